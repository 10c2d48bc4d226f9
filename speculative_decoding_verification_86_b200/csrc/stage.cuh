// Per-thread staging of streamed logits in shared memory with asynchronous
// copies (cp.async, 16 bytes each, sm_80+).
//
// A streaming pass reads its row segment in steps of kStepVecs 16-byte vectors
// per thread.  Instead of holding the next step's loads in registers, each
// thread keeps kStageSlots steps in flight as asynchronous copies into its own
// slots of a shared buffer -- three times the bytes in flight of register
// double buffering, at no register cost -- and reads a step back once its
// copy group has landed.  Thread t's vector u of slot s lives at
// buf[(s * kStepVecs + u) * kThreads + t]: consecutive threads touch
// consecutive 16-byte words (no bank conflicts), and no thread ever touches
// another thread's words, so no barrier is needed.  Vectors past the row end
// are not copied (zero-fill) and are replaced by masked logits when read.
#pragma once
#include "common.cuh"

namespace sv {

constexpr int kStageSlots = 3;
constexpr int kStepVecs = 4;
constexpr size_t kStageBytes = static_cast<size_t>(kStageSlots) * kStepVecs * kThreads * 16;  // 48 KB

__device__ __forceinline__ void cp_async16(uint4* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most n copy groups of this thread are still in flight (n <= 2).
__device__ __forceinline__ void cp_async_wait(int n) {
  if (n <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
  else if (n == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else asm volatile("cp.async.wait_group 2;" ::: "memory");
}

// A stream of `steps` steps; step s copies, for u < kStepVecs, the vector
// addr(s, u) (a global vector index, valid when < limit(s, u)) of row rows(s, u).
struct Stager {
  uint4* buf;
  int issued = 0;

  __device__ __forceinline__ uint4* slot(int s, int u) const {
    return buf + (static_cast<size_t>(s % kStageSlots) * kStepVecs + u) * kThreads + threadIdx.x;
  }
};

}  // namespace sv
