"""The refinement path's fp64 exp2 (csrc/fp64.cuh) against CUDA's exp2(double).

A probe kernel including the header is compiled with nvcc at test time and run
on 2^22 arguments spread over the whole range the refinement uses (x in
[-1075, 0], denser near 0) plus special points; the result must lie within a
few ulp of exp2() (relative error < 1e-15 for normal results, exact 0 below
the double range, NaN kept).
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from speculative_decoding_verification_86_b200 import build

pytestmark = pytest.mark.gpu

PROBE = r'''
#include "fp64.cuh"
__global__ void probe(const double* x, double* got, double* ref, int n) {
  __shared__ double tab[sv::kExp2Table];
  sv::exp2_table_init(tab);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    got[i] = sv::exp2_fast(x[i], tab);
    ref[i] = exp2(x[i]);
  }
}
extern "C" int run_probe(const double* x, double* got, double* ref, int n) {
  probe<<<296, 256>>>(x, got, ref, n);
  return (int)cudaDeviceSynchronize();
}
'''


@pytest.fixture(scope="module")
def probe_lib(tmp_path_factory):
    d = tmp_path_factory.mktemp("exp2probe")
    src = d / "probe.cu"
    src.write_text(PROBE)
    out = d / "probe.so"
    subprocess.check_call([build._nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-Xcompiler", "-fPIC", "-shared", "-I", build.CSRC, str(src), "-o", str(out)])
    lib = ctypes.CDLL(str(out))
    lib.run_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    return lib


def test_exp2_fast_matches_cuda_exp2(probe_lib, cuda_device):
    rng = np.random.default_rng(0)
    n = 1 << 22
    x = np.concatenate([
        -rng.random(n // 2) * 60.0,                  # where weights live
        -rng.random(n // 2 - 64) * 1075.0,           # the whole range
        [0.0, -0.0, -1e-300, -1.0, -0.5, -1 / 64, -1 / 32, -1021.0, -1022.0, -1022.5, -1060.0,
         -1069.99, -1070.0, -1074.0, -1075.0, -2000.0, -np.inf, np.nan, 1e-17, 2e-16],
    ])
    x = np.concatenate([x, -np.arange(0, 44) / 32.0])
    xd = torch.from_numpy(x).to(cuda_device)
    got = torch.empty_like(xd)
    ref = torch.empty_like(xd)
    assert probe_lib.run_probe(xd.data_ptr(), got.data_ptr(), ref.data_ptr(), xd.numel()) == 0
    g, r = got.cpu().numpy(), ref.cpu().numpy()
    nan = np.isnan(x)
    assert np.all(np.isnan(g[nan]))
    g, r, xs = g[~nan], r[~nan], x[~nan]
    below = xs < -1070.0
    assert np.all(g[below] == 0.0)
    normal = (~below) & (r >= 2.0 ** -1022)
    rel = np.abs(g[normal] - r[normal]) / r[normal]
    assert rel.max() < 1e-15, rel.max()
    sub = (~below) & (r < 2.0 ** -1022)
    assert np.all(np.abs(g[sub] - r[sub]) <= 2.0 ** -1074 * 8)
