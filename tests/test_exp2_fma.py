"""The FMA-pipe exp2 of the attention softmax against CUDA's exp2f on the GPU.

The device function is compiled from the library's own header into a small
test program; its relative error over the softmax's input range must stay
within the 7.5e-5 bound of its Remez fit (plus fp32 rounding)."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "dynamic_block_sparse_rr_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#include <cmath>
#include "sm100.cuh"
__global__ void k(const float* x, float* a, float* b, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) { a[i] = rr::ex2_fma(x[i]); b[i] = exp2f(x[i]); }
}
int main() {
  const int n = 1 << 22;
  float *x, *a, *b;
  cudaMallocManaged(&x, n * 4); cudaMallocManaged(&a, n * 4); cudaMallocManaged(&b, n * 4);
  for (int i = 0; i < n; ++i) x[i] = -120.0f + 128.0f * (float)i / (float)(n - 1);
  k<<<(n + 255) / 256, 256>>>(x, a, b, n);
  if (cudaDeviceSynchronize() != cudaSuccess) return 2;
  double worst = 0; int at = 0;
  for (int i = 0; i < n; ++i) {
    double e = fabs((double)a[i] / (double)b[i] - 1.0);
    if (e > worst) { worst = e; at = i; }
  }
  printf("%.9e %.9e\n", worst, x[at]);
  return 0;
}
'''


def test_ex2_fma_matches_exp2f():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "t.cu")
        exe = os.path.join(d, "t")
        open(src, "w").write(PROGRAM)
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                               "-I", CSRC, "-I", os.path.join(ROOT, "include"), "-o", exe, src])
        out = subprocess.check_output([exe], text=True).split()
    worst, at = float(out[0]), float(out[1])
    assert worst < 8e-5, (worst, at)
