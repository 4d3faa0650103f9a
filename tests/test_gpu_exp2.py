"""The FMA-pipe exp2 forms of csrc/exp2_poly.cuh (degree 3 for the attention
softmax, degree 5 for the heat map's row sums) against fp64 exp2 and CUDA's
exp2f, on inputs covering the range the kernels feed them ([-125, 8])."""
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "dynamic_block_sparse_fractal_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <vector>
#include <cuda_runtime.h>
#include "exp2_poly.cuh"
__global__ void k(const float* x, float* poly, float* poly5, float* ref, int n) {
  int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 >= n) return;
  uint64_t e = sa::exp2_poly_x2(sa::f2_pack(x[i], x[i + 1]));
  float a, b;
  sa::f2_unpack(e, a, b);
  poly[i] = a; poly[i + 1] = b;
  e = sa::exp2_poly5_x2(sa::f2_pack(x[i], x[i + 1]));
  sa::f2_unpack(e, a, b);
  poly5[i] = a; poly5[i + 1] = b;
  ref[i] = exp2f(x[i]); ref[i + 1] = exp2f(x[i + 1]);
}
int main(int argc, char** argv) {
  const int n = 1 << 22;
  std::vector<float> hx(n);
  for (int i = 0; i < n; ++i) hx[i] = -125.0f + 133.0f * float(i) / float(n - 1);
  float *x, *p, *p5, *r;
  cudaMalloc(&x, n * 4); cudaMalloc(&p, n * 4); cudaMalloc(&p5, n * 4); cudaMalloc(&r, n * 4);
  cudaMemcpy(x, hx.data(), n * 4, cudaMemcpyHostToDevice);
  k<<<n / 512, 256>>>(x, p, p5, r, n);
  if (cudaDeviceSynchronize() != cudaSuccess) return 1;
  std::vector<float> hp(n), hp5(n), hr(n);
  cudaMemcpy(hp.data(), p, n * 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(hp5.data(), p5, n * 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(hr.data(), r, n * 4, cudaMemcpyDeviceToHost);
  FILE* f = fopen(argv[1], "wb");
  fwrite(hx.data(), 4, n, f); fwrite(hp.data(), 4, n, f); fwrite(hp5.data(), 4, n, f);
  fwrite(hr.data(), 4, n, f);
  fclose(f);
  return 0;
}
"""


def test_poly_exp2_relative_error():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "h.cu")
        exe = os.path.join(d, "h")
        out = os.path.join(d, "out.bin")
        open(src, "w").write(HARNESS)
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-std=c++17", "-I", CSRC, "-o", exe, src], check=True)
        subprocess.run([exe, out], check=True)
        raw = np.fromfile(out, dtype=np.float32)
    n = raw.size // 4
    x, poly, poly5, ref = (raw[:n].astype(np.float64), raw[n:2 * n], raw[2 * n:3 * n],
                           raw[3 * n:])
    exact = np.exp2(x)
    rel = np.abs(poly / exact - 1.0)
    # polynomial bound 7.5e-5 plus fp32 evaluation rounding
    assert rel.max() < 1.0e-4, rel.max()
    # and it agrees with CUDA's exp2f to the same order
    assert np.abs(poly / ref.astype(np.float64) - 1.0).max() < 1.0e-4
    # degree 5: 1.5e-7 polynomial bound plus the rounding of five fp32 FMAs
    rel5 = np.abs(poly5 / exact - 1.0)
    assert rel5.max() < 6.0e-7, rel5.max()
