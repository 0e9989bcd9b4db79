"""The FMA-pipe exp2 (exp2_poly2 in csrc/sm100.cuh) against CUDA's exp2f and
an fp64 reference, over every fp32 step of [-125, 10] at a coarse stride and
densely around integers (where the range reduction switches n).

The kernel uses it for one exponential in four on non-diagonal causal tiles;
its relative error must stay far below bf16's 2^-9 (P is rounded to bf16).
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mla_causal_attention_attn_b200", "csrc")

pytestmark = pytest.mark.gpu

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "sm100.cuh"
__global__ void run(const float* x, float* poly, float* ref, int n) {
  int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    float e0, e1;
    mla::exp2_poly2(x[i], x[i + 1], e0, e1);
    poly[i] = e0; poly[i + 1] = e1;
    ref[i] = exp2f(x[i]); ref[i + 1] = exp2f(x[i + 1]);
  }
}
int main() {
  const int n = 1 << 22;
  std::vector<float> hx(n);
  FILE* f = fopen("x.bin", "rb"); fread(hx.data(), 4, n, f); fclose(f);
  float *x, *p, *r;
  cudaMalloc(&x, 4 * n); cudaMalloc(&p, 4 * n); cudaMalloc(&r, 4 * n);
  cudaMemcpy(x, hx.data(), 4 * n, cudaMemcpyHostToDevice);
  run<<<n / 512, 256>>>(x, p, r, n);
  if (cudaDeviceSynchronize() != cudaSuccess) return 2;
  std::vector<float> hp(n), hr(n);
  cudaMemcpy(hp.data(), p, 4 * n, cudaMemcpyDeviceToHost);
  cudaMemcpy(hr.data(), r, 4 * n, cudaMemcpyDeviceToHost);
  f = fopen("poly.bin", "wb"); fwrite(hp.data(), 4, n, f); fclose(f);
  f = fopen("ref.bin", "wb"); fwrite(hr.data(), 4, n, f); fclose(f);
  return 0;
}
"""


def test_exp2_poly_error_bound():
    n = 1 << 22
    g = np.random.default_rng(0)
    coarse = np.linspace(-125.0, 10.0, n // 2, dtype=np.float64)
    ints = np.repeat(np.arange(-125, 11), (n // 2) // 136 + 1)[: n // 2].astype(np.float64)
    near = ints + g.uniform(-1e-3, 1e-3, size=n // 2)
    x = np.concatenate([coarse, near]).astype(np.float32)
    x = np.clip(x, -125.0, 10.0)
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "t.cu")
        open(src, "w").write(PROGRAM)
        exe = os.path.join(d, "t")
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-std=c++17", "-I", CSRC, src, "-o", exe], check=True)
        x.tofile(os.path.join(d, "x.bin"))
        subprocess.run([exe], check=True, cwd=d)
        poly = np.fromfile(os.path.join(d, "poly.bin"), dtype=np.float32).astype(np.float64)
        ref = np.fromfile(os.path.join(d, "ref.bin"), dtype=np.float32).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel_exact = np.abs(poly - exact) / exact
    rel_cuda = np.abs(poly - ref) / ref
    assert np.all(np.isfinite(poly))
    assert rel_exact.max() < 1.2e-4, rel_exact.max()
    assert rel_cuda.max() < 1.3e-4, rel_cuda.max()
    # far below the bf16 rounding P goes through afterwards
    assert rel_exact.max() < 2.0 ** -9 / 10
