// oproj_gemm.h -- launcher of the tcgen05 output-projection GEMM.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mla {

// C[M, N] = A[M, K] . W[N, K]^T, all bf16 row-major, fp32 accumulation.
// Requires N % 128 == 0, K % 64 == 0, 16-byte aligned pointers. M <= 128 (with
// K % 128 == 0) runs the small-M kernel, which reads W once with two CTAs per
// 128 rows of W (K halves) and swaps the MMA operands; otherwise the output
// tile (128 x 128, 224 or 256, or 256 x 224) is chosen for wave efficiency
// unless `force_bn` (non-zero) fixes a 128-row tile of that width.
// test_stall (failure-detection tests only): in the first cluster of the
// small-M kernel the rank-1 CTA never reports its partial sum.
cudaError_t launch_oproj_gemm(const void* A, const void* W, void* C, int64_t M, int N, int K,
                              int num_sms, unsigned long long wait_limit_ns, int force_bn,
                              unsigned int* err_word, cudaStream_t stream, int test_stall = 0);

// Up-projection of the compressed KV latent: kv = c_kv [B*T, R] . W [64*256, R]^T,
// stored per head as k_nope [B, 64, T, 128] (columns h*256 .. +127) and
// v [B, 64, T, 128] (columns h*256+128 .. +255), bf16, fp32 accumulation. The
// tiled GEMM with 128 x 256 tiles (one head per column tile); R % 64 == 0.
cudaError_t launch_kv_up(const void* c_kv, const void* W, void* k_nope, void* v, int B, int T,
                         int R, int num_sms, unsigned long long wait_limit_ns,
                         unsigned int* err_word, cudaStream_t stream);

// Output tile the launcher picks for an M x N problem (M > 128) on `num_sms`
// SMs: mt row blocks of 128 by bn columns.
struct OprojTile {
  int bn, mt;
};
OprojTile oproj_pick_tile(int64_t M, int N, int num_sms);

}  // namespace mla
