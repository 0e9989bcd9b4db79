// fp8_oproj.h -- launchers of the e4m3 quantisers and the block-scaled FP8
// output-projection GEMM (fp8_oproj.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mla {

// x [M, K] bf16 (row stride ld elements, ld >= K, ld % 8 == 0, 16-byte
// aligned) -> q [M, K] e4m3 codes and scale [K/128][M] fp32. K % 128 == 0.
cudaError_t launch_quant_rows_fp8(const void* x, int64_t ld, int64_t M, int K, void* q,
                                  float* scale, cudaStream_t stream);

// W [N, K] bf16 (16-byte aligned) -> q [N, K] codes and scale [N/128][K/128].
// N % 128 == 0, K % 128 == 0.
cudaError_t launch_quant_weight_fp8(const void* W, int N, int K, void* q, float* scale,
                                    cudaStream_t stream);

// C[M, N] bf16 = block-scaled product of qa [M, K] (a_scale [K/128][M]) and
// qw [N, K] (w_scale [N/128][K/128]). N % 128 == 0, K % 512 == 0; code
// pointers and C 16-byte aligned. Output tiles are 128 x oproj_fp8_pick_bn().
cudaError_t launch_oproj_fp8(const void* qa, const float* a_scale, const void* qw,
                             const float* w_scale, void* C, int64_t M, int N, int K, int num_sms,
                             unsigned long long wait_limit_ns, unsigned int* err_word,
                             cudaStream_t stream);

// Tile width (128 or 256 columns) the FP8 GEMM uses for an M x N problem.
int oproj_fp8_pick_bn(int64_t M, int N, int num_sms);
}  // namespace mla
