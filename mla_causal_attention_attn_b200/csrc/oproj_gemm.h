// oproj_gemm.h -- launcher of the tcgen05 output-projection GEMM.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mla {

// C[M, N] = A[M, K] . W[N, K]^T, all bf16 row-major, fp32 accumulation.
// Requires N % 256 == 0, K % 64 == 0, 16-byte aligned pointers. `force_bn`
// (0, 64, 128 or 256) overrides the tile-width choice.
cudaError_t launch_oproj_gemm(const void* A, const void* W, void* C, int64_t M, int N, int K,
                              int num_sms, unsigned long long wait_limit_ns, int force_bn,
                              unsigned int* err_word, cudaStream_t stream);

// Tile width the launcher picks for an M x N problem on `num_sms` SMs.
int oproj_pick_bn(int64_t M, int N, int num_sms);

}  // namespace mla
