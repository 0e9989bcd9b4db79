// attn_prefill.h -- launchers of the MLA prefill attention kernel and of the
// mask-tile classifier.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mla {

// Class of one 128x128 (query, key) tile of an explicit additive mask.
enum : uint8_t {
  kTileSkip = 0,   // every entry -inf: the tile contributes nothing
  kTileZero = 1,   // every entry +-0: scores need no mask add
  kTileMixed = 2,  // anything else: the kernel adds the mask entries
  kTileCausal = 3, // a diagonal tile holding the causal pattern: +-0 where key <= query,
                   // -inf above (no mask loads; the causal kernel's per-row limit)
  kTilePrefix = 4, // kTilePrefix + lim (lim in 0..126): every row is +-0 for the
                   // tile's keys 0..lim and -inf after (no mask loads)
};

// Bytes of the tile-class array for a [B,1,T,T] mask (B x ceil(T/128)^2).
size_t attn_class_bytes(int B, int T);

// Classify every 128x128 tile of `mask` ([B,1,T,mask_ld] bf16) into `cls`.
cudaError_t launch_mask_classify(const void* mask, int64_t mask_ld, int B, int T, void* cls,
                                 cudaStream_t stream);

// Prefill attention for all 64 heads; writes out[b, t, h*128 + e] (bf16).
// mask == null: causal. tile_class may be null when mask is given (every key
// tile is then visited and masked element-wise). valid_len (device, [B] int32,
// only without mask): causal with keys j >= valid_len[b] masked (values are
// clamped to [0, T]); null means every sequence has all T keys. rope_cs
// (device, [B*T][32] float2 of (f cos, f sin), from launch_rope_prepass):
// q_pe arrives unrotated and each query tile's rotary part is rotated in
// shared memory (k_pe must then be the rotated key); null: q_pe is rotated.
cudaError_t launch_attn_prefill(const void* q_nope, const void* q_pe, const void* k_nope,
                                const void* k_pe, const void* v, const void* mask,
                                int64_t mask_ld, const void* tile_class, int B, int T,
                                float softmax_scale, void* out,
                                unsigned long long wait_limit_ns, unsigned int* err_word,
                                int test_stall, cudaStream_t stream,
                                const int* valid_len = nullptr, const void* rope_cs = nullptr);

}  // namespace mla
