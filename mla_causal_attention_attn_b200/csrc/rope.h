// rope.h -- YaRN rotary embedding: frequencies (host) and the per-call
// pre-pass that rotates the shared rotary key and tabulates cos / sin.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace mla {

constexpr int kRopePairs = 32;  // qk_rope_head_dim / 2

// Rotation frequencies of the 32 pairs (radians per position) and the factor
// applied to cos and sin; passed to the kernel by value.
struct RopeFreqs {
  double inv_freq[kRopePairs];
  double attn_factor;
};

// YaRN frequencies and attention factor from config.json's rope_theta and
// rope_scaling fields. False if a parameter is not finite or out of range
// (theta <= 1, factor, original_max_position_embeddings or a beta <= 0).
bool yarn_frequencies(double theta, double factor, double orig_max_pos, double beta_fast,
                      double beta_slow, double mscale, double mscale_all_dim, RopeFreqs* out);

// Bytes of the cos / sin table ([B*T][32] float2) and of the rotated key
// ([B, 1, T, 64] bf16).
size_t rope_cs_bytes(int B, int T);
size_t rope_krot_bytes(int B, int T);

// For every (b, t): cs[b*T + t][i] = (f cos a, f sin a) with a = position *
// inv_freq[i], and k_rot[b, 0, t, :] = k_pe[b, 0, t, :] rotated. position_ids
// [B, T] int32, or null for t. Angles, cos and sin in double; k_rot rounded
// once to bf16.
cudaError_t launch_rope_prepass(const void* k_pe, const int* position_ids, int B, int T,
                                const RopeFreqs& f, void* cs, void* k_rot, cudaStream_t stream);

}  // namespace mla
