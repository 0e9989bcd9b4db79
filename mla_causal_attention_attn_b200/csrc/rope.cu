// rope.cu -- YaRN rotary embedding of the rotary parts, for callers that pass
// q_pe and k_pe unrotated (page "Kimi K2 · Mix and project", excerpt
// modeling_deepseek.py 799-840: cos, sin = self.rotary_emb(...);
// apply_rotary_pos_emb(q_pe, k_pe, cos, sin, position_ids); parameters from
// config.json on page "Kimi K2 · Block input": rope_theta 50000 and
// rope_scaling {yarn, factor 32, original_max_position_embeddings 4096,
// beta_fast 1, beta_slow 1, mscale 1, mscale_all_dim 1}).
//
// Pair i of a rotary vector (elements 2i, 2i+1) turns by position *
// inv_freq[i], scaled by the attention factor f:
//   y0 = f (x0 cos a - x1 sin a),  y1 = f (x1 cos a + x0 sin a).
// YaRN (NTK-by-parts): inv_freq[i] = theta^(-2i/64) * ((1 - r_i) + r_i / factor)
// with r_i a ramp from 0 to 1 between the pair indices that complete
// beta_fast and beta_slow turns over the original context length.
//
// The shared rotary key is rotated once per call here (it serves all 64
// heads; rotating it inside every attention CTA would repeat the same work
// 64 x (query tile pairs) times), and the same pass writes (f cos, f sin) for
// every (b, t) and pair, which the attention kernel uses to rotate each query
// tile's q_pe in shared memory right after its TMA load.
#include "rope.h"

#include <cmath>

#include <cuda_bf16.h>

namespace mla {

namespace {

__global__ void __launch_bounds__(256)
    rope_prepass_kernel(const __nv_bfloat162* __restrict__ k_pe, const int* __restrict__ pos,
                        int64_t n_rows, int T, RopeFreqs f, float2* __restrict__ cs,
                        __nv_bfloat162* __restrict__ k_rot) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // (row, pair)
  if (idx >= n_rows * kRopePairs) return;
  const int64_t row = idx / kRopePairs;  // b * T + t
  const int i = int(idx % kRopePairs);
  const double p = pos ? double(pos[row]) : double(row % T);
  double s, c;
  sincos(p * f.inv_freq[i], &s, &c);
  c *= f.attn_factor;
  s *= f.attn_factor;
  cs[idx] = make_float2(float(c), float(s));
  const __nv_bfloat162 x = k_pe[idx];
  const double x0 = __bfloat162float(x.x), x1 = __bfloat162float(x.y);
  __nv_bfloat162 y;
  y.x = __double2bfloat16(x0 * c - x1 * s);
  y.y = __double2bfloat16(x1 * c + x0 * s);
  k_rot[idx] = y;
}

}  // namespace

bool yarn_frequencies(double theta, double factor, double orig_max_pos, double beta_fast,
                      double beta_slow, double mscale, double mscale_all_dim, RopeFreqs* out) {
  const double v[7] = {theta, factor, orig_max_pos, beta_fast, beta_slow, mscale, mscale_all_dim};
  for (double x : v)
    if (!std::isfinite(x)) return false;
  if (!(theta > 1.0) || !(factor > 0.0) || !(orig_max_pos > 0.0) || !(beta_fast > 0.0) ||
      !(beta_slow > 0.0))
    return false;
  constexpr int kDim = 2 * kRopePairs;
  const double kTwoPi = 6.283185307179586476925286766559;
  // pair index that completes n turns over orig_max_pos positions
  auto turns_index = [&](double n) {
    return kDim * std::log(orig_max_pos / (kTwoPi * n)) / (2.0 * std::log(theta));
  };
  double lo = std::floor(turns_index(beta_fast));
  double hi = std::ceil(turns_index(beta_slow));
  lo = std::max(lo, 0.0);
  hi = std::min(hi, double(kDim - 1));
  if (hi == lo) hi += 0.001;
  for (int i = 0; i < kRopePairs; ++i) {
    const double base = std::pow(theta, -2.0 * i / kDim);
    const double r = std::min(std::max((i - lo) / (hi - lo), 0.0), 1.0);
    out->inv_freq[i] = base * (1.0 - r) + base / factor * r;
  }
  auto m = [&](double k) { return factor <= 1.0 ? 1.0 : 0.1 * k * std::log(factor) + 1.0; };
  out->attn_factor = m(mscale) / m(mscale_all_dim);
  return std::isfinite(out->attn_factor);
}

cudaError_t launch_rope_prepass(const void* k_pe, const int* position_ids, int B, int T,
                                const RopeFreqs& f, void* cs, void* k_rot, cudaStream_t stream) {
  const int64_t n_rows = int64_t(B) * T;
  const int64_t threads = n_rows * kRopePairs;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  rope_prepass_kernel<<<unsigned(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat162*>(k_pe), position_ids, n_rows, T, f,
      static_cast<float2*>(cs), static_cast<__nv_bfloat162*>(k_rot));
  return cudaGetLastError();
}

size_t rope_cs_bytes(int B, int T) { return size_t(B) * size_t(T) * kRopePairs * sizeof(float2); }

size_t rope_krot_bytes(int B, int T) { return size_t(B) * size_t(T) * 2 * kRopePairs * 2; }

}  // namespace mla
