// attn_prefill.cu -- causal / additively-masked MLA prefill attention for the
// Kimi K2 head layout (page "Kimi K2 · Mix and project", code excerpt
// modeling_deepseek.py 799-840, and the head merge of excerpt 848-852):
//
//   per batch b, head h (64 heads), query row i:
//     s_ij = softmax_scale * (q_nope_i . k_nope_j + q_pe_i . k_pe_j) + M_ij
//     p_ij = softmax_j(s_ij)            (fp32; P fed to the MMA as bf16)
//     out[b, i, h*128 + e] = sum_j p_ij v_je
//   with k_pe one [B,1,T,64] tensor shared by all heads and M either the
//   implicit causal mask (mask == NULL) or an explicit additive [B,1,T,T] mask.
//   The causal kernel also takes the compact form of causal + key padding
//   (page "Kimi K2 · Transformer blocks", excerpt modeling_deepseek.py
//   1443-1457: the 2-D padding mask of the flash path): key j is allowed for
//   query i iff j <= i and j < valid_len[b].
//
// One CTA computes two 128-row query tiles (2p, 2p+1) of one (b, h), so that
// every K/V tile brought into shared memory serves 256 query rows and the
// softmax of one query tile overlaps the tensor-core work of the other.
// Roles (384 threads = three warpgroups):
//   warp 0       TMA producer: query tile 0 (nope + rope, 48 KB) and the first
//                key tile's K blocks (issued by thread 0 right after it sets up
//                the barriers), query tile 1, then for every visited 128-key
//                tile five 16 KB blocks (k_nope lo/hi, the shared k_pe,
//                v lo/hi) into an 8-block ring;
//   warp 1       tensor-memory owner; warps 1 and 2: one MMA-issuing thread
//                per query tile i, per key tile j in order
//                  Oi += Pi_{j-1} V_{j-1},  Si = Qi K_j^T
//                (S: 128x128, K = 128 nope + 64 rope, both operands in shared
//                memory; PV: 128x128, K = 128 keys, P read from tensor memory),
//                with the S MMAs of the two tiles kept in the order
//                S0_j, S1_j, S0_{j+1}, ... Because PV_{j-1} of a tile is issued
//                before its S_j, the commit that announces S_j also guarantees
//                O holds PV_{j-1};
//   warp 3       idle, or (half-tile scores, long sequences) the PV issuer
//                described below;
//   warps 4..7   softmax of query tile 0, one thread per row (TMEM lane);
//   warps 8..11  softmax of query tile 1. Each reads S, scales, masks, keeps a
//                running max (rescaling O only when the max grows by more than
//                2^8), exponentiates, sums, writes P as bf16 over the first 64
//                columns of its S buffer, and at the end O / l -> bf16, staged in
//                its query tile's freed Q buffer and written by TMA stores.
//                Tiles that need no mask entries added (every causal tile, the
//                all-zero tiles of an explicit mask) take a single pass
//                against the running max; the others two passes.
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).
//
// Half-tile scores (the default): with 128-key tiles a
// query tile's chain S_j -> softmax_j -> PV_j -> S_{j+1} is serial, and the
// tensor pipe idles whenever both softmax warpgroups are busy. There each
// 128-column S buffer is split into two 64-key buffers, and an issuer runs
// S(0), S(1), then PV(u), S(u+2) for every 64-key half tile u, so the scores
// of the next half tile are computed while the softmax works on this one;
// the softmax waits for PV(u-1) only before it rescales O. The O accumulators
// and the K/V ring are unchanged. The issue order needs each query tile's
// active key tiles to be a prefix of the visited ones: always true for
// causal and valid-length calls. Under an explicit mask the CTA checks its
// tile classes and keeps 128-key tiles when a query tile skips a key tile
// that a later one of its key tiles follows (the half-tile issuers would
// have to release the skipped tile's ring blocks in between); a mask
// tile's class maps onto its two halves (zero; causal, limit r - 64 half;
// prefix L, limit L - 64 half; mixed, its 64 entries).
//
// Separate PV issuer (half tiles, T >= kPvIssuerMinT unless MLA_ATTN_PV_ISSUER
// says otherwise): an issuer that waits for a K block of S(u+2) cannot issue
// PV(u+1), however early P(u+1) is written. Then warps 1 and 2 issue only the
// S products, and one thread of warp 3 issues the PV products of both query
// tiles, polling P and V readiness of each tile in turn. S(u+2) overwrites
// the buffer PV(u) reads, so the S issuer waits until PV(u) has been issued
// (pv_issued); the tensor pipe keeps that order across the two threads
// through the tcgen05 fences around the barrier.
#include "attn_prefill.h"

#include <cstdlib>
#include <cstring>

#include "host_util.h"
#include "sm100.cuh"

namespace mla {

namespace {

constexpr int kBQ = 128;     // query rows per tile
constexpr int kBKV = 128;    // keys per tile
constexpr int kDN = 128;     // qk_nope_head_dim
constexpr int kDR = 64;      // qk_rope_head_dim
constexpr int kDV = 128;     // v_head_dim
constexpr int kH = 64;       // heads
// Heads whose CTAs are scheduled together (L2 reuse of K/V): 8 (a group's
// K/V of 8 x 2 MB at T = 4096 stays in L2), more for short sequences, where
// a group's K/V is small and a longer longest-first run packs the SMs
// better.
constexpr int kHeadGroup = 8;
__host__ __device__ constexpr int head_group_for(int T) { return T <= 2048 ? 16 : kHeadGroup; }
constexpr int kRing = 8;     // 16 KB blocks in the K/V ring
// Sequences at least this long issue their half-tile PV products from a
// thread of their own. Shorter ones keep one issuer per query tile: there
// the last query tile runs alone for a larger share of a CTA, and the extra
// hand-off between S and PV issuers sits on its serial chain (B=16 T=1024:
// 0.549 against 0.516 ms; B=1 T=4096: 0.342 against 0.345 ms; B=1 T=32768:
// 20.1-20.2 against 20.8-21.0 ms).
constexpr int kPvIssuerMinT = 4096;
constexpr int kBlocksPerTile = 5;
constexpr int kThreads = 384;
// ptxas budgets 168 registers a thread for 384 threads; setmaxnreg moves
// them: 128 x 88 (warpgroup 0) + 256 x 208 (softmax) = 384 x 168.
constexpr uint32_t kRegsControl = 88;
constexpr uint32_t kRegsSoftmax = 208;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= 384 * 168, "register split");
constexpr int kBarTeardown = 1;  // named barrier for the final hand-off
constexpr int kBarStage0 = 2;    // + query tile: its output rows are staged
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t kBlock = kBQ * 64 * 2;  // one 128 x 64 bf16 swizzled block: 16 KB
constexpr uint32_t kQBytes = 3 * kBlock;   // nope lo, nope hi, rope
constexpr uint32_t kOffQ = 0;              // Q0, then Q1
constexpr uint32_t kOffRing = 2 * kQBytes;
constexpr uint32_t kSmemUsed = kOffRing + kRing * kBlock;
constexpr size_t kSmemBytes = kSmemUsed + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;  // S_i at kColS + 128 i, O_i at kColO + 128 i

static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

struct AttnArgs {
  const __nv_bfloat16* mask;   // [B,1,T,mask_ld] or null (causal)
  const int* valid_len;        // [B] keys per sequence (causal kernel), or null (all T)
  int64_t mask_ld;
  int mask_vec;                // rows 16-byte aligned: vector loads
  const uint8_t* tile_class;   // [B, n_qt, n_kv] or null
  __nv_bfloat16* out;          // [B, T, 64*128]
  int B, T, n_qt, n_kv, n_pairs;
  float scale_log2;            // softmax_scale * log2(e)
  unsigned long long wait_limit_ns;
  unsigned int* err_word;      // device status word
  int test_stall;              // failure-detection test: one wait that never completes
  const float2* rope_cs;       // [B*T][32] (f cos, f sin) of each query's rotary pairs, or
                               // null when q_pe arrives rotated
};

// Which key tiles the two query tiles of a CTA visit. Causal: tile qt visits
// 0..qt, and none at or past the sequence's key count (kv_end tiles). Explicit
// mask: every key tile whose class is not "all -inf" (every tile when no
// classification is given).
template <bool kMasked>
struct PairTiles {
  int qt[2];
  bool exists[2];
  const uint8_t* cls[2];
  int kv_end;  // causal: key tiles holding at least one of the sequence's keys
  int end;     // one past the last candidate key tile

  __device__ __forceinline__ bool active(int i, int kt) const {
    if (!exists[i]) return false;
    if (kMasked) return cls[i] ? cls[i][kt] != kTileSkip : true;
    return kt <= qt[i] && kt < kv_end;
  }
  __device__ __forceinline__ int next(int kt) const {
    ++kt;
    while (kt < end && !active(0, kt) && !active(1, kt)) ++kt;
    return kt;
  }
  __device__ __forceinline__ int first() const { return next(-1); }
};

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// One row's view of a 128x128 score tile: turns 32 consecutive raw scores
// (chunk c, already read from tensor memory) into
// s * scale_log2 + mask * log2(e) - shift, with keys that are excluded
// (causal, past T, invalid row) at -inf.
template <bool kMasked>
struct ScoreChunk {
  uint8_t cls;                // class of this (query, key) tile
  bool row_valid;
  const __nv_bfloat16* mrow;  // mask row at the tile's first key (kMasked)
  int kvalid;                 // keys of the tile below T
  int mask_vec;               // 16-byte mask loads allowed
  int diag_row;               // keys c > diag_row are excluded (the causal kernel's
                              // diagonal; a causal-pattern or prefix tile of a mask)

  __device__ __forceinline__ void apply(const uint32_t* rr, int c, float scale_log2, float shift,
                                        float (&x)[32]) const {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = fmaf(__uint_as_float(rr[i]), scale_log2, -shift);
    if (!kMasked) {
      if (diag_row < kBKV) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c * 32 + i > diag_row) x[i] = -INFINITY;
      }
      return;
    }
    if (!row_valid) {
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = -INFINITY;
      return;
    }
    if (diag_row < kBKV) {
      // causal-pattern and prefix tiles: their mask entries are +-0 up to the
      // limit and -inf after it (only a non-positive scale brings them here)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c * 32 + i > diag_row) x[i] = -INFINITY;
    }
    if (cls == kTileMixed) {
      // 8 keys per 16-byte load when rows are 16-byte aligned; a chunk that
      // starts below T then lies inside the row (mask_ld >= T, mask_ld % 8 ==
      // 0). Chunks past the last key re-read the last existing one; their keys
      // are set to -inf below.
      const int klast = min(kvalid, kBKV) - 1;
      const int c8_last = klast >> 3;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c8 = 4 * c + j;
        uint32_t ws[4];
        if (mask_vec) {
          const uint4 w = ld_nc_v4_ordered(reinterpret_cast<const uint4*>(mrow) + min(c8, c8_last));
          ws[0] = w.x, ws[1] = w.y, ws[2] = w.z, ws[3] = w.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            ws[e] = ld_nc_u16_ordered(mrow + min(c8 * 8 + 2 * e, klast)) |
                    (ld_nc_u16_ordered(mrow + min(c8 * 8 + 2 * e + 1, klast)) << 16);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[8 * j + 2 * e] = fmaf(bf16_bits_to_float(ws[e] & 0xffffu), kLog2e, x[8 * j + 2 * e]);
          x[8 * j + 2 * e + 1] = fmaf(bf16_bits_to_float(ws[e] >> 16), kLog2e, x[8 * j + 2 * e + 1]);
        }
      }
    }
    if (kvalid < (c + 1) * 32) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c * 32 + i >= kvalid) x[i] = -INFINITY;
    }
  }
};

// Maximum of a row of W (128 or 64) raw scores; on the diagonal tile keys
// c > r are excluded (causal).
template <bool kDiag, int W = kBKV>
__device__ __forceinline__ float raw_row_max(const uint32_t (&raw)[W], int r) {
  float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int i = 0; i < W; i += 8) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      v[e] = __uint_as_float(raw[i + e]);
      if (kDiag && i + e > r) v[e] = -INFINITY;
    }
    m4[0] = fmax3(m4[0], v[0], v[1]);
    m4[1] = fmax3(m4[1], v[2], v[3]);
    m4[2] = fmax3(m4[2], v[4], v[5]);
    m4[3] = fmax3(m4[3], v[6], v[7]);
  }
  return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
}

// Causal tile, 32 raw scores of chunk c: p = 2^(s*scale_log2 - m) (MUFU
// ex2, which maps -inf to exactly 0), packed as bf16 pairs into pk and summed
// (unrounded, fp32) into the paired partial sums acc. On the diagonal tile
// keys c > r give 0. With kTrackMax, xmax[0..1] also collect the largest
// s*scale_log2 - m seen (the caller's running-max check).
template <bool kDiag, bool kTrackMax = false>
__device__ __forceinline__ void p_chunk_causal(const uint32_t* raw, int c, int r, float scale_log2,
                                               float m, uint32_t (&pk)[16], float (&acc)[8],
                                               float* xmax = nullptr) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1;
    ffma2(x0, x1, __uint_as_float(raw[2 * i]), __uint_as_float(raw[2 * i + 1]), scale_log2,
          scale_log2, -m, -m);
    float p0, p1;
    if (kDiag) {
      if (c * 32 + 2 * i > r) x0 = -INFINITY;
      if (c * 32 + 2 * i + 1 > r) x1 = -INFINITY;
    }
    if (kTrackMax) xmax[i & 1] = fmax3(xmax[i & 1], x0, x1);
    p0 = fast_exp2(x0);
    p1 = fast_exp2(x1);
    const int a = 2 * (i & 3);
    fadd2(acc[a], acc[a + 1], acc[a], acc[a + 1], p0, p1);
    pk[i] = pack_bf16x2(p0, p1);
  }
}

// One softmax step of a query row (one thread, one TMEM lane) over kW keys:
// a 128-key tile, or a 64-key half tile. Reads the raw scores at TMEM column
// colS, folds them into the running max m (log2 units) and the running sum
// l, writes P as bf16 over the first kW / 2 columns, and rescales O (column
// colO) when the max grew past the headroom. Tiles that need no mask entries
// added (fast_route: every causal tile, the all-zero, causal-pattern and
// prefix tiles of an explicit mask; positive scale) take a single pass
// against the running max; keys c > lim are excluded there when diag is set.
// The others, and the first tile, take two passes through sc. False when a
// bounded wait gave up.
template <bool kMasked, int kW>
__device__ __forceinline__ bool softmax_step(const AttnArgs& args, uint32_t lane_base,
                                             uint32_t colS, uint32_t colO,
                                             const ScoreChunk<kMasked>& sc, bool fast_route,
                                             bool diag, int lim, int r, uint32_t n, float& m,
                                             float& l, uint64_t* pv_bar, uint32_t pv_par,
                                             const WaitCtl& ctl) {
  constexpr int kC = kW / 32;  // 32-key chunks
  static_assert(kW == 64 || kW == kBKV, "tile width");
  uint32_t raw[kW];
#pragma unroll
  for (int c = 0; c < kC; ++c)
    tmem_ld32(lane_base + colS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(raw + c * 32));
  tmem_ld_wait();
  reg_fence(raw);
  float alpha = 1.f;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 4 paired partial sums
  // Fast-route tiles after the first: one pass against the running max m,
  // writing P (64 keys per store). Every p is then <= 2^8 unless the max
  // grew by more than the headroom, so a row sum <= 2^8 proves no rescale
  // is due; otherwise (rare: many keys near the max, or a new max) the
  // tile's true max is taken and, only if it grew past the headroom, the
  // tile is redone exactly below (new max, O rescaled). The first tile and
  // the tiles that need their mask entries added take the exact two-pass
  // route. The choice is warp-uniform (a row whose max is still -inf fails
  // the row-sum test).
  bool exact = !(fast_route && n > 0);
  float rowsum = 0.f;
  if (!exact) {
#pragma unroll
    for (int c2 = 0; c2 < kC; c2 += 2) {
      uint32_t pk[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t(&ph)[16] = *reinterpret_cast<uint32_t(*)[16]>(pk + 16 * h2);
        if (diag)
          p_chunk_causal<true>(raw + (c2 + h2) * 32, c2 + h2, lim, args.scale_log2, m, ph,
                               acc);
        else
          p_chunk_causal<false>(raw + (c2 + h2) * 32, c2 + h2, r, args.scale_log2, m, ph,
                                acc);
      }
      tmem_st32(lane_base + colS + 16 * c2, pk);
    }
    rowsum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    if (__any_sync(0xffffffffu, !(rowsum <= 256.f))) {
      const float mt = (diag ? raw_row_max<true>(raw, lim) : raw_row_max<false>(raw, r)) *
                       args.scale_log2;
      exact = __any_sync(0xffffffffu, !(mt <= m + kRescaleThreshold));
      if (exact) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      }
    }
  }
  if (exact) {
    float mt;
    if (fast_route) {
      // positive scale: the maximum of the raw scores gives the maximum of
      // the scaled ones
      mt = diag ? raw_row_max<true>(raw, lim) : raw_row_max<false>(raw, r);
      mt *= args.scale_log2;
    } else {
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        float x[32];
        sc.apply(raw + c * 32, c, args.scale_log2, 0.f, x);
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          m4[0] = fmax3(m4[0], x[i], x[i + 1]);
          m4[1] = fmax3(m4[1], x[i + 2], x[i + 3]);
          m4[2] = fmax3(m4[2], x[i + 4], x[i + 5]);
          m4[3] = fmax3(m4[3], x[i + 6], x[i + 7]);
        }
        // keep the scaled, masked scores: the exponentials below need
        // neither the mask nor the scale again
#pragma unroll
        for (int i = 0; i < 32; ++i) raw[c * 32 + i] = __float_as_uint(x[i]);
      }
      mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
    }
    float m_new = m;
    if (n == 0) {
      m_new = mt;
    } else if (mt > m + kRescaleThreshold) {
      m_new = mt;
      alpha = fast_exp2(m - m_new);
    }
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    m = m_new;

    // P as bf16 pairs over the first kW / 2 columns of the S buffer (every
    // score is in registers by now), 32 keys per store.
#pragma unroll
    for (int c = 0; c < kC; ++c) {
      const uint32_t* rc = raw + c * 32;
      uint32_t pk[16];
      if (fast_route) {
        if (diag)
          p_chunk_causal<true>(rc, c, lim, args.scale_log2, m_use, pk, acc);
        else
          p_chunk_causal<false>(rc, c, r, args.scale_log2, m_use, pk, acc);
      } else {
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(rc[i]) - m_use;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = fast_exp2(x[2 * i]);
          const float p1 = fast_exp2(x[2 * i + 1]);
          fadd2(acc[2 * (i & 3)], acc[2 * (i & 3) + 1], acc[2 * (i & 3)],
                acc[2 * (i & 3) + 1], p0, p1);
          pk[i] = pack_bf16x2(p0, p1);
        }
      }
      tmem_st16(lane_base + colS + 16 * c, pk);
    }
    rowsum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));

    // The rescale needs O to hold P_{n-1} V_{n-1}. On 128-key tiles that PV
    // was issued before this S, and the commit behind s_full covers every
    // earlier MMA (pv_bar null); on half tiles it is issued after this S and
    // its own commit (pv_bar) is awaited. The rescale lands before PV_n, which
    // waits for p_full. (Only the exact route can change the max.)
    if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
      if (pv_bar) {
        if (!mbar_wait_warp(pv_bar, pv_par, ctl, 23)) return false;
        tc_fence_after();
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + colO + c * 32, rr);
        tmem_ld_wait();
        reg_fence(rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
        tmem_st32(lane_base + colO + c * 32, rr);
      }
    }
  }  // exact
  l = l * alpha + rowsum;
  return true;
}

template <bool kMasked, bool kRope, bool kHalf, bool kPvIssuer>
__global__ void __launch_bounds__(kThreads, 1)
    mla_attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQn,
                            const __grid_constant__ CUtensorMap tmQp,
                            const __grid_constant__ CUtensorMap tmKn,
                            const __grid_constant__ CUtensorMap tmKp,
                            const __grid_constant__ CUtensorMap tmV,
                            const __grid_constant__ CUtensorMap tmOut, const AttnArgs args) {
  static_assert(kHalf || !kPvIssuer, "the PV issuer serves half-tile scores");
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[2];     // query tile i is in shared memory
  __shared__ uint64_t q_rot[2];      // its rotary part is rotated (rotary calls only)
  __shared__ uint64_t ring_full[kRing], ring_empty[kRing];
  // S ready / P written: [query tile] on 128-key tiles, [2 * query tile +
  // half] on half tiles
  __shared__ uint64_t s_full[4], p_full[4];
  __shared__ uint64_t pv_done[2];   // half tiles: a PV product of query tile i completed
  // half tiles with a PV issuer: PV(u) of query tile i has been issued,
  // [2 * i + u % 2]
  __shared__ uint64_t pv_issued[4];
  __shared__ uint64_t o_final[2];
  __shared__ uint64_t drain_bar[3];  // issuer i's MMAs (i = 2: the PV issuer) have completed
  __shared__ uint64_t s_issued[2];  // issuer i has issued (or skipped) S of its next tile
  __shared__ uint64_t never_bar;    // no thread ever arrives (failure-detection test)
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int mask_n_act[2];  // half tiles under a mask: each query tile's active prefix
  __shared__ int mask_half;      // ... and whether both are prefixes (else 128-key tiles)

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // CTA -> (b, h, pair): groups of head_group_for(T) heads, longest pairs first
  // within a group.
  const int hg = head_group_for(args.T);
  const int per_group = hg * args.n_pairs;
  const int grp = blockIdx.x / per_group;
  const int rem = blockIdx.x - grp * per_group;
  const int b = grp / (kH / hg);
  const int h = (grp % (kH / hg)) * hg + rem % hg;
  const int pair = args.n_pairs - 1 - rem / hg;
  const int bh = b * kH + h;
  // Keys of this sequence: T, or valid_len[b] clamped to [0, T].
  const int n_keys =
      (!kMasked && args.valid_len) ? min(max(args.valid_len[b], 0), args.T) : args.T;

  PairTiles<kMasked> tiles;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    tiles.qt[i] = 2 * pair + i;
    tiles.exists[i] = tiles.qt[i] < args.n_qt;
    tiles.cls[i] = (kMasked && args.tile_class && tiles.exists[i])
                       ? args.tile_class + (size_t(b) * args.n_qt + tiles.qt[i]) * args.n_kv
                       : nullptr;
  }
  tiles.kv_end = (n_keys + kBKV - 1) / kBKV;
  tiles.end = kMasked ? args.n_kv : min(min(2 * pair + 2, args.n_qt), tiles.kv_end);
  const bool has_work = tiles.first() < tiles.end;

  WaitCtl ctl{&abort_flag, args.wait_limit_ns, kErrKernelAttn, args.err_word};

  // TMA loads (thread 0, the producer): query tile i (nope lo, nope hi, rope:
  // 48 KB), and block i of key tile k0 into ring slot `slot`.
  auto load_q = [&](uint32_t i) {
    uint8_t* sQ = smem + kOffQ + i * kQBytes;
    const int q0 = tiles.qt[i] * kBQ;
    mbar_arrive_expect_tx(&q_full[i], kQBytes);
    tma_load_3d(sQ, &tmQn, &q_full[i], 0, q0, bh);
    tma_load_3d(sQ + kBlock, &tmQn, &q_full[i], 64, q0, bh);
    tma_load_3d(sQ + 2 * kBlock, &tmQp, &q_full[i], 0, q0, bh);
  };
  auto load_block = [&](int i, uint32_t slot, int k0) {
    uint8_t* dst = smem + kOffRing + slot * kBlock;
    mbar_arrive_expect_tx(&ring_full[slot], kBlock);
    switch (i) {
      case 0: tma_load_3d(dst, &tmKn, &ring_full[slot], 0, k0, bh); break;
      case 1: tma_load_3d(dst, &tmKn, &ring_full[slot], 64, k0, bh); break;
      case 2: tma_load_3d(dst, &tmKp, &ring_full[slot], 0, k0, b); break;
      default: {
        // V for 64 keys, all 128 value dims: two 64 x 64 boxes, 8 KB apart
        const int kv = k0 + (i - 3) * 64;
        tma_load_3d(dst, &tmV, &ring_full[slot], 0, kv, bh);
        tma_load_3d(dst + kBlock / 2, &tmV, &ring_full[slot], 64, kv, bh);
        break;
      }
    }
  };
  // The first key tile's K blocks (ring slots 0..2) and query tile 0 are
  // loaded as soon as the barriers exist, overlapping the tensor-memory
  // allocation and the block-wide barrier; the producer loop skips them.
  constexpr uint32_t kPreBlocks = 3;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&q_full[0], 1);
    mbar_init(&q_full[1], 1);
    mbar_init(&q_rot[0], 128);
    mbar_init(&q_rot[1], 128);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&ring_full[s], 1);
      // released once per query tile: K blocks by its S issuer, V blocks by
      // its PV issuer (the same thread unless warp 3 issues the PVs)
      mbar_init(&ring_empty[s], tiles.exists[1] ? 2 : 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      if (kPvIssuer) mbar_init(&pv_issued[i], 1);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&drain_bar[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&o_final[i], 1);
      mbar_init(&s_issued[i], 1);
      mbar_init(&pv_done[i], 1);
      mbar_init(&never_bar, 1);
    }
    fence_barrier_init();
    if (has_work) {
      load_q(0);
      for (uint32_t i = 0; i < kPreBlocks; ++i) load_block(int(i), i, tiles.first() * kBKV);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if constexpr (kMasked && kHalf) {
    // Half tiles take a query tile's active key tiles as a prefix [0, n_act).
    // Under an explicit mask warp 3 reads the tile classes of both query
    // tiles (32 per ballot): n_act is the index of the first skipped tile,
    // and the CTA keeps 128-key tiles if an active tile follows a skipped one
    // in either query tile.
    if (warp == 3) {
      bool prefix = true;
#pragma unroll 1
      for (int i = 0; i < 2; ++i) {
        int f = 0;
        if (tiles.exists[i]) {
          f = args.n_kv;
          const uint8_t* cls = tiles.cls[i];
          for (int base = 0; base < args.n_kv; base += 32) {
            const int kt = base + lane;
            const bool in = kt < args.n_kv;
            const bool act = in && (cls == nullptr || cls[kt] != kTileSkip);
            const unsigned am = __ballot_sync(0xffffffffu, act);
            const unsigned im = __ballot_sync(0xffffffffu, in && !act);
            if (f == args.n_kv && im != 0u) f = base + __ffs(int(im)) - 1;
            if (f < args.n_kv) {
              const int sh = f - base;  // f lies in this chunk or an earlier one
              const unsigned later = sh <= 0 ? am : (am & (0xffffffffu << sh));
              if (later != 0u) prefix = false;
            }
          }
        }
        if (lane == 0) mask_n_act[i] = f;
      }
      if (lane == 0) mask_half = prefix ? 1 : 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  // Half-tile scores (kHalf): always for causal and valid-length calls; under
  // an explicit mask when both query tiles' active key tiles are prefixes.
  // n_act: active key tiles of each query tile, visited [0, vis_end).
  const bool half = kHalf && (!kMasked || mask_half != 0);
  auto n_act_of = [&](int i) -> int {
    if constexpr (kMasked) return mask_n_act[i];
    return tiles.exists[i] ? min(tiles.qt[i] + 1, tiles.end) : 0;
  };
  const int vis_end = kMasked ? max(n_act_of(0), n_act_of(1)) : tiles.end;

  if (warp < 4) {
  // Warpgroup 0 (TMA producer, MMA issuer, two idle warps) hands registers
  // to the two softmax warpgroups.
  setmaxnreg_dec<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && has_work) {
      prefetch_tensormap(&tmQn);
      prefetch_tensormap(&tmQp);
      prefetch_tensormap(&tmKn);
      prefetch_tensormap(&tmKp);
      prefetch_tensormap(&tmV);
      // Query tile 0 and the first key tile's K blocks came with the
      // barriers; query tile 1 follows them, so the first S MMA waits for
      // 96 KB rather than 144 KB.
      bool q1_issued = false;
      uint32_t issued = 0, issued_par = 0;
      uint32_t s = 0;  // block sequence number
      bool ok = true;
      // Key tiles are prefetched into L2 two visited tiles ahead of their
      // loads (the first CTA of a head group to reach a tile otherwise waits
      // on DRAM with the ring slots already committed).
      auto prefetch_tile = [&](int pt) {
        if (pt >= tiles.end) return;
        const int p0 = pt * kBKV;
        tma_prefetch_l2_3d(&tmKn, 0, p0, bh);
        tma_prefetch_l2_3d(&tmKn, 64, p0, bh);
        tma_prefetch_l2_3d(&tmKp, 0, p0, b);
        tma_prefetch_l2_3d(&tmV, 0, p0, bh);
        tma_prefetch_l2_3d(&tmV, 64, p0, bh);
        tma_prefetch_l2_3d(&tmV, 0, p0 + 64, bh);
        tma_prefetch_l2_3d(&tmV, 64, p0 + 64, bh);
      };
      int pf = tiles.next(tiles.first());
      prefetch_tile(pf);
      for (int kt = tiles.first(); ok && kt < tiles.end; kt = tiles.next(kt)) {
        const int k0 = kt * kBKV;
        if (pf < tiles.end) {
          pf = tiles.next(pf);
          prefetch_tile(pf);
        }
#pragma unroll 1
        for (int i = 0; i < kBlocksPerTile; ++i, ++s) {
          const uint32_t slot = s % kRing;
          const uint32_t par = (s / kRing) & 1u;
          if (s >= kPreBlocks) {
            if (!mbar_wait(&ring_empty[slot], par ^ 1u, ctl, 1)) { ok = false; break; }
            load_block(i, slot, k0);
          }
          issued |= 1u << slot;
          issued_par = (issued_par & ~(1u << slot)) | (par << slot);
          if (s == 2 && tiles.exists[1]) {
            load_q(1);
            q1_issued = true;
          }
        }
      }
      if (ok && tiles.exists[1] && !q1_issued) {  // not reached: every tile has 5 blocks
        load_q(1);
        q1_issued = true;
      }
      if (!ok) {
        // let the copies already issued land before the CTA's memory goes away
        int zero = 0;
        WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
        mbar_wait(&q_full[0], 0, drain, 2);
        if (q1_issued) mbar_wait(&q_full[1], 0, drain, 2);
        for (int k = 0; k < kRing; ++k)
          if (issued & (1u << k)) mbar_wait(&ring_full[k], (issued_par >> k) & 1u, drain, 3);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues the MMAs of query tile 0, warp 2 those of query tile 1,
    // so a tile's PV is never held up behind the other tile's queued MMAs in
    // one issuing thread. Per visited key tile j an issuer runs
    //   O += P_{j-1} V_{j-1}, release V_{j-1};  S = Q K_j^T, release K_j.
    // The S MMAs keep a strict order S0_0, S1_0, S0_1, S1_1, ... (s_issued),
    // which keeps the two softmax warpgroups out of phase.
    const int qi = warp - 1;
    if (lane == 0 && has_work && tiles.exists[qi]) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBQ, kBKV, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBQ, kDV, false, true);
      const uint32_t ring0 = smem_u32(smem + kOffRing);
      const uint32_t sQ = smem_u32(smem + kOffQ + qi * kQBytes);
      const uint32_t s_tmem = tmem_base + kColS + 128 * qi;  // S, and P over it
      const uint32_t o_tmem = tmem_base + kColO + 128 * qi;
      const bool pair = tiles.exists[1];
      bool ok = mbar_wait(&q_full[qi], 0, ctl, 10);
      if (kRope && ok) ok = mbar_wait(&q_rot[qi], 0, ctl, 16);
      bool issued_any = false;

      auto wait_block = [&](uint32_t seq, uint32_t site) -> bool {
        return mbar_wait(&ring_full[seq % kRing], (seq / kRing) & 1u, ctl, site);
      };
      auto block_addr = [&](uint32_t seq) -> uint32_t { return ring0 + (seq % kRing) * kBlock; };
      // Each issuer releases every ring block once: a commit after its MMAs
      // that read the block, or a plain arrive when its query tile did not use
      // the key tile. Either comes after the block has landed, so it cannot
      // count toward an earlier fill of the same slot.
      auto release = [&](uint32_t seq, bool used) {
        if (used)
          mma_commit(&ring_empty[seq % kRing]);
        else
          mbar_arrive(&ring_empty[seq % kRing]);
      };
      if (half) {
        // Half tiles: sub-tile u = 2 kt + hb is keys kt*128 + 64 hb .. +63 of
        // this query tile's active key tiles 0 .. n_act-1 (a prefix of the
        // visited ones); its scores go to buffer hb (64 TMEM columns, P over
        // the first 32). Order: S(0), S(1), then for each u: PV(u), S(u+2),
        // so the scores of the next half tile are ready while the softmax
        // works on this one. S(u+2) reuses the buffer PV(u) reads; the tensor
        // pipe runs one thread's MMAs in order.
        constexpr uint32_t idesc_sh = idesc_bf16_f32(kBQ, kBKV / 2, false, false);
        const int n_act = n_act_of(qi);
        const int n_sub = 2 * n_act;
        auto issue_s = [&](int u) -> bool {
          const int kt = u >> 1, hb = u & 1;
          const uint32_t base = kBlocksPerTile * uint32_t(kt);
          if (hb == 0 &&
              (!wait_block(base, 13) || !wait_block(base + 1, 13) || !wait_block(base + 2, 13)))
            return false;
          tc_fence_after();
          const uint32_t s_buf = s_tmem + 64 * hb;
#pragma unroll
          for (int blk = 0; blk < 3; ++blk) {
            const uint32_t kb = block_addr(base + blk) + hb * (kBlock / 2);  // keys 64 hb ..
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t qd = sdesc_sw128(sQ + blk * kBlock + kk * 32, 16, 1024);
              const uint64_t kd = sdesc_sw128(kb + kk * 32, 16, 1024);
              mma_ss(s_buf, qd, kd, idesc_sh, (blk | kk) != 0 ? 1u : 0u);
            }
          }
          issued_any = true;
          mma_commit(&s_full[2 * qi + hb]);
          if (hb == 1) {  // both halves read the K blocks
            release(base, true);
            release(base + 1, true);
            release(base + 2, true);
          }
          return true;
        };
        // O += P V over the 64 keys of one V block, then release it.
        auto issue_pv = [&](int u) -> bool {
          const int kt = u >> 1, hb = u & 1;
          const uint32_t vseq = kBlocksPerTile * uint32_t(kt) + 3 + hb;
          if (!wait_block(vseq, 12)) return false;
          if (!mbar_wait(&p_full[2 * qi + hb], uint32_t(u >> 1) & 1u, ctl, 11)) return false;
          tc_fence_after();
          const uint32_t vb = block_addr(vseq);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t vd = sdesc_sw128(vb + kk * 16 * 128, kBlock / 2, 1024);
            mma_ts(o_tmem, s_tmem + 64 * hb + kk * 8, vd, idesc_o, (u | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&pv_done[qi]);
          release(vseq, true);
          return true;
        };
        if (ok && n_sub > 0) ok = issue_s(0);
        if (ok && n_sub > 0) ok = issue_s(1);
        if constexpr (kPvIssuer) {
          // PV(u) comes from warp 3; S(u+2) follows it into the buffer.
          (void)issue_pv;
          for (int u = 0; ok && u + 2 < n_sub; ++u) {
            ok = mbar_wait(&pv_issued[2 * qi + (u & 1)], uint32_t(u >> 1) & 1u, ctl, 18);
            if (ok) {
              tc_fence_after();
              ok = issue_s(u + 2);
            }
          }
        } else {
          for (int u = 0; ok && u < n_sub; ++u) {
            ok = issue_pv(u);
            if (ok && u + 2 < n_sub) ok = issue_s(u + 2);
          }
          if (ok) mma_commit(&o_final[qi]);
        }
        // The visited key tiles past this query tile's last one (causal: the
        // other query tile's diagonal; under a mask, up to the other query
        // tile's prefix) are released unused, block by block once landed,
        // after every block this tile used.
        for (int kt = n_act; ok && kt < vis_end; ++kt)
          for (uint32_t i = 0; ok && i < uint32_t(kBlocksPerTile); ++i) {
            const uint32_t seq = kBlocksPerTile * uint32_t(kt) + i;
            ok = wait_block(seq, 13);
            if (ok) release(seq, false);
          }
      } else {
        uint32_t n_pv = 0;       // PVs issued
        uint32_t n_tiles = 0;    // visited key tiles so far
        int prev = -1;           // previous visited key tile
        bool prev_act = false;   // did this query tile use it
        uint32_t prev_base = 0;  // block sequence number of prev's first block
        // O += P V for the previous key tile, then release its two V blocks.
        auto finish_prev = [&]() -> bool {
          if (!wait_block(prev_base + 3, 12) || !wait_block(prev_base + 4, 12)) return false;
          if (prev_act) {
            if (!mbar_wait(&p_full[qi], n_pv & 1u, ctl, 11)) return false;
            tc_fence_after();
            // Each V block holds 64 keys x 128 value dims, MN-major: value dims
            // 0..63 and 64..127 are two 8 KB halves (LBO), 8-key groups 1 KB
            // apart (SBO). 16 keys per MMA = 8 packed TMEM columns of P.
#pragma unroll
            for (int vh = 0; vh < 2; ++vh) {
              const uint32_t vb = block_addr(prev_base + 3 + vh);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t acc = (n_pv > 0 || vh > 0 || kk > 0) ? 1u : 0u;
                const uint64_t vd = sdesc_sw128(vb + kk * 16 * 128, kBlock / 2, 1024);
                mma_ts(o_tmem, s_tmem + (vh * 4 + kk) * 8, vd, idesc_o, acc);
              }
            }
            ++n_pv;
            issued_any = true;
          }
          release(prev_base + 3, prev_act);
          release(prev_base + 4, prev_act);
          return true;
        };

        uint32_t base = 0;
        for (int kt = tiles.first(); ok && kt < tiles.end;
             kt = tiles.next(kt), base += kBlocksPerTile, ++n_tiles) {
          const bool act = tiles.active(qi, kt);
          if (prev >= 0 && !finish_prev()) { ok = false; break; }
          if (!wait_block(base, 13) || !wait_block(base + 1, 13) || !wait_block(base + 2, 13)) {
            ok = false;
            break;
          }
          // S order: tile 1 waits for tile 0's S of this key tile, tile 0 for
          // tile 1's S of the previous one.
          if (pair) {
            if (qi == 1) {
              if (!mbar_wait(&s_issued[0], n_tiles & 1u, ctl, 15)) { ok = false; break; }
            } else if (n_tiles > 0) {
              if (!mbar_wait(&s_issued[1], (n_tiles - 1) & 1u, ctl, 15)) { ok = false; break; }
            }
          }
          if (act) {
            tc_fence_after();
            const uint32_t k_addr[3] = {block_addr(base), block_addr(base + 1),
                                        block_addr(base + 2)};
#pragma unroll
            for (int blk = 0; blk < 3; ++blk) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t qd = sdesc_sw128(sQ + blk * kBlock + kk * 32, 16, 1024);
                const uint64_t kd = sdesc_sw128(k_addr[blk] + kk * 32, 16, 1024);
                mma_ss(s_tmem, qd, kd, idesc_s, (blk | kk) != 0 ? 1u : 0u);
              }
            }
            issued_any = true;
            mma_commit(&s_full[qi]);
          }
          if (pair) mbar_arrive(&s_issued[qi]);
          release(base, act);
          release(base + 1, act);
          release(base + 2, act);
          prev = kt;
          prev_act = act;
          prev_base = base;
        }
        if (ok && prev >= 0) ok = finish_prev();
        if (ok && n_pv > 0) mma_commit(&o_final[qi]);
      }
      if (!ok && issued_any) {
        mma_commit(&drain_bar[qi]);
        int zero = 0;
        WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
        mbar_wait(&drain_bar[qi], 0, drain, 14);
      }
    }
  }
  if constexpr (kPvIssuer) {
    if (warp == 3 && lane == 0 && has_work && half) {
      // ------------------------------------------------------------ PV issuer
      // For each query tile in turn: once P(u) is written and the V block of
      // half tile u has landed, O += P(u) V, release the V block, and tell
      // the tile's S issuer (pv_issued). Spins on non-blocking tests: parking
      // on one tile's barrier would hold up the other tile's PV. The tile
      // loop stays rolled: unrolled, the tighter spin measured slower
      // (B=1 T=32768: 20.5-20.6 against 19.8-19.9 ms), the thread sharing
      // its SM sub-partition with two softmax warps.
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBQ, kDV, false, true);
      const uint32_t ring0 = smem_u32(smem + kOffRing);
      int n_sub[2], next[2] = {0, 0};
#pragma unroll
      for (int t = 0; t < 2; ++t)
        n_sub[t] = 2 * n_act_of(t);
      bool ok = true, issued_any = false;
      unsigned long long last = globaltimer_ns();
      while (ok && (next[0] < n_sub[0] || next[1] < n_sub[1])) {
        bool progress = false;
#pragma unroll 1
        for (int t = 0; t < 2; ++t) {
          const int u = next[t];
          if (u >= n_sub[t]) continue;
          const int kt = u >> 1, hb = u & 1;
          const uint32_t vseq = kBlocksPerTile * uint32_t(kt) + 3 + hb;
          if (!mbar_test(&p_full[2 * t + hb], uint32_t(u >> 1) & 1u) ||
              !mbar_test(&ring_full[vseq % kRing], (vseq / kRing) & 1u))
            continue;
          tc_fence_after();
          const uint32_t o_tmem = tmem_base + kColO + 128 * t;
          const uint32_t p_tmem = tmem_base + kColS + 128 * t + 64 * hb;
          const uint32_t vb = ring0 + (vseq % kRing) * kBlock;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t vd = sdesc_sw128(vb + kk * 16 * 128, kBlock / 2, 1024);
            mma_ts(o_tmem, p_tmem + kk * 8, vd, idesc_o, (u | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&pv_done[t]);
          mma_commit(&ring_empty[vseq % kRing]);
          if (u + 1 == n_sub[t]) mma_commit(&o_final[t]);
          tc_fence_before();
          mbar_arrive(&pv_issued[2 * t + hb]);
          issued_any = true;
          next[t] = u + 1;
          progress = true;
        }
        if (progress) {
          last = globaltimer_ns();
        } else if (abort_flag) {
          ok = false;
        } else if (globaltimer_ns() - last > args.wait_limit_ns) {
          abort_flag = 1;
          atomicCAS(args.err_word, 0u, kErrTimeoutFlag | kErrKernelAttn | 19u);
          __threadfence();
          ok = false;
        }
      }
      if (!ok && issued_any) {
        mma_commit(&drain_bar[2]);
        int zero = 0;
        WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
        mbar_wait(&drain_bar[2], 0, drain, 14);
      }
    }
  }
  named_barrier_sync(kBarTeardown, kThreads);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  } else {
  setmaxnreg_inc<kRegsSoftmax>();
  {
    // ------------------------------------------------------------ softmax / epilogue
    const int wi = (warp - 4) >> 2;  // query tile of this warpgroup
    const int quad = warp & 3;       // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;  // row within the tile == TMEM lane
    const int qt = tiles.qt[wi];
    const int q = qt * kBQ + r;
    const uint32_t lane_base = tmem_addr(tmem_base, quad * 32, 0);
    const uint32_t colS = kColS + 128 * wi;
    const uint32_t colO = kColO + 128 * wi;
    const bool row_valid = tiles.exists[wi] && q < args.T;
    const __nv_bfloat16* mrow =
        (kMasked && row_valid) ? args.mask + (size_t(b) * args.T + q) * args.mask_ld : nullptr;

    bool ok = true;
    if (kRope && has_work && tiles.exists[wi]) {
      // Rotary calls: rotate this row's q_pe (64 values, the tile's third
      // 16 KB block, 128-byte rows with the 16-byte chunks XOR-swizzled by
      // row % 8) in shared memory once its TMA load has landed; pair i =
      // elements 2i, 2i+1 turns by the (f cos, f sin) tabulated for this
      // query's position. The MMA issuer waits for all 128 rows (q_rot).
      ok = mbar_wait(&q_full[wi], 0, ctl, 24);
      if (ok && row_valid) {
        uint8_t* rowp = smem + kOffQ + wi * kQBytes + 2 * kBlock + r * 128;
        const float4* cs = reinterpret_cast<const float4*>(args.rope_cs + (size_t(b) * args.T + q) * 32);
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 16-byte chunk c holds pairs 4c .. 4c+3
          uint4* chunk = reinterpret_cast<uint4*>(rowp + ((c ^ (r & 7)) << 4));
          uint4 w = *chunk;
          const float4 a = __ldg(cs + 2 * c), bq = __ldg(cs + 2 * c + 1);
          const float csn[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
          uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_bits_to_float(wp[e] & 0xffffu);
            const float x1 = bf16_bits_to_float(wp[e] >> 16);
            const float cc = csn[2 * e], ss = csn[2 * e + 1];
            wp[e] = pack_bf16x2(fmaf(x0, cc, -x1 * ss), fmaf(x1, cc, x0 * ss));
          }
          *chunk = w;
        }
        fence_proxy_async_smem();  // the MMA reads it through the async proxy
      }
      mbar_arrive(&q_rot[wi]);
    }
    float m = -INFINITY;  // running max, log2 units
    float l = 0.f;        // running sum of p (fp32, unrounded)
    uint32_t n = 0;
    if (half) {
      // Half tiles: 64 keys per step, the two score buffers of this query
      // tile in turn.
      const int n_sub = (has_work && tiles.exists[wi]) ? 2 * n_act_of(wi) : 0;
      for (int u = 0; u < n_sub; ++u) {
        const int kt = u >> 1, hb = u & 1;
        const int k0 = kt * kBKV + 64 * hb;
        if (args.test_stall && wi == 0 && blockIdx.x == 0 &&
            !mbar_wait_warp(&never_bar, 0, ctl, 30)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(&s_full[2 * wi + hb], uint32_t(u >> 1) & 1u, ctl, 20)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // keys c <= lim of the half tile: c + 64 hb <= r on the diagonal tile
        // (none for rows r < 64 in its second half), and none at or past the
        // sequence's key count. Under a mask the tile's class gives the
        // limit: the causal pattern as above, a prefix class its last key
        // minus 64 hb; mixed tiles add their 64 mask entries.
        ScoreChunk<kMasked> sc;
        bool diag, fast_route;
        int lim;
        if constexpr (kMasked) {
          // A second half that starts at or past T (the last key tile, T not a
          // multiple of 128) holds no keys: class zero, so no mask entry is
          // read for it and the limit below cuts every key.
          const uint8_t tile_cls = args.T - k0 <= 0 ? uint8_t(kTileZero)
                                   : tiles.cls[wi] ? tiles.cls[wi][kt] : uint8_t(kTileMixed);
          const bool causal_tile = tile_cls == kTileCausal;
          const bool prefix_tile = tile_cls >= kTilePrefix;
          diag = causal_tile || prefix_tile || args.T - k0 < kBKV / 2;
          lim = min(causal_tile ? r - 64 * hb
                                : (prefix_tile ? int(tile_cls) - kTilePrefix - 64 * hb : kBKV / 2 - 1),
                    args.T - 1 - k0);
          fast_route = (tile_cls == kTileZero || causal_tile || prefix_tile) && args.scale_log2 > 0.f;
          sc.cls = row_valid ? tile_cls : uint8_t(kTileZero);
          sc.row_valid = row_valid;
          sc.mrow = mrow + (row_valid ? k0 : 0);
          sc.kvalid = args.T - k0;
          sc.mask_vec = args.mask_vec;
          sc.diag_row = (causal_tile || prefix_tile) ? lim : kBKV;
        } else {
          const bool causal_tile = kt == qt;
          diag = causal_tile || n_keys - k0 < kBKV / 2;
          lim = min(causal_tile ? r - 64 * hb : kBKV / 2 - 1, n_keys - 1 - k0);
          fast_route = args.scale_log2 > 0.f;
          sc.cls = kTileZero;
          sc.row_valid = row_valid;
          sc.mrow = nullptr;
          sc.kvalid = args.T - k0;
          sc.mask_vec = 0;
          sc.diag_row = diag ? lim : kBKV;
        }
        // Before rescaling O the step waits for PV(u-1): at most one PV of
        // this query tile is outstanding here (S(u), awaited above, was issued
        // after PV(u-2)), so the parity of pv_done is unambiguous.
        if (!softmax_step<kMasked, kBKV / 2>(args, lane_base, colS + 64 * hb, colO, sc,
                                             fast_route, diag, lim, r, n, m, l,
                                             &pv_done[wi], (n - 1) & 1u, ctl)) {
          ok = false;
          break;
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[2 * wi + hb]);
        ++n;
      }
    } else {
      for (int kt = tiles.first(); kt < tiles.end; kt = tiles.next(kt)) {
        if (!tiles.active(wi, kt)) continue;
        const int k0 = kt * kBKV;
        // Failure-detection test: query tile 0 of the first CTA waits on a
        // barrier nothing arrives on; the bounded wait must time out, abort the
        // CTA cleanly and report through the status word.
        if (args.test_stall && wi == 0 && blockIdx.x == 0 &&
            !mbar_wait_warp(&never_bar, 0, ctl, 30)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(&s_full[wi], n & 1u, ctl, 20)) { ok = false; break; }
        tc_fence_after();
        // The 128 scores of this thread's row are read from tensor memory once
        // and kept in registers for both passes (row maximum, exponentials).
        ScoreChunk<kMasked> sc;
        sc.cls = (kMasked && row_valid)
                     ? (tiles.cls[wi] ? tiles.cls[wi][kt] : uint8_t(kTileMixed))
                     : uint8_t(kTileZero);
        sc.row_valid = row_valid;
        sc.mrow = mrow + (kMasked && row_valid ? k0 : 0);
        sc.kvalid = args.T - k0;
        sc.mask_vec = args.mask_vec;
        // The fast route (scores need no mask add): every tile of the causal
        // kernel, and the all-zero and causal-pattern tiles of an explicit
        // mask. It needs a positive scale (the raw maximum is then the scaled
        // one).
        const uint8_t tile_cls =
            kMasked ? (tiles.cls[wi] ? tiles.cls[wi][kt] : uint8_t(kTileMixed)) : uint8_t(kTileZero);
        const bool causal_tile = !kMasked ? kt == qt : tile_cls == kTileCausal;
        const bool prefix_tile = kMasked && tile_cls >= kTilePrefix;
        const bool fast_route =
            (tile_cls == kTileZero || tile_cls == kTileCausal || prefix_tile) &&
            args.scale_log2 > 0.f;
        // Keys c <= lim of the tile are allowed on the fast route: c <= r on a
        // causal diagonal tile, c <= the class's limit on a prefix tile, and
        // none at or past the sequence's key count (T, or valid_len[b]). `diag`
        // marks the tiles where that limit cuts (warp-uniform).
        const int key_end = kMasked ? args.T : n_keys;
        const bool diag = causal_tile || prefix_tile || key_end - k0 < kBKV;
        const int lim = min(causal_tile ? r : (prefix_tile ? int(tile_cls) - kTilePrefix : kBKV - 1),
                            key_end - 1 - k0);
        sc.diag_row = (kMasked ? (causal_tile || prefix_tile) : diag) ? lim : kBKV;
        if (!softmax_step<kMasked, kBKV>(args, lane_base, colS, colO, sc, fast_route, diag, lim, r,
                                         n, m, l, nullptr, 0, ctl)) {
          ok = false;
          break;
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[wi]);
        ++n;
      }
    }

    // epilogue: O / l -> bf16 -> out[b, q, h*128 + e]. The rows are staged
    // in this query tile's Q buffer (free: its last S product has completed)
    // as two 128-row x 64-dim boxes in the TMA 128-byte swizzle (16-byte
    // chunk c of row r at chunk c ^ (r % 8), so the warp's stores spread
    // over all banks), then written by two TMA stores. Rows at or past T
    // fall outside the output map's T extent and are not written.
    // A query tile with no key tiles to visit writes zeros; its buffer may
    // still be receiving its query rows, which land first. Every warp of the
    // warpgroup reaches the staging barrier whatever happened before it; the
    // rows are stored only if all four staged theirs.
    bool stage_ok = false;
    if (ok && n > 0) {
      stage_ok = mbar_wait_warp(&o_final[wi], 0, ctl, 22);
      if (stage_ok) tc_fence_after();
    } else if (ok) {
      stage_ok = !(has_work && tiles.exists[wi]) || mbar_wait_warp(&q_full[wi], 0, ctl, 25);
    }
    uint8_t* stage = smem + kOffQ + wi * kQBytes;
    if (stage_ok) {
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        if (n > 0) {
          tmem_ld32(lane_base + colO + c * 32, rr);
          tmem_ld_wait();
          reg_fence(rr);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = 0u;
        }
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * inv_l,
                                  __uint_as_float(rr[2 * i + 1]) * inv_l);
        // dims 32c .. 32c+31: box c / 2, 16-byte chunks 4 (c % 2) .. + 3
        uint8_t* rowp = stage + (c >> 1) * kBlock + r * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int chunk = 4 * (c & 1) + i;
          *reinterpret_cast<uint4*>(rowp + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
      fence_proxy_async_smem();
    }
    const bool all_staged = named_barrier_and(kBarStage0 + wi, 128, stage_ok);
    if (all_staged && tiles.exists[wi] && quad == 0 && lane == 0) {
      tma_store_3d(&tmOut, stage, h * kDV, qt * kBQ, b);
      tma_store_3d(&tmOut, stage + kBlock, h * kDV + 64, qt * kBQ, b);
      bulk_commit_group();
      bulk_wait_group_read<0>();  // the staging buffer stays valid until read
    }
  }

  tc_fence_before();
  named_barrier_sync(kBarTeardown, kThreads);
  }
}

// ---------------------------------------------------------------- CTA-pair kernel
// The attention kernel on a pair of SMs. A cluster of two CTAs computes query
// tiles 2p (even CTA) and 2p+1 (odd CTA) of one (b, h): each SM holds one
// 128-row query tile, and each score and PV product is ONE
// tcgen05.mma.cta_group::2 of M = 256 rows issued by the even CTA:
//   S (256 x 128 keys, K = 128 nope + 64 rope): each CTA holds its 128 query
//     rows and 64 of the 128 keys (the B operand is split by columns);
//   PV (256 x 128 value dims, K = 128 keys): P comes from each CTA's tensor
//     memory, each CTA holds 64 of the 128 value dims of all 128 keys.
// So every K/V byte a CTA loads serves 256 query rows, as in the one-SM
// kernel, while each SM runs a single softmax warpgroup (its 128 rows), and
// S is triple-buffered in tensor memory: the scores of the next two key tiles
// are computed or queued while the softmax of one tile runs. Issue order of
// the even CTA's MMA thread:
//   S_0, S_1, S_2, [P_0] PV_0, S_3, [P_1] PV_1, S_4, ...
// (P_j aliases S_j's buffer; S_{j+3} reuses it after PV_j in issue order).
//
// A cluster works on two items, query-tile pairs p and n_pairs - 1 - p of the
// same (b, h) (one item for the middle pair when n_pairs is odd), so every
// cluster visits the same number of key tiles and one launch, barrier set and
// tensor-memory allocation serve both. Both items' query tiles are loaded up
// front (two query buffers); the key-tile sequence runs on across the item
// boundary, and the items share one O accumulator (the second item's first
// PV, which overwrites O, waits for its first P, which the softmax threads
// write only after they have read the first item's O).
//
// Cross-CTA signals, chosen for their cost on B200 (a remote mbarrier arrive
// with release at cluster scope stalls its thread for about 0.7 us, so no
// per-block or per-softmax-warp thread handshake crosses the pair):
//  - ring blocks: both CTAs' TMA copies complete on the even CTA's barrier
//    (cp.async.bulk.tensor .cta_group::2); the even CTA arms both CTAs' bytes;
//  - query tiles: each CTA's copies complete on its own barrier (the odd
//    CTA's softmax warps rotate them under the rotary calls), and a helper
//    thread of the odd CTA forwards "ready" once per item;
//  - P: the softmax warps arrive on a barrier of their own CTA; the odd CTA's
//    helper forwards its CTA's P once per key tile.
// Roles (256 threads):
//   warp 0       K producer of this CTA: its two query tiles, then per
//                visited key tile its halves of k_nope lo / hi and k_pe (64
//                keys; three 8 KB blocks) into a 9-block ring;
//   warp 1       tensor-memory allocation for the pair; in the even CTA, the
//                MMA-issuing thread;
//   warp 2       odd CTA only: the helper forwarding query and P readiness;
//   warp 3       V producer: per visited key tile V of all 128 keys for this
//                CTA's 64 value dims (two 8 KB blocks) into a 6-block ring.
//                K and V have rings and producers of their own because their
//                slots free up at different times (a K block after its S
//                product, a V block only after its PV product, a softmax
//                later): one ring filled in order would hold the K blocks of
//                tile j+3 behind the V blocks of tile j+2, and so behind
//                PV_{j-1};
//   warps 4..7   softmax of this CTA's 128 rows (one row per thread) and the
//                epilogue O / l -> bf16 -> out of each item.
// Tensor memory (512 columns, allocated for the pair): S buffers at columns
// 0, 128 and 256, O at 384.
//
// Teardown: after a first cluster barrier no CTA issues another copy; the
// even CTA then makes the last phase of every slot of both rings complete (arming, or
// completing with mbarrier.complete_tx, the bytes of a copy that only one of
// the two CTAs issued before an abort) and waits for it, so no copy is in
// flight toward either CTA; a second cluster barrier precedes the release of
// tensor memory and the exit.
constexpr int kThreadsPair = 256;
constexpr uint32_t kHalfBlock = 64 * 64 * 2;  // 64 rows x 64 bf16, 128-byte swizzle: 8 KB
constexpr int kKRing = 9;                      // K blocks: three key tiles
constexpr int kVRing = 6;                      // V blocks: three key tiles
constexpr int kKPerTile = 3, kVPerTile = 2;
constexpr int kSBufs = 3;                      // score buffers in tensor memory
constexpr uint32_t kOffKRing = 2 * kQBytes;    // after the two query tiles (96 KB)
constexpr uint32_t kOffVRing = kOffKRing + kKRing * kHalfBlock;
constexpr uint32_t kSmemPairUsed = kOffVRing + kVRing * kHalfBlock;
constexpr size_t kSmemPairBytes = kSmemPairUsed + 1024;
constexpr uint32_t kColOPair = 384;
constexpr uint16_t kPairMask = 0x3;  // both CTAs of the cluster
static_assert(kSmemPairBytes <= 227 * 1024, "shared memory budget");

// The items of a cluster and the tiles each visits.
template <bool kMasked>
struct PairItems {
  int n_items;
  int pair[2];
  PairTiles<kMasked> tiles[2];
  int n_visit[2];
  __device__ __forceinline__ int total() const { return n_visit[0] + (n_items > 1 ? n_visit[1] : 0); }
};

template <bool kMasked, bool kRope>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsPair, 1)
    mla_attn_prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQn,
                                 const __grid_constant__ CUtensorMap tmQp,
                                 const __grid_constant__ CUtensorMap tmKn,
                                 const __grid_constant__ CUtensorMap tmKp,
                                 const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[2];   // this CTA's query tile of item i landed
  __shared__ uint64_t q_rot[2];    // its rotary part is rotated (4 softmax warps)
  __shared__ uint64_t q_peer[2];   // even CTA: the odd CTA's query tile of item i is ready
  __shared__ uint64_t k_full[kKRing];   // even CTA: both CTAs' halves of a K block landed
  __shared__ uint64_t k_empty[kKRing];  // this CTA's K slot is free again
  __shared__ uint64_t v_full[kVRing];   // even CTA: both CTAs' halves of a V block landed
  __shared__ uint64_t v_empty[kVRing];
  __shared__ uint64_t s_full[kSBufs];  // S buffer b holds the next scores
  __shared__ uint64_t p_full[kSBufs];  // even CTA: P in buffer b is complete (4 warps + helper);
                                       // odd CTA: its 4 softmax warps wrote their P
  __shared__ uint64_t pv_done[kSBufs];  // PV of the tile whose P was in buffer b landed
                                        // (per buffer: a waiter is never two phases behind)
  __shared__ uint64_t o_final;     // one phase per item: its last PV product has landed
  __shared__ uint64_t drain_bar;
  __shared__ uint64_t never_bar;   // no thread ever arrives (failure-detection test)
  __shared__ uint32_t n_issued[2];  // K and V blocks this CTA's producers issued
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  // cluster -> (b, h, item pair): groups of kHeadGroup heads; within a group
  // the clusters of the longest item first
  const int n_cl = (args.n_pairs + 1) / 2;  // clusters per (b, h)
  const int cid = int(blockIdx.x >> 1);
  const int per_group = kHeadGroup * n_cl;
  const int grp = cid / per_group;
  const int rem = cid - grp * per_group;
  const int b = grp / (kH / kHeadGroup);
  const int h = (grp % (kH / kHeadGroup)) * kHeadGroup + rem % kHeadGroup;
  const int ci = rem / kHeadGroup;
  const int bh = b * kH + h;
  const int n_keys =
      (!kMasked && args.valid_len) ? min(max(args.valid_len[b], 0), args.T) : args.T;

  PairItems<kMasked> items;
  items.pair[0] = args.n_pairs - 1 - ci;
  items.pair[1] = ci;
  items.n_items = items.pair[1] < items.pair[0] ? 2 : 1;
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    PairTiles<kMasked>& t = items.tiles[it];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      t.qt[i] = 2 * items.pair[it] + i;
      t.exists[i] = it < items.n_items && t.qt[i] < args.n_qt;
      t.cls[i] = (kMasked && args.tile_class && t.exists[i])
                     ? args.tile_class + (size_t(b) * args.n_qt + t.qt[i]) * args.n_kv
                     : nullptr;
    }
    t.kv_end = (n_keys + kBKV - 1) / kBKV;
    t.end = kMasked ? args.n_kv : min(min(2 * items.pair[it] + 2, args.n_qt), t.kv_end);
    int nv = 0;
    if (it < items.n_items)
      for (int kt = t.first(); kt < t.end; kt = t.next(kt)) ++nv;
    items.n_visit[it] = nv;
  }
  const int n_total = items.total();

  WaitCtl ctl{&abort_flag, args.wait_limit_ns, kErrKernelAttn, args.err_word};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    n_issued[0] = 0;
    n_issued[1] = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_rot[i], 4);
      mbar_init(&q_peer[i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], leader ? 5 : 4);
      mbar_init(&pv_done[i], 1);
    }
    for (int s = 0; s < kKRing; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVRing; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&o_final, 1);
    mbar_init(&drain_bar, 1);
    mbar_init(&never_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  __syncwarp();  // the .aligned cluster barrier wants converged warps
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: the query tiles and the K blocks; warp 3: the V blocks
    if (lane == 0 && n_total > 0) {
      const bool kprod = warp == 0;
      uint32_t q_issued = 0;
      if (kprod) {
        prefetch_tensormap(&tmQn);
        prefetch_tensormap(&tmQp);
        prefetch_tensormap(&tmKn);
        prefetch_tensormap(&tmKp);
        for (int it = 0; it < items.n_items; ++it) {
          if (items.n_visit[it] == 0) continue;
          const int q0 = items.tiles[it].qt[rank] * kBQ;
          uint8_t* sQ = smem + it * kQBytes;
          mbar_arrive_expect_tx(&q_full[it], kQBytes);
          tma_load_3d(sQ, &tmQn, &q_full[it], 0, q0, bh);
          tma_load_3d(sQ + kBlock, &tmQn, &q_full[it], 64, q0, bh);
          tma_load_3d(sQ + 2 * kBlock, &tmQp, &q_full[it], 0, q0, bh);
          q_issued |= 1u << it;
        }
      } else {
        prefetch_tensormap(&tmV);
      }
      const int kh = int(rank) * 64;  // this CTA's keys of a tile / its value dims
      const int per_tile = kprod ? kKPerTile : kVPerTile;
      const uint32_t ring = kprod ? kKRing : kVRing;
      uint64_t* full = kprod ? k_full : v_full;
      uint64_t* empty = kprod ? k_empty : v_empty;
      uint8_t* ring0 = smem + (kprod ? kOffKRing : kOffVRing);
      auto prefetch_tile = [&](int pt) {
        const int p0 = pt * kBKV;
        if (kprod) {
          tma_prefetch_l2_3d(&tmKn, 0, p0 + kh, bh);
          tma_prefetch_l2_3d(&tmKn, 64, p0 + kh, bh);
          tma_prefetch_l2_3d(&tmKp, 0, p0 + kh, b);
        } else {
          tma_prefetch_l2_3d(&tmV, kh, p0, bh);
          tma_prefetch_l2_3d(&tmV, kh, p0 + 64, bh);
        }
      };
      uint32_t s = 0;
      bool ok = true;
      for (int it = 0; ok && it < items.n_items; ++it) {
        const PairTiles<kMasked>& t = items.tiles[it];
        int pf = t.next(t.first());
        if (pf < t.end) prefetch_tile(pf);
        for (int kt = t.first(); ok && kt < t.end; kt = t.next(kt)) {
          const int k0 = kt * kBKV;
          if (pf < t.end) {
            pf = t.next(pf);
            if (pf < t.end) prefetch_tile(pf);
          }
#pragma unroll 1
          for (int i = 0; i < per_tile; ++i, ++s) {
            const uint32_t slot = s % ring;
            const uint32_t par = (s / ring) & 1u;
            if (!mbar_wait(&empty[slot], par ^ 1u, ctl, 1)) { ok = false; break; }
            uint8_t* dst = ring0 + slot * kHalfBlock;
            // both CTAs' copies of this block complete on the even CTA's barrier
            if (leader) mbar_arrive_expect_tx(&full[slot], 2 * kHalfBlock);
            const uint32_t fb = mapa_shared(smem_u32(&full[slot]), 0);
            if (kprod) {
              if (i < 2) tma_load_3d_pair(dst, &tmKn, fb, 64 * i, k0 + kh, bh);
              else tma_load_3d_pair(dst, &tmKp, fb, 0, k0 + kh, b);
            } else {
              tma_load_3d_pair(dst, &tmV, fb, kh, k0 + 64 * i, bh);
            }
            n_issued[kprod ? 0 : 1] = s + 1;
          }
        }
      }
      // the query copies complete on this CTA's own barriers: drain them here
      int zero = 0;
      WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
      if (!ok)
        for (int it = 0; it < 2; ++it)
          if (q_issued & (1u << it)) mbar_wait(&q_full[it], 0, drain, 2);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader && n_total > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(2 * kBQ, kBKV, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(2 * kBQ, kDV, false, true);
      const uint32_t kring0 = smem_u32(smem + kOffKRing);
      const uint32_t vring0 = smem_u32(smem + kOffVRing);
      const uint32_t o_tmem = tmem_base + kColOPair;
      const int n0 = items.n_visit[0];  // the first item's tiles come first
      bool ok = true;
      bool issued_any = false;
      uint32_t q_ready = 0;
      auto k_addr = [&](uint32_t seq) { return kring0 + (seq % kKRing) * kHalfBlock; };
      auto v_addr = [&](uint32_t seq) { return vring0 + (seq % kVRing) * kHalfBlock; };
      auto wait_k = [&](uint32_t seq) -> bool {
        return mbar_wait(&k_full[seq % kKRing], (seq / kKRing) & 1u, ctl, 13);
      };
      auto wait_v = [&](uint32_t seq) -> bool {
        return mbar_wait(&v_full[seq % kVRing], (seq / kVRing) & 1u, ctl, 12);
      };
      auto issue_s = [&](int j) -> bool {
        const int it = j < n0 ? 0 : 1;
        if (!(q_ready & (1u << it))) {
          // both CTAs' query tiles of this item are in shared memory (rotated)
          if (!mbar_wait(&q_full[it], 0, ctl, 10) ||
              !mbar_wait_cluster_sleep(&q_peer[it], 0, ctl, 10))
            return false;
          if (kRope && !mbar_wait(&q_rot[it], 0, ctl, 16)) return false;
          q_ready |= 1u << it;
        }
        const uint32_t base = uint32_t(j) * kKPerTile;
        if (!wait_k(base) || !wait_k(base + 1) || !wait_k(base + 2)) return false;
        tc_fence_after();
        const uint32_t sQ = smem_u32(smem + it * kQBytes);
        const uint32_t s_tmem = tmem_base + 128u * uint32_t(j % kSBufs);
#pragma unroll
        for (int blk = 0; blk < 3; ++blk) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t qd = sdesc_sw128(sQ + blk * kBlock + kk * 32, 16, 1024);
            const uint64_t kd = sdesc_sw128(k_addr(base + blk) + kk * 32, 16, 1024);
            mma_ss_pair(s_tmem, qd, kd, idesc_s, (blk | kk) != 0 ? 1u : 0u);
          }
        }
        issued_any = true;
        mma_commit_pair_mc(&s_full[j % kSBufs], kPairMask);
        for (uint32_t i = 0; i < uint32_t(kKPerTile); ++i)
          mma_commit_pair_mc(&k_empty[(base + i) % kKRing], kPairMask);
        return true;
      };
      for (int j = 0; ok && j < min(n_total, kSBufs); ++j) ok = issue_s(j);
      for (int j = 0; ok && j < n_total; ++j) {
        const int it = j < n0 ? 0 : 1;
        const int first = it == 0 ? 0 : n0;  // the item's first tile overwrites O
        const uint32_t vbase = uint32_t(j) * kVPerTile;
        // (acquire at cluster scope: the odd CTA's P is forwarded by a remote arrive)
        if (!mbar_wait_cluster_sleep(&p_full[j % kSBufs], uint32_t(j / kSBufs) & 1u, ctl, 11) ||
            !wait_v(vbase) || !wait_v(vbase + 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // P_j: 128 keys as 64 packed columns of its S buffer; V: each CTA's 64
        // value dims of 64 keys per block, MN-major, 8-key groups 1 KB apart.
        const uint32_t p_tmem = tmem_base + 128u * uint32_t(j % kSBufs);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t vb = v_addr(vbase + half);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (j > first || half > 0 || kk > 0) ? 1u : 0u;
            const uint64_t vd = sdesc_sw128(vb + kk * 16 * 128, kHalfBlock, 1024);
            mma_ts_pair(o_tmem, p_tmem + (half * 4 + kk) * 8, vd, idesc_o, acc);
          }
        }
        mma_commit_pair_mc(&pv_done[j % kSBufs], kPairMask);
        if (j == first + items.n_visit[it] - 1) mma_commit_pair_mc(&o_final, kPairMask);
        mma_commit_pair_mc(&v_empty[vbase % kVRing], kPairMask);
        mma_commit_pair_mc(&v_empty[(vbase + 1) % kVRing], kPairMask);
        if (j + kSBufs < n_total && !issue_s(j + kSBufs)) { ok = false; break; }
      }
      if (!ok && issued_any) {
        mma_commit_pair_mc(&drain_bar, 0x1);
        int zero = 0;
        WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
        mbar_wait(&drain_bar, 0, drain, 14);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ helper (odd CTA)
    if (lane == 0 && !leader && n_total > 0) {
      bool ok = true;
      for (int it = 0; ok && it < items.n_items; ++it) {
        if (items.n_visit[it] == 0) continue;
        ok = mbar_wait(&q_full[it], 0, ctl, 17);
        if (kRope && ok) ok = mbar_wait(&q_rot[it], 0, ctl, 17);
        if (ok) mbar_arrive_cluster(mapa_shared(smem_u32(&q_peer[it]), 0));
      }
      for (int j = 0; ok && j < n_total; ++j) {
        if (!mbar_wait(&p_full[j % kSBufs], uint32_t(j / kSBufs) & 1u, ctl, 18)) break;
        mbar_arrive_cluster(mapa_shared(smem_u32(&p_full[j % kSBufs]), 0));
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_base = tmem_addr(tmem_base, quad * 32, 0);
    bool ok = true;
    if (kRope) {
      // rotate this row's q_pe in shared memory, for each item (see the
      // one-SM kernel)
      for (int it = 0; it < items.n_items; ++it) {
        if (items.n_visit[it] == 0) continue;
        const int q = items.tiles[it].qt[rank] * kBQ + r;
        if (ok) ok = mbar_wait(&q_full[it], 0, ctl, 24);
        if (ok && items.tiles[it].exists[rank] && q < args.T) {
          uint8_t* rowp = smem + it * kQBytes + 2 * kBlock + r * 128;
          const float4* cs =
              reinterpret_cast<const float4*>(args.rope_cs + (size_t(b) * args.T + q) * 32);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* chunk = reinterpret_cast<uint4*>(rowp + ((c ^ (r & 7)) << 4));
            uint4 w = *chunk;
            const float4 a = __ldg(cs + 2 * c), bq = __ldg(cs + 2 * c + 1);
            const float csn[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = bf16_bits_to_float(wp[e] & 0xffffu);
              const float x1 = bf16_bits_to_float(wp[e] >> 16);
              const float cc = csn[2 * e], ss = csn[2 * e + 1];
              wp[e] = pack_bf16x2(fmaf(x0, cc, -x1 * ss), fmaf(x1, cc, x0 * ss));
            }
            *chunk = w;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_rot[it]);
      }
    }

    int j = 0;  // visited key tiles so far (the pair's sequence, over both items)
    for (int it = 0; it < items.n_items; ++it) {
      const PairTiles<kMasked>& tiles = items.tiles[it];
      const int qt_me = tiles.qt[rank];
      const int q = qt_me * kBQ + r;
      const bool row_valid = tiles.exists[rank] && q < args.T;
      const __nv_bfloat16* mrow =
          (kMasked && row_valid) ? args.mask + (size_t(b) * args.T + q) * args.mask_ld : nullptr;
      float m = -INFINITY;  // running max, log2 units
      float l = 0.f;        // running sum of p (fp32, unrounded)
      uint32_t n = 0;       // key tiles used by this row's tile so far
      for (int kt = tiles.first(); ok && kt < tiles.end; kt = tiles.next(kt), ++j) {
        const int buf = j % kSBufs;
        const uint32_t colS = 128u * uint32_t(buf);
        const int k0 = kt * kBKV;
        if (args.test_stall && rank == 0 && blockIdx.x == 0 &&
            !mbar_wait_warp(&never_bar, 0, ctl, 30)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(&s_full[buf], uint32_t(j / kSBufs) & 1u, ctl, 20)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (!tiles.active(int(rank), kt)) {
          // No key of this tile is allowed for this CTA's rows (causal: the
          // odd CTA's diagonal tile seen from the even CTA; a mask: a skipped
          // tile): P = 0 for the pair's PV.
          uint32_t z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = 0u;
          tmem_st32(lane_base + colS, z);
          tmem_st32(lane_base + colS + 32, z);
        } else {
          // as in the one-SM kernel: the fast route for tiles that need no
          // mask entries added (every causal tile; all-zero, causal-pattern
          // and prefix tiles of a mask) with a per-row key limit, the exact
          // two-pass route for the others and for a non-positive scale
          const uint8_t tile_cls = kMasked ? (tiles.cls[rank] ? tiles.cls[rank][kt]
                                                              : uint8_t(kTileMixed))
                                           : uint8_t(kTileZero);
          ScoreChunk<kMasked> sc;
          sc.cls = (kMasked && row_valid) ? tile_cls : uint8_t(kTileZero);
          sc.row_valid = row_valid;
          sc.mrow = mrow + (kMasked && row_valid ? k0 : 0);
          sc.kvalid = args.T - k0;
          sc.mask_vec = args.mask_vec;
          const bool causal_tile = !kMasked ? kt == qt_me : tile_cls == kTileCausal;
          const bool prefix_tile = kMasked && tile_cls >= kTilePrefix;
          const bool fast_route =
              (tile_cls == kTileZero || tile_cls == kTileCausal || prefix_tile) &&
              args.scale_log2 > 0.f;
          const int key_end = kMasked ? args.T : n_keys;
          const bool diag = causal_tile || prefix_tile || key_end - k0 < kBKV;
          const int lim =
              min(causal_tile ? r : (prefix_tile ? int(tile_cls) - kTilePrefix : kBKV - 1),
                  key_end - 1 - k0);
          sc.diag_row = (kMasked ? (causal_tile || prefix_tile) : diag) ? lim : kBKV;
          uint32_t raw[kBKV];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(lane_base + colS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(raw + c * 32));
          tmem_ld_wait();
          reg_fence(raw);
          float alpha = 1.f;
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          bool exact = !(fast_route && n > 0);
          float rowsum = 0.f;
          if (!exact) {
#pragma unroll
            for (int c2 = 0; c2 < 4; c2 += 2) {
              uint32_t pk[32];
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t(&ph)[16] = *reinterpret_cast<uint32_t(*)[16]>(pk + 16 * h2);
                if (diag)
                  p_chunk_causal<true>(raw + (c2 + h2) * 32, c2 + h2, lim, args.scale_log2, m,
                                       ph, acc);
                else
                  p_chunk_causal<false>(raw + (c2 + h2) * 32, c2 + h2, r, args.scale_log2, m,
                                        ph, acc);
              }
              tmem_st32(lane_base + colS + 16 * c2, pk);
            }
            rowsum =
                ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
            if (__any_sync(0xffffffffu, !(rowsum <= 256.f))) {
              const float mt = (diag ? raw_row_max<true>(raw, lim) : raw_row_max<false>(raw, r)) *
                               args.scale_log2;
              exact = __any_sync(0xffffffffu, !(mt <= m + kRescaleThreshold));
              if (exact) {
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = 0.f;
              }
            }
          }
          if (exact) {
            float mt;
            if (fast_route) {
              mt = diag ? raw_row_max<true>(raw, lim) : raw_row_max<false>(raw, r);
              mt *= args.scale_log2;
            } else {
              float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                float x[32];
                sc.apply(raw + c * 32, c, args.scale_log2, 0.f, x);
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                  m4[0] = fmax3(m4[0], x[i], x[i + 1]);
                  m4[1] = fmax3(m4[1], x[i + 2], x[i + 3]);
                  m4[2] = fmax3(m4[2], x[i + 4], x[i + 5]);
                  m4[3] = fmax3(m4[3], x[i + 6], x[i + 7]);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) raw[c * 32 + i] = __float_as_uint(x[i]);
              }
              mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            }
            float m_new = m;
            if (n == 0) {
              m_new = mt;
            } else if (mt > m + kRescaleThreshold) {
              m_new = mt;
              alpha = fast_exp2(m - m_new);
            }
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            m = m_new;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint32_t* rc = raw + c * 32;
              uint32_t pk[16];
              if (fast_route) {
                if (diag)
                  p_chunk_causal<true>(rc, c, lim, args.scale_log2, m_use, pk, acc);
                else
                  p_chunk_causal<false>(rc, c, r, args.scale_log2, m_use, pk, acc);
              } else {
                float x[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(rc[i]) - m_use;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float p0 = fast_exp2(x[2 * i]);
                  const float p1 = fast_exp2(x[2 * i + 1]);
                  fadd2(acc[2 * (i & 3)], acc[2 * (i & 3) + 1], acc[2 * (i & 3)],
                        acc[2 * (i & 3) + 1], p0, p1);
                  pk[i] = pack_bf16x2(p0, p1);
                }
              }
              tmem_st16(lane_base + colS + 16 * c, pk);
            }
            rowsum =
                ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
            // Rescale O once PV_{j-1} (the last product issued before this
            // tile's, into this item's O since n > 0) has landed; PV_j waits
            // for this tile's P below.
            if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
              if (!mbar_wait_warp(&pv_done[(j - 1) % kSBufs], uint32_t((j - 1) / kSBufs) & 1u,
                                  ctl, 21)) {
                ok = false;
              } else {
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                  uint32_t rr[32];
                  tmem_ld32(lane_base + kColOPair + c * 32, rr);
                  tmem_ld_wait();
                  reg_fence(rr);
#pragma unroll
                  for (int i = 0; i < 32; ++i)
                    rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
                  tmem_st32(lane_base + kColOPair + c * 32, rr);
                }
              }
            }
          }  // exact
          l = l * alpha + rowsum;
          ++n;
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[buf]);  // own CTA; the helper forwards the odd CTA's
      }
      if (!ok) break;

      // epilogue of this item: O / l -> bf16 -> out[b, q, h*128 + e]. Every
      // softmax thread waits for the item's last product (so no MMA is in
      // flight at teardown) and reads O before it writes the next item's
      // first P (whose PV overwrites O).
      const bool have = items.n_visit[it] > 0 && mbar_wait_warp(&o_final, uint32_t(it) & 1u, ctl, 22);
      if (items.n_visit[it] > 0 && !have) {
        ok = false;
        break;
      }
      if (have) tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = args.out + (size_t(b) * args.T + q) * size_t(kH * kDV) + h * kDV;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        if (n > 0) {
          tmem_ld32(lane_base + kColOPair + c * 32, rr);
          tmem_ld_wait();
          reg_fence(rr);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = 0u;
        }
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * inv_l,
                                  __uint_as_float(rr[2 * i + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                packed[4 * i + 3]);
        }
      }
      tc_fence_before();
    }
  }

  // Teardown, first barrier: from here on neither CTA issues a copy.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (leader && (warp == 0 || warp == 3) && lane == 0 && n_total > 0) {
    // Every ring copy completes on this CTA's barriers (warp 0: the K ring,
    // warp 3: the V ring). Account for a block that only one CTA issued
    // (possible only after an abort), then wait for the last phase of every
    // slot; each slot has at most one phase pending.
    const int which = warp == 0 ? 0 : 1;
    uint64_t* full = which == 0 ? k_full : v_full;
    const uint32_t ring = which == 0 ? kKRing : kVRing;
    const uint32_t n_own = n_issued[which];
    const uint32_t n_peer = ld_shared_cluster_u32(mapa_shared(smem_u32(&n_issued[which]), 1));
    const uint32_t lo = min(n_own, n_peer), hi = max(n_own, n_peer);
    for (uint32_t seq = lo; seq < hi; ++seq) {
      uint64_t* fb = &full[seq % ring];
      if (seq < n_own)  // armed for both CTAs' bytes, the odd CTA's copy never came
        mbar_complete_tx_cluster(mapa_shared(smem_u32(fb), 0), kHalfBlock);
      else              // the odd CTA's copy came, this CTA never armed the phase
        mbar_arrive_expect_tx(fb, kHalfBlock);
    }
    int zero = 0;
    WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
    const uint32_t first = hi > ring ? hi - ring : 0;
    for (uint32_t seq = first; seq < hi; ++seq)
      mbar_wait(&full[seq % ring], (seq / ring) & 1u, drain, 3);
  }
  // Second barrier: no copy is in flight toward either CTA; neither leaves,
  // nor frees the pair's tensor memory, before both get here.
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- classifier
// One pass over the additive mask: each 128x128 (query, key) tile, clipped to
// T, becomes kTileSkip (every entry -inf), kTileZero (every entry +-0),
// kTileCausal (the causal pattern on a diagonal tile), kTilePrefix + L (every
// row +-0 on keys 0..L, -inf after) or kTileMixed. One CTA per tile, 256
// threads, 16-byte loads when the rows are 16-byte aligned (vec != 0),
// element loads otherwise.
__global__ void __launch_bounds__(256)
    mask_tile_classify_kernel(const __nv_bfloat16* __restrict__ mask, int64_t mask_ld, int vec,
                              int T, int n_qt, int n_kv, uint8_t* __restrict__ cls) {
  const int kt = blockIdx.x, qt = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kBQ, k0 = kt * kBKV;
  const int rows = min(kBQ, T - q0);
  const int cols = min(kBKV, T - k0);
  const uint16_t* base =
      reinterpret_cast<const uint16_t*>(mask) + (size_t(b) * T + q0) * mask_ld + k0;
  bool all_ninf = true, all_zero = true;
  bool all_causal = kt == qt;  // diagonal tile: +-0 where key <= query, -inf above
  // prefix pattern: every entry +-0 or -inf, the last +-0 column before the
  // first -inf column in every row
  bool zero_or_ninf = true;
  int max_zero_col = -1, min_ninf_col = kBKV;
  __shared__ int s_max_zero, s_min_ninf;
  if (threadIdx.x == 0) {
    s_max_zero = -1;
    s_min_ninf = kBKV;
  }
  auto track = [&](uint32_t v, int c) {
    if ((v & 0x7fffu) == 0u) max_zero_col = max(max_zero_col, c);
    else if (v == 0xff80u) min_ninf_col = min(min_ninf_col, c);
    else zero_or_ninf = false;
  };
  auto causal_ok = [](uint32_t v, int rr, int c) {
    return c <= rr ? (v & 0x7fffu) == 0u : v == 0xff80u;
  };
  if (vec && cols == kBKV) {
    // 16 uint4 per row
    for (int idx = threadIdx.x; idx < rows * 16; idx += blockDim.x) {
      const int rr = idx >> 4, c8 = idx & 15;
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(base + size_t(rr) * mask_ld) + c8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = ws[e] & 0xffffu, hi = ws[e] >> 16;
        all_ninf &= (lo == 0xff80u) && (hi == 0xff80u);
        all_zero &= ((lo & 0x7fffu) == 0u) && ((hi & 0x7fffu) == 0u);
        all_causal &= causal_ok(lo, rr, c8 * 8 + 2 * e) && causal_ok(hi, rr, c8 * 8 + 2 * e + 1);
        track(lo, c8 * 8 + 2 * e);
        track(hi, c8 * 8 + 2 * e + 1);
      }
    }
  } else {
    for (int idx = threadIdx.x; idx < rows * cols; idx += blockDim.x) {
      const int rr = idx / cols, c = idx - rr * cols;
      const uint32_t v = base[size_t(rr) * mask_ld + c];
      all_ninf &= (v == 0xff80u);
      all_zero &= ((v & 0x7fffu) == 0u);
      all_causal &= causal_ok(v, rr, c);
      track(v, c);
    }
  }
  __syncthreads();  // s_max_zero / s_min_ninf initialised
  atomicMax(&s_max_zero, max_zero_col);
  atomicMin(&s_min_ninf, min_ninf_col);
  const int any_not_ninf = __syncthreads_or(!all_ninf);
  const int any_not_zero = __syncthreads_or(!all_zero);
  const int any_not_causal = __syncthreads_or(!all_causal);
  const int any_other = __syncthreads_or(!zero_or_ninf);  // also orders the atomics
  if (threadIdx.x == 0) {
    uint8_t c = kTileMixed;
    if (!any_not_ninf) c = kTileSkip;
    else if (!any_not_zero) c = kTileZero;
    else if (!any_not_causal) c = kTileCausal;
    else if (!any_other && s_max_zero >= 0 && s_max_zero + 1 == s_min_ninf &&
             s_max_zero <= kBKV - 2)
      c = uint8_t(kTilePrefix + s_max_zero);
    cls[(size_t(b) * n_qt + qt) * n_kv + kt] = c;
  }
}

// Which attention kernel runs (MLA_ATTN_KERNEL, read once): "pair" selects
// the CTA-pair kernel; "tile" the one-SM kernel with 128-key score tiles for
// every call; anything else the one-SM kernel with half-tile scores (under
// an explicit mask where the CTA's active key tiles allow it).
bool kernel_env_is(const char* name) {
  const char* s = std::getenv("MLA_ATTN_KERNEL");
  return s && std::strcmp(s, name) == 0;
}
bool pair_kernel_selected() {
  static const bool v = kernel_env_is("pair");
  return v;
}
bool tile_kernel_selected() {
  static const bool v = kernel_env_is("tile");
  return v;
}

// Half-tile PV products from their own issuing thread: for T >=
// kPvIssuerMinT, or as MLA_ATTN_PV_ISSUER (read once) says: "1" always,
// "0" never.
bool pv_issuer_for(int T) {
  static const int env = [] {
    const char* s = std::getenv("MLA_ATTN_PV_ISSUER");
    if (s && std::strcmp(s, "1") == 0) return 1;
    if (s && std::strcmp(s, "0") == 0) return 0;
    return -1;
  }();
  return env >= 0 ? env == 1 : T >= kPvIssuerMinT;
}

// Rows of the mask can be read with 16-byte loads.
bool mask_rows_vec_ok(const void* mask, int64_t mask_ld) {
  return (reinterpret_cast<uintptr_t>(mask) & 15u) == 0 && (mask_ld % 8) == 0;
}

// [outer][T][inner] bf16 tensor, boxes of 64 (inner) x box_rows (T) x 1.
bool make_map_3d(CUtensorMap* m, const void* p, int inner, int T, int outer,
                 uint32_t box_rows = kBQ) {
  const uint64_t dims[3] = {uint64_t(inner), uint64_t(T), uint64_t(outer)};
  const uint64_t strides[2] = {uint64_t(inner) * 2, uint64_t(inner) * 2 * uint64_t(T)};
  const uint32_t box[3] = {64, box_rows, 1};
  return encode_tmap_bf16(m, p, 3, dims, strides, box, true);
}

}  // namespace

size_t attn_class_bytes(int B, int T) {
  const size_t nt = size_t((T + kBQ - 1) / kBQ);
  return size_t(B) * nt * nt;
}

cudaError_t launch_mask_classify(const void* mask, int64_t mask_ld, int B, int T, void* cls,
                                 cudaStream_t stream) {
  const int nt = (T + kBQ - 1) / kBQ;
  dim3 grid(nt, nt, B);
  mask_tile_classify_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(mask), mask_ld, mask_rows_vec_ok(mask, mask_ld) ? 1 : 0,
      T, nt, nt, static_cast<uint8_t*>(cls));
  return cudaGetLastError();
}

cudaError_t launch_attn_prefill(const void* q_nope, const void* q_pe, const void* k_nope,
                                const void* k_pe, const void* v, const void* mask,
                                int64_t mask_ld, const void* tile_class, int B, int T,
                                float softmax_scale, void* out,
                                unsigned long long wait_limit_ns, unsigned int* err_word,
                                int test_stall, cudaStream_t stream, const int* valid_len,
                                const void* rope_cs) {
  if (mask && valid_len) return cudaErrorInvalidValue;
  CUtensorMap tmQn, tmQp, tmKn, tmKp, tmV;
  const int BH = B * kH;
  if (pair_kernel_selected()) {
    // CTA pairs: K maps with 64-key boxes (each CTA loads half the keys)
    if (!make_map_3d(&tmQn, q_nope, kDN, T, BH) || !make_map_3d(&tmQp, q_pe, kDR, T, BH) ||
        !make_map_3d(&tmKn, k_nope, kDN, T, BH, 64) || !make_map_3d(&tmKp, k_pe, kDR, T, B, 64) ||
        !make_map_3d(&tmV, v, kDV, T, BH, 64))
      return cudaErrorInvalidValue;
    auto kern = mask ? (rope_cs ? mla_attn_prefill_pair_kernel<true, true>
                                : mla_attn_prefill_pair_kernel<true, false>)
                     : (rope_cs ? mla_attn_prefill_pair_kernel<false, true>
                                : mla_attn_prefill_pair_kernel<false, false>);
    static ContextCache pair_attr[4];
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), int(kSmemPairBytes),
                                     &pair_attr[(mask ? 1 : 0) + (rope_cs ? 2 : 0)]);
    if (e != cudaSuccess) return e;
    AttnArgs a{};
    a.mask = static_cast<const __nv_bfloat16*>(mask);
    a.mask_ld = mask_ld;
    a.mask_vec = mask_rows_vec_ok(mask, mask_ld) ? 1 : 0;
    a.tile_class = static_cast<const uint8_t*>(tile_class);
    a.valid_len = valid_len;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.B = B;
    a.T = T;
    a.n_qt = (T + kBQ - 1) / kBQ;
    a.n_kv = a.n_qt;
    a.n_pairs = (a.n_qt + 1) / 2;
    a.scale_log2 = softmax_scale * kLog2e;
    a.wait_limit_ns = wait_limit_ns;
    a.err_word = err_word;
    a.test_stall = test_stall;
    a.rope_cs = static_cast<const float2*>(rope_cs);
    const long long ctas = 2LL * B * kH * ((a.n_pairs + 1) / 2);  // a cluster per two items
    if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
    kern<<<unsigned(ctas), kThreadsPair, kSmemPairBytes, stream>>>(tmQn, tmQp, tmKn, tmKp, tmV,
                                                                  a);
    return cudaGetLastError();
  }
  CUtensorMap tmOut;  // out [B, T, 64 * 128]: 64-dim x 128-row boxes
  if (!make_map_3d(&tmQn, q_nope, kDN, T, BH) || !make_map_3d(&tmQp, q_pe, kDR, T, BH) ||
      !make_map_3d(&tmKn, k_nope, kDN, T, BH) || !make_map_3d(&tmKp, k_pe, kDR, T, B) ||
      !make_map_3d(&tmV, v, kDV, T, BH, 64) || !make_map_3d(&tmOut, out, kH * kDV, T, B))
    return cudaErrorInvalidValue;
  // half-tile scores unless MLA_ATTN_KERNEL=tile (under an explicit mask the
  // kernel falls back to 128-key tiles per CTA where needed)
  const bool half = !tile_kernel_selected();
  const bool pv = half && pv_issuer_for(T);
  auto kern = pv ? (mask ? (rope_cs ? mla_attn_prefill_kernel<true, true, true, true>
                                    : mla_attn_prefill_kernel<true, false, true, true>)
                         : (rope_cs ? mla_attn_prefill_kernel<false, true, true, true>
                                    : mla_attn_prefill_kernel<false, false, true, true>))
              : half ? (mask ? (rope_cs ? mla_attn_prefill_kernel<true, true, true, false>
                                        : mla_attn_prefill_kernel<true, false, true, false>)
                             : (rope_cs ? mla_attn_prefill_kernel<false, true, true, false>
                                        : mla_attn_prefill_kernel<false, false, true, false>))
                     : (mask ? (rope_cs ? mla_attn_prefill_kernel<true, true, false, false>
                                        : mla_attn_prefill_kernel<true, false, false, false>)
                             : (rope_cs ? mla_attn_prefill_kernel<false, true, false, false>
                                        : mla_attn_prefill_kernel<false, false, false, false>));
  static ContextCache attr_done[16];  // index: mask + 2 rope + 4 half + 8 PV issuer
  cudaError_t e = ensure_smem_attr(
      reinterpret_cast<const void*>(kern), int(kSmemBytes),
      &attr_done[(mask ? 1 : 0) + (rope_cs ? 2 : 0) + (half ? 4 : 0) + (pv ? 8 : 0)]);
  if (e != cudaSuccess) return e;
  AttnArgs a;
  a.mask = static_cast<const __nv_bfloat16*>(mask);
  a.mask_ld = mask_ld;
  a.valid_len = valid_len;
  a.mask_vec = mask_rows_vec_ok(mask, mask_ld) ? 1 : 0;
  a.tile_class = static_cast<const uint8_t*>(tile_class);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.B = B;
  a.T = T;
  a.n_qt = (T + kBQ - 1) / kBQ;
  a.n_kv = a.n_qt;
  a.n_pairs = (a.n_qt + 1) / 2;
  a.scale_log2 = softmax_scale * kLog2e;
  a.wait_limit_ns = wait_limit_ns;
  a.err_word = err_word;
  a.test_stall = test_stall;
  a.rope_cs = static_cast<const float2*>(rope_cs);
  const long long ctas = (long long)B * kH * a.n_pairs;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
  kern<<<unsigned(ctas), kThreads, kSmemBytes, stream>>>(tmQn, tmQp, tmKn, tmKp, tmV, tmOut, a);
  return cudaGetLastError();
}

}  // namespace mla
