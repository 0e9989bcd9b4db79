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
//
// One CTA computes one (b, h, 128-row query tile); the longest causal tiles
// are scheduled first. Roles:
//   warp 0      TMA producer: the Q tile (nope + rope, 48 KB) once, then per
//               128-key tile the K tile (k_nope + the shared k_pe, 48 KB) and
//               the V tile (32 KB) into 2-deep rings;
//   warp 1      tensor-memory owner and MMA issuer:
//                 S_j = Q K_j^T     128x128, K = 128 (nope) + 64 (rope), SS
//                 O  += P_j V_j     128x128, K = 128 keys, P from TMEM (TS)
//               S is double-buffered so S_{j+1} runs while row softmax j does;
//   warps 2..5  one thread per query row: read S_j from TMEM, scale, mask,
//               online max (rescaling O only when the max grows by more than
//               2^8), exponentials, row sum, write P_j as bf16 back into the S
//               buffer, and at the end O / l -> bf16 -> out[b, i, h*128 ..].
// Tensor memory: S0 cols [0,128), S1 [128,256), O [256,384).
#include "attn_prefill.h"
#include "host_util.h"
#include "sm100.cuh"

namespace mla {

namespace {

constexpr int kBQ = 128;     // query rows per CTA
constexpr int kBKV = 128;    // keys per tile
constexpr int kDN = 128;     // qk_nope_head_dim
constexpr int kDR = 64;      // qk_rope_head_dim
constexpr int kDV = 128;     // v_head_dim
constexpr int kH = 64;       // heads
constexpr int kNSK = 2;      // K ring depth
constexpr int kNSV = 2;      // V ring depth
constexpr int kThreads = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t kBlock = kBQ * 64 * 2;      // one 128 x 64 bf16 swizzled block: 16 KB
constexpr uint32_t kQBytes = 3 * kBlock;       // nope lo, nope hi, rope
constexpr uint32_t kKBytes = 3 * kBlock;
constexpr uint32_t kVBytes = 2 * kBlock;       // value dims 0..63, 64..127
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQBytes;
constexpr uint32_t kOffV = kOffK + kNSK * kKBytes;
constexpr uint32_t kSmemUsed = kOffV + kNSV * kVBytes;
constexpr size_t kSmemBytes = kSmemUsed + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256;

static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

struct AttnArgs {
  const __nv_bfloat16* mask;   // [B,1,T,mask_ld] or null (causal)
  int64_t mask_ld;
  int mask_vec;                // rows 16-byte aligned: vector loads
  const uint8_t* tile_class;   // [B, n_qt, n_kv] or null
  __nv_bfloat16* out;          // [B, T, 64*128]
  int B, T, n_qt, n_kv;
  float scale_log2;            // softmax_scale * log2(e)
  unsigned long long wait_limit_ns;
  unsigned int* err_word;      // device status word
};

// Tiles of key blocks a query tile visits, in order. Causal: 0..qt. Explicit
// mask: every key tile whose class is not "all -inf" (all of them when no
// classification is given).
struct KvTiles {
  const uint8_t* cls;  // class row of this (b, qt), or null
  int end;             // one past the last candidate tile
  __device__ __forceinline__ int first() const { return next(-1); }
  __device__ __forceinline__ int next(int kt) const {
    ++kt;
    if (cls)
      while (kt < end && cls[kt] == kTileSkip) ++kt;
    return kt;
  }
  __device__ __forceinline__ int count() const {
    int n = 0;
    for (int kt = first(); kt < end; kt = next(kt)) ++n;
    return n;
  }
};

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

template <bool kMasked>
__global__ void __launch_bounds__(kThreads, 1)
    mla_attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQn,
                            const __grid_constant__ CUtensorMap tmQp,
                            const __grid_constant__ CUtensorMap tmKn,
                            const __grid_constant__ CUtensorMap tmKp,
                            const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full;
  __shared__ uint64_t k_full[kNSK], k_empty[kNSK];
  __shared__ uint64_t v_full[kNSV], v_empty[kNSV];
  __shared__ uint64_t s_full[2], p_full[2];
  __shared__ uint64_t o_done;
  __shared__ uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int b = blockIdx.y;
  const int qt = args.n_qt - 1 - int(blockIdx.z);  // longest causal tiles first
  const int q0 = qt * kBQ;
  const int bh = b * kH + h;

  KvTiles tiles;
  if (kMasked) {
    tiles.cls = args.tile_class ? args.tile_class + (size_t(b) * args.n_qt + qt) * args.n_kv
                                : nullptr;
    tiles.end = args.n_kv;
  } else {
    tiles.cls = nullptr;
    tiles.end = qt + 1;
  }
  const int n = tiles.count();

  WaitCtl ctl{&abort_flag, args.wait_limit_ns, kErrKernelAttn, args.err_word};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&q_full, 1);
    for (int s = 0; s < kNSK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kNSV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
    }
    mbar_init(&o_done, 1);
    mbar_init(&drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n > 0) {
      prefetch_tensormap(&tmQn);
      prefetch_tensormap(&tmQp);
      prefetch_tensormap(&tmKn);
      prefetch_tensormap(&tmKp);
      prefetch_tensormap(&tmV);
      uint8_t* sQ = smem + kOffQ;
      mbar_arrive_expect_tx(&q_full, kQBytes);
      tma_load_3d(sQ, &tmQn, &q_full, 0, q0, bh);
      tma_load_3d(sQ + kBlock, &tmQn, &q_full, 64, q0, bh);
      tma_load_3d(sQ + 2 * kBlock, &tmQp, &q_full, 0, q0, bh);
      uint32_t k_issued = 0, k_par = 0, v_issued = 0, v_par = 0;
      bool ok = true;
      int j = 0;
      for (int kt = tiles.first(); kt < tiles.end; kt = tiles.next(kt), ++j) {
        const int k0 = kt * kBKV;
        const int sk = j % kNSK;
        const uint32_t pk = (j / kNSK) & 1;
        if (!mbar_wait(&k_empty[sk], pk ^ 1u, ctl, 1)) { ok = false; break; }
        uint8_t* sK = smem + kOffK + sk * kKBytes;
        mbar_arrive_expect_tx(&k_full[sk], kKBytes);
        tma_load_3d(sK, &tmKn, &k_full[sk], 0, k0, bh);
        tma_load_3d(sK + kBlock, &tmKn, &k_full[sk], 64, k0, bh);
        tma_load_3d(sK + 2 * kBlock, &tmKp, &k_full[sk], 0, k0, b);
        k_issued |= 1u << sk;
        k_par = (k_par & ~(1u << sk)) | (pk << sk);

        const int sv = j % kNSV;
        const uint32_t pv = (j / kNSV) & 1;
        if (!mbar_wait(&v_empty[sv], pv ^ 1u, ctl, 2)) { ok = false; break; }
        uint8_t* sV = smem + kOffV + sv * kVBytes;
        mbar_arrive_expect_tx(&v_full[sv], kVBytes);
        tma_load_3d(sV, &tmV, &v_full[sv], 0, k0, bh);
        tma_load_3d(sV + kBlock, &tmV, &v_full[sv], 64, k0, bh);
        v_issued |= 1u << sv;
        v_par = (v_par & ~(1u << sv)) | (pv << sv);
      }
      if (!ok) {
        int zero = 0;
        WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
        mbar_wait(&q_full, 0, drain, 3);
        for (int s = 0; s < kNSK; ++s)
          if (k_issued & (1u << s)) mbar_wait(&k_full[s], (k_par >> s) & 1u, drain, 4);
        for (int s = 0; s < kNSV; ++s)
          if (v_issued & (1u << s)) mbar_wait(&v_full[s], (v_par >> s) & 1u, drain, 5);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBQ, kBKV, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBQ, kDV, false, true);
      const uint32_t sQ = smem_u32(smem + kOffQ);
      bool ok = mbar_wait(&q_full, 0, ctl, 10);
      bool issued_any = false;

      auto issue_pv = [&](int i) -> bool {
        const int sv = i % kNSV;
        const int pb = i & 1;
        if (!mbar_wait(&p_full[pb], (i >> 1) & 1, ctl, 11)) return false;
        if (!mbar_wait(&v_full[sv], (i / kNSV) & 1, ctl, 12)) return false;
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + kOffV + sv * kVBytes);
        const uint32_t p_tmem = tmem_base + kColS0 + pb * 128;
#pragma unroll
        for (int kk = 0; kk < kBKV / 16; ++kk) {
          // 16 keys = 8 packed TMEM columns of P; 16 V rows of 128 bytes.
          const uint64_t vd = sdesc_sw128(sV + kk * 16 * 128, kBlock, 1024);
          mma_ts(tmem_base + kColO, p_tmem + kk * 8, vd, idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&o_done);
        mma_commit(&v_empty[sv]);
        return true;
      };

      int j = 0;
      for (int kt = tiles.first(); ok && kt < tiles.end; kt = tiles.next(kt), ++j) {
        const int sk = j % kNSK;
        const int sb = j & 1;
        if (!mbar_wait(&k_full[sk], (j / kNSK) & 1, ctl, 13)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + kOffK + sk * kKBytes);
        const uint32_t s_tmem = tmem_base + kColS0 + sb * 128;
#pragma unroll
        for (int blk = 0; blk < 3; ++blk) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t qd = sdesc_sw128(sQ + blk * kBlock + kk * 32, 16, 1024);
            const uint64_t kd = sdesc_sw128(sK + blk * kBlock + kk * 32, 16, 1024);
            mma_ss(s_tmem, qd, kd, idesc_s, (blk | kk) != 0 ? 1u : 0u);
          }
        }
        issued_any = true;
        mma_commit(&s_full[sb]);
        mma_commit(&k_empty[sk]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && !issue_pv(n - 1)) ok = false;
      if (!ok && issued_any) {
        mma_commit(&drain_bar);
        int zero = 0;
        WaitCtl drain{&zero, args.wait_limit_ns, kErrKernelAttn, args.err_word};
        mbar_wait(&drain_bar, 0, drain, 14);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // row within the tile == TMEM lane
    const int q = q0 + r;
    const uint32_t lane_base = tmem_addr(tmem_base, quad * 32, 0);
    const bool row_valid = q < args.T;
    const __nv_bfloat16* mrow =
        (kMasked && row_valid) ? args.mask + (size_t(b) * args.T + q) * args.mask_ld : nullptr;

    float m = -INFINITY;  // running max, log2 units
    float l = 0.f;        // running sum of p (fp32, unrounded)
    bool ok = true;
    int j = 0;
    for (int kt = tiles.first(); kt < tiles.end; kt = tiles.next(kt), ++j) {
      const int sb = j & 1;
      const int k0 = kt * kBKV;
      if (!mbar_wait_warp(&s_full[sb], (j >> 1) & 1, ctl, 20)) { ok = false; break; }
      tc_fence_after();
      // scores in log2 units, with the explicit mask added chunk by chunk
      const uint8_t cls =
          (kMasked && row_valid) ? (tiles.cls ? tiles.cls[kt] : uint8_t(kTileMixed))
                                   : uint8_t(kTileZero);
      const int kvalid = args.T - k0;  // keys of this tile that exist
      // 8 keys per 16-byte load when the rows are 16-byte aligned; a chunk
      // that starts below T then lies inside the row (mask_ld >= T and
      // mask_ld % 8 == 0).
      const uint4* mv = reinterpret_cast<const uint4*>(mrow + k0);
      const int c8_last = (min(kvalid, kBKV) - 1) >> 3;
      float x[kBKV];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + kColS0 + sb * 128 + c * 32, rr);
        tmem_ld_wait();
        reg_fence(rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(rr[i]) * args.scale_log2;
        if (cls == kTileMixed) {
#pragma unroll
          for (int c8 = 4 * c; c8 < 4 * c + 4; ++c8) {
            // Chunks past the last key re-read the last existing chunk; their
            // keys are set to -inf below.
            const int c8c = min(c8, c8_last);
            uint32_t ws[4];
            if (args.mask_vec) {
              const uint4 w = ld_nc_v4_ordered(mv + c8c);
              ws[0] = w.x, ws[1] = w.y, ws[2] = w.z, ws[3] = w.w;
            } else {
              // rows not 16-byte aligned: element loads, clamped to the row
              const __nv_bfloat16* mc = mrow + k0;
              const int klast = min(kvalid, kBKV) - 1;
#pragma unroll
              for (int e = 0; e < 4; ++e)
                ws[e] = ld_nc_u16_ordered(mc + min(c8 * 8 + 2 * e, klast)) |
                        (ld_nc_u16_ordered(mc + min(c8 * 8 + 2 * e + 1, klast)) << 16);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              x[c8 * 8 + 2 * e] += bf16_bits_to_float(ws[e] & 0xffffu) * kLog2e;
              x[c8 * 8 + 2 * e + 1] += bf16_bits_to_float(ws[e] >> 16) * kLog2e;
            }
          }
        }
      }
      if (!kMasked) {
        if (kt == qt) {  // diagonal tile: key k0+c allowed iff c <= r
#pragma unroll
          for (int c = 0; c < kBKV; ++c)
            if (c > r) x[c] = -INFINITY;
        }
      } else if (!row_valid) {
#pragma unroll
        for (int c = 0; c < kBKV; ++c) x[c] = -INFINITY;
      } else if (kvalid < kBKV) {
#pragma unroll
        for (int c = 0; c < kBKV; ++c)
          if (c >= kvalid) x[c] = -INFINITY;
      }
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBKV; ++c) mt = fmaxf(mt, x[c]);
      float alpha = 1.f;
      float m_new = m;
      if (j == 0) {
        m_new = mt;
      } else if (mt > m + kRescaleThreshold) {
        m_new = mt;
        alpha = fast_exp2(m - m_new);
      }
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      m = m_new;

      if (j >= 1) {
        // O must hold P_{j-1} V_{j-1} before it is rescaled.
        if (!mbar_wait_warp(&o_done, (j - 1) & 1, ctl, 21)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t rr[32];
            tmem_ld32(lane_base + kColO + c * 32, rr);
            tmem_ld_wait();
            reg_fence(rr);
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st32(lane_base + kColO + c * 32, rr);
          }
        }
      }
      // P_j as bf16 pairs over the first 64 columns of its S buffer, written
      // 32 columns (64 keys) at a time.
      float rowsum = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = fast_exp2(x[64 * half + 2 * c] - m_use);
          const float p1 = fast_exp2(x[64 * half + 2 * c + 1] - m_use);
          rowsum += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        tmem_st32(lane_base + kColS0 + sb * 128 + 32 * half, pk);
      }
      l = l * alpha + rowsum;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }

    // epilogue: O / l -> bf16 -> out[b, q, h*128 + e]
    const bool have = ok && n > 0 && mbar_wait_warp(&o_done, (n - 1) & 1, ctl, 22);
    if (have) tc_fence_after();
    if (n == 0 || have) {
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = args.out + (size_t(b) * args.T + q) * size_t(kH * kDV) + h * kDV;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        if (n > 0) {
          tmem_ld32(lane_base + kColO + c * 32, rr);
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- classifier
// One pass over the additive mask: each 128x128 (query, key) tile, clipped to
// T, becomes kTileSkip (every entry -inf), kTileZero (every entry +-0) or
// kTileMixed. One CTA per tile, 256 threads, 16-byte loads when the rows are
// 16-byte aligned (vec != 0), element loads otherwise.
__global__ void __launch_bounds__(256)
    mask_tile_classify_kernel(const __nv_bfloat16* __restrict__ mask, int64_t mask_ld, int vec,
                              int T, int n_qt, int n_kv, uint8_t* __restrict__ cls) {
  const int kt = blockIdx.x, qt = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kBQ, k0 = kt * kBKV;
  const int rows = min(kBQ, T - q0);
  const int cols = min(kBKV, T - k0);
  const uint16_t* base = reinterpret_cast<const uint16_t*>(mask) + (size_t(b) * T + q0) * mask_ld + k0;
  bool all_ninf = true, all_zero = true;
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
      }
    }
  } else {
    for (int idx = threadIdx.x; idx < rows * cols; idx += blockDim.x) {
      const int rr = idx / cols, c = idx - rr * cols;
      const uint32_t v = base[size_t(rr) * mask_ld + c];
      all_ninf &= (v == 0xff80u);
      all_zero &= ((v & 0x7fffu) == 0u);
    }
  }
  const int any_not_ninf = __syncthreads_or(!all_ninf);
  const int any_not_zero = __syncthreads_or(!all_zero);
  if (threadIdx.x == 0) {
    uint8_t c = kTileMixed;
    if (!any_not_ninf) c = kTileSkip;
    else if (!any_not_zero) c = kTileZero;
    cls[(size_t(b) * n_qt + qt) * n_kv + kt] = c;
  }
}

// Rows of the mask can be read with 16-byte loads.
bool mask_rows_vec_ok(const void* mask, int64_t mask_ld) {
  return (reinterpret_cast<uintptr_t>(mask) & 15u) == 0 && (mask_ld % 8) == 0;
}

bool make_map_3d(CUtensorMap* m, const void* p, int inner, int T, int outer) {
  const uint64_t dims[3] = {uint64_t(inner), uint64_t(T), uint64_t(outer)};
  const uint64_t strides[2] = {uint64_t(inner) * 2, uint64_t(inner) * 2 * uint64_t(T)};
  const uint32_t box[3] = {64, kBQ, 1};
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
                                cudaStream_t stream) {
  CUtensorMap tmQn, tmQp, tmKn, tmKp, tmV;
  const int BH = B * kH;
  if (!make_map_3d(&tmQn, q_nope, kDN, T, BH) || !make_map_3d(&tmQp, q_pe, kDR, T, BH) ||
      !make_map_3d(&tmKn, k_nope, kDN, T, BH) || !make_map_3d(&tmKp, k_pe, kDR, T, B) ||
      !make_map_3d(&tmV, v, kDV, T, BH))
    return cudaErrorInvalidValue;
  auto kern = mask ? mla_attn_prefill_kernel<true> : mla_attn_prefill_kernel<false>;
  static unsigned attr_done[2] = {0, 0};
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), int(kSmemBytes),
                                   &attr_done[mask ? 1 : 0]);
  if (e != cudaSuccess) return e;
  AttnArgs a;
  a.mask = static_cast<const __nv_bfloat16*>(mask);
  a.mask_ld = mask_ld;
  a.mask_vec = mask_rows_vec_ok(mask, mask_ld) ? 1 : 0;
  a.tile_class = static_cast<const uint8_t*>(tile_class);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.B = B;
  a.T = T;
  a.n_qt = (T + kBQ - 1) / kBQ;
  a.n_kv = a.n_qt;
  a.scale_log2 = softmax_scale * kLog2e;
  a.wait_limit_ns = wait_limit_ns;
  a.err_word = err_word;
  dim3 grid(kH, B, a.n_qt);
  kern<<<grid, kThreads, kSmemBytes, stream>>>(tmQn, tmQp, tmKn, tmKp, tmV, a);
  return cudaGetLastError();
}

}  // namespace mla
