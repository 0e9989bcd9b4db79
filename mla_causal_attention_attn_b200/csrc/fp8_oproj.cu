// fp8_oproj.cu -- the output projection with 8-bit (e4m3) operands and block
// scales, the weight format of the checkpoint (page "Kimi K2 · Transformer
// blocks", configuration excerpt config.json, quantization_config:
// quant_method fp8, fmt e4m3, activation_scheme dynamic, weight_block_size
// [128, 128]).
//
// Format (the readings of those four fields):
//   * W_o [N, K] is stored as e4m3 codes with one fp32 scale per 128 x 128
//     block, w_scale [N/128][K/128], W_o ~= value(code) * scale;
//   * the activations are quantised at run time ("dynamic"), one scale per
//     token and per 128-wide group of input features, a_scale [K/128][M];
//   * a group's scale is amax / 448 (1 for a group of zeros) and each code is
//     the e4m3 value nearest to x / scale, both in fp32, saturating at 448.
// The product is out[m, n] = sum_g a_scale[g][m] * w_scale[n/128][g] *
// (sum over the group's 128 features of the decoded codes' products).
//
// Kernels:
//   * quant_rows_fp8_kernel: one half-warp per (token, group); bf16 in, codes
//     and the group's scale out (bound by HBM);
//   * quant_weight_fp8_kernel: one CTA per 128 x 128 weight block;
//   * oproj_fp8_kernel<BN>: persistent tcgen05 GEMM on 128 x BN output tiles
//     (BN = 128 or 256, one or two weight blocks wide). Each 128-wide K group
//     is one shared-memory stage (128 x 128 bytes of A, BN x 128 bytes of
//     W_o, 128-byte swizzle, K = 32 per kind::f8f6f4 MMA), and its four MMAs
//     write a fresh fp32 partial product into one of 512 / BN tensor-memory
//     buffers. Eight warps read each partial back, multiply it by the group's
//     two scales and add it into fp32 accumulators held in registers; the
//     partial buffer is released as soon as it has been read, so the MMAs of
//     the next groups run meanwhile.
//   Measured on B200 (M = 4096 and 16384, N = 7168, K = 8192): 256-wide
//   tiles ran 14-20 % faster than 128-wide ones (less shared-memory traffic
//   and half the MMA instructions per FLOP), with bit-identical results;
//   without the promotion step (a timing experiment only) the MMA and TMA
//   side alone reached 2.05-2.25 PFLOP/s, so the promotion is what bounds
//   the kernel.
#include "fp8_oproj.h"

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "../../include/mla.h"
#include "fp8_codes.cuh"
#include "host_util.h"
#include "sm100.cuh"

namespace mla {

namespace {

constexpr int kGroup = 128;        // quantisation group along K, and weight block edge

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---------------------------------------------------------------- quantisers
// x [M, K] bf16 (row stride ld elements) -> q [M, K] codes, scale [K/128][M].
// Items are (token, group) pairs, m = item / G, g = item % G; a half-warp
// takes one item, each of its 16 lanes 8 features (one 16-byte load, one
// 8-byte store), and every lane loads kQuantUnroll items before converting
// any, so enough loads are in flight to keep HBM busy.
constexpr int kQuantWarps = 8;
constexpr int kQuantUnroll = 4;
constexpr int64_t kQuantMaxBlocks = int64_t(1) << 20;

__global__ void __launch_bounds__(kQuantWarps * 32)
    quant_rows_fp8_kernel(const __nv_bfloat16* __restrict__ x, int64_t ld, int64_t M, int K,
                          uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int G = K / kGroup;
  const int64_t items = M * G;
  const int sub = (threadIdx.x >> 4) & 1;  // half-warp
  const int l16 = threadIdx.x & 15;
  // Half-warp `sub` of warp w takes items 2w + sub + k * per_iter. The loop
  // runs on the warp's first item, so both halves (and their shuffles) stay
  // converged; items past the end are skipped after the shuffles.
  const int64_t per_iter = int64_t(gridDim.x) * kQuantWarps * 2;
  const int64_t w2 = (int64_t(blockIdx.x) * kQuantWarps + (threadIdx.x >> 5)) * 2;
  for (int64_t base = w2; base < items; base += per_iter * kQuantUnroll) {
    uint4 raw[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t item = base + sub + u * per_iter;
      if (item < items) {
        const int64_t m = item / G;
        const int g = int(item - m * G);
        raw[u] = *reinterpret_cast<const uint4*>(x + size_t(m) * size_t(ld) + size_t(g) * kGroup +
                                                 l16 * 8);
      } else {
        raw[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t item = base + sub + u * per_iter;
      const uint32_t w4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      float v[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = bf16_lo(w4[e]);
        v[2 * e + 1] = bf16_hi(w4[e]);
      }
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
      // reduce over the 16 lanes of this half-warp (xor offsets below 16 stay inside it)
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (item < items) {
        const int64_t m = item / G;
        const int g = int(item - m * G);
        const float s = group_scale(amax);
        const uint32_t lo = e4m3_code(v[0], s) | (e4m3_code(v[1], s) << 8) |
                            (e4m3_code(v[2], s) << 16) | (e4m3_code(v[3], s) << 24);
        const uint32_t hi = e4m3_code(v[4], s) | (e4m3_code(v[5], s) << 8) |
                            (e4m3_code(v[6], s) << 16) | (e4m3_code(v[7], s) << 24);
        *reinterpret_cast<uint2*>(q + size_t(m) * K + size_t(g) * kGroup + l16 * 8) =
            make_uint2(lo, hi);
        if (l16 == 0) scale[size_t(g) * size_t(M) + size_t(m)] = s;
      }
    }
  }
}

// W [N, K] bf16 -> q [N, K] codes, scale [N/128][K/128]. CTA (kb, nb) takes
// one block; thread t holds 64 features of row t / 2 of the block.
__global__ void __launch_bounds__(256)
    quant_weight_fp8_kernel(const __nv_bfloat16* __restrict__ W, int N, int K,
                            uint8_t* __restrict__ q, float* __restrict__ scale) {
  __shared__ float warp_max[8];
  const int kb = blockIdx.x, nb = blockIdx.y;
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const size_t off = size_t(nb * kGroup + r) * size_t(K) + size_t(kb) * kGroup + half * 64;
  uint4 raw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) raw[i] = reinterpret_cast<const uint4*>(W + off)[i];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w4[e])), fabsf(bf16_hi(w4[e]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
  const float s = group_scale(amax);
  if (threadIdx.x == 0) scale[size_t(nb) * size_t(K / kGroup) + kb] = s;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint4 a = raw[2 * i + j];
      out[2 * j] = e4m3_code(bf16_lo(a.x), s) | (e4m3_code(bf16_hi(a.x), s) << 8) |
                   (e4m3_code(bf16_lo(a.y), s) << 16) | (e4m3_code(bf16_hi(a.y), s) << 24);
      out[2 * j + 1] = e4m3_code(bf16_lo(a.z), s) | (e4m3_code(bf16_hi(a.z), s) << 8) |
                       (e4m3_code(bf16_lo(a.w), s) << 16) | (e4m3_code(bf16_hi(a.w), s) << 24);
    }
    reinterpret_cast<uint4*>(q + off)[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// ---------------------------------------------------------------- GEMM
constexpr int kBM = 128;
// Warpgroup 0: TMA producer (warp 0), tensor-memory owner and MMA issuer
// (warp 1), two idle warps. Warpgroups 1 and 2: the promotion warps 4..11, two
// sets of four, BN/2 columns each. The roles are warpgroup-aligned so that
// setmaxnreg can move registers to the promotion warps (BN = 256 holds 128
// fp32 accumulators a thread): 128 x 72 + 256 x 216 = 384 x 168.
constexpr int kPromoWarps = 8;
constexpr int kThreads = 128 + 32 * kPromoWarps;
constexpr uint32_t kRegsCtl = 72;
constexpr uint32_t kRegsPromo = 216;
static_assert(128 * kRegsCtl + 32 * kPromoWarps * kRegsPromo <= kThreads * 168, "register split");
constexpr uint32_t kABytes = kBM * kGroup;
constexpr int kGroupM = 16;          // row blocks visited together (L2 reuse)
constexpr int kScaleAhead = 4;       // groups of scales loaded ahead
// The promotion loop walks the K groups kScaleAhead at a time, so the
// launcher needs K to be a multiple of kGroup * kScaleAhead; the o_proj
// width (8192 input features) is one.
static_assert(MLA_OPROJ_IN % (kGroup * kScaleAhead) == 0,
              "o_proj input width must be a multiple of the promotion step");

template <int BN>
struct Fp8Cfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kParts = 512 / BN;        // partial-product buffers in tensor memory
  static constexpr int kCols = BN / 2;           // columns of one promotion warp
  static constexpr int kChunk = BN == 256 ? 32 : 64;  // columns read per tensor-memory wait
  static constexpr uint32_t kBBytes = BN * kGroup;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = kParts * BN;
  static constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + 1024;
  static_assert(BN == 128 || BN == 256, "BN");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kTmemCols == 512, "TMEM columns must be a power of two <= 512");
};

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int& mb, int& nb) {
  const int group_tiles = kGroupM * n_tiles;
  const int group = tile / group_tiles;
  const int first_m = group * kGroupM;
  const int gm = min(kGroupM, m_tiles - first_m);
  const int in_group = tile - group * group_tiles;
  mb = first_m + in_group % gm;
  nb = in_group / gm;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    oproj_fp8_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, const float* __restrict__ a_scale,
                     const float* __restrict__ w_scale, __nv_bfloat16* __restrict__ C, int M,
                     int N, int K, unsigned long long wait_limit_ns, unsigned int* err_word) {
  using Cfg = Fp8Cfg<BN>;
  constexpr int kBN = BN, kStages = Cfg::kStages, kParts = Cfg::kParts;
  constexpr uint32_t kStageBytes = Cfg::kStageBytes, kTmemCols = Cfg::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[kStages];
  __shared__ uint64_t empty_bar[kStages];
  __shared__ uint64_t part_full[kParts];   // the MMAs of a group finished
  __shared__ uint64_t part_empty[kParts];  // the promotion warps have read it
  __shared__ uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + kBM - 1) / kBM;
  const int n_tiles = N / kBN;
  const int num_tiles = m_tiles * n_tiles;
  const int G = K / kGroup;

  WaitCtl ctl{&abort_flag, wait_limit_ns, kErrKernelOprojFp8, err_word};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int p = 0; p < kParts; ++p) {
      mbar_init(&part_full[p], 1);
      mbar_init(&part_empty[p], kPromoWarps);
    }
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

  if (warp < 4) {
  setmaxnreg_dec<kRegsCtl>();
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, m_tiles, n_tiles, mb, nb);
        for (int g = 0; g < G; ++g) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, ctl, 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + size_t(stage) * kStageBytes;
          mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
          tma_load_2d(sa, &tmA, &full_bar[stage], g * kGroup, mb * kBM);
          tma_load_2d(sa + kABytes, &tmB, &full_bar[stage], g * kGroup, nb * kBN);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA's memory goes away.
        int zero = 0;
        WaitCtl drain{&zero, wait_limit_ns, kErrKernelOprojFp8, err_word};
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) mbar_wait(&full_bar[s], (issued_par >> s) & 1u, drain, 2);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int part = 0;
      uint32_t part_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int g = 0; g < G; ++g) {
          if (!mbar_wait(&part_empty[part], part_phase ^ 1u, ctl, 3) ||
              !mbar_wait(&full_bar[stage], phase, ctl, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + size_t(stage) * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int kk = 0; kk < kGroup / 32; ++kk) {
            // 32 e4m3 = 32 bytes along K inside the 128-byte swizzled row
            const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_addr + kk * 32, 16, 1024);
            mma_ss_f8(tmem_base + uint32_t(part * kBN), ad, bd, idesc, kk != 0 ? 1u : 0u);
          }
          issued_any = true;
          mma_commit(&empty_bar[stage]);   // frees the stage once these MMAs finish
          mma_commit(&part_full[part]);    // the group's partial product is ready
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
          if (++part == kParts) {
            part = 0;
            part_phase ^= 1u;
          }
        }
      }
      if (!ok && issued_any) {
        // Wait for the MMAs in flight before the tensor memory is released.
        mma_commit(&drain_bar);
        int zero = 0;
        WaitCtl drain{&zero, wait_limit_ns, kErrKernelOprojFp8, err_word};
        mbar_wait(&drain_bar, 0, drain, 5);
      }
    }
  }
  } else {
    setmaxnreg_inc<kRegsPromo>();
    // ---------------------------------------------------------------- promotion + epilogue
    constexpr int kCols = Cfg::kCols, kChunk = Cfg::kChunk;
    const int quad = warp & 3;                     // TMEM lane quadrant this warp may access
    const int col0 = ((warp - 4) >> 2) * kCols;    // this warp's columns of the tile
    const int row_in_tile = quad * 32 + lane;
    int part = 0;
    uint32_t part_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, m_tiles, n_tiles, mb, nb);
      const int row = mb * kBM + row_in_tile;
      const bool row_ok = row < M;
      // the warp's columns lie in one 128-wide weight block
      const float* ws = w_scale + size_t(nb * (kBN / kGroup) + col0 / kGroup) * size_t(G);
      float sa[kScaleAhead], sw[kScaleAhead];
#pragma unroll
      for (int u = 0; u < kScaleAhead; ++u) {
        sa[u] = row_ok ? __ldg(a_scale + size_t(u) * size_t(M) + size_t(row)) : 0.f;
        sw[u] = __ldg(ws + u);
      }
      float acc[kCols];
#pragma unroll
      for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
      for (int g0 = 0; g0 < G && ok; g0 += kScaleAhead) {
#pragma unroll
        for (int u = 0; u < kScaleAhead; ++u) {
          const int g = g0 + u;
          if (!mbar_wait_warp(&part_full[part], part_phase, ctl, 6)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float sc = sa[u] * sw[u];
          if (g + kScaleAhead < G) {
            sa[u] = row_ok ? __ldg(a_scale + size_t(g + kScaleAhead) * size_t(M) + size_t(row))
                           : 0.f;
            sw[u] = __ldg(ws + g + kScaleAhead);
          }
          const uint32_t taddr = tmem_addr(tmem_base, quad * 32, uint32_t(part * kBN + col0));
#pragma unroll
          for (int c = 0; c < kCols / kChunk; ++c) {
            uint32_t v[kChunk];
#pragma unroll
            for (int j = 0; j < kChunk / 32; ++j)
              tmem_ld32(taddr + c * kChunk + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * j));
            tmem_ld_wait();
            reg_fence(v);
            if (c == kCols / kChunk - 1) {
              // every column of the partial is in registers: release the buffer
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&part_empty[part]);
              if (++part == kParts) {
                part = 0;
                part_phase ^= 1u;
              }
            }
#pragma unroll
            for (int i = 0; i < kChunk; i += 2)
              ffma2(acc[c * kChunk + i], acc[c * kChunk + i + 1], __uint_as_float(v[i]),
                    __uint_as_float(v[i + 1]), sc, sc, acc[c * kChunk + i],
                    acc[c * kChunk + i + 1]);
          }
        }
      }
      if (!ok) break;
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(C + size_t(row) * size_t(N) + size_t(nb) * kBN + col0);
#pragma unroll
        for (int i = 0; i < kCols / 8; ++i)
          dst[i] = make_uint4(pack_bf16x2(acc[8 * i], acc[8 * i + 1]),
                              pack_bf16x2(acc[8 * i + 2], acc[8 * i + 3]),
                              pack_bf16x2(acc[8 * i + 4], acc[8 * i + 5]),
                              pack_bf16x2(acc[8 * i + 6], acc[8 * i + 7]));
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

}  // namespace

cudaError_t launch_quant_rows_fp8(const void* x, int64_t ld, int64_t M, int K, void* q,
                                  float* scale, cudaStream_t stream) {
  if (M <= 0 || K <= 0 || K % kGroup != 0 || ld < K || ld % 8 != 0) return cudaErrorInvalidValue;
  const int64_t items = M * (K / kGroup);
  int64_t blocks = (items + 2 * kQuantWarps * kQuantUnroll - 1) / (2 * kQuantWarps * kQuantUnroll);
  if (blocks > kQuantMaxBlocks) blocks = kQuantMaxBlocks;
  quant_rows_fp8_kernel<<<unsigned(blocks), kQuantWarps * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), ld, M, K, static_cast<uint8_t*>(q), scale);
  return cudaGetLastError();
}

cudaError_t launch_quant_weight_fp8(const void* W, int N, int K, void* q, float* scale,
                                    cudaStream_t stream) {
  if (N <= 0 || K <= 0 || N % kGroup != 0 || K % kGroup != 0 || N / kGroup > 65535)
    return cudaErrorInvalidValue;
  dim3 grid(K / kGroup, N / kGroup);
  quant_weight_fp8_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(W), N, K,
                                                    static_cast<uint8_t*>(q), scale);
  return cudaGetLastError();
}

namespace {

template <int BN>
cudaError_t launch_fp8_bn(const CUtensorMap& tmA, const void* qw, const float* a_scale,
                          const float* w_scale, void* C, int64_t M, int N, int K, int num_sms,
                          unsigned long long wait_limit_ns, unsigned int* err_word,
                          cudaStream_t stream) {
  using Cfg = Fp8Cfg<BN>;
  CUtensorMap tmB;
  const uint64_t b_dims[2] = {uint64_t(K), uint64_t(N)};
  const uint64_t strides[1] = {uint64_t(K)};
  const uint32_t b_box[2] = {kGroup, BN};
  if (!encode_tmap_u8(&tmB, qw, 2, b_dims, strides, b_box, true)) return cudaErrorInvalidValue;
  auto kern = oproj_fp8_kernel<BN>;
  static ContextCache attr_done;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), int(Cfg::kSmemBytes),
                                   &attr_done);
  if (e != cudaSuccess) return e;
  const int64_t num_tiles = ((M + kBM - 1) / kBM) * (N / BN);
  const int grid = num_tiles < num_sms ? int(num_tiles) : num_sms;
  kern<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(tmA, tmB, a_scale, w_scale,
                                                   static_cast<__nv_bfloat16*>(C), int(M), N, K,
                                                   wait_limit_ns, err_word);
  return cudaGetLastError();
}

}  // namespace

int oproj_fp8_pick_bn(int64_t M, int N, int num_sms) {
  // Largest expected throughput: fraction of the last wave's SMs kept busy,
  // times the tile's measured efficiency (128-wide tiles ran at 0.83-0.88 of
  // the 256-wide ones on B200).
  struct Cand { int bn; double eff; };
  const Cand cand[2] = {{256, 1.0}, {128, 0.85}};
  int best = 128;
  double best_score = -1.0;
  for (const Cand& c : cand) {
    if (N % c.bn != 0) continue;
    const int64_t tiles = ((M + kBM - 1) / kBM) * (N / c.bn);
    const int64_t waves = (tiles + num_sms - 1) / num_sms;
    const double score = double(tiles) / double(waves * num_sms) * c.eff;
    if (score > best_score + 1e-9) {
      best_score = score;
      best = c.bn;
    }
  }
  return best;
}

cudaError_t launch_oproj_fp8(const void* qa, const float* a_scale, const void* qw,
                             const float* w_scale, void* C, int64_t M, int N, int K, int num_sms,
                             unsigned long long wait_limit_ns, unsigned int* err_word,
                             cudaStream_t stream) {
  if (M <= 0 || M > (int64_t(1) << 31) - kBM || N % 128 != 0 || K % (kGroup * kScaleAhead) != 0 ||
      num_sms <= 0)
    return cudaErrorInvalidValue;
  CUtensorMap tmA;
  const uint64_t a_dims[2] = {uint64_t(K), uint64_t(M)};
  const uint64_t strides[1] = {uint64_t(K)};
  const uint32_t a_box[2] = {kGroup, kBM};
  if (!encode_tmap_u8(&tmA, qa, 2, a_dims, strides, a_box, true)) return cudaErrorInvalidValue;
  if (oproj_fp8_pick_bn(M, N, num_sms) == 256)
    return launch_fp8_bn<256>(tmA, qw, a_scale, w_scale, C, M, N, K, num_sms, wait_limit_ns,
                              err_word, stream);
  return launch_fp8_bn<128>(tmA, qw, a_scale, w_scale, C, M, N, K, num_sms, wait_limit_ns,
                            err_word, stream);
}

}  // namespace mla
