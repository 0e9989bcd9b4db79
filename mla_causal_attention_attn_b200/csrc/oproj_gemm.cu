// oproj_gemm.cu -- the output projection C[M, N] = A[M, K] . W[N, K]^T in bf16
// with fp32 accumulation (page "Kimi K2 · Mix and project": o_proj is
// nn.Linear(64*128 -> 7168, bias=False) applied to the merged heads; the
// page's parameter table gives W 8,192 x 7,168).
//
// Design (sm_100a):
//   * persistent CTAs, one per SM, walking MT*128 x BN output tiles in a
//     grouped order (row groups for 128-row tiles, column groups for 256-row
//     ones) so concurrently running CTAs share A and W tiles in L2;
//   * warp 0 issues TMA loads of 128x64 A and BNx64 W tiles (128-byte
//     swizzle) into a STAGES-deep shared-memory ring;
//   * warp 1 allocates tensor memory and one elected thread issues
//     tcgen05.mma (M=128, N=BN, K=16) into one of two TMEM accumulators;
//   * warps 2..5 drain the finished accumulator (tcgen05.ld), convert to bf16
//     and store, while the MMA warp already fills the other accumulator.
// For M <= 128 the product is bound by reading W and runs in
// oproj_small_m_kernel (below): operands swapped, K split over a cluster of
// two CTAs, partial sums combined through distributed shared memory.
#include "oproj_gemm.h"
#include "host_util.h"
#include "sm100.cuh"

namespace mla {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
// Output tiles are visited in groups, so the tiles in flight share A rows
// and W_o columns in L2. 128-row tiles: groups of kGroupM row blocks, all
// column blocks of a group before the next (A band resident, W_o streamed);
// groups of 8, 16 and 32 ran at the same speed (M = 4096 .. 32768), 16 moved
// the least DRAM data. 256-row tiles: groups of kGroupN column blocks, all
// row blocks of a group before the next (W_o band resident, A streamed):
// measured against row groups at M = 16384 (ncu, one launch) 1.66 against
// 1.84 GB of DRAM traffic, and 1-9 % less time at M = 16384 and 32768; at M
// = 4096 (128-row tiles) column groups moved more data (540-617 against 462
// MB) and were not faster.
constexpr int kGroupM = 16;
constexpr int kGroupN = 16;
constexpr int kThreads = 192;
constexpr int64_t kSmallMMax = 128;  // M up to this goes to oproj_small_m_kernel

template <int MT>
__device__ __forceinline__ void gemm_tile_coords(int tile, int m_tiles, int n_tiles, int& mb,
                                                 int& nb) {
  if (MT == 1) {
    const int group_tiles = kGroupM * n_tiles;
    const int group = tile / group_tiles;
    const int first_m = group * kGroupM;
    const int gm = min(kGroupM, m_tiles - first_m);
    const int in_group = tile - group * group_tiles;
    mb = first_m + in_group % gm;
    nb = in_group / gm;
  } else {
    const int group_tiles = kGroupN * m_tiles;
    const int group = tile / group_tiles;
    const int first_n = group * kGroupN;
    const int gn = min(kGroupN, n_tiles - first_n);
    const int in_group = tile - group * group_tiles;
    nb = first_n + in_group % gn;
    mb = in_group / gn;
  }
}

// An output tile is MT x 128 rows by BN columns. MT = 1: two accumulators in
// tensor memory, so the epilogue of one tile overlaps the next tile's MMAs.
// MT = 2: the two 128-row halves share each W tile (a third less L2 traffic
// per FLOP) and fill the same columns, so there is one accumulator set.
template <int BN, int STAGES, int MT>
struct GemmCfg {
  static constexpr uint32_t kASub = kBM * kBK * 2;
  static constexpr uint32_t kABytes = MT * kASub;
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kNumAcc = MT == 1 ? 2 : 1;
  // rounded up to the power-of-two allocation granule
  static constexpr uint32_t kTmemCols = 2 * BN <= 128 ? 128u : (2 * BN <= 256 ? 256u : 512u);
  static_assert(MT == 1 || MT == 2, "MT");
  static constexpr size_t kSmemBytes = size_t(STAGES) * kStageBytes + 1024;
  static_assert(BN == 128 || BN == 224 || BN == 256, "BN");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                "TMEM columns must be a power of two in [32, 512]");
};

// kSplit (the latent up-projection): the 256 columns of column tile nb are
// head nb's 128 non-rotary key parts and 128 values; row m is token
// (m / T, m % T). They are stored into C = k_nope [B, 64, T, 128] and
// C2 = v [B, 64, T, 128] instead of a row-major [M, N] C.
template <int BN, int STAGES, int MT, bool kSplit = false>
__global__ void __launch_bounds__(kThreads, 1)
    oproj_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, __nv_bfloat16* __restrict__ C,
                      int M, int N, int K, unsigned long long wait_limit_ns,
                      unsigned int* err_word, __nv_bfloat16* __restrict__ C2, int T) {
  using Cfg = GemmCfg<BN, STAGES, MT>;
  static_assert(!kSplit || (BN == 256 && MT == 1), "head split: one head per 256-wide tile");
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[STAGES];
  __shared__ uint64_t empty_bar[STAGES];
  __shared__ uint64_t acc_full[2];
  __shared__ uint64_t acc_empty[2];
  __shared__ uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  // 1024-byte aligned start of the stage ring (128B-swizzle atoms).
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kTileM = MT * kBM;
  const int m_tiles = (M + kTileM - 1) / kTileM;
  const int n_tiles = N / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int k_blocks = K / kBK;
  // accumulator buffer of the local-th tile, and the parity of its use
  auto acc_buf = [](int local) { return Cfg::kNumAcc == 2 ? (local & 1) : 0; };
  auto acc_phase = [](int local) -> uint32_t {
    return Cfg::kNumAcc == 2 ? uint32_t((local >> 1) & 1) : uint32_t(local & 1);
  };
  // TMEM column of the accumulator of row half t in buffer buf
  auto acc_col = [](int buf, int t) -> uint32_t { return uint32_t((MT == 1 ? buf : t) * BN); };

  WaitCtl ctl{&abort_flag, wait_limit_ns, kErrKernelOproj, err_word};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

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
        gemm_tile_coords<MT>(tile, m_tiles, n_tiles, mb, nb);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, ctl, 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + size_t(stage) * Cfg::kStageBytes;
          uint8_t* sb = sa + Cfg::kABytes;
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::kStageBytes);
#pragma unroll
          for (int t = 0; t < MT; ++t)
            tma_load_2d(sa + t * Cfg::kASub, &tmA, &full_bar[stage], kb * kBK, mb * kTileM + t * kBM);
          tma_load_2d(sb, &tmB, &full_bar[stage], kb * kBK, nb * BN);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA's memory goes away.
        int zero = 0;
        WaitCtl drain{&zero, wait_limit_ns, kErrKernelOproj, err_word};
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_wait(&full_bar[s], (issued_par >> s) & 1u, drain, 2);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int buf = acc_buf(local);
        const uint32_t acc_par = acc_phase(local);
        if (!mbar_wait(&acc_empty[buf], acc_par ^ 1u, ctl, 3)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, ctl, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + size_t(stage) * Cfg::kStageBytes);
          const uint32_t b_addr = a_addr + Cfg::kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(b_addr + kk * 32, 16, 1024);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              const uint64_t ad = sdesc_sw128(a_addr + t * Cfg::kASub + kk * 32, 16, 1024);
              mma_ss(tmem_base + acc_col(buf, t), ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          issued_any = true;
          mma_commit(&empty_bar[stage]);  // frees the stage once these MMAs finish
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
      if (!ok && issued_any) {
        // Wait for the MMAs in flight before the tensor memory is released.
        mma_commit(&drain_bar);
        int zero = 0;
        WaitCtl drain{&zero, wait_limit_ns, kErrKernelOproj, err_word};
        mbar_wait(&drain_bar, 0, drain, 5);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int row_in_tile = quad * 32 + lane;
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      int mb, nb;
      gemm_tile_coords<MT>(tile, m_tiles, n_tiles, mb, nb);
      const int buf = acc_buf(local);
      const uint32_t acc_par = acc_phase(local);
      if (!mbar_wait_warp(&acc_full[buf], acc_par, ctl, 6)) break;
      tc_fence_after();
#pragma unroll 1
      for (int t = 0; t < MT; ++t) {
      const int row = mb * kTileM + t * kBM + row_in_tile;
      __nv_bfloat16* crow = C + size_t(row) * size_t(N) + size_t(nb) * BN;
      __nv_bfloat16* vrow = nullptr;
      if constexpr (kSplit) {
        const int bi = row / T;  // row = bi * T + ti
        const size_t off =
            ((size_t(bi) * size_t(N / BN) + nb) * size_t(T) + (row - bi * T)) * (BN / 2);
        crow = C + off;
        vrow = C2 + off;
      }
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tmem_base, quad * 32, acc_col(buf, t) + c * 32), r);
        tmem_ld_wait();
        reg_fence(r);
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        if (row < M) {
          uint4* dst = reinterpret_cast<uint4*>(crow + c * 32);
          if constexpr (kSplit)  // chunks 0..3: key part, 4..7: value
            dst = reinterpret_cast<uint4*>((c < 4 ? crow : vrow) + (c & 3) * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                packed[4 * i + 3]);
        }
      }
      }  // row halves
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

template <int BN, int STAGES, int MT>
cudaError_t launch_bn(const CUtensorMap& tmA, const void* W, __nv_bfloat16* C, int M, int N,
                      int K, int num_sms, unsigned long long wait_limit_ns,
                      unsigned int* err_word, cudaStream_t stream) {
  using Cfg = GemmCfg<BN, STAGES, MT>;
  CUtensorMap tmB;
  const uint64_t dims[2] = {uint64_t(K), uint64_t(N)};
  const uint64_t strides[1] = {uint64_t(K) * 2};
  const uint32_t box[2] = {kBK, BN};
  if (!encode_tmap_bf16(&tmB, W, 2, dims, strides, box, true)) return cudaErrorInvalidValue;
  auto kern = oproj_gemm_kernel<BN, STAGES, MT>;
  static ContextCache attr_done;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), int(Cfg::kSmemBytes),
                                   &attr_done);
  if (e != cudaSuccess) return e;
  const int m_tiles = (M + MT * kBM - 1) / (MT * kBM);
  const int num_tiles = m_tiles * (N / BN);
  const int grid = num_tiles < num_sms ? num_tiles : num_sms;
  kern<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(tmA, tmB, C, M, N, K, wait_limit_ns,
                                                   err_word, nullptr, 0);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- latent up-projection
cudaError_t launch_kv_up_impl(const void* c_kv, const void* W, void* k_nope, void* v, int B, int T,
                              int R, int num_sms, unsigned long long wait_limit_ns,
                              unsigned int* err_word, cudaStream_t stream) {
  constexpr int BN = 256, STAGES = 4;
  using Cfg = GemmCfg<BN, STAGES, 1>;
  const int64_t M64 = int64_t(B) * T;
  const int N = 64 * BN;
  if (M64 <= 0 || M64 > (int64_t(1) << 31) - kBM || R % kBK != 0) return cudaErrorInvalidValue;
  const int M = int(M64);
  CUtensorMap tmA, tmB;
  const uint64_t a_dims[2] = {uint64_t(R), uint64_t(M)};
  const uint64_t w_dims[2] = {uint64_t(R), uint64_t(N)};
  const uint64_t strides[1] = {uint64_t(R) * 2};
  const uint32_t a_box[2] = {kBK, kBM};
  const uint32_t w_box[2] = {kBK, BN};
  if (!encode_tmap_bf16(&tmA, c_kv, 2, a_dims, strides, a_box, true) ||
      !encode_tmap_bf16(&tmB, W, 2, w_dims, strides, w_box, true))
    return cudaErrorInvalidValue;
  auto kern = oproj_gemm_kernel<BN, STAGES, 1, true>;
  static ContextCache attr_done;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), int(Cfg::kSmemBytes),
                                   &attr_done);
  if (e != cudaSuccess) return e;
  const int num_tiles = ((M + kBM - 1) / kBM) * (N / BN);
  const int grid = num_tiles < num_sms ? num_tiles : num_sms;
  kern<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(
      tmA, tmB, static_cast<__nv_bfloat16*>(k_nope), M, N, R, wait_limit_ns, err_word,
      static_cast<__nv_bfloat16*>(v), T);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- small M
// C[M, N] = A[M, K] . W[N, K]^T for M <= 128, where the product is bound by
// reading W once from HBM. The operands swap roles: each CTA computes
// D = W_tile . A^T (M = 128 rows of W, N = NM >= M columns, one per token),
// so the shared-memory ring holds mostly W and the MMA accumulates
// C^T[128, NM] in tensor memory. K is split in two halves over the two CTAs
// of a cluster: the CTA of rank 1 writes its fp32 partial sum into its own
// (now idle) ring, the CTA of rank 0 adds it through distributed shared
// memory, rounds to bf16 and stores. Both hand-offs between the two CTAs are
// mbarriers with bounded waits: part_ready (in rank 0, the partial is written)
// and part_done (in rank 1, rank 0 has read it; rank 1 keeps its shared
// memory until then).
constexpr int kSmallThreads = 192;
constexpr int kSmallWRows = 128;

template <int NM, int STAGES>
struct SmallCfg {
  static constexpr uint32_t kWBytes = kSmallWRows * kBK * 2;  // 16 KB
  static constexpr uint32_t kABytes = NM * kBK * 2;
  static constexpr uint32_t kStageBytes = kWBytes + kABytes;
  static constexpr uint32_t kRowFloats = NM + 4;  // padded partial row (bank spread)
  static constexpr uint32_t kPartBytes = kSmallWRows * kRowFloats * 4;
  static constexpr uint32_t kTmemCols = NM;
  static constexpr size_t kSmemBytes = size_t(STAGES) * kStageBytes + 1024;
  static_assert(NM == 32 || NM == 64 || NM == 128, "NM");
  static_assert(kPartBytes <= STAGES * kStageBytes, "partial fits in the ring");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

template <int NM, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSmallThreads, 1)
    oproj_small_m_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmW, __nv_bfloat16* __restrict__ C,
                         int M, int N, int K, unsigned long long wait_limit_ns,
                         unsigned int* err_word, int test_stall) {
  using Cfg = SmallCfg<NM, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[STAGES];
  __shared__ uint64_t empty_bar[STAGES];
  __shared__ uint64_t acc_full;
  __shared__ uint64_t part_ready;  // rank 0: rank 1's partial is in its shared memory
  __shared__ uint64_t part_done;   // rank 1: rank 0 has read the partial
  __shared__ uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int n0 = int(blockIdx.x >> 1) * kSmallWRows;  // first W row (output column)
  const int k_blocks = K / kBK / 2;                    // this CTA's half of K
  const int kb0 = int(rank) * k_blocks;

  WaitCtl ctl{&abort_flag, wait_limit_ns, kErrKernelOprojSmallM, err_word};

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&part_ready, 128);
    mbar_init(&part_done, 128);
    mbar_init(&drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before();
  // Both CTAs' barriers are initialised before either can touch the other's.
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmW);
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int i = 0; i < k_blocks; ++i) {
        const int stage = i % STAGES;
        const uint32_t phase = uint32_t(i / STAGES) & 1u;
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, ctl, 1)) {
          ok = false;
          break;
        }
        uint8_t* sw = smem + size_t(stage) * Cfg::kStageBytes;
        uint8_t* sa = sw + Cfg::kWBytes;
        mbar_arrive_expect_tx(&full_bar[stage], Cfg::kStageBytes);
        tma_load_2d(sw, &tmW, &full_bar[stage], (kb0 + i) * kBK, n0);
        tma_load_2d(sa, &tmA, &full_bar[stage], (kb0 + i) * kBK, 0);
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
      }
      if (!ok) {
        int zero = 0;
        WaitCtl drain{&zero, wait_limit_ns, kErrKernelOprojSmallM, err_word};
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_wait(&full_bar[s], (issued_par >> s) & 1u, drain, 2);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kSmallWRows, NM, false, false);
      bool ok = true;
      bool issued_any = false;
      for (int i = 0; i < k_blocks; ++i) {
        const int stage = i % STAGES;
        const uint32_t phase = uint32_t(i / STAGES) & 1u;
        if (!mbar_wait(&full_bar[stage], phase, ctl, 4)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t w_addr = smem_u32(smem + size_t(stage) * Cfg::kStageBytes);
        const uint32_t a_addr = w_addr + Cfg::kWBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t wd = sdesc_sw128(w_addr + kk * 32, 16, 1024);
          const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
          mma_ss(tmem_base, wd, ad, idesc, (i | kk) != 0 ? 1u : 0u);
        }
        issued_any = true;
        mma_commit(&empty_bar[stage]);
      }
      if (ok) mma_commit(&acc_full);
      if (!ok && issued_any) {
        mma_commit(&drain_bar);
        int zero = 0;
        WaitCtl drain{&zero, wait_limit_ns, kErrKernelOprojSmallM, err_word};
        mbar_wait(&drain_bar, 0, drain, 5);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // Thread = TMEM lane = W row n0 + r; its TMEM columns are the tokens.
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    float* part = reinterpret_cast<float*>(smem);  // rank 1's partial, [128][kRowFloats]
    if (mbar_wait_warp(&acc_full, 0, ctl, 6)) {
      tc_fence_after();
      if (rank == 1) {
        // All MMAs (the ring's last readers) are done: the ring holds the partial.
#pragma unroll 1
        for (int c = 0; c < NM / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem_addr(tmem_base, quad * 32, c * 32), v);
          tmem_ld_wait();
          reg_fence(v);
          float4* dst = reinterpret_cast<float4*>(part + r * Cfg::kRowFloats + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                 __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
        // (Failure-detection test: the first cluster's rank 1 never reports,
        // so both CTAs' waits below must run out.)
        if (!(test_stall && blockIdx.x == 1))
          mbar_arrive_cluster(mapa_shared(smem_u32(&part_ready), 0));
        // Keep this CTA's shared memory until rank 0 has read the partial.
        mbar_wait_cluster(&part_done, 0, ctl, 8);
      } else if (mbar_wait_cluster(&part_ready, 0, ctl, 7)) {
        const uint32_t remote = mapa_shared(smem_u32(part + r * Cfg::kRowFloats), 1);
        const int n = n0 + r;
#pragma unroll 1
        for (int c = 0; c < NM / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem_addr(tmem_base, quad * 32, c * 32), v);
          tmem_ld_wait();
          reg_fence(v);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 p = ld_shared_cluster_f4(remote + (c * 32 + 4 * i) * 4);
            const float s4[4] = {__uint_as_float(v[4 * i]) + p.x,
                                 __uint_as_float(v[4 * i + 1]) + p.y,
                                 __uint_as_float(v[4 * i + 2]) + p.z,
                                 __uint_as_float(v[4 * i + 3]) + p.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int m = c * 32 + 4 * i + e;
              if (m < M) C[size_t(m) * size_t(N) + n] = __float2bfloat16_rn(s4[e]);
            }
          }
        }
        mbar_arrive_cluster(mapa_shared(smem_u32(&part_done), 1));
      }
    }
  }

  // Exit rule: neither CTA leaves while its peer may still touch its shared
  // memory (rank 1 arriving on rank 0's part_ready, rank 0 reading rank 1's
  // partial or arriving on its part_done). After a timeout on either side
  // those accesses can still come late, so both CTAs meet here first. Every
  // wait above is bounded, so every thread of both CTAs reaches this barrier.
  __syncwarp();  // the .aligned cluster barrier wants converged warps
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

template <int NM, int STAGES>
cudaError_t launch_small_m(const void* A, const void* W, __nv_bfloat16* C, int M, int N, int K,
                           unsigned long long wait_limit_ns, unsigned int* err_word,
                           cudaStream_t stream, int test_stall) {
  using Cfg = SmallCfg<NM, STAGES>;
  CUtensorMap tmA, tmW;
  const uint64_t a_dims[2] = {uint64_t(K), uint64_t(M)};
  const uint64_t w_dims[2] = {uint64_t(K), uint64_t(N)};
  const uint64_t strides[1] = {uint64_t(K) * 2};
  const uint32_t a_box[2] = {kBK, uint32_t(NM)};  // rows >= M read as zero
  const uint32_t w_box[2] = {kBK, kSmallWRows};
  if (!encode_tmap_bf16(&tmA, A, 2, a_dims, strides, a_box, true) ||
      !encode_tmap_bf16(&tmW, W, 2, w_dims, strides, w_box, true))
    return cudaErrorInvalidValue;
  auto kern = oproj_small_m_kernel<NM, STAGES>;
  static ContextCache attr_done;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), int(Cfg::kSmemBytes),
                                   &attr_done);
  if (e != cudaSuccess) return e;
  const int grid = (N / kSmallWRows) * 2;  // two CTAs (the K halves) per cluster
  kern<<<grid, kSmallThreads, Cfg::kSmemBytes, stream>>>(tmA, tmW, C, M, N, K, wait_limit_ns,
                                                        err_word, test_stall);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_up(const void* c_kv, const void* W, void* k_nope, void* v, int B, int T,
                         int R, int num_sms, unsigned long long wait_limit_ns,
                         unsigned int* err_word, cudaStream_t stream) {
  return launch_kv_up_impl(c_kv, W, k_nope, v, B, T, R, num_sms, wait_limit_ns, err_word, stream);
}

OprojTile oproj_pick_tile(int64_t M, int N, int num_sms) {
  // Largest expected throughput: fraction of the last wave's SMs kept busy,
  // times a per-tile efficiency (measured on B200: 128x256 tiles ran 3 %
  // faster than 128x224 at M = 16384, where both fill their last wave
  // equally; 256x224 tiles ran 3-7 % faster than 128x224 at M = 16384 and
  // 32768).
  struct Cand { int bn, mt; double eff; };
  const Cand cand[4] = {{256, 1, 1.0}, {224, 1, 0.97}, {128, 1, 0.95}, {224, 2, 1.03}};
  OprojTile best{128, 1};
  double best_score = -1.0;
  for (const Cand& c : cand) {
    if (N % c.bn != 0) continue;
    const int64_t m_tiles = (M + c.mt * kBM - 1) / (c.mt * kBM);
    const int64_t tiles = m_tiles * (N / c.bn);
    const int64_t waves = (tiles + num_sms - 1) / num_sms;
    const double score = double(tiles) / double(waves * num_sms) * c.eff;
    if (score > best_score + 1e-9) {
      best_score = score;
      best = OprojTile{c.bn, c.mt};
    }
  }
  return best;
}

cudaError_t launch_oproj_gemm(const void* A, const void* W, void* C, int64_t M, int N, int K,
                              int num_sms, unsigned long long wait_limit_ns, int force_bn,
                              unsigned int* err_word, cudaStream_t stream, int test_stall) {
  if (M <= 0 || N % 128 != 0 || K % kBK != 0 || M > (int64_t(1) << 31) - kBM)
    return cudaErrorInvalidValue;
  CUtensorMap tmA;
  const uint64_t dims[2] = {uint64_t(K), uint64_t(M)};
  const uint64_t strides[1] = {uint64_t(K) * 2};
  const uint32_t box[2] = {kBK, kBM};
  if (!encode_tmap_bf16(&tmA, A, 2, dims, strides, box, true)) return cudaErrorInvalidValue;
  auto* Cb = static_cast<__nv_bfloat16*>(C);
  if (!force_bn && M <= kSmallMMax && N % kSmallWRows == 0 && K % (2 * kBK) == 0) {
    // As many stages as shared memory holds: the kernel is bound by the bytes
    // of W in flight.
    if (M <= 32)
      return launch_small_m<32, 11>(A, W, Cb, int(M), N, K, wait_limit_ns, err_word, stream,
                                    test_stall);
    if (M <= 64)
      return launch_small_m<64, 9>(A, W, Cb, int(M), N, K, wait_limit_ns, err_word, stream,
                                   test_stall);
    return launch_small_m<128, 7>(A, W, Cb, int(M), N, K, wait_limit_ns, err_word, stream,
                                  test_stall);
  }
  const OprojTile tile = force_bn ? OprojTile{force_bn, 1} : oproj_pick_tile(M, N, num_sms);
  if (N % tile.bn != 0) return cudaErrorInvalidValue;
  if (tile.mt == 2) {
    if (tile.bn != 224) return cudaErrorInvalidValue;
    return launch_bn<224, 3, 2>(tmA, W, Cb, int(M), N, K, num_sms, wait_limit_ns, err_word,
                                stream);
  }
  switch (tile.bn) {
    case 256:
      return launch_bn<256, 4, 1>(tmA, W, Cb, int(M), N, K, num_sms, wait_limit_ns, err_word,
                                 stream);
    case 224:
      return launch_bn<224, 5, 1>(tmA, W, Cb, int(M), N, K, num_sms, wait_limit_ns, err_word,
                                 stream);
    case 128:
      return launch_bn<128, 6, 1>(tmA, W, Cb, int(M), N, K, num_sms, wait_limit_ns, err_word,
                                 stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace mla
