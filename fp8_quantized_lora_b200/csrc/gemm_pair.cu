// Two-SM FP8 GEMMs (tcgen05 cta_group::2) of the melded FP8 linear layer (sm_100a).
//
// The forward and dX products (the plain ones of gemm.cu: no adapter
// segment, no addend) run here:
//   forward    Y  = Xq  . Wq^T   / (s_X s_W)    A K-major, B K-major
//   dX         dX = dYq . Wq     / (s_dY s_W)   A K-major, B MN-major
// A cluster of two CTAs, one per SM, owns a 256 x 256 output tile.  Each CTA
// stages its 128 rows of A and its 128 of the tile's 256 columns of B; one
// thread of the even CTA issues M = 256 UMMAs that read the operands of both
// CTAs and leave each CTA's 128 rows of the accumulator in its own TMEM.
// Per SM and K block (128 codes) the shared memory takes 32 KB from TMA and
// feeds 32 KB to the tensor core for 128 x 256 x 128 multiply-adds; the
// one-SM 128 x 256 tile of gemm.cu moves 48 KB each way for the same work,
// more than 128 bytes per clock can carry at the FP8 tensor rate.
//
// Roles (per CTA; the MMA roles work in the even CTA only):
//   warp 0      TMA producer (one lane): this CTA's A and B tiles of a
//               `kStages`-deep ring.  The bytes of both CTAs complete on the
//               even CTA's full barrier, which the even producer arms.
//   warp 1      TMEM allocation (both CTAs, together); in the even CTA the
//               UMMA issuer (one lane).
//   warps 2-5   epilogue: this CTA's 128 rows of the accumulator, scaled, bf16.
//   warp 6      even CTA: MMA waiter.  It does the mbarrier waits and releases
//               the issuer through a named barrier (an mbarrier wait in the
//               issuing thread would hold back its MMA stream).
// The issuer's commits arrive on the barrier at the same offset in both
// CTAs (stage free, accumulator full); the epilogue warps of both CTAs
// arrive on the even CTA's accumulator-drained barrier.  Every wait is
// bounded (FALQON_DEV_TIMEOUT).
//
// Scheduling: persistent, one pair per two SMs as far as the device can
// co-schedule clusters of two; pairs take 256 x 256 tiles round robin.  A
// partial last wave of at most half the pairs runs as 256 x 128 halves
// (N = 128 pair MMAs, 64 columns of B per CTA).  An MN-major half is 64
// bytes wide, so it is staged with the 64-byte swizzle (8-row x 64-byte
// atoms) and described to the MMA as such.
#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace falqon {
namespace {

constexpr int kPairMmaBar = 1;  // named barrier between the issuer and its waiter (even CTA)

struct PairArgs {
  int32_t m_tiles, n_tiles, kb_total;
  int32_t n_full, n_half;  // items [0, n_full) whole tiles; then n_half 128-column halves
  int64_t M, N;
  void* out;               // bf16 [M][ldo]
  int64_t ldo;
  const float* scale_a;
  const float* scale_b;
  int32_t* dev_status;
};

template <bool kBMn, uint32_t kAFmt, int kStages>
struct PairCfg {
  static constexpr bool BMn = kBMn;
  static constexpr int Stages = kStages;
  static constexpr int TileM = 2 * kBM;         // 256: 128 rows per CTA
  static constexpr int TileN = 256;             // 128 columns of B staged per CTA
  static constexpr int BK = kRowBytes;          // 128 codes per K block
  static constexpr int KSteps = kRowBytes / 32; // UMMA K = 32 codes
  static constexpr int ABytes = kBM * kRowBytes;          // 16 KB
  static constexpr int BBytes = (TileN / 2) * kRowBytes;  // 16 KB
  static constexpr int StageBytes = ABytes + BBytes;
  static constexpr int Acc = 2;
  static constexpr uint32_t TmemCols = 512;     // two accumulators of 256 columns
  static constexpr int EpiWarps = 4;
  static constexpr int WaiterWarp = 6;
  static constexpr int Threads = 32 * (WaiterWarp + 1);
  static constexpr int BarBytes = 8 * (2 * kStages + 2 * Acc + 1) + 16;
  static constexpr int SmemBytes = kStages * StageBytes + BarBytes + 1024;
  static constexpr uint32_t IDesc = idesc_f32acc(kAFmt, 0u, 0u, kBMn ? 1u : 0u, 256, TileN);
  static constexpr uint32_t IDescHalf = idesc_f32acc(kAFmt, 0u, 0u, kBMn ? 1u : 0u, 256, TileN / 2);
  static_assert(SmemBytes <= 232448, "shared memory per CTA");
};

template <class C>
__global__ void __launch_bounds__(C::Threads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmBh, const PairArgs g) {
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::Stages * C::StageBytes);
  uint64_t* full = bars;                      // [Stages] both CTAs' tiles landed (even CTA's copy is used)
  uint64_t* empty = bars + C::Stages;         // [Stages] the MMAs are done with this CTA's slot
  uint64_t* acc_full = bars + 2 * C::Stages;  // [Acc] accumulator ready (both CTAs)
  uint64_t* acc_empty = acc_full + C::Acc;    // [Acc] drained by both epilogues (even CTA's copy)
  uint64_t* drain = acc_empty + C::Acc;       // the even CTA's MMAs retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the pair's MMAs
  const bool lead = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int total = g.n_full + g.n_half;
  auto item = [&](int w, int& mt, int& nt, int& nh) {
    int t = w;
    nh = -1;
    if (w >= g.n_full) {
      t = g.n_full + ((w - g.n_full) >> 1);
      nh = (w - g.n_full) & 1;
    }
    nt = t % g.n_tiles;
    mt = t / g.n_tiles;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::Acc; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * C::EpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();  // visible to the other CTA's copies and arrivals
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmBh);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();  // the next kernel may start launching; it waits for this one
  pdl_wait();     // the previous kernel's results are complete and visible

  auto fail = [&]() {
    *abort_flag = 1;
    raise_status(g.dev_status, kDevTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_lead = dsmem_addr(full, 0);  // the even CTA's full[0]
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;
      bool ok = true;
      for (int w = pair; w < total && ok; w += npairs) {
        int mt, nt, nh;
        item(w, mt, nt, nh);
        const bool halfi = nh >= 0;
        const int bcols = halfi ? C::TileN / 4 : C::TileN / 2;  // B columns this CTA stages
        const int m0 = mt * C::TileM + static_cast<int>(rank) * kBM;
        const int n0 = nt * C::TileN + (nh > 0 ? C::TileN / 2 : 0) + static_cast<int>(rank) * bcols;
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { fail(); ok = false; break; }
          uint8_t* sA = smem + stage * C::StageBytes;
          uint8_t* sB = sA + C::ABytes;
          if (lead) mbar_arrive_expect_tx(&full[stage], 2u * static_cast<uint32_t>(C::ABytes + bcols * kRowBytes));
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          const uint32_t fb = full_lead + 8u * static_cast<uint32_t>(stage);
          tma_load_2d_pair(sA, &tmA, fb, kb * C::BK, m0);
          if constexpr (C::BMn)  // [K rows][128 columns]: one 128-byte block (64 for a half: 64-byte swizzle)
            tma_load_2d_pair(sB, halfi ? &tmBh : &tmB, fb, n0, kb * C::BK);
          else
            tma_load_2d_pair(sB, halfi ? &tmBh : &tmB, fb, kb * C::BK, n0);
          if (++stage == C::Stages) { stage = 0; phase ^= 1; }
        }
      }
      // Teardown: every slot this lane filled has been consumed by the MMAs
      // (or, after an abort, the bounded wait has outlasted the copies).
      for (int s = 0; s < C::Stages; ++s)
        if (issued & (1u << s))
          if (!mbar_wait_budget(&empty[s], (issued_parity >> s) & 1u)) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lead) {
      int stage = 0;
      int acc = 0;
      for (int w = pair; w < total; w += npairs) {
        if (bar_red_or(kPairMmaBar, 64, false)) break;
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + static_cast<uint32_t>(acc * C::TileN);
        const bool halfi = w >= g.n_full;
        const uint32_t idesc = halfi ? C::IDescHalf : C::IDesc;
        bool abort = false;
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (bar_red_or(kPairMmaBar, 64, false)) { abort = true; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_base = smem_u32(smem + stage * C::StageBytes);
            const uint32_t b_base = a_base + C::ABytes;
#pragma unroll
            for (int ks = 0; ks < C::KSteps; ++ks) {
              // an MN-major half tile: [K rows][64 bytes], 64-byte swizzle, 8-row atoms 512 B apart
              const uint64_t bd = (C::BMn && halfi) ? sdesc_sw64(b_base + ks * 32 * 64, 64 * C::BK, 512)
                                                    : operand_desc<C::BMn, 1, C::BK>(b_base, ks);
              umma_f8_pair(tmem_d, operand_desc<false, 1, C::BK>(a_base, ks), bd, idesc,
                           (kb > 0 || ks > 0) ? 1u : 0u);
            }
            umma_commit_pair_both(&empty[stage]);
          }
          __syncwarp();
          if (++stage == C::Stages) stage = 0;
        }
        if (abort) break;
        if (lane == 0) umma_commit_pair_both(&acc_full[acc]);
        __syncwarp();
        if (++acc == C::Acc) acc = 0;
      }
      if (lane == 0) {
        umma_commit_pair_local(drain);
        mbar_wait_budget(drain, 0);
      }
      __syncwarp();
    }
  } else if (warp == C::WaiterWarp) {
    // ------------------------------------------------------------ MMA waiter (even CTA)
    if (lead) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int w = pair; w < total; w += npairs) {
        const bool ok_acc = warp_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag);
        if (!ok_acc && lane == 0) fail();
        __syncwarp();
        if (bar_red_or(kPairMmaBar, 64, !ok_acc)) break;
        bool abort = false;
        for (int kb = 0; kb < g.kb_total; ++kb) {
          const bool ok = warp_wait(&full[stage], phase, abort_flag);
          if (!ok && lane == 0) fail();
          __syncwarp();
          if (bar_red_or(kPairMmaBar, 64, !ok)) { abort = true; break; }
          if (++stage == C::Stages) { stage = 0; phase ^= 1; }
        }
        if (abort) break;
        if (++acc == C::Acc) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t empty_lead = dsmem_addr(acc_empty, 0);
    float alpha = 1.0f;
    {
      double den = g.scale_a ? static_cast<double>(*g.scale_a) : 1.0;
      if (g.scale_b) den *= static_cast<double>(*g.scale_b);
      alpha = static_cast<float>(1.0 / den);
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = pair; w < total; w += npairs) {
      int mt, nt, nh;
      item(w, mt, nt, nh);
      if (!warp_wait(&acc_full[acc], acc_phase, abort_flag)) { if (lane == 0) fail(); break; }
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mt) * C::TileM + rank * kBM + q * 32 + lane;
      const int64_t col_base = static_cast<int64_t>(nt) * C::TileN + (nh > 0 ? C::TileN / 2 : 0);
      const int chunks = (nh >= 0 ? C::TileN / 2 : C::TileN) / 32;
#pragma unroll 1
      for (int c = 0; c < chunks; ++c) {
        uint32_t r[32];
        tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::TileN + c * 32),
                       r);
        tmem_ld_wait();
        if (row < g.M) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.out) + row * g.ldo;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int64_t col = col_base + c * 32 + 8 * j;
            if (col < g.N) {  // N % 8 == 0: eight columns in or out together
              uint32_t pk[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 2 * h]) * alpha,
                                                               __uint_as_float(r[8 * j + 2 * h + 1]) * alpha);
                memcpy(&pk[h], &b, 4);
              }
              *reinterpret_cast<uint4*>(dst + col) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(empty_lead + 8u * static_cast<uint32_t>(acc));
      if (++acc == C::Acc) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // the even CTA's MMAs have retired: no copy or MMA touches either CTA any more
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TmemCols);
  }
}

// ---------------------------------------------------------------- host side
// Six stages of 32 KB (seven measured the same).
using PairFwdCfg = PairCfg<false, 0u, 6>;
using PairDxCfg = PairCfg<true, 0u, 6>;
using PairDxE5Cfg = PairCfg<true, 1u, 6>;  // dYq in E5M2

// Pairs the device can keep resident at once (cached per device): the grid
// never exceeds it, so the persistent pairs all run in one wave.
template <class C>
int resident_pairs(const DeviceInfo* di) {
  static int cached[32] = {0};
  const int dev = di->device;
  if (dev >= 0 && dev < 32 && cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(di->sm_count & ~1));
  cfg.blockDim = dim3(C::Threads);
  cfg.dynamicSmemBytes = C::SmemBytes;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_pair_kernel<C>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = di->sm_count / 2;
  }
  if (n > di->sm_count / 2) n = di->sm_count / 2;
  if (dev >= 0 && dev < 32) cached[dev] = n;
  return n;
}

template <class C>
cudaError_t pair_gemm(const uint8_t* a, const float* sa, const uint8_t* b, const float* sb, int64_t M,
                      int64_t Ncols, int64_t Kc, void* out, int32_t* dev_status, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  static int configured_mask = 0;  // one bit per device ordinal < 31
  const int bit = di->device < 31 ? (1 << di->device) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SmemBytes);
    if (e != cudaSuccess) return e;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_ACQ_REL);
  }
  CUtensorMap tA, tB, tBh;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  if (!make_tmap_2d(&tA, U8, 1, a, Kc, M, C::BK, kBM, true)) return cudaErrorInvalidValue;
  if constexpr (C::BMn) {
    // B [Kc, Ncols] row-major: boxes of 128 columns (one 128-byte block) x BK rows
    if (!make_tmap_2d(&tB, U8, 1, b, Ncols, Kc, C::TileN / 2, C::BK, true)) return cudaErrorInvalidValue;
    if (!make_tmap_2d_sw64(&tBh, U8, 1, b, Ncols, Kc, C::TileN / 4, C::BK)) return cudaErrorInvalidValue;
  } else {
    // B [Ncols, Kc] K-major: boxes of BK codes x 128 rows (64 for half tiles)
    if (!make_tmap_2d(&tB, U8, 1, b, Kc, Ncols, C::BK, C::TileN / 2, true)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tBh, U8, 1, b, Kc, Ncols, C::BK, C::TileN / 4, true)) return cudaErrorInvalidValue;
  }
  PairArgs g{};
  g.m_tiles = ceil_div(M, C::TileM);
  g.n_tiles = ceil_div(Ncols, C::TileN);
  g.kb_total = ceil_div(Kc, C::BK);
  g.M = M;
  g.N = Ncols;
  g.out = out;
  g.ldo = Ncols;
  g.scale_a = sa;
  g.scale_b = sb;
  g.dev_status = dev_status;
  const int tiles = g.m_tiles * g.n_tiles;
  if (tiles == 0) return cudaSuccess;
  const int slots = resident_pairs<C>(di);
  const int pairs = tiles < slots ? tiles : slots;
  // a partial last wave of at most half the pairs runs as 256 x 128 halves
  const int tail = tiles % pairs;
  g.n_full = tiles;
  g.n_half = 0;
  if (tiles > pairs && tail > 0 && 2 * tail <= pairs) {
    g.n_full = tiles - tail;
    g.n_half = 2 * tail;
  }
  return launch_pdl(tc_gemm_pair_kernel<C>, dim3(static_cast<unsigned>(2 * pairs)), dim3(C::Threads), C::SmemBytes,
                    stream, 2u, tA, tB, tBh, g);
}

}  // namespace

cudaError_t launch_fp8_gemm_fwd_pair(const uint8_t* xq, const float* s_x, const uint8_t* wq, const float* s_w,
                                     int64_t M, int64_t N, int64_t K, void* y, int32_t* dev_status,
                                     cudaStream_t stream) {
  return pair_gemm<PairFwdCfg>(xq, s_x, wq, s_w, M, N, K, y, dev_status, stream);
}

cudaError_t launch_fp8_gemm_dx_pair(const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
                                    int64_t M, int64_t N, int64_t K, void* dx, int32_t* dev_status,
                                    cudaStream_t stream, bool dy_e5m2) {
  // contraction over N: A = dYq [M, N] K-major; B = Wq [N, K] read MN-major (K contiguous)
  if (dy_e5m2) return pair_gemm<PairDxE5Cfg>(dyq, s_dy, wq, s_w, M, K, N, dx, dev_status, stream);
  return pair_gemm<PairDxCfg>(dyq, s_dy, wq, s_w, M, K, N, dx, dev_status, stream);
}

}  // namespace falqon
