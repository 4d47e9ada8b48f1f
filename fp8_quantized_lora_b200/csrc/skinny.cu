// Rank-r adapter products of the melded FP8 linear backward (sm_100a).
//
// FALQON, OpenReview rebuttal (reviewer 4, Q1): B's gradient comes from the
// precomputable product A x, and A's from B^T dL/dO; both reuse the E4M3
// codes the quantize step produced.  With T = Xq A^T / s_X and
// U = dYq B / s_dY (fp32 tiles kept as bf16 hi/lo pairs):
//   T   = Xq . A^T          [M, r]   A-op Xq   K-major,  B-op A   [r, K]  K-major
//   U   = dYq . B           [M, r]   A-op dYq  K-major,  B-op B   [N, r]  MN-major
//   dB  = dYq^T . T / s_dY  [N, r]   A-op dYq^T MN-major, B-op T (hi + lo) MN-major
//   dA^T= Xq^T . U / s_X    [K, r]   A-op Xq^T  MN-major, B-op U (hi + lo) MN-major
//
// The E4M3 codes are expanded exactly to bf16 in shared memory and fed to
// tcgen05 kind::f16 (every E4M3 value is a bf16 value).  One launch runs two
// independent products (T with U, then dB with dA): the first `ctas0` CTAs
// work on problem 0, the others on problem 1, two CTAs per SM where the tiles
// allow, so the start-up and reduction phases of one CTA overlap the main
// loop of its neighbour.  Each CTA owns one (row tile, K split) work item;
// the `splits` CTAs of a row tile form one cluster and sum their fp32 tiles
// through DSMEM in rank order (deterministic).
//
// Roles per CTA:
//   warp 0       TMA producer for the small bf16 operand (one lane)
//   warp 1       TMEM owner and UMMA issuer (one lane issues)
//   warps 2-5    epilogue: TMEM -> fp32 reduction tile in shared memory
//   warps 6-13   converters: raw E4M3 tile -> bf16, 128-byte-swizzled
//   warp 14      TMA producer for the raw E4M3 tiles (one lane)
#include "internal.h"
#include "tc_common.cuh"

namespace falqon {
namespace {

struct SkinnyProblem {
  int32_t m_tiles, n_tiles, splits, kb_total, kb_per_split;
  int64_t M, N;        // output rows (UMMA M side) and columns (r)
  void* out;           // bf16 [M][ldo] (or [N][ldo] when transposed)
  void* out_lo;        // optional low half of a hi/lo pair
  int64_t ldo;
  int transpose;       // store out[col * ldo + row]
  int b_mn;            // the bf16 operand is MN-major (else K-major)
  const float* scale;  // alpha = 1 / *scale
};

struct SkinnyArgs {
  SkinnyProblem p[2];
  int ctas0;           // CTAs of problem 0; the rest work on problem 1
  int32_t* dev_status;
};

template <int kBN, bool kAMn, bool kBSplit, int kSA, int kSB, int kSR, int kMinBlocks>
struct SkCfg {
  static constexpr int BN = kBN;
  static constexpr bool AMn = kAMn;
  static constexpr bool BSplit = kBSplit;  // B = B_hi + B_lo: two tiles, two MMAs per k-step
  static constexpr int SA = kSA, SB = kSB, SR = kSR;
  static constexpr int MinBlocks = kMinBlocks;
  static constexpr int BK = 64;                             // bf16 K per stage
  static constexpr int KSteps = 4;                          // UMMA K = 16
  static constexpr int ABytes = kBM * BK * 2;               // expanded A tile, 16 KB
  static constexpr int BBytes = kBN * BK * 2;
  static constexpr int BSlotBytes = BBytes * (kBSplit ? 2 : 1);
  static constexpr int RawSlotBytes = kBM * BK;             // 8 KB of codes
  static constexpr int ConvWarps = 8;
  static constexpr int RawWarp = 6 + ConvWarps;
  static constexpr int Threads = 32 * (RawWarp + 1);        // 480
  static constexpr uint32_t TmemCols = kBN < 32 ? 32 : kBN;
  static constexpr int ARing = kSA * ABytes, BRing = kSB * BSlotBytes, RawRing = kSR * RawSlotBytes;
  static constexpr int BarBytes = 8 * (2 * kSA + 2 * kSB + 2 * kSR + 2) + 16;
  static constexpr int SmemBytes = ARing + BRing + RawRing + BarBytes + 1024;
  static constexpr int RedStride = kBN + 4;  // fp32 words per row of the reduction tile
  static_assert(kBM * RedStride * 4 <= ARing + BRing, "reduction tile");
  static_assert(kBN % 64 == 0 && kBN <= 256, "UMMA N, 128-byte MN-major blocks");
  static_assert(RawSlotBytes == 2 * 16 * 32 * ConvWarps, "two 16-byte chunks per converter thread");
  static_assert(kSA >= 2 && kSB >= 2 && kSR >= 2, "ring depths");
  static_assert(SmemBytes * kMinBlocks <= 228 * 1024 - 1024 * kMinBlocks, "shared memory per SM");
};

template <class C>
__global__ void __launch_bounds__(C::Threads, C::MinBlocks)
    skinny_kernel(const __grid_constant__ CUtensorMap raw0, const __grid_constant__ CUtensorMap b0,
                  const __grid_constant__ CUtensorMap b20, const __grid_constant__ CUtensorMap raw1,
                  const __grid_constant__ CUtensorMap b1, const __grid_constant__ CUtensorMap b21,
                  const SkinnyArgs args) {
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_ring = smem;                                 // expanded A tiles
  uint8_t* b_ring = smem + C::ARing;                      // bf16 operand tiles
  uint8_t* raw_ring = b_ring + C::BRing;                  // raw E4M3 tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw_ring + C::RawRing);
  uint64_t* full = bars;                                  // [SB] B landed
  uint64_t* empty = full + C::SB;                         // [SB] MMAs done with the B slot
  uint64_t* conv = empty + C::SB;                         // [SA] A expanded
  uint64_t* aempty = conv + C::SA;                        // [SA] MMAs done with the A slot
  uint64_t* rawfull = aempty + C::SA;                     // [SR] raw codes landed
  uint64_t* rawempty = rawfull + C::SR;                   // [SR] converters done reading
  uint64_t* acc_full = rawempty + C::SR;                  // accumulator complete
  uint64_t* drain = acc_full + 1;                         // all MMAs retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool second = static_cast<int>(blockIdx.x) >= args.ctas0;
  const SkinnyProblem& g = args.p[second ? 1 : 0];
  const CUtensorMap* tmRaw = second ? &raw1 : &raw0;
  const CUtensorMap* tmB = second ? &b1 : &b0;
  const CUtensorMap* tmB2 = second ? &b21 : &b20;
  const int w = static_cast<int>(blockIdx.x) - (second ? args.ctas0 : 0);  // work item
  const int split = w % g.splits;
  const int nt = (w / g.splits) % g.n_tiles;
  const int mt = w / (g.splits * g.n_tiles);
  const int kb0 = split * g.kb_per_split;
  const int kb1 = min(g.kb_total, kb0 + g.kb_per_split);
  const bool b_mn = g.b_mn != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(&conv[s], C::ConvWarps);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < C::SR; ++s) {
      mbar_init(&rawfull[s], 1);
      mbar_init(&rawempty[s], C::ConvWarps);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(tmRaw);
    tma_prefetch_desc(tmB);
    if constexpr (C::BSplit) tma_prefetch_desc(tmB2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    raise_status(args.dev_status, kDevTimeout);
  };
  // one producer lane: waits `emp`, then fills `ful` with `load(slot, kb)`
  auto produce = [&](uint64_t* ful, uint64_t* emp, int depth, uint32_t bytes, auto load) {
    int s = 0;
    uint32_t ph = 0, issued = 0, issued_parity = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&emp[s], ph ^ 1, abort_flag)) { fail(); break; }
      mbar_arrive_expect_tx(&ful[s], bytes);
      issued |= 1u << s;
      issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
      load(s, kb);
      if (++s == depth) { s = 0; ph ^= 1; }
    }
    // every load issued must land before shared memory is reused or released
    for (int t = 0; t < depth; ++t)
      if (issued & (1u << t)) mbar_wait_budget(&ful[t], (issued_parity >> t) & 1u);
  };

  constexpr int kTileRows = C::AMn ? C::BK : kBM;  // rows of the A tile (and of its raw box)
  constexpr int kTileCols = C::AMn ? kBM : C::BK;  // codes per row
  if (warp == 0) {
    // ------------------------------------------------------------ bf16 operand producer
    if (lane == 0) {
      const int n0 = nt * C::BN;
      produce(full, empty, C::SB, static_cast<uint32_t>(C::BSlotBytes), [&](int s, int kb) {
        uint8_t* sB = b_ring + s * C::BSlotBytes;
        if (b_mn) {
          // [K rows][N] row-major: 128-byte column blocks of 64 K rows each
#pragma unroll
          for (int c = 0; c < C::BN / 64; ++c) {
            tma_load_2d(sB + c * C::BK * kRowBytes, tmB, &full[s], n0 + c * 64, kb * C::BK);
            if constexpr (C::BSplit)
              tma_load_2d(sB + C::BBytes + c * C::BK * kRowBytes, tmB2, &full[s], n0 + c * 64, kb * C::BK);
          }
        } else {
          tma_load_2d(sB, tmB, &full[s], kb * C::BK, n0);
          if constexpr (C::BSplit) tma_load_2d(sB + C::BBytes, tmB2, &full[s], kb * C::BK, n0);
        }
      });
    }
    __syncwarp();
  } else if (warp == C::RawWarp) {
    // ------------------------------------------------------------ raw-code producer
    // K-major A = codes[m0 .. +128, kb*64 .. +64]; MN-major A = codes[kb*64 .. +64, m0 .. +128]
    if (lane == 0) {
      produce(rawfull, rawempty, C::SR, static_cast<uint32_t>(C::RawSlotBytes), [&](int s, int kb) {
        if constexpr (C::AMn)
          tma_load_2d(raw_ring + s * C::RawSlotBytes, tmRaw, &rawfull[s], mt * kBM, kb * C::BK);
        else
          tma_load_2d(raw_ring + s * C::RawSlotBytes, tmRaw, &rawfull[s], kb * C::BK, mt * kBM);
      });
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_f32acc(1u, 1u, C::AMn ? 1u : 0u, b_mn ? 1u : 0u, kBM, C::BN);
    int sb = 0, sa = 0;
    uint32_t pb = 0, pa = 0;
    bool ok = true;
    tc_fence_after();
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!warp_wait(&conv[sa], pa, abort_flag) || !warp_wait(&full[sb], pb, abort_flag)) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_base = smem_u32(a_ring + sa * C::ABytes);
        const uint32_t b_base = smem_u32(b_ring + sb * C::BSlotBytes);
#pragma unroll
        for (int ks = 0; ks < C::KSteps; ++ks) {
          const uint64_t ad = operand_desc_rt<2, C::BK>(C::AMn, a_base, ks);
          const uint64_t bd = operand_desc_rt<2, C::BK>(b_mn, b_base, ks);
          umma_bf16(tmem_base, ad, bd, idesc, (kb > kb0 || ks > 0) ? 1u : 0u);
          if constexpr (C::BSplit)
            umma_bf16(tmem_base, ad, operand_desc_rt<2, C::BK>(b_mn, b_base + C::BBytes, ks), idesc, 1u);
        }
        umma_commit(&empty[sb]);
        umma_commit(&aempty[sa]);
      }
      __syncwarp();
      if (++sb == C::SB) { sb = 0; pb ^= 1; }
      if (++sa == C::SA) { sa = 0; pa ^= 1; }
    }
    if (lane == 0) {
      if (ok) umma_commit(acc_full);
      umma_commit(drain);
      mbar_wait_budget(drain, 0);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    // fp32 accumulator rows -> reduction tile in shared memory (the rings are
    // idle once every MMA has completed)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    if (warp_wait(acc_full, 0, abort_flag)) {
      tc_fence_after();
      float* red_row = reinterpret_cast<float*>(smem) + (q * 32 + lane) * C::RedStride;
      const bool empty_split = kb1 <= kb0;  // no K blocks: the partial sum is zero
#pragma unroll 1
      for (int c = 0; c < C::BN / 16; ++c) {
        uint32_t r[16];
        if (!empty_split) {
          tmem_ld_16cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + c * 16, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] = 0u;
        }
        float4* red = reinterpret_cast<float4*>(red_row + c * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          red[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                               __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
      }
    } else if (lane == 0) {
      fail();
    }
    tc_fence_before();
  } else {
    // ------------------------------------------------------------ converters
    // 256 threads; each expands two 16-byte chunks (32 codes) of every A tile:
    //   K-major  [128 rows][64 codes]:  rows t/4 and t/4 + 64,  columns (t % 4) * 16 ..
    //   MN-major [64 rows][128 codes]:  rows t/8 and t/8 + 32,  columns (t % 8) * 16 ..
    constexpr int kThrPerRow = kTileCols / 16;
    constexpr int kRowStep = 256 / kThrPerRow;  // second chunk: this many rows further down
    const int t = threadIdx.x - 6 * 32;
    const int trow = t / kThrPerRow;
    const int tcol = (t % kThrPerRow) * 16;
    const uint32_t raw_off0 = trow * kTileCols + tcol;
    const uint32_t raw_off1 = (trow + kRowStep) * kTileCols + tcol;
    const int blk = tcol / 64;
    const int unit0 = (tcol % 64) / 8;
    auto dst_off = [&](int row, int unit) {
      return static_cast<uint32_t>(blk * (kTileRows * kRowBytes) + row * kRowBytes +
                                   ((unit ^ (row & 7)) << 4));
    };
    const uint32_t d00 = dst_off(trow, unit0), d01 = dst_off(trow, unit0 + 1);
    const uint32_t d10 = dst_off(trow + kRowStep, unit0), d11 = dst_off(trow + kRowStep, unit0 + 1);
    int sa = 0, sr = 0;
    uint32_t pa = 0, pr = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!warp_wait(&rawfull[sr], pr, abort_flag)) { if (lane == 0) fail(); break; }
      const uint4 q0 = *reinterpret_cast<const uint4*>(raw_ring + sr * C::RawSlotBytes + raw_off0);
      const uint4 q1 = *reinterpret_cast<const uint4*>(raw_ring + sr * C::RawSlotBytes + raw_off1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&rawempty[sr]);
      if (++sr == C::SR) { sr = 0; pr ^= 1; }
      uint32_t o0[8], o1[8];
      e4m3x16_to_bf16(q0, o0);
      e4m3x16_to_bf16(q1, o1);
      if (!warp_wait(&aempty[sa], pa ^ 1, abort_flag)) { if (lane == 0) fail(); break; }
      uint8_t* sA = a_ring + sa * C::ABytes;
      *reinterpret_cast<uint4*>(sA + d00) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
      *reinterpret_cast<uint4*>(sA + d01) = make_uint4(o0[4], o0[5], o0[6], o0[7]);
      *reinterpret_cast<uint4*>(sA + d10) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
      *reinterpret_cast<uint4*>(sA + d11) = make_uint4(o1[4], o1[5], o1[6], o1[7]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&conv[sa]);
      if (++sa == C::SA) { sa = 0; pa ^= 1; }
    }
  }

  // ---------------------------------------------------------------- split-K reduction
  // Sum the cluster's tiles row slice by row slice (this CTA owns rows
  // [q0, q1) of the tile), in rank order, and write bf16 (or hi/lo pairs).
  __syncthreads();
  cluster_sync_all();
  {
    const int S = g.splits;
    const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
    const int rows_per = (kBM + S - 1) / S;
    const int q0 = static_cast<int>(rank) * rows_per;
    const int q1 = min(kBM, q0 + rows_per);
    const float* red = reinterpret_cast<const float*>(smem);
    uint32_t peer[kMaxSplits];
#pragma unroll
    for (int sidx = 0; sidx < kMaxSplits; ++sidx) peer[sidx] = dsmem_addr(red, sidx < S ? sidx : 0);
    const float alpha = g.scale ? static_cast<float>(1.0 / static_cast<double>(*g.scale)) : 1.0f;
    const int nrows = q1 - q0;
    constexpr int G = C::BN / 4;  // float4 groups per row
    const int ngroups = nrows > 0 ? nrows * G : 0;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
    __nv_bfloat16* out_lo = static_cast<__nv_bfloat16*>(g.out_lo);
    for (int e = threadIdx.x; e < ngroups; e += blockDim.x) {
      int lr, lg;
      if (g.transpose) { lr = q0 + e % nrows; lg = e / nrows; }  // walk rows: coalesced out[col][row]
      else { lr = q0 + e / G; lg = e % G; }
      const uint32_t off = static_cast<uint32_t>((lr * C::RedStride + 4 * lg) * 4);
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int s0 = 0; s0 < kMaxSplits; s0 += 4) {  // fixed order: rank 0, 1, ...
        float4 part[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (s0 + k < S) part[k] = dsmem_load_f32x4(peer[s0 + k] + off);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (s0 + k < S) {
            acc.x += part[k].x;
            acc.y += part[k].y;
            acc.z += part[k].z;
            acc.w += part[k].w;
          }
        }
      }
      const int64_t grow = static_cast<int64_t>(mt) * kBM + lr;
      const int64_t gcol0 = static_cast<int64_t>(nt) * C::BN + 4 * lg;
      if (grow >= g.M || gcol0 >= g.N) continue;  // N % 16 == 0: groups of 4 in or out
      const float vals[4] = {acc.x * alpha, acc.y * alpha, acc.z * alpha, acc.w * alpha};
      __nv_bfloat16 hi[4], lo[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        hi[k] = __float2bfloat16_rn(vals[k]);
        lo[k] = __float2bfloat16_rn(vals[k] - __bfloat162float(hi[k]));
      }
      if (g.transpose) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          out[(gcol0 + k) * g.ldo + grow] = hi[k];
          if (out_lo) out_lo[(gcol0 + k) * g.ldo + grow] = lo[k];
        }
      } else {
        uint2 ph, pl;
        memcpy(&ph, hi, 8);
        memcpy(&pl, lo, 8);
        *reinterpret_cast<uint2*>(out + grow * g.ldo + gcol0) = ph;
        if (out_lo) *reinterpret_cast<uint2*>(out_lo + grow * g.ldo + gcol0) = pl;
      }
    }
  }
  cluster_sync_all();  // no CTA leaves while a peer still reads its tile

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TmemCols);
  }
}

// ---------------------------------------------------------------- host side
// Stage depths <A (expanded), B (bf16 operand), raw codes>: two CTAs per SM
// where 64-wide (and 128-wide K-major) tiles allow, one otherwise.
template <int BN> using KCfg = SkCfg<BN, false, false, 3, (BN == 128 ? 2 : 3), (BN == 128 ? 3 : 4), (BN <= 128 ? 2 : 1)>;
template <int BN> using MCfg = SkCfg<BN, true, true, (BN == 256 ? 2 : 3), (BN == 64 ? 2 : (BN == 128 ? 3 : 2)),
                                     (BN == 64 ? 3 : 4), (BN == 64 ? 2 : 1)>;

template <class C>
cudaError_t launch_skinny(const CUtensorMap (&maps)[6], const SkinnyArgs& args, int grid,
                          cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  static int configured_mask = 0;  // one bit per device ordinal < 31
  const int bit = di->device < 31 ? (1 << di->device) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(skinny_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SmemBytes);
    if (e != cudaSuccess) return e;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_ACQ_REL);
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(args.p[0].splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::Threads);
  cfg.dynamicSmemBytes = C::SmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, skinny_kernel<C>, maps[0], maps[1], maps[2], maps[3], maps[4],
                            maps[5], args);
}

int skinny_bn(int64_t r) { return r <= 64 ? 64 : (r <= 128 ? 128 : 256); }

// One product: rows_out x r output, contraction kc.
struct Product {
  int64_t rows_out, kc;
  void* out;
  void* out_lo;
  int64_t ldo;
  bool transpose, b_mn;
  const float* scale;
  CUtensorMap raw, b, b2;
};

// Launches one or two products (the second may be null) as one grid.
template <template <int> class CF>
cudaError_t run_products(const Product* p0, const Product* p1, int64_t r, const DeviceInfo* di,
                         int32_t* dev_status, cudaStream_t stream) {
  const int bn = skinny_bn(r);
  const int n_tiles = ceil_div(r, bn);
  const int per_sm = bn == 64 || (bn == 128 && !CF<128>::AMn) ? 2 : 1;
  const Product* ps[2] = {p0, p1};
  int tiles[2] = {0, 0}, kbt[2] = {0, 0};
  for (int i = 0; i < 2; ++i) {
    if (!ps[i]) continue;
    tiles[i] = ceil_div(ps[i]->rows_out, kBM) * n_tiles;
    kbt[i] = ceil_div(ps[i]->kc, 64);
  }
  // one split count for the whole grid (the cluster size is per launch)
  const int kb_min = p1 ? std::min(kbt[0], kbt[1]) : kbt[0];
  const int splits = choose_splits(tiles[0] + tiles[1], kb_min, per_sm * di->sm_count);
  SkinnyArgs args{};
  args.dev_status = dev_status;
  CUtensorMap maps[6];
  for (int i = 0; i < 2; ++i) {
    const Product* p = ps[i] ? ps[i] : ps[0];
    SkinnyProblem& q = args.p[i];
    q.m_tiles = ceil_div(p->rows_out, kBM);
    q.n_tiles = n_tiles;
    q.splits = splits;
    q.kb_total = ceil_div(p->kc, 64);
    q.kb_per_split = ceil_div(q.kb_total, splits);
    q.M = p->rows_out;
    q.N = r;
    q.out = p->out;
    q.out_lo = p->out_lo;
    q.ldo = p->ldo;
    q.transpose = p->transpose ? 1 : 0;
    q.b_mn = p->b_mn ? 1 : 0;
    q.scale = p->scale;
    maps[3 * i] = p->raw;
    maps[3 * i + 1] = p->b;
    maps[3 * i + 2] = p->b2;
  }
  args.ctas0 = args.p[0].m_tiles * n_tiles * splits;
  const int grid = args.ctas0 + (p1 ? args.p[1].m_tiles * n_tiles * splits : 0);
  switch (bn) {
    case 64: return launch_skinny<CF<64>>(maps, args, grid, stream);
    case 128: return launch_skinny<CF<128>>(maps, args, grid, stream);
    default: return launch_skinny<CF<256>>(maps, args, grid, stream);
  }
}

// Tensor map over an E4M3 code matrix [rows, cols] for the raw-code ring,
// unswizzled: K-major (contraction along cols) boxes are 128 rows x 64 codes;
// MN-major (contraction along rows) boxes are 64 rows x 128 codes.
bool codes_tmap(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t cols, bool mn_major) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, codes, static_cast<uint64_t>(cols),
                      static_cast<uint64_t>(rows), mn_major ? 128 : 64, mn_major ? 64 : 128, false);
}

}  // namespace

// Workspace: T_hi, T_lo, U_hi, U_lo, each bf16 [M, r].  T and U are carried
// as bf16 hi/lo pairs (about 16 significant bits): a single bf16 rounding of
// T would move small dB entries by more than one bf16 ulp of the tensor's
// scale.  The split-K sums never leave the chip (cluster reduction).
size_t adapter_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, bool want_da) {
  (void)N;
  (void)K;
  (void)want_da;
  const size_t tu = align_up(static_cast<size_t>(M) * r * 2, 256);
  return 4 * tu;
}

cudaError_t launch_adapter_grads(const uint8_t* dyq, const float* s_dy, const uint8_t* xq,
                                 const float* s_x, const void* A, const void* B, int64_t M,
                                 int64_t N, int64_t K, int64_t r, void* dA, void* dB,
                                 int32_t* dev_status, void* workspace, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t tu = align_up(static_cast<size_t>(M) * r * 2, 256);
  void* T_hi = ws;
  void* T_lo = ws + tu;
  void* U_hi = ws + 2 * tu;
  void* U_lo = ws + 3 * tu;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int bn = skinny_bn(r);
  const uint32_t bn_box = static_cast<uint32_t>(bn);

  // stage 1: T = Xq . A^T / s_x (for dB) and U = dYq . B / s_dy (for dA), one grid
  Product t{}, u{};
  if (dB) {
    t.rows_out = M; t.kc = K; t.out = T_hi; t.out_lo = T_lo; t.ldo = r;
    t.transpose = false; t.b_mn = false; t.scale = s_x;
    if (!codes_tmap(&t.raw, xq, M, K, false) || !make_tmap_2d(&t.b, BF, 2, A, K, r, 64, bn_box, true))
      return cudaErrorInvalidValue;
    t.b2 = t.b;
  }
  if (dA) {
    u.rows_out = M; u.kc = N; u.out = U_hi; u.out_lo = U_lo; u.ldo = r;
    u.transpose = false; u.b_mn = true; u.scale = s_dy;
    if (!codes_tmap(&u.raw, dyq, M, N, false) || !make_tmap_2d(&u.b, BF, 2, B, r, N, 64, 64, true))
      return cudaErrorInvalidValue;
    u.b2 = u.b;
  }
  cudaError_t e;
  if (dB && dA) e = run_products<KCfg>(&t, &u, r, di, dev_status, stream);
  else e = run_products<KCfg>(dB ? &t : &u, nullptr, r, di, dev_status, stream);
  if (e != cudaSuccess) return e;

  // stage 2: dB = dYq^T . (T_hi + T_lo) / s_dy and dA^T = Xq^T . (U_hi + U_lo) / s_x
  Product db{}, da{};
  if (dB) {
    db.rows_out = N; db.kc = M; db.out = dB; db.out_lo = nullptr; db.ldo = r;
    db.transpose = false; db.b_mn = true; db.scale = s_dy;
    if (!codes_tmap(&db.raw, dyq, M, N, true) || !make_tmap_2d(&db.b, BF, 2, T_hi, r, M, 64, 64, true) ||
        !make_tmap_2d(&db.b2, BF, 2, T_lo, r, M, 64, 64, true))
      return cudaErrorInvalidValue;
  }
  if (dA) {
    // stored transposed into dA [r, K]
    da.rows_out = K; da.kc = M; da.out = dA; da.out_lo = nullptr; da.ldo = K;
    da.transpose = true; da.b_mn = true; da.scale = s_x;
    if (!codes_tmap(&da.raw, xq, M, K, true) || !make_tmap_2d(&da.b, BF, 2, U_hi, r, M, 64, 64, true) ||
        !make_tmap_2d(&da.b2, BF, 2, U_lo, r, M, 64, 64, true))
      return cudaErrorInvalidValue;
  }
  if (dB && dA) return run_products<MCfg>(&db, &da, r, di, dev_status, stream);
  return run_products<MCfg>(dB ? &db : &da, nullptr, r, di, dev_status, stream);
}

}  // namespace falqon
