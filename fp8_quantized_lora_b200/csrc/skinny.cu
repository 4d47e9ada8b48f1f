// Rank-r adapter products of the melded FP8 linear backward (sm_100a).
//
// FALQON, OpenReview rebuttal (reviewer 4, Q1): B's gradient comes from the
// precomputable product A x, and A's from B^T dL/dO; both reuse the E4M3
// codes the quantize step produced.  Every product puts the small rank
// dimension on the UMMA M side and 256 tokens or features on the N side, so
// one 128 x 256 x 16 MMA does the most work a single instruction can:
//   T^T  = A . Xq^T / s_X          [r, M]  A-op A [r, K] K-major,  B-op Xq codes K-major
//   U^T  = B^T . dYq^T / s_dY      [r, M]  A-op B [N, r] MN-major, B-op dYq codes K-major
//   dB^T = (T_hi + T_lo)^T . dYq / s_dY   [r, N]  A-op T^T hi over lo, B-op dYq codes MN-major
//   dA   = (U_hi + U_lo)^T . Xq / s_X     [r, K]  A-op U^T hi over lo, B-op Xq codes MN-major
// T and U are kept as bf16 hi/lo pairs, stored transposed ([r, M]).  In dB
// and dA the hi and lo operands fill the upper and lower 64 rows of one
// M = 128 tile; each CTA adds the two halves of its fp32 tile before the
// cluster sums its split-K partners.
//
// The E4M3 codes are expanded exactly to bf16 in shared memory (every E4M3
// value is a bf16 value) and fed to tcgen05 kind::f16 as the B operand.  One
// launch runs two independent products (T with U, then dB with dA): the first
// `ctas0` CTAs work on problem 0, the rest on problem 1.  Each CTA owns one
// (rank tile, column tile, K split) work item; the `splits` CTAs of an output
// tile form one cluster and sum their fp32 tiles through DSMEM in rank order
// (deterministic).
//
// Two warps issue MMAs, on alternate pairs of K blocks, into two TMEM
// accumulators: a warp that waits on a barrier stalls its own MMA stream, and
// the other warp's keeps the tensor pipe busy meanwhile.  The epilogue adds
// the two accumulators in a fixed order.
//
// Roles per CTA:
//   warp 0       TMA producer for the bf16 A operand (one lane)
//   warp 1       TMEM owner; MMA issuer for even K-block pairs (one lane)
//   warps 2-5    idle until the drain
// After the last MMA all 16 warps drain TMEM into an fp32 tile in shared
// memory (warp w: lane quarter w % 4, 64-column slice w / 4).
//   warps 6-13   converters: raw E4M3 tile -> bf16, 128-byte-swizzled
//   warp 14      TMA producer for the raw E4M3 tiles (one lane)
//   warp 15      MMA issuer for odd K-block pairs (one lane)
#include "internal.h"
#include "tc_common.cuh"

namespace falqon {
namespace {

constexpr int kSkN = 256;  // UMMA N: tokens or features per tile
constexpr int kSkK = 64;   // bf16 K per stage (one 128-byte swizzle row)

struct SkinnyProblem {
  int32_t m_tiles, n_tiles, splits, kb_total, kb_per_split;
  int64_t rows;        // r: ranks (output rows before any transpose)
  int64_t cols;        // tokens or features (output columns before any transpose)
  void* out;           // bf16 [rows][ldo], or [cols][ldo] when transposed
  void* out_lo;        // optional low half of a hi/lo pair
  int64_t ldo;
  int transpose;       // store out[col * ldo + row]
  int a_mn;            // the A operand is MN-major (B for U^T) instead of K-major
  int hilo;            // A rows [0, 64) hi and [64, 128) lo of the same ranks: add the halves
  int code_e5;         // the codes are E5M2 (dY of E5M2 gradients) instead of E4M3
  const float* scale;  // alpha = 1 / *scale
};

struct SkinnyArgs {
  SkinnyProblem p[2];
  int ctas0;           // CTAs of problem 0; the rest work on problem 1
  int32_t* dev_status;
};

template <bool kBMn, int kStages, int kRawStages>
struct SkCfg {
  static constexpr bool BMn = kBMn;  // codes are the MN-major B operand (dB^T, dA)
  static constexpr int S = kStages, SR = kRawStages;
  static constexpr int KSteps = kSkK / 16;                // UMMA K = 16
  static constexpr int ABytes = kBM * kSkK * 2;           // bf16 A tile, 16 KB
  static constexpr int BBytes = kSkN * kSkK * 2;          // expanded B tile, 32 KB
  static constexpr int StageBytes = ABytes + BBytes;
  static constexpr int RawBytes = kSkN * kSkK;            // raw codes, 16 KB
  static constexpr int RawRowBytes = kBMn ? kSkN : kSkK;  // row length of the raw box
  static constexpr int ConvWarps = 8;
  static constexpr int ChunksPerThread = RawBytes / 16 / (32 * ConvWarps);  // 4
  static constexpr int RawWarp = 6 + ConvWarps;
  static constexpr int Mma2Warp = RawWarp + 1;
  static constexpr int Threads = 32 * (Mma2Warp + 1);     // 512
  static constexpr uint32_t TmemCols = 2 * kSkN;          // two accumulators
  static constexpr int Ring = kStages * StageBytes, RawRing = kRawStages * RawBytes;
  static constexpr int BarBytes = 8 * (2 * kStages + 2 * kRawStages + 5) + 16;
  static constexpr int SmemBytes = Ring + RawRing + BarBytes + 1024;
  static constexpr int RedStride = kSkN + 4;   // [rank][col] reduction tile, fp32 words per row
  static constexpr int RedStrideT = kBM + 4;   // [col][rank] reduction tile (transposed outputs)
  static_assert(kBM * RedStride * 4 <= Ring && kSkN * RedStrideT * 4 <= Ring, "reduction tile");
  static_assert(ChunksPerThread * 16 * 32 * ConvWarps == RawBytes, "chunks per converter");
  static_assert(kStages >= 2 && kRawStages >= 2, "ring depths");
  // pconv[m] may not complete a pair's phase before its issuer saw the previous
  // one: the converters' last stage of pair p + 2 must reuse a slot of pair p
  static_assert(kStages <= 4, "pair barriers");
  static_assert(SmemBytes <= 232448, "shared memory per CTA");
};

template <class C>
__global__ void __launch_bounds__(C::Threads, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap raw0, const __grid_constant__ CUtensorMap a0,
                  const __grid_constant__ CUtensorMap a20, const __grid_constant__ CUtensorMap raw1,
                  const __grid_constant__ CUtensorMap a1, const __grid_constant__ CUtensorMap a21,
                  const SkinnyArgs args) {
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;                                   // stages of [A 16 KB][B 32 KB]
  uint8_t* raw_ring = smem + C::Ring;                     // raw E4M3 tiles (TMA)
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw_ring + C::RawRing);
  uint64_t* full = bars;                                  // [S] A landed
  uint64_t* empty = full + C::S;                          // [S] MMAs done with the stage
  uint64_t* pconv = empty + C::S;                         // [2] a pair of stages ready, per issuer
  uint64_t* rawfull = pconv + 2;                          // [SR] raw codes landed
  uint64_t* rawempty = rawfull + C::SR;                   // [SR] converters done reading
  uint64_t* acc_full = rawempty + C::SR;                  // both accumulators complete
  uint64_t* drain = acc_full + 1;                         // [2] each issuer's MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool second = static_cast<int>(blockIdx.x) >= args.ctas0;
  const SkinnyProblem& g = args.p[second ? 1 : 0];
  const CUtensorMap* tmRaw = second ? &raw1 : &raw0;
  const CUtensorMap* tmA = second ? &a1 : &a0;
  const CUtensorMap* tmA2 = second ? &a21 : &a20;
  const int w = static_cast<int>(blockIdx.x) - (second ? args.ctas0 : 0);  // work item
  const int split = w % g.splits;
  const int nt = (w / g.splits) % g.n_tiles;
  const int mt = w / (g.splits * g.n_tiles);
  const int kb0 = split * g.kb_per_split;
  const int nkb = max(0, min(g.kb_total, kb0 + g.kb_per_split) - kb0);
  const int npairs = (nkb + 1) / 2;
  const bool a_mn = g.a_mn != 0;
  const bool hilo = g.hilo != 0;
  const bool e5 = g.code_e5 != 0;
  const int row_span = hilo ? 64 : kBM;  // ranks per tile
  const int i0 = mt * row_span;
  const int n0 = nt * kSkN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&pconv[0], C::ConvWarps);
    mbar_init(&pconv[1], C::ConvWarps);
    for (int s = 0; s < C::SR; ++s) {
      mbar_init(&rawfull[s], 1);
      mbar_init(&rawempty[s], C::ConvWarps);
    }
    mbar_init(acc_full, 2);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(tmRaw);
    tma_prefetch_desc(tmA);
    if (hilo) tma_prefetch_desc(tmA2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();  // the next kernel may start launching; it waits for this one
  pdl_wait();     // the previous kernel's results are complete and visible

  auto fail = [&]() {
    *abort_flag = 1;
    raise_status(args.dev_status, kDevTimeout);
  };
  // one producer lane: waits `emp`, then fills `ful` with `load(slot, k-block)`
  auto produce = [&](uint64_t* ful, uint64_t* emp, int depth, uint32_t bytes, auto load) {
    int s = 0;
    uint32_t ph = 0, issued = 0, issued_parity = 0;
    for (int i = 0; i < nkb; ++i) {
      if (!mbar_wait(&emp[s], ph ^ 1, abort_flag)) { fail(); break; }
      mbar_arrive_expect_tx(&ful[s], bytes);
      issued |= 1u << s;
      issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
      load(s, kb0 + i);
      if (++s == depth) { s = 0; ph ^= 1; }
    }
    // every load issued must land before shared memory is reused or released
    for (int t = 0; t < depth; ++t)
      if (issued & (1u << t)) mbar_wait_budget(&ful[t], (issued_parity >> t) & 1u);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ A producer
    if (lane == 0) {
      produce(full, empty, C::S, static_cast<uint32_t>(C::ABytes), [&](int s, int kb) {
        uint8_t* sA = ring + s * C::StageBytes;
        const int k0 = kb * kSkK;
        if (hilo) {
          // ranks i0 .. +64 of the hi operand in rows 0-63, of the lo operand in rows 64-127
          tma_load_2d(sA, tmA, &full[s], k0, i0);
          tma_load_2d(sA + 64 * kRowBytes, tmA2, &full[s], k0, i0);
        } else if (a_mn) {
          // [K rows][ranks] row-major: two 128-byte column blocks of 64 ranks
          tma_load_2d(sA, tmA, &full[s], i0, k0);
          tma_load_2d(sA + kSkK * kRowBytes, tmA, &full[s], i0 + 64, k0);
        } else {
          tma_load_2d(sA, tmA, &full[s], k0, i0);
        }
      });
    }
    __syncwarp();
  } else if (warp == C::RawWarp) {
    // ------------------------------------------------------------ raw-code producer
    // K-major codes[n0 .. +256][kb*64 .. +64]; MN-major codes[kb*64 .. +64][n0 .. +256]
    if (lane == 0) {
      produce(rawfull, rawempty, C::SR, static_cast<uint32_t>(C::RawBytes), [&](int s, int kb) {
        if constexpr (C::BMn)
          tma_load_2d(raw_ring + s * C::RawBytes, tmRaw, &rawfull[s], n0, kb * kSkK);
        else
          tma_load_2d(raw_ring + s * C::RawBytes, tmRaw, &rawfull[s], kb * kSkK, n0);
      });
    }
    __syncwarp();
  } else if (warp == 1 || warp == C::Mma2Warp) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer m takes K-block pairs m, m + 2, ... into accumulator m, and
    // waits once per pair on its own barrier pconv[m], whose phases it sees
    // one by one: the converters arrive there when both stages of the pair
    // are expanded and both A tiles have landed.  (A wait on a per-stage
    // barrier could not tell its phases apart here: the issuer that did not
    // see a stage's previous use may find it two phases behind.)
    const int m = warp == 1 ? 0 : 1;
    const uint32_t idesc = idesc_f32acc(1u, 1u, a_mn ? 1u : 0u, C::BMn ? 1u : 0u, kBM, kSkN);
    const uint32_t acc = tmem_base + static_cast<uint32_t>(m * kSkN);
    bool ok = true;
    tc_fence_after();
    for (int p = m; p < npairs; p += 2) {
      const int i_first = 2 * p;
      const int i_last = min(2 * p + 1, nkb - 1);
      if (!warp_wait(&pconv[m], static_cast<uint32_t>((p >> 1) & 1), abort_flag)) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        for (int i = i_first; i <= i_last; ++i) {
          const int s = i % C::S;
          const uint32_t a_base = smem_u32(ring + s * C::StageBytes);
          const uint32_t b_base = a_base + C::ABytes;
#pragma unroll
          for (int ks = 0; ks < C::KSteps; ++ks)
            umma_bf16(acc, operand_desc_rt<2, kSkK>(a_mn, a_base, ks),
                      operand_desc_rt<2, kSkK>(C::BMn, b_base, ks), idesc,
                      (p > m || i > i_first || ks > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
      }
      __syncwarp();
    }
    if (lane == 0) {
      if (ok) umma_commit(acc_full);
      umma_commit(&drain[m]);
      mbar_wait_budget(&drain[m], 0);
    }
    __syncwarp();
  } else if (warp < 6) {
    // epilogue warps: they join the drain below with every other warp
  } else {
    // ------------------------------------------------------------ converters
    // 256 threads; each expands four 16-byte chunks (64 codes) of every tile:
    //   K-major  raw [256 rows][64 codes]:  rows t/4 + 64j,  codes (t % 4) * 16 ..
    //   MN-major raw [64 rows][256 codes]:  rows t/16 + 16j, codes (t % 16) * 16 ..
    // into the 128-byte-swizzled bf16 tile (MN-major: four 64-column blocks).
    constexpr int kThrPerRow = C::RawRowBytes / 16;
    constexpr int kRowStep = 256 / kThrPerRow;
    constexpr int kBlkBytes = (C::BMn ? kSkK : kSkN) * kRowBytes;  // one 128-byte column block
    const int t = threadIdx.x - 6 * 32;
    const int trow = t / kThrPerRow;
    const int tcol = (t % kThrPerRow) * 16;
    const int blk = tcol / 64;
    const int unit0 = (tcol % 64) / 8;
    for (int i = 0; i < nkb; ++i) {
      const int sr = i % C::SR, s = i % C::S;
      if (!warp_wait(&rawfull[sr], static_cast<uint32_t>((i / C::SR) & 1), abort_flag)) {
        if (lane == 0) fail();
        break;
      }
      uint4 q[C::ChunksPerThread];
#pragma unroll
      for (int j = 0; j < C::ChunksPerThread; ++j)
        q[j] = *reinterpret_cast<const uint4*>(raw_ring + sr * C::RawBytes +
                                               (trow + j * kRowStep) * C::RawRowBytes + tcol);
      __syncwarp();
      if (lane == 0) mbar_arrive(&rawempty[sr]);
      // codes the bit placement cannot take (E4M3 NaN; E5M2 infinity / NaN)
      // send the batch through the hardware conversion
      uint32_t nan_acc = 0u;
#pragma unroll
      for (int j = 0; j < C::ChunksPerThread; ++j)
        nan_acc = e5 ? special5_fold(nan_acc, q[j]) : nan_fold(nan_acc, q[j]);
      const bool nan = nan_found(nan_acc);
      if (!warp_wait(&empty[s], static_cast<uint32_t>(((i / C::S) & 1) ^ 1), abort_flag)) {
        if (lane == 0) fail();
        break;
      }
      uint8_t* sB = ring + s * C::StageBytes + C::ABytes + blk * kBlkBytes;
      // MN-major tiles: the 16 lanes of a half-warp share one row and cover
      // four column blocks; odd blocks store their two 16-byte units in the
      // other order, so that each store instruction meets every bank pair twice
      const int swap = C::BMn ? (blk & 1) : 0;
#pragma unroll
      for (int j = 0; j < C::ChunksPerThread; ++j) {
        uint32_t o[8];
        if (e5) e5m2x16_to_bf16(q[j], nan, o);
        else e4m3x16_to_bf16(q[j], nan, o);
        const int row = trow + j * kRowStep;
        const uint4 lo = make_uint4(o[0], o[1], o[2], o[3]), hi = make_uint4(o[4], o[5], o[6], o[7]);
        *reinterpret_cast<uint4*>(sB + row * kRowBytes + (((unit0 + swap) ^ (row & 7)) << 4)) = swap ? hi : lo;
        *reinterpret_cast<uint4*>(sB + row * kRowBytes + (((unit0 + 1 - swap) ^ (row & 7)) << 4)) = swap ? lo : hi;
      }
      fence_proxy_async_smem();
      // the stage's A tile must have landed too: pconv[] then covers both operands
      if (!warp_wait(&full[s], static_cast<uint32_t>((i / C::S) & 1), abort_flag)) {
        if (lane == 0) fail();
        break;
      }
      __syncwarp();
      // K blocks 2p and 2p + 1 form pair p, issued from accumulator p % 2's warp
      if (lane == 0 && ((i & 1) || i == nkb - 1)) mbar_arrive(&pconv[(i >> 1) & 1]);
    }
  }

  // ---------------------------------------------------------------- drain
  // acc0 + acc1 -> fp32 reduction tile in shared memory (the ring is idle once
  // every MMA has completed), by all 16 warps: warp w reads TMEM lane quarter
  // w % 4 and the 64 columns of slice w / 4.  [rank][col] for row-major
  // outputs, [col][rank] for transposed ones, so that the reduction reads
  // float4 along the output's contiguous dimension.
  __syncwarp();
  {
    const int q = warp & 3, slice = warp >> 2;
    if (warp_wait(acc_full, 0, abort_flag)) {
      tc_fence_after();
      const int row = q * 32 + lane;
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      float* red = reinterpret_cast<float*>(smem);
#pragma unroll 1
      for (int c = slice * 4; c < slice * 4 + 4; ++c) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          if (npairs > a) {
            uint32_t r[16];
            tmem_ld_16cols(lane_base + a * kSkN + c * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += __uint_as_float(r[j]);
          }
        }
        if (g.transpose) {
#pragma unroll
          for (int j = 0; j < 16; ++j) red[(c * 16 + j) * C::RedStrideT + row] = v[j];
        } else {
          float4* dst = reinterpret_cast<float4*>(red + row * C::RedStride + c * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
    } else if (lane == 0) {
      fail();
    }
    tc_fence_before();
  }
  __syncthreads();
  if (hilo) {
    // the lo operand's rows (64 .. 127) onto the hi operand's (0 .. 63), in
    // this CTA: the cluster then sums one 64-rank tile per CTA
    float* red = reinterpret_cast<float*>(smem);
    const bool tr = g.transpose != 0;
    for (int e = static_cast<int>(threadIdx.x); e < 64 * (kSkN / 4); e += blockDim.x) {
      // 4096 float4 groups either way: [col][rank] 256 columns x 16 groups of
      // four hi ranks; [rank][col] 64 hi ranks x 64 groups of four columns
      float* h = tr ? red + (e / 16) * C::RedStrideT + 4 * (e % 16)
                    : red + (e / (kSkN / 4)) * C::RedStride + 4 * (e % (kSkN / 4));
      const float* l = h + (tr ? 64 : 64 * C::RedStride);
      float4 x = *reinterpret_cast<float4*>(h);
      const float4 y = *reinterpret_cast<const float4*>(l);
      x.x += y.x;
      x.y += y.y;
      x.z += y.z;
      x.w += y.w;
      *reinterpret_cast<float4*>(h) = x;
    }
  }

  // ---------------------------------------------------------------- split-K reduction
  // The cluster's tiles are summed in rank order over a flat range of float4
  // groups (this CTA owns one slice), scaled by 1/s and written as bf16 (or
  // hi/lo pairs).  Each thread issues the peer loads of both its groups
  // before it sums either.
  __syncthreads();
  cluster_sync_all();
  {
    const int S = g.splits;
    const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
    const int nvalid = static_cast<int>(g.rows - i0 < row_span ? g.rows - i0 : row_span);  // ranks, % 4 == 0
    const bool tr = g.transpose != 0;
    const int ng = tr ? nvalid / 4 : kSkN / 4;  // float4 groups along the contiguous dimension
    const int total = tr ? kSkN * ng : nvalid * ng;
    const int chunk = (total + S - 1) / S;
    const int e_begin = static_cast<int>(rank) * chunk;
    const int e_end = min(total, e_begin + chunk);
    const float* red = reinterpret_cast<const float*>(smem);
    uint32_t peer[kMaxSplits];
#pragma unroll
    for (int sidx = 0; sidx < kMaxSplits; ++sidx) peer[sidx] = dsmem_addr(red, sidx < S ? sidx : 0);
    const float alpha = g.scale ? static_cast<float>(1.0 / static_cast<double>(*g.scale)) : 1.0f;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
    __nv_bfloat16* out_lo = static_cast<__nv_bfloat16*>(g.out_lo);
    for (int e0 = e_begin + static_cast<int>(threadIdx.x); e0 < e_end; e0 += 2 * blockDim.x) {
      float4 part[2][kMaxSplits];
      int64_t gcol[2];
      bool live[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = e0 + u * static_cast<int>(blockDim.x);
        const int major = e / ng, lg = e % ng;  // tr: (col, rank group); else (rank, col group)
        gcol[u] = n0 + (tr ? major : 4 * lg);
        live[u] = e < e_end && gcol[u] < g.cols;  // row-major outputs: ldo covers the whole group
        const uint32_t off = static_cast<uint32_t>(
            (tr ? major * C::RedStrideT + 4 * lg : major * C::RedStride + 4 * lg) * 4);
#pragma unroll
        for (int sidx = 0; sidx < kMaxSplits; ++sidx)
          if (live[u] && sidx < S) part[u][sidx] = dsmem_load_f32x4(peer[sidx] + off);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (!live[u]) continue;
        const int e = e0 + u * static_cast<int>(blockDim.x);
        const int major = e / ng, lg = e % ng;
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int sidx = 0; sidx < kMaxSplits; ++sidx) {  // fixed order: rank 0, 1, ...
          if (sidx < S) {
            acc.x += part[u][sidx].x;
            acc.y += part[u][sidx].y;
            acc.z += part[u][sidx].z;
            acc.w += part[u][sidx].w;
          }
        }
        const float vals[4] = {acc.x * alpha, acc.y * alpha, acc.z * alpha, acc.w * alpha};
        __nv_bfloat16 hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          hi[k] = __float2bfloat16_rn(vals[k]);
          lo[k] = __float2bfloat16_rn(vals[k] - __bfloat162float(hi[k]));
        }
        const int64_t o = tr ? gcol[u] * g.ldo + i0 + 4 * lg : static_cast<int64_t>(i0 + major) * g.ldo + gcol[u];
        uint2 ph, pl;
        memcpy(&ph, hi, 8);
        memcpy(&pl, lo, 8);
        *reinterpret_cast<uint2*>(out + o) = ph;
        if (out_lo) *reinterpret_cast<uint2*>(out_lo + o) = pl;
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
// Stages of [A 16 KB | expanded codes 32 KB] and a deeper ring of 16 KB raw
// code tiles, which carries the HBM latency more cheaply.
using KCfg = SkCfg<false, 3, 4>;  // T^T, U^T: codes are the K-major operand
using MCfg = SkCfg<true, 3, 4>;   // dB^T, dA: codes are the MN-major operand

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
  return launch_pdl(skinny_kernel<C>, dim3(static_cast<unsigned>(grid)), dim3(C::Threads), C::SmemBytes,
                    stream, static_cast<unsigned>(args.p[0].splits), maps[0], maps[1], maps[2], maps[3],
                    maps[4], maps[5], args);
}

// One product: out (r x cols, or its transpose) = A-op . codes, contraction kc.
struct Product {
  int64_t cols, kc;
  void* out;
  void* out_lo;
  int64_t ldo;
  bool transpose, a_mn, hilo, code_e5;
  const float* scale;
  CUtensorMap raw, a, a2;
};

// Launches one or two products (the second may be null) as one grid.
template <class C>
cudaError_t run_products(const Product* p0, const Product* p1, int64_t r, const DeviceInfo* di,
                         int32_t* dev_status, cudaStream_t stream) {
  const Product* ps[2] = {p0, p1};
  int tiles[2] = {0, 0}, kbt[2] = {0, 0};
  for (int i = 0; i < 2; ++i) {
    if (!ps[i]) continue;
    tiles[i] = ceil_div(r, ps[i]->hilo ? 64 : kBM) * ceil_div(ps[i]->cols, kSkN);
    kbt[i] = ceil_div(ps[i]->kc, kSkK);
  }
  // one split count for the whole grid (the cluster size is per launch)
  const int kb_min = p1 ? std::min(kbt[0], kbt[1]) : kbt[0];
  const int splits = choose_splits(tiles[0] + tiles[1], kb_min, di->sm_count);
  SkinnyArgs args{};
  args.dev_status = dev_status;
  CUtensorMap maps[6];
  for (int i = 0; i < 2; ++i) {
    const Product* p = ps[i] ? ps[i] : ps[0];
    SkinnyProblem& q = args.p[i];
    q.m_tiles = ceil_div(r, p->hilo ? 64 : kBM);
    q.n_tiles = ceil_div(p->cols, kSkN);
    q.splits = splits;
    q.kb_total = ceil_div(p->kc, kSkK);
    q.kb_per_split = ceil_div(q.kb_total, splits);
    q.rows = r;
    q.cols = p->cols;
    q.out = p->out;
    q.out_lo = p->out_lo;
    q.ldo = p->ldo;
    q.transpose = p->transpose ? 1 : 0;
    q.a_mn = p->a_mn ? 1 : 0;
    q.hilo = p->hilo ? 1 : 0;
    q.code_e5 = p->code_e5 ? 1 : 0;
    q.scale = p->scale;
    maps[3 * i] = p->raw;
    maps[3 * i + 1] = p->a;
    maps[3 * i + 2] = p->a2;
  }
  args.ctas0 = args.p[0].m_tiles * args.p[0].n_tiles * splits;
  const int grid = args.ctas0 + (p1 ? args.p[1].m_tiles * args.p[1].n_tiles * splits : 0);
  return launch_skinny<C>(maps, args, grid, stream);
}

// Tensor map over an E4M3 code matrix [rows, cols] for the raw-code ring,
// unswizzled: K-major (contraction along cols) boxes are 256 rows x 64 codes;
// MN-major (contraction along rows) boxes are 64 rows x 256 codes.
bool codes_tmap(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t cols, bool mn_major) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, codes, static_cast<uint64_t>(cols),
                      static_cast<uint64_t>(rows), mn_major ? kSkN : kSkK, mn_major ? kSkK : kSkN, false);
}

// Row stride (elements) of the transposed T / U workspace: M rounded up so
// that rows start 16-byte aligned.
int64_t tu_ld(int64_t M) { return adapter_tu_ld(M); }

}  // namespace

// Workspace: T_hi^T, T_lo^T, U_hi^T, U_lo^T, each bf16 [r, M] (rows padded to
// a multiple of 8 elements).  T and U are carried as bf16 hi/lo pairs (about
// 16 significant bits): a single bf16 rounding of T would move small dB
// entries by more than one bf16 ulp of the tensor's scale.  The split-K sums
// never leave the chip (cluster reduction).
size_t adapter_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, bool want_da) {
  (void)want_da;
  if (adapter_gemm_path(M, r)) return adapter_gemm_workspace_bytes(M, N, K, r);
  const size_t tu = align_up(static_cast<size_t>(tu_ld(M)) * r * 2, 256);
  return 4 * tu;
}

cudaError_t launch_adapter_grads(const uint8_t* dyq, const float* s_dy, const uint8_t* xq,
                                 const float* s_x, const void* A, const void* B, int64_t M,
                                 int64_t N, int64_t K, int64_t r, void* dA, void* dB,
                                 int32_t* dev_status, void* workspace, cudaStream_t stream, bool dy_e5m2) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  // past a few hundred ranks the rank-on-M kernel below would expand every
  // code r / 128 times: the products run as plain bf16 GEMMs instead
  if (adapter_gemm_path(M, r))
    return launch_adapter_grads_gemm(dyq, s_dy, xq, s_x, A, B, M, N, K, r, dA, dB, dev_status, workspace, stream,
                                     dy_e5m2);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t ld = tu_ld(M);
  const size_t tu = align_up(static_cast<size_t>(ld) * r * 2, 256);
  void* T_hi = ws;
  void* T_lo = ws + tu;
  void* U_hi = ws + 2 * tu;
  void* U_lo = ws + 3 * tu;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

  // stage 1: T^T = A . Xq^T / s_x (for dB) and U^T = B^T . dYq^T / s_dy (for dA), one grid
  Product t{}, u{};
  if (dB) {
    t.cols = M; t.kc = K; t.out = T_hi; t.out_lo = T_lo; t.ldo = ld;
    t.transpose = false; t.a_mn = false; t.hilo = false; t.scale = s_x;
    if (!codes_tmap(&t.raw, xq, M, K, false) || !make_tmap_2d(&t.a, BF, 2, A, K, r, kSkK, kBM, true))
      return cudaErrorInvalidValue;
    t.a2 = t.a;
  }
  if (dA) {
    u.cols = M; u.kc = N; u.out = U_hi; u.out_lo = U_lo; u.ldo = ld;
    u.transpose = false; u.a_mn = true; u.hilo = false; u.code_e5 = dy_e5m2; u.scale = s_dy;
    if (!codes_tmap(&u.raw, dyq, M, N, false) || !make_tmap_2d(&u.a, BF, 2, B, r, N, 64, kSkK, true))
      return cudaErrorInvalidValue;
    u.a2 = u.a;
  }
  cudaError_t e;
  if (dB && dA) e = run_products<KCfg>(&t, &u, r, di, dev_status, stream);
  else e = run_products<KCfg>(dB ? &t : &u, nullptr, r, di, dev_status, stream);
  if (e != cudaSuccess) return e;
  return launch_adapter_stage2(dyq, s_dy, xq, s_x, T_hi, T_lo, U_hi, U_lo, ld, M, N, K, r, dA, dB, dev_status,
                               stream, dy_e5m2);
}

// Stage 2 on T and U given as transposed bf16 hi/lo planes [r][ld] (from
// stage 1 above, or from the folded FP8 GEMMs' adapter columns):
//   dB^T = (T_hi + T_lo)^T . dYq / s_dy, stored as dB [N, r]
//   dA   = (U_hi + U_lo)^T . Xq / s_x   [r, K]
cudaError_t launch_adapter_stage2(const uint8_t* dyq, const float* s_dy, const uint8_t* xq, const float* s_x,
                                  const void* T_hi, const void* T_lo, const void* U_hi, const void* U_lo,
                                  int64_t ld, int64_t M, int64_t N, int64_t K, int64_t r, void* dA, void* dB,
                                  int32_t* dev_status, cudaStream_t stream, bool dy_e5m2) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  if (!dA && !dB) return cudaSuccess;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  Product db{}, da{};
  if (dB) {
    db.cols = N; db.kc = M; db.out = dB; db.out_lo = nullptr; db.ldo = r;
    db.transpose = true; db.a_mn = false; db.hilo = true; db.code_e5 = dy_e5m2; db.scale = s_dy;
    if (!codes_tmap(&db.raw, dyq, M, N, true) ||
        !make_tmap_2d(&db.a, BF, 2, T_hi, M, r, kSkK, 64, true, ld) ||
        !make_tmap_2d(&db.a2, BF, 2, T_lo, M, r, kSkK, 64, true, ld))
      return cudaErrorInvalidValue;
  }
  if (dA) {
    da.cols = K; da.kc = M; da.out = dA; da.out_lo = nullptr; da.ldo = K;
    da.transpose = false; da.a_mn = false; da.hilo = true; da.scale = s_x;
    if (!codes_tmap(&da.raw, xq, M, K, true) ||
        !make_tmap_2d(&da.a, BF, 2, U_hi, M, r, kSkK, 64, true, ld) ||
        !make_tmap_2d(&da.a2, BF, 2, U_lo, M, r, kSkK, 64, true, ld))
      return cudaErrorInvalidValue;
  }
  if (dB && dA) return run_products<MCfg>(&db, &da, r, di, dev_status, stream);
  return run_products<MCfg>(dB ? &db : &da, nullptr, r, di, dev_status, stream);
}

}  // namespace falqon
