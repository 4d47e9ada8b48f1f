// tcgen05 FP8 GEMMs of the melded FP8 linear layer (sm_100a).
//
// One persistent, warp-specialised kernel template serves the two large
// products of the step:
//   forward    Y  = Xq  . Wq^T   / (s_X s_W)    kind::f8f6f4, A K-major, B K-major
//   dX         dX = dYq . Wq     / (s_dY s_W)   kind::f8f6f4, A K-major, B MN-major
// FALQON's point (paper introduction) is that both run on the FP8 backbone
// alone: the adapter is merged into Wq, so there is no separate LoRA path.
//
// Folded quantized adapters (the paper's Fig. 2 with quantized A~ and B~):
// the same kernel appends the adapter columns to either product,
//   [Y | T]  = Xq  . [Wq ; A~q]^T     T = Xq . A~q^T / (s_X s_A)
//   [dX | U] = dYq . [Wq | B~q]       U = dYq . B~q / (s_dY s_B)
// as a second B segment: output tiles past the backbone's read their B tile
// from a second tensor map (rows past r are zero-filled by TMA) and write
// their columns transposed, as a bf16 hi/lo pair [r][ld] (about 16
// significant bits), the layout the dB / dA products read.
//
// Roles (persistent over 128 x 256 output tiles; when the last wave would
// leave at least half the SMs idle, its tiles run as 128 x 128 halves):
//   warp 0      TMA producer (one lane): fills a `kStages`-deep smem ring.
//   warp 1      TMEM owner and UMMA issuer (one lane issues).
//   warps 2-5   epilogue: tcgen05.ld of the accumulator, scale, bf16 store.
//   warp 6      MMA waiter: waits on the stage and accumulator mbarriers and
//               releases the issuer through a named barrier.  An mbarrier
//               wait in the issuing thread holds back its MMA stream until
//               the MMAs in flight retire (measured: half the tensor rate
//               with a wait every 4 UMMAs); a named barrier does not.
// The accumulator lives in TMEM (kAcc buffers of BN fp32 columns); with two
// buffers the epilogue of one tile overlaps the MMAs of the next.  (Two CTAs
// per SM with a 2-stage ring and one accumulator each measured slower.)
//
// Every operand tile in smem is a stack of 128-byte rows in the SWIZZLE_128B
// layout TMA writes: K-major tiles are [rows][128 B of K]; MN-major tiles are
// 128-byte-wide column blocks of [K rows][128 B of N], LBO apart.
#include <algorithm>
#include <cfloat>

#include "internal.h"
#include "tc_common.cuh"

namespace falqon {
namespace {

constexpr int kMmaBar = 1;  // named barrier between the MMA issuer and its waiter

struct GemmArgs {
  int32_t m_tiles, n_tiles, kb_total;
  // Work items: items [0, n_full) are whole tiles (tile = item); the last
  // n_half items are the 128-column halves of the tiles n_full ..
  // n_full + n_half/2 - 1 (the partial last wave, split so that it takes
  // about half as long).  total = n_full + n_half.
  int32_t n_full, n_half;
  int32_t n_tiles0;        // tiles of the backbone segment; tiles nt >= n_tiles0 are the adapter's
  int64_t M, N;            // output extent of the backbone segment
  void* out;               // bf16 output, row-major [M][ldo]
  int64_t ldo;
  const float* scale_a;    // alpha = 1 / (scale_a * scale_b); either may be null (= 1)
  const float* scale_b;
  int64_t N2;              // adapter columns (r); 0 without an adapter segment
  void* out2_hi;           // adapter columns transposed: bf16 [N2][ld2], hi + lo = value
  void* out2_lo;
  int64_t ld2;
  const float* scale_b2;   // alpha2 = 1 / (scale_a * scale_b2)
  const void* addend;      // bf16 [M][ldo] added to the rounded product (nullable)
  int32_t f32_accumulate;  // out is float32 [M][ldo]: 1: out = fl32(out + alpha * product); 2: out = alpha * product
  // grouped launch (kMode 2): up to three B segments sharing A, each with its
  // own scale and row-major bf16 output; segment s owns the tiles from
  // seg_tile0[s] on (seg_tile0[nseg] = n_tiles)
  int32_t nseg;
  int32_t seg_tile0[4];
  void* seg_out[3];
  const float* seg_scale[3];
  int64_t seg_n[3];
  int32_t* dev_status;
};

template <bool kBMn, int kBN, int kStages, int kAcc, int kMinBlocks, int kHalves, int kAFmt = 0, bool kBf16 = false>
struct Cfg {
  static constexpr bool BMn = kBMn;
  static constexpr bool Bf16 = kBf16;                 // bf16 operands (kind::f16), else 8-bit codes
  static constexpr int ElemBytes = kBf16 ? 2 : 1;
  static constexpr int BN = kBN;
  static constexpr int Stages = kStages;
  static constexpr int Acc = kAcc;              // accumulator buffers in TMEM
  static constexpr int MinBlocks = kMinBlocks;  // CTAs per SM
  static constexpr int Halves = kHalves;        // 128-row halves of a tile (one MMA each per K step)
  static constexpr int TileM = kHalves * kBM;
  static constexpr int BK = kRowBytes / ElemBytes;    // K per stage: one 128-byte row (128 codes or 64 bf16)
  static constexpr int KSteps = kRowBytes / 32;       // UMMA K is 32 bytes of K (32 codes or 16 bf16)
  static constexpr int BNBlock = kRowBytes / ElemBytes;  // N elements of one MN-major 128-byte column block
  static constexpr int AHalfBytes = kBM * kRowBytes;  // 16 KB
  static constexpr int ABytes = kHalves * AHalfBytes;
  static constexpr int BBytes = kBN * kRowBytes;
  static constexpr int StageBytes = ABytes + BBytes;
  static constexpr int EpiWarps = 4 * kHalves;        // warps 2 .. 2 + EpiWarps - 1
  static constexpr int WaiterWarp = 2 + EpiWarps;
  static constexpr int Threads = 32 * (WaiterWarp + 1);
  // kAcc accumulators of Halves x BN columns; allocations are powers of two >= 32
  static constexpr int AccCols = kAcc * kHalves * kBN;
  static constexpr uint32_t TmemCols = AccCols <= 32 ? 32 : (AccCols <= 64 ? 64 : (AccCols <= 128 ? 128 : (AccCols <= 256 ? 256 : 512)));
  static constexpr int BarBytes = 8 * (2 * kStages + 2 * kAcc + 1) + 16;
  // float32-accumulate epilogue (bf16 configurations only): one 32 x 33 float
  // transpose buffer per epilogue warp, so that P moves in contiguous rows
  static constexpr int EpiStageBytes = kBf16 ? EpiWarps * 32 * 33 * 4 : 0;
  static constexpr int SmemBytes = kStages * StageBytes + BarBytes + EpiStageBytes + 1024;
  // 8-bit kinds: A in E4M3 (kAFmt 0) or E5M2 (1; the dX GEMM of E5M2 gradients), B in E4M3;
  // kind::f16: A and B bf16 (format 1)
  static constexpr uint32_t AFmt = kBf16 ? 1u : static_cast<uint32_t>(kAFmt);
  static constexpr uint32_t BFmt = kBf16 ? 1u : 0u;
  static constexpr uint32_t IDesc = idesc_f32acc(AFmt, BFmt, 0u, kBMn ? 1u : 0u, kBM, kBN);
  // a half tile: the first 128 columns of the B tile
  static constexpr int HalfN = 128;
  static constexpr uint32_t IDescHalf = idesc_f32acc(AFmt, BFmt, 0u, kBMn ? 1u : 0u, kBM, HalfN);
  static constexpr int HalfStageBytes = ABytes + BBytes / 2;
  static_assert(kBN % 16 == 0 && kBN >= 16 && kBN <= 256, "UMMA N");
  static_assert(!kBMn || kBN % BNBlock == 0, "MN-major B needs whole 128-byte blocks");
  static_assert(SmemBytes <= 232448, "shared memory per CTA");
  static_assert(kMinBlocks * (SmemBytes + 1024) <= 233472, "shared memory per SM");
  static_assert(kMinBlocks * TmemCols <= 512, "tensor memory per SM");
  static_assert(kAcc == 1 || kAcc == 2, "accumulator buffers");
  static_assert(kHalves == 1 || kHalves == 2, "tile halves");
  static_assert(AccCols <= 512, "tensor memory");
};

// kMode 0: a plain product.  1 (kSeg2): the grid also carries adapter tiles
// (a second B segment written transposed).  2 (kGroup): up to three B
// segments (tmB, tmB2, tmBh) share the A operand, each written row-major
// with its own scale.  The plain GEMMs are compiled without the other code.
template <class C, int kMode>
__global__ void __launch_bounds__(C::Threads, C::MinBlocks)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmBh,
                   const GemmArgs g) {
  constexpr bool kSeg2 = kMode == 1;
  constexpr bool kGroup = kMode == 2;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::Stages * C::StageBytes);
  uint64_t* full = bars;                      // [Stages] TMA landed
  uint64_t* empty = bars + C::Stages;         // [Stages] MMAs done with the slot
  uint64_t* acc_full = bars + 2 * C::Stages;  // [Acc] accumulator ready
  uint64_t* acc_empty = acc_full + C::Acc;    // [Acc] accumulator drained
  uint64_t* drain = acc_empty + C::Acc;       // all issued MMAs retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total = g.n_full + g.n_half;
  // work item -> (tile, column half): nh = -1 for a whole tile, else 0 or 1
  auto item = [&](int w, int& mt, int& nt, int& nh) {
    int t = w;
    nh = -1;
    if constexpr (kMode == 2) {
      // segment by segment (each segment's backbone stays in L2 while its
      // tiles run), row band by row band within a segment
      const int sg = w >= g.m_tiles * g.seg_tile0[2] ? 2 : (w >= g.m_tiles * g.seg_tile0[1] ? 1 : 0);
      const int nts = g.seg_tile0[sg + 1] - g.seg_tile0[sg];
      const int local = w - g.m_tiles * g.seg_tile0[sg];
      mt = local / nts;
      nt = g.seg_tile0[sg] + local % nts;
      return;
    }
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
      mbar_init(&acc_empty[b], C::EpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (kSeg2 || kGroup) tma_prefetch_desc(&tmB2);
    if (kGroup && g.nseg > 2) tma_prefetch_desc(&tmBh);
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
    raise_status(g.dev_status, kDevTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage: ever loaded / parity of last load
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        int mt, nt, nh;
        item(w, mt, nt, nh);
        const bool seg2 = kSeg2 && nt >= g.n_tiles0;  // an adapter tile
        const CUtensorMap* tb = seg2 ? &tmB2 : &tmB;
        int ntl = seg2 ? nt - g.n_tiles0 : nt;  // tile index within its segment
        if constexpr (kGroup) {
          const int sg = nt >= g.seg_tile0[2] ? 2 : (nt >= g.seg_tile0[1] ? 1 : 0);
          tb = sg == 0 ? &tmB : (sg == 1 ? &tmB2 : &tmBh);
          ntl = nt - g.seg_tile0[sg];
        }
        const int m0 = mt * C::TileM;
        const int n0 = ntl * C::BN + (nh > 0 ? C::HalfN : 0);
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { fail(); ok = false; break; }
          uint8_t* sA = smem + stage * C::StageBytes;
          uint8_t* sB = sA + C::ABytes;
          mbar_arrive_expect_tx(&full[stage], nh >= 0 ? C::HalfStageBytes : C::StageBytes);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
#pragma unroll
          for (int h = 0; h < C::Halves; ++h)  // rows m0 + 128 h .., K block kb
            tma_load_2d(sA + h * C::AHalfBytes, &tmA, &full[stage], kb * C::BK, m0 + h * kBM);
          if constexpr (C::BMn) {
            // B is [K][N] row-major: 128-byte column blocks of BK rows each (the first
            // 128 columns for a half tile)
            const int blocks = (nh >= 0 ? C::HalfN : C::BN) / C::BNBlock;
            for (int c = 0; c < blocks; ++c)
              tma_load_2d(sB + c * C::BK * kRowBytes, tb, &full[stage], n0 + c * C::BNBlock, kb * C::BK);
          } else {
            // a half tile loads 128 rows of B through the half-height box
            tma_load_2d(sB, nh >= 0 ? &tmBh : tb, &full[stage], kb * C::BK, n0);
          }
          if (++stage == C::Stages) { stage = 0; phase ^= 1; }
        }
      }
      // every load this lane issued must land before the CTA exits (matters
      // only after an abort; otherwise the MMA warp already consumed them)
      for (int s = 0; s < C::Stages; ++s)
        if (issued & (1u << s)) mbar_wait_budget(&full[s], (issued_parity >> s) & 1u);
    }
    __syncwarp();  // the warp reaches the CTA barrier below together
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Released by the waiter once per tile (accumulator free) and once per K
    // block (stage landed); the barrier's OR carries an abort, and both warps
    // leave their loops at the same point.
    int stage = 0;
    int acc = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      if (bar_red_or(kMmaBar, 64, false)) break;
      tc_fence_after();
      const uint32_t tmem_d = tmem_base + acc * C::Halves * C::BN;
      const uint32_t idesc = w >= g.n_full ? C::IDescHalf : C::IDesc;
      bool abort = false;
      for (int kb = 0; kb < g.kb_total; ++kb) {
        if (bar_red_or(kMmaBar, 64, false)) { abort = true; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_u32(smem + stage * C::StageBytes);
          const uint32_t b_base = a_base + C::ABytes;
#pragma unroll
          for (int ks = 0; ks < C::KSteps; ++ks) {
            const uint64_t bd = operand_desc<C::BMn, C::ElemBytes, C::BK>(b_base, ks);
#pragma unroll
            for (int h = 0; h < C::Halves; ++h) {  // the halves share the B tile
              const uint64_t ad = operand_desc<false, C::ElemBytes, C::BK>(a_base + h * C::AHalfBytes, ks);
              if constexpr (C::Bf16)
                umma_bf16(tmem_d + h * C::BN, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
              else
                umma_f8(tmem_d + h * C::BN, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::Stages) stage = 0;
      }
      if (abort) break;
      if (lane == 0) umma_commit(&acc_full[acc]);
      __syncwarp();
      if (++acc == C::Acc) acc = 0;
    }
    // drain the tensor pipe before TMEM is released
    if (lane == 0) {
      umma_commit(drain);
      mbar_wait_budget(drain, 0);
    }
    __syncwarp();
  } else if (warp == C::WaiterWarp) {
    // ------------------------------------------------------------ MMA waiter
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const bool ok_acc = warp_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag);
      if (!ok_acc && lane == 0) fail();
      __syncwarp();  // converged at the (aligned) named barrier
      if (bar_red_or(kMmaBar, 64, !ok_acc)) break;
      bool abort = false;
      for (int kb = 0; kb < g.kb_total; ++kb) {
        const bool ok = warp_wait(&full[stage], phase, abort_flag);
        if (!ok && lane == 0) fail();
        __syncwarp();
        if (bar_red_or(kMmaBar, 64, !ok)) { abort = true; break; }
        if (++stage == C::Stages) { stage = 0; phase ^= 1; }
      }
      if (abort) break;
      if (++acc == C::Acc) { acc = 0; acc_phase ^= 1; }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;  // 128-row half this warp drains
    float alpha = 1.0f, alpha2 = 1.0f;
    {
      const double sa = g.scale_a ? static_cast<double>(*g.scale_a) : 1.0;
      double den = sa;
      if (g.scale_b) den *= static_cast<double>(*g.scale_b);
      alpha = static_cast<float>(1.0 / den);
      if (kSeg2) {
        double den2 = sa;
        if (g.scale_b2) den2 *= static_cast<double>(*g.scale_b2);
        alpha2 = static_cast<float>(1.0 / den2);
      }
    }
    float seg_alpha[3] = {alpha, alpha, alpha};
    if constexpr (kGroup) {
      const double sa = g.scale_a ? static_cast<double>(*g.scale_a) : 1.0;
      for (int sg = 0; sg < g.nseg && sg < 3; ++sg)
        seg_alpha[sg] = static_cast<float>(1.0 / (g.seg_scale[sg] ? sa * static_cast<double>(*g.seg_scale[sg]) : sa));
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      int mt, nt, nh;
      item(w, mt, nt, nh);
      if (!warp_wait(&acc_full[acc], acc_phase, abort_flag)) { if (lane == 0) fail(); break; }
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mt) * C::TileM + half * kBM + q * 32 + lane;
      if (kSeg2 && nt >= g.n_tiles0) {
        // adapter columns: rank i of token `row` goes to out2[i][row]; the 32
        // lanes of a warp hold 32 consecutive tokens, so each store is 64 bytes
        const int64_t i0 = static_cast<int64_t>(nt - g.n_tiles0) * C::BN;
        __nv_bfloat16* hi_out = static_cast<__nv_bfloat16*>(g.out2_hi);
        __nv_bfloat16* lo_out = static_cast<__nv_bfloat16*>(g.out2_lo);
#pragma unroll 1
        for (int c = 0; c < C::BN / 32 && i0 + c * 32 < g.N2; ++c) {  // warp-uniform bound
          uint32_t r[32];
          tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (acc * C::Halves + half) * C::BN +
                             c * 32, r);
          tmem_ld_wait();
          if (row < g.M) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int64_t i = i0 + c * 32 + j;
              if (i < g.N2) {
                const float v = __uint_as_float(r[j]) * alpha2;
                const __nv_bfloat16 h = __float2bfloat16_rn(v);
                hi_out[i * g.ld2 + row] = h;
                lo_out[i * g.ld2 + row] = __float2bfloat16_rn(v - __bfloat162float(h));
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        if (++acc == C::Acc) { acc = 0; acc_phase ^= 1; }
        continue;
      }
      int64_t col_base = static_cast<int64_t>(nt) * C::BN + (nh > 0 ? C::HalfN : 0);
      void* out = g.out;
      int64_t ldo = g.ldo, ncols = g.N;
      float alpha_t = alpha;
      if constexpr (kGroup) {
        const int sg = nt >= g.seg_tile0[2] ? 2 : (nt >= g.seg_tile0[1] ? 1 : 0);
        col_base = static_cast<int64_t>(nt - g.seg_tile0[sg]) * C::BN;
        out = g.seg_out[sg];
        ldo = ncols = g.seg_n[sg];
        alpha_t = seg_alpha[sg];
      }
      const int chunks = (nh >= 0 ? C::HalfN : C::BN) / 32;
#pragma unroll 1
      for (int c = 0; c < chunks; ++c) {
        uint32_t r[32];
        tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (acc * C::Halves + half) * C::BN +
                           c * 32, r);
        tmem_ld_wait();
        if constexpr (C::EpiStageBytes > 0) {
          if (g.f32_accumulate) {
            // float32 output accumulated in place, out = fl32(out + alpha * D)
            // (or written, out = fl32(alpha * D), in mode 2).
            // Lane l holds row l of the warp's 32 rows; the 32 x 32 chunk goes
            // through shared memory so that every access below covers four
            // rows of 128 contiguous bytes.
            float* stg = reinterpret_cast<float*>(smem + C::Stages * C::StageBytes + C::BarBytes) +
                         (warp - 2) * (32 * 33);
#pragma unroll
            for (int j = 0; j < 32; ++j) stg[lane * 33 + j] = __fmul_rn(__uint_as_float(r[j]), alpha);
            __syncwarp();
            const int64_t row0 = row - lane;  // the warp's first row
            const int64_t col = col_base + c * 32 + 4 * (lane & 7);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int rr = 4 * it + (lane >> 3);
              const int64_t grow = row0 + rr;
              if (grow < g.M && col < g.N) {  // Ncols % 4 == 0: four columns in or out together
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out) + grow * g.ldo + col);
                float4 p = g.f32_accumulate == 2 ? make_float4(0.f, 0.f, 0.f, 0.f) : *dst;
                const float* src = stg + rr * 33 + 4 * (lane & 7);
                p.x = __fadd_rn(p.x, src[0]);
                p.y = __fadd_rn(p.y, src[1]);
                p.z = __fadd_rn(p.z, src[2]);
                p.w = __fadd_rn(p.w, src[3]);
                *dst = p;
              }
            }
            __syncwarp();  // the buffer is reused by the next chunk
            continue;
          }
        }
        if (row < g.M) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(out) + row * ldo;
          const __nv_bfloat16* add = g.addend ? static_cast<const __nv_bfloat16*>(g.addend) + row * ldo : nullptr;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int64_t col = col_base + c * 32 + 8 * j;
            if (col < ncols) {
              uint32_t pk[4];
              uint4 ad = make_uint4(0u, 0u, 0u, 0u);
              if (add) ad = *reinterpret_cast<const uint4*>(add + col);
              const uint32_t aw[4] = {ad.x, ad.y, ad.z, ad.w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 2 * h]) * alpha_t,
                                                         __uint_as_float(r[8 * j + 2 * h + 1]) * alpha_t);
                if (add) {
                  // the product rounded to bf16, then added as bf16 tensors add:
                  // a float32 sum rounded once to bf16
                  const float2 pf = __bfloat1622float2(b);
                  b = __floats2bfloat162_rn(__fadd_rn(pf.x, __uint_as_float(aw[h] << 16)),
                                            __fadd_rn(pf.y, __uint_as_float(aw[h] & 0xFFFF0000u)));
                }
                memcpy(&pk[h], &b, 4);
              }
              *reinterpret_cast<uint4*>(dst + col) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == C::Acc) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TmemCols);
  }
}

// ---------------------------------------------------------------- host side
template <class C, int kMode>
cudaError_t launch_gemm(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tB2, const CUtensorMap& tBh,
                        GemmArgs g, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  static int configured_mask = 0;  // one bit per device ordinal < 31
  const int bit = di->device < 31 ? (1 << di->device) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<C, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SmemBytes);
    if (e != cudaSuccess) return e;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_ACQ_REL);
  }
  const int tiles = g.m_tiles * g.n_tiles;
  const int slots = C::MinBlocks * di->sm_count;
  const int grid = tiles < slots ? tiles : slots;
  // A partial last wave of at most half the grid's width runs as half tiles
  // (twice as many items, each about half as long).  The adapter-tile
  // launches keep whole tiles.
  const int tail = tiles % grid;
  g.n_full = tiles;
  g.n_half = 0;
  if (kMode == 0 && C::BN == 2 * C::HalfN && tiles > grid && tail > 0 && 2 * tail <= grid) {
    g.n_full = tiles - tail;
    g.n_half = 2 * tail;
  }
  return launch_pdl(tc_gemm_kernel<C, kMode>, dim3(grid), dim3(C::Threads), C::SmemBytes, stream, 1u, tA, tB, tB2,
                    tBh, g);
}

// 128 x 256 tiles, 4-stage ring, double-buffered accumulator, one CTA per SM.
// Measured slower on the 4096-square product: 128 x 192 and 128 x 128 tiles
// (more L2 bytes per flop), 256 x 256 tiles (two MMAs per K step sharing B;
// 1.73 waves, no accumulator double buffer) and two CTAs per SM.
using FwdCfg = Cfg<false, 256, 4, 2, 1, 1>;
using DxCfg = Cfg<true, 256, 4, 2, 1, 1>;

// The adapter segment, when present: B2 (A~q [N2, Kc] K-major, or B~q
// [Kc, N2] MN-major) with scale sb2, written transposed to the hi/lo planes
// out2_hi / out2_lo [N2][ld2].  `out` may be null (no backbone segment: the
// grid then covers the adapter tiles alone).
struct Segment2 {
  const void* b = nullptr;
  const float* sb = nullptr;
  int64_t n = 0;
  void* hi = nullptr;
  void* lo = nullptr;
  int64_t ld = 0;
};

template <class C>
constexpr CUtensorMapDataType tmap_dtype() {
  return C::Bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
}

template <class C>
bool b_tmap(CUtensorMap* t, const void* b, int64_t Ncols, int64_t Kc) {
  // B K-major [Ncols, Kc] or MN-major [Kc, Ncols]; boxes are one 128-byte row wide
  return C::BMn ? make_tmap_2d(t, tmap_dtype<C>(), C::ElemBytes, b, Ncols, Kc, C::BNBlock, C::BK, true)
                : make_tmap_2d(t, tmap_dtype<C>(), C::ElemBytes, b, Kc, Ncols, C::BK, C::BN, true);
}

// C[M, Ncols] = bf16(A . B / (sa sb)) (+ addend, rounded as bf16 tensors add);
// A [M, Kc] K-major; B per C::BMn.  Operands are 8-bit codes, or bf16 when C::Bf16.
template <class C>
cudaError_t tc_gemm(const void* a, const float* sa, const void* b, const float* sb,
                    int64_t M, int64_t Ncols, int64_t Kc, void* out, int32_t* dev_status,
                    cudaStream_t stream, const Segment2& s2 = Segment2{}, const void* addend = nullptr,
                    int64_t lda = 0, int f32_accumulate = 0) {
  CUtensorMap tA, tB, tB2, tBh;
  // A [M, Kc] K-major, rows lda elements apart (0: Kc)
  if (!make_tmap_2d(&tA, tmap_dtype<C>(), C::ElemBytes, a, Kc, M, C::BK, kBM, true, static_cast<uint64_t>(lda)))
    return cudaErrorInvalidValue;
  const bool seg1 = out != nullptr;
  if (seg1 && !b_tmap<C>(&tB, b, Ncols, Kc)) return cudaErrorInvalidValue;
  if (s2.n > 0 && !b_tmap<C>(&tB2, s2.b, s2.n, Kc)) return cudaErrorInvalidValue;
  if (!seg1) tB = tB2;
  if (s2.n <= 0) tB2 = tB;
  // K-major half tiles load 128 rows of B through a half-height box
  tBh = tB;
  if (!C::BMn && seg1 &&
      !make_tmap_2d(&tBh, tmap_dtype<C>(), C::ElemBytes, b, Kc, Ncols, C::BK, C::HalfN, true))
    return cudaErrorInvalidValue;
  GemmArgs g{};
  g.m_tiles = ceil_div(M, C::TileM);
  g.n_tiles0 = seg1 ? ceil_div(Ncols, C::BN) : 0;
  g.n_tiles = g.n_tiles0 + (s2.n > 0 ? ceil_div(s2.n, C::BN) : 0);
  g.kb_total = ceil_div(Kc, C::BK);
  g.M = M;
  g.N = seg1 ? Ncols : 0;
  g.out = out;
  g.ldo = Ncols;
  g.scale_a = sa;
  g.scale_b = sb;
  g.N2 = s2.n > 0 ? s2.n : 0;
  g.out2_hi = s2.hi;
  g.out2_lo = s2.lo;
  g.ld2 = s2.ld;
  g.scale_b2 = s2.sb;
  g.addend = addend;
  g.f32_accumulate = f32_accumulate;
  g.dev_status = dev_status;
  if (g.n_tiles == 0) return cudaSuccess;
  if (g.n_tiles0 < g.n_tiles) return launch_gemm<C, 1>(tA, tB, tB2, tBh, g, stream);
  return launch_gemm<C, 0>(tA, tB, tB2, tBh, g, stream);
}

template <class C>
cudaError_t fp8_gemm(const uint8_t* a, const float* sa, const uint8_t* b, const float* sb,
                     int64_t M, int64_t Ncols, int64_t Kc, void* out, int32_t* dev_status,
                     cudaStream_t stream, const Segment2& s2 = Segment2{}) {
  return tc_gemm<C>(a, sa, b, sb, M, Ncols, Kc, out, dev_status, stream, s2);
}

// Grouped forward (kMode 2): Y_s = bf16(Xq . Wq_s^T / (s_X s_W_s)) for up to
// three backbones Wq_s [N_s, Kc] that read the same quantized activation.
cudaError_t fp8_gemm_grouped(const uint8_t* a, const float* sa, int nseg, const uint8_t* const* b,
                             const float* const* sb, const int64_t* n, void* const* out, int64_t M, int64_t Kc,
                             int32_t* dev_status, cudaStream_t stream) {
  using C = FwdCfg;
  CUtensorMap tA, tb[3];
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a, Kc, M, C::BK, kBM, true)) return cudaErrorInvalidValue;
  GemmArgs g{};
  g.nseg = nseg;
  int tiles = 0;
  for (int sg = 0; sg < 3; ++sg) {
    g.seg_tile0[sg] = tiles;
    if (sg < nseg) {
      if (!b_tmap<C>(&tb[sg], b[sg], n[sg], Kc)) return cudaErrorInvalidValue;
      g.seg_out[sg] = out[sg];
      g.seg_scale[sg] = sb[sg];
      g.seg_n[sg] = n[sg];
      tiles += ceil_div(n[sg], C::BN);
    } else {
      tb[sg] = tb[0];  // an absent segment owns no tile: its first tile is the end
    }
  }
  g.seg_tile0[3] = tiles;
  g.m_tiles = ceil_div(M, C::TileM);
  g.n_tiles = g.n_tiles0 = tiles;
  g.kb_total = ceil_div(Kc, C::BK);
  g.M = M;
  g.N = n[0];
  g.out = out[0];
  g.ldo = n[0];
  g.scale_a = sa;
  g.scale_b = sb[0];
  g.dev_status = dev_status;
  if (tiles == 0) return cudaSuccess;
  return launch_gemm<C, 2>(tA, tb[0], tb[1], tb[2], g, stream);
}

using BfFwdCfg = Cfg<false, 256, 4, 2, 1, 1, 0, true>;  // bf16 operands, B K-major
using BfDxCfg = Cfg<true, 256, 4, 2, 1, 1, 0, true>;    // bf16 operands, B MN-major

}  // namespace

// The plain forward and dX products run on SM pairs (gemm_pair.cu); the
// one-SM kernel keeps the adapter-segment, grouped and addend variants.
cudaError_t launch_fp8_gemm_fwd(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                const float* s_w, int64_t M, int64_t N, int64_t K, void* y,
                                int32_t* dev_status, cudaStream_t stream) {
  return launch_fp8_gemm_fwd_pair(xq, s_x, wq, s_w, M, N, K, y, dev_status, stream);
}

cudaError_t launch_fp8_gemm_dx(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                               const float* s_w, int64_t M, int64_t N, int64_t K, void* dx,
                               int32_t* dev_status, cudaStream_t stream, bool dy_e5m2) {
  return launch_fp8_gemm_dx_pair(dyq, s_dy, wq, s_w, M, N, K, dx, dev_status, stream, dy_e5m2);
}

cudaError_t launch_fp8_gemm_fwd_folded(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                       const float* s_w, const uint8_t* aq, const float* s_a, int64_t M,
                                       int64_t N, int64_t K, int64_t r, void* y, void* t_hi, void* t_lo,
                                       int64_t ld, int32_t* dev_status, cudaStream_t stream) {
  Segment2 s2;
  s2.b = aq; s2.sb = s_a; s2.n = r; s2.hi = t_hi; s2.lo = t_lo; s2.ld = ld;
  return fp8_gemm<FwdCfg>(xq, s_x, wq, s_w, M, N, K, y, dev_status, stream, s2);
}

cudaError_t launch_fp8_gemm_dx_folded(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                                      const float* s_w, const uint8_t* bq, const float* s_b, int64_t M,
                                      int64_t N, int64_t K, int64_t r, void* dx, void* u_hi, void* u_lo,
                                      int64_t ld, int32_t* dev_status, cudaStream_t stream) {
  // contraction over N: B~q [N, r] is the MN-major second segment beside Wq [N, K]
  Segment2 s2;
  s2.b = bq; s2.sb = s_b; s2.n = bq ? r : 0; s2.hi = u_hi; s2.lo = u_lo; s2.ld = ld;
  return fp8_gemm<DxCfg>(dyq, s_dy, wq, s_w, M, K, N, dx, dev_status, stream, s2);
}

cudaError_t launch_gemm_nt(bool bf16, const void* a, const float* sa, const void* b, const float* sb, int64_t M,
                           int64_t Ncols, int64_t Kc, void* out, const void* addend, int32_t* dev_status,
                           cudaStream_t stream) {
  return bf16 ? tc_gemm<BfFwdCfg>(a, sa, b, sb, M, Ncols, Kc, out, dev_status, stream, Segment2{}, addend)
              : tc_gemm<FwdCfg>(a, sa, b, sb, M, Ncols, Kc, out, dev_status, stream, Segment2{}, addend);
}

cudaError_t launch_gemm_nn(bool bf16, const void* a, const float* sa, const void* b, const float* sb, int64_t M,
                           int64_t Ncols, int64_t Kc, void* out, const void* addend, int32_t* dev_status,
                           cudaStream_t stream, int64_t lda) {
  return bf16 ? tc_gemm<BfDxCfg>(a, sa, b, sb, M, Ncols, Kc, out, dev_status, stream, Segment2{}, addend, lda)
              : tc_gemm<DxCfg>(a, sa, b, sb, M, Ncols, Kc, out, dev_status, stream, Segment2{}, addend, lda);
}

cudaError_t launch_fp8_gemm_fwd_grouped(const uint8_t* xq, const float* s_x, int nseg, const uint8_t* const* wq,
                                        const float* const* s_w, const int64_t* n, void* const* y, int64_t M,
                                        int64_t K, int32_t* dev_status, cudaStream_t stream) {
  return fp8_gemm_grouped(xq, s_x, nseg, wq, s_w, n, y, M, K, dev_status, stream);
}

cudaError_t launch_gemm_nn_f32acc(const void* a, const void* b, int64_t M, int64_t Ncols, int64_t Kc, float* out,
                                  int32_t* dev_status, cudaStream_t stream) {
  return tc_gemm<BfDxCfg>(a, nullptr, b, nullptr, M, Ncols, Kc, out, dev_status, stream, Segment2{}, nullptr, 0, 1);
}

cudaError_t launch_gemm_bf16_f32out(bool b_mn, const void* a, int64_t lda, const void* b, const float* sb, int64_t M,
                                    int64_t Ncols, int64_t Kc, float* out, int32_t* dev_status, cudaStream_t stream) {
  return b_mn ? tc_gemm<BfDxCfg>(a, nullptr, b, sb, M, Ncols, Kc, out, dev_status, stream, Segment2{}, nullptr, lda, 2)
              : tc_gemm<BfFwdCfg>(a, nullptr, b, sb, M, Ncols, Kc, out, dev_status, stream, Segment2{}, nullptr, lda, 2);
}

}  // namespace falqon
