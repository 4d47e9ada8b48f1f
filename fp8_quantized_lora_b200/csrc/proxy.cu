// Row-wise proxy update of the FP8 backbone.
//
// FALQON (abstract and introduction): a row-wise proxy accumulates the
// adapter updates and only the substantial ones are applied to the quantized
// backbone; updates that would vanish under quantization are skipped.  The
// rule implemented here: row n is selected iff adding its proxy would change
// the value of at least one of its E4M3 codes; selected rows take the new
// value of every code whose value changes and have their proxy cleared;
// other rows keep their codes bit-for-bit and their accumulated proxy.
//
// Two launches per update (one of the first two kernels, then the clear), no
// cross-CTA synchronisation:
//   proxy_ws_kernel  (accumulation with r <= 64, r % 8 == 0; persistent,
//     two CTAs per SM) walks a contiguous range of 32 x 256 tiles of P,
//     column block by column block.  Four math warps run only the FMA chains
//     (8 rows x 8 columns per thread) from A's columns and the tile's dB_inc
//     values in shared memory and hand D over in shared memory; four epilogue
//     warps stage those operands one tile ahead, hold the tile's P and Wq in
//     registers while D is computed, and run the epilogue below (registers
//     are split 104 / 152 between the roles).  The roles meet on mbarriers
//     with bounded waits.  The arithmetic is the one below.
//   proxy_stream_kernel  (grid over 32 x 256 tiles of P; two CTAs per SM;
//     any r)
//     Each thread owns 8 rows x 4 columns.  Its P and Wq slices stream in
//     with cp.async while the tile's A columns and dB_inc rows are staged
//     in shared memory (A as bf16, dB_inc as duplicated float pairs so that
//     the packed FMA takes its operand straight from a broadcast load).
//     D = dB_inc . A is a float32 FMA chain in index order i = 0..r-1 from
//     +0 (__ffma2_rn: two independent round-to-nearest FMAs), P' = P + D is
//     written back, and t = dec(c) + s_W * P' (no FMA) is re-encoded.  Codes
//     whose value changes are written at once -- such a change already
//     selects the row -- and the row's flag is set.
//   proxy_clear_kernel  (one warp per row)
//     Selected rows get P = +0; writes the row mask and the selected count.
//     With a deferred clear it writes only the mask and the count, and the
//     next call's accumulation reads the masked rows' P as +0.
//
// Every step is reproduced bit-for-bit by the float32 arithmetic.
#include <cuda_fp16.h>

#include "codes.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace falqon {
namespace {

using namespace codes;

// Selection mode of the accumulation kernels.
constexpr int kModeNone = 0;    // accumulate only
constexpr int kModeSelect = 1;  // threshold rule: changed codes written at once, per-block row flags

constexpr int kThreads = 256;
constexpr int kTileRows = 32;   // 4 row groups of kRT rows
constexpr int kTileCols = 256;  // 64 column groups of 4 columns
constexpr int kRT = 8;          // rows per thread
constexpr int kIChunk = 64;     // ranks staged per pass

// dynamic shared memory layout (bytes)
constexpr int kAsBytes = kIChunk * kTileCols * 2;                  // bf16 A chunk   32 KB
constexpr int kBsBytes = kIChunk * kTileRows * 8;                  // (b, b) pairs   16 KB
constexpr int kPBytes = kRT * kThreads * 16;                       // P slices       32 KB
constexpr int kWBytes = kRT * kThreads * 4;                        // Wq slices       8 KB
constexpr int kSmemBytes = kAsBytes + kBsBytes + kPBytes + kWBytes;  // 88 KB

// Residual-keeping clear: for the codes in byte mask m (their value changes
// from w_old to w_new) the proxy keeps what the new code does not apply,
// P - (dec(new) - dec(old)) / s_w (the difference of two E4M3 values is exact
// in float32; one IEEE division, one subtraction); other lanes keep P.
__device__ __forceinline__ float4 residual4(float4 p, uint32_t w_old, uint32_t w_new, uint32_t m, float s_w) {
  const float2 o01 = e4m3x2_values(w_old), o23 = e4m3x2_values(w_old >> 16);
  const float2 n01 = e4m3x2_values(w_new), n23 = e4m3x2_values(w_new >> 16);
  if (m & 0x000000FFu) p.x = __fsub_rn(p.x, __fdiv_rn(__fsub_rn(n01.x, o01.x), s_w));
  if (m & 0x0000FF00u) p.y = __fsub_rn(p.y, __fdiv_rn(__fsub_rn(n01.y, o01.y), s_w));
  if (m & 0x00FF0000u) p.z = __fsub_rn(p.z, __fdiv_rn(__fsub_rn(n23.x, o23.x), s_w));
  if (m & 0xFF000000u) p.w = __fsub_rn(p.w, __fdiv_rn(__fsub_rn(n23.y, o23.y), s_w));
  return p;
}

template <bool kAcc, int kSel>
__global__ void __launch_bounds__(kThreads, 2)
    proxy_stream_kernel(uint8_t* __restrict__ wq, const float* __restrict__ s_w_ptr,
                        float* __restrict__ proxy, const uint16_t* __restrict__ dB_inc,
                        const uint16_t* __restrict__ A, int64_t N, int64_t K, int r,
                        uint8_t* __restrict__ rowflag, int32_t* __restrict__ n_selected,
                        int32_t* __restrict__ dev_status, int keep_residual,
                        const uint8_t* __restrict__ zero_rows) {
  pdl_trigger();  // the next kernel may start launching; it waits for this one
  pdl_wait();     // the previous kernel's results are complete and visible
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ int tile_flag[kTileRows];  // a code of the row changed
  uint16_t* As = reinterpret_cast<uint16_t*>(sm);                              // [kIChunk][256]
  float2* Bs = reinterpret_cast<float2*>(sm + kAsBytes);                       // [kIChunk][32]
  float4* pbuf = reinterpret_cast<float4*>(sm + kAsBytes + kBsBytes);          // [kRT][256]
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(sm + kAsBytes + kBsBytes + kPBytes);  // [kRT][256]

  const int tid = threadIdx.x;
  const int tc = tid & 63;  // columns c0 + 4*tc .. +3
  const int tr = tid >> 6;  // rows r0 + 8*tr .. +7
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTileRows;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTileCols;
  const int64_t col = c0 + 4 * tc;
  const bool col_ok = col < K;  // K % 16 == 0: four columns in or out together

  // this thread's P and Wq slices start streaming first
#pragma unroll
  for (int j = 0; j < kRT; ++j) {
    const int64_t n = r0 + tr * kRT + j;
    const bool ok = col_ok && n < N;
    const bool pz = ok && zero_rows && zero_rows[n];  // a deferred clear: P reads as +0
    cp_async16(pbuf + j * kThreads + tid, ok ? static_cast<const void*>(proxy + n * K + col) : proxy,
               ok && !pz ? 16u : 0u);
    if (kSel != kModeNone)
      cp_async4(wbuf + j * kThreads + tid, ok ? static_cast<const void*>(wq + n * K + col) : wq,
                ok ? 4u : 0u);
  }
  cp_async_commit();

  float2 acc[kRT][2];
#pragma unroll
  for (int j = 0; j < kRT; ++j) acc[j][0] = acc[j][1] = make_float2(0.0f, 0.0f);

  if constexpr (kAcc) {
    for (int i0 = 0; i0 < r; i0 += kIChunk) {
      const int ni = r - i0 < kIChunk ? r - i0 : kIChunk;
      // A[i0 : i0+64, c0 : c0+256] as bf16, 16-byte chunks (zero outside the tensor)
#pragma unroll
      for (int k = 0; k < (kIChunk * kTileCols / 8) / kThreads; ++k) {
        const int e = tid + k * kThreads;
        const int i = e / (kTileCols / 8), c8 = e % (kTileCols / 8);
        const int64_t gc = c0 + 8 * c8;
        const bool ok = i < ni && gc < K;
        cp_async16(As + i * kTileCols + 8 * c8,
                   ok ? static_cast<const void*>(A + static_cast<int64_t>(i0 + i) * K + gc) : A,
                   ok ? 16u : 0u);
      }
      cp_async_commit();
      // dB_inc[r0 : r0+32, i0 : i0+64] -> (b, b) pairs, [i][row]
#pragma unroll
      for (int k = 0; k < (kIChunk * kTileRows) / kThreads; ++k) {
        const int e = tid + k * kThreads;
        const int row = e / kIChunk, i = e % kIChunk;
        const int64_t n = r0 + row;
        float f = 0.0f;
        if (i < ni && n < N) f = bf16_bits_to_f32(dB_inc[n * r + i0 + i]);
        Bs[i * kTileRows + row] = make_float2(f, f);
      }
      cp_async_wait_all();
      __syncthreads();
      const uint16_t* arow = As + 4 * tc;
      const float2* brow = Bs + tr * kRT;
#pragma unroll 4
      for (int i = 0; i < ni; ++i) {
        const uint2 a2 = *reinterpret_cast<const uint2*>(arow + i * kTileCols);
        const float2 a01 = make_float2(__uint_as_float(a2.x << 16), __uint_as_float(a2.x & 0xFFFF0000u));
        const float2 a23 = make_float2(__uint_as_float(a2.y << 16), __uint_as_float(a2.y & 0xFFFF0000u));
        float2 bb[kRT];
#pragma unroll
        for (int j = 0; j < kRT; j += 2) {
          const float4 q = *reinterpret_cast<const float4*>(brow + i * kTileRows + j);
          bb[j] = make_float2(q.x, q.y);
          bb[j + 1] = make_float2(q.z, q.w);
        }
#pragma unroll
        for (int j = 0; j < kRT; ++j) {
          acc[j][0] = __ffma2_rn(bb[j], a01, acc[j][0]);
          acc[j][1] = __ffma2_rn(bb[j], a23, acc[j][1]);
        }
      }
      __syncthreads();  // the next chunk overwrites As and Bs
    }
  }
  cp_async_wait_all();

  const float s_w = kSel != kModeNone ? *s_w_ptr : 1.0f;
  bool nonfinite = false;
  if (kSel != kModeNone) {
    if (tid < kTileRows) tile_flag[tid] = 0;
    if (kSel == kModeSelect && n_selected && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0)
      *n_selected = 0;  // the clear pass counts
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < kRT; ++j) {
    const int64_t n = r0 + tr * kRT + j;
    if (!(col_ok && n < N)) continue;
    float4 p = pbuf[j * kThreads + tid];
    if constexpr (kAcc) {
      p.x = __fadd_rn(p.x, acc[j][0].x);
      p.y = __fadd_rn(p.y, acc[j][0].y);
      p.z = __fadd_rn(p.z, acc[j][1].x);
      p.w = __fadd_rn(p.w, acc[j][1].y);
      *reinterpret_cast<float4*>(proxy + n * K + col) = p;
    }
    nonfinite |= !(isfinite(p.x) && isfinite(p.y) && isfinite(p.z) && isfinite(p.w));
    if constexpr (kSel != kModeNone) {
      const uint32_t w = wbuf[j * kThreads + tid];
      const uint32_t cn = requantized4(w, s_w, p);
      const uint32_t m = changed_bytes(w, cn);
      if (m) {
        *reinterpret_cast<uint32_t*>(wq + n * K + col) = (cn & m) | (w & ~m);
        tile_flag[tr * kRT + j] = 1;  // every writer stores the same value
        if (keep_residual) *reinterpret_cast<float4*>(proxy + n * K + col) = residual4(p, w, cn, m, s_w);
      }
    }
  }
  if (kSel != kModeNone) {
    // this tile's verdict for each of its rows, written in every case
    __syncthreads();
    const int64_t ncb = gridDim.x;
    if (tid < kTileRows && r0 + tid < N) rowflag[(r0 + tid) * ncb + blockIdx.x] = static_cast<uint8_t>(tile_flag[tid]);
  }
  if (__any_sync(0xFFFFFFFFu, nonfinite) && (tid & 31) == 0 && dev_status)
    atomicOr(dev_status, kDevNonfinite);
}

// ---------------------------------------------------------------- warp-specialised pipeline
// Persistent, two CTAs per SM, 32 x 256 tiles of P taken column block by
// column block.  Warps 4-7 run only the float32 FMA chains: warp 4 + w owns
// columns 64w .. 64w+63 of the tile, lane (g, c) = (l / 8, l % 8) rows
// 8g .. 8g+7 and columns 64w + 8c .. +7, 8 x 8 accumulators per thread (32
// packed FMAs per rank against one 16-byte load of A and two of dB_inc
// values, whose (b, b) pairs are formed in registers).  Warps 0-3 stage the
// operands (A's columns of the block when it changes, the next tile's
// dB_inc values as floats), prefetch the tile's P and Wq into registers and
// run the epilogue from D, which the math warps hand over in shared memory
// (the epilogue warps come first: at r = 16 that measured 3 % faster than
// the other order).  The two roles meet on mbarriers whose waits are
// bounded.
constexpr int kWsThreads = 256;
constexpr int kWsRows = 32;
constexpr int kWsRMax = 64;                                   // ranks held in shared memory
constexpr int kWsAsBytes = kWsRMax * kTileCols * 2;           // A columns, bf16      32 KB
constexpr int kWsBsBytes = kWsRMax * kWsRows * 4;             // dB_inc values, each   8 KB
constexpr int kWsDBytes = kWsRows * kTileCols * 4;            // D of one tile        32 KB
constexpr int kWsSmemBytes = kWsAsBytes + 2 * kWsBsBytes + kWsDBytes + 64;  // 80 KB + 6 mbarriers
// Registers per thread of the two roles after the split (setmaxnreg): the
// launch gives 65536 / (2 CTAs x 256 threads) = 128 per thread, and the
// split must return exactly the CTA's pool, or the increase never completes.
constexpr int kWsMathRegs = 104, kWsEpiRegs = 152;
static_assert(128 * kWsMathRegs + 128 * kWsEpiRegs == kWsThreads * (65536 / (2 * kWsThreads)),
              "the register split must balance the CTA's launch allocation");
static_assert(kWsMathRegs % 8 == 0 && kWsEpiRegs % 8 == 0, "setmaxnreg takes multiples of 8");

template <int kSel>
__global__ void __launch_bounds__(kWsThreads, 2)
    proxy_ws_kernel(uint8_t* __restrict__ wq, const float* __restrict__ s_w_ptr, float* __restrict__ proxy,
                    const uint16_t* __restrict__ dB_inc, const uint16_t* __restrict__ A, int64_t N, int64_t K,
                    int r, int row_groups, int units, int ncb, uint8_t* __restrict__ rowflag,
                    int32_t* __restrict__ n_selected, int32_t* __restrict__ dev_status, int keep_residual,
                    const uint8_t* __restrict__ zero_rows) {
  // No early trigger: the clear kernel that follows would only sit on the SMs.
  pdl_wait();
  extern __shared__ __align__(128) uint8_t sm[];
  uint16_t* As = reinterpret_cast<uint16_t*>(sm);                                     // [r][256]
  float* Bs = reinterpret_cast<float*>(sm + kWsAsBytes);                              // [2][64][32]
  float* Ds = reinterpret_cast<float*>(sm + kWsAsBytes + 2 * kWsBsBytes);             // [32][256]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kWsAsBytes + 2 * kWsBsBytes + kWsDBytes);
  uint64_t* full_ops = bars;      // [2] operands of a tile staged (epilogue -> math)
  uint64_t* empty_ops = bars + 2; // [2] a tile's operands consumed (math -> epilogue)
  uint64_t* full_d = bars + 4;    // D of a tile written (math -> epilogue)
  uint64_t* empty_d = bars + 5;   // D read (epilogue -> math)
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * units / gridDim.x);
  const int u_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * units / gridDim.x);
  if (u_begin >= u_end) return;
  const int ntiles = u_end - u_begin;
  if (tid == 0) {
    for (int b = 0; b < 6; ++b) mbar_init(bars + b, 128);
    abort_flag = 0;
    fence_barrier_init();
    if (kSel == kModeSelect && n_selected && blockIdx.x == 0) *n_selected = 0;  // the clear pass counts
  }
  __syncthreads();
  auto give_up = [&]() {
    abort_flag = 1;
    if (dev_status) atomicOr(dev_status, kDevTimeout);
  };

  // Register split between the roles: the math warps need about 90 registers
  // (64 accumulators and the operands of one rank step) and hand the rest to
  // the epilogue warps, which hold a tile's P and Wq slices (at 128 each,
  // the epilogue spilled).
  if (warp >= 4) {
    // ------------------------------------------------------------ math warps (4-7)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kWsMathRegs));
    const int g = lane >> 3, c = lane & 7;
    const int colw = 64 * (warp - 4) + 8 * c;
    for (int t = 0; t < ntiles; ++t) {
      if (!mbar_wait(&full_ops[t & 1], (t >> 1) & 1, &abort_flag)) {
        give_up();
        break;
      }
      float2 acc[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int h = 0; h < 4; ++h) acc[j][h] = make_float2(0.0f, 0.0f);
      // shared-memory bytes per 32 packed FMAs are what bounds this loop: A
      // arrives as 8 bf16 (16 bytes), the 8 rows' dB_inc values as floats (32
      // bytes) and their (b, b) pairs are formed in registers
      const uint16_t* arow = As + colw;
      const float* brow = Bs + (t & 1) * (kWsRMax * kWsRows) + 8 * g;
#pragma unroll 2
      for (int i = 0; i < r; ++i) {
        const uint4 a4 = *reinterpret_cast<const uint4*>(arow + i * kTileCols);
        const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w};
        float2 av[4];
#pragma unroll
        for (int h = 0; h < 4; ++h)
          av[h] = make_float2(__uint_as_float(aw[h] << 16), __uint_as_float(aw[h] & 0xFFFF0000u));
        const float4 q0 = *reinterpret_cast<const float4*>(brow + i * kWsRows);
        const float4 q1 = *reinterpret_cast<const float4*>(brow + i * kWsRows + 4);
        const float bv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 b = make_float2(bv[j], bv[j]);
#pragma unroll
          for (int h = 0; h < 4; ++h) acc[j][h] = __ffma2_rn(b, av[h], acc[j][h]);
        }
      }
      mbar_arrive(&empty_ops[t & 1]);
      if (!mbar_wait(empty_d, (t & 1) ^ 1, &abort_flag)) {
        give_up();
        break;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4* dst = reinterpret_cast<float4*>(Ds + (8 * g + j) * kTileCols + colw);
        dst[0] = make_float4(acc[j][0].x, acc[j][0].y, acc[j][1].x, acc[j][1].y);
        dst[1] = make_float4(acc[j][2].x, acc[j][2].y, acc[j][3].x, acc[j][3].y);
      }
      mbar_arrive(full_d);
    }
    return;
  }

  // -------------------------------------------------------------- epilogue warps
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kWsEpiRegs));
  const int et = tid;  // epilogue warps 0-3
  const int ew = et >> 5;  // rows 8ew .. 8ew+7 of the tile; lane: columns 4l .. 4l+3 and 128 + 4l .. +3
  const int chunks_per_row = r / 8;
  auto stage = [&](int v, bool with_a) {
    const int64_t r0 = static_cast<int64_t>(v % row_groups) * kWsRows;
    float* B = Bs + ((v - u_begin) & 1) * (kWsRMax * kWsRows);
    // lane = row: each store instruction of a warp writes 32 consecutive words
    for (int e = et; e < kWsRows * chunks_per_row; e += 128) {
      const int row = e % kWsRows, c8 = e / kWsRows;
      const int64_t n = r0 + row;
      uint4 q = make_uint4(0u, 0u, 0u, 0u);
      if (n < N) q = *reinterpret_cast<const uint4*>(dB_inc + n * r + 8 * c8);
      const uint32_t wds[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        B[(8 * c8 + 2 * h) * kWsRows + row] = __uint_as_float(wds[h] << 16);
        B[(8 * c8 + 2 * h + 1) * kWsRows + row] = __uint_as_float(wds[h] & 0xFFFF0000u);
      }
    }
    if (with_a) {
      const int64_t cb = v / row_groups;
      for (int e = et; e < r * (kTileCols / 8); e += 128) {
        const int i = e / (kTileCols / 8), c8 = e % (kTileCols / 8);
        const int64_t gc = cb * kTileCols + 8 * c8;
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (gc < K) q = *reinterpret_cast<const uint4*>(A + static_cast<int64_t>(i) * K + gc);
        *reinterpret_cast<uint4*>(As + i * kTileCols + 8 * c8) = q;
      }
    }
  };
  stage(u_begin, true);
  mbar_arrive(&full_ops[0]);
  const float s_w = kSel != kModeNone ? *s_w_ptr : 1.0f;
  uint32_t maxmag = 0;  // largest |P'| bit pattern: >= 0x7F800000 means inf or NaN
  for (int t = 0; t < ntiles; ++t) {
    const int v = u_begin + t;
    const int cb = v / row_groups;
    const int64_t r0 = static_cast<int64_t>(v % row_groups) * kWsRows;
    const int64_t cbase = static_cast<int64_t>(cb) * kTileCols + 4 * lane;
    // 1. this tile's P and Wq slices, in registers while the math warps compute D
    float4 p[8][2];
    uint32_t w[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t n = r0 + 8 * ew + j;
      const bool pz = zero_rows && n < N && zero_rows[n];  // a deferred clear: P reads as +0
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t col = cbase + 128 * h;
        const bool ok = n < N && col < K;  // K % 16 == 0: four columns in or out together
        p[j][h] = ok && !pz ? *reinterpret_cast<const float4*>(proxy + n * K + col) : make_float4(0.f, 0.f, 0.f, 0.f);
        w[j][h] = (ok && kSel != kModeNone) ? *reinterpret_cast<const uint32_t*>(wq + n * K + col) : 0u;
      }
    }
    // 2. operands of the next tile (its A columns only when the column block changes)
    if (t + 1 < ntiles) {
      const int tn = t + 1;
      const bool new_block = (v + 1) / row_groups != cb;
      bool ok = true;
      if (new_block) ok = mbar_wait(&empty_ops[t & 1], (t >> 1) & 1, &abort_flag);  // As free
      if (ok) ok = mbar_wait(&empty_ops[tn & 1], ((tn >> 1) & 1) ^ 1, &abort_flag);   // Bs[tn & 1] free
      if (!ok) {
        give_up();
        break;
      }
      stage(v + 1, new_block);
      mbar_arrive(&full_ops[tn & 1]);
    }
    // 3. D of this tile
    if (!mbar_wait(full_d, t & 1, &abort_flag)) {
      give_up();
      break;
    }
    // 4. P' = P + D, requantize, write P' and the changed codes, the tile's row verdicts
    //    (D is read row by row; the math warps need its buffer only after their next tile)
    uint32_t changed = 0;  // bit j: a code of row 8ew + j changed in this lane's columns
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t n = r0 + 8 * ew + j;  // uniform across the warp
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t col = cbase + 128 * h;
        const float4 dv = *reinterpret_cast<const float4*>(Ds + (8 * ew + j) * kTileCols + 4 * lane + 128 * h);
        if (n < N && col < K) {
          float4 q = p[j][h];
          q.x = __fadd_rn(q.x, dv.x);
          q.y = __fadd_rn(q.y, dv.y);
          q.z = __fadd_rn(q.z, dv.z);
          q.w = __fadd_rn(q.w, dv.w);
          const uint32_t mg = 0x7FFFFFFFu;
          maxmag = max(maxmag, max(max(__float_as_uint(q.x) & mg, __float_as_uint(q.y) & mg),
                                   max(__float_as_uint(q.z) & mg, __float_as_uint(q.w) & mg)));
          float4 out = q;
          if constexpr (kSel != kModeNone) {
            const uint32_t wv = w[j][h];
            const uint32_t cn = requantized4(wv, s_w, q);
            // identical words change only where they hold NaN codes (the common case)
            const uint32_t m = cn == wv ? nan_bytes(wv) : changed_bytes(wv, cn);
            if (m) {
              *reinterpret_cast<uint32_t*>(wq + n * K + col) = (cn & m) | (wv & ~m);
              changed |= 1u << j;
              if (keep_residual) out = residual4(q, wv, cn, m, s_w);
            }
          }
          *reinterpret_cast<float4*>(proxy + n * K + col) = out;
        }
      }
    }
    if constexpr (kSel == kModeSelect) {
      // the tile's verdicts for its rows 8ew .. 8ew+7, written whether or not a code changed
      const uint32_t any = __reduce_or_sync(0xFFFFFFFFu, changed);
      if (lane < 8 && r0 + 8 * ew + lane < N)
        rowflag[(r0 + 8 * ew + lane) * ncb + cb] = static_cast<uint8_t>((any >> lane) & 1u);
    }
    mbar_arrive(empty_d);
  }
  if (__any_sync(0xFFFFFFFFu, maxmag >= 0x7F800000u) && lane == 0 && dev_status)
    atomicOr(dev_status, kDevNonfinite);
}

constexpr int kClearThreads = 256;
constexpr int kClearWarps = kClearThreads / 32;

// One warp per row: the lanes read the row's verdict bytes once each and
// agree on their OR; a selected row is then cleared by the same warp with
// 16-byte stores.
__global__ void __launch_bounds__(kClearThreads)
    proxy_clear_kernel(float* __restrict__ proxy, int64_t N, int64_t K, int ncb,
                       const uint8_t* __restrict__ rowflag, uint8_t* __restrict__ row_mask,
                       int32_t* __restrict__ n_selected, int clear) {
  pdl_trigger();  // the next kernel may start launching; it waits for this one
  pdl_wait();     // the previous kernel's results are complete and visible
  __shared__ int warp_count[kClearWarps];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int count = 0;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * kClearWarps + warp; n < N;
       n += static_cast<int64_t>(gridDim.x) * kClearWarps) {
    uint32_t f = 0;
    for (int c = lane; c < ncb; c += 32) f |= rowflag[n * ncb + c];
    const bool sel = __any_sync(0xFFFFFFFFu, f != 0u);
    if (lane == 0) {
      if (row_mask) row_mask[n] = sel ? 1 : 0;
      count += sel ? 1 : 0;
    }
    if (!sel || !clear) continue;
    float4* row = reinterpret_cast<float4*>(proxy + n * K);
    for (int64_t c = lane; c < K / 4; c += 32) row[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (lane == 0) warp_count[warp] = count;
  __syncthreads();
  if (threadIdx.x == 0 && n_selected) {
    int total = 0;
    for (int w = 0; w < kClearWarps; ++w) total += warp_count[w];
    if (total) atomicAdd(n_selected, total);
  }
}

template <bool kAcc, int kSel>
cudaError_t launch_stream(dim3 grid, uint8_t* wq, const float* s_w, float* proxy, const void* dB_inc,
                          const void* A, int64_t N, int64_t K, int r, uint8_t* rowflag,
                          int32_t* n_selected, int32_t* dev_status, int keep_residual, const uint8_t* zero_rows,
                          cudaStream_t stream) {
  static int configured_mask = 0;  // one bit per device ordinal < 31
  int dev = 0;
  cudaGetDevice(&dev);
  const int bit = dev < 31 ? (1 << dev) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(proxy_stream_kernel<kAcc, kSel>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_ACQ_REL);
  }
  return launch_pdl(proxy_stream_kernel<kAcc, kSel>, grid, dim3(kThreads), kSmemBytes, stream, 1u, wq, s_w,
                    proxy, static_cast<const uint16_t*>(dB_inc), static_cast<const uint16_t*>(A), N, K, r,
                    rowflag, n_selected, dev_status, keep_residual, zero_rows);
}

template <int kSel>
cudaError_t launch_pipe(int grid, uint8_t* wq, const float* s_w, float* proxy, const void* dB_inc,
                        const void* A, int64_t N, int64_t K, int r, int row_groups, int units,
                        int ncb, uint8_t* rowflag, int32_t* n_selected, int32_t* dev_status,
                        int keep_residual, const uint8_t* zero_rows, cudaStream_t stream) {
  static int configured_mask = 0;  // one bit per device ordinal < 31
  int dev = 0;
  cudaGetDevice(&dev);
  const int bit = dev < 31 ? (1 << dev) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(proxy_ws_kernel<kSel>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kWsSmemBytes);
    if (e != cudaSuccess) return e;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_ACQ_REL);
  }
  return launch_pdl(proxy_ws_kernel<kSel>, dim3(grid), dim3(kWsThreads), kWsSmemBytes, stream, 1u, wq,
                    s_w, proxy, static_cast<const uint16_t*>(dB_inc), static_cast<const uint16_t*>(A), N, K, r,
                    row_groups, units, ncb, rowflag, n_selected, dev_status, keep_residual, zero_rows);
}

}  // namespace

size_t proxy_workspace_bytes(int64_t N, int64_t K) {
  // one verdict byte per (row, 256-column block)
  return align_up(static_cast<size_t>(N) * static_cast<size_t>((K + kTileCols - 1) / kTileCols), 256);
}

cudaError_t launch_proxy_update(uint8_t* wq, const float* s_w, float* proxy, const void* dB_inc,
                                const void* A, int64_t N, int64_t K, int64_t r, uint32_t flags,
                                uint8_t* row_mask, int32_t* n_selected, int32_t* dev_status,
                                void* workspace, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  bool acc = flags & 1u;
  const bool sel = flags & 2u;
  const int keep_res = (flags & 4u) ? 1 : 0;  // residual-keeping clear instead of P = +0
  const bool defer = flags & 32u;              // the clear is carried to the next call through row_mask
  const uint8_t* zero_rows = defer ? row_mask : nullptr;
  if (r > (int64_t(1) << 30)) return cudaErrorInvalidValue;
  if (acc && (flags & 16u)) {
    // tensor-core accumulation: P = fl32(P + dB_inc . A), float32 accumulation
    // in the tensor cores' order; the selection below reads the result
    cudaError_t e = launch_gemm_nn_f32acc(dB_inc, A, N, K, r, proxy, dev_status, stream);
    if (e != cudaSuccess || !sel) return e;
    acc = false;
  }
  const dim3 grid(static_cast<unsigned>((K + kTileCols - 1) / kTileCols),
                  static_cast<unsigned>((N + kTileRows - 1) / kTileRows));
  const int rr = acc ? static_cast<int>(r) : 0;
  const int64_t row_groups = (N + kWsRows - 1) / kWsRows;
  const int64_t units = row_groups * grid.x;
  // the persistent kernel accumulates with A and dB_inc slices of up to 64
  // ranks held in 16-byte chunks; selection alone streams through the grid kernel
  const bool pipe = acc && rr >= 1 && rr <= kWsRMax && rr % 8 == 0 &&
                    units <= (int64_t(1) << 30) && di->max_smem_optin >= kWsSmemBytes;
  if (!pipe && grid.y > 65535u) return cudaErrorInvalidValue;
  // per (row, 256-column block) verdicts, each written by the tile that owns it:
  // nothing to clear beforehand
  uint8_t* rowflag = static_cast<uint8_t*>(workspace);
  const int ncb = static_cast<int>(grid.x);
  cudaError_t e;
  if (pipe) {
    const int64_t resident = 2 * static_cast<int64_t>(di->sm_count);  // two CTAs per SM
    const int g = static_cast<int>(units < resident ? units : resident);
    const int rg = static_cast<int>(row_groups), un = static_cast<int>(units);
    if (sel)
      e = launch_pipe<kModeSelect>(g, wq, s_w, proxy, dB_inc, A, N, K, rr, rg, un, ncb, rowflag, n_selected,
                                   dev_status, keep_res, zero_rows, stream);
    else
      e = launch_pipe<kModeNone>(g, wq, s_w, proxy, dB_inc, A, N, K, rr, rg, un, ncb, rowflag, n_selected,
                                 dev_status, keep_res, zero_rows, stream);
  } else if (acc && sel)
    e = launch_stream<true, kModeSelect>(grid, wq, s_w, proxy, dB_inc, A, N, K, rr, rowflag, n_selected,
                                         dev_status, keep_res, zero_rows, stream);
  else if (acc)
    e = launch_stream<true, kModeNone>(grid, wq, s_w, proxy, dB_inc, A, N, K, rr, rowflag, n_selected,
                                       dev_status, keep_res, zero_rows, stream);
  else
    e = launch_stream<false, kModeSelect>(grid, wq, s_w, proxy, dB_inc, A, N, K, rr, rowflag, n_selected,
                                          dev_status, keep_res, zero_rows, stream);
  if (e != cudaSuccess || !sel) return e;
  const int64_t row_blocks = (N + kClearWarps - 1) / kClearWarps;
  const int64_t blocks = row_blocks < static_cast<int64_t>(di->sm_count) * 8 ? row_blocks
                                                                              : static_cast<int64_t>(di->sm_count) * 8;
  return launch_pdl(proxy_clear_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kClearThreads), 0, stream, 1u,
                    proxy, N, K, ncb, rowflag, row_mask, n_selected, keep_res || defer ? 0 : 1);
}

}  // namespace falqon
