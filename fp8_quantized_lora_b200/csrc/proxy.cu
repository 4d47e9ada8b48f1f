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
//   proxy_pipe_kernel  (accumulation with r <= 64, r % 8 == 0; persistent,
//     two CTAs per SM) walks a contiguous range of 32 x 256 tiles of P,
//     column block by column block, keeping the block's A columns in shared
//     memory.  The next tile's dB_inc rows are fetched with cp.async one tile
//     ahead; each thread's P and Wq slices of the current tile are fetched when
//     the tile starts and land while its FMA chains run (8 rows x 8 columns per
//     thread).  The arithmetic is the one below.
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
                        int32_t* __restrict__ dev_status, int keep_residual) {
  pdl_trigger();  // the next kernel may start launching; it waits for this one
  pdl_wait();     // the previous kernel's results are complete and visible
  extern __shared__ __align__(16) uint8_t sm[];
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
    cp_async16(pbuf + j * kThreads + tid, ok ? static_cast<const void*>(proxy + n * K + col) : proxy,
               ok ? 16u : 0u);
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

// ---------------------------------------------------------------- persistent pipeline
// Tiles of 32 rows x 256 columns, four warps per CTA, two CTAs per SM: while
// one CTA runs its epilogue (memory and integer work) the other keeps the FMA
// pipe busy.  Warp w owns rows 8w .. 8w+7 of the tile and lane l the columns
// 8l .. 8l+7, so every thread keeps 8 x 8 accumulators (32 packed FMAs per
// rank against one 16-byte load of A and four broadcast loads of dB_inc pairs).
constexpr int kPipeThreads = 128;
constexpr int kPipeRows = 32;
constexpr int kPipeRT = 8;                          // rows per thread
constexpr int kPipeCT = 8;                          // columns per thread
constexpr int kPipeRMax = 64;                       // ranks held in shared memory
constexpr int kDbStride = kPipeRMax * 2 + 16;       // bytes per staged dB_inc row (padded)
constexpr int kPipePBytes = kPipeRows * kTileCols * 4;            // P tile          32 KB
constexpr int kPipeWBytes = kPipeRows * kTileCols;                // Wq tile          8 KB
constexpr int kPipeDbBytes = kPipeRows * kDbStride;               // dB_inc rows    4.5 KB
constexpr int kPipeAsBytes = kPipeRMax * kTileCols * 2;           // A columns       32 KB
constexpr int kPipeBsBytes = kPipeRMax * kPipeRows * 8;           // (b, b) pairs    16 KB
constexpr int kPipeSmemBytes =
    kPipePBytes + kPipeWBytes + 2 * kPipeDbBytes + kPipeAsBytes + kPipeBsBytes;  // 97 KB

template <int kSel>
__global__ void __launch_bounds__(kPipeThreads, 2)
    proxy_pipe_kernel(uint8_t* __restrict__ wq, const float* __restrict__ s_w_ptr,
                      float* __restrict__ proxy, const uint16_t* __restrict__ dB_inc,
                      const uint16_t* __restrict__ A, int64_t N, int64_t K, int r, int row_groups,
                      int units, int ncb, uint8_t* __restrict__ rowflag,
                      int32_t* __restrict__ n_selected, int32_t* __restrict__ dev_status,
                      int keep_residual) {
  // No early trigger: the clear kernel that follows needs no shared memory, so
  // its CTAs would sit beside this kernel's on the SMs while they wait.
  pdl_wait();  // the previous kernel's results are complete and visible
  extern __shared__ __align__(16) uint8_t sm[];
  float4* pst = reinterpret_cast<float4*>(sm);                                 // [8][2][128]
  uint2* wst = reinterpret_cast<uint2*>(sm + kPipePBytes);                     // [8][128]
  uint8_t* dbraw = sm + kPipePBytes + kPipeWBytes;                             // [2][32][kDbStride]
  uint16_t* As = reinterpret_cast<uint16_t*>(dbraw + 2 * kPipeDbBytes);       // [r][256]
  float2* Bs = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(As) + kPipeAsBytes);  // [r][32]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int tr = tid >> 5;  // rows r0 + 8*tr .. +7
  const int u_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * units / gridDim.x);
  const int u_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * units / gridDim.x);
  if (u_begin >= u_end) return;
  const int chunks_per_row = r / 8;  // 16-byte chunks of one dB_inc row

  auto tile_r0 = [&](int v) { return static_cast<int64_t>(v % row_groups) * kPipeRows; };
  auto tile_col = [&](int v) {
    return static_cast<int64_t>(v / row_groups) * kTileCols + kPipeCT * lane;
  };
  // this thread's P and Wq slices of tile v (read back only by this thread)
  auto issue_pw = [&](int v) {
    const int64_t r0 = tile_r0(v), col = tile_col(v);
    const bool col_ok = col < K;
#pragma unroll
    for (int j = 0; j < kPipeRT; ++j) {
      const int64_t n = r0 + tr * kPipeRT + j;
      const bool ok = col_ok && n < N;
      const float* src = ok ? proxy + n * K + col : proxy;
      cp_async16(pst + (2 * j) * kPipeThreads + tid, src, ok ? 16u : 0u);
      cp_async16(pst + (2 * j + 1) * kPipeThreads + tid, ok ? src + 4 : proxy, ok ? 16u : 0u);
      if (kSel != kModeNone) {
        const uint8_t* wsrc = ok ? wq + n * K + col : wq;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(wst + j * kPipeThreads + tid)),
                     "l"(wsrc), "r"(ok ? 8u : 0u)
                     : "memory");
      }
    }
  };
  // dB_inc rows of tile v -> dbraw[buf] (shared by the CTA)
  auto issue_db = [&](int v, int buf) {
    const int64_t r0 = tile_r0(v);
    for (int e = tid; e < kPipeRows * chunks_per_row; e += kPipeThreads) {
      const int row = e / chunks_per_row, c8 = e % chunks_per_row;
      const int64_t n = r0 + row;
      const bool ok = n < N;
      cp_async16(dbraw + buf * kPipeDbBytes + row * kDbStride + 16 * c8,
                 ok ? static_cast<const void*>(dB_inc + n * r + 8 * c8) : dB_inc, ok ? 16u : 0u);
    }
  };
  // A[0:r, cb*256 : cb*256+256] -> As (zero beyond K)
  auto issue_A = [&](int cb) {
    for (int e = tid; e < r * (kTileCols / 8); e += kPipeThreads) {
      const int i = e / (kTileCols / 8), c8 = e % (kTileCols / 8);
      const int64_t gc = static_cast<int64_t>(cb) * kTileCols + 8 * c8;
      const bool ok = gc < K;
      cp_async16(As + i * kTileCols + 8 * c8,
                 ok ? static_cast<const void*>(A + static_cast<int64_t>(i) * K + gc) : A,
                 ok ? 16u : 0u);
    }
  };

  // prologue: dB_inc rows of the first tile
  issue_db(u_begin, 0);
  cp_async_commit();

  const float s_w = kSel != kModeNone ? *s_w_ptr : 1.0f;
  if (kSel == kModeSelect && n_selected && blockIdx.x == 0 && threadIdx.x == 0)
    *n_selected = 0;  // the clear pass counts
  uint32_t maxmag = 0;  // largest |P'| bit pattern: >= 0x7F800000 means inf or NaN
  int cur_cb = -1, dbuf = 0;
  for (int v = u_begin; v < u_end; ++v) {
    cp_async_wait_all();  // dB_inc rows of tile v (this thread's copies)
    __syncthreads();      // everyone's copies visible; tile v-1 finished everywhere
    // groups, oldest first: A (empty unless the column block changes), P / Wq of
    // tile v, dB_inc rows of tile v+1
    const int cb = v / row_groups;
    const bool new_block = cb != cur_cb;
    if (new_block) issue_A(cb);
    cp_async_commit();
    issue_pw(v);
    cp_async_commit();
    if (v + 1 < u_end) issue_db(v + 1, dbuf ^ 1);
    cp_async_commit();
    cur_cb = cb;
    // dB_inc rows of tile v -> (b, b) pairs, [i][row]
    {
      const uint8_t* raw = dbraw + dbuf * kPipeDbBytes;
      for (int e = tid; e < kPipeRows * chunks_per_row; e += kPipeThreads) {
        const int row = e % kPipeRows, c8 = e / kPipeRows;
        const uint4 q = *reinterpret_cast<const uint4*>(raw + row * kDbStride + 16 * c8);
        const uint32_t wds[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float f0 = __uint_as_float(wds[h] << 16);
          const float f1 = __uint_as_float(wds[h] & 0xFFFF0000u);
          Bs[(8 * c8 + 2 * h) * kPipeRows + row] = make_float2(f0, f0);
          Bs[(8 * c8 + 2 * h + 1) * kPipeRows + row] = make_float2(f1, f1);
        }
      }
    }
    if (new_block) cp_async_wait_group<2>();  // this thread's share of A has landed
    __syncthreads();                           // Bs and A complete

    float2 acc[kPipeRT][4];
#pragma unroll
    for (int j = 0; j < kPipeRT; ++j)
#pragma unroll
      for (int h = 0; h < 4; ++h) acc[j][h] = make_float2(0.0f, 0.0f);
    const uint16_t* arow = As + kPipeCT * lane;
    const float2* brow = Bs + tr * kPipeRT;
#pragma unroll 4
    for (int i = 0; i < r; ++i) {
      const uint4 a4 = *reinterpret_cast<const uint4*>(arow + i * kTileCols);
      const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w};
      float2 av[4];
#pragma unroll
      for (int h = 0; h < 4; ++h)
        av[h] = make_float2(__uint_as_float(aw[h] << 16), __uint_as_float(aw[h] & 0xFFFF0000u));
#pragma unroll
      for (int j = 0; j < kPipeRT; j += 2) {
        const float4 q = *reinterpret_cast<const float4*>(brow + i * kPipeRows + j);
        const float2 b0 = make_float2(q.x, q.y), b1 = make_float2(q.z, q.w);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          acc[j][h] = __ffma2_rn(b0, av[h], acc[j][h]);
          acc[j + 1][h] = __ffma2_rn(b1, av[h], acc[j + 1][h]);
        }
      }
    }

    // epilogue: P' = P + D; requantize; write P' and the changed codes
    cp_async_wait_group<1>();  // P / Wq of tile v (not dB_inc of tile v+1)
    const int64_t r0 = tile_r0(v), col = tile_col(v);
    const bool col_ok = col < K;
#pragma unroll
    for (int j = 0; j < kPipeRT; ++j) {
      const int64_t n = r0 + tr * kPipeRT + j;  // the warp's row: uniform across the warp
      bool changed = false;
      if (col_ok && n < N) {
        float4 p0 = pst[(2 * j) * kPipeThreads + tid];
        float4 p1 = pst[(2 * j + 1) * kPipeThreads + tid];
        p0.x = __fadd_rn(p0.x, acc[j][0].x);
        p0.y = __fadd_rn(p0.y, acc[j][0].y);
        p0.z = __fadd_rn(p0.z, acc[j][1].x);
        p0.w = __fadd_rn(p0.w, acc[j][1].y);
        p1.x = __fadd_rn(p1.x, acc[j][2].x);
        p1.y = __fadd_rn(p1.y, acc[j][2].y);
        p1.z = __fadd_rn(p1.z, acc[j][3].x);
        p1.w = __fadd_rn(p1.w, acc[j][3].y);
        float4* dst = reinterpret_cast<float4*>(proxy + n * K + col);
        dst[0] = p0;
        dst[1] = p1;
        const uint32_t mg = 0x7FFFFFFFu;
        maxmag = max(maxmag, max(max(max(__float_as_uint(p0.x) & mg, __float_as_uint(p0.y) & mg),
                                     max(__float_as_uint(p0.z) & mg, __float_as_uint(p0.w) & mg)),
                                 max(max(__float_as_uint(p1.x) & mg, __float_as_uint(p1.y) & mg),
                                     max(__float_as_uint(p1.z) & mg, __float_as_uint(p1.w) & mg))));
        if constexpr (kSel != kModeNone) {
          const uint2 w = wst[j * kPipeThreads + tid];
          const uint32_t c0 = requantized4(w.x, s_w, p0);
          const uint32_t c1 = requantized4(w.y, s_w, p1);
          // identical words change only where they hold NaN codes (the common case)
          const uint32_t m0 = c0 == w.x ? nan_bytes(w.x) : changed_bytes(w.x, c0);
          const uint32_t m1 = c1 == w.y ? nan_bytes(w.y) : changed_bytes(w.y, c1);
          if (m0 | m1) {
            *reinterpret_cast<uint2*>(wq + n * K + col) =
                make_uint2((c0 & m0) | (w.x & ~m0), (c1 & m1) | (w.y & ~m1));
            changed = true;
            if (keep_residual) {
              dst[0] = residual4(p0, w.x, c0, m0, s_w);
              dst[1] = residual4(p1, w.y, c1, m1, s_w);
            }
          }
        }
      }
      if constexpr (kSel == kModeSelect) {
        // the tile's verdict for row n, written whether or not a code changed
        const bool any = __any_sync(0xFFFFFFFFu, changed);
        if (lane == 0 && n < N) rowflag[n * ncb + v / row_groups] = any ? 1 : 0;
      }
    }
    dbuf ^= 1;
  }
  cp_async_wait_all();
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
                          int32_t* n_selected, int32_t* dev_status, int keep_residual, cudaStream_t stream) {
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
                    rowflag, n_selected, dev_status, keep_residual);
}

template <int kSel>
cudaError_t launch_pipe(int grid, uint8_t* wq, const float* s_w, float* proxy, const void* dB_inc,
                        const void* A, int64_t N, int64_t K, int r, int row_groups, int units,
                        int ncb, uint8_t* rowflag, int32_t* n_selected, int32_t* dev_status,
                        int keep_residual, cudaStream_t stream) {
  static int configured_mask = 0;  // one bit per device ordinal < 31
  int dev = 0;
  cudaGetDevice(&dev);
  const int bit = dev < 31 ? (1 << dev) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(proxy_pipe_kernel<kSel>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPipeSmemBytes);
    if (e != cudaSuccess) return e;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_ACQ_REL);
  }
  return launch_pdl(proxy_pipe_kernel<kSel>, dim3(grid), dim3(kPipeThreads), kPipeSmemBytes, stream, 1u, wq,
                    s_w, proxy, static_cast<const uint16_t*>(dB_inc), static_cast<const uint16_t*>(A), N, K, r,
                    row_groups, units, ncb, rowflag, n_selected, dev_status, keep_residual);
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
  const bool acc = flags & 1u, sel = flags & 2u;
  const int keep_res = (flags & 4u) ? 1 : 0;  // residual-keeping clear instead of P = +0
  if (r > (int64_t(1) << 30)) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((K + kTileCols - 1) / kTileCols),
                  static_cast<unsigned>((N + kTileRows - 1) / kTileRows));
  const int rr = acc ? static_cast<int>(r) : 0;
  const int64_t row_groups = (N + kPipeRows - 1) / kPipeRows;
  const int64_t units = row_groups * grid.x;
  // the persistent kernel accumulates with A and dB_inc slices of up to 64
  // ranks held in 16-byte chunks; selection alone streams through the grid kernel
  const bool pipe = acc && rr >= 1 && rr <= kPipeRMax && rr % 8 == 0 &&
                    units <= (int64_t(1) << 30) && di->max_smem_optin >= kPipeSmemBytes;
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
                                   dev_status, keep_res, stream);
    else
      e = launch_pipe<kModeNone>(g, wq, s_w, proxy, dB_inc, A, N, K, rr, rg, un, ncb, rowflag, n_selected,
                                 dev_status, keep_res, stream);
  } else if (acc && sel)
    e = launch_stream<true, kModeSelect>(grid, wq, s_w, proxy, dB_inc, A, N, K, rr, rowflag, n_selected,
                                         dev_status, keep_res, stream);
  else if (acc)
    e = launch_stream<true, kModeNone>(grid, wq, s_w, proxy, dB_inc, A, N, K, rr, rowflag, n_selected,
                                       dev_status, keep_res, stream);
  else
    e = launch_stream<false, kModeSelect>(grid, wq, s_w, proxy, dB_inc, A, N, K, rr, rowflag, n_selected,
                                          dev_status, keep_res, stream);
  if (e != cudaSuccess || !sel) return e;
  const int64_t row_blocks = (N + kClearWarps - 1) / kClearWarps;
  const int64_t blocks = row_blocks < static_cast<int64_t>(di->sm_count) * 8 ? row_blocks
                                                                              : static_cast<int64_t>(di->sm_count) * 8;
  return launch_pdl(proxy_clear_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kClearThreads), 0, stream, 1u,
                    proxy, N, K, ncb, rowflag, row_mask, n_selected, keep_res ? 0 : 1);
}

}  // namespace falqon
