// Top-k proxy update over the r rank components of the adapter.
//
// FALQON's OpenReview rebuttal (reviewer 3, Q1; reviewer 2, W7): the top-k
// step runs over the r rows of the adapter's proxy, r much smaller than the
// layer's dimension, and shrinks the inner dimension of the weight update
// from r to k.  The proxy Q [r, N] float32 holds in row i the part of B's
// column i (rank component i, whose update to the weight is the outer
// product Q[i,:]^T A[i,:]) not yet merged into the backbone.  One call:
//   accumulate  Q[i,n] = fl32(Q[i,n] + dB_inc[n,i]);
//   score       score_i = max_n |Q[i,n]| * max_k |A[i,k]|, a float64 product
//               of two float32 magnitudes (exact); a non-finite value in the
//               component's Q or A row scores +inf and sets NONFINITE;
//   select      the k components of highest positive score, ties to the
//               lower index;
//   merge       D = float32 FMA chain over the chosen components in
//               increasing index order from +0, t = dec(c) + s_W * D (no
//               FMA), every code whose value changes becomes E4M3(t);
//   clear       the chosen rows of Q become +0.
// Four launches, no waits between CTAs:
//   topk_accum_kernel   Q += dB_inc^T through a shared-memory transpose (64
//                       features x 32 components per CTA), with each CTA's
//                       maxima of |Q| per component; extra CTAs take the row
//                       maxima of |A| (one warp per row and 2048 columns).
//   topk_select_kernel  one CTA: the scores as the bit patterns of the
//                       float64 products (non-negative doubles order like
//                       their bits), each component's rank counted against
//                       every other in shared memory, the chosen
//                       components listed in index order.
//   topk_merge_kernel   persistent, 32 x 256 tiles of Wq taken column block
//                       by column block, the chosen rows of A for the block
//                       kept in shared memory, the chosen Q entries of the
//                       next tile's rows fetched one tile ahead and expanded
//                       into duplicated float pairs; each
//                       thread holds 8 rows x 8 columns of D (packed FMAs)
//                       and writes the codes whose value changes.  2 N K k
//                       flops and one pass over Wq.
//   topk_clear_kernel   Q[S, :] = +0.
// Every result is reproduced bit-for-bit by the float32 arithmetic.
#include "codes.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace falqon {
namespace {

using namespace codes;

constexpr int kAccThreads = 256;
constexpr int kAccN = 64;        // features per accumulation CTA
constexpr int kAccI = 32;        // components per accumulation CTA
constexpr int kAmaxCols = 2048;  // columns of A per warp in the |A| maxima
constexpr int kSelThreads = 1024;

constexpr int kMThreads = 128;  // 4 warps: warp w owns rows 8w .. 8w+7 of the tile
constexpr int kMRows = 32;
constexpr int kMCols = 256;     // lane l owns columns 8l .. 8l+7
constexpr int kMRT = 8;
constexpr int kMChunk = 64;     // components staged per pass
constexpr int kMCtasPerSm = 3;
constexpr int kMAsBytes = kMChunk * kMCols * 2;  // chosen rows of A, bf16    32 KB
constexpr int kMBsBytes = kMChunk * kMRows * 8;  // (q, q) pairs              16 KB
constexpr int kMQBytes = 2 * kMChunk * kMRows * 4;  // raw Q entries, two tiles  16 KB
constexpr int kMWBytes = kMRT * kMThreads * 8;   // this thread's Wq slices    8 KB
constexpr int kMSmemBytes = kMAsBytes + kMBsBytes + kMQBytes + kMWBytes;  // 72 KB

constexpr int kClearThreads = 256;

// Q += dB_inc^T (when accumulate) and per-CTA maxima of |Q| per component:
// partQ[i * nq_x + bx] = largest |Q[i, 64 bx .. 64 bx + 63]| bit pattern.
// The CTAs past nq_blocks write partA[i * kchunks + kc] = largest |A[i, c]|
// bit pattern (bf16) over 2048-column chunk kc.
__global__ void __launch_bounds__(kAccThreads)
    topk_accum_kernel(float* __restrict__ Q, const uint16_t* __restrict__ dB_inc,
                      const uint16_t* __restrict__ A, int64_t N, int64_t K, int r, int accumulate, int nq_x,
                      int nq_blocks, int kchunks, uint32_t* __restrict__ partQ, uint32_t* __restrict__ partA) {
  pdl_trigger();  // the next kernel may start launching; it waits for this one
  pdl_wait();     // the previous kernel's results are complete and visible
  const int tid = threadIdx.x;
  if (static_cast<int>(blockIdx.x) < nq_blocks) {
    __shared__ float tile[kAccI][kAccN + 1];
    __shared__ uint32_t qmax[kAccI];
    const int bx = static_cast<int>(blockIdx.x) % nq_x, by = static_cast<int>(blockIdx.x) / nq_x;
    const int64_t n0 = static_cast<int64_t>(bx) * kAccN;
    const int i0 = by * kAccI;
    if (tid < kAccI) qmax[tid] = 0u;
    if (accumulate) {
      // dB_inc[n0 .. n0+63, i0 .. i0+31], read along the rank (contiguous), stored transposed
      for (int e = tid; e < kAccN * kAccI; e += kAccThreads) {
        const int nn = e / kAccI, ii = e % kAccI;
        const int64_t n = n0 + nn;
        const int i = i0 + ii;
        tile[ii][nn] = (n < N && i < r) ? bf16_bits_to_f32(dB_inc[n * r + i]) : 0.0f;
      }
    }
    __syncthreads();
    const int nn = tid % kAccN;
    const int64_t n = n0 + nn;
    // warp w covers half a row of the tile: the component index is uniform
    // across the warp.  All of a thread's loads are issued before any use.
    constexpr int kPer = kAccI / (kAccThreads / kAccN);
    float v[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = i0 + tid / kAccN + q * (kAccThreads / kAccN);
      v[q] = (i < r && n < N) ? Q[static_cast<int64_t>(i) * N + n] : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int ii = tid / kAccN + q * (kAccThreads / kAccN);
      const int i = i0 + ii;
      if (accumulate && i < r && n < N) {
        v[q] = __fadd_rn(v[q], tile[ii][nn]);
        Q[static_cast<int64_t>(i) * N + n] = v[q];
      }
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int ii = tid / kAccN + q * (kAccThreads / kAccN);
      uint32_t m = __float_as_uint(v[q]) & 0x7FFFFFFFu;  // NaN patterns lie above infinity's
      m = __reduce_max_sync(0xFFFFFFFFu, m);
      if ((tid & 31) == 0 && m) atomicMax(&qmax[ii], m);
    }
    __syncthreads();
    if (partQ && tid < kAccI && i0 + tid < r) partQ[static_cast<int64_t>(i0 + tid) * nq_x + bx] = qmax[tid];
    return;
  }
  if (!partA) return;
  const int b = static_cast<int>(blockIdx.x) - nq_blocks;
  const int warp = tid >> 5, lane = tid & 31;
  const int rb = b / kchunks, kc = b % kchunks;
  const int i = rb * (kAccThreads / 32) + warp;
  if (i >= r) return;  // uniform across the warp
  const int64_t c_begin = static_cast<int64_t>(kc) * kAmaxCols;
  const int64_t c_end = c_begin + kAmaxCols < K ? c_begin + kAmaxCols : K;
  const uint16_t* row = A + static_cast<int64_t>(i) * K;
  uint32_t m = 0u;
  // K % 16 == 0: every 8-column unit that starts below c_end ends by it
  for (int64_t c = c_begin + 8 * lane; c < c_end; c += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) m = max(m, max(w[h] & 0x7FFFu, (w[h] >> 16) & 0x7FFFu));
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if (lane == 0) partA[static_cast<int64_t>(i) * kchunks + kc] = m;
}

// Exclusive prefix sum of v over the CTA in thread order; *total = the sum.
__device__ __forceinline__ int select_block_scan(int v, int* red, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, d);
    if (lane >= d) x += y;
  }
  __syncthreads();  // red is free again
  if (lane == 31) red[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) {
    if (w < warp) before += red[w];
    all += red[w];
  }
  *total = all;
  return before + x - v;
}

__global__ void __launch_bounds__(kSelThreads, 1)
    topk_select_kernel(const uint32_t* __restrict__ partQ, int nq_x, const uint32_t* __restrict__ partA,
                       int kchunks, int r, int64_t k, uint8_t* __restrict__ comp_mask,
                       int32_t* __restrict__ n_selected, int32_t* __restrict__ sel,
                       int32_t* __restrict__ n_sel, int32_t* __restrict__ dev_status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t sm[];
  uint64_t* key = reinterpret_cast<uint64_t*>(sm);  // [r]
  __shared__ int red[kSelThreads / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // one warp per component: the maxima of its partials, then its score's bits
  bool nonfinite = false;
  for (int i = warp; i < r; i += kSelThreads / 32) {
    uint32_t mq = 0u, ma = 0u;
    for (int b = lane; b < nq_x; b += 32) mq = max(mq, partQ[static_cast<int64_t>(i) * nq_x + b]);
    for (int b = lane; b < kchunks; b += 32) ma = max(ma, partA[static_cast<int64_t>(i) * kchunks + b]);
    mq = __reduce_max_sync(0xFFFFFFFFu, mq);
    ma = __reduce_max_sync(0xFFFFFFFFu, ma);
    if (lane == 0) {
      uint64_t kv;
      if (mq >= 0x7F800000u || ma >= 0x7F80u) {
        kv = 0x7FF0000000000000ull;  // +infinity
        nonfinite = true;
      } else {
        const double s = static_cast<double>(__uint_as_float(mq)) * static_cast<double>(__uint_as_float(ma << 16));
        kv = static_cast<uint64_t>(__double_as_longlong(s));
      }
      key[i] = kv;
    }
  }
  if (__syncthreads_or(nonfinite) && tid == 0 && dev_status) atomicOr(dev_status, kDevNonfinite);
  // rank of each component (higher score first, ties to the lower index);
  // chosen iff its rank is below k and its score is positive
  int out = 0;
  for (int base = 0; base < r; base += kSelThreads) {
    const int i = base + tid;
    int chosen = 0;
    if (i < r) {
      const uint64_t ki = key[i];
      if (ki != 0ull && k > 0) {
        int64_t rank = 0;
        for (int j = 0; j < r && rank < k; ++j) {
          const uint64_t kj = key[j];
          rank += (kj > ki || (kj == ki && j < i)) ? 1 : 0;
        }
        chosen = rank < k ? 1 : 0;
      }
      if (comp_mask) comp_mask[i] = static_cast<uint8_t>(chosen);
    }
    int total = 0;
    const int pos = out + select_block_scan(chosen, red, &total);
    if (chosen) sel[pos] = i;
    out += total;
  }
  if (tid == 0) {
    *n_sel = out;
    if (n_selected) *n_selected = out;
  }
}

__global__ void __launch_bounds__(kMThreads, kMCtasPerSm)
    topk_merge_kernel(uint8_t* __restrict__ wq, const float* __restrict__ s_w_ptr, const float* __restrict__ Q,
                      const uint16_t* __restrict__ A, int64_t N, int64_t K, const int32_t* __restrict__ sel,
                      const int32_t* __restrict__ n_sel, int row_groups, int units) {
  pdl_trigger();
  pdl_wait();
  const int ns = *n_sel;
  if (ns <= 0) return;
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t* As = reinterpret_cast<uint16_t*>(sm);                                   // [kMChunk][256]
  float2* Bs = reinterpret_cast<float2*>(sm + kMAsBytes);                           // [kMChunk][32]
  float* qraw = reinterpret_cast<float*>(sm + kMAsBytes + kMBsBytes);               // [2][kMChunk][32]
  uint2* wst = reinterpret_cast<uint2*>(sm + kMAsBytes + kMBsBytes + kMQBytes);     // [8][128]
  __shared__ int s_sel[kMChunk];  // the chosen components of the first chunk

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int tr = tid >> 5;
  const int u_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * units / gridDim.x);
  const int u_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * units / gridDim.x);
  if (u_begin >= u_end) return;
  const int n0c = ns < kMChunk ? ns : kMChunk;  // components of the first chunk
  for (int j = tid; j < n0c; j += kMThreads) s_sel[j] = sel[j];
  __syncthreads();
  // Q entries of the first chunk for the rows of tile v -> qraw[buf] (one tile ahead)
  auto issue_q = [&](int v, int buf) {
    const int64_t r0 = static_cast<int64_t>(v % row_groups) * kMRows;
    float* dst = qraw + buf * (kMChunk * kMRows);
    for (int e = tid; e < n0c * kMRows; e += kMThreads) {
      const int j = e / kMRows, row = e % kMRows;
      const int64_t n = r0 + row;
      const bool ok = n < N;
      cp_async4(dst + e, ok ? static_cast<const void*>(Q + static_cast<int64_t>(s_sel[j]) * N + n) : Q,
                ok ? 4u : 0u);
    }
  };
  issue_q(u_begin, 0);
  cp_async_commit();
  const float s_w = *s_w_ptr;
  int cur_cb = -1;
  for (int v = u_begin; v < u_end; ++v) {
    const int buf = (v - u_begin) & 1;
    const int cb = v / row_groups;
    const int64_t r0 = static_cast<int64_t>(v % row_groups) * kMRows;
    const int64_t c0 = static_cast<int64_t>(cb) * kMCols;
    const int64_t col = c0 + 8 * lane;
    const bool col_ok = col < K;  // K % 16 == 0: the 8 columns are in or out together
    cp_async_wait_all();  // this thread's copies of tile v's Q entries
    __syncthreads();      // everyone's copies visible; the previous tile's FMA loop is done everywhere
    // groups, oldest first: A of the first chunk (empty while it stays), Wq slices of
    // tile v, Q entries of tile v+1
    if (ns > kMChunk || cb != cur_cb) {
      for (int e = tid; e < n0c * (kMCols / 8); e += kMThreads) {
        const int j = e / (kMCols / 8), c8 = e % (kMCols / 8);
        const int64_t gc = c0 + 8 * c8;
        const bool ok = gc < K;
        cp_async16(As + j * kMCols + 8 * c8,
                   ok ? static_cast<const void*>(A + static_cast<int64_t>(s_sel[j]) * K + gc) : A, ok ? 16u : 0u);
      }
    }
    cp_async_commit();
#pragma unroll
    for (int j = 0; j < kMRT; ++j) {
      const int64_t n = r0 + tr * kMRT + j;
      const bool ok = col_ok && n < N;
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(wst + j * kMThreads + tid)),
                   "l"(ok ? wq + n * K + col : wq), "r"(ok ? 8u : 0u)
                   : "memory");
    }
    cp_async_commit();
    if (v + 1 < u_end) issue_q(v + 1, buf ^ 1);
    cp_async_commit();
    // (q, q) pairs of the first chunk, [j][row]
    const float* qsrc = qraw + buf * (kMChunk * kMRows);
    for (int e = tid; e < n0c * kMRows; e += kMThreads) Bs[e] = make_float2(qsrc[e], qsrc[e]);
    cp_async_wait_group<2>();  // A of the first chunk
    __syncthreads();           // As and Bs complete
    cur_cb = cb;

    float2 acc[kMRT][4];
#pragma unroll
    for (int j = 0; j < kMRT; ++j)
#pragma unroll
      for (int h = 0; h < 4; ++h) acc[j][h] = make_float2(0.0f, 0.0f);
    int nj = n0c;
    for (int j0 = 0;;) {
      const uint16_t* arow = As + 8 * lane;
      const float2* brow = Bs + tr * kMRT;
#pragma unroll 4
      for (int j = 0; j < nj; ++j) {
        const uint4 a4 = *reinterpret_cast<const uint4*>(arow + j * kMCols);
        const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w};
        float2 av[4];
#pragma unroll
        for (int h = 0; h < 4; ++h)
          av[h] = make_float2(__uint_as_float(aw[h] << 16), __uint_as_float(aw[h] & 0xFFFF0000u));
#pragma unroll
        for (int rr = 0; rr < kMRT; rr += 2) {
          const float4 q = *reinterpret_cast<const float4*>(brow + j * kMRows + rr);
          const float2 b0 = make_float2(q.x, q.y), b1 = make_float2(q.z, q.w);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            acc[rr][h] = __ffma2_rn(b0, av[h], acc[rr][h]);
            acc[rr + 1][h] = __ffma2_rn(b1, av[h], acc[rr + 1][h]);
          }
        }
      }
      j0 += nj;
      if (j0 >= ns) break;
      // a further chunk of components (more than kMChunk chosen): staged in place
      nj = ns - j0 < kMChunk ? ns - j0 : kMChunk;
      __syncthreads();  // every thread is done with As and Bs
      for (int e = tid; e < nj * (kMCols / 8); e += kMThreads) {
        const int j = e / (kMCols / 8), c8 = e % (kMCols / 8);
        const int64_t gc = c0 + 8 * c8;
        const bool ok = gc < K;
        const int64_t i = sel[j0 + j];
        cp_async16(As + j * kMCols + 8 * c8, ok ? static_cast<const void*>(A + i * K + gc) : A, ok ? 16u : 0u);
      }
      cp_async_commit();
      for (int e = tid; e < nj * kMRows; e += kMThreads) {
        const int j = e / kMRows, row = e % kMRows;
        const int64_t n = r0 + row;
        const float q = n < N ? Q[static_cast<int64_t>(sel[j0 + j]) * N + n] : 0.0f;
        Bs[j * kMRows + row] = make_float2(q, q);
      }
      cp_async_wait_all();
      __syncthreads();
    }
    cp_async_wait_group<1>();  // this thread's Wq slices (tile v+1's Q entries may still be in flight)
#pragma unroll
    for (int j = 0; j < kMRT; ++j) {
      const int64_t n = r0 + tr * kMRT + j;
      if (!(col_ok && n < N)) continue;
      const uint2 w = wst[j * kMThreads + tid];
      const float4 p0 = make_float4(acc[j][0].x, acc[j][0].y, acc[j][1].x, acc[j][1].y);
      const float4 p1 = make_float4(acc[j][2].x, acc[j][2].y, acc[j][3].x, acc[j][3].y);
      const uint32_t c0w = requantized4(w.x, s_w, p0);
      const uint32_t c1w = requantized4(w.y, s_w, p1);
      // identical words change only where they hold NaN codes (the common case)
      const uint32_t m0 = c0w == w.x ? nan_bytes(w.x) : changed_bytes(w.x, c0w);
      const uint32_t m1 = c1w == w.y ? nan_bytes(w.y) : changed_bytes(w.y, c1w);
      if (m0 | m1)
        *reinterpret_cast<uint2*>(wq + n * K + col) = make_uint2((c0w & m0) | (w.x & ~m0), (c1w & m1) | (w.y & ~m1));
    }
  }
  cp_async_wait_all();
}

__global__ void __launch_bounds__(kClearThreads)
    topk_clear_kernel(float* __restrict__ Q, int64_t N, const int32_t* __restrict__ sel,
                      const int32_t* __restrict__ n_sel) {
  pdl_trigger();
  pdl_wait();
  const int64_t ns = *n_sel;
  const int64_t total = ns * N;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * kClearThreads + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * kClearThreads) {
    const int64_t j = e / N, n = e % N;
    Q[static_cast<int64_t>(sel[j]) * N + n] = 0.0f;
  }
}

struct TopkWorkspace {
  uint32_t* partQ;  // [r][nq_x]
  uint32_t* partA;  // [r][kchunks]
  int32_t* sel;     // [r]
  int32_t* n_sel;   // [1]
};

TopkWorkspace topk_layout(void* ws, int64_t N, int64_t K, int64_t r, size_t* bytes) {
  const int64_t nq_x = (N + kAccN - 1) / kAccN, kchunks = (K + kAmaxCols - 1) / kAmaxCols;
  const size_t a = align_up(static_cast<size_t>(r) * static_cast<size_t>(nq_x) * 4, 256);
  const size_t b = align_up(static_cast<size_t>(r) * static_cast<size_t>(kchunks) * 4, 256);
  const size_t c = align_up(static_cast<size_t>(r) * 4, 256);
  TopkWorkspace t{};
  uint8_t* p = static_cast<uint8_t*>(ws);
  if (p) {
    t.partQ = reinterpret_cast<uint32_t*>(p);
    t.partA = reinterpret_cast<uint32_t*>(p + a);
    t.sel = reinterpret_cast<int32_t*>(p + a + b);
    t.n_sel = reinterpret_cast<int32_t*>(p + a + b + c);
  }
  if (bytes) *bytes = a + b + c + 256;
  return t;
}

// cudaFuncSetAttribute once per device ordinal below 31.
template <typename Kern>
cudaError_t ensure_smem(Kern* kernel, int bytes, int* configured_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int bit = dev < 31 ? (1 << dev) : 0;
  if (bit && (__atomic_load_n(configured_mask, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) __atomic_fetch_or(configured_mask, bit, __ATOMIC_ACQ_REL);
  return e;
}

}  // namespace

size_t proxy_topk_workspace_bytes(int64_t N, int64_t K, int64_t r) {
  size_t bytes = 0;
  topk_layout(nullptr, N, K, r, &bytes);
  return bytes;
}

cudaError_t launch_proxy_update_topk(uint8_t* wq, const float* s_w, float* Q, const void* dB_inc, const void* A,
                                     int64_t N, int64_t K, int64_t r, int64_t k, uint32_t flags,
                                     uint8_t* comp_mask, int32_t* n_selected, int32_t* dev_status,
                                     void* workspace, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  const bool acc = flags & 1u, sel = flags & 2u;
  if (r < 1 || r > kTopkMaxRank || N > (int64_t(1) << 31) - 1) return cudaErrorInvalidValue;
  const int rr = static_cast<int>(r);
  const int64_t nq_x = (N + kAccN - 1) / kAccN;
  const int64_t nq_blocks = nq_x * ((r + kAccI - 1) / kAccI);
  const int64_t kchunks = (K + kAmaxCols - 1) / kAmaxCols;
  const int64_t na_blocks = sel ? ((r + 7) / 8) * kchunks : 0;
  if (nq_blocks + na_blocks > (int64_t(1) << 31) - 1) return cudaErrorInvalidValue;
  const TopkWorkspace t = topk_layout(workspace, N, K, r, nullptr);
  // 1. Q += dB_inc^T, maxima of |Q| and |A|
  cudaError_t e = launch_pdl(topk_accum_kernel, dim3(static_cast<unsigned>(nq_blocks + na_blocks)),
                             dim3(kAccThreads), 0, stream, 1u, Q, static_cast<const uint16_t*>(dB_inc),
                             static_cast<const uint16_t*>(A), N, K, rr, acc ? 1 : 0, static_cast<int>(nq_x),
                             static_cast<int>(nq_blocks), static_cast<int>(kchunks), sel ? t.partQ : nullptr,
                             sel ? t.partA : nullptr);
  if (e != cudaSuccess || !sel) return e;
  // 2. scores and the chosen components
  static int sel_configured = 0;
  const int sel_smem = rr * 8;
  if (sel_smem > 48 * 1024) {
    e = ensure_smem(topk_select_kernel, sel_smem, &sel_configured);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(topk_select_kernel, dim3(1), dim3(kSelThreads), static_cast<size_t>(sel_smem), stream, 1u,
                 static_cast<const uint32_t*>(t.partQ), static_cast<int>(nq_x),
                 static_cast<const uint32_t*>(t.partA), static_cast<int>(kchunks), rr, k, comp_mask, n_selected,
                 t.sel, t.n_sel, dev_status);
  if (e != cudaSuccess || k == 0) return e;
  // 3. merge them into the codes
  static int merge_configured = 0;
  e = ensure_smem(topk_merge_kernel, kMSmemBytes, &merge_configured);
  if (e != cudaSuccess) return e;
  const int64_t row_groups = (N + kMRows - 1) / kMRows;
  const int64_t units = row_groups * ((K + kMCols - 1) / kMCols);
  if (units > (int64_t(1) << 30)) return cudaErrorInvalidValue;
  const int64_t resident = static_cast<int64_t>(kMCtasPerSm) * di->sm_count;
  const int grid = static_cast<int>(units < resident ? units : resident);
  e = launch_pdl(topk_merge_kernel, dim3(grid), dim3(kMThreads), kMSmemBytes, stream, 1u, wq, s_w,
                 static_cast<const float*>(Q), static_cast<const uint16_t*>(A), N, K,
                 static_cast<const int32_t*>(t.sel), static_cast<const int32_t*>(t.n_sel),
                 static_cast<int>(row_groups), static_cast<int>(units));
  if (e != cudaSuccess) return e;
  // 4. clear their rows of Q
  const int64_t kk = k < r ? k : r;
  const int64_t work = (kk * N + kClearThreads - 1) / kClearThreads;
  const int64_t cap = static_cast<int64_t>(di->sm_count) * 4;
  const int cgrid = static_cast<int>(work < 1 ? 1 : (work < cap ? work : cap));
  return launch_pdl(topk_clear_kernel, dim3(cgrid), dim3(kClearThreads), 0, stream, 1u, Q, N,
                    static_cast<const int32_t*>(t.sel), static_cast<const int32_t*>(t.n_sel));
}

}  // namespace falqon
