// Route preprocessing for exact route-set QSA.
//
// Route membership is a set: invalid IDs (negative or >= T_kv) are padding and
// duplicates collapse ("fa4_qsa" page, `_preprocess`; "flex_qsa" page,
// `_routes_to_membership`).  These kernels turn the raw [T, n_sel] routes into
//   * per-row ascending de-duplicated lists (row_cnt, row_cols), consumed by the
//     per-query forward and dQ kernels, and
//   * the key->query transpose at the granularity of aligned key quads
//     (quad_ptr, quad_ent), each list in ascending query order, consumed by the
//     per-quad dK/dV kernel.  A fixed list order makes the dK/dV summation order,
//     and so its result bits, independent of scheduling.
#include <climits>

#include "qsa_device.cuh"
#include "qsa_internal.h"

namespace qsa {
namespace {

constexpr int kRowThreads = 256;
constexpr int kSortThreads = 256;
constexpr int kSortCap = 4096;  // int64 entries sorted in shared memory (32 KB)

// Ascending bitonic sort of s[0, n2) where n2 is a power of two and elements at
// or beyond `len` are treated as +infinity (never read or written).  Every
// comparator moves the smaller value to the lower index (the "flip" form of the
// bitonic merge), so the virtual padding at the end never has to move.  All
// threads of the block must call it.  `T` is int32_t or int64_t; `s` may point
// to shared or global memory (global memory writes are ordered by the
// __syncthreads between steps).
template <typename T>
__device__ void block_sort(T* s, int64_t len, int64_t n2) {
  const int64_t half_n = n2 >> 1;
  for (int64_t k = 2; k <= n2; k <<= 1) {
    const int64_t half = k >> 1;
    for (int64_t p = threadIdx.x; p < half_n; p += blockDim.x) {
      const int64_t blk = p / half, off = p - blk * half;
      const int64_t i = blk * k + off, j = blk * k + (k - 1 - off);
      if (j < len) {
        const T a = s[i], b = s[j];
        if (b < a) { s[i] = b; s[j] = a; }
      }
    }
    __syncthreads();
    for (int64_t h = half >> 1; h >= 1; h >>= 1) {
      for (int64_t p = threadIdx.x; p < half_n; p += blockDim.x) {
        const int64_t i = (p / h) * 2 * h + (p % h), j = i + h;
        if (j < len) {
          const T a = s[i], b = s[j];
          if (b < a) { s[i] = b; s[j] = a; }
        }
      }
      __syncthreads();
    }
  }
}

// Exclusive prefix sum of one int per thread over the block; returns the
// thread's offset and writes the block total to *total.
__device__ int block_exclusive_scan(int x, int* scratch /* >= 32 ints */, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nwarps) scratch[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int base = warp > 0 ? scratch[warp - 1] : 0;
  *total = scratch[nwarps - 1];
  __syncthreads();
  return base + incl - x;
}

// One block per query row: filter invalid IDs, sort, de-duplicate, compact.
__global__ void __launch_bounds__(kRowThreads) route_rows_kernel(
    const int32_t* __restrict__ routes, int32_t T_kv, int n_sel, int n2,
    int32_t* __restrict__ row_cnt, int32_t* __restrict__ row_cols, int32_t* __restrict__ quad_cnt) {
  extern __shared__ int32_t sv[];  // n2 values, then 32 ints of scan scratch
  int* scratch = sv + n2;
  const int64_t t = blockIdx.x;
  const int32_t* row = routes + t * n_sel;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    int32_t x = INT_MAX;
    if (i < n_sel) {
      const int32_t r = row[i];
      if (r >= 0 && r < T_kv) x = r;
    }
    sv[i] = x;
  }
  __syncthreads();
  block_sort<int32_t>(sv, n2, n2);

  // Each thread owns a contiguous run of the sorted values.
  const int per = (n2 + blockDim.x - 1) / blockDim.x;
  const int lo = min(n2, static_cast<int>(threadIdx.x) * per), hi = min(n2, lo + per);
  int mine = 0;
  for (int i = lo; i < hi; ++i) {
    const int32_t x = sv[i];
    if (x != INT_MAX && (i == 0 || sv[i - 1] != x)) {
      ++mine;
      if (quad_cnt != nullptr && (i == 0 || (sv[i - 1] >> 2) != (x >> 2))) atomicAdd(quad_cnt + (x >> 2), 1);
    }
  }
  int total;
  int pos = block_exclusive_scan(mine, scratch, &total);
  int32_t* out = row_cols + t * n_sel;
  for (int i = lo; i < hi; ++i) {
    const int32_t x = sv[i];
    if (x != INT_MAX && (i == 0 || sv[i - 1] != x)) out[pos++] = x;
  }
  if (threadIdx.x == 0) row_cnt[t] = total;
}

// Single block: exclusive scan of quad counts (n_quads + 1 offsets).
__global__ void __launch_bounds__(1024) quad_scan_kernel(const int32_t* __restrict__ cnt, int64_t n,
                                                         int32_t* __restrict__ ptr, int32_t* __restrict__ fill) {
  __shared__ int scratch[32];
  const int64_t per = (n + blockDim.x - 1) / blockDim.x;
  const int64_t lo = min(n, static_cast<int64_t>(threadIdx.x) * per), hi = min(n, lo + per);
  int mine = 0;
  for (int64_t i = lo; i < hi; ++i) mine += cnt[i];
  int total;
  int run = block_exclusive_scan(mine, scratch, &total);
  for (int64_t i = lo; i < hi; ++i) {
    ptr[i] = run;
    fill[i] = run;
    run += cnt[i];
  }
  if (threadIdx.x == 0) ptr[n] = total;
}

// One warp per row: emit one entry per key quad the row meets.
__global__ void __launch_bounds__(256) quad_fill_kernel(const int32_t* __restrict__ row_cnt,
                                                        const int32_t* __restrict__ row_cols, int64_t T,
                                                        int n_sel, int32_t* __restrict__ fill,
                                                        int64_t* __restrict__ ent) {
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int cnt = row_cnt[t];
  const int32_t* cols = row_cols + t * n_sel;
  for (int i = lane; i < cnt; i += 32) {
    const int32_t x = cols[i];
    const int32_t qd = x >> 2;
    if (i == 0 || (cols[i - 1] >> 2) != qd) {
      int mask = 1 << (x & 3);
#pragma unroll
      for (int d = 1; d < 4; ++d) {
        if (i + d < cnt) {
          const int32_t y = cols[i + d];
          if ((y >> 2) == qd) mask |= 1 << (y & 3);
        }
      }
      const int p = atomicAdd(fill + qd, 1);
      ent[p] = (t << 32) | (static_cast<int64_t>(i) << 4) | mask;
    }
  }
}

// One block per quad: sort its list ascending (by query, the high word).
__global__ void __launch_bounds__(kSortThreads) quad_sort_kernel(const int32_t* __restrict__ ptr,
                                                                 int64_t* __restrict__ ent) {
  __shared__ int64_t sv[kSortCap];
  const int64_t b = blockIdx.x;
  const int64_t lo = ptr[b], len = ptr[b + 1] - lo;
  if (len <= 1) return;
  int64_t n2 = 1;
  while (n2 < len) n2 <<= 1;
  int64_t* seg = ent + lo;
  if (n2 <= kSortCap) {
    for (int64_t i = threadIdx.x; i < n2; i += blockDim.x) sv[i] = i < len ? seg[i] : LLONG_MAX;
    __syncthreads();
    block_sort<int64_t>(sv, n2, n2);
    for (int64_t i = threadIdx.x; i < len; i += blockDim.x) seg[i] = sv[i];
  } else {
    block_sort<int64_t>(seg, len, n2);  // in place, in global memory
  }
}

int next_pow2(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

}  // namespace

cudaError_t launch_route_rows(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel, int32_t* row_cnt,
                              int32_t* row_cols, int32_t* quad_cnt, cudaStream_t s) {
  const int n2 = next_pow2(n_sel < 2 ? 2 : n_sel);
  const size_t smem = static_cast<size_t>(n2 + 32) * sizeof(int32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  route_rows_kernel<<<static_cast<unsigned>(T), kRowThreads, smem, s>>>(
      routes, static_cast<int32_t>(T_kv), n_sel, n2, row_cnt, row_cols, quad_cnt);
  return cudaGetLastError();
}

cudaError_t launch_quad_scan(const int32_t* quad_cnt, int64_t n_quads, int32_t* quad_ptr, int32_t* quad_fill,
                             cudaStream_t s) {
  quad_scan_kernel<<<1, 1024, 0, s>>>(quad_cnt, n_quads, quad_ptr, quad_fill);
  return cudaGetLastError();
}

cudaError_t launch_quad_fill(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int n_sel,
                             int32_t* quad_fill, int64_t* quad_ent, cudaStream_t s) {
  const int64_t blocks = (T * 32 + 255) / 256;
  quad_fill_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(row_cnt, row_cols, T, n_sel, quad_fill, quad_ent);
  return cudaGetLastError();
}

cudaError_t launch_quad_sort(const int32_t* quad_ptr, int64_t n_quads, int64_t* quad_ent, cudaStream_t s) {
  quad_sort_kernel<<<static_cast<unsigned>(n_quads), kSortThreads, 0, s>>>(quad_ptr, quad_ent);
  return cudaGetLastError();
}

}  // namespace qsa
