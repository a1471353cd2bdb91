// Block-selection bitmap -> route IDs.
//
// The cuDNN-Frontend "Query Sparse Attention (QSA)" page ("Tensors", "Selection
// and components") specifies selection by a bitmap sel_blocks [T, NB] and
// per-query metadata: key token j is allowed for query t iff
// lo[t] <= j <= hi[t], 0 <= b < NB and sel_blocks[t, b] != 0, where
// b = blk_base[t] + floor((j - tok_base[t]) / block_size).  The allowed set of a
// query is a route set, so route-set QSA over the converted rows is the bitmap
// API's attention.
//
// One warp per query row.  Only the blocks that keys inside [lo, hi] can map to
// are read: b in [blk_base + floor((max(lo, 0) - tok_base) / bs),
// blk_base + floor((min(hi, T_kv - 1) - tok_base) / bs)] clipped to [0, NB).  The
// warp walks that range 128 blocks per pass (4 consecutive blocks per lane);
// each selected block contributes its tokens clipped to [lo, hi]; a warp prefix
// sum places them, so every row comes out ascending.  Rows longer than n_sel
// keep their n_sel smallest keys; row_cnt reports the true size.
#include "qsa_internal.h"

namespace qsa {
namespace {

__device__ __forceinline__ int64_t floor_div(int64_t a, int64_t b) {  // b > 0
  return a >= 0 ? a / b : -((-a + b - 1) / b);
}

__global__ void __launch_bounds__(256)
bitmap_routes_kernel(const uint8_t* __restrict__ sel, const int32_t* __restrict__ lo,
                     const int32_t* __restrict__ hi, const int32_t* __restrict__ blk_base,
                     const int32_t* __restrict__ tok_base, int64_t T, int64_t NB, int64_t T_kv, int bs, int n_sel,
                     int32_t* __restrict__ routes, int32_t* __restrict__ row_cnt, int32_t* __restrict__ max_cnt) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  const int64_t jlo = max(static_cast<int64_t>(__ldg(lo + t)), int64_t{0});
  const int64_t jhi = min(static_cast<int64_t>(__ldg(hi + t)), T_kv - 1);
  const int64_t bb = __ldg(blk_base + t), tb = __ldg(tok_base + t);
  int32_t* out = routes + t * n_sel;
  const uint8_t* row = sel + t * NB;
  int64_t cnt = 0;
  if (jlo <= jhi) {
    const int64_t b_lo = max(bb + floor_div(jlo - tb, bs), int64_t{0});
    const int64_t b_hi = min(bb + floor_div(jhi - tb, bs), NB - 1);
    for (int64_t p = b_lo; p <= b_hi; p += 128) {
      // this lane's 4 blocks: p + 4 lane .. p + 4 lane + 3
      int n[4];
      int64_t first[4];
      int total = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t b = p + 4 * lane + i;
        n[i] = 0;
        first[i] = 0;
        if (b <= b_hi && __ldg(row + b) != 0) {
          // tokens j with floor((j - tb) / bs) == b - bb, clipped to [jlo, jhi]
          const int64_t s = tb + (b - bb) * bs;
          const int64_t a = max(s, jlo), e = min(s + bs - 1, jhi);
          if (a <= e) {
            n[i] = static_cast<int>(e - a + 1);
            first[i] = a;
          }
        }
        total += n[i];
      }
      // warp exclusive prefix sum of the lane totals
      int incl = total;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += x;
      }
      int64_t pos = cnt + (incl - total);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        for (int k = 0; k < n[i]; ++k, ++pos)
          if (pos < n_sel) out[pos] = static_cast<int32_t>(first[i] + k);
      cnt += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  for (int64_t i = min(cnt, static_cast<int64_t>(n_sel)) + lane; i < n_sel; i += 32) out[i] = -1;
  if (lane == 0) {
    const int32_t c = static_cast<int32_t>(min(cnt, static_cast<int64_t>(INT32_MAX)));
    if (row_cnt) row_cnt[t] = c;
    if (max_cnt) atomicMax(max_cnt, c);
  }
}

}  // namespace

cudaError_t launch_bitmap_routes(const uint8_t* sel, const int32_t* lo, const int32_t* hi, const int32_t* blk_base,
                                 const int32_t* tok_base, int64_t T, int64_t NB, int64_t T_kv, int block_size,
                                 int n_sel, int32_t* routes, int32_t* row_cnt, int32_t* max_cnt, cudaStream_t s) {
  if (max_cnt) {
    cudaError_t e = cudaMemsetAsync(max_cnt, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  const int64_t blocks = (T + 7) / 8;  // 8 rows (warps) per 256-thread block
  bitmap_routes_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(sel, lo, hi, blk_base, tok_base, T, NB, T_kv,
                                                                      block_size, n_sel, routes, row_cnt, max_cnt);
  return cudaGetLastError();
}

}  // namespace qsa
