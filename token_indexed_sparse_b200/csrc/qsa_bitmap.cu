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
// warp walks that range with 16-byte loads (16 blocks per lane, 512 per pass,
// four passes in flight); each selected block contributes its tokens clipped
// to [lo, hi]; a warp prefix sum places them, so every row comes out ascending.
// Rows longer than n_sel keep their n_sel smallest keys; row_cnt reports the
// true size.
#include "qsa_internal.h"

namespace qsa {
namespace {

__device__ __forceinline__ int64_t floor_div(int64_t a, int64_t b) {  // b > 0
  return a >= 0 ? a / b : -((-a + b - 1) / b);
}
__device__ __forceinline__ int kBlkOff(int lane) { return 16 * lane; }

constexpr int kBmBlkPerLane = 16;                  // one 16-byte load per lane
constexpr int kBmPass = 32 * kBmBlkPerLane;        // 512 blocks per warp pass
constexpr int kBmUnroll = 4;                       // passes loaded before any is scanned

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
  const uint8_t* sel_end = sel + T * NB;
  int64_t cnt = 0;
  if (jlo <= jhi) {
    const int64_t b_lo = max(bb + floor_div(jlo - tb, bs), int64_t{0});
    const int64_t b_hi = min(bb + floor_div(jhi - tb, bs), NB - 1);
    // passes start at a 16-byte aligned address at or before block b_lo (the
    // bytes before b_lo and after b_hi are loaded but never selected); every
    // load stays inside the bitmap: its base is 16-byte aligned (checked by the
    // C ABI) and the last partial vector is read byte by byte
    const uint8_t* a0 = reinterpret_cast<const uint8_t*>(reinterpret_cast<uintptr_t>(row + b_lo) & ~uintptr_t{15});
    const int64_t b0 = a0 - row;  // block index of a0's first byte (may be negative)
    for (int64_t p = b0; p <= b_hi; p += int64_t{kBmPass} * kBmUnroll) {
      uint4 w[kBmUnroll];
#pragma unroll
      for (int u = 0; u < kBmUnroll; ++u) {
        const uint8_t* a = row + p + int64_t{u} * kBmPass + kBlkOff(lane);
        w[u] = make_uint4(0, 0, 0, 0);
        if (p + int64_t{u} * kBmPass + kBlkOff(lane) <= b_hi) {
          if (a + 16 <= sel_end) {
            w[u] = __ldg(reinterpret_cast<const uint4*>(a));
          } else {  // the bitmap's last partial vector: byte loads up to its end
            uint32_t x[4] = {0, 0, 0, 0};
            for (int i = 0; a + i < sel_end; ++i) x[i >> 2] |= static_cast<uint32_t>(__ldg(a + i)) << (8 * (i & 3));
            w[u] = make_uint4(x[0], x[1], x[2], x[3]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kBmUnroll; ++u) {
        // 32-bit arithmetic relative to the row: block r = base + i - b_lo covers
        // tokens [f0 + bs r, f0 + bs r + bs - 1] clipped to [jlo, jhi], where
        // f0 = tok_base + bs (b_lo - blk_base) (all inside int32: keys < T_kv)
        const int64_t base = p + int64_t{u} * kBmPass + kBlkOff(lane);  // this lane's first block
        const uint32_t words[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        const int rb = static_cast<int>(base - b_lo);                    // may be negative
        const int nrel = static_cast<int>(b_hi - b_lo);
        const int lo32 = static_cast<int>(jlo), hi32 = static_cast<int>(jhi);
        const int64_t f0l = tb + (b_lo - bb) * bs;                        // first token of block b_lo
        const int f0 = static_cast<int>(max(min(f0l, int64_t{INT32_MAX}), int64_t{INT32_MIN + 1}));
        uint32_t selmask = 0;
        int total = 0;
#pragma unroll
        for (int i = 0; i < kBmBlkPerLane; ++i) {
          const int r = rb + i;
          const bool on = ((words[i >> 2] >> (8 * (i & 3))) & 0xffu) != 0 && r >= 0 && r <= nrel;
          if (on) {
            const int s0 = f0 + bs * r;
            const int a = max(s0, lo32), e = min(s0 + bs - 1, hi32);
            if (a <= e) {
              selmask |= 1u << i;
              total += e - a + 1;
            }
          }
        }
        int incl = total;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int x = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += x;
        }
        int64_t pos = cnt + (incl - total);
        while (selmask) {
          const int i = __ffs(selmask) - 1;
          selmask &= selmask - 1;
          const int s0 = f0 + bs * (rb + i);
          const int a = max(s0, lo32), e = min(s0 + bs - 1, hi32);
          for (int j = a; j <= e; ++j, ++pos)
            if (pos < n_sel) out[pos] = j;
        }
        cnt += __shfl_sync(0xffffffffu, incl, 31);
      }
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
