// Route preprocessing for exact route-set QSA.
//
// Route membership is a set: invalid IDs (negative or >= T_kv) are padding and
// duplicates collapse ("fa4_qsa" page, `_preprocess`; "flex_qsa" page,
// `_routes_to_membership`).  These kernels turn the raw [T, n_sel] routes into
//   * per-row ascending de-duplicated lists (row_cnt, row_cols), consumed by the
//     per-query forward and dQ kernels,
//   * the key->query transpose over aligned 128-key tiles (tile_ptr, tile_ent:
//     one entry per (row, tile) naming the row's run of keys in the tile), each
//     list written directly in ascending query order (no sort), and the
//     per-phase work lists the dK/dV kernel claims its units from, and
//   * the same transpose over aligned key quads with 4-bit owner masks
//     (quad_ptr, quad_ent), exposed by qsa_route_plan, and
//   * the query-union lists of adjacent rows (qsa_union_plan).
// Rows are sorted by a warp in registers (bitonic networks over shfl.xor) up to
// 1024 slots, 513-768 slots as 512 + the rest merged in shared memory, and by a
// CTA above 1024 (register-sorted 256-slot chunks, merge-path rounds).  The
// forward's lists stay in its workspace with a tag of their sizes, so that the
// backward can reuse them (row_delta_masks_kernel) instead of sorting again.
// A fixed list order makes the dK/dV summation order, and so its result bits,
// independent of scheduling.
#include <climits>

#include "qsa_device.cuh"
#include "qsa_internal.h"

namespace qsa {
namespace {

constexpr int kRowThreads = 256;
constexpr int kSortThreads = 256;
constexpr int kSortCap = 4096;  // int64 entries sorted in shared memory (32 KB)
constexpr int kMaxUnionGroup = 8;  // rows per union group at most

// Ascending bitonic sort of s[0, n2) where n2 is a power of two and elements at
// or beyond `len` are treated as +infinity (never read or written).  Every
// comparator moves the smaller value to the lower index (the "flip" form of the
// bitonic merge), so the virtual padding at the end never has to move.  All
// threads of the block must call it.  `T` is int32_t or int64_t; `s` may point
// to shared or global memory (global memory writes are ordered by the
// __syncthreads between steps).  Index arithmetic is 32-bit shifts and masks:
// n2 <= 2^30.
template <typename T>
__device__ void block_sort(T* s, int len, int n2) {
  const int half_n = n2 >> 1;
  for (int lk = 1; (1 << lk) <= n2; ++lk) {
    const int k = 1 << lk, lh = lk - 1;
    for (int p = threadIdx.x; p < half_n; p += blockDim.x) {
      const int off = p & ((1 << lh) - 1);
      const int base = (p >> lh) << lk;
      const int i = base + off, j = base + (k - 1 - off);
      if (j < len) {
        const T a = s[i], b = s[j];
        if (b < a) { s[i] = b; s[j] = a; }
      }
    }
    __syncthreads();
    for (int lg = lh - 1; lg >= 0; --lg) {
      for (int p = threadIdx.x; p < half_n; p += blockDim.x) {
        const int i = ((p >> lg) << (lg + 1)) | (p & ((1 << lg) - 1)), j = i + (1 << lg);
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

// Ascending bitonic sort of the 32*NPL values a warp holds in registers
// (element e = lane * NPL + r lives in v[r] of lane e / NPL).  Same "flip" network
// as block_sort: comparators whose partner is in another lane exchange values
// with shfl.xor, the others compare registers of one lane.  Fully unrolled.
template <int NPL>
__device__ __forceinline__ void warp_sort(int32_t (&v)[NPL], int lane) {
#pragma unroll
  for (int k = 2; k <= 32 * NPL; k <<= 1) {
    // flip step: e <-> e ^ (k - 1)
    if (k <= NPL) {
#pragma unroll
      for (int r = 0; r < NPL; ++r) {
        const int p = r ^ (k - 1);
        if (p > r) {
          const int32_t a = v[r], b = v[p];
          v[r] = min(a, b);
          v[p] = max(a, b);
        }
      }
    } else {
      // partner of (lane, r) is (lane ^ m, r ^ (NPL - 1)); the lower half of the
      // k-block (bit k/2 of the element index clear) keeps the minimum
      const int m = k / NPL - 1;
      const bool lower = (lane & (k / (2 * NPL))) == 0;
      if (NPL == 1) {  // register 0 pairs with register 0 of lane ^ m
        const int32_t t = __shfl_xor_sync(0xffffffffu, v[0], m);
        v[0] = lower ? min(v[0], t) : max(v[0], t);
      }
#pragma unroll
      for (int r = 0; r < NPL / 2; ++r) {
        const int r2 = NPL - 1 - r;
        const int32_t x = v[r], y = v[r2];
        const int32_t tx = __shfl_xor_sync(0xffffffffu, y, m);  // partner of register r
        const int32_t ty = __shfl_xor_sync(0xffffffffu, x, m);  // partner of register r2
        v[r] = lower ? min(x, tx) : max(x, tx);
        v[r2] = lower ? min(y, ty) : max(y, ty);
      }
    }
    // half-cleaners: e <-> e ^ h
#pragma unroll
    for (int h = k / 4; h >= 1; h >>= 1) {
      if (h < NPL) {
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
          if ((r & h) == 0) {
            const int32_t a = v[r], b = v[r | h];
            v[r] = min(a, b);
            v[r | h] = max(a, b);
          }
        }
      } else {
        const int m = h / NPL;
        const bool lower = (lane & m) == 0;
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
          const int32_t t = __shfl_xor_sync(0xffffffffu, v[r], m);
          v[r] = lower ? min(v[r], t) : max(v[r], t);
        }
      }
    }
  }
}

// Keys per 128-key tile: 2^kTileShift.  Query rows form blocks of kBlockRows
// for the tile masks (one 64-bit mask per block and tile).
constexpr int kTileShift = 7;
constexpr int kBlockRows = 64;
constexpr int kRowWarps = 8;  // rows (warps) per CTA of route_rows_warp_kernel

// Route-list tag: a route kernel that zeroes a call's status word also writes,
// in words 4..7 of the same 256-byte slot, {kPlanMagic, T, T_kv, n_sel}, so a
// later call that reuses the route lists (qsa_backward_saved) can check, on the
// device, that they come from a route kernel run on rows of these sizes.
constexpr int32_t kPlanMagic = 0x51534131;
__device__ __forceinline__ void write_plan_tag(int* status, int64_t T, int32_t T_kv, int n_sel) {
  status[0] = 0;
  status[4] = kPlanMagic;
  status[5] = static_cast<int32_t>(T);
  status[6] = T_kv;
  status[7] = n_sel;
}

// Sets row t's bit in the mask of (its 64-row block, 128-key tile tl); the
// masks [ceil(T / 64), n_tiles] are zeroed by the caller.
__device__ __forceinline__ void mark_tile(unsigned long long* masks, int64_t n_tiles, int64_t t, int32_t tl) {
  static_assert(kBlockRows == 64, "one 64-bit mask per block of rows");
  atomicOr(masks + (t / kBlockRows) * n_tiles + tl, 1ull << (t % kBlockRows));
}

// delta[t, h] = rowsum(dO * out) for heads h0 .. h0 + 3 of row t, h0 = first,
// first + step, ... below H (H a multiple of 4), by one warp with the four
// heads' loads in flight together.
__device__ __forceinline__ void row_delta(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
                                          float* __restrict__ delta, int64_t t, int H, int lane, int first, int step) {
  for (int h0 = first; h0 < H; h0 += step) {
    uint4 a[4], b[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t off = (t * H + h0 + j) * kHeadDim + lane * 8;
      a[j] = __ldg(reinterpret_cast<const uint4*>(dout + off));
      b[j] = __ldg(reinterpret_cast<const uint4*>(out + off));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float x = bf16_lo(a[j].x) * bf16_lo(b[j].x) + bf16_hi(a[j].x) * bf16_hi(b[j].x) +
                bf16_lo(a[j].y) * bf16_lo(b[j].y) + bf16_hi(a[j].y) * bf16_hi(b[j].y) +
                bf16_lo(a[j].z) * bf16_lo(b[j].z) + bf16_hi(a[j].z) * bf16_hi(b[j].z) +
                bf16_lo(a[j].w) * bf16_lo(b[j].w) + bf16_hi(a[j].w) * bf16_hi(b[j].w);
      x = warp_sum(x);
      if (lane == 0) delta[t * H + h0 + j] = x;
    }
  }
}

// Emits a warp's sorted values (element e = lane * NPL + r in v[r], +infinity
// as INT_MAX at the end): de-duplicates and compacts them to dst, and
// optionally adds per-bucket row counts (a bucket is 2^cnt_shift consecutive
// keys) and sets the row's bits in the tile masks.  Returns the row's count.
template <int NPL>
__device__ __forceinline__ int emit_sorted(const int32_t (&v)[NPL], int lane, int64_t t, int32_t* __restrict__ dst,
                                           int32_t* __restrict__ quad_cnt, int cnt_shift,
                                           unsigned long long* __restrict__ masks, int64_t n_tiles) {
  // the previous element of v[0] is the previous lane's v[NPL - 1]
  int32_t prev = __shfl_up_sync(0xffffffffu, v[NPL - 1], 1);
  if (lane == 0) prev = INT_MIN;
  int mine = 0;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const int32_t p = r == 0 ? prev : v[r - 1];
    const int32_t x = v[r];
    if (x != INT_MAX && x != p) {
      ++mine;
      if (quad_cnt != nullptr && (p == INT_MIN || (p >> cnt_shift) != (x >> cnt_shift)))
        atomicAdd(quad_cnt + (x >> cnt_shift), 1);
      if (masks != nullptr && (p == INT_MIN || (p >> kTileShift) != (x >> kTileShift)))
        mark_tile(masks, n_tiles, t, x >> kTileShift);
    }
  }
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int pos = incl - mine;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const int32_t p = r == 0 ? prev : v[r - 1];
    const int32_t x = v[r];
    if (x != INT_MAX && x != p) dst[pos++] = x;
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

// Loads slots [first, first + 32 * NPL) of a route row into registers
// (coalesced: slot first + r * 32 + lane in v[r]; the sort does not care where
// a value starts), invalid IDs and slots past n_sel as INT_MAX.
template <int NPL>
__device__ __forceinline__ void load_slots(int32_t (&v)[NPL], const int32_t* __restrict__ row, int first, int n_sel,
                                           int32_t T_kv, int lane) {
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const int i = first + r * 32 + lane;
    int32_t x = INT_MAX;
    if (i < n_sel) {
      const int32_t y = __ldg(row + i);
      if (y >= 0 && y < T_kv) x = y;
    }
    v[r] = x;
  }
}

// One warp per query row (rows of up to 32*NPL route slots): filter, sort in
// registers, de-duplicate, compact; optionally per-bucket row counts, the
// row's bits in the tile masks, and delta.
// (A shared-memory bitmap of the row's key range in place of the sort, with
// word popcounts scanned across the warp, ran the seq32k rows in 0.30 ms
// against 0.25 ms for this sort: the bit-by-bit read-back diverges across lanes.)
template <int NPL>
__global__ void __launch_bounds__(kRowWarps * 32, 3) route_rows_warp_kernel(
    const int32_t* __restrict__ routes, int64_t T, int32_t T_kv, int n_sel, int32_t* __restrict__ row_cnt,
    int32_t* __restrict__ row_cols, int32_t* __restrict__ quad_cnt, int cnt_shift, int* __restrict__ status,
    const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out, float* __restrict__ delta,
    int H, unsigned long long* __restrict__ masks, int64_t n_tiles) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) write_plan_tag(status, T, T_kv, n_sel);
  if (t >= T) return;
  int32_t v[NPL];
  load_slots<NPL>(v, routes + t * n_sel, 0, n_sel, T_kv, lane);
  warp_sort<NPL>(v, lane);
  const int cnt = emit_sorted<NPL>(v, lane, t, row_cols + t * n_sel, quad_cnt, cnt_shift, masks, n_tiles);
  if (lane == 0) row_cnt[t] = cnt;
  if (delta != nullptr) row_delta(dout, out, delta, t, H, lane, 0, 4);
}

// Rows of 513 .. 512 + 32 * NB slots (NB <= 8): the first 512 slots and the
// rest are sorted apart in registers (bitonic networks of 512 and 32 NB
// elements, about 40-95 % fewer compare-exchanges than one network of 1024),
// stored to shared memory and merged: lane l produces the merged elements
// l * (16 + NB) ... of the stable merge (ties from the first part first), its
// split of the two parts found by a binary search on its diagonal.
constexpr int kSplitA = 512;
template <int NB>
__global__ void __launch_bounds__(kRowWarps * 32, 3) route_rows_split_kernel(
    const int32_t* __restrict__ routes, int64_t T, int32_t T_kv, int n_sel, int32_t* __restrict__ row_cnt,
    int32_t* __restrict__ row_cols, int32_t* __restrict__ quad_cnt, int cnt_shift, int* __restrict__ status,
    const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out, float* __restrict__ delta,
    int H, unsigned long long* __restrict__ masks, int64_t n_tiles) {
  constexpr int NA = kSplitA / 32, kLenB = 32 * NB, kPer = NA + NB;
  __shared__ int32_t parts[kRowWarps][kSplitA + kLenB];
  const int lane = threadIdx.x & 31;
  int32_t* sa = parts[threadIdx.x >> 5];
  int32_t* sb = sa + kSplitA;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) write_plan_tag(status, T, T_kv, n_sel);
  if (t >= T) return;
  const int32_t* row = routes + t * n_sel;
  {
    int32_t a[NA];
    load_slots<NA>(a, row, 0, n_sel, T_kv, lane);
    warp_sort<NA>(a, lane);
#pragma unroll
    for (int r = 0; r < NA; ++r) sa[lane * NA + r] = a[r];
  }
  {
    int32_t b[NB];
    load_slots<NB>(b, row, kSplitA, n_sel, T_kv, lane);
    warp_sort<NB>(b, lane);
#pragma unroll
    for (int r = 0; r < NB; ++r) sb[lane * NB + r] = b[r];
  }
  __syncwarp();
  // merge path: the first d merged elements take i from the first part and
  // d - i from the second, i the least value with sa[i] > sb[d - i - 1]
  const int d = lane * kPer;
  int lo = d > kLenB ? d - kLenB : 0, hi = d < kSplitA ? d : kSplitA;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (sa[mid] <= sb[d - mid - 1]) lo = mid + 1;
    else hi = mid;
  }
  int ia = lo, ib = d - lo;
  int32_t v[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int32_t x = ia < kSplitA ? sa[ia] : INT_MAX;
    const int32_t y = ib < kLenB ? sb[ib] : INT_MAX;
    const bool take_a = ib >= kLenB || (ia < kSplitA && x <= y);
    v[r] = take_a ? x : y;
    ia += take_a ? 1 : 0;
    ib += take_a ? 0 : 1;
  }
  const int cnt = emit_sorted<kPer>(v, lane, t, row_cols + t * n_sel, quad_cnt, cnt_shift, masks, n_tiles);
  if (lane == 0) row_cnt[t] = cnt;
  if (delta != nullptr) row_delta(dout, out, delta, t, H, lane, 0, 4);
}

// The backward's route work when the forward's row lists are at hand (same
// routes): no sort, only delta and the row's tile-mask bits, a tile run
// starting wherever a key's tile differs from the previous key's.  One warp
// per row.
__global__ void __launch_bounds__(256) row_delta_masks_kernel(
    const int32_t* __restrict__ row_cnt, const int32_t* __restrict__ row_cols, int64_t T, int32_t T_kv, int n_sel,
    const int* __restrict__ plan_tag, int* __restrict__ status, const __nv_bfloat16* __restrict__ dout,
    const __nv_bfloat16* __restrict__ out, float* __restrict__ delta, int H, unsigned long long* __restrict__ masks,
    int64_t n_tiles) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  // the lists must carry the tag of rows of these sizes; without it nothing
  // reads them (here, in the tile fill or in dQ: those see the status word)
  const bool ok = plan_tag[4] == kPlanMagic && plan_tag[5] == static_cast<int32_t>(T) && plan_tag[6] == T_kv &&
                  plan_tag[7] == n_sel;
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = ok ? 0 : kStatusBadPlan;
  if (t >= T || !ok) return;
  const int cnt = row_cnt[t];
  const int32_t* cols = row_cols + t * n_sel;
  int32_t carry = -1;  // tile of the last key of the previous 32 (none: -1)
  for (int base = 0; base < cnt; base += 32) {
    const int i = base + lane;
    const int32_t tl = i < cnt ? (__ldg(cols + i) >> kTileShift) : INT_MAX;
    int32_t prev = __shfl_up_sync(0xffffffffu, tl, 1);
    if (lane == 0) prev = carry;
    carry = __shfl_sync(0xffffffffu, tl, 31);
    if (i < cnt && tl != prev) mark_tile(masks, n_tiles, t, tl);
  }
  row_delta(dout, out, delta, t, H, lane, 0, 4);
}

// Sorts a row of n2 slots (n2 a power of two >= 2048, slots past n_sel and
// invalid IDs as INT_MAX) with the CTA's 8 warps: every 256-slot chunk is
// sorted in registers by one warp (warp_sort), then rounds of pairwise merges
// double the sorted runs until one remains, each thread producing n2 / 256
// consecutive outputs of its pair of runs after a binary search on its
// diagonal (merge path).  b0 and b1 are n2 ints each of shared memory; returns
// the one holding the sorted row.  All threads of the CTA must call it.
__device__ int32_t* block_merge_sort(int32_t* b0, int32_t* b1, const int32_t* __restrict__ row, int n_sel,
                                     int32_t T_kv, int n2) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int c = warp; c < n2 / 256; c += nw) {
    int32_t v[8];
    load_slots<8>(v, row, c * 256, n_sel, T_kv, lane);
    warp_sort<8>(v, lane);
#pragma unroll
    for (int r = 0; r < 8; ++r) b0[c * 256 + lane * 8 + r] = v[r];
  }
  __syncthreads();
  const int per = n2 / static_cast<int>(blockDim.x);
  int32_t* src = b0;
  int32_t* dst = b1;
  for (int len = 256; len < n2; len <<= 1) {
    const int o0 = static_cast<int>(threadIdx.x) * per;
    const int base = o0 & ~(2 * len - 1);  // the pair of runs [base, base + len), [base + len, base + 2 len)
    const int32_t* a = src + base;
    const int32_t* b = a + len;
    const int d = o0 - base;
    int lo = d > len ? d - len : 0, hi = d < len ? d : len;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (a[mid] <= b[d - mid - 1]) lo = mid + 1;
      else hi = mid;
    }
    int ia = lo, ib = d - lo;
    for (int r = 0; r < per; ++r) {
      const int32_t x = ia < len ? a[ia] : INT_MAX;
      const int32_t y = ib < len ? b[ib] : INT_MAX;
      const bool take_a = ib >= len || (ia < len && x <= y);
      dst[o0 + r] = take_a ? x : y;
      ia += take_a ? 1 : 0;
      ib += take_a ? 0 : 1;
    }
    __syncthreads();
    int32_t* tmp = src;
    src = dst;
    dst = tmp;
  }
  return src;
}

// One block per query row (rows of more than 1024 slots): filter invalid IDs,
// sort (block_merge_sort), de-duplicate, compact.
__global__ void __launch_bounds__(kRowThreads) route_rows_kernel(
    const int32_t* __restrict__ routes, int32_t T_kv, int n_sel, int n2,
    int32_t* __restrict__ row_cnt, int32_t* __restrict__ row_cols, int32_t* __restrict__ quad_cnt, int cnt_shift,
    int* __restrict__ status, const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
    float* __restrict__ delta, int H, unsigned long long* __restrict__ masks, int64_t n_tiles) {
  extern __shared__ int32_t smem_rows[];  // two buffers of n2 values, then 32 ints of scan scratch
  int* scratch = smem_rows + 2 * n2;
  const int64_t t = blockIdx.x;
  if (status != nullptr && t == 0 && threadIdx.x == 0) write_plan_tag(status, gridDim.x, T_kv, n_sel);
  const int32_t* sv = block_merge_sort(smem_rows, smem_rows + n2, routes + t * n_sel, n_sel, T_kv, n2);

  // Each thread owns a contiguous run of the sorted values.
  const int per = (n2 + blockDim.x - 1) / blockDim.x;
  const int lo = min(n2, static_cast<int>(threadIdx.x) * per), hi = min(n2, lo + per);
  int mine = 0;
  for (int i = lo; i < hi; ++i) {
    const int32_t x = sv[i];
    if (x != INT_MAX && (i == 0 || sv[i - 1] != x)) {
      ++mine;
      if (quad_cnt != nullptr && (i == 0 || (sv[i - 1] >> cnt_shift) != (x >> cnt_shift)))
        atomicAdd(quad_cnt + (x >> cnt_shift), 1);
      if (masks != nullptr && (i == 0 || (sv[i - 1] >> kTileShift) != (x >> kTileShift)))
        mark_tile(masks, n_tiles, t, x >> kTileShift);
    }
  }
  int total;
  int pos = block_exclusive_scan(mine, scratch, &total);
  int32_t* dst = row_cols + t * n_sel;
  for (int i = lo; i < hi; ++i) {
    const int32_t x = sv[i];
    if (x != INT_MAX && (i == 0 || sv[i - 1] != x)) dst[pos++] = x;
  }
  if (threadIdx.x == 0) row_cnt[t] = total;
  if (delta != nullptr) row_delta(dout, out, delta, t, H, threadIdx.x & 31, 4 * (threadIdx.x >> 5), 4 * (blockDim.x >> 5));
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

// First index in sorted entries s[0, len) whose query (high word) is >= q.
template <typename P>
__device__ int lower_bound_query(const P* s, int len, int64_t q) {
  int lo = 0, hi = len;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((s[mid] >> 32) < q) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// One block per quad: sort its list ascending (by query, the high word), then
// record where each query phase [p*C, (p+1)*C) starts in the sorted list:
// phase_ptr[b*(P+1) + p], p = 0..P (phase P ends the list).
__global__ void __launch_bounds__(kSortThreads) quad_sort_kernel(const int32_t* __restrict__ ptr,
                                                                 int64_t* __restrict__ ent, int P, int C,
                                                                 int32_t* __restrict__ phase_ptr) {
  __shared__ int64_t sv[kSortCap];
  const int64_t b = blockIdx.x;
  const int lo = ptr[b], len = ptr[b + 1] - lo;
  int32_t* pp = phase_ptr + b * (P + 1);
  int64_t* seg = ent + lo;
  if (len <= 1) {
    for (int p = threadIdx.x; p <= P; p += blockDim.x)
      pp[p] = lo + ((len == 1 && (seg[0] >> 32) < static_cast<int64_t>(p) * C) ? 1 : 0);
    return;
  }
  int n2 = 1;
  while (n2 < len) n2 <<= 1;
  if (n2 <= kSortCap) {
    for (int i = threadIdx.x; i < n2; i += blockDim.x) sv[i] = i < len ? seg[i] : LLONG_MAX;
    __syncthreads();
    block_sort<int64_t>(sv, n2, n2);
    for (int i = threadIdx.x; i < len; i += blockDim.x) seg[i] = sv[i];
    for (int p = threadIdx.x; p <= P; p += blockDim.x)
      pp[p] = lo + lower_bound_query(sv, len, static_cast<int64_t>(p) * C);
  } else {
    block_sort<int64_t>(seg, len, n2);  // in place, in global memory
    for (int p = threadIdx.x; p <= P; p += blockDim.x)
      pp[p] = lo + lower_bound_query(seg, len, static_cast<int64_t>(p) * C);
  }
}

// ---- key->query transpose at the granularity of 128-key tiles ----
// Entry of a (query row, tile) pair, the "union" of the row's keys in the tile:
// (t << 32) | (i0 << 8) | (n - 1), where row_cols[t][i0, i0 + n) are the row's
// keys inside the tile (ascending, so one contiguous run of the sorted row).

// Rows come in blocks of 64 (kBlockRows).  Per block and tile, a 64-bit mask of
// the block's rows that meet the tile (set by the route-rows kernels, which see
// each row's tiles as they sort it); a scan down each tile's column of mask
// popcounts gives every block its first slot in the tile's list; an entry's
// place inside its block is the popcount of the mask below its row.  So every
// (row, tile) entry is written straight to its place in ascending query order,
// with no sort and no atomics on the list, and a query phase (a multiple of 64
// rows) starts at a block's first slot.

// One warp per tile: exclusive scan of the blocks' mask popcounts down the
// tile's column (blk_base), and the tile's row count.
__global__ void __launch_bounds__(256) tile_scan_kernel(const unsigned long long* __restrict__ masks, int64_t n_blocks,
                                                        int64_t n_tiles, int32_t* __restrict__ blk_base,
                                                        int32_t* __restrict__ tile_cnt) {
  const int lane = threadIdx.x & 31;
  const int64_t j = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (j >= n_tiles) return;
  int carry = 0;
  for (int64_t b0 = 0; b0 < n_blocks; b0 += 32) {
    const int64_t b = b0 + lane;
    const int c = b < n_blocks ? __popcll(masks[b * n_tiles + j]) : 0;
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (b < n_blocks) blk_base[b * n_tiles + j] = carry + x - c;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) tile_cnt[j] = carry;
}

// Writes the entry (t << 32) | (i0 << 8) | (n - 1) of row t's run in tile tl.
__device__ __forceinline__ void tile_put(int64_t t, int32_t tl, int i0, int n, int64_t n_tiles,
                                         const unsigned long long* __restrict__ masks,
                                         const int32_t* __restrict__ blk_base, const int32_t* __restrict__ ptr,
                                         int64_t* __restrict__ ent) {
  const int64_t cell = (t >> 6) * n_tiles + tl;
  const unsigned long long below = masks[cell] & ((1ull << (t & 63)) - 1ull);
  const int64_t p = static_cast<int64_t>(ptr[tl]) + blk_base[cell] + __popcll(below);
  ent[p] = (t << 32) | (static_cast<int64_t>(i0) << 8) | static_cast<int64_t>(n - 1);
}

// One entry per (row, tile) run, (t << 32) | (i0 << 8) | (n - 1), at
// ptr[tile] + blk_base[block, tile] + (rows of the block below t that meet the tile).
// A run ends where the next one starts: within a 32-key window the next start
// above a lane comes from the window's ballot of starts; the last run of a
// window stays pending until the first start of a later window (or the row's end).
// Rows are independent here (every slot comes from the masks, the block bases
// and the tile pointers), so each warp takes one row (against a CTA per 64-row
// block: seq32k tile lists 0.13 -> 0.10 ms, cp128k 0.20 -> 0.11 ms).
__global__ void __launch_bounds__(256) tile_fill_kernel(const int32_t* __restrict__ row_cnt,
                                                        const int32_t* __restrict__ row_cols, int64_t T, int n_sel,
                                                        int64_t n_tiles, const unsigned long long* __restrict__ masks,
                                                        const int32_t* __restrict__ blk_base,
                                                        const int32_t* __restrict__ ptr, int64_t* __restrict__ ent,
                                                        const int* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T || (status != nullptr && *status == kStatusBadPlan)) return;
  const int cnt = row_cnt[t];
  const int32_t* cols = row_cols + t * n_sel;
  int32_t carry = -1;             // tile of the last key of the previous window (none: -1)
  int pend_i = -1;                // start of the run still open at the end of the previous windows
  int32_t pend_tl = 0;
  for (int base = 0; base < cnt; base += 32) {
    const int i = base + lane;
    const int32_t tl = i < cnt ? (cols[i] >> kTileShift) : INT_MAX;
    int32_t prev = __shfl_up_sync(0xffffffffu, tl, 1);
    if (lane == 0) prev = carry;
    carry = __shfl_sync(0xffffffffu, tl, 31);
    const bool start = i < cnt && tl != prev;
    const uint32_t m = __ballot_sync(0xffffffffu, start);
    if (m == 0) continue;
    const int first = __ffs(m) - 1, last = 31 - __clz(m);
    if (pend_i >= 0 && lane == 0) tile_put(t, pend_tl, pend_i, base + first - pend_i, n_tiles, masks, blk_base, ptr, ent);
    const uint32_t above = lane == 31 ? 0u : (m >> (lane + 1)) << (lane + 1);
    if (start && above != 0) tile_put(t, tl, i, base + __ffs(above) - 1 - i, n_tiles, masks, blk_base, ptr, ent);
    pend_i = base + last;
    pend_tl = __shfl_sync(0xffffffffu, tl, last);
  }
  if (pend_i >= 0 && lane == 0) tile_put(t, pend_tl, pend_i, cnt - pend_i, n_tiles, masks, blk_base, ptr, ent);
}

// Union lists of groups of `group` adjacent query rows (the paired-query gather
// of the "Query Sparse Attention (QSA)" page, "Selection and components":
// adjacent queries gather the union of their selected keys once, owner bits
// keeping each query's own set).  One CTA per group.  The rows are sorted
// already, so their merge needs no sort: key x at position k of row q goes to
// k + (keys of the rows below q that are <= x) + (keys of the rows above q
// that are < x) (binary searches in shared memory), a stable merge in which
// equal keys end up adjacent in row order.  Every distinct key is then placed
// by a CTA scan over "first of its key" flags, with the OR of its owners.
// Group gi's list is ukey / uown [gi * group * n_sel, ...), its length ucnt[gi].
__device__ __forceinline__ int count_below(const int32_t* a, int n, int32_t x, bool or_equal) {
  int lo = 0, hi = n;  // the number of a[0 .. n) that are < x (or <= x)
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x || (or_equal && a[mid] == x)) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kRowThreads) union_lists_kernel(
    const int32_t* __restrict__ row_cnt, const int32_t* __restrict__ row_cols, int64_t T, int n_sel, int group,
    int32_t* __restrict__ ucnt, int32_t* __restrict__ ukey, uint8_t* __restrict__ uown) {
  extern __shared__ int32_t us[];  // the rows' keys [total], then the merged (key, row) pairs [total] as int64
  __shared__ int scratch[32];
  __shared__ int off[kMaxUnionGroup + 1];
  const int64_t gi = blockIdx.x, t0 = gi * group;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int q = 0; q < group; ++q) {
      off[q] = acc;
      acc += t0 + q < T ? row_cnt[t0 + q] : 0;
    }
    off[group] = acc;
  }
  __syncthreads();
  const int total = off[group];
  int64_t* mv = reinterpret_cast<int64_t*>(us + ((total + 1) & ~1));
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    int q = 0;
    while (i >= off[q + 1]) ++q;
    us[i] = row_cols[(t0 + q) * n_sel + (i - off[q])];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    int q = 0;
    while (i >= off[q + 1]) ++q;
    const int32_t x = us[i];
    int pos = i - off[q];
    for (int q2 = 0; q2 < group; ++q2)
      if (q2 != q) pos += count_below(us + off[q2], off[q2 + 1] - off[q2], x, q2 < q);
    mv[pos] = (static_cast<int64_t>(x) << 8) | q;
  }
  __syncthreads();
  const int per = (total + blockDim.x - 1) / blockDim.x;
  const int lo = min(total, static_cast<int>(threadIdx.x) * per), hi = min(total, lo + per);
  int mine = 0;
  for (int i = lo; i < hi; ++i)
    if (i == 0 || (mv[i] >> 8) != (mv[i - 1] >> 8)) ++mine;
  int cnt;
  int pos = block_exclusive_scan(mine, scratch, &cnt);
  const int64_t cap = static_cast<int64_t>(group) * n_sel;
  int32_t* kd = ukey + gi * cap;
  uint8_t* od = uown + gi * cap;
  for (int i = lo; i < hi; ++i) {
    if (i > 0 && (mv[i] >> 8) == (mv[i - 1] >> 8)) continue;
    const int64_t key = mv[i] >> 8;
    uint32_t own = 0;
    for (int k = i; k < total && (mv[k] >> 8) == key; ++k) own |= 1u << (mv[k] & 0xff);
    kd[pos] = static_cast<int32_t>(key);
    od[pos] = static_cast<uint8_t>(own);
    ++pos;
  }
  if (threadIdx.x == 0) ucnt[gi] = cnt;
}

// One warp per tile: lane 0 appends the tile's non-empty phase ranges to the
// per-phase work lists, wl[p][*] = (tile, first entry, end entry, flags), flags
// bit 0: no entries of the tile before this range, bit 1: none after it, bits
// 2..: the number of earlier non-empty phases of the tile (the range's place in
// the tile's accumulation order).  A tile that no query routes to gets its
// dK/dV rows zeroed by the warp.
__global__ void __launch_bounds__(256) tile_worklist_kernel(
    const int32_t* __restrict__ ptr, const int32_t* __restrict__ blk_base, int64_t n_blocks, int64_t n_tiles,
    int64_t T_kv, int G, int P, int C, int32_t* __restrict__ wl_cnt, int4* __restrict__ wl, uint8_t* __restrict__ dk,
    uint8_t* __restrict__ dv, int out_bytes) {
  const int lane = threadIdx.x & 31;
  const int64_t b = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (b >= n_tiles) return;
  const int q0 = ptr[b], q1 = ptr[b + 1];
  if (q0 == q1) {
    const int64_t k0 = b << kTileShift, k1 = min(T_kv, (b + 1) << kTileShift);
    const int64_t row = static_cast<int64_t>(G) * kHeadDim * out_bytes;  // bytes per key, a multiple of 16
    uint4* rk = reinterpret_cast<uint4*>(dk + k0 * row);
    uint4* rv = reinterpret_cast<uint4*>(dv + k0 * row);
    for (int64_t i = lane; i < (k1 - k0) * row / 16; i += 32) rk[i] = rv[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  if (lane != 0) return;
  // phase p (rows p C .. (p + 1) C - 1, C a multiple of 64) starts at the first
  // slot of block p C / 64 in the tile's list
  auto start = [&](int p) {
    const int64_t blk = static_cast<int64_t>(p) * C / kBlockRows;
    return q0 + (blk < n_blocks ? blk_base[blk * n_tiles + b] : q1 - q0);
  };
  int ord = 0;
  for (int p = 0; p < P; ++p) {
    const int lo = start(p), hi = start(p + 1);
    if (hi > lo) {
      const int slot = atomicAdd(wl_cnt + p, 1);
      wl[static_cast<int64_t>(p) * n_tiles + slot] =
          make_int4(static_cast<int>(b), lo, hi, (lo == q0 ? 1 : 0) | (hi == q1 ? 2 : 0) | (ord << 2));
      ++ord;
    }
  }
}

}  // namespace

static int next_pow2(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

cudaError_t launch_route_rows(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel, int32_t* row_cnt,
                              int32_t* row_cols, int32_t* bucket_cnt, int cnt_shift, int* status, const void* dout,
                              const void* out, float* delta, int H, unsigned long long* tile_masks, cudaStream_t s) {
  const auto* dq = static_cast<const __nv_bfloat16*>(dout);
  const auto* o = static_cast<const __nv_bfloat16*>(out);
  const unsigned wblocks = static_cast<unsigned>((T + kRowWarps - 1) / kRowWarps);
  const int32_t tkv = static_cast<int32_t>(T_kv);
  const int64_t n_tiles = (T_kv + 127) >> kTileShift;
#define QSA_ROWS_WARP(NPL)                                                                                         \
  route_rows_warp_kernel<NPL><<<wblocks, kRowWarps * 32, 0, s>>>(routes, T, tkv, n_sel, row_cnt, row_cols,        \
                                                                 bucket_cnt, cnt_shift, status, dq, o, delta, H, \
                                                                 tile_masks, n_tiles);                            \
  return cudaGetLastError()
  if (n_sel <= 64) { QSA_ROWS_WARP(2); }
  if (n_sel <= 128) { QSA_ROWS_WARP(4); }
  if (n_sel <= 256) { QSA_ROWS_WARP(8); }
  if (n_sel <= 512) { QSA_ROWS_WARP(16); }
#undef QSA_ROWS_WARP
#define QSA_ROWS_SPLIT(NB)                                                                                        \
  route_rows_split_kernel<NB><<<wblocks, kRowWarps * 32, 0, s>>>(routes, T, tkv, n_sel, row_cnt, row_cols,         \
                                                                 bucket_cnt, cnt_shift, status, dq, o, delta, H, \
                                                                 tile_masks, n_tiles);                            \
  return cudaGetLastError()
  if (n_sel <= kSplitA + 32) { QSA_ROWS_SPLIT(1); }
  if (n_sel <= kSplitA + 64) { QSA_ROWS_SPLIT(2); }
  if (n_sel <= kSplitA + 128) { QSA_ROWS_SPLIT(4); }
  if (n_sel <= kSplitA + 256) { QSA_ROWS_SPLIT(8); }
#undef QSA_ROWS_SPLIT
#define QSA_ROWS_WARP(NPL)                                                                                         \
  route_rows_warp_kernel<NPL><<<wblocks, kRowWarps * 32, 0, s>>>(routes, T, tkv, n_sel, row_cnt, row_cols,        \
                                                                 bucket_cnt, cnt_shift, status, dq, o, delta, H, \
                                                                 tile_masks, n_tiles);                            \
  return cudaGetLastError()
  if (n_sel <= 1024) { QSA_ROWS_WARP(32); }
#undef QSA_ROWS_WARP
  const int n2 = next_pow2(n_sel);
  const size_t smem = static_cast<size_t>(2 * n2 + 32) * sizeof(int32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  route_rows_kernel<<<static_cast<unsigned>(T), kRowThreads, smem, s>>>(
      routes, tkv, n_sel, n2, row_cnt, row_cols, bucket_cnt, cnt_shift, status, dq, o, delta, H, tile_masks, n_tiles);
  return cudaGetLastError();
}

cudaError_t launch_row_delta_masks(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int64_t T_kv,
                                   int n_sel, const int* plan_tag, int* status, const void* dout, const void* out,
                                   float* delta, int H, unsigned long long* tile_masks, cudaStream_t s) {
  row_delta_masks_kernel<<<static_cast<unsigned>((T + 7) / 8), 256, 0, s>>>(
      row_cnt, row_cols, T, static_cast<int32_t>(T_kv), n_sel, plan_tag, status,
      static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out), delta, H, tile_masks,
      (T_kv + 127) >> kTileShift);
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

cudaError_t launch_quad_sort(const int32_t* quad_ptr, int64_t n_quads, int64_t* quad_ent, int P, int C,
                             int32_t* phase_ptr, cudaStream_t s) {
  quad_sort_kernel<<<static_cast<unsigned>(n_quads), kSortThreads, 0, s>>>(quad_ptr, quad_ent, P, C, phase_ptr);
  return cudaGetLastError();
}

int union_group(int n_sel) { return n_sel <= kUnionSortCap / kUnionGroup ? kUnionGroup : 1; }

cudaError_t launch_union_lists(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int n_sel, int group,
                               int32_t* ucnt, int32_t* ukey, uint8_t* uown, cudaStream_t s) {
  if (group < 1 || group > kMaxUnionGroup || static_cast<int64_t>(group) * n_sel > kUnionSortCap)
    return cudaErrorInvalidValue;
  const int cap = group * n_sel;
  const size_t smem = static_cast<size_t>((cap + 1) & ~1) * 4 + static_cast<size_t>(cap) * 8;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(union_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const int64_t n_groups = (T + group - 1) / group;
  union_lists_kernel<<<static_cast<unsigned>(n_groups), kRowThreads, smem, s>>>(row_cnt, row_cols, T, n_sel, group,
                                                                               ucnt, ukey, uown);
  return cudaGetLastError();
}

size_t tile_masks_bytes(int64_t T, int64_t T_kv) {
  const size_t nb = static_cast<size_t>((T + kBlockRows - 1) / kBlockRows);
  const size_t nt = static_cast<size_t>((T_kv + 127) / 128);
  return nb * nt * 8;
}

size_t tile_lists_bytes(int64_t T, int64_t T_kv) {
  return tile_masks_bytes(T, T_kv) / 8 * 12;  // a mask (8 bytes) and a block base (4 bytes) per (block, tile)
}

cudaError_t launch_tile_lists(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int n_sel,
                              int64_t n_tiles, void* scratch, int32_t* tile_cnt, int32_t* tile_ptr,
                              int32_t* tile_fill, int64_t* tile_ent, const int* status, cudaStream_t s) {
  const int64_t nb = (T + kBlockRows - 1) / kBlockRows;
  const auto* masks = static_cast<const unsigned long long*>(scratch);
  auto* blk_base = reinterpret_cast<int32_t*>(static_cast<unsigned long long*>(scratch) + nb * n_tiles);
  tile_scan_kernel<<<static_cast<unsigned>((n_tiles * 32 + 255) / 256), 256, 0, s>>>(masks, nb, n_tiles, blk_base,
                                                                                    tile_cnt);
  cudaError_t e = launch_quad_scan(tile_cnt, n_tiles, tile_ptr, tile_fill, s);
  if (e != cudaSuccess) return e;
  tile_fill_kernel<<<static_cast<unsigned>((T + 7) / 8), 256, 0, s>>>(row_cnt, row_cols, T, n_sel, n_tiles, masks,
                                                                     blk_base, tile_ptr, tile_ent, status);
  return cudaGetLastError();
}

cudaError_t launch_tile_worklist(const int32_t* tile_ptr, const void* scratch, int64_t T, int64_t n_tiles,
                                 int64_t T_kv, int G, int P, int C, int32_t* wl_cnt, int4* wl, void* dk, void* dv,
                                 bool f32_out, cudaStream_t s) {
  if (C % kBlockRows != 0) return cudaErrorInvalidValue;
  const int64_t nb = (T + kBlockRows - 1) / kBlockRows;
  const auto* blk_base =
      reinterpret_cast<const int32_t*>(static_cast<const unsigned long long*>(scratch) + nb * n_tiles);
  tile_worklist_kernel<<<static_cast<unsigned>((n_tiles * 32 + 255) / 256), 256, 0, s>>>(
      tile_ptr, blk_base, nb, n_tiles, T_kv, G, P, C, wl_cnt, wl, static_cast<uint8_t*>(dk), static_cast<uint8_t*>(dv),
      f32_out ? 4 : 2);
  return cudaGetLastError();
}

}  // namespace qsa
