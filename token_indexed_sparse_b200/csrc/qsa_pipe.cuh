// Chunked K/V gather pipeline shared by the forward and dQ kernels.
//
// Both kernels are persistent.  Work items are (query t, KV group g) pairs, item
// `it` = t * G + g, dealt round-robin: CTA b takes items b, b + gridDim.x, ...
// Item t's de-duplicated keys R_t are cut into chunks of KEYS = 8 x (warps per
// CTA) keys (an empty row still has one chunk, with 0 keys).  Every thread of
// the CTA walks the same chunk sequence with a Cursor; the gather of a chunk is
// issued while earlier chunks are computed.
//
// Each chunk's K and V rows land in an XOR-swizzled [KEYS][256] BF16 tile through
// 16-byte cp.async copies; warp w copies rows 8w .. 8w + 7, one whole 512-byte
// row per instruction, with the rows' key IDs loaded one chunk ahead.  Rows past
// the end of R_t are zero-filled by the copies themselves.
#pragma once

#include "qsa_device.cuh"

namespace qsa {

template <int KEYS>
__device__ __forceinline__ int pipe_chunks(int cnt) { return cnt > 0 ? (cnt + KEYS - 1) / KEYS : 1; }

// The item index is tracked as (t, g) and advanced by the grid stride without
// any division in the loop: the stride's quotient and remainder by G are taken
// once, at initialisation.
struct Cursor {
  int64_t it;    // current item; >= n_items once the CTA's sequence is exhausted
  int64_t t;     // its query token, it / G
  int g;         // its KV group, it % G
  int dt, dg;    // gridDim.x / G and gridDim.x % G
  int ch;        // chunk index within the item
  int nch;       // chunks of the item
  int cnt;       // |R_t| of the item
  int cnt_next;  // |R_t| of the CTA's next item (prefetched)
};

// |R_t| of the item one grid stride after (t, g), or 0 past the end.
__device__ __forceinline__ int pipe_cnt_next(const Cursor& c, const int32_t* row_cnt, int64_t n_items, int G) {
  const int64_t t_next = c.t + c.dt + (c.g + c.dg >= G ? 1 : 0);
  return c.it + gridDim.x < n_items ? __ldg(row_cnt + t_next) : 0;
}

template <int KEYS>
__device__ __forceinline__ void cursor_init(Cursor& c, const int32_t* row_cnt, int64_t n_items, int G) {
  c.it = blockIdx.x;
  c.t = static_cast<int>(blockIdx.x) / G;
  c.g = static_cast<int>(blockIdx.x) % G;
  c.dt = static_cast<int>(gridDim.x) / G;
  c.dg = static_cast<int>(gridDim.x) % G;
  c.ch = 0;
  c.cnt = c.it < n_items ? __ldg(row_cnt + c.t) : 0;
  c.cnt_next = pipe_cnt_next(c, row_cnt, n_items, G);
  c.nch = pipe_chunks<KEYS>(c.cnt);
}

template <int KEYS>
__device__ __forceinline__ void cursor_next(Cursor& c, const int32_t* row_cnt, int64_t n_items, int G) {
  if (++c.ch == c.nch) {
    c.it += gridDim.x;
    c.t += c.dt;
    c.g += c.dg;
    if (c.g >= G) {
      c.g -= G;
      ++c.t;
    }
    c.ch = 0;
    c.cnt = c.cnt_next;
    c.nch = pipe_chunks<KEYS>(c.cnt);
    c.cnt_next = pipe_cnt_next(c, row_cnt, n_items, G);
  }
}

// Keys in the cursor's current chunk (0 for an empty row or past the end).
template <int KEYS>
__device__ __forceinline__ int cursor_nk(const Cursor& c, int64_t n_items) {
  if (c.it >= n_items || c.cnt <= 0) return 0;
  return min(KEYS, c.cnt - c.ch * KEYS);
}

// Key IDs of the rows this thread gathers in the cursor's current chunk: rows
// 8 * warp + j, j = 0..7 (0 for rows past the end of the chunk, whose copies are
// then zero-fills).  Every lane of a warp loads the same eight IDs.
template <int KEYS>
__device__ __forceinline__ void cursor_keys(int32_t (&key)[8], const Cursor& c, int64_t n_items, int G,
                                            const int32_t* row_cols, int n_sel) {
  const int nk = cursor_nk<KEYS>(c, n_items);
  const int r0 = 8 * (threadIdx.x >> 5);
  const int32_t* src = row_cols + c.t * n_sel + c.ch * KEYS + r0;
#pragma unroll
  for (int j = 0; j < 8; ++j) key[j] = (r0 + j < nk) ? __ldg(src + j) : 0;
}

// Gathers rows 8 * warp + j (j = 0..7) of K and of V into swizzled tiles at kt / vt
// (shared addresses): lane l copies 16-byte column l, so one warp instruction
// moves one whole contiguous 512-byte row, and each warp walks a run of eight
// consecutive (ascending) keys: four-token route blocks are contiguous in K/V,
// and contiguous runs gather markedly faster than scattered rows.
__device__ __forceinline__ void gather_rows(uint32_t kt, uint32_t vt, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                            const int32_t (&key)[8], int g, int G, int nk) {
  const int r0 = 8 * (threadIdx.x >> 5), l = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int r = r0 + j;
    const int64_t off = (static_cast<int64_t>(key[j]) * G + g) * kHeadDim + l * 8;
    cp_async16(kt + swz512(r, l), k + off, r < nk);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int r = r0 + j;
    const int64_t off = (static_cast<int64_t>(key[j]) * G + g) * kHeadDim + l * 8;
    cp_async16(vt + swz512(r, l), v + off, r < nk);
  }
}

// Gathers the 12 rows of a query group ([12][256] BF16, contiguous at `src`) into
// a swizzled tile: with NW warps, warp w copies rows w, w + NW, ..., one 512-byte
// row per instruction.
template <int NW = 8>
__device__ __forceinline__ void gather_heads(uint32_t dst, const __nv_bfloat16* src) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < kHeadsPerGroup; r += NW)
    if (r + w < kHeadsPerGroup) cp_async16(dst + swz512(r + w, l), src + (r + w) * kHeadDim + l * 8, true);
}

}  // namespace qsa
