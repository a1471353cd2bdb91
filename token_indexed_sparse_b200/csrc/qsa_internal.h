// Host-side launchers of the QSA kernels, shared by the C ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qsa {

// Route preprocessing (qsa_routes.cu).
// Per-row ascending, de-duplicated valid route IDs; optionally counts, per
// bucket of 2^cnt_shift consecutive keys (2: quads), the rows that meet it
// (bucket_cnt must be zeroed by the caller).
// `status` (nullable) is zeroed by this kernel, the first of every call.  With
// `delta` non-null it also writes delta[t, h] = sum_d dO[t,h,d] * out[t,h,d]
// (FP32 from the BF16 tensors, [T, H]).  With `tile_masks` non-null (the first
// tile_masks_bytes of a tile-lists scratch, zeroed by the caller) it sets row
// t's bit in the mask of (t / 64, tile) for every 128-key tile the row meets,
// the input of launch_tile_lists.
cudaError_t launch_route_rows(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel,
                              int32_t* row_cnt, int32_t* row_cols, int32_t* bucket_cnt, int cnt_shift,
                              int* status, const void* dout, const void* out, float* delta, int H,
                              unsigned long long* tile_masks, cudaStream_t s);
// The backward's route work from row lists sorted already (a forward's, same
// routes): delta and the tile masks as launch_route_rows would set them.
// plan_tag: the status slot of the call that wrote the lists; `status` is set
// to kStatusBadPlan unless it carries the route-list tag of rows of these sizes.
constexpr int kStatusBadPlan = 2;
cudaError_t launch_row_delta_masks(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int64_t T_kv,
                                   int n_sel, const int* plan_tag, int* status, const void* dout, const void* out,
                                   float* delta, int H, unsigned long long* tile_masks, cudaStream_t s);
// quad_cnt -> quad_ptr (exclusive scan, n_quads+1 entries) and quad_fill (copy
// of quad_ptr used as fill cursors).
cudaError_t launch_quad_scan(const int32_t* quad_cnt, int64_t n_quads, int32_t* quad_ptr,
                             int32_t* quad_fill, cudaStream_t s);
// Fill the key-quad lists (unordered), then sort each list by query.
cudaError_t launch_quad_fill(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int n_sel,
                             int32_t* quad_fill, int64_t* quad_ent, cudaStream_t s);
// Sorts each quad's list by query and records where each query phase
// [p*C, (p+1)*C) starts in it: phase_ptr[b*(P+1) + p].
cudaError_t launch_quad_sort(const int32_t* quad_ptr, int64_t n_quads, int64_t* quad_ent, int P, int C,
                             int32_t* phase_ptr, cudaStream_t s);
// The key->query transpose over 128-key tiles: one entry per (row, tile) pair,
// (t << 32) | (i0 << 8) | (n - 1) with row_cols[t][i0, i0 + n) the row's keys in
// the tile, every list in ascending query order without a sort: per block of 64
// rows a mask of the rows meeting each tile (set by launch_route_rows), block
// bases from a scan down each tile's column, ranks from mask popcounts.
// `scratch` holds the masks (its first tile_masks_bytes) and the block bases
// (tile_lists_bytes in all); tile_cnt, tile_ptr (n_tiles + 1) and tile_fill
// (n_tiles) are written.
size_t tile_masks_bytes(int64_t T, int64_t T_kv);
size_t tile_lists_bytes(int64_t T, int64_t T_kv);
cudaError_t launch_tile_lists(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int n_sel,
                              int64_t n_tiles, void* scratch, int32_t* tile_cnt, int32_t* tile_ptr,
                              int32_t* tile_fill, int64_t* tile_ent, const int* status, cudaStream_t s);
// Per-phase work lists of non-empty (tile, entry range) items (wl_cnt zeroed by
// the caller), phase p = rows [p C, (p + 1) C) with C a multiple of 64, its
// start in a tile's list read from the block bases in `scratch` (written by
// launch_tile_lists); zeroes dK/dV of tiles that no query routes to.
cudaError_t launch_tile_worklist(const int32_t* tile_ptr, const void* scratch, int64_t T, int64_t n_tiles,
                                 int64_t T_kv, int G, int P, int C, int32_t* wl_cnt, int4* wl, void* dk, void* dv,
                                 bool f32_out, cudaStream_t s);

// Union lists of groups of `group` adjacent query rows (qsa_routes.cu): per
// group gi, the ascending union of the rows' route sets in ukey[gi * group *
// n_sel, + ucnt[gi]) and per key a mask of the rows that selected it (uown).
// group * n_sel <= kUnionSortCap; union_group(n_sel) is the group size the
// forward uses (kUnionGroup rows, or 1 for rows too long to merge in shared memory).
constexpr int kUnionGroup = 4;
constexpr int kUnionSortCap = 16384;
int union_group(int n_sel);
cudaError_t launch_union_lists(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int n_sel, int group,
                               int32_t* ucnt, int32_t* ukey, uint8_t* uown, cudaStream_t s);

// Attention kernels (qsa_forward.cu, qsa_backward.cu, qsa_dkdv_union.cu).
cudaError_t launch_forward(const void* q, const void* k, const void* v, const int32_t* row_cnt,
                           const int32_t* row_cols, int64_t T, int G, int n_sel, float scale,
                           void* out, float* lse, int* status, cudaStream_t s);
// dQ per query; also writes the BF16 probabilities / score gradients of every
// routed pair, pds [T, G, n_sel, 24] ([P h0..h11 | dS h0..h11] per pair).
cudaError_t launch_backward_dq(const void* grad_out, const void* q, const void* k, const void* v,
                               const float* lse, const float* delta, const int32_t* row_cnt,
                               const int32_t* row_cols, int64_t T, int G, int n_sel, float scale,
                               void* dq, uint16_t* pds, const int* status, cudaStream_t s);
// SM count of the current device (cached).
int sm_count();
// Query phases of the dK/dV pass for T queries of H heads: P phases of C
// queries each (C a multiple of 256).
void dkdv_phases(int64_t T, int H, int* P, int* C);
// dK/dV over 128-key tiles on the tensor cores, all P query phases in one
// launch: units (tile, group, tensor) of the per-phase work lists claimed from
// *claim_ctr in phase order; the FP32 partial of a (tile, group, tensor) passes
// from phase to phase through `partial`, ordered by its counter in `done`
// (n_tiles * 2G ints; claim_ctr and done zeroed by the caller); final dK/dV BF16,
// or FP32 when f32_out.  Sets *status = 3 if a bounded wait expired.  P <= 64.
cudaError_t launch_backward_dkdv_union(const void* grad_out, const void* q, const uint16_t* pds,
                                       const int32_t* row_cols, const int64_t* tile_ent, const int32_t* wl_cnt,
                                       const int4* wl, int* claim_ctr, int* done, int P, int64_t n_tiles,
                                       int64_t T_kv, int G, int n_sel, float scale, float* partial, void* dk, void* dv,
                                       bool f32_out, int* status, cudaStream_t s);

// FP32 -> BF16 (round to nearest even) of n contiguous values (qsa_cast.cu);
// x and y 16-byte aligned.
cudaError_t launch_cast_f32_bf16(const float* x, void* y, int64_t n, cudaStream_t s);

// Bitmap selection -> route IDs (qsa_bitmap.cu); zeroes *max_cnt first when given.
cudaError_t launch_bitmap_routes(const uint8_t* sel, const int32_t* lo, const int32_t* hi, const int32_t* blk_base,
                                 const int32_t* tok_base, int64_t T, int64_t NB, int64_t T_kv, int block_size,
                                 int n_sel, int32_t* routes, int32_t* row_cnt, int32_t* max_cnt, cudaStream_t s);

// Selector (qsa_selector.cu): scores of the candidate blocks, then top-k and route expansion.
cudaError_t launch_selector_scores(const void* qi, const void* kbar, int64_t T, int64_t NB, int Hi, float scale,
                                   const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base,
                                   float* scores, int64_t stride, int* status, cudaStream_t s);
cudaError_t launch_selector_topk(const float* scores, int64_t stride, int64_t T, int64_t NB, int k,
                                 const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base,
                                 int32_t* blocks, int32_t* routes, cudaStream_t s);

}  // namespace qsa
