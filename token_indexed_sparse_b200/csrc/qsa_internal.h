// Host-side launchers of the QSA kernels, shared by the C ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qsa {

// Route preprocessing (qsa_routes.cu).
// Per-row ascending, de-duplicated valid route IDs; optionally counts, per key
// quad, the rows that meet it (quad_cnt must be zeroed by the caller).
cudaError_t launch_route_rows(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel,
                              int32_t* row_cnt, int32_t* row_cols, int32_t* quad_cnt,
                              cudaStream_t s);
// quad_cnt -> quad_ptr (exclusive scan, n_quads+1 entries) and quad_fill (copy
// of quad_ptr used as fill cursors).
cudaError_t launch_quad_scan(const int32_t* quad_cnt, int64_t n_quads, int32_t* quad_ptr,
                             int32_t* quad_fill, cudaStream_t s);
// Fill the key-quad lists (unordered), then sort each list by query.
cudaError_t launch_quad_fill(const int32_t* row_cnt, const int32_t* row_cols, int64_t T, int n_sel,
                             int32_t* quad_fill, int64_t* quad_ent, cudaStream_t s);
cudaError_t launch_quad_sort(const int32_t* quad_ptr, int64_t n_quads, int64_t* quad_ent,
                             cudaStream_t s);

// Attention kernels (qsa_forward.cu, qsa_backward.cu).
cudaError_t launch_forward(const void* q, const void* k, const void* v, const int32_t* row_cnt,
                           const int32_t* row_cols, int64_t T, int G, int n_sel, float scale,
                           void* out, float* lse, cudaStream_t s);
// dQ per query; also writes delta [T, H] and the BF16 probabilities / score
// gradients of every routed pair, pds [T, G, n_sel, 24].
cudaError_t launch_backward_dq(const void* grad_out, const void* q, const void* k, const void* v,
                               const void* out, const float* lse, const int32_t* row_cnt,
                               const int32_t* row_cols, int64_t T, int G, int n_sel, float scale,
                               void* dq, float* delta, uint16_t* pds, cudaStream_t s);
// dK/dV per key quad over the sorted key-quad lists.
cudaError_t launch_backward_dkdv(const void* grad_out, const void* q, const uint16_t* pds,
                                 const int32_t* quad_ptr, const int64_t* quad_ent, int64_t T,
                                 int64_t T_kv, int G, int n_sel, float scale, void* dk, void* dv,
                                 cudaStream_t s);

}  // namespace qsa
