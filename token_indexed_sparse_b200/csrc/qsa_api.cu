// C ABI of the QSA library: host-side argument checks, workspace layout and the
// launch sequences of the forward, backward and route-plan calls.  Nothing here
// reads device memory or synchronises; every launch goes to the caller's stream.
#include <climits>
#include <cmath>
#include <cstdint>

#include "qsa.h"
#include "qsa_device.cuh"
#include "qsa_internal.h"

namespace {

constexpr int kMaxSel = 16384;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

qsa_status_t check_sizes(int64_t T, int64_t T_kv, int H, int G, int n_sel) {
  if (T < 1 || T_kv < 1 || n_sel < 1 || n_sel > kMaxSel || G < 1 || H < 1) return QSA_ERR_INVALID_ARGUMENT;
  if (T_kv > INT32_MAX || T > INT32_MAX / n_sel || T > (int64_t{1} << 30)) return QSA_ERR_INVALID_ARGUMENT;
  if (H % G != 0 || H / G != qsa::kHeadsPerGroup) return QSA_ERR_UNSUPPORTED;
  if (T > INT32_MAX / G || (T_kv + 3) / 4 > INT32_MAX / G) return QSA_ERR_INVALID_ARGUMENT;
  return QSA_OK;
}


struct Layout {
  size_t status = 0, row_cnt = 0, row_cols = 0, tile_ctr = 0, tile_ptr = 0, tile_fill = 0, tile_ent = 0, delta = 0,
         pds = 0, lists = 0, wl = 0, partial = 0, total = 0;
  int P = 1, C = 1;
};

// Counters zeroed by one memset at the start of a backward call: per-tile row
// counts [n_tiles], per-phase work-list sizes [P], the dK/dV unit claim counter
// [1], and per (tile, group, tensor) the number of phases accumulated [n_tiles * 2G].
size_t tile_ctr_ints(int64_t n_tiles, int P, int G) {
  return static_cast<size_t>(n_tiles) * (1 + 2 * static_cast<size_t>(G)) + static_cast<size_t>(P) + 1;
}

Layout make_layout(int64_t T, int64_t T_kv, int H, int G, int n_sel, bool backward) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const size_t nt = static_cast<size_t>((T_kv + 127) / 128);  // 128-key tiles
  const size_t pairs = static_cast<size_t>(T) * static_cast<size_t>(n_sel);
  L.status = take(4);
  L.row_cnt = take(static_cast<size_t>(T) * 4);
  L.row_cols = take(pairs * 4);
  if (backward) {
    qsa::dkdv_phases(T, H, &L.P, &L.C);
    L.tile_ctr = take(tile_ctr_ints(static_cast<int64_t>(nt), L.P, G) * 4);
    L.lists = take(qsa::tile_lists_bytes(T, T_kv));  // tile masks first (zeroed with the counters), block bases
    L.tile_ptr = take((nt + 1) * 4);
    L.tile_fill = take(nt * 4);
    L.tile_ent = take(pairs * 8);  // at most one entry per routed pair
    L.delta = take(static_cast<size_t>(T) * H * 4);
    L.pds = take(pairs * G * 48);  // BF16 [P | dS] of every routed pair, 12 heads each
    L.wl = take(static_cast<size_t>(L.P) * nt * 16);
    L.partial = take(nt * G * 2 * 128 * 256 * 4);  // FP32 dK and dV of every (tile, group)
  }
  L.total = off;
  return L;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

#define QSA_TRY(expr)                         \
  do {                                        \
    cudaError_t e_ = (expr);                  \
    if (e_ != cudaSuccess) return QSA_ERR_CUDA; \
  } while (0)

// Records stage event i (if supplied) on the stream.
struct StageEvents {
  const qsa_event_t* ev;
  int n;
  cudaStream_t s;
  cudaError_t mark(int i) const {
    if (ev == nullptr || i >= n || ev[i] == nullptr) return cudaSuccess;
    return cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[i]), s);
  }
};

}  // namespace

// The forward sequence.
static qsa_status_t forward_impl(const void* q, const void* k, const void* v, const int32_t* routes, int64_t T,
                                 int64_t T_kv, int H, int G, int n_sel, float scale, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                                 const qsa_event_t* stage_events, int n_stage_events, qsa_event_t kv_ready) {
  if (!q || !k || !v || !routes || !out || !lse || !workspace) return QSA_ERR_INVALID_ARGUMENT;
  const qsa_status_t st = check_sizes(T, T_kv, H, G, n_sel);
  if (st != QSA_OK) return st;
  if (!(scale > 0.f) || !std::isfinite(scale)) return QSA_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(routes, 4) ||
      !aligned(lse, 4) || !aligned(workspace, 256))
    return QSA_ERR_MISALIGNED;
  const Layout L = make_layout(T, T_kv, H, G, n_sel, false);
  if (workspace_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, L.status);
  int32_t* row_cnt = at<int32_t>(workspace, L.row_cnt);
  int32_t* row_cols = at<int32_t>(workspace, L.row_cols);
  const StageEvents ev{stage_events, n_stage_events, s};
  QSA_TRY(qsa::launch_route_rows(routes, T, T_kv, n_sel, row_cnt, row_cols, nullptr, 2, status, nullptr, nullptr,
                                 nullptr, H, nullptr, s));
  QSA_TRY(ev.mark(0));
  // k and v are read from here on; the route work above ran without them
  if (kv_ready != nullptr) QSA_TRY(cudaStreamWaitEvent(s, reinterpret_cast<cudaEvent_t>(kv_ready), 0));
  QSA_TRY(qsa::launch_forward(q, k, v, row_cnt, row_cols, T, G, n_sel, scale, out, lse, status, s));
  QSA_TRY(ev.mark(1));
  return QSA_OK;
}

// The backward sequence; dk / dv are BF16, or FP32 when kv_f32.
static qsa_status_t backward_impl(const void* grad_out, const void* q, const void* k, const void* v, const void* out,
                           const float* lse, const int32_t* routes, int64_t T, int64_t T_kv, int H, int G, int n_sel,
                           float scale, void* dq, void* dk, void* dv, bool kv_f32, void* workspace,
                           size_t workspace_bytes, qsa_stream_t stream, const qsa_event_t* stage_events,
                           int n_stage_events, qsa_event_t kv_ready, const void* fwd_workspace,
                           size_t fwd_workspace_bytes) {
  // with fwd_workspace the route lists come from a forward call's workspace, and routes is not read
  const bool saved = fwd_workspace != nullptr;
  if (!grad_out || !q || !k || !v || !out || !lse || (!routes && !saved) || !dq || !dk || !dv || !workspace)
    return QSA_ERR_INVALID_ARGUMENT;
  const qsa_status_t st = check_sizes(T, T_kv, H, G, n_sel);
  if (st != QSA_OK) return st;
  if (!(scale > 0.f) || !std::isfinite(scale)) return QSA_ERR_INVALID_ARGUMENT;
  if (!aligned(grad_out, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) ||
      (!saved && !aligned(routes, 4)) || !aligned(workspace, 256) || (saved && !aligned(fwd_workspace, 256)))
    return QSA_ERR_MISALIGNED;
  const Layout L = make_layout(T, T_kv, H, G, n_sel, true);
  if (workspace_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
  const Layout LF = make_layout(T, T_kv, H, G, n_sel, false);
  if (saved && fwd_workspace_bytes < LF.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nt = (T_kv + 127) / 128;
  int* status = at<int>(workspace, L.status);
  void* rows_ws = saved ? const_cast<void*>(fwd_workspace) : workspace;  // read only when saved
  int32_t* row_cnt = at<int32_t>(rows_ws, saved ? LF.row_cnt : L.row_cnt);
  int32_t* row_cols = at<int32_t>(rows_ws, saved ? LF.row_cols : L.row_cols);
  int32_t* tile_cnt = at<int32_t>(workspace, L.tile_ctr);
  int32_t* wl_cnt = tile_cnt + nt;
  int32_t* claim = wl_cnt + L.P;
  int32_t* done = claim + 1;
  int32_t* tile_ptr = at<int32_t>(workspace, L.tile_ptr);
  int32_t* tile_fill = at<int32_t>(workspace, L.tile_fill);
  int64_t* tile_ent = at<int64_t>(workspace, L.tile_ent);
  float* delta = at<float>(workspace, L.delta);
  uint16_t* pds = at<uint16_t>(workspace, L.pds);  // [T, G, n_sel, 24]
  void* lists = at<void>(workspace, L.lists);
  int4* wl = at<int4>(workspace, L.wl);
  float* partial = at<float>(workspace, L.partial);
  const StageEvents ev{stage_events, n_stage_events, s};
  // one memset: the counters and the tile masks after them
  QSA_TRY(cudaMemsetAsync(tile_cnt, 0, L.lists - L.tile_ctr + qsa::tile_masks_bytes(T, T_kv), s));
  if (saved)
    QSA_TRY(qsa::launch_row_delta_masks(row_cnt, row_cols, T, T_kv, n_sel, at<int>(rows_ws, LF.status), status,
                                        grad_out, out, delta, H, static_cast<unsigned long long*>(lists), s));
  else
    QSA_TRY(qsa::launch_route_rows(routes, T, T_kv, n_sel, row_cnt, row_cols, nullptr, 0, status, grad_out, out,
                                   delta, H, static_cast<unsigned long long*>(lists), s));
  QSA_TRY(ev.mark(0));
  QSA_TRY(qsa::launch_tile_lists(row_cnt, row_cols, T, n_sel, nt, lists, tile_cnt, tile_ptr, tile_fill, tile_ent,
                                 status, s));
  QSA_TRY(ev.mark(1));
  QSA_TRY(qsa::launch_tile_worklist(tile_ptr, lists, T, nt, T_kv, G, L.P, L.C, wl_cnt, wl, dk, dv, kv_f32, s));
  QSA_TRY(ev.mark(2));
  // k and v are read from here on; the route work above ran without them
  if (kv_ready != nullptr) QSA_TRY(cudaStreamWaitEvent(s, reinterpret_cast<cudaEvent_t>(kv_ready), 0));
  QSA_TRY(qsa::launch_backward_dq(grad_out, q, k, v, lse, delta, row_cnt, row_cols, T, G, n_sel, scale, dq, pds,
                                  status, s));
  QSA_TRY(ev.mark(3));
  QSA_TRY(qsa::launch_backward_dkdv_union(grad_out, q, pds, row_cols, tile_ent, wl_cnt, wl, claim, done,
                                          L.P, nt, T_kv, G, n_sel, scale, partial, dk, dv, kv_f32, status, s));
  QSA_TRY(ev.mark(4));
  return QSA_OK;
}

extern "C" {

const char* qsa_status_string(qsa_status_t status) {
  switch (status) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARGUMENT: return "QSA_ERR_INVALID_ARGUMENT";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_MISALIGNED: return "QSA_ERR_MISALIGNED";
    case QSA_ERR_WORKSPACE_TOO_SMALL: return "QSA_ERR_WORKSPACE_TOO_SMALL";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
  }
  return "QSA_ERR_UNKNOWN";
}

const char* qsa_version(void) { return "qsa_b200 0.1 (sm_100a)"; }

size_t qsa_forward_workspace_size(int64_t T, int64_t T_kv, int H, int G, int n_sel) {
  if (check_sizes(T, T_kv, H, G, n_sel) != QSA_OK) return 0;
  return make_layout(T, T_kv, H, G, n_sel, false).total;
}

size_t qsa_backward_workspace_size(int64_t T, int64_t T_kv, int H, int G, int n_sel) {
  if (check_sizes(T, T_kv, H, G, n_sel) != QSA_OK) return 0;
  return make_layout(T, T_kv, H, G, n_sel, true).total;
}

qsa_status_t qsa_forward(const void* q, const void* k, const void* v, const int32_t* routes, int64_t T,
                         int64_t T_kv, int H, int G, int n_sel, float scale, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, qsa_stream_t stream) {
  return qsa_forward_ex(q, k, v, routes, T, T_kv, H, G, n_sel, scale, out, lse, workspace, workspace_bytes, stream,
                        nullptr, 0);
}

qsa_status_t qsa_forward_ex(const void* q, const void* k, const void* v, const int32_t* routes, int64_t T,
                            int64_t T_kv, int H, int G, int n_sel, float scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                            const qsa_event_t* stage_events, int n_stage_events) {
  return forward_impl(q, k, v, routes, T, T_kv, H, G, n_sel, scale, out, lse, workspace, workspace_bytes, stream,
                      stage_events, n_stage_events, nullptr);
}

qsa_status_t qsa_forward_kvwait(const void* q, const void* k, const void* v, const int32_t* routes, int64_t T,
                                int64_t T_kv, int H, int G, int n_sel, float scale, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, qsa_stream_t stream, qsa_event_t kv_ready,
                                const qsa_event_t* stage_events, int n_stage_events) {
  return forward_impl(q, k, v, routes, T, T_kv, H, G, n_sel, scale, out, lse, workspace, workspace_bytes, stream,
                      stage_events, n_stage_events, kv_ready);
}

qsa_status_t qsa_backward(const void* grad_out, const void* q, const void* k, const void* v, const void* out,
                          const float* lse, const int32_t* routes, int64_t T, int64_t T_kv, int H, int G,
                          int n_sel, float scale, void* dq, void* dk, void* dv, void* workspace,
                          size_t workspace_bytes, qsa_stream_t stream) {
  return qsa_backward_ex(grad_out, q, k, v, out, lse, routes, T, T_kv, H, G, n_sel, scale, dq, dk, dv, workspace,
                         workspace_bytes, stream, nullptr, 0);
}

qsa_status_t qsa_backward_ex(const void* grad_out, const void* q, const void* k, const void* v, const void* out,
                             const float* lse, const int32_t* routes, int64_t T, int64_t T_kv, int H, int G,
                             int n_sel, float scale, void* dq, void* dk, void* dv, void* workspace,
                             size_t workspace_bytes, qsa_stream_t stream, const qsa_event_t* stage_events,
                             int n_stage_events) {
  return backward_impl(grad_out, q, k, v, out, lse, routes, T, T_kv, H, G, n_sel, scale, dq, dk, dv, false, workspace,
                       workspace_bytes, stream, stage_events, n_stage_events, nullptr, nullptr, 0);
}

qsa_status_t qsa_backward_kvwait(const void* grad_out, const void* q, const void* k, const void* v, const void* out,
                                 const float* lse, const int32_t* routes, int64_t T, int64_t T_kv, int H, int G,
                                 int n_sel, float scale, void* dq, void* dk, void* dv, int kv_fp32, void* workspace,
                                 size_t workspace_bytes, qsa_stream_t stream, qsa_event_t kv_ready,
                                 const qsa_event_t* stage_events, int n_stage_events) {
  return backward_impl(grad_out, q, k, v, out, lse, routes, T, T_kv, H, G, n_sel, scale, dq, dk, dv, kv_fp32 != 0,
                       workspace, workspace_bytes, stream, stage_events, n_stage_events, kv_ready, nullptr, 0);
}

qsa_status_t qsa_backward_saved(const void* grad_out, const void* q, const void* k, const void* v, const void* out,
                                const float* lse, const void* fwd_workspace, size_t fwd_workspace_bytes, int64_t T,
                                int64_t T_kv, int H, int G, int n_sel, float scale, void* dq, void* dk, void* dv,
                                int kv_fp32, void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                                qsa_event_t kv_ready, const qsa_event_t* stage_events, int n_stage_events) {
  if (!fwd_workspace) return QSA_ERR_INVALID_ARGUMENT;
  return backward_impl(grad_out, q, k, v, out, lse, nullptr, T, T_kv, H, G, n_sel, scale, dq, dk, dv, kv_fp32 != 0,
                       workspace, workspace_bytes, stream, stage_events, n_stage_events, kv_ready, fwd_workspace,
                       fwd_workspace_bytes);
}

qsa_status_t qsa_backward_fp32kv(const void* grad_out, const void* q, const void* k, const void* v, const void* out,
                                 const float* lse, const int32_t* routes, int64_t T, int64_t T_kv, int H, int G,
                                 int n_sel, float scale, void* dq, float* dk, float* dv, void* workspace,
                                 size_t workspace_bytes, qsa_stream_t stream) {
  return backward_impl(grad_out, q, k, v, out, lse, routes, T, T_kv, H, G, n_sel, scale, dq, dk, dv, true, workspace,
                       workspace_bytes, stream, nullptr, 0, nullptr, nullptr, 0);
}

int qsa_launch_count(int64_t T, int64_t T_kv, int H, int G, int n_sel, int backward) {
  if (check_sizes(T, T_kv, H, G, n_sel) != QSA_OK) return 0;
  // backward: route rows (+ tile masks), column scans, tile-pointer scan, tile fill, work lists, dQ, dK/dV
  return backward ? 7 : 2;
}

qsa_status_t qsa_bitmap_routes(const uint8_t* sel_blocks, const int32_t* lo, const int32_t* hi,
                               const int32_t* blk_base, const int32_t* tok_base, int64_t T, int64_t NB,
                               int64_t T_kv, int block_size, int n_sel, int32_t* routes, int32_t* row_cnt,
                               int32_t* max_cnt, qsa_stream_t stream) {
  if (!sel_blocks || !lo || !hi || !blk_base || !tok_base || !routes) return QSA_ERR_INVALID_ARGUMENT;
  if (T < 1 || NB < 1 || T_kv < 1 || n_sel < 1 || block_size < 1) return QSA_ERR_INVALID_ARGUMENT;
  if (T_kv > INT32_MAX || T > INT32_MAX / n_sel) return QSA_ERR_INVALID_ARGUMENT;
  if (!aligned(sel_blocks, 16) || !aligned(lo, 4) || !aligned(hi, 4) || !aligned(blk_base, 4) || !aligned(tok_base, 4) ||
      !aligned(routes, 4) || (row_cnt && !aligned(row_cnt, 4)) || (max_cnt && !aligned(max_cnt, 4)))
    return QSA_ERR_MISALIGNED;
  QSA_TRY(qsa::launch_bitmap_routes(sel_blocks, lo, hi, blk_base, tok_base, T, NB, T_kv, block_size, n_sel, routes,
                                    row_cnt, max_cnt, reinterpret_cast<cudaStream_t>(stream)));
  return QSA_OK;
}

qsa_status_t qsa_selector_scores(const void* qi, const void* kbar, int64_t T, int64_t NB, int Hi, int Di,
                                 float scale, const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base,
                                 float* scores, int64_t score_stride, int* status, qsa_stream_t stream) {
  if (!qi || !kbar || !scores) return QSA_ERR_INVALID_ARGUMENT;
  if (T < 1 || NB < 1 || score_stride < NB || !(scale > 0.f) || !std::isfinite(scale))
    return QSA_ERR_INVALID_ARGUMENT;
  if (Di != 128 || (Hi != 32 && Hi != 64 && Hi != 128 && Hi != 256)) return QSA_ERR_UNSUPPORTED;
  if (T > INT32_MAX / Hi || NB > INT32_MAX || T > INT64_MAX / score_stride) return QSA_ERR_INVALID_ARGUMENT;
  if (!aligned(qi, 16) || !aligned(kbar, 16) || !aligned(scores, 4) || (pos && !aligned(pos, 4)) ||
      (blk_base && !aligned(blk_base, 4)) || (tok_base && !aligned(tok_base, 4)) || (status && !aligned(status, 4)))
    return QSA_ERR_MISALIGNED;
  QSA_TRY(qsa::launch_selector_scores(qi, kbar, T, NB, Hi, scale, pos, blk_base, tok_base, scores, score_stride,
                                      status, reinterpret_cast<cudaStream_t>(stream)));
  return QSA_OK;
}

qsa_status_t qsa_selector_topk(const float* scores, int64_t score_stride, int64_t T, int64_t NB, int k,
                               const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base, int32_t* blocks,
                               int32_t* routes, qsa_stream_t stream) {
  if (!scores || !blocks || !routes) return QSA_ERR_INVALID_ARGUMENT;
  if (T < 1 || NB < 1 || k < 1 || score_stride < NB) return QSA_ERR_INVALID_ARGUMENT;
  if (T > INT32_MAX || k > (INT32_MAX / 4) - 1 || T > INT32_MAX / (4 * (k + 1))) return QSA_ERR_INVALID_ARGUMENT;
  if (!aligned(scores, 4) || !aligned(blocks, 4) || !aligned(routes, 4) || (pos && !aligned(pos, 4)) ||
      (blk_base && !aligned(blk_base, 4)) || (tok_base && !aligned(tok_base, 4)))
    return QSA_ERR_MISALIGNED;
  QSA_TRY(qsa::launch_selector_topk(scores, score_stride, T, NB, k, pos, blk_base, tok_base, blocks, routes,
                                    reinterpret_cast<cudaStream_t>(stream)));
  return QSA_OK;
}

size_t qsa_route_plan_scratch_size(int64_t T, int64_t T_kv) {
  if (T < 1 || T_kv < 1 || T_kv > INT32_MAX) return 0;
  const size_t nq = static_cast<size_t>((T_kv + 3) / 4);
  return 2 * align256(nq * 4) + align256(nq * 8);
}

qsa_status_t qsa_route_plan(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel, int32_t* row_cnt,
                            int32_t* row_cols, int32_t* quad_ptr, int64_t* quad_ent, void* scratch,
                            size_t scratch_bytes, qsa_stream_t stream) {
  if (!routes || !row_cnt || !row_cols || !quad_ptr || !quad_ent || !scratch) return QSA_ERR_INVALID_ARGUMENT;
  const qsa_status_t st = check_sizes(T, T_kv, qsa::kHeadsPerGroup, 1, n_sel);
  if (st != QSA_OK) return st;
  if (!aligned(routes, 4) || !aligned(row_cnt, 4) || !aligned(row_cols, 4) || !aligned(quad_ptr, 4) ||
      !aligned(quad_ent, 8) || !aligned(scratch, 256))
    return QSA_ERR_MISALIGNED;
  if (scratch_bytes < qsa_route_plan_scratch_size(T, T_kv)) return QSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nq = (T_kv + 3) / 4;
  int32_t* quad_cnt = static_cast<int32_t*>(scratch);
  int32_t* quad_fill = at<int32_t>(scratch, align256(static_cast<size_t>(nq) * 4));
  int32_t* phase_ptr = at<int32_t>(scratch, 2 * align256(static_cast<size_t>(nq) * 4));
  QSA_TRY(cudaMemsetAsync(quad_cnt, 0, static_cast<size_t>(nq) * 4, s));
  QSA_TRY(qsa::launch_route_rows(routes, T, T_kv, n_sel, row_cnt, row_cols, quad_cnt, 2, nullptr, nullptr, nullptr,
                                 nullptr, qsa::kHeadsPerGroup, nullptr, s));
  QSA_TRY(qsa::launch_quad_scan(quad_cnt, nq, quad_ptr, quad_fill, s));
  QSA_TRY(qsa::launch_quad_fill(row_cnt, row_cols, T, n_sel, quad_fill, quad_ent, s));
  QSA_TRY(qsa::launch_quad_sort(quad_ptr, nq, quad_ent, 1, static_cast<int>(T), phase_ptr, s));
  return QSA_OK;
}

int qsa_union_group(int n_sel) { return n_sel < 1 || n_sel > kMaxSel ? 0 : qsa::union_group(n_sel); }

qsa_status_t qsa_union_plan(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel, int32_t* row_cnt,
                            int32_t* row_cols, int32_t* ucnt, int32_t* ukey, uint8_t* uown, qsa_stream_t stream) {
  if (!routes || !row_cnt || !row_cols || !ucnt || !ukey || !uown) return QSA_ERR_INVALID_ARGUMENT;
  const qsa_status_t st = check_sizes(T, T_kv, qsa::kHeadsPerGroup, 1, n_sel);
  if (st != QSA_OK) return st;
  if (!aligned(routes, 4) || !aligned(row_cnt, 4) || !aligned(row_cols, 4) || !aligned(ucnt, 4) || !aligned(ukey, 4))
    return QSA_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  QSA_TRY(qsa::launch_route_rows(routes, T, T_kv, n_sel, row_cnt, row_cols, nullptr, 0, nullptr, nullptr, nullptr,
                                 nullptr, qsa::kHeadsPerGroup, nullptr, s));
  QSA_TRY(qsa::launch_union_lists(row_cnt, row_cols, T, n_sel, qsa::union_group(n_sel), ucnt, ukey, uown, s));
  return QSA_OK;
}

size_t qsa_tile_plan_scratch_size(int64_t T, int64_t T_kv) {
  if (T < 1 || T_kv < 1 || T_kv > INT32_MAX) return 0;
  const size_t nt = static_cast<size_t>((T_kv + 127) / 128);
  return 2 * align256(nt * 4) + align256(qsa::tile_lists_bytes(T, T_kv));
}

qsa_status_t qsa_tile_plan(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel, int32_t* row_cnt,
                           int32_t* row_cols, int32_t* tile_ptr, int64_t* tile_ent, void* scratch,
                           size_t scratch_bytes, qsa_stream_t stream) {
  if (!routes || !row_cnt || !row_cols || !tile_ptr || !tile_ent || !scratch) return QSA_ERR_INVALID_ARGUMENT;
  const qsa_status_t st = check_sizes(T, T_kv, qsa::kHeadsPerGroup, 1, n_sel);
  if (st != QSA_OK) return st;
  if (!aligned(routes, 4) || !aligned(row_cnt, 4) || !aligned(row_cols, 4) || !aligned(tile_ptr, 4) ||
      !aligned(tile_ent, 8) || !aligned(scratch, 256))
    return QSA_ERR_MISALIGNED;
  if (scratch_bytes < qsa_tile_plan_scratch_size(T, T_kv)) return QSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nt = (T_kv + 127) / 128;
  int32_t* tile_cnt = static_cast<int32_t*>(scratch);
  int32_t* tile_fill = at<int32_t>(scratch, align256(static_cast<size_t>(nt) * 4));
  void* lists = at<void>(scratch, 2 * align256(static_cast<size_t>(nt) * 4));
  QSA_TRY(cudaMemsetAsync(lists, 0, qsa::tile_masks_bytes(T, T_kv), s));
  QSA_TRY(qsa::launch_route_rows(routes, T, T_kv, n_sel, row_cnt, row_cols, nullptr, 0, nullptr, nullptr, nullptr,
                                 nullptr, qsa::kHeadsPerGroup, static_cast<unsigned long long*>(lists), s));
  QSA_TRY(qsa::launch_tile_lists(row_cnt, row_cols, T, n_sel, nt, lists, tile_cnt, tile_ptr, tile_fill, tile_ent,
                                 nullptr, s));
  return QSA_OK;
}

}  // extern "C"
