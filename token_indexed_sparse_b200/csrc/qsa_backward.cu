// QSA backward, following the backward equations of the cuDNN-Frontend
// "Query Sparse Attention (QSA)" page ("Selection and components"), per query
// head h and its KV head g:
//   S = scale Q K^T,  P = exp(S - lse) (zero outside R_t),
//   delta = rowsum(dO * out),  dP = dO V^T,  dS = P * (dP - delta),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO  (dK/dV summed over heads).
//
// This file holds dq_kernel, persistent over (query t, group g) items: it
// recomputes S and dP over R_t (K/V rows gathered like the forward), forms P
// and dS with delta from the route kernel, accumulates dQ, and stores the BF16
// P and dS of every routed pair for the dK/dV pass (qsa_dkdv_union.cu): one
// 48-byte record [P h0..h11 | dS h0..h11] per (t, g, position in R_t), pds
// [T, G, n_sel, 24].  No floating-point atomics.
#include "qsa_internal.h"
#include "qsa_pipe.cuh"

namespace qsa {
namespace {

// ---------------------------------------------------------------------------
// dQ (+ P/dS records): persistent, CPS CTAs of NW warps per SM
// ---------------------------------------------------------------------------
// Same pipeline as the forward kernel (qsa_pipe.cuh): chunks of KEYS = 8 NW keys
// of K and V rows gathered STAGES - 1 chunks ahead into a ring of swizzled tiles
// (rows past the end of R_t zero-filled: dQ multiplies their zero dS by their K
// rows).  Once per item the 12 Q and dO rows, the 12 LSE values and the 12 delta
// values (delta = rowsum(dO * out), computed by the route kernel) go to an item
// buffer.  Per chunk, warp w computes S = Q K^T and dP = dO V^T for keys
// 8w..8w+7, P = exp2(S*scale*log2e - lse*log2e), dS = P (dP - delta), stores the
// BF16 P / dS records and accumulates dQ[:, DPW*w : DPW*(w+1)] += dS K.  The
// next chunk's gather is issued right after the landing barrier, except at an
// item's first chunk: there it waits for a second barrier, once every warp has
// taken the item buffer into registers (seq32k dQ 5.04 -> 5.01 ms, cp128k
// 2.49 -> 2.39 ms against issuing after that barrier in every chunk).
constexpr int kRec = 24;  // bf16 per (t, g, key) record: 12 P + 12 dS
constexpr int kFirst = 1, kLast = 2, kSlot = 4;

template <int NW, int STAGES, int CPS>
struct DqShape {
  static constexpr int kThreads = NW * 32;
  static constexpr int kKeys = 8 * NW;
  static constexpr int kDpw = kHeadDim / NW;  // dQ dims per warp
  static constexpr int kNt = kDpw / 8;
  static constexpr int kKs = kKeys / 16;
  static constexpr int kTile = kKeys * 512;
  static constexpr int kStageBytes = 2 * kTile;
  // Item buffers: with a 2-stage ring the next item's buffer is issued after
  // every warp has read the current one, so one buffer suffices; deeper rings
  // keep an item pending and alternate two.
  static constexpr int kSlots = STAGES == 2 ? 1 : 2;
  static constexpr int kItemQ = 0, kItemDO = kHeadsPerGroup * 512, kItemLse = 2 * kHeadsPerGroup * 512;
  static constexpr int kItemDelta = kItemLse + 64, kItemBytes = kItemDelta + 64;
  static constexpr int kOffItem = STAGES * kStageBytes;
  static constexpr int kOffZero = kOffItem + kSlots * kItemBytes;
  static constexpr int kDsStride = kKeys + 8;  // bf16 per dS row (conflict-free ldmatrix)
  static constexpr int kOffDS = kOffZero + 512;
  static constexpr int kOffRec = kOffDS + ((kRowTile * kDsStride * 2 + 15) / 16) * 16;
  static constexpr int kOffDesc = kOffRec + kKeys * kRec * 2;
  static constexpr int kSmemBytes = kOffDesc + STAGES * 16;
  static_assert(kSmemBytes * CPS + 1024 * CPS <= 233472, "shared memory per SM");
  static_assert(kOffItem % 16 == 0 && kItemBytes % 16 == 0 && kOffZero % 16 == 0 && kOffDS % 16 == 0 &&
                    kOffRec % 16 == 0 && kOffDesc % 16 == 0,
                "alignment");
  static_assert(kKs >= 1 && kNt % 2 == 0 && kThreads >= 24, "shape");
};

template <int NW, int STAGES, int CPS>
__global__ void __launch_bounds__(NW * 32, CPS)
dq_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ q,
          const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
          const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ row_cnt,
          const int32_t* __restrict__ row_cols, int64_t n_items, int G, int n_sel, float scale, float scale_log2,
          __nv_bfloat16* __restrict__ dq, uint16_t* __restrict__ pds, const int* __restrict__ status) {
  using S_ = DqShape<NW, STAGES, CPS>;
  constexpr int KEYS = S_::kKeys, kTile = S_::kTile, kStageBytes = S_::kStageBytes, kDsStride = S_::kDsStride;
  constexpr int kNt = S_::kNt, kKs = S_::kKs, kItemBytes = S_::kItemBytes, kThreads = S_::kThreads;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, cq = lane & 3, mi = lane >> 3;
  const int H = G * kHeadsPerGroup;
  int4* desc = reinterpret_cast<int4*>(smem + S_::kOffDesc);
  __nv_bfloat16* sDS = reinterpret_cast<__nv_bfloat16*>(smem + S_::kOffDS);
  uint16_t* sRec = reinterpret_cast<uint16_t*>(smem + S_::kOffRec);
  const uint32_t sDSa = smem_u32(sDS);
  // route lists that failed their tag check are not read (the status word
  // already reports it; dq is left unwritten)
  if (status != nullptr && *status == kStatusBadPlan) return;
  if (tid < 32) reinterpret_cast<uint4*>(smem + S_::kOffZero)[tid] = make_uint4(0, 0, 0, 0);

  Cursor cur;
  cursor_init<KEYS>(cur, row_cnt, n_items, G);
  int32_t key[8];
  cursor_keys<KEYS>(key, cur, n_items, G, row_cols, n_sel);
  int islot = 0;  // item buffer of the next non-empty item
  auto issue = [&](int stage) {
    const uint32_t st = sbase + stage * kStageBytes;
    if (cur.it < n_items) {
      const int64_t t = cur.t;
      const int g = cur.g;
      const int nk = cursor_nk<KEYS>(cur, n_items);
      int flags = (cur.ch == 0 ? kFirst : 0) | (cur.ch == cur.nch - 1 ? kLast : 0);
      if (nk > 0) {
        gather_rows(st, st + kTile, k, v, key, g, G, nk);
        if (cur.ch == 0) {
          const int64_t qrow0 = t * H + g * kHeadsPerGroup;
          const uint32_t ib = sbase + S_::kOffItem + islot * kItemBytes;
          gather_heads<NW>(ib + S_::kItemQ, q + qrow0 * kHeadDim);
          gather_heads<NW>(ib + S_::kItemDO, dout + qrow0 * kHeadDim);
          const int j = tid - (kThreads - 24);  // the last 24 threads: 12 LSE + 12 delta values
          if (j >= 0 && j < kHeadsPerGroup) cp_async4(ib + S_::kItemLse + 4 * j, lse + qrow0 + j);
          if (j >= kHeadsPerGroup) cp_async4(ib + S_::kItemDelta + 4 * (j - 12), delta + qrow0 + (j - 12));
          flags |= islot ? kSlot : 0;
          if (S_::kSlots > 1) islot ^= 1;
        } else {
          // the item's slot was flipped at its first chunk
          flags |= (S_::kSlots > 1 ? (islot ? 0 : kSlot) : 0);
        }
      }
      if (tid == 0) desc[stage] = make_int4(static_cast<int>(t), g, nk, flags | ((cur.ch) << 3));
    } else if (tid == 0) {
      desc[stage] = make_int4(0, 0, -1, 0);
    }
    cp_async_commit();
    cursor_next<KEYS>(cur, row_cnt, n_items, G);
    cursor_keys<KEYS>(key, cur, n_items, G, row_cols, n_sel);
  };
#pragma unroll
  for (int s0 = 0; s0 < STAGES - 1; ++s0) issue(s0);

  uint32_t qa[16][4], da[16][4];
  float acc[kNt][4];
  float ls0 = INFINITY, ls1 = INFINITY, dl0 = 0.f, dl1 = 0.f;

  for (int c = 0;; ++c) {
    const int stage = c % STAGES;
    const uint32_t st = sbase + stage * kStageBytes;
    cp_async_wait<STAGES - 2>();
    __syncthreads();  // chunk c has landed; every warp is done with chunk c - 1
    const int4 d = desc[stage];
    const int nk = d.z;
    if (nk < 0) break;
    const int64_t t = d.x;
    const int g = d.y;
    const int64_t qrow0 = t * H + g * kHeadsPerGroup;
    if (nk == 0) {  // padding query: dQ = 0 (no item buffer is used)
      issue((c + STAGES - 1) % STAGES);
      uint4* orow = reinterpret_cast<uint4*>(dq + qrow0 * kHeadDim);
      for (int i = tid; i < kHeadsPerGroup * 32; i += kThreads) orow[i] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const bool first = (d.w & kFirst) != 0;
    if (!first) issue((c + STAGES - 1) % STAGES);  // the item buffer was read at the item's first chunk
    if (first) {
      const uint32_t ib = sbase + S_::kOffItem + ((d.w & kSlot) ? kItemBytes : 0);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const int r = ((mi & 1) << 3) + (lane & 7);
        const int cc = 2 * ks + (mi >> 1);
        const bool real = r < kHeadsPerGroup;
        ldsm_x4(qa[ks], real ? ib + S_::kItemQ + swz512(r, cc) : sbase + S_::kOffZero + (cc << 4));
        ldsm_x4(da[ks], real ? ib + S_::kItemDO + swz512(r, cc) : sbase + S_::kOffZero + (cc << 4));
      }
      const float* il = reinterpret_cast<const float*>(smem + (ib - sbase) + S_::kItemLse);
      const float* idl = reinterpret_cast<const float*>(smem + (ib - sbase) + S_::kItemDelta);
      ls0 = il[gq] * kLog2e;
      dl0 = idl[gq];
      ls1 = gq + 8 < kHeadsPerGroup ? il[gq + 8] * kLog2e : INFINITY;
      dl1 = gq + 8 < kHeadsPerGroup ? idl[gq + 8] : 0.f;
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    }
    // S = Q K^T and dP = dO V^T for this warp's 8 keys, two chains each
    float s[4], dp[4];
    {
      float sa[2][4], pa[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) sa[j][i] = pa[j][i] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 16; ks += 2) {
        uint32_t b[4], e[4];
        const uint32_t off = swz512(warp * 8 + (lane & 7), 2 * ks + mi);
        ldsm_x4(b, st + off);
        ldsm_x4(e, st + kTile + off);
        mma_16816(sa[(ks >> 1) & 1], qa[ks], b[0], b[1]);
        mma_16816(pa[(ks >> 1) & 1], da[ks], e[0], e[1]);
        mma_16816(sa[(ks >> 1) & 1], qa[ks + 1], b[2], b[3]);
        mma_16816(pa[(ks >> 1) & 1], da[ks + 1], e[2], e[3]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        s[i] = sa[0][i] + sa[1][i];
        dp[i] = pa[0][i] + pa[1][i];
      }
    }
    if (first) {
      __syncthreads();  // every warp has read this item's buffer: its slot may be refilled
      issue((c + STAGES - 1) % STAGES);
    }

    const int key0 = warp * 8 + 2 * cq;
    const bool v0 = key0 < nk, v1 = key0 + 1 < nk;
    const float p0 = v0 ? exp2f(s[0] * scale_log2 - ls0) : 0.f;
    const float p1 = v1 ? exp2f(s[1] * scale_log2 - ls0) : 0.f;
    const float p2 = v0 ? exp2f(s[2] * scale_log2 - ls1) : 0.f;
    const float p3 = v1 ? exp2f(s[3] * scale_log2 - ls1) : 0.f;
    const uint32_t P01 = pack_bf16(p0, p1), P23 = pack_bf16(p2, p3);
    const uint32_t D01 = pack_bf16(p0 * (dp[0] - dl0), p1 * (dp[1] - dl0));
    const uint32_t D23 = pack_bf16(p2 * (dp[2] - dl1), p3 * (dp[3] - dl1));
    *reinterpret_cast<uint32_t*>(sDS + gq * kDsStride + key0) = D01;
    *reinterpret_cast<uint32_t*>(sDS + (gq + 8) * kDsStride + key0) = D23;
    // records: [key][P h0..h11 | dS h0..h11]
    sRec[key0 * kRec + gq] = static_cast<uint16_t>(P01 & 0xffff);
    sRec[(key0 + 1) * kRec + gq] = static_cast<uint16_t>(P01 >> 16);
    sRec[key0 * kRec + 12 + gq] = static_cast<uint16_t>(D01 & 0xffff);
    sRec[(key0 + 1) * kRec + 12 + gq] = static_cast<uint16_t>(D01 >> 16);
    if (gq + 8 < kHeadsPerGroup) {
      sRec[key0 * kRec + gq + 8] = static_cast<uint16_t>(P23 & 0xffff);
      sRec[(key0 + 1) * kRec + gq + 8] = static_cast<uint16_t>(P23 >> 16);
      sRec[key0 * kRec + 20 + gq] = static_cast<uint16_t>(D23 & 0xffff);
      sRec[(key0 + 1) * kRec + 20 + gq] = static_cast<uint16_t>(D23 >> 16);
    }
    __syncthreads();
    {
      // the chunk's records, 48 bytes per key, to their run of the record array
      const int base = (d.w >> 3) * KEYS;
      const uint4* src = reinterpret_cast<const uint4*>(sRec);
      uint4* dst = reinterpret_cast<uint4*>(pds + ((t * G + g) * n_sel + base) * kRec);
      for (int i = tid; i < nk * 3; i += kThreads) dst[i] = src[i];
    }
    // dQ[:, DPW*w : DPW*(w+1)] += dS K over the chunk's keys
#pragma unroll
    for (int ks = 0; ks < kKs; ++ks) {
      uint32_t a[4];
      ldsm_x4(a, sDSa + (((((mi & 1) << 3) + (lane & 7)) * kDsStride + 16 * ks + ((mi >> 1) << 3)) << 1));
#pragma unroll
      for (int nt = 0; nt < kNt; nt += 2) {
        uint32_t b[4];
        ldsm_x4_t(b, st + swz512(16 * ks + ((mi & 1) << 3) + (lane & 7), warp * kNt + nt + (mi >> 1)));
        mma_16816(acc[nt], a, b[0], b[1]);
        mma_16816(acc[nt + 1], a, b[2], b[3]);
      }
    }
    if (d.w & kLast) {
      __nv_bfloat16* drow = dq + qrow0 * kHeadDim;
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) {
        const int dim = warp * S_::kDpw + nt * 8 + 2 * cq;
        *reinterpret_cast<uint32_t*>(drow + gq * kHeadDim + dim) = pack_bf16(acc[nt][0] * scale, acc[nt][1] * scale);
        if (gq + 8 < kHeadsPerGroup)
          *reinterpret_cast<uint32_t*>(drow + (gq + 8) * kHeadDim + dim) =
              pack_bf16(acc[nt][2] * scale, acc[nt][3] * scale);
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace

// dQ kernel shape used by launch_backward_dq: 2 CTAs of 4 warps per SM, 32-key
// chunks, 2-stage ring.
constexpr int kDqWarps = 4, kDqStages = 2, kDqCtasPerSm = 2;

cudaError_t launch_backward_dq(const void* grad_out, const void* q, const void* k, const void* v,
                               const float* lse, const float* delta, const int32_t* row_cnt,
                               const int32_t* row_cols, int64_t T, int G, int n_sel, float scale, void* dq,
                               uint16_t* pds, const int* status, cudaStream_t s) {
  using S_ = DqShape<kDqWarps, kDqStages, kDqCtasPerSm>;
  auto kern = dq_kernel<kDqWarps, kDqStages, kDqCtasPerSm>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S_::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t n_items = T * G;
  const int64_t slots = static_cast<int64_t>(kDqCtasPerSm) * sm_count();
  const int64_t grid = n_items < slots ? n_items : slots;
  kern<<<static_cast<unsigned>(grid), S_::kThreads, S_::kSmemBytes, s>>>(
      static_cast<const __nv_bfloat16*>(grad_out), static_cast<const __nv_bfloat16*>(q),
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), lse, delta, row_cnt, row_cols,
      n_items, G, n_sel, scale, scale * kLog2e, static_cast<__nv_bfloat16*>(dq), pds, status);
  return cudaGetLastError();
}

}  // namespace qsa
