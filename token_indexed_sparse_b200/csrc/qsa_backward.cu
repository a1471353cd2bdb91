// QSA backward, following the backward equations of the cuDNN-Frontend
// "Query Sparse Attention (QSA)" page ("Selection and components"), per query
// head h and its KV head g:
//   S = scale Q K^T,  P = exp(S - lse) (zero outside R_t),
//   delta = rowsum(dO * out),  dP = dO V^T,  dS = P * (dP - delta),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO  (dK/dV summed over heads).
//
// Two kernels, neither using floating-point atomics:
//   * dq_kernel, one CTA per (query t, group g): recomputes S and dP over R_t
//     (K/V rows gathered like the forward), forms P and dS, accumulates dQ, and
//     stores delta and the BF16 P / dS of every routed pair (`pds`, one 48-byte
//     record [P h0..h11 | dS h0..h11] per (t, g, position in R_t)).
//   * dkdv_kernel, one CTA per (aligned key quad, group g): walks the quad's
//     query list in ascending query order and accumulates dK^T = Q^T dS and
//     dV^T = dO^T P on tensor cores.  Each warp owns 64 of the 256 dims and loads
//     its Q / dO slices straight from global memory into A fragments, so the
//     kernel uses no shared memory; the fixed list order makes dK/dV bitwise
//     reproducible.
#include "qsa_device.cuh"
#include "qsa_internal.h"

namespace qsa {
namespace {

// ---------------------------------------------------------------------------
// dQ (+ delta, P/dS records)
// ---------------------------------------------------------------------------
constexpr int kDqThreads = 128;
constexpr int kChunk = 32;
constexpr int kDsStride = 40;  // bf16 per row of the dS tile (80 B)
constexpr int kTileBytes = kChunk * 512;
constexpr int kRec = 24;       // bf16 per (t, g, key) record: 12 P + 12 dS
constexpr int kOffDO = 16 * 512;
constexpr int kOffK = kOffDO + 16 * 512;
constexpr int kOffV = kOffK + 2 * kTileBytes;
constexpr int kOffDS = kOffV + 2 * kTileBytes;
constexpr int kOffRec = kOffDS + kRowTile * kDsStride * 2;
constexpr int kOffDelta = kOffRec + kChunk * kRec * 2;
constexpr int kOffLse = kOffDelta + kRowTile * 4;
constexpr int kOffCols = kOffLse + kRowTile * 4;

__global__ void __launch_bounds__(kDqThreads, 2)
dq_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ q,
          const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
          const __nv_bfloat16* __restrict__ out, const float* __restrict__ lse,
          const int32_t* __restrict__ row_cnt, const int32_t* __restrict__ row_cols, int G, int n_sel,
          float scale, float scale_log2, __nv_bfloat16* __restrict__ dq, float* __restrict__ delta_out,
          uint16_t* __restrict__ pds) {
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sDS = reinterpret_cast<__nv_bfloat16*>(smem + kOffDS);
  uint16_t* sRec = reinterpret_cast<uint16_t*>(smem + kOffRec);
  float* sDelta = reinterpret_cast<float*>(smem + kOffDelta);
  float* sLse = reinterpret_cast<float*>(smem + kOffLse);
  int32_t* sCols = reinterpret_cast<int32_t*>(smem + kOffCols);

  const int H = G * kHeadsPerGroup;
  const int64_t t = blockIdx.x / G;
  const int g = static_cast<int>(blockIdx.x - t * G);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, cq = lane & 3;
  const int cnt = row_cnt[t];
  const int64_t qrow0 = t * H + g * kHeadsPerGroup;

  if (cnt == 0) {  // padding query: dQ = 0, nothing else is read later
    uint4* o = reinterpret_cast<uint4*>(dq + qrow0 * kHeadDim);
    for (int i = tid; i < kHeadsPerGroup * 32; i += kDqThreads) o[i] = make_uint4(0, 0, 0, 0);
    if (tid < kHeadsPerGroup) delta_out[qrow0 + tid] = 0.f;
    return;
  }

  for (int i = tid; i < cnt; i += kDqThreads) sCols[i] = row_cols[t * n_sel + i];
  const uint32_t sQa = smem_u32(smem), sDOa = smem_u32(smem + kOffDO);
  const uint32_t sKa = smem_u32(smem + kOffK), sVa = smem_u32(smem + kOffV);
  for (int i = tid; i < 2 * kRowTile * 32; i += kDqThreads) {
    const int tensor = i >> 9, r = (i >> 5) & 15, c = i & 31;
    const bool ok = r < kHeadsPerGroup;
    const __nv_bfloat16* src = (tensor ? dout : q) + (qrow0 + (ok ? r : 0)) * kHeadDim + c * 8;
    cp_async16((tensor ? sDOa : sQa) + swz512(r, c), src, ok);
  }
  cp_async_commit();
  if (tid < kRowTile) sLse[tid] = tid < kHeadsPerGroup ? lse[qrow0 + tid] * kLog2e : INFINITY;
  __syncthreads();

  const int n_chunks = (cnt + kChunk - 1) / kChunk;
  auto issue = [&](int ch) {
    const int stage = ch & 1, base = ch * kChunk;
    const int nk = min(kChunk, cnt - base);
#pragma unroll 4
    for (int i = tid; i < 2 * kChunk * 32; i += kDqThreads) {
      const int tensor = i / (kChunk * 32);
      const int r = (i >> 5) & (kChunk - 1), c = i & 31;
      const bool ok = r < nk;
      const int64_t key = ok ? sCols[base + r] : 0;
      const __nv_bfloat16* src = (tensor ? v : k) + (key * G + g) * kHeadDim + c * 8;
      cp_async16((tensor ? sVa : sKa) + stage * kTileBytes + swz512(r, c), src, ok);
    }
  };
  issue(0);
  cp_async_commit();
  if (n_chunks > 1) issue(1);
  cp_async_commit();
  cp_async_wait<2>();  // Q and dO tiles have landed
  __syncthreads();

  // delta = rowsum(dO * out) in fp32 from the BF16 forward output; warp w owns rows 3w..3w+2.
  for (int r = warp * 3; r < warp * 3 + 3; ++r) {
    const uint4 ov = *reinterpret_cast<const uint4*>(out + (qrow0 + r) * kHeadDim + lane * 8);
    uint4 dv;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(dv.x), "=r"(dv.y), "=r"(dv.z), "=r"(dv.w) : "r"(sDOa + swz512(r, lane)));
    float acc = bf16_lo(ov.x) * bf16_lo(dv.x) + bf16_hi(ov.x) * bf16_hi(dv.x) +
                bf16_lo(ov.y) * bf16_lo(dv.y) + bf16_hi(ov.y) * bf16_hi(dv.y) +
                bf16_lo(ov.z) * bf16_lo(dv.z) + bf16_hi(ov.z) * bf16_hi(dv.z) +
                bf16_lo(ov.w) * bf16_lo(dv.w) + bf16_hi(ov.w) * bf16_hi(dv.w);
    acc = warp_sum(acc);
    if (lane == 0) {
      sDelta[r] = acc;
      delta_out[qrow0 + r] = acc;
    }
  }
  if (tid < kRowTile - kHeadsPerGroup) sDelta[kHeadsPerGroup + tid] = 0.f;

  uint32_t qa[16][4], da[16][4];
#pragma unroll
  for (int ks = 0; ks < 16; ++ks) {
    const int mi = lane >> 3;
    const uint32_t off = swz512(((mi & 1) << 3) + (lane & 7), 2 * ks + (mi >> 1));
    ldsm_x4(qa[ks], sQa + off);
    ldsm_x4(da[ks], sDOa + off);
  }
  __syncthreads();  // sDelta
  const float dl0 = sDelta[gq], dl1 = sDelta[gq + 8];
  const float ls0 = sLse[gq], ls1 = sLse[gq + 8];

  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  const uint32_t sDSa = smem_u32(sDS);
  uint16_t* pds_row = pds + (t * G + g) * static_cast<int64_t>(n_sel) * kRec;

  for (int ch = 0; ch < n_chunks; ++ch) {
    const int stage = ch & 1, base = ch * kChunk;
    const int nk = min(kChunk, cnt - base);
    cp_async_wait<1>();
    __syncthreads();

    float s[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t kb = sKa + stage * kTileBytes, vb = sVa + stage * kTileBytes;
#pragma unroll
    for (int ks = 0; ks < 16; ks += 2) {
      uint32_t b[4], c[4];
      const uint32_t off = swz512(warp * 8 + (lane & 7), 2 * ks + (lane >> 3));
      ldsm_x4(b, kb + off);
      ldsm_x4(c, vb + off);
      mma_16816(s, qa[ks], b[0], b[1]);
      mma_16816(s, qa[ks + 1], b[2], b[3]);
      mma_16816(dp, da[ks], c[0], c[1]);
      mma_16816(dp, da[ks + 1], c[2], c[3]);
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

    // records of this chunk: nk * 48 contiguous bytes
    {
      const uint4* src = reinterpret_cast<const uint4*>(sRec);
      uint4* dst = reinterpret_cast<uint4*>(pds_row + static_cast<int64_t>(base) * kRec);
      for (int i = tid; i < nk * 3; i += kDqThreads) dst[i] = src[i];
    }
    // dQ[:, 64w:64w+64] += dS K
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      const int mi = lane >> 3;
      ldsm_x4(a, sDSa + (((((mi & 1) << 3) + (lane & 7)) * kDsStride + 16 * ks + ((mi >> 1) << 3)) << 1));
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t b[4];
        ldsm_x4_t(b, kb + swz512(16 * ks + ((mi & 1) << 3) + (lane & 7), warp * 8 + nt + (mi >> 1)));
        mma_16816(acc[nt], a, b[0], b[1]);
        mma_16816(acc[nt + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();
    if (ch + 2 < n_chunks) issue(ch + 2);
    cp_async_commit();
  }
  cp_async_wait<0>();

  __nv_bfloat16* drow = dq + qrow0 * kHeadDim;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int dim = warp * 64 + nt * 8 + 2 * cq;
    *reinterpret_cast<uint32_t*>(drow + gq * kHeadDim + dim) = pack_bf16(acc[nt][0] * scale, acc[nt][1] * scale);
    if (gq + 8 < kHeadsPerGroup)
      *reinterpret_cast<uint32_t*>(drow + (gq + 8) * kHeadDim + dim) =
          pack_bf16(acc[nt][2] * scale, acc[nt][3] * scale);
  }
}

// ---------------------------------------------------------------------------
// dK / dV per key quad
// ---------------------------------------------------------------------------
constexpr int kKvThreads = 128;
constexpr int kUnroll = 4;  // entries in flight per warp

// Loads this thread's slice of one query's 12 head rows for the A operand of
// X^T (dims x heads): rows {2c, 2c+1, 2c+8, 2c+9} (rows >= 12 are zero), dims
// [4g, 4g+4) and [32+4g, 32+4g+4) of the warp's 64-dim slice.
struct RowSlice {
  uint2 x[4], y[4];
};
__device__ __forceinline__ void load_slice(RowSlice& r, const __nv_bfloat16* base, int gq, int cq, bool live) {
  const int rows[4] = {2 * cq, 2 * cq + 1, 2 * cq + 8, 2 * cq + 9};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (live && rows[i] < kHeadsPerGroup) {
      const __nv_bfloat16* p = base + rows[i] * kHeadDim + 4 * gq;
      r.x[i] = __ldg(reinterpret_cast<const uint2*>(p));
      r.y[i] = __ldg(reinterpret_cast<const uint2*>(p + 32));
    } else {
      r.x[i] = make_uint2(0, 0);
      r.y[i] = make_uint2(0, 0);
    }
  }
}
// A fragment of m-tile mt (dims 4g+mt and 32+4g+mt; k = head rows).
__device__ __forceinline__ void slice_frag(uint32_t (&a)[4], const RowSlice& r, int mt) {
  const uint32_t sel = (mt & 1) ? kHiHi : kLoLo;
  const bool hiw = mt >= 2;
  a[0] = prmt(hiw ? r.x[0].y : r.x[0].x, hiw ? r.x[1].y : r.x[1].x, sel);
  a[1] = prmt(hiw ? r.y[0].y : r.y[0].x, hiw ? r.y[1].y : r.y[1].x, sel);
  a[2] = prmt(hiw ? r.x[2].y : r.x[2].x, hiw ? r.x[3].y : r.x[3].x, sel);
  a[3] = prmt(hiw ? r.y[2].y : r.y[2].x, hiw ? r.y[3].y : r.y[3].x, sel);
}

__global__ void __launch_bounds__(kKvThreads)
dkdv_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ q,
            const uint16_t* __restrict__ pds, const int32_t* __restrict__ quad_ptr,
            const int64_t* __restrict__ quad_ent, int64_t T_kv, int G, int n_sel, float scale,
            __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  const int H = G * kHeadsPerGroup;
  const int64_t b = blockIdx.x / G;
  const int g = static_cast<int>(blockIdx.x - b * G);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, cq = lane & 3;
  const int e0 = quad_ptr[b], e1 = quad_ptr[b + 1];

  float ak[4][4], av[4][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) ak[mt][j] = av[mt][j] = 0.f;

  for (int base = e0; base < e1; base += 32) {
    const int64_t my_ent = base + lane < e1 ? quad_ent[base + lane] : -1;
    const int n_here = min(32, e1 - base);
    for (int u0 = 0; u0 < n_here; u0 += kUnroll) {
      RowSlice sq[kUnroll], sd[kUnroll];
      uint32_t pb[kUnroll][2], sb[kUnroll][2];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t ent = __shfl_sync(0xffffffffu, my_ent, (u0 + u) & 31);
        const bool live = u0 + u < n_here;
        const int64_t t = live ? (ent >> 32) : 0;
        const int i0 = static_cast<int>((ent >> 4) & 0x0fffffff);
        const int mask = static_cast<int>(ent & 15);
        const int64_t row0 = (t * H + g * kHeadsPerGroup) * kHeadDim + warp * 64;
        load_slice(sq[u], q + row0, gq, cq, live);
        load_slice(sd[u], dout + row0, gq, cq, live);
        pb[u][0] = pb[u][1] = sb[u][0] = sb[u][1] = 0u;
        if (live && gq < 4 && ((mask >> gq) & 1)) {
          const int idx = i0 + __popc(mask & ((1 << gq) - 1));
          const uint16_t* rec = pds + ((t * G + g) * n_sel + idx) * kRec;
          pb[u][0] = __ldg(reinterpret_cast<const uint32_t*>(rec + 2 * cq));
          sb[u][0] = __ldg(reinterpret_cast<const uint32_t*>(rec + 12 + 2 * cq));
          if (cq < 2) {
            pb[u][1] = __ldg(reinterpret_cast<const uint32_t*>(rec + 8 + 2 * cq));
            sb[u][1] = __ldg(reinterpret_cast<const uint32_t*>(rec + 20 + 2 * cq));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t a[4];
          slice_frag(a, sq[u], mt);
          mma_16816(ak[mt], a, sb[u][0], sb[u][1]);
          slice_frag(a, sd[u], mt);
          mma_16816(av[mt], a, pb[u][0], pb[u][1]);
        }
      }
    }
  }

  // C fragment: (dim 4g+mt | 32+4g+mt, key 2c | 2c+1) of the warp's slice; keys 0..3 valid.
  if (cq < 2) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int64_t key = 4 * b + 2 * cq + j;
      if (key >= T_kv) continue;
      const int64_t off = (key * G + g) * kHeadDim + warp * 64 + 4 * gq;
      uint2 wk, wv;
      wk.x = pack_bf16(ak[0][j] * scale, ak[1][j] * scale);
      wk.y = pack_bf16(ak[2][j] * scale, ak[3][j] * scale);
      wv.x = pack_bf16(av[0][j], av[1][j]);
      wv.y = pack_bf16(av[2][j], av[3][j]);
      *reinterpret_cast<uint2*>(dk + off) = wk;
      *reinterpret_cast<uint2*>(dv + off) = wv;
      wk.x = pack_bf16(ak[0][2 + j] * scale, ak[1][2 + j] * scale);
      wk.y = pack_bf16(ak[2][2 + j] * scale, ak[3][2 + j] * scale);
      wv.x = pack_bf16(av[0][2 + j], av[1][2 + j]);
      wv.y = pack_bf16(av[2][2 + j], av[3][2 + j]);
      *reinterpret_cast<uint2*>(dk + off + 32) = wk;
      *reinterpret_cast<uint2*>(dv + off + 32) = wv;
    }
  }
}

}  // namespace

cudaError_t launch_backward_dq(const void* grad_out, const void* q, const void* k, const void* v,
                               const void* out, const float* lse, const int32_t* row_cnt,
                               const int32_t* row_cols, int64_t T, int G, int n_sel, float scale, void* dq,
                               float* delta, uint16_t* pds, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(kOffCols) + static_cast<size_t>(n_sel) * 4;
  cudaError_t e = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dq_kernel<<<static_cast<unsigned>(T * G), kDqThreads, smem, s>>>(
      static_cast<const __nv_bfloat16*>(grad_out), static_cast<const __nv_bfloat16*>(q),
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
      static_cast<const __nv_bfloat16*>(out), lse, row_cnt, row_cols, G, n_sel, scale, scale * kLog2e,
      static_cast<__nv_bfloat16*>(dq), delta, pds);
  return cudaGetLastError();
}

cudaError_t launch_backward_dkdv(const void* grad_out, const void* q, const uint16_t* pds,
                                 const int32_t* quad_ptr, const int64_t* quad_ent, int64_t T, int64_t T_kv,
                                 int G, int n_sel, float scale, void* dk, void* dv, cudaStream_t s) {
  (void)T;
  const int64_t n_quads = (T_kv + 3) / 4;
  dkdv_kernel<<<static_cast<unsigned>(n_quads * G), kKvThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(grad_out), static_cast<const __nv_bfloat16*>(q), pds, quad_ptr,
      quad_ent, T_kv, G, n_sel, scale, static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv));
  return cudaGetLastError();
}

}  // namespace qsa
