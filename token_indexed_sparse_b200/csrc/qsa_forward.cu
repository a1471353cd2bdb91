// QSA forward: one CTA per (query token t, KV group g).
//
// Computes, for the 12 query heads of group g, the softmax attention of
// "Query Sparse Attention (QSA)" (cuDNN-Frontend page, "Selection and
// components": scaled QK over the selected keys, online softmax, PV, FP32
// output cast to BF16, natural-log LSE; empty rows give zero output and -inf
// LSE) over the row's de-duplicated route set R_t.
//
// Data flow per CTA (4 warps):
//   * R_t (ascending) is staged in shared memory; Q's 12 rows (padded to the
//     16-row MMA tile with zeros) are loaded once into A fragments.
//   * K and V rows of R_t are gathered in chunks of 32 keys with 16-byte
//     cp.async copies into a double-buffered, XOR-swizzled shared tile; rows past
//     the end of R_t are zero-filled, so unselected K/V values are never read.
//   * Per chunk: warp w forms S = Q K^T for keys 8w..8w+7 (mma.sync bf16,
//     fp32 accumulate), the chunk row maximum is combined across warps through
//     shared memory, P = exp2(S*scale*log2e - m) is written as BF16, and warp w
//     accumulates O[:, 64w:64w+64] += P V with running-max rescaling.
#include "qsa_device.cuh"
#include "qsa_internal.h"

namespace qsa {
namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 32;       // keys per pipeline stage
constexpr int kPStride = 40;     // bf16 per row of the P tile (80 B: conflict-free ldmatrix)
constexpr int kTileBytes = kChunk * 512;
constexpr int kOffK = 16 * 512;                 // after the Q tile
constexpr int kOffV = kOffK + 2 * kTileBytes;
constexpr int kOffP = kOffV + 2 * kTileBytes;
constexpr int kOffMax = kOffP + kRowTile * kPStride * 2;
constexpr int kOffSum = kOffMax + 4 * kRowTile * 4;
constexpr int kOffCols = kOffSum + 4 * kRowTile * 4;

__global__ void __launch_bounds__(kThreads, 2)
fwd_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
           const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ row_cnt,
           const int32_t* __restrict__ row_cols, int G, int n_sel, float scale_log2,
           __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sP = reinterpret_cast<__nv_bfloat16*>(smem + kOffP);
  float* sMax = reinterpret_cast<float*>(smem + kOffMax);
  float* sSum = reinterpret_cast<float*>(smem + kOffSum);
  int32_t* sCols = reinterpret_cast<int32_t*>(smem + kOffCols);

  const int H = G * kHeadsPerGroup;
  const int64_t t = blockIdx.x / G;
  const int g = static_cast<int>(blockIdx.x - t * G);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, cq = lane & 3;
  const int cnt = row_cnt[t];
  const int64_t qrow0 = t * H + g * kHeadsPerGroup;  // first of the group's 12 query-head rows

  if (cnt == 0) {  // padding query: zero output, -inf LSE
    uint4* o = reinterpret_cast<uint4*>(out + qrow0 * kHeadDim);
    for (int i = tid; i < kHeadsPerGroup * 32; i += kThreads) o[i] = make_uint4(0, 0, 0, 0);
    if (tid < kHeadsPerGroup) lse[qrow0 + tid] = -INFINITY;
    return;
  }

  for (int i = tid; i < cnt; i += kThreads) sCols[i] = row_cols[t * n_sel + i];
  const uint32_t sQa = smem_u32(smem), sKa = smem_u32(smem + kOffK), sVa = smem_u32(smem + kOffV);
  for (int i = tid; i < kRowTile * 32; i += kThreads) {
    const int r = i >> 5, c = i & 31;
    const bool ok = r < kHeadsPerGroup;
    cp_async16(sQa + swz512(r, c), q + (qrow0 + (ok ? r : 0)) * kHeadDim + c * 8, ok);
  }
  cp_async_commit();
  __syncthreads();  // sCols visible to every issuing thread

  const int n_chunks = (cnt + kChunk - 1) / kChunk;
  auto issue = [&](int ch) {
    const int stage = ch & 1, base = ch * kChunk;
    const int nk = min(kChunk, cnt - base);
#pragma unroll 4
    for (int i = tid; i < 2 * kChunk * 32; i += kThreads) {
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
  cp_async_wait<2>();  // the Q tile has landed
  __syncthreads();

  uint32_t qa[16][4];
#pragma unroll
  for (int ks = 0; ks < 16; ++ks) {
    const int mi = lane >> 3;
    ldsm_x4(qa[ks], sQa + swz512(((mi & 1) << 3) + (lane & 7), 2 * ks + (mi >> 1)));
  }

  float o[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running max, rows gq and gq+8 (log2 domain)
  float l0 = 0.f, l1 = 0.f;              // running sum of exp2(s - m)
  const uint32_t sPa = smem_u32(sP);

  for (int ch = 0; ch < n_chunks; ++ch) {
    const int stage = ch & 1;
    const int nk = min(kChunk, cnt - ch * kChunk);
    cp_async_wait<1>();
    __syncthreads();

    // S = Q K^T for this warp's 8 keys.
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t kb = sKa + stage * kTileBytes;
#pragma unroll
    for (int ks = 0; ks < 16; ks += 2) {
      uint32_t b[4];
      ldsm_x4(b, kb + swz512(warp * 8 + (lane & 7), 2 * ks + (lane >> 3)));
      mma_16816(s, qa[ks], b[0], b[1]);
      mma_16816(s, qa[ks + 1], b[2], b[3]);
    }
    const int key0 = warp * 8 + 2 * cq;
    const bool v0 = key0 < nk, v1 = key0 + 1 < nk;
    s[0] = v0 ? s[0] * scale_log2 : -INFINITY;
    s[1] = v1 ? s[1] * scale_log2 : -INFINITY;
    s[2] = v0 ? s[2] * scale_log2 : -INFINITY;
    s[3] = v1 ? s[3] * scale_log2 : -INFINITY;
    float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]);
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    if (cq == 0) {
      sMax[warp * kRowTile + gq] = mx0;
      sMax[warp * kRowTile + gq + 8] = mx1;
    }
    __syncthreads();
    float n0 = m0, n1 = m1;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      n0 = fmaxf(n0, sMax[w * kRowTile + gq]);
      n1 = fmaxf(n1, sMax[w * kRowTile + gq + 8]);
    }
    const float p0 = exp2f(s[0] - n0), p1 = exp2f(s[1] - n0);
    const float p2 = exp2f(s[2] - n1), p3 = exp2f(s[3] - n1);
    *reinterpret_cast<uint32_t*>(sP + gq * kPStride + key0) = pack_bf16(p0, p1);
    *reinterpret_cast<uint32_t*>(sP + (gq + 8) * kPStride + key0) = pack_bf16(p2, p3);
    float ps0 = p0 + p1, ps1 = p2 + p3;
    ps0 += __shfl_xor_sync(0xffffffffu, ps0, 1);
    ps0 += __shfl_xor_sync(0xffffffffu, ps0, 2);
    ps1 += __shfl_xor_sync(0xffffffffu, ps1, 1);
    ps1 += __shfl_xor_sync(0xffffffffu, ps1, 2);
    if (cq == 0) {
      sSum[warp * kRowTile + gq] = ps0;
      sSum[warp * kRowTile + gq + 8] = ps1;
    }
    const float a0 = exp2f(m0 - n0), a1 = exp2f(m1 - n1);
    m0 = n0;
    m1 = n1;
    __syncthreads();
    float cs0 = 0.f, cs1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      cs0 += sSum[w * kRowTile + gq];
      cs1 += sSum[w * kRowTile + gq + 8];
    }
    l0 = l0 * a0 + cs0;
    l1 = l1 * a1 + cs1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      o[nt][0] *= a0;
      o[nt][1] *= a0;
      o[nt][2] *= a1;
      o[nt][3] *= a1;
    }

    // O[:, 64w:64w+64] += P V
    const uint32_t vb = sVa + stage * kTileBytes;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t pa[4];
      const int mi = lane >> 3;
      ldsm_x4(pa, sPa + (((((mi & 1) << 3) + (lane & 7)) * kPStride + 16 * ks + ((mi >> 1) << 3)) << 1));
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t b[4];
        ldsm_x4_t(b, vb + swz512(16 * ks + ((mi & 1) << 3) + (lane & 7), warp * 8 + nt + (mi >> 1)));
        mma_16816(o[nt], pa, b[0], b[1]);
        mma_16816(o[nt + 1], pa, b[2], b[3]);
      }
    }
    __syncthreads();  // every warp is done with this stage
    if (ch + 2 < n_chunks) issue(ch + 2);
    cp_async_commit();
  }
  cp_async_wait<0>();

  const float i0 = 1.f / l0, i1 = 1.f / l1;
  __nv_bfloat16* orow = out + qrow0 * kHeadDim;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int dim = warp * 64 + nt * 8 + 2 * cq;
    *reinterpret_cast<uint32_t*>(orow + gq * kHeadDim + dim) = pack_bf16(o[nt][0] * i0, o[nt][1] * i0);
    if (gq + 8 < kHeadsPerGroup)
      *reinterpret_cast<uint32_t*>(orow + (gq + 8) * kHeadDim + dim) = pack_bf16(o[nt][2] * i1, o[nt][3] * i1);
  }
  if (warp == 0 && cq == 0) {
    lse[qrow0 + gq] = (m0 + log2f(l0)) * kLn2;
    if (gq + 8 < kHeadsPerGroup) lse[qrow0 + gq + 8] = (m1 + log2f(l1)) * kLn2;
  }
}

}  // namespace

cudaError_t launch_forward(const void* q, const void* k, const void* v, const int32_t* row_cnt,
                           const int32_t* row_cols, int64_t T, int G, int n_sel, float scale, void* out,
                           float* lse, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(kOffCols) + static_cast<size_t>(n_sel) * 4;
  cudaError_t e = cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  fwd_kernel<<<static_cast<unsigned>(T * G), kThreads, smem, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), row_cnt, row_cols, G, n_sel, scale * kLog2e,
      static_cast<__nv_bfloat16*>(out), lse);
  return cudaGetLastError();
}

}  // namespace qsa
