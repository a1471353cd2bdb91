// QSA forward: persistent, four CTAs of two warps per SM (the shape set at the
// launcher below).
//
// Computes, for the 12 query heads of every (query token t, KV group g), the
// softmax attention of the cuDNN-Frontend "Query Sparse Attention (QSA)" page
// ("Selection and components": scaled QK over the selected keys, online softmax,
// PV, FP32 output cast to BF16, natural-log LSE; empty rows give zero output and
// -inf LSE) over the row's de-duplicated route set R_t.
//
// Pipeline (qsa_pipe.cuh): the CTA's items are cut into chunks of 8 keys per
// warp (16 at the launch shape) that flow through a ring of swizzled K / V tiles
// (plus the item's 12 Q rows on its first chunk), gathered with 16-byte
// cp.async copies STAGES - 1 chunks ahead of the compute (one at the launch
// shape).  Rows past the end of R_t are zero-filled, so unselected K/V
// values never reach an output.  Per chunk, warp w forms S = Q K^T for keys
// 8w..8w+7 (mma.sync m16n8k16 BF16, FP32 accumulate, Q fragments held in
// registers for the whole item), P = exp2(S*scale*log2e - m) is written as BF16
// against the running row maximum m, and warp w accumulates
// O[:, DPW w : DPW (w + 1)] += P V (DPW = 256 / warps, 128 at the launch shape).
// m may lag the true maximum by up to 2^8 (P < 256): only a chunk in which some
// score passes m by more than that exchanges the warps' maxima, rescales O and
// the sums and rewrites P, so most chunks take one barrier between S and P V.
// Each lane keeps its part of the row sums; they are combined once per item.
// (seq32k forward: 3.80 ms with a maximum exchange and a sum exchange in every
// chunk, 3.53 ms with the lag.)
#include "qsa_internal.h"
#include "qsa_pipe.cuh"

namespace qsa {
namespace {

// Kernel shape: NW warps per CTA (chunks of KEYS = 8 * NW keys, warp w owns keys
// 8w..8w+7 of S and dims [DPW * w, DPW * (w + 1)) of O), STAGES-deep gather ring
// (gathers run STAGES - 1 chunks ahead), CPS CTAs resident per SM.
template <int NW, int STAGES, int CPS>
struct FwdShape {
  static constexpr int kThreads = NW * 32;
  static constexpr int kKeys = 8 * NW;
  static constexpr int kDpw = kHeadDim / NW;                   // output dims per warp
  static constexpr int kNt = kDpw / 8;                         // n8 tiles of P V per warp
  static constexpr int kKs = kKeys / 16;                       // k16 steps of P V
  static constexpr int kTile = kKeys * 512;                    // one swizzled [KEYS][256] BF16 tile
  static constexpr int kStageBytes = 2 * kTile + kHeadsPerGroup * 512;  // K | V | Q rows
  static constexpr int kPStride = kKeys + 8;                   // bf16 per P row (conflict-free ldmatrix)
  static constexpr int kOffZero = STAGES * kStageBytes;        // 512 zero bytes: Q rows 12..15
  static constexpr int kOffP = kOffZero + 512;
  static constexpr int kOffMax = kOffP + kRowTile * kPStride * 2;
  static constexpr int kOffSum = kOffMax + NW * kRowTile * 4;
  static constexpr int kOffDesc = kOffSum + NW * kRowTile * 4;
  static constexpr int kOffJump = kOffDesc + STAGES * 16;       // one flag per warp
  static constexpr int kSmemBytes = kOffJump + ((NW * 4 + 15) / 16) * 16;
  static_assert(kSmemBytes * CPS + 1024 * CPS <= 233472, "shared memory per SM");
  static_assert(kKs >= 1 && kNt % 2 == 0, "shape");
};
constexpr int kFirst = 1, kLast = 2;
// The running maximum of a row may lag its true maximum by up to kLag (log2
// units): P stays below 2^kLag, and O and the sums are rescaled only when a
// score passes the maximum by more than that.
constexpr float kLag = 8.f;
__device__ __forceinline__ float p_of(float s, float m) { return s == -INFINITY ? 0.f : exp2f(s - m); }

template <int NW, int STAGES, int CPS>
__global__ void __launch_bounds__(NW * 32, CPS)
fwd_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
           const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ row_cnt,
           const int32_t* __restrict__ row_cols, int64_t n_items, int G, int n_sel, float scale_log2,
           __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  using S_ = FwdShape<NW, STAGES, CPS>;
  constexpr int KEYS = S_::kKeys, kTile = S_::kTile, kStageBytes = S_::kStageBytes, kPStride = S_::kPStride;
  constexpr int kNt = S_::kNt, kKs = S_::kKs;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, cq = lane & 3, mi = lane >> 3;
  const int H = G * kHeadsPerGroup;
  int4* desc = reinterpret_cast<int4*>(smem + S_::kOffDesc);
  __nv_bfloat16* sP = reinterpret_cast<__nv_bfloat16*>(smem + S_::kOffP);
  float* sMax = reinterpret_cast<float*>(smem + S_::kOffMax);
  float* sSum = reinterpret_cast<float*>(smem + S_::kOffSum);
  int* sJump = reinterpret_cast<int*>(smem + S_::kOffJump);
  if (tid < 32) reinterpret_cast<uint4*>(smem + S_::kOffZero)[tid] = make_uint4(0, 0, 0, 0);

  Cursor cur;
  cursor_init<KEYS>(cur, row_cnt, n_items, G);
  int32_t key[8];
  cursor_keys<KEYS>(key, cur, n_items, G, row_cols, n_sel);
  // Issues the cursor's chunk into `stage`, records its descriptor, advances.
  auto issue = [&](int stage) {
    const uint32_t st = sbase + stage * kStageBytes;
    if (cur.it < n_items) {
      const int64_t t = cur.t;
      const int g = cur.g;
      const int nk = cursor_nk<KEYS>(cur, n_items);
      if (nk > 0) {
        gather_rows(st, st + kTile, k, v, key, g, G, nk);
        if (cur.ch == 0) gather_heads<NW>(st + 2 * kTile, q + (t * H + g * kHeadsPerGroup) * kHeadDim);
      }
      if (tid == 0)
        desc[stage] = make_int4(static_cast<int>(t), g, nk,
                                (cur.ch == 0 ? kFirst : 0) | (cur.ch == cur.nch - 1 ? kLast : 0));
    } else if (tid == 0) {
      desc[stage] = make_int4(0, 0, -1, 0);  // end of the CTA's sequence
    }
    cp_async_commit();
    cursor_next<KEYS>(cur, row_cnt, n_items, G);
    cursor_keys<KEYS>(key, cur, n_items, G, row_cols, n_sel);
  };
#pragma unroll
  for (int s0 = 0; s0 < STAGES - 1; ++s0) issue(s0);

  uint32_t qa[16][4];
  float o[kNt][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const uint32_t spa = smem_u32(sP);

  for (int c = 0;; ++c) {
    const int stage = c % STAGES;
    const uint32_t st = sbase + stage * kStageBytes;
    cp_async_wait<STAGES - 2>();
    __syncthreads();  // chunk c has landed; every warp is done with chunk c - 1
    const int4 d = desc[stage];
    issue((c + STAGES - 1) % STAGES);
    const int nk = d.z;
    if (nk < 0) break;
    const int64_t qrow0 = static_cast<int64_t>(d.x) * H + d.y * kHeadsPerGroup;
    if (nk == 0) {  // padding query: zero output, -inf LSE
      uint4* orow = reinterpret_cast<uint4*>(out + qrow0 * kHeadDim);
      for (int i = tid; i < kHeadsPerGroup * 32; i += S_::kThreads) orow[i] = make_uint4(0, 0, 0, 0);
      if (tid < kHeadsPerGroup) lse[qrow0 + tid] = -INFINITY;
      continue;
    }
    if (d.w & kFirst) {
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const int r = ((mi & 1) << 3) + (lane & 7);
        const int cc = 2 * ks + (mi >> 1);
        ldsm_x4(qa[ks], r < kHeadsPerGroup ? st + 2 * kTile + swz512(r, cc) : sbase + S_::kOffZero + (cc << 4));
      }
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    }
    // S = Q K^T for this warp's 8 keys, as four independent accumulation chains
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    {
      float sp[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) sp[j][0] = sp[j][1] = sp[j][2] = sp[j][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 16; ks += 2) {
        uint32_t b[4];
        ldsm_x4(b, st + swz512(warp * 8 + (lane & 7), 2 * ks + mi));
        mma_16816(sp[(ks >> 1) & 3], qa[ks], b[0], b[1]);
        mma_16816(sp[(ks >> 1) & 3], qa[ks + 1], b[2], b[3]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) s[i] = (sp[0][i] + sp[1][i]) + (sp[2][i] + sp[3][i]);
    }
    const int key0 = warp * 8 + 2 * cq;
    const bool v0 = key0 < nk, v1 = key0 + 1 < nk;
    s[0] = v0 ? s[0] * scale_log2 : -INFINITY;
    s[1] = v1 ? s[1] * scale_log2 : -INFINITY;
    s[2] = v0 ? s[2] * scale_log2 : -INFINITY;
    s[3] = v1 ? s[3] * scale_log2 : -INFINITY;
    // P against the running maximum as it stands; it is replaced only when a
    // score exceeds it by more than kLag (then every warp rescales together)
    const bool jump = fmaxf(s[0], s[1]) > m0 + kLag || fmaxf(s[2], s[3]) > m1 + kLag;
    const unsigned any_jump = __any_sync(0xffffffffu, jump);
    float p0 = p_of(s[0], m0), p1 = p_of(s[1], m0), p2 = p_of(s[2], m1), p3 = p_of(s[3], m1);
    if (!any_jump) {
      *reinterpret_cast<uint32_t*>(sP + gq * kPStride + key0) = pack_bf16(p0, p1);
      *reinterpret_cast<uint32_t*>(sP + (gq + 8) * kPStride + key0) = pack_bf16(p2, p3);
    }
    float x0 = fmaxf(s[0], s[1]), x1 = fmaxf(s[2], s[3]);
    x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
    x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
    x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
    x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
    if (cq == 0) {
      sMax[warp * kRowTile + gq] = x0;
      sMax[warp * kRowTile + gq + 8] = x1;
    }
    if (lane == 0) sJump[warp] = any_jump ? 1 : 0;
    __syncthreads();
    bool rescale = false;
#pragma unroll
    for (int w = 0; w < NW; ++w) rescale |= sJump[w] != 0;
    if (rescale) {  // CTA-uniform
      float n0 = m0, n1 = m1;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        n0 = fmaxf(n0, sMax[w * kRowTile + gq]);
        n1 = fmaxf(n1, sMax[w * kRowTile + gq + 8]);
      }
      const float a0 = n0 == -INFINITY ? 1.f : exp2f(m0 - n0), a1 = n1 == -INFINITY ? 1.f : exp2f(m1 - n1);
      m0 = n0;
      m1 = n1;
      l0 *= a0;
      l1 *= a1;
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) {
        o[nt][0] *= a0;
        o[nt][1] *= a0;
        o[nt][2] *= a1;
        o[nt][3] *= a1;
      }
      p0 = p_of(s[0], m0);
      p1 = p_of(s[1], m0);
      p2 = p_of(s[2], m1);
      p3 = p_of(s[3], m1);
      *reinterpret_cast<uint32_t*>(sP + gq * kPStride + key0) = pack_bf16(p0, p1);
      *reinterpret_cast<uint32_t*>(sP + (gq + 8) * kPStride + key0) = pack_bf16(p2, p3);
      __syncthreads();
    }
    l0 += p0 + p1;  // this lane's part of the row sums
    l1 += p2 + p3;
    // O[:, DPW*w : DPW*(w+1)] += P V over the chunk's keys
#pragma unroll
    for (int ks = 0; ks < kKs; ++ks) {
      uint32_t pa[4];
      ldsm_x4(pa, spa + (((((mi & 1) << 3) + (lane & 7)) * kPStride + 16 * ks + ((mi >> 1) << 3)) << 1));
#pragma unroll
      for (int nt = 0; nt < kNt; nt += 2) {
        uint32_t b[4];
        ldsm_x4_t(b, st + kTile + swz512(16 * ks + ((mi & 1) << 3) + (lane & 7), warp * kNt + nt + (mi >> 1)));
        mma_16816(o[nt], pa, b[0], b[1]);
        mma_16816(o[nt + 1], pa, b[2], b[3]);
      }
    }
    if (d.w & kLast) {  // CTA-uniform
      float c0 = l0, c1 = l1;
      c0 += __shfl_xor_sync(0xffffffffu, c0, 1);
      c0 += __shfl_xor_sync(0xffffffffu, c0, 2);
      c1 += __shfl_xor_sync(0xffffffffu, c1, 1);
      c1 += __shfl_xor_sync(0xffffffffu, c1, 2);
      if (cq == 0) {
        sSum[warp * kRowTile + gq] = c0;
        sSum[warp * kRowTile + gq + 8] = c1;
      }
      __syncthreads();
      float t0 = 0.f, t1 = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        t0 += sSum[w * kRowTile + gq];
        t1 += sSum[w * kRowTile + gq + 8];
      }
      const float i0 = 1.f / t0, i1 = 1.f / t1;
      __nv_bfloat16* orow = out + qrow0 * kHeadDim;
#pragma unroll
      for (int nt = 0; nt < kNt; ++nt) {
        const int dim = warp * S_::kDpw + nt * 8 + 2 * cq;
        *reinterpret_cast<uint32_t*>(orow + gq * kHeadDim + dim) = pack_bf16(o[nt][0] * i0, o[nt][1] * i0);
        if (gq + 8 < kHeadsPerGroup)
          *reinterpret_cast<uint32_t*>(orow + (gq + 8) * kHeadDim + dim) = pack_bf16(o[nt][2] * i1, o[nt][3] * i1);
      }
      if (warp == 0 && cq == 0) {
        lse[qrow0 + gq] = (m0 + log2f(t0)) * kLn2;
        if (gq + 8 < kHeadsPerGroup) lse[qrow0 + gq + 8] = (m1 + log2f(t1)) * kLn2;
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace

int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Forward kernel shape used by launch_forward: 4 CTAs of 2 warps per SM, 16-key
// chunks, 2-stage ring (more independent items per SM beat wider CTAs: at 8 warps
// per SM, 4 x 2 ran the seq32k forward in 4.7 ms, 2 x 4 in 4.9 ms, 1 x 8 in 6.5 ms).
constexpr int kFwdWarps = 2, kFwdStages = 2, kFwdCtasPerSm = 4;

cudaError_t launch_forward(const void* q, const void* k, const void* v, const int32_t* row_cnt,
                           const int32_t* row_cols, int64_t T, int G, int n_sel, float scale, void* out,
                           float* lse, int* status, cudaStream_t s) {
  (void)status;  // the forward has no wait that can expire: nothing to report
  using S_ = FwdShape<kFwdWarps, kFwdStages, kFwdCtasPerSm>;
  auto kern = fwd_kernel<kFwdWarps, kFwdStages, kFwdCtasPerSm>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S_::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t n_items = T * G;
  const int64_t slots = static_cast<int64_t>(kFwdCtasPerSm) * sm_count();
  const int64_t grid = n_items < slots ? n_items : slots;
  kern<<<static_cast<unsigned>(grid), S_::kThreads, S_::kSmemBytes, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), row_cnt, row_cols, n_items, G, n_sel, scale * kLog2e,
      static_cast<__nv_bfloat16*>(out), lse);
  return cudaGetLastError();
}

}  // namespace qsa
