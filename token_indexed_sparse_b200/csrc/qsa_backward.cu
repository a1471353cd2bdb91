// QSA backward, following the backward equations of the cuDNN-Frontend
// "Query Sparse Attention (QSA)" page ("Selection and components"), per query
// head h and its KV head g:
//   S = scale Q K^T,  P = exp(S - lse) (zero outside R_t),
//   delta = rowsum(dO * out),  dP = dO V^T,  dS = P * (dP - delta),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO  (dK/dV summed over heads).
//
// Two kernels, neither using floating-point atomics:
//   * dq_kernel, persistent over (query t, group g) items: recomputes S and dP
//     over R_t (K/V rows gathered like the forward), forms P and dS with delta
//     from the route kernel, accumulates dQ, and stores the BF16 P / dS of every
//     routed pair (`pds`, one 48-byte record [P h0..h11 | dS h0..h11] per
//     (t, g, position in R_t)).
//   * dkdv_kernel, persistent over (aligned key quad, group g, query-phase range)
//     work items: walks the quad's query list in ascending query order, stages
//     each entry's Q / dO rows and P / dS records in shared memory and
//     accumulates dK^T = Q^T dS and dV^T = dO^T P on tensor cores; the fixed list
//     order makes dK/dV bitwise reproducible.
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
// BF16 P / dS records and accumulates dQ[:, DPW*w : DPW*(w+1)] += dS K.
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
          __nv_bfloat16* __restrict__ dq, uint16_t* __restrict__ pds) {
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
    if (d.w & kFirst) {
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
    __syncthreads();  // every warp has read this item's buffer: its slot may be refilled
    issue((c + STAGES - 1) % STAGES);

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

// ---------------------------------------------------------------------------
// dK / dV per key quad, one query phase per launch
// ---------------------------------------------------------------------------
// Work item = (quad b, group g, entries [lo, hi) of b's ascending query list that
// fall in the launch's query phase).  Items are dealt round-robin to persistent
// CTAs (8 warps); each item's entries flow in chunks of 4 through a 4-stage ring:
// all 12 Q rows and 12 dO rows of each entry (whole 512-byte rows, cp.async,
// swizzled) and the entry's P/dS records placed by key slot (absent keys and
// missing entries zero-filled).  Warp w owns dims [32w, 32w+32) and accumulates
// dK^T += Q^T dS and dV^T += dO^T P with mma.sync: the A fragments come from
// ldmatrix.trans of the staged rows and the K dimension packs head rows of
// different entries of the same quad: k-step 0 = heads 0..7 of entries 0 and 1,
// k-step 1 = the same for entries 2 and 3, k-step 2 = heads 8..11 of all four,
// so no MMA slot or shared-memory read is spent on padding heads.  An item
// starts from zero or from the FP32 partial of the previous phase and ends with
// a partial or, on its last range, the BF16 result: the summation order is the
// fixed list order, so dK/dV are bitwise reproducible.
constexpr int kKvThreads = 256;
constexpr int kKvStages = 2;
constexpr int kKvCtasPerSm = 2;
constexpr int kEnt = 4;                                   // entries per chunk
constexpr int kKvRows = kEnt * 2 * kHeadsPerGroup;        // 96 staged rows per chunk
constexpr int kKvRecOff = kKvRows * 512;                  // records after the rows
constexpr int kKvRecBytes = kEnt * 4 * kRec * 2;          // 4 entries x 4 key slots x 48 B
constexpr int kKvStageBytes = kKvRecOff + kKvRecBytes;
constexpr int kKvOffDesc = kKvStages * kKvStageBytes;
constexpr int kKvSmem = kKvOffDesc + kKvStages * 16;
static_assert(kKvSmem <= 232448, "shared memory per block");
static_assert(kKvStageBytes % 128 == 0, "alignment");
constexpr int kItemFirst = 1, kItemLast = 2, kChFirst = 4, kChLast = 8;

// Byte offset of 16-byte column c of stage row r, which belongs to entry u: the
// 512-byte-row XOR swizzle with the phase of odd entries shifted by 4.
__device__ __forceinline__ uint32_t swz_ent(int u, int r, int c) {
  return static_cast<uint32_t>(r) * 512u + (static_cast<uint32_t>(c ^ ((r & 7) ^ ((u & 1) << 2))) << 4);
}

struct KvCursor {
  int64_t w;        // work index (item = w / G, g = w % G); >= n_work when exhausted
  int64_t wi;       // w / G, kept incrementally (no division in the loop)
  int wg;           // w % G
  int dt, dg;       // gridDim.x / G and gridDim.x % G
  int4 item;        // (quad, lo, hi, flags) of the current work index
  int4 item_next;   // of the next one (prefetched)
  int ch, nch;
};

// Work-list item one grid stride after the cursor's, or zeros past the end.
__device__ __forceinline__ int4 kv_item_next(const KvCursor& c, const int4* wl, int64_t n_work, int G) {
  const int64_t wi_next = c.wi + c.dt + (c.wg + c.dg >= G ? 1 : 0);
  return c.w + gridDim.x < n_work ? __ldg(wl + wi_next) : make_int4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(kKvThreads, kKvCtasPerSm)
dkdv_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ q,
            const uint16_t* __restrict__ pds, const int64_t* __restrict__ quad_ent,
            const int32_t* __restrict__ wl_cnt, const int4* __restrict__ wl, int64_t T_kv, int G, int n_sel,
            float scale, float* __restrict__ partial, void* __restrict__ dk_out, void* __restrict__ dv_out,
            bool f32_out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, cq = lane & 3, mat = lane >> 3, rr = lane & 7;
  const int H = G * kHeadsPerGroup;
  int4* desc = reinterpret_cast<int4*>(smem + kKvOffDesc);
  const int64_t n_work = static_cast<int64_t>(__ldg(wl_cnt)) * G;

  KvCursor cur;
  cur.w = blockIdx.x;
  cur.wi = static_cast<int>(blockIdx.x) / G;
  cur.wg = static_cast<int>(blockIdx.x) % G;
  cur.dt = static_cast<int>(gridDim.x) / G;
  cur.dg = static_cast<int>(gridDim.x) % G;
  cur.item = cur.w < n_work ? __ldg(wl + cur.wi) : make_int4(0, 0, 0, 0);
  cur.item_next = kv_item_next(cur, wl, n_work, G);
  cur.ch = 0;
  cur.nch = (cur.item.z - cur.item.y + kEnt - 1) / kEnt;
  // Warp w copies the 12 rows (one contiguous 6 KB block) of entry w / 2,
  // tensor w % 2, to rows u * 24 + tn * 12 + h of the stage; warps 0, 2, 4, 6
  // also copy their entry's P/dS records.  Each warp loads only its own entry.
  const int u_w = warp >> 1, tn_w = warp & 1;
  const uint32_t row_off = static_cast<uint32_t>(u_w * 24 + tn_w * kHeadsPerGroup) * 512;
  // Stage rows use the 512-byte-row swizzle with the phase of odd entries
  // shifted by 4 (swz_ent): the k-step that packs heads 8..11 of entries 2j and
  // 2j + 1 then reads eight distinct 16-byte bank groups.  For row
  // u*24 + tn*12 + h the phase is (h & 7) ^ 4 (tn ^ (u & 1)).
  const uint32_t xl4 = static_cast<uint32_t>(lane ^ ((tn_w ^ (u_w & 1)) << 2)) << 4;
  int64_t ent = -1;
  auto load_ent = [&]() {
    const int e = cur.item.y + cur.ch * kEnt + u_w;
    ent = (cur.w < n_work && e < cur.item.z) ? __ldg(quad_ent + e) : -1;
  };
  load_ent();

  auto issue = [&](int stage) {
    const uint32_t st = sbase + stage * kKvStageBytes;
    if (cur.w < n_work) {
      const int g = cur.wg;
      const int n_ent = min(kEnt, cur.item.z - (cur.item.y + cur.ch * kEnt));
      const bool live_u = u_w < n_ent;
      const int64_t t = live_u ? (ent >> 32) : 0;
      {
        const __nv_bfloat16* src = (tn_w ? dout : q) + ((t * H + g * kHeadsPerGroup) * kHeadDim + lane * 8);
        const uint32_t dst = st + row_off;
#pragma unroll
        for (int h = 0; h < kHeadsPerGroup; ++h)
          cp_async16(dst + h * 512 + (xl4 ^ ((h & 7) << 4)), src + h * kHeadDim, live_u);
      }
      // records: lanes 0..11 of the tensor-0 warp of entry u copy (key slot, 16-byte part)
      if (tn_w == 0 && lane < 12) {
        const int slot = lane / 3, part = lane - 3 * slot;
        const int mask = static_cast<int>(ent & 15);
        const bool live = live_u && ((mask >> slot) & 1);
        const int i0 = static_cast<int>((ent >> 4) & 0x0fffffff);
        const int idx = live ? i0 + __popc(mask & ((1 << slot) - 1)) : 0;
        const uint16_t* src = pds + (((live ? t : 0) * G + g) * n_sel + idx) * kRec + part * 8;
        cp_async16(st + kKvRecOff + (u_w * 4 + slot) * (kRec * 2) + part * 16, src, live);
      }
      if (tid == 0) {
        const int fl = (cur.item.w & 3) | (cur.ch == 0 ? kChFirst : 0) | (cur.ch == cur.nch - 1 ? kChLast : 0);
        desc[stage] = make_int4(cur.item.x, g, n_ent, fl);
      }
    } else if (tid == 0) {
      desc[stage] = make_int4(0, 0, -1, 0);
    }
    cp_async_commit();
    // advance
    if (cur.w < n_work && ++cur.ch == cur.nch) {
      cur.w += gridDim.x;
      cur.wi += cur.dt;
      cur.wg += cur.dg;
      if (cur.wg >= G) {
        cur.wg -= G;
        ++cur.wi;
      }
      cur.item = cur.item_next;
      cur.item_next = kv_item_next(cur, wl, n_work, G);
      cur.ch = 0;
      cur.nch = (cur.item.z - cur.item.y + kEnt - 1) / kEnt;
    }
    load_ent();
  };
  for (int s0 = 0; s0 < kKvStages - 1; ++s0) issue(s0);

  float ak[2][4], av[2][4];
  for (int c = 0;; ++c) {
    const int stage = c % kKvStages;
    const uint32_t st = sbase + stage * kKvStageBytes;
    cp_async_wait<kKvStages - 2>();
    __syncthreads();  // chunk c has landed; every warp is done with chunk c - 1
    const int4 d = desc[stage];
    issue((c + kKvStages - 1) % kKvStages);
    if (d.z < 0) break;
    const int64_t b = d.x;
    const int g = d.y;
    const int fl = d.w;
    float* part = partial + ((b * G + g) * 128 + warp * 16 + gq * 2 + (cq & 1)) * 16;
    if (fl & kChFirst) {
      if ((fl & kItemFirst) || cq >= 2) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) ak[mt][i] = av[mt][i] = 0.f;
      } else {
        const float4* src = reinterpret_cast<const float4*>(part);
        const float4 x0 = src[0], x1 = src[1], x2 = src[2], x3 = src[3];
        ak[0][0] = x0.x; ak[0][1] = x0.y; ak[0][2] = x0.z; ak[0][3] = x0.w;
        ak[1][0] = x1.x; ak[1][1] = x1.y; ak[1][2] = x1.z; ak[1][3] = x1.w;
        av[0][0] = x2.x; av[0][1] = x2.y; av[0][2] = x2.z; av[0][3] = x2.w;
        av[1][0] = x3.x; av[1][1] = x3.y; av[1][2] = x3.z; av[1][3] = x3.w;
      }
    }
#pragma unroll
    for (int ks = 0; ks < 3; ++ks) {
      // B fragments: P (dV) and dS (dK) of key slot gq for the k-step's head slots
      uint32_t pb0 = 0, pb1 = 0, sb0 = 0, sb1 = 0;
      if (gq < 4) {
        int u0, u1, wp;
        if (ks < 2) {
          u0 = 2 * ks;
          u1 = 2 * ks + 1;
          wp = cq;
        } else {
          u0 = cq >> 1;
          u1 = 2 + (cq >> 1);
          wp = 4 + (cq & 1);
        }
        const uint32_t r0 = st + kKvRecOff + (u0 * 4 + gq) * (kRec * 2);
        const uint32_t r1 = st + kKvRecOff + (u1 * 4 + gq) * (kRec * 2);
        asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(pb0) : "r"(r0 + wp * 4));
        asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(pb1) : "r"(r1 + wp * 4));
        asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(sb0) : "r"(r0 + (6 + wp) * 4));
        asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(sb1) : "r"(r1 + (6 + wp) * 4));
      }
      // A fragments: this lane addresses row (entry, head) of matrix `mat`
      int u, h;
      if (ks < 2) {
        u = 2 * ks + (mat >> 1);
        h = rr;
      } else {
        u = 2 * (mat >> 1) + (rr >> 2);
        h = 8 + (rr & 3);
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int dch = warp * 4 + mt * 2 + (mat & 1);
        uint32_t aq[4], ad[4];
        ldsm_x4_t(aq, st + swz_ent(u, u * 24 + h, dch));
        ldsm_x4_t(ad, st + swz_ent(u, u * 24 + kHeadsPerGroup + h, dch));
        mma_16816(ak[mt], aq, sb0, sb1);
        mma_16816(av[mt], ad, pb0, pb1);
      }
    }
    if ((fl & kChLast) && cq < 2) {
      if (fl & kItemLast) {
        // C fragment of m-tile mt: (dim 32w+16mt+g | +8, key 2c | 2c+1)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int64_t key = 4 * b + 2 * cq + j;
          if (key < T_kv) {
            const int64_t o = (key * G + g) * kHeadDim + warp * 32 + gq;
            if (f32_out) {  // FP32 sums for callers that add partials before rounding
              float* rk = static_cast<float*>(dk_out) + o;
              float* rv = static_cast<float*>(dv_out) + o;
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) {
                rk[16 * mt] = ak[mt][j] * scale;
                rk[16 * mt + 8] = ak[mt][2 + j] * scale;
                rv[16 * mt] = av[mt][j];
                rv[16 * mt + 8] = av[mt][2 + j];
              }
            } else {
              __nv_bfloat16* rk = static_cast<__nv_bfloat16*>(dk_out) + o;
              __nv_bfloat16* rv = static_cast<__nv_bfloat16*>(dv_out) + o;
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) {
                rk[16 * mt] = __float2bfloat16_rn(ak[mt][j] * scale);
                rk[16 * mt + 8] = __float2bfloat16_rn(ak[mt][2 + j] * scale);
                rv[16 * mt] = __float2bfloat16_rn(av[mt][j]);
                rv[16 * mt + 8] = __float2bfloat16_rn(av[mt][2 + j]);
              }
            }
          }
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(part);
        dst[0] = make_float4(ak[0][0], ak[0][1], ak[0][2], ak[0][3]);
        dst[1] = make_float4(ak[1][0], ak[1][1], ak[1][2], ak[1][3]);
        dst[2] = make_float4(av[0][0], av[0][1], av[0][2], av[0][3]);
        dst[3] = make_float4(av[1][0], av[1][1], av[1][2], av[1][3]);
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
                               uint16_t* pds, cudaStream_t s) {
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
      n_items, G, n_sel, scale, scale * kLog2e, static_cast<__nv_bfloat16*>(dq), pds);
  return cudaGetLastError();
}

cudaError_t launch_backward_dkdv(const void* grad_out, const void* q, const uint16_t* pds, const int64_t* quad_ent,
                                 const int32_t* wl_cnt, const int4* wl, int p, int64_t n_quads, int64_t T_kv,
                                 int G, int n_sel, float scale, float* partial, void* dk, void* dv,
                                 bool f32_out, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem);
  if (e != cudaSuccess) return e;
  dkdv_kernel<<<static_cast<unsigned>(kKvCtasPerSm * sm_count()), kKvThreads, kKvSmem, s>>>(
      static_cast<const __nv_bfloat16*>(grad_out), static_cast<const __nv_bfloat16*>(q), pds, quad_ent, wl_cnt + p,
      wl + static_cast<int64_t>(p) * n_quads, T_kv, G, n_sel, scale, partial, dk, dv, f32_out);
  return cudaGetLastError();
}

}  // namespace qsa
