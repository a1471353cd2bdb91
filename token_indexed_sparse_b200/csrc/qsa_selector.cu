// QSA block selector: scores, ratio-causal top-k and expansion to token routes.
//
// cuDNN-Frontend "Query Sparse Attention (QSA)", "Finding QSA attention and its
// indexer": each complete compressed block is scored as
// scale * sum_h relu(qi[t, h] . kbar[block]) (compression ratio four, constant
// head weights); a ratio-causal top-k keeps the best blocks, returned as local
// block IDs, which are expanded to the attention input format with the
// incomplete causal tail and the packed sequence's token origin ("cudnn_qsa"
// page, _pack_indices: four-slot groups hold one complete block or the tail).
//
// Query t sits at key position pos[t] of a sequence starting at token
// tok_base[t] and compressed block blk_base[t]; its own block is
// o = (pos - tok_base) / 4 and its candidates are the local blocks c < o
// (global block blk_base + c).
//
// selector_scores_kernel (tcgen05): one CTA per tile of Q = 256 / Hi queries,
// i.e. 256 (query, head) rows of qi.  It loops over 128-block tiles of kbar
// covering the tile's candidates:  D[128 blocks][256 rows] = kbar_tile .
// qi_tile^T with K = Di = 128, BF16 operands staged by TMA in 128B-swizzled
// shared memory (K-major; kbar tiles up to four ahead, a stage refilled as soon
// as the MMA that read it has completed), FP32 accumulators in tensor memory,
// double-buffered so that the MMA of block tile i + 1 runs under the epilogue
// of tile i.  The
// epilogue thread of TMEM lane r (block g0 + r) reads its 256 columns, sums
// relu over each query's Hi heads and writes the scaled score.
//
// selector_topk_kernel: one CTA per query; radix select on the score bits
// (scores are >= 0, so their bit patterns order like the values) finds the
// k-th largest value; blocks above it and the lowest-ID blocks equal to it
// are kept, written ascending, and expanded to routes.
#include <cuda.h>

#include "qsa_internal.h"
#include "qsa_device.cuh"

namespace qsa {
namespace {

constexpr int kSelDi = 128;        // indexer dims (K of the MMA)
constexpr int kSelRows = 256;      // (query, head) rows per CTA: the MMA N
constexpr int kSelBlk = 128;       // compressed blocks per tile: the MMA M
constexpr int kSelThreads = 128;   // 4 warps: one TMEM lane quarter each
constexpr int kQiBytes = kSelRows * kSelDi * 2;   // 64 KB: two [256][64] SW128 K-blocks
constexpr int kKbBytes = kSelBlk * kSelDi * 2;    // 32 KB: two [128][64] SW128 K-blocks
constexpr int kSelKbStages = 4;                   // kbar tiles loaded ahead of their MMA
constexpr int kSelOffKb = kQiBytes;
constexpr int kSelOffBar = kSelOffKb + kSelKbStages * kKbBytes;
// barriers: qi, kSelKbStages kbar stages, 2 accumulators; then the TMEM address
constexpr int kSelBarQ = 0, kSelBarK0 = 8, kSelBarM0 = kSelBarK0 + 8 * kSelKbStages, kSelTmemSlot = kSelBarM0 + 16;
constexpr int kSelSmem = kSelOffBar + kSelTmemSlot + 8 + 1024;  // + 1 KB alignment slack
static_assert(kSelSmem <= 232448, "shared memory per block");
constexpr uint32_t kSelSpin = 1u << 24;

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
// Bounded wait on phase `parity`; returns false if the wait gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  uint32_t done = 0;
  for (uint32_t it = 0; it < kSelSpin && !done; ++it)
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(done) : "r"(bar), "r"(parity) : "memory");
  return done != 0;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle
// layout (8-row x 128-byte atoms, 1024 bytes apart), sm_100 descriptor version.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3fff);          // start address
  d |= static_cast<uint64_t>(1) << 16;                       // leading byte offset (unused for swizzled K-major)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride byte offset: next 8-row group
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                       // layout: 128-byte swizzle
  return d;
}
// Instruction descriptor, kind::f16: FP32 accumulate, BF16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kSelIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kSelRows >> 3) << 17) |
                               (static_cast<uint32_t>(kSelBlk >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kSelIdesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ int own_block(const int32_t* pos, const int32_t* tok_base, int64_t t) {
  const int64_t p = pos ? __ldg(pos + t) : t;
  const int64_t tb = tok_base ? __ldg(tok_base + t) : 0;
  return p >= tb ? static_cast<int>((p - tb) >> 2) : 0;
}
// Candidates of query t: local blocks [0, n) with n = min(own block, NB - blk_base).
__device__ __forceinline__ int n_cand(const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base,
                                      int64_t t, int64_t NB) {
  const int64_t bb = blk_base ? __ldg(blk_base + t) : 0;
  const int64_t n = min(static_cast<int64_t>(own_block(pos, tok_base, t)), NB - bb);
  return n > 0 ? static_cast<int>(n) : 0;
}

__global__ void __launch_bounds__(kSelThreads, 1)
selector_scores_kernel(const __grid_constant__ CUtensorMap qi_map, const __grid_constant__ CUtensorMap kb_map,
                       int64_t T, int64_t NB, int Hi, float scale, const int32_t* __restrict__ pos,
                       const int32_t* __restrict__ blk_base, const int32_t* __restrict__ tok_base,
                       float* __restrict__ scores, int64_t stride, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Q = kSelRows / Hi;                 // queries per CTA
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * Q;
  const uint32_t bar_q = sb + kSelOffBar + kSelBarQ, bar_k0 = sb + kSelOffBar + kSelBarK0,
                 bar_m0 = sb + kSelOffBar + kSelBarM0;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSelOffBar + kSelTmemSlot);

  // the tile's global candidate blocks: union over its queries of [blk_base, blk_base + own)
  int64_t g_lo = INT64_MAX, g_hi = 0;
  for (int q = 0; q < Q; ++q) {
    const int64_t t = t0 + q;
    if (t >= T) break;
    const int64_t bb = blk_base ? __ldg(blk_base + t) : 0;
    const int n = n_cand(pos, blk_base, tok_base, t, NB);
    if (n > 0) {
      g_lo = min(g_lo, bb);
      g_hi = max(g_hi, bb + n);
    }
  }
  if (g_lo >= g_hi) return;  // no candidate anywhere in the tile (uniform across the CTA)
  const int n_tiles = static_cast<int>((g_hi - g_lo + kSelBlk - 1) / kSelBlk);

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int j = 0; j < kSelKbStages; ++j) mbar_init(bar_k0 + 8 * j, 1);
    mbar_init(bar_m0, 1);
    mbar_init(bar_m0 + 8, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {  // 2 accumulators x 256 FP32 columns = all 512 columns (one CTA per SM)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  const int qi_row0 = static_cast<int>(t0 * Hi);
  auto load_kb = [&](int i) {  // kbar tile i -> stage i % kSelKbStages
    const uint32_t bar = bar_k0 + 8 * (i % kSelKbStages);
    const uint32_t dst = sb + kSelOffKb + (i % kSelKbStages) * kKbBytes;
    mbar_expect_tx(bar, kKbBytes);
    const int g = static_cast<int>(g_lo + static_cast<int64_t>(i) * kSelBlk);
    tma_load_2d(dst, &kb_map, 0, g, bar);
    tma_load_2d(dst + kKbBytes / 2, &kb_map, 64, g, bar);
  };
  auto issue_mma = [&](int i) {  // D[i & 1] = kbar tile i . qi tile^T
    const uint32_t d = tmem + (i & 1) * kSelRows;
    const uint32_t a0 = sb + kSelOffKb + (i % kSelKbStages) * kKbBytes, b0 = sb;
#pragma unroll
    for (int kk = 0; kk < kSelDi / 16; ++kk) {
      // k-step kk: K-block kk / 4, byte offset 32 (kk % 4) inside the 128-byte row
      const uint32_t a = a0 + (kk >> 2) * (kKbBytes / 2) + (kk & 3) * 32;
      const uint32_t b = b0 + (kk >> 2) * (kQiBytes / 2) + (kk & 3) * 32;
      umma_bf16(d, smem_desc_sw128(a), smem_desc_sw128(b), kk > 0 ? 1u : 0u);
    }
    umma_commit(bar_m0 + 8 * (i & 1));
  };

  bool ok = true;
  if (tid == 0) {
    mbar_expect_tx(bar_q, kQiBytes);
    tma_load_2d(sb, &qi_map, 0, qi_row0, bar_q);
    tma_load_2d(sb + kQiBytes / 2, &qi_map, 64, qi_row0, bar_q);
    for (int j = 0; j < min(n_tiles, kSelKbStages); ++j) load_kb(j);
    ok = mbar_wait(bar_q, 0) && mbar_wait(bar_k0, 0);
    if (ok) {
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      issue_mma(0);
    }
  }
  ok = __syncthreads_and(ok) != 0;

  int i = 0;
  for (; ok && i < n_tiles; ++i) {
    // issue the next tile's MMA before this tile's epilogue
    if (tid == 0 && i + 1 < n_tiles) {
      ok = mbar_wait(bar_k0 + 8 * ((i + 1) % kSelKbStages), ((i + 1) / kSelKbStages) & 1);
      if (ok) {
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        issue_mma(i + 1);
      }
    }
    const bool got = mbar_wait(bar_m0 + 8 * (i & 1), (i >> 1) & 1);
    ok = __syncthreads_and(ok && got) != 0;
    if (!ok) break;
    // MMA i has read its kbar stage: refill it kSelKbStages tiles ahead, under the epilogue
    if (tid == 0 && i + kSelKbStages < n_tiles) load_kb(i + kSelKbStages);
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    // epilogue: thread = TMEM lane = block row r of the tile
    const int r = warp * 32 + lane;
    const int64_t g = g_lo + static_cast<int64_t>(i) * kSelBlk + r;
    const uint32_t row_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + (i & 1) * kSelRows;
    for (int q = 0; q < Q; ++q) {
      float s = 0.f;
      for (int h0 = 0; h0 < Hi; h0 += 32) {
        float v[32];
        tmem_ld32(row_addr + q * Hi + h0, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) s += fmaxf(v[j], 0.f);
      }
      const int64_t t = t0 + q;
      if (t < T && g < NB) {
        const int64_t c = g - (blk_base ? __ldg(blk_base + t) : 0);
        if (c >= 0 && c < n_cand(pos, blk_base, tok_base, t, NB) && c < stride) scores[t * stride + c] = scale * s;
      }
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();  // accumulator i & 1 is free again
  }
  if (!ok) {
    if (tid == 0 && status) atomicExch(status, 2);
    // wait (bounded) for this CTA's copies and MMAs still in flight
    if (tid == 0) {
      mbar_wait(bar_q, 0);
      for (int j = i; j < min(n_tiles, i + kSelKbStages); ++j) mbar_wait(bar_k0 + 8 * (j % kSelKbStages), (j / kSelKbStages) & 1);
      for (int j = i; j < min(n_tiles, i + 2); ++j) mbar_wait(bar_m0 + 8 * (j & 1), (j >> 1) & 1);
    }
    __syncthreads();
  }
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(512));
}

// ---------------------------------------------------------------------------
// top-k + expansion: one CTA (256 threads) per query
// ---------------------------------------------------------------------------
constexpr int kTopThreads = 256;

__global__ void __launch_bounds__(kTopThreads)
selector_topk_kernel(const float* __restrict__ scores, int64_t stride, int64_t T, int64_t NB, int k,
                     const int32_t* __restrict__ pos, const int32_t* __restrict__ blk_base,
                     const int32_t* __restrict__ tok_base, int32_t* __restrict__ blocks,
                     int32_t* __restrict__ routes) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_need;
  __shared__ int s_base;
  __shared__ uint32_t s_warp[kTopThreads / 32];
  const int tid = threadIdx.x;
  const int64_t t = blockIdx.x;
  const int n = static_cast<int>(min(static_cast<int64_t>(n_cand(pos, blk_base, tok_base, t, NB)), stride));
  const int own = own_block(pos, tok_base, t);
  const float* row = scores + t * stride;
  // radix select: the k-th largest key among row[0..n) (keys = score bits, >= 0)
  uint32_t prefix = 0, mask = 0;
  uint32_t need = static_cast<uint32_t>(min(k, n));  // rank of the threshold from the top
  for (int shift = 24; shift >= 0 && need > 0 && n > k; shift -= 8) {
    hist[tid] = 0;
    __syncthreads();
    for (int c = tid; c < n; c += kTopThreads) {
      const uint32_t key = __float_as_uint(row[c]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t acc = 0;
      int d = 255;
      for (; d > 0; --d) {
        if (acc + hist[d] >= need) break;
        acc += hist[d];
      }
      s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
      s_need = need - acc;
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    mask |= 255u << shift;
  }
  // keep: key > threshold, plus the `need` lowest-ID blocks with key == threshold
  // (all candidates when n <= k); write them ascending by block ID
  const bool all = n <= k;
  const uint32_t thr = prefix;
  if (tid == 0) s_base = 0;
  __syncthreads();
  int32_t* brow = blocks + t * k;
  int eq_seen = 0;  // running count of threshold-equal keys before this chunk (uniform)
  for (int c0 = 0; c0 < n; c0 += kTopThreads) {
    const int c = c0 + tid;
    uint32_t key = 0;
    bool gt = false, eq = false;
    if (c < n) {
      key = __float_as_uint(row[c]);
      gt = all || key > thr;
      eq = !all && key == thr;
    }
    // rank of this thread's equal key among the chunk's equal keys
    const uint32_t eq_ball = __ballot_sync(0xffffffffu, eq);
    const int lane = tid & 31, w = tid >> 5;
    if (lane == 0) s_warp[w] = __popc(eq_ball);
    __syncthreads();
    int eq_before = eq_seen;
    for (int j = 0; j < w; ++j) eq_before += s_warp[j];
    eq_before += __popc(eq_ball & ((1u << lane) - 1));
    int eq_total = 0;
    for (int j = 0; j < kTopThreads / 32; ++j) eq_total += s_warp[j];
    const bool keep = gt || (eq && eq_before < static_cast<int>(need));
    __syncthreads();
    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) s_warp[w] = __popc(kb);
    __syncthreads();
    int kbefore = s_base;
    for (int j = 0; j < w; ++j) kbefore += s_warp[j];
    kbefore += __popc(kb & ((1u << lane) - 1));
    if (keep) brow[kbefore] = c;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int j = 0; j < kTopThreads / 32; ++j) tot += s_warp[j];
      s_base += tot;
    }
    eq_seen += eq_total;
    __syncthreads();
  }
  const int kept = s_base;
  for (int j = kept + tid; j < k; j += kTopThreads) brow[j] = -1;
  __syncthreads();
  // routes: the kept blocks' tokens, the causal tail, then -1
  const int64_t p = pos ? __ldg(pos + t) : t;
  const int64_t tb = tok_base ? __ldg(tok_base + t) : 0;
  int32_t* rrow = routes + t * static_cast<int64_t>(4 * (k + 1));
  for (int j = tid; j < 4 * (k + 1); j += kTopThreads) {
    const int grp = j >> 2, slot = j & 3;
    int32_t val = -1;
    if (grp < kept) {
      val = static_cast<int32_t>(tb + 4 * static_cast<int64_t>(brow[grp]) + slot);
    } else if (grp == kept) {
      const int64_t tok = tb + 4 * static_cast<int64_t>(own) + slot;
      val = tok <= p ? static_cast<int32_t>(tok) : -1;
    }
    rrow[j] = val;
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D BF16 map over rows of 128 elements (256 bytes), box {64, box_rows}, 128B swizzle.
bool encode_rows(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kSelDi), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kSelDi) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_selector_scores(const void* qi, const void* kbar, int64_t T, int64_t NB, int Hi, float scale,
                                   const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base,
                                   float* scores, int64_t stride, int* status, cudaStream_t s) {
  CUtensorMap qi_map, kb_map;
  if (!encode_rows(&qi_map, qi, static_cast<uint64_t>(T) * Hi, kSelRows) ||
      !encode_rows(&kb_map, kbar, static_cast<uint64_t>(NB), kSelBlk))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(selector_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelSmem);
  if (e != cudaSuccess) return e;
  const int Q = kSelRows / Hi;
  const int64_t grid = (T + Q - 1) / Q;
  selector_scores_kernel<<<static_cast<unsigned>(grid), kSelThreads, kSelSmem, s>>>(
      qi_map, kb_map, T, NB, Hi, scale, pos, blk_base, tok_base, scores, stride, status);
  return cudaGetLastError();
}

cudaError_t launch_selector_topk(const float* scores, int64_t stride, int64_t T, int64_t NB, int k,
                                 const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base,
                                 int32_t* blocks, int32_t* routes, cudaStream_t s) {
  selector_topk_kernel<<<static_cast<unsigned>(T), kTopThreads, 0, s>>>(scores, stride, T, NB, k, pos, blk_base,
                                                                        tok_base, blocks, routes);
  return cudaGetLastError();
}

}  // namespace qsa
