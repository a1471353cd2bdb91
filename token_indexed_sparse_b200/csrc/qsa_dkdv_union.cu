// dK / dV over 128-key tiles on the tensor cores (tcgen05), all query phases in
// one launch.
//
// Backward equations of the cuDNN-Frontend "Query Sparse Attention (QSA)" page
// ("Selection and components"), per KV group g, summed over its 12 heads:
//   dK [key] = scale * sum_t sum_h dS[t, h, key] Q[t, h],   dV [key] = sum_t sum_h P[t, h, key] dO[t, h].
// A work unit is (tile of 128 keys, group g, tensor dK or dV).  Its queries are
// the tile's transpose list for the phase: one entry per query row that routes
// into the tile (its "union": the row's keys inside the tile, a contiguous run
// of the sorted row), so a query's 12 Q (or dO) rows are gathered once per tile
// however many of the tile's keys it selected.  Per chunk of 8 unions:
//   D [128 keys x 256 dims] += A [128 keys x 96] . B [96 x 256 dims]
// with K row 12 u + h = head h of union u; A holds the BF16 dS (for dK) or P
// (for dV) halves of the 48-byte records the dQ kernel wrote, zero where a
// union did not select the key; B holds the gathered Q (or dO) rows.  That is
// 6 tcgen05.mma kind::f16 (M 128, N 256, K 16), A K-major without swizzle, B
// MN-major with the 128-byte swizzle, the accumulator in tensor memory (two
// 256-column buffers, so the epilogue of one unit overlaps the next unit's MMAs).
// Chunks of 8 unions rather than 4 halve the MMA thread's fixed cost per union,
// at three 72 KB stages instead of six of 36 KB, and four warps per stage keep
// more copies in flight (seq32k 7.3 -> 5.6 ms, thd16k 1.53 -> 1.14 ms).
//
// Warp roles (576 threads): warp 16 schedules (claims units, cuts them into
// chunks of 8 entries, publishes each chunk's descriptor in a shared-memory ring
// and prefetches its records and keys into L2); warps 0-11 fill the chunks,
// warps s, s + 3, s + 6 and s + 9 every chunk of stage s of the 3-stage
// shared-memory ring, each two of its unions (clear A, copy the records' P or
// dS halves straight into their A rows and gather the B rows, all with
// cp.async; a warp keeps only about eight 512-byte copies in flight, so the
// rows of a chunk are split over four warps);
// warp 17 (one thread) issues the MMAs; warps 12-15 (tensor-memory lane
// quarters 0-3) run the epilogue, thread = key row.  Units are claimed from one counter in
// phase order (phase 0's units, then phase 1's, ...; inside a phase every dK
// unit before every dV unit), so the
// CTAs work on about one phase and one tensor at a time and its Q (or dO) rows
// stay in L2.  A unit sums its entries in list order; its epilogue waits until
// the unit of the same (tile, group, tensor) in the previous non-empty phase has
// stored its FP32 partial (a per-(tile, group, tensor) counter in global
// memory), adds it, and stores its own partial or the final dK / dV.  The
// summation order is fixed, whichever CTA ran what: no floating-point atomics,
// bitwise reproducible.  A wait only ever targets a unit claimed earlier, by a
// CTA that is running, so the waits cannot form a cycle.  Every wait is
// bounded; on expiry the kernel sets the status word, stops all roles, waits
// (bounded) for its MMAs, frees its tensor memory and returns.
#include "qsa_internal.h"
#include "qsa_device.cuh"

namespace qsa {
namespace {

// CTAs per SM and accumulator buffers per CTA (tensor memory: 256 columns per
// buffer, 512 per SM)
constexpr int kUCtasPerSm = 1, kUAccBufs = 2;
constexpr int kUTmemCols = 256 * kUAccBufs;
constexpr int kUStages = 3;
constexpr int kUWorkersPerStage = 4;                // warps per stage, kUUnions / 4 unions each
constexpr int kUWorkers = kUStages * kUWorkersPerStage;  // warps 0-11 fill chunks
constexpr int kUEpiWarp0 = 12, kUSchedWarp = 16, kUMmaWarp = 17;
constexpr int kUWarps = 18;
constexpr int kUThreads = 32 * kUWarps;
constexpr int kURec = 24;                           // bf16 per (t, g, key) record: 12 P + 12 dS
constexpr int kUKeys = 128;                         // keys per tile (MMA M)
constexpr int kUUnions = 8;                         // unions per chunk
constexpr int kUK = kUUnions * kHeadsPerGroup;      // 96 K rows per chunk
constexpr int kUBBlk = kUK * 128;                   // one 64-dim column block of B (12 KB)
constexpr int kUBBytes = 4 * kUBBlk;                // 48 KB
constexpr int kUASbo = (kUK / 8) * 128;             // A: bytes between 8-key core-matrix rows (768)
constexpr int kUABytes = kUKeys * kUK * 2;          // 24 KB
constexpr int kUStage = kUBBytes + kUABytes;        // 72 KB
constexpr int kURing = 16;                          // chunk descriptors the scheduler may run ahead
constexpr int kUOffCtl = kUStages * kUStage;
// control block: stage descriptors, accumulator descriptors, the chunk ring
// (header int4 + 4 list entries), phase prefix, barriers, tmem slot, abort flag
constexpr int kUOffDesc = kUOffCtl;                          // kUStages x int4
constexpr int kUOffAcc = kUOffDesc + kUStages * 16;          // 2 x int4
constexpr int kURingSlot = 16 + 8 * kUUnions;                // header int4 + the chunk's entries
constexpr int kUOffRing = kUOffAcc + 2 * 16;                 // kURing x kURingSlot bytes
constexpr int kUMaxPhases = 64;
constexpr int kUOffPref = kUOffRing + kURing * kURingSlot;   // kUMaxPhases + 1 ints: units before each phase
constexpr int kUOffBar = (kUOffPref + 4 * (kUMaxPhases + 1) + 7) & ~7;
constexpr int kUBarFull = kUOffBar, kUBarEmpty = kUBarFull + 8 * kUStages;
constexpr int kUBarRingFull = kUBarEmpty + 8 * kUStages, kUBarRingEmpty = kUBarRingFull + 8 * kURing;
constexpr int kUBarAccFull = kUBarRingEmpty + 8 * kURing, kUBarAccEmpty = kUBarAccFull + 16;
constexpr int kUBarDrain = kUBarAccEmpty + 16;
constexpr int kUOffTmem = kUBarDrain + 8, kUOffAbort = kUOffTmem + 4;
constexpr int kUSmem = kUOffAbort + 4 + 1024;      // + alignment slack
static_assert(kUStage % 1024 == 0, "stage alignment (128-byte swizzle atoms)");
static_assert(kUSmem <= 232448, "shared memory per block");
static_assert((kUUnions & (kUUnions - 1)) == 0 && 32 % kUUnions == 0 && kURingSlot % 16 == 0,
              "chunks of a power-of-two number of unions, a divisor of the scheduler's 32-entry window");
// kUWorkersPerStage workers per stage: chunk c goes to warps c % kUStages + h
// kUStages, so every wait on a stage's barriers comes from those warps, each in
// chunk order, at most one phase ahead of the barrier (a
// parity wait two phases early would pass at once).  The descriptor ring is at
// least as deep as the stage count for the same reason.
static_assert(kUWorkers == kUStages * kUWorkersPerStage && kUUnions % kUWorkersPerStage == 0 &&
                  kURing >= kUStages,
              "a fixed set of workers per stage, an equal share of the unions each");
static_assert(kUEpiWarp0 % 4 == 0 && kUEpiWarp0 + 4 <= kUWarps && kUSchedWarp >= kUWorkers &&
                  kUSchedWarp < kUWarps && kUMmaWarp >= kUWorkers && kUMmaWarp < kUWarps &&
                  kUSchedWarp != kUMmaWarp && (kUMmaWarp < kUEpiWarp0 || kUMmaWarp >= kUEpiWarp0 + 4) &&
                  (kUSchedWarp < kUEpiWarp0 || kUSchedWarp >= kUEpiWarp0 + 4),
              "warp roles (epilogue warps cover tensor-memory lane quarters 0-3 in order)");
static_assert(kUTmemCols * kUCtasPerSm <= 512, "tensor memory per SM");
static_assert((kUSmem + 1024) * kUCtasPerSm <= 233472, "shared memory per SM");
constexpr uint32_t kUSpin = 1u << 22;
constexpr int kChFirst = 1, kChLast = 2;
// kind::f16: FP32 accumulate, BF16 A (K-major) and B (MN-major), N = 256, M = 128.
constexpr uint32_t kUIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

// Bounded wait that also gives up once another role has aborted.
__device__ __forceinline__ bool u_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t it = 0; it < kUSpin; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 255) == 255 && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}
// A: K-major, no swizzle; core matrices of 8 rows x 16 bytes, 128 bytes apart
// along K (LBO) and kUASbo apart along M (SBO).
__device__ __forceinline__ uint64_t u_desc_a(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3fff) | (static_cast<uint64_t>(128 >> 4) << 16) |
         (static_cast<uint64_t>(kUASbo >> 4) << 32) | (static_cast<uint64_t>(1) << 46);
}
// B: MN-major, 128-byte swizzle; 64-dim column blocks kUBBlk apart (LBO), 8-row
// groups 1024 bytes apart (SBO).
__device__ __forceinline__ uint64_t u_desc_b(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3fff) | (static_cast<uint64_t>(kUBBlk >> 4) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}
__device__ __forceinline__ void u_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(kUIdesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void u_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void u_ld32(uint32_t taddr, float (&v)[32]) {
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

__global__ void __launch_bounds__(kUThreads, kUCtasPerSm)
dkdv_union_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ q,
                  const uint16_t* __restrict__ pds, const int32_t* __restrict__ row_cols,
                  const int64_t* __restrict__ ent, const int32_t* __restrict__ wl_cnt, const int4* __restrict__ wl,
                  int* __restrict__ claim_ctr, int* __restrict__ done, int P, int64_t n_tiles, int64_t T_kv, int G,
                  int n_sel, float scale,
                  float* __restrict__ partial, void* __restrict__ dk_out, void* __restrict__ dv_out, bool f32_out,
                  int* __restrict__ status) {
  extern __shared__ uint8_t u_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(u_smem_raw) + 1023) & ~uintptr_t{1023});
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = G * kHeadsPerGroup;
  const int units_per_item = 2 * G;
  volatile int* pref = reinterpret_cast<volatile int*>(smem + kUOffPref);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kUOffAbort);
  int4* desc = reinterpret_cast<int4*>(smem + kUOffDesc);
  int4* acc_desc = reinterpret_cast<int4*>(smem + kUOffAcc);
  uint8_t* ring = smem + kUOffRing;  // chunk c: header int4 at kURingSlot (c % kURing), entries after it

  if (tid == 0) {
    for (int s = 0; s < kUStages; ++s) {
      mbar_init(sbase + kUBarFull + 8 * s, kUWorkersPerStage);  // the worker warps that filled the stage
      mbar_init(sbase + kUBarEmpty + 8 * s, 1);  // the MMAs that read it
    }
    for (int r = 0; r < kURing; ++r) {
      mbar_init(sbase + kUBarRingFull + 8 * r, 1);   // the scheduler wrote the descriptor
      mbar_init(sbase + kUBarRingEmpty + 8 * r, kUWorkersPerStage);  // its workers read it
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sbase + kUBarAccFull + 8 * b, 2);   // MMA completion + the issuing thread's descriptor arrival
      mbar_init(sbase + kUBarAccEmpty + 8 * b, 4);  // one arrival per epilogue warp
    }
    mbar_init(sbase + kUBarDrain, 1);
    *abort_flag = 0;
    int acc = 0;
    for (int p = 0; p < P; ++p) {
      pref[p] = acc;
      acc += __ldg(wl_cnt + p) * units_per_item;
    }
    pref[P] = acc;
    mbar_fence_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(sbase + kUOffTmem),
                 "r"(kUTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kUOffTmem);
  const int n_units = pref[P];

  if (warp < kUWorkers) {
    // ------------------------------------------------------------ workers
    // Warps s + 3 h (h < kUWorkersPerStage) fill chunks s, s + 3, s + 6, ...
    // together, each taking kMy of the chunk's unions: each takes the chunk's
    // descriptor from the scheduler's ring, loads its unions' keys, waits for
    // the chunk's stage to be free, clears its unions' A slots, copies their
    // records into the A rows of their keys and gathers their 24 Q (or dO) rows
    // into B (cp.async, 8 and 16 bytes), waits for its copies and arrives on the
    // stage's full barrier (complete when all have).  Up to kUStages chunks are
    // in flight at once, with no barrier between stages.  (Records loaded into
    // registers first and stored after the gather, with keys past 32 of a run
    // loaded one after another, ran thd16k's dK/dV in 1.16 ms against 0.89 ms.)
    const int s = warp % kUStages, half = warp / kUStages;
    constexpr int kMy = kUUnions / kUWorkersPerStage;  // unions per warp
    const int u0 = kMy * half;                         // this warp's first union of a chunk
    // A rows this lane wrote in the warp's previous chunk (its stage still holds
    // them; keys lane and lane + 32 of each union): clearing those 24-byte slots
    // restores zeros in this warp's unions' columns without rewriting the tile;
    // they are cleared for all 128 rows on the stage's first use and after a
    // chunk whose records were not all tracked (runs > 64 keys)
    int prev_m[kMy], prev_m2[kMy];  // A rows of keys 0..31 and 32..63 of the warp's unions
#pragma unroll
    for (int j = 0; j < kMy; ++j) prev_m[j] = prev_m2[j] = -1;
    bool zero_all = true;
    for (int c = s;; c += kUStages) {
      const int rs = c % kURing;
      bool got = true;
      if (lane == 0) got = u_wait(sbase + kUBarRingFull + 8 * rs, (c / kURing) & 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      __syncwarp();  // every lane reads the descriptor after lane 0 saw it published
      const volatile int* hv = reinterpret_cast<const volatile int*>(ring + kURingSlot * rs);
      const int4 hd = make_int4(hv[0], hv[1], hv[2], hv[3]);
      int64_t e[kMy];
#pragma unroll
      for (int j = 0; j < kMy; ++j) e[j] = reinterpret_cast<const volatile int64_t*>(ring + kURingSlot * rs + 16)[u0 + j];
      __syncwarp();
      if (lane == 0) mbar_arrive(sbase + kUBarRingEmpty + 8 * rs);
      const bool end = hd.x < 0;
      if (end && hd.y == 0) break;  // an end marker for a stage whose chunk the MMA never reaches
      const int n = hd.z & 255, r = hd.z >> 10, g = r >> 1, tensor = r & 1, tile = hd.w;
      // the keys of this warp's unions (positions lane and lane + 32 of each
      // run), loaded first so that their latency overlaps the wait for the
      // stage; record i of union u goes to A row (key - tile base), K columns
      // 12 u .. 12 u + 11 (dK takes the record's dS half, dV its P half)
      const int key0 = tile * kUKeys;
      int32_t key[kMy], key2[kMy];
#pragma unroll
      for (int j = 0; j < kMy; ++j) {
        const int64_t t = e[j] >> 32;
        const int i0 = static_cast<int>((e[j] >> 8) & 0x3fff), cnt = static_cast<int>(e[j] & 0x7f) + 1;
        const bool ok_j = u0 + j < n && lane < cnt;
        key[j] = ok_j ? __ldg(row_cols + t * n_sel + i0 + lane) : -1;
        key2[j] = u0 + j < n && lane + 32 < cnt ? __ldg(row_cols + t * n_sel + i0 + 32 + lane) : -1;
      }
      // stage s is free once the MMAs of chunk c - kUStages completed
      if (c >= kUStages) {
        if (lane == 0) got = u_wait(sbase + kUBarEmpty + 8 * s, ((c / kUStages) - 1) & 1, abort_flag);
        if (!__shfl_sync(0xffffffffu, got, 0)) break;
      }
      const uint32_t st = sbase + s * kUStage;
      if (end) {  // the first chunk past the last unit: end marker for the MMA warp
        if (lane == 0) {
          if (half == 0) desc[s] = make_int4(0, -1, 0, 0);
          mbar_arrive(sbase + kUBarFull + 8 * s);
        }
        break;
      }
      // A must read 0 in every (union, key) slot this chunk does not fill
      uint8_t* abase = smem + s * kUStage + kUBBytes;
      auto slot = [&](int u, int m, int hq) -> uint2* {
        const int kk = u * kHeadsPerGroup + 4 * hq;
        return reinterpret_cast<uint2*>(abase + (m >> 3) * kUASbo + (m & 7) * 16 + (kk >> 3) * 128 + (kk & 7) * 2);
      };
      if (zero_all) {
#pragma unroll 4
        for (int i = lane; i < kMy * kUKeys * 3; i += 32) {
          const int j = i / (kUKeys * 3), rem = i - j * (kUKeys * 3);
          *slot(u0 + j, rem / 3, rem % 3) = make_uint2(0, 0);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kMy; ++j)
          if (prev_m[j] >= 0) {
#pragma unroll
            for (int hq = 0; hq < 3; ++hq) *slot(u0 + j, prev_m[j], hq) = make_uint2(0, 0);
          }
#pragma unroll
        for (int j = 0; j < kMy; ++j)
          if (prev_m2[j] >= 0) {
#pragma unroll
            for (int hq = 0; hq < 3; ++hq) *slot(u0 + j, prev_m2[j], hq) = make_uint2(0, 0);
          }
      }
      __syncwarp();  // the clearing above before the record copies below
      // record i of union u (its P or dS half: 3 x 8 bytes) straight into the A
      // row of its key; returns that row, or -1
      auto copy_rec = [&](int j, int32_t k, int i) -> int {
        const int m = k - key0;
        if (k < 0 || static_cast<unsigned>(m) >= static_cast<unsigned>(kUKeys)) return -1;  // never for a well-formed list
        const int64_t t = e[j] >> 32;
        const int i0 = static_cast<int>((e[j] >> 8) & 0x3fff);
        const uint2* rec = reinterpret_cast<const uint2*>(pds + ((t * G + g) * n_sel + i0 + i) * kURec) + (tensor ? 0 : 3);
#pragma unroll
        for (int hq = 0; hq < 3; ++hq)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(slot(u0 + j, m, hq))), "l"(rec + hq)
                       : "memory");
        return m;
      };
#pragma unroll
      for (int j = 0; j < kMy; ++j) {
        prev_m[j] = copy_rec(j, key[j], lane);
        prev_m2[j] = copy_rec(j, key2[j], lane + 32);
      }
      // B: the 12 head rows of each of this warp's unions (zero-filled for missing unions)
      {
        const __nv_bfloat16* base = (tensor ? dout : q) + (g * kHeadsPerGroup * kHeadDim + lane * 8);
        const uint32_t dst = st + (lane >> 3) * kUBBlk;
        const int unit = lane & 7;
#pragma unroll
        for (int j = 0; j < kMy; ++j) {
          const bool mine = u0 + j < n;
          const __nv_bfloat16* src = base + (mine ? (e[j] >> 32) : 0) * H * kHeadDim;
#pragma unroll
          for (int h = 0; h < kHeadsPerGroup; ++h) {
            const int kr = (u0 + j) * kHeadsPerGroup + h;
            cp_async16(dst + kr * 128 + ((unit ^ (kr & 7)) << 4), src + h * kHeadDim, mine);
          }
        }
      }
      cp_async_commit();
      // stores record j of union u; returns its A row, or -1
      auto put = [&](int u, int32_t k, const uint2 (&v)[3]) -> int {
        const int m = k - key0;
        if (k < 0 || static_cast<unsigned>(m) >= static_cast<unsigned>(kUKeys)) return -1;  // never for a well-formed list
#pragma unroll
        for (int hq = 0; hq < 3; ++hq) *slot(u, m, hq) = v[hq];
        return m;
      };
      // unions with more than 64 keys in the tile (rare for sparse routes); their
      // extra rows are not tracked, so the next chunk of this stage clears all
      // of this warp's slots
      zero_all = false;
#pragma unroll
      for (int j = 0; j < kMy; ++j) {
        const int64_t t = e[j] >> 32;
        const int i0 = static_cast<int>((e[j] >> 8) & 0x3fff), cnt = static_cast<int>(e[j] & 0x7f) + 1;
        if (u0 + j >= n || cnt <= 64) continue;
        zero_all = true;
        const uint2* rec = reinterpret_cast<const uint2*>(pds + ((t * G + g) * n_sel + i0) * kURec) + (tensor ? 0 : 3);
        for (int jj = lane + 64; jj < cnt; jj += 32) {
          const uint2 v[3] = {__ldg(rec + jj * 6), __ldg(rec + jj * 6 + 1), __ldg(rec + jj * 6 + 2)};
          put(u0 + j, __ldg(row_cols + t * n_sel + i0 + jj), v);
        }
      }
      if (half == 0 && lane == 0) desc[s] = make_int4(hd.x, n, (hd.z >> 8) & 3, r);
      // this warp's part of the stage is complete once its copies landed: make
      // it visible to the tensor cores, arrive on the stage's full barrier
      cp_async_wait<0>();
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(sbase + kUBarFull + 8 * s);
    }
  } else if (warp == kUMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int useq = 0;
      bool ok = true;
      for (int c = 0;; ++c) {
        const int s = c % kUStages;
        if (!u_wait(sbase + kUBarFull + 8 * s, (c / kUStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int4 d = desc[s];
        if (d.y < 0) break;
        const int buf = useq % kUAccBufs;
        if ((d.z & kChFirst) && useq >= kUAccBufs &&
            !u_wait(sbase + kUBarAccEmpty + 8 * buf, ((useq / kUAccBufs) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        const uint32_t st = sbase + s * kUStage;
        const int nks = (d.y * kHeadsPerGroup + 15) / 16;
        for (int ks = 0; ks < nks; ++ks)
          u_mma(tmem + buf * 256, u_desc_a(st + kUBBytes + ks * 256), u_desc_b(st + ks * 2048),
                ((d.z & kChFirst) && ks == 0) ? 0u : 1u);
        u_commit(sbase + kUBarEmpty + 8 * s);
        if (d.z & kChLast) {
          acc_desc[buf] = make_int4(d.x, d.w, 0, 0);
          u_commit(sbase + kUBarAccFull + 8 * buf);
          mbar_arrive(sbase + kUBarAccFull + 8 * buf);
          ++useq;
        }
      }
      if (ok) {  // end marker for the epilogue
        const int buf = useq % kUAccBufs;
        if (useq < kUAccBufs || u_wait(sbase + kUBarAccEmpty + 8 * buf, ((useq / kUAccBufs) - 1) & 1, abort_flag)) {
          acc_desc[buf] = make_int4(-1, 0, 0, 0);
          mbar_arrive(sbase + kUBarAccFull + 8 * buf);
          mbar_arrive(sbase + kUBarAccFull + 8 * buf);
        }
      }
      // all issued MMAs complete before the tensor memory is released
      u_commit(sbase + kUBarDrain);
      for (uint32_t it = 0; it < kUSpin && !mbar_try(sbase + kUBarDrain, 0); ++it) {
      }
    }
    __syncwarp();
  } else if (warp >= kUEpiWarp0 && warp < kUEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp - kUEpiWarp0;      // tensor-memory lanes 32 quarter .. + 31
    const int m = quarter * 32 + lane;          // key row within the tile
    const bool leader = quarter == 0 && lane == 0;
    for (int useq = 0;; ++useq) {
      const int buf = useq % kUAccBufs;
      // the four warps leave together: one warp whose wait expired must not
      // leave the others in the named barriers below
      const bool got = u_wait(sbase + kUBarAccFull + 8 * buf, (useq / kUAccBufs) & 1, abort_flag);
      if (bar_or(3, 128, !got)) break;
      const int idx = acc_desc[buf].x, r = acc_desc[buf].y;
      if (idx < 0) break;
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      const int4 it = __ldg(wl + idx);
      const int g = r >> 1, tensor = r & 1;
      const int ord = it.w >> 2;                 // earlier non-empty phases of this tile
      const bool last = it.w & 2;
      const int64_t key = static_cast<int64_t>(it.x) * kUKeys + m;
      const int64_t slot = (static_cast<int64_t>(it.x) * G + g) * 2 + tensor;
      float* part = partial + slot * (kUKeys * kHeadDim) + static_cast<int64_t>(m) * kHeadDim;
      const float f = tensor ? 1.f : scale;
      if (ord > 0) {
        // the previous phase's partial of this (tile, group, tensor) must be stored
        bool fail = false;
        if (leader) {
          uint32_t it2 = 0;
          for (;; ++it2) {
            int v;
            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(done + slot) : "memory");
            if (v >= ord) break;
            if (it2 >= kUSpin || ((it2 & 255) == 255 && *abort_flag)) {
              *abort_flag = 1;
              fail = true;
              break;
            }
            __nanosleep(64);
          }
        }
        if (bar_or(3, 128, fail)) break;
      }
      for (int j = 0; j < kHeadDim / 32; ++j) {
        float v[32];
        u_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * 256 + j * 32, v);
        if (ord > 0) {
          const float4* pr = reinterpret_cast<const float4*>(part + j * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 x = __ldcg(pr + i);
            v[4 * i] += x.x;
            v[4 * i + 1] += x.y;
            v[4 * i + 2] += x.z;
            v[4 * i + 3] += x.w;
          }
        }
        if (last) {
          if (key < T_kv) {
            const int64_t o = (key * G + g) * kHeadDim + j * 32;
            if (f32_out) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(tensor ? dv_out : dk_out) + o);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(v[4 * i] * f, v[4 * i + 1] * f, v[4 * i + 2] * f, v[4 * i + 3] * f);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(tensor ? dv_out : dk_out) + o);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pack_bf16(v[8 * i] * f, v[8 * i + 1] * f), pack_bf16(v[8 * i + 2] * f, v[8 * i + 3] * f),
                                    pack_bf16(v[8 * i + 4] * f, v[8 * i + 5] * f),
                                    pack_bf16(v[8 * i + 6] * f, v[8 * i + 7] * f));
            }
          }
        } else {
          float4* pw = reinterpret_cast<float4*>(part + j * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) __stcg(pw + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(sbase + kUBarAccEmpty + 8 * buf);
      if (!last) {
        // publish the partial: every epilogue thread's stores, then the counter
        bar_sync(3, 128);
        if (leader) {
          __threadfence();
          asm volatile("st.release.gpu.global.b32 [%0], %1;\n" ::"l"(done + slot), "r"(ord + 1) : "memory");
        }
      }
    }
  } else if (warp == kUSchedWarp) {
    // ------------------------------------------------------------ scheduler
    // Claims units (one ahead) in phase order, cuts them into chunks of up to 4
    // entries, writes each chunk's descriptor and entries into the ring, and
    // prefetches into L2 the record runs and key runs the chunk's worker will
    // load into registers (up to kURing chunks ahead).
    int claim_p = 0;
    // unit U -> its phase p, and inside the phase tensor-major order (every dK
    // unit, then every dV unit, so one tensor's rows are live in L2 at a time):
    // {work item index, r = 2 g + tensor}; item.x < 0 when the list is exhausted
    auto claim = [&](int4& item, int& idx, int& r) {
      int U = 0;
      if (lane == 0) U = atomicAdd(claim_ctr, 1);
      U = __shfl_sync(0xffffffffu, U, 0);
      if (U >= n_units) {
        item = make_int4(-1, 0, 0, 0);
        return;
      }
      while (pref[claim_p + 1] <= U) ++claim_p;  // claims only grow
      const int local = U - pref[claim_p];
      const int per_tensor = (pref[claim_p + 1] - pref[claim_p]) >> 1;  // items x G
      const int tensor = local >= per_tensor ? 1 : 0;
      const int rem = local - tensor * per_tensor;
      idx = static_cast<int>(claim_p * n_tiles) + rem / G;
      r = 2 * (rem % G) + tensor;
      item = __ldg(wl + idx);
    };
    // L2 prefetch of the 128-byte lines of [p, p + bytes) (a plain per-line hint:
    // the bulk prefetch goes through the bulk-copy unit, one operation at a time)
    auto prefetch_l2 = [&](const void* p, int64_t bytes) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(p);
      for (uintptr_t a = a0 & ~uintptr_t{127}; a < a0 + bytes; a += 128)
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(a < a0 ? a0 : a) : "memory");
    };
    int c = 0;
    bool ok = true;
    int4 cur, nxt;
    int cur_idx = 0, cur_r = 0, nxt_idx = 0, nxt_r = 0;
    claim(cur, cur_idx, cur_r);
    if (cur.x >= 0) claim(nxt, nxt_idx, nxt_r);
    while (ok && cur.x >= 0) {
      const int g = cur_r >> 1;
      // windows of up to 32 entries, lane i holding entry w0 + i; the next
      // window's entries are loaded while this one is published
      int64_t el_next = cur.y + lane < cur.z ? __ldg(ent + cur.y + lane) : 0;
      for (int w0 = cur.y; ok && w0 < cur.z; w0 += 32) {
        const bool have = w0 + lane < cur.z;
        const int64_t el = el_next;
        el_next = w0 + 32 + lane < cur.z ? __ldg(ent + w0 + 32 + lane) : 0;
        if (have) {  // the records and keys the workers load into registers
          const int64_t t = el >> 32;
          const int i0 = static_cast<int>((el >> 8) & 0x3fff), cnt = static_cast<int>(el & 0x7f) + 1;
          prefetch_l2(pds + ((t * G + g) * n_sel + i0) * kURec, cnt * kURec * 2);
          prefetch_l2(row_cols + t * n_sel + i0, cnt * 4);
        }
        const int w1 = min(cur.z, w0 + 32);
        for (int p = w0; p < w1; p += kUUnions) {
          const int n = min(kUUnions, cur.z - p);
          const int rs = c % kURing;
          bool got = true;
          if (c >= kURing && lane == 0) got = u_wait(sbase + kUBarRingEmpty + 8 * rs, ((c / kURing) - 1) & 1, abort_flag);
          if (!__shfl_sync(0xffffffffu, got, 0)) {
            ok = false;
            break;
          }
          const int64_t eu = __shfl_sync(0xffffffffu, el, (p - w0) + (lane & (kUUnions - 1)));
          if (lane < kUUnions) reinterpret_cast<int64_t*>(ring + kURingSlot * rs + 16)[lane] = lane < n ? eu : 0;
          const int flags = (p == cur.y ? kChFirst : 0) | (p + n >= cur.z ? kChLast : 0);
          if (lane == 0) *reinterpret_cast<int4*>(ring + kURingSlot * rs) = make_int4(cur_idx, p, n | (flags << 8) | (cur_r << 10), cur.x);
          __syncwarp();
          if (lane == 0) mbar_arrive(sbase + kUBarRingFull + 8 * rs);
          ++c;
        }
      }
      cur = nxt;
      cur_idx = nxt_idx;
      cur_r = nxt_r;
      if (cur.x >= 0) claim(nxt, nxt_idx, nxt_r);
    }
    // end markers: chunk c (the first past the list) ends the MMA loop; each of
    // the other stages' worker pairs gets one that only ends their own loop
    for (int k = 0; ok && k < kUStages; ++k, ++c) {
      const int rs = c % kURing;
      bool got = true;
      if (c >= kURing && lane == 0) got = u_wait(sbase + kUBarRingEmpty + 8 * rs, ((c / kURing) - 1) & 1, abort_flag);
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      if (lane == 0) {
        *reinterpret_cast<int4*>(ring + kURingSlot * rs) = make_int4(-1, k == 0 ? 1 : 0, 0, 0);
        mbar_arrive(sbase + kUBarRingFull + 8 * rs);
      }
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  if (*abort_flag && tid == 0 && status) atomicExch(status, 3);
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kUTmemCols));
}

}  // namespace

// Query phases of the dK/dV pass: each phase covers C consecutive queries, chosen
// so that one phase's Q and dO rows (C * H * 1 KB; the pass reads one tensor at
// a time) stay resident in L2 (48 MiB), but at least 4096 queries: every phase
// boundary costs an FP32 partial read and write per (tile, group, tensor), and
// with many heads the L2 bound alone makes phases so short that this dominates
// (seq32k, 24 heads: 2048 queries per phase ran dK/dV in 7.7 ms, 4096 in 7.1 ms;
// with 12 heads the bound is 4096 already).  At most 64 phases.  It lives with
// the kernel because the launch's DRAM traffic depends on both.
void dkdv_phases(int64_t T, int H, int* P, int* C) {
  int64_t c = (int64_t{48} << 20) / (static_cast<int64_t>(H) * 1024);
  c = c < 4096 ? 4096 : (c / 256) * 256;
  int64_t p = (T + c - 1) / c;
  if (p > 64) {
    c = (((T + 63) / 64) + 255) / 256 * 256;
    p = (T + c - 1) / c;
  }
  *P = static_cast<int>(p);
  *C = static_cast<int>(c);
}

cudaError_t launch_backward_dkdv_union(const void* grad_out, const void* q, const uint16_t* pds,
                                       const int32_t* row_cols, const int64_t* tile_ent, const int32_t* wl_cnt,
                                       const int4* wl, int* claim_ctr, int* done, int P, int64_t n_tiles,
                                       int64_t T_kv, int G, int n_sel, float scale, float* partial, void* dk, void* dv,
                                       bool f32_out, int* status, cudaStream_t s) {
  if (P < 1 || P > kUMaxPhases) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(dkdv_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUSmem);
  if (e != cudaSuccess) return e;
  dkdv_union_kernel<<<static_cast<unsigned>(kUCtasPerSm * sm_count()), kUThreads, kUSmem, s>>>(
      static_cast<const __nv_bfloat16*>(grad_out), static_cast<const __nv_bfloat16*>(q), pds, row_cols, tile_ent,
      wl_cnt, wl, claim_ctr, done, P, n_tiles, T_kv, G, n_sel, scale, partial, dk, dv, f32_out, status);
  return cudaGetLastError();
}

}  // namespace qsa
