// tcgen05 (5th-generation tensor core) split-KV decode kernel for the bf16
// workloads: r = 512 latent columns, 64 RoPE columns, 64-token pages,
// up to 128 query rows (heads x query tokens) per sequence.
//
// One CTA pair (a cluster of 2 on one TPC) per worker. The pair walks the
// worker's split segments (see common.cuh) in groups of 4 pages = 256 tokens:
//
//   QK  (cta_group::2, M = 128 rows, N = 256 tokens, K = 576): S = Q . [cKV ||
//       k_rope]^T. CTA c holds query rows [64c, 64c+64) of Q in shared memory
//       and supplies tokens [128c, 128c+128) (group pages 2c, 2c+1) as the B
//       operand, streamed in 64-column chunks through a TMA ring. Each CTA's
//       tensor memory receives its 64 rows x 256 tokens, folded over the 128
//       lanes (lanes 0-63: tokens 0-127, lanes 64-127: tokens 128-255).
//       N = 256 matters: a tcgen05.mma costs ~60 cycles whatever its size, and
//       only N = 256 (64 rows x 256 x 16 per SM = 64 cycles of math) keeps the
//       tensor pipe efficient.
//   softmax (4 warps per CTA and shard, fp32, log2 domain): per row online max / sum;
//       the max is moved (and O rescaled) only when it grows by more than 2^8,
//       so every P value lies in [0, 256] and rescales are rare. One pass
//       over the thread's 128 scores in tensor memory (exp2 on the SFU), the
//       row maximum combined with the other token half through shared memory.
//   PV  (cta_group::2, M = 128 rows, N = 256 latent columns, K = 256 tokens,
//       two N blocks): O_lat += P . cKV. CTA c supplies latent columns
//       [256 nb + 128 c, +128) of every token, streamed page by page through
//       a second TMA ring (these tokens were just read for QK, so the re-read
//       is served by L2). One 16 KB P buffer holds pages 0-1 of the group, then
//       pages 2-3 once the PV MMAs are done with the first half.
//   TPLA (S = 2 shards): one S tile per shard (latent chunks 0-3 or 4-7, each
//       with the RoPE chunk), one softmax per shard, PV N block nb = shard nb.
//       The QK chunk order puts the RoPE chunk between the shards, so shard
//       0's tile is complete (and released) on its own; each shard has its
//       own softmax warpgroup (384 threads per CTA, so 168 registers: the
//       scores are read from tensor memory twice, for the max and for P) and
//       its own 16 KB P buffer with the one-shard hand-off; V items run shard
//       by shard within each page half.
//
// QK and PV are issued by two different threads of the leader CTA, so that the
// QK stream (HBM) and the V stream (L2) drain independently; they touch
// disjoint tensor memory and shared memory and meet only through the softmax.
//
// Each CTA's O accumulator covers its 64 rows x 512 latent columns (256 tensor
// memory columns). At the end of a split segment the softmax warps write
// O / l (fp16) and the log2-sum-exp per row into the workspace; the combine
// kernel merges the segments and applies W_UV.
//
// Sources: TPLA abstract (latent cache, shard-and-sum), TransMLA abstract
// (absorbed decode over the compressed cache), pith.science verdict record for
// 2502.07864 (one RoPE key per token, common to all heads).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace mla {

constexpr bool kTcDecodeAvailable = true;

namespace tc {

constexpr int kWidth = 576;                 // r + d_rope at r = 512
constexpr int kChunks = 9;                  // 64-column chunks of a row at r = 512 (8 latent + 1 rope)
constexpr int kGroupPages = 4;              // pages per pair step (256 tokens)
// warps: 0 Q/QK loads, 1 QK MMA, 2 V loads, 3-6 softmax, 7 PV MMA; two
// latent shards add warps 8-11, the softmax of shard 1 (warps 3-6: shard 0)
constexpr int kThreads = 256;
template <int S>
constexpr int threads_of() { return S == 2 ? 384 : 256; }
constexpr uint32_t kQChunkBytes = 64 * 128;  // 64 rows x 128 B
constexpr uint32_t kQBytes = kChunks * kQChunkBytes;
// The latent width R of one launch: 512 (every workload on one GPU), or 256
// (one latent shard per GPU of a tensor-parallel pair: TPLA across GPUs).
// Per R: 64-column chunks of a cached row (latent + RoPE), PV N blocks of 256
// latent columns, and the tensor-memory columns of this CTA's O accumulator.
template <int R>
struct Width {
  static_assert(R == 256 || R == 512, "latent width 256 or 512");
  static constexpr int kChunks = R / 64 + 1;
  static constexpr int kNBlocks = R / 256;
  static constexpr uint32_t kQBytes = kChunks * kQChunkBytes;
  static constexpr uint32_t kOCols = R / 2;
};
// Chunk order within a group. One shard: latent chunks 0..R/64-1, then the
// RoPE chunk. Two shards (r = 512): shard 0's latent chunks 0-3, the RoPE
// chunk (added to both shards' scores), then shard 1's chunks 4-7, so shard
// 0's scores are complete after five chunks and the softmax starts on them
// while shard 1's QK is still running.
template <int S>
__device__ __forceinline__ int chunk_at(int pos) {
  if constexpr (S == 2) return pos < 4 ? pos : (pos == 4 ? 8 : pos - 1);
  return pos;
}
constexpr uint32_t kSlotBytes = 16384;       // QK slot: 128 tokens x 64 cols; V slot: 64 tokens x 128 cols
constexpr uint32_t kPChunkBytes = 64 * 128;  // 64 rows x 64 tokens bf16
constexpr uint32_t kPBytes = 4 * kPChunkBytes;  // 64 rows x 256 tokens
constexpr float kRescaleThreshold = 8.0f;    // log2 units
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;
// A thread's TMA loads are processed one after another (about 4-5 cycles per
// 128-byte row on B200); issuing the two boxes of every ring item from two
// lanes doubles what a producer can stream.
constexpr int kIssueLanes = 2;

#ifndef MLA_QK_SLOTS
#define MLA_QK_SLOTS 4
#endif
#ifndef MLA_V_SLOTS
#define MLA_V_SLOTS 4
#endif
#ifndef MLA_QK_SLOTS_2SHARD
#define MLA_QK_SLOTS_2SHARD 3
#endif
#ifndef MLA_V_SLOTS_2SHARD
#define MLA_V_SLOTS_2SHARD 4
#endif
template <int S, int R = 512>
struct Cfg {
  static constexpr int kQkSlots = S == 1 ? MLA_QK_SLOTS : MLA_QK_SLOTS_2SHARD;
  static constexpr int kVSlots = S == 1 ? MLA_V_SLOTS : MLA_V_SLOTS_2SHARD;
  static constexpr int kSBufs = S == 1 ? 2 : 1;   // S tiles in tensor memory (128 columns each per shard)
  // P per shard: one 16 KB buffer holds group pages 0, 1 and then 2, 3 (the
  // second half is written once PV is done with the first). Against P for all
  // four pages this frees 16 KB per shard for the TMA rings, whose depth sets
  // the streaming rate.
  static constexpr uint32_t kPShard = kPBytes / 2;
  static constexpr uint32_t kPRegion = S * kPShard;
};

template <int S, int R = 512>
struct Smem {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t qk = q + Width<R>::kQBytes;
  static constexpr uint32_t v = qk + Cfg<S, R>::kQkSlots * kSlotBytes;
  static constexpr uint32_t p = v + Cfg<S, R>::kVSlots * kSlotBytes;
  // float [2][S][128] row max (double-buffered by group parity) + [S][128] l
  static constexpr uint32_t xch = p + Cfg<S, R>::kPRegion;
  static constexpr uint32_t bars = xch + 3 * S * 128 * 4;
  static constexpr uint32_t nbars = 56;
  static constexpr uint32_t misc = bars + nbars * 8;  // tmem slot, abort flag
  static_assert(Cfg<S, R>::kQkSlots <= 6 && Cfg<S, R>::kVSlots <= 6, "barrier arrays hold 6 slots");
  static constexpr uint32_t total = misc + 64;
  static constexpr uint32_t alloc = total + 1024;     // alignment slack
  static_assert(alloc <= 227 * 1024, "shared memory of one CTA");
};

// barrier indices (leader = only the leader CTA's copy is used)
enum : int {
  B_Q_FULL = 0,       // (unused: the query arrives chunk by chunk, B_QC_FULL)
  B_QK_FULL = 1,      // [6] leader, count 2 (+tx)
  B_V_FULL = 7,       // [6] leader, count 2 (+tx)
  B_S_FREE = 13,      // [2] leader, count 8 (4 softmax warps x 2 CTAs): by S buffer (one shard) or by shard
  B_P_FULL = 15,      // leader, count 8: P pages 0, 1 written (2 warps x 2 CTAs) and O rescaled (all 8)
  B_O_FREE = 16,      // leader, count 8 S (every softmax warp of both CTAs)
  B_QK_FREE = 17,     // [6] both, count 1 (MMA commit)
  B_V_FREE = 23,      // [6] both, count 1
  B_S_FULL = 29,      // [2] both, count 1: by S buffer (one shard) or by shard (two)
  B_PV_DONE = 31,     // both, count 1
  B_FINAL_QK = 32,    // leader, count 1
  B_FINAL_PV = 33,    // leader, count 1
  B_P_FREE_LO = 34,   // both, count 1: PV is done with P of group pages 0, 1
  B_P_FREE_HI = 35,   // both, count 1: PV is done with P of group pages 2, 3
  B_QC_FULL = 36,     // [9] leader, count 2 (+tx): query chunk k of the current segment
  B_P_FULL_HI = 45,   // leader, count 4: P pages 2, 3 written by 2 warps x 2 CTAs
  // threshold skipping (kSkip): the pair's keep / skip decision of group gi
  B_DECIDE = 46,      // [2] both, count 1 (+4 tx bytes: the peer's vote), by group parity
  B_VSEEN = 48,       // [2] both, count 1: the V producer has read the decision of group gi
  // two shards: shard 1's copies of B_P_FULL, B_P_FULL_HI, B_P_FREE_LO, B_P_FREE_HI
  B_P_FULL_1 = 50,
  B_P_FULL_HI_1 = 51,
  B_P_FREE_LO_1 = 52,
  B_P_FREE_HI_1 = 53,
  B_COUNT = 54
};
// the P hand-off barriers of shard s
__host__ __device__ constexpr int bar_p_full(int s) { return s ? B_P_FULL_1 : B_P_FULL; }
__host__ __device__ constexpr int bar_p_full_hi(int s) { return s ? B_P_FULL_HI_1 : B_P_FULL_HI; }
__host__ __device__ constexpr int bar_p_free_lo(int s) { return s ? B_P_FREE_LO_1 : B_P_FREE_LO; }
__host__ __device__ constexpr int bar_p_free_hi(int s) { return s ? B_P_FREE_HI_1 : B_P_FREE_HI; }
static_assert(B_COUNT <= 56, "barrier array");

// V ring order within a group: item i -> (page q, N block nb). One shard:
// page-major. Two shards (N block nb = shard nb): pages 0, 1 of shard 0,
// pages 0, 1 of shard 1, then pages 2, 3 of each, so that PV releases each
// shard's first P half as early as the one-shard order does.
template <int S, int NB>
__device__ __forceinline__ void v_item(int i, int& q, int& nb) {
  if constexpr (S == 2) {
    nb = (i >> 1) & 1;
    q = 2 * (i >> 2) + (i & 1);
  } else {
    q = i / NB;
    nb = i % NB;
  }
}

// Optional event trace (compile with -DMLA_TRACE): SM clock of per-group events
// of the first kTraceWorkers workers, read back with mla_debug_trace_read().
#ifdef MLA_TRACE
constexpr int kTraceWorkers = 4, kTraceKinds = 15, kTraceSteps = 64;
__device__ unsigned long long g_trace[kTraceWorkers * 2 * kTraceKinds * kTraceSteps];
__device__ unsigned long long g_trace_ns[kTraceWorkers * 2 * kTraceKinds * kTraceSteps];
#define MLA_TRACE_EV(w, rank, kind, step)                                                \
  do {                                                                                   \
    if ((w) < kTraceWorkers && (step) < kTraceSteps) {                                   \
      unsigned long long t_, n_;                                                         \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_));                                 \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(n_));                             \
      g_trace[(((w) * 2 + (rank)) * kTraceKinds + (kind)) * kTraceSteps + (step)] = t_;   \
      g_trace_ns[(((w) * 2 + (rank)) * kTraceKinds + (kind)) * kTraceSteps + (step)] = n_;\
    }                                                                                    \
  } while (0)
// per CTA: globaltimer at entry, after setup, at the start of teardown, at exit
__device__ unsigned long long g_trace_cta[1024 * 4];
#define MLA_TRACE_CTA(k)                                                                  \
  do {                                                                                   \
    if (threadIdx.x == 0 && blockIdx.x < 1024) {                                         \
      unsigned long long n_;                                                             \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(n_));                             \
      g_trace_cta[blockIdx.x * 4 + (k)] = n_;                                            \
    }                                                                                    \
  } while (0)
// chunk-level events of worker 0's leader CTA: QK issue / full, V issue / full
constexpr int kTraceChunks = 1024;
__device__ unsigned long long g_trace_chunk[4 * kTraceChunks];
#define MLA_TRACE_CHUNK(w, rank, kind, idx)                                              \
  do {                                                                                   \
    if ((w) == 0 && (rank) == 0 && (idx) < (uint32_t)kTraceChunks) {                     \
      unsigned long long t_;                                                             \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_));                                 \
      g_trace_chunk[(kind) * kTraceChunks + (idx)] = t_;                                 \
    }                                                                                    \
  } while (0)
#else
#define MLA_TRACE_EV(w, rank, kind, step) do {} while (0)
#define MLA_TRACE_CHUNK(w, rank, kind, idx) do {} while (0)
#define MLA_TRACE_CTA(k) do {} while (0)
#endif
enum { EV_QK_START = 0, EV_QK_END, EV_PV_START, EV_PV_END, EV_S_READY, EV_P_DONE, EV_PBUF_FREE, EV_LOAD,
       EV_PASS1, EV_PASS2, EV_SYNC1, EV_LD0, EV_LD1, EV_LD2, EV_LD3 };

// Sequential walk over a worker's page groups: sequence b, first page and
// page count of the group (1..4), first-group-of-segment flag, segment index.
struct GroupCursor {
  int b, page, pe, npages, seg;
  bool first;
  int64_t g1;
  __device__ __forceinline__ void set_group() { npages = min(kGroupPages, pe - page); }
  // returns false when the worker has no pages
  __device__ __forceinline__ bool init(const RunParams& p, int w) {
    const int64_t g0 = worker_page_start(w, p.cum, p.B, p.W);
    g1 = worker_page_start(w + 1, p.cum, p.B, p.W);
    if (g0 >= g1) return false;
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cum[mid] <= g0) lo = mid; else hi = mid - 1;
    }
    b = lo;
    page = (int)(g0 - p.cum[b]);
    pe = (int)(min(p.cum[b + 1], g1) - p.cum[b]);
    seg = 0;
    first = true;
    set_group();
    return true;
  }
  // advances to the next group; returns false after the last one
  __device__ __forceinline__ bool next(const RunParams& p) {
    page += npages;
    first = false;
    if (page >= pe) {
      if (b + 1 >= p.B || p.cum[b + 1] >= g1) return false;
      ++b;
      ++seg;
      page = 0;
      pe = (int)(min(p.cum[b + 1], g1) - p.cum[b]);
      first = true;
    }
    set_group();
    return true;
  }
  __device__ __forceinline__ bool last_of_segment() const { return page + npages >= pe; }
};

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk16) {
  return row * 128 + ((chunk16 ^ (row & 7)) << 4);
}

template <int S, int R, bool kSkip = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_of<S>(), 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_q, RunParams p) {
  using namespace ptx;
  using L = Smem<S, R>;
  using C = Cfg<S, R>;
  using Wd = Width<R>;
  static_assert(S == 1 || R == 512, "two shards in one launch split r = 512");
  static_assert(!kSkip || S == 1, "threshold skipping: one latent shard");
  constexpr int kChunks = Wd::kChunks;
  extern __shared__ uint8_t smem_raw[];
  MLA_TRACE_CTA(0);

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t rank = cluster_ctarank();
  const int w = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return base + L::bars + 8u * i; };
  auto leader_bar = [&](int i) -> uint32_t { return map_to_cta(bar(i), 0); };
  // arrival on a leader-owned barrier: CTA-local release on the leader itself
  auto arrive_leader = [&](int i) {
    if (rank == 0) mbar_arrive_local(bar(i)); else mbar_arrive_cluster(leader_bar(i));
  };
  auto expect_leader = [&](int i, uint32_t bytes) {
    if (rank == 0) mbar_arrive_expect_tx_local(bar(i), bytes);
    else mbar_arrive_expect_tx_cluster(leader_bar(i), bytes);
  };
  auto commit_both = [&](int i) {
    tc_commit<2>(bar(i));
    tc_commit<2>(map_to_cta(bar(i), 1));
  };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc + 8);
  // threshold skipping: votes [group parity][CTA rank] (nonzero: some row of
  // that CTA keeps the group)
  volatile uint32_t* votes = reinterpret_cast<volatile uint32_t*>(gbase + L::misc + 16);
  auto pair_keeps = [&](int gi) { return (votes[2 * (gi & 1)] | votes[2 * (gi & 1) + 1]) != 0; };
  float* xch = reinterpret_cast<float*>(gbase + L::xch);

  if (threadIdx.x == 0) {
    uint32_t counts[B_COUNT];
    for (int i = 0; i < B_COUNT; ++i) counts[i] = 1;

    for (int i = 0; i < kChunks; ++i) counts[B_QC_FULL + i] = 2;
    for (int i = 0; i < 6; ++i) counts[B_QK_FULL + i] = 2;
    for (int i = 0; i < 6; ++i) counts[B_V_FULL + i] = 2;
    counts[B_S_FREE] = counts[B_S_FREE + 1] = 8;
    counts[B_P_FULL] = counts[B_P_FULL_1] = 8;
    counts[B_P_FULL_HI] = counts[B_P_FULL_HI_1] = 4;
    counts[B_O_FREE] = 8 * S;  // every softmax warp of both CTAs
    counts[B_VSEEN] = counts[B_VSEEN + 1] = 2;  // both CTAs' V producers
    for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), counts[i]);
    fence_mbarrier_init_cluster();
    *abort_flag = 0;
  }
  if (warp == 1) {
    tmem_alloc<2>(base + L::misc, kTmemCols);
    tmem_relinquish<2>();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // the setup above overlaps the previous kernel; from here on its results
  // (the absorbed queries, the page prefix sums) are read
  grid_launch_dependents();
  grid_dependency_wait();
  const bool run = *p.lengths_ok != 0;  // uniform across the pair
  MLA_TRACE_CTA(1);

  auto fail = [&](int code) {
    record_error(p.status, code);
    *abort_flag = 1;
  };
  // Row coordinate of page `page` of sequence b in the pool viewed as
  // [num_blocks * 64, 576]; pages past the group's end and invalid block ids
  // read past the tensor (TMA fills zeros) and are masked by the softmax.
  const int oob_row = (int)(p.num_blocks * 64);
  auto page_row = [&](int b, int page, bool exists) -> int {
    if (!exists) return oob_row;
    const int32_t blk = p.block_table[(int64_t)b * p.bt_stride + page];
    if (blk < 0 || blk >= p.num_blocks) {
      record_error(p.status, MLA_ERR_BOUNDS);
      return oob_row;
    }
    return blk * 64;
  };

  if (!run) {
    // invalid lengths (reported by the length scan): nothing to do
  } else if (warp == 0) {
    // --------------------------------------------- Q and QK chunk producer --
    // lanes 0 and 1: lane k loads this CTA's page 2 rank + k of every chunk
    if (lane < kIssueLanes) {
      if (lane == 0) {
        prefetch_tmap(&tm_kv);
        prefetch_tmap(&tm_q);
      }
      GroupCursor g;
      bool ok = true;
      bool have = g.init(p, w);
      uint32_t cc = 0;  // chunk counter over all groups
      for (int gi = 0; have && ok; ++gi) {
        const int yq = g.b * p.rows + 64 * (int)rank;  // this CTA's query rows of the segment
        const int pg = 2 * (int)rank + lane;            // this lane's page within the group
        const int y = page_row(g.b, g.page + pg, pg < g.npages);
        if (lane == 0) MLA_TRACE_EV(w, rank, EV_LOAD, gi);
        for (int pos = 0; pos < kChunks && ok; ++pos, ++cc) {
          const int kc = chunk_at<S>(pos);
          const int slot = cc % C::kQkSlots;
          if (cc >= (uint32_t)C::kQkSlots)
            ok = mbar_wait(bar(B_QK_FREE + slot), ((cc / C::kQkSlots) - 1) & 1, p.wait_limit_ns);
          if (!ok) break;
          if (g.first && lane == 1) {
            // New segment: reload query chunk kc. Its last reader, chunk kc of
            // the previous group (kChunks items back), is done: the QK issuer
            // consumes items in order and item cc - kQkSlots has been released.
            expect_leader(B_QC_FULL + kc, kQChunkBytes);
            tma_load_2d_pair(base + L::q + kc * kQChunkBytes, &tm_q, 64 * kc, yq,
                             leader_bar(B_QC_FULL + kc));
          }
          if (lane == 0) expect_leader(B_QK_FULL + slot, kSlotBytes);
          tma_load_2d_pair(base + L::qk + slot * kSlotBytes + lane * (kSlotBytes / 2), &tm_kv, 64 * kc, y,
                           leader_bar(B_QK_FULL + slot));
          if (lane == 0) MLA_TRACE_CHUNK(w, rank, 0, cc);
        }
        if (ok) have = g.next(p);
      }
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------ V chunk producer --
    // lanes 0 and 1: lane k loads latent chunk 4 nb + 2 rank + k of every page
    if (lane < kIssueLanes) {
      GroupCursor g;
      bool ok = true;
      bool have = g.init(p, w);
      uint32_t vc = 0;  // V slot counter
      int gi = 0;
      while (have && ok) {
        bool keep = true;
        if constexpr (kSkip) {
          // the pair's decision for this group: a skipped group's V is not loaded
          ok = mbar_wait(bar(B_DECIDE + (gi & 1)), (gi >> 1) & 1, p.wait_limit_ns);
          ok = __all_sync(0x3u, ok);
          if (!ok) break;
          keep = pair_keeps(gi);
          __syncwarp(0x3u);
          if (lane == 0) {  // both CTAs' publishers may now reuse this vote slot
            mbar_arrive_local(bar(B_VSEEN + (gi & 1)));
            mbar_arrive_cluster(map_to_cta(bar(B_VSEEN + (gi & 1)), rank ^ 1u));
          }
        }
        ++gi;
        int rows[kGroupPages];
        for (int q = 0; q < kGroupPages; ++q) rows[q] = page_row(g.b, g.page + q, q < g.npages);
        for (int i = 0; i < kGroupPages * Wd::kNBlocks && ok && keep; ++i, ++vc) {
          int q, nb;
          v_item<S, Wd::kNBlocks>(i, q, nb);
          const int slot = vc % C::kVSlots;
          if (vc >= (uint32_t)C::kVSlots)
            ok = mbar_wait(bar(B_V_FREE + slot), ((vc / C::kVSlots) - 1) & 1, p.wait_limit_ns);
          if (!ok) break;
          if (lane == 0) expect_leader(B_V_FULL + slot, kSlotBytes);
          const int chunk = 4 * nb + 2 * (int)rank + lane;
          tma_load_2d_pair(base + L::v + slot * kSlotBytes + lane * (kSlotBytes / 2), &tm_kv, 64 * chunk,
                           rows[q], leader_bar(B_V_FULL + slot));
          if (lane == 0) MLA_TRACE_CHUNK(w, rank, 2, vc);
        }
        if (ok) have = g.next(p);
      }
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ QK MMA issuer --
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, 256, 0, 0);
      // descriptors of offset 0; the 14-bit start-address field (address >> 4)
      // advances by adding the byte offset >> 4
      const uint64_t q_desc0 = smem_desc_sw128(base + L::q, 16, 1024);
      const uint64_t qk_desc0 = smem_desc_sw128(base + L::qk, 16, 1024);
      bool ok = true;
      uint32_t cc = 0;
      GroupCursor g;
      bool have = g.init(p, w);
      for (int gi = 0; have && ok; ++gi) {
        // one shard: S buffer sb must be free; two shards (one buffer, a
        // 128-column tile per shard): shard 0's tile now, shard 1's at the RoPE chunk
        const int sb = gi % C::kSBufs;
        if (ok && gi >= C::kSBufs) ok = mbar_wait(bar(B_S_FREE + sb), ((gi / C::kSBufs) - 1) & 1, p.wait_limit_ns);
        if (!ok) break;
        MLA_TRACE_EV(w, 0, EV_QK_START, gi);
        const uint32_t s_tmem = tbase + sb * 128 * S;
        for (int pos = 0; pos < kChunks && ok; ++pos, ++cc) {
          const int kc = chunk_at<S>(pos);
          const int slot = cc % C::kQkSlots;
          if (g.first) ok = mbar_wait(bar(B_QC_FULL + kc), g.seg & 1, p.wait_limit_ns);  // this segment's query chunk
          ok = ok && mbar_wait(bar(B_QK_FULL + slot), (cc / C::kQkSlots) & 1, p.wait_limit_ns);
          if (!ok) break;
          MLA_TRACE_CHUNK(w, 0, 1, cc);
          tc_fence_after();
          const uint64_t ad = q_desc0 + (uint64_t)(kc * (kQChunkBytes >> 4));
          const uint64_t bd = qk_desc0 + (uint64_t)((slot * kSlotBytes) >> 4);
          auto qk_mma = [&](int shard, bool first_k) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16<2>(s_tmem + 128 * shard, ad + (uint64_t)(2 * ks), bd + (uint64_t)(2 * ks),
                         idesc_qk, (first_k && ks == 0) ? 0u : 1u);
          };
          if constexpr (S == 1) {
            qk_mma(0, kc == 0);
          } else {
            // shard 0: chunks 0-3 and the RoPE chunk, which completes it
            if (kc < 4 || kc == 8) qk_mma(0, kc == 0);
            if (kc == 8) {
              commit_both(B_S_FULL + 0);
              if (gi >= 1) ok = mbar_wait(bar(B_S_FREE + 1), (gi - 1) & 1, p.wait_limit_ns);
              if (!ok) break;
              tc_fence_after();
            }
            // shard 1: the RoPE chunk first, then chunks 4-7
            if (kc >= 4) qk_mma(1, kc == 8);
          }
          commit_both(B_QK_FREE + slot);
        }
        if (!ok) break;
        MLA_TRACE_EV(w, 0, EV_QK_END, gi);
        commit_both(B_S_FULL + (S == 2 ? 1 : sb));
        have = g.next(p);
      }
      tc_commit<2>(bar(B_FINAL_QK));
      if (!mbar_wait(bar(B_FINAL_QK), 0, p.wait_limit_ns)) ok = false;
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 7) {
    // ------------------------------------------------------ PV MMA issuer --
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      const uint64_t p_desc0 = smem_desc_sw128(base + L::p, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(base + L::v, kSlotBytes / 2, 1024);
      bool ok = true;
      uint32_t vc = 0;
      GroupCursor g;
      bool have = g.init(p, w);
      int n_groups = 0, n_skipped = 0;
      for (int gi = 0; have && ok; ++gi) {
        ok = mbar_wait(bar(B_P_FULL), gi & 1, p.wait_limit_ns);
        if (ok && g.first && g.seg > 0) ok = mbar_wait(bar(B_O_FREE), (g.seg - 1) & 1, p.wait_limit_ns);
        if (!ok) break;
        MLA_TRACE_EV(w, 0, EV_PV_START, gi);
        // threshold skipping: both CTAs' softmax warps read the pair's decision
        // before arriving on B_P_FULL, so it is final here
        bool keep = true;
        if constexpr (kSkip) {
          keep = pair_keeps(gi);
          ++n_groups;
          n_skipped += keep ? 0 : 1;
        }
        // A shard's P buffer holds pages 0, 1, then pages 2, 3: PV waits for
        // each half as it is written and releases it once its MMAs are issued
        // (the commit completes when they are done). Items in V ring order.
        if constexpr (S == 1) {
          // page-major, both N blocks of a page (kept in this form: one loop
          // over the items in ring order measured ~10% slower per step)
          for (int q = 0; q < kGroupPages && ok; ++q) {
            if (q == 2) {
              ok = mbar_wait(bar(B_P_FULL_HI), gi & 1, p.wait_limit_ns);
              if (!ok) break;
            }
            for (int nb = 0; nb < Wd::kNBlocks && ok && keep; ++nb, ++vc) {
              const int slot = vc % C::kVSlots;
              ok = mbar_wait(bar(B_V_FULL + slot), (vc / C::kVSlots) & 1, p.wait_limit_ns);
              if (!ok) break;
              MLA_TRACE_CHUNK(w, 0, 3, vc);
              tc_fence_after();
              const uint64_t pd = p_desc0 + (uint64_t)(((q & 1) * kPChunkBytes) >> 4);
              const uint64_t vd = v_desc0 + (uint64_t)((slot * kSlotBytes) >> 4);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_f16<2>(tbase + kTmemO + 128 * nb, pd + (uint64_t)(2 * ks),
                           vd + (uint64_t)(128 * ks), idesc_pv,
                           (g.first && q == 0 && ks == 0) ? 0u : 1u);
              commit_both(B_V_FREE + slot);
            }
            if (q == 1) commit_both(B_P_FREE_LO);
          }
          if (ok) commit_both(B_P_FREE_HI);
        } else {
          auto pv_item = [&](int q, int shard) {  // N block nb = shard
            const int nb = shard;
            const int slot = vc % C::kVSlots;
            ok = mbar_wait(bar(B_V_FULL + slot), (vc / C::kVSlots) & 1, p.wait_limit_ns);
            if (!ok) return;
            MLA_TRACE_CHUNK(w, 0, 3, vc);
            tc_fence_after();
            const uint64_t pd = p_desc0 + (uint64_t)((shard * C::kPShard + (q & 1) * kPChunkBytes) >> 4);
            const uint64_t vd = v_desc0 + (uint64_t)((slot * kSlotBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16<2>(tbase + kTmemO + 128 * nb, pd + (uint64_t)(2 * ks),
                         vd + (uint64_t)(128 * ks), idesc_pv,
                         (g.first && q == 0 && ks == 0) ? 0u : 1u);
            commit_both(B_V_FREE + slot);
            ++vc;
          };
          // page half, then shard (= N block), then the half's two pages
          for (int hf = 0; hf < 2 && ok; ++hf) {
            for (int sh = 0; sh < 2 && ok; ++sh) {
              if (hf + sh > 0) {
                ok = mbar_wait(bar(hf ? bar_p_full_hi(sh) : bar_p_full(sh)), gi & 1, p.wait_limit_ns);
                if (!ok) break;
              }
              for (int qq = 0; qq < 2 && ok; ++qq) pv_item(2 * hf + qq, sh);
              if (ok) commit_both(hf ? bar_p_free_hi(sh) : bar_p_free_lo(sh));
            }
          }
        }
        if (!ok) break;
        MLA_TRACE_EV(w, 0, EV_PV_END, gi);
        commit_both(B_PV_DONE);
        have = g.next(p);
      }
      tc_commit<2>(bar(B_FINAL_PV));
      if (!mbar_wait(bar(B_FINAL_PV), 0, p.wait_limit_ns)) ok = false;
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
      if constexpr (kSkip) {
        atomicAdd(p.skip_stats, n_skipped);
        atomicAdd(p.skip_stats + 1, n_groups);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps --
    // Every softmax thread executes the same sequence of named barriers
    // whatever happens: after a failed (timed-out) wait the flag `ok` turns
    // false for the whole warp and the remaining groups only skip their work.
    // two shards: one softmax warpgroup per shard (warps 3-6 and 8-11), each
    // with its own named barrier; one shard: warps 3-6
    const int my_shard = (S == 2 && warp >= 8) ? 1 : 0;
    const int lq = (warp & 3) * 32 + lane;         // tensor-memory lane of this thread
    const int half = lq >> 6;                      // token half: group tokens [128 half, +128)
    const int rloc = lq & 63;                      // row within this CTA's 64
    const int row = 64 * (int)rank + rloc;         // query row within the sequence
    const bool row_real = row < p.rows;
    const int t_row = row_real ? row / p.H : 0;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    bool ok = true;
    float* xl = xch + 2 * S * 128;                 // [S][128]
    const uint32_t sync_id = 1u + 2u * (uint32_t)my_shard;
    auto named_sync = [sync_id] { asm volatile("bar.sync %0, 128;" :: "r"(sync_id) : "memory"); };
    auto wait = [&](int b, uint32_t parity) {
      if (ok && *abort_flag) ok = false;
      if (ok) ok = mbar_wait(bar(b), parity, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
    };
    GroupCursor g;
    bool have = g.init(p, w);
    int gi = 0;
    float m_run = -INFINITY, l_run = 0.f;  // this thread's row: running max (log2 units) and sum
    float mm = -INFINITY;  // threshold skipping: the row's true running max of the segment (log2 units)
    while (have) {
      if (g.first) {
        m_run = -INFINITY;
        l_run = 0.f;
        mm = -INFINITY;
      }
      const int sb = gi % C::kSBufs;
      float* xmax = xch + (gi & 1) * S * 128;      // this group's [S][128] row maxima
      const int64_t L = p.seq_lens[g.b];
      // this thread's 128 tokens: group pages 2 half, 2 half + 1; the visible
      // ones are the first nvis (pages past the group's end or past the causal
      // limit are masked); nvis is uniform across the warp
      const int64_t key0 = (int64_t)(g.page + 2 * half) * 64;
      const int64_t lim = row_real ? L - p.Lq + t_row : -1;  // last visible key
      int64_t nv = lim - key0 + 1;
      const int64_t in_group = (int64_t)(g.npages - 2 * half) * 64;
      nv = nv > in_group ? in_group : nv;
      nv = nv < 0 ? 0 : (nv > 128 ? 128 : nv);
      const int nvis = (int)nv;

      if constexpr (S == 1) {
        wait(B_S_FULL + sb, (gi / C::kSBufs) & 1);
        if (lq == 0) MLA_TRACE_EV(w, rank, EV_S_READY, gi);
        if (ok) tc_fence_after();
      }
#pragma unroll 1
      for (int s = my_shard; s <= my_shard; ++s) {  // this warpgroup's shard
        if constexpr (S == 2) {
          // two shards: each tile is complete (and released) on its own
          wait(B_S_FULL + s, gi & 1);
          if (lq == 0 && s == 0) MLA_TRACE_EV(w, rank, EV_S_READY, gi);
          if (ok) tc_fence_after();
        }
        // The thread's 128 scores of shard s. One shard: one pass over tensor
        // memory into registers. Two shards (a warpgroup each, 384 threads,
        // 168 registers): two passes in 32-column pieces, for the row max and
        // then for P, so that no 128-score array is live; the tile is released
        // after the second.
        const uint32_t s_addr = tbase + lane_off + sb * 128 * S + 128 * s;
        constexpr int kRegScores = S == 2 ? 1 : 128;
        uint32_t r[kRegScores];
        float mx0 = -INFINITY, mx1 = -INFINITY;
        if constexpr (S == 2) {
          if (ok) {
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 64) {
              uint32_t v[64];
              tmem_ld32(s_addr + c0, *reinterpret_cast<uint32_t(*)[32]>(v));
              tmem_ld32(s_addr + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
              tmem_wait_ld();
              // masked keys (past the group or the causal limit) count as -inf
              if (nvis >= 128) {
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                  mx0 = fmaxf(mx0, __uint_as_float(v[k]));
                  mx1 = fmaxf(mx1, __uint_as_float(v[k + 1]));
                }
              } else {
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                  mx0 = fmaxf(mx0, c0 + k < nvis ? __uint_as_float(v[k]) : -INFINITY);
                  mx1 = fmaxf(mx1, c0 + k + 1 < nvis ? __uint_as_float(v[k + 1]) : -INFINITY);
                }
              }
            }
          }
        } else {
          if (ok) {
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32)
              tmem_ld32(s_addr + c0, *reinterpret_cast<uint32_t(*)[32]>(r + c0));
            tmem_wait_ld();
          }
          // every score of this S buffer is in registers: QK may reuse it
          if (ok) tc_fence_before();
          __syncwarp();
          if (ok && lane == 0 && !p.withhold_s_free) arrive_leader(B_S_FREE + sb);
          // masked keys (past the group or the causal limit) become -inf: they
          // drop out of the max and 2^-inf = 0 in the sum and in P
          if (nvis < 128) {
#pragma unroll
            for (int j = 0; j < 128; ++j)
              if (j >= nvis) r[j] = 0xff800000u;
          }
          if (ok) {
#pragma unroll
            for (int j = 0; j < 128; j += 2) {
              mx0 = fmaxf(mx0, __uint_as_float(r[j]));
              mx1 = fmaxf(mx1, __uint_as_float(r[j + 1]));
            }
          }
        }
        const float mt_own = fmaxf(mx0, mx1) * p.scale_log2;
        xmax[s * 128 + lq] = mt_own;
        if (lq == 0 && s == 0) MLA_TRACE_EV(w, rank, EV_PASS1, gi);
        named_sync();
        // row max over both token halves (the other half lives in lane lq ^ 64)
        const float mt = fmaxf(mt_own, xmax[s * 128 + (lq ^ 64)]);
        // Threshold skipping (BLASST abstract on the kk6lht.com listing: a fixed
        // threshold against the online softmax's running max marks negligible
        // scores; their exp, value loads and PV are skipped). A row keeps the
        // group if its maximum reaches its running max + skip_log2 (or it is the
        // row's first visible group); the group is skipped when no row of the
        // pair keeps it. Votes: a barrier reduction over this CTA's 128 softmax
        // threads, exchanged with the peer by an async store on its barrier.
        bool skip = false;
        if constexpr (kSkip) {
          const bool keep_row = row_real && mt != -INFINITY && (mm == -INFINITY || mt >= mm + p.skip_log2);
          mm = fmaxf(mm, mt);
          uint32_t any_keep;
          asm volatile("{\n\t.reg .pred pk, pa;\n\tsetp.ne.u32 pk, %1, 0;\n\t"
                       "barrier.cta.red.or.pred pa, 2, 128, pk;\n\tselp.u32 %0, 1, 0, pa;\n\t}"
                       : "=r"(any_keep) : "r"((uint32_t)keep_row) : "memory");
          const int par = gi & 1;
          if (lq == 0) {
            // the vote slot of group gi - 2 is free once both V producers read it
            if (ok && gi >= 2) ok = mbar_wait(bar(B_VSEEN + par), ((gi - 2) >> 1) & 1, p.wait_limit_ns);
            if (ok) {
              votes[2 * par + rank] = any_keep;
              const uint32_t slot = smem_u32(const_cast<uint32_t*>(votes + 2 * par + rank));
              st_async_b32(map_to_cta(slot, rank ^ 1u), any_keep, map_to_cta(bar(B_DECIDE + par), rank ^ 1u));
              mbar_arrive_expect_tx_local(bar(B_DECIDE + par), 4);
            }
          }
          wait(B_DECIDE + par, (gi >> 1) & 1);
          skip = ok && !pair_keeps(gi);
        }
        float mu = m_run;
        if (!skip && (m_run == -INFINITY || mt > m_run + kRescaleThreshold)) mu = fmaxf(mt, m_run);
        float alpha = 1.f;
        const bool rescale = mu != m_run && m_run != -INFINITY;
        if (rescale) alpha = ex2_approx(m_run - mu);
        m_run = mu;
        // P = 2^(score * scale - m) in bf16 pairs, row sum in four partial sums
        // (a row that has seen no key yet keeps m = -inf, all its scores are
        // -inf and P = 0)
        uint32_t pk[64];
        float ps0 = 0.f, ps1 = 0.f, ps2 = 0.f, ps3 = 0.f;
        const float nmu = mu == -INFINITY ? 0.f : -mu;
        auto p_of4 = [&](int j, float x0, float x1, float x2, float x3) {
          const float p0 = ex2_approx(fmaf(x0, p.scale_log2, nmu));
          const float p1 = ex2_approx(fmaf(x1, p.scale_log2, nmu));
          const float p2 = ex2_approx(fmaf(x2, p.scale_log2, nmu));
          const float p3 = ex2_approx(fmaf(x3, p.scale_log2, nmu));
          ps0 += p0; ps1 += p1; ps2 += p2; ps3 += p3;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(p0, p1);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(p2, p3);
          pk[j >> 1] = *reinterpret_cast<uint32_t*>(&h0);
          pk[(j >> 1) + 1] = *reinterpret_cast<uint32_t*>(&h1);
        };
        if constexpr (S == 2) {
          // second pass over the tile, 32 columns at a time; then release it
          if (ok) {
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
              uint32_t v[32];
              tmem_ld32(s_addr + c0, v);
              tmem_wait_ld();
              if (nvis >= 128) {
#pragma unroll
                for (int k = 0; k < 32; k += 4)
                  p_of4(c0 + k, __uint_as_float(v[k]), __uint_as_float(v[k + 1]), __uint_as_float(v[k + 2]),
                        __uint_as_float(v[k + 3]));
              } else {
#pragma unroll
                for (int k = 0; k < 32; k += 4) {
                  const int j = c0 + k;
                  p_of4(j, j < nvis ? __uint_as_float(v[k]) : -INFINITY,
                        j + 1 < nvis ? __uint_as_float(v[k + 1]) : -INFINITY,
                        j + 2 < nvis ? __uint_as_float(v[k + 2]) : -INFINITY,
                        j + 3 < nvis ? __uint_as_float(v[k + 3]) : -INFINITY);
                }
              }
            }
            tc_fence_before();
          }
          __syncwarp();
          if (ok && lane == 0 && !p.withhold_s_free) arrive_leader(B_S_FREE + s);
        } else if (!skip) {
#pragma unroll
          for (int j = 0; j < 128; j += 4)
            p_of4(j, __uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                  __uint_as_float(r[j + 3]));
        }
        l_run = l_run * alpha + ((ps0 + ps1) + (ps2 + ps3));
        if (lq == 0 && s == 0) MLA_TRACE_EV(w, rank, EV_PASS2, gi);
        auto rescale_o = [&](int c0, int ncols) {
          tc_fence_after();
#pragma unroll 1
          for (int c = c0; c < c0 + ncols; c += 32) {
            uint32_t o[32];
            tmem_ld32(tbase + lane_off + kTmemO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(tbase + lane_off + kTmemO + c, o);
          }
          tmem_wait_st();
        };
        // P -> shared memory, K-major 128-byte swizzle: row rloc, this
        // thread's 128 tokens as two 64-token chunks, 16-byte units 0..7 each
        auto write_p = [&](uint8_t* chunk0) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            uint8_t* chunk = chunk0 + t * kPChunkBytes;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(chunk + sw128(rloc, u)) =
                  make_uint4(pk[32 * t + 4 * u], pk[32 * t + 4 * u + 1],
                             pk[32 * t + 4 * u + 2], pk[32 * t + 4 * u + 3]);
          }
        };
        // Shard s's P buffer: pages 0, 1 (this half 0 thread's tokens) go in
        // once the previous group's PV is done with pages 2, 3; pages 2, 3
        // (half 1) replace them once this group's PV is done with pages 0, 1.
        // Shard s's O columns are rescaled (after the previous group's PV)
        // before this group's PV adds to them; both halves signal that
        // through the shard's P_FULL barrier.
        if (!g.first && __any_sync(0xffffffffu, rescale)) wait(B_PV_DONE, (gi - 1) & 1);
        if (ok && !g.first && __any_sync(0xffffffffu, rescale))
          rescale_o((Wd::kOCols / S) * s, Wd::kOCols / S);
        if (half == 0) {
          if (gi >= 1) wait(bar_p_free_hi(s), (gi - 1) & 1);
        } else {
          if (ok) tc_fence_before();
          __syncwarp();
          if (ok && lane == 0) arrive_leader(bar_p_full(s));
          wait(bar_p_free_lo(s), gi & 1);
        }
        if (lq == 0 && s == 0) MLA_TRACE_EV(w, rank, EV_PBUF_FREE, gi);
        if (ok && !skip) {
          write_p(gbase + L::p + s * C::kPShard);
          fence_proxy_async_smem();
          tc_fence_before();
        }
        __syncwarp();
        if (ok && lane == 0) arrive_leader(half == 0 ? bar_p_full(s) : bar_p_full_hi(s));
      }
      if (lq == 0) MLA_TRACE_EV(w, rank, EV_P_DONE, gi);

      if (g.last_of_segment()) {
        // ---- segment epilogue: O / l and log2-sum-exp of this segment
        wait(B_PV_DONE, gi & 1);
        if (lq == 0) MLA_TRACE_EV(w, rank, EV_SYNC1, gi);
        if (ok) tc_fence_after();
        // (this warpgroup's shard: its l, log2-sum-exp and O columns)
        const int s = my_shard;
        xl[s * 128 + lq] = l_run;
        named_sync();
        const int64_t slot = w + g.b;
        const float lt = l_run + xl[s * 128 + (lq ^ 64)];
        const float iv = lt > 0.f ? 1.f / lt : 0.f;
        if (ok && half == 0 && row_real)
          p.lse_part[(slot * p.rows + row) * S + s] = lt > 0.f ? m_run + log2f(lt) : kEmptyLse;
        if (ok) {
          // O / l goes out as fp16 (the combine kernel reads it back once).
          // A warp holds 32 consecutive rows; per round it loads 64 columns of
          // them from tensor memory and transposes the 32 x 128-byte block
          // through 4 KB of the P buffer (free: this group's PV has completed),
          // so that each store instruction writes four whole 128-byte row
          // segments. Swizzle: 16-byte unit u of staged row r sits at u ^ (r & 7).
          uint8_t* stage = gbase + L::p + s * C::kPShard + (warp & 3) * 4096;
          const int rbase = 64 * (int)rank + 32 * ((warp & 3) & 1);  // row of lane 0
          const int j = lane & 7;
          __half* oh = reinterpret_cast<__half*>(p.o_part);
          constexpr int kCols = (int)Wd::kOCols / S;  // this shard's O columns
#pragma unroll 1
          for (int c = kCols * s; c < kCols * (s + 1); c += 64) {
            uint32_t o[64];
            tmem_ld32(tbase + lane_off + kTmemO + c, *reinterpret_cast<uint32_t(*)[32]>(o));
            tmem_ld32(tbase + lane_off + kTmemO + c + 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32));
            tmem_wait_ld();
            const int nb = c >> 7;
            const int col0 = 256 * nb + 128 * half + (c & 127);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              uint32_t hv[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                __half2 h2 = __floats2half2_rn(__uint_as_float(o[8 * u + 2 * k]) * iv,
                                               __uint_as_float(o[8 * u + 2 * k + 1]) * iv);
                hv[k] = *reinterpret_cast<uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(stage + lane * 128 + 16 * (u ^ (lane & 7))) =
                  make_uint4(hv[0], hv[1], hv[2], hv[3]);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = (lane >> 3) + 4 * i;
              const uint4 v = *reinterpret_cast<const uint4*>(stage + r * 128 + 16 * (j ^ (r & 7)));
              if (rbase + r < p.rows)
                *reinterpret_cast<uint4*>(oh + (slot * p.rows + rbase + r) * (int64_t)p.r + col0 + 8 * j) = v;
            }
            __syncwarp();
          }
          tc_fence_before();
          __threadfence();  // this thread's partial rows, before the CTA's segment-done count
        }
        named_sync();  // xl and the O reads of the warpgroup's four warps are done
        // one count per CTA and shard: the combine waits for 2 S per segment
        if (ok && lq == 0) publish_segment_half(p.seg_done + g.b);
        if (lq == 0) MLA_TRACE_EV(w, rank, EV_LD0, gi);
        __syncwarp();
        if (ok && lane == 0) arrive_leader(B_O_FREE);
      }
      ++gi;
      have = g.next(p);
    }
    if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
  }
  __syncwarp();

  MLA_TRACE_CTA(2);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<2>(tbase, kTmemCols);
  MLA_TRACE_CTA(3);
}

// ------------------------------------------------------------------ host ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 2-D bf16 row-major [rows, width] (width = r + d_rope) with a (64 columns x
// 64 rows) 128B-swizzled box.
inline bool make_rows_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t width = kWidth) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)width * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

namespace tc {
template <int S, int R, bool kSkip = false>
inline cudaError_t launch_decode_variant(const RunParams& p, const CUtensorMap& tm_kv, const CUtensorMap& tm_q,
                                         cudaStream_t stream, bool pdl) {
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(decode_tc_kernel<S, R, kSkip>),
                                    (int)Smem<S, R>::alloc);
  if (e != cudaSuccess) return e;
  return launch_dependent_opt(pdl, decode_tc_kernel<S, R, kSkip>, dim3(2 * p.W), dim3(threads_of<S>()), Smem<S, R>::alloc,
                              stream, tm_kv, tm_q, p);
}
}  // namespace tc

// r = 512 with one or two latent shards, or r = 256 with one (a TPLA shard per GPU)
// skip: the threshold-skipping variant (r = 512, one shard; p.skip_log2, p.skip_stats)
inline cudaError_t launch_tc_decode(const RunParams& p, cudaStream_t stream, bool pdl = true, bool skip = false) {
  const uint64_t width = (uint64_t)p.r + p.dr;
  CUtensorMap tm_kv, tm_q;
  if (!tc::make_rows_map(&tm_kv, p.kv, (uint64_t)p.num_blocks * 64, width)) return cudaErrorInvalidValue;
  if (!tc::make_rows_map(&tm_q, p.q, (uint64_t)p.B * p.rows, width)) return cudaErrorInvalidValue;
  if (skip) {
    if (p.r != 512 || p.S != 1) return cudaErrorInvalidValue;
    return tc::launch_decode_variant<1, 512, true>(p, tm_kv, tm_q, stream, pdl);
  }
  if (p.r == 256 && p.S == 1) return tc::launch_decode_variant<1, 256>(p, tm_kv, tm_q, stream, pdl);
  if (p.r != 512) return cudaErrorInvalidValue;
  return p.S == 1 ? tc::launch_decode_variant<1, 512>(p, tm_kv, tm_q, stream, pdl)
                  : tc::launch_decode_variant<2, 512>(p, tm_kv, tm_q, stream, pdl);
}

}  // namespace mla
