// tcgen05 (5th-generation tensor core) split-KV decode kernel for the bf16
// workloads: r = 512 latent columns, 64 RoPE columns, 64-token pages,
// up to 128 query rows (heads x query tokens) per sequence.
//
// One CTA pair (a cluster of 2 on one TPC) per worker; the pair walks the
// worker's page range (split segments, see common.cuh). Per 64-token page:
//
//   QK  (cta_group::2, M = 128 rows, N = 64 tokens, K = 576):
//       S = Q . [cKV || k_rope]^T. CTA c holds query rows [64c, 64c+64) of Q in
//       shared memory and tokens [32c, 32c+32) of the page; each CTA's tensor
//       memory receives its 64 rows x all 64 tokens, folded over the 128
//       lanes (lanes 0-63: tokens 0-31, lanes 64-127: tokens 32-63).
//   softmax (4 warps per CTA, fp32): online max / sum per row in the log2
//       domain; the max is only moved (and O rescaled) when it grows by more
//       than 2^8, which keeps every P value in [0, 256] and makes the rescale
//       of O rare. P is written in bf16 to shared memory.
//   PV  (cta_group::2, M = 128 rows, N = 256 latent columns, K = 64 tokens,
//       two N blocks): O_lat += P . cKV. The B operand (the cKV page, MN-major)
//       is split along N: CTA0 supplies latent chunks 4nb, 4nb+2 and CTA1 4nb+1,
//       4nb+3. Each CTA already holds its own 32 tokens of the page; after the
//       QK MMAs have read the stage, the 32 tokens of the other half of its
//       latent chunks are re-read from L2 into the slots it no longer needs.
//   TPLA (S = 2 shards): two S tiles per page (latent chunks 0-3 or 4-7, both
//       with the RoPE chunk), one softmax per shard, and PV N-block nb = shard nb.
//
// Each CTA's O accumulator covers its 64 rows x 512 latent columns (256 tensor
// memory columns). At the end of a split segment the softmax warps write
// O / l and log2-sum-exp per row into the workspace; the combine kernel
// merges the segments and applies W_UV.
//
// Sources: TPLA abstract (latent cache, shard-and-sum), TransMLA abstract
// (absorbed decode over the compressed cache), pith.science verdict record for
// 2502.07864 (shared multi-query RoPE key).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace mla {

constexpr bool kTcDecodeAvailable = true;

namespace tc {

constexpr int kWidth = 576;          // r + d_rope
constexpr int kChunks = 9;           // 64-column chunks of a row (8 latent + 1 rope)
constexpr int kStages = 3;
constexpr int kThreads = 192;        // warp 0 TMA, warp 1 MMA, warps 2-5 softmax
constexpr uint32_t kQChunkBytes = 64 * 128;            // 64 rows x 128 B
constexpr uint32_t kKvChunkBytes = 32 * 128;           // 32 rows x 128 B
constexpr uint32_t kQBytes = kChunks * kQChunkBytes;   // 72 KB
constexpr uint32_t kStageBytes = kChunks * kKvChunkBytes;  // 36 KB
constexpr uint32_t kPBytes = 64 * 128;                 // 64 rows x 64 tokens bf16
constexpr float kRescaleThreshold = 8.0f;              // log2 units

// tensor-memory columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;

template <int S>
struct Smem {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t kv = q + kQBytes;
  static constexpr uint32_t p = kv + kStages * kStageBytes;
  static constexpr uint32_t xch = p + 2 * S * kPBytes;          // float [2][S][128] + l [S][128]
  static constexpr uint32_t bars = xch + (2 * S * 128 + S * 128) * 4;
  static constexpr uint32_t nbars = 32;
  static constexpr uint32_t misc = bars + nbars * 8;             // tmem slot, flags
  static constexpr uint32_t total = misc + 64;
  static constexpr uint32_t alloc = total + 1024;                // alignment slack
};

// barrier indices
enum : int {
  B_Q_FULL = 0,                 // leader, count 2 (+tx)
  B_KV_FULL = 1,                // [3] leader, count 2 (+tx)
  B_V_FULL = 4,                 // [3] leader, count 2 (+tx)
  B_S_FREE = 7,                 // [2] leader, count 8
  B_P_FULL = 9,                 // [2] leader, count 8
  B_O_FREE = 11,                // leader, count 8
  B_QK_DONE = 12,               // [3] both, count 1 (MMA commit)
  B_STAGE_FREE = 15,            // [3] both, count 1
  B_S_FULL = 18,                // [2] both, count 1
  B_PV_DONE = 20,               // [2] both, count 1
  B_FINAL = 22,                 // leader, count 1
  B_COUNT = 23
};

// Optional event trace (compile with -DMLA_TRACE): SM clock of each role's
// per-step events for the first kTraceWorkers workers, read back on the host
// with mla_debug_trace_read(). Off in normal builds.
#ifdef MLA_TRACE
constexpr int kTraceWorkers = 4, kTraceKinds = 8, kTraceSteps = 64;
__device__ unsigned long long g_trace[kTraceWorkers * 2 * kTraceKinds * kTraceSteps];
#define MLA_TRACE_EV(w, rank, kind, step)                                                \
  do {                                                                                   \
    if ((w) < kTraceWorkers && (step) < kTraceSteps) {                                   \
      unsigned long long t_;                                                             \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_));                                 \
      g_trace[(((w) * 2 + (rank)) * kTraceKinds + (kind)) * kTraceSteps + (step)] = t_;   \
    }                                                                                    \
  } while (0)
#else
#define MLA_TRACE_EV(w, rank, kind, step) do {} while (0)
#endif
enum { EV_LOAD = 0, EV_RELOAD, EV_QK, EV_PV, EV_S_READY, EV_P_DONE, EV_PBUF_FREE, EV_PV_READY };

// Walks the worker's split segments: calls f(seg_index, b, first_page, end_page).
template <typename F>
__device__ __forceinline__ void for_each_segment(const RunParams& p, int w, F&& f) {
  const int64_t G = p.cum[p.B];
  const int64_t g0 = worker_page_start(w, G, p.W), g1 = worker_page_start(w + 1, G, p.W);
  if (g0 >= g1) return;
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.cum[mid] <= g0) lo = mid; else hi = mid - 1;
  }
  int seg = 0;
  for (int b = lo; b < p.B && p.cum[b] < g1; ++b, ++seg) {
    const int64_t pb = max(p.cum[b], g0) - p.cum[b];
    const int64_t pe = min(p.cum[b + 1], g1) - p.cum[b];
    if (!f(seg, b, (int)pb, (int)pe)) return;
  }
}

// Sequential walk over the worker's steps (one page each): sequence b, page
// within the sequence, end page of the segment, first-of-segment flag.
struct StepCursor {
  int b, page, pe;
  bool first;
  int64_t g1;
  // returns the number of steps of worker w
  __device__ __forceinline__ int init(const RunParams& p, int w) {
    const int64_t G = p.cum[p.B];
    const int64_t g0 = worker_page_start(w, G, p.W);
    g1 = worker_page_start(w + 1, G, p.W);
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cum[mid] <= g0) lo = mid; else hi = mid - 1;
    }
    b = lo;
    page = (int)(g0 - p.cum[b]);
    pe = (int)(min(p.cum[b + 1], g1) - p.cum[b]);
    first = true;
    return (int)(g1 - g0);
  }
  __device__ __forceinline__ void next(const RunParams& p) {
    first = false;
    if (++page >= pe && b + 1 < p.B && p.cum[b + 1] < g1) {
      ++b;
      page = 0;
      pe = (int)(min(p.cum[b + 1], g1) - p.cum[b]);
      first = true;
    }
  }
};

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk16) {
  return row * 128 + ((chunk16 ^ (row & 7)) << 4);
}

template <int S>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_q, RunParams p) {
  using namespace ptx;
  using L = Smem<S>;
  extern __shared__ uint8_t smem_raw[];
  if (!*p.lengths_ok) return;  // uniform across the pair

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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc + 8);
  float* xch = reinterpret_cast<float*>(gbase + L::xch);

  if (threadIdx.x == 0) {
    const uint32_t counts[B_COUNT] = {2, 2, 2, 2, 2, 2, 2, 8, 8, 8, 8, 8, 1, 1, 1, 1, 1, 1, 1, 1,
                                      1, 1, 1};
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

  auto fail = [&](int code) {
    record_error(p.status, code);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tmap(&tm_kv);
      prefetch_tmap(&tm_q);
      // The worker's pages, in order, are its steps. Loads run two steps ahead
      // of the V re-reads; Q is (re)loaded at each segment start once the
      // previous segment's QK MMAs are done with it. Two sequential cursors
      // walk the steps; the block id of each stage is kept for its re-read.
      StepCursor ld, rl;
      const int nsteps = ld.init(p, w);
      rl.init(p, w);
      int32_t stage_blk[kStages] = {0, 0, 0};
      auto block_of = [&](const StepCursor& c) -> int32_t {
        int32_t blk = p.block_table[(int64_t)c.b * p.bt_stride + c.page];
        if (blk < 0 || blk >= p.num_blocks) {
          record_error(p.status, MLA_ERR_BOUNDS);
          blk = 0;  // in-bounds stand-in; the result is flagged by the status word
        }
        return blk;
      };
      auto load_step = [&](int i, int32_t blk) -> bool {
        if (ld.first) {
          if (i > 0) {
            // previous segment's last QK must be done before Q is overwritten
            const int j = i - 1;
            if (!mbar_wait<false>(bar(B_QK_DONE + j % kStages), (j / kStages) & 1)) return false;
          }
          const uint32_t qb = leader_bar(B_Q_FULL);
          expect_leader(B_Q_FULL, kQBytes);
          const int y = ld.b * p.rows + 64 * (int)rank;
          for (int k = 0; k < kChunks; ++k)
            tma_load_2d_pair(base + L::q + k * kQChunkBytes, &tm_q, 64 * k, y, qb);
        }
        const int st = i % kStages;
        stage_blk[st] = blk;
        const uint32_t kb = leader_bar(B_KV_FULL + st);
        expect_leader(B_KV_FULL + st, kStageBytes);
        const int y = blk * 64 + 32 * (int)rank;
        const uint32_t sb = base + L::kv + st * kStageBytes;
        for (int k = 0; k < kChunks; ++k) tma_load_2d_pair(sb + k * kKvChunkBytes, &tm_kv, 64 * k, y, kb);
        MLA_TRACE_EV(w, rank, EV_LOAD, i);
        ld.next(p);
        return true;
      };
      auto reload_step = [&](int i) -> bool {
        const int st = i % kStages;
        if (!mbar_wait<false>(bar(B_QK_DONE + st), (i / kStages) & 1)) return false;
        const uint32_t vb = leader_bar(B_V_FULL + st);
        expect_leader(B_V_FULL + st, 4 * kKvChunkBytes);
        // CTA c takes latent chunk 2q + c for the other 32 tokens of the page
        // into slot 2q + 1 - c (a chunk this CTA's PV never reads).
        const int y = stage_blk[st] * 64 + 32 * (1 - (int)rank);
        const uint32_t sb = base + L::kv + st * kStageBytes;
        for (int q = 0; q < 4; ++q)
          tma_load_2d_pair(sb + (2 * q + 1 - rank) * kKvChunkBytes, &tm_kv, 64 * (2 * q + (int)rank), y, vb);
        MLA_TRACE_EV(w, rank, EV_RELOAD, i);
        return true;
      };
      bool ok = true;
      for (int i = 0; i < nsteps && i < 2 && ok; ++i) ok = load_step(i, block_of(ld));
      for (int i = 0; i < nsteps && ok; ++i) {
        const int32_t next_blk = (i + 2 < nsteps) ? block_of(ld) : 0;  // fetched before the waits
        ok = reload_step(i);
        if (ok && i + 2 < nsteps) {
          // stage of step i+2 was used by step i-1: wait for its PV
          if (i >= 1) {
            const int j = i - 1;
            ok = mbar_wait<false>(bar(B_STAGE_FREE + j % kStages), (j / kStages) & 1);
          }
          if (ok) ok = load_step(i + 2, next_blk);
        }
      }
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      // descriptors of chunk 0 / k-step 0; the 14-bit start-address field
      // (address >> 4) advances by adding the byte offset >> 4
      const uint64_t q_desc0 = smem_desc_sw128(base + L::q, 16, 1024);
      const uint64_t kv_desc0 = smem_desc_sw128(base + L::kv, 16, 1024);
      const uint64_t p_desc0 = smem_desc_sw128(base + L::p, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(base + L::kv, 8192, 1024);
      bool ok = true;
      int i = 0;
      int prev_seg = -1;
      bool prev_first = false;  // is step i-1 the first of its segment
      int prev_segidx = 0;
      auto commit_both = [&](int b) {
        tc_commit<2>(bar(b));
        tc_commit<2>(map_to_cta(bar(b), 1));
      };
      auto issue_pv = [&](int j, bool first_of_seg, int segidx) -> bool {
        if (!mbar_wait(bar(B_P_FULL + (j & 1)), (j >> 1) & 1)) return false;
        if (!mbar_wait(bar(B_V_FULL + j % kStages), (j / kStages) & 1)) return false;
        if (first_of_seg && segidx > 0 && !mbar_wait(bar(B_O_FREE), (segidx - 1) & 1)) return false;
        MLA_TRACE_EV(w, 0, EV_PV_READY, j);
        tc_fence_after();
        const uint64_t vd = v_desc0 + (uint64_t)(((j % kStages) * kStageBytes) >> 4);
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          const int shard = S == 2 ? nb : 0;
          const uint64_t pd = p_desc0 + (uint64_t)((((j & 1) * S + shard) * kPBytes) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16<2>(tbase + kTmemO + 128 * nb, pd + (uint64_t)(2 * ks),
                       vd + (uint64_t)(1024 * nb + 128 * ks), idesc_pv,
                       (first_of_seg && ks == 0) ? 0u : 1u);
        }
        MLA_TRACE_EV(w, 0, EV_PV, j);
        commit_both(B_STAGE_FREE + j % kStages);
        commit_both(B_PV_DONE + (j & 1));
        return true;
      };
      for_each_segment(p, w, [&](int seg, int, int pb, int pe) {
        for (int page = pb; page < pe && ok; ++page, ++i) {
          const bool first = page == pb;
          if (first) ok = mbar_wait(bar(B_Q_FULL), seg & 1);
          if (ok) ok = mbar_wait(bar(B_KV_FULL + i % kStages), (i / kStages) & 1);
          if (ok && i >= 2) ok = mbar_wait(bar(B_S_FREE + (i & 1)), ((i >> 1) - 1) & 1);
          if (!ok) break;
          MLA_TRACE_EV(w, 0, EV_QK, i);
          tc_fence_after();
          const uint64_t bd0 = kv_desc0 + (uint64_t)(((i % kStages) * kStageBytes) >> 4);
#pragma unroll
          for (int shard = 0; shard < S; ++shard) {
            const uint32_t d = tbase + 64 * (i & 1) + 32 * shard;
#pragma unroll
            for (int kc = 0; kc < kChunks; ++kc) {
              if (S == 2 && kc < 8 && (kc / 4) != shard) continue;
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const bool first_k = (S == 2) ? (kc == 4 * shard && ks == 0) : (kc == 0 && ks == 0);
                mma_f16<2>(d, q_desc0 + (uint64_t)(kc * (kQChunkBytes >> 4) + 2 * ks),
                           bd0 + (uint64_t)(kc * (kKvChunkBytes >> 4) + 2 * ks), idesc_qk,
                           first_k ? 0u : 1u);
              }
            }
          }
          commit_both(B_S_FULL + (i & 1));
          commit_both(B_QK_DONE + i % kStages);
          if (i >= 1) ok = issue_pv(i - 1, prev_first, prev_segidx);
          prev_first = first;
          prev_segidx = seg;
          prev_seg = seg;
        }
        return ok;
      });
      if (ok && i >= 1) ok = issue_pv(i - 1, prev_first, prev_segidx);
      (void)prev_seg;
      tc_commit<2>(bar(B_FINAL));
      if (!mbar_wait(bar(B_FINAL), 0)) ok = false;
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps --
    // Every softmax thread executes the same sequence of named barriers
    // whatever happens: after a failed (timed-out) wait the flag `ok` turns
    // false for the whole warp and the remaining steps only skip their work.
    const int lq = (warp & 3) * 32 + lane;         // tensor-memory lane of this thread
    const int half = lq >> 6;                      // token half (0: 0-31, 1: 32-63)
    const int rloc = lq & 63;                      // row within this CTA's 64
    const int row = 64 * (int)rank + rloc;         // query row within the sequence
    const bool row_real = row < p.rows;
    const int t_row = row_real ? row / p.H : 0;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    bool ok = true;
    int i = 0;
    float* xmax = xch;                             // [2][S][128]
    float* xl = xch + 2 * S * 128;                 // [S][128]
    auto named_sync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };
    auto wait = [&](int b, uint32_t parity) {
      if (ok && *abort_flag) ok = false;
      if (ok) ok = mbar_wait<false>(bar(b), parity);
      ok = __all_sync(0xffffffffu, ok);
    };
    for_each_segment(p, w, [&](int, int b, int pb, int pe) {
      const int64_t L = p.seq_lens[b];
      float m[S], l[S];
#pragma unroll
      for (int s = 0; s < S; ++s) { m[s] = -INFINITY; l[s] = 0.f; }
      for (int page = pb; page < pe; ++page, ++i) {
        const int sbuf = i & 1;
        uint32_t sr[S][32];
        wait(B_S_FULL + sbuf, (i >> 1) & 1);
        if (lq == 0) MLA_TRACE_EV(w, rank, EV_S_READY, i);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < S; ++s) tmem_ld32(tbase + lane_off + 64 * sbuf + 32 * s, sr[s]);
          tmem_wait_ld();
          tc_fence_before();
        } else {
#pragma unroll
          for (int s = 0; s < S; ++s)
#pragma unroll
            for (int j = 0; j < 32; ++j) sr[s][j] = 0u;
        }
        __syncwarp();
        if (ok && lane == 0) arrive_leader(B_S_FREE + sbuf);
        // visible part of this thread's 32 tokens [tok0, tok0 + 32)
        const int64_t tok0 = (int64_t)page * 64 + 32 * half;
        const int64_t lim = row_real ? L - p.Lq + t_row : -1;  // last visible key
        int64_t nv = lim - tok0 + 1;
        nv = nv < 0 ? 0 : (nv > 32 ? 32 : nv);
        const int nvis = (int)nv;
        float alpha[S];
        bool rescale = false;
#pragma unroll
        for (int s = 0; s < S; ++s) {
          float mx = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float x = j < nvis ? __uint_as_float(sr[s][j]) * p.scale_log2 : -INFINITY;
            sr[s][j] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
          xmax[(sbuf * S + s) * 128 + lq] = mx;
        }
        named_sync();
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const float mt = fmaxf(xmax[(sbuf * S + s) * 128 + lq], xmax[(sbuf * S + s) * 128 + (lq ^ 64)]);
          float mu = m[s];
          if (m[s] == -INFINITY || mt > m[s] + kRescaleThreshold) mu = fmaxf(mt, m[s]);
          alpha[s] = 1.f;
          if (mu != m[s] && m[s] != -INFINITY) {
            alpha[s] = exp2f(m[s] - mu);
            rescale = true;
          }
          m[s] = mu;
          float ps = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float pj = (mu == -INFINITY) ? 0.f : exp2f(__uint_as_float(sr[s][j]) - mu);
            sr[s][j] = __float_as_uint(pj);
            ps += pj;
          }
          l[s] = l[s] * alpha[s] + ps;
        }
        // the P buffer (i & 1) was last read by PV(i - 2)
        if (i >= 2) wait(B_PV_DONE + sbuf, ((i >> 1) - 1) & 1);
        if (lq == 0) MLA_TRACE_EV(w, rank, EV_PBUF_FREE, i);
        if (__any_sync(0xffffffffu, rescale) && page > pb) {
          // O holds PV(i - 1) of this segment: wait for it, then scale in place
          const int j = i - 1;
          wait(B_PV_DONE + (j & 1), (j >> 1) & 1);
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 256; c += 32) {
              const float a = alpha[S == 2 ? (c >> 7) : 0];
              uint32_t o[32];
              tmem_ld32(tbase + lane_off + kTmemO + c, o);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * a);
              tmem_st32(tbase + lane_off + kTmemO + c, o);
            }
            tmem_wait_st();
          }
        }
        if (ok) {
          // P (bf16) -> shared memory, K-major 128-byte swizzle: row rloc,
          // tokens [32 half, 32 half + 32) = 16-byte chunks 4 half .. 4 half + 3
#pragma unroll
          for (int s = 0; s < S; ++s) {
            uint8_t* pbuf = gbase + L::p + (sbuf * S + s) * kPBytes;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t v[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(sr[s][8 * c + 2 * k]),
                                                          __uint_as_float(sr[s][8 * c + 2 * k + 1]));
                v[k] = *reinterpret_cast<uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(pbuf + sw128(rloc, 4 * half + c)) =
                  make_uint4(v[0], v[1], v[2], v[3]);
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
        }
        __syncwarp();
        if (ok && lane == 0) arrive_leader(B_P_FULL + sbuf);
        if (lq == 0) MLA_TRACE_EV(w, rank, EV_P_DONE, i);
      }
      // ---- segment epilogue: O / l and log2-sum-exp of this segment
      const int j = i - 1;
      wait(B_PV_DONE + (j & 1), (j >> 1) & 1);
      if (ok) tc_fence_after();
#pragma unroll
      for (int s = 0; s < S; ++s) xl[s * 128 + lq] = l[s];
      named_sync();
      float inv[S];
      const int64_t slot = w + b;
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const float lt = l[s] + xl[s * 128 + (lq ^ 64)];
        inv[s] = lt > 0.f ? 1.f / lt : 0.f;
        if (ok && half == 0 && row_real)
          p.lse_part[(slot * p.rows + row) * S + s] = lt > 0.f ? m[s] + log2f(lt) : kEmptyLse;
      }
      if (ok) {
        float* orow = p.o_part + (slot * p.rows + row) * (int64_t)p.r;
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t o[32];
          tmem_ld32(tbase + lane_off + kTmemO + c, o);
          tmem_wait_ld();
          const int nb = c >> 7, cc = c & 127;
          const float iv = inv[S == 2 ? nb : 0];
          const int chunk = 4 * nb + 2 * (cc >> 6) + half;
          const int col0 = 64 * chunk + (cc & 63);
          if (row_real) {
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<float4*>(orow + col0 + k) =
                  make_float4(__uint_as_float(o[k]) * iv, __uint_as_float(o[k + 1]) * iv,
                              __uint_as_float(o[k + 2]) * iv, __uint_as_float(o[k + 3]) * iv);
          }
        }
        tc_fence_before();
      }
      named_sync();  // xl and the O reads of all four warps are done
      __syncwarp();
      if (ok && lane == 0) arrive_leader(B_O_FREE);
      return true;
    });
    if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
  }
  __syncwarp();

  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<2>(tbase, kTmemCols);
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

// 2-D bf16 row-major [rows, 576] with a (64 columns x box_rows) 128B-swizzled box.
inline bool make_rows_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kWidth, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kWidth * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

inline cudaError_t launch_tc_decode(const RunParams& p, cudaStream_t stream) {
  CUtensorMap tm_kv, tm_q;
  if (!tc::make_rows_map(&tm_kv, p.kv, (uint64_t)p.num_blocks * 64, 32)) return cudaErrorInvalidValue;
  if (!tc::make_rows_map(&tm_q, p.q, (uint64_t)p.B * p.rows, 64)) return cudaErrorInvalidValue;
  cudaError_t e;
  if (p.S == 1) {
    e = cudaFuncSetAttribute(tc::decode_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc::Smem<1>::alloc);
    if (e != cudaSuccess) return e;
    tc::decode_tc_kernel<1><<<2 * p.W, tc::kThreads, tc::Smem<1>::alloc, stream>>>(tm_kv, tm_q, p);
  } else {
    e = cudaFuncSetAttribute(tc::decode_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc::Smem<2>::alloc);
    if (e != cudaSuccess) return e;
    tc::decode_tc_kernel<2><<<2 * p.W, tc::kThreads, tc::Smem<2>::alloc, stream>>>(tm_kv, tm_q, p);
  }
  return cudaGetLastError();
}

}  // namespace mla
