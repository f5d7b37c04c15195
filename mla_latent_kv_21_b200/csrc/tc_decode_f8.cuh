// tcgen05 split-KV decode over an FP8 latent cache (dims.dtype = MLA_FP8_CACHE):
// per token 512 E4M3 codes of cKV, one fp32 scale s_t and a bf16 RoPE key
// stored divided by s_t, so that cKV_t = s_t * code_t and k_rope_t = s_t *
// stored_t. Activations, weights and the output are bf16; r = 512, d_rope =
// 64, 64-token pages, up to 128 query rows, one latent shard.
//
// The CTA pair, its split of query rows and tokens, the group of 4 pages, the
// tensor-memory layout, the online softmax and the segment epilogue are those
// of the bf16 kernel (tc_decode.cuh). What changes is what crosses HBM, how it
// is multiplied, and the softmax's code shape:
//
//   QK  per group five ring items instead of nine: four of 128 tokens x 128
//       code bytes (one 128-column chunk of cKV) and the RoPE chunk (128 tokens
//       x 64 bf16). The absorbed query arrives from the absorb kernel split
//       into q_hi = e4m3(q) and q_lo = e5m2(q - q_hi); each cKV chunk takes two
//       tcgen05.mma kind::f8f6f4 per K step of 32 (q_hi . code and q_lo .
//       code, both accumulating into S), the RoPE chunk four kind::f16 MMAs.
//       S then holds S'_t = score_t / s_t (the RoPE key is stored divided by
//       s_t), and the softmax multiplies column t by s_t from a per-group
//       table of scales (one 1 KB bulk copy per group).
//   PV  the cached codes themselves are V: V items of 128 tokens x 128 code
//       bytes (one column block per CTA), four per group instead of eight.
//       P' = 2^kp * p_t * s_t goes to shared memory as P'_hi = e4m3(P') and
//       P'_lo = e4m3(P' - P'_hi) and each K step of 32 tokens takes two
//       kind::f8f6f4 MMAs (P'_hi . code and P'_lo . code), so O accumulates
//       2^kp sum_t p_t cKV_t. The power of two 2^kp, chosen per group from the
//       group's largest scale, puts P' as high in e4m3's range as the lazy max
//       allows (28 < 2^kp * s_max <= 56 and P <= 2^3: P' <= 448), so that
//       every weight P >= (s_max / s_t) / 112 has P' >= 1/4, where the split
//       keeps 8 significant bits; it is carried by O and the row sum like a
//       shift of the running max.
//   softmax  the per-element work is about three times the bf16 kernel's, so
//       both passes (row max; P, P' and its split) walk a thread's 128 columns
//       32 at a time through one copy of their loop body, reading S from
//       tensor memory twice, and P' goes to shared memory 32 tokens at a time:
//       unrolled over 128 columns the code outgrows the instruction cache.
//       Each token half has its own P' buffer (the QK ring has three slots to
//       make room), so neither half waits for PV of the other's tokens.
//
// The two-term splits keep the operands near bf16 precision while the cache
// bytes per token fall from 1152 to 644: the e4m3 term leaves a residual below
// 2^-4 of the value, which the query's e5m2 term (any magnitude) carries to
// within 2^-3 of itself and P's e4m3 term to within 2^-4 while the residual is
// an e4m3 normal (P' >= 1/4), or to an absolute 2^-10 below that.
//
// Sources: as tc_decode.cuh (TPLA abstract, TransMLA abstract, pith.science
// verdict record for 2502.07864); the FP8 cache itself is a format of this
// library.
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tc_decode.cuh"

namespace mla {
namespace tc8 {

using tc::GroupCursor;
using tc::kGroupPages;
// The running max moves (and O is rescaled) when a group's row max exceeds it
// by more than 2^3, so P <= 2^3 and P' = 2^kp * P * s_t <= 8 * kPScaleTarget
// = 448, e4m3's largest finite value.
constexpr float kRescaleThreshold = 3.0f;   // log2 units
constexpr float kPScaleTarget = 56.0f;      // 2^kp * s_max <= 56
using tc::kThreads;
using tc::kTmemCols;
using tc::kTmemO;
using tc::sw128;
#ifdef MLA_TRACE
using tc::g_trace;
using tc::g_trace_chunk;
using tc::g_trace_ns;
using tc::kTraceChunks;
using tc::kTraceKinds;
using tc::kTraceSteps;
using tc::kTraceWorkers;
#endif

constexpr int kLatChunks = 4;                         // 128-column chunks of cKV (e4m3 codes)
constexpr int kItems = kLatChunks + 1;                // QK ring items per group (+ the RoPE chunk)
constexpr int kQChunks = 2 * kLatChunks + 1;          // query chunks: hi 0-3, lo 0-3, RoPE
constexpr uint32_t kQChunkBytes = 64 * 128;           // 64 rows x 128 B
constexpr uint32_t kQBytes = kQChunks * kQChunkBytes;  // 72 KB
constexpr uint32_t kQRowBytes = 1152;                 // workspace query row: hi 512 | lo 512 | RoPE 128
constexpr uint32_t kSlotBytes = 16384;                // 128 tokens x 128 B
constexpr int kQkSlots = 3;
constexpr int kVSlots = 4;
constexpr uint32_t kPHalfBytes = 64 * 128;            // one token half of P': 64 rows x 128 tokens
constexpr uint32_t kPRegion = 2 * kPHalfBytes;        // P'_hi and P'_lo of one token half (two buffers)
constexpr uint32_t kScaleBytes = kGroupPages * 64 * 4;  // token scales of one group
constexpr int kScaleBufs = 4;                         // groups of scales in flight (producer runs ahead)

struct Smem {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t qk = q + kQBytes;
  static constexpr uint32_t v = qk + kQkSlots * kSlotBytes;
  static constexpr uint32_t p = v + kVSlots * kSlotBytes;
  static constexpr uint32_t xch = p + 2 * kPRegion;    // float [2][128] row max, [128] l, [2][4] scale max
  static constexpr uint32_t sc = xch + 3 * 128 * 4 + 2 * 4 * 4;  // float [kScaleBufs][256] token scales
  static constexpr uint32_t bars = sc + kScaleBufs * kScaleBytes;
  static constexpr uint32_t nbars = 48;
  static constexpr uint32_t misc = bars + nbars * 8;   // tmem slot, abort flag
  static constexpr uint32_t total = misc + 64;
  static constexpr uint32_t alloc = total + 1024;
};

enum : int {
  B_QK_FULL = 0,     // [4] leader, count 2 (+tx)
  B_V_FULL = 4,      // [4] leader, count 2 (+tx)
  B_S_FREE = 8,      // [2] leader, count 8
  B_P_FULL = 10,     // leader, count 8: P' of pages 0, 1 written and O rescaled
  B_O_FREE = 11,     // leader, count 8
  B_QK_FREE = 12,    // [4] both, count 1 (MMA commit)
  B_V_FREE = 16,     // [4] both, count 1
  B_S_FULL = 20,     // [2] both, count 1
  B_PV_DONE = 22,    // both, count 1
  B_FINAL_QK = 23,   // leader, count 1
  B_FINAL_PV = 24,   // leader, count 1
  B_P_FREE_LO = 25,  // both, count 1: PV is done with P' of pages 0, 1
  B_P_FREE_HI = 26,  // both, count 1: PV is done with P' of pages 2, 3
  B_QC_FULL = 27,    // [5] leader, count 2 (+tx): query chunks of ring item c (segment start)
  B_P_FULL_HI = 32,  // leader, count 4: P' of pages 2, 3 written
  B_SC_FULL = 33,    // [4] local, count 1 (+tx): token scales of the group
  B_SC_FREE = 37,    // [4] local, count 4: the softmax warps are done with them
  B_COUNT = 41
};
static_assert(B_COUNT <= (int)Smem::nbars, "barrier region");

// instruction descriptors: dense, f32 accumulator, M = 128, N = 256
constexpr uint32_t kIdescBase = (1u << 4) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t kE5M2A = 1u << 7;   // A format e5m2 (e4m3 = 0)
constexpr uint32_t kMnMajorB = 1u << 16;

__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// (P_hi, P_lo) bytes of four values: two words, byte j = value j. The values
// go to f16 first (11 significant bits, below the residual's step); hi =
// e4m3(x), lo = e4m3(x - hi), the difference taken exactly in f16. The P pass
// scales P' into e4m3's normal range, where a residual of at least 2^-6 keeps
// four significant bits and a smaller one an absolute step of 2^-9.
__device__ __forceinline__ void split4(float a, float b, float c, float d, uint32_t& hi, uint32_t& lo) {
  const uint32_t x01 = ptx::cvt_f16x2(a, b), x23 = ptx::cvt_f16x2(c, d);
  const uint32_t h01 = ptx::e4m3x2_of_f16x2(x01), h23 = ptx::e4m3x2_of_f16x2(x23);
  const uint32_t l01 = ptx::e4m3x2_of_f16x2(ptx::sub_f16x2(x01, ptx::f16x2_of_e4m3x2(h01)));
  const uint32_t l23 = ptx::e4m3x2_of_f16x2(ptx::sub_f16x2(x23, ptx::f16x2_of_e4m3x2(h23)));
  hi = h01 | (h23 << 16);
  lo = l01 | (l23 << 16);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_f8_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_rope,
                     const __grid_constant__ CUtensorMap tm_q, RunParams p) {
  using namespace ptx;
  using L = Smem;
  extern __shared__ uint8_t smem_raw[];

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t rank = cluster_ctarank();
  const int w = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return base + L::bars + 8u * i; };
  auto leader_bar = [&](int i) -> uint32_t { return map_to_cta(bar(i), 0); };
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
  float* xch = reinterpret_cast<float*>(gbase + L::xch);
  float* scales = reinterpret_cast<float*>(gbase + L::sc);

  if (threadIdx.x == 0) {
    uint32_t counts[B_COUNT];
    for (int i = 0; i < B_COUNT; ++i) counts[i] = 1;
    for (int i = 0; i < kItems; ++i) counts[B_QC_FULL + i] = 2;
    for (int i = 0; i < kQkSlots; ++i) counts[B_QK_FULL + i] = 2;
    for (int i = 0; i < kVSlots; ++i) counts[B_V_FULL + i] = 2;
    counts[B_S_FREE] = counts[B_S_FREE + 1] = 8;
    counts[B_P_FULL] = 8;
    counts[B_P_FULL_HI] = 4;
    counts[B_O_FREE] = 8;
    for (int i = 0; i < kScaleBufs; ++i) counts[B_SC_FREE + i] = 4;
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
  grid_launch_dependents();
  grid_dependency_wait();
  const bool run = *p.lengths_ok != 0;

  auto fail = [&](int code) {
    record_error(p.status, code);
    *abort_flag = 1;
  };
  // Block of page `page` of sequence b, or -1 (past the group's end, or an
  // invalid id, which is reported). Rows of missing pages are read past the
  // tensors (TMA fills zeros) and masked by the softmax.
  const int oob_row = (int)(p.num_blocks * 64);
  auto page_block = [&](int b, int page, bool exists) -> int {
    if (!exists) return -1;
    const int32_t blk = p.block_table[(int64_t)b * p.bt_stride + page];
    if (blk < 0 || blk >= p.num_blocks) {
      record_error(p.status, MLA_ERR_BOUNDS);
      return -1;
    }
    return blk;
  };

  if (!run) {
    // invalid lengths (reported by the length scan): nothing to do
  } else if (warp == 0) {
    // ------------------------------- query, QK item and token-scale producer --
    // lanes 0 and 1: lane k loads this CTA's page 2 rank + k of every item;
    // lane 0 also copies the group's token scales, lane 1 reloads the query
    // at segment starts
    if (lane < 2) {
      if (lane == 0) {
        prefetch_tmap(&tm_codes);
        prefetch_tmap(&tm_rope);
        prefetch_tmap(&tm_q);
      }
      const int k = lane;
      GroupCursor g;
      bool ok = true;
      bool have = g.init(p, w);
      uint32_t cc = 0;  // item counter over all groups
      for (int gi = 0; have && ok; ++gi) {
        const int yq = g.b * p.rows + 64 * (int)rank;  // this CTA's query rows of the segment
        const int pg = 2 * (int)rank + k;
        const int blk = page_block(g.b, g.page + pg, pg < g.npages);
        const int y = blk >= 0 ? blk * 64 : oob_row;
        if (k == 0) MLA_TRACE_EV(w, rank, tc::EV_LOAD, gi);
        if (k == 0) {
          // token scales of the group's four pages -> table gi % kScaleBufs
          const int sbuf = gi % kScaleBufs;
          if (gi >= kScaleBufs) ok = mbar_wait(bar(B_SC_FREE + sbuf), ((gi / kScaleBufs) - 1) & 1);
          if (!ok) break;
          int blks[kGroupPages];
          uint32_t bytes = 0;
          for (int q = 0; q < kGroupPages; ++q) {
            blks[q] = page_block(g.b, g.page + q, q < g.npages);
            if (blks[q] >= 0) bytes += 256;
          }
          mbar_arrive_expect_tx_local(bar(B_SC_FULL + sbuf), bytes);
          for (int q = 0; q < kGroupPages; ++q)
            if (blks[q] >= 0)
              bulk_load_g2s(base + L::sc + sbuf * kScaleBytes + q * 256, p.kv_scale + (int64_t)blks[q] * 64, 256,
                            bar(B_SC_FULL + sbuf));
        }
        for (int c = 0; c < kItems && ok; ++c, ++cc) {
          const int slot = cc % kQkSlots;
          if (cc >= (uint32_t)kQkSlots) ok = mbar_wait(bar(B_QK_FREE + slot), ((cc / kQkSlots) - 1) & 1);
          if (!ok) break;
          if (g.first && k == 1) {
            // New segment: reload the query chunks item c reads (hi and lo of
            // cKV chunk c, or the RoPE chunk). Their last reader, item c of the
            // previous group (5 items back), is done: the QK issuer consumes
            // items in order and item cc - kQkSlots has been released.
            if (c < kLatChunks) {
              expect_leader(B_QC_FULL + c, 2 * kQChunkBytes);
              tma_load_2d_pair(base + L::q + c * kQChunkBytes, &tm_q, 128 * c, yq, leader_bar(B_QC_FULL + c));
              tma_load_2d_pair(base + L::q + (kLatChunks + c) * kQChunkBytes, &tm_q, 512 + 128 * c, yq,
                               leader_bar(B_QC_FULL + c));
            } else {
              expect_leader(B_QC_FULL + c, kQChunkBytes);
              tma_load_2d_pair(base + L::q + 2 * kLatChunks * kQChunkBytes, &tm_q, 1024, yq,
                               leader_bar(B_QC_FULL + c));
            }
          }
          if (k == 0) expect_leader(B_QK_FULL + slot, kSlotBytes);
          if (c < kLatChunks)
            tma_load_2d_pair(base + L::qk + slot * kSlotBytes + k * (kSlotBytes / 2), &tm_codes, 128 * c, y,
                             leader_bar(B_QK_FULL + slot));
          else
            tma_load_2d_pair(base + L::qk + slot * kSlotBytes + k * (kSlotBytes / 2), &tm_rope, 0, y,
                             leader_bar(B_QK_FULL + slot));
          if (k == 0) MLA_TRACE_CHUNK(w, rank, 0, cc);
        }
        if (ok) have = g.next(p);
      }
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------ V item producer --
    // item (token half th, column block nb): pages 2 th, 2 th + 1 of the code
    // columns [256 nb + 128 rank, +128); lane k loads page 2 th + k
    if (lane < 2) {
      const int k = lane;
      GroupCursor g;
      bool ok = true;
      bool have = g.init(p, w);
      uint32_t vc = 0;
      while (have && ok) {
        int rows[2];
        for (int th = 0; th < 2; ++th) {
          const int q = 2 * th + k;
          const int blk = page_block(g.b, g.page + q, q < g.npages);
          rows[th] = blk >= 0 ? blk * 64 : oob_row;
        }
        for (int th = 0; th < 2 && ok; ++th) {
          for (int nb = 0; nb < 2 && ok; ++nb, ++vc) {
            const int slot = vc % kVSlots;
            if (vc >= (uint32_t)kVSlots) ok = mbar_wait(bar(B_V_FREE + slot), ((vc / kVSlots) - 1) & 1);
            if (!ok) break;
            if (k == 0) expect_leader(B_V_FULL + slot, kSlotBytes);
            tma_load_2d_pair(base + L::v + slot * kSlotBytes + k * (kSlotBytes / 2), &tm_codes,
                             256 * nb + 128 * (int)rank, rows[th], leader_bar(B_V_FULL + slot));
            if (k == 0) MLA_TRACE_CHUNK(w, rank, 2, vc);
          }
        }
        if (ok) have = g.next(p);
      }
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ QK MMA issuer --
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_hi = kIdescBase;
      const uint32_t idesc_lo = kIdescBase | kE5M2A;
      const uint32_t idesc_rope = idesc_bf16_f32(128, 256, 0, 0);
      const uint64_t q_desc0 = smem_desc_sw128(base + L::q, 16, 1024);
      const uint64_t qk_desc0 = smem_desc_sw128(base + L::qk, 16, 1024);
      bool ok = true;
      uint32_t cc = 0;
      GroupCursor g;
      bool have = g.init(p, w);
      for (int gi = 0; have && ok; ++gi) {
        const int sb = gi & 1;
        if (gi >= 2) ok = mbar_wait(bar(B_S_FREE + sb), ((gi >> 1) - 1) & 1);
        if (!ok) break;
        const uint32_t s_tmem = tbase + sb * 128;
        MLA_TRACE_EV(w, 0, tc::EV_QK_START, gi);
        for (int c = 0; c < kItems && ok; ++c, ++cc) {
          const int slot = cc % kQkSlots;
          if (g.first) ok = mbar_wait(bar(B_QC_FULL + c), g.seg & 1);  // this segment's query chunks
          ok = ok && mbar_wait(bar(B_QK_FULL + slot), (cc / kQkSlots) & 1);
          if (!ok) break;
          MLA_TRACE_CHUNK(w, 0, 1, cc);
          tc_fence_after();
          const uint64_t bd = qk_desc0 + (uint64_t)((slot * kSlotBytes) >> 4);
          if (c < kLatChunks) {
            const uint64_t ah = q_desc0 + (uint64_t)((c * kQChunkBytes) >> 4);
            const uint64_t al = q_desc0 + (uint64_t)(((kLatChunks + c) * kQChunkBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // K = 128 = 4 x 32 (32 bytes per step)
              mma_f8(s_tmem, ah + (uint64_t)(2 * ks), bd + (uint64_t)(2 * ks), idesc_hi,
                     (c == 0 && ks == 0) ? 0u : 1u);
              mma_f8(s_tmem, al + (uint64_t)(2 * ks), bd + (uint64_t)(2 * ks), idesc_lo, 1u);
            }
          } else {
            const uint64_t ar = q_desc0 + (uint64_t)((2 * kLatChunks * kQChunkBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)  // K = 64 = 4 x 16 (bf16)
              mma_f16<2>(s_tmem, ar + (uint64_t)(2 * ks), bd + (uint64_t)(2 * ks), idesc_rope, 1u);
          }
          commit_both(B_QK_FREE + slot);
        }
        if (!ok) break;
        MLA_TRACE_EV(w, 0, tc::EV_QK_END, gi);
        commit_both(B_S_FULL + sb);
        have = g.next(p);
      }
      tc_commit<2>(bar(B_FINAL_QK));
      if (!mbar_wait(bar(B_FINAL_QK), 0)) ok = false;
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 7) {
    // ------------------------------------------------------ PV MMA issuer --
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_hi = kIdescBase | kMnMajorB;
      const uint32_t idesc_lo = kIdescBase | kMnMajorB;  // P'_lo is e4m3 too
      const uint64_t p_desc0 = smem_desc_sw128(base + L::p, 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(base + L::v, kSlotBytes, 1024);
      bool ok = true;
      uint32_t vc = 0;
      GroupCursor g;
      bool have = g.init(p, w);
      for (int gi = 0; have && ok; ++gi) {
        ok = mbar_wait(bar(B_P_FULL), gi & 1);
        if (ok && g.first && g.seg > 0) ok = mbar_wait(bar(B_O_FREE), (g.seg - 1) & 1);
        if (!ok) break;
        MLA_TRACE_EV(w, 0, tc::EV_PV_START, gi);
        for (int th = 0; th < 2 && ok; ++th) {
          if (th == 1) {
            ok = mbar_wait(bar(B_P_FULL_HI), gi & 1);  // P' of pages 2, 3 in its buffer
            if (!ok) break;
          }
          for (int nb = 0; nb < 2 && ok; ++nb, ++vc) {
            const int slot = vc % kVSlots;
            ok = mbar_wait(bar(B_V_FULL + slot), (vc / kVSlots) & 1);
            if (!ok) break;
            MLA_TRACE_CHUNK(w, 0, 3, vc);
            tc_fence_after();
            const uint64_t vd = v_desc0 + (uint64_t)((slot * kSlotBytes) >> 4);
            const uint64_t pd = p_desc0 + (uint64_t)((th * kPRegion) >> 4);  // this token half's P
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // K = 128 tokens = 4 x 32; V steps 32 rows x 128 B
              mma_f8(tbase + kTmemO + 128 * nb, pd + (uint64_t)(2 * ks), vd + (uint64_t)(256 * ks),
                     idesc_hi, (g.first && th == 0 && ks == 0) ? 0u : 1u);
              mma_f8(tbase + kTmemO + 128 * nb, pd + (uint64_t)((kPHalfBytes >> 4) + 2 * ks),
                     vd + (uint64_t)(256 * ks), idesc_lo, 1u);
            }
            commit_both(B_V_FREE + slot);
          }
          if (th == 0) commit_both(B_P_FREE_LO);
        }
        if (!ok) break;
        MLA_TRACE_EV(w, 0, tc::EV_PV_END, gi);
        commit_both(B_P_FREE_HI);
        commit_both(B_PV_DONE);
        have = g.next(p);
      }
      tc_commit<2>(bar(B_FINAL_PV));
      if (!mbar_wait(bar(B_FINAL_PV), 0)) ok = false;
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps --
    // As in the bf16 kernel; every softmax thread executes the same sequence
    // of named barriers whatever happens.
    const int lq = (warp & 3) * 32 + lane;         // tensor-memory lane of this thread
    const int half = lq >> 6;                      // token half: group tokens [128 half, +128)
    const int rloc = lq & 63;                      // row within this CTA's 64
    const int row = 64 * (int)rank + rloc;         // query row within the sequence
    const bool row_real = row < p.rows;
    const int t_row = row_real ? row / p.H : 0;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    bool ok = true;
    float* xl = xch + 2 * 128;                     // [128]
    auto named_sync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };
    auto wait = [&](int b, uint32_t parity) {
      if (ok && *abort_flag) ok = false;
      if (ok) ok = mbar_wait(bar(b), parity);
      ok = __all_sync(0xffffffffu, ok);
    };
    GroupCursor g;
    bool have = g.init(p, w);
    int gi = 0;
    float m = -INFINITY, l = 0.f;
    int kp = 0;                                    // P' is held as 2^kp * P * s_t
    while (have) {
      if (g.first) { m = -INFINITY; l = 0.f; }
      const int sb = gi & 1;
      float* xmax = xch + (gi & 1) * 128;
      const int64_t Lb = p.seq_lens[g.b];
      const int64_t key0 = (int64_t)(g.page + 2 * half) * 64;
      const int64_t lim = row_real ? Lb - p.Lq + t_row : -1;  // last visible key
      int64_t nv = lim - key0 + 1;
      const int64_t in_group = (int64_t)(g.npages - 2 * half) * 64;
      nv = nv > in_group ? in_group : nv;
      nv = nv < 0 ? 0 : (nv > 128 ? 128 : nv);
      const int nvis = (int)nv;

      wait(B_S_FULL + sb, (gi >> 1) & 1);
      if (lq == 0) MLA_TRACE_EV(w, rank, tc::EV_S_READY, gi);
      if (ok) tc_fence_after();
      const uint32_t s_col = tbase + lane_off + sb * 128;  // this thread's 128 S columns
      // S holds score / s_t: column t is multiplied by its token scale
      wait(B_SC_FULL + gi % kScaleBufs, (gi / kScaleBufs) & 1);
      float* sc_tab = scales + (gi % kScaleBufs) * (kScaleBytes / 4);
      const float* sct = sc_tab + 128 * half;
      float* xsmax = xch + 3 * 128 + (gi & 1) * 4;  // [4] per-warp largest scale of this group
      if (ok) {
        // entries of keys past the sequence (or of pages the group lacks) hold
        // whatever the pool or an older group left there: zero them, so that a
        // masked key's P' = 0 * s is 0 whatever it held; the named barrier
        // below orders these stores before the P pass reads the table. The
        // largest valid scale of the group goes to xsmax (scales are > 0, so
        // their bits order as unsigned integers).
        uint32_t smax_bits = 0u;
#pragma unroll
        for (int e = lq; e < 4 * 64; e += 128) {
          const int q = e >> 6;
          if (q >= g.npages || (int64_t)(g.page + q) * 64 + (e & 63) >= Lb) sc_tab[e] = 0.f;
          else smax_bits = max(smax_bits, __float_as_uint(sc_tab[e]));
        }
        smax_bits = __reduce_max_sync(0xffffffffu, smax_bits);
        if (lane == 0) xsmax[warp & 3] = __uint_as_float(smax_bits);
      }
      if (lq == 0) MLA_TRACE_EV(w, rank, tc::EV_PASS1, gi);
      // 32 S columns from tensor memory times their token scales; keys masked
      // for this row (past the group or the causal limit) become -inf
      auto load_scaled = [&](int c0, uint32_t (&r)[32]) {
        tmem_ld32(s_col + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 s4 = *reinterpret_cast<const float4*>(sct + c0 + j);
          r[j] = __float_as_uint(__uint_as_float(r[j]) * s4.x);
          r[j + 1] = __float_as_uint(__uint_as_float(r[j + 1]) * s4.y);
          r[j + 2] = __float_as_uint(__uint_as_float(r[j + 2]) * s4.z);
          r[j + 3] = __float_as_uint(__uint_as_float(r[j + 3]) * s4.w);
        }
        if (nvis < c0 + 32) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j >= nvis) r[j] = 0xff800000u;
        }
      };
      // Both passes walk the 128 columns 32 at a time through one copy of
      // their loop body and read tensor memory twice: a fully unrolled
      // 128-column pass is more code than the instruction cache holds.
      float mx0 = -INFINITY, mx1 = -INFINITY;
      if (ok) {
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t r[32];
          load_scaled(c0, r);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            mx0 = fmaxf(mx0, __uint_as_float(r[j]));
            mx1 = fmaxf(mx1, __uint_as_float(r[j + 1]));
          }
        }
      }
      const float mt_own = fmaxf(mx0, mx1) * p.scale_log2;
      xmax[lq] = mt_own;
      if (lq == 0) MLA_TRACE_EV(w, rank, tc::EV_SYNC1, gi);
      if (lq == 64) MLA_TRACE_EV(w, rank, tc::EV_LD0, gi);
      named_sync();
      if (lq == 0) MLA_TRACE_EV(w, rank, tc::EV_LD1, gi);
      const float mt = fmaxf(mt_own, xmax[lq ^ 64]);
      float mu = m;
      if (m == -INFINITY || mt > m + kRescaleThreshold) mu = fmaxf(mt, m);
      // P' is kept as 2^kp * P * s_t with 2^kp * s_max <= 56, so that with
      // P <= 2^3 (the lazy max) it stays at or below e4m3's 448 and weights
      // P >= (s_max / s_t) / 112 reach P' >= 1/4 (8 bits in the split); kp
      // only falls within a segment. O and l carry the same 2^kp: the exponent
      // offset is m - kp, and a change of either rescales them like a new max.
      const float smax = fmaxf(fmaxf(xsmax[0], xsmax[1]), fmaxf(xsmax[2], xsmax[3]));
      int kg = smax > 0.f ? (int)((__float_as_uint(kPScaleTarget / smax) >> 23) & 0xFF) - 127 : kp;
      kg = kg < -64 ? -64 : (kg > 64 ? 64 : kg);
      const int kn = g.first ? kg : min(kp, kg);
      const float off_old = m - (float)kp, off_new = mu - (float)kn;
      float alpha = 1.f;
      const bool rescale = m != -INFINITY && off_new != off_old;
      if (rescale) alpha = ex2_approx(off_old - off_new);
      m = mu;
      kp = kn;
      auto rescale_o = [&]() {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t o[32];
          tmem_ld32(tbase + lane_off + kTmemO + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(tbase + lane_off + kTmemO + c, o);
        }
        tmem_wait_st();
      };
      // O is rescaled (after the previous group's PV) before this group's PV
      // adds to it: B_P_FULL counts half 0's P' writes and half 1's rescale.
      // Each token half has its own P' buffer, free once the previous group's
      // PV of that half is done.
      if (!g.first && __any_sync(0xffffffffu, rescale)) wait(B_PV_DONE, (gi - 1) & 1);
      if (ok && !g.first && __any_sync(0xffffffffu, rescale)) rescale_o();
      if (half == 1) {
        if (ok) tc_fence_before();
        __syncwarp();
        if (ok && lane == 0) arrive_leader(B_P_FULL);
      }
      if (gi >= 1) wait(half == 0 ? B_P_FREE_LO : B_P_FREE_HI, (gi - 1) & 1);
      if (lq == 0) MLA_TRACE_EV(w, rank, tc::EV_PBUF_FREE, gi);
      // P = 2^(score * scale - m + kp); P' = P * s_t split into two e4m3 bytes,
      // written 32 tokens at a time into row rloc of this half's P' buffer
      // (K-major, 128-byte swizzle: 16-byte units c0 / 16 and c0 / 16 + 1);
      // the row sum takes P itself
      uint8_t* pbuf = gbase + L::p + half * kPRegion;
      float ps0 = 0.f, ps1 = 0.f, ps2 = 0.f, ps3 = 0.f;
      const float nmu = mu == -INFINITY ? 0.f : -off_new;
      if (ok) {
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t r[32];
          load_scaled(c0, r);
          uint32_t ph[8], pl[8];
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(r[j]), p.scale_log2, nmu));
            const float p1 = ex2_approx(fmaf(__uint_as_float(r[j + 1]), p.scale_log2, nmu));
            const float p2 = ex2_approx(fmaf(__uint_as_float(r[j + 2]), p.scale_log2, nmu));
            const float p3 = ex2_approx(fmaf(__uint_as_float(r[j + 3]), p.scale_log2, nmu));
            ps0 += p0; ps1 += p1; ps2 += p2; ps3 += p3;
            // a key masked for this row has P = 0 (score -inf) and a finite table entry
            const float4 s4 = *reinterpret_cast<const float4*>(sct + c0 + j);
            split4(p0 * s4.x, p1 * s4.y, p2 * s4.z, p3 * s4.w, ph[j >> 2], pl[j >> 2]);
          }
          const int u0 = c0 >> 4;
          *reinterpret_cast<uint4*>(pbuf + sw128(rloc, u0)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
          *reinterpret_cast<uint4*>(pbuf + sw128(rloc, u0 + 1)) = make_uint4(ph[4], ph[5], ph[6], ph[7]);
          *reinterpret_cast<uint4*>(pbuf + kPHalfBytes + sw128(rloc, u0)) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
          *reinterpret_cast<uint4*>(pbuf + kPHalfBytes + sw128(rloc, u0 + 1)) =
              make_uint4(pl[4], pl[5], pl[6], pl[7]);
        }
        // P' (and the table's zeroing stores) before the MMAs and the next bulk
        // copy into the table (async proxy); the S reads before QK reuses S
        fence_proxy_async_smem();
        tc_fence_before();
      }
      l = l * alpha + ((ps0 + ps1) + (ps2 + ps3));
      if (lq == 0) MLA_TRACE_EV(w, rank, tc::EV_PASS2, gi);
      __syncwarp();
      if (ok && lane == 0) {
        arrive_leader(B_S_FREE + sb);
        mbar_arrive_local(bar(B_SC_FREE + gi % kScaleBufs));
        arrive_leader(half == 0 ? B_P_FULL : B_P_FULL_HI);
      }
      if (lq == 0) MLA_TRACE_EV(w, rank, tc::EV_P_DONE, gi);

      if (g.last_of_segment()) {
        // ---- segment epilogue: O / l (fp16) and log2-sum-exp of this segment
        wait(B_PV_DONE, gi & 1);
        if (ok) tc_fence_after();
        xl[lq] = l;
        named_sync();
        const int64_t slot = w + g.b;
        const float lt = l + xl[lq ^ 64];
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        if (ok && half == 0 && row_real) p.lse_part[slot * p.rows + row] = lt > 0.f ? m - (float)kp + log2f(lt) : kEmptyLse;
        if (ok) {
          // a warp's 32 rows x 64 columns per round, transposed through 4 KB
          // of the (idle) P' buffer into whole 128-byte row segments
          uint8_t* stage = gbase + L::p + (warp & 3) * 4096;
          const int rbase = 64 * (int)rank + 32 * ((warp & 3) & 1);
          const int j = lane & 7;
          __half* oh = reinterpret_cast<__half*>(p.o_part);
#pragma unroll 1
          for (int c = 0; c < 256; c += 64) {
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
                __half2 h2 = __floats2half2_rn(__uint_as_float(o[8 * u + 2 * k]) * inv,
                                               __uint_as_float(o[8 * u + 2 * k + 1]) * inv);
                hv[k] = *reinterpret_cast<uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(stage + lane * 128 + 16 * (u ^ (lane & 7))) =
                  make_uint4(hv[0], hv[1], hv[2], hv[3]);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = (lane >> 3) + 4 * i;
              const uint4 v = *reinterpret_cast<const uint4*>(stage + rr * 128 + 16 * (j ^ (rr & 7)));
              if (rbase + rr < p.rows)
                *reinterpret_cast<uint4*>(oh + (slot * p.rows + rbase + rr) * (int64_t)p.r + col0 + 8 * j) = v;
            }
            __syncwarp();
          }
          tc_fence_before();
          __threadfence();  // this thread's partial rows, before the CTA's segment-done count
        }
        named_sync();
        if (ok && lq == 0) publish_segment_half(p.seg_done + g.b);
        __syncwarp();
        if (ok && lane == 0) arrive_leader(B_O_FREE);
      }
      ++gi;
      have = g.next(p);
    }
    if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
  }
  __syncwarp();

  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<2>(tbase, kTmemCols);
}

// 2-D tensor maps: u8 or bf16 [rows, cols] row-major with a 128-byte-wide,
// 64-row, 128B-swizzled box
inline bool make_map_bytes(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t row_bytes, bool bf16) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) return false;
  const uint64_t elt = bf16 ? 2 : 1;
  cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / elt), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(128 / elt), 64};
  cuuint32_t es[2] = {1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
             const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc8

inline cudaError_t launch_tc_decode_f8(const RunParams& p, cudaStream_t stream, bool pdl = true) {
  CUtensorMap tm_codes, tm_rope, tm_q;
  const uint64_t pool_rows = (uint64_t)p.num_blocks * 64;
  if (!tc8::make_map_bytes(&tm_codes, p.kv, pool_rows, 512, false)) return cudaErrorInvalidValue;
  if (!tc8::make_map_bytes(&tm_rope, p.kv_rope, pool_rows, 128, true)) return cudaErrorInvalidValue;
  if (!tc8::make_map_bytes(&tm_q, p.q, (uint64_t)p.B * p.rows, tc8::kQRowBytes, false)) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(tc8::decode_f8_kernel), (int)tc8::Smem::alloc);
  if (e != cudaSuccess) return e;
  return launch_dependent_opt(pdl, tc8::decode_f8_kernel, dim3(2 * p.W), dim3(tc8::kThreads), tc8::Smem::alloc, stream,
                          tm_codes, tm_rope, tm_q, p);
}

}  // namespace mla
