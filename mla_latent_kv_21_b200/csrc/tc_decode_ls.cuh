// Latent-split tcgen05 decode kernel (bf16, r = 512, d_rope = 64, one shard).
//
// A CTA pair (cluster of 2) works through a worker's pages one 64-token page
// at a time. Unlike the row-split kernel (tc_decode.cuh), each CTA of the pair
// takes all 128 query rows and half of the columns of every cached row:
// latent columns [256 c, 256 c + 256) and RoPE columns [512 + 32 c, +32).
//
//   QK (cta_group::1, M = 128 rows, N = 64 tokens, K = 288): the partial score
//       S_c = Q[:, cols_c] . KV[:, cols_c]^T into tensor memory.
//   exchange: each CTA sends the rows the peer owns (64 of the 128) of its
//       partial score, in fp16, to the peer (st.async, completing on the
//       peer's barrier); the owner adds the two halves: S = S_0 + S_1.
//   softmax: one thread per owned row holds its 64 scores (the full row, so
//       no cross-thread max or sum); online max with lazy rescale, fp32, log2
//       domain; P in bf16.
//   P: written into this CTA's P buffer (its 64 rows) and copied with one bulk
//       shared-to-shared copy into the peer's P buffer, so both CTAs hold P for
//       all 128 rows.
//   PV (cta_group::1, M = 128, N = 256 latent columns of this CTA, K = 64):
//       O_c += P . cKV[:, latent cols_c] from the same shared-memory tile that
//       QK read: every cached byte crosses HBM -> SM once.
//   The row owner sends each group's rescale factor (and, at the end of a
//   split segment, the row sum) to the peer, whose O half of the row it is.
//
// Sources: TPLA abstract (latent cache), TransMLA abstract (absorbed decode
// over the compressed cache), pith.science verdict record for 2502.07864
// (shared multi-query RoPE key).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tc_decode.cuh"

namespace mla {
namespace ls {

#ifdef MLA_TRACE
using tc::g_trace;
using tc::g_trace_ns;
using tc::kTraceKinds;
using tc::kTraceSteps;
using tc::kTraceWorkers;
#endif

constexpr int kThreads = 256;                      // warps: 0 loads, 1 QK, 2 P-free relay, 3 PV, 4-7 rows
constexpr int kLat = 4;                            // latent chunks of 64 columns per CTA
constexpr uint32_t kQLatChunk = 128 * 128;         // 128 rows x 64 columns, 128-byte swizzle
constexpr uint32_t kQRope = 128 * 64;              // 128 rows x 32 columns, 64-byte swizzle
constexpr uint32_t kQBytes = kLat * kQLatChunk + kQRope;
constexpr uint32_t kTLat = 64 * 128;               // 64 tokens x 64 columns
constexpr uint32_t kTRope = 64 * 64;               // 64 tokens x 32 columns
constexpr uint32_t kTileBytes = kLat * kTLat + kTRope;
constexpr int kTiles = 3;
constexpr uint32_t kPBytes = 128 * 128;            // 128 rows x 64 tokens bf16
constexpr uint32_t kRecvBytes = 64 * 128;          // 64 owned rows x 64 tokens fp16
constexpr int kPBufs = 2;                          // P double-buffered: a page's softmax overlaps the previous PV
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                     // 256 columns: O of this CTA's latent half
constexpr uint32_t kTmemS = 256;                   // 2 x 64 columns: partial scores
constexpr float kRescaleThreshold = 8.0f;          // log2 units

struct Smem {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t tiles = q + kQBytes;
  static constexpr uint32_t p = tiles + kTiles * kTileBytes;
  static constexpr uint32_t recv = p + kPBufs * kPBytes;    // [64 rows][128 B], swizzled
  static constexpr uint32_t alpha = recv + kRecvBytes;      // float [2][64]
  static constexpr uint32_t lsum = alpha + 2 * 64 * 4;      // float [64]
  static constexpr uint32_t bars = lsum + 64 * 4;
  static constexpr uint32_t nbars = 32;
  static constexpr uint32_t misc = bars + nbars * 8;        // tmem slot, abort flag
  static constexpr uint32_t total = misc + 64;
  static constexpr uint32_t alloc = total + 1024;
  static_assert(tiles % 1024 == 0 && p % 1024 == 0 && recv % 1024 == 0, "alignment");
  static_assert(alloc <= 232448, "shared memory");
};

// Arrays of 2 are indexed by page parity (except S / recv: see their use).
enum : int {
  B_Q_FULL = 0,        // count 1 (+tx); phase = segment
  B_TILE_FULL = 1,     // [3] count 1 (+tx)
  B_TILE_FREE = 4,     // [3] count 1 (PV commit)
  B_S_FULL = 7,        // [2] count 1 (QK commit)
  B_S_FREE = 9,        // [2] count 4 (2 softmax + 2 export warps)
  B_RECV_FULL = 11,    // count 1 (+tx): the peer's score half for the owned rows
  B_RECV_FREE = 12,    // count 2: the peer's softmax warps have read what this CTA sent
  B_P_FULL = 13,       // [2] count 2 (+tx): own P rows written, own O rows rescaled, peer's rows copied in
  B_P_FREE = 15,       // [2] count 1 (PV commit)
  B_P_PEER_FREE = 17,  // [2] count 1: the peer's PV is done with its P buffer (relayed)
  B_O_READY = 19,      // [2] count 2: the peer's rows of O rescaled (export warps)
  B_PV_DONE = 21,      // count 1 (PV commit)
  B_ALPHA_FULL = 22,   // [2] count 1 (+tx): the peer's rescale factors for its rows
  B_ALPHA_FREE = 24,   // [2] count 2: the peer's export warps have read this CTA's factors
  B_L_FULL = 26,       // count 1 (+tx): the peer's row sums at a segment end
  B_L_FREE = 27,       // count 2: the peer's export warps have read this CTA's row sums
  B_O_FREE = 28,       // count 4: O read out at a segment end
  B_FINAL_QK = 29,
  B_FINAL_PV = 30,
  B_COUNT = 31
};

// Sequential walk over a worker's pages (one 64-token page per step).
struct PageCursor {
  int b, page, pe, seg;
  bool first;
  int64_t g1;
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
    return true;
  }
  __device__ __forceinline__ bool next(const RunParams& p) {
    ++page;
    first = false;
    if (page >= pe) {
      if (b + 1 >= p.B || p.cum[b + 1] >= g1) return false;
      ++b;
      ++seg;
      page = 0;
      pe = (int)(min(p.cum[b + 1], g1) - p.cum[b]);
      first = true;
    }
    return true;
  }
  __device__ __forceinline__ bool last_of_segment() const { return page + 1 >= pe; }
};

// 16-byte unit u of row l in a 128-byte-row buffer, swizzled so that the 8
// units of 8 consecutive rows fall in different banks.
__device__ __forceinline__ uint32_t unit_off(uint32_t l, uint32_t u) {
  return l * 128 + ((u ^ (l & 7)) << 4);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_ls_kernel(const __grid_constant__ CUtensorMap tm_kv128,
                     const __grid_constant__ CUtensorMap tm_kv64,
                     const __grid_constant__ CUtensorMap tm_q128,
                     const __grid_constant__ CUtensorMap tm_q64, RunParams p) {
  using namespace ptx;
  using L = Smem;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int w = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return base + L::bars + 8u * i; };
  auto peer_of = [&](uint32_t local) -> uint32_t { return map_to_cta(local, peer); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc + 8);

  if (threadIdx.x == 0) {
    uint32_t counts[B_COUNT];
    for (int i = 0; i < B_COUNT; ++i) counts[i] = 1;
    counts[B_S_FREE] = counts[B_S_FREE + 1] = 4;
    counts[B_RECV_FREE] = 2;
    counts[B_P_FULL] = counts[B_P_FULL + 1] = 2;
    counts[B_O_READY] = counts[B_O_READY + 1] = 2;
    counts[B_ALPHA_FREE] = counts[B_ALPHA_FREE + 1] = 2;
    counts[B_L_FREE] = 2;
    counts[B_O_FREE] = 4;
    for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), counts[i]);
    fence_mbarrier_init_cluster();
    *abort_flag = 0;
  }
  if (warp == 1) {
    tmem_alloc<1>(base + L::misc, kTmemCols);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  grid_launch_dependents();
  grid_dependency_wait();
  const bool run = *p.lengths_ok != 0;  // uniform across the pair

  auto fail = [&](int code) {
    record_error(p.status, code);
    *abort_flag = 1;
  };
  const int oob_row = (int)(p.num_blocks * 64);
  auto page_row = [&](int b, int page) -> int {
    const int32_t blk = p.block_table[(int64_t)b * p.bt_stride + page];
    if (blk < 0 || blk >= p.num_blocks) {
      record_error(p.status, MLA_ERR_BOUNDS);
      return oob_row;  // past the tensor: TMA fills zeros
    }
    return blk * 64;
  };
  const int col_lat = 256 * (int)rank;       // this CTA's latent columns
  const int col_rope = 512 + 32 * (int)rank;  // this CTA's RoPE columns

  if (!run) {
    // invalid lengths (reported by the length scan): nothing to do
  } else if (warp == 0) {
    // ------------------------------------------------------- tile producer --
    // lanes 0-3 load latent chunk `lane` of every page, lane 4 the RoPE half
    if (lane < kLat + 1) {
      if (lane == 0) {
        prefetch_tmap(&tm_kv128);
        prefetch_tmap(&tm_kv64);
        prefetch_tmap(&tm_q128);
        prefetch_tmap(&tm_q64);
      }
      PageCursor g;
      bool ok = true;
      bool have = g.init(p, w);
      for (int gi = 0; have && ok; ++gi) {
        const int slot = gi % kTiles;
        if (gi >= kTiles) ok = mbar_wait(bar(B_TILE_FREE + slot), ((gi / kTiles) - 1) & 1);
        if (ok && g.first) {
          // new segment: the previous page's QK must be done with Q
          if (gi > 0) ok = mbar_wait(bar(B_S_FULL + ((gi - 1) & 1)), ((gi - 1) >> 1) & 1);
          if (ok) {
            if (lane == 0) mbar_arrive_expect_tx_local(bar(B_Q_FULL), kQBytes);
            const int yq = g.b * p.rows;
            if (lane < kLat)
              tma_load_2d(base + L::q + lane * kQLatChunk, &tm_q128, col_lat + 64 * lane, yq, bar(B_Q_FULL));
            else
              tma_load_2d(base + L::q + kLat * kQLatChunk, &tm_q64, col_rope, yq, bar(B_Q_FULL));
          }
        }
        if (!ok) break;
        if (lane == 0) MLA_TRACE_EV(w, rank, 7, gi);
        const int y = page_row(g.b, g.page);
        const uint32_t dst = base + L::tiles + slot * kTileBytes;
        if (lane == 0) mbar_arrive_expect_tx_local(bar(B_TILE_FULL + slot), kTileBytes);
        if (lane < kLat)
          tma_load_2d(dst + lane * kTLat, &tm_kv128, col_lat + 64 * lane, y, bar(B_TILE_FULL + slot));
        else
          tma_load_2d(dst + kLat * kTLat, &tm_kv64, col_rope, y, bar(B_TILE_FULL + slot));
        have = g.next(p);
      }
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ QK MMA issuer --
    if (lane == 0) {
      const uint32_t idq = idesc_bf16_f32(128, 64, 0, 0);
      const uint64_t qd = smem_desc_sw128(base + L::q, 16, 1024);
      const uint64_t qr = smem_desc_sw64(base + L::q + kLat * kQLatChunk, 16, 512);
      const uint64_t td = smem_desc_sw128(base + L::tiles, 16, 1024);
      const uint64_t tr = smem_desc_sw64(base + L::tiles + kLat * kTLat, 16, 512);
      bool ok = true;
      PageCursor g;
      bool have = g.init(p, w);
      for (int gi = 0; have && ok; ++gi) {
        const int slot = gi % kTiles, sb = gi & 1;
        if (g.first) ok = mbar_wait(bar(B_Q_FULL), g.seg & 1);
        ok = ok && mbar_wait(bar(B_TILE_FULL + slot), (gi / kTiles) & 1);
        if (ok && gi >= 2) ok = mbar_wait(bar(B_S_FREE + sb), ((gi >> 1) - 1) & 1);
        if (!ok) break;
        MLA_TRACE_EV(w, rank, 0, gi);
        tc_fence_after();
        const uint32_t d = tbase + kTmemS + 64 * sb;
        const uint64_t toff = (uint64_t)((slot * kTileBytes) >> 4);
#pragma unroll
        for (int j = 0; j < kLat; ++j)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16<1>(d, qd + (uint64_t)(j * (kQLatChunk >> 4) + 2 * ks),
                       td + toff + (uint64_t)(j * (kTLat >> 4) + 2 * ks), idq, (j | ks) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_f16<1>(d, qr + (uint64_t)(2 * ks), tr + toff + (uint64_t)(2 * ks), idq, 1u);
        tc_commit<1>(bar(B_S_FULL + sb));
        MLA_TRACE_EV(w, rank, 1, gi);
        have = g.next(p);
      }
      tc_commit<1>(bar(B_FINAL_QK));
      if (!mbar_wait(bar(B_FINAL_QK), 0)) ok = false;
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------- P-buffer release relay --
    // the peer copies its P rows into this CTA's P buffer: tell it when this
    // CTA's PV is done with the buffer
    if (lane == 0) {
      bool ok = true;
      PageCursor g;
      bool have = g.init(p, w);
      for (int gi = 0; have && ok; ++gi) {
        const int pb = gi & 1;
        ok = mbar_wait(bar(B_P_FREE + pb), (gi >> 1) & 1);
        if (ok) mbar_arrive_cluster(peer_of(bar(B_P_PEER_FREE + pb)));
        have = g.next(p);
      }
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------ PV MMA issuer --
    if (lane == 0) {
      const uint32_t idp = idesc_bf16_f32(128, 256, 0, 1);
      const uint64_t pd0 = smem_desc_sw128(base + L::p, 16, 1024);
      // MN-major V: the 4 latent chunks of a tile, 8 KB apart
      const uint64_t vd = smem_desc_sw128(base + L::tiles, kTLat, 1024);
      bool ok = true;
      PageCursor g;
      bool have = g.init(p, w);
      for (int gi = 0; have && ok; ++gi) {
        const int slot = gi % kTiles, pb = gi & 1;
        ok = mbar_wait(bar(B_P_FULL + pb), (gi >> 1) & 1) && mbar_wait(bar(B_O_READY + pb), (gi >> 1) & 1);
        if (ok && g.first && g.seg > 0) ok = mbar_wait(bar(B_O_FREE), (g.seg - 1) & 1);
        if (!ok) break;
        MLA_TRACE_EV(w, rank, 2, gi);
        tc_fence_after();
        const uint64_t voff = (uint64_t)((slot * kTileBytes) >> 4);
        const uint64_t pd = pd0 + (uint64_t)((pb * kPBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16<1>(tbase + kTmemO, pd + (uint64_t)(2 * ks), vd + voff + (uint64_t)(128 * ks), idp,
                     (g.first && ks == 0) ? 0u : 1u);
        tc_commit<1>(bar(B_TILE_FREE + slot));
        tc_commit<1>(bar(B_P_FREE + pb));
        tc_commit<1>(bar(B_PV_DONE));
        MLA_TRACE_EV(w, rank, 3, gi);
        have = g.next(p);
      }
      tc_commit<1>(bar(B_FINAL_PV));
      if (!mbar_wait(bar(B_FINAL_PV), 0)) ok = false;
      if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- row warps --
    // warp 4 + q covers tensor-memory lanes (rows) [32 q, 32 q + 32); rows
    // [64 c, 64 c + 64) are owned by CTA c (softmax), the others are the
    // peer's (their partial scores are sent there, their O half rescaled here)
    const int q = warp & 3;
    const int row = 32 * q + lane;                  // query row within the sequence
    const bool own = (q >> 1) == (int)rank;
    const int l = row & 63;                         // index among the owner's 64 rows
    const bool first_warp = (q & 1) == 0;           // the first of the two warps of a role
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const bool row_real = row < p.rows;
    const int t_row = row_real ? row / p.H : 0;
    bool ok = true;
    auto wait = [&](int b, uint32_t parity) {
      if (ok && *abort_flag) ok = false;
      if (ok) ok = mbar_wait(bar(b), parity);
      ok = __all_sync(0xffffffffu, ok);
    };
    auto rescale_o = [&](float a) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t o[32];
        tmem_ld32(tbase + lane_off + kTmemO + c, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * a);
        tmem_st32(tbase + lane_off + kTmemO + c, o);
      }
      tmem_wait_st();
    };
    // O row / lsum -> partial slot of this segment (this CTA's latent half)
    auto write_o = [&](int64_t slot, float inv) {  // fp16, as the combine kernel reads it
      __half* orow = reinterpret_cast<__half*>(p.o_part) + (slot * p.rows + row) * (int64_t)p.r + col_lat;
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t o[32];
        tmem_ld32(tbase + lane_off + kTmemO + c, o);
        tmem_wait_ld();
        if (row_real) {
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint32_t hv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __half2 h2 = __floats2half2_rn(__uint_as_float(o[k + 2 * e]) * inv,
                                             __uint_as_float(o[k + 2 * e + 1]) * inv);
              hv[e] = *reinterpret_cast<uint32_t*>(&h2);
            }
            *reinterpret_cast<uint4*>(orow + c + k) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          }
        }
      }
    };
    // export side: the previous page's rescale factor, O rows of the peer's
    // rows rescaled, O_READY for that page's PV, and its segment end
    struct PageInfo {
      bool first, last;
      int64_t slot;
      int seg;
    };
    PageInfo prev{};
    auto export_tail = [&](int gj, const PageInfo& pg) {
      const int jb = gj & 1;
      if (first_warp && lane == 0 && ok) mbar_arrive_expect_tx_local(bar(B_ALPHA_FULL + jb), 64 * 4);
      wait(B_ALPHA_FULL + jb, (gj >> 1) & 1);
      if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 8, gj);
      const float a = ok ? *reinterpret_cast<const volatile float*>(gbase + L::alpha + (jb * 64 + l) * 4) : 1.f;
      __syncwarp();
      if (ok && lane == 0) mbar_arrive_cluster(peer_of(bar(B_ALPHA_FREE + jb)));
      if (!pg.first && __any_sync(0xffffffffu, a != 1.f)) wait(B_PV_DONE, (gj - 1) & 1);
      if (ok && !pg.first && __any_sync(0xffffffffu, a != 1.f)) rescale_o(a);
      if (ok) tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive_local(bar(B_O_READY + jb));
      if (pg.last) {
        wait(B_PV_DONE, gj & 1);
        if (first_warp && lane == 0 && ok) mbar_arrive_expect_tx_local(bar(B_L_FULL), 64 * 4);
        wait(B_L_FULL, pg.seg & 1);
        const float lv = ok ? *reinterpret_cast<const volatile float*>(gbase + L::lsum + l * 4) : 0.f;
        __syncwarp();
        if (ok && lane == 0) mbar_arrive_cluster(peer_of(bar(B_L_FREE)));
        if (ok) {
          tc_fence_after();
          write_o(pg.slot, lv > 0.f ? 1.f / lv : 0.f);
          tc_fence_before();
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive_local(bar(B_O_FREE));
      }
    };
    PageCursor g;
    bool have = g.init(p, w);
    float m = -INFINITY, lrow = 0.f;
    int gi = 0;
    for (; have; ++gi) {
      const int sb = gi & 1, ab = gi & 1, pb = gi & 1;
      const int64_t slot = w + g.b;
      if (g.first) { m = -INFINITY; lrow = 0.f; }
      if (own) {
        // ---------------------------------------------------- softmax (owner)
        const int64_t Lb = p.seq_lens[g.b];
        const int64_t key0 = (int64_t)g.page * 64;
        const int64_t lim = row_real ? Lb - p.Lq + t_row : -1;  // last visible key
        int64_t nv = lim - key0 + 1;
        nv = nv < 0 ? 0 : (nv > 64 ? 64 : nv);
        const int nvis = (int)nv;
        if (first_warp && lane == 0 && ok) mbar_arrive_expect_tx_local(bar(B_RECV_FULL), kRecvBytes);
        wait(B_S_FULL + sb, (gi >> 1) & 1);
        wait(B_RECV_FULL, gi & 1);
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 4, gi);
        float sc[64];
        if (ok) {
          tc_fence_after();
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + lane_off + kTmemS + 64 * sb, r0);
          tmem_ld32(tbase + lane_off + kTmemS + 64 * sb + 32, r1);
          tmem_wait_ld();
          const uint8_t* rb = gbase + L::recv;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 v = *reinterpret_cast<const uint4*>(rb + unit_off(l, u));
            const uint32_t hv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hv[k]));
              const int j = 8 * u + 2 * k;
              const uint32_t a0 = j < 32 ? r0[j] : r1[j - 32];
              const uint32_t a1 = j + 1 < 32 ? r0[j + 1] : r1[j + 1 - 32];
              sc[j] = __uint_as_float(a0) + f.x;
              sc[j + 1] = __uint_as_float(a1) + f.y;
            }
          }
          tc_fence_before();
        }
        __syncwarp();
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 10, gi);
        if (ok && lane == 0) {
          mbar_arrive_local(bar(B_S_FREE + sb));
          mbar_arrive_cluster(peer_of(bar(B_RECV_FREE)));  // the buffer may be refilled
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j >= nvis) sc[j] = -INFINITY;
          mx = fmaxf(mx, sc[j]);
        }
        const float mt = mx * p.scale_log2;
        float mu = m;
        if (m == -INFINITY || mt > m + kRescaleThreshold) mu = fmaxf(mt, m);
        float alpha = 1.f;
        const bool rescale = mu != m && m != -INFINITY;
        if (rescale) alpha = ex2_approx(m - mu);
        m = mu;
        const float nmu = mu == -INFINITY ? 0.f : -mu;
        uint32_t pk[32];
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const float p0 = ex2_approx(fmaf(sc[j], p.scale_log2, nmu));
          const float p1 = ex2_approx(fmaf(sc[j + 1], p.scale_log2, nmu));
          ps0 += p0;
          ps1 += p1;
          __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
          pk[j >> 1] = *reinterpret_cast<uint32_t*>(&h);
        }
        lrow = lrow * alpha + (ps0 + ps1);
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 11, gi);
        // the rescale factor, to the peer (its O half of this row)
        if (gi >= 2) wait(B_ALPHA_FREE + ab, ((gi >> 1) - 1) & 1);
        if (ok)
          st_async_b32(peer_of(base + L::alpha + (ab * 64 + l) * 4), __float_as_uint(alpha),
                       peer_of(bar(B_ALPHA_FULL + ab)));
        // this CTA's O half of the row, after the previous page's PV
        if (!g.first && __any_sync(0xffffffffu, rescale)) wait(B_PV_DONE, (gi - 1) & 1);
        if (ok && !g.first && __any_sync(0xffffffffu, rescale)) rescale_o(alpha);
        // P buffer pb, here and at the peer, must be free (PV of page gi - 2)
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 12, gi);
        if (gi >= 2) {
          wait(B_P_FREE + pb, ((gi >> 1) - 1) & 1);
          wait(B_P_PEER_FREE + pb, ((gi >> 1) - 1) & 1);
        }
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 13, gi);
        if (ok) {
          uint8_t* prow = gbase + L::p + pb * kPBytes;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(prow + unit_off(row, u)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          fence_proxy_async_smem();
          tc_fence_before();
        }
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 9, gi);
        named_barrier(1, 64);  // both owner warps: their rows are in the P buffer
        if (ok && first_warp && lane == 0) {
          // the peer's rows arrive in this CTA's buffer by bulk copy
          const uint32_t off = L::p + pb * kPBytes + rank * (kPBytes / 2);
          mbar_arrive_expect_tx_local(bar(B_P_FULL + pb), kPBytes / 2);
          bulk_copy_s2s(peer_of(base + off), base + off, kPBytes / 2, peer_of(bar(B_P_FULL + pb)));
        } else if (ok && lane == 0) {
          mbar_arrive_local(bar(B_P_FULL + pb));
        }
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 5, gi);
        if (g.last_of_segment()) {
          // ---- segment end: O / l of this CTA's half, l to the peer, LSE
          wait(B_PV_DONE, gi & 1);
          if (g.seg >= 1) wait(B_L_FREE, (g.seg - 1) & 1);
          if (ok)
            st_async_b32(peer_of(base + L::lsum + l * 4), __float_as_uint(lrow), peer_of(bar(B_L_FULL)));
          if (ok && row_real) p.lse_part[slot * p.rows + row] = lrow > 0.f ? m + log2f(lrow) : kEmptyLse;
          if (ok) {
            tc_fence_after();
            write_o(slot, lrow > 0.f ? 1.f / lrow : 0.f);
            tc_fence_before();
          }
          __syncwarp();
          if (ok && lane == 0) mbar_arrive_local(bar(B_O_FREE));
        }
      } else {
        // --------------------------------------- the peer's rows (export)
        // This page's partial scores go out first; the owner's rescale factor
        // for the previous page (and that page's segment end, if it was one)
        // is handled after, so the peer's softmax never waits a round trip.
        wait(B_S_FULL + sb, (gi >> 1) & 1);
        if (first_warp && lane == 0) MLA_TRACE_EV(w, rank, 6, gi);
        if (gi >= 1) wait(B_RECV_FREE, (gi - 1) & 1);
        uint32_t r0[32], r1[32];
        if (ok) {
          tc_fence_after();
          tmem_ld32(tbase + lane_off + kTmemS + 64 * sb, r0);
          tmem_ld32(tbase + lane_off + kTmemS + 64 * sb + 32, r1);
          tmem_wait_ld();
          tc_fence_before();
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive_local(bar(B_S_FREE + sb));
        if (ok) {
          const uint32_t dst = peer_of(base + L::recv);
          const uint32_t rbar = peer_of(bar(B_RECV_FULL));
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint32_t hv[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int j = 8 * u + 2 * k;
              const float a0 = __uint_as_float(j < 32 ? r0[j] : r1[j - 32]);
              const float a1 = __uint_as_float(j + 1 < 32 ? r0[j + 1] : r1[j + 1 - 32]);
              __half2 h = __floats2half2_rn(a0, a1);
              hv[k] = *reinterpret_cast<uint32_t*>(&h);
            }
            st_async_v4(dst + unit_off(l, u), hv[0], hv[1], hv[2], hv[3], rbar);
          }
        }
        if (gi >= 1) export_tail(gi - 1, prev);
        prev = PageInfo{g.first, g.last_of_segment(), slot, g.seg};
      }
      have = g.next(p);
    }
    if (!own && gi >= 1) export_tail(gi - 1, prev);  // the last page
    if (!ok) fail(MLA_ERR_DEVICE_TIMEOUT);
  }
  __syncwarp();

  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<1>(tbase, kTmemCols);
}

// 2-D bf16 row-major [rows, 576] map with a (box_cols x box_rows) box.
inline bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                     CUtensorMapSwizzle swz) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)576, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)576 * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ls

inline cudaError_t launch_ls_decode(const RunParams& p, cudaStream_t stream) {
  CUtensorMap kv128, kv64, q128, q64;
  const uint64_t kv_rows = (uint64_t)p.num_blocks * 64, q_rows = (uint64_t)p.B * p.rows;
  if (!ls::make_map(&kv128, p.kv, kv_rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !ls::make_map(&kv64, p.kv, kv_rows, 32, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !ls::make_map(&q128, p.q, q_rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !ls::make_map(&q64, p.q, q_rows, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(ls::decode_ls_kernel), (int)ls::Smem::alloc);
  if (e != cudaSuccess) return e;
  return launch_dependent(ls::decode_ls_kernel, dim3(2 * p.W), dim3(ls::kThreads), ls::Smem::alloc, stream,
                          kv128, kv64, q128, q64, p);
}

}  // namespace mla
