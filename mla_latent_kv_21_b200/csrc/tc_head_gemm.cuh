// tcgen05 per-head GEMMs of the bf16 decode path (r = 512 or 256, d_nope =
// d_v = 128):
//
//   absorb : q_lat[row, :] = q_nope[row, h, :] . W_UK[h]            (K = 128, 512 outputs)
//            (TransMLA abstract: W_UK is absorbed into the query)
//   combine: out[row, h, :] = o_lat[row, h, :] . W_UV[h]             (K = 512, 128 outputs)
//            where o_lat is the log-sum-exp merge of the split partials
//            (per TPLA shard, then the shards are contracted together, which
//            sums the shard outputs; TPLA abstract)
//
// Both are computed transposed, out^T = W^T . X^T, so that the 128 output
// features of a tile are the MMA's M = 128 rows (tensor-memory lanes) and the
// query rows (batch x query tokens) are N: one CTA owns one head and one tile
// of 128 output features; the weight tile arrives by TMA as an MN-major A
// operand, the query rows as a K-major B operand, and the fp32 accumulator
// lives in tensor memory. These kernels are bound by reading the weights
// (16.8 MB each for 128 heads) and, for the up-projection, the partials.
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "simt_kernels.cuh"
#include "tc_decode.cuh"

namespace mla {
namespace hg {

constexpr int kThreads = 256;

#ifdef MLA_TRACE
// per CTA (blockIdx.x < 256): globaltimer at entry, operands landed, MMA done, exit
__device__ unsigned long long g_hg_trace[2][256 * 4];
#define MLA_HG_TRACE(kern, k)                                                             \
  do {                                                                                   \
    if (blockIdx.x < 256 && blockIdx.y == 0) {                                           \
      unsigned long long n_;                                                             \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(n_));                             \
      g_hg_trace[kern][blockIdx.x * 4 + (k)] = n_;                                       \
    }                                                                                    \
  } while (0)
#else
#define MLA_HG_TRACE(kern, k) do {} while (0)
#endif

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk16) {
  return row * 128 + ((chunk16 ^ (row & 7)) << 4);
}

// ---------------------------------------------------------------------------
// absorb: grid (H, r / 128 latent tiles, ceil(rows / 128)); block 256. One CTA per
// (head, 128-column latent tile): W_UK[h][:, tile] (32 KB, two MN-major groups
// of 64 latent columns) as the A operand, q_nope rows [N][128] as 2 K-major
// chunks; 8 MMAs into one tensor-memory accumulator. Small CTAs (shared
// memory sized to the query rows: ~41 KB for 32 rows, 64 registers) so that
// four share an SM: the 4 H CTAs of a step (512 at 128 heads) run as one wave
// and spread the 16.8 MB of W_UK over every SM.
// ---------------------------------------------------------------------------
constexpr int kAbsorbMaxN = 128;         // query rows per absorb CTA
struct AbsorbSmem {
  static constexpr uint32_t w = 0;                             // 32 KB
  static constexpr uint32_t x = 32768;                         // 2 x n_pad x 128 B <= 32 KB
  static constexpr uint32_t bars(int n_pad) { return x + 2u * (uint32_t)n_pad * 128u; }
  static constexpr uint32_t misc(int n_pad) { return bars(n_pad) + 64; }
  static constexpr uint32_t alloc(int n_pad) { return misc(n_pad) + 64 + 1024; }
};

__global__ void __launch_bounds__(kThreads, 4)
    absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_wuk,
                     const __grid_constant__ CUtensorMap tm_qn, RunParams p, int n_pad) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  if (threadIdx.x == 0) MLA_HG_TRACE(0, 0);
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int h = blockIdx.x, mt = blockIdx.y;  // head, latent tile [128 mt, +128)
  const int nbt = p.B * p.Lq;
  const int row0 = blockIdx.z * kAbsorbMaxN;
  const int nrows = min(kAbsorbMaxN, nbt - row0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_w = base + AbsorbSmem::bars(n_pad), bar_x = bar_w + 8, bar_done = bar_w + 16;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gbase + AbsorbSmem::misc(n_pad));
  const uint32_t tcols = n_pad <= 32 ? 32 : n_pad <= 64 ? 64 : 128;
  if (threadIdx.x == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_x, 1);
    mbar_init(bar_done, 1);
    fence_mbarrier_init_cluster();
    // the weights do not depend on the previous kernel: fetch them at once
    prefetch_tmap(&tm_wuk);
    prefetch_tmap(&tm_qn);
    mbar_arrive_expect_tx_local(bar_w, 2 * 16384);
  }
  __syncwarp();
  // W_UK[h][:, 128 mt + 64 j .. +64], all 128 d rows: one box per lane
  if (warp == 0 && lane < 2)
    tma_load_2d(base + AbsorbSmem::w + 16384 * lane, &tm_wuk, 128 * mt + 64 * lane, h * p.dn, bar_w);
  if (warp == 0) {
    tmem_alloc<1>(base + AbsorbSmem::misc(n_pad), tcols);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  // q_nope may come from the previous kernel, and that kernel may still read
  // the workspace (prefix sums, query buffer) this kernel writes
  grid_launch_dependents();
  grid_dependency_wait();
  // page prefix sums and length check of this run (all 256 threads of one block)
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) scan_lengths(p);
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx_local(bar_x, 2 * n_pad * 128);
    for (int kc = 0; kc < 2; ++kc)  // q_nope rows [row0, row0 + n_pad), d chunk kc
      tma_load_2d(base + AbsorbSmem::x + kc * n_pad * 128, &tm_qn, h * p.dn + 64 * kc, row0, bar_x);
    if (mbar_wait(bar_w, 0) && mbar_wait(bar_x, 0)) {
      MLA_HG_TRACE(0, 1);
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, n_pad, 1, 0);
      const uint64_t b0 = smem_desc_sw128(base + AbsorbSmem::x, 16, 1024);
      const uint64_t a0 = smem_desc_sw128(base + AbsorbSmem::w, 16384, 1024);
      for (int ks = 0; ks < 8; ++ks) {  // K = 128 = 8 x 16
        const uint64_t ad = a0 + (uint64_t)(128 * ks);  // 16 K rows x 128 B
        const uint64_t bd = b0 + (uint64_t)(((ks >> 2) * n_pad * 128) >> 4) + (uint64_t)(2 * (ks & 3));
        mma_f16<1>(tbase, ad, bd, idesc, ks > 0 ? 1u : 0u);
      }
      tc_commit<1>(bar_done);
    } else {
      record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
  }
  // q_rope columns of the packed query rows (the tile-0 CTA of each head), in
  // 16-byte pieces (d_rope = 64: 8 per row, at most 4 per thread for 128 rows),
  // every load issued before the first store
  if (mt == 0) {
    const uint4* q_rope = static_cast<const uint4*>(p.q_rope);
    uint4* q = static_cast<uint4*>(p.q);
    constexpr int kPer = (kAbsorbMaxN * 8 + kThreads - 1) / kThreads;
    const int total = nrows * 8;
    uint4 v[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int idx = threadIdx.x + k * kThreads;
      if (idx < total) {
        const int64_t row = (int64_t)(row0 + idx / 8) * p.H + h;
        v[k] = __ldg(q_rope + row * 8 + (idx % 8));
      }
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int idx = threadIdx.x + k * kThreads;
      if (idx < total) {
        const int64_t row = (int64_t)(row0 + idx / 8) * p.H + h;
        q[row * ((p.r + p.dr) / 8) + p.r / 8 + (idx % 8)] = v[k];  // row of (r + d_rope) bf16 = 72 pieces
      }
    }
  }
  __syncwarp();
  {
    // warps w and w + 4 share lane quadrant w % 4 (latent columns
    // 32 (w % 4) .. +32 of the tile) and split the rows by 32-row chunks
    const bool done = mbar_wait(bar_done, 0);
    if (threadIdx.x == 0) MLA_HG_TRACE(0, 2);
    if (__all_sync(0xffffffffu, done)) {
      tc_fence_after();
      __nv_bfloat16* q = static_cast<__nv_bfloat16*>(p.q);
      const int quad = warp & 3;
      const int m = 128 * mt + 32 * quad + lane;  // latent column
      for (int c0 = 32 * (warp >> 2); c0 < n_pad; c0 += 64) {
        uint32_t r[32];
        tmem_ld32(tbase + ((uint32_t)(32 * quad) << 16) + c0, r);
        tmem_wait_ld();
        for (int j = 0; j < 32; ++j) {
          const int i = c0 + j;
          if (i >= nrows) continue;
          const int64_t qrow = (int64_t)(row0 + i) * p.H + h;
          const float v = __uint_as_float(r[j]);
          if (p.fp8) {
            // FP8 cache: the query row is [e4m3(q) x r | e5m2(q - e4m3(q)) x r |
            // bf16 q_rope], 2 (r + d_rope) bytes like the bf16 row
            uint8_t* qb = static_cast<uint8_t*>(p.q) + qrow * 2 * (p.r + p.dr);
            const uint32_t hi = cvt_e4m3x2(v, 0.f);
            const float back = e4m3x2_to_float2(hi).x;
            qb[m] = (uint8_t)(hi & 0xFF);
            qb[p.r + m] = (uint8_t)(cvt_e5m2x2(v - back, 0.f) & 0xFF);
          } else {
            q[qrow * (p.r + p.dr) + m] = __float2bfloat16_rn(v);
          }
        }
      }
    } else if (lane == 0) {
      record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc<1>(tbase, tcols);
  if (threadIdx.x == 0) MLA_HG_TRACE(0, 3);
}

// ---------------------------------------------------------------------------
// combine: out[row, h, :] = o_lat[row, h, :] . W_UV[h], where o_lat is the
// log-sum-exp merge of the row's split partials (per TPLA shard; contracting
// over all r latent columns then sums the shard outputs). One kernel:
//   1. W_UV[h] (128 KB, [K = 512][M = 128] as 2 MN-major groups of 64 output
//      columns) is fetched by TMA before the dependency wait, so it overlaps
//      the tail of the decode kernel;
//   2. after the wait, the 512 threads merge the fp16 partials of the CTA's
//      rows (a thread takes a row x 32 latent columns and issues the loads of
//      all its segments at once) and write bf16 o_lat straight into shared
//      memory as the K-major B operand (8 chunks of 64 latent columns,
//      128-byte swizzle), so o_lat never goes to HBM;
//   3. one thread issues the 32 MMAs (M = 128 outputs, N = rows, K = 512);
//   4. 4 warps read the accumulator and write the bf16 output rows.
// grid (H, ceil(rows / 64)); block 512.
// ---------------------------------------------------------------------------
struct CombineSmem {
  static constexpr int kMaxRows = 64;                  // query rows per CTA
  static constexpr uint32_t w = 0;                     // 128 KB
  static constexpr uint32_t x = 131072;                // 8 x N x 128 B
  static constexpr uint32_t bars = x + 8 * kMaxRows * 128;
  static constexpr uint32_t misc = bars + 64;
  static constexpr uint32_t alloc = misc + 64 + 1024;
};

constexpr int kCombineThreads = 512;

template <int S>
__global__ void __launch_bounds__(kCombineThreads, 1)
    combine_tc_kernel(const __grid_constant__ CUtensorMap tm_wuv, RunParams p, int n_pad) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  if (threadIdx.x == 0) MLA_HG_TRACE(1, 0);
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int h = blockIdx.x;
  const int nbt = p.B * p.Lq;
  const int row0 = blockIdx.y * CombineSmem::kMaxRows;
  const int nrows = min(CombineSmem::kMaxRows, nbt - row0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_w = base + CombineSmem::bars, bar_done = bar_w + 16;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gbase + CombineSmem::misc);
  if (threadIdx.x == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_done, 1);
    fence_mbarrier_init_cluster();
    // the weights do not depend on the previous kernels: fetch them at once
    prefetch_tmap(&tm_wuv);
    mbar_arrive_expect_tx_local(bar_w, (uint32_t)p.r * 256u);  // r latent rows x 128 outputs, bf16
  }
  __syncwarp();
  if (warp == 0 && lane < 2 * (p.r / 256)) {  // one 32 KB box per lane
    const int j = lane & 1, k = lane >> 1;  // output columns [64 j, +64), latent rows [256 k, +256)
    tma_load_2d(base + CombineSmem::w + 65536 * j + 32768 * k, &tm_wuv, 64 * j, h * p.r + 256 * k, bar_w);
  }
  if (warp == 0) {
    tmem_alloc<1>(base + CombineSmem::misc, 128);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  grid_launch_dependents();
  // No grid-wide wait for the decode kernel: this grid starts once every decode
  // CTA has passed its setup (all of them resident), and each merge item waits
  // below for its own sequence's segments only, so the sequences that finish
  // early are merged while the last decode pairs still run. The prefix sums and
  // the length flag come from the absorb kernel, complete before the decode
  // kernel started.
  const bool run = *p.lengths_ok != 0;
  if (run) {
    // ---- merge: one item = one row x 32 latent columns (64 bytes of each fp16
    // partial row; the 16 items of a row read it as 1 KB of consecutive
    // bytes). Each thread issues all loads of an item's first 4 segments at
    // once, so the merge costs about two L2 round trips per item.
    const int64_t Gv = virtual_pages(p.cum[p.B], p.B);
    const int64_t lstride = (int64_t)p.rows * S;
    const int64_t ostride = (int64_t)p.rows * p.r;
    const __half* opart = reinterpret_cast<const __half*>(p.o_part);
    const int sl_shift = p.r == 512 ? 4 : 3;  // log2 of the 32-column items per row (r = 512 or 256)
    for (int it = threadIdx.x; it < (n_pad << sl_shift); it += kCombineThreads) {
      const int i = it >> sl_shift, slice = it & ((1 << sl_shift) - 1);
      const int c0 = 32 * slice;
      uint4 packed[4] = {};  // padding rows stay zero
      if (i < nrows) {
        const int bt = row0 + i, b = bt / p.Lq, t = bt % p.Lq, row = t * p.H + h;
        const int sh = c0 / (p.r / S);
        const int64_t lo = page_owner(p.cum[b], b, Gv, p.W) + b;
        const int64_t hi = page_owner(p.cum[b + 1] - 1, b, Gv, p.W) + b;
        // both CTAs of each of the sequence's segments publish their rows, once
        // per latent shard (bounded wait)
        const int32_t want = 2 * S * (int32_t)(hi - lo + 1);
        if (load_acquire_gpu(p.seg_done + b) < want) {
          const uint64_t t0 = ptx::globaltimer_ns();
          bool waited = true;
          while (load_acquire_gpu(p.seg_done + b) < want) {
            if (ptx::globaltimer_ns() - t0 > p.wait_limit_ns) {
              waited = false;
              break;
            }
            __nanosleep(128);
          }
          if (!waited) record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
        }
        const float* lse = p.lse_part + (int64_t)row * S + sh;
        const __half* op = opart + (int64_t)row * p.r + c0;
        // one round of loads per 4 segments; the running maximum moves as the
        // rounds go (a row has at most a few segments, so usually one round)
        float mx = -INFINITY, sum = 0.f, acc[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) acc[k] = 0.f;
        for (int64_t j0 = lo; j0 <= hi; j0 += 4) {
          float l[4];
          uint4 v[4][4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int64_t slot = j0 + k;
            if (slot <= hi) {
              l[k] = lse[slot * lstride];
              const uint4* src = reinterpret_cast<const uint4*>(op + slot * ostride);
#pragma unroll
              for (int q = 0; q < 4; ++q) v[k][q] = src[q];
            } else {
              l[k] = -INFINITY;
#pragma unroll
              for (int q = 0; q < 4; ++q) v[k][q] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          const float mn = fmaxf(mx, fmaxf(fmaxf(l[0], l[1]), fmaxf(l[2], l[3])));  // slot j0 exists
          const float sc = exp2f(mx - mn);  // 0 on the first round
          sum *= sc;
#pragma unroll
          for (int k = 0; k < 32; ++k) acc[k] *= sc;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float wk = exp2f(l[k] - mn);
            sum += wk;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t hw[4] = {v[k][q].x, v[k][q].y, v[k][q].z, v[k][q].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hw[e]));
                acc[8 * q + 2 * e] = fmaf(wk, f.x, acc[8 * q + 2 * e]);
                acc[8 * q + 2 * e + 1] = fmaf(wk, f.y, acc[8 * q + 2 * e + 1]);
              }
            }
          }
          mx = mn;
        }
        const float inv = 1.f / sum;  // sum >= 1: the largest weight is 2^0
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pk[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[8 * q + 2 * k] * inv, acc[8 * q + 2 * k + 1] * inv);
            pk[k] = *reinterpret_cast<uint32_t*>(&h2);
          }
          packed[q] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      // o_lat[row0 + i, h, 8u .. +8] for u = 4 slice + q -> chunk u / 8, row i,
      // 16-byte unit u % 8 of the 128-byte-swizzled K-major operand
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int u = 4 * slice + q;
        *reinterpret_cast<uint4*>(gbase + CombineSmem::x + (u >> 3) * n_pad * 128 + sw128(i, u & 7)) = packed[q];
      }
    }
    fence_proxy_async_smem();  // generic writes -> tensor core reads
  }
  __syncthreads();
  if (run && threadIdx.x == 0) {
    if (mbar_wait(bar_w, 0)) {
      MLA_HG_TRACE(1, 1);
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, n_pad, 1, 0);
      const uint64_t a0 = smem_desc_sw128(base + CombineSmem::w, 65536, 1024);
      const uint64_t b0 = smem_desc_sw128(base + CombineSmem::x, 16, 1024);
      for (int ks = 0; ks < p.r / 16; ++ks) {  // K = r in steps of 16
        const uint64_t ad = a0 + (uint64_t)(128 * ks);
        const uint64_t bd = b0 + (uint64_t)(((ks >> 2) * n_pad * 128) >> 4) + (uint64_t)(2 * (ks & 3));
        mma_f16<1>(tbase, ad, bd, idesc, ks > 0 ? 1u : 0u);
      }
      tc_commit<1>(bar_done);
    } else {
      record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
  }
  __syncwarp();
  if (run && warp < 4) {
    const bool done = mbar_wait(bar_done, 0);
    if (threadIdx.x == 0) MLA_HG_TRACE(1, 2);
    if (__all_sync(0xffffffffu, done)) {
      tc_fence_after();
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      const int e = 32 * warp + lane;  // output feature
      for (int c0 = 0; c0 < n_pad; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tbase + ((uint32_t)(32 * warp) << 16) + c0, r);
        tmem_wait_ld();
        for (int j = 0; j < 32; ++j) {
          const int i = c0 + j;
          if (i < nrows)
            out[((int64_t)(row0 + i) * p.H + h) * p.dv + e] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
      }
    } else if (lane == 0) {
      record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc<1>(tbase, 128);
  if (threadIdx.x == 0) MLA_HG_TRACE(1, 3);
}

// 2-D bf16 row-major [rows, cols] with a (64 columns x box_rows) 128B-swizzled box.
inline bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int pad16(int n) { return (n + 15) / 16 * 16; }



}  // namespace hg

// absorb on tensor cores (bf16, d_nope = 128, r = 512 or 256); also scans the lengths
inline cudaError_t launch_absorb_tc(const RunParams& p, cudaStream_t stream) {
  const int nbt = p.B * p.Lq;
  const int n_pad = hg::pad16(nbt < hg::kAbsorbMaxN ? nbt : hg::kAbsorbMaxN);
  CUtensorMap tm_wuk, tm_qn;
  if (!hg::make_map(&tm_wuk, p.w_uk, (uint64_t)p.H * p.dn, (uint64_t)p.r, 128)) return cudaErrorInvalidValue;
  if (!hg::make_map(&tm_qn, p.q_nope, (uint64_t)nbt, (uint64_t)p.H * p.dn, (uint32_t)n_pad))
    return cudaErrorInvalidValue;
  const uint32_t smem = hg::AbsorbSmem::alloc(n_pad);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(hg::absorb_tc_kernel),
                                    (int)hg::AbsorbSmem::alloc(hg::kAbsorbMaxN));
  if (e != cudaSuccess) return e;
  const dim3 grid(p.H, p.r / 128, (nbt + hg::kAbsorbMaxN - 1) / hg::kAbsorbMaxN);  // 128-column latent tiles
  return launch_dependent(hg::absorb_tc_kernel, grid, dim3(hg::kThreads), smem,
                              stream, tm_wuk, tm_qn, p, n_pad);
}

// split merge (bf16 o_lat into the query buffer) + up-projection on tensor
// cores (bf16, r = 512 or 256, d_v = 128)
inline cudaError_t launch_combine_tc(const RunParams& p, cudaStream_t stream) {
  const int nbt = p.B * p.Lq;
  const int rows_cta = hg::CombineSmem::kMaxRows;
  const int n_pad = hg::pad16(nbt < rows_cta ? nbt : rows_cta);
  CUtensorMap tm_wuv;
  if (!hg::make_map(&tm_wuv, p.w_uv, (uint64_t)p.H * p.r, (uint64_t)p.dv, 256)) return cudaErrorInvalidValue;
  const void* fn = p.S == 1 ? reinterpret_cast<const void*>(hg::combine_tc_kernel<1>)
                            : reinterpret_cast<const void*>(hg::combine_tc_kernel<2>);
  cudaError_t e = ensure_smem_limit(fn, (int)hg::CombineSmem::alloc);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.H, (nbt + rows_cta - 1) / rows_cta);
  return p.S == 1 ? launch_dependent(hg::combine_tc_kernel<1>, grid, dim3(hg::kCombineThreads),
                                     hg::CombineSmem::alloc, stream, tm_wuv, p, n_pad)
                  : launch_dependent(hg::combine_tc_kernel<2>, grid, dim3(hg::kCombineThreads),
                                     hg::CombineSmem::alloc, stream, tm_wuv, p, n_pad);
}

}  // namespace mla
