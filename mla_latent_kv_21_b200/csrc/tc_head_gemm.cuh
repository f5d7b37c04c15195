// tcgen05 per-head GEMMs of the bf16 decode path (r = 512, d_nope = d_v = 128):
//
//   absorb : q_lat[row, :] = q_nope[row, h, :] . W_UK[h]            (K = 128, 512 outputs)
//            (TransMLA abstract: W_UK is absorbed into the query)
//   up-proj: out[row, h, :] = o_lat[row, h, :] . W_UV[h]             (K = 512, 128 outputs)
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
constexpr int kMaxN = 256;               // query rows per CTA (MMA N)

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk16) {
  return row * 128 + ((chunk16 ^ (row & 7)) << 4);
}

// ---------------------------------------------------------------------------
// absorb: grid (H, 4 latent tiles of 128, ceil(rows / 256)); block 256.
// Shared memory: W tile [K = 128 d_nope][M = 128 latent] as 2 MN-major groups
// of 64 latent columns (16 KB each); q_nope rows [N][128] as 2 K-major chunks.
// ---------------------------------------------------------------------------
struct AbsorbSmem {
  static constexpr uint32_t w = 0;                   // 32 KB
  static constexpr uint32_t x = 32768;               // 2 x N x 128 B <= 64 KB
  static constexpr uint32_t bars = x + 2 * kMaxN * 128;
  static constexpr uint32_t misc = bars + 64;
  static constexpr uint32_t alloc = misc + 64 + 1024;
};

__global__ void __launch_bounds__(kThreads, 1)
    absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_wuk,
                     const __grid_constant__ CUtensorMap tm_qn, RunParams p, int n_pad) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  // page prefix sums and length check of this run (all 256 threads of one block)
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) scan_lengths(p);
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int h = blockIdx.x, mt = blockIdx.y, nt = blockIdx.z;
  const int nbt = p.B * p.Lq;
  const int row0 = nt * kMaxN;
  const int nrows = min(kMaxN, nbt - row0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = base + AbsorbSmem::bars, bar_done = bar_full + 8;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gbase + AbsorbSmem::misc);
  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_done, 1);
    fence_mbarrier_init_cluster();
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc<1>(base + AbsorbSmem::misc, 256);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  bool ok = true;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_wuk);
    prefetch_tmap(&tm_qn);
    const uint32_t bytes = 2 * 16384 + 2 * n_pad * 128;
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(bar_full), "r"(bytes) : "memory");
    for (int j = 0; j < 2; ++j)  // W_UK[h][:, 128 mt + 64 j .. +64], all 128 d rows
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
          :: "r"(base + AbsorbSmem::w + 16384 * j), "l"(reinterpret_cast<uint64_t>(&tm_wuk)),
             "r"(128 * mt + 64 * j), "r"(h * p.dn), "r"(bar_full) : "memory");
    for (int kc = 0; kc < 2; ++kc)  // q_nope rows [row0, row0 + n_pad), d chunk kc
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
          :: "r"(base + AbsorbSmem::x + kc * n_pad * 128), "l"(reinterpret_cast<uint64_t>(&tm_qn)),
             "r"(h * p.dn + 64 * kc), "r"(row0), "r"(bar_full) : "memory");
    ok = mbar_wait<false>(bar_full, 0);
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, n_pad, 1, 0);
      const uint64_t a0 = smem_desc_sw128(base + AbsorbSmem::w, 16384, 1024);
      const uint64_t b0 = smem_desc_sw128(base + AbsorbSmem::x, 16, 1024);
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
  // q_rope columns of the packed query rows (tile 0 only)
  if (mt == 0) {
    const __nv_bfloat16* q_rope = static_cast<const __nv_bfloat16*>(p.q_rope);
    __nv_bfloat16* q = static_cast<__nv_bfloat16*>(p.q);
    for (int idx = threadIdx.x; idx < nrows * p.dr; idx += blockDim.x) {
      const int i = idx / p.dr, e = idx % p.dr, bt = row0 + i;
      q[((int64_t)bt * p.H + h) * (p.r + p.dr) + p.r + e] = q_rope[((int64_t)bt * p.H + h) * p.dr + e];
    }
  }
  __syncwarp();
  if (warp < 4) {
    const bool done = mbar_wait<false>(bar_done, 0);
    if (__all_sync(0xffffffffu, done)) {
      tc_fence_after();
      __nv_bfloat16* q = static_cast<__nv_bfloat16*>(p.q);
      const int m = 32 * warp + lane;  // latent column within the tile
      for (int c0 = 0; c0 < n_pad; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tbase + ((uint32_t)(32 * warp) << 16) + c0, r);
        tmem_wait_ld();
        for (int j = 0; j < 32; ++j) {
          const int i = c0 + j;
          if (i < nrows)
            q[((int64_t)(row0 + i) * p.H + h) * (p.r + p.dr) + 128 * mt + m] =
                __float2bfloat16_rn(__uint_as_float(r[j]));
        }
      }
    } else if (lane == 0) {
      record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc<1>(tbase, 256);
}

// ---------------------------------------------------------------------------
// combine + up-projection: grid (H, ceil(rows / 256)); block 256.
// Shared memory: W_UV[h] [K = 512][M = 128] as 2 MN-major groups of 64 output
// columns (64 KB each); o_lat [N][512] bf16 as 8 K-major chunks.
// ---------------------------------------------------------------------------
struct UprojSmem {
  static constexpr int kMaxRows = 64;                  // query rows per CTA
  static constexpr uint32_t w = 0;                     // 128 KB
  static constexpr uint32_t x = 131072;                // 8 x N x 128 B
  static constexpr uint32_t lse = x + 8 * kMaxRows * 128;  // float [N][2] totals, int64 [N][2] slot range
  static constexpr uint32_t bars = lse + kMaxRows * 2 * 4 + kMaxRows * 2 * 8;
  static constexpr uint32_t misc = bars + 64;
  static constexpr uint32_t alloc = misc + 64 + 1024;
};

template <int S>
__global__ void __launch_bounds__(kThreads, 1)
    uproj_tc_kernel(const __grid_constant__ CUtensorMap tm_wuv, RunParams p, int n_pad) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  if (!*p.lengths_ok) return;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int h = blockIdx.x;
  const int nbt = p.B * p.Lq;
  const int row0 = blockIdx.y * UprojSmem::kMaxRows;
  const int nrows = min(UprojSmem::kMaxRows, nbt - row0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = base + UprojSmem::bars, bar_done = bar_full + 8;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gbase + UprojSmem::misc);
  float* lse_tot = reinterpret_cast<float*>(gbase + UprojSmem::lse);  // [N][S]
  int64_t* seg = reinterpret_cast<int64_t*>(gbase + UprojSmem::lse + UprojSmem::kMaxRows * 2 * 4);
  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_done, 1);
    fence_mbarrier_init_cluster();
    prefetch_tmap(&tm_wuv);
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(bar_full), "r"(131072u) : "memory");
    for (int j = 0; j < 2; ++j)      // output columns [64 j, 64 j + 64)
      for (int k = 0; k < 2; ++k)    // latent rows [256 k, 256 k + 256)
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
            :: "r"(base + UprojSmem::w + 65536 * j + 32768 * k),
               "l"(reinterpret_cast<uint64_t>(&tm_wuv)), "r"(64 * j), "r"(h * p.r + 256 * k),
               "r"(bar_full) : "memory");
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc<1>(base + UprojSmem::misc, 128);
    tmem_relinquish<1>();
  }
  // per-row log2-sum-exp totals over the row's split segments (one warp per row)
  const int64_t G = p.cum[p.B];
  for (int i = warp; i < n_pad; i += kThreads / 32) {
    const int bt = row0 + i;
    if (i >= nrows) continue;
    const int b = bt / p.Lq, t = bt % p.Lq, row = t * p.H + h;
    const int64_t w_lo = page_owner(p.cum[b], G, p.W);
    const int64_t w_hi = page_owner(p.cum[b + 1] - 1, G, p.W);
    for (int s = 0; s < S; ++s) {
      float mx = -INFINITY;
      for (int64_t w = w_lo + lane; w <= w_hi; w += 32)
        mx = fmaxf(mx, p.lse_part[((w + b) * p.rows + row) * S + s]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
      for (int64_t w = w_lo + lane; w <= w_hi; w += 32)
        sum += exp2f(p.lse_part[((w + b) * p.rows + row) * S + s] - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) lse_tot[i * S + s] = mx + log2f(sum);
    }
    if (lane == 0) {
      seg[2 * i] = w_lo;
      seg[2 * i + 1] = w_hi;
    }
  }
  __syncthreads();
  // o_lat rows -> bf16 B operand, K-major 128B swizzle: row i, latent column c
  // in chunk c / 64, 16-byte unit (c % 64) / 8
  const int rs = p.r / S;
  for (int idx = threadIdx.x; idx < n_pad * 64; idx += blockDim.x) {
    const int i = idx >> 6, unit = idx & 63;       // unit = 8 latent columns
    const int c0 = unit * 8;
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = 0.f;
    if (i < nrows) {
      const int bt = row0 + i;
      const int b = bt / p.Lq, t = bt % p.Lq, row = t * p.H + h, s = c0 / rs;
      const float tot = lse_tot[i * S + s];
      for (int64_t w = seg[2 * i]; w <= seg[2 * i + 1]; ++w) {
        const int64_t slot = w + b;
        const float wt = exp2f(p.lse_part[(slot * p.rows + row) * S + s] - tot);
        const float4* src = reinterpret_cast<const float4*>(p.o_part + (slot * p.rows + row) * (int64_t)p.r + c0);
        const float4 v0 = src[0], v1 = src[1];
        a[0] = fmaf(wt, v0.x, a[0]); a[1] = fmaf(wt, v0.y, a[1]);
        a[2] = fmaf(wt, v0.z, a[2]); a[3] = fmaf(wt, v0.w, a[3]);
        a[4] = fmaf(wt, v1.x, a[4]); a[5] = fmaf(wt, v1.y, a[5]);
        a[6] = fmaf(wt, v1.z, a[6]); a[7] = fmaf(wt, v1.w, a[7]);
      }
    }
    uint32_t pk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(a[2 * k], a[2 * k + 1]);
      pk[k] = *reinterpret_cast<uint32_t*>(&h2);
    }
    const int chunk = unit >> 3, u16 = unit & 7;
    *reinterpret_cast<uint4*>(gbase + UprojSmem::x + chunk * n_pad * 128 + sw128(i, u16)) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  if (threadIdx.x == 0) {
    if (mbar_wait<false>(bar_full, 0)) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, n_pad, 1, 0);
      const uint64_t a0 = smem_desc_sw128(base + UprojSmem::w, 65536, 1024);
      const uint64_t b0 = smem_desc_sw128(base + UprojSmem::x, 16, 1024);
      for (int ks = 0; ks < 32; ++ks) {  // K = 512 = 32 x 16
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
  if (warp < 4) {
    const bool done = mbar_wait<false>(bar_done, 0);
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

// absorb on tensor cores (bf16, d_nope = 128, r = 512); also scans the lengths
inline cudaError_t launch_absorb_tc(const RunParams& p, cudaStream_t stream) {
  const int nbt = p.B * p.Lq;
  const int n_pad = hg::pad16(nbt < hg::kMaxN ? nbt : hg::kMaxN);
  CUtensorMap tm_wuk, tm_qn;
  if (!hg::make_map(&tm_wuk, p.w_uk, (uint64_t)p.H * p.dn, (uint64_t)p.r, 128)) return cudaErrorInvalidValue;
  if (!hg::make_map(&tm_qn, p.q_nope, (uint64_t)nbt, (uint64_t)p.H * p.dn, (uint32_t)n_pad))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(hg::absorb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)hg::AbsorbSmem::alloc);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.H, p.r / 128, (nbt + hg::kMaxN - 1) / hg::kMaxN);
  hg::absorb_tc_kernel<<<grid, hg::kThreads, hg::AbsorbSmem::alloc, stream>>>(tm_wuk, tm_qn, p, n_pad);
  return cudaGetLastError();
}

// combine + up-projection on tensor cores (bf16, r = 512, d_v = 128)
inline cudaError_t launch_uproj_tc(const RunParams& p, cudaStream_t stream) {
  const int nbt = p.B * p.Lq;
  const int rows_cta = hg::UprojSmem::kMaxRows;
  const int n_pad = hg::pad16(nbt < rows_cta ? nbt : rows_cta);
  CUtensorMap tm_wuv;
  if (!hg::make_map(&tm_wuv, p.w_uv, (uint64_t)p.H * p.r, (uint64_t)p.dv, 256)) return cudaErrorInvalidValue;
  const dim3 grid(p.H, (nbt + rows_cta - 1) / rows_cta);
  cudaError_t e;
  if (p.S == 1) {
    e = cudaFuncSetAttribute(hg::uproj_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)hg::UprojSmem::alloc);
    if (e != cudaSuccess) return e;
    hg::uproj_tc_kernel<1><<<grid, hg::kThreads, hg::UprojSmem::alloc, stream>>>(tm_wuv, p, n_pad);
  } else {
    e = cudaFuncSetAttribute(hg::uproj_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)hg::UprojSmem::alloc);
    if (e != cudaSuccess) return e;
    hg::uproj_tc_kernel<2><<<grid, hg::kThreads, hg::UprojSmem::alloc, stream>>>(tm_wuv, p, n_pad);
  }
  return cudaGetLastError();
}

}  // namespace mla
