// Prefill in the MLA (non-absorbed) form on tcgen05 tensor cores (bf16,
// r = 512, d_rope = 64, d_nope = d_v = 128).
//
// TPLA's abstract separates the two phases: prefill, compute-bound, keeps the
// MLA form; decode, memory-bound, uses the absorbed (or TPLA) form. In the MLA
// form every head's keys and values are recovered from the latent rows:
//
//   K_nope[h, t, :] = cKV[t] . W_UK[h]^T     V[h, t, :] = cKV[t] . W_UV[h]
//   out[t, h, :] = softmax_j<=t(scale (q_nope[t,h] . K_nope[h,j] + q_rope[t,h] . k_rope[j])) . V[h, :]
//
// with causal attention inside each sequence (the prompt's tokens attend to
// themselves and to earlier tokens). Two kernels:
//
//   uproj: per 128-token tile the latent rows (128 x 512, 128 KB) stay in
//          shared memory while the CTA walks its heads; per head W_UK[h]
//          (K-major) and W_UV[h] (MN-major) stream through a 3-stage TMA ring
//          in 64-column K chunks, 8 MMAs (M = 128 tokens, N = 128, K = 64) per
//          chunk into two tensor-memory accumulators (K_nope and V), double
//          buffered across heads so the epilogue of one head overlaps the
//          MMAs of the next. K_nope and V go to the workspace as [H, T, 128].
//   attn:  flash attention, one CTA per (128-query tile, head, sequence),
//          longest tiles launched first. Q (128 x 192: two q_nope chunks and
//          the q_rope chunk) stays in shared memory; key tiles of 128 stream
//          through a 5-slot ring of 16 KB items (two K_nope chunks, the k_rope
//          chunk read straight from the latent rows) and a 2-slot ring of
//          V tiles (32 KB, MN-major). S = Q K^T (M = 128, N = 128, K = 192) in
//          one of two tensor-memory buffers; four softmax warps (one query
//          row per thread, fp32, log2 domain, lazy max with threshold 2^8)
//          write P (bf16 pairs) to tensor memory; O += P V (N = 128, K = 128)
//          in tensor memory, P the MMA's A operand straight from there. The QK of tile j + 1 is issued before the PV of
//          tile j, so the tensor core works while the softmax of tile j runs.
//
// Every wait is bounded (p.wait_limit_ns) and records MLA_ERR_DEVICE_TIMEOUT.
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tc_decode.cuh"

namespace mla {

struct PrefillParams {
  const void* q_nope;          // [T, H, dn] bf16
  const void* q_rope;          // [T, H, dr] bf16
  const void* kv;              // [T, r + dr] bf16 latent rows of the prompt tokens
  const int32_t* cu_seqlens;   // [B + 1] device: sequence b owns tokens [cu[b], cu[b+1])
  const void* w_uk;            // [H, dn, r]
  const void* w_uv;            // [H, r, dv]
  void* out;                   // [T, H, dv] bf16
  int32_t* status;             // workspace status word
  void* k_nope;                // workspace [H, T, dn] bf16
  void* v;                     // workspace [H, T, dv] bf16
  int64_t T;
  int32_t B, H, r, dr, dn, dv;
  int32_t num_q_tiles;         // ceil(max length / 128)
  float scale_log2;            // softmax_scale * log2(e)
  uint64_t wait_limit_ns;
};

namespace pf {

using tc::sw128;

constexpr int kThreads = 256;
constexpr int kTile = 128;       // tokens per up-projection tile, queries / keys per attention tile
constexpr int kUpHeads = 16;     // heads per up-projection CTA

// ------------------------------------------------------------ up-projection --
struct UpSmem {
  static constexpr uint32_t a = 0;                    // 8 chunks x [128 tokens][64] bf16
  static constexpr uint32_t ring = 8 * 16384;         // 3 stages x (UK chunk 16 KB + UV chunk 16 KB)
  static constexpr int kStages = 3;
  static constexpr uint32_t kStageBytes = 32768;
  static constexpr uint32_t bars = ring + kStages * kStageBytes;
  static constexpr uint32_t misc = bars + 128;
  static constexpr uint32_t alloc = misc + 64 + 1024;
  static_assert(alloc <= 227 * 1024, "shared memory of one CTA");
};
enum : int { U_A_FULL = 0, U_B_FULL = 1, U_B_EMPTY = 4, U_D_FULL = 7, U_D_EMPTY = 9, U_COUNT = 11 };

__global__ void __launch_bounds__(kThreads, 1)
    uproj_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_wuk,
                 const __grid_constant__ CUtensorMap tm_wuv, PrefillParams p) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)blockIdx.x * kTile;
  const int h0 = blockIdx.y * kUpHeads;
  const int nh = min(kUpHeads, p.H - h0);
  auto bar = [&](int i) -> uint32_t { return base + UpSmem::bars + 8u * i; };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gbase + UpSmem::misc);

  if (threadIdx.x == 0) {
    mbar_init(bar(U_A_FULL), 1);
    for (int i = 0; i < UpSmem::kStages; ++i) {
      mbar_init(bar(U_B_FULL + i), 1);
      mbar_init(bar(U_B_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(U_D_FULL + i), 1);
      mbar_init(bar(U_D_EMPTY + i), 4);  // the four epilogue warps
    }
    fence_mbarrier_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc<1>(base + UpSmem::misc, 512);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tmap(&tm_kv);
      prefetch_tmap(&tm_wuk);
      prefetch_tmap(&tm_wuv);
      // the latent rows of this token tile: 8 boxes of 64 columns x 128 rows
      mbar_arrive_expect_tx_local(bar(U_A_FULL), 8 * 16384);
      for (int kc = 0; kc < 8; ++kc)
        tma_load_2d(base + UpSmem::a + kc * 16384, &tm_kv, 64 * kc, (int32_t)t0, bar(U_A_FULL));
      uint32_t it = 0;
      for (int hi = 0; hi < nh && ok; ++hi) {
        const int h = h0 + hi;
        for (int kc = 0; kc < 8 && ok; ++kc, ++it) {
          const int st = it % UpSmem::kStages;
          if (it >= (uint32_t)UpSmem::kStages)
            ok = mbar_wait(bar(U_B_EMPTY + st), ((it / UpSmem::kStages) - 1) & 1, p.wait_limit_ns);
          if (!ok) break;
          const uint32_t dst = base + UpSmem::ring + st * UpSmem::kStageBytes;
          mbar_arrive_expect_tx_local(bar(U_B_FULL + st), UpSmem::kStageBytes);
          // W_UK[h][:, 64 kc .. +64]: 128 rows (d_nope) x 64 latent columns, K-major
          tma_load_2d(dst, &tm_wuk, 64 * kc, h * p.dn, bar(U_B_FULL + st));
          // W_UV[h][64 kc .. +64, :]: 64 latent rows x 128 outputs as two 64-column halves (MN-major)
          tma_load_2d(dst + 16384, &tm_wuv, 0, h * p.r + 64 * kc, bar(U_B_FULL + st));
          tma_load_2d(dst + 16384 + 8192, &tm_wuv, 64, h * p.r + 64 * kc, bar(U_B_FULL + st));
        }
      }
      if (!ok) record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idesc_k = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_v = idesc_bf16_f32(128, 128, 0, 1);
      const uint64_t a0 = smem_desc_sw128(base + UpSmem::a, 16, 1024);
      ok = mbar_wait(bar(U_A_FULL), 0, p.wait_limit_ns);
      uint32_t it = 0;
      for (int hi = 0; hi < nh && ok; ++hi) {
        const int db = hi & 1;
        if (hi >= 2) ok = mbar_wait(bar(U_D_EMPTY + db), ((hi >> 1) - 1) & 1, p.wait_limit_ns);
        if (!ok) break;
        const uint32_t d_k = tbase + db * 256, d_v = d_k + 128;
        for (int kc = 0; kc < 8 && ok; ++kc, ++it) {
          const int st = it % UpSmem::kStages;
          ok = mbar_wait(bar(U_B_FULL + st), (it / UpSmem::kStages) & 1, p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sbase = base + UpSmem::ring + st * UpSmem::kStageBytes;
          const uint64_t bk = smem_desc_sw128(sbase, 16, 1024);
          const uint64_t bv = smem_desc_sw128(sbase + 16384, 8192, 1024);
          const uint64_t ad = a0 + (uint64_t)((kc * 16384) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint32_t acc = (kc | ks) ? 1u : 0u;
            mma_f16<1>(d_k, ad + (uint64_t)(2 * ks), bk + (uint64_t)(2 * ks), idesc_k, acc);
            mma_f16<1>(d_v, ad + (uint64_t)(2 * ks), bv + (uint64_t)(128 * ks), idesc_v, acc);
          }
          tc_commit<1>(bar(U_B_EMPTY + st));
        }
        if (ok) tc_commit<1>(bar(U_D_FULL + db));
      }
      if (!ok) record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const int row = 32 * quad + lane;
    const int64_t t = t0 + row;
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    __nv_bfloat16* kout = static_cast<__nv_bfloat16*>(p.k_nope);
    __nv_bfloat16* vout = static_cast<__nv_bfloat16*>(p.v);
    for (int hi = 0; hi < nh; ++hi) {
      const int db = hi & 1;
      if (ok) ok = mbar_wait(bar(U_D_FULL + db), (hi >> 1) & 1, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int h = h0 + hi;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        __nv_bfloat16* dst = (half ? vout : kout) + ((int64_t)h * p.T + t) * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t v[32];
          tmem_ld32(tbase + lane_off + db * 256 + half * 128 + c, v);
          tmem_wait_ld();
          if (t < p.T) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint32_t w4[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * u + 2 * k]),
                                                          __uint_as_float(v[8 * u + 2 * k + 1]));
                w4[k] = *reinterpret_cast<uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(dst + c + 8 * u) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_local(bar(U_D_EMPTY + db));
    }
    if (!ok && lane == 0) record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
  }
  // the attention kernel may start its setup now; it waits for this grid's
  // K_nope / V before reading them
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<1>(tbase, 512);
}

// ---------------------------------------------------------------- attention --
struct AttnSmem {
  static constexpr uint32_t q = 0;                    // 3 chunks x [128 rows][64] bf16
  static constexpr int kKSlots = 5;                   // 16 KB: K_nope chunk 0, 1, k_rope
  static constexpr int kVSlots = 2;                   // 32 KB: V tile, two 64-column halves
  static constexpr uint32_t k = 3 * 16384;
  static constexpr uint32_t v = k + kKSlots * 16384;
  static constexpr uint32_t bars = v + kVSlots * 32768;
  static constexpr uint32_t misc = bars + 256;
  static constexpr uint32_t alloc = misc + 64 + 1024;
  static_assert(alloc <= 227 * 1024, "shared memory of one CTA");
};
enum : int {
  A_Q_FULL = 0, A_K_FULL = 1, A_K_EMPTY = 6, A_V_FULL = 11, A_V_EMPTY = 13, A_S_FULL = 15,
  A_S_EMPTY = 17, A_P_FULL = 19, A_P_EMPTY = 20, A_COUNT = 21
};
constexpr float kPrefillRescaleThreshold = 8.0f;  // log2 units

// Paired float arithmetic of sm_100 (one instruction for two lanes' worth of
// work, each element rounded as the scalar instruction rounds it) and the
// three-input max: the softmax issues fewer instructions per score.
__device__ __forceinline__ uint64_t pair_f32(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpair_f32(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// D += A x B with A in tensor memory (cta_group::1): A's M rows are the lanes
// from a_tmem on, its K elements run along the columns, two 16-bit elements
// per 32-bit column (element 2c in the low half of column c); B is a shared
// memory descriptor as for ptx::mma_f16.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      :: "r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Optional event trace (compile with -DMLA_TRACE): SM clock of per-item
// events of the first attention CTA (its longest query tile), read back with
// mla_debug_trace_pf_read(). Kinds: 0 K item load issued, 1 K item seen full
// by the MMA issuer, 2 V tile load issued, 3 P seen full by the MMA issuer,
// 4 V seen full (PV issued), 5 S seen full by the softmax, 6 the softmax may
// write P, 7 P written.
#ifdef MLA_TRACE
constexpr int kPfTraceItems = 256;
__device__ unsigned long long g_pf_trace[8 * kPfTraceItems];
#define MLA_PF_TRACE(kind, idx)                                                          \
  do {                                                                                   \
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (idx) < kPfTraceItems) { \
      unsigned long long t_;                                                             \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_));                                 \
      g_pf_trace[(kind) * kPfTraceItems + (idx)] = t_;                                   \
    }                                                                                    \
  } while (0)
#else
#define MLA_PF_TRACE(kind, idx) do {} while (0)
#endif

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_qr,
                const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_kr,
                const __grid_constant__ CUtensorMap tm_v, PrefillParams p) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  const int b = blockIdx.z, h = blockIdx.y;
  const int qt = p.num_q_tiles - 1 - (int)blockIdx.x;   // longest tiles first
  const int64_t seq0 = p.cu_seqlens[b];
  const int64_t L = (int64_t)p.cu_seqlens[b + 1] - seq0;
  if (L <= 0 || (int64_t)qt * kTile >= L) return;       // this sequence has no such tile (uniform)
  const int nkt = qt + 1;                                 // causal: key tiles 0 .. qt

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return base + AttnSmem::bars + 8u * i; };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gbase + AttnSmem::misc);

  if (threadIdx.x == 0) {
    uint32_t counts[A_COUNT];
    for (int i = 0; i < A_COUNT; ++i) counts[i] = 1;
    counts[A_S_EMPTY] = counts[A_S_EMPTY + 1] = 4;  // the four softmax warps
    counts[A_P_FULL] = 4;
    for (int i = 0; i < A_COUNT; ++i) mbar_init(bar(i), counts[i]);
    fence_mbarrier_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc<1>(base + AttnSmem::misc, 512);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t kTmemO = 256;  // O: columns [256, 384); S: two buffers of 128 columns from 0
  const uint32_t kTmemP = 384;  // P (bf16 pairs): columns [384, 448), the A operand of P V
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tmap(&tm_qn);
      prefetch_tmap(&tm_qr);
      prefetch_tmap(&tm_kn);
      prefetch_tmap(&tm_kr);
      prefetch_tmap(&tm_v);
      // the queries are inputs: load them before waiting for the up-projection
      const int32_t q0 = (int32_t)(seq0 + (int64_t)qt * kTile);
      mbar_arrive_expect_tx_local(bar(A_Q_FULL), 3 * 16384);
      tma_load_3d(base + AttnSmem::q, &tm_qn, 0, h, q0, bar(A_Q_FULL));
      tma_load_3d(base + AttnSmem::q + 16384, &tm_qn, 64, h, q0, bar(A_Q_FULL));
      tma_load_3d(base + AttnSmem::q + 32768, &tm_qr, 0, h, q0, bar(A_Q_FULL));
      grid_dependency_wait();  // K_nope and V of the up-projection
      uint32_t kc = 0;
      for (int j = 0; j < nkt && ok; ++j) {
        const int32_t key0 = (int32_t)(seq0 + (int64_t)j * kTile);   // token row of the tile's first key
        const int32_t krow = (int32_t)((int64_t)h * p.T + key0);     // its row in [H * T, 128]
        for (int i = 0; i < 3 && ok; ++i, ++kc) {
          const int slot = kc % AttnSmem::kKSlots;
          if (kc >= (uint32_t)AttnSmem::kKSlots)
            ok = mbar_wait(bar(A_K_EMPTY + slot), ((kc / AttnSmem::kKSlots) - 1) & 1, p.wait_limit_ns);
          if (!ok) break;
          const uint32_t dst = base + AttnSmem::k + slot * 16384;
          MLA_PF_TRACE(0, kc);
          mbar_arrive_expect_tx_local(bar(A_K_FULL + slot), 16384);
          if (i < 2) tma_load_2d(dst, &tm_kn, 64 * i, krow, bar(A_K_FULL + slot));
          else tma_load_2d(dst, &tm_kr, p.r, key0, bar(A_K_FULL + slot));  // k_rope: latent-row columns [r, r + 64)
        }
        if (!ok) break;
        const int vs = j % AttnSmem::kVSlots;
        if (j >= AttnSmem::kVSlots)
          ok = mbar_wait(bar(A_V_EMPTY + vs), ((j / AttnSmem::kVSlots) - 1) & 1, p.wait_limit_ns);
        if (!ok) break;
        const uint32_t dst = base + AttnSmem::v + vs * 32768;
        MLA_PF_TRACE(2, j);
        mbar_arrive_expect_tx_local(bar(A_V_FULL + vs), 32768);
        tma_load_2d(dst, &tm_v, 0, krow, bar(A_V_FULL + vs));
        tma_load_2d(dst + 16384, &tm_v, 64, krow, bar(A_V_FULL + vs));
      }
      if (!ok) record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
      const uint64_t q_desc = smem_desc_sw128(base + AttnSmem::q, 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(base + AttnSmem::k, 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(base + AttnSmem::v, 16384, 1024);
      uint32_t kc = 0;
      ok = mbar_wait(bar(A_Q_FULL), 0, p.wait_limit_ns);
      auto issue_qk = [&](int j) {
        const int sb = j & 1;
        if (j >= 2) ok = ok && mbar_wait(bar(A_S_EMPTY + sb), ((j >> 1) - 1) & 1, p.wait_limit_ns);
        for (int i = 0; i < 3 && ok; ++i, ++kc) {
          const int slot = kc % AttnSmem::kKSlots;
          ok = mbar_wait(bar(A_K_FULL + slot), (kc / AttnSmem::kKSlots) & 1, p.wait_limit_ns);
          if (!ok) break;
          MLA_PF_TRACE(1, kc);
          tc_fence_after();
          const uint64_t ad = q_desc + (uint64_t)((i * 16384) >> 4);
          const uint64_t bd = k_desc + (uint64_t)((slot * 16384) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16<1>(tbase + sb * 128, ad + (uint64_t)(2 * ks), bd + (uint64_t)(2 * ks), idesc_s,
                       (i | ks) ? 1u : 0u);
          tc_commit<1>(bar(A_K_EMPTY + slot));
        }
        if (ok) tc_commit<1>(bar(A_S_FULL + sb));
      };
      if (ok) issue_qk(0);
      for (int j = 0; j < nkt && ok; ++j) {
        if (j + 1 < nkt) issue_qk(j + 1);
        if (!ok) break;
        const int vs = j % AttnSmem::kVSlots;
        ok = mbar_wait(bar(A_P_FULL), j & 1, p.wait_limit_ns);
        MLA_PF_TRACE(3, j);
        ok = ok && mbar_wait(bar(A_V_FULL + vs), (j / AttnSmem::kVSlots) & 1, p.wait_limit_ns);
        if (!ok) break;
        MLA_PF_TRACE(4, j);
        tc_fence_after();
        const uint64_t vd = v_desc + (uint64_t)((vs * 32768) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // K = 16 keys per MMA: 8 columns of P
          mma_f16_ts(tbase + kTmemO, tbase + kTmemP + 8 * ks, vd + (uint64_t)(128 * ks), idesc_o,
                     (j | ks) ? 1u : 0u);
        tc_commit<1>(bar(A_V_EMPTY + vs));
        tc_commit<1>(bar(A_P_EMPTY));
      }
      if (!ok) record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax --
    const int quad = warp & 3;
    const int row = 32 * quad + lane;                    // query row of the tile
    const int64_t tq = (int64_t)qt * kTile + row;        // its position in the sequence
    const bool row_real = tq < L;
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    float m = -INFINITY, l = 0.f;
    auto wait = [&](int bi, uint32_t parity) {
      if (ok) ok = mbar_wait(bar(bi), parity, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
    };
    for (int j = 0; j < nkt; ++j) {
      const int sb = j & 1;
      wait(A_S_FULL + sb, (j >> 1) & 1);
      if (row == 0) MLA_PF_TRACE(5, j);
      uint32_t r[128];
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32)
          tmem_ld32(tbase + lane_off + sb * 128 + c0, *reinterpret_cast<uint32_t(*)[32]>(r + c0));
        tmem_wait_ld();
        tc_fence_before();
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive_local(bar(A_S_EMPTY + sb));
      // visible keys of this row in tile j: k <= tq (causal) and k < L
      const int64_t lim = row_real ? tq : -1;
      int64_t nv = lim - (int64_t)j * kTile + 1;
      nv = nv < 0 ? 0 : (nv > 128 ? 128 : nv);
      const int nvis = (int)nv;
      if (nvis < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= nvis) r[c] = 0xff800000u;
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        mx0 = max3(mx0, __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
        mx1 = max3(mx1, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
      }
      const float mt = fmaxf(mx0, mx1) * p.scale_log2;
      float mu = m;
      if (m == -INFINITY || mt > m + kPrefillRescaleThreshold) mu = fmaxf(mt, m);
      float alpha = 1.f;
      const bool rescale = mu != m && m != -INFINITY;
      if (rescale) alpha = ex2_approx(m - mu);
      m = mu;
      const float nmu = mu == -INFINITY ? 0.f : -mu;
      uint32_t pk[64];
      // two pairs of running sums (the same four sums, added pairwise)
      uint64_t ps01 = pair_f32(0.f, 0.f), ps23 = pair_f32(0.f, 0.f);
      const uint64_t sc2 = pair_f32(p.scale_log2, p.scale_log2), nmu2 = pair_f32(nmu, nmu);
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        float x0, x1, x2, x3;
        unpair_f32(fma2(pair_f32(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sc2, nmu2), x0, x1);
        unpair_f32(fma2(pair_f32(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])), sc2, nmu2), x2, x3);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1), p2 = ex2_approx(x2), p3 = ex2_approx(x3);
        ps01 = add2(ps01, pair_f32(p0, p1));
        ps23 = add2(ps23, pair_f32(p2, p3));
        __nv_bfloat162 h0 = __floats2bfloat162_rn(p0, p1);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(p2, p3);
        pk[c >> 1] = *reinterpret_cast<uint32_t*>(&h0);
        pk[(c >> 1) + 1] = *reinterpret_cast<uint32_t*>(&h1);
      }
      float ps0, ps1, ps2, ps3;
      unpair_f32(ps01, ps0, ps1);
      unpair_f32(ps23, ps2, ps3);
      l = l * alpha + ((ps0 + ps1) + (ps2 + ps3));
      // the PV of tile j - 1 is done with P and has added to O
      if (j >= 1) wait(A_P_EMPTY, (j - 1) & 1);
      if (row == 0) MLA_PF_TRACE(6, j);
      if (ok && j >= 1 && __any_sync(0xffffffffu, rescale)) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t o[32];
          tmem_ld32(tbase + lane_off + kTmemO + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(tbase + lane_off + kTmemO + c, o);
        }
        tmem_wait_st();
      }
      if (ok) {
        // P row -> tensor memory: this thread's lane, keys 2c and 2c + 1 in column c
        tmem_st32(tbase + lane_off + kTmemP, *reinterpret_cast<uint32_t(*)[32]>(pk));
        tmem_st32(tbase + lane_off + kTmemP + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
        tmem_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive_local(bar(A_P_FULL));
      if (row == 0) MLA_PF_TRACE(7, j);
    }
    // ---- epilogue: O / l of this row
    wait(A_P_EMPTY, (nkt - 1) & 1);
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + ((seq0 + tq) * p.H + h) * (int64_t)p.dv;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        uint32_t o[32];
        tmem_ld32(tbase + lane_off + kTmemO + c, o);
        tmem_wait_ld();
        if (row_real) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[8 * u + 2 * k]) * inv,
                                                        __uint_as_float(o[8 * u + 2 * k + 1]) * inv);
              w4[k] = *reinterpret_cast<uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(out + c + 8 * u) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      tc_fence_before();
    }
    if (!ok && lane == 0) record_error(p.status, MLA_ERR_DEVICE_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<1>(tbase, 512);
}

// ------------------------------------------------------------------ host ---
// 2-D bf16 row-major [rows, cols] with a (64 columns x box_rows) 128B-swizzled box.
inline bool make_map2(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 [T, H, d] viewed as (d, H, T): box of 64 features x 1 head x 128 tokens.
inline bool make_map_thd(CUtensorMap* m, const void* ptr, uint64_t T, uint64_t H, uint64_t d) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)(H * d * 2)};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kTile};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pf

inline cudaError_t launch_prefill(const PrefillParams& p, cudaStream_t stream, cudaEvent_t ev_start = nullptr,
                                  cudaEvent_t ev_stop = nullptr) {
  const uint64_t width = (uint64_t)p.r + p.dr;
  CUtensorMap tm_kv, tm_wuk, tm_wuv, tm_qn, tm_qr, tm_kn, tm_kr, tm_v;
  if (!pf::make_map2(&tm_kv, p.kv, (uint64_t)p.T, width, pf::kTile) ||
      !pf::make_map2(&tm_wuk, p.w_uk, (uint64_t)p.H * p.dn, (uint64_t)p.r, 128) ||
      !pf::make_map2(&tm_wuv, p.w_uv, (uint64_t)p.H * p.r, (uint64_t)p.dv, 64) ||
      !pf::make_map_thd(&tm_qn, p.q_nope, (uint64_t)p.T, (uint64_t)p.H, (uint64_t)p.dn) ||
      !pf::make_map_thd(&tm_qr, p.q_rope, (uint64_t)p.T, (uint64_t)p.H, (uint64_t)p.dr) ||
      !pf::make_map2(&tm_kn, p.k_nope, (uint64_t)p.H * p.T, (uint64_t)p.dn, pf::kTile) ||
      !pf::make_map2(&tm_kr, p.kv, (uint64_t)p.T, width, pf::kTile) ||
      !pf::make_map2(&tm_v, p.v, (uint64_t)p.H * p.T, (uint64_t)p.dv, pf::kTile))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(pf::uproj_kernel), (int)pf::UpSmem::alloc);
  if (e != cudaSuccess) return e;
  e = ensure_smem_limit(reinterpret_cast<const void*>(pf::attn_kernel), (int)pf::AttnSmem::alloc);
  if (e != cudaSuccess) return e;
  const dim3 gu((unsigned)((p.T + pf::kTile - 1) / pf::kTile), (unsigned)((p.H + pf::kUpHeads - 1) / pf::kUpHeads));
  pf::uproj_kernel<<<gu, pf::kThreads, pf::UpSmem::alloc, stream>>>(tm_kv, tm_wuk, tm_wuv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ev_start && (e = cudaEventRecord(ev_start, stream)) != cudaSuccess) return e;
  const dim3 ga((unsigned)p.num_q_tiles, (unsigned)p.H, (unsigned)p.B);
  e = launch_dependent_opt(ev_start == nullptr, pf::attn_kernel, ga, dim3(pf::kThreads), pf::AttnSmem::alloc, stream,
                           tm_qn, tm_qr, tm_kn, tm_kr, tm_v, p);
  if (e == cudaSuccess && ev_stop) e = cudaEventRecord(ev_stop, stream);
  return e;
}

}  // namespace mla
