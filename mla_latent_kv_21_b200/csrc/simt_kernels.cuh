// CUDA-core kernels of the decode path. They serve every supported shape and
// are the only path for fp32 inputs (the tiny fp32 workload needs 1e-5
// relative accuracy, which bf16 tensor-core operands cannot give). For the
// bf16 workloads the tcgen05 kernels in tc_decode.cuh replace the decode step.
//
// Three steps per run (TPLA abstract, TransMLA abstract "Absorb"):
//   absorb  : q[b,t,h] = [q_nope . W_UK[h] || q_rope]       (+ length scan)
//   decode  : per split segment, online softmax over the latent pages,
//             O_lat / l and log2-sum-exp per row (and per TPLA shard)
//   combine : log-sum-exp merge of the segments, then o_lat . W_UV[h]
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kSimtThreads = 256;
constexpr int kSimtRowGroup = 8;     // query rows per decode CTA
constexpr int kAbsorbRows = 16;      // (b, t) rows per absorb CTA
constexpr int kCombineRows = 8;      // (b, t) rows per combine CTA
constexpr int kMaxNope = 128;

// Page prefix sums and length validation of this run's seq_lens, done by one
// block (all its threads must call it). L_b must lie in [Lq, stride * P].
__device__ void scan_lengths(const RunParams& p) {
  __shared__ int64_t part[kSimtThreads];
  __shared__ int bad;
  const int nt = blockDim.x, tid = threadIdx.x;
  const int chunk = (p.B + nt - 1) / nt;
  const int b0 = min(p.B, tid * chunk), b1 = min(p.B, b0 + chunk);
  if (tid == 0) bad = 0;
  __syncthreads();
  int64_t s = 0;
  int ok = 1;
  const int64_t maxlen = (int64_t)p.bt_stride * p.P;
  for (int b = b0; b < b1; ++b) {
    const int64_t L = p.seq_lens[b];
    if (L < p.Lq || L > maxlen) ok = 0;
    s += ceil_div64(L > 0 ? L : 0, p.P);
  }
  part[tid] = s;
  if (!ok) atomicOr(&bad, 1);
  __syncthreads();
  if (tid == 0) {
    int64_t acc = 0;
    for (int i = 0; i < nt; ++i) {
      const int64_t v = part[i];
      part[i] = acc;
      acc += v;
    }
    p.cum[p.B] = acc;
    *p.lengths_ok = bad ? 0 : 1;
    if (bad) record_error(p.status, MLA_ERR_BOUNDS);
  }
  __syncthreads();
  int64_t acc = part[tid];
  for (int b = b0; b < b1; ++b) {
    p.cum[b] = acc;
    if (p.seg_done) p.seg_done[b] = 0;
    const int64_t L = p.seq_lens[b];
    acc += ceil_div64(L > 0 ? L : 0, p.P);
  }
}

// Largest b with cum[b] <= g (cum strictly increasing; cum[0] = 0 <= g).
__device__ __forceinline__ int find_sequence(const int64_t* cum, int B, int64_t g) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cum[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// absorb: grid (H, ceil(r / 128), ceil(B*Lq / 16)), 128 threads.
// q row (b, t, h) = [sum_d q_nope[b,t,h,d] W_UK[h,d,:] || q_rope[b,t,h,:]]
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) absorb_simt_kernel(RunParams p) {
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) scan_lengths(p);
  __shared__ float qn[kAbsorbRows][kMaxNope + 1];
  const int h = blockIdx.x;
  const int c = blockIdx.y * 128 + threadIdx.x;
  const int bt0 = blockIdx.z * kAbsorbRows;
  const int nbt = p.B * p.Lq;
  const int width = p.r + p.dr;
  const T* q_nope = static_cast<const T*>(p.q_nope);
  const T* q_rope = static_cast<const T*>(p.q_rope);
  const T* w_uk = static_cast<const T*>(p.w_uk);
  T* q = static_cast<T*>(p.q);
  for (int idx = threadIdx.x; idx < kAbsorbRows * p.dn; idx += blockDim.x) {
    const int i = idx / p.dn, d = idx % p.dn, bt = bt0 + i;
    qn[i][d] = bt < nbt ? to_float(q_nope[((int64_t)bt * p.H + h) * p.dn + d]) : 0.f;
  }
  __syncthreads();
  if (c < p.r) {
    float acc[kAbsorbRows];
#pragma unroll
    for (int i = 0; i < kAbsorbRows; ++i) acc[i] = 0.f;
    const T* wcol = w_uk + (int64_t)h * p.dn * p.r + c;
    for (int d = 0; d < p.dn; ++d) {
      const float w = to_float(wcol[(int64_t)d * p.r]);
#pragma unroll
      for (int i = 0; i < kAbsorbRows; ++i) acc[i] = fmaf(qn[i][d], w, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < kAbsorbRows; ++i) {
      const int bt = bt0 + i;
      if (bt < nbt) q[((int64_t)bt * p.H + h) * width + c] = from_float<T>(acc[i]);
    }
  }
  if (blockIdx.y == 0) {
    for (int idx = threadIdx.x; idx < kAbsorbRows * p.dr; idx += blockDim.x) {
      const int i = idx / p.dr, e = idx % p.dr, bt = bt0 + i;
      if (bt < nbt)
        q[((int64_t)bt * p.H + h) * width + p.r + e] = q_rope[((int64_t)bt * p.H + h) * p.dr + e];
    }
  }
}

// ---------------------------------------------------------------------------
// decode: grid (W, ceil(rows / 8)), 256 threads, dynamic shared memory.
// Worker w walks its page range [start(w), start(w+1)) sequence by sequence.
// Query row `row` of sequence b is token t = row / H of head h = row % H.
// ---------------------------------------------------------------------------
inline size_t simt_decode_smem_bytes(int width, int shards, int P) {
  return sizeof(float) * ((size_t)(kSimtRowGroup + P) * (width + 1) +
                          (size_t)shards * kSimtRowGroup * P + 3 * shards * kSimtRowGroup);
}

template <typename T, int S>
__global__ void __launch_bounds__(kSimtThreads) decode_simt_kernel(RunParams p) {
  if (!*p.lengths_ok) return;
  extern __shared__ float smem[];
  const int width = p.r + p.dr, ld = width + 1, P = p.P;
  float* q_s = smem;                                  // [RG][ld]
  float* tile = q_s + kSimtRowGroup * ld;             // [P][ld]
  float* s_s = tile + P * ld;                         // [S][RG][P]
  float* m_s = s_s + S * kSimtRowGroup * P;           // [S][RG]
  float* l_s = m_s + S * kSimtRowGroup;
  float* a_s = l_s + S * kSimtRowGroup;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int w = blockIdx.x, row0 = blockIdx.y * kSimtRowGroup;
  const int64_t g0 = worker_page_start(w, p.cum, p.B, p.W), g1 = worker_page_start(w + 1, p.cum, p.B, p.W);
  if (g0 >= g1) return;
  const T* pool = static_cast<const T*>(p.kv);
  const T* qg = static_cast<const T*>(p.q);
  const int rs = p.r / S;  // latent columns per shard
  constexpr int kCols = 2; // r <= 512 = 2 * 256 columns per thread

  for (int b = find_sequence(p.cum, p.B, g0); b < p.B && p.cum[b] < g1; ++b) {
    const int64_t pb = max(p.cum[b], g0) - p.cum[b];
    const int64_t pe = min(p.cum[b + 1], g1) - p.cum[b];
    const int64_t L = p.seq_lens[b];
    const int64_t slot = w + b;
    for (int idx = tid; idx < kSimtRowGroup * width; idx += blockDim.x) {
      const int i = idx / width, k = idx % width, row = row0 + i;
      q_s[i * ld + k] = row < p.rows ? to_float(qg[((int64_t)b * p.rows + row) * width + k]) : 0.f;
    }
    if (tid < S * kSimtRowGroup) {
      m_s[tid] = -INFINITY;
      l_s[tid] = 0.f;
    }
    float acc[kCols][kSimtRowGroup];
#pragma unroll
    for (int u = 0; u < kCols; ++u)
#pragma unroll
      for (int i = 0; i < kSimtRowGroup; ++i) acc[u][i] = 0.f;
    __syncthreads();

    for (int64_t page = pb; page < pe; ++page) {
      const int32_t blk = p.block_table[(int64_t)b * p.bt_stride + page];
      int valid = (int)(L - page * P < P ? L - page * P : P);
      if (blk < 0 || blk >= p.num_blocks) {
        if (tid == 0) record_error(p.status, MLA_ERR_BOUNDS);
        valid = 0;
      }
      const T* src = pool + (int64_t)(valid > 0 ? blk : 0) * P * width;
      for (int idx = tid; idx < P * width; idx += blockDim.x) {
        const int j = idx / width, k = idx % width;
        tile[j * ld + k] = j < valid ? to_float(src[idx]) : 0.f;
      }
      __syncthreads();
      // scores, log2 domain
      for (int pr = tid; pr < kSimtRowGroup * P; pr += blockDim.x) {
        const int i = pr / P, j = pr % P, row = row0 + i;
        const int t = row / p.H;
        const bool vis = row < p.rows && j < valid && page * P + j <= L - p.Lq + t;
        const float* qr = q_s + i * ld;
        const float* kr = tile + j * ld;
        float rope = 0.f;
        for (int k = p.r; k < width; ++k) rope = fmaf(qr[k], kr[k], rope);
#pragma unroll
        for (int s = 0; s < S; ++s) {
          float dot = rope;
          for (int k = s * rs; k < (s + 1) * rs; ++k) dot = fmaf(qr[k], kr[k], dot);
          s_s[(s * kSimtRowGroup + i) * P + j] = vis ? dot * p.scale_log2 : -INFINITY;
        }
      }
      __syncthreads();
      // online softmax, one warp per (shard, row); P = 64 -> two keys per lane
      for (int sr = warp; sr < S * kSimtRowGroup; sr += kSimtThreads / 32) {
        float* sv = s_s + sr * P;
        const float v0 = sv[lane], v1 = sv[lane + 32];
        float mx = fmaxf(v0, v1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_old = m_s[sr];
        const float m_new = fmaxf(m_old, mx);
        float p0 = 0.f, p1 = 0.f, alpha = 1.f;
        if (m_new != -INFINITY) {
          p0 = exp2f(v0 - m_new);
          p1 = exp2f(v1 - m_new);
          alpha = exp2f(m_old - m_new);
        }
        float sum = p0 + p1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        sv[lane] = p0;
        sv[lane + 32] = p1;
        __syncwarp();
        if (lane == 0) {
          l_s[sr] = l_s[sr] * alpha + sum;
          m_s[sr] = m_new;
          a_s[sr] = alpha;
        }
      }
      __syncthreads();
      // O_lat += P . cKV
#pragma unroll
      for (int u = 0; u < kCols; ++u) {
        const int c = tid + u * kSimtThreads;
        if (c < p.r) {
          const int s = c / rs;
#pragma unroll
          for (int i = 0; i < kSimtRowGroup; ++i) {
            const float* pv = s_s + (s * kSimtRowGroup + i) * P;
            float a = acc[u][i] * a_s[s * kSimtRowGroup + i];
            for (int j = 0; j < P; ++j) a = fmaf(pv[j], tile[j * ld + c], a);
            acc[u][i] = a;
          }
        }
      }
      __syncthreads();
    }
    // segment partials: O_lat / l and log2(sum) + max
#pragma unroll
    for (int u = 0; u < kCols; ++u) {
      const int c = tid + u * kSimtThreads;
      if (c < p.r) {
        const int s = c / rs;
#pragma unroll
        for (int i = 0; i < kSimtRowGroup; ++i) {
          const int row = row0 + i;
          if (row < p.rows) {
            const float l = l_s[s * kSimtRowGroup + i];
            p.o_part[(slot * p.rows + row) * p.r + c] = l > 0.f ? acc[u][i] / l : 0.f;
          }
        }
      }
    }
    if (tid < S * kSimtRowGroup) {
      const int s = tid / kSimtRowGroup, i = tid % kSimtRowGroup, row = row0 + i;
      if (row < p.rows) {
        const float l = l_s[tid];
        p.lse_part[(slot * p.rows + row) * S + s] = l > 0.f ? m_s[tid] + log2f(l) : kEmptyLse;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// combine + up-projection: grid (H, ceil(B*Lq / 8)), 256 threads.
// out[b,t,h,:] = (sum over segments of 2^(lse - LSE) O_seg) . W_UV[h]
// (per TPLA shard: its own LSE over its own columns; the shards' columns are
// then contracted together with W_UV[h], which sums the shard outputs).
// ---------------------------------------------------------------------------
template <typename T, int S>
__global__ void __launch_bounds__(kSimtThreads) combine_simt_kernel(RunParams p) {
  if (!*p.lengths_ok) return;
  extern __shared__ float smem[];
  float* o_lat = smem;                              // [8][r]
  float* red = o_lat + kCombineRows * p.r;          // [8][128]
  __shared__ float lse_tot[kCombineRows][2];
  __shared__ int64_t seg_lo[kCombineRows], seg_hi[kCombineRows];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x, bt0 = blockIdx.y * kCombineRows;
  const int nbt = p.B * p.Lq;
  const int64_t Gv = virtual_pages(p.cum[p.B], p.B);
  const int rs = p.r / S;
  if (warp < kCombineRows) {
    const int i = warp, bt = bt0 + i;
    if (bt < nbt) {
      const int b = bt / p.Lq, t = bt % p.Lq, row = t * p.H + h;
      const int64_t w_lo = page_owner(p.cum[b], b, Gv, p.W);
      const int64_t w_hi = page_owner(p.cum[b + 1] - 1, b, Gv, p.W);
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
        if (lane == 0) lse_tot[i][s] = mx + log2f(sum);
      }
      if (lane == 0) {
        seg_lo[i] = w_lo;
        seg_hi[i] = w_hi;
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < kCombineRows * p.r; idx += blockDim.x) {
    const int i = idx / p.r, c = idx % p.r, bt = bt0 + i;
    float a = 0.f;
    if (bt < nbt) {
      const int b = bt / p.Lq, t = bt % p.Lq, row = t * p.H + h, s = c / rs;
      const float tot = lse_tot[i][s];
      for (int64_t w = seg_lo[i]; w <= seg_hi[i]; ++w) {
        const int64_t slot = w + b;
        const float wt = exp2f(p.lse_part[(slot * p.rows + row) * S + s] - tot);
        a = fmaf(wt, p.o_part[(slot * p.rows + row) * p.r + c], a);
      }
    }
    o_lat[idx] = a;
  }
  __syncthreads();
  const T* w_uv = static_cast<const T*>(p.w_uv) + (int64_t)h * p.r * p.dv;
  const int e = tid & 127, half = tid >> 7;
  float acc[kCombineRows];
#pragma unroll
  for (int i = 0; i < kCombineRows; ++i) acc[i] = 0.f;
  if (e < p.dv) {
    const int c0 = half * (p.r / 2), c1 = half ? p.r : p.r / 2;
    for (int c = c0; c < c1; ++c) {
      const float wv = to_float(w_uv[(int64_t)c * p.dv + e]);
#pragma unroll
      for (int i = 0; i < kCombineRows; ++i) acc[i] = fmaf(o_lat[i * p.r + c], wv, acc[i]);
    }
  }
  if (half == 1) {
#pragma unroll
    for (int i = 0; i < kCombineRows; ++i) red[i * 128 + e] = acc[i];
  }
  __syncthreads();
  if (half == 0 && e < p.dv) {
    T* out = static_cast<T*>(p.out);
#pragma unroll
    for (int i = 0; i < kCombineRows; ++i) {
      const int bt = bt0 + i;
      if (bt < nbt) out[((int64_t)bt * p.H + h) * p.dv + e] = from_float<T>(acc[i] + red[i * 128 + e]);
    }
  }
}

inline size_t simt_combine_smem_bytes(int r) {
  return sizeof(float) * ((size_t)kCombineRows * r + kCombineRows * 128);
}

}  // namespace mla
