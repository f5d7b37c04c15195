// Host side of the C ABI declared in include/mla_decode.h: dims validation,
// the plan (worker count, workspace size, split partition export) and the
// launch sequence of one decode step.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "common.cuh"
#include "simt_kernels.cuh"
#include "tc_decode.cuh"
#include "tc_decode_f8.cuh"
#include "tc_head_gemm.cuh"
#include "tc_prefill.cuh"

using namespace mla;

struct mla_plan {
  mla_dims_t dims;
  int32_t B;
  int32_t W;
  int32_t kernel;
  int32_t num_sms;
  int64_t G;
  std::vector<int32_t> lens;
  WorkspaceLayout layout;
};

namespace {

// The tensor-core kernels: r = 512 (bf16 with one or two latent shards, or the
// FP8 cache), or r = 256 with one shard (bf16; a TPLA shard per GPU).
bool tc_supported(const mla_dims_t& d) {
  if (!(kTcDecodeAvailable && d.rope_dim == 64 && d.page_size == 64 && d.num_heads * d.q_len <= 128 &&
        d.nope_dim == 128 && d.v_dim == 128))
    return false;
  if (d.latent_rank == 512)
    return d.dtype == MLA_BF16 ? (d.latent_shards == 1 || d.latent_shards == 2)
                               : (d.dtype == MLA_FP8_CACHE && d.latent_shards == 1);
  return d.latent_rank == 256 && d.dtype == MLA_BF16 && d.latent_shards == 1;
}

mla_status_t check_dims(const mla_dims_t& d) {
  if (d.num_heads < 1 || d.latent_rank < 1 || d.rope_dim < 0 || d.nope_dim < 1 || d.v_dim < 1 ||
      d.q_len < 1 || d.page_size < 1 || d.latent_shards < 1 || !std::isfinite(d.softmax_scale) ||
      d.softmax_scale <= 0.f)
    return MLA_ERR_INVALID_ARG;
  if (d.dtype != MLA_BF16 && d.dtype != MLA_FP32 && d.dtype != MLA_FP8_CACHE) return MLA_ERR_INVALID_ARG;
  if (d.page_size != 64) return MLA_ERR_UNSUPPORTED;
  if (d.latent_shards > 2 || d.latent_rank % d.latent_shards != 0) return MLA_ERR_UNSUPPORTED;
  if (d.latent_rank > 512 || d.latent_rank + d.rope_dim > 576 || d.nope_dim > kMaxNope ||
      d.v_dim > 128 || d.num_heads * d.q_len > 4096)
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

int device_sm_count(int32_t* out) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  *out = n;
  return 1;
}

}  // namespace

extern "C" {

int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported dimensions";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MLA_ERR_CUDA: return "CUDA runtime error";
    case MLA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MLA_ERR_BOUNDS: return "block id or sequence length out of range";
    case MLA_ERR_NO_DEVICE: return "no usable CUDA device";
  }
  return "unknown status";
}

mla_status_t mla_decode_plan_ex(const mla_dims_t* dims, int32_t batch, const int32_t* seq_lens_host,
                                const mla_plan_options_t* opts, mla_plan_t* plan_out,
                                size_t* workspace_bytes) {
  if (!dims || !seq_lens_host || !plan_out || batch < 1) return MLA_ERR_INVALID_ARG;
  *plan_out = nullptr;
  mla_status_t st = check_dims(*dims);
  if (st != MLA_OK) return st;
  mla_plan_options_t o{};
  if (opts) o = *opts;
  int32_t sms = o.num_sms;
  if (sms < 0) return MLA_ERR_INVALID_ARG;
  if (sms == 0 && !device_sm_count(&sms)) return MLA_ERR_NO_DEVICE;
  int64_t G = 0;
  for (int b = 0; b < batch; ++b) {
    const int32_t L = seq_lens_host[b];
    if (L < dims->q_len) return MLA_ERR_INVALID_ARG;
    G += ceil_div64(L, dims->page_size);
  }
  int32_t kernel = o.kernel;
  if (kernel == MLA_KERNEL_AUTO) kernel = tc_supported(*dims) ? MLA_KERNEL_TCGEN05 : MLA_KERNEL_SIMT;
  // the FP8 cache has one kernel: tcgen05, one latent shard
  if (dims->dtype == MLA_FP8_CACHE && (kernel != MLA_KERNEL_TCGEN05 || !tc_supported(*dims)))
    return MLA_ERR_UNSUPPORTED;
  if (kernel == MLA_KERNEL_TCGEN05 && !tc_supported(*dims)) return MLA_ERR_UNSUPPORTED;
  if (kernel != MLA_KERNEL_SIMT && kernel != MLA_KERNEL_TCGEN05) return MLA_ERR_INVALID_ARG;
  int64_t W;
  if (o.num_workers > 0) {
    W = o.num_workers;
  } else if (kernel == MLA_KERNEL_TCGEN05) {
    // one CTA pair per worker (a cluster of two SMs); a pair step is one page
    W = std::max<int64_t>(1, std::min<int64_t>(sms / 2, G));
  } else {
    W = std::max<int64_t>(1, std::min<int64_t>(sms, G));
  }
  W = std::min<int64_t>(W, G);
  mla_plan* p = new (std::nothrow) mla_plan();
  if (!p) return MLA_ERR_INVALID_ARG;
  p->dims = *dims;
  p->B = batch;
  p->W = (int32_t)W;
  p->kernel = kernel;
  p->num_sms = sms;
  p->G = G;
  p->lens.assign(seq_lens_host, seq_lens_host + batch);
  const int elt = dims->dtype == MLA_FP32 ? 4 : 2;  // FP8 cache: query rows of 2 (r + d_rope) bytes
  p->layout = workspace_layout(batch, dims->q_len, dims->num_heads, dims->latent_rank,
                               dims->rope_dim, dims->latent_shards, elt, W + batch - 1);
  *plan_out = p;
  if (workspace_bytes) *workspace_bytes = p->layout.total;
  return MLA_OK;
}

mla_status_t mla_decode_plan(const mla_dims_t* dims, int32_t batch, const int32_t* seq_lens_host,
                             int32_t num_sms, mla_plan_t* plan_out, size_t* workspace_bytes) {
  mla_plan_options_t o{};
  o.num_sms = num_sms;
  return mla_decode_plan_ex(dims, batch, seq_lens_host, &o, plan_out, workspace_bytes);
}

void mla_plan_destroy(mla_plan_t plan) { delete plan; }

}  // extern "C"

bool mla::plan_is_fp8(const mla_plan* plan) { return plan && plan->dims.dtype == MLA_FP8_CACHE; }

extern "C" {

mla_status_t mla_plan_get_info(mla_plan_t plan, mla_plan_info_t* info) {
  if (!plan || !info) return MLA_ERR_INVALID_ARG;
  info->batch = plan->B;
  info->rows = plan->dims.num_heads * plan->dims.q_len;
  info->kernel = plan->kernel;
  info->num_workers = plan->W;
  info->num_split_slots = plan->W + plan->B - 1;
  // absorb, decode, combine (split merge fused with the up-projection)
  info->launches_per_run = 3;
  info->total_pages = plan->G;
  info->workspace_bytes = plan->layout.total;
  return MLA_OK;
}

mla_status_t mla_plan_segments(mla_plan_t plan, int32_t* out, int64_t capacity, int64_t* count) {
  if (!plan || !count || capacity < 0 || (capacity > 0 && !out)) return MLA_ERR_INVALID_ARG;
  const int64_t P = plan->dims.page_size, W = plan->W;
  std::vector<int64_t> cum(plan->B + 1, 0);
  for (int b = 0; b < plan->B; ++b) cum[b + 1] = cum[b] + ceil_div64(plan->lens[b], P);
  int64_t n = 0;
  for (int64_t w = 0; w < W; ++w) {
    const int64_t g0 = worker_page_start(w, cum.data(), plan->B, W),
                  g1 = worker_page_start(w + 1, cum.data(), plan->B, W);
    if (g0 >= g1) continue;
    int b = 0;
    while (cum[b + 1] <= g0) ++b;
    for (; b < plan->B && cum[b] < g1; ++b) {
      if (n < capacity) {
        int32_t* e = out + 5 * n;
        e[0] = (int32_t)w;
        e[1] = b;
        e[2] = (int32_t)(std::max(cum[b], g0) - cum[b]);
        e[3] = (int32_t)(std::min(cum[b + 1], g1) - cum[b]);
        e[4] = (int32_t)(w + b);
      }
      ++n;
    }
  }
  *count = n;
  return MLA_OK;
}

mla_status_t mla_decode_run(mla_plan_t plan, const void* q_nope, const void* q_rope,
                            const void* kv_cache, int64_t num_blocks, const int32_t* block_table,
                            int32_t block_table_stride, const int32_t* seq_lens_dev,
                            const void* w_uk, const void* w_uv, void* out, void* workspace,
                            size_t workspace_bytes, void* stream_) {
  return mla_decode_run_ex(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                           block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace,
                           workspace_bytes, stream_, nullptr);
}

}  // extern "C"

namespace {

// Device-wait settings of one run: the normal limit, or a self-test of the
// timeout path (short limit, one arrival withheld in the decode kernel).
struct WaitKnobs {
  uint64_t limit_ns = ptx::kWaitLimitNs;
  int32_t withhold_s_free = 0;
  bool skip = false;        // threshold-skipping decode
  float skip_log2 = 0.f;
};

mla_status_t run_impl(mla_plan_t plan, const void* q_nope, const void* q_rope, const void* kv_cache,
                      const void* kv_rope, const float* kv_scale, int64_t num_blocks,
                      const int32_t* block_table, int32_t block_table_stride, const int32_t* seq_lens_dev,
                      const void* w_uk, const void* w_uv, void* out, void* workspace, size_t workspace_bytes,
                      void* stream_, const mla_run_options_t* opts, WaitKnobs knobs = WaitKnobs{}) {
  if (!plan || !q_nope || !q_rope || !kv_cache || !block_table || !seq_lens_dev || !w_uk ||
      !w_uv || !out || !workspace || num_blocks < 1 || block_table_stride < 1)
    return MLA_ERR_INVALID_ARG;
  if (plan->dims.rope_dim > 0 && !q_rope) return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < plan->layout.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const mla_dims_t& d = plan->dims;
  char* ws = static_cast<char*>(workspace);
  RunParams p{};
  p.q_nope = q_nope;
  p.q_rope = q_rope;
  p.kv = kv_cache;
  p.kv_rope = kv_rope;
  p.kv_scale = kv_scale;
  p.fp8 = plan->dims.dtype == MLA_FP8_CACHE ? 1 : 0;
  p.block_table = block_table;
  p.seq_lens = seq_lens_dev;
  p.w_uk = w_uk;
  p.w_uv = w_uv;
  p.out = out;
  p.status = reinterpret_cast<int32_t*>(ws);
  p.lengths_ok = reinterpret_cast<int32_t*>(ws + 4);
  p.cum = reinterpret_cast<int64_t*>(ws + plan->layout.cum);
  p.seg_done = reinterpret_cast<int32_t*>(ws + plan->layout.done);
  p.q = ws + plan->layout.q;
  p.o_part = reinterpret_cast<float*>(ws + plan->layout.o_part);
  p.lse_part = reinterpret_cast<float*>(ws + plan->layout.lse_part);
  p.num_blocks = num_blocks;
  p.bt_stride = block_table_stride;
  p.B = plan->B;
  p.Lq = d.q_len;
  p.H = d.num_heads;
  p.r = d.latent_rank;
  p.dr = d.rope_dim;
  p.dn = d.nope_dim;
  p.dv = d.v_dim;
  p.P = d.page_size;
  p.S = d.latent_shards;
  p.rows = d.num_heads * d.q_len;
  p.W = plan->W;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.wait_limit_ns = knobs.limit_ns;
  p.withhold_s_free = knobs.withhold_s_free;
  p.skip_log2 = knobs.skip_log2;
  p.skip_stats = reinterpret_cast<int32_t*>(ws + 8);
  if (knobs.skip && cudaMemsetAsync(ws + 8, 0, 8, stream) != cudaSuccess) return MLA_ERR_CUDA;

  const bool bf16 = d.dtype == MLA_BF16;
  const int nbt = p.B * p.Lq;
  const bool tc = plan->kernel == MLA_KERNEL_TCGEN05;
  if (tc) {
    if (launch_absorb_tc(p, stream) != cudaSuccess) return MLA_ERR_CUDA;
  } else {
    const dim3 ga(p.H, (p.r + 127) / 128, (nbt + kAbsorbRows - 1) / kAbsorbRows);
    if (bf16) absorb_simt_kernel<__nv_bfloat16><<<ga, 128, 0, stream>>>(p);
    else absorb_simt_kernel<float><<<ga, 128, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  }

  cudaEvent_t ev_start = opts ? static_cast<cudaEvent_t>(opts->decode_start_event) : nullptr;
  cudaEvent_t ev_stop = opts ? static_cast<cudaEvent_t>(opts->decode_stop_event) : nullptr;
  if (ev_start && cudaEventRecord(ev_start, stream) != cudaSuccess) return MLA_ERR_CUDA;
  // The decode keeps its programmatic launch when bracketed by the caller's
  // events (its setup overlaps the absorb kernel, as in an untimed step): the
  // events then time its critical-path share, within ~2% of its kernel-only
  // duration in an ncu launch list, while a plain-order launch adds the launch
  // gap and the setup (10-40 us, run to run).
  const bool pdl = true;
  if (p.fp8) {
    if (launch_tc_decode_f8(p, stream, pdl) != cudaSuccess) return MLA_ERR_CUDA;
  } else if (plan->kernel == MLA_KERNEL_TCGEN05) {
    if (launch_tc_decode(p, stream, pdl, knobs.skip) != cudaSuccess) return MLA_ERR_CUDA;
  } else {
    const size_t smem = simt_decode_smem_bytes(p.r + p.dr, p.S, p.P);
    const dim3 gd(p.W, (p.rows + kSimtRowGroup - 1) / kSimtRowGroup);
    cudaError_t e;
#define MLA_LAUNCH_DECODE(T, S)                                                              \
  e = ensure_smem_limit(reinterpret_cast<const void*>(decode_simt_kernel<T, S>), (int)smem);  \
  if (e == cudaSuccess) decode_simt_kernel<T, S><<<gd, kSimtThreads, smem, stream>>>(p);
    if (bf16 && p.S == 1) { MLA_LAUNCH_DECODE(__nv_bfloat16, 1) }
    else if (bf16) { MLA_LAUNCH_DECODE(__nv_bfloat16, 2) }
    else if (p.S == 1) { MLA_LAUNCH_DECODE(float, 1) }
    else { MLA_LAUNCH_DECODE(float, 2) }
#undef MLA_LAUNCH_DECODE
    if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  }
  if (ev_stop && cudaEventRecord(ev_stop, stream) != cudaSuccess) return MLA_ERR_CUDA;

  if (tc) {
    if (launch_combine_tc(p, stream) != cudaSuccess) return MLA_ERR_CUDA;
  } else {
    const size_t csmem = simt_combine_smem_bytes(p.r);
    const dim3 gc(p.H, (nbt + kCombineRows - 1) / kCombineRows);
    if (bf16 && p.S == 1) combine_simt_kernel<__nv_bfloat16, 1><<<gc, kSimtThreads, csmem, stream>>>(p);
    else if (bf16) combine_simt_kernel<__nv_bfloat16, 2><<<gc, kSimtThreads, csmem, stream>>>(p);
    else if (p.S == 1) combine_simt_kernel<float, 1><<<gc, kSimtThreads, csmem, stream>>>(p);
    else combine_simt_kernel<float, 2><<<gc, kSimtThreads, csmem, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status_t mla_decode_run_ex(mla_plan_t plan, const void* q_nope, const void* q_rope,
                               const void* kv_cache, int64_t num_blocks,
                               const int32_t* block_table, int32_t block_table_stride,
                               const int32_t* seq_lens_dev, const void* w_uk, const void* w_uv,
                               void* out, void* workspace, size_t workspace_bytes, void* stream_,
                               const mla_run_options_t* opts) {
  if (plan && plan->dims.dtype == MLA_FP8_CACHE) return MLA_ERR_INVALID_ARG;  // mla_decode_run_fp8
  return run_impl(plan, q_nope, q_rope, kv_cache, nullptr, nullptr, num_blocks, block_table,
                  block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace, workspace_bytes, stream_, opts);
}

mla_status_t mla_decode_run_fp8(mla_plan_t plan, const void* q_nope, const void* q_rope,
                                const void* kv_codes, const void* kv_rope, const float* kv_scale,
                                int64_t num_blocks, const int32_t* block_table,
                                int32_t block_table_stride, const int32_t* seq_lens_dev,
                                const void* w_uk, const void* w_uv, void* out, void* workspace,
                                size_t workspace_bytes, void* stream_, const mla_run_options_t* opts) {
  if (!plan || plan->dims.dtype != MLA_FP8_CACHE || !kv_rope || !kv_scale) return MLA_ERR_INVALID_ARG;
  return run_impl(plan, q_nope, q_rope, kv_codes, kv_rope, kv_scale, num_blocks, block_table,
                  block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace, workspace_bytes, stream_, opts);
}

mla_status_t mla_decode_run_blasst(mla_plan_t plan, const void* q_nope, const void* q_rope,
                                   const void* kv_cache, int64_t num_blocks, const int32_t* block_table,
                                   int32_t block_table_stride, const int32_t* seq_lens_dev, const void* w_uk,
                                   const void* w_uv, void* out, void* workspace, size_t workspace_bytes,
                                   float skip_log2, void* stream_, const mla_run_options_t* opts) {
  if (!plan || plan->dims.dtype != MLA_BF16 || plan->kernel != MLA_KERNEL_TCGEN05 || plan->dims.latent_rank != 512 ||
      plan->dims.latent_shards != 1)
    return MLA_ERR_UNSUPPORTED;
  if (!(skip_log2 <= 0.f)) return MLA_ERR_INVALID_ARG;  // NaN and positive thresholds refused
  WaitKnobs k;
  k.skip = true;
  k.skip_log2 = skip_log2;
  return run_impl(plan, q_nope, q_rope, kv_cache, nullptr, nullptr, num_blocks, block_table, block_table_stride,
                  seq_lens_dev, w_uk, w_uv, out, workspace, workspace_bytes, stream_, opts, k);
}

mla_status_t mla_decode_selftest_timeout(mla_plan_t plan, const void* q_nope, const void* q_rope,
                                         const void* kv_cache, int64_t num_blocks,
                                         const int32_t* block_table, int32_t block_table_stride,
                                         const int32_t* seq_lens_dev, const void* w_uk, const void* w_uv,
                                         void* out, void* workspace, size_t workspace_bytes,
                                         uint64_t wait_limit_ns, void* stream_) {
  // the bf16 tensor-core decode kernel is the one whose waits take the limit
  if (!plan || plan->dims.dtype != MLA_BF16 || plan->kernel != MLA_KERNEL_TCGEN05) return MLA_ERR_UNSUPPORTED;
  if (wait_limit_ns < 1000 || wait_limit_ns > ptx::kWaitLimitNs) return MLA_ERR_INVALID_ARG;
  WaitKnobs k;
  k.limit_ns = wait_limit_ns;
  k.withhold_s_free = 1;
  return run_impl(plan, q_nope, q_rope, kv_cache, nullptr, nullptr, num_blocks, block_table,
                  block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace, workspace_bytes, stream_,
                  nullptr, k);
}

}  // extern "C"

struct mla_prefill_plan {
  mla_dims_t dims;
  int32_t B;
  int64_t T;
  int32_t max_len;
  size_t k_off, v_off, total;
};

extern "C" {

mla_status_t mla_prefill_plan(const mla_dims_t* dims, int32_t batch, const int32_t* seq_lens_host,
                              mla_prefill_plan_t* plan_out, size_t* workspace_bytes) {
  if (!dims || !seq_lens_host || !plan_out || batch < 1) return MLA_ERR_INVALID_ARG;
  *plan_out = nullptr;
  const mla_dims_t& d = *dims;
  if (d.num_heads < 1 || !std::isfinite(d.softmax_scale) || d.softmax_scale <= 0.f) return MLA_ERR_INVALID_ARG;
  if (d.dtype != MLA_BF16 || d.latent_rank != 512 || d.rope_dim != 64 || d.nope_dim != 128 || d.v_dim != 128 ||
      d.latent_shards != 1)
    return MLA_ERR_UNSUPPORTED;
  int64_t T = 0;
  int32_t mx = 0;
  for (int b = 0; b < batch; ++b) {
    if (seq_lens_host[b] < 1) return MLA_ERR_INVALID_ARG;
    T += seq_lens_host[b];
    mx = std::max(mx, seq_lens_host[b]);
  }
  // row coordinates of the K_nope / V workspace ([H * T, 128]) are 32-bit
  if ((int64_t)d.num_heads * (T + pf::kTile) >= (int64_t(1) << 31)) return MLA_ERR_UNSUPPORTED;
  struct mla_prefill_plan* p = new (std::nothrow) struct mla_prefill_plan();
  if (!p) return MLA_ERR_INVALID_ARG;
  p->dims = d;
  p->B = batch;
  p->T = T;
  p->max_len = mx;
  p->k_off = 1024;
  p->v_off = align_up(p->k_off + (size_t)T * d.num_heads * d.nope_dim * 2, 1024);
  p->total = align_up(p->v_off + (size_t)T * d.num_heads * d.v_dim * 2, 1024);
  *plan_out = p;
  if (workspace_bytes) *workspace_bytes = p->total;
  return MLA_OK;
}

mla_status_t mla_prefill_run(mla_prefill_plan_t plan, const void* q_nope, const void* q_rope,
                             const void* kv_rows, const int32_t* cu_seqlens_dev, const void* w_uk,
                             const void* w_uv, void* out, void* workspace, size_t workspace_bytes,
                             void* stream_) {
  return mla_prefill_run_ex(plan, q_nope, q_rope, kv_rows, cu_seqlens_dev, w_uk, w_uv, out, workspace,
                            workspace_bytes, stream_, nullptr);
}

mla_status_t mla_prefill_run_ex(mla_prefill_plan_t plan, const void* q_nope, const void* q_rope,
                                const void* kv_rows, const int32_t* cu_seqlens_dev, const void* w_uk,
                                const void* w_uv, void* out, void* workspace, size_t workspace_bytes,
                                void* stream_, const mla_run_options_t* opts) {
  if (!plan || !q_nope || !q_rope || !kv_rows || !cu_seqlens_dev || !w_uk || !w_uv || !out || !workspace)
    return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < plan->total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  const mla_dims_t& d = plan->dims;
  char* ws = static_cast<char*>(workspace);
  PrefillParams p{};
  p.q_nope = q_nope;
  p.q_rope = q_rope;
  p.kv = kv_rows;
  p.cu_seqlens = cu_seqlens_dev;
  p.w_uk = w_uk;
  p.w_uv = w_uv;
  p.out = out;
  p.status = reinterpret_cast<int32_t*>(ws);
  p.k_nope = ws + plan->k_off;
  p.v = ws + plan->v_off;
  p.T = plan->T;
  p.B = plan->B;
  p.H = d.num_heads;
  p.r = d.latent_rank;
  p.dr = d.rope_dim;
  p.dn = d.nope_dim;
  p.dv = d.v_dim;
  p.num_q_tiles = (plan->max_len + pf::kTile - 1) / pf::kTile;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.wait_limit_ns = ptx::kWaitLimitNs;
  cudaEvent_t ev0 = opts ? static_cast<cudaEvent_t>(opts->decode_start_event) : nullptr;
  cudaEvent_t ev1 = opts ? static_cast<cudaEvent_t>(opts->decode_stop_event) : nullptr;
  if (launch_prefill(p, static_cast<cudaStream_t>(stream_), ev0, ev1) != cudaSuccess) {
    (void)cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

void mla_prefill_plan_destroy(mla_prefill_plan_t plan) { delete plan; }

mla_status_t mla_workspace_init(void* workspace, size_t workspace_bytes, void* stream_) {
  if (!workspace || workspace_bytes < 1024) return MLA_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, 1024, static_cast<cudaStream_t>(stream_)) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status_t mla_decode_read_status(const void* workspace, void* stream_, int32_t* device_status) {
  if (!workspace || !device_status) return MLA_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  int32_t v = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemset(const_cast<void*>(workspace), 0, sizeof(v)) != cudaSuccess) return MLA_ERR_CUDA;
  *device_status = v;
  return MLA_OK;
}

#ifdef MLA_TRACE
// Debug builds only: copies the event trace (see tc_decode.cuh) to host memory.
int mla_debug_trace_read(unsigned long long* host, size_t n) {
  const size_t cap = sizeof(tc::g_trace) / sizeof(unsigned long long);
  if (n > cap) n = cap;
  return cudaMemcpyFromSymbol(host, tc::g_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 1;
}
int mla_debug_trace_ns_read(unsigned long long* host, size_t n) {
  const size_t cap = sizeof(tc::g_trace_ns) / sizeof(unsigned long long);
  if (n > cap) n = cap;
  return cudaMemcpyFromSymbol(host, tc::g_trace_ns, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 1;
}
int mla_debug_trace_cta_read(unsigned long long* host, size_t n) {
  const size_t cap = sizeof(tc::g_trace_cta) / sizeof(unsigned long long);
  if (n > cap) n = cap;
  return cudaMemcpyFromSymbol(host, tc::g_trace_cta, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 1;
}
int mla_debug_trace_hg_read(unsigned long long* host, size_t n) {
  const size_t cap = sizeof(hg::g_hg_trace) / sizeof(unsigned long long);
  if (n > cap) n = cap;
  return cudaMemcpyFromSymbol(host, hg::g_hg_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 1;
}
int mla_debug_trace_pf_read(unsigned long long* host, size_t n) {
  const size_t cap = sizeof(pf::g_pf_trace) / sizeof(unsigned long long);
  if (n > cap) n = cap;
  return cudaMemcpyFromSymbol(host, pf::g_pf_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 1;
}
int mla_debug_trace_chunks_read(unsigned long long* host, size_t n) {
  const size_t cap = sizeof(tc::g_trace_chunk) / sizeof(unsigned long long);
  if (n > cap) n = cap;
  return cudaMemcpyFromSymbol(host, tc::g_trace_chunk, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 1;
}
#endif

}  // extern "C"
