// Shared definitions of the decode library: the split partition (evaluated
// identically by the host plan and by every kernel), the workspace layout and
// the kernel parameter block.
#pragma once

#include <cstdint>
#include <mutex>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/mla_decode.h"

#define MLA_HD __host__ __device__ __forceinline__

namespace mla {

// ---------------------------------------------------------------------------
// Split partition.
//
// The pages of all sequences are concatenated (sequence b owns global pages
// [cum[b], cum[b+1]), cum[b] = sum_{i<b} ceil(L_i / P)) and cut into W
// contiguous page ranges. A worker's range meets one or more sequences; each
// (worker, sequence) intersection is one split segment whose partial result
// goes to slot w + b. Along the concatenated page order both w and b are
// non-decreasing and at least one of them grows from one segment to the next,
// so w + b is strictly increasing: slots are unique, and W + B - 1 slots always
// suffice whatever the lengths are.
//
// The cut balances cost, not pages: a worker whose range crosses a sequence
// boundary writes one more segment partial and reloads the query, which costs
// about as much as kSegmentCostPages pages. So every boundary takes that many
// places on a "virtual" page line (page x of sequence b sits at x + c b, and
// the line is G' = G + c (B - 1) long), the line is cut evenly, at
// floor(w G' / W), and each cut moves to the first real page at or after it.
// ---------------------------------------------------------------------------
constexpr int64_t kSegmentCostPages = 4;

MLA_HD int64_t virtual_pages(int64_t G, int64_t B) { return G + kSegmentCostPages * (B - 1); }

// start(w): the first global page of worker w (start(W) = G). cum has B + 1
// entries, strictly increasing (every sequence has at least one page).
MLA_HD int64_t worker_page_start(int64_t w, const int64_t* cum, int64_t B, int64_t W) {
  const int64_t v = (w * virtual_pages(cum[B], B)) / W;
  int64_t lo = 0, hi = B - 1;  // the last sequence b with cum[b] + c b <= v
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (cum[mid] + kSegmentCostPages * mid <= v) lo = mid; else hi = mid - 1;
  }
  const int64_t x = v - kSegmentCostPages * lo;
  return x < cum[lo + 1] ? x : cum[lo + 1];  // a cut inside a boundary moves to the next sequence
}

// The worker whose range holds page x of sequence b: the largest w with
// start(w) <= x, i.e. with floor(w G' / W) <= x + c b, clamped to W - 1.
MLA_HD int64_t page_owner(int64_t x, int64_t b, int64_t Gv, int64_t W) {
  const int64_t xv = x + kSegmentCostPages * b;
  const int64_t w = ((xv + 1) * W + Gv - 1) / Gv - 1;
  return w < W - 1 ? w : W - 1;
}

MLA_HD int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------
// Workspace layout (byte offsets from the workspace base; all 1 KiB aligned).
//   [0]            int32 status word (first device-side error, sticky)
//   [4]            int32 lengths_ok (written by the first kernel of a run)
//   cum            int64 [B + 1] page prefix sums of this run's seq_lens
//   done           int32 [B] segment halves of sequence b written this run
//                  (each CTA of a pair adds 1 per segment once its rows are out)
//   q              [B * Lq * H, r + d_rope] absorbed query rows (dims.dtype)
//   o_part         [slots, rows, r]  per-segment O_lat / l: fp32 on the SIMT
//                  path, fp16 on the tensor-core paths (room for fp32 either way)
//   lse_part       fp32 [slots, rows, S]  per-segment log2-sum-exp per shard
// ---------------------------------------------------------------------------
struct WorkspaceLayout {
  size_t cum, done, q, o_part, lse_part, total;
};

MLA_HD size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WorkspaceLayout workspace_layout(int64_t B, int64_t Lq, int64_t H, int64_t r,
                                        int64_t dr, int64_t shards, int64_t elt_bytes,
                                        int64_t slots) {
  WorkspaceLayout L{};
  size_t off = 1024;
  L.cum = off;
  off = align_up(off + sizeof(int64_t) * (B + 1), 1024);
  L.done = off;
  off = align_up(off + sizeof(int32_t) * B, 1024);
  L.q = off;
  off = align_up(off + (size_t)(B * Lq * H) * (r + dr) * elt_bytes, 1024);
  L.o_part = off;
  off = align_up(off + (size_t)slots * (Lq * H) * r * sizeof(float), 1024);
  L.lse_part = off;
  off = align_up(off + (size_t)slots * (Lq * H) * shards * sizeof(float), 1024);
  L.total = off;
  return L;
}

// Finite stand-in for log(0): a segment row that saw no key.
constexpr float kEmptyLse = -1.0e30f;

// ---------------------------------------------------------------------------
// Parameters shared by the kernels of one run.
// ---------------------------------------------------------------------------
struct RunParams {
  // inputs
  const void* q_nope;
  const void* q_rope;
  const void* kv;          // pool (bf16 / fp32 rows, or the e4m3 codes of an FP8 cache)
  const void* kv_rope;     // FP8 cache: bf16 RoPE keys stored divided by the token scale
  const float* kv_scale;   // FP8 cache: fp32 scale per token [num_blocks, page_size]
  const int32_t* block_table;
  const int32_t* seq_lens;
  const void* w_uk;
  const void* w_uv;
  void* out;
  // workspace
  int32_t* status;
  int32_t* lengths_ok;
  int64_t* cum;
  int32_t* seg_done;       // [B] zeroed by the absorb kernel, counted up by the decode kernels
  void* q;                 // absorbed query rows
  float* o_part;           // fp32 (SIMT kernels) or fp16 (tensor-core kernels)
  float* lse_part;
  // sizes
  int64_t num_blocks;
  int32_t bt_stride;
  int32_t B, Lq, H, r, dr, dn, dv, P, S;
  int32_t rows;            // H * Lq
  int32_t W;               // workers
  int32_t fp8;             // 1: FP8 cache (the absorbed query is written as e4m3 + e5m2 bytes)
  float scale_log2;        // softmax_scale * log2(e)
  // bounded waits of the bf16 tensor-core decode kernel (2 s in a normal run)
  uint64_t wait_limit_ns;
  // self-test of the timeout path only: the decode kernel's softmax withholds
  // the release of its score buffers, so the QK issuer's wait runs out
  int32_t withhold_s_free;
  // threshold skipping (the skipping decode only): log2 threshold below the
  // running max, and the workspace counters (skipped groups, groups)
  float skip_log2;
  int32_t* skip_stats;
};

// True for a plan over the FP8 latent cache (host; defined with the ABI).
bool plan_is_fp8(const mla_plan* plan);

__device__ __forceinline__ void record_error(int32_t* status, int32_t code) {
  atomicCAS(status, 0, code);
}

// A CTA of a decode pair has written its rows of a segment's partials: every
// writing thread fenced its stores before the CTA barrier that precedes this
// call, so the release-ordered add publishes them at GPU scope.
__device__ __forceinline__ void publish_segment_half(int32_t* done) {
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" :: "l"(done) : "memory");
}

__device__ __forceinline__ int32_t load_acquire_gpu(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_float(float x);
template <> __device__ __forceinline__ float from_float<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device) and
// remembers it, so that repeated runs (and runs captured into a CUDA graph)
// make no further attribute calls.
inline cudaError_t ensure_smem_limit(const void* func, int bytes) {
  struct Entry { const void* func; int dev; int bytes; };
  static Entry table[256];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (table[i].func == func && table[i].dev == dev && table[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  // Every kernel of a run asks for the largest shared-memory carveout, so that
  // consecutive kernels find the SM already configured.
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && used < 256) table[used++] = Entry{func, dev, bytes};
  return e;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream runs and waits for it in
// grid_dependency_wait(). pdl = false launches it in plain stream order (a
// kernel bracketed by timing events: an event recorded between two kernels
// chained this way does not mark the second one's start).
template <typename... Params, typename... Args>
inline cudaError_t launch_dependent_opt(bool pdl, void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                        cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... Params, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args&&... args) {
  return launch_dependent_opt(true, kernel, grid, block, smem, stream, std::forward<Args>(args)...);
}

}  // namespace mla
