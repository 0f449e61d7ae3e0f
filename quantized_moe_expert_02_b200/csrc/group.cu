// Token-to-expert grouping: the (token, slot) pairs p = t*k + j sorted by
// expert, stable in p -- the per-expert token lists that the expert GEMMs
// of the "llama-halo-hybrid" post's MoE path consume.
#include "moe_internal.cuh"
#include "trace.h"

namespace moe {

constexpr int GROUP_CHUNK = 2048;   // pairs per block of the large path
constexpr int GROUP_SMALL_MAX = 16384;

// Whole grouping in one block (P = T*k <= GROUP_SMALL_MAX, E <= EMAX).
__global__ void __launch_bounds__(1024)
    group_small_kernel(const int32_t* __restrict__ idx, int P, int E,
                       int32_t* __restrict__ offsets,
                       int32_t* __restrict__ pair_ids,
                       int32_t* __restrict__ active,
                       int32_t* __restrict__ n_active, int32_t* err) {
  __shared__ int32_t cnt[EMAX + 1];
  __shared__ int32_t flag[EMAX + 1];
  __shared__ int32_t tmp[32];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) { cnt[e] = 0; flag[e] = 0; }
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int e = idx[p];
    if (e < 0 || e >= E) { set_err(err, MOE_ERR_DEVICE); continue; }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) flag[e] = cnt[e] > 0;
  __syncthreads();
  block_exclusive_scan(cnt, E + 1, tmp);   // cnt[E] (=0) becomes the total
  const int na = block_exclusive_scan(flag, E + 1, tmp);
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    offsets[e] = cnt[e];
    if (e < E && ((e + 1 <= E ? flag[e + 1] : na) != flag[e]))
      active[flag[e]] = e;
  }
  if (threadIdx.x == 0) *n_active = na;
  __syncthreads();
  // stable scatter by warp 0: 32 pairs per step, ranks by __match_any_sync
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int base = 0; base < P; base += 32) {
      const int p = base + lane;
      const int e = (p < P) ? idx[p] : -1;
      const bool ok = (p < P) && e >= 0 && e < E;
      const unsigned m = __match_any_sync(0xffffffffu, ok ? e : -1 - lane);
      const int rank = __popc(m & ((1u << lane) - 1u));
      if (ok) pair_ids[cnt[e] + rank] = p;
      __syncwarp();
      if (ok && rank == 0) cnt[e] += __popc(m);
      __syncwarp();
    }
  }
}

// Large path, step 1: per-chunk histograms hist[blk][E].
__global__ void __launch_bounds__(256)
    group_hist_kernel(const int32_t* __restrict__ idx, int P, int E,
                      int32_t* __restrict__ hist, int32_t* err) {
  __shared__ int32_t cnt[EMAX];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * GROUP_CHUNK;
  for (int i = threadIdx.x; i < GROUP_CHUNK; i += blockDim.x) {
    const int p = p0 + i;
    if (p >= P) break;
    const int e = idx[p];
    if (e < 0 || e >= E) { set_err(err, MOE_ERR_DEVICE); continue; }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    hist[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// Step 2 (one block): offsets, active list, per-chunk bases (in place).
__global__ void __launch_bounds__(1024)
    group_scan_kernel(int32_t* __restrict__ hist, int nblk, int E,
                      int32_t* __restrict__ offsets,
                      int32_t* __restrict__ active,
                      int32_t* __restrict__ n_active) {
  __shared__ int32_t tot[EMAX + 1];
  __shared__ int32_t flag[EMAX + 1];
  __shared__ int32_t tmp[32];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    int s = 0;
    if (e < E)
      for (int b = 0; b < nblk; ++b) s += hist[(int64_t)b * E + e];
    tot[e] = s;
    flag[e] = (e < E) && s > 0;
  }
  __syncthreads();
  block_exclusive_scan(tot, E + 1, tmp);
  const int na = block_exclusive_scan(flag, E + 1, tmp);
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    offsets[e] = tot[e];
    if (e < E && ((e + 1 <= E ? flag[e + 1] : na) != flag[e]))
      active[flag[e]] = e;
  }
  if (threadIdx.x == 0) *n_active = na;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = tot[e];
    for (int b = 0; b < nblk; ++b) {
      const int c = hist[(int64_t)b * E + e];
      hist[(int64_t)b * E + e] = run;
      run += c;
    }
  }
}

// Step 3: stable scatter, one warp per chunk.
__global__ void __launch_bounds__(32)
    group_scatter_kernel(const int32_t* __restrict__ idx, int P, int E,
                         const int32_t* __restrict__ base,
                         int32_t* __restrict__ pair_ids) {
  __shared__ int32_t cur[EMAX];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32)
    cur[e] = base[(int64_t)blockIdx.x * E + e];
  __syncwarp();
  const int p0 = blockIdx.x * GROUP_CHUNK;
  for (int b = 0; b < GROUP_CHUNK; b += 32) {
    const int p = p0 + b + lane;
    const int e = (p < P) ? idx[p] : -1;
    const bool ok = (p < P) && e >= 0 && e < E;
    const unsigned m = __match_any_sync(0xffffffffu, ok ? e : -1 - lane);
    const int rank = __popc(m & ((1u << lane) - 1u));
    if (ok) pair_ids[cur[e] + rank] = p;
    __syncwarp();
    if (ok && rank == 0) cur[e] += __popc(m);
    __syncwarp();
  }
}

size_t group_ws_bytes(int T, int k, int E) {
  const int64_t P = (int64_t)T * k;
  if (P <= GROUP_SMALL_MAX) return 256;
  const int64_t nblk = (P + GROUP_CHUNK - 1) / GROUP_CHUNK;
  return (size_t)(nblk * E * 4 + 256);
}

moe_status launch_group(const int32_t* idx, int T, int k, int E,
                        int32_t* offsets, int32_t* pair_ids, int32_t* active,
                        int32_t* n_active, int32_t* scratch, int32_t* err,
                        cudaStream_t s) {
  const int P = T * k;
  if (P <= GROUP_SMALL_MAX) {
    group_small_kernel<<<1, 1024, 0, s>>>(idx, P, E, offsets, pair_ids,
                                          active, n_active, err);
    return launch_status();
  }
  const int nblk = (P + GROUP_CHUNK - 1) / GROUP_CHUNK;
  group_hist_kernel<<<nblk, 256, 0, s>>>(idx, P, E, scratch, err);
  group_scan_kernel<<<1, 1024, 0, s>>>(scratch, nblk, E, offsets, active,
                                       n_active);
  group_scatter_kernel<<<nblk, 32, 0, s>>>(idx, P, E, scratch, pair_ids);
  return launch_status();
}

// The grouping restricted to a list of experts: the first block builds
// the sub-offsets (counts of the listed experts, exclusive scan) and the
// active list; every block then copies the listed experts' pair ranges.
// One launch of SUB_BLOCKS blocks; block 0's scan is redone by every block
// (E <= EMAX words in shared memory), so no inter-block sync is needed.
constexpr int SUB_BLOCKS = 64;

__global__ void __launch_bounds__(1024)
    group_subset_kernel(const int32_t* __restrict__ offsets,
                        const int32_t* __restrict__ pair_ids, int E,
                        const int32_t* __restrict__ experts, int n,
                        int32_t* __restrict__ sub_offsets,
                        int32_t* __restrict__ sub_pairs,
                        int32_t* __restrict__ sub_active,
                        int32_t* __restrict__ sub_n_active, int32_t* err) {
  __shared__ int32_t cnt[EMAX + 1];
  __shared__ int32_t mark[EMAX + 1];
  __shared__ int32_t tmp[32];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) { cnt[e] = 0; mark[e] = 0; }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = experts[i];
    if (e < 0 || e >= E) {
      if (blockIdx.x == 0) set_err(err, MOE_ERR_DEVICE);
      continue;
    }
    mark[e] = 1;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = mark[e] ? offsets[e + 1] - offsets[e] : 0;
    cnt[e] = c;
    mark[e] = c > 0;
  }
  __syncthreads();
  block_exclusive_scan(cnt, E + 1, tmp);
  const int na = block_exclusive_scan(mark, E + 1, tmp);
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
      sub_offsets[e] = cnt[e];
      if (e < E && mark[e + 1] != mark[e]) sub_active[mark[e]] = e;
    }
    if (threadIdx.x == 0) *sub_n_active = na;
  }
  // copy: expert e's pairs go to sub_pairs[cnt[e] ..), block b takes the
  // experts e with e % gridDim.x == b
  for (int e = blockIdx.x; e < E; e += gridDim.x) {
    const int c = cnt[e + 1] - cnt[e];
    if (c <= 0) continue;
    const int src = offsets[e];
    for (int i = threadIdx.x; i < c; i += blockDim.x)
      sub_pairs[cnt[e] + i] = pair_ids[src + i];
  }
}

}  // namespace moe

// ---------------------------------------------------------------------
// Grouping without a caller workspace.  For callers that cannot allocate
// device memory at the call site -- a plugin or custom operator that is
// handed only its input and output pointers by a host framework, code
// running where an allocation would synchronise the device or break a
// capture that the caller does not own, real-time loops that forbid
// allocation -- this variant keeps its scratch in a fixed array in the
// library's own device memory instead of a workspace.
#include <cuda.h>

#include <mutex>

namespace moe {
namespace {

constexpr int STATIC_GROUP_MAX_PAIRS = 262144;   // T*k
constexpr int STATIC_GROUP_MAX_E = 1024;
constexpr int STATIC_GROUP_MAX_CHUNKS =
    (STATIC_GROUP_MAX_PAIRS + GROUP_CHUNK - 1) / GROUP_CHUNK;
// word 0: error word; from word 64: per-chunk histograms [chunk][E].
// 512.25 KiB, held by every device that loads the library until exit.
constexpr size_t STATIC_GROUP_WORDS =
    64 + (size_t)STATIC_GROUP_MAX_CHUNKS * STATIC_GROUP_MAX_E;

static __device__ __align__(256) int32_t g_group_scratch[STATIC_GROUP_WORDS];

// Device address of the scratch array in the current context, looked up
// once per (device, context) with that device current (the array's name is
// only a host-side stand-in).  A symbol's address belongs to a context: a
// second context on the device gets its own lookup.
moe_status group_scratch_address(int32_t** out) {
  using CtxGetCurrent = CUresult (*)(CUcontext*);
  struct Entry { int dev; CUcontext ctx; int32_t* addr; };
  static Entry seen[64];
  static int n_seen = 0;
  static CtxGetCurrent ctx_get = nullptr;
  static std::mutex mu;
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(mu);
  if (!ctx_get) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault,
                                &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !f)
      return MOE_ERR_CUDA;
    ctx_get = reinterpret_cast<CtxGetCurrent>(f);
  }
  CUcontext ctx = nullptr;
  if (ctx_get(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  if (ctx)
    for (int i = 0; i < n_seen; ++i)
      if (seen[i].dev == dev && seen[i].ctx == ctx) {
        *out = seen[i].addr;
        return MOE_OK;
      }
  // the lookup makes the device's primary context current if none was
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_group_scratch);
  if (e != cudaSuccess || !p) return MOE_ERR_CUDA;
  if (!ctx && (ctx_get(&ctx) != CUDA_SUCCESS || !ctx)) return MOE_ERR_CUDA;
  if (n_seen < 64) seen[n_seen++] = Entry{dev, ctx, static_cast<int32_t*>(p)};
  *out = static_cast<int32_t*>(p);
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_group_subset(
    const int32_t* expert_offsets, const int32_t* pair_ids, int E,
    const int32_t* experts, int n, int32_t* sub_offsets, int32_t* sub_pairs,
    int32_t* sub_active, int32_t* sub_n_active, int32_t* err, void* stream) {
  MOE_TRACE();
  if (!expert_offsets || !pair_ids || !experts || !sub_offsets ||
      !sub_pairs || !sub_active || !sub_n_active || !err)
    return MOE_ERR_INVALID;
  if (E <= 0 || E > EMAX || n < 0 || n > E) return MOE_ERR_SHAPE;
  group_subset_kernel<<<SUB_BLOCKS, 1024, 0, (cudaStream_t)stream>>>(
      expert_offsets, pair_ids, E, experts, n, sub_offsets, sub_pairs,
      sub_active, sub_n_active, err);
  return launch_status();
}

extern "C" moe_status moe_group_tokens_static(
    const int32_t* topk_idx, int T, int k, int E, int32_t* expert_offsets,
    int32_t* pair_ids, int32_t* active, int32_t* n_active, int32_t* err,
    void* stream) {
  if (!topk_idx || !expert_offsets || !pair_ids || !active || !n_active)
    return MOE_ERR_INVALID;
  if (T <= 0 || k <= 0 || E <= 0) return MOE_ERR_SHAPE;
  if ((int64_t)T * k > STATIC_GROUP_MAX_PAIRS || E > STATIC_GROUP_MAX_E)
    return MOE_ERR_SHAPE;   // beyond the fixed scratch array
  int32_t* base = nullptr;
  const moe_status st = group_scratch_address(&base);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* e = err;
  if (!e) {
    e = base;   // the array's own error word, cleared for this call
    MOE_CUDA_TRY(cudaMemsetAsync(e, 0, sizeof(int32_t), s));
  }
  return launch_group(topk_idx, T, k, E, expert_offsets, pair_ids, active,
                      n_active, base + 64, e, s);
}
