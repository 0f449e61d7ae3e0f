// Expert staging without a host round trip per layer.  The "Betelgeuse"
// post fills missed slots with a host pager that a doorbell in the decode
// stream wakes.  Here the host copies of the blobs already sit in pinned
// host memory, so the GPU pulls them itself: after the slot resolve, one
// kernel on the same stream reads each missed blob from mapped pinned host
// memory (over PCIe) and writes it into its victim slot.  Nothing waits on
// the host or on another stream, the step stays capturable in one CUDA
// graph, and the layer's FFN that follows on the stream sees the blobs.
//
// A host thread that copies the misses while the stream waits on a flag
// cannot be made safe here: streams share hardware queues, so its copies
// can sit behind the very launches that the waiting kernel holds up.
#include <vector>

#include "moe_internal.cuh"
#include "trace.h"

namespace moe {
namespace {

constexpr int STAGE_THREADS = 512;
constexpr int STAGE_UNROLL = 4;   // 16-byte loads in flight per thread

// Grid-stride over (miss, 16-byte word); each thread has STAGE_UNROLL loads
// from host memory in flight before it stores them.
__global__ void __launch_bounds__(STAGE_THREADS)
    stage_misses_kernel(const int32_t* n_miss, const int32_t* miss_expert,
                        const int32_t* miss_slot, int P, int layer, int E,
                        int slot_base, int n_slots, int64_t pool_slots,
                        const uint64_t* table, uint8_t* pool, int64_t stride,
                        int64_t blob_bytes, int32_t* err) {
  const int n = *n_miss;
  if (n < 0 || n > P) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_err(err, MOE_ERR_DEVICE);
    return;
  }
  const int64_t words = blob_bytes / 16;          // per blob
  const int64_t total = (int64_t)n * words;
  const int64_t step = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
       i0 < total; i0 += step * STAGE_UNROLL) {
    uint4 v[STAGE_UNROLL];
    uint4* dst[STAGE_UNROLL];
#pragma unroll
    for (int u = 0; u < STAGE_UNROLL; ++u) {
      const int64_t i = i0 + u * step;
      dst[u] = nullptr;
      if (i >= total) continue;
      const int m = (int)(i / words);
      const int64_t w = i % words;
      const int e = miss_expert[m];
      const int ls = miss_slot[m];   // slot inside the layer's partition
      const int64_t slot = (int64_t)slot_base + ls;
      const uint64_t src = (e >= 0 && e < E) ? table[(int64_t)layer * E + e]
                                             : 0ull;
      // no host copy, or a slot outside the layer's partition: skipped
      if (src == 0ull || ls < 0 || ls >= n_slots || slot >= pool_slots) {
        if (w == 0) set_err(err, MOE_ERR_CAPACITY);
        continue;
      }
      v[u] = reinterpret_cast<const uint4*>(src)[w];
      dst[u] = reinterpret_cast<uint4*>(pool + slot * stride) + w;
    }
#pragma unroll
    for (int u = 0; u < STAGE_UNROLL; ++u)
      if (dst[u]) *dst[u] = v[u];
  }
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_stage_table(const void* const* host_blob, int n,
                                      uint64_t* table, void* stream) {
  MOE_TRACE();
  if (!host_blob || !table || n < 1) return MOE_ERR_INVALID;
  std::vector<uint64_t> t((size_t)n, 0ull);
  for (int i = 0; i < n; ++i) {
    if (!host_blob[i]) continue;
    if (reinterpret_cast<uintptr_t>(host_blob[i]) % 16)
      return MOE_ERR_INVALID;
    // only pinned (registered, mapped) host memory may be read by the
    // kernel; pageable memory is rejected even where the device could
    // reach it
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, host_blob[i]) != cudaSuccess ||
        a.type != cudaMemoryTypeHost || !a.devicePointer) {
      cudaGetLastError();
      return MOE_ERR_INVALID;
    }
    // (the attributes may describe the allocation's start: keep the offset)
    t[(size_t)i] =
        reinterpret_cast<uint64_t>(a.devicePointer) +
        (reinterpret_cast<uint64_t>(host_blob[i]) -
         reinterpret_cast<uint64_t>(a.hostPointer ? a.hostPointer
                                                  : host_blob[i]));
  }
  cudaStream_t s = (cudaStream_t)stream;
  MOE_CUDA_TRY(cudaMemcpyAsync(table, t.data(), (size_t)n * 8,
                               cudaMemcpyHostToDevice, s));
  // the host vector dies on return: wait for the copy
  MOE_CUDA_TRY(cudaStreamSynchronize(s));
  return MOE_OK;
}

extern "C" moe_status moe_stage_misses(const int32_t* n_miss,
                                       const int32_t* miss_expert,
                                       const int32_t* miss_slot, int P,
                                       int layer, int L, int E,
                                       const uint64_t* table,
                                       uint8_t* pool, int slot_base,
                                       int n_slots, int64_t pool_slots,
                                       int64_t blob_stride,
                                       int64_t blob_bytes, int32_t* err,
                                       void* stream) {
  MOE_TRACE();
  if (!n_miss || !miss_expert || !miss_slot || !table || !pool)
    return MOE_ERR_INVALID;
  if (P < 1 || layer < 0 || layer >= L || E < 1 || slot_base < 0 ||
      n_slots < 1 || pool_slots < 1 ||
      slot_base + (int64_t)n_slots > pool_slots ||
      blob_bytes < 16 || blob_bytes % 16 || blob_stride % 16 ||
      blob_stride < blob_bytes || reinterpret_cast<uintptr_t>(pool) % 16)
    return MOE_ERR_SHAPE;
  moe::stage_misses_kernel<<<moe::num_sms(), moe::STAGE_THREADS, 0,
                             (cudaStream_t)stream>>>(
      n_miss, miss_expert, miss_slot, P, layer, E, slot_base, n_slots,
      pool_slots,
      table, pool, blob_stride, blob_bytes, err);
  return moe::launch_status();
}
