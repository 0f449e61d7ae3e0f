// Expert-slot resolution on the device ("Betelgeuse" post: a VRAM pool of
// expert slots with non-uniform per-layer capacity; an in-stream kernel
// resolves hits and reports only the misses).  One block per call.
#include "moe_internal.cuh"
#include "trace.h"

namespace moe {

constexpr int SLOT_EMAX = 8192;
constexpr int SLOT_NMAX = 8192;
constexpr int SLOT_PMAX = 1024;

__global__ void __launch_bounds__(1024)
    slot_resolve_kernel(const int32_t* __restrict__ topk_idx, int P, int E,
                        int32_t* __restrict__ table, int32_t* __restrict__ owner,
                        uint32_t* __restrict__ last_use, int n_slots,
                        int slot_base, uint32_t stamp_arg,
                        uint32_t* stamp_ctr,
                        int32_t* __restrict__ blob_index,
                        int32_t* __restrict__ miss_expert,
                        int32_t* __restrict__ miss_slot,
                        int32_t* __restrict__ n_miss, int32_t* err) {
  __shared__ uint8_t chosen[SLOT_EMAX];
  __shared__ uint8_t used[SLOT_NMAX];
  __shared__ int32_t misses[SLOT_PMAX];
  __shared__ int32_t victims[SLOT_PMAX];
  __shared__ int32_t s_nmiss, s_nhit, s_bad;
  __shared__ unsigned long long s_best;
  const int tid = threadIdx.x;
  // with a device counter, this call's stamp is the counter + 1 (stored
  // back below, once the call updates the partition)
  const uint32_t stamp = stamp_ctr ? *stamp_ctr + 1u : stamp_arg;
  for (int e = tid; e < E; e += blockDim.x) chosen[e] = 0;
  for (int s = tid; s < n_slots; s += blockDim.x) used[s] = 0;
  if (tid == 0) { s_nmiss = 0; s_nhit = 0; s_bad = 0; }
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = topk_idx[p];
    if (e < 0 || e >= E) { s_bad = 1; continue; }
    chosen[e] = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) { set_err(err, MOE_ERR_DEVICE); *n_miss = 0; }
    return;
  }
  // hits mark their slot; misses are collected below in ascending id
  for (int e = tid; e < E; e += blockDim.x) {
    if (!chosen[e]) continue;
    const int s = table[e];
    if (s >= 0 && s < n_slots) {
      used[s] = 1;
      atomicAdd(&s_nhit, 1);
    }
  }
  __syncthreads();
  if (tid < 32) {  // ascending compaction of the misses by warp 0
    int count = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + tid;
      const bool miss = e < E && chosen[e] &&
                        !(table[e] >= 0 && table[e] < n_slots);
      const unsigned b = __ballot_sync(0xffffffffu, miss);
      if (miss) misses[count + __popc(b & ((1u << tid) - 1u))] = e;
      count += __popc(b);
    }
    if (tid == 0) s_nmiss = count;
  }
  __syncthreads();
  const int nm = s_nmiss;
  if (nm > n_slots - s_nhit) {
    if (tid == 0) { set_err(err, MOE_ERR_CAPACITY); *n_miss = 0; }
    return;
  }
  // victims: the i-th miss takes the unused slot with the i-th smallest
  // (last_use, slot); one block-wide arg-min per miss
  for (int i = 0; i < nm; ++i) {
    if (tid == 0) s_best = ~0ull;
    __syncthreads();
    unsigned long long best = ~0ull;
    for (int s = tid; s < n_slots; s += blockDim.x)
      if (!used[s]) {
        const unsigned long long key =
            ((unsigned long long)last_use[s] << 32) | (unsigned)s;
        if (key < best) best = key;
      }
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long ob = __shfl_xor_sync(0xffffffffu, best, o);
      if (ob < best) best = ob;
    }
    if ((tid & 31) == 0) atomicMin(&s_best, best);
    __syncthreads();
    if (tid == 0) {
      const int v = (int)(s_best & 0xffffffffu);
      victims[i] = v;
      used[v] = 1;
    }
    __syncthreads();
  }
  // apply: evict, fill, stamp
  if (tid == 0) {
    for (int i = 0; i < nm; ++i) {
      const int e = misses[i], v = victims[i];
      const int old = owner[v];
      if (old >= 0 && old < E) table[old] = -1;
      owner[v] = e;
      table[e] = v;
      miss_expert[i] = e;
      miss_slot[i] = v;
    }
    *n_miss = nm;
    if (stamp_ctr) *stamp_ctr = stamp;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x)
    if (chosen[e]) blob_index[e] = slot_base + table[e];
  for (int s = tid; s < n_slots; s += blockDim.x)
    if (used[s]) last_use[s] = stamp;
}

}  // namespace moe

using namespace moe;

static moe_status slot_resolve(const int32_t* topk_idx, int T, int k, int E,
                               int32_t* slot_table, int32_t* slot_owner,
                               uint32_t* last_use, int n_slots, int slot_base,
                               uint32_t stamp, uint32_t* stamp_ctr,
                               int32_t* blob_index, int32_t* miss_expert,
                               int32_t* miss_slot, int32_t* n_miss,
                               int32_t* err, void* stream) {
  if (!topk_idx || !slot_table || !slot_owner || !last_use || !blob_index ||
      !miss_expert || !miss_slot || !n_miss || !err)
    return MOE_ERR_INVALID;
  if (T <= 0 || k <= 0 || E <= 0 || n_slots <= 0 || slot_base < 0)
    return MOE_ERR_SHAPE;
  if ((int64_t)T * k > SLOT_PMAX || E > SLOT_EMAX || n_slots > SLOT_NMAX)
    return MOE_ERR_SHAPE;
  slot_resolve_kernel<<<1, 1024, 0, (cudaStream_t)stream>>>(
      topk_idx, T * k, E, slot_table, slot_owner, last_use, n_slots,
      slot_base, stamp, stamp_ctr, blob_index, miss_expert, miss_slot, n_miss,
      err);
  return launch_status();
}

extern "C" moe_status moe_slot_resolve(const int32_t* topk_idx, int T, int k,
                                       int E, int32_t* slot_table,
                                       int32_t* slot_owner,
                                       uint32_t* last_use, int n_slots,
                                       int slot_base, uint32_t stamp,
                                       int32_t* blob_index,
                                       int32_t* miss_expert,
                                       int32_t* miss_slot, int32_t* n_miss,
                                       int32_t* err, void* stream) {
  MOE_TRACE();
  return slot_resolve(topk_idx, T, k, E, slot_table, slot_owner, last_use,
                      n_slots, slot_base, stamp, nullptr, blob_index,
                      miss_expert, miss_slot, n_miss, err, stream);
}

extern "C" moe_status moe_slot_resolve_dev(
    const int32_t* topk_idx, int T, int k, int E, int32_t* slot_table,
    int32_t* slot_owner, uint32_t* last_use, int n_slots, int slot_base,
    uint32_t* stamp, int32_t* blob_index, int32_t* miss_expert,
    int32_t* miss_slot, int32_t* n_miss, int32_t* err, void* stream) {
  MOE_TRACE();
  if (!stamp) return MOE_ERR_INVALID;
  return slot_resolve(topk_idx, T, k, E, slot_table, slot_owner, last_use,
                      n_slots, slot_base, 0u, stamp, blob_index, miss_expert,
                      miss_slot, n_miss, err, stream);
}
