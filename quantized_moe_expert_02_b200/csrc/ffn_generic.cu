// Expert FFN, general path (any number of tokens): per expert, the weight
// rows are dequantised into shared memory as fp32 and dotted with the
// expert's token rows.  h = silu(Wg x) * (Wu x), y = Wd h (SwiGLU expert of
// the Avalon model; up/gate/down tensors of the model card).
#include "moe_internal.cuh"

namespace moe {

constexpr int GEN_UP_ROWS = 4;    // F rows per block (x2 tensors)
constexpr int GEN_DN_ROWS = 8;    // H rows per block

struct ExpertRef {
  const uint8_t* pool;
  int64_t stride;
  const int32_t* blob_index;
  int E;
};

__device__ inline const uint8_t* expert_blob(const ExpertRef& r, int e,
                                             int32_t* err) {
  int64_t b = e;
  if (r.blob_index) b = r.blob_index[e];
  if (b < 0) { set_err(err, MOE_ERR_DEVICE); return nullptr; }
  return r.pool + b * r.stride;
}

__global__ void __launch_bounds__(256)
    ffn_up_generic_kernel(ExpertRef ref, int fmt, int H, int F,
                          int64_t gate_off, const uint16_t* __restrict__ x,
                          int k, const int32_t* __restrict__ offsets,
                          const int32_t* __restrict__ pair_ids,
                          const int32_t* __restrict__ active,
                          const int32_t* __restrict__ n_active,
                          float* __restrict__ h, int32_t* err) {
  extern __shared__ float wsm[];  // [2][GEN_UP_ROWS][H]
  const int u = blockIdx.y;
  if (u >= *n_active) return;
  const int e = active[u];
  if (e < 0 || e >= ref.E) { set_err(err, MOE_ERR_DEVICE); return; }
  const uint8_t* blob = expert_blob(ref, e, err);
  if (!blob) return;
  const int f0 = blockIdx.x * GEN_UP_ROWS;
  for (int i = threadIdx.x; i < 2 * GEN_UP_ROWS * H; i += blockDim.x) {
    const int tz = i / (GEN_UP_ROWS * H);
    const int r = (i / H) % GEN_UP_ROWS, c = i % H;
    wsm[i] = dq_packed(fmt, blob + tz * gate_off, H, f0 + r, c);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int p0 = offsets[e], np = offsets[e + 1] - p0;
  for (int i = warp; i < np; i += blockDim.x >> 5) {
    const int p = pair_ids[p0 + i];
    const uint16_t* xr = x + (int64_t)(p / k) * H;
    float acc[2 * GEN_UP_ROWS] = {};
    for (int c = lane; c < H; c += 32) {
      const float xv = bf16_to_f32(xr[c]);
#pragma unroll
      for (int q = 0; q < 2 * GEN_UP_ROWS; ++q)
        acc[q] = fmaf(wsm[q * H + c], xv, acc[q]);
    }
#pragma unroll
    for (int q = 0; q < 2 * GEN_UP_ROWS; ++q)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
    if (lane < GEN_UP_ROWS) {
      float uu = acc[0], gg = acc[GEN_UP_ROWS];
#pragma unroll
      for (int q = 1; q < GEN_UP_ROWS; ++q)
        if (lane == q) { uu = acc[q]; gg = acc[GEN_UP_ROWS + q]; }
      const float sg = gg / (1.0f + expf(-gg));
      h[(int64_t)p * F + f0 + lane] = sg * uu;
    }
  }
}

__global__ void __launch_bounds__(256)
    ffn_down_generic_kernel(ExpertRef ref, int fmt, int H, int F,
                            int64_t down_off, int k,
                            const int32_t* __restrict__ offsets,
                            const int32_t* __restrict__ pair_ids,
                            const int32_t* __restrict__ active,
                            const int32_t* __restrict__ n_active,
                            const float* __restrict__ h,
                            float* __restrict__ y, int32_t* err) {
  extern __shared__ float wsm[];  // [GEN_DN_ROWS][F]
  const int u = blockIdx.y;
  if (u >= *n_active) return;
  const int e = active[u];
  if (e < 0 || e >= ref.E) { set_err(err, MOE_ERR_DEVICE); return; }
  const uint8_t* blob = expert_blob(ref, e, err);
  if (!blob) return;
  const int r0 = blockIdx.x * GEN_DN_ROWS;
  for (int i = threadIdx.x; i < GEN_DN_ROWS * F; i += blockDim.x)
    wsm[i] = dq_packed(fmt, blob + down_off, F, r0 + i / F, i % F);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int p0 = offsets[e], np = offsets[e + 1] - p0;
  for (int i = warp; i < np; i += blockDim.x >> 5) {
    const int p = pair_ids[p0 + i];
    const float* hr = h + (int64_t)p * F;
    float acc[GEN_DN_ROWS] = {};
    for (int c = lane; c < F; c += 32) {
      const float hv = hr[c];
#pragma unroll
      for (int q = 0; q < GEN_DN_ROWS; ++q)
        acc[q] = fmaf(wsm[q * F + c], hv, acc[q]);
    }
#pragma unroll
    for (int q = 0; q < GEN_DN_ROWS; ++q)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < GEN_DN_ROWS; ++q)
        y[(int64_t)p * H + r0 + q] = acc[q];
    }
  }
}

static moe_status set_smem(const void* fn, size_t bytes) {
  if (bytes > 200 * 1024) return MOE_ERR_SHAPE;
  return ensure_smem(fn, bytes);
}

moe_status launch_up_generic(const moe_layer_desc& d, const uint16_t* x,
                             int T, int k, const int32_t* offsets,
                             const int32_t* pair_ids, const int32_t* active,
                             const int32_t* n_active,
                             const int32_t* blob_index, float* h,
                             int32_t* err, cudaStream_t s) {
  ExpertRef ref{d.pool, d.blob_stride, blob_index, d.E};
  const int64_t ug = tensor_bytes_of(d.fmt_up_gate, d.F, d.H);
  const int max_u = T * k < d.E ? T * k : d.E;
  const size_t smem = (size_t)2 * GEN_UP_ROWS * d.H * sizeof(float);
  moe_status st = set_smem((const void*)ffn_up_generic_kernel, smem);
  if (st != MOE_OK) return st;
  ffn_up_generic_kernel<<<dim3(d.F / GEN_UP_ROWS, max_u), 256, smem, s>>>(
      ref, d.fmt_up_gate, d.H, d.F, ug, x, k, offsets, pair_ids, active,
      n_active, h, err);
  return launch_status();
}

moe_status launch_down_generic(const moe_layer_desc& d, int T, int k,
                               const int32_t* offsets,
                               const int32_t* pair_ids, const int32_t* active,
                               const int32_t* n_active,
                               const int32_t* blob_index, const float* h,
                               float* y, int32_t* err, cudaStream_t s) {
  ExpertRef ref{d.pool, d.blob_stride, blob_index, d.E};
  const int64_t ug = tensor_bytes_of(d.fmt_up_gate, d.F, d.H);
  const int max_u = T * k < d.E ? T * k : d.E;
  const size_t smem = (size_t)GEN_DN_ROWS * d.F * sizeof(float);
  moe_status st = set_smem((const void*)ffn_down_generic_kernel, smem);
  if (st != MOE_OK) return st;
  ffn_down_generic_kernel<<<dim3(d.H / GEN_DN_ROWS, max_u), 256, smem, s>>>(
      ref, d.fmt_down, d.H, d.F, 2 * ug, k, offsets, pair_ids, active,
      n_active, h, y, err);
  return launch_status();
}

}  // namespace moe
