// Router logits and top-k ("Avalon" README: 512 routed experts, 10 active
// per token; softmax over all experts, top-k by probability with equal
// values to the lower index, weights renormalised over the k chosen).
#include <float.h>

#include "moe_internal.cuh"

namespace moe {

// ---------------------------------------------------------------------
// Decode-sized logits (T <= 8): one warp per expert row, the x rows staged
// in shared memory as bf16.  Each lane accumulates its 8-element chunks in
// fp32, then a fixed xor-butterfly reduces the warp (deterministic).
__global__ void __launch_bounds__(256)
    route_logits_small_kernel(const uint16_t* __restrict__ x, int T, int H,
                              const uint16_t* __restrict__ wr, int E,
                              const float* __restrict__ bias,
                              float* __restrict__ logits) {
  extern __shared__ __align__(16) uint16_t xs[];  // [T][H]
  const int nchunk = H / 8;
  for (int i = threadIdx.x; i < T * nchunk; i += blockDim.x)
    reinterpret_cast<uint4*>(xs)[i] = reinterpret_cast<const uint4*>(x)[i];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); e < E;
       e += nwarps) {
    float acc[DEC_TMAX];
#pragma unroll
    for (int t = 0; t < DEC_TMAX; ++t) acc[t] = 0.f;
    const uint4* row = reinterpret_cast<const uint4*>(wr + (int64_t)e * H);
    for (int ch = lane; ch < nchunk; ch += 32) {
      const uint4 w = __ldg(row + ch);
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int t = 0; t < DEC_TMAX; ++t) {
        if (t < T) {
          const uint4 xv = reinterpret_cast<const uint4*>(xs + t * H)[ch];
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
          float a = acc[t];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            a = fmaf(__uint_as_float(wv[q] << 16), __uint_as_float(xw[q] << 16),
                     a);
            a = fmaf(__uint_as_float(wv[q] & 0xFFFF0000u),
                     __uint_as_float(xw[q] & 0xFFFF0000u), a);
          }
          acc[t] = a;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < DEC_TMAX; ++t) {
      float a = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      acc[t] = a;
    }
    if (lane == 0) {
      const float b = bias ? bias[e] : 0.f;
      for (int t = 0; t < T; ++t) logits[(int64_t)t * E + e] = acc[t] + b;
    }
  }
}

// Prefill-sized logits: 64 tokens x 64 experts per block, 256 threads each
// holding a 4x4 fp32 tile; K in steps of 32, accumulated in ascending k.
__global__ void __launch_bounds__(256)
    route_logits_tiled_kernel(const uint16_t* __restrict__ x, int T, int H,
                              const uint16_t* __restrict__ wr, int E,
                              const float* __restrict__ bias,
                              float* __restrict__ logits) {
  __shared__ float xs[32][65];
  __shared__ float ws[32][65];
  const int t0 = blockIdx.y * 64, e0 = blockIdx.x * 64;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < H; k0 += 32) {
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      const int r = i / 32, kk = i % 32;
      const int t = t0 + r, e = e0 + r;
      xs[kk][r] = (t < T && k0 + kk < H)
                      ? bf16_to_f32(x[(int64_t)t * H + k0 + kk]) : 0.f;
      ws[kk][r] = (e < E && k0 + kk < H)
                      ? bf16_to_f32(wr[(int64_t)e * H + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  for (int i = 0; i < 4; ++i)
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + ty * 4 + i, e = e0 + tx * 4 + j;
      if (t < T && e < E)
        logits[(int64_t)t * E + e] = acc[i][j] + (bias ? bias[e] : 0.f);
    }
}

// One warp per token: k rounds of a warp arg-max over the token's logits
// (value descending, index ascending), then the renormalised softmax
// weights w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max) over the chosen.
__global__ void __launch_bounds__(128)
    topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  extern __shared__ float sl[];  // [4 warps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + warp;
  if (t >= T) return;
  float* my = sl + (size_t)warp * E;
  for (int e = lane; e < E; e += 32) my[e] = logits[(int64_t)t * E + e];
  __syncwarp();
  float my_v = 0.f;   // lane r keeps round r's winner
  int my_i = 0;
  for (int r = 0; r < k; ++r) {
    float bv = -FLT_MAX;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float v = my[e];
      if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == r) { my_v = bv; my_i = bi; }
    if (lane == 0 && bi < E) my[bi] = -INFINITY;
    __syncwarp();
  }
  // weights: exp(l_r - l_0) summed in round order, as a serial loop would
  const float m = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = lane < k ? expf(my_v - m) : 0.f;
  float s = 0.f;
  for (int r = 0; r < k; ++r) s += __shfl_sync(0xffffffffu, ex, r);
  if (lane < k) {
    topk_idx[(int64_t)t * k + lane] = my_i;
    topk_w[(int64_t)t * k + lane] = ex / s;
  }
}

bool route_tc_supported(int T, int H);
moe_status launch_route_tc(const uint16_t* x, int T, int H,
                           const uint16_t* wr, int E, const float* bias,
                           float* logits, int32_t* err, cudaStream_t s);

moe_status launch_route(const uint16_t* x, int T, int H, const uint16_t* wr,
                        int E, const float* bias, int k, int32_t* topk_idx,
                        float* topk_w, float* logits, int32_t* err,
                        cudaStream_t s) {
  if (route_tc_supported(T, H)) {
    const moe_status st =
        launch_route_tc(x, T, H, wr, E, bias, logits, err, s);
    if (st != MOE_OK) return st;
  } else if (T <= DEC_TMAX) {
    const size_t smem = (size_t)T * H * 2;
    const moe_status st =
        ensure_smem((const void*)route_logits_small_kernel, smem);
    if (st != MOE_OK) return st;
    int grid = (E + 7) / 8;
    if (grid > num_sms()) grid = num_sms();
    route_logits_small_kernel<<<grid, 256, smem, s>>>(x, T, H, wr, E, bias,
                                                      logits);
  } else {
    dim3 grid((E + 63) / 64, (T + 63) / 64);
    route_logits_tiled_kernel<<<grid, 256, 0, s>>>(x, T, H, wr, E, bias,
                                                   logits);
  }
  MOE_CUDA_TRY(cudaGetLastError());
  const size_t smem = (size_t)4 * E * sizeof(float);
  const moe_status st = ensure_smem((const void*)topk_kernel, smem);
  if (st != MOE_OK) return st;
  topk_kernel<<<(T + 3) / 4, 128, smem, s>>>(logits, T, E, k, topk_idx,
                                             topk_w);
  return launch_status();
}

}  // namespace moe
