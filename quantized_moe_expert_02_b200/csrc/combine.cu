// Weighted combine of the k expert outputs of each token, and the
// row-wise RMS normalisation used between the layers of a stack.
#include "moe_internal.cuh"
#include "trace.h"

namespace moe {

// out[t,h] = sum_j w[t,j] * y[t*k+j, h]  (j ascending)  + residual[t,h]
__global__ void combine_kernel(const float* __restrict__ y,
                               const float* __restrict__ w, int T, int k,
                               int H, const float* residual, float* out,
                               uint16_t* __restrict__ out_bf16) {
  const int64_t n = (int64_t)T * H;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / H), h = (int)(i % H);
    float acc = 0.f;
    for (int j = 0; j < k; ++j)
      acc = fmaf(w[(int64_t)t * k + j], y[((int64_t)t * k + j) * H + h], acc);
    if (residual) acc += residual[i];
    out[i] = acc;
    if (out_bf16) out_bf16[i] = f32_to_bf16_rne(acc);
  }
}

// The same sum, one block per token and four columns per thread: four of
// the k rows' float4 loads are issued before their multiply-adds, which
// run in the same order (j ascending, then the residual), so the result
// is bit-identical to the one-column form.  H a multiple of 4, 16-byte
// aligned y/residual/out.
__global__ void __launch_bounds__(256)
    combine_row_kernel(const float4* __restrict__ y,
                       const float* __restrict__ w, int k, int H4,
                       const float4* residual, float4* out,
                       uint2* __restrict__ out_bf16) {
  constexpr int CH = 4;
  const int64_t t = blockIdx.x;
  const float* wt = w + t * k;
  const float4* yt = y + t * k * H4;
  for (int h = threadIdx.x; h < H4; h += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < k; j0 += CH) {
      float4 v[CH];
#pragma unroll
      for (int jj = 0; jj < CH; ++jj)
        if (j0 + jj < k) v[jj] = __ldcs(yt + (int64_t)(j0 + jj) * H4 + h);
#pragma unroll
      for (int jj = 0; jj < CH; ++jj)
        if (j0 + jj < k) {
          const float wj = __ldg(wt + j0 + jj);
          acc.x = fmaf(wj, v[jj].x, acc.x);
          acc.y = fmaf(wj, v[jj].y, acc.y);
          acc.z = fmaf(wj, v[jj].z, acc.z);
          acc.w = fmaf(wj, v[jj].w, acc.w);
        }
    }
    const int64_t i = t * H4 + h;
    if (residual) {
      const float4 r = residual[i];
      acc.x += r.x;
      acc.y += r.y;
      acc.z += r.z;
      acc.w += r.w;
    }
    out[i] = acc;
    if (out_bf16)
      out_bf16[i] = make_uint2(
          (uint32_t)f32_to_bf16_rne(acc.x) |
              ((uint32_t)f32_to_bf16_rne(acc.y) << 16),
          (uint32_t)f32_to_bf16_rne(acc.z) |
              ((uint32_t)f32_to_bf16_rne(acc.w) << 16));
  }
}

// x = bf16(r / sqrt(mean(r^2) + eps)), one block per row.
__global__ void __launch_bounds__(256)
    rmsnorm_bf16_kernel(const float* __restrict__ r, int H,
                        uint16_t* __restrict__ x) {
  __shared__ float red[8];
  const float* row = r + (int64_t)blockIdx.x * H;
  float s = 0.f;
  for (int h = threadIdx.x; h < H; h += blockDim.x) s = fmaf(row[h], row[h], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
  const float inv = 1.0f / sqrtf(tot / (float)H + 1e-6f);
  for (int h = threadIdx.x; h < H; h += blockDim.x)
    x[(int64_t)blockIdx.x * H + h] = f32_to_bf16_rne(row[h] * inv);
}

moe_status launch_combine(const float* y, const float* w, int T, int k,
                          int H, const float* residual, float* out,
                          uint16_t* out_bf16, cudaStream_t s) {
  auto a16 = [](const void* q) {
    return (reinterpret_cast<uintptr_t>(q) & 15) == 0;
  };
  const bool vec = H % 4 == 0 && a16(y) && a16(out) &&
                   (!residual || a16(residual)) &&
                   (!out_bf16 || (reinterpret_cast<uintptr_t>(out_bf16) & 7) == 0);
  if (vec) {
    combine_row_kernel<<<T, 256, 0, s>>>(
        reinterpret_cast<const float4*>(y), w, k, H / 4,
        reinterpret_cast<const float4*>(residual),
        reinterpret_cast<float4*>(out), reinterpret_cast<uint2*>(out_bf16));
  } else {
    const int64_t n = (int64_t)T * H;
    int64_t g = (n + 255) / 256;
    if (g > (int64_t)num_sms() * 8) g = (int64_t)num_sms() * 8;
    combine_kernel<<<(int)g, 256, 0, s>>>(y, w, T, k, H, residual, out,
                                          out_bf16);
  }
  return launch_status();
}

moe_status launch_rmsnorm_bf16(const float* r, int T, int H, uint16_t* x,
                               cudaStream_t s) {
  rmsnorm_bf16_kernel<<<T, 256, 0, s>>>(r, H, x);
  return launch_status();
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_combine(const float* y_pairs, const float* topk_w,
                                  int T, int k, int H, const float* residual,
                                  float* out, uint16_t* out_bf16,
                                  void* stream) {
  MOE_TRACE();
  if (!y_pairs || !topk_w || !out) return MOE_ERR_INVALID;
  if (T <= 0 || k <= 0 || H <= 0) return MOE_ERR_SHAPE;
  return launch_combine(y_pairs, topk_w, T, k, H, residual, out, out_bf16,
                        (cudaStream_t)stream);
}

extern "C" moe_status moe_rmsnorm_bf16(const float* r, int T, int H,
                                       uint16_t* x_out, void* stream) {
  MOE_TRACE();
  if (!r || !x_out) return MOE_ERR_INVALID;
  if (T <= 0 || H <= 0) return MOE_ERR_SHAPE;
  return launch_rmsnorm_bf16(r, T, H, x_out, (cudaStream_t)stream);
}
