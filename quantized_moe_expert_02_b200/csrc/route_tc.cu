// Router logits for many tokens on the 5th-generation tensor cores:
//   logits[t][e] = sum_h x[t][h] * Wr[e][h] + bias[e]
// (the router of the MoE layer in the "Avalon" README: 512 experts, top-10
// chosen from the softmax over all of them).  bf16 operands, exact
// products, fp32 accumulation in tensor memory, one fp32 bias add.
//
// One persistent CTA per SM; a unit is 128 experts x 128 tokens.  Warps 0-3
// move accumulators out of TMEM, warp 4 owns TMEM and issues the MMAs,
// warp 5 issues the TMA copies of both operands (128-byte swizzle, rows
// past E or T read as zeros).
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace moe {
namespace {

constexpr int RT_BM = 128, RT_BN = 128, RT_BK = 64, RT_STAGES = 6;
constexpr int RT_THREADS = 192;
constexpr int RT_TILE_BYTES = RT_BM * RT_BK * 2;   // 16 KB (A and B alike)
constexpr int RT_STAGE_BYTES = 2 * RT_TILE_BYTES;
constexpr int RT_BAR_OFF = RT_STAGES * RT_STAGE_BYTES;
constexpr int RT_SMEM = RT_BAR_OFF + 256 + 1024;
constexpr int RT_TMEM_COLS = 256;   // two 128-column accumulators

struct RtParams {
  int T, E, H;
  const float* bias;
  float* logits;
  int32_t* err;
};

__global__ void __launch_bounds__(RT_THREADS, 1)
    route_tc_kernel(const RtParams p, const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_x) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RT_BAR_OFF);
  uint64_t* empty = full + RT_STAGES;
  uint64_t* acc_full = empty + RT_STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RT_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    tc::tmem_alloc(tmem_slot, RT_TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int mt = (p.E + RT_BM - 1) / RT_BM;
  const int n_units = mt * ((p.T + RT_BN - 1) / RT_BN);
  const int nk = p.H / RT_BK;
  int32_t* err = p.err;

  if (warp == 5) {
    if (lane == 0) {   // ------------------------------- TMA producer ---
      uint32_t kstep = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
        const int m = u % mt, n = u / mt;
        for (int ks = 0; ks < nk; ++ks, ++kstep) {
          const int s = (int)(kstep % RT_STAGES);
          const uint32_t use = kstep / RT_STAGES;
          if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, err)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + (uint32_t)(s * RT_STAGE_BYTES);
          mbar_arrive_expect_tx(&full[s], RT_STAGE_BYTES);
          tc::tma_load_2d(st, &map_w, ks * RT_BK, m * RT_BM, &full[s]);
          tc::tma_load_2d(st + RT_TILE_BYTES, &map_x, ks * RT_BK, n * RT_BN,
                          &full[s]);
        }
      }
    }
  } else if (warp == 4) {
    if (lane == 0) {   // ------------------------------------ MMA --------
      // bf16 A and B (K-major), fp32 D, M = N = 128
      const uint32_t idesc = tc::idesc_f16_f32(RT_BM, RT_BN) | (1u << 7) |
                             (1u << 10);
      uint32_t kstep = 0;
      bool ok = true;
      int it = 0;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++it) {
        const int ab = it & 1, use_ab = it >> 1;
        if (use_ab > 0 && !mbar_wait(&acc_empty[ab], (use_ab - 1) & 1, err))
          break;
        tc::fence_after_sync();
        const uint32_t d = tmem + (uint32_t)(ab * RT_BN);
        for (int ks = 0; ks < nk; ++ks, ++kstep) {
          const int s = (int)(kstep % RT_STAGES);
          if (!mbar_wait(&full[s], (kstep / RT_STAGES) & 1, err)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t st = sbase + (uint32_t)(s * RT_STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_f16(d, tc::sdesc_sw128(st + 32 * kk),
                        tc::sdesc_sw128(st + RT_TILE_BYTES + 32 * kk), idesc,
                        (ks | kk) != 0);
          tc::commit(&empty[s]);
        }
        if (!ok) break;
        tc::commit(&acc_full[ab]);
      }
      tc::commit(drain);
      mbar_wait(drain, 0, err);
    }
  } else {   // ------------------------------------------- epilogue -------
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int it = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++it) {
      const int m = u % mt, n = u / mt;
      const int ab = it & 1, use_ab = it >> 1;
      const int e = m * RT_BM + warp * 32 + lane;
      const bool ev = e < p.E;
      const float b = (ev && p.bias) ? p.bias[e] : 0.f;
      if (!mbar_wait(&acc_full[ab], use_ab & 1, err)) break;
      tc::fence_after_sync();
      const int t0 = n * RT_BN;
      float* lp = p.logits + (int64_t)t0 * p.E + e;
      for (int c0 = 0; c0 < RT_BN && t0 + c0 < p.T; c0 += 32) {
        float acc[32];
        const uint32_t ta = tmem + lane_base + (uint32_t)(ab * RT_BN + c0);
        tc::ld_32x32b_x16(ta, *(float(*)[16])&acc[0]);
        tc::ld_32x32b_x16(ta + 16, *(float(*)[16])&acc[16]);
        tc::wait_ld();
        if (ev) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (t0 + c0 + i < p.T) lp[(int64_t)(c0 + i) * p.E] = acc[i] + b;
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 4) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, RT_TMEM_COLS);
  }
}

moe_status encode_bf16_map(CUtensorMap* m, const void* base, uint64_t inner,
                           uint64_t outer, uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!fn) {
      void* f = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f,
                                  cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !f)
        return MOE_ERR_CUDA;
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
  }
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {(cuuint32_t)RT_BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
         dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

bool route_tc_supported(int T, int H) {
  return T > DEC_TMAX && H % RT_BK == 0;
}

moe_status launch_route_tc(const uint16_t* x, int T, int H,
                           const uint16_t* wr, int E, const float* bias,
                           float* logits, int32_t* err, cudaStream_t s) {
  CUtensorMap mw, mx;
  moe_status st = encode_bf16_map(&mw, wr, (uint64_t)H, (uint64_t)E, RT_BM);
  if (st != MOE_OK) return st;
  st = encode_bf16_map(&mx, x, (uint64_t)H, (uint64_t)T, RT_BN);
  if (st != MOE_OK) return st;
  st = ensure_smem(reinterpret_cast<const void*>(&route_tc_kernel), RT_SMEM);
  if (st != MOE_OK) return st;
  RtParams p{T, E, H, bias, logits, err};
  route_tc_kernel<<<num_sms(), RT_THREADS, RT_SMEM, s>>>(p, mw, mx);
  return launch_status();
}

}  // namespace moe
