// Natural -> packed tile layout, and the dequantisation export.
// Formats: the expert quant types of the Avalon GGUF model card ("Files"):
// the 3.25-bpw super-block variant (one scale per 256 weights, 4-bit
// sub-scales per 32), the 4-bit non-uniform-codebook type, and this
// library's 3-bit non-uniform-codebook super-block (NL3).
#include "moe_internal.cuh"
#include "trace.h"

namespace moe {

// ---- natural layout readers ------------------------------------------
// SB3 natural: codes plane (96 B per super-block, code i at bit 3i), then
// sub-scale words, then fp16 d.
__device__ inline int nat_sb3_code(const uint8_t* codes, int cols, int row,
                                   int col) {
  const int64_t sb = (int64_t)row * (cols / 256) + col / 256;
  const int bit = 3 * (col % 256);
  const uint8_t* p = codes + sb * 96 + bit / 8;
  const uint32_t v = p[0] | ((bit / 8 + 1 < 96) ? ((uint32_t)p[1] << 8) : 0u);
  return (v >> (bit % 8)) & 7;
}
// SB2 natural: codes plane (64 B per super-block, code i at bit 2i).
__device__ inline int nat_sb2_code(const uint8_t* codes, int cols, int row,
                                   int col) {
  const int64_t sb = (int64_t)row * (cols / 256) + col / 256;
  const int i = col % 256;
  return (codes[sb * 64 + i / 4] >> (2 * (i % 4))) & 3;
}
__device__ inline int nat_b32_code(const uint8_t* codes, int cols, int row,
                                   int col) {
  const int64_t i = (int64_t)row * cols + col;
  const uint8_t b = codes[i / 2];
  return (i & 1) ? (b >> 4) : (b & 15);
}

// One thread per 32-bit word of the packed tensor.  SB3 and NL3 (the NL3
// tile appends the codebook-shift bytes of its 16 rows); SB2 below.
template <bool NL3>
__global__ void pack_sb3_kernel(const uint8_t* __restrict__ nat, int rows,
                                int cols, uint32_t* __restrict__ out) {
  constexpr int TBW = (NL3 ? NL3_TILE_BYTES : SB3_TILE_BYTES) / 4;
  const int ntc = cols / 256;
  const int64_t ntiles = (int64_t)(rows / 16) * ntc;
  const int64_t nwords = ntiles * TBW;
  const int64_t nsb = (int64_t)rows * ntc;
  const uint8_t* codes = nat;
  const uint32_t* scales = (const uint32_t*)(nat + nsb * 96);
  const uint16_t* dplane = (const uint16_t*)(nat + nsb * 100);
  const uint8_t* extra = nat + nsb * 102;   // NL3 only
  for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
       wi < nwords; wi += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = wi / TBW;
    const int w = (int)(wi % TBW);
    const int rt = (int)(tile / ntc), kb = (int)(tile % ntc);
    uint32_t word = 0;
    if (w < 384) {
      const int seg = w / 128, lane = (w % 128) / 4, iw = w % 4;
      const int g = lane / 4, c = lane % 4;
      if (seg < 2) {  // LO[j]
        const int j = 4 * seg + iw;
        for (int r = 0; r < 4; ++r)
          for (int e = 0; e < 4; ++e) {
            const int row = 16 * rt + g + 8 * (r & 1);
            const int col = 256 * kb + 32 * j + 16 * (r >> 1) + 4 * c + e;
            const int q = nat_sb3_code(codes, cols, row, col);
            const int n = 4 * (r & 1) + e;
            word |= (uint32_t)(q & 3) << (4 * n + 2 * (r >> 1));
          }
      } else {  // HI[m]: blocks 2m, 2m+1
        const int m = iw;
        for (int jj = 0; jj < 2; ++jj)
          for (int r = 0; r < 4; ++r)
            for (int e = 0; e < 4; ++e) {
              const int j = 2 * m + jj;
              const int row = 16 * rt + g + 8 * (r & 1);
              const int col = 256 * kb + 32 * j + 16 * (r >> 1) + 4 * c + e;
              const int q = nat_sb3_code(codes, cols, row, col);
              const int n = 4 * (r & 1) + e;
              word |= (uint32_t)(q >> 2) << (4 * n + 2 * jj + (r >> 1));
            }
      }
    } else if (w < 400) {  // sub-scale words, packed index pi
      const int pi = w - 384;
      const int r = pi / 2 + 8 * (pi % 2);
      word = scales[(int64_t)(16 * rt + r) * ntc + kb];
    } else if (w < 408) {  // d: two fp16 per word
      const int p0 = 2 * (w - 400);
      uint32_t lohi[2];
      for (int h = 0; h < 2; ++h) {
        const int pi = p0 + h;
        const int r = pi / 2 + 8 * (pi % 2);
        lohi[h] = dplane[(int64_t)(16 * rt + r) * ntc + kb];
      }
      word = lohi[0] | (lohi[1] << 16);
    } else {  // NL3 codebook-shift bytes: four per word
      for (int h = 0; h < 4; ++h) {
        const int pi = 4 * (w - 408) + h;
        const int r = pi / 2 + 8 * (pi % 2);
        word |= (uint32_t)extra[(int64_t)(16 * rt + r) * ntc + kb] << (8 * h);
      }
    }
    out[wi] = word;
  }
}

// SB2: the LO words of the SB3 tile (the 2-bit codes), then the sub-scale
// words and the fp16 d, one thread per 32-bit word.
__global__ void pack_sb2_kernel(const uint8_t* __restrict__ nat, int rows,
                                int cols, uint32_t* __restrict__ out) {
  constexpr int TBW = SB2_TILE_BYTES / 4;
  const int ntc = cols / 256;
  const int64_t ntiles = (int64_t)(rows / 16) * ntc;
  const int64_t nwords = ntiles * TBW;
  const int64_t nsb = (int64_t)rows * ntc;
  const uint8_t* codes = nat;
  const uint32_t* scales = (const uint32_t*)(nat + nsb * 64);
  const uint16_t* dplane = (const uint16_t*)(nat + nsb * 68);
  for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
       wi < nwords; wi += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = wi / TBW;
    const int w = (int)(wi % TBW);
    const int rt = (int)(tile / ntc), kb = (int)(tile % ntc);
    uint32_t word = 0;
    if (w < 256) {  // LO[j]
      const int seg = w / 128, lane = (w % 128) / 4, iw = w % 4;
      const int g = lane / 4, c = lane % 4;
      const int j = 4 * seg + iw;
      for (int r = 0; r < 4; ++r)
        for (int e = 0; e < 4; ++e) {
          const int row = 16 * rt + g + 8 * (r & 1);
          const int col = 256 * kb + 32 * j + 16 * (r >> 1) + 4 * c + e;
          const int q = nat_sb2_code(codes, cols, row, col);
          const int n = 4 * (r & 1) + e;
          word |= (uint32_t)q << (4 * n + 2 * (r >> 1));
        }
    } else if (w < 272) {  // sub-scale words, packed index pi
      const int pi = w - 256;
      const int r = pi / 2 + 8 * (pi % 2);
      word = scales[(int64_t)(16 * rt + r) * ntc + kb];
    } else {  // d: two fp16 per word
      const int p0 = 2 * (w - 272);
      uint32_t lohi[2];
      for (int h = 0; h < 2; ++h) {
        const int pi = p0 + h;
        const int r = pi / 2 + 8 * (pi % 2);
        lohi[h] = dplane[(int64_t)(16 * rt + r) * ntc + kb];
      }
      word = lohi[0] | (lohi[1] << 16);
    }
    out[wi] = word;
  }
}

__global__ void pack_b32_kernel(const uint8_t* __restrict__ nat, int rows,
                                int cols, uint32_t* __restrict__ out) {
  const int ntc = cols / 64;
  const int64_t ntiles = (int64_t)(rows / 16) * ntc;
  const int64_t nwords = ntiles * (B32_TILE_BYTES / 4);
  const uint8_t* codes = nat;
  const uint16_t* dplane = (const uint16_t*)(nat + (int64_t)rows * cols / 2);
  const int nb = cols / 32;
  for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
       wi < nwords; wi += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = wi / (B32_TILE_BYTES / 4);
    const int w = (int)(wi % (B32_TILE_BYTES / 4));
    const int rt = (int)(tile / ntc), kt = (int)(tile % ntc);
    uint32_t word = 0;
    if (w < 128) {
      const int lane = w / 4, iw = w % 4;
      const int g = lane / 4, c = lane % 4;
      const int b = iw / 2, h = iw % 2;
      for (int n = 0; n < 8; ++n) {
        const int row = 16 * rt + g + 8 * (n >> 2);
        const int col = 64 * kt + 32 * b + 16 * h + 4 * c + (n & 3);
        word |= (uint32_t)nat_b32_code(codes, cols, row, col) << (4 * n);
      }
    } else {
      const int p0 = 2 * (w - 128);
      uint32_t lohi[2];
      for (int hh = 0; hh < 2; ++hh) {
        const int idx = p0 + hh;  // = 4g + 2*half + b
        const int b = idx % 2, half = (idx / 2) % 2, g = idx / 4;
        const int row = 16 * rt + g + 8 * half;
        lohi[hh] = dplane[(int64_t)row * nb + 2 * kt + b];
      }
      word = lohi[0] | (lohi[1] << 16);
    }
    out[wi] = word;
  }
}

__global__ void dequant_kernel(int fmt, const uint8_t* __restrict__ t,
                               int rows, int cols, float* __restrict__ out) {
  const int64_t n = (int64_t)rows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    out[i] = dq_packed(fmt, t, cols, (int)(i / cols), (int)(i % cols));
  }
}

static int grid_for(int64_t n, int block) {
  int64_t g = (n + block - 1) / block;
  const int64_t cap = (int64_t)num_sms() * 32;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_tensor_bytes(int fmt, int rows, int cols) {
  if (!packed_shape_ok(fmt, rows, cols)) return 0;
  return (size_t)tensor_bytes_of(fmt, rows, cols);
}

extern "C" size_t moe_blob_bytes(int fmt_up_gate, int fmt_down, int H,
                                 int F) {
  const size_t a = moe_tensor_bytes(fmt_up_gate, F, H);
  const size_t b = moe_tensor_bytes(fmt_down, H, F);
  if (!a || !b) return 0;
  return 2 * a + b;
}

extern "C" moe_status moe_pack_tensor(int fmt, const uint8_t* natural,
                                      int rows, int cols, uint8_t* packed,
                                      void* stream) {
  MOE_TRACE();
  if (!natural || !packed) return MOE_ERR_INVALID;
  if (!fmt_valid(fmt)) return MOE_ERR_INVALID;
  if (!packed_shape_ok(fmt, rows, cols)) return MOE_ERR_SHAPE;
  if (((uintptr_t)packed & 3) || ((uintptr_t)natural & 3))
    return MOE_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t words = tensor_bytes_of(fmt, rows, cols) / 4;
  if (fmt == MOE_SB3_256)
    pack_sb3_kernel<false><<<grid_for(words, 256), 256, 0, s>>>(
        natural, rows, cols, (uint32_t*)packed);
  else if (fmt == MOE_NL3_256)
    pack_sb3_kernel<true><<<grid_for(words, 256), 256, 0, s>>>(
        natural, rows, cols, (uint32_t*)packed);
  else if (fmt == MOE_SB2_256)
    pack_sb2_kernel<<<grid_for(words, 256), 256, 0, s>>>(
        natural, rows, cols, (uint32_t*)packed);
  else
    pack_b32_kernel<<<grid_for(words, 256), 256, 0, s>>>(natural, rows, cols,
                                                         (uint32_t*)packed);
  return launch_status();
}

extern "C" moe_status moe_dequant(int fmt, const uint8_t* packed, int rows,
                                  int cols, float* out, void* stream) {
  MOE_TRACE();
  if (!packed || !out) return MOE_ERR_INVALID;
  if (!fmt_valid(fmt)) return MOE_ERR_INVALID;
  if (!packed_shape_ok(fmt, rows, cols)) return MOE_ERR_SHAPE;
  if ((uintptr_t)packed & 3) return MOE_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  dequant_kernel<<<grid_for((int64_t)rows * cols, 256), 256, 0, s>>>(
      fmt, packed, rows, cols, out);
  return launch_status();
}
