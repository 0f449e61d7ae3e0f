// moe_dequant_path: the dequantised weights as the hot-path decoders
// produce them, so that those decoders -- not only the generic dequant of
// moe_dequant -- can be checked bit for bit against the closed forms of the
// formats (Avalon GGUF model card, "Files": the expert quant types).
//
//  decode  : the int8 tensor-core tile decoders of the decode kernels
//            (piece_sb3 / piece_b32: byte-table codes, sub-scale folds,
//            fp32 scale products), fed one-hot activations.  With x = e_i
//            the exact int32 block sum is the integer code value of
//            column i (times (2s+1) for SB3), and the fp32 scale product
//            gives w[row][i] -- exact, since every weight of these formats
//            is exact in fp32.
//  prefill : the fp16 A-operand tiles that the dequant warps of the
//            grouped GEMM write to shared memory (prefill.cu), un-swizzled.
#include "decode_pieces.cuh"
#include "trace.h"

namespace moe {

bool pf_export_supported(int fmt, int rows, int cols);
moe_status launch_pf_dequant_export(int fmt, const uint8_t* t, int rows,
                                    int cols, uint16_t* out, cudaStream_t s);

namespace {

constexpr int XW = 4;   // warps per block, one 16-row tile each

// One warp per packed tile (16 rows x TC columns).  Call c of the warp
// feeds eight one-hot activation columns (token tok carries e_i for tile
// column i = 8c + tok) and stores the eight result columns of the tile's
// 16 rows.
template <int FMT>
__global__ void __launch_bounds__(XW * 32)
    dq_decode_export_kernel(const uint8_t* __restrict__ t, int rows,
                            int cols, float* __restrict__ out) {
  constexpr bool SB3 =
      FMT == MOE_SB3_256 || FMT == MOE_NL3_256 || FMT == MOE_SB2_256;
  constexpr int TC = SB3 ? SB3_TILE_COLS : B32_TILE_COLS;
  constexpr int TB = FMT == MOE_SB3_256   ? SB3_TILE_BYTES
                     : FMT == MOE_NL3_256 ? NL3_TILE_BYTES
                     : FMT == MOE_SB2_256 ? SB2_TILE_BYTES
                                          : B32_TILE_BYTES;
  constexpr int NBLK = TC / 32;                 // 32-blocks per tile
  constexpr int FW = NBLK * BF_NT * 64;         // B fragment words
  __shared__ __align__(16) uint32_t frag_all[XW][FW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* frag = frag_all[warp];
  const int ntc = cols / TC;
  const int64_t tile = (int64_t)blockIdx.x * XW + warp;
  if (tile >= (int64_t)(rows / TILE_ROWS) * ntc) return;   // whole warp
  const int64_t rt = tile / ntc;
  const int kt = (int)(tile % ntc);
  const uint8_t* tp = t + tile * TB;   // row-tile major, column-tile minor
  const int g = lane >> 2, c = lane & 3;
  for (int cg = 0; cg < TC / 8; ++cg) {
    // B fragment entry i = (j * BF_NT + nt) * 32 + L: lane L = 4n + cq
    // holds k = 4cq..4cq+3 (.x) and 16+4cq..16+4cq+3 (.y) of column n,
    // the high (n even) or low (n odd) int8 half of token 4nt + n/2
    for (int i = lane; i < FW / 2; i += 32) {
      const int L = i & 31, nt = (i >> 5) % BF_NT, j = i / (32 * BF_NT);
      const int n = L >> 2, cq = L & 3;
      const int col = 8 * cg + 4 * nt + (n >> 1);
      uint2 wv = make_uint2(0u, 0u);
      if ((n & 1) && col / 32 == j) {   // v = 1: low half 1, high half 0
        const int kk = col % 32, kb = kk & 15;
        if ((kb >> 2) == cq) {
          const uint32_t bit = 1u << (8 * (kb & 3));
          if (kk >> 4) wv.y = bit; else wv.x = bit;
        }
      }
      reinterpret_cast<uint2*>(frag)[i] = wv;
    }
    __syncwarp();
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    if constexpr (SB3) {
      // 2^-sigma / 8 (SB3), / 16 (NL3) or / 4 (SB2), sigma = 0
      const float xs[2] = {fmt_xfold(FMT), fmt_xfold(FMT)};
      piece_sbx<FMT>(tp, frag, BF_NT, xs, acc, lane, BF_NT);
    } else {
      const float cs[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
      piece_b32<FMT>(tp, frag, BF_NT, cs, 0, acc, lane, BF_NT);
    }
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < BF_NT; ++nt) {
      const int64_t col = (int64_t)kt * TC + 8 * cg + c + 4 * nt;
      out[(rt * TILE_ROWS + g) * cols + col] = acc[nt][0];
      out[(rt * TILE_ROWS + g + 8) * cols + col] = acc[nt][1];
    }
  }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dequant_path(int fmt, int path,
                                       const uint8_t* packed, int rows,
                                       int cols, void* out, void* stream) {
  MOE_TRACE();
  if (!packed || !out) return MOE_ERR_INVALID;
  if (!fmt_valid(fmt)) return MOE_ERR_INVALID;
  if (path != MOE_DQ_DECODE && path != MOE_DQ_PREFILL) return MOE_ERR_INVALID;
  if (!packed_shape_ok(fmt, rows, cols)) return MOE_ERR_SHAPE;
  if (((uintptr_t)packed & 15) || ((uintptr_t)out & 15))
    return MOE_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  if (path == MOE_DQ_PREFILL) {
    if (!pf_export_supported(fmt, rows, cols)) return MOE_ERR_SHAPE;
    return launch_pf_dequant_export(fmt, packed, rows, cols,
                                    static_cast<uint16_t*>(out), s);
  }
  const int tc = tile_cols(fmt);
  const int64_t tiles = (int64_t)(rows / TILE_ROWS) * (cols / tc);
  const unsigned grid = (unsigned)((tiles + XW - 1) / XW);
  float* o = static_cast<float*>(out);
  switch (fmt) {
    case MOE_SB3_256:
      dq_decode_export_kernel<MOE_SB3_256><<<grid, XW * 32, 0, s>>>(
          packed, rows, cols, o);
      break;
    case MOE_NL4_B32:
      dq_decode_export_kernel<MOE_NL4_B32><<<grid, XW * 32, 0, s>>>(
          packed, rows, cols, o);
      break;
    case MOE_NL3_256:
      dq_decode_export_kernel<MOE_NL3_256><<<grid, XW * 32, 0, s>>>(
          packed, rows, cols, o);
      break;
    case MOE_SB2_256:
      dq_decode_export_kernel<MOE_SB2_256><<<grid, XW * 32, 0, s>>>(
          packed, rows, cols, o);
      break;
    default:
      dq_decode_export_kernel<MOE_Q4_B32><<<grid, XW * 32, 0, s>>>(
          packed, rows, cols, o);
  }
  return launch_status();
}
