// Tile decoders of the decode path: packed SB3 / NL3 / SB2 / Q4 / NL4 tiles -> int8 A
// fragments of mma.m16n8k32 (byte-table lookups with prmt), multiplied by
// int8 B fragments of the activations (v = 256*hi + lo), exact int32 sums
// per 32-block, scales applied in fp32.
#pragma once

#include "moe_internal.cuh"

namespace moe {

// ---- tile decoders ----------------------------------------------------
// SB3 tile (16 x 256): acc[nt][0/1] += rows g / g+8 for column token
// (lane&3) + 4nt.  xfb = B fragments of the tile's first 32-block,
// [blk][bnt][32][2] words; xs[nt] = 2^-sigma_t / 8 of the lane's token.
// NL3 tile (same planes plus a shift byte per row): the byte table is the
// codebook cb3, each row's bytes raised by its block's shift bit e_j, and
// xs[nt] = 2^-sigma_t / 16.  SB2 tile (no HI plane): the 2-bit code is the
// selector, the table c = 2q - 3, xs[nt] = 2^-sigma_t / 4.
template <int FMT>
__device__ __forceinline__ void piece_sbx(const uint8_t* tp,
                                          const uint32_t* xfb, int NT,
                                          const float (&xs)[2],
                                          float (&acc)[2][2], int lane,
                                          int bnt) {
  constexpr bool NL3 = FMT == MOE_NL3_256;
  constexpr bool SB2 = FMT == MOE_SB2_256;
  constexpr uint32_t T0 = NL3 ? NL3_TAB0 : SB2 ? SB2_TAB0 : SB3_TAB0;
  constexpr uint32_t T1 = NL3 ? NL3_TAB1 : SB2 ? 0u : SB3_TAB1;
  constexpr int SC_OFF = SB2 ? 1024 : 1536, D_OFF = SB2 ? 1088 : 1600;
  const int g = lane >> 2;
  const uint4 L0 = *reinterpret_cast<const uint4*>(tp + 16 * lane);
  const uint4 L1 = *reinterpret_cast<const uint4*>(tp + 512 + 16 * lane);
  const uint4 HV =
      SB2 ? make_uint4(0u, 0u, 0u, 0u)
          : *reinterpret_cast<const uint4*>(tp + 1024 + 16 * lane);
  const uint2 SC = *reinterpret_cast<const uint2*>(tp + SC_OFF + 8 * g);
  const uint32_t DD = *reinterpret_cast<const uint32_t*>(tp + D_OFF + 4 * g);
  const uint32_t lo[8] = {L0.x, L0.y, L0.z, L0.w, L1.x, L1.y, L1.z, L1.w};
  const uint32_t hi[4] = {HV.x, HV.y, HV.z, HV.w};
  // NL3: shift bits of rows g (pi = 2g) and g+8 (pi = 2g + 1)
  const uint32_t EX =
      NL3 ? *reinterpret_cast<const uint16_t*>(tp + SB3_TILE_BYTES + 2 * g)
          : 0u;
  int32_t S[2][2] = {{0, 0}, {0, 0}};
  const int32_t zero[4] = {0, 0, 0, 0};
  // (2s+1) of the eight 32-blocks as bytes: even blocks, odd blocks
  const uint32_t mge = (SC.x & 0x0F0F0F0Fu) * 2u + 0x01010101u;
  const uint32_t mgo = ((SC.x >> 4) & 0x0F0F0F0Fu) * 2u + 0x01010101u;
  const uint32_t m8e = (SC.y & 0x0F0F0F0Fu) * 2u + 0x01010101u;
  const uint32_t m8o = ((SC.y >> 4) & 0x0F0F0F0Fu) * 2u + 0x01010101u;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t LO = lo[j], HH = hi[j >> 1];
    const uint32_t ha = (j & 1) ? HH : (HH << 2);
    const uint32_t hb = (j & 1) ? (HH >> 1) : (HH << 1);
    // selector nibbles: the 3-bit code (SB3, NL3) or the 2-bit code (SB2)
    const uint32_t sa = SB2 ? (LO & 0x33333333u)
                            : (LO & 0x33333333u) | (ha & 0x44444444u);
    const uint32_t sb = SB2 ? ((LO >> 2) & 0x33333333u)
                            : ((LO >> 2) & 0x33333333u) | (hb & 0x44444444u);
    uint32_t a[4];
    a[0] = prmt(T0, T1, sa);          // row g,   k 4c..4c+3
    a[1] = prmt(T0, T1, sa >> 16);    // row g+8
    a[2] = prmt(T0, T1, sb);          // row g,   k 16+4c..
    a[3] = prmt(T0, T1, sb >> 16);    // row g+8
    if (NL3) {
      const uint32_t inc = ((EX >> j) & 1u) * 0x01010101u;
      const uint32_t inc8 = ((EX >> (8 + j)) & 1u) * 0x01010101u;
      a[0] += inc;
      a[2] += inc;
      a[1] += inc8;
      a[3] += inc8;
    }
    // byte j/2 of the even/odd word, zero-extended (prmt selector 0x444m)
    const uint32_t bsel = 0x4440u | (uint32_t)(j >> 1);
    const int mg = (int)prmt((j & 1) ? mgo : mge, 0u, bsel);
    const int mg8 = (int)prmt((j & 1) ? m8o : m8e, 0u, bsel);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (nt < NT) {
        const uint2 b = *reinterpret_cast<const uint2*>(
            xfb + (j * bnt + nt) * 64 + 2 * lane);
        int32_t d[4];
        mma_s8(d, a, b.x, b.y, zero);
        S[nt][0] += (d[0] * 256 + d[1]) * mg;
        S[nt][1] += (d[2] * 256 + d[3]) * mg8;
      }
    }
  }
  const float2 dv = __half22float2(*reinterpret_cast<const __half2*>(&DD));
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    if (nt < NT) {
      acc[nt][0] = fmaf((float)S[nt][0], dv.x * xs[nt], acc[nt][0]);
      acc[nt][1] = fmaf((float)S[nt][1], dv.y * xs[nt], acc[nt][1]);
    }
  }
}

__device__ __forceinline__ void piece_sb3(const uint8_t* tp,
                                          const uint32_t* xfb, int NT,
                                          const float (&xs)[2],
                                          float (&acc)[2][2], int lane,
                                          int bnt = BF_NT) {
  piece_sbx<MOE_SB3_256>(tp, xfb, NT, xs, acc, lane, bnt);
}
__device__ __forceinline__ void piece_nl3(const uint8_t* tp,
                                          const uint32_t* xfb, int NT,
                                          const float (&xs)[2],
                                          float (&acc)[2][2], int lane,
                                          int bnt = BF_NT) {
  piece_sbx<MOE_NL3_256>(tp, xfb, NT, xs, acc, lane, bnt);
}
// Scale that folds the fixed denominator of a super-block format's value
// into the activation scale: 1/8 (SB3), 1/16 (NL3), 1/4 (SB2), 1 (the
// 4-bit formats).
__host__ __device__ constexpr float fmt_xfold(int fmt) {
  return fmt == MOE_SB3_256   ? 0.125f
         : fmt == MOE_NL3_256 ? 0.0625f
         : fmt == MOE_SB2_256 ? 0.25f
                              : 1.0f;
}

// Q4 / NL4 tile (16 x 64, two 32-blocks).  cs = column scales of the
// lane's columns: value for (local block bl, nt) at cs[bl*cs_stride + 4nt].
template <int FMT>
__device__ __forceinline__ void piece_b32(const uint8_t* tp,
                                          const uint32_t* bfb, int NT,
                                          const float* cs, int cs_stride,
                                          float (&acc)[2][2], int lane,
                                          int bnt = BF_NT) {
  constexpr uint32_t TA0 = FMT == MOE_NL4_B32 ? NL4_TA0 : Q4_TA0;
  constexpr uint32_t TA1 = FMT == MOE_NL4_B32 ? NL4_TA1 : Q4_TA1;
  constexpr uint32_t TB0 = FMT == MOE_NL4_B32 ? NL4_TB0 : Q4_TB0;
  constexpr uint32_t TB1 = FMT == MOE_NL4_B32 ? NL4_TB1 : Q4_TB1;
  const int g = lane >> 2;
  const uint4 W = *reinterpret_cast<const uint4*>(tp + 16 * lane);
  const uint2 DV = *reinterpret_cast<const uint2*>(tp + 512 + 8 * g);
  const float2 dg = __half22float2(*reinterpret_cast<const __half2*>(&DV.x));
  const float2 dg8 = __half22float2(*reinterpret_cast<const __half2*>(&DV.y));
  const uint32_t w[4] = {W.x, W.y, W.z, W.w};
  const int32_t zero[4] = {0, 0, 0, 0};
#pragma unroll
  for (int bl = 0; bl < 2; ++bl) {
    const uint32_t w0 = w[2 * bl], w1 = w[2 * bl + 1];
    const uint32_t x0 = w0 ^ 0x88888888u, x1 = w1 ^ 0x88888888u;
    uint32_t a1[4], a2[4];
    a1[0] = prmt(TA0, TA1, w0);
    a1[1] = prmt(TA0, TA1, w0 >> 16);
    a1[2] = prmt(TA0, TA1, w1);
    a1[3] = prmt(TA0, TA1, w1 >> 16);
    a2[0] = prmt(TB0, TB1, x0);
    a2[1] = prmt(TB0, TB1, x0 >> 16);
    a2[2] = prmt(TB0, TB1, x1);
    a2[3] = prmt(TB0, TB1, x1 >> 16);
    const float d0 = bl ? dg.y : dg.x, d8 = bl ? dg8.y : dg8.x;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (nt < NT) {
        const uint2 b = *reinterpret_cast<const uint2*>(
            bfb + (bl * bnt + nt) * 64 + 2 * lane);
        // the two table halves as independent products (exact int32 sum)
        int32_t d[4], e[4];
        mma_s8(d, a1, b.x, b.y, zero);
        mma_s8(e, a2, b.x, b.y, zero);
#pragma unroll
        for (int q = 0; q < 4; ++q) d[q] += e[q];
        const float c = cs[bl * cs_stride + 4 * nt];
        acc[nt][0] = fmaf((float)(d[0] * 256 + d[1]), d0 * c, acc[nt][0]);
        acc[nt][1] = fmaf((float)(d[2] * 256 + d[3]), d8 * c, acc[nt][1]);
      }
    }
  }
}

// Columns of x that share one activation scale in the decode kernels: a
// large value in one channel coarsens only the other values of its block.
constexpr int XB_COLS = 256;

// max |v| of 8 bf16 values packed in a 16-byte word.
__device__ __forceinline__ float absmax8_bf16(const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    m = fmaxf(m, fabsf(__uint_as_float(w[q] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w[q] & 0xFFFF0000u)));
  }
  return m;
}

// 2^sigma with sigma chosen so that max|v| * 2^sigma < 2^14.
__device__ __forceinline__ int pow2_sigma(float m) {
  if (!(m > 0.f) || !isfinite(m)) return 0;
  const int e = (int)((__float_as_uint(m) >> 23) & 255u) - 126;  // m < 2^e
  int s = 14 - e;
  if (s > 100) s = 100;
  if (s < -100) s = -100;
  return s;
}
__device__ __forceinline__ float exp2i(int s) {
  return __uint_as_float((uint32_t)(127 + s) << 23);
}


}  // namespace moe
