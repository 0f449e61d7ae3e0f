// Prefill expert FFN (many tokens per expert) on the 5th-generation tensor
// cores: grouped GEMMs over the per-expert token lists of the MoE layer of
// the "Avalon" README (512 experts, 10 active), with the expert tensors in
// the quant types of the Avalon GGUF model card ("Files").
//
// One persistent CTA per SM walks a list of units.  A unit is 128 weight
// rows of one expert times up to 256 of that expert's token rows:
//   up   : [u | g] = W_{up,gate}[128 rows x H] . x[tokens]^T, then
//          h = silu(g) * u  -> fp16, grouped row order
//   down : y = W_down[128 rows x F] . h[tokens]^T -> fp32 rows of y_pairs
// Warp roles inside the CTA:
//   warps 0..E-1  epilogue: TMEM -> registers -> global (warp w reads TMEM
//                 lane quadrant w % 4; with E = 8 (up/gate, whose single
//                 accumulator buffer makes the epilogue stall the MMAs)
//                 warp w / 4 takes every other 32 columns)
//   warp  E     TMEM owner; lane 0 issues tcgen05.mma and the commits
//   warp  E+1   B operand: TMA copies of 16-row boxes of activations in
//               grouped row order (up: x gathered to fp16 by a pre-pass;
//               down: h as the up/gate epilogue wrote it)
//   warps E+2.. A operand: quantised tiles -> fp16 in shared memory (8)
// Operands are K-major fp16 with the 128-byte swizzle, accumulators fp32 in
// tensor memory.  The A tiles hold the round-to-nearest-even fp16 value of
// each dequantised weight (d * (2s+1) * c / 8 or d * cb[q], formed with
// exact fp16 products and one rounding).
#include "moe_internal.cuh"
#include "tc_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace moe {
namespace {

constexpr int PF_BM = 128;   // weight rows per unit (MMA M)
constexpr int PF_BK = 64;    // K per pipeline stage (one swizzle row)
constexpr int PF_BN = 256;   // token rows per unit at most (MMA N)
constexpr int PF_NDQ = 8;    // dequant warps
constexpr int PF_A_BYTES = PF_BM * PF_BK * 2;         // 16 KB
constexpr int PF_B_BYTES = PF_BN * PF_BK * 2;         // 32 KB
constexpr int PF_TMEM_COLS = 512;
// A operand formats of the GEMM kernels: the 4-bit 32-weight blocks (Q4,
// NL4), the 3-bit super-blocks SB3 and NL3, and the 2-bit super-block SB2.
constexpr int AF_B32 = 0, AF_SB3 = 1, AF_NL3 = 2, AF_SB2 = 3;
__host__ __device__ constexpr int af_of(int fmt) {
  return fmt == MOE_SB3_256   ? AF_SB3
         : fmt == MOE_NL3_256 ? AF_NL3
         : fmt == MOE_SB2_256 ? AF_SB2
                              : AF_B32;
}
__host__ __device__ constexpr int af_tile_bytes(int af) {
  return af == AF_SB3   ? SB3_TILE_BYTES
         : af == AF_NL3 ? NL3_TILE_BYTES
         : af == AF_SB2 ? SB2_TILE_BYTES
                        : B32_TILE_BYTES;
}

template <bool UP>
struct PfCfg {
  static constexpr int EPI = UP ? 8 : 4;           // epilogue warps
  static constexpr int WMMA = EPI, WLOAD = EPI + 1, WDQ0 = EPI + 2;
  static constexpr int THREADS = (WDQ0 + PF_NDQ) * 32;
  static constexpr int NA = UP ? 2 : 1;            // A tensors per unit
  static constexpr int STAGES = UP ? 3 : 4;
  static constexpr int STAGE_BYTES = NA * PF_A_BYTES + PF_B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int META_OFF = BAR_OFF + 256;   // epilogue row metadata
  static constexpr int META_BYTES = EPI * PF_BN * 4;
  static constexpr int SMEM = META_OFF + META_BYTES + 1024;   // + alignment
};

// B operand tensor maps: the same fp16 [P][K] tensor with box heights
// 256, 128, 64, 32, 16 rows (a tile of n rows takes at most one of each).
constexpr int PF_NMAPS = 5;
struct PfMaps {
  CUtensorMap m[PF_NMAPS];
};

struct PfParams {
  const uint8_t* pool;
  int64_t blob_stride;
  const int32_t* blob_index;   // [E] or null (blob e)
  int64_t off_a0, off_a1;      // A tensors inside a blob (bytes)
  int K;                       // contraction length
  int rows;                    // rows of the A tensors
  int k;                       // pairs per token
  const int32_t* pair_ids;     // grouped order
  const int4* tiles;           // {expert, first grouped row, rows, 0}
  const int32_t* n_tiles;
  const float* xscale;         // up: 2^sigma per grouped row
  __half* h16;                 // up output [P][rows], grouped rows
  float* y;                    // down output [P][rows], pair order
  uint32_t tab[4];             // B32 decode tables (NL4 or Q4)
  int32_t* err;
};

__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a),
                      *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hsub2u(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a),
                      *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t half_bcast(uint16_t h) {
  return (uint32_t)h | ((uint32_t)h << 16);
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a,
                                             uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a),
               "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ uint32_t ldg_u32(const uint8_t* p) {
  return __ldg(reinterpret_cast<const uint32_t*>(p));
}
__device__ __forceinline__ uint2 ldg_u64(const uint8_t* p) {
  return __ldg(reinterpret_cast<const uint2*>(p));
}
__device__ __forceinline__ uint4 ldg_u128(const uint8_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Byte offset of 16-byte chunk `chunk` of row `r` in a swizzled K-major
// operand tile (rows of 128 bytes).
__device__ __forceinline__ uint32_t sw128(int r, int chunk) {
  return (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4));
}

// ------------------------------------------------------------- SB3 ----
// fp16 high bytes of c = 2q - 7 for q = 0..3 and 4..7 (the low bytes are 0).
constexpr uint32_t SB3_H16_LO = 0xBCC2C5C7u;   // -1,-3,-5,-7 (bytes 3..0)
constexpr uint32_t SB3_H16_HI = 0x4745423Cu;   //  7, 5, 3, 1
// SB2: fp16 high bytes of c = 2q - 3 for q = 0..3 (the low bytes are 0)
constexpr uint32_t SB2_H16 = 0x423CBCC2u;      //  3, 1,-1,-3 (bytes 3..0)

// One thread's share of a 16-row SB3 tile (one super-block per row) for
// one of the two dequant groups: group gamma takes k-steps q = gamma and
// gamma + 2 of the super-block's four 64-column k-steps.  Holds, for lanes
// L0 = 4g + 2p and L0 + 1, the LO words 2*gamma, 2*gamma+1 of both
// segments and the HI words gamma, gamma+2, plus the sub-scale words and
// fp16 d of rows g and g+8.
struct Sb3Half {
  uint2 lo[2][2];   // [segment][lane]
  uint2 hi[2];      // [lane]: HI[gamma], HI[gamma+2]
  uint2 sc;         // sub-scale words of rows g, g+8
  uint32_t d;       // fp16 d of rows g (low), g+8 (high)
  uint32_t ex;      // NL3: shift bytes of rows g (bits 0-7), g+8 (8-15)
};

template <bool SB2>
__device__ __forceinline__ void sbq_load(const uint8_t* tp, int g, int p,
                                         int gamma, Sb3Half& q) {
  const int L0 = 4 * g + 2 * p;
#pragma unroll
  for (int l = 0; l < 2; ++l) {
    const uint8_t* lw = tp + 16 * (L0 + l);
    q.lo[0][l] = ldg_u64(lw + 8 * gamma);
    q.lo[1][l] = ldg_u64(lw + 512 + 8 * gamma);
    q.hi[l] = SB2 ? make_uint2(0u, 0u)
                  : make_uint2(ldg_u32(lw + 1024 + 4 * gamma),
                               ldg_u32(lw + 1024 + 8 + 4 * gamma));
  }
  q.sc = ldg_u64(tp + (SB2 ? 1024 : 1536) + 8 * g);
  q.d = ldg_u32(tp + (SB2 ? 1088 : 1600) + 4 * g);
}
__device__ __forceinline__ void sb3_load(const uint8_t* tp, int g, int p,
                                         int gamma, Sb3Half& q) {
  sbq_load<false>(tp, g, p, gamma, q);
}
__device__ __forceinline__ void nl3_load(const uint8_t* tp, int g, int p,
                                         int gamma, Sb3Half& q) {
  sb3_load(tp, g, p, gamma, q);
  q.ex = __ldg(reinterpret_cast<const uint16_t*>(tp + SB3_TILE_BYTES + 2 * g));
}

// 8 codes of one lane word (nibble n = 4*rowhalf + w) -> fp16 c values as
// two half2 words per row: out[0..1] row g (w = 0,1 | 2,3), out[2..3] row
// g+8.  Q holds one 3-bit code per nibble (bit 3 clear).
template <bool SB2>
__device__ __forceinline__ void sbq_codes_to_h16(uint32_t Q,
                                                 uint32_t (&o)[4]) {
  // SB3: table bytes 0..7; SB2: bytes 0..3, and byte 4 (a zero) for C
  constexpr uint32_t TL = SB2 ? SB2_H16 : SB3_H16_LO;
  constexpr uint32_t TH = SB2 ? 0u : SB3_H16_HI;
  const uint32_t S = Q << 4;
  // selector nibbles [C, q(n), C, q(n+1)]: C = 0xC picks a zero byte (the
  // sign, replicated, of a byte whose top bit is clear)
  const uint32_t X0 = (prmt(Q, S, 0x1504u) & 0xF0F0F0F0u) | 0x0C0C0C0Cu;
  const uint32_t X1 = (prmt(Q, S, 0x3726u) & 0xF0F0F0F0u) | 0x0C0C0C0Cu;
  o[0] = prmt(TL, TH, X0);
  o[1] = prmt(TL, TH, X0 >> 16);
  o[2] = prmt(TL, TH, X1);
  o[3] = prmt(TL, TH, X1 >> 16);
}

// The group's k-step qh (0/1) of the super-block, i.e. k-step
// q = gamma + 2*qh: sub-blocks j0 = 2q and 2q+1 -> fp16 rows g and g+8 of
// the swizzled A tile.
template <bool SB2>
__device__ __forceinline__ void sbq_store(const Sb3Half& sb, int g, int p,
                                          int gamma, int qh, int row0,
                                          uint32_t a_smem) {
  constexpr float FOLD = SB2 ? 0.25f : 0.125f;   // (2s+1)/4 or /8
  const int q = gamma + 2 * qh;
  const int j0 = 2 * q;
  const uint32_t dg = half_bcast((uint16_t)(sb.d & 0xFFFFu));
  const uint32_t dg8 = half_bcast((uint16_t)(sb.d >> 16));
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    const int j = j0 + jj;
    const int sg = (sb.sc.x >> (4 * j)) & 15, sg8 = (sb.sc.y >> (4 * j)) & 15;
    // (2s+1)/8 (SB3) or /4 (SB2), exact in fp16
    const __half tg = __float2half_rn((float)(2 * sg + 1) * FOLD);
    const __half tg8 = __float2half_rn((float)(2 * sg8 + 1) * FOLD);
    const uint32_t t2g = half_bcast(__half_as_ushort(tg));
    const uint32_t t2g8 = half_bcast(__half_as_ushort(tg8));
    uint32_t w[2][2][4];   // [lane][h][words]
#pragma unroll
    for (int l = 0; l < 2; ++l) {
      const uint32_t lo = jj ? sb.lo[qh][l].y : sb.lo[qh][l].x;
      const uint32_t hi = (qh ? sb.hi[l].y : sb.hi[l].x) >> (2 * jj);
      const uint32_t Q0 = SB2 ? (lo & 0x33333333u)
                              : (lo & 0x33333333u) | ((hi << 2) & 0x44444444u);
      const uint32_t Q1 = SB2 ? ((lo >> 2) & 0x33333333u)
                              : ((lo >> 2) & 0x33333333u) |
                                    ((hi << 1) & 0x44444444u);
      sbq_codes_to_h16<SB2>(Q0, w[l][0]);
      sbq_codes_to_h16<SB2>(Q1, w[l][1]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        w[l][h][0] = hmul2u(hmul2u(w[l][h][0], t2g), dg);
        w[l][h][1] = hmul2u(hmul2u(w[l][h][1], t2g), dg);
        w[l][h][2] = hmul2u(hmul2u(w[l][h][2], t2g8), dg8);
        w[l][h][3] = hmul2u(hmul2u(w[l][h][3], t2g8), dg8);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int chunk = 4 * jj + 2 * h + p;
      st_shared_v4(a_smem + sw128(row0 + g, chunk), w[0][h][0], w[0][h][1],
                   w[1][h][0], w[1][h][1]);
      st_shared_v4(a_smem + sw128(row0 + g + 8, chunk), w[0][h][2],
                   w[0][h][3], w[1][h][2], w[1][h][3]);
    }
  }
}

__device__ __forceinline__ void sb3_store(const Sb3Half& sb, int g, int p,
                                          int gamma, int qh, int row0,
                                          uint32_t a_smem) {
  sbq_store<false>(sb, g, p, gamma, qh, row0, a_smem);
}

// ------------------------------------------------------------- NL3 ----
// cb3[q] + 16 as unsigned bytes (1..30), q = 0..3 and 4..7
constexpr uint32_t NL3_U0 = 0x0E0A0601u;
constexpr uint32_t NL3_U1 = 0x1E191511u;
constexpr uint32_t H16_1040 = 0x64106410u;   // fp16 1040 = 1024 + 16, twice

// 8 codes of one lane word (as sb3_codes_to_h16) -> fp16 cb3[q] + e, with
// inc / inc8 the byte-replicated shift bits of rows g and g+8: the bytes
// u = cb3[q] + 16 + e go under a 0x64 high byte (fp16 1024 + u, exact),
// minus fp16 1040.
__device__ __forceinline__ void nl3_codes_to_h16(uint32_t Q, uint32_t inc,
                                                 uint32_t inc8,
                                                 uint32_t (&o)[4]) {
  const uint32_t P0 = prmt(NL3_U0, NL3_U1, Q) + inc;          // row g
  const uint32_t P1 = prmt(NL3_U0, NL3_U1, Q >> 16) + inc8;   // row g+8
  o[0] = hsub2u(prmt(P0, 0x64646464u, 0x5140u), H16_1040);
  o[1] = hsub2u(prmt(P0, 0x64646464u, 0x7362u), H16_1040);
  o[2] = hsub2u(prmt(P1, 0x64646464u, 0x5140u), H16_1040);
  o[3] = hsub2u(prmt(P1, 0x64646464u, 0x7362u), H16_1040);
}

// The NL3 counterpart of sb3_store: value (cb3[q] + e_j) * (2s+1)/16 (exact
// in fp16) times d, one rounding.
__device__ __forceinline__ void nl3_store(const Sb3Half& sb, int g, int p,
                                          int gamma, int qh, int row0,
                                          uint32_t a_smem) {
  const int q = gamma + 2 * qh;
  const int j0 = 2 * q;
  const uint32_t dg = half_bcast((uint16_t)(sb.d & 0xFFFFu));
  const uint32_t dg8 = half_bcast((uint16_t)(sb.d >> 16));
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    const int j = j0 + jj;
    const int sg = (sb.sc.x >> (4 * j)) & 15, sg8 = (sb.sc.y >> (4 * j)) & 15;
    const __half tg = __float2half_rn((float)(2 * sg + 1) * 0.0625f);
    const __half tg8 = __float2half_rn((float)(2 * sg8 + 1) * 0.0625f);
    const uint32_t t2g = half_bcast(__half_as_ushort(tg));
    const uint32_t t2g8 = half_bcast(__half_as_ushort(tg8));
    const uint32_t inc = ((sb.ex >> j) & 1u) * 0x01010101u;
    const uint32_t inc8 = ((sb.ex >> (8 + j)) & 1u) * 0x01010101u;
    uint32_t w[2][2][4];   // [lane][h][words]
#pragma unroll
    for (int l = 0; l < 2; ++l) {
      const uint32_t lo = jj ? sb.lo[qh][l].y : sb.lo[qh][l].x;
      const uint32_t hi = (qh ? sb.hi[l].y : sb.hi[l].x) >> (2 * jj);
      const uint32_t Q0 = (lo & 0x33333333u) | ((hi << 2) & 0x44444444u);
      const uint32_t Q1 = ((lo >> 2) & 0x33333333u) | ((hi << 1) & 0x44444444u);
      nl3_codes_to_h16(Q0, inc, inc8, w[l][0]);
      nl3_codes_to_h16(Q1, inc, inc8, w[l][1]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        w[l][h][0] = hmul2u(hmul2u(w[l][h][0], t2g), dg);
        w[l][h][1] = hmul2u(hmul2u(w[l][h][1], t2g), dg);
        w[l][h][2] = hmul2u(hmul2u(w[l][h][2], t2g8), dg8);
        w[l][h][3] = hmul2u(hmul2u(w[l][h][3], t2g8), dg8);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int chunk = 4 * jj + 2 * h + p;
      st_shared_v4(a_smem + sw128(row0 + g, chunk), w[0][h][0], w[0][h][1],
                   w[1][h][0], w[1][h][1]);
      st_shared_v4(a_smem + sw128(row0 + g + 8, chunk), w[0][h][2],
                   w[0][h][3], w[1][h][2], w[1][h][3]);
    }
  }
}

// Super-block format of a GEMM's A operand: SB3, NL3 or SB2 load / store.
template <int AF>
__device__ __forceinline__ void sbx_load(const uint8_t* tp, int g, int p,
                                         int gamma, Sb3Half& q) {
  if constexpr (AF == AF_NL3) nl3_load(tp, g, p, gamma, q);
  else if constexpr (AF == AF_SB2) sbq_load<true>(tp, g, p, gamma, q);
  else sb3_load(tp, g, p, gamma, q);
}
template <int AF>
__device__ __forceinline__ void sbx_store(const Sb3Half& sb, int g, int p,
                                          int gamma, int qh, int row0,
                                          uint32_t a_smem) {
  if constexpr (AF == AF_NL3) nl3_store(sb, g, p, gamma, qh, row0, a_smem);
  else if constexpr (AF == AF_SB2)
    sbq_store<true>(sb, g, p, gamma, qh, row0, a_smem);
  else sb3_store(sb, g, p, gamma, qh, row0, a_smem);
}

// ------------------------------------------------------------- B32 ----
struct B32Q {
  uint4 w0, w1;   // W[0..3] of lanes L0, L0+1
  uint2 d;        // fp16 d: (row g, b0), (g, b1), (g+8, b0), (g+8, b1)
};

__device__ __forceinline__ B32Q b32_load(const uint8_t* tp, int g, int p) {
  const int L0 = 4 * g + 2 * p;
  B32Q q;
  q.w0 = ldg_u128(tp + 16 * L0);
  q.w1 = ldg_u128(tp + 16 * L0 + 16);
  q.d = ldg_u64(tp + 512 + 8 * g);
  return q;
}

// 4 codes (selector nibbles in the low 16 bits of `sel`) -> two half2
// words of d * value(q).  A1 + A2 = value (the byte-table split of the
// packed layout); both halves are widened to 16 bits and offset into the
// fp16 range [1024, 2048) so one subtraction gives the exact integer.
struct B32Tab {
  uint32_t a0, a1, b0, b1;
};

__device__ __forceinline__ void b32_codes(uint32_t sel, const B32Tab tab,
                                          uint32_t d2, uint32_t& o01,
                                          uint32_t& o23) {
  const uint32_t A1 = prmt(tab.a0, tab.a1, sel);
  const uint32_t A2 = prmt(tab.b0, tab.b1, sel ^ 0x8888u);
  // u8(A1) + A2 = 256 + value, no carry across the 16-bit halves
  const uint32_t v01 = prmt(A1, A2, 0xC1C0u) + prmt(A2, A2, 0x8180u) +
                       0x64006400u;
  const uint32_t v23 = prmt(A1, A2, 0xC3C2u) + prmt(A2, A2, 0x8382u) +
                       0x64006400u;
  const uint32_t k1280 = 0x65006500u;   // fp16 1280
  o01 = hmul2u(hsub2u(v01, k1280), d2);
  o23 = hmul2u(hsub2u(v23, k1280), d2);
}

__device__ __forceinline__ void b32_store(const B32Q& q, int g, int p,
                                          int rh, int row0,
                                          const B32Tab tab,
                                          uint32_t a_smem) {
  const uint32_t dw = rh ? q.d.y : q.d.x;
  const uint32_t d2[2] = {half_bcast((uint16_t)(dw & 0xFFFFu)),
                          half_bcast((uint16_t)(dw >> 16))};
  const uint32_t W0[4] = {q.w0.x, q.w0.y, q.w0.z, q.w0.w};
  const uint32_t W1[4] = {q.w1.x, q.w1.y, q.w1.z, q.w1.w};
  const int r = row0 + g + 8 * rh;
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t a0, a1, c0, c1;
      b32_codes(W0[2 * b + h] >> (16 * rh), tab, d2[b], a0, a1);
      b32_codes(W1[2 * b + h] >> (16 * rh), tab, d2[b], c0, c1);
      st_shared_v4(a_smem + sw128(r, 4 * b + 2 * h + p), a0, a1, c0, c1);
    }
}

// ------------------------------------------------------ tile export --
// The A operand tiles exactly as the dequant warps of pf_gemm_kernel write
// them (same loads, same stores, same thread mapping), for one 128-row
// block and one group of k-steps -- SB3: the four 64-column k-steps of a
// super-block (group gamma writes k-steps gamma and gamma + 2); Q4/NL4: two
// k-steps, one per group -- then un-swizzled to fp16 [rows][cols].  Used
// only by moe_dequant_path, to check these decoders bit for bit.
template <int AF>
__global__ void __launch_bounds__(256)
    pf_dequant_export_kernel(const uint8_t* __restrict__ t, int cols,
                             uint4 tab4, uint16_t* __restrict__ out) {
  constexpr bool SB3 = AF != AF_B32;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint8_t* smem = smem_raw + (sbase - raw);
  constexpr int NKS = SB3 ? 4 : 2;   // k-steps of one block
  const int gamma = threadIdx.x >> 7, tt = threadIdx.x & 127;
  const int tg = tt & 7, tp_ = (tt >> 3) & 1, tti = tt >> 4;
  const int m = blockIdx.x, kg = blockIdx.y;
  const int tcols = SB3 ? SB3_TILE_COLS : B32_TILE_COLS;
  const int tbytes = af_tile_bytes(AF);
  const int64_t trow_stride = (int64_t)(cols / tcols) * tbytes;
  const uint8_t* ptp = t + (int64_t)(m * (PF_BM / 16) + tti) * trow_stride;
  const int nks_total = cols / PF_BK;
  if constexpr (SB3) {
    Sb3Half q;
    sbx_load<AF>(ptp + (int64_t)kg * tbytes, tg, tp_, gamma, q);
#pragma unroll
    for (int qh = 0; qh < 2; ++qh)
      sbx_store<AF>(q, tg, tp_, gamma, qh, 16 * tti,
                    sbase + (uint32_t)((gamma + 2 * qh) * PF_A_BYTES));
  } else {
    const B32Tab tab = {tab4.x, tab4.y, tab4.z, tab4.w};
    const int ks = NKS * kg + gamma;
    if (ks < nks_total) {
      const B32Q q = b32_load(ptp + (int64_t)ks * B32_TILE_BYTES, tg, tp_);
#pragma unroll
      for (int rh = 0; rh < 2; ++rh)
        b32_store(q, tg, tp_, rh, 16 * tti, tab,
                  sbase + (uint32_t)(gamma * PF_A_BYTES));
    }
  }
  __syncthreads();
  // 16-byte chunk ch of row r of k-step q holds columns 8ch .. 8ch+7
  for (int i = threadIdx.x; i < NKS * PF_BM * 8; i += blockDim.x) {
    const int q = i / (PF_BM * 8), r = (i / 8) % PF_BM, ch = i % 8;
    const int ksg = kg * NKS + q;
    if (ksg >= nks_total) continue;
    const uint4 v = *reinterpret_cast<const uint4*>(smem + q * PF_A_BYTES +
                                                    sw128(r, ch));
    *reinterpret_cast<uint4*>(out + (int64_t)(PF_BM * m + r) * cols +
                              ksg * PF_BK + 8 * ch) = v;
  }
}

// --------------------------------------------------------------- kernel --
// maps: up: x_g [P][H], down: h16 [P][F], both fp16 in grouped row
// order, boxes of 64 columns, 128-byte swizzle.
template <bool UP, int AF>
__global__ void __launch_bounds__(PfCfg<UP>::THREADS, 1)
    pf_gemm_kernel(const PfParams p, const __grid_constant__ PfMaps maps) {
  constexpr bool SB3 = AF != AF_B32;   // a super-block format (SB3, NL3, SB2)
  using C = PfCfg<UP>;
  constexpr int NA = C::NA, S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* full_a = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* full_b = full_a + S;
  uint64_t* empty = full_b + S;
  uint64_t* acc_full = empty + S;      // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_a[s], PF_NDQ / 2);   // the warps of one dequant group
      mbar_init(&full_b[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::EPI);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == C::WMMA) {
    tc::tmem_alloc(tmem_slot, PF_TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const int MT = p.rows / PF_BM;   // row blocks per expert tensor
  const int nk = p.K / PF_BK;
  const int n_units = *p.n_tiles * MT;
  int32_t* err = p.err;

  if (warp == C::WMMA) {
    // ------------------------------------------------ MMA issuer ------
    if (lane == 0) {
      uint32_t kstep = 0;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++it) {
        const int4 tile = p.tiles[u / MT];
        const int nmma = (tile.z + 15) & ~15;
        const int ab = UP ? 0 : (it & 1);
        const int use_ab = UP ? it : (it >> 1);   // earlier uses of buffer ab
        if (use_ab > 0 && !mbar_wait(&acc_empty[ab], (use_ab - 1) & 1, err)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_f16_f32(PF_BM, nmma);
        const uint32_t d0 = tmem + (uint32_t)(ab * 256);
        for (int ks = 0; ks < nk; ++ks, ++kstep) {
          const int s = (int)(kstep % S);
          const uint32_t par = (kstep / S) & 1;
          if (!mbar_wait(&full_a[s], par, err) ||
              !mbar_wait(&full_b[s], par, err)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t st = sbase + (uint32_t)(s * C::STAGE_BYTES);
          const uint32_t bst = st + NA * PF_A_BYTES;
#pragma unroll
          for (int a = 0; a < NA; ++a)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc::mma_f16(d0 + (uint32_t)(a * 256),
                          tc::sdesc_sw128(st + a * PF_A_BYTES + 32 * kk),
                          tc::sdesc_sw128(bst + 32 * kk), idesc,
                          (ks | kk) != 0);
          tc::commit(&empty[s]);
        }
        if (!ok) break;
        tc::commit(&acc_full[ab]);
      }
      // all issued MMAs complete before the allocation is released
      tc::commit(drain);
      mbar_wait(drain, 0, err);
    }
  } else if (warp == C::WLOAD) {
    // ------------------------------------------- B operand loader -----
    // Lane 0 issues the TMA copies of every k-step: the unit's grouped
    // rows in boxes of 256/128/64/32/16 rows; rows past the tile (up to the
    // 16-row MMA granularity) belong to the next expert or read zeros past
    // the end.
    if (lane == 0) {
      uint32_t kstep = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
        const int4 tile = p.tiles[u / MT];
        const int nmma = (tile.z + 15) & ~15;
        const uint32_t bytes = (uint32_t)nmma * (PF_BK * 2);
        for (int ks = 0; ks < nk; ++ks, ++kstep) {
          const int s = (int)(kstep % S);
          const uint32_t use = kstep / S;
          if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, err)) {
            ok = false;
            break;
          }
          const uint32_t bst =
              sbase + (uint32_t)(s * C::STAGE_BYTES + NA * PF_A_BYTES);
          mbar_arrive_expect_tx(&full_b[s], bytes);
          int n = 0;
#pragma unroll
          for (int b = 0; b < PF_NMAPS; ++b) {
            const int rows = 256 >> b;
            if (nmma - n >= rows) {
              tc::tma_load_2d(bst + n * 128, &maps.m[b], ks * PF_BK,
                              tile.y + n, &full_b[s]);
              n += rows;
            }
          }
        }
      }
    }
  } else if (warp >= C::WDQ0) {
    // ------------------------------------------ A operand dequant -----
    // Two groups of four warps take alternate k-steps (group gamma the
    // steps whose index in this CTA's sequence has parity gamma); each
    // thread covers one (tile, g, p) position of every A tensor of the
    // stage: rows g and g+8 (both row halves), columns 8p..8p+7 of each
    // 16-column half of the stage's 64 columns.
    const int gamma = (warp - C::WDQ0) >> 2;
    const int t = threadIdx.x - (C::WDQ0 + 4 * gamma) * 32;   // 0..127
    const int tg = t & 7, tp_ = (t >> 3) & 1, tti = t >> 4;
    const int tcols = SB3 ? SB3_TILE_COLS : B32_TILE_COLS;
    const int tbytes = af_tile_bytes(AF);
    const int64_t trow_stride = (int64_t)(p.K / tcols) * tbytes;  // 16 rows
    const B32Tab tab = {p.tab[0], p.tab[1], p.tab[2], p.tab[3]};
    // tile pointers of the prefetch position's unit
    const uint8_t* ptp[NA];
    int pf_it = -1;
    auto set_unit = [&](int it) {
      pf_it = it;
      const int u = blockIdx.x + it * gridDim.x;
      if (u >= n_units) return;
      const int4 tile = p.tiles[u / MT];
      const int m = u % MT;
      const int e = tile.x;
      int64_t bi = p.blob_index ? (int64_t)p.blob_index[e] : (int64_t)e;
      if (bi < 0) {   // no blob: report, and read blob 0 so the unit completes
        if (t == 0) set_err(err, MOE_ERR_DEVICE);
        bi = 0;
      }
      const uint8_t* blob = p.pool + bi * p.blob_stride;
#pragma unroll
      for (int a = 0; a < NA; ++a)
        ptp[a] = blob + (a ? p.off_a1 : p.off_a0) +
                 (int64_t)(m * (PF_BM / 16) + tti) * trow_stride;
    };
    auto stage_begin = [&](uint32_t ks_glob, uint32_t& st) -> bool {
      const int s = (int)(ks_glob % S);
      const uint32_t use = ks_glob / S;
      if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, err)) return false;
      st = sbase + (uint32_t)(s * C::STAGE_BYTES);
      return true;
    };
    auto stage_end = [&](uint32_t ks_glob) {
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_a[ks_glob % S]);
    };
    const int n_my = (n_units - (int)blockIdx.x + (int)gridDim.x - 1) /
                     (int)gridDim.x;   // units of this CTA
    bool ok = true;
    if constexpr (SB3) {
      // super-block granularity (the group's two k-steps of it),
      // prefetched one super-block ahead
      const int nsb = nk / 4;
      const int total_sb = n_my * nsb;
      int pf_sb = 0;
      auto fetch = [&](Sb3Half (&q)[NA]) {
        if (pf_sb >= total_sb) return;
        const int it = pf_sb / nsb, sb = pf_sb % nsb;
        if (it != pf_it) set_unit(it);
#pragma unroll
        for (int a = 0; a < NA; ++a)
          sbx_load<AF>(ptp[a] + (int64_t)sb * tbytes, tg, tp_, gamma, q[a]);
        ++pf_sb;
      };
      Sb3Half cur[NA], nxt[NA];
      fetch(cur);
      for (int gsb = 0; ok && gsb < total_sb; ++gsb) {
        fetch(nxt);
#pragma unroll
        for (int qh = 0; qh < 2; ++qh) {
          const uint32_t ksg = (uint32_t)gsb * 4 + gamma + 2 * qh;
          uint32_t st;
          if (!stage_begin(ksg, st)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int a = 0; a < NA; ++a)
            sbx_store<AF>(cur[a], tg, tp_, gamma, qh, 16 * tti,
                          st + a * PF_A_BYTES);
          stage_end(ksg);
        }
#pragma unroll
        for (int a = 0; a < NA; ++a) cur[a] = nxt[a];
      }
    } else {
      // the group's k-steps, prefetched two of them ahead
      const uint32_t total = (uint32_t)n_my * nk;
      uint32_t pf_k = gamma;   // global k-step of the next fetch
      auto fetch = [&](B32Q (&q)[NA]) {
        if (pf_k >= total) return;
        const int it = (int)(pf_k / nk), ks = (int)(pf_k % nk);
        if (it != pf_it) set_unit(it);
#pragma unroll
        for (int a = 0; a < NA; ++a)
          q[a] = b32_load(ptp[a] + (int64_t)ks * B32_TILE_BYTES, tg, tp_);
        pf_k += 2;
      };
      B32Q q0[NA], q1[NA], q2[NA];
      fetch(q0);
      fetch(q1);
      for (uint32_t ksg = gamma; ok && ksg < total; ksg += 2) {
        fetch(q2);
        uint32_t st;
        if (!stage_begin(ksg, st)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int a = 0; a < NA; ++a)
#pragma unroll
          for (int rh = 0; rh < 2; ++rh)
            b32_store(q0[a], tg, tp_, rh, 16 * tti, tab,
                      st + a * PF_A_BYTES);
        stage_end(ksg);
#pragma unroll
        for (int a = 0; a < NA; ++a) {
          q0[a] = q1[a];
          q1[a] = q2[a];
        }
      }
    }
  } else {
    // ------------------------------------------------- epilogue -------
    // Per unit, the rows' metadata (up: the token's x scale; down: the
    // pair id) goes to this warp's slice of shared memory before the
    // accumulator wait, so its global latency overlaps the MMAs.
    int it = 0;
    const int quad = warp & 3, chalf = warp >> 2;
    constexpr int CSTEP = 32 * (C::EPI / 4);   // column stride of a warp
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    float* meta_f = reinterpret_cast<float*>(smem + C::META_OFF) + warp * PF_BN;
    int32_t* meta_i = reinterpret_cast<int32_t*>(meta_f);
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++it) {
      const int4 tile = p.tiles[u / MT];
      const int nlen = tile.z, row0 = tile.y;
      const int ab = UP ? 0 : (it & 1);
      __syncwarp();
      for (int n = 32 * chalf + lane; n < ((nlen + 31) & ~31); n += CSTEP) {
        if constexpr (UP)
          meta_f[n] = n < nlen ? p.xscale[row0 + n] : 1.f;
        else
          meta_i[n] = n < nlen ? p.pair_ids[row0 + n] : 0;
      }
      __syncwarp();
      const int use_ab = UP ? it : (it >> 1);
      if (!mbar_wait(&acc_full[ab], use_ab & 1, err)) break;
      tc::fence_after_sync();
      const int col = (u % MT) * PF_BM + quad * 32 + lane;  // output column
      // Each 32-column chunk reads its metadata into registers first, so
      // no shared-memory load waits behind a global store.
      if constexpr (UP) {
        float hmax = 0.f;
        __half* hp = p.h16 + (int64_t)row0 * p.rows + col;
        for (int c0 = 32 * chalf; c0 < nlen; c0 += CSTEP) {
          float ua[32], ga[32], sc[32];
          tc::ld_32x32b_x16(tmem + lane_base + (uint32_t)c0, *(float(*)[16])&ua[0]);
          tc::ld_32x32b_x16(tmem + lane_base + (uint32_t)(c0 + 16),
                            *(float(*)[16])&ua[16]);
          tc::ld_32x32b_x16(tmem + lane_base + 256u + (uint32_t)c0,
                            *(float(*)[16])&ga[0]);
          tc::ld_32x32b_x16(tmem + lane_base + 256u + (uint32_t)(c0 + 16),
                            *(float(*)[16])&ga[16]);
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 v = *reinterpret_cast<const float4*>(meta_f + c0 + i);
            sc[i] = v.x; sc[i + 1] = v.y; sc[i + 2] = v.z; sc[i + 3] = v.w;
          }
          tc::wait_ld();
          // silu(g) u = g u (1 + tanh(g/2)) / 2, one hardware tanh each
          __half2 hv2[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float hv[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float uu = ua[i + j] * sc[i + j];
              const float gg = ga[i + j] * sc[i + j];
              const float th = tanh_approx(0.5f * gg);
              hv[j] = (0.5f * gg * uu) * (1.0f + th);
              if (c0 + i + j < nlen) hmax = fmaxf(hmax, fabsf(hv[j]));
            }
            hv2[i / 2] = __floats2half2_rn(hv[0], hv[1]);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            if (c0 + i < nlen)
              hp[(int64_t)(c0 + i) * p.rows] = __low2half(hv2[i / 2]);
            if (c0 + i + 1 < nlen)
              hp[(int64_t)(c0 + i + 1) * p.rows] = __high2half(hv2[i / 2]);
          }
        }
        if (!(hmax < 65520.f)) set_err(err, MOE_ERR_DEVICE);   // fp16 range
      } else {
        float* yp = p.y + col;
        for (int c0 = 32 * chalf; c0 < nlen; c0 += CSTEP) {
          float acc[32];
          int pr[32];
          tc::ld_32x32b_x16(tmem + lane_base + (uint32_t)(ab * 256 + c0),
                            *(float(*)[16])&acc[0]);
          tc::ld_32x32b_x16(tmem + lane_base + (uint32_t)(ab * 256 + c0 + 16),
                            *(float(*)[16])&acc[16]);
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const int4 v = *reinterpret_cast<const int4*>(meta_i + c0 + i);
            pr[i] = v.x; pr[i + 1] = v.y; pr[i + 2] = v.z; pr[i + 3] = v.w;
          }
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < nlen) yp[(int64_t)pr[i] * p.rows] = acc[i];
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == C::WMMA) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, PF_TMEM_COLS);
  }
}

// ---------------------------------------------------- plan and inputs ---
// Unit list.  Expert e's cnt grouped rows are cut into nt = ceil(cnt/256)
// tiles of nearly equal size in whole 16-row blocks (so no expert leaves a
// small remainder tile; the last tile holds the partial block), and the
// tiles are ordered by size in 16-row blocks, largest first; one expert's
// tiles of one size stay contiguous.  The order inside a size class
// depends on atomics; every unit writes its own outputs, so results do
// not depend on it.
__global__ void __launch_bounds__(1024)
    pf_plan_kernel(const int32_t* __restrict__ offsets, int E,
                   int4* __restrict__ tiles, int32_t* __restrict__ n_tiles) {
  __shared__ int32_t hist[18], base[18];
  const int tid = threadIdx.x;
  if (tid < 18) hist[tid] = 0;
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int cnt = offsets[e + 1] - offsets[e];
    if (!cnt) continue;
    const int nb = (cnt + 15) >> 4, nt = (nb + 15) >> 4;
    const int q = nb / nt, r = nb % nt;   // r tiles of q+1 blocks, rest q
    if (r) atomicAdd(&hist[q + 1], r);
    atomicAdd(&hist[q], nt - r);
  }
  __syncthreads();
  if (tid == 0) {
    int b0 = 0;
    for (int b = 16; b >= 1; --b) {
      base[b] = b0;
      b0 += hist[b];
    }
    *n_tiles = b0;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int o = offsets[e], cnt = offsets[e + 1] - o;
    if (!cnt) continue;
    const int nb = (cnt + 15) >> 4, nt = (nb + 15) >> 4;
    const int q = nb / nt, r = nb % nt;
    int p1 = 0, p0;
    if (r) p1 = atomicAdd(&base[q + 1], r);
    p0 = atomicAdd(&base[q], nt - r);
    int row = o;
    for (int i = 0; i < nt; ++i) {
      const int blocks = i < r ? q + 1 : q;
      const int rows = min(16 * blocks, o + cnt - row);
      tiles[i < r ? p1 + i : p0 + (i - r)] = make_int4(e, row, rows, 0);
      row += rows;
    }
  }
}

// inv[pair_ids[r]] = r: the grouped row of every pair (pair_ids is a
// permutation of 0 .. P-1, as the grouping produces it).
// Grouped row of each pair: inv[pair_ids[r]] = r for the n_rows listed
// pairs (the grouping may list a subset of the P pairs); unlisted pairs
// keep -1 (inv is filled with -1 first by pf_fill_kernel).
__global__ void pf_inv_kernel(const int32_t* __restrict__ pair_ids,
                              const int32_t* __restrict__ offsets, int E,
                              int P, int32_t* __restrict__ inv) {
  const int n_rows = offsets[E];
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < n_rows && r < P) {
    const int q = pair_ids[r];
    if (q >= 0 && q < P) inv[q] = r;
  }
}
__global__ void pf_fill_kernel(int32_t* __restrict__ v, int n, int32_t val) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] = val;
}

// One block per token t: x[t] as fp16, scaled by a power of two 2^-sigma
// that keeps every value below 2^15 (sigma = 0 unless max|x_t| >= 2^15),
// written to the grouped rows of the token's k pairs; xscale of those rows
// = 2^sigma.  H a multiple of 8.
__global__ void __launch_bounds__(256)
    pf_xg_kernel(const uint16_t* __restrict__ x, int H, int k,
                 const int32_t* __restrict__ inv, __half* __restrict__ xg,
                 float* __restrict__ xscale) {
  __shared__ float red[8];
  __shared__ int32_t rows[32];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) rows[threadIdx.x] = inv[t * k + threadIdx.x];
  __syncthreads();
  // a token none of whose pairs the grouping lists is not needed
  bool any = false;
  for (int j = 0; j < k; ++j) any |= rows[j] >= 0;
  if (!any) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + t * H);
  const int nch = H / 8;
  float m = 0.f;
  for (int c = threadIdx.x; c < nch; c += blockDim.x) {
    const uint4 v = __ldg(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[i] << 16)),
                         fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  int sigma = 0;
  if (m >= 32768.f && m <= 3.0e38f) sigma = ilogbf(m) - 14;
  const float inv_s = ldexpf(1.f, -sigma);
  if (threadIdx.x < k && rows[threadIdx.x] >= 0)
    xscale[rows[threadIdx.x]] = ldexpf(1.f, sigma);
  for (int c = threadIdx.x; c < nch; c += blockDim.x) {
    const uint4 v = __ldg(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 q = __floats2half2_rn(__uint_as_float(w[i] << 16) * inv_s,
                                          __uint_as_float(w[i] & 0xFFFF0000u) * inv_s);
      h[i] = *reinterpret_cast<const uint32_t*>(&q);
    }
    const uint4 hv = make_uint4(h[0], h[1], h[2], h[3]);
    for (int j = 0; j < k; ++j)
      if (rows[j] >= 0)
        reinterpret_cast<uint4*>(xg + (int64_t)rows[j] * H)[c] = hv;
  }
}

}  // namespace

// ------------------------------------------------------------ launchers --
bool pf_supported(const moe_layer_desc& d, int T) {
  return T > DEC_TMAX && d.F % PF_BM == 0 && d.H % PF_BM == 0 &&
         d.H % PF_BK == 0 && d.F % PF_BK == 0;
}

int64_t pf_max_tiles(int64_t P) { return P / PF_BN + P + 1; }

static void pf_tables(int fmt, uint32_t (&t)[4]) {
  if (fmt == MOE_NL4_B32) {
    t[0] = NL4_TA0; t[1] = NL4_TA1; t[2] = NL4_TB0; t[3] = NL4_TB1;
  } else {
    t[0] = Q4_TA0; t[1] = Q4_TA1; t[2] = Q4_TB0; t[3] = Q4_TB1;
  }
}

bool pf_export_supported(int fmt, int rows, int cols) {
  return rows > 0 && cols > 0 && rows % PF_BM == 0 &&
         cols % tile_cols(fmt) == 0;
}

moe_status launch_pf_dequant_export(int fmt, const uint8_t* t, int rows,
                                    int cols, uint16_t* out, cudaStream_t s) {
  uint32_t tb[4] = {0u, 0u, 0u, 0u};
  if (!fmt_sb(fmt)) pf_tables(fmt, tb);
  const uint4 tab4 = make_uint4(tb[0], tb[1], tb[2], tb[3]);
  const bool sb3 = fmt_sb(fmt);
  const int nks = sb3 ? 4 : 2;
  const size_t smem = (size_t)nks * PF_A_BYTES + 1024;
  const int af = af_of(fmt);
  const void* fn = af == AF_SB3   ? (const void*)&pf_dequant_export_kernel<AF_SB3>
                   : af == AF_NL3 ? (const void*)&pf_dequant_export_kernel<AF_NL3>
                   : af == AF_SB2 ? (const void*)&pf_dequant_export_kernel<AF_SB2>
                                  : (const void*)&pf_dequant_export_kernel<AF_B32>;
  moe_status st = ensure_smem(fn, smem);
  if (st != MOE_OK) return st;
  const dim3 grid(rows / PF_BM, sb3 ? cols / SB3_TILE_COLS
                                    : (cols / PF_BK + 1) / 2);
  if (af == AF_SB3)
    pf_dequant_export_kernel<AF_SB3><<<grid, 256, smem, s>>>(t, cols, tab4,
                                                             out);
  else if (af == AF_NL3)
    pf_dequant_export_kernel<AF_NL3><<<grid, 256, smem, s>>>(t, cols, tab4,
                                                             out);
  else if (af == AF_SB2)
    pf_dequant_export_kernel<AF_SB2><<<grid, 256, smem, s>>>(t, cols, tab4,
                                                             out);
  else
    pf_dequant_export_kernel<AF_B32><<<grid, 256, smem, s>>>(t, cols, tab4,
                                                             out);
  return launch_status();
}

// fp16 [outer][inner] row-major tensor map with the 128-byte swizzle and
// zero fill out of range; encoded through the driver entry point.
static moe_status encode_f16_map(CUtensorMap* m, const void* base,
                                 uint64_t inner, uint64_t outer,
                                 uint32_t box_rows) {
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
  const cuuint32_t box[2] = {(cuuint32_t)PF_BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims,
         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

static moe_status encode_maps(PfMaps* maps, const void* base, uint64_t inner,
                              uint64_t outer) {
  for (int b = 0; b < PF_NMAPS; ++b) {
    const moe_status st =
        encode_f16_map(&maps->m[b], base, inner, outer, 256u >> b);
    if (st != MOE_OK) return st;
  }
  return MOE_OK;
}

template <bool UP, int AF>
static moe_status pf_launch(const PfParams& prm, const PfMaps& map,
                            cudaStream_t s) {
  const void* fn = reinterpret_cast<const void*>(&pf_gemm_kernel<UP, AF>);
  moe_status st = ensure_smem(fn, PfCfg<UP>::SMEM);
  if (st != MOE_OK) return st;
  pf_gemm_kernel<UP, AF>
      <<<num_sms(), PfCfg<UP>::THREADS, PfCfg<UP>::SMEM, s>>>(prm, map);
  return launch_status();
}
template <bool UP>
static moe_status pf_launch_fmt(int fmt, const PfParams& prm,
                                const PfMaps& map, cudaStream_t s) {
  switch (af_of(fmt)) {
    case AF_SB3: return pf_launch<UP, AF_SB3>(prm, map, s);
    case AF_NL3: return pf_launch<UP, AF_NL3>(prm, map, s);
    case AF_SB2: return pf_launch<UP, AF_SB2>(prm, map, s);
    default: return pf_launch<UP, AF_B32>(prm, map, s);
  }
}

// The up/gate GEMM launch alone, on the grouped activations, row scales
// and unit plan that launch_pf_up staged in the workspace.
moe_status launch_pf_up_gemm(const moe_layer_desc& d, int T, int k,
                             const int32_t* pair_ids,
                             const int32_t* blob_index, const FfnWs& w,
                             cudaStream_t s) {
  const int64_t P = (int64_t)T * k;
  PfMaps map;
  moe_status st = encode_maps(&map, w.x16, (uint64_t)d.H, (uint64_t)P);
  if (st != MOE_OK) return st;
  PfParams prm{};
  prm.pool = d.pool;
  prm.blob_stride = d.blob_stride;
  prm.blob_index = blob_index;
  prm.off_a0 = 0;
  prm.off_a1 = tensor_bytes_of(d.fmt_up_gate, d.F, d.H);
  prm.K = d.H;
  prm.rows = d.F;
  prm.k = k;
  prm.pair_ids = pair_ids;
  prm.tiles = w.tiles;
  prm.n_tiles = w.n_tiles;
  prm.xscale = w.xscale;
  prm.h16 = reinterpret_cast<__half*>(w.h);
  prm.err = w.err;
  pf_tables(d.fmt_up_gate, prm.tab);
  return pf_launch_fmt<true>(d.fmt_up_gate, prm, map, s);
}

moe_status launch_pf_up(const moe_layer_desc& d, const uint16_t* x, int T,
                        int k, const int32_t* offsets,
                        const int32_t* pair_ids, const int32_t* blob_index,
                        const FfnWs& w, cudaStream_t s) {
  const int64_t P = (int64_t)T * k;
  pf_fill_kernel<<<(unsigned)((P + 255) / 256), 256, 0, s>>>(w.inv, (int)P,
                                                            -1);
  pf_inv_kernel<<<(unsigned)((P + 255) / 256), 256, 0, s>>>(
      pair_ids, offsets, d.E, (int)P, w.inv);
  pf_xg_kernel<<<T, 256, 0, s>>>(x, d.H, k, w.inv, w.x16, w.xscale);
  pf_plan_kernel<<<1, 1024, 0, s>>>(offsets, d.E, w.tiles, w.n_tiles);
  const moe_status st = launch_status();
  if (st != MOE_OK) return st;
  return launch_pf_up_gemm(d, T, k, pair_ids, blob_index, w, s);
}

moe_status launch_pf_down(const moe_layer_desc& d, int T, int k,
                          const int32_t* pair_ids, const int32_t* blob_index,
                          const FfnWs& w, float* y, cudaStream_t s) {
  const int64_t P = (int64_t)T * k;
  PfMaps map;
  moe_status st = encode_maps(&map, w.h, (uint64_t)d.F, (uint64_t)P);
  if (st != MOE_OK) return st;
  PfParams prm{};
  prm.pool = d.pool;
  prm.blob_stride = d.blob_stride;
  prm.blob_index = blob_index;
  prm.off_a0 = 2 * tensor_bytes_of(d.fmt_up_gate, d.F, d.H);
  prm.off_a1 = prm.off_a0;
  prm.K = d.F;
  prm.rows = d.H;
  prm.k = k;
  prm.pair_ids = pair_ids;
  prm.tiles = w.tiles;
  prm.n_tiles = w.n_tiles;
  prm.y = y;
  prm.err = w.err;
  pf_tables(d.fmt_down, prm.tab);
  return pf_launch_fmt<false>(d.fmt_down, prm, map, s);
}

}  // namespace moe
