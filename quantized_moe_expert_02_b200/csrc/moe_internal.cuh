// Internal definitions of the MoE library: packed tile layouts, workspace
// carving, PTX wrappers.  sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ------------------------------------------------------------ formats ----
// Packed GPU tile layout (this library's own; the natural layout is in
// moe.h).  A tensor [R x C] is cut into tiles of 16 rows; tiles are stored
// row-tile major, column-tile minor.  Inside a tile, the codes are ordered
// so that lane L = 4*g + c of a warp finds, in one 16-byte word per plane,
// the int8 A fragment of `mma.sync.m16n8k32` (rows g and g+8, columns
// 4c..4c+3 and 16+4c..16+4c+3 of each 32-column block) after a byte-table
// lookup; scales of rows g and g+8 sit next to each other.
//
// SB3 tile = 16 rows x 256 columns (one super-block per row), 1632 bytes:
//   [   0, 512)  LO[0..3]  lane L at 16L: 2-bit low parts of the codes of
//                          32-blocks j = 0..3 (one 32-bit word per block)
//   [ 512,1024)  LO[4..7]
//   [1024,1536)  HI[0..3]  high code bits, word m covers blocks 2m, 2m+1
//   [1536,1600)  sub-scale words, row r at 4*pi(r)   (natural nibble order)
//   [1600,1632)  fp16 d, row r at 2*pi(r)
// with pi(r) = 2*(r%8) + r/8.  For block j, A register r (0..3), element w
// (0..3) of lane (g, c): tile row g + 8*(r&1), column 32j + 16*(r>>1) +
// 4c + w; nibble n = 4*(r&1) + w; the 2-bit low part sits at bit
// 4n + 2*(r>>1) of LO[j]; the high bit at bit 4n + 2*(j&1) + (r>>1) of
// HI[j>>1].
//
// B32 tile (Q4 / NL4) = 16 rows x 64 columns (two 32-blocks), 576 bytes:
//   [  0,512)  lane L at 16L: words W[2b+h] (b = block 0/1, h = half):
//              nibble n of W[2b+h] = code of row g + 8*(n>>2), column
//              32b + 16h + 4c + (n&3)
//   [512,576)  fp16 d: row r, block b at 2*(4*(r%8) + 2*(r/8) + b)
//
// NL3 tile (MOE_NL3_256) = the SB3 tile (codes, sub-scales, d at the same
// offsets) followed by
//   [1632,1648)  codebook-shift bytes, row r at 1632 + pi(r) (bit j = e_j
//                of 32-block j)
// 1648 bytes.
//
// SB2 tile (MOE_SB2_256) = 16 rows x 256 columns of 2-bit codes, 1120
// bytes: the SB3 tile without its HI plane --
//   [   0,1024)  LO[0..7] as in SB3 (the 2-bit code of each weight)
//   [1024,1088)  sub-scale words, row r at 4*pi(r)
//   [1088,1120)  fp16 d, row r at 2*pi(r)
constexpr int SB3_TILE_BYTES = 1632;
constexpr int SB2_TILE_BYTES = 1120;
constexpr int SB3_TILE_COLS = 256;
constexpr int NL3_TILE_BYTES = 1648;
constexpr int B32_TILE_BYTES = 576;
constexpr int B32_TILE_COLS = 64;
constexpr int TILE_ROWS = 16;

// The super-block formats (256 columns per tile, codes in the LO plane and,
// for the 3-bit ones, the HI plane): SB3, NL3 and SB2.
__host__ __device__ inline bool fmt_sb(int fmt) {
  return fmt == MOE_SB3_256 || fmt == MOE_NL3_256 || fmt == MOE_SB2_256;
}
__host__ __device__ inline int tile_bytes(int fmt) {
  return fmt == MOE_SB3_256   ? SB3_TILE_BYTES
         : fmt == MOE_NL3_256 ? NL3_TILE_BYTES
         : fmt == MOE_SB2_256 ? SB2_TILE_BYTES
                              : B32_TILE_BYTES;
}
__host__ __device__ inline int tile_cols(int fmt) {
  return fmt_sb(fmt) ? SB3_TILE_COLS : B32_TILE_COLS;
}
inline bool fmt_valid(int fmt) {
  return fmt == MOE_Q4_B32 || fmt == MOE_SB3_256 || fmt == MOE_NL4_B32 ||
         fmt == MOE_NL3_256 || fmt == MOE_SB2_256;
}
// Shape accepted by the packed layout.
inline bool packed_shape_ok(int fmt, int rows, int cols) {
  return fmt_valid(fmt) && rows > 0 && cols > 0 && rows % TILE_ROWS == 0 &&
         cols % tile_cols(fmt) == 0;
}
__host__ __device__ inline int64_t tensor_bytes_of(int fmt, int rows,
                                                   int cols) {
  return (int64_t)(rows / TILE_ROWS) * (cols / tile_cols(fmt)) *
         tile_bytes(fmt);
}

// int8 byte tables of the decoders (see the PRMT-based decode).
// SB3: code q (0..7) -> c = 2q - 7.
constexpr uint32_t SB3_TAB0 = 0xFFFDFBF9u;  // q=0..3 -> -7,-5,-3,-1
constexpr uint32_t SB3_TAB1 = 0x07050301u;  // q=4..7 ->  1, 3, 5, 7
// NL4: A1 table holds cb[q] for q < 8 (all negative, so a selector with
// bit 3 set replicates their sign: 0xFF = -1); A2 table holds cb[q] + 1
// for q >= 8 (all positive, so a set bit 3 gives 0).  A1 + A2 = cb[q].
constexpr uint32_t NL4_TA0 = 0xBFAD9881u;   // -127,-104,-83,-65
constexpr uint32_t NL4_TA1 = 0xF6EADDCFu;   //  -49, -35,-22,-10
constexpr uint32_t NL4_TB0 = 0x271A0E02u;   //    2,  14, 26, 39
constexpr uint32_t NL4_TB1 = 0x725A4636u;   //   54,  70, 90,114
// NL3: the 3-bit codebook {-15,-10,-6,-2,1,5,9,14} as int8 bytes, q = 0..3
// and 4..7; a set shift bit e adds 1 to every byte (no byte is -1, so the
// 32-bit add never carries across bytes).
constexpr uint32_t NL3_TAB0 = 0xFEFAF6F1u;  // -15,-10, -6, -2
constexpr uint32_t NL3_TAB1 = 0x0E090501u;  //   1,  5,  9, 14
// SB2: code q (0..3) -> c = 2q - 3.
constexpr uint32_t SB2_TAB0 = 0x0301FFFDu;  // -3,-1, 1, 3
// Q4: q - 8 in the same split.
constexpr uint32_t Q4_TA0 = 0xFBFAF9F8u;    // -8..-5
constexpr uint32_t Q4_TA1 = 0xFFFEFDFCu;    // -4..-1
constexpr uint32_t Q4_TB0 = 0x04030201u;    //  1..4  (= q-8+1, q=8..11)
constexpr uint32_t Q4_TB1 = 0x08070605u;    //  5..8

// ------------------------------------------------------------ status -----
#define MOE_CUDA_TRY(expr)                       \
  do {                                           \
    cudaError_t e__ = (expr);                    \
    if (e__ != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

inline moe_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Device error word: first error wins.
__device__ inline void set_err(int32_t* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

int num_sms();  // SM count of the current device (cached)
// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device (cached per kernel and device; thread-safe).
moe_status ensure_smem(const void* kernel, size_t bytes);

// ------------------------------------------------------- workspace -------
// Decode path limits.
constexpr int DEC_TMAX = 8;     // tokens per decode call (two N tiles)
constexpr int NSPLIT_MAX = 4;   // K split of the up/gate units
constexpr int BF_NT = 2;        // N tiles (4 tokens each) of the B layouts

// Modes of one launch of the one-kernel decode layer.  DL_ROUTE then
// DL_FFN computes exactly what DL_FULL does (same router partition, same
// top-k and weights, same FFN), so a caller can act between routing and
// the FFN (the expert-slot cache fills its misses there) without changing
// a bit of the result.
constexpr int DL_FULL = 0, DL_ROUTE = 1, DL_FFN = 2;

// In-kernel staging of a slot-cache layer's misses (DL_FFN): the slot
// resolve's miss list, the host blob table and the layer's partition.
struct StageArgs {
  const int32_t* n_miss;
  const int32_t* miss_expert;
  const int32_t* miss_slot;
  const uint64_t* table;
  int layer;
  int slot_base, n_slots;
  int64_t pool_slots, blob_bytes;
};

struct FfnWs {
  int32_t* err;       // [4]  error word, route counter, spare
  int32_t* up_cnt;    // [P * F/32]   arrival counters, 32-row up tiles
  int32_t* dn_cnt;    // [H/16]       arrival counters, down row tiles
  float* up_part;     // [P][F/32][4][2][32][8] split-K partials
  uint32_t* bfrag;    // [P][F/32][2][32][2] down B fragments (int8 hi/lo)
  float* bscale;      // [P][F/32][8]   2^-sigma per (expert, block, slot)
  float* y_int;       // [T*k][H]       y_pairs of the fused combine
  float* h;           // [T*k][F]       generic path: SwiGLU output
  float* logits;      // [T][Emax]      route scratch when no logits_out
  int32_t* grp;       // grouping scratch
  // tensor-core path (T > DEC_TMAX); h above then holds fp16 [T*k][F] in
  // grouped row order
  __half* x16;        // [T*k][H] activations as fp16, grouped row order
  float* xscale;      // [T*k]    2^sigma per grouped row
  int32_t* inv;       // [T*k]    grouped row of each pair
  int4* tiles;        // unit list: {expert, first grouped row, rows, 0}
  int32_t* n_tiles;
  size_t bytes;
};

// Largest E the route kernels accept.
constexpr int EMAX = 4096;

size_t group_ws_bytes(int T, int k, int E);
FfnWs carve_ffn_ws(void* base, int T, int k, int H, int F);

// --------------------------------------------------------------- PTX -----
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b,
                                         uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// D = A(16x32 s8) * B(32x8 s8) + C, int32 accumulate.
__device__ __forceinline__ void mma_s8(int32_t (&d)[4], const uint32_t (&a)[4],
                                       uint32_t b0, uint32_t b1,
                                       const int32_t (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1),
        "r"(c[0]), "r"(c[1]), "r"(c[2]), "r"(c[3]));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(void* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(void* bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive(void* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// One arrival that counts `n` times toward the barrier's expected count.
__device__ __forceinline__ void mbar_arrive_n(void* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(n)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(void* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// The same test, but a thread whose phase is not complete is suspended
// (issuing nothing) until the phase completes or about `ns` nanoseconds
// pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(void* bar, uint32_t parity,
                                                    uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete; give up after 0.5 s of
// %globaltimer, set MOE_ERR_TIMEOUT and return false.  Once any wait of the
// launch has given up, later waits return false at once.
__device__ __forceinline__ bool mbar_wait(void* bar, uint32_t parity,
                                          int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  if (err && *reinterpret_cast<volatile int32_t*>(err) == MOE_ERR_TIMEOUT)
    return false;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
    if (globaltimer() - t0 > 500000000ull) {
      set_err(err, MOE_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Wait for the phase of `parity` to complete, bounded by 0.5 s of
// %globaltimer but without mbar_wait's early return after another wait of
// the launch gave up: for draining copies that are in flight.
__device__ __forceinline__ bool mbar_wait_drain(void* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_sleep(bar, parity, 20000u))
    if (globaltimer() - t0 > 500000000ull) return false;
  return true;
}

// 1-D bulk copy global -> shared, completion counted on `bar`.  Addresses
// 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src,
                                         uint32_t bytes, void* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Arrive on named barrier `id` without waiting (the barrier's other
// participants wait with bar.sync); this thread's earlier memory accesses
// are performed for them when the barrier completes.
__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// Exclusive scan of v[0..n) in place by one block of 1024 threads;
// returns the total.  n <= 8 * 1024.
__device__ inline int block_exclusive_scan(int32_t* v, int n, int32_t* tmp) {
  const int tid = threadIdx.x, per = (n + 1023) / 1024;
  int local = 0;
  for (int i = 0; i < per; ++i) {
    const int idx = tid * per + i;
    if (idx < n) local += v[idx];
  }
  // warp inclusive scan
  const int lane = tid & 31, warp = tid >> 5;
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = tmp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    tmp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int run = x - local + (warp ? tmp[warp - 1] : 0);
  const int total = tmp[31];
  __syncthreads();
  for (int i = 0; i < per; ++i) {
    const int idx = tid * per + i;
    if (idx < n) {
      const int c = v[idx];
      v[idx] = run;
      run += c;
    }
  }
  __syncthreads();
  return total;
}

// ---------------------------------------------------- packed decoding ----
// Value of element (row, col) of a packed tensor (generic, slow path).
__device__ inline float dq_packed(int fmt, const uint8_t* t, int cols,
                                  int row, int col) {
  const int tc = tile_cols(fmt);
  const int ntc = cols / tc;
  const uint8_t* tile =
      t + ((int64_t)(row / TILE_ROWS) * ntc + col / tc) * tile_bytes(fmt);
  const int r = row % TILE_ROWS, g = r % 8, half = r / 8;
  const int pi = 2 * g + half;
  if (fmt_sb(fmt)) {
    const int kk = col % 256, j = kk / 32, k32 = kk % 32;
    const int hsel = k32 / 16, c = (k32 % 16) / 4, w = k32 % 4;
    const int lane = 4 * g + c;
    const int reg_odd = half, reg_hi = hsel;  // r&1, r>>1
    const int n = 4 * reg_odd + w;
    const uint32_t lo =
        *(const uint32_t*)(tile + 512 * (j / 4) + 16 * lane + 4 * (j % 4));
    if (fmt == MOE_SB2_256) {
      const int q2 = (lo >> (4 * n + 2 * reg_hi)) & 3;
      const int s2 = (*(const uint32_t*)(tile + 1024 + 4 * pi) >> (4 * j)) & 15;
      const float d2 = __half2float(*(const __half*)(tile + 1088 + 2 * pi));
      return d2 * (float)((2 * s2 + 1) * (2 * q2 - 3)) * 0.25f;
    }
    const uint32_t hi = *(const uint32_t*)(tile + 1024 + 16 * lane +
                                           4 * (j / 2));
    const int q = ((lo >> (4 * n + 2 * reg_hi)) & 3) |
                  (((hi >> (4 * n + 2 * (j & 1) + reg_hi)) & 1) << 2);
    const uint32_t sw = *(const uint32_t*)(tile + 1536 + 4 * pi);
    const int s = (sw >> (4 * j)) & 15;
    const float d =
        __half2float(*(const __half*)(tile + 1600 + 2 * pi));
    if (fmt == MOE_NL3_256) {
      const int8_t cb[8] = {-15, -10, -6, -2, 1, 5, 9, 14};
      const int e = (tile[1632 + pi] >> j) & 1;
      return d * (float)((2 * s + 1) * (cb[q] + e)) * 0.0625f;
    }
    return d * (float)(2 * s + 1) * (float)(2 * q - 7) * 0.125f;
  } else {
    const int kk = col % 64, b = kk / 32, k32 = kk % 32;
    const int hsel = k32 / 16, c = (k32 % 16) / 4, w = k32 % 4;
    const int lane = 4 * g + c;
    const uint32_t word =
        *(const uint32_t*)(tile + 16 * lane + 4 * (2 * b + hsel));
    const int n = 4 * half + w;
    const int q = (word >> (4 * n)) & 15;
    const float d = __half2float(
        *(const __half*)(tile + 512 + 2 * (4 * g + 2 * half + b)));
    float v;
    if (fmt == MOE_Q4_B32) {
      v = (float)(q - 8);
    } else {
      const int8_t cb[16] = {-127, -104, -83, -65, -49, -35, -22, -10,
                             1,    13,   25,  38,  53,  69,  89,  113};
      v = (float)cb[q];
    }
    return d * v;
  }
}

}  // namespace moe
