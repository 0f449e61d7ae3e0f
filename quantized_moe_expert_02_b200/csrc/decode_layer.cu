// One whole decode layer (T <= 8 tokens) in one persistent cooperative
// kernel: router + top-k, grouping, up/gate + SwiGLU, down, combine.
//
// One block per SM.  Warps 0..15 compute; warp 16 is a producer that
// streams the chosen experts' packed tiles into a ring of four shared-
// memory slots with 1-D bulk copies (cp.async.bulk + mbarrier), first the
// up/gate units (one per slot), then -- without waiting for the up phase to
// finish -- the down units (four per slot), so the expert stream does not
// stop at the phase boundaries; warp 17 publishes finished up units to the
// other blocks; warps 18 and 19 finish the up units of the two up groups
// (reduction, SwiGLU, h stores), so that the compute warps go on to their
// next unit at once.  Only the warps that use a slot wait on it and
// release it.
//
// Phases (grid barriers marked ||):
//   P0  router logits: the E rows are split over the blocks; x staged in
//       shared memory (or computed as bf16(rmsnorm(r)) from a residual)
//   ||
//   P1  every block: top-k of every token from the logits (a warp per
//       token, one redux.sync arg-max per round), softmax weights, grouping
//       of the T*k pairs by expert -- all in shared memory; meanwhile the
//       other warps turn x into int8 hi/lo B fragments (2^-sigma per token
//       and 256-column block)
//   P2  up/gate units (expert, 16 rows of F, all of H), two groups of eight
//       warps taking alternate units, three tiles per warp, partial sums
//       -> shared memory; the group's epilogue warp reduces them,
//       h = silu(g) * u of each of the expert's tokens -> global,
//       |h| max per pair -> global; each finished unit counts towards its
//       expert's completion counter
//   P3  down B fragments: once the (at most two) experts of this block's
//       down units are complete (their counters, not a grid barrier), h is
//       quantised with one scale per pair
//   P4  down units (expert, 16 rows of H, all of F), four per slot, one per
//       group of four warps: y of each pair -> global
//   ||
//   P5  combine: out[t] = sum_j w[t,j] y[t,j] (+ residual), j ascending
//
// Staged FFN variant (STG, expert-slot cache): one more warp per block
// pulls this block's share of every missed expert's blob from pinned host
// memory into its slot while the others compute; the grouping puts the
// missed experts after the hits, and the producer waits (bounded) for a
// missed expert's blob to be complete in every block before it copies that
// expert's tiles.
#include <float.h>

#include "decode_pieces.cuh"

namespace moe {

namespace {

constexpr int CW = 16;                      // compute warps
constexpr int LAYER_THREADS = (CW + 4) * 32;
constexpr int PRODUCER = CW;                // warp index of the producer
constexpr int SIGNALER = CW + 1;            // publishes finished up units
constexpr int UPEPI = CW + 2;               // up epilogue warps: 18, 19
constexpr int NSLOT = 4;                    // ring slots
constexpr int MAXP = 96;                    // max pairs (T*k) per call
constexpr int BAR_ALL = 1;                  // named barrier: all 16 warps
constexpr int BAR_RDY = 2;                  // 2, 3: up partials written
constexpr int BAR_FREE = 9;                 // 9, 10: up partials read
constexpr int BAR_DN = 4;                   // 4..7: down groups
constexpr int BAR_XF = 8;                   // warps that build x fragments
constexpr int UPG = 2, UPW = CW / UPG;      // up: 2 groups of 8 warps
constexpr int DNG = 4, DNW = CW / DNG;      // down: 4 groups of 4 warps
constexpr int EMAX_FUSED = 1024;            // widest router of this kernel
constexpr int PULLER = CW + 4;              // STG: pulls missed blobs
constexpr int LAYER_THREADS_STG = LAYER_THREADS + 32;
#ifndef MOE_PULL_DEPTH
#define MOE_PULL_DEPTH 8
#endif
constexpr int PULL_DEPTH = MOE_PULL_DEPTH;  // STG: 16-byte loads in flight per lane

struct LayerParams {
  const uint8_t* pool;
  int64_t stride;
  const int32_t* blob_index;
  int E, H, F, T, k;
  int64_t gate_off, down_off;
  const uint16_t* x;       // bf16 [T][H] (or null: use r_in)
  const float* r_in;       // fp32 [T][H]: x = bf16(rmsnorm(r_in))
  const uint16_t* wr;      // bf16 [E][H]
  const float* bias;       // fp32 [E] or null
  int32_t* topk_idx;       // [T][k]
  float* topk_w;           // [T][k]
  float* logits;           // [T][E]
  const float* residual;   // fp32 [T][H] or null (may alias out)
  float* out;              // fp32 [T][H]
  uint16_t* out_bf16;      // bf16 [T][H] or null
  float* h;                // ws [T*k][F]
  uint32_t* hmax;          // ws [T*k]
  float* y;                // ws [T*k][H]
  int32_t* bar;            // ws [2]: grid barrier, exit counter
  int32_t* up_done;        // ws [MAXP]: finished up units per expert
  int32_t* err;
  // STG: the slot resolve's misses, pulled from pinned host memory
  const int32_t* n_miss;
  const int32_t* miss_expert;    // [P], ascending expert id
  const int32_t* miss_slot;      // [P], slot inside the partition
  const uint64_t* stage_table;   // device addresses of the host blobs
  int stage_layer;               // row stage_layer * E of the table
  int slot_base, n_slots;        // the layer's partition of the pool
  int64_t pool_slots, blob_bytes;
  int32_t* ready;                // ws [MAXP]: blocks done with miss m
  int mode;                // DL_FULL, DL_ROUTE (P0-P1 top-k only) or
                           // DL_FFN (top-k read from topk_idx/topk_w)
};


struct Smem {  // offsets into dynamic shared memory
  int slot_bytes, ring, frag, red, misc, xsc, total;
};

__host__ __device__ inline int dn_unit_bytes(int F) {
  return (F / B32_TILE_COLS) * B32_TILE_BYTES;
}
// Reduction buffers: an up group holds [UPW][32 lanes][NT][2 rows][2]
// floats, a down group [DNW][32][NT][2] (double-buffered).
__host__ __device__ inline int red_up_floats(int NT) {
  return UPW * 32 * NT * 4;
}
__host__ __device__ inline int red_dn_floats(int NT) {
  return DNW * 32 * NT * 2;
}
__host__ __device__ inline Smem smem_layout_slot(int slot, int H, int F,
                                                 int T) {
  Smem L;
  slot = (slot + 127) / 128 * 128;
  const int NT = (T + 3) / 4;
  const int xfrag = (H / 32) * NT * 64 * 4;
  const int hfrag = 2 * (F / 32) * NT * 64 * 4;
  const int red_up = UPG * red_up_floats(NT) * 4;
  const int red_dn = DNG * 2 * red_dn_floats(NT) * 4;
  L.slot_bytes = slot;
  L.ring = 0;
  L.frag = NSLOT * slot;
  L.red = L.frag + ((xfrag > hfrag ? xfrag : hfrag) + 127) / 128 * 128;
  L.misc = L.red + (red_up > red_dn ? red_up : red_dn);
  // activation scales: float 2^-sigma, then int sigma, [nxb][DEC_TMAX] each
  L.xsc = L.misc + 3072;
  L.total = L.xsc + ((H + XB_COLS - 1) / XB_COLS) * DEC_TMAX * 8;
  return L;
}
// A ring slot holds one up unit (up and gate row tiles) or up to DNG down
// units: it is sized for DNG down units where that fits, so that a format
// with small up tiles (SB2) keeps the down phase's copies as deep as SB3.
__host__ __device__ inline Smem smem_layout(int fmt_ug, int H, int F, int T) {
  const int up = 2 * (H / tile_cols(fmt_ug)) * tile_bytes(fmt_ug);
  const int dn = dn_unit_bytes(F);
  const int base = up > dn ? up : dn;
  const int deep = base > DNG * dn ? base : DNG * dn;
  const Smem L = smem_layout_slot(deep, H, F, T);
  return L.total <= 227 * 1024 ? L : smem_layout_slot(base, H, F, T);
}

// Small shared state (at the misc offset).
struct Misc {
  uint64_t full[NSLOT];
  uint64_t empty[NSLOT];
  int32_t tk_idx[MAXP];
  float tk_w[MAXP];
  int32_t sorted[MAXP];      // pair ids sorted by (expert, pair)
  int32_t active[MAXP];      // experts with pairs, ascending
  int32_t off[MAXP + 1];     // pairs of active[u]: sorted[off[u]..off[u+1])
  float hsc[2][8];           // 2^-sigma of each pair slot, down experts
  int32_t up_fin[MAXP];      // up units of each expert finished here
  uint32_t missmap[EMAX_FUSED / 32];   // STG: experts pulled this call
  int U;
  int Uhit;                  // STG: active experts before the misses
  int nmiss;
  int flag;
};

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
__device__ __forceinline__ void red_release_add(int32_t* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v)
               : "memory");
}
// Spin until *cnt >= target (acquire); gives up after 0.5 s of
// %globaltimer (MOE_ERR_TIMEOUT, or at once when an earlier wait of this
// launch gave up).  The timer is read every 64 polls.
__device__ __forceinline__ void spin_until(const int32_t* cnt, int target,
                                           int32_t* err) {
  if (ld_acquire(cnt) >= target) return;
  if (*reinterpret_cast<volatile int32_t*>(err) == MOE_ERR_TIMEOUT) return;
  const uint64_t t0 = globaltimer();
  for (int it = 1; ld_acquire(cnt) < target; ++it) {
    if ((it & 63) == 0 && globaltimer() - t0 > 500000000ull) {
      set_err(err, MOE_ERR_TIMEOUT);
      return;
    }
  }
}

// Grid barrier among the compute warps of all blocks: barrier number `n`
// (1, 2, 3) completes when the counter reaches n * gridDim.x.  Bounded:
// gives up after 0.5 s (MOE_ERR_TIMEOUT) so the launch always ends.
__device__ void grid_barrier(const LayerParams& p, int n) {
  named_bar_sync(BAR_ALL, CW * 32);
  if (threadIdx.x == 0) {
    // the block's writes (ordered before this thread by the bar.sync) are
    // released with the arrival
    red_release_add(p.bar, 1);
    spin_until(p.bar, n * (int)gridDim.x, p.err);
  }
  named_bar_sync(BAR_ALL, CW * 32);
}
// The same barrier in two halves: the arrival (called by one thread after
// a __syncthreads that orders the block's writes before it; its release
// may take a while, so it is made by a warp with nothing else to do),
// other work, then the wait.
__device__ void grid_arrive(const LayerParams& p) {
  red_release_add(p.bar, 1);
}
__device__ void grid_wait(const LayerParams& p, int n) {
  if (threadIdx.x == 0) spin_until(p.bar, n * (int)gridDim.x, p.err);
  named_bar_sync(BAR_ALL, CW * 32);
}

__device__ __forceinline__ const uint8_t* expert_base(const LayerParams& p,
                                                      int e) {
  if (e < 0 || e >= p.E) { set_err(p.err, MOE_ERR_DEVICE); return nullptr; }
  const int64_t b = p.blob_index ? (int64_t)p.blob_index[e] : e;
  if (b < 0) { set_err(p.err, MOE_ERR_DEVICE); return nullptr; }
  return p.pool + b * p.stride;
}

// Order-preserving uint32 of a float (-0 taken as +0).
__device__ __forceinline__ uint32_t ord_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// int8 hi/lo B fragment word of 4 values: column n of the fragment is the
// high (n even) or low (n odd) half of v = round(value * 2^sigma).
__device__ __forceinline__ uint32_t frag_word(const float (&v)[4], float sc,
                                              bool low) {
  uint32_t word = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int vq = __float2int_rn(v[q] * sc);
    const int hi = (vq + 128) >> 8, lo = vq - hi * 256;
    word |= ((uint32_t)(low ? lo : hi) & 0xFFu) << (8 * q);
  }
  return word;
}

}  // namespace

template <int FUG, int FDN, int NTT, int EPL, bool STG>
__global__ void __launch_bounds__(STG ? LAYER_THREADS_STG : LAYER_THREADS, 1)
    decode_layer_kernel(LayerParams p) {
  constexpr int NTHR = STG ? LAYER_THREADS_STG : LAYER_THREADS;
  extern __shared__ __align__(128) uint8_t smem[];
  const Smem L = smem_layout(FUG, p.H, p.F, p.T);
  Misc& M = *reinterpret_cast<Misc*>(smem + L.misc);
  uint8_t* ring = smem + L.ring;
  uint32_t* frag = reinterpret_cast<uint32_t*>(smem + L.frag);
  float* red = reinterpret_cast<float*>(smem + L.red);
  // per (256-column block b, token t) at b * DEC_TMAX + t: 2^-sigma (/8 for
  // SB3) and sigma of the activations' fixed-point scale
  float* xsc = reinterpret_cast<float*>(smem + L.xsc);
  const int nxb = (p.H + XB_COLS - 1) / XB_COLS;
  int* xsig = reinterpret_cast<int*>(xsc + nxb * DEC_TMAX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, F = p.F, T = p.T, k = p.k, E = p.E;
  constexpr int NT = NTT;            // N tiles of 4 tokens: T <= 4 * NT
  constexpr int TM = 4 * NTT;
  const int G = gridDim.x;
  constexpr bool SBU = FUG == MOE_SB3_256 || FUG == MOE_NL3_256 ||
                      FUG == MOE_SB2_256;
  constexpr int TCU = SBU ? SB3_TILE_COLS : B32_TILE_COLS;
  constexpr int TBU = FUG == MOE_SB3_256   ? SB3_TILE_BYTES
                      : FUG == MOE_NL3_256 ? NL3_TILE_BYTES
                      : FUG == MOE_SB2_256 ? SB2_TILE_BYTES
                                           : B32_TILE_BYTES;
  const int nk = H / TCU;                      // up tiles per row tile
  const int nkd = F / B32_TILE_COLS;           // down tiles per row tile

  // ---------------------------------------------------------------- P0 --
  if (tid == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&M.full[s], 1);
      mbar_init(&M.empty[s], CW);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < MAXP; i += NTHR) M.up_fin[i] = 0;
  if (STG && tid < EMAX_FUSED / 32) M.missmap[tid] = 0u;
  // router rows of this block (not in DL_FFN): four warps per row, each a
  // quarter of H.  The kernel is launched as a programmatic dependent of
  // the previous kernel on the stream, and the router weights are the one
  // input that kernel does not produce: the first row chunk of every warp
  // is loaded BEFORE the wait for it (griddepcontrol.wait), so that the
  // load overlaps the end of the previous kernel; nothing else in global
  // memory is touched before the wait.
  constexpr int RQ = 4, RCH = 4;
  const bool route = p.mode != DL_FFN;
  const int e0 = (int)((int64_t)E * blockIdx.x / G);
  const int e1 = (int)((int64_t)E * (blockIdx.x + 1) / G);
  const int nrow = e1 - e0;
  const int nch = H / 8, qch = (nch + RQ - 1) / RQ;
  uint4 wpre[RCH];
  {
    const int r = warp / RQ, q = warp % RQ;
    const uint4* row =
        reinterpret_cast<const uint4*>(p.wr + (int64_t)(e0 + r) * H);
#pragma unroll
    for (int i = 0; i < RCH; ++i) {
      const int ch = q * qch + lane + 32 * i;
      wpre[i] = (route && warp < CW && r < nrow && ch < (q + 1) * qch &&
                 ch < nch)
                    ? __ldg(row + ch)
                    : make_uint4(0, 0, 0, 0);
    }
  }
  grid_dep_wait();
  uint16_t* xs = reinterpret_cast<uint16_t*>(ring);   // [T][H] bf16
  if (p.x) {
    for (int i = tid; i < T * H / 8; i += NTHR)
      reinterpret_cast<uint4*>(xs)[i] = reinterpret_cast<const uint4*>(p.x)[i];
  } else {
    for (int t = warp; t < T; t += NTHR / 32) {
      const float* r = p.r_in + (int64_t)t * H;
      float s = 0.f;
      for (int h = lane; h < H; h += 32) s = fmaf(r[h], r[h], s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float inv = 1.0f / sqrtf(s / (float)H + 1e-6f);
      for (int h = lane; h < H; h += 32)
        xs[t * H + h] = f32_to_bf16_rne(r[h] * inv);
    }
  }
  if (blockIdx.x == 0)
    for (int i = tid; i < T * k; i += NTHR) p.hmax[i] = 0u;
  __syncthreads();
  if (STG) {
    // the experts this call pulls (the slot resolve's misses)
    int nm = *p.n_miss;
    if (nm < 0 || nm > T * k) {
      if (tid == 0) set_err(p.err, MOE_ERR_DEVICE);
      nm = 0;
    }
    for (int i = tid; i < nm; i += NTHR) {
      const int e = p.miss_expert[i];
      if (e >= 0 && e < E) atomicOr(&M.missmap[e >> 5], 1u << (e & 31));
    }
    if (tid == 0) M.nmiss = nm;
  }
  // a lane issues all its loads of the row first (up to RCH 16-byte
  // chunks), then accumulates in fp32; lane sums by a fixed butterfly and
  // the quarters in fixed order (deterministic)
  if (route) {
    float* part = reinterpret_cast<float*>(smem + L.red);   // [rows][RQ][T]
    for (int base = 0; base < nrow; base += CW / RQ) {
      const int r = base + warp / RQ, q = warp % RQ;
      if (warp < CW && r < nrow) {
        const uint4* row =
            reinterpret_cast<const uint4*>(p.wr + (int64_t)(e0 + r) * H);
        float acc[TM];
#pragma unroll
        for (int t = 0; t < TM; ++t) acc[t] = 0.f;
        for (int c0 = q * qch; c0 < (q + 1) * qch && c0 < nch; c0 += 32 * RCH) {
          uint4 w[RCH];
          const bool pre = base == 0 && c0 == q * qch;
#pragma unroll
          for (int i = 0; i < RCH; ++i) {
            const int ch = c0 + lane + 32 * i;
            w[i] = pre ? wpre[i]
                       : (ch < (q + 1) * qch && ch < nch) ? __ldg(row + ch)
                                                          : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int i = 0; i < RCH; ++i) {
            const int ch = c0 + lane + 32 * i;
            if (!(ch < (q + 1) * qch && ch < nch)) continue;
            const uint32_t wv[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
            for (int t = 0; t < TM; ++t) {
              if (t < T) {
                const uint4 xv = reinterpret_cast<const uint4*>(xs + t * H)[ch];
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                float a = acc[t];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                  a = fmaf(__uint_as_float(wv[qq] << 16),
                           __uint_as_float(xw[qq] << 16), a);
                  a = fmaf(__uint_as_float(wv[qq] & 0xFFFF0000u),
                           __uint_as_float(xw[qq] & 0xFFFF0000u), a);
                }
                acc[t] = a;
              }
            }
          }
        }
#pragma unroll
        for (int t = 0; t < TM; ++t) {
          float a = acc[t];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          if (lane == 0 && t < T) part[(r * RQ + q) * DEC_TMAX + t] = a;
        }
      }
    }
    __syncthreads();
    for (int i = tid; i < nrow * T; i += NTHR) {
      const int r = i / T, t = i % T;
      float a = 0.f;
      for (int q = 0; q < RQ; ++q) a += part[(r * RQ + q) * DEC_TMAX + t];
      const float b = p.bias ? p.bias[e0 + r] : 0.f;
      p.logits[(int64_t)t * E + e0 + r] = a + b;
    }
  }
  __syncthreads();

  // ------------------------------------------------------------- P0|P1 --
  if (warp == SIGNALER && lane == 0) grid_arrive(p);
  if (warp < CW) {
    grid_wait(p, 1);
  }

  // ---------------------------------------------------------------- P1 --
  if (warp < CW) {
    if (warp >= T && p.mode != DL_ROUTE) {
      // the warps without a top-k: per-token activation scale, then the
      // int8 hi/lo B fragments of x
      const int xt = tid - T * 32, xn = (CW - T) * 32;
      // max |x| per (token, 256-column block): one warp per pair, a lane
      // per 8 values
      for (int item = warp - T; item < T * nxb; item += CW - T) {
        const int t = item / nxb, b = item % nxb;
        const int ch = b * (XB_COLS / 8) + lane;
        const float m0 =
            ch < nch ? absmax8_bf16(reinterpret_cast<const uint4*>(xs)[t * nch + ch])
                     : 0.f;
        float m = m0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) {
          const int sg = pow2_sigma(m);
          xsig[b * DEC_TMAX + t] = sg;
          xsc[b * DEC_TMAX + t] =
              exp2i(-sg) * fmt_xfold(FUG);
        }
      }
      named_bar_sync(BAR_XF, xn);
      const int nent = (H / 32) * NT * 32;
      for (int i = xt; i < nent; i += xn) {
        const int Ln = i & 31, nt = (i >> 5) % NT, blk = i / (32 * NT);
        const int n = Ln >> 2, cq = Ln & 3;
        const int t = 4 * nt + (n >> 1);
        uint2 wv = make_uint2(0u, 0u);
        if (t < T) {
          const float sc = exp2i(xsig[(32 * blk / XB_COLS) * DEC_TMAX + t]);
          const uint16_t* xr = xs + t * H + 32 * blk + 4 * cq;
          const uint2 a = *reinterpret_cast<const uint2*>(xr);
          const uint2 b = *reinterpret_cast<const uint2*>(xr + 16);
          const float va[4] = {__uint_as_float(a.x << 16),
                               __uint_as_float(a.x & 0xFFFF0000u),
                               __uint_as_float(a.y << 16),
                               __uint_as_float(a.y & 0xFFFF0000u)};
          const float vb[4] = {__uint_as_float(b.x << 16),
                               __uint_as_float(b.x & 0xFFFF0000u),
                               __uint_as_float(b.y << 16),
                               __uint_as_float(b.y & 0xFFFF0000u)};
          wv.x = frag_word(va, sc, n & 1);
          wv.y = frag_word(vb, sc, n & 1);
        }
        reinterpret_cast<uint2*>(frag)[i] = wv;
      }
    }
    if (warp < T && p.mode == DL_FFN) {
      // the caller's top-k (as a DL_ROUTE launch wrote it)
      const int t = warp;
      if (lane < k) {
        M.tk_idx[t * k + lane] = p.topk_idx[t * k + lane];
        M.tk_w[t * k + lane] = p.topk_w[t * k + lane];
      }
    } else if (warp < T) {
      // top-k of token t: lane-local candidates in registers, one
      // redux.sync arg-max per round, ties to the lowest expert index;
      // the weights exp(l_j - l_0) / sum are computed by lanes j < k
      const int t = warp;
      constexpr int PER = EPL;
      uint32_t key[PER];
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int e = lane + 32 * q;
        key[q] = e < E ? ord_key(__ldcg(p.logits + (int64_t)t * E + e)) : 0u;
      }
      uint32_t my_key = 0u;   // lane r keeps round r's winner
      int my_idx = 0;
#pragma unroll 1
      for (int r = 0; r < k; ++r) {
        // lane-local arg-max by a balanced tree; on equal keys the left
        // (lower index) side wins
        uint32_t tk[PER];
        int tq[PER];
#pragma unroll
        for (int q = 0; q < PER; ++q) { tk[q] = key[q]; tq[q] = q; }
#pragma unroll
        for (int w = 1; w < PER; w <<= 1)
#pragma unroll
          for (int q = 0; q + w < PER; q += 2 * w)
            if (tk[q + w] > tk[q]) { tk[q] = tk[q + w]; tq[q] = tq[q + w]; }
        const uint32_t bk = tk[0];
        const int bi = lane + 32 * tq[0];
        const uint32_t gk = __reduce_max_sync(0xffffffffu, bk);
        const int gi = (int)__reduce_min_sync(
            0xffffffffu, (uint32_t)(bk == gk ? bi : 0x7fffffff));
#pragma unroll
        for (int q = 0; q < PER; ++q)
          if (lane + 32 * q == gi) key[q] = 0u;
        if (lane == r) { my_key = gk; my_idx = gi; }
      }
      // the key is order-preserving and invertible: recover the logits
      const float v = __uint_as_float((my_key & 0x80000000u)
                                          ? (my_key & 0x7FFFFFFFu) : ~my_key);
      const float v0 = __shfl_sync(0xffffffffu, v, 0);
      const float ex = lane < k ? expf(v - v0) : 0.f;
      // sum in index order (lane 0 first), as a serial loop would
      float s = 0.f;
      for (int r = 0; r < k; ++r) s += __shfl_sync(0xffffffffu, ex, r);
      if (lane < k) {
        const float w = ex / s;
        M.tk_idx[t * k + lane] = my_idx;
        M.tk_w[t * k + lane] = w;
        if (blockIdx.x == 0) {
          p.topk_idx[t * k + lane] = my_idx;
          p.topk_w[t * k + lane] = w;
        }
      }
    }
    named_bar_sync(BAR_ALL, CW * 32);
    // grouping: rank of pair q = #{r : (e_r, r) < (e_q, q)}
    const int P = p.mode == DL_ROUTE ? 0 : T * k;   // DL_ROUTE: no units
    // STG: the pulled experts sort after the others (their units come
    // last, so the hits are computed while the pulls fly)
    auto gkey = [&](int e) -> int {
      return (STG && e >= 0 && e < E &&
              ((M.missmap[e >> 5] >> (e & 31)) & 1u)) ? e + EMAX_FUSED : e;
    };
    if (tid < P) {
      const int eq = M.tk_idx[tid];
      const int kq = gkey(eq);
      int rank = 0;
      for (int r = 0; r < P; ++r) {
        const int kr = gkey(M.tk_idx[r]);
        rank += (kr < kq) || (kr == kq && r < tid);
      }
      M.sorted[rank] = tid;
      if (eq < 0 || eq >= E) set_err(p.err, MOE_ERR_DEVICE);
    }
    named_bar_sync(BAR_ALL, CW * 32);
    if (warp == 0) {
      int U = 0;
      for (int i0 = 0; i0 < P; i0 += 32) {
        const int i = i0 + lane;
        bool head = false;
        if (i < P) {
          const int e = M.tk_idx[M.sorted[i]];
          head = (i == 0) || (e != M.tk_idx[M.sorted[i - 1]]);
        }
        const unsigned b = __ballot_sync(0xffffffffu, head);
        if (head) {
          const int u = U + __popc(b & ((1u << lane) - 1u));
          M.active[u] = M.tk_idx[M.sorted[i]];
          M.off[u] = i;
        }
        U += __popc(b);
      }
      if (lane == 0) {
        M.U = U;
        M.off[U] = P;
        if (STG) {
          int uh = 0;
          while (uh < U && gkey(M.active[uh]) < EMAX_FUSED) ++uh;
          M.Uhit = uh;
          // every miss must be a chosen expert of this call
          if (U - uh != M.nmiss) set_err(p.err, MOE_ERR_DEVICE);
        }
      }
    }
  }
  __syncthreads();   // the producer may start now

  const int U = M.U;
  const int nrt_f = F / 16, nrt_h = H / 16;
  // up units: (u, rt) over U x F/16; down units: (u, rt) over U x H/16
  const int nu_all = U * nrt_f, nd_all = U * nrt_h;
  // up units are dealt round-robin (unit b + i*G is this block's i-th), so
  // the experts' up units finish in expert order across the grid and a
  // down unit rarely waits; down units are contiguous ranges (at most two
  // experts per block)
  const int b0 = blockIdx.x;
  const int n_up = nu_all > b0 ? (nu_all - 1 - b0) / G + 1 : 0;
  // Down ranges are dealt in reverse block order and sized so that each
  // block's work is about even, counting an up unit as four down units
  // (their bytes) and the extra up unit of the first nu_all % G blocks as
  // eight: those blocks also take the last experts' down units, whose up
  // units are the last to finish, so they wait for them before their down
  // phase.  Plain even split when that weighting does not fit (ranges must
  // stay within two experts), and for one token: with its ten experts a
  // block has only four or five up units, and the even split is the faster
  // deal there (30.3 vs 30.8 us per layer on one B200).
  int d0, d1;
  {
    const int q_up = nu_all / G, extra = nu_all % G;
    const int64_t ctot = 4LL * q_up * G + 8LL * extra + nd_all;
    const bool weighted = T > 1 && (4LL * q_up + 8) * G <= ctot &&
                          (ctot + G - 1) / G - 4LL * q_up <= nrt_h;
    if (weighted) {
      auto before = [&](int pos) -> int {   // down units of positions < pos
        const int64_t up = 4LL * pos * q_up +
                           8LL * (pos > G - extra ? pos - (G - extra) : 0);
        return (int)(((int64_t)pos * ctot - (int64_t)G * up) / G);
      };
      const int pos = G - 1 - b0;
      d0 = before(pos);
      d1 = before(pos + 1);
    } else {
      d0 = (int)((int64_t)nd_all * b0 / G);
      d1 = (int)((int64_t)nd_all * (b0 + 1) / G);
    }
  }
  const int dnb = dn_unit_bytes(F);
  int dps = L.slot_bytes / dnb;                // down units per slot
  if (dps > DNG) dps = DNG;

  // ---------------------------------------------------------- producer --
  if (warp == PRODUCER) {
    if (lane == 0) {
      int i = 0;
      bool ok = true;   // false once a wait for a free slot gave up
      // STG: a pulled expert's tiles are copied only once every block has
      // written its share of the blob (bounded wait; the bulk copies read
      // through the async proxy what other SMs stored)
      uint32_t seen[MAXP / 32] = {0u, 0u, 0u};
      auto pulled = [&](int u) -> bool {
        if (!STG) return true;
        const int m = u - M.Uhit;
        if (m < 0 || m >= M.nmiss) return true;
        if ((seen[m >> 5] >> (m & 31)) & 1u) return true;
        spin_until(p.ready + m, G, p.err);
        if (ld_acquire(p.ready + m) < G) return false;
        asm volatile("fence.proxy.async.global;" ::: "memory");
        seen[m >> 5] |= 1u << (m & 31);
        return true;
      };
      auto acquire = [&](int slot_i) {
        const int s = slot_i % NSLOT;
        if (slot_i >= NSLOT &&
            !mbar_wait(&M.empty[s], ((slot_i / NSLOT) - 1) & 1, p.err))
          ok = false;
        return s;
      };
      for (; i < n_up; ++i) {
        const int v = b0 + i * G;
        const int s = acquire(i);
        if (!ok) break;
        const int u = v / nrt_f, rt = v % nrt_f;
        if (!pulled(u)) {
          ok = false;
          break;
        }
        const uint8_t* b = expert_base(p, M.active[u]);
        if (!b) { mbar_arrive_expect_tx(&M.full[s], 0); continue; }
        const uint32_t nb = (uint32_t)(nk * TBU);
        mbar_arrive_expect_tx(&M.full[s], 2 * nb);
        uint8_t* dst = ring + s * L.slot_bytes;
        bulk_g2s(dst, b + (int64_t)rt * nb, nb, &M.full[s]);
        bulk_g2s(dst + nb, b + p.gate_off + (int64_t)rt * nb, nb, &M.full[s]);
      }
      for (int v = d0; ok && v < d1; v += dps, ++i) {
        const int s = acquire(i);
        if (!ok) break;
        const int n = (d1 - v) < dps ? (d1 - v) : dps;
        for (int j = 0; j < n && ok; ++j) ok = pulled((v + j) / nrt_h);
        if (!ok) break;
        uint32_t tot = 0;
        const uint8_t* src[DNG];
        for (int j = 0; j < n; ++j) {
          const int uu = (v + j) / nrt_h, rt = (v + j) % nrt_h;
          const uint8_t* b = expert_base(p, M.active[uu]);
          src[j] = b ? b + p.down_off + (int64_t)rt * dnb : nullptr;
          if (src[j]) tot += (uint32_t)dnb;
        }
        mbar_arrive_expect_tx(&M.full[s], tot);
        for (int j = 0; j < n; ++j)
          if (src[j])
            bulk_g2s(ring + s * L.slot_bytes + j * dnb, src[j], (uint32_t)dnb,
                     &M.full[s]);
      }
      // Fills 0 .. i-1 were issued.  None may still be in flight when the
      // block exits (after a timed-out wait the compute warps stop waiting
      // for them), so wait -- bounded, and without the early give-up of
      // mbar_wait -- for the last fill of every slot to land.
      for (int s = 0; s < NSLOT && s < i; ++s) {
        const int last = s + ((i - 1 - s) / NSLOT) * NSLOT;
        if (!mbar_wait_drain(&M.full[s], (last / NSLOT) & 1))
          set_err(p.err, MOE_ERR_TIMEOUT);
      }
    }
    return;
  }

  // ---------------------------------------------------------- signaler --
  // Publishes this block's finished up units to the per-expert counters
  // (gpu-scope release), so that the compute warps never wait on a fence.
  if (warp == SIGNALER) {
    if (n_up > 0) {
      // lane l watches experts l, l + 32, l + 64 (U <= MAXP)
      int pub[MAXP / 32];
#pragma unroll
      for (int i = 0; i < MAXP / 32; ++i) pub[i] = 0;
      int left = n_up;
      const uint64_t t0 = globaltimer();
      while (left > 0) {
        int got = 0;
#pragma unroll
        for (int i = 0; i < MAXP / 32; ++i) {
          const int u = lane + 32 * i;
          if (u < U) {
            const int d = *reinterpret_cast<volatile int32_t*>(&M.up_fin[u]);
            if (d > pub[i]) {
              fence_acq_rel();
              atomicAdd(p.up_done + u, d - pub[i]);
              got += d - pub[i];
              pub[i] = d;
            }
          }
        }
        left -= __reduce_add_sync(0xffffffffu, (unsigned)got);
        if (left > 0) {
          __nanosleep(64);
          if (__any_sync(0xffffffffu, globaltimer() - t0 > 500000000ull)) {
            if (lane == 0) set_err(p.err, MOE_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
    return;
  }

  // ------------------------------------------------------- puller (STG) --
  // Copies this block's share (a contiguous 16-byte range) of every missed
  // blob from its pinned host copy into its slot, PULL_DEPTH loads in flight
  // per lane, and counts each finished share in ready[m] (release).  A missing
  // host copy or a slot outside the partition sets MOE_ERR_CAPACITY and the
  // share is skipped -- and still counted, so that no wait runs out.
  if (STG && warp == PULLER) {
    const int nm = M.nmiss;
    const int64_t words = p.blob_bytes / 16;
    const int64_t per = (words + G - 1) / G;
    const int64_t w0 = per * blockIdx.x;
    const int64_t w1 = w0 + per < words ? w0 + per : words;
    for (int m = 0; m < nm; ++m) {
      const int e = p.miss_expert[m];
      const int ls = p.miss_slot[m];
      const uint64_t src =
          (e >= 0 && e < E) ? p.stage_table[(int64_t)p.stage_layer * E + e]
                            : 0ull;
      const int64_t slot = (int64_t)p.slot_base + ls;
      if (src != 0ull && ls >= 0 && ls < p.n_slots && slot < p.pool_slots) {
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        uint4* d4 = reinterpret_cast<uint4*>(const_cast<uint8_t*>(p.pool) +
                                             slot * p.stride);
        for (int64_t i0 = w0 + lane; i0 < w1; i0 += 32 * PULL_DEPTH) {
          uint4 v[PULL_DEPTH];
#pragma unroll
          for (int u = 0; u < PULL_DEPTH; ++u)
            if (i0 + 32 * u < w1) v[u] = s4[i0 + 32 * u];
#pragma unroll
          for (int u = 0; u < PULL_DEPTH; ++u)
            if (i0 + 32 * u < w1) d4[i0 + 32 * u] = v[u];
        }
      } else if (lane == 0 && blockIdx.x == 0) {
        set_err(p.err, MOE_ERR_CAPACITY);
      }
      __syncwarp();
      if (lane == 0) {
        __threadfence();
        atomicAdd(p.ready + m, 1);
      }
    }
    return;
  }

  // ------------------------------------------------ up epilogue warps --
  // Warp UPEPI + ug, for each unit of up group ug: the group's partial
  // sums (eight warps) -> u, g of the unit's 16 rows for each of the
  // expert's pairs (lane o + 32i: pair slot o / 16, row o % 16); the buffer
  // is released before h = silu(g) * u goes to global memory, |h| max per
  // pair to hmax, and the unit is counted for the signaler.
  if (warp >= UPEPI) {
    const int ug = warp - UPEPI;
    const float* rb = red + ug * red_up_floats(NT);
    constexpr int OPL = TM / 2;   // outputs per lane: TM pairs x 16 rows
    for (int i = ug; i < n_up; i += UPG) {
      const int v = b0 + i * G;
      const int u = v / nrt_f, rt = v % nrt_f;
      const int pb = M.off[u], Tu = M.off[u + 1] - pb;
      named_bar_sync(BAR_RDY + ug, (UPW + 1) * 32);
      float su[OPL], sg[OPL];
      int pp[OPL];
#pragma unroll
      for (int i = 0; i < OPL; ++i) {
        const int o = lane + 32 * i, slot = o >> 4, rho = o & 15;
        su[i] = 0.f;
        sg[i] = 0.f;
        pp[i] = -1;
        if (slot < Tu) {
          pp[i] = M.sorted[pb + slot];
          const int t = pp[i] / k;
          const int Ln = 4 * (rho & 7) + (t & 3), nt = t >> 2, hh = rho >> 3;
#pragma unroll
          for (int w = 0; w < UPW; ++w) {
            su[i] += rb[(w * 32 + Ln) * NT * 4 + (nt * 2 + hh) * 2 + 0];
            sg[i] += rb[(w * 32 + Ln) * NT * 4 + (nt * 2 + hh) * 2 + 1];
          }
        }
      }
      named_bar_arrive(BAR_FREE + ug, (UPW + 1) * 32);
#pragma unroll
      for (int i = 0; i < OPL; ++i) {
        const int rho = lane & 15;
        float hv = 0.f;
        if (pp[i] >= 0) {
          hv = __fdividef(sg[i], 1.0f + __expf(-sg[i])) * su[i];
          p.h[(int64_t)pp[i] * F + 16 * rt + rho] = hv;
        }
        float m = fabsf(hv);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (rho == 0 && pp[i] >= 0)
          atomicMax(p.hmax + pp[i], __float_as_uint(m));
      }
      // the unit's h / hmax writes, then its count; the signaler releases
      // them at gpu scope
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        atomicAdd(&M.up_fin[u], 1);
      }
    }
    return;
  }

  // ------------------------------------------------------------ compute --
  const int c = lane & 3;
  int slot_i = 0;

  // P2: up/gate partial sums.  Group ug takes this block's units i with
  // i % 2 == ug; its epilogue warp finishes them (one partial-sum buffer
  // per group: written after the epilogue warp has read the previous
  // unit's).
  {
    const int ug = warp / UPW, wg = warp % UPW;
    float* rb = red + ug * red_up_floats(NT);
    int mine = 0;
    for (int i = 0; i < n_up; ++i, ++slot_i) {
      if ((i & 1) != ug) continue;            // the other group's unit
      const int s = slot_i % NSLOT;
      mbar_wait(&M.full[s], (slot_i / NSLOT) & 1, p.err);
      const uint8_t* unit = ring + s * L.slot_bytes;
      float au[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      float ag[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      for (int pc = wg; pc < 2 * nk; pc += UPW) {
        const int tz = pc / nk, kt = pc % nk;
        const uint8_t* tp = unit + pc * TBU;
        const uint32_t* xf = frag + kt * (TCU / 32) * NT * 64;
        const float* xb = xsc + (kt * TCU / XB_COLS) * DEC_TMAX;
        if (SBU) {
          const float xs2[2] = {xb[c], xb[4 + c]};
          if (tz == 0) piece_sbx<FUG>(tp, xf, NT, xs2, au, lane, NT);
          else piece_sbx<FUG>(tp, xf, NT, xs2, ag, lane, NT);
        } else {
          if (tz == 0) piece_b32<FUG>(tp, xf, NT, xb + c, 0, au, lane, NT);
          else piece_b32<FUG>(tp, xf, NT, xb + c, 0, ag, lane, NT);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_n(&M.empty[s], CW / UPW);
      if (mine > 0) named_bar_sync(BAR_FREE + ug, (UPW + 1) * 32);
      float* rw = rb + (wg * 32 + lane) * NT * 4;
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          rw[(nt * 2 + hh) * 2 + 0] = au[nt][hh];
          rw[(nt * 2 + hh) * 2 + 1] = ag[nt][hh];
        }
      named_bar_arrive(BAR_RDY + ug, (UPW + 1) * 32);
      ++mine;
    }
    if (mine > 0) named_bar_sync(BAR_FREE + ug, (UPW + 1) * 32);
  }

  // P3: B fragments of h for this block's down experts (at most two),
  // one scale per pair: 2^-sigma with sigma from max |h| of the pair
  const int uf = d1 > d0 ? d0 / nrt_h : 0;
  const int ul = d1 > d0 ? (d1 - 1) / nrt_h : -1;
  if (ul - uf > 1) set_err(p.err, MOE_ERR_DEVICE);
  const int nexp = ul - uf + 1 < 2 ? ul - uf + 1 : 2;
  const int hwords = (F / 32) * NT * 64;      // words per expert
  {
    // wait until every up unit of this block's down experts is done
    if (tid < nexp) spin_until(p.up_done + uf + tid, nrt_f, p.err);
    named_bar_sync(BAR_ALL, CW * 32);
    if (tid < 16) {
      const int b = tid >> 3, sl = tid & 7;
      float sc = 0.f;
      if (b < nexp) {
        const int u = uf + b;
        const int pb = M.off[u], Tu = M.off[u + 1] - pb;
        if (sl < Tu) {
          const int pp = M.sorted[pb + sl];
          sc = exp2i(-pow2_sigma(__uint_as_float(__ldcg(p.hmax + pp))));
        }
      }
      M.hsc[b][sl] = sc;
    }
    named_bar_sync(BAR_ALL, CW * 32);
    const int nent = (F / 32) * NT * 32;      // entries per expert
    for (int i = tid; i < nexp * nent; i += CW * 32) {
      const int b = i / nent, j = i % nent;
      const int Ln = j & 31, nt = (j >> 5) % NT, blk = j / (32 * NT);
      const int n = Ln >> 2, cc = Ln & 3;
      const int sl = 4 * nt + (n >> 1);
      const int u = uf + b;
      const int pb = M.off[u], Tu = M.off[u + 1] - pb;
      uint2 wv = make_uint2(0u, 0u);
      if (sl < Tu) {
        const int pp = M.sorted[pb + sl];
        const float sc = 1.0f / M.hsc[b][sl];
        const float* hr = p.h + (int64_t)pp * F + 32 * blk + 4 * cc;
        const float4 ha = __ldcg(reinterpret_cast<const float4*>(hr));
        const float4 hb = __ldcg(reinterpret_cast<const float4*>(hr + 16));
        const float va[4] = {ha.x, ha.y, ha.z, ha.w};
        const float vb[4] = {hb.x, hb.y, hb.z, hb.w};
        wv.x = frag_word(va, sc, n & 1);
        wv.y = frag_word(vb, sc, n & 1);
      }
      reinterpret_cast<uint2*>(frag + b * hwords)[j] = wv;
    }
    named_bar_sync(BAR_ALL, CW * 32);
  }

  // P4: down projection.  Slot = up to DNG units; group dg takes unit dg.
  {
    const int dg = warp / DNW, wd = warp % DNW;
    const int gtid = tid - dg * DNW * 32;
    const int rfl = red_dn_floats(NT);
    const int kt0 = wd * nkd / DNW, kt1 = (wd + 1) * nkd / DNW;
    int it = 0;
    for (int v = d0; v < d1; v += dps, ++slot_i) {
      const int n = (d1 - v) < dps ? (d1 - v) : dps;
      const bool have = dg < n;               // a unit for this group?
      const int s = slot_i % NSLOT;
      mbar_wait(&M.full[s], (slot_i / NSLOT) & 1, p.err);
      const int u = (v + dg) / nrt_h, rt = (v + dg) % nrt_h;
      const int b = u - uf;
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      if (have && b >= 0 && b < nexp) {
        const uint8_t* unit = ring + s * L.slot_bytes + dg * dnb;
#pragma unroll 4
        for (int kt = kt0; kt < kt1; ++kt)
          piece_b32<FDN>(unit + kt * B32_TILE_BYTES,
                         frag + b * hwords + (2 * kt) * NT * 64, NT,
                         &M.hsc[b][c], 0, acc, lane, NT);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.empty[s]);   // all CW warps use a slot
      if (!have) continue;
      ++it;
      float* rb = red + (dg * 2 + (it & 1)) * rfl;   // it counts this group's units
      float* rw = rb + (wd * 32 + lane) * NT * 2;
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) rw[nt * 2 + hh] = acc[nt][hh];
      named_bar_sync(BAR_DN + dg, DNW * 32);
      {
        const int pb = M.off[u], Tu = M.off[u + 1] - pb;
        const int sl = gtid >> 4, rho = gtid & 15;   // gtid < 128
        if (sl < Tu && b >= 0 && b < nexp) {
          const int Ln = 4 * (rho & 7) + (sl & 3), nt = sl >> 2;
          const int hh = rho >> 3;
          float yv = 0.f;
#pragma unroll
          for (int w = 0; w < DNW; ++w)
            yv += rb[(w * 32 + Ln) * NT * 2 + nt * 2 + hh];
          const int pp = M.sorted[pb + sl];
          p.y[(int64_t)pp * H + 16 * rt + rho] = yv;
        }
      }
    }
  }

  grid_barrier(p, 2);
  // the next kernel on the stream may start its launch (it waits for this
  // one to finish before it reads or writes global memory)
  grid_dep_launch();

  // P5: combine (not in DL_ROUTE), then the exit count that re-arms the
  // grid barrier
  if (p.mode != DL_ROUTE) {
    const int64_t n = (int64_t)T * H;
    const int64_t i0 = n * blockIdx.x / G, i1 = n * (blockIdx.x + 1) / G;
    for (int64_t i = i0 + tid; i < i1; i += CW * 32) {
      const int t = (int)(i / H), col = (int)(i % H);
      float a = 0.f;
      for (int j = 0; j < k; ++j)
        a = fmaf(M.tk_w[t * k + j], __ldcg(p.y + ((int64_t)t * k + j) * H + col),
                 a);
      if (p.residual) a += p.residual[i];
      p.out[i] = a;
      if (p.out_bf16) p.out_bf16[i] = f32_to_bf16_rne(a);
    }
  }
  named_bar_sync(BAR_ALL, CW * 32);
  if (tid == 0) {
    fence_acq_rel();
    M.flag = atomicAdd(p.bar + 1, 1) == G - 1;
  }
  named_bar_sync(BAR_ALL, CW * 32);
  if (M.flag) {   // last block out: re-arm the counters for the next call
    for (int i = tid; i < U; i += CW * 32) p.up_done[i] = 0;
    if (STG)
      for (int i = tid; i < M.nmiss; i += CW * 32) p.ready[i] = 0;
    if (tid == 0) {
      p.bar[0] = 0;
      p.bar[1] = 0;
    }
  }
}

// ---------------------------------------------------------------- host --
bool decode_layer_supported(const moe_layer_desc& d, int T, int k) {
  if (T < 1 || T > DEC_TMAX || T * k > MAXP || k > 32) return false;
  if (d.E > EMAX_FUSED) return false;
  if (d.fmt_down != MOE_NL4_B32 && d.fmt_down != MOE_Q4_B32) return false;
  if (d.F % 64 || d.H % 64) return false;
  if (T * k > num_sms()) return false;
  const Smem L = smem_layout(d.fmt_up_gate, d.H, d.F, T);
  if (L.total > 227 * 1024) return false;
  if ((int64_t)T * d.H * 2 > NSLOT * L.slot_bytes) return false;
  return (int)sizeof(Misc) <= 3072;
}

size_t decode_layer_ws_bytes(int T, int k, int H, int F) {
  const size_t P = (size_t)T * k;
  return 1024 + ((P * F * 4 + 255) & ~(size_t)255) +
         ((P * 4 + 255) & ~(size_t)255) + ((P * H * 4 + 255) & ~(size_t)255);
}

moe_status launch_decode_layer(const moe_layer_desc& d, const uint16_t* x,
                               const float* r_in, int T, int k,
                               const uint16_t* wr, const float* bias,
                               const int32_t* blob_index,
                               const float* residual, float* out,
                               uint16_t* out_bf16, int32_t* topk_idx,
                               float* topk_w, float* logits, void* ws,
                               int32_t* err, cudaStream_t s, int mode,
                               const StageArgs* stg) {
  LayerParams p;
  p.mode = mode;
  p.pool = d.pool;
  p.stride = d.blob_stride;
  p.blob_index = blob_index;
  p.E = d.E;
  p.H = d.H;
  p.F = d.F;
  p.T = T;
  p.k = k;
  p.gate_off = tensor_bytes_of(d.fmt_up_gate, d.F, d.H);
  p.down_off = 2 * p.gate_off;
  p.x = x;
  p.r_in = r_in;
  p.wr = wr;
  p.bias = bias;
  p.topk_idx = topk_idx;
  p.topk_w = topk_w;
  p.logits = logits;
  p.residual = residual;
  p.out = out;
  p.out_bf16 = out_bf16;
  uint8_t* b = static_cast<uint8_t*>(ws);
  const size_t P = (size_t)T * k;
  p.bar = reinterpret_cast<int32_t*>(b);
  p.up_done = reinterpret_cast<int32_t*>(b + 64);
  b += 1024;
  p.h = reinterpret_cast<float*>(b);
  b += (P * d.F * 4 + 255) & ~(size_t)255;
  p.hmax = reinterpret_cast<uint32_t*>(b);
  b += (P * 4 + 255) & ~(size_t)255;
  p.y = reinterpret_cast<float*>(b);
  p.err = err;
  p.n_miss = stg ? stg->n_miss : nullptr;
  p.miss_expert = stg ? stg->miss_expert : nullptr;
  p.miss_slot = stg ? stg->miss_slot : nullptr;
  p.stage_table = stg ? stg->table : nullptr;
  p.stage_layer = stg ? stg->layer : 0;
  p.slot_base = stg ? stg->slot_base : 0;
  p.n_slots = stg ? stg->n_slots : 0;
  p.pool_slots = stg ? stg->pool_slots : 0;
  p.blob_bytes = stg ? stg->blob_bytes : 0;
  p.ready = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + 512);
  const Smem L = smem_layout(d.fmt_up_gate, d.H, d.F, T);
  void (*kern)(LayerParams) = nullptr;
  const bool q4d = d.fmt_down == MOE_Q4_B32;
  const bool two = T > 4;
  const bool wide = d.E > 512;
#define MOE_K(FU, FD, NTT, EPLV)                                            \
  (stg ? decode_layer_kernel<FU, FD, NTT, EPLV, true>                        \
       : decode_layer_kernel<FU, FD, NTT, EPLV, false>)
#define MOE_PICK2(FU, FD, NTT)                                               \
  (wide ? MOE_K(FU, FD, NTT, 32) : MOE_K(FU, FD, NTT, 16))
#define MOE_PICK(FU)                                                        \
  kern = q4d ? (two ? MOE_PICK2(FU, MOE_Q4_B32, 2)                          \
                    : MOE_PICK2(FU, MOE_Q4_B32, 1))                         \
             : (two ? MOE_PICK2(FU, MOE_NL4_B32, 2)                         \
                    : MOE_PICK2(FU, MOE_NL4_B32, 1))
  switch (d.fmt_up_gate) {
    case MOE_SB3_256: MOE_PICK(MOE_SB3_256); break;
    case MOE_NL3_256: MOE_PICK(MOE_NL3_256); break;
    case MOE_SB2_256: MOE_PICK(MOE_SB2_256); break;
    case MOE_NL4_B32: MOE_PICK(MOE_NL4_B32); break;
    default: MOE_PICK(MOE_Q4_B32);
  }
#undef MOE_PICK
#undef MOE_PICK2
#undef MOE_K
  moe_status st = ensure_smem((const void*)kern, (size_t)L.total);
  if (st != MOE_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(stg ? LAYER_THREADS_STG : LAYER_THREADS);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, p));
  return MOE_OK;
}

}  // namespace moe
