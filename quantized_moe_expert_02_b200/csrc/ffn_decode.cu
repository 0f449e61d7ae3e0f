// Expert FFN, decode path (T <= 8 tokens): fused dequant-GEMV on the int8
// tensor-core path.  HBM-bound: every expert byte is read once.
//
// Structure (both kernels): a persistent grid of one block per SM; warp 8
// is a producer that streams packed expert tiles global -> shared memory
// with 1-D bulk copies (cp.async.bulk) into a ring of stages guarded by
// mbarriers; warps 0..7 are two consumer groups of four warps that take
// alternate units.  A consumer turns the codes of its tile into the int8
// A fragment of mma.m16n8k32 with byte-table lookups (prmt), and the
// activations enter as the B fragment split into two int8 halves
// (v = 256*hi + lo, v = round(a * 2^sigma), |v| < 2^14, with one sigma per
// token and 256-column block of x), so the products
// and their sums over a 32-block are exact integers.  Scales are applied
// in fp32 per block (per super-block for SB3, whose sub-scales multiply
// the integer partials).
//
// Up/gate kernel: unit = (expert, 32 rows of F, quarter of H).  Its four
// chunks (up/gate x two 16-row tiles) go to the four warps of a group.  The
// partials of the quarters are summed in fixed order by whichever block
// finishes a 32-row tile last (arrival counter), which applies SwiGLU and
// writes h of each of the expert's tokens as the int8 B fragments of the
// down projection (one scale per token and 32-block).
//
// Down kernel: unit = (expert, 16 rows of H), all of F; the four warps of
// a group split F.  y of each pair is written per row tile; with the fused
// combine, the block that finishes a row tile last (over all experts) sums
// the k expert outputs of each token in j order.
#include "decode_pieces.cuh"

namespace moe {

constexpr int NGRP = 2;                    // consumer groups
constexpr int GRP_WARPS = 4;               // warps per group
constexpr int DEC_THREADS = (NGRP * GRP_WARPS + 1) * 32;
constexpr int PROD_WARP = NGRP * GRP_WARPS;
constexpr int UP_STAGES = 4;
constexpr int DN_STAGES = 8;

struct DecParams {
  const uint8_t* pool;
  int64_t stride;
  const int32_t* blob_index;
  int E, H, F, T, k;
  int64_t gate_off, down_off;
  const uint16_t* x;
  const int32_t* offsets;
  const int32_t* pair_ids;
  const int32_t* active;
  const int32_t* n_active;
  int32_t* err;
  int32_t* up_cnt;
  int32_t* dn_cnt;
  float* up_part;
  uint32_t* bfrag;
  float* bscale;
  float* y;               // y of each pair [T*k][H]
  const float* topk_w;    // fused combine (out != nullptr)
  const float* residual;
  float* out;
  uint16_t* out_bf16;
};

__device__ __forceinline__ const uint8_t* blob_of(const DecParams& p, int e) {
  if (e < 0 || e >= p.E) { set_err(p.err, MOE_ERR_DEVICE); return nullptr; }
  const int64_t b = p.blob_index ? (int64_t)__ldcg(p.blob_index + e) : e;
  if (b < 0) { set_err(p.err, MOE_ERR_DEVICE); return nullptr; }
  return p.pool + b * p.stride;
}

// ---------------------------------------------------------------- up ---
template <int FMT>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    ffn_up_decode_kernel(DecParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr bool SBF = FMT == MOE_SB3_256 || FMT == MOE_NL3_256 ||
                      FMT == MOE_SB2_256;
  constexpr int TB = FMT == MOE_SB3_256   ? SB3_TILE_BYTES
                     : FMT == MOE_NL3_256 ? NL3_TILE_BYTES
                     : FMT == MOE_SB2_256 ? SB2_TILE_BYTES
                                          : B32_TILE_BYTES;
  constexpr int TC = SBF ? SB3_TILE_COLS : B32_TILE_COLS;
  const int nk = p.H / TC;
  const int nsplit = nk < NSPLIT_MAX ? nk : NSPLIT_MAX;
  const int kmax = (nk + nsplit - 1) / nsplit;
  const int chunk_bytes = kmax * TB;
  const int stage_bytes = 4 * chunk_bytes;
  const int NT = (p.T + 3) / 4;
  const int nblk = p.H / 32;
  const int nrt = p.F / 32;
  uint8_t* stages = smem;
  uint32_t* xf = reinterpret_cast<uint32_t*>(smem + UP_STAGES * stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(xf + nblk * BF_NT * 64);
  uint64_t* empty = full + UP_STAGES;
  // activation scales per (256-column block, token): [nxb][8]
  const int nxb = (p.H + XB_COLS - 1) / XB_COLS;
  float* xsc = reinterpret_cast<float*>(empty + UP_STAGES);
  int* xsig = reinterpret_cast<int*>(xsc + nxb * DEC_TMAX);
  int* flag = xsig + nxb * DEC_TMAX;                         // [NGRP]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < UP_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], GRP_WARPS);
    }
    fence_mbar_init();
  }
  // scale of the activations per token and 256-column block (x is an
  // input of this layer): one warp per (token, block), a lane per 8 values
  for (int item = warp; item < p.T * nxb; item += DEC_THREADS / 32) {
    const int t = item / nxb, b = item % nxb;
    const int h0 = b * XB_COLS + 8 * lane;
    float m = 0.f;
    if (h0 < p.H) {
      const uint4 v =
          *reinterpret_cast<const uint4*>(p.x + (int64_t)t * p.H + h0);
      m = absmax8_bf16(v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      const int s = pow2_sigma(m);
      xsig[b * DEC_TMAX + t] = s;
      xsc[b * DEC_TMAX + t] =
          exp2i(-s) * fmt_xfold(FMT);
    }
  }
  __syncthreads();
  // B fragments of x: [blk][nt][lane][reg], 4 int8 of column n = g:
  // token 4nt + n/2, n even = high half, odd = low half of v.
  for (int i = tid; i < nblk * BF_NT * 64; i += DEC_THREADS) {
    const int reg = i & 1, L = (i >> 1) & 31, nt = (i >> 6) % BF_NT;
    const int blk = i / (64 * BF_NT);
    const int n = L >> 2, c = L & 3;
    const int t = 4 * nt + (n >> 1);
    uint32_t word = 0;
    if (t < p.T) {
      const float sc = exp2i(xsig[(32 * blk / XB_COLS) * DEC_TMAX + t]);
      const uint16_t* xr = p.x + (int64_t)t * p.H + 32 * blk + 16 * reg + 4 * c;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int v = __float2int_rn(bf16_to_f32(xr[q]) * sc);
        const int hi = (v + 128) >> 8, lo = v - hi * 256;
        word |= (uint32_t)((n & 1) ? lo : hi) << (8 * q) & (0xFFu << (8 * q));
      }
    }
    xf[i] = word;
  }
  __syncthreads();
  grid_dep_wait();      // routing of this layer is complete and visible
  grid_dep_launch();

  const int n_act = *p.n_active;
  const int64_t n_units = (int64_t)n_act * nrt * nsplit;
  const int64_t v0 = n_units * blockIdx.x / gridDim.x;
  const int64_t v1 = n_units * (blockIdx.x + 1) / gridDim.x;
  const int nu = (int)(v1 - v0);

  if (warp == PROD_WARP) {
    if (lane == 0) {
      for (int i = 0; i < nu; ++i) {
        const int s = i % UP_STAGES;
        if (i >= UP_STAGES)
          mbar_wait(&empty[s], ((i / UP_STAGES) - 1) & 1, p.err);
        const int64_t v = v0 + i;
        const int u = (int)(v / (nrt * nsplit));
        const int rt = (int)((v / nsplit) % nrt), kq = (int)(v % nsplit);
        const int k0 = kq * nk / nsplit, k1 = (kq + 1) * nk / nsplit;
        const uint32_t nbytes = (uint32_t)((k1 - k0) * TB);
        const uint8_t* blob = blob_of(p, p.active[u]);
        if (!blob) { mbar_arrive_expect_tx(&full[s], 0); continue; }
        mbar_arrive_expect_tx(&full[s], 4 * nbytes);
        for (int w = 0; w < 4; ++w) {
          const int tz = w >> 1, rg = w & 1;
          const uint8_t* src = blob + tz * p.gate_off +
                               ((int64_t)(2 * rt + rg) * nk + k0) * TB;
          bulk_g2s(stages + s * stage_bytes + w * chunk_bytes, src, nbytes,
                   &full[s]);
        }
      }
    }
    return;
  }

  const int grp = warp / GRP_WARPS, wg = warp % GRP_WARPS;
  const int gtid = tid - grp * GRP_WARPS * 32;   // 0..127 within the group
  const int tz = wg >> 1, rg = wg & 1;
  const int g = lane >> 2, c = lane & 3;
  for (int i = grp; i < nu; i += NGRP) {
    const int s = i % UP_STAGES;
    mbar_wait(&full[s], (i / UP_STAGES) & 1, p.err);
    const int64_t v = v0 + i;
    const int u = (int)(v / (nrt * nsplit));
    const int rt = (int)((v / nsplit) % nrt), kq = (int)(v % nsplit);
    const int k0 = kq * nk / nsplit, k1 = (kq + 1) * nk / nsplit;
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    const uint8_t* chunk = stages + s * stage_bytes + wg * chunk_bytes;
    for (int kt = 0; kt < k1 - k0; ++kt) {
      const int blk0 = (k0 + kt) * (TC / 32);
      const float* xb = xsc + ((k0 + kt) * TC / XB_COLS) * DEC_TMAX;
      if (SBF) {
        const float xs[2] = {xb[c], xb[4 + c]};
        piece_sbx<FMT>(chunk + kt * TB,
                                      xf + blk0 * BF_NT * 64, NT, xs, acc,
                                      lane, BF_NT);
      } else {
        piece_b32<FMT>(chunk + kt * TB, xf + blk0 * BF_NT * 64, NT, xb + c,
                       0, acc, lane);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    // split-K partial of this quarter
    float* part = p.up_part +
                  ((((int64_t)u * nrt + rt) * NSPLIT_MAX + kq) * 2 + tz) * 256;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int t = 4 * nt + c;
      if (t < p.T) {
        part[(rg * 16 + g) * 8 + t] = acc[nt][0];
        part[(rg * 16 + g + 8) * 8 + t] = acc[nt][1];
      }
    }
    __threadfence();
    named_bar_sync(1 + grp, GRP_WARPS * 32);
    if (gtid == 0) {
      const int old = atomicAdd(&p.up_cnt[u * nrt + rt], 1);
      flag[grp] = (old == nsplit - 1);
    }
    named_bar_sync(1 + grp, GRP_WARPS * 32);
    if (flag[grp]) {
      __threadfence();
      // finalize the 32-row tile: SwiGLU, then the down B fragments
      const int e = p.active[u];
      const int off = p.offsets[e], Tu = p.offsets[e + 1] - off;
      const int slot = gtid >> 4, r0 = (gtid & 15) * 2;
      float hv[2] = {0.f, 0.f};
      if (slot < Tu) {
        const int pp = p.pair_ids[off + slot];
        const int t = pp / p.k;
        const float* pb = p.up_part +
                          (((int64_t)u * nrt + rt) * NSPLIT_MAX) * 2 * 256;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int r = r0 + q;
          float su = 0.f, sg = 0.f;
          for (int kk = 0; kk < nsplit; ++kk) {
            su += __ldcg(pb + (kk * 2 + 0) * 256 + r * 8 + t);
            sg += __ldcg(pb + (kk * 2 + 1) * 256 + r * 8 + t);
          }
          hv[q] = sg / (1.0f + expf(-sg)) * su;
        }
      }
      float m = fmaxf(fabsf(hv[0]), fabsf(hv[1]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int sig = pow2_sigma(m);
      const float sc = exp2i(sig);
      uint8_t* bf8 = reinterpret_cast<uint8_t*>(p.bfrag);
      const int nt = slot >> 2, nhi = 2 * (slot & 3);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int r = r0 + q;
        const int vq = slot < Tu ? __float2int_rn(hv[q] * sc) : 0;
        const int hi = (vq + 128) >> 8, lo = vq - hi * 256;
        const int cc = (r & 15) >> 2, reg = r >> 4, byte = r & 3;
        const int64_t base =
            (((int64_t)u * nrt + rt) * BF_NT + nt) * 32 * 8 + reg * 4 + byte;
        bf8[base + (4 * nhi + cc) * 8] = (uint8_t)hi;
        bf8[base + (4 * (nhi + 1) + cc) * 8] = (uint8_t)lo;
      }
      if ((gtid & 15) == 0)
        p.bscale[((int64_t)u * nrt + rt) * 8 + slot] = exp2i(-sig);
      if (gtid == 0) p.up_cnt[u * nrt + rt] = 0;
    }
  }
}

// -------------------------------------------------------------- down ---
template <int FMT>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    ffn_down_decode_kernel(DecParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int nk = p.F / B32_TILE_COLS;
  const int nrt = p.H / TILE_ROWS;
  const int nblk = p.F / 32;
  const int stage_bytes = nk * B32_TILE_BYTES;
  const int NT = (p.T + 3) / 4;
  const int bwords = nblk * BF_NT * 64;
  uint8_t* stages = smem;
  uint32_t* bbuf = reinterpret_cast<uint32_t*>(smem + DN_STAGES * stage_bytes);
  float* bsc = reinterpret_cast<float*>(bbuf + 2 * bwords);     // [2][nblk*8]
  float* red = bsc + 2 * nblk * 8;                 // [NGRP][4][2][2][32]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + NGRP * 4 * 2 * 2 * 32);
  uint64_t* empty = full + DN_STAGES;
  uint64_t* bfull = empty + DN_STAGES;
  int* flag = reinterpret_cast<int*>(bfull + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < DN_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], GRP_WARPS);
    }
    mbar_init(bfull, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // The routing (two launches back) is complete: the up kernel waited for
  // it before it allowed this grid to start.  Read it through L2.
  const int n_act = __ldcg(p.n_active);
  const int64_t n_units = (int64_t)n_act * nrt;
  const int64_t v0 = n_units * blockIdx.x / gridDim.x;
  const int64_t v1 = n_units * (blockIdx.x + 1) / gridDim.x;
  const int nu = (int)(v1 - v0);
  const int u_first = nu > 0 ? (int)(v0 / nrt) : 0;
  const int u_last = nu > 0 ? (int)((v1 - 1) / nrt) : -1;

  if (warp == PROD_WARP) {
    if (lane == 0) {
      auto issue = [&](int i) {
        const int s = i % DN_STAGES;
        const int64_t v = v0 + i;
        const int u = (int)(v / nrt), rt = (int)(v % nrt);
        const uint8_t* blob = blob_of(p, __ldcg(p.active + u));
        if (!blob) { mbar_arrive_expect_tx(&full[s], 0); return; }
        mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
        bulk_g2s(stages + s * stage_bytes,
                 blob + p.down_off + (int64_t)rt * stage_bytes,
                 (uint32_t)stage_bytes, &full[s]);
      };
      const int pre = nu < DN_STAGES ? nu : DN_STAGES;
      for (int i = 0; i < pre; ++i) issue(i);
      grid_dep_wait();    // the up kernel's B fragments are complete
      grid_dep_launch();
      if (u_last >= u_first && u_last - u_first <= 1) {
        const uint32_t nb = (uint32_t)(bwords * 4 + nblk * 8 * 4);
        mbar_arrive_expect_tx(bfull, (u_last - u_first + 1) * nb);
        for (int u = u_first; u <= u_last; ++u) {
          const int bi = u - u_first;
          bulk_g2s(bbuf + bi * bwords, p.bfrag + (int64_t)u * bwords,
                   (uint32_t)(bwords * 4), bfull);
          bulk_g2s(bsc + bi * nblk * 8, p.bscale + (int64_t)u * nblk * 8,
                   (uint32_t)(nblk * 8 * 4), bfull);
        }
      } else {
        if (u_last - u_first > 1) set_err(p.err, MOE_ERR_DEVICE);
        mbar_arrive_expect_tx(bfull, 0);
      }
      for (int i = pre; i < nu; ++i) {
        const int s = i % DN_STAGES;
        mbar_wait(&empty[s], ((i / DN_STAGES) - 1) & 1, p.err);
        issue(i);
      }
    }
    return;
  }

  grid_dep_wait();
  const int grp = warp / GRP_WARPS, wg = warp % GRP_WARPS;
  const int gtid = tid - grp * GRP_WARPS * 32;
  const int c = lane & 3;
  mbar_wait(bfull, 0, p.err);
  const int kt0 = wg * nk / GRP_WARPS, kt1 = (wg + 1) * nk / GRP_WARPS;
  float* myred = red + grp * (4 * 2 * 2 * 32);
  for (int i = grp; i < nu; i += NGRP) {
    const int s = i % DN_STAGES;
    mbar_wait(&full[s], (i / DN_STAGES) & 1, p.err);
    const int64_t v = v0 + i;
    const int u = (int)(v / nrt), rt = (int)(v % nrt);
    const int bi = u - u_first;
    const bool bok = bi >= 0 && bi <= 1;
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    if (bok) {
      const uint32_t* bb = bbuf + bi * bwords;
      const float* bs = bsc + bi * nblk * 8;
      for (int kt = kt0; kt < kt1; ++kt)
        piece_b32<FMT>(stages + s * stage_bytes + kt * B32_TILE_BYTES,
                       bb + (2 * kt) * BF_NT * 64, NT, bs + (2 * kt) * 8 + c,
                       8, acc, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        myred[((wg * 2 + nt) * 2 + h) * 32 + lane] = acc[nt][h];
    named_bar_sync(1 + grp, GRP_WARPS * 32);
    {
      const int rho = gtid >> 3, slot = gtid & 7;
      const int L = 4 * (rho & 7) + (slot & 3), nt = slot >> 2, h = rho >> 3;
      float yv = 0.f;
#pragma unroll
      for (int w = 0; w < GRP_WARPS; ++w)
        yv += myred[((w * 2 + nt) * 2 + h) * 32 + L];
      const int e = __ldcg(p.active + u);
      const int off = __ldcg(p.offsets + e);
      const int Tu = __ldcg(p.offsets + e + 1) - off;
      if (slot < Tu && bok) {
        const int pp = __ldcg(p.pair_ids + off + slot);
        p.y[(int64_t)pp * p.H + 16 * rt + rho] = yv;
      }
    }
    if (p.out) {
      __threadfence();
      named_bar_sync(1 + grp, GRP_WARPS * 32);
      if (gtid == 0) {
        const int old = atomicAdd(&p.dn_cnt[rt], 1);
        flag[grp] = (old == n_act - 1);
      }
      named_bar_sync(1 + grp, GRP_WARPS * 32);
      if (flag[grp]) {
        __threadfence();
        const int t = gtid >> 4, rho = gtid & 15;
        if (t < p.T) {
          const int64_t col = 16 * rt + rho;
          float a = 0.f;
          for (int j = 0; j < p.k; ++j) {
            const int64_t pp = (int64_t)t * p.k + j;
            a = fmaf(p.topk_w[pp], __ldcg(p.y + pp * p.H + col), a);
          }
          if (p.residual) a += p.residual[(int64_t)t * p.H + col];
          p.out[(int64_t)t * p.H + col] = a;
          if (p.out_bf16) p.out_bf16[(int64_t)t * p.H + col] = f32_to_bf16_rne(a);
        }
        if (gtid == 0) p.dn_cnt[rt] = 0;
      }
    }
    named_bar_sync(1 + grp, GRP_WARPS * 32);
  }
}

// ------------------------------------------------------------ launch ---
static size_t up_smem_bytes(int fmt, int H) {
  const int TB = tile_bytes(fmt), TC = tile_cols(fmt);
  const int nk = H / TC;
  const int nsplit = nk < NSPLIT_MAX ? nk : NSPLIT_MAX;
  const int kmax = (nk + nsplit - 1) / nsplit;
  const int nxb = (H + XB_COLS - 1) / XB_COLS;
  return (size_t)UP_STAGES * 4 * kmax * TB + (size_t)(H / 32) * BF_NT * 64 * 4 +
         2 * UP_STAGES * 8 + (size_t)2 * nxb * DEC_TMAX * 4 + 64;
}
static size_t dn_smem_bytes(int F) {
  const int nk = F / B32_TILE_COLS, nblk = F / 32;
  return (size_t)DN_STAGES * nk * B32_TILE_BYTES +
         (size_t)2 * nblk * BF_NT * 64 * 4 + (size_t)2 * nblk * 8 * 4 +
         (size_t)NGRP * 4 * 2 * 2 * 32 * 4 + (2 * DN_STAGES + 1) * 8 + 64;
}

bool ffn_decode_supported(const moe_layer_desc& d, int T, int k) {
  if (T < 1 || T > DEC_TMAX) return false;
  if (d.fmt_down != MOE_NL4_B32 && d.fmt_down != MOE_Q4_B32) return false;
  if (d.F % 32 != 0 || d.H % 16 != 0) return false;
  if ((int64_t)T * k > num_sms()) return false;
  if (up_smem_bytes(d.fmt_up_gate, d.H) > 220 * 1024) return false;
  if (dn_smem_bytes(d.F) > 220 * 1024) return false;
  return true;
}

template <typename K>
static moe_status launch_pdl(K kernel, int grid, size_t smem, cudaStream_t s,
                             bool pdl, const DecParams& prm) {
  const moe_status st = ensure_smem((const void*)kernel, smem);
  if (st != MOE_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, kernel, prm));
  return MOE_OK;
}

static DecParams make_params(const moe_layer_desc& d, const uint16_t* x,
                             int T, int k, const int32_t* offsets,
                             const int32_t* pair_ids, const int32_t* active,
                             const int32_t* n_active,
                             const int32_t* blob_index, const FfnWs& ws,
                             float* y, const float* topk_w,
                             const float* residual, float* out,
                             uint16_t* out_bf16) {
  DecParams prm;
  prm.pool = d.pool;
  prm.stride = d.blob_stride;
  prm.blob_index = blob_index;
  prm.E = d.E;
  prm.H = d.H;
  prm.F = d.F;
  prm.T = T;
  prm.k = k;
  prm.gate_off = tensor_bytes_of(d.fmt_up_gate, d.F, d.H);
  prm.down_off = 2 * prm.gate_off;
  prm.x = x;
  prm.offsets = offsets;
  prm.pair_ids = pair_ids;
  prm.active = active;
  prm.n_active = n_active;
  prm.err = ws.err;
  prm.up_cnt = ws.up_cnt;
  prm.dn_cnt = ws.dn_cnt;
  prm.up_part = ws.up_part;
  prm.bfrag = ws.bfrag;
  prm.bscale = ws.bscale;
  prm.y = y;
  prm.topk_w = topk_w;
  prm.residual = residual;
  prm.out = out;
  prm.out_bf16 = out_bf16;
  return prm;
}

moe_status launch_up_decode(const moe_layer_desc& d, const uint16_t* x,
                            int T, int k, const int32_t* offsets,
                            const int32_t* pair_ids, const int32_t* active,
                            const int32_t* n_active, const int32_t* blob_index,
                            const FfnWs& ws, cudaStream_t s, bool pdl) {
  const DecParams prm =
      make_params(d, x, T, k, offsets, pair_ids, active, n_active, blob_index,
                  ws, nullptr, nullptr, nullptr, nullptr, nullptr);
  const int grid = num_sms();
  const size_t su = up_smem_bytes(d.fmt_up_gate, d.H);
  switch (d.fmt_up_gate) {
    case MOE_SB3_256:
      return launch_pdl(ffn_up_decode_kernel<MOE_SB3_256>, grid, su, s, pdl,
                        prm);
    case MOE_NL4_B32:
      return launch_pdl(ffn_up_decode_kernel<MOE_NL4_B32>, grid, su, s, pdl,
                        prm);
    case MOE_NL3_256:
      return launch_pdl(ffn_up_decode_kernel<MOE_NL3_256>, grid, su, s, pdl,
                        prm);
    case MOE_SB2_256:
      return launch_pdl(ffn_up_decode_kernel<MOE_SB2_256>, grid, su, s, pdl,
                        prm);
    default:
      return launch_pdl(ffn_up_decode_kernel<MOE_Q4_B32>, grid, su, s, pdl,
                        prm);
  }
}

moe_status launch_down_decode(const moe_layer_desc& d, int T, int k,
                              const int32_t* offsets, const int32_t* pair_ids,
                              const int32_t* active, const int32_t* n_active,
                              const int32_t* blob_index, const FfnWs& ws,
                              float* y, const float* topk_w,
                              const float* residual, float* out,
                              uint16_t* out_bf16, cudaStream_t s, bool pdl) {
  const DecParams prm =
      make_params(d, nullptr, T, k, offsets, pair_ids, active, n_active,
                  blob_index, ws, y, topk_w, residual, out, out_bf16);
  const int grid = num_sms();
  const size_t sd = dn_smem_bytes(d.F);
  if (d.fmt_down == MOE_NL4_B32)
    return launch_pdl(ffn_down_decode_kernel<MOE_NL4_B32>, grid, sd, s, pdl,
                      prm);
  return launch_pdl(ffn_down_decode_kernel<MOE_Q4_B32>, grid, sd, s, pdl, prm);
}

}  // namespace moe
