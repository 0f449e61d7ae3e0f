// Device twin of synth/__init__.py: draws the natural-layout bytes of
// expert tensors from the same counter-based SplitMix64 streams, so that
// multi-gigabyte expert pools can be generated where they are used.  It
// holds no part of the layer's arithmetic.  Must produce exactly the bytes
// the host generator produces (checked by a GPU test).
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t GAMMA = 0x9E3779B97F4A7C15ull;
constexpr uint64_t MUL1 = 0xBF58476D1CE4E5B9ull;
constexpr uint64_t MUL2 = 0x94D049BB133111EBull;
constexpr uint64_t KEY0 = 0x243F6A8885A308D3ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * MUL1;
  z = (z ^ (z >> 27)) * MUL2;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, uint64_t layer,
                                               uint64_t expert, uint64_t tensor,
                                               uint64_t plane) {
  uint64_t k = KEY0;
  const uint64_t f[5] = {seed, layer, expert, tensor, plane};
  for (int i = 0; i < 5; ++i) k = mix64((k ^ f[i]) + GAMMA);
  return k;
}

__device__ inline uint64_t word(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * GAMMA);
}

struct Plane {
  int64_t offset;   // byte offset in the tensor
  int64_t bytes;
  int id;           // 0 codes, 1 scales, 2 d, 3 extra (NL3)
};

struct TensorSpec {
  Plane planes[4];
  int nplanes;
  int64_t bytes;
  int tensor_id;
  double lo, hi;
};

// One grid-stride pass over chunks of CW generator words of one tensor kind
// (the stream key is computed once per chunk).
constexpr int CW = 32;

__device__ inline int64_t plane_words(const Plane& pl) {
  return pl.id == 2 ? pl.bytes / 2 : (pl.bytes + 7) / 8;
}

__global__ void fill_kernel(uint8_t* __restrict__ dst, int64_t blob_stride,
                            int64_t tensor_offset, TensorSpec spec,
                            uint64_t seed, int layer, int expert0,
                            int nexperts) {
  int64_t cpe = 0;  // chunks per expert
  for (int p = 0; p < spec.nplanes; ++p)
    cpe += (plane_words(spec.planes[p]) + CW - 1) / CW;
  const int64_t total = cpe * nexperts;
  for (int64_t gi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
       gi < total; gi += (int64_t)gridDim.x * blockDim.x) {
    const int ei = (int)(gi / cpe);
    int64_t ci = gi % cpe;
    int p = 0;
    for (; p < spec.nplanes; ++p) {
      const int64_t nc = (plane_words(spec.planes[p]) + CW - 1) / CW;
      if (ci < nc) break;
      ci -= nc;
    }
    const Plane pl = spec.planes[p];
    const uint64_t key =
        stream_key(seed, (uint64_t)layer, (uint64_t)(expert0 + ei),
                   (uint64_t)spec.tensor_id, (uint64_t)pl.id);
    uint8_t* t = dst + (int64_t)ei * blob_stride + tensor_offset + pl.offset;
    const int64_t nw = plane_words(pl);
    for (int64_t wi = ci * CW; wi < nw && wi < (ci + 1) * CW; ++wi) {
      const uint64_t w = word(key, (uint64_t)wi);
      if (pl.id == 2) {  // fp16 scales, one word per value
        const double u = (double)(w >> 11) * 0x1.0p-53;
        const double d = __dadd_rn(spec.lo, __dmul_rn(spec.hi - spec.lo, u));
        *reinterpret_cast<__half*>(t + 2 * wi) = __double2half(d);
      } else {
        const int64_t b0 = wi * 8;
        const int nb = (int)(pl.bytes - b0 < 8 ? pl.bytes - b0 : 8);
        uint8_t* q = t + b0;
        if (nb == 8 && ((uintptr_t)q & 7) == 0)
          *reinterpret_cast<uint64_t*>(q) = w;  // little-endian
        else
          for (int b = 0; b < nb; ++b) q[b] = (uint8_t)(w >> (8 * b));
      }
    }
  }
}

TensorSpec make_spec(int fmt, int rows, int cols, int tensor_id, double lo,
                     double hi) {
  TensorSpec s{};
  s.tensor_id = tensor_id;
  s.lo = lo;
  s.hi = hi;
  if (fmt == 2 || fmt == 4 || fmt == 5) {
    // SB3, NL3 (+ one shift byte per block), SB2 (64 code bytes per block)
    const int64_t nsb = (int64_t)rows * (cols / 256);
    const int64_t cb = fmt == 5 ? 64 : 96;
    s.planes[0] = {0, nsb * cb, 0};
    s.planes[1] = {nsb * cb, nsb * 4, 1};
    s.planes[2] = {nsb * (cb + 4), nsb * 2, 2};
    s.nplanes = 3;
    s.bytes = nsb * (cb + 6);
    if (fmt == 4) {
      s.planes[3] = {nsb * 102, nsb, 3};
      s.nplanes = 4;
      s.bytes = nsb * 103;
    }
  } else {  // Q4 / NL4
    const int64_t nb = (int64_t)rows * (cols / 32);
    s.planes[0] = {0, nb * 16, 0};
    s.planes[1] = {nb * 16, nb * 2, 2};
    s.nplanes = 2;
    s.bytes = nb * 18;
  }
  return s;
}

}  // namespace

extern "C" {

// Natural-layout expert blobs (up | gate | down) of experts
// expert0 .. expert0+nexperts-1 of one layer, written at dst + i*blob_stride.
// Returns 0 or a cudaError_t.
int synth_fill_experts(uint8_t* dst, int64_t blob_stride, int fmt_up_gate,
                       int fmt_down, int H, int F, double ug_lo, double ug_hi,
                       double dn_lo, double dn_hi, uint64_t seed, int layer,
                       int expert0, int nexperts, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  const TensorSpec up = make_spec(fmt_up_gate, F, H, 0, ug_lo, ug_hi);
  TensorSpec gate = make_spec(fmt_up_gate, F, H, 1, ug_lo, ug_hi);
  const TensorSpec down = make_spec(fmt_down, H, F, 2, dn_lo, dn_hi);
  const int64_t offs[3] = {0, up.bytes, 2 * up.bytes};
  const TensorSpec specs[3] = {up, gate, down};
  for (int t = 0; t < 3; ++t) {
    const int64_t total = ((specs[t].bytes + 7) / 8 / CW + 3) * nexperts;
    int64_t grid = (total + 255) / 256;
    if (grid > 148 * 64) grid = 148 * 64;
    fill_kernel<<<(int)grid, 256, 0, s>>>(dst, blob_stride, offs[t], specs[t],
                                         seed, layer, expert0, nexperts);
  }
  return (int)cudaGetLastError();
}

}  // extern "C"
