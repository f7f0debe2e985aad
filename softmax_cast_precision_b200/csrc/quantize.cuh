// quantize.cuh -- Q/K/V quantisation in front of the attention path: an
// optional rotation by R = diag(signs) H_d / sqrt(d) (H_d the Sylvester
// Hadamard matrix), one power-of-two descale per block of rows, and the E4M3
// cast ("Attenzione flash e domanda sulla lunghezza della sequenza", section
// "FA3: Meccanica della tramoggia", point 3: a random rotation spreads
// outlier channels over all coordinates before block quantisation).
//
// Four threads own one row: thread part t (0..3) holds elements
// [t*E, t*E + E), E = d / 4, so a warp covers eight consecutive rows with
// contiguous 16-byte loads and stores.  The rotation is the radix-2 fast
// transform with stages of half-width 1, 2, ..., d/2 (pair i, i + h: sum at
// i, difference at i + h); stages below E stay inside a thread, the last two
// pair threads through shuffles.  Every operation rounds to float32 once, in
// that fixed order.
//
// Descale of a block: the smallest power of two s >= 2^-126 with
// amax <= 448 s; with amax = m 2^E (m in [1, 2)) that is 2^(E - 8) when
// m <= 1.75 and 2^(E - 7) otherwise.  x / s is then exact and within E4M3
// range, and the cast is round-to-nearest-even with saturation.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fp8attn {

struct QuantParams {
  const void* x;      // [Z, N, d] bfloat16 (x_f32 == 0) or float32
  uint8_t* xq;        // [Z, N, d] E4M3
  float* scales;      // [Z, nblocks] descales (per-slab mode: [Z], amax words during the pass)
  int Z, N, d;
  int block_rows;     // rows per block (per-slab mode: 128, the rows one CTA covers)
  int nblocks;        // blocks per slab in `scales`
  int x_f32;
  int rotate;
  uint32_t sign_bits[4];  // bit i set: signs[i] = -1 (d <= 128)
};

constexpr int kQuantWarps = 8;
constexpr int kQuantThreadsPerRow = 4;
constexpr int kQuantRowsPerPass = kQuantWarps * 32 / kQuantThreadsPerRow;  // 64

// Binary exponent e of the descale s = 2^e of a block whose largest
// magnitude is amax (e = 0 for an all-zero block).
__device__ __forceinline__ int quant_scale_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  int ex;
  const float m = frexpf(amax, &ex);  // amax = m 2^ex, m in [0.5, 1): mantissa 2m, exponent ex - 1
  const int e = (m <= 0.875f) ? ex - 9 : ex - 8;
  return e < -126 ? -126 : e;
}

// Raw 16-byte words of one thread's E elements of a row: bfloat16 E/8 words,
// float32 E/4.
template <int E>
struct RowBits {
  uint4 w[E / 4];
};

template <int E>
__device__ __forceinline__ RowBits<E> quant_fetch_row(const QuantParams& p, int z, int row, int part) {
  RowBits<E> r;
  const int64_t base = (static_cast<int64_t>(z) * p.N + row) * p.d + part * E;
  if (p.x_f32) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(p.x) + base);
#pragma unroll
    for (int i = 0; i < E / 4; ++i) r.w[i] = __ldg(src + i);
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + base);
#pragma unroll
    for (int i = 0; i < E / 8; ++i) r.w[i] = __ldg(src + i);
  }
  return r;
}

__device__ __forceinline__ uint32_t quant_word(const uint4& q, int i) {
  return i == 0 ? q.x : i == 1 ? q.y : i == 2 ? q.z : q.w;
}

// The thread's E values of the row as float32, with the signs and the
// unnormalised transform x H_d applied when the rotation is enabled (the
// factor 1/sqrt(d) is applied by the caller).  `sb` holds this thread's E
// sign bits (bit e set: element e is negated).
template <int E>
__device__ __forceinline__ void quant_transform_row(const QuantParams& p, const RowBits<E>& r, int part, uint32_t sb,
                                                    float (&v)[E]) {
  if (p.x_f32) {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = __uint_as_float(quant_word(r.w[e / 4], e % 4));
  } else {
    // bfloat16 -> float32 is exact: the 16 bits become the high half.
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint32_t w = quant_word(r.w[e / 8], (e / 2) % 4);
      v[e] = __uint_as_float(w << 16);
      v[e + 1] = __uint_as_float(w & 0xFFFF0000u);
    }
  }
  if (!p.rotate) return;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if ((sb >> e) & 1u) v[e] = -v[e];
  }
  // Stage h = 1 inside the thread, one rounding per sum or difference.
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const float a = v[e], b = v[e + 1];
    v[e] = a + b;
    v[e + 1] = a - b;
  }
  // Stages h = 2 .. E/2: both members of a pair (e, e + 1) meet (e + h, e + 1 + h), in packed f32x2.
#pragma unroll
  for (int h = 2; h < E; h *= 2) {
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      if ((e & h) == 0) {
        const uint64_t a = f2_pack(v[e], v[e + 1]), b = f2_pack(v[e + h], v[e + 1 + h]);
        f2_unpack(f2_add(a, b), v[e], v[e + 1]);
        f2_unpack(f2_add(a, f2_mul(b, f2_pack(-1.0f, -1.0f))), v[e + h], v[e + 1 + h]);
      }
    }
  }
  // The two stages across the row's four threads: the partner of element
  // i = part*E + e is i ^ h, in part ^ (h / E) at the same e; the lower
  // member keeps v + other, the upper other - v (one rounding each).
#pragma unroll
  for (int hp = 1; hp < kQuantThreadsPerRow; hp *= 2) {
    const float sg = (part & hp) ? -1.0f : 1.0f;
    const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float o0 = __shfl_xor_sync(0xffffffffu, v[e], hp);
      const float o1 = __shfl_xor_sync(0xffffffffu, v[e + 1], hp);
      f2_unpack(f2_fma(f2_pack(v[e], v[e + 1]), sg2, f2_pack(o0, o1)), v[e], v[e + 1]);
    }
  }
}

// Stores E4M3(v * mul): mul = c / s, with c = float32(1/sqrt(d)) after a
// rotation (else 1) and s the block's power-of-two descale, so that
// v * mul = (v * c) / s exactly (s is a power of two).
template <int E>
__device__ __forceinline__ void quant_store_row(const QuantParams& p, int z, int row, int part, const float (&v)[E],
                                                float mul) {
  uint4* dst = reinterpret_cast<uint4*>(p.xq + (static_cast<int64_t>(z) * p.N + row) * p.d + part * E);
  const uint64_t m2 = f2_pack(mul, mul);
#pragma unroll
  for (int c = 0; c < E / 16; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = c * 16 + 4 * j;
      float a, b, cc, dd;
      f2_unpack(f2_mul(f2_pack(v[e], v[e + 1]), m2), a, b);
      f2_unpack(f2_mul(f2_pack(v[e + 2], v[e + 3]), m2), cc, dd);
      w[j] = cvt_e4m3x4(a, b, cc, dd);
    }
    dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// MODE 0: scale per block of p.block_rows rows (one CTA per block, rows kept
//         in registers between the amax and the cast).
// MODE 1: per-slab pass 1 -- amax of the CTA's 128 rows, atomicMax into
//         p.scales[z] (float bits of a value >= 0 order like integers).
// MODE 2: per-slab pass 2 -- cast with the descale of the slab's amax.
template <int E, int MODE>
__global__ void __launch_bounds__(kQuantWarps * 32, 2) quantize_kernel(const QuantParams p) {
  constexpr int kPasses = 128 / kQuantRowsPerPass;  // rows per thread held in registers (block_rows <= 128)
  __shared__ float warp_amax[kQuantWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = lane & (kQuantThreadsPerRow - 1);
  const int rsub = threadIdx.x / kQuantThreadsPerRow;  // 0..63
  const int blk = blockIdx.x, z = blockIdx.y;
  const int r0 = blk * p.block_rows;
  const int rows = min(p.block_rows, p.N - r0);
  // All of the thread's rows are fetched before any is transformed, so their
  // loads are in flight together.
  RowBits<E> raw[kPasses];
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int r = rsub + i * kQuantRowsPerPass;
    if (r < rows) {
      raw[i] = quant_fetch_row<E>(p, z, r0 + r, part);
    } else {
#pragma unroll
      for (int j = 0; j < E / 4; ++j) raw[i].w[j] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // This thread's E sign bits: E = 32 is one whole word, E = 16 half of one.
  uint32_t sb;
  {
    const int i0 = part * E;
    const int wi = i0 >> 5;
    sb = (wi == 0 ? p.sign_bits[0] : wi == 1 ? p.sign_bits[1] : wi == 2 ? p.sign_bits[2] : p.sign_bits[3]) >>
         (i0 & 31);
  }
  // float32(1/sqrt(d)) after a rotation: applied to the block maximum here
  // (positive scaling is monotone, so max |v c| = max|v| c) and folded into
  // the cast's multiplier.
  const float cnorm = p.rotate ? ((E == 32) ? 0.08838834764831845f : 0.125f) : 1.0f;
  float v[kPasses][E];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    // Every lane transforms (rows past the block's end hold zeros), so the
    // full-warp shuffles of the rotation always have all 32 lanes.
    const int r = rsub + i * kQuantRowsPerPass;
    quant_transform_row<E>(p, raw[i], part, sb, v[i]);
    if (r < rows) {
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
    }
  }
  amax *= cnorm;
  int e;
  if constexpr (MODE == 2) {
    e = quant_scale_exponent(__uint_as_float(reinterpret_cast<const uint32_t*>(p.scales)[z]));
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) warp_amax[warp] = amax;
    __syncthreads();
    float a = warp_amax[0];
#pragma unroll
    for (int w = 1; w < kQuantWarps; ++w) a = fmaxf(a, warp_amax[w]);
    if constexpr (MODE == 1) {
      if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned int*>(p.scales + z), __float_as_uint(a));
      return;
    }
    e = quant_scale_exponent(a);
    if (threadIdx.x == 0) p.scales[static_cast<int64_t>(z) * p.nblocks + blk] = ldexpf(1.0f, e);
  }
  const float mul = cnorm * ldexpf(1.0f, -e);  // c / s, exact (s a power of two)
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int r = rsub + i * kQuantRowsPerPass;
    if (r < rows) quant_store_row<E>(p, z, r0 + r, part, v[i], mul);
  }
}

// Per-slab pass 3: amax words -> descales.
__global__ void quantize_finish_kernel(float* scales, int Z) {
  const int z = blockIdx.x * blockDim.x + threadIdx.x;
  if (z < Z) scales[z] = ldexpf(1.0f, quant_scale_exponent(__uint_as_float(reinterpret_cast<const uint32_t*>(scales)[z])));
}

}  // namespace fp8attn
