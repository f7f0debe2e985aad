// quantize.cuh -- Q/K/V quantisation in front of the attention path: an
// optional rotation by R = diag(signs) H_d / sqrt(d) (H_d the Sylvester
// Hadamard matrix), one power-of-two descale per block of rows, and the E4M3
// cast ("Attenzione flash e domanda sulla lunghezza della sequenza", section
// "FA3: Meccanica della tramoggia", point 3: a random rotation spreads
// outlier channels over all coordinates before block quantisation).
//
// The pass is a stream: each block's rows are contiguous in memory, so a
// persistent CTA pulls whole blocks into a ring of shared-memory stages with
// untiled bulk copies (one elected thread issues them, an mbarrier per stage
// counts the bytes), and its 256 threads transform, reduce and cast one block
// while the next ones are in flight.  A stage is handed back to the copy
// engine at the block's amax barrier, when every thread has its rows in
// registers.
//
// Four threads own one row.  The row is cut into 8-element chunks and thread
// part t (0..3) holds chunks t, t + 4, t + 8, ... (E = d / 4 elements), so the
// index of element i splits as i = 32 k + 8 t + j: j (bits 0-2) and k (bits
// 5 and up) lie inside a thread, t (bits 3-4) across the row's four lanes.
// The rotation is the radix-2 fast transform with stages of half-width 1, 2,
// ..., d/2, in that order (pair i, i + h: sum at i, difference at i + h):
// half-widths 1, 2, 4 inside the thread, 8 and 16 through shuffles, 32 and 64
// inside the thread again.  Every operation rounds to float32 once, in that
// fixed order.
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
constexpr int kQuantMaxStages = 8;
constexpr int kQuantMaxChunks = 4;  // 8-element chunks per thread at d = 128
constexpr int kQuantStageBudget = 96 * 1024;  // shared bytes of the ring (two CTAs per SM)

// Binary exponent e of the descale s = 2^e of a block whose largest
// magnitude is amax (e = 0 for an all-zero block).
__device__ __forceinline__ int quant_scale_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  int ex;
  const float m = frexpf(amax, &ex);  // amax = m 2^ex, m in [0.5, 1): mantissa 2m, exponent ex - 1
  const int e = (m <= 0.875f) ? ex - 9 : ex - 8;
  return e < -126 ? -126 : e;
}

// One thread's E elements of a row, read from the staged block: slot c
// (elements 8c .. 8c + 7 of the thread's list) holds chunk c ^ sw, row
// elements 32 (c ^ sw) + 8 part ..  With sw = 1 on odd rows, the two rows of
// a quarter-warp read opposite 64-byte halves of their 256-byte rows, so the
// 16-byte reads hit distinct banks.  Rows past the block's end read as zeros.
template <int E>
__device__ __forceinline__ void quant_read_row(const uint8_t* stage, int row_bytes, int r, int rows, int part,
                                               int x_f32, const uint4* sign_masks, int sw, float (&v)[E]) {
  if (r >= rows) {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = 0.0f;
    return;
  }
  if (x_f32) {
    const float* src = reinterpret_cast<const float*>(stage + static_cast<int64_t>(r) * row_bytes) + 8 * part;
#pragma unroll
    for (int c = 0; c < E / 8; ++c) {
      const float4 a = *reinterpret_cast<const float4*>(src + 32 * (c ^ sw));
      const float4 b = *reinterpret_cast<const float4*>(src + 32 * (c ^ sw) + 4);
      v[8 * c + 0] = a.x; v[8 * c + 1] = a.y; v[8 * c + 2] = a.z; v[8 * c + 3] = a.w;
      v[8 * c + 4] = b.x; v[8 * c + 5] = b.y; v[8 * c + 6] = b.z; v[8 * c + 7] = b.w;
    }
  } else {
    // bfloat16 -> float32 is exact: the 16 bits become the high half.
    const uint16_t* src = reinterpret_cast<const uint16_t*>(stage + static_cast<int64_t>(r) * row_bytes) + 8 * part;
#pragma unroll
    for (int c = 0; c < E / 8; ++c) {
      const uint4 q = *reinterpret_cast<const uint4*>(src + 32 * (c ^ sw));
      // With a rotation, the signs flip the bfloat16 sign bits (bits 15 and 31 of each word).
      const uint4 sm = sign_masks ? sign_masks[(c ^ sw) * kQuantThreadsPerRow + part] : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w[4] = {q.x ^ sm.x, q.y ^ sm.y, q.z ^ sm.z, q.w ^ sm.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * c + 2 * i] = __uint_as_float(w[i] << 16);
        v[8 * c + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
  }
}

// One in-thread stage of the transform over the thread's list: pairs (e, e + h)
// with bit h of e clear, taken two at a time in packed f32x2.
template <int E, int H>
__device__ __forceinline__ void quant_stage(float (&v)[E]) {
  if constexpr (H == 1) {
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float a = v[e], b = v[e + 1];
      v[e] = a + b;
      v[e + 1] = a - b;
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      if ((e & H) == 0) {
        const uint64_t a = f2_pack(v[e], v[e + 1]), b = f2_pack(v[e + H], v[e + 1 + H]);
        f2_unpack(f2_add(a, b), v[e], v[e + 1]);
        f2_unpack(f2_fma(b, f2_pack(-1.0f, -1.0f), a), v[e + H], v[e + 1 + H]);  // a - b, one rounding
      }
    }
  }
}

// The stage of half-width 32 (slot bit 0) when slots 2i and 2i + 1 may hold
// chunks 2i + 1 and 2i (sw = 1): the member in slot 2i is then the upper
// one.  new slot 2i = s1 * slot 2i + slot 2i+1, new slot 2i+1 = s2 * slot
// 2i+1 + slot 2i, with (s1, s2) = (1, -1) or (-1, 1): a sum or a difference,
// one rounding each, exactly as in the unswapped order.
template <int E>
__device__ __forceinline__ void quant_stage32(float (&v)[E], int sw) {
  const float s1 = sw ? -1.0f : 1.0f;
  const uint64_t sg1 = f2_pack(s1, s1), sg2 = f2_pack(-s1, -s1);
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    if ((e & 8) == 0) {
      const uint64_t a = f2_pack(v[e], v[e + 1]), b = f2_pack(v[e + 8], v[e + 9]);
      f2_unpack(f2_fma(a, sg1, b), v[e], v[e + 1]);
      f2_unpack(f2_fma(b, sg2, a), v[e + 8], v[e + 9]);
    }
  }
}

// The signs and the unnormalised transform x H_d over the thread's E values
// (the factor 1/sqrt(d) is applied by the caller).  sb[c] holds the 8 sign
// bits of chunk c (bit j set: element j of the chunk is negated); they are
// applied here only when not already applied to the raw words (and then the
// slots are not swapped, sw = 0).
template <int E>
__device__ __forceinline__ void quant_rotate_row(int part, const uint32_t (&sb)[E / 8], bool signs_applied, int sw,
                                                 float (&v)[E]) {
  if (!signs_applied) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((sb[e / 8] >> (e % 8)) & 1u) v[e] = -v[e];
    }
  }
  quant_stage<E, 1>(v);
  quant_stage<E, 2>(v);
  quant_stage<E, 4>(v);
  // Half-widths 8 and 16: the partner of element i is i ^ h, in lane part ^ (h / 8)
  // at the same position; the lower member keeps v + other, the upper other - v.
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
  // Half-widths 32 and 64: chunk bits of the thread's list (8 and 16 in it).
  quant_stage32<E>(v, sw);
  if constexpr (E > 16) quant_stage<E, 16>(v);
}

// Stores E4M3(v * mul): mul = c / s, with c = float32(1/sqrt(d)) after a
// rotation (else 1) and s the block's power-of-two descale, so that
// v * mul = (v * c) / s exactly (s is a power of two).  Slot c (chunk c ^ sw)
// goes to row bytes 32 (c ^ sw) + 8 part .. + 7.
template <int E>
__device__ __forceinline__ void quant_store_row(uint8_t* dst_row, int part, const float (&v)[E], float mul, int sw) {
  const uint64_t m2 = f2_pack(mul, mul);
#pragma unroll
  for (int c = 0; c < E / 8; ++c) {
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int e = 8 * c + 4 * j;
      float a, b, cc, dd;
      f2_unpack(f2_mul(f2_pack(v[e], v[e + 1]), m2), a, b);
      f2_unpack(f2_mul(f2_pack(v[e + 2], v[e + 3]), m2), cc, dd);
      w[j] = cvt_e4m3x4(a, b, cc, dd);
    }
    *reinterpret_cast<uint2*>(dst_row + 32 * (c ^ sw) + 8 * part) = make_uint2(w[0], w[1]);
  }
}

// Ring geometry of one launch: a stage holds one block of p.block_rows rows.
__host__ __device__ inline int quant_stage_bytes(const QuantParams& p) {
  return p.block_rows * p.d * (p.x_f32 ? 4 : 2);
}
__host__ __device__ inline int quant_stages(const QuantParams& p) {
  const int n = kQuantStageBudget / quant_stage_bytes(p);
  return n < 1 ? 1 : (n > kQuantMaxStages ? kQuantMaxStages : n);
}

// MODE 0: scale per block of p.block_rows rows (rows kept in registers
//         between the amax and the cast).
// MODE 1: per-slab pass 1 -- amax of each 128-row block, atomicMax into
//         p.scales[z] (float bits of a value >= 0 order like integers).
// MODE 2: per-slab pass 2 -- cast with the descale of the slab's amax.
// The CTA walks the blocks u = blockIdx.x, blockIdx.x + gridDim.x, ... of the
// Z * nblocks blocks (slab z = u / nblocks).
template <int E, int MODE>
__global__ void __launch_bounds__(kQuantWarps * 32, 2) quantize_kernel(const QuantParams p, uint32_t* err_word) {
  constexpr int kPasses = 128 / kQuantRowsPerPass;  // rows per thread held in registers (block_rows <= 128)
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ __align__(8) uint64_t full[kQuantMaxStages];
  __shared__ float warp_amax[2][kQuantWarps];
  // bfloat16 inputs with a rotation: XOR masks of the signs, per (chunk, part),
  // for the four 32-bit words (two elements each) of a chunk.
  __shared__ uint4 sign_masks[kQuantMaxChunks * kQuantThreadsPerRow];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = lane & (kQuantThreadsPerRow - 1);
  const int rsub = threadIdx.x / kQuantThreadsPerRow;  // 0..63
  const int row_bytes = p.d * (p.x_f32 ? 4 : 2);
  const int stage_bytes = quant_stage_bytes(p);
  const int stages = quant_stages(p);
  const int nunits = p.Z * p.nblocks;
  const uint8_t* xb = static_cast<const uint8_t*>(p.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  const bool word_signs = p.rotate && !p.x_f32;
  if (word_signs && threadIdx.x < (E / 8) * kQuantThreadsPerRow) {
    const int c = threadIdx.x / kQuantThreadsPerRow, pt = threadIdx.x % kQuantThreadsPerRow;
    // (no run-time index into the parameter array, which would copy it to local memory)
    const uint32_t word = c == 0 ? p.sign_bits[0] : c == 1 ? p.sign_bits[1] : c == 2 ? p.sign_bits[2] : p.sign_bits[3];
    const uint32_t x = (word >> (8 * pt)) & 0xFFu;  // elements 32 c + 8 pt + j, bit j
    uint32_t m[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) m[j] = (((x >> (2 * j)) & 1u) << 15) | (((x >> (2 * j + 1)) & 1u) << 31);
    sign_masks[threadIdx.x] = make_uint4(m[0], m[1], m[2], m[3]);
  }
  __syncthreads();
  // Copy of the CTA's local block k into stage k % stages (thread 0 only).
  auto issue = [&](int k) {
    const int u = blockIdx.x + k * gridDim.x;
    if (u >= nunits) return;
    const int z = u / p.nblocks, blk = u - z * p.nblocks;
    const int r0 = blk * p.block_rows;
    const uint32_t bytes = static_cast<uint32_t>(min(p.block_rows, p.N - r0) * row_bytes);
    uint64_t* bar = &full[k % stages];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(ring + (k % stages) * stage_bytes, xb + (static_cast<int64_t>(z) * p.N + r0) * row_bytes, bytes, bar);
  };
  if (threadIdx.x == 0) {
    for (int k = 0; k < stages; ++k) issue(k);
  }

  // This thread's sign bits: chunk c covers row elements 32 c + 8 part .. + 7.
  uint32_t sb[E / 8];
#pragma unroll
  for (int c = 0; c < E / 8; ++c) sb[c] = (p.sign_bits[c] >> (8 * part)) & 0xFFu;
  // float32(1/sqrt(d)) after a rotation: applied to the block maximum here
  // (positive scaling is monotone, so max |v c| = max|v| c) and folded into
  // the cast's multiplier.
  const float cnorm = p.rotate ? ((E == 32) ? 0.08838834764831845f : 0.125f) : 1.0f;
  // Odd rows hold their chunk pairs swapped (bfloat16 inputs; see quant_read_row).
  // Every row this thread handles has the parity of rsub (rows rsub + 64 i).
  const int sw = p.x_f32 ? 0 : (rsub & 1);

  int k = 0;
  bool aborted = false;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++k) {
    const int z = u / p.nblocks, blk = u - z * p.nblocks;
    const int r0 = blk * p.block_rows;
    const int rows = min(p.block_rows, p.N - r0);
    const bool ok = mbar_wait_bounded(&full[k % stages], (k / stages) & 1, err_word, kErrTimeoutLoad);
    const uint8_t* stage = ring + (k % stages) * stage_bytes;
    float v[kPasses][E];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      // Every lane transforms (rows past the block's end hold zeros), so the
      // full-warp shuffles of the rotation always have all 32 lanes.
      quant_read_row<E>(stage, row_bytes, rsub + i * kQuantRowsPerPass, ok ? rows : 0, part, p.x_f32,
                        word_signs ? sign_masks : nullptr, sw, v[i]);
      if (p.rotate) quant_rotate_row<E>(part, sb, word_signs, sw, v[i]);
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
    }
    if constexpr (MODE != 2) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (lane == 0) warp_amax[k & 1][warp] = amax;
    }
    // Every thread holds its rows: the stage goes back to the copy engine.
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    if (threadIdx.x == 0) issue(k + stages);
    int e;
    if constexpr (MODE == 2) {
      e = quant_scale_exponent(__uint_as_float(reinterpret_cast<const uint32_t*>(p.scales)[z]));
    } else {
      float a = warp_amax[k & 1][0];
#pragma unroll
      for (int w = 1; w < kQuantWarps; ++w) a = fmaxf(a, warp_amax[k & 1][w]);
      a *= cnorm;
      if constexpr (MODE == 1) {
        if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned int*>(p.scales + z), __float_as_uint(a));
        continue;
      }
      e = quant_scale_exponent(a);
      if (threadIdx.x == 0) p.scales[static_cast<int64_t>(z) * p.nblocks + blk] = ldexpf(1.0f, e);
    }
    const float mul = cnorm * ldexpf(1.0f, -e);  // c / s, exact (s a power of two)
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      const int r = rsub + i * kQuantRowsPerPass;
      if (r < rows) quant_store_row<E>(p.xq + (static_cast<int64_t>(z) * p.N + r0 + r) * p.d, part, v[i], mul, sw);
    }
  }
  // After a wait ran out: let the copies still in flight land before the CTA's
  // shared memory is released (each wait again bounded).
  if (threadIdx.x == 0 && aborted) {
    for (int j = k; j < k + stages; ++j) {
      if (blockIdx.x + j * gridDim.x >= nunits) break;
      mbar_wait_bounded(&full[j % stages], (j / stages) & 1, err_word, kErrTimeoutLoad, 100000000ull);
    }
  }
}

// Per-slab pass 3: amax words -> descales.
__global__ void quantize_finish_kernel(float* scales, int Z) {
  const int z = blockIdx.x * blockDim.x + threadIdx.x;
  if (z < Z) scales[z] = ldexpf(1.0f, quant_scale_exponent(__uint_as_float(reinterpret_cast<const uint32_t*>(scales)[z])));
}

}  // namespace fp8attn
