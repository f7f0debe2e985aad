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
// Two adjacent lanes own one row.  The row is cut into 8-element chunks and
// lane t (0, 1) of the pair holds chunks t, t + 2, t + 4, ... (E = d / 2
// elements), so the index of element i splits as i = 16 m + 8 t + j: j (bits
// 0-2) and m (bits 4 and up) lie inside a thread, t (bit 3) across the pair.
// The rotation is the radix-2 fast transform with stages of half-width 1, 2,
// ..., d/2, in that order (pair i, i + h: sum at i, difference at i + h):
// half-widths 1, 2, 4 inside the thread, 8 through one shuffle, 16 and up
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

constexpr int kQuantWarps = 8;  // the block maximum reads the warps' maxima as two float4
constexpr int kQuantThreadsPerRow = 2;
constexpr int kQuantRowsPerPass = kQuantWarps * 32 / kQuantThreadsPerRow;  // 128: one block per pass
constexpr int kQuantMaxStages = 8;
constexpr int kQuantMaxChunks = 16;  // 8-element chunks per row at d = 128
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

// One thread's E elements of a row, read from the staged block.  Thread t
// (0, 1) of a row holds its chunks 2 m + t (8 elements each, m = 0 .. E/8 - 1):
// slot k (elements 8 k .. 8 k + 7 of the thread's list) holds chunk
// 2 (k ^ s) + t, where s = row % 4 for bfloat16 rows (0 otherwise), so the
// four rows of a quarter-warp read distinct 16-byte banks.  Row element i
// = 16 (k ^ s) + 8 t + j.  Rows past the block's end read as zeros.
template <int E>
__device__ __forceinline__ void quant_read_row(const uint8_t* stage, int row_bytes, int r, int rows, int t, int s,
                                               int x_f32, const uint4* sign_masks, float (&v)[E]) {
  if (r >= rows) {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = 0.0f;
    return;
  }
  if (x_f32) {
    const float* src = reinterpret_cast<const float*>(stage + static_cast<int64_t>(r) * row_bytes);
#pragma unroll
    for (int k = 0; k < E / 8; ++k) {
      const int c = 2 * (k ^ s) + t;
      const float4 a = *reinterpret_cast<const float4*>(src + 8 * c);
      const float4 b = *reinterpret_cast<const float4*>(src + 8 * c + 4);
      v[8 * k + 0] = a.x; v[8 * k + 1] = a.y; v[8 * k + 2] = a.z; v[8 * k + 3] = a.w;
      v[8 * k + 4] = b.x; v[8 * k + 5] = b.y; v[8 * k + 6] = b.z; v[8 * k + 7] = b.w;
    }
  } else {
    // bfloat16 -> float32 is exact: the 16 bits become the high half.
    const uint16_t* src = reinterpret_cast<const uint16_t*>(stage + static_cast<int64_t>(r) * row_bytes);
#pragma unroll
    for (int k = 0; k < E / 8; ++k) {
      const int c = 2 * (k ^ s) + t;
      const uint4 q = *reinterpret_cast<const uint4*>(src + 8 * c);
      // With a rotation, the signs flip the bfloat16 sign bits (bits 15 and 31 of each word).
      const uint4 sm = sign_masks ? sign_masks[c] : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w[4] = {q.x ^ sm.x, q.y ^ sm.y, q.z ^ sm.z, q.w ^ sm.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * k + 2 * i] = __uint_as_float(w[i] << 16);
        v[8 * k + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
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

// An in-thread stage over a slot bit that s may flip: pairs (e, e + H) with
// bit H of e clear; when flip is set, slot e holds the pair's upper member and
// slot e + H its lower one.  Slot e becomes s1 v[e] + v[e + H] and slot e + H
// becomes v[e] - s1 v[e + H] (s1 = -1 when flipped, else 1): the lower slot
// gets the sum and the upper the difference, each rounded once, exactly as in
// the unflipped order.
template <int E, int H>
__device__ __forceinline__ void quant_stage_flip(float (&v)[E], int flip) {
  const float s1 = flip ? -1.0f : 1.0f;
  const uint64_t sg1 = f2_pack(s1, s1), sg2 = f2_pack(-s1, -s1);
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    if ((e & H) == 0) {
      const uint64_t a = f2_pack(v[e], v[e + 1]), b = f2_pack(v[e + H], v[e + 1 + H]);
      f2_unpack(f2_fma(a, sg1, b), v[e], v[e + 1]);
      f2_unpack(f2_fma(b, sg2, a), v[e + H], v[e + 1 + H]);
    }
  }
}

// The signs and the unnormalised transform x H_d over the thread's E values
// (the factor 1/sqrt(d) is applied by the caller), stages of half-width 1, 2,
// 4 inside the slots, 8 across the row's two threads, then 16, 32 (and 64)
// over the slot bits.  sb[k] holds the 8 sign bits of slot k (bit j set:
// element j is negated); they are applied here only when not already applied
// to the raw words (and then s = 0).
template <int E>
__device__ __forceinline__ void quant_rotate_row(int t, int s, const uint32_t (&sb)[E / 8], bool signs_applied,
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
  // Half-width 8: the partner of element i is i ^ 8, in the row's other
  // thread at the same position; the lower member keeps v + other, the upper
  // other - v.
  {
    const float sg = t ? -1.0f : 1.0f;
    const uint64_t sg2 = f2_pack(sg, sg);
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float o0 = __shfl_xor_sync(0xffffffffu, v[e], 1);
      const float o1 = __shfl_xor_sync(0xffffffffu, v[e + 1], 1);
      f2_unpack(f2_fma(f2_pack(v[e], v[e + 1]), sg2, f2_pack(o0, o1)), v[e], v[e + 1]);
    }
  }
  // Half-widths 16, 32, 64: slot bits 0, 1, 2 (8, 16, 32 in the list); s flips bits 0 and 1.
  quant_stage_flip<E, 8>(v, s & 1);
  quant_stage_flip<E, 16>(v, (s >> 1) & 1);
  if constexpr (E > 32) quant_stage<E, 32>(v);
}

// Stores E4M3(v * mul): mul = c / s, with c = float32(1/sqrt(d)) after a
// rotation (else 1) and s the block's power-of-two descale, so that
// v * mul = (v * c) / s exactly (s is a power of two).  Slot k holds chunk
// 2 (k ^ sx) + t, row bytes 8 (2 (k ^ sx) + t) .. + 7; the two lanes of the
// row swap half their slots so that each stores whole 16-byte pieces.  Every
// lane calls this (the swap is a full-warp shuffle); `live` says whether the
// row exists.
template <int E>
__device__ __forceinline__ void quant_store_row(uint8_t* dst_row, bool live, int t, int sx, const float (&v)[E],
                                                float mul) {
  const uint64_t m2 = f2_pack(mul, mul);
  uint2 w[E / 8];
#pragma unroll
  for (int k = 0; k < E / 8; ++k) {
    float a, b, cc, dd;
    f2_unpack(f2_mul(f2_pack(v[8 * k], v[8 * k + 1]), m2), a, b);
    f2_unpack(f2_mul(f2_pack(v[8 * k + 2], v[8 * k + 3]), m2), cc, dd);
    w[k].x = cvt_e4m3x4(a, b, cc, dd);
    f2_unpack(f2_mul(f2_pack(v[8 * k + 4], v[8 * k + 5]), m2), a, b);
    f2_unpack(f2_mul(f2_pack(v[8 * k + 6], v[8 * k + 7]), m2), cc, dd);
    w[k].y = cvt_e4m3x4(a, b, cc, dd);
  }
  // Slots 2 q and 2 q + 1: lane t keeps slot 2 q + t and takes the partner's
  // slot 2 q + t, which holds the other half of the same 16 bytes (chunks
  // 2 m and 2 m + 1, m = (2 q + t) ^ sx), so that each lane stores 16 bytes.
#pragma unroll
  for (int q = 0; q < E / 16; ++q) {
    const uint2 mine = t ? w[2 * q + 1] : w[2 * q];
    const uint2 give = t ? w[2 * q] : w[2 * q + 1];
    uint2 got;
    got.x = __shfl_xor_sync(0xffffffffu, give.x, 1);
    got.y = __shfl_xor_sync(0xffffffffu, give.y, 1);
    const uint4 out = t ? make_uint4(got.x, got.y, mine.x, mine.y) : make_uint4(mine.x, mine.y, got.x, got.y);
    if (live) *reinterpret_cast<uint4*>(dst_row + 16 * ((2 * q + t) ^ sx)) = out;
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
  __shared__ __align__(16) float warp_amax[2][kQuantWarps];
  // bfloat16 inputs with a rotation: XOR masks of the signs, per 8-element
  // chunk of the row, for the four 32-bit words (two elements each) of a chunk.
  __shared__ uint4 sign_masks[kQuantMaxChunks];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = lane & 1;                               // which chunks of the row: 2 m + t
  const int rsub = threadIdx.x / kQuantThreadsPerRow;  // 0..127
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
    const int c = threadIdx.x, wi = c >> 2;  // chunk c: row elements 8 c .. 8 c + 7
    // (no run-time index into the parameter array, which would copy it to local memory)
    const uint32_t word = wi == 0 ? p.sign_bits[0] : wi == 1 ? p.sign_bits[1] : wi == 2 ? p.sign_bits[2] : p.sign_bits[3];
    const uint32_t x = (word >> (8 * (c & 3))) & 0xFFu;  // elements 8 c + j, bit j
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

  // This thread's sign bits for float32 rows (no slot rotation there): slot k
  // holds chunk 2 k + t, row elements 16 k + 8 t .. + 7, in sign word k / 2.
  uint32_t sb[E / 8];
#pragma unroll
  for (int k = 0; k < E / 8; ++k) sb[k] = (p.sign_bits[k >> 1] >> (8 * ((2 * k + t) & 3))) & 0xFFu;
  // float32(1/sqrt(d)) after a rotation: applied to the block maximum here
  // (positive scaling is monotone, so max |v c| = max|v| c) and folded into
  // the cast's multiplier.
  const float cnorm = p.rotate ? ((E == 64) ? 0.08838834764831845f : 0.125f) : 1.0f;
  // Slot rotation of bfloat16 rows (see quant_read_row); the thread's row is rsub.
  const int sx = p.x_f32 ? 0 : (rsub & 3);

  int k = 0;
  bool aborted = false;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++k) {
    const int z = u / p.nblocks, blk = u - z * p.nblocks;
    const int r0 = blk * p.block_rows;
    const int rows = min(p.block_rows, p.N - r0);
    const bool ok = mbar_wait_bounded(&full[k % stages], (k / stages) & 1, err_word, kErrTimeoutLoad);
    const uint8_t* stage = ring + (k % stages) * stage_bytes;
    float v[kPasses][E];
    // Block maximum of |v| in four independent chains (max is exact in any order).
    float am4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      // Every lane transforms (rows past the block's end hold zeros), so the
      // full-warp shuffles of the rotation always have all 32 lanes.
      quant_read_row<E>(stage, row_bytes, rsub + i * kQuantRowsPerPass, ok ? rows : 0, t, sx, p.x_f32,
                        word_signs ? sign_masks : nullptr, v[i]);
      if (p.rotate) quant_rotate_row<E>(t, sx, sb, word_signs, v[i]);
#pragma unroll
      for (int e = 0; e < E; e += 4) {
        const float m01 = fmaxf(fabsf(v[i][e]), fabsf(v[i][e + 1])), m23 = fmaxf(fabsf(v[i][e + 2]), fabsf(v[i][e + 3]));
        am4[(e / 4) & 3] = fmaxf(am4[(e / 4) & 3], fmaxf(m01, m23));
      }
    }
    float amax = fmaxf(fmaxf(am4[0], am4[1]), fmaxf(am4[2], am4[3]));
    if constexpr (MODE != 2) {
      amax = warp_max_f32(amax);
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
      const float4 w0 = reinterpret_cast<const float4*>(warp_amax[k & 1])[0];
      const float4 w1 = reinterpret_cast<const float4*>(warp_amax[k & 1])[1];
      float a = fmaxf(fmaxf(fmaxf(w0.x, w0.y), fmaxf(w0.z, w0.w)), fmaxf(fmaxf(w1.x, w1.y), fmaxf(w1.z, w1.w)));
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
      // (every lane takes part: the exchange inside is a full-warp shuffle)
      quant_store_row<E>(p.xq + (static_cast<int64_t>(z) * p.N + r0 + r) * p.d, r < rows, t, sx, v[i], mul);
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
