// decode.cuh -- decode / split-KV form of the P-cast attention forward pass
// (d = 128): one query row per (batch, head) attends to all N keys.
//
// The keys are cut into splits of `split_tiles` consecutive 128-key tiles.
// One CTA handles one split of one (batch, kv-head) for the G = H / Hkv query
// heads that share it, running the blockwise online softmax with the P-cast
// over the split's tiles (walked forward or in reverse inside the split):
// running maximum, P * S = 2^(x - m + log2 S), l from the unquantised
// values, P^ = E4M3(P * S), O += P^ V ("Attenzione flash e domanda sulla
// lunghezza della sequenza", sections "L'algoritmo Flash Attention" and "La
// ricorrenza softmax online"; "P-Cast Precision in FP8 Attention", technical
// summary, section 1).  It writes (m, l, acc) per query row to a workspace;
// decode_combine_kernel merges the splits exactly through their maxima and
// sums and writes O / (S l) and lse.
//
// With one query row per head there is no M dimension for the tensor cores:
// products run on the FP32 pipes.  E4M3 x E4M3 products are exact in FP32.
// Thread t owns key t of a tile for S = q K^T; for P^ V it owns the four
// output columns 4 (t % 32) .. + 3 over the keys 32 (t / 32) .. + 31 of each
// tile (one 32-bit load of V per key), and the four key quarters are summed
// once per split.
// K rows are stored with their 16-byte chunks XOR-swizzled by (row & 7), so
// that a warp reading one chunk of 32 different rows hits 32 distinct banks.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fp8attn {

constexpr int kDecodeMaxG = 8;       // query heads per kv head
constexpr int kDecodePartStride = 130;  // floats per (query row, split): acc[128], m, l

struct DecodeParams {
  const uint8_t* q;  // [B, H, 128] E4M3
  const uint8_t* k;  // [B, Hkv, N, 128] E4M3
  const uint8_t* v;  // [B, Hkv, N, 128] E4M3
  float* part;       // [B * H, splits, 130]
  void* o;           // [B, H, 128] bfloat16
  float* lse;        // [B, H] or nullptr
  int B, H, Hkv, N, G;
  int splits, split_tiles, ntiles;
  int reverse;
  float scale_log2;    // log2(e) / sqrt(128)
  float log2_p_scale;  // log2(S)
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Four E4M3 bytes of a 32-bit word to float32 (exact).
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float& a, float& b, float& c, float& d) {
  uint32_t lo, hi;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(lo) : "h"(static_cast<uint16_t>(w & 0xFFFFu)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hi) : "h"(static_cast<uint16_t>(w >> 16)));
  const __half2 l2 = *reinterpret_cast<const __half2*>(&lo);
  const __half2 h2 = *reinterpret_cast<const __half2*>(&hi);
  a = __low2float(l2), b = __high2float(l2), c = __low2float(h2), d = __high2float(h2);
}

// The E4M3 value nearest to x (round to nearest even, saturating), as float32.
__device__ __forceinline__ float e4m3_round(float x) {
  const uint32_t c = cvt_e4m3x2(x, 0.0f);
  float a, b, cc, dd;
  e4m3x4_to_f32(c, a, b, cc, dd);
  return a;
}

__global__ void __launch_bounds__(128) decode_split_kernel(const DecodeParams p) {
  constexpr int kTile = 128 * 128;  // bytes of one K or V tile
  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t* sK = dsm;                            // 2 x 16 KB, swizzled rows
  uint8_t* sV = dsm + 2 * kTile;                // 2 x 16 KB
  float* sQ = reinterpret_cast<float*>(dsm + 4 * kTile);  // [G][128]
  float* sP = sQ + kDecodeMaxG * 128;                     // [128 keys][8] P^ values
  float* sRed = sP + kDecodeMaxG * 128;                   // [4 warps][G]
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int split = blockIdx.x, zkv = blockIdx.y;  // zkv = b * Hkv + hkv
  const int b = zkv / p.Hkv, hkv = zkv - b * p.Hkv;
  const int G = p.G;
  const int tile0 = split * p.split_tiles;
  const int nt = min(p.split_tiles, p.ntiles - tile0);
  const uint8_t* kbase = p.k + static_cast<int64_t>(zkv) * p.N * 128;
  const uint8_t* vbase = p.v + static_cast<int64_t>(zkv) * p.N * 128;

  // Query rows of the G heads, decoded.
  for (int i = t; i < G * 128; i += 128) {
    const int g = i >> 7, c = i & 127;
    const uint8_t code = p.q[(static_cast<int64_t>(b) * p.H + hkv * G + g) * 128 + c];
    float a, bb, cc, dd;
    e4m3x4_to_f32(code, a, bb, cc, dd);
    sQ[i] = a;
  }

  auto tile_of = [&](int i) { return tile0 + (p.reverse ? nt - 1 - i : i); };
  // Issues the copies of tile `tile` into buffer `buf`; rows at or past N are zero-filled.
  auto fetch = [&](int tile, int buf) {
    const uint32_t dK = smem_u32(sK + buf * kTile), dV = smem_u32(sV + buf * kTile);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = t + 128 * r, row = i >> 3, chunk = i & 7;
      const int key = tile * 128 + row;
      const bool in = key < p.N;
      const int64_t off = static_cast<int64_t>(in ? key : 0) * 128 + chunk * 16;
      cp_async16(dK + row * 128 + ((chunk ^ (row & 7)) << 4), kbase + off, in ? 16u : 0u);
      cp_async16(dV + row * 128 + (chunk << 4), vbase + off, in ? 16u : 0u);
    }
    cp_async_commit();
  };

  float m[kDecodeMaxG], l[kDecodeMaxG], acc[kDecodeMaxG][4];
#pragma unroll
  for (int g = 0; g < kDecodeMaxG; ++g) {
    m[g] = -INFINITY, l[g] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[g][j] = 0.0f;
  }
  const float c = p.scale_log2;

  fetch(tile_of(0), 0);
  for (int i = 0; i < nt; ++i) {
    const int buf = i & 1;
    const int tile = tile_of(i);
    if (i + 1 < nt) {
      fetch(tile_of(i + 1), buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    // S for key t of this tile, against every query row.
    float s[kDecodeMaxG];
#pragma unroll
    for (int g = 0; g < kDecodeMaxG; ++g) s[g] = 0.0f;
    const uint8_t* krow = sK + buf * kTile + t * 128;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 w = *reinterpret_cast<const uint4*>(krow + ((ch ^ (t & 7)) << 4));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float k0, k1, k2, k3;
        e4m3x4_to_f32(ws[j], k0, k1, k2, k3);
        const int col = ch * 16 + j * 4;
#pragma unroll
        for (int g = 0; g < kDecodeMaxG; ++g) {
          if (g < G) {
            const float* qg = sQ + g * 128 + col;
            s[g] = fmaf(k0, qg[0], s[g]);
            s[g] = fmaf(k1, qg[1], s[g]);
            s[g] = fmaf(k2, qg[2], s[g]);
            s[g] = fmaf(k3, qg[3], s[g]);
          }
        }
      }
    }
    const bool valid = tile * 128 + t < p.N;
    // Tile maximum of every row: warp, then across the four warps.
#pragma unroll
    for (int g = 0; g < kDecodeMaxG; ++g) {
      if (g < G) {
        float x = valid ? s[g] : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
        if (lane == 0) sRed[warp * kDecodeMaxG + g] = x;
      }
    }
    __syncthreads();
    float alpha[kDecodeMaxG];
#pragma unroll
    for (int g = 0; g < kDecodeMaxG; ++g) {
      alpha[g] = 1.0f;
      if (g < G) {
        const float tmax = fmaxf(fmaxf(sRed[g], sRed[kDecodeMaxG + g]),
                                 fmaxf(sRed[2 * kDecodeMaxG + g], sRed[3 * kDecodeMaxG + g]));
        const float m_new = fmaxf(m[g], tmax * c);
        alpha[g] = (m_new == m[g]) ? 1.0f : ex2_approx(m[g] - m_new);
        m[g] = m_new;
        // P * S for key t: the scale enters the exponent; masked keys give 0.
        const float ps = valid ? ex2_approx(fmaf(s[g], c, p.log2_p_scale - m_new)) : 0.0f;
        s[g] = ps;
        sP[t * kDecodeMaxG + g] = e4m3_round(ps);
      }
    }
    __syncthreads();  // every thread has read sRed (maxima) and written sP
#pragma unroll
    for (int g = 0; g < kDecodeMaxG; ++g) {
      if (g < G) {
        float x = s[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) sRed[warp * kDecodeMaxG + g] = x;
      }
    }
    // P^ V: columns 4 cg .. 4 cg + 3 over this thread's quarter of the keys.
#pragma unroll
    for (int g = 0; g < kDecodeMaxG; ++g) {
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[g][j] *= alpha[g];
    }
    const uint8_t* vtile = sV + buf * kTile + (lane << 2);
#pragma unroll 4
    for (int kk = 0; kk < 32; ++kk) {
      const int key = (warp << 5) + kk;
      float v0, v1, v2, v3;
      e4m3x4_to_f32(*reinterpret_cast<const uint32_t*>(vtile + key * 128), v0, v1, v2, v3);
      const float4 pa = *reinterpret_cast<const float4*>(sP + key * kDecodeMaxG);
      const float4 pb = *reinterpret_cast<const float4*>(sP + key * kDecodeMaxG + 4);
      const float pg[kDecodeMaxG] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int g = 0; g < kDecodeMaxG; ++g) {
        if (g < G) {
          acc[g][0] = fmaf(pg[g], v0, acc[g][0]);
          acc[g][1] = fmaf(pg[g], v1, acc[g][1]);
          acc[g][2] = fmaf(pg[g], v2, acc[g][2]);
          acc[g][3] = fmaf(pg[g], v3, acc[g][3]);
        }
      }
    }
    __syncthreads();  // sums in sRed; every read of sP and of this buffer done
#pragma unroll
    for (int g = 0; g < kDecodeMaxG; ++g) {
      if (g < G) {
        const float tsum = (sRed[g] + sRed[kDecodeMaxG + g]) + (sRed[2 * kDecodeMaxG + g] + sRed[3 * kDecodeMaxG + g]);
        l[g] = l[g] * alpha[g] + tsum;  // l * S
      }
    }
    __syncthreads();  // sRed is rewritten by the next tile's maxima
  }
  // Sum of the four key quarters (through the K buffers, free now), then
  // the partial results of this split.
  float* sAcc = reinterpret_cast<float*>(dsm);  // [4 quarters][G][128]
#pragma unroll
  for (int g = 0; g < kDecodeMaxG; ++g) {
    if (g < G) {
      *reinterpret_cast<float4*>(sAcc + (warp * kDecodeMaxG + g) * 128 + (lane << 2)) =
          make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int g = 0; g < kDecodeMaxG; ++g) {
    if (g < G) {
      const float sum = (sAcc[(0 * kDecodeMaxG + g) * 128 + t] + sAcc[(1 * kDecodeMaxG + g) * 128 + t]) +
                        (sAcc[(2 * kDecodeMaxG + g) * 128 + t] + sAcc[(3 * kDecodeMaxG + g) * 128 + t]);
      float* dst = p.part + (static_cast<int64_t>(b * p.H + hkv * G + g) * p.splits + split) * kDecodePartStride;
      dst[t] = sum;
      if (t == 0) {
        dst[128] = m[g];
        dst[129] = l[g];
      }
    }
  }
}

// Merge of the splits of one query row: O = sum_s 2^(m_s - M) acc_s /
// sum_s 2^(m_s - M) l_s (l carries the factor S), lse = (M + log2 L - log2 S) ln 2.
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  const int row = blockIdx.x;  // b * H + h
  const int t = threadIdx.x;
  const float* part = p.part + static_cast<int64_t>(row) * p.splits * kDecodePartStride;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, part[s * kDecodePartStride + 128]);
  float num = 0.0f, den = 0.0f;
  for (int s = 0; s < p.splits; ++s) {
    const float* ps = part + s * kDecodePartStride;
    const float w = ex2_approx(ps[128] - M);
    num = fmaf(w, ps[t], num);
    den = fmaf(w, ps[129], den);
  }
  const float o = num / den;
  uint16_t* orow = static_cast<uint16_t*>(p.o) + static_cast<int64_t>(row) * 128;
  orow[t] = static_cast<uint16_t>(pack_bf16x2(o, 0.0f) & 0xFFFFu);
  if (t == 0 && p.lse != nullptr) p.lse[row] = (M + (log2f(den) - p.log2_p_scale)) * 0.6931471805599453f;
}

}  // namespace fp8attn
