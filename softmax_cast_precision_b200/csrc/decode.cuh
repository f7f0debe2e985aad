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
// The products run as tcgen05 FP8 MMAs with the keys (and, for P^ V, the
// head dimension) as the M = 128 side and the query heads padded to N = 16:
//   S^T [128 keys x 16]  = K [128 keys x d] . Q^T          (K K-major from TMA, Q K-major)
//   O^T [d x 16]        += V^T [d x 128 keys] . P^^T       (V MN-major straight from TMA, P^ K-major)
// Thread t holds key t's 16 logits (TMEM lane t of S^T) and, for the
// rescale and the partials, column d = t of O^T.  The maxima and sums of
// each query head run over the keys: warp shuffles, then the four warps
// through shared memory.  S^T is double-buffered in tensor memory so the
// next tile's product runs during this tile's softmax and P^ V.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
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

constexpr int kTcN = 16;         // query heads padded to the MMA's N

struct DecodeLayout {
  static constexpr int OFF_K = 0;                       // 2 stages x 16 KB (TMA, 128-byte swizzle)
  static constexpr int OFF_V = 2 * 16384;               // 2 stages x 16 KB
  static constexpr int OFF_Q = 4 * 16384;               // Q: 16 rows x 128 B, K-major (B of S^T)
  static constexpr int OFF_P = OFF_Q + 2048;            // P^: 16 rows x 128 keys, K-major (B of O^T)
  static constexpr int OFF_RED = OFF_P + 2048;          // float [2][4 warps][16]: maxima, sums
  static constexpr int OFF_BAR = OFF_RED + 2 * 4 * kTcN * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;
};
static_assert(DecodeLayout::OFF_Q % 1024 == 0 && DecodeLayout::OFF_P % 1024 == 0, "swizzled tiles 1024-aligned");

__global__ void __launch_bounds__(128) decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                         const __grid_constant__ CUtensorMap tm_v,
                                                         const DecodeParams p, uint32_t* err_word) {
  using L = DecodeLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sMax = reinterpret_cast<float*>(base + L::OFF_RED);  // [4][16]
  float* sSum = sMax + 4 * kTcN;                               // [4][16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L::OFF_BAR);
  uint64_t* bar_k = bars + 0;      // per stage: K of a tile landed
  uint64_t* bar_v = bars + 2;      // per stage: V of a tile landed
  uint64_t* bar_s = bars + 4;      // S^T of the next tile computed
  uint64_t* bar_o = bars + 5;      // O^T += P^ V of this tile complete
  uint64_t* bar_drain = bars + 6;  // every product issued so far complete (abort path)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7);

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int split = blockIdx.x, zkv = blockIdx.y;  // zkv = b * Hkv + hkv
  const int b = zkv / p.Hkv, hkv = zkv - b * p.Hkv;
  const int G = p.G;
  const int tile0 = split * p.split_tiles;
  const int nt = min(p.split_tiles, p.ntiles - tile0);
  auto tile_of = [&](int i) { return tile0 + (p.reverse ? nt - 1 - i : i); };

  if (t == 0) {
    for (int i = 0; i < 7; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  // Q rows of the G heads (rows G..15 zero) and an all-zero P^ tile, both in
  // the 128-byte-swizzled K-major layout: row r, 16-byte chunk c at
  // r * 128 + ((c ^ (r & 7)) << 4).
  {
    const int r = t >> 3, c = t & 7;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (r < G) {
      const uint8_t* src = p.q + (static_cast<int64_t>(b) * p.H + hkv * G + r) * 128 + c * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i >> 2] |= static_cast<uint32_t>(src[i]) << (8 * (i & 3));
    }
    const uint32_t off = r * 128 + ((c ^ (r & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(base + L::OFF_Q) + off), "r"(w[0]),
                 "r"(w[1]), "r"(w[2]), "r"(w[3])
                 : "memory");
    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(smem_u32(base + L::OFF_P) + off), "r"(0u)
                 : "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tO = tmem + 32;  // O^T: columns 32 .. 47; S^T buffers at 0 .. 15 and 16 .. 31

  // Thread 0 issues the copies and the products.  K and V of tile i go to
  // stage i % 2 on barriers of their own: a K stage is free once the S^T it
  // fed has completed, so K runs two tiles ahead; a V stage is free once the
  // P^ V it fed has completed.
  int k_issued = 0, k_landed = 0, v_issued = 0, v_landed = 0;  // thread 0: tiles issued / waited for
  auto issue_k = [&](int i) {
    k_issued = i + 1;
    mbar_arrive_expect_tx(bar_k + (i & 1), 16384);
    tma_load_3d(base + L::OFF_K + (i & 1) * 16384, &tm_k, bar_k + (i & 1), 0, tile_of(i) * 128, zkv);
  };
  auto issue_v = [&](int i) {
    v_issued = i + 1;
    mbar_arrive_expect_tx(bar_v + (i & 1), 16384);
    tma_load_3d(base + L::OFF_V + (i & 1) * 16384, &tm_v, bar_v + (i & 1), 0, tile_of(i) * 128, zkv);
  };
  constexpr uint32_t idesc_s = idesc_e4m3_f32(128, kTcN, false, false);
  constexpr uint32_t idesc_o = idesc_e4m3_f32(128, kTcN, true, false);  // A = V^T read MN-major
  const uint64_t dQ = smem_desc(smem_u32(base + L::OFF_Q), 16, 1024, 2);
  const uint64_t dP = smem_desc(smem_u32(base + L::OFF_P), 16, 1024, 2);
  // S^T of tile i into TMEM buffer i % 2, once its K has landed.
  auto issue_s = [&](int i) -> bool {
    if (!mbar_wait_bounded(bar_k + (i & 1), (i >> 1) & 1, err_word, kErrTimeoutKV)) return false;
    k_landed = i + 1;
    tc_fence_after();
    const uint64_t dK = smem_desc(smem_u32(base + L::OFF_K + (i & 1) * 16384), 16, 1024, 2);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tmem + (i & 1) * 16, dK + 2 * kk, dQ + 2 * kk, idesc_s, kk > 0);
    mma_commit(bar_s);
    return true;
  };

  bool fail = false;
  if (t == 0) {
    issue_k(0);
    issue_v(0);
    if (nt > 1) {
      issue_k(1);
      issue_v(1);
    }
    fail = !issue_s(0);
  }

  // m: running maximum of each query head's logits (uniform over the CTA);
  // l: this thread's share of l * S (its keys' unquantised P * S), summed
  // over the CTA once at the end.
  float m[kTcN], l[kTcN];
#pragma unroll
  for (int g = 0; g < kTcN; ++g) m[g] = -INFINITY, l[g] = 0.0f;
  const float c = p.scale_log2;
  bool abort = false;

  for (int i = 0; i < nt; ++i) {
    const int key = tile_of(i) * 128 + t;
    const bool valid = key < p.N;
    // This tile's logits.
    if (!mbar_wait_bounded(bar_s, i & 1, err_word, kErrTimeoutMMA)) fail = true;
    tc_fence_after();
    // S^T(i) is complete, so K stage i % 2 is free for tile i + 2.
    if (t == 0 && !fail && i + 2 < nt) issue_k(i + 2);
    uint32_t rs[16];
    tmem_ld16(tmem + (i & 1) * 16 + lane_off, rs);
    tmem_wait_ld();
    float s[kTcN];
#pragma unroll
    for (int g = 0; g < kTcN; ++g) s[g] = __uint_as_float(rs[g]);
    // Tile maximum of every query head: one warp reduction, then the four warps.
#pragma unroll
    for (int g = 0; g < kTcN; ++g) {
      if (g < G) {
        const float x = warp_max_f32(valid ? s[g] : -INFINITY);
        if (lane == 0) sMax[warp * kTcN + g] = x;
      }
    }
    // The previous P^ V must be complete before P^ and O^T are touched; its
    // V stage is then free for tile i + 1.
    if (i > 0) {
      if (!mbar_wait_bounded(bar_o, (i - 1) & 1, err_word, kErrTimeoutMMA)) fail = true;
      tc_fence_after();
      if (t == 0 && !fail && i + 1 < nt) issue_v(i + 1);
    }
    abort = __syncthreads_or(fail) != 0;
    if (abort) break;
    const float* tm = sMax;
    float alpha[kTcN];
    bool any_rescale = false;
#pragma unroll
    for (int g = 0; g < kTcN; ++g) {
      alpha[g] = 1.0f;
      if (g < G) {
        const float tmax = fmaxf(fmaxf(tm[g], tm[kTcN + g]), fmaxf(tm[2 * kTcN + g], tm[3 * kTcN + g]));
        const float m_new = fmaxf(m[g], tmax * c);
        alpha[g] = (m_new == m[g]) ? 1.0f : ex2_approx(m[g] - m_new);
        any_rescale |= alpha[g] != 1.0f;
        m[g] = m_new;
        // P * S for key t: the scale enters the exponent; masked keys give 0.
        const float ps = valid ? ex2_approx(fmaf(s[g], c, p.log2_p_scale - m_new)) : 0.0f;
        l[g] = l[g] * alpha[g] + ps;
        const uint32_t code = cvt_e4m3x2(ps, 0.0f) & 0xFFu;
        const uint32_t off = g * 128 + ((((t >> 4) ^ (g & 7))) << 4) + (t & 15);
        asm volatile("st.shared.u8 [%0], %1;" ::"r"(smem_u32(base + L::OFF_P) + off), "r"(code) : "memory");
      }
    }
    // O^T *= alpha per query head (column), when any maximum grew; every
    // thread computed the same alphas.
    if (i > 0 && any_rescale) {
      uint32_t o[16];
      tmem_ld16(tO + lane_off, o);
      tmem_wait_ld();
#pragma unroll
      for (int g = 0; g < kTcN; ++g) o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
      tmem_st16(tO + lane_off, o);
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (t == 0) {
      // O^T += V^T P^^T once V(i) has landed: V stage i % 2 read MN-major (32 keys = 32 rows of 128 B per step).
      if (mbar_wait_bounded(bar_v + (i & 1), (i >> 1) & 1, err_word, kErrTimeoutKV)) {
        v_landed = i + 1;
        tc_fence_after();
        const uint64_t dV = smem_desc(smem_u32(base + L::OFF_V + (i & 1) * 16384), 16384, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tO, dV + 256 * kk, dP + 2 * kk, idesc_o, (i > 0) || (kk > 0));
        mma_commit(bar_o);
        if (i + 1 < nt && !issue_s(i + 1)) fail = true;
      } else {
        fail = true;
      }
    }
    // Every thread read this tile's maxima before the barrier above, so the
    // next tile may overwrite them.
  }
  abort = __syncthreads_or(fail || abort) != 0;
  if (!abort && nt > 0) {
    if (!mbar_wait_bounded(bar_o, (nt - 1) & 1, err_word, kErrTimeoutMMA)) abort = true;
    tc_fence_after();
  }
  // l * S of each query head: the threads' shares, summed over the warp, then the warps.
#pragma unroll
  for (int g = 0; g < kTcN; ++g) {
    if (g < G) {
      float x = l[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane == 0) sSum[warp * kTcN + g] = x;
    }
  }
  abort = __syncthreads_or(abort) != 0;
  if (!abort) {
    // Partials of this split: column d = t of O^T for every query head.
    uint32_t o[16];
    tmem_ld16(tO + lane_off, o);
    tmem_wait_ld();
#pragma unroll
    for (int g = 0; g < kTcN; ++g) {
      if (g < G) {
        float* dst = p.part + (static_cast<int64_t>(b * p.H + hkv * G + g) * p.splits + split) * kDecodePartStride;
        dst[t] = __uint_as_float(o[g]);
        if (t == 0) {
          dst[128] = m[g];
          dst[129] = (sSum[g] + sSum[kTcN + g]) + (sSum[2 * kTcN + g] + sSum[3 * kTcN + g]);
        }
      }
    }
  }
  if (abort && t == 0) {
    // A wait ran out: let this CTA's products and tile loads still in flight
    // land before its tensor and shared memory are released (each wait again
    // bounded).
    mma_commit(bar_drain);
    mbar_wait_bounded(bar_drain, 0, err_word, kErrTimeoutMMA, 100000000ull);
    for (int j = k_landed; j < k_issued; ++j)
      mbar_wait_bounded(bar_k + (j & 1), (j >> 1) & 1, err_word, kErrTimeoutKV, 100000000ull);
    for (int j = v_landed; j < v_issued; ++j)
      mbar_wait_bounded(bar_v + (j & 1), (j >> 1) & 1, err_word, kErrTimeoutKV, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
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
