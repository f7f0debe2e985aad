// fwd_v1.cuh -- straightforward sm_100a forward kernel: one CTA (one
// warpgroup) per 128-row query tile, TMA tile loads into a two-stage K/V ring,
// tcgen05 FP8 MMAs into tensor memory, the online softmax with the E4M3
// P-cast in registers, and the P V product from shared memory.
//
// Method: "P-Cast Precision in FP8 Attention: Sink-Induced Collapse and the
// Optimality of S=2^8", technical summary, section 1 (P * S cast to E4M3
// before P V, S divided out in the epilogue; forward or reverse KV order).
// Algorithm: "Attenzione flash e domanda sulla lunghezza della sequenza",
// sections "L'algoritmo Flash Attention" (tiling, running max and sum,
// retroactive rescale) and the causal-masking section (blocks entirely above
// the diagonal are skipped); normalisation deferred to the end as in its
// "FA2" section, item 1.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fp8attn {

struct FwdParams {
  void* o;                      // bf16 [B, H, N, D]          (unused when counting)
  float* lse;                   // f32  [B, H, N] or nullptr  (unused when counting)
  unsigned long long* counts;   // u64  [B, H]                (counting only)
  int B, H, Hkv, N;
  int h_per_kv;                 // H / Hkv
  int causal;
  int reverse;                  // 0: KV block 0 first; 1: last block first
  int n_sink;                   // keys j < n_sink are not counted
  int num_q_tiles;
  int num_kv_tiles;
  int group_heads;               // persistent kernel: (b, h) slabs per scheduling group
  unsigned int* sched;           // persistent kernel: work-unit counter, zero at launch
  float p_scale;                // S
  float scale_log2;             // log2(e) / sqrt(D)
  float log2_p_scale;           // log2(S), rounded to float
  // Descaled inputs (persistent kernel, SCALED instance only): q = q_scale *
  // E4M3 codes per 128-row query tile, k likewise per key tile, v per head.
  const float* q_scales;        // [B * H, num_q_tiles]
  const float* k_scales;        // [B * Hkv, num_kv_tiles]
  const float* v_scales;        // [B * Hkv]
  int unrotate;                 // rotate each output row back by R^T = H_D diag(signs) / sqrt(D)
  uint32_t sign_bits[4];        // bit i set: signs[i] = -1
  // Persistent kernel: how long a wait may last before it gives up (2 s in
  // normal use), and the test switch that makes the producer skip the load
  // of the first K tile, so that a wait runs out on purpose.
  unsigned long long wait_limit_ns;
  int test_withhold_k;
  // Persistent kernel, streamed host calls (nullptr otherwise): the inputs
  // arrive piece by piece, a piece being heads_per_piece consecutive (b, h)
  // slabs.  Word kPieceReady + c is set by the copy stream once piece c is on
  // the device; the kernel counts finished query tiles in kPieceDone + c and
  // sets kPieceFlag + c when piece c's outputs are all stored.
  unsigned int* stream_flags;
  int heads_per_piece;
};

// Word offsets in FwdParams::stream_flags, a 512-byte block (word 0 is the
// work-unit counter when the same block holds both).
constexpr int kMaxPieces = 32;
constexpr int kPieceReady = 32;
constexpr int kPieceDone = 64;
constexpr int kPieceFlag = 96;
constexpr int kPieceBlockBytes = 512;

template <int D>
struct V1Config {
  static constexpr int BM = 128;                    // query rows per tile (TMEM lanes)
  static constexpr int BN = (D == 128) ? 128 : 64;  // keys per KV block
  static constexpr int Q_BYTES = BM * D;
  static constexpr int KV_BYTES = BN * D;
  static constexpr int P_BYTES = BM * BN;
  // Row pitch equals the swizzle span: 128-byte rows use the 128-byte
  // swizzle, 64-byte rows the 64-byte swizzle (tcgen05 descriptor modes).
  static constexpr uint32_t SWZ_QKV = (D == 128) ? 2u : 4u;
  static constexpr uint32_t SWZ_P = (BN == 128) ? 2u : 4u;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K0 = OFF_Q + Q_BYTES;
  static constexpr int OFF_V0 = OFF_K0 + 2 * KV_BYTES;
  static constexpr int OFF_P = OFF_V0 + 2 * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;  // barriers + TMEM slot + alignment slack
  static constexpr uint32_t TMEM_COLS = 256;               // S in [0, BN), O in [128, 128 + D)
  static constexpr uint32_t TMEM_O = 128;
};

// Byte offset of 16-byte chunk `c` of row `r` in a tile whose rows are
// `row_bytes` (128 or 64) long, under the matching hardware swizzle: the
// chunk index is XORed with address bits 7..9 (128-byte) or 7..8 (64-byte).
__device__ __forceinline__ uint32_t swizzled_chunk(int r, int c, int row_bytes) {
  const int x = (row_bytes == 128) ? (r & 7) : ((r >> 1) & 3);
  return static_cast<uint32_t>(r * row_bytes + ((c ^ x) << 4));
}

template <int D, bool COUNT>
__global__ void __launch_bounds__(128, 1)
    fwd_v1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p, uint32_t* err_word) {
  using C = V1Config<D>;
  constexpr int BM = C::BM, BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base + C::OFF_Q;
  uint8_t* sP = base + C::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_kv = bars + 1;  // two stages
  uint64_t* bar_s = bars + 3;
  uint64_t* bar_o = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int qt = p.num_q_tiles - 1 - static_cast<int>(blockIdx.x);  // longest causal rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * BM;
  const int zq = b * p.H + h;
  const int zkv = b * p.Hkv + h / p.h_per_kv;
  int last = p.num_kv_tiles - 1;
  if (p.causal) last = min(last, (q0 + BM - 1) / BN);
  const int ntiles = last + 1;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_kv + 0, 1);
    mbar_init(bar_kv + 1, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + C::TMEM_O;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

  auto kv_tile = [&](int it) { return p.reverse ? (last - it) : it; };

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
    tma_load_3d(sQ, &tm_q, bar_q, 0, q0, zq);
    for (int s = 0; s < 2 && s < ntiles; ++s) {
      mbar_arrive_expect_tx(bar_kv + s, 2 * C::KV_BYTES);
      tma_load_3d(base + C::OFF_K0 + s * C::KV_BYTES, &tm_k, bar_kv + s, 0, kv_tile(s) * BN, zkv);
      tma_load_3d(base + C::OFF_V0 + s * C::KV_BYTES, &tm_v, bar_kv + s, 0, kv_tile(s) * BN, zkv);
    }
  }

  constexpr uint32_t idesc_qk = idesc_e4m3_f32(BM, BN, false, false);
  constexpr uint32_t idesc_pv = idesc_e4m3_f32(BM, D, false, true);
  const uint32_t sQ_a = smem_u32(sQ), sP_a = smem_u32(sP);

  const int row = q0 + tid;
  float m = -INFINITY;  // running max, log2 units
  float l = 0.0f;       // running sum of unquantised P
  uint32_t nzero = 0;
  bool fail = false;
  bool abort = false;

  for (int it = 0; it < ntiles; ++it) {
    const int t = kv_tile(it);
    const int stage = it & 1;
    const int j0 = t * BN;
    const uint32_t sK_a = smem_u32(base + C::OFF_K0 + stage * C::KV_BYTES);
    const uint32_t sV_a = smem_u32(base + C::OFF_V0 + stage * C::KV_BYTES);

    // S = Q K_t^T, FP32 in TMEM columns [0, BN).
    if (tid == 0) {
      bool ready = (it > 0) || mbar_wait_bounded(bar_q, 0, err_word, kErrTimeoutQ);
      ready = ready && mbar_wait_bounded(bar_kv + stage, (it >> 1) & 1, err_word, kErrTimeoutKV);
      if (ready) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t a = smem_desc(sQ_a + kk * 32, 16, 8 * D, C::SWZ_QKV);
          const uint64_t bd = smem_desc(sK_a + kk * 32, 16, 8 * D, C::SWZ_QKV);
          mma_f8_ss(tS, a, bd, idesc_qk, kk > 0);
        }
        mma_commit(bar_s);
      } else {
        fail = true;
      }
    }
    if (!mbar_wait_bounded(bar_s, it & 1, err_word, kErrTimeoutMMA)) fail = true;
    tc_fence_after();

    // Logits of this thread's row, scaled to log2 units and masked.
    float s[BN];
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tS + lane_off + c * 32, r);
#pragma unroll
      for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
    }
    tmem_wait_ld();
    const bool edge = (j0 + BN > p.N) || (p.causal && j0 + BN - 1 > q0);
    float mt = -INFINITY;
#pragma unroll
    for (int c = 0; c < BN; ++c) {
      float x = s[c] * p.scale_log2;
      if (edge) {
        const int j = j0 + c;
        if (j >= p.N || (p.causal && j > row)) x = -INFINITY;
      }
      s[c] = x;
      mt = fmaxf(mt, x);
    }
    // Running max over every block, then P = 2^(x - m_new).
    const float m_new = fmaxf(m, mt);
    const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
    const float alpha = ex2_approx(m - m_use);  // 0 before the first visible key
    float rowsum = 0.0f;
    uint32_t packed[BN / 4];
#pragma unroll
    for (int c = 0; c < BN; c += 4) {
      const float p0 = ex2_approx(s[c + 0] - m_use);
      const float p1 = ex2_approx(s[c + 1] - m_use);
      const float p2 = ex2_approx(s[c + 2] - m_use);
      const float p3 = ex2_approx(s[c + 3] - m_use);
      rowsum += (p0 + p1) + (p2 + p3);
      // The P-cast: P * S rounded to E4M3 (nearest even, saturating).
      const uint32_t lo = cvt_e4m3x2(p0 * p.p_scale, p1 * p.p_scale);
      const uint32_t hi = cvt_e4m3x2(p2 * p.p_scale, p3 * p.p_scale);
      packed[c / 4] = lo | (hi << 16);
      if constexpr (COUNT) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j0 + c + e;
          const bool visible = row < p.N && j < p.N && j >= p.n_sink && (!p.causal || j <= row);
          const uint32_t byte = (packed[c / 4] >> (8 * e)) & 0xFFu;
          nzero += (visible && byte == 0u) ? 1u : 0u;
        }
      }
    }
    l = l * alpha + rowsum;
    m = m_new;

    // The previous P V product must be done before P and O are touched.
    if (it > 0) {
      if (!mbar_wait_bounded(bar_o, (it - 1) & 1, err_word, kErrTimeoutMMA)) fail = true;
      tc_fence_after();
      if (tid == 0 && !fail && it + 1 < ntiles) {
        const int s2 = (it + 1) & 1;
        mbar_arrive_expect_tx(bar_kv + s2, 2 * C::KV_BYTES);
        tma_load_3d(base + C::OFF_K0 + s2 * C::KV_BYTES, &tm_k, bar_kv + s2, 0, kv_tile(it + 1) * BN, zkv);
        tma_load_3d(base + C::OFF_V0 + s2 * C::KV_BYTES, &tm_v, bar_kv + s2, 0, kv_tile(it + 1) * BN, zkv);
      }
    }

    // P^ into shared memory in the K-major swizzled layout the MMA reads.
#pragma unroll
    for (int c = 0; c < BN / 16; ++c) {
      const uint32_t off = swizzled_chunk(tid, c, BN);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sP_a + off), "r"(packed[4 * c + 0]),
                   "r"(packed[4 * c + 1]), "r"(packed[4 * c + 2]), "r"(packed[4 * c + 3])
                   : "memory");
    }

    // Retroactive rescale of the accumulated O by 2^(m_old - m_new) when the
    // running max grew (skipped when alpha == 1 for the whole warp: exact).
    if (it > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
        tmem_st32(tO + lane_off + c * 32, r);
      }
      tmem_wait_st();
    }

    fence_proxy_async_smem();
    tc_fence_before();
    abort = __syncthreads_or(fail) != 0;
    if (abort) break;

    // O += P^ V_t (V is MN-major: d contiguous).
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BN / 32; ++kk) {
        const uint64_t a = smem_desc(sP_a + kk * 32, 16, 8 * BN, C::SWZ_P);
        const uint64_t bd = smem_desc(sV_a + kk * 32 * D, BN * D, 8 * D, C::SWZ_QKV);
        mma_f8_ss(tO, a, bd, idesc_pv, (it > 0) || (kk > 0));
      }
      mma_commit(bar_o);
    }
  }

  if (!abort) {
    if (!mbar_wait_bounded(bar_o, (ntiles - 1) & 1, err_word, kErrTimeoutMMA)) fail = true;
    tc_fence_after();
  }
  abort = __syncthreads_or(fail || abort) != 0;

  if (!abort) {
    if constexpr (COUNT) {
      const uint32_t total = __reduce_add_sync(0xffffffffu, nzero);
      if ((tid & 31) == 0 && total) atomicAdd(p.counts + zq, static_cast<unsigned long long>(total));
    } else {
      // Epilogue: O / (S * l) to bfloat16; lse = (m + log2 l) * ln 2.
      const float den = p.p_scale * l;
      uint8_t* orow = static_cast<uint8_t*>(p.o) + ((static_cast<int64_t>(zq) * p.N + row) * D) * 2;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + lane_off + c * 32, r);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__fdiv_rn(__uint_as_float(r[2 * i]), den), __fdiv_rn(__uint_as_float(r[2 * i + 1]), den));
        if (row < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (p.lse != nullptr && row < p.N) p.lse[static_cast<int64_t>(zq) * p.N + row] = (m + log2f(l)) * 0.6931471805599453f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fp8attn
