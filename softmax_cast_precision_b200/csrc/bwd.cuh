// bwd.cuh -- backward pass of the P-cast attention on sm_100a (d = 128).
//
// The gradients are those of the recomputation form of "Attenzione flash e
// domanda sulla lunghezza della sequenza" (FlashAttention keeps O and the
// log-sum-exp and recomputes P from them), with the P-cast of "P-Cast
// Precision in FP8 Attention", technical summary, section 1, kept where the
// forward pass applies it, on the probabilities that multiply V:
//
//   P_ij  = exp(s_ij - lse_i),  s_ij = q_i . k_j / sqrt(d)   (masked: 0)
//   dV_j  = sum_i E4M3(P_ij S) dO_i / S
//   dP_ij = dO_i . v_j,   D_i = dO_i . O_i,   dS_ij = P_ij (dP_ij - D_i)
//   dQ_i  = sum_j dS_ij k_j / sqrt(d),   dK_j = sum_i dS_ij q_i / sqrt(d)
//
// The cast is the identity for differentiation (dS uses the unquantised P).
//
// Four kernels, all on the caller's stream:
//   bwd_delta_kernel  D_i = dO_i . O_i (one warp per row);
//   bwd_widen_kernel  bfloat16 copies of K and V, written into the dK and dV
//                     output buffers (free until bwd_dkdv_kernel writes them);
//   bwd_dkdv_kernel   one CTA per (batch, kv head, 128-key tile): for every
//                     query head of the group and every query tile that sees
//                     the keys, S^T = K Q^T and dP^T = V dO^T on the tensor
//                     cores, P^T, E4M3(P^T S) and dS^T in registers, then
//                     dV += E4M3(P^T S) dO and dK += dS^T Q accumulated in
//                     tensor memory; no atomics (the group's heads are summed
//                     in the CTA);
//   bwd_dq_kernel     one CTA per (batch, head, 128-row query tile): S and dP
//                     recomputed per key tile, dQ += dS K in tensor memory,
//                     K and V loaded in bfloat16 from the widened copies;
//                     it runs before bwd_dkdv_kernel, which overwrites them.
//
// Operands.  Q, K and V are E4M3 and dO is bfloat16.  S (S^T) multiplies two
// E4M3 tiles (kind::f8f6f4).  The products with dO or dS take both operands
// in bfloat16 (kind::f16): the E4M3 tiles are converted, exactly (every E4M3
// value is a bfloat16 value) -- V and each Q tile in shared memory by the dK/dV
// kernel, K and V once in global memory for the dQ kernel -- and so are the
// cast probabilities E4M3(P S); dS is rounded to bfloat16 (nearest even).  Every
// 16-bit tile is 128 rows x 128 columns stored as two 64-column panels under
// the 128-byte swizzle (16 KB apart), the layout a TMA box of 64 bfloat16
// columns writes; the MMAs read it K-major (K along the row) or MN-major (M
// or N along the row) as each product needs.  Accumulators are FP32 in
// tensor memory and the gradients are written in FP32.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace fp8attn {

struct BwdParams {
  const void* o;       // bf16 [B, H, N, 128]
  const void* dout;    // bf16 [B, H, N, 128]
  const float* lse;    // f32  [B, H, N], natural log
  float* delta;        // f32  [B, H, N]: D_i (written by bwd_delta_kernel)
  float* dq;           // f32  [B, H, N, 128]
  float* dk;           // f32  [B, Hkv, N, 128]
  float* dv;           // f32  [B, Hkv, N, 128]
  int B, H, Hkv, N;
  int h_per_kv;        // H / Hkv
  int causal;
  int num_tiles;       // ceil(N / 128), query and key tiles alike
  float p_scale;       // S
  float scale_log2;    // log2(e) / sqrt(128)
  float inv_sqrt_d;    // 1 / sqrt(128)
};

struct BwdConfig {
  static constexpr int T = 128;                   // rows of every tile (queries or keys)
  static constexpr int F8_TILE = T * 128;         // one E4M3 tile: 16 KB
  static constexpr int BF_PANEL = T * 128;        // one 64-column bfloat16 panel: 16 KB
  static constexpr int BF_TILE = 2 * BF_PANEL;    // one bfloat16 tile: 32 KB
  static constexpr uint32_t TMEM_COLS = 512;
};

// Shared-memory layout of bwd_dkdv_kernel (offsets from a 1024-byte aligned base).
struct DkdvLayout {
  static constexpr int OFF_K = 0;                                   // K_j   E4M3
  static constexpr int OFF_VB = OFF_K + BwdConfig::F8_TILE;         // V_j   bf16
  static constexpr int OFF_Q = OFF_VB + BwdConfig::BF_TILE;         // Q_i   E4M3 (first V_j E4M3, converted once)
  static constexpr int OFF_QB = OFF_Q + BwdConfig::F8_TILE;         // Q_i   bf16
  static constexpr int OFF_DO = OFF_QB + BwdConfig::BF_TILE;        // dO_i  bf16, two buffers (step parity)
  static constexpr int OFF_PT = OFF_DO + 2 * BwdConfig::BF_TILE;    // E4M3(P^T S) as bf16
  static constexpr int OFF_DST = OFF_PT + BwdConfig::BF_TILE;       // dS^T  bf16
  static constexpr int OFF_VEC = OFF_DST + BwdConfig::BF_TILE;      // lse_i * log2(e) [128], D_i [128]
  static constexpr int OFF_BAR = OFF_VEC + 2 * 128 * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 192 + 1024;           // barriers, TMEM slot, alignment slack
};

// Shared-memory layout of bwd_dq_kernel.
struct DqLayout {
  static constexpr int OFF_Q = 0;                                   // Q_i   E4M3
  static constexpr int OFF_DO = OFF_Q + BwdConfig::F8_TILE;         // dO_i  bf16
  static constexpr int OFF_K = OFF_DO + BwdConfig::BF_TILE;         // K_j   E4M3
  static constexpr int OFF_KB = OFF_K + BwdConfig::F8_TILE;         // K_j   bf16, two buffers (step parity)
  static constexpr int OFF_VB = OFF_KB + 2 * BwdConfig::BF_TILE;    // V_j   bf16
  static constexpr int OFF_DS = OFF_VB + BwdConfig::BF_TILE;        // dS    bf16
  static constexpr int OFF_BAR = OFF_DS + BwdConfig::BF_TILE;
  static constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;
};

// Every swizzled tile starts on a 1024-byte boundary (the 128-byte swizzle
// pattern repeats every 8 rows of 128 bytes and is keyed to address bits
// 7..9), and each kernel fits the 227 KB a CTA may opt into.
static_assert(DkdvLayout::OFF_VB % 1024 == 0 && DkdvLayout::OFF_Q % 1024 == 0 &&
                  DkdvLayout::OFF_QB % 1024 == 0 && DkdvLayout::OFF_DO % 1024 == 0 &&
                  DkdvLayout::OFF_PT % 1024 == 0 && DkdvLayout::OFF_DST % 1024 == 0,
              "dK/dV tiles must be 1024-byte aligned");
static_assert(DqLayout::OFF_DO % 1024 == 0 && DqLayout::OFF_K % 1024 == 0 &&
                  DqLayout::OFF_KB % 1024 == 0 && DqLayout::OFF_VB % 1024 == 0 && DqLayout::OFF_DS % 1024 == 0,
              "dQ tiles must be 1024-byte aligned");
static_assert(DkdvLayout::OFF_BAR % 8 == 0 && DqLayout::OFF_BAR % 8 == 0, "mbarriers are 8-byte aligned");
static_assert(DkdvLayout::SMEM_BYTES <= 227 * 1024 && DqLayout::SMEM_BYTES <= 227 * 1024,
              "shared memory beyond the per-CTA opt-in limit");

// Instruction descriptor for kind::f16 with bfloat16 A and B and an FP32
// accumulator, with the operand majors given (bit 15: A MN-major, bit 16: B
// MN-major).
__host__ __device__ constexpr uint32_t bwd_idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of 16-byte chunk `c` (0..15, eight bfloat16 columns each) of
// row `r` in a two-panel bfloat16 tile: panel c / 8, chunk c % 8 of the
// panel's 128-byte row, XORed with r % 8 (the 128-byte swizzle).
__device__ __forceinline__ uint32_t bf16_tile_chunk(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * BwdConfig::BF_PANEL + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Four E4M3 codes (one 32-bit word, lowest byte first) to four bfloat16
// values in two words (exact: E4M3 -> f16 -> f32 -> bf16 loses nothing).
__device__ __forceinline__ uint2 bwd_e4m3x4_to_bf16x4(uint32_t w) {
  uint32_t lo, hi;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(lo) : "h"(static_cast<uint16_t>(w & 0xFFFFu)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hi) : "h"(static_cast<uint16_t>(w >> 16)));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  return make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(b.x, b.y));
}

// Part h of row `r` of an E4M3 tile (128 bytes per row, 128-byte swizzle, as
// TMA wrote it) into row `r` of a two-panel bfloat16 tile: E4M3 columns
// 16 NC h .. 16 NC (h + 1) - 1, so that 8 / NC threads share a row.
template <int NC>
__device__ __forceinline__ void bwd_convert_part_row(const uint8_t* src, uint8_t* dst, int r, int h) {
  const uint32_t s = smem_u32(src), d = smem_u32(dst);
#pragma unroll
  for (int cc = 0; cc < NC; ++cc) {
    const int c = NC * h + cc;
    uint32_t w0, w1, w2, w3;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                 : "r"(s + r * 128 + ((c ^ (r & 7)) << 4))
                 : "memory");
    const uint2 a = bwd_e4m3x4_to_bf16x4(w0), b = bwd_e4m3x4_to_bf16x4(w1);
    const uint2 e = bwd_e4m3x4_to_bf16x4(w2), f = bwd_e4m3x4_to_bf16x4(w3);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(d + bf16_tile_chunk(r, 2 * c)), "r"(a.x),
                 "r"(a.y), "r"(b.x), "r"(b.y)
                 : "memory");
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(d + bf16_tile_chunk(r, 2 * c + 1)), "r"(e.x),
                 "r"(e.y), "r"(f.x), "r"(f.y)
                 : "memory");
  }
}

// Shared-memory float stores and 16-byte loads by shared address.
__device__ __forceinline__ void sts_f32(uint32_t addr, float x) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(x) : "memory");
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Stores 32 FP32 values (columns 32*g .. 32*g+31 of row `r`) as bfloat16
// chunks 4g .. 4g+3 of a two-panel tile.
__device__ __forceinline__ void bwd_store_bf16_32(uint8_t* dst, int r, int g, const float (&x)[32]) {
  const uint32_t d = smem_u32(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w0 = pack_bf16x2(x[8 * q + 0], x[8 * q + 1]);
    const uint32_t w1 = pack_bf16x2(x[8 * q + 2], x[8 * q + 3]);
    const uint32_t w2 = pack_bf16x2(x[8 * q + 4], x[8 * q + 5]);
    const uint32_t w3 = pack_bf16x2(x[8 * q + 6], x[8 * q + 7]);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(d + bf16_tile_chunk(r, 4 * g + q)), "r"(w0),
                 "r"(w1), "r"(w2), "r"(w3)
                 : "memory");
  }
}

// bfloat16 pair (lo in the low half) of the E4M3 values nearest to lo and
// hi (nearest even, saturating): exact, every E4M3 value being a bfloat16.
__device__ __forceinline__ uint32_t bwd_e4m3_pair_bf16(float lo, float hi) {
  const uint32_t code = cvt_e4m3x2(lo, hi);
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(code)));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x, f.y);
}

// 16 values (columns 8 c0 .. 8 c0 + 15 of row `r`) as bfloat16 chunks c0 and
// c0 + 1 of a two-panel tile: from FP32 values, or already packed in pairs.
__device__ __forceinline__ void bwd_store_bf16_16(uint8_t* dst, int r, int c0, const float (&x)[16]) {
  const uint32_t d = smem_u32(dst);
#pragma unroll
  for (int q = 0; q < 2; ++q)
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(d + bf16_tile_chunk(r, c0 + q)),
                 "r"(pack_bf16x2(x[8 * q + 0], x[8 * q + 1])), "r"(pack_bf16x2(x[8 * q + 2], x[8 * q + 3])),
                 "r"(pack_bf16x2(x[8 * q + 4], x[8 * q + 5])), "r"(pack_bf16x2(x[8 * q + 6], x[8 * q + 7]))
                 : "memory");
}
__device__ __forceinline__ void bwd_store_bf16_16_packed(uint8_t* dst, int r, int c0, const uint32_t (&w)[8]) {
  const uint32_t d = smem_u32(dst);
#pragma unroll
  for (int q = 0; q < 2; ++q)
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(d + bf16_tile_chunk(r, c0 + q)), "r"(w[4 * q]),
                 "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                 : "memory");
}

// Descriptors of the three operand forms (start address, LBO, SBO, 128-byte
// swizzle), with the per-step start-address advance of a K step:
//   E4M3 tile, K-major:     32 columns = 32 bytes per step (+2 in the >> 4 field);
//   (kmajor_desc serves both K-major forms: only the step differs)
//   bf16 tile, K-major:     16 columns = 32 bytes (+2), four steps per panel,
//                           then the next panel (+16 KB);
//   bf16 tile, MN-major:    16 rows = 2048 bytes (+128); the N (or M) extent of
//                           128 spans both panels, LBO = 16 KB apart.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }

// Warpgroups of the two tensor-core backward kernels: each thread keeps one
// TMEM lane (row) and takes 4 / kBwdGroups of the row's four 32-column chunks.
constexpr int kBwdGroups = 4;
constexpr int kBwdChunks = 4 / kBwdGroups;
__device__ __forceinline__ uint64_t bf16_kmajor_step(int kk) {
  return static_cast<uint64_t>((kk >> 2) * (BwdConfig::BF_PANEL >> 4) + 2 * (kk & 3));
}
__device__ __forceinline__ uint64_t bf16_mnmajor_desc(uint32_t saddr) {
  return smem_desc(saddr, BwdConfig::BF_PANEL, 1024, 2);
}

// --------------------------------------------------------------------------
// D_i = dO_i . O_i in FP32, one warp per row (4 columns per lane).
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_delta_kernel(const BwdParams p) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.N;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint2 a = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.dout) + row * 128)[lane];
  const uint2 b = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.o) + row * 128)[lane];
  auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
  auto hi = [](uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); };
  float s = lo(a.x) * lo(b.x);
  s = fmaf(hi(a.x), hi(b.x), s);
  s = fmaf(lo(a.y), lo(b.y), s);
  s = fmaf(hi(a.y), hi(b.y), s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) p.delta[row] = s;
}

// E4M3 rows [n16 / 8][128] to bfloat16 rows [n16 / 8][128], 16 codes per
// thread and step (exact, as in the shared-memory conversions).
__global__ void __launch_bounds__(256) bwd_widen_kernel(const uint8_t* src, uint16_t* dst, int64_t n16) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 w = reinterpret_cast<const uint4*>(src)[i];
    const uint2 a = bwd_e4m3x4_to_bf16x4(w.x), b = bwd_e4m3x4_to_bf16x4(w.y);
    const uint2 c = bwd_e4m3x4_to_bf16x4(w.z), e = bwd_e4m3x4_to_bf16x4(w.w);
    uint4* out = reinterpret_cast<uint4*>(dst) + 2 * i;
    out[0] = make_uint4(a.x, a.y, b.x, b.y);
    out[1] = make_uint4(c.x, c.y, e.x, e.y);
  }
}

// --------------------------------------------------------------------------
// dK and dV: one CTA per (batch, kv head, key tile).
//
// Roles: a TMA/MMA warp (warp 16, lane 0 issues) and two pairs of
// warpgroups.  Pair p owns query half p (queries 64 p .. 64 p + 63) of every
// step (query tile), with its own S^T / dP^T buffers in tensor memory (64
// columns each), its own panel of the P^ and dS^T tiles and its own half of
// Q's bfloat16 copy; within a pair, thread (key r, chunk c) takes 32 of the
// half's 64 queries.  The MMA warp issues, for each step, each half's
// products in a fixed order (so dV and dK sum in a fixed order): S^T and dP^T
// of a half as soon as its inputs have landed, dV and dK of a half as soon as
// its pair has written P^ and dS^T.  While one pair computes, the tensor core
// works for the other.
// --------------------------------------------------------------------------
constexpr int kDkdvCompute = 512;                 // two pairs of warpgroups
constexpr int kDkdvThreads = kDkdvCompute + 32;   // + the TMA/MMA warp

struct DkdvBars {
  uint64_t kv;           // K_j and V_j landed
  uint64_t q[2];         // Q half p of the step landed
  uint64_t dout[2];      // dO of the step landed, one barrier per buffer (step parity)
  uint64_t s_full[2];    // S^T and dP^T of half p computed
  uint64_t qb_ready[2];  // pair p has converted its half of Q to bfloat16 (256 arrivals)
  uint64_t p_full[2];    // pair p has written P^ and dS^T (256 arrivals)
  uint64_t g_done[2];    // dV and dK products of half p complete
  uint64_t drain;        // every product issued so far complete (end of the kernel)
  uint32_t tmem_base;
};

// Pair-wide OR of `v` over the 256 threads of pair p (named barrier 1 + p).
__device__ __forceinline__ bool pair_any(int p, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "barrier.red.or.pred b, %2, 256, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(1 + p)
      : "memory");
  return r != 0;
}

static_assert(sizeof(DkdvBars) <= 192, "dK/dV control block exceeds its shared-memory slot");

__global__ void __launch_bounds__(kDkdvThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p, uint32_t* err_word) {
  using L = DkdvLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // lse_i * log2(e) and D_i of the step's queries; written and read through
  // shared-memory addresses (generic pointers here would become generic loads).
  const uint32_t sLse2 = smem_u32(base + L::OFF_VEC), sDelta = sLse2 + 128 * 4;
  DkdvBars* bars = reinterpret_cast<DkdvBars*>(base + L::OFF_BAR);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int jt = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int k0 = jt * 128;
  const int zkv = b * p.Hkv + hk;
  const int i_first = p.causal ? jt : 0;  // query tiles before the key tile see none of its keys
  const int per_head = p.num_tiles - i_first;
  const int n_iter = p.h_per_kv * per_head;
  auto step_geom = [&](int it, int& zq, int& q0) {
    const int hl = it / per_head;
    q0 = (i_first + (it - hl * per_head)) * 128;
    zq = b * p.H + hk * p.h_per_kv + hl;
  };

  if (tid == kDkdvCompute) {
    mbar_init(&bars->kv, 1);
    mbar_init(&bars->drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q[i], 1);
      mbar_init(&bars->dout[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->qb_ready[i], 256);
      mbar_init(&bars->p_full[i], 256);
      mbar_init(&bars->g_done[i], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_q64);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, BwdConfig::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tDV = tmem + 256, tDK = tmem + 384;  // S^T / dP^T of half p at 128 p / 128 p + 64

  // Loads (lane 0 of the MMA warp).
  auto issue_q_half = [&](int it, int h) {
    int zq, q0;
    step_geom(it, zq, q0);
    mbar_arrive_expect_tx(&bars->q[h], BwdConfig::F8_TILE / 2);
    tma_load_3d(base + L::OFF_Q + h * (BwdConfig::F8_TILE / 2), &tm_q64, &bars->q[h], 0, q0 + 64 * h, zq);
  };
  auto issue_do = [&](int it) {
    int zq, q0;
    step_geom(it, zq, q0);
    uint8_t* dst = base + L::OFF_DO + (it & 1) * BwdConfig::BF_TILE;
    mbar_arrive_expect_tx(&bars->dout[it & 1], BwdConfig::BF_TILE);
    tma_load_3d(dst, &tm_do, &bars->dout[it & 1], 0, q0, zq);
    tma_load_3d(dst + BwdConfig::BF_PANEL, &tm_do, &bars->dout[it & 1], 64, q0, zq);
  };
  if (tid == kDkdvCompute) {
    // V_j (E4M3) lands in the Q buffer, to be converted once.
    mbar_arrive_expect_tx(&bars->kv, 2 * BwdConfig::F8_TILE);
    tma_load_3d(base + L::OFF_K, &tm_k, &bars->kv, 0, k0, zkv);
    tma_load_3d(base + L::OFF_Q, &tm_v, &bars->kv, 0, k0, zkv);
    if (n_iter > 0) issue_do(0);
    if (n_iter > 1) issue_do(1);
  }
  bool fail = false;
  if (tid < kDkdvCompute) {
    fail = !mbar_wait_bounded(&bars->kv, 0, err_word, kErrTimeoutKV);
    if (!fail) bwd_convert_part_row<2>(base + L::OFF_Q, base + L::OFF_VB, tid & 127, tid >> 7);
    fence_proxy_async_smem();  // every thread has read V out of the Q buffer before Q may overwrite it
  }
  bool abort = __syncthreads_or(fail) != 0;

  const uint32_t sK = smem_u32(base + L::OFF_K), sVB = smem_u32(base + L::OFF_VB);
  const uint32_t sQ = smem_u32(base + L::OFF_Q), sQB = smem_u32(base + L::OFF_QB);
  const uint32_t sPT = smem_u32(base + L::OFF_PT), sDST = smem_u32(base + L::OFF_DST);
  const uint32_t sDO0 = smem_u32(base + L::OFF_DO);
  int q_issued[2] = {0, 0}, q_landed[2] = {0, 0}, do_issued = n_iter > 1 ? 2 : n_iter, do_landed = 0;

  if (tid == kDkdvCompute && !abort && n_iter > 0) {
    // ----------------------------- TMA / MMA lane -----------------------------
    constexpr uint32_t idesc_s = idesc_e4m3_f32(128, 64, false, false);   // S^T = K Q_h^T (N = 64 queries)
    constexpr uint32_t idesc_dp = bwd_idesc_bf16(128, 64, false, false);  // dP^T = V dO_h^T
    constexpr uint32_t idesc_grad = bwd_idesc_bf16(128, 128, false, true);  // dV += P^T dO_h, dK += dS^T Q_h
    auto q_half = [&](int it, int h) {
      issue_q_half(it, h);
      ++q_issued[h];
    };
    // S^T and dP^T of half h of step it, once Q_h and dO of the step have landed.
    auto issue_sdp = [&](int it, int h) -> bool {
      if (!mbar_wait_bounded(&bars->q[h], it & 1, err_word, kErrTimeoutQ)) return false;
      q_landed[h] = it + 1;
      if (!mbar_wait_bounded(&bars->dout[it & 1], (it >> 1) & 1, err_word, kErrTimeoutQ)) return false;
      do_landed = it + 1;
      tc_fence_after();
      const uint32_t tS = tmem + 128 * h, tDP = tS + 64;
      const uint32_t sQh = sQ + h * (BwdConfig::F8_TILE / 2);
      const uint32_t sDOh = sDO0 + (it & 1) * BwdConfig::BF_TILE + h * (BwdConfig::BF_PANEL / 2);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tS, kmajor_desc(sK) + 2 * kk, kmajor_desc(sQh) + 2 * kk, idesc_s, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tDP, kmajor_desc(sVB) + bf16_kmajor_step(kk), kmajor_desc(sDOh) + bf16_kmajor_step(kk), idesc_dp,
                    kk > 0);
      mma_commit(&bars->s_full[h]);
      return true;
    };
    q_half(0, 0);
    q_half(0, 1);
    bool ok = issue_sdp(0, 0) && issue_sdp(0, 1);
    for (int it = 0; ok && it < n_iter; ++it) {
      // dO of step it + 1 goes to the buffer of step it - 1 once both halves' products of that step completed.
      if (it >= 1 && it + 1 < n_iter) {
        ok = mbar_wait_bounded(&bars->g_done[0], (it - 1) & 1, err_word, kErrTimeoutMMA) &&
             mbar_wait_bounded(&bars->g_done[1], (it - 1) & 1, err_word, kErrTimeoutMMA);
        if (!ok) break;
        issue_do(it + 1);
        do_issued = it + 2;
      }
      // Q half h of step it + 1 once S^T(h, it) has completed and pair h has converted its half.
      if (it + 1 < n_iter) {
        for (int h = 0; ok && h < 2; ++h) {
          ok = mbar_wait_bounded(&bars->s_full[h], it & 1, err_word, kErrTimeoutMMA) &&
               mbar_wait_bounded(&bars->qb_ready[h], it & 1, err_word, kErrTimeoutPipe);
          if (ok) q_half(it + 1, h);
        }
        if (!ok) break;
      }
      const uint32_t sDO = sDO0 + (it & 1) * BwdConfig::BF_TILE;
      for (int h = 0; ok && h < 2; ++h) {
        ok = mbar_wait_bounded(&bars->p_full[h], it & 1, err_word, kErrTimeoutPipe);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const bool acc = (it > 0) || (h > 0) || (kk > 0);
          const uint32_t rows = h * (BwdConfig::BF_PANEL / 2);  // queries 64 h .. of the MN-major operands
          mma_bf16_ss(tDV, kmajor_desc(sPT + h * BwdConfig::BF_PANEL) + 2 * kk, bf16_mnmajor_desc(sDO + rows) + 128 * kk,
                      idesc_grad, acc);
          mma_bf16_ss(tDK, kmajor_desc(sDST + h * BwdConfig::BF_PANEL) + 2 * kk,
                      bf16_mnmajor_desc(sQB + rows) + 128 * kk, idesc_grad, acc);
        }
        mma_commit(&bars->g_done[h]);
        if (it + 1 < n_iter) ok = issue_sdp(it + 1, h);
      }
    }
    fail = !ok;
  } else if (tid < kDkdvCompute && !abort) {
    // ----------------------------- compute pairs ------------------------------
    const int pr = tid >> 8, tp = tid & 255, c = tp >> 7, r = tid & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128 * pr + lane_off, tDP = tS + 64;
    const int key = k0 + r;
    // lse (threads 0..63 of the pair) and D (64..127) of the pair's 64 queries, fetched one step ahead.
    auto fetch = [&](int it) -> float {
      if (it >= n_iter || tp >= 128) return 0.0f;
      int zq, q0;
      step_geom(it, zq, q0);
      const int qi = q0 + 64 * pr + (tp & 63);
      if (qi >= p.N) return 0.0f;
      const int64_t idx = static_cast<int64_t>(zq) * p.N + qi;
      return tp < 64 ? p.lse[idx] : p.delta[idx];
    };
    float next_vec = fetch(0);
    for (int it = 0; it < n_iter; ++it) {
      int zq, q0;
      step_geom(it, zq, q0);
      // This pair's previous products read P^, dS^T and its half of Q's bfloat16 copy.
      if (it > 0 && !fail && !mbar_wait_bounded(&bars->g_done[pr], (it - 1) & 1, err_word, kErrTimeoutMMA))
        fail = true;
      if (tp < 64)
        sts_f32(sLse2 + 4 * (64 * pr + tp), next_vec * 1.4426950408889634f);  // lse in log2 units
      else if (tp < 128)
        sts_f32(sDelta + 4 * (64 * pr + tp - 64), next_vec);
      next_vec = fetch(it + 1);
      if (!fail && !mbar_wait_bounded(&bars->q[pr], it & 1, err_word, kErrTimeoutQ)) fail = true;
      // Rows 64 pr .. 64 pr + 63 of Q to bfloat16, a quarter row per thread.
      if (!fail) bwd_convert_part_row<2>(base + L::OFF_Q, base + L::OFF_QB, 64 * pr + (tp & 63), tp >> 6);
      fence_proxy_async_smem();
      mbar_arrive(&bars->qb_ready[pr]);
      // One decision per pair (the barrier also makes the pair's lse/D writes visible).
      if (pair_any(pr, fail)) {
        fail = true;
        break;
      }
      const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->s_full[pr], it & 1, err_word, kErrTimeoutMMA));
      if (ok) {
        tc_fence_after();
        // P^T, E4M3(P^T S) and dS^T for this thread's key and queries 64 pr + 32 c .. + 31,
        // 16 at a time (fewer live registers).
        const int qh0 = q0 + 64 * pr;
        const bool edge = qh0 + 64 > p.N || k0 + 128 > p.N || (p.causal && k0 + 127 > qh0);
#pragma unroll
        for (int sc = 0; sc < 2; ++sc) {
          const int qc0 = 64 * pr + 32 * c + 16 * sc;  // first query column (in the tile) of the piece
          uint32_t rs[16], rdp[16];
          tmem_ld16(tS + 32 * c + 16 * sc, rs);
          tmem_ld16(tDP + 32 * c + 16 * sc, rdp);
          tmem_wait_ld();
          uint32_t php[8];
          float ds[16];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 lv = lds_f32x4(sLse2 + 4 * qc0 + 16 * e4);
            const float4 dv = lds_f32x4(sDelta + 4 * qc0 + 16 * e4);
            const float la[4] = {lv.x, lv.y, lv.z, lv.w}, da[4] = {dv.x, dv.y, dv.z, dv.w};
            float pb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int e = 4 * e4 + i;
              pb[i] = ex2_approx(__uint_as_float(rs[e]) * p.scale_log2 - la[i]);
              if (edge) {
                const int qi = q0 + qc0 + e;
                const bool visible = qi < p.N && key < p.N && (!p.causal || key <= qi);
                pb[i] = visible ? pb[i] : 0.0f;
              }
              ds[e] = pb[i] * (__uint_as_float(rdp[e]) - da[i]);
            }
            php[2 * e4] = bwd_e4m3_pair_bf16(pb[0] * p.p_scale, pb[1] * p.p_scale);
            php[2 * e4 + 1] = bwd_e4m3_pair_bf16(pb[2] * p.p_scale, pb[3] * p.p_scale);
          }
          bwd_store_bf16_16_packed(base + L::OFF_PT, r, qc0 / 8, php);
          bwd_store_bf16_16(base + L::OFF_DST, r, qc0 / 8, ds);
        }
        tc_fence_before();  // the loads of S^T / dP^T are ordered before p_full, which frees them
      } else {
        fail = true;
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->p_full[pr]);
    }
    // The last step's products of both halves.
    if (!fail && n_iter > 0 &&
        (!mbar_wait_bounded(&bars->g_done[0], (n_iter - 1) & 1, err_word, kErrTimeoutMMA) ||
         !mbar_wait_bounded(&bars->g_done[1], (n_iter - 1) & 1, err_word, kErrTimeoutMMA)))
      fail = true;
    tc_fence_after();
  }
  abort = __syncthreads_or(fail || abort) != 0;

  if (!abort && tid < kDkdvCompute) {
    // dV / S and dK / sqrt(d): eight 32-column jobs, two per warpgroup.  Every
    // lane takes part in the warp-wide TMEM loads; lanes past N store nothing.
    const int wg = tid >> 7, r = tid & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = k0 + r;
    const int64_t row = static_cast<int64_t>(zkv) * p.N + key;
#pragma unroll 1
    for (int job = 2 * wg; job < 2 * wg + 2; ++job) {
      const bool is_dv = job < 4;
      const int g = job & 3;
      float* dst = (is_dv ? p.dv : p.dk) + row * 128;
      uint32_t a[32];
      tmem_ld32((is_dv ? tDV : tDK) + lane_off + 32 * g, a);
      tmem_wait_ld();
      if (key < p.N) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 x;
          if (is_dv)
            x = make_float4(__fdiv_rn(__uint_as_float(a[e]), p.p_scale), __fdiv_rn(__uint_as_float(a[e + 1]), p.p_scale),
                            __fdiv_rn(__uint_as_float(a[e + 2]), p.p_scale), __fdiv_rn(__uint_as_float(a[e + 3]), p.p_scale));
          else
            x = make_float4(__uint_as_float(a[e]) * p.inv_sqrt_d, __uint_as_float(a[e + 1]) * p.inv_sqrt_d,
                            __uint_as_float(a[e + 2]) * p.inv_sqrt_d, __uint_as_float(a[e + 3]) * p.inv_sqrt_d);
          reinterpret_cast<float4*>(dst + 32 * g)[e / 4] = x;
        }
      }
    }
  }
  if (tid == kDkdvCompute) {
    // Every product issued has completed before tensor memory is released;
    // after an abort, also the loads still in flight (each wait bounded).
    mma_commit(&bars->drain);
    mbar_wait_bounded(&bars->drain, 0, err_word, kErrTimeoutMMA, 100000000ull);
    if (abort) {
      mbar_wait_bounded(&bars->kv, 0, err_word, kErrTimeoutKV, 100000000ull);
      for (int h = 0; h < 2; ++h)
        for (int j = q_landed[h]; j < q_issued[h]; ++j)
          mbar_wait_bounded(&bars->q[h], j & 1, err_word, kErrTimeoutQ, 100000000ull);
      for (int j = do_landed; j < do_issued; ++j)
        mbar_wait_bounded(&bars->dout[j & 1], (j >> 1) & 1, err_word, kErrTimeoutQ, 100000000ull);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, BwdConfig::TMEM_COLS);
  }
}

// --------------------------------------------------------------------------
// dQ: one CTA (one warpgroup) per (batch, head, query tile).
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(128 * kBwdGroups, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_kb, const __grid_constant__ CUtensorMap tm_vb,
                  const __grid_constant__ CUtensorMap tm_do, const BwdParams p, uint32_t* err_word) {
  using L = DqLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L::OFF_BAR);
  uint64_t* bar_q = bars + 0;   // Q_i and dO_i landed
  uint64_t* bar_kv = bars + 1;  // K_j (E4M3 and bfloat16) and V_j (bfloat16) landed
  uint64_t* bar_s = bars + 2;   // S and dP computed
  uint64_t* bar_g = bars + 3;      // dQ product of this step complete
  uint64_t* bar_drain = bars + 4;  // every product issued so far complete (abort path)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);

  // kBwdGroups warpgroups: thread tid owns TMEM lane (query row) r = tid % 128
  // and, in each step, part wg = tid / 128 of the keys (kBwdChunks chunks of
  // 32).
  const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, r = tid & 127;
  const int it_q = p.num_tiles - 1 - static_cast<int>(blockIdx.x);  // longest causal rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int q0 = it_q * 128;
  const int zq = b * p.H + h;
  const int zkv = b * p.Hkv + h / p.h_per_kv;
  const int last = p.causal ? it_q : p.num_tiles - 1;  // key tiles 0 .. last

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_kb);
    tma_prefetch_desc(&tm_vb);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, BwdConfig::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 256;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;

  int kv_issued = 0, kv_landed = 0;  // thread 0: key tiles issued / waited for (drain after an abort)
  // Key tile j: E4M3 K (for S), and bfloat16 K (for dQ, into buffer j % 2)
  // and V (for dP) as two 64-column boxes each.
  auto issue_kv = [&](int j) {
    kv_issued = j + 1;
    mbar_arrive_expect_tx(bar_kv, BwdConfig::F8_TILE + 2 * BwdConfig::BF_TILE);
    tma_load_3d(base + L::OFF_K, &tm_k, bar_kv, 0, j * 128, zkv);
    uint8_t* kb = base + L::OFF_KB + (j & 1) * BwdConfig::BF_TILE;
    tma_load_3d(kb, &tm_kb, bar_kv, 0, j * 128, zkv);
    tma_load_3d(kb + BwdConfig::BF_PANEL, &tm_kb, bar_kv, 64, j * 128, zkv);
    tma_load_3d(base + L::OFF_VB, &tm_vb, bar_kv, 0, j * 128, zkv);
    tma_load_3d(base + L::OFF_VB + BwdConfig::BF_PANEL, &tm_vb, bar_kv, 64, j * 128, zkv);
  };
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_q, BwdConfig::F8_TILE + BwdConfig::BF_TILE);
    tma_load_3d(base + L::OFF_Q, &tm_q, bar_q, 0, q0, zq);
    tma_load_3d(base + L::OFF_DO, &tm_do, bar_q, 0, q0, zq);
    tma_load_3d(base + L::OFF_DO + BwdConfig::BF_PANEL, &tm_do, bar_q, 64, q0, zq);
    issue_kv(0);
  }

  const uint32_t sQ = smem_u32(base + L::OFF_Q), sDO = smem_u32(base + L::OFF_DO);
  const uint32_t sK = smem_u32(base + L::OFF_K), sKB = smem_u32(base + L::OFF_KB);
  const uint32_t sVB = smem_u32(base + L::OFF_VB), sDS = smem_u32(base + L::OFF_DS);
  constexpr uint32_t idesc_s = idesc_e4m3_f32(128, 128, false, false);   // S = Q K^T
  constexpr uint32_t idesc_dp = bwd_idesc_bf16(128, 128, false, false);  // dP = dO V^T
  constexpr uint32_t idesc_dq = bwd_idesc_bf16(128, 128, false, true);   // dQ += dS K

  const int row = q0 + r;  // this thread's TMEM lane: one query
  const int64_t ridx = static_cast<int64_t>(zq) * p.N + row;
  const float lse2 = row < p.N ? p.lse[ridx] * 1.4426950408889634f : 0.0f;
  const float dlt = row < p.N ? p.delta[ridx] : 0.0f;
  bool fail = !mbar_wait_bounded(bar_q, 0, err_word, kErrTimeoutQ);
  bool abort = false;

  for (int j = 0; j <= last; ++j) {
    const int j0 = j * 128;
    if (!fail && !mbar_wait_bounded(bar_kv, j & 1, err_word, kErrTimeoutKV)) fail = true;
    if (!fail && tid == 0) kv_landed = j + 1;
    tc_fence_before();
    abort = __syncthreads_or(fail) != 0;
    if (abort) break;

    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_f8_ss(tS, kmajor_desc(sQ) + 2 * kk, kmajor_desc(sK) + 2 * kk, idesc_s, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tDP, kmajor_desc(sDO) + bf16_kmajor_step(kk), kmajor_desc(sVB) + bf16_kmajor_step(kk),
                    idesc_dp, kk > 0);
      mma_commit(bar_s);
    }
    if (!mbar_wait_bounded(bar_s, j & 1, err_word, kErrTimeoutMMA)) fail = true;
    tc_fence_after();
    // S and dP have read K and V, and (the products of one thread completing
    // in order) the dQ product of step j - 1 has read the other bfloat16 K
    // buffer: fetch the next key tile while this one is finished.
    if (tid == 0 && !fail && j < last) issue_kv(j + 1);

    // Only tiles on the diagonal or past N mask any (query, key) pair.
    const bool edge = q0 + 128 > p.N || j0 + 128 > p.N || (p.causal && j0 + 127 > q0);
    // dS is single-buffered: the previous step's dQ product must have read it.
    if (j > 0 && !mbar_wait_bounded(bar_g, (j - 1) & 1, err_word, kErrTimeoutMMA)) fail = true;
#pragma unroll 1
    for (int g = kBwdChunks * wg; g < kBwdChunks * (wg + 1); ++g) {
      uint32_t rs[32], rdp[32];
      tmem_ld32(tS + lane_off + 32 * g, rs);
      tmem_ld32(tDP + lane_off + 32 * g, rdp);
      tmem_wait_ld();
      float ds[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float pr = ex2_approx(__uint_as_float(rs[e]) * p.scale_log2 - lse2);
        if (edge) {
          const int kj = j0 + 32 * g + e;
          const bool visible = row < p.N && kj < p.N && (!p.causal || kj <= row);
          pr = visible ? pr : 0.0f;
        }
        ds[e] = pr * (__uint_as_float(rdp[e]) - dlt);
      }
      bwd_store_bf16_32(base + L::OFF_DS, r, g, ds);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    abort = __syncthreads_or(fail) != 0;
    if (abort) break;

    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tDQ, kmajor_desc(sDS) + bf16_kmajor_step(kk),
                    bf16_mnmajor_desc(sKB + (j & 1) * BwdConfig::BF_TILE) + 128 * kk, idesc_dq, (j > 0) || (kk > 0));
      mma_commit(bar_g);
    }
    // Not waited here: the next step converts into the other K buffer and
    // issues its S and dP behind this product; it waits for this product only
    // before it rewrites dS.
  }
  // The last dQ product.
  if (!abort && last >= 0 && !mbar_wait_bounded(bar_g, last & 1, err_word, kErrTimeoutMMA)) fail = true;
  tc_fence_after();
  abort = __syncthreads_or(fail || abort) != 0;

  if (!abort) {
    float* dqrow = p.dq + ridx * 128;
#pragma unroll 1
    for (int g = kBwdChunks * wg; g < kBwdChunks * (wg + 1); ++g) {
      uint32_t a[32];
      tmem_ld32(tDQ + lane_off + 32 * g, a);
      tmem_wait_ld();
      if (row < p.N) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          reinterpret_cast<float4*>(dqrow + 32 * g)[e / 4] =
              make_float4(__uint_as_float(a[e]) * p.inv_sqrt_d, __uint_as_float(a[e + 1]) * p.inv_sqrt_d,
                          __uint_as_float(a[e + 2]) * p.inv_sqrt_d, __uint_as_float(a[e + 3]) * p.inv_sqrt_d);
      }
    }
  }

  if (abort && tid == 0) {
    // A wait ran out: let the products and loads still in flight land before
    // the CTA's tensor and shared memory are released (each wait again bounded).
    mma_commit(bar_drain);
    mbar_wait_bounded(bar_drain, 0, err_word, kErrTimeoutMMA, 100000000ull);
    mbar_wait_bounded(bar_q, 0, err_word, kErrTimeoutQ, 100000000ull);
    for (int j = kv_landed; j < kv_issued; ++j) mbar_wait_bounded(bar_kv, j & 1, err_word, kErrTimeoutKV, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, BwdConfig::TMEM_COLS);
  }
}

}  // namespace fp8attn
