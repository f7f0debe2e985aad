// fwd_v2.cuh -- persistent, warp-specialised sm_100a forward kernel (d = 128).
//
// One CTA per SM claims work units from a global counter, in a head-grouped,
// heaviest-first order; a unit is a pair of adjacent 128-row query tiles
// (Q0, Q1) of one (batch, head).  Roles:
//   warps 0-3  softmax for Q0  (TMEM lanes 0..127 of S0 and O0)
//   warps 4-7  softmax for Q1  (TMEM lanes 0..127 of S1 and O1)
//   warp  8    TMA producer: Q pair per unit, K and V tiles through a ring
//   warps 9-10 MMA issuers for Q0 and Q1: S_k = Q_k K^T and O_k += P^_k V
//              (tcgen05, FP8 E4M3); warp 9 owns the tensor-memory allocation
//   warp  11   idle (it completes the producer warpgroup for setmaxnreg)
// Tensor memory: S0 cols [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// The two softmax warpgroups alternate on the tensor core: while one turns
// its S tile into P^, the other query tile's MMA warp runs its products, so
// the tensor core and the exponential/convert pipes overlap.
//
// Per KV tile and query row the arithmetic is that of the simple kernel:
// running max over every block, P = 2^(x - m), l from unquantised P, the
// P-cast E4M3(P * S), exact retroactive rescale of O when the max grew, and
// O / (S * l) at the end ("P-Cast Precision in FP8 Attention", technical
// summary, section 1; "Attenzione flash e domanda sulla lunghezza della
// sequenza", sections "L'algoritmo Flash Attention" and the causal-masking
// section).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

#include "fwd_v1.cuh"
#include "sm100_ptx.cuh"

namespace fp8attn {

struct V2Config {
  static constexpr int D = 128;
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int STAGES = 4;              // largest ring depth (barrier arrays)
  static constexpr int TILE_BYTES = 128 * 128;  // one 128 x 128 E4M3 tile
  static constexpr int THREADS = 384;  // 3 warpgroups
  // Register split (setmaxnreg): the block launches with 168 registers per
  // thread (65536 / 384 rounded down to a multiple of 8); the producer
  // warpgroup gives registers back and the two softmax warpgroups take them.
  static constexpr int LAUNCH_REGS = 168;
  static constexpr int SOFTMAX_REGS = 208;
  static constexpr int PRODUCER_REGS = 80;
  static constexpr uint32_t TMEM_COLS = 512;
};

// Shared-memory layout.  QK16 = false: Q and K are E4M3 (16 KB tiles, one
// 128-byte swizzle panel), K and V rings of 4 stages.  QK16 = true: Q and K
// are bfloat16 (32 KB tiles: two 64-column panels of 128-byte rows), rings
// of 2 stages; V and P^ stay E4M3 either way.
template <bool QK16>
struct V2Layout {
  static constexpr int STAGES = QK16 ? 2 : 4;
  static constexpr int QK_TILE = QK16 ? 2 * V2Config::TILE_BYTES : V2Config::TILE_BYTES;
  static constexpr int OFF_Q = 0;                                         // Q0, Q1
  static constexpr int OFF_K = OFF_Q + 2 * QK_TILE;                       // K ring
  static constexpr int OFF_V = OFF_K + STAGES * QK_TILE;                  // V ring
  static constexpr int OFF_P = OFF_V + STAGES * V2Config::TILE_BYTES;     // P0 x2, P1 x2 (double-buffered)
  static constexpr int OFF_BAR = OFF_P + 4 * V2Config::TILE_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 320 + 1024;  // control block + alignment slack
};

// Shared-memory control block.
struct V2Bars {
  uint64_t q_full[2], q_free;  // q_full[k]: Q_k landed (only for units where Q_k is used)
  uint64_t k_full[V2Config::STAGES], v_full[V2Config::STAGES];
  // Ring stages and the Q pair are released by the softmax threads (256
  // arrivals: each thread arrives twice when the other query tile does not
  // use the tile), not by tensor-core commits, which stall the MMA pipe.
  uint64_t k_free[V2Config::STAGES], v_free[V2Config::STAGES];
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2], o_free[2];
  uint64_t drain[2];  // MMA warps: all issued tensor-core work complete
  // Dynamic schedule: the producer fetches unit ids from a global counter and
  // hands them to the other roles through a two-slot queue.
  uint64_t unit_full[2], unit_empty[2];
  int unit_id[2];
  uint64_t wait_limit_ns;  // bound of every wait (FwdParams::wait_limit_ns)
  uint32_t tmem_base;
  volatile uint32_t abort;
};
static_assert(V2Layout<false>::SMEM_BYTES <= 232448 && V2Layout<true>::SMEM_BYTES <= 232448,
              "exceeds the 227 KB shared-memory limit per block");
static_assert(sizeof(V2Bars) <= 320, "control block exceeds its shared-memory slot");
static_assert(2 * 128 * V2Config::SOFTMAX_REGS + 128 * V2Config::PRODUCER_REGS <=
                  V2Config::THREADS * V2Config::LAUNCH_REGS,
              "register split exceeds the registers the block launches with");
static_assert(V2Config::SOFTMAX_REGS % 8 == 0 && V2Config::PRODUCER_REGS % 8 == 0, "setmaxnreg needs multiples of 8");

// Work-unit geometry shared by every role so that all of them walk the same
// tile sequence.
struct UnitGeom {
  int zq, zkv;         // query (b*H + h) and key/value (b*Hkv + hk) slab
  int q0;              // first query row of Q0 (Q1 starts at q0 + 128)
  int last[2];         // last KV tile index Q_k needs, -1 if Q_k is empty
  int ntiles;          // KV tiles in the stream: last[1] + 1 (or last[0] + 1)
};

__device__ __forceinline__ UnitGeom unit_geom(const FwdParams& p, int u) {
  UnitGeom g;
  const int num_pairs = (p.N + 255) / 256;
  const int bh = p.B * p.H;
  // Units come in groups of p.group_heads consecutive (b, h) slabs, so that
  // the CTAs running at any moment share a few heads' K and V in L2; within a
  // group the longest (latest) query pairs come first for causal balance.
  const int per_group = p.group_heads * num_pairs;
  const int grp = u / per_group;
  const int idx = u - grp * per_group;
  const int h0 = grp * p.group_heads;
  const int gsz = min(p.group_heads, bh - h0);
  const int pair = num_pairs - 1 - idx / gsz;
  const int zq = h0 + idx % gsz;
  g.zq = zq;
  const int b = zq / p.H, h = zq % p.H;
  g.zkv = b * p.Hkv + h / p.h_per_kv;
  g.q0 = pair * 256;
  const int nkv = p.num_kv_tiles;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int qk = g.q0 + 128 * k;
    if (qk >= p.N) {
      g.last[k] = -1;
    } else {
      g.last[k] = p.causal ? min(nkv - 1, (qk + 127) / 128) : nkv - 1;
    }
  }
  g.ntiles = max(g.last[0], g.last[1]) + 1;
  return g;
}

// KV tile at stream position `idx` (forward: idx; reverse: ntiles-1-idx).
__device__ __forceinline__ int stream_tile(const FwdParams& p, const UnitGeom& g, int idx) {
  return p.reverse ? (g.ntiles - 1 - idx) : idx;
}

// Wait with a time limit (bars->wait_limit_ns); also gives up as soon as
// another role aborted.
// Between checks the thread sleeps inside try_wait (suspend hint), so a
// waiting warp takes no issue slots from the warps sharing its scheduler and
// still wakes as soon as the phase completes.
__device__ __forceinline__ bool v2_wait(V2Bars* bars, uint64_t* bar, uint32_t parity, uint32_t* err_word,
                                        uint32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (bars->abort) return false;
    if (globaltimer_ns() - t0 > bars->wait_limit_ns) {
      atomicOr(err_word, code);
      bars->abort = 1u;
      return false;
    }
  }
}

// Bounded wait used while draining after an abort: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 500000000ull) return;
  }
}

// Streamed calls: wait until piece c of the inputs is on the device (the
// copy stream sets its ready word after the piece's copies), then order the
// tensor-memory loads that follow after the copies.  Bounded like every
// other wait; on timeout the CTA aborts.
__device__ __forceinline__ bool wait_piece_ready(const FwdParams& p, int c, V2Bars* bars, uint32_t* err_word) {
  const unsigned int* w = p.stream_flags + kPieceReady + c;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(w) : "memory");
    if (v != 0u) break;
    if (bars->abort) return false;
    if (globaltimer_ns() - t0 > bars->wait_limit_ns) {
      atomicOr(err_word, kErrTimeoutLoad);
      bars->abort = 1u;
      return false;
    }
    __nanosleep(1000);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// Streamed calls: each of the four warps of a query tile arrives once on its
// piece after storing its rows of O and lse; the arrival that completes the
// piece raises the piece's flag for the copy stream.
__device__ __forceinline__ void piece_tile_stored(const FwdParams& p, int zq, int lane) {
  __syncwarp();
  if (lane == 0) {
    const int c = zq / p.heads_per_piece;
    const int heads = min(p.heads_per_piece, p.B * p.H - c * p.heads_per_piece);
    const unsigned int expected = 4u * static_cast<unsigned int>(heads) * static_cast<unsigned int>(p.num_q_tiles);
    __threadfence();
    const unsigned int before = atomicAdd(p.stream_flags + kPieceDone + c, 1u);
    if (before + 1u == expected) {
      __threadfence_system();
      atomicExch(p.stream_flags + kPieceFlag + c, 1u);
    }
  }
}

// Readers of each published unit id: lane 0 of the two MMA warps and every
// thread of the two softmax warpgroups.
constexpr uint32_t kUnitReaders = 2 + 256;

// Pairs out of every eight (16 keys) whose exponentials use the FMA-pipe
// polynomial instead of MUFU ex2.  Measured at the 32K prefill: 0 pairs
// 1440 TFLOP/s, 1 pair 1311, 2 pairs 1294 (with the packed conversion
// below).  The exponential loop is limited by issue and dependency latency
// as much as by MUFU throughput, and the polynomial's longer dependency
// chains cost more than the MUFU work they remove, so every exponential
// uses MUFU.
constexpr int kPolyPairs = 0;

// SCALED: the inputs carry descales (FwdParams q/k/v_scales) and optionally
// a rotation to undo on the output; the running maximum is then kept in
// log2 units of the descaled logits, whose scale changes from tile to tile.
// QK16: Q and K are bfloat16 and S = Q K^T runs as a kind::f16 product (the
// P-cast and P V are unchanged).
// STREAMED: the inputs arrive piece by piece (FwdParams::stream_flags); its
// own instance, so that the other instances carry no streaming code.
template <bool COUNT, bool SCALED = false, bool QK16 = false, bool STREAMED = false>
__global__ void __launch_bounds__(V2Config::THREADS, 1)
    fwd_v2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p, uint32_t* err_word) {
  using C = V2Config;
  using L = V2Layout<QK16>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  V2Bars* bars = reinterpret_cast<V2Bars*>(base + L::OFF_BAR);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int num_units = p.B * p.H * ((p.N + 255) / 256);
  // Work units are handed out dynamically in the heaviest-first, head-grouped
  // order of unit_geom: the producer takes the next index from the global
  // counter p.sched (zero at launch) and passes it to the other roles.
  // next_unit(it) returns the it-th unit of this CTA (-1 when none is left).
  auto next_unit = [&](uint32_t it, bool reader_arrives) -> int {
    const int slot = it & 1;
    if (!v2_wait(bars, &bars->unit_full[slot], (it >> 1) & 1, err_word, kErrTimeoutPipe)) return -1;
    const int u = *reinterpret_cast<volatile int*>(&bars->unit_id[slot]);
    if (reader_arrives) mbar_arrive(&bars->unit_empty[slot]);
    return u;
  };

  if (tid == 0) {
    mbar_init(&bars->q_full[0], 1);
    mbar_init(&bars->q_full[1], 1);
    mbar_init(&bars->q_free, 256);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_free[s], 256);
      mbar_init(&bars->v_free[s], 256);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bars->s_full[k], 1);
      mbar_init(&bars->s_free[k], 128);
      mbar_init(&bars->p_full[k], 128);
      mbar_init(&bars->o_done[k], 1);
      mbar_init(&bars->o_free[k], 128);
    }
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    for (int s2 = 0; s2 < 2; ++s2) {
      mbar_init(&bars->unit_full[s2], 1);
      mbar_init(&bars->unit_empty[s2], kUnitReaders);
    }
    bars->abort = 0u;
    bars->wait_limit_ns = p.wait_limit_ns;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp >= 8) {
    // Each role's code sits inside the branch that set its register budget.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::PRODUCER_REGS));
  if (warp == 8) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t kv_it = 0, q_it = 0, q_done[2] = {0, 0};
      int ready_piece = -1;  // streamed calls: the last piece seen on the device
      bool ok = true;
      for (uint32_t u_it = 0; ok; ++u_it) {
        // Claim the next unit and publish it (slot reuse waits until every
        // reader has taken the unit published two claims ago).
        const int slot = u_it & 1;
        if (u_it >= 2 && !v2_wait(bars, &bars->unit_empty[slot], ((u_it >> 1) - 1) & 1, err_word, kErrTimeoutPipe))
          break;
        int u = static_cast<int>(atomicAdd(p.sched, 1u));
        if (u >= num_units) u = -1;
        bars->unit_id[slot] = u;
        mbar_arrive(&bars->unit_full[slot]);
        if (u < 0) break;
        const UnitGeom g = unit_geom(p, u);
        if (STREAMED && g.zq / p.heads_per_piece != ready_piece) {
          ready_piece = g.zq / p.heads_per_piece;
          if (!wait_piece_ready(p, ready_piece, bars, err_word)) break;
        }
        if (q_it > 0) ok = v2_wait(bars, &bars->q_free, (q_it - 1) & 1, err_word, kErrTimeoutPipe);
        if (!ok) break;
        // A Q or K tile is one box, or for bfloat16 two boxes of 64 columns
        // (one 128-byte swizzle panel each, 16 KB apart).
        auto load_qk = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row, int slab) {
          mbar_arrive_expect_tx(bar, L::QK_TILE);
          tma_load_3d(dst, map, bar, 0, row, slab);
          if constexpr (QK16) tma_load_3d(dst + C::TILE_BYTES, map, bar, 64, row, slab);
        };
        load_qk(base + L::OFF_Q, &tm_q, &bars->q_full[0], g.q0, g.zq);
        ++q_done[0];
        if (g.last[1] >= 0) {
          load_qk(base + L::OFF_Q + L::QK_TILE, &tm_q, &bars->q_full[1], g.q0 + 128, g.zq);
          ++q_done[1];
        }
        ++q_it;
        for (int idx = 0; idx < g.ntiles; ++idx) {
          const int t = stream_tile(p, g, idx);
          const int st = kv_it % L::STAGES;
          // K is released once both query tiles have read their S for it, V
          // once both have seen its P V products complete.
          if (kv_it >= L::STAGES) {
            ok = v2_wait(bars, &bars->k_free[st], ((kv_it / L::STAGES) - 1) & 1, err_word, kErrTimeoutPipe);
            if (!ok) break;
          }
          // (The test switch skips the first K tile: its readers' waits run out.)
          if (!(p.test_withhold_k && kv_it == 0))
            load_qk(base + L::OFF_K + st * L::QK_TILE, &tm_k, &bars->k_full[st], t * 128, g.zkv);
          if (kv_it >= L::STAGES) {
            ok = v2_wait(bars, &bars->v_free[st], ((kv_it / L::STAGES) - 1) & 1, err_word, kErrTimeoutPipe);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(&bars->v_full[st], C::TILE_BYTES);
          tma_load_3d(base + L::OFF_V + st * C::TILE_BYTES, &tm_v, &bars->v_full[st], 0, t * 128, g.zkv);
          ++kv_it;
        }
      }
      if (bars->abort) {
        // Let the loads already issued land before the CTA's shared memory is
        // released: the last Q pair and the last STAGES K/V tiles.
        if (q_done[0] > 0) drain_wait(&bars->q_full[0], (q_done[0] - 1) & 1);
        if (q_done[1] > 0) drain_wait(&bars->q_full[1], (q_done[1] - 1) & 1);
        for (uint32_t i = (kv_it > L::STAGES ? kv_it - L::STAGES : 0); i < kv_it; ++i) {
          if (!(p.test_withhold_k && i == 0)) drain_wait(&bars->k_full[i % L::STAGES], (i / L::STAGES) & 1);
          drain_wait(&bars->v_full[i % L::STAGES], (i / L::STAGES) & 1);
        }
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------- MMA issuers ------------------------------
    // Warp 9 issues query tile 0's products, warp 10 query tile 1's, each in
    // a fixed order S_k(i), P V_k(i-1), ... that only depends on its own
    // softmax warpgroup; both wait with try_wait, which suspends the warp and
    // takes no issue slots from the softmax warps sharing its scheduler.  The
    // whole warp runs the loop; lane 0 issues the MMAs and commits (a commit
    // tracks the MMAs of its own thread).
    // The role is instantiated once per query tile so that k, and with it
    // every MMA operand (TMEM addresses and shared-memory descriptors), is a
    // compile-time constant: with k computed from the warp index at run time
    // the S products came out wrong on the GPU for every row but the first,
    // while this form (and an unrolled single-warp form) is exact.
    auto mma_role = [&](auto kc) {
    constexpr int k = decltype(kc)::value;
    constexpr uint32_t idesc_qk = QK16 ? idesc_bf16_f32(128, 128) : idesc_e4m3_f32(128, 128, false, false);
    constexpr uint32_t idesc_pv = idesc_e4m3_f32(128, 128, false, true);
    // Descriptors are built once: a K step of 32 keys/columns moves the
    // start-address field (bytes >> 4) by 2 for the K-major operands (32
    // bytes along the row) and by 256 for V (32 rows of 128 bytes).
    constexpr uint64_t kTile = C::TILE_BYTES >> 4;  // one 16 KB tile (or panel) in the address field
    constexpr uint64_t kQKTile = L::QK_TILE >> 4;
    const uint64_t dQ = smem_desc(smem_u32(base + L::OFF_Q), 16, 1024, 2) + k * kQKTile;
    const uint64_t dK0 = smem_desc(smem_u32(base + L::OFF_K), 16, 1024, 2);
    const uint64_t dV0 = smem_desc(smem_u32(base + L::OFF_V), 128 * 128, 1024, 2);
    const uint64_t dP = smem_desc(smem_u32(base + L::OFF_P), 16, 1024, 2) + 2 * k * kTile;
    const uint32_t tS = tmem + 128 * k;
    const uint32_t tO = tmem + 256 + 128 * k;
    uint32_t kv_base = 0, q_it = 0, s_cnt = 0, p_cnt = 0, units = 0;
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, v2_wait(bars, bar, parity, err_word, code));
    };
    for (uint32_t u_it = 0; ok; ++u_it) {
      const int u = __shfl_sync(0xffffffffu, next_unit(u_it, lane == 0), 0);
      if (u < 0) break;
      const UnitGeom g = unit_geom(p, u);
      const uint32_t unit_base = kv_base;
      kv_base += g.ntiles;
      const int nk = (k ? g.last[1] : g.last[0]) + 1;  // tiles this query tile needs (0 if empty)
      if (nk == 0) continue;
      ok = wait_all(&bars->q_full[k], q_it & 1, kErrTimeoutQ);
      ++q_it;
      if (!ok) break;
      const int lo = p.reverse ? g.ntiles - nk : 0;
      for (int idx = lo; idx <= lo + nk && ok; ++idx) {
        if (idx < lo + nk) {
          // S_k = Q_k K^T once K has landed and softmax k has read its previous S.
          const uint32_t it = unit_base + idx;
          const int st = it % L::STAGES;
          ok = wait_all(&bars->k_full[st], (it / L::STAGES) & 1, kErrTimeoutKV);
          if (ok && s_cnt > 0) ok = wait_all(&bars->s_free[k], (s_cnt - 1) & 1, kErrTimeoutPipe);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint64_t db = dK0 + st * kQKTile;
            if constexpr (QK16) {
              // K = 16 per instruction: 32 bytes along the row (+2), four
              // steps per 128-byte panel, then the next panel (+16 KB).
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint64_t off = (kk >> 2) * kTile + 2 * (kk & 3);
                mma_bf16_ss(tS, dQ + off, db + off, idesc_qk, kk > 0);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tS, dQ + 2 * kk, db + 2 * kk, idesc_qk, kk > 0);
            }
            mma_commit(&bars->s_full[k]);
          }
          __syncwarp();
          ++s_cnt;
        }
        if (idx > lo) {
          // O_k += P^_k V for the previous tile once softmax k has written P^_k
          // (and, at a unit's first tile, has read out the previous unit's O_k).
          const uint32_t it = unit_base + idx - 1;
          const int st = it % L::STAGES;
          const bool first = (idx - 1 == lo);
          ok = wait_all(&bars->p_full[k], p_cnt & 1, kErrTimeoutPipe);
          if (ok) ok = wait_all(&bars->v_full[st], (it / L::STAGES) & 1, kErrTimeoutKV);
          if (ok && first && units > 0) ok = wait_all(&bars->o_free[k], (units - 1) & 1, kErrTimeoutPipe);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint64_t da = dP + (p_cnt & 1) * kTile, db = dV0 + st * kTile;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tO, da + 2 * kk, db + 256 * kk, idesc_pv, !(first && kk == 0));
            mma_commit(&bars->o_done[k]);
          }
          __syncwarp();
          ++p_cnt;
        }
      }
      ++units;
    }
    // Every MMA lane 0 issued has completed before TMEM is released.
    if (lane == 0) {
      mma_commit(&bars->drain[k]);
      drain_wait(&bars->drain[k], 0);
    }
    __syncwarp();
    };
    if (warp == 9) {
      mma_role(std::integral_constant<int, 0>{});
    } else {
      mma_role(std::integral_constant<int, 1>{});
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFTMAX_REGS));
    // ------------------------------- softmax WGs ------------------------------
    const int k = warp >> 2;  // which query tile of the pair
    const int r = tid & 127;  // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128 * k + lane_off;
    const uint32_t tO = tmem + 256 + 128 * k + lane_off;
    const uint32_t sPk = smem_u32(base + L::OFF_P + 2 * k * C::TILE_BYTES);
    uint32_t s_it = 0, o_it = 0, p_cnt = 0;
    uint32_t kv_base = 0;  // stream position of the unit's first KV tile (ring stage bookkeeping)
    bool ok = true;
    for (uint32_t u_it = 0; ok; ++u_it) {
      const int u = __shfl_sync(0xffffffffu, next_unit(u_it, true), 0);
      if (u < 0) break;
      const UnitGeom g = unit_geom(p, u);
      const int last = k ? g.last[1] : g.last[0];  // no dynamic indexing: keeps g in registers
      const int last_other = k ? g.last[0] : g.last[1];
      const uint32_t unit_base = kv_base;
      kv_base += g.ntiles;
      if (last < 0) continue;
      int prev_stage = 0;
      uint32_t prev_cnt = 2;
      const int qk = g.q0 + 128 * k;
      const int row = qk + r;
      // Running maximum: of the raw logits, or for SCALED inputs of the
      // descaled logits in log2 units (x = s * c_t with a per-tile c_t).
      float m = -INFINITY;
      float c_q = p.scale_log2;  // log2(e) / sqrt(d), times the query tile's descale when SCALED
      if constexpr (SCALED) c_q *= p.q_scales[static_cast<int64_t>(g.zq) * p.num_q_tiles + (qk >> 7)];
      float l = 0.0f;
      uint32_t nzero = 0;
      int j = 0;
      for (int idx = 0; idx < g.ntiles; ++idx) {
        const int t = stream_tile(p, g, idx);
        if (t > last) continue;
        const int j0 = t * 128;
        float c_t = c_q;  // scale of this tile's logits into log2 units
        if constexpr (SCALED) c_t *= __ldg(p.k_scales + static_cast<int64_t>(g.zkv) * p.num_kv_tiles + t);
        ok = __all_sync(0xffffffffu, v2_wait(bars, &bars->s_full[k], s_it & 1, err_word, kErrTimeoutMMA));
        if (!ok) break;  // warp-uniform, so the collective TMEM loads below stay converged
        ++s_it;
        tc_fence_after();
        float s[128];
        // Two halves: the second load is in flight while the first half's
        // maximum is formed.
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t rr[32];
          tmem_ld32(tS + c * 32, rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(rr[i]);
        }
        tmem_wait_ld();
#pragma unroll
        for (int c = 2; c < 4; ++c) {
          uint32_t rr[32];
          tmem_ld32(tS + c * 32, rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(rr[i]);
        }
        // Keys j0 + c with c >= lim are masked: beyond N, or after this query
        // row under the causal mask (edge blocks only).
        const bool edge = (j0 + 128 > p.N) || (p.causal && j0 + 127 > qk);
        const int lim = edge ? min(p.N, p.causal ? row + 1 : p.N) - j0 : 128;
        if (edge) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
        }
        float half_max;
        {
          float h1[22];
#pragma unroll
          for (int i = 0; i < 21; ++i) h1[i] = fmax3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
          h1[21] = SCALED ? s[63] : fmaxf(s[63], m);
          float h2[8];
#pragma unroll
          for (int i = 0; i < 7; ++i) h2[i] = fmax3(h1[3 * i], h1[3 * i + 1], h1[3 * i + 2]);
          h2[7] = h1[21];
          half_max = fmaxf(fmax3(fmax3(h2[0], h2[1], h2[2]), fmax3(h2[3], h2[4], h2[5]), h2[6]), h2[7]);
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->s_free[k]);  // the S buffer may now be overwritten
        // This S has completed, so the K stage it read (and, at the unit's
        // last tile, the Q pair) may be refilled once the other query tile is
        // done with them too; a tile it does not use counts twice here.
        const int stage = static_cast<int>((unit_base + idx) % L::STAGES);
        const uint32_t cnt = (t <= last_other) ? 1u : 2u;
        mbar_arrive_cnt(&bars->k_free[stage], cnt);
        if (p.reverse ? (t == 0) : (t == last)) mbar_arrive_cnt(&bars->q_free, last_other >= 0 ? 1u : 2u);

        if (edge) {
#pragma unroll
          for (int c = 64; c < 128; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
        }
        // Running max over this block and the previous maximum: trees of
        // three-input maxima (short dependency chains).
        float m_new;
        {
          float t1[22];
#pragma unroll
          for (int i = 0; i < 21; ++i) t1[i] = fmax3(s[64 + 3 * i], s[65 + 3 * i], s[66 + 3 * i]);
          t1[21] = fmaxf(s[127], half_max);
          float t2[8];
#pragma unroll
          for (int i = 0; i < 7; ++i) t2[i] = fmax3(t1[3 * i], t1[3 * i + 1], t1[3 * i + 2]);
          t2[7] = t1[21];
          m_new = fmaxf(fmax3(fmax3(t2[0], t2[1], t2[2]), fmax3(t2[3], t2[4], t2[5]), t2[6]), t2[7]);
        }
        if constexpr (SCALED) m_new = fmaxf(m_new * c_t, m);
        const float ms = (m_new == -INFINITY) ? 0.0f : (SCALED ? m_new : m_new * p.scale_log2);
        // P * S = 2^(x - m_new + log2 S) with x = s * log2(e) / sqrt(d)
        // (packed pairs): the scale enters the exponent, so one exponential
        // gives the scaled probability.  Its row sum, l * S, is kept (eight
        // independent pair sums) and divided out at the end; P^ = E4M3(P * S)
        // goes straight to the P buffer this tile uses (its previous reader,
        // the P V product two tiles back, is known to be complete).
        const uint32_t sPb = sPk + (p_cnt & 1) * C::TILE_BYTES;
        const uint64_t sc2 = f2_pack(c_t, c_t);
        const float bias = p.log2_p_scale - ms;
        const uint64_t nm2 = f2_pack(bias, bias);
        uint64_t acc[8];
#pragma unroll
        for (int c = 0; c < 128; c += 16) {
          uint32_t w[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int cc = c + 4 * q4;
            float x0, x1, x2, x3;
            f2_unpack(f2_fma(f2_pack(s[cc], s[cc + 1]), sc2, nm2), x0, x1);
            f2_unpack(f2_fma(f2_pack(s[cc + 2], s[cc + 3]), sc2, nm2), x2, x3);
            // Of every 16 keys, the last kPolyPairs pairs take the FMA-pipe
            // polynomial, the rest the MUFU exponential.
            const uint64_t pa = (2 * q4 >= 8 - kPolyPairs) ? exp2_poly2(x0, x1) : f2_pack(ex2_approx(x0), ex2_approx(x1));
            const uint64_t pb = (2 * q4 + 1 >= 8 - kPolyPairs) ? exp2_poly2(x2, x3)
                                                                : f2_pack(ex2_approx(x2), ex2_approx(x3));
            const int ai = (cc / 4) & 3;
            if (c == 0) {
              acc[2 * ai] = pa;
              acc[2 * ai + 1] = pb;
            } else {
              acc[2 * ai] = f2_add(acc[2 * ai], pa);
              acc[2 * ai + 1] = f2_add(acc[2 * ai + 1], pb);
            }
            float y0, y1, y2, y3;
            f2_unpack(pa, y0, y1);
            f2_unpack(pb, y2, y3);
            w[q4] = cvt_e4m3x4(y0, y1, y2, y3);
            if constexpr (COUNT) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int jj = j0 + cc + e;
                const bool visible = row < p.N && jj < p.N && jj >= p.n_sink && (!p.causal || jj <= row);
                nzero += (visible && ((w[q4] >> (8 * e)) & 0xFFu) == 0u) ? 1u : 0u;
              }
            }
          }
          const uint32_t off = swizzled_chunk(r, c / 16, 128);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sPb + off), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                       "r"(w[3])
                       : "memory");
        }
        float rowsum;
        {
          const uint64_t a01 = f2_add(acc[0], acc[1]), a23 = f2_add(acc[2], acc[3]);
          const uint64_t a45 = f2_add(acc[4], acc[5]), a67 = f2_add(acc[6], acc[7]);
          float lo, hi;
          f2_unpack(f2_add(f2_add(a01, a23), f2_add(a45, a67)), lo, hi);
          rowsum = lo + hi;
        }
        // Rescale factor 2^(m_old - m_new): exactly 1 when the maximum did not
        // change (the product m * c is then not recomputed), 0 before the
        // first visible key.  Formed after the exponentials so that this one
        // MUFU operation never waits behind them.
        const float alpha = (m_new == m) ? 1.0f : ex2_approx(SCALED ? m - ms : fmaf(m, p.scale_log2, -ms));
        l = l * alpha + rowsum;  // l * S
        m = m_new;

        if (j > 0) {
          // O_k holds the previous P V only once that product has completed.
          ok = __all_sync(0xffffffffu, v2_wait(bars, &bars->o_done[k], o_it & 1, err_word, kErrTimeoutMMA));
          if (!ok) break;
          ++o_it;
          mbar_arrive_cnt(&bars->v_free[prev_stage], prev_cnt);  // the previous tile's V has been read
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.0f)) {
            // O_k *= alpha: four loads, one wait, packed multiplies, four stores.
            uint32_t o[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tO + c * 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32 * c));
            tmem_wait_ld();
            const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
            for (int i = 0; i < 128; i += 2) {
              float lo, hi;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2), lo, hi);
              o[i] = __float_as_uint(lo);
              o[i + 1] = __float_as_uint(hi);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_st32(tO + c * 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32 * c));
            tmem_wait_st();
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->p_full[k]);
        prev_stage = stage;
        prev_cnt = cnt;
        ++p_cnt;
        ++j;
      }
      if (!ok) break;
      // Epilogue: the last P V of the unit, then O / (S * l) (l already
      // carries the factor S).
      ok = __all_sync(0xffffffffu, v2_wait(bars, &bars->o_done[k], o_it & 1, err_word, kErrTimeoutMMA));
      if (!ok) break;
      ++o_it;
      mbar_arrive_cnt(&bars->v_free[prev_stage], prev_cnt);
      tc_fence_after();
      if constexpr (COUNT) {
        const uint32_t total = __reduce_add_sync(0xffffffffu, nzero);
        if (lane == 0 && total) atomicAdd(p.counts + g.zq, static_cast<unsigned long long>(total));
      } else {
        float inv = __frcp_rn(l);  // l holds l * S
        if constexpr (SCALED) inv *= p.v_scales[g.zkv];
        uint8_t* orow = static_cast<uint8_t*>(p.o) + ((static_cast<int64_t>(g.zq) * p.N + row) * 128) * 2;
        if (SCALED && p.unrotate) {
          // O_row R^T: the Walsh-Hadamard transform of the whole row (radix-2
          // stages of half-width 1, 2, ..., 64, sum first), times
          // float32(1/sqrt(128)), then the signs.
          float y[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t rr[32];
            tmem_ld32(tO + c * 32, rr);
#pragma unroll
            for (int i = 0; i < 32; ++i) y[c * 32 + i] = __uint_as_float(rr[i]);
          }
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 128; ++i) y[i] *= inv;
#pragma unroll
          for (int h = 1; h < 128; h *= 2) {
#pragma unroll
            for (int i = 0; i < 128; ++i) {
              if ((i & h) == 0) {
                const float a = y[i], b = y[i + h];
                y[i] = a + b;
                y[i + h] = a - b;
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 128; ++i) {
            const float t = y[i] * 0.08838834764831845f;  // float32(1/sqrt(128))
            y[i] = ((p.sign_bits[i >> 5] >> (i & 31)) & 1u) ? -t : t;
          }
          if (row < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              dst[i] = make_uint4(pack_bf16x2(y[8 * i], y[8 * i + 1]), pack_bf16x2(y[8 * i + 2], y[8 * i + 3]),
                                  pack_bf16x2(y[8 * i + 4], y[8 * i + 5]), pack_bf16x2(y[8 * i + 6], y[8 * i + 7]));
          }
        } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t rr[32];
          tmem_ld32(tO + c * 32, rr);
          tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * inv, __uint_as_float(rr[2 * i + 1]) * inv);
          if (row < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
        }
        if (p.lse != nullptr && row < p.N)
          p.lse[static_cast<int64_t>(g.zq) * p.N + row] =
              ((SCALED ? m : m * p.scale_log2) + (log2f(l) - p.log2_p_scale)) * 0.6931471805599453f;
        if constexpr (STREAMED) piece_tile_stored(p, g.zq, lane);
      }
      tc_fence_before();
      mbar_arrive(&bars->o_free[k]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (STREAMED && bars->abort && tid == 0) {
    // This CTA gave up: raise every piece flag, so that no copy stream waits
    // for outputs that will not come (the error word reports the failure).
    const int pieces = (p.B * p.H + p.heads_per_piece - 1) / p.heads_per_piece;
    for (int c = 0; c < pieces; ++c) atomicExch(p.stream_flags + kPieceFlag + c, 1u);
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fp8attn
