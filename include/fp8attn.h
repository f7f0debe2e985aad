/*
 * fp8attn.h -- C ABI of libfp8attn: FP8 (E4M3) attention forward pass on
 * NVIDIA B200 (sm_100a) with a static P-cast scale.
 *
 * The operation (the page "P-Cast Precision in FP8 Attention: Sink-Induced
 * Collapse and the Optimality of S=2^8", technical summary, section 1):
 * blockwise online-softmax attention O = softmax(Q K^T / sqrt(d)) V in which
 * each probability tile P is multiplied by a static scale S, cast to E4M3
 * before the P V product, and S is divided back out in the epilogue; the KV
 * blocks are walked forward (block 0 first) or in reverse (last block first).
 * The blockwise algorithm and its online-softmax recurrence are those of the
 * page "Attenzione flash e domanda sulla lunghezza della sequenza", sections
 * "L'algoritmo Flash Attention" and "La ricorrenza softmax online"; causal
 * block skipping is its section on causal masking.
 *
 * Conventions shared by the calls (each call's comment states its exceptions):
 *   - All tensor arguments are DEVICE pointers to caller-owned memory; the
 *     library keeps no pointer after a call returns.  Pointers must be
 *     16-byte aligned (descale and lse arrays: 4-byte).  The rotation signs
 *     of fp8attn_quantize and fp8attn_fwd_scaled are a HOST array.
 *   - The persistent-kernel calls (fp8attn_fwd, fp8attn_pzero_count,
 *     fp8attn_fwd_scaled, fp8attn_fwd_bf16qk at d = 128) each take a 256-byte
 *     work-unit counter from a per-device stream-ordered memory pool the
 *     library creates on first use (cudaMallocFromPoolAsync on the call's
 *     stream, returned with cudaFreeAsync on the same stream before the call
 *     returns; the pool keeps its memory mapped for reuse), so concurrent
 *     calls on different streams are independent.  fp8attn_fwd_noalloc,
 *     fp8attn_quantize, fp8attn_decode and fp8attn_bwd allocate nothing.
 *   - Layouts are contiguous, row-major, with the head dimension innermost:
 *       q    [B, H,   N, d]  E4M3 bytes (OCP E4M3FN)
 *       k, v [B, Hkv, N, d]  E4M3 bytes
 *       o    [B, H,   N, d]  bfloat16
 *       lse  [B, H,   N]     float32
 *     Query head h reads key/value head h / (H / Hkv) (grouped-query
 *     attention; Hkv == H is ordinary multi-head attention).
 *   - d must be 64 or 128.  N >= 0 is arbitrary (a ragged last tile is
 *     masked).  B * H * N == 0 is a valid empty problem: nothing is launched.
 *   - causal != 0 applies the square, top-left aligned mask (query i sees keys
 *     0..i); KV blocks entirely above the diagonal are skipped.
 *   - The logit scale is fixed at 1/sqrt(d).
 *   - p_scale is the static scale S, 2^-64 <= S <= 2^64 (anything else, NaN
 *     included, is FP8ATTN_ERR_INVALID_ARG).  S > 448 saturates the largest
 *     probabilities.
 *   - kv_order: 0 = forward (KV block 0 first), 1 = reverse (last block
 *     first).
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous with respect to the host: a return of
 *     FP8ATTN_OK means the arguments were valid and the launch succeeded.
 *   - On any error nothing is launched and outputs are left untouched; the
 *     library never aborts the process and never traps on the device.
 *   - Device-side waits are bounded.  A wait that runs out sets a device
 *     error word instead of hanging; fp8attn_check_error() reports it.
 */
#ifndef FP8ATTN_H
#define FP8ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every call. */
enum fp8attn_status {
    FP8ATTN_OK = 0,
    FP8ATTN_ERR_INVALID_ARG = 1, /* a size, pointer, alignment or scale is invalid */
    FP8ATTN_ERR_UNSUPPORTED = 2, /* valid but not supported here (d, device)       */
    FP8ATTN_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed            */
    FP8ATTN_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out              */
    FP8ATTN_ERR_SCRATCH_LIMIT = 5 /* too large for fp8attn_fwd_noalloc's fixed scratch */
};

/* Size of the device array that fp8attn_fwd_noalloc uses as scratch (one per
 * device), and the most work units (B * H * ceil(N / 256), d = 128) one of
 * its calls accepts: its counter is one 32-bit word of that array. */
#define FP8ATTN_NOALLOC_SCRATCH_BYTES 256
#define FP8ATTN_NOALLOC_MAX_UNITS 2147418112LL /* 2^31 - 2^16 */

/*
 * Forward pass.  Writes o (bfloat16, O = sum_j P^_j v_j / (S * l)) and, when
 * lse is not NULL, lse = m + ln(l): the natural log of the softmax
 * denominator in units of the scaled logits q.k/sqrt(d), l being the sum of
 * the unquantised probabilities.
 */
int fp8attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int H, int Hkv, int N, int d, int causal,
                float p_scale, int kv_order, void* stream);

/*
 * P-collapse count.  Runs the same forward pass (same tiles, order, scale and
 * cast) without writing O, and writes counts[b * H + h] = the number of
 * (query, key) pairs of head (b, h) with key index j >= n_sink, not masked,
 * whose cast value E4M3(P * S) is zero.  counts is a device array of B * H
 * unsigned 64-bit integers; it is overwritten.  n_sink >= 0.  (Underflow of
 * non-sink probabilities to zero is the "P-collapse" of the P-cast summary,
 * section 1; passing n_sink equal to fp8attn_kv_tile(d) counts only keys
 * outside the block that holds the sinks.)
 */
int fp8attn_pzero_count(const void* q, const void* k, const void* v,
                        unsigned long long* counts,
                        int B, int H, int Hkv, int N, int d, int causal,
                        float p_scale, int kv_order, int n_sink, void* stream);

/*
 * Quantisation in front of the attention path ("Attenzione flash e domanda
 * sulla lunghezza della sequenza", section "FA3: Meccanica della tramoggia",
 * point 3: block quantisation to FP8, after a random rotation that spreads
 * outlier channels over all coordinates).
 *
 * x is a device array [Z, N, d] of bfloat16 (x_dtype = 0) or float32
 * (x_dtype = 1), contiguous, 16-byte aligned, finite.  Each row is optionally
 * rotated by R = diag(signs) H_d / sqrt(d) (H_d the Sylvester Hadamard
 * matrix; signs is a HOST array of d values, each +1 or -1, read during the
 * call; NULL = no rotation), evaluated as the radix-2 fast transform in
 * float32.  Rows are then cast to E4M3 (xq: device [Z, N, d], 16-byte
 * aligned) with one descale per block: the smallest power of two s >= 2^-126
 * with max|x| <= 448 s, so that x = s * E4M3 code up to the cast's rounding
 * and nothing saturates.  Blocks are block_rows (1..128) consecutive rows of
 * one slab, scales is then a device float array [Z, ceil(N / block_rows)];
 * block_rows = 0 gives one descale per slab, scales [Z]: an amax pass, a
 * cast pass, and one launch that turns the maxima into descales (the array
 * holds intermediate maxima until that last launch).
 * d must be 64 or 128, and Z * ceil(N / block_rows) at most 2^30
 * (FP8ATTN_ERR_UNSUPPORTED otherwise).
 * For fp8attn_fwd_scaled: Q and K with block_rows = 128, V with 0, the same
 * signs for all three.
 */
int fp8attn_quantize(const void* x, int x_dtype, void* xq, float* scales,
                     int Z, int N, int d, int block_rows, const float* signs, void* stream);

/*
 * Forward pass on quantised inputs: q = q_scales * q codes per 128-row query
 * tile ([B * H, ceil(N / 128)]), k = k_scales * k codes per 128-key tile
 * ([B * Hkv, ceil(N / 128)]), v = v_scales * v codes per head ([B * Hkv]),
 * all scales device float arrays (powers of two as fp8attn_quantize writes
 * them).  The P-cast, orders, masks and outputs are those of fp8attn_fwd on
 * the descaled values; when signs (HOST, d values of +-1, the ones used to
 * quantize) is not NULL, each output row is rotated back by R^T before the
 * bfloat16 rounding, so o is the attention of the unrotated inputs.  d must
 * be 128 (FP8ATTN_ERR_UNSUPPORTED otherwise).  The scratch is that of
 * fp8attn_fwd.
 */
int fp8attn_fwd_scaled(const void* q, const void* k, const void* v, void* o, float* lse,
                       const float* q_scales, const float* k_scales, const float* v_scales,
                       const float* signs, int B, int H, int Hkv, int N, int d, int causal,
                       float p_scale, int kv_order, void* stream);

/*
 * Forward pass with bfloat16 Q and K: q [B, H, N, d] and k [B, Hkv, N, d]
 * bfloat16, v [B, Hkv, N, d] E4M3 (device, contiguous, 16-byte aligned).
 * S = Q K^T runs on the tensor cores' 16-bit path with FP32 accumulation;
 * the running maximum, the P-cast E4M3(P * S), P^ V in FP8 and the epilogue
 * are those of fp8attn_fwd.  This is the setting of the P-cast summary's
 * kernel-faithful experiments, which keep Q and K in high precision to
 * isolate the cast of P ("P-Cast Precision in FP8 Attention", section 3,
 * point 4, and section 4).  d must be 128
 * (FP8ATTN_ERR_UNSUPPORTED otherwise); the scratch is that of fp8attn_fwd.
 */
int fp8attn_fwd_bf16qk(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int H, int Hkv, int N, int d, int causal,
                       float p_scale, int kv_order, void* stream);

/*
 * Decode / split-KV forward pass: one query row per (batch, head) against
 * all N keys, q [B, H, d] E4M3, k and v [B, Hkv, N, d] E4M3 (device), o
 * [B, H, d] bfloat16, lse [B, H] float32 (may be NULL).  The keys are cut
 * into splits of split_tiles consecutive 128-key tiles; each split runs the
 * blockwise online softmax with the P-cast on its own, its tiles walked in
 * kv_order, and the splits are merged exactly through their maxima and
 * sums ("Attenzione flash e domanda sulla lunghezza della sequenza", section
 * "La ricorrenza softmax online"; "P-Cast Precision in FP8 Attention",
 * technical summary, section 1).  No causal mask (the query is the last
 * position).  workspace is caller-owned device memory of at least
 * fp8attn_decode_workspace_bytes(B, H, N, split_tiles) bytes, 16-byte
 * aligned, overwritten by the call.  d must be 128 and H / Hkv at most 8
 * (FP8ATTN_ERR_UNSUPPORTED otherwise); N >= 1; k, v, o 16-byte aligned.
 */
int fp8attn_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                   void* workspace, unsigned long long workspace_bytes,
                   int B, int H, int Hkv, int N, int d, float p_scale, int kv_order,
                   int split_tiles, void* stream);

/* Workspace bytes fp8attn_decode needs (0 for invalid sizes). */
unsigned long long fp8attn_decode_workspace_bytes(int B, int H, int N, int split_tiles);

/*
 * Backward pass of fp8attn_fwd.  Given the forward inputs q, k, v (E4M3), its
 * outputs o (bfloat16 [B, H, N, d]) and lse (float32 [B, H, N], natural log,
 * as fp8attn_fwd writes it) and the output gradient dout (bfloat16 [B, H, N,
 * d]), writes the float32 gradients
 *   dq [B, H, N, d],  dk [B, Hkv, N, d],  dv [B, Hkv, N, d]
 * and delta [B, H, N], delta_i = dout_i . o_i.  The probabilities are
 * recomputed from lse, P_ij = exp(q_i.k_j/sqrt(d) - lse_i), as in the
 * recomputation form of "Attenzione flash e domanda sulla lunghezza della
 * sequenza"; the P-cast of "P-Cast Precision in FP8 Attention", technical
 * summary, section 1, is kept where the forward pass applies it:
 *   dv_j = sum_i E4M3(P_ij S) dout_i / S
 *   dS_ij = P_ij (dout_i . v_j - delta_i)   (the cast is the identity here)
 *   dq_i = sum_j dS_ij k_j / sqrt(d),   dk_j = sum_i dS_ij q_i / sqrt(d)
 * dk and dv sum over the H / Hkv query heads that share a kv head.  dS is
 * rounded to bfloat16 before its two products; everything else accumulates
 * in float32.  The gradients do not depend on the forward call's kv_order.
 * d must be 128 (FP8ATTN_ERR_UNSUPPORTED otherwise); B * H * N at most 2^34.
 * All pointers are device pointers, caller-owned, 16-byte aligned (lse and
 * delta: 4-byte); the outputs are overwritten, and no output may overlap
 * another argument.  Allocates nothing: dk and dv also serve as scratch
 * during the call (bfloat16 copies of k and v that the dq kernel reads,
 * replaced by the gradients before the call's work ends).  Launches five
 * kernels on stream: the row dots, the two bfloat16 copies, dq, then dk
 * and dv.
 */
int fp8attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                const void* dout, float* dq, float* dk, float* dv, float* delta,
                int B, int H, int Hkv, int N, int d, int causal, float p_scale, void* stream);

/*
 * Allocation-free forward pass.  The pages have no counterpart of this call:
 * it is an interface for callers that cannot let the library allocate device
 * memory -- programs that hand the whole device memory to their own allocator
 * up front and budget it exactly, and latency-bound loops in which an
 * allocation (which may block, grow a pool or fail under fragmentation) at an
 * unpredictable moment is not acceptable.
 *
 * Arguments, layouts, results and status codes are those of fp8attn_fwd, and
 * so are the outputs on every input both accept.  The differences:
 *   - Scratch.  For d = 128 the persistent kernel's work-unit counter is word
 *     0 of one library-static device array of FP8ATTN_NOALLOC_SCRATCH_BYTES
 *     bytes (one array per device), not a per-call block.  Each call zeroes
 *     the counter on `stream` (cudaMemsetAsync) before its launch.  No call
 *     allocates or frees device memory.  d = 64 runs a kernel that needs no
 *     scratch.
 *   - Set-up.  The first call on a device (the device current at the call)
 *     looks up the array's address with cudaGetSymbolAddress, loads both
 *     forward kernels and sets their shared-memory limits; it returns
 *     FP8ATTN_ERR_CUDA if any of that fails.  Make that first call before any
 *     stream capture begins.
 *   - Sharing.  Every call on a device uses the same array.  Calls that can
 *     overlap on the device (streams without ordering between them, or
 *     several host threads) race on the counter and give wrong results:
 *     order them, e.g. issue them all on one stream.
 *   - Limit.  A d = 128 problem with more than FP8ATTN_NOALLOC_MAX_UNITS work
 *     units is rejected with FP8ATTN_ERR_SCRATCH_LIMIT before anything is
 *     launched.
 */
int fp8attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int Hkv, int N, int d, int causal,
                        float p_scale, int kv_order, void* stream);

/*
 * The forward pass of fp8attn_fwd on inputs and outputs in HOST memory, with
 * the host<->device copies overlapped with the computation ("P-Cast
 * Precision in FP8 Attention", technical summary, section 1, for what is
 * computed; the overlap is this library's).
 *
 * q_host, k_host, v_host (E4M3 bytes), o_host (bfloat16) and lse_host
 * (float32, or NULL) have the layouts of fp8attn_fwd and should be pinned
 * (cudaHostAlloc / cudaHostRegister) for the copies to overlap; pageable
 * memory works, but its copies then run one after another.  q_dev, k_dev,
 * v_dev, o_dev and lse_dev (NULL exactly when lse_host is NULL) are
 * caller-owned device buffers of the same sizes, used as staging (16-byte
 * aligned; lse_dev 4-byte aligned); their contents afterwards are those of
 * an fp8attn_fwd call on them.
 *
 * The problem is cut into `pieces` (1..32; 0 picks 24; never more than the
 * number of (batch, kv head) slabs) pieces of whole (batch, kv head) slabs
 * with their query heads.  The inputs are copied on a copy stream of the
 * library, in runs of neighbouring pieces (one piece first, then two, then
 * three at a time, then two and one at the end), each run followed by the
 * ready words of its pieces.  One persistent kernel on `stream` processes the
 * pieces in order, its producer waiting for each piece's ready word; as the
 * last query tile of a piece is stored the kernel raises the piece's flag, and
 * a second copy stream copies each run's outputs back once the flags of all
 * its pieces are up.  The copy streams are non-blocking streams the library
 * creates once per device; the work on them is joined back into `stream`
 * before the call's later work.  The ready words, flags and work-unit counter
 * of a call sit in a 512-byte block of a ring of eight that the library
 * allocates once per device (stream memory operations cannot address pool
 * allocations); a block is reused only after the stream of its previous call
 * has passed that call's end.  Calls from several host threads on one device
 * must be ordered by the caller.
 * With d = 64 or pieces = 1 the copies in, the pass and the copies out simply
 * run in order on `stream`.
 *
 * Asynchronous like fp8attn_fwd: the outputs are on the host once `stream`
 * has reached this point.  If a device wait runs out, the kernel still
 * raises every flag (so no copy stream waits for good), the outputs are
 * undefined, and fp8attn_check_error() returns FP8ATTN_ERR_TIMEOUT.
 * Returns FP8ATTN_ERR_INVALID_ARG for a NULL host pointer, pieces outside
 * 0..32 or the checks of fp8attn_fwd (on the device buffers);
 * FP8ATTN_ERR_UNSUPPORTED if the driver has no stream memory operations.
 */
int fp8attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                     void* o_host, float* lse_host,
                     void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_dev,
                     int B, int H, int Hkv, int N, int d, int causal,
                     float p_scale, int kv_order, int pieces, void* stream);

/* KV block size B_c the kernels use for head dimension d (0 if d is
 * unsupported).  The query block is always 128 rows. */
int fp8attn_kv_tile(int d);

/* Human-readable name of a status code (static string, never NULL). */
const char* fp8attn_status_str(int status);

/*
 * Synchronises stream, then reads and clears the device error word that
 * bounded waits set.  Returns FP8ATTN_ERR_TIMEOUT if a wait ran out since the
 * last check, FP8ATTN_ERR_CUDA if the synchronisation itself failed, else
 * FP8ATTN_OK.
 */
int fp8attn_check_error(void* stream);

/*
 * Test switch for the bounded waits (the pages have no counterpart).  Arms
 * the next launch of the d = 128 forward kernel in this process
 * (fp8attn_fwd, fp8attn_pzero_count, fp8attn_fwd_scaled, fp8attn_fwd_bf16qk):
 * its producer skips the load of the first K tile, so the waits for that tile
 * run out after wait_limit_ns nanoseconds instead of the normal 2 s.  The
 * kernel then stops every role, lets its in-flight copies and products land,
 * releases its tensor memory and returns; outputs of that launch are
 * undefined and fp8attn_check_error() returns FP8ATTN_ERR_TIMEOUT.  Nothing
 * faults or traps.  The switch is consumed by that one launch.  Returns
 * FP8ATTN_ERR_INVALID_ARG unless 0 < wait_limit_ns <= 2e9.
 */
int fp8attn_test_withhold_load(unsigned long long wait_limit_ns);

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
int fp8attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8ATTN_H */
