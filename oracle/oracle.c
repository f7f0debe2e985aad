/*
 * oracle.c -- plain CPU oracle for FP8 (E4M3) attention with a static P-cast scale.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may link, load or call this file; only the test suite,
 * the smoke check and the CPU-baseline leg of the benchmark do.  It shares no
 * code, header, table or constant with the CUDA path.
 *
 * Sources it follows (cited by page title and section):
 *   [PCAST]  "P-Cast Precision in FP8 Attention: Sink-Induced Collapse and the
 *            Optimality of S=2^8" (Reed Lau), technical summary, sections 1-4;
 *            the Italian summary "Riepilogo Tecnico: Precisione P-Cast in FP8
 *            Attention" says the same, section by section.
 *   [FLASH]  "Un contesto di un'intera giornata batte uno di dieci minuti?
 *            Attenzione flash e domanda sulla lunghezza della sequenza",
 *            sections "Perche l'attenzione e legata alla memoria",
 *            "L'algoritmo Flash Attention", "La ricorrenza softmax online",
 *            "Il mascheramento causale ...".
 *   [OCP]    the OCP 8-bit floating point definition of E4M3 ("E4M3FN": bias 7,
 *            no infinities, S.1111.111 is NaN, largest finite 448, smallest
 *            normal 2^-6, smallest subnormal 2^-9), which [PCAST] relies on
 *            (section 2: round-to-zero threshold 2^-10, normal range down to
 *            2^-6, S <= 448).
 *
 * Everything here is deliberately slow and direct: one query row at a time,
 * the steps in the order the pages give them.  Parallelism is only over
 * independent query rows (OpenMP), which changes no arithmetic.
 *
 * Build: gcc -O3 -mavx2 -mfma -ffp-contract=off -fopenmp -shared -fPIC
 * (-ffp-contract=off keeps every FP32 multiply and add separately rounded, as
 * written.)
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* E4M3 codec from the [OCP] definition.                                    */
/* ------------------------------------------------------------------------ */

/* Value of one E4M3 code: sign bit 7, exponent field bits 6..3 (bias 7),
 * mantissa bits 2..0.  Exponent field 0 is subnormal (m * 2^-9); exponent
 * field 15 with mantissa 7 is NaN; there is no infinity. */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Round a real number to E4M3: round to nearest, ties to even; subnormals
 * kept; anything beyond the largest finite value saturates to +-448
 * ("satfinite", never NaN for a finite input); NaN maps to the NaN code.
 *
 * Method: find the binade [2^e, 2^(e+1)) of |x| (e >= -6; below that the
 * subnormal spacing 2^-9 applies), express |x| in units of that binade's
 * spacing 2^(e-3), and round that (exactly representable) quotient to an
 * integer with nearbyint() under the default round-to-nearest-even mode.
 * The integer is then the code's low seven bits, because codes are monotone
 * in magnitude and consecutive within and across binades. */
uint8_t oracle_e4m3_encode(double x)
{
    if (isnan(x))
        return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0)
        return sign | 0x7E;                  /* largest finite, 1.75 * 2^8 */
    int e;
    if (a < ldexp(1.0, -6)) {
        e = -6;                              /* subnormal spacing 2^-9 */
    } else {
        int ex;
        (void)frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1) */
        e = ex - 1;                          /* a in [2^e, 2^(e+1)) */
    }
    double units = ldexp(a, 3 - e);          /* |x| / 2^(e-3), exact */
    double q = nearbyint(units);             /* ties to even */
    /* Codes 0..7 are the subnormals m * 2^-9 and code 8 is 2^-6; from there
     * each binade [2^e, 2^(e+1)) holds 8 codes of spacing 2^(e-3), starting
     * at code (e + 7) * 8.  With q = |x| / 2^(e-3) in [8, 16] for a normal
     * (in [0, 8] for the subnormal range, where e = -6), the code is
     * (e + 6) * 8 + q; q = 16 carries into the next binade's first code. */
    int code = (e + 6) * 8 + (int)q;
    if (code > 0x7E)
        code = 0x7E;                         /* rounding up past 448 saturates */
    return sign | (uint8_t)code;
}

void oracle_e4m3_encode_array(const float* x, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_encode((double)x[i]);
}

/* The same rounding of float64 values (no intermediate float32 rounding). */
void oracle_e4m3_encode_array_f64(const double* x, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_decode_array(const uint8_t* c, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)oracle_e4m3_decode(c[i]);
}

/* Round an FP32 value to bfloat16 (8 significant bits), nearest-even, and
 * return the bfloat16 bit pattern (the upper half of the rounded FP32).
 * Same binade method as above; finite inputs only (outputs here are bounded
 * by max|V| <= 448). */
uint16_t oracle_bf16_round(float xf)
{
    double x = (double)xf;
    if (x == 0.0 || isnan(x) || isinf(x)) {
        uint32_t b;
        memcpy(&b, &xf, 4);
        return (uint16_t)(b >> 16);
    }
    int ex;
    (void)frexp(fabs(x), &ex);
    int e = ex - 1;
    if (e < -126)
        e = -126;                            /* bf16 subnormal spacing 2^-133 */
    double q = nearbyint(ldexp(x, 7 - e));
    float r = (float)ldexp(q, e - 7);        /* exact: 8 significant bits */
    uint32_t b;
    memcpy(&b, &r, 4);
    return (uint16_t)(b >> 16);
}

void oracle_bf16_round_array(const float* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_round(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Shared row plumbing (layout only, no arithmetic).                        */
/* ------------------------------------------------------------------------ */

/* q: [B, H, N, d]; k, v: [B, Hkv, N, d]; grouped-query attention maps query
 * head h to key/value head h / (H / Hkv). */
static const float* q_row(const float* q, int b, int h, int i, int H, int N, int d)
{
    return q + (((int64_t)b * H + h) * N + i) * (int64_t)d;
}
static const float* kv_head(const float* kv, int b, int h, int H, int Hkv, int N, int d)
{
    int hk = h / (H / Hkv);
    return kv + ((int64_t)b * Hkv + hk) * (int64_t)N * d;
}

/* Dot product of two rows, accumulated in FP64.  For E4M3 inputs each product
 * is a multiple of 2^-18 below 2^18 and a sum of up to 2^14 of them stays
 * below 2^53 units, so the result is the exact dot product whatever the
 * summation order; the eight partial sums only let the compiler vectorise. */
static double dot64(const float* a, const float* b, int d)
{
    double s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int c = 0;
    for (; c + 8 <= d; c += 8)
        for (int u = 0; u < 8; ++u)
            s[u] += (double)a[c + u] * (double)b[c + u];
    for (; c < d; ++c)
        s[0] += (double)a[c] * (double)b[c];
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

/* ------------------------------------------------------------------------ */
/* (1) Exact attention in FP64: O = softmax(Q K^T / sqrt(d)) V.             */
/* ------------------------------------------------------------------------ */

/* [FLASH] "Perche l'attenzione e legata alla memoria": attention is
 * softmax(Q K^T / sqrt(d_k)) V.  [FLASH] causal masking section: a query
 * attends only to keys at or before its own position (top-left aligned
 * square mask).  Two passes over the row (max, then normalised sum), which
 * is the "naive" softmax the online recurrence re-associates.
 *
 * rows: the query positions to evaluate (the same for every (b, h)); the
 * outputs are o [B, H, nrows, d] and lse [B, H, nrows] (natural log of the
 * softmax denominator, in units of the scaled logits). */
void oracle_attention_fp64(const float* q, const float* k, const float* v,
                           int B, int H, int Hkv, int N, int d, int causal,
                           const int32_t* rows, int nrows, double* o, double* lse)
{
    const double scale = 1.0 / sqrt((double)d);
    int64_t total = (int64_t)B * H * nrows;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 4)
        for (int64_t u = 0; u < total; ++u) {
            int r = (int)(u % nrows);
            int h = (int)((u / nrows) % H);
            int b = (int)(u / ((int64_t)nrows * H));
            int i = rows[r];
            const float* qi = q_row(q, b, h, i, H, N, d);
            const float* K = kv_head(k, b, h, H, Hkv, N, d);
            const float* V = kv_head(v, b, h, H, Hkv, N, d);
            int jend = causal ? i + 1 : N;   /* keys 0..jend-1 are visible */
            double m = -INFINITY;
            for (int j = 0; j < jend; ++j) {
                s[j] = dot64(qi, K + (int64_t)j * d, d) * scale;
                if (s[j] > m)
                    m = s[j];
            }
            double z = 0.0;
            double* oi = o + u * d;
            for (int c = 0; c < d; ++c)
                oi[c] = 0.0;
            for (int j = 0; j < jend; ++j) {
                double w = exp(s[j] - m);
                z += w;
                const float* vj = V + (int64_t)j * d;
                for (int c = 0; c < d; ++c)
                    oi[c] += w * (double)vj[c];
            }
            for (int c = 0; c < d; ++c)
                oi[c] /= z;
            lse[u] = m + log(z);
        }
        free(s);
    }
}

/* ------------------------------------------------------------------------ */
/* (2) Blockwise online-softmax attention with the E4M3 P-cast.             */
/* ------------------------------------------------------------------------ */

/* One query row of the tiled forward pass.
 *
 * [FLASH] "L'algoritmo Flash Attention": K and V are split into column
 * blocks of B_c keys; for each block the logits S_ij = Q_i K_j^T / sqrt(d)
 * are formed, the running maximum is updated to m_new = max(m, rowmax), the
 * probabilities P = exp(S - m_new) are formed, the running sum l and the
 * output accumulator O are rescaled by exp(m_old - m_new) and the block's
 * contribution P V_j is added.  [FLASH] "La ricorrenza softmax online": the
 * rescale is retroactive and exact in exact arithmetic.  Normalisation by l
 * is deferred to the end (the FlashAttention-2 change in [FLASH] "FA2:
 * parallelismo", item 1).
 *
 * [PCAST] section 1: before the P V product, P is multiplied by a static
 * scale S and cast to E4M3; S is divided back out in the epilogue.  The
 * running sum l is kept from the unquantised FP32 P (so the epilogue divides
 * by S * l); values that round to zero are therefore lost mass, which is the
 * "P-collapse" of [PCAST] section 1.
 *
 * [PCAST] section 1, implementation choice 1: the KV blocks are walked
 * forward (block 0 first) or in reverse (last block first).
 *
 * Arithmetic: logits, P, l, the accumulator and the epilogue in FP32 (the
 * kernel's precision); each block's P^ V product is exact (E4M3 x E4M3
 * products summed in FP64) and rounded once to FP32 when it is added, as an
 * FP32-accumulating tensor core adds a block product into its accumulator.
 *
 * Counting: a key j >= n_sink that is visible (not causally masked) and whose
 * cast value P^_j is zero is an underflow; counts[0] tallies those in the
 * block that holds key 0 (the sink block), counts[1] those in every other
 * block; eligible[0..1] tallies the visible non-sink keys likewise. */
static void emulate_row(const float* qi, const float* K, const float* V,
                        int N, int d, int causal, int i, int Bc, float S,
                        int reverse, int cast, int n_sink,
                        float* acc, float* s, double* pv,
                        float* o_f32, float* lse_out, int64_t* counts, int64_t* eligible)
{
    const double rsd = sqrt((double)d);
    const int nblocks = (N + Bc - 1) / Bc;
    /* causal: blocks after the one holding key i are entirely masked and are
     * skipped ([FLASH] causal masking section). */
    const int last = causal ? (i / Bc) : (nblocks - 1);

    float m = -INFINITY;
    float l = 0.0f;
    for (int c = 0; c < d; ++c)
        acc[c] = 0.0f;
    counts[0] = counts[1] = 0;
    eligible[0] = eligible[1] = 0;

    for (int step = 0; step <= last; ++step) {
        const int t = reverse ? (last - step) : step;
        const int j0 = t * Bc;
        const int j1 = (j0 + Bc < N) ? (j0 + Bc) : N;

        /* S_ij = Q_i K_j^T / sqrt(d), rounded to FP32; masked keys get -inf. */
        float mt = -INFINITY;
        for (int j = j0; j < j1; ++j) {
            if (causal && j > i) {
                s[j - j0] = -INFINITY;
                continue;
            }
            s[j - j0] = (float)(dot64(qi, K + (int64_t)j * d, d) / rsd);
            if (s[j - j0] > mt)
                mt = s[j - j0];
        }
        /* m_new = max(m_old, rowmax(S_ij)), updated on every block. */
        const float m_new = (mt > m) ? mt : m;
        /* Rescale factor exp(m_old - m_new); zero before the first block. */
        const float alpha = (m == -INFINITY) ? 0.0f : (float)exp((double)(m - m_new));

        float rowsum = 0.0f;
        for (int c = 0; c < d; ++c)
            pv[c] = 0.0;
        for (int j = j0; j < j1; ++j) {
            if (causal && j > i)
                continue;                     /* masked: no mass, not counted */
            const float x = s[j - j0] - m_new;
            const float p = (float)exp((double)x);        /* P = exp(S - m_new) */
            rowsum += p;                                  /* l from FP32 P */
            const float ps = p * S;                       /* P * S in FP32 */
            const float phat = cast ? (float)oracle_e4m3_decode(oracle_e4m3_encode((double)ps))
                                    : ps;                 /* the P-cast */
            if (j >= n_sink) {
                const int where = (t == 0) ? 0 : 1;
                eligible[where] += 1;
                if (phat == 0.0f)
                    counts[where] += 1;
            }
            const float* vj = V + (int64_t)j * d;
            for (int c = 0; c < d; ++c)
                pv[c] += (double)phat * (double)vj[c];
        }
        /* l_new = l_old * exp(m_old - m_new) + rowsum(P);
         * O_new = O_old * exp(m_old - m_new) + P^ V_j. */
        l = l * alpha + rowsum;
        for (int c = 0; c < d; ++c)
            acc[c] = acc[c] * alpha + (float)pv[c];
        m = m_new;
    }
    /* Epilogue: divide S back out together with the softmax denominator. */
    const float den = S * l;
    for (int c = 0; c < d; ++c)
        o_f32[c] = acc[c] / den;
    *lse_out = m + (float)log((double)l);
}

/* Blockwise emulator over a set of query rows (the same positions for every
 * (b, h)).  Outputs: o_f32 [B,H,nrows,d] (FP32 before the output rounding),
 * o_bf16 [B,H,nrows,d] (bfloat16 bits of o_f32, nearest-even), lse
 * [B,H,nrows], counts and eligible [B,H,nrows,2] (sink block, other blocks).
 * reverse: 0 walks KV blocks 0 -> last, 1 walks last -> 0.  cast: 1 applies
 * the E4M3 P-cast, 0 keeps P * S in FP32 (for re-association checks). */
void oracle_emulate(const float* q, const float* k, const float* v,
                    int B, int H, int Hkv, int N, int d, int causal,
                    int Bc, float S, int reverse, int cast, int n_sink,
                    const int32_t* rows, int nrows,
                    float* o_f32, uint16_t* o_bf16, float* lse,
                    int64_t* counts, int64_t* eligible)
{
    int64_t total = (int64_t)B * H * nrows;
#pragma omp parallel
    {
        float* acc = (float*)malloc(sizeof(float) * (size_t)d);
        float* s = (float*)malloc(sizeof(float) * (size_t)Bc);
        double* pv = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (int64_t u = 0; u < total; ++u) {
            int r = (int)(u % nrows);
            int h = (int)((u / nrows) % H);
            int b = (int)(u / ((int64_t)nrows * H));
            int i = rows[r];
            emulate_row(q_row(q, b, h, i, H, N, d), kv_head(k, b, h, H, Hkv, N, d),
                        kv_head(v, b, h, H, Hkv, N, d), N, d, causal, i, Bc, S, reverse,
                        cast, n_sink, acc, s, pv, o_f32 + u * d, lse + u,
                        counts + 2 * u, eligible + 2 * u);
            for (int c = 0; c < d; ++c)
                o_bf16[u * d + c] = oracle_bf16_round(o_f32[u * d + c]);
        }
        free(acc);
        free(s);
        free(pv);
    }
}

/* Threads the OpenMP loops above use (the CPU-baseline core count). */
int oracle_num_threads(void)
{
    return omp_get_max_threads();
}
