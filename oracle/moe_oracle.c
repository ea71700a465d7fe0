/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU reference for one
 * Mixture-of-Experts FFN layer forward and its dense baselines.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library path may link, import or
 * call this file: it exists so that tests, the smoke check and the CPU
 * baseline of the benchmark can check the CUDA path against the definitions.
 * It shares no code, header, table or helper with the CUDA sources.
 *
 * Arithmetic is IEEE double throughout (inputs are widened exactly: a bf16
 * value is the upper 16 bits of an fp32 value), plain loops in the order the
 * definitions are written, no blocking or fusion.
 *
 * Sources (web pages on "Demystifying the Mixture of Experts Serving Tax",
 * MLSys 2026):
 *   - notes.yuuk.io talk notes, section "MoE serving tax: definition"
 *     (Eq. 1, DenseFA / DensePA definitions);
 *   - same page, "Key findings 5" (the stages of the MoE block: router, top-K
 *     selection, alignment, GroupGEMM, local sum);
 *   - same page, "Padding model (Section 5.1)" (block-wise padding
 *     P = sum_i ceil(N_i / B) * B);
 *   - same page, "Balls-Bins-Buckets" (token-count vector N = [N_1..N_E],
 *     m tokens x K assignments);
 *   - same page, Table 2 (shared experts);
 *   - the MoE-Prism write-up (routing top-k as a per-request runtime knob):
 *     per-token dynamic K, k_t <= K, unused slots -1;
 *   - talk notes, "Reduction techniques" (decode: weight quantisation cuts
 *     the expert weights loaded from HBM): FP8 E4M3 expert weights with row
 *     scales (format and scaling are this oracle's reading, stated below).
 * Concrete gating (softmax renormalised over the selected K, or sigmoid
 * normalised over the selected K), SwiGLU experts and the tile size come from
 * the layer definitions of the workloads (Mixtral-, Qwen2-MoE-,
 * DeepSeek-V3-shaped layers).  Readings where the pages are silent:
 *   - top-K is taken on the fp32 router logit, descending, ties broken by
 *     the lower expert index, IEEE comparison (so -0.0 ties +0.0); a NaN
 *     logit is rejected (return -1);
 *   - the K outputs of a token are listed in that order, which fixes k;
 *   - shared experts have weight 1 and no gate; S experts of width I_s are
 *     one dense SwiGLU FFN of width S*I_s;
 *   - padding slots of sorted_ids are -1; blocks past P in block_expert are
 *     -1; experts with N_e = 0 get no rows.
 *
 * Parity status: every function below is pinned by the CPU tests (brute force
 * over subsets, closed forms, invariants, hand-worked fixtures, reductions).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes: 0 = bf16 (uint16 bit patterns), 1 = fp32 */
static double ld(const void* p, size_t i, int dtype)
{
    if (dtype == 0) {
        uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float*)p)[i];
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* ---------------------------------------------------------------- router */
/* logits[t][e] = sum_h x[t][h] * w_r[e][h]  (router GEMM, x.W_r^T) */
int oracle_router_logits(int T, int H, int E, int dtype, const void* x,
                         const void* w_r, double* logits)
{
    if (T < 0 || H <= 0 || E <= 0) return -1;
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += ld(x, (size_t)t * H + h, dtype) * ld(w_r, (size_t)e * H + h, dtype);
            logits[(size_t)t * E + e] = s;
        }
    return 0;
}

/* ------------------------------------------------------------------ top-K */
/* K passes; each pass picks the not-yet-selected expert with the largest
 * logit, the lowest index winning a tie.  ids[t][0..K-1] in selection order. */
/* Per-token dynamic K (the MoE-Prism write-up: the routing top-k as a
 * runtime control knob, per request): token t selects its k_t largest logits,
 * 0 <= k_t <= K, in the same order; slots k >= k_t hold -1 (no assignment).
 * k_per_token == NULL means k_t = K for every token. */
int oracle_topk_k(int T, int E, int K, const int32_t* k_per_token, const float* logits, int32_t* ids)
{
    if (T < 0 || E <= 0 || K <= 0 || K > E) return -1;
    char* taken = (char*)malloc((size_t)E);
    if (!taken) return -2;
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        int kt = k_per_token ? k_per_token[t] : K;
        if (kt < 0 || kt > K) { free(taken); return -1; }
        for (int e = 0; e < E; ++e) {
            if (isnan(l[e])) { free(taken); return -1; }
            taken[e] = 0;
        }
        for (int k = kt; k < K; ++k) ids[(size_t)t * K + k] = -1;
        for (int k = 0; k < kt; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: ties keep lower e */
            }
            taken[best] = 1;
            ids[(size_t)t * K + k] = best;
        }
    }
    free(taken);
    return 0;
}

int oracle_topk(int T, int E, int K, const float* logits, int32_t* ids)
{
    return oracle_topk_k(T, E, K, NULL, logits, ids);
}

/* ---------------------------------------------------------------- weights */
/* score_fn 0 = softmax, 1 = sigmoid.
 * softmax, renorm=1: w_j = exp(l_j - m) / sum_{i in sel} exp(l_i - m), m = max over sel
 * softmax, renorm=0: w_j = exp(l_j - m) / sum_{all e} exp(l_e - m), m = max over all
 * sigmoid, renorm=1: w_j = s_j / sum_{i in sel} s_i,  s = 1/(1+exp(-l))
 * sigmoid, renorm=0: w_j = s_j */
int oracle_gate_weights(int T, int E, int K, int score_fn, int renorm,
                        const float* logits, const int32_t* ids, double* w)
{
    if (T < 0 || E <= 0 || K <= 0 || K > E) return -1;
    if (score_fn != 0 && score_fn != 1) return -1;
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        const int32_t* id = ids + (size_t)t * K;
        double* wt = w + (size_t)t * K;
        /* slots with id -1 (no assignment) get weight 0 and stay out of the sums */
        for (int k = 0; k < K; ++k) if (id[k] >= E || id[k] < -1) return -1;
        if (score_fn == 0) {
            double m = -INFINITY, den = 0.0;
            if (renorm) {
                for (int k = 0; k < K; ++k) if (id[k] >= 0 && (double)l[id[k]] > m) m = l[id[k]];
                for (int k = 0; k < K; ++k) if (id[k] >= 0) den += exp((double)l[id[k]] - m);
            } else {
                for (int e = 0; e < E; ++e) if ((double)l[e] > m) m = l[e];
                for (int e = 0; e < E; ++e) den += exp((double)l[e] - m);
            }
            for (int k = 0; k < K; ++k) wt[k] = id[k] >= 0 ? exp((double)l[id[k]] - m) / den : 0.0;
        } else {
            double den = 0.0;
            for (int k = 0; k < K; ++k) if (id[k] >= 0) den += sigmoid((double)l[id[k]]);
            for (int k = 0; k < K; ++k)
                wt[k] = id[k] < 0 ? 0.0 : (renorm ? sigmoid((double)l[id[k]]) / den : sigmoid((double)l[id[k]]));
        }
    }
    return 0;
}

/* ---------------------------------------------------------- align + pad */
/* Assignments a = t*K + k, expert e(a) = ids[a], A = T*K.
 *   counts[e]  = N_e = #{a : e(a) = e}
 *   padded N^_e = ceil(N_e / B) * B                    (mode 0, block-wise padding)
 *              = ceil(max_i N_i / B) * B for every e    (mode 1, max-value padding:
 *                all experts take the size of the most loaded one; same page,
 *                "Padding model (Section 5.1)", P_g = E_g * ceil(max N_i / B) * B
 *                with E_g = E on one GPU)
 *   offsets    = exclusive scan of N^, offsets[E] = P = sum_e N^_e
 *   sorted_ids[p] = a, a ascending within each expert's segment; -1 elsewhere
 *   pos[a]     = the slot p holding a
 *   block_expert[b] = e for b in [offsets[e]/B, offsets[e+1]/B), -1 for b >= P/B
 *   E_active   = #{e : N_e > 0}
 * sorted_ids has P_max slots, block_expert ceil(P_max/B) entries. */
int oracle_align(int T, int K, int E, int B, int mode, const int32_t* ids, int64_t P_max,
                 int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                 int32_t* block_expert, int32_t* pos, int32_t* P_out,
                 int32_t* E_active_out)
{
    if (T < 0 || K <= 0 || E <= 0 || B <= 0 || (mode != 0 && mode != 1)) return -1;
    int64_t A = (int64_t)T * K;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < A; ++a) {
        if (ids[a] == -1) continue;  /* an empty slot (dynamic K): no assignment */
        if (ids[a] < 0 || ids[a] >= E) return -1;
        counts[ids[a]] += 1;
    }
    int32_t n_max = 0;
    for (int e = 0; e < E; ++e) if (counts[e] > n_max) n_max = counts[e];
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int32_t n = mode == 0 ? counts[e] : n_max;
        int32_t padded = ((n + B - 1) / B) * B;
        offsets[e + 1] = offsets[e] + padded;
    }
    int32_t P = offsets[E];
    if (P > P_max) return -1;
    for (int64_t p = 0; p < P_max; ++p) sorted_ids[p] = -1;
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    if (!cursor) return -2;
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t a = 0; a < A; ++a) {
        int e = ids[a];
        if (e < 0) { pos[a] = -1; continue; }
        sorted_ids[cursor[e]] = (int32_t)a;
        pos[a] = cursor[e];
        cursor[e] += 1;
    }
    free(cursor);
    int64_t nblk = (P_max + B - 1) / B;
    for (int64_t b = 0; b < nblk; ++b) block_expert[b] = -1;
    for (int e = 0; e < E; ++e)
        for (int32_t b = offsets[e] / B; b < offsets[e + 1] / B; ++b) block_expert[b] = e;
    int ea = 0;
    for (int e = 0; e < E; ++e) if (counts[e] > 0) ++ea;
    *P_out = P;
    *E_active_out = ea;
    return 0;
}

/* ---------------------------------------------------------------- permute */
/* x_perm[p] = x[sorted_ids[p] / K] for p < P; a zero row where sorted_ids[p]
 * is -1 (a padding slot).  Rows are H elements of `dtype`; the output is
 * double. */
int oracle_permute(int H, int K, int dtype, const void* x, const int32_t* sorted_ids, int P,
                   double* x_perm)
{
    if (H <= 0 || K <= 0 || P < 0) return -1;
    for (int p = 0; p < P; ++p) {
        int a = sorted_ids[p];
        for (int h = 0; h < H; ++h)
            x_perm[(size_t)p * H + h] = a < 0 ? 0.0 : ld(x, (size_t)(a / K) * H + h, dtype);
    }
    return 0;
}

/* --------------------------------------------------------------- combine */
/* Local sum: out[t] = sum_{k=0..K-1} w[t][k] * y[pos[t*K+k]] + shared[t]
 * (shared may be NULL).  y and shared rows are H elements of `dtype`. */
int oracle_combine(int T, int H, int K, int dtype, const void* y, const int32_t* pos,
                   const double* w, const void* shared, double* out)
{
    if (T < 0 || H <= 0 || K <= 0) return -1;
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double s = 0.0;
            for (int k = 0; k < K; ++k) {
                int32_t p = pos[(size_t)t * K + k];
                if (p >= 0) s += w[(size_t)t * K + k] * ld(y, (size_t)p * H + h, dtype);
            }
            if (shared) s += ld(shared, (size_t)t * H + h, dtype);
            out[(size_t)t * H + h] = s;
        }
    return 0;
}

/* ------------------------------------------------------------- SwiGLU FFN */
/* One token through one SwiGLU expert.  w13 is [2I, H]: rows 0..I-1 are the
 * gate projection W1, rows I..2I-1 the up projection W3; w2 is [H, I].
 *   g_i = sum_h W1[i][h] x[h];  u_i = sum_h W3[i][h] x[h]
 *   a_i = silu(g_i) * u_i,      silu(v) = v * sigmoid(v)
 *   y_h = sum_i W2[h][i] a_i
 * x is given as an element offset into a typed array. */
/* --------------------------------------------------------- FP8 weights */
/* Quantised expert weights for the decode streaming path (talk notes,
 * "Reduction techniques / decode optimisation": weight quantisation cuts the
 * expert weights loaded from HBM, more so for MoE than for dense models).
 * The pages fix no format; the reading is FP8 E4M3 with one fp32 scale per
 * output row:
 *   E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent
 *   field 0 holds subnormals m/8 * 2^-6; no infinities; S.1111.111 is NaN;
 *   the largest finite value is 448 (S.1111.110).
 *   Row scale s_r = max_c |w[r][c]| / 448 (fp32; 1 for an all-zero row);
 *   code q[r][c] = E4M3(w[r][c] / s_r), the fp32 quotient rounded to the
 *   nearest E4M3 value, ties to the even mantissa, saturating at +-448;
 *   dequantised weight = value(q) * s_r. */
double oracle_e4m3_value(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10); /* (1 + m/8) 2^(e-7) */
    return sgn ? -v : v;
}

uint8_t oracle_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sgn = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sgn | 0x7E;
    if (a == 0.0) return sgn;
    int k;
    frexp(a, &k);             /* a in [2^(k-1), 2^k) */
    int eb = k - 1;           /* binade exponent */
    double step = eb < -6 ? ldexp(1.0, -9) : ldexp(1.0, eb - 3);
    double q = nearbyint(a / step) * step; /* exact quotient; ties to even (default rounding) */
    if (q == 0.0) return sgn;
    frexp(q, &k);
    eb = k - 1;
    if (eb < -6) return sgn | (uint8_t)(q / ldexp(1.0, -9));      /* subnormal: m = q / 2^-9 */
    int m = (int)((q / ldexp(1.0, eb) - 1.0) * 8.0);
    return sgn | (uint8_t)((eb + 7) << 3) | (uint8_t)m;
}

/* Row-wise quantisation of w [rows, cols] (dtype 0 bf16 / 1 fp32). */
int oracle_quantize_fp8(int rows, int cols, int dtype, const void* w, uint8_t* q, float* scales)
{
    if (rows < 0 || cols <= 0 || (dtype != 0 && dtype != 1)) return -1;
    for (int r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int c = 0; c < cols; ++c) {
            float a = fabsf((float)ld(w, (size_t)r * cols + c, dtype));
            if (a > amax) amax = a;
        }
        float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        scales[r] = sc;
        for (int c = 0; c < cols; ++c) {
            float v = (float)ld(w, (size_t)r * cols + c, dtype) / sc;
            q[(size_t)r * cols + c] = oracle_e4m3_encode(v);
        }
    }
    return 0;
}

/* One token through one FP8 expert: as ffn_one with w = value(q) * s_row. */
static void ffn_one_fp8(int H, int I, int dtype, const void* x, size_t x_off, const uint8_t* q13,
                        const float* s13, const uint8_t* q2, const float* s2, double* a_scratch, double* y)
{
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = ld(x, x_off + h, dtype);
            g += oracle_e4m3_value(q13[(size_t)i * H + h]) * (double)s13[i] * xv;
            u += oracle_e4m3_value(q13[(size_t)(I + i) * H + h]) * (double)s13[I + i] * xv;
        }
        a_scratch[i] = g * sigmoid(g) * u;
    }
    for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += oracle_e4m3_value(q2[(size_t)h * I + i]) * (double)s2[h] * a_scratch[i];
        y[h] = acc;
    }
}

static void ffn_one(int H, int I, int dtype, const void* x, size_t x_off,
                    const void* w13, const void* w2, double* a_scratch, double* y)
{
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            double xv = ld(x, x_off + h, dtype);
            g += ld(w13, (size_t)i * H + h, dtype) * xv;
            u += ld(w13, (size_t)(I + i) * H + h, dtype) * xv;
        }
        a_scratch[i] = g * sigmoid(g) * u;
    }
    for (int h = 0; h < H; ++h) {
        double s = 0.0;
        for (int i = 0; i < I; ++i) s += ld(w2, (size_t)h * I + i, dtype) * a_scratch[i];
        y[h] = s;
    }
}

/* y[H] for one token row x[H] through one expert (exported for the tests). */
int oracle_swiglu_ffn(int H, int I, int dtype, const void* x, const void* w13,
                      const void* w2, double* y)
{
    if (H <= 0 || I <= 0) return -1;
    double* a = (double*)malloc(sizeof(double) * (size_t)I);
    if (!a) return -2;
    ffn_one(H, I, dtype, x, 0, w13, w2, a, y);
    free(a);
    return 0;
}

/* Dense SwiGLU FFN over T tokens (DenseFA / DensePA / shared experts):
 * out[t] = W2 (silu(W1 x_t) * (W3 x_t)).  Its own loops: no routing. */
int oracle_dense_ffn(int T, int H, int I, int dtype, const void* x,
                     const void* w13, const void* w2, double* out, int nthreads)
{
    if (T < 0 || H <= 0 || I <= 0) return -1;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)I);
        double* u = (double*)malloc(sizeof(double) * (size_t)I);
        if (!g || !u) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int t = 0; t < T; ++t) {
                for (int i = 0; i < I; ++i) {
                    g[i] = 0.0;
                    u[i] = 0.0;
                }
                for (int i = 0; i < I; ++i)
                    for (int h = 0; h < H; ++h) {
                        double xv = ld(x, (size_t)t * H + h, dtype);
                        g[i] += ld(w13, (size_t)i * H + h, dtype) * xv;
                        u[i] += ld(w13, (size_t)(I + i) * H + h, dtype) * xv;
                    }
                for (int h = 0; h < H; ++h) {
                    double s = 0.0;
                    for (int i = 0; i < I; ++i)
                        s += ld(w2, (size_t)h * I + i, dtype) * (g[i] * sigmoid(g[i]) * u[i]);
                    out[(size_t)t * H + h] = s;
                }
            }
        }
        free(g);
        free(u);
    }
    return err;
}

/* ------------------------------------------------------------- MoE layer */
/* Full layer forward for the tokens listed in `tokens` (n_tok of them; NULL
 * means all T in order).  For each listed token t:
 *   1. l = logits_in[t] if given, else fp32(x_t . W_r^T) from the router GEMM;
 *   2. top-K ids (descending logit, lower index on ties);
 *   3. gate weights (softmax / sigmoid, renormalised or not);
 *   4. y_k = SwiGLU expert ids[k] applied to x_t directly (no permutation);
 *   5. shared: y_s = SwiGLU with the shared weights (I_sh = S*I_s; 0 = none);
 *   6. out[j] = sum_k w_k y_k + y_s.
 * w13[e] / w2[e] point at expert e's [2I,H] and [H,I] weights (entries for
 * experts no listed token selects may be NULL).  ids_out / w_out (nullable)
 * receive the routing of each listed token.  Returns -1 on bad input
 * (NaN logit, NULL weight of a selected expert). */
/* wfmt 0: weights of `dtype`; wfmt 1: FP8 codes (uint8) with fp32 row scales
 * s13 / s2 (per expert) and s13_sh / s2_sh. */
static int layer_impl(int T, int H, int E, int K, int I, int I_sh, int score_fn,
                      int renorm, int dtype, int wfmt, const void* x, const void* w_r,
                      const void* const* w13, const void* const* w2,
                      const float* const* s13, const float* const* s2,
                      const void* w13_sh, const void* w2_sh, const float* s13_sh, const float* s2_sh,
                      const float* logits_in, const int32_t* k_per_token,
                      const int32_t* tokens, int n_tok, double* out,
                      int32_t* ids_out, double* w_out, int nthreads)
{
    if (T < 0 || H <= 0 || E <= 0 || K <= 0 || K > E || I <= 0 || I_sh < 0) return -1;
    if (n_tok < 0) return -1;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        float* l = (float*)malloc(sizeof(float) * (size_t)E);
        double* ld_logits = (double*)malloc(sizeof(double) * (size_t)E);
        int32_t* id = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
        double* w = (double*)malloc(sizeof(double) * (size_t)K);
        int Imax = I > I_sh ? I : I_sh;
        double* a = (double*)malloc(sizeof(double) * (size_t)(Imax > 0 ? Imax : 1));
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        if (!l || !ld_logits || !id || !w || !a || !y) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int j = 0; j < n_tok; ++j) {
                int t = tokens ? tokens[j] : j;
                if (t < 0 || t >= T) {
#pragma omp atomic write
                    err = -1;
                    continue;
                }
                size_t xo = (size_t)t * H;
                if (logits_in) {
                    for (int e = 0; e < E; ++e) l[e] = logits_in[(size_t)t * E + e];
                } else {
                    for (int e = 0; e < E; ++e) {
                        double s = 0.0;
                        for (int h = 0; h < H; ++h)
                            s += ld(x, xo + h, dtype) * ld(w_r, (size_t)e * H + h, dtype);
                        ld_logits[e] = s;
                        l[e] = (float)s;
                    }
                }
                if (oracle_topk_k(1, E, K, k_per_token ? k_per_token + t : NULL, l, id) != 0 ||
                    oracle_gate_weights(1, E, K, score_fn, renorm, l, id, w) != 0) {
#pragma omp atomic write
                    err = -1;
                    continue;
                }
                double* o = out + (size_t)j * H;
                for (int h = 0; h < H; ++h) o[h] = 0.0;
                for (int k = 0; k < K; ++k) {
                    int e = id[k];
                    if (e < 0) continue;  /* empty slot */
                    if (!w13[e] || !w2[e] || (wfmt == 1 && (!s13[e] || !s2[e]))) {
#pragma omp atomic write
                        err = -1;
                        break;
                    }
                    if (wfmt == 1)
                        ffn_one_fp8(H, I, dtype, x, xo, (const uint8_t*)w13[e], s13[e], (const uint8_t*)w2[e],
                                    s2[e], a, y);
                    else
                        ffn_one(H, I, dtype, x, xo, w13[e], w2[e], a, y);
                    for (int h = 0; h < H; ++h) o[h] += w[k] * y[h];
                }
                if (I_sh > 0) {
                    if (wfmt == 1)
                        ffn_one_fp8(H, I_sh, dtype, x, xo, (const uint8_t*)w13_sh, s13_sh, (const uint8_t*)w2_sh,
                                    s2_sh, a, y);
                    else
                        ffn_one(H, I_sh, dtype, x, xo, w13_sh, w2_sh, a, y);
                    for (int h = 0; h < H; ++h) o[h] += y[h];
                }
                if (ids_out)
                    for (int k = 0; k < K; ++k) ids_out[(size_t)j * K + k] = id[k];
                if (w_out)
                    for (int k = 0; k < K; ++k) w_out[(size_t)j * K + k] = w[k];
            }
        }
        free(l);
        free(ld_logits);
        free(id);
        free(w);
        free(a);
        free(y);
    }
    return err;
}

int oracle_moe_layer(int T, int H, int E, int K, int I, int I_sh, int score_fn,
                     int renorm, int dtype, const void* x, const void* w_r,
                     const void* const* w13, const void* const* w2,
                     const void* w13_sh, const void* w2_sh, const float* logits_in,
                     const int32_t* k_per_token,
                     const int32_t* tokens, int n_tok, double* out,
                     int32_t* ids_out, double* w_out, int nthreads)
{
    return layer_impl(T, H, E, K, I, I_sh, score_fn, renorm, dtype, 0, x, w_r, w13, w2, NULL, NULL, w13_sh,
                      w2_sh, NULL, NULL, logits_in, k_per_token, tokens, n_tok, out, ids_out, w_out, nthreads);
}

/* The layer with FP8 expert weights (routed and shared): q13[e] / q2[e] the
 * E4M3 codes of expert e ([2I,H], [H,I]), s13[e] / s2[e] its row scales ([2I],
 * [H]); x and the router are of `dtype`. */
int oracle_moe_layer_fp8(int T, int H, int E, int K, int I, int I_sh, int score_fn,
                         int renorm, int dtype, const void* x, const void* w_r,
                         const void* const* q13, const void* const* q2,
                         const float* const* s13, const float* const* s2,
                         const void* q13_sh, const void* q2_sh, const float* s13_sh, const float* s2_sh,
                         const float* logits_in, const int32_t* k_per_token,
                         const int32_t* tokens, int n_tok, double* out, int nthreads)
{
    return layer_impl(T, H, E, K, I, I_sh, score_fn, renorm, dtype, 1, x, w_r, q13, q2, s13, s2, q13_sh,
                      q2_sh, s13_sh, s2_sh, logits_in, k_per_token, tokens, n_tok, out, NULL, NULL, nthreads);
}
