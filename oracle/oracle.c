/*
 * oracle.c -- plain, slow fp64 CPU oracle for the multi-tenant LoRA hot path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library. The CUDA product path never links,
 * imports or calls it, and it shares no code, header or table with it.
 *
 * What it computes, and where that is defined:
 *   - The LoRA algebra and the batched multi-adapter output
 *       y = x.W + x.A.B,   Y = X.W + (x1.A1.B1, ..., xn.An.Bn)
 *     (Punica README, section "How?"). Here W is stored [N][K] (nn.Linear
 *     layout), so the base term reads x.W^T; A_i is [h_in][r], B_i is [r][h_out],
 *     and every adapter carries a scale s_i: the added term is s_i.(x.A_i).B_i.
 *   - Tokens of many tenants in one batch, each with its own adapter, and an
 *     adapter id of -1 meaning "base model only" (EpiLoRA abstract, sentence 1;
 *     Punica README, "How?": a batch X that maps to each LoRA model).
 *   - Grouping of tokens by adapter (the "segmented gather" of SGMV, Punica
 *     README "How?"): a stable counting sort.
 *   - The 8-bit base GEMM whose epilogue adds every tenant's up-projection
 *     (EpiLoRA abstract, sentences 2-4). The pages do not fix the 8-bit
 *     format or its scaling; this oracle reads it as OCP FP8 E4M3 weights with
 *     one fp32 scale per output channel and E4M3 activations with one fp32
 *     scale per token (amax / 448), rounded to nearest-even with saturation.
 *
 * Every function below is the plain definition: loops in the order the
 * definition states, fp64 accumulation, no blocking, fusion or reordering.
 * Loops over independent output elements are spread over threads with
 * OpenMP; that changes no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Number formats, decoded from their field definitions.               */
/* ------------------------------------------------------------------ */

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double orc_bf16_decode(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 7) & 0xFF;
    int m = h & 0x7F;
    double v;
    if (e == 0xFF)
        v = m ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)m, -126 - 7);           /* subnormal: 0.m * 2^-126 */
    else
        v = ldexp((double)(128 + m), e - 127 - 7); /* normal: 1.m * 2^(e-127) */
    return s ? -v : v;
}

/* OCP FP8 E4M3: 1 sign, 4 exponent bits (bias 7), 3 fraction bits;
 * no infinities; S.1111.111 is NaN; largest finite magnitude 448. */
double orc_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -6 - 3);             /* subnormal: 0.m * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 7 - 3);    /* normal: 1.m * 2^(e-7) */
    return s ? -v : v;
}

/* Round a binary32 value to E4M3: nearest representable value, ties to
 * the code with an even fraction field, magnitudes beyond 448 clamped to
 * 448 (saturating conversion), NaN to the NaN code. Brute force over the
 * 127 non-negative finite codes; the sign is kept, zero included. */
uint8_t orc_e4m3_encode(float f)
{
    if (isnan(f))
        return 0x7F;
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (a >= 448.0)
        return sign | 0x7E;
    int best = 0;
    double best_d = a; /* distance to code 0 (value 0) */
    for (int c = 1; c <= 0x7E; ++c) {
        double d = fabs(a - orc_e4m3_decode((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return sign | (uint8_t)best;
}

/* OCP MX FP4 element (E2M1): 1 sign, 2 exponent bits (bias 1), 1 fraction
 * bit; no infinities or NaN; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double orc_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1;
    int e = (c >> 1) & 3;
    int m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* OCP MX E8M0 block scale: 2^(E - 127); 255 is NaN. */
double orc_e8m0_decode(uint8_t e)
{
    return e == 255 ? NAN : ldexp(1.0, (int)e - 127);
}

/* Nearest E2M1 code to a (finite) value, ties to the code whose fraction bit
 * is 0, magnitudes beyond 6 saturated to 6 (brute force over the 8 codes). */
uint8_t orc_e2m1_encode(double f)
{
    uint8_t sign = signbit(f) ? 8 : 0;
    double a = fabs(f);
    if (a >= 6.0)
        return sign | 7;
    int best = 0;
    double best_d = a;
    for (int c = 1; c <= 7; ++c) {
        double d = fabs(a - orc_e2m1_decode((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return sign | (uint8_t)best;
}

/* ------------------------------------------------------------------ */
/* Segments: stable group-by of token indices by adapter id.           */
/* ------------------------------------------------------------------ */

/*
 * ids[T]: adapter id per token; -1 (and any id outside [0, n_adapters),
 * counted as bad) means "no adapter".
 * perm[T]: token indices with a valid id, ordered by ascending id and, within
 *   one id, by ascending token index; then the no-adapter tokens in ascending
 *   token index.
 * indptr[n_adapters+1]: indptr[a] = first position of adapter a in perm;
 *   indptr[n_adapters] = number of valid tokens.
 * active[n_adapters]: ids with at least one token, ascending (first n_active
 *   entries meaningful; the rest are set to -1).
 * tok_adapter[T]: the id each token is served with (-1 for none or bad).
 * counts[3]: n_valid, n_active, n_bad.
 * This is the grouping the segmented gather needs and nothing more: how a
 * kernel cuts the segments into units of work is not part of it.
 */
void orc_build_segments(const int32_t* ids, int T, int n_adapters,
                        int32_t* perm, int32_t* indptr, int32_t* active,
                        int32_t* tok_adapter, int32_t* counts)
{
    int32_t* cnt = (int32_t*)calloc((size_t)n_adapters + 1, sizeof(int32_t));
    int32_t* cursor = (int32_t*)calloc((size_t)n_adapters + 1, sizeof(int32_t));
    int n_bad = 0;
    for (int t = 0; t < T; ++t) {
        int id = ids[t];
        int bin;
        if (id >= 0 && id < n_adapters) {
            bin = id;
        } else {
            bin = n_adapters;
            if (id != -1)
                ++n_bad;
        }
        tok_adapter[t] = (bin < n_adapters) ? id : -1;
        ++cnt[bin];
    }
    int pos = 0;
    for (int a = 0; a <= n_adapters; ++a) {
        indptr[a] = pos; /* for a == n_adapters: start of the no-adapter tail */
        cursor[a] = pos;
        pos += cnt[a];
    }
    for (int t = 0; t < T; ++t) {
        int id = ids[t];
        int bin = (id >= 0 && id < n_adapters) ? id : n_adapters;
        perm[cursor[bin]++] = t;
    }
    int n_active = 0;
    for (int a = 0; a < n_adapters; ++a)
        if (cnt[a] > 0)
            active[n_active++] = a;
    for (int s = n_active; s < n_adapters; ++s)
        active[s] = -1;
    counts[0] = indptr[n_adapters];
    counts[1] = n_active;
    counts[2] = n_bad;
    free(cnt);
    free(cursor);
}

/* ------------------------------------------------------------------ */
/* LoRA shrink (down-projection) and expand (up-projection).           */
/* ------------------------------------------------------------------ */

static int valid_id(const int32_t* ids, int t, int n_adapters)
{
    int a = ids[t];
    return (a >= 0 && a < n_adapters) ? a : -1;
}

static int rank_of(const int32_t* ranks, int a, int r_max)
{
    return ranks ? ranks[a] : r_max;
}

/*
 * v[t][j] = sum_k x[t][k] * A[id_t][k][j] for j < r_{id_t}; 0 for j >= r_{id_t}
 * and for tokens without an adapter. x bf16 [T][h_in], A bf16
 * [n_adapters][h_in][r_max], v fp64 [T][r_max].
 * (Punica README "How?": the x_i.A_i half of x_i.A_i.B_i.)
 */
void orc_lora_shrink(const uint16_t* x, int T, int h_in, const uint16_t* A,
                     int n_adapters, int r_max, const int32_t* ranks,
                     const int32_t* ids, double* v)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        int a = valid_id(ids, t, n_adapters);
        for (int j = 0; j < r_max; ++j)
            v[(size_t)t * r_max + j] = 0.0;
        if (a < 0)
            continue;
        int r = rank_of(ranks, a, r_max);
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int k = 0; k < h_in; ++k)
                acc += orc_bf16_decode(x[(size_t)t * h_in + k]) *
                       orc_bf16_decode(A[((size_t)a * h_in + k) * r_max + j]);
            v[(size_t)t * r_max + j] = acc;
        }
    }
}

/*
 * y_out[t][n] = y_in[t][n] + s_{id_t} * sum_{j < r_{id_t}} v[t][j] * B[id_t][j][n]
 * for tokens with an adapter; y_out = y_in for the others.
 * v fp64 [T][r_max], B bf16 [n_adapters][r_max][h_out], y_in bf16 [T][h_out],
 * y_out fp64 [T][h_out]. scales NULL means s = 1.
 * (Punica README "How?": the (x_i.A_i).B_i half, added to the base output.)
 */
void orc_lora_expand(const double* v, int T, int r_max, const uint16_t* B,
                     int n_adapters, int h_out, const int32_t* ranks,
                     const float* scales, const int32_t* ids,
                     const uint16_t* y_in, double* y_out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        int a = valid_id(ids, t, n_adapters);
        for (int n = 0; n < h_out; ++n) {
            double y = orc_bf16_decode(y_in[(size_t)t * h_out + n]);
            if (a >= 0) {
                int r = rank_of(ranks, a, r_max);
                double s = scales ? (double)scales[a] : 1.0;
                double acc = 0.0;
                for (int j = 0; j < r; ++j)
                    acc += v[(size_t)t * r_max + j] *
                           orc_bf16_decode(B[((size_t)a * r_max + j) * h_out + n]);
                y += s * acc;
            }
            y_out[(size_t)t * h_out + n] = y;
        }
    }
}

/* Shrink then expand, with v kept in fp64 (never rounded). */
void orc_lora_apply(const uint16_t* x, int T, int h_in, int h_out,
                    const uint16_t* A, const uint16_t* B, int n_adapters,
                    int r_max, const int32_t* ranks, const float* scales,
                    const int32_t* ids, const uint16_t* y_in, double* y_out)
{
    double* v = (double*)malloc(sizeof(double) * (size_t)T * (size_t)r_max);
    orc_lora_shrink(x, T, h_in, A, n_adapters, r_max, ranks, ids, v);
    orc_lora_expand(v, T, r_max, B, n_adapters, h_out, ranks, scales, ids, y_in, y_out);
    free(v);
}

/* ------------------------------------------------------------------ */
/* Base linear layers.                                                 */
/* ------------------------------------------------------------------ */

/* y[m][n] = sum_k x[m][k] * W[n][k] for the listed (m, n) samples;
 * x bf16 [M][K], W bf16 [N][K]. (Punica README "How?": the X.W term.) */
void orc_linear_bf16_sampled(const uint16_t* x, const uint16_t* W, int K,
                             const int32_t* rows, const int32_t* cols,
                             int n_samples, double* out)
{
#pragma omp parallel for schedule(static)
    for (int i = 0; i < n_samples; ++i) {
        const uint16_t* xr = x + (size_t)rows[i] * K;
        const uint16_t* wr = W + (size_t)cols[i] * K;
        double acc = 0.0;
        for (int k = 0; k < K; ++k)
            acc += orc_bf16_decode(xr[k]) * orc_bf16_decode(wr[k]);
        out[i] = acc;
    }
}

/*
 * Per-row FP8 quantisation (one scale per row):
 *   amax = max_k |x[m][k]|;  sx[m] = fl32(amax / 448), or 1 when amax == 0;
 *   xq[m][k] = E4M3(fl32(x[m][k] / sx[m])).
 * Both divisions are IEEE binary32 divisions, rounded to nearest.
 * Serves activations (per token) and weights (per output channel) alike.
 */
void orc_quantize_rows(const uint16_t* x, int M, int K, uint8_t* xq, float* sx)
{
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) {
        double amax = 0.0;
        for (int k = 0; k < K; ++k) {
            double a = fabs(orc_bf16_decode(x[(size_t)m * K + k]));
            if (a > amax)
                amax = a;
        }
        float famax = (float)amax; /* exact: a bf16 magnitude */
        volatile float s = (famax == 0.0f) ? 1.0f : famax / 448.0f;
        sx[m] = s;
        for (int k = 0; k < K; ++k) {
            float xv = (float)orc_bf16_decode(x[(size_t)m * K + k]); /* exact */
            volatile float q = xv / s;
            xq[(size_t)m * K + k] = orc_e4m3_encode(q);
        }
    }
}

/*
 * FP8 base GEMM with the LoRA up-projection added in its epilogue, at the
 * listed (m, n) samples:
 *   y[m][n] = sx[m] * sw[n] * sum_k E4M3(xq[m][k]) * E4M3(Wq[n][k])
 *           + s_a * sum_{j < r_a} (sum_k x[m][k] * A[a][k][j]) * B[a][j][n],
 *   a = ids[m]; the LoRA term is absent when a is -1 / out of range or A is
 *   NULL. The LoRA term uses the unquantised bf16 x.
 * (EpiLoRA abstract, sentences 3-4: the GEMM adds every tenant's
 * up-projection of the down-projected x in its epilogue.)
 */
void orc_fp8_gemm_lora_sampled(const uint8_t* xq, const float* sx,
                               const uint8_t* Wq, const float* sw, int K,
                               const uint16_t* x, const uint16_t* A,
                               const uint16_t* B, int n_adapters, int r_max,
                               int h_out, const int32_t* ranks,
                               const float* scales, const int32_t* ids,
                               const int32_t* rows, const int32_t* cols,
                               int n_samples, double* out)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int i = 0; i < n_samples; ++i) {
        int m = rows[i], n = cols[i];
        double acc = 0.0;
        for (int k = 0; k < K; ++k)
            acc += orc_e4m3_decode(xq[(size_t)m * K + k]) *
                   orc_e4m3_decode(Wq[(size_t)n * K + k]);
        double y = (double)sx[m] * (double)sw[n] * acc;
        if (A != NULL) {
            int a = valid_id(ids, m, n_adapters);
            if (a >= 0) {
                int r = rank_of(ranks, a, r_max);
                double s = scales ? (double)scales[a] : 1.0;
                double l = 0.0;
                for (int j = 0; j < r; ++j) {
                    double vj = 0.0;
                    for (int k = 0; k < K; ++k)
                        vj += orc_bf16_decode(x[(size_t)m * K + k]) *
                              orc_bf16_decode(A[((size_t)a * K + k) * r_max + j]);
                    l += vj * orc_bf16_decode(B[((size_t)a * r_max + j) * h_out + n]);
                }
                y += s * l;
            }
        }
        out[i] = y;
    }
}

/*
 * Token-wise merge of the selected adapters into the backbone (LoRA-Switch
 * abstract on the shd-paper.top page: for each token a router picks LoRA
 * adapters, which are merged into the backbone weights before the token is
 * decoded, all selected adapters in one fused operation). With W stored
 * [N][K] (y = x.W^T) and the Punica README's identity x.(W + A.B) =
 * x.W + x.A.B, merging adapter a with router gate g adds g.s_a.(A_a.B_a)^T:
 *   out[n][k] = W[n][k] + sum_e gates[e] * s_{sel[e]}
 *                         * sum_{j < r_{sel[e]}} A[sel[e]][k][j] * B[sel[e]][j][n]
 * over the n_sel selected entries; an entry with sel[e] outside [0, n_adapters)
 * (-1: no adapter) adds nothing. W, A, B bf16; out fp64 [N][K].
 */
void orc_lora_switch_merge(const uint16_t* W, int N, int K, const uint16_t* A,
                           const uint16_t* B, int n_adapters, int r_max,
                           const int32_t* ranks, const float* scales,
                           const int32_t* sel, const float* gates, int n_sel,
                           double* out)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int k = 0; k < K; ++k) {
            double w = orc_bf16_decode(W[(size_t)n * K + k]);
            for (int e = 0; e < n_sel; ++e) {
                int a = sel[e];
                if (a < 0 || a >= n_adapters)
                    continue;
                int r = rank_of(ranks, a, r_max);
                double s = scales ? (double)scales[a] : 1.0;
                double d = 0.0;
                for (int j = 0; j < r; ++j)
                    d += orc_bf16_decode(A[((size_t)a * K + k) * r_max + j]) *
                         orc_bf16_decode(B[((size_t)a * r_max + j) * N + n]);
                w += (double)gates[e] * s * d;
            }
            out[(size_t)n * K + k] = w;
        }
    }
}

/*
 * Gradients of the LoRA layer for training adapters on a frozen 8-bit base
 * (EpiLoRA abstract, sentence 6: a trainer that keeps the base weights in
 * FP8). The forward is y = x.W^T + s_a.(x.A_a).B_a (the Punica README's
 * "How?" with a scale); for an upstream gradient dY [M][N] the chain rule
 * gives, per token m with adapter a (nothing from the adapter term for -1):
 *   dX[m][k]    = sum_n dY[m][n] W[n][k] + s_a sum_j u[m][j] A_a[k][j],
 *                 u[m][j] = sum_n dY[m][n] B_a[j][n]            (j < r_a)
 *   dA_a[k][j]  = s_a sum_{m with adapter a} x[m][k] u[m][j]     (j < r_a)
 *   dB_a[j][n]  = s_a sum_{m with adapter a} v[m][j] dY[m][n],   v = x.A_a
 * The base weight's term of dX is the 8-bit GEMM of the backward: W^T
 * quantised per input channel (WqT [K][N] E4M3 with fp32 scales swT [K], made
 * once from the frozen W like the forward's Wq) and dY quantised per token
 * the way the forward quantises x (sd[m] = amax_n |dY[m][n]| / 448, dYq =
 * E4M3(dY / sd)), both given here:
 *   base[m][k] = sd[m] swT[k] sum_n E4M3(dYq[m][n]) E4M3(WqT[k][n]).
 * WqT == NULL leaves the base term out. Entries past each adapter's rank
 * (padding) are neither read nor written: dA / dB keep zero there, and they
 * are zero for adapters without tokens. x, dY, A, B bf16; outputs fp64.
 */
void orc_lora_backward(const uint16_t* x, const uint16_t* dY, int M, int K, int N,
                       const uint8_t* dYq, const float* sd, const uint8_t* WqT,
                       const float* swT, const uint16_t* A, const uint16_t* B,
                       int n_adapters, int r_max, const int32_t* ranks,
                       const float* scales, const int32_t* ids, double* dX,
                       double* dA, double* dB)
{
    double* u = (double*)calloc((size_t)M * r_max, sizeof(double));
    double* v = (double*)calloc((size_t)M * r_max, sizeof(double));
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M; ++m) {
        int a = valid_id(ids, m, n_adapters);
        if (a < 0)
            continue;
        int r = rank_of(ranks, a, r_max);
        for (int j = 0; j < r; ++j) {
            double su = 0.0, sv = 0.0;
            for (int n = 0; n < N; ++n)
                su += orc_bf16_decode(dY[(size_t)m * N + n]) *
                      orc_bf16_decode(B[((size_t)a * r_max + j) * N + n]);
            for (int k = 0; k < K; ++k)
                sv += orc_bf16_decode(x[(size_t)m * K + k]) *
                      orc_bf16_decode(A[((size_t)a * K + k) * r_max + j]);
            u[(size_t)m * r_max + j] = su;
            v[(size_t)m * r_max + j] = sv;
        }
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < M; ++m) {
        int a = valid_id(ids, m, n_adapters);
        int r = a >= 0 ? rank_of(ranks, a, r_max) : 0;
        double s = (a >= 0 && scales) ? (double)scales[a] : 1.0;
        for (int k = 0; k < K; ++k) {
            double g = 0.0;
            if (WqT != NULL) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n)
                    acc += orc_e4m3_decode(dYq[(size_t)m * N + n]) *
                           orc_e4m3_decode(WqT[(size_t)k * N + n]);
                g = (double)sd[m] * (double)swT[k] * acc;
            }
            double l = 0.0;
            for (int j = 0; j < r; ++j)
                l += u[(size_t)m * r_max + j] * orc_bf16_decode(A[((size_t)a * K + k) * r_max + j]);
            dX[(size_t)m * K + k] = g + s * l;
        }
    }
    memset(dA, 0, sizeof(double) * (size_t)n_adapters * K * r_max);
    memset(dB, 0, sizeof(double) * (size_t)n_adapters * r_max * N);
#pragma omp parallel for schedule(dynamic, 1)
    for (int a = 0; a < n_adapters; ++a) {
        int r = rank_of(ranks, a, r_max);
        double s = scales ? (double)scales[a] : 1.0;
        for (int m = 0; m < M; ++m) {
            if (valid_id(ids, m, n_adapters) != a)
                continue;
            for (int k = 0; k < K; ++k) {
                double xv = orc_bf16_decode(x[(size_t)m * K + k]);
                for (int j = 0; j < r; ++j)
                    dA[((size_t)a * K + k) * r_max + j] += s * xv * u[(size_t)m * r_max + j];
            }
            for (int j = 0; j < r; ++j)
                for (int n = 0; n < N; ++n)
                    dB[((size_t)a * r_max + j) * N + n] +=
                        s * v[(size_t)m * r_max + j] * orc_bf16_decode(dY[(size_t)m * N + n]);
        }
    }
    free(u);
    free(v);
}

/*
 * MXFP4 quantisation of weight rows (the 4-bit base of the EpiLoRA abstract,
 * sentence 2, read as the OCP MX format): every block of 32 consecutive
 * values of a row shares one E8M0 scale X = 2^(floor(log2(amax)) - 2) (2 is
 * the exponent of E2M1's largest value, 6 = 1.5 * 2^2; the E8M0 exponent is
 * clamped to 0..254, and an all-zero block takes the smallest scale), and
 * each value is rounded to E2M1 as v / X (nearest, ties to even fraction,
 * saturating to +-6). W bf16 [N][K], K a multiple of 32; codes [N][K]
 * (one E2M1 code per byte); scales [N][K / 32] (E8M0 bytes).
 */
void orc_mxfp4_quantize(const uint16_t* W, int N, int K, uint8_t* codes, uint8_t* scales)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int b = 0; b < K / 32; ++b) {
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs(orc_bf16_decode(W[(size_t)n * K + b * 32 + i]));
                if (a > amax)
                    amax = a;
            }
            int e = 0;
            if (amax > 0.0) {
                e = (int)floor(log2(amax)) - 2 + 127;
                if (e < 0)
                    e = 0;
                if (e > 254)
                    e = 254;
            }
            scales[(size_t)n * (K / 32) + b] = (uint8_t)e;
            double x = orc_e8m0_decode((uint8_t)e);
            for (int i = 0; i < 32; ++i) {
                double v = orc_bf16_decode(W[(size_t)n * K + b * 32 + i]);
                codes[(size_t)n * K + b * 32 + i] = orc_e2m1_encode(v / x);
            }
        }
    }
}

/*
 * The MXFP4 base GEMM with the LoRA term, at the listed (m, n) samples, with
 * the activations kept in bf16 (the 16-bit activation engine of the EpiLoRA
 * abstract, sentence 6):
 *   y[m][n] = sum_k x[m][k] * E2M1(codes[n][k]) * E8M0(scales[n][k / 32])
 *           + s_a * sum_{j < r_a} (sum_k x[m][k] A[a][k][j]) * B[a][j][n].
 * A == NULL: no LoRA term. Layouts as orc_mxfp4_quantize.
 */
void orc_mxfp4_gemm_lora_sampled(const uint16_t* x, const uint8_t* codes, const uint8_t* scales,
                                 int K, const uint16_t* A, const uint16_t* B, int n_adapters,
                                 int r_max, int h_out, const int32_t* ranks,
                                 const float* scales_lora, const int32_t* ids,
                                 const int32_t* rows, const int32_t* cols, int n_samples,
                                 double* out)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int i = 0; i < n_samples; ++i) {
        int m = rows[i], n = cols[i];
        double acc = 0.0;
        for (int k = 0; k < K; ++k)
            acc += orc_bf16_decode(x[(size_t)m * K + k]) *
                   orc_e2m1_decode(codes[(size_t)n * K + k]) *
                   orc_e8m0_decode(scales[(size_t)n * (K / 32) + k / 32]);
        double y = acc;
        if (A != NULL) {
            int a = valid_id(ids, m, n_adapters);
            if (a >= 0) {
                int r = rank_of(ranks, a, r_max);
                double s = scales_lora ? (double)scales_lora[a] : 1.0;
                double l = 0.0;
                for (int j = 0; j < r; ++j) {
                    double vj = 0.0;
                    for (int k = 0; k < K; ++k)
                        vj += orc_bf16_decode(x[(size_t)m * K + k]) *
                              orc_bf16_decode(A[((size_t)a * K + k) * r_max + j]);
                    l += vj * orc_bf16_decode(B[((size_t)a * r_max + j) * h_out + n]);
                }
                y += s * l;
            }
        }
        out[i] = y;
    }
}

/*
 * The 8-bit-weight GEMM with the activations kept in bf16 (W8A16: the FP8
 * weights of the EpiLoRA abstract, sentence 2, under its 16-bit activation
 * engine, sentence 6) and the LoRA term, at the listed (m, n) samples:
 *   y[m][n] = sw[n] * sum_k x[m][k] * E4M3(Wq[n][k])
 *           + s_a * sum_{j < r_a} (sum_k x[m][k] A[a][k][j]) * B[a][j][n].
 * A == NULL: no LoRA term. Wq / sw as orc_quantize_rows makes them.
 */
void orc_w8a16_gemm_lora_sampled(const uint16_t* x, const uint8_t* Wq, const float* sw, int K,
                                 const uint16_t* A, const uint16_t* B, int n_adapters, int r_max,
                                 int h_out, const int32_t* ranks, const float* scales,
                                 const int32_t* ids, const int32_t* rows, const int32_t* cols,
                                 int n_samples, double* out)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int i = 0; i < n_samples; ++i) {
        int m = rows[i], n = cols[i];
        double acc = 0.0;
        for (int k = 0; k < K; ++k)
            acc += orc_bf16_decode(x[(size_t)m * K + k]) * orc_e4m3_decode(Wq[(size_t)n * K + k]);
        double y = (double)sw[n] * acc;
        if (A != NULL) {
            int a = valid_id(ids, m, n_adapters);
            if (a >= 0) {
                int r = rank_of(ranks, a, r_max);
                double s = scales ? (double)scales[a] : 1.0;
                double l = 0.0;
                for (int j = 0; j < r; ++j) {
                    double vj = 0.0;
                    for (int k = 0; k < K; ++k)
                        vj += orc_bf16_decode(x[(size_t)m * K + k]) *
                              orc_bf16_decode(A[((size_t)a * K + k) * r_max + j]);
                    l += vj * orc_bf16_decode(B[((size_t)a * r_max + j) * h_out + n]);
                }
                y += s * l;
            }
        }
        out[i] = y;
    }
}

/* Threads the OpenMP loops above use. */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
