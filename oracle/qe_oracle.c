/*
 * Plain CPU oracle for the Quant Experts (QE) compensated quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library. The product
 * path never calls it. It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes, and where each step is defined:
 *   Quant Experts (MCISLAB DeepRead summary), Method: token-aware important
 *     channel partitioning: w = Meanrow(|W_f|) per input channel, and per
 *     token Top-k(|x_t| * w). Channel frequencies are counted over calibration
 *     tokens.                                           -> oracle_topk, w_mean
 *   same page, Method, Shared Expert: channel-wise scaling, with activations
 *     divided by s and weights multiplied by s, before low-bit quantization.
 *     E = W_f - W_q is reconstructed by low-rank adapters.
 *                                       -> oracle_quantize_weights, oracle_act_quant
 *   same page, Method, Routed Experts: one router picks, per token, the routed
 *     expert with the smallest predicted residual error. Every token uses the
 *     shared expert plus that one routed expert.
 *                                       -> oracle_route, oracle_qe_forward
 *   Quant Experts (thelatestinai listing), Table 7: the QE linear costs
 *     s*d^2 + s*d(2r + N_r), so the router is one d x N_r linear map.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   symmetric RTN. Weights use one fp32 scale per (output row, K group) and
 *   activations one fp32 scale per token. qmax = 2^(b-1)-1. A scale is
 *   absmax/qmax and a code is clamp(rint(v/scale), -qmax, qmax) with
 *   round-half-to-even. A zero absmax gives a zero scale and zero codes.
 *   Every one of those steps is one IEEE fp32 operation, so the integer codes
 *   are defined bit-exactly. v = x*s_inv for activations (s_inv = fl32(1/s)
 *   is the stored smoothing factor) and v = w*s for weights. The adapters
 *   read the raw X. The router is L = X*G and e = argmin (ties -> lowest e).
 *   W3A16/W4A16 weight-only layers round x*s_inv to bf16 (the 16-bit
 *   activation) and keep the dequantized weight q*sw exact.
 *
 * Everything after the integer codes is exact: int64 dot products and fp64
 * sums of exactly representable products.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fPIC -shared [-fopenmp]
 * (compiled by oracle/build.py). The optional OpenMP pragma only runs
 * independent tokens in parallel. It changes no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

static int qmax_of(int bits) { return (1 << (bits - 1)) - 1; }

/* Round-to-nearest-even fp32 -> bf16 (returned widened to fp32). Not used on NaN/Inf. */
static float round_bf16(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u = u + 0x7FFFu + lsb;
    u &= 0xFFFF0000u;
    float r;
    memcpy(&r, &u, 4);
    return r;
}

/*
 * fp32 -> fp16 (IEEE binary16) with round-to-nearest-even, returned widened to fp32: the value is
 * rounded to a multiple of its binary16 quantum, 2^(e-10) in the normal range (e >= -14, where
 * 2^e <= |v| < 2^(e+1)) and 2^-24 below it (subnormals). A magnitude that rounds beyond the
 * largest finite binary16 (65504) saturates to it: the stored scale stays finite (a reading of
 * the library's; the pages give no fp16 format). Not used on NaN/Inf.
 */
static float round_fp16(float v) {
    if (v == 0.0f) return v;
    int e;
    frexpf(v, &e);          /* |v| = m * 2^e, m in [0.5, 1): 2^(e-1) <= |v| < 2^e */
    e -= 1;
    if (e < -14) e = -14;   /* subnormal range: quantum 2^-24 */
    const float quantum = ldexpf(1.0f, e - 10);
    volatile float q = v / quantum;   /* exact: division by a power of two */
    float r = rintf(q) * quantum;     /* ties to even */
    if (r > 65504.0f) r = 65504.0f;
    if (r < -65504.0f) r = -65504.0f;
    return r;
}

/* One symmetric RTN code: clamp(rint(fl32(v / scale)), -qmax, qmax); zero scale -> 0. */
static int rtn_code(float v, float scale, int qmax) {
    if (scale == 0.0f) return 0;
    volatile float quot = v / scale;  /* one IEEE fp32 division */
    float r = rintf(quot);            /* ties to even in the default rounding mode */
    if (r > (float)qmax) r = (float)qmax;
    if (r < (float)-qmax) r = (float)-qmax;
    return (int)r;
}

/*
 * Weight quantization with channel scaling (Shared Expert paragraph, DeepRead
 * summary: weights are multiplied by the per-channel factor s). scale_fp16 != 0
 * stores every group scale as fp16 (an optional byte saving the pages do not
 * fix: the fp32 scale is rounded to fp16 and the codes are computed from the
 * stored value).
 *   W [N][K] fp32 values (bf16-stored weights widened exactly), s [K].
 *   codes [N][K] int8, scales [N][K/group] (natural row-major layout),
 *   w_mean [K] = Meanrow(|W|) (mean over the N output rows, fp64 sum, one
 *   rounding), w_colmax [K] = max_o |W[o][k]|.
 */
int oracle_quantize_weights(const float* W, const float* s, int N, int K, int group, int bits, int scale_fp16,
                            int8_t* codes, float* scales, float* w_mean, float* w_colmax) {
    if (N <= 0 || K <= 0 || group <= 0 || K % group != 0 || bits < 2 || bits > 8) return ORACLE_BAD_ARG;
    const int qmax = qmax_of(bits);
    const int G = K / group;
    for (int o = 0; o < N; ++o) {
        for (int j = 0; j < G; ++j) {
            float amax = 0.0f;
            for (int k = j * group; k < (j + 1) * group; ++k) {
                volatile float ws = W[(size_t)o * K + k] * s[k];
                float a = fabsf(ws);
                if (a > amax) amax = a;
            }
            volatile float sc = amax / (float)qmax;
            /* fp16 scales: the stored scale is fp16(sc), and the codes are recomputed from it */
            if (scale_fp16) sc = round_fp16(sc);
            scales[(size_t)o * G + j] = sc;
            for (int k = j * group; k < (j + 1) * group; ++k) {
                volatile float ws = W[(size_t)o * K + k] * s[k];
                codes[(size_t)o * K + k] = (int8_t)rtn_code(ws, sc, qmax);
            }
        }
    }
    if (w_mean || w_colmax) {
        for (int k = 0; k < K; ++k) {
            double sum = 0.0;
            float cmax = 0.0f;
            for (int o = 0; o < N; ++o) {
                float a = fabsf(W[(size_t)o * K + k]);
                sum += (double)a;
                if (a > cmax) cmax = a;
            }
            if (w_mean) w_mean[k] = (float)(sum / (double)N);
            if (w_colmax) w_colmax[k] = cmax;
        }
    }
    return ORACLE_OK;
}

/*
 * Per-token symmetric activation quantization of X/s (Shared Expert
 * paragraph: activations are divided by s). X [T][K] fp32 values.
 * q [T][K] int8, sa [T].
 */
int oracle_act_quant(const float* X, const float* s_inv, int T, int K, int bits, int8_t* q, float* sa) {
    if (T < 0 || K <= 0 || bits < 2 || bits > 8) return ORACLE_BAD_ARG;
    const int qmax = qmax_of(bits);
    for (int t = 0; t < T; ++t) {
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            volatile float v = X[(size_t)t * K + k] * s_inv[k];
            float a = fabsf(v);
            if (a > amax) amax = a;
        }
        volatile float sc = amax / (float)qmax;
        sa[t] = sc;
        for (int k = 0; k < K; ++k) {
            volatile float v = X[(size_t)t * K + k] * s_inv[k];
            q[(size_t)t * K + k] = (int8_t)rtn_code(v, sc, qmax);
        }
    }
    return ORACLE_OK;
}

/*
 * Router (Routed Experts paragraph: the router estimates each expert's
 * remaining error and the token takes the smallest). Table 7 prices it at
 * s*d*N_r, so it is one linear map G [K][Nr].
 * L [T][Nr] = X G in fp64. e[t] = argmin_e L[t][e], with exact ties going to the lowest e.
 */
int oracle_route(const float* X, const float* G, int T, int K, int Nr, double* L, int32_t* e) {
    if (T < 0 || K <= 0 || Nr <= 0) return ORACLE_BAD_ARG;
    for (int t = 0; t < T; ++t) {
        int best = 0;
        double bestv = 0.0;
        for (int r = 0; r < Nr; ++r) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += (double)X[(size_t)t * K + k] * (double)G[(size_t)k * Nr + r];
            if (L) L[(size_t)t * Nr + r] = acc;
            if (r == 0 || acc < bestv) { best = r; bestv = acc; }
        }
        e[t] = best;
    }
    return ORACLE_OK;
}

/*
 * Token -> expert buckets: a stable counting sort by e. perm[p] is the token
 * at sorted position p, and offsets[r]..offsets[r+1] is expert r's range.
 */
int oracle_bucket(const int32_t* e, int T, int Nr, int32_t* perm, int32_t* offsets) {
    if (T < 0 || Nr <= 0) return ORACLE_BAD_ARG;
    for (int r = 0; r <= Nr; ++r) offsets[r] = 0;
    for (int t = 0; t < T; ++t) {
        if (e[t] < 0 || e[t] >= Nr) return ORACLE_BAD_ARG;
        offsets[e[t] + 1] += 1;
    }
    for (int r = 0; r < Nr; ++r) offsets[r + 1] += offsets[r];
    int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)Nr);
    if (!fill) return ORACLE_BAD_ARG;
    for (int r = 0; r < Nr; ++r) fill[r] = offsets[r];
    for (int t = 0; t < T; ++t) perm[fill[e[t]]++] = t;
    free(fill);
    return ORACLE_OK;
}

/* acc[t][o][j] = sum_{k in group j} xq[t][k] * wq[o][k] (exact int64). */
int oracle_group_acc(const int8_t* xq, const int8_t* wq, int T, int N, int K, int group, int64_t* acc) {
    if (T < 0 || N <= 0 || K <= 0 || group <= 0 || K % group != 0) return ORACLE_BAD_ARG;
    const int G = K / group;
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < N; ++o)
            for (int j = 0; j < G; ++j) {
                int64_t a = 0;
                for (int k = j * group; k < (j + 1) * group; ++k)
                    a += (int64_t)xq[(size_t)t * K + k] * (int64_t)wq[(size_t)o * K + k];
                acc[((size_t)t * N + o) * G + j] = a;
            }
    return ORACLE_OK;
}

/*
 * The QE linear layer, one token row at a time:
 *   Y[t] = dequant(Q_A(x_t/s)) . dequant(Q_W(W s))^T + (x_t A_s) B_s + (x_t A_r[e]) B_r[e]
 * with e = e(t) from the router (or expert_override[i] when given).
 *
 * Inputs (fp32 values; bf16-stored tensors widened exactly):
 *   X [T][K]; wcodes [N][K] int8; wscales [N][K/group]; s_inv [K];
 *   A_s [K][rs]; B_s [rs][N]; A_r [Nr][K][rr]; B_r [Nr][rr][N]; G [K][Nr].
 *   a_bits in {2..8}: per-token activation quantization (W4A8/W4A6 ...).
 *   a_bits == 16: weight-only layer. The activation is bf16(fl32(x*s_inv)) and
 *                 the weight is the exact q*sw.
 *   rows [n_rows] token indices to evaluate (NULL: all T in order).
 * Outputs, for each evaluated row i: Y [n_rows][N] fp64, expert [n_rows].
 */
int oracle_qe_forward(const float* X, int T, int K, int N, int group, int a_bits,
                      const int8_t* wcodes, const float* wscales, const float* s_inv,
                      const float* A_s, const float* B_s, int rs,
                      const float* A_r, const float* B_r, int Nr, int rr,
                      const float* G, const int32_t* rows, int n_rows,
                      const int32_t* expert_override, double* Y, int32_t* expert) {
    if (T < 0 || K <= 0 || N <= 0 || group <= 0 || K % group != 0 || Nr <= 0) return ORACLE_BAD_ARG;
    if (!(a_bits == 16 || (a_bits >= 2 && a_bits <= 8))) return ORACLE_BAD_ARG;
    const int nr_eval = rows ? n_rows : T;
    const int Gk = K / group;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < nr_eval; ++i) {
        const int t = rows ? rows[i] : i;
        if (t < 0 || t >= T) { bad = 1; continue; }
        const float* x = X + (size_t)t * K;
        int8_t* xq = (int8_t*)malloc((size_t)K);
        double* xb = (double*)malloc(sizeof(double) * (size_t)K);
        double* u = (double*)malloc(sizeof(double) * (size_t)(rs + rr + 1));
        double* Lt = (double*)malloc(sizeof(double) * (size_t)Nr);
        float sa = 0.0f;
        /* router */
        int e = 0;
        {
            int32_t et;
            oracle_route(x, G, 1, K, Nr, Lt, &et);
            e = expert_override ? expert_override[i] : et;
        }
        if (expert) expert[i] = e;
        /* activation */
        if (a_bits == 16) {
            for (int k = 0; k < K; ++k) {
                volatile float v = x[k] * s_inv[k];
                xb[k] = (double)round_bf16(v);
            }
        } else {
            oracle_act_quant(x, s_inv, 1, K, a_bits, xq, &sa);
        }
        /* adapter down-projections from the raw x */
        for (int r = 0; r < rs; ++r) {
            double a = 0.0;
            for (int k = 0; k < K; ++k) a += (double)x[k] * (double)A_s[(size_t)k * rs + r];
            u[r] = a;
        }
        for (int r = 0; r < rr; ++r) {
            double a = 0.0;
            for (int k = 0; k < K; ++k) a += (double)x[k] * (double)A_r[((size_t)e * K + k) * rr + r];
            u[rs + r] = a;
        }
        for (int o = 0; o < N; ++o) {
            double y0 = 0.0;
            if (a_bits == 16) {
                for (int j = 0; j < Gk; ++j) {
                    double part = 0.0;
                    for (int k = j * group; k < (j + 1) * group; ++k)
                        part += xb[k] * (double)wcodes[(size_t)o * K + k];
                    y0 += part * (double)wscales[(size_t)o * Gk + j];
                }
            } else {
                for (int j = 0; j < Gk; ++j) {
                    int64_t acc = 0;
                    for (int k = j * group; k < (j + 1) * group; ++k)
                        acc += (int64_t)xq[k] * (int64_t)wcodes[(size_t)o * K + k];
                    y0 += (double)wscales[(size_t)o * Gk + j] * (double)acc;
                }
                y0 *= (double)sa;
            }
            double ad = 0.0;
            for (int r = 0; r < rs; ++r) ad += u[r] * (double)B_s[(size_t)r * N + o];
            for (int r = 0; r < rr; ++r) ad += u[rs + r] * (double)B_r[((size_t)e * rr + r) * N + o];
            Y[(size_t)i * N + o] = y0 + ad;
        }
        free(xq); free(xb); free(u); free(Lt);
    }
    return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* Top-k ordering: larger score first, equal scores -> lower channel index first. */
typedef struct { float score; int32_t idx; } scored_t;
static int cmp_scored(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

/*
 * Token-aware importance (DeepRead summary, Method: Top-k(|x_t| * w) with
 * w = Meanrow(|W_f|); the channel frequency is counted over the tokens).
 * score[t][c] = fl32(|x[t][c]| * w_mean[c]). idx[t][0..k) holds the k
 * largest by full sort. hist[c] += number of tokens whose Top-k holds c.
 */
int oracle_topk(const float* X, const float* w_mean, int T, int K, int k, int32_t* idx, int32_t* hist) {
    if (T < 0 || K <= 0 || k <= 0 || k > K) return ORACLE_BAD_ARG;
    scored_t* buf = (scored_t*)malloc(sizeof(scored_t) * (size_t)K);
    if (!buf) return ORACLE_BAD_ARG;
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < K; ++c) {
            volatile float sc = fabsf(X[(size_t)t * K + c]) * w_mean[c];
            buf[c].score = sc;
            buf[c].idx = c;
        }
        qsort(buf, (size_t)K, sizeof(scored_t), cmp_scored);
        for (int i = 0; i < k; ++i) {
            idx[(size_t)t * k + i] = buf[i].idx;
            if (hist) hist[buf[i].idx] += 1;
        }
    }
    free(buf);
    return ORACLE_OK;
}

/* The bf16 rounding used above, exported so that tests can pin it against torch. */
float oracle_round_bf16(float v) { return round_bf16(v); }
/* The fp16 rounding of the weight scales, exported so that tests can pin it against numpy. */
float oracle_round_fp16(float v) { return round_fp16(v); }
