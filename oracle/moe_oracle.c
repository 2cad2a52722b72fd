/*
 * CPU oracle for the FP8 MoE expert layer -- TEST INFRASTRUCTURE ONLY.
 * See moe_oracle.h for the sources and the readings this file follows.
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared -lm -lpthread
 * (-ffp-contract=off: every multiply and add below rounds exactly where written).
 */
#include "moe_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

#define GROUP 128

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* E4M3FN: sign, 4 exponent bits (bias 7), 3 mantissa bits. Exponent field 0
 * holds subnormals m/8 * 2^-6; there is no infinity; S.1111.111 is NaN; the
 * largest finite magnitude is 1.75 * 2^8 = 448 (the clamp bound of [P1] 3.3). */
double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round v to the nearest E4M3 value, ties to even, clamping magnitudes at 448
 * ([P1] 3.3: x_fp8 = clamp(round(x / scale), -448, 448)). The sign of zero is kept. */
uint8_t orc_e4m3_encode(float v) {
    uint8_t sign;
    double a, q, r;
    int ex, eu;
    if (isnan(v)) return 0x7F;
    sign = signbit(v) ? 0x80 : 0x00;
    a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    frexp(a, &ex);               /* a = f * 2^ex, f in [0.5, 1) */
    eu = ex - 1;                 /* floor(log2(a)) */
    if (eu < -6) eu = -6;        /* subnormal range shares the 2^-9 spacing */
    q = ldexp(1.0, eu - 3);      /* spacing of representable values near a */
    r = rint(a / q) * q;         /* a / q is exact; rint rounds half to even */
    if (r == 0.0) return sign;
    frexp(r, &ex);
    eu = ex - 1;
    if (eu < -6) return sign | (uint8_t)(r / ldexp(1.0, -9));           /* subnormal */
    return sign | (uint8_t)((eu + 7) << 3) | (uint8_t)(r / ldexp(1.0, eu - 3) - 8.0);
}

float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double once to bf16 (8 significant bits), ties to even ([P1] 3.3). */
uint16_t orc_f64_to_bf16(double v) {
    double a, q, r;
    int ex, eu;
    float f;
    uint32_t u;
    if (isnan(v)) return 0x7FC0;
    a = fabs(v);
    if (a == 0.0 || isinf(v)) {
        f = (float)v;
        memcpy(&u, &f, 4);
        return (uint16_t)(u >> 16);
    }
    frexp(a, &ex);
    eu = ex - 1;
    if (eu < -126) eu = -126;
    q = ldexp(1.0, eu - 7);
    r = rint(a / q) * q;
    if (r >= ldexp(1.0, 128)) r = INFINITY;
    f = (float)(v < 0 ? -r : r);    /* exact: r has at most 8 significant bits */
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* A tiny static-partition thread helper (work split only; the          */
/* arithmetic of each output never depends on the thread count).       */
/* ------------------------------------------------------------------ */
typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end);
typedef struct { range_fn fn; void* ctx; int64_t b, e; } range_job;

static void* range_thread(void* p) {
    range_job* j = (range_job*)p;
    j->fn(j->ctx, j->b, j->e);
    return NULL;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx) {
    pthread_t th[256];
    range_job jobs[256];
    int t, nt = nthreads < 1 ? 1 : (nthreads > 256 ? 256 : nthreads);
    if (nt > n) nt = (int)(n > 0 ? n : 1);
    if (nt == 1) { fn(ctx, 0, n); return; }
    for (t = 0; t < nt; ++t) {
        jobs[t].fn = fn; jobs[t].ctx = ctx;
        jobs[t].b = n * t / nt; jobs[t].e = n * (t + 1) / nt;
        pthread_create(&th[t], NULL, range_thread, &jobs[t]);
    }
    for (t = 0; t < nt; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------ */
/* Router ([P1] 2.2: s = softmax(W_g x + b); [P3] 2.3: fp32 softmax)    */
/* ------------------------------------------------------------------ */
/* Canonical fp32 order for one logit (a reading: the pages fix no order, and
 * bit-identical expert selection needs one). With 32 partial sums:
 *   p_j = fma-chain over h = 128 s + 4 j + i (i = 0..3, s = 0, 1, ...), that
 *         is four consecutive h in every 128-wide block, ascending, from +0;
 *   then pairwise halving p_j <- p_j + p_{j+w} for w = 16, 8, 4, 2, 1;
 *   l = p_0 + b_e. */
typedef struct { int H, E; const uint16_t* x; const float* Wg; const float* bias; float* logits; } logit_ctx;

static void logits_range(void* vctx, int64_t b, int64_t e) {
    logit_ctx* c = (logit_ctx*)vctx;
    float* xf = (float*)malloc(sizeof(float) * (size_t)c->H);
    int64_t t;
    for (t = b; t < e; ++t) {
        int h, ex, j, w;
        for (h = 0; h < c->H; ++h) xf[h] = orc_bf16_to_f32(c->x[t * c->H + h]);
        for (ex = 0; ex < c->E; ++ex) {
            const float* wr = c->Wg + (int64_t)ex * c->H;
            float p[32];
            for (j = 0; j < 32; ++j) {
                float acc = 0.0f;
                int s0, i;
                for (s0 = 0; s0 < c->H; s0 += 128)
                    for (i = 0; i < 4; ++i) {
                        h = s0 + 4 * j + i;
                        if (h < c->H) acc = fmaf(xf[h], wr[h], acc);
                    }
                p[j] = acc;
            }
            for (w = 16; w >= 1; w >>= 1)
                for (j = 0; j < w; ++j) p[j] = p[j] + p[j + w];
            c->logits[t * c->E + ex] = c->bias ? p[0] + c->bias[ex] : p[0];
        }
    }
    free(xf);
}

void orc_router_logits(int T, int H, int E, const uint16_t* x, const float* Wg,
                       const float* bias, float* logits, int nthreads) {
    logit_ctx c = {H, E, x, Wg, bias, logits};
    parallel_for(T, nthreads, logits_range, &c);
}

/* Top-k ([P2] 3.1, [P4] ch.1): the k largest logits, ties to the lower expert
 * index, in descending order. Softmax is monotone, so this is the top-k of s.
 * Weights renormalised over the selected experts ([P4] ch.1 pseudo-code):
 *   w_j = exp(l_j - m) / sum_{i in top-k} exp(l_i - m),  m = the largest logit,
 * which equals s_j / sum_{top-k} s_i. Computed in fp64, rounded to fp32. */
void orc_topk_softmax(int T, int E, int k, const float* logits, int32_t* topk_idx, float* topk_w) {
    int t, j, e;
    char* taken = (char*)malloc((size_t)E);
    for (t = 0; t < T; ++t) {
        const float* l = logits + (int64_t)t * E;
        double den = 0.0, m;
        memset(taken, 0, (size_t)E);
        for (j = 0; j < k; ++j) {
            int best = -1;
            for (e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: ties keep the lower index */
            }
            taken[best] = 1;
            topk_idx[(int64_t)t * k + j] = best;
        }
        m = (double)l[topk_idx[(int64_t)t * k]];
        for (j = 0; j < k; ++j) den += exp((double)l[topk_idx[(int64_t)t * k + j]] - m);
        for (j = 0; j < k; ++j)
            topk_w[(int64_t)t * k + j] = (float)(exp((double)l[topk_idx[(int64_t)t * k + j]] - m) / den);
    }
    free(taken);
}

/* Hash routing ([P3] 2.2: hash(token_id) % num_experts): one expert per token. */
void orc_route_hash(int T, int E, const int32_t* token_ids, int32_t* topk_idx, float* topk_w) {
    int t;
    for (t = 0; t < T; ++t) {
        uint32_t h = (uint32_t)token_ids[t] * 2654435761u;   /* mod 2^32 */
        topk_idx[t] = (int32_t)(h % (uint32_t)E);
        topk_w[t] = 1.0f;
    }
}

/* Capacity ([P4] 2.5: ceil(top-k * N / E) * alpha, truncated as in its worked
 * example int(64 * 1.2) = 76). alpha = cap_num / cap_den, exact integers. */
int64_t orc_capacity(int T, int k, int E, int cap_num, int cap_den) {
    int64_t R = (int64_t)T * k, c;
    if (cap_num <= 0 || cap_den <= 0) return -1;
    c = (R + E - 1) / E;
    return c * cap_num / cap_den;
}

/* ------------------------------------------------------------------ */
/* Dispatch ([P1] 2.1 Concat of the per-expert token sets; [P4] 2.5     */
/* overflow dropped in token order)                                    */
/* ------------------------------------------------------------------ */
int orc_dispatch(int T, int k, int E, const int32_t* topk_idx, int64_t cap, int layout, int pad,
                 int masked_max_m, int64_t rows_cap, int32_t* counts, int32_t* kept,
                 int32_t* offsets, int32_t* row_src, int32_t* slot_row) {
    int e, t, j, overflow = 0;
    int64_t r;
    int32_t* rank = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (e = 0; e < E; ++e) counts[e] = 0;
    for (t = 0; t < T; ++t)
        for (j = 0; j < k; ++j) counts[topk_idx[(int64_t)t * k + j]] += 1;
    for (e = 0; e < E; ++e) {
        int64_t kk = counts[e];
        if (cap >= 0 && kk > cap) kk = cap;
        if (layout == 1 && kk > masked_max_m) { kk = masked_max_m; overflow = 1; }
        kept[e] = (int32_t)kk;
    }
    offsets[0] = 0;
    for (e = 0; e < E; ++e) {
        if (layout == 0) offsets[e + 1] = offsets[e] + (kept[e] + pad - 1) / pad * pad;
        else offsets[e + 1] = (e + 1) * masked_max_m;
    }
    for (r = 0; r < rows_cap; ++r) row_src[r] = -1;
    /* token order: the i-th slot of expert e (by token index) gets rank i */
    for (t = 0; t < T; ++t) {
        for (j = 0; j < k; ++j) {
            int64_t s = (int64_t)t * k + j;
            int ee = topk_idx[s];
            int rk = rank[ee]++;
            if (rk < kept[ee]) {
                int64_t row = (int64_t)offsets[ee] + rk;
                slot_row[s] = (int32_t)row;
                row_src[row] = (int32_t)s;
            } else {
                slot_row[s] = -1;
            }
        }
    }
    free(rank);
    return overflow;
}

/* ------------------------------------------------------------------ */
/* Activation quantisation ([P1] 3.3; fine-grained 1x128 groups)         */
/* ------------------------------------------------------------------ */
void orc_quant_rows(int64_t rows, int K, const float* v, uint8_t* q, float* s) {
    int64_t r;
    int g, i, G = K / GROUP;
    for (r = 0; r < rows; ++r) {
        for (g = 0; g < G; ++g) {
            const float* vv = v + r * K + (int64_t)g * GROUP;
            uint8_t* qq = q + r * K + (int64_t)g * GROUP;
            float amax = 0.0f, sc;
            for (i = 0; i < GROUP; ++i) if (fabsf(vv[i]) > amax) amax = fabsf(vv[i]);
            if (amax == 0.0f) {
                sc = 1.0f;
                for (i = 0; i < GROUP; ++i) qq[i] = orc_e4m3_encode(vv[i]);  /* signed zeros */
            } else {
                sc = amax / 448.0f;                       /* fp32, correctly rounded */
                for (i = 0; i < GROUP; ++i) qq[i] = orc_e4m3_encode(vv[i] / sc);
            }
            s[r * G + g] = sc;
        }
    }
}

/* One quantisation group of n values with one scale (the same rule as a
 * 1x128 group: scale = max|v| / 448 in fp32, 1 for an all-zero group; code =
 * E4M3 of v / scale). Used for the 128x128 blocks of the weight-gradient
 * operands of the backward pass. */
void orc_quant_group(int64_t n, const float* v, uint8_t* q, float* s) {
    int64_t i;
    float amax = 0.0f, sc;
    for (i = 0; i < n; ++i) if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
    if (amax == 0.0f) {
        sc = 1.0f;
        for (i = 0; i < n; ++i) q[i] = orc_e4m3_encode(v[i]);
    } else {
        sc = amax / 448.0f;
        for (i = 0; i < n; ++i) q[i] = orc_e4m3_encode(v[i] / sc);
    }
    *s = sc;
}

/* ------------------------------------------------------------------ */
/* Expert math (SwiGLU FFN E_i(x) = W2 (silu(W1 x) * W3 x))              */
/* ------------------------------------------------------------------ */
/* Dequantised value: the E4M3 value times its block scale, rounded to fp32. */
static float deq(uint8_t code, float scale) {
    float v = (float)orc_e4m3_decode(code);
    return v * scale;
}

/* One output of a K-major FP8 GEMM row: sum_k deq(a[k]) * deq(w[k]) in fp64.
 * a_s holds the row's K/128 scales; w_s the weight row's K/128 block scales. */
static double dot_row(int K, const uint8_t* a, const float* a_s, const uint8_t* w, const float* w_s) {
    double acc = 0.0;
    int kk;
    for (kk = 0; kk < K; ++kk)
        acc += (double)deq(a[kk], a_s[kk / GROUP]) * (double)deq(w[kk], w_s[kk / GROUP]);
    return acc;
}

/* 4-bit weight codes ([P3] 3.1): the integer levels -7..7 of a block scaled by
 * its max-abs, round((w / max|w|) * (2^3 - 1)), stored as a sign and a 3-bit
 * magnitude. A row holds K/8 little-endian 32-bit words, each with the levels
 * of eight consecutive k (k = 8 q + i): the magnitude of level i (i = 0..3) in
 * bits 4i..4i+2 and its sign in bit 8i+7; the magnitude of level 4+i in bits
 * 16+4i..16+4i+2 and its sign in bit 8i+3. Returns the level of element k. */
int orc_w4_decode(const uint8_t* row, int k) {
    const uint8_t* b = row + 4 * (k / 8);
    const uint32_t w = (uint32_t)b[0] | ((uint32_t)b[1] << 8) | ((uint32_t)b[2] << 16) | ((uint32_t)b[3] << 24);
    const int i = k % 8;
    int mag, neg;
    if (i < 4) {
        mag = (int)((w >> (4 * i)) & 7u);
        neg = (int)((w >> (8 * i + 7)) & 1u);
    } else {
        mag = (int)((w >> (16 + 4 * (i - 4))) & 7u);
        neg = (int)((w >> (8 * (i - 4) + 3)) & 1u);
    }
    return neg ? -mag : mag;
}

/* As dot_row, with a row of 4-bit weight codes and the row's K/128 scales
 * (max-abs / 7 per block), w_s[kb * ws_stride]; the dequantised weight is
 * code * scale in fp32. */
static double dot_row_w4(int K, const uint8_t* a, const float* a_s, const uint8_t* w, const float* w_s,
                         int64_t ws_stride) {
    double acc = 0.0;
    int kk;
    for (kk = 0; kk < K; ++kk) {
        float wd = (float)orc_w4_decode(w, kk) * w_s[(int64_t)(kk / GROUP) * ws_stride];
        acc += (double)deq(a[kk], a_s[kk / GROUP]) * (double)wd;
    }
    return acc;
}

static double silu(double a) { return a / (1.0 + exp(-a)); }

typedef struct {
    int H, I;
    const uint8_t *xq; const float* xs;
    const uint8_t *W1q, *W3q, *W2q; const float *S1, *S3, *S2;
    uint8_t* hq; float* hs; uint16_t* o;
    float* h;          /* [n, I] fp32 h before its quantisation */
} expert_ctx;

/* Work items are (row, output column); the split is over items only, so
 * every output is the same sum in the same order whatever the thread count. */
static void expert_up_range(void* vctx, int64_t b, int64_t e) {
    expert_ctx* c = (expert_ctx*)vctx;
    int H = c->H, I = c->I;
    int64_t it;
    for (it = b; it < e; ++it) {
        int64_t r = it / I;
        int n = (int)(it % I);
        const uint8_t* xr = c->xq + r * H;
        const float* xsr = c->xs + r * (H / GROUP);
        double a = dot_row(H, xr, xsr, c->W1q + (int64_t)n * H, c->S1 + (int64_t)(n / GROUP) * (H / GROUP));
        double bb = dot_row(H, xr, xsr, c->W3q + (int64_t)n * H, c->S3 + (int64_t)(n / GROUP) * (H / GROUP));
        c->h[r * I + n] = (float)(silu(a) * bb);
    }
}

static void expert_down_range(void* vctx, int64_t b, int64_t e) {
    expert_ctx* c = (expert_ctx*)vctx;
    int H = c->H, I = c->I;
    int64_t it;
    for (it = b; it < e; ++it) {
        int64_t r = it / H;
        int n = (int)(it % H);
        double o = dot_row(I, c->hq + r * I, c->hs + r * (I / GROUP),
                           c->W2q + (int64_t)n * I, c->S2 + (int64_t)(n / GROUP) * (I / GROUP));
        c->o[r * H + n] = orc_f64_to_bf16(o);
    }
}

void orc_expert_rows(int n, int H, int I, const uint8_t* xq, const float* xs,
                     const uint8_t* W1q, const float* S1, const uint8_t* W3q, const float* S3,
                     const uint8_t* W2q, const float* S2,
                     uint8_t* hq, float* hs, uint16_t* o, int nthreads) {
    expert_ctx c = {H, I, xq, xs, W1q, W3q, W2q, S1, S3, S2, hq, hs, o, NULL};
    c.h = (float*)malloc(sizeof(float) * (size_t)n * (size_t)I);
    parallel_for((int64_t)n * I, nthreads, expert_up_range, &c);     /* a, b, h = silu(a) * b */
    orc_quant_rows(n, I, c.h, hq, hs);                                /* h -> E4M3 + 1x128 scales */
    parallel_for((int64_t)n * H, nthreads, expert_down_range, &c);    /* o = W2 h, -> bf16 */
    free(c.h);
}

/* ------------------------------------------------------------------ */
/* Grouped GEMM with the boundary's semantics ([P1] 2.1, 3.2: each group */
/* its own M, shared N and K; "nt" operands, bf16 output)                */
/* ------------------------------------------------------------------ */
typedef struct {
    int layout, E, N, K, M_rows, epilogue;
    int w4;            /* 0: E4M3 weights, 128x128 block scales; 1: 4-bit weights, 1x128 row scales */
    const uint8_t* A; const float* As; const int32_t* gi;
    const uint8_t* B; const float* Bs;
    void* D; float* Ds;
    int64_t nrows;
} gg_ctx;

/* expert of a row, or -1 if the row lies in no group */
static int gg_row_expert(const gg_ctx* c, int64_t row) {
    int e;
    if (c->layout == 0) {
        for (e = 0; e < c->E; ++e) if (row >= c->gi[e] && row < c->gi[e + 1]) return e;
        return -1;
    }
    e = (int)(row / c->M_rows);
    return (row % c->M_rows) < c->gi[e] ? e : -1;
}

/* Output column n of expert e for one activation row: E4M3 weights are [E, N, K]
 * with scales [E, N/128, K/128]; 4-bit weights are [E, N, K/2] with scales
 * [E, K/128, N] (K-block-major: the scales of one K block for consecutive rows
 * lie together). */
static double gg_dot(const gg_ctx* c, const uint8_t* ar, const float* a_s, int e, int64_t n) {
    const int K = c->K, KB = K / GROUP;
    const int64_t row = (int64_t)e * c->N + n;
    if (!c->w4)
        return dot_row(K, ar, a_s, c->B + row * K, c->Bs + ((int64_t)e * (c->N / GROUP) + n / GROUP) * KB);
    return dot_row_w4(K, ar, a_s, c->B + row * (K / 2), c->Bs + (int64_t)e * KB * c->N + n, c->N);
}

static void gg_range(void* vctx, int64_t b, int64_t end) {
    gg_ctx* c = (gg_ctx*)vctx;
    int K = c->K, N = c->N, KB = K / GROUP, n, kb;
    float* a_s = (float*)malloc(sizeof(float) * (size_t)KB);
    float* h = (float*)malloc(sizeof(float) * (size_t)(N / 2 + 1));
    int64_t row;
    for (row = b; row < end; ++row) {
        int e = gg_row_expert(c, row);
        const uint8_t* ar;
        const float* As_base;
        int64_t srow;
        if (e < 0) continue;
        ar = c->A + row * K;
        srow = (c->layout == 0) ? row : row % c->M_rows;              /* scale column */
        As_base = (c->layout == 0) ? c->As : c->As + (int64_t)e * KB * c->M_rows;
        for (kb = 0; kb < KB; ++kb) a_s[kb] = As_base[(int64_t)kb * c->M_rows + srow];
        if (c->epilogue == 0) {
            uint16_t* D = (uint16_t*)c->D;
            for (n = 0; n < N; ++n)
                D[row * N + n] = orc_f64_to_bf16(gg_dot(c, ar, a_s, e, n));
        } else {
            int I = N / 2, G = I / GROUP, g;
            uint8_t* Dq = (uint8_t*)c->D;
            float hsr[64];
            float* Ds_base = (c->layout == 0) ? c->Ds : c->Ds + (int64_t)e * G * c->M_rows;
            for (n = 0; n < I; ++n) {
                int blk = n / GROUP, w = n % GROUP;
                int64_t r1 = (int64_t)(2 * blk) * GROUP + w;       /* gate row (W1) */
                int64_t r3 = (int64_t)(2 * blk + 1) * GROUP + w;   /* up row (W3) */
                double a = gg_dot(c, ar, a_s, e, r1);
                double bb = gg_dot(c, ar, a_s, e, r3);
                h[n] = (float)(silu(a) * bb);
            }
            for (g = 0; g < G; g += 64) {
                int gn = (G - g) < 64 ? (G - g) : 64, q;
                orc_quant_rows(1, gn * GROUP, h + (int64_t)g * GROUP, Dq + row * I + (int64_t)g * GROUP, hsr);
                for (q = 0; q < gn; ++q) Ds_base[(int64_t)(g + q) * c->M_rows + srow] = hsr[q];
            }
        }
    }
    free(a_s);
    free(h);
}

static void grouped_gemm(int w4, int layout, int E, int N, int K, const uint8_t* A, const float* As,
                         const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                         int epilogue, void* D, float* Ds, int nthreads) {
    gg_ctx c;
    c.layout = layout; c.E = E; c.N = N; c.K = K; c.M_rows = M_rows; c.epilogue = epilogue; c.w4 = w4;
    c.A = A; c.As = As; c.gi = group_info; c.B = B; c.Bs = Bs; c.D = D; c.Ds = Ds;
    c.nrows = (layout == 0) ? group_info[E] : (int64_t)E * M_rows;
    parallel_for(c.nrows, nthreads, gg_range, &c);
}

void orc_grouped_gemm(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                      const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                      int epilogue, void* D, float* Ds, int nthreads) {
    grouped_gemm(0, layout, E, N, K, A, As, group_info, M_rows, B, Bs, epilogue, D, Ds, nthreads);
}

void orc_grouped_gemm_w4(int layout, int E, int N, int K, const uint8_t* A, const float* As,
                         const int32_t* group_info, int M_rows, const uint8_t* B, const float* Bs,
                         int epilogue, void* D, float* Ds, int nthreads) {
    grouped_gemm(1, layout, E, N, K, A, As, group_info, M_rows, B, Bs, epilogue, D, Ds, nthreads);
}

/* ------------------------------------------------------------------ */
/* Combine ([P1] 2.1: y = sum_{i in TopK} G(x)_i * E_i(x))               */
/* ------------------------------------------------------------------ */
void orc_combine(int T, int k, int H, const int32_t* slot_row, const float* topk_w,
                 const uint16_t* O, uint16_t* y) {
    int t, j, n;
    double* acc = (double*)malloc(sizeof(double) * (size_t)H);
    for (t = 0; t < T; ++t) {
        for (n = 0; n < H; ++n) acc[n] = 0.0;
        for (j = 0; j < k; ++j) {
            int64_t row = slot_row[(int64_t)t * k + j];
            double w = (double)topk_w[(int64_t)t * k + j];
            if (row < 0) continue;                 /* dropped slot: no contribution */
            for (n = 0; n < H; ++n) acc[n] += w * (double)orc_bf16_to_f32(O[row * H + n]);
        }
        for (n = 0; n < H; ++n) y[(int64_t)t * H + n] = orc_f64_to_bf16(acc[n]);
    }
    free(acc);
}

/* Auxiliary-loss-free load balancing ([P1] 2.2): every expert keeps a routing
 * bias; the load each expert received is tallied over the update interval and,
 * when the interval ends, an expert that received more than the mean has its
 * bias lowered by the step gamma, one that received less has it raised, and
 * one exactly at the mean keeps it. The mean is compared exactly, in integers:
 * E * load[e] against the total. The bias is stored in fp32, so the step is
 * one fp32 addition or subtraction. The tally restarts after an update. */
void orc_balance_bias(int E, const int32_t* counts, int64_t* load, float* bias, float gamma, int update) {
    int e;
    int64_t total = 0;
    for (e = 0; e < E; ++e) load[e] += counts[e];
    if (!update) return;
    for (e = 0; e < E; ++e) total += load[e];
    for (e = 0; e < E; ++e) {
        const int64_t scaled = (int64_t)E * load[e];
        if (scaled > total) bias[e] = bias[e] - gamma;        /* overloaded: lower */
        else if (scaled < total) bias[e] = bias[e] + gamma;   /* underloaded: raise */
        load[e] = 0;
    }
}
