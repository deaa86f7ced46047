/*
 * fmoe_oracle.c — plain CPU oracle (test infrastructure only; see fmoe_oracle.h).
 *
 * Written for a reader who checks it against the pages by eye: one loop per definition, no
 * blocking, no fusion, no reordering. Build: gcc -O2 -ffp-contract=off -fPIC -shared.
 * -ffp-contract=off keeps every binary32 operation of the quantiser separately rounded.
 *
 * ORC_MUTANT (compile-time, default 0) plants one known mistake; the test suite compiles
 * each mutant and checks that at least one pin catches it. It is never set in normal builds.
 */
#include "fmoe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif

int orc_mutant(void) { return ORC_MUTANT; }

/* ---------------------------------------------------------------- bf16 (own bit arithmetic) */
uint16_t orc_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u); /* NaN: keep it a (quiet) NaN */
    uint32_t lsb = (u >> 16) & 1u;               /* round to nearest, ties to even */
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ---------------------------------------------------------------- sizes */
/* Any positive row count; columns in whole groups of 64. */
static int legal(int rows, int cols, int bits) {
    return rows > 0 && cols > 0 && cols % 64 == 0 && (bits == 2 || bits == 4);
}

size_t orc_qmat_bytes(int rows, int cols, int bits) {
    if (!legal(rows, cols, bits)) return 0;
    size_t n = (size_t)rows * (size_t)cols;
    return n * (size_t)bits / 8 + (n / 64) * 4;
}

size_t orc_expert_bytes(int hidden, int inter, int bits) {
    return 2 * orc_qmat_bytes(inter, hidden, bits) + orc_qmat_bytes(hidden, inter, bits);
}

/* ---------------------------------------------------------------- quantiser (binary32) */
static float rint_half_even(float v) {
#if ORC_MUTANT == 11
    return floorf(v + 0.5f); /* planted: ties away from even */
#else
    return rintf(v); /* default rounding mode: to nearest, ties to even */
#endif
}

void orc_quantise(const float* w, int rows, int cols, int bits, uint8_t* dst) {
    const int per_word = 32 / bits;
    const int qmax = (1 << bits) - 1;
    const size_t code_bytes = (size_t)rows * cols * bits / 8;
    const int groups = cols / 64;
    uint32_t* words = (uint32_t*)dst;
    uint32_t* sb = (uint32_t*)(dst + code_bytes);
    memset(dst, 0, code_bytes);
    for (int r = 0; r < rows; ++r) {
        for (int g = 0; g < groups; ++g) {
            const float* v = w + (size_t)r * cols + (size_t)g * 64;
            float mn = v[0], mx = v[0];
            for (int i = 1; i < 64; ++i) {
                if (v[i] < mn) mn = v[i];
                if (v[i] > mx) mx = v[i];
            }
            float range = mx - mn;
            float step = range / (float)qmax;
            uint16_t s16 = orc_bf16_rne(step);
            uint16_t z16 = orc_bf16_rne(mn);
            float s = orc_bf16_to_f32(s16);
            float z = orc_bf16_to_f32(z16);
            sb[(size_t)r * groups + g] = (uint32_t)s16 | ((uint32_t)z16 << 16);
            for (int i = 0; i < 64; ++i) {
                int q = 0;
                if (s != 0.0f) {
                    float d = v[i] - z;
                    float t = d / s;
                    float rq = rint_half_even(t);
                    if (rq < 0.0f) rq = 0.0f;
                    if (rq > (float)qmax) rq = (float)qmax;
                    q = (int)rq;
                }
                int c = g * 64 + i;
                size_t word = (size_t)r * (cols / per_word) + (size_t)(c / per_word);
                int pos = (c % per_word) * bits;
                words[word] |= (uint32_t)q << pos;
            }
        }
    }
}

/* ---------------------------------------------------------------- decoder */
int orc_code(const uint8_t* qm, int rows, int cols, int bits, int r, int c) {
    (void)rows;
    const int per_word = 32 / bits;
    const uint32_t* words = (const uint32_t*)qm;
    uint32_t word = words[(size_t)r * (cols / per_word) + (size_t)(c / per_word)];
#if ORC_MUTANT == 1
    int pos = (per_word - 1 - c % per_word) * bits; /* planted: highest column in lowest bits */
#else
    int pos = (c % per_word) * bits;
#endif
    return (int)((word >> pos) & ((1u << bits) - 1u));
}

void orc_scale_bias(const uint8_t* qm, int rows, int cols, int bits, int r, int g, double* s,
                    double* z) {
    const size_t code_bytes = (size_t)rows * cols * bits / 8;
    const uint32_t* sb = (const uint32_t*)(qm + code_bytes);
    const int groups = cols / 64;
#if ORC_MUTANT == 4
    g = (g + 1) % groups; /* planted: neighbouring group's scale and bias */
#endif
    uint32_t word = sb[(size_t)r * groups + g];
#if ORC_MUTANT == 3
    *s = (double)orc_bf16_to_f32((uint16_t)(word >> 16)); /* planted: halves swapped */
    *z = (double)orc_bf16_to_f32((uint16_t)(word & 0xffffu));
#else
    *s = (double)orc_bf16_to_f32((uint16_t)(word & 0xffffu));
    *z = (double)orc_bf16_to_f32((uint16_t)(word >> 16));
#endif
}

double orc_weight(const uint8_t* qm, int rows, int cols, int bits, int r, int c) {
    double s, z;
    orc_scale_bias(qm, rows, cols, bits, r, c / 64, &s, &z);
    int q = orc_code(qm, rows, cols, bits, r, c);
#if ORC_MUTANT == 2
    return (double)q * s; /* planted: bias dropped */
#else
    return (double)q * s + z;
#endif
}

void orc_dequant(const uint8_t* qm, int rows, int cols, int bits, double* out) {
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c) out[(size_t)r * cols + c] = orc_weight(qm, rows, cols, bits, r, c);
}

void orc_gemv(const uint8_t* qm, int rows, int cols, int bits, const double* x, double* y) {
    for (int r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int c = 0; c < cols; ++c) acc += orc_weight(qm, rows, cols, bits, r, c) * x[c];
        y[r] = acc;
    }
}

double orc_group_dot(int form, const int* q, double s, double z, const double* x, int n) {
    double acc = 0.0;
    if (form == 0) {
        for (int i = 0; i < n; ++i) acc += ((double)q[i] * s + z) * x[i];
    } else if (form == 1) {
        for (int i = 0; i < n; ++i) acc += fma((double)q[i], s * x[i], z * x[i]);
    } else if (form == 2) {
        for (int i = 0; i < n; ++i) acc += fma((double)q[i] * x[i], s, z * x[i]);
    } else {
        double qx = 0.0, sx = 0.0;
        for (int i = 0; i < n; ++i) {
            qx += (double)q[i] * x[i];
            sx += x[i];
        }
        acc = s * qx + z * sx;
    }
    return acc;
}

/* ---------------------------------------------------------------- expert */
static double silu(double a) {
#if ORC_MUTANT == 5
    return a / (1.0 + exp(a)); /* planted: sign error */
#else
    return a / (1.0 + exp(-a));
#endif
}

void orc_expert(const uint8_t* blob, int H, int I, int bits, const double* x, double* y,
                double* h_out) {
    const uint8_t* gate = blob;
    const uint8_t* up = blob + orc_qmat_bytes(I, H, bits);
#if ORC_MUTANT == 13
    const uint8_t* down = up; /* planted: reads the up matrix (same byte size) as down */
#else
    const uint8_t* down = blob + 2 * orc_qmat_bytes(I, H, bits);
#endif
    double* a = (double*)malloc(sizeof(double) * I);
    double* u = (double*)malloc(sizeof(double) * I);
    double* h = (double*)malloc(sizeof(double) * I);
    orc_gemv(gate, I, H, bits, x, a);
    orc_gemv(up, I, H, bits, x, u);
    for (int r = 0; r < I; ++r) h[r] = silu(a[r]) * u[r];
    orc_gemv(down, H, I, bits, h, y);
    if (h_out) memcpy(h_out, h, sizeof(double) * I);
    free(a);
    free(u);
    free(h);
}

/* ---------------------------------------------------------------- router */
void orc_route(const double* x, const float* router, const float* bias, int H, int E, int K,
               int* idx, double* w, double* logits_out, double* p_out) {
    double* logit = (double*)malloc(sizeof(double) * E);
    double* p = (double*)malloc(sizeof(double) * E);
    char* taken = (char*)calloc((size_t)E, 1);
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int i = 0; i < H; ++i) acc += (double)router[(size_t)e * H + i] * x[i];
        if (bias) acc += (double)bias[e];
        logit[e] = acc;
    }
    /* softmax over all experts */
    double mx = logit[0];
    for (int e = 1; e < E; ++e)
        if (logit[e] > mx) mx = logit[e];
    double den = 0.0;
    for (int e = 0; e < E; ++e) {
        p[e] = exp(logit[e] - mx);
        den += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= den;
    /* top-K by probability, ties to the lower index */
    double sel = 0.0;
    for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
#if ORC_MUTANT == 8
            if (best < 0 || p[e] >= p[best]) best = e; /* planted: ties to the higher index */
#else
            if (best < 0 || p[e] > p[best]) best = e;
#endif
        }
        taken[best] = 1;
        idx[k] = best;
        sel += p[best];
    }
    for (int k = 0; k < K; ++k) {
#if ORC_MUTANT == 9
        w[k] = p[idx[k]]; /* planted: no renormalisation */
#else
        w[k] = p[idx[k]] / sel;
#endif
    }
    if (logits_out) memcpy(logits_out, logit, sizeof(double) * E);
    if (p_out) memcpy(p_out, p, sizeof(double) * E);
    free(logit);
    free(p);
    free(taken);
}

/* ---------------------------------------------------------------- layer */
static double sigmoid(double a) { return 1.0 / (1.0 + exp(-a)); }

int orc_layer_forced(const orc_layer* L, const double* x, const double* res, const int* idx,
                     const double* w, double* out) {
    const int H = L->H;
    double* y = (double*)malloc(sizeof(double) * H);
    for (int j = 0; j < H; ++j) {
#if ORC_MUTANT == 6
        out[j] = 0.0; /* planted: residual dropped */
#else
        out[j] = res ? res[j] : 0.0;
#endif
    }
    for (int k = 0; k < L->K; ++k) {
        const uint8_t* blob = L->experts[idx[k]];
        if (!blob) {
            free(y);
            return -1;
        }
        orc_expert(blob, H, L->I, L->bits, x, y, NULL);
        for (int j = 0; j < H; ++j) out[j] += w[k] * y[j];
    }
    if (L->shared) {
        double gate = 1.0;
        if (L->shared_gate) {
            double gx = 0.0;
            for (int i = 0; i < H; ++i) gx += (double)L->shared_gate[i] * x[i];
#if ORC_MUTANT == 7
            gate = gx; /* planted: sigmoid dropped */
#else
            gate = sigmoid(gx);
#endif
        }
        orc_expert(L->shared, H, L->I, L->bits, x, y, NULL);
        for (int j = 0; j < H; ++j) out[j] += gate * y[j];
    }
    free(y);
    return 0;
}

int orc_layer_forward(const orc_layer* L, const double* x, const double* res, const float* bias,
                      double* out, int* idx, double* w) {
    int* ix = (int*)malloc(sizeof(int) * L->K);
    double* wk = (double*)malloc(sizeof(double) * L->K);
    orc_route(x, L->router, bias, L->H, L->E, L->K, ix, wk, NULL, NULL);
    int rc = orc_layer_forced(L, x, res, ix, wk, out);
    if (idx) memcpy(idx, ix, sizeof(int) * L->K);
    if (w) memcpy(w, wk, sizeof(double) * L->K);
    free(ix);
    free(wk);
    return rc;
}

/* ---------------------------------------------------------------- norm and stack */
void orc_rmsnorm(const double* h, int H, double eps, double* x) {
    double ss = 0.0;
    for (int i = 0; i < H; ++i) ss += h[i] * h[i];
#if ORC_MUTANT == 10
    double r = 1.0 / sqrt(ss / H); /* planted: eps dropped */
#else
    double r = 1.0 / sqrt(ss / H + eps);
#endif
    for (int i = 0; i < H; ++i) x[i] = h[i] * r;
}

int orc_stack(const orc_layer* layers, int L, const double* h_in, const float* bias, double eps,
              double* h_out, int* idx_trace, double* x_trace) {
    const int H = layers[0].H;
    double* h = (double*)malloc(sizeof(double) * H);
    double* x = (double*)malloc(sizeof(double) * H);
    double* o = (double*)malloc(sizeof(double) * H);
    memcpy(h, h_in, sizeof(double) * H);
    int rc = 0;
    for (int l = 0; l < L && rc == 0; ++l) {
        const orc_layer* ly = &layers[l];
#if ORC_MUTANT == 14
        orc_rmsnorm(h, H, eps, x); /* planted: layer 0 normalised too */
#else
        if (l == 0)
            memcpy(x, h, sizeof(double) * H);
        else
            orc_rmsnorm(h, H, eps, x);
#endif
        if (x_trace) memcpy(x_trace + (size_t)l * H, x, sizeof(double) * H);
        int* ix = idx_trace ? idx_trace + (size_t)l * ly->K : NULL;
        rc = orc_layer_forward(ly, x, h, bias ? bias + (size_t)l * ly->E : NULL, o, ix, NULL);
        memcpy(h, o, sizeof(double) * H);
    }
    memcpy(h_out, h, sizeof(double) * H);
    free(h);
    free(x);
    free(o);
    return rc;
}
