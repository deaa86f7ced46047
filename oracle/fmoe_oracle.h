/*
 * fmoe_oracle.h — plain, slow CPU oracle of the batch-1 MoE layer with group-affine
 * dequantising expert GEMVs. TEST INFRASTRUCTURE ONLY: it is linked by the tests, by
 * __graft_entry__.smoke() and by the CPU-baseline leg of bench.py, never by the product
 * library. It shares no code, header, table or helper with the CUDA path; it decodes the
 * packed bytes with its own decoder written from the layout text (codes row-major, n =
 * 32/bits codes per little-endian uint32 word, lowest column in the lowest bits; then one
 * uint32 per 64-column group: bf16 scale in bits 0..15, bf16 bias in bits 16..31).
 *
 * Arithmetic: binary64 everywhere except the quantiser, which is defined in binary32 so that
 * a GPU packer can reproduce it bit for bit. Sums are naive left-to-right loops.
 *
 * Pages followed (cited by title and section):
 *   [FR-A] "Qu'est-ce que Flash-MoE ? ..." (a2a-mcp.org/blog/what-is-flash-moe-fr)
 *   [SK]   "Flash-MoE: Ako spustiť 397-miliardový AI model na bežnom notebooku"
 *   [JA-O] "Flash-MoE：純粋なC/MetalでMacBook Pro上で397BパラメータのQwenモデルを実行"
 *   [JA-A] "Flash-MoEとは何か？..." (a2a-mcp.org/blog/what-is-flash-moe-ja)
 */
#ifndef FMOE_ORACLE_H
#define FMOE_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16: round binary32 to nearest-even bf16 (NaN kept quiet), and widen back. */
uint16_t orc_bf16_rne(float f);
float orc_bf16_to_f32(uint16_t h);

/* Byte size of a packed matrix: codes R*C*bits/8 plus one uint32 per 64-column group. */
size_t orc_qmat_bytes(int rows, int cols, int bits);
size_t orc_expert_bytes(int hidden, int inter, int bits);

/* Quantiser (binary32 arithmetic, IEEE rounding):
 *   mn, mx = group min/max; s = bf16(fl((mx - mn) / (2^bits - 1))); z = bf16(mn);
 *   q = s == 0 ? 0 : clamp(rint(fl(fl(w - z) / s)), 0, 2^bits - 1)  (rint ties to even). */
void orc_quantise(const float* w, int rows, int cols, int bits, uint8_t* dst);

/* Decoder. */
int orc_code(const uint8_t* qm, int rows, int cols, int bits, int r, int c);
void orc_scale_bias(const uint8_t* qm, int rows, int cols, int bits, int r, int g, double* s,
                    double* z);
/* w_hat = q*s + z ([FR-A] §2 "Noyaux de Déquantification Optimisés pour FMA", the form
 * before the rewrite). */
double orc_weight(const uint8_t* qm, int rows, int cols, int bits, int r, int c);
void orc_dequant(const uint8_t* qm, int rows, int cols, int bits, double* out /* R*C */);

/* y_r = sum_c (q_rc*s + z) * x_c, the naive (pre-FMA) form, fp64, left to right. */
void orc_gemv(const uint8_t* qm, int rows, int cols, int bits, const double* x, double* y);

/* Dot of n codes of one group with x in one of the four algebraically equal forms:
 *   0: sum (q*s + z) * x                      (naive, [FR-A] §2 "Avant")
 *   1: sum fma(q, s*x, z*x)                   ([FR-A] §2 "Après"; [JA-O] "FMA最適化デカントカーネル")
 *   2: sum fma(q*x, s, z*x)                   ([SK] "FMA-optimalizovaný dequantizačný kernel")
 *   3: s * sum(q*x) + z * sum(x)              (group-factored: the same sum, distributed) */
double orc_group_dot(int form, const int* q, double s, double z, const double* x, int n);

/* One expert: h = SiLU(gate x) * (up x);  y = down h.  SiLU(a) = a / (1 + exp(-a)).
 * blob: gate qmat (I x H) | up qmat (I x H) | down qmat (H x I). h_out nullable [I]. */
void orc_expert(const uint8_t* blob, int H, int I, int bits, const double* x, double* y,
                double* h_out);

/* Router ([JA-O] "パイプラインパフォーマンス": routing GEMV, then softmax + topK):
 *   logit_e = sum_i R[e,i] x_i (+ bias_e);  p = softmax(logit) over all E (max-subtracted);
 *   top-K by p, ties to the lower index;  w_k = p_k / sum_sel p.
 * idx/w in selection order. logits_out, p_out nullable [E]. */
void orc_route(const double* x, const float* router, const float* bias, int H, int E, int K,
               int* idx, double* w, double* logits_out, double* p_out);

typedef struct orc_layer {
    int H, I, E, K, bits;
    const uint8_t* const* experts; /* [E] blob pointers; only the selected ones are read   */
    const uint8_t* shared;         /* nullable                                              */
    const float* router;           /* [E x H]                                               */
    const float* shared_gate;      /* nullable [H]                                          */
} orc_layer;

/* out = res + sum_k w_k expert_{idx_k}(x) + sigmoid(g . x) * shared(x)   ([FR-A] §3, MoE
 * combine + residual + sigmoid gating). res nullable (0). Returns 0, or -1 if a selected
 * expert pointer is NULL. idx/w nullable outputs. */
int orc_layer_forward(const orc_layer* L, const double* x, const double* res, const float* bias,
                      double* out, int* idx, double* w);
/* Same combine with the routing decision given (used where two routings are both correct). */
int orc_layer_forced(const orc_layer* L, const double* x, const double* res, const int* idx,
                     const double* w, double* out);

/* x = h / sqrt(sum h^2 / H + eps)  ([FR-A] §3: RMSNorm, sum of squares then apply). */
void orc_rmsnorm(const double* h, int H, double eps, double* x);

/* One token through L layers: h_0 = h_in; x_0 = h_0; x_l = rmsnorm(h_l) for l >= 1;
 * h_{l+1} = layer_l(x_l, res = h_l). bias nullable [L x E]. idx_trace nullable [L x K],
 * x_trace nullable [L x H]. Returns 0 or -1 (missing expert blob). */
int orc_stack(const orc_layer* layers, int L, const double* h_in, const float* bias, double eps,
              double* h_out, int* idx_trace, double* x_trace);

/* Which planted mistake this build carries (0 = none); see the test of the pins. */
int orc_mutant(void);

#ifdef __cplusplus
}
#endif
#endif
