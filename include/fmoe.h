/*
 * fmoe.h — C ABI of the batch-1 Mixture-of-Experts layer forward with 4-bit / 2-bit
 * group-affine dequantising expert GEMVs (B200, sm_100a).
 *
 * Sources. The operation is the per-token MoE layer of the Flash-MoE engine as described on
 * five web pages (no code or equations are published there):
 *   [FR-A] "Qu'est-ce que Flash-MoE ? Exécuter des modèles d'IA de 397B paramètres sur un
 *          ordinateur portable" (a2a-mcp.org/blog/what-is-flash-moe-fr)
 *   [FR-D] "L'IA Massive Devient Accessible aux Développeurs" (deepthix.com)
 *   [SK]   "Flash-MoE: Ako spustiť 397-miliardový AI model na bežnom notebooku"
 *          (education.sardonicrepulsion.com)
 *   [JA-O] "Flash-MoE：純粋なC/MetalでMacBook Pro上で397BパラメータのQwenモデルを実行"
 *          (openclawradar.com)
 *   [JA-A] "Flash-MoEとは何か？ラップトップで397BパラメーターのAIモデルを実行する技術"
 *          (a2a-mcp.org/blog/what-is-flash-moe-ja)
 * Where a page leaves a step open, the reading taken is stated beside the declaration.
 *
 * Conventions for every entry point
 *   - Every pointer argument is DEVICE memory owned by the caller unless stated otherwise
 *     ("host" in the comment). The library never frees caller memory.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream). A status of FMOE_OK means the work was enqueued.
 *   - Arguments are validated on the host BEFORE anything is enqueued; on a validation
 *     failure nothing is launched and a negative status is returned. The message for the
 *     last failure on the calling host thread is in fmoe_last_error().
 *   - Errors raised inside a kernel (a bounded wait that ran out) are sticky per device and
 *     are read with fmoe_sync_status().
 *   - The layer entry points run one persistent kernel with one CTA per SM whose CTAs wait
 *     on each other; it is launched cooperatively, so a launch whose CTAs cannot all be
 *     resident at once (another kernel holding SMs, MPS limits) fails at launch with
 *     FMOE_ERR_CUDA instead of waiting out its budget.
 *   - Device pointers to packed weights, activations and outputs must be 16-byte aligned
 *     (FMOE_ERR_ALIGN otherwise).
 *   - Shapes: hidden H and intermediate I are multiples of 64 with 64 <= H,I <= 8192;
 *     bits is 4 or 2; 1 <= top_k <= min(n_experts, 8); 1 <= n_experts <= 4096;
 *     top_k * I <= 8192. Larger shapes return FMOE_ERR_UNSUPPORTED.
 *
 * Packed matrix layout ("qmat"), shared by the pack kernels, the GEMV kernels and the oracle.
 *   A weight matrix W has R rows (outputs) and C columns (inputs); y = W x. Groups of G = 64
 *   consecutive columns of one row share one scale s and one bias z (both bf16), and every
 *   weight is stored as an unsigned code q of `bits` bits:  w_hat = q * s + z.
 *   [FR-A] §2 "Noyaux de Déquantification Optimisés pour FMA"; [SK] "Kvantizácia" table;
 *   [JA-O] "主要技術". The pages fix 4-bit and 2-bit codes and a scale and bias per group;
 *   the group size 64, bf16 scale/bias and the 6.75 MB expert size follow from
 *   "~6.75MB per expert" for 3 x 4096 x 1024 weights ([FR-A] §1, [JA-O] "SSDエキスパート
 *   ストリーミング"): 3*4096*1024*(4/8 + 4/64) B = 7,077,888 B = 6.75 MiB.
 *   Byte layout of one qmat (R, C, bits):
 *     codes: R * C * bits / 8 bytes, row-major; row r starts at byte r*C*bits/8.
 *            A row is a sequence of little-endian uint32 words. With n = 32/bits codes per
 *            word, word j of a row holds columns j*n .. j*n+n-1; column j*n+i occupies bits
 *            [i*bits, i*bits+bits-1] (lowest column in the lowest bits).
 *     sb:    R * (C/64) uint32 words, row-major, directly after the codes. Word r*(C/64)+g
 *            holds the scale of group g of row r in bits 0..15 and its bias in bits 16..31,
 *            both as bf16 (a bf16 is the upper 16 bits of an IEEE-754 binary32).
 *   fmoe_qmat_bytes(R, C, bits) = R*C*bits/8 + R*C/16.
 *   Every section size is a multiple of 256 bytes for legal shapes.
 *
 * Expert blob layout (one contiguous blob per expert, all experts resident in HBM):
 *   gate qmat (I x H) | up qmat (I x H) | down qmat (H x I)
 *   fmoe_expert_bytes(H, I, bits) = 2*fmoe_qmat_bytes(I, H, bits) + fmoe_qmat_bytes(H, I, bits).
 *   The routed experts of one layer are `n_experts` blobs at a constant `expert_stride`
 *   (>= fmoe_expert_bytes, multiple of 16) from `experts`.
 */
#ifndef FMOE_H
#define FMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every int-returning entry point. */
enum {
    FMOE_OK = 0,
    FMOE_ERR_INVALID = -1,     /* a shape, count or required pointer is invalid            */
    FMOE_ERR_ALIGN = -2,       /* a pointer or stride is not 16-byte aligned               */
    FMOE_ERR_CUDA = -3,        /* a CUDA runtime call failed; text in fmoe_last_error()    */
    FMOE_ERR_NOMEM = -4,       /* device memory for library scratch could not be obtained  */
    FMOE_ERR_TIMEOUT = -5,     /* a bounded device-side wait ran out (see fmoe_sync_status) */
    FMOE_ERR_UNSUPPORTED = -6  /* legal shape beyond the limits stated above               */
};

/* Message describing the last failure on the calling host thread ("" if none).
 * The returned pointer stays valid until the next call on the same thread. */
const char* fmoe_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fmoe_version(void);

/* Waits for all work on `stream`, then returns and clears the sticky device-side status of
 * the current device: FMOE_OK, or FMOE_ERR_TIMEOUT if a kernel of this library gave up on a
 * bounded wait since the last call (its outputs are then undefined). FMOE_ERR_CUDA if the
 * synchronisation itself failed. */
int fmoe_sync_status(void* stream);

/* Sets the budget of every device-side bounded wait of kernels launched afterwards on the
 * calling host thread, in nanoseconds (default 1e9 = 1 s; values < 1000 are clamped). */
void fmoe_set_wait_budget_ns(uint64_t ns);

/* Test hook: bit 0 makes every kernel launched afterwards on the calling host thread compute
 * its router logits but never write them for the other CTAs, so every wait that depends on
 * them runs out of its budget and the launch ends with FMOE_ERR_TIMEOUT (a host-made failure
 * for testing the timeout path; nothing faults). 0 restores normal operation. */
void fmoe_set_fault_injection(int flags);

/* ---------------------------------------------------------------------------------------
 * Sizes (host only; no CUDA call). Return 0 for an illegal (rows, cols, bits).
 * --------------------------------------------------------------------------------------- */
size_t fmoe_qmat_bytes(int rows, int cols, int bits);
size_t fmoe_expert_bytes(int hidden, int inter, int bits);

/* ---------------------------------------------------------------------------------------
 * Pack (offline conversion; [FR-A] "Conclusion" mentions the weight-conversion scripts,
 * the pages do not state how scale and bias are formed). Reading taken: asymmetric
 * min/max affine per group, computed in binary32 with IEEE-correct rounding:
 *     mn, mx = min, max of the 64 weights of the group
 *     s = bf16_rne((mx - mn) / (2^bits - 1)),  z = bf16_rne(mn)
 *     q = (s == 0) ? 0 : clamp(rint((w - z) / s), 0, 2^bits - 1)   (rint: ties to even)
 *
 * w:   device, rows x cols binary32, row-major (row stride = cols).
 * dst: device, fmoe_qmat_bytes(rows, cols, bits) bytes, receives the qmat described above.
 * Returns FMOE_ERR_INVALID if rows or cols is not a positive multiple of 64 (rows up to
 * 1<<20, cols up to 1<<16) or bits is not 2 or 4; FMOE_ERR_ALIGN for unaligned pointers.
 * w and dst must not overlap.
 * --------------------------------------------------------------------------------------- */
int fmoe_pack(const float* w, int rows, int cols, int bits, void* dst, void* stream);
int fmoe_pack_q4(const float* w, int rows, int cols, void* dst, void* stream);
int fmoe_pack_q2(const float* w, int rows, int cols, void* dst, void* stream);

/* ---------------------------------------------------------------------------------------
 * Router: logits, softmax, top-K. The pages run "routing" on the GPU inside the second
 * command buffer and "softmax + topK" on the CPU ([JA-O] "パイプラインパフォーマンス").
 *   logit_e = sum_i router[e*hidden + i] * x[i]  (+ logit_bias[e] if non-NULL)
 *   p = softmax(logit) over all n_experts; select the top_k experts by p (ties to the lower
 *   expert index); weight_k = p_k / sum of the selected p.
 * Dot products are accumulated in binary64 on the GPU; weights are returned as binary32.
 * idx[k], weight[k] are written in decreasing logit order (k = 0 is the largest).
 *
 * x: [hidden] fp32. router: [n_experts x hidden] fp32 row-major. logit_bias: nullable
 * [n_experts] fp32 (added before the softmax; used to force routing in benchmarks).
 * idx: [top_k] int32 out. weight: [top_k] fp32 out.
 * --------------------------------------------------------------------------------------- */
int fmoe_route(const float* x, const float* router, const float* logit_bias, int hidden,
               int n_experts, int top_k, int32_t* idx, float* weight, void* stream);

/* ---------------------------------------------------------------------------------------
 * One expert: y = down( SiLU(gate x) * (up x) )  ([FR-A] §3 "Compute Shaders Metal Optimisés
 * à la Main": tiled 4-/2-bit dequant matvec and fused SwiGLU). SiLU(a) = a / (1 + exp(-a)).
 * expert: device blob in the expert layout above. x: [hidden] fp32. y: [hidden] fp32 out.
 * --------------------------------------------------------------------------------------- */
int fmoe_expert_gemv(const void* expert, int hidden, int inter, int bits, const float* x,
                     float* y, void* stream);

/* Description of one MoE layer. All pointers are device memory owned by the caller and
 * must stay valid while work that uses them is pending. */
typedef struct fmoe_layer_desc {
    int hidden;                 /* H                                                    */
    int inter;                  /* I (routed and shared experts)                        */
    int n_experts;              /* E routed experts                                     */
    int top_k;                  /* K                                                    */
    int bits;                   /* 4 or 2                                               */
    const void* experts;        /* E expert blobs                                       */
    size_t expert_stride;       /* bytes between consecutive expert blobs               */
    const void* shared_expert;  /* nullable: one more expert blob applied to every token */
    const float* router;        /* [E x H] fp32                                          */
    const float* shared_gate;   /* nullable [H] fp32: sigmoid gate of the shared expert  */
} fmoe_layer_desc;

/* ---------------------------------------------------------------------------------------
 * One MoE layer for one token ([FR-A] §3 and [JA-O] "Metalコンピュートシェーダー": MoE
 * combine + residual + sigmoid gate in one pass; [JA-O] "技術実装": K = 4 routed + 1 shared
 * out of 512 experts per layer):
 *   (idx, w) = route(x)
 *   out = residual + sum_k w_k * expert_{idx_k}(x) + sigmoid(shared_gate . x) * shared(x)
 * The shared term is dropped when shared_expert is NULL; sigmoid(..) is taken as 1 when
 * shared_gate is NULL. residual is nullable (treated as 0) and may alias out; x must not
 * alias out. idx_out [K] / w_out [K] are nullable outputs of the routing decision.
 * logit_bias: nullable [E].
 * --------------------------------------------------------------------------------------- */
int fmoe_moe_layer(const fmoe_layer_desc* layer, const float* x, const float* residual,
                   const float* logit_bias, float* out, int32_t* idx_out, float* w_out,
                   void* stream);

/* n_tokens independent decode tokens, strictly one after another in ONE launch: token t
 * goes through layers[t % n_layers] with input x[t*H..], residual[t*H..] (nullable),
 * logit_bias[t*E..] (nullable), and writes out[t*H..], idx_out[t*K..], w_out[t*K..]
 * (both nullable). Token t+1 starts computing only after token t's output is complete
 * (weights of token t+1 may be fetched earlier). All layers must share H, I, E, K, bits.
 * 1 <= n_layers <= 128. */
int fmoe_moe_layer_seq(const fmoe_layer_desc* layers, int n_layers, const float* x,
                       const float* residual, int n_tokens, const float* logit_bias,
                       float* out, int32_t* idx_out, float* w_out, void* stream);

/* Same as fmoe_moe_layer_seq with the token data in HOST memory: x_host, residual_host
 * (nullable), logit_bias_host (nullable), out_host, idx_host and w_host (both nullable) are
 * host pointers (page-locked for the copies to be asynchronous). The call stages them
 * through library-owned device memory on `stream` with one cudaMemcpyAsync per buffer:
 * inputs host->device, the launch, outputs device->host. Host buffers must stay valid and
 * unmodified until `stream` has completed the call. Layer descriptors are device memory as
 * usual. */
int fmoe_moe_layer_seq_host(const fmoe_layer_desc* layers, int n_layers, const float* x_host,
                            const float* residual_host, int n_tokens,
                            const float* logit_bias_host, float* out_host, int32_t* idx_host,
                            float* w_host, void* stream);

/* ---------------------------------------------------------------------------------------
 * MoE-only decode stack: n_tokens tokens, each through n_layers layers in order, token by
 * token ([JA-O] "遅延GPUエキスパート計算": the combine + residual + norm output feeds the next
 * layer with no host round trip). For token t:
 *   h_0 = h_in[t]
 *   x_0 = h_0 (layer 0 is not normalised);  x_l = h_l / sqrt(mean(h_l^2) + eps) for l >= 1
 *   h_{l+1} = MoE layer l (x_l, residual = h_l)
 *   h_out[t] = h_L
 * logit_bias: nullable [T x L x E]. idx_trace: nullable [T x L x K] int32 (chosen experts).
 * h_trace: nullable [T x L x H] fp32: the input h_l of every layer before its RMSNorm (h_0 =
 * h_in), for teacher-forced checking of single layers.
 * 1 <= n_layers <= 128; all layers share H, I, E, K, bits. h_out must not alias h_in.
 * --------------------------------------------------------------------------------------- */
int fmoe_moe_stack(const fmoe_layer_desc* layers, int n_layers, const float* h_in,
                   int n_tokens, const float* logit_bias, float eps, float* h_out,
                   int32_t* idx_trace, float* h_trace, void* stream);

/* Same computation as fmoe_moe_stack, captured once into a CUDA graph that owns its scratch
 * memory; fmoe_stack_graph_launch replays it on `stream` (same buffers every replay).
 * tokens_per_launch: tokens per kernel launch inside the graph (0 = all tokens in one
 * launch). The graph handle is freed with fmoe_stack_graph_destroy (after its last replay
 * has completed). */
typedef struct fmoe_graph fmoe_graph;
int fmoe_stack_graph_create(const fmoe_layer_desc* layers, int n_layers, const float* h_in,
                            int n_tokens, const float* logit_bias, float eps, float* h_out,
                            int32_t* idx_trace, float* h_trace, int tokens_per_launch,
                            fmoe_graph** graph);
int fmoe_stack_graph_launch(fmoe_graph* graph, void* stream);
int fmoe_stack_graph_destroy(fmoe_graph* graph);

/* Launch geometry of the engine kernel for a shape on a GPU with `sms` SMs and `max_smem`
 * bytes of shared memory per block (host only; no CUDA call). flags: bit 0 router, bit 1
 * shared expert, bit 2 routed experts, bit 3 shared-expert gate. Writes up to n_out int64
 * values in the order documented in FMOE_GEOMETRY_FIELDS and returns how many were written,
 * or a negative status for an unsupported shape. For checking the launch layout against
 * buffer bounds on a machine without a GPU. */
#define FMOE_GEOMETRY_FIELDS                                                                  \
    "H I E K bits route_on shared_on routed_on gate_on rc_h rs_h rc_i rs_i q_gu nr rseg rcols " \
    "rrows au hr ad dr nseg sh wh gh si wi pi ji stage_bytes nA nB o_ringA o_ringB o_x o_h "    \
    "o_red o_oacc o_misc o_bar oacc_n smem_bytes consumer_warps max_rows_thread max_rows_warp " \
    "red_slot gpass"
int fmoe_describe_geometry(int hidden, int inter, int n_experts, int top_k, int bits, int flags,
                           int max_smem, int sms, int64_t* out, int n_out);

/* Selects how the expert GEMVs evaluate each group-affine dot product, for kernels launched
 * afterwards on the calling host thread (all give the same value in real arithmetic):
 *   0  default: s * sum(q * x) + z * sum(x) per 32-column slice, sum(q * x) as integer dp4a
 *      products of the codes with three signed 8-bit digit planes of x;
 *   1  the pages' literal form per weight: sum of fma(q, s * x, z * x) ([FR-A] §2 "Noyaux de
 *      Déquantification Optimisés pour FMA", the form after the rewrite);
 *   2  the naive form per weight: sum of (q * s + z) * x ([FR-A] §2, the form before it).
 * Returns FMOE_ERR_INVALID for another value (the setting is then unchanged). */
int fmoe_set_dot_form(int form);

/* Number of kernel launches of this library enqueued on the calling host thread so far
 * (graph replays count the kernels inside the graph). For accounting in benchmarks. */
uint64_t fmoe_launch_count(void);

/* ---------------------------------------------------------------------------------------
 * fmoe_moe_layer with no allocation. The pages have no counterpart: it is an interface
 * variant for callers that must not allocate device memory at call time, such as a decode
 * loop that reserved all free device memory for weights and caches up front, or a latency-
 * bound caller that must never wait on the allocator growing a pool (which can synchronise
 * the device).
 *
 * Same arguments, layout, validation and result as fmoe_moe_layer (one token). The library
 * scratch of the call (unit-done words, tagged router logits, tagged h vectors) lives in
 * one fixed device array of FMOE_NOALLOC_SCRATCH_BYTES per device, compiled into the library;
 * the call makes no cudaMalloc, cudaFree, pool or other allocating call.
 *   - The first call on a device does the setup: it obtains the array's address with
 *     cudaGetSymbolAddress (which also loads the library's kernels on that device), zeroes the
 *     array's error word and sets the kernel's shared-memory limit. Make that first call with
 *     the device current and outside any stream capture; later calls only enqueue work.
 *   - The exchange words must start at zero for every launch: each call zeroes the scratch
 *     it uses with one cudaMemsetAsync on `stream` before its launch.
 *   - Shapes whose scratch exceeds the array (beyond FMOE_NOALLOC_SCRATCH_BYTES minus 256
 *     bytes for the error word; e.g. 4096 experts with top_k = 8 and I = 1024) return
 *     FMOE_ERR_UNSUPPORTED with the needed size in fmoe_last_error(); nothing is enqueued.
 *     The full-size layer (H = 4096, I = 1024, E = 512, K = 4) needs 91,392 bytes.
 *   - There is one array per device: two calls of this function on one device whose work can
 *     overlap (different streams, or host threads without ordering) race on it and give
 *     undefined results. Calls on one stream are ordered and safe.
 *   - A device-side wait that runs out of budget is recorded in the array's error word and
 *     reported (and cleared) by fmoe_sync_status like the other entry points' errors.
 * --------------------------------------------------------------------------------------- */
#define FMOE_NOALLOC_SCRATCH_BYTES (128u * 1024u)
int fmoe_moe_layer_noalloc(const fmoe_layer_desc* layer, const float* x, const float* residual,
                           const float* logit_bias, float* out, int32_t* idx_out, float* w_out,
                           void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FMOE_H */
