// engine.h — host/device description of one launch of the MoE engine kernel.
//
// A launch runs a sequence of "units"; a unit is one MoE layer applied to one token, and units
// run strictly one after another (unit u+1 computes only after every output of unit u is
// written; its weights may be fetched earlier). One CTA per SM. Every CTA owns a contiguous,
// equal share of the rows of every phase of a unit:
//   router rows      [E router rows, then the shared-gate vector as row E]  -> logits
//   h-rows           I rows of every expert's gate and up matrices (the same rows for the
//                    shared expert and for each routed expert)            -> h = SiLU(g) * u
//   output rows      H rows of every expert's down matrix                  -> out
// The share of each phase is cut into chunks of at most one shared-memory stage and streamed
// through two rings of stages:
//   ring A (data-independent weights, streamed ahead across units): the CTA's router chunks,
//          shared-expert gate/up chunks and shared-expert down chunks of each unit;
//   ring B (weights that depend on the routing decision): the routed experts' gate/up chunks
//          (expert k = 0..K-1 in turn), then their down chunks.
// The consumer warps work through a unit in the order
//   router (A) -> shared gate/up (A) -> shared down (A) -> routed gate/up k (B) -> routed down k (B)
// with every warp taking part in every chunk.
// Cross-CTA data moves as self-validating 64-bit words, written without fences and read by
// polling: each word carries the unit it belongs to (a tag), so a reader that sees the right
// tag has the value, and no flag, release fence or second round trip is needed:
//   router logits   binary64, the tag in the 13 lowest mantissa bits;
//   h values        {binary32 value, 32-bit tag};
//   stack outputs   {binary32 value, 32-bit tag} (the next layer's input).
// Where nothing is read (one token's output before an independent next token), each CTA
// stores a per-CTA "unit done" word instead; the buffers alternate between units, so unit u
// of independent tokens with expert rows starts once every CTA's word shows unit u-2 (a
// router-only launch, and a stack's next token, once it shows unit u-1). Every exchange buffer is zeroed before each launch; tags are
// never zero.
#pragma once
#include <stdint.h>

namespace fmoe {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kCtrlWarps = 3;                      // producer A, producer B, controller
constexpr int kThreads = kConsumers + 32 * kCtrlWarps;
constexpr int kMaxLayers = 128;
constexpr int kMaxK = 8;
constexpr unsigned kStage = 36864;                 // bytes per ring stage
constexpr int kRouterCols = 4 * 4 * 256;           // router columns per chunk (4 float4 per thread)
constexpr int kMaxStages = 16;                     // per ring
constexpr int kMaxRowsThread = 8;                  // gate/up rows one consumer thread holds
constexpr int kMaxRowsWarp = 4;                    // down rows (per side-by-side lane group) a warp holds
constexpr int kMaxHr = 64;                         // h-rows per gate/up chunk (cap)
constexpr int kRouterBatch = 4;                    // router rows reduced together

// Per-CTA "unit done" words (Scratch::ctrl[cta]): the number of units whose output rows the
// CTA has written.
constexpr int kMaxCtas = 256;                      // grid size limit (one CTA per SM)
constexpr int kCtrlWords = kMaxCtas;
constexpr int kMiscBytes = 4096;                   // small shared state (Smem)

enum ModeBits { MODE_SEQ = 0, MODE_STACK = 1 };

struct LayerW {
  const uint8_t* experts;
  unsigned long long expert_stride;
  const uint8_t* shared;       // nullable
  const float* router;         // [E x H]
  const float* gate;           // nullable [H]
};

struct Geo {
  int H, I, E, K, bits;
  int route_on, shared_on, routed_on, gate_on;
  unsigned rc_h, rs_h, rc_i, rs_i;  // bytes per row of codes / scale-bias words (H or I wide)
  unsigned long long q_gu;          // bytes of one I x H packed matrix (gate or up)
  // router chunks
  int nr;                      // router rows: E + gate_on
  int rseg;                    // column segments per router row (1 when a row fits a stage)
  int rcols;                   // columns per segment
  int rrows;                   // router rows per chunk (rseg == 1)
  // gate/up chunks
  int au;                      // h-row alignment unit (rows whose sb bytes are a multiple of 16)
  int hr;                      // h-rows per chunk (a multiple of au)
  int gpass;                   // gate/up chunks processed together (1 or 2)
  // down chunks
  int ad;                      // output-row alignment unit
  int dr;                      // output rows per chunk (a multiple of ad)
  int nseg;                    // down segments per output row: shared_on + K (routed)
  // consumer thread layout for H-wide rows: slices S_h = H/32, W_h threads per row (a power
  // of two >= S_h up to 32, else a multiple of 32), G_h = 256 / W_h row groups
  int sh, wh, gh;
  // consumer layout for I-wide rows: slices S_i = I/32; W_i lanes per row (power of two
  // >= S_i, at most 32); P_i = 32 / W_i rows side by side in a warp; J_i slices per lane
  int si, wi, pi, ji;
  // shared memory carve-up (byte offsets from the dynamic smem base)
  unsigned stage_bytes;
  int nA, nB;                  // stages of ring A and ring B
  unsigned o_ringA, o_ringB, o_x, o_h, o_red, o_oacc, o_misc, o_bar;
  int oacc_n;                  // output accumulators (most output rows a CTA owns)
  unsigned red_slot;           // bytes of the reduction area per stage (both rings)
  unsigned smem_bytes;
};

// Exchange buffers, indexed by unit parity; all zeroed before each launch.
struct Scratch {
  unsigned* ctrl;                 // kCtrlWords unit-done words
  int* err;                       // sticky per-device error word
  unsigned long long* logits;     // [2][rseg][nr] tagged binary64 partial logits per column segment
  unsigned long long* hx;         // [2][nseg][I] tagged h values: shared expert first, then routed k
  unsigned long long* hbuf;       // [2][H] tagged stack outputs (STACK mode only; else null)
};

struct Prog {
  int mode;
  int n_units, n_layers, n_tokens;
  const float* x;        // SEQ: [T x H] inputs; STACK: h_in
  const float* res;      // SEQ: nullable [T x H]
  float* out;            // SEQ: [T x H]; STACK: h_out
  const float* bias;     // SEQ: [T x E]; STACK: [T x L x E]; nullable
  int* idx_out;          // SEQ: [T x K]; STACK: [T x L x K]; nullable
  float* w_out;          // SEQ: [T x K]; nullable
  float* h_trace;        // STACK: [T x L x H] layer inputs before the norm; nullable
  float eps;
  int form;              // dot-product form (DotForm)
  unsigned long long wait_ns;
  int debug;             // bit 0: the router signal is never raised (timeout test)
  Scratch s;
  LayerW layers[kMaxLayers];
};

// Evaluation of one group-affine dot product over a 32-column slice (same value in real
// arithmetic): integer products of the codes with three 8-bit digit planes of x (default),
// the pages' literal fma(q, s*x, z*x) per weight, or the naive (q*s + z)*x per weight.
enum DotForm { FORM_DIGITS = 0, FORM_FMA = 1, FORM_NAIVE = 2, FORM_COUNT = 3 };

// error codes written to Scratch::err (first one wins)
enum DevErr { DE_NONE = 0, DE_TIMEOUT_FULL = 1, DE_TIMEOUT_EMPTY = 2, DE_TIMEOUT_ROUTE = 3,
              DE_TIMEOUT_DEP = 4, DE_TIMEOUT_DRAIN = 5 };

// The contiguous share [lo, hi) of n items (in units of `unit` items) that CTA c of nc owns.
__host__ __device__ __forceinline__ void share_of(int n, int unit, int c, int nc, int* lo,
                                                  int* hi) {
  const long long nu = n / unit;
  *lo = (int)(nu * c / nc) * unit;
  *hi = (int)(nu * (c + 1) / nc) * unit;
}

}  // namespace fmoe
