// engine.h — host/device description of one launch of the MoE engine kernel.
//
// A launch runs a sequence of "units"; a unit is one MoE layer applied to one token. The work
// of a unit is cut into chunks of one shared-memory stage each, listed in dependency order:
//   K_ROUTER  a column segment of one or more router rows (fp32 weights, binary64 sums); the
//             shared-gate vector is router row E
//   K_SGU     R rows of the shared expert's gate matrix and the same R rows of its up matrix
//   K_RGU     the same for routed expert k (needs the routing decision)
//   K_DN      Rd output rows of the fused down projection: output row j is the dot product of
//             the concatenated rows j of every active down matrix (shared expert first, then
//             routed k = 0..K-1) with the concatenated inputs [sigma*h_s | w_0*h_0 | ...]
// Completion is counted per class: CL_ROUTER (router chunks), CL_GU (shared and routed gate/
// up chunks) and CL_DN. Chunk g of the launch (g = unit * chunks_per_unit + index) belongs to
// CTA g mod gridDim; inside a CTA, local chunk i goes to consumer warp i mod kConsumerWarps and
// ring stage i mod nstage. The transforms of a unit's x and down input are shared by the
// consumer warps that hold the unit's gate/up (down) chunks, an equal part each, done at the
// warp's first chunk that needs it, after which it waits for the other parts; those first
// chunks are at most kConsumerWarps - 1 local chunks apart, and the ring holds at least
// kConsumerWarps stages, so they are all in flight together. Every other wait
// a chunk makes is on chunks with smaller g, so with all CTAs resident (one per SM) the
// schedule cannot deadlock, and every wait is bounded in time.
#pragma once
#include <stdint.h>

namespace fmoe {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kCtrlWarps = 2;                      // producer + stager
constexpr int kThreads = kConsumers + 32 * kCtrlWarps;
constexpr int kMaxLayers = 128;
constexpr int kMaxK = 8;
constexpr int kRowsPerLane = 8;                    // rows one lane accumulates per chunk
constexpr int kStageTarget = 11520;                // bytes of weights per chunk (target)
constexpr int kMaxStages = 32;

enum Kind { K_ROUTER = 0, K_SGU = 1, K_RGU = 2, K_DN = 3, K_COUNT = 4 };
enum Class { CL_ROUTER = 0, CL_GU = 1, CL_DN = 2, CL_COUNT = 3 };

// Control words (uint32, zeroed before every launch). Class counters take one atomic per CTA
// per run of same-class chunks; class c is complete for units 0..u when its counter reaches
// (u + 1) * ncl[c], which the waiters (one warp per CTA) read directly.
enum Ctrl {
  C_CNT = 0,                    // C_CNT + 32*class: chunks of that class completed (all units)
  C_WORDS = 32 * CL_COUNT       // every counter on its own 128-byte line
};

enum ModeBits { MODE_SEQ = 0, MODE_STACK = 1 };

struct LayerW {
  const uint8_t* experts;
  unsigned long long expert_stride;
  const uint8_t* shared;       // nullable
  const float* router;         // [E x H]
  const float* gate;           // nullable [H]
};

// Lane layout of a dot-product chunk inside one warp: S lanes share a row (S a power of two,
// >= the row's 32-column slices when they are fewer than 32), P = 32 / S rows side by side.
struct LaneMap {
  int nsl;                     // 32-column slices per (virtual) row
  int S, P;                    // lanes per row, rows side by side
  int nrl;                     // rows per lane (<= kRowsPerLane)
};

struct Geo {
  int H, I, E, K, bits;
  int route_on, shared_on, routed_on, gate_on;
  unsigned rc_h, rs_h, rc_i, rs_i;  // bytes per row of codes / scale-bias words (H or I wide)
  unsigned long long q_gu;          // bytes of one I x H packed matrix (gate or up)
  // router chunks
  int nr;                      // router rows: E + gate_on
  int rseg;                    // column segments per router row
  int rcols;                   // columns per segment (H / rseg)
  int rrows;                   // router rows per chunk (1 when rseg > 1)
  int nrb;                     // router row blocks: ceil(nr / rrows)
  // gate/up chunks
  int R;                       // rows of gate (and as many of up) per chunk
  int nb;                      // chunks per expert: ceil(I / R)
  // down chunks
  int nseg;                    // segments of a down virtual row: shared_on + K (routed)
  int Rd;                      // virtual rows per chunk
  int n[K_COUNT];
  int off[K_COUNT + 1];        // off[K_COUNT] = chunks per unit
  int ncl[CL_COUNT];           // chunks per unit of each class
  LaneMap gu, dn;
  // shared memory carve-up (byte offsets from the dynamic smem base)
  unsigned stage_bytes;
  int nstage;
  unsigned o_ring, o_full, o_empty, o_xa, o_xg, o_red, o_misc;
  unsigned smem_bytes;
};

struct Scratch {
  unsigned* ctrl;        // C_WORDS
  int* err;              // sticky per-device error word
  double* logits;        // [2][rseg][nr] partial logits per column segment
  float* hs;             // [2][I]
  float* hk;             // [2][K][I]
  float* normsq;         // [n_units]
  float* hbuf;           // [2][H]
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
  unsigned long long wait_ns;
  int debug;             // bit 0: the routing decision is never published (timeout test)
  Scratch s;
  LayerW layers[kMaxLayers];
};

// error codes written to Scratch::err (first one wins)
enum DevErr { DE_NONE = 0, DE_TIMEOUT_FULL = 1, DE_TIMEOUT_EMPTY = 2, DE_TIMEOUT_ROUTE = 3,
              DE_TIMEOUT_DEP = 4, DE_TIMEOUT_DRAIN = 5 };

}  // namespace fmoe
