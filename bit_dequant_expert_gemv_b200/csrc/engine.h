// engine.h — host/device description of one launch of the MoE engine kernel.
//
// A launch runs a sequence of "units"; a unit is one MoE layer applied to one token. The work
// of a unit is cut into chunks, listed in dependency order by phase:
//   P_ROUTER   router rows (fp32, binary64 accumulation) + the shared-gate row; the CTA whose
//              completion brings the router count to its target selects the top-K experts
//   P_SGU      shared expert gate/up rows + SwiGLU            (needs x)
//   P_SDN      shared expert down rows + residual             (needs the shared h and sigma)
//   P_RGU      routed experts gate/up rows + SwiGLU           (needs the routing decision)
//   P_RDN      routed experts down rows + weighted combine    (needs all routed h)
// Chunk g of the launch (g = unit * chunks_per_unit + index) belongs to CTA g mod gridDim, and
// every CTA works through its chunks in increasing g; every wait a chunk makes is on chunks with
// smaller g, so with all CTAs resident (one per SM) the schedule cannot deadlock, and every wait
// is bounded in time in any case.
#pragma once
#include <stdint.h>

namespace fmoe {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;    // 256 consumer threads
constexpr int kThreads = kConsumers + 64;          // + one producer warp + one signal warp
constexpr int kMaxLayers = 128;
constexpr int kMaxK = 8;
constexpr int kMaxSlices = 256;                    // 32-column slices per (virtual) row
constexpr int kSliceCols = 32;
constexpr int kBoxes = 4;                          // outbox depth (chunks)

enum Phase { P_ROUTER = 0, P_SGU = 1, P_SDN = 2, P_RGU = 3, P_RDN = 4, P_COUNT = 5 };

// Control words (uint32, zeroed before every launch). Phase counters take one atomic per CTA
// per run of chunks; the CTA whose atomic completes a phase of a unit writes "phase p of unit
// u is complete" into every CTA's own flag line, and waiters poll only their own line.
enum Ctrl {
  C_CNT = 0,                    // C_CNT + 32*phase: chunks of that phase completed (all units)
  C_WORDS = 32 * P_COUNT,       // every counter on its own 128-byte line
  F_WORDS = 32                  // per-CTA flag line: word p = units whose phase p is complete
};

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
  // bytes per row
  unsigned rc_h, rs_h, rc_i, rs_i;
  unsigned long long q_gu, q_dn;  // bytes of an I x H (gate/up) and an H x I (down) packed matrix
  // rows per chunk
  int rr, rcg, rsd, rrd;
  int nr;                      // router rows: E + gate_on
  int nb;                      // gate/up chunks per expert
  int n[P_COUNT];
  int off[P_COUNT + 1];        // off[P_COUNT] = chunks per unit
  // thread mapping: slices of 32 columns, padded per virtual row
  int sl_h, sp_h, p_h;         // H-wide rows (gate/up)
  int sl_i, sp_i, p_i;         // I-wide rows (shared down)
  int sl_d, sp_d, p_d;         // K*I-wide virtual rows (routed down)
  int w_gu, w_sd, w_rd;        // waves per chunk
  // shared memory carve-up (byte offsets from the dynamic smem base)
  unsigned stage_bytes;
  int nstage;
  unsigned o_ring, o_full, o_empty, o_meta, o_xr, o_xg, o_sxg, o_xs, o_sxs, o_xd, o_sxd, o_red,
      o_rows, o_misc;
  unsigned smem_bytes;
  unsigned o_box;              // reduction slots: kBoxes x box_floats (partials + prefetched base)
  int box_floats;
  int red_part;                // floats of per-warp partials at the start of a slot (then bases)
};

struct Scratch {
  unsigned* ctrl;        // C_WORDS
  unsigned* flags;       // [gridDim][F_WORDS]
  int* err;              // sticky per-device error word
  double* logits;        // [2][nr]
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
