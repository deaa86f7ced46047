// engine.cu — the persistent MoE-layer engine for sm_100a.
//
// What it computes (per unit = one token through one MoE layer), after the Flash-MoE pages:
//   router GEMV over E experts, softmax and top-K with renormalised weights
//     ("Flash-MoE：純粋なC/Metal…" (openclawradar.com), "パイプラインパフォーマンス": CMD2 routing,
//      then softmax + topK);
//   per selected expert and for the shared expert: gate and up dequantising GEMVs with a fused
//   SwiGLU, then the down GEMV; the routing-weighted combine with the sigmoid-gated shared
//   expert and the residual, in one pass
//     ("Qu'est-ce que Flash-MoE ?" (a2a-mcp.org, fr), §3 "Compute Shaders Metal Optimisés à la
//      Main");
//   each 4-/2-bit weight is q*s + z with one bf16 scale/bias per 64-weight group. The default
//   evaluation is s * sum(q*x) + z * sum(x) per 32-column slice: the pages' fma(nibble,
//   scale*x, bias*x) with the scale and bias factored out of the slice sum (same value in real
//   arithmetic; "Qu'est-ce que Flash-MoE ?" (a2a-mcp.org, fr), §2 "Noyaux de Déquantification
//   Optimisés pour FMA"), where sum(q*x) is taken as integer dot products of the codes with
//   three 8-bit digit planes of x (x ~ s_x (d0 + d1/128 + d2/16384), within 1e-6 of the
//   slice's largest |x|), one dp4a per four weights. The pages' literal form
//   fma(q, s*x, z*x) and the naive (q*s + z)*x per weight are compiled as selectable
//   alternatives (DotForm), for the comparison the pages make between them.
//
// How (one CTA per SM, 11 warps):
//   warp 0  producer A: streams the CTA's data-independent chunks (router rows, shared-expert
//           gate/up and down rows) unit after unit into ring A, as far ahead as the ring
//           allows, with 1-D TMA bulk copies (no multicast) completing on the stage barriers;
//   warp 1  producer B: once a unit's routing decision is known, streams the CTA's rows of
//           the K routed experts (gate/up, then down) into ring B;
//   warp 2  controller: brings each unit's x into shared memory, waits for the router signal
//           and selects the top-K (redundantly in every CTA, so no second broadcast), brings in
//           each expert's h as soon as its signal completes;
//   warps 3-10  consumers: all eight take part in every chunk. For gate/up rows each thread
//           owns one 32-column slice of x (its digit planes in registers for the whole unit) and
//           a few of the chunk's rows; for down rows each lane owns a slice of h and each warp a
//           few output rows, accumulated over the shared and the routed experts.
// Every spin-wait is bounded by a global-timer budget; on expiry the kernel records an error
// word, every role leaves its loop, the producers wait for their copies in flight and return.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "engine.h"
#include "ptx.cuh"

// Timeline hooks (a point of a unit's progress reached by one role), defined by the profiling
// build of timeline/timeline.py (timeline/marks.cuh); they expand to nothing in the library.
#ifndef FMOE_MARK
#define FMOE_MARK(u, ev) ((void)0)
#endif

namespace fmoe {

enum MarkEv {
  MK_C_UNIT = 0, MK_C_PREV_DONE, MK_C_X, MK_C_S1, MK_C_RT, MK_C_XFREE, MK_C_SS, MK_C_HS,
  MK_C_S2 = 8, MK_C_HK = 16,
  MK_K_X = 24, MK_K_ROUTER, MK_K_XD, MK_K_SGU, MK_K_HS, MK_K_DS,
  MK_K_P2F = 30, MK_K_P2 = 38, MK_K_HK = 46, MK_K_D = 54, MK_K_OUT = 62,
  MK_B_RT = 63, MK_B_LAST, MK_A_FIRST, MK_A_LAST,
  MK_R_DOT = 67, MK_R_RED, MK_R_LAST, MK_R_PUB,   // router batch: first and last consumer warp
  MK_R_DOT_W = 71, MK_R_RED_W, MK_R_LAST_W,
  MK_G_DOT = 74, MK_G_RED, MK_G_LAST, MK_G_PUB,   // first gate/up pass of routed expert 0
  MK_G_DOT_W = 78, MK_G_RED_W, MK_G_LAST_W,
  MK_J1_TOP = 81, MK_J1_W0, MK_B_I2, MK_B_I3, MK_G_EPI_END
};
// marks from the first (w == 0) and the last consumer warp inside a phase
#define FMOE_MARK_W(u, ev0, evw)                                   \
  do {                                                             \
    const int w_ = ((int)threadIdx.x >> 5) - kCtrlWarps;           \
    if (w_ == 0) FMOE_MARK(u, ev0);                                \
    if (w_ == kConsumerWarps - 1) FMOE_MARK(u, evw);               \
  } while (0)

// ------------------------------------------------------------------------------------------
// small shared state
// ------------------------------------------------------------------------------------------
struct Smem {
  uint64_t xbar;               // the controller's bulk-copy barrier for x
  // Readiness published by the controller (and one by the consumers): a monotone counter (the
  // truth) and an mbarrier that completes one phase per increment, used only to sleep until
  // the next increment.
  uint64_t x_bar, rt_bar, hs_bar, hk_bar, xfree_bar;
  unsigned x_ready;            // units whose x is in the x buffer
  unsigned rt_ready;           // units whose routing decision is in rt_e / rt_w
  unsigned hs_ready;           // units whose h_s is in the h buffer
  unsigned hk_ready;           // routed segments ready, counted over units: u*K + k + 1
  unsigned xfree;              // units whose x buffer the consumers no longer read
  unsigned xd_arrive;          // consumer warps done loading x digits (8 per unit)
  unsigned chunk_arrive[2 * kMaxStages];  // per stage (ring A, then B): warps done with it
  float xf[2];                 // RMSNorm factor of the unit's x (1 without a norm)
  float sigma[2];              // sigmoid(g . x) of the unit (1 without a shared gate)
  int rt_e[2][kMaxK];          // routing of unit u (index u & 1): experts and weights
  float rt_w[2][kMaxK];
  // top-K candidates: each consumer warp's K best packed keys and their binary64 logits
  unsigned long long cand_key[kConsumerWarps * kMaxK];
  double cand_l[kConsumerWarps * kMaxK];
  volatile int abort;
};
static_assert(sizeof(Smem) <= kMiscBytes, "small shared state exceeds its area");

__device__ __forceinline__ void raise_error(const Prog& P, Smem* sm, int code) {
  atomicCAS(P.s.err, 0, code);
  sm->abort = 1;
}

// ------------------------------------------------------------------------------------------
// exchange words (see engine.h): tags, packing, unit-done words
// ------------------------------------------------------------------------------------------
constexpr unsigned long long kTag13 = 0x1FFFull;               // logit words: low mantissa bits
constexpr unsigned long long kTag32 = 0xFFFFFFFF00000000ull;   // value words: high half

__device__ __forceinline__ unsigned long long tag13(int u) {
  return (unsigned long long)(u % 8191 + 1);
}
__device__ __forceinline__ unsigned long long tag32(int u) {
  return (unsigned long long)(unsigned)(u + 1) << 32;
}
// A binary64 logit with the unit's tag in its 13 lowest mantissa bits (a change of at most
// 2^-39 relative, inside the band where the top-K treats logits as tied).
__device__ __forceinline__ unsigned long long logit_word(double l, int u) {
  return ((unsigned long long)__double_as_longlong(l) & ~kTag13) | tag13(u);
}
__device__ __forceinline__ double logit_of(unsigned long long w) {
  return __longlong_as_double((long long)(w & ~kTag13));
}
__device__ __forceinline__ unsigned long long value_word(float v, int u) {
  return tag32(u) | (unsigned long long)__float_as_uint(v);
}
__device__ __forceinline__ float value_of(unsigned long long w) {
  return __uint_as_float((unsigned)w);
}

// This lane: poll the word at p until its tag bits (mask) equal `want`, the budget runs out,
// the CTA aborts or another CTA has recorded an error. Returns the last word read; if its tag
// differs from `want`, the wait failed (and the failure is recorded).
__device__ __noinline__ unsigned long long await_word(const Prog& P, Smem* sm,
                                                      const unsigned long long* p,
                                                      unsigned long long mask,
                                                      unsigned long long want, int code) {
  unsigned long long v = ld_relaxed_gpu_u64(p);
  if ((v & mask) == want) return v;
  const uint64_t deadline = global_ns() + P.wait_ns;
#pragma unroll 1
  for (unsigned it = 0;; ++it) {
    __nanosleep(32);
    v = ld_relaxed_gpu_u64(p);
    if ((v & mask) == want) return v;
    if ((it & 7) == 7) {
      if (sm->abort || ld_volatile_int(P.s.err) != 0) {
        sm->abort = 1;
        return v;
      }
      if (global_ns() > deadline) {
        raise_error(P, sm, code);
        return v;
      }
    }
  }
}

// This lane's N words v[j] (already loaded from addr(j)): re-read every word whose tag bits
// (mask) differ from `want`, all those loads in flight together, with a short sleep between
// rounds, until every word matches, the budget runs out, the CTA aborts or another CTA has
// recorded an error (the failure is then recorded). False on failure.
template <int N, typename Addr>
__device__ __forceinline__ bool settle(const Prog& P, Smem* sm, unsigned long long (&v)[N],
                                       Addr addr, unsigned long long mask,
                                       unsigned long long want, int code) {
  unsigned miss = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) miss |= ((v[j] & mask) != want ? 1u : 0u) << j;
  if (!miss) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
#pragma unroll 1
  for (unsigned it = 0;; ++it) {
    __nanosleep(64);
#pragma unroll
    for (int j = 0; j < N; ++j)
      if ((miss >> j) & 1u) v[j] = ld_relaxed_gpu_u64(addr(j));
    miss = 0;
#pragma unroll
    for (int j = 0; j < N; ++j) miss |= ((v[j] & mask) != want ? 1u : 0u) << j;
    if (!miss) return true;
    if ((it & 7) == 7) {
      if (sm->abort || ld_volatile_int(P.s.err) != 0) {
        sm->abort = 1;
        return false;
      }
      if (global_ns() > deadline) {
        raise_error(P, sm, code);
        return false;
      }
    }
  }
}

// This CTA has written every output row of units 0..u (one lane). Nothing is read through
// this word: it only orders the start of the next unit after the end of this one.
__device__ __forceinline__ void unit_done(const Prog& P, int u) {
  st_relaxed_gpu(P.s.ctrl + blockIdx.x, (unsigned)(u + 1));
}

// ------------------------------------------------------------------------------------------
// bounded waits
// ------------------------------------------------------------------------------------------
// Whole warp: spin until every CTA's unit-done word has reached `target` (wrap-safe), the
// budget runs out, the CTA aborts or another CTA has recorded an error. Lane l polls words
// 4l..4l+3 and 128+4l.. with relaxed 16-byte loads.
__device__ __noinline__ bool warp_wait_done(const Prog& P, Smem* sm, unsigned target, int code) {
  const int lane = threadIdx.x & 31;
  const int nc = gridDim.x;
  const unsigned* row = P.s.ctrl;
  uint64_t deadline = 0;
#pragma unroll 1
  for (unsigned it = 0;; ++it) {
    bool ok = true;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int w0 = 4 * lane + 128 * h;
      if (w0 < nc) {
        const uint4 v = ld_relaxed_gpu_v4(row + w0);
        ok = ok && (int)(v.x - target) >= 0;
        ok = ok && (w0 + 1 >= nc || (int)(v.y - target) >= 0);
        ok = ok && (w0 + 2 >= nc || (int)(v.z - target) >= 0);
        ok = ok && (w0 + 3 >= nc || (int)(v.w - target) >= 0);
      }
    }
    if (__all_sync(0xffffffffu, ok)) return true;
    if (it == 0) deadline = global_ns() + P.wait_ns;
    int bad = 0;
    if (lane == 0 && (it & 7) == 7) {
      if (sm->abort || ld_volatile_int(P.s.err) != 0) {
        sm->abort = 1;
        bad = 1;
      } else if (global_ns() > deadline) {
        raise_error(P, sm, code);
        bad = 1;
      }
    }
    if (__shfl_sync(0xffffffffu, bad, 0)) return false;
    __nanosleep(20);
  }
}

// Waits on shared-memory barriers and counters poll with short sleeps in between by default;
// a positive FMOE_WAIT_SUSPEND_NS selects a try_wait that suspends the thread with that time
// hint instead (the two measured the same).
#ifndef FMOE_WAIT_SUSPEND_NS
#define FMOE_WAIT_SUSPEND_NS 0
#endif

__device__ __forceinline__ bool mbar_poll(uint64_t* bar, unsigned parity) {
  if (FMOE_WAIT_SUSPEND_NS > 0) return mbar_try_wait_sleep(bar, parity, FMOE_WAIT_SUSPEND_NS);
  if (mbar_try_wait(bar, parity)) return true;
  __nanosleep(20);
  return false;
}

__device__ __noinline__ bool wait_mbar(const Prog& P, Smem* sm, uint64_t* bar, unsigned parity,
                                       int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
#pragma unroll 1
  for (unsigned it = 0;; ++it) {
    if (mbar_poll(bar, parity)) return true;
    if ((it & 7) == 7) {
      if (sm->abort) return false;
      if (global_ns() > deadline) {
        raise_error(P, sm, code);
        return false;
      }
    }
  }
}

// Wait until the readiness counter *cnt reaches target (the publisher stores the counter
// with release semantics; it also arrives on `bar`, which the suspending form sleeps on).
__device__ __noinline__ bool wait_ready(const Prog& P, Smem* sm, const unsigned* cnt,
                                        uint64_t* bar, unsigned target, int code) {
  unsigned c = ld_acquire_cta_smem(cnt);
  if ((int)(c - target) >= 0) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
#pragma unroll 1
  for (unsigned it = 0;; ++it) {
    if (FMOE_WAIT_SUSPEND_NS > 0) {
      if (!mbar_try_wait_sleep(bar, c & 1u, FMOE_WAIT_SUSPEND_NS)) __nanosleep(64);
    } else {
      __nanosleep(20);
    }
    c = ld_acquire_cta_smem(cnt);
    if ((int)(c - target) >= 0) return true;
    if ((it & 7) == 7) {
      if (sm->abort) return false;
      if (global_ns() > deadline) {
        raise_error(P, sm, code);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void signal_ready(unsigned* cnt, uint64_t* bar, unsigned v) {
  st_release_cta_smem(cnt, v);
  mbar_arrive(bar);
}

// Whole-warp wrappers: lane 0 waits, every lane gets the verdict.
__device__ __forceinline__ bool warp_wait_ready(const Prog& P, Smem* sm, const unsigned* cnt,
                                                uint64_t* bar, unsigned target, int code) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_ready(P, sm, cnt, bar, target, code);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ bool warp_wait_mbar(const Prog& P, Smem* sm, uint64_t* bar,
                                               unsigned parity, int code) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_mbar(P, sm, bar, parity, code);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Named barrier of the 256 consumer threads (barrier 0 is __syncthreads).
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}

// ------------------------------------------------------------------------------------------
// per-CTA shares and chunk lists
// ------------------------------------------------------------------------------------------
struct Share {
  int r0, r1;    // router rows
  int h0, h1;    // h-rows (gate/up rows of every expert)
  int d0, d1;    // output rows (down rows of every expert)
  int nrc;       // router chunks per unit
  int ngc;       // gate/up chunks per expert
  int ndc;       // down chunks per expert
  int na;        // ring-A chunks per unit
  int nb;        // ring-B chunks per unit
};

__device__ __forceinline__ Share make_share(const Geo& G) {
  Share s;
  const int c = blockIdx.x, nc = gridDim.x;
  share_of(G.nr, 1, c, nc, &s.r0, &s.r1);
  share_of(G.I, G.au, c, nc, &s.h0, &s.h1);
  share_of(G.H, G.ad, c, nc, &s.d0, &s.d1);
  const int nrr = s.r1 - s.r0;
  s.nrc = !G.route_on ? 0 : (G.rseg > 1 ? nrr * G.rseg : (nrr + G.rrows - 1) / G.rrows);
  const bool gu = G.shared_on || G.routed_on;
  s.ngc = gu ? (s.h1 - s.h0 + G.hr - 1) / G.hr : 0;
  s.ndc = G.nseg > 0 ? (s.d1 - s.d0 + G.dr - 1) / G.dr : 0;
  s.na = s.nrc + (G.shared_on ? s.ngc + s.ndc : 0);
  s.nb = G.routed_on ? G.K * (s.ngc + s.ndc) : 0;
  return s;
}

// A chunk of ring A or B decoded from its index i within the unit's list.
struct Chunk {
  int kind;      // CK_ROUTER, CK_GU, CK_DN
  int e;         // -1: shared expert; else routed slot k (0..K-1)
  int r0, n;     // first row (router row, h-row or output row) and valid rows
  int seg;       // router column segment
};
enum { CK_ROUTER = 0, CK_GU = 1, CK_DN = 2 };

__device__ __forceinline__ Chunk chunk_a(const Geo& G, const Share& S, int i) {
  Chunk c;
  c.seg = 0;
  c.e = -1;
  if (i < S.nrc) {
    c.kind = CK_ROUTER;
    if (G.rseg > 1) {
      const int rr = i / G.rseg;
      c.seg = i - rr * G.rseg;
      c.r0 = S.r0 + rr;
      c.n = 1;
    } else {
      c.r0 = S.r0 + i * G.rrows;
      c.n = min(G.rrows, S.r1 - c.r0);
    }
    return c;
  }
  i -= S.nrc;
  if (i < S.ngc) {
    c.kind = CK_GU;
    c.r0 = S.h0 + i * G.hr;
    c.n = min(G.hr, S.h1 - c.r0);
    return c;
  }
  i -= S.ngc;
  c.kind = CK_DN;
  c.r0 = S.d0 + i * G.dr;
  c.n = min(G.dr, S.d1 - c.r0);
  return c;
}

__device__ __forceinline__ Chunk chunk_b(const Geo& G, const Share& S, int i) {
  Chunk c;
  c.seg = 0;
  const int gu = G.K * S.ngc;
  if (i < gu) {
    c.kind = CK_GU;
    c.e = i / S.ngc;
    const int j = i - c.e * S.ngc;
    c.r0 = S.h0 + j * G.hr;
    c.n = min(G.hr, S.h1 - c.r0);
    return c;
  }
  i -= gu;
  c.kind = CK_DN;
  c.e = i / S.ndc;
  const int j = i - c.e * S.ndc;
  c.r0 = S.d0 + j * G.dr;
  c.n = min(G.dr, S.d1 - c.r0);
  return c;
}

// ------------------------------------------------------------------------------------------
// units
// ------------------------------------------------------------------------------------------
struct UnitView {
  int t, l, slot;
  const LayerW* L;
  const float* xin;                 // x from an input buffer (null: xw)
  const unsigned long long* xw;     // x as the previous unit's tagged output words (stack
                                    // layers after the first; x = rmsnorm of them)
  const float* res;                 // residual from an input buffer (nullable)
  const unsigned long long* resw;   // residual as tagged words (with xw)
  float* out;                       // output to a result buffer (null: outw)
  unsigned long long* outw;         // output as tagged words for the next layer
  const float* bias;                // nullable [E]
  int* idx_out;
  float* w_out;
  float* h_trace;
};

__device__ __forceinline__ UnitView unit_view(const Prog& P, const Geo& G, int u) {
  UnitView v;
  v.slot = u & 1;
  v.xw = nullptr;
  v.resw = nullptr;
  v.outw = nullptr;
  if (P.mode == MODE_SEQ) {
    v.t = u;
    v.l = u % P.n_layers;
    v.xin = P.x + (size_t)u * G.H;
    v.res = P.res ? P.res + (size_t)u * G.H : nullptr;
    v.out = P.out + (size_t)u * G.H;
    v.bias = P.bias ? P.bias + (size_t)u * G.E : nullptr;
    v.idx_out = P.idx_out ? P.idx_out + (size_t)u * G.K : nullptr;
    v.w_out = P.w_out ? P.w_out + (size_t)u * G.K : nullptr;
    v.h_trace = nullptr;
  } else {
    const int L = P.n_layers;
    v.t = u / L;
    v.l = u % L;
    if (v.l == 0) {
      v.xin = P.x + (size_t)v.t * G.H;
      v.res = v.xin;
    } else {
      v.xin = nullptr;
      v.res = nullptr;
      v.xw = P.s.hbuf + (size_t)((u - 1) & 1) * G.H;
      v.resw = v.xw;
    }
    if (v.l == L - 1) {
      v.out = P.out + (size_t)v.t * G.H;
    } else {
      v.out = nullptr;
      v.outw = P.s.hbuf + (size_t)(u & 1) * G.H;
    }
    const size_t tl = (size_t)v.t * L + v.l;
    v.bias = P.bias ? P.bias + tl * G.E : nullptr;
    v.idx_out = P.idx_out ? P.idx_out + tl * G.K : nullptr;
    v.w_out = nullptr;
    v.h_trace = P.h_trace ? P.h_trace + tl * G.H : nullptr;
  }
  v.L = &P.layers[v.l];
  return v;
}

// ------------------------------------------------------------------------------------------
// producers: the bulk copies of a chunk
// ------------------------------------------------------------------------------------------
// Copy q of chunk c (q < 4): returns its byte count (0: no such copy) and sets the source
// and the offset in the stage. `eb` is the expert blob (shared or routed). Stage layouts:
//   router:  rows r0..r0+n-1 (row E is the shared-gate vector), or one column segment;
//   gate/up: gate codes | up codes | gate sb | up sb, hr rows each (n valid);
//   down:    codes | sb, dr rows each (n valid).
__device__ __forceinline__ unsigned copy_desc(const Geo& G, const LayerW& L, const uint8_t* eb,
                                              const Chunk& c, int q, const uint8_t** src,
                                              unsigned* dst_off) {
  if (c.kind == CK_ROUTER) {
    const unsigned rowb = 4u * (unsigned)G.H;
    if (G.rseg > 1) {
      if (q != 0) return 0u;
      const float* row = c.r0 < G.E ? L.router + (size_t)c.r0 * G.H : L.gate;
      *src = reinterpret_cast<const uint8_t*>(row + (size_t)c.seg * G.rcols);
      *dst_off = 0;
      return 4u * (unsigned)G.rcols;
    }
    const int a = c.r0, b = min(c.r0 + c.n, G.E);
    if (q == 0) {
      if (b <= a) return 0u;
      *src = reinterpret_cast<const uint8_t*>(L.router + (size_t)a * G.H);
      *dst_off = 0;
      return (unsigned)(b - a) * rowb;
    }
    if (q == 1 && c.r0 + c.n > G.E) {
      *src = reinterpret_cast<const uint8_t*>(L.gate);
      *dst_off = (unsigned)(G.E - c.r0) * rowb;
      return rowb;
    }
    return 0u;
  }
  if (c.kind == CK_GU) {
    const bool up = (q & 1) != 0, sbq = q >= 2;
    const size_t mat = up ? G.q_gu : 0;
    if (!sbq) {
      *src = eb + mat + (size_t)c.r0 * G.rc_h;
      *dst_off = (up ? (unsigned)G.hr : 0u) * G.rc_h;
      return (unsigned)c.n * G.rc_h;
    }
    *src = eb + mat + (size_t)G.I * G.rc_h + (size_t)c.r0 * G.rs_h;
    *dst_off = 2u * (unsigned)G.hr * G.rc_h + (up ? (unsigned)G.hr : 0u) * G.rs_h;
    return (unsigned)c.n * G.rs_h;
  }
  if (q >= 2) return 0u;
  const uint8_t* dn = eb + 2 * G.q_gu;
  if (q == 0) {
    *src = dn + (size_t)c.r0 * G.rc_i;
    *dst_off = 0;
    return (unsigned)c.n * G.rc_i;
  }
  *src = dn + (size_t)G.H * G.rc_i + (size_t)c.r0 * G.rs_i;
  *dst_off = (unsigned)G.dr * G.rc_i;
  return (unsigned)c.n * G.rs_i;
}

__device__ __forceinline__ unsigned chunk_bytes(const Geo& G, const Chunk& c) {
  if (c.kind == CK_ROUTER) return G.rseg > 1 ? 4u * (unsigned)G.rcols : 4u * (unsigned)G.H * c.n;
  if (c.kind == CK_GU) return 2u * (unsigned)c.n * (G.rc_h + G.rs_h);
  return (unsigned)c.n * (G.rc_i + G.rs_i);
}

// Issue one chunk into a stage (one thread): wait for the stage to be free, register the
// chunk's bytes on its full barrier, issue its copies one after another. (Issuing from a
// single thread whose warp has no other live lanes streams fastest: several lanes issuing one
// copy each, or one lane of a full warp, measured markedly slower on this part.)
__device__ __forceinline__ bool issue_chunk(const Prog& P, const Geo& G, Smem* sm,
                                            uint8_t* stage, uint64_t* full, uint64_t* empty,
                                            unsigned use, const LayerW& L, const uint8_t* eb,
                                            const Chunk& c) {
  if (!wait_mbar(P, sm, empty, (use & 1u) ^ 1u, DE_TIMEOUT_EMPTY)) return false;
  mbar_arrive_expect_tx(full, chunk_bytes(G, c));
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint8_t* src = nullptr;
    unsigned dst_off = 0;
    const unsigned bytes = copy_desc(G, L, eb, c, q, &src, &dst_off);
    if (bytes) tma_load_1d(stage + dst_off, src, bytes, full);
  }
  return true;
}

// Never leave the CTA with bulk copies in flight: wait for the last use of every stage.
__device__ void drain_ring(const Prog& P, uint64_t* full, int ns, unsigned issued) {
  const uint64_t deadline = global_ns() + 100000000ull;
  const unsigned first = issued > (unsigned)ns ? issued - (unsigned)ns : 0u;
#pragma unroll 1
  for (unsigned j = first; j < issued; ++j) {
    while (!mbar_try_wait(&full[j % (unsigned)ns], (j / (unsigned)ns) & 1u)) {
      if (global_ns() > deadline) {
        atomicCAS(P.s.err, 0, DE_TIMEOUT_DRAIN);
        return;
      }
    }
  }
}

// The first ring-B chunks of unit u (min(nB, nb) of them, lane i taking chunk i), issued by the
// consumer warp that made the routing decision, as soon as it has: both stages are free then
// (the previous unit's chunks were all consumed before this unit began), and this warp's code
// is hot, where the producer thread's first issue after its wait measured ~0.8 µs.
__device__ __forceinline__ int first_b_chunks(const Geo& G, const Share& S) {
  return G.routed_on ? min(G.nB, S.nb) : 0;
}

__device__ __forceinline__ void issue_first_b(const Prog& P, const Geo& G, const Share& S,
                                              uint8_t* smem, Smem* sm, int u) {
  const int lane = threadIdx.x & 31;
  if (lane < first_b_chunks(G, S)) {
    const LayerW& L = P.layers[u % P.n_layers];
    const Chunk c = chunk_b(G, S, lane);
    const int e = min(max(sm->rt_e[u & 1][c.e], 0), G.E - 1);
    const uint8_t* eb = L.experts + (size_t)e * L.expert_stride;
    const unsigned pos = (unsigned)u * (unsigned)S.nb + (unsigned)lane;  // ring-B position
    const unsigned st = pos % (unsigned)G.nB;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_bar) + 2 * G.nA + st;
    uint8_t* stage = smem + G.o_ringB + (size_t)st * G.stage_bytes;
    mbar_arrive_expect_tx(full, chunk_bytes(G, c));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint8_t* src = nullptr;
      unsigned dst_off = 0;
      const unsigned bytes = copy_desc(G, L, eb, c, q, &src, &dst_off);
      if (bytes) tma_load_1d(stage + dst_off, src, bytes, full);
    }
  }
  __syncwarp();
}

// Producers run on one thread each (lane 0 of warps 0 and 1; the other lanes have left).
__device__ void producer_a(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm,
                           const Share& S) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_bar);
  uint64_t* empty = full + G.nA;
  unsigned issued = 0;
  bool failed = false;
#pragma unroll 1
  for (int u = 0; u < P.n_units && !failed; ++u) {
    const LayerW& L = P.layers[u % P.n_layers];
#pragma unroll 1
    for (int i = 0; i < S.na; ++i) {
      const Chunk c = chunk_a(G, S, i);
      const unsigned st = issued % (unsigned)G.nA;
      if (!issue_chunk(P, G, sm, smem + G.o_ringA + (size_t)st * G.stage_bytes, &full[st],
                       &empty[st], issued / (unsigned)G.nA, L, L.shared, c)) {
        failed = true;
        break;
      }
      if (i == 0) FMOE_MARK(u, MK_A_FIRST);
      if (i == S.na - 1) FMOE_MARK(u, MK_A_LAST);
      ++issued;
    }
  }
  if (failed) drain_ring(P, full, G.nA, issued);
}

__device__ void producer_b(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm,
                           const Share& S) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_bar) + 2 * G.nA;
  uint64_t* empty = full + G.nB;
  unsigned issued = 0;
  bool failed = false;
  if (S.nb == 0) return;
#pragma unroll 1
  for (int u = 0; u < P.n_units && !failed; ++u) {
    const LayerW& L = P.layers[u % P.n_layers];
    if (!wait_ready(P, sm, &sm->rt_ready, &sm->rt_bar, (unsigned)(u + 1), DE_TIMEOUT_ROUTE)) {
      failed = true;
      break;
    }
    FMOE_MARK(u, MK_B_RT);
    const int* rte = sm->rt_e[u & 1];
    const int i0 = first_b_chunks(G, S);  // issued by the consumer warp of the decision
    issued += (unsigned)i0;
#pragma unroll 1
    for (int i = i0; i < S.nb; ++i) {
      const Chunk c = chunk_b(G, S, i);
      const int e = min(max(rte[c.e], 0), G.E - 1);
      const uint8_t* eb = L.experts + (size_t)e * L.expert_stride;
      const unsigned st = issued % (unsigned)G.nB;
      if (!issue_chunk(P, G, sm, smem + G.o_ringB + (size_t)st * G.stage_bytes, &full[st],
                       &empty[st], issued / (unsigned)G.nB, L, eb, c)) {
        failed = true;
        break;
      }
      if (i == S.nb - 1) FMOE_MARK(u, MK_B_LAST);
      if (i == 2) FMOE_MARK(u, MK_B_I2);
      if (i == 3) FMOE_MARK(u, MK_B_I3);
      ++issued;
    }
  }
  if (failed) drain_ring(P, full, G.nB, issued);
}

// ------------------------------------------------------------------------------------------
// top-K (controller warp)
// ------------------------------------------------------------------------------------------
// Order-preserving 64-bit key of a binary64 value (larger value <=> larger unsigned key).
__device__ __forceinline__ unsigned long long dkey(double d) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(d);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Packed selection key: the upper 51 bits of the logit's key, then 13 bits of (8191 - e), so
// that one unsigned compare orders by logit and breaks exact ties toward the lower index.
// Dropping 13 low mantissa bits merges logits that differ by less than ~2^-39 relative (about
// 1e-10 at |logit| = 64), far inside the 1e-6 band where either order is correct.
__device__ __forceinline__ unsigned long long pkey(double l, int e) {
  return (dkey(l) & ~0x1FFFull) | (unsigned long long)(0x1FFF - e);
}

// Word `sg` (column segment) of expert e's logit of unit u, polled until it carries the unit's
// tag; `bad` is set if the wait failed.
__device__ __forceinline__ double logit_part(const Prog& P, Smem* sm, const unsigned long long* lg,
                                             unsigned long long wd, size_t at, int u, bool& bad) {
  const unsigned long long want = tag13(u);
  if ((wd & kTag13) != want) {
    wd = await_word(P, sm, lg + at, kTag13, want, DE_TIMEOUT_ROUTE);
    bad = bad || (wd & kTag13) != want;
  }
  return logit_of(wd);
}

// Top-K of the unit's logits by the consumer warps, after every CTA's router rows are in.
// Warp w takes experts e = e0 + 32 w + lane + 32 W i (i = 0, 1; W consumer warps) of each
// block of 64 W experts: their binary64 logits (bias first, then the column-segment partials
// in order) and packed keys (pkey). Rounds of a warp maximum (two 32-bit reductions: high
// word, then low word among the lanes holding it; the lane holding the winner drops it)
// leave the warp's K best in lanes 0..K-1; further blocks' K best are merged into them the
// same way. The warps' candidates go to shared memory; after a consumer barrier warp 0 merges
// them and forms the weights w_k = exp(l_k - l_max) / sum_sel exp(l_j - l_max): the softmax
// over all experts followed by renormalisation over the selected ones, where the full softmax
// denominator cancels. Keys carry the index, so no two are equal; logits within ~2^-39
// relative of each other count as tied and go to the lower index.

// K rounds of a warp maximum over the M keys per lane; lane k < K ends with the k-th best key
// and its logit (others: 0).
template <int M>
__device__ __forceinline__ void warp_topk(int K, unsigned long long (&key)[M], double (&lv)[M],
                                          unsigned long long& out_key, double& out_l) {
  const int lane = threadIdx.x & 31;
  out_key = 0ull;
  out_l = 0.0;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    unsigned long long bk = key[0];
    int bi = 0;
#pragma unroll
    for (int i = 1; i < M; ++i)
      if (key[i] > bk) bk = key[i], bi = i;
    const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(bk >> 32));
    const unsigned lo =
        __reduce_max_sync(0xffffffffu, (unsigned)(bk >> 32) == hi ? (unsigned)bk : 0u);
    const unsigned long long win = ((unsigned long long)hi << 32) | lo;
    const bool mine = bk == win && win != 0ull;  // at most one lane holds it
    double l = 0.0;
#pragma unroll
    for (int i = 0; i < M; ++i) l = i == bi ? lv[i] : l;
    const unsigned holder = __ballot_sync(0xffffffffu, mine);
    const double wl = __shfl_sync(0xffffffffu, l, holder ? __ffs(holder) - 1 : 0);
    if (mine) {
#pragma unroll
      for (int i = 0; i < M; ++i) key[i] = i == bi ? 0ull : key[i];
    }
    if (lane == k) {
      out_key = win;
      out_l = wl;
    }
  }
}

__device__ __noinline__ bool topk_block(const Prog& P, const Geo& G, Smem* sm, int u,
                                        const unsigned long long* lg, const float* bias,
                                        int* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  bool bad = false;
  float gate_l = 0.f;
  // the shared-gate row's logit (sigma): its first word is loaded now, with the experts' words
  // below in flight beside it, and settled after them
  const bool gate_lane = w == 0 && lane == 0 && G.gate_on;
  const unsigned long long gate_w0 = gate_lane ? ld_relaxed_gpu_u64(lg + G.E) : 0ull;
  unsigned long long best_key = 0ull;  // lane k < K: the warp's k-th best so far
  double best_l = 0.0;
  constexpr int kBlock = 64 * kConsumerWarps;
#pragma unroll 1
  for (int e0 = 0; e0 < G.E; e0 += kBlock) {
    unsigned long long key[2];
    double lv[2];
    int ec[2];
    unsigned long long w0[2], w1[2];
    float bv[2];
    // words of the first two column segments of both experts: every load first, then one
    // wait for all of them
    const size_t s1 = G.rseg > 1 ? (size_t)G.nr : 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      ec[i] = min(e0 + 32 * w + lane + 32 * kConsumerWarps * i, G.E - 1);
      bv[i] = bias ? __ldcg(bias + ec[i]) : 0.f;
    }
    unsigned long long wd[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) wd[j] = ld_relaxed_gpu_u64(lg + (j >> 1) * s1 + ec[j & 1]);
    const int ec0 = ec[0], ec1 = ec[1];
    if (!settle<4>(P, sm, wd, [=](int j) { return lg + (j >> 1) * s1 + ((j & 1) ? ec1 : ec0); }, kTag13,
                   tag13(u), DE_TIMEOUT_ROUTE))
      bad = true;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      w0[i] = wd[i];
      w1[i] = wd[2 + i];
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int e = e0 + 32 * w + lane + 32 * kConsumerWarps * i;
      // the bias first, then the column-segment partials in order
      double l = (double)bv[i] + logit_of(w0[i]);
      if (G.rseg > 1) l += logit_of(w1[i]);
#pragma unroll 1
      for (int sg = 2; sg < G.rseg; ++sg) {
        const size_t at = (size_t)sg * G.nr + ec[i];
        l += logit_part(P, sm, lg, ld_relaxed_gpu_u64(lg + at), at, u, bad);
      }
      lv[i] = l;
      key[i] = e < G.E ? pkey(l, e) : 0ull;
    }
    unsigned long long bk;
    double bl;
    warp_topk<2>(G.K, key, lv, bk, bl);
    if (e0 == 0) {
      best_key = bk;
      best_l = bl;
    } else {  // merge the block's K best (lanes 0..K-1) into the running K best
      key[0] = best_key;
      lv[0] = best_l;
      key[1] = bk;
      lv[1] = bl;
      warp_topk<2>(G.K, key, lv, best_key, best_l);
    }
  }
  if (gate_lane) {
    double a = 0.0;
    a += logit_part(P, sm, lg, gate_w0, (size_t)G.E, u, bad);
#pragma unroll 1
    for (int sg = 1; sg < G.rseg; ++sg) {
      const size_t at = (size_t)sg * G.nr + G.E;
      a += logit_part(P, sm, lg, ld_relaxed_gpu_u64(lg + at), at, u, bad);
    }
    gate_l = (float)a;
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane < G.K) {
    sm->cand_key[w * kMaxK + lane] = best_key;
    sm->cand_l[w * kMaxK + lane] = best_l;
  }
  consumers_sync();
  if (w != 0) return bad;
  // merge: lane l holds candidates l + 32 i of the W K (missing ones are 0)
  constexpr int kM = (kConsumerWarps * kMaxK + 31) / 32;
  const int nc = kConsumerWarps * G.K;
  unsigned long long key[kM];
  double lv[kM];
#pragma unroll
  for (int i = 0; i < kM; ++i) {
    const int c = lane + 32 * i;
    const int wk = c / G.K, kk = c - wk * G.K;  // candidate kk of warp wk
    const bool ok = c < nc;
    key[i] = ok ? sm->cand_key[wk * kMaxK + kk] : 0ull;
    lv[i] = ok ? sm->cand_l[wk * kMaxK + kk] : 0.0;
  }
  unsigned long long sel_key;
  double sel_l;
  warp_topk<kM>(G.K, key, lv, sel_key, sel_l);
  const bool mine = lane < G.K;
  const int e = min(max(0x1FFF - (int)(sel_key & 0x1FFFull), 0), G.E - 1);
  const double l0 = __shfl_sync(0xffffffffu, sel_l, 0);
  const float ex = mine ? expf((float)(sel_l - l0)) : 0.f;
  float den = ex;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (mine) {
    const float wk = __fdividef(ex, den);
    sm->rt_e[u & 1][lane] = e;
    sm->rt_w[u & 1][lane] = wk;
    if (idx_out) idx_out[lane] = e;
    if (w_out) w_out[lane] = wk;
  }
  gate_l = __shfl_sync(0xffffffffu, gate_l, 0);
  if (lane == 0) sm->sigma[u & 1] = G.gate_on ? 1.f / (1.f + expf(-gate_l)) : 1.f;
  __syncwarp();
  if (lane == 0) signal_ready(&sm->rt_ready, &sm->rt_bar, (unsigned)(u + 1));
  return bad;
}

// ------------------------------------------------------------------------------------------
// digit form of a vector in shared memory (in place)
// ------------------------------------------------------------------------------------------
// A slice is 32 consecutive columns = 128 bytes of binary32 values. In digit form the same
// 128 bytes hold, as 16-byte chunks at position (i ^ (slice & 7)) (swizzled so that the 8
// lanes of a quarter-warp loading chunk i of 8 consecutive slices hit distinct banks):
//   chunks 0..5: digit plane p = i/2, words 4(i%2) .. 4(i%2)+3, one signed byte per column;
//   chunk 6:     {s, sum of the slice's values}.
// Word n of a plane pairs with the bytes the kernel cuts from the codes:
//   4 bits: word n = 2j + h holds columns 8j + 2b + h (b = 0..3): code word j's low nibbles
//           (h = 0) or its high nibbles, left in place as 16 q (h = 1);
//   2 bits: word n = 4j + p holds columns 16j + 4b + p: bit-pair p of code word j, left in
//           place as 4^p q.
// The digits of column c are those of q_c = rint(v_c * k / m_n) with k = 127 * 2^14 / max|v|
// and m_n the in-place factor of its word (1, 16, or 4^p), split exactly into
// q = d0 * 2^14 + d1 * 2^7 + d2; then sum over the slice of code * v ~ s * sum_p 2^(14-7p) *
// dp4a(codes, plane p) with s = max|v| / (127 * 2^14).
__device__ __forceinline__ int dslot(int s, int i) { return 32 * s + 4 * (i ^ (s & 7)); }

// Three signed 8-bit digits of q = rint(v * k) (|q| <= 127 * 2^14): q = d0 * 2^14 + d1 * 2^7
// + d2 with d0 in [-127, 127], d1 in [-64, 64], d2 in [-64, 63]. Adding 1.5 * 2^23 in the same
// fused operation leaves the rounded product in the low mantissa bits.
__device__ __forceinline__ void digits3(float v, float k, int& d0, int& d1, int& d2) {
  const int q = __float_as_int(fmaf(v, k, 12582912.f)) - 0x4B400000;
  d0 = (q + 8192) >> 14;
  const int r = q - (d0 << 14);
  d1 = (r + 64) >> 7;
  d2 = r - (d1 << 7);
}

// low bytes of four ints, in order, as one word
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return __byte_perm(__byte_perm((uint32_t)a, (uint32_t)b, 0x0040),
                     __byte_perm((uint32_t)c, (uint32_t)d, 0x0040), 0x5410);
}

// Column of byte b (b = 0..3) of digit word n of a slice (see the layout above).
template <int BITS>
__device__ __forceinline__ int word_col(int n, int b) {
  return BITS == 4 ? 8 * (n >> 1) + 2 * b + (n & 1) : 16 * (n >> 2) + 4 * b + (n & 3);
}

// Transform nsl slices of src (binary32, scaled by `scale`) into digit form in dst (dst may
// be src: in place), by nthr threads (tid = this thread's index among them, nthr a multiple of
// 32, the threads whole warps): 8 threads per slice, thread n of a slice making digit word n
// of the three planes from its four columns. The 8 threads of a slice are consecutive lanes of
// one warp, and every lane reads its values before any lane writes.
template <int BITS>
__device__ void transform(const float* src, float* dst, int nsl, float scale, int tid, int nthr) {
  const int items = nsl * 8;
  const int rounds = (items + nthr - 1) / nthr;
  uint32_t* base = reinterpret_cast<uint32_t*>(dst);
#pragma unroll 1
  for (int r = 0; r < rounds; ++r) {
    const int it = tid + nthr * r;
    const bool act = it < items;
    const int s = act ? it >> 3 : 0, n = it & 7;
    float v[4];
    float m = 0.f, sum = 0.f;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      v[b] = act ? src[32 * s + word_col<BITS>(n, b)] * scale : 0.f;
      m = fmaxf(m, fabsf(v[b]));
    }
    sum = (v[0] + v[1]) + (v[2] + v[3]);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    __syncwarp();
    if (act) {
      // the in-place factor of word n: 1 / 16 for high nibbles, 4^-p for bit-pair p
      const float fw = BITS == 4 ? ((n & 1) ? 0.0625f : 1.f)
                                 : ((n & 3) == 0 ? 1.f : (n & 3) == 1 ? 0.25f
                                                       : (n & 3) == 2 ? 0.0625f : 0.015625f);
      const float k = m > 0.f ? __fdividef(2080768.f, m) * fw : 0.f;
      int d[3][4];
#pragma unroll
      for (int b = 0; b < 4; ++b) digits3(v[b], k, d[0][b], d[1][b], d[2][b]);
#pragma unroll
      for (int p = 0; p < 3; ++p)
        base[dslot(s, 2 * p + (n >> 2)) + (n & 3)] = pack4(d[p][0], d[p][1], d[p][2], d[p][3]);
      if (n == 0)
        *reinterpret_cast<float2*>(base + dslot(s, 6)) = make_float2(m * (1.f / 2080768.f), sum);
    }
    __syncwarp();
  }
}

// The consumers' form: all 256 consumer threads, in place.
template <int BITS>
__device__ __forceinline__ void transform(float* buf, int nsl, float scale) {
  transform<BITS>(buf, buf, nsl, scale, (int)threadIdx.x - 32 * kCtrlWarps, kConsumers);
}

// The digit form of slice s of buf: xd[8p + n] = word n of plane p; {sc, sx}.
struct XDig {
  int d[24];
  float sc, sx;
};

__device__ __forceinline__ void load_digits(const float* buf, int s, XDig& x) {
#pragma unroll
  for (int i = 0; i < 6; ++i) {
    const uint4 a = *reinterpret_cast<const uint4*>(buf + dslot(s, i));
    x.d[4 * i] = (int)a.x; x.d[4 * i + 1] = (int)a.y; x.d[4 * i + 2] = (int)a.z;
    x.d[4 * i + 3] = (int)a.w;
  }
  const float2 b = *reinterpret_cast<const float2*>(buf + dslot(s, 6));
  x.sc = b.x;
  x.sx = b.y;
}

// The binary32 values of slice s of buf, scaled (the literal and naive forms).
struct XVal {
  float v[32];
};

__device__ __forceinline__ void load_values(const float* buf, int s, float scale, XVal& x) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 a = *reinterpret_cast<const float4*>(buf + 32 * s + 4 * q);
    x.v[4 * q] = a.x * scale; x.v[4 * q + 1] = a.y * scale;
    x.v[4 * q + 2] = a.z * scale; x.v[4 * q + 3] = a.w * scale;
  }
}

// ------------------------------------------------------------------------------------------
// controller warp
// ------------------------------------------------------------------------------------------
// Bring `bytes` from global memory (written by other CTAs or by the caller) into shared
// memory with one bulk copy issued by lane 0 on `bar`.
__device__ __forceinline__ void copy_in(void* dst, const void* src, unsigned bytes,
                                        uint64_t* bar) {
  if ((threadIdx.x & 31) == 0) {
    fence_proxy_async();  // order earlier generic accesses before the async-proxy copy
    mbar_arrive_expect_tx(bar, bytes);
    tma_load_1d(dst, src, bytes, bar);
  }
  __syncwarp();
}

__device__ __forceinline__ bool wait_copy(const Prog& P, Smem* sm, uint64_t* bar,
                                          unsigned& phase) {
  const bool ok = warp_wait_mbar(P, sm, bar, phase, DE_TIMEOUT_DEP);
  phase ^= 1u;
  return ok;
}

// Whole warp: the n tagged value words of unit u at src into dst as binary32, 16 words per
// lane in flight; each word polled until it carries the unit's tag. False if a wait failed.
__device__ __noinline__ bool fetch_values(const Prog& P, Smem* sm, const unsigned long long* src,
                                          float* dst, int n, int u, int code) {
  const int lane = threadIdx.x & 31;
  const unsigned long long want = tag32(u);
  bool ok = true;
#pragma unroll 1
  for (int b = 0; b < n; b += 32 * 16) {
    const unsigned long long* sb = src + b + lane;
    const int lim = n - 1 - b - lane;  // words j with 32 j <= lim are inside the vector
    unsigned long long v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = ld_relaxed_gpu_u64(sb + min(32 * j, lim));
    ok = settle<16>(P, sm, v, [=](int j) { return sb + min(32 * j, lim); }, kTag32, want, code) &&
         ok;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (32 * j <= lim) dst[b + lane + 32 * j] = value_of(v[j]);
  }
  return __all_sync(0xffffffffu, ok);
}

__device__ void controller(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm, bool need_h) {
  const int lane = threadIdx.x & 31;
  float* XB = reinterpret_cast<float*>(smem + G.o_x);
  float* HB = reinterpret_cast<float*>(smem + G.o_h);
  unsigned px = 0;          // phase of the x copy barrier
  bool x_issued = false;    // the next unit's x copy is already in flight
  const bool x_digits = G.shared_on || G.routed_on;
#pragma unroll 1
  for (int u = 0; u < P.n_units; ++u) {
    const UnitView uv = unit_view(P, G, u);
    const bool owner = (u % (int)gridDim.x) == (int)blockIdx.x;
    FMOE_MARK(u, MK_C_UNIT);
    // ---- x(u) from an input buffer. Independent tokens with expert rows: unit u starts once
    // every CTA has finished unit u-2 (the logit and h buffers alternate between units and
    // every word carries its unit, so a CTA one unit ahead overwrites only words of unit u-2,
    // which no CTA reads any more; this CTA's x buffer is refilled only after its consumers
    // freed it). Otherwise (router only, whose x copy nothing else orders after the
    // consumers' reads; a stack's first layer) once unit u-1 is done everywhere. Stack layers
    // after the first read the previous layer's words in the consumers.
    if (uv.xin) {
      const int lag = P.mode == MODE_SEQ && x_digits ? 2 : 1;
      if (u >= lag && !warp_wait_done(P, sm, (unsigned)(u + 1 - lag), DE_TIMEOUT_DEP)) break;
      FMOE_MARK(u, MK_C_PREV_DONE);
      if (!x_issued) copy_in(XB, uv.xin, 4u * (unsigned)G.H, &sm->xbar);
      x_issued = false;
      if (!wait_copy(P, sm, &sm->xbar, px)) break;
      FMOE_MARK(u, MK_C_X);
      if (owner && uv.h_trace)
#pragma unroll 1
        for (int c = lane * 4; c < G.H; c += 128)
          *reinterpret_cast<float4*>(uv.h_trace + c) = *reinterpret_cast<const float4*>(XB + c);
      if (lane == 0) {
        sm->xf[u & 1] = 1.f;
        signal_ready(&sm->x_ready, &sm->x_bar, (unsigned)(u + 1));
      }
      __syncwarp();
    }
    if (G.route_on && uv.bias)  // the unit's logit bias into L2 while the router runs
#pragma unroll 1
      for (int e = lane * 32; e < G.E; e += 32 * 32) prefetch_l2(uv.bias + e);

    // ---- independent tokens: the next unit's x, once the consumers hold this unit's x
    // digits in registers (its computation still waits for this unit to complete)
    if (P.mode == MODE_SEQ && x_digits && u + 1 < P.n_units) {
      if (!warp_wait_ready(P, sm, &sm->xfree, &sm->xfree_bar, (unsigned)(u + 1), DE_TIMEOUT_DEP))
        break;
      FMOE_MARK(u, MK_C_XFREE);
      copy_in(XB, P.x + (size_t)(u + 1) * G.H, 4u * (unsigned)G.H, &sm->xbar);
      x_issued = true;
    }
    if (G.nseg == 0 || !need_h) continue;  // (no output rows: no h needed)
    // the h buffer is refilled only after this CTA's consumers have left unit u-1 (they hold
    // unit u's x): without a router nothing else orders the two
    if (!warp_wait_ready(P, sm, &sm->xfree, &sm->xfree_bar, (unsigned)(u + 1), DE_TIMEOUT_DEP))
      break;
    // ---- h of unit u, segment by segment (shared expert, then routed k), as its words arrive
    bool ok = true;
#pragma unroll 1
    for (int sg = 0; sg < G.nseg && ok; ++sg) {
      const bool sh = G.shared_on && sg == 0;
      const int k = sg - G.shared_on;
      ok = fetch_values(P, sm, P.s.hx + ((size_t)uv.slot * G.nseg + sg) * G.I,
                        HB + (size_t)sg * G.I, G.I, u, DE_TIMEOUT_DEP);
      if (!ok) break;
      FMOE_MARK(u, sh ? MK_C_HS : MK_C_HK + k);
      if (lane == 0) {
        if (sh) signal_ready(&sm->hs_ready, &sm->hs_bar, (unsigned)(u + 1));
        else signal_ready(&sm->hk_ready, &sm->hk_bar, (unsigned)(u * G.K + k + 1));
      }
      __syncwarp();
    }
    if (!ok) break;
  }
  // never leave with a copy in flight
  if (x_issued && lane == 0) {
    const uint64_t deadline = global_ns() + 100000000ull;
    while (!mbar_try_wait(&sm->xbar, px))
      if (global_ns() > deadline) break;
  }
}

// ------------------------------------------------------------------------------------------
// one row x one 32-column slice
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// s * sum(q x) + z * sum(x) over the slice: codes at `ca`, scale/bias word `sbw`.
template <int BITS>
__device__ __forceinline__ float slice_dot(const uint8_t* ca, uint32_t sbw, const XDig& x) {
  int c0 = 0, c1 = 0, c2 = 0;
  if constexpr (BITS == 4) {
    const uint4 q = *reinterpret_cast<const uint4*>(ca);
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = qw[j] & 0x0F0F0F0Fu, hi = qw[j] & 0xF0F0F0F0u;
      c0 = dp4a_us(hi, x.d[2 * j + 1], dp4a_us(lo, x.d[2 * j], c0));
      c1 = dp4a_us(hi, x.d[8 + 2 * j + 1], dp4a_us(lo, x.d[8 + 2 * j], c1));
      c2 = dp4a_us(hi, x.d[16 + 2 * j + 1], dp4a_us(lo, x.d[16 + 2 * j], c2));
    }
  } else {
    const uint2 q = *reinterpret_cast<const uint2*>(ca);
    const uint32_t qw[2] = {q.x, q.y};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint32_t cp = qw[j] & (0x03030303u << (2 * p));
        c0 = dp4a_us(cp, x.d[4 * j + p], c0);
        c1 = dp4a_us(cp, x.d[8 + 4 * j + p], c1);
        c2 = dp4a_us(cp, x.d[16 + 4 * j + p], c2);
      }
    }
  }
  const int tq = c0 * 16384 + c1 * 128 + c2;
  const float s = __uint_as_float(sbw << 16);
  const float z = __uint_as_float(sbw & 0xFFFF0000u);
  return fmaf(s * x.sc, (float)tq, z * x.sx);
}

// The code of column c of a slice from its code words (lowest column in the lowest bits).
template <int BITS>
__device__ __forceinline__ float code_at(const uint32_t* qw, int c) {
  constexpr int per = 32 / BITS;
  return (float)((qw[c / per] >> (BITS * (c % per))) & ((1u << BITS) - 1u));
}

// The pages' literal FMA form per weight: sum over the slice of fma(q, s*x, z*x).
template <int BITS>
__device__ __forceinline__ float slice_dot_fma(const uint8_t* ca, uint32_t sbw, const XVal& x) {
  uint32_t qw[4];
  if constexpr (BITS == 4) {
    const uint4 q = *reinterpret_cast<const uint4*>(ca);
    qw[0] = q.x; qw[1] = q.y; qw[2] = q.z; qw[3] = q.w;
  } else {
    const uint2 q = *reinterpret_cast<const uint2*>(ca);
    qw[0] = q.x; qw[1] = q.y; qw[2] = 0u; qw[3] = 0u;
  }
  const float s = __uint_as_float(sbw << 16);
  const float z = __uint_as_float(sbw & 0xFFFF0000u);
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    a0 = a0 + fmaf(code_at<BITS>(qw, c), s * x.v[c], z * x.v[c]);
    a1 = a1 + fmaf(code_at<BITS>(qw, c + 1), s * x.v[c + 1], z * x.v[c + 1]);
  }
  return a0 + a1;
}

// The naive form per weight: sum over the slice of (q*s + z) * x.
template <int BITS>
__device__ __forceinline__ float slice_dot_naive(const uint8_t* ca, uint32_t sbw, const XVal& x) {
  uint32_t qw[4];
  if constexpr (BITS == 4) {
    const uint4 q = *reinterpret_cast<const uint4*>(ca);
    qw[0] = q.x; qw[1] = q.y; qw[2] = q.z; qw[3] = q.w;
  } else {
    const uint2 q = *reinterpret_cast<const uint2*>(ca);
    qw[0] = q.x; qw[1] = q.y; qw[2] = 0u; qw[3] = 0u;
  }
  const float s = __uint_as_float(sbw << 16);
  const float z = __uint_as_float(sbw & 0xFFFF0000u);
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    a0 = a0 + __fmul_rn(__fadd_rn(__fmul_rn(code_at<BITS>(qw, c), s), z), x.v[c]);
    a1 = a1 + __fmul_rn(__fadd_rn(__fmul_rn(code_at<BITS>(qw, c + 1), s), z), x.v[c + 1]);
  }
  return a0 + a1;
}

template <int BITS, int FORM, typename XT>
__device__ __forceinline__ float slice_any(const uint8_t* ca, uint32_t sbw, const XT& x) {
  if constexpr (FORM == FORM_DIGITS)
    return slice_dot<BITS>(ca, sbw, x);
  else if constexpr (FORM == FORM_FMA)
    return slice_dot_fma<BITS>(ca, sbw, x);
  else
    return slice_dot_naive<BITS>(ca, sbw, x);
}

template <int FORM>
struct XOf {
  using T = XVal;
};
template <>
struct XOf<FORM_DIGITS> {
  using T = XDig;
};

// ------------------------------------------------------------------------------------------
// reductions
// ------------------------------------------------------------------------------------------
// Transposing butterfly over `width` lanes (a power of two <= 32, the lane's segment): NR row
// partials per lane become one fully reduced value per row; store(i, v) is called for row i
// on exactly one lane of the segment.
template <int NR, typename T, typename Store>
__device__ __forceinline__ void seg_reduce(T (&v)[NR], int lane_in_seg, int width, Store store) {
  int lo = 0;
  int nlive = NR;
#pragma unroll
  for (int i = 0; (1 << i) < NR; ++i) {
    const int o = 1 << i;
    const int half = (NR >> i) >> 1;
    if (o < width) {
      const bool upper = (lane_in_seg & o) != 0;
#pragma unroll
      for (int a = 0; a < (NR >> 1); ++a) {
        if (a < half) {
          const T send = upper ? v[a] : v[a + half];
          const T keep = upper ? v[a + half] : v[a];
          v[a] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      if (upper) lo += half;
      nlive = half;
    }
  }
  if (nlive == 1) {
#pragma unroll 1
    for (int o = NR; o < width; o <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    if (lane_in_seg < NR && lane_in_seg < width) store(lo, v[0]);
  } else {
#pragma unroll
    for (int a = 0; a < NR; ++a)
      if (a < nlive) store(lo + a, v[a]);
  }
}

// ------------------------------------------------------------------------------------------
// consumer warps
// ------------------------------------------------------------------------------------------
// A ring of stages (ring A or ring B); the consumers' count of chunks taken from each ring is
// kept in registers beside it. Copied by value (never addressed) so that it stays in registers.
struct Ring {
  uint8_t* base;
  uint64_t* full;
  uint64_t* empty;
  int ns;
  int slot0;       // first chunk_arrive / red slot of this ring
};

__device__ __forceinline__ const uint8_t* ring_stage(const Geo& G, const Ring& R, unsigned use) {
  return R.base + (size_t)(use % (unsigned)R.ns) * G.stage_bytes;
}
__device__ __forceinline__ uint64_t* ring_empty(const Ring& R, unsigned use) {
  return &R.empty[use % (unsigned)R.ns];
}
__device__ __forceinline__ int ring_slot(const Ring& R, unsigned use) {
  return R.slot0 + (int)(use % (unsigned)R.ns);
}
// Wait (whole warp) for chunk `use` of the ring to have landed.
__device__ __forceinline__ void ring_wait(const Prog& P, Smem* sm, const Ring& R, unsigned use,
                                          bool& dead) {
  if (!dead && !warp_wait_mbar(P, sm, &R.full[use % (unsigned)R.ns], (use / (unsigned)R.ns) & 1u,
                               DE_TIMEOUT_FULL))
    dead = true;
}

// Every warp arrives once per chunk use of a stage; the warp that completes the count of 8
// returns true (it has acquired every other warp's writes of the chunk) and resets it.
__device__ __forceinline__ bool chunk_last(Smem* sm, int slot) {
  int last = 0;
  if ((threadIdx.x & 31) == 0) {
    const unsigned old = atom_add_acq_rel_cta_smem(&sm->chunk_arrive[slot], 1u);
    last = old == (unsigned)(kConsumerWarps - 1);
    if (last) atom_exch_cta_smem(&sm->chunk_arrive[slot], 0u);
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  __syncwarp();
  return last != 0;
}

__device__ __forceinline__ void release_stage(uint64_t* empty) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
}

// Router rows of a chunk: binary64 sums of fp32 products over the chunk's columns; each
// thread takes float4 columns t, t + 256, ...; per row a warp reduction, the 8 warp
// partials through shared memory, summed in warp order by the chunk's last warp.
// The x columns (float4 group f) of router segment `seg`, converted to binary64.
struct X4 {
  double a, b, c, d;
};

__device__ __forceinline__ X4 router_x4(const Geo& G, const float* XB, int seg, int f) {
  const float4 v = reinterpret_cast<const float4*>(XB + (size_t)seg * G.rcols)[f];
  return X4{(double)v.x, (double)v.y, (double)v.z, (double)v.w};
}

// four products of a float4 group of weights with x, the weights converted to binary64 (the
// products are exact), accumulated in binary64 onto `acc`
__device__ __forceinline__ double dot4(const float4 wv, const X4& x, double acc) {
  acc = fma((double)wv.x, x.a, acc);
  acc = fma((double)wv.y, x.b, acc);
  acc = fma((double)wv.z, x.c, acc);
  return fma((double)wv.w, x.d, acc);
}

// Whole router rows, up to kRouterBatch of them from consecutive chunks of G.rrows rows each
// (row r of the batch is row r % rrows of chunk use0 + r / rrows): each thread takes float4
// columns t + 256 j of every row, x converted once per column group, one independent binary64
// chain per row; one transposing warp reduction for all rows; the warp partials through
// shared memory, summed in warp order by the batch's last warp, which stores the logits.
__device__ __forceinline__ void router_batch(const Prog& P, const Geo& G, Smem* sm, int u,
                                             int r0, int nrows, int nchunks, const Ring& R,
                                             unsigned use0, double* red, const float* XB) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  const int t = w * 32 + lane;
  const int nf = G.rcols / 4;
  const float4* ws[kRouterBatch];
#pragma unroll
  for (int r = 0; r < kRouterBatch; ++r) {
    const int rr = r < nrows ? r : 0;
    const int q = rr / G.rrows;
    ws[r] = reinterpret_cast<const float4*>(ring_stage(G, R, use0 + (unsigned)q)) +
            (size_t)(rr - q * G.rrows) * nf;
  }
  double v[kRouterBatch];
#pragma unroll
  for (int r = 0; r < kRouterBatch; ++r) v[r] = 0.0;
  // every x and weight group of this thread loaded first (clamped to a valid group; the
  // clamped ones are not used), then the binary64 chains in the same order as one at a time
  float4 xv[4], wv[4][kRouterBatch];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int f = min(t + kConsumers * j, nf - 1);
    xv[j] = reinterpret_cast<const float4*>(XB)[f];
#pragma unroll
    for (int r = 0; r < kRouterBatch; ++r) wv[j][r] = ws[r][f];
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (t + kConsumers * j < nf) {
      const X4 x{(double)xv[j].x, (double)xv[j].y, (double)xv[j].z, (double)xv[j].w};
#pragma unroll
      for (int r = 0; r < kRouterBatch; ++r)
        if (r < nrows) v[r] = dot4(wv[j][r], x, v[r]);
    }
  }
  FMOE_MARK_W(u, MK_R_DOT, MK_R_DOT_W);
  const int slot = ring_slot(R, use0);
  double* rs = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(red) + (size_t)slot * G.red_slot);
  seg_reduce<kRouterBatch>(v, lane, 32, [&](int r, double x) {
    if (r < nrows) rs[r * kConsumerWarps + w] = x;
  });
  FMOE_MARK_W(u, MK_R_RED, MK_R_RED_W);
  const bool last = chunk_last(sm, slot);
  FMOE_MARK_W(u, MK_R_LAST, MK_R_LAST_W);
  if (last) {
    const double xf = (double)sm->xf[u & 1];
    unsigned long long* lg = P.s.logits + (size_t)(u & 1) * G.rseg * G.nr + r0;
    if (lane < nrows && !(P.debug & 1)) {  // debug bit 0: the logits are never written
      double x = 0.0;
#pragma unroll
      for (int q = 0; q < kConsumerWarps; ++q) x += rs[lane * kConsumerWarps + q];
      st_relaxed_gpu_u64(lg + lane, logit_word(x * xf, u));  // norm factor applied to the sum
    }
    FMOE_MARK(u, MK_R_PUB);
  }
#pragma unroll 1
  for (int q = 0; q < nchunks; ++q) release_stage(ring_empty(R, use0 + (unsigned)q));
}

__device__ __forceinline__ bool router_chunk(const Prog& P, const Geo& G, Smem* sm,
                                             const Chunk& c, int u, const uint8_t* stage,
                                             uint64_t* empty, int slot, double* red,
                                             const float* XB) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  const int t = w * 32 + lane;
  const int nf = G.rcols / 4;
  const float4* ws = reinterpret_cast<const float4*>(stage);
  double* rs = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(red) + (size_t)slot * G.red_slot);
#pragma unroll 1
  for (int r = 0; r < c.n; ++r) {
    double a = 0.0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int f = t + kConsumers * j;
      if (f < nf) a = dot4(ws[(size_t)r * nf + f], router_x4(G, XB, c.seg, f), a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) rs[r * kConsumerWarps + w] = a;
  }
  const bool last = chunk_last(sm, slot);
  if (last) {
    const double xf = (double)sm->xf[u & 1];
    unsigned long long* lg = P.s.logits + ((size_t)(u & 1) * G.rseg + c.seg) * G.nr + c.r0;
#pragma unroll 1
    for (int r = lane; r < c.n && !(P.debug & 1); r += 32) {
      double a = 0.0;
#pragma unroll
      for (int q = 0; q < kConsumerWarps; ++q) a += rs[r * kConsumerWarps + q];
      st_relaxed_gpu_u64(lg + r, logit_word(a * xf, u));  // norm factor applied to the sum
    }
  }
  release_stage(empty);
  return true;
}

// Gate/up rows of up to two chunks of one expert at once (a "pass"): chunk c's stage holds hr
// gate rows then hr up rows (n_c valid each); row slot q = 2 hr c + rho. Thread (group g,
// slice s) takes slots g + gh i (i < NR); every slot reads a copied row (row 0 of chunk 0
// stands in for slots without a valid row), so the loads and products of all NR slots are
// issued without branches. Partial sums are reduced over the row's threads (lanes of its
// segment, then warps through shared memory); the pass's last warp applies SwiGLU and stores
// the h values as tagged words of unit u. `tr` marks the pass traced by a profiling build.
template <int BITS, int FORM, int NR>
__device__ __forceinline__ void gu_pass(const Prog& P, const Geo& G, Smem* sm, int np,
                                        const Chunk& c0, const Chunk& c1, const Ring& R,
                                        unsigned use0, float* red,
                                        const typename XOf<FORM>::T& x, unsigned long long* h,
                                        int u, bool tr) {
  const uint8_t* st0 = ring_stage(G, R, use0);
  const uint8_t* st1 = ring_stage(G, R, use0 + (unsigned)(np - 1));
  const int slot = ring_slot(R, use0);
  const int lane = threadIdx.x & 31;
  const int t = (int)threadIdx.x - 32 * kCtrlWarps;
  const int g = t / G.wh, s = t - g * G.wh;
  const bool act = g < G.gh && s < G.sh;
  const int sc = act ? s : 0;
  const int hr = G.hr;
  constexpr unsigned cb = BITS == 4 ? 16u : 8u;
  const unsigned sbo = 2u * (unsigned)hr * G.rc_h;  // offset of the sb words in a stage
  float acc[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int q = g + G.gh * i;
    const int c = q >= 2 * hr ? 1 : 0;
    const int rho = q - 2 * hr * c;
    const int rr = rho < hr ? rho : rho - hr;
    const bool ok = act && c < np && rr < (c ? c1.n : c0.n);
    const int rc = ok ? rho : 0;
    const uint8_t* st = (ok && c) ? st1 : st0;
    const uint32_t sbw =
        reinterpret_cast<const uint32_t*>(st + sbo)[(unsigned)rc * (G.rs_h >> 2) + (sc >> 1)];
    const float v = slice_any<BITS, FORM>(st + (unsigned)rc * G.rc_h + (unsigned)sc * cb, sbw, x);
    acc[i] = ok ? v : 0.f;
  }
  if (tr) FMOE_MARK_W(u, MK_G_DOT, MK_G_DOT_W);
  // the stages are no longer read: reduce over the row's threads
  const int width = G.wh < 32 ? G.wh : 32;
  const int wn = G.wh > 32 ? G.wh / 32 : 1;  // warps per row group
  const int om = G.wh > 32 ? s >> 5 : 0;     // this warp's index within its group
  float* rs = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(red) + (size_t)slot * G.red_slot);
  seg_reduce<NR>(acc, lane & (width - 1), width, [&](int i, float v) {
    const int q = g + G.gh * i;
    if (act && q < 2 * hr * np) rs[q * wn + om] = v;
  });
  if (tr) FMOE_MARK_W(u, MK_G_RED, MK_G_RED_W);
  const bool last = chunk_last(sm, slot);
  if (tr) FMOE_MARK_W(u, MK_G_LAST, MK_G_LAST_W);
  if (last) {
#pragma unroll 1
    for (int c = 0; c < np; ++c) {
      const int n = c ? c1.n : c0.n, r0 = c ? c1.r0 : c0.r0;
#pragma unroll 1
      for (int i = lane; i < n; i += 32) {
        float a = 0.f, b = 0.f;
#pragma unroll 1
        for (int q = 0; q < wn; ++q) {
          a += rs[(2 * hr * c + i) * wn + q];
          b += rs[(2 * hr * c + hr + i) * wn + q];
        }
        // SwiGLU: SiLU(gate) * up
        st_relaxed_gpu_u64(h + r0 + i, value_word(__fdividef(a, 1.f + __expf(-a)) * b, u));
      }
    }
    if (tr) FMOE_MARK(u, MK_G_PUB);
  }
  if (tr && last) FMOE_MARK(u, MK_G_EPI_END);
  release_stage(ring_empty(R, use0));
  if (np > 1) release_stage(ring_empty(R, use0 + 1));
}

// Down rows of a chunk (one expert segment): rows rho = w * P_i + lane_p + 8 P_i i of the
// stage's dr rows (n valid); lane_s takes slices lane_s + W_i j of the segment's digit form in
// the h buffer. Row totals are added to the CTA's output accumulators oacc (one per output
// row of the share; each row always handled by the same lane).
template <int BITS, int FORM, int NR>
__device__ __forceinline__ void dn_chunk(const Geo& G, const Chunk& c, const uint8_t* stage,
                                         uint64_t* empty, const float* hseg, float hscale,
                                         float* oacc, int d0) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  const int lane_s = lane & (G.wi - 1), lane_p = lane / G.wi;
  const int n = c.n;
  constexpr unsigned cb = BITS == 4 ? 16u : 8u;
  const uint32_t* sbb = reinterpret_cast<const uint32_t*>(stage + (unsigned)G.dr * G.rc_i);
  float acc[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) acc[i] = 0.f;
#pragma unroll 1
  for (int j = 0; j < G.ji; ++j) {
    const int s = lane_s + G.wi * j;
    const bool sok = s < G.si;
    const int sc = sok ? s : 0;
    typename XOf<FORM>::T x;
    if constexpr (FORM == FORM_DIGITS)
      load_digits(hseg, sc, x);
    else
      load_values(hseg, sc, hscale, x);
    const uint8_t* code0 = stage + (unsigned)sc * cb;
    const uint32_t* sbp = sbb + (sc >> 1);
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int rho = w * G.pi + lane_p + kConsumerWarps * G.pi * i;
      const bool ok = sok && rho < n;
      const int rc = ok ? rho : 0;  // row 0 stands in for slots without a valid row
      const uint32_t sbw = sbp[(unsigned)rc * (G.rs_i >> 2)];
      const float v = slice_any<BITS, FORM>(code0 + (unsigned)rc * G.rc_i, sbw, x);
      acc[i] += ok ? v : 0.f;
    }
  }
  release_stage(empty);
  const int r_off = c.r0 - d0;
  seg_reduce<NR>(acc, lane_s, G.wi, [&](int i, float v) {
    const int rho = w * G.pi + lane_p + kConsumerWarps * G.pi * i;
    if (rho < n) oacc[r_off + rho] += v;
  });
}

// Stack layers after the first: x is the previous unit's output, read as its tagged words by
// the 256 consumer threads (each word polled until it carries that unit's tag) into the x
// buffer; the norm factor 1 / sqrt(mean(x^2) + eps) from a binary64 sum of squares taken in
// the same order in every CTA; the owner CTA records x before the norm. While the words are
// in flight, warp 0 also waits for every CTA's unit-done word of the previous unit: CTAs that
// own no output rows write no words, and this keeps every CTA within one unit of the others
// (the exchange buffers are reused every second unit). False (this warp) if a wait failed.
__device__ __noinline__ bool fetch_x(const Prog& P, const Geo& G, Smem* sm,
                                     const unsigned long long* xw, float* h_trace, int u,
                                     float* XB, double* red) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  const int t = w * 32 + lane;
  const unsigned long long want = tag32(u - 1);
  bool bad = false;
  double ss = 0.0;
#pragma unroll 1
  for (int b = 0; b < G.H; b += kConsumers * 16) {
    unsigned long long v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = ld_relaxed_gpu_u64(xw + min(b + t + kConsumers * j, G.H - 1));
    if (b == 0 && w == 0) bad = !warp_wait_done(P, sm, (unsigned)u, DE_TIMEOUT_DEP);
    const int H = G.H;
    if (!settle<16>(P, sm, v, [=](int j) { return xw + min(b + t + kConsumers * j, H - 1); },
                    kTag32, want, DE_TIMEOUT_DEP))
      bad = true;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int i = b + t + kConsumers * j;
      if (i < G.H) {
        const float x = value_of(v[j]);
        XB[i] = x;
        if (h_trace) h_trace[i] = x;
        ss = fma((double)x, (double)x, ss);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[w] = ss;
  consumers_sync();
  if (t == 0) {
    double a = 0.0;
#pragma unroll
    for (int q = 0; q < kConsumerWarps; ++q) a += red[q];
    sm->xf[u & 1] = (float)(1.0 / sqrt(a / (double)G.H + (double)P.eps));
  }
  consumers_sync();
  return !__any_sync(0xffffffffu, bad);
}

template <int BITS, int FORM, int NRG, int NRD>
__device__ void consumer(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm, const Share& S) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  const int t = w * 32 + lane;
  float* XB = reinterpret_cast<float*>(smem + G.o_x);
  float* HB = reinterpret_cast<float*>(smem + G.o_h);
  float* red = reinterpret_cast<float*>(smem + G.o_red);
  float* oacc = reinterpret_cast<float*>(smem + G.o_oacc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G.o_bar);
  const Ring A{smem + G.o_ringA, bars, bars + G.nA, G.nA, 0};
  const Ring B{smem + G.o_ringB, bars + 2 * G.nA, bars + 2 * G.nA + G.nB, G.nB, G.nA};
  unsigned a_used = 0, b_used = 0;  // chunks taken from each ring so far
  const int gslice = t % G.wh;           // this thread's x slice in gate/up rows
  const bool gu_on = G.shared_on || G.routed_on;
  // A wait that fails (its budget ran out, or the CTA aborted) marks the warp dead: it skips
  // every later wait but keeps walking the same sequence of chunks and consumer barriers as
  // the other warps, so that no warp is left at a barrier; the results are then undefined and
  // the error word reports the failure.
  bool dead = false;
  typename XOf<FORM>::T xg;              // x of this thread's slice (digits or values)
#pragma unroll 1
  for (int u = 0; u < P.n_units; ++u) {
    const int slot_u = u & 1;
    if (P.mode == MODE_STACK && u % P.n_layers != 0) {
      const UnitView uv = unit_view(P, G, u);
      const bool owner = (u % (int)gridDim.x) == (int)blockIdx.x;
      if (!fetch_x(P, G, sm, uv.xw, owner ? uv.h_trace : nullptr, u, XB,
                   reinterpret_cast<double*>(red)))
        dead = true;
    } else if (!dead && !warp_wait_ready(P, sm, &sm->x_ready, &sm->x_bar, (unsigned)(u + 1),
                                         DE_TIMEOUT_DEP)) {
      dead = true;
    }
    if (t == 0 && !G.route_on) sm->sigma[slot_u] = 1.f;
    if (w == 0) FMOE_MARK(u, MK_K_X);
    // ---- router rows: whole rows in batches of up to kRouterBatch rows, else chunk by chunk
    if (G.route_on && S.nrc > 0) {
      if (G.rseg == 1 && G.rrows <= kRouterBatch) {
        const int cmax = max(1, min(kRouterBatch / G.rrows, A.ns));  // chunks per batch
#pragma unroll 1
        for (int i0 = 0; i0 < S.nrc; i0 += cmax) {
          const int nc = min(cmax, S.nrc - i0);
#pragma unroll 1
          for (int q = 0; q < nc; ++q) ring_wait(P, sm, A, a_used + (unsigned)q, dead);
          const int rb = S.r0 + i0 * G.rrows;
          router_batch(P, G, sm, u, rb, min(nc * G.rrows, S.r1 - rb), nc, A, a_used,
                       reinterpret_cast<double*>(red), XB);
          a_used += (unsigned)nc;
        }
      } else {
#pragma unroll 1
        for (int i = 0; i < S.nrc; ++i) {
          const Chunk c = chunk_a(G, S, i);
          ring_wait(P, sm, A, a_used, dead);
          router_chunk(P, G, sm, c, u, ring_stage(G, A, a_used), ring_empty(A, a_used),
                       ring_slot(A, a_used), reinterpret_cast<double*>(red), XB);
          ++a_used;
        }
      }
    }
    if (w == 0) FMOE_MARK(u, MK_K_ROUTER);
    // ---- x of this thread's slice: digit form (in place, after every router read of x)
    if (gu_on) {
      if constexpr (FORM == FORM_DIGITS) {
        consumers_sync();
        transform<BITS>(XB, G.sh, sm->xf[slot_u]);
        consumers_sync();
        load_digits(XB, gslice < G.sh ? gslice : 0, xg);
      } else {
        consumers_sync();
        load_values(XB, gslice < G.sh ? gslice : 0, sm->xf[slot_u], xg);
      }
      // the x buffer and the digit form are free once every warp holds its slice
      if (lane == 0) {
        const unsigned old = atom_add_acq_rel_cta_smem(&sm->xd_arrive, 1u);
        if (old == (unsigned)(kConsumerWarps * (u + 1) - 1))
          signal_ready(&sm->xfree, &sm->xfree_bar, (unsigned)(u + 1));
      }
      __syncwarp();
      if (w == 0) FMOE_MARK(u, MK_K_XD);
    }
    // ---- gate/up rows, in passes of up to gpass chunks: the shared expert (ring A) first,
    // while the other CTAs' logits arrive; then the routing decision; then routed expert k
    // (ring B) in turn
    const int jobs = gu_on ? G.shared_on + (G.routed_on ? G.K : 0) : 0;
#pragma unroll 1
    for (int phase = 0; phase < 2; ++phase) {
      if (phase == 1) {
        // ---- routing decision: from every CTA's logit words of the unit, as they arrive
        if (G.route_on) {
          if (w == 0) FMOE_MARK(u, MK_C_S1);
          const UnitView uv = unit_view(P, G, u);
          const bool owner = (u % (int)gridDim.x) == (int)blockIdx.x;
          if (topk_block(P, G, sm, u, P.s.logits + (size_t)slot_u * G.rseg * G.nr, uv.bias,
                         owner ? uv.idx_out : nullptr, owner ? uv.w_out : nullptr))
            dead = true;
          if (w == 0) issue_first_b(P, G, S, smem, sm, u);
          consumers_sync();
          if (w == 0) FMOE_MARK(u, MK_C_RT);
        }
        if (G.nseg == 0 && t == 0) unit_done(P, u);  // no output rows: the unit ends here
      }
      const int j0 = phase == 0 ? 0 : G.shared_on;
      const int j1 = phase == 0 ? min(G.shared_on, jobs) : jobs;
#pragma unroll 1
      for (int job = j0; job < j1; ++job) {
        const bool sh = G.shared_on && job == 0;
        const int k = job - G.shared_on;  // routed expert slot
        if (w == 0 && k == 1) FMOE_MARK(u, MK_J1_TOP);
        unsigned long long* hdst = P.s.hx + ((size_t)slot_u * G.nseg + job) * G.I;
        const Ring R = sh ? A : B;
        unsigned use = sh ? a_used : b_used;
#pragma unroll 1
        for (int i0 = 0; i0 < S.ngc; i0 += G.gpass) {
          const int np = min(G.gpass, S.ngc - i0);
          const Chunk c0 = sh ? chunk_a(G, S, S.nrc + i0) : chunk_b(G, S, k * S.ngc + i0);
          const Chunk c1 = sh ? chunk_a(G, S, S.nrc + i0 + np - 1)
                              : chunk_b(G, S, k * S.ngc + i0 + np - 1);
          ring_wait(P, sm, R, use, dead);
          if (w == 0 && k == 1 && i0 == 0) FMOE_MARK(u, MK_J1_W0);
          if (np > 1) ring_wait(P, sm, R, use + 1, dead);
          if (w == 0 && i0 == 0 && !sh) FMOE_MARK(u, MK_K_P2F + k);
          gu_pass<BITS, FORM, NRG>(P, G, sm, np, c0, c1, R, use, red, xg, hdst, u,
                                   !sh && k == 0 && i0 == 0);
          use += (unsigned)np;
        }
        if (sh) a_used = use;
        else b_used = use;
        if (w == 0) FMOE_MARK(u, sh ? MK_K_SGU : MK_K_P2 + k);
      }
    }
    if (!gu_on) continue;
    // ---- down rows: segment 0 the shared expert (ring A), then routed expert k (ring B), each
    // as soon as every CTA's h-rows of it are in; accumulated into this CTA's output rows
    if (S.ndc > 0) {
#pragma unroll 1
      for (int sgm = 0; sgm < G.nseg; ++sgm) {
        const bool sh = G.shared_on && sgm == 0;
        const int k = sgm - G.shared_on;
        const bool okw = sh ? warp_wait_ready(P, sm, &sm->hs_ready, &sm->hs_bar, (unsigned)(u + 1),
                                              DE_TIMEOUT_DEP)
                            : warp_wait_ready(P, sm, &sm->hk_ready, &sm->hk_bar,
                                              (unsigned)(u * G.K + k + 1), DE_TIMEOUT_DEP);
        if (!dead && !okw) dead = true;
        if (w == 0) FMOE_MARK(u, sh ? MK_K_HS : MK_K_HK + k);
        float* hseg = HB + (size_t)sgm * G.I;
        const float hsc = sh ? sm->sigma[slot_u] : sm->rt_w[slot_u][k];
        if constexpr (FORM == FORM_DIGITS) {
          transform<BITS>(hseg, G.si, hsc);
          consumers_sync();
        }
        const Ring R = sh ? A : B;
        unsigned use = sh ? a_used : b_used;
#pragma unroll 1
        for (int i = 0; i < S.ndc; ++i) {
          const Chunk c = sh ? chunk_a(G, S, S.nrc + S.ngc + i)
                             : chunk_b(G, S, G.K * S.ngc + k * S.ndc + i);
          ring_wait(P, sm, R, use, dead);
          dn_chunk<BITS, FORM, NRD>(G, c, ring_stage(G, R, use), ring_empty(R, use), hseg, hsc,
                                    oacc, S.d0);
          ++use;
        }
        if (sh) a_used = use;
        else b_used = use;
        if (w == 0) FMOE_MARK(u, sh ? MK_K_DS : MK_K_D + k);
      }
    }
    // ---- outputs of this CTA's rows: residual + accumulated experts; sum of squares
    if (G.nseg > 0) {
      if (S.d1 > S.d0) consumers_sync();
      if (w == 0) {
        const UnitView uv = unit_view(P, G, u);  // (recomputed: not held through the unit)
#pragma unroll 1
        for (int r = S.d0 + lane; r < S.d1; r += 32) {
          const float res = uv.resw ? value_of(__ldcg(uv.resw + r))
                                    : (uv.res ? __ldcg(uv.res + r) : 0.f);
          const float o = res + oacc[r - S.d0];
          oacc[r - S.d0] = 0.f;
          if (uv.outw) st_relaxed_gpu_u64(uv.outw + r, value_word(o, u));
          else uv.out[r] = o;
        }
        __syncwarp();
        if (lane == 0) unit_done(P, u);
        FMOE_MARK(u, MK_K_OUT);
      }
    }
  }
}

template <int BITS, int FORM>
__global__ void __launch_bounds__(kThreads, 1)
    engine_kernel(const __grid_constant__ Prog P, const __grid_constant__ Geo G) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Smem* sm = reinterpret_cast<Smem*>(smem + G.o_misc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G.o_bar);
  if (threadIdx.x == 0) {
    sm->abort = 0;
    sm->x_ready = sm->rt_ready = sm->hs_ready = sm->hk_ready = sm->xfree = 0;
    sm->xd_arrive = 0;
#pragma unroll 1
    for (int i = 0; i < 2 * kMaxStages; ++i) sm->chunk_arrive[i] = 0;
    mbar_init(&sm->xbar, 1);
    mbar_init(&sm->x_bar, 1);
    mbar_init(&sm->rt_bar, 1);
    mbar_init(&sm->hs_bar, 1);
    mbar_init(&sm->hk_bar, 1);
    mbar_init(&sm->xfree_bar, 1);
#pragma unroll 1
    for (int i = 0; i < G.nA; ++i) {
      mbar_init(&bars[i], 1);
      mbar_init(&bars[G.nA + i], kConsumerWarps);
    }
#pragma unroll 1
    for (int i = 0; i < G.nB; ++i) {
      mbar_init(&bars[2 * G.nA + i], 1);
      mbar_init(&bars[2 * G.nA + G.nB + i], kConsumerWarps);
    }
    fence_mbar_init();
  }
  float* oacc = reinterpret_cast<float*>(smem + G.o_oacc);
#pragma unroll 1
  for (int i = threadIdx.x; i < G.oacc_n; i += blockDim.x) oacc[i] = 0.f;
  __syncthreads();
  const Share S = make_share(G);
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) producer_a(P, G, smem, sm, S);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) producer_b(P, G, smem, sm, S);
  } else if (warp == 2) {
    controller(P, G, smem, sm, S.ndc > 0);
  } else {
    consumer<BITS, FORM, kMaxRowsThread, kMaxRowsWarp>(P, G, smem, sm, S);
  }
}

template <int BITS, int FORM>
cudaError_t launch_t(const Prog* P, const Geo* G, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)kThreads);
  cfg.dynamicSmemBytes = G->smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, engine_kernel<BITS, FORM>, *P, *G);
}

template <int BITS, int FORM>
cudaError_t configure_t(int max_smem) {
  return cudaFuncSetAttribute(engine_kernel<BITS, FORM>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
}

}  // namespace fmoe

// ------------------------------------------------------------------------------------------
// launchers used by the C ABI layer
// ------------------------------------------------------------------------------------------
extern "C" cudaError_t fmoe_engine_configure(int max_smem) {
  using namespace fmoe;
  cudaError_t e;
  if ((e = configure_t<4, FORM_DIGITS>(max_smem)) != cudaSuccess) return e;
  if ((e = configure_t<2, FORM_DIGITS>(max_smem)) != cudaSuccess) return e;
  if ((e = configure_t<4, FORM_FMA>(max_smem)) != cudaSuccess) return e;
  if ((e = configure_t<2, FORM_FMA>(max_smem)) != cudaSuccess) return e;
  if ((e = configure_t<4, FORM_NAIVE>(max_smem)) != cudaSuccess) return e;
  return configure_t<2, FORM_NAIVE>(max_smem);
}

// The CTAs of one launch wait on each other's progress, so they must all be resident at
// once: the launch is cooperative, which makes a grid that cannot be co-resident a launch
// error instead of a wait that runs out of budget.
extern "C" cudaError_t fmoe_engine_launch(const fmoe::Prog* P, const fmoe::Geo* G, int grid,
                                          cudaStream_t stream) {
  using namespace fmoe;
  const int f = P->form;
  if (G->bits == 4) {
    if (f == FORM_FMA) return launch_t<4, FORM_FMA>(P, G, grid, stream);
    if (f == FORM_NAIVE) return launch_t<4, FORM_NAIVE>(P, G, grid, stream);
    return launch_t<4, FORM_DIGITS>(P, G, grid, stream);
  }
  if (f == FORM_FMA) return launch_t<2, FORM_FMA>(P, G, grid, stream);
  if (f == FORM_NAIVE) return launch_t<2, FORM_NAIVE>(P, G, grid, stream);
  return launch_t<2, FORM_DIGITS>(P, G, grid, stream);
}

// CTAs of the engine kernel that fit on one SM with `smem` bytes of dynamic shared memory.
extern "C" cudaError_t fmoe_engine_occupancy(int smem, int* ctas_per_sm) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      ctas_per_sm, fmoe::engine_kernel<4, fmoe::FORM_DIGITS>, fmoe::kThreads, (size_t)smem);
}
