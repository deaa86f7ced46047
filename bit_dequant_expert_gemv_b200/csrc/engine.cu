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

namespace fmoe {

// ------------------------------------------------------------------------------------------
// small shared state
// ------------------------------------------------------------------------------------------
struct Smem {
  uint64_t xbar;               // the controller's bulk-copy barrier for x
  uint64_t hbar;               // the controller's bulk-copy barrier for h
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
  volatile int abort;
};

__device__ __forceinline__ void raise_error(const Prog& P, Smem* sm, int code) {
  atomicCAS(P.s.err, 0, code);
  sm->abort = 1;
}

__device__ __forceinline__ unsigned* sig_word(const Prog& P, int s) { return P.s.ctrl + 32 * s; }

// ------------------------------------------------------------------------------------------
// bounded waits
// ------------------------------------------------------------------------------------------
// Spin until *a - target >= 0 (wrap-safe) on a gpu-scope counter, the budget runs out, the
// CTA aborts or another CTA has recorded an error. Polls with relaxed loads and makes one
// acquire fence once the target is seen.
__device__ __noinline__ bool spin_geq(const Prog& P, Smem* sm, const unsigned* a, unsigned target,
                                      int code) {
  if ((int)(ld_acquire(a) - target) >= 0) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (unsigned it = 0;; ++it) {
    if ((int)(ld_relaxed_gpu(a) - target) >= 0) {
      fence_acq_rel_gpu();
      return true;
    }
    if (sm->abort) return false;
    if ((it & 15) == 15) {
      if (ld_volatile_int(P.s.err) != 0) {
        sm->abort = 1;
        return false;
      }
      if (global_ns() > deadline) {
        raise_error(P, sm, code);
        return false;
      }
    }
    __nanosleep(32);
  }
}

__device__ __noinline__ bool wait_mbar(const Prog& P, Smem* sm, uint64_t* bar, unsigned parity,
                                       int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 2000u)) return true;
    if (sm->abort) return false;
    if (global_ns() > deadline) {
      raise_error(P, sm, code);
      return false;
    }
  }
}

// Wait until the readiness counter *cnt reaches target. Sleeps on the phase that the next
// increment completes (the publisher stores the counter before it arrives on the barrier),
// re-reading the counter after every wake-up or after at most ~1 us.
__device__ __noinline__ bool wait_ready(const Prog& P, Smem* sm, const unsigned* cnt,
                                        uint64_t* bar, unsigned target, int code) {
  unsigned c = ld_acquire_cta_smem(cnt);
  if ((int)(c - target) >= 0) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (;;) {
    if (!mbar_try_wait_sleep(bar, c & 1u, 1000u)) __nanosleep(64);
    c = ld_acquire_cta_smem(cnt);
    if ((int)(c - target) >= 0) return true;
    if (sm->abort) return false;
    if (global_ns() > deadline) {
      raise_error(P, sm, code);
      return false;
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

__device__ __forceinline__ bool warp_spin_geq(const Prog& P, Smem* sm, int s, unsigned target,
                                              int code) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = spin_geq(P, sm, sig_word(P, s), target, code);
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
  const float* xin;   // raw input h (x before the norm)
  bool norm;          // x = rmsnorm(h) using normsq[u-1]
  const float* res;   // nullable
  float* out;
  const float* bias;  // nullable [E]
  int* idx_out;
  float* w_out;
  float* h_trace;
};

__device__ __forceinline__ UnitView unit_view(const Prog& P, const Geo& G, int u) {
  UnitView v;
  v.slot = u & 1;
  if (P.mode == MODE_SEQ) {
    v.t = u;
    v.l = u % P.n_layers;
    v.xin = P.x + (size_t)u * G.H;
    v.norm = false;
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
    v.xin = v.l == 0 ? P.x + (size_t)v.t * G.H : P.s.hbuf + (size_t)((u - 1) & 1) * G.H;
    v.norm = v.l > 0;
    v.res = v.xin;
    v.out = v.l == L - 1 ? P.out + (size_t)v.t * G.H : P.s.hbuf + (size_t)(u & 1) * G.H;
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

// Issue one chunk into a stage: lane 0 waits for the stage to be free and registers the
// bytes on its full barrier; lanes 0..3 issue the copies.
__device__ __forceinline__ bool issue_chunk(const Prog& P, const Geo& G, Smem* sm,
                                            uint8_t* stage, uint64_t* full, uint64_t* empty,
                                            unsigned use, const LayerW& L, const uint8_t* eb,
                                            const Chunk& c) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) {
    ok = wait_mbar(P, sm, empty, (use & 1u) ^ 1u, DE_TIMEOUT_EMPTY);
    if (ok) mbar_arrive_expect_tx(full, chunk_bytes(G, c));
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (!ok) return false;
  if (lane < 4) {
    const uint8_t* src = nullptr;
    unsigned dst_off = 0;
    const unsigned bytes = copy_desc(G, L, eb, c, lane, &src, &dst_off);
    if (bytes) tma_load_1d(stage + dst_off, src, bytes, full);
  }
  __syncwarp();
  return true;
}

// Never leave the CTA with bulk copies in flight: wait for the last use of every stage.
__device__ void drain_ring(const Prog& P, uint64_t* full, int ns, unsigned issued) {
  if ((threadIdx.x & 31) != 0) return;
  const uint64_t deadline = global_ns() + 100000000ull;
  const unsigned first = issued > (unsigned)ns ? issued - (unsigned)ns : 0u;
  for (unsigned j = first; j < issued; ++j) {
    while (!mbar_try_wait(&full[j % (unsigned)ns], (j / (unsigned)ns) & 1u)) {
      if (global_ns() > deadline) {
        atomicCAS(P.s.err, 0, DE_TIMEOUT_DRAIN);
        return;
      }
    }
  }
}

__device__ void producer_a(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm,
                           const Share& S) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_bar);
  uint64_t* empty = full + G.nA;
  unsigned issued = 0;
  bool failed = false;
  for (int u = 0; u < P.n_units && !failed; ++u) {
    const LayerW& L = P.layers[u % P.n_layers];
    for (int i = 0; i < S.na; ++i) {
      const Chunk c = chunk_a(G, S, i);
      const unsigned st = issued % (unsigned)G.nA;
      if (!issue_chunk(P, G, sm, smem + G.o_ringA + (size_t)st * G.stage_bytes, &full[st],
                       &empty[st], issued / (unsigned)G.nA, L, L.shared, c)) {
        failed = true;
        break;
      }
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
  for (int u = 0; u < P.n_units && !failed; ++u) {
    const LayerW& L = P.layers[u % P.n_layers];
    if (!warp_wait_ready(P, sm, &sm->rt_ready, &sm->rt_bar, (unsigned)(u + 1), DE_TIMEOUT_ROUTE)) {
      failed = true;
      break;
    }
    const int* rte = sm->rt_e[u & 1];
    for (int i = 0; i < S.nb; ++i) {
      const Chunk c = chunk_b(G, S, i);
      const int e = min(max(rte[c.e], 0), G.E - 1);
      const uint8_t* eb = L.experts + (size_t)e * L.expert_stride;
      const unsigned st = issued % (unsigned)G.nB;
      if (!issue_chunk(P, G, sm, smem + G.o_ringB + (size_t)st * G.stage_bytes, &full[st],
                       &empty[st], issued / (unsigned)G.nB, L, eb, c)) {
        failed = true;
        break;
      }
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

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

// Sort 16 keys in descending order (bitonic network, fully unrolled).
__device__ __forceinline__ void sort16_desc(unsigned long long (&k)[16]) {
#pragma unroll
  for (int size = 2; size <= 16; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = k[i], b = k[j];
          const bool sw = desc ? (a < b) : (a > b);
          k[i] = sw ? b : a;
          k[j] = sw ? a : b;
        }
      }
    }
  }
}

// Logits e0 + lane + 32 i (i < 16) of the unit: the bias plus the column-segment partials,
// in segment order.
__device__ __forceinline__ void load_logits(const Geo& G, const double* lg, const float* bias,
                                            int e0, double (&lv)[16]) {
  const int lane = threadIdx.x & 31;
  double p1[16];
  float bv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {  // the bias and the first two segments in one round trip
    const int ec = min(e0 + lane + 32 * i, G.E - 1);
    bv[i] = bias ? __ldcg(bias + ec) : 0.f;
    lv[i] = __ldcg(lg + ec);
    p1[i] = G.rseg > 1 ? __ldcg(lg + (size_t)G.nr + ec) : 0.0;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) lv[i] = ((double)bv[i] + lv[i]) + p1[i];
  for (int sg = 2; sg < G.rseg; ++sg) {
    double part[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      part[i] = __ldcg(lg + (size_t)sg * G.nr + min(e0 + lane + 32 * i, G.E - 1));
#pragma unroll
    for (int i = 0; i < 16; ++i) lv[i] += part[i];
  }
}

// The binary64 logit of expert e (bias first, then the segments in order, as load_logits).
__device__ __forceinline__ double one_logit(const Geo& G, const double* lg, const float* bias,
                                            int e) {
  double l = ((double)(bias ? __ldcg(bias + e) : 0.f) + __ldcg(lg + e)) +
             (G.rseg > 1 ? __ldcg(lg + (size_t)G.nr + e) : 0.0);
  for (int sg = 2; sg < G.rseg; ++sg) l += __ldcg(lg + (size_t)sg * G.nr + e);
  return l;
}

// Top-K of the unit's logits by one warp. Lane l holds experts l + 32 i of each block of 512;
// with more than 512 experts every lane keeps its 16 largest keys across blocks (bitonic
// merge). K rounds: the warp maximum of the lanes' best packed keys (two 32-bit reductions:
// high word, then low word among the lanes holding that high word); the lane that held it
// drops it. The winners' binary64 logits give the weights w_k = exp(l_k - l_max) /
// sum_sel exp(l_j - l_max): the softmax over all experts followed by renormalisation over the
// selected ones, where the full softmax denominator cancels.
__device__ void topk_warp(const Geo& G, const double* lg, const float* bias, int* rt_e,
                          float* rt_w, int* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  unsigned long long key[16];
  {
    double lv[16];
    load_logits(G, lg, bias, 0, lv);
#pragma unroll
    for (int i = 0; i < 16; ++i) key[i] = lane + 32 * i < G.E ? pkey(lv[i], lane + 32 * i) : 0ull;
  }
  if (G.E > 512) {
    sort16_desc(key);
    for (int e0 = 512; e0 < G.E; e0 += 512) {
      double lw[16];
      unsigned long long k2[16];
      load_logits(G, lg, bias, e0, lw);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int e = e0 + lane + 32 * i;
        k2[i] = e < G.E ? pkey(lw[i], e) : 0ull;
      }
      sort16_desc(k2);
#pragma unroll
      for (int i = 0; i < 16; ++i) key[i] = umax64(key[i], k2[15 - i]);
      sort16_desc(key);
    }
  }
  unsigned long long bk = key[0];
  int bi = 0;
#pragma unroll
  for (int i = 1; i < 16; ++i)
    if (key[i] > bk) bk = key[i], bi = i;
  int sel_e = 0;
  for (int k = 0; k < G.K; ++k) {
    const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(bk >> 32));
    const unsigned lo =
        __reduce_max_sync(0xffffffffu, (unsigned)(bk >> 32) == hi ? (unsigned)bk : 0u);
    const unsigned long long win = ((unsigned long long)hi << 32) | lo;
    if (bk == win && win != 0ull) {  // exactly one lane holds it: drop it, find the next
#pragma unroll
      for (int i = 0; i < 16; ++i) key[i] = i == bi ? 0ull : key[i];
      bk = key[0];
      bi = 0;
#pragma unroll
      for (int i = 1; i < 16; ++i)
        if (key[i] > bk) bk = key[i], bi = i;
    }
    if (lane == k) sel_e = 0x1FFF - (int)(win & 0x1FFFull);
  }
  const bool mine = lane < G.K;
  const int e = min(max(sel_e, 0), G.E - 1);  // NaN logits must not make an address
  const double sel_l = mine ? one_logit(G, lg, bias, e) : 0.0;
  const double l0 = __shfl_sync(0xffffffffu, sel_l, 0);
  const float ex = mine ? expf((float)(sel_l - l0)) : 0.f;
  float den = ex;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (mine) {
    const float wk = __fdividef(ex, den);
    rt_e[lane] = e;
    rt_w[lane] = wk;
    if (idx_out) idx_out[lane] = e;
    if (w_out) w_out[lane] = wk;
  }
  __syncwarp();
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

// The signal whose completion means "unit u is done" and its rows per unit.
__device__ __forceinline__ int final_sig(const Geo& G) { return G.nseg > 0 ? SG_OUT : SG_ROUTER; }
__device__ __forceinline__ unsigned final_rows(const Geo& G) {
  return G.nseg > 0 ? (unsigned)G.H : (unsigned)(G.nr * G.rseg);
}

__device__ void controller(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm) {
  const int lane = threadIdx.x & 31;
  float* XB = reinterpret_cast<float*>(smem + G.o_x);
  float* HB = reinterpret_cast<float*>(smem + G.o_h);
  unsigned px = 0, ph = 0;  // phases of the x and h copy barriers
  bool x_issued = false;    // the next unit's x copy is already in flight
  const int fsig = final_sig(G);
  const unsigned frows = final_rows(G);
  bool x_digits = G.shared_on || G.routed_on;
  for (int u = 0; u < P.n_units; ++u) {
    const UnitView uv = unit_view(P, G, u);
    const bool owner = (u % (int)gridDim.x) == (int)blockIdx.x;
    // ---- x(u): computed on only after unit u-1 is complete everywhere
    if (u > 0 && !warp_spin_geq(P, sm, fsig, (unsigned)u * frows, DE_TIMEOUT_DEP)) break;
    if (!x_issued) copy_in(XB, uv.xin, 4u * (unsigned)G.H, &sm->xbar);
    x_issued = false;
    float f = 1.f;
    if (uv.norm) f = rsqrtf(__ldcg(P.s.normsq + (u - 1)) / (float)G.H + P.eps);
    if (!wait_copy(P, sm, &sm->xbar, px)) break;
    if (owner && uv.h_trace)
      for (int c = lane * 4; c < G.H; c += 128)
        *reinterpret_cast<float4*>(uv.h_trace + c) = *reinterpret_cast<const float4*>(XB + c);
    if (lane == 0) {
      sm->xf[u & 1] = f;
      signal_ready(&sm->x_ready, &sm->x_bar, (unsigned)(u + 1));
    }
    __syncwarp();
    // ---- routing decision: needs every router row of unit u
    const double* lg = P.s.logits + (size_t)uv.slot * G.rseg * G.nr;
    if (G.route_on) {
      if (uv.bias)  // the unit's logit bias into L2 while the router runs
        for (int e = lane * 32; e < G.E; e += 32 * 32) prefetch_l2(uv.bias + e);
      if (!warp_spin_geq(P, sm, SG_ROUTER, (unsigned)(u + 1) * (unsigned)(G.nr * G.rseg),
                         DE_TIMEOUT_ROUTE))
        break;
      topk_warp(G, lg, uv.bias, sm->rt_e[u & 1], sm->rt_w[u & 1], owner ? uv.idx_out : nullptr,
                owner ? uv.w_out : nullptr);
      float sigma = 1.f;
      if (G.gate_on) {
        double a = 0.0;
        for (int s = 0; s < G.rseg; ++s) a += __ldcg(lg + (size_t)s * G.nr + G.E);
        sigma = (float)(1.0 / (1.0 + exp(-a)));
      }
      if (lane == 0) {
        sm->sigma[u & 1] = sigma;
        signal_ready(&sm->rt_ready, &sm->rt_bar, (unsigned)(u + 1));
      }
      __syncwarp();
    } else if (lane == 0) {
      sm->sigma[u & 1] = 1.f;
    }
    // ---- independent tokens: the next unit's x, once the consumers hold this unit's x
    // digits in registers (its computation still waits for this unit to complete)
    if (P.mode == MODE_SEQ && x_digits && u + 1 < P.n_units) {
      if (!warp_wait_ready(P, sm, &sm->xfree, &sm->xfree_bar, (unsigned)(u + 1), DE_TIMEOUT_DEP))
        break;
      copy_in(XB, P.x + (size_t)(u + 1) * G.H, 4u * (unsigned)G.H, &sm->xbar);
      x_issued = true;
    }
    if (G.nseg == 0) continue;
    // ---- h_s: every shared-expert h-row of unit u
    if (G.shared_on) {
      if (!warp_spin_geq(P, sm, SG_SHARED, (unsigned)(u + 1) * (unsigned)G.I, DE_TIMEOUT_DEP))
        break;
      copy_in(HB, P.s.hs + (size_t)uv.slot * G.I, 4u * (unsigned)G.I, &sm->hbar);
      if (!wait_copy(P, sm, &sm->hbar, ph)) break;
      if (lane == 0) signal_ready(&sm->hs_ready, &sm->hs_bar, (unsigned)(u + 1));
      __syncwarp();
    }
    // ---- h_k: routed expert k's h-rows of unit u, in order
    if (G.routed_on) {
      bool ok = true;
      for (int k = 0; k < G.K && ok; ++k) {
        ok = warp_spin_geq(P, sm, SG_EXP0 + k, (unsigned)(u + 1) * (unsigned)G.I, DE_TIMEOUT_DEP);
        if (!ok) break;
        copy_in(HB + (size_t)(G.shared_on + k) * G.I, P.s.hk + ((size_t)uv.slot * G.K + k) * G.I,
                4u * (unsigned)G.I, &sm->hbar);
        ok = wait_copy(P, sm, &sm->hbar, ph);
        if (!ok) break;
        if (lane == 0) signal_ready(&sm->hk_ready, &sm->hk_bar, (unsigned)(u * G.K + k + 1));
        __syncwarp();
      }
      if (!ok) break;
    }
  }
  // never leave with a copy in flight
  if (x_issued && lane == 0) {
    const uint64_t deadline = global_ns() + 100000000ull;
    while (!mbar_try_wait(&sm->xbar, px))
      if (global_ns() > deadline) break;
  }
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

// Transform nsl slices of buf (binary32, scaled by `scale`) into digit form, in place, by the
// 256 consumer threads: TS threads per slice, each owning one code word's columns (8 at
// 4 bits, 16 at 2 bits). Every lane of a warp reads its values before any lane writes (the
// TS threads of a slice are consecutive lanes of one warp).
template <int BITS>
__device__ void transform(float* buf, int nsl, float scale) {
  constexpr int TS = BITS == 4 ? 4 : 2;
  constexpr int NV = 32 / TS;
  const int t = (int)threadIdx.x - 32 * kCtrlWarps;
  const int items = nsl * TS;
  const int rounds = (items + kConsumers - 1) / kConsumers;
  for (int r = 0; r < rounds; ++r) {
    const int it = t + kConsumers * r;
    const bool act = it < items;
    const int s = act ? it / TS : 0, j = it % TS;
    float v[NV];
    float m = 0.f, sum = 0.f;
    if (act) {
#pragma unroll
      for (int q = 0; q < NV / 4; ++q) {
        const float4 a = *reinterpret_cast<const float4*>(buf + 32 * s + NV * j + 4 * q);
        v[4 * q] = a.x * scale; v[4 * q + 1] = a.y * scale;
        v[4 * q + 2] = a.z * scale; v[4 * q + 3] = a.w * scale;
      }
#pragma unroll
      for (int q = 0; q < NV; ++q) {
        m = fmaxf(m, fabsf(v[q]));
        sum += v[q];
      }
    }
#pragma unroll
    for (int o = 1; o < TS; o <<= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    __syncwarp();
    if (act) {
      const float k = m > 0.f ? __fdividef(2080768.f, m) : 0.f;
      uint32_t* base = reinterpret_cast<uint32_t*>(buf);
      if (BITS == 4) {
        uint32_t w[3][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float kh = h ? k * 0.0625f : k;
          int d[3][4];
#pragma unroll
          for (int b = 0; b < 4; ++b) digits3(v[2 * b + h], kh, d[0][b], d[1][b], d[2][b]);
#pragma unroll
          for (int p = 0; p < 3; ++p) w[p][h] = pack4(d[p][0], d[p][1], d[p][2], d[p][3]);
        }
        // words 2j, 2j+1 of plane p: chunk 2p + j/2, word positions 2(j%2), 2(j%2)+1
#pragma unroll
        for (int p = 0; p < 3; ++p)
          *reinterpret_cast<uint2*>(base + dslot(s, 2 * p + (j >> 1)) + 2 * (j & 1)) =
              make_uint2(w[p][0], w[p][1]);
      } else {
        uint32_t w[3][4];
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          const float kp = k * (pc == 0 ? 1.f : pc == 1 ? 0.25f : pc == 2 ? 0.0625f : 0.015625f);
          int d[3][4];
#pragma unroll
          for (int b = 0; b < 4; ++b) digits3(v[4 * b + pc], kp, d[0][b], d[1][b], d[2][b]);
#pragma unroll
          for (int p = 0; p < 3; ++p) w[p][pc] = pack4(d[p][0], d[p][1], d[p][2], d[p][3]);
        }
        // words 4j .. 4j+3 of plane p: chunk 2p + j
#pragma unroll
        for (int p = 0; p < 3; ++p)
          *reinterpret_cast<uint4*>(base + dslot(s, 2 * p + j)) =
              make_uint4(w[p][0], w[p][1], w[p][2], w[p][3]);
      }
      if (j == 0)
        *reinterpret_cast<float2*>(base + dslot(s, 6)) = make_float2(m * (1.f / 2080768.f), sum);
    }
    __syncwarp();
  }
}

// The digit form of slice s of buf: xd[8p + n] = word n of plane p; {sc, sx}.
struct XDig {
  int d[24];
  float sc, sx;
};

__device__ __forceinline__ void load_digits(const float* buf, int s, XDig& x) {
  const uint32_t base = smem_u32(buf);
#pragma unroll
  for (int i = 0; i < 6; ++i) {
    const uint4 a = lds128(base + 4u * (unsigned)dslot(s, i));
    x.d[4 * i] = (int)a.x; x.d[4 * i + 1] = (int)a.y; x.d[4 * i + 2] = (int)a.z;
    x.d[4 * i + 3] = (int)a.w;
  }
  const uint2 b = lds64(base + 4u * (unsigned)dslot(s, 6));
  x.sc = __uint_as_float(b.x);
  x.sx = __uint_as_float(b.y);
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
// one row x one 32-column slice
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// s * sum(q x) + z * sum(x) over the slice: codes at `ca`, scale/bias word `sbw`.
template <int BITS>
__device__ __forceinline__ float slice_dot(uint32_t ca, uint32_t sbw, const XDig& x) {
  int c0 = 0, c1 = 0, c2 = 0;
  if constexpr (BITS == 4) {
    const uint4 q = lds128(ca);
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = qw[j] & 0x0F0F0F0Fu, hi = qw[j] & 0xF0F0F0F0u;
      c0 = dp4a_us(hi, x.d[2 * j + 1], dp4a_us(lo, x.d[2 * j], c0));
      c1 = dp4a_us(hi, x.d[8 + 2 * j + 1], dp4a_us(lo, x.d[8 + 2 * j], c1));
      c2 = dp4a_us(hi, x.d[16 + 2 * j + 1], dp4a_us(lo, x.d[16 + 2 * j], c2));
    }
  } else {
    const uint2 q = lds64(ca);
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
__device__ __forceinline__ float slice_dot_fma(uint32_t ca, uint32_t sbw, const XVal& x) {
  uint32_t qw[4];
  if constexpr (BITS == 4) {
    const uint4 q = lds128(ca);
    qw[0] = q.x; qw[1] = q.y; qw[2] = q.z; qw[3] = q.w;
  } else {
    const uint2 q = lds64(ca);
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
__device__ __forceinline__ float slice_dot_naive(uint32_t ca, uint32_t sbw, const XVal& x) {
  uint32_t qw[4];
  if constexpr (BITS == 4) {
    const uint4 q = lds128(ca);
    qw[0] = q.x; qw[1] = q.y; qw[2] = q.z; qw[3] = q.w;
  } else {
    const uint2 q = lds64(ca);
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
__device__ __forceinline__ float slice_any(uint32_t ca, uint32_t sbw, const XT& x) {
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
template <int NR, typename Store>
__device__ __forceinline__ void seg_reduce(float (&v)[NR], int lane_in_seg, int width,
                                           Store store) {
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
          const float send = upper ? v[a] : v[a + half];
          const float keep = upper ? v[a + half] : v[a];
          v[a] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      if (upper) lo += half;
      nlive = half;
    }
  }
  if (nlive == 1) {
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
struct Ring {
  uint8_t* base;
  uint64_t* full;
  uint64_t* empty;
  int ns;
  int slot0;       // first chunk_arrive / red slot of this ring
  unsigned used;   // chunks consumed so far
};

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
struct XRouter {
  double v[5][4];   // this thread's x columns (binary64) of the current segment
  int seg;          // which segment they hold (-1: none)
};

__device__ __forceinline__ void router_x(const Geo& G, const float* XB, int seg, XRouter& xr) {
  const int t = (int)threadIdx.x - 32 * kCtrlWarps;
  const int nf = G.rcols / 4;
  const float4* xs = reinterpret_cast<const float4*>(XB + (size_t)seg * G.rcols);
#pragma unroll
  for (int j = 0; j < 5; ++j) {
    const int f = t + kConsumers * j;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    if (f < nf) a = xs[f];
    xr.v[j][0] = (double)a.x; xr.v[j][1] = (double)a.y;
    xr.v[j][2] = (double)a.z; xr.v[j][3] = (double)a.w;
  }
  xr.seg = seg;
}

__device__ __forceinline__ bool router_chunk(const Prog& P, const Geo& G, Smem* sm,
                                             const Chunk& c, int u, const uint8_t* stage,
                                             uint64_t* empty, int slot, double* red,
                                             const XRouter& xr, bool last_of_cta,
                                             unsigned cta_rows) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  const int t = w * 32 + lane;
  const int nf = G.rcols / 4;
  const float4* ws = reinterpret_cast<const float4*>(stage);
  double* rs = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(red) + (size_t)slot * G.red_slot);
  for (int r = 0; r < c.n; ++r) {
    double a = 0.0;
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      const int f = t + kConsumers * j;
      if (f < nf) {
        const float4 wv = ws[(size_t)r * nf + f];
        a = fma((double)wv.x, xr.v[j][0], a);
        a = fma((double)wv.y, xr.v[j][1], a);
        a = fma((double)wv.z, xr.v[j][2], a);
        a = fma((double)wv.w, xr.v[j][3], a);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) rs[r * kConsumerWarps + w] = a;
  }
  const bool last = chunk_last(sm, slot);
  if (last) {
    const double xf = (double)sm->xf[u & 1];
    double* lg = P.s.logits + ((size_t)(u & 1) * G.rseg + c.seg) * G.nr + c.r0;
    for (int r = lane; r < c.n; r += 32) {
      double a = 0.0;
#pragma unroll
      for (int q = 0; q < kConsumerWarps; ++q) a += rs[r * kConsumerWarps + q];
      lg[r] = a * xf;  // the norm factor of x, applied to the sum
    }
    __syncwarp();
    if (last_of_cta && lane == 0 && !(P.debug & 1))
      red_release_gpu(sig_word(P, SG_ROUTER), cta_rows);
  }
  release_stage(empty);
  return true;
}

// Gate/up rows of a chunk: hr gate rows then hr up rows (n valid each) in the stage. Thread
// (group g, slice s) takes rows rho = g + gh * i; partial sums are reduced over the row's
// threads (lanes of its segment, then warps through shared memory); the chunk's last warp
// applies SwiGLU and stores h. Returns whether the stage was handed back normally.
template <int BITS, int FORM, int NR>
__device__ __forceinline__ void gu_chunk(const Prog& P, const Geo& G, Smem* sm, const Chunk& c,
                                         const uint8_t* stage, uint64_t* empty, int slot,
                                         float* red, const typename XOf<FORM>::T& x, float* h,
                                         int sig, bool last_of_k, unsigned cta_rows) {
  const int lane = threadIdx.x & 31;
  const int t = (int)threadIdx.x - 32 * kCtrlWarps;
  const int g = t / G.wh, s = t - g * G.wh;
  const bool act = g < G.gh && s < G.sh;
  const int hr = G.hr, n = c.n;
  constexpr unsigned cb = BITS == 4 ? 16u : 8u;
  const uint32_t st = smem_u32(stage);
  const uint32_t sb0 = st + 2u * (unsigned)hr * G.rc_h + (unsigned)(s >> 1) * 4u;
  float acc[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    acc[i] = 0.f;
    const int rho = g + G.gh * i;
    const int rr = rho < hr ? rho : rho - hr;
    if (act && rho < 2 * hr && rr < n) {
      const uint32_t sbw = lds32(sb0 + (unsigned)rho * G.rs_h);
      acc[i] = slice_any<BITS, FORM>(st + (unsigned)rho * G.rc_h + (unsigned)s * cb, sbw, x);
    }
  }
  // reduce over the row's threads: its segment of lanes, then (wide rows) its warps
  const int width = G.wh < 32 ? G.wh : 32;
  const int wn = G.wh > 32 ? G.wh / 32 : 1;  // warps per row group
  const int om = G.wh > 32 ? s >> 5 : 0;     // this warp's index within its group
  float* rs = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(red) + (size_t)slot * G.red_slot);
  seg_reduce<NR>(acc, lane & (width - 1), width, [&](int i, float v) {
    const int rho = g + G.gh * i;
    if (act && rho < 2 * hr) rs[rho * wn + om] = v;
  });
  const bool last = chunk_last(sm, slot);
  if (last) {
    for (int i = lane; i < n; i += 32) {
      float a = 0.f, b = 0.f;
      for (int q = 0; q < wn; ++q) {
        a += rs[i * wn + q];
        b += rs[(hr + i) * wn + q];
      }
      h[c.r0 + i] = __fdividef(a, 1.f + __expf(-a)) * b;  // SwiGLU: SiLU(gate) * up
    }
    __syncwarp();
    if (last_of_k && lane == 0) red_release_gpu(sig_word(P, sig), cta_rows);
  }
  release_stage(empty);
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
  const uint32_t st = smem_u32(stage);
  const uint32_t sbb = st + (unsigned)G.dr * G.rc_i;
  float acc[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) acc[i] = 0.f;
  for (int j = 0; j < G.ji; ++j) {
    const int s = lane_s + G.wi * j;
    const bool sok = s < G.si;
    typename XOf<FORM>::T x;
    if constexpr (FORM == FORM_DIGITS)
      load_digits(hseg, sok ? s : 0, x);
    else
      load_values(hseg, sok ? s : 0, hscale, x);
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int rho = w * G.pi + lane_p + kConsumerWarps * G.pi * i;
      if (sok && rho < n) {
        const uint32_t sbw = lds32(sbb + (unsigned)rho * G.rs_i + (unsigned)(s >> 1) * 4u);
        acc[i] += slice_any<BITS, FORM>(st + (unsigned)rho * G.rc_i + (unsigned)s * cb, sbw, x);
      }
    }
  }
  release_stage(empty);
  const int r_off = c.r0 - d0;
  seg_reduce<NR>(acc, lane_s, G.wi, [&](int i, float v) {
    const int rho = w * G.pi + lane_p + kConsumerWarps * G.pi * i;
    if (rho < n) oacc[r_off + rho] += v;
  });
}

template <int BITS, int FORM, int NR>
__device__ void consumer(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm, const Share& S) {
  const int lane = threadIdx.x & 31;
  const int w = ((int)threadIdx.x >> 5) - kCtrlWarps;
  const int t = w * 32 + lane;
  float* XB = reinterpret_cast<float*>(smem + G.o_x);
  float* HB = reinterpret_cast<float*>(smem + G.o_h);
  float* red = reinterpret_cast<float*>(smem + G.o_red);
  float* oacc = reinterpret_cast<float*>(smem + G.o_oacc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G.o_bar);
  Ring A{smem + G.o_ringA, bars, bars + G.nA, G.nA, 0, 0u};
  Ring B{smem + G.o_ringB, bars + 2 * G.nA, bars + 2 * G.nA + G.nB, G.nB, G.nA, 0u};
  const int gslice = t % G.wh;           // this thread's x slice in gate/up rows
  const bool gu_on = G.shared_on || G.routed_on;
  XRouter xr;
  xr.seg = -1;
  // A wait that fails (its budget ran out, or the CTA aborted) marks the warp dead: it skips
  // every later wait but keeps walking the same sequence of chunks and consumer barriers as
  // the other warps, so that no warp is left at a barrier; the results are then undefined and
  // the error word reports the failure.
  bool dead = false;
  typename XOf<FORM>::T xg;              // x of this thread's slice (digits or values)
  for (int u = 0; u < P.n_units; ++u) {
    const int slot_u = u & 1;
    if (!dead && !warp_wait_ready(P, sm, &sm->x_ready, &sm->x_bar, (unsigned)(u + 1), DE_TIMEOUT_DEP))
      dead = true;
    // ---- router rows
    xr.seg = -1;
    for (int i = 0; i < S.nrc; ++i) {
      const Chunk c = chunk_a(G, S, i);
      const unsigned st = A.used % (unsigned)A.ns;
      if (!dead && !warp_wait_mbar(P, sm, &A.full[st], (A.used / (unsigned)A.ns) & 1u, DE_TIMEOUT_FULL))
        dead = true;
      if (xr.seg != c.seg) router_x(G, XB, c.seg, xr);
      router_chunk(P, G, sm, c, u, A.base + (size_t)st * G.stage_bytes, &A.full[A.ns + st],
                   A.slot0 + (int)st, reinterpret_cast<double*>(red), xr, i == S.nrc - 1,
                   (unsigned)((S.r1 - S.r0) * G.rseg));
      ++A.used;
    }
    if (!gu_on) continue;
    // ---- x of this thread's slice: digit form (in place, after every router read of x)
    consumers_sync();
    const float xf = sm->xf[slot_u];
    if constexpr (FORM == FORM_DIGITS) {
      transform<BITS>(XB, G.sh, xf);
      consumers_sync();
      load_digits(XB, gslice < G.sh ? gslice : 0, xg);
    } else {
      load_values(XB, gslice < G.sh ? gslice : 0, xf, xg);
    }
    // the x buffer is free once every warp holds its slice
    if (lane == 0) {
      const unsigned old = atom_add_acq_rel_cta_smem(&sm->xd_arrive, 1u);
      if (old == (unsigned)(kConsumerWarps * (u + 1) - 1))
        signal_ready(&sm->xfree, &sm->xfree_bar, (unsigned)(u + 1));
    }
    __syncwarp();
    const unsigned hrows = (unsigned)(S.h1 - S.h0);
    // ---- shared expert: gate/up rows, then (once every CTA's are done) down rows
    if (G.shared_on) {
      for (int i = 0; i < S.ngc; ++i) {
        const Chunk c = chunk_a(G, S, S.nrc + i);
        const unsigned st = A.used % (unsigned)A.ns;
        if (!dead && !warp_wait_mbar(P, sm, &A.full[st], (A.used / (unsigned)A.ns) & 1u, DE_TIMEOUT_FULL))
          dead = true;
        gu_chunk<BITS, FORM, NR>(P, G, sm, c, A.base + (size_t)st * G.stage_bytes,
                                 &A.full[A.ns + st], A.slot0 + (int)st, red, xg,
                                 P.s.hs + (size_t)slot_u * G.I, SG_SHARED, i == S.ngc - 1, hrows);
        ++A.used;
      }
      if (S.ndc > 0) {
        if (!dead && !warp_wait_ready(P, sm, &sm->hs_ready, &sm->hs_bar, (unsigned)(u + 1), DE_TIMEOUT_DEP))
          dead = true;
        const float sg = sm->sigma[slot_u];
        if constexpr (FORM == FORM_DIGITS) {
          transform<BITS>(HB, G.si, sg);
          consumers_sync();
        }
        for (int i = 0; i < S.ndc; ++i) {
          const Chunk c = chunk_a(G, S, S.nrc + S.ngc + i);
          const unsigned st = A.used % (unsigned)A.ns;
          if (!dead && !warp_wait_mbar(P, sm, &A.full[st], (A.used / (unsigned)A.ns) & 1u,
                                       DE_TIMEOUT_FULL))
            dead = true;
          dn_chunk<BITS, FORM, NR>(G, c, A.base + (size_t)st * G.stage_bytes, &A.full[A.ns + st],
                                   HB, sg, oacc, S.d0);
          ++A.used;
        }
      }
    }
    // ---- routed experts: gate/up rows of k = 0..K-1, then down rows as each h_k completes
    if (G.routed_on) {
      for (int k = 0; k < G.K; ++k) {
        float* hk = P.s.hk + ((size_t)slot_u * G.K + k) * G.I;
        for (int i = 0; i < S.ngc; ++i) {
          const Chunk c = chunk_b(G, S, k * S.ngc + i);
          const unsigned st = B.used % (unsigned)B.ns;
          if (!dead && !warp_wait_mbar(P, sm, &B.full[st], (B.used / (unsigned)B.ns) & 1u,
                                       DE_TIMEOUT_FULL))
            dead = true;
          gu_chunk<BITS, FORM, NR>(P, G, sm, c, B.base + (size_t)st * G.stage_bytes,
                                   &B.full[B.ns + st], B.slot0 + (int)st, red, xg, hk,
                                   SG_EXP0 + k, i == S.ngc - 1, hrows);
          ++B.used;
        }
      }
      if (S.ndc > 0) {
        for (int k = 0; k < G.K; ++k) {
          if (!dead && !warp_wait_ready(P, sm, &sm->hk_ready, &sm->hk_bar,
                                        (unsigned)(u * G.K + k + 1), DE_TIMEOUT_DEP))
            dead = true;
          float* hseg = HB + (size_t)(G.shared_on + k) * G.I;
          const float wk = sm->rt_w[slot_u][k];
          if constexpr (FORM == FORM_DIGITS) {
            transform<BITS>(hseg, G.si, wk);
            consumers_sync();
          }
          for (int i = 0; i < S.ndc; ++i) {
            const Chunk c = chunk_b(G, S, G.K * S.ngc + k * S.ndc + i);
            const unsigned st = B.used % (unsigned)B.ns;
            if (!dead && !warp_wait_mbar(P, sm, &B.full[st], (B.used / (unsigned)B.ns) & 1u,
                                         DE_TIMEOUT_FULL))
              dead = true;
            dn_chunk<BITS, FORM, NR>(G, c, B.base + (size_t)st * G.stage_bytes,
                                     &B.full[B.ns + st], hseg, wk, oacc, S.d0);
            ++B.used;
          }
        }
      }
    }
    // ---- outputs of this CTA's rows: residual + accumulated experts; sum of squares
    if (G.nseg > 0 && S.d1 > S.d0) {
      consumers_sync();
      if (w == 0) {
        const UnitView uv = unit_view(P, G, u);
        float sq = 0.f;
        for (int r = S.d0 + lane; r < S.d1; r += 32) {
          const float o = (uv.res ? __ldcg(uv.res + r) : 0.f) + oacc[r - S.d0];
          oacc[r - S.d0] = 0.f;
          uv.out[r] = o;
          sq += o * o;
        }
        if (P.mode == MODE_STACK) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
          if (lane == 0) atomicAdd(P.s.normsq + u, sq);
        }
        __syncwarp();
        if (lane == 0) red_release_gpu(sig_word(P, SG_OUT), (unsigned)(S.d1 - S.d0));
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
    for (int i = 0; i < 2 * kMaxStages; ++i) sm->chunk_arrive[i] = 0;
    mbar_init(&sm->xbar, 1);
    mbar_init(&sm->hbar, 1);
    mbar_init(&sm->x_bar, 1);
    mbar_init(&sm->rt_bar, 1);
    mbar_init(&sm->hs_bar, 1);
    mbar_init(&sm->hk_bar, 1);
    mbar_init(&sm->xfree_bar, 1);
    for (int i = 0; i < G.nA; ++i) {
      mbar_init(&bars[i], 1);
      mbar_init(&bars[G.nA + i], kConsumerWarps);
    }
    for (int i = 0; i < G.nB; ++i) {
      mbar_init(&bars[2 * G.nA + i], 1);
      mbar_init(&bars[2 * G.nA + G.nB + i], kConsumerWarps);
    }
    fence_mbar_init();
  }
  float* oacc = reinterpret_cast<float*>(smem + G.o_oacc);
  for (int i = threadIdx.x; i < G.oacc_n; i += blockDim.x) oacc[i] = 0.f;
  __syncthreads();
  const Share S = make_share(G);
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    producer_a(P, G, smem, sm, S);
  } else if (warp == 1) {
    producer_b(P, G, smem, sm, S);
  } else if (warp == 2) {
    controller(P, G, smem, sm);
  } else {
    const int nrg = (2 * G.hr + G.gh - 1) / G.gh;
    const int nrd = (G.dr + kConsumerWarps * G.pi - 1) / (kConsumerWarps * G.pi);
    if (max(nrg, nrd) <= 4)
      consumer<BITS, FORM, 4>(P, G, smem, sm, S);
    else
      consumer<BITS, FORM, 8>(P, G, smem, sm, S);
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
