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
//   each 4-/2-bit weight is q*s + z with one bf16 scale/bias per 64-weight group, evaluated as
//   s * sum(q*x) + z * sum(x) per 32-column slice: the pages' fma(nibble, scale*x, bias*x)
//   with the scale and bias factored out of the slice sum (same value in real arithmetic;
//     "Qu'est-ce que Flash-MoE ?" (a2a-mcp.org, fr), §2 "Noyaux de Déquantification Optimisés
//      pour FMA"); sum(q*x) is taken as integer dot products of the codes with three 8-bit
//   digit planes of x (x ~ s_x (d0 + d1/128 + d2/16384), within 1e-6 of the slice's largest
//   |x|), so that one dp4a covers four weights.
//
// How: one CTA per SM, every CTA working through a static share of every unit's chunks.
//   producer warp   streams each chunk's weight rows into a ring of shared-memory stages with
//                   1-D TMA bulk copies that complete on the stage's mbarrier;
//   stager warp     per unit: brings x into shared memory (TMA; the raw copy is the router's
//                   input), selects the top-K experts once the router is complete, and brings
//                   in the down input [h_s | h_k] once every gate/up chunk is complete;
//   consumer warps  each owns whole chunks (local chunk i -> warp i mod kConsumerWarps); each
//                   puts its part of the unit's x and of its down input
//                   [sigma*h_s | w_k*h_k] into digit form; cuts codes into bytes (nibbles or
//                   bit-planes) for dp4a against the digit planes, reduces its row sums
//                   inside the warp and runs the chunk's epilogue (logit store, SwiGLU, or
//                   residual + combine) itself -- no block-wide barrier and no cross-warp
//                   reduction on the hot path.
// Completion is counted per run of same-class chunks of a CTA: the warp finishing a CTA's run
// makes one gpu-scope release-acquire atomic on the class counter, and the stager warps poll
// that counter (it is performed in L2, so no second hop is needed). Every spin-wait is
// bounded by a global-timer budget; on expiry the kernel records an error word, waits for
// its own copies in flight and returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include "engine.h"
#include "ptx.cuh"

namespace fmoe {

__device__ __forceinline__ int cnt_word(int cls) { return C_CNT + 32 * cls; }

// ------------------------------------------------------------------------------------------
// unit and chunk views
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

struct Chunk {
  int u, c, kind, j, r0, n, k, seg;
};

// The chunks g0, g0 + step, g0 + 2 step, ... of a launch, walked without divisions: (u, c) is
// the current chunk's unit and index within the unit (one division at the start only).
struct ChunkWalk {
  int u, c, step, ntot;
  __device__ __forceinline__ void init(const Geo& G, unsigned long long g0, int step_) {
    ntot = G.off[K_COUNT];
    u = (int)(g0 / (unsigned)ntot);
    c = (int)(g0 - (unsigned long long)u * (unsigned)ntot);
    step = step_;
  }
  __device__ __forceinline__ void next() {
    c += step;
    while (c >= ntot) {
      c -= ntot;
      ++u;
    }
  }
};

// The chunk (u, c) decoded (no 64-bit arithmetic).
__device__ __forceinline__ Chunk chunk_view(const Geo& G, int u, int c) {
  Chunk v;
  v.u = u;
  v.c = c;
  int kd = 0;
  while (c >= G.off[kd + 1]) ++kd;
  v.kind = kd;
  v.j = c - G.off[kd];
  v.k = 0;
  v.seg = 0;
  switch (kd) {
    case K_ROUTER: {
      const int rb = v.j / G.rseg;
      v.seg = v.j - rb * G.rseg;
      v.r0 = rb * G.rrows;
      v.n = min(G.rrows, G.nr - v.r0);
      break;
    }
    case K_SGU:
      v.r0 = v.j * G.R;
      v.n = min(G.R, G.I - v.r0);
      break;
    case K_RGU:
      v.k = v.j / G.nb;
      v.r0 = (v.j - v.k * G.nb) * G.R;
      v.n = min(G.R, G.I - v.r0);
      break;
    default:
      v.r0 = v.j * G.Rd;
      v.n = min(G.Rd, G.H - v.r0);
      break;
  }
  return v;
}

__device__ __forceinline__ int class_of(int kind) {
  return kind == K_ROUTER ? CL_ROUTER : (kind == K_DN ? CL_DN : CL_GU);
}

// the class whose completion means "the unit is complete"
__device__ __forceinline__ int final_class(const Geo& G) {
  return G.nseg > 0 ? CL_DN : CL_ROUTER;
}

__device__ __forceinline__ int class_lo(const Geo& G, int cls) {
  return cls == CL_ROUTER ? G.off[K_ROUTER] : (cls == CL_GU ? G.off[K_SGU] : G.off[K_DN]);
}
__device__ __forceinline__ int class_hi(const Geo& G, int cls) {
  return cls == CL_ROUTER ? G.off[K_SGU] : (cls == CL_GU ? G.off[K_DN] : G.off[K_COUNT]);
}

// number of x in [lo, hi) with x mod m == r (r < m)
__device__ __forceinline__ unsigned count_cong(unsigned long long lo, unsigned long long hi,
                                               unsigned r, unsigned m) {
  const unsigned long long a = lo > r ? (lo - r + m - 1) / m : 0ull;
  const unsigned long long b = hi > r ? (hi - r + m - 1) / m : 0ull;
  return (unsigned)(b - a);
}

__device__ __forceinline__ unsigned local_chunks(const Prog& P, const Geo& G) {
  const unsigned long long total = (unsigned long long)P.n_units * (unsigned)G.off[K_COUNT];
  return count_cong(0ull, total, blockIdx.x, gridDim.x);
}

// ------------------------------------------------------------------------------------------
// bounded waits
// ------------------------------------------------------------------------------------------
struct Smem {  // small shared state (in the misc area)
  uint64_t xbar;               // the stager's TMA barrier
  // Readiness per unit: a monotone counter (units ready so far; the truth) and an mbarrier
  // that completes one phase per unit, used only to sleep until the next increment. Waiters
  // may run several units ahead of the stager, so the counter decides, never the parity.
  uint64_t x_bar;              // raw x of the unit in XA (the router's input)
  uint64_t rt_bar;             // routing decision in rt_e / rt_w
  uint64_t xd_bar;             // raw down input [h_s | h_k] of the unit in XA
  unsigned x_ready, rt_ready, xd_ready;
  // The transforms of x (into XG) and of the down input (in place in XA) are shared by the
  // consumer warps holding the unit's chunks that need them; per unit parity, the number of
  // slices transformed so far.
  unsigned xg_done[2], xd_done[2];
  // per unit parity: the warps holding the unit's gate/up (down) chunks share its x (down
  // input) transform; the first of them (local chunk index mod 8) and how many chunks there are
  int xg_w0[2], xg_n[2], xd_w0[2], xd_n[2];
  unsigned run_n[2][CL_COUNT];  // per unit parity: this CTA's chunks of each class
  float xf[2];                 // RMSNorm factor of the unit's x (1 without a norm)
  float sigma[2];              // sigmoid(g . x) of the unit (1 without a shared gate)
  volatile int abort;
  unsigned run_cnt[CL_COUNT];  // chunks of the current run of each class finished here
  int rt_e[2][kMaxK];          // routing of unit u (index u & 1): experts and weights
  float rt_w[2][kMaxK];
};

__device__ __forceinline__ void raise_error(const Prog& P, Smem* sm, int code) {
  atomicCAS(P.s.err, 0, code);
  sm->abort = 1;
}

// Spin until *a - target >= 0 (wrap-safe) on a gpu-scope counter, the budget runs out, the
// CTA aborts or another CTA has recorded an error.
// Polls with relaxed loads (an acquire per poll would be a gpu-scope ordering operation each
// time) and makes one acquire fence once the flag is seen.
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
    __nanosleep(64);
  }
}

__device__ __forceinline__ bool wait_mbar(const Prog& P, Smem* sm, uint64_t* bar, unsigned parity,
                                          int code) {
  if (mbar_try_wait(bar, parity)) return true;
  // back off between polls: every poll is a shared-memory operation that competes with the
  // working warps' loads
  const uint64_t deadline = global_ns() + P.wait_ns;
  unsigned ns = 32;
  for (;;) {
    __nanosleep(ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (sm->abort) return false;
    if (global_ns() > deadline) {
      raise_error(P, sm, code);
      return false;
    }
    ns = ns < 256 ? 2 * ns : 256;
  }
}

// Wait until the readiness counter *cnt reaches target. Sleeps on the phase that the next
// increment completes (the stager stores the counter before it arrives on the barrier), and
// re-reads the counter after every wake-up or after at most ~1 us.
// Returns the counter value seen (>= target), or 0 if the wait failed.
__device__ __noinline__ unsigned wait_ready(const Prog& P, Smem* sm, const unsigned* cnt,
                                            uint64_t* bar, unsigned target, int code) {
  unsigned c = ld_acquire_cta_smem(cnt);
  if ((int)(c - target) >= 0) return c;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (;;) {
    if (!mbar_try_wait_sleep(bar, c & 1u, 1000u)) __nanosleep(256);
    c = ld_acquire_cta_smem(cnt);
    if ((int)(c - target) >= 0) return c;
    if (sm->abort) return 0u;
    if (global_ns() > deadline) {
      raise_error(P, sm, code);
      return 0u;
    }
  }
}

// Wait until the shared counter *cnt reaches target (a few warps' transform shares away).
__device__ __noinline__ bool wait_count(const Prog& P, Smem* sm, const unsigned* cnt,
                                        unsigned target, int code) {
  if (ld_acquire_cta_smem(cnt) >= target) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (;;) {
    __nanosleep(64);
    if (ld_acquire_cta_smem(cnt) >= target) return true;
    if (sm->abort) return false;
    if (global_ns() > deadline) {
      raise_error(P, sm, code);
      return false;
    }
  }
}

// the stager's side: publish "unit u is ready" on a counter and wake sleepers
__device__ __forceinline__ void signal_ready(unsigned* cnt, uint64_t* bar, int u) {
  st_release_cta_smem(cnt, (unsigned)(u + 1));
  mbar_arrive(bar);
}

// Whole-warp wrappers: lane 0 waits, every lane gets the verdict, and what was published
// before the counter's value is visible to every lane afterwards.
// Class cls complete for `units` units: its counter has reached units * (chunks per unit).
__device__ __forceinline__ bool warp_wait_class(const Prog& P, const Geo& G, Smem* sm, int cls,
                                                unsigned units, int code) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0)
    ok = spin_geq(P, sm, P.s.ctrl + cnt_word(cls), units * (unsigned)G.ncl[cls], code);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Returns the number of ready units seen (>= target), or 0 if the wait failed.
__device__ __forceinline__ unsigned warp_wait_ready(const Prog& P, Smem* sm, const unsigned* cnt,
                                                    uint64_t* bar, unsigned target, int code) {
  unsigned c = 0;
  if ((threadIdx.x & 31) == 0) c = wait_ready(P, sm, cnt, bar, target, code);
  c = __shfl_sync(0xffffffffu, c, 0);
  __syncwarp();
  return c;
}

__device__ __forceinline__ bool warp_wait_count(const Prog& P, Smem* sm, const unsigned* cnt,
                                                unsigned target, int code) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_count(P, sm, cnt, target, code);
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

// ------------------------------------------------------------------------------------------
// completion of a chunk: counted per run of same-class chunks, published per run
// ------------------------------------------------------------------------------------------
// Called by the whole warp after the global stores of its last chunk of a run were issued,
// with `mine` = the number of chunks of the run this warp did. One CTA-scope release-acquire
// add per warp and run; the warp that completes the CTA's run of (unit, class) has acquired
// every warp's stores of the run and adds the run's chunks to the class counter with one
// gpu-scope release-acquire atomic (withheld for the router class under the timeout-test
// flag, so that the routing decision never comes).
__device__ __forceinline__ void finish_run(const Prog& P, const Geo& G, Smem* sm, int cls, int u,
                                           unsigned mine) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    const unsigned old = atom_add_acq_rel_cta_smem(&sm->run_cnt[cls], mine);
    const unsigned nrun = sm->run_n[u & 1][cls];  // recorded by the stager before x(u)
    if (old + mine == nrun) {
      atom_exch_cta_smem(&sm->run_cnt[cls], 0u);
      if (!(cls == CL_ROUTER && (P.debug & 1)))
        atom_add_acq_rel_gpu(P.s.ctrl + cnt_word(cls), nrun);
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------------------------------------
// producer: stream the rows of this CTA's chunks into the ring (lane 0 of warp 0)
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void copy_rows(uint8_t* dst, const uint8_t* src, unsigned bytes,
                                          uint64_t* bar) {
  if (bytes) tma_load_1d(dst, src, bytes, bar);
}

// One bulk copy of a chunk: copy number q of the chunk (q < copies_of(chunk)). Returns the
// byte count (0 when chunk has no copy q) and sets the source and the offset in the stage.
__device__ __forceinline__ unsigned copy_desc(const Geo& G, const LayerW& L, const Smem* sm,
                                              const Chunk& cv, int q, const uint8_t** src,
                                              unsigned* dst_off) {
  switch (cv.kind) {
    case K_ROUTER: {
      if (G.rseg == 1) {  // whole rows r0 .. r0+n-1; row E is the shared-gate vector
        const unsigned rowb = 4u * (unsigned)G.H;
        const int a = cv.r0, b = min(cv.r0 + cv.n, G.E);
        if (q == 0 && b > a) {
          *src = reinterpret_cast<const uint8_t*>(L.router + (size_t)a * G.H);
          *dst_off = 0;
          return (unsigned)(b - a) * rowb;
        }
        if (q == 1 && cv.r0 + cv.n > G.E) {
          *src = reinterpret_cast<const uint8_t*>(L.gate);
          *dst_off = (unsigned)(G.E - cv.r0) * rowb;
          return rowb;
        }
        return 0u;
      }
      if (q != 0) return 0u;  // one column segment of row r0
      const float* row = cv.r0 < G.E ? L.router + (size_t)cv.r0 * G.H : L.gate;
      *src = reinterpret_cast<const uint8_t*>(row + (size_t)cv.seg * G.rcols);
      *dst_off = 0;
      return 4u * (unsigned)G.rcols;
    }
    case K_SGU:
    case K_RGU: {  // stage: gate codes | up codes | gate sb | up sb, R rows each
      if (q >= 4) return 0u;
      const uint8_t* base =
          cv.kind == K_SGU
              ? L.shared
              : L.experts + (size_t)min(max(sm->rt_e[cv.u & 1][cv.k], 0), G.E - 1) * L.expert_stride;
      const bool up = (q & 1) != 0, sbq = q >= 2;
      const size_t mat = up ? G.q_gu : 0;
      if (!sbq) {
        *src = base + mat + (size_t)cv.r0 * G.rc_h;
        *dst_off = (up ? (unsigned)G.R : 0u) * G.rc_h;
        return (unsigned)cv.n * G.rc_h;
      }
      *src = base + mat + (size_t)G.I * G.rc_h + (size_t)cv.r0 * G.rs_h;
      *dst_off = 2u * (unsigned)G.R * G.rc_h + (up ? (unsigned)G.R : 0u) * G.rs_h;
      return (unsigned)cv.n * G.rs_h;
    }
    default: {  // K_DN: per segment s (shared first, then routed k) Rd rows of codes | sb
      const int sgm = q >> 1;
      if (sgm >= G.nseg) return 0u;
      const uint8_t* eb =
          (G.shared_on && sgm == 0)
              ? L.shared
              : L.experts + (size_t)min(max(sm->rt_e[cv.u & 1][sgm - G.shared_on], 0), G.E - 1) *
                                L.expert_stride;
      const uint8_t* dn = eb + 2 * G.q_gu;
      if ((q & 1) == 0) {
        *src = dn + (size_t)cv.r0 * G.rc_i;
        *dst_off = (unsigned)sgm * G.Rd * G.rc_i;
        return (unsigned)cv.n * G.rc_i;
      }
      *src = dn + (size_t)G.H * G.rc_i + (size_t)cv.r0 * G.rs_i;
      *dst_off = (unsigned)G.nseg * G.Rd * G.rc_i + (unsigned)sgm * G.Rd * G.rs_i;
      return (unsigned)cv.n * G.rs_i;
    }
  }
}

// Bulk copies a chunk takes (some may be empty, see copy_desc) and its total bytes.
__device__ __forceinline__ int copies_of(const Geo& G, const Chunk& cv) {
  return cv.kind == K_ROUTER ? (G.rseg == 1 ? 2 : 1) : (cv.kind == K_DN ? 2 * G.nseg : 4);
}

__device__ __forceinline__ unsigned chunk_bytes(const Geo& G, const Chunk& cv) {
  switch (cv.kind) {
    case K_ROUTER:
      if (G.rseg > 1) return 4u * (unsigned)G.rcols;
      return (unsigned)cv.n * 4u * (unsigned)G.H;  // router rows and the gate row alike
    case K_SGU:
    case K_RGU:
      return 2u * (unsigned)cv.n * (G.rc_h + G.rs_h);
    default:
      return (unsigned)G.nseg * (unsigned)cv.n * (G.rc_i + G.rs_i);
  }
}

// The whole producer warp walks this CTA's chunks in order, several chunks per step: the
// lanes are dealt out to the copies of consecutive chunks (at most 8 chunks, 32 copies), the
// first lane of each chunk waits for its stage to be free and registers the chunk's bytes on
// the stage's barrier, then every lane issues its copy. Routed chunks of a unit wait, once,
// for the CTA's routing decision of that unit; a step never spans that wait.
__device__ void producer(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
  const int lane = threadIdx.x & 31;
  const unsigned NS = (unsigned)G.nstage;
  const unsigned n_local = local_chunks(P, G);
  int rt_u = -1;  // unit whose routing decision this warp has seen
  ChunkWalk cw;
  cw.init(G, blockIdx.x, (int)gridDim.x);
  unsigned i = 0;
  bool failed = false;
  while (i < n_local) {
    // Plan a step (the same plan in every lane): lane j <= 8 decodes the step's chunk j (the
    // walk advanced j chunks), a warp scan of the chunks' copy counts takes the leading
    // chunks that fit 32 copies (at most 8, never across the routing boundary of a unit), and
    // each lane picks up its copy. Planned before the wait for that routing decision, so that
    // the copies go out as soon as it is made.
    ChunkWalk wj = cw;
    const int jl = lane < 8 ? lane : 8;
    wj.c += jl * wj.step;
    while (wj.c >= wj.ntot) {
      wj.c -= wj.ntot;
      ++wj.u;
    }
    const Chunk cj = chunk_view(G, wj.u, wj.c);
    const int c0_u = __shfl_sync(0xffffffffu, cj.u, 0);
    const int c0_kind = __shfl_sync(0xffffffffu, cj.kind, 0);
    const bool wait_rt =
        (c0_kind == K_RGU || (c0_kind == K_DN && G.routed_on)) && c0_u != rt_u;
    const int bu = wait_rt ? c0_u : rt_u;  // the unit whose routing this step may use
    const bool ok_j = lane < 8 && i + (unsigned)lane < n_local &&
                      !((cj.kind == K_RGU || (cj.kind == K_DN && G.routed_on)) && cj.u != bu);
    const int nc_j = ok_j ? copies_of(G, cj) : 0;
    int incl = nc_j;  // inclusive prefix sum of the copy counts over lanes 0..lane
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const unsigned take = __ballot_sync(0xffffffffu, ok_j && incl <= 32);
    const int nb = __ffs(~take) - 1;  // leading chunks taken (chunk 0 always fits)
    int my_j = 0, my_lo = 0;
    for (int j = 0; j < 8; ++j) {
      const int ij = __shfl_sync(0xffffffffu, incl, j);
      if (j < nb && lane >= ij) my_j = j + 1, my_lo = ij;
    }
    const int my_q = my_j < nb ? lane - my_lo : -1;
    const unsigned my_i = i + (unsigned)my_j;
    Chunk my;
    my.u = __shfl_sync(0xffffffffu, cj.u, my_j);
    my.c = __shfl_sync(0xffffffffu, cj.c, my_j);
    my.kind = __shfl_sync(0xffffffffu, cj.kind, my_j);
    my.j = __shfl_sync(0xffffffffu, cj.j, my_j);
    my.r0 = __shfl_sync(0xffffffffu, cj.r0, my_j);
    my.n = __shfl_sync(0xffffffffu, cj.n, my_j);
    my.k = __shfl_sync(0xffffffffu, cj.k, my_j);
    my.seg = __shfl_sync(0xffffffffu, cj.seg, my_j);
    ChunkWalk w = cw;  // the walk after the step's nb chunks (lane nb decoded it)
    w.u = __shfl_sync(0xffffffffu, wj.u, nb);
    w.c = __shfl_sync(0xffffffffu, wj.c, nb);
    if (wait_rt) {  // the CTA's routing decision of the step's unit
      int ok = 1;
      if (lane == 0)
        ok = wait_ready(P, sm, &sm->rt_ready, &sm->rt_bar, (unsigned)(c0_u + 1),
                        DE_TIMEOUT_ROUTE) != 0u;
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        failed = true;
        break;
      }
      __syncwarp();
      rt_u = c0_u;
    }
    // stages free?
    int ok = 1;
    if (my_q == 0)
      ok = wait_mbar(P, sm, &empty[my_i % NS], ((my_i / NS) & 1u) ^ 1u, DE_TIMEOUT_EMPTY);
    if (!__all_sync(0xffffffffu, ok)) {
      failed = true;
      break;
    }
    if (my_q == 0) mbar_arrive_expect_tx(&full[my_i % NS], chunk_bytes(G, my));
    __syncwarp();
    if (my_q >= 0) {
      const LayerW& L = P.layers[my.u % P.n_layers];
      const uint8_t* src = nullptr;
      unsigned dst_off = 0;
      const unsigned bytes = copy_desc(G, L, sm, my, my_q, &src, &dst_off);
      if (bytes)
        tma_load_1d(smem + G.o_ring + (size_t)(my_i % NS) * G.stage_bytes + dst_off, src, bytes,
                    &full[my_i % NS]);
    }
    __syncwarp();
    i += (unsigned)nb;
    cw = w;
  }
  // never leave the CTA with bulk copies in flight: wait for the last copies of every stage
  if (lane == 0 && failed) {
    const uint64_t deadline = global_ns() + 100000000ull;
    const unsigned first = i > NS ? i - NS : 0u;
    for (unsigned j = first; j < i; ++j) {
      const int st = (int)(j % NS);
      while (!mbar_try_wait(&full[st], (j / NS) & 1u)) {
        if (global_ns() > deadline) {
          atomicCAS(P.s.err, 0, DE_TIMEOUT_DRAIN);
          return;
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// top-K (stager warp)
// ------------------------------------------------------------------------------------------
// Order-preserving 64-bit key of a binary64 value (larger value <=> larger unsigned key).
__device__ __forceinline__ unsigned long long dkey(double d) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(d);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Packed selection key: the upper 51 bits of the logit's key, then 13 bits of (8191 - e), so
// that one unsigned compare orders by logit and breaks exact ties toward the lower index.
// Dropping 13 low mantissa bits merges logits that differ by less than ~2^-39 relative, far
// inside the tie band where either order is correct.
__device__ __forceinline__ unsigned long long pkey(double l, int e) {
  return (dkey(l) & ~0x1FFFull) | (unsigned long long)(0x1FFF - e);
}

__device__ __forceinline__ double dkey_inv(unsigned long long k) {
  const unsigned long long b = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double((long long)b);
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

// Sort 16 keys in descending order (bitonic network: 80 independent compare-exchanges in 10
// layers, fully unrolled so the layers' exchanges overlap).
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

// logit of expert e: the sum of its column-segment partials, in segment order
__device__ __forceinline__ double unit_logit(const Geo& G, const double* lg, int e) {
  double a = 0.0;
  for (int s = 0; s < G.rseg; ++s) a += __ldcg(lg + (size_t)s * G.nr + e);
  return a;
}

// Top-K over at most 512 experts by one warp (lane l holds experts l + 32 i). K rounds: the
// warp maximum of the lanes' best packed keys (pkey: the binary64 logit's order-preserving key
// with its 13 lowest bits replaced by 8191 - e, so that one unsigned compare orders by logit and
// breaks ties toward the lower index; logits within ~2^-39 relative of each other count as
// tied, far inside the 1e-6 band where either order is correct, at any logit magnitude), taken
// as two 32-bit warp reductions (high word, then low word among the lanes holding that high
// word). The winners' binary64 logits are carried along for the weights
// w_k = exp(l_k - l_max) / sum_sel exp(l_j - l_max): the softmax over all experts followed by
// renormalisation over the selected ones, where the full softmax denominator cancels.
__device__ void topk_warp_512(const Geo& G, const double* lg, const float* bias, int* rt_e,
                              float* rt_w, int* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = 16;
  double lv[kPer], p1[kPer];
  float bv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {  // the bias and the first two segments in one round trip
    const int ec = min(lane + 32 * i, G.E - 1);
    bv[i] = bias ? __ldcg(bias + ec) : 0.f;
    lv[i] = __ldcg(lg + ec);
    p1[i] = G.rseg > 1 ? __ldcg(lg + (size_t)G.nr + ec) : 0.0;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) lv[i] = ((double)bv[i] + lv[i]) + p1[i];
  for (int sg = 2; sg < G.rseg; ++sg) {
    double part[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) part[i] = __ldcg(lg + (size_t)sg * G.nr + min(lane + 32 * i, G.E - 1));
#pragma unroll
    for (int i = 0; i < kPer; ++i) lv[i] += part[i];
  }
  unsigned long long key[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) key[i] = lane + 32 * i < G.E ? pkey(lv[i], lane + 32 * i) : 0ull;
  // the lane's best: largest key (the lowest index among equal logits by construction)
  auto lane_best = [&](unsigned long long& bk, int& bi) {
    bk = key[0];
    bi = 0;
#pragma unroll
    for (int i = 1; i < kPer; ++i)
      if (key[i] > bk) bk = key[i], bi = i;
  };
  unsigned long long bk;
  int bi;
  lane_best(bk, bi);
  int sel_e = 0;
  double sel_l = 0.0;
  for (int k = 0; k < G.K; ++k) {
    const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(bk >> 32));
    const unsigned lo =
        __reduce_max_sync(0xffffffffu, (unsigned)(bk >> 32) == hi ? (unsigned)bk : 0u);
    const unsigned long long win = ((unsigned long long)hi << 32) | lo;
    const int we = 0x1FFF - (int)(win & 0x1FFFull);  // winning expert
    const bool mine_w = bk == win && win != 0ull;     // exactly one lane holds it
    double wl = 0.0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) wl = (mine_w && i == bi) ? lv[i] : wl;
    wl = __shfl_sync(0xffffffffu, wl, we & 31);
    if (mine_w) {
#pragma unroll
      for (int i = 0; i < kPer; ++i) key[i] = i == bi ? 0ull : key[i];
      lane_best(bk, bi);
    }
    if (lane == k) {
      sel_e = we;
      sel_l = wl;
    }
  }
  const double l0 = __shfl_sync(0xffffffffu, sel_l, 0);
  const bool mine = lane < G.K;
  const float ex = mine ? expf((float)(sel_l - l0)) : 0.f;
  float den = ex;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (mine) {
    const int e = min(max(sel_e, 0), G.E - 1);  // NaN logits must not make an address
    const float wk = __fdividef(ex, den);
    rt_e[lane] = e;
    rt_w[lane] = wk;
    if (idx_out) idx_out[lane] = e;
    if (w_out) w_out[lane] = wk;
  }
  __syncwarp();
}

// Top-K of the unit's logits by one warp for more than 512 experts. Every lane sorts its 16
// packed keys; passes over 512 experts at a time keep each lane's best 16 by a bitonic merge.
// Then K rounds of a warp maximum over the lanes' heads (two 32-bit reductions), the winning
// lane dropping its head. The weights as in topk_warp_512; the logits come back from the keys
// with 40 significant bits.
__device__ void topk_warp(const Geo& G, const double* lg, const float* bias, int* rt_e,
                          float* rt_w, int* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = 16;
  unsigned long long best[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) best[i] = 0ull;
  for (int e0 = 0; e0 < G.E; e0 += 32 * kPer) {
    // the bias and the first two segments' partials are loaded together (one round trip)
    double lv[kPer], p1[kPer];
    float bv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int ec = min(e0 + lane + 32 * i, G.E - 1);
      bv[i] = bias ? __ldcg(bias + ec) : 0.f;
      lv[i] = __ldcg(lg + ec);
      p1[i] = G.rseg > 1 ? __ldcg(lg + (size_t)G.nr + ec) : 0.0;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) lv[i] = ((double)bv[i] + lv[i]) + p1[i];
    for (int s = 2; s < G.rseg; ++s) {
      double part[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        part[i] = __ldcg(lg + (size_t)s * G.nr + min(e0 + lane + 32 * i, G.E - 1));
#pragma unroll
      for (int i = 0; i < kPer; ++i) lv[i] += part[i];
    }
    unsigned long long key[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = e0 + lane + 32 * i;
      key[i] = e < G.E ? pkey(lv[i], e) : 0ull;
    }
    if (G.E <= 32 * kPer) {  // one block: the lane's 16 keys are its candidates, unsorted
#pragma unroll
      for (int i = 0; i < kPer; ++i) best[i] = key[i];
    } else {
      // keep each lane's 16 largest keys: both lists sorted descending, best[i] vs key[15-i]
      // is a bitonic sequence holding the 16 largest, which one more sort puts in order
      sort16_desc(key);
      if (e0 == 0) {
#pragma unroll
        for (int i = 0; i < kPer; ++i) best[i] = key[i];
      } else {
#pragma unroll
        for (int i = 0; i < kPer; ++i) best[i] = umax64(best[i], key[kPer - 1 - i]);
        sort16_desc(best);
      }
    }
  }
  // K rounds: the warp maximum of the lanes' largest candidates (two 32-bit reductions); the
  // lane that held it drops it and finds its next largest
  unsigned long long m = 0ull;
#pragma unroll
  for (int i = 0; i < kPer; ++i) m = umax64(m, best[i]);
  int sel_e = 0;  // lane k < K ends up holding winner k
  unsigned long long sel_k = 0ull;
  for (int k = 0; k < G.K; ++k) {
    const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(m >> 32));
    const unsigned lo =
        __reduce_max_sync(0xffffffffu, (unsigned)(m >> 32) == hi ? (unsigned)m : 0u);
    const unsigned long long win = ((unsigned long long)hi << 32) | lo;
    if (m == win && win != 0ull) {
      unsigned long long nm = 0ull;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        best[i] = best[i] == win ? 0ull : best[i];
        nm = umax64(nm, best[i]);
      }
      m = nm;
    }
    if (lane == k) {
      sel_k = win;
      sel_e = 0x1FFF - (int)(win & 0x1FFFull);
    }
  }
  const double l0 = dkey_inv(__shfl_sync(0xffffffffu, sel_k, 0) & ~0x1FFFull);
  const bool mine = lane < G.K;
  const float ex = mine ? expf((float)(dkey_inv(sel_k & ~0x1FFFull) - l0)) : 0.f;
  float den = ex;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (mine) {
    const int e = min(max(sel_e, 0), G.E - 1);  // NaN logits must not make an address
    const float wk = __fdividef(ex, den);
    rt_e[lane] = e;
    rt_w[lane] = wk;
    if (idx_out) idx_out[lane] = e;
    if (w_out) w_out[lane] = wk;
  }
  __syncwarp();
}

// ------------------------------------------------------------------------------------------
// stager warp: per unit, x in, routing decision, down input
// ------------------------------------------------------------------------------------------
// Position of float4 number i of 32-column slice t in a transformed vector: swizzled so that
// the 8 lanes of a quarter-warp reading "float4 i of their own slices" hit distinct banks.
__device__ __forceinline__ int xpos(int t, int i) { return 32 * t + 4 * (i ^ (t & 7)); }

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

// Column of byte b of digit word n of a slice, matching the bytes the slice kernels cut from
// a code word: at 4 bits word n pairs with the low (n even) or high (n odd) nibbles of code
// word n/2 (columns 8(n/2) + 2b + n%2); at 2 bits with bit-plane n%4 of code word n/4
// (columns 16(n/4) + 4b + n%4).
template <int BITS>
__device__ __forceinline__ constexpr int digit_col(int n, int b) {
  return BITS == 4 ? 8 * (n >> 1) + 2 * b + (n & 1) : 16 * (n >> 2) + 4 * b + (n & 3);
}

// The digit form of one 32-value slice v (already scaled): scale s = max|v| / 127 and the
// digits of v/s, so that v ~ s * (d0 + d1/128 + d2/16384) to within 1e-6 * max|v|. Chunk
// i < 6 of the slice (at xpos(t, i)) holds digit plane i/2, words 4(i%2) .. 4(i%2)+3; chunk 6
// holds {s, sum of v}.
template <int BITS>
__device__ __forceinline__ void store_digits(const float (&v)[32], float* xt, int t) {
  float mq[4] = {0.f, 0.f, 0.f, 0.f}, sq[4] = {0.f, 0.f, 0.f, 0.f};  // four short chains each
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    mq[j & 3] = fmaxf(mq[j & 3], fabsf(v[j]));
    sq[j & 3] += v[j];
  }
  const float m = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
  const float sum = (sq[0] + sq[1]) + (sq[2] + sq[3]);
  // 127 * 2^14 / max|v|; a few ulp of error in k only shift |q| by a few units near its
  // limit, which the digit ranges absorb, and the scale below is taken from m directly
  const float k = m > 0.f ? __fdividef(2080768.f, m) : 0.f;
  uint32_t w[3][8];
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    int d[3][4];
#pragma unroll
    for (int b = 0; b < 4; ++b) digits3(v[digit_col<BITS>(n, b)], k, d[0][b], d[1][b], d[2][b]);
#pragma unroll
    for (int p = 0; p < 3; ++p) w[p][n] = pack4(d[p][0], d[p][1], d[p][2], d[p][3]);
  }
#pragma unroll
  for (int i = 0; i < 6; ++i) {
    const int p = i >> 1, n0 = 4 * (i & 1);
    *reinterpret_cast<uint4*>(xt + xpos(t, i)) =
        make_uint4(w[p][n0], w[p][n0 + 1], w[p][n0 + 2], w[p][n0 + 3]);
  }
  *reinterpret_cast<float2*>(xt + xpos(t, 6)) = make_float2(m * (1.f / 127.f), sum);
}

// Bring up to two blocks from global memory (written by other CTAs or by the caller) into
// shared memory with bulk copies on one barrier, and wait for both.
__device__ __forceinline__ bool stage_in(const Prog& P, Smem* sm, void* dst, const void* src,
                                         unsigned bytes, unsigned& xphase,
                                         void* dst2 = nullptr, const void* src2 = nullptr,
                                         unsigned bytes2 = 0) {
  if ((threadIdx.x & 31) == 0) {
    fence_proxy_async();  // order earlier generic accesses before the async-proxy copies
    mbar_arrive_expect_tx(&sm->xbar, bytes + bytes2);
    if (bytes) tma_load_1d(dst, src, bytes, &sm->xbar);
    if (bytes2) tma_load_1d(dst2, src2, bytes2, &sm->xbar);
  }
  const bool ok = warp_wait_mbar(P, sm, &sm->xbar, xphase, DE_TIMEOUT_DEP);
  xphase ^= 1u;
  return ok;
}

// Share r (of ns) of a transform: slices [r*nsl/ns, (r+1)*nsl/ns) of the raw values in `raw`
// (linear layout), slice t scaled by scale_of(t), go into `xt` in digit form (store_digits).
// One lane per slice; raw and xt may be the same array (a lane reads its whole slice before
// it writes it). Returns the number of slices done.
template <typename ScaleOf>
__device__ __forceinline__ int transform_share(const float* raw, float* xt, int nsl, int r,
                                               int ns, int bits, ScaleOf scale_of) {
  const int lane = threadIdx.x & 31;
  const int t0 = r * nsl / ns, t1 = (r + 1) * nsl / ns;
  for (int t = t0 + lane; t < t1; t += 32) {
    const float f = scale_of(t);
    float v[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 a = *reinterpret_cast<const float4*>(raw + 32 * t + 4 * q);
      v[4 * q] = a.x * f; v[4 * q + 1] = a.y * f; v[4 * q + 2] = a.z * f; v[4 * q + 3] = a.w * f;
    }
    if (bits == 4)
      store_digits<4>(v, xt, t);
    else
      store_digits<2>(v, xt, t);
  }
  __syncwarp();
  return t1 - t0;
}

// Local index range [lo, hi) of this CTA's chunks with unit index in [u*ntot + c0, u*ntot + c1).
__device__ __forceinline__ void local_range(const Geo& G, int u, int c0, int c1, unsigned* lo,
                                            unsigned* hi) {
  const unsigned long long base = (unsigned long long)u * (unsigned)G.off[K_COUNT];
  *lo = count_cong(0ull, base + (unsigned)c0, blockIdx.x, gridDim.x);
  *hi = *lo + count_cong(base + (unsigned)c0, base + (unsigned)c1, blockIdx.x, gridDim.x);
}

// The share of consumer warp w among the n_sh warps that hold a range of n chunks whose first
// local chunk goes to warp w0 (local chunk i -> warp i mod 8); the caller holds one of them.
__device__ __forceinline__ int share_rank(int w0, int n, int w, int* n_sh) {
  *n_sh = n < kConsumerWarps ? n : kConsumerWarps;
  return n < kConsumerWarps ? (w - w0 + kConsumerWarps) % kConsumerWarps : w;
}

// The scale of down-input slice t: sigma for the shared expert's segment, w_k for routed k.
__device__ __forceinline__ float xd_scale(const Geo& G, const Smem* sm, int u, int t) {
  const int s = t / (G.I / 32);
  return (G.shared_on && s == 0) ? sm->sigma[u & 1] : sm->rt_w[u & 1][s - G.shared_on];
}

__device__ void stager(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm) {
  const int lane = threadIdx.x & 31;
  float* XA = reinterpret_cast<float*>(smem + G.o_xa);
  float* XG = reinterpret_cast<float*>(smem + G.o_xg);
  const int fcl = final_class(G);
  const unsigned ntot = (unsigned)G.off[K_COUNT];
  const bool gu_on = G.shared_on || G.routed_on;
  unsigned xphase = 0;
  (void)lane;
  for (int u = 0; u < P.n_units; ++u) {
    const UnitView uv = unit_view(P, G, u);
    const bool owner = ((unsigned long long)u * ntot) % gridDim.x == blockIdx.x;
    // ---- x(u): needs unit u-1 complete (its output is this input, its buffers are free)
    if (u > 0 && !warp_wait_class(P, G, sm, fcl, (unsigned)u, DE_TIMEOUT_DEP)) break;
    float f = 1.f;
    if (uv.norm) f = rsqrtf(__ldcg(P.s.normsq + (u - 1)) / (float)G.H + P.eps);
    if (!stage_in(P, sm, XA, uv.xin, 4u * (unsigned)G.H, xphase)) break;
    if (owner && uv.h_trace)
      for (int c = lane * 4; c < G.H; c += 128)
        *reinterpret_cast<float4*>(uv.h_trace + c) = *reinterpret_cast<const float4*>(XA + c);
    if (lane == 0) {
      unsigned lo, hi;
      sm->xf[u & 1] = f;
      sm->xg_done[u & 1] = 0u;
      local_range(G, u, G.off[K_SGU], G.off[K_DN], &lo, &hi);
      sm->xg_w0[u & 1] = (int)(lo % kConsumerWarps);
      sm->xg_n[u & 1] = (int)(hi - lo);
      sm->run_n[u & 1][CL_GU] = hi - lo;
      local_range(G, u, G.off[K_DN], G.off[K_COUNT], &lo, &hi);
      sm->xd_w0[u & 1] = (int)(lo % kConsumerWarps);
      sm->xd_n[u & 1] = (int)(hi - lo);
      sm->run_n[u & 1][CL_DN] = hi - lo;
      local_range(G, u, G.off[K_ROUTER], G.off[K_SGU], &lo, &hi);
      sm->run_n[u & 1][CL_ROUTER] = hi - lo;
    }
    __syncwarp();
    if (lane == 0) signal_ready(&sm->x_ready, &sm->x_bar, u);
    // ---- routing decision: needs every router chunk of unit u
    float sigma = 1.f;
    if (G.route_on) {
      // the unit's logit bias into L2 while the router runs (it streams from HBM otherwise)
      if (uv.bias)
        for (int e = lane * 32; e < G.E; e += 32 * 32) prefetch_l2(uv.bias + e);
      if (!warp_wait_class(P, G, sm, CL_ROUTER, (unsigned)(u + 1), DE_TIMEOUT_ROUTE)) break;
      const double* lg = P.s.logits + (size_t)uv.slot * G.rseg * G.nr;
      if (G.E <= 512)
        topk_warp_512(G, lg, uv.bias, sm->rt_e[u & 1], sm->rt_w[u & 1],
                      owner ? uv.idx_out : nullptr, owner ? uv.w_out : nullptr);
      else
        topk_warp(G, lg, uv.bias, sm->rt_e[u & 1], sm->rt_w[u & 1], owner ? uv.idx_out : nullptr,
                  owner ? uv.w_out : nullptr);
      __syncwarp();
      if (lane == 0) signal_ready(&sm->rt_ready, &sm->rt_bar, u);
      // sigma(g . x) (the shared-gate row is router row E) is needed only by the down input
      if (G.gate_on) sigma = (float)(1.0 / (1.0 + exp(-unit_logit(G, lg, G.E))));
      if (lane == 0) sm->sigma[u & 1] = sigma;
    }
    // ---- down input [sigma*h_s | w_0*h_0 | ...]: needs every gate/up chunk of unit u
    if (G.nseg > 0) {
      if (!warp_wait_class(P, G, sm, CL_GU, (unsigned)(u + 1), DE_TIMEOUT_DEP)) break;
      const unsigned bs = G.shared_on ? 4u * (unsigned)G.I : 0u;
      const unsigned bk = G.routed_on ? 4u * (unsigned)(G.K * G.I) : 0u;
      if (lane == 0) {
        sm->xd_done[u & 1] = 0u;
        if (!G.route_on) sm->sigma[u & 1] = 1.f;
      }
      if (!stage_in(P, sm, XA, P.s.hs + (size_t)uv.slot * G.I, bs, xphase,
                    XA + (size_t)G.shared_on * G.I, P.s.hk + (size_t)uv.slot * G.K * G.I, bk))
        break;
      __syncwarp();
      if (lane == 0) signal_ready(&sm->xd_ready, &sm->xd_bar, u);
    }
  }
}

// ------------------------------------------------------------------------------------------
// dequantising dot products: W rows x one 32-column slice
// ------------------------------------------------------------------------------------------
// acc[w] += s_w * sum(q x) + z_w * sum(x) over the slice, for W rows whose codes start at
// stage + coff[w] and whose scale/bias word is at stage + soff[w]; rows with ok[w] false add
// 0 (their offsets must still point inside the stage). sum(q x) comes from integer dot
// products of the codes with the slice's three digit planes xd (store_digits), scaled by sc;
// sx is sum(x).
template <int BITS, int W>
__device__ __forceinline__ void qslice(uint32_t stage, const unsigned (&coff)[W],
                                       const unsigned (&soff)[W], const bool (&ok)[W],
                                       const int (&xd)[24], float sc, float sx, float* acc) {
  constexpr int kWords = BITS == 4 ? 4 : 2;
  uint32_t q[W][kWords];
  uint32_t sbw[W];
#pragma unroll
  for (int w = 0; w < W; ++w) {
    if constexpr (BITS == 4) {
      const uint4 t = lds128(stage + coff[w]);
      q[w][0] = t.x; q[w][1] = t.y; q[w][2] = t.z; q[w][3] = t.w;
    } else {
      const uint2 t = lds64(stage + coff[w]);
      q[w][0] = t.x; q[w][1] = t.y;
    }
    sbw[w] = lds32(stage + soff[w]);
  }
  int c0[W], c1[W], c2[W];
#pragma unroll
  for (int w = 0; w < W; ++w) c0[w] = c1[w] = c2[w] = 0;
#pragma unroll
  for (int wi = 0; wi < kWords; ++wi) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
      if constexpr (BITS == 4) {  // low nibbles: digit word 2wi, high nibbles: 2wi + 1
        const int lo = (int)(q[w][wi] & 0x0F0F0F0Fu);
        const int hi = (int)((q[w][wi] >> 4) & 0x0F0F0F0Fu);
        c0[w] = __dp4a(hi, xd[2 * wi + 1], __dp4a(lo, xd[2 * wi], c0[w]));
        c1[w] = __dp4a(hi, xd[8 + 2 * wi + 1], __dp4a(lo, xd[8 + 2 * wi], c1[w]));
        c2[w] = __dp4a(hi, xd[16 + 2 * wi + 1], __dp4a(lo, xd[16 + 2 * wi], c2[w]));
      } else {  // bit-plane p of code word wi: digit word 4wi + p
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int c = (int)((q[w][wi] >> (2 * p)) & 0x03030303u);
          c0[w] = __dp4a(c, xd[4 * wi + p], c0[w]);
          c1[w] = __dp4a(c, xd[8 + 4 * wi + p], c1[w]);
          c2[w] = __dp4a(c, xd[16 + 4 * wi + p], c2[w]);
        }
      }
    }
  }
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const float s = __uint_as_float(sbw[w] << 16);
    const float z = __uint_as_float(sbw[w] & 0xFFFF0000u);
    const float qx =
        sc * ((float)c0[w] + ((float)c1[w] * 0.0078125f + (float)c2[w] * 6.103515625e-05f));
    acc[w] += ok[w] ? fmaf(s, qx, z * sx) : 0.f;
  }
}

// Transposing butterfly over `width` lanes (a power of two <= 32): W row partials per lane
// become one fully reduced value per distinct row; results land in red[lo + i].
template <int W>
__device__ __forceinline__ void reduce_rows(float (&v)[W], int lane_in_seg, int width,
                                            float* red) {
  int lo = 0;
  int nlive = W;
#pragma unroll
  for (int i = 0; (1 << i) < W; ++i) {
    const int o = 1 << i;
    const int half = (W >> i) >> 1;
    if (o < width) {
      const bool upper = (lane_in_seg & o) != 0;
#pragma unroll
      for (int a = 0; a < (W >> 1); ++a) {
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
    for (int o = W; o < width; o <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    if (lane_in_seg < W && lane_in_seg < width) red[lo] = v[0];
  } else {
#pragma unroll
    for (int a = 0; a < W; ++a)
      if (a < nlive) red[lo + a] = v[a];
  }
}

// Where a chunk's rows live in its stage.
struct RowGeom {
  unsigned rc, rs;        // row strides (codes, sb) inside a segment
  unsigned seg_c, seg_s;  // segment strides (codes, sb)
  unsigned sb0;           // offset of the sb area
  int spseg;              // slices per segment
};

// A chunk's rows x slices on one warp: rows rho = lane_p + P*i (i < NRL), slices
// t = lane_s + S*j; rows are processed in lock-step groups of GW (3 or 4) per slice. Row rho
// takes part when valid(rho). The reduced value of row rho ends in
// red[(rho % P) * kRowsPerLane + rho / P].
template <int BITS, int NRL, typename Valid>
__device__ __forceinline__ void dot_chunk(uint32_t st, const LaneMap& M, const RowGeom& RG,
                                          int nrows, Valid valid, uint32_t xs,
                                          float* red) {
  constexpr int NRLP = NRL <= 4 ? 4 : 8;         // padded to a power of two for the butterfly
  constexpr int GW = (NRL % 4 == 0) ? 4 : 3;     // rows per lock-step group
  const int lane = threadIdx.x & 31;
  const int lane_s = lane & (M.S - 1), lane_p = lane / M.S;
  constexpr unsigned cb = BITS == 4 ? 16u : 8u;
  float acc[NRLP];
#pragma unroll
  for (int i = 0; i < NRLP; ++i) acc[i] = 0.f;
  const int nj = (M.nsl + M.S - 1) / M.S;
  for (int j = 0; j < nj; ++j) {
    const int t = lane_s + M.S * j;
    const bool tok = t < M.nsl;
    const int tc = tok ? t : M.nsl - 1;
    int xd[24];
#pragma unroll
    for (int i = 0; i < 6; ++i) {
      const uint4 a = lds128(xs + 4u * (unsigned)xpos(tc, i));
      xd[4 * i] = (int)a.x; xd[4 * i + 1] = (int)a.y; xd[4 * i + 2] = (int)a.z;
      xd[4 * i + 3] = (int)a.w;
    }
    const uint2 ss = lds64(xs + 4u * (unsigned)xpos(tc, 6));
    const float sc = __uint_as_float(ss.x), sx = __uint_as_float(ss.y);
    const int seg = tc / RG.spseg, loc = tc - seg * RG.spseg;
    const unsigned cbase = (unsigned)seg * RG.seg_c + (unsigned)loc * cb;
    const unsigned sbase = RG.sb0 + (unsigned)seg * RG.seg_s + (unsigned)(loc >> 1) * 4u;
#pragma unroll
    for (int g = 0; g < NRL; g += GW) {
      if (g == 0 || M.P * g < nrows) {  // some lane has rows in this group
        unsigned coff[GW], soff[GW];
        bool ok[GW];
#pragma unroll
        for (int w = 0; w < GW; ++w) {
          const int rho = lane_p + M.P * (g + w);
          ok[w] = tok && valid(rho);
          const unsigned rr = ok[w] ? (unsigned)rho : 0u;
          coff[w] = cbase + rr * RG.rc;
          soff[w] = sbase + rr * RG.rs;
        }
        qslice<BITS, GW>(st, coff, soff, ok, xd, sc, sx, acc + g);
      }
    }
  }
  reduce_rows<NRLP>(acc, lane_s, M.S, red + lane_p * kRowsPerLane);
}

__device__ __forceinline__ float red_row(const float* red, const LaneMap& M, int rho) {
  return red[(rho % M.P) * kRowsPerLane + rho / M.P];
}

// ------------------------------------------------------------------------------------------
// consumer warps
// ------------------------------------------------------------------------------------------
// Every lane's reads of the stage have returned (their values fed the row sums already
// reduced across the warp), so a relaxed arrival is enough to hand the stage back.
__device__ __forceinline__ void release_stage(uint64_t* empty) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_relaxed(empty);
}

// router rows r0..r0+n-1, columns seg*rcols .. +rcols: binary64 sums of fp32 products
__device__ __forceinline__ void router_chunk(const Prog& P, const Geo& G, const Chunk& cv,
                                             const uint8_t* stage, uint64_t* empty,
                                             const float* XR, float xf) {
  const int lane = threadIdx.x & 31;
  const float4* xr = reinterpret_cast<const float4*>(XR + (size_t)cv.seg * G.rcols);
  const int nf = G.rcols / 4;
  double* lg = P.s.logits + ((size_t)(cv.u & 1) * G.rseg + cv.seg) * G.nr + cv.r0;
  double res = 0.0;
  for (int r = 0; r < cv.n; ++r) {
    const float4* wr = reinterpret_cast<const float4*>(stage) + (size_t)r * nf;
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    for (int f = lane; f < nf; f += 32) {
      const float4 w = wr[f], x = xr[f];
      a0 = fma((double)w.x, (double)x.x, a0);
      a1 = fma((double)w.y, (double)x.y, a1);
      a2 = fma((double)w.z, (double)x.z, a2);
      a3 = fma((double)w.w, (double)x.w, a3);
    }
    double a = (a0 + a1) + (a2 + a3);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == (r & 31)) res = a * (double)xf;  // the norm factor of x, applied to the sum
    if ((r & 31) == 31 || r == cv.n - 1) {  // flush up to 32 results, one per lane
      const int rb = r & ~31;
      if (lane <= (r & 31)) lg[rb + lane] = res;
    }
  }
  release_stage(empty);
}

template <int BITS, int NRL>
__device__ __forceinline__ void gu_chunk(const Prog& P, const Geo& G, const Chunk& cv,
                                         const uint8_t* stage, uint64_t* empty, const float* XG,
                                         float* red) {
  const int lane = threadIdx.x & 31;
  RowGeom RG;
  RG.rc = G.rc_h; RG.rs = G.rs_h; RG.seg_c = 0; RG.seg_s = 0;
  RG.sb0 = 2u * (unsigned)G.R * G.rc_h;
  RG.spseg = G.H / 32;
  const int R = G.R, n = cv.n;
  dot_chunk<BITS, NRL>(
      smem_u32(stage), G.gu, RG, 2 * R,
      [&](int rho) { return rho < 2 * R && (rho < R ? rho : rho - R) < n; }, smem_u32(XG),
      red);
  release_stage(empty);
  __syncwarp();
  float* h = cv.kind == K_SGU ? P.s.hs + (size_t)(cv.u & 1) * G.I
                              : P.s.hk + ((size_t)(cv.u & 1) * G.K + cv.k) * G.I;
  for (int r = lane; r < n; r += 32) {
    const float a = red_row(red, G.gu, r);
    const float b = red_row(red, G.gu, R + r);
    h[cv.r0 + r] = __fdividef(a, 1.f + __expf(-a)) * b;  // SwiGLU: SiLU(gate) * up
  }
  __syncwarp();
}

template <int BITS, int NRL>
__device__ __forceinline__ void dn_chunk(const Prog& P, const Geo& G, const Chunk& cv,
                                         const UnitView& uv, const uint8_t* stage,
                                         uint64_t* empty, const float* XD,
                                         float* red) {
  const int lane = threadIdx.x & 31;
  // the residual each output row adds is fetched first so its latency hides behind the dots
  const float rv = (uv.res && lane < cv.n) ? __ldcg(uv.res + cv.r0 + lane) : 0.f;
  RowGeom RG;
  RG.rc = G.rc_i; RG.rs = G.rs_i;
  RG.seg_c = (unsigned)G.Rd * G.rc_i;
  RG.seg_s = (unsigned)G.Rd * G.rs_i;
  RG.sb0 = (unsigned)G.nseg * G.Rd * G.rc_i;
  RG.spseg = G.I / 32;
  const int n = cv.n;
  dot_chunk<BITS, NRL>(smem_u32(stage), G.dn, RG, n, [&](int rho) { return rho < n; },
                       smem_u32(XD), red);
  release_stage(empty);
  __syncwarp();
  float sq = 0.f;
  for (int r = lane; r < n; r += 32) {
    const float base = r < 32 ? rv : (uv.res ? __ldcg(uv.res + cv.r0 + r) : 0.f);
    const float o = base + red_row(red, G.dn, r);
    uv.out[cv.r0 + r] = o;
    sq += o * o;
  }
  if (P.mode == MODE_STACK) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) atomicAdd(P.s.normsq + cv.u, sq);
  }
  __syncwarp();
}

// rows per lane -> the compiled variant that covers them (3, 4, 6 or 8 rows)
__device__ __forceinline__ int nrl_class(int nrl) {
  return nrl <= 3 ? 3 : (nrl == 4 ? 4 : (nrl <= 6 ? 6 : 8));
}

template <int BITS>
__device__ __forceinline__ void dispatch_dot(const Prog& P, const Geo& G, const Chunk& cv,
                                             const UnitView& uv, const uint8_t* stage,
                                             uint64_t* empty, uint8_t* smem, float* red) {
  if (cv.kind == K_DN) {
    const float* XD = reinterpret_cast<const float*>(smem + G.o_xa);
    switch (nrl_class(G.dn.nrl)) {
      case 3: dn_chunk<BITS, 3>(P, G, cv, uv, stage, empty, XD, red); break;
      case 4: dn_chunk<BITS, 4>(P, G, cv, uv, stage, empty, XD, red); break;
      case 6: dn_chunk<BITS, 6>(P, G, cv, uv, stage, empty, XD, red); break;
      default: dn_chunk<BITS, 8>(P, G, cv, uv, stage, empty, XD, red); break;
    }
  } else {
    const float* XG = reinterpret_cast<const float*>(smem + G.o_xg);
    switch (nrl_class(G.gu.nrl)) {
      case 3: gu_chunk<BITS, 3>(P, G, cv, stage, empty, XG, red); break;
      case 4: gu_chunk<BITS, 4>(P, G, cv, stage, empty, XG, red); break;
      case 6: gu_chunk<BITS, 6>(P, G, cv, stage, empty, XG, red); break;
      default: gu_chunk<BITS, 8>(P, G, cv, stage, empty, XG, red); break;
    }
  }
}

__device__ void consumer(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm, int w) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
  float* red = reinterpret_cast<float*>(smem + G.o_red) + (size_t)w * 16 * kRowsPerLane;
  float* XA = reinterpret_cast<float*>(smem + G.o_xa);
  float* XG = reinterpret_cast<float*>(smem + G.o_xg);
  const int lane = threadIdx.x & 31;
  const unsigned NS = (unsigned)G.nstage;
  const unsigned n_local = local_chunks(P, G);
  int cur_u = -1;
  UnitView uv;
  unsigned x_seen = 0, xd_seen = 0;  // units known ready (counter values already acquired)
  unsigned xg_mine = 0, xd_mine = 0; // units (+1) whose transform share this warp has done
  unsigned mine = 0;                 // chunks of the current run done by this warp
  ChunkWalk cw;
  cw.init(G, (unsigned long long)blockIdx.x + (unsigned long long)w * gridDim.x,
          kConsumerWarps * (int)gridDim.x);
  for (unsigned i = (unsigned)w; i < n_local; i += kConsumerWarps, cw.next()) {
    const int slot = (int)(i % NS);
    const Chunk cv = chunk_view(G, cw.u, cw.c);
    if (cv.u != cur_u) {
      cur_u = cv.u;
      uv = unit_view(P, G, cv.u);
    }
    const unsigned need = (unsigned)(cv.u + 1);
    // the input of the chunk; at the warp's first chunk of the unit that needs a transformed
    // input, its share of the transform, done before the chunk's weights are waited for
    bool share_wait = false;
    if (cv.kind == K_DN) {
      if ((int)(xd_seen - need) < 0) {
        xd_seen = warp_wait_ready(P, sm, &sm->xd_ready, &sm->xd_bar, need, DE_TIMEOUT_DEP);
        if (xd_seen == 0u) break;
      }
      if (xd_mine != need) {
        xd_mine = need;
        share_wait = true;
        int n_sh;
        const int rk = share_rank(sm->xd_w0[cv.u & 1], sm->xd_n[cv.u & 1], w, &n_sh);
        const int d = transform_share(XA, XA, G.nseg * (G.I / 32), rk, n_sh, G.bits,
                                      [&](int t) { return xd_scale(G, sm, cv.u, t); });
        if (lane == 0 && d) red_release_cta_smem(&sm->xd_done[cv.u & 1], (unsigned)d);
      }
    } else {
      if ((int)(x_seen - need) < 0) {
        x_seen = warp_wait_ready(P, sm, &sm->x_ready, &sm->x_bar, need, DE_TIMEOUT_DEP);
        if (x_seen == 0u) break;
      }
      if (cv.kind != K_ROUTER && xg_mine != need) {
        xg_mine = need;
        share_wait = true;
        const float f = sm->xf[cv.u & 1];
        int n_sh;
        const int rk = share_rank(sm->xg_w0[cv.u & 1], sm->xg_n[cv.u & 1], w, &n_sh);
        const int d = transform_share(XA, XG, G.H / 32, rk, n_sh, G.bits,
                                      [&](int) { return f; });
        if (lane == 0 && d) red_release_cta_smem(&sm->xg_done[cv.u & 1], (unsigned)d);
      }
    }
    if (!warp_wait_mbar(P, sm, &full[slot], (i / NS) & 1u, DE_TIMEOUT_FULL)) break;
    if (share_wait) {  // every other share of the transform
      const bool dn = cv.kind == K_DN;
      if (!warp_wait_count(P, sm, dn ? &sm->xd_done[cv.u & 1] : &sm->xg_done[cv.u & 1],
                           (unsigned)(dn ? G.nseg * (G.I / 32) : G.H / 32), DE_TIMEOUT_DEP))
        break;
    }
    const uint8_t* stage = smem + G.o_ring + (size_t)slot * G.stage_bytes;
    if (cv.kind == K_ROUTER)
      router_chunk(P, G, cv, stage, &empty[slot], XA, sm->xf[cv.u & 1]);
    else if (G.bits == 4)
      dispatch_dot<4>(P, G, cv, uv, stage, &empty[slot], smem, red);
    else
      dispatch_dot<2>(P, G, cv, uv, stage, &empty[slot], smem, red);
    ++mine;
    // publish when this warp's next chunk belongs to another (unit, class) run, or there is none
    const int cls = class_of(cv.kind);
    bool run_end = i + kConsumerWarps >= n_local;
    if (!run_end) {
      ChunkWalk nw = cw;
      nw.next();
      run_end = nw.u != cv.u || class_of(chunk_view(G, nw.u, nw.c).kind) != cls;
    }
    if (run_end) {
      finish_run(P, G, sm, cls, cv.u, mine);
      mine = 0;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    engine_kernel(const __grid_constant__ Prog P, const __grid_constant__ Geo G) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Smem* sm = reinterpret_cast<Smem*>(smem + G.o_misc);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
  if (threadIdx.x == 0) {
    sm->abort = 0;
    for (int c = 0; c < CL_COUNT; ++c) sm->run_cnt[c] = 0;
    sm->x_ready = sm->rt_ready = sm->xd_ready = 0;
    mbar_init(&sm->x_bar, 1);
    mbar_init(&sm->rt_bar, 1);
    mbar_init(&sm->xd_bar, 1);
    for (int i = 0; i < G.nstage; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&sm->xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    producer(P, G, smem, sm);
    return;
  }
  if (warp == 1) {
    stager(P, G, smem, sm);
    return;
  }
  consumer(P, G, smem, sm, warp - kCtrlWarps);
}

}  // namespace fmoe

// launcher used by the C ABI layer
extern "C" cudaError_t fmoe_engine_configure(int max_smem) {
  return cudaFuncSetAttribute(fmoe::engine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              max_smem);
}

// The CTAs of one launch wait on each other's progress, so they must all be resident at
// once: the launch is cooperative, which makes a grid that cannot be co-resident a launch
// error instead of a wait that runs out of budget.
extern "C" cudaError_t fmoe_engine_launch(const fmoe::Prog* P, const fmoe::Geo* G, int grid,
                                          cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)fmoe::kThreads);
  cfg.dynamicSmemBytes = G->smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fmoe::engine_kernel, *P, *G);
}

// CTAs of the engine kernel that fit on one SM with `smem` bytes of dynamic shared memory.
extern "C" cudaError_t fmoe_engine_occupancy(int smem, int* ctas_per_sm) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, fmoe::engine_kernel,
                                                       fmoe::kThreads, (size_t)smem);
}
