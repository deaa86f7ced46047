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
//      pour FMA").
//
// How: one CTA per SM with three roles.
//   producer warp   streams the weight rows of the CTA's chunks into a ring of shared-memory
//                   stages with 1-D TMA bulk copies completing on mbarriers;
//   8 consumer warps own fixed 32-column slices, keep the matching (pre-transformed) x values
//                   in registers, unpack codes with one byte-permute per byte into a binary32
//                   "32768 + byte" pattern and finish the exact code values with packed f32x2
//                   arithmetic; row partials are reduced with a transposing warp butterfly and
//                   across warps in shared memory, then the epilogue (SwiGLU or combine) runs;
//   signal warp     moves each chunk's epilogue results from a shared-memory outbox to global
//                   memory, publishes completions to the other CTAs (one gpu-scope fence and
//                   one reduction per run of same-phase chunks) and, in the CTA that completes
//                   the router, selects the top-K experts -- so the consumers never wait on a
//                   global store, fence or atomic.
// Every spin-wait is bounded by a global-timer budget; on expiry the kernel records an error
// word, waits for its own copies in flight and returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include "engine.h"
#include "ptx.cuh"

namespace fmoe {

constexpr int kMaxW = 8;
// Warp roles: warp 0 producer, warp 1 signal, warps 2..9 consumers. The control warps get the
// lowest warp ids so that, sharing sub-partitions with busy consumer warps, they are not
// starved of issue slots.
constexpr int kCtrlThreads = 64;
__device__ __forceinline__ int ctid() { return (int)threadIdx.x - kCtrlThreads; }

__device__ __forceinline__ int cnt_word(int phase) { return C_CNT + 32 * phase; }
// this CTA's flag word `w` (units whose phase w is complete)
__device__ __forceinline__ const unsigned* my_flag(const Prog& P, int w) {
  return P.s.flags + blockIdx.x * F_WORDS + w;
}

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

struct ChunkView {
  int u, c, phase, j, r0, n, k;
};

// The chunks of this CTA in order: g = blockIdx + it * gridDim, decoded incrementally.
struct ChunkIter {
  unsigned it, total;
  int u, c, ntot, step;
  __device__ __forceinline__ ChunkIter(const Prog& P, const Geo& G) {
    ntot = G.off[P_COUNT];
    total = (unsigned)P.n_units * (unsigned)ntot;
    step = (int)gridDim.x;
    it = 0;
    u = (int)(blockIdx.x / (unsigned)ntot);
    c = (int)(blockIdx.x - (unsigned)u * (unsigned)ntot);
  }
  __device__ __forceinline__ bool valid() const {
    return (unsigned)u * (unsigned)ntot + (unsigned)c < total;
  }
  __device__ __forceinline__ void next() {
    ++it;
    c += step;
    while (c >= ntot) {
      c -= ntot;
      ++u;
    }
  }
  __device__ __forceinline__ ChunkView view(const Geo& G) const {
    ChunkView v;
    v.u = u;
    v.c = c;
    int p = 0;
    while (c >= G.off[p + 1]) ++p;
    v.phase = p;
    v.j = c - G.off[p];
    v.k = 0;
    switch (p) {
      case P_ROUTER: v.r0 = v.j * G.rr; v.n = min(G.rr, G.nr - v.r0); break;
      case P_SGU: v.r0 = v.j * G.rcg; v.n = min(G.rcg, G.I - v.r0); break;
      case P_SDN: v.r0 = v.j * G.rsd; v.n = min(G.rsd, G.H - v.r0); break;
      case P_RGU: {
        v.k = v.j / G.nb;
        const int jj = v.j - v.k * G.nb;
        v.r0 = jj * G.rcg;
        v.n = min(G.rcg, G.I - v.r0);
        break;
      }
      default: v.r0 = v.j * G.rrd; v.n = min(G.rrd, G.H - v.r0); break;
    }
    return v;
  }
};

// the phase whose completion means "the unit is complete"
__device__ __forceinline__ int final_phase(const Geo& G) {
  return G.routed_on ? P_RDN : (G.shared_on ? P_SDN : P_ROUTER);
}

// ------------------------------------------------------------------------------------------
// bounded waits
// ------------------------------------------------------------------------------------------
struct Smem {  // small shared state (in the misc area)
  volatile int abort;
  volatile int prod_done;
  volatile unsigned issued;
  unsigned done_count;         // consumer warps x chunks completed (CTA-scope release counter)
  volatile unsigned sig_done;  // chunks whose outbox the signal warp has emptied
  volatile int cons_done;
  int rt_e[2][kMaxK];    // routing of units u (index u & 1): experts and weights, by the producer
  float rt_w[2][kMaxK];
};

__device__ __forceinline__ void raise_error(const Prog& P, Smem* sm, int code) {
  atomicCAS(P.s.err, 0, code);
  sm->abort = 1;
}

// Spin until ctrl[word] - target >= 0 (wrap-safe), the budget runs out or an abort is seen.
__device__ __noinline__ bool spin_geq(const Prog& P, Smem* sm, const unsigned* a, unsigned target,
                                      int code) {
  if ((int)(ld_acquire(a) - target) >= 0) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (unsigned it = 0;; ++it) {
    if ((int)(ld_acquire(a) - target) >= 0) return true;
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
    __nanosleep(100);
  }
}

__device__ __forceinline__ bool wait_mbar(const Prog& P, Smem* sm, uint64_t* bar, unsigned parity,
                                          int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (unsigned it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (sm->abort) return false;
    if ((it & 63) == 63) {
      if (ld_volatile_int(P.s.err) != 0) {
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

// Consumer-wide wait: thread 0 spins, all consumers get the same verdict at the barrier.
__device__ __forceinline__ bool consumer_wait(const Prog& P, Smem* sm, int word, unsigned target,
                                              int code) {
  if (ctid() == 0) spin_geq(P, sm, my_flag(P, word), target, code);
  return !consumer_any(sm->abort != 0);
}

// ------------------------------------------------------------------------------------------
// producer: stream the rows of this CTA's chunks into the ring
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void stage_rows(uint8_t* dst, const uint8_t* src, unsigned bytes,
                                           uint64_t* bar) {
  if (bytes) tma_load_1d(dst, src, bytes, bar);
}

__device__ void topk_warp(const Prog& P, const Geo& G, int u, int slot, const float* bias,
                          int* idx_out, float* w_out, Smem* sm);

// The whole producer warp runs this loop; lane 0 issues the copies, and all 32 lanes select
// the top-K experts of a unit when its first routed chunk comes up (every CTA computes the
// same selection from the same logits, so no second broadcast is needed).
__device__ void producer(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
  const int lane = threadIdx.x & 31;
  const int NS = G.nstage;
  int route_unit = -1;
  int eidx[kMaxK];
  for (ChunkIter ci(P, G); ci.valid(); ci.next()) {
    const unsigned it = ci.it;
    const int slot = (int)(it % NS);
    const unsigned ph = (it / NS) & 1u;
    int ok = 1;
    if (lane == 0) ok = wait_mbar(P, sm, &empty[slot], ph ^ 1u, DE_TIMEOUT_EMPTY);
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    const ChunkView cv = ci.view(G);
    const UnitView uv = unit_view(P, G, cv.u);
    const LayerW& L = *uv.L;
    if ((cv.phase == P_RGU || cv.phase == P_RDN) && route_unit != cv.u) {
      if (lane == 0) ok = spin_geq(P, sm, my_flag(P, P_ROUTER), (unsigned)(cv.u + 1), DE_TIMEOUT_ROUTE);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      // the CTA owning the unit's first routed chunk writes the caller's routing outputs
      const unsigned first = (unsigned)cv.u * (unsigned)ci.ntot + (unsigned)G.off[P_RGU];
      const bool outs = first % gridDim.x == blockIdx.x;
      topk_warp(P, G, cv.u, uv.slot, uv.bias, outs ? uv.idx_out : nullptr,
                outs ? uv.w_out : nullptr, sm);
      for (int k = 0; k < G.K; ++k) eidx[k] = min(max(sm->rt_e[cv.u & 1][k], 0), G.E - 1);
      route_unit = cv.u;
    }
    if (lane == 0) {
      uint8_t* dst = smem + G.o_ring + (size_t)slot * G.stage_bytes;
      switch (cv.phase) {
        case P_ROUTER: {
          const unsigned rowb = 4u * G.H;
          const int a = cv.r0, b = min(cv.r0 + cv.n, G.E);
          const unsigned bytes =
              (b > a ? (unsigned)(b - a) * rowb : 0u) + (cv.r0 + cv.n > G.E ? rowb : 0u);
          mbar_arrive_expect_tx(&full[slot], bytes);
          if (b > a)
            stage_rows(dst, reinterpret_cast<const uint8_t*>(L.router + (size_t)a * G.H),
                       (unsigned)(b - a) * rowb, &full[slot]);
          if (cv.r0 + cv.n > G.E)
            stage_rows(dst + (size_t)(G.E - cv.r0) * rowb,
                       reinterpret_cast<const uint8_t*>(L.gate), rowb, &full[slot]);
          break;
        }
        case P_SGU:
        case P_RGU: {
          const uint8_t* base =
              cv.phase == P_SGU ? L.shared : L.experts + (size_t)eidx[cv.k] * L.expert_stride;
          const unsigned cb = (unsigned)cv.n * G.rc_h, sbb = (unsigned)cv.n * G.rs_h;
          mbar_arrive_expect_tx(&full[slot], 2u * (cb + sbb));
          const size_t sbo = (size_t)G.I * G.rc_h;
          stage_rows(dst, base + (size_t)cv.r0 * G.rc_h, cb, &full[slot]);
          stage_rows(dst + (size_t)G.rcg * G.rc_h, base + G.q_gu + (size_t)cv.r0 * G.rc_h, cb,
                     &full[slot]);
          uint8_t* dsb = dst + (size_t)2 * G.rcg * G.rc_h;
          stage_rows(dsb, base + sbo + (size_t)cv.r0 * G.rs_h, sbb, &full[slot]);
          stage_rows(dsb + (size_t)G.rcg * G.rs_h,
                     base + G.q_gu + sbo + (size_t)cv.r0 * G.rs_h, sbb, &full[slot]);
          break;
        }
        case P_SDN: {
          const uint8_t* base = L.shared + 2 * G.q_gu;
          const unsigned cb = (unsigned)cv.n * G.rc_i, sbb = (unsigned)cv.n * G.rs_i;
          mbar_arrive_expect_tx(&full[slot], cb + sbb);
          stage_rows(dst, base + (size_t)cv.r0 * G.rc_i, cb, &full[slot]);
          stage_rows(dst + (size_t)G.rsd * G.rc_i,
                     base + (size_t)G.H * G.rc_i + (size_t)cv.r0 * G.rs_i, sbb, &full[slot]);
          break;
        }
        default: {  // P_RDN
          const unsigned cb = (unsigned)cv.n * G.rc_i, sbb = (unsigned)cv.n * G.rs_i;
          mbar_arrive_expect_tx(&full[slot], (unsigned)G.K * (cb + sbb));
          uint8_t* dsb = dst + (size_t)G.K * G.rrd * G.rc_i;
          for (int k = 0; k < G.K; ++k) {
            const uint8_t* base = L.experts + (size_t)eidx[k] * L.expert_stride + 2 * G.q_gu;
            stage_rows(dst + (size_t)k * G.rrd * G.rc_i, base + (size_t)cv.r0 * G.rc_i, cb,
                       &full[slot]);
            stage_rows(dsb + (size_t)k * G.rrd * G.rs_i,
                       base + (size_t)G.H * G.rc_i + (size_t)cv.r0 * G.rs_i, sbb, &full[slot]);
          }
          break;
        }
      }
      sm->issued = it + 1;
    }
    __syncwarp();
  }
  if (lane == 0) sm->prod_done = 1;
}

// ------------------------------------------------------------------------------------------
// signal warp: move epilogue results to global memory, publish completions, top-K
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

// Top-K of the unit's logits by one warp. Every lane sorts its 16 packed keys; passes over
// more than 512 experts keep each lane's best 16 by a bitonic merge. Then K rounds of a warp
// maximum over the lanes' heads (two 32-bit reductions), the winning lane dropping its head.
// w_k = exp(l_k - l_max) / sum_sel exp(l_j - l_max): the softmax over all experts followed by
// renormalisation over the selected ones, where the full softmax denominator cancels; the
// logits come back from the keys with 40 significant bits.
__device__ __noinline__ void topk_warp(const Prog& P, const Geo& G, int u, int slot,
                                       const float* bias, int* idx_out, float* w_out,
                                       Smem* sm) {
  const int lane = threadIdx.x & 31;
  const double* lg = P.s.logits + (size_t)slot * G.nr;
  constexpr int kPer = 16;
  unsigned long long best[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) best[i] = 0ull;
  for (int e0 = 0; e0 < G.E; e0 += 32 * kPer) {
    double lv[kPer];
    float bv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = min(e0 + lane + 32 * i, G.E - 1);
      lv[i] = __ldcg(lg + e);
      bv[i] = bias ? __ldcg(bias + e) : 0.f;
    }
    unsigned long long key[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = e0 + lane + 32 * i;
      key[i] = e < G.E ? pkey(lv[i] + (double)bv[i], e) : 0ull;
    }
    sort16_desc(key);
    if (e0 == 0) {
#pragma unroll
      for (int i = 0; i < kPer; ++i) best[i] = key[i];
    } else {
      // both lists sorted descending: best[i] vs key[15-i] keeps the 16 largest as a bitonic
      // sequence, which one more sort puts in order
#pragma unroll
      for (int i = 0; i < kPer; ++i) best[i] = best[i] > key[kPer - 1 - i] ? best[i] : key[kPer - 1 - i];
      sort16_desc(best);
    }
  }
  int sel_e = 0;             // lane k < K ends up holding winner k
  unsigned long long sel_k = 0ull;
#pragma unroll
  for (int k = 0; k < kMaxK; ++k) {
    if (k < G.K) {
      const unsigned long long head = best[0];
      const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(head >> 32));
      const unsigned lo =
          __reduce_max_sync(0xffffffffu, (unsigned)(head >> 32) == hi ? (unsigned)head : 0u);
      const unsigned long long win = ((unsigned long long)hi << 32) | lo;
      if (head == win && win != 0ull) {
#pragma unroll
        for (int j = 0; j + 1 < kMaxK; ++j) best[j] = best[j + 1];
        best[kMaxK - 1] = 0ull;
      }
      if (lane == k) {
        sel_k = win;
        sel_e = 0x1FFF - (int)(win & 0x1FFFull);
      }
    }
  }
  // weights on lanes 0..K-1
  const double l0 = dkey_inv(__shfl_sync(0xffffffffu, sel_k, 0) & ~0x1FFFull);
  const bool mine = lane < G.K;
  const float ex = mine ? expf((float)(dkey_inv(sel_k & ~0x1FFFull) - l0)) : 0.f;
  float den = ex;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (mine) {
    const int e = min(max(sel_e, 0), G.E - 1);  // NaN logits must not make an address
    const float wk = __fdividef(ex, den);
    sm->rt_e[u & 1][lane] = e;
    sm->rt_w[u & 1][lane] = wk;
    if (idx_out) idx_out[lane] = e;
    if (w_out) w_out[lane] = wk;
  }
  __syncwarp();
}

// Sum of virtual row vr (wave w = vr / Pn, row-lane p = vr % Pn) from a reduction slot.
__device__ __forceinline__ float slot_row_sum(const float* part, int vr, int sp, int Pn) {
  const int p = vr % Pn, w = vr / Pn;
  if (sp >= 32) {
    const int nw = sp / 32;
    float a = 0.f;
    for (int i = 0; i < nw; ++i) a += part[(p * nw + i) * kMaxW + w];
    return a;
  }
  return part[p * kMaxW + w];
}

// The signal warp finishes every chunk of its CTA in order: it waits for the eight consumer
// warps' partials, sums them across warps, applies the epilogue (logit store; SwiGLU;
// residual/combine), stores the results, frees the slot, and publishes each run of same-
// (unit, phase) chunks with one gpu-scope fence and one reduction on the phase counter.
__device__ void signaller(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm) {
  const int lane = threadIdx.x & 31;
  float* boxes = reinterpret_cast<float*>(smem + G.o_box);
  unsigned run_n = 0;
  int cur_u = -1;
  UnitView uv;
  for (ChunkIter ci(P, G); ci.valid(); ci.next()) {
    const unsigned it = ci.it;
    // wait until all consumer warps have delivered chunk `it`
    int ok = 1;
    if (lane == 0) {
      const unsigned want = (it + 1) * kConsumerWarps;
      if ((int)(ld_acquire_cta_smem(&sm->done_count) - want) < 0) {
        const uint64_t deadline = global_ns() + P.wait_ns;
        for (unsigned k = 0;; ++k) {
          if ((int)(ld_acquire_cta_smem(&sm->done_count) - want) >= 0) break;
          if (sm->abort || sm->cons_done) {
            __threadfence_block();
            ok = !sm->abort && (int)(ld_acquire_cta_smem(&sm->done_count) - want) >= 0;
            break;
          }
          if ((k & 63) == 63 && global_ns() > deadline) {
            raise_error(P, sm, DE_TIMEOUT_DEP);
            ok = 0;
            break;
          }
          __nanosleep(20);
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    const ChunkView cv = ci.view(G);
    if (cv.u != cur_u) {
      cur_u = cv.u;
      uv = unit_view(P, G, cv.u);
    }
    const float* part = boxes + (size_t)(it % kBoxes) * G.box_floats;
    const float* base = part + G.red_part;
    float sq = 0.f;
    for (int r = lane; r < cv.n; r += 32) {
      switch (cv.phase) {
        case P_ROUTER: {
          const double* pd = reinterpret_cast<const double*>(part);
          double a = 0.0;
          for (int w = 0; w < kConsumerWarps; ++w) a += pd[w * G.rr + r];
          P.s.logits[(size_t)uv.slot * G.nr + cv.r0 + r] = a;
          break;
        }
        case P_SGU:
        case P_RGU: {
          const float a = slot_row_sum(part, r, G.sp_h, G.p_h);
          const float u = slot_row_sum(part, G.rcg + r, G.sp_h, G.p_h);
          const float h = __fdividef(a, 1.f + __expf(-a)) * u;  // SwiGLU: SiLU(gate) * up
          if (cv.phase == P_SGU)
            P.s.hs[(size_t)uv.slot * G.I + cv.r0 + r] = h;
          else
            P.s.hk[((size_t)uv.slot * G.K + cv.k) * G.I + cv.r0 + r] = h;
          break;
        }
        default: {
          const bool routed = cv.phase == P_RDN;
          const float o = base[r] + slot_row_sum(part, r, routed ? G.sp_d : G.sp_i,
                                                 routed ? G.p_d : G.p_i);
          uv.out[cv.r0 + r] = o;
          sq += o * o;
        }
      }
    }
    const bool final_out = cv.phase == P_RDN || (cv.phase == P_SDN && !G.routed_on);
    if (final_out && P.mode == MODE_STACK) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (lane == 0) atomicAdd(P.s.normsq + cv.u, sq);
    }
    __syncwarp();
    if (lane == 0) sm->sig_done = it + 1;  // the slot may be reused
    ++run_n;
    // Publish when this CTA's run of (unit, phase) ends: the next chunk of the schedule
    // belongs to another unit or phase, or there is none.
    ChunkIter nx = ci;
    nx.next();
    bool run_end = !nx.valid();
    if (!run_end) {
      const ChunkView nv = nx.view(G);
      run_end = nv.u != cv.u || nv.phase != cv.phase;
    }
    if (run_end) {
      fence_acq_rel_gpu();  // every lane: its stores come first
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        const unsigned old = atom_add_acq_rel_gpu(P.s.ctrl + cnt_word(cv.phase), run_n);
        last = old + run_n == (unsigned)(cv.u + 1) * (unsigned)G.n[cv.phase];
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        // this CTA completed the phase for the unit: tell every CTA through its own flag line
        if (cv.phase == P_ROUTER && !G.routed_on)  // routing-only launches: outputs from here
          topk_warp(P, G, cv.u, uv.slot, uv.bias, uv.idx_out, uv.w_out, sm);
        if (!(cv.phase == P_ROUTER && (P.debug & 1))) {
          fence_acq_rel_gpu();
          for (int c = lane; c < (int)gridDim.x; c += 32)
            P.s.flags[c * F_WORDS + cv.phase] = (unsigned)(cv.u + 1);
        }
      }
      run_n = 0;
    }
  }
}

// ------------------------------------------------------------------------------------------
// dequantising dot products of W rows with one thread's 32-column slice
// ------------------------------------------------------------------------------------------
// One byte of codes becomes the binary32 32768 + byte (exponent 15, byte in mantissa bits
// 8..15); clearing the low code(s) gives 32768 + the high part. Subtracting 32768 is exact.
__device__ __forceinline__ uint32_t magic_byte(uint32_t word, int k) {
  return __byte_perm(word, 0x47000000u, 0x7604u | ((uint32_t)k << 4));
}

// v[w] = s_w * sum(q x) + z_w * sum(x) over the slice, for the W rows vr = p + w*P; all W
// rows are loaded first and unpacked in lock step so their instruction streams interleave.
// Rows that are not valid read a clamped (in-stage) address and are returned as 0.
template <int BITS, int W>
__device__ __forceinline__ void qrows(const uint8_t* slot, int p, int P, bool s_ok,
                                      unsigned a_row, unsigned a_slice, unsigned b_base,
                                      unsigned b_row, unsigned b_slice, int n, int half_rows,
                                      int vmax, const float (&xq)[32], float sx, float (&v)[W]) {
  constexpr int kWords = BITS == 4 ? 4 : 2;
  uint32_t q[W][kWords];
  uint32_t sbw[W];
  bool ok[W];
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int vr = p + w * P;
    ok[w] = s_ok && (half_rows > 0 ? (vr < half_rows ? vr < n : (vr - half_rows) < n) : vr < n);
    const int vc = min(vr, vmax);
    const uint8_t* ca = slot + a_slice + (size_t)vc * a_row;
    if constexpr (BITS == 4) {
      const uint4 t = *reinterpret_cast<const uint4*>(ca);
      q[w][0] = t.x; q[w][1] = t.y; q[w][2] = t.z; q[w][3] = t.w;
    } else {
      const uint2 t = *reinterpret_cast<const uint2*>(ca);
      q[w][0] = t.x; q[w][1] = t.y;
    }
    sbw[w] = *reinterpret_cast<const uint32_t*>(slot + b_base + b_slice + (size_t)vc * b_row);
  }
  const float2 m = make_float2(-32768.f, -32768.f);
  float2 acc0[W], acc1[W];
#pragma unroll
  for (int w = 0; w < W; ++w) {
    acc0[w] = make_float2(0.f, 0.f);
    acc1[w] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int wi = 0; wi < kWords; ++wi) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int b = wi * 4 + k;
      if constexpr (BITS == 4) {
        // (16*hi + lo, 16*hi) paired with (x_lo, x_hi/16 - x_lo)
        const float2 xv = make_float2(xq[2 * b], xq[2 * b + 1]);
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const uint32_t t = magic_byte(q[w][wi], k);
          const float2 f = __fadd2_rn(make_float2(__uint_as_float(t), __uint_as_float(t & 0xFFFFF0FFu)), m);
          if (b & 1)
            acc1[w] = __ffma2_rn(f, xv, acc1[w]);
          else
            acc0[w] = __ffma2_rn(f, xv, acc0[w]);
        }
      } else {
        // (c0+4c1+16c2+64c3, 4c1+16c2+64c3) and (16c2+64c3, 64c3)
        const float2 xa = make_float2(xq[4 * b], xq[4 * b + 1]);
        const float2 xb = make_float2(xq[4 * b + 2], xq[4 * b + 3]);
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const uint32_t t = magic_byte(q[w][wi], k);
          const float2 f01 = __fadd2_rn(make_float2(__uint_as_float(t), __uint_as_float(t & 0xFFFFFCFFu)), m);
          const float2 f23 = __fadd2_rn(make_float2(__uint_as_float(t & 0xFFFFF0FFu), __uint_as_float(t & 0xFFFFC0FFu)), m);
          acc0[w] = __ffma2_rn(f01, xa, acc0[w]);
          acc1[w] = __ffma2_rn(f23, xb, acc1[w]);
        }
      }
    }
  }
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const float s = __uint_as_float(sbw[w] << 16);
    const float z = __uint_as_float(sbw[w] & 0xFFFF0000u);
    const float qx = (acc0[w].x + acc0[w].y) + (acc1[w].x + acc1[w].y);
    v[w] = ok[w] ? fmaf(s, qx, z * sx) : 0.f;
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

// x' transform of a vector into the layout the slice kernels read (see qrows): 4-bit pairs
// (x0, x1/16 - x0); 2-bit quads (x0, x1/4 - x0, x2/16 - x1/4, x3/64 - x2/16).
__device__ __forceinline__ void transform_store4(float* xq, int c, float v0, float v1, float v2,
                                                 float v3, int bits) {
  float4 o;
  if (bits == 4)
    o = make_float4(v0, v1 * 0.0625f - v0, v2, v3 * 0.0625f - v2);
  else
    o = make_float4(v0, v1 * 0.25f - v0, v2 * 0.0625f - v1 * 0.25f, v3 * 0.015625f - v2 * 0.0625f);
  *reinterpret_cast<float4*>(xq + c) = o;
}

// ------------------------------------------------------------------------------------------
// consumers
// ------------------------------------------------------------------------------------------
struct Map {  // one thread's place in a virtual-row layout: row-lane p, slice s (clamped sc)
  int p, s, sc;
  bool ok;
};

__device__ __forceinline__ Map make_map(int sp, int Pn, int sl) {
  Map m;
  m.p = ctid() / sp;
  m.s = ctid() - m.p * sp;
  m.ok = m.p < Pn && m.s < sl;
  m.sc = min(m.s, sl - 1);
  return m;
}

struct Consumer {
  const Prog& P;
  const Geo& G;
  uint8_t* smem;
  Smem* sm;
  float* XR;
  float* XG;
  float* SXG;
  float* XS;
  float* SXS;
  float* XD;
  float* SXD;
  float* boxes;
  Map mgu, msd, mrd;
  int x_unit = -1, xs_unit = -1, xd_unit = -1;
  int tag_unit = -1, tag_buf = -1;
  float xq[32];
  float sx = 0.f;

  __device__ Consumer(const Prog& P_, const Geo& G_, uint8_t* smem_, Smem* sm_)
      : P(P_), G(G_), smem(smem_), sm(sm_) {
    XR = reinterpret_cast<float*>(smem + G.o_xr);
    XG = reinterpret_cast<float*>(smem + G.o_xg);
    SXG = reinterpret_cast<float*>(smem + G.o_sxg);
    XS = reinterpret_cast<float*>(smem + G.o_xs);
    SXS = reinterpret_cast<float*>(smem + G.o_sxs);
    XD = reinterpret_cast<float*>(smem + G.o_xd);
    SXD = reinterpret_cast<float*>(smem + G.o_sxd);
    boxes = reinterpret_cast<float*>(smem + G.o_box);
    mgu = make_map(G.sp_h, G.p_h, G.sl_h);
    msd = make_map(G.sp_i, G.p_i, G.sl_i);
    mrd = make_map(G.sp_d, G.p_d, G.sl_d);
  }

  __device__ __forceinline__ bool wait_unit_done(int u) {
    return consumer_wait(P, sm, final_phase(G), (unsigned)(u + 1), DE_TIMEOUT_DEP);
  }

  // slice sums of a vector in shared memory (32 columns per slice), bank-conflict free
  __device__ __forceinline__ void slice_sums(const float* x, float* sxo, int nsl) {
    for (int s = ctid(); s < nsl; s += kConsumers) {
      float a = 0.f;
      for (int i = 0; i < 32; ++i) a += x[s * 32 + ((i + s) & 31)];
      sxo[s] = a;
    }
  }

  // x of unit u: raw in XR (router), transformed in XG + slice sums (gate/up)
  __device__ __forceinline__ bool ensure_x(int u, const UnitView& uv) {
    if (x_unit == u) return true;
    if (u > 0 && !wait_unit_done(u - 1)) return false;
    float f = 1.f;
    if (uv.norm) f = rsqrtf(__ldcg(P.s.normsq + (u - 1)) / (float)G.H + P.eps);
    for (int c = ctid() * 4; c < G.H; c += kConsumers * 4) {
      const float4 a = ldcg4(uv.xin + c);
      const float v0 = a.x * f, v1 = a.y * f, v2 = a.z * f, v3 = a.w * f;
      *reinterpret_cast<float4*>(XR + c) = make_float4(v0, v1, v2, v3);
      transform_store4(XG, c, v0, v1, v2, v3, G.bits);
    }
    consumer_sync();
    slice_sums(XR, SXG, G.sl_h);
    consumer_sync();
    x_unit = u;
    return true;
  }

  // sigma * h_shared, transformed, for the shared-expert down rows
  __device__ __forceinline__ bool ensure_xs(int u, const UnitView& uv) {
    if (xs_unit == u) return true;
    if (!consumer_wait(P, sm, P_SGU, (unsigned)(u + 1), DE_TIMEOUT_DEP)) return false;
    float sig = 1.f;
    if (G.gate_on) {  // sigma(g . x): the shared-gate row is the last router row
      if (!consumer_wait(P, sm, P_ROUTER, (unsigned)(u + 1), DE_TIMEOUT_DEP)) return false;
      sig = (float)(1.0 / (1.0 + exp(-__ldcg(P.s.logits + (size_t)uv.slot * G.nr + G.E))));
    }
    const float* hs = P.s.hs + (size_t)uv.slot * G.I;
    float* raw = XD;  // XD is rebuilt before its next use in this unit
    for (int c = ctid() * 4; c < G.I; c += kConsumers * 4) {
      const float4 a = ldcg4(hs + c);
      const float v0 = sig * a.x, v1 = sig * a.y, v2 = sig * a.z, v3 = sig * a.w;
      *reinterpret_cast<float4*>(raw + c) = make_float4(v0, v1, v2, v3);
      transform_store4(XS, c, v0, v1, v2, v3, G.bits);
    }
    consumer_sync();
    slice_sums(raw, SXS, G.sl_i);
    xd_unit = -1;
    consumer_sync();
    xs_unit = u;
    return true;
  }

  // w_k * h_k of the routed experts, transformed, for the routed down rows
  __device__ __forceinline__ bool ensure_xd(int u, const UnitView& uv) {
    if (xd_unit == u) return true;
    if (!consumer_wait(P, sm, P_RGU, (unsigned)(u + 1), DE_TIMEOUT_DEP)) return false;
    if (G.shared_on && !consumer_wait(P, sm, P_SDN, (unsigned)(u + 1), DE_TIMEOUT_DEP))
      return false;
    const float* hk = P.s.hk + (size_t)uv.slot * G.K * G.I;
    const int KI = G.K * G.I;
    float* raw = XR;  // XR (the router's x) is no longer needed in this unit
    for (int c = ctid() * 4; c < KI; c += kConsumers * 4) {
      const float wk = sm->rt_w[u & 1][c / G.I];
      const float4 a = ldcg4(hk + c);
      const float v0 = wk * a.x, v1 = wk * a.y, v2 = wk * a.z, v3 = wk * a.w;
      if (KI <= G.H) *reinterpret_cast<float4*>(raw + c) = make_float4(v0, v1, v2, v3);
      transform_store4(XD, c, v0, v1, v2, v3, G.bits);
    }
    consumer_sync();
    if (KI <= G.H) {
      slice_sums(raw, SXD, G.sl_d);
    } else {
      for (int s = ctid(); s < G.sl_d; s += kConsumers) {
        const float wk = sm->rt_w[u & 1][(s * 32) / G.I];
        float a = 0.f;
        for (int i = 0; i < 32; ++i) a += wk * __ldcg(hk + s * 32 + i);
        SXD[s] = a;
      }
    }
    if (KI <= G.H) x_unit = -1;  // XR was overwritten
    consumer_sync();
    xd_unit = u;
    return true;
  }

  __device__ __forceinline__ void load_xq(int unit, int buf, const float* X, const float* SX,
                                          const Map& m) {
    if (tag_unit == unit && tag_buf == buf) return;
    tag_unit = unit;
    tag_buf = buf;
    if (m.ok) {
      const float4* src = reinterpret_cast<const float4*>(X + m.s * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 a = src[i];
        xq[4 * i] = a.x;
        xq[4 * i + 1] = a.y;
        xq[4 * i + 2] = a.z;
        xq[4 * i + 3] = a.w;
      }
      sx = SX[m.s];
    }
  }

  // Slot of chunk `it` may be written once the signal warp has finished chunk it - kBoxes.
  // Each warp checks for itself (no CTA-wide barrier per chunk).
  __device__ __forceinline__ void wait_slot(unsigned it) {
    if ((threadIdx.x & 31) == 0 && it >= (unsigned)kBoxes) {
      const unsigned want = it - kBoxes + 1;
      if ((int)(sm->sig_done - want) < 0) {
        const uint64_t deadline = global_ns() + P.wait_ns;
        for (unsigned k = 0;; ++k) {
          if ((int)(sm->sig_done - want) >= 0) break;
          if (sm->abort) break;
          if ((k & 63) == 63 && global_ns() > deadline) {
            raise_error(P, sm, DE_TIMEOUT_DEP);
            break;
          }
          __nanosleep(20);
        }
      }
    }
    __syncwarp();
  }

  // Warp-level reduction of the row partials straight into the chunk's slot.
  template <int W>
  __device__ __forceinline__ void reduce_to_slot(float (&v)[W], int sp, unsigned it,
                                                 float* part) {
    const int lane = threadIdx.x & 31, warp = (ctid() >> 5);
    const int width = sp < 32 ? sp : 32;
    float* dst = sp >= 32 ? part + warp * kMaxW : part + (warp * (32 / sp) + lane / sp) * kMaxW;
    const int lane_in_seg = sp >= 32 ? lane : (lane % sp);
    wait_slot(it);
    reduce_rows<W>(v, lane_in_seg, width, dst);
  }

  // Epilogue row of this thread for prefetches: rows go round-robin over the warps (row r ->
  // warp r % 8, lane r / 8) so that no single warp carries them.
  __device__ __forceinline__ int epi_row() const {
    return (threadIdx.x & 31) * kConsumerWarps + ((ctid() >> 5));
  }

  __device__ __forceinline__ void release(uint64_t* empty) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
  }

  // ---------------------------------------------------------------- router rows
  __device__ __forceinline__ void router_chunk(const ChunkView& cv, const uint8_t* slot,
                                               uint64_t* empty, float* part, unsigned it) {
    const float* rows = reinterpret_cast<const float*>(slot);
    const int H = G.H, t = ctid(), lane = t & 31, warp = t >> 5;
    if (lane == 0) wait_slot_lane0(it);
    __syncwarp();
    for (int r = 0; r < cv.n; ++r) {
      double a = 0.0;
      const float4* wr = reinterpret_cast<const float4*>(rows + (size_t)r * H);
      const float4* xr = reinterpret_cast<const float4*>(XR);
      for (int c4 = t; c4 < H / 4; c4 += kConsumers) {
        const float4 p = wr[c4], b = xr[c4];
        a = fma((double)p.x, (double)b.x, a);
        a = fma((double)p.y, (double)b.y, a);
        a = fma((double)p.z, (double)b.z, a);
        a = fma((double)p.w, (double)b.w, a);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) reinterpret_cast<double*>(part)[warp * G.rr + r] = a;
    }
    release(empty);
  }

  __device__ __forceinline__ void wait_slot_lane0(unsigned it) {
    if (it >= (unsigned)kBoxes) {
      const unsigned want = it - kBoxes + 1;
      const uint64_t deadline = global_ns() + P.wait_ns;
      for (unsigned k = 0; (int)(sm->sig_done - want) < 0; ++k) {
        if (sm->abort) break;
        if ((k & 63) == 63 && global_ns() > deadline) {
          raise_error(P, sm, DE_TIMEOUT_DEP);
          break;
        }
        __nanosleep(20);
      }
    }
  }

  // ---------------------------------------------------------------- gate/up (SwiGLU in the signal warp)
  template <int BITS, int W>
  __device__ __forceinline__ void gateup_chunk(const ChunkView& cv, const uint8_t* slot,
                                               uint64_t* empty, float* part, unsigned it) {
    load_xq(cv.u, 0, XG, SXG, mgu);
    float v[W];
    qrows<BITS, W>(slot, mgu.p, G.p_h, mgu.ok, G.rc_h, (unsigned)mgu.sc * (BITS == 4 ? 16u : 8u),
                   2u * G.rcg * G.rc_h, G.rs_h, (unsigned)(mgu.sc >> 1) * 4u, cv.n, G.rcg,
                   2 * G.rcg - 1, xq, sx, v);
    release(empty);
    reduce_to_slot<W>(v, G.sp_h, it, part);
  }

  // ---------------------------------------------------------------- down (+ base for the combine)
  template <int BITS, int W>
  __device__ __forceinline__ void down_chunk(const ChunkView& cv, const UnitView& uv,
                                             const uint8_t* slot, uint64_t* empty, float* part,
                                             unsigned it, bool fail) {
    const bool routed = cv.phase == P_RDN;
    const Map& m = routed ? mrd : msd;
    const int sp = routed ? G.sp_d : G.sp_i, Pn = routed ? G.p_d : G.p_i;
    const int rows = routed ? G.rrd : G.rsd;
    // the base each output row adds to (residual, or the shared expert's combine) is fetched
    // now so its latency hides behind the dot products; the signal warp adds it
    float base[2];
    const int er = epi_row();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = er + i * kConsumers;
      base[i] = 0.f;
      if (r < cv.n && !fail) {
        const int j = cv.r0 + r;
        if (routed && G.shared_on)
          base[i] = __ldcg(uv.out + j);
        else if (uv.res)
          base[i] = __ldcg(uv.res + j);
      }
    }
    unsigned a_slice, b_slice;
    const unsigned b_base = (unsigned)(routed ? G.K : 1) * rows * G.rc_i;
    const unsigned cbytes = BITS == 4 ? 16u : 8u;
    if (routed) {
      const int k = m.sc / G.sl_i, si = m.sc - k * G.sl_i;
      a_slice = (unsigned)k * rows * G.rc_i + (unsigned)si * cbytes;
      b_slice = (unsigned)k * rows * G.rs_i + (unsigned)(si >> 1) * 4u;
      load_xq(cv.u, 2, XD, SXD, m);
    } else {
      a_slice = (unsigned)m.sc * cbytes;
      b_slice = (unsigned)(m.sc >> 1) * 4u;
      load_xq(cv.u, 1, XS, SXS, m);
    }
    float v[W];
    qrows<BITS, W>(slot, m.p, Pn, m.ok, G.rc_i, a_slice, b_base, G.rs_i, b_slice, cv.n, 0,
                   rows - 1, xq, sx, v);
    release(empty);
    reduce_to_slot<W>(v, sp, it, part);
    float* bs = part + G.red_part;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = er + i * kConsumers;
      if (r < cv.n) bs[r] = base[i];
    }
  }

  template <int BITS>
  __device__ __forceinline__ void dispatch(const ChunkView& cv, const UnitView& uv,
                                           const uint8_t* slot, uint64_t* empty, float* part,
                                           unsigned it, bool fail) {
    if (cv.phase == P_SGU || cv.phase == P_RGU) {
      if (G.w_gu == 4)
        gateup_chunk<BITS, 4>(cv, slot, empty, part, it);
      else
        gateup_chunk<BITS, 8>(cv, slot, empty, part, it);
    } else {
      down_chunk<BITS, 4>(cv, uv, slot, empty, part, it, fail);
    }
  }

  __device__ __forceinline__ void run() {
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
    const int NS = G.nstage;
    int cur_u = -1;
    UnitView uv;
    ChunkIter ci(P, G);
    for (; ci.valid(); ci.next()) {
      const unsigned it = ci.it;
      const int slot_i = (int)(it % NS);
      // A failed wait sets the CTA's abort flag; this warp then runs on in skip mode (reads of
      // in-bounds shared memory only) and every collective wait below returns at once.
      const bool fail = !wait_mbar(P, sm, &full[slot_i], (it / NS) & 1u, DE_TIMEOUT_FULL);
      const ChunkView cv = ci.view(G);
      if (cv.u != cur_u) {
        cur_u = cv.u;
        uv = unit_view(P, G, cv.u);
      }
      const uint8_t* slot = smem + G.o_ring + (size_t)slot_i * G.stage_bytes;
      bool ok;
      if (cv.phase == P_ROUTER || cv.phase == P_SGU || cv.phase == P_RGU) ok = ensure_x(cv.u, uv);
      else if (cv.phase == P_SDN) ok = ensure_xs(cv.u, uv);
      else ok = ensure_xd(cv.u, uv);
      if (!ok) break;
      if (cv.c == 0 && uv.h_trace && !fail)
        for (int c = ctid(); c < G.H; c += kConsumers) uv.h_trace[c] = __ldcg(uv.xin + c);
      float* part = boxes + (size_t)(it % kBoxes) * G.box_floats;
      if (cv.phase == P_ROUTER)
        router_chunk(cv, slot, &empty[slot_i], part, it);
      else if (G.bits == 4)
        dispatch<4>(cv, uv, slot, &empty[slot_i], part, it, fail);
      else
        dispatch<2>(cv, uv, slot, &empty[slot_i], part, it, fail);
      // this warp's share of the chunk's slot is written: tell the signal warp
      __syncwarp();
      if ((threadIdx.x & 31) == 0) red_release_cta_smem(&sm->done_count, 1u);
    }
    consumer_sync();  // every consumer warp's last delivery is published before this
    if (ctid() == 0) sm->cons_done = 1;
    // drain: never leave the CTA with bulk copies in flight
    if (ctid() == 0 && sm->abort) {
      const uint64_t deadline = global_ns() + 100000000ull;
      while (!sm->prod_done && global_ns() < deadline) __nanosleep(1000);
      const unsigned issued = sm->issued;
      for (unsigned j = ci.it; j < issued; ++j) {
        const int si = (int)(j % NS);
        while (!mbar_try_wait(&full[si], (j / NS) & 1u) && global_ns() < deadline) {
        }
      }
    }
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    engine_kernel(const __grid_constant__ Prog P, const __grid_constant__ Geo G) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Smem* sm = reinterpret_cast<Smem*>(smem + G.o_misc);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
  if (threadIdx.x == 0) {
    sm->abort = 0;
    sm->prod_done = 0;
    sm->issued = 0;
    sm->done_count = 0;
    sm->sig_done = 0;
    sm->cons_done = 0;
    for (int i = 0; i < G.nstage; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    producer(P, G, smem, sm);
    return;
  }
  if (warp == 1) {
    signaller(P, G, smem, sm);
    return;
  }
  Consumer c(P, G, smem, sm);
  c.run();
}

}  // namespace fmoe

// launcher used by the C ABI layer
extern "C" cudaError_t fmoe_engine_configure(int max_smem) {
  return cudaFuncSetAttribute(fmoe::engine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              max_smem);
}

extern "C" cudaError_t fmoe_engine_launch(const fmoe::Prog* P, const fmoe::Geo* G, int grid,
                                          cudaStream_t stream) {
  fmoe::engine_kernel<<<grid, fmoe::kThreads, G->smem_bytes, stream>>>(*P, *G);
  return cudaGetLastError();
}
