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
// How: one CTA per SM, 8 consumer warps + 1 producer warp. The producer claims chunks from a
// global counter (in dependency order) and streams their weight rows into a ring of shared
// memory stages with 1-D TMA bulk copies completing on mbarriers. Consumers own fixed 32-column
// slices, keep the matching (pre-transformed) x values in registers and unpack codes with one
// byte-permute per byte into a binary32 "32768 + byte" pattern; subtracting the magic with
// packed f32x2 arithmetic yields two exact code values per pair of instructions. Row partials
// are reduced with a transposing warp butterfly, then across warps in shared memory.
// Every spin-wait is bounded by a global-timer budget; on expiry the kernel records an error
// word, waits for its own copies in flight and returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include "engine.h"
#include "ptx.cuh"

namespace fmoe {

constexpr int kMaxW = 8;
constexpr unsigned kEnd = 0xFFFFFFFFu;

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

__device__ __forceinline__ ChunkView chunk_view(const Geo& G, unsigned g) {
  ChunkView v;
  const int ntot = G.off[P_COUNT];
  v.u = (int)(g / (unsigned)ntot);
  v.c = (int)(g - (unsigned)v.u * (unsigned)ntot);
  int p = 0;
  while (v.c >= G.off[p + 1]) ++p;
  v.phase = p;
  v.j = v.c - G.off[p];
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

// target of "unit u is complete" on the control words
__device__ __forceinline__ void unit_done_target(const Geo& G, int u, int* word, unsigned* target) {
  if (G.routed_on) {
    *word = C_CNT + P_RDN;
    *target = (unsigned)(u + 1) * (unsigned)G.n[P_RDN];
  } else if (G.shared_on) {
    *word = C_CNT + P_SDN;
    *target = (unsigned)(u + 1) * (unsigned)G.n[P_SDN];
  } else {
    *word = C_ROUTE;
    *target = (unsigned)(u + 1);
  }
}

// ------------------------------------------------------------------------------------------
// bounded waits
// ------------------------------------------------------------------------------------------
struct Smem {  // small shared state (in the misc area)
  volatile int abort;
  volatile int prod_done;
  volatile unsigned issued;
  int do_topk;
  int sel_e[kMaxK];
  double sel_l[kMaxK];
  double cand_l[2][kConsumerWarps];
  int cand_e[2][kConsumerWarps];
  float nsq[kConsumerWarps];
};

__device__ __forceinline__ void raise_error(const Prog& P, Smem* sm, int code) {
  atomicCAS(P.s.err, 0, code);
  sm->abort = 1;
}

// Spin until ctrl[word] - target >= 0 (wrap-safe), the budget runs out or an abort is seen.
__device__ __noinline__ bool spin_geq(const Prog& P, Smem* sm, int word, unsigned target, int code) {
  const unsigned* a = P.s.ctrl + word;
  if ((int)(ld_acquire(a) - target) >= 0) return true;
  const uint64_t deadline = global_ns() + P.wait_ns;
  for (unsigned it = 0;; ++it) {
    if ((int)(ld_acquire(a) - target) >= 0) return true;
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
    __nanosleep(64);
  }
}

__device__ __forceinline__ bool wait_mbar(const Prog& P, Smem* sm, uint64_t* bar, unsigned parity, int code) {
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

// Consumer-wide wait: thread 0 spins, the others learn the outcome at the barrier.
__device__ __forceinline__ bool consumer_wait(const Prog& P, Smem* sm, int word, unsigned target,
                                              int code) {
  if (threadIdx.x == 0) spin_geq(P, sm, word, target, code);
  return !consumer_any(sm->abort != 0);
}

// ------------------------------------------------------------------------------------------
// producer: claim chunks, stream their rows into the ring
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ unsigned stage_rows(uint8_t* dst, const uint8_t* src, unsigned bytes,
                                               uint64_t* bar) {
  if (bytes) tma_load_1d(dst, src, bytes, bar);
  return bytes;
}

__device__ void producer(const Prog& P, const Geo& G, uint8_t* smem, Smem* sm) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
  unsigned* meta = reinterpret_cast<unsigned*>(smem + G.o_meta);
  const unsigned ntot = (unsigned)G.off[P_COUNT];
  const unsigned total = (unsigned)P.n_units * ntot;
  const int NS = G.nstage;
  int route_unit = -1;
  int eidx[kMaxK];
  for (unsigned it = 0;; ++it) {
    const int slot = (int)(it % NS);
    const unsigned ph = (it / NS) & 1u;
    if (!wait_mbar(P, sm, &empty[slot], ph ^ 1u, DE_TIMEOUT_EMPTY)) break;
    const unsigned g = atomicAdd(P.s.ctrl + C_NEXT, 1u);
    if (g >= total) {
      meta[slot] = kEnd;
      mbar_arrive(&full[slot]);
      sm->issued = it + 1;
      break;
    }
    const ChunkView cv = chunk_view(G, g);
    const UnitView uv = unit_view(P, G, cv.u);
    const LayerW& L = *uv.L;
    if ((cv.phase == P_RGU || cv.phase == P_RDN) && route_unit != cv.u) {
      if (!spin_geq(P, sm, C_ROUTE, (unsigned)(cv.u + 1), DE_TIMEOUT_ROUTE)) break;
      const int* si = P.s.sidx + uv.slot * G.K;
      for (int k = 0; k < G.K; ++k) eidx[k] = min(max(__ldcg(si + k), 0), G.E - 1);
      route_unit = cv.u;
    }
    meta[slot] = g;
    uint8_t* dst = smem + G.o_ring + (size_t)slot * G.stage_bytes;
    unsigned bytes = 0;
    switch (cv.phase) {
      case P_ROUTER: {
        const unsigned rowb = 4u * G.H;
        const int a = cv.r0, b = min(cv.r0 + cv.n, G.E);
        bytes = (b > a ? (unsigned)(b - a) * rowb : 0u) + (cv.r0 + cv.n > G.E ? rowb : 0u);
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
        const uint8_t* base = cv.phase == P_SGU
                                  ? L.shared
                                  : L.experts + (size_t)eidx[cv.k] * L.expert_stride;
        const unsigned cb = (unsigned)cv.n * G.rc_h, sbb = (unsigned)cv.n * G.rs_h;
        bytes = 2u * (cb + sbb);
        mbar_arrive_expect_tx(&full[slot], bytes);
        const size_t sbo = (size_t)G.I * G.rc_h;
        stage_rows(dst, base + (size_t)cv.r0 * G.rc_h, cb, &full[slot]);
        stage_rows(dst + (size_t)G.rcg * G.rc_h, base + G.q_gu + (size_t)cv.r0 * G.rc_h, cb,
                   &full[slot]);
        uint8_t* dsb = dst + (size_t)2 * G.rcg * G.rc_h;
        stage_rows(dsb, base + sbo + (size_t)cv.r0 * G.rs_h, sbb, &full[slot]);
        stage_rows(dsb + (size_t)G.rcg * G.rs_h, base + G.q_gu + sbo + (size_t)cv.r0 * G.rs_h,
                   sbb, &full[slot]);
        break;
      }
      case P_SDN: {
        const uint8_t* base = L.shared + 2 * G.q_gu;
        const unsigned cb = (unsigned)cv.n * G.rc_i, sbb = (unsigned)cv.n * G.rs_i;
        bytes = cb + sbb;
        mbar_arrive_expect_tx(&full[slot], bytes);
        stage_rows(dst, base + (size_t)cv.r0 * G.rc_i, cb, &full[slot]);
        stage_rows(dst + (size_t)G.rsd * G.rc_i, base + (size_t)G.H * G.rc_i + (size_t)cv.r0 * G.rs_i,
                   sbb, &full[slot]);
        break;
      }
      default: {  // P_RDN
        const unsigned cb = (unsigned)cv.n * G.rc_i, sbb = (unsigned)cv.n * G.rs_i;
        bytes = (unsigned)G.K * (cb + sbb);
        mbar_arrive_expect_tx(&full[slot], bytes);
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
  sm->prod_done = 1;
}

// ------------------------------------------------------------------------------------------
// dequantising slice dot products
// ------------------------------------------------------------------------------------------
// One byte of codes becomes the binary32 32768 + byte (exponent 15, byte in mantissa bits
// 8..15); clearing the low code(s) gives 32768 + the high part. Subtracting 32768 is exact.
__device__ __forceinline__ float2 magic_pair(uint32_t word, int k, uint32_t clear) {
  const uint32_t t = __byte_perm(word, 0x47000000u, 0x7604u | ((uint32_t)k << 4));
  return make_float2(__uint_as_float(t), __uint_as_float(t & clear));
}

template <int BITS>
__device__ __forceinline__ float slice_dot(const uint8_t* code, const uint8_t* sbp,
                                           const float (&xq)[32], float sx) {
  const float2 m = make_float2(-32768.f, -32768.f);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
  if constexpr (BITS == 4) {
    const uint4 q = *reinterpret_cast<const uint4*>(code);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // (16*hi + lo, 16*hi): paired with (x_lo, x_hi/16 - x_lo)
        const float2 f = __fadd2_rn(magic_pair(w[wi], k, 0xFFFFF0FFu), m);
        const int b = wi * 4 + k;
        const float2 xv = make_float2(xq[2 * b], xq[2 * b + 1]);
        if (b & 1)
          acc1 = __ffma2_rn(f, xv, acc1);
        else
          acc0 = __ffma2_rn(f, xv, acc0);
      }
    }
  } else {
    const uint2 q = *reinterpret_cast<const uint2*>(code);
    const uint32_t w[2] = {q.x, q.y};
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t t = __byte_perm(w[wi], 0x47000000u, 0x7604u | ((uint32_t)k << 4));
        // (c0+4c1+16c2+64c3, 4c1+16c2+64c3) and (16c2+64c3, 64c3)
        const float2 f01 = __fadd2_rn(make_float2(__uint_as_float(t), __uint_as_float(t & 0xFFFFFCFFu)), m);
        const float2 f23 = __fadd2_rn(make_float2(__uint_as_float(t & 0xFFFFF0FFu), __uint_as_float(t & 0xFFFFC0FFu)), m);
        const int b = wi * 4 + k;
        acc0 = __ffma2_rn(f01, make_float2(xq[4 * b], xq[4 * b + 1]), acc0);
        acc1 = __ffma2_rn(f23, make_float2(xq[4 * b + 2], xq[4 * b + 3]), acc1);
      }
    }
  }
  const uint32_t sb = *reinterpret_cast<const uint32_t*>(sbp);
  const float s = __uint_as_float(sb << 16);
  const float z = __uint_as_float(sb & 0xFFFF0000u);
  const float qx = (acc0.x + acc0.y) + (acc1.x + acc1.y);
  return fmaf(s, qx, z * sx);
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

// ------------------------------------------------------------------------------------------
// consumers
// ------------------------------------------------------------------------------------------
// ------------------------------------------------------------------------------------------
// top-K over the unit's logits by the 256 consumers of the CTA that completed the last router
// chunk: K rounds of a block-wide argmax (larger logit first, ties to the lower index), then
// w_k = exp(l_k - l_max) / sum_sel exp(l_j - l_max) -- the softmax over all experts followed by
// renormalisation over the selected ones, where the full denominator cancels.
// ------------------------------------------------------------------------------------------
__device__ __noinline__ void topk(const Prog& P, const Geo& G, Smem* sm, int u, int slot,
                                  const float* bias, int* idx_out, float* w_out) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (t == 0) __threadfence();
  consumer_sync();
  const double* lg = P.s.logits + (size_t)slot * G.nr;
  constexpr int kPer = 16;  // E <= 4096
  double lv[kPer];
  unsigned taken = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = t + i * kConsumers;
    lv[i] = -INFINITY;
    if (e < G.E) {
      double l = __ldcg(lg + e);
      if (bias) l += (double)__ldcg(bias + e);
      lv[i] = l;
    }
  }
  for (int k = 0; k < G.K; ++k) {
    double bl = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = t + i * kConsumers;
      if (e < G.E && !(taken >> i & 1u) && (lv[i] > bl || (lv[i] == bl && e < be))) {
        bl = lv[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ol = __shfl_xor_sync(0xffffffffu, bl, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ol > bl || (ol == bl && oe < be)) {
        bl = ol;
        be = oe;
      }
    }
    if (lane == 0) {
      sm->cand_l[k & 1][warp] = bl;
      sm->cand_e[k & 1][warp] = be;
    }
    consumer_sync();
    bl = sm->cand_l[k & 1][0];
    be = sm->cand_e[k & 1][0];
    for (int w = 1; w < kConsumerWarps; ++w) {
      const double ol = sm->cand_l[k & 1][w];
      const int oe = sm->cand_e[k & 1][w];
      if (ol > bl || (ol == bl && oe < be)) {
        bl = ol;
        be = oe;
      }
    }
    if (be - t >= 0 && (be - t) % kConsumers == 0) taken |= 1u << ((be - t) / kConsumers);
    if (t == 0) {
      sm->sel_e[k] = be;
      sm->sel_l[k] = bl;
    }
  }
  consumer_sync();
  if (t == 0) {
    const int K = G.K;
    double den = 0.0, ex[kMaxK];
    for (int k = 0; k < K; ++k) {
      ex[k] = exp(sm->sel_l[k] - sm->sel_l[0]);
      den += ex[k];
    }
    for (int k = 0; k < K; ++k) {
      const float wk = (float)(ex[k] / den);
      const int e = min(max(sm->sel_e[k], 0), G.E - 1);  // NaN logits must not make an address
      sm->sel_e[k] = e;
      P.s.sidx[slot * K + k] = e;
      P.s.sw[slot * K + k] = wk;
      if (idx_out) idx_out[k] = sm->sel_e[k];
      if (w_out) w_out[k] = wk;
    }
    float sig = 1.f;
    if (G.gate_on) sig = (float)(1.0 / (1.0 + exp(-__ldcg(lg + G.E))));
    P.s.ssig[slot] = sig;
    __threadfence();
    if (!(P.debug & 1)) st_release(P.s.ctrl + C_ROUTE, (unsigned)(u + 1));
  }
}


struct XTag {
  int unit;
  int buf;
};

// x' transform of a vector into the layout the slice kernels read (see slice_dot): 4-bit
// pairs (x0, x1/16 - x0); 2-bit quads (x0, x1/4 - x0, x2/16 - x1/4, x3/64 - x2/16).
__device__ __forceinline__ void transform_store(float* xq, int c, const float* v, int bits) {
  if (bits == 4) {
    xq[c] = v[0];
    xq[c + 1] = v[1] * 0.0625f - v[0];
  } else {
    xq[c] = v[0];
    xq[c + 1] = v[1] * 0.25f - v[0];
    xq[c + 2] = v[2] * 0.0625f - v[1] * 0.25f;
    xq[c + 3] = v[3] * 0.015625f - v[2] * 0.0625f;
  }
}

// slice sums of a vector held in shared memory (n columns, n/32 slices)
__device__ __forceinline__ void slice_sums(const float* x, float* sx, int nsl) {
  for (int s = threadIdx.x; s < nsl; s += kConsumers) {
    float a = 0.f;
    for (int i = 0; i < 32; ++i) a += x[s * 32 + ((i + s) & 31)];
    sx[s] = a;
  }
}

template <int BITS, int W>
__device__ __forceinline__ void qrows(const uint8_t* slot, int p, int P, int s, bool s_ok,
                                      unsigned a_row, unsigned a_slice, unsigned b_base,
                                      unsigned b_row, unsigned b_slice, int n, int half_rows,
                                      const float (&xq)[32], float sx, float (&v)[W]) {
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int vr = p + w * P;
    bool ok = s_ok;
    if (half_rows > 0)
      ok = ok && (vr < half_rows ? vr < n : (vr - half_rows) < n) && vr < 2 * half_rows;
    else
      ok = ok && vr < n;
    v[w] = ok ? slice_dot<BITS>(slot + a_slice + (size_t)vr * a_row,
                                slot + b_base + b_slice + (size_t)vr * b_row, xq, sx)
              : 0.f;
  }
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
  float* red;
  int x_unit = -1, xs_unit = -1, xd_unit = -1;
  XTag tag{-1, -1};
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
    red = reinterpret_cast<float*>(smem + G.o_red);
  }

  __device__ __forceinline__ bool wait_unit_done(int u) {
    int word;
    unsigned target;
    unit_done_target(G, u, &word, &target);
    return consumer_wait(P, sm, word, target, DE_TIMEOUT_DEP);
  }

  // x of unit u in XR (raw) and XG (transformed) + slice sums
  __device__ __forceinline__ bool ensure_x(int u, const UnitView& uv) {
    if (x_unit == u) return true;
    if (u > 0 && !wait_unit_done(u - 1)) return false;
    float f = 1.f;
    if (uv.norm) f = rsqrtf(__ldcg(P.s.normsq + (u - 1)) / (float)G.H + P.eps);
    const int H = G.H;
    const int step = G.bits == 4 ? 2 : 4;
    for (int c = threadIdx.x * step; c < H; c += kConsumers * step) {
      float v[4];
      if (step == 2) {
        const float2 a = __ldcg(reinterpret_cast<const float2*>(uv.xin + c));
        v[0] = a.x * f;
        v[1] = a.y * f;
      } else {
        const float4 a = ldcg4(uv.xin + c);
        v[0] = a.x * f;
        v[1] = a.y * f;
        v[2] = a.z * f;
        v[3] = a.w * f;
      }
      for (int i = 0; i < step; ++i) XR[c + i] = v[i];
      transform_store(XG, c, v, G.bits);
    }
    consumer_sync();
    slice_sums(XR, SXG, G.sl_h);
    consumer_sync();
    x_unit = u;
    return true;
  }

  __device__ __forceinline__ bool ensure_xs(int u, const UnitView& uv) {
    if (xs_unit == u) return true;
    if (!consumer_wait(P, sm, C_CNT + P_SGU, (unsigned)(u + 1) * G.n[P_SGU], DE_TIMEOUT_DEP))
      return false;
    float sig = 1.f;
    if (G.gate_on) {
      if (!consumer_wait(P, sm, C_ROUTE, (unsigned)(u + 1), DE_TIMEOUT_DEP)) return false;
      sig = __ldcg(P.s.ssig + uv.slot);
    }
    const float* hs = P.s.hs + (size_t)uv.slot * G.I;
    const int step = G.bits == 4 ? 2 : 4;
    for (int c = threadIdx.x * step; c < G.I; c += kConsumers * step) {
      float v[4];
      for (int i = 0; i < step; ++i) v[i] = sig * __ldcg(hs + c + i);
      transform_store(XS, c, v, G.bits);
    }
    // slice sums of sig*h straight from global (L2)
    for (int s = threadIdx.x; s < G.sl_i; s += kConsumers) {
      float a = 0.f;
      for (int i = 0; i < 32; ++i) a += sig * __ldcg(hs + s * 32 + i);
      SXS[s] = a;
    }
    consumer_sync();
    xs_unit = u;
    return true;
  }

  __device__ __forceinline__ bool ensure_xd(int u, const UnitView& uv) {
    if (xd_unit == u) return true;
    if (!consumer_wait(P, sm, C_CNT + P_RGU, (unsigned)(u + 1) * G.n[P_RGU], DE_TIMEOUT_DEP))
      return false;
    if (G.shared_on &&
        !consumer_wait(P, sm, C_CNT + P_SDN, (unsigned)(u + 1) * G.n[P_SDN], DE_TIMEOUT_DEP))
      return false;
    const float* hk = P.s.hk + (size_t)uv.slot * G.K * G.I;
    const int step = G.bits == 4 ? 2 : 4;
    const int KI = G.K * G.I;
    for (int c = threadIdx.x * step; c < KI; c += kConsumers * step) {
      const float wk = __ldcg(P.s.sw + uv.slot * G.K + c / G.I);
      float v[4];
      for (int i = 0; i < step; ++i) v[i] = wk * __ldcg(hk + c + i);
      transform_store(XD, c, v, G.bits);
    }
    for (int s = threadIdx.x; s < G.sl_d; s += kConsumers) {
      const float wk = __ldcg(P.s.sw + uv.slot * G.K + (s * 32) / G.I);
      float a = 0.f;
      for (int i = 0; i < 32; ++i) a += wk * __ldcg(hk + s * 32 + i);
      SXD[s] = a;
    }
    consumer_sync();
    xd_unit = u;
    return true;
  }

  __device__ __forceinline__ void load_xq(int unit, int buf, const float* X, const float* SX, int s, bool s_ok) {
    if (tag.unit == unit && tag.buf == buf) return;
    tag.unit = unit;
    tag.buf = buf;
    if (s_ok) {
      const float4* src = reinterpret_cast<const float4*>(X + s * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 a = src[i];
        xq[4 * i] = a.x;
        xq[4 * i + 1] = a.y;
        xq[4 * i + 2] = a.z;
        xq[4 * i + 3] = a.w;
      }
      sx = SX[s];
    }
  }

  // Reduce the per-thread row partials of a chunk into red, then return (after a barrier).
  template <int W>
  __device__ __forceinline__ void reduce_chunk(float (&v)[W], int sp, int p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int width = sp < 32 ? sp : 32;
    float* dst;
    if (sp >= 32)
      dst = red + warp * kMaxW;
    else
      dst = red + (warp * (32 / sp) + lane / sp) * kMaxW;
    const int lane_in_seg = sp >= 32 ? lane : (lane % sp);
    (void)p;
    reduce_rows<W>(v, lane_in_seg, width, dst);
    consumer_sync();
  }

  // Sum of virtual row vr (wave w, row-lane p) from red.
  __device__ __forceinline__ float row_sum(int vr, int sp, int P_) const {
    const int p = vr % P_, w = vr / P_;
    if (sp >= 32) {
      const int nw = sp / 32;
      float a = 0.f;
      for (int i = 0; i < nw; ++i) a += red[(p * nw + i) * kMaxW + w];
      return a;
    }
    return red[p * kMaxW + w];
  }

  __device__ __forceinline__ void release(uint64_t* empty) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
  }

  // completion of a chunk: all consumer writes are done before the counter moves
  __device__ __forceinline__ unsigned complete(int phase) {
    consumer_sync();
    unsigned old = 0;
    if (threadIdx.x == 0) {
      __threadfence();
      old = atomicAdd(P.s.ctrl + C_CNT + phase, 1u);
      sm->do_topk = (int)old;
    }
    return old;
  }

  // ---------------------------------------------------------------- router rows
  __device__ __forceinline__ void router_chunk(const ChunkView& cv, const UnitView& uv, const uint8_t* slot,
                               uint64_t* empty) {
    const float* rows = reinterpret_cast<const float*>(slot);
    const int H = G.H, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    double* redd = reinterpret_cast<double*>(red);
    for (int r = 0; r < cv.n; ++r) {
      double acc = 0.0;
      const float4* wr = reinterpret_cast<const float4*>(rows + (size_t)r * H);
      const float4* xr = reinterpret_cast<const float4*>(XR);
      for (int c4 = t; c4 < H / 4; c4 += kConsumers) {
        const float4 a = wr[c4], b = xr[c4];
        acc = fma((double)a.x, (double)b.x, acc);
        acc = fma((double)a.y, (double)b.y, acc);
        acc = fma((double)a.z, (double)b.z, acc);
        acc = fma((double)a.w, (double)b.w, acc);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) redd[warp * 32 + r] = acc;
    }
    release(empty);
    consumer_sync();
    if (t < cv.n) {
      double a = 0.0;
      for (int w = 0; w < kConsumerWarps; ++w) a += redd[w * 32 + t];
      P.s.logits[(size_t)uv.slot * G.nr + cv.r0 + t] = a;
    }
    const unsigned old = complete(P_ROUTER);
    (void)old;
    consumer_sync();
    const unsigned last = (unsigned)(cv.u + 1) * (unsigned)G.n[P_ROUTER] - 1u;
    if ((unsigned)sm->do_topk == last) topk(P, G, sm, cv.u, uv.slot, uv.bias, uv.idx_out, uv.w_out);
  }

  // ---------------------------------------------------------------- gate/up + SwiGLU
  template <int BITS, int W>
  __device__ __forceinline__ void gateup_chunk(const ChunkView& cv, const UnitView& uv, const uint8_t* slot,
                               uint64_t* empty) {
    const int t = threadIdx.x, sp = G.sp_h, Pn = G.p_h;
    const int p = t / sp, s = t % sp;
    const bool s_ok = p < Pn && s < G.sl_h;
    load_xq(cv.u, 0, XG, SXG, s, s_ok);
    float v[W];
    qrows<BITS, W>(slot, p, Pn, s, s_ok, G.rc_h, (unsigned)s * (BITS == 4 ? 16u : 8u),
                   2u * G.rcg * G.rc_h, G.rs_h, (unsigned)(s >> 1) * 4u, cv.n, G.rcg, xq, sx, v);
    release(empty);
    reduce_chunk<W>(v, sp, p);
    if (t < cv.n) {
      const float a = row_sum(t, sp, Pn);
      const float u = row_sum(G.rcg + t, sp, Pn);
      const float h = a / (1.f + expf(-a)) * u;
      float* dst = cv.phase == P_SGU ? P.s.hs + (size_t)uv.slot * G.I
                                     : P.s.hk + ((size_t)uv.slot * G.K + cv.k) * G.I;
      dst[cv.r0 + t] = h;
    }
    complete(cv.phase);
  }

  // ---------------------------------------------------------------- down + combine
  template <int BITS, int W>
  __device__ __forceinline__ void down_chunk(const ChunkView& cv, const UnitView& uv, const uint8_t* slot,
                             uint64_t* empty) {
    const int t = threadIdx.x;
    const bool routed = cv.phase == P_RDN;
    const int sp = routed ? G.sp_d : G.sp_i, Pn = routed ? G.p_d : G.p_i;
    const int p = t / sp, s = t % sp;
    const int sl = routed ? G.sl_d : G.sl_i;
    const bool s_ok = p < Pn && s < sl;
    const int rows = routed ? G.rrd : G.rsd;
    unsigned a_slice, b_slice, b_base = (unsigned)(routed ? G.K : 1) * rows * G.rc_i;
    const unsigned sb_bytes = BITS == 4 ? 16u : 8u;
    if (routed) {
      const int k = s / G.sl_i, si = s - k * G.sl_i;
      a_slice = (unsigned)k * rows * G.rc_i + (unsigned)si * sb_bytes;
      b_slice = (unsigned)k * rows * G.rs_i + (unsigned)(si >> 1) * 4u;
      load_xq(cv.u, 2, XD, SXD, s, s_ok);
    } else {
      a_slice = (unsigned)s * sb_bytes;
      b_slice = (unsigned)(s >> 1) * 4u;
      load_xq(cv.u, 1, XS, SXS, s, s_ok);
    }
    float v[W];
    qrows<BITS, W>(slot, p, Pn, s, s_ok, G.rc_i, a_slice, b_base, G.rs_i, b_slice, cv.n, 0, xq,
                   sx, v);
    release(empty);
    reduce_chunk<W>(v, sp, p);
    const bool final_out = routed || !G.routed_on;
    float sq = 0.f;
    if (t < cv.n) {
      const int j = cv.r0 + t;
      float base;
      if (routed && G.shared_on)
        base = __ldcg(uv.out + j);
      else
        base = uv.res ? __ldcg(uv.res + j) : 0.f;
      const float o = base + row_sum(t, sp, Pn);
      uv.out[j] = o;
      sq = o * o;
    }
    if (final_out && P.mode == MODE_STACK) {
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if ((t & 31) == 0 && t < cv.n) atomicAdd(P.s.normsq + cv.u, sq);
    }
    complete(cv.phase);
  }

  template <int BITS, int W1, int W2>
  __device__ __forceinline__ void dispatch(const ChunkView& cv, const UnitView& uv, const uint8_t* slot,
                           uint64_t* empty) {
    if (cv.phase == P_SGU || cv.phase == P_RGU) {
      if (G.w_gu == W1)
        gateup_chunk<BITS, W1>(cv, uv, slot, empty);
      else
        gateup_chunk<BITS, W2>(cv, uv, slot, empty);
    } else {
      down_chunk<BITS, 4>(cv, uv, slot, empty);
    }
  }

  __device__ __forceinline__ void run() {
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G.o_full);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + G.o_empty);
    const unsigned* meta = reinterpret_cast<const unsigned*>(smem + G.o_meta);
    const int NS = G.nstage;
    unsigned it = 0;
    int cur_u = -1;
    UnitView uv;
    for (;; ++it) {
      const int slot_i = (int)(it % NS);
      const bool got = wait_mbar(P, sm, &full[slot_i], (it / NS) & 1u, DE_TIMEOUT_FULL);
      if (consumer_any(!got || sm->abort != 0)) break;
      const unsigned g = meta[slot_i];
      if (g == kEnd) {
        ++it;
        break;
      }
      const ChunkView cv = chunk_view(G, g);
      if (cv.u != cur_u) {
        cur_u = cv.u;
        uv = unit_view(P, G, cv.u);
      }
      const uint8_t* slot = smem + G.o_ring + (size_t)slot_i * G.stage_bytes;
      bool ok = true;
      if (cv.phase == P_ROUTER || cv.phase == P_SGU || cv.phase == P_RGU) ok = ensure_x(cv.u, uv);
      else if (cv.phase == P_SDN) ok = ensure_xs(cv.u, uv);
      else ok = ensure_xd(cv.u, uv);
      if (!ok) {
        ++it;
        break;
      }
      if (cv.c == 0 && uv.h_trace)
        for (int c = threadIdx.x; c < G.H; c += kConsumers) uv.h_trace[c] = __ldcg(uv.xin + c);
      if (cv.phase == P_ROUTER)
        router_chunk(cv, uv, slot, &empty[slot_i]);
      else if (G.bits == 4)
        dispatch<4, 4, 8>(cv, uv, slot, &empty[slot_i]);
      else
        dispatch<2, 4, 8>(cv, uv, slot, &empty[slot_i]);
    }
    // drain: never leave the CTA with bulk copies in flight
    consumer_sync();
    if (threadIdx.x == 0 && sm->abort) {
      const uint64_t deadline = global_ns() + 100000000ull;
      while (!sm->prod_done && global_ns() < deadline) __nanosleep(1000);
      const unsigned issued = sm->issued;
      for (unsigned j = it; j < issued; ++j) {
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
    for (int i = 0; i < G.nstage; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x >= kConsumers) {
    if (threadIdx.x == kConsumers) producer(P, G, smem, sm);
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
