// api.cu — the C ABI declared in include/fmoe.h: argument validation, launch geometry, scratch
// memory and CUDA-graph capture around the engine kernel (engine.cu) and the pack kernel.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "engine.h"
#include "fmoe.h"

extern "C" cudaError_t fmoe_engine_launch(const fmoe::Prog* P, const fmoe::Geo* G, int grid,
                                          cudaStream_t stream);
extern "C" cudaError_t fmoe_engine_configure(int max_smem);
extern "C" cudaError_t fmoe_engine_occupancy(int smem, int* ctas_per_sm);
extern "C" cudaError_t fmoe_pack_launch(const float* w, int rows, int cols, int bits, void* dst,
                                        int sms, cudaStream_t stream);

using namespace fmoe;

namespace {

thread_local std::string g_err;
thread_local uint64_t g_launches = 0;
thread_local uint64_t g_wait_ns = 1000000000ull;
thread_local int g_debug = 0;
thread_local int g_form = FORM_DIGITS;
constexpr int kMaxUnits = 1 << 24;  // units per launch (chunk and signal counters stay in range)

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FMOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define CK(call)                                        \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- per-device state
struct DevState {
  bool init = false;
  int sms = 0;
  int max_smem = 0;
  int* err = nullptr;          // sticky device error word
  cudaMemPool_t pool = nullptr;
};
std::mutex g_mu;
DevState g_dev[64];

// State of fmoe_moe_layer_noalloc, set up on its first call on a device. `base` is the device
// address of the fixed scratch array; its last 256 bytes hold the sticky error word.
struct NoAllocState {
  bool init = false;
  int sms = 0;
  int max_smem = 0;
  uint8_t* base = nullptr;
};
NoAllocState g_na[64];
constexpr size_t kNoAllocErrOff = FMOE_NOALLOC_SCRATCH_BYTES - 256;

int dev_state(DevState** out) {
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(FMOE_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& d = g_dev[dev];
  if (!d.init) {
    CK(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    CK(cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    CK(cudaMalloc(&d.err, sizeof(int)));
    CK(cudaMemset(d.err, 0, sizeof(int)));
    cudaMemPoolProps props;
    memset(&props, 0, sizeof props);
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    CK(cudaMemPoolCreate(&d.pool, &props));
    uint64_t keep = 64ull << 20;  // keep up to 64 MiB of scratch cached between calls
    CK(cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep));
    CK(fmoe_engine_configure(d.max_smem));
    int per_sm = 0;
    CK(fmoe_engine_occupancy(d.max_smem, &per_sm));
    if (per_sm < 1)
      return fail(FMOE_ERR_UNSUPPORTED, "the engine kernel does not fit one SM (%d CTAs)", per_sm);
    d.init = true;
  }
  *out = &d;
  return FMOE_OK;
}

unsigned align_up(unsigned v, unsigned a) { return (v + a - 1) / a * a; }

// rows whose byte size times this count is a multiple of 16 (TMA bulk copy granularity)
int rows_for_16(unsigned row_bytes) {
  int r = 1;
  while ((row_bytes * (unsigned)r) % 16u) r <<= 1;
  return r;
}

int pow2ceil(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// ---------------------------------------------------------------- validation and geometry
int check_shape(int H, int I, int E, int K, int bits) {
  if (bits != 2 && bits != 4) return fail(FMOE_ERR_INVALID, "bits must be 2 or 4 (got %d)", bits);
  if (H <= 0 || I <= 0 || H % 64 || I % 64)
    return fail(FMOE_ERR_INVALID, "hidden (%d) and inter (%d) must be positive multiples of 64", H, I);
  if (E < 1 || K < 1 || K > E) return fail(FMOE_ERR_INVALID, "need 1 <= top_k (%d) <= n_experts (%d)", K, E);
  if (H > 8192 || I > 8192) return fail(FMOE_ERR_UNSUPPORTED, "hidden/inter above 8192");
  if (K > kMaxK) return fail(FMOE_ERR_UNSUPPORTED, "top_k above %d", kMaxK);
  if (E > 4096) return fail(FMOE_ERR_UNSUPPORTED, "n_experts above 4096");
  if ((long long)K * I > 8192) return fail(FMOE_ERR_UNSUPPORTED, "top_k * inter above 8192");
  return FMOE_OK;
}

// Chunk sizes, consumer thread layouts and the shared-memory carve-up of one launch on a GPU
// with `sms` SMs (one CTA each) and `max_smem` bytes of shared memory per CTA.
int make_geo(int H, int I, int E, int K, int bits, bool route_on, bool shared_on, bool routed_on,
             bool gate_on, int max_smem, int sms, Geo* G) {
  memset(G, 0, sizeof *G);
  G->H = H; G->I = I; G->E = E; G->K = K; G->bits = bits;
  G->route_on = route_on; G->shared_on = shared_on; G->routed_on = routed_on;
  G->gate_on = gate_on && route_on && shared_on;
  G->rc_h = (unsigned)H * bits / 8; G->rs_h = (unsigned)H / 16;
  G->rc_i = (unsigned)I * bits / 8; G->rs_i = (unsigned)I / 16;
  G->q_gu = (unsigned long long)I * (G->rc_h + G->rs_h);
  if (sms < 1 || sms > kMaxCtas) return fail(FMOE_ERR_UNSUPPORTED, "SM count %d", sms);
  const bool gu_on = shared_on || routed_on;
  G->nseg = (shared_on ? 1 : 0) + (routed_on ? K : 0);
  G->au = rows_for_16(G->rs_h);
  G->ad = rows_for_16(G->rs_i);
  // a stage holds at least one aligned group of gate + up rows and of down rows
  const unsigned stage = align_up(
      std::max({kStage, gu_on ? 2u * (unsigned)G->au * (G->rc_h + G->rs_h) : 0u,
                G->nseg > 0 ? (unsigned)G->ad * (G->rc_i + G->rs_i) : 0u}),
      128);
  G->stage_bytes = stage;
  // router: whole rows when a row fits kRouterCols columns, else column segments of one row
  // (a consumer thread holds 4 float4 columns of a segment)
  G->nr = route_on ? E + (G->gate_on ? 1 : 0) : 0;
  if (H <= kRouterCols) {
    G->rseg = 1;
    G->rcols = H;
    G->rrows = std::max(1, std::min(32, (int)(kStage / (4u * H))));
  } else {
    int d = (H + kRouterCols - 1) / kRouterCols;
    while (H % d || (H / d) % 4) ++d;
    G->rseg = d;
    G->rcols = H / d;
    G->rrows = 1;
  }
  // gate/up: thread layout, then hr h-rows (gate + up) per chunk
  G->sh = H / 32;
  G->wh = G->sh <= 32 ? pow2ceil(G->sh) : 32 * ((G->sh + 31) / 32);
  G->gh = kConsumers / G->wh;
  {
    int hr = (int)(stage / (2u * (G->rc_h + G->rs_h)));
    hr = std::min(hr, kMaxHr);
    hr = std::min(hr, I);
    hr = std::min(hr, kMaxRowsThread * G->gh / 2);
    hr = hr / G->au * G->au;
    if (!gu_on) hr = G->au;  // no gate/up rows in this launch
    if (hr < G->au) return fail(FMOE_ERR_UNSUPPORTED, "gate/up rows do not fit a stage (H=%d)", H);
    G->hr = hr;
    // two chunks in one pass when their rows fit the threads' row slots
    G->gpass = (2 * 2 * hr <= kMaxRowsThread * G->gh) ? 2 : 1;
  }
  // down: lane layout, then dr output rows per chunk
  G->si = I / 32;
  if (G->si <= 32) {
    G->wi = pow2ceil(G->si);
    G->pi = 32 / G->wi;
    G->ji = 1;
  } else {
    G->wi = 32;
    G->pi = 1;
    G->ji = (G->si + 31) / 32;
  }
  {
    int dr = (int)(stage / (G->rc_i + G->rs_i));
    dr = std::min(dr, kMaxRowsWarp * kConsumerWarps * G->pi);
    dr = std::min(dr, H);
    dr = dr / G->ad * G->ad;
    if (G->nseg == 0) dr = G->ad;  // no down rows in this launch
    if (dr < G->ad) return fail(FMOE_ERR_UNSUPPORTED, "down rows do not fit a stage (I=%d)", I);
    G->dr = dr;
  }
  {
    const int nu = H / G->ad;
    G->oacc_n = G->nseg > 0 ? ((nu + sms - 1) / sms) * G->ad : 0;
  }
  // shared memory: ring A | ring B | x | h | reductions | output accumulators | misc | barriers
  unsigned o = 0;
  auto take = [&](unsigned bytes) {
    unsigned at = o;
    o = align_up(o + bytes, 128);
    return at;
  };
  const unsigned x_b = 4u * (unsigned)H;
  // the h area also holds the digit form of x (written by the controller while the router
  // reads x, read by the consumers before any h value arrives)
  const unsigned h_b = std::max(4u * (unsigned)(G->nseg * I), x_b);
  const unsigned wn = G->wh > 32 ? (unsigned)G->wh / 32 : 1u;
  const unsigned red_slot =
      std::max(8u * (unsigned)std::max(G->rrows, kRouterBatch) * kConsumerWarps,
               4u * 2u * (unsigned)(G->gpass * G->hr) * wn);
  const unsigned oacc_b = 4u * (unsigned)std::max(G->oacc_n, 1);
  const unsigned misc_b = kMiscBytes;
  const unsigned fixed = align_up(x_b, 128) + align_up(std::max(h_b, 128u), 128) +
                         align_up(oacc_b, 128) + misc_b;
  const unsigned per_stage = stage + red_slot + 16;
  if ((unsigned)max_smem < fixed + 4 * per_stage + 256)
    return fail(FMOE_ERR_UNSUPPORTED, "shared memory too small for 4 stages");
  int ns = (int)(((unsigned)max_smem - fixed - 256) / per_stage);
  const bool a_used = route_on || shared_on, b_used = routed_on;
  int nb = b_used ? std::min(kMaxStages, a_used ? ns / 2 : ns - 1) : 1;
  int na = std::min(kMaxStages, ns - nb);
  if (na < 1 || (a_used && na < 2) || (b_used && nb < 2))
    return fail(FMOE_ERR_UNSUPPORTED, "not enough stages (%d)", ns);
  G->nA = na;
  G->nB = nb;
  G->o_ringA = take((unsigned)na * stage);
  G->o_ringB = take((unsigned)nb * stage);
  G->o_x = take(x_b);
  G->o_h = take(std::max(h_b, 128u));
  G->red_slot = red_slot;
  G->o_red = take(red_slot * (unsigned)(na + nb));
  G->o_oacc = take(oacc_b);
  G->o_misc = take(misc_b);
  G->o_bar = o;
  o += 16u * (unsigned)(na + nb);
  G->smem_bytes = o;
  if (G->smem_bytes > (unsigned)max_smem)
    return fail(FMOE_ERR_UNSUPPORTED, "shared memory layout too large (%u)", G->smem_bytes);
  return FMOE_OK;
}

int check_layer(const fmoe_layer_desc* L, const fmoe_layer_desc* L0) {
  if (!L) return fail(FMOE_ERR_INVALID, "layer descriptor is NULL");
  if (L0 && (L->hidden != L0->hidden || L->inter != L0->inter || L->n_experts != L0->n_experts ||
             L->top_k != L0->top_k || L->bits != L0->bits))
    return fail(FMOE_ERR_INVALID, "all layers must share hidden, inter, n_experts, top_k, bits");
  int rc = check_shape(L->hidden, L->inter, L->n_experts, L->top_k, L->bits);
  if (rc) return rc;
  if (!L->experts || !L->router) return fail(FMOE_ERR_INVALID, "experts and router are required");
  const size_t eb = fmoe_expert_bytes(L->hidden, L->inter, L->bits);
  if (L->expert_stride < eb) return fail(FMOE_ERR_INVALID, "expert_stride (%zu) < expert bytes (%zu)", L->expert_stride, eb);
  if (L->expert_stride % 16) return fail(FMOE_ERR_ALIGN, "expert_stride must be a multiple of 16");
  if (!aligned16(L->experts) || !aligned16(L->router) || !aligned16(L->shared_expert) ||
      !aligned16(L->shared_gate))
    return fail(FMOE_ERR_ALIGN, "layer pointers must be 16-byte aligned");
  return FMOE_OK;
}

// ---------------------------------------------------------------- scratch
struct ScratchPlan {
  size_t off_ctrl, off_logits, off_hx, off_hbuf, total;
};

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

// Every part of the scratch is an exchange buffer that must start at zero (the whole plan is
// zeroed before each launch); the stack buffer exists only for MODE_STACK programs.
ScratchPlan plan_scratch(const Geo& G, int mode) {
  ScratchPlan s;
  size_t o = 0;
  s.off_ctrl = o; o = up256(o + 4 * (size_t)kCtrlWords);
  s.off_logits = o; o = up256(o + 8 * 2 * (size_t)std::max(G.rseg, 1) * std::max(G.nr, 1));
  s.off_hx = o; o = up256(o + 8 * 2 * (size_t)G.nseg * G.I);
  s.off_hbuf = o; o = up256(o + (mode == MODE_STACK ? 8 * 2 * (size_t)G.H : 0));
  s.total = o;
  return s;
}

void bind_scratch(Prog* P, const ScratchPlan& sp, uint8_t* base, int* err) {
  P->s.ctrl = reinterpret_cast<unsigned*>(base + sp.off_ctrl);
  P->s.logits = reinterpret_cast<unsigned long long*>(base + sp.off_logits);
  P->s.hx = reinterpret_cast<unsigned long long*>(base + sp.off_hx);
  P->s.hbuf = sp.total > sp.off_hbuf ? reinterpret_cast<unsigned long long*>(base + sp.off_hbuf)
                                     : nullptr;
  P->s.err = err;
}

void fill_layers(Prog* P, const fmoe_layer_desc* layers, int n) {
  for (int l = 0; l < n; ++l) {
    P->layers[l].experts = static_cast<const uint8_t*>(layers[l].experts);
    P->layers[l].expert_stride = layers[l].expert_stride;
    P->layers[l].shared = static_cast<const uint8_t*>(layers[l].shared_expert);
    P->layers[l].router = layers[l].router;
    P->layers[l].gate = layers[l].shared_gate;
  }
}

// Enqueue one engine run: zero the exchange buffers, launch.
int enqueue_engine(Prog* P, const Geo& G, const ScratchPlan& sp, uint8_t* base, int sms,
                   cudaStream_t st) {
  CK(cudaMemsetAsync(base, 0, sp.total, st));
  cudaError_t e = fmoe_engine_launch(P, &G, sms, st);
  if (e != cudaSuccess) return cuda_fail(e, "engine launch");
  ++g_launches;
  return FMOE_OK;
}

// Run a program with scratch taken from the library's stream-ordered pool.
int run_pooled(Prog* P, const Geo& G, DevState* d, cudaStream_t st) {
  const ScratchPlan sp = plan_scratch(G, P->mode);
  void* base = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&base, sp.total, d->pool, st);
  if (e != cudaSuccess) return fail(FMOE_ERR_NOMEM, "scratch allocation: %s", cudaGetErrorString(e));
  bind_scratch(P, sp, static_cast<uint8_t*>(base), d->err);
  int rc = enqueue_engine(P, G, sp, static_cast<uint8_t*>(base), d->sms, st);
  cudaError_t e2 = cudaFreeAsync(base, st);
  if (rc) return rc;
  if (e2 != cudaSuccess) return cuda_fail(e2, "scratch free");
  return FMOE_OK;
}

void base_prog(Prog* P, int mode) {
  memset(P, 0, sizeof *P);
  P->mode = mode;
  P->wait_ns = g_wait_ns;
  P->debug = g_debug;
  P->form = g_form;
}

}  // namespace

// =============================================================================================
extern "C" {

const char* fmoe_last_error(void) { return g_err.c_str(); }

int fmoe_version(void) { return 10000; }

void fmoe_set_wait_budget_ns(uint64_t ns) { g_wait_ns = ns < 1000 ? 1000 : ns; }

void fmoe_set_fault_injection(int flags) { g_debug = flags; }

int fmoe_set_dot_form(int form) {
  if (form < 0 || form >= FORM_COUNT) return fail(FMOE_ERR_INVALID, "dot form %d", form);
  g_form = form;
  return FMOE_OK;
}

uint64_t fmoe_launch_count(void) { return g_launches; }

int fmoe_describe_geometry(int hidden, int inter, int n_experts, int top_k, int bits, int flags,
                           int max_smem, int sms, int64_t* out, int n_out) {
  int rc = check_shape(hidden, inter, n_experts, top_k, bits);
  if (rc) return rc;
  Geo G;
  if ((rc = make_geo(hidden, inter, n_experts, top_k, bits, flags & 1, flags & 2, flags & 4,
                     flags & 8, max_smem, sms, &G)))
    return rc;
  const int64_t v[] = {G.H, G.I, G.E, G.K, G.bits, G.route_on, G.shared_on, G.routed_on,
                       G.gate_on, G.rc_h, G.rs_h, G.rc_i, G.rs_i, (int64_t)G.q_gu, G.nr, G.rseg,
                       G.rcols, G.rrows, G.au, G.hr, G.ad, G.dr, G.nseg, G.sh, G.wh, G.gh, G.si,
                       G.wi, G.pi, G.ji, G.stage_bytes, G.nA, G.nB, G.o_ringA, G.o_ringB, G.o_x,
                       G.o_h, G.o_red, G.o_oacc, G.o_misc, G.o_bar, G.oacc_n, G.smem_bytes,
                       kConsumerWarps, kMaxRowsThread, kMaxRowsWarp, G.red_slot, G.gpass};
  const int n = (int)(sizeof v / sizeof v[0]);
  for (int i = 0; i < n && i < n_out; ++i) out[i] = v[i];
  return n < n_out ? n : n_out;
}

int fmoe_sync_status(void* stream) {
  // Reads the error words of whatever this library has set up on the current device and
  // creates nothing: a caller that only uses fmoe_moe_layer_noalloc must not see the pooled
  // path's error word or memory pool allocated here.
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(FMOE_ERR_UNSUPPORTED, "device ordinal %d", dev);
  int* pooled_err = nullptr;
  int* na_err = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_dev[dev].init) pooled_err = g_dev[dev].err;
    if (g_na[dev].init) na_err = reinterpret_cast<int*>(g_na[dev].base + kNoAllocErrOff);
  }
  CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0;
  for (int* w : {pooled_err, na_err}) {
    if (!w) continue;
    int x = 0;
    CK(cudaMemcpy(&x, w, sizeof x, cudaMemcpyDeviceToHost));
    if (x != 0) {
      CK(cudaMemset(w, 0, sizeof(int)));
      if (v == 0) v = x;
    }
  }
  if (v == 0) return FMOE_OK;
  static const char* what[] = {"", "waiting for a weight stage", "waiting for a free stage",
                               "waiting for the routing decision", "waiting for a dependency",
                               "draining copies"};
  return fail(FMOE_ERR_TIMEOUT, "a device-side wait ran out of budget (%s)",
              v > 0 && v < 6 ? what[v] : "?");
}

size_t fmoe_qmat_bytes(int rows, int cols, int bits) {
  if (rows <= 0 || cols <= 0 || rows % 64 || cols % 64 || (bits != 2 && bits != 4)) return 0;
  const size_t n = (size_t)rows * (size_t)cols;
  return n * (size_t)bits / 8 + n / 16;
}

size_t fmoe_expert_bytes(int hidden, int inter, int bits) {
  const size_t a = fmoe_qmat_bytes(inter, hidden, bits), b = fmoe_qmat_bytes(hidden, inter, bits);
  if (!a || !b) return 0;
  return 2 * a + b;
}

int fmoe_pack(const float* w, int rows, int cols, int bits, void* dst, void* stream) {
  if (bits != 2 && bits != 4) return fail(FMOE_ERR_INVALID, "bits must be 2 or 4 (got %d)", bits);
  if (rows <= 0 || cols <= 0 || rows % 64 || cols % 64 || rows > (1 << 20) || cols > (1 << 16))
    return fail(FMOE_ERR_INVALID, "rows (%d) and cols (%d) must be positive multiples of 64", rows, cols);
  if (!w || !dst) return fail(FMOE_ERR_INVALID, "NULL pointer");
  if (!aligned16(w) || !aligned16(dst)) return fail(FMOE_ERR_ALIGN, "pointers must be 16-byte aligned");
  const char* wb = reinterpret_cast<const char*>(w);
  const char* db = static_cast<const char*>(dst);
  if (wb < db + fmoe_qmat_bytes(rows, cols, bits) && db < wb + (size_t)rows * cols * 4)
    return fail(FMOE_ERR_INVALID, "w and dst overlap");
  DevState* d;
  int rc = dev_state(&d);
  if (rc) return rc;
  cudaError_t e = fmoe_pack_launch(w, rows, cols, bits, dst, d->sms, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  ++g_launches;
  return FMOE_OK;
}

int fmoe_pack_q4(const float* w, int rows, int cols, void* dst, void* stream) {
  return fmoe_pack(w, rows, cols, 4, dst, stream);
}

int fmoe_pack_q2(const float* w, int rows, int cols, void* dst, void* stream) {
  return fmoe_pack(w, rows, cols, 2, dst, stream);
}

int fmoe_route(const float* x, const float* router, const float* logit_bias, int hidden,
               int n_experts, int top_k, int32_t* idx, float* weight, void* stream) {
  int rc = check_shape(hidden, 64, n_experts, top_k, 4);
  if (rc) return rc;
  if (!x || !router || !idx || !weight) return fail(FMOE_ERR_INVALID, "NULL pointer");
  if (!aligned16(x) || !aligned16(router))
    return fail(FMOE_ERR_ALIGN, "x and router must be 16-byte aligned");
  DevState* d;
  if ((rc = dev_state(&d))) return rc;
  Geo G;
  if ((rc = make_geo(hidden, 64, n_experts, top_k, 4, true, false, false, false, d->max_smem,
                     d->sms, &G)))
    return rc;
  Prog P;
  base_prog(&P, MODE_SEQ);
  P.n_units = 1; P.n_layers = 1; P.n_tokens = 1;
  P.x = x; P.bias = logit_bias; P.idx_out = idx; P.w_out = weight;
  P.out = nullptr;
  P.layers[0].router = router;
  return run_pooled(&P, G, d, static_cast<cudaStream_t>(stream));
}

int fmoe_expert_gemv(const void* expert, int hidden, int inter, int bits, const float* x,
                     float* y, void* stream) {
  int rc = check_shape(hidden, inter, 1, 1, bits);
  if (rc) return rc;
  if (!expert || !x || !y) return fail(FMOE_ERR_INVALID, "NULL pointer");
  if (!aligned16(expert) || !aligned16(x) || !aligned16(y))
    return fail(FMOE_ERR_ALIGN, "pointers must be 16-byte aligned");
  if (x == y) return fail(FMOE_ERR_INVALID, "x and y must not alias");
  DevState* d;
  if ((rc = dev_state(&d))) return rc;
  Geo G;
  if ((rc = make_geo(hidden, inter, 1, 1, bits, false, true, false, false, d->max_smem, d->sms,
                     &G)))
    return rc;
  Prog P;
  base_prog(&P, MODE_SEQ);
  P.n_units = 1; P.n_layers = 1; P.n_tokens = 1;
  P.x = x; P.out = y;
  P.layers[0].shared = static_cast<const uint8_t*>(expert);
  return run_pooled(&P, G, d, static_cast<cudaStream_t>(stream));
}

static int prep_layers(const fmoe_layer_desc* layers, int n_layers, DevState* d, Geo* G) {
  if (!layers || n_layers < 1 || n_layers > kMaxLayers)
    return fail(FMOE_ERR_INVALID, "need 1 <= n_layers <= %d", kMaxLayers);
  int rc;
  for (int l = 0; l < n_layers; ++l)
    if ((rc = check_layer(&layers[l], l ? &layers[0] : nullptr))) return rc;
  bool shared = layers[0].shared_expert != nullptr, gate = layers[0].shared_gate != nullptr;
  for (int l = 1; l < n_layers; ++l)
    if ((layers[l].shared_expert != nullptr) != shared || (layers[l].shared_gate != nullptr) != gate)
      return fail(FMOE_ERR_INVALID, "all layers must agree on having a shared expert / gate");
  const fmoe_layer_desc& L = layers[0];
  return make_geo(L.hidden, L.inter, L.n_experts, L.top_k, L.bits, true, shared, true,
                  gate && shared, d->max_smem, d->sms, G);
}

int fmoe_moe_layer_seq(const fmoe_layer_desc* layers, int n_layers, const float* x,
                       const float* residual, int n_tokens, const float* logit_bias, float* out,
                       int32_t* idx_out, float* w_out, void* stream) {
  DevState* d;
  int rc = dev_state(&d);
  if (rc) return rc;
  Geo G;
  if ((rc = prep_layers(layers, n_layers, d, &G))) return rc;
  if (n_tokens < 1) return fail(FMOE_ERR_INVALID, "n_tokens must be >= 1");
  if (n_tokens > kMaxUnits) return fail(FMOE_ERR_UNSUPPORTED, "more than %d tokens", kMaxUnits);
  if (!x || !out) return fail(FMOE_ERR_INVALID, "x and out are required");
  if (!aligned16(x) || !aligned16(out) || !aligned16(residual))
    return fail(FMOE_ERR_ALIGN, "x, residual, out must be 16-byte aligned");
  if (x == out) return fail(FMOE_ERR_INVALID, "x must not alias out");
  Prog P;
  base_prog(&P, MODE_SEQ);
  P.n_units = n_tokens; P.n_layers = n_layers; P.n_tokens = n_tokens;
  P.x = x; P.res = residual; P.out = out; P.bias = logit_bias; P.idx_out = idx_out; P.w_out = w_out;
  fill_layers(&P, layers, n_layers);
  return run_pooled(&P, G, d, static_cast<cudaStream_t>(stream));
}

int fmoe_moe_layer_seq_host(const fmoe_layer_desc* layers, int n_layers, const float* x_host,
                            const float* residual_host, int n_tokens,
                            const float* logit_bias_host, float* out_host, int32_t* idx_host,
                            float* w_host, void* stream) {
  DevState* d;
  int rc = dev_state(&d);
  if (rc) return rc;
  Geo G;
  if ((rc = prep_layers(layers, n_layers, d, &G))) return rc;
  if (n_tokens < 1) return fail(FMOE_ERR_INVALID, "n_tokens must be >= 1");
  if (!x_host || !out_host) return fail(FMOE_ERR_INVALID, "x_host and out_host are required");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t T = (size_t)n_tokens, H = (size_t)G.H, E = (size_t)G.E, K = (size_t)G.K;
  size_t o = 0;
  const size_t ox = o; o = up256(o + T * H * 4);
  const size_t orr = o; o = up256(o + (residual_host ? T * H * 4 : 0));
  const size_t ob = o; o = up256(o + (logit_bias_host ? T * E * 4 : 0));
  const size_t oo = o; o = up256(o + T * H * 4);
  const size_t oi = o; o = up256(o + T * K * 4);
  const size_t ow = o; o = up256(o + T * K * 4);
  void* dev = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&dev, o, d->pool, st);
  if (e != cudaSuccess) return fail(FMOE_ERR_NOMEM, "staging allocation: %s", cudaGetErrorString(e));
  uint8_t* b = static_cast<uint8_t*>(dev);
  auto h2d = [&](size_t off, const void* src, size_t n) {
    return n ? cudaMemcpyAsync(b + off, src, n, cudaMemcpyHostToDevice, st) : cudaSuccess;
  };
  if ((e = h2d(ox, x_host, T * H * 4)) != cudaSuccess ||
      (residual_host && (e = h2d(orr, residual_host, T * H * 4)) != cudaSuccess) ||
      (logit_bias_host && (e = h2d(ob, logit_bias_host, T * E * 4)) != cudaSuccess)) {
    cudaFreeAsync(dev, st);
    return cuda_fail(e, "host->device copy");
  }
  rc = fmoe_moe_layer_seq(layers, n_layers, reinterpret_cast<float*>(b + ox),
                          residual_host ? reinterpret_cast<float*>(b + orr) : nullptr, n_tokens,
                          logit_bias_host ? reinterpret_cast<float*>(b + ob) : nullptr,
                          reinterpret_cast<float*>(b + oo), idx_host ? reinterpret_cast<int32_t*>(b + oi) : nullptr,
                          w_host ? reinterpret_cast<float*>(b + ow) : nullptr, stream);
  if (rc == FMOE_OK) {
    if ((e = cudaMemcpyAsync(out_host, b + oo, T * H * 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (idx_host && (e = cudaMemcpyAsync(idx_host, b + oi, T * K * 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess) ||
        (w_host && (e = cudaMemcpyAsync(w_host, b + ow, T * K * 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess))
      rc = cuda_fail(e, "device->host copy");
  }
  cudaFreeAsync(dev, st);
  return rc;
}

int fmoe_moe_layer(const fmoe_layer_desc* layer, const float* x, const float* residual,
                   const float* logit_bias, float* out, int32_t* idx_out, float* w_out,
                   void* stream) {
  return fmoe_moe_layer_seq(layer, 1, x, residual, 1, logit_bias, out, idx_out, w_out, stream);
}

// ---------------------------------------------------------------- fixed-scratch variant
// The scratch of fmoe_moe_layer_noalloc: one array per device, reserved with the library's
// module image when it is loaded, so that the call itself never allocates.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FMOE_NOALLOC_SCRATCH_BYTES];

static int noalloc_state(NoAllocState** out) {
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(FMOE_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  NoAllocState& s = g_na[dev];
  if (!s.init) {
    CK(cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev));
    CK(cudaDeviceGetAttribute(&s.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    void* p = nullptr;
    CK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    CK(cudaMemset(static_cast<uint8_t*>(p) + kNoAllocErrOff, 0, sizeof(int)));
    CK(fmoe_engine_configure(s.max_smem));
    s.base = static_cast<uint8_t*>(p);
    s.init = true;
  }
  *out = &s;
  return FMOE_OK;
}

int fmoe_moe_layer_noalloc(const fmoe_layer_desc* layer, const float* x, const float* residual,
                           const float* logit_bias, float* out, int32_t* idx_out, float* w_out,
                           void* stream) {
  NoAllocState* s;
  int rc = noalloc_state(&s);
  if (rc) return rc;
  DevState shape_limits;  // prep_layers only reads the shared-memory limit
  shape_limits.sms = s->sms;
  shape_limits.max_smem = s->max_smem;
  Geo G;
  if ((rc = prep_layers(layer, 1, &shape_limits, &G))) return rc;
  if (!x || !out) return fail(FMOE_ERR_INVALID, "x and out are required");
  if (!aligned16(x) || !aligned16(out) || !aligned16(residual))
    return fail(FMOE_ERR_ALIGN, "x, residual, out must be 16-byte aligned");
  if (x == out) return fail(FMOE_ERR_INVALID, "x must not alias out");
  const ScratchPlan sp = plan_scratch(G, MODE_SEQ);
  if (sp.total > kNoAllocErrOff)
    return fail(FMOE_ERR_UNSUPPORTED,
                "fmoe_moe_layer_noalloc: this shape needs %zu bytes of scratch, the fixed area "
                "holds %zu",
                sp.total, kNoAllocErrOff);
  Prog P;
  base_prog(&P, MODE_SEQ);
  P.n_units = 1; P.n_layers = 1; P.n_tokens = 1;
  P.x = x; P.res = residual; P.out = out; P.bias = logit_bias; P.idx_out = idx_out; P.w_out = w_out;
  fill_layers(&P, layer, 1);
  bind_scratch(&P, sp, s->base, reinterpret_cast<int*>(s->base + kNoAllocErrOff));
  return enqueue_engine(&P, G, sp, s->base, s->sms, static_cast<cudaStream_t>(stream));
}

static int stack_prog(const fmoe_layer_desc* layers, int n_layers, const float* h_in,
                      int n_tokens, const float* logit_bias, float eps, float* h_out,
                      int32_t* idx_trace, float* h_trace, DevState* d, Geo* G, Prog* P) {
  int rc = prep_layers(layers, n_layers, d, G);
  if (rc) return rc;
  if (n_tokens < 1) return fail(FMOE_ERR_INVALID, "n_tokens must be >= 1");
  if ((long long)n_tokens * n_layers > kMaxUnits)
    return fail(FMOE_ERR_UNSUPPORTED, "more than %d tokens x layers in one launch", kMaxUnits);
  if (!h_in || !h_out) return fail(FMOE_ERR_INVALID, "h_in and h_out are required");
  if (!aligned16(h_in) || !aligned16(h_out) || !aligned16(h_trace))
    return fail(FMOE_ERR_ALIGN, "h_in, h_out, h_trace must be 16-byte aligned");
  if (h_in == h_out) return fail(FMOE_ERR_INVALID, "h_out must not alias h_in");
  if (!(eps >= 0.f)) return fail(FMOE_ERR_INVALID, "eps must be >= 0");
  base_prog(P, MODE_STACK);
  P->n_units = n_tokens * n_layers; P->n_layers = n_layers; P->n_tokens = n_tokens;
  P->x = h_in; P->out = h_out; P->bias = logit_bias; P->idx_out = idx_trace; P->h_trace = h_trace;
  P->eps = eps;
  fill_layers(P, layers, n_layers);
  return FMOE_OK;
}

int fmoe_moe_stack(const fmoe_layer_desc* layers, int n_layers, const float* h_in, int n_tokens,
                   const float* logit_bias, float eps, float* h_out, int32_t* idx_trace,
                   float* h_trace, void* stream) {
  DevState* d;
  int rc = dev_state(&d);
  if (rc) return rc;
  Geo G;
  Prog P;
  if ((rc = stack_prog(layers, n_layers, h_in, n_tokens, logit_bias, eps, h_out, idx_trace,
                       h_trace, d, &G, &P)))
    return rc;
  return run_pooled(&P, G, d, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

struct fmoe_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  void* scratch = nullptr;
  int kernels = 0;
};

extern "C" {

int fmoe_stack_graph_create(const fmoe_layer_desc* layers, int n_layers, const float* h_in,
                            int n_tokens, const float* logit_bias, float eps, float* h_out,
                            int32_t* idx_trace, float* h_trace, int tokens_per_launch,
                            fmoe_graph** graph) {
  if (!graph) return fail(FMOE_ERR_INVALID, "graph out-pointer is NULL");
  *graph = nullptr;
  DevState* d;
  int rc = dev_state(&d);
  if (rc) return rc;
  Geo G;
  Prog P;
  if ((rc = stack_prog(layers, n_layers, h_in, n_tokens, logit_bias, eps, h_out, idx_trace,
                       h_trace, d, &G, &P)))
    return rc;
  if (tokens_per_launch <= 0 || tokens_per_launch > n_tokens) tokens_per_launch = n_tokens;
  const int H = G.H, E = G.E, K = G.K, L = n_layers;
  const ScratchPlan sp = plan_scratch(G, MODE_STACK);
  fmoe_graph* g = new fmoe_graph();
  cudaError_t e = cudaMalloc(&g->scratch, sp.total);
  if (e != cudaSuccess) {
    delete g;
    return fail(FMOE_ERR_NOMEM, "graph scratch: %s", cudaGetErrorString(e));
  }
  cudaStream_t cs;
  if ((e = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking)) != cudaSuccess) {
    cudaFree(g->scratch);
    delete g;
    return cuda_fail(e, "capture stream");
  }
  const uint64_t launches_before = g_launches;
  e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (e == cudaSuccess) {
    for (int t0 = 0; t0 < n_tokens && rc == FMOE_OK; t0 += tokens_per_launch) {
      const int nt = std::min(tokens_per_launch, n_tokens - t0);
      Prog Q = P;
      Q.n_tokens = nt;
      Q.n_units = nt * L;
      Q.x = h_in + (size_t)t0 * H;
      Q.out = h_out + (size_t)t0 * H;
      Q.bias = logit_bias ? logit_bias + (size_t)t0 * L * E : nullptr;
      Q.idx_out = idx_trace ? idx_trace + (size_t)t0 * L * K : nullptr;
      Q.h_trace = h_trace ? h_trace + (size_t)t0 * L * H : nullptr;
      bind_scratch(&Q, sp, static_cast<uint8_t*>(g->scratch), d->err);
      rc = enqueue_engine(&Q, G, sp, static_cast<uint8_t*>(g->scratch), d->sms, cs);
    }
    cudaError_t e2 = cudaStreamEndCapture(cs, &g->graph);
    if (rc == FMOE_OK && e2 != cudaSuccess) rc = cuda_fail(e2, "end capture");
  } else {
    rc = cuda_fail(e, "begin capture");
  }
  cudaStreamDestroy(cs);
  g->kernels = (int)(g_launches - launches_before);
  g_launches = launches_before;
  if (rc == FMOE_OK) {
    e = cudaGraphInstantiate(&g->exec, g->graph, 0);
    if (e != cudaSuccess) rc = cuda_fail(e, "graph instantiate");
  }
  if (rc != FMOE_OK) {
    if (g->graph) cudaGraphDestroy(g->graph);
    cudaFree(g->scratch);
    delete g;
    return rc;
  }
  *graph = g;
  return FMOE_OK;
}

int fmoe_stack_graph_launch(fmoe_graph* g, void* stream) {
  if (!g || !g->exec) return fail(FMOE_ERR_INVALID, "graph is NULL");
  cudaError_t e = cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "graph launch");
  g_launches += (uint64_t)g->kernels;
  return FMOE_OK;
}

int fmoe_stack_graph_destroy(fmoe_graph* g) {
  if (!g) return FMOE_OK;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  if (g->scratch) cudaFree(g->scratch);
  delete g;
  return FMOE_OK;
}

}  // extern "C"
