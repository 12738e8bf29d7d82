// C ABI entry points: argument checks, workspace layout, kernel choice.
#include <string.h>

#include <atomic>

#include "launch.h"

namespace gdn {
namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_cc[kMaxDevices];

// SM count and compute capability (major*10+minor) of the current device.
int device_info(int *sm_count, int *cc) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_NO_DEVICE;
  int sms = g_sm_count[dev].load(std::memory_order_relaxed);
  int c = g_cc[dev].load(std::memory_order_relaxed);
  if (sms <= 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return GDN_ERR_CUDA;
    c = major * 10 + minor;
    g_cc[dev].store(c, std::memory_order_relaxed);
    g_sm_count[dev].store(sms, std::memory_order_relaxed);
  }
  *sm_count = sms;
  *cc = c;
  return GDN_OK;
}

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_sizes(int B, int H, int F, int L, int dk, int dv) {
  if (B < 1 || H < 1 || F < 1 || L < 1 || dk < 1 || dv < 1) return GDN_ERR_INVALID_ARG;
  if (dk > 128 || dv > 128) return GDN_ERR_UNSUPPORTED;
  // every index fits in int64; unit counts fit in int32 tickets
  const long long units = (long long)B * H * F;
  if (units > (1LL << 30)) return GDN_ERR_UNSUPPORTED;
  if ((long long)B * H * F * L > (1LL << 40)) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

int pick_gdn_impl(const gdn_opts_t *o, int dk, int dv) {
  if (o->impl != GDN_IMPL_AUTO) return o->impl;
  if (o->in_dtype == GDN_DTYPE_BF16 && gdn_tc_supported(dk, dv)) return GDN_IMPL_TC;
  return GDN_IMPL_FRAME_SIMT;
}

int pick_relu_impl(const gdn_opts_t *o, int dk, int dv) {
  if (o->impl != GDN_IMPL_AUTO) return o->impl;
  if (o->in_dtype == GDN_DTYPE_BF16 && relu_tc_supported(dk, dv)) return GDN_IMPL_TC;
  return GDN_IMPL_FRAME_SIMT;
}

size_t gdn_state_elems(int impl, int dk, int dv) {
  if (impl == GDN_IMPL_TC) return gdn_tc_state_elems(dk, dv);
  return (size_t)dk * dv;
}

// Chunk segments per frame (GDN_IMPL_TC).  The automatic choice considers
// segments only for launches of at most kSegUnitsMax frames, and at most
// kMaxSegs of them.
constexpr long kSegUnitsMax = 128;
constexpr int kMaxSegs = 8;

// The most segments a launch with these sizes and options may use; sizes the
// workspace without asking the device.
int gdn_seg_bound(int impl, const gdn_opts_t *o, long units, int L) {
  if (impl != GDN_IMPL_TC) return 1;
  const int nch = (L + 63) / 64;
  if (o->segments > 0) return o->segments < nch ? o->segments : nch;
  if (units > kSegUnitsMax) return 1;
  return nch < kMaxSegs ? nch : kMaxSegs;
}

// The segments of a launch on `sms` SMs: all units * P CTAs must be resident
// at once.  Automatic: P > 1 only when the frames alone would fill at most
// half the grid, and then about sqrt(chunks per frame) of them.  A call's time
// grows by one chunk's latency per chunk in a segment and by one chain step's
// per segment, and the two were measured about equal (~5.5-6 us each for one
// 920-token frame of 20 heads: 109 us at P = 1, 74 at 2, 62 at 4, 69 at 8).
int gdn_segs(int impl, const gdn_opts_t *o, int sms, long units, int L) {
  int bound = gdn_seg_bound(impl, o, units, L);
  if (bound <= 1) return 1;
  long g = sms;
  if (o->max_ctas > 0 && o->max_ctas < g) g = o->max_ctas;
  if (o->segments <= 0) {
    if (2 * units > g) return 1;
    const int nch = (L + 63) / 64;
    int want = 1;
    while (want * want < nch) ++want;
    if (want < bound) bound = want;
  }
  const long fit = g / units;
  const long P = fit < bound ? fit : bound;
  return (int)(P < 1 ? 1 : P);
}

// Workspace of gdn with P segments: the chain scratch over units * P segment
// units, then (P > 1) each frame's end state as bf16 high/low pairs, d_k
// words per row of S^T.
size_t gdn_ws_bytes_p(int impl, int B, int H, int F, int dk, int dv, int P) {
  if (impl == GDN_IMPL_SEQ) return 0;
  const long units = (long)B * H * F;
  size_t b = chain_workspace_bytes(units * P, (long)gdn_state_elems(impl, dk, dv));
  if (P > 1) b += align_up(sizeof(uint32_t) * (size_t)units * dk * dv, 256);
  return b;
}

size_t gdn_ws_bytes(int impl, const gdn_opts_t *o, int B, int H, int F, int L, int dk, int dv) {
  return gdn_ws_bytes_p(impl, B, H, F, dk, dv, gdn_seg_bound(impl, o, (long)B * H * F, L));
}

size_t relu_ws_bytes(int B, int H, int F, int dk, int dv) {
  return chain_workspace_bytes((long)B * H * F, (long)(dv + 1) * dk);
}

unsigned long long spin_ns(const gdn_opts_t *o) {
  const long long us = o->spin_limit_us > 0 ? o->spin_limit_us : 2000000;
  return (unsigned long long)us * 1000ull;
}

int grid_for(const gdn_opts_t *o, int sms, long units) {
  long g = sms;
  if (o->max_ctas > 0 && o->max_ctas < g) g = o->max_ctas;
  if (units < g) g = units;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" int gdn_abi_version(void) { return GDN_ABI_VERSION; }

extern "C" const char *gdn_status_string(int s) {
  switch (s) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer, bad size or workspace)";
    case GDN_ERR_UNSUPPORTED: return "unsupported sizes or options for this build";
    case GDN_ERR_CUDA: return "CUDA runtime error";
    case GDN_ERR_TIMEOUT: return "device: a bounded in-kernel wait expired; outputs are invalid";
    case GDN_ERR_NO_DEVICE: return "no usable sm_100 device";
    default: return "unknown status";
  }
}

extern "C" size_t gdn_workspace_bytes(int op, int B, int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts || check_sizes(B, H, F, L, dk, dv) != GDN_OK) return 0;
  if (op == GDN_OP_GDN) return gdn_ws_bytes(pick_gdn_impl(opts, dk, dv), opts, B, H, F, L, dk, dv);
  if (op == GDN_OP_RELU_LA) return relu_ws_bytes(B, H, F, dk, dv);
  return 0;
}

extern "C" int gdn_frame_fwd(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                             const float *state_in, float *state_out, float *o, int B, int H, int F, int L,
                             int dk, int dv, const gdn_opts_t *opts) {
  if (!opts) return GDN_ERR_INVALID_ARG;
  if (!q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  if (opts->impl < GDN_IMPL_AUTO || opts->impl > GDN_IMPL_TC) return GDN_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, F, L, dk, dv);
  if (rc != GDN_OK) return rc;
  const void *ptrs[] = {q, k, v, alpha, beta, state_in, state_out, o, opts->workspace, opts->status};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return GDN_ERR_INVALID_ARG;
  int sms = 0, cc = 0;
  rc = device_info(&sms, &cc);
  if (rc != GDN_OK) return rc;
  if (cc != 100) return GDN_ERR_NO_DEVICE;
  const int impl = pick_gdn_impl(opts, dk, dv);
  if (impl == GDN_IMPL_TC && (opts->in_dtype != GDN_DTYPE_BF16 || !gdn_tc_supported(dk, dv)))
    return GDN_ERR_UNSUPPORTED;

  cudaStream_t st = (cudaStream_t)opts->stream;
  GdnParams p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta;
  p.state_in = state_in; p.state_out = state_out; p.o = o;
  p.B = B; p.H = H; p.F = F; p.L = L; p.dk = dk; p.dv = dv;
  p.gates_are_logits = opts->gates_are_logits ? 1 : 0;
  p.status = opts->status;
  p.spin_limit_ns = spin_ns(opts);
  p.withhold = opts->test_withhold_unit > 0 ? (long)opts->test_withhold_unit - 1 : -1;
  p.segs = 1;

  cudaError_t e;
  if (impl == GDN_IMPL_SEQ) {
    e = launch_gdn_seq(p, opts->in_dtype, st);
  } else {
    const long units = (long)B * H * F;
    const int P = gdn_segs(impl, opts, sms, units, L);
    const size_t need = gdn_ws_bytes_p(impl, B, H, F, dk, dv, P);
    if (!opts->workspace || opts->workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
    p.ws = chain_workspace(opts->workspace, units * P);
    p.segs = P;
    if (P > 1)
      p.ro_states = reinterpret_cast<uint32_t *>(
          (char *)opts->workspace + chain_workspace_bytes(units * P, (long)gdn_state_elems(impl, dk, dv)));
    e = cudaMemsetAsync(opts->workspace, 0, chain_workspace_zero_bytes(units * P), st);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    const int grid = P > 1 ? (int)(units * P) : grid_for(opts, sms, units);
    e = impl == GDN_IMPL_TC ? launch_gdn_tc(p, grid, P > 1, st)
                            : launch_gdn_frame_simt(p, opts->in_dtype, grid, st);
  }
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" int relu_la_block_fwd(const void *q, const void *k, const void *v, const float *kv_in, const float *z_in,
                                 float *kv_out, float *z_out, float *o, int B, int H, int F, int L, int dk, int dv,
                                 float eps, const gdn_opts_t *opts) {
  if (!opts) return GDN_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  if (opts->impl != GDN_IMPL_AUTO && opts->impl != GDN_IMPL_FRAME_SIMT && opts->impl != GDN_IMPL_TC)
    return GDN_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return GDN_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, F, L, dk, dv);
  if (rc != GDN_OK) return rc;
  const void *ptrs[] = {q, k, v, kv_in, z_in, kv_out, z_out, o, opts->workspace, opts->status};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return GDN_ERR_INVALID_ARG;
  int sms = 0, cc = 0;
  rc = device_info(&sms, &cc);
  if (rc != GDN_OK) return rc;
  if (cc != 100) return GDN_ERR_NO_DEVICE;
  const int impl = pick_relu_impl(opts, dk, dv);
  if (impl == GDN_IMPL_TC && (opts->in_dtype != GDN_DTYPE_BF16 || !relu_tc_supported(dk, dv)))
    return GDN_ERR_UNSUPPORTED;
  const long units = (long)B * H * F;
  const size_t need = relu_ws_bytes(B, H, F, dk, dv);
  if (!opts->workspace || opts->workspace_bytes < need) return GDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;

  cudaStream_t st = (cudaStream_t)opts->stream;
  ReluParams p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.kv_in = kv_in; p.z_in = z_in; p.kv_out = kv_out; p.z_out = z_out; p.o = o;
  p.B = B; p.H = H; p.F = F; p.L = L; p.dk = dk; p.dv = dv; p.eps = eps;
  p.status = opts->status;
  p.spin_limit_ns = spin_ns(opts);
  p.withhold = opts->test_withhold_unit > 0 ? (long)opts->test_withhold_unit - 1 : -1;
  p.ws = chain_workspace(opts->workspace, units);
  cudaError_t e = cudaMemsetAsync(opts->workspace, 0, chain_workspace_zero_bytes(units), st);
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  const int grid = grid_for(opts, sms, units);
  e = impl == GDN_IMPL_TC ? launch_relu_tc(p, grid, st) : launch_relu_frame_simt(p, opts->in_dtype, grid, st);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// ---------------------------------------------------------------- host I/O

namespace {
struct HostLayout {
  size_t q, k, v, alpha, beta, s_in, o, s_out, ws, total;
};

HostLayout host_layout(int B, int H, int F, int L, int dk, int dv, int in_dtype, size_t ws_bytes) {
  const size_t esz = in_dtype == GDN_DTYPE_F32 ? 4 : 2;
  const size_t N = (size_t)F * L, BH = (size_t)B * H;
  HostLayout h;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  h.q = take(BH * N * dk * esz);
  h.k = take(BH * N * dk * esz);
  h.v = take(BH * N * dv * esz);
  h.alpha = take(BH * F * 4);
  h.beta = take(BH * N * 4);
  h.s_in = take(BH * dk * dv * 4);
  h.o = take(BH * N * dv * 4);
  h.s_out = take(BH * dk * dv * 4);
  h.ws = take(ws_bytes);
  h.total = off;
  return h;
}
}  // namespace

extern "C" size_t gdn_workspace_bytes_host(int B, int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts || check_sizes(B, H, F, L, dk, dv) != GDN_OK) return 0;
  const size_t ws = gdn_ws_bytes(pick_gdn_impl(opts, dk, dv), opts, B, H, F, L, dk, dv);
  return host_layout(B, H, F, L, dk, dv, opts->in_dtype, ws).total;
}

extern "C" int gdn_frame_fwd_host(const void *q, const void *k, const void *v, const float *alpha,
                                  const float *beta, const float *state_in, float *state_out, float *o, int B,
                                  int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts || !q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, F, L, dk, dv);
  if (rc != GDN_OK) return rc;
  const size_t ws = gdn_ws_bytes(pick_gdn_impl(opts, dk, dv), opts, B, H, F, L, dk, dv);
  const HostLayout h = host_layout(B, H, F, L, dk, dv, opts->in_dtype, ws);
  if (!opts->workspace || opts->workspace_bytes < h.total) return GDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
  char *base = (char *)opts->workspace;
  cudaStream_t st = (cudaStream_t)opts->stream;
  const size_t esz = opts->in_dtype == GDN_DTYPE_F32 ? 4 : 2;
  const size_t N = (size_t)F * L, BH = (size_t)B * H;
  struct Cp { void *dst; const void *src; size_t n; };
  const Cp in[] = {{base + h.q, q, BH * N * dk * esz}, {base + h.k, k, BH * N * dk * esz},
                   {base + h.v, v, BH * N * dv * esz}, {base + h.alpha, alpha, BH * F * 4},
                   {base + h.beta, beta, BH * N * 4},  {base + h.s_in, state_in, BH * dk * dv * 4}};
  for (const Cp &c : in) {
    if (!c.src) continue;
    if (cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, st) != cudaSuccess) return GDN_ERR_CUDA;
  }
  gdn_opts_t inner = *opts;
  inner.workspace = base + h.ws;
  inner.workspace_bytes = ws;
  rc = gdn_frame_fwd(base + h.q, base + h.k, base + h.v, (const float *)(base + h.alpha),
                     (const float *)(base + h.beta), state_in ? (const float *)(base + h.s_in) : nullptr,
                     state_out ? (float *)(base + h.s_out) : nullptr, (float *)(base + h.o), B, H, F, L, dk, dv,
                     &inner);
  if (rc != GDN_OK) return rc;
  if (cudaMemcpyAsync(o, base + h.o, BH * N * dv * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (state_out &&
      cudaMemcpyAsync(state_out, base + h.s_out, BH * dk * dv * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GDN_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
