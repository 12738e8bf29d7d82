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
  if (o->impl == GDN_IMPL_TC_PFORM) return GDN_IMPL_TC;
  if (o->impl != GDN_IMPL_AUTO) return o->impl;
  if (o->in_dtype == GDN_DTYPE_BF16 && gdn_tc_supported(dk, dv)) return GDN_IMPL_TC;
  return GDN_IMPL_FRAME_SIMT;
}

int pick_relu_impl(const gdn_opts_t *o, int dk, int dv) {
  if (o->impl != GDN_IMPL_AUTO) return o->impl;
  if (o->in_dtype == GDN_DTYPE_BF16 && relu_tc_supported(dk, dv)) return GDN_IMPL_TC;
  return GDN_IMPL_FRAME_SIMT;
}

// Floats of scratch per published frame state of the frame-chain kernels other
// than the product-form one (which gdn_ws_bytes_p sizes on its own).
size_t gdn_state_elems(int impl, int dk, int dv) {
  if (impl == GDN_IMPL_TC) return gdn_tc_state_elems(dk, dv);
  return (size_t)dk * dv;
}

// The product-form tensor-core kernel runs when it is asked for (one segment per frame).
bool use_pform(int impl, const gdn_opts_t *o, int P, int dk, int dv) {
  return impl == GDN_IMPL_TC && o->impl == GDN_IMPL_TC_PFORM && P == 1 && gdn_pform_supported(dk, dv);
}

// Chunk segments per frame (GDN_IMPL_TC).  The automatic choice considers
// segments only for launches of at most kSegUnitsMax frames, and at most
// kMaxSegs of them.
constexpr long kSegUnitsMax = 128;
constexpr int kMaxSegs = 8;

// The most segments a launch with these sizes and options may use; sizes the
// workspace without asking the device.
int gdn_seg_bound(int impl, const gdn_opts_t *o, long units, int L) {
  if (impl != GDN_IMPL_TC || o->impl == GDN_IMPL_TC_PFORM) return 1;
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
size_t gdn_ws_bytes_p(int impl, const gdn_opts_t *o, int B, int H, int F, int dk, int dv, int P) {
  if (impl == GDN_IMPL_SEQ) return 0;
  const long units = (long)B * H * F;
  if (use_pform(impl, o, P, dk, dv))
    return chain_workspace_bytes(units, (long)(gdn_pform_state_bytes(dk, dv) / sizeof(float)));
  size_t b = chain_workspace_bytes(units * P, (long)gdn_state_elems(impl, dk, dv));
  if (P > 1) b += align_up(sizeof(uint32_t) * (size_t)units * dk * dv, 256);
  return b;
}

// Bytes of the 3D RoPE table (after the chain scratch in the workspace).
size_t gdn_rope_bytes(const gdn_opts_t *o, int F, int L, int dk) {
  if (o->rope_grid_w <= 0 || L % o->rope_grid_w) return 0;
  return align_up(sizeof(float2) * rope_table_entries(F, L, o->rope_grid_w, dk), 256);
}

// Workspace for any launch these sizes and options may lead to: the segment
// count is chosen on the device, so both the most segments and one segment
// (the product-form kernel) are covered; then the RoPE table.
size_t gdn_ws_chain_bytes(int impl, const gdn_opts_t *o, int B, int H, int F, int L, int dk, int dv) {
  const int bound = gdn_seg_bound(impl, o, (long)B * H * F, L);
  size_t b = gdn_ws_bytes_p(impl, o, B, H, F, dk, dv, bound);
  if (bound > 1) {
    const size_t b1 = gdn_ws_bytes_p(impl, o, B, H, F, dk, dv, 1);
    if (b1 > b) b = b1;
  }
  return b;
}

size_t gdn_ws_bytes(int impl, const gdn_opts_t *o, int B, int H, int F, int L, int dk, int dv) {
  return gdn_ws_chain_bytes(impl, o, B, H, F, L, dk, dv) + gdn_rope_bytes(o, F, L, dk);
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

namespace gdn {
namespace {
bool overlap(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
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
    case GDN_ERR_RANGE:
      return "device: a value met the fp16 range of the tensor-core operands (|q|, |v| or |S| >= 65504, or "
             "NaN); outputs are invalid";
    default: return "unknown status";
  }
}

extern "C" const char *gdn_status_str(int s) { return gdn_status_string(s); }

namespace gdn {
namespace {
// The backward's forward recompute: the tensor-core kernel for bf16 inputs where it
// applies (one unit per frame), else the fp32 CUDA-core frame kernel.
int pick_bwd_fwd_impl(const gdn_opts_t *o, int dk, int dv) {
  if (o->impl == GDN_IMPL_FRAME_SIMT) return GDN_IMPL_FRAME_SIMT;
  if (o->impl == GDN_IMPL_TC) return GDN_IMPL_TC;
  return o->in_dtype == GDN_DTYPE_BF16 && gdn_tc_supported(dk, dv) ? GDN_IMPL_TC : GDN_IMPL_FRAME_SIMT;
}

// Backward workspace: the recompute's chain scratch, then A_f^T and S_f of every
// frame, G_f of every frame, the per-column-group dalpha partial sums, (bf16
// inputs) each chunk's Linv and the residuals, and (with the 3D RoPE) its table.
struct BwdLayout {
  size_t maps, states, gbuf, part, linv, rbuf, rope, total;
};
BwdLayout bwd_layout(const gdn_opts_t *o, int B, int H, int F, int L, int dk, int dv) {
  BwdLayout w;
  const size_t fr = (size_t)B * H * F;
  w.maps = align_up(gdn_ws_bytes_p(pick_bwd_fwd_impl(o, dk, dv), o, B, H, F, dk, dv, 1), 256);
  w.states = w.maps + align_up(sizeof(float) * fr * dk * dk, 256);
  w.gbuf = w.states + align_up(sizeof(float) * fr * dk * dv, 256);
  w.part = w.gbuf + align_up(sizeof(float) * fr * dk * dv, 256);
  w.linv = w.part + align_up(sizeof(float) * fr * ((dv + 15) / 16), 256);
  w.rbuf = w.linv;
  w.total = w.linv;
  if (o->in_dtype == GDN_DTYPE_BF16) {  // the tensor-core frame kernel keeps each chunk's Linv and residuals
    w.rbuf = w.linv + align_up(sizeof(float) * fr * gdn_bwd_chunks(L) * 48 * 48, 256);
    w.total = w.rbuf + (dv > dk ? align_up(sizeof(float) * fr * L * dv, 256) : 0);
  }
  w.rope = w.total;
  w.total += gdn_rope_bytes(o, F, L, dk);
  return w;
}
}  // namespace
}  // namespace gdn

extern "C" size_t gdn_workspace_bytes(int op, int B, int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts || check_sizes(B, H, F, L, dk, dv) != GDN_OK) return 0;
  if (op == GDN_OP_GDN) return gdn_ws_bytes(pick_gdn_impl(opts, dk, dv), opts, B, H, F, L, dk, dv);
  if (op == GDN_OP_RELU_LA) return relu_ws_bytes(B, H, F, dk, dv);
  if (op == GDN_OP_GDN_BWD) return bwd_layout(opts, B, H, F, L, dk, dv).total;
  return 0;
}

extern "C" int gdn_frame_bwd(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                             const float *state_in, const float *d_o, const float *dstate_out, float *dq,
                             float *dk_out, float *dv_out, float *dalpha, float *dbeta, float *dstate_in, int B,
                             int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts) return GDN_ERR_INVALID_ARG;
  if (!q || !k || !v || !alpha || !beta || !d_o || !dq || !dk_out || !dv_out || !dalpha || !dbeta)
    return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  if (opts->impl != GDN_IMPL_AUTO && opts->impl != GDN_IMPL_FRAME_SIMT && opts->impl != GDN_IMPL_TC)
    return GDN_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, F, L, dk, dv);
  if (rc != GDN_OK) return rc;
  if (!gdn_bwd_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
  const bool rope = opts->rope_grid_w != 0;
  if (rope && (opts->rope_grid_w < 0 || L % opts->rope_grid_w || dk % 2 || !(opts->rope_base >= 0.0f) ||
               opts->rope_frame_offset < 0))
    return GDN_ERR_INVALID_ARG;
  const void *ptrs[] = {q, k, v, alpha, beta, state_in, d_o, dstate_out, dq, dk_out, dv_out, dalpha, dbeta,
                        dstate_in, opts->workspace, opts->status};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return GDN_ERR_INVALID_ARG;
  // the outputs overlap neither one another nor the inputs
  const size_t N = (size_t)B * H * F * L, nsq = (size_t)B * H * dk * dv, nf = (size_t)B * H * F;
  const size_t isz = opts->in_dtype == GDN_DTYPE_F32 ? 4 : 2;
  const void *outs[] = {dq, dk_out, dv_out, dalpha, dbeta, dstate_in};
  const size_t osz[] = {N * dk * 4, N * dk * 4, N * dv * 4, nf * 4, N * 4, nsq * 4};
  const void *ins[] = {q, k, v, alpha, beta, state_in, d_o, dstate_out};
  const size_t insz[] = {N * dk * isz, N * dk * isz, N * dv * isz, nf * 4, N * 4, nsq * 4, N * dv * 4, nsq * 4};
  for (int a = 0; a < 6; ++a) {
    for (int c = a + 1; c < 6; ++c)
      if (overlap(outs[a], osz[a], outs[c], osz[c])) return GDN_ERR_INVALID_ARG;
    for (int c = 0; c < 8; ++c)
      if (overlap(outs[a], osz[a], ins[c], insz[c])) return GDN_ERR_INVALID_ARG;
  }
  int sms = 0, cc = 0;
  rc = device_info(&sms, &cc);
  if (rc != GDN_OK) return rc;
  if (cc != 100) return GDN_ERR_NO_DEVICE;
  const int fimpl = pick_bwd_fwd_impl(opts, dk, dv);
  if (fimpl == GDN_IMPL_TC && (opts->in_dtype != GDN_DTYPE_BF16 || !gdn_tc_supported(dk, dv)))
    return GDN_ERR_UNSUPPORTED;
  const BwdLayout w = bwd_layout(opts, B, H, F, L, dk, dv);
  if (!opts->workspace || opts->workspace_bytes < w.total) return GDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
  char *ws = static_cast<char *>(opts->workspace);
  float *maps = reinterpret_cast<float *>(ws + w.maps);
  float *states = reinterpret_cast<float *>(ws + w.states);
  cudaStream_t st = (cudaStream_t)opts->stream;

  // 1. forward recompute: every frame's A_f^T and S_f (no read-out)
  GdnParams p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta;
  p.state_in = state_in;
  p.B = B; p.H = H; p.F = F; p.L = L; p.dk = dk; p.dv = dv;
  p.gates_are_logits = opts->gates_are_logits ? 1 : 0;
  p.status = opts->status;
  p.spin_limit_ns = spin_ns(opts);
  p.withhold = opts->test_withhold_unit > 0 ? (long)opts->test_withhold_unit - 1 : -1;
  p.segs = 1;
  p.save_maps = maps;
  p.save_states = states;
  const long units = (long)B * H * F;
  p.ws = chain_workspace(ws, units);
  cudaError_t e = cudaMemsetAsync(ws, 0, chain_workspace_zero_bytes(units), st);
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  if (rope) {  // the table, filled on the stream before the recompute; the backward kernels read it too
    p.rope_on = 1;
    p.rope_gw = opts->rope_grid_w;
    p.rope_dh = 2 * (dk / 6);
    p.rope_dt = dk - 2 * p.rope_dh;
    p.rope_tab = reinterpret_cast<const float2 *>(ws + w.rope);
    e = launch_rope_table(p, opts->rope_frame_offset, opts->rope_base > 0.0f ? opts->rope_base : 10000.0f, st);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
  }
  const int grid = grid_for(opts, sms, units);
  e = fimpl == GDN_IMPL_TC ? launch_gdn_tc(p, grid, false, st) : launch_gdn_frame_simt(p, opts->in_dtype, grid, st);
  if (e != cudaSuccess) return GDN_ERR_CUDA;

  // 2-3. the adjoint frame chain, then the frame-parallel backward
  BwdParams b;
  memset(&b, 0, sizeof(b));
  b.q = q; b.k = k; b.v = v; b.alpha = alpha; b.beta = beta; b.state_in = state_in;
  b.d_o = d_o; b.dstate_out = dstate_out;
  b.maps = maps; b.states = states;
  b.gbuf = reinterpret_cast<float *>(ws + w.gbuf);
  b.dal_part = reinterpret_cast<float *>(ws + w.part);
  b.linv_buf = w.rbuf > w.linv ? reinterpret_cast<float *>(ws + w.linv) : nullptr;  // bf16 inputs only
  b.rbuf = w.rope > w.rbuf ? reinterpret_cast<float *>(ws + w.rbuf) : nullptr;  // own rows only when dv > dk
  b.dq = dq; b.dk_out = dk_out; b.dv_out = dv_out; b.dalpha = dalpha; b.dbeta = dbeta; b.dstate_in = dstate_in;
  b.B = B; b.H = H; b.F = F; b.L = L; b.dk = dk; b.dv = dv;
  b.gates_are_logits = p.gates_are_logits;
  e = launch_gdn_bwd(b, p, opts->in_dtype, st);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}


extern "C" int gdn_frame_fwd(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                             const float *state_in, float *state_out, float *o, int B, int H, int F, int L,
                             int dk, int dv, const gdn_opts_t *opts) {
  if (!opts) return GDN_ERR_INVALID_ARG;
  if (!q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  if (opts->impl < GDN_IMPL_AUTO || opts->impl > GDN_IMPL_TC_PFORM) return GDN_ERR_INVALID_ARG;
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
  if (opts->impl == GDN_IMPL_TC_PFORM && !gdn_pform_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
  const bool rope = opts->rope_grid_w != 0;
  if (rope) {
    if (opts->rope_grid_w < 0 || L % opts->rope_grid_w || dk % 2 || !(opts->rope_base >= 0.0f) ||
        opts->rope_frame_offset < 0)
      return GDN_ERR_INVALID_ARG;
    if (opts->impl == GDN_IMPL_TC_PFORM) return GDN_ERR_UNSUPPORTED;
  }

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
  if (rope) {
    // the table after the chain scratch; filled on the stream before the recurrence
    const size_t chain = impl == GDN_IMPL_SEQ ? 0 : gdn_ws_chain_bytes(impl, opts, B, H, F, L, dk, dv);
    const size_t need = chain + gdn_rope_bytes(opts, F, L, dk);
    if (!opts->workspace || opts->workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
    p.rope_on = 1;
    p.rope_gw = opts->rope_grid_w;
    p.rope_dh = 2 * (dk / 6);
    p.rope_dt = dk - 2 * p.rope_dh;
    p.rope_tab = reinterpret_cast<const float2 *>((char *)opts->workspace + chain);
    e = launch_rope_table(p, opts->rope_frame_offset, opts->rope_base > 0.0f ? opts->rope_base : 10000.0f, st);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
  }
  if (impl == GDN_IMPL_SEQ) {
    e = launch_gdn_seq(p, opts->in_dtype, st);
  } else {
    const long units = (long)B * H * F;
    const int P = gdn_segs(impl, opts, sms, units, L);
    const size_t need = gdn_ws_bytes_p(impl, opts, B, H, F, dk, dv, P);
    if (!opts->workspace || opts->workspace_bytes < need) return GDN_ERR_INVALID_ARG;
    // (with RoPE the table follows the scratch of the most segments; checked above)
    if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
    p.ws = chain_workspace(opts->workspace, units * P);
    p.segs = P;
    if (P > 1)
      p.ro_states = reinterpret_cast<uint32_t *>(
          (char *)opts->workspace + chain_workspace_bytes(units * P, (long)gdn_state_elems(impl, dk, dv)));
    e = cudaMemsetAsync(opts->workspace, 0, chain_workspace_zero_bytes(units * P), st);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    const int grid = P > 1 ? (int)(units * P) : grid_for(opts, sms, units);
    if (use_pform(impl, opts, P, dk, dv))
      e = launch_gdn_pform(p, grid, st);
    else if (impl == GDN_IMPL_TC)
      e = launch_gdn_tc(p, grid, P > 1, st);
    else
      e = launch_gdn_frame_simt(p, opts->in_dtype, grid, st);
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
  if (opts->rope_grid_w != 0) return GDN_ERR_UNSUPPORTED;  // the position embedding is built for gdn only
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


extern "C" int temporal_conv_fwd(const void *x, const float *w, const float *bias, const void *cache_in,
                                 void *cache_out, void *y, int B, int F, int HW, int C, const gdn_opts_t *opts) {
  using namespace gdn;
  if (!opts || !x || !w || !y) return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  if (B < 1 || F < 1 || HW < 1 || C < 1) return GDN_ERR_INVALID_ARG;
  if ((long long)B * F * HW * C > (1LL << 40)) return GDN_ERR_UNSUPPORTED;
  const void *ptrs[] = {x, w, bias, cache_in, cache_out, y};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return GDN_ERR_INVALID_ARG;
  const size_t es = opts->in_dtype == GDN_DTYPE_BF16 ? 2 : 4;
  const size_t nx = es * (size_t)B * F * HW * C, nc = es * (size_t)B * HW * C;
  if (overlap(x, nx, y, nx) || overlap(cache_in, nc, y, nx) || overlap(cache_out, nc, y, nx) ||
      overlap(cache_out, nc, x, nx) || (cache_in != cache_out && overlap(cache_in, nc, cache_out, nc)))
    return GDN_ERR_INVALID_ARG;
  int sms = 0, cc = 0;
  int rc = device_info(&sms, &cc);
  if (rc != GDN_OK) return rc;
  if (cc != 100) return GDN_ERR_NO_DEVICE;
  const cudaError_t e = launch_temporal_conv(x, w, bias, cache_in, cache_out, y, B, F, HW, C, opts->in_dtype,
                                             opts->max_ctas, (cudaStream_t)opts->stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" int softmax_window_fwd(const void *q, const void *k, const void *v, float *o, int B, int H, int F, int L,
                                  int dk, int dv, int W, float scale, const gdn_opts_t *opts) {
  using namespace gdn;
  if (!opts || !q || !k || !v || !o) return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  if (W < 1 || !(scale >= 0.0f)) return GDN_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, F, L, dk, dv);
  if (rc != GDN_OK) return rc;
  if (opts->impl != GDN_IMPL_AUTO && opts->impl != GDN_IMPL_FRAME_SIMT && opts->impl != GDN_IMPL_TC)
    return GDN_ERR_INVALID_ARG;
  const bool tc_ok = opts->in_dtype == GDN_DTYPE_BF16 && softmax_window_supported(dk, dv);
  if (opts->impl == GDN_IMPL_TC && !tc_ok) return GDN_ERR_UNSUPPORTED;
  const bool use_tc = tc_ok && opts->impl != GDN_IMPL_FRAME_SIMT;
  const void *ptrs[] = {q, k, v, o, opts->status};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return GDN_ERR_INVALID_ARG;
  const size_t N = (size_t)B * H * F * L, es = opts->in_dtype == GDN_DTYPE_BF16 ? 2 : 4;
  if (overlap(o, N * dv * 4, q, N * dk * es) || overlap(o, N * dv * 4, k, N * dk * es) ||
      overlap(o, N * dv * 4, v, N * dv * es))
    return GDN_ERR_INVALID_ARG;
  int sms = 0, cc = 0;
  rc = device_info(&sms, &cc);
  if (rc != GDN_OK) return rc;
  if (cc != 100) return GDN_ERR_NO_DEVICE;
  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)dk);
  const cudaError_t e =
      use_tc ? launch_softmax_window(q, k, v, o, B, H, F, L, dk, dv, W, sc, opts->status, spin_ns(opts),
                                     (cudaStream_t)opts->stream)
             : launch_softmax_window_simt(q, k, v, o, B, H, F, L, dk, dv, W, sc, opts->in_dtype,
                                          (cudaStream_t)opts->stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// ---------------------------------------------------------------- host I/O
//
// gdn_frame_fwd_host streams the sequence through the device in groups of
// frames: while group g runs, the inputs of group g + 1 are copied in and the
// output of group g - 1 is copied out, on three streams.  The state passes
// from group to group through state_out / state_in in fp32.

namespace {

// Frames per group: about 16 groups, so the first copy in and the last copy
// out (the parts that cannot overlap) are short.
int host_group_frames(int F) { return F <= 16 ? 1 : (F + 15) / 16; }

struct HostLayout {
  int Fg;                          // frames per group (the last group may have fewer)
  size_t slot;                     // bytes of one staging slot
  size_t q, k, v, alpha, beta, o;  // offsets inside a slot
  size_t s_in, s_out, s_a, s_b;    // fp32 states: caller's in / out, the two group hand-off buffers
  size_t ws;                       // kernel workspace (sized for Fg frames)
  size_t ws_bytes, total;
};

HostLayout host_layout(const gdn_opts_t *opts, int B, int H, int F, int L, int dk, int dv) {
  const size_t esz = opts->in_dtype == GDN_DTYPE_F32 ? 4 : 2;
  HostLayout h;
  h.Fg = host_group_frames(F);
  const size_t BH = (size_t)B * H, Ng = (size_t)h.Fg * L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  h.q = take(BH * Ng * dk * esz);
  h.k = take(BH * Ng * dk * esz);
  h.v = take(BH * Ng * dv * esz);
  h.alpha = take(BH * h.Fg * 4);
  h.beta = take(BH * Ng * 4);
  h.o = take(BH * Ng * dv * 4);
  h.slot = off;
  off = 2 * h.slot;
  const size_t sb = BH * dk * dv * 4;
  h.s_in = take(sb);
  h.s_out = take(sb);
  h.s_a = take(sb);
  h.s_b = take(sb);
  h.ws_bytes = gdn_ws_bytes(pick_gdn_impl(opts, dk, dv), opts, B, H, h.Fg, L, dk, dv);
  h.ws = take(h.ws_bytes);
  h.total = off;
  return h;
}

// Streams and events of one host call, released on every path out.
struct HostStreams {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t ev[4][2] = {};  // per slot: inputs in, group computed, output out, (spare)
  bool ok = true;
  HostStreams() {
    ok = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) == cudaSuccess;
    for (auto &pair : ev)
      for (auto &e : pair) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
  }
  ~HostStreams() {
    for (auto &pair : ev)
      for (auto &e : pair)
        if (e) cudaEventDestroy(e);
    if (up) cudaStreamDestroy(up);
    if (down) cudaStreamDestroy(down);
  }
};

}  // namespace

extern "C" size_t gdn_workspace_bytes_host(int B, int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts || check_sizes(B, H, F, L, dk, dv) != GDN_OK) return 0;
  return host_layout(opts, B, H, F, L, dk, dv).total;
}

extern "C" int gdn_frame_fwd_host(const void *q, const void *k, const void *v, const float *alpha,
                                  const float *beta, const float *state_in, float *state_out, float *o, int B,
                                  int H, int F, int L, int dk, int dv, const gdn_opts_t *opts) {
  if (!opts || !q || !k || !v || !alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
  if (opts->in_dtype != GDN_DTYPE_F32 && opts->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, F, L, dk, dv);
  if (rc != GDN_OK) return rc;
  const HostLayout h = host_layout(opts, B, H, F, L, dk, dv);
  if (!opts->workspace || opts->workspace_bytes < h.total) return GDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(opts->workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
  char *base = (char *)opts->workspace;
  cudaStream_t st = (cudaStream_t)opts->stream;
  const size_t esz = opts->in_dtype == GDN_DTYPE_F32 ? 4 : 2;
  const size_t N = (size_t)F * L, BH = (size_t)B * H;
  const size_t sbytes = BH * dk * dv * 4;
  HostStreams hs;
  if (!hs.ok) return GDN_ERR_CUDA;
  // the up and down streams start after whatever the caller queued on opts->stream
  if (cudaEventRecord(hs.ev[3][0], st) != cudaSuccess || cudaStreamWaitEvent(hs.up, hs.ev[3][0], 0) != cudaSuccess ||
      cudaStreamWaitEvent(hs.down, hs.ev[3][0], 0) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (state_in && cudaMemcpyAsync(base + h.s_in, state_in, sbytes, cudaMemcpyHostToDevice, hs.up) != cudaSuccess)
    return GDN_ERR_CUDA;
  const int G = (F + h.Fg - 1) / h.Fg;
  gdn_opts_t inner = *opts;
  inner.workspace = base + h.ws;
  inner.workspace_bytes = h.ws_bytes;
  for (int gi = 0; gi < G; ++gi) {
    const int f0 = gi * h.Fg, Fn = F - f0 < h.Fg ? F - f0 : h.Fg;
    const int sl = gi & 1;
    char *slot = base + (size_t)sl * h.slot;
    const size_t t0 = (size_t)f0 * L, nt = (size_t)Fn * L;
    cudaEvent_t in_done = hs.ev[sl][0], computed = hs.ev[sl][1], out_done = hs.ev[2][sl];
    // inputs of group gi (the slot's previous group must have been computed)
    if (gi >= 2 && cudaStreamWaitEvent(hs.up, computed, 0) != cudaSuccess) return GDN_ERR_CUDA;
    struct Cp2 { void *dst; const void *src; size_t row, pitch; };
    const Cp2 ins[] = {
        {slot + h.q, (const char *)q + t0 * dk * esz, nt * dk * esz, N * dk * esz},
        {slot + h.k, (const char *)k + t0 * dk * esz, nt * dk * esz, N * dk * esz},
        {slot + h.v, (const char *)v + t0 * dv * esz, nt * dv * esz, N * dv * esz},
        {slot + h.alpha, (const char *)alpha + (size_t)f0 * 4, (size_t)Fn * 4, (size_t)F * 4},
        {slot + h.beta, (const char *)beta + t0 * 4, nt * 4, N * 4}};
    for (const Cp2 &c : ins)
      if (cudaMemcpy2DAsync(c.dst, c.row, c.src, c.pitch, c.row, BH, cudaMemcpyHostToDevice, hs.up) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaEventRecord(in_done, hs.up) != cudaSuccess) return GDN_ERR_CUDA;
    // the group on the caller's stream, once its inputs are in and the slot's previous
    // output has been copied out
    if (cudaStreamWaitEvent(st, in_done, 0) != cudaSuccess) return GDN_ERR_CUDA;
    if (gi >= 2 && cudaStreamWaitEvent(st, out_done, 0) != cudaSuccess) return GDN_ERR_CUDA;
    const float *sin = gi == 0 ? (state_in ? (const float *)(base + h.s_in) : nullptr)
                               : (const float *)(base + ((gi - 1) & 1 ? h.s_b : h.s_a));
    float *sout = gi == G - 1 ? (state_out ? (float *)(base + h.s_out) : nullptr)
                              : (float *)(base + (gi & 1 ? h.s_b : h.s_a));
    inner.rope_frame_offset = opts->rope_frame_offset + f0;  // the group's first frame in the sequence
    rc = gdn_frame_fwd(slot + h.q, slot + h.k, slot + h.v, (const float *)(slot + h.alpha),
                       (const float *)(slot + h.beta), sin, sout, (float *)(slot + h.o), B, H, Fn, L, dk, dv,
                       &inner);
    if (rc != GDN_OK) return rc;
    if (cudaEventRecord(computed, st) != cudaSuccess) return GDN_ERR_CUDA;
    // output of group gi
    if (cudaStreamWaitEvent(hs.down, computed, 0) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMemcpy2DAsync((char *)o + t0 * dv * 4, N * dv * 4, slot + h.o, nt * dv * 4, nt * dv * 4, BH,
                          cudaMemcpyDeviceToHost, hs.down) != cudaSuccess)
      return GDN_ERR_CUDA;
    if (cudaEventRecord(out_done, hs.down) != cudaSuccess) return GDN_ERR_CUDA;
  }
  if (state_out &&
      cudaMemcpyAsync(state_out, base + h.s_out, sbytes, cudaMemcpyDeviceToHost, hs.down) != cudaSuccess)
    return GDN_ERR_CUDA;
  // the caller's stream waits for the last copy out, then the call returns
  if (cudaEventRecord(hs.ev[3][1], hs.down) != cudaSuccess || cudaStreamWaitEvent(st, hs.ev[3][1], 0) != cudaSuccess)
    return GDN_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
