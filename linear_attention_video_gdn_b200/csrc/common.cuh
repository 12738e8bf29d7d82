// Shared device-side helpers: workspace layout, bounded waits, element loads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn_b200.h"

namespace gdn {

// Key normalisation floor: khat = k / max(||k||, kKeyNormEps).
constexpr float kKeyNormEps = 1e-6f;

// Workspace of the frame-chain kernels:
//   [0, 256)                 : int counters (ticket counter at [0])
//   [256, 256 + 4*units)     : int flag per (b, h, f) unit: 1 once its state is published
//   then, 256-byte aligned   : published state per unit, in the layout of the kernel that runs:
//                              the SIMT frame kernel fp32 St[j][i] (dv rows of dk), the tcgen05
//                              kernel fp16 rows S^T[j][l] (half the bytes; sized in floats)
struct Workspace {
  int *counter;
  int *flags;
  float *states;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline size_t chain_workspace_bytes(long units, long state_elems) {
  size_t b = 256;
  b += align_up(sizeof(int) * (size_t)units, 256);
  b += align_up(sizeof(float) * (size_t)units * (size_t)state_elems, 256);
  return b;
}

inline Workspace chain_workspace(void *base, long units) {
  char *p = (char *)base;
  Workspace w;
  w.counter = (int *)p;
  w.flags = (int *)(p + 256);
  w.states = (float *)(p + 256 + align_up(sizeof(int) * (size_t)units, 256));
  return w;
}

// Bytes of the zero-initialised head of the workspace (counter + flags).
inline size_t chain_workspace_zero_bytes(long units) { return 256 + align_up(sizeof(int) * (size_t)units, 256); }

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(int *p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Latch the first device-side error code into *status (if given).
__device__ __forceinline__ void latch_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Spin (with back-off) until *flag >= target or limit_ns elapses.  Returns
// false on timeout.  Called by one thread.
__device__ __forceinline__ bool wait_flag(const int *flag, int target, unsigned long long limit_ns) {
  if (ld_acquire(flag) >= target) return true;
  const unsigned long long t0 = global_timer_ns();
  unsigned ns = 32;
  while (true) {
    __nanosleep(ns);
    if (ld_acquire(flag) >= target) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
    if (ns < 256) ns *= 2;
  }
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Gate activations (fp32): alpha = exp(-softplus(a)) = 1 / (1 + e^a); beta = sigmoid(b).
__device__ __forceinline__ float gate_alpha(float a) { return 1.0f / (1.0f + expf(a)); }
__device__ __forceinline__ float gate_beta(float b) { return 1.0f / (1.0f + expf(-b)); }

struct GdnParams {
  const void *q, *k, *v;
  const float *alpha, *beta;
  const float *state_in;
  float *state_out;
  float *o;
  int B, H, F, L, dk, dv;
  int gates_are_logits;
  int *status;
  unsigned long long spin_limit_ns;
  long withhold;  // unit that never publishes (testing), -1 = none
  Workspace ws;   // flags and published states per segment unit ((b, h, f), then segment)
  int segs;       // chunk segments per frame (tcgen05 kernel; 1 elsewhere)
  uint32_t *ro_states;  // segs > 1: per (b, h, f) the end-of-frame S^T rows as bf16 high/low pairs
  // 3D rotary position embedding of q and k (rope_on != 0): cos/sin of the angle of every
  // (axis position, pair) as float2, time part [F][dt/2], then height [L/gw][dh/2], then width [gw][dh/2]
  const float2 *rope_tab;
  int rope_on, rope_gw, rope_dt, rope_dh;
  // backward recompute (non-null together, one unit per frame, no position embedding):
  // every frame's map A_f^T [b, h, f][r][i] = A_f[i][r] and end state S_f [b, h, f][l][j], fp32
  float *save_maps;
  float *save_states;
};

// Backward of the Gated DeltaNet (gdn_bwd.cu).  Buffers are [b, h] then as named.
struct BwdParams {
  const void *q, *k, *v;        // [N][dk], [N][dk], [N][dv] (bf16 or fp32)
  const float *alpha, *beta;    // [F], [N] (logits when gates_are_logits)
  const float *state_in;        // [dk][dv] or null (zero)
  const float *d_o;             // [N][dv]
  const float *dstate_out;      // [dk][dv] or null (zero)
  const float *maps;            // [F][dk][dk]: A_f^T (recomputed forward)
  const float *states;          // [F][dk][dv]: S_f, the end state of every frame
  float *gbuf;                  // [F][dk][dv]: G_f = dL/dS_f (adjoint chain -> frame kernel)
  float *dal_part;              // [F][ceil(dv / 16)]: dalpha_f per column group
  float *linv_buf;              // [F][chunks][48][48]: each chunk's Linv (bf16-input frame kernel)
  float *rbuf;                  // [N][dv]: each token's residual, or null (then kept in dk_out's rows, dv <= dk)
  float *dq, *dk_out, *dv_out;  // [N][dk], [N][dk], [N][dv]; dv_out is also scratch
  float *dalpha, *dbeta;        // [F], [N]
  float *dstate_in;             // [dk][dv] or null
  int B, H, F, L, dk, dv;
  int gates_are_logits;
};

// Rotated element i of the d_k-vector x (i's pair is i ^ 1) of the token at
// index tf of frame f, with the table of the 3D rotary position embedding.
template <typename T>
__device__ __forceinline__ float rope_elem(const T *x, int i, int f, int tf, const GdnParams &p) {
  const int pr = i & ~1;
  int a_off, idx;
  if (pr < p.rope_dt) {
    a_off = f * (p.rope_dt / 2);
    idx = pr / 2;
  } else if (pr < p.rope_dt + p.rope_dh) {
    a_off = p.F * (p.rope_dt / 2) + (tf / p.rope_gw) * (p.rope_dh / 2);
    idx = (pr - p.rope_dt) / 2;
  } else {
    a_off = p.F * (p.rope_dt / 2) + (p.L / p.rope_gw) * (p.rope_dh / 2) + (tf % p.rope_gw) * (p.rope_dh / 2);
    idx = (pr - p.rope_dt - p.rope_dh) / 2;
  }
  const float2 cs = __ldg(p.rope_tab + a_off + idx);
  const float x0 = to_f32(x[pr]), x1 = to_f32(x[pr + 1]);
  return (i & 1) ? fmaf(x0, cs.y, x1 * cs.x) : fmaf(x0, cs.x, -x1 * cs.y);
}

// The pair (dd, dd + 1) (dd even) of a token at index tf of frame f, rotated.
__device__ __forceinline__ float2 rope_pair(float2 x, int dd, int f, int tf, const GdnParams &p) {
  int a_off, idx;
  if (dd < p.rope_dt) {
    a_off = f * (p.rope_dt / 2);
    idx = dd / 2;
  } else if (dd < p.rope_dt + p.rope_dh) {
    a_off = p.F * (p.rope_dt / 2) + (tf / p.rope_gw) * (p.rope_dh / 2);
    idx = (dd - p.rope_dt) / 2;
  } else {
    a_off = p.F * (p.rope_dt / 2) + (p.L / p.rope_gw) * (p.rope_dh / 2) + (tf % p.rope_gw) * (p.rope_dh / 2);
    idx = (dd - p.rope_dt - p.rope_dh) / 2;
  }
  const float2 cs = __ldg(p.rope_tab + a_off + idx);
  return make_float2(fmaf(x.x, cs.x, -x.y * cs.y), fmaf(x.x, cs.y, x.y * cs.x));
}

// Entries of the RoPE table for these sizes (float2 each).
inline size_t rope_table_entries(int F, int L, int gw, int dk) {
  const int dh = 2 * (dk / 6), dt = dk - 2 * dh;
  return (size_t)F * (dt / 2) + (size_t)(L / gw) * (dh / 2) + (size_t)gw * (dh / 2);
}

struct ReluParams {
  const void *q, *k, *v;
  const float *kv_in, *z_in;
  float *kv_out, *z_out;
  float *o;
  int B, H, F, L, dk, dv;
  float eps;
  int *status;
  unsigned long long spin_limit_ns;
  long withhold;  // unit that never publishes (testing), -1 = none
  Workspace ws;
};

}  // namespace gdn
