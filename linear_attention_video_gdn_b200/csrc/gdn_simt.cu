// CUDA-core (SIMT) kernels of the two frame recurrences, fp32 arithmetic.
//
//  * gdn_seq_kernel: the per-token Gated DeltaNet recurrence exactly as
//    defined, one CTA per head, one thread per d_v column of the state
//    (column j of S depends only on column j of v and S0).  Simple and
//    sequential over all F*L tokens: the correctness baseline.
//  * gdn_frame_simt_kernel: the same recurrence reorganised around the frame
//    map (S_f = alpha_f A_f S_{f-1} + B_f, A_f the ordered product of the
//    frame's (I - beta khat khat^T) factors, B_f the frame's update from a
//    zero state).  Frames are independent work units taken from a ticket
//    counter; only the d x d chain step waits on the previous frame.
//  * relu_frame_simt_kernel: block-causal ReLU linear attention with the
//    same ticketed frame chain (additive block state and normaliser).
//
// Frame-wise Gated DeltaNet: SANA-WM GeekNews summary, "Core design and
// generation pipeline"; block KV cache: SANA-Video ICLR 2026 oral talk,
// block KV cache passage.
#include "common.cuh"

namespace gdn {

constexpr int kTile = 16;  // tokens staged in shared memory per step

// ----------------------------------------------------------------------------
// gdn_seq_kernel<DK, T>: grid = B*H, block = round_up(dv, 32) <= 128.
// ----------------------------------------------------------------------------
template <int DK, typename T>
__global__ void __launch_bounds__(128) gdn_seq_kernel(GdnParams p) {
  const int bh = blockIdx.x;
  const int j = threadIdx.x;
  const int nthr = blockDim.x;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const long N = (long)F * L;
  const T *q = (const T *)p.q + (long)bh * N * dk;
  const T *k = (const T *)p.k + (long)bh * N * dk;
  const T *v = (const T *)p.v + (long)bh * N * dv;
  const float *beta = p.beta + (long)bh * N;
  const float *alpha = p.alpha + (long)bh * F;

  __shared__ float sk[kTile][DK];
  __shared__ float sv[kTile][128];
  __shared__ float sb[kTile];
  __shared__ float sinv[kTile];

  float S[DK];
#pragma unroll
  for (int i = 0; i < DK; ++i)
    S[i] = (p.state_in && j < dv && i < dk) ? p.state_in[(long)bh * dk * dv + (long)i * dv + j] : 0.f;

  for (int f = 0; f < F; ++f) {
    const float a = alpha[f];
    const float al = p.gates_are_logits ? gate_alpha(a) : a;
#pragma unroll
    for (int i = 0; i < DK; ++i) S[i] *= al;
    const long t_end = (long)(f + 1) * L;
    for (long t0 = (long)f * L; t0 < t_end; t0 += kTile) {
      const int nt = (int)min((long)kTile, t_end - t0);
      __syncthreads();
      for (int e = j; e < kTile * DK; e += nthr) {
        const int tt = e / DK, i = e % DK;
        sk[tt][i] = (tt < nt && i < dk) ? (p.rope_on ? rope_elem(k + (t0 + tt) * dk, i, f, (int)(t0 + tt - (long)f * L), p)
                                                      : to_f32(k[(t0 + tt) * dk + i]))
                                        : 0.f;
      }
      for (int e = j; e < kTile * 128; e += nthr) {
        const int tt = e / 128, c = e % 128;
        sv[tt][c] = (tt < nt && c < dv) ? to_f32(v[(t0 + tt) * dv + c]) : 0.f;
      }
      if (j < kTile) {
        const float b = j < nt ? beta[t0 + j] : 0.f;
        sb[j] = p.gates_are_logits ? gate_beta(b) : b;
      }
      __syncthreads();
      if (j < kTile) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < DK; ++i) ss += sk[j][i] * sk[j][i];
        sinv[j] = 1.0f / fmaxf(sqrtf(ss), kKeyNormEps);
      }
      __syncthreads();
      for (int tt = 0; tt < nt; ++tt) {
        const float inv = sinv[tt];
        float pr = 0.f;
#pragma unroll
        for (int i = 0; i < DK; ++i) pr += S[i] * sk[tt][i];
        const float r = pr * inv - sv[tt][j];
        const float c = sb[tt] * r * inv;
#pragma unroll
        for (int i = 0; i < DK; ++i) S[i] -= c * sk[tt][i];
      }
    }
    // read-out with the end-of-frame state
    for (long t0 = (long)f * L; t0 < t_end; t0 += kTile) {
      const int nt = (int)min((long)kTile, t_end - t0);
      __syncthreads();
      for (int e = j; e < kTile * DK; e += nthr) {
        const int tt = e / DK, i = e % DK;
        sk[tt][i] = (tt < nt && i < dk) ? (p.rope_on ? rope_elem(q + (t0 + tt) * dk, i, f, (int)(t0 + tt - (long)f * L), p)
                                                      : to_f32(q[(t0 + tt) * dk + i]))
                                        : 0.f;
      }
      __syncthreads();
      if (j < dv) {
        for (int tt = 0; tt < nt; ++tt) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < DK; ++i) acc += S[i] * sk[tt][i];
          p.o[((long)bh * N + t0 + tt) * dv + j] = acc;
        }
      }
    }
  }
  if (p.state_out && j < dv) {
#pragma unroll
    for (int i = 0; i < DK; ++i)
      if (i < dk) p.state_out[(long)bh * dk * dv + (long)i * dv + j] = S[i];
  }
}

// ----------------------------------------------------------------------------
// gdn_frame_simt_kernel<DK, T>: persistent, block = 256 threads.
// Thread c < dk owns column c of A_f; thread dk + j owns column j of B_f.
// ----------------------------------------------------------------------------
template <int DK>
struct FrameSimtSmem {
  float sk[kTile][DK];
  float sv[kTile][128];
  float sb[kTile];
  float sinv[kTile];
  float sAt[DK][DK];    // sAt[l][i] = A_f[i][l]
  float sS[DK][128];    // S_{f-1}[l][j]
  int ticket;
  int abort;
};

template <int DK, typename T>
__global__ void __launch_bounds__(256) gdn_frame_simt_kernel(GdnParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FrameSimtSmem<DK> &sm = *reinterpret_cast<FrameSimtSmem<DK> *>(smem_raw);
  const int c = threadIdx.x;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const int BH = p.B * p.H;
  const long N = (long)F * L;
  const long units = (long)BH * F;
  const int ncol = dk + dv;
  const bool is_b = c >= dk && c < ncol;
  const int j = c - dk;

  for (;;) {
    if (c == 0) {
      sm.ticket = atomicAdd(p.ws.counter, 1);
      sm.abort = 0;
    }
    __syncthreads();
    const long ticket = sm.ticket;
    if (ticket >= units) break;
    const int f = (int)(ticket / BH);
    const int bh = (int)(ticket % BH);
    const T *q = (const T *)p.q + (long)bh * N * dk;
    const T *k = (const T *)p.k + (long)bh * N * dk;
    const T *v = (const T *)p.v + (long)bh * N * dv;
    const float *beta = p.beta + (long)bh * N;

    // Y = [A | B], A starts at I, B at 0; target 0 for A columns, v for B.
    float y[DK];
#pragma unroll
    for (int i = 0; i < DK; ++i) y[i] = (c < dk && i == c) ? 1.f : 0.f;

    const long t_beg = (long)f * L, t_end = t_beg + L;
    for (long t0 = t_beg; t0 < t_end; t0 += kTile) {
      const int nt = (int)min((long)kTile, t_end - t0);
      __syncthreads();
      for (int e = c; e < kTile * DK; e += 256) {
        const int tt = e / DK, i = e % DK;
        sm.sk[tt][i] = (tt < nt && i < dk) ? (p.rope_on ? rope_elem(k + (t0 + tt) * dk, i, f, (int)(t0 + tt - t_beg), p)
                                                         : to_f32(k[(t0 + tt) * dk + i]))
                                           : 0.f;
      }
      for (int e = c; e < kTile * 128; e += 256) {
        const int tt = e / 128, x = e % 128;
        sm.sv[tt][x] = (tt < nt && x < dv) ? to_f32(v[(t0 + tt) * dv + x]) : 0.f;
      }
      if (c < kTile) {
        const float b = c < nt ? beta[t0 + c] : 0.f;
        sm.sb[c] = p.gates_are_logits ? gate_beta(b) : b;
      }
      __syncthreads();
      if (c < kTile) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < DK; ++i) ss += sm.sk[c][i] * sm.sk[c][i];
        sm.sinv[c] = 1.0f / fmaxf(sqrtf(ss), kKeyNormEps);
      }
      __syncthreads();
      if (c < ncol) {
        for (int tt = 0; tt < nt; ++tt) {
          const float inv = sm.sinv[tt];
          float pr = 0.f;
#pragma unroll
          for (int i = 0; i < DK; ++i) pr += y[i] * sm.sk[tt][i];
          const float target = is_b ? sm.sv[tt][j] : 0.f;
          const float cc = sm.sb[tt] * (pr * inv - target) * inv;
#pragma unroll
          for (int i = 0; i < DK; ++i) y[i] -= cc * sm.sk[tt][i];
        }
      }
    }

    // ---- chain step: S_f = alpha_f A_f S_{f-1} + B_f ----
    __syncthreads();
    if (c < dk) {
#pragma unroll
      for (int i = 0; i < DK; ++i) sm.sAt[c][i] = y[i];
    }
    for (int e = c; e < DK * dk; e += 256) {  // zero-pad unused rows of sAt
      const int l = e / DK, i = e % DK;
      if (i >= dk) sm.sAt[l][i] = 0.f;
    }
    if (p.save_maps) {  // A_f^T rows for the backward (written by threads c < dk above)
      __syncthreads();
      float *mp = p.save_maps + ((long)bh * F + f) * (long)dk * dk;
      for (int e = c; e < dk * dk; e += 256) mp[e] = sm.sAt[e / dk][e % dk];
    }
    const float a = p.alpha[(long)bh * F + f];
    const float al = p.gates_are_logits ? gate_alpha(a) : a;
    bool have_prev = true;
    if (f > 0) {
      if (c == 0) {
        if (!wait_flag(p.ws.flags + (long)bh * F + (f - 1), 1, p.spin_limit_ns)) {
          latch_status(p.status, GDN_ERR_TIMEOUT);
          sm.abort = 1;
        }
      }
      __syncthreads();
      if (sm.abort) break;
      const float *prev = p.ws.states + ((long)bh * F + (f - 1)) * (long)dk * dv;  // St[j][l]
      for (int e = c; e < DK * 128; e += 256) {
        const int l = e / 128, x = e % 128;
        sm.sS[l][x] = (l < dk && x < dv) ? __ldcg(prev + (long)x * dk + l) : 0.f;
      }
    } else if (p.state_in) {
      const float *s0 = p.state_in + (long)bh * dk * dv;
      for (int e = c; e < DK * 128; e += 256) {
        const int l = e / 128, x = e % 128;
        sm.sS[l][x] = (l < dk && x < dv) ? s0[(long)l * dv + x] : 0.f;
      }
    } else {
      have_prev = false;
    }
    __syncthreads();
    if (is_b && have_prev) {
      for (int l = 0; l < dk; ++l) {
        const float s = al * sm.sS[l][j];
#pragma unroll
        for (int i = 0; i < DK; ++i) y[i] += sm.sAt[l][i] * s;
      }
    }
    // publish S_f^T (row j = column j of S_f)
    float *cur = p.ws.states + ((long)bh * F + f) * (long)dk * dv;
    if (is_b) {
#pragma unroll
      for (int i = 0; i < DK; ++i)
        if (i < dk) cur[(long)j * dk + i] = y[i];
      if (f == F - 1 && p.state_out) {
#pragma unroll
        for (int i = 0; i < DK; ++i)
          if (i < dk) p.state_out[(long)bh * dk * dv + (long)i * dv + j] = y[i];
      }
      if (p.save_states) {
        float *sp = p.save_states + ((long)bh * F + f) * (long)dk * dv;
#pragma unroll
        for (int i = 0; i < DK; ++i)
          if (i < dk) sp[(long)i * dv + j] = y[i];
      }
    }
    __syncthreads();
    if (c == 0 && ticket != p.withhold) {
      __threadfence();
      st_release(p.ws.flags + (long)bh * F + f, 1);
    }

    // ---- read-out: o_t = S_f^T q_t for the frame's tokens (none for the backward's recompute) ----
    for (long t0 = t_beg; p.o && t0 < t_end; t0 += kTile) {
      const int nt = (int)min((long)kTile, t_end - t0);
      __syncthreads();
      for (int e = c; e < kTile * DK; e += 256) {
        const int tt = e / DK, i = e % DK;
        sm.sk[tt][i] = (tt < nt && i < dk) ? (p.rope_on ? rope_elem(q + (t0 + tt) * dk, i, f, (int)(t0 + tt - t_beg), p)
                                                         : to_f32(q[(t0 + tt) * dk + i]))
                                           : 0.f;
      }
      __syncthreads();
      if (is_b) {
        for (int tt = 0; tt < nt; ++tt) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < DK; ++i) acc += y[i] * sm.sk[tt][i];
          p.o[((long)bh * N + t0 + tt) * dv + j] = acc;
        }
      }
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// relu_frame_simt_kernel<DK, T>: persistent, block = 256 threads.
// Thread j < dv owns column j of the frame's contribution relu(K)^T V;
// thread dv owns the normaliser contribution sum relu(k).
// Published per unit: St[j][i] for j < dv, and z at row dv.
// ----------------------------------------------------------------------------
template <int DK>
struct ReluSimtSmem {
  float sk[kTile][DK];
  float sv[kTile][128];
  float sden[kTile];
  int ticket;
  int abort;
};

template <int DK, typename T>
__global__ void __launch_bounds__(256) relu_frame_simt_kernel(ReluParams p) {
  __shared__ ReluSimtSmem<DK> sm;
  const int c = threadIdx.x;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const int BH = p.B * p.H;
  const long N = (long)F * L;
  const long units = (long)BH * F;
  const bool owner = c <= dv;  // c == dv: normaliser
  const long slot = (long)(dv + 1) * dk;

  for (;;) {
    if (c == 0) {
      sm.ticket = atomicAdd(p.ws.counter, 1);
      sm.abort = 0;
    }
    __syncthreads();
    const long ticket = sm.ticket;
    if (ticket >= units) break;
    const int f = (int)(ticket / BH);
    const int bh = (int)(ticket % BH);
    const T *q = (const T *)p.q + (long)bh * N * dk;
    const T *k = (const T *)p.k + (long)bh * N * dk;
    const T *v = (const T *)p.v + (long)bh * N * dv;

    float s[DK];
#pragma unroll
    for (int i = 0; i < DK; ++i) s[i] = 0.f;
    const long t_beg = (long)f * L, t_end = t_beg + L;
    for (long t0 = t_beg; t0 < t_end; t0 += kTile) {
      const int nt = (int)min((long)kTile, t_end - t0);
      __syncthreads();
      for (int e = c; e < kTile * DK; e += 256) {
        const int tt = e / DK, i = e % DK;
        sm.sk[tt][i] = (tt < nt && i < dk) ? fmaxf(to_f32(k[(t0 + tt) * dk + i]), 0.f) : 0.f;
      }
      for (int e = c; e < kTile * 128; e += 256) {
        const int tt = e / 128, x = e % 128;
        sm.sv[tt][x] = (tt < nt && x < dv) ? to_f32(v[(t0 + tt) * dv + x]) : 0.f;
      }
      __syncthreads();
      if (owner) {
        for (int tt = 0; tt < nt; ++tt) {
          const float w = c < dv ? sm.sv[tt][c] : 1.0f;
#pragma unroll
          for (int i = 0; i < DK; ++i) s[i] += sm.sk[tt][i] * w;
        }
      }
    }
    // chain: S_f = S_{f-1} + dS_f (same for z)
    if (f > 0) {
      if (c == 0) {
        if (!wait_flag(p.ws.flags + (long)bh * F + (f - 1), 1, p.spin_limit_ns)) {
          latch_status(p.status, GDN_ERR_TIMEOUT);
          sm.abort = 1;
        }
      }
      __syncthreads();
      if (sm.abort) break;
      if (owner) {
        const float *prev = p.ws.states + ((long)bh * F + (f - 1)) * slot + (long)c * dk;
#pragma unroll
        for (int i = 0; i < DK; ++i)
          if (i < dk) s[i] += __ldcg(prev + i);
      }
    } else if (owner) {
      if (c < dv && p.kv_in) {
#pragma unroll
        for (int i = 0; i < DK; ++i)
          if (i < dk) s[i] += p.kv_in[(long)bh * dk * dv + (long)i * dv + c];
      }
      if (c == dv && p.z_in) {
#pragma unroll
        for (int i = 0; i < DK; ++i)
          if (i < dk) s[i] += p.z_in[(long)bh * dk + i];
      }
    }
    if (owner) {
      float *cur = p.ws.states + ((long)bh * F + f) * slot + (long)c * dk;
#pragma unroll
      for (int i = 0; i < DK; ++i)
        if (i < dk) cur[i] = s[i];
      if (f == F - 1) {
        if (c < dv && p.kv_out) {
#pragma unroll
          for (int i = 0; i < DK; ++i)
            if (i < dk) p.kv_out[(long)bh * dk * dv + (long)i * dv + c] = s[i];
        }
        if (c == dv && p.z_out) {
#pragma unroll
          for (int i = 0; i < DK; ++i)
            if (i < dk) p.z_out[(long)bh * dk + i] = s[i];
        }
      }
    }
    __syncthreads();
    if (c == 0 && ticket != p.withhold) {
      __threadfence();
      st_release(p.ws.flags + (long)bh * F + f, 1);
    }
    // read-out
    for (long t0 = t_beg; t0 < t_end; t0 += kTile) {
      const int nt = (int)min((long)kTile, t_end - t0);
      __syncthreads();
      for (int e = c; e < kTile * DK; e += 256) {
        const int tt = e / DK, i = e % DK;
        sm.sk[tt][i] = (tt < nt && i < dk) ? fmaxf(to_f32(q[(t0 + tt) * dk + i]), 0.f) : 0.f;
      }
      __syncthreads();
      if (c == dv) {
        for (int tt = 0; tt < nt; ++tt) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < DK; ++i) acc += s[i] * sm.sk[tt][i];
          sm.sden[tt] = acc + p.eps;
        }
      }
      __syncthreads();
      if (c < dv) {
        for (int tt = 0; tt < nt; ++tt) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < DK; ++i) acc += s[i] * sm.sk[tt][i];
          p.o[((long)bh * N + t0 + tt) * dv + c] = acc / sm.sden[tt];
        }
      }
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// host launchers
// ----------------------------------------------------------------------------
template <int DK, typename T>
static cudaError_t launch_seq_t(const GdnParams &p, cudaStream_t st) {
  const int threads = ((p.dv + 31) / 32) * 32;
  gdn_seq_kernel<DK, T><<<p.B * p.H, threads, 0, st>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_seq(const GdnParams &p, cudaStream_t st) {
  if (p.dk <= 32) return launch_seq_t<32, T>(p, st);
  if (p.dk <= 64) return launch_seq_t<64, T>(p, st);
  return launch_seq_t<128, T>(p, st);
}

cudaError_t launch_gdn_seq(const GdnParams &p, int in_dtype, cudaStream_t st) {
  return in_dtype == GDN_DTYPE_F32 ? launch_seq<float>(p, st) : launch_seq<__nv_bfloat16>(p, st);
}

template <int DK, typename T>
static cudaError_t launch_frame_simt_t(const GdnParams &p, int grid, cudaStream_t st) {
  const size_t smem = sizeof(FrameSimtSmem<DK>);
  cudaError_t e = cudaFuncSetAttribute(gdn_frame_simt_kernel<DK, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  gdn_frame_simt_kernel<DK, T><<<grid, 256, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_frame_simt(const GdnParams &p, int grid, cudaStream_t st) {
  if (p.dk <= 32) return launch_frame_simt_t<32, T>(p, grid, st);
  if (p.dk <= 64) return launch_frame_simt_t<64, T>(p, grid, st);
  return launch_frame_simt_t<128, T>(p, grid, st);
}

cudaError_t launch_gdn_frame_simt(const GdnParams &p, int in_dtype, int grid, cudaStream_t st) {
  return in_dtype == GDN_DTYPE_F32 ? launch_frame_simt<float>(p, grid, st)
                                   : launch_frame_simt<__nv_bfloat16>(p, grid, st);
}

template <int DK, typename T>
static cudaError_t launch_relu_simt_t(const ReluParams &p, int grid, cudaStream_t st) {
  relu_frame_simt_kernel<DK, T><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_relu_simt(const ReluParams &p, int grid, cudaStream_t st) {
  if (p.dk <= 32) return launch_relu_simt_t<32, T>(p, grid, st);
  if (p.dk <= 64) return launch_relu_simt_t<64, T>(p, grid, st);
  return launch_relu_simt_t<128, T>(p, grid, st);
}

cudaError_t launch_relu_frame_simt(const ReluParams &p, int in_dtype, int grid, cudaStream_t st) {
  return in_dtype == GDN_DTYPE_F32 ? launch_relu_simt<float>(p, grid, st)
                                   : launch_relu_simt<__nv_bfloat16>(p, grid, st);
}

}  // namespace gdn
