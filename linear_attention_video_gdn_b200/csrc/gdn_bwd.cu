// Backward of the frame-wise Gated DeltaNet (no position embedding).
//
// Source of the method: SANA-WM GeekNews summary, "Core design and generation
// pipeline" (frame-wise Gated DeltaNet; the model is trained, on 64 H100s).
// Forward, per head: S <- alpha_f S at each frame start, then per token
// S <- S + beta khat (v - S^T khat)^T, khat = k / max(||k||, eps); every token
// of frame f reads o = S_f^T q with S_f the state after the frame.
//
// Given dL/do and dL/dS_out the gradients are taken in three passes:
//  1. (gdn_tc / gdn_frame_simt, recompute) every frame's map A_f (the ordered
//     product of the frame's I - beta khat khat^T factors, saved as A_f^T) and
//     end state S_f, fp32.
//  2. gdn_bwd_adjoint_kernel: the frame chain in reverse.  With
//     G_f = dL/dS_f (end of frame f),
//        G_{F-1} = dS_out + Q_{F-1}^T dO_{F-1},
//        G_{f-1} = Q_{f-1}^T dO_{f-1} + alpha_f A_f^T G_f,
//     dalpha_f = <A_f^T G_f, S_{f-1}>, dS_in = alpha_0 A_0^T G_0.  Columns j
//     of G are independent: one CTA per (head, 16 columns), serial over
//     frames.
//  3. gdn_bwd_frame_kernel: one CTA per frame, from S^(0) = alpha_f S_{f-1}
//     and H = G_f, in chunks of C = 48 tokens (UT form; Linv = (I + N)^-1,
//     N = strict_lower(diag(beta) Khat Khat^T)):
//       forward sweep: E = V - Khat S, U = Linv diag(beta) E, S += Khat^T U
//                      (U kept for the reverse sweep); then dq = dO S_f^T;
//       reverse sweep: S -= Khat^T U (the chunk's start state again),
//                      E = V - Khat S, R = E - strict_lower(Khat Khat^T) U
//                      (row t: the token's residual v_t - S_{t-1}^T khat_t),
//                      Gm = Linv^T Khat H (row t: g_t = H_t^T khat_t with H_t
//                      the gradient after token t),
//                      dv = diag(beta) Gm, dbeta_t = g_t . R_t,
//                      dkhat = diag(beta) (R H^T - Gm S^T - M Khat), where
//                        M[t][s] = beta_s R_t . g_s (s > t), g_t . u_s (s < t)
//                      (the in-chunk terms of H_t r_t and S_{t-1} g_t),
//                      H -= Khat^T diag(beta) Gm;
//     dk from dkhat through the normalisation.
// Products run on CUDA cores in fp32 (register tiles over shared memory).
#include "launch.h"

namespace gdn {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kC = 48;      // tokens per chunk (frame kernel)
constexpr int kLdC = kC + 1;
constexpr int kQt = 64;     // tokens per tile (adjoint kernel)

template <typename T>
__device__ __forceinline__ float ldf(const T *p) {
  return to_f32(*p);
}

// acc[i][j] += sum_{k < K} fa(ty + 16 i, k) * fb(k, tx + 16 j): the thread's
// rows and columns interleave with stride 16, so that a warp reads two rows
// of A (broadcast) and 16 consecutive columns of B per k, conflict-free for
// odd leading dimensions in either orientation.
template <int TM, int TN, class FA, class FB>
__device__ __forceinline__ void mm(float (&acc)[TM][TN], int K, int ty, int tx, FA fa, FB fb) {
#pragma unroll 2
  for (int k = 0; k < K; ++k) {
    float a[TM], b[TN];
#pragma unroll
    for (int i = 0; i < TM; ++i) a[i] = fa(ty + 16 * i, k);
#pragma unroll
    for (int j = 0; j < TN; ++j) b[j] = fb(k, tx + 16 * j);
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

template <int TM, int TN>
__device__ __forceinline__ void zero(float (&acc)[TM][TN]) {
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

// ---------------------------------------------------------------- pass 2
// Shared memory: A_f^T [DP][DP + 1], G [DP][17], q tile [kQt][DP + 1], dO tile [kQt][17].
template <int ND>
struct AdjSmem {
  static constexpr int DP = 16 * ND, LD = DP + 1;
  float a[DP * LD];
  float g[DP * 17];
  float q[kQt * LD];
  float d[kQt * 17];
  float red[kThreads / 32];
};

template <int ND, typename T>
__global__ void __launch_bounds__(kThreads) gdn_bwd_adjoint_kernel(BwdParams p) {
  using SM = AdjSmem<ND>;
  constexpr int LD = SM::LD;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SM &sm = *reinterpret_cast<SM *>(smem_raw);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const long N = (long)F * L;
  const int ncg = (dv + 15) / 16;
  const int bh = blockIdx.x / ncg, cg = blockIdx.x % ncg;
  const int j = cg * 16 + tx;  // this thread's column of G
  const bool jok = j < dv;
  const long SS = (long)dk * dv;
  const T *q = static_cast<const T *>(p.q) + (long)bh * N * dk;
  const float *d_o = p.d_o + (long)bh * N * dv;

  for (int e = tid; e < (int)(sizeof(SM) / 4); e += kThreads) reinterpret_cast<float *>(&sm)[e] = 0.f;
  float carry[ND];  // alpha_{f+1} A_{f+1}^T G_{f+1} (or dS_out), rows ty + 16 r
#pragma unroll
  for (int r = 0; r < ND; ++r) {
    const int i = ty + 16 * r;
    carry[r] = (p.dstate_out && jok && i < dk) ? p.dstate_out[(long)bh * SS + (long)i * dv + j] : 0.f;
  }
  __syncthreads();
  for (int f = F - 1; f >= 0; --f) {
    // A_f^T into shared memory
    const float *mp = p.maps + ((long)bh * F + f) * (long)dk * dk;
    for (int e = tid; e < dk * dk; e += kThreads) sm.a[(e / dk) * LD + e % dk] = __ldg(mp + e);
    // C = Q_f^T dO_f (columns of this CTA)
    float c[ND][1];
    zero(c);
    for (int t0 = 0; t0 < L; t0 += kQt) {
      const int nt = min(kQt, L - t0);
      const long base = (long)f * L + t0;
      for (int e = tid; e < nt * dk; e += kThreads) sm.q[(e / dk) * LD + e % dk] = ldf(q + base * dk + e);
      for (int e = tid; e < nt * 16; e += kThreads) {
        const int jj = cg * 16 + (e & 15);
        sm.d[(e >> 4) * 17 + (e & 15)] = jj < dv ? __ldg(d_o + (base + (e >> 4)) * dv + jj) : 0.f;
      }
      __syncthreads();
      mm(c, nt, ty, tx, [&](int m, int k) { return sm.q[k * LD + m]; }, [&](int k, int n) { return sm.d[k * 17 + n]; });
      __syncthreads();
    }
    // G_f = C + carry -> global (for the frame kernel) and shared memory
    float *gout = p.gbuf + ((long)bh * F + f) * SS;
#pragma unroll
    for (int r = 0; r < ND; ++r) {
      const int i = ty + 16 * r;
      const float gv = c[r][0] + carry[r];
      sm.g[i * 17 + tx] = gv;
      if (jok && i < dk) gout[(long)i * dv + j] = gv;
    }
    __syncthreads();
    // H0 = A_f^T G_f
    float h[ND][1];
    zero(h);
    mm(h, dk, ty, tx, [&](int m, int k) { return sm.a[m * LD + k]; }, [&](int k, int n) { return sm.g[k * 17 + n]; });
    // dalpha_f (this CTA's columns) = <H0, S_{f-1}>
    const float *sprev = f > 0 ? p.states + ((long)bh * F + f - 1) * SS
                               : (p.state_in ? p.state_in + (long)bh * SS : nullptr);
    float part = 0.f;
    if (sprev && jok) {
#pragma unroll
      for (int r = 0; r < ND; ++r) {
        const int i = ty + 16 * r;
        if (i < dk) part = fmaf(h[r][0], __ldg(sprev + (long)i * dv + j), part);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if ((tid & 31) == 0) sm.red[tid >> 5] = part;
    const float araw = p.alpha[(long)bh * F + f];
    const float al = p.gates_are_logits ? gate_alpha(araw) : araw;
#pragma unroll
    for (int r = 0; r < ND; ++r) carry[r] = al * h[r][0];
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) s += sm.red[w];
      p.dal_part[((long)bh * F + f) * ncg + cg] = s;
    }
  }
  if (p.dstate_in && jok) {
#pragma unroll
    for (int r = 0; r < ND; ++r) {
      const int i = ty + 16 * r;
      if (i < dk) p.dstate_in[(long)bh * SS + (long)i * dv + j] = carry[r];
    }
  }
}

// ---------------------------------------------------------------- pass 3
template <int ND>
struct FrameSmem {
  static constexpr int DP = 16 * ND, LD = DP + 1;
  float S[DP * LD];   // S[i][j]
  float H[DP * LD];   // H[i][j]
  float K[kC * LD];   // khat rows
  float E[kC * LD];   // v -> E -> R rows
  float U[kC * LD];   // U rows
  float G[kC * LD];   // Khat H -> Gm rows; dO rows for dq
  float M[kC * kLdC]; // Gram (upper, with diagonal) | Linv (strict lower); then the dkhat coupling M
  float T[3 * 16 * 17];  // inverse scratch
  float b[kC], inv[kC], nrm[kC], red[kC];
};

// Rows t0 .. t0 + nc - 1 of the frame: khat (normalised), beta, v.
template <int ND, typename T>
__device__ __forceinline__ void load_chunk(FrameSmem<ND> &sm, const BwdParams &p, const T *k, const T *v,
                                           const float *beta, long t0, int nc, int tid) {
  constexpr int LD = FrameSmem<ND>::LD;
  const int dk = p.dk, dv = p.dv;
  for (int e = tid; e < kC * dk; e += kThreads) {
    const int t = e / dk, i = e % dk;
    sm.K[t * LD + i] = t < nc ? ldf(k + (t0 + t) * dk + i) : 0.f;
  }
  for (int e = tid; e < kC * dv; e += kThreads) {
    const int t = e / dv, jj = e % dv;
    sm.E[t * LD + jj] = t < nc ? ldf(v + (t0 + t) * dv + jj) : 0.f;
  }
  if (tid < kC) {
    const float braw = tid < nc ? beta[t0 + tid] : 0.f;
    sm.b[tid] = tid < nc ? (p.gates_are_logits ? gate_beta(braw) : braw) : 0.f;
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < kC; t += kThreads / 32) {
    float ss = 0.f;
    for (int i = lane; i < dk; i += 32) ss = fmaf(sm.K[t * LD + i], sm.K[t * LD + i], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) {
      const float n = sqrtf(ss);
      sm.nrm[t] = n;
      sm.inv[t] = 1.0f / fmaxf(n, kKeyNormEps);
    }
  }
  __syncthreads();
  for (int e = tid; e < kC * dk; e += kThreads) {
    const int t = e / dk, i = e % dk;
    sm.K[t * LD + i] *= sm.inv[t];
  }
  __syncthreads();
}

// Gram matrix into the upper triangle (with the diagonal) of M, then
// Linv = (I + N)^-1, N[t][s] = beta_t (khat_t . khat_s) for s < t, into the
// strict lower triangle (its unit diagonal implied): 16 x 16 blocks, the
// diagonal ones by forward substitution, the others by block substitution.
template <int ND>
__device__ __forceinline__ void gram_inverse(FrameSmem<ND> &sm, int nc, int dk, int tid) {
  constexpr int LD = FrameSmem<ND>::LD;
  const int ty = tid >> 4, tx = tid & 15;
  {
    float g[3][3];
    zero(g);
    mm(g, dk, ty, tx, [&](int m, int k) { return sm.K[m * LD + k]; },
       [&](int k, int n) { return sm.K[n * LD + k]; });
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int jj = 0; jj < 3; ++jj) {
        const int t = ty + 16 * i, s = tx + 16 * jj;
        if (s >= t) sm.M[t * kLdC + s] = g[i][jj];
      }
  }
  __syncthreads();
  // N[t][s] (s < t) = beta_t M[s][t]
  auto Nv = [&](int t, int s) { return sm.b[t] * sm.M[s * kLdC + t]; };
  const int nb = (nc + 15) / 16;
  // diagonal blocks: thread (block kb, column c) solves column c of D_kb
  if (tid < 16 * nb) {
    const int kb = tid >> 4, c = tid & 15, o = 16 * kb;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a = (r == c) ? 1.f : 0.f;
#pragma unroll
      for (int u = 0; u < r; ++u) a -= (u >= c) ? Nv(o + r, o + u) * x[u] : 0.f;
      x[r] = r >= c ? a : 0.f;
    }
    // a thread writes only its own column's entries, read by no other thread before the barrier
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r > c) sm.M[(o + r) * kLdC + o + c] = x[r];
  }
  __syncthreads();
  // off-diagonal blocks, by distance: Linv_{i,j} = -D_i sum_{m=j}^{i-1} N_{i,m} Linv_{m,j}
  for (int d = 1; d < nb; ++d) {
    // T_{i,j} = sum_m N_{i,m} Linv_{m,j}  (Linv_{m,m} = D_m with its unit diagonal)
    for (int e = tid; e < (nb - d) * 256; e += kThreads) {
      const int jb = e >> 8, r = (e >> 4) & 15, c = e & 15, ib = jb + d;
      float a = 0.f;
      for (int mb = jb; mb < ib; ++mb)
        for (int u = 0; u < 16; ++u) {
          const int s = 16 * mb + u, col = 16 * jb + c;
          const float lv = s == col ? 1.f : (s > col ? sm.M[s * kLdC + col] : 0.f);
          a = fmaf(Nv(16 * ib + r, s), lv, a);
        }
      sm.T[jb * 272 + r * 17 + c] = a;
    }
    __syncthreads();
    // Linv_{i,j} = -D_i T_{i,j}
    for (int e = tid; e < (nb - d) * 256; e += kThreads) {
      const int jb = e >> 8, r = (e >> 4) & 15, c = e & 15, ib = jb + d;
      float a = sm.T[jb * 272 + r * 17 + c];  // D_i's unit diagonal
      for (int u = 0; u < r; ++u) a = fmaf(sm.M[(16 * ib + r) * kLdC + 16 * ib + u], sm.T[jb * 272 + u * 17 + c], a);
      sm.M[(16 * ib + r) * kLdC + 16 * jb + c] = -a;
    }
    __syncthreads();
  }
}

// Linv[t][s] with its unit diagonal and zero upper part
template <int ND>
__device__ __forceinline__ float linv(const FrameSmem<ND> &sm, int t, int s) {
  return s < t ? sm.M[t * kLdC + s] : (s == t ? 1.f : 0.f);
}

template <int ND, typename T>
__global__ void __launch_bounds__(kThreads, 1) gdn_bwd_frame_kernel(BwdParams p) {
  using SM = FrameSmem<ND>;
  constexpr int LD = SM::LD;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SM &sm = *reinterpret_cast<SM *>(smem_raw);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const long N = (long)F * L;
  const long SS = (long)dk * dv;
  const int f = blockIdx.x % F, bh = blockIdx.x / F;
  const T *k = static_cast<const T *>(p.k) + (long)bh * N * dk;
  const T *v = static_cast<const T *>(p.v) + (long)bh * N * dv;
  const float *beta = p.beta + (long)bh * N;
  const float *d_o = p.d_o + (long)bh * N * dv;
  float *dq = p.dq + (long)bh * N * dk;
  float *dkg = p.dk_out + (long)bh * N * dk;
  float *dvg = p.dv_out + (long)bh * N * dv;  // also the U scratch of the forward sweep
  float *dbg = p.dbeta + (long)bh * N;
  const int nch = (L + kC - 1) / kC;

  for (int e = tid; e < (int)(sizeof(SM) / 4); e += kThreads) reinterpret_cast<float *>(&sm)[e] = 0.f;
  __syncthreads();
  const float araw = p.alpha[(long)bh * F + f];
  const float al = p.gates_are_logits ? gate_alpha(araw) : araw;
  {
    const float *sprev = f > 0 ? p.states + ((long)bh * F + f - 1) * SS
                               : (p.state_in ? p.state_in + (long)bh * SS : nullptr);
    const float *gf = p.gbuf + ((long)bh * F + f) * SS;
    for (int e = tid; e < dk * dv; e += kThreads) {
      const int i = e / dv, jj = e % dv;
      sm.S[i * LD + jj] = sprev ? al * __ldg(sprev + e) : 0.f;
      sm.H[i * LD + jj] = __ldg(gf + e);
    }
  }
  __syncthreads();

  // ---- forward sweep
  for (int c = 0; c < nch; ++c) {
    const long t0 = (long)f * L + c * kC;
    const int nc = min(kC, L - c * kC);
    load_chunk<ND, T>(sm, p, k, v, beta, t0, nc, tid);
    gram_inverse<ND>(sm, nc, dk, tid);
    {  // E = V - Khat S
      float a[3][ND];
      zero(a);
      mm(a, dk, ty, tx, [&](int m, int kk) { return sm.K[m * LD + kk]; },
         [&](int kk, int n) { return sm.S[kk * LD + n]; });
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) sm.E[(ty + 16 * i) * LD + tx + 16 * jj] -= a[i][jj];
    }
    __syncthreads();
    {  // U = Linv diag(beta) E
      float a[3][ND];
      zero(a);
      mm(a, nc, ty, tx, [&](int m, int s) { return linv(sm, m, s) * sm.b[s]; },
         [&](int s, int n) { return sm.E[s * LD + n]; });
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) {
          const int t = ty + 16 * i, n = tx + 16 * jj;
          sm.U[t * LD + n] = a[i][jj];
          if (t < nc && n < dv) dvg[(t0 + t) * dv + n] = a[i][jj];
        }
    }
    __syncthreads();
    {  // S += Khat^T U
      float a[ND][ND];
      zero(a);
      mm(a, nc, ty, tx, [&](int m, int t) { return sm.K[t * LD + m]; },
         [&](int t, int n) { return sm.U[t * LD + n]; });
#pragma unroll
      for (int i = 0; i < ND; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) sm.S[(ty + 16 * i) * LD + tx + 16 * jj] += a[i][jj];
    }
    __syncthreads();
  }

  // ---- dq = dO S_f^T
  for (int c = 0; c < nch; ++c) {
    const long t0 = (long)f * L + c * kC;
    const int nc = min(kC, L - c * kC);
    for (int e = tid; e < kC * dv; e += kThreads) {
      const int t = e / dv, jj = e % dv;
      sm.G[t * LD + jj] = t < nc ? __ldg(d_o + (t0 + t) * dv + jj) : 0.f;
    }
    __syncthreads();
    float a[3][ND];
    zero(a);
    mm(a, dv, ty, tx, [&](int m, int jj) { return sm.G[m * LD + jj]; },
       [&](int jj, int n) { return sm.S[n * LD + jj]; });
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int jj = 0; jj < ND; ++jj) {
        const int t = ty + 16 * i, n = tx + 16 * jj;
        if (t < nc && n < dk) dq[(t0 + t) * dk + n] = a[i][jj];
      }
    __syncthreads();
  }

  // ---- reverse sweep
  for (int c = nch - 1; c >= 0; --c) {
    const long t0 = (long)f * L + c * kC;
    const int nc = min(kC, L - c * kC);
    for (int e = tid; e < kC * dv; e += kThreads) {
      const int t = e / dv, jj = e % dv;
      sm.U[t * LD + jj] = t < nc ? dvg[(t0 + t) * dv + jj] : 0.f;
    }
    load_chunk<ND, T>(sm, p, k, v, beta, t0, nc, tid);  // (its barriers order the U loads too)
    {  // S -= Khat^T U: the chunk's start state
      float a[ND][ND];
      zero(a);
      mm(a, nc, ty, tx, [&](int m, int t) { return sm.K[t * LD + m]; },
         [&](int t, int n) { return sm.U[t * LD + n]; });
#pragma unroll
      for (int i = 0; i < ND; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) sm.S[(ty + 16 * i) * LD + tx + 16 * jj] -= a[i][jj];
    }
    gram_inverse<ND>(sm, nc, dk, tid);  // (starts with reads of K only; its barriers order S)
    {  // E = V - Khat S
      float a[3][ND];
      zero(a);
      mm(a, dk, ty, tx, [&](int m, int kk) { return sm.K[m * LD + kk]; },
         [&](int kk, int n) { return sm.S[kk * LD + n]; });
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) sm.E[(ty + 16 * i) * LD + tx + 16 * jj] -= a[i][jj];
    }
    __syncthreads();
    {  // R = E - strict_lower(Khat Khat^T) U  (in place: each thread owns its elements)
      float a[3][ND];
      zero(a);
      mm(a, nc, ty, tx, [&](int m, int s) { return s < m ? sm.M[s * kLdC + m] : 0.f; },
         [&](int s, int n) { return sm.U[s * LD + n]; });
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) sm.E[(ty + 16 * i) * LD + tx + 16 * jj] -= a[i][jj];
    }
    {  // Khat H -> G
      float a[3][ND];
      zero(a);
      mm(a, dk, ty, tx, [&](int m, int kk) { return sm.K[m * LD + kk]; },
         [&](int kk, int n) { return sm.H[kk * LD + n]; });
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) sm.G[(ty + 16 * i) * LD + tx + 16 * jj] = a[i][jj];
    }
    __syncthreads();
    {  // Gm = Linv^T (Khat H), in place after a barrier
      float a[3][ND];
      zero(a);
      mm(a, nc, ty, tx, [&](int m, int s) { return linv(sm, s, m); },
         [&](int s, int n) { return sm.G[s * LD + n]; });
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) {
          const int t = ty + 16 * i, n = tx + 16 * jj;
          sm.G[t * LD + n] = a[i][jj];
          if (t < nc && n < dv) dvg[(t0 + t) * dv + n] = sm.b[t] * a[i][jj];
        }
    }
    __syncthreads();
    {  // dbeta_t = g_t . R_t
      const int warp = tid >> 5, lane = tid & 31;
      for (int t = warp; t < nc; t += kThreads / 32) {
        float s = 0.f;
        for (int jj = lane; jj < dv; jj += 32) s = fmaf(sm.G[t * LD + jj], sm.E[t * LD + jj], s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
          const float bt = sm.b[t];
          dbg[t0 + t] = p.gates_are_logits ? s * bt * (1.f - bt) : s;
        }
      }
    }
    // dkhat = diag(beta) (R H^T - Gm S^T - M Khat)
    float dkh[3][ND];
    zero(dkh);
    mm(dkh, dv, ty, tx, [&](int m, int jj) { return sm.E[m * LD + jj]; },
       [&](int jj, int n) { return sm.H[n * LD + jj]; });
    {
      float a[3][ND];
      zero(a);
      mm(a, dv, ty, tx, [&](int m, int jj) { return sm.G[m * LD + jj]; },
         [&](int jj, int n) { return sm.S[n * LD + jj]; });
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) dkh[i][jj] -= a[i][jj];
    }
    {  // M: upper beta_s R_t . g_s, lower g_t . u_s (Gram and Linv are dead)
      float r1[3][3], r2[3][3];
      zero(r1);
      zero(r2);
      mm(r1, dv, ty, tx, [&](int m, int jj) { return sm.E[m * LD + jj]; },
         [&](int jj, int n) { return sm.G[n * LD + jj]; });
      mm(r2, dv, ty, tx, [&](int m, int jj) { return sm.G[m * LD + jj]; },
         [&](int jj, int n) { return sm.U[n * LD + jj]; });
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int jj = 0; jj < 3; ++jj) {
          const int t = ty + 16 * i, s = tx + 16 * jj;
          sm.M[t * kLdC + s] = s > t ? sm.b[s] * r1[i][jj] : (s < t ? r2[i][jj] : 0.f);
        }
    }
    __syncthreads();
    {
      float a[3][ND];
      zero(a);
      mm(a, nc, ty, tx, [&](int m, int s) { return sm.M[m * kLdC + s]; },
         [&](int s, int n) { return sm.K[s * LD + n]; });
      // dk = (dkhat - khat (khat . dkhat)) / ||k|| (||k|| > eps), dkhat / eps (otherwise)
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        const int t = ty + 16 * i;
        const float bt = sm.b[t];
        float dot = 0.f;
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) {
          dkh[i][jj] = bt * (dkh[i][jj] - a[i][jj]);
          dot = fmaf(sm.K[t * LD + tx + 16 * jj], dkh[i][jj], dot);
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const bool proj = sm.nrm[t] > kKeyNormEps;
        const float sc = sm.inv[t];
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) {
          const int n = tx + 16 * jj;
          const float g = proj ? dkh[i][jj] - sm.K[t * LD + n] * dot : dkh[i][jj];
          if (t < nc && n < dk) dkg[(t0 + t) * dk + n] = g * sc;
        }
      }
    }
    {  // H -= Khat^T diag(beta) Gm
      float a[ND][ND];
      zero(a);
      mm(a, nc, ty, tx, [&](int m, int t) { return sm.K[t * LD + m] * sm.b[t]; },
         [&](int t, int n) { return sm.G[t * LD + n]; });
      __syncthreads();
#pragma unroll
      for (int i = 0; i < ND; ++i)
#pragma unroll
        for (int jj = 0; jj < ND; ++jj) sm.H[(ty + 16 * i) * LD + tx + 16 * jj] -= a[i][jj];
    }
    __syncthreads();
  }
  if (tid == 0) {
    const int ncg = (dv + 15) / 16;
    float s = 0.f;
    for (int cg = 0; cg < ncg; ++cg) s += p.dal_part[((long)bh * F + f) * ncg + cg];
    p.dalpha[(long)bh * F + f] = p.gates_are_logits ? s * (-al * (1.f - al)) : s;
  }
}

template <int ND, typename T>
cudaError_t launch_nd(const BwdParams &p, cudaStream_t st) {
  const size_t sa = sizeof(AdjSmem<ND>), sf = sizeof(FrameSmem<ND>);
  cudaError_t e = cudaFuncSetAttribute(gdn_bwd_adjoint_kernel<ND, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sa);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gdn_bwd_frame_kernel<ND, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sf);
  if (e != cudaSuccess) return e;
  const int BH = p.B * p.H;
  const int ncg = (p.dv + 15) / 16;
  gdn_bwd_adjoint_kernel<ND, T><<<BH * ncg, kThreads, sa, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gdn_bwd_frame_kernel<ND, T><<<(unsigned)((long)BH * p.F), kThreads, sf, st>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const BwdParams &p, cudaStream_t st) {
  const int d = p.dk > p.dv ? p.dk : p.dv;
  if (d <= 32) return launch_nd<2, T>(p, st);
  if (d <= 64) return launch_nd<4, T>(p, st);
  return launch_nd<7, T>(p, st);
}

}  // namespace bwd

bool gdn_bwd_supported(int dk, int dv) { return dk >= 1 && dv >= 1 && dk <= 112 && dv <= 112; }

cudaError_t launch_gdn_bwd(const BwdParams &p, int in_dtype, cudaStream_t st) {
  if (!gdn_bwd_supported(p.dk, p.dv)) return cudaErrorInvalidValue;
  return in_dtype == GDN_DTYPE_F32 ? bwd::launch_t<float>(p, st) : bwd::launch_t<__nv_bfloat16>(p, st);
}

}  // namespace gdn
