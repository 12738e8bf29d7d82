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
//  2. gdn_bwd_qdo_kernel: C_f = Q_f^T dO_f for every frame (frame-parallel);
//     gdn_bwd_adjoint_kernel: the frame chain in reverse.  With
//     G_f = dL/dS_f (end of frame f),
//        G_{F-1} = dS_out + C_{F-1},   G_{f-1} = C_{f-1} + alpha_f A_f^T G_f,
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
//                      (row t: the token's residual v_t - S_{t-1}^T khat_t;
//                      the warp-MMA kernel keeps R and Linv from the forward
//                      sweep instead),
//                      Gm = Linv^T Khat H (row t: g_t = H_t^T khat_t with H_t
//                      the gradient after token t),
//                      dv = diag(beta) Gm, dbeta_t = g_t . R_t,
//                      dkhat = diag(beta) (R H^T - Gm S^T - M Khat), where
//                        M[t][s] = beta_s R_t . g_s (s > t), g_t . u_s (s < t)
//                      (the in-chunk terms of H_t r_t and S_{t-1} g_t),
//                      H -= Khat^T diag(beta) Gm;
//     dk from dkhat through the normalisation.
// Products: bf16 inputs on the tensor cores through warp-level mma.sync
// (tf32 operands, fp32 accumulation); fp32 inputs on CUDA cores in fp32
// (register tiles over shared memory), except Q^T dO, on the tensor cores with
// tf32 high/low operand splits (about fp32).
#include <type_traits>

#include "launch.h"

namespace gdn {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kC = 48;      // tokens per chunk (frame kernel)
constexpr int kQt = 64;     // tokens per tile (Q^T dO kernel)

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

// x rounded to the nearest tf32 value (10-bit significand), as a float
__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// Global -> shared copies of fp32 tiles: dst[r * ldd + c] = scale * src[r * gs + c]
// for r < rows, c < cols (rows >= nvalid read as zero).  Each thread keeps eight
// loads in flight before storing, four elements per load where the rows allow
// it (cols % 4 == 0); loads go through L2 (__ldcg), so that data this kernel
// wrote earlier is seen.
__device__ __forceinline__ float4 ld4(const float *p) { return __ldcg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
  const uint2 u = __ldcg(reinterpret_cast<const uint2 *>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float ld1(const float *p) { return __ldcg(p); }
__device__ __forceinline__ float ld1(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// kTf32: the stored values rounded to tf32 (tiles used only as warp-MMA operands).
template <bool kTf32 = false, typename T>
__device__ __forceinline__ void tile_load(float *dst, int ldd, const T *src, long gs, int rows, int nvalid, int cols,
                                          float scale = 1.f) {
  auto rnd = [](float x) { return kTf32 ? tf32_round(x) : x; };
  constexpr int kB = 8;
  if ((cols & 3) == 0 && (gs & 3) == 0) {
    const int cv = cols >> 2, nv = rows * cv;
    for (int base = threadIdx.x; base < nv; base += kB * (int)blockDim.x) {
      float4 r[kB];
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int e = base + b * (int)blockDim.x;
        const int row = e / cv, c4 = e - row * cv;
        r[b] = (e < nv && row < nvalid) ? ld4(src + row * gs + 4 * c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int e = base + b * (int)blockDim.x;
        if (e < nv) {
          const int row = e / cv, c4 = e - row * cv;
          float *d = dst + row * ldd + 4 * c4;
          d[0] = rnd(scale * r[b].x);
          d[1] = rnd(scale * r[b].y);
          d[2] = rnd(scale * r[b].z);
          d[3] = rnd(scale * r[b].w);
        }
      }
    }
  } else {
    const int nv = rows * cols;
    for (int base = threadIdx.x; base < nv; base += kB * (int)blockDim.x) {
      float r[kB];
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int e = base + b * (int)blockDim.x;
        const int row = e / cols, c = e - row * cols;
        r[b] = (e < nv && row < nvalid) ? ld1(src + row * gs + c) : 0.f;
      }
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int e = base + b * (int)blockDim.x;
        if (e < nv) {
          const int row = e / cols, c = e - row * cols;
          dst[row * ldd + c] = rnd(scale * r[b]);
        }
      }
    }
  }
}

// Asynchronous global -> shared copies of fp32 rows, 16 bytes per cp.async:
// dst[r * ldd + c] = src[r * gs + c] for r < rows, c < cols (cols, gs and ldd
// multiples of 4, both bases 16-byte aligned).  The caller commits the group,
// waits for it and then synchronises the block before the rows are read.
__device__ __forceinline__ void tile_load_async(float *dst, int ldd, const float *src, long gs, int rows, int cols) {
  const int cv = cols >> 2, nv = rows * cv;
  for (int e = threadIdx.x; e < nv; e += blockDim.x) {
    const int row = e / cv, c4 = e - row * cv;
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst + row * ldd + 4 * c4);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src + row * gs + 4 * c4) : "memory");
  }
}

// Ask L2 for [base, base + bytes) (128-byte lines spread over the block's threads).
__device__ __forceinline__ void prefetch_l2(const void *base, long bytes) {
  const char *b = static_cast<const char *>(base);
  for (long off = (long)threadIdx.x * 128; off < bytes; off += (long)blockDim.x * 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(b + off));
}

template <int TM, int TN>
__device__ __forceinline__ void zero(float (&acc)[TM][TN]) {
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

// ---------------------------------------------------------------- pass 2
// Shared memory: A_f^T [DP][DP + 1], G [DP][17].
template <int ND>
struct AdjSmem {
  static constexpr int DP = 16 * ND, LD = DP + 1;
  float a[DP * LD];
  float g[DP * 17];
  float red[kThreads / 32];
};

template <int ND>
__global__ void __launch_bounds__(kThreads) gdn_bwd_adjoint_kernel(BwdParams p) {
  using SM = AdjSmem<ND>;
  constexpr int LD = SM::LD;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SM &sm = *reinterpret_cast<SM *>(smem_raw);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int dk = p.dk, dv = p.dv, F = p.F;
  const int ncg = (dv + 15) / 16;
  const int bh = blockIdx.x / ncg, cg = blockIdx.x % ncg;
  const int j = cg * 16 + tx;  // this thread's column of G
  const bool jok = j < dv;
  const long SS = (long)dk * dv;

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
    tile_load(sm.a, LD, p.maps + ((long)bh * F + f) * (long)dk * dk, dk, dk, dk, dk);
    // G_f = C_f + carry (C_f = Q_f^T dO_f, from gdn_bwd_qdo_kernel in gbuf) -> gbuf and shared memory
    float *gout = p.gbuf + ((long)bh * F + f) * SS;
#pragma unroll
    for (int r = 0; r < ND; ++r) {
      const int i = ty + 16 * r;
      const float gv = (jok && i < dk ? __ldcg(gout + (long)i * dv + j) : 0.f) + carry[r];
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
// Row-major fp32 tiles with padded rows: LD = DP + PAD for d-wide rows, LDC =
// kC + PAD for chunk-wide rows (PAD 1 for the CUDA-core products, 4 for the
// warp-MMA fragments).
template <int ND, int PAD>
struct FrameSmemT {
  static constexpr int DP = 16 * ND, LD = DP + PAD, LDC = kC + PAD;
  float S[DP * LD];   // S[i][j]
  float H[DP * LD];   // H[i][j]
  float K[kC * LD];   // khat rows
  float E[kC * LD];   // v -> E -> R rows
  float U[kC * LD];   // U rows; dkhat rows (warp-MMA kernel)
  float G[kC * LD];   // Khat H -> Gm rows; dO rows for dq
  float M[kC * LDC];  // Gram (upper, with diagonal) | Linv (strict lower); then the dkhat coupling M
  float T[3 * 16 * 17];  // inverse scratch
  float b[kC], inv[kC], nrm[kC], red[kC];
};
template <int ND>
using FrameSmem = FrameSmemT<ND, 1>;

// 3D RoPE of one token: the start of its time, height and width rows in the angle
// table (time [F][dt/2], height [L/gw][dh/2], width [gw][dh/2]), each less the pair
// index of its band's first pair, so that pair j of any band is entry off + j.
struct RopeRow {
  int t_off, h_off, w_off;
};
__device__ __forceinline__ RopeRow rope_row(int f, int tf, const GdnParams &rp) {
  const int row = tf / rp.rope_gw, col = tf - row * rp.rope_gw;
  const int ht = rp.F * (rp.rope_dt / 2), hp = rp.rope_dh / 2;
  return {f * (rp.rope_dt / 2), ht + row * hp - rp.rope_dt / 2,
          ht + (rp.L / rp.rope_gw) * hp + col * hp - (rp.rope_dt + rp.rope_dh) / 2};
}
// (cos, sin) of the pair (dd, dd + 1), dd even: the band is a select, not a branch
__device__ __forceinline__ float2 rope_cs(int dd, const RopeRow &r, const GdnParams &rp) {
  const int off = dd < rp.rope_dt ? r.t_off : (dd < rp.rope_dt + rp.rope_dh ? r.h_off : r.w_off);
  return __ldg(rp.rope_tab + off + (dd >> 1));
}

// The 3D rotary position embedding of rows [0, rows) of an fp32 tile (row t = the
// token at index tf0 + t of frame f), in place: a warp per row, its lanes over the pairs.
__device__ __forceinline__ void rope_rows(float *x, int ld, int rows, int d, int f, int tf0, const GdnParams &rp) {
  const int lane = threadIdx.x & 31, nw = (int)(blockDim.x >> 5);
  for (int t = (int)(threadIdx.x >> 5); t < rows; t += nw) {
    const RopeRow r = rope_row(f, tf0 + t, rp);
    float *px = x + t * ld;
    for (int dd = 2 * lane; dd < d; dd += 64) {
      const float2 cs = rope_cs(dd, r, rp);
      const float x0 = px[dd], x1 = px[dd + 1];
      px[dd] = fmaf(x0, cs.x, -x1 * cs.y);
      px[dd + 1] = fmaf(x0, cs.y, x1 * cs.x);
    }
  }
}

// Rows t0 .. t0 + nc - 1 of the frame: khat (normalised), beta and (kV) v.  With
// the embedding (rp.rope_on), k is rotated before its normalisation.
template <class SM, typename T, bool kV = true, bool kTf32 = false>
__device__ __forceinline__ void load_chunk(SM &sm, const BwdParams &p, const GdnParams &rp, const T *k, const T *v,
                                           const float *beta, long t0, int nc, int tid) {
  constexpr int LD = SM::LD;
  const int dk = p.dk, dv = p.dv;
  tile_load(sm.K, LD, k + t0 * dk, dk, kC, nc, dk);
  if (kV) tile_load(sm.E, LD, v + t0 * dv, dv, kC, nc, dv);
  if (tid < kC) {
    const float braw = tid < nc ? beta[t0 + tid] : 0.f;
    sm.b[tid] = tid < nc ? (p.gates_are_logits ? gate_beta(braw) : braw) : 0.f;
  }
  __syncthreads();
  if (rp.rope_on) {
    const int f = (int)(t0 / p.L);
    rope_rows(sm.K, LD, nc, dk, f, (int)(t0 - (long)f * p.L), rp);
    __syncthreads();
  }
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < kC; t += (int)(blockDim.x >> 5)) {
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
  for (int e = tid; e < kC * dk; e += (int)blockDim.x) {
    const int t = e / dk, i = e % dk;
    const float x = sm.K[t * LD + i] * sm.inv[t];
    sm.K[t * LD + i] = kTf32 ? tf32_round(x) : x;
  }
  __syncthreads();
}

// Linv = (I + N)^-1, N[t][s] = beta_t (khat_t . khat_s) for s < t, into the
// strict lower triangle of M (its unit diagonal implied), from the Gram matrix
// in the upper triangle: 16 x 16 blocks, the diagonal ones by forward
// substitution, the others by block substitution.
template <class SM>
__device__ __forceinline__ void inverse(SM &sm, int nc, int tid) {
  constexpr int kLdC = SM::LDC;
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
    for (int e = tid; e < (nb - d) * 256; e += (int)blockDim.x) {
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
    for (int e = tid; e < (nb - d) * 256; e += (int)blockDim.x) {
      const int jb = e >> 8, r = (e >> 4) & 15, c = e & 15, ib = jb + d;
      float a = sm.T[jb * 272 + r * 17 + c];  // D_i's unit diagonal
      for (int u = 0; u < r; ++u) a = fmaf(sm.M[(16 * ib + r) * kLdC + 16 * ib + u], sm.T[jb * 272 + u * 17 + c], a);
      sm.M[(16 * ib + r) * kLdC + 16 * jb + c] = -a;
    }
    __syncthreads();
  }
}

// Gram matrix (CUDA cores) into the upper triangle of M, with the diagonal; then the inverse.
template <int ND>
__device__ __forceinline__ void gram_inverse(FrameSmem<ND> &sm, int nc, int dk, int tid) {
  constexpr int LD = FrameSmem<ND>::LD, kLdC = FrameSmem<ND>::LDC;
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
  inverse(sm, nc, tid);
}

// Linv[t][s] with its unit diagonal and zero upper part
template <class SM>
__device__ __forceinline__ float linv(const SM &sm, int t, int s) {
  return s < t ? sm.M[t * SM::LDC + s] : (s == t ? 1.f : 0.f);
}

template <int ND, typename T>
__global__ void __launch_bounds__(kThreads, 1) gdn_bwd_frame_kernel(BwdParams p, GdnParams rp) {
  using SM = FrameSmem<ND>;
  constexpr int LD = SM::LD, kLdC = SM::LDC;
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
    if (sprev) tile_load(sm.S, LD, sprev, dv, dk, dk, dv, al);
    tile_load(sm.H, LD, p.gbuf + ((long)bh * F + f) * SS, dv, dk, dk, dv);
  }
  __syncthreads();

  // ---- forward sweep
  for (int c = 0; c < nch; ++c) {
    const long t0 = (long)f * L + c * kC;
    const int nc = min(kC, L - c * kC);
    load_chunk(sm, p, rp, k, v, beta, t0, nc, tid);
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
    tile_load(sm.G, LD, d_o + t0 * dv, dv, kC, nc, dv);
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
    tile_load(sm.U, LD, dvg + t0 * dv, dv, kC, nc, dv);
    load_chunk(sm, p, rp, k, v, beta, t0, nc, tid);  // (its barriers order the U loads too)
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

// ---------------------------------------------------------------- pass 3 on warp MMAs (bf16 inputs)
// The same frame kernel with every product on the tensor cores through
// mma.sync m16n8k8 (tf32 operands, fp32 accumulation).  NP = 1: operands
// rounded to tf32 (10-bit significands); NP = 3: each operand split into tf32
// high and low parts and the three leading products summed (about fp32).
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc += the (16 MT) x (8 NT) block at (m0, n0) of sum_{k < K} fa(m, k) fb(k, n),
// in the m16n8 accumulator layout (lane: g = lane / 4 rows g, g + 8; t = lane % 4
// columns 2t, 2t + 1).  A fragments: rows g, g + 8, k = t, t + 4; B: k = t, t + 4, column g.
// RA / RB false: that operand already holds tf32 values (rounded where it was
// written), so its fragments skip the conversion (one-pass products only).
template <int MT, int NT, int NP, bool RA = true, bool RB = true, class FA, class FB>
__device__ __forceinline__ void wmm(float (&acc)[MT][NT][4], int m0, int n0, int K, FA fa, FB fb) {
  constexpr bool ca = RA || NP != 1, cb = RB || NP != 1;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 1
  for (int k0 = 0; k0 < K; k0 += 8) {
    const int ka = k0 + t, kb = k0 + t + 4;
    const bool va = ka < K, vb = kb < K;
    uint32_t ah[MT][4], al[MT][4], bh[NT][2], bl[NT][2];
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      const int r = m0 + 16 * i + g;
      const float x[4] = {va ? fa(r, ka) : 0.f, va ? fa(r + 8, ka) : 0.f, vb ? fa(r, kb) : 0.f,
                          vb ? fa(r + 8, kb) : 0.f};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ah[i][e] = ca ? to_tf32(x[e]) : __float_as_uint(x[e]);
        if (NP == 3) al[i][e] = to_tf32(x[e] - __uint_as_float(ah[i][e]));
      }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int n = n0 + 8 * j + g;
      const float y[2] = {va ? fb(ka, n) : 0.f, vb ? fb(kb, n) : 0.f};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        bh[j][e] = cb ? to_tf32(y[e]) : __float_as_uint(y[e]);
        if (NP == 3) bl[j][e] = to_tf32(y[e] - __uint_as_float(bh[j][e]));
      }
    }
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        mma_tf32(acc[i][j], ah[i], bh[j]);
        if (NP == 3) {
          mma_tf32(acc[i][j], ah[i], bl[j]);
          mma_tf32(acc[i][j], al[i], bh[j]);
        }
      }
  }
}

template <int MT, int NT, class EP>
__device__ __forceinline__ void each(const float (&acc)[MT][NT][4], int m0, int n0, EP ep) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) ep(m0 + 16 * i + g + 8 * (e >> 1), n0 + 8 * j + 2 * t + (e & 1), acc[i][j][e]);
}

// An M x N product over all warps, blocks of (16 MT) x (8 NT) taken round-robin;
// ep(m, n, value) for every element inside M x N.
template <int MT, int NT, int NP, bool RA = true, bool RB = true, class FA, class FB, class EP>
__device__ __forceinline__ void wrun(int M, int N, int K, FA fa, FB fb, EP ep) {
  const int warp = threadIdx.x >> 5;
  const int nmb = (M + 16 * MT - 1) / (16 * MT), nnb = (N + 8 * NT - 1) / (8 * NT);
  for (int blk = warp; blk < nmb * nnb; blk += (int)(blockDim.x >> 5)) {
    const int m0 = (blk % nmb) * 16 * MT, n0 = (blk / nmb) * 8 * NT;
    float acc[MT][NT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
    wmm<MT, NT, NP, RA, RB>(acc, m0, n0, K, fa, fb);
    each(acc, m0, n0, [&](int m, int n, float v) {
      if (m < M && n < N) ep(m, n, v);
    });
  }
}

// The same with at most one block per warp and a barrier between the products
// and the epilogue (for results written over an operand).  All threads call it.
template <int MT, int NT, int NP, bool RA = true, bool RB = true, class FA, class FB, class EP>
__device__ __forceinline__ void wrun_sync(int M, int N, int K, FA fa, FB fb, EP ep) {
  const int warp = threadIdx.x >> 5;
  const int nmb = (M + 16 * MT - 1) / (16 * MT), nnb = (N + 8 * NT - 1) / (8 * NT);
  const bool has = warp < nmb * nnb;
  const int m0 = (warp % nmb) * 16 * MT, n0 = (warp / nmb) * 8 * NT;
  float acc[MT][NT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
  if (has) wmm<MT, NT, NP, RA, RB>(acc, m0, n0, K, fa, fb);
  __syncthreads();
  if (has)
    each(acc, m0, n0, [&](int m, int n, float v) {
      if (m < M && n < N) ep(m, n, v);
    });
}

template <int ND, typename T, int NP, int NW>
__global__ void __launch_bounds__(32 * NW, 1) gdn_bwd_frame_mma_kernel(BwdParams p, GdnParams rp) {
  constexpr int kTh = 32 * NW;
  constexpr int NB = NW >= 16 ? 1 : 2;  // 8-column tiles per warp block: more warps, narrower blocks
  using SM = FrameSmemT<ND, 4>;
  constexpr int LD = SM::LD, LDC = SM::LDC;
  static_assert(2 * ND <= NB * NW, "one block per warp");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SM &sm = *reinterpret_cast<SM *>(smem_raw);
  const int tid = threadIdx.x;
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
  const int warp = tid >> 5, lane = tid & 31;
  // each token's residual R (kept by the forward sweep for the reverse one): in the
  // workspace, or in dk_out's rows (dv <= dk), which the reverse sweep overwrites after reading
  float *rdst = p.rbuf ? p.rbuf + (long)bh * N * dv : dkg;
  const int rld = p.rbuf ? dv : dk;
  float *lbuf = p.linv_buf + ((long)bh * F + f) * nch * (kC * kC);  // each chunk's Linv, [48][48]

  for (int e = tid; e < (int)(sizeof(SM) / 4); e += kTh) reinterpret_cast<float *>(&sm)[e] = 0.f;
  __syncthreads();
  const float araw = p.alpha[(long)bh * F + f];
  const float al = p.gates_are_logits ? gate_alpha(araw) : araw;
  {
    const float *sprev = f > 0 ? p.states + ((long)bh * F + f - 1) * SS
                               : (p.state_in ? p.state_in + (long)bh * SS : nullptr);
    if (sprev) tile_load(sm.S, LD, sprev, dv, dk, dk, dv, al);
    tile_load(sm.H, LD, p.gbuf + ((long)bh * F + f) * SS, dv, dk, dk, dv);
  }
  __syncthreads();
  auto Krow = [&](int m, int kk) { return sm.K[m * LD + kk]; };  // Khat (t, i)
  auto Kcol = [&](int m, int kk) { return sm.K[kk * LD + m]; };  // Khat^T (i, t)
  auto gram = [&]() {
    wrun<3, NB, NP, false, false>(kC, kC, dk, Krow, [&](int kk, int n) { return sm.K[n * LD + kk]; },
                                  [&](int m, int n, float x) {
                                    if (n >= m) sm.M[m * LDC + n] = x;
                                  });
  };

  // ---- forward sweep
  for (int c = 0; c < nch; ++c) {
    const long t0 = (long)f * L + c * kC;
    const int nc = min(kC, L - c * kC);
    if (c + 1 < nch) {
      const int nn = min(kC, L - (c + 1) * kC);
      prefetch_l2(k + (t0 + kC) * dk, (long)nn * dk * sizeof(T));
      prefetch_l2(v + (t0 + kC) * dv, (long)nn * dv * sizeof(T));
    }
    load_chunk<SM, T, true, true>(sm, p, rp, k, v, beta, t0, nc, tid);
    gram();
    __syncthreads();
    inverse(sm, nc, tid);
    wrun<3, NB, NP, false, true>(kC, dv, dk, Krow, [&](int kk, int n) { return sm.S[kk * LD + n]; },
                                 [&](int m, int n, float x) { sm.E[m * LD + n] -= x; });  // E = V - Khat S
    __syncthreads();
    wrun<3, NB, NP>(kC, dv, nc, [&](int m, int s2) { return linv(sm, m, s2) * sm.b[s2]; },
                   [&](int s2, int n) { return sm.E[s2 * LD + n]; }, [&](int m, int n, float x) {
                     const float xr = tf32_round(x);  // U = Linv diag(beta) E (an operand from here on)
                     sm.U[m * LD + n] = xr;
                     if (m < nc) dvg[(t0 + m) * dv + n] = xr;
                   });
    __syncthreads();
    wrun<ND, NB, NP, false, false>(dk, dv, nc, Kcol, [&](int t, int n) { return sm.U[t * LD + n]; },
                                   [&](int m, int n, float x) { sm.S[m * LD + n] += x; });  // S += Khat^T U
    // R = E - strict_lower(Gram) U, and Linv, kept for the reverse sweep
    wrun<3, NB, NP, true, false>(kC, dv, nc, [&](int m, int s2) { return s2 < m ? sm.M[s2 * LDC + m] : 0.f; },
                                 [&](int s2, int n) { return sm.U[s2 * LD + n]; }, [&](int m, int n, float x) {
                                   if (m < nc) rdst[(t0 + m) * rld + n] = tf32_round(sm.E[m * LD + n] - x);
                                 });
    for (int e = tid; e < kC * kC; e += kTh) lbuf[c * (kC * kC) + e] = sm.M[(e / kC) * LDC + e % kC];
    __syncthreads();
  }

  // ---- dq = dO S_f^T, the dO rows double-buffered in G and U (free here): the next
  // chunk's arrive by asynchronous copies while this chunk's product runs
  auto fetch_do = [&](int cc) {
    const long tt = (long)f * L + cc * kC;
    const int n = min(kC, L - cc * kC);
    float *dst = (cc & 1) ? sm.U : sm.G;
    if (dv % 4 == 0) {
      tile_load_async(dst, LD, d_o + tt * dv, dv, n, dv);
      asm volatile("cp.async.commit_group;" ::: "memory");
      for (int e = tid; e < (kC - n) * dv; e += kTh) dst[(n + e / dv) * LD + e % dv] = 0.f;
    } else {
      tile_load(dst, LD, d_o + tt * dv, dv, kC, n, dv);
    }
  };
  fetch_do(0);
  for (int c = 0; c < nch; ++c) {
    const long t0 = (long)f * L + c * kC;
    const int nc = min(kC, L - c * kC);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();  // chunk c's rows are visible; chunk c - 1's product is done with the other buffer
    if (c + 1 < nch) fetch_do(c + 1);
    const float *dcur = (c & 1) ? sm.U : sm.G;
    wrun<3, NB, NP>(kC, dk, dv, [&](int m, int jj) { return dcur[m * LD + jj]; },
                    [&](int jj, int n) { return sm.S[n * LD + jj]; }, [&](int m, int n, float x) {
                      if (m < nc) dq[(t0 + m) * dk + n] = x;
                    });
  }
  __syncthreads();

  // ---- reverse sweep (U, R and Linv kept by the forward sweep).  Chunk c's U, R and
  // Linv arrive by asynchronous copies issued during chunk c + 1's H update.
  const bool async_rows = dv % 4 == 0 && rld % 4 == 0;
  auto fetch = [&](int cc) {  // U, R and Linv of chunk cc -> U, E and M (rows past the frame zero)
    const long tt = (long)f * L + cc * kC;
    const int n = min(kC, L - cc * kC);
    if (async_rows) {
      tile_load_async(sm.U, LD, dvg + tt * dv, dv, n, dv);
      tile_load_async(sm.E, LD, rdst + tt * rld, rld, n, dv);
      tile_load_async(sm.M, LDC, lbuf + cc * (kC * kC), kC, kC, kC);
      asm volatile("cp.async.commit_group;" ::: "memory");
      for (int e = tid; e < (kC - n) * dv; e += kTh) {
        const int row = n + e / dv, col = e % dv;
        sm.U[row * LD + col] = 0.f;
        sm.E[row * LD + col] = 0.f;
      }
    } else {
      tile_load(sm.U, LD, dvg + tt * dv, dv, kC, n, dv);
      tile_load(sm.E, LD, rdst + tt * rld, rld, kC, n, dv);
      tile_load(sm.M, LDC, lbuf + cc * (kC * kC), kC, kC, kC, kC);
    }
  };
  fetch(nch - 1);
  for (int c = nch - 1; c >= 0; --c) {
    const long t0 = (long)f * L + c * kC;
    const int nc = min(kC, L - c * kC);
    if (c > 0) prefetch_l2(k + (t0 - kC) * dk, (long)kC * dk * sizeof(T));
    asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's copies; load_chunk's barrier publishes them
    load_chunk<SM, T, false, true>(sm, p, rp, k, v, beta, t0, nc, tid);
    wrun<ND, NB, NP, false, false>(dk, dv, nc, Kcol, [&](int t, int n) { return sm.U[t * LD + n]; },
                                   [&](int m, int n, float x) { sm.S[m * LD + n] -= x; });  // the chunk's start state
    wrun<3, NB, NP, false, true>(kC, dv, dk, Krow, [&](int kk, int n) { return sm.H[kk * LD + n]; },
                                 [&](int m, int n, float x) { sm.G[m * LD + n] = tf32_round(x); });  // Khat H
    __syncthreads();
    wrun_sync<3, NB, NP, true, false>(kC, dv, nc, [&](int m, int s2) { return linv(sm, s2, m); },
                                      [&](int s2, int n) { return sm.G[s2 * LD + n]; }, [&](int m, int n, float x) {
                          sm.G[m * LD + n] = tf32_round(x);  // Gm = Linv^T (Khat H), an operand from here on
                          if (m < nc) dvg[(t0 + m) * dv + n] = sm.b[m] * x;
                        });
    __syncthreads();
    for (int t = warp; t < nc; t += NW) {  // dbeta_t = g_t . R_t
      float s2 = 0.f;
      for (int jj = lane; jj < dv; jj += 32) s2 = fmaf(sm.G[t * LD + jj], sm.E[t * LD + jj], s2);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, off);
      if (lane == 0) {
        const float bt = sm.b[t];
        dbg[t0 + t] = p.gates_are_logits ? s2 * bt * (1.f - bt) : s2;
      }
    }
    // M: upper beta_s R_t . g_s, lower g_t . u_s (Gram and Linv are dead): 8 NB columns of
    // all 48 rows per warp, the first 6 / NB warps for R Gm^T, the next for Gm U^T
    if (warp < 12 / NB) {
      const int half = warp / (6 / NB), n0 = (warp % (6 / NB)) * 8 * NB;
      float r[3][NB][4] = {};
      if (half == 0) {
        wmm<3, NB, NP, false, false>(r, 0, n0, dv, [&](int m, int jj) { return sm.E[m * LD + jj]; },
                                     [&](int jj, int n) { return sm.G[n * LD + jj]; });
        each(r, 0, n0, [&](int m, int n, float x) {
          if (n >= m) sm.M[m * LDC + n] = n > m ? sm.b[n] * x : 0.f;
        });
      } else {
        wmm<3, NB, NP, false, false>(r, 0, n0, dv, [&](int m, int jj) { return sm.G[m * LD + jj]; },
                                     [&](int jj, int n) { return sm.U[n * LD + jj]; });
        each(r, 0, n0, [&](int m, int n, float x) {
          if (n < m) sm.M[m * LDC + n] = x;
        });
      }
    }
    __syncthreads();
    {  // dkhat = diag(beta) (R H^T - Gm S^T - M Khat) -> U rows (U is dead)
      const int n0 = warp * 8 * NB;
      const bool has = n0 < dk;
      float a[3][NB][4] = {};
      if (has) {
        wmm<3, NB, NP, false, true>(a, 0, n0, dv, [&](int m, int jj) { return sm.E[m * LD + jj]; },
                                    [&](int jj, int n) { return sm.H[n * LD + jj]; });
        wmm<3, NB, NP, false, true>(a, 0, n0, dv, [&](int m, int jj) { return -sm.G[m * LD + jj]; },
                                    [&](int jj, int n) { return sm.S[n * LD + jj]; });
        wmm<3, NB, NP, true, false>(a, 0, n0, nc, [&](int m, int s2) { return -sm.M[m * LDC + s2]; },
                                    [&](int s2, int n) { return sm.K[s2 * LD + n]; });
      }
      __syncthreads();
      if (has) each(a, 0, n0, [&](int m, int n, float x) { sm.U[m * LD + n] = sm.b[m] * x; });
    }
    __syncthreads();
    for (int t = warp; t < nc; t += NW) {
      // dk = (dkhat - khat (khat . dkhat)) / ||k|| (||k|| > eps), dkhat / eps (otherwise)
      float dot = 0.f;
      for (int i = lane; i < dk; i += 32) dot = fmaf(sm.K[t * LD + i], sm.U[t * LD + i], dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const bool proj = sm.nrm[t] > kKeyNormEps;
      const float sc = sm.inv[t];
      for (int i = lane; i < dk; i += 32) {
        const float gk = proj ? sm.U[t * LD + i] - sm.K[t * LD + i] * dot : sm.U[t * LD + i];
        dkg[(t0 + t) * dk + i] = gk * sc;
      }
    }
    __syncthreads();  // U (dkhat), E (R) and M are dead: the next chunk's arrive under the H update
    if (c > 0) fetch(c - 1);
    wrun<ND, NB, NP, true, false>(dk, dv, nc, [&](int m, int t) { return sm.K[t * LD + m] * sm.b[t]; },
                                  [&](int t, int n) { return sm.G[t * LD + n]; },
                    [&](int m, int n, float x) { sm.H[m * LD + n] -= x; });  // H -= Khat^T diag(beta) Gm
    __syncthreads();
  }
  if (tid == 0) {
    const int ncg = (dv + 15) / 16;
    float s2 = 0.f;
    for (int cg = 0; cg < ncg; ++cg) s2 += p.dal_part[((long)bh * F + f) * ncg + cg];
    p.dalpha[(long)bh * F + f] = p.gates_are_logits ? s2 * (-al * (1.f - al)) : s2;
  }
}

// ---------------------------------------------------------------- pass 2a
// C_f = Q_f^T dO_f for every frame, into gbuf (the adjoint chain adds its carry
// there): one CTA per frame, 64-token tiles of q and dO in shared memory, warp
// MMAs (tf32 operands with NP passes) over all d_k rows and 16 columns per warp.
template <int ND>
struct QdoSmem {
  static constexpr int DP = 16 * ND, LD = DP + 8;  // LD % 32 in {8, 24}: conflict-free k-major fragments
  float q[kQt * LD];
  float d[kQt * LD];
};

template <int ND, typename T, int NP>
__global__ void __launch_bounds__(kThreads) gdn_bwd_qdo_kernel(BwdParams p, GdnParams rp) {
  using SM = QdoSmem<ND>;
  constexpr int LD = SM::LD;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SM &sm = *reinterpret_cast<SM *>(smem_raw);
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const long N = (long)F * L;
  const int f = blockIdx.x % F, bh = blockIdx.x / F;
  const T *q = static_cast<const T *>(p.q) + (long)bh * N * dk + (long)f * L * dk;
  const float *d_o = p.d_o + (long)bh * N * dv + (long)f * L * dv;
  const int warp = threadIdx.x >> 5;
  const bool has = warp < (dv + 15) / 16;
  float acc[ND][2][4];
#pragma unroll
  for (int i = 0; i < ND; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
  for (int t0 = 0; t0 < L; t0 += kQt) {
    const int nt = min(kQt, L - t0);
    tile_load(sm.q, LD, q + (long)t0 * dk, dk, nt, nt, dk);
    tile_load(sm.d, LD, d_o + (long)t0 * dv, dv, nt, nt, dv);
    __syncthreads();
    if (rp.rope_on) {
      rope_rows(sm.q, LD, nt, dk, f, t0, rp);
      __syncthreads();
    }
    if (has)
      wmm<ND, 2, NP>(acc, 0, warp * 16, nt, [&](int m, int t) { return sm.q[t * LD + m]; },
                     [&](int t, int n) { return sm.d[t * LD + n]; });
    __syncthreads();
  }
  float *c = p.gbuf + ((long)bh * F + f) * (long)dk * dv;
  if (has)
    each(acc, 0, warp * 16, [&](int m, int n, float x) {
      if (m < dk && n < dv) c[(long)m * dv + n] = x;
    });
}

// With the embedding: dq and dk hold the gradients with respect to the rotated q
// and k; each pair is turned back by the transpose rotation (cos, -sin).  A warp
// per token, its lanes over the pairs.
__global__ void gdn_bwd_rope_back_kernel(float *dq, float *dk, long ntok, int F, int L, int d, GdnParams rp) {
  const int lane = threadIdx.x & 31;
  const long nwarps = (long)gridDim.x * (blockDim.x >> 5);
  for (long tok = blockIdx.x * (long)(blockDim.x >> 5) + (threadIdx.x >> 5); tok < ntok; tok += nwarps) {
    const long tt = tok % ((long)F * L);  // token index in its head's sequence
    const int f = (int)(tt / L), tf = (int)(tt - (long)f * L);
    const RopeRow r = rope_row(f, tf, rp);
    for (int dd = 2 * lane; dd < d; dd += 64) {
      const float2 cs = rope_cs(dd, r, rp);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        float2 *px = reinterpret_cast<float2 *>((w ? dk : dq) + tok * d + dd);
        const float2 x = *px;
        *px = make_float2(fmaf(x.x, cs.x, x.y * cs.y), fmaf(x.y, cs.x, -x.x * cs.y));
      }
    }
  }
}

// tf32 passes of the warp-MMA frame kernel (bf16 inputs): 3 = high/low split
constexpr int kMmaPasses = 1;
constexpr int kMmaWarps = 8;  // warps of the warp-MMA frame kernel (16 measured slower: a phase is as long as its k-loop)

template <int ND, typename T>
cudaError_t launch_nd(const BwdParams &p, const GdnParams &rp, cudaStream_t st) {
  constexpr bool mma = std::is_same<T, __nv_bfloat16>::value;
  const size_t sa = sizeof(AdjSmem<ND>);
  const size_t sf = mma ? sizeof(FrameSmemT<ND, 4>) : sizeof(FrameSmem<ND>);
  const size_t sq = sizeof(QdoSmem<ND>);
  constexpr int qnp = mma ? kMmaPasses : 3;  // fp32 inputs: high/low split (about fp32)
  cudaError_t e = cudaFuncSetAttribute(gdn_bwd_qdo_kernel<ND, T, qnp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sq);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gdn_bwd_adjoint_kernel<ND>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sa);
  if (e != cudaSuccess) return e;
  const int BH = p.B * p.H;
  const int ncg = (p.dv + 15) / 16;
  gdn_bwd_qdo_kernel<ND, T, qnp><<<(unsigned)((long)BH * p.F), kThreads, sq, st>>>(p, rp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gdn_bwd_adjoint_kernel<ND><<<BH * ncg, kThreads, sa, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((long)BH * p.F);
  if constexpr (mma) {
    e = cudaFuncSetAttribute(gdn_bwd_frame_mma_kernel<ND, T, kMmaPasses, kMmaWarps>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sf);
    if (e != cudaSuccess) return e;
    gdn_bwd_frame_mma_kernel<ND, T, kMmaPasses, kMmaWarps><<<grid, 32 * kMmaWarps, sf, st>>>(p, rp);
  } else {
    e = cudaFuncSetAttribute(gdn_bwd_frame_kernel<ND, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sf);
    if (e != cudaSuccess) return e;
    gdn_bwd_frame_kernel<ND, T><<<grid, kThreads, sf, st>>>(p, rp);
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const BwdParams &p, const GdnParams &rp, cudaStream_t st) {
  const int d = p.dk > p.dv ? p.dk : p.dv;
  cudaError_t e = d <= 32 ? launch_nd<2, T>(p, rp, st) : (d <= 64 ? launch_nd<4, T>(p, rp, st) : launch_nd<7, T>(p, rp, st));
  if (e != cudaSuccess || !rp.rope_on) return e;
  const long ntok = (long)p.B * p.H * p.F * p.L;
  const int blocks = (int)(ntok / 8 + 1 < 148 * 16 ? ntok / 8 + 1 : 148 * 16);  // 8 tokens (warps) per block
  gdn_bwd_rope_back_kernel<<<blocks, 256, 0, st>>>(p.dq, p.dk_out, ntok, p.F, p.L, p.dk, rp);
  return cudaGetLastError();
}

}  // namespace bwd

bool gdn_bwd_supported(int dk, int dv) { return dk >= 1 && dv >= 1 && dk <= 112 && dv <= 112; }
int gdn_bwd_chunks(int L) { return (L + bwd::kC - 1) / bwd::kC; }

cudaError_t launch_gdn_bwd(const BwdParams &p, const GdnParams &rope, int in_dtype, cudaStream_t st) {
  if (!gdn_bwd_supported(p.dk, p.dv)) return cudaErrorInvalidValue;
  return in_dtype == GDN_DTYPE_F32 ? bwd::launch_t<float>(p, rope, st) : bwd::launch_t<__nv_bfloat16>(p, rope, st);
}

}  // namespace gdn
