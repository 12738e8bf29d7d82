/*
 * CPU oracle for the frame-wise linear-attention recurrences (fp64).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code
 * with the CUDA path and is deliberately plain: per-token loops in double,
 * in the order the method states them, with no chunking, no blocking and no
 * re-association.  Inputs are read as float (bf16 inputs are passed as the
 * exact float values of the bf16 numbers) and widened to double.
 *
 * Sources for what is computed:
 *  - "SANA-WM, an open-source 2.6B world model for 1-minute 720p video"
 *    (GeekNews, vi.news.hada.io/topic?id=29572 and its Turkish twin
 *    tr.news.hada.io/topic?id=29572), section "Core design and generation
 *    pipeline": attention is a frame-wise (frame-level) Gated DeltaNet.
 *  - "How NVIDIA SANA-WM generates 60-second 720p video on one GPU"
 *    (dothoosh.com): the Gated DeltaNet keeps a fixed-size recurrent state,
 *    independent of video length.
 *  - "SANA-Video: Efficient Video Generation with Block Linear Diffusion
 *    Transformer (ICLR 2026 oral)" talk transcript (shadowingenglish.com),
 *    block KV cache passage: the linear-attention state is a fixed D x D
 *    matrix; block i adds its own KV contribution to the cached state of
 *    block i-1, and every token of a block reads that state.
 *
 * The pages print no equation.  The update rules below are the library's
 * definition of the two modes (the plainest reading consistent with the
 * pages), written in the stored layout S[i][j], i over d_k, j over d_v:
 *
 *  Gated DeltaNet, per (b, h), S starts at state_in (or 0):
 *    for each frame f:  alpha_f = exp(-softplus(a_f))   (or given)
 *                       S <- alpha_f * S
 *      for each token t of f, in order:
 *                       khat = k_t / max(||k_t||_2, 1e-6)
 *                       beta = sigmoid(b_t)              (or given)
 *                       r    = S^T khat - v_t            (length d_v)
 *                       S   <- S - beta * khat r^T
 *      for each token t of f:  o_t = S^T q_t  (state after the whole frame)
 *    state_out = S.
 *
 *  Block-causal ReLU linear attention, per (b, h), S = kv_in (or 0),
 *  z = z_in (or 0):
 *    for each frame f:  S += sum_{t in f} relu(k_t) v_t^T
 *                       z += sum_{t in f} relu(k_t)
 *      for each token t of f:
 *        o_t = relu(q_t)^T S / (relu(q_t)^T z + eps)
 *
 * Threads split the work over independent (b, h) heads and blocks of d_v
 * columns (column j of S and o depends only on column j of v and S0), which
 * changes no arithmetic.
 *
 * The backward of the Gated DeltaNet recurrence (oracle_gdn_bwd, below) is its
 * reverse-mode derivative, token by token in fp64; its pins are finite
 * differences of the forward and torch autograd through a separate loop.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GDN_KEY_NORM_EPS 1e-6

/* alpha = exp(-softplus(a)) with softplus(a) = log(1 + exp(a)). */
static double gate_alpha(double a) { return exp(-log1p(exp(a))); }
/* beta = sigmoid(b) = 1 / (1 + exp(-b)). */
static double gate_beta(double b) { return 1.0 / (1.0 + exp(-b)); }

double oracle_gate_alpha(double a) { return gate_alpha(a); }
double oracle_gate_beta(double b) { return gate_beta(b); }

/*
 * 3D rotary position embedding (SANA-Video talk, "3D RoPE for the linear
 * attention"; the talk gives no formula, this is the library's reading): a
 * d-vector at latent position (frame, row, column) is split into a time part
 * of dt dimensions, then a height and a width part of dh = dw = 2 * floor(d / 6)
 * each (dt = d - dh - dw); in each part the pair (2i, 2i + 1) is rotated by
 * the angle pos * base^(-2i / part_length), pos being that part's coordinate.
 * The token at index t of a frame of a grid_w-wide latent grid sits at row
 * t / grid_w and column t % grid_w.
 */
typedef struct {
  int on;
  int64_t grid_w;       /* latent grid width (tokens per row) */
  int64_t frame_offset; /* time coordinate of the first frame */
  double base;
} rope_t;

static void rope3d(const float *x, int64_t d, int64_t frame, int64_t row, int64_t col, double base, double *out) {
  const int64_t dh = 2 * (d / 6), dw = dh, dt = d - dh - dw;
  const int64_t len[3] = {dt, dh, dw}, pos[3] = {frame, row, col};
  int64_t o = 0;
  for (int a = 0; a < 3; ++a) {
    for (int64_t i = 0; i < len[a] / 2; ++i) {
      const double theta = pow(base, -2.0 * (double)i / (double)len[a]);
      const double phi = (double)pos[a] * theta;
      const double c = cos(phi), sn = sin(phi);
      const double x0 = (double)x[o + 2 * i], x1 = (double)x[o + 2 * i + 1];
      out[o + 2 * i] = x0 * c - x1 * sn;
      out[o + 2 * i + 1] = x0 * sn + x1 * c;
    }
    o += len[a];
  }
}

/* The rotation of a double d-vector by sign times rope3d's angles (sign = -1:
 * the transpose, which maps a gradient with respect to the rotated vector to
 * one with respect to the vector). */
static void rope3d_rot(const double *x, int64_t d, int64_t frame, int64_t row, int64_t col, double base, double sign,
                       double *out) {
  const int64_t dh = 2 * (d / 6), dw = dh, dt = d - dh - dw;
  const int64_t len[3] = {dt, dh, dw}, pos[3] = {frame, row, col};
  int64_t o = 0;
  for (int a = 0; a < 3; ++a) {
    for (int64_t i = 0; i < len[a] / 2; ++i) {
      const double phi = sign * (double)pos[a] * pow(base, -2.0 * (double)i / (double)len[a]);
      const double c = cos(phi), sn = sin(phi);
      const double x0 = x[o + 2 * i], x1 = x[o + 2 * i + 1];
      out[o + 2 * i] = x0 * c - x1 * sn;
      out[o + 2 * i + 1] = x0 * sn + x1 * c;
    }
    o += len[a];
  }
}

/* The embedding alone: x [n_heads, F*L, d] -> out (double), for tests. */
int oracle_rope3d(const float *x, double *out, int64_t nh, int64_t F, int64_t L, int64_t d, int64_t grid_w,
                  int64_t frame_offset, double base) {
  if (d <= 0 || d % 2 || grid_w <= 0 || L % grid_w) return 1;
  for (int64_t h = 0; h < nh; ++h)
    for (int64_t f = 0; f < F; ++f)
      for (int64_t t = 0; t < L; ++t) {
        const int64_t n = (h * F + f) * L + t;
        rope3d(x + n * d, d, frame_offset + f, t / grid_w, t % grid_w, base, out + n * d);
      }
  return 0;
}

typedef struct {
  const float *q, *k, *v, *alpha, *beta;
  int logits;
  const double *s_in;
  double *s_out, *o;
  int64_t F, L, dk, dv;
  int64_t bh;          /* flat head index */
  int64_t c0, c1;      /* column range [c0, c1) of d_v */
  rope_t rope;         /* 3D RoPE on q and k (k before its normalisation) */
} gdn_unit_t;

static void gdn_unit(const gdn_unit_t *u) {
  const int64_t F = u->F, L = u->L, dk = u->dk, dv = u->dv, N = F * L;
  const int64_t nc = u->c1 - u->c0;
  const float *q = u->q + u->bh * N * dk;
  const float *k = u->k + u->bh * N * dk;
  const float *v = u->v + u->bh * N * dv;
  const float *al = u->alpha + u->bh * F;
  const float *be = u->beta + u->bh * N;
  double *S = (double *)calloc((size_t)(dk * nc), sizeof(double)); /* S[i][j - c0] */
  double *kh = (double *)malloc(sizeof(double) * (size_t)dk);
  double *qr = (double *)malloc(sizeof(double) * (size_t)dk);
  double *r = (double *)malloc(sizeof(double) * (size_t)nc);
  if (u->s_in)
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < nc; ++j) S[i * nc + j] = u->s_in[u->bh * dk * dv + i * dv + u->c0 + j];
  for (int64_t f = 0; f < F; ++f) {
    const double alpha = u->logits ? gate_alpha((double)al[f]) : (double)al[f];
    for (int64_t e = 0; e < dk * nc; ++e) S[e] *= alpha;
    for (int64_t t = f * L; t < (f + 1) * L; ++t) {
      if (u->rope.on) {
        rope3d(k + t * dk, dk, u->rope.frame_offset + f, (t - f * L) / u->rope.grid_w, (t - f * L) % u->rope.grid_w,
               u->rope.base, kh);
      } else {
        for (int64_t i = 0; i < dk; ++i) kh[i] = (double)k[t * dk + i];
      }
      double ss = 0.0;
      for (int64_t i = 0; i < dk; ++i) ss += kh[i] * kh[i];
      double nrm = sqrt(ss);
      double den = nrm > GDN_KEY_NORM_EPS ? nrm : GDN_KEY_NORM_EPS;
      for (int64_t i = 0; i < dk; ++i) kh[i] = kh[i] / den;
      const double beta = u->logits ? gate_beta((double)be[t]) : (double)be[t];
      for (int64_t j = 0; j < nc; ++j) {
        double p = 0.0;
        for (int64_t i = 0; i < dk; ++i) p += S[i * nc + j] * kh[i];
        r[j] = p - (double)v[t * dv + u->c0 + j];
      }
      for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < nc; ++j) S[i * nc + j] -= beta * kh[i] * r[j];
    }
    if (u->o)
      for (int64_t t = f * L; t < (f + 1) * L; ++t) {
        if (u->rope.on) {
          rope3d(q + t * dk, dk, u->rope.frame_offset + f, (t - f * L) / u->rope.grid_w,
                 (t - f * L) % u->rope.grid_w, u->rope.base, qr);
        } else {
          for (int64_t i = 0; i < dk; ++i) qr[i] = (double)q[t * dk + i];
        }
        for (int64_t j = 0; j < nc; ++j) {
          double acc = 0.0;
          for (int64_t i = 0; i < dk; ++i) acc += S[i * nc + j] * qr[i];
          u->o[(u->bh * N + t) * dv + u->c0 + j] = acc;
        }
      }
  }
  if (u->s_out)
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < nc; ++j) u->s_out[u->bh * dk * dv + i * dv + u->c0 + j] = S[i * nc + j];
  free(S);
  free(kh);
  free(qr);
  free(r);
}

typedef struct {
  gdn_unit_t *units;
  int64_t n;
  int64_t next;
  pthread_mutex_t mu;
} pool_t;

static void *gdn_worker(void *p) {
  pool_t *pl = (pool_t *)p;
  for (;;) {
    pthread_mutex_lock(&pl->mu);
    int64_t i = pl->next++;
    pthread_mutex_unlock(&pl->mu);
    if (i >= pl->n) return NULL;
    gdn_unit(&pl->units[i]);
  }
}

/*
 * Gated DeltaNet frame recurrence (optionally with the 3D RoPE on q and k).
 * Layouts (row-major, contiguous):
 *   q, k [B,H,F*L,dk]; v [B,H,F*L,dv]; alpha [B,H,F]; beta [B,H,F*L];
 *   state_in/state_out [B,H,dk,dv] (nullable); o [B,H,F*L,dv] (nullable).
 * Only d_v columns [col_lo, col_hi) of o and state_out are written.
 * heads: optional list of nheads flat head indices to compute (NULL = all).
 */
int oracle_gdn(const float *q, const float *k, const float *v, const float *alpha, const float *beta,
               int gates_are_logits, const double *state_in, double *state_out, double *o,
               int64_t B, int64_t H, int64_t F, int64_t L, int64_t dk, int64_t dv,
               int64_t col_lo, int64_t col_hi, const int64_t *heads, int64_t nheads,
               int64_t col_block, int nthreads, int64_t rope_grid_w, int64_t rope_frame_offset,
               double rope_base) {
  if (B < 0 || H < 0 || F < 0 || L < 0 || dk <= 0 || dv <= 0) return 1;
  /* rope_grid_w > 0 turns the 3D RoPE on (q and k; needs even d_k and L a multiple of it) */
  if (rope_grid_w > 0 && (dk % 2 || L % rope_grid_w)) return 1;
  if (col_lo < 0 || col_hi > dv || col_lo > col_hi) return 1;
  if (col_block <= 0) col_block = dv;
  int64_t nh = heads ? nheads : B * H;
  int64_t nb = (col_hi - col_lo + col_block - 1) / col_block;
  int64_t n = nh * nb;
  if (n == 0) return 0;
  gdn_unit_t *units = (gdn_unit_t *)calloc((size_t)n, sizeof(gdn_unit_t));
  for (int64_t h = 0; h < nh; ++h)
    for (int64_t c = 0; c < nb; ++c) {
      gdn_unit_t *u = &units[h * nb + c];
      u->q = q; u->k = k; u->v = v; u->alpha = alpha; u->beta = beta;
      u->logits = gates_are_logits; u->s_in = state_in; u->s_out = state_out; u->o = o;
      u->F = F; u->L = L; u->dk = dk; u->dv = dv;
      u->bh = heads ? heads[h] : h;
      u->c0 = col_lo + c * col_block;
      u->c1 = u->c0 + col_block < col_hi ? u->c0 + col_block : col_hi;
      u->rope.on = rope_grid_w > 0;
      u->rope.grid_w = rope_grid_w > 0 ? rope_grid_w : 1;
      u->rope.frame_offset = rope_frame_offset;
      u->rope.base = rope_base;
    }
  pool_t pl;
  pl.units = units; pl.n = n; pl.next = 0;
  pthread_mutex_init(&pl.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > n) nthreads = (int)n;
  if (nthreads > 512) nthreads = 512;
  pthread_t th[512];
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, gdn_worker, &pl);
  gdn_worker(&pl);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&pl.mu);
  free(units);
  return 0;
}

/*
 * Backward of the Gated DeltaNet frame recurrence.
 *
 * The model is trained (SANA-WM GeekNews summary, "Core design and generation
 * pipeline": 64 H100 GPUs over 15 days), so the recurrence above needs its
 * gradient.  Given dL/do [B,H,F*L,dv] (do) and dL/dstate_out [B,H,dk,dv]
 * (dstate_out, nullable = 0) for a loss L, this returns dL/dq, dL/dk, dL/dv,
 * dL/d(alpha input) [B,H,F] and dL/d(beta input) [B,H,F*L] (with respect to
 * the logits a, b when gates_are_logits, else the gate values), and
 * dL/dstate_in [B,H,dk,dv] (also when state_in is NULL: the gradient with
 * respect to the zero start state).
 *
 * With the 3D RoPE (rope_grid_w > 0), q_t and k_t are rotated as in the
 * forward (k before its normalisation) and the gradients with respect to the
 * rotated vectors are rotated back by the transpose rotation.
 *
 * Reverse-mode differentiation of the forward above, one head at a time:
 *   1. Forward over the frames, keeping S_{f-1} (the state before frame f's
 *      decay) for every frame.
 *   2. Frames in reverse.  Frame f is run forward again from alpha_f S_{f-1},
 *      keeping each token's r_t = S^T khat_t - v_t; with S_f its end state,
 *      the read-out o_t = S_f^T q_t gives dq_t = S_f do_t and adds
 *      sum_t q_t do_t^T to H = dL/dS_f.  Tokens in reverse: with
 *      H = dL/dS after token t and S the state after it,
 *        S    <- S + beta khat r^T           (the state before token t: the
 *                                             update undone, exact in real
 *                                             arithmetic)
 *        g     = H^T khat                    (length d_v)
 *        dv_t  = beta g
 *        dbeta = -(g . r)
 *        dkhat = -beta (H r + S g)
 *        H    <- H - beta khat g^T           (dL/dS before token t)
 *      then dk_t from dkhat through khat = k / max(||k||, eps):
 *        dk = (dkhat - khat (khat . dkhat)) / ||k||   if ||k|| > eps,
 *        dk = dkhat / eps                             otherwise.
 *      At the frame start H = dL/d(alpha_f S_{f-1}):
 *        dalpha_f = <H, S_{f-1}>,  dL/dS_{f-1} = alpha_f H  (carried to frame f-1).
 *   3. Gate logits: dalpha/da = -alpha (1 - alpha) (alpha = 1 / (1 + e^a)),
 *      dbeta/db = beta (1 - beta).
 * The derivation is pinned by central finite differences of the forward.
 * heads: optional list of nheads flat head indices (NULL = all); only their
 * outputs are written.
 */
typedef struct {
  const float *q, *k, *v, *alpha, *beta, *d_o;
  int logits;
  const double *s_in, *ds_out;
  double *dq, *dk, *dv, *dal, *dbe, *ds_in;
  int64_t F, L, dk_, dv_, bh;
  rope_t rope;         /* 3D RoPE on q and k (k before its normalisation) */
} gdn_bwd_unit_t;

static void gdn_bwd_unit(const gdn_bwd_unit_t *u) {
  const int64_t F = u->F, L = u->L, dk = u->dk_, dv = u->dv_, N = F * L, bh = u->bh;
  const int64_t SS = dk * dv;
  const float *q = u->q + bh * N * dk, *k = u->k + bh * N * dk, *v = u->v + bh * N * dv;
  const float *al = u->alpha + bh * F, *be = u->beta + bh * N, *d_o = u->d_o + bh * N * dv;
  double *Sprev = (double *)calloc((size_t)(F * SS), sizeof(double)); /* S_{f-1} for each frame f */
  double *S = (double *)calloc((size_t)SS, sizeof(double));
  double *H = (double *)calloc((size_t)SS, sizeof(double));
  double *kh = (double *)malloc(sizeof(double) * (size_t)(L * dk)); /* the frame's khat rows */
  double *nrm = (double *)malloc(sizeof(double) * (size_t)L);
  double *r = (double *)malloc(sizeof(double) * (size_t)(L * dv));   /* the frame's residuals */
  double *g = (double *)malloc(sizeof(double) * (size_t)dv);
  double *dkh = (double *)malloc(sizeof(double) * (size_t)dk);
  double *qr = (double *)malloc(sizeof(double) * (size_t)dk); /* q_t (rotated with the embedding) */
  double *grot = (double *)malloc(sizeof(double) * (size_t)dk); /* a gradient with respect to a rotated vector */
  if (u->s_in)
    for (int64_t e = 0; e < SS; ++e) S[e] = u->s_in[bh * SS + e];
  /* khat_t and ||k_t|| for token t of frame f (index tl in the frame) */
#define GDN_BWD_KEY(f, tl)                                                        \
  do {                                                                            \
    const float *kt = k + ((f) * L + (tl)) * dk;                                  \
    double *kx = kh + (tl) * dk;                                                  \
    if (u->rope.on)                                                               \
      rope3d(kt, dk, u->rope.frame_offset + (f), (tl) / u->rope.grid_w,           \
             (tl) % u->rope.grid_w, u->rope.base, kx);                            \
    else                                                                          \
      for (int64_t i = 0; i < dk; ++i) kx[i] = (double)kt[i];                     \
    double ss = 0.0;                                                              \
    for (int64_t i = 0; i < dk; ++i) ss += kx[i] * kx[i];                         \
    const double n_ = sqrt(ss);                                                   \
    const double den = n_ > GDN_KEY_NORM_EPS ? n_ : GDN_KEY_NORM_EPS;             \
    nrm[tl] = n_;                                                                 \
    for (int64_t i = 0; i < dk; ++i) kx[i] = kx[i] / den;                         \
  } while (0)
  /* 1. forward over the frames */
  for (int64_t f = 0; f < F; ++f) {
    memcpy(Sprev + f * SS, S, sizeof(double) * (size_t)SS);
    const double alpha = u->logits ? gate_alpha((double)al[f]) : (double)al[f];
    for (int64_t e = 0; e < SS; ++e) S[e] *= alpha;
    for (int64_t tl = 0; tl < L; ++tl) {
      GDN_BWD_KEY(f, tl);
      const double *x = kh + tl * dk;
      const double beta = u->logits ? gate_beta((double)be[f * L + tl]) : (double)be[f * L + tl];
      for (int64_t j = 0; j < dv; ++j) {
        double p = 0.0;
        for (int64_t i = 0; i < dk; ++i) p += S[i * dv + j] * x[i];
        r[j] = p - (double)v[(f * L + tl) * dv + j];
      }
      for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= beta * x[i] * r[j];
    }
  }
  /* 2. frames in reverse; H = dL/dS after the last frame */
  if (u->ds_out)
    for (int64_t e = 0; e < SS; ++e) H[e] = u->ds_out[bh * SS + e];
  for (int64_t f = F - 1; f >= 0; --f) {
    const double alpha = u->logits ? gate_alpha((double)al[f]) : (double)al[f];
    for (int64_t e = 0; e < SS; ++e) S[e] = alpha * Sprev[f * SS + e];
    for (int64_t tl = 0; tl < L; ++tl) { /* the frame again, keeping khat and r */
      GDN_BWD_KEY(f, tl);
      const double *x = kh + tl * dk;
      double *rt = r + tl * dv;
      const double beta = u->logits ? gate_beta((double)be[f * L + tl]) : (double)be[f * L + tl];
      for (int64_t j = 0; j < dv; ++j) {
        double p = 0.0;
        for (int64_t i = 0; i < dk; ++i) p += S[i * dv + j] * x[i];
        rt[j] = p - (double)v[(f * L + tl) * dv + j];
      }
      for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] -= beta * x[i] * rt[j];
    }
    /* read-out: o_t = S_f^T q_t (q_t rotated with the embedding; its gradient rotated back) */
    for (int64_t tl = 0; tl < L; ++tl) {
      const int64_t t = f * L + tl;
      if (u->rope.on)
        rope3d(q + t * dk, dk, u->rope.frame_offset + f, tl / u->rope.grid_w, tl % u->rope.grid_w, u->rope.base, qr);
      else
        for (int64_t i = 0; i < dk; ++i) qr[i] = (double)q[t * dk + i];
      for (int64_t i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < dv; ++j) acc += S[i * dv + j] * (double)d_o[t * dv + j];
        grot[i] = acc;
      }
      if (u->rope.on)
        rope3d_rot(grot, dk, u->rope.frame_offset + f, tl / u->rope.grid_w, tl % u->rope.grid_w, u->rope.base, -1.0,
                   u->dq + (bh * N + t) * dk);
      else
        for (int64_t i = 0; i < dk; ++i) u->dq[(bh * N + t) * dk + i] = grot[i];
      for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) H[i * dv + j] += qr[i] * (double)d_o[t * dv + j];
    }
    /* tokens in reverse */
    for (int64_t tl = L - 1; tl >= 0; --tl) {
      const int64_t t = f * L + tl;
      const double *x = kh + tl * dk, *rt = r + tl * dv;
      const double beta = u->logits ? gate_beta((double)be[t]) : (double)be[t];
      for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += beta * x[i] * rt[j];
      for (int64_t j = 0; j < dv; ++j) {
        double p = 0.0;
        for (int64_t i = 0; i < dk; ++i) p += H[i * dv + j] * x[i];
        g[j] = p;
        u->dv[(bh * N + t) * dv + j] = beta * p;
      }
      double gr = 0.0;
      for (int64_t j = 0; j < dv; ++j) gr += g[j] * rt[j];
      const double dbeta = -gr;
      for (int64_t i = 0; i < dk; ++i) {
        double hr = 0.0, sg = 0.0;
        for (int64_t j = 0; j < dv; ++j) {
          hr += H[i * dv + j] * rt[j];
          sg += S[i * dv + j] * g[j];
        }
        dkh[i] = -beta * (hr + sg);
      }
      for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) H[i * dv + j] -= beta * x[i] * g[j];
      if (nrm[tl] > GDN_KEY_NORM_EPS) {
        double kd = 0.0;
        for (int64_t i = 0; i < dk; ++i) kd += x[i] * dkh[i];
        for (int64_t i = 0; i < dk; ++i) grot[i] = (dkh[i] - x[i] * kd) / nrm[tl];
      } else {
        for (int64_t i = 0; i < dk; ++i) grot[i] = dkh[i] / GDN_KEY_NORM_EPS;
      }
      /* grot = dL/d(the rotated key); the key's own gradient is its transpose rotation */
      if (u->rope.on)
        rope3d_rot(grot, dk, u->rope.frame_offset + f, tl / u->rope.grid_w, tl % u->rope.grid_w, u->rope.base, -1.0,
                   u->dk + (bh * N + t) * dk);
      else
        for (int64_t i = 0; i < dk; ++i) u->dk[(bh * N + t) * dk + i] = grot[i];
      u->dbe[bh * N + t] = u->logits ? dbeta * beta * (1.0 - beta) : dbeta;
    }
    /* frame start: H = dL/d(alpha_f S_{f-1}) */
    double da = 0.0;
    for (int64_t e = 0; e < SS; ++e) da += H[e] * Sprev[f * SS + e];
    u->dal[bh * F + f] = u->logits ? da * (-alpha * (1.0 - alpha)) : da;
    for (int64_t e = 0; e < SS; ++e) H[e] *= alpha;
  }
#undef GDN_BWD_KEY
  if (u->ds_in)
    for (int64_t e = 0; e < SS; ++e) u->ds_in[bh * SS + e] = H[e];
  free(Sprev);
  free(S);
  free(H);
  free(kh);
  free(nrm);
  free(r);
  free(g);
  free(dkh);
  free(qr);
  free(grot);
}

typedef struct {
  gdn_bwd_unit_t *units;
  int64_t n, next;
  pthread_mutex_t mu;
} bwd_pool_t;

static void *gdn_bwd_worker(void *p) {
  bwd_pool_t *pl = (bwd_pool_t *)p;
  for (;;) {
    pthread_mutex_lock(&pl->mu);
    int64_t i = pl->next++;
    pthread_mutex_unlock(&pl->mu);
    if (i >= pl->n) return NULL;
    gdn_bwd_unit(&pl->units[i]);
  }
}

int oracle_gdn_bwd(const float *q, const float *k, const float *v, const float *alpha, const float *beta,
                   int gates_are_logits, const double *state_in, const float *d_o, const double *dstate_out,
                   double *dq, double *dk, double *dv, double *dalpha, double *dbeta, double *dstate_in,
                   int64_t B, int64_t H, int64_t F, int64_t L, int64_t dk_, int64_t dv_,
                   const int64_t *heads, int64_t nheads, int nthreads, int64_t rope_grid_w,
                   int64_t rope_frame_offset, double rope_base) {
  if (B < 0 || H < 0 || F < 0 || L < 0 || dk_ <= 0 || dv_ <= 0) return 1;
  if (!dq || !dk || !dv || !dalpha || !dbeta) return 1;
  if (rope_grid_w > 0 && (dk_ % 2 || L % rope_grid_w)) return 1;
  const int64_t n = heads ? nheads : B * H;
  if (n <= 0) return 0;
  gdn_bwd_unit_t *units = (gdn_bwd_unit_t *)calloc((size_t)n, sizeof(gdn_bwd_unit_t));
  for (int64_t h = 0; h < n; ++h) {
    gdn_bwd_unit_t *u = &units[h];
    u->q = q; u->k = k; u->v = v; u->alpha = alpha; u->beta = beta; u->d_o = d_o;
    u->logits = gates_are_logits; u->s_in = state_in; u->ds_out = dstate_out;
    u->dq = dq; u->dk = dk; u->dv = dv; u->dal = dalpha; u->dbe = dbeta; u->ds_in = dstate_in;
    u->F = F; u->L = L; u->dk_ = dk_; u->dv_ = dv_;
    u->bh = heads ? heads[h] : h;
    u->rope.on = rope_grid_w > 0;
    u->rope.grid_w = rope_grid_w > 0 ? rope_grid_w : 1;
    u->rope.frame_offset = rope_frame_offset;
    u->rope.base = rope_base;
  }
  bwd_pool_t pl;
  pl.units = units; pl.n = n; pl.next = 0;
  pthread_mutex_init(&pl.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > n) nthreads = (int)n;
  if (nthreads > 512) nthreads = 512;
  pthread_t th[512];
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, gdn_bwd_worker, &pl);
  gdn_bwd_worker(&pl);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&pl.mu);
  free(units);
  return 0;
}

/*
 * Block-causal ReLU linear attention, one (b, h) head.  Layouts: q, k
 * [B,H,F*L,dk]; v [B,H,F*L,dv]; kv_in/kv_out [B,H,dk,dv]; z_in/z_out [B,H,dk]
 * (nullable); o [B,H,F*L,dv].
 */
typedef struct {
  const float *q, *k, *v;
  const double *kv_in, *z_in;
  double *kv_out, *z_out, *o;
  int64_t F, L, dk, dv;
  double eps;
  int64_t bh;
} relu_unit_t;

static void relu_unit(const relu_unit_t *u) {
  const int64_t F = u->F, L = u->L, dk = u->dk, dv = u->dv, N = F * L, bh = u->bh;
  double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
  double *z = (double *)malloc(sizeof(double) * (size_t)dk);
  double *rq = (double *)malloc(sizeof(double) * (size_t)dk);
  const float *qh = u->q + bh * N * dk, *kh = u->k + bh * N * dk, *vh = u->v + bh * N * dv;
  for (int64_t e = 0; e < dk * dv; ++e) S[e] = u->kv_in ? u->kv_in[bh * dk * dv + e] : 0.0;
  for (int64_t i = 0; i < dk; ++i) z[i] = u->z_in ? u->z_in[bh * dk + i] : 0.0;
  for (int64_t f = 0; f < F; ++f) {
    for (int64_t t = f * L; t < (f + 1) * L; ++t)
      for (int64_t i = 0; i < dk; ++i) {
        double rk = (double)kh[t * dk + i];
        if (rk < 0.0) rk = 0.0;
        z[i] += rk;
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += rk * (double)vh[t * dv + j];
      }
    for (int64_t t = f * L; t < (f + 1) * L; ++t) {
      double den = 0.0;
      for (int64_t i = 0; i < dk; ++i) {
        double x = (double)qh[t * dk + i];
        rq[i] = x > 0.0 ? x : 0.0;
        den += rq[i] * z[i];
      }
      den += u->eps;
      for (int64_t j = 0; j < dv; ++j) {
        double num = 0.0;
        for (int64_t i = 0; i < dk; ++i) num += rq[i] * S[i * dv + j];
        u->o[(bh * N + t) * dv + j] = num / den;
      }
    }
  }
  if (u->kv_out) memcpy(u->kv_out + bh * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
  if (u->z_out) memcpy(u->z_out + bh * dk, z, sizeof(double) * (size_t)dk);
  free(S);
  free(z);
  free(rq);
}

typedef struct {
  relu_unit_t *units;
  int64_t n;
  int64_t next;
  pthread_mutex_t mu;
} relu_pool_t;

static void *relu_worker(void *p) {
  relu_pool_t *pl = (relu_pool_t *)p;
  for (;;) {
    pthread_mutex_lock(&pl->mu);
    int64_t i = pl->next++;
    pthread_mutex_unlock(&pl->mu);
    if (i >= pl->n) return NULL;
    relu_unit(&pl->units[i]);
  }
}

/*
 * Block-causal ReLU linear attention over all B*H heads; nthreads threads take
 * whole heads (heads are independent, so this changes no arithmetic).
 */
int oracle_relu_la(const float *q, const float *k, const float *v, const double *kv_in,
                   const double *z_in, double *kv_out, double *z_out, double *o,
                   int64_t B, int64_t H, int64_t F, int64_t L, int64_t dk, int64_t dv, double eps,
                   int nthreads) {
  if (B < 0 || H < 0 || F < 0 || L < 0 || dk <= 0 || dv <= 0) return 1;
  const int64_t n = B * H;
  if (n == 0) return 0;
  relu_unit_t *units = (relu_unit_t *)calloc((size_t)n, sizeof(relu_unit_t));
  for (int64_t bh = 0; bh < n; ++bh) {
    relu_unit_t *u = &units[bh];
    u->q = q; u->k = k; u->v = v; u->kv_in = kv_in; u->z_in = z_in;
    u->kv_out = kv_out; u->z_out = z_out; u->o = o;
    u->F = F; u->L = L; u->dk = dk; u->dv = dv; u->eps = eps; u->bh = bh;
  }
  relu_pool_t pl;
  pl.units = units; pl.n = n; pl.next = 0;
  pthread_mutex_init(&pl.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > n) nthreads = (int)n;
  if (nthreads > 512) nthreads = 512;
  pthread_t th[512];
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, relu_worker, &pl);
  relu_worker(&pl);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&pl.mu);
  free(units);
  return 0;
}

/*
 * Causal temporal convolution of one block of frames with the block-boundary
 * cache (SANA-Video talk, causal Mix-FFN passage: in training a zero token
 * separates two blocks so that block one cannot see block two, and block
 * two is prefixed with block one's last token; both are removed after the
 * convolution).  The library's reading: a depthwise convolution of kernel 3
 * along the frame axis, per latent position n and channel c,
 *   y[f][n][c] = w[c][0] x[f-1][n][c] + w[c][1] x[f][n][c] + w[c][2] x[f+1][n][c] + bias[c]
 * where x[-1] is the cached last frame of the previous block (zero without
 * one) and x[F] is zero (the block cannot see the next one).  cache_out is
 * the block's last frame.  Layouts: x, y [B, F, HW, C]; cache [B, HW, C];
 * w [C][3]; bias [C] (nullable).
 */
int oracle_temporal_conv(const float *x, const float *w, const float *bias, const float *cache_in, double *y,
                         double *cache_out, int64_t B, int64_t F, int64_t HW, int64_t C) {
  if (B < 0 || F <= 0 || HW <= 0 || C <= 0) return 1;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t f = 0; f < F; ++f)
      for (int64_t n = 0; n < HW; ++n)
        for (int64_t c = 0; c < C; ++c) {
          const int64_t at = ((b * F + f) * HW + n) * C + c;
          const double prev = f > 0 ? (double)x[at - HW * C] : (cache_in ? (double)cache_in[(b * HW + n) * C + c] : 0.0);
          const double next = f + 1 < F ? (double)x[at + HW * C] : 0.0;
          double acc = (double)w[c * 3 + 0] * prev + (double)w[c * 3 + 1] * (double)x[at] + (double)w[c * 3 + 2] * next;
          if (bias) acc += (double)bias[c];
          y[at] = acc;
        }
  if (cache_out)
    for (int64_t b = 0; b < B; ++b)
      for (int64_t n = 0; n < HW; ++n)
        for (int64_t c = 0; c < C; ++c)
          cache_out[(b * HW + n) * C + c] = (double)x[((b * F + F - 1) * HW + n) * C + c];
  return 0;
}

/*
 * Windowed block-causal softmax attention: the softmax layers that SANA-WM's
 * hybrid interleaves with the frame-wise Gated DeltaNet (GeekNews summary of
 * SANA-WM, "Core design and generation pipeline": periodic softmax; the
 * Vietnamese post: Gated DeltaNet for most of the sequence, softmax windows
 * in between; SANA-Video talk: long videos keep softmax inside a sliding
 * window).  The library's reading: token t of frame f attends to every token
 * of frames max(0, f-W+1) .. f (its own frame in full, as in the linear
 * modes), o_t = sum_s softmax_s(scale q_t . k_s) v_s.  Per (b, h) and per
 * frame f the key set is shared; rows of o outside frame_mask (if given, one
 * byte per frame) are left untouched.  q, k: [B, H, F*L, dk]; v, o: [B, H, F*L, dv].
 */
typedef struct {
  const float *q, *k, *v;
  double *o;
  int64_t BH, F, L, dk, dv, W;
  double scale;
  const unsigned char *frame_mask;
  int64_t next; /* shared work counter over (bh, f) */
  pthread_mutex_t mu;
} sw_job_t;

static void sw_unit(sw_job_t *j, int64_t bh, int64_t f) {
  const int64_t N = j->F * j->L;
  const int64_t f0 = f - j->W + 1 < 0 ? 0 : f - j->W + 1;
  const int64_t nk = (f - f0 + 1) * j->L;
  double *sc = (double *)malloc(sizeof(double) * (size_t)nk);
  for (int64_t t = f * j->L; t < (f + 1) * j->L; ++t) {
    const float *qt = j->q + (bh * N + t) * j->dk;
    double m = -INFINITY;
    for (int64_t s = 0; s < nk; ++s) {
      const float *ks = j->k + (bh * N + f0 * j->L + s) * j->dk;
      double acc = 0.0;
      for (int64_t i = 0; i < j->dk; ++i) acc += (double)qt[i] * (double)ks[i];
      sc[s] = acc * j->scale;
      if (sc[s] > m) m = sc[s];
    }
    double den = 0.0;
    for (int64_t s = 0; s < nk; ++s) {
      sc[s] = exp(sc[s] - m);
      den += sc[s];
    }
    double *ot = j->o + (bh * N + t) * j->dv;
    for (int64_t c = 0; c < j->dv; ++c) ot[c] = 0.0;
    for (int64_t s = 0; s < nk; ++s) {
      const float *vs = j->v + (bh * N + f0 * j->L + s) * j->dv;
      const double p = sc[s] / den;
      for (int64_t c = 0; c < j->dv; ++c) ot[c] += p * (double)vs[c];
    }
  }
  free(sc);
}

static void *sw_worker(void *arg) {
  sw_job_t *j = (sw_job_t *)arg;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    const int64_t u = j->next++;
    pthread_mutex_unlock(&j->mu);
    if (u >= j->BH * j->F) break;
    const int64_t bh = u / j->F, f = u % j->F;
    if (j->frame_mask && !j->frame_mask[f]) continue;
    sw_unit(j, bh, f);
  }
  return NULL;
}

int oracle_softmax_window(const float *q, const float *k, const float *v, double *o, int64_t B, int64_t H, int64_t F,
                          int64_t L, int64_t dk, int64_t dv, int64_t W, double scale,
                          const unsigned char *frame_mask, int nthreads) {
  if (B <= 0 || H <= 0 || F <= 0 || L <= 0 || dk <= 0 || dv <= 0 || W <= 0) return 1;
  sw_job_t j = {q, k, v, o, B * H, F, L, dk, dv, W, scale, frame_mask, 0};
  pthread_mutex_init(&j.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, sw_worker, &j);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&j.mu);
  return 0;
}
