// Frame-wise Gated DeltaNet on tcgen05 tensor cores (bf16 q, k, v; fp32 state).
//
// Source of the method: SANA-WM GeekNews summary, "Core design and generation
// pipeline" (frame-wise Gated DeltaNet); dothoosh.com SANA-WM article (fixed-
// size recurrent state).  Update rule per token: S <- S - beta khat (S^T khat
// - v)^T after a per-frame decay S <- alpha S; every token of a frame reads
// o = S^T q with the state after the whole frame.
//
// Work unit = one (b, h, f) frame, taken from a ticket counter (f-major) by a
// persistent CTA; with P segments per frame (few frames, e.g. a streaming
// call) a unit is one run of consecutive chunks of a frame, and the map below
// is the segment's, chained through the frame's segments in order (alpha_f on
// the first only), every segment reading out against the frame's last state.
// For its frame the CTA builds the frame map
//     S_f = A_f (alpha_f S_{f-1}) + B_f,
// A_f = ordered product of (I - beta_t khat_t khat_t^T), B_f = the frame's
// update from a zero state, by running the delta rule on Y = [A | B] from
// [I | 0] with targets [0 | V], chunked 64 tokens at a time in the UT form
//     Y <- Y + W^T ([0 | V] - Khat Y),   W^T = Khat^T T,
//     T = (I + N)^-1 diag(beta),  N = strict_lower(diag(beta) Khat Khat^T),
// kept transposed in TMEM (lanes = columns of A and B, fp32).  Only the
// d x d chain step S_f = ... waits on the previous frame's published state.
// Then O_f = Q_f S_f.
//
// Warp roles (512 threads):
//   warps 0-3, 4-7  tile chains A and B, one per 128-lane TMEM tile of Y^T
//                   (rows of A^T, rows of B^T).  Per chunk: R^T = -Y^T Khat^T
//                   on tcgen05, R^T back into TMEM as fp16 pairs, Y^T += R^T W
//                   (+ V^T W for tile B, the [0 | V] target) with R^T read from
//                   TMEM, and an fp16 copy of Y^T in shared memory for the next
//                   chunk.  The first chunk of a frame starts from Y = [I | 0],
//                   so its R^T is -Khat^T and [0 | V] directly.  Together the
//                   eight warps run the chain step and publish S_f; in the
//                   read-out thread 0 issues the MMAs and warps 4-7 store O.
//   warps 8-11, 12-15  two prep groups for even and odd chunks: gates beta,
//                   key normalisation (fp16 khat), v to fp16, Gram matrix Khat
//                   Khat^T on tcgen05, T by blocked inversion of the unit lower
//                   triangular I + N (16 x 16 fp32 blocks on CUDA cores), W^T =
//                   Khat^T T on tcgen05, fp16 W for the chains.
// k and v reach a 3-slot ring by TMA, issued by the chains as soon as a slot's
// last MMA has completed (chunk c + 3 after chunk c; a frame's first three
// chunks as soon as its ticket is taken).
// The frame chain passes S_f between CTAs as fp16 rows S_f^T[j][l] (one bulk
// store out, 16-byte loads in); alpha_f is folded into the fp16 copy of A_f.
// The read-out takes S_f as a bf16 high/low pair (two MMAs on bf16 q) in
// 64-token tiles: thread 0 issues the MMAs one tile ahead while warps 4-7 move
// the previous tile through shared memory to a bulk store.
// Operands that are not exact in bf16 (khat, v after the cast, Y, R, T, W, A_f,
// S_{f-1}) enter the tensor cores as fp16 (11-bit significands); all
// accumulation is fp32.
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {

constexpr int kChain = 256;      // warps 0-7
constexpr int kGThreads = 512;   // + two prep warpgroups
constexpr int kC = 64;           // tokens per chunk
constexpr int kSlots = 3;        // chunks in flight (k, v, W)
constexpr int kQTok = 64;        // tokens per read-out tile

// shared memory map (bytes from the 1024-aligned base)
constexpr uint32_t OFF_MIRROR = 0;       // 64 KB: Y^T as fp16, [tile][k-block][128 rows][128 B]
constexpr uint32_t OFF_SLOT = 65536;     // 3 slots of 48 KB:
constexpr uint32_t SLOT_BYTES = 49152;
constexpr uint32_t SL_KHAT = 0;          //   khat fp16 (TMA'd bf16 k, normalised in place) [k-block][64 t][128 B]
constexpr uint32_t SL_V = 16384;         //   v fp16 (TMA'd bf16, cast in place) [j-block][64 t][128 B]
constexpr uint32_t SL_W = 32768;         //   W fp16, [128 rows i][128 B (64 t)]; fp32 16 x 16 blocks of the
                                         //   inversion while the prep group works on the slot
constexpr uint32_t OFF_T = OFF_SLOT + kSlots * SLOT_BYTES;  // 2 x 8 KB: T fp16 [64 rows u][128 B (64 t)]
constexpr uint32_t OFF_BAR = OFF_T + 2 * 8192;              // barriers and small state
// frame-end aliases: the tile-B half of the mirror is free after the last
// chunk, the tile-A half once the chain step has read alpha A_f^T
constexpr uint32_t OFF_STAGE = OFF_MIRROR;        // 32 KB: fp16 rows of S_f, then fp32 rows of O (64 tokens)
constexpr uint32_t OFF_QB = OFF_MIRROR + 32768;   // two q tiles (bf16) [k-block][64 t][128 B], 16 KB each

struct Bars {
  uint64_t kv_full[kSlots];     // TMA bytes of k and v
  uint64_t khat_ready[kSlots];  // prep: khat normalised
  uint64_t w_ready[kSlots];     // prep: W written
  uint64_t slot_free[kSlots];   // the last MMA of each tile chain on the slot (2 arrivals)
  uint64_t g_bar[2];            // per prep group: its MMAs
  uint64_t mma_bar[2];          // per tile chain
  uint64_t fr_bar;              // frame-level MMAs (chain step)
  uint64_t q_full[2];           // read-out: q tile in buffer b
  uint64_t q_conv[2];           // read-out with the position embedding: q tile b rotated, as fp16
  uint64_t o_full[2];           // read-out: the MMAs into O buffer b are done
  uint64_t o_free[2];           // read-out: the epilogue has read O buffer b
  uint64_t tkt_bar[2];          // chain group -> prep groups: next frame's ticket
  uint32_t tmem_base;
  int abort;
  uint32_t loads;               // chunks whose k, v loads have been issued
  int ticket_ring[4];
  __align__(16) float beta[kSlots][64];
};
constexpr size_t kGdnSmemBytes = OFF_BAR + sizeof(Bars) + 1024;
static_assert(kGdnSmemBytes <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t TM_Y = 0;     // Y^T: tile A [0,128), tile B [128,256); read-out: S_f^T as bf16 pairs,
                                 // high parts [0,64), low parts [64,128)
constexpr uint32_t TM_R = 256;   // R^T: tile A [256,320), tile B [320,384); chain step: S^T pairs
                                 // [256,320); read-out: O buffers, 64 columns each, [256,320) and
                                 // [320,384)
constexpr uint32_t TM_P = 384;   // prep group g: [384 + 64 g, 448 + 64 g): Gram matrix, then W^T

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// 16 fp32 values -> two 16-byte fp16 chunks of a 128B-swizzled row.
__device__ __forceinline__ void store_row16_f16(uint8_t *tile, uint32_t row, uint32_t col0, const float (&r)[16]) {
  uint4 a = make_uint4(pack_h2(r[0], r[1]), pack_h2(r[2], r[3]), pack_h2(r[4], r[5]), pack_h2(r[6], r[7]));
  uint4 b = make_uint4(pack_h2(r[8], r[9]), pack_h2(r[10], r[11]), pack_h2(r[12], r[13]), pack_h2(r[14], r[15]));
  *reinterpret_cast<uint4 *>(tile + sw128_offset(row, col0)) = a;
  *reinterpret_cast<uint4 *>(tile + sw128_offset(row, col0 + 8)) = b;
}

// bf16 x 8 -> fp16 x 8 (one 16-byte chunk); amax takes the largest |value|
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 u, float &amax) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v2 = __bfloat1622float2(h[e]);
    amax = fmaxf(amax, fmaxf(fabsf(v2.x), fabsf(v2.y)));
    o[e] = pack_h2(v2.x, v2.y);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Largest finite fp16 value: an operand at or beyond it (or NaN) leaves the fp16 range.
constexpr float kF16Max = 65504.0f;

// ---------------------------------------------------------------- blocked inversion
// The 64 x 64 unit lower triangular I + N is handled as 4 x 4 blocks of 16 x 16.
// Shared-memory scratch (the slot's W area, 16 KB): blocks of 1 KB, fp32,
// row r = 16 floats whose four float4 groups are permuted by q ^ ((r >> 1) & 3)
// (eight consecutive rows of one group fall in distinct bank groups).
//   lblk(i, j), i >= j (10 blocks): N's block (i, j); the diagonal ones are
//              replaced by D_i = (I + N_ii)^-1, the others (once E is formed)
//              by block (i, j) of (I + N)^-1;
//   iblk(i, j), i > j (6 blocks): E_ij = D_i N_ij.
// With Linv_jj = D_j, block (i, j) of the inverse is -sum_{k=j}^{i-1} E_ik Linv_kj
// (forward block substitution), computed by distance i - j = 1, 2, 3.
__device__ __forceinline__ int bofs(int r, int q) { return r * 16 + ((q ^ ((r >> 1) & 3)) << 2); }
__device__ __forceinline__ float *lblk(float *scr, int i, int j) { return scr + (i * (i + 1) / 2 + j) * 256; }
__device__ __forceinline__ float *iblk(float *scr, int i, int j) {
  const int d = i - j;
  return scr + (10 + (d - 1) * (8 - d) / 2 + j) * 256;
}
__device__ __forceinline__ float4 ld_blk4(const float *b, int r, int q) {
  return *reinterpret_cast<const float4 *>(b + bofs(r, q));
}
__device__ __forceinline__ void st_blk4(float *b, int r, int q, float4 v) {
  *reinterpret_cast<float4 *>(b + bofs(r, q)) = v;
}
__device__ __forceinline__ void fma4(float4 &acc, float a, float4 b) {
  acc.x = fmaf(a, b.x, acc.x);
  acc.y = fmaf(a, b.y, acc.y);
  acc.z = fmaf(a, b.z, acc.z);
  acc.w = fmaf(a, b.w, acc.w);
}
// acc += (row r of A) x (columns 4q .. 4q+3 of B), 16 x 16 blocks.  The rows of
// B are loaded eight at a time ahead of their FMAs, into two accumulators, so
// that one thread keeps several shared-memory loads in flight.
__device__ __forceinline__ void blk_row_mul(float4 &acc, const float *A, const float *B, int r, int q) {
  float4 a4[4], b[8];
#pragma unroll
  for (int g = 0; g < 4; ++g) a4[g] = ld_blk4(A, r, g);
  float4 acc1 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int s = 0; s < 8; ++s) b[s] = ld_blk4(B, 8 * h + s, q);
#pragma unroll
    for (int s = 0; s < 8; s += 4) {
      const float4 a = a4[2 * h + s / 4];
      fma4(acc, a.x, b[s]);
      fma4(acc1, a.y, b[s + 1]);
      fma4(acc, a.z, b[s + 2]);
      fma4(acc1, a.w, b[s + 3]);
    }
  }
  acc.x += acc1.x;
  acc.y += acc1.y;
  acc.z += acc1.z;
  acc.w += acc1.w;
}
__device__ __forceinline__ float4 neg4(float4 v) { return make_float4(-v.x, -v.y, -v.z, -v.w); }

// 3D RoPE of one token: where its time, height and width rows start in the angle
// table (time [F][dt/2], height [L/gw][dh/2], width [gw][dh/2]), each less the
// pair index of its band's first pair, so that pair j of any band is entry off + j.
// The division by the grid width is taken once per token, not once per pair.
struct RopeTok {
  int t_off, h_off, w_off;
};
__device__ __forceinline__ RopeTok rope_tok(int f, int tf, const GdnParams &p) {
  const int row = tf / p.rope_gw, col = tf - row * p.rope_gw;
  const int ht = p.F * (p.rope_dt / 2), hp = p.rope_dh / 2;
  return {f * (p.rope_dt / 2), ht + row * hp - p.rope_dt / 2,
          ht + (p.L / p.rope_gw) * hp + col * hp - (p.rope_dt + p.rope_dh) / 2};
}
// The pair (dd, dd + 1) (dd even) rotated by its angle: the band is a select, not a
// branch (lanes of a warp hold pairs of different bands).
__device__ __forceinline__ float2 rope_at(float2 x, int dd, const RopeTok &r, const GdnParams &p) {
  const int off = dd < p.rope_dt ? r.t_off : (dd < p.rope_dt + p.rope_dh ? r.h_off : r.w_off);
  const float2 cs = __ldg(p.rope_tab + off + (dd >> 1));
  return make_float2(fmaf(x.x, cs.x, -x.y * cs.y), fmaf(x.x, cs.y, x.y * cs.x));
}

// kSeg: frames split into p.segs chunk segments (else one unit per frame; the
// segment arithmetic folds away)
// kRope: the 3D rotary position embedding on q and k (a separate instantiation,
// so that the kernel without it carries none of its code)
// kSave: the backward's recompute: every frame's map A_f^T and end state S_f
// go to p.save_maps / p.save_states (fp32) and there is no read-out
template <bool kSeg, bool kRope, bool kSave = false>
__global__ void __launch_bounds__(kGThreads, 1)
    gdn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, GdnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars &bar = *reinterpret_cast<Bars *>(sm + OFF_BAR);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const int BH = p.B * p.H;
  const int P = kSeg ? p.segs : 1;     // chunk segments per frame
  const long units = (long)BH * F * P; // tickets
  const long N = (long)F * L;
  const unsigned long long lim = p.spin_limit_ns;
  const int nkd = dk / 16;            // k-steps over d_k
  const int nch = (L + kC - 1) / kC;  // chunks per frame
  volatile int *abort_flag = &bar.abort;
  // ticket (f-major, then segment, then b*H + h) -> frame, segment, head and
  // the segment's chunks [c0, c1)
  struct Unit {
    int f, s, bh, c0, c1;
  };
  auto unit_of = [&](int tk) -> Unit {
    Unit u;
    if (!kSeg) {
      u.f = tk / BH;
      u.s = 0;
      u.bh = tk - u.f * BH;
      u.c0 = 0;
      u.c1 = nch;
      return u;
    }
    u.f = tk / (BH * P);
    const int r = tk - u.f * BH * P;
    u.s = r / BH;
    u.bh = r - u.s * BH;
    u.c0 = u.s * nch / P;
    u.c1 = (u.s + 1) * nch / P;
    return u;
  };

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar.kv_full[s], 1);
      mbar_init(&bar.khat_ready[s], 1);
      mbar_init(&bar.w_ready[s], 1);
      mbar_init(&bar.slot_free[s], 2);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.g_bar[s], 1);
      mbar_init(&bar.mma_bar[s], 1);
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_conv[s], 1);
      mbar_init(&bar.o_full[s], 1);
      mbar_init(&bar.o_free[s], 1);
      mbar_init(&bar.tkt_bar[s], 1);
    }
    mbar_init(&bar.fr_bar, 1);
    bar.abort = 0;
    bar.loads = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  if (warp == 0) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  // Issue the k, v loads of chunk c of frame (f, bh), the g-th chunk of this
  // CTA, into slot g % 3 once the slot's previous chunk is done with it.
  // Called by one thread; false on a timeout.
  auto issue_kv = [&](uint32_t gg, int f, int bh, int c) -> bool {
    const int s = (int)(gg % kSlots);
    if (!mbar_wait(&bar.slot_free[s], ((gg / kSlots) & 1u) ^ 1u, lim)) return false;
    uint8_t *slot = sm + OFF_SLOT + s * SLOT_BYTES;
    const int t0 = c * kC;
    mbar_expect_tx(&bar.kv_full[s], 32768);
    tma_load_4d(slot + SL_KHAT, &tmap_k, &bar.kv_full[s], 0, t0, f, bh);
    tma_load_4d(slot + SL_KHAT + 8192, &tmap_k, &bar.kv_full[s], 64, t0, f, bh);
    tma_load_4d(slot + SL_V, &tmap_v, &bar.kv_full[s], 0, t0, f, bh);
    tma_load_4d(slot + SL_V + 8192, &tmap_v, &bar.kv_full[s], 64, t0, f, bh);
    bar.loads = gg + 1;
    return true;
  };
  // the first (up to) three chunks of ticket tk's unit, the g0-th chunk on
  auto issue_frame_kv = [&](int tk, uint32_t g0) -> bool {
    if (tk < 0) return true;
    const Unit u = unit_of(tk);
    for (int c = u.c0; c < u.c1 && c < u.c0 + kSlots; ++c)
      if (!issue_kv(g0 + (c - u.c0), u.f, u.bh, c)) return false;
    return true;
  };

  if (warp >= 8) {
    // ============================================================ prep groups
    regs_dec<120>();  // the block launches with 512 x 128; the chains take 2 x 128 x 136
    const int grp = (warp - 8) >> 2;     // 0: even chunks, 1: odd chunks
    const int pt = tid - kChain - 128 * grp;  // 0..127
    const int pbar = 2 + grp;            // named barrier of the group
    const uint32_t tmP = tmem + TM_P + 64 * grp;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint8_t *tbuf = sm + OFF_T + grp * 8192;
    uint32_t gph = 0;  // phase of g_bar[grp]
    uint32_t g = 0;
    bool stop = false;
    auto group_fail = [&](int timed_out) {
      if (pt == 0 && timed_out) latch_status(p.status, GDN_ERR_TIMEOUT);  // the first code latched wins
      *abort_flag = 1;
      stop = true;
    };
    for (int k = 0; !stop; ++k) {
      {
        const int bad = pt == 0 ? !mbar_wait(&bar.tkt_bar[k & 1], (k >> 1) & 1u, lim) : 0;
        if (bar_sync_or(pbar, 128, bad || *abort_flag)) {
          group_fail(bad);
          break;
        }
      }
      const int tk = bar.ticket_ring[k & 3];
      if (tk < 0) break;
      const int c0 = unit_of(tk).c0, c1 = unit_of(tk).c1;
      for (int c = c0; c < c1; ++c, ++g) {
        if ((int)(g & 1u) != grp) continue;
        const int s = (int)(g % kSlots);
        const uint32_t ph = (g / kSlots) & 1u;
        uint8_t *slot = sm + OFF_SLOT + s * SLOT_BYTES;
        // gate of token pt of the chunk (used from step 3 on, so its load latency is hidden)
        float braw = 0.f;
        const bool bvalid = pt < 64 && c * kC + pt < L;
        if (bvalid) {  // the unit decoded again here keeps fewer registers live across the loop
          const Unit un = unit_of(tk);
          braw = p.beta[(long)un.bh * N + (long)un.f * L + c * kC + pt];
        }
        {
          const int bad = pt == 0 ? !mbar_wait(&bar.kv_full[s], ph, lim) : 0;
          if (bar_sync_or(pbar, 128, bad || *abort_flag)) {
            group_fail(bad);
            break;
          }
        }
        // 1. normalise keys in place (fp16): thread -> token pt/2, block pt%2
        {
          const int t = pt >> 1, kb = pt & 1;
          uint8_t *krow = slot + SL_KHAT + kb * 8192;
          uint4 ku[8];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) ku[ch] = *reinterpret_cast<const uint4 *>(krow + sw128_offset(t, ch * 8));
          float ssp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&ku[ch]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 v2 = __bfloat1622float2(h[e]);
              ssp[e] = fmaf(v2.x, v2.x, fmaf(v2.y, v2.y, ssp[e]));
            }
          }
          float ss = (ssp[0] + ssp[1]) + (ssp[2] + ssp[3]);
          ss += __shfl_xor_sync(0xffffffffu, ss, 1);
          const float inv = 1.0f / fmaxf(sqrtf(ss), kKeyNormEps);  // the rotation keeps the norm
          const int tf = c * kC + t;  // token index in the frame
          const bool rot = kRope && tf < L;
          RopeTok rtok = {0, 0, 0};
          if (rot) rtok = rope_tok(unit_of(tk).f, tf, p);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&ku[ch]);
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float2 v2 = __bfloat1622float2(h[e]);
              const int dd = kb * 64 + ch * 8 + 2 * e;  // this pair's first dimension
              if (rot && dd < dk) v2 = rope_at(v2, dd, rtok, p);
              o[e] = pack_h2(v2.x * inv, v2.y * inv);
            }
            *reinterpret_cast<uint4 *>(krow + sw128_offset(t, ch * 8)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(pbar, 128);
        // 2. khat ready for the chains; Gram matrix G = Khat Khat^T (lanes 0..63 = tokens)
        if (pt == 0) {
          mbar_arrive_only(&bar.khat_ready[s]);
          tc_fence_after();
          const uint32_t idg = idesc_f16(128, 64, 0, 0, 0);
          for (int kk = 0; kk < nkd; ++kk) {
            const uint32_t a = smem_u32(slot + SL_KHAT + (kk >> 2) * 8192 + (kk & 3) * 32);
            mma_f16_ss(tmP, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), idg, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bar.g_bar[grp]);
        }
        // v to fp16 in place while the Gram matrix is computed (the chains read
        // it after w_ready, which follows the fence below)
        {
          const int t = pt >> 1, kb = pt & 1;
          uint8_t *vrow = slot + SL_V + kb * 8192;
          uint4 vu[8];
          float vmax = 0.f;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) vu[ch] = *reinterpret_cast<const uint4 *>(vrow + sw128_offset(t, ch * 8));
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4 *>(vrow + sw128_offset(t, ch * 8)) = bf16x8_to_f16x8(vu[ch], vmax);
          if (!(vmax < kF16Max)) latch_status(p.status, GDN_ERR_RANGE);
        }
        {
          const int bad = pt == 0 ? !mbar_wait(&bar.g_bar[grp], gph, lim) : 0;
          gph ^= 1u;
          if (bar_sync_or(pbar, 128, bad)) {
            group_fail(bad);
            break;
          }
        }
        tc_fence_after();
        float *scr = reinterpret_cast<float *>(slot + SL_W);
        const float *bet = bar.beta[s];
        // 3. N's blocks: row t of N = beta_t G[t][u] for u < t (warps 0-1 hold TMEM lanes 0..63)
        if (pt < 64) {
          const int t = pt;
          const float bt = bvalid ? (p.gates_are_logits ? gate_beta(braw) : braw) : 0.f;
          bar.beta[s][t] = bt;
          const int ib = t >> 4, r = t & 15;
          float gr[4][16];
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) tmem_ld16(tmP + lane_off + jb * 16, gr[jb]);
          tmem_ld_wait();
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            if (jb > ib) continue;
            float *dst = lblk(scr, ib, jb);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int u = jb * 16 + q * 4;
              float4 v;
              v.x = (u + 0 < t) ? bt * gr[jb][q * 4 + 0] : 0.f;
              v.y = (u + 1 < t) ? bt * gr[jb][q * 4 + 1] : 0.f;
              v.z = (u + 2 < t) ? bt * gr[jb][q * 4 + 2] : 0.f;
              v.w = (u + 3 < t) ? bt * gr[jb][q * 4 + 3] : 0.f;
              st_blk4(dst, r, q, v);
            }
          }
        }
        tc_fence_before();
        __syncwarp();  // block k's rows of N come from the 16 threads that invert it, in one warp
        // 4. D_k = (I + N_kk)^-1: thread (k, c) solves column c by forward substitution
        if (pt < 64) {
          const int kq = pt >> 4, c = pt & 15;
          float *Dk = lblk(scr, kq, kq);
          float x[16];
#pragma unroll
          for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
          float4 cur[4], nxt[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) cur[q] = ld_blk4(Dk, 1, q);
#pragma unroll
          for (int r = 1; r < 16; ++r) {
            if (r + 1 < 16) {  // the next row's loads do not depend on x
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if (4 * q < r + 1) nxt[q] = ld_blk4(Dk, r + 1, q);
            }
            float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (4 * q < r) a[0] = fmaf(cur[q].x, x[4 * q], a[0]);
              if (4 * q + 1 < r) a[1] = fmaf(cur[q].y, x[4 * q + 1], a[1]);
              if (4 * q + 2 < r) a[2] = fmaf(cur[q].z, x[4 * q + 2], a[2]);
              if (4 * q + 3 < r) a[3] = fmaf(cur[q].w, x[4 * q + 3], a[3]);
            }
            x[r] = (r > c) ? -((a[0] + a[1]) + (a[2] + a[3])) : x[r];
#pragma unroll
            for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
          }
          __syncwarp();  // the block's 16 threads share this warp: all reads of N_kk are done
#pragma unroll
          for (int r = 0; r < 16; ++r) Dk[bofs(r, c >> 2) + (c & 3)] = x[r];
        }
        named_bar(pbar, 128);
        // 5. E_ik = D_i N_ik for the six blocks below the diagonal; item = (block,
        //    float4 column group q, row r), 64 per block
#pragma unroll 1
        for (int it = pt; it < 6 * 64; it += 128) {
          const int e = it >> 6, q = (it >> 4) & 3, r = it & 15;
          const int d = e < 3 ? 1 : (e < 5 ? 2 : 3), kq = e < 3 ? e : (e < 5 ? e - 3 : 0);
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          blk_row_mul(acc, lblk(scr, kq + d, kq + d), lblk(scr, kq + d, kq), r, q);
          st_blk4(iblk(scr, kq + d, kq), r, q, acc);
        }
        named_bar(pbar, 128);
        // 6-8. distance d = 1, 2, 3: Linv_{k+d,k} = -(E_{k+d,k} D_k + sum_{m=1}^{d-1}
        //      E_{k+d,k+m} Linv_{k+m,k}), written over N's (dead) block
#pragma unroll 1
        for (int d = 1; d <= 3; ++d) {
#pragma unroll 1
          for (int it = pt; it < (4 - d) * 64; it += 128) {
            const int kq = it >> 6, q = (it >> 4) & 3, r = it & 15;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
            for (int m = 0; m < d; ++m) blk_row_mul(acc, iblk(scr, kq + d, kq + m), lblk(scr, kq + m, kq), r, q);
            st_blk4(lblk(scr, kq + d, kq), r, q, neg4(acc));
          }
          named_bar(pbar, 128);
        }
        // 9. T[u][t] = Linv[u][t] beta_t as fp16, rows u (MN-major B operand: N = t, K = u)
        {
          const int u = pt >> 1, half = pt & 1;
          const int ub = u >> 4, r = u & 15;
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int tb = half * 2 + h2;
            float v[16];
            if (tb > ub) {
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = 0.f;
            } else {
              const float *src = lblk(scr, ub, tb);  // D_ub on the diagonal, the inverse's block below it
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 t4 = ld_blk4(src, r, q);
                const float4 b4 = *reinterpret_cast<const float4 *>(bet + tb * 16 + q * 4);
                v[4 * q] = t4.x * b4.x;
                v[4 * q + 1] = t4.y * b4.y;
                v[4 * q + 2] = t4.z * b4.z;
                v[4 * q + 3] = t4.w * b4.w;
              }
            }
            store_row16_f16(tbuf, u, tb * 16, v);
          }
        }
        fence_async_smem();
        named_bar(pbar, 128);
        // 10. W^T = Khat^T T (lanes i, columns t): A = khat read MN-major, B = T MN-major
        if (pt == 0) {
          tc_fence_after();
          const uint32_t kb0 = smem_u32(slot + SL_KHAT), tb0 = smem_u32(tbuf);
          const uint32_t idw = idesc_f16(128, 64, 0, 1, 1);
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(tmP, sdesc_sw128(kb0 + kk * 2048, 8192, 1024), sdesc_sw128(tb0 + kk * 2048, 8192, 1024), idw,
                       kk > 0 ? 1u : 0u);
          mma_commit(&bar.g_bar[grp]);
        }
        {
          const int bad = pt == 0 ? !mbar_wait(&bar.g_bar[grp], gph, lim) : 0;
          gph ^= 1u;
          if (bar_sync_or(pbar, 128, bad)) {
            group_fail(bad);
            break;
          }
        }
        tc_fence_after();
        // 11. row i of the K-major B operand W (N = i, K = t); the scratch blocks are dead
        {
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            float r[2][16];
            tmem_ld16(tmP + lane_off + hb * 32, r[0]);
            tmem_ld16(tmP + lane_off + hb * 32 + 16, r[1]);
            tmem_ld_wait();
            if (pt < dk) {
              store_row16_f16(slot + SL_W, pt, hb * 32, r[0]);
              store_row16_f16(slot + SL_W, pt, hb * 32 + 16, r[1]);
            }
          }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(pbar, 128);
        if (pt == 0) mbar_arrive_only(&bar.w_ready[s]);
      }
    }
  } else {
    // ============================================================ tile chains
    regs_inc<136>();
    const int tile = warp >> 2;           // 0: tile A (rows of A^T), 1: tile B (rows of B^T)
    const int row = tid & 127;            // TMEM lane / operand row within the tile
    const bool issuer = row == 0;         // threads 0 and 128 issue their tile's MMAs
    const int tbar = 4 + tile;            // named barrier of one tile chain (128 threads)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tmY = tmem + TM_Y + tile * 128;
    const uint32_t tmR = tmem + TM_R + tile * 64;
    uint8_t *mir = sm + OFF_MIRROR + tile * 32768;
    uint32_t tphase = 0;                  // phase of mma_bar[tile]
    uint32_t fphase = 0;                  // phase of fr_bar
    // read-out tiles over the CTA's lifetime (thread 0): q loads issued /
    // waited for, MMAs issued / waited for; tile n uses q buffer n & 1 and O
    // buffer n & 1
    uint32_t qi = 0, qw = 0, oi = 0, ow = 0;
    uint32_t rt = 0;  // read-out tiles of earlier units
    int frames = 0;
    bool failed = false;
    uint32_t g = 0;
    const uint32_t id_r = idesc_f16(128, 64, 0, 0, 0, 1, 0);   // -(Y^T) x Khat^T
    const uint32_t id_y = idesc_f16(128, dk, 0, 0, 0);          // R^T (TMEM) x W
    const uint32_t id_vw = idesc_f16(128, dk, 0, 1, 0);         // V^T (MN) x W
    const uint32_t id_kw = idesc_f16(128, dk, 0, 1, 0, 1, 0);   // -(Khat^T) (MN) x W
    const uint32_t id_s = idesc_f16(128, dk, 0, 0, 1);          // (alpha S^T, TMEM) x A^T (MN)
    // S^T (bf16 pairs, TMEM) x Q^T (bf16); with the position embedding fp16 pairs x rotated fp16 q
    const uint32_t id_o = idesc_f16(128, kQTok, kRope ? 0 : 1, 0, 0);
    uint8_t *qbuf = sm + OFF_QB;                                 // q buffers, 16 KB each
    const uint32_t tmO = tmem + TM_R;                            // O buffers, 64 columns each

    // Wait for this tile's MMAs: the issuing thread polls the mbarrier, the
    // others wait on the named barrier (which takes no issue slots from the
    // warps doing work).  False, for all 128 threads of the tile, on a
    // timeout, on `extra` from any of them, or once another role gave up.
    auto tile_wait = [&](int extra) -> bool {
      int bad = extra;
      if (issuer) bad |= !mbar_wait(&bar.mma_bar[tile], tphase, lim);
      tphase ^= 1u;
      return !bar_sync_or(tbar, 128, bad || *abort_flag);
    };
    // the same for one thread's mbarrier over all 256 chain threads
    auto group_wait = [&](uint64_t *b, uint32_t parity) -> bool {
      int bad = 0;
      if (tid == 0) bad = !mbar_wait(b, parity, lim);
      return !bar_sync_or(1, kChain, bad || *abort_flag);
    };
    auto issue_q = [&](int f, int bh, int t0) {  // thread 0
      const int bq = qi & 1;
      mbar_expect_tx(&bar.q_full[bq], 16384);
      uint8_t *qb = qbuf + bq * 16384;
      tma_load_4d(qb, &tmap_q, &bar.q_full[bq], 0, t0, f, bh);
      tma_load_4d(qb + 8192, &tmap_q, &bar.q_full[bq], 64, t0, f, bh);
      ++qi;
    };

    // The chain group takes the tickets: the first here, each next one right
    // after the current frame's state is published (before its read-out), and
    // hands each to the prep groups.  A ticket is thus started a fixed read-out
    // time after it is taken, whatever the frame chain's waits were; taking it
    // earlier (for the prep groups to run on across the frame boundary) was
    // measured slower, the longer hold lengthening the frame chain's waits.
    if (tid == 0) {
      const long t = atomicAdd(p.ws.counter, 1);
      const int tk0 = (int)(t < units ? t : -1);
      bar.ticket_ring[0] = tk0;
      mbar_arrive_only(&bar.tkt_bar[0]);
      if (!issue_frame_kv(tk0, 0)) failed = true;
    }
    if (bar_sync_or(1, kChain, failed ? 1 : 0)) failed = true;
    for (; !failed;) {
      const int tk = bar.ticket_ring[frames & 3];
      ++frames;
      if (tk < 0) break;
      const long ticket = tk;
      const Unit un = unit_of(tk);
      // (one unit per frame: the 64-bit forms, which leave the register allocation as it was)
      const int f = kSeg ? un.f : (int)(ticket / BH), bh = kSeg ? un.bh : (int)(ticket % BH);
      const int seg = un.s, c0 = un.c0, c1 = un.c1;
      const float a_raw = p.alpha[(long)bh * F + f];
      const float alpha = seg > 0 ? 1.f : (p.gates_are_logits ? gate_alpha(a_raw) : a_raw);

      // Y_A^T = I in TMEM (the first chunk accumulates onto it); Y_B^T starts
      // from the first chunk's product
      if (tile == 0) {
#pragma unroll 1
        for (int cb = 0; cb < nkd; ++cb) {
          float r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = (cb * 16 + e == row) ? 1.f : 0.f;
          tmem_st16(tmY + lane_off + cb * 16, r);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      named_bar(tbar, 128);

      // ---- the frame's chunks, one independent chain per tile
      for (int c = c0; c < c1; ++c, ++g) {
        const int s = (int)(g % kSlots);
        const uint32_t ph = (g / kSlots) & 1u;
        uint8_t *slot = sm + OFF_SLOT + s * SLOT_BYTES;
        int cbad = 0;
        if (c > c0) {
          // R^T = -Y^T Khat^T (the [0 ; V^T] target enters with the W product)
          if (issuer) {
            if (!mbar_wait(&bar.khat_ready[s], ph, lim)) cbad = 1;
            tc_fence_after();
            const uint32_t kh = smem_u32(slot + SL_KHAT);
            const uint32_t mb = smem_u32(mir);
            for (int kk = 0; kk < nkd; ++kk) {
              const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
              const uint32_t kho = (kk >> 2) * 8192 + (kk & 3) * 32;
              mma_f16_ss(tmR, sdesc_sw128(mb + ko, 16, 1024), sdesc_sw128(kh + kho, 16, 1024), id_r,
                         kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar.mma_bar[tile]);
          }
          if (!tile_wait(cbad)) {
            failed = true;
            break;
          }
          tc_fence_after();
          {
            // row of R^T -> fp16 pairs in the first 32 columns (A operand of the next MMA)
            float r[4][16];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tmem_ld16(tmR + lane_off + cb * 16, r[cb]);
            tmem_ld_wait();
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
              uint32_t h[16];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                h[e] = pack_h2(r[2 * hp][2 * e], r[2 * hp][2 * e + 1]);
                h[8 + e] = pack_h2(r[2 * hp + 1][2 * e], r[2 * hp + 1][2 * e + 1]);
              }
              tmem_st16u(tmR + lane_off + hp * 16, h);
            }
            tmem_st_wait();
          }
          tc_fence_before();
          named_bar(tbar, 128);
        }
        // Y^T += R^T W  (tile B also + V^T W); the last MMA of this tile on slot s releases it
        if (issuer) {
          if (!mbar_wait(&bar.w_ready[s], ph, lim)) cbad = 1;
          tc_fence_after();
          const uint32_t wb = smem_u32(slot + SL_W);
          if (c > c0) {
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ts(tmY, tmR + kk * 8, sdesc_sw128(wb + kk * 32, 16, 1024), id_y, 1u);
          } else if (tile == 0) {
            const uint32_t kb = smem_u32(slot + SL_KHAT);
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(tmY, sdesc_sw128(kb + kk * 2048, 8192, 1024), sdesc_sw128(wb + kk * 32, 16, 1024), id_kw,
                         1u);
          }
          if (tile == 1) {
            const uint32_t vb = smem_u32(slot + SL_V);
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(tmY, sdesc_sw128(vb + kk * 2048, 8192, 1024), sdesc_sw128(wb + kk * 32, 16, 1024), id_vw,
                         (c > c0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar.mma_bar[tile]);
          mma_commit(&bar.slot_free[s]);
        }
        if (!tile_wait(cbad)) {
          failed = true;
          break;
        }
        tc_fence_after();
        // slot s is free once both tiles' last MMAs on it are done: chunk c + 3 goes there
        if (tile == 1 && issuer && c + kSlots < c1 && !issue_kv(g + kSlots, f, bh, c + kSlots)) {
          *abort_flag = 1;
          latch_status(p.status, GDN_ERR_TIMEOUT);
        }
        // Y^T rows -> fp16 mirror (tile B's rows are not needed after the last
        // chunk; tile A's last copy is alpha_f A_f^T for the chain step)
        if (c + 1 < c1 || tile == 0) {
          const float sc = c + 1 < c1 ? 1.f : alpha;
#pragma unroll
          for (int hb = 0; hb < 4; ++hb) {  // batches of up to 2 column blocks
            if (2 * hb >= nkd) break;
            float r[2][16];
#pragma unroll
            for (int e = 0; e < 2; ++e)
              if (2 * hb + e < nkd) tmem_ld16(tmY + lane_off + (2 * hb + e) * 16, r[e]);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 2; ++e)
              if (2 * hb + e < nkd) {
                const int cb = 2 * hb + e;
#pragma unroll
                for (int x = 0; x < 16; ++x) r[e][x] *= sc;
                store_row16_f16(mir + (cb >> 2) * 16384, row, (cb & 3) * 16, r[e]);
              }
          }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(tbar, 128);
      }
      if (bar_sync_or(1, kChain, failed ? 1 : 0)) {
        failed = true;
        break;
      }
      if (kSave && tile == 0) {  // A_f^T row `row` (TMEM lane) -> the backward's frame maps
        tc_fence_after();
        float *mrow = p.save_maps + (((long)bh * F + f) * dk + row) * dk;
#pragma unroll 1
        for (int cb = 0; cb < nkd; ++cb) {
          float r[16];
          tmem_ld16(tmY + lane_off + cb * 16, r);
          tmem_ld_wait();
          if (row < dk) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4 *>(mrow + cb * 16 + e) = make_float4(r[e], r[e + 1], r[e + 2], r[e + 3]);
          }
        }
      }

      // ---- chain step: S_f^T = B_f^T + S_{f-1}^T (alpha A_f^T)
      const long uidx = ((long)bh * F + f) * P + seg;  // this unit's flag and published state
      // read-out tiles of this chain: tile-chain A takes tiles 0, 2, 4, ...; B 1, 3, 5, ...
      const int tb0 = c0 * kC, tb1 = (kSeg && c1 * kC < L) ? c1 * kC : L;  // the unit's tokens
      const int nt = kSave ? 0 : (tb1 - tb0 + kQTok - 1) / kQTok;  // read-out tiles
      if (!kSave && tid == 0) {  // the first q tiles -> the tile-B half of the mirror (free now)
        issue_q(f, bh, tb0);
        if (nt > 1) issue_q(f, bh, tb0 + kQTok);
      }
      // the state before this unit: the previous segment's, or the previous
      // frame's last segment's (unit uidx - 1 either way), else state_in
      const bool chained = f > 0 || seg > 0;
      const bool have_prev = chained || p.state_in != nullptr;
      {
        int bad = 0;
        if (tid == 0 && chained) bad = !wait_flag(p.ws.flags + uidx - 1, 1, lim);
        if (bar_sync_or(1, kChain, bad || *abort_flag)) {
          failed = true;
          break;
        }
      }
      const int j = row;
      const int l0 = tile * 64;                                        // this thread's half of the d_k columns
      const int nl = dk - l0 < 64 ? (dk - l0 > 0 ? dk - l0 : 0) : 64;  // columns in it (a multiple of 16)
      if (have_prev) {
        // S_{f-1}^T row j as fp16 pairs into TMEM columns [256, 256 + d_k / 2) (the A operand
        // of the chain product); the caller's fp32 state_in also as the fp16 low parts of its
        // values into [320, 320 + d_k / 2), for a second product
        if (nl > 0) {
          if (chained) {
            // published rows S^T[j][l] (fp16, d_k per row): the pairs are the loaded words
            const __half *base = reinterpret_cast<const __half *>(p.ws.states) + (uidx - 1) * (long)dk * dv;
            {
              const uint4 *src = reinterpret_cast<const uint4 *>(base + (long)j * dk + l0);
              uint4 u[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                u[e] = (j < dv && 8 * e < nl) ? __ldcg(src + e) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                if (32 * h2 < nl) {
                  const uint32_t w[16] = {u[4 * h2].x,     u[4 * h2].y,     u[4 * h2].z,     u[4 * h2].w,
                                          u[4 * h2 + 1].x, u[4 * h2 + 1].y, u[4 * h2 + 1].z, u[4 * h2 + 1].w,
                                          u[4 * h2 + 2].x, u[4 * h2 + 2].y, u[4 * h2 + 2].z, u[4 * h2 + 2].w,
                                          u[4 * h2 + 3].x, u[4 * h2 + 3].y, u[4 * h2 + 3].z, u[4 * h2 + 3].w};
                  tmem_st16u(tmem + TM_R + lane_off + (l0 + 32 * h2) / 2, w);
                }
              }
            }
          } else {
            // the caller's fp32 state S[l][j] (d_v contiguous: lanes j read consecutive addresses),
            // split into fp16 high and low parts
            const float *prev = p.state_in + (long)bh * dk * dv;
            float smax = 0.f;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
              if (32 * h2 >= nl) break;
              uint32_t wh[16], wl[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int l = l0 + 32 * h2 + 2 * e;
                const float v0 = (j < dv && l < dk) ? __ldcg(prev + (long)l * dv + j) : 0.f;
                const float v1 = (j < dv && l + 1 < dk) ? __ldcg(prev + (long)(l + 1) * dv + j) : 0.f;
                smax = fmaxf(smax, fmaxf(fabsf(v0), fabsf(v1)));
                const float h0 = __half2float(__float2half_rn(v0)), h1 = __half2float(__float2half_rn(v1));
                wh[e] = pack_h2(h0, h1);
                wl[e] = pack_h2(v0 - h0, v1 - h1);
              }
              tmem_st16u(tmem + TM_R + lane_off + (l0 + 32 * h2) / 2, wh);
              tmem_st16u(tmem + TM_R + 64 + lane_off + (l0 + 32 * h2) / 2, wl);
            }
            if (!(smax < kF16Max)) latch_status(p.status, GDN_ERR_RANGE);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(1, kChain);
        if (tid == 0) {
          tc_fence_after();
          const uint32_t ab = smem_u32(sm + OFF_MIRROR);  // tile A of the mirror = alpha A_f^T rows, read MN-major
          for (int part = 0; part < (chained ? 1 : 2); ++part)  // state_in: high + low parts
            for (int kk = 0; kk < nkd; ++kk)
              mma_f16_ts(tmem + TM_Y + 128, tmem + TM_R + 64 * part + kk * 8, sdesc_sw128(ab + kk * 2048, 16384, 1024),
                         id_s, 1u);
          mma_commit(&bar.fr_bar);
        }
        const bool ok = group_wait(&bar.fr_bar, fphase);
        fphase ^= 1u;
        if (!ok) {
          failed = true;
          break;
        }
        tc_fence_after();
      }
      // S_f^T row j (this thread's half of l), in two passes over TMEM: first an
      // fp16 row into the staging area (one bulk store to the workspace, for
      // the next unit) and the fp32 state_out after the last frame; then, while
      // that store drains, bf16 high/low pairs into TMEM [0, 128) (the
      // read-out's A operand) and, from a frame's last segment of several, to
      // the workspace for the others' read-outs.  The flag follows both.
      const bool last_seg = seg == P - 1;
      {
        float *sout = (f == F - 1 && last_seg && p.state_out) ? p.state_out + (long)bh * dk * dv : nullptr;
        float *sall = kSave ? p.save_states + ((long)bh * F + f) * dk * dv : nullptr;
        __half *srow = reinterpret_cast<__half *>(sm + OFF_STAGE) + (long)j * dk + l0;
        float smax = 0.f;
#pragma unroll 1
        for (int h2 = 0; h2 < 4; ++h2) {  // 16 columns l at a time
          if (16 * h2 >= nl) break;
          const int lb = l0 + 16 * h2;
          float r[16];
          tmem_ld16(tmem + TM_Y + 128 + lane_off + lb, r);
          tmem_ld_wait();
          if (j < dv) {
            uint32_t hf[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              smax = fmaxf(smax, fmaxf(fabsf(r[2 * e]), fabsf(r[2 * e + 1])));
              hf[e] = pack_h2(r[2 * e], r[2 * e + 1]);
            }
            *reinterpret_cast<uint4 *>(srow + 16 * h2) = make_uint4(hf[0], hf[1], hf[2], hf[3]);
            *reinterpret_cast<uint4 *>(srow + 16 * h2 + 8) = make_uint4(hf[4], hf[5], hf[6], hf[7]);
            if (sout) {
#pragma unroll
              for (int e = 0; e < 16; ++e) sout[(long)(lb + e) * dv + j] = r[e];
            }
            if (kSave) {
#pragma unroll
              for (int e = 0; e < 16; ++e) sall[(long)(lb + e) * dv + j] = r[e];
            }
          }
        }
        if (!(smax < kF16Max)) latch_status(p.status, GDN_ERR_RANGE);
      }
      fence_async_smem();
      named_bar(1, kChain);
      if (tid == 0) {
        __half *dst = reinterpret_cast<__half *>(p.ws.states) + uidx * (long)dk * dv;
        bulk_store(dst, sm + OFF_STAGE, (uint32_t)(dk * dv * 2));
        bulk_commit();
      }
      uint32_t *ro = (P > 1 && last_seg && j < dv) ? p.ro_states + (((long)bh * F + f) * dv + j) * dk : nullptr;
#pragma unroll 1
      for (int h2 = 0; h2 < 4; ++h2) {
        if (16 * h2 >= nl) break;
        const int lb = l0 + 16 * h2;
        float r[16];
        tmem_ld16(tmem + TM_Y + 128 + lane_off + lb, r);
        tmem_ld_wait();
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a = j < dv ? r[2 * e] : 0.f;
          const float b = j < dv ? r[2 * e + 1] : 0.f;
          if (kRope) {  // the read-out's q is fp16 (rotated): fp16 pairs
            const __half2 h = __floats2half2_rn(a, b);
            const float2 hb = __half22float2(h);
            const __half2 lw = __floats2half2_rn(a - hb.x, b - hb.y);
            hi[e] = *reinterpret_cast<const uint32_t *>(&h);
            lo[e] = *reinterpret_cast<const uint32_t *>(&lw);
          } else {
            const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
            const float2 hb = __bfloat1622float2(h);
            const __nv_bfloat162 lw = __floats2bfloat162_rn(a - hb.x, b - hb.y);
            hi[e] = *reinterpret_cast<const uint32_t *>(&h);
            lo[e] = *reinterpret_cast<const uint32_t *>(&lw);
          }
        }
        tmem_st8u(tmem + TM_Y + lane_off + lb / 2, hi);
        tmem_st8u(tmem + TM_Y + 64 + lane_off + lb / 2, lo);
        if (ro) {  // row j: high pairs in words [0, d_k / 2), low pairs in [d_k / 2, d_k)
          uint4 *rh = reinterpret_cast<uint4 *>(ro + lb / 2);
          uint4 *rl = reinterpret_cast<uint4 *>(ro + dk / 2 + lb / 2);
          rh[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          rh[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
          rl[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          rl[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
        }
      }
      if (ro) __threadfence();  // before thread 0 releases the flag
      tmem_st_wait();
      tc_fence_before();
      named_bar(1, kChain);
      if (tid == 0) {
        bulk_wait_all();
        if (ticket != p.withhold) {
          fence_async_global();
          __threadfence();
          st_release(p.ws.flags + uidx, 1);
        }
      }

      // ---- read-out: O_f = Q_f S_f in 64-token tiles.  Thread 0 runs
      // O^T = S_f^T Q^T (bf16 high and low parts of S_f from TMEM, bf16 q) into
      // TMEM buffer n & 1 while warps 4-7 (all 128 TMEM lanes) move tile n - 1
      // through shared memory into O's row-major layout and bulk-store it.  An
      // MMA's issue holds its thread for its whole duration, so the issuing
      // thread takes no part in the epilogue.
      named_bar(1, kChain);  // thread 0's bulk store of S_f has read the staging area
      if (!last_seg) {
        // the frame's state is the last segment's: its bf16 high/low rows
        // replace this unit's in TMEM [0, 128)
        int bad = 0;
        if (tid == 0) bad = !wait_flag(p.ws.flags + uidx - seg + (P - 1), 1, lim);
        if (bar_sync_or(1, kChain, bad || *abort_flag)) {
          failed = true;
          break;
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(p.ro_states + (((long)bh * F + f) * dv + j) * dk);
#pragma unroll 1
        for (int h2 = 0; h2 < 4; ++h2) {
          if (16 * h2 >= nl) break;
          const int lb = l0 + 16 * h2;
          uint4 a[4];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            a[e] = j < dv ? __ldcg(src + lb / 8 + e) : make_uint4(0u, 0u, 0u, 0u);
            a[2 + e] = j < dv ? __ldcg(src + dk / 8 + lb / 8 + e) : make_uint4(0u, 0u, 0u, 0u);
          }
          const uint32_t hi[8] = {a[0].x, a[0].y, a[0].z, a[0].w, a[1].x, a[1].y, a[1].z, a[1].w};
          const uint32_t lo[8] = {a[2].x, a[2].y, a[2].z, a[2].w, a[3].x, a[3].y, a[3].z, a[3].w};
          tmem_st8u(tmem + TM_Y + lane_off + lb / 2, hi);
          tmem_st8u(tmem + TM_Y + 64 + lane_off + lb / 2, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(1, kChain);
      }
      // the next ticket, and its first k, v loads, from a thread that is idle in
      // the read-out (thread 0 issues the read-out MMAs)
      if (tid == 32) {
        const long t = atomicAdd(p.ws.counter, 1);
        const int tkn = (int)(t < units ? t : -1);
        bar.ticket_ring[frames & 3] = tkn;
        mbar_arrive_only(&bar.tkt_bar[frames & 1]);
        if (!issue_frame_kv(tkn, g)) {
          *abort_flag = 1;
          latch_status(p.status, GDN_ERR_TIMEOUT);
        }
      }
      if (tid == 0) {
        int bad = 0;
        for (int n = 0; n < nt; ++n) {
          const uint32_t gt = rt + n, b = gt & 1u, ph = (gt >> 1) & 1u;
          if (!mbar_wait(kRope ? &bar.q_conv[b] : &bar.q_full[b], ph, lim)) {
            bad = 1;
            break;
          }
          ++qw;
          if (gt >= 2 && !mbar_wait(&bar.o_free[b], ph ^ 1u, lim)) {  // tile n - 2 has left O buffer b
            bad = 1;
            break;
          }
          tc_fence_after();
          const uint32_t b0 = smem_u32(qbuf + b * 16384);
          for (int hl = 0; hl < 2; ++hl)
            for (int kk = 0; kk < nkd; ++kk)
              mma_f16_ts(tmO + b * 64, tmem + TM_Y + hl * 64 + kk * 8,
                         sdesc_sw128(b0 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_o,
                         (hl > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bar.o_full[b]);
          ++oi;
          // q buffer b is free once these MMAs are done: tile n + 2 goes there
          if (!mbar_wait(&bar.o_full[b], ph, lim)) {
            bad = 1;
            break;
          }
          ++ow;
          if (n + 2 < nt) issue_q(f, bh, tb0 + (n + 2) * kQTok);
        }
        if (bad) {
          *abort_flag = 1;
          latch_status(p.status, GDN_ERR_TIMEOUT);
          failed = true;
        }
      } else if (kRope && warp >= 1 && warp < 4) {
        // position embedding: warps 1-3 rotate each q tile and convert it to fp16 in place
        const int ct = tid - 32;
        for (int n = 0; n < nt; ++n) {
          const uint32_t gt = rt + n, b = gt & 1u, ph = (gt >> 1) & 1u;
          {
            const int bad = ct == 0 ? !mbar_wait(&bar.q_full[b], ph, lim) : 0;
            if (bar_sync_or(6, 96, bad || *abort_flag)) {
              if (bad) {
                *abort_flag = 1;
                latch_status(p.status, GDN_ERR_TIMEOUT);
              }
              failed = true;
              break;
            }
          }
          uint8_t *qb = qbuf + b * 16384;
          float qmax = 0.f;
          for (int i = ct; i < 1024; i += 96) {  // [column block][64 rows][8 x 16 B], swizzled
            const int kb = i >> 9, rw = (i >> 3) & 63, pc = i & 7;
            const int ch = pc ^ (rw & 7);
            const int tf = tb0 + n * kQTok + rw;  // token index in the frame
            const RopeTok rtok = rope_tok(f, tf < L ? tf : 0, p);
            uint4 *cp = reinterpret_cast<uint4 *>(qb + kb * 8192 + rw * 128 + pc * 16);
            const uint4 u = *cp;
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float2 v2 = __bfloat1622float2(h[e]);
              const int dd = kb * 64 + ch * 8 + 2 * e;
              if (tf < L && dd < dk) v2 = rope_at(v2, dd, rtok, p);
              qmax = fmaxf(qmax, fmaxf(fabsf(v2.x), fabsf(v2.y)));
              o4[e] = pack_h2(v2.x, v2.y);
            }
            *cp = make_uint4(o4[0], o4[1], o4[2], o4[3]);
          }
          if (!(qmax < kF16Max)) latch_status(p.status, GDN_ERR_RANGE);
          fence_async_smem();
          named_bar(6, 96);
          if (ct == 0) mbar_arrive_only(&bar.q_conv[b]);
        }
      } else if (tile == 1) {
        float *stg = reinterpret_cast<float *>(sm + OFF_STAGE);
        for (int n = 0; n < nt; ++n) {
          const uint32_t gt = rt + n, b = gt & 1u, ph = (gt >> 1) & 1u;
          {
            int bad = 0;
            if (issuer) bad = !mbar_wait(&bar.o_full[b], ph, lim);
            if (bar_sync_or(tbar, 128, bad || *abort_flag)) {
              failed = true;
              break;
            }
          }
          tc_fence_after();
          if (issuer) bulk_wait_read();  // the previous tile's bulk store has read the staging rows
          named_bar(tbar, 128);
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {  // 32 tokens at a time
            float r[2][16];
            tmem_ld16(tmO + b * 64 + lane_off + 32 * hh, r[0]);
            tmem_ld16(tmO + b * 64 + lane_off + 32 * hh + 16, r[1]);
            tmem_ld_wait();
            if (j < dv) {
#pragma unroll
              for (int e = 0; e < 32; ++e) stg[(32 * hh + e) * dv + j] = r[e >> 4][e & 15];
            }
          }
          tc_fence_before();
          fence_async_smem();
          named_bar(tbar, 128);
          if (issuer) {
            mbar_arrive_only(&bar.o_free[b]);
            const int t0 = tb0 + n * kQTok;
            const int tl = tb1 - t0 < kQTok ? tb1 - t0 : kQTok;  // tokens of this tile
            bulk_store(p.o + ((long)bh * N + (long)f * L + t0) * dv, stg, (uint32_t)(tl * dv * 4));
            bulk_commit();
          }
        }
      }
      rt += (uint32_t)nt;
      // the staging rows (the tile-A half of the mirror) are rewritten by the next frame
      if (tid == 128) bulk_wait_read();
      if (bar_sync_or(1, kChain, failed ? 1 : 0)) {
        failed = true;
        break;
      }
    }
    if (failed) {
      if (tid == 0) latch_status(p.status, GDN_ERR_TIMEOUT);  // the first code latched wins
      *abort_flag = 1;
    }
    // loads and MMAs issued by thread 0 complete before the CTA exits
    if (tid == 0) {
      for (; qw < qi; ++qw) mbar_wait(&bar.q_full[qw & 1], (qw >> 1) & 1u, lim);
      for (; ow < oi; ++ow) mbar_wait(&bar.o_full[ow & 1], (ow >> 1) & 1u, lim);
    }
    if (issuer) bulk_wait_all();
    named_bar(1, kChain);
    if (tid == 0) {  // the last k, v loads issued (earlier ones were waited for by the prep groups)
      const uint32_t n = bar.loads;
      for (uint32_t gg = n > (uint32_t)kSlots ? n - kSlots : 0u; gg < n; ++gg)
        mbar_wait(&bar.kv_full[gg % kSlots], (gg / kSlots) & 1u, lim);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace tc

bool gdn_tc_supported(int dk, int dv) {
  return dk % 16 == 0 && dv % 16 == 0 && dk >= 16 && dk <= 128 && dv >= 16 && dv <= 128;
}

// published frame states are fp16 rows S^T[j][l]: d_k * d_v halves = d_k * d_v / 2 floats
size_t gdn_tc_state_elems(int dk, int dv) { return (size_t)dk * dv / 2; }

template <bool kRope>
static cudaError_t launch_tc(const GdnParams &p, int grid, bool cooperative, cudaStream_t st, const CUtensorMap &mq,
                             const CUtensorMap &mk, const CUtensorMap &mv) {
  using namespace tc;
  if (!cooperative) {  // one unit per frame
    cudaError_t e = cudaFuncSetAttribute(gdn_tc_kernel<false, kRope>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kGdnSmemBytes);
    if (e != cudaSuccess) return e;
    gdn_tc_kernel<false, kRope><<<grid, kGThreads, kGdnSmemBytes, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(gdn_tc_kernel<true, kRope>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGdnSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = kGdnSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gdn_tc_kernel<true, kRope>, mq, mk, mv, p);
}

// the backward's recompute (kSave): maps and end states, no read-out
template <bool kRope>
static cudaError_t launch_save(const GdnParams &p, int grid, cudaStream_t st, const CUtensorMap &mq,
                               const CUtensorMap &mk, const CUtensorMap &mv) {
  using namespace tc;
  cudaError_t e = cudaFuncSetAttribute(gdn_tc_kernel<false, kRope, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGdnSmemBytes);
  if (e != cudaSuccess) return e;
  gdn_tc_kernel<false, kRope, true><<<grid, kGThreads, kGdnSmemBytes, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

cudaError_t launch_gdn_tc(const GdnParams &p, int grid, bool cooperative, cudaStream_t st) {
  using namespace tc;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_bf16_map(&mq, p.q, p.dk, p.L, p.F, BH, kQTok) || !make_bf16_map(&mk, p.k, p.dk, p.L, p.F, BH, 64) ||
      !make_bf16_map(&mv, p.v, p.dv, p.L, p.F, BH, 64))
    return cudaErrorInvalidValue;
  if (p.save_maps) {  // the backward's recompute: one unit per frame
    if (cooperative || !p.save_states) return cudaErrorInvalidValue;
    return p.rope_on ? launch_save<true>(p, grid, st, mq, mk, mv) : launch_save<false>(p, grid, st, mq, mk, mv);
  }
  return p.rope_on ? launch_tc<true>(p, grid, cooperative, st, mq, mk, mv)
                   : launch_tc<false>(p, grid, cooperative, st, mq, mk, mv);
}

}  // namespace gdn
