// Frame-wise Gated DeltaNet on tcgen05 tensor cores, chunk maps in product form.
//
// Source of the method: SANA-WM GeekNews summary, "Core design and generation
// pipeline" (frame-wise Gated DeltaNet); dothoosh.com SANA-WM article (fixed-
// size recurrent state).  Update rule per token: S <- S - beta khat (S^T khat
// - v)^T after a per-frame decay S <- alpha S; every token of a frame reads
// o = S^T q with the state after the whole frame.
//
// Work unit = one (b, h, f) frame, taken from a ticket counter (f-major) by a
// persistent CTA.  The CTA builds the frame map S_f = A_f (alpha_f S_{f-1}) +
// B_f by running the delta rule on Y = [A | B] (d_k x (d_k + d_v)) from
// [I | 0], 64 tokens (one chunk) at a time.  With the chunk's UT transform
//     T = (I + N)^-1 diag(beta),  N = strict_lower(diag(beta) Khat Khat^T),
//     W^T = Khat^T T                                    (d_k x 64)
// one chunk moves Y to
//     Y <- P Y + W^T [0 | V],    P = I - W^T Khat        (d_k x d_k),
// i.e. Y += M^T Y + W^T [0 | V] with M^T = -W^T Khat: ONE accumulation into Y
// per chunk (Y lives in TMEM, lanes = rows of Y) whose operands (M^T, W^T) do
// not depend on Y and are made ahead by the prep warps.  Then
//     S_f = alpha_f A_f S_{f-1} + B_f          (one d_k x d_k x d_v product)
// waits on the previous frame's published state, and O_f = Q_f S_f.
//
// Warp roles (512 threads):
//   warps 8-11, 12-15  two prep groups for even and odd chunks: gates beta,
//       key normalisation (fp16 khat), v to fp16, Gram matrix Khat Khat^T on
//       tcgen05, the inverse (I + N)^-1 by column-parallel forward
//       substitution in registers (one thread per column, rows of N read as
//       shared-memory broadcasts), T as a K-major fp16 tile, W^T = Khat^T T and
//       M^T = -W^T Khat on tcgen05, both left in TMEM as fp16 pairs (the A
//       operands of the chain's accumulation).
//   warps 0-7  the chain: per chunk thread 0 issues Y += M^T Ycopy (N = d_k +
//       d_v) and Y_B += W^T V, then all eight warps copy Y to shared memory as
//       fp16 (the next chunk's B operand).  At the frame end the chain step
//       (alpha A_f from the copy, S_{f-1} as fp16 high/low images) and the
//       publish of S_f; then the read-out in 128-token tiles: thread 0 issues
//       the MMAs (q converted to fp16 in place by warps 1-3, S_f as an fp16
//       B operand), warps 4-7 store O rows straight from TMEM.
// k and v reach a 3-slot ring by TMA; the frame's q tiles are prefetched into
// L2 during its last chunks.  S_f is handed to the next frame as fp16 high and
// low parts (about 22 significant bits), written in the swizzled layout of
// the consumer's MMA operand and fetched with one bulk copy each.
// Operands that are not exact in bf16 (khat, v, q after the cast, Y, T, W, M,
// alpha A_f, the S images) enter the tensor cores as fp16 (11-bit
// significands); all accumulation is fp32.
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace pf {

using namespace tc;

constexpr int kThreads = 512;
constexpr int kChain = 256;
constexpr int kC = 64;               // tokens per chunk
constexpr int kSlots = 3;            // chunks of k, v in flight
constexpr int kMaxQT = 64;           // most tokens per read-out tile
constexpr int kQBuf = 3;             // q tiles in flight in the read-out
constexpr int kStageTok = 32;        // tokens per bulk store of o
constexpr uint32_t kSlotBytes = 32768;
constexpr uint32_t kSlK = 0;         // khat: [col block][64 t][128 B] (TMA'd bf16, fp16 in place)
constexpr uint32_t kSlV = 16384;     // v:    [col block][64 t][128 B]
constexpr uint32_t kPrepBytes = 16384;   // per prep group: N (fp32 64 x 64), then T (fp16, 64 rows t x 128 B)

constexpr int kMaxSmem = 232448;

struct Bars {
  uint64_t kv_full[kSlots];    // TMA bytes of k and v of the chunk in the slot
  uint64_t slot_free[kSlots];  // the chain's MMAs of the slot's chunk are done
  uint64_t g_mma[2];           // prep group: its own MMAs (Gram, W, M)
  uint64_t prep_ready[2];      // prep group -> chain: W^T, M^T (TMEM) and V (fp16) of its chunk
  uint64_t chain_done[2];      // chain -> prep group: the MMAs reading its TMEM region are done
  uint64_t y_mma;              // chain: the chunk's MMAs are done
  uint64_t fr_bar;             // chain step MMAs
  uint64_t s_full[2];          // bulk copies of S_{f-1}: low, high image
  uint64_t q_full[kQBuf];      // read-out: q tile in buffer b (TMA)
  uint64_t o_full[2];          // read-out: the MMAs into O buffer b are done
  uint64_t o_free[2];          // read-out: the epilogue has read O buffer b
  uint64_t tkt_bar[2];         // chain -> prep groups: next frame's ticket
  uint64_t drain;              // exit: every MMA issued by the three issuing threads is done
  uint32_t tmem_base;
  int abort;
  uint32_t loads;              // chunks whose k, v loads have been issued
  uint32_t q_used;             // read-out q tiles consumed by the converters
  int ticket_ring[4];
};

// Shared-memory and TMEM map for one (d_k, d_v).  Byte offsets from the
// 1024-aligned base of dynamic shared memory.
struct Layout {
  int ok;
  uint32_t yb;        // bytes of one 64-column block of an operand with d_k rows: d_k * 128
  uint32_t nyb;       // 64-column blocks of the Y copy (d_k + d_v columns)
  uint32_t nab;       // blocks holding A (the first d_k columns)
  uint32_t nvb;       // blocks of an S image (d_v columns)
  uint32_t s_img;     // bytes of one S image (nvb * yb)
  uint32_t off_y;     // Y copy, fp16, MN-major B operand: [block][d_k rows][128 B]
  uint32_t off_fr;    // frame area (low image of S_{f-1}; part of the read-out buffers)
  uint32_t off_slot;  // k, v ring
  uint32_t off_prep;  // two prep scratch areas
  uint32_t off_bar;
  uint32_t smem;      // dynamic shared memory to request (with the alignment slack)
  uint32_t off_shi;   // high image of S_{f-1}: the Y copy's blocks after A (free after the last chunk)
  uint32_t off_slo;   // low image of S_{f-1}
  uint32_t off_sf;    // read-out: S_f image (fp16) over the A blocks of the copy
  uint32_t off_q;     // read-out: two q tiles
  uint32_t qt;        // tokens per read-out tile: two O^T buffers of qt TMEM columns fit in Y's columns
  uint32_t qtile;     // bytes of one q tile: [col block][qt t][128 B]
  uint32_t off_stage; // read-out: o staging, kStageTok rows of d_v fp32 (the bulk store's source)
  uint32_t stage;     // bytes of the staging area
  uint32_t ny;        // d_k + d_v: TMEM columns of Y
  uint32_t prep_cols; // TMEM columns of one prep group: 32 (W^T pairs) + d_k (M^T, fp32 then pairs)
};

__host__ __device__ inline Layout make_layout(int dk, int dv) {
  Layout l;
  l.ok = 0;
  if (dk % 16 || dv % 16 || dk < 16 || dv < 16 || dk > 128 || dv > dk) return l;
  l.ny = (uint32_t)(dk + dv);
  l.prep_cols = 32u + (uint32_t)dk;
  if (l.ny + 2 * l.prep_cols > 512) return l;                 // TMEM
  l.qt = (l.ny / 2) / kStageTok * kStageTok;                  // whole bulk stores per tile
  if (l.qt > (uint32_t)kMaxQT) l.qt = kMaxQT;
  if (l.qt == 0) return l;
  l.qtile = 2u * l.qt * 128u;
  l.yb = (uint32_t)dk * 128u;
  l.nyb = (l.ny + 63) / 64;
  l.nab = (uint32_t)(dk + 63) / 64;
  l.nvb = (uint32_t)(dv + 63) / 64;
  if (l.nyb < l.nab + l.nvb) return l;                        // room for the high image after A
  l.s_img = l.nvb * l.yb;
  const uint32_t ycopy = l.nyb * l.yb;
  l.stage = (uint32_t)kStageTok * (uint32_t)dv * 4u;
  const uint32_t ro = l.s_img + kQBuf * l.qtile + l.stage;     // read-out: S_f image, q tiles, staging
  uint32_t fr = l.s_img;
  if (ro > ycopy + fr) fr = ro - ycopy;
  fr = (fr + 1023) / 1024 * 1024;
  l.off_y = 0;
  l.off_fr = ycopy;
  l.off_slot = l.off_fr + fr;
  l.off_prep = l.off_slot + kSlots * kSlotBytes;
  l.off_bar = l.off_prep + 2 * kPrepBytes;
  l.smem = l.off_bar + (uint32_t)sizeof(Bars) + 1024;
  if (l.smem > (uint32_t)kMaxSmem) return l;
  l.off_shi = l.off_y + l.nab * l.yb;
  l.off_slo = l.off_fr;
  l.off_sf = l.off_y;
  l.off_q = l.off_y + l.s_img;
  l.off_stage = l.off_q + kQBuf * l.qtile;
  l.ok = 1;
  return l;
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// 16 fp32 values -> two 16-byte fp16 chunks at columns col0 .. col0+15 of row
// `row` of a 128B-swizzled tile (col0 a multiple of 8, col0 + 15 < 64).
__device__ __forceinline__ void st_row16_f16(uint8_t *tile, uint32_t row, uint32_t col0, const float (&r)[16]) {
  uint4 a = make_uint4(pack_h2(r[0], r[1]), pack_h2(r[2], r[3]), pack_h2(r[4], r[5]), pack_h2(r[6], r[7]));
  uint4 b = make_uint4(pack_h2(r[8], r[9]), pack_h2(r[10], r[11]), pack_h2(r[12], r[13]), pack_h2(r[14], r[15]));
  *reinterpret_cast<uint4 *>(tile + sw128_offset(row, col0)) = a;
  *reinterpret_cast<uint4 *>(tile + sw128_offset(row, col0 + 8)) = b;
}

// bf16 x 8 -> fp16 x 8 (one 16-byte chunk); sets *big if a value is beyond the fp16 range
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

// Largest finite fp16 value; anything at or beyond it (or NaN) is out of range.
constexpr float kF16Max = 65504.0f;
__device__ __forceinline__ bool out_of_f16_range(float amax) { return !(amax < kF16Max); }

__global__ void __launch_bounds__(kThreads, 1)
    gdn_pform_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, GdnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const Layout lay = make_layout(dk, dv);
  Bars &bar = *reinterpret_cast<Bars *>(sm + lay.off_bar);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int BH = p.B * p.H;
  const long units = (long)BH * F;
  const long N = (long)F * L;
  const unsigned long long lim = p.spin_limit_ns;
  const int nkd = dk / 16;            // k-steps over d_k
  const int nvc = dv / 16;            // 16-column chunks of d_v
  const int nch = (L + kC - 1) / kC;  // chunks per frame
  const int qt = (int)lay.qt;         // tokens per read-out tile
  volatile int *abort_flag = &bar.abort;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar.kv_full[s], 1);
      mbar_init(&bar.slot_free[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.g_mma[s], 1);
      mbar_init(&bar.prep_ready[s], 1);
      mbar_init(&bar.chain_done[s], 1);
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.o_full[s], 1);
      mbar_init(&bar.o_free[s], 1);
      mbar_init(&bar.tkt_bar[s], 1);
    }
    mbar_init(&bar.q_full[2], 1);
    mbar_init(&bar.y_mma, 1);
    mbar_init(&bar.fr_bar, 1);
    mbar_init(&bar.drain, 3);
    bar.abort = 0;
    bar.loads = 0;
    bar.q_used = 0;
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
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

  // k, v of chunk c of frame (f, bh), the gg-th chunk of this CTA, into slot
  // gg % 3 once the chain is done with the slot's previous chunk.  One thread.
  auto issue_kv = [&](uint32_t gg, int f, int bh, int c) -> bool {
    const int s = (int)(gg % kSlots);
    if (gg >= (uint32_t)kSlots && !mbar_wait(&bar.slot_free[s], ((gg / kSlots) & 1u) ^ 1u, lim)) return false;
    uint8_t *slot = sm + lay.off_slot + s * kSlotBytes;
    const int t0 = c * kC;
    mbar_expect_tx(&bar.kv_full[s], 32768);
    tma_load_4d(slot + kSlK, &tmap_k, &bar.kv_full[s], 0, t0, f, bh);
    tma_load_4d(slot + kSlK + 8192, &tmap_k, &bar.kv_full[s], 64, t0, f, bh);
    tma_load_4d(slot + kSlV, &tmap_v, &bar.kv_full[s], 0, t0, f, bh);
    tma_load_4d(slot + kSlV + 8192, &tmap_v, &bar.kv_full[s], 64, t0, f, bh);
    bar.loads = gg + 1;
    if (c + 2 < nch) {  // two chunks further on towards L2, so that their loads find them there
      const int t2 = t0 + 2 * kC;
      tma_prefetch_l2_4d(&tmap_k, 0, t2, f, bh);
      tma_prefetch_l2_4d(&tmap_k, 64, t2, f, bh);
      tma_prefetch_l2_4d(&tmap_v, 0, t2, f, bh);
      tma_prefetch_l2_4d(&tmap_v, 64, t2, f, bh);
    }
    return true;
  };
  auto issue_frame_kv = [&](int tk, uint32_t g0) -> bool {
    if (tk < 0) return true;
    const int f = tk / BH, bh = tk - (tk / BH) * BH;
    for (int c = 0; c < nch && c < kSlots; ++c)
      if (!issue_kv(g0 + c, f, bh, c)) return false;
    return true;
  };

  if (warp >= 8) {
    // ============================================================ prep groups
    regs_dec<120>();  // the block launches with 512 x 128; the chain takes 256 x 136
    const int grp = (warp - 8) >> 2;          // 0: even chunks, 1: odd chunks
    const int pt = tid - kChain - 128 * grp;  // 0..127; TMEM lane of this thread = pt
    const int pbar = 2 + grp;                 // named barrier of the group
    const uint32_t tmP = tmem + lay.ny + (uint32_t)grp * lay.prep_cols;
    uint8_t *scr = sm + lay.off_prep + grp * kPrepBytes;
    float *nsm = reinterpret_cast<float *>(scr);  // N rows: float4 group q of row r at q ^ (r & 7)
    uint32_t gph = 0;  // phase of g_mma[grp]
    uint32_t g = 0;
    bool stop = false;
    auto group_fail = [&](int timed_out) {
      if (pt == 0 && timed_out) latch_status(p.status, GDN_ERR_TIMEOUT);
      *abort_flag = 1;
      stop = true;
    };
    auto group_mma_wait = [&]() -> bool {  // pt 0 committed to g_mma[grp]
      const int bad = pt == 0 ? !mbar_wait(&bar.g_mma[grp], gph, lim) : 0;
      gph ^= 1u;
      if (bar_sync_or(pbar, 128, bad)) {
        group_fail(bad);
        return false;
      }
      tc_fence_after();
      return true;
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
      for (int c = 0; c < nch; ++c, ++g) {
        if ((int)(g & 1u) != grp) continue;
        const int s = (int)(g % kSlots);
        const uint32_t ph = (g / kSlots) & 1u;
        uint8_t *slot = sm + lay.off_slot + s * kSlotBytes;
        // gate of token pt of the chunk (used from the N step on, so its load latency is hidden)
        // (threads pt and pt + 64 both hold token pt % 64's: one makes N's row, the other, in
        // group 1, T's column)
        float bt = 0.f;
        if (c * kC + (pt & 63) < L) {
          const int f = tk / BH, bh = tk - (tk / BH) * BH;
          const float braw = p.beta[(long)bh * N + (long)f * L + c * kC + (pt & 63)];
          bt = p.gates_are_logits ? gate_beta(braw) : braw;
        }
        {
          const int bad = pt == 0 ? !mbar_wait(&bar.kv_full[s], ph, lim) : 0;
          if (bar_sync_or(pbar, 128, bad || *abort_flag)) {
            group_fail(bad);
            break;
          }
        }
        // 1. keys normalised in place (fp16 khat), v to fp16: thread -> token pt/2, column block pt%2
        float vmax = 0.f;
        {
          const int t = pt >> 1, kb = pt & 1;
          uint8_t *krow = slot + kSlK + kb * 8192;
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
          const float inv = 1.0f / fmaxf(sqrtf(ss), kKeyNormEps);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&ku[ch]);
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 v2 = __bfloat1622float2(h[e]);
              o[e] = pack_h2(v2.x * inv, v2.y * inv);
            }
            *reinterpret_cast<uint4 *>(krow + sw128_offset(t, ch * 8)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
          uint8_t *vrow = slot + kSlV + kb * 8192;
          uint4 vu[8];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) vu[ch] = *reinterpret_cast<const uint4 *>(vrow + sw128_offset(t, ch * 8));
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4 *>(vrow + sw128_offset(t, ch * 8)) = bf16x8_to_f16x8(vu[ch], vmax);
        }
        if (out_of_f16_range(vmax)) latch_status(p.status, GDN_ERR_RANGE);
        fence_async_smem();
        tc_fence_before();
        named_bar(pbar, 128);
        // 2. Gram matrix G = Khat Khat^T into the group's TMEM (lanes 0..63 = tokens), once the
        //    chain's MMAs of this group's previous chunk (which read the region) are done
        {
          int bad = 0;
          if (pt == 0) {
            if (g >= 2 && !mbar_wait(&bar.chain_done[grp], ((g >> 1) & 1u) ^ 1u, lim)) bad = 1;
            tc_fence_after();
            const uint32_t idg = idesc_f16(128, 64, 0, 0, 0);
            const uint32_t kb0 = smem_u32(slot + kSlK);
            for (int kk = 0; kk < nkd; ++kk) {
              const uint32_t a = kb0 + (kk >> 2) * 8192 + (kk & 3) * 32;
              mma_f16_ss(tmP, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), idg, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar.g_mma[grp]);
          }
          if (bar_sync_or(pbar, 128, bad)) {
            group_fail(bad);
            break;
          }
        }
        if (!group_mma_wait()) break;
        // 3. rows of N = strict_lower(diag(beta) G) into the scratch (warps 0-1 hold TMEM lanes 0..63)
        if (pt < kC) {
          const int t = pt;
          float gr[4][16];
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) tmem_ld16(tmP + lane_off + jb * 16, gr[jb]);
          tmem_ld_wait();
          float *row = nsm + t * 64;
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float4 v;
            v.x = (4 * q + 0 < t) ? bt * gr[q >> 2][(q & 3) * 4 + 0] : 0.f;
            v.y = (4 * q + 1 < t) ? bt * gr[q >> 2][(q & 3) * 4 + 1] : 0.f;
            v.z = (4 * q + 2 < t) ? bt * gr[q >> 2][(q & 3) * 4 + 2] : 0.f;
            v.w = (4 * q + 3 < t) ? bt * gr[q >> 2][(q & 3) * 4 + 3] : 0.f;
            *reinterpret_cast<float4 *>(row + 4 * (q ^ (t & 7))) = v;
          }
        }
        tc_fence_before();
        named_bar(pbar, 128);
        // 4. (I + N)^-1 = [[Ai, 0], [X, Bi]] from its 32 x 32 blocks: Ai = (I + N_aa)^-1 and
        //    Bi = (I + N_bb)^-1 by forward substitution (one thread per column, the column in
        //    registers, each row of N read as a shared-memory broadcast; the two blocks on two
        //    warps at once), then X = -Bi (N_ba Ai) by two 32 x 32 products on all 128 threads.
        //    Every block is written over N's own block once no thread reads it.  Then
        //    T = (I + N)^-1 diag(beta): column t of T is row t of the K-major B operand of the W
        //    product.  Group 0 substitutes on its warps 0-1, group 1 on its warps 2-3, so the
        //    two groups' substitutions issue from different SM sub-partitions.
        const int inv0 = grp ? kC : 0;
        auto nrow = [&](int r, int col) -> float * {  // address of N[r][col] (col % 4 == 0)
          return nsm + r * 64 + 4 * ((col >> 2) ^ (r & 7));
        };
        if (pt >= inv0 && pt < inv0 + kC) {
          const int sb = (pt - inv0) >> 5, cc = (pt - inv0) & 31, r0 = 32 * sb;
          // element (r0 + i, r0 + 4 q) of the block at a constant offset from one base
          // (r0 is a multiple of 32: (8 sb + q) ^ (i & 7) = 8 sb + (q ^ (i & 7)) for q < 8)
          const float *blk = nsm + r0 * 64 + 32 * sb;
          float x[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = (i == cc) ? 1.f : 0.f;
#pragma unroll
          for (int i = 1; i < 32; ++i) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int q = 0; q < (i + 3) / 4; ++q) {
              const float4 n4 = *reinterpret_cast<const float4 *>(blk + i * 64 + 4 * (q ^ (i & 7)));
              if (4 * q + 0 < i) a0 = fmaf(n4.x, x[4 * q + 0], a0);
              if (4 * q + 1 < i) a1 = fmaf(n4.y, x[4 * q + 1], a1);
              if (4 * q + 2 < i) a2 = fmaf(n4.z, x[4 * q + 2], a2);
              if (4 * q + 3 < i) a3 = fmaf(n4.w, x[4 * q + 3], a3);
            }
            // rows above the diagonal come out 0: every term there multiplies a 0
            x[i] = (i == cc) ? 1.f : -((a0 + a1) + (a2 + a3));
          }
          __syncwarp();  // the warp's 32 columns are done with N's diagonal block
#pragma unroll
          for (int i = 0; i < 32; ++i) nrow(r0 + i, r0 + (cc & ~3))[cc & 3] = x[i];
        }
        named_bar(pbar, 128);
        {
          // P = N_ba Ai, then X = -Bi P: thread (row i, columns 8 jg .. 8 jg + 7); the thread's
          // own row is read a float4 at a time, the 8 columns as broadcasts
          const int i = pt & 31, jg = pt >> 5;
          auto row_times = [&](int arow_r, int arow_c0, int brow0, float (&acc)[8]) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 2
            for (int kq = 0; kq < 8; ++kq) {
              const float4 a4 = *reinterpret_cast<const float4 *>(nrow(arow_r, arow_c0 + 4 * kq));
              const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int kk = 4 * kq + e;
                const float4 b0 = *reinterpret_cast<const float4 *>(nrow(brow0 + kk, 8 * jg));
                const float4 b1 = *reinterpret_cast<const float4 *>(nrow(brow0 + kk, 8 * jg + 4));
                acc[0] = fmaf(av[e], b0.x, acc[0]); acc[1] = fmaf(av[e], b0.y, acc[1]);
                acc[2] = fmaf(av[e], b0.z, acc[2]); acc[3] = fmaf(av[e], b0.w, acc[3]);
                acc[4] = fmaf(av[e], b1.x, acc[4]); acc[5] = fmaf(av[e], b1.y, acc[5]);
                acc[6] = fmaf(av[e], b1.z, acc[6]); acc[7] = fmaf(av[e], b1.w, acc[7]);
              }
            }
          };
          float acc[8];
          row_times(32 + i, 0, 0, acc);  // P[i][.] = N_ba[i][.] Ai
          named_bar(pbar, 128);          // every row of N_ba has been read: P goes over it
          *reinterpret_cast<float4 *>(nrow(32 + i, 8 * jg)) = make_float4(acc[0], acc[1], acc[2], acc[3]);
          *reinterpret_cast<float4 *>(nrow(32 + i, 8 * jg + 4)) = make_float4(acc[4], acc[5], acc[6], acc[7]);
          named_bar(pbar, 128);          // P complete
          row_times(32 + i, 32, 32, acc);  // (Bi P)[i][.] = Bi[i][.] P
          named_bar(pbar, 128);          // every row of P has been read: X goes over it
          *reinterpret_cast<float4 *>(nrow(32 + i, 8 * jg)) = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
          *reinterpret_cast<float4 *>(nrow(32 + i, 8 * jg + 4)) = make_float4(-acc[4], -acc[5], -acc[6], -acc[7]);
        }
        named_bar(pbar, 128);
        {
          // T: thread (column t, half h of the rows u) reads its half column of (I + N)^-1
          // (rows 0..31 of columns 32..63 hold N's zeros), then writes it as half of the
          // K-major row t once every thread has read (T takes N's first 8 KB)
          const int t = pt & 63, h = pt >> 6;
          float x[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) x[u] = nrow(32 * h + u, t & ~3)[t & 3];
          named_bar(pbar, 128);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const uint4 u = make_uint4(pack_h2(x[8 * ch + 0] * bt, x[8 * ch + 1] * bt),
                                       pack_h2(x[8 * ch + 2] * bt, x[8 * ch + 3] * bt),
                                       pack_h2(x[8 * ch + 4] * bt, x[8 * ch + 5] * bt),
                                       pack_h2(x[8 * ch + 6] * bt, x[8 * ch + 7] * bt));
            *reinterpret_cast<uint4 *>(scr + sw128_offset(t, 32 * h + ch * 8)) = u;
          }
        }
        fence_async_smem();
        named_bar(pbar, 128);
        // 5. W^T = Khat^T T (lanes i over d_k, 64 columns t): A = khat read MN-major, B = T K-major
        if (pt == 0) {
          tc_fence_after();
          const uint32_t kb0 = smem_u32(slot + kSlK), tb0 = smem_u32(scr);
          const uint32_t idw = idesc_f16(128, 64, 0, 1, 0);
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(tmP, sdesc_sw128(kb0 + kk * 2048, 8192, 1024), sdesc_sw128(tb0 + kk * 32, 16, 1024), idw,
                       kk > 0 ? 1u : 0u);
          mma_commit(&bar.g_mma[grp]);
        }
        if (!group_mma_wait()) break;
        // 6. W^T -> fp16 pairs in place (columns [0, 32) of the region)
        {
          float r[4][16];
#pragma unroll
          for (int e = 0; e < 4; ++e) tmem_ld16(tmP + lane_off + e * 16, r[e]);
          tmem_ld_wait();
#pragma unroll
          for (int hp = 0; hp < 2; ++hp) {
            uint32_t h[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              h[e] = pack_h2(r[2 * hp][2 * e], r[2 * hp][2 * e + 1]);
              h[8 + e] = pack_h2(r[2 * hp + 1][2 * e], r[2 * hp + 1][2 * e + 1]);
            }
            tmem_st16u(tmP + lane_off + hp * 16, h);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        named_bar(pbar, 128);
        // 7. M^T = -W^T Khat (lanes i, columns l over d_k) at column 32: A = W^T pairs (TMEM),
        //    B = khat MN-major (K = t)
        if (pt == 0) {
          tc_fence_after();
          const uint32_t kb0 = smem_u32(slot + kSlK);
          const uint32_t idm = idesc_f16(128, dk, 0, 0, 1);
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ts(tmP + 32, tmP + kk * 8, sdesc_sw128(kb0 + kk * 2048, 8192, 1024), idm, kk > 0 ? 1u : 0u);
          mma_commit(&bar.g_mma[grp]);
        }
        if (!group_mma_wait()) break;
        // 8. M^T -> negated fp16 pairs in place (columns [32, 32 + d_k / 2))
#pragma unroll 1
        for (int cb = 0; cb < nkd; cb += 2) {
          const bool two = cb + 1 < nkd;
          float r[2][16];
          tmem_ld16(tmP + 32 + lane_off + cb * 16, r[0]);
          if (two) tmem_ld16(tmP + 32 + lane_off + cb * 16 + 16, r[1]);
          tmem_ld_wait();
          uint32_t h[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            h[e] = pack_h2(-r[0][2 * e], -r[0][2 * e + 1]);
            h[8 + e] = two ? pack_h2(-r[1][2 * e], -r[1][2 * e + 1]) : 0u;
          }
          if (two) {
            tmem_st16u(tmP + 32 + lane_off + cb * 8, h);
          } else {
            const uint32_t h8[8] = {h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7]};
            tmem_st8u(tmP + 32 + lane_off + cb * 8, h8);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(pbar, 128);
        if (pt == 0) mbar_arrive_only(&bar.prep_ready[grp]);
      }
    }
    if (pt == 0) {  // every MMA of this group has completed before TMEM is released
      mma_commit(&bar.drain);
    }
  } else {
    // ============================================================ chain, chain step, read-out
    regs_inc<136>();
    const int row = tid & 127;              // TMEM lane of this thread
    const bool right = warp >= 4;           // warps 4-7: the B columns of Y / the second half of S columns
    uint8_t *ycp = sm + lay.off_y;
    uint32_t yph = 0, fph = 0, sph = 0;     // phases of y_mma, fr_bar, s_full
    uint32_t rt = 0;                        // read-out tiles of earlier frames
    uint32_t qi = 0;                        // q tiles issued (thread 0)
    bool s_pending = false;                 // thread 0: S bulk copies issued, not yet waited for
    int frames = 0;
    bool failed = false;
    uint32_t g = 0;
    const uint32_t id_y = idesc_f16(128, (int)lay.ny, 0, 0, 1);   // M^T (TMEM) x Ycopy (MN-major)
    const uint32_t id_wv = idesc_f16(128, dv, 0, 0, 1);           // W^T (TMEM) x V (MN-major)
    const uint32_t id_s = idesc_f16(128, dv, 0, 0, 1);            // alpha A (K-major) x S image (MN-major)
    const uint32_t id_o = idesc_f16(128, qt, 0, 1, 0);            // S_f image (MN-major) x q (K-major): O^T
    const int h = (nvc + 1) / 2;                                  // S column chunks of warps 0-3
    const int sc0 = right ? h : 0, sc1 = right ? nvc : h;
    float ymax = 0.f;  // largest |value| written as an fp16 operand (range check)

    auto issue_q = [&](int f, int bh, int t0) {  // thread 0: q tile (qt tokens, both column blocks)
      const int bq = qi % kQBuf;
      uint8_t *qb = sm + lay.off_q + bq * lay.qtile;
      mbar_expect_tx(&bar.q_full[bq], lay.qtile);
      tma_load_4d(qb, &tmap_q, &bar.q_full[bq], 0, t0, f, bh);
      tma_load_4d(qb + lay.qtile / 2, &tmap_q, &bar.q_full[bq], 64, t0, f, bh);
      ++qi;
    };

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
      const int f = tk / BH, bh = tk - (tk / BH) * BH;
      const float a_raw = p.alpha[(long)bh * F + f];
      const float alpha = p.gates_are_logits ? gate_alpha(a_raw) : a_raw;
      const long uidx = (long)bh * F + f;  // this frame's flag and published state

      // ---- Y <- [I | 0] in TMEM and in the fp16 copy (every lane takes part in the TMEM
      //      stores, which the warp executes together; rows past d_k are never read)
      {
        const int col0 = right ? dk : 0;
        const int n16 = right ? nvc : nkd;
#pragma unroll 1
        for (int cb = 0; cb < n16; ++cb) {
          float r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = (!right && cb * 16 + e == row) ? 1.f : 0.f;
          tmem_st16(tmem + lane_off + col0 + cb * 16, r);
          const int col = col0 + cb * 16;
          if (row < dk) st_row16_f16(ycp + (col >> 6) * lay.yb, row, col & 63, r);
        }
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      named_bar(1, kChain);

      // ---- the frame's chunks: Y += M^T Ycopy (+ W^T V on the B columns)
      for (int c = 0; c < nch; ++c, ++g) {
        const int s = (int)(g % kSlots);
        const int grp = (int)(g & 1u);
        const uint32_t tmP = tmem + lay.ny + (uint32_t)grp * lay.prep_cols;
        int cbad = 0;
        if (tid == 0) {
          if (!mbar_wait(&bar.prep_ready[grp], (g >> 1) & 1u, lim)) cbad = 1;
          tc_fence_after();
          const uint32_t yb0 = smem_u32(ycp);
          for (int kk = 0; kk < nkd; ++kk)
            mma_f16_ts(tmem, tmP + 32 + kk * 8, sdesc_sw128(yb0 + kk * 2048, lay.yb, 1024), id_y, 1u);
          const uint32_t vb0 = smem_u32(sm + lay.off_slot + s * kSlotBytes + kSlV);
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ts(tmem + dk, tmP + kk * 8, sdesc_sw128(vb0 + kk * 2048, 8192, 1024), id_wv, 1u);
          mma_commit(&bar.y_mma);
          mma_commit(&bar.slot_free[s]);
          mma_commit(&bar.chain_done[grp]);
          if (c == (nch > 4 ? nch - 4 : 0)) {  // the frame's q tiles towards L2 for the read-out
            for (int t0 = 0; t0 < L; t0 += qt) {
              tma_prefetch_l2_4d(&tmap_q, 0, t0, f, bh);
              tma_prefetch_l2_4d(&tmap_q, 64, t0, f, bh);
            }
          }
        }
        {
          int bad = cbad;
          if (tid == 0) bad |= !mbar_wait(&bar.y_mma, yph, lim);
          yph ^= 1u;
          if (bar_sync_or(1, kChain, bad || *abort_flag)) {
            failed = true;
            break;
          }
        }
        tc_fence_after();
        // slot s is free (its chunk's MMAs are done): chunk c + 3 goes there
        if (tid == 0 && c + kSlots < nch && !issue_kv(g + kSlots, f, bh, c + kSlots)) {
          *abort_flag = 1;
          latch_status(p.status, GDN_ERR_TIMEOUT);
        }
        // Y -> fp16 copy (the B operand of the next chunk).  After the last chunk only
        // alpha_f A_f is copied (the chain step's A operand); B_f stays in TMEM.
        const bool last = c + 1 == nch;
        if (!(last && right)) {
          const float sc = last ? alpha : 1.f;
          const int col0 = right ? dk : 0;
          const int n16 = right ? nvc : nkd;
#pragma unroll 1
          for (int cb = 0; cb < n16; cb += 2) {
            const bool two = cb + 1 < n16;
            float r[2][16];
            tmem_ld16(tmem + lane_off + col0 + cb * 16, r[0]);
            if (two) tmem_ld16(tmem + lane_off + col0 + cb * 16 + 16, r[1]);
            tmem_ld_wait();
            if (row < dk) {
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                if (e == 1 && !two) break;
                const int col = col0 + (cb + e) * 16;
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                  r[e][x] *= sc;
                  ymax = fmaxf(ymax, fabsf(r[e][x]));
                }
                st_row16_f16(ycp + (col >> 6) * lay.yb, row, col & 63, r[e]);
              }
            }
          }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(1, kChain);
      }
      if (bar_sync_or(1, kChain, failed ? 1 : 0)) {
        failed = true;
        break;
      }
      if (out_of_f16_range(ymax)) latch_status(p.status, GDN_ERR_RANGE);

      // ---- chain step: S_f = B_f + (alpha A_f) S_{f-1}, S_{f-1} as fp16 high + low images
      const bool chained = f > 0;
      const bool have_prev = chained || p.state_in != nullptr;
      if (chained) {
        int bad = 0;
        if (tid == 0) {
          bad = !wait_flag(p.ws.flags + uidx - 1, 1, lim);
          if (!bad) {
            fence_async_global();  // the producer's generic stores before this thread's async-proxy reads
            const uint8_t *img = reinterpret_cast<const uint8_t *>(p.ws.states) + (uidx - 1) * 2 * (long)lay.s_img;
            mbar_expect_tx(&bar.s_full[0], lay.s_img);
            bulk_load(sm + lay.off_slo, img + lay.s_img, lay.s_img, &bar.s_full[0]);
            mbar_expect_tx(&bar.s_full[1], lay.s_img);
            bulk_load(sm + lay.off_shi, img, lay.s_img, &bar.s_full[1]);
            s_pending = true;
          }
        }
        if (bar_sync_or(1, kChain, bad || *abort_flag)) {
          failed = true;
          break;
        }
      } else if (p.state_in != nullptr) {
        // the caller's fp32 S[l][j]: row l = this thread's lane, its half of the columns
        if (row < dk) {
          const float *src = p.state_in + ((long)bh * dk + row) * dv;
#pragma unroll 1
          for (int cb = sc0; cb < sc1; ++cb) {
            float hi[16], lo[16];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 v4 = __ldg(reinterpret_cast<const float4 *>(src + cb * 16 + e));
              const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
              for (int z = 0; z < 4; ++z) {
                hi[e + z] = __half2float(__float2half_rn(vv[z]));
                lo[e + z] = vv[z] - hi[e + z];
                ymax = fmaxf(ymax, fabsf(vv[z]));
              }
            }
            const int col = cb * 16;
            st_row16_f16(sm + lay.off_shi + (col >> 6) * lay.yb, row, col & 63, hi);
            st_row16_f16(sm + lay.off_slo + (col >> 6) * lay.yb, row, col & 63, lo);
          }
        }
        if (out_of_f16_range(ymax)) latch_status(p.status, GDN_ERR_RANGE);
        fence_async_smem();
      }
      tc_fence_before();
      named_bar(1, kChain);
      if (have_prev) {
        int bad = 0;
        if (tid == 0) {
          if (chained) {
            bad = !mbar_wait(&bar.s_full[0], sph, lim) || !mbar_wait(&bar.s_full[1], sph, lim);
            if (!bad) {
              sph ^= 1u;
              s_pending = false;
            }
          }
          tc_fence_after();
          const uint32_t ab = smem_u32(ycp);
          const uint32_t img[2] = {smem_u32(sm + lay.off_slo), smem_u32(sm + lay.off_shi)};
          for (int part = 0; part < 2; ++part)
            for (int kk = 0; kk < nkd; ++kk)
              mma_f16_ss(tmem + dk, sdesc_sw128(ab + (kk >> 2) * lay.yb + (kk & 3) * 32, 16, 1024),
                         sdesc_sw128(img[part] + kk * 2048, lay.yb, 1024), id_s, 1u);
          mma_commit(&bar.fr_bar);
          if (!bad) bad = !mbar_wait(&bar.fr_bar, fph, lim);
        }
        fph ^= 1u;
        if (bar_sync_or(1, kChain, bad || *abort_flag)) {
          failed = true;
          break;
        }
        tc_fence_after();
      }

      // ---- publish S_f: fp16 high and low images for the next frame (bulk-copied by its
      //      CTA), the high image also as this frame's read-out operand, state_out at the end
      {
        uint8_t *img = reinterpret_cast<uint8_t *>(p.ws.states) + uidx * 2 * (long)lay.s_img;
        float *sout = (f == F - 1 && p.state_out) ? p.state_out + ((long)bh * dk + row) * dv : nullptr;
        float smax = 0.f;
#pragma unroll 1
        for (int cb = sc0; cb < sc1; ++cb) {
          float r[16];
          tmem_ld16(tmem + lane_off + dk + cb * 16, r);
          tmem_ld_wait();
          if (row < dk) {
            float hi[16], lo[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              hi[e] = __half2float(__float2half_rn(r[e]));
              lo[e] = r[e] - hi[e];
              smax = fmaxf(smax, fabsf(r[e]));
            }
            const int col = cb * 16;
            const uint32_t off = (col >> 6) * lay.yb;
            uint4 hw[2], lw[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              hw[z] = make_uint4(pack_h2(hi[8 * z + 0], hi[8 * z + 1]), pack_h2(hi[8 * z + 2], hi[8 * z + 3]),
                                 pack_h2(hi[8 * z + 4], hi[8 * z + 5]), pack_h2(hi[8 * z + 6], hi[8 * z + 7]));
              lw[z] = make_uint4(pack_h2(lo[8 * z + 0], lo[8 * z + 1]), pack_h2(lo[8 * z + 2], lo[8 * z + 3]),
                                 pack_h2(lo[8 * z + 4], lo[8 * z + 5]), pack_h2(lo[8 * z + 6], lo[8 * z + 7]));
              const uint32_t o16 = off + sw128_offset(row, (col & 63) + 8 * z);
              *reinterpret_cast<uint4 *>(img + o16) = hw[z];
              *reinterpret_cast<uint4 *>(img + lay.s_img + o16) = lw[z];
              *reinterpret_cast<uint4 *>(sm + lay.off_sf + o16) = hw[z];
            }
            if (sout) {
#pragma unroll
              for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4 *>(sout + col + e) = make_float4(r[e], r[e + 1], r[e + 2], r[e + 3]);
            }
          }
        }
        if (out_of_f16_range(smax)) latch_status(p.status, GDN_ERR_RANGE);
      }
      __threadfence();
      fence_async_smem();
      tc_fence_before();
      named_bar(1, kChain);
      if (tid == 0 && ticket != p.withhold) st_release(p.ws.flags + uidx, 1);
      // the next ticket, and its first k, v loads (the prep groups run ahead into it
      // while this frame is read out)
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

      // ---- read-out O_f = Q_f S_f in qt-token tiles: O^T = S_f^T Q^T into TMEM buffer n & 1
      //      (columns [b qt, (b+1) qt)); q tiles come through kQBuf shared-memory buffers
      const int nt = (L + qt - 1) / qt;
      if (warp < 4) {
        // warps 0-3 convert each q tile to fp16 in place (8 16-byte chunks per thread); thread 0
        // also issues the q loads (kQBuf ahead) and each tile's MMAs
        if (tid == 0) {
          tc_fence_after();
          for (int n = 0; n < nt && n < kQBuf; ++n) issue_q(f, bh, n * qt);
        }
        for (int n = 0; n < nt; ++n) {
          const uint32_t gt = rt + n, qb = gt % kQBuf, qph = (gt / kQBuf) & 1u;
          const uint32_t b = gt & 1u, ph = (gt >> 1) & 1u;
          {
            const int bad = tid == 0 ? !mbar_wait(&bar.q_full[qb], qph, lim) : 0;
            if (bar_sync_or(6, 128, bad || *abort_flag)) {
              if (bad) {
                *abort_flag = 1;
                latch_status(p.status, GDN_ERR_TIMEOUT);
              }
              break;
            }
          }
          if (tid == 0) bar.q_used = gt + 1;
          uint4 *qv = reinterpret_cast<uint4 *>(sm + lay.off_q + qb * lay.qtile);
          float qmax = 0.f;
          const int nq16 = (int)(lay.qtile / 16);
#pragma unroll 2
          for (int i0 = 0; i0 < nq16; i0 += 4 * 128) {
            uint4 u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (i0 + e * 128 + tid < nq16) u[e] = qv[i0 + e * 128 + tid];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (i0 + e * 128 + tid < nq16) qv[i0 + e * 128 + tid] = bf16x8_to_f16x8(u[e], qmax);
          }
          if (out_of_f16_range(qmax)) latch_status(p.status, GDN_ERR_RANGE);
          fence_async_smem();
          named_bar(6, 128);
          if (tid == 0) {
            int bad = gt >= 2 && !mbar_wait(&bar.o_free[b], ph ^ 1u, lim);  // tile n - 2 has left buffer b
            if (!bad) {
              tc_fence_after();
              const uint32_t q0 = smem_u32(sm + lay.off_q + qb * lay.qtile), sf = smem_u32(sm + lay.off_sf);
              for (int kk = 0; kk < nkd; ++kk)
                mma_f16_ss(tmem + b * qt, sdesc_sw128(sf + kk * 2048, lay.yb, 1024),
                           sdesc_sw128(q0 + (kk >> 2) * (lay.qtile / 2) + (kk & 3) * 32, 16, 1024), id_o,
                           kk > 0 ? 1u : 0u);
              mma_commit(&bar.o_full[b]);
              // tile n - 1's MMAs done: its q buffer takes tile n - 1 + kQBuf
              if (n >= 1 && n - 1 + kQBuf < nt) {
                const uint32_t gp = gt - 1;
                bad = !mbar_wait(&bar.o_full[gp & 1u], (gp >> 1) & 1u, lim);
                if (!bad) issue_q(f, bh, (n - 1 + kQBuf) * qt);
              }
            }
            if (bad) {
              *abort_flag = 1;
              latch_status(p.status, GDN_ERR_TIMEOUT);
            }
          }
        }
      } else {
        // epilogue: O^T (lane = column j of o, TMEM columns = tokens of the tile) through the
        // staging rows into o's row-major layout (for each token the 32 lanes of a warp write
        // 32 consecutive floats), kStageTok tokens per bulk store of contiguous rows
        const int et = tid - 128;
        float *stg = reinterpret_cast<float *>(sm + lay.off_stage);
        for (int n = 0; n < nt; ++n) {
          const uint32_t gt = rt + n, b = gt & 1u, ph = (gt >> 1) & 1u;
          bool stop_ro = false;
          for (int hh = 0; hh < qt / kStageTok && !stop_ro; ++hh) {
            {
              int bad = (et == 0 && hh == 0) ? !mbar_wait(&bar.o_full[b], ph, lim) : 0;
              if (et == 0) bulk_wait_read();  // the previous bulk store has read the staging rows
              if (bar_sync_or(7, 128, bad || *abort_flag)) {
                if (bad) {
                  *abort_flag = 1;
                  latch_status(p.status, GDN_ERR_TIMEOUT);
                }
                stop_ro = true;
                break;
              }
            }
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < kStageTok / 16; ++cb) {
              float r[16];
              tmem_ld16(tmem + lane_off + b * qt + hh * kStageTok + cb * 16, r);
              tmem_ld_wait();
              if (row < dv) {
#pragma unroll
                for (int z = 0; z < 16; ++z) stg[(cb * 16 + z) * dv + row] = r[z];
              }
            }
            tc_fence_before();
            fence_async_smem();
            named_bar(7, 128);
            if (et == 0) {
              if (hh + 1 == qt / kStageTok) mbar_arrive_only(&bar.o_free[b]);
              const int t0 = n * qt + hh * kStageTok;
              const int nv = L - t0 < kStageTok ? L - t0 : kStageTok;  // tokens inside the frame
              if (nv > 0) {
                bulk_store(p.o + ((long)bh * N + (long)f * L + t0) * dv, stg, (uint32_t)(nv * dv * 4));
                bulk_commit();
              }
            }
          }
          if (stop_ro) break;
        }
      }
      rt += (uint32_t)nt;
      if (tid == 128) bulk_wait_read();  // the next frame's Y copy overwrites the staging rows
      if (bar_sync_or(1, kChain, *abort_flag)) {
        failed = true;
        break;
      }
    }
    if (failed) {
      if (tid == 0) latch_status(p.status, GDN_ERR_TIMEOUT);  // the first code latched wins
      *abort_flag = 1;
    }
    if (tid == 128) bulk_wait_all();  // o rows written before the CTA exits
    named_bar(1, kChain);
    if (tid == 0) {
      // loads still in flight complete before the CTA exits: the last k, v load of each
      // slot, the q tiles no converter took, the S images not waited for
      const uint32_t n = bar.loads;
      for (uint32_t gg = n > (uint32_t)kSlots ? n - kSlots : 0u; gg < n; ++gg)
        mbar_wait(&bar.kv_full[gg % kSlots], (gg / kSlots) & 1u, lim);
      for (uint32_t gq = bar.q_used; gq < qi; ++gq) mbar_wait(&bar.q_full[gq % kQBuf], (gq / kQBuf) & 1u, lim);
      if (s_pending) {
        mbar_wait(&bar.s_full[0], sph, lim);
        mbar_wait(&bar.s_full[1], sph, lim);
      }
      mma_commit(&bar.drain);
    }
  }
  // every MMA issued by thread 0 and the two prep leaders has completed
  if (tid == 0 || tid == kChain || tid == kChain + 128) mbar_wait(&bar.drain, 0, lim);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace pf

bool gdn_pform_supported(int dk, int dv) { return pf::make_layout(dk, dv).ok != 0; }

// bytes of one published frame state: fp16 high and low images of d_k rows x d_v columns
size_t gdn_pform_state_bytes(int dk, int dv) {
  const pf::Layout l = pf::make_layout(dk, dv);
  return l.ok ? 2 * (size_t)l.s_img : 0;
}

cudaError_t launch_gdn_pform(const GdnParams &p, int grid, cudaStream_t st) {
  using namespace pf;
  const Layout lay = make_layout(p.dk, p.dv);
  if (!lay.ok) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!tc::make_bf16_map(&mq, p.q, p.dk, p.L, p.F, BH, (int)lay.qt) || !tc::make_bf16_map(&mk, p.k, p.dk, p.L, p.F, BH, 64) ||
      !tc::make_bf16_map(&mv, p.v, p.dv, p.L, p.F, BH, 64))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gdn_pform_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.smem);
  if (e != cudaSuccess) return e;
  gdn_pform_kernel<<<grid, kThreads, lay.smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn
