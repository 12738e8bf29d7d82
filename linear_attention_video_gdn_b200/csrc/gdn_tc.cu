// Frame-wise Gated DeltaNet on tcgen05 tensor cores (bf16 q, k, v; fp32 state).
//
// Source of the method: SANA-WM GeekNews summary, "Core design and generation
// pipeline" (frame-wise Gated DeltaNet); dothoosh.com SANA-WM article (fixed-
// size recurrent state).  Update rule per token: S <- S - beta khat (S^T khat
// - v)^T after a per-frame decay S <- alpha S; every token of a frame reads
// o = S^T q with the state after the whole frame.
//
// Work unit = one (b, h, f) frame, taken from a ticket counter (f-major) by a
// persistent CTA.  For its frame the CTA builds the frame map
//     S_f = A_f (alpha_f S_{f-1}) + B_f,
// A_f = ordered product of (I - beta_t khat_t khat_t^T), B_f = the frame's
// update from a zero state, by running the delta rule on Y = [A | B] from
// [I | 0] with targets [0 | V], chunked 64 tokens at a time in the UT form
//     R = [0 | V] - Khat Y,   Y <- Y + Khat^T T R = Y + W^T R,
//     T = (I + N)^-1 diag(beta),  N = strict_lower(diag(beta) Khat Khat^T),
//     W = T^T Khat = diag(beta) Z,  (I + N^T) Z = Khat  (back substitution),
// kept transposed in TMEM (lanes = columns of A and B, fp32).  Only the
// d x d chain step S_f = ... waits on the previous frame's published state.
// Then O_f = Q_f S_f.
//
// Warp roles (384 threads):
//   warps 0-3  "tile A" and warps 4-7 "tile B": two independent chains, one
//              per 128-lane TMEM tile of Y^T (A^T rows, B^T rows).  Per chunk
//              each runs R^T = [0 ; V^T] - Y^T Khat^T and Y^T += R^T W on
//              tcgen05 with a TMEM -> fp16 shared-memory conversion after
//              each; the first thread of each issues its MMAs.  Together they
//              run the chain step, the read-out MMAs and the fp32 epilogue.
//   warps 8-11 "prep": TMA loads of k, v; key normalisation (fp16 khat);
//              Gram matrix Khat Khat^T on tcgen05; the back substitution for
//              W on CUDA cores (one thread per d_k column).  Runs up to two
//              chunks ahead.
// Operands that are not exact in bf16 (khat, Y, R, U, T, S, q) enter the
// tensor cores as fp16 (11-bit significands); all accumulation is fp32.
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {

constexpr int kGThreads = 384;  // 8 chain warps + 1 prep warpgroup
constexpr int kChain = 256;  // warps 0-7
constexpr int kC = 64;       // tokens per chunk

// shared memory map (bytes from the 1024-aligned base)
constexpr uint32_t OFF_MIRROR = 0;         // 64 KB: Y^T as fp16, [tile][k-block][128 rows][128 B]
constexpr uint32_t OFF_RU = 65536;         // 32 KB: R^T fp16, [tile][128 rows][128 B]
constexpr uint32_t OFF_KHAT = 98304;       // 48 KB: khat ring, [k-block][3 slots][64 rows][128 B]
constexpr uint32_t KHAT_KB_STRIDE = 24576;
constexpr uint32_t OFF_V = 147456;         // 32 KB: v ring (bf16, raw), [slot][dv-block][64 rows][128 B]
constexpr uint32_t OFF_W = 180224;         // 32 KB: W ring fp16, [slot][128 rows i][128 B (64 tokens)];
                                           //        while the prep group works on a slot it first holds
                                           //        N (fp32 64 x 64, float4-XOR-swizzled rows)
constexpr uint32_t OFF_I = 212992;         // 8 KB: identity 64 x 64 bf16 (K-major)
constexpr uint32_t OFF_NHL = 221184;       // 4 KB: fp16 block N[32 + u][t] (t, u < 32), rows t, K-major
constexpr uint32_t OFF_BAR = 225280;       // barriers and small state
// read-out phase aliases
constexpr uint32_t OFF_S16 = OFF_MIRROR;           // S_f as fp16 B operand [k-block][128 rows j][128 B]
constexpr uint32_t OFF_SPREV = OFF_MIRROR + 32768; // alpha S_{f-1}^T fp16 A operand (mirror tile-B region)
constexpr uint32_t OFF_Q0 = OFF_RU;                // q tile buffer 0 (32 KB)
constexpr uint32_t OFF_Q1 = OFF_MIRROR + 32768;    // q tile buffer 1 (32 KB, after the chain MMA)

struct Bars {
  uint64_t kv_full[2];
  uint64_t khat_ready[2];
  uint64_t w_ready[2];
  uint64_t slot_free[2];  // two arrivals: the last MMA of each tile chain on the slot
  uint64_t g_bar;
  uint64_t mma_bar[2];    // per tile chain
  uint64_t fr_bar;        // frame-level MMAs (chain step, read-out)
  uint64_t q_full[2];
  uint64_t tkt_bar[2];    // chain group -> prep group: the next frame's ticket is in ticket_ring
  uint32_t tmem_base;
  int abort;
  int ticket_ring[4];
  __align__(16) float beta[2][64];
};
constexpr size_t kGdnSmemBytes = OFF_BAR + sizeof(Bars) + 1024;

// TMEM columns
constexpr uint32_t TM_Y = 0;     // tile A [0,128), tile B [128,256)
constexpr uint32_t TM_RU = 256;  // R^T: tile A [256,320), tile B [320,384); read-out O uses [256,384)
constexpr uint32_t TM_G = 384;   // Gram matrix, 64 columns

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
  const long units = (long)BH * F;
  const long N = (long)F * L;
  const unsigned long long lim = p.spin_limit_ns;
  const int nkd = dk / 16;          // k-steps over d_k
  const int nch = (L + kC - 1) / kC;  // chunks per frame

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.kv_full[s], 1);
      mbar_init(&bar.khat_ready[s], 1);
      mbar_init(&bar.w_ready[s], 1);
      mbar_init(&bar.slot_free[s], 2);
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.mma_bar[s], 1);
    }
    mbar_init(&bar.g_bar, 1);
    mbar_init(&bar.fr_bar, 1);
    mbar_init(&bar.tkt_bar[0], 1);
    mbar_init(&bar.tkt_bar[1], 1);
    bar.abort = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  // identity (bf16, K-major 64 x 64) and zero pad slot of the khat ring
  for (int e = tid; e < 64 * 64; e += kGThreads) {
    const int r = e / 64, c = e % 64;
    *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_I + sw128_offset(r, c)) = __float2bfloat16(r == c ? 1.f : 0.f);
  }
  for (int e = tid; e < 2 * 8192 / 16; e += kGThreads) {
    const int kb = e / 512, w = e % 512;
    *reinterpret_cast<uint4 *>(sm + OFF_KHAT + kb * KHAT_KB_STRIDE + 2 * 8192 + w * 16) = make_uint4(0, 0, 0, 0);
  }
  fence_async_smem();
  if (warp == 0) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp >= 8) {
    // ============================================================ prep group
    regs_inc<232>();  // the back substitution keeps 64 values per thread live
    const int pt = tid - kChain;  // 0..127
    const int pbar = 2;           // named barrier of the prep group
    const uint32_t tmG = tmem + TM_G;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t g_phase = 0;
    uint32_t g = 0;          // chunks processed so far (all frames)
    float bnext = 0.f;       // gate input of token pt of the chunk whose loads are in flight
    bool bvalid = false;     // token pt exists in that chunk
    bool loaded = false;     // loads of chunk g already issued
    bool stop = false;
    // Issue the TMA loads of chunk c of frame (f, bh) into slot gg & 1 once the
    // chain group has released it, and prefetch its gates into bnext.
    auto issue_loads = [&](uint32_t gg, int f, int bh, int c) -> int {
      const int s = gg & 1;
      int bad = 0;
      if (pt == 0) {
        if (!mbar_wait(&bar.slot_free[s], ((gg >> 1) & 1u) ^ 1u, lim)) {
          bad = 1;
        } else {
          const int t0 = c * kC;
          mbar_expect_tx(&bar.kv_full[s], 32768);
          tma_load_4d(sm + OFF_KHAT + s * 8192, &tmap_k, &bar.kv_full[s], 0, t0, f, bh);
          tma_load_4d(sm + OFF_KHAT + KHAT_KB_STRIDE + s * 8192, &tmap_k, &bar.kv_full[s], 64, t0, f, bh);
          tma_load_4d(sm + OFF_V + s * 16384, &tmap_v, &bar.kv_full[s], 0, t0, f, bh);
          tma_load_4d(sm + OFF_V + s * 16384 + 8192, &tmap_v, &bar.kv_full[s], 64, t0, f, bh);
        }
      }
      if (pt < 64) {  // raw gate of the token; activated when stored (keeps the load latency off this path)
        const int t = c * kC + pt;
        bnext = t < L ? p.beta[(long)bh * N + (long)f * L + t] : 0.f;
        bvalid = t < L;
      }
      return bad;
    };
    for (int k = 0; !stop; ++k) {
      // the chain group takes each frame's ticket and hands it over
      {
        const int bad = (pt == 0) ? !mbar_wait(&bar.tkt_bar[k & 1], (k >> 1) & 1u, lim) : 0;
        if (bar_sync_or(pbar, 128, bad || *((volatile int *)&bar.abort))) {
          if (pt == 0 && bad) latch_status(p.status, GDN_ERR_TIMEOUT);
          bar.abort = 1;
          break;
        }
      }
      const int tk = bar.ticket_ring[k & 3];
      if (tk < 0) break;
      const int f = tk / BH;
      const int bh = tk % BH;
      for (int c = 0; c < nch; ++c, ++g) {
      const int s = g & 1;
      const uint32_t ph = (g >> 1) & 1u;
      int pbad = 0;
      if (!loaded) pbad = issue_loads(g, f, bh, c);
      if (pt < 64) bar.beta[s][pt] = bvalid ? (p.gates_are_logits ? gate_beta(bnext) : bnext) : 0.f;
      if (bar_sync_or(pbar, 128, pbad || *((volatile int *)&bar.abort))) {
        if (pt == 0 && pbad) latch_status(p.status, GDN_ERR_TIMEOUT);
        bar.abort = 1;
        stop = true;
        break;
      }
      if (bar_sync_or(pbar, 128, pt == 0 ? !mbar_wait(&bar.kv_full[s], ph, lim) : 0)) {
        if (pt == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
        bar.abort = 1;
        stop = true;
        break;
      }
      // 2. normalise keys in place: thread pt -> token pt/2, k-block pt%2
      {
        const int t = pt >> 1, kb = pt & 1;
        uint8_t *row = sm + OFF_KHAT + kb * KHAT_KB_STRIDE + s * 8192;
        float x[64];
        float ss = 0.f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 u = *reinterpret_cast<const uint4 *>(row + sw128_offset(t, ch * 8));
          const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 v2 = __bfloat1622float2(h[e]);
            x[ch * 8 + 2 * e] = v2.x;
            x[ch * 8 + 2 * e + 1] = v2.y;
            ss += v2.x * v2.x + v2.y * v2.y;
          }
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        const float inv = 1.0f / fmaxf(sqrtf(ss), kKeyNormEps);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 u = make_uint4(pack_h2(x[ch * 8] * inv, x[ch * 8 + 1] * inv),
                                     pack_h2(x[ch * 8 + 2] * inv, x[ch * 8 + 3] * inv),
                                     pack_h2(x[ch * 8 + 4] * inv, x[ch * 8 + 5] * inv),
                                     pack_h2(x[ch * 8 + 6] * inv, x[ch * 8 + 7] * inv));
          *reinterpret_cast<uint4 *>(row + sw128_offset(t, ch * 8)) = u;
        }
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(pbar, 128);
      // 3. khat ready; Gram matrix G = Khat Khat^T (rows: this chunk and the next slot)
      if (pt == 0) {
        mbar_arrive_only(&bar.khat_ready[s]);
        tc_fence_after();
        const uint32_t idg = idesc_f16(128, 64, 0, 0, 0);
        for (int kk = 0; kk < nkd; ++kk) {
          const uint32_t a = smem_u32(sm + OFF_KHAT + (kk >> 2) * KHAT_KB_STRIDE + s * 8192 + (kk & 3) * 32);
          mma_f16_ss(tmG, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), idg, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.g_bar);
      }
      // prefetch the next chunk of this frame while the Gram matrix is computed
      loaded = c + 1 < nch;
      const int nbad = loaded ? issue_loads(g + 1, f, bh, c + 1) : 0;
      const int gbad = pt == 0 ? !mbar_wait(&bar.g_bar, g_phase, lim) : 0;
      g_phase ^= 1u;
      if (bar_sync_or(pbar, 128, gbad || nbad)) {
        if (pt == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
        bar.abort = 1;
        stop = true;
        break;
      }
      tc_fence_after();
      // 4. Nt[t][u] = N[u][t] = beta_u G[u][t] for u > t.  G is symmetric, so lane
      //    t (the group's first two warps) reads row t of G and writes row t of Nt (fp32, float4
      //    index XOR (t & 15)); Nt occupies the W slot until step 5.
      float *Nt = reinterpret_cast<float *>(sm + OFF_W + s * 16384);
      if (pt < 64) {  // the group's first two warps hold TMEM lanes 0..63
        const int t = pt;  // lane
        float r[4][16];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tmem_ld16(tmG + lane_off + cb * 16, r[cb]);
        tmem_ld_wait();
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            const int u = cb * 16 + e;
            const float4 b4 = *reinterpret_cast<const float4 *>(&bar.beta[s][u]);
            float4 o4;
            o4.x = (u + 0 > t) ? b4.x * r[cb][e + 0] : 0.f;
            o4.y = (u + 1 > t) ? b4.y * r[cb][e + 1] : 0.f;
            o4.z = (u + 2 > t) ? b4.z * r[cb][e + 2] : 0.f;
            o4.w = (u + 3 > t) ? b4.w * r[cb][e + 3] : 0.f;
            *reinterpret_cast<float4 *>(Nt + t * 64 + (((u >> 2) ^ (t & 15)) << 2)) = o4;
          }
        if (t < 32) {
          // B operand of the cross-term MMA: row t holds N[32 + u][t] = beta_{32+u} G[t][32+u]
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t h4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int u = 32 + ch * 8 + 2 * e;
              h4[e] = pack_h2(bar.beta[s][u] * r[u >> 4][u & 15], bar.beta[s][u + 1] * r[(u + 1) >> 4][(u + 1) & 15]);
            }
            *reinterpret_cast<uint4 *>(sm + OFF_NHL + sw128_offset(t, ch * 8)) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
          }
        }
      }
      tc_fence_before();
      named_bar(pbar, 128);
      // 5. W = diag(beta) Z with (I + N^T) Z = Khat: thread i < d_k owns column i
      //    of Z and back-substitutes from the last token,
      //        z[t] = khat[t][i] - sum_{u > t} N[u][t] z[u],
      //    in two halves: rows 63..32 on CUDA cores; the hi -> lo coupling
      //    sum_{u >= 32} N[u][t] z[u] for t < 32 as one tcgen05 MMA (z_hi^T in
      //    TMEM as A, the fp16 N block as B); then rows 31..0.
      float z[64];
      const bool solver = pt < dk;
      if (solver) {
        const int i = pt;
        const uint8_t *kt = sm + OFF_KHAT + (i >> 6) * KHAT_KB_STRIDE + s * 8192;
#pragma unroll
        for (int t = 0; t < 64; ++t) z[t] = __half2float(*reinterpret_cast<const __half *>(kt + sw128_offset(t, i & 63)));
      }
      // rows in blocks of four: the four rows' sums over already final z[u] are
      // independent (two partial sums each), then the 4 x 4 triangle in order
      auto solve_rows = [&](int hi_block, int u_end) {
#pragma unroll
        for (int tb = 60; tb >= 0; tb -= 4) {
          if ((tb >= 32) != (hi_block != 0)) continue;
          float a[4][2];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            a[r][0] = z[tb + r];
            a[r][1] = 0.f;
          }
#pragma unroll
          for (int u4 = tb + 4; u4 < 64; u4 += 4) {
            if (u4 >= u_end) continue;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const int t = tb + r;
              const float4 n4 = *reinterpret_cast<const float4 *>(Nt + t * 64 + (((u4 >> 2) ^ (t & 15)) << 2));
              a[r][0] = fmaf(-n4.x, z[u4 + 0], a[r][0]);
              a[r][1] = fmaf(-n4.y, z[u4 + 1], a[r][1]);
              a[r][0] = fmaf(-n4.z, z[u4 + 2], a[r][0]);
              a[r][1] = fmaf(-n4.w, z[u4 + 3], a[r][1]);
            }
          }
#pragma unroll
          for (int r = 3; r >= 0; --r) {
            const int t = tb + r;
            const float4 n4 = *reinterpret_cast<const float4 *>(Nt + t * 64 + (((tb >> 2) ^ (t & 15)) << 2));
            float v = a[r][0] + a[r][1];
            if (r < 3) v = fmaf(-n4.w, z[tb + 3], v);
            if (r < 2) v = fmaf(-n4.z, z[tb + 2], v);
            if (r < 1) v = fmaf(-n4.y, z[tb + 1], v);
            z[t] = v;
          }
        }
      };
      if (solver) solve_rows(1, 64);
      {
        // z_hi^T as the MMA's A operand: lane i, 16 columns of packed fp16 (zeros past d_k)
        uint32_t hz[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) hz[e] = solver ? pack_h2(z[32 + 2 * e], z[33 + 2 * e]) : 0u;
        tmem_st16u(tmG + lane_off, hz);
        tmem_st_wait();
      }
      tc_fence_before();
      named_bar(pbar, 128);
      if (pt == 0) {
        tc_fence_after();
        const uint32_t idc = idesc_f16(128, 32, 0, 0, 0);
        const uint32_t nb = smem_u32(sm + OFF_NHL);
        for (int kk = 0; kk < 2; ++kk)
          mma_f16_ts(tmG + 32, tmG + kk * 8, sdesc_sw128(nb + kk * 32, 16, 1024), idc, kk > 0 ? 1u : 0u);
        mma_commit(&bar.g_bar);
      }
      {
        const int cbad = pt == 0 ? !mbar_wait(&bar.g_bar, g_phase, lim) : 0;
        g_phase ^= 1u;
        if (bar_sync_or(pbar, 128, cbad)) {
          if (pt == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
          bar.abort = 1;
          stop = true;
          break;
        }
      }
      tc_fence_after();
      {
        float cr[2][16];
        tmem_ld16(tmG + 32 + lane_off, cr[0]);
        tmem_ld16(tmG + 48 + lane_off, cr[1]);
        tmem_ld_wait();
        if (solver) {
#pragma unroll
          for (int t = 0; t < 32; ++t) z[t] -= cr[t >> 4][t & 15];
          solve_rows(0, 32);
        }
      }
      named_bar(pbar, 128);  // every read of N is done before W overwrites it
      if (solver) {
        // row i of the K-major B operand W^T-as-(K = token, N = i): W[t][i] = beta_t z[t]
        uint8_t *wrow = sm + OFF_W + s * 16384;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = ch * 8 + 2 * e;
            w4[e] = pack_h2(bar.beta[s][t] * z[t], bar.beta[s][t + 1] * z[t + 1]);
          }
          *reinterpret_cast<uint4 *>(wrow + sw128_offset(pt, ch * 8)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_async_smem();
      named_bar(pbar, 128);
      if (pt == 0) mbar_arrive_only(&bar.w_ready[s]);
      }
    }
  } else {
    // ============================================================ chain group
    regs_dec<128>();
    const int tile = warp >> 2;           // 0: tile A (rows of A^T), 1: tile B (rows of B^T)
    const int row = tid & 127;            // TMEM lane / operand row within the tile
    const bool issuer = row == 0;         // threads 0 and 128 issue their tile's MMAs
    const int tbar = 3 + tile;            // named barrier of one tile chain (128 threads)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t tphase = 0;                  // phase of mma_bar[tile]
    uint32_t fphase = 0;                  // phase of fr_bar
    uint32_t qcount[2] = {0, 0};
    int frames = 0;
    bool failed = false;
    uint32_t g = 0;
    const uint32_t id_vi = idesc_f16(128, 64, 1, 1, 0);          // V^T (MN) x I (K), bf16
    const uint32_t id_r = idesc_f16(128, 64, 0, 0, 0, 1, 0);     // -(Y^T) x Khat^T, fp16
    const uint32_t id_y = idesc_f16(128, dk, 0, 0, 0);           // R^T x W (both K-major)
    const uint32_t id_s = idesc_f16(128, dk, 0, 0, 1);           // (alpha S^T) x A^T (MN)
    const uint32_t id_o = idesc_f16(128, 128, 0, 0, 0);          // S^T x Q^T (128 tokens)

    // Wait for this tile's MMAs: the issuing thread polls the mbarrier, the
    // others wait on the named barrier (which takes no issue slots from the
    // warps doing work).  False, for all 128 threads of the tile, on a
    // timeout, on `extra` from any of them, or once the prep group gave up.
    auto tile_wait = [&](int extra) -> bool {
      int bad = extra;
      if (issuer) bad |= !mbar_wait(&bar.mma_bar[tile], tphase, lim);
      tphase ^= 1u;
      return !bar_sync_or(tbar, 128, bad || *((volatile int *)&bar.abort));
    };
    // the same for frame-level MMAs, over all 256 chain threads
    auto frame_wait = [&](int extra) -> bool {
      int bad = extra;
      if (tid == 0) bad |= !mbar_wait(&bar.fr_bar, fphase, lim);
      fphase ^= 1u;
      return !bar_sync_or(1, kChain, bad || *((volatile int *)&bar.abort));
    };

    // The chain group takes the tickets: the first here, each next one right
    // after the current frame's state is published (before its read-out), and
    // hands each to the prep group.  A ticket is thus started a fixed read-out
    // time after it is taken, whatever the frame chain's waits were.
    if (tid == 0) {
      const long t = atomicAdd(p.ws.counter, 1);
      bar.ticket_ring[0] = (int)(t < units ? t : -1);
      mbar_arrive_only(&bar.tkt_bar[0]);
    }
    named_bar(1, kChain);
    for (;;) {
      const int tk = bar.ticket_ring[frames & 3];
      ++frames;
      if (tk < 0) break;
      {
        const int s = g & 1;
        const uint32_t ph = (g >> 1) & 1u;
        const int kbad = tid == 0 ? !mbar_wait(&bar.khat_ready[s], ph, lim) : 0;
        if (bar_sync_or(1, kChain, kbad)) {
          failed = true;
          break;
        }
      }
      const long ticket = tk;
      const int f = (int)(ticket / BH);
      const int bh = (int)(ticket % BH);

      // Y = [I | 0] in TMEM (fp32) and in the fp16 mirror, rows of this tile
      {
        const int rdim = tile == 0 ? dk : dv;
#pragma unroll 1
        for (int cb = 0; cb < nkd; ++cb) {
          float r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = (tile == 0 && cb * 16 + e == row && row < rdim) ? 1.f : 0.f;
          tmem_st16(tmem + TM_Y + tile * 128 + lane_off + cb * 16, r);
          store_row16_f16(sm + OFF_MIRROR + tile * 32768 + (cb >> 2) * 16384, row, (cb & 3) * 16, r);
        }
        tmem_st_wait();
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(tbar, 128);

      // ---- the frame's chunks, one independent chain per tile
      for (int c = 0; c < nch; ++c, ++g) {
        const int s = g & 1;
        const uint32_t ph = (g >> 1) & 1u;
        int cbad = 0;
        // R^T = [0 ; V^T] - Y^T Khat^T  (the V^T part for tile B only)
        if (issuer) {
          if (c > 0 && !mbar_wait(&bar.khat_ready[s], ph, lim)) cbad = 1;
          tc_fence_after();
          const uint32_t kh = smem_u32(sm + OFF_KHAT + s * 8192);
          const uint32_t mb = smem_u32(sm + OFF_MIRROR + tile * 32768);
          const uint32_t dR = tmem + TM_RU + tile * 64;
          if (tile == 1) {
            const uint32_t vb = smem_u32(sm + OFF_V + s * 16384);
            const uint32_t ib = smem_u32(sm + OFF_I);
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(dR, sdesc_sw128(vb + kk * 2048, 8192, 1024), sdesc_sw128(ib + kk * 32, 16, 1024), id_vi,
                         kk > 0 ? 1u : 0u);
          }
          for (int kk = 0; kk < nkd; ++kk) {
            const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t kho = (kk >> 2) * KHAT_KB_STRIDE + (kk & 3) * 32;
            mma_f16_ss(dR, sdesc_sw128(mb + ko, 16, 1024), sdesc_sw128(kh + kho, 16, 1024), id_r,
                       (tile == 1 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar.mma_bar[tile]);
        }
        if (!tile_wait(cbad)) { failed = true; break; }
        tc_fence_after();
        {
          float r[4][16];
#pragma unroll
          for (int cb = 0; cb < 4; ++cb) tmem_ld16(tmem + TM_RU + tile * 64 + lane_off + cb * 16, r[cb]);
          tmem_ld_wait();
#pragma unroll
          for (int cb = 0; cb < 4; ++cb) store_row16_f16(sm + OFF_RU + tile * 16384, row, cb * 16, r[cb]);
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(tbar, 128);
        // Y^T += R^T W ; the last MMA of this tile on slot s releases it
        if (issuer) {
          if (!mbar_wait(&bar.w_ready[s], ph, lim)) cbad = 1;
          tc_fence_after();
          const uint32_t rb = smem_u32(sm + OFF_RU + tile * 16384);
          const uint32_t wb = smem_u32(sm + OFF_W + s * 16384);
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(tmem + TM_Y + tile * 128, sdesc_sw128(rb + kk * 32, 16, 1024),
                       sdesc_sw128(wb + kk * 32, 16, 1024), id_y, 1u);
          mma_commit(&bar.mma_bar[tile]);
          mma_commit(&bar.slot_free[s]);
        }
        if (!tile_wait(cbad)) { failed = true; break; }
        tc_fence_after();
        // Y^T rows -> fp16 mirror (tile B's rows are not needed after the last chunk)
        if (c + 1 < nch || tile == 0) {
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {  // two batches of up to 4 column blocks
            float r[4][16];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (hb * 4 + e < nkd) tmem_ld16(tmem + TM_Y + tile * 128 + lane_off + (hb * 4 + e) * 16, r[e]);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (hb * 4 + e < nkd) store_row16_f16(sm + OFF_MIRROR + tile * 32768 + hb * 16384, row, e * 16, r[e]);
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

      // ---- chain step: S_f^T = B_f^T + (alpha S_{f-1}^T) A_f^T
      const int n3 = (L + 127) / 128;
      if (tid == 0) {
        // q tile 0 -> the R/U region (free now)
        mbar_expect_tx(&bar.q_full[0], 32768);
        tma_load_4d(sm + OFF_Q0, &tmap_q, &bar.q_full[0], 0, 0, f, bh);
        tma_load_4d(sm + OFF_Q0 + 16384, &tmap_q, &bar.q_full[0], 64, 0, f, bh);
      }
      const float a_raw = p.alpha[(long)bh * F + f];
      const float alpha = p.gates_are_logits ? gate_alpha(a_raw) : a_raw;
      const bool have_prev = f > 0 || p.state_in != nullptr;
      int bad = 0;
      if (tid == 0 && f > 0) bad = !wait_flag(p.ws.flags + (long)bh * F + (f - 1), 1, lim);
      if (bar_sync_or(1, kChain, bad)) {
        if (tid == 0) mbar_wait(&bar.q_full[0], qcount[0] & 1u, lim);  // drain the q load in flight
        failed = true;
        break;
      }
      if (have_prev) {
        // rows j of alpha * S_{f-1}^T (threads of both tiles split the d_k
        // columns); states are stored S[l][j] (d_v contiguous), so lanes j read
        // consecutive addresses
        const int j = row;
        const int half = tile;  // 0: k-block 0, 1: k-block 1
        const float *prev = f > 0 ? p.ws.states + ((long)bh * F + (f - 1)) * (long)dk * dv
                                  : p.state_in + (long)bh * dk * dv;
#pragma unroll 1
        for (int cb = half * 4; cb < half * 4 + 4; ++cb) {
          if (cb >= nkd) break;
          float r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = j < dv ? alpha * __ldcg(prev + (long)(cb * 16 + e) * dv + j) : 0.f;
          store_row16_f16(sm + OFF_SPREV + (cb >> 2) * 16384, j, (cb & 3) * 16, r);
        }
        fence_async_smem();
        named_bar(1, kChain);
        if (tid == 0) {
          tc_fence_after();
          const uint32_t sb = smem_u32(sm + OFF_SPREV);
          const uint32_t ab = smem_u32(sm + OFF_MIRROR);  // tile A of the mirror = A_f^T rows, read MN-major
          for (int kk = 0; kk < nkd; ++kk)
            mma_f16_ss(tmem + TM_Y + 128, sdesc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                       sdesc_sw128(ab + kk * 2048, 16384, 1024), id_s, 1u);
          mma_commit(&bar.fr_bar);
        }
        if (!frame_wait(0)) { failed = true; break; }
        tc_fence_after();
      }
      // S_f^T rows: publish fp32 as S[i][j] (lanes j write consecutive
      // addresses), state_out, fp16 operand for the read-out
      {
        const int j = row;
        const int half = tile;
        float *cur = p.ws.states + ((long)bh * F + f) * (long)dk * dv;
        float *sout = (f == F - 1 && p.state_out) ? p.state_out + (long)bh * dk * dv : nullptr;
#pragma unroll 1
        for (int cb = half * 4; cb < half * 4 + 4; ++cb) {
          if (cb >= nkd) break;
          float r[16];
          tmem_ld16(tmem + TM_Y + 128 + lane_off + cb * 16, r);
          tmem_ld_wait();
          if (j < dv) {
#pragma unroll
            for (int e = 0; e < 16; ++e) cur[(long)(cb * 16 + e) * dv + j] = r[e];
            if (sout) {
#pragma unroll
              for (int e = 0; e < 16; ++e) sout[(long)(cb * 16 + e) * dv + j] = r[e];
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = 0.f;
          }
          store_row16_f16(sm + OFF_S16 + (cb >> 2) * 16384, j, (cb & 3) * 16, r);
        }
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(1, kChain);
      if (tid == 0) {
        if (ticket != p.withhold) {
          __threadfence();
          st_release(p.ws.flags + (long)bh * F + f, 1);
        }
        const long t = atomicAdd(p.ws.counter, 1);
        bar.ticket_ring[frames & 3] = (int)(t < units ? t : -1);
        mbar_arrive_only(&bar.tkt_bar[frames & 1]);
        if (n3 > 1) {
          mbar_expect_tx(&bar.q_full[1], 32768);
          tma_load_4d(sm + OFF_Q1, &tmap_q, &bar.q_full[1], 0, 128, f, bh);
          tma_load_4d(sm + OFF_Q1 + 16384, &tmap_q, &bar.q_full[1], 64, 128, f, bh);
        }
      }

      // ---- read-out: O_f = Q_f S_f, 128 tokens per tile
      for (int qc = 0; qc < n3; ++qc) {
        const int b = qc & 1;
        uint8_t *qb = sm + (b == 0 ? OFF_Q0 : OFF_Q1);
        const int qbad = tid == 0 ? !mbar_wait(&bar.q_full[b], qcount[b] & 1u, lim) : 0;
        ++qcount[b];
        if (bar_sync_or(1, kChain, qbad)) { failed = true; break; }
        // bf16 -> fp16 in place
        for (int i = tid * 16; i < 32768; i += kChain * 16) {
          uint4 u = *reinterpret_cast<uint4 *>(qb + i);
          __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 v2 = __bfloat1622float2(h[e]);
            o[e] = pack_h2(v2.x, v2.y);
          }
          *reinterpret_cast<uint4 *>(qb + i) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_async_smem();
        named_bar(1, kChain);
        if (tid == 0) {
          tc_fence_after();
          // O^T = S_f^T Q^T: lanes = output columns j, TMEM columns = tokens
          const uint32_t a0 = smem_u32(sm + OFF_S16), b0 = smem_u32(qb);
          for (int kk = 0; kk < nkd; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_f16_ss(tmem + TM_RU, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024), id_o,
                       kk > 0 ? 1u : 0u);
          }
          mma_commit(&bar.fr_bar);
        }
        if (!frame_wait(0)) { failed = true; break; }
        tc_fence_after();
        if (tid == 0 && qc + 2 < n3) {
          mbar_expect_tx(&bar.q_full[b], 32768);
          tma_load_4d(qb, &tmap_q, &bar.q_full[b], 0, (qc + 2) * 128, f, bh);
          tma_load_4d(qb + 16384, &tmap_q, &bar.q_full[b], 64, (qc + 2) * 128, f, bh);
        }
        // epilogue: lane j holds O[t][j] for the tile's tokens t; warps 0-3
        // store tokens [0, 64), warps 4-7 tokens [64, 128); for each token a
        // warp writes 32 consecutive floats of row t
        {
          const int j = row;
          float *obase = p.o + ((long)bh * N + (long)f * L + (long)qc * 128) * dv + j;
          const int tl = L - qc * 128;  // tokens of this tile
#pragma unroll 1
          for (int tb = tile * 4; tb < tile * 4 + 4; ++tb) {
            float r[16];
            tmem_ld16(tmem + TM_RU + lane_off + tb * 16, r);
            tmem_ld_wait();
            if (j < dv) {
#pragma unroll
              for (int e = 0; e < 16; ++e)
                if (tb * 16 + e < tl) obase[(long)(tb * 16 + e) * dv] = r[e];
            }
          }
        }
        tc_fence_before();
        named_bar(1, kChain);
      }
      if (failed) break;
    }
    if (failed) {
      if (tid == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
      bar.abort = 1;
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

size_t gdn_tc_state_elems(int dk, int dv) { return (size_t)dk * dv; }

cudaError_t launch_gdn_tc(const GdnParams &p, int grid, cudaStream_t st) {
  using namespace tc;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_bf16_map(&mq, p.q, p.dk, p.L, p.F, BH, 128) || !make_bf16_map(&mk, p.k, p.dk, p.L, p.F, BH, 64) ||
      !make_bf16_map(&mv, p.v, p.dv, p.L, p.F, BH, 64))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(gdn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGdnSmemBytes);
  if (e != cudaSuccess) return e;
  gdn_tc_kernel<<<grid, kGThreads, kGdnSmemBytes, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn
