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
//     R = [0 | V] - Khat Y,   U = T R,   Y <- Y + Khat^T U,
//     T = (I + strict_lower(diag(beta) Khat Khat^T))^-1 diag(beta),
// kept transposed in TMEM (lanes = columns of A and B, fp32).  Only the
// d x d chain step S_f = ... waits on the previous frame's published state.
// Then O_f = Q_f S_f.
//
// Warp roles (384 threads):
//   warps 0-7  "chain": the three recurrence MMAs per chunk and their
//              TMEM -> fp16 shared-memory conversions, the chain step, the
//              read-out MMAs and the fp32 output epilogue.  Thread 0 issues
//              their tcgen05.mma and TMA loads of q.
//   warps 8-11 "prep": TMA loads of k, v; key normalisation (fp16 khat);
//              Gram matrix Khat Khat^T on tcgen05; the 64 x 64 triangular
//              solve for T on CUDA cores.  Runs up to two chunks ahead.
// Operands that are not exact in bf16 (khat, Y, R, U, T, S, q) enter the
// tensor cores as fp16 (11-bit significands); all accumulation is fp32.
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {

constexpr int kGThreads = 384;
constexpr int kChain = 256;  // warps 0-7
constexpr int kC = 64;       // tokens per chunk

// shared memory map (bytes from the 1024-aligned base)
constexpr uint32_t OFF_MIRROR = 0;         // 64 KB: Y^T as fp16, [tile][k-block][128 rows][128 B]
constexpr uint32_t OFF_RU = 65536;         // 32 KB: R^T / U^T fp16, [tile][128 rows][128 B]
constexpr uint32_t OFF_KHAT = 98304;       // 48 KB: khat ring, [k-block][3 slots][64 rows][128 B]
constexpr uint32_t KHAT_KB_STRIDE = 24576;
constexpr uint32_t OFF_V = 147456;         // 32 KB: v ring (bf16, raw), [slot][dv-block][64 rows][128 B]
constexpr uint32_t OFF_T = 180224;         // 16 KB: T ring fp16, [slot][64 rows][128 B]
constexpr uint32_t OFF_N = 196608;         // 17 KB: N = strict_lower(diag(beta) G) fp32, 64 rows x 68
constexpr uint32_t N_STRIDE = 68;
constexpr uint32_t OFF_I = 214016;         // 8 KB: identity 64 x 64 bf16 (K-major)
constexpr uint32_t OFF_BAR = 222208;       // barriers and small state
// read-out phase aliases
constexpr uint32_t OFF_S16 = OFF_MIRROR;           // S_f as fp16 B operand [k-block][128 rows j][128 B]
constexpr uint32_t OFF_SPREV = OFF_MIRROR + 32768; // alpha S_{f-1}^T fp16 A operand (mirror tile-B region)
constexpr uint32_t OFF_Q0 = OFF_RU;                // q tile buffer 0 (32 KB)
constexpr uint32_t OFF_Q1 = OFF_MIRROR + 32768;    // q tile buffer 1 (32 KB, after the chain MMA)

struct Bars {
  uint64_t kv_full[2];
  uint64_t khat_ready[2];
  uint64_t t_ready[2];
  uint64_t slot_free[2];
  uint64_t g_bar;
  uint64_t mma_bar;
  uint64_t q_full[2];
  uint32_t tmem_base;
  int abort;
  int ticket_ring[4];
  __align__(16) float beta[2][64];
};
constexpr size_t kGdnSmemBytes = OFF_BAR + sizeof(Bars) + 1024;

// TMEM columns
constexpr uint32_t TM_Y = 0;     // tile A [0,128), tile B [128,256)
constexpr uint32_t TM_RU = 256;  // tile A [256,320), tile B [320,384); read-out O uses [256,384)
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
      mbar_init(&bar.t_ready[s], 1);
      mbar_init(&bar.slot_free[s], 1);
      mbar_init(&bar.q_full[s], 1);
    }
    mbar_init(&bar.g_bar, 1);
    mbar_init(&bar.mma_bar, 1);
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
    const int pt = tid - kChain;  // 0..127
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t g_phase = 0;
    long ticket = -1;
    int f = 0, bh = 0, c = 0;
    int frames = 0;
    for (uint32_t g = 0;; ++g) {
      const int s = g & 1;
      const uint32_t ph = (g >> 1) & 1u;
      // next chunk of the current frame, or the next frame
      if (ticket < 0 || c == nch) {
        if (pt == 0) {
          const long t = atomicAdd(p.ws.counter, 1);
          bar.ticket_ring[frames & 3] = (int)(t < units ? t : -1);
        }
        named_bar(2, 128);
        const int t = bar.ticket_ring[frames & 3];
        ++frames;
        if (t < 0) {
          // end of work: wake the chain group on this slot without loading
          if (pt == 0) {
            bool ok = mbar_wait(&bar.slot_free[s], ph ^ 1u, lim);
            (void)ok;
            mbar_arrive_only(&bar.khat_ready[s]);
          }
          break;
        }
        ticket = t;
        f = (int)(ticket / BH);
        bh = (int)(ticket % BH);
        c = 0;
      }
      if (bar_sync_or(2, 128, *((volatile int *)&bar.abort))) break;
      const int t0 = c * kC;
      const int nvalid = min(kC, L - t0);
      // 1. slot free -> TMA k, v
      int pbad = 0;
      if (pt == 0) {
        if (!mbar_wait(&bar.slot_free[s], ph ^ 1u, lim)) {
          pbad = 1;
        } else {
          mbar_expect_tx(&bar.kv_full[s], 32768);
          tma_load_4d(sm + OFF_KHAT + s * 8192, &tmap_k, &bar.kv_full[s], 0, t0, f, bh);
          tma_load_4d(sm + OFF_KHAT + KHAT_KB_STRIDE + s * 8192, &tmap_k, &bar.kv_full[s], 64, t0, f, bh);
          tma_load_4d(sm + OFF_V + s * 16384, &tmap_v, &bar.kv_full[s], 0, t0, f, bh);
          tma_load_4d(sm + OFF_V + s * 16384 + 8192, &tmap_v, &bar.kv_full[s], 64, t0, f, bh);
        }
      }
      // gates of the chunk (padding tokens get beta = 0)
      if (pt < 64) {
        float b = 0.f;
        if (pt < nvalid) {
          const float x = p.beta[(long)bh * N + (long)f * L + t0 + pt];
          b = p.gates_are_logits ? gate_beta(x) : x;
        }
        bar.beta[s][pt] = b;
      }
      if (bar_sync_or(2, 128, pbad)) {
        if (pt == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
        bar.abort = 1;
        break;
      }
      if (bar_sync_or(2, 128, !mbar_wait(&bar.kv_full[s], ph, lim))) {
        if (pt == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
        bar.abort = 1;
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
      named_bar(2, 128);
      // 3. khat ready; Gram matrix G = Khat Khat^T (rows: this chunk and the next slot)
      if (pt == 0) {
        // (for a frame's first chunk the chain group reads the ticket after this arrival)
        mbar_arrive_only(&bar.khat_ready[s]);
        tc_fence_after();
        const uint32_t idg = idesc_f16(128, 64, 0, 0, 0);
        for (int kk = 0; kk < nkd; ++kk) {
          const uint32_t a = smem_u32(sm + OFF_KHAT + (kk >> 2) * KHAT_KB_STRIDE + s * 8192 + (kk & 3) * 32);
          mma_f16_ss(tmem + TM_G, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), idg, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.g_bar);
      }
      const int gbad = !mbar_wait(&bar.g_bar, g_phase, lim);
      g_phase ^= 1u;
      if (bar_sync_or(2, 128, gbad)) {
        if (pt == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
        bar.abort = 1;
        break;
      }
      tc_fence_after();
      // 4. Nt[u][t] = N[t][u] = beta_t G[t][u] for t > u (G is symmetric, so lane u
      //    reads row u of G); TMEM lanes 0..63 live in warps 8 and 9.
      float *Nt = reinterpret_cast<float *>(sm + OFF_N);
      if (warp < 10) {
        const int u = pt;  // lane
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          float r[16];
          tmem_ld16(tmem + TM_G + lane_off + cb * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            const int t = cb * 16 + e;
            const float4 b4 = *reinterpret_cast<const float4 *>(&bar.beta[s][t]);
            float4 o4;
            o4.x = (t + 0 > u) ? b4.x * r[e + 0] : 0.f;
            o4.y = (t + 1 > u) ? b4.y * r[e + 1] : 0.f;
            o4.z = (t + 2 > u) ? b4.z * r[e + 2] : 0.f;
            o4.w = (t + 3 > u) ? b4.w * r[e + 3] : 0.f;
            *reinterpret_cast<float4 *>(Nt + u * N_STRIDE + t) = o4;
          }
        }
      }
      tc_fence_before();
      named_bar(2, 128);
      // 5. T = (I + N)^-1 diag(beta): thread `col` < 64 solves column col of
      //    X = (I + N)^-1 by forward substitution in axpy form: once x_u is
      //    final, acc[t] += N[t][u] x_u for every later t (independent FMAs),
      //    and x_t = -acc[t].  The critical path is one FMA per step.
      if (pt < 64) {
        const int col = pt;
        float acc[64];
#pragma unroll
        for (int t = 0; t < 64; ++t) acc[t] = 0.f;
#pragma unroll
        for (int u = 0; u < 64; ++u) {
          const float xu = (u == col) ? 1.f : (u < col ? 0.f : -acc[u]);
          acc[u] = xu;
#pragma unroll
          for (int t4 = ((u + 1) >> 2) << 2; t4 < 64; t4 += 4) {
            const float4 n4 = *reinterpret_cast<const float4 *>(Nt + u * N_STRIDE + t4);
            if (t4 + 0 > u) acc[t4 + 0] = fmaf(n4.x, xu, acc[t4 + 0]);
            if (t4 + 1 > u) acc[t4 + 1] = fmaf(n4.y, xu, acc[t4 + 1]);
            if (t4 + 2 > u) acc[t4 + 2] = fmaf(n4.z, xu, acc[t4 + 2]);
            if (t4 + 3 > u) acc[t4 + 3] = fmaf(n4.w, xu, acc[t4 + 3]);
          }
        }
        const float bc = bar.beta[s][col];
        uint8_t *Tt = sm + OFF_T + s * 8192;
#pragma unroll
        for (int t = 0; t < 64; ++t)
          *reinterpret_cast<__half *>(Tt + sw128_offset(t, col)) = __float2half_rn(acc[t] * bc);
      }
      fence_async_smem();
      named_bar(2, 128);
      if (pt == 0) mbar_arrive_only(&bar.t_ready[s]);
      ++c;
    }
  } else {
    // ============================================================ chain group
    const int tile = warp >> 2;                       // 0: A rows, 1: B rows
    const int row = tid & 127;                        // TMEM lane / operand row
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t mma_phase = 0;
    uint32_t qcount[2] = {0, 0};
    int frames = 0;
    bool failed = false;
    uint32_t g = 0;
    const uint32_t id_vi = idesc_f16(128, 64, 1, 1, 0);          // V^T (MN) x I (K), bf16
    const uint32_t id_r = idesc_f16(128, 64, 0, 0, 0, 1, 0);     // -(Y^T) x Khat^T, fp16
    const uint32_t id_u = idesc_f16(128, 64, 0, 0, 0);           // R^T x T^T
    const uint32_t id_y = idesc_f16(128, dk, 0, 0, 1);           // U^T x Khat (MN)
    const uint32_t id_s = idesc_f16(128, dk, 0, 0, 1);           // (alpha S^T) x A^T (MN)
    const uint32_t id_o = idesc_f16(128, dv, 0, 0, 0);           // Q x S

    // wait for the MMAs committed to mma_bar; false (for every chain thread) on a
    // timeout, on `extra` from any thread, or if the prep group gave up
    auto wait_mma = [&](int extra) -> bool {
      const bool ok = mbar_wait(&bar.mma_bar, mma_phase, lim);
      mma_phase ^= 1u;
      return !bar_sync_or(1, kChain, !ok || extra || *((volatile int *)&bar.abort));
    };

    for (;;) {
      // ---- frame start: the prep group has taken the ticket
      {
        const int s = g & 1;
        const uint32_t ph = (g >> 1) & 1u;
        if (bar_sync_or(1, kChain, !mbar_wait(&bar.khat_ready[s], ph, lim))) {
          failed = true;
          break;
        }
      }
      const int tk = bar.ticket_ring[frames & 3];
      ++frames;
      if (tk < 0) break;
      const long ticket = tk;
      const int f = (int)(ticket / BH);
      const int bh = (int)(ticket % BH);

      // Y = [I | 0] in TMEM (fp32) and in the fp16 mirror
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
      named_bar(1, kChain);

      for (int c = 0; c < nch; ++c, ++g) {
        const int s = g & 1;
        const uint32_t ph = (g >> 1) & 1u;
        int cbad = 0;
        // MMA 1: R^T = [0 ; V^T] - Y^T Khat^T
        if (tid == 0) {
          if (c > 0 && !mbar_wait(&bar.khat_ready[s], ph, lim)) cbad = 1;
          tc_fence_after();
          const uint32_t kh = smem_u32(sm + OFF_KHAT + s * 8192);
          const uint32_t vb = smem_u32(sm + OFF_V + s * 16384);
          const uint32_t ib = smem_u32(sm + OFF_I);
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(tmem + TM_RU + 64, sdesc_sw128(vb + kk * 2048, 8192, 1024), sdesc_sw128(ib + kk * 32, 16, 1024),
                       id_vi, kk > 0 ? 1u : 0u);
          for (int t2 = 0; t2 < 2; ++t2) {
            const uint32_t mb = smem_u32(sm + OFF_MIRROR + t2 * 32768);
            for (int kk = 0; kk < nkd; ++kk) {
              const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
              const uint32_t kho = (kk >> 2) * KHAT_KB_STRIDE + (kk & 3) * 32;
              mma_f16_ss(tmem + TM_RU + t2 * 64, sdesc_sw128(mb + ko, 16, 1024), sdesc_sw128(kh + kho, 16, 1024), id_r,
                         (t2 == 1 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&bar.mma_bar);
        }
        if (!wait_mma(cbad)) { failed = true; break; }
        tc_fence_after();
        // conv 1: R^T rows -> fp16
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          float r[16];
          tmem_ld16(tmem + TM_RU + tile * 64 + lane_off + cb * 16, r);
          tmem_ld_wait();
          store_row16_f16(sm + OFF_RU + tile * 16384, row, cb * 16, r);
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(1, kChain);
        // MMA 2: U^T = R^T T^T
        if (tid == 0) {
          if (!mbar_wait(&bar.t_ready[s], ph, lim)) cbad = 1;
          tc_fence_after();
          const uint32_t tb = smem_u32(sm + OFF_T + s * 8192);
          for (int t2 = 0; t2 < 2; ++t2) {
            const uint32_t rb = smem_u32(sm + OFF_RU + t2 * 16384);
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(tmem + TM_RU + t2 * 64, sdesc_sw128(rb + kk * 32, 16, 1024), sdesc_sw128(tb + kk * 32, 16, 1024),
                         id_u, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bar.mma_bar);
        }
        if (!wait_mma(cbad)) { failed = true; break; }
        tc_fence_after();
        // conv 2: U^T rows -> fp16
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          float r[16];
          tmem_ld16(tmem + TM_RU + tile * 64 + lane_off + cb * 16, r);
          tmem_ld_wait();
          store_row16_f16(sm + OFF_RU + tile * 16384, row, cb * 16, r);
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(1, kChain);
        // MMA 3: Y^T += U^T Khat ; then release the khat/v slot
        if (tid == 0) {
          tc_fence_after();
          const uint32_t kh = smem_u32(sm + OFF_KHAT + s * 8192);
          for (int t2 = 0; t2 < 2; ++t2) {
            const uint32_t ub = smem_u32(sm + OFF_RU + t2 * 16384);
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(tmem + TM_Y + t2 * 128, sdesc_sw128(ub + kk * 32, 16, 1024),
                         sdesc_sw128(kh + kk * 2048, KHAT_KB_STRIDE, 1024), id_y, 1u);
          }
          mma_commit(&bar.mma_bar);
          mma_commit(&bar.slot_free[s]);
        }
        if (!wait_mma(0)) { failed = true; break; }
        tc_fence_after();
        // conv 3: Y^T rows -> fp16 mirror (tile B not needed after the last chunk)
        if (c + 1 < nch || tile == 0) {
#pragma unroll 1
          for (int cb = 0; cb < nkd; ++cb) {
            float r[16];
            tmem_ld16(tmem + TM_Y + tile * 128 + lane_off + cb * 16, r);
            tmem_ld_wait();
            store_row16_f16(sm + OFF_MIRROR + tile * 32768 + (cb >> 2) * 16384, row, (cb & 3) * 16, r);
          }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(1, kChain);
      }
      if (failed) break;

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
        // rows j of alpha * S_{f-1}^T (threads of both tiles split the d_k columns)
        const int j = row;
        const int half = tile;  // 0: k-block 0, 1: k-block 1
        const float *prev = p.ws.states + ((long)bh * F + (f - 1)) * (long)dk * dv + (long)j * dk;
#pragma unroll 1
        for (int cb = half * 4; cb < half * 4 + 4; ++cb) {
          if (cb >= nkd) break;
          float r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = 0.f;
          if (j < dv) {
            if (f > 0) {
#pragma unroll
              for (int e = 0; e < 16; e += 4) {
                const float4 x = __ldcg(reinterpret_cast<const float4 *>(prev + cb * 16 + e));
                r[e] = alpha * x.x; r[e + 1] = alpha * x.y; r[e + 2] = alpha * x.z; r[e + 3] = alpha * x.w;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) r[e] = alpha * p.state_in[(long)bh * dk * dv + (long)(cb * 16 + e) * dv + j];
            }
          }
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
          mma_commit(&bar.mma_bar);
        }
        if (!wait_mma(0)) { failed = true; break; }
        tc_fence_after();
      }
      // S_f^T rows: publish fp32, state_out, fp16 B operand for the read-out
      {
        const int j = row;
        const int half = tile;
        float *cur = p.ws.states + ((long)bh * F + f) * (long)dk * dv + (long)j * dk;
#pragma unroll 1
        for (int cb = half * 4; cb < half * 4 + 4; ++cb) {
          if (cb >= nkd) break;
          float r[16];
          tmem_ld16(tmem + TM_Y + 128 + lane_off + cb * 16, r);
          tmem_ld_wait();
          if (j < dv) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4 *>(cur + cb * 16 + e) = make_float4(r[e], r[e + 1], r[e + 2], r[e + 3]);
            if (f == F - 1 && p.state_out) {
#pragma unroll
              for (int e = 0; e < 16; ++e) p.state_out[(long)bh * dk * dv + (long)(cb * 16 + e) * dv + j] = r[e];
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
        const bool ok = mbar_wait(&bar.q_full[b], qcount[b] & 1u, lim);
        ++qcount[b];
        if (bar_sync_or(1, kChain, !ok)) { failed = true; break; }
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
          const uint32_t a0 = smem_u32(qb), b0 = smem_u32(sm + OFF_S16);
          for (int kk = 0; kk < nkd; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_f16_ss(tmem + TM_RU, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024), id_o,
                       kk > 0 ? 1u : 0u);
          }
          mma_commit(&bar.mma_bar);
        }
        if (!wait_mma(0)) { failed = true; break; }
        tc_fence_after();
        if (tid == 0 && qc + 2 < n3) {
          mbar_expect_tx(&bar.q_full[b], 32768);
          tma_load_4d(qb, &tmap_q, &bar.q_full[b], 0, (qc + 2) * 128, f, bh);
          tma_load_4d(qb + 16384, &tmap_q, &bar.q_full[b], 64, (qc + 2) * 128, f, bh);
        }
        // epilogue: token row = lane; warps 0-3 take column blocks [0, nb0), warps 4-7 the rest
        {
          const int t = qc * 128 + row;
          const int nb = dv / 16, nb0 = (nb + 1) / 2;
          float *orow = p.o + ((long)bh * N + (long)f * L + t) * dv;
          const int cb0 = tile == 0 ? 0 : nb0, cb1 = tile == 0 ? nb0 : nb;
#pragma unroll 1
          for (int cb = cb0; cb < cb1; ++cb) {
            float r[16];
            tmem_ld16(tmem + TM_RU + lane_off + cb * 16, r);
            tmem_ld_wait();
            if (t < L) {
              float4 *dst = reinterpret_cast<float4 *>(orow + cb * 16);
#pragma unroll
              for (int e = 0; e < 4; ++e) dst[e] = make_float4(r[4 * e], r[4 * e + 1], r[4 * e + 2], r[4 * e + 3]);
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
