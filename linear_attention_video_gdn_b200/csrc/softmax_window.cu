// Windowed block-causal softmax attention on tcgen05 tensor cores (bf16 q, k, v).
//
// SANA-WM's hybrid interleaves the frame-wise Gated DeltaNet with softmax
// attention ("SANA-WM, an open-source 2.6B world model for 1-minute 720p
// video", GeekNews, "Core design and generation pipeline": periodic softmax;
// the Vietnamese post: Gated DeltaNet for most of the sequence, softmax windows
// in between; the SANA-Video talk: minute-long video keeps softmax inside a
// sliding window).  The library's reading: token t of frame f attends to every
// token of frames max(0, f-W+1) .. f,
//   o_t = sum_s softmax_s(scale q_t . k_s) v_s.
//
// One CTA per (b, h, frame, 128-query tile); the window's keys stream in
// 64-key tiles through a 4-slot TMA ring whose K and V halves are refilled
// separately (K after its S product, V after its PV product).  Per key tile:
//   S = Q K^T         tcgen05, M=128 queries x N=64 keys, bf16 operands, into
//                     one of two TMEM buffers;
//   P = exp(S - m)    warps 0-7: warps w and w+4 share the query rows of TMEM
//                     lane quarter w and take 32 keys each; P is written to
//                     shared memory as bf16 high and low parts (truncated
//                     upper halves, about 16 significant bits);
//   O += P V          tcgen05, M=128 x N=dv, two MMAs per 16 keys (high and
//                     low parts against the bf16 V tile as loaded), fp32 in
//                     TMEM.
// The running maximum m moves only when a tile's maximum exceeds it by more
// than 2^8 in exp2 units; then O (in TMEM) and the row sums are rescaled.  The
// result is exact for any m, since P and the row sums use the same m.  One
// thread each in warps 8-11 issues the S MMAs, the PV MMAs, the K loads and the
// V loads, so no role waits on another's issue cost, and S of the next tile and
// PV of the tile before run on the tensor pipe while warps 0-7 exponentiate.
#include "f32x2.cuh"
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kSwThreads = 384;  // warps 0-7: softmax; warps 8-11: S MMAs, PV MMAs, K loads, V loads
constexpr int kSoftmax = 256;    // softmax threads
constexpr int kQRows = 128;      // queries per CTA
constexpr int kKeys = 64;        // keys per tile
constexpr int kHalf = kKeys / 2; // keys per softmax thread
constexpr int kRing = 4;         // K/V tiles in flight
constexpr uint32_t kTileBytes = 32768;  // K (2 x 8 KB) + V (2 x 8 KB)
constexpr float kRescale = 8.0f;        // exp2 units the running maximum may lag behind

struct __align__(1024) SwSmem {
  uint8_t q[2][16384];             // Q tile: two 64-column atoms of 128 rows (K-major A operand)
  uint8_t kv[kRing][kTileBytes];   // K tile (64 keys x 2 atoms), then V tile (64 keys x 2 atoms)
  uint8_t p[2][2][16384];          // P buffer b, high / low part: bf16, 128 rows x 64 keys (K-major)
  float part[2][kQRows];           // the two halves' tile maxima of each row (row sums at the end)
  uint64_t q_full;
  uint64_t k_full[kRing];    // the K half of slot s has landed
  uint64_t v_full[kRing];    // the V half of slot s has landed
  uint64_t k_empty[kRing];   // the S MMAs reading the K half have completed
  uint64_t v_empty[kRing];   // the PV MMAs reading the V half have completed
  uint64_t s_full[2];        // S buffer b holds tile j's scores
  uint64_t s_free[2];        // the softmax warps have read S buffer b
  uint64_t p_full[2];        // P buffer b holds tile j's probabilities
  uint64_t o_done[2];        // the PV MMAs of tile j (buffer j & 1) have completed
  uint64_t fin;              // every MMA of the CTA has completed (teardown)
  uint32_t tmem_base;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two values as bf16 high parts (the upper 16 bits) and bf16 low parts (the upper
// 16 bits of what the high part leaves, formed exactly in fp32): about 16
// significant bits in all, with integer and add instructions only, so the
// conversion unit stays free for the exponentials.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  const float ra = a - __uint_as_float(ua & 0xffff0000u), rb = b - __uint_as_float(ub & 0xffff0000u);
  hi = __byte_perm(ua, ub, 0x7632);  // (b's upper half << 16) | a's upper half
  lo = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
}

__device__ __forceinline__ void sw_named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void sw_st_v8(float *p, const float *v, float scale) {
  asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0] * scale), "f"(v[1] * scale),
               "f"(v[2] * scale), "f"(v[3] * scale), "f"(v[4] * scale), "f"(v[5] * scale), "f"(v[6] * scale),
               "f"(v[7] * scale)
               : "memory");
}

// Key tile j of the window: frame f0 + j / tiles_per_frame, tile j % tiles_per_frame.
struct KeyTile {
  int frame, row0, valid;
};
__device__ __forceinline__ KeyTile key_tile(int j, int f0, int tpf, int L) {
  KeyTile t;
  t.frame = f0 + j / tpf;
  t.row0 = (j % tpf) * kKeys;
  t.valid = min(kKeys, L - t.row0);
  return t;
}

struct SwParams {
  float *o;
  int BH, F, L, dk, dv, W;
  float scale_log2;  // scale * log2(e): scores in exp2 units
  int *status;
  unsigned long long spin_limit_ns;
};

__global__ void __launch_bounds__(kSwThreads, 1)
    softmax_window_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v, SwParams p) {
  extern __shared__ uint8_t smem_raw[];
  SwSmem &sm = *reinterpret_cast<SwSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int L = p.L, dk = p.dk, dv = p.dv;
  const int nqt = (L + kQRows - 1) / kQRows;
  const long unit = blockIdx.x;
  const int qt = (int)(unit % nqt);
  const int f = (int)((unit / nqt) % p.F);
  const int bh = (int)(unit / ((long)nqt * p.F));
  const int f0 = max(0, f - p.W + 1);
  const int tpf = (L + kKeys - 1) / kKeys;  // key tiles per frame
  const int nt = (f - f0 + 1) * tpf;        // key tiles of the window
  const unsigned long long lim = p.spin_limit_ns;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_free[b], 2);  // one arrival per key half
      mbar_init(&sm.p_full[b], 2);
      mbar_init(&sm.o_done[b], 1);
    }
    mbar_init(&sm.fin, 2);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tS[2] = {tmem, tmem + 64};        // scores, 64 columns each
  const uint32_t tO[2] = {tmem + 128, tmem + 256};  // output accumulator of each key half, dv columns

  if (warp >= 8) {
    // ---------------- one thread per role: S MMAs, PV MMAs, K loads, V loads ----------------
    const bool lead = (tid & 31) == 0;
    bool ok = true;
    // K and V of tile j go into slot j % kRing with barriers of their own: a K half is
    // free once the tile's S MMAs are done, well before its V half (free after PV)
    if (warp == 8 && lead) {  // S_j = Q K_j^T
      const uint32_t idesc_s = idesc_f16(kQRows, kKeys, 1, 0, 0);  // bf16; Q and K both K-major
      ok = mbar_wait(&sm.q_full, 0, lim);
      // descriptors built once; a k-step only advances their start-address field (address / 16)
      const uint64_t qdesc = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing, b = j & 1;
        ok = mbar_wait(&sm.k_full[s], (uint32_t)(j / kRing) & 1u, lim);
        if (ok && j >= 2) ok = mbar_wait(&sm.s_free[b], (uint32_t)((j - 2) >> 1) & 1u, lim);
        if (!ok) break;
        tc_fence_after();
        const uint64_t kd = sdesc_sw128(smem_u32(sm.kv[s]), 16, 1024);
        for (int kk = 0; kk < dk / 16; ++kk) {
          const uint32_t qo = (uint32_t)(kk / 4) * 16384u + (uint32_t)(kk % 4) * 32u;
          const uint32_t ko = (uint32_t)(kk / 4) * 8192u + (uint32_t)(kk % 4) * 32u;
          mma_f16_ss(tS[b], qdesc + (qo >> 4), kd + (ko >> 4), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[b]);
        mma_commit(&sm.k_empty[s]);
      }
      mma_commit(&sm.fin);  // TMEM is released only after every MMA of both issuers
    } else if (warp == 9 && lead) {  // O_h += P_i,h V_i,h for each key half h, high then low part of P
      const uint32_t idesc_pv = idesc_f16(kQRows, dv, 1, 0, 1);  // bf16; P K-major, V MN-major
      for (int i = 0; i < nt && ok; ++i) {
        const int b = i & 1, s = i % kRing;
        ok = mbar_wait(&sm.p_full[b], (uint32_t)(i >> 1) & 1u, lim) &&
             mbar_wait(&sm.v_full[s], (uint32_t)(i / kRing) & 1u, lim);
        if (!ok) break;
        tc_fence_after();
        const uint64_t vd = sdesc_sw128(smem_u32(sm.kv[s] + 16384), 8192, 1024);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint64_t pd = sdesc_sw128(smem_u32(sm.p[b][part]), 16, 1024);
#pragma unroll
            for (int kk = 2 * h; kk < 2 * h + 2; ++kk)  // keys 16 kk .. 16 kk + 15 of the tile
              mma_f16_ss(tO[h], pd + (uint64_t)(kk * 32 / 16), vd + (uint64_t)(kk * 2048 / 16), idesc_pv,
                         (i > 0 || part > 0 || kk > 2 * h) ? 1u : 0u);
          }
        mma_commit(&sm.o_done[b]);
        mma_commit(&sm.v_empty[s]);
      }
      mma_commit(&sm.fin);
      if (!mbar_wait(&sm.fin, 0, lim)) ok = false;
    } else if (warp == 10 && lead) {  // Q, then K tiles as their slots free up
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      mbar_expect_tx(&sm.q_full, 32768);
      tma_load_4d(sm.q[0], &tmap_q, &sm.q_full, 0, qt * kQRows, f, bh);
      tma_load_4d(sm.q[1], &tmap_q, &sm.q_full, 64, qt * kQRows, f, bh);
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing;
        if (j >= kRing) ok = mbar_wait(&sm.k_empty[s], (uint32_t)((j - kRing) / kRing) & 1u, lim);
        if (!ok) break;
        const KeyTile t = key_tile(j, f0, tpf, L);
        mbar_expect_tx(&sm.k_full[s], kTileBytes / 2);
        tma_load_4d(sm.kv[s] + 0, &tmap_k, &sm.k_full[s], 0, t.row0, t.frame, bh);
        tma_load_4d(sm.kv[s] + 8192, &tmap_k, &sm.k_full[s], 64, t.row0, t.frame, bh);
      }
      // the last loads land before the CTA can exit
      for (int j = max(0, nt - kRing); j < nt && ok; ++j)
        ok = mbar_wait(&sm.k_full[j % kRing], (uint32_t)(j / kRing) & 1u, lim);
    } else if (warp == 11 && lead) {  // V tiles as their slots free up
      tma_prefetch_desc(&tmap_v);
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing;
        if (j >= kRing) ok = mbar_wait(&sm.v_empty[s], (uint32_t)((j - kRing) / kRing) & 1u, lim);
        if (!ok) break;
        const KeyTile t = key_tile(j, f0, tpf, L);
        mbar_expect_tx(&sm.v_full[s], kTileBytes / 2);
        tma_load_4d(sm.kv[s] + 16384, &tmap_v, &sm.v_full[s], 0, t.row0, t.frame, bh);
        tma_load_4d(sm.kv[s] + 24576, &tmap_v, &sm.v_full[s], 64, t.row0, t.frame, bh);
      }
      for (int j = max(0, nt - kRing); j < nt && ok; ++j)
        ok = mbar_wait(&sm.v_full[j % kRing], (uint32_t)(j / kRing) & 1u, lim);
    }
    if (lead && !ok) latch_status(p.status, GDN_ERR_TIMEOUT);
  } else {
    // ---------------- softmax: warps 4h .. 4h+3 take keys 32h .. 32h+31 of every tile ----------------
    // Each half keeps its own running maximum, row sum and accumulator O_h, so the
    // halves never wait for each other inside the key loop; they combine once at the end.
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + (tid & 31);
    const int hb = 1 + half;  // the half's named barrier
    const bool hlead = (tid & 127) == 0;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int qrow = qt * kQRows + row;
    float m = -INFINITY, l = 0.0f;  // this half's running maximum (exp2 units) and row sum
    bool failed = false;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      const KeyTile t = key_tile(j, f0, tpf, L);
      int bad = !mbar_wait(&sm.s_full[b], (uint32_t)(j >> 1) & 1u, lim);
      if (bar_sync_or(hb, 128, bad)) { failed = true; break; }
      tc_fence_after();
      float x[kHalf];
      tmem_ld16(tS[b] + lane_off + half * kHalf, *reinterpret_cast<float(*)[16]>(x));
      tmem_ld16(tS[b] + lane_off + half * kHalf + 16, *reinterpret_cast<float(*)[16]>(x + 16));
      tmem_ld_wait();
      // the maximum of the raw scores over this half's keys inside the frame
      const int nvalid = t.valid - half * kHalf;
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kHalf; ++c)
        if (c < nvalid) mx[c & 3] = fmaxf(mx[c & 3], x[c]);
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      // P buffer b was last read by PV_{j-2}
      bad = j >= 2 && !mbar_wait(&sm.o_done[b], (uint32_t)((j - 2) >> 1) & 1u, lim);
      // move the running maximum only when this tile exceeds it by more than 2^kRescale;
      // the warp rescales its rows of O_h together (TMEM access is warp-wide)
      const bool up = mt > m + kRescale;
      if (__any_sync(0xffffffffu, up) && !__any_sync(0xffffffffu, bad)) {
        const float m_new = up ? mt : m;
        if (j >= 1) {
          bad = !mbar_wait(&sm.o_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, lim);
          tc_fence_after();
          const float a = up ? ex2(m - m_new) : 1.0f;  // 0 while m is still -inf (O_h and l are 0)
          l *= a;
          for (int cb = 0; cb < dv / 16; ++cb) {
            float r[16];
            tmem_ld16(tO[half] + lane_off + cb * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] *= a;
            tmem_st16(tO[half] + lane_off + cb * 16, r);
          }
          tmem_st_wait();
        }
        m = m_new;
      }
      // p = exp2(s * scale_log2 - m): the argument of two keys in one packed FMA
      const uint64_t c2 = pack2(__float_as_uint(p.scale_log2), __float_as_uint(p.scale_log2));
      const uint64_t nm2 = pack2(__float_as_uint(-m), __float_as_uint(-m));
      float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      uint32_t hi[kHalf / 2], lo[kHalf / 2];
#pragma unroll
      for (int c = 0; c < kHalf; c += 2) {
        const uint64_t arg = fma2(pack2(__float_as_uint(x[c]), __float_as_uint(x[c + 1])), c2, nm2);
        const float p0 = c < nvalid ? ex2(__uint_as_float((uint32_t)arg)) : 0.0f;
        const float p1 = c + 1 < nvalid ? ex2(__uint_as_float((uint32_t)(arg >> 32))) : 0.0f;
        rs[(c >> 1) & 3] += p0 + p1;
        split_bf16x2(p0, p1, hi[c / 2], lo[c / 2]);
      }
      l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
#pragma unroll
      for (int c8 = 0; c8 < kHalf / 8; ++c8) {
        const uint32_t off = sw128_offset((uint32_t)row, (uint32_t)((half * (kHalf / 8) + c8) * 8));
        *reinterpret_cast<uint4 *>(sm.p[b][0] + off) = make_uint4(hi[4 * c8], hi[4 * c8 + 1], hi[4 * c8 + 2], hi[4 * c8 + 3]);
        *reinterpret_cast<uint4 *>(sm.p[b][1] + off) = make_uint4(lo[4 * c8], lo[4 * c8 + 1], lo[4 * c8 + 2], lo[4 * c8 + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      if (bar_sync_or(hb, 128, bad)) { failed = true; break; }
      if (hlead) {
        mbar_arrive_only(&sm.s_free[b]);  // this half of S buffer b was read at the top of the tile
        mbar_arrive_only(&sm.p_full[b]);
      }
    }
    if (!failed && nt >= 1) {
      const int last = nt - 1;
      const int bad = !mbar_wait(&sm.o_done[last & 1], (uint32_t)(last >> 1) & 1u, lim);
      if (bar_sync_or(hb, 128, bad)) failed = true;
    }
    // combine the halves once: M = max(m_0, m_1), o = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / (l_0 2^(m_0-M) + l_1 2^(m_1-M));
    // every softmax thread takes part in the barriers below, failed or not, so both halves pass them
    const int fail_any = bar_sync_or(3, kSoftmax, failed ? 1 : 0);
    sm.part[half][row] = m;
    sw_named_bar(3, kSoftmax);
    const float M = fmaxf(sm.part[0][row], sm.part[1][row]);
    const float sc0 = ex2(sm.part[0][row] - M), sc1 = ex2(sm.part[1][row] - M);  // 0 for a half with no key
    sw_named_bar(3, kSoftmax);
    sm.part[half][row] = l * (half ? sc1 : sc0);
    sw_named_bar(3, kSoftmax);
    if (!fail_any) {
      tc_fence_after();
      const float inv = 1.0f / (sm.part[0][row] + sm.part[1][row]);
      const float w0 = sc0 * inv, w1 = sc1 * inv;
      float *orow = p.o + ((long)bh * p.F * L + (long)f * L + qrow) * dv;
      const bool aligned32 = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
#pragma unroll 1
      for (int cb = half; cb < dv / 16; cb += 2) {
        float r0[16], r1[16];
        tmem_ld16(tO[0] + lane_off + cb * 16, r0);
        tmem_ld16(tO[1] + lane_off + cb * 16, r1);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) r0[e] = r0[e] * w0 + r1[e] * w1;
        if (qrow < L) {
          if (aligned32) {
            sw_st_v8(orow + cb * 16, r0, 1.0f);
            sw_st_v8(orow + cb * 16 + 8, r0 + 8, 1.0f);
          } else {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4 *>(orow + cb * 16 + e) = make_float4(r0[e], r0[e + 1], r0[e + 2], r0[e + 3]);
          }
        }
      }
    } else if (tid == 0) {
      latch_status(p.status, GDN_ERR_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace
}  // namespace tc

bool softmax_window_supported(int dk, int dv) {
  return dk % 16 == 0 && dv % 16 == 0 && dk >= 16 && dk <= 128 && dv >= 16 && dv <= 128;
}

cudaError_t launch_softmax_window(const void *q, const void *k, const void *v, float *o, int B, int H, int F, int L,
                                  int dk, int dv, int W, float scale, int *status, unsigned long long spin_limit_ns,
                                  cudaStream_t st) {
  using namespace tc;
  CUtensorMap mq, mk, mv;
  const int BH = B * H;
  if (!make_bf16_map(&mq, q, dk, L, F, BH, kQRows) || !make_bf16_map(&mk, k, dk, L, F, BH, kKeys) ||
      !make_bf16_map(&mv, v, dv, L, F, BH, kKeys))
    return cudaErrorInvalidValue;
  SwParams p;
  p.o = o;
  p.BH = BH; p.F = F; p.L = L; p.dk = dk; p.dv = dv; p.W = W;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);  // log2(e)
  p.status = status;
  p.spin_limit_ns = spin_limit_ns;
  const size_t smem = sizeof(SwSmem) + 1024;
  static_assert(sizeof(SwSmem) + 1024 <= 232448, "shared memory of one CTA");
  cudaError_t e = cudaFuncSetAttribute(softmax_window_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long grid = (long)BH * F * ((L + kQRows - 1) / kQRows);
  if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
  softmax_window_kernel<<<(unsigned)grid, kSwThreads, smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn
