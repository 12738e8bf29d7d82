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
// One CTA per (b, h, frame, pair of 128-query tiles X = 0, 1); the window's keys
// stream in 64-key tiles through a 3-slot TMA ring whose K and V halves are
// refilled separately (K after its S products, V after its PV products), and
// each key tile serves both query tiles.  Per key tile and query tile X:
//   S_X = Q_X K^T     tcgen05, M=128 queries x N=64 keys, bf16 operands, into
//                     one of two TMEM buffers of tile X;
//   P_X = exp(S - m)  warps 4X .. 4X+3, one query row per thread, written to
//                     shared memory as fp16 (11-bit significands); warps
//                     12-13 convert the V tile to fp16 in place (exact for
//                     bf16 values inside the fp16 range);
//   O_X += P_X V      tcgen05, M=128 x N=dv, fp16 operands, fp32 in TMEM.
// While one query tile's warps exponentiate, the tensor pipe runs the other
// tile's products.  The running maximum m moves only when a tile's maximum
// exceeds it by more than 2^8 in exp2 units; then the row of O (in TMEM) and
// the row sum are rescaled.  The result is exact for any m, since P and the
// row sum use the same m.  One thread each in warps 8-11 issues the S MMAs,
// the PV MMAs, the K loads and the V loads.
#include "f32x2.cuh"
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kSwThreads = 448;  // warps 0-3: query tile 0; 4-7: query tile 1; 8-11: S, PV, K, V; 12-13: V to fp16
constexpr int kQRows = 128;      // queries per query tile
constexpr int kKeys = 64;        // keys per key tile
constexpr int kRing = 4;         // K/V tiles in flight
constexpr uint32_t kHalfBytes = 16384;  // the K (or V) half of a ring slot: 64 keys x 2 atoms
constexpr float kRescale = 8.0f;        // exp2 units the running maximum may lag behind

struct __align__(1024) SwSmem {
  uint8_t q[2][2][16384];          // query tile X: two 64-column atoms of 128 rows (K-major A operand)
  uint8_t kv[kRing][2][16384];     // slot: K half, V half (64 keys x 2 atoms each)
  uint8_t p[2][16384];             // query tile X: fp16 probabilities, 128 rows x 64 keys (K-major)
  uint64_t q_full;
  uint64_t k_full[kRing], v_full[kRing];
  uint64_t k_empty[kRing];   // both query tiles' S MMAs reading the K half have completed
  uint64_t v_empty[kRing];   // both query tiles' PV MMAs reading the V half have completed
  uint64_t v_conv[kRing];    // the V half has been converted to fp16 (one arrival per converting warp)
  uint64_t s_full[2][2];     // [X][b]: S buffer b of tile X holds its scores
  uint64_t s_free[2][2];     // [X][b]: tile X's four softmax warps have read it
  uint64_t p_full[2];        // [X]: P_X holds the current key tile's probabilities (one arrival per warp)
  uint64_t o_done[2];        // [X]: the PV MMAs of tile X's latest key tile have completed
  uint64_t fin;              // every MMA of the CTA has completed (teardown)
  uint32_t tmem_base;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
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

// Maximum of the raw scores over the first nvalid keys (kFull: all 64), four
// partial maxima to shorten the dependent chain.
template <bool kFull>
__device__ __forceinline__ float tile_max(const float (&sc)[kKeys], int nvalid) {
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < kKeys; ++c)
    if (kFull || c < nvalid) mx[c & 3] = fmaxf(mx[c & 3], sc[c]);
  return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// p = exp2(s * c - m) over the row's 64 keys (zero past nvalid), written to the
// K-major P tile as fp16 8 keys at a time; returns the sum.
template <bool kFull>
__device__ __forceinline__ float tile_exp(const float (&sc)[kKeys], int nvalid, float c, float m, int row,
                                          uint8_t *p_tile) {
  const uint64_t c2 = pack2(__float_as_uint(c), __float_as_uint(c));
  const uint64_t nm2 = pack2(__float_as_uint(-m), __float_as_uint(-m));
  float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int c8 = 0; c8 < kKeys / 8; ++c8) {
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k0 = c8 * 8 + 2 * e;
      const uint64_t arg = fma2(pack2(__float_as_uint(sc[k0]), __float_as_uint(sc[k0 + 1])), c2, nm2);
      float p0 = ex2(__uint_as_float((uint32_t)arg)), p1 = ex2(__uint_as_float((uint32_t)(arg >> 32)));
      if (!kFull) {
        p0 = k0 < nvalid ? p0 : 0.0f;
        p1 = k0 + 1 < nvalid ? p1 : 0.0f;
      }
      rs[e] += p0 + p1;
      h[e] = pack_f16x2(p0, p1);
    }
    const uint32_t off = sw128_offset((uint32_t)row, (uint32_t)(c8 * 8));
    *reinterpret_cast<uint4 *>(p_tile + off) = make_uint4(h[0], h[1], h[2], h[3]);
  }
  return (rs[0] + rs[1]) + (rs[2] + rs[3]);
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
  const int warp = tid >> 5, lane = tid & 31;
  const int L = p.L, dk = p.dk, dv = p.dv;
  const int npair = (L + 2 * kQRows - 1) / (2 * kQRows);  // pairs of query tiles per frame
  const long unit = blockIdx.x;
  const int qp = (int)(unit % npair);
  const int f = (int)((unit / npair) % p.F);
  const int bh = (int)(unit / ((long)npair * p.F));
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
      mbar_init(&sm.v_conv[s], 2);
    }
    for (int x = 0; x < 2; ++x) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.s_full[x][b], 1);
        mbar_init(&sm.s_free[x][b], 4);  // one arrival per softmax warp of the tile
      }
      mbar_init(&sm.p_full[x], 4);
      mbar_init(&sm.o_done[x], 1);
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
  // TMEM: [0, 256) scores, two 64-column buffers per query tile; [256, 512) O of each query tile
  auto tS = [&](int x, int b) { return tmem + (uint32_t)(x * 128 + b * 64); };
  auto tO = [&](int x) { return tmem + 256u + (uint32_t)(x * 128); };

  if (warp >= 8 && warp < 12) {
    // ---------------- one thread per role: S MMAs, PV MMAs, Q and K loads, V loads ----------------
    const bool lead = lane == 0;
    bool ok = true;
    if (warp == 8 && lead) {  // S_X = Q_X K_j^T for both query tiles
      const uint32_t idesc_s = idesc_f16(kQRows, kKeys, 1, 0, 0);  // bf16; Q and K both K-major
      ok = mbar_wait(&sm.q_full, 0, lim);
      // descriptors built once; a k-step only advances their start-address field (address / 16)
      const uint64_t qdesc[2] = {sdesc_sw128(smem_u32(sm.q[0][0]), 16, 1024),
                                 sdesc_sw128(smem_u32(sm.q[1][0]), 16, 1024)};
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing, b = j & 1;
        ok = mbar_wait(&sm.k_full[s], (uint32_t)(j / kRing) & 1u, lim);
        const uint64_t kd = sdesc_sw128(smem_u32(sm.kv[s][0]), 16, 1024);
        for (int x = 0; x < 2 && ok; ++x) {
          if (j >= 2) ok = mbar_wait(&sm.s_free[x][b], (uint32_t)((j - 2) >> 1) & 1u, lim);
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < dk / 16; ++kk) {
            const uint32_t qo = (uint32_t)(kk / 4) * 16384u + (uint32_t)(kk % 4) * 32u;
            const uint32_t ko = (uint32_t)(kk / 4) * 8192u + (uint32_t)(kk % 4) * 32u;
            mma_f16_ss(tS(x, b), qdesc[x] + (qo >> 4), kd + (ko >> 4), idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&sm.s_full[x][b]);
        }
        if (ok) mma_commit(&sm.k_empty[s]);
      }
      mma_commit(&sm.fin);  // TMEM is released only after every MMA of both issuers
    } else if (warp == 9 && lead) {  // O_X += P_X V_j
      const uint32_t idesc_pv = idesc_f16(kQRows, dv, 0, 0, 1);  // fp16; P K-major, V MN-major
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing;
        ok = mbar_wait(&sm.v_conv[s], (uint32_t)(j / kRing) & 1u, lim);
        const uint64_t vd = sdesc_sw128(smem_u32(sm.kv[s][1]), 8192, 1024);
        for (int x = 0; x < 2 && ok; ++x) {
          ok = mbar_wait(&sm.p_full[x], (uint32_t)j & 1u, lim);
          if (!ok) break;
          tc_fence_after();
          const uint64_t pd = sdesc_sw128(smem_u32(sm.p[x]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            mma_f16_ss(tO(x), pd + (uint64_t)(kk * 32 / 16), vd + (uint64_t)(kk * 2048 / 16), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sm.o_done[x]);
        }
        if (ok) mma_commit(&sm.v_empty[s]);
      }
      mma_commit(&sm.fin);
      if (!mbar_wait(&sm.fin, 0, lim)) ok = false;
    } else if (warp == 10 && lead) {  // both Q tiles, then K halves as their slots free up
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      mbar_expect_tx(&sm.q_full, 65536);
      for (int x = 0; x < 2; ++x) {
        const int r0 = (2 * qp + x) * kQRows;
        tma_load_4d(sm.q[x][0], &tmap_q, &sm.q_full, 0, r0, f, bh);
        tma_load_4d(sm.q[x][1], &tmap_q, &sm.q_full, 64, r0, f, bh);
      }
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing;
        if (j >= kRing) ok = mbar_wait(&sm.k_empty[s], (uint32_t)((j - kRing) / kRing) & 1u, lim);
        if (!ok) break;
        const KeyTile t = key_tile(j, f0, tpf, L);
        mbar_expect_tx(&sm.k_full[s], kHalfBytes);
        tma_load_4d(sm.kv[s][0], &tmap_k, &sm.k_full[s], 0, t.row0, t.frame, bh);
        tma_load_4d(sm.kv[s][0] + 8192, &tmap_k, &sm.k_full[s], 64, t.row0, t.frame, bh);
      }
      // the last loads land before the CTA can exit
      for (int j = max(0, nt - kRing); j < nt && ok; ++j)
        ok = mbar_wait(&sm.k_full[j % kRing], (uint32_t)(j / kRing) & 1u, lim);
    } else if (warp == 11 && lead) {  // V halves as their slots free up
      tma_prefetch_desc(&tmap_v);
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing;
        if (j >= kRing) ok = mbar_wait(&sm.v_empty[s], (uint32_t)((j - kRing) / kRing) & 1u, lim);
        if (!ok) break;
        const KeyTile t = key_tile(j, f0, tpf, L);
        mbar_expect_tx(&sm.v_full[s], kHalfBytes);
        tma_load_4d(sm.kv[s][1], &tmap_v, &sm.v_full[s], 0, t.row0, t.frame, bh);
        tma_load_4d(sm.kv[s][1] + 8192, &tmap_v, &sm.v_full[s], 64, t.row0, t.frame, bh);
      }
      for (int j = max(0, nt - kRing); j < nt && ok; ++j)
        ok = mbar_wait(&sm.v_full[j % kRing], (uint32_t)(j / kRing) & 1u, lim);
    }
    if (lead && !ok) latch_status(p.status, GDN_ERR_TIMEOUT);
  } else if (warp >= 12) {
    // ---------------- V halves to fp16 in place, each warp half of the 16 KB ----------------
    const int part = warp - 12;
    bool range_bad = false, failed = false;
    for (int j = 0; j < nt; ++j) {
      const int s = j % kRing;
      if (__any_sync(0xffffffffu, !mbar_wait(&sm.v_full[s], (uint32_t)(j / kRing) & 1u, lim))) {
        failed = true;
        break;
      }
      uint4 *vt = reinterpret_cast<uint4 *>(sm.kv[s][1]) + part * 512;
#pragma unroll 4
      for (int e = 0; e < 16; ++e) {
        const uint4 w = vt[lane + 32 * e];
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t out[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(in[i] << 16), hi = __uint_as_float(in[i] & 0xffff0000u);
          range_bad |= !(fmaxf(fabsf(lo), fabsf(hi)) < 65504.0f);
          out[i] = pack_f16x2(lo, hi);
        }
        vt[lane + 32 * e] = make_uint4(out[0], out[1], out[2], out[3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_only(&sm.v_conv[s]);
    }
    if (__any_sync(0xffffffffu, range_bad) && lane == 0) latch_status(p.status, GDN_ERR_RANGE);
    if (failed && lane == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
  } else {
    // ---------------- softmax: query tile x = warp / 4, one query row per thread ----------------
    const int x = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int qrow = (2 * qp + x) * kQRows + row;
    float m = -INFINITY, l = 0.0f;  // running maximum (exp2 units) and row sum
    bool failed = false;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      const KeyTile t = key_tile(j, f0, tpf, L);
      // each warp runs its own rows: mbarriers only, no barrier with the tile's other warps
      int bad = !mbar_wait(&sm.s_full[x][b], (uint32_t)(j >> 1) & 1u, lim);
      if (__any_sync(0xffffffffu, bad)) { failed = true; break; }
      tc_fence_after();
      float sc[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys / 16; ++c)
        tmem_ld16(tS(x, b) + lane_off + c * 16, *reinterpret_cast<float(*)[16]>(sc + c * 16));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_only(&sm.s_free[x][b]);  // this warp's rows of S buffer b are read
      // the maximum of the raw scores over the keys inside the frame (most tiles are full)
      const bool full = t.valid == kKeys;
      const float mt = (full ? tile_max<true>(sc, kKeys) : tile_max<false>(sc, t.valid)) * p.scale_log2;
      // P_x (one buffer) and O_x: the previous key tile's PV MMAs must be done
      bad = j >= 1 && !mbar_wait(&sm.o_done[x], (uint32_t)(j - 1) & 1u, lim);
      // move the running maximum only when this tile exceeds it by more than 2^kRescale;
      // the warp rescales its rows of O_x together (TMEM access is warp-wide)
      const bool up = mt > m + kRescale;
      if (__any_sync(0xffffffffu, up) && !__any_sync(0xffffffffu, bad)) {
        const float m_new = up ? mt : m;
        if (j >= 1) {
          tc_fence_after();
          const float a = up ? ex2(m - m_new) : 1.0f;
          l *= a;
          for (int cb = 0; cb < dv / 16; ++cb) {
            float r[16];
            tmem_ld16(tO(x) + lane_off + cb * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] *= a;
            tmem_st16(tO(x) + lane_off + cb * 16, r);
          }
          tmem_st_wait();
        }
        m = m_new;
      }
      // p = exp2(s * scale_log2 - m), written 8 keys at a time as bf16 high and low parts
      l += full ? tile_exp<true>(sc, kKeys, p.scale_log2, m, row, sm.p[x])
                : tile_exp<false>(sc, t.valid, p.scale_log2, m, row, sm.p[x]);
      fence_async_smem();
      tc_fence_before();
      if (__any_sync(0xffffffffu, bad)) { failed = true; break; }
      if (lane == 0) mbar_arrive_only(&sm.p_full[x]);  // this warp's rows of P_x are written
    }
    if (!failed && nt >= 1) {
      const int bad = !mbar_wait(&sm.o_done[x], (uint32_t)(nt - 1) & 1u, lim);
      if (__any_sync(0xffffffffu, bad)) failed = true;
    }
    if (!failed) {
      tc_fence_after();
      const float inv = 1.0f / l;
      float *orow = p.o + ((long)bh * p.F * L + (long)f * L + qrow) * dv;
      const bool aligned32 = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
#pragma unroll 1
      for (int cb = 0; cb < dv / 16; ++cb) {
        float r[16];
        tmem_ld16(tO(x) + lane_off + cb * 16, r);
        tmem_ld_wait();
        if (qrow < L) {
          if (aligned32) {
            sw_st_v8(orow + cb * 16, r, inv);
            sw_st_v8(orow + cb * 16 + 8, r + 8, inv);
          } else {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4 *>(orow + cb * 16 + e) =
                  make_float4(r[e] * inv, r[e + 1] * inv, r[e + 2] * inv, r[e + 3] * inv);
          }
        }
      }
    } else if (lane == 0) {
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
  const long grid = (long)BH * F * ((L + 2 * kQRows - 1) / (2 * kQRows));
  if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
  softmax_window_kernel<<<(unsigned)grid, kSwThreads, smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn
