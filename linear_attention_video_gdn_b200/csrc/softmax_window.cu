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
// 64-key tiles through a 4-slot TMA ring.  Per key tile:
//   S = Q K^T         tcgen05, M=128 queries x N=64 keys, bf16 operands, into
//                     one of two TMEM buffers;
//   P = exp(S - m)    warps 0-3, one query row per thread, written to shared
//                     memory as fp16 (11-bit significand); the V tile is
//                     converted to fp16 in place (exact for bf16 values);
//   O += P V          tcgen05, M=128 x N=dv, fp16 operands, fp32 in TMEM.
// The running maximum m moves only when a tile's maximum exceeds it by more
// than 2^8 in exp2 units; then O (in TMEM) and the row sum are rescaled.  The
// result is exact for any m, since P and the row sum use the same m.  Warp 4
// (one thread) issues the loads and the MMAs, so S of the next tile and PV of
// the tile before run on the tensor pipe while warps 0-3 exponentiate.
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {
namespace {

constexpr int kSwThreads = 160;  // warps 0-3: softmax rows; warp 4: loads and MMAs
constexpr int kQRows = 128;      // queries per CTA
constexpr int kKeys = 64;        // keys per tile
constexpr int kRing = 4;         // K/V tiles in flight
constexpr uint32_t kTileBytes = 32768;  // K (2 x 8 KB) + V (2 x 8 KB)
constexpr float kRescale = 8.0f;        // exp2 units the running maximum may lag behind

struct __align__(1024) SwSmem {
  uint8_t q[2][16384];             // Q tile: two 64-column atoms of 128 rows (K-major A operand)
  uint8_t kv[kRing][kTileBytes];   // K tile (64 keys x 2 atoms), then V tile (64 keys x 2 atoms)
  uint8_t p[2][16384];             // P tiles (fp16, 128 rows x 64 keys, K-major A operand)
  uint64_t q_full;
  uint64_t kv_full[kRing];
  uint64_t kv_empty[kRing];  // the PV MMA reading the tile has completed
  uint64_t s_full[2];        // S buffer b holds tile j's scores
  uint64_t s_free[2];        // the softmax warps have read S buffer b
  uint64_t p_full[2];        // P buffer b and tile j's V (fp16) are ready
  uint64_t o_done[2];        // the PV MMA of tile j (buffer j & 1) has completed
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
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_free[b], 1);
      mbar_init(&sm.p_full[b], 1);
      mbar_init(&sm.o_done[b], 1);
    }
    mbar_init(&sm.fin, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tS[2] = {tmem, tmem + 64};  // scores, 64 columns each
  const uint32_t tO = tmem + 128;            // output accumulator, dv columns

  if (warp == 4) {
    // ---------------- loads and MMAs (one thread) ----------------
    if ((tid & 31) == 0) {
      const uint32_t idesc_s = idesc_f16(kQRows, kKeys, 1, 0, 0);  // bf16; Q and K both K-major
      const uint32_t idesc_pv = idesc_f16(kQRows, dv, 0, 0, 1);    // fp16; P K-major, V MN-major
      bool ok = true;
      auto issue_kv = [&](int j) {
        const int s = j % kRing;
        const KeyTile t = key_tile(j, f0, tpf, L);
        uint64_t *bar = &sm.kv_full[s];
        mbar_expect_tx(bar, kTileBytes);
        tma_load_4d(sm.kv[s] + 0, &tmap_k, bar, 0, t.row0, t.frame, bh);
        tma_load_4d(sm.kv[s] + 8192, &tmap_k, bar, 64, t.row0, t.frame, bh);
        tma_load_4d(sm.kv[s] + 16384, &tmap_v, bar, 0, t.row0, t.frame, bh);
        tma_load_4d(sm.kv[s] + 24576, &tmap_v, bar, 64, t.row0, t.frame, bh);
      };
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      mbar_expect_tx(&sm.q_full, 32768);
      tma_load_4d(sm.q[0], &tmap_q, &sm.q_full, 0, qt * kQRows, f, bh);
      tma_load_4d(sm.q[1], &tmap_q, &sm.q_full, 64, qt * kQRows, f, bh);
      for (int j = 0; j < nt && j < kRing; ++j) issue_kv(j);
      ok = mbar_wait(&sm.q_full, 0, lim);
      auto pv = [&](int i) {  // O += P_i V_i, then refill the slot PV_{i-1} released with tile i + 3
        const int b = i & 1, s = i % kRing;
        ok = ok && mbar_wait(&sm.p_full[b], (uint32_t)(i >> 1) & 1u, lim);
        if (!ok) return;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sm.p[b]), v0 = smem_u32(sm.kv[s] + 16384);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_f16_ss(tO, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(v0 + kk * 2048, 8192, 1024), idesc_pv,
                     (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.o_done[b]);
        mma_commit(&sm.kv_empty[s]);
        if (i >= 1 && i + 3 < nt) {
          ok = mbar_wait(&sm.kv_empty[(i - 1) % kRing], (uint32_t)((i - 1) / kRing) & 1u, lim);
          if (ok) issue_kv(i + 3);
        }
      };
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kRing, b = j & 1;
        ok = mbar_wait(&sm.kv_full[s], (uint32_t)(j / kRing) & 1u, lim);
        if (ok && j >= 2) ok = mbar_wait(&sm.s_free[b], (uint32_t)((j - 2) >> 1) & 1u, lim);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sm.q[0]), k0 = smem_u32(sm.kv[s]);
        for (int kk = 0; kk < dk / 16; ++kk) {
          const uint32_t qa = a0 + (uint32_t)(kk / 4) * 16384u + (uint32_t)(kk % 4) * 32u;
          const uint32_t kb = k0 + (uint32_t)(kk / 4) * 8192u + (uint32_t)(kk % 4) * 32u;
          mma_f16_ss(tS[b], sdesc_sw128(qa, 16, 1024), sdesc_sw128(kb, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[b]);
        if (j >= 1) pv(j - 1);
      }
      if (ok && nt >= 1) pv(nt - 1);
      if (!ok) latch_status(p.status, GDN_ERR_TIMEOUT);
      mma_commit(&sm.fin);  // TMEM is released only after every MMA issued here
      mbar_wait(&sm.fin, 0, lim);
    }
  } else {
    // ---------------- softmax rows (warps 0-3, one query row per thread) ----------------
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int qrow = qt * kQRows + tid;
    float m = -INFINITY, l = 0.0f;
    bool failed = false, range_bad = false;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1, s = j % kRing;
      const KeyTile t = key_tile(j, f0, tpf, L);
      int bad = !mbar_wait(&sm.s_full[b], (uint32_t)(j >> 1) & 1u, lim) ||
                !mbar_wait(&sm.kv_full[s], (uint32_t)(j / kRing) & 1u, lim);
      if (bar_sync_or(1, 128, bad)) { failed = true; break; }
      tc_fence_after();
      float x[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys / 16; ++c)
        tmem_ld16(tS[b] + lane_off + c * 16, *reinterpret_cast<float(*)[16]>(x + c * 16));
      tmem_ld_wait();
      tc_fence_before();
      sw_named_bar(1, 128);
      if (tid == 0) mbar_arrive_only(&sm.s_free[b]);
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        x[c] = c < t.valid ? x[c] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, x[c]);
      }
      // P buffer b was last read by PV_{j-2}
      bad = j >= 2 && !mbar_wait(&sm.o_done[b], (uint32_t)((j - 2) >> 1) & 1u, lim);
      // move the running maximum only when this tile exceeds it by more than 2^kRescale;
      // the warp rescales its O rows together (TMEM access is warp-wide)
      const bool up = mt > m + kRescale;
      if (__any_sync(0xffffffffu, up) && !__any_sync(0xffffffffu, bad)) {
        const float m_new = up ? mt : m;
        if (j >= 1) {
          bad = !mbar_wait(&sm.o_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, lim);
          tc_fence_after();
          const float a = up ? ex2(m - m_new) : 1.0f;
          l *= a;
          for (int cb = 0; cb < dv / 16; ++cb) {
            float r[16];
            tmem_ld16(tO + lane_off + cb * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] *= a;
            tmem_st16(tO + lane_off + cb * 16, r);
          }
          tmem_st_wait();
        }
        m = m_new;
      }
      float rs = 0.0f;
      uint32_t h[kKeys / 2];
#pragma unroll
      for (int c = 0; c < kKeys; c += 2) {
        const float p0 = ex2(x[c] - m), p1 = ex2(x[c + 1] - m);
        rs += p0 + p1;
        h[c / 2] = pack_f16x2(p0, p1);
      }
      l += rs;
#pragma unroll
      for (int c8 = 0; c8 < kKeys / 8; ++c8)
        *reinterpret_cast<uint4 *>(sm.p[b] + sw128_offset((uint32_t)tid, (uint32_t)(c8 * 8))) =
            make_uint4(h[4 * c8], h[4 * c8 + 1], h[4 * c8 + 2], h[4 * c8 + 3]);
      // the tile's V to fp16 in place (exact for bf16 values inside the fp16 range)
      uint4 *vt = reinterpret_cast<uint4 *>(sm.kv[s] + 16384);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        uint4 w = vt[tid + 128 * e];
        uint32_t in[4] = {w.x, w.y, w.z, w.w}, out[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(in[i] << 16), hi = __uint_as_float(in[i] & 0xffff0000u);
          range_bad |= !(fabsf(lo) < 65504.0f) || !(fabsf(hi) < 65504.0f);
          out[i] = pack_f16x2(lo, hi);
        }
        vt[tid + 128 * e] = make_uint4(out[0], out[1], out[2], out[3]);
      }
      fence_async_smem();
      tc_fence_before();
      if (bar_sync_or(1, 128, bad)) { failed = true; break; }
      if (tid == 0) mbar_arrive_only(&sm.p_full[b]);
    }
    if (range_bad) latch_status(p.status, GDN_ERR_RANGE);
    if (!failed && nt >= 1) {
      const int last = nt - 1;
      const int bad = !mbar_wait(&sm.o_done[last & 1], (uint32_t)(last >> 1) & 1u, lim);
      if (bar_sync_or(1, 128, bad)) failed = true;
    }
    if (!failed) {
      tc_fence_after();
      const float inv = 1.0f / l;
      float *orow = p.o + ((long)bh * p.F * L + (long)f * L + qrow) * dv;
      const bool aligned32 = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0 && (dv % 8) == 0;
#pragma unroll 1
      for (int cb = 0; cb < dv / 16; ++cb) {
        float r[16];
        tmem_ld16(tO + lane_off + cb * 16, r);
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
    } else if (tid == 0) {
      latch_status(p.status, GDN_ERR_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
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
