// Block-causal ReLU linear attention on tcgen05 tensor cores (bf16 inputs).
//
// SANA-Video ICLR 2026 oral talk transcript, block KV cache passage: the
// linear-attention state is a fixed D x D matrix; block f adds its own KV
// contribution to the cached state of block f-1 and every token of the block
// reads the result.  Per (b, h, f) work unit, one persistent CTA:
//
//  1. dS_f^T and dz_f^T in one MMA chain: D1 = [V_f | 1]^T relu(K_f), an
//     M=128 x N=dk fp32 accumulator in TMEM (row j < dv holds column j of dS,
//     row dv holds dz).  K_f, V_f stream through a 3-stage TMA ring in
//     64-token chunks; relu is applied in shared memory, the ones column is
//     written into the V tile's padding.
//  2. Chain: S_f = S_{f-1} + dS_f (and z), S_{f-1} read from the workspace
//     once its producer's flag is set (bounded wait), S_f published.
//  3. Read-out: [num | den] = relu(Q_f) [S_f | z_f] as bf16 hi + lo halves of
//     the fp32 state (two MMAs, ~16 significant bits), M=128 tokens x N=128;
//     o = num / (den + eps) in the epilogue, stored as fp32.  Warps 0-3 apply
//     relu to each q tile and thread 0 issues its MMAs into TMEM buffer n & 1
//     (D1's columns are free by then) while warps 4-7 run the epilogue of the
//     tile before.
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {

constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr uint32_t kStageBytes = 32768;

struct __align__(1024) ReluSmem {
  uint8_t ring[kStages][kStageBytes];  // K/V chunk: K at +0 (2 x 8 KB), V at +16 KB; Q chunk: 2 x 16 KB
  uint8_t bhi[32768];                  // K-major B operand: [k-block][128 rows][128 B]
  uint8_t blo[32768];
  uint64_t full[kStages];
  uint64_t mma_bar;
  uint64_t d2_full[2];  // read-out: the MMAs into accumulator buffer b are done
  uint64_t d2_free[2];  // read-out: the epilogue has read buffer b
  uint32_t tmem_base;
  int ticket;
};

__device__ __forceinline__ void relu_inplace(uint8_t *p, int nbytes, int tid, int nthreads) {
  const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
  for (int i = tid * 16; i < nbytes; i += nthreads * 16) {
    uint4 x = *reinterpret_cast<uint4 *>(p + i);
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __hmax2(h[e], zero);
    *reinterpret_cast<uint4 *>(p + i) = x;
  }
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

__global__ void __launch_bounds__(kThreads, 1)
    relu_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, ReluParams p) {
  extern __shared__ uint8_t smem_raw[];
  ReluSmem &sm = *reinterpret_cast<ReluSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const int BH = p.B * p.H;
  const long units = (long)BH * F;
  const long N = (long)F * L;
  const long slot = (long)(dv + 1) * dk;
  const unsigned long long lim = p.spin_limit_ns;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
    mbar_init(&sm.mma_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.d2_full[b], 1);
      mbar_init(&sm.d2_free[b], 1);
    }
    mbar_fence_init();
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tD1 = tmem;        // columns [0, 128)
  const uint32_t tD2 = tmem + 128;  // columns [128, 256)
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

  const uint32_t idesc1 = idesc_f16(128, dk, 1, 1, 1);   // A = [V|1]^T (MN-major), B = relu(K) (MN-major)
  const uint32_t idesc3 = idesc_f16(128, 128, 1, 0, 0);  // A = relu(Q) (K-major), B = S (K-major)
  const int nk3 = dk / 16;

  uint32_t loads = 0;     // loads issued (all threads track the same count)
  uint32_t consumed = 0;  // loads consumed
  uint32_t mma_phase = 0;
  uint32_t rt = 0;        // read-out tiles of earlier units (buffer n & 1 and its phases)
  bool failed = false;

  auto issue_kv = [&](int chunk, int f, int bh) {
    const int s = loads % kStages;
    uint64_t *bar = &sm.full[s];
    mbar_expect_tx(bar, kStageBytes);
    const int t0 = chunk * 64;
    tma_load_4d(sm.ring[s] + 0, &tmap_k, bar, 0, t0, f, bh);
    tma_load_4d(sm.ring[s] + 8192, &tmap_k, bar, 64, t0, f, bh);
    tma_load_4d(sm.ring[s] + 16384, &tmap_v, bar, 0, t0, f, bh);
    tma_load_4d(sm.ring[s] + 24576, &tmap_v, bar, 64, t0, f, bh);
  };
  auto issue_q = [&](int chunk, int f, int bh) {
    const int s = loads % kStages;
    uint64_t *bar = &sm.full[s];
    mbar_expect_tx(bar, kStageBytes);
    const int t0 = chunk * 128;
    tma_load_4d(sm.ring[s] + 0, &tmap_q, bar, 0, t0, f, bh);
    tma_load_4d(sm.ring[s] + 16384, &tmap_q, bar, 64, t0, f, bh);
  };
  // all threads: wait for the oldest issued load; returns false on timeout (collective)
  auto wait_load = [&]() -> bool {
    const int s = consumed % kStages;
    const bool ok = mbar_wait(&sm.full[s], (consumed / kStages) & 1u, lim);
    return !__syncthreads_or(!ok);
  };
  auto wait_mma = [&]() -> bool {
    const bool ok = mbar_wait(&sm.mma_bar, mma_phase, lim);
    mma_phase ^= 1u;
    return !__syncthreads_or(!ok);
  };

  for (;;) {
    if (tid == 0) sm.ticket = atomicAdd(p.ws.counter, 1);
    __syncthreads();
    const long ticket = sm.ticket;
    if (ticket >= units) break;
    const int f = (int)(ticket / BH);
    const int bh = (int)(ticket % BH);
    const int n1 = (L + 63) / 64;
    const int n3 = (L + 127) / 128;

    // ---- 1. D1 = [V | 1]^T relu(K) over the frame ----
    if (tid == 0)
      for (int c = 0; c < n1 && c < kStages; ++c) {
        issue_kv(c, f, bh);
        ++loads;
      }
    if (tid != 0) loads += (uint32_t)min(n1, kStages);
    for (int c = 0; c < n1; ++c) {
      const int s = consumed % kStages;
      if (!wait_load()) { failed = true; break; }
      ++consumed;
      relu_inplace(sm.ring[s], 16384, tid, kThreads);
      if (tid < 64) {
        const uint32_t off = 16384u + (uint32_t)(dv / 64) * 8192u + sw128_offset((uint32_t)tid, (uint32_t)(dv % 64));
        *reinterpret_cast<__nv_bfloat16 *>(sm.ring[s] + off) = __float2bfloat16(1.0f);
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t a0 = smem_u32(sm.ring[s] + 16384), b0 = smem_u32(sm.ring[s]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tD1, sdesc_sw128(a0 + kk * 2048, 8192, 1024), sdesc_sw128(b0 + kk * 2048, 8192, 1024),
                     idesc1, (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.mma_bar);
      }
      if (!wait_mma()) { failed = true; break; }
      if (c + kStages < n1) {
        if (tid == 0) issue_kv(c + kStages, f, bh);
        ++loads;
      }
    }
    if (failed) break;

    // ---- 2. chain: S_f = S_{f-1} + dS_f ----
    int bad = 0;
    if (tid == 0 && f > 0) {
      if (!wait_flag(p.ws.flags + (long)bh * F + (f - 1), 1, lim)) bad = 1;
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
      failed = true;
      break;
    }
    tc_fence_after();
    if (warp >= 4) {
      const int j = tid - 128;  // TMEM lane = row of D1 = column j of [S | z]
      const bool live = j <= dv;
      const float *prev = p.ws.states + ((long)bh * F + (f - 1)) * slot + (long)j * dk;
      float *cur = p.ws.states + ((long)bh * F + f) * slot + (long)j * dk;
      // 16 columns (i = d_k index) at a time: add the cached state, publish, and
      // write the bf16 hi/lo B-operand row j.
#pragma unroll 1
      for (int cb = 0; cb < 8; ++cb) {
        float r[16];
        if (cb * 16 < dk) {
          tmem_ld16(tD1 + lane_off + cb * 16, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = 0.f;
        }
        if (live && cb * 16 < dk) {
          const int i0 = cb * 16;
          if (f > 0) {
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 x = __ldcg(reinterpret_cast<const float4 *>(prev + i0 + e));
              r[e] += x.x; r[e + 1] += x.y; r[e + 2] += x.z; r[e + 3] += x.w;
            }
          } else if (j < dv && p.kv_in) {
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] += p.kv_in[(long)bh * dk * dv + (long)(i0 + e) * dv + j];
          } else if (j == dv && p.z_in) {
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] += p.z_in[(long)bh * dk + i0 + e];
          }
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4 *>(cur + i0 + e) = make_float4(r[e], r[e + 1], r[e + 2], r[e + 3]);
          if (f == F - 1) {
            if (j < dv && p.kv_out) {
#pragma unroll
              for (int e = 0; e < 16; ++e) p.kv_out[(long)bh * dk * dv + (long)(i0 + e) * dv + j] = r[e];
            } else if (j == dv && p.z_out) {
#pragma unroll
              for (int e = 0; e < 16; ++e) p.z_out[(long)bh * dk + i0 + e] = r[e];
            }
          }
        } else if (!live) {
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = 0.f;
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = r[half * 8 + 2 * e], x1 = r[half * 8 + 2 * e + 1];
            const float h0 = __bfloat162float(__float2bfloat16(x0));
            const float h1 = __bfloat162float(__float2bfloat16(x1));
            hi[e] = pack_bf16x2(h0, h1);
            lo[e] = pack_bf16x2(x0 - h0, x1 - h1);
          }
          const int ch = cb * 2 + half;  // 8-element chunk index along d_k
          const uint32_t off = (uint32_t)(ch / 8) * 16384u + sw128_offset((uint32_t)j, (uint32_t)((ch % 8) * 8));
          *reinterpret_cast<uint4 *>(sm.bhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4 *>(sm.blo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (ticket != p.withhold) {
        __threadfence();
        st_release(p.ws.flags + (long)bh * F + f, 1);
      }
      for (int c = 0; c < n3 && c < kStages; ++c) {
        issue_q(c, f, bh);
        ++loads;
      }
    }
    if (tid != 0) loads += (uint32_t)min(n3, kStages);

    // ---- 3. read-out: o = relu(Q) S / (relu(Q) z + eps) ----
    if (warp < 4) {
      for (int c = 0; c < n3; ++c) {
        const int s = consumed % kStages;
        {
          int bad = 0;
          if (tid == 0) bad = !mbar_wait(&sm.full[s], (consumed / kStages) & 1u, lim);
          if (bar_sync_or(1, 128, bad)) {
            failed = true;
            break;
          }
        }
        ++consumed;
        relu_inplace(sm.ring[s], 32768, tid, 128);
        fence_async_smem();
        named_bar(1, 128);
        int bad = 0;
        if (tid == 0) {
          const uint32_t gt = rt + c, b = gt & 1u, ph = (gt >> 1) & 1u;
          const uint32_t tD = b ? tD1 : tD2;
          bad = gt >= 2 && !mbar_wait(&sm.d2_free[b], ph ^ 1u, lim);  // tile n - 2 has left buffer b
          if (!bad) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(sm.ring[s]), bh0 = smem_u32(sm.bhi), bl0 = smem_u32(sm.blo);
            for (int kk = 0; kk < nk3; ++kk) {
              const uint32_t off = (uint32_t)(kk / 4) * 16384u + (uint32_t)(kk % 4) * 32u;
              mma_f16_ss(tD, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(bh0 + off, 16, 1024), idesc3,
                         kk > 0 ? 1u : 0u);
            }
            for (int kk = 0; kk < nk3; ++kk) {
              const uint32_t off = (uint32_t)(kk / 4) * 16384u + (uint32_t)(kk % 4) * 32u;
              mma_f16_ss(tD, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(bl0 + off, 16, 1024), idesc3, 1u);
            }
            mma_commit(&sm.d2_full[b]);
            // the ring stage is free once these MMAs are done: q tile c + 3 goes there
            if (c + kStages < n3) {
              bad = !mbar_wait(&sm.d2_full[b], ph, lim);
              if (!bad) issue_q(c + kStages, f, bh);
            }
          }
        }
        if (c + kStages < n3) ++loads;
        if (bar_sync_or(1, 128, bad)) {
          failed = true;
          break;
        }
      }
    } else {
      for (int c = 0; c < n3; ++c) {
        const uint32_t gt = rt + c, b = gt & 1u;
        const uint32_t tD = b ? tD1 : tD2;
        {
          int bad = 0;
          if (tid == 128) bad = !mbar_wait(&sm.d2_full[b], (gt >> 1) & 1u, lim);
          if (bar_sync_or(2, 128, bad)) {
            failed = true;
            break;
          }
        }
        tc_fence_after();
        const int t = c * 128 + (tid - 128);
        float inv;  // 1 / (relu(q)^T z + eps), one division per token
        {
          float r[16];
          tmem_ld16(tD + lane_off + (uint32_t)(dv & ~15), r);
          tmem_ld_wait();
          inv = 1.0f / (r[dv & 15] + p.eps);
        }
        float *orow = p.o + ((long)bh * N + (long)f * L + t) * dv;
#pragma unroll 1
        for (int cb = 0; cb < dv / 16; cb += 2) {  // 32 columns per TMEM wait
          float r[2][16];
          tmem_ld16(tD + lane_off + cb * 16, r[0]);
          if (cb + 1 < dv / 16) tmem_ld16(tD + lane_off + (cb + 1) * 16, r[1]);
          tmem_ld_wait();
          if (t < L) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (cb + h >= dv / 16) break;
              float4 *dst = reinterpret_cast<float4 *>(orow + (cb + h) * 16);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_float4(r[h][4 * e] * inv, r[h][4 * e + 1] * inv, r[h][4 * e + 2] * inv,
                                     r[h][4 * e + 3] * inv);
            }
          }
        }
        tc_fence_before();
        named_bar(2, 128);
        if (tid == 128) mbar_arrive_only(&sm.d2_free[b]);
      }
      consumed += (uint32_t)n3;
      loads += (uint32_t)(n3 > kStages ? n3 - kStages : 0);
    }
    rt += (uint32_t)n3;
    if (__syncthreads_or(failed ? 1 : 0)) {
      failed = true;
      break;
    }
  }
  if (failed && tid == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace tc

bool relu_tc_supported(int dk, int dv) {
  return dk % 16 == 0 && dv % 16 == 0 && dk >= 16 && dk <= 128 && dv >= 16 && dv <= 112;
}

cudaError_t launch_relu_tc(const ReluParams &p, int grid, cudaStream_t st) {
  using namespace tc;
  CUtensorMap mq, mk, mv;
  const int BH = p.B * p.H;
  if (!make_bf16_map(&mq, p.q, p.dk, p.L, p.F, BH, 128) || !make_bf16_map(&mk, p.k, p.dk, p.L, p.F, BH, 64) ||
      !make_bf16_map(&mv, p.v, p.dv, p.L, p.F, BH, 64))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(ReluSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(relu_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  relu_tc_kernel<<<grid, kThreads, smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn
