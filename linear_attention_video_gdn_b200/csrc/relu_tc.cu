// Block-causal ReLU linear attention on tcgen05 tensor cores (bf16 inputs).
//
// SANA-Video ICLR 2026 oral talk transcript, block KV cache passage: the
// linear-attention state is a fixed D x D matrix; block f adds its own KV
// contribution to the cached state of block f-1 and every token of the block
// reads the result.  Per (b, h, f) work unit:
//
//  1. dS_f^T and dz_f^T in one MMA chain: D1 = [V_f | 1]^T relu(K_f), an
//     M=128 x N=dk fp32 accumulator in TMEM (row j < dv holds column j of dS,
//     row dv holds dz).  K_f, V_f stream through a 3-slot TMA ring in 64-token
//     chunks; relu is applied in shared memory, the ones column is written into
//     the V tile's padding.
//  2. Chain: S_f = S_{f-1} + dS_f (and z), S_{f-1} read from the workspace
//     once its producer's flag is set (bounded wait), S_f published, and S_f
//     written as the bf16 high / low B operands of the read-out.
//  3. Read-out: [num | den] = relu(Q_f) [S_f | z_f] as two MMAs over the
//     high and low halves (about 16 significant bits), M=128 tokens x N=128;
//     o = num / (den + eps) in the epilogue, stored as fp32.
//
// One persistent CTA per SM runs two pipelines on consecutive units, so the
// K/V stream of one unit and the Q / o stream of the one before are both in
// flight (each alone leaves HBM idle half the time):
//  - warps 0-3 (group A) take a ticket, run steps 1 and 2 and hand the unit
//    to group B through the high / low operands, then take the next ticket;
//  - warps 4-7 (group B, issue) load q tiles through a 2-slot ring, apply relu
//    and issue the read-out MMAs into one of two TMEM accumulators;
//  - warps 8-11 (group B, epilogue) divide and store the tile before.
// The high / low operands are single-buffered: group A writes the next unit's
// operands once the last read-out MMA of the unit before has completed.
// Group A announces each ticket when it takes it, so group B loads the first q
// tiles of the next unit while A still builds that unit's state.  S_{f-1}
// arrives in one bulk copy into the (then idle) K/V ring.  The epilogue writes
// o rows with 32-byte stores (full sectors) when o starts on a sector.
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace tc {

constexpr int kThreads = 384;
constexpr int kKvStages = 3;
constexpr int kQStages = 2;
constexpr uint32_t kStageBytes = 32768;

struct __align__(1024) ReluSmem {
  uint8_t kv[kKvStages][kStageBytes];  // K/V chunk: K at +0 (2 x 8 KB), V at +16 KB (2 x 8 KB)
  uint8_t q[kQStages][kStageBytes];    // q tile of 128 tokens: 2 x 16 KB
  uint8_t bhi[32768];                  // K-major B operand: [k-block][128 rows][128 B]
  uint8_t blo[32768];
  uint64_t kv_full[kKvStages];   // the chunk's TMA loads have landed
  uint64_t kv_empty[kKvStages];  // the MMAs reading the chunk have completed
  uint64_t q_full[kQStages];
  uint64_t q_empty[kQStages];
  uint64_t d1_done;    // step 1's MMAs of the unit have completed
  uint64_t d2_full[2]; // read-out: the MMAs into accumulator buffer b are done and tile_unit/tile_c
                       // name its tile (two arrivals: the issuing thread, then the MMA commit)
  uint64_t d2_free[2]; // read-out: the epilogue has read buffer b
  uint64_t b_ready;    // A -> B: the high / low operands hold unit b_unit (or b_unit < 0: stop)
  uint64_t b_free;     // B -> A: every read-out MMA of the unit has completed
  uint64_t fin;        // teardown: both MMA-issuing threads' MMAs have completed
  uint64_t prev_full;  // group A: the cached state S_{f-1} has landed in kv[0..1]
  uint64_t next_known[2];  // A -> B: ticket k of the CTA is next_unit[k & 1] (< 0: none), so that B
                           // loads its first q tiles while A still builds its state
  uint32_t tmem_base;
  int a_ticket;
  int abort;           // a bounded wait ran out somewhere in the CTA
  long long b_unit;
  long long tile_unit[2];  // unit of the tile in accumulator buffer b (< 0: stop)
  long long next_unit[2];
  int tile_c[2];           // its 128-token tile index within the frame
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

// 32-byte store (one full sector); p must be 32-byte aligned
__device__ __forceinline__ void st_v8(float *p, const float *v, float scale) {
  asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0] * scale), "f"(v[1] * scale),
               "f"(v[2] * scale), "f"(v[3] * scale), "f"(v[4] * scale), "f"(v[5] * scale), "f"(v[6] * scale),
               "f"(v[7] * scale)
               : "memory");
}

// named barriers (0 is __syncthreads)
constexpr int kBarA = 1;     // group A, 128 threads
constexpr int kBarIss = 2;   // group B issue warps, 128 threads
constexpr int kBarEpi = 3;   // group B epilogue warps, 128 threads

// Group A (warps 0-3): tickets, step 1 (D1 over the frame's K/V chunks) and
// step 2 (chain, publish, high / low operands), then the hand-over to group B.
__device__ __forceinline__ void relu_group_a(ReluSmem &sm, const CUtensorMap *tmap_k, const CUtensorMap *tmap_v,
                                             const ReluParams &p, uint32_t tD1) {
  const int tid = threadIdx.x;  // 0..127: TMEM lane = row of D1 = column j of [S | z]
  const int warp = tid >> 5;
  const int dk = p.dk, dv = p.dv, L = p.L, F = p.F;
  const int BH = p.B * p.H;
  const long units = (long)BH * F;
  const long slot = (long)(dv + 1) * dk;
  const unsigned long long lim = p.spin_limit_ns;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t idesc1 = idesc_f16(128, dk, 1, 1, 1);  // A = [V|1]^T (MN-major), B = relu(K) (MN-major)

  uint32_t loads = 0;  // K/V chunk loads issued (thread 0's count; slot = loads % 3)
  uint32_t used = 0;   // chunks consumed (all threads)
  uint32_t d1_phase = 0, prev_phase = 0;
  uint32_t handoffs = 0, tickets = 0;
  bool failed = false;

  // thread 0: load chunk `chunk` of unit (f, bh) into the next slot, once the
  // MMAs of that slot's previous chunk have completed
  auto issue_kv = [&](int chunk, int f, int bh) -> bool {
    const uint32_t g = loads++;
    const int s = (int)(g % kKvStages);
    if (g >= (uint32_t)kKvStages && !mbar_wait(&sm.kv_empty[s], ((g - kKvStages) / kKvStages) & 1u, lim))
      return false;
    uint64_t *bar = &sm.kv_full[s];
    mbar_expect_tx(bar, kStageBytes);
    const int t0 = chunk * 64;
    tma_load_4d(sm.kv[s] + 0, tmap_k, bar, 0, t0, f, bh);
    tma_load_4d(sm.kv[s] + 8192, tmap_k, bar, 64, t0, f, bh);
    tma_load_4d(sm.kv[s] + 16384, tmap_v, bar, 0, t0, f, bh);
    tma_load_4d(sm.kv[s] + 24576, tmap_v, bar, 64, t0, f, bh);
    return true;
  };

  for (;;) {
    // thread 0 decides for the group: a ticket, or past the end once the CTA aborts
    if (tid == 0) {
      const int tk = *(volatile int *)&sm.abort ? 0x7fffffff : atomicAdd(p.ws.counter, 1);
      sm.a_ticket = tk;
      sm.next_unit[tickets & 1u] = tk < units ? tk : -1;
      mbar_arrive_only(&sm.next_known[tickets & 1u]);
    }
    ++tickets;
    named_bar(kBarA, 128);
    const long ticket = sm.a_ticket;
    if (ticket >= units) break;
    const int f = (int)(ticket / BH);
    const int bh = (int)(ticket % BH);
    const int n1 = (L + 63) / 64;

    // ---- 1. D1 = [V | 1]^T relu(K) over the frame ----
    int bad = 0;
    if (tid == 0)
      for (int c = 0; c < n1 && c < kKvStages && !bad; ++c) bad = !issue_kv(c, f, bh);
    if (bar_sync_or(kBarA, 128, bad)) { failed = true; break; }
    for (int c = 0; c < n1; ++c) {
      const int s = (int)(used % kKvStages);
      bad = !mbar_wait(&sm.kv_full[s], (used / kKvStages) & 1u, lim);
      ++used;
      if (bar_sync_or(kBarA, 128, bad)) { failed = true; break; }
      relu_inplace(sm.kv[s], 16384, tid, 128);
      if (tid < 64) {
        const uint32_t off = 16384u + (uint32_t)(dv / 64) * 8192u + sw128_offset((uint32_t)tid, (uint32_t)(dv % 64));
        *reinterpret_cast<__nv_bfloat16 *>(sm.kv[s] + off) = __float2bfloat16(1.0f);
      }
      fence_async_smem();
      named_bar(kBarA, 128);
      if (tid == 0) {
        tc_fence_after();
        const uint32_t a0 = smem_u32(sm.kv[s] + 16384), b0 = smem_u32(sm.kv[s]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tD1, sdesc_sw128(a0 + kk * 2048, 8192, 1024), sdesc_sw128(b0 + kk * 2048, 8192, 1024),
                     idesc1, (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.kv_empty[s]);
        // chunk c + 2 goes into the slot of chunk c - 1, whose MMAs were issued
        // one chunk ago (chunks 0..2 were loaded up front)
        if (c >= 1 && c + 2 < n1 && !issue_kv(c + 2, f, bh)) bad = 1;
        if (c == n1 - 1) mma_commit(&sm.d1_done);
      }
    }
    if (failed) break;
    bad = !mbar_wait(&sm.d1_done, d1_phase, lim) || bad;
    d1_phase ^= 1u;

    // ---- 2. chain: S_f = S_{f-1} + dS_f, once group B is done with the operands ----
    // S_{f-1} comes in one bulk copy into the K/V ring (idle until the next
    // unit's loads), so the rows below read shared memory instead of paying an
    // L2 round trip per 16 columns
    if (tid == 0 && f > 0 && !bad) {
      bad = !wait_flag(p.ws.flags + (long)bh * F + (f - 1), 1, lim);
      if (!bad) {
        fence_async_global();  // the producer's generic stores before the async-proxy read
        const uint32_t bytes = (uint32_t)(slot * sizeof(float));
        mbar_expect_tx(&sm.prev_full, bytes);
        bulk_load(sm.kv[0], p.ws.states + ((long)bh * F + (f - 1)) * slot, bytes, &sm.prev_full);
      }
    }
    if (handoffs > 0 && !bad) bad = !mbar_wait(&sm.b_free, (handoffs - 1) & 1u, lim);
    if (bar_sync_or(kBarA, 128, bad)) { failed = true; break; }
    if (f > 0) {
      bad = !mbar_wait(&sm.prev_full, prev_phase, lim);
      prev_phase ^= 1u;
      if (bar_sync_or(kBarA, 128, bad)) { failed = true; break; }
    }
    tc_fence_after();
    {
      const int j = tid;
      const bool live = j <= dv;
      const float *prev = reinterpret_cast<const float *>(sm.kv[0]) + (long)j * dk;
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
              const float4 x = *reinterpret_cast<const float4 *>(prev + i0 + e);
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
    }
    fence_async_smem();
    tc_fence_before();
    named_bar(kBarA, 128);
    if (tid == 0) {
      if (ticket != p.withhold) {
        __threadfence();
        st_release(p.ws.flags + (long)bh * F + f, 1);
      }
      sm.b_unit = ticket;
      mbar_arrive_only(&sm.b_ready);
    }
    ++handoffs;
  }
  if (failed) {
    if (tid == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
    *(volatile int *)&sm.abort = 1;
  }
  // stop group B once it is done with the last unit handed over
  if (tid == 0) {
    if (handoffs > 0 && !failed && !mbar_wait(&sm.b_free, (handoffs - 1) & 1u, lim)) {
      latch_status(p.status, GDN_ERR_TIMEOUT);
      *(volatile int *)&sm.abort = 1;
    }
    sm.b_unit = -1;
    mbar_arrive_only(&sm.b_ready);
    // drain the K/V loads still in flight (a failed unit may leave some)
    for (uint32_t g = used; g < loads; ++g) mbar_wait(&sm.kv_full[g % kKvStages], (g / kKvStages) & 1u, lim);
  }
}

// Group B issue warps (4-7): q tiles of the unit handed over, relu, read-out
// MMAs into accumulator buffer (tile count & 1).
__device__ __forceinline__ void relu_group_b_issue(ReluSmem &sm, const CUtensorMap *tmap_q, const ReluParams &p,
                                                   uint32_t tD2a, uint32_t tD2b) {
  const int it = threadIdx.x - 128;
  const int dk = p.dk, L = p.L;
  const int BH = p.B * p.H;
  const unsigned long long lim = p.spin_limit_ns;
  const uint32_t idesc3 = idesc_f16(128, 128, 1, 0, 0);  // A = relu(Q) (K-major), B = S (K-major)
  const int nk3 = dk / 16;

  uint32_t handled = 0, loads = 0, used = 0, rt = 0;
  uint32_t known = 0;        // next_known waits done (thread 128)
  long long pf_unit = -1;    // unit whose first q tiles are already loading (thread 128)
  bool failed = false;
  auto issue_q = [&](int chunk, int f, int bh) -> bool {  // thread 128
    const uint32_t g = loads++;
    const int s = (int)(g % kQStages);
    if (g >= (uint32_t)kQStages && !mbar_wait(&sm.q_empty[s], ((g - kQStages) / kQStages) & 1u, lim)) return false;
    uint64_t *bar = &sm.q_full[s];
    mbar_expect_tx(bar, kStageBytes);
    tma_load_4d(sm.q[s] + 0, tmap_q, bar, 0, chunk * 128, f, bh);
    tma_load_4d(sm.q[s] + 16384, tmap_q, bar, 64, chunk * 128, f, bh);
    return true;
  };
  // thread 128: learn the CTA's next ticket and load its first q tiles
  auto prefetch_next = [&]() -> bool {
    const uint32_t k = known++;
    if (!mbar_wait(&sm.next_known[k & 1u], (k >> 1) & 1u, lim)) return false;
    pf_unit = sm.next_unit[k & 1u];
    if (pf_unit < 0) return true;
    const int f = (int)(pf_unit / BH), bh = (int)(pf_unit % BH);
    const int n3 = (L + 127) / 128;
    for (int c = 0; c < n3 && c < kQStages; ++c)
      if (!issue_q(c, f, bh)) return false;
    return true;
  };
  // thread 128: tell the epilogue to stop, at the next accumulator buffer
  auto send_stop = [&]() {
    const uint32_t b = rt & 1u;
    if (rt >= 2) mbar_wait(&sm.d2_free[b], ((rt >> 1) & 1u) ^ 1u, lim);
    sm.tile_unit[b] = -1;
    mbar_arrive_only(&sm.d2_full[b]);
    mbar_arrive_only(&sm.d2_full[b]);
  };

  int bad = 0;
  if (it == 0) bad = !prefetch_next();
  for (;;) {
    const bool ok = !bad && mbar_wait(&sm.b_ready, handled & 1u, lim);
    if (bar_sync_or(kBarIss, 128, !ok)) { failed = true; break; }
    const long long unit = sm.b_unit;
    if (unit < 0) break;
    ++handled;
    const int f = (int)(unit / BH);
    const int bh = (int)(unit % BH);
    const int n3 = (L + 127) / 128;
    // the first tiles were loaded ahead: the hand-over order is the ticket order
    if (it == 0 && unit != pf_unit) bad = 1;
    for (int c = 0; c < n3; ++c) {
      const int s = (int)(used % kQStages);
      if (it == 0 && !bad) bad = !mbar_wait(&sm.q_full[s], (used / kQStages) & 1u, lim);
      ++used;
      if (bar_sync_or(kBarIss, 128, bad)) { failed = true; break; }
      relu_inplace(sm.q[s], 32768, it, 128);
      fence_async_smem();
      named_bar(kBarIss, 128);
      if (it == 0) {
        const uint32_t gt = rt + c, b = gt & 1u, ph = (gt >> 1) & 1u;
        const uint32_t tD = b ? tD2b : tD2a;
        bad = gt >= 2 && !mbar_wait(&sm.d2_free[b], ph ^ 1u, lim);  // tile gt - 2 has left buffer b
        if (!bad) {
          sm.tile_unit[b] = unit;
          sm.tile_c[b] = c;
          mbar_arrive_only(&sm.d2_full[b]);
          tc_fence_after();
          const uint32_t a0 = smem_u32(sm.q[s]), bh0 = smem_u32(sm.bhi), bl0 = smem_u32(sm.blo);
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
          mma_commit(&sm.q_empty[s]);
          if (c == n3 - 1) mma_commit(&sm.b_free);  // group A may overwrite the operands
          // tile c + 1 goes into the slot of tile c - 1, whose MMAs were issued one tile ago
          if (c >= 1 && c + 1 < n3) bad = !issue_q(c + 1, f, bh);
        }
      }
    }
    rt += (uint32_t)n3;
    if (failed) break;
    if (it == 0 && !bad) bad = !prefetch_next();
  }
  if (failed) {
    if (it == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
    *(volatile int *)&sm.abort = 1;
  }
  if (it == 0) {
    send_stop();
    for (uint32_t g = used; g < loads; ++g) mbar_wait(&sm.q_full[g % kQStages], (g / kQStages) & 1u, lim);
  }
}

// Group B epilogue warps (8-11): o = num / (den + eps) of each read-out tile,
// in the order the issue warps filled the accumulator buffers.
__device__ __forceinline__ void relu_group_b_epilogue(ReluSmem &sm, const ReluParams &p, uint32_t tD2a,
                                                      uint32_t tD2b) {
  const int et = threadIdx.x - 256;  // TMEM lane = token row of the tile
  const int warp = threadIdx.x >> 5;
  const int dv = p.dv, L = p.L, F = p.F;
  const int BH = p.B * p.H;
  const long N = (long)F * L;
  const unsigned long long lim = p.spin_limit_ns;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  // rows are dv * 4 bytes (a multiple of 32): 32-byte stores when o starts on a sector
  const bool o_sector_aligned = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
  bool failed = false;
  for (uint32_t gt = 0;; ++gt) {
    const uint32_t b = gt & 1u;
    const uint32_t tD = b ? tD2b : tD2a;
    int bad = 0;
    if (et == 0) bad = !mbar_wait(&sm.d2_full[b], (gt >> 1) & 1u, lim);
    if (bar_sync_or(kBarEpi, 128, bad)) { failed = true; break; }
    const long long unit = sm.tile_unit[b];
    if (unit < 0) break;
    const int f = (int)(unit / BH), bh = (int)(unit % BH), c = sm.tile_c[b];
    tc_fence_after();
    const int t = c * 128 + et;
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
          float *dst = orow + (cb + h) * 16;
          if (o_sector_aligned) {  // full 32-byte sectors: half the store instructions
            st_v8(dst, r[h], inv);
            st_v8(dst + 8, r[h] + 8, inv);
          } else {
            float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_float4(r[h][4 * e] * inv, r[h][4 * e + 1] * inv, r[h][4 * e + 2] * inv,
                                  r[h][4 * e + 3] * inv);
          }
        }
      }
    }
    tc_fence_before();
    named_bar(kBarEpi, 128);
    if (et == 0) mbar_arrive_only(&sm.d2_free[b]);
  }
  if (failed) {
    if (et == 0) latch_status(p.status, GDN_ERR_TIMEOUT);
    *(volatile int *)&sm.abort = 1;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    relu_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, ReluParams p) {
  extern __shared__ uint8_t smem_raw[];
  ReluSmem &sm = *reinterpret_cast<ReluSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  if (tid == 0) {
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
    }
    mbar_init(&sm.d1_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.d2_full[b], 2);
      mbar_init(&sm.d2_free[b], 1);
    }
    mbar_init(&sm.b_ready, 1);
    mbar_init(&sm.b_free, 1);
    mbar_init(&sm.fin, 2);
    mbar_init(&sm.prev_full, 1);
    mbar_init(&sm.next_known[0], 1);
    mbar_init(&sm.next_known[1], 1);
    sm.abort = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tD1 = tmem;                                // columns [0, 128): step 1
  const uint32_t tD2a = tmem + 128, tD2b = tmem + 256;      // read-out accumulators

  if (warp < 4)
    relu_group_a(sm, &tmap_k, &tmap_v, p, tD1);
  else if (warp < 8)
    relu_group_b_issue(sm, &tmap_q, p, tD2a, tD2b);
  else
    relu_group_b_epilogue(sm, p, tD2a, tD2b);

  // every MMA of both issuing threads has completed before TMEM is released
  if (tid == 0 || tid == 128) mma_commit(&sm.fin);
  if (tid == 0) mbar_wait(&sm.fin, 0, p.spin_limit_ns);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
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
  static_assert(sizeof(ReluSmem) + 1024 <= 232448, "shared memory of one CTA");
  if ((size_t)(p.dv + 1) * p.dk * sizeof(float) > 2 * kStageBytes) return cudaErrorInvalidValue;  // S in kv[0..1]
  cudaError_t e = cudaFuncSetAttribute(relu_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  relu_tc_kernel<<<grid, kThreads, smem, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn
