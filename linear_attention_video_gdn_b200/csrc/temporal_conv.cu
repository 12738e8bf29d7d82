// Causal temporal convolution of one block of latent frames with the
// block-boundary cache (SANA-Video talk, causal FFN passage: in training a zero
// token separates consecutive blocks and the later block is prefixed with the
// earlier block's last frame; generated block by block, the same result comes
// from carrying that last frame in a cache).
//
//   y[b,f,n,c] = w[c][0] x[b,f-1,n,c] + w[c][1] x[b,f,n,c] + w[c][2] x[b,f+1,n,c] + bias[c]
//   x[b,-1] = cache_in[b] (zero without one), x[b,F] = 0, cache_out[b] = x[b,F-1]
//
// HBM-bound streaming kernel: every element of x is read once and every
// element of y written once.  A thread owns one 16-byte column of channels
// (8 bf16 or 4 fp32) at one latent position and walks it along the frame
// axis over a run of up to kRun frames, keeping x[f-1] and x[f] in registers;
// the frames after f are prefetched 8-12 deep by asynchronous copies
// (cp.async, 16 bytes each) into the thread's own slots of a shared-memory
// ring, so the bytes in flight cost no registers and no thread waits on
// another.  The arithmetic runs on packed fp32 pairs (fma.rn.f32x2).  When C is
// not a multiple of the vector, single elements are walked the same way with
// register prefetch.  One CTA takes one run of one tile of kThreads columns;
// the runs of a tile are neighbouring CTAs, so the frame a run re-reads on
// each side (halo) is usually still in L2.  Many small CTAs (several waves)
// let the hardware balance the SMs, and each CTA's start-up latency overlaps
// other CTAs' transfers.
#include <cuda_bf16.h>

#include "f32x2.cuh"
#include "launch.h"
#include "tc_ptx.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 128;
constexpr int kRun = 32;  // frames per CTA run
constexpr int kAhead = 4;  // frames loaded ahead per step (single-element columns)
// frames prefetched per thread into shared memory (16-byte columns): deeper
// where fewer CTAs fit an SM (bf16 columns hold more registers)
template <int V> __host__ __device__ constexpr int ring_depth() { return V == 8 ? 12 : 8; }

// A vector of V channels as it sits in memory (Raw) and in registers (float[V]).
template <typename T, int V> struct Col;

template <> struct Col<__nv_bfloat16, 8> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw load(const void *p) { return __ldcs(reinterpret_cast<const uint4 *>(p)); }
  static __device__ __forceinline__ Raw load_keep(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }
  static __device__ __forceinline__ Raw zero() { return make_uint4(0u, 0u, 0u, 0u); }
  static __device__ __forceinline__ void to_float(const Raw &r, float (&v)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void store(void *p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(w[0], w[1], w[2], w[3]));
  }
  static __device__ __forceinline__ void store_raw(void *p, const Raw &r) { *reinterpret_cast<uint4 *>(p) = r; }
  // channel pairs (2i, 2i+1) as packed fp32 pairs (low word = channel 2i)
  static __device__ __forceinline__ void to_pairs(const Raw &r, uint64_t (&v)[4]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = pack2(w[i] << 16, w[i] & 0xffff0000u);
  }
  static __device__ __forceinline__ void store_pairs(void *p, const uint64_t (&v)[4]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = (uint32_t)v[i], hi = (uint32_t)(v[i] >> 32);
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[i]) : "f"(__uint_as_float(hi)), "f"(__uint_as_float(lo)));
    }
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(w[0], w[1], w[2], w[3]));
  }
};

template <> struct Col<float, 4> {
  using Raw = float4;
  static __device__ __forceinline__ Raw load(const void *p) { return __ldcs(reinterpret_cast<const float4 *>(p)); }
  static __device__ __forceinline__ Raw load_keep(const void *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
  static __device__ __forceinline__ Raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  static __device__ __forceinline__ void to_float(const Raw &r, float (&v)[4]) {
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
  }
  static __device__ __forceinline__ void store(void *p, const float (&v)[4]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
  }
  static __device__ __forceinline__ void store_raw(void *p, const Raw &r) { *reinterpret_cast<float4 *>(p) = r; }
  static __device__ __forceinline__ void to_pairs(const Raw &r, uint64_t (&v)[2]) {
    v[0] = pack2(__float_as_uint(r.x), __float_as_uint(r.y));
    v[1] = pack2(__float_as_uint(r.z), __float_as_uint(r.w));
  }
  static __device__ __forceinline__ void store_pairs(void *p, const uint64_t (&v)[2]) {
    __stcs(reinterpret_cast<float4 *>(p),
           make_float4(__uint_as_float((uint32_t)v[0]), __uint_as_float((uint32_t)(v[0] >> 32)),
                       __uint_as_float((uint32_t)v[1]), __uint_as_float((uint32_t)(v[1] >> 32))));
  }
};

template <typename T> struct Col<T, 1> {
  using Raw = T;
  static __device__ __forceinline__ Raw load(const void *p) { return *reinterpret_cast<const T *>(p); }
  static __device__ __forceinline__ Raw load_keep(const void *p) { return *reinterpret_cast<const T *>(p); }
  static __device__ __forceinline__ Raw zero() { return T(0.0f); }
  static __device__ __forceinline__ void to_float(const Raw &r, float (&v)[1]) { v[0] = (float)r; }
  static __device__ __forceinline__ void store(void *p, const float (&v)[1]) { *reinterpret_cast<T *>(p) = T(v[0]); }
  static __device__ __forceinline__ void store_raw(void *p, const Raw &r) { *reinterpret_cast<T *>(p) = r; }
};

struct ConvArgs {
  const void *x;
  const float *w, *bias;
  const void *cache_in;
  void *cache_out, *y;
  long long frame_cols;  // HW * C / V columns of one frame of one batch
  long long cols;        // B * frame_cols
  long long tiles;       // ceil(cols / kThreads)
  int F, C;
};

// One frame run [fa, fb) of column j (caller checks j < cols).
template <typename T, int V>
__device__ __forceinline__ void conv_run(const ConvArgs &a, long long j, int fa, int fb) {
  using K = Col<T, V>;
  using Raw = typename K::Raw;
  constexpr int es = (int)sizeof(T);
  const long long b = j / a.frame_cols, r = j - b * a.frame_cols;
  const long long fstride = a.frame_cols * V * es;  // bytes from one frame to the next
  const char *xb = static_cast<const char *>(a.x) + (b * a.F * a.frame_cols + r) * V * es;
  char *yb = static_cast<char *>(a.y) + (b * a.F * a.frame_cols + r) * V * es;
  const int c0 = (int)((r * V) % a.C);
  float w0[V], w1[V], w2[V], bb[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    w0[i] = __ldg(a.w + 3 * (c0 + i));
    w1[i] = __ldg(a.w + 3 * (c0 + i) + 1);
    w2[i] = __ldg(a.w + 3 * (c0 + i) + 2);
    bb[i] = a.bias ? __ldg(a.bias + c0 + i) : 0.0f;
  }
  const long long cofs = (b * a.frame_cols + r) * V * es;  // this column in a [B, HW, C] cache
  Raw prev_raw;
  if (fa > 0)
    prev_raw = K::load_keep(xb + (long long)(fa - 1) * fstride);
  else
    prev_raw = a.cache_in ? K::load_keep(static_cast<const char *>(a.cache_in) + cofs) : K::zero();
  Raw cur_raw = K::load(xb + (long long)fa * fstride);
  // frames f+1 .. f+kAhead of the current step; the next step's are loaded
  // before this step's outputs are formed (two steps of loads in flight)
  Raw nx[kAhead];
  auto fetch = [&](Raw(&dst)[kAhead], int first) {
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int g = first + u;  // frame fb is the run's right halo
      dst[u] = (g <= fb && g < a.F) ? (g == fb ? K::load_keep(xb + (long long)g * fstride)
                                               : K::load(xb + (long long)g * fstride))
                                    : K::zero();
    }
  };
  fetch(nx, fa + 1);
  for (int f = fa; f < fb; f += kAhead) {
    Raw nn[kAhead];
    fetch(nn, f + 1 + kAhead);
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      if (f + u < fb) {
        // x values stay in their stored form (exact) until used
        float prev[V], cur[V], nxt[V], out[V];
        K::to_float(prev_raw, prev);
        K::to_float(cur_raw, cur);
        K::to_float(nx[u], nxt);
#pragma unroll
        for (int i = 0; i < V; ++i) out[i] = fmaf(w2[i], nxt[i], fmaf(w1[i], cur[i], fmaf(w0[i], prev[i], bb[i])));
        K::store(yb + (long long)(f + u) * fstride, out);
        prev_raw = cur_raw;
        cur_raw = nx[u];
      }
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) nx[u] = nn[u];
  }
  // The owner of frame 0 read cache_in above and now writes cache_out, so one
  // thread touches both (cache_in == cache_out is allowed).
  if (fa == 0 && a.cache_out) {
    const Raw last = K::load_keep(xb + (long long)(a.F - 1) * fstride);
    K::store_raw(static_cast<char *>(a.cache_out) + cofs, last);
  }
}

__device__ __forceinline__ void cp_async16(void *sdst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One frame run [fa, fb) of 16-byte column j; frames fa+1 .. fb (fb is the
// run's right halo) come through the thread's ring slots
// ring[s * kThreads + threadIdx.x], s < R, R = ring_depth frames ahead.
template <typename T, int V>
__device__ __forceinline__ void conv_run_ring(const ConvArgs &a, long long j, int fa, int fb, uint4 *ring) {
  using K = Col<T, V>;
  using Raw = typename K::Raw;
  static_assert(sizeof(Raw) == 16, "ring slots hold 16-byte columns");
  constexpr int R = ring_depth<V>();
  constexpr int es = (int)sizeof(T);
  const long long b = j / a.frame_cols, r = j - b * a.frame_cols;
  const long long fstride = a.frame_cols * V * es;  // bytes from one frame to the next
  const char *xb = static_cast<const char *>(a.x) + (b * a.F * a.frame_cols + r) * V * es;
  char *yb = static_cast<char *>(a.y) + (b * a.F * a.frame_cols + r) * V * es;
  uint4 *mine = ring + threadIdx.x;
  const int last = fb < a.F ? fb : a.F - 1;  // last frame the run reads
  const char *src = xb + (long long)(fa + 1) * fstride;  // next frame to prefetch
  int next = fa + 1;
#pragma unroll
  for (int k = 0; k < R; ++k) {  // slot k <- frame fa + 1 + k
    if (next <= last) cp_async16(mine + k * kThreads, src);
    cp_async_commit();
    ++next;
    src += fstride;
  }
  constexpr int NP = V / 2;  // channel pairs
  const int c0 = (int)((r * V) % a.C);
  uint64_t w0[NP], w1[NP], w2[NP], bb[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const float *wa = a.w + 3 * (c0 + 2 * i);  // rows c0+2i and c0+2i+1 of w
    w0[i] = pack2(__float_as_uint(__ldg(wa)), __float_as_uint(__ldg(wa + 3)));
    w1[i] = pack2(__float_as_uint(__ldg(wa + 1)), __float_as_uint(__ldg(wa + 4)));
    w2[i] = pack2(__float_as_uint(__ldg(wa + 2)), __float_as_uint(__ldg(wa + 5)));
    bb[i] = a.bias ? pack2(__float_as_uint(__ldg(a.bias + c0 + 2 * i)), __float_as_uint(__ldg(a.bias + c0 + 2 * i + 1)))
                   : 0ull;
  }
  const long long cofs = (b * a.frame_cols + r) * V * es;  // this column in a [B, HW, C] cache
  Raw prev_raw;
  if (fa > 0)
    prev_raw = K::load_keep(xb + (long long)(fa - 1) * fstride);
  else
    prev_raw = a.cache_in ? K::load_keep(static_cast<const char *>(a.cache_in) + cofs) : K::zero();
  Raw cur_raw = K::load(xb + (long long)fa * fstride);
  uint64_t prev[NP], cur[NP];  // x[f-1], x[f] as fp32 pairs (exact)
  K::to_pairs(prev_raw, prev);
  K::to_pairs(cur_raw, cur);
  char *dst = yb + (long long)fa * fstride;
  for (int f = fa; f < fb; f += R) {
#pragma unroll
    for (int u = 0; u < R; ++u) {  // frame f + u reads slot u (frame f + u + 1)
      if (f + u < fb) {
        cp_async_wait<R - 1>();
        Raw nx_raw = K::zero();
        if (f + u + 1 <= last) nx_raw = *reinterpret_cast<const Raw *>(mine + u * kThreads);
        // refill the slot just read with frame f + u + 1 + R
        if (next <= last) cp_async16(mine + u * kThreads, src);
        cp_async_commit();
        ++next;
        src += fstride;
        uint64_t nxt[NP], out[NP];
        K::to_pairs(nx_raw, nxt);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          out[i] = fma2(w2[i], nxt[i], fma2(w1[i], cur[i], fma2(w0[i], prev[i], bb[i])));
          prev[i] = cur[i];
          cur[i] = nxt[i];
        }
        K::store_pairs(dst, out);
        dst += fstride;
      }
    }
  }
  cp_async_wait<0>();
  // The owner of frame 0 read cache_in above and now writes cache_out, so one
  // thread touches both (cache_in == cache_out is allowed).
  if (fa == 0 && a.cache_out)  // the last frame, as stored (exact)
    K::store_raw(static_cast<char *>(a.cache_out) + cofs, K::load_keep(xb + (long long)(a.F - 1) * fstride));
}

template <typename T, int V>
__global__ void __launch_bounds__(kThreads, V == 8 ? 4 : 6) temporal_conv_kernel(ConvArgs a) {
  extern __shared__ uint4 ring[];  // [ring_depth][kThreads] (16-byte columns)
  const long long runs = (a.F + kRun - 1) / kRun;  // runs per tile
  const long long items = a.tiles * runs;          // one item = one run of one tile
  for (long long id = blockIdx.x; id < items; id += gridDim.x) {
    const long long t = id / runs;
    const int fa = (int)(id - t * runs) * kRun;
    const int fb = fa + kRun < a.F ? fa + kRun : a.F;
    const long long j = t * kThreads + threadIdx.x;
    if (j < a.cols) {
      if constexpr (V == 1)
        conv_run<T, V>(a, j, fa, fb);
      else
        conv_run_ring<T, V>(a, j, fa, fb, ring);
    }
  }
}

template <typename T, int V>
cudaError_t launch_typed(ConvArgs a, int max_ctas, cudaStream_t st) {
  const size_t ring_bytes = V == 1 ? 0 : sizeof(uint4) * ring_depth<V>() * kThreads;
  static_assert(sizeof(uint4) * ring_depth<8>() * kThreads <= 48 * 1024, "ring within the default shared memory");
  a.frame_cols /= V;
  a.cols /= V;
  a.tiles = (a.cols + kThreads - 1) / kThreads;
  long long grid = a.tiles * ((a.F + kRun - 1) / kRun);  // one CTA per item
  if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;  // fewer CTAs loop over the items
  if (grid > 0x7fffffffLL) grid = 0x7fffffffLL;
  temporal_conv_kernel<T, V><<<(unsigned)grid, kThreads, ring_bytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_temporal_conv(const void *x, const float *w, const float *bias, const void *cache_in,
                                 void *cache_out, void *y, int B, int F, int HW, int C, int in_dtype, int max_ctas,
                                 cudaStream_t st) {
  ConvArgs a;
  a.x = x; a.w = w; a.bias = bias; a.cache_in = cache_in; a.cache_out = cache_out; a.y = y;
  a.F = F; a.C = C;
  a.frame_cols = (long long)HW * C;
  a.cols = (long long)B * a.frame_cols;
  a.tiles = 0;
  if (in_dtype == GDN_DTYPE_BF16)
    return C % 8 == 0 ? launch_typed<__nv_bfloat16, 8>(a, max_ctas, st)
                      : launch_typed<__nv_bfloat16, 1>(a, max_ctas, st);
  return C % 4 == 0 ? launch_typed<float, 4>(a, max_ctas, st) : launch_typed<float, 1>(a, max_ctas, st);
}

}  // namespace gdn
