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
// (8 bf16 or 4 fp32; single elements when C is not a multiple of that) at one
// latent position and walks it along the frame axis, keeping x[f-1], x[f] and
// the next frames in registers, with two steps of kAhead frames loaded ahead.  The grid
// is one resident wave; each CTA takes an equal contiguous share of the
// (column tile, frame) index space, so its work is a few frame runs of one or
// two column tiles and no CTA waits on a tail.  A run re-reads one frame on
// each side (halo), about 2 frames per run of a few hundred.
#include <cuda_bf16.h>

#include <atomic>

#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kAhead = 4;  // frames loaded ahead per step

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

template <typename T, int V>
__global__ void __launch_bounds__(kThreads, 2) temporal_conv_kernel(ConvArgs a) {
  const long long total = a.tiles * a.F;  // (column tile, frame) items
  const long long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  for (long long t = lo / a.F; t * a.F < hi; ++t) {
    const long long s = t * a.F;
    const int fa = (int)((lo > s ? lo : s) - s);
    const int fb = (int)((hi < s + a.F ? hi : s + a.F) - s);
    const long long j = t * kThreads + threadIdx.x;
    if (fa < fb && j < a.cols) conv_run<T, V>(a, j, fa, fb);
  }
}

template <typename T, int V>
cudaError_t launch_typed(ConvArgs a, int sms, int max_ctas, cudaStream_t st) {
  static std::atomic<int> resident{0};  // CTAs of this kernel per SM (register-limited)
  int per_sm = resident.load(std::memory_order_relaxed);
  if (per_sm <= 0) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, temporal_conv_kernel<T, V>, kThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    resident.store(per_sm, std::memory_order_relaxed);
  }
  a.frame_cols /= V;
  a.cols /= V;
  a.tiles = (a.cols + kThreads - 1) / kThreads;
  long long grid = (long long)sms * per_sm;
  if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
  if (grid > a.tiles * a.F) grid = a.tiles * a.F;
  temporal_conv_kernel<T, V><<<(unsigned)grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_temporal_conv(const void *x, const float *w, const float *bias, const void *cache_in,
                                 void *cache_out, void *y, int B, int F, int HW, int C, int in_dtype, int sms,
                                 int max_ctas, cudaStream_t st) {
  ConvArgs a;
  a.x = x; a.w = w; a.bias = bias; a.cache_in = cache_in; a.cache_out = cache_out; a.y = y;
  a.F = F; a.C = C;
  a.frame_cols = (long long)HW * C;
  a.cols = (long long)B * a.frame_cols;
  a.tiles = 0;
  if (in_dtype == GDN_DTYPE_BF16)
    return C % 8 == 0 ? launch_typed<__nv_bfloat16, 8>(a, sms, max_ctas, st)
                      : launch_typed<__nv_bfloat16, 1>(a, sms, max_ctas, st);
  return C % 4 == 0 ? launch_typed<float, 4>(a, sms, max_ctas, st) : launch_typed<float, 1>(a, sms, max_ctas, st);
}

}  // namespace gdn
