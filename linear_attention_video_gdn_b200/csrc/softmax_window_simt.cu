// Windowed block-causal softmax attention on CUDA cores, fp32 arithmetic: the
// path for fp32 inputs (1e-5 tolerance) and for head sizes the tensor-core
// kernel does not take (d_k or d_v not a multiple of 16).  Same definition as
// softmax_window.cu: token t of frame f attends to every token of frames
// max(0, f-W+1) .. f, o_t = sum_s softmax_s(scale q_t . k_s) v_s.
//
// One warp per query row: lane i holds q and the output accumulator at
// dimensions i, i+32, i+64, i+96.  Keys are visited in order with the running
// maximum updated at every key (exact online softmax); k and v rows are read
// by the warp as whole 128-byte lines.
#include <cuda_bf16.h>

#include "launch.h"

namespace gdn {
namespace {

constexpr int kSwsWarps = 8;  // query rows per CTA

template <typename T>
__device__ __forceinline__ float ld_elem(const T *p) {
  return (float)p[0];
}
template <>
__device__ __forceinline__ float ld_elem<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(p[0]);
}

template <typename T>
__global__ void __launch_bounds__(32 * kSwsWarps)
    softmax_window_simt_kernel(const T *q, const T *k, const T *v, float *o, int F, int L, int dk, int dv, int W,
                               float scale) {
  const int lane = threadIdx.x & 31;
  const int nqt = (L + kSwsWarps - 1) / kSwsWarps;
  const long unit = blockIdx.x;
  const int qt = (int)(unit % nqt);
  const int f = (int)((unit / nqt) % F);
  const long bh = unit / ((long)nqt * F);
  const int t = qt * kSwsWarps + (threadIdx.x >> 5);  // query row in the frame
  if (t >= L) return;
  const long N = (long)F * L;
  const T *qt_row = q + (bh * N + (long)f * L + t) * dk;
  float qr[4], acc[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int i = lane + 32 * e;
    qr[e] = i < dk ? ld_elem(qt_row + i) : 0.0f;
    acc[e] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  const int f0 = max(0, f - W + 1);
  const long s0 = bh * N + (long)f0 * L, s1 = bh * N + (long)(f + 1) * L;
  for (long s = s0; s < s1; ++s) {
    const T *ks = k + s * dk;
    float dot = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = lane + 32 * e;
      if (i < dk) dot = fmaf(qr[e], ld_elem(ks + i), dot);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float x = dot * scale;
    const T *vs = v + s * dv;
    if (x > m) {  // new maximum: rescale what was accumulated
      const float a = expf(m - x);  // 0 for the first key (m = -inf)
      l = l * a + 1.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = lane + 32 * e;
        acc[e] = c < dv ? fmaf(acc[e], a, ld_elem(vs + c)) : 0.0f;
      }
      m = x;
    } else {
      const float pr = expf(x - m);
      l += pr;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = lane + 32 * e;
        if (c < dv) acc[e] = fmaf(pr, ld_elem(vs + c), acc[e]);
      }
    }
  }
  float *orow = o + (bh * N + (long)f * L + t) * dv;
  const float inv = 1.0f / l;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = lane + 32 * e;
    if (c < dv) orow[c] = acc[e] * inv;
  }
}

}  // namespace

cudaError_t launch_softmax_window_simt(const void *q, const void *k, const void *v, float *o, int B, int H, int F,
                                       int L, int dk, int dv, int W, float scale, int in_dtype, cudaStream_t st) {
  const long grid = (long)B * H * F * ((L + kSwsWarps - 1) / kSwsWarps);
  if (grid > 0x7fffffffL) return cudaErrorInvalidValue;
  if (in_dtype == GDN_DTYPE_F32)
    softmax_window_simt_kernel<float><<<(unsigned)grid, 32 * kSwsWarps, 0, st>>>(
        static_cast<const float *>(q), static_cast<const float *>(k), static_cast<const float *>(v), o, F, L, dk, dv,
        W, scale);
  else
    softmax_window_simt_kernel<__nv_bfloat16><<<(unsigned)grid, 32 * kSwsWarps, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), o, F, L, dk, dv, W, scale);
  return cudaGetLastError();
}

}  // namespace gdn
