// Internal kernel launchers (host side), one per kernel family.
#pragma once

#include "common.cuh"

namespace gdn {

cudaError_t launch_gdn_seq(const GdnParams &p, int in_dtype, cudaStream_t st);
cudaError_t launch_gdn_frame_simt(const GdnParams &p, int in_dtype, int grid, cudaStream_t st);
cudaError_t launch_relu_frame_simt(const ReluParams &p, int in_dtype, int grid, cudaStream_t st);
// fills p.rope_tab (the 3D RoPE table) on the stream
cudaError_t launch_rope_table(const GdnParams &p, int frame_offset, float base, cudaStream_t st);

// tcgen05 / TMEM / TMA kernels (bf16 inputs, dk = dv in {16..128} multiples of 16).
bool gdn_tc_supported(int dk, int dv);
size_t gdn_tc_state_elems(int dk, int dv);
// cooperative: p.segs > 1; all CTAs resident at once (segments wait across CTAs both ways)
cudaError_t launch_gdn_tc(const GdnParams &p, int grid, bool cooperative, cudaStream_t st);
// product-form tensor-core kernel: one CTA per frame, sizes where its shared memory and
// TMEM maps fit (make_layout in gdn_pform.cu)
bool gdn_pform_supported(int dk, int dv);
size_t gdn_pform_state_bytes(int dk, int dv);  // published bytes per frame
cudaError_t launch_gdn_pform(const GdnParams &p, int grid, cudaStream_t st);
// causal temporal convolution with the block-boundary cache (one CTA per run of frames of a column tile)
cudaError_t launch_temporal_conv(const void *x, const float *w, const float *bias, const void *cache_in,
                                 void *cache_out, void *y, int B, int F, int HW, int C, int in_dtype, int max_ctas,
                                 cudaStream_t st);
// windowed block-causal softmax attention (bf16 q, k, v on tcgen05; fp32 o)
bool softmax_window_supported(int dk, int dv);
cudaError_t launch_softmax_window(const void *q, const void *k, const void *v, float *o, int B, int H, int F, int L,
                                  int dk, int dv, int W, float scale, int *status, unsigned long long spin_limit_ns,
                                  cudaStream_t st);
// the same on CUDA cores in fp32 (fp32 or bf16 inputs, any d_k, d_v up to 128)
cudaError_t launch_softmax_window_simt(const void *q, const void *k, const void *v, float *o, int B, int H, int F,
                                       int L, int dk, int dv, int W, float scale, int in_dtype, cudaStream_t st);
// backward of the Gated DeltaNet (after the recompute has filled p.maps and p.states):
// Q^T dO per frame, the adjoint frame chain, then the frame-parallel chunked backward;
// d_k, d_v <= 112.  rope: the 3D RoPE's table fields (rope.rope_on = 0: none)
bool gdn_bwd_supported(int dk, int dv);
int gdn_bwd_chunks(int L);  // 48-token chunks per frame of the frame kernel
cudaError_t launch_gdn_bwd(const BwdParams &p, const GdnParams &rope, int in_dtype, cudaStream_t st);
bool relu_tc_supported(int dk, int dv);
cudaError_t launch_relu_tc(const ReluParams &p, int grid, cudaStream_t st);

}  // namespace gdn
