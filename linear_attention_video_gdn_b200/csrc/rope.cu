// The table of the 3D rotary position embedding: cos and sin of every angle
// pos * base^(-2i / part_length) a call uses, one float2 per (axis position,
// pair), time part first (one row per frame of the call), then the height
// rows, then the width columns of the latent grid.  The angles are formed in
// double and rounded once.
#include "launch.h"

namespace gdn {

__global__ void rope_table_kernel(float2 *tab, int F, int rows, int gw, int dt, int dh, int frame_offset,
                                  double base) {
  const int nt = F * (dt / 2), nh = rows * (dh / 2), nw = gw * (dh / 2);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < nt + nh + nw; e += gridDim.x * blockDim.x) {
    int pos, i, len;
    if (e < nt) {
      pos = frame_offset + e / (dt / 2);
      i = e % (dt / 2);
      len = dt;
    } else if (e < nt + nh) {
      pos = (e - nt) / (dh / 2);
      i = (e - nt) % (dh / 2);
      len = dh;
    } else {
      pos = (e - nt - nh) / (dh / 2);
      i = (e - nt - nh) % (dh / 2);
      len = dh;
    }
    const double phi = (double)pos * pow(base, -2.0 * (double)i / (double)len);
    double sn, cs;
    sincos(phi, &sn, &cs);
    tab[e] = make_float2((float)cs, (float)sn);
  }
}

cudaError_t launch_rope_table(const GdnParams &p, int frame_offset, float base, cudaStream_t st) {
  const int rows = p.L / p.rope_gw;
  const size_t n = rope_table_entries(p.F, p.L, p.rope_gw, p.dk);
  const int threads = 256;
  int blocks = (int)((n + threads - 1) / threads);
  if (blocks > 1024) blocks = 1024;
  if (blocks < 1) blocks = 1;
  rope_table_kernel<<<blocks, threads, 0, st>>>(const_cast<float2 *>(p.rope_tab), p.F, rows, p.rope_gw, p.rope_dt,
                                                p.rope_dh, frame_offset, (double)base);
  return cudaGetLastError();
}

}  // namespace gdn
