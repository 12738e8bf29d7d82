// Host helpers of the tcgen05 kernels.
#pragma once

#include <cuda.h>

namespace gdn {
namespace tc {

// bf16 tensor [BH, F, L, d] (row-major) as a 4-D TMA map whose boxes are 64
// elements of d by `rows` tokens of one frame, 128-byte swizzled.  Rows past
// the frame's end read as zeros.  False if the driver entry point is missing
// or the encoder rejects the map.
bool make_bf16_map(CUtensorMap *m, const void *base, int d, int L, int F, int BH, int rows);

}  // namespace tc
}  // namespace gdn
