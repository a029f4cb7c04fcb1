// inst_tile_f16_nk.cu -- one-CTA tile kernels, f16 operands, weight N x K.
#include "inst_tile.cuh"

namespace ge_inst {
TileKernelFn tile_f16_nk(int bn, int epi) { return tile_any<false, true>(bn, epi); }
}  // namespace ge_inst
