// inst_tile_f16_mn.cu -- one-CTA tile kernels, f16 operands, weight K x N.
#include "inst_tile.cuh"

namespace ge_inst {
TileKernelFn tile_f16_mn(int bn, int epi) { return tile_any<false, false>(bn, epi); }
}  // namespace ge_inst
