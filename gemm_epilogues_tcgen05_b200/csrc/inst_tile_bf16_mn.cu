// inst_tile_bf16_mn.cu -- one-CTA tile kernels, bf16 operands, weight K x N.
#include "inst_tile.cuh"

namespace ge_inst {
TileKernelFn tile_bf16_mn(int bn, int epi) { return tile_any<true, false>(bn, epi); }
}  // namespace ge_inst
