// inst_tile_bf16_nk.cu -- one-CTA tile kernels, bf16 operands, weight N x K.
#include "inst_tile.cuh"

namespace ge_inst {
TileKernelFn tile_bf16_nk(int bn, int epi) { return tile_any<true, true>(bn, epi); }
}  // namespace ge_inst
