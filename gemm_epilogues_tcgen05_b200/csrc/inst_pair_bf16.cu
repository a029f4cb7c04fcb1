// inst_pair_bf16.cu -- CTA-pair tile kernels, bf16 operands.
#include "inst_pair.cuh"

namespace ge_inst {
TileKernelFn pair_bf16(int epi, bool bk) { return bk ? pair_epi<true, true, false>(epi) : pair_epi<true, false, false>(epi); }
}  // namespace ge_inst
