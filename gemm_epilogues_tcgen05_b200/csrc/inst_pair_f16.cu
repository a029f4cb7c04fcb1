// inst_pair_f16.cu -- CTA-pair tile kernels, f16 operands.
#include "inst_pair.cuh"

namespace ge_inst {
TileKernelFn pair_f16(int epi, bool bk) { return bk ? pair_epi<false, true, false>(epi) : pair_epi<false, false, false>(epi); }
}  // namespace ge_inst
