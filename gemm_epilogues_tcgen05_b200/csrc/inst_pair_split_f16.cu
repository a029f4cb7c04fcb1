// inst_pair_split_f16.cu -- CTA-pair tile kernels in stream-K mode (fewer
// tiles than pairs), f16 operands, weight K x N or N x K.
#include "inst_pair.cuh"

namespace ge_inst {
TileKernelFn pair_split_f16(int epi, bool bk) {
  return bk ? pair_epi<false, true, true>(epi) : pair_epi<false, false, true>(epi);
}
}  // namespace ge_inst
