// inst_pair_split_bf16.cu -- CTA-pair tile kernels in stream-K mode (fewer
// tiles than pairs), bf16 operands, weight K x N or N x K.
#include "inst_pair.cuh"

namespace ge_inst {
TileKernelFn pair_split_bf16(int epi, bool bk) {
  return bk ? pair_epi<true, true, true>(epi) : pair_epi<true, false, true>(epi);
}
}  // namespace ge_inst
