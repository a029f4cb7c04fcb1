// inst_skinny_f16_kps1.cu -- few-row kernels, f16 operands, 1 k-block(s) per stage.
#include "inst_skinny.cuh"

namespace ge_inst {
SkinnyKernelFn skinny_f16_kps1(int tp, int epi) { return skinny_any<1, false>(tp, epi); }
}  // namespace ge_inst
