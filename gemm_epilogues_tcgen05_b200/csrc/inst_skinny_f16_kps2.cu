// inst_skinny_f16_kps2.cu -- few-row kernels, f16 operands, 2 k-block(s) per stage.
#include "inst_skinny.cuh"

namespace ge_inst {
SkinnyKernelFn skinny_f16_kps2(int tp, int epi) { return skinny_any<2, false>(tp, epi); }
}  // namespace ge_inst
