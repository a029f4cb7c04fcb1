// inst_skinny_bf16_kps1.cu -- few-row kernels, bf16 operands, 1 k-block(s) per stage.
#include "inst_skinny.cuh"

namespace ge_inst {
SkinnyKernelFn skinny_bf16_kps1(int tp, int epi) { return skinny_any<1, true>(tp, epi); }
}  // namespace ge_inst
