// inst_skinny.cuh -- instances of the few-row kernel for one operand type and
// stage depth (included by inst_skinny_*.cu).
#pragma once

#include "kernel_table.h"
#include "skinny_kernel.cuh"

namespace ge_inst {

template <int TP, int KPS, bool BF>
SkinnyKernelFn skinny_epi(int epi) {
  switch (epi) {
    case ge::EPI_BIAS: return ge::skinny_kernel<TP, KPS, ge::EPI_BIAS, BF>;
    case ge::EPI_RELU_BIAS: return ge::skinny_kernel<TP, KPS, ge::EPI_RELU_BIAS, BF>;
    case ge::EPI_RELU_AUX_BIAS: return ge::skinny_kernel<TP, KPS, ge::EPI_RELU_AUX_BIAS, BF>;
    case ge::EPI_DRELU_BGRAD: return ge::skinny_kernel<TP, KPS, ge::EPI_DRELU_BGRAD, BF>;
    case ge::EPI_GELU_BIAS: return ge::skinny_kernel<TP, KPS, ge::EPI_GELU_BIAS, BF>;
    case ge::EPI_GELU_AUX_BIAS: return ge::skinny_kernel<TP, KPS, ge::EPI_GELU_AUX_BIAS, BF>;
    case ge::EPI_STORE: return ge::skinny_kernel<TP, KPS, ge::EPI_STORE, BF>;
    default: return nullptr;  // WGRAD never runs on the few-row kernel
  }
}

template <int KPS, bool BF>
SkinnyKernelFn skinny_any(int tp, int epi) {
  switch (tp) {
    case 16: return skinny_epi<16, KPS, BF>(epi);
    case 32: return skinny_epi<32, KPS, BF>(epi);
    case 64: return skinny_epi<64, KPS, BF>(epi);
    case 128: return skinny_epi<128, KPS, BF>(epi);
    case 256: return skinny_epi<256, KPS, BF>(epi);
    default: return nullptr;
  }
}

}  // namespace ge_inst
