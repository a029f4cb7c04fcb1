// inst_pair.cuh -- instances of the CTA-pair tile kernel for one operand
// type, both weight layouts (included by inst_pair_*.cu).
#pragma once

#include "kernel_table.h"
#include "tile2_kernel.cuh"

namespace ge_inst {

template <bool BF, bool BK, bool SPLIT>
TileKernelFn pair_epi(int epi) {
  switch (epi) {
    case ge::EPI_BIAS: return ge::tile2_kernel<256, 6, ge::EPI_BIAS, BF, BK, SPLIT>;
    case ge::EPI_RELU_BIAS: return ge::tile2_kernel<256, 6, ge::EPI_RELU_BIAS, BF, BK, SPLIT>;
    case ge::EPI_RELU_AUX_BIAS: return ge::tile2_kernel<256, 6, ge::EPI_RELU_AUX_BIAS, BF, BK, SPLIT>;
    case ge::EPI_DRELU_BGRAD: return ge::tile2_kernel<256, 6, ge::EPI_DRELU_BGRAD, BF, BK, SPLIT>;
    // eight epilogue warps (whole tiles): their staging leaves room for 5 stages
    case ge::EPI_GELU_BIAS: return ge::tile2_kernel<256, SPLIT ? 6 : 5, ge::EPI_GELU_BIAS, BF, BK, SPLIT>;
    case ge::EPI_GELU_AUX_BIAS: return ge::tile2_kernel<256, SPLIT ? 6 : 5, ge::EPI_GELU_AUX_BIAS, BF, BK, SPLIT>;
    case ge::EPI_WGRAD:
      if constexpr (BK)
        return nullptr;
      else
        return ge::tile2_kernel<256, 6, ge::EPI_WGRAD, BF, false, SPLIT>;
    case ge::EPI_STORE: return ge::tile2_kernel<256, 6, ge::EPI_STORE, BF, BK, SPLIT>;
    default: return nullptr;
  }
}

}  // namespace ge_inst
