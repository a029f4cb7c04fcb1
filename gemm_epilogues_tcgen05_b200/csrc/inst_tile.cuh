// inst_tile.cuh -- instances of the one-CTA tile kernel for one operand type
// and weight layout (included by inst_tile_*.cu).
#pragma once

#include "kernel_table.h"
#include "tile_kernel.cuh"

namespace ge_inst {

template <int BN, int ST, bool BF, bool BK>
TileKernelFn tile_epi(int epi) {
  switch (epi) {
    case ge::EPI_BIAS: return ge::tile_kernel<BN, ST, ge::EPI_BIAS, BF, BK>;
    case ge::EPI_RELU_BIAS: return ge::tile_kernel<BN, ST, ge::EPI_RELU_BIAS, BF, BK>;
    case ge::EPI_RELU_AUX_BIAS: return ge::tile_kernel<BN, ST, ge::EPI_RELU_AUX_BIAS, BF, BK>;
    case ge::EPI_DRELU_BGRAD: return ge::tile_kernel<BN, ST, ge::EPI_DRELU_BGRAD, BF, BK>;
    case ge::EPI_GELU_BIAS: return ge::tile_kernel<BN, ST, ge::EPI_GELU_BIAS, BF, BK>;
    case ge::EPI_GELU_AUX_BIAS: return ge::tile_kernel<BN, ST, ge::EPI_GELU_AUX_BIAS, BF, BK>;
    case ge::EPI_WGRAD:
      if constexpr (BK)
        return nullptr;  // the weight gradient's operands have no weight layout to choose
      else
        return ge::tile_kernel<BN, ST, ge::EPI_WGRAD, BF>;
    case ge::EPI_STORE: return ge::tile_kernel<BN, ST, ge::EPI_STORE, BF, BK>;
    default: return nullptr;
  }
}

template <bool BF, bool BK>
TileKernelFn tile_any(int bn, int epi) {
  if (bn == 256) return tile_epi<256, 4, BF, BK>(epi);
  if (bn == 192) return tile_epi<192, 4, BF, BK>(epi);
  if (bn == 128) return tile_epi<128, 6, BF, BK>(epi);
  if (bn == 64) return tile_epi<64, 8, BF, BK>(epi);
  return nullptr;
}

}  // namespace ge_inst
