// kernel_table.h -- the compiled kernel instances, as host-side function
// pointers. The instances live in separate translation units (inst_*.cu),
// grouped by operand type, weight layout and stage depth, so that the build
// compiles them in parallel; gemm_epi.cu picks them through these functions
// and launches them through the pointers.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace ge {
struct TileParams;
struct SkinnyParams;
}  // namespace ge

namespace ge_inst {

using TileKernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, ge::TileParams);
using SkinnyKernelFn = void (*)(CUtensorMap, CUtensorMap, ge::SkinnyParams);

// One CTA per tile, BN = 64, 128, 192 or 256 columns (8, 6, 4 or 4 stages); `epi` is
// a ge::EpiKind. _mn: the weight is K x N; _nk: N x K (no WGRAD: nullptr).
TileKernelFn tile_f16_mn(int bn, int epi);
TileKernelFn tile_f16_nk(int bn, int epi);
TileKernelFn tile_bf16_mn(int bn, int epi);
TileKernelFn tile_bf16_nk(int bn, int epi);

// CTA pairs, 256 x 256 tiles, 6 stages; bk: the weight is N x K. _split:
// stream-K over the pairs (fewer tiles than pairs).
TileKernelFn pair_f16(int epi, bool bk);
TileKernelFn pair_bf16(int epi, bool bk);
TileKernelFn pair_split_f16(int epi, bool bk);
TileKernelFn pair_split_bf16(int epi, bool bk);

// Few-row kernel: TP = 16, 32, 64, 128 or 256 padded rows, KPS = 1 or 2
// k-blocks per stage; every epilog but WGRAD.
SkinnyKernelFn skinny_f16_kps1(int tp, int epi);
SkinnyKernelFn skinny_f16_kps2(int tp, int epi);
SkinnyKernelFn skinny_bf16_kps1(int tp, int epi);
SkinnyKernelFn skinny_bf16_kps2(int tp, int epi);

}  // namespace ge_inst
