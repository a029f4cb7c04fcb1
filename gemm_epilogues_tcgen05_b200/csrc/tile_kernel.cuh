// tile_kernel.cuh -- persistent tcgen05 GEMM with the fused linear-layer
// epilogues (BIAS, RELU_BIAS, RELU_AUX_BIAS, DRELU_BGRAD, and a plain store
// for the unfused measurement path).
//
// One CTA per SM walks a static tile schedule. Warp roles:
//   warp 0      TMA producer: X tile (128 x 64, K-major) and W tile
//               (64 x BN, N-major) per stage into a STAGES-deep ring of
//               128-byte-swizzled shared memory, guarded by full/empty mbarriers
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma
//               (M=128, N=BN, K=16) into one of two fp32 accumulators and
//               commits each stage back to the producer
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one row per thread,
//               32 consecutive columns per load), bias from shared memory,
//               ReLU, mask words, 16-bit stores; for DRELU_BGRAD the mask is
//               applied and each tile's column sums are reduced in a fixed
//               order and written as one partial row per 128-row tile.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.
//
// Every wait on an mbarrier is bounded: on expiry the kernel records a code
// in the plan's status word, raises a CTA-wide abort flag, lets its issued
// copies and MMAs finish, frees its tensor memory and returns.
#pragma once

#include "ptx.cuh"

namespace ge {

// The values match gemm_epi_epilog; EPI_STORE (plain store of X.W) is the
// public NONE and the unfused ablation's GEMM.
enum EpiKind : int {
  EPI_BIAS = 0,
  EPI_RELU_BIAS = 1,
  EPI_RELU_AUX_BIAS = 2,
  EPI_DRELU_BGRAD = 3,
  EPI_GELU_BIAS = 4,
  EPI_WGRAD = 5,
  EPI_STORE = 6,
  EPI_GELU_AUX_BIAS = 7  // GELU_BIAS, and the pre-activation Z stored (16-bit) as the auxiliary output
};

// Epilogs that apply GELU.
template <int EPI>
struct AppliesGelu {
  static constexpr bool value = EPI == EPI_GELU_BIAS || EPI == EPI_GELU_AUX_BIAS;
};

// The weight gradient dW = X^T dZ reads its A operand (X^T, M = the features
// of X) straight from row-major X: M is the contiguous index, so A is
// MN-major and staged like W, as two 64-wide chunks per 128-row tile.
template <int EPI>
struct AOperandMN {
  static constexpr bool value = EPI == EPI_WGRAD;
};
constexpr uint32_t kAChunkMN = 64 * 64 * 2;  // one 64-wide M chunk x 64 k (8 KB)

// Epilogs whose output is the plain rounded accumulator.
template <int EPI>
struct PlainStore {
  static constexpr bool value = EPI == EPI_STORE || EPI == EPI_WGRAD;
};

// A operand descriptor for K step kk (16 elements) of a stage at a0:
// K-major: 128-byte rows, 8-row groups 1024 B apart, a K step is 32 bytes
// inside the swizzle atom; MN-major: 64-wide M chunks 8 KB apart (LBO), 8
// K-rows 1024 B apart (SBO), a K step is 16 rows = 2048 bytes.
// B operand descriptor for K step kk of a stage at b0. MN-major (W is K x N):
// 64-wide N chunks `chunk` bytes apart (LBO), 8 K-rows 1024 B apart (SBO), a
// K step of 16 rows is 2048 bytes. K-major (W is N x K): 128-byte rows of 64
// k, 8-row groups 1024 B apart, a K step is 32 bytes inside the swizzle atom.
__device__ __forceinline__ uint64_t b_desc(uint32_t b0, int kk, bool k_major, uint32_t chunk) {
  return k_major ? smem_desc_sw128(b0 + kk * 32, 16, 1024) : smem_desc_sw128(b0 + kk * 2048, chunk, 1024);
}

template <bool A_MN>
__device__ __forceinline__ uint64_t a_desc(uint32_t a0, int kk) {
  if constexpr (A_MN)
    return smem_desc_sw128(a0 + kk * 2048, kAChunkMN, 1024);
  else
    return smem_desc_sw128(a0 + kk * 32, 16, 1024);
}

// Epilogs that add the bias.
template <int EPI>
struct AddsBias {
  static constexpr bool value =
      EPI == EPI_BIAS || EPI == EPI_RELU_BIAS || EPI == EPI_RELU_AUX_BIAS || EPI == EPI_GELU_BIAS ||
      EPI == EPI_GELU_AUX_BIAS;
};

// GELU(z) = z * Phi(z), Phi the standard normal CDF, through CUDA's erff.
__device__ __forceinline__ float gelu_erf(float z) { return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f)); }

struct TileParams {
  int32_t T, N, K;
  int32_t m_tiles, n_tiles, k_blocks, num_tiles;
  int32_t aux_words;        // ceil(N / 32)
  int32_t group_m;          // row (or, with raster_n, column) tiles per raster group (see tile_coords)
  const void* bias;         // N values of the 16-bit type (forward)
  void* out;                // T x N, 16-bit: Y, dZ, or the unfused intermediate
  uint32_t* aux_out;        // RELU_AUX_BIAS mask words (GELU_AUX_BIAS: T x N 16-bit Z, stored through tmAux)
  const uint32_t* aux_in;   // DRELU_BGRAD mask words
  float* partials;          // DRELU_BGRAD: m_tiles x N column partial sums
  int* status;              // watchdog report (host-visible)
  uint64_t timeout_ns;
  int32_t inject_stall;     // fault injection for tests: withhold the first tile's tmem_full commit
                            // (one-CTA kernel: the CTA's first tile; CTA pairs: the leader's first unit)
  int32_t aux_tma;          // RELU_AUX_BIAS: mask words go out by TMA store (see AuxByTma)
  int* col_tickets;         // DRELU_BGRAD: per column block, zero between launches; null = no in-kernel finish
  float* dbias;             // DRELU_BGRAD: written by the tile that takes a column block's last ticket
  int32_t tail_split;       // pair kernel: split the last round's tiles into column halves
  int32_t bias_f32;         // the bias is N fp32 values (else the 16-bit type)
  int32_t out_f32;          // the output (Y, dZ or dW) is fp32 (else the 16-bit type)
  int32_t raster_n;         // tile order by column groups (see tile_coords)
  // CTA-pair stream-K (few tiles): the k-blocks of all tiles are cut into one
  // contiguous range per pair; a tile's later segments leave fp32 partials
  float* sk_slots;          // [pairs][2 ranks][128 rows][256 cols]: a pair's later segment
  int* sk_flags;            // [pairs][2 ranks]: segments in for the tile the pair finishes; zero between launches
  int32_t sk_max_segs;
  int32_t sk_first;         // stream-K tiles before the whole tiles (else after them)
};

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;
// output staging: each epilogue warp owns two 32 x 32 16-bit blocks (2 KB
// each), written to global memory by TMA stores
constexpr uint32_t kStageBytesPerWarp = 2 * 2048;
// mask-word staging: each epilogue warp's 32 rows x (BN / 32) words of a tile
constexpr uint32_t kAuxStageBytesPerWarp = 1024;

template <int BN, int STAGES>
struct TileSmem {
  static constexpr uint32_t A_BYTES = kBM * kBK * 2;          // 16 KB
  static constexpr uint32_t B_CHUNK = kBK * 64 * 2;           // 8 KB: 64 K-rows x 64 N
  static constexpr uint32_t B_BYTES = (BN / 64) * B_CHUNK;
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_B + STAGES * B_BYTES;
  static constexpr uint32_t N_BARS = 2 * STAGES + 5;          // full, empty, tfull[2], tempty[2], drain
  static constexpr uint32_t OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem slot, abort flag
  static constexpr uint32_t OFF_BIAS = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr uint32_t OFF_COLP = OFF_BIAS + 2 * BN * 4;
  static constexpr uint32_t OFF_STG = (OFF_COLP + 2 * 4 * BN * 4 + 1023) / 1024 * 1024;
  static constexpr uint32_t OFF_AUXSTG = OFF_STG + kStageBytesPerWarp * 4;
  static constexpr uint32_t END = OFF_AUXSTG + kAuxStageBytesPerWarp * 4;
  static constexpr uint32_t BYTES = END + 1024;               // + alignment slack
};

// Tile order (raster). By rows (by_n = 0): groups of `group` row tiles;
// inside a group the row tile varies fastest, then the column tile, so
// consecutive CTAs share W's column block and the group's rows of X stay in
// L2 while the group sweeps every column block. By columns (by_n = 1): the
// same with the roles swapped -- groups of `group` column tiles whose block
// of W stays in L2 while the group sweeps every row tile of X; the better
// order when X is much larger than W.
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int group, int by_n, int& mb,
                                            int& nb) {
  const int outer = by_n ? n_tiles : m_tiles;  // the dimension that is grouped
  const int inner = by_n ? m_tiles : n_tiles;
  const int per_group = group * inner;
  const int g = tile / per_group;
  const int first = g * group;
  const int gsize = min(outer - first, group);
  const int r = tile - g * per_group;
  const int a = first + r % gsize, b = r / gsize;
  mb = by_n ? b : a;
  nb = by_n ? a : b;
}

static __device__ __noinline__ void report_timeout(int* status, volatile int* abort_flag, int site) {
  *abort_flag = 1;
  if (status) {
    *reinterpret_cast<volatile int*>(status) = 0x7100 | site;
    __threadfence_system();
  }
}

// Wait for the phase of parity `parity` on `bar`. Returns false if the CTA
// is aborting or the wait exceeded the time limit (then it raises the abort).
// Each test suspends the thread for up to ~20 us (mbar_try_wait), so the
// abort flag and the clock are checked after every test.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const TileParams& p,
                                             volatile int* abort_flag, int site, bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (globaltimer_ns() - t0 > p.timeout_ns) {
      report_timeout(p.status, abort_flag, site);
      return false;
    }
  }
}

template <bool BF16>
__device__ __forceinline__ float load_16(const void* base, int64_t i) {
  if constexpr (BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  else
    return __half2float(reinterpret_cast<const __half*>(base)[i]);
}

// bias[n] as fp32, stored either as fp32 or in the 16-bit type
template <bool BF16>
__device__ __forceinline__ float load_bias(const void* bias, int bias_f32, int64_t n) {
  return bias_f32 ? reinterpret_cast<const float*>(bias)[n] : load_16<BF16>(bias, n);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

// Sum 32 per-lane vectors across the warp: on return, v[0] of lane j holds
// the sum over all 32 lanes of their v[j]. Each step halves the columns a
// lane keeps and swaps the other half with its partner, in a fixed order.
__device__ __forceinline__ void warp_transpose_reduce32(float (&v)[32]) {
  const uint32_t lane = lane_id();
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = keep + recv;
    }
  }
}

// ---------------------------------------------------------------------------
// Epilogue pieces shared by the one-CTA and the CTA-pair tile kernels. One
// epilogue thread owns one accumulator row (its TMEM lane) of a 128-row block.

// Stage the tile's bias values (fp32) in shared memory.
template <int BN, int EPI, bool BF16, int NT = 128>
__device__ __forceinline__ void epi_stage_bias(const TileParams& p, int n0, float* bs, uint32_t et, int ncols = BN) {
  if constexpr (AddsBias<EPI>::value) {
    for (int c = et; c < ncols; c += NT) {
      const int n = n0 + c;
      bs[c] = n < p.N ? load_bias<BF16>(p.bias, p.bias_f32, n) : 0.f;
    }
  }
}

// Drain row `row` (columns n0 .. n0+BN) of the accumulator at TMEM address
// `tbase` (this warp's lane quarter, the buffer's first column) through the
// epilogue: bias, ReLU, mask word, 16-bit stores; for DRELU_BGRAD the mask
// select and this warp's column sums into cpw[0..BN).
// Mask words go out through shared memory and one TMA store per warp and
// tile when a row's words are a multiple of 16 bytes (BN = 128, 256); with
// BN = 64 or 192 (8 or 24 bytes) they are stored directly.
template <int BN>
struct AuxByTma {
  static constexpr bool value = BN == 128 || BN == 256;  // a TMA box row must be a multiple of 16 bytes
};

// DRELU_BGRAD: this row's mask words for a tile. The epilogue loads them
// before it waits for the tile's accumulator, so the loads overlap the MMAs
// (and no load follows a store it could not be moved above).
template <int BN>
struct MaskWords {
  uint32_t w[BN / 32];
};

template <int BN>
__device__ __forceinline__ MaskWords<BN> load_mask_words(const TileParams& p, int row, int n0) {
  MaskWords<BN> m;
  const bool row_ok = row < p.T;
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    const int nc0 = n0 + c * 32;
    m.w[c] = (row_ok && nc0 < p.N) ? __ldg(p.aux_in + static_cast<int64_t>(row) * p.aux_words + (nc0 >> 5)) : 0u;
  }
  return m;
}

// Stage a warp's 32 x 32 block of 16-bit values (row = lane, 64 bytes) with
// the 64-byte swizzle -- 16-byte chunk q of row r at chunk q ^ ((r >> 1) & 3)
// -- so the 16-byte shared stores are conflict-free, then one lane writes the
// block with a TMA store at column x, row y (rows and columns past the
// tensor's extent are clipped by the tensor map). The buffer used two blocks
// ago must have been read by its store before it is overwritten.
template <bool BF16>
__device__ __forceinline__ void store_block16(const float (&v)[32], const CUtensorMap* map, uint8_t* stg,
                                              uint32_t& scount, int x, int y) {
  const uint32_t lane = lane_id();
  uint8_t* buf = stg + (scount & 1u) * 2048;
  if (lane == 0) bulk_wait_group_read<1>();
  __syncwarp();
  const uint32_t rbase = smem_u32(buf) + lane * 64;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack2<BF16>(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack2<BF16>(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack2<BF16>(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack2<BF16>(v[8 * q + 6], v[8 * q + 7]);
    st_shared_v4(rbase + ((q ^ ((lane >> 1) & 3u)) * 16), w);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, buf, x, y);
    bulk_commit_group();
  }
  ++scount;
}

// This thread's 32 consecutive values of row `row` from column nc0, rounded
// to the 16-bit type, into the T x N auxiliary output (GELU_AUX_BIAS):
// four 16-byte stores when the whole segment is inside the tensor (and
// 16-byte aligned, as it is when N is a multiple of 8), else element by
// element up to N.
template <bool BF16>
__device__ __forceinline__ void store_row16(const float (&v)[32], const TileParams& p, int row, int nc0) {
  if (row >= p.T) return;
  uint16_t* base = reinterpret_cast<uint16_t*>(p.aux_out) + static_cast<int64_t>(row) * p.N + nc0;
  if (nc0 + 32 <= p.N) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack2<BF16>(v[8 * q + 0], v[8 * q + 1]);
      w.y = pack2<BF16>(v[8 * q + 2], v[8 * q + 3]);
      w.z = pack2<BF16>(v[8 * q + 4], v[8 * q + 5]);
      w.w = pack2<BF16>(v[8 * q + 6], v[8 * q + 7]);
      reinterpret_cast<uint4*>(base)[q] = w;
    }
  } else {
    for (int j = 0; j < 32 && nc0 + j < p.N; ++j) {
      const uint32_t h = pack2<BF16>(v[j], 0.f);
      base[j] = static_cast<uint16_t>(h & 0xffffu);
    }
  }
}

template <int BN, int EPI, bool BF16>
__device__ __forceinline__ void epi_rows(const TileParams& p, uint32_t tbase, int row, int n0, const float* bs,
                                         float* cpw, const CUtensorMap* tmY, uint8_t* stg, uint32_t& scount,
                                         int wrow0, const CUtensorMap* tmAux, uint8_t* auxstg,
                                         const MaskWords<BN>& mw, int ncols = BN, bool aux_block = true,
                                         const float* addp = nullptr, int nadd = 0, int64_t add_stride = 0,
                                         bool add_smem = false) {
  const uint32_t lane = lane_id();
  const bool row_ok = row < p.T;
  constexpr bool kAuxTma = EPI == EPI_RELU_AUX_BIAS && AuxByTma<BN>::value;
  const bool aux_by_tma = kAuxTma && p.aux_tma && aux_block;  // a tile narrower than BN stores its words directly
  uint32_t auxw[kAuxTma ? BN / 32 : 1];
  if constexpr (kAuxTma) {
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) auxw[c] = 0u;
  }
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    const int nc0 = n0 + c * 32;
    if (nc0 >= p.N || c * 32 >= ncols) break;  // warp-uniform
    uint32_t r[32];
    tmem_ld_32x32b_x32(tbase + c * 32, r);
    tmem_wait_ld();
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    // stream-K: this thread's row of the other k-segments' fp32 partial
    // accumulators (written by other CTA pairs; in global memory, or brought
    // into shared memory), added in segment order. A partial is this warp's
    // 16 blocks of 32 rows x 16 columns (2 KB each, rows of 64 bytes whose
    // 16-byte chunks are XOR-swizzled like the output staging); `addp` is the
    // warp's first block of the first segment.
    for (int sg = 0; sg < nadd; ++sg) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float* blk = addp + sg * add_stride + (2 * c + h) * 512 + lane * 16;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4* src = reinterpret_cast<const float4*>(blk + ((q ^ ((lane >> 1) & 3u)) * 4));
          const float4 x = add_smem ? *src : __ldcg(src);
          v[16 * h + 4 * q] += x.x;
          v[16 * h + 4 * q + 1] += x.y;
          v[16 * h + 4 * q + 2] += x.z;
          v[16 * h + 4 * q + 3] += x.w;
        }
      }
    }
    if constexpr (EPI == EPI_DRELU_BGRAD) {
      const uint32_t m = mw.w[c];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = ((m >> j) & 1u) ? v[j] : 0.f;
    } else if constexpr (!PlainStore<EPI>::value) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += bs[c * 32 + j];
      // GELU_AUX_BIAS: the pre-activation Z goes out (16-bit) before GELU, this
      // thread's 32 columns as one 64-byte row segment written directly (the
      // staging buffers and TMA stores are Y's; sharing them doubles the
      // epilogue's store waits)
      if constexpr (EPI == EPI_GELU_AUX_BIAS) store_row16<BF16>(v, p, row, nc0);
      if constexpr (AppliesGelu<EPI>::value) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = gelu_erf(v[j]);
      }
      if constexpr (EPI == EPI_RELU_BIAS || EPI == EPI_RELU_AUX_BIAS) {
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const bool pos = v[j] > 0.f;
          m |= (pos ? 1u : 0u) << j;
          v[j] = pos ? v[j] : 0.f;
        }
        if constexpr (EPI == EPI_RELU_AUX_BIAS) {
          const int valid = p.N - nc0;
          if (valid < 32) m &= (1u << valid) - 1u;
          if (aux_by_tma)
            auxw[kAuxTma ? c : 0] = m;
          else if (row_ok)
            p.aux_out[static_cast<int64_t>(row) * p.aux_words + (nc0 >> 5)] = m;
        }
      }
    }
    if (p.out_f32) {
      // fp32 output: the chunk goes out as two 16-column blocks, whose 64-byte
      // rows are staged and stored exactly like the 16-bit blocks below (a
      // second block that would start at or past N is not stored)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h == 1 && nc0 + 16 >= p.N) break;  // warp-uniform
        uint8_t* buf = stg + (scount & 1u) * 2048;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        const uint32_t rbase = smem_u32(buf) + lane * 64;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(rbase + ((q ^ ((lane >> 1) & 3u)) * 16),
                       make_uint4(__float_as_uint(v[16 * h + 4 * q]), __float_as_uint(v[16 * h + 4 * q + 1]),
                                  __float_as_uint(v[16 * h + 4 * q + 2]), __float_as_uint(v[16 * h + 4 * q + 3])));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tmY, buf, nc0 + 16 * h, wrow0);
          bulk_commit_group();
        }
        ++scount;
      }
    } else {
      store_block16<BF16>(v, tmY, stg, scount, nc0, wrow0);
    }
    if constexpr (EPI == EPI_DRELU_BGRAD) {
      warp_transpose_reduce32(v);
      cpw[c * 32 + lane] = v[0];
    }
  }
  if (aux_by_tma) {
    // row `lane` of the warp's [32][BN/32] word block; the previous tile's
    // block was read by its store before any later chunk's wait returned
    constexpr int WB = BN / 32 * 4;  // bytes per row
    const uint32_t rb = smem_u32(auxstg) + lane * WB;
#pragma unroll
    for (int q = 0; q < WB / 16; ++q) st_shared_v4(rb + q * 16, make_uint4(auxw[4 * q], auxw[4 * q + 1], auxw[4 * q + 2], auxw[4 * q + 3]));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmAux, auxstg, n0 >> 5, wrow0);
      bulk_commit_group();
    }
  }
}

// DRELU_BGRAD: combine the four warps' column sums (rows in lane-quarter
// order) into the partial row `prow` of the workspace.
template <int BN>
__device__ __forceinline__ void epi_write_partials(const TileParams& p, int prow, int n0, const float* cp, uint32_t et,
                                                   int ncols = BN) {
  for (int c = et; c < ncols; c += 128) {
    const int n = n0 + c;
    if (n < p.N)
      p.partials[static_cast<int64_t>(prow) * p.N + n] = ((cp[0 * BN + c] + cp[1 * BN + c]) + cp[2 * BN + c]) + cp[3 * BN + c];
  }
}

// Column sums of the partial rows 0 .. m_tiles-1 for up to two columns na, nb
// (used where ua / ub), each in ascending row order, one row at a time -- the
// same order whichever tile runs it. The loads of 16 rows of both columns are
// issued together (32 L2 round trips in flight): issued one by one they were
// most of the finishing time at few row blocks.
__device__ __forceinline__ void sum_partials2(const TileParams& p, int na, bool ua, int nb, bool ub, float& sa,
                                              float& sb) {
  sa = 0.f;
  sb = 0.f;
  const float* ca = p.partials + na;
  const float* cb = p.partials + nb;
  for (int m0 = 0; m0 < p.m_tiles; m0 += 16) {
    float xa[16], xb[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const bool v = m0 + j < p.m_tiles;
      const int64_t off = static_cast<int64_t>(m0 + j) * p.N;
      xa[j] = (ua && v) ? __ldcg(ca + off) : 0.f;
      xb[j] = (ub && v) ? __ldcg(cb + off) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (m0 + j < p.m_tiles) {
        sa += xa[j];
        sb += xb[j];
      }
    }
  }
}

// DRELU_BGRAD, second pass inside the kernel: after its partial rows are
// written, a tile takes `rows` tickets on each of its `nblocks` column blocks
// of `ncols` columns (nb, nb + 1, ...; a whole CTA-pair tile spans two); for
// each block where it takes the last ticket it sums every partial row of the
// block in ascending row order -- the same order whichever tile is last --
// writes dbias and resets the counter for the next launch. Called by the 128
// epilogue threads, each taking columns et and et + 128 of the tile;
// `flag` is a shared-memory word.
template <int BN>
__device__ __forceinline__ void epi_finish_dbias(const TileParams& p, int nb, int n0, int rows, uint32_t et,
                                                 volatile int* flag, int ncols = BN, int nblocks = 1) {
  __threadfence();
  named_bar_sync(1, 128);
  if (et == 0) {
    int bits = 0;
    for (int b = 0; b < nblocks; ++b) {
      const int prev = atomicAdd(p.col_tickets + nb + b, rows);
      if (prev + rows == p.m_tiles) {
        p.col_tickets[nb + b] = 0;
        bits |= 1 << b;
      }
    }
    *flag = bits;
  }
  named_bar_sync(1, 128);
  const int bits = *flag;
  if (bits) {
    __threadfence();
    const int total = nblocks * ncols;
    const int ca = static_cast<int>(et), cb = static_cast<int>(et) + 128;
    const bool ua = ca < total && ((bits >> (ca / ncols)) & 1) && n0 + ca < p.N;
    const bool ub = cb < total && ((bits >> (cb / ncols)) & 1) && n0 + cb < p.N;
    if (ua || ub) {
      float sa, sb;
      sum_partials2(p, n0 + ca, ua, n0 + cb, ub, sa, sb);
      if (ua) p.dbias[n0 + ca] = sa;
      if (ub) p.dbias[n0 + cb] = sb;
    }
  }
  named_bar_sync(1, 128);  // the flag word is reused by the next tile
}

// BK: the weight is N x K (K contiguous) and B is staged K-major; a template
// parameter, not a runtime flag -- a branch on it in the producer and MMA
// loops cost 3-4 % on the FFN shape (their issue path is latency-critical)
template <int BN, int STAGES, int EPI, bool BF16, bool BK = false>
__global__ void __launch_bounds__(kThreads, 1)
    tile_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmAux,
                const TileParams p) {
  using L = TileSmem<BN, STAGES>;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be 64, 128, 192 or 256");
  constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                 : (2 * BN <= 256) ? 256 : 512;
  constexpr bool A_MN = AOperandMN<EPI>::value;
  constexpr uint32_t IDESC = idesc_f16(BF16, /*A MN-major*/ A_MN, /*B MN-major*/ true, kBM, BN);
  constexpr uint32_t IDESC_BK = idesc_f16(BF16, A_MN, /*B MN-major*/ false, kBM, BN);
  constexpr uint32_t STAGE_TX = L::A_BYTES + L::B_BYTES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + L::OFF_A;
  uint8_t* sB = smem + L::OFF_B;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  float* bias_s = reinterpret_cast<float*>(smem + L::OFF_BIAS);  // [2][BN]
  float* colp_s = reinterpret_cast<float*>(smem + L::OFF_COLP);  // [2][4][BN]
  uint8_t* stg_s = smem + L::OFF_STG;                             // [4 warps][2][2 KB]
  uint8_t* auxstg_s = smem + L::OFF_AUXSTG;                       // [4 warps][1 KB]
  volatile int* dflag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);

  const uint32_t warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p.m_tiles, p.n_tiles, p.group_m, p.raster_n, mb, nb);
        const int m0 = mb * kBM, n0 = nb * BN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&empty[s], ph ^ 1u, p, abort_flag, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], STAGE_TX);
          if constexpr (A_MN) {
            tma_load_2d(sA + s * L::A_BYTES, &tmA, &full[s], m0, kb * kBK);
            tma_load_2d(sA + s * L::A_BYTES + kAChunkMN, &tmA, &full[s], m0 + 64, kb * kBK);
          } else {
            tma_load_2d(sA + s * L::A_BYTES, &tmA, &full[s], kb * kBK, m0);
          }
          if constexpr (BK) {
            tma_load_2d(sB + s * L::B_BYTES, &tmB, &full[s], kb * kBK, n0);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(sB + s * L::B_BYTES + j * L::B_CHUNK, &tmB, &full[s], n0 + j * 64, kb * kBK);
          }
        }
      }
      // let every issued copy land before the CTA can exit
      const uint32_t inflight = it < STAGES ? it : STAGES;
      for (uint32_t i = it - inflight; i < it; ++i)
        wait_bounded(&full[i % STAGES], (i / STAGES) & 1u, p, abort_flag, 2, /*honour_abort=*/false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      constexpr uint32_t idesc = BK ? IDESC_BK : IDESC;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1u;
        const uint32_t tph = (tcount >> 1) & 1u;
        if (!wait_bounded(&tempty[buf], tph ^ 1u, p, abort_flag, 3)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&full[s], ph, p, abort_flag, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * L::A_BYTES);
          const uint32_t b0 = smem_u32(sB + s * L::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t adesc = a_desc<A_MN>(a0, kk);
            const uint64_t bdesc = b_desc(b0, kk, BK, L::B_CHUNK);
            umma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        // (fault injection: the epilogue then waits on a barrier nothing arrives on)
        if (!(p.inject_stall && tcount == 0)) umma_commit(&tfull[buf]);
      }
      // every MMA issued above must finish before tensor memory is freed
      umma_commit(drain);
      wait_bounded(drain, 0, p, abort_flag, 5, /*honour_abort=*/false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t ew = warp & 3u;        // TMEM lane quarter this warp may access
    const uint32_t et = threadIdx.x - 64;  // 0..127
    uint8_t* stg = stg_s + ew * kStageBytesPerWarp;
    uint32_t scount = 0;
    uint32_t tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, p.group_m, p.raster_n, mb, nb);
      const int m0 = mb * kBM, n0 = nb * BN;
      const uint32_t buf = tcount & 1u;
      const uint32_t tph = (tcount >> 1) & 1u;
      float* bs = bias_s + buf * BN;
      float* cp = colp_s + buf * 4 * BN;
      epi_stage_bias<BN, EPI, BF16>(p, n0, bs, et);
      MaskWords<BN> mw{};
      if constexpr (EPI == EPI_DRELU_BGRAD) mw = load_mask_words<BN>(p, m0 + static_cast<int>(ew * 32 + lane), n0);
      named_bar_sync(1, 128);
      if (ok) ok = wait_bounded(&tfull[buf], tph, p, abort_flag, 6);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        epi_rows<BN, EPI, BF16>(p, tmem_base + ((ew * 32u) << 16) + buf * BN, m0 + static_cast<int>(ew * 32 + lane), n0,
                                bs, cp + ew * BN, &tmY, stg, scount, m0 + static_cast<int>(ew * 32), &tmAux,
                                auxstg_s + ew * kAuxStageBytesPerWarp, mw);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
      }
      if constexpr (EPI == EPI_DRELU_BGRAD) {
        named_bar_sync(1, 128);
        if (ok) epi_write_partials<BN>(p, mb, n0, cp, et);
        if (p.col_tickets) epi_finish_dbias<BN>(p, nb, n0, ok ? 1 : 0, et, dflag);
      }
    }
    if (lane == 0) bulk_wait_group_all();  // this warp's output stores are complete
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace ge
