// tile2_kernel.cuh -- the CTA-pair (cluster of 2, tcgen05 cta_group::2)
// variant of the persistent tile kernel, for large problems.
//
// A pair computes a 256 x BN output tile with one MMA stream: the leader CTA
// (rank 0) issues tcgen05.mma.cta_group::2 with M = 256, reading rows 0..127
// of the X tile and columns 0..BN/2-1 of the W tile from its own shared
// memory and rows 128..255 / columns BN/2..BN-1 from its peer's (same
// offsets); each CTA's TMEM receives its 128 rows of the accumulator, all BN
// columns. Per CTA and k-block that is 16 KB of X and BN/2 x 64 of W instead
// of the single-CTA kernel's 16 KB + BN x 64, so each SM needs two thirds of
// the operand traffic per FLOP and the ring can be deeper.
//
// Synchronisation across the pair:
//   full[s]   (leader's) one arrival -- the leader's expect_tx for both CTAs'
//             bytes -- plus both CTAs' TMA transaction bytes (the peer's loads
//             name the leader's barrier)
//   empty[s]  (each CTA's) one arrival from the leader's MMA commit,
//             multicast to both CTAs
//   tfull[b]  (each CTA's) the leader's commit after a tile, multicast
//   tempty[b] (leader's) one arrival per epilogue warp of each CTA (4 or 8),
//             the peer's through its shared::cluster address
// No load uses TMA multicast. Every wait is bounded as in the 1-CTA kernel.
//
// Tail split: when the tiles left for the last round fill at most half of
// the pairs, each of them is processed as two 128-column halves (MMA N =
// 128), so the last round takes half a tile's time instead of a whole one.
//
// Stream-K (SPLIT): the tiles that would leave the last round of whole
// tiles partly idle (between one and two waves of them; all tiles when there
// are fewer tiles than pairs) are cut into one contiguous k-range per pair,
// so every pair does the same share of the MMAs. A tile covered by several
// pairs has one segment per pair; segment 0 (the one that starts at k-block
// 0) finishes the tile. The others write their fp32 accumulator (each CTA
// its 128 rows) to a workspace slot and count themselves on the tile's flag;
// segment 0 waits (bounded) until all are in, adds them to its own in
// segment order (so the sum is the same on every run) and runs the epilogue.
// Only segment 0 waits, and it waits only on segments that never wait, and
// every pair is resident (one CTA per SM), so the waits always end. By
// default the stream-K tiles come before the whole tiles, so that the fixups
// overlap later MMAs instead of ending the kernel.
#pragma once

#include "tile_kernel.cuh"

namespace ge {

// Epilogue warps of the pair kernel: one per TMEM lane quarter, or two for
// the GELU epilogs (each with half of a tile's columns). A warp reaches only
// its own quarter of the TMEM lanes, so the four quarters sit on the four
// SM sub-partitions, one warp each; with one warp per sub-partition a GELU
// epilogue (erff per element, a chain of dependent operations) ran about
// five times longer than a ReLU one and bounded the launch, and a second
// warp per sub-partition overlaps two such chains. Stream-K instances keep
// four (their partial slots are laid out per quarter).
template <int EPI, bool SPLIT>
struct PairEpiWarps {
  static constexpr int value = AppliesGelu<EPI>::value && !SPLIT ? 8 : 4;
};

template <int BN, int STAGES, int EW = 4>
struct Tile2Smem {
  static constexpr uint32_t A_BYTES = kBM * kBK * 2;          // this CTA's 128 rows x 64 k
  static constexpr uint32_t B_CHUNK = kBK * 64 * 2;           // 64 k x 64 n
  static constexpr uint32_t B_BYTES = (BN / 128) * B_CHUNK;   // this CTA's BN/2 columns
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_B + STAGES * B_BYTES;
  static constexpr uint32_t N_BARS = 2 * STAGES + 6;  // full, empty, tfull[2], tempty[2], drain, stream-K fixup
  static constexpr uint32_t OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr uint32_t OFF_BIAS = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr uint32_t OFF_COLP = OFF_BIAS + 2 * BN * 4;
  static constexpr uint32_t OFF_STG = (OFF_COLP + 2 * 4 * BN * 4 + 1023) / 1024 * 1024;
  static constexpr uint32_t OFF_AUXSTG = OFF_STG + kStageBytesPerWarp * EW;
  static constexpr uint32_t END = OFF_AUXSTG + kAuxStageBytesPerWarp * EW;
  static constexpr uint32_t BYTES = END + 1024;
};

// Work unit u of the pair schedule: a whole tile, or (in the split tail) one
// column half of a tile; under stream-K, one k-range of a tile.
struct PairUnit {
  int mb, nb;
  int half;          // -1 for a whole tile, else 0 or 1
  int kb0, kb1;      // k-blocks [kb0, kb1)
  int tile, seg, nsegs;  // stream-K: the tile's index, this pair's segment of it, their count
};

// largest pair whose stream-K range starts at or before k-block x
__device__ __host__ __forceinline__ int64_t pair_owner(int64_t x, int64_t npairs, int64_t total) {
  return ((x + 1) * npairs - 1) / total;
}

struct PairSchedule {
  int num_tiles, full_units, num_units;
  __device__ __forceinline__ PairSchedule(int tiles, int npairs, bool allow_split) {
    num_tiles = tiles;
    const int tail = tiles % npairs;
    const bool split = allow_split && tail > 0 && 2 * tail <= npairs;
    full_units = split ? tiles - tail : tiles;
    num_units = split ? tiles + tail : tiles;
  }
  __device__ __forceinline__ PairUnit unit(int u, int m2_tiles, int n_tiles, int group, int by_n) const {
    PairUnit r;
    int t = u;
    r.half = -1;
    if (u >= full_units) {
      t = full_units + (u - full_units) / 2;
      r.half = (u - full_units) & 1;
    }
    tile_coords(t, m2_tiles, n_tiles, group, by_n, r.mb, r.nb);
    r.tile = t;
    r.seg = 0;
    r.nsegs = 1;
    return r;
  }
};

// Stream-K part of a split schedule: with at least two waves of tiles,
// rounds - 1 waves stay whole tiles, one per pair as without the split, and
// only the rest (between one and two waves of tiles) is cut into equal
// k-ranges, so every range spans at least one tile's k-blocks and a tile has
// at most two segments; with fewer tiles every tile is cut.
__device__ __host__ __forceinline__ int pair_dp_rounds(int tiles, int npairs) {
  const int rounds = tiles / npairs;
  return rounds >= 2 ? rounds - 1 : 0;
}

// The sequence of units of one pair. Without SPLIT: units pair, pair +
// npairs, ... of the schedule, each over every k-block. With SPLIT: the
// pieces of the pair's contiguous range [lo, hi) of the flattened (tile,
// k-block) space of the stream-K tiles, tile by tile, and the pair's whole
// tiles of the data-parallel rounds. With sk_first the stream-K pieces come
// first (they are the first sk_tiles tiles of the raster order): a tile's
// fixup then runs in an epilogue that the next whole tile's MMAs overlap,
// and every pair ends on a whole tile. Otherwise the whole tiles come first
// and the stream-K tiles are the last ones.
template <bool SPLIT>
struct PairWork {
  PairSchedule sched;
  int pair, npairs, m2_tiles, n_tiles, group, by_n, k_blocks;
  int dp_units, dp_tiles, sk_tiles, dp_done;  // SPLIT: the data-parallel rounds' whole tiles
  bool sk_first;
  int64_t total, lo, hi, cur;
  __device__ __forceinline__ PairWork(const TileParams& p, int pair_, int npairs_, int m2)
      : sched(m2 * p.n_tiles, npairs_, !SPLIT && p.tail_split != 0),
        pair(pair_), npairs(npairs_), m2_tiles(m2), n_tiles(p.n_tiles), group(p.group_m), by_n(p.raster_n),
        k_blocks(p.k_blocks) {
    if constexpr (SPLIT) {
      const int tiles = m2 * p.n_tiles;
      dp_units = pair_dp_rounds(tiles, npairs);
      dp_tiles = dp_units * npairs;
      sk_tiles = tiles - dp_tiles;
      dp_done = 0;
      sk_first = p.sk_first != 0;
      total = static_cast<int64_t>(sk_tiles) * p.k_blocks;
      lo = static_cast<int64_t>(pair) * total / npairs;
      hi = static_cast<int64_t>(pair + 1) * total / npairs;
      cur = 0;
    } else {
      cur = pair;
      hi = sched.num_units;
    }
  }
  // this is the pair's last unit (after next() returned it)
  __device__ __forceinline__ bool done() const {
    return SPLIT ? (lo + cur >= hi && dp_done >= dp_units) : cur >= hi;
  }
  __device__ __forceinline__ bool next(PairUnit& w) {
    if constexpr (SPLIT) {
      const bool sk_left = lo + cur < hi;
      if (dp_done < dp_units && !(sk_first && sk_left)) {  // a whole tile of the data-parallel rounds
        const int t = (sk_first ? sk_tiles : 0) + pair + dp_done * npairs;
        tile_coords(t, m2_tiles, n_tiles, group, by_n, w.mb, w.nb);
        w.half = -1;
        w.kb0 = 0;
        w.kb1 = k_blocks;
        w.tile = t;
        w.seg = 0;
        w.nsegs = 1;
        ++dp_done;
        return true;
      }
      if (!sk_left) return false;
      const int64_t g = lo + cur;  // stream-K index
      const int tl = static_cast<int>(g / k_blocks);  // tile among the stream-K tiles
      const int64_t tb = static_cast<int64_t>(tl) * k_blocks;
      const int64_t end = hi < tb + k_blocks ? hi : tb + k_blocks;
      const int t = (sk_first ? 0 : dp_tiles) + tl;
      tile_coords(t, m2_tiles, n_tiles, group, by_n, w.mb, w.nb);
      w.half = -1;
      w.kb0 = static_cast<int>(g - tb);
      w.kb1 = static_cast<int>(end - tb);
      w.tile = t;
      const int64_t first = pair_owner(tb, npairs, total);
      w.nsegs = static_cast<int>(pair_owner(tb + k_blocks - 1, npairs, total) - first + 1);
      w.seg = static_cast<int>(pair - first);
      cur = end - lo;
      return true;
    } else {
      if (cur >= hi) return false;
      w = sched.unit(static_cast<int>(cur), m2_tiles, n_tiles, group, by_n);
      w.kb0 = 0;
      w.kb1 = k_blocks;
      cur += npairs;
      return true;
    }
  }
};

template <int BN, int STAGES, int EPI, bool BF16, bool BK = false, bool SPLIT = false>
__global__ void __launch_bounds__(64 + 32 * PairEpiWarps<EPI, SPLIT>::value, 1)
    tile2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmAux,
                 const TileParams p) {
  constexpr int EW = PairEpiWarps<EPI, SPLIT>::value;  // epilogue warps
  constexpr int ET = 32 * EW;                          // epilogue threads
  using L = Tile2Smem<BN, STAGES, EW>;
  static_assert(BN == 128 || BN == 256, "the pair kernel splits BN in 64-column chunks per CTA");
  constexpr uint32_t TMEM_COLS = 2 * BN;
  static_assert(BN == 256, "the tail split halves 256-column tiles");
  constexpr bool A_MN = AOperandMN<EPI>::value;
  constexpr uint32_t IDESC = idesc_f16(BF16, /*A MN-major*/ A_MN, /*B MN-major*/ true, 2 * kBM, BN);
  constexpr uint32_t IDESC_HALF = idesc_f16(BF16, A_MN, true, 2 * kBM, BN / 2);
  constexpr uint32_t IDESC_BK = idesc_f16(BF16, A_MN, /*B MN-major*/ false, 2 * kBM, BN);
  constexpr uint32_t PAIR_TX = 2 * (L::A_BYTES + L::B_BYTES);
  constexpr uint32_t PAIR_TX_HALF = 2 * (L::A_BYTES + L::B_CHUNK);
  constexpr uint16_t BOTH = 0x3;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + L::OFF_A;
  uint8_t* sB = smem + L::OFF_B;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* fixbar = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  float* bias_s = reinterpret_cast<float*>(smem + L::OFF_BIAS);  // [2][BN]
  float* colp_s = reinterpret_cast<float*>(smem + L::OFF_COLP);  // [2][4][BN]
  uint8_t* stg_s = smem + L::OFF_STG;                             // [EW warps][2][2 KB]
  uint8_t* auxstg_s = smem + L::OFF_AUXSTG;                       // [EW warps][1 KB]
  volatile int* dflag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);
  volatile int* sflag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 12);  // stream-K wait result

  const uint32_t warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * EW);
    }
    mbar_init(drain, 1);
    mbar_init(fixbar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before either side signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int m2_tiles = (p.m_tiles + 1) / 2;  // 256-row tiles
  // half units would need a 64-row box of a K-major W: with BK every unit is a whole tile
  TileParams pw = p;
  if constexpr (BK) pw.tail_split = 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
      PairWork<SPLIT> work(pw, pair, npairs, m2_tiles);
      PairUnit w;
      while (ok && work.next(w)) {
        const int m0 = w.mb * 2 * kBM + static_cast<int>(rank) * kBM;
        // this CTA's columns: half of the tile (two 64-wide chunks), or half of a half (one chunk)
        const int nchunks = w.half < 0 ? BN / 128 : 1;
        const int nh0 = w.nb * BN + (w.half < 0 ? 0 : w.half * (BN / 2)) + static_cast<int>(rank) * nchunks * 64;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&empty[s], ph ^ 1u, p, abort_flag, 1)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], w.half < 0 ? PAIR_TX : PAIR_TX_HALF);
          const uint32_t fbar = full0 + s * 8;  // the leader's full[s]
          if constexpr (A_MN) {
            tma_load_2d_pair(sA + s * L::A_BYTES, &tmA, fbar, m0, kb * kBK);
            tma_load_2d_pair(sA + s * L::A_BYTES + kAChunkMN, &tmA, fbar, m0 + 64, kb * kBK);
          } else {
            tma_load_2d_pair(sA + s * L::A_BYTES, &tmA, fbar, kb * kBK, m0);
          }
          if constexpr (BK) {  // this CTA's 128 rows of the N x K weight in one box
            tma_load_2d_pair(sB + s * L::B_BYTES, &tmB, fbar, kb * kBK, nh0);
          } else {
            for (int j = 0; j < nchunks; ++j)
              tma_load_2d_pair(sB + s * L::B_BYTES + j * L::B_CHUNK, &tmB, fbar, nh0 + j * 64, kb * kBK);
          }
        }
      }
      // the last fills have landed once the MMA has released them
      const uint32_t inflight = it < STAGES ? it : STAGES;
      for (uint32_t i = it - inflight; i < it; ++i)
        wait_bounded(&empty[i % STAGES], ((i / STAGES) & 1u), p, abort_flag, 2, /*honour_abort=*/false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      if (rank == 0) {
        uint32_t it = 0, tcount = 0;
        bool ok = true;
        PairWork<SPLIT> work(pw, pair, npairs, m2_tiles);
        PairUnit w;
        for (; ok && work.next(w); ++tcount) {
          const uint32_t idesc = BK ? IDESC_BK : w.half < 0 ? IDESC : IDESC_HALF;
          const uint32_t buf = tcount & 1u;
          const uint32_t tph = (tcount >> 1) & 1u;
          if (!wait_bounded(&tempty[buf], tph ^ 1u, p, abort_flag, 3)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + buf * BN;
          for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
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
              umma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb > w.kb0 || kk != 0) ? 1u : 0u);
            }
            umma_commit_pair(&empty[s], BOTH);
          }
          if (!ok) break;
          // (fault injection: both CTAs' epilogues then wait on a barrier nothing arrives on)
          if (!(p.inject_stall && tcount == 0)) umma_commit_pair(&tfull[buf], BOTH);
        }
        umma_commit_pair(drain, BOTH);
      }
      // both CTAs: the leader's MMAs write this CTA's TMEM; they must be done
      wait_bounded(drain, 0, p, abort_flag, 5, /*honour_abort=*/false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t ew = warp & 3u;             // TMEM lane quarter
    const uint32_t eh = (warp - 2u) >> 2;      // column half (EW == 8), else 0
    const uint32_t et = threadIdx.x - 64;      // 0 .. ET - 1
    uint8_t* stg = stg_s + (warp - 2u) * kStageBytesPerWarp;
    uint32_t scount = 0;
    uint32_t tcount = 0;
    bool ok = true;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    PairWork<SPLIT> work(pw, pair, npairs, m2_tiles);
    PairUnit w;
    for (; work.next(w); ++tcount) {
      const int prow = w.mb * 2 + static_cast<int>(rank);  // this CTA's 128-row block
      const int m0 = prow * kBM;
      const int n0 = w.nb * BN + (w.half < 0 ? 0 : w.half * (BN / 2));
      const int ncols = w.half < 0 ? BN : BN / 2;
      const uint32_t buf = tcount & 1u;
      const uint32_t tph = (tcount >> 1) & 1u;
      float* bs = bias_s + buf * BN;
      float* cp = colp_s + buf * 4 * BN;
      epi_stage_bias<BN, EPI, BF16, ET>(p, n0, bs, et, ncols);
      MaskWords<BN> mw{};
      if constexpr (EPI == EPI_DRELU_BGRAD) mw = load_mask_words<BN>(p, m0 + static_cast<int>(ew * 32 + lane), n0);
      named_bar_sync(1, ET);
      if (ok) ok = wait_bounded(&tfull[buf], tph, p, abort_flag, 6);
      ok = __all_sync(0xffffffffu, ok);
      const uint32_t trow = tmem_base + ((ew * 32u) << 16) + buf * BN;
      const int r = static_cast<int>(ew * 32 + lane);  // this thread's row of the CTA's 128
      // stream-K slots, one per pair and CTA: a pair's only later segment is
      // its first stream-K piece, so segment s of the tile that pair `pair` finishes
      // is in pair (pair + s)'s slot; the flag of a tile is its finisher's
      const int64_t slot_stride = 2 * kBM * BN;
      float* own_slot = SPLIT ? p.sk_slots + (static_cast<int64_t>(pair) * 2 + rank) * (kBM * BN) : nullptr;
      if (SPLIT && w.seg > 0) {
        // a later segment: hand the fp32 accumulator to segment 0 and count it
        // in. Each warp stages its rows as 2 KB blocks of 32 rows x 16 columns
        // (the swizzled layout of the output staging) and writes each block
        // with one bulk copy into its 32 KB of the slot.
        if (ok) {
          tc_fence_after();
          float* dst = own_slot + ew * (16 * 512);
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(trow + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint8_t* sbuf = stg + (scount & 1u) * 2048;
              if (lane == 0) bulk_wait_group_read<1>();
              __syncwarp();
              const uint32_t rbase = smem_u32(sbuf) + lane * 64;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                st_shared_v4(rbase + ((q ^ ((lane >> 1) & 3u)) * 16),
                             make_uint4(v[16 * h + 4 * q], v[16 * h + 4 * q + 1], v[16 * h + 4 * q + 2],
                                        v[16 * h + 4 * q + 3]));
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                bulk_store_s2g(dst + (2 * c + h) * 512, sbuf, 2048);
                bulk_commit_group();
              }
              ++scount;
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty0 + buf * 8);
          if (lane == 0) {
            bulk_wait_group_all();  // the partial is in global memory
            fence_proxy_async_global();
          }
          __syncwarp();
        }
        __threadfence();
        named_bar_sync(1, ET);
        if (et == 0 && ok) atomicAdd(p.sk_flags + (pair - w.seg) * 2 + rank, 1);
        continue;
      }
      int nadd = 0;
      const float* addp = nullptr;
      bool add_smem = false;
      if (SPLIT && w.nsegs > 1) {
        // segment 0: wait until the other segments' partials are in (bounded)
        int* flag = p.sk_flags + pair * 2 + rank;
        // the pair's last unit with one other segment (stream-K tiles last,
        // or no whole tiles): its operand stages are idle (the MMAs that read
        // them are complete), so that segment's 128 KB comes in with bulk
        // copies and is added from shared memory; otherwise the epilogue
        // reads it from global memory while the next tile's MMAs run
        const bool bulk = w.nsegs == 2 && work.done();
        if (et == 0) {
          int got = ok ? 1 : 0;
          if (got) {
            const uint64_t t0 = globaltimer_ns();
            while (*reinterpret_cast<volatile int*>(flag) < w.nsegs - 1) {
              __nanosleep(100);
              if (*abort_flag || globaltimer_ns() - t0 > p.timeout_ns) {
                report_timeout(p.status, abort_flag, 7);
                got = 0;
                break;
              }
            }
            if (got) *flag = 0;  // ready for the next launch
          }
          __threadfence();
          if (got && bulk) {
            fence_proxy_async_global();  // the bulk copies below read what the flag announced
            constexpr uint32_t kPart = kBM * BN * 4, kPiece = 32768;
            const float* src = own_slot + slot_stride;  // pair + 1's slot
            mbar_arrive_expect_tx(fixbar, kPart);
            for (uint32_t off = 0; off < kPart; off += kPiece)
              bulk_load_g2s(smem + off, reinterpret_cast<const uint8_t*>(src) + off, kPiece, fixbar);
          }
          *sflag = got;
        }
        named_bar_sync(1, ET);
        ok = ok && *sflag != 0;
        if (ok && bulk) ok = wait_bounded(fixbar, 0, p, abort_flag, 8);
        ok = __all_sync(0xffffffffu, ok);
        nadd = w.nsegs - 1;
        addp = bulk ? reinterpret_cast<const float*>(smem) + ew * (16 * 512) : own_slot + slot_stride + ew * (16 * 512);
        add_smem = bulk;
      }
      if (ok) {
        tc_fence_after();
        if constexpr (EW == 8) {
          // this warp's half of the columns (the GELU epilogs: no mask words,
          // no column sums, no stream-K addends)
          const int hc = ncols / 2, c0 = static_cast<int>(eh) * hc;
          epi_rows<BN, EPI, BF16>(p, trow + c0, m0 + r, n0 + c0, bs + c0, nullptr, &tmY, stg, scount,
                                  m0 + static_cast<int>(ew * 32), &tmAux, nullptr, mw, hc, false);
        } else {
          epi_rows<BN, EPI, BF16>(p, trow, m0 + r, n0, bs, cp + ew * BN, &tmY, stg, scount,
                                  m0 + static_cast<int>(ew * 32), &tmAux, auxstg_s + ew * kAuxStageBytesPerWarp, mw,
                                  ncols, w.half < 0, addp, nadd, slot_stride, add_smem);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty0 + buf * 8);
      }
      if constexpr (EPI == EPI_DRELU_BGRAD) {
        named_bar_sync(1, ET);
        const bool has_row = prow < p.m_tiles;
        if (ok && has_row) epi_write_partials<BN>(p, prow, n0, cp, et, ncols);
        // tickets count per 128-column half block, so whole tiles and tail halves mix
        if (p.col_tickets) {
          const int rows = (ok && has_row) ? 1 : 0;
          if (w.half < 0)
            epi_finish_dbias<BN>(p, 2 * w.nb, n0, rows, et, dflag, BN / 2, 2);
          else
            epi_finish_dbias<BN>(p, 2 * w.nb + w.half, n0, rows, et, dflag, BN / 2);
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();  // this warp's output stores are complete
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the other may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

}  // namespace ge
