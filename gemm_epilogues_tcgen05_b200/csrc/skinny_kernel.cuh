// skinny_kernel.cuh -- the few-row case (T <= 256) of the fused linear-layer
// GEMM + epilogue: there the weight W (K x N) is the only large operand, and
// the kernel's job is to stream it from HBM once at full bandwidth.
//
// Swap-AB: the MMA computes D^T[n][t] = sum_k W[k][n] * X[t][k], with 128
// features n in the MMA's M slot (A = W^T, read N-major straight from W's
// row-major layout) and the T rows, padded to TP (a power of two >= 16), in
// its N slot (B = X, K-major). The accumulator has one TMEM lane per feature
// and one column per row t, so in the epilogue each thread owns one feature:
// the bias is a per-thread constant, the mask word of 32 consecutive features
// is one __ballot_sync per row, and the bias gradient is a per-thread sum
// over t.
//
// Work split (stream-K): the (feature tile, k-block) space is flattened and
// cut into `grid` contiguous ranges, one per persistent CTA, so every SM
// streams the same share of W. A tile covered by one range is finished
// directly; a tile shared by several CTAs ("segments") has each segment write
// its fp32 partial to the workspace and take a ticket, and the CTA that takes
// the last ticket sums the segments in segment order (fixed, so results are
// reproducible) and runs the epilogue. Nobody waits for another CTA.
#pragma once

#include "tile_kernel.cuh"

namespace ge {

struct SkinnyParams {
  int32_t T, N, K;
  int32_t n_tiles, kbt, total_kb;  // 128-feature tiles, stages of 64·KPS k per tile, n_tiles * kbt
  int32_t aux_words;
  int32_t max_segs;                // workspace slots per tile
  int32_t prefetch;                // k-blocks of W prefetched into L2 ahead of the ring (0 = none)
  const void* bias;
  void* out;                       // Y or dZ, T x N
  uint32_t* aux_out;               // RELU_AUX_BIAS mask words; GELU_AUX_BIAS: T x N 16-bit Z
  const uint32_t* aux_in;
  float* dbias;
  float* partials;                 // [n_tiles][max_segs][TP][128] fp32
  int* tickets;                    // [n_tiles], zero between launches
  int* status;
  uint64_t timeout_ns;
  int32_t bias_f32;                // the bias is N fp32 values (else the 16-bit type)
  int32_t out_f32;                 // the output is fp32 (else the 16-bit type)
  int32_t cache_hints;             // W streamed once: evict_first; X read by every CTA: evict_last
  int32_t inject_stall;            // fault injection for tests: withhold the first segment's tfull commit
};

// A stage holds KPS consecutive 64-deep k-blocks: W as one box of 64 features
// x 64·KPS k-rows per 64-feature chunk, X as KPS boxes of TP rows x 64 k.
// Stages of 32 KB or more kept one SM's TMA stream up to 1.5x faster than
// 16 KB stages with the same bytes in flight (a load-only stream of W, 4096 x
// 11008, over 86 CTAs).
template <int TP, int KPS>
struct SkinnySmem {
  static constexpr int BK = kBK * KPS;                 // k per stage
  static constexpr uint32_t A_CHUNK = 64 * BK * 2;     // one 64-feature chunk x BK k-rows
  static constexpr uint32_t A_BYTES = 2 * A_CHUNK;     // 128 features
  static constexpr uint32_t A_SUB = 64 * kBK * 2;      // 64 k-rows of one chunk (8 KB)
  static constexpr uint32_t B_SUB = TP * kBK * 2;      // TP rows x 128 B (one 64-k block of X)
  static constexpr uint32_t B_BYTES = KPS * B_SUB;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (230400 / STAGE) > 12 ? 12 : (230400 / STAGE);
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_B + STAGES * B_BYTES;
  static constexpr uint32_t N_BARS = 2 * STAGES + 5;
  static constexpr uint32_t OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem slot, abort flag, last flag
  static constexpr uint32_t END = OFF_MISC + 16;
  static constexpr uint32_t BYTES = END + 1024;
  static_assert(STAGES >= 2, "few-row stage too large");
  static_assert(BYTES <= 232448, "few-row shared memory above the per-CTA limit");
};

// largest CTA index whose range starts at or before k-block x
__device__ __host__ __forceinline__ int64_t skinny_owner(int64_t x, int64_t grid, int64_t total) {
  return ((x + 1) * grid - 1) / total;
}

// The same in 32-bit arithmetic, for the kernel: the plan keeps (k-blocks + 1)
// x grid below 2^31. (64-bit divisions in the range and segment arithmetic
// sit between the kernel's start and its first load.)
__device__ __forceinline__ uint32_t skinny_owner32(uint32_t x, uint32_t grid, uint32_t total) {
  return ((x + 1u) * grid - 1u) / total;
}

struct Segment {
  int tile, kb0, kb1;  // k-blocks [kb0, kb1) of the tile, local to it
  int seg, nsegs;      // index among the CTAs sharing the tile, and their count
};

// The next segment of this CTA's k-block range [g, hi), or false when there
// are no more.
__device__ __forceinline__ bool skinny_segment(const SkinnyParams& p, uint32_t hi, uint32_t& g, Segment& s) {
  if (g >= hi) return false;
  const uint32_t kbt = static_cast<uint32_t>(p.kbt), total = static_cast<uint32_t>(p.total_kb);
  const uint32_t tile = g / kbt;
  const uint32_t tbeg = tile * kbt;
  const uint32_t tend = tbeg + kbt;
  const uint32_t end = hi < tend ? hi : tend;
  s.tile = static_cast<int>(tile);
  s.kb0 = static_cast<int>(g - tbeg);
  s.kb1 = static_cast<int>(end - tbeg);
  const uint32_t first = skinny_owner32(tbeg, gridDim.x, total);
  const uint32_t last = skinny_owner32(tend - 1u, gridDim.x, total);
  s.nsegs = static_cast<int>(last - first + 1u);
  s.seg = static_cast<int>(blockIdx.x - first);
  g = end;
  return true;
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

template <bool BF16>
__device__ __forceinline__ void store_16(void* base, int64_t i, float v) {
  if constexpr (BF16)
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<__half*>(base)[i] = __float2half_rn(v);
}

// the output element i: fp32 or rounded to the 16-bit type, chosen by OUTM
// (0: 16-bit, 1: fp32, 2: the plan's out_f32 flag at run time)
template <bool BF16, int OUTM>
__device__ __forceinline__ void store_out(const SkinnyParams& p, int64_t i, float v) {
  const bool f32 = OUTM == 2 ? p.out_f32 != 0 : OUTM == 1;
  if (f32)
    reinterpret_cast<float*>(p.out)[i] = v;
  else
    store_16<BF16>(p.out, i, v);
}

// DRELU_BGRAD: the mask words of rows t0 .. t0+15 for this warp's 32
// features (one word per row), held by every lane. A whole tile's words are
// all loaded before the accumulator wait and handed out 16 rows at a time by
// shuffles; the split-tile fixup loads a batch's words before it reads the
// partials, so the loads are in flight together.
struct Mask16 {
  uint32_t m[16];
};

__device__ __forceinline__ Mask16 skinny_mask16(const SkinnyParams& p, int t0, int word) {
  Mask16 r;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int t = t0 + j;
    r.m[j] = (t < p.T && word < p.aux_words) ? __ldg(p.aux_in + static_cast<int64_t>(t) * p.aux_words + word) : 0u;
  }
  return r;
}

// Epilogue of 16 rows t = t0 .. t0+15 of one feature n (this thread). With
// FULL the caller guarantees that all 16 rows are below T and that every lane
// of the warp has a feature below N, so the stores go out without a
// per-element check: a check around each store (a divergent branch and its
// reconvergence) made 16 rows of the few-row epilogue take 0.65 instead of
// 0.40 us, measured with %globaltimer stamps in an instrumented copy.
template <int EPI, bool BF16, int OUTM, bool FULL>
__device__ __forceinline__ void skinny_finish16_rows(const SkinnyParams& p, float (&v)[16], int t0, int n, bool n_ok,
                                                     int word, float bias_n, float& dbias_acc, const Mask16& mk) {
  const uint32_t lane = lane_id();
  if constexpr (EPI == EPI_DRELU_BGRAD) {
    const uint32_t* m = mk.m;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = t0 + j;
      if (FULL || t < p.T) {
        const float dz = ((m[j] >> lane) & 1u) ? v[j] : 0.f;
        if (FULL || n_ok) store_out<BF16, OUTM>(p, static_cast<int64_t>(t) * p.N + n, dz);
        dbias_acc += dz;
      }
    }
  } else {
    uint32_t myword = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float z = v[j] + bias_n;
      const int t = t0 + j;
      const bool ok = FULL || (t < p.T && n_ok);
      if constexpr (EPI == EPI_GELU_AUX_BIAS)  // the pre-activation, 16-bit, before GELU
        if (ok) store_16<BF16>(p.aux_out, static_cast<int64_t>(t) * p.N + n, z);
      if constexpr (AppliesGelu<EPI>::value) z = gelu_erf(z);
      if constexpr (EPI == EPI_RELU_BIAS || EPI == EPI_RELU_AUX_BIAS) {
        const bool pos = z > 0.f;
        if constexpr (EPI == EPI_RELU_AUX_BIAS) {
          const uint32_t w = __ballot_sync(0xffffffffu, pos && n_ok);
          if (lane == static_cast<uint32_t>(j)) myword = w;
        }
        z = pos ? z : 0.f;
      }
      if (ok) store_out<BF16, OUTM>(p, static_cast<int64_t>(t) * p.N + n, z);
    }
    if constexpr (EPI == EPI_RELU_AUX_BIAS) {
      const int t = t0 + static_cast<int>(lane);
      if (lane < 16 && t < p.T && word < p.aux_words) p.aux_out[static_cast<int64_t>(t) * p.aux_words + word] = myword;
    }
  }
}

// Whole-tile rows: the unchecked form where the 16 rows and the warp's 32
// features are all in range (warp_ok: every lane's feature is below N), for
// 16-bit and fp32 outputs. Instances for at most 16 rows (TP = 16) keep only
// the checked form: their one block of rows is full only at T = 16, and the
// larger code made T = 1 and 8 about 0.3 us slower.
template <int EPI, bool BF16, bool TRY_FULL>
__device__ __forceinline__ void skinny_finish16(const SkinnyParams& p, float (&v)[16], int t0, int n, bool n_ok,
                                                bool warp_ok, int word, float bias_n, float& dbias_acc,
                                                const Mask16& mk) {
  if (TRY_FULL && warp_ok && t0 + 16 <= p.T) {
    if (p.out_f32)
      skinny_finish16_rows<EPI, BF16, 1, true>(p, v, t0, n, n_ok, word, bias_n, dbias_acc, mk);
    else
      skinny_finish16_rows<EPI, BF16, 0, true>(p, v, t0, n, n_ok, word, bias_n, dbias_acc, mk);
  } else {
    skinny_finish16_rows<EPI, BF16, 2, false>(p, v, t0, n, n_ok, word, bias_n, dbias_acc, mk);
  }
}

// Sum the segments' partials of one tile, 32 rows at a time, in segment
// order, and finish those rows. With S > 0 the segment loop is unrolled so
// that all S x 32 loads of a batch are in flight together (the reads are
// L2 round trips; issued one by one they would dominate the kernel).
template <int S, int TP, int EPI, bool BF16>
__device__ __forceinline__ void skinny_fixup(const SkinnyParams& p, const float* base, int nsegs, int n, bool n_ok,
                                             int word, float bias_n, float& dbias_acc) {
  constexpr int SEG = TP * 128;
  constexpr int RB = TP < 32 ? TP : 32;  // rows per batch
#pragma unroll 1
  for (int t0 = 0; t0 < TP; t0 += RB) {
    if (t0 >= p.T) break;
    Mask16 mk[RB / 16];
    if constexpr (EPI == EPI_DRELU_BGRAD) {
#pragma unroll
      for (int h = 0; h < RB / 16; ++h) mk[h] = skinny_mask16(p, t0 + h * 16, word);
    }
    float v[RB];
#pragma unroll
    for (int j = 0; j < RB; ++j) v[j] = 0.f;
    if constexpr (S > 0) {
      float x[S][RB];
#pragma unroll
      for (int sg = 0; sg < S; ++sg)
#pragma unroll
        for (int j = 0; j < RB; ++j) x[sg][j] = __ldcg(base + sg * SEG + (t0 + j) * 128);
#pragma unroll
      for (int sg = 0; sg < S; ++sg)
#pragma unroll
        for (int j = 0; j < RB; ++j) v[j] += x[sg][j];
    } else {
      for (int sg = 0; sg < nsegs; ++sg) {
        float x[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j) x[j] = __ldcg(base + sg * SEG + (t0 + j) * 128);
#pragma unroll
        for (int j = 0; j < RB; ++j) v[j] += x[j];
      }
    }
#pragma unroll
    for (int h = 0; h < RB / 16; ++h) {
      float w[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) w[j] = v[h * 16 + j];
      skinny_finish16_rows<EPI, BF16, 2, false>(p, w, t0 + h * 16, n, n_ok, word, bias_n, dbias_acc, mk[h]);
    }
  }
}

template <int TP, int KPS, int EPI, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const SkinnyParams p) {
  using L = SkinnySmem<TP, KPS>;
  constexpr int STAGES = L::STAGES;
  static_assert(TP == 16 || TP == 32 || TP == 64 || TP == 128 || TP == 256, "TP must be a power of two in [16, 256]");
  constexpr uint32_t TMEM_COLS = 2 * TP < 32 ? 32 : 2 * TP;
  constexpr uint32_t IDESC = idesc_f16(BF16, /*A MN-major*/ true, /*B MN-major*/ false, 128, TP);

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
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);

  const uint32_t warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  const uint32_t lo = blockIdx.x * static_cast<uint32_t>(p.total_kb) / gridDim.x;
  const uint32_t hi = (blockIdx.x + 1u) * static_cast<uint32_t>(p.total_kb) / gridDim.x;

  // the tile kernel's bounded wait reads its timeout and status from TileParams
  TileParams wp{};
  wp.status = p.status;
  wp.timeout_ns = p.timeout_ns;

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
    *last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
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
      uint32_t g = lo;
      Segment s;
      // W tiles may also be prefetched into L2 p.prefetch k-blocks ahead of
      // the shared-memory ring, so that the ring's loads hit L2.
      uint32_t pf = lo;
      const auto prefetch_upto = [&](uint32_t upto) {
        for (; pf < upto && pf < hi; ++pf) {
          const int t = static_cast<int>(pf / static_cast<uint32_t>(p.kbt));
          const int kb = static_cast<int>(pf - static_cast<uint32_t>(t) * static_cast<uint32_t>(p.kbt));
          tma_prefetch_l2_2d(&tmW, t * 128, kb * L::BK);
          tma_prefetch_l2_2d(&tmW, t * 128 + 64, kb * L::BK);
        }
      };
      uint32_t gk = lo;  // global k-block index of the next load
      const uint64_t pol_w = l2_policy_evict_first(), pol_x = l2_policy_evict_last();
      while (ok && skinny_segment(p, hi, g, s)) {
        const int n0 = s.tile * 128;
        for (int kb = s.kb0; kb < s.kb1; ++kb, ++it, ++gk) {
          if (p.prefetch > 0) prefetch_upto(gk + static_cast<uint32_t>(p.prefetch));
          const uint32_t st = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&empty[st], ph ^ 1u, wp, abort_flag, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[st], L::STAGE);
          if (p.cache_hints) {
            tma_load_2d_hint(sA + st * L::A_BYTES, &tmW, &full[st], n0, kb * L::BK, pol_w);
            tma_load_2d_hint(sA + st * L::A_BYTES + L::A_CHUNK, &tmW, &full[st], n0 + 64, kb * L::BK, pol_w);
#pragma unroll
            for (int j = 0; j < KPS; ++j)
              tma_load_2d_hint(sB + st * L::B_BYTES + j * L::B_SUB, &tmX, &full[st], kb * L::BK + j * kBK, 0, pol_x);
          } else {
            tma_load_2d(sA + st * L::A_BYTES, &tmW, &full[st], n0, kb * L::BK);
            tma_load_2d(sA + st * L::A_BYTES + L::A_CHUNK, &tmW, &full[st], n0 + 64, kb * L::BK);
#pragma unroll
            for (int j = 0; j < KPS; ++j)
              tma_load_2d(sB + st * L::B_BYTES + j * L::B_SUB, &tmX, &full[st], kb * L::BK + j * kBK, 0);
          }
        }
      }
      const uint32_t inflight = it < STAGES ? it : STAGES;
      for (uint32_t i = it - inflight; i < it; ++i)
        wait_bounded(&full[i % STAGES], (i / STAGES) & 1u, wp, abort_flag, 2, /*honour_abort=*/false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0, scount = 0;
      bool ok = true;
      uint32_t g = lo;
      Segment s;
      while (ok && skinny_segment(p, hi, g, s)) {
        const uint32_t buf = scount & 1u;
        const uint32_t tph = (scount >> 1) & 1u;
        ++scount;
        if (!wait_bounded(&tempty[buf], tph ^ 1u, wp, abort_flag, 3)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * TP;
        for (int kb = s.kb0; kb < s.kb1; ++kb, ++it) {
          const uint32_t st = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&full[st], ph, wp, abort_flag, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + st * L::A_BYTES);
          const uint32_t b0 = smem_u32(sB + st * L::B_BYTES);
#pragma unroll
          for (int j = 0; j < KPS; ++j) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              // A = W^T: feature-major, 64-feature chunks A_CHUNK apart (LBO), 8 k-rows 1 KB apart (SBO)
              const uint64_t adesc = smem_desc_sw128(a0 + j * L::A_SUB + kk * 2048, L::A_CHUNK, 1024);
              // B = X: K-major 128-byte rows, 8-row groups 1 KB apart, one TP-row block per 64 k
              const uint64_t bdesc = smem_desc_sw128(b0 + j * L::B_SUB + kk * 32, 16, 1024);
              umma_f16(d_tmem, adesc, bdesc, IDESC, (kb > s.kb0 || j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[st]);
        }
        if (!ok) break;
        // (fault injection: the epilogue then waits on a barrier nothing arrives on)
        if (!(p.inject_stall && scount == 1)) umma_commit(&tfull[buf]);
      }
      umma_commit(drain);
      wait_bounded(drain, 0, wp, abort_flag, 5, /*honour_abort=*/false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t ew = warp & 3u;
    const uint32_t et = threadIdx.x - 64;
    uint32_t scount = 0;
    bool ok = true;
    uint32_t g = lo;
    Segment s;
    while (skinny_segment(p, hi, g, s)) {
      const uint32_t buf = scount & 1u;
      const uint32_t tph = (scount >> 1) & 1u;
      ++scount;
      const int n_local = static_cast<int>(ew * 32 + lane);
      const int n = s.tile * 128 + n_local;
      const bool n_ok = n < p.N;
      const bool warp_ok = __all_sync(0xffffffffu, n_ok);  // all 32 features of this warp in range
      const int word = (s.tile * 128 + static_cast<int>(ew) * 32) >> 5;
      float bias_n = 0.f;
      if constexpr (AddsBias<EPI>::value)
        bias_n = n_ok ? load_bias<BF16>(p.bias, p.bias_f32, n) : 0.f;
      float dbias_acc = 0.f;
      const bool whole = s.kb0 == 0 && s.kb1 == p.kbt;
      // DRELU_BGRAD, whole tile: every mask word the tile needs, loaded before
      // the accumulator wait so that none of them is fetched while the
      // epilogue runs (lane l holds the word of row 32·i + l in mrow[i])
      constexpr int MR = (TP + 31) / 32;
      uint32_t mrow[MR];
#pragma unroll
      for (int i = 0; i < MR; ++i) mrow[i] = 0u;
      if constexpr (EPI == EPI_DRELU_BGRAD)
        if (whole)
#pragma unroll
          for (int i = 0; i < MR; ++i) {
            const int t = i * 32 + static_cast<int>(lane);
            if (t < p.T && word < p.aux_words) mrow[i] = __ldg(p.aux_in + static_cast<int64_t>(t) * p.aux_words + word);
          }
      if (ok) ok = wait_bounded(&tfull[buf], tph, wp, abort_flag, 6);
      ok = __all_sync(0xffffffffu, ok);
      const uint32_t tbase = tmem_base + ((ew * 32u) << 16) + buf * TP;
      float* slot = p.partials + (static_cast<int64_t>(s.tile) * p.max_segs + s.seg) * (TP * 128);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < TP / 16; ++c) {
          if (c * 16 >= p.T) break;  // warp-uniform
          Mask16 mk{};
          if constexpr (EPI == EPI_DRELU_BGRAD)
            if (whole) {
#pragma unroll
              for (int j = 0; j < 16; ++j) mk.m[j] = __shfl_sync(0xffffffffu, mrow[0], (c & 1) * 16 + j);
              if (c & 1)
#pragma unroll
                for (int i = 0; i + 1 < MR; ++i) mrow[i] = mrow[i + 1];
            }
          uint32_t r[16];
          tmem_ld_32x32b_x16(tbase + c * 16, r);
          tmem_wait_ld();
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
          if (whole) {
            skinny_finish16<EPI, BF16, (TP > 16)>(p, v, c * 16, n, n_ok, warp_ok, word, bias_n, dbias_acc, mk);
          } else if (TP > 16 && c * 16 + 16 <= p.T) {
#pragma unroll
            for (int j = 0; j < 16; ++j) slot[(c * 16 + j) * 128 + n_local] = v[j];
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c * 16 + j < p.T) slot[(c * 16 + j) * 128 + n_local] = v[j];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
      }
      if (whole) {
        if constexpr (EPI == EPI_DRELU_BGRAD)
          if (ok && n_ok) p.dbias[n] = dbias_acc;
      } else {
        // publish this segment's partial, take a ticket; the last segment finishes the tile
        __threadfence();
        named_bar_sync(1, 128);
        if (et == 0) {
          int last = 0;
          if (ok) {
            const int prev = atomicAdd(p.tickets + s.tile, 1);
            last = prev == s.nsegs - 1;
            if (last) p.tickets[s.tile] = 0;  // ready for the next launch
          }
          *last_flag = last;
        }
        named_bar_sync(1, 128);
        const bool last = *last_flag != 0;
        if (ok && last) {
          __threadfence();
          const float* base = p.partials + static_cast<int64_t>(s.tile) * p.max_segs * (TP * 128) + n_local;
          switch (s.nsegs) {
            case 2: skinny_fixup<2, TP, EPI, BF16>(p, base, s.nsegs, n, n_ok, word, bias_n, dbias_acc); break;
            case 3: skinny_fixup<3, TP, EPI, BF16>(p, base, s.nsegs, n, n_ok, word, bias_n, dbias_acc); break;
            case 4: skinny_fixup<4, TP, EPI, BF16>(p, base, s.nsegs, n, n_ok, word, bias_n, dbias_acc); break;
            default: skinny_fixup<0, TP, EPI, BF16>(p, base, s.nsegs, n, n_ok, word, bias_n, dbias_acc); break;
          }
          if constexpr (EPI == EPI_DRELU_BGRAD)
            if (n_ok) p.dbias[n] = dbias_acc;
        }
        named_bar_sync(1, 128);  // last_flag is reused by the next segment
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace ge
