// gemm_epi.cu -- C ABI of the fused linear-layer GEMM + epilogue library
// (declared in include/gemm_epi.h): plan validation and kernel choice,
// TMA descriptor encoding, launches, the watchdog status word and errors.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_set>

#include "../../include/gemm_epi.h"
#include "aux_kernels.cuh"
#include "kernel_table.h"
#include "skinny_kernel.cuh"
#include "tile2_kernel.cuh"
#include "tile_kernel.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(GEMM_EPI_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

// ---------------------------------------------------------------- registry
std::mutex g_mu;
std::unordered_set<gemm_epi_plan_s*>& live_plans() {
  static std::unordered_set<gemm_epi_plan_s*> s;
  return s;
}

// ----------------------------------------------------- driver entry points
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Fault-injection hooks for the tests take effect only while
// GEMM_EPI_TEST_HOOKS=1 is set as well, so that one stray variable inherited
// by a production process cannot make its plans stall or fail.
bool test_hooks_on() {
  const char* f = getenv("GEMM_EPI_TEST_HOOKS");
  return f && atoi(f) == 1;
}
bool test_hook(const char* name) {
  const char* f = test_hooks_on() ? getenv(name) : nullptr;
  return f && atoi(f) != 0;
}

// GEMM_EPI_INJECT_ENCODE_FAILURE makes every tensor-map encode fail, so an
// execute call must return GEMM_EPI_ERR_CUDA before it launches anything.
bool inject_encode_failure() { return test_hook("GEMM_EPI_INJECT_ENCODE_FAILURE"); }

// The watchdog settings a launch carries: the limit of each bounded wait
// (2 s; GEMM_EPI_WAIT_TIMEOUT_MS overrides) and, for the watchdog tests,
// GEMM_EPI_INJECT_STALL -- the MMA issuer withholds its first tile's
// completion signal, so the epilogue's wait runs out and the kernel reports
// ERR_TIMEOUT. Read when a plan is created and on every call of the
// allocation-free entry point.
struct WatchdogEnv {
  uint64_t timeout_ns = 2000000000ull;
  int inject_stall = 0;
};
WatchdogEnv watchdog_env() {
  WatchdogEnv w;
  if (const char* t = getenv("GEMM_EPI_WAIT_TIMEOUT_MS")) {
    const long long ms = atoll(t);
    if (ms > 0) w.timeout_ns = (uint64_t)ms * 1000000ull;
  }
  w.inject_stall = test_hook("GEMM_EPI_INJECT_STALL") ? 1 : 0;
  return w;
}

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor of 16-bit elements: `inner` contiguous columns,
// `outer` rows; box of box_inner x box_outer with 128-byte swizzle (operand
// tiles) or 64-byte swizzle (32 x 32 output staging blocks).
int encode_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer, const char* name,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(GEMM_EPI_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (inject_encode_failure()) return fail(GEMM_EPI_ERR_CUDA, "injected tensor map encode failure");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GEMM_EPI_ERR_CUDA, "tensor map encode for %s failed (CUresult %d)", name, (int)r);
  return GEMM_EPI_OK;
}

using ge_inst::SkinnyKernelFn;
using ge_inst::TileKernelFn;

// the output (Y, dZ or an unfused intermediate) as the tile kernels' TMA
// stores see it: 32 x 32 blocks, 64-byte swizzle
int encode_out(CUtensorMap* map, const void* out, int64_t T, int64_t N) {
  return encode_2d(map, out, (uint64_t)N, (uint64_t)T, 32, 32, "the output", CU_TENSOR_MAP_SWIZZLE_64B);
}

// fp32 output: 16 x 32 blocks (64-byte rows, the 16-bit blocks' staging layout)
int encode_out_f32(CUtensorMap* map, const void* out, int64_t T, int64_t N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(GEMM_EPI_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (inject_encode_failure()) return fail(GEMM_EPI_ERR_CUDA, "injected tensor map encode failure");
  const cuuint64_t dims[2] = {(uint64_t)N, (uint64_t)T};
  const cuuint64_t strides[1] = {(uint64_t)N * 4};
  const cuuint32_t box[2] = {16, 32};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(out), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GEMM_EPI_ERR_CUDA, "tensor map encode for the fp32 output failed (CUresult %d)", (int)r);
  return GEMM_EPI_OK;
}

// the mask words as the tile kernels' TMA stores see them: per warp and tile
// a block of BN/32 words x 32 rows. Usable when a row of words is a multiple
// of 16 bytes and the pointer is 16-byte aligned; otherwise the kernels store
// the words directly.
bool aux_tma_ok(const void* aux, int64_t N, int bn) {
  const int64_t words = (N + 31) / 32;
  return (bn == 128 || bn == 256) && (words % 4) == 0 && (reinterpret_cast<uintptr_t>(aux) & 15) == 0;
}

int encode_aux(CUtensorMap* map, const void* aux, int64_t T, int64_t N, int bn) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(GEMM_EPI_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (inject_encode_failure()) return fail(GEMM_EPI_ERR_CUDA, "injected tensor map encode failure");
  const uint64_t words = (uint64_t)((N + 31) / 32);
  const cuuint64_t dims[2] = {words, (uint64_t)T};
  const cuuint64_t strides[1] = {words * 4};
  const cuuint32_t box[2] = {(cuuint32_t)(bn / 32), 32};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(aux), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GEMM_EPI_ERR_CUDA, "tensor map encode for the mask words failed (CUresult %d)", (int)r);
  return GEMM_EPI_OK;
}

static_assert(static_cast<int>(GEMM_EPI_BIAS) == ge::EPI_BIAS && static_cast<int>(GEMM_EPI_RELU_BIAS) == ge::EPI_RELU_BIAS &&
                  static_cast<int>(GEMM_EPI_RELU_AUX_BIAS) == ge::EPI_RELU_AUX_BIAS &&
                  static_cast<int>(GEMM_EPI_DRELU_BGRAD) == ge::EPI_DRELU_BGRAD &&
                  static_cast<int>(GEMM_EPI_GELU_BIAS) == ge::EPI_GELU_BIAS &&
                  static_cast<int>(GEMM_EPI_WGRAD) == ge::EPI_WGRAD &&
                  static_cast<int>(GEMM_EPI_NONE) == ge::EPI_STORE &&
                  static_cast<int>(GEMM_EPI_GELU_AUX_BIAS) == ge::EPI_GELU_AUX_BIAS,
              "the public epilog values are the kernels' epilog kinds");

struct TileCfg {
  int BN = 256, stages = 4;
  TileKernelFn fn = nullptr;
  uint32_t smem = 0;
  bool pair = false;  // CTA-pair kernel, launched in clusters of 2
  int threads = ge::kThreads;
};

// bk: the weight is given N x K (GEMM_EPI_FLAG_W_NK); never with WGRAD
TileCfg pair_cfg(int epi, bool bf16, bool bk, bool split = false) {
  TileCfg c;
  c.BN = 256;
  c.stages = 6;
  c.smem = ge::Tile2Smem<256, 6>::BYTES;
  if (!split && (epi == ge::EPI_GELU_BIAS || epi == ge::EPI_GELU_AUX_BIAS)) {
    // eight epilogue warps (ge::PairEpiWarps), five stages
    c.stages = 5;
    c.smem = ge::Tile2Smem<256, 5, 8>::BYTES;
    c.threads = 64 + 32 * 8;
  }
  if (split)
    c.fn = bf16 ? ge_inst::pair_split_bf16(epi, bk) : ge_inst::pair_split_f16(epi, bk);
  else
    c.fn = bf16 ? ge_inst::pair_bf16(epi, bk) : ge_inst::pair_f16(epi, bk);
  c.pair = true;
  return c;
}

// How many CTA pairs of this kernel the device holds at once (clusters of
// two must sit in one GPC); one pair per two SMs if the query fails.
int max_resident_pairs(const TileCfg& c, int sms) {
  if (cudaFuncSetAttribute(c.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)c.smem) != cudaSuccess) {
    cudaGetLastError();
    return sms / 2;
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)(sms / 2 * 2), 1, 1);
  lc.blockDim = dim3((unsigned)c.threads, 1, 1);
  lc.dynamicSmemBytes = c.smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)c.fn, &lc) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return sms / 2;
  }
  return n < sms / 2 ? n : sms / 2;
}

TileCfg tile_cfg(int BN, int epi, bool bf16, bool bk) {
  TileCfg c;
  c.BN = BN == 256 || BN == 192 || BN == 128 ? BN : 64;
  if (c.BN == 256) {
    c.stages = 4;
    c.smem = ge::TileSmem<256, 4>::BYTES;
  } else if (c.BN == 192) {
    c.stages = 4;
    c.smem = ge::TileSmem<192, 4>::BYTES;
  } else if (c.BN == 128) {
    c.stages = 6;
    c.smem = ge::TileSmem<128, 6>::BYTES;
  } else {
    c.stages = 8;
    c.smem = ge::TileSmem<64, 8>::BYTES;
  }
  c.fn = bk ? (bf16 ? ge_inst::tile_bf16_nk(c.BN, epi) : ge_inst::tile_f16_nk(c.BN, epi))
            : (bf16 ? ge_inst::tile_bf16_mn(c.BN, epi) : ge_inst::tile_f16_mn(c.BN, epi));
  return c;
}

int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

struct SkinnyCfg {
  int TP = 16;
  int KPS = 1;  // 64-deep k-blocks per pipeline stage
  SkinnyKernelFn fn = nullptr;
  uint32_t smem = 0;
  int stages = 0;
};

template <int TP, int KPS>
SkinnyCfg skinny_cfg_kps(int epi, bool bf16) {
  SkinnyCfg c;
  c.TP = TP;
  c.KPS = KPS;
  if constexpr (KPS == 2)
    c.fn = bf16 ? ge_inst::skinny_bf16_kps2(TP, epi) : ge_inst::skinny_f16_kps2(TP, epi);
  else
    c.fn = bf16 ? ge_inst::skinny_bf16_kps1(TP, epi) : ge_inst::skinny_f16_kps1(TP, epi);
  c.smem = ge::SkinnySmem<TP, KPS>::BYTES;
  c.stages = ge::SkinnySmem<TP, KPS>::STAGES;
  return c;
}

template <int TP>
SkinnyCfg skinny_cfg_tp(int epi, bool bf16, int kps) {
  if (kps >= 2) return skinny_cfg_kps<TP, 2>(epi, bf16);
  return skinny_cfg_kps<TP, 1>(epi, bf16);
}

// Two k-blocks per stage (W stages of 32 KB) while X's share of a stage is
// small: at T = 1 and 8 (N = 11008, K = 4096) 26.7 us against 28.7 us with
// one, at T = 64 28.7 against 32.8 us, at T = 128 32.8 / 36.8 against
// 36.8 / 38.9 us (forward / backward, current sources; an older build had
// one k-block ahead at T = 128). Four per stage never beat two.
int default_kps(int64_t T) { return T <= 128 ? 2 : 1; }

SkinnyCfg skinny_cfg(int64_t T, int epi, bool bf16) {
  int kps = default_kps(T);
  if (const char* f = getenv("GEMM_EPI_SKINNY_KPS")) {  // tuning override: 1 or 2
    const int v = atoi(f);
    if (v == 1 || v == 2) kps = v;
  }
  if (T <= 16) return skinny_cfg_tp<16>(epi, bf16, kps);
  if (T <= 32) return skinny_cfg_tp<32>(epi, bf16, kps);
  if (T <= 64) return skinny_cfg_tp<64>(epi, bf16, kps);
  if (T <= 128) return skinny_cfg_tp<128>(epi, bf16, kps);
  return skinny_cfg_tp<256>(epi, bf16, kps);
}

// Kernel and tile choice by a small cost model, fitted to measurements on
// one B200 (bf16, K = 4096, one tile per CTA, events around each call):
// the one-CTA kernel's throughput per SM grows with the tile width, because
// every stage brings the same 16 KB of X for BN/64 times the MMA work --
// about 3.1, 5.4, 7.5 and 9.3 TFLOP/s per SM at BN = 64, 128, 192 and 256
// (e.g. T = 512, N = K = 4096: 49.1 us with 256 tiles of BN = 64, 30.7 us
// with 128 of BN = 128). CTA pairs (256 x 256 tiles, two thirds of the
// operand bytes per FLOP) run about 10 per SM. A plan's estimate is rounds
// of tiles x time per tile; the pair kernel's last round counts half when its
// tiles fit the half-width tail split.
double tile_rate(int bn) { return bn == 256 ? 9.3 : bn == 192 ? 7.5 : bn == 128 ? 5.4 : 3.1; }
constexpr double kPairRate = 10.0;

double est_tile_us(int64_t T, int64_t N, int64_t K, int bn, int sms) {
  const int64_t tiles = ((T + ge::kBM - 1) / ge::kBM) * ((N + bn - 1) / bn);
  const int64_t rounds = (tiles + sms - 1) / sms;
  return double(rounds) * 2.0 * ge::kBM * bn * double(K) / (tile_rate(bn) * 1e6);
}

double est_pair_us(int64_t T, int64_t N, int64_t K, int pairs) {
  const int64_t tiles = ((T + 255) / 256) * ((N + 255) / 256);
  const int64_t full = tiles / pairs, tail = tiles % pairs;
  const double rounds = double(full) + (tail == 0 ? 0.0 : 2 * tail <= pairs ? 0.5 : 1.0);
  return rounds * 2.0 * 256 * 256 * double(K) / (2.0 * kPairRate * 1e6);
}

// one-CTA tile width: the fastest estimate (the wider on a tie)
int choose_bn(int64_t T, int64_t N, int64_t K, int num_sms) {
  if (const char* f = getenv("GEMM_EPI_FORCE_BN")) {
    int v = atoi(f);
    if (v == 64 || v == 128 || v == 192 || v == 256) return v;
  }
  int best = 256;
  double best_us = est_tile_us(T, N, K, 256, num_sms);
  for (int bn : {192, 128, 64}) {
    const double us = est_tile_us(T, N, K, bn, num_sms);
    if (us < best_us * 0.999) {
      best = bn;
      best_us = us;
    }
  }
  return best;
}

// CTA pairs when there is at least one full wave of pair tiles (fewer would
// leave pairs idle, and half-width tail units are fed less efficiently), X is
// at most 1 GiB, and the estimate beats the best one-CTA tile. The size limit
// is measured: on the 65536 x 16384 x 8192 fp16 problem (X = 2 GiB) the pair
// kernel read 46.0 GB from DRAM per launch against the one-CTA kernel's 24.3
// (ncu), and under the 1 kW power cap ran at 908 against 1106 TFLOP/s.
// GEMM_EPI_FORCE_KERNEL=tile / pair overrides.
bool use_pair(int64_t T, int64_t N, int64_t K, int num_sms) {
  if (const char* f = getenv("GEMM_EPI_FORCE_KERNEL")) {
    if (!strcmp(f, "tile") || !strcmp(f, "skinny")) return false;
    if (!strcmp(f, "pair")) return T > 128;
  }
  if (T <= 128 || T * K * 2 > ((int64_t)1 << 30)) return false;
  const int pairs = num_sms / 2;
  const int64_t pair_tiles = ((T + 255) / 256) * ((N + 255) / 256);
  if (pair_tiles < pairs) return false;
  const int bn = choose_bn(T, N, K, num_sms);
  return est_pair_us(T, N, K, pairs) <= est_tile_us(T, N, K, bn, num_sms);
}

// The few-row kernel for T <= 128; from 129 rows on, one-CTA tiles of 192
// columns beat it (T = 256, N = 11008, K = 4096: 34.7 / 36.9 us against
// 47.1 / 51.2 us, and against the CTA pair's 36.6 / 40.9 us).
// The few-row kernel's range arithmetic is 32-bit: (k-blocks + 1) x grid must
// stay below 2^31 (k-blocks of 64 at most, grid at most one CTA per SM).
bool skinny_fits(int64_t N, int64_t K, int sms) {
  const int64_t kblocks = ((N + 127) / 128) * ((K + 63) / 64);
  return (kblocks + 1) * (int64_t)sms < (int64_t(1) << 31);
}

bool use_skinny(int64_t T) {
  if (const char* f = getenv("GEMM_EPI_FORCE_KERNEL")) {
    if (!strcmp(f, "tile")) return false;
    if (!strcmp(f, "skinny")) return T <= 256;
    if (!strcmp(f, "pair")) return T <= 128;
  }
  return T <= 128;
}

}  // namespace

struct gemm_epi_plan_s {
  int64_t T, N, K;   // the kernels' rows, columns and contraction length
  int64_t uT, uK;    // the caller's T and K (WGRAD: rows = uK, contraction = uT)
  int dtype, epilog;
  int device, num_sms;
  int m_tiles, n_tiles, k_blocks, num_tiles, aux_words, grid, group_m;
  int raster_n = 0;  // tile order by column groups (see choose_raster)
  int pair_split = 0;        // CTA pairs in stream-K mode
  int pair_sk_first = 1;     // stream-K tiles before the whole tiles
  int pair_max_segs = 1;
  float* pair_slots = nullptr;  // stream-K fp32 partials
  int* pair_flags = nullptr;    // stream-K segment counters, zero between launches
  int n_pair_flags = 0;
  size_t pair_bytes = 0;
  TileCfg cfg;       // fused kernel
  TileCfg cfg_store; // unfused GEMM (plain store)
  float* partials = nullptr;  // DRELU_BGRAD: m_tiles x N
  size_t partial_bytes = 0;
  int* col_tickets = nullptr;  // DRELU_BGRAD on the tile kernels: n_tickets counters
  int n_tickets = 0;
  int* status_host = nullptr;
  int* status_dev = nullptr;
  uint64_t timeout_ns = 0;
  int inject_stall = 0;  // GEMM_EPI_INJECT_STALL at plan time (watchdog tests)
  int tail_split = 1;    // GEMM_EPI_TAIL_SPLIT=0 keeps whole tiles in the pair kernel's last round
  int bias_f32 = 0;      // gemm_epi_set_bias_f32: the forward bias is fp32
  int w_nk = 0;          // GEMM_EPI_FLAG_W_NK: W / W2 given N x K (K contiguous)
  int out_f32 = 0;       // GEMM_EPI_FLAG_OUT_F32: Y / dZ / dW written as fp32
  int cache_hints = 0;   // few-row kernel: L2 eviction policies on the operand loads (GEMM_EPI_CACHE_HINTS)
  // tensor-map cache
  const void* a_ptr = nullptr;
  const void* b_ptr = nullptr;
  const void* y_ptr = nullptr;
  const void* aux_ptr = nullptr;
  CUtensorMap tmA, tmB, tmY, tmAux;
  // few-row kernel (kernel == 1)
  int kernel = 0;
  SkinnyCfg sk;
  int sk_grid = 0, sk_kbt = 0, sk_total = 0, sk_max_segs = 1, sk_prefetch = 0;
  float* sk_partials = nullptr;
  int* sk_tickets = nullptr;
  size_t sk_bytes = 0;
  const void* xs_ptr = nullptr;
  CUtensorMap tmXs;  // the row operand with a TP-row box
  const void* ws_ptr = nullptr;
  CUtensorMap tmWs;  // the weight operand with a 64·KPS-row box
};

namespace {

gemm_epi_plan_s* lookup(gemm_epi_plan_t p) {
  std::lock_guard<std::mutex> g(g_mu);
  return live_plans().count(p) ? p : nullptr;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int take_status(gemm_epi_plan_s* p) {
  volatile int* s = p->status_host;
  const int v = *s;
  if (v != 0) {
    *s = 0;
    // an interrupted launch may have left split-tile tickets counted
    if (p->sk_tickets) cudaMemset(p->sk_tickets, 0, sizeof(int) * (size_t)ceil_div(p->N, 128));
    if (p->col_tickets) cudaMemset(p->col_tickets, 0, sizeof(int) * (size_t)p->n_tickets);
    if (p->pair_flags) cudaMemset(p->pair_flags, 0, sizeof(int) * (size_t)p->n_pair_flags);
    return fail(GEMM_EPI_ERR_TIMEOUT, "a kernel of this plan gave up waiting (watchdog code 0x%x)", v);
  }
  return GEMM_EPI_OK;
}

int prepare_maps(gemm_epi_plan_s* p, const void* A, const void* B) {
  if (A != p->a_ptr && p->epilog == GEMM_EPI_WGRAD) {
    // X (uT x uK) read as the MN-major A = X^T: boxes of 64 features x 64 rows
    int rc = encode_2d(&p->tmA, A, (uint64_t)p->T, (uint64_t)p->K, 64, ge::kBK, "X");
    if (rc) return rc;
    p->a_ptr = A;
  } else if (A != p->a_ptr) {
    int rc = encode_2d(&p->tmA, A, (uint64_t)p->K, (uint64_t)p->T, ge::kBK, ge::kBM, "the row operand");
    if (rc) return rc;
    p->a_ptr = A;
  }
  if (B != p->b_ptr && p->w_nk) {
    // N x K weight, K-major: one box of 64 k x (the CTA's) BN rows per stage
    const uint32_t rows = p->kernel == 2 ? 128u : (uint32_t)p->cfg.BN;
    int rc = encode_2d(&p->tmB, B, (uint64_t)p->K, (uint64_t)p->N, ge::kBK, rows, "the N x K weight operand");
    if (rc) return rc;
    p->b_ptr = B;
  } else if (B != p->b_ptr) {
    int rc = encode_2d(&p->tmB, B, (uint64_t)p->N, (uint64_t)p->K, 64, ge::kBK, "the weight operand");
    if (rc) return rc;
    p->b_ptr = B;
  }
  return GEMM_EPI_OK;
}

ge::TileParams base_params(const gemm_epi_plan_s* p) {
  ge::TileParams k{};
  k.T = (int32_t)p->T;
  k.N = (int32_t)p->N;
  k.K = (int32_t)p->K;
  k.m_tiles = p->m_tiles;
  k.n_tiles = p->n_tiles;
  k.k_blocks = p->k_blocks;
  k.num_tiles = p->num_tiles;
  k.aux_words = p->aux_words;
  k.group_m = p->group_m;
  k.raster_n = p->raster_n;
  k.sk_slots = p->pair_slots;
  k.sk_flags = p->pair_flags;
  k.sk_max_segs = p->pair_max_segs;
  k.sk_first = p->pair_sk_first;
  k.status = p->status_dev;
  k.timeout_ns = p->timeout_ns;
  k.inject_stall = p->inject_stall;
  k.tail_split = p->tail_split;
  k.bias_f32 = p->bias_f32;
  k.out_f32 = p->out_f32;
  return k;
}

int prepare_out_map(gemm_epi_plan_s* p, const void* out) {
  if (out != p->y_ptr) {
    int rc = p->out_f32 ? encode_out_f32(&p->tmY, out, p->T, p->N) : encode_out(&p->tmY, out, p->T, p->N);
    if (rc) return rc;
    p->y_ptr = out;
  }
  return GEMM_EPI_OK;
}

int launch_tile(gemm_epi_plan_s* p, const TileCfg& c, const ge::TileParams& k_in, cudaStream_t s) {
  ge::TileParams k = k_in;
  int rc = prepare_out_map(p, k.out);
  if (rc) return rc;
  k.aux_tma = 0;
  if (p->epilog == GEMM_EPI_GELU_AUX_BIAS) {
    // the pre-activation Z (T x N, 16-bit) is stored directly by the epilogue threads
  } else if (k.aux_out && aux_tma_ok(k.aux_out, p->N, c.BN)) {
    if (k.aux_out != p->aux_ptr) {
      rc = encode_aux(&p->tmAux, k.aux_out, p->T, p->N, c.BN);
      if (rc) return rc;
      p->aux_ptr = k.aux_out;
    }
    k.aux_tma = 1;
  }
  const CUtensorMap& tmAux = k.aux_tma ? p->tmAux : p->tmY;  // unused by the kernel unless aux_tma
  if (c.pair) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p->grid, 1, 1);
    cfg.blockDim = dim3((unsigned)c.threads, 1, 1);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, c.fn, p->tmA, p->tmB, p->tmY, tmAux, k);
    if (e != cudaSuccess) return cuda_fail(e, "pair kernel launch");
    return GEMM_EPI_OK;
  }
  c.fn<<<p->grid, ge::kThreads, c.smem, s>>>(p->tmA, p->tmB, p->tmY, tmAux, k);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "tile kernel launch");
  return GEMM_EPI_OK;
}

// Raster: which operand's block stays in L2 while the other streams past
// it. Holding a group of R row tiles of X (about 48 MB, a little under half
// of the 126 MB L2) while the group sweeps every column block streams W from
// HBM once per group -- once in all when all of X fits (FFN, square). When X
// is both larger than the L2 and at least 4x W, a group of column tiles of W
// (about 64 MB) is held instead and X streams past it. Measured on the
// 65536 x 16384 x 8192 fp16 problem (X 2 GiB, W 256 MiB; ncu, DRAM bytes read
// per launch, one-CTA kernel, 256-column tiles): row groups 24.3 GB; column
// groups of 6, 8 and 12 tiles 20.1, 18.0 and 19.2 GB, at equal time (13.4 to
// 13.8 ms). Every order reads several times the operands there: a wave of
// 148 tiles touches 1.8 GB of operands at K = 16384, 14 times the L2.
// GEMM_EPI_RASTER=m|n and GEMM_EPI_GROUP_M (the group size in tiles)
// override, for measurement.
struct Raster {
  int group = 1;
  int by_n = 0;
};

Raster choose_raster(int64_t T, int64_t N, int64_t K, int tile_rows, int tile_cols) {
  const int64_t m_tiles = (T + tile_rows - 1) / tile_rows, n_tiles = (N + tile_cols - 1) / tile_cols;
  const double x_bytes = 2.0 * T * K, w_bytes = 2.0 * K * N;
  int64_t R = (int64_t)(double(48 << 20) / (2.0 * tile_rows * K));
  int64_t C = (int64_t)(double(64 << 20) / (2.0 * tile_cols * K));
  R = R < 1 ? 1 : R > m_tiles ? m_tiles : R;
  C = C < 1 ? 1 : C > n_tiles ? n_tiles : C;
  Raster r;
  r.by_n = (x_bytes > double(128 << 20) && x_bytes >= 4.0 * w_bytes) ? 1 : 0;
  r.group = (int)(r.by_n ? C : R);
  if (const char* f = getenv("GEMM_EPI_RASTER")) {  // tuning override
    if (!strcmp(f, "m") || !strcmp(f, "n")) {
      r.by_n = f[0] == 'n';
      r.group = (int)(r.by_n ? C : R);
    }
  }
  if (const char* f = getenv("GEMM_EPI_GROUP_M")) {  // tuning override: the group size in tiles
    const int v = atoi(f);
    if (v >= 1) r.group = v;
  }
  const int64_t outer = r.by_n ? n_tiles : m_tiles;
  if (r.group > outer) r.group = (int)outer;
  return r;
}

int prepare_skinny_maps(gemm_epi_plan_s* p, const void* A, const void* B) {
  if (A != p->xs_ptr) {
    int rc = encode_2d(&p->tmXs, A, (uint64_t)p->K, (uint64_t)p->T, ge::kBK, (uint32_t)p->sk.TP, "the row operand");
    if (rc) return rc;
    p->xs_ptr = A;
  }
  if (B != p->ws_ptr) {  // W in boxes of 64 features x 64·KPS k-rows (the tile kernels' map is tmB)
    int rc = encode_2d(&p->tmWs, B, (uint64_t)p->N, (uint64_t)p->K, 64, (uint32_t)(ge::kBK * p->sk.KPS),
                       "the weight operand");
    if (rc) return rc;
    p->ws_ptr = B;
  }
  return GEMM_EPI_OK;
}

ge::SkinnyParams skinny_params(const gemm_epi_plan_s* p) {
  ge::SkinnyParams k{};
  k.T = (int32_t)p->T;
  k.N = (int32_t)p->N;
  k.K = (int32_t)p->K;
  k.n_tiles = ceil_div(p->N, 128);
  k.kbt = p->sk_kbt;
  k.total_kb = p->sk_total;
  k.aux_words = p->aux_words;
  k.max_segs = p->sk_max_segs;
  k.prefetch = p->sk_prefetch;
  k.partials = p->sk_partials;
  k.tickets = p->sk_tickets;
  k.status = p->status_dev;
  k.timeout_ns = p->timeout_ns;
  k.bias_f32 = p->bias_f32;
  k.out_f32 = p->out_f32;
  k.cache_hints = p->cache_hints;
  k.inject_stall = p->inject_stall;
  return k;
}

int launch_skinny(const gemm_epi_plan_s* p, const ge::SkinnyParams& k, cudaStream_t s) {
  p->sk.fn<<<p->sk_grid, ge::kThreads, p->sk.smem, s>>>(p->tmWs, p->tmXs, k);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "few-row kernel launch");
  return GEMM_EPI_OK;
}

}  // namespace

extern "C" {

gemm_epi_plan_t gemm_epi_plan(int64_t T, int64_t N, int64_t K, gemm_epi_dtype dtype, gemm_epi_epilog epilog) {
  return gemm_epi_plan_ex(T, N, K, dtype, epilog, 0u);
}

gemm_epi_plan_t gemm_epi_plan_ex(int64_t T, int64_t N, int64_t K, gemm_epi_dtype dtype, gemm_epi_epilog epilog,
                                 uint32_t flags) {
  if ((flags & ~(uint32_t)(GEMM_EPI_FLAG_W_NK | GEMM_EPI_FLAG_OUT_F32)) != 0) {
    fail(GEMM_EPI_ERR_INVALID_ARG, "unknown plan flags 0x%x", flags);
    return nullptr;
  }
  const bool w_nk = (flags & GEMM_EPI_FLAG_W_NK) != 0;
  if (w_nk && epilog == GEMM_EPI_WGRAD) {
    fail(GEMM_EPI_ERR_INVALID_ARG, "GEMM_EPI_FLAG_W_NK applies to the weight of forward and DRELU_BGRAD plans");
    return nullptr;
  }
  if (T < 1 || N < 8 || K < 8 || (N % 8) != 0 || (K % 8) != 0) {
    fail(GEMM_EPI_ERR_INVALID_ARG, "bad shape T=%lld N=%lld K=%lld (need T>=1, N,K>=8 and multiples of 8)",
         (long long)T, (long long)N, (long long)K);
    return nullptr;
  }
  if (T > (int64_t)1 << 30 || N > (int64_t)1 << 24 || K > (int64_t)1 << 24 || T * N > ((int64_t)1 << 40)) {
    fail(GEMM_EPI_ERR_INVALID_ARG, "shape too large for 32-bit tile coordinates");
    return nullptr;
  }
  if (dtype != GEMM_EPI_F16 && dtype != GEMM_EPI_BF16) {
    fail(GEMM_EPI_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    return nullptr;
  }
  if (epilog < GEMM_EPI_BIAS || epilog > GEMM_EPI_GELU_AUX_BIAS) {
    fail(GEMM_EPI_ERR_INVALID_ARG, "unknown epilog %d", (int)epilog);
    return nullptr;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cuda_fail(e, "cudaGetDevice");
    return nullptr;
  }
  int major = 0, minor = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || minor != 0) {
    fail(GEMM_EPI_ERR_UNSUPPORTED, "device %d has compute capability %d.%d; this library needs 10.0 (sm_100a)", dev,
         major, minor);
    return nullptr;
  }

  if (epilog == GEMM_EPI_WGRAD && K * N > ((int64_t)1 << 40)) {
    fail(GEMM_EPI_ERR_INVALID_ARG, "shape too large for 32-bit tile coordinates");
    return nullptr;
  }
  auto* p = new gemm_epi_plan_s();
  p->uT = T;
  p->uK = K;
  if (epilog == GEMM_EPI_WGRAD) {  // dW (K x N) = X^T dZ: K output rows, contraction over the T rows
    const int64_t rows = K;
    K = T;
    T = rows;
  }
  p->T = T;
  p->N = N;
  p->K = K;
  p->dtype = dtype;
  p->epilog = epilog;
  p->w_nk = w_nk ? 1 : 0;
  p->out_f32 = (flags & GEMM_EPI_FLAG_OUT_F32) ? 1 : 0;
  p->device = dev;
  p->num_sms = sms;
  const bool bf16 = dtype == GEMM_EPI_BF16;
  const bool pair = use_pair(T, N, K, sms);
  const int bn = pair ? 256 : choose_bn(T, N, K, sms);
  p->cfg = pair ? pair_cfg((int)epilog, bf16, w_nk) : tile_cfg(bn, (int)epilog, bf16, w_nk);
  p->cfg_store = pair ? pair_cfg(ge::EPI_STORE, bf16, w_nk) : tile_cfg(bn, ge::EPI_STORE, bf16, w_nk);
  p->kernel = pair ? 2 : 0;
  p->m_tiles = ceil_div(T, ge::kBM);
  p->n_tiles = ceil_div(N, bn);
  p->k_blocks = ceil_div(K, ge::kBK);
  p->num_tiles = p->m_tiles * p->n_tiles;
  p->aux_words = ceil_div(N, 32);
  const Raster raster = choose_raster(T, N, K, pair ? 2 * ge::kBM : ge::kBM, bn);
  p->group_m = raster.group;
  p->raster_n = raster.by_n;
  p->grid = p->num_tiles < sms ? p->num_tiles : sms;
  const WatchdogEnv wd = watchdog_env();
  p->timeout_ns = wd.timeout_ns;
  p->inject_stall = wd.inject_stall;
  if (const char* f = getenv("GEMM_EPI_TAIL_SPLIT")) p->tail_split = atoi(f) != 0;


  auto cleanup = [&](int rc) {
    if (p->pair_slots) cudaFree(p->pair_slots);
    if (p->pair_flags) cudaFree(p->pair_flags);
    if (p->col_tickets) cudaFree(p->col_tickets);
    if (p->sk_partials) cudaFree(p->sk_partials);
    if (p->sk_tickets) cudaFree(p->sk_tickets);
    if (p->partials) cudaFree(p->partials);
    if (p->status_host) cudaFreeHost(p->status_host);
    delete p;
    (void)rc;
    return nullptr;
  };

  if (pair) {
    // One cluster of two CTAs per 256-row x 256-column tile, up to the number
    // of clusters the device can hold at once (a GPC with an odd number of
    // free SMs cannot place a pair on its last one).
    const int pair_tiles = ceil_div(T, 256) * p->n_tiles;
    const int max_pairs = max_resident_pairs(p->cfg, sms);
    int pairs = pair_tiles < max_pairs ? pair_tiles : max_pairs;
    // Stream-K (the last waves cut into k-ranges) is opt-in,
    // GEMM_EPI_PAIR_SPLIT=1. It evened out the end of the FFN forward while
    // the MMA stream ran at 83 % of the tensor peak (244.0 against 256.8 us),
    // but since the waits suspend instead of spinning and a tile runs at the
    // peak rate, whole tiles are as fast or faster everywhere measured
    // (interleaved runs on one box, forward / backward, us, whole against
    // stream-K): FFN 252.9 / 257.0 against 252.9 / 255.0; T = 1024, N = 5120
    // 51.2 / 56.3 against 53.3 / 60.4; T = 1000, N = 5000, K = 1024
    // 23.6 / 29.7 against 34.8 / 42.0; square 97.3 / 104.7 against
    // 98.3 / 109.6; T = 2048, N = 8192 94.2 / 99.3 against 97.3 / 103.5.
    // The GELU epilogs slow down most with it (FFN GELU_BIAS 443 against 316).
    bool split = false;
    if (const char* f = getenv("GEMM_EPI_PAIR_SPLIT")) split = atoi(f) != 0 && p->k_blocks >= 16;
    if (split && pair_tiles < max_pairs) {
      const int64_t want = (int64_t)pair_tiles * p->k_blocks / 8;  // at least 8 k-blocks per pair
      const int sp = (int)(want < max_pairs ? want : max_pairs);
      split = sp > pair_tiles;
      if (split) pairs = sp;
    }
    p->grid = 2 * pairs;
    if (split) {
      p->pair_split = 1;
      // the stream-K tiles first, so their fixups overlap the whole tiles'
      // MMAs: FFN forward 275.5 against 277.4 us with them last, backward
      // 277.5 against 279.6 (interleaved runs on one box); square equal
      if (const char* f = getenv("GEMM_EPI_PAIR_SK_FIRST")) p->pair_sk_first = atoi(f) != 0;
      p->cfg = pair_cfg((int)epilog, bf16, w_nk, true);
      p->cfg_store = pair_cfg(ge::EPI_STORE, bf16, w_nk, true);
      const int dp_tiles = ge::pair_dp_rounds(pair_tiles, pairs) * pairs;
      const int64_t total = (int64_t)(pair_tiles - dp_tiles) * p->k_blocks;
      p->pair_max_segs = 1;
      for (int t = 0; t < pair_tiles - dp_tiles; ++t) {
        const int64_t a = ge::pair_owner((int64_t)t * p->k_blocks, pairs, total);
        const int64_t b = ge::pair_owner((int64_t)(t + 1) * p->k_blocks - 1, pairs, total);
        if (b - a + 1 > p->pair_max_segs) p->pair_max_segs = (int)(b - a + 1);
      }
      // one slot per pair and CTA (a pair hands on at most one segment: its first unit)
      p->pair_bytes = (size_t)pairs * 2 * ge::kBM * 256 * sizeof(float);
      e = cudaMalloc((void**)&p->pair_slots, p->pair_bytes);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMalloc(stream-K partials)"));
      e = cudaMalloc((void**)&p->pair_flags, sizeof(int) * 2 * (size_t)pairs);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMalloc(stream-K flags)"));
      e = cudaMemset(p->pair_flags, 0, sizeof(int) * 2 * (size_t)pairs);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMemset(stream-K flags)"));
      p->n_pair_flags = 2 * pairs;
      p->pair_bytes += sizeof(int) * 2 * (size_t)pairs;
    }
  }
  for (const TileCfg* c : {&p->cfg, &p->cfg_store}) {
    if (!c->fn) return cleanup(fail(GEMM_EPI_ERR_INVALID_ARG, "no kernel instance for this epilog and layout"));
    e = cudaFuncSetAttribute(c->fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)c->smem);
    if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)"));
  }
  // L2 eviction hints on the few-row kernel's operand loads (W evict_first, X
  // evict_last), where W streams through L2 once (measured at N = 11008, K =
  // 4096: T = 1 25.1 / 24.5 us against 27.3 / 26.8, T = 64 32.6 / 33.4 against
  // 33.2 / 34.3). The tile kernels load without hints: there they did not help
  // the FFN and square shapes and slowed the large one (17.6 against 16.8 ms).
  if (!pair && epilog != GEMM_EPI_WGRAD && !w_nk && use_skinny(T) && skinny_fits(N, K, sms)) {
    p->kernel = 1;
    p->cache_hints = 1;
    p->sk = skinny_cfg(T, (int)epilog, bf16);
    const int n_tiles = ceil_div(N, 128);
    p->sk_kbt = ceil_div(K, (int64_t)ge::kBK * p->sk.KPS);
    p->sk_total = n_tiles * p->sk_kbt;
    const int min_stages = 8 / p->sk.KPS;  // at least 512 k per CTA under stream-K
    // every CTA gets at least 8 k-blocks, so a tile is shared by few CTAs
    // With at least half as many feature tiles as SMs (and no more than
    // SMs), every CTA takes whole tiles: no split-tile partials or fixups,
    // whose dependent round trips cost more than the idle SMs would give.
    // Otherwise stream-K over up to one CTA per SM, at least 8 k-blocks each.
    if (n_tiles * 2 >= sms && n_tiles <= sms) {
      p->sk_grid = n_tiles;
    } else {
      int g = p->sk_total / min_stages;
      g = g < 1 ? 1 : g;
      p->sk_grid = g < sms ? g : sms;
    }
    if (const char* f = getenv("GEMM_EPI_SKINNY_GRID")) {  // tuning override
      const int v = atoi(f);
      if (v >= 1 && v <= p->sk_total && (int64_t)(p->sk_total + 1) * v < (int64_t(1) << 31)) p->sk_grid = v;
    }
    if (const char* f = getenv("GEMM_EPI_SKINNY_PREFETCH")) p->sk_prefetch = atoi(f) > 0 ? atoi(f) : 0;
    p->sk_max_segs = 1;
    for (int t = 0; t < n_tiles; ++t) {
      const int64_t first = ge::skinny_owner((int64_t)t * p->sk_kbt, p->sk_grid, p->sk_total);
      const int64_t last = ge::skinny_owner((int64_t)(t + 1) * p->sk_kbt - 1, p->sk_grid, p->sk_total);
      if (last - first + 1 > p->sk_max_segs) p->sk_max_segs = (int)(last - first + 1);
    }
    e = cudaFuncSetAttribute(p->sk.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p->sk.smem);
    if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)"));
    if (p->sk_max_segs > 1) {
      p->sk_bytes = (size_t)n_tiles * p->sk_max_segs * p->sk.TP * 128 * sizeof(float);
      e = cudaMalloc((void**)&p->sk_partials, p->sk_bytes);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMalloc(split-tile partials)"));
      e = cudaMalloc((void**)&p->sk_tickets, sizeof(int) * (size_t)n_tiles);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMalloc(tickets)"));
      e = cudaMemset(p->sk_tickets, 0, sizeof(int) * (size_t)n_tiles);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMemset(tickets)"));
      p->sk_bytes += sizeof(int) * (size_t)n_tiles;
    }
  }
  e = cudaHostAlloc((void**)&p->status_host, sizeof(int), cudaHostAllocMapped);
  if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaHostAlloc(status word)"));
  *p->status_host = 0;
  e = cudaHostGetDevicePointer((void**)&p->status_dev, p->status_host, 0);
  if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaHostGetDevicePointer(status word)"));
  // the column partials are needed by the fused and the unfused backward
  p->partial_bytes = (size_t)p->m_tiles * (size_t)N * sizeof(float);
  if (epilog == GEMM_EPI_DRELU_BGRAD) {
    if (test_hook("GEMM_EPI_INJECT_PLAN_ALLOC_FAILURE"))
      return cleanup(fail(GEMM_EPI_ERR_CUDA, "injected workspace allocation failure"));
    e = cudaMalloc((void**)&p->partials, p->partial_bytes);
    if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMalloc(workspace)"));
    if (p->kernel != 1) {  // the tile kernels finish dbias themselves (last ticket per column block)
      p->n_tickets = p->kernel == 2 ? 2 * p->n_tiles : p->n_tiles;  // pair kernel: 128-column half blocks
      e = cudaMalloc((void**)&p->col_tickets, sizeof(int) * (size_t)p->n_tickets);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMalloc(column tickets)"));
      e = cudaMemset(p->col_tickets, 0, sizeof(int) * (size_t)p->n_tickets);
      if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMemset(column tickets)"));
    }
  } else if (epilog == GEMM_EPI_WGRAD) {  // partials of the optional bias gradient (sum of X over its rows)
    p->partial_bytes = (size_t)ceil_div(p->uT, 128) * (size_t)p->uK * sizeof(float);
    e = cudaMalloc((void**)&p->partials, p->partial_bytes);
    if (e != cudaSuccess) return cleanup(cuda_fail(e, "cudaMalloc(workspace)"));
  }
  if (const char* f = getenv("GEMM_EPI_CACHE_HINTS")) p->cache_hints = atoi(f) != 0;  // A/B override
  {
    std::lock_guard<std::mutex> g(g_mu);
    live_plans().insert(p);
  }
  g_last_error.clear();
  return p;
}

void gemm_epi_free(gemm_epi_plan_t plan) {
  if (!plan) return;
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (!live_plans().erase(plan)) {
      g_last_error = "gemm_epi_free: not a live plan (ignored)";
      return;
    }
  }
  if (plan->partials) cudaFree(plan->partials);
  if (plan->col_tickets) cudaFree(plan->col_tickets);
  if (plan->pair_slots) cudaFree(plan->pair_slots);
  if (plan->pair_flags) cudaFree(plan->pair_flags);
  if (plan->sk_partials) cudaFree(plan->sk_partials);
  if (plan->sk_tickets) cudaFree(plan->sk_tickets);
  if (plan->status_host) cudaFreeHost(plan->status_host);
  delete plan;
}

const char* gemm_epi_last_error(void) { return g_last_error.c_str(); }

int gemm_epi_query(gemm_epi_plan_t plan, gemm_epi_info* info) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p || !info) return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_query: unknown plan or NULL info");
  memset(info, 0, sizeof(*info));
  info->T = p->uT;
  info->N = p->N;
  info->K = p->uK;
  info->dtype = p->dtype;
  info->epilog = p->epilog;
  info->kernel = p->kernel;
  info->num_sms = p->num_sms;
  if (p->kernel == 1) {
    info->tile_m = 128;  // features per tile (the MMA's M)
    info->tile_n = p->sk.TP;  // padded rows (the MMA's N)
    info->tile_k = ge::kBK * p->sk.KPS;  // k per pipeline stage
    info->stages = p->sk.stages;
    info->split_k = p->sk_max_segs;
    info->grid = p->sk_grid;
    info->launches = 1;
    info->workspace_bytes = p->sk_bytes + (p->epilog == GEMM_EPI_DRELU_BGRAD ? p->partial_bytes : 0);
  } else {
    info->tile_m = p->kernel == 2 ? 2 * ge::kBM : ge::kBM;
    info->tile_n = p->cfg.BN;
    info->tile_k = ge::kBK;
    info->stages = p->cfg.stages;
    info->split_k = p->pair_split ? p->pair_max_segs : 1;
    info->grid = p->grid;
    info->launches = 1;
    info->workspace_bytes = p->pair_bytes +
                            (p->epilog == GEMM_EPI_DRELU_BGRAD ? p->partial_bytes + sizeof(int) * (size_t)p->n_tickets
                             : p->epilog == GEMM_EPI_WGRAD     ? p->partial_bytes
                                                               : 0);
  }
  return GEMM_EPI_OK;
}

int gemm_epi_status(gemm_epi_plan_t plan) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p) return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_status: unknown plan");
  return take_status(p);
}

int gemm_epi_execute(gemm_epi_plan_t plan, const void* X, const void* W, const void* bias, void* Y, uint32_t* aux,
                     cudaStream_t stream) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p) return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_execute: unknown plan");
  if (p->epilog == GEMM_EPI_DRELU_BGRAD || p->epilog == GEMM_EPI_WGRAD)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "gemm_epi_execute called on a %s plan",
                p->epilog == GEMM_EPI_WGRAD ? "WGRAD" : "DRELU_BGRAD");
  if (!X || !W || !Y || (!bias && p->epilog != GEMM_EPI_NONE))
    return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_execute: NULL X, W, bias or Y");
  const bool gelu_aux = p->epilog == GEMM_EPI_GELU_AUX_BIAS;
  if ((p->epilog == GEMM_EPI_RELU_AUX_BIAS || gelu_aux) && !aux)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "%s needs an aux buffer", gelu_aux ? "GELU_AUX_BIAS" : "RELU_AUX_BIAS");
  if (!aligned(X, 16) || !aligned(W, 16) || !aligned(Y, 16) || !aligned(bias, p->bias_f32 ? 4 : 2) ||
      (p->epilog == GEMM_EPI_RELU_AUX_BIAS && !aligned(aux, 4)) || (gelu_aux && !aligned(aux, 16)))
    return fail(GEMM_EPI_ERR_MISALIGNED,
                "gemm_epi_execute: X, W, Y need 16-byte, bias 2-byte, aux 4-byte (GELU_AUX_BIAS: 16-byte) alignment");
  int rc = take_status(p);
  if (rc) return rc;
  if (p->kernel == 1) {
    rc = prepare_skinny_maps(p, X, W);
    if (rc) return rc;
    ge::SkinnyParams k = skinny_params(p);
    k.bias = bias;
    k.out = Y;
    k.aux_out = aux;
    return launch_skinny(p, k, stream);
  }
  rc = prepare_maps(p, X, W);
  if (rc) return rc;
  ge::TileParams k = base_params(p);
  k.bias = bias;
  k.out = Y;
  k.aux_out = aux;
  return launch_tile(p, p->cfg, k, stream);
}

int drelu_bgrad_execute(gemm_epi_plan_t plan, const void* dY2, const void* W2, const uint32_t* aux, void* dZ,
                        float* dbias, cudaStream_t stream) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p) return fail(GEMM_EPI_ERR_INVALID_ARG, "drelu_bgrad_execute: unknown plan");
  if (p->epilog != GEMM_EPI_DRELU_BGRAD)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "drelu_bgrad_execute called on a forward plan");
  if (!dY2 || !W2 || !aux || !dZ || !dbias)
    return fail(GEMM_EPI_ERR_INVALID_ARG, "drelu_bgrad_execute: NULL dY2, W2, aux, dZ or dbias");
  if (!aligned(dY2, 16) || !aligned(W2, 16) || !aligned(dZ, 16) || !aligned(aux, 4) || !aligned(dbias, 4))
    return fail(GEMM_EPI_ERR_MISALIGNED,
                "drelu_bgrad_execute: dY2, W2, dZ need 16-byte, aux and dbias 4-byte alignment");
  int rc = take_status(p);
  if (rc) return rc;
  if (p->kernel == 1) {
    rc = prepare_skinny_maps(p, dY2, W2);
    if (rc) return rc;
    ge::SkinnyParams k = skinny_params(p);
    k.out = dZ;
    k.aux_in = aux;
    k.dbias = dbias;
    return launch_skinny(p, k, stream);
  }
  rc = prepare_maps(p, dY2, W2);
  if (rc) return rc;
  ge::TileParams k = base_params(p);
  k.out = dZ;
  k.aux_in = aux;
  k.partials = p->partials;
  k.col_tickets = p->col_tickets;
  k.dbias = dbias;
  return launch_tile(p, p->cfg, k, stream);
}

int gemm_epi_unfused_execute(gemm_epi_plan_t plan, const void* X, const void* W, const void* bias, void* T1, void* T2,
                             void* Y, uint32_t* aux, cudaStream_t stream) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p) return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_unfused_execute: unknown plan");
  if (p->epilog == GEMM_EPI_DRELU_BGRAD || p->epilog == GEMM_EPI_WGRAD || p->epilog == GEMM_EPI_NONE)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "gemm_epi_unfused_execute: the plan's epilog has nothing to unfuse");
  if (p->out_f32)
    return fail(GEMM_EPI_ERR_UNSUPPORTED, "the unfused path keeps 16-bit intermediates and outputs (no fp32 output)");
  const bool gelu_aux = p->epilog == GEMM_EPI_GELU_AUX_BIAS;
  if ((p->epilog == GEMM_EPI_RELU_AUX_BIAS || gelu_aux) && !aux)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "%s needs an aux buffer", gelu_aux ? "GELU_AUX_BIAS" : "RELU_AUX_BIAS");
  if (gelu_aux) T2 = aux;  // the bias kernel's output is the auxiliary output Z itself
  if (!X || !W || !bias || !T1 || !T2 || !Y) return fail(GEMM_EPI_ERR_INVALID_ARG, "unfused: NULL pointer");
  if (!aligned(X, 16) || !aligned(W, 16) || !aligned(T1, 16) || !aligned(T2, 16) || !aligned(Y, 16) ||
      !aligned(bias, p->bias_f32 ? 4 : 2) || (aux && !aligned(aux, 4)))
    return fail(GEMM_EPI_ERR_MISALIGNED, "unfused: misaligned pointer");
  int rc = take_status(p);
  if (rc) return rc;
  rc = prepare_maps(p, X, W);
  if (rc) return rc;
  ge::TileParams k = base_params(p);
  k.out = T1;
  rc = launch_tile(p, p->cfg_store, k, stream);
  if (rc) return rc;
  const bool bf16 = p->dtype == GEMM_EPI_BF16;
  const int blocks = p->num_sms * 8;
  if (bf16)
    ge::bias_add_kernel<true><<<blocks, 256, 0, stream>>>((const uint4*)T1, bias, (uint4*)T2, p->T, (int)p->N,
                                                          p->bias_f32);
  else
    ge::bias_add_kernel<false><<<blocks, 256, 0, stream>>>((const uint4*)T1, bias, (uint4*)T2, p->T, (int)p->N,
                                                           p->bias_f32);
  if (p->epilog == GEMM_EPI_GELU_BIAS || gelu_aux) {
    const int64_t n_vec = p->T * p->N / 8;
    if (bf16)
      ge::gelu_kernel<true><<<blocks, 256, 0, stream>>>((const uint4*)T2, (uint4*)Y, n_vec);
    else
      ge::gelu_kernel<false><<<blocks, 256, 0, stream>>>((const uint4*)T2, (uint4*)Y, n_vec);
  } else if (p->epilog != GEMM_EPI_BIAS) {
    const bool want_aux = p->epilog == GEMM_EPI_RELU_AUX_BIAS;
    auto* in = (const uint16_t*)T2;
    auto* out = (uint16_t*)Y;
    if (bf16) {
      if (want_aux)
        ge::relu_mask_kernel<true, true><<<blocks, 256, 0, stream>>>(in, out, aux, p->T, (int)p->N, p->aux_words);
      else
        ge::relu_mask_kernel<true, false><<<blocks, 256, 0, stream>>>(in, out, aux, p->T, (int)p->N, p->aux_words);
    } else {
      if (want_aux)
        ge::relu_mask_kernel<false, true><<<blocks, 256, 0, stream>>>(in, out, aux, p->T, (int)p->N, p->aux_words);
      else
        ge::relu_mask_kernel<false, false><<<blocks, 256, 0, stream>>>(in, out, aux, p->T, (int)p->N, p->aux_words);
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "unfused elementwise launch");
  return GEMM_EPI_OK;
}

int gemm_epi_set_bias_f32(gemm_epi_plan_t plan, int bias_f32) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p) return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_set_bias_f32: unknown plan");
  if (p->epilog == GEMM_EPI_DRELU_BGRAD || p->epilog == GEMM_EPI_WGRAD)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "gemm_epi_set_bias_f32: only forward plans take a bias");
  p->bias_f32 = bias_f32 ? 1 : 0;
  return GEMM_EPI_OK;
}

int gemm_epi_wgrad_execute(gemm_epi_plan_t plan, const void* X, const void* dZ, void* dW, float* dbias,
                           cudaStream_t stream) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p) return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_wgrad_execute: unknown plan");
  if (p->epilog != GEMM_EPI_WGRAD)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "gemm_epi_wgrad_execute called on a plan whose epilog is not WGRAD");
  if (!X || !dZ || !dW) return fail(GEMM_EPI_ERR_INVALID_ARG, "gemm_epi_wgrad_execute: NULL X, dZ or dW");
  if (!aligned(X, 16) || !aligned(dZ, 16) || !aligned(dW, 16) || (dbias && !aligned(dbias, 4)))
    return fail(GEMM_EPI_ERR_MISALIGNED, "gemm_epi_wgrad_execute: X, dZ, dW need 16-byte, dbias 4-byte alignment");
  int rc = take_status(p);
  if (rc) return rc;
  rc = prepare_maps(p, X, dZ);
  if (rc) return rc;
  ge::TileParams k = base_params(p);
  k.out = dW;
  rc = launch_tile(p, p->cfg, k, stream);
  if (rc || !dbias) return rc;
  // dbias[k] = sum over the uT rows of X[t][k]: per-128-row partials, then a fixed-order sum
  const int row_blocks = ceil_div(p->uT, 128);
  dim3 cgrid(ceil_div(p->uK, 256), row_blocks);
  if (p->dtype == GEMM_EPI_BF16)
    ge::colsum_partial_kernel<true><<<cgrid, 256, 0, stream>>>((const uint16_t*)X, p->uT, (int)p->uK, p->partials);
  else
    ge::colsum_partial_kernel<false><<<cgrid, 256, 0, stream>>>((const uint16_t*)X, p->uT, (int)p->uK, p->partials);
  ge::dbias_finish_kernel<<<ceil_div(p->uK, 256), 256, 0, stream>>>(p->partials, row_blocks, (int)p->uK, dbias);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wgrad bias-gradient launch");
  return GEMM_EPI_OK;
}

int drelu_bgrad_unfused_execute(gemm_epi_plan_t plan, const void* dY2, const void* W2, const uint32_t* aux, void* G,
                                void* dZ, float* dbias, cudaStream_t stream) {
  gemm_epi_plan_s* p = lookup(plan);
  if (!p) return fail(GEMM_EPI_ERR_INVALID_ARG, "drelu_bgrad_unfused_execute: unknown plan");
  if (p->epilog != GEMM_EPI_DRELU_BGRAD)
    return fail(GEMM_EPI_ERR_EPILOG_MISMATCH, "drelu_bgrad_unfused_execute called on a forward plan");
  if (p->out_f32)
    return fail(GEMM_EPI_ERR_UNSUPPORTED, "the unfused path keeps 16-bit intermediates and outputs (no fp32 output)");
  if (!dY2 || !W2 || !aux || !G || !dZ || !dbias) return fail(GEMM_EPI_ERR_INVALID_ARG, "unfused: NULL pointer");
  if (!aligned(dY2, 16) || !aligned(W2, 16) || !aligned(G, 16) || !aligned(dZ, 16) || !aligned(aux, 4) ||
      !aligned(dbias, 4))
    return fail(GEMM_EPI_ERR_MISALIGNED, "unfused: misaligned pointer");
  int rc = take_status(p);
  if (rc) return rc;
  rc = prepare_maps(p, dY2, W2);
  if (rc) return rc;
  ge::TileParams k = base_params(p);
  k.out = G;
  rc = launch_tile(p, p->cfg_store, k, stream);
  if (rc) return rc;
  const int blocks = p->num_sms * 8;
  const bool bf16 = p->dtype == GEMM_EPI_BF16;
  if (bf16)
    ge::mask_apply_kernel<true><<<blocks, 256, 0, stream>>>((const uint16_t*)G, aux, (uint16_t*)dZ, p->T, (int)p->N,
                                                             p->aux_words);
  else
    ge::mask_apply_kernel<false><<<blocks, 256, 0, stream>>>((const uint16_t*)G, aux, (uint16_t*)dZ, p->T, (int)p->N,
                                                              p->aux_words);
  dim3 cgrid(ceil_div(p->N, 256), p->m_tiles);
  if (bf16)
    ge::colsum_partial_kernel<true><<<cgrid, 256, 0, stream>>>((const uint16_t*)dZ, p->T, (int)p->N, p->partials);
  else
    ge::colsum_partial_kernel<false><<<cgrid, 256, 0, stream>>>((const uint16_t*)dZ, p->T, (int)p->N, p->partials);
  ge::dbias_finish_kernel<<<ceil_div(p->N, 256), 256, 0, stream>>>(p->partials, p->m_tiles, (int)p->N, dbias);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "unfused backward launch");
  return GEMM_EPI_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free DRELU_BGRAD (drelu_bgrad_execute_noalloc).
//
// For callers that may not allocate device memory: the column partials and
// the watchdog word live in this fixed, file-scope device array instead of a
// plan's workspace. In host code `g_noalloc_scratch` only names the symbol;
// its device address comes from cudaGetSymbolAddress, looked up once per
// device (with that device current) on the first call there.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocStatusBytes = 256;  // status word, padded to keep the partials 256-byte aligned
constexpr size_t kNoAllocPartialBytes = GEMM_EPI_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocStatusBytes + kNoAllocPartialBytes];

constexpr int kNoAllocMaxDevices = 64;

struct NoAllocDevice {
  std::mutex mu;
  bool ready = false;                // set only once the set-up below succeeded
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

// dbias[n] = sum of partials over row tiles, ascending; NaN everywhere if
// the tile kernel's watchdog fired during this call.
__global__ void noalloc_dbias_finish_kernel(const float* __restrict__ partials, int m_tiles, int N,
                                            float* __restrict__ dbias, const int* __restrict__ status) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  if (*reinterpret_cast<const volatile int*>(status) != 0) {
    dbias[n] = __int_as_float(0x7fc00000);
    return;
  }
  float s = 0.f;
  for (int m = 0; m < m_tiles; ++m) s += partials[static_cast<int64_t>(m) * N + n];
  dbias[n] = s;
}

// Once per device, with that device current: the scratch array's device
// address and the kernels' shared-memory limit. A failed attempt (for
// instance one made during a stream capture) leaves the device not ready, so
// the next call tries again.
int noalloc_setup(int dev, NoAllocDevice*& out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(GEMM_EPI_ERR_UNSUPPORTED, "device index %d out of range", dev);
  NoAllocDevice& d = g_noalloc_dev[dev];
  std::lock_guard<std::mutex> g(d.mu);
  if (!d.ready) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    for (int bn : {64, 128, 256}) {
      for (bool bf16 : {false, true}) {
        TileCfg c = tile_cfg(bn, ge::EPI_DRELU_BGRAD, bf16, false);
        e = cudaFuncSetAttribute(c.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)c.smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
      }
    }
    d.scratch = static_cast<unsigned char*>(p);
    d.ready = true;
  }
  out = &d;
  return GEMM_EPI_OK;
}

}  // namespace

extern "C" int drelu_bgrad_execute_noalloc(int64_t T, int64_t N, int64_t K, gemm_epi_dtype dtype, const void* dY2,
                                           const void* W2, const uint32_t* aux, void* dZ, float* dbias,
                                           cudaStream_t stream) {
  if (T < 1 || N < 8 || K < 8 || (N % 8) != 0 || (K % 8) != 0 || T > ((int64_t)1 << 30) || N > ((int64_t)1 << 24) ||
      K > ((int64_t)1 << 24))
    return fail(GEMM_EPI_ERR_INVALID_ARG, "bad shape T=%lld N=%lld K=%lld (need T>=1, N,K>=8 and multiples of 8)",
                (long long)T, (long long)N, (long long)K);
  if (dtype != GEMM_EPI_F16 && dtype != GEMM_EPI_BF16)
    return fail(GEMM_EPI_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  const int64_t m_tiles = (T + ge::kBM - 1) / ge::kBM;
  const uint64_t need = (uint64_t)m_tiles * (uint64_t)N * sizeof(float);
  if (need > kNoAllocPartialBytes)
    return fail(GEMM_EPI_ERR_INVALID_ARG,
                "drelu_bgrad_execute_noalloc: T=%lld, N=%lld needs %llu bytes of column partials, more than its "
                "fixed %u-byte scratch (ceil(T/128) * N * 4 must fit); use a plan instead",
                (long long)T, (long long)N, (unsigned long long)need, (unsigned)kNoAllocPartialBytes);
  if (!dY2 || !W2 || !aux || !dZ || !dbias)
    return fail(GEMM_EPI_ERR_INVALID_ARG, "drelu_bgrad_execute_noalloc: NULL dY2, W2, aux, dZ or dbias");
  if (!aligned(dY2, 16) || !aligned(W2, 16) || !aligned(dZ, 16) || !aligned(aux, 4) || !aligned(dbias, 4))
    return fail(GEMM_EPI_ERR_MISALIGNED,
                "drelu_bgrad_execute_noalloc: dY2, W2, dZ need 16-byte, aux and dbias 4-byte alignment");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || minor != 0)
    return fail(GEMM_EPI_ERR_UNSUPPORTED, "device %d has compute capability %d.%d; this library needs 10.0", dev,
                major, minor);
  NoAllocDevice* nd = nullptr;
  int rc = noalloc_setup(dev, nd);
  if (rc) return rc;
  int* status = reinterpret_cast<int*>(nd->scratch);
  float* partials = reinterpret_cast<float*>(nd->scratch + kNoAllocStatusBytes);

  const int bn = choose_bn(T, N, K, sms);
  const TileCfg cfg = tile_cfg(bn, ge::EPI_DRELU_BGRAD, dtype == GEMM_EPI_BF16, false);
  CUtensorMap tmA, tmB, tmY;
  rc = encode_2d(&tmA, dY2, (uint64_t)K, (uint64_t)T, ge::kBK, ge::kBM, "dY2");
  if (rc) return rc;
  rc = encode_2d(&tmB, W2, (uint64_t)N, (uint64_t)K, 64, ge::kBK, "W2");
  if (rc) return rc;
  rc = encode_out(&tmY, dZ, T, N);
  if (rc) return rc;

  ge::TileParams k{};
  k.T = (int32_t)T;
  k.N = (int32_t)N;
  k.K = (int32_t)K;
  k.m_tiles = (int32_t)m_tiles;
  k.n_tiles = ceil_div(N, bn);
  k.k_blocks = ceil_div(K, ge::kBK);
  k.num_tiles = k.m_tiles * k.n_tiles;
  k.aux_words = ceil_div(N, 32);
  const Raster raster = choose_raster(T, N, K, ge::kBM, bn);
  k.group_m = raster.group;
  k.raster_n = raster.by_n;
  k.out = dZ;
  k.aux_in = aux;
  k.partials = partials;
  k.status = status;
  const WatchdogEnv wd = watchdog_env();  // the same limit (and test hook) as a plan's
  k.timeout_ns = wd.timeout_ns;
  k.inject_stall = wd.inject_stall;
  const int grid = k.num_tiles < sms ? k.num_tiles : sms;

  // the status word must start each call at zero; the partials are fully
  // rewritten by the tile kernel before the finishing kernel reads them
  e = cudaMemsetAsync(status, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  cfg.fn<<<grid, ge::kThreads, cfg.smem, stream>>>(tmA, tmB, tmY, tmY, k);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "tile kernel launch");
  noalloc_dbias_finish_kernel<<<ceil_div(N, 256), 256, 0, stream>>>(partials, k.m_tiles, (int)N, dbias, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "dbias finish launch");
  return GEMM_EPI_OK;
}
