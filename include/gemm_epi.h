/*
 * gemm_epi.h -- C ABI of the fused linear-layer GEMM + epilogue library for
 * NVIDIA B200 (sm_100a).
 *
 * The library mirrors the plan / execute / free life cycle of the pages'
 * stateful matmul object ("Fusing bias addition into matrix multiplication
 * with nvmath-python", life-cycle and stream items of its checklist;
 * "nvmath-python cuBLASLt bindings for PyTorch fusion", the three-step
 * init / plan / execute pattern): a plan fixes the shape, the 16-bit type and
 * the epilog once, and is then executed any number of times.
 *
 * Layouts (all row-major, every 16-bit tensor of a call has the plan's dtype):
 *   X     T x K      activations                 (K contiguous)
 *   W     K x N      weight                      (N contiguous)
 *   bias  N          one value per output feature, broadcast over the T rows
 *   Y     T x N      output
 *   aux   T x ceil(N/32) uint32 ReLU mask words: bit (n % 32) of word
 *         [t][n / 32] is 1 iff the pre-activation Z[t][n] > 0 (strictly),
 *         least significant bit first; bits past N are 0.
 *   dY2   T x K      gradient input of the backward product (K plays D2)
 *   W2    K x N      second operand of the backward product
 *   dZ    T x N      masked gradient
 *   dbias N          fp32 bias gradient
 *
 * Arithmetic: products accumulate in fp32 (tensor cores, fp32 accumulators in
 * tensor memory); the bias is converted to fp32 and added; outputs are rounded
 * to the 16-bit type with round-to-nearest-even.
 *
 * Streams and ownership: every execute call is asynchronous on the caller's
 * stream and never synchronises (the pages' execute is non-blocking; the
 * caller synchronises before reading results). The caller owns every tensor.
 * A plan owns only its workspace and host state, allocated by gemm_epi_plan
 * and released by gemm_epi_free; execute calls allocate nothing. One plan
 * must not run concurrently on two streams (its workspace is shared).
 *
 * Errors: functions return GEMM_EPI_OK (0) or a negative code; a message is
 * kept per thread and read with gemm_epi_last_error(). Argument errors are
 * detected before anything is launched.
 *
 * Environment variables, read when a plan is created (and by every call of
 * drelu_bgrad_execute_noalloc); none is needed in normal use:
 *   GEMM_EPI_WAIT_TIMEOUT_MS      limit of each bounded wait inside a kernel
 *                                 (default 2000 ms; see GEMM_EPI_ERR_TIMEOUT)
 *   tuning overrides of the plan's choices, for measurement and tests:
 *   GEMM_EPI_FORCE_KERNEL=tile|pair|skinny, GEMM_EPI_FORCE_BN=64|128|192|256,
 *   GEMM_EPI_RASTER=m|n, GEMM_EPI_GROUP_M, GEMM_EPI_SKINNY_GRID, GEMM_EPI_SKINNY_KPS=1|2,
 *   GEMM_EPI_SKINNY_PREFETCH, GEMM_EPI_TAIL_SPLIT=0|1, GEMM_EPI_CACHE_HINTS=0|1,
 *   GEMM_EPI_PAIR_SPLIT=0|1 (stream-K CTA pairs; off by default),
 *   GEMM_EPI_PAIR_SK_FIRST=0|1 (with stream-K: its tiles before the whole tiles, the
 *   default, or after them)
 *   fault injection for the library's own tests, honoured only while
 *   GEMM_EPI_TEST_HOOKS=1 is also set: GEMM_EPI_INJECT_STALL (a kernel
 *   withholds its first tile's completion signal, so its watchdog fires),
 *   GEMM_EPI_INJECT_ENCODE_FAILURE (every tensor-map encode fails),
 *   GEMM_EPI_INJECT_PLAN_ALLOC_FAILURE (the DRELU_BGRAD workspace
 *   allocation fails).
 */
#ifndef GEMM_EPI_H
#define GEMM_EPI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GEMM_EPI_API __attribute__((visibility("default")))
#else
#define GEMM_EPI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA runtime stream handle (same type as cuda_runtime_api.h's). */
typedef struct CUstream_st* cudaStream_t;

typedef enum { GEMM_EPI_F16 = 0, GEMM_EPI_BF16 = 1 } gemm_epi_dtype;

/* The pages' epilog names ("Fusing bias addition into matrix multiplication
 * with nvmath-python": BIAS, RELU_BIAS, RELU_AUX_BIAS; "nvmath-python fused
 * epilogs for linear layers": DRELU_BGRAD; "nvmath-python cuBLASLt bindings
 * for PyTorch fusion", its list of predefined epilogs: GELU_BIAS, bias then
 * GELU). The pages do not say which GELU; this library computes the
 * definition GELU(z) = z * Phi(z) = 0.5 * z * (1 + erf(z / sqrt(2))) in fp32
 * with CUDA's erff, not the tanh approximation. */
typedef enum {
  GEMM_EPI_BIAS = 0,          /* Y = X.W + bias                              */
  GEMM_EPI_RELU_BIAS = 1,     /* Y = relu(X.W + bias)                        */
  GEMM_EPI_RELU_AUX_BIAS = 2, /* Y = relu(X.W + bias), aux = mask (Z > 0)    */
  GEMM_EPI_DRELU_BGRAD = 3,   /* dZ = (dY2.W2) masked by aux, dbias = sum_t dZ */
  GEMM_EPI_GELU_BIAS = 4,     /* Y = gelu(X.W + bias); aux is ignored         */
  GEMM_EPI_WGRAD = 5,         /* dW = X^T . dZ, see gemm_epi_wgrad_execute    */
  GEMM_EPI_NONE = 6,          /* Y = X.W, no bias (may be NULL) or activation */
  GEMM_EPI_GELU_AUX_BIAS = 7  /* Y = gelu(Z), aux = Z = X.W + bias (16-bit)   */
} gemm_epi_epilog;

/* GELU_AUX_BIAS is to GELU_BIAS what RELU_AUX_BIAS is to RELU_BIAS: it also
 * returns what the backward pass of the activation needs. The pages define
 * that auxiliary output only for ReLU (the mask); GELU's derivative depends
 * on the pre-activation itself, not only on its sign, so this library
 * returns Z = X.W + bias, rounded to the plan's 16-bit type (round to
 * nearest even), T x N row-major in the aux buffer. */

enum {
  GEMM_EPI_OK = 0,
  GEMM_EPI_ERR_INVALID_ARG = -1,     /* bad dimension, enum, NULL pointer or unknown plan */
  GEMM_EPI_ERR_MISALIGNED = -2,      /* a pointer is not aligned as required below        */
  GEMM_EPI_ERR_EPILOG_MISMATCH = -3, /* call does not fit the plan's epilog              */
  GEMM_EPI_ERR_CUDA = -4,            /* CUDA runtime / driver error (message kept)        */
  GEMM_EPI_ERR_TIMEOUT = -5,         /* a kernel's bounded wait expired (watchdog)        */
  GEMM_EPI_ERR_UNSUPPORTED = -6      /* no device of compute capability 10.0             */
};

typedef struct gemm_epi_plan_s* gemm_epi_plan_t;

/* What a plan chose, for logs and tests. */
typedef struct {
  int64_t T, N, K;
  int dtype, epilog;
  int kernel;          /* 0 = tile kernel (one CTA per tile), 1 = few-row kernel (swap-AB,
                          stream-K), 2 = tile kernel on CTA pairs (256-row tiles) */
  int tile_m, tile_n, tile_k, stages;
  int split_k;         /* K slices per output tile (1 = none) */
  int grid;            /* CTAs launched by the main kernel */
  int launches;        /* kernel launches per execute call */
  int num_sms;
  size_t workspace_bytes;
} gemm_epi_info;

/*
 * gemm_epi_plan: validate a problem and choose its kernel configuration.
 *   T >= 1 rows; N >= 8 and K >= 8, both multiples of 8 (16-byte row
 *   strides); dtype and epilog from the enums above. For DRELU_BGRAD, K is
 *   the contraction length D2 of G = dY2 . W2 (a backward plan is separate
 *   from the forward plan, as the pages build a separate matmul for it). For
 *   WGRAD, (T, N, K) are the forward's: dW is K x N, summed over T (any T).
 *   Uses the current CUDA device; allocates the plan's workspace there.
 * Returns a plan, or NULL with gemm_epi_last_error() set.
 */
GEMM_EPI_API gemm_epi_plan_t gemm_epi_plan(int64_t T, int64_t N, int64_t K, gemm_epi_dtype dtype,
                              gemm_epi_epilog epilog);

/* Flags of gemm_epi_plan_ex. */
enum { GEMM_EPI_FLAG_W_NK = 1u, GEMM_EPI_FLAG_OUT_F32 = 2u };

/*
 * gemm_epi_plan_ex: gemm_epi_plan with flags (gemm_epi_plan passes 0).
 *   GEMM_EPI_FLAG_W_NK: the weight operand -- W of a forward plan, W2 of a
 *   DRELU_BGRAD plan -- is given N x K row-major (K contiguous: the
 *   [out_features, in_features] layout of a framework's linear layer)
 *   instead of K x N. Chaining two layers needs both orientations of one
 *   weight (the forward reads it as N x K, the backward through it as
 *   K x N); with this flag neither has to be transposed in memory. Such plans
 *   run on the one-CTA or CTA-pair kernels, never the few-row kernel. Not
 *   valid for WGRAD plans.
 *   GEMM_EPI_FLAG_OUT_F32: the output -- Y, dZ or dW -- is written as fp32
 *   (the accumulator, not rounded; 16-byte aligned) while the operands stay
 *   16-bit ("Fusing bias addition into matrix multiplication with
 *   nvmath-python", engineering checklist: operand and result types need
 *   only be compatible). The mask words and dbias are unchanged. The unfused
 *   entry points return GEMM_EPI_ERR_UNSUPPORTED on such a plan.
 * Returns a plan, or NULL with gemm_epi_last_error() set (unknown flags:
 * GEMM_EPI_ERR_INVALID_ARG).
 */
GEMM_EPI_API gemm_epi_plan_t gemm_epi_plan_ex(int64_t T, int64_t N, int64_t K, gemm_epi_dtype dtype,
                                              gemm_epi_epilog epilog, uint32_t flags);

/*
 * gemm_epi_execute: the forward epilogs (BIAS, RELU_BIAS, RELU_AUX_BIAS,
 * GELU_BIAS, GELU_AUX_BIAS) and the plain product (NONE).
 *   X, W, Y: device pointers, 16-byte aligned (W is K x N, or N x K with
 *   GEMM_EPI_FLAG_W_NK; Y is fp32 with GEMM_EPI_FLAG_OUT_F32). bias: device
 *   pointer, 2-byte aligned (4-byte for an fp32 bias, gemm_epi_set_bias_f32),
 *   never NULL except for NONE, where it is ignored. aux: device pointer,
 *   required for RELU_AUX_BIAS (the mask words, 4-byte aligned) and for
 *   GELU_AUX_BIAS (T x N values of the plan's 16-bit type even with
 *   GEMM_EPI_FLAG_OUT_F32, 16-byte aligned; pass it cast to uint32_t*), and
 *   ignored (may be NULL) otherwise.
 * Returns GEMM_EPI_OK once the work is enqueued on `stream`;
 * GEMM_EPI_ERR_EPILOG_MISMATCH on a DRELU_BGRAD or WGRAD plan or a missing
 * aux; GEMM_EPI_ERR_MISALIGNED for a misaligned pointer; GEMM_EPI_ERR_CUDA if
 * a tensor map cannot be encoded or the launch fails (nothing is launched
 * then); GEMM_EPI_ERR_TIMEOUT if an earlier call on this plan reported a
 * watchdog expiry (the report is cleared by reading it).
 */
GEMM_EPI_API int gemm_epi_execute(gemm_epi_plan_t plan, const void* X, const void* W, const void* bias, void* Y,
                     uint32_t* aux, cudaStream_t stream);

/*
 * drelu_bgrad_execute: DRELU_BGRAD ("nvmath-python fused epilogs for linear
 * layers", DRELU_BGRAD section): G = dY2 . W2, dZ = G where the mask bit of
 * aux is set, else 0 (rounded to dtype), and dbias[n] = sum over t of the
 * fp32 masked G, reduced in a fixed order (bitwise reproducible).
 *   dY2 (T x K), W2 (K x N), dZ (T x N): device, 16-byte aligned.
 *   aux: device, 4-byte aligned, the forward's relu_aux (T x ceil(N/32)).
 *   dbias: device, 4-byte aligned, N floats.
 * Returns as gemm_epi_execute; GEMM_EPI_ERR_EPILOG_MISMATCH on a forward plan.
 */
GEMM_EPI_API int drelu_bgrad_execute(gemm_epi_plan_t plan, const void* dY2, const void* W2, const uint32_t* aux,
                        void* dZ, float* dbias, cudaStream_t stream);

/*
 * gemm_epi_set_bias_f32: forward plans only. With bias_f32 != 0, later
 * execute calls of this plan read the bias as N fp32 values (4-byte aligned)
 * instead of the plan's 16-bit type; 0 restores the default. "Fusing bias
 * addition into matrix multiplication with nvmath-python" (engineering
 * checklist, types and device) allows a float32 bias with float16 operands
 * and has the library convert it. The bias is added in fp32 either way.
 * Takes effect for calls enqueued after it returns (host-side state).
 * Returns GEMM_EPI_OK; GEMM_EPI_ERR_INVALID_ARG for an unknown plan;
 * GEMM_EPI_ERR_EPILOG_MISMATCH on a DRELU_BGRAD or WGRAD plan.
 */
GEMM_EPI_API int gemm_epi_set_bias_f32(gemm_epi_plan_t plan, int bias_f32);

/*
 * gemm_epi_wgrad_execute: the weight gradient of the linear layer,
 * dW[k][n] = sum over t of X[t][k] * dZ[t][n], rounded to dtype. The pages
 * name no epilog for it: "nvmath-python fused epilogs for linear layers"
 * (FAQ) says DRELU_BGRAD covers the mask and the bias gradient but not the
 * whole backward pass; this is the remaining product of that pass, with the
 * dZ that drelu_bgrad_execute returns. Plan it with epilog GEMM_EPI_WGRAD and
 * the forward's (T, N, K): the contraction runs over the T rows.
 *   X (T x K), dZ (T x N), dW (K x N): device, 16-byte aligned, row-major.
 *   dbias: NULL, or K floats (4-byte aligned) receiving sum over t of
 *   X[t][k] in fp32, reduced in a fixed order (a second launch in the same
 *   call). With a layer weight in the [out, in] layout, dW = dY^T . H is
 *   called with X = dY, and dbias is then that layer's bias gradient.
 * Returns as gemm_epi_execute; GEMM_EPI_ERR_EPILOG_MISMATCH on a plan whose
 * epilog is not WGRAD (and gemm_epi_execute / drelu_bgrad_execute return it
 * on a WGRAD plan).
 */
GEMM_EPI_API int gemm_epi_wgrad_execute(gemm_epi_plan_t plan, const void* X, const void* dZ, void* dW,
                                        float* dbias, cudaStream_t stream);

/* Release a plan and its workspace. NULL and already-freed plans are
 * ignored. The caller must make sure no work of the plan is still running
 * (synchronise its stream first). */
GEMM_EPI_API void gemm_epi_free(gemm_epi_plan_t plan);

/* The calling thread's last error message ("" if none). */
GEMM_EPI_API const char* gemm_epi_last_error(void);

/* Fill *info with the plan's choices. Returns GEMM_EPI_OK or ERR_INVALID_ARG. */
GEMM_EPI_API int gemm_epi_query(gemm_epi_plan_t plan, gemm_epi_info* info);

/* After the caller synchronised the plan's stream: GEMM_EPI_OK, or
 * GEMM_EPI_ERR_TIMEOUT if a kernel of this plan gave up on a wait (and then
 * left its outputs incomplete). Reading clears the report. */
GEMM_EPI_API int gemm_epi_status(gemm_epi_plan_t plan);

/*
 * Unfused path, for measurement only (the pages' three-kernel baseline,
 * "AI inference compiler optimisation: operator fusion", section 2.2:
 * MatMul writes an intermediate, BiasAdd reads it and writes another, ReLU
 * reads that and writes the output).
 *   gemm_epi_unfused_execute: GEMM -> T1 (T x N, dtype), T1 + bias -> T2,
 *   relu(T2) -> Y (and, for RELU_AUX_BIAS, the mask from T2 > 0 -> aux), or
 *   gelu(T2) -> Y for GELU_BIAS. For GELU_AUX_BIAS the bias kernel writes
 *   into aux (the auxiliary output Z; T2 is ignored and may be NULL), and
 *   gelu(aux) -> Y. For BIAS the activation kernel is skipped and T2 is the
 *   output: pass Y as T2.
 *   drelu_bgrad_unfused_execute: GEMM -> G (dtype), mask apply -> dZ,
 *   column sum of dZ -> dbias (fixed order).
 * T1, T2, G: caller-owned device scratch of T x N dtype, 16-byte aligned.
 * Plans with epilog NONE or WGRAD return GEMM_EPI_ERR_EPILOG_MISMATCH, plans
 * with GEMM_EPI_FLAG_OUT_F32 GEMM_EPI_ERR_UNSUPPORTED (the unfused path
 * keeps 16-bit intermediates).
 */
GEMM_EPI_API int gemm_epi_unfused_execute(gemm_epi_plan_t plan, const void* X, const void* W, const void* bias,
                             void* T1, void* T2, void* Y, uint32_t* aux, cudaStream_t stream);
GEMM_EPI_API int drelu_bgrad_unfused_execute(gemm_epi_plan_t plan, const void* dY2, const void* W2,
                                const uint32_t* aux, void* G, void* dZ, float* dbias,
                                cudaStream_t stream);

/* Capacity of the fixed scratch used by drelu_bgrad_execute_noalloc: the
 * backward needs ceil(T/128) * N floats of column partials. */
#define GEMM_EPI_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * drelu_bgrad_execute_noalloc: the same DRELU_BGRAD computation as
 * drelu_bgrad_execute, for callers that must not allocate device memory.
 * (The pages have no counterpart: this is a deployment variant, not part of
 * the method.)
 *
 * Who needs it: code that runs inside a host that owns all device memory --
 * a framework's caching allocator or an inference engine with a fixed,
 * pre-reserved budget -- where a raw cudaMalloc would bypass its accounting
 * or fail once the pool has claimed the device; and enqueue-time plugin
 * callbacks, which must not call cudaMalloc/cudaFree because those can
 * synchronise the device and stall every other stream. Such callers cannot
 * create a plan (gemm_epi_plan allocates its workspace), so this entry point
 * takes the shape directly and allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library call.
 *
 * Scratch: the column partial sums live in one fixed array of
 * GEMM_EPI_NOALLOC_SCRATCH_BYTES (4 MiB) plus a 256-byte status block, in
 * static device memory of this library; every GPU that loads the library
 * keeps it until the process exits. Shapes whose partials exceed it
 * (ceil(T/128) * N * 4 bytes > 4 MiB, e.g. T = 4096 needs N <= 32768) are
 * rejected with GEMM_EPI_ERR_INVALID_ARG and a message, before any work.
 * All calls share that array: two calls that overlap on the GPU (other
 * streams, other host threads, same device) race on it and corrupt each
 * other's dbias. Serialise them, e.g. on one stream.
 *
 * Arguments: T, N, K (K is D2) and dtype as for gemm_epi_plan with epilog
 * DRELU_BGRAD; the pointers, alignment and layouts as drelu_bgrad_execute.
 * First call on a device: it looks up the scratch array's device address
 * and sets the kernel's shared-memory limit for that device, once; make
 * that first call before any stream capture begins (a set-up that fails is
 * tried again by the next call). Each call clears the status block, then
 * launches two kernels on `stream` and returns without synchronising. The
 * product always runs on the one-CTA tile kernel: at few-row shapes
 * (T <= 256), where a plan picks the few-row kernel, this entry point is
 * slower than drelu_bgrad_execute. Its waits are bounded like a plan's
 * (GEMM_EPI_WAIT_TIMEOUT_MS); if one expires (the watchdog), every dbias
 * entry is written as NaN instead of a sum, and dZ may be incomplete.
 */
GEMM_EPI_API int drelu_bgrad_execute_noalloc(int64_t T, int64_t N, int64_t K, gemm_epi_dtype dtype,
                                             const void* dY2, const void* W2, const uint32_t* aux, void* dZ,
                                             float* dbias, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GEMM_EPI_H */
