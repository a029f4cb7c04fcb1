// aux_kernels.cuh -- the bias-gradient finishing pass and the elementwise
// kernels of the unfused measurement path.
#pragma once

#include "ptx.cuh"

namespace ge {

// dbias[n] = sum over row tiles m (ascending) of partials[m][n]. One thread
// per feature; reads are coalesced across n. Fixed order => reproducible.
__global__ void dbias_finish_kernel(const float* __restrict__ partials, int m_tiles, int N,
                                    float* __restrict__ dbias) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float s = 0.f;
  for (int m = 0; m < m_tiles; ++m) s += partials[static_cast<int64_t>(m) * N + n];
  dbias[n] = s;
}

template <bool BF16>
__device__ __forceinline__ void unpack8(uint4 w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (BF16) {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&u[i]);
      f[2 * i] = __low2float(h);
      f[2 * i + 1] = __high2float(h);
    } else {
      __half2 h = *reinterpret_cast<const __half2*>(&u[i]);
      f[2 * i] = __low2float(h);
      f[2 * i + 1] = __high2float(h);
    }
  }
}

template <bool BF16>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 w;
  uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (BF16) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      u[i] = *reinterpret_cast<uint32_t*>(&h);
    } else {
      __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
      u[i] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
  return w;
}

// Unfused GELU: out = gelu(in), 8 elements per thread (n_vec = T * N / 8).
template <bool BF16>
__global__ void gelu_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t n_vec) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float f[8];
    unpack8<BF16>(in[i], f);
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = 0.5f * f[j] * (1.0f + erff(f[j] * 0.70710678118654752f));
    out[i] = pack8<BF16>(f);
  }
}

// Unfused BiasAdd: out[t][n] = in[t][n] + bias[n] (8 elements per thread).
template <bool BF16>
__global__ void bias_add_kernel(const uint4* __restrict__ in, const void* __restrict__ bias, uint4* __restrict__ out,
                                int64_t T, int N, int bias_f32) {
  const int vec_per_row = N / 8;
  const int64_t total = T * vec_per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int n0 = static_cast<int>(i % vec_per_row) * 8;
    float f[8];
    unpack8<BF16>(in[i], f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (bias_f32)
        f[j] += reinterpret_cast<const float*>(bias)[n0 + j];
      else if constexpr (BF16)
        f[j] += __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(bias)[n0 + j]);
      else
        f[j] += __half2float(reinterpret_cast<const __half*>(bias)[n0 + j]);
    }
    out[i] = pack8<BF16>(f);
  }
}

// Unfused ReLU (+ mask): one thread per (row, 32-column word).
template <bool BF16, bool AUX>
__global__ void relu_mask_kernel(const uint16_t* __restrict__ in, uint16_t* __restrict__ out,
                                 uint32_t* __restrict__ aux, int64_t T, int N, int aux_words) {
  const int64_t total = T * aux_words;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / aux_words;
    const int w = static_cast<int>(i % aux_words);
    uint32_t m = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = w * 32 + q * 8;
      if (n < N) {
        const int64_t off = t * N + n;
        float f[8];
        unpack8<BF16>(*reinterpret_cast<const uint4*>(in + off), f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const bool pos = f[j] > 0.f;
          m |= (pos ? 1u : 0u) << (q * 8 + j);
          f[j] = pos ? f[j] : 0.f;
        }
        *reinterpret_cast<uint4*>(out + off) = pack8<BF16>(f);
      }
    }
    if (AUX) aux[i] = m;
  }
}

// Unfused mask application: dZ = bit ? G : 0, one thread per (row, word).
template <bool BF16>
__global__ void mask_apply_kernel(const uint16_t* __restrict__ G, const uint32_t* __restrict__ aux,
                                  uint16_t* __restrict__ dZ, int64_t T, int N, int aux_words) {
  const int64_t total = T * aux_words;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / aux_words;
    const int w = static_cast<int>(i % aux_words);
    const uint32_t m = aux[i];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = w * 32 + q * 8;
      if (n < N) {
        const int64_t off = t * N + n;
        uint4 g = *reinterpret_cast<const uint4*>(G + off);
        uint32_t* u = reinterpret_cast<uint32_t*>(&g);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t lo = (m >> (q * 8 + 2 * j)) & 1u, hi = (m >> (q * 8 + 2 * j + 1)) & 1u;
          u[j] &= (lo ? 0x0000FFFFu : 0u) | (hi ? 0xFFFF0000u : 0u);
        }
        *reinterpret_cast<uint4*>(dZ + off) = g;
      }
    }
  }
}

// Unfused column sum, first pass: partials[m][n] = sum of dZ over rows
// [128 m, 128 m + 128), one thread per column, rows in ascending order.
template <bool BF16>
__global__ void colsum_partial_kernel(const uint16_t* __restrict__ dZ, int64_t T, int N, float* __restrict__ partials) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int m = blockIdx.y;
  if (n >= N) return;
  const int64_t t0 = static_cast<int64_t>(m) * 128;
  const int64_t t1 = t0 + 128 < T ? t0 + 128 : T;
  float s = 0.f;
  for (int64_t t = t0; t < t1; ++t) {
    const uint16_t h = dZ[t * N + n];
    if constexpr (BF16)
      s += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&h));
    else
      s += __half2float(*reinterpret_cast<const __half*>(&h));
  }
  partials[static_cast<int64_t>(m) * N + n] = s;
}

}  // namespace ge
