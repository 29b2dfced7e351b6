// Eq. 1 (per-channel MinMax int8 container) and Eq. 6 (MSB slicing) packed
// into dense r-bit planes. Both are one-time, HBM-bound passes over a weight
// matrix ("Matryoshka Quantization" explainer page, section 3.4 Eq. 1 and
// "The Bit-Slicing Operator" Eq. 6).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "mq_internal.h"

namespace mq {
namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ float ld_w(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_w(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// One IEEE-binary32 quantization step of Eq. 1, every operation correctly
// rounded: t = (w / alpha) + z, q = clamp(round-half-even(t), 0, 255).
__device__ __forceinline__ uint32_t quant1(float w, float alpha, float zero) {
  const float t = __fadd_rn(__fdiv_rn(w, alpha), zero);
  const float r = fminf(fmaxf(rintf(t), 0.0f), 255.0f);
  return static_cast<uint32_t>(r);
}

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// One CTA per row (grid-stride over rows). Pass 1 reduces min and max; one
// thread derives alpha and z; pass 2 re-reads the row (an L2 hit) and writes
// the codes. `vec` selects 8-element vector accesses (K % 16 == 0 and every
// pointer 16-byte aligned), else element accesses. With `gamma` and `beta`
// (one pair per row) the range is OmniQuant's clipped [beta*min, gamma*max]
// (Eq. 3) and weights outside it saturate; without them it is Eq. 1's.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
quantize_rows_kernel(const T* __restrict__ w, int64_t N, int64_t K, bool vec,
                     const float* __restrict__ gamma, const float* __restrict__ beta,
                     uint8_t* __restrict__ q, float* __restrict__ alpha,
                     float* __restrict__ zero) {
  __shared__ float s_mn[kQuantThreads / 32], s_mx[kQuantThreads / 32];
  __shared__ float s_alpha, s_zero;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
    const T* row = w + n * K;
    uint8_t* qrow = q + n * K;
    float mn = FLT_MAX, mx = -FLT_MAX;
    if (vec) {
      for (int64_t k = int64_t(tid) * 8; k < K; k += int64_t(kQuantThreads) * 8) {
        float v[8];
        load8<T>(row + k, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
      }
    } else {
      for (int64_t k = tid; k < K; k += kQuantThreads) {
        const float v = ld_w(row + k);
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) { s_mn[warp] = mn; s_mx[warp] = mx; }
    __syncthreads();
    if (tid == 0) {
      float a = s_mn[0], b = s_mx[0];
      for (int i = 1; i < kQuantThreads / 32; ++i) { a = fminf(a, s_mn[i]); b = fmaxf(b, s_mx[i]); }
      if (gamma) {  // Eq. 3: the clipped range [beta * min, gamma * max]
        b = __fmul_rn(gamma[n], b);
        a = __fmul_rn(beta[n], a);
      }
      // Eq. 1: alpha = (max - min) / (2^8 - 1), z = -min / alpha.
      float al = __fdiv_rn(__fsub_rn(b, a), 255.0f);
      // constant row (or an empty clipped range): alpha = max(|min| 2^-8,
      // 2^-126), both exact, so z = -min / alpha is -256 sign(min) (or
      // min 2^126) and alpha (0 - z) = min exactly
      if (!(al > 0.0f)) al = fmaxf(fabsf(a) * 0.00390625f, 1.17549435e-38f);
      const float z = __fdiv_rn(-a, al);
      s_alpha = al;
      s_zero = z;
      alpha[n] = al;
      zero[n] = z;
    }
    __syncthreads();
    const float al = s_alpha, z = s_zero;
    if (vec) {
      for (int64_t k = int64_t(tid) * 8; k < K; k += int64_t(kQuantThreads) * 8) {
        float v[8];
        load8<T>(row + k, v);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          lo |= quant1(v[i], al, z) << (8 * i);
          hi |= quant1(v[4 + i], al, z) << (8 * i);
        }
        *reinterpret_cast<uint2*>(qrow + k) = make_uint2(lo, hi);
      }
    } else {
      for (int64_t k = tid; k < K; k += kQuantThreads) {
        qrow[k] = static_cast<uint8_t>(quant1(ld_w(row + k), al, z));
      }
    }
    __syncthreads();  // s_alpha / s_zero / s_mn are reused by the next row
  }
}

// Eq. 6 code of one container value: round half up on q / 2^(8-R) (the first
// dropped bit decides), then clamp to 2^R - 1.
template <int R>
__device__ __forceinline__ uint32_t slice_code(uint32_t qv) {
  if constexpr (R == 8) {
    return qv;
  } else {
    constexpr int s = 8 - R;
    const uint32_t k = (qv + (1u << (s - 1))) >> s;
    return k < ((1u << R) - 1) ? k : ((1u << R) - 1);
  }
}

// Bit offset of local code u inside a 32-bit word of a plane of width B.
template <int B>
__device__ __forceinline__ constexpr int plane_bitpos(int u) {
  return B == 8 ? 8 * u : 16 * (u & 1) + B * (u >> 1);
}

// Loads the C = 32/B consecutive container bytes that feed one plane word.
template <int C>
__device__ __forceinline__ void load_bytes(const uint8_t* p, uint8_t (&v)[C]) {
  if constexpr (C == 32) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    *reinterpret_cast<uint4*>(v) = a;
    *reinterpret_cast<uint4*>(v + 16) = b;
  } else if constexpr (C == 16) {
    *reinterpret_cast<uint4*>(v) = __ldg(reinterpret_cast<const uint4*>(p));
  } else if constexpr (C == 8) {
    *reinterpret_cast<uint2*>(v) = __ldg(reinterpret_cast<const uint2*>(p));
  } else {
    *reinterpret_cast<uint32_t*>(v) = __ldg(reinterpret_cast<const uint32_t*>(p));
  }
}

// Builds one 32-bit word of plane `plane` (width B, bit shift SH into the
// code) for row n, word index wi.
template <int R, int B, int SH>
__device__ __forceinline__ uint32_t plane_word(const uint8_t* __restrict__ q, int64_t K,
                                               int64_t n, int64_t wi) {
  constexpr int C = 32 / B;
  alignas(16) uint8_t v[C];
  load_bytes<C>(q + n * K + wi * C, v);
  uint32_t word = 0;
#pragma unroll
  for (int u = 0; u < C; ++u) {
    const uint32_t field = (slice_code<R>(v[u]) >> SH) & ((1u << B) - 1u);
    word |= field << plane_bitpos<B>(u);
  }
  return word;
}

template <int R, int B0, int B1>
__global__ void __launch_bounds__(256)
slice_pack_kernel(const uint8_t* __restrict__ q, int64_t N, int64_t K,
                  uint32_t* __restrict__ out) {
  const int64_t wpr0 = K * B0 / 32;
  const int64_t words0 = N * wpr0;
  const int64_t wpr1 = B1 ? K * B1 / 32 : 1;
  const int64_t total = words0 + (B1 ? N * wpr1 : 0);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    uint32_t word;
    if (i < words0) {
      word = plane_word<R, B0, 0>(q, K, i / wpr0, i % wpr0);
    } else {
      if constexpr (B1 != 0) {
        const int64_t j = i - words0;
        word = plane_word<R, (B1 ? B1 : 1), B0>(q, K, j / wpr1, j % wpr1);
      } else {
        word = 0;
      }
    }
    out[i] = word;
  }
}

int grid_for(int64_t work, int threads, int sms) {
  int64_t g = (work + threads - 1) / threads;
  const int64_t cap = int64_t(sms) * 16;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_quantize(const void* w, int dtype, int64_t N, int64_t K, const float* gamma,
                            const float* beta, uint8_t* q, float* alpha, float* zero,
                            cudaStream_t stream, int sms) {
  const bool aligned = ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(q)) & 15) == 0;
  const bool vec = aligned && (K % 16 == 0);
  int64_t grid = N < int64_t(sms) * 8 ? N : int64_t(sms) * 8;
  if (grid < 1) grid = 1;
  if (dtype == 0) {
    quantize_rows_kernel<float><<<static_cast<int>(grid), kQuantThreads, 0, stream>>>(
        static_cast<const float*>(w), N, K, vec, gamma, beta, q, alpha, zero);
  } else {
    quantize_rows_kernel<__nv_bfloat16><<<static_cast<int>(grid), kQuantThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(w), N, K, vec, gamma, beta, q, alpha, zero);
  }
  return cudaGetLastError();
}

cudaError_t launch_slice_pack(const uint8_t* q, int64_t N, int64_t K, int r, void* packed,
                              cudaStream_t stream, int sms) {
  const int64_t words = N * K * r / 32;
  const int grid = grid_for(words, 256, sms);
  uint32_t* out = static_cast<uint32_t*>(packed);
  switch (r) {
    case 8: slice_pack_kernel<8, 8, 0><<<grid, 256, 0, stream>>>(q, N, K, out); break;
    case 6: slice_pack_kernel<6, 4, 2><<<grid, 256, 0, stream>>>(q, N, K, out); break;
    case 4: slice_pack_kernel<4, 4, 0><<<grid, 256, 0, stream>>>(q, N, K, out); break;
    case 3: slice_pack_kernel<3, 2, 1><<<grid, 256, 0, stream>>>(q, N, K, out); break;
    case 2: slice_pack_kernel<2, 2, 0><<<grid, 256, 0, stream>>>(q, N, K, out); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace mq
