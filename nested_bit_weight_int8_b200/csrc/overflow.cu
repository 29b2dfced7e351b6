// Extra Precision positions ("Matryoshka Quantization" explainer page, errata
// section 7, Eq. 8 without the clamp of Eq. 6). At width r, s = 8 - r, the
// unclamped code of a container value q is one step above the clamped code
// exactly when q + 2^(s-1) >= 256, i.e. q >= 256 - 2^(s-1): the "extra
// bucket". These kernels list, per row, the positions k of those values as
// a compressed sparse row structure (row offsets + 16-bit column indices),
// so that the r-bit planes of Eq. 6 plus the list serve Eq. 8 with one extra
// activation per listed position.
//
// Three steps, all on the device: count per row (one warp per row), one
// exclusive scan of the counts (one CTA), then fill (one warp per row, the
// columns of a row in increasing order).
#include <cuda_runtime.h>

#include <cstdint>

#include "mq_device.cuh"
#include "mq_internal.h"

namespace mq {
namespace {

constexpr int kOvfThreads = 256;
constexpr int kScanThreads = 1024;

// Bit i of the result is set when byte i of the 16 bytes is >= thr (thr4 =
// thr in every byte).
__device__ __forceinline__ uint32_t ovf_mask16(const uint4& v, uint32_t thr4) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t c = __vcmpgeu4(w[i], thr4);  // 0xFF in each byte that is >= thr
#pragma unroll
    for (int b = 0; b < 4; ++b) m |= ((c >> (8 * b + 7)) & 1u) << (4 * i + b);
  }
  return m;
}

// counts: row_ptr[n + 1] = number of positions of row n; row_ptr[0] = 0.
__global__ void __launch_bounds__(kOvfThreads)
ovf_count_kernel(const uint8_t* __restrict__ q, int64_t N, int64_t K, uint32_t thr4,
                 int32_t* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (kOvfThreads / 32);
  if (blockIdx.x == 0 && threadIdx.x == 0) row_ptr[0] = 0;
  for (int64_t n = int64_t(blockIdx.x) * (kOvfThreads / 32) + (threadIdx.x >> 5); n < N; n += warps) {
    const uint8_t* row = q + n * K;
    int cnt = 0;
    for (int64_t k = int64_t(lane) * 16; k < K; k += 32 * 16) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + k);
      cnt += __popc(ovf_mask16(v, thr4));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) row_ptr[n + 1] = cnt;
  }
}

// In-place inclusive scan of row_ptr[1 .. N] (row_ptr[0] = 0 stays): one CTA,
// each thread owns a contiguous chunk.
__global__ void __launch_bounds__(kScanThreads) ovf_scan_kernel(int32_t* __restrict__ row_ptr, int64_t N) {
  __shared__ int64_t s_part[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t chunk = (N + kScanThreads - 1) / kScanThreads;
  const int64_t b = 1 + int64_t(tid) * chunk;
  const int64_t e = b + chunk < N + 1 ? b + chunk : N + 1;
  int64_t sum = 0;
  for (int64_t i = b; i < e; ++i) sum += row_ptr[i];
  // exclusive scan of the chunk sums over the CTA
  int64_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_part[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < kScanThreads / 32 ? s_part[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    if (lane < kScanThreads / 32) s_part[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int64_t run = (incl - sum) + (warp > 0 ? s_part[warp - 1] : 0);
  for (int64_t i = b; i < e; ++i) {
    run += row_ptr[i];
    row_ptr[i] = static_cast<int32_t>(run);
  }
}

// cols[row_ptr[n] ..] = the positions of row n, increasing.
__global__ void __launch_bounds__(kOvfThreads)
ovf_fill_kernel(const uint8_t* __restrict__ q, int64_t N, int64_t K, uint32_t thr4,
                const int32_t* __restrict__ row_ptr, uint16_t* __restrict__ cols, uint32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (kOvfThreads / 32);
  for (int64_t n = int64_t(blockIdx.x) * (kOvfThreads / 32) + (threadIdx.x >> 5); n < N; n += warps) {
    const uint8_t* row = q + n * K;
    int base = row_ptr[n];
    const int row_end = row_ptr[n + 1];
    (void)row_end;  // read only by the debug build's checks
    for (int64_t k0 = 0; k0 < K; k0 += 32 * 16) {
      const int64_t k = k0 + int64_t(lane) * 16;
      uint32_t m = 0;
      if (k < K) m = ovf_mask16(*reinterpret_cast<const uint4*>(row + k), thr4);
      const int cnt = __popc(m);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int pos = base + incl - cnt;
      while (m) {
        const int bit = __ffs(m) - 1;
        if (MQ_IN_BOUNDS(pos < row_end, err)) cols[pos] = static_cast<uint16_t>(k + bit);
        ++pos;
        m &= m - 1;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

int ovf_grid(int64_t N, int sms) {
  const int64_t blocks = (N + kOvfThreads / 32 - 1) / (kOvfThreads / 32);
  const int64_t cap = int64_t(sms) * 8;
  return static_cast<int>(blocks < cap ? (blocks < 1 ? 1 : blocks) : cap);
}

uint32_t threshold4(int r) {
  const uint32_t thr = 256u - (1u << (7 - r));  // 256 - 2^(s-1), s = 8 - r
  return thr * 0x01010101u;
}

// The list as a dense bit plane for the prefill GEMM: bit (k % 32) of word
// n * words + k / 32 is set when position k of row n is listed. One warp per
// row: it clears the row's words, then sets the listed bits.
__global__ void __launch_bounds__(kOvfThreads)
ep_bits_kernel(const int32_t* __restrict__ row_ptr, const uint16_t* __restrict__ cols, int64_t N, int words,
               uint32_t* __restrict__ bits) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (kOvfThreads / 32);
  for (int64_t n = (int64_t(blockIdx.x) * kOvfThreads + threadIdx.x) / 32; n < N; n += warps) {
    uint32_t* row = bits + n * words;
    for (int w = lane; w < words; w += 32) row[w] = 0u;
    __syncwarp();
    const int beg = row_ptr[n], end = row_ptr[n + 1];
    for (int j = beg + lane; j < end; j += 32) {
      const int k = cols[j];
      if (k / 32 < words) atomicOr(row + k / 32, 1u << (k % 32));
    }
  }
}

}  // namespace

cudaError_t launch_ep_bits(const int32_t* row_ptr, const uint16_t* cols, int64_t N, int64_t K, uint32_t* bits,
                           cudaStream_t stream, int sms) {
  ep_bits_kernel<<<ovf_grid(N, sms), kOvfThreads, 0, stream>>>(row_ptr, cols, N, static_cast<int>(K / 32), bits);
  return cudaGetLastError();
}

cudaError_t launch_ovf_rows(const uint8_t* q, int64_t N, int64_t K, int r, int32_t* row_ptr,
                            cudaStream_t stream, int sms) {
  ovf_count_kernel<<<ovf_grid(N, sms), kOvfThreads, 0, stream>>>(q, N, K, threshold4(r), row_ptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ovf_scan_kernel<<<1, kScanThreads, 0, stream>>>(row_ptr, N);
  return cudaGetLastError();
}

cudaError_t launch_ovf_cols(const uint8_t* q, int64_t N, int64_t K, int r, const int32_t* row_ptr,
                            uint16_t* cols, cudaStream_t stream, int sms) {
  uint32_t* err = nullptr;
  cudaError_t e = get_error_word(&err);
  if (e != cudaSuccess) return e;
  ovf_fill_kernel<<<ovf_grid(N, sms), kOvfThreads, 0, stream>>>(q, N, K, threshold4(r), row_ptr, cols, err);
  return cudaGetLastError();
}

}  // namespace mq
