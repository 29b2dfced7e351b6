// mq_linear_noalloc: the decode GEMV (M <= 32) for callers that must not
// allocate device memory. Its scratch (the fragment-ordered activation
// blocks, the activation class sums and the wait-error word) lives in one
// file-scope device array that every GPU loading this library holds until the
// process exits; the entry point itself never calls cudaMalloc or cudaFree.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <vector>

#include "../../include/mq.h"
#include "mq_internal.h"

namespace mq {
namespace {

// Layout of the array: [0, 256) the wait-error word (zeroed at set-up),
// [256, kNoAllocScratchBytes) the decode path's scratch.
constexpr size_t kNoAllocHeader = 256;
constexpr size_t kNoAllocScratchBytes = MQ_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
std::vector<void*> g_noalloc_addr;  // per device ordinal; null until set up

// Once per device, with that device current: resolves the array's device
// address (in host code the symbol itself is only a host-side stand-in) and
// zeroes the error word.
cudaError_t noalloc_base(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_noalloc_mutex);
  if (g_noalloc_addr.size() <= static_cast<size_t>(dev)) g_noalloc_addr.resize(dev + 1, nullptr);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    e = cudaMemset(p, 0, kNoAllocHeader);
    if (e != cudaSuccess) return e;
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

mq_status noalloc_fail(mq_status s, const char* fmt, ...) {
  char buf[384];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  set_last_error(buf);
  return s;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

// Reads and clears the array's wait-error word on the current device (0 if
// mq_linear_noalloc was never set up there: then nothing can have set it).
// Synchronous; allocates nothing.
cudaError_t noalloc_take_error(uint32_t* flags) {
  *flags = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mutex);
    if (static_cast<size_t>(dev) < g_noalloc_addr.size()) p = g_noalloc_addr[dev];
  }
  if (!p) return cudaSuccess;
  e = cudaMemcpy(flags, p, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess || *flags == 0) return e;
  return cudaMemset(p, 0, sizeof(uint32_t));
}

}  // namespace mq

using namespace mq;

extern "C" mq_status mq_linear_noalloc(const void* x, int64_t M, int64_t K, const void* packed,
                                       const float* alpha, const float* zero, int64_t N, int r,
                                       float* y, void* stream) {
  mq::TraceRange trace_("mq_linear_noalloc");
  set_last_error("");
  if (!x || !packed || !alpha || !zero || !y) return noalloc_fail(MQ_ERR_INVALID_ARG, "mq_linear_noalloc: null pointer");
  if (r != 8 && r != 6 && r != 4 && r != 3 && r != 2)
    return noalloc_fail(MQ_ERR_INVALID_ARG, "mq_linear_noalloc: r=%d not in {8,6,4,3,2}", r);
  if (M < 1 || M > 32) return noalloc_fail(MQ_ERR_INVALID_ARG, "mq_linear_noalloc: M=%lld must be in [1, 32]", (long long)M);
  if (N < 1) return noalloc_fail(MQ_ERR_INVALID_ARG, "mq_linear_noalloc: N must be >= 1");
  // every plane row a whole number of 16-byte units (as mq_linear)
  const int kmult = r == 3 ? 128 : (r == 6 || r == 2) ? 64 : 32;
  if (K < kmult || K % kmult != 0)
    return noalloc_fail(MQ_ERR_INVALID_ARG, "mq_linear_noalloc: K must be a positive multiple of %d at r = %d (K=%lld)",
                        kmult, r, (long long)K);
  if (!aligned(x, 16) || !aligned(packed, 16))
    return noalloc_fail(MQ_ERR_INVALID_ARG, "mq_linear_noalloc: x and packed must be 16-byte aligned");
  if (!aligned(alpha, 4) || !aligned(zero, 4) || !aligned(y, 4))
    return noalloc_fail(MQ_ERR_INVALID_ARG, "mq_linear_noalloc: alpha, zero, y must be 4-byte aligned");
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 24))
    return noalloc_fail(MQ_ERR_UNSUPPORTED, "mq_linear_noalloc: N or K too large");
  LinearJob job{x, static_cast<const uint8_t*>(packed), alpha, zero, y, N, K, r};
  const size_t need = gemv_scratch_bytes(job, static_cast<int>(M));
  const size_t have = kNoAllocScratchBytes - kNoAllocHeader;
  if (need > have)
    return noalloc_fail(MQ_ERR_INVALID_ARG,
                        "mq_linear_noalloc: M=%lld, K=%lld needs %zu scratch bytes, more than the fixed "
                        "%zu (M*K up to 524288 fits; K up to 174592 at M = 1)",
                        (long long)M, (long long)K, need, have);
  void* base = nullptr;
  cudaError_t e = noalloc_base(&base);
  if (e != cudaSuccess) return noalloc_fail(MQ_ERR_CUDA, "mq_linear_noalloc: set-up: %s", cudaGetErrorString(e));
  unsigned char* b = static_cast<unsigned char*>(base);
  // header: the error word at byte 0, the grid-barrier words at byte 128
  FixedScratch fs{b + kNoAllocHeader, have, reinterpret_cast<uint32_t*>(b), reinterpret_cast<uint32_t*>(b + 128)};
  e = run_gemv_fixed(job, static_cast<int>(M), static_cast<cudaStream_t>(stream), fs);
  if (e != cudaSuccess) return noalloc_fail(MQ_ERR_CUDA, "mq_linear_noalloc: %s", cudaGetErrorString(e));
  return MQ_OK;
}
