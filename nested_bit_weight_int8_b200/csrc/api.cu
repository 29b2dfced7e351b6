// C ABI entry points: argument checks, status codes, the per-(device, stream)
// workspace and the device error word. Every compute step runs in the
// library's own kernels; nothing here computes on the host.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "../../include/mq.h"
#include "mq_device.cuh"
#include "mq_internal.h"

namespace mq {

// The container file (container_io.cu); nonzero return = failure with `why`
// (2: a file of another shape).
int container_save(const char* path, const uint8_t* q, const float* alpha, const float* zero, int64_t N,
                   int64_t K, char* why, size_t why_len);
int container_info(const char* path, int64_t* N, int64_t* K, char* why, size_t why_len);
int container_load(const char* path, uint8_t* q, float* alpha, float* zero, int64_t N, int64_t K, char* why,
                   size_t why_len);

namespace {

thread_local std::string g_last_error;
std::mutex g_ws_mutex;
std::map<std::pair<int, cudaStream_t>, Workspace> g_workspaces;
std::map<int, uint32_t*> g_error_words;
uint64_t g_wait_limit_ns = 2000000000ull;
std::map<int, int> g_sm_counts;

mq_status fail(mq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

mq_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }


bool valid_r(int r) { return r == 8 || r == 6 || r == 4 || r == 3 || r == 2; }

// The K a width's planes need: every plane row (K b / 8 bytes for a plane of
// width b) must be a whole number of 16-byte units, the row pitch of a TMA
// box. r = 8 and 4 need K % 32 (with the pages' K % 32 as the floor), r = 6
// and 2 (a 2-bit plane) K % 64, r = 3 (a 1-bit plane) K % 128. The int8
// container (one byte per weight) serves every width from K % 32.
int plane_kmult(int r) { return r == 3 ? 128 : (r == 6 || r == 2) ? 64 : 32; }

}  // namespace

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_ws_mutex);
  auto it = g_sm_counts.find(dev);
  if (it != g_sm_counts.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
  g_sm_counts[dev] = n;
  return n;
}

cudaError_t get_workspace(cudaStream_t stream, size_t bytes, void** out, uint32_t** sync) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  bytes += kSyncBytes;
  std::lock_guard<std::mutex> lk(g_ws_mutex);
  Workspace& w = g_workspaces[std::make_pair(dev, stream)];
  if (w.bytes < bytes) {
    if (w.ptr) {
      e = cudaDeviceSynchronize();  // in-flight kernels may still read the old buffer
      if (e != cudaSuccess) return e;
      cudaFree(w.ptr);
      w.ptr = nullptr;
      w.bytes = 0;
    }
    size_t sz = bytes < (1u << 20) ? (1u << 20) : bytes;
    sz = (sz + 4095) & ~size_t(4095);
    void* p = nullptr;
    e = cudaMalloc(&p, sz);
    if (e != cudaSuccess) return e;
    // the barrier words start at zero, ahead of any kernel on this stream;
    // the workspace is kept only once that is enqueued
    e = cudaMemsetAsync(p, 0, kSyncBytes, stream);
    if (e != cudaSuccess) {
      cudaFree(p);
      return e;
    }
    w.ptr = p;
    w.bytes = sz;
  }
  *out = static_cast<uint8_t*>(w.ptr) + kSyncBytes;
  if (sync) *sync = static_cast<uint32_t*>(w.ptr);
  return cudaSuccess;
}

cudaError_t get_error_word(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_ws_mutex);
  auto it = g_error_words.find(dev);
  if (it == g_error_words.end()) {
    uint32_t* p = nullptr;
    e = cudaMalloc(&p, 256);
    if (e != cudaSuccess) return e;
    e = cudaMemset(p, 0, 256);
    if (e != cudaSuccess) return e;
    it = g_error_words.emplace(dev, p).first;
  }
  *out = it->second;
  return cudaSuccess;
}

uint32_t* find_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lk(g_ws_mutex);
  auto it = g_error_words.find(dev);
  return it == g_error_words.end() ? nullptr : it->second;
}

uint64_t wait_limit_ns() { return g_wait_limit_ns; }

void set_last_error(const char* msg) { g_last_error = msg; }

}  // namespace mq

using namespace mq;

extern "C" {

int mq_version(void) { return (0 << 16) | 3; }

const char* mq_last_error(void) { return g_last_error.c_str(); }

size_t mq_packed_bytes(int64_t N, int64_t K, int r) {
  if (N < 1 || K < 1 || !valid_r(r) || K % plane_kmult(r) != 0) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) * static_cast<size_t>(r) / 8;
}

mq_status mq_quantize_int8(const void* w, int dtype, int64_t N, int64_t K, uint8_t* q,
                           float* alpha, float* zero, void* stream) {
  TraceRange trace_("mq_quantize_int8");
  g_last_error.clear();
  if (!w || !q || !alpha || !zero) return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8: null pointer");
  if (dtype != MQ_F32 && dtype != MQ_BF16) return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8: dtype must be MQ_F32 or MQ_BF16");
  if (N < 1 || K < 1) return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8: N and K must be >= 1");
  if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return fail(MQ_ERR_UNSUPPORTED, "mq_quantize_int8: N or K too large");
  if (!aligned(w, 4) || !aligned(alpha, 4) || !aligned(zero, 4))
    return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8: w, alpha, zero must be 4-byte aligned");
  cudaError_t e = launch_quantize(w, dtype, N, K, nullptr, nullptr, q, alpha, zero,
                                  static_cast<cudaStream_t>(stream), sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "mq_quantize_int8");
  return MQ_OK;
}

mq_status mq_quantize_int8_clipped(const void* w, int dtype, int64_t N, int64_t K,
                                   const float* gamma, const float* beta, uint8_t* q, float* alpha,
                                   float* zero, void* stream) {
  TraceRange trace_("mq_quantize_int8_clipped");
  g_last_error.clear();
  if (!w || !gamma || !beta || !q || !alpha || !zero)
    return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8_clipped: null pointer");
  if (dtype != MQ_F32 && dtype != MQ_BF16) return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8_clipped: dtype must be MQ_F32 or MQ_BF16");
  if (N < 1 || K < 1) return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8_clipped: N and K must be >= 1");
  if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return fail(MQ_ERR_UNSUPPORTED, "mq_quantize_int8_clipped: N or K too large");
  if (!aligned(w, 4) || !aligned(alpha, 4) || !aligned(zero, 4) || !aligned(gamma, 4) || !aligned(beta, 4))
    return fail(MQ_ERR_INVALID_ARG, "mq_quantize_int8_clipped: w, gamma, beta, alpha, zero must be 4-byte aligned");
  cudaError_t e = launch_quantize(w, dtype, N, K, gamma, beta, q, alpha, zero,
                                  static_cast<cudaStream_t>(stream), sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "mq_quantize_int8_clipped");
  return MQ_OK;
}

mq_status mq_slice_pack(const uint8_t* q, int64_t N, int64_t K, int r, void* packed, void* stream) {
  TraceRange trace_("mq_slice_pack");
  g_last_error.clear();
  if (!q || !packed) return fail(MQ_ERR_INVALID_ARG, "mq_slice_pack: null pointer");
  if (!valid_r(r)) return fail(MQ_ERR_INVALID_ARG, "mq_slice_pack: r=%d not in {8,6,4,3,2}", r);
  if (N < 1 || K < 1 || K % plane_kmult(r) != 0)
    return fail(MQ_ERR_INVALID_ARG, "mq_slice_pack: need N >= 1 and K a positive multiple of %d at r = %d (K=%lld)",
                plane_kmult(r), r, (long long)K);
  if (!aligned(q, 16) || !aligned(packed, 16)) return fail(MQ_ERR_INVALID_ARG, "mq_slice_pack: q and packed must be 16-byte aligned");
  if (N * K > (int64_t(1) << 40)) return fail(MQ_ERR_UNSUPPORTED, "mq_slice_pack: matrix too large");
  cudaError_t e = launch_slice_pack(q, N, K, r, packed, static_cast<cudaStream_t>(stream), sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "mq_slice_pack");
  return MQ_OK;
}

// kmult: the K multiple the weights' layout needs (plane_kmult(r) for
// planes, 32 for the container).
static mq_status check_linear(const char* who, const void* x, int64_t M, int64_t K, const void* packed,
                              const float* alpha, const float* zero, int64_t N, int r, const float* y,
                              int kmult) {
  if (!x || !packed || !alpha || !zero || !y) return fail(MQ_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!valid_r(r)) return fail(MQ_ERR_INVALID_ARG, "%s: r=%d not in {8,6,4,3,2}", who, r);
  if (M < 1) return fail(MQ_ERR_INVALID_ARG, "%s: M must be >= 1", who);
  if (N < 1) return fail(MQ_ERR_INVALID_ARG, "%s: N must be >= 1", who);
  if (K < kmult || K % kmult != 0)
    return fail(MQ_ERR_INVALID_ARG, "%s: K must be a positive multiple of %d at r = %d (K=%lld)", who, kmult, r,
                (long long)K);
  if (!aligned(x, 16) || !aligned(packed, 16)) return fail(MQ_ERR_INVALID_ARG, "%s: x and packed must be 16-byte aligned", who);
  if (!aligned(alpha, 4) || !aligned(zero, 4) || !aligned(y, 4)) return fail(MQ_ERR_INVALID_ARG, "%s: alpha, zero, y must be 4-byte aligned", who);
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 24)) return fail(MQ_ERR_UNSUPPORTED, "%s: N or K too large", who);
  return MQ_OK;
}

mq_status mq_linear(const void* x, int64_t M, int64_t K, const void* packed, const float* alpha,
                    const float* zero, int64_t N, int r, float* y, void* stream) {
  TraceRange trace_("mq_linear");
  g_last_error.clear();
  mq_status st = check_linear("mq_linear", x, M, K, packed, alpha, zero, N, r, y, valid_r(r) ? plane_kmult(r) : 32);
  if (st != MQ_OK) return st;
  LinearJob job{x, static_cast<const uint8_t*>(packed), alpha, zero, y, N, K, r};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (M <= 32) {
    e = run_gemv(&job, 1, static_cast<int>(M), s);
  } else {
    if (M > (int64_t(1) << 24)) return fail(MQ_ERR_UNSUPPORTED, "mq_linear: M too large");
    e = run_gemm(job, static_cast<int>(M), s);
  }
  if (e == cudaErrorNotSupported) return fail(MQ_ERR_UNSUPPORTED, "mq_linear: shape not served by this build");
  if (e != cudaSuccess) return cuda_fail(e, "mq_linear");
  return MQ_OK;
}

mq_status mq_linear_container(const void* x, int64_t M, int64_t K, const uint8_t* q,
                              const float* alpha, const float* zero, int64_t N, int r, int clamp,
                              float* y, void* stream) {
  TraceRange trace_("mq_linear_container");
  g_last_error.clear();
  mq_status st = check_linear("mq_linear_container", x, M, K, q, alpha, zero, N, r, y, 32);
  if (st != MQ_OK) return st;
  if (clamp != 0 && clamp != 1) return fail(MQ_ERR_INVALID_ARG, "mq_linear_container: clamp must be 0 or 1");
  LinearJob job{x, q, alpha, zero, y, N, K, r, clamp ? kContainer : kContainerEP};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (M <= 32) {
    e = run_gemv(&job, 1, static_cast<int>(M), s);
  } else {
    if (M > (int64_t(1) << 24)) return fail(MQ_ERR_UNSUPPORTED, "mq_linear_container: M too large");
    e = run_gemm(job, static_cast<int>(M), s);
  }
  if (e == cudaErrorNotSupported) return fail(MQ_ERR_UNSUPPORTED, "mq_linear_container: shape not served by this build");
  if (e != cudaSuccess) return cuda_fail(e, "mq_linear_container");
  return MQ_OK;
}

static mq_status check_ovf(const char* who, const uint8_t* q, int64_t N, int64_t K, int r) {
  if (!q) return fail(MQ_ERR_INVALID_ARG, "%s: null q", who);
  if (r != 6 && r != 4 && r != 3 && r != 2) return fail(MQ_ERR_INVALID_ARG, "%s: r=%d not in {6,4,3,2}", who, r);
  if (N < 1 || K < 16 || K % 16 != 0) return fail(MQ_ERR_INVALID_ARG, "%s: need N >= 1 and K a positive multiple of 16", who);
  if (K > 65536 || N * K >= (int64_t(1) << 31)) return fail(MQ_ERR_UNSUPPORTED, "%s: K > 65536 or N*K >= 2^31", who);
  if (!aligned(q, 16)) return fail(MQ_ERR_INVALID_ARG, "%s: q must be 16-byte aligned", who);
  return MQ_OK;
}

mq_status mq_ep_overflow_rows(const uint8_t* q, int64_t N, int64_t K, int r, int32_t* row_ptr,
                              void* stream) {
  TraceRange trace_("mq_ep_overflow_rows");
  g_last_error.clear();
  mq_status st = check_ovf("mq_ep_overflow_rows", q, N, K, r);
  if (st != MQ_OK) return st;
  if (!row_ptr || !aligned(row_ptr, 4)) return fail(MQ_ERR_INVALID_ARG, "mq_ep_overflow_rows: row_ptr null or not 4-byte aligned");
  cudaError_t e = launch_ovf_rows(q, N, K, r, row_ptr, static_cast<cudaStream_t>(stream), sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "mq_ep_overflow_rows");
  return MQ_OK;
}

mq_status mq_ep_overflow_cols(const uint8_t* q, int64_t N, int64_t K, int r, const int32_t* row_ptr,
                              uint16_t* cols, void* stream) {
  TraceRange trace_("mq_ep_overflow_cols");
  g_last_error.clear();
  mq_status st = check_ovf("mq_ep_overflow_cols", q, N, K, r);
  if (st != MQ_OK) return st;
  if (!row_ptr || !aligned(row_ptr, 4)) return fail(MQ_ERR_INVALID_ARG, "mq_ep_overflow_cols: row_ptr null or not 4-byte aligned");
  if (!cols || !aligned(cols, 2)) return fail(MQ_ERR_INVALID_ARG, "mq_ep_overflow_cols: cols null or not 2-byte aligned");
  cudaError_t e = launch_ovf_cols(q, N, K, r, row_ptr, cols, static_cast<cudaStream_t>(stream), sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "mq_ep_overflow_cols");
  return MQ_OK;
}

mq_status mq_linear_ep(const void* x, int64_t M, int64_t K, const void* packed, const float* alpha,
                       const float* zero, int64_t N, int r, const int32_t* row_ptr,
                       const uint16_t* cols, float* y, void* stream) {
  TraceRange trace_("mq_linear_ep");
  g_last_error.clear();
  mq_status st = check_linear("mq_linear_ep", x, M, K, packed, alpha, zero, N, r, y, valid_r(r) ? plane_kmult(r) : 32);
  if (st != MQ_OK) return st;
  if (r == 8) return fail(MQ_ERR_INVALID_ARG, "mq_linear_ep: r=8 has no extra bucket");
  if (!row_ptr || !cols || !aligned(row_ptr, 4) || !aligned(cols, 2))
    return fail(MQ_ERR_INVALID_ARG, "mq_linear_ep: row_ptr / cols null or misaligned");
  if (K > 65536) return fail(MQ_ERR_UNSUPPORTED, "mq_linear_ep: K > 65536");
  LinearJob job{x, static_cast<const uint8_t*>(packed), alpha, zero, y, N, K, r, kPlanes, row_ptr, cols};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (M <= 32) {
    e = run_gemv(&job, 1, static_cast<int>(M), s);
  } else {
    if (M > (int64_t(1) << 24)) return fail(MQ_ERR_UNSUPPORTED, "mq_linear_ep: M too large");
    e = run_gemm(job, static_cast<int>(M), s);
  }
  if (e == cudaErrorNotSupported) return fail(MQ_ERR_UNSUPPORTED, "mq_linear_ep: shape not served by this build");
  if (e != cudaSuccess) return cuda_fail(e, "mq_linear_ep");
  return MQ_OK;
}

size_t mq_chain_scratch_bytes(int64_t M, int64_t D, int64_t Dkv, int64_t F) {
  if (M < 1 || M > 32 || D < 128 || Dkv < 1 || F < 128) return 0;
  return chain_scratch_bytes(M, D, Dkv, F);
}

mq_status mq_chain_scratch_views(int64_t M, int64_t D, int64_t Dkv, int64_t F, mq_chain_views* out) {
  g_last_error.clear();
  if (!out) return fail(MQ_ERR_INVALID_ARG, "mq_chain_scratch_views: null out");
  if (mq_chain_scratch_bytes(M, D, Dkv, F) == 0) return fail(MQ_ERR_INVALID_ARG, "mq_chain_scratch_views: bad sizes");
  size_t v[10];
  chain_views(M, D, Dkv, F, v);
  *out = mq_chain_views{v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], v[8], v[9]};
  return MQ_OK;
}

mq_status mq_chain_forward(const mq_chain_layer* layers, int n_layers, int64_t M, int64_t D,
                           int64_t Dkv, int64_t F, int64_t head_dim, float* h, void* scratch,
                           size_t scratch_bytes, int flags, void* stream) {
  TraceRange trace_("mq_chain_forward");
  g_last_error.clear();
  const char* who = "mq_chain_forward";
  if (!layers || !h || !scratch) return fail(MQ_ERR_INVALID_ARG, "%s: null pointer", who);
  if (n_layers < 1) return fail(MQ_ERR_INVALID_ARG, "%s: n_layers must be >= 1", who);
  if (M < 1 || M > 32) return fail(MQ_ERR_INVALID_ARG, "%s: M must be in [1, 32]", who);
  if (D < 128 || D % 128 || F < 128 || F % 128) return fail(MQ_ERR_INVALID_ARG, "%s: D and F must be positive multiples of 128", who);
  if (head_dim < 1 || Dkv < head_dim || Dkv % head_dim || D % head_dim || (D / head_dim) % (Dkv / head_dim))
    return fail(MQ_ERR_INVALID_ARG, "%s: head_dim must divide Dkv and D, and D / head_dim be a multiple of Dkv / head_dim", who);
  if (D > (int64_t(1) << 20) || F > (int64_t(1) << 20) || Dkv > (int64_t(1) << 20))
    return fail(MQ_ERR_UNSUPPORTED, "%s: dimensions too large", who);
  if (flags & ~MQ_CHAIN_GRAPH) return fail(MQ_ERR_INVALID_ARG, "%s: unknown flags", who);
  if (!aligned(h, 4) || !aligned(scratch, 256)) return fail(MQ_ERR_INVALID_ARG, "%s: h must be 4-byte and scratch 256-byte aligned", who);
  if (scratch_bytes < chain_scratch_bytes(M, D, Dkv, F)) return fail(MQ_ERR_INVALID_ARG, "%s: scratch smaller than mq_chain_scratch_bytes", who);
  const int64_t nout[5] = {D + 2 * Dkv, D, F, F, D};
  const int64_t nin[5] = {D, D, D, D, F};
  for (int l = 0; l < n_layers; ++l) {
    const mq_chain_layer& L = layers[l];
    for (int i = 0; i < 5; ++i) {
      char w[64];
      std::snprintf(w, sizeof(w), "%s[layer %d, linear %d]", who, l, i);
      // a 16-byte-aligned stand-in for x: the chain's own bf16 buffers
      mq_status st = check_linear(w, scratch, M, nin[i], L.packed[i], L.alpha[i], L.zero[i], nout[i], L.r, h,
                                  valid_r(L.r) ? plane_kmult(L.r) : 32);
      if (st != MQ_OK) return st;
    }
  }
  cudaError_t e = run_chain(layers, n_layers, static_cast<int>(M), static_cast<int>(D), static_cast<int>(Dkv),
                            static_cast<int>(F), static_cast<int>(head_dim), h, scratch,
                            (flags & MQ_CHAIN_GRAPH) != 0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, who);
  return MQ_OK;
}

mq_status mq_container_save(const char* path, const uint8_t* q, const float* alpha, const float* zero,
                            int64_t N, int64_t K) {
  TraceRange trace_("mq_container_save");
  g_last_error.clear();
  if (!path || !q || !alpha || !zero) return fail(MQ_ERR_INVALID_ARG, "mq_container_save: null pointer");
  if (N < 1 || K < 1) return fail(MQ_ERR_INVALID_ARG, "mq_container_save: N and K must be >= 1");
  char why[512];
  if (container_save(path, q, alpha, zero, N, K, why, sizeof(why)) != 0) return fail(MQ_ERR_IO, "%s", why);
  return MQ_OK;
}

mq_status mq_container_info(const char* path, int64_t* N, int64_t* K) {
  g_last_error.clear();
  if (!path || !N || !K) return fail(MQ_ERR_INVALID_ARG, "mq_container_info: null pointer");
  char why[512];
  if (container_info(path, N, K, why, sizeof(why)) != 0) return fail(MQ_ERR_IO, "%s", why);
  return MQ_OK;
}

mq_status mq_container_load(const char* path, uint8_t* q, float* alpha, float* zero, int64_t N, int64_t K) {
  TraceRange trace_("mq_container_load");
  g_last_error.clear();
  if (!path || !q || !alpha || !zero) return fail(MQ_ERR_INVALID_ARG, "mq_container_load: null pointer");
  if (N < 1 || K < 1) return fail(MQ_ERR_INVALID_ARG, "mq_container_load: N and K must be >= 1");
  char why[512];
  const int rc = container_load(path, q, alpha, zero, N, K, why, sizeof(why));
  if (rc == 2) return fail(MQ_ERR_INVALID_ARG, "%s", why);
  if (rc != 0) return fail(MQ_ERR_IO, "%s", why);
  return MQ_OK;
}

mq_status mq_stack_forward(const mq_linear_desc* lins, const int* layer_of_lin, int n_lins,
                           const int* widths, int n_layers, int64_t M, void* stream) {
  TraceRange trace_("mq_stack_forward");
  g_last_error.clear();
  if (!lins || !layer_of_lin || !widths) return fail(MQ_ERR_INVALID_ARG, "mq_stack_forward: null host array");
  if (n_lins < 1 || n_layers < 1) return fail(MQ_ERR_INVALID_ARG, "mq_stack_forward: need n_lins >= 1 and n_layers >= 1");
  if (M < 1 || M > 32) return fail(MQ_ERR_INVALID_ARG, "mq_stack_forward: M must be in [1, 32]");
  std::vector<LinearJob> jobs(n_lins);
  for (int i = 0; i < n_lins; ++i) {
    const int layer = layer_of_lin[i];
    if (layer < 0 || layer >= n_layers) return fail(MQ_ERR_INVALID_ARG, "mq_stack_forward: layer_of_lin[%d]=%d out of range", i, layer);
    const int r = widths[layer];
    const mq_linear_desc& d = lins[i];
    char who[64];
    std::snprintf(who, sizeof(who), "mq_stack_forward[lin %d]", i);
    mq_status st = check_linear(who, d.x, M, d.K, d.packed, d.alpha, d.zero, d.N, r, d.y, valid_r(r) ? plane_kmult(r) : 32);
    if (st != MQ_OK) return st;
    jobs[i] = LinearJob{d.x, static_cast<const uint8_t*>(d.packed), d.alpha, d.zero, d.y, d.N, d.K, r};
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int b = 0; b < n_lins; b += kGemvMaxLinears) {
    const int cnt = (n_lins - b) < kGemvMaxLinears ? (n_lins - b) : kGemvMaxLinears;
    cudaError_t e = run_gemv(jobs.data() + b, cnt, static_cast<int>(M), s);
    if (e != cudaSuccess) return cuda_fail(e, "mq_stack_forward");
  }
  return MQ_OK;
}

mq_status mq_device_status(void* stream) {
  TraceRange trace_("mq_device_status");
  g_last_error.clear();
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "mq_device_status");
  // The device's error word exists once any allocating call ran here; this
  // call does not create it, so a caller of mq_linear_noalloc alone still
  // allocates nothing.
  uint32_t v = 0;
  if (uint32_t* err = find_error_word()) {
    e = cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "mq_device_status");
    if (v != 0) {
      e = cudaMemset(err, 0, sizeof(uint32_t));
      if (e != cudaSuccess) return cuda_fail(e, "mq_device_status");
    }
  }
  // mq_linear_noalloc's kernels flag a give-up in its fixed array instead
  uint32_t vn = 0;
  e = noalloc_take_error(&vn);
  if (e != cudaSuccess) return cuda_fail(e, "mq_device_status");
  v |= vn;
  if (v != 0) {
    if (v & kErrBounds)
      return fail(MQ_ERR_BOUNDS, "a device index check failed (flags 0x%x); its outputs are undefined", v);
    return fail(MQ_ERR_TIMEOUT, "a kernel gave up a bounded wait (flags 0x%x); its outputs are undefined", v);
  }
  return MQ_OK;
}

mq_status mq_release_workspace(void) {
  g_last_error.clear();
  std::lock_guard<std::mutex> lk(g_ws_mutex);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_workspaces) {
    if (kv.second.ptr) {
      cudaSetDevice(kv.first.first);
      cudaDeviceSynchronize();
      cudaFree(kv.second.ptr);
    }
  }
  g_workspaces.clear();
  cudaSetDevice(cur);
  release_chain_graphs();
  release_map_tables();
  return MQ_OK;
}

int64_t mq_debug_map_table_count(void) { return static_cast<int64_t>(map_table_count()); }

mq_status mq_debug_set_wait_limit_ns(uint64_t ns) {
  g_last_error.clear();
  g_wait_limit_ns = ns;
  return MQ_OK;
}

}  // extern "C"
