// A chained decoder stack over the sliced linears: each layer's output feeds
// the next layer's input, so a token's decode step is a long chain of
// dependent launches (the measure here is that chain's latency, and how much
// of it a CUDA graph replay removes).
//
// The Matryoshka Quantization pages quantize the linear layers only and
// define no glue between them (explainer page, section 3.4; the Mix'n'Match
// paragraph gives each layer its own width). The stand-in glue, per layer:
//   xn  = bf16(rmsnorm(h))                 RMSNorm, no learned scale, eps 1e-6
//   qkv = xn . Wqkv^T                      decode GEMV
//   a   = bf16(v of the head's kv group)   attention over a one-token context
//   h1  = h + a . Wo^T                     decode GEMV, residual
//   xn1 = bf16(rmsnorm(h1))
//   g, u = xn1 . Wgate^T, xn1 . Wup^T      one decode launch over both
//   act = bf16(silu(g) u)                  SwiGLU
//   h   = h1 + act . Wdown^T               decode GEMV, residual
// The residual stream h is fp32; every linear reads bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <vector>

#include "../../include/mq.h"
#include "mq_device.cuh"
#include "mq_internal.h"

namespace mq {
namespace {

constexpr int kGlueThreads = 256;
constexpr float kEps = 1e-6f;

// One CTA per batch row: v = h + add (add may be null), written to h_out if
// given; xn = bf16(v / sqrt(mean(v^2) + eps)) if xn is given. `clear` (may be
// null) is a word set to zero once the previous grid has finished.
__global__ void __launch_bounds__(kGlueThreads)
rmsnorm_kernel(const float* __restrict__ h, const float* __restrict__ add, float* __restrict__ h_out,
               __nv_bfloat16* __restrict__ xn, int D, uint32_t* clear) {
  __shared__ float red[kGlueThreads / 32];
  __shared__ float s_inv;
  pdl_launch_dependents();
  pdl_wait_primary();
  const int m = blockIdx.x, tid = threadIdx.x;
  if (clear && m == 0 && tid == 0) *clear = 0u;
  const float* hr = h + int64_t(m) * D;
  const float* ar = add ? add + int64_t(m) * D : nullptr;
  float ss = 0.f;
  for (int k = tid; k < D; k += kGlueThreads) {
    const float v = ar ? hr[k] + ar[k] : hr[k];
    if (h_out) h_out[int64_t(m) * D + k] = v;
    ss = fmaf(v, v, ss);
  }
  if (!xn) return;  // the last layer's residual add alone
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((tid & 31) == 0) red[tid >> 5] = ss;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int i = 0; i < kGlueThreads / 32; ++i) t += red[i];
    s_inv = 1.0f / sqrtf(t / static_cast<float>(D) + kEps);
  }
  __syncthreads();
  const float inv = s_inv;
  for (int k = tid; k < D; k += kGlueThreads) {
    const float v = ar ? hr[k] + ar[k] : hr[k];
    xn[int64_t(m) * D + k] = __float2bfloat16_rn(v * inv);
  }
}

// a[m, j] = bf16(v[m, g(j) hd + j % hd]), g(j) = (j / hd) / (heads per kv group).
__global__ void __launch_bounds__(kGlueThreads)
attn_one_token_kernel(const float* __restrict__ qkv, __nv_bfloat16* __restrict__ a, int M, int D,
                      int Dkv, int hd) {
  pdl_launch_dependents();
  pdl_wait_primary();
  const int per_group = (D / hd) / (Dkv / hd);
  const int nq = D + 2 * Dkv;
  const int64_t total = int64_t(M) * D;
  for (int64_t i = int64_t(blockIdx.x) * kGlueThreads + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * kGlueThreads) {
    const int m = static_cast<int>(i / D), j = static_cast<int>(i % D);
    const int g = (j / hd) / per_group;
    a[i] = __float2bfloat16_rn(qkv[int64_t(m) * nq + D + Dkv + g * hd + j % hd]);
  }
}

// act = bf16(silu(g) u), silu(g) = g / (1 + exp(-g)).
__global__ void __launch_bounds__(kGlueThreads)
swiglu_kernel(const float* __restrict__ g, const float* __restrict__ u, __nv_bfloat16* __restrict__ act,
              int64_t total) {
  pdl_launch_dependents();
  pdl_wait_primary();
  for (int64_t i = int64_t(blockIdx.x) * kGlueThreads + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * kGlueThreads) {
    const float gv = g[i];
    act[i] = __float2bfloat16_rn(gv / (1.0f + expf(-gv)) * u[i]);
  }
}

int glue_grid(int64_t total, int sms) {
  const int64_t b = (total + kGlueThreads - 1) / kGlueThreads;
  return static_cast<int>(b < 1 ? 1 : (b > 4 * sms ? 4 * sms : b));
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// Byte offsets of the chain's buffers inside the caller's scratch.
struct ChainLayout {
  size_t xn, qkv, a, o, h1, xn1, g, u, act, dn, ws, ws_bytes, sync, total;
};

ChainLayout chain_layout(int64_t M, int64_t D, int64_t Dkv, int64_t F) {
  ChainLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
  L.xn = take(size_t(M) * D * 2);
  L.qkv = take(size_t(M) * (D + 2 * Dkv) * 4);
  L.a = take(size_t(M) * D * 2);
  L.o = take(size_t(M) * D * 4);
  L.h1 = take(size_t(M) * D * 4);
  L.xn1 = take(size_t(M) * D * 2);
  L.g = take(size_t(M) * F * 4);
  L.u = take(size_t(M) * F * 4);
  L.act = take(size_t(M) * F * 2);
  L.dn = take(size_t(M) * D * 4);
  // decode-path workspace: the largest need of any call, over every width
  size_t need = 0;
  for (int r : {8, 6, 4, 3, 2}) {
    for (int64_t K : {D, F}) {
      LinearJob j{};
      j.r = r;
      j.K = K;
      j.N = F;
      const size_t b = 2 * gemv_scratch_bytes(j, static_cast<int>(M));  // two linears share a call
      if (b > need) need = b;
    }
  }
  L.ws_bytes = align256(need);
  L.ws = take(L.ws_bytes);
  // grid-barrier words of the short integer decode launches (the arrival
  // count is cleared by the chain's first kernel on every call)
  L.sync = take(256);
  L.total = off;
  return L;
}

struct ChainArgs {
  const mq_chain_layer* layers;
  int n_layers;
  int M, D, Dkv, F, hd;
  float* h;
  uint8_t* scratch;
  uint32_t* err;
};

// Enqueues the whole chain on `s`.
cudaError_t enqueue_chain(const ChainArgs& c, const ChainLayout& L, cudaStream_t s, int sms) {
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(c.scratch + off); };
  auto fp = [&](size_t off) { return reinterpret_cast<float*>(c.scratch + off); };
  uint32_t* sync = reinterpret_cast<uint32_t*>(c.scratch + L.sync);
  const FixedScratch fx{c.scratch + L.ws, L.ws_bytes, c.err, sync};
  const int M = c.M, D = c.D, Dkv = c.Dkv, F = c.F;
  cudaError_t e;
  // xn = bf16(rmsnorm(h)) for the first layer; later layers get it from the
  // previous layer's last norm
  const float* no_add = nullptr;
  float* no_out = nullptr;
  e = launch_pdl(rmsnorm_kernel, dim3(M), dim3(kGlueThreads), 0, s, static_cast<const float*>(c.h), no_add,
                 no_out, bf(L.xn), D, sync);
  if (e != cudaSuccess) return e;
  for (int l = 0; l < c.n_layers; ++l) {
    const mq_chain_layer& Ly = c.layers[l];
    auto job = [&](int which, const void* x, int64_t N, int64_t K, float* y) {
      LinearJob j{};
      j.x = x;
      j.packed = static_cast<const uint8_t*>(Ly.packed[which]);
      j.alpha = Ly.alpha[which];
      j.zero = Ly.zero[which];
      j.y = y;
      j.N = N;
      j.K = K;
      j.r = Ly.r;
      return j;
    };
    LinearJob jq = job(0, bf(L.xn), D + 2 * Dkv, D, fp(L.qkv));
    if ((e = run_gemv_fixed_n(&jq, 1, M, s, fx)) != cudaSuccess) return e;
    e = launch_pdl(attn_one_token_kernel, dim3(glue_grid(int64_t(M) * D, sms)), dim3(kGlueThreads), 0, s,
                   static_cast<const float*>(fp(L.qkv)), bf(L.a), M, D, Dkv, c.hd);
    if (e != cudaSuccess) return e;
    LinearJob jo = job(1, bf(L.a), D, D, fp(L.o));
    if ((e = run_gemv_fixed_n(&jo, 1, M, s, fx)) != cudaSuccess) return e;
    e = launch_pdl(rmsnorm_kernel, dim3(M), dim3(kGlueThreads), 0, s, static_cast<const float*>(c.h),
                   static_cast<const float*>(fp(L.o)), fp(L.h1), bf(L.xn1), D, static_cast<uint32_t*>(nullptr));
    if (e != cudaSuccess) return e;
    LinearJob jgu[2] = {job(2, bf(L.xn1), F, D, fp(L.g)), job(3, bf(L.xn1), F, D, fp(L.u))};
    if ((e = run_gemv_fixed_n(jgu, 2, M, s, fx)) != cudaSuccess) return e;
    e = launch_pdl(swiglu_kernel, dim3(glue_grid(int64_t(M) * F, sms)), dim3(kGlueThreads), 0, s,
                   static_cast<const float*>(fp(L.g)), static_cast<const float*>(fp(L.u)), bf(L.act),
                   int64_t(M) * F);
    if (e != cudaSuccess) return e;
    LinearJob jd = job(4, bf(L.act), D, F, fp(L.dn));
    if ((e = run_gemv_fixed_n(&jd, 1, M, s, fx)) != cudaSuccess) return e;
    // h = h1 + down, and the next layer's normalized input (none after the
    // last layer, whose intermediates then all stay in the scratch)
    __nv_bfloat16* next_xn = l + 1 < c.n_layers ? bf(L.xn) : nullptr;
    e = launch_pdl(rmsnorm_kernel, dim3(M), dim3(kGlueThreads), 0, s, static_cast<const float*>(fp(L.h1)),
                   static_cast<const float*>(fp(L.dn)), c.h, next_xn, D, static_cast<uint32_t*>(nullptr));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Instantiated graphs of earlier identical calls, keyed by every argument.
std::mutex g_graph_mutex;
std::map<std::vector<uint64_t>, cudaGraphExec_t> g_graphs;

}  // namespace

size_t chain_scratch_bytes(int64_t M, int64_t D, int64_t Dkv, int64_t F) {
  return chain_layout(M, D, Dkv, F).total;
}

void chain_views(int64_t M, int64_t D, int64_t Dkv, int64_t F, size_t out[10]) {
  const ChainLayout L = chain_layout(M, D, Dkv, F);
  const size_t v[10] = {L.xn, L.qkv, L.a, L.o, L.h1, L.xn1, L.g, L.u, L.act, L.dn};
  for (int i = 0; i < 10; ++i) out[i] = v[i];
}

cudaError_t run_chain(const mq_chain_layer* layers, int n_layers, int M, int D, int Dkv, int F, int hd,
                      float* h, void* scratch, bool use_graph, cudaStream_t stream) {
  const ChainLayout L = chain_layout(M, D, Dkv, F);
  uint32_t* err = nullptr;
  cudaError_t e = get_error_word(&err);
  if (e != cudaSuccess) return e;
  const ChainArgs c{layers, n_layers, M, D, Dkv, F, hd, h, static_cast<uint8_t*>(scratch), err};
  const int sms = sm_count();
  if (!use_graph || stream == nullptr) return enqueue_chain(c, L, stream, sms);

  int dev = 0;
  cudaGetDevice(&dev);
  std::vector<uint64_t> key = {uint64_t(dev), reinterpret_cast<uint64_t>(stream), uint64_t(n_layers),
                               uint64_t(M), uint64_t(D), uint64_t(Dkv), uint64_t(F), uint64_t(hd),
                               reinterpret_cast<uint64_t>(h), reinterpret_cast<uint64_t>(scratch),
                               wait_limit_ns()};
  for (int l = 0; l < n_layers; ++l) {
    key.push_back(uint64_t(layers[l].r));
    for (int i = 0; i < 5; ++i) {
      key.push_back(reinterpret_cast<uint64_t>(layers[l].packed[i]));
      key.push_back(reinterpret_cast<uint64_t>(layers[l].alpha[i]));
      key.push_back(reinterpret_cast<uint64_t>(layers[l].zero[i]));
    }
  }
  std::lock_guard<std::mutex> lk(g_graph_mutex);
  auto it = g_graphs.find(key);
  if (it != g_graphs.end()) return cudaGraphLaunch(it->second, stream);
  // The first call of a new argument set runs directly (it also completes
  // every lazy set-up of the decode path, none of which may happen inside a
  // capture); the second one is captured and instantiated.
  static std::map<std::vector<uint64_t>, int> seen;
  if (seen[key]++ == 0) return enqueue_chain(c, L, stream, sms);
  e = cudaStreamBeginCapture(stream, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) return e;
  const cudaError_t eq = enqueue_chain(c, L, stream, sms);
  cudaGraph_t graph = nullptr;
  e = cudaStreamEndCapture(stream, &graph);
  if (eq != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return eq;
  }
  if (e != cudaSuccess) return e;
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiateWithFlags(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) return e;
  seen.erase(key);
  g_graphs.emplace(std::move(key), exec);
  return cudaGraphLaunch(exec, stream);
}

void release_chain_graphs() {
  std::lock_guard<std::mutex> lk(g_graph_mutex);
  for (auto& kv : g_graphs) cudaGraphExecDestroy(kv.second);
  g_graphs.clear();
}

}  // namespace mq
