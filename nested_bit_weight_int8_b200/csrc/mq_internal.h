// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include <cstdint>
#include <vector>

namespace mq {

// One sliced linear as the host planner sees it (device pointers).
struct LinearJob {
  const void* x;        // M x K bf16
  const uint8_t* packed;
  const float* alpha;
  const float* zero;
  float* y;             // M x N fp32
  int64_t N;
  int64_t K;
  int r;
  // Where the codes come from: kPlanes (packed r-bit planes of width r), or
  // the int8 container itself, sliced on load with Eq. 6 (kContainer) or
  // with the unclamped Eq. 8 (kContainerEP, 2^r + 1 levels).
  int src = 0;
  // Extra Precision on the planes (Eq. 8 from Eq. 6 planes plus a sparse
  // list): per row n the positions ep_cols[ep_rows[n] .. ep_rows[n+1]) whose
  // code is one step higher; null for none.
  const int32_t* ep_rows = nullptr;
  const uint16_t* ep_cols = nullptr;
};
constexpr int kPlanes = 0, kContainer = 1, kContainerEP = 2;

// Plane widths of a width r: b0 (low bits) and b1 (high bits, 0 if none).
inline void plane_widths(int r, int& b0, int& b1) {
  switch (r) {
    case 8: b0 = 8; b1 = 0; return;
    case 6: b0 = 4; b1 = 2; return;
    case 4: b0 = 4; b1 = 0; return;
    case 3: b0 = 2; b1 = 1; return;
    case 2: b0 = 2; b1 = 0; return;
    default: b0 = 0; b1 = 0; return;
  }
}
// Plane widths a job streams: the container is one 8-bit plane.
inline void job_planes(const LinearJob& j, int& b0, int& b1) {
  if (j.src != kPlanes) { b0 = 8; b1 = 0; return; }
  plane_widths(j.r, b0, b1);
}
// Decode kind of a job in the decode kernel: the width r for planes (and for
// the container at r = 8, whose bytes are the r = 8 plane), 10 for the
// container sliced with Eq. 6, 11 for the container with Eq. 8.
inline int decode_kind(const LinearJob& j) {
  if (j.src == kPlanes || j.r == 8) return j.r;
  return j.src == kContainer ? 10 : 11;
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while its predecessor in the stream finishes, so it must execute
// griddepcontrol.wait before touching any memory the predecessor may use.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Per-(device, stream) scratch owned by the library.
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
// Returns a workspace of at least `bytes` for the current device and
// `stream`, growing it if needed (growth synchronizes the device). Each
// workspace starts with kSyncBytes of grid-barrier words, zeroed when it is
// allocated, that the decode launches without a prep kernel use: `sync` (if
// not null) receives their address, `out` the bytes after them.
constexpr size_t kSyncBytes = 256;
cudaError_t get_workspace(cudaStream_t stream, size_t bytes, void** out, uint32_t** sync = nullptr);
// Device error word of the current device (zero-initialized).
cudaError_t get_error_word(uint32_t** out);
uint64_t wait_limit_ns();
// Replaces the calling thread's mq_last_error() text.
void set_last_error(const char* msg);

// 2-D tensor map over a row-major matrix of `rows` x `row_elems` elements of
// `elem_bytes` bytes (1: uint8, 2: bf16), box `box_inner` x `box_rows`,
// out-of-bounds elements read as zero. `swizzle_bytes` 0 stores the box
// plainly; 32, 64 or 128 stores its rows in swizzled atoms of that span
// (box_inner * elem_bytes must equal it; the 16-byte chunk c of row r then sits
// at chunk c ^ ((r / (128 / span)) % (span / 16)) and the destination must be
// aligned to 8 rows of the span). Cached per arguments.
cudaError_t encode_map_2d(CUtensorMap* out, const void* base, uint64_t rows, uint64_t row_elems,
                          uint32_t box_inner, uint32_t box_rows, int elem_bytes,
                          int swizzle_bytes = 0);
int sm_count();

// gamma, beta: per-row clipping factors of Eq. 3, or null for Eq. 1.
cudaError_t launch_quantize(const void* w, int dtype, int64_t N, int64_t K, const float* gamma,
                            const float* beta, uint8_t* q, float* alpha, float* zero,
                            cudaStream_t stream, int sms);
cudaError_t launch_slice_pack(const uint8_t* q, int64_t N, int64_t K, int r, void* packed,
                              cudaStream_t stream, int sms);

// Decode path (M <= 32): plans, stages activations and launches the
// persistent stream-K GEMV over all jobs (at most kGemvMaxLinears).
constexpr int kGemvMaxLinears = 256;
cudaError_t run_gemv(const LinearJob* jobs, int n_jobs, int M, cudaStream_t stream);

// Caller-provided device scratch for the decode path: `ptr` (256-byte
// aligned, `bytes` long) replaces the per-stream workspace and `err` the
// per-device error word. Used by the entry point that allocates nothing.
struct FixedScratch {
  void* ptr;
  size_t bytes;
  uint32_t* err;
  uint32_t* sync;  // grid-barrier words (zero-initialized)
};
// Reads and clears the wait-error word of mq_linear_noalloc's fixed array on
// the current device (0 if that entry point never ran there).
cudaError_t noalloc_take_error(uint32_t* flags);
// The per-device error word if it exists already (null otherwise); never
// allocates.
uint32_t* find_error_word();
// Scratch bytes the decode path needs for one linear at batch M.
size_t gemv_scratch_bytes(const LinearJob& job, int M);
// Decode path for one linear on caller-provided scratch; returns
// cudaErrorMemoryAllocation if the scratch is too small (nothing launched).
cudaError_t run_gemv_fixed(const LinearJob& job, int M, cudaStream_t stream,
                           const FixedScratch& scratch);

// Extra Precision positions of a container at width r (Eq. 8 vs Eq. 6):
// row offsets (count + scan), then the columns.
cudaError_t launch_ovf_rows(const uint8_t* q, int64_t N, int64_t K, int r, int32_t* row_ptr,
                            cudaStream_t stream, int sms);
cudaError_t launch_ovf_cols(const uint8_t* q, int64_t N, int64_t K, int r, const int32_t* row_ptr,
                            uint16_t* cols, cudaStream_t stream, int sms);

// Decode path for up to 8 linears on caller-provided scratch.
cudaError_t run_gemv_fixed_n(const LinearJob* jobs, int n_jobs, int M, cudaStream_t stream,
                             const FixedScratch& scratch);

// Chained decoder stack (mq_chain_forward): scratch bytes, and the run, with
// graph capture and replay of repeated identical calls when `use_graph`.
size_t chain_scratch_bytes(int64_t M, int64_t D, int64_t Dkv, int64_t F);
// Offsets of the last layer's intermediates (xn, qkv, a, o, h1, xn1, g, u,
// act, down) inside the chain's scratch.
void chain_views(int64_t M, int64_t D, int64_t Dkv, int64_t F, size_t out[10]);
cudaError_t run_chain(const struct mq_chain_layer* layers, int n_layers, int M, int D, int Dkv, int F,
                      int hd, float* h, void* scratch, bool use_graph, cudaStream_t stream);
void release_chain_graphs();
// The bounded cache of tensor-map tables of large decode launches: frees all
// of it (after the devices finish), and its current size.
void release_map_tables();
size_t map_table_count();

// Prefill path (M > 32): tcgen05 GEMM for one linear. Returns
// cudaErrorNotSupported for shapes it does not serve (nothing launched).
cudaError_t run_gemm(const LinearJob& job, int M, cudaStream_t stream);
// An Extra Precision list as a bit plane (N rows of K / 32 words; K % 32 == 0)
// for the prefill GEMM.
cudaError_t launch_ep_bits(const int32_t* row_ptr, const uint16_t* cols, int64_t N, int64_t K, uint32_t* bits,
                           cudaStream_t stream, int sms);

// An NVTX range around every entry point that launches work, so a timeline
// tool shows each library call (without a tool attached it costs a branch).
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace mq
