/*
 * mq.h -- C ABI of the nested-bit int8 (Matryoshka Quantization) serving path
 * for NVIDIA B200 (sm_100a).
 *
 * One int8 container per weight matrix serves every width r in {8, 6, 4, 3, 2}:
 * the r most significant bits are sliced out (Eq. 6), stored as dense r-bit
 * planes and consumed by a fused unpack -> dequantize -> matmul.
 * Sources ("Matryoshka Quantization" explainer page): section 3.4 Eq. 1
 * (MinMax quantizer), "The Bit-Slicing Operator" Eq. 6, section 3.2
 * ("at deployment, only the int8-quantized model needs to be stored; lower
 * precisions are extracted by slicing") and "Mix'n'Match and Interpolative
 * Slicing" (per-layer widths, r = 3 and 6 from the same container).
 *
 * Conventions for every call:
 *  - Tensor pointers are DEVICE pointers owned by the caller, unless a
 *    comment says otherwise. Every tensor is dense and row-major.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Calls enqueue work on it and return without synchronizing.
 *  - Arguments are checked on the host before anything is launched. A
 *    rejected call launches nothing and returns MQ_ERR_INVALID_ARG (bad
 *    value, null or misaligned pointer) or MQ_ERR_UNSUPPORTED (a valid value
 *    this build does not serve); mq_last_error() then describes it.
 *  - A CUDA launch failure returns MQ_ERR_CUDA. A bounded device-side wait
 *    that gave up is reported by mq_device_status() as MQ_ERR_TIMEOUT.
 *  - A library built with MQ_DEBUG_BOUNDS (libmq_debug.so) checks its device
 *    indices (activation layout, shared-memory reads, Extra Precision
 *    columns); a failed check skips the access and mq_device_status()
 *    reports MQ_ERR_BOUNDS. The normal build compiles the checks out.
 *  - No C++ exception crosses this interface.
 *  - The library keeps a small per-(device, stream) workspace of device
 *    memory for its own scratch (activation copies, row sums, the two
 *    grid-barrier words of short decode calls, error word). It is allocated
 *    on first use by a call on that stream; make one call before capturing
 *    such a stream into a CUDA graph. Calls on one stream use its workspace
 *    in order, so a graph captured on a stream must not run concurrently
 *    with other calls on that stream's workspace. mq_release_workspace()
 *    frees all of it.
 */
#ifndef MQ_H_
#define MQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MQ_API __attribute__((visibility("default")))
#else
#define MQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mq_status {
  MQ_OK = 0,
  MQ_ERR_INVALID_ARG = 1,
  MQ_ERR_UNSUPPORTED = 2,
  MQ_ERR_CUDA = 3,
  MQ_ERR_TIMEOUT = 4,
  MQ_ERR_BOUNDS = 5,
  MQ_ERR_IO = 6
} mq_status;

typedef enum mq_dtype { MQ_F32 = 0, MQ_BF16 = 1 } mq_dtype;

/* Library version, (major << 16) | minor. */
MQ_API int mq_version(void);

/* Text of the last error raised on the calling thread ("" if none). The
 * pointer stays valid until the next mq_* call on the same thread. */
MQ_API const char* mq_last_error(void);

/*
 * Bytes of the dense r-bit planes of an N x K matrix: N*K*r/8.
 * Returns 0 for N < 1, r not in {8, 6, 4, 3, 2}, or K not a positive multiple
 * of the width's K unit: every plane row (K*b/8 bytes for a plane of width b)
 * must be a whole number of 16-byte units, so K % 32 at r = 8 and 4, K % 64
 * at r = 6 and 2 (a 2-bit plane), K % 128 at r = 3 (a 1-bit plane).
 * Layout (this library's own; the pages fix only that a slice is an r-bit
 * integer per weight): r = 8 -> one plane of bytes (the container itself);
 * r = 4, 2 -> one plane of width r; r = 3 -> planes of widths (2, 1);
 * r = 6 -> planes of widths (4, 2). Plane 0 holds the low bits of each code,
 * plane 1 the code shifted right by plane 0's width; the planes follow one
 * another, each row-major with a row pitch of K*b/8 bytes. In a plane of
 * width b < 8 every little-endian 32-bit word holds 32/b codes; local code
 * u sits at bit 16*(u % 2) + b*(u / 2) (even codes in the low half-word, odd
 * codes in the high half-word). In the byte plane code u sits at bit 8u.
 */
MQ_API size_t mq_packed_bytes(int64_t N, int64_t K, int r);

/*
 * Eq. 1, MinMax asymmetric quantization of each output channel (row) of a
 * weight matrix into the int8 container:
 *   alpha_n = (max_k w[n,k] - min_k w[n,k]) / 255,  z_n = -min_k w[n,k] / alpha_n,
 *   q[n,k]  = clamp(round(w[n,k] / alpha_n + z_n), 0, 255).
 * Arithmetic contract (IEEE binary32, each operation correctly rounded, no
 * contraction): d = max - min; alpha = d / 255; z = -min / alpha;
 * t = (w / alpha) + z; q = clamp(round-half-to-even(t), 0, 255). A row whose
 * alpha rounds to 0 (max == min) gets alpha = max(|min| 2^-8, 2^-126) and
 * z = -min / alpha (exact: all codes 0 and alpha (0 - z) = min).
 *   w     : N x K, fp32 (dtype MQ_F32) or bf16 (MQ_BF16), 4-byte aligned.
 *   q     : N x K uint8 out.   alpha, zero : N fp32 out.
 * Requires N >= 1, K >= 1; weights finite with a finite range.
 */
MQ_API mq_status mq_quantize_int8(const void* w, int dtype, int64_t N, int64_t K,
                           uint8_t* q, float* alpha, float* zero, void* stream);

/*
 * Eq. 3, OmniQuant's clipped MinMax quantization into the int8 container,
 * with the clipping factors given (learning them is training, not serving):
 *   alpha_n = (gamma_n * max_k w[n,k] - beta_n * min_k w[n,k]) / 255,
 *   z_n     = -(beta_n * min_k w[n,k]) / alpha_n,
 *   q[n,k]  = clamp(round(w[n,k] / alpha_n + z_n), 0, 255),
 * so weights outside [beta_n min, gamma_n max] saturate at 0 or 255. Same
 * arithmetic contract as mq_quantize_int8, with gmax = gamma * max and
 * bmin = beta * min rounded first; a row whose clipped range is empty or
 * inverted (alpha <= 0) gets alpha = max(|bmin| 2^-8, 2^-126) and
 * z = -bmin / alpha. gamma = beta = 1 gives
 * exactly mq_quantize_int8.
 *   gamma, beta : N fp32 (device), 4-byte aligned, finite (OmniQuant keeps
 *                 them in (0, 1)). Other arguments as mq_quantize_int8.
 */
MQ_API mq_status mq_quantize_int8_clipped(const void* w, int dtype, int64_t N, int64_t K,
                                          const float* gamma, const float* beta, uint8_t* q,
                                          float* alpha, float* zero, void* stream);

/*
 * Eq. 6 slicing of the container into width r, packed as dense r-bit planes:
 *   code[n,k] = clamp(round_half_up(q[n,k] / 2^(8-r)), 0, 2^r - 1)
 * (S(q, r) = code * 2^(8-r); r = 8 is the identity). The first dropped bit
 * decides the rounding, as the slicing paragraph states.
 *   q      : N x K uint8 container (from mq_quantize_int8), 16-byte aligned.
 *   packed : mq_packed_bytes(N, K, r) bytes out, 16-byte aligned.
 * Requires r in {8, 6, 4, 3, 2} and K a multiple of the width's K unit (see
 * mq_packed_bytes: 32, 64 or 128).
 */
MQ_API mq_status mq_slice_pack(const uint8_t* q, int64_t N, int64_t K, int r,
                        void* packed, void* stream);

/*
 * Fused unpack -> dequantize -> matmul with a sliced width r:
 *   y[m,n] = sum_k x[m,k] * alpha_n * (S(q[n,k], r) - z_n)
 * (dequantization alpha * (q - z) of Eq. 1 with the sliced code in place of
 * q). x is bf16, accumulation is fp32, y is fp32.
 *   x      : M x K bf16, 16-byte aligned.
 *   packed : planes of width r from mq_slice_pack, 16-byte aligned.
 *   alpha, zero : N fp32 (from mq_quantize_int8).
 *   y      : M x N fp32 out (overwritten), 4-byte aligned.
 * Requires 1 <= M, N >= 1, and K a multiple of the width's K unit (32 at
 * r = 8, 4; 64 at r = 6, 2; 128 at r = 3: every plane row a whole number of
 * 16-byte units for the TMA boxes). M <= 32 runs the decode GEMV (legacy
 * tensor-core tiles fed from TMA-staged planes: at M = 1 and r = 8, 4, 2 the
 * integer m16n8k32 with exact sums, otherwise bf16 m16n8k16); M > 32 runs the
 * prefill GEMM (tcgen05, accumulators in tensor memory).
 * Accuracy: |y - y_exact| <= 1e-3 * sum_k |x[m,k]| |W_r[n,k]| + 1e-6.
 */
MQ_API mq_status mq_linear(const void* x, int64_t M, int64_t K, const void* packed,
                    const float* alpha, const float* zero, int64_t N, int r,
                    float* y, void* stream);

/*
 * Slice on load: the product of mq_linear served straight from the int8
 * container, with no repacked planes (the pages' "extracted on the fly by
 * slicing"). Each byte is sliced as the weights stream, s = 8 - r:
 *   clamp = 1, Eq. 6:  code = min(round_half_up(q / 2^s), 2^r - 1);
 *   clamp = 0, Eq. 8 (the Extra Precision variant of the errata section):
 *                      code = round_half_up(q / 2^s), which reaches 2^r for
 *                      q >= 256 - 2^(s-1), so 2^r + 1 levels;
 *   y[m,n] = sum_k x[m,k] * alpha_n * (code[n,k] * 2^s - z_n).
 * It streams 8 bits per weight: it saves the planes' storage, not bandwidth.
 *   q : N x K uint8 container (row pitch K bytes), 16-byte aligned.
 *   Other arguments and the accuracy bound as mq_linear: M <= 32 runs the
 *   decode GEMV, larger M the prefill GEMM, both slicing while they decode.
 *   Requires K % 32 == 0, clamp in {0, 1}. At r = 8 both forms are the
 *   container.
 */
MQ_API mq_status mq_linear_container(const void* x, int64_t M, int64_t K, const uint8_t* q,
                                     const float* alpha, const float* zero, int64_t N, int r,
                                     int clamp, float* y, void* stream);

/*
 * Extra Precision on the planes (the errata section's Eq. 8, the clamp of
 * Eq. 6 removed): at width r, s = 8 - r, the unclamped code of q is one step
 * (2^s on the 8-bit scale) above the clamped one exactly for
 * q >= 256 - 2^(s-1), the "extra bucket". Those positions are few, so they
 * are kept as a sparse list beside the r-bit planes of Eq. 6, in compressed
 * sparse rows: row n's columns are cols[row_ptr[n] .. row_ptr[n+1]),
 * increasing. Build it in two calls: mq_ep_overflow_rows fills row_ptr
 * (N + 1 int32: counts and their scan, row_ptr[0] = 0); read row_ptr[N]
 * (the total) to size cols; mq_ep_overflow_cols fills cols (uint16).
 *   q : N x K uint8 container, 16-byte aligned, K % 16 == 0, K <= 65536,
 *       N * K < 2^31. r in {6, 4, 3, 2} (r = 8 has no extra bucket).
 *   row_ptr : N + 1 int32 (device), 4-byte aligned. cols : row_ptr[N]
 *       uint16 (device), 2-byte aligned.
 */
MQ_API mq_status mq_ep_overflow_rows(const uint8_t* q, int64_t N, int64_t K, int r,
                                     int32_t* row_ptr, void* stream);
MQ_API mq_status mq_ep_overflow_cols(const uint8_t* q, int64_t N, int64_t K, int r,
                                     const int32_t* row_ptr, uint16_t* cols, void* stream);

/*
 * The Extra Precision product from the Eq. 6 planes plus the sparse list:
 *   y[m,n] = sum_k x[m,k] alpha_n (code8[n,k] 2^s - z_n),
 * code8 the unclamped Eq. 8 code. At M <= 32 (decode) it is the planes'
 * product plus alpha_n 2^s times the sum over row n's listed positions of
 * x[m,k] (the "sparse additions"), gathered by the prep kernel and added in
 * the decode epilogue. At M > 32 (prefill) the list is first laid out as a
 * bit plane (N x K/32 words in the library's workspace) and the GEMM's
 * decode adds one step to each listed code before the tensor cores sum
 * x (code8 - c0). Arguments as mq_linear plus the list of mq_ep_overflow_*;
 * r in {6, 4, 3, 2}, K <= 65536. Accuracy as mq_linear, against W with the
 * Eq. 8 codes.
 */
MQ_API mq_status mq_linear_ep(const void* x, int64_t M, int64_t K, const void* packed,
                              const float* alpha, const float* zero, int64_t N, int r,
                              const int32_t* row_ptr, const uint16_t* cols, float* y,
                              void* stream);

/* One linear of a stack: its input, its packed planes, its scales, its output. */
typedef struct mq_linear_desc {
  const void* x;       /* M x K bf16 input, 16-byte aligned */
  const void* packed;  /* planes at the width of the linear's layer */
  const float* alpha;  /* N */
  const float* zero;   /* N */
  float* y;            /* M x N fp32 output (overwritten) */
  int64_t N;
  int64_t K;
} mq_linear_desc;

/*
 * Mix'n'Match serving: every linear i runs at the width widths[layer_of_lin[i]]
 * of its layer (the pages' per-layer precision assignment; e.g. int8 on the
 * outer layers, int2 in the middle). All linears are independent (each reads
 * its own x), so the whole stack is streamed by one persistent kernel whose
 * work units run across linear boundaries.
 *   lins[n_lins], layer_of_lin[n_lins] : HOST arrays.
 *   widths[n_layers]                  : HOST array, each in {8, 6, 4, 3, 2}.
 * Requires 1 <= M <= 32 and the mq_linear conditions for every linear.
 * Stacks longer than 256 linears are split into several launches.
 * A launch of more than 8 linears reads their plane tensor maps from a device
 * table: one per distinct list (device, planes addresses, N, K, widths),
 * encoded and uploaded with an asynchronous copy on `stream` the first time
 * the list is served, then reused. At most 64 tables (16 MiB) are kept; a new
 * one evicts the least recently used, synchronizing that table's device
 * before freeing it. A table served during a CUDA graph capture is pinned
 * until mq_release_workspace (the graph holds its address); a list first seen
 * during a capture returns MQ_ERR_CUDA (make one call before capturing).
 */
MQ_API mq_status mq_stack_forward(const mq_linear_desc* lins, const int* layer_of_lin,
                           int n_lins, const int* widths, int n_layers,
                           int64_t M, void* stream);

/*
 * A chained decoder stack: each layer's output is the next layer's input, so
 * one call is one token's decode step through n_layers dependent layers. The
 * pages quantize the linears only (each layer at its own Mix'n'Match width)
 * and define no glue between them; the stand-in glue per layer is
 *   xn  = bf16(rmsnorm(h));  qkv = xn Wqkv^T;
 *   a   = bf16(v of each query head's kv group)   (attention over a context
 *         of one token: the softmax over a single score is 1);
 *   h1  = h + a Wo^T;  xn1 = bf16(rmsnorm(h1));
 *   act = bf16(silu(xn1 Wgate^T) * (xn1 Wup^T));  h = h1 + act Wdown^T,
 * with rmsnorm(v) = v / sqrt(mean(v^2) + 1e-6) (no learned scale),
 * silu(g) = g / (1 + exp(-g)), the residual stream h in fp32 and every
 * linear run by the decode path of mq_linear at the layer's width.
 *   layers  : n_layers host descriptors; packed/alpha/zero index 0..4 =
 *             qkv ((D + 2 Dkv) x D), o (D x D), gate (F x D), up (F x D),
 *             down (D x F), each packed at width r.
 *   h       : M x D fp32 (device), the residual stream in and out.
 *   D, Dkv, F, head_dim : model width, key/value width, MLP width, head
 *             size; D and F multiples of 128, head_dim dividing Dkv, and
 *             D / head_dim a multiple of Dkv / head_dim.
 *   scratch : mq_chain_scratch_bytes(M, D, Dkv, F) bytes (device), 256-byte
 *             aligned, owned by the caller; the chain allocates nothing.
 *   flags   : MQ_CHAIN_GRAPH to capture the call into a CUDA graph on its
 *             second identical call (same stream, pointers and sizes) and
 *             replay it from then on; the first call runs directly. Graphs
 *             are freed by mq_release_workspace. Needs a stream other than
 *             the legacy default stream (there the flag is ignored).
 * Requires 1 <= M <= 32.
 */
typedef struct mq_chain_layer {
  int r;
  const void* packed[5];
  const float* alpha[5];
  const float* zero[5];
} mq_chain_layer;
#define MQ_CHAIN_GRAPH 1
MQ_API size_t mq_chain_scratch_bytes(int64_t M, int64_t D, int64_t Dkv, int64_t F);

/*
 * Where mq_chain_forward leaves the intermediate values of its LAST layer
 * inside the caller's scratch: byte offsets from the scratch pointer, valid
 * once the call's stream has completed, for inspecting a token's step (and
 * for checking each step against a reference on the chain's own inputs).
 * Every buffer is row-major with M rows:
 *   xn   M x D bf16           bf16(rmsnorm(h_in)), the input of qkv
 *   qkv  M x (D + 2 Dkv) fp32
 *   a    M x D bf16           the attention output, the input of o
 *   o    M x D fp32           a Wo^T
 *   h1   M x D fp32           h_in + o (fp32 add)
 *   xn1  M x D bf16           bf16(rmsnorm(h1))
 *   g, u M x F fp32           gate and up products
 *   act  M x F bf16           bf16(silu(g) u)
 *   down M x D fp32           act Wdown^T; h_out = h1 + down (fp32 add)
 * Returns MQ_ERR_INVALID_ARG for sizes mq_chain_scratch_bytes rejects.
 */
typedef struct mq_chain_views {
  size_t xn, qkv, a, o, h1, xn1, g, u, act, down;
} mq_chain_views;
MQ_API mq_status mq_chain_scratch_views(int64_t M, int64_t D, int64_t Dkv, int64_t F,
                                        mq_chain_views* out);
MQ_API mq_status mq_chain_forward(const mq_chain_layer* layers, int n_layers, int64_t M, int64_t D,
                                  int64_t Dkv, int64_t F, int64_t head_dim, float* h,
                                  void* scratch, size_t scratch_bytes, int flags, void* stream);

/*
 * The int8 container as a file: the one stored artifact, from which every
 * width is sliced. Host buffers (the caller copies device data). Layout,
 * little-endian: "MQC8", version 1 (uint32), N, K (int64), q (N x K uint8,
 * row-major), alpha, zero (N fp32 each), then the CRC-32 (IEEE, reflected) of
 * everything before it. Errors: MQ_ERR_INVALID_ARG for null pointers, sizes
 * below 1, or a file of another shape (load); MQ_ERR_IO for a file that
 * cannot be opened, written or read, is truncated, has trailing bytes, is not
 * a container of this version, or fails its checksum.
 * mq_container_save writes the file under a temporary name beside `path`
 * (path.tmp.<pid>), checks that it closed cleanly, then renames it over
 * `path`: readers see the old file or the complete new one, and a failed save
 * leaves `path` untouched. mq_container_load reads straight into q, alpha and
 * zero; if it returns an error, their contents are undefined (partly
 * overwritten).
 */
MQ_API mq_status mq_container_save(const char* path, const uint8_t* q, const float* alpha,
                                   const float* zero, int64_t N, int64_t K);
MQ_API mq_status mq_container_info(const char* path, int64_t* N, int64_t* K);
MQ_API mq_status mq_container_load(const char* path, uint8_t* q, float* alpha, float* zero,
                                   int64_t N, int64_t K);

/* Bytes of the device array that mq_linear_noalloc works in (1.25 MiB). */
#define MQ_NOALLOC_SCRATCH_BYTES (1280u * 1024u)

/*
 * mq_linear_noalloc -- the decode GEMV of mq_linear (1 <= M <= 32) without any
 * device allocation. The paper has no counterpart: this is a deployment aid.
 *
 * Who needs it: callers that may not, or cannot afford to, call cudaMalloc. For
 * example, a serving engine whose own allocator owns every byte of HBM. Or a
 * plugin loaded into a host program that forbids it to allocate. Or a
 * latency-critical decode loop where an allocation, and the device-wide
 * synchronization it can imply, is not acceptable. mq_linear would allocate
 * its per-stream workspace and error word on first use; this entry point
 * does not.
 *
 * Instead its scratch lives in one file-scope device array of
 * MQ_NOALLOC_SCRATCH_BYTES. The first 256 bytes hold a wait-error word; the
 * rest holds the fragment-ordered activation blocks and activation sums.
 * Every GPU that loads the library holds this array until the process exits.
 * It is enough for M * K up to 524288 (e.g. M = 32 with K = 16384), except
 * at M = 1 with r = 8, 4 or 2, whose inputs are staged as seven integer
 * digits (7.1 to 7.5 bytes each): there K up to 174592, 180480 and 183808.
 * A call that needs more returns MQ_ERR_INVALID_ARG with the sizes in
 * mq_last_error() and launches nothing.
 *
 * Arguments, layouts and accuracy: as mq_linear, with 1 <= M <= 32.
 *
 * Set-up: the first call on each device (with that device current) looks up
 * the array's device address and zeroes its error word with a synchronous
 * cudaMemset plus a device synchronization. Make that first call before any
 * stream capture.
 *
 * Sharing: every call uses the same array, and the array keeps what the last
 * call wrote. Each call rewrites on the device all the scratch it reads, and
 * zeroes y there before accumulating. Calls whose kernels overlap on the GPU race: two streams,
 * or two host threads on one device. Serialize them. A bounded wait that gave
 * up leaves y undefined and is recorded in the array's error word;
 * mq_device_status() reads and clears that word too (as MQ_ERR_TIMEOUT) and
 * allocates nothing, so such a caller can check its calls with it.
 */
MQ_API mq_status mq_linear_noalloc(const void* x, int64_t M, int64_t K, const void* packed,
                                   const float* alpha, const float* zero, int64_t N, int r,
                                   float* y, void* stream);

/*
 * Synchronizes `stream`, then reports whether any kernel launched by this
 * library on the current device gave up a bounded wait (MQ_ERR_TIMEOUT; the
 * outputs of that call are then undefined) and clears the flag. It reads the
 * error word of the per-device workspace and that of mq_linear_noalloc's
 * fixed array, and allocates nothing. Returns MQ_ERR_CUDA if the
 * synchronization itself failed.
 */
MQ_API mq_status mq_device_status(void* stream);

/* Frees every workspace of this library (all devices and streams) and its
 * tensor-map tables (see mq_stack_forward). The caller must ensure no mq_*
 * work is still in flight, and must not replay a CUDA graph that captured an
 * mq_* call afterwards. */
MQ_API mq_status mq_release_workspace(void);

/*
 * Testing hook: the number of tensor-map tables the library holds (a stack
 * with more linears than fit in one launch's parameters reads its plane maps
 * from a device table, one per distinct list of linears; at most 64 are kept,
 * least recently used first out). Allocates nothing.
 */
MQ_API int64_t mq_debug_map_table_count(void);

/*
 * Testing hook: the time (ns) a kernel waits on a pipeline barrier before it
 * gives up, sets the device error flag and exits cleanly. 0 makes every such
 * wait give up at once (deterministic exercise of the timeout path). The
 * default is 2 s. Applies to launches made after the call.
 */
MQ_API mq_status mq_debug_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* MQ_H_ */
