// Prefill path (M > 32): y = x . W_r^T with W_r[n,k] = alpha_n (S(q[n,k], r) - z_n)
// on the fifth-generation tensor cores ("Matryoshka Quantization" explainer
// page: Eq. 1 dequantization alpha*(q - z), Eq. 6 slicing; "Mix'n'Match and
// Interpolative Slicing" for the widths 6 and 3 served from the same int8
// container).
//
// With codes c[n,k] = S(q[n,k], r) / 2^(8-r) and c0_n the code nearest to
// z_n / 2^(8-r), the product factors as
//   y[m,n] = A_n * sum_k x[m,k] (c[n,k] - c0_n) - B_n * Sx[m],
//   A_n = alpha_n 2^(8-r),  B_n = alpha_n (z_n - c0_n 2^(8-r)),  Sx[m] = sum_k x[m,k],
// so the contraction runs on exact integer operands (c - c0 lies in
// [-255, 255], exact in bf16; products and sums are fp32), and the sums stay
// small where the dequantized weights are small.
//
// Tile: 128 weight rows (n) x 256 batch rows (m), K in stages of 64 codes.
// The weights are the MMA's A operand and live in tensor memory; x is the B
// operand in shared memory (128-byte swizzled, K-major), so D = W x^T sits in
// tensor memory with one weight row per lane and one batch row per column.
// The 256-wide batch tile (the largest MMA N) spends each decoded weight on
// twice the arithmetic of a square tile: the decode is ALU work that must
// stay below the MMA time of a stage.
//   warp 0      : TMA producer (x box, plane boxes) into a ring of stages
//   warp 1      : allocates tensor memory, issues tcgen05.mma (one thread)
//   warps 4..19 : decode, two groups of eight taking alternate stages: each
//                 thread owns one weight row (its TMEM lane) and
//                 32 of the stage's 64 codes, unpacks them from the staged
//                 planes to bf16 and writes them to tensor memory
//                 (tcgen05.st); then the same warps run the epilogue.
// Every mbarrier wait is bounded; a wait that gives up sets the device error
// word, the CTA drains its copies and MMAs, frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <map>
#include <mutex>

#include "mq_device.cuh"
#include "mq_internal.h"
#include "tc05.cuh"

namespace mq {
namespace {

constexpr int kBN = 128;          // weight rows per CTA (MMA M, TMEM lanes)
constexpr int kBM = 256;          // batch rows per CTA (MMA N, TMEM columns)
constexpr int kBK = 64;           // codes of K per stage
constexpr int kStages = 5;
constexpr int kGemmThreads = 20 * 32;
constexpr int kDecodeWarp0 = 4;   // warps 4..19 decode, then run the epilogue
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;                 // D: columns [0, 256)
constexpr uint32_t kASlotCol = 256;             // A slot s: columns [256 + 32 s, +32)
constexpr uint32_t kXStageBytes = kBM * kBK * 2;      // one 64-code swizzled tile, 32 KB
constexpr uint32_t kHeaderBytes = 1024;

struct GemmParams {
  CUtensorMap map_x;       // x: M x K bf16, box 64 x 256, 128-byte swizzle
  CUtensorMap map_p0;      // plane 0: N rows x K*b0/8 bytes, box 8*b0 x 128
  CUtensorMap map_p1;      // plane 1 (widths 3, 6): box 16 bytes x 128
  const float* alpha;
  const float* zero;
  const float* sx;         // Sx[m] = sum_k x[m,k]
  float* y;                // M x N fp32
  uint32_t* err;
  unsigned long long wait_ns;
  int M, N, K, r;
  uint32_t stage_bytes;    // x sub-tiles + plane 0 box + plane 1 box, 1024-aligned
  uint32_t off_p0, off_p1; // plane boxes within a stage
  // Extra Precision (Eq. 8): the listed positions as a bit plane, row n's
  // bit k at word n * ep_words + k / 32, bit k % 32 (null without a list)
  const uint32_t* ep_bits;
  int ep_words;
};

// ------------------------------------------------------------ Sx kernel
// Sx[m] = sum_k x[m,k] in fp32, one CTA per batch row.
__global__ void __launch_bounds__(256) rowsum_kernel(const __nv_bfloat16* __restrict__ x, int K,
                                                     float* __restrict__ sx) {
  const __nv_bfloat16* row = x + static_cast<int64_t>(blockIdx.x) * K;
  float acc = 0.f;
  for (int k0 = threadIdx.x * 8; k0 < K; k0 += blockDim.x * 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + k0);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xFFFF0000u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) v += red[i];
    sx[blockIdx.x] = v;
  }
}

// ------------------------------------------------------------ decode
// bf16x2 128.0 in both halves: OR-ing a code c < 128 into the mantissa gives
// 128 + c exactly. Each decode thread owns one weight row and subtracts
// 128 + c0 of that row, c0 the code nearest to the row's zero point (sub2),
// which leaves the integer c - c0: the MMA then sums x (c - c0), small where
// the dequantized weights are small, instead of x c.
constexpr uint32_t kMag128x2 = 0x43004300u;

__device__ __forceinline__ uint32_t exact_pair(uint32_t codes2, uint32_t sub2) {
  uint32_t d;
  // bf16x2 subtract (exact: both operands and the result are small integers)
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(codes2 | kMag128x2), "r"(sub2));
  return d;
}

// Two container bytes (0..255) minus c0 as an exact bf16x2 pair, through
// fp32: 2^23 + c is built by placing c in the low mantissa byte, and subf =
// 2^23 + c0 is subtracted.
__device__ __forceinline__ uint32_t exact_pair_bytes(uint32_t w, uint32_t sel_lo, uint32_t sel_hi, float subf) {
  const float f0 = __uint_as_float(__byte_perm(w, 0x4B000000u, sel_lo)) - subf;
  const float f1 = __uint_as_float(__byte_perm(w, 0x4B000000u, sel_hi)) - subf;
  const __nv_bfloat162 b = __floats2bfloat162_rn(f0, f1);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// Unpacks 32 consecutive codes of one weight row into 16 bf16x2 registers
// (register j holds codes 2j, 2j+1: the even code in the low half, as the
// A operand in tensor memory expects). `p0` / `p1` point at this row's 32-code
// slice of plane 0 / plane 1 in shared memory. Plane word layout: local code
// u of a width-b word sits at bit 16*(u%2) + b*(u/2) (b < 8), at 8u for b = 8.
// R = 10 / 11: the int8 container sliced on load by Eq. 6 / Eq. 8 (runtime
// width r): code = min(q + 2^(s-1), 255) >> s, or (q + 2^(s-1)) >> s, on the
// two 16-bit halves at once (h2 = 2^(s-1) in both halves, kmask the code's
// bits in both halves after the shift by s).
// epw (planes of width 2, 3, 4, 6): the Extra Precision steps of the 32
// codes, bit j for code 2j and bit 16 + j for code 2j + 1; each set bit adds
// one to its code (the Eq. 8 code is the Eq. 6 code plus one there, at most
// 2^r <= 64, still under the magic 128).
template <int R>
__device__ __forceinline__ void decode32(const uint8_t* p0, const uint8_t* p0b, const uint8_t* p1,
                                         uint32_t (&v)[16], uint32_t sub2, float subf, uint32_t h2 = 0,
                                         uint32_t kmask = 0, int sh = 0, uint32_t epw = 0) {
  if constexpr (R == 10 || R == 11) {
    const uint4 a = *reinterpret_cast<const uint4*>(p0);
    const uint4 b = *reinterpret_cast<const uint4*>(p0b);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      // codes 2j, 2j+1 are bytes (0, 1) or (2, 3) of word j / 2
      const uint32_t t = __byte_perm(w[j / 2], 0u, (j % 2 == 0) ? 0x4140u : 0x4342u);
      const uint32_t u = (R == 10) ? __viaddmin_u16x2(t, h2, 0x00FF00FFu) : t + h2;
      v[j] = exact_pair((u >> sh) & kmask, sub2);
    }
  } else if constexpr (R == 2) {
    const uint2 a = *reinterpret_cast<const uint2*>(p0);
    const uint32_t w[2] = {a.x, a.y};
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = exact_pair(((w[j / 8] >> (2 * (j % 8))) & 0x00030003u) + ((epw >> j) & 0x00010001u), sub2);
  } else if constexpr (R == 4) {
    const uint4 a = *reinterpret_cast<const uint4*>(p0);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = exact_pair(((w[j / 4] >> (4 * (j % 4))) & 0x000F000Fu) + ((epw >> j) & 0x00010001u), sub2);
  } else if constexpr (R == 3) {
    const uint2 a = *reinterpret_cast<const uint2*>(p0);
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p1);
    const uint32_t w[2] = {a.x, a.y};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t lo = (w[j / 8] >> (2 * (j % 8))) & 0x00030003u;
      const uint32_t hi = ((u >> j) & 0x00010001u) << 2;
      v[j] = exact_pair((lo | hi) + ((epw >> j) & 0x00010001u), sub2);
    }
  } else if constexpr (R == 6) {
    const uint4 a = *reinterpret_cast<const uint4*>(p0);
    const uint2 h = *reinterpret_cast<const uint2*>(p1);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
    const uint32_t u[2] = {h.x, h.y};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t lo = (w[j / 4] >> (4 * (j % 4))) & 0x000F000Fu;
      const uint32_t hi = ((u[j / 8] >> (2 * (j % 8))) & 0x00030003u) << 4;
      v[j] = exact_pair((lo | hi) + ((epw >> j) & 0x00010001u), sub2);
    }
  } else {  // R == 8: bytes, 4 codes per word
    const uint4 a = *reinterpret_cast<const uint4*>(p0);
    const uint4 b = *reinterpret_cast<const uint4*>(p0b);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = (j % 2 == 0) ? exact_pair_bytes(w[j / 2], 0x7440u, 0x7441u, subf)
                          : exact_pair_bytes(w[j / 2], 0x7442u, 0x7443u, subf);
  }
}

// The 32 position bits m of a half stage (bit i: code i) rearranged for
// decode32: the even codes' bits to bits 0..15, the odd codes' to 16..31.
__device__ __forceinline__ uint32_t spread_even_odd(uint32_t m) {
  auto compact = [](uint32_t e) {  // bits 0, 2, 4, ... of e to bits 0, 1, 2, ...
    e &= 0x55555555u;
    e = (e | (e >> 1)) & 0x33333333u;
    e = (e | (e >> 2)) & 0x0F0F0F0Fu;
    e = (e | (e >> 4)) & 0x00FF00FFu;
    e = (e | (e >> 8)) & 0x0000FFFFu;
    return e;
  };
  return compact(m) | (compact(m >> 1) << 16);
}

// ------------------------------------------------------------ kernel
// EP: the planes carry an Extra Precision bit plane (widths 2, 3, 4, 6).
template <int R, bool EP = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc05_kernel(const __grid_constant__ GemmParams p) {
  static_assert(!EP || R == 2 || R == 3 || R == 4 || R == 6, "Extra Precision needs planes of width <= 6");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base: the swizzled x sub-tiles need it.
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);       // TMA -> decode
  uint64_t* decoded = full + kStages;                        // decode -> MMA
  uint64_t* empty = decoded + kStages;                       // MMA -> TMA, decode
  uint64_t* acc_full = empty + kStages;                      // MMA -> epilogue
  uint64_t* drain = acc_full + 1;                            // MMA completion at exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* stages = smem + kHeaderBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  // a ragged last stage reads past K: the TMA boxes fill it with zeros, and a
  // zero input times any decoded weight adds nothing
  const int n_k = (p.K + kBK - 1) / kBK;
  constexpr int kDecodeWarps = 8;   // per stage: one of the two decode groups

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&decoded[i], kDecodeWarps);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tc05::alloc(smem_u32(tmem_slot), kTmemCols);
    tc05::relinquish();
    tc05::fence_before_sync();
  }
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&p.map_x);
      prefetch_tmap(&p.map_p0);
      int issued = 0;
      // plane 0: 8*b0 bytes (64 codes) per row; plane 1: the 16-byte chunk
      // that holds the stage's codes (64 codes at b1 = 2, 128 at b1 = 1)
      constexpr uint32_t b0 = (R == 8 || R >= 10) ? 8 : (R == 4 || R == 6) ? 4 : 2;
      const uint32_t p0_bytes = 128u * 8u * b0;
      const uint32_t p1_bytes = (R == 3 || R == 6) ? 128u * 16u : 0u;
      for (int it = 0; it < n_k; ++it, ++issued) {
        const int s = it % kStages;
        if (it >= kStages &&
            (*s_abort || !mbar_wait_bounded(&empty[s], ((it / kStages) - 1) & 1, p.wait_ns))) {
          atomicOr(p.err, kErrWaitEmpty);
          *s_abort = 1;
          break;
        }
        uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
        mbar_arrive_expect_tx(&full[s], kXStageBytes + p0_bytes + p1_bytes);
        const int k0 = it * kBK;
        tma_load_2d(st, &p.map_x, k0, m0, &full[s]);
        tma_load_2d(st + p.off_p0, &p.map_p0, it * static_cast<int>(8 * b0), n0, &full[s]);
        if (p1_bytes) {
          const int x1 = (R == 3) ? (it / 2) * 16 : it * 16;
          tma_load_2d(st + p.off_p1, &p.map_p1, x1, n0, &full[s]);
        }
      }
      // no bulk copy may be in flight when this thread leaves
      const int first = issued > kStages ? issued - kStages : 0;
      for (int j = first; j < issued; ++j)
        if (!mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, 1000000000ull)) atomicOr(p.err, kErrDrain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = tc05::idesc_bf16_f32(kBN, kBM);
      bool ok = true;
      for (int it = 0; it < n_k; ++it) {
        const int s = it % kStages;
        if (*s_abort || !mbar_wait_bounded(&decoded[s], (it / kStages) & 1, p.wait_ns)) {
          atomicOr(p.err, kErrMma);
          *s_abort = 1;
          ok = false;
          break;
        }
        tc05::fence_after_sync();
        const uint32_t xs = smem_u32(stages + static_cast<size_t>(s) * p.stage_bytes);
#pragma unroll
        for (int j = 0; j < kBK / 16; ++j) {
          // k16 step j: A columns advance by 8 (two bf16 per column); B advances
          // 32 bytes along its 128-byte swizzled rows.
          const uint64_t bdesc = tc05::desc_kmajor_sw128(xs + j * 32);
          tc05::mma_ts(tmem + kAccCol, tmem + kASlotCol + s * 32 + j * 8, bdesc, idesc,
                       it > 0 || j > 0);
        }
        tc05::commit(smem_u32(&empty[s]));
      }
      if (ok) tc05::commit(smem_u32(acc_full));
      // all MMAs this thread issued have finished before the CTA moves on
      tc05::commit(smem_u32(drain));
      if (!mbar_wait_bounded(drain, 0, 1000000000ull)) atomicOr(p.err, kErrDrain);
    }
  } else if (warp >= kDecodeWarp0) {
    // ---------------------------------------------------------- decode
    // Two groups of eight warps take alternate stages: the decode of a stage
    // is a chain of waits and a tensor-memory store whose latency exceeds the
    // MMA time of one stage, so each group gets two stages' time for it.
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int h = ((warp - kDecodeWarp0) >> 2) & 1;  // which 32 codes of the stage
    const int grp = (warp - kDecodeWarp0) >> 3;      // which stages: it % 2 == grp
    const int row = 32 * q + lane;             // weight row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    constexpr int b0 = (R == 8 || R >= 10) ? 8 : (R == 4 || R == 6) ? 4 : 2;
    // slice-on-load constants (container kinds 10, 11)
    const int cs = 8 - p.r;
    const uint32_t ch2 = (R >= 10) ? (1u << (cs - 1)) * 0x10001u : 0u;
    const uint32_t ckm = (R >= 10) ? ((1u << (R == 10 ? p.r : p.r + 1)) - 1u) * 0x10001u : 0u;
    constexpr int b1 = (R == 3) ? 1 : (R == 6) ? 2 : 0;
    // c0, the code nearest to this row's zero point (clamped to the code
    // range): the decode subtracts it and the epilogue adds alpha c0 2^s back
    const int rw = R >= 10 ? p.r : R;
    const int cmax = R == 11 ? (1 << rw) : (1 << rw) - 1;
    int c0 = 0;
    if (n0 + row < p.N) {
      const float zc = rintf(__ldg(p.zero + n0 + row) * (1.0f / static_cast<float>(1 << (8 - rw))));
      c0 = zc <= 0.f ? 0 : zc >= static_cast<float>(cmax) ? cmax : static_cast<int>(zc);
    }
    const uint32_t sub2 = (0x4300u | static_cast<uint32_t>(c0 & 0x7F)) * 0x10001u;  // 128 + c0 (c0 < 128)
    const float subf = 8388608.0f + static_cast<float>(c0);
    bool ok = true;
    for (int it = grp; it < n_k; it += 2) {
      const int s = it % kStages;
      // this row's Extra Precision steps in the warp's 32 codes of the stage
      // (the bit plane is ready before the launch, so it loads ahead of the wait)
      uint32_t epw = 0;
      if constexpr (EP) {
        const int kw = (it * kBK + 32 * h) >> 5;
        if (n0 + row < p.N && kw < p.ep_words)
          epw = spread_even_odd(__ldg(p.ep_bits + static_cast<int64_t>(n0 + row) * p.ep_words + kw));
      }
      // Every lane waits (each needs the barrier's ordering for the staged
      // bytes); the warp then decides together, since the tensor-memory
      // store below must be executed by all of its lanes.
      bool mine = *s_abort == 0 && mbar_wait_bounded(&full[s], (it / kStages) & 1, p.wait_ns) &&
                  (it < kStages || mbar_wait_bounded(&empty[s], ((it / kStages) - 1) & 1, p.wait_ns));
      if (!__all_sync(0xffffffffu, mine)) {
        if (lane == 0) { atomicOr(p.err, kErrWaitFull); *s_abort = 1; }
        ok = false;
        break;
      }
      const uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
      // plane 0 rows hold 64 codes (8*b0 bytes); this warp's 32 codes are half
      // of them. Plane 1 rows hold a 16-byte chunk: 64 codes at b1 = 2, 128 at
      // b1 = 1 (of which this stage uses the half it % 2).
      // plane-0 rows of 32 bytes (b0 = 4) and 64 bytes (b0 = 8) are stored in
      // 32- and 64-byte swizzled atoms: 16-byte chunk c of row `row` sits at
      // chunk c ^ ((row / 4) % 2), resp. c ^ ((row / 2) % 4)
      const uint8_t* p0row = st + p.off_p0 + row * (8 * b0);
      const uint8_t* r0;
      const uint8_t* r0b;
      if constexpr (b0 == 8) {
        const int x = (row >> 1) & 3;
        r0 = p0row + 16 * ((2 * h) ^ x);
        r0b = p0row + 16 * ((2 * h + 1) ^ x);
      } else if constexpr (b0 == 4) {
        r0 = p0row + 16 * (h ^ ((row >> 2) & 1));
        r0b = r0;
      } else {
        r0 = p0row + h * (4 * b0);
        r0b = r0;
      }
      const uint8_t* r1 = st + p.off_p1 + row * 16 +
                          (b1 == 1 ? (it % 2) * 8 + h * 4 : h * 8);
      uint32_t v[16] = {};
      const uint8_t* st_end = st + p.stage_bytes;
      (void)st_end;  // read only by the debug build's checks
      // (r1 is read only by widths with a second plane)
      if (MQ_IN_BOUNDS(r0 + 16 <= st_end && r0b + 16 <= st_end && (b1 == 0 || r1 + 8 <= st_end), p.err))
        decode32<R>(r0, r0b, r1, v, sub2, subf, ch2, ckm, cs, epw);
      tc05::st_32x32b_x16(tmem + lane_addr + kASlotCol + s * 32 + h * 16, v);
      tc05::wait_st();
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&decoded[s]);
    }
    // ---------------------------------------------------------- epilogue
    // Warp (q, h, grp) writes batch columns [128 h + 64 grp, +64) of its 32
    // weight rows.
    const bool acc_ready = ok && __all_sync(0xffffffffu, mbar_wait_bounded(acc_full, 0, p.wait_ns));
    if (acc_ready) {
      tc05::fence_after_sync();
      const int n = n0 + row;
      const bool row_ok = n < p.N;
      float A = 0.f, B = 0.f;
      if (row_ok) {
        // y = A sum x (c - c0) - alpha (z - c0 2^s) Sx
        const float a = __ldg(p.alpha + n);
        const float sc = static_cast<float>(1 << (8 - rw));
        A = a * sc;
        B = a * (__ldg(p.zero + n) - static_cast<float>(c0) * sc);
      }
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int col = 128 * h + 64 * grp + 32 * c;
        uint32_t d[32];
        tc05::ld_32x32b_x32(tmem + lane_addr + kAccCol + col, d);
        tc05::wait_ld();
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + col + j;
            if (m < p.M) {
              const float sx = __ldg(p.sx + m);
              p.y[static_cast<int64_t>(m) * p.N + n] = A * __uint_as_float(d[j]) - B * sx;
            }
          }
        }
      }
    } else if (ok) {
      if (lane == 0) { atomicOr(p.err, kErrMma); *s_abort = 1; }
    }
    tc05::fence_before_sync();
  }
  if (warp == 1) tc05::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc05::fence_after_sync();
    tc05::dealloc(tmem, kTmemCols);
  }
}


template <int R, bool EP = false>
cudaError_t launch_gemm_r(const GemmParams& gp, dim3 grid, size_t smem, cudaStream_t stream) {
  auto kern = gemm_tc05_kernel<R, EP>;
  static std::mutex mu;
  static std::map<int, bool> attr_set;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  kern<<<grid, kGemmThreads, smem, stream>>>(gp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t run_gemm(const LinearJob& job, int M, cudaStream_t stream) {
  if (M < 1 || job.K < 32 || job.K % 32 != 0 || job.N < 1) return cudaErrorNotSupported;
  if ((job.N + kBN - 1) / kBN > 0x7FFFFFFF || (M + kBM - 1) / kBM > 65535) return cudaErrorNotSupported;
  int b0, b1;
  job_planes(job, b0, b1);
  if (b0 == 0) return cudaErrorInvalidValue;
  const bool ep = job.ep_rows != nullptr;
  if (ep && (job.r == 8 || job.src != kPlanes)) return cudaErrorNotSupported;  // Eq. 8 lists: planes of width <= 6

  static thread_local GemmParams gp;
  cudaError_t e = encode_map_2d(&gp.map_x, job.x, uint64_t(M), uint64_t(job.K), 64, kBM, 2, 128);
  if (e != cudaSuccess) return e;
  // plane-0 rows of 32 or 64 bytes arrive swizzled, so that the decode
  // threads (one weight row each) read them without bank conflicts
  e = encode_map_2d(&gp.map_p0, job.packed, uint64_t(job.N), uint64_t(job.K) * b0 / 8,
                    8u * b0, kBN, 1, b0 == 8 ? 64 : b0 == 4 ? 32 : 0);
  if (e != cudaSuccess) return e;
  if (b1) {
    e = encode_map_2d(&gp.map_p1, job.packed + job.N * job.K * b0 / 8, uint64_t(job.N),
                      uint64_t(job.K) * b1 / 8, 16u, kBN, 1);
    if (e != cudaSuccess) return e;
  } else {
    gp.map_p1 = gp.map_p0;
  }

  void* ws = nullptr;
  // Sx, then (Extra Precision) the list's bit plane: N rows of K / 32 words
  const size_t sx_bytes = (size_t(M) * sizeof(float) + 255) & ~size_t(255);
  const size_t ep_bytes = ep ? size_t(job.N) * size_t(job.K / 32) * sizeof(uint32_t) : 0;
  e = get_workspace(stream, sx_bytes + ep_bytes + 256, &ws);
  if (e != cudaSuccess) return e;
  float* sx = static_cast<float*>(ws);
  uint32_t* err = nullptr;
  e = get_error_word(&err);
  if (e != cudaSuccess) return e;

  gp.alpha = job.alpha;
  gp.zero = job.zero;
  gp.sx = sx;
  gp.ep_bits = nullptr;
  gp.ep_words = static_cast<int>(job.K / 32);
  if (ep) {
    uint32_t* bits = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + sx_bytes);
    e = launch_ep_bits(job.ep_rows, job.ep_cols, job.N, job.K, bits, stream, sm_count());
    if (e != cudaSuccess) return e;
    gp.ep_bits = bits;
  }
  gp.y = job.y;
  gp.err = err;
  gp.wait_ns = wait_limit_ns();
  gp.M = M;
  gp.N = static_cast<int>(job.N);
  gp.K = static_cast<int>(job.K);
  gp.r = job.r;
  gp.off_p0 = kXStageBytes;
  const uint32_t p0_bytes = 128u * 8u * b0;
  gp.off_p1 = gp.off_p0 + p0_bytes;
  const uint32_t p1_bytes = b1 ? 128u * 16u : 0u;
  gp.stage_bytes = (gp.off_p1 + p1_bytes + 1023u) & ~1023u;
  const size_t smem = 1024 /* alignment slack */ + kHeaderBytes + size_t(kStages) * gp.stage_bytes;

  rowsum_kernel<<<M, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(job.x),
                                        static_cast<int>(job.K), sx);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const dim3 grid(static_cast<unsigned>((job.N + kBN - 1) / kBN), static_cast<unsigned>((M + kBM - 1) / kBM));
  if (ep) {
    switch (decode_kind(job)) {
      case 6: return launch_gemm_r<6, true>(gp, grid, smem, stream);
      case 4: return launch_gemm_r<4, true>(gp, grid, smem, stream);
      case 3: return launch_gemm_r<3, true>(gp, grid, smem, stream);
      case 2: return launch_gemm_r<2, true>(gp, grid, smem, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (decode_kind(job)) {
    case 10: return launch_gemm_r<10>(gp, grid, smem, stream);
    case 11: return launch_gemm_r<11>(gp, grid, smem, stream);
    case 8: return launch_gemm_r<8>(gp, grid, smem, stream);
    case 6: return launch_gemm_r<6>(gp, grid, smem, stream);
    case 4: return launch_gemm_r<4>(gp, grid, smem, stream);
    case 3: return launch_gemm_r<3>(gp, grid, smem, stream);
    case 2: return launch_gemm_r<2>(gp, grid, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mq
