// Decode path (M <= 32): y = x . W_r^T with W_r[n,k] = alpha_n (S(q[n,k], r) - z_n),
// streaming dense r-bit planes ("Matryoshka Quantization" explainer page:
// Eq. 1 dequantization alpha*(q - z), Eq. 6 slicing, and the statement that
// decode latency is set by how fast the weights move out of HBM).
//
// Work decomposition. A "unit" is 128 weight rows x KC codes of one linear.
// All units of all linears of a launch form one list; CTA c of a persistent
// grid of G CTAs takes the contiguous range [c*U/G, (c+1)*U/G) ("stream-K"),
// so every CTA streams the same number of units whatever the shapes. Partial
// row sums are added into y with fp32 atomics; the prep kernel zeroes y.
//
// CTA = 4 consumer warps + 1 producer warp. The producer stages each unit in
// shared memory with 1-D bulk copies (cp.async.bulk, one per row and plane)
// plus one copy of the activation block, signalling an mbarrier. Each
// consumer warp owns 2 tiles of 16 rows and runs mma.sync m16n8k16 (bf16 in,
// fp32 accumulate) with the weights as the A operand and the batch (M <= 32,
// n8 tiles) as B.
//
// Exactness of the operands. A code c (0 <= c < 2^b, b <= 4) is OR-ed into
// the mantissa of a bf16 power of two 2^e at a bit position p, which yields
// exactly 2^e + c * 2^(e-7+p); choosing p and e so that the code weight is 1
// (or 4, 16 for the high plane of r = 3, 6; 16 for the high nibble of r = 8)
// gives the integer value off + weight*c, exact in bf16. The offsets "off"
// sum to O_m = sum_k x[m,k] off(k), which depends only on k mod 8 and is
// removed in the epilogue from per-class activation sums computed once:
//   y = A_n (acc - O_m) - B_n Sx_m,  A_n = alpha_n 2^(8-r),  B_n = alpha_n z_n.
// Offsets stay <= 384, so fp32 partial sums stay small (accuracy), and
// two codes are decoded per shift+LOP3 pair (issue budget at r = 2).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <map>
#include <utility>
#include <vector>

#include "mq_device.cuh"
#include "mq_internal.h"

namespace mq {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kTilesPerWarp = 2;
constexpr int kRowsPerUnit = kConsumerWarps * kTilesPerWarp * 16;  // 128
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxStages = 8;
constexpr int kBarrierBytes = 256;

// Per-linear descriptor, passed by value in the kernel parameters.
struct LinDesc {
  const uint8_t* plane0;
  const uint8_t* plane1;
  const float* alpha;
  const float* zero;
  float* y;
  const uint8_t* xf;   // activations in fragment order, n_kc blocks of M*KC bf16
  const float* psum;   // [M][4] activation sums per class (k >> 1) & 3
  int N, K, r, kc, n_kc, unit_begin;
};

template <int CAP>
struct GemvParams {
  int n_lin, M, total_units, stages;
  uint32_t stage_bytes, off_plane1, off_x;
  int pitch0, pitch1;
  uint32_t* err;
  unsigned long long wait_ns;
  LinDesc lin[CAP];
};

// Geometry of one width: the high-plane width b1 (0 if one plane), the
// 8-code activation groups per 16-byte low-plane chunk (W8) and the MMAs fed
// by one group (MPG: 2 when each code fills one k-slot, 4 when it fills two).
template <int R> struct Geo;
template <> struct Geo<2> { static constexpr int b1 = 0, W8 = 8, MPG = 2; };
template <> struct Geo<4> { static constexpr int b1 = 0, W8 = 4, MPG = 2; };
template <> struct Geo<8> { static constexpr int b1 = 0, W8 = 2, MPG = 4; };
template <> struct Geo<3> { static constexpr int b1 = 1, W8 = 8, MPG = 4; };
template <> struct Geo<6> { static constexpr int b1 = 2, W8 = 4, MPG = 4; };

__device__ __forceinline__ void plane_widths_dev(int r, int& b0, int& b1) {
  b0 = (r == 8) ? 8 : (r == 4 || r == 6) ? 4 : 2;
  b1 = (r == 3) ? 1 : (r == 6) ? 2 : 0;
}

template <int SIG>
__device__ __forceinline__ uint32_t shift_to(uint32_t w) {
  if constexpr (SIG < 0) return w << (-SIG);
  else return w >> SIG;
}

// bf16x2 magic constants 2^e in both halves.
constexpr uint32_t kMag4 = 0x40804080u, kMag8 = 0x41004100u, kMag16 = 0x41804180u,
                   kMag32 = 0x42004200u, kMag64 = 0x42804280u, kMag128 = 0x43004300u,
                   kMag256 = 0x43804380u;

// Decodes the two A registers (x0: slots {2t, 2t+1}; x1: slots {2t+8, 2t+9})
// of MMA J for one weight row from its low-plane words lo[4] and high-plane
// words hi[2]. Each register holds the bf16 values of two neighbouring codes.
template <int R, int J>
__device__ __forceinline__ void decode_pair(const uint32_t (&lo)[4], const uint32_t (&hi)[2],
                                            uint32_t& x0, uint32_t& x1) {
  if constexpr (R == 2) {
    // codes 4J..4J+3: pair 2jj at half-bit 4jj -> bits 3-4 (16+c), pair 2jj+1 -> bits 5-6 (4+c)
    constexpr int jj = J % 4;
    const uint32_t sh = shift_to<4 * jj - 3>(lo[J / 4]);
    x0 = (sh & 0x00180018u) | kMag16;
    x1 = (sh & 0x00600060u) | kMag4;
  } else if constexpr (R == 4) {
    // codes 4J..4J+3: pairs pa, pa+1 at half-bits 4pa, 4pa+4 -> bits 3-6 (16+c)
    constexpr int pa = 2 * (J % 2);
    const uint32_t w = lo[J / 2];
    x0 = (shift_to<4 * pa - 3>(w) & 0x00780078u) | kMag16;
    x1 = (shift_to<4 * (pa + 1) - 3>(w) & 0x00780078u) | kMag16;
  } else if constexpr (R == 8) {
    // codes 2J, 2J+1 (bytes): low nibble -> 128+l, high nibble -> 256+16h
    const uint32_t d = __byte_perm(lo[J / 2], 0u, (J % 2) ? 0x4342u : 0x4140u);
    x0 = (d & 0x000F000Fu) | kMag128;
    x1 = ((d >> 1) & 0x00780078u) | kMag256;
  } else if constexpr (R == 3) {
    // codes 2J, 2J+1: low 2-bit plane -> 16+c or 4+c; high 1-bit plane (weight 4)
    constexpr int pl = J % 8;
    const uint32_t sl = shift_to<4 * (pl / 2) - 3>(lo[J / 8]);
    if constexpr (pl % 2 == 0) x0 = (sl & 0x00180018u) | kMag16;
    else x0 = (sl & 0x00600060u) | kMag4;
    constexpr int ph = J % 16;
    constexpr int p = 3 + ph % 4;
    constexpr uint32_t mask = (1u << p) | (1u << (16 + p));
    constexpr uint32_t mag = (ph % 4 == 0) ? kMag64 : (ph % 4 == 1) ? kMag32 : (ph % 4 == 2) ? kMag16 : kMag8;
    x1 = (shift_to<4 * (ph / 4) - 3>(hi[J / 16]) & mask) | mag;
  } else {  // R == 6
    // codes 2J, 2J+1: low 4-bit plane -> 16+c; high 2-bit plane (weight 16) -> 256+16h or 64+16h
    constexpr int pl = J % 4;
    x0 = (shift_to<4 * pl - 3>(lo[J / 4]) & 0x00780078u) | kMag16;
    constexpr int ph = J % 8;
    const uint32_t sh = shift_to<4 * (ph / 2) - 3>(hi[J / 8]);
    if constexpr (ph % 2 == 0) x1 = (sh & 0x00180018u) | kMag256;
    else x1 = (sh & 0x00600060u) | kMag64;
  }
}

// Offset coefficients per activation class (k >> 1) & 3 for each width.
__device__ __forceinline__ void offset_coeffs(int r, float (&c)[4]) {
  switch (r) {
    case 8: c[0] = c[1] = c[2] = c[3] = 384.f; break;
    case 4: c[0] = c[1] = c[2] = c[3] = 16.f; break;
    case 2: c[0] = 16.f; c[1] = 4.f; c[2] = 16.f; c[3] = 4.f; break;
    case 3: c[0] = 80.f; c[1] = 36.f; c[2] = 32.f; c[3] = 12.f; break;
    default: c[0] = 272.f; c[1] = 80.f; c[2] = 272.f; c[3] = 80.f; break;  // 6
  }
}

template <int R, int MMA_J, int NT>
__device__ __forceinline__ void mma_step(const uint32_t (&lo)[kTilesPerWarp][2][4],
                                         const uint32_t (&hi)[kTilesPerWarp][2][2],
                                         const uint4 (&xb)[NT],
                                         float (&ch)[kTilesPerWarp][NT][2][4]) {
  using G = Geo<R>;
  uint32_t b0[NT], b1[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint32_t comp[4] = {xb[nt].x, xb[nt].y, xb[nt].z, xb[nt].w};
    if constexpr (G::MPG == 2) {
      b0[nt] = comp[2 * (MMA_J % 2)];
      b1[nt] = comp[2 * (MMA_J % 2) + 1];
    } else {
      b0[nt] = comp[MMA_J % 4];
      b1[nt] = b0[nt];
    }
  }
#pragma unroll
  for (int tau = 0; tau < kTilesPerWarp; ++tau) {
    uint32_t a0, a1, a2, a3;
    decode_pair<R, MMA_J>(lo[tau][0], hi[tau][0], a0, a2);
    decode_pair<R, MMA_J>(lo[tau][1], hi[tau][1], a1, a3);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(ch[tau][nt][MMA_J & 1], a0, a1, a2, a3, b0[nt], b1[nt]);
  }
}

template <int R, int NT, int Q>
__device__ __forceinline__ void group_steps(const uint32_t (&lo)[kTilesPerWarp][2][4],
                                            const uint32_t (&hi)[kTilesPerWarp][2][2],
                                            const uint8_t* xq, uint32_t xstride, bool (&mval)[NT],
                                            float (&ch)[kTilesPerWarp][NT][2][4]) {
  using G = Geo<R>;
  uint4 xb[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    xb[nt] = mval[nt] ? *reinterpret_cast<const uint4*>(xq + nt * xstride) : make_uint4(0, 0, 0, 0);
  if constexpr (G::MPG >= 1) mma_step<R, Q * G::MPG + 0, NT>(lo, hi, xb, ch);
  if constexpr (G::MPG >= 2) mma_step<R, Q * G::MPG + 1, NT>(lo, hi, xb, ch);
  if constexpr (G::MPG >= 3) mma_step<R, Q * G::MPG + 2, NT>(lo, hi, xb, ch);
  if constexpr (G::MPG >= 4) mma_step<R, Q * G::MPG + 3, NT>(lo, hi, xb, ch);
}

template <int R, int NT, int... Qs>
__device__ __forceinline__ void all_groups(const uint32_t (&lo)[kTilesPerWarp][2][4],
                                           const uint32_t (&hi)[kTilesPerWarp][2][2],
                                           const uint8_t* xs, int M, uint32_t xstride_q,
                                           uint32_t xstride_nt, bool (&mval)[NT],
                                           float (&ch)[kTilesPerWarp][NT][2][4],
                                           std::integer_sequence<int, Qs...>) {
  (group_steps<R, NT, Qs>(lo, hi, xs + Qs * xstride_q, xstride_nt, mval, ch), ...);
}

// Processes one staged unit for this warp's two 16-row tiles.
template <int R, int NT>
__device__ __forceinline__ void process_unit(const uint8_t* st0, const uint8_t* st1,
                                             const uint8_t* stx, int pitch0, int pitch1,
                                             int nsub, int M, int warp, int lane,
                                             float (&ch)[kTilesPerWarp][NT][2][4]) {
  using G = Geo<R>;
  const int g = lane >> 2, t = lane & 3;
  bool mval[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) mval[nt] = (nt * 8 + g) < M;
  for (int s = 0; s < nsub; ++s) {
    const int ci = 4 * s + t;  // this thread's 16-byte chunk of the low plane
    uint32_t lo[kTilesPerWarp][2][4];
    uint32_t hi[kTilesPerWarp][2][2];
#pragma unroll
    for (int tau = 0; tau < kTilesPerWarp; ++tau) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = warp * 32 + tau * 16 + g + 8 * h;
        const uint4 v = *reinterpret_cast<const uint4*>(st0 + row * pitch0 + ci * 16);
        lo[tau][h][0] = v.x; lo[tau][h][1] = v.y; lo[tau][h][2] = v.z; lo[tau][h][3] = v.w;
        if constexpr (G::b1 != 0) {
          const uint2 u = *reinterpret_cast<const uint2*>(st1 + row * pitch1 + ci * 8);
          hi[tau][h][0] = u.x; hi[tau][h][1] = u.y;
        } else {
          hi[tau][h][0] = 0; hi[tau][h][1] = 0;
        }
      }
    }
    // Activation group q of chunk ci for batch row m sits at
    // ((((s*W8 + q)*M + m)*4 + t) * 16) bytes of the staged block.
    const uint8_t* xs = stx + ((static_cast<uint32_t>(s * G::W8) * M + g) * 4 + t) * 16;
    all_groups<R, NT>(lo, hi, xs, M, static_cast<uint32_t>(M) * 64u, 8u * 64u, mval, ch,
                      std::make_integer_sequence<int, G::W8>{});
  }
}

template <int NT, int CAP>
__device__ void flush_rows(const GemvParams<CAP>& p, int l, int rb, int kc0, int warp, int lane,
                           float (&tot)[kTilesPerWarp][NT][4]) {
  const LinDesc& L = p.lin[l];
  const int g = lane >> 2, t = lane & 3;
  const float scale = static_cast<float>(1 << (8 - L.r));
  float c[4];
  offset_coeffs(L.r, c);
#pragma unroll
  for (int tau = 0; tau < kTilesPerWarp; ++tau) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = rb * kRowsPerUnit + warp * 32 + tau * 16 + g + 8 * h;
      if (n >= L.N) continue;
      const float a = L.alpha[n], z = L.zero[n];
      const float A = a * scale, B = a * z;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int m = nt * 8 + 2 * t + e;
          if (m >= p.M) continue;
          float v = tot[tau][nt][2 * h + e];
          if (kc0 == 0) {
            const float* P = L.psum + m * 4;
            const float O = c[0] * P[0] + c[1] * P[1] + c[2] * P[2] + c[3] * P[3];
            const float Sx = (P[0] + P[1]) + (P[2] + P[3]);
            v = A * (v - O) - B * Sx;
          } else {
            v = A * v;
          }
          atomicAdd(L.y + static_cast<int64_t>(m) * L.N + n, v);
        }
      }
    }
  }
}

template <int NT, int CAP>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv_streamk_kernel(const __grid_constant__ GemvParams<CAP> p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kMaxStages);
  uint8_t* stages = smem + kBarrierBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t G = gridDim.x, c = blockIdx.x;
  const int u0 = static_cast<int>(int64_t(p.total_units) * c / G);
  const int u1 = static_cast<int>(int64_t(p.total_units) * (c + 1) / G);

  // Activations, class sums and the zeroed outputs come from the prep kernel.
  pdl_wait_primary();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    int l = 0, issued = 0;
    bool aborted = false;
    for (int u = u0; u < u1; ++u, ++issued) {
      const int s = issued % S;
      if (issued >= S) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&empty[s], ((issued / S) - 1) & 1, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) {
          if (lane == 0) { atomicOr(p.err, kErrWaitEmpty); *s_abort = 1; }
          aborted = true;
          break;
        }
      }
      if (*s_abort) { aborted = true; break; }
      while (l + 1 < p.n_lin && u >= p.lin[l + 1].unit_begin) ++l;
      const LinDesc& L = p.lin[l];
      const int local = u - L.unit_begin;
      const int rb = local / L.n_kc, kc = local - rb * L.n_kc;
      const int ncodes = min(L.kc, L.K - kc * L.kc);
      const int rows = min(kRowsPerUnit, L.N - rb * kRowsPerUnit);
      int b0, b1;
      plane_widths_dev(L.r, b0, b1);
      const uint32_t bytes0 = static_cast<uint32_t>(ncodes * b0 / 8);
      const uint32_t bytes1 = static_cast<uint32_t>(ncodes * b1 / 8);
      const uint32_t bytesx = static_cast<uint32_t>(p.M * L.kc * 2);
      uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
      if (lane == 0)
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(rows) * (bytes0 + bytes1) + bytesx);
      __syncwarp();
      const int64_t row0 = int64_t(rb) * kRowsPerUnit;
      const int64_t gp0 = int64_t(L.K) * b0 / 8, gp1 = int64_t(L.K) * b1 / 8;
      const int ncopies = rows * (b1 ? 2 : 1) + 1;
      for (int cidx = lane; cidx < ncopies; cidx += 32) {
        if (cidx == ncopies - 1) {
          bulk_g2s(st + p.off_x, L.xf + int64_t(kc) * bytesx, bytesx, &full[s]);
        } else if (cidx < rows) {
          bulk_g2s(st + cidx * p.pitch0,
                   L.plane0 + (row0 + cidx) * gp0 + int64_t(kc) * (L.kc * b0 / 8), bytes0, &full[s]);
        } else {
          const int i = cidx - rows;
          bulk_g2s(st + p.off_plane1 + i * p.pitch1,
                   L.plane1 + (row0 + i) * gp1 + int64_t(kc) * (L.kc * b1 / 8), bytes1, &full[s]);
        }
      }
    }
    if (aborted && lane == 0) {
      // Leave no bulk copy in flight: wait for the last issue of every stage.
      const int first = issued > S ? issued - S : 0;
      for (int j = first; j < issued; ++j) {
        if (!mbar_wait_bounded(&full[j % S], (j / S) & 1, 1000000000ull)) atomicOr(p.err, kErrDrain);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  float ch[kTilesPerWarp][NT][2][4];
  float tot[kTilesPerWarp][NT][4];
#pragma unroll
  for (int a = 0; a < kTilesPerWarp; ++a)
#pragma unroll
    for (int b = 0; b < NT; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) { ch[a][b][0][i] = 0.f; ch[a][b][1][i] = 0.f; tot[a][b][i] = 0.f; }

  int l = 0, cur_l = -1, cur_rb = -1, cur_kc0 = 0;
  bool aborted = false;
  int it = 0;
  for (int u = u0; u < u1; ++u, ++it) {
    const int s = it % S;
    if (*s_abort || !mbar_wait_bounded(&full[s], (it / S) & 1, p.wait_ns)) {
      if (lane == 0) { atomicOr(p.err, kErrWaitFull); *s_abort = 1; }
      aborted = true;
      break;
    }
    while (l + 1 < p.n_lin && u >= p.lin[l + 1].unit_begin) ++l;
    const LinDesc& L = p.lin[l];
    const int local = u - L.unit_begin;
    const int rb = local / L.n_kc, kc = local - rb * L.n_kc;
    if (l != cur_l || rb != cur_rb) {
      if (cur_l >= 0) flush_rows<NT>(p, cur_l, cur_rb, cur_kc0, warp, lane, tot);
#pragma unroll
      for (int a = 0; a < kTilesPerWarp; ++a)
#pragma unroll
        for (int b = 0; b < NT; ++b)
#pragma unroll
          for (int i = 0; i < 4; ++i) tot[a][b][i] = 0.f;
      cur_l = l; cur_rb = rb; cur_kc0 = kc;
    }
    const int rows = min(kRowsPerUnit, L.N - rb * kRowsPerUnit);
    if (warp * 32 < rows) {
      const int ncodes = min(L.kc, L.K - kc * L.kc);
      const uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
      int b0, b1;
      plane_widths_dev(L.r, b0, b1);
      const int per_sub = 512 / b0;  // codes covered by one sub-step (4 chunks of 16 bytes)
      const int nsub = (ncodes + per_sub - 1) / per_sub;
      switch (L.r) {
        case 2: process_unit<2, NT>(st, st + p.off_plane1, st + p.off_x, p.pitch0, p.pitch1, nsub, p.M, warp, lane, ch); break;
        case 4: process_unit<4, NT>(st, st + p.off_plane1, st + p.off_x, p.pitch0, p.pitch1, nsub, p.M, warp, lane, ch); break;
        case 8: process_unit<8, NT>(st, st + p.off_plane1, st + p.off_x, p.pitch0, p.pitch1, nsub, p.M, warp, lane, ch); break;
        case 3: process_unit<3, NT>(st, st + p.off_plane1, st + p.off_x, p.pitch0, p.pitch1, nsub, p.M, warp, lane, ch); break;
        default: process_unit<6, NT>(st, st + p.off_plane1, st + p.off_x, p.pitch0, p.pitch1, nsub, p.M, warp, lane, ch); break;
      }
      // Fold the two MMA chains into the row totals once per unit.
#pragma unroll
      for (int a = 0; a < kTilesPerWarp; ++a)
#pragma unroll
        for (int b = 0; b < NT; ++b)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            tot[a][b][i] += ch[a][b][0][i] + ch[a][b][1][i];
            ch[a][b][0][i] = 0.f;
            ch[a][b][1][i] = 0.f;
          }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (!aborted && cur_l >= 0) flush_rows<NT>(p, cur_l, cur_rb, cur_kc0, warp, lane, tot);
}

// ------------------------------------------------------------------ prep
struct PrepLayout {
  const __nv_bfloat16* x;
  uint8_t* xf;
  int K, kc, w8, n_kc;
};
struct PrepSum {
  const __nv_bfloat16* x;
  float* psum;
  int K;
};
struct PrepZero {
  float* y;
  int64_t count;
};
template <int CAP>
struct PrepParams {
  int M, n_layout, n_sum, n_zero;
  PrepLayout lay[CAP];
  PrepSum sum[CAP];
  PrepZero zero[CAP];
};

// Builds the fragment-ordered activation blocks (zero-padded to whole
// k-chunks), the per-class activation sums and zeroes every output.
template <int CAP>
__global__ void __launch_bounds__(256) gemv_prep_kernel(const __grid_constant__ PrepParams<CAP> p) {
  pdl_launch_dependents();
  const int M = p.M;
  // (1) class sums: one CTA per (sum job, batch row)
  if (blockIdx.x < p.n_sum * M) {
    const PrepSum& J = p.sum[blockIdx.x / M];
    const int m = blockIdx.x % M;
    const __nv_bfloat16* row = J.x + int64_t(m) * J.K;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    // 8 consecutive elements k0..k0+7 (k0 % 8 == 0): classes 0,0,1,1,2,2,3,3
    for (int k0 = threadIdx.x * 8; k0 < J.K; k0 += blockDim.x * 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + k0);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        acc[i] += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xFFFF0000u);
    }
    __shared__ float red[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = acc[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((threadIdx.x & 31) == 0) red[i][threadIdx.x >> 5] = v;
    }
    __syncthreads();
    if (threadIdx.x < 4) {
      float v = 0.f;
      for (int w8 = 0; w8 < (int)(blockDim.x >> 5); ++w8) v += red[threadIdx.x][w8];
      J.psum[m * 4 + threadIdx.x] = v;
    }
  }
  // (2) fragment-ordered activation groups: thread per (layout, m, 8-code group)
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t tid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int li = 0; li < p.n_layout; ++li) {
    const PrepLayout& L = p.lay[li];
    const int groups_per_chunk = L.kc / 8;
    const int64_t total = int64_t(L.n_kc) * groups_per_chunk * M;
    for (int64_t i = tid; i < total; i += stride) {
      const int m = static_cast<int>(i % M);
      const int64_t gg = i / M;                 // global group index
      const int kc = static_cast<int>(gg / groups_per_chunk);
      const int grp = static_cast<int>(gg % groups_per_chunk);
      const int k0 = kc * L.kc + grp * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (k0 < L.K) v = *reinterpret_cast<const uint4*>(L.x + int64_t(m) * L.K + k0);
      const int s = grp / (4 * L.w8);
      const int rem = grp % (4 * L.w8);
      const int t = rem / L.w8, q = rem % L.w8;
      const int64_t off = int64_t(kc) * M * L.kc * 2 +
                          ((int64_t(s * L.w8 + q) * M + m) * 4 + t) * 16;
      *reinterpret_cast<uint4*>(L.xf + off) = v;
    }
  }
  // (3) zero the outputs
  for (int zi = 0; zi < p.n_zero; ++zi) {
    float* y = p.zero[zi].y;
    const int64_t cnt = p.zero[zi].count;
    for (int64_t i = tid; i < cnt; i += stride) y[i] = 0.f;
  }
}

template <int NT>
cudaError_t launch_gemv_nt(const GemvParams<kGemvMaxLinears>& gp, int grid, size_t smem,
                           cudaStream_t stream) {
  auto kern = gemv_streamk_kernel<NT, kGemvMaxLinears>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, gp);
}

template <int NT>
int occupancy_nt(size_t smem) {
  int blocks = 0;
  auto kern = gemv_streamk_kernel<NT, kGemvMaxLinears>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kGemvThreads, smem) != cudaSuccess)
    return 1;
  return blocks < 1 ? 1 : blocks;
}

}  // namespace

cudaError_t run_gemv(const LinearJob* jobs, int n_jobs, int M, cudaStream_t stream) {
  if (n_jobs < 1 || n_jobs > kGemvMaxLinears || M < 1 || M > 32) return cudaErrorInvalidValue;
  // Bytes of low plane per row per unit: 192 keeps consecutive rows 64 bytes
  // apart modulo 128 (conflict-free 16-byte shared loads) with few copies;
  // larger batches use 64 to bound the staged activation block.
  const int P0 = M <= 8 ? 192 : 64;
  const int NT = (M + 7) / 8;

  static thread_local GemvParams<kGemvMaxLinears> gp;
  static thread_local PrepParams<kGemvMaxLinears> pp;
  std::memset(&gp, 0, sizeof(gp));
  std::memset(&pp, 0, sizeof(pp));

  // Distinct inputs (class sums) and distinct (input, layout) pairs.
  std::map<const void*, int> sum_of_x;
  std::map<std::pair<const void*, int>, int> layout_of;
  struct LayoutInfo { const void* x; int K, kc, w8, n_kc; size_t off; };
  std::vector<LayoutInfo> layouts;
  std::vector<std::pair<const void*, int>> sums;
  bool two_planes = false;
  int units = 0;
  size_t xf_bytes = 0;
  for (int i = 0; i < n_jobs; ++i) {
    const LinearJob& j = jobs[i];
    int b0, b1;
    plane_widths(j.r, b0, b1);
    if (b1) two_planes = true;
    const int kc = P0 * 8 / b0;
    const int n_kc = static_cast<int>((j.K + kc - 1) / kc);
    if (!sum_of_x.count(j.x)) {
      sum_of_x[j.x] = static_cast<int>(sums.size());
      sums.push_back({j.x, static_cast<int>(j.K)});
    }
    auto key = std::make_pair(j.x, b0);
    if (!layout_of.count(key)) {
      layout_of[key] = static_cast<int>(layouts.size());
      layouts.push_back({j.x, static_cast<int>(j.K), kc, (128 / b0) / 8, n_kc, xf_bytes});
      xf_bytes += size_t(n_kc) * M * kc * 2;
      xf_bytes = (xf_bytes + 255) & ~size_t(255);
    }
    const int nrb = static_cast<int>((j.N + kRowsPerUnit - 1) / kRowsPerUnit);
    LinDesc& d = gp.lin[i];
    d.plane0 = j.packed;
    d.plane1 = b1 ? j.packed + j.N * j.K * b0 / 8 : nullptr;
    d.alpha = j.alpha;
    d.zero = j.zero;
    d.y = j.y;
    d.N = static_cast<int>(j.N);
    d.K = static_cast<int>(j.K);
    d.r = j.r;
    d.kc = kc;
    d.n_kc = n_kc;
    d.unit_begin = units;
    units += nrb * n_kc;
  }
  const size_t psum_off = xf_bytes;
  const size_t ws_bytes = psum_off + sums.size() * size_t(M) * 4 * sizeof(float) + 256;
  void* ws = nullptr;
  cudaError_t e = get_workspace(stream, ws_bytes, &ws);
  if (e != cudaSuccess) return e;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* psum_base = reinterpret_cast<float*>(wsb + psum_off);
  for (int i = 0; i < n_jobs; ++i) {
    int b0, b1;
    plane_widths(jobs[i].r, b0, b1);
    gp.lin[i].xf = wsb + layouts[layout_of[std::make_pair(jobs[i].x, b0)]].off;
    gp.lin[i].psum = psum_base + size_t(sum_of_x[jobs[i].x]) * M * 4;
  }

  // Prep launch.
  pp.M = M;
  pp.n_layout = static_cast<int>(layouts.size());
  pp.n_sum = static_cast<int>(sums.size());
  pp.n_zero = n_jobs;
  for (size_t i = 0; i < layouts.size(); ++i) {
    pp.lay[i] = {static_cast<const __nv_bfloat16*>(layouts[i].x), wsb + layouts[i].off,
                 layouts[i].K, layouts[i].kc, layouts[i].w8, layouts[i].n_kc};
  }
  for (size_t i = 0; i < sums.size(); ++i) {
    pp.sum[i] = {static_cast<const __nv_bfloat16*>(sums[i].first), psum_base + i * M * 4,
                 sums[i].second};
  }
  for (int i = 0; i < n_jobs; ++i) pp.zero[i] = {jobs[i].y, int64_t(M) * jobs[i].N};
  const int sms = sm_count();
  int prep_grid = std::max(pp.n_sum * M, sms);
  prep_grid = std::min(prep_grid, 4 * sms);
  gemv_prep_kernel<kGemvMaxLinears><<<prep_grid, 256, 0, stream>>>(pp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // Stage layout: [128 rows x P0][128 rows x P1][M x KC bf16 activations].
  const int P1 = two_planes ? P0 / 2 : 0;
  const uint32_t off_plane1 = static_cast<uint32_t>(kRowsPerUnit * P0);
  const uint32_t off_x = off_plane1 + static_cast<uint32_t>(kRowsPerUnit * P1);
  const uint32_t x_bytes = static_cast<uint32_t>(M * (P0 * 8 / 2) * 2);  // largest KC (b0 = 2)
  uint32_t stage_bytes = off_x + x_bytes;
  stage_bytes = (stage_bytes + 127) & ~127u;
  const size_t budget = 110 * 1024;
  int stages = static_cast<int>(budget / stage_bytes);
  stages = std::max(2, std::min(stages, kMaxStages));
  const size_t smem = kBarrierBytes + size_t(stages) * stage_bytes;

  gp.n_lin = n_jobs;
  gp.M = M;
  gp.total_units = units;
  gp.stages = stages;
  gp.stage_bytes = stage_bytes;
  gp.off_plane1 = off_plane1;
  gp.off_x = off_x;
  gp.pitch0 = P0;
  gp.pitch1 = P1;
  uint32_t* err = nullptr;
  e = get_error_word(&err);
  if (e != cudaSuccess) return e;
  gp.err = err;
  gp.wait_ns = wait_limit_ns();

  int occ = 1;
  switch (NT) {
    case 1: occ = occupancy_nt<1>(smem); break;
    case 2: occ = occupancy_nt<2>(smem); break;
    case 3: occ = occupancy_nt<3>(smem); break;
    default: occ = occupancy_nt<4>(smem); break;
  }
  const int grid = std::max(1, std::min(units, sms * occ));
  switch (NT) {
    case 1: return launch_gemv_nt<1>(gp, grid, smem, stream);
    case 2: return launch_gemv_nt<2>(gp, grid, smem, stream);
    case 3: return launch_gemv_nt<3>(gp, grid, smem, stream);
    default: return launch_gemv_nt<4>(gp, grid, smem, stream);
  }
}

}  // namespace mq
