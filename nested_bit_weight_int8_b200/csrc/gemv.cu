// Decode path (M <= 32): y = x . W_r^T with W_r[n,k] = alpha_n (S(q[n,k], r) - z_n),
// streaming dense r-bit planes ("Matryoshka Quantization" explainer page:
// Eq. 1 dequantization alpha*(q - z), Eq. 6 slicing, and the statement that
// decode latency is set by how fast the weights move out of HBM).
//
// Work decomposition. A "unit" is 128 weight rows x KC codes of one linear.
// All units of all linears of a launch form one list; CTA c of a persistent
// grid of G CTAs takes a contiguous range of it ("stream-K"). The ranges are
// cut on the host so that every CTA gets the same estimated cost: a unit's
// cost depends on its width (at r = 2 a unit holds four times the codes of
// an r = 8 unit in the same bytes). A CTA walks its range one row block at a
// time; a row block it owns whole is stored into y directly, a row block
// shared with a neighbour is added into y with fp32 atomics, and the prep
// kernel zeroes exactly those shared row blocks first.
//
// CTA = 8 consumer warps + 1 producer warp. The producer stages each unit in
// shared memory with 1-D bulk copies (cp.async.bulk, one per row and plane)
// plus one copy of the activation block, signalling an mbarrier. Each
// consumer warp owns one tile of 16 rows and runs mma.sync m16n8k16 (bf16 in,
// fp32 accumulate) with the weights as the A operand and the batch (M <= 32,
// n8 tiles) as B.
//
// Exactness of the operands. A code c (0 <= c < 2^b, b <= 4) is OR-ed into
// the mantissa of a bf16 power of two 2^e at a bit position p, which yields
// exactly 2^e + c * 2^(e-7+p); choosing p and e so that the code weight is 1
// (or 4, 16 for the high plane of r = 3, 6) gives the integer value
// off + weight*c, exact in bf16. A byte (r = 8) has one significant bit too
// many for this; it goes through fp32 instead (below). The offsets "off"
// sum to O_m = sum_k x[m,k] off(k), which depends only on k mod 16 and is
// removed in the epilogue from per-class activation sums computed once:
//   y = A_n (acc - O_m) - B_n Sx_m,  A_n = alpha_n 2^(8-r),  B_n = alpha_n z_n.
// Offsets stay <= 272 (none at r = 8), so fp32 partial sums stay small
// (accuracy), and two codes are decoded per LOP3 (issue budget at r = 2).
//
// Slicing on load. A linear may also stream the int8 container itself (the
// r = 8 plane) and slice each byte while decoding, so one stored matrix serves
// every width with no repack ("extracted on the fly by slicing"): the code is
// (q + 2^(s-1)) >> s, s = 8 - r, clamped to 2^r - 1 by Eq. 6 or left at up to
// 2^r by the unclamped Eq. 8 (the Extra Precision variant). Two bytes sit in
// the 16-bit halves of a register; the rounding add (and Eq. 6's clamp) runs
// on both halves at once, and a shift and a LOP3 place the code under a bf16
// power of two, as for the planes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "mq_device.cuh"
#include "mq_internal.h"

namespace mq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxStages = 8;
constexpr int kHeaderBytes = 1024;  // barriers, abort flag; last 64 bytes: zero block
constexpr int kMaxDynSmem = 227 * 1024;
constexpr size_t kStageBudget = 108 * 1024;  // two CTAs per SM with the header and alignment slack
constexpr int kMaxCtas = 320;       // persistent grid cap (2 CTAs on each of 148 SMs fit)
constexpr int kClasses = 8;         // activation classes (k >> 1) & 7

// Geometry of a launch with NT batch tiles of 8. Up to 8 batch rows, each
// consumer warp owns two 16-row tiles (four independent MMA chains; one
// activation fragment load feeds two MMAs) over 128-byte plane rows staged in
// 128-byte swizzled boxes, so a unit is 256 rows. Larger batches keep one
// tile per warp over 64-byte rows (128-row units): their accumulators take
// the registers.
template <int NT>
struct Tiling {
  static constexpr int TW = (NT == 1) ? 2 : 1;       // 16-row tiles per warp
  static constexpr int RPW = 16 * TW;                // weight rows per warp
  static constexpr int RPU = kConsumerWarps * RPW;   // weight rows per unit
  static constexpr int P0 = (NT == 1) ? 128 : 64;    // plane-0 bytes per row per unit
  static constexpr bool SWZ = (NT == 1);             // plane-0 box in 128-byte swizzle
  static constexpr int NSUB = P0 / 64;               // 64-byte sub-steps per unit
};
// The same choice on the host, by batch size.
inline int tiling_p0(int M) { return M <= 8 ? 128 : 64; }
inline int tiling_rows(int M) { return M <= 8 ? 256 : 128; }

// Per-linear descriptor, passed by value in the kernel parameters.
struct LinDesc {
  const uint8_t* plane0;
  const uint8_t* plane1;
  const float* alpha;
  const float* zero;
  float* y;
  const uint8_t* xf;   // activations in fragment order, n_kc blocks of M*KC bf16
  const float* psum;   // [M][8] activation sums per class (k >> 1) & 7
  int N, K, r, kc, n_kc, unit_begin;
  int dk;  // decode kind: r for planes, 10 / 11 for the container sliced by Eq. 6 / Eq. 8
  // Extra Precision on the planes (or null): epc[m * N + n] is the sum of
  // x[m, k] over row n's positions whose Eq. 8 code is one step above the
  // Eq. 6 code, computed by the prep kernel.
  const float* epc;
};

template <int CAP>
struct GemvParams {
  // Tensor maps of the planes (plane 0, plane 1 per linear): inline for small
  // launches, else in a device table built once per distinct stack.
  CUtensorMap maps[CAP <= 8 ? 2 * CAP : 1];
  const CUtensorMap* map_table;
  int n_lin, M, total_units, stages;
  uint32_t stage_bytes, off_plane1, off_x;
  int pitch0, pitch1;
  uint32_t* err;
  unsigned long long wait_ns;
  int cta_begin[kMaxCtas + 1];  // unit range of CTA c: [cta_begin[c], cta_begin[c + 1])
  LinDesc lin[CAP];
};
// kernel parameters are limited to 32764 bytes
static_assert(sizeof(GemvParams<kGemvMaxLinears>) <= 32764, "decode kernel parameters too large");

// Geometry of one width: plane widths, 8-code activation groups per 16-byte
// low-plane chunk (W8).
template <int R> struct Geo;
template <> struct Geo<2> { static constexpr int b0 = 2, b1 = 0, W8 = 8; };
template <> struct Geo<4> { static constexpr int b0 = 4, b1 = 0, W8 = 4; };
template <> struct Geo<8> { static constexpr int b0 = 8, b1 = 0, W8 = 2; };
template <> struct Geo<3> { static constexpr int b0 = 2, b1 = 1, W8 = 8; };
template <> struct Geo<6> { static constexpr int b0 = 4, b1 = 2, W8 = 4; };
// The container sliced on load (Eq. 6: kind 10, Eq. 8: kind 11) streams the
// 8-bit plane.
template <> struct Geo<10> { static constexpr int b0 = 8, b1 = 0, W8 = 2; };
template <> struct Geo<11> { static constexpr int b0 = 8, b1 = 0, W8 = 2; };

// Per-linear constants of the slice-on-load decode (both 16-bit halves):
// h2 the rounding addend 2^(s-1), kmask the code's bits after the shift, mag
// the bf16 power of two the code is OR-ed under (code weight 1).
struct Cdec {
  uint32_t h2, kmask, mag;
};
__device__ __forceinline__ Cdec make_cdec(int dk, int r) {
  Cdec c{0u, 0u, 0u};
  if (dk == 10 || dk == 11) {
    const int s = 8 - r;
    c.h2 = (1u << (s - 1)) * 0x10001u;
    // Eq. 6: min(q + h, 255) >> 1 holds the r-bit code at bits 7-r .. 6, under
    // 2^r. Eq. 8: (q + h) >> 2 holds the (r+1)-bit code at bits 6-r .. 6,
    // under 2^(r+1).
    const int e = dk == 10 ? r : r + 1;
    const uint32_t bits = dk == 10 ? ((1u << r) - 1u) << (7 - r) : ((1u << (r + 1)) - 1u) << (6 - r);
    c.kmask = bits * 0x10001u;
    c.mag = (static_cast<uint32_t>(127 + e) << 7) * 0x10001u;
  }
  return c;
}

__device__ __forceinline__ void plane_widths_dev(int r, int& b0, int& b1) {
  b0 = (r == 8 || r >= 10) ? 8 : (r == 4 || r == 6) ? 4 : 2;  // 10, 11: the container
  b1 = (r == 3) ? 1 : (r == 6) ? 2 : 0;
}

template <int SIG>
__device__ __forceinline__ uint32_t shift_to(uint32_t w) {
  if constexpr (SIG < 0) return w << (-SIG);
  else if constexpr (SIG == 0) return w;
  else return w >> SIG;
}

// (a & mask) | magic in one LOP3: both constants travel in registers, so the
// instruction needs no second immediate.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t mask, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
  return d;
}

// bf16x2 powers of two 2^e in both halves (OR-ing a code into the mantissa
// gives 2^e + code * 2^(e-7+p) exactly).
constexpr uint32_t kMag4 = 0x40804080u, kMag8 = 0x41004100u, kMag16 = 0x41804180u,
                   kMag32 = 0x42004200u, kMag64 = 0x42804280u,
                   kMag256 = 0x43804380u;
constexpr uint32_t kMaskP3b2 = 0x00180018u, kMaskP5b2 = 0x00600060u, kMaskP3b4 = 0x00780078u;

// Two bytes of w (chosen by the byte_perm selectors, which put the byte under
// the exponent of 2^23) as an exact bf16x2 pair of integers 0..255.
__device__ __forceinline__ uint32_t bytes_bf16x2(uint32_t w, uint32_t sel_lo, uint32_t sel_hi) {
  const float lo = __uint_as_float(__byte_perm(w, 0x4B000000u, sel_lo)) - 8388608.0f;
  const float hi = __uint_as_float(__byte_perm(w, 0x4B000000u, sel_hi)) - 8388608.0f;
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// The pair of 2-bit codes at half-word position P (0, 2, ..., 14) of a plane
// word as bf16x2. A left shift by 1 puts positions 0-4 at bits 1, 3, 5 of
// each half, right shifts by 5 and 11 do the same for 6-10 and 12-14, so a
// word costs three shifts and eight LOP3s. The code sits under the magic
// 2^(7-p) that gives it weight 1: offsets 64, 16, 4 (the bits shifted in
// from the other half fall outside the mask). An earlier form used shifts of
// 0, 6, 12 and took the offset 128 of bit 0 out with a bf16x2 subtract: one
// instruction more per word.
template <int P>
__device__ __forceinline__ uint32_t pick2(uint32_t w) {
  constexpr int sh = P <= 4 ? -1 : (P <= 10 ? 5 : 11);
  constexpr int p = P - sh;
  constexpr uint32_t mask = 0x00030003u << p;
  return and_or(shift_to<sh>(w), mask, p == 1 ? kMag64 : p == 3 ? kMag16 : kMag4);
}

// Decoded A registers of one MMA for one weight row: x0 fills k-slots
// {2t, 2t+1}, x1 fills {2t+8, 2t+9}. PLANE 0 is the low plane, 1 the high
// plane; Q is the 8-code group of the chunk, HF the 4-code half of it.
template <int R, int PLANE, int Q, int HF>
__device__ __forceinline__ void decode_quad(const uint32_t (&lo)[4], const uint32_t (&hi)[2],
                                            const Cdec& cd, uint32_t& x0, uint32_t& x1) {
  if constexpr (R == 10 || R == 11) {
    // container bytes c0..c3 of one word, registers pair (c0, c2) and (c1, c3)
    // as the r = 8 plane does; q + h never leaves its 16-bit half
    const uint32_t w = lo[2 * Q + HF];
    const uint32_t ev = w & 0x00FF00FFu;
    const uint32_t od = __byte_perm(w, 0u, 0x4341);
    if constexpr (R == 10) {
      x0 = and_or(__viaddmin_u16x2(ev, cd.h2, 0x00FF00FFu) >> 1, cd.kmask, cd.mag);
      x1 = and_or(__viaddmin_u16x2(od, cd.h2, 0x00FF00FFu) >> 1, cd.kmask, cd.mag);
    } else {
      x0 = and_or((ev + cd.h2) >> 2, cd.kmask, cd.mag);
      x1 = and_or((od + cd.h2) >> 2, cd.kmask, cd.mag);
    }
  } else if constexpr (R == 2) {
    // 2-bit codes, word = 16 codes; x0 holds codes 4j, 4j+1 (half-word
    // position 4j), x1 codes 4j+2, 4j+3 (position 4j+2), j = 2(Q%2)+HF.
    constexpr int j = 2 * (Q % 2) + HF;
    x0 = pick2<4 * j>(lo[Q / 2]);
    x1 = pick2<4 * j + 2>(lo[Q / 2]);
  } else if constexpr (R == 3 && PLANE == 0) {
    // 2-bit codes, word = 16 codes; pairs 2j, 2j+1 (j = 2(Q%2)+HF) at half-bits
    // 4j, 4j+2 -> bits 3-4 (16 + c) and bits 5-6 (4 + c) after one shift.
    constexpr int j = 2 * (Q % 2) + HF;
    const uint32_t sh = shift_to<4 * j - 3>(lo[Q / 2]);
    x0 = and_or(sh, kMaskP3b2, kMag16);
    x1 = and_or(sh, kMaskP5b2, kMag4);
  } else if constexpr (R == 4 || (R == 6 && PLANE == 0)) {
    // 4-bit codes, word = 8 codes; pairs 2HF, 2HF+1 at half-bits 8HF, 8HF+4 -> bits 3-6 (16 + c)
    const uint32_t w = lo[Q];
    x0 = and_or(shift_to<8 * HF - 3>(w), kMaskP3b4, kMag16);
    x1 = and_or(shift_to<8 * HF + 1>(w), kMaskP3b4, kMag16);
  } else if constexpr (R == 8) {
    // bytes c0..c3 of one word; registers pair (c0, c2) and (c1, c3). A byte
    // has 8 significant bits, one more than a bf16 mantissa holds under a
    // magic exponent, so it goes through fp32: 2^23 + c minus 2^23 is c, and
    // its conversion to bf16 is exact. No offset remains.
    const uint32_t w = lo[2 * Q + HF];
    x0 = bytes_bf16x2(w, 0x7440u, 0x7442u);
    x1 = bytes_bf16x2(w, 0x7441u, 0x7443u);
  } else if constexpr (R == 3) {
    // high 1-bit plane (weight 4), word = 32 codes; pairs P = 4(Q%4)+2HF, +1 at
    // half-bit P; one shift puts the group's 4 pairs at bits 3..6 (64/32/16/8 + 4h)
    const uint32_t sh = shift_to<4 * (Q % 4) - 3>(hi[Q / 4]);
    constexpr int p0 = 3 + 2 * HF;
    constexpr uint32_t m0 = (1u << p0) | (1u << (16 + p0));
    constexpr uint32_t m1 = (1u << (p0 + 1)) | (1u << (17 + p0));
    x0 = and_or(sh, m0, HF == 0 ? kMag64 : kMag16);
    x1 = and_or(sh, m1, HF == 0 ? kMag32 : kMag8);
  } else {  // R == 6, high 2-bit plane (weight 16), word = 16 codes
    constexpr int j = 2 * (Q % 2) + HF;
    const uint32_t sh = shift_to<4 * j - 3>(hi[Q / 2]);
    x0 = and_or(sh, kMaskP3b2, kMag256);
    x1 = and_or(sh, kMaskP5b2, kMag64);
  }
}

// Offset of the decoded value per activation class (k >> 1) & 7 for each
// width (the sum over the planes of the magic added to the code). The offsets
// stay small next to the code unit (at most 32 at r = 2), so the fp32 sums
// lose little to cancellation when the offsets are taken out again.
__device__ __forceinline__ void offset_coeffs(int dk, int r, float (&c)[kClasses]) {
  constexpr float r2[kClasses] = {64.f, 16.f, 4.f, 64.f, 16.f, 4.f, 64.f, 16.f};
  constexpr float r3[4] = {80.f, 36.f, 32.f, 12.f};
  constexpr float r6[4] = {272.f, 80.f, 272.f, 80.f};
  // the container sliced on load: one magic for every class
  const float cont = static_cast<float>(1 << (dk == 10 ? r : r + 1));
#pragma unroll
  for (int i = 0; i < kClasses; ++i) {
    c[i] = dk >= 10 ? cont : r == 8 ? 0.f : r == 4 ? 16.f : r == 2 ? r2[i] : r == 3 ? r3[i & 3] : r6[i & 3];
  }
}

// All MMAs of one 8-code activation group: for each 4-code half and each
// plane, one m16n8k16 per batch tile, the B registers shared by the planes.
template <int R, int NT, int TW, int Q>
__device__ __forceinline__ void group_mmas(const uint32_t (&lo)[TW][2][4], const uint32_t (&hi)[TW][2][2],
                                           const uint32_t (&xaddr)[NT], const uint32_t (&xstep)[NT],
                                           int gbase, const Cdec& cd, uint32_t* errp,
                                           float (&ch)[TW][NT][2][4]) {
  uint4 xb[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    // a plain shared-memory load (the CTA's dynamic shared array plus an
    // offset), so the compiler may hoist it ahead of the decode work; the
    // mbarrier wait before the unit is a memory barrier it cannot cross
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t a = xaddr[nt] + static_cast<uint32_t>(gbase + Q) * xstep[nt];
    xb[nt] = make_uint4(0u, 0u, 0u, 0u);
    if (MQ_IN_BOUNDS(a + 16u <= dynamic_smem_bytes(), errp))
      xb[nt] = *reinterpret_cast<const uint4*>(smem + a);
  }
  // two operand planes for r = 3, 6 (low/high bit planes)
  constexpr int NPL = (Geo<R>::b1 != 0) ? 2 : 1;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
    for (int pl = 0; pl < NPL; ++pl) {
#pragma unroll
      for (int T = 0; T < TW; ++T) {
        uint32_t a0, a1, a2, a3;
        if (hf == 0 && pl == 0) { decode_quad<R, 0, Q, 0>(lo[T][0], hi[T][0], cd, a0, a2); decode_quad<R, 0, Q, 0>(lo[T][1], hi[T][1], cd, a1, a3); }
        if (hf == 0 && pl == 1) { decode_quad<R, 1, Q, 0>(lo[T][0], hi[T][0], cd, a0, a2); decode_quad<R, 1, Q, 0>(lo[T][1], hi[T][1], cd, a1, a3); }
        if (hf == 1 && pl == 0) { decode_quad<R, 0, Q, 1>(lo[T][0], hi[T][0], cd, a0, a2); decode_quad<R, 0, Q, 1>(lo[T][1], hi[T][1], cd, a1, a3); }
        if (hf == 1 && pl == 1) { decode_quad<R, 1, Q, 1>(lo[T][0], hi[T][0], cd, a0, a2); decode_quad<R, 1, Q, 1>(lo[T][1], hi[T][1], cd, a1, a3); }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t b0 = hf ? xb[nt].z : xb[nt].x;
          const uint32_t b1 = hf ? xb[nt].w : xb[nt].y;
          mma_bf16_16816(ch[T][nt][(2 * Q + hf + pl) & 1], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
}

template <int R, int NT, int TW, int... Qs>
__device__ __forceinline__ void chunk_mmas(const uint32_t (&lo)[TW][2][4], const uint32_t (&hi)[TW][2][2],
                                           const uint32_t (&xaddr)[NT], const uint32_t (&xstep)[NT],
                                           int gbase, const Cdec& cd, uint32_t* errp,
                                           float (&ch)[TW][NT][2][4],
                                           std::integer_sequence<int, Qs...>) {
  (group_mmas<R, NT, TW, Qs>(lo, hi, xaddr, xstep, gbase, cd, errp, ch), ...);
}

// One staged unit for this warp's 16-row tiles. All sub-steps are unrolled
// and their plane loads issued first. Sub-steps past the unit's valid codes
// read zero-filled planes and zero activations and add nothing. Activation
// group q of chunk 4s+t for batch row m sits at ((((s*W8 + q)*M + m)*4 + t)
// * 16) bytes of the staged block; lanes whose batch row is past M read a
// zero block instead (step 0). With 128-byte plane rows the box is stored in
// 128-byte swizzled atoms: chunk c of row r at chunk c ^ (r % 8).
template <int R, int NT>
__device__ __forceinline__ void process_unit(const uint8_t* st0, const uint8_t* st1,
                                             const uint32_t (&xaddr)[NT],
                                             const uint32_t (&xstep)[NT], int warp, int lane,
                                             const Cdec& cd, uint32_t* errp,
                                             float (&ch)[Tiling<NT>::TW][NT][2][4]) {
  using G = Geo<R>;
  using TL = Tiling<NT>;
  constexpr int TW = TL::TW, NSUB = TL::NSUB, P0 = TL::P0, P1 = TL::P0 / 2;
  const int g = lane >> 2, t = lane & 3;
  uint32_t lo[NSUB][TW][2][4];
  uint32_t hi[NSUB][TW][2][2];
#pragma unroll
  for (int s = 0; s < NSUB; ++s) {
    const int ci = 4 * s + t;  // this thread's 16-byte chunk of the low plane
#pragma unroll
    for (int T = 0; T < TW; ++T) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = warp * TL::RPW + 16 * T + g + 8 * h;
        const int cs = TL::SWZ ? (ci ^ (row & 7)) : ci;
        const uint4 v = *reinterpret_cast<const uint4*>(st0 + row * P0 + cs * 16);
        lo[s][T][h][0] = v.x; lo[s][T][h][1] = v.y; lo[s][T][h][2] = v.z; lo[s][T][h][3] = v.w;
        if constexpr (G::b1 != 0) {
          const uint2 u = *reinterpret_cast<const uint2*>(st1 + row * P1 + ci * 8);
          hi[s][T][h][0] = u.x; hi[s][T][h][1] = u.y;
        } else {
          hi[s][T][h][0] = 0; hi[s][T][h][1] = 0;
        }
      }
    }
  }
#pragma unroll
  for (int s = 0; s < NSUB; ++s)
    chunk_mmas<R, NT, TW>(lo[s], hi[s], xaddr, xstep, s * G::W8, cd, errp, ch,
                          std::make_integer_sequence<int, G::W8>{});
}

// The current linear of a CTA's walk over its unit range, cached in registers.
struct Cursor {
  int l, rb, kc;          // linear, row block, k-chunk of the current unit
  int nrb, n_kc, r, N;    // of linear l
  int dk;                 // its decode kind (width, or 10 / 11 for the container)
};

template <int RPU, int CAP>
__device__ __forceinline__ void cursor_load(const GemvParams<CAP>& p, Cursor& c) {
  const LinDesc& L = p.lin[c.l];
  c.n_kc = L.n_kc;
  c.nrb = (L.N + RPU - 1) / RPU;
  c.r = L.r;
  c.N = L.N;
  c.dk = L.dk;
}

template <int RPU, int CAP>
__device__ __forceinline__ void cursor_init(const GemvParams<CAP>& p, int u, Cursor& c) {
  int l = 0;
  while (l + 1 < p.n_lin && u >= p.lin[l + 1].unit_begin) ++l;
  c.l = l;
  cursor_load<RPU>(p, c);
  const int local = u - p.lin[l].unit_begin;
  c.rb = local / c.n_kc;
  c.kc = local - c.rb * c.n_kc;
}

template <int RPU, int CAP>
__device__ __forceinline__ void cursor_next(const GemvParams<CAP>& p, Cursor& c) {
  if (++c.kc == c.n_kc) {
    c.kc = 0;
    if (++c.rb == c.nrb) {
      c.rb = 0;
      ++c.l;
      if (c.l < p.n_lin) cursor_load<RPU>(p, c);
    }
  }
}

// Epilogue of one row block of this warp's 16 rows: scales the raw sums,
// removes the decoding offsets and the zero point (once per row, by the part
// that starts at k-chunk 0) and writes y. A row block this CTA owns whole is
// stored; a shared one is added atomically into y, which the prep kernel
// zeroed.
template <int NT, int CAP>
__device__ void flush_rows(const GemvParams<CAP>& p, int l, int rb, int kc0, bool whole, int warp,
                           int T, int lane, const float (&tot)[NT][4]) {
  const LinDesc& L = p.lin[l];
  const int g = lane >> 2, t = lane & 3;
  const float scale = static_cast<float>(1 << (8 - L.r));
  float c[kClasses];
  offset_coeffs(L.dk, L.r, c);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int n = rb * Tiling<NT>::RPU + warp * Tiling<NT>::RPW + 16 * T + g + 8 * h;
    if (n >= L.N) continue;
    const float a = L.alpha[n], z = L.zero[n];
    const float A = a * scale, B = a * z;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int m = nt * 8 + 2 * t + e;
        if (m >= p.M) continue;
        float v = tot[nt][2 * h + e];
        if (kc0 == 0) {
          // Extra Precision: each listed position adds one code step
          if (L.epc) v += L.epc[static_cast<int64_t>(m) * L.N + n];
          const float* P = L.psum + m * kClasses;
          float O = 0.f, Sx = 0.f;
#pragma unroll
          for (int i = 0; i < kClasses; ++i) {
            O = fmaf(c[i], P[i], O);
            Sx += P[i];
          }
          v = A * (v - O) - B * Sx;
        } else {
          v = A * v;
        }
        float* dst = L.y + static_cast<int64_t>(m) * L.N + n;
        if (whole) *dst = v;
        else atomicAdd(dst, v);
      }
    }
  }
}

// Consumes `seg` consecutive staged units of one row block at width R and
// adds them into `tot`. The two MMA accumulator chains are folded into `tot`
// after every unit, which keeps each fp32 chain short. Returns false if a wait
// gave up (the abort flag is then set for the whole CTA).
template <int R, int NT, int CAP>
__device__ __forceinline__ bool run_segment(const GemvParams<CAP>& p, const uint8_t* stages,
                                            uint64_t* full, uint64_t* empty,
                                            volatile int* s_abort, int seg, int& s, uint32_t& ph,
                                            bool active, const uint32_t (&xaddr)[NT],
                                            const uint32_t (&xstep)[NT], int warp, int lane,
                                            const Cdec& cd, float (&tot)[Tiling<NT>::TW][NT][4]) {
  constexpr int TW = Tiling<NT>::TW;
  for (int i = 0; i < seg; ++i) {
    if (*s_abort || !mbar_wait_bounded(&full[s], ph, p.wait_ns)) {
      if (lane == 0) { atomicOr(p.err, kErrWaitFull); *s_abort = 1; }
      return false;
    }
    if (active) {
      const uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
      extern __shared__ __align__(128) uint8_t smem[];
      const uint32_t xs = static_cast<uint32_t>(st + p.off_x - smem);  // offset in shared memory
      uint32_t xa[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) xa[nt] = xstep[nt] ? xs + xaddr[nt] : xaddr[nt];
      float ch[TW][NT][2][4];
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int b = 0; b < NT; ++b)
#pragma unroll
          for (int j = 0; j < 4; ++j) { ch[T][b][0][j] = 0.f; ch[T][b][1][j] = 0.f; }
      // the plane pitches and rows follow from the batch tiles (Tiling)
      process_unit<R, NT>(st, st + Tiling<NT>::RPU * Tiling<NT>::P0, xa, xstep, warp, lane, cd, p.err, ch);
#pragma unroll
      for (int T = 0; T < TW; ++T)
#pragma unroll
        for (int b = 0; b < NT; ++b)
#pragma unroll
          for (int j = 0; j < 4; ++j) tot[T][b][j] += ch[T][b][0][j] + ch[T][b][1][j];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == p.stages) { s = 0; ph ^= 1u; }
  }
  return true;
}

template <int NT, int CAP>
__global__ void __launch_bounds__(kGemvThreads, (NT <= 2 ? 2 : 1))
gemv_streamk_kernel(const __grid_constant__ GemvParams<CAP> p) {
  using TL = Tiling<NT>;
  extern __shared__ __align__(128) uint8_t smem[];
  // 1024-byte aligned header and stages: the swizzled plane boxes need it
  const uint32_t raw = smem_u32(smem);
  uint8_t* base = smem + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base);
  uint64_t* empty = full + kMaxStages;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kMaxStages);
  uint8_t* zero_block = base + kHeaderBytes - 64;  // 64 zero bytes read by lanes past M
  uint8_t* stages = base + kHeaderBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.stages;
  // The next kernel in the stream may be scheduled once every CTA of this
  // grid is resident; it waits for this grid's completion before it reads.
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) reinterpret_cast<uint32_t*>(zero_block)[threadIdx.x] = 0u;
  __syncthreads();

  const int u0 = p.cta_begin[blockIdx.x];
  const int u1 = p.cta_begin[blockIdx.x + 1];
  if (u0 >= u1) return;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    // Weight boxes do not depend on the prep kernel, so the first stages'
    // boxes are requested before waiting for it; their activation blocks
    // follow once the prep grid has finished.
    bool aborted = false;
    int issued = 0;
    if (lane == 0) {
      Cursor c;
      cursor_init<TL::RPU>(p, u0, c);
      Cursor pre_c = c;
      auto issue_weights = [&](const Cursor& cc, int s) {
        int b0, b1;
        plane_widths_dev(cc.dk, b0, b1);
        uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
        const CUtensorMap* tm = p.map_table ? p.map_table + 2 * cc.l : &p.maps[2 * cc.l];
        const uint32_t box = TL::RPU * (p.pitch0 + (b1 ? p.pitch1 : 0));
        const uint32_t bytesx = static_cast<uint32_t>(p.M * p.lin[cc.l].kc * 2);
        // One 2-D box per plane (128 rows x the unit's bytes; rows past N and
        // bytes past K read as zero) plus the unit's activation block.
        mbar_arrive_expect_tx(&full[s], box + bytesx);
        tma_load_2d(st, tm, cc.kc * p.pitch0, cc.rb * TL::RPU, &full[s]);
        if (b1) tma_load_2d(st + p.off_plane1, tm + 1, cc.kc * p.pitch1, cc.rb * TL::RPU, &full[s]);
      };
      auto issue_x = [&](const Cursor& cc, int s) {
        const LinDesc& L = p.lin[cc.l];
        const uint32_t bytesx = static_cast<uint32_t>(p.M * L.kc * 2);
        uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
        bulk_g2s(st + p.off_x, L.xf + int64_t(cc.kc) * bytesx, bytesx, &full[s]);
      };
      const int pre = min(S, u1 - u0);
      for (int i = 0; i < pre; ++i) { issue_weights(c, i); cursor_next<TL::RPU>(p, c); }
      pdl_wait_primary();
      for (int i = 0; i < pre; ++i) { issue_x(pre_c, i); cursor_next<TL::RPU>(p, pre_c); }
      issued = pre;
      for (int u = u0 + pre; u < u1; ++u, ++issued) {
        const int s = issued % S;
        if (!mbar_wait_bounded(&empty[s], ((issued / S) - 1) & 1, p.wait_ns)) {
          atomicOr(p.err, kErrWaitEmpty);
          *s_abort = 1;
          aborted = true;
          break;
        }
        if (*s_abort) { aborted = true; break; }
        issue_weights(c, s);
        issue_x(c, s);
        cursor_next<TL::RPU>(p, c);
      }
      // Leave no bulk copy in flight when this thread exits, whether or not
      // the consumers took the data (they stop early after a wait gave up):
      // wait for the last issue of every stage.
      (void)aborted;
      const int first = issued > S ? issued - S : 0;
      for (int j = first; j < issued; ++j) {
        if (!mbar_wait_bounded(&full[j % S], (j / S) & 1, 1000000000ull)) atomicOr(p.err, kErrDrain);
      }
    } else {
      pdl_wait_primary();
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // Class sums and the zeroed outputs come from the prep kernel.
  pdl_wait_primary();
  const int g = lane >> 2, t = lane & 3;
  uint32_t xaddr[NT], xstep[NT];
  const uint32_t zero_addr = static_cast<uint32_t>(zero_block - smem) + t * 16;  // shared offset
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int m = nt * 8 + g;
    xaddr[nt] = zero_addr;
    xstep[nt] = 0;
    if (m < p.M) {
      xaddr[nt] = static_cast<uint32_t>((m * 4 + t) * 16);  // + stage x base, per unit
      xstep[nt] = static_cast<uint32_t>(p.M) * 64u;
    }
  }
  Cursor c;
  cursor_init<TL::RPU>(p, u0, c);
  int s = 0;
  uint32_t ph = 0;
  for (int u = u0; u < u1;) {
    // One row block: units kc0 .. kc0 + seg - 1 of (linear c.l, row block c.rb).
    const int seg = min(c.n_kc - c.kc, u1 - u);
    const int kc0 = c.kc;
    const bool whole = kc0 == 0 && seg == c.n_kc;
    const bool active = warp * TL::RPW < c.N - c.rb * TL::RPU;
    float tot[TL::TW][NT][4];
#pragma unroll
    for (int T = 0; T < TL::TW; ++T)
#pragma unroll
      for (int b = 0; b < NT; ++b)
#pragma unroll
        for (int i = 0; i < 4; ++i) tot[T][b][i] = 0.f;
    bool ok;
    const Cdec cd = make_cdec(c.dk, c.r);
    switch (c.dk) {
      case 2: ok = run_segment<2, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, tot); break;
      case 4: ok = run_segment<4, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, tot); break;
      case 8: ok = run_segment<8, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, tot); break;
      case 3: ok = run_segment<3, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, tot); break;
      case 10: ok = run_segment<10, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, tot); break;
      case 11: ok = run_segment<11, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, tot); break;
      default: ok = run_segment<6, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, tot); break;
    }
    if (!ok) break;  // outputs are undefined after a give-up; the flag says so
    if (active) {
#pragma unroll
      for (int T = 0; T < TL::TW; ++T) flush_rows<NT>(p, c.l, c.rb, kc0, whole, warp, T, lane, tot[T]);
    }
    u += seg;
    c.kc += seg;
    if (c.kc == c.n_kc) {
      c.kc = 0;
      if (++c.rb == c.nrb) {
        c.rb = 0;
        if (++c.l < p.n_lin) cursor_load<TL::RPU>(p, c);
      }
    }
  }
}

// ------------------------------------------------------------------ prep
struct PrepLayout {
  const __nv_bfloat16* x;
  uint8_t* xf;
  int K, kc, w8, n_kc;
  int perm02;  // byte planes pair codes (c0, c2), (c1, c3): store x0, x2, x1, x3
};
struct PrepSum {
  const __nv_bfloat16* x;
  float* psum;
  int K;
};
// A row block of an output that two or more CTAs add into: y[m, 128 rb ..
// 128 rb + 127] for every m (columns past N excluded).
struct PrepZero {
  float* y;
  int N, rb;
};
// Extra Precision sums of one linear: out[m * N + n] = sum over row n's
// listed positions k (cols[rows[n] .. rows[n + 1])) of x[m, k].
struct PrepEp {
  const int* rows;
  const uint16_t* cols;
  const __nv_bfloat16* x;
  float* out;
  int N, K;
};
constexpr int kMaxEpJobs = 8;
template <int CAP>
struct PrepParams {
  uint32_t* err;  // device error word (index checks of the debug build)
  int M, n_layout, n_sum, n_zero, n_ep;
  int rows;  // weight rows per unit: the height of a zeroed row block
  PrepLayout lay[CAP];
  PrepSum sum[CAP];
  PrepZero zero[kMaxCtas];
  PrepEp ep[kMaxEpJobs];
};
static_assert(sizeof(PrepParams<kGemvMaxLinears>) <= 32764, "prep kernel parameters too large");

// Builds the fragment-ordered activation blocks (zero-padded to whole
// k-chunks) and the per-class activation sums, and zeroes the output row
// blocks that several CTAs add into.
template <int CAP>
__global__ void __launch_bounds__(256) gemv_prep_kernel(const __grid_constant__ PrepParams<CAP> p) {
  // The decode kernel may start now (its weight boxes do not depend on this
  // grid); this grid itself may have started before its predecessor in the
  // stream finished, so it waits for it before touching memory.
  pdl_launch_dependents();
  pdl_wait_primary();
  const int M = p.M;
  // (1) class sums: one CTA per (sum job, batch row)
  if (blockIdx.x < p.n_sum * M) {
    const PrepSum& J = p.sum[blockIdx.x / M];
    const int m = blockIdx.x % M;
    const __nv_bfloat16* row = J.x + int64_t(m) * J.K;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    // 8 consecutive elements k0..k0+7 (k0 % 8 == 0) fall in classes
    // 4h, 4h, 4h+1, 4h+1, ..., 4h+3 with h = (k0 >> 3) & 1; the stride of
    // the loop is a multiple of 16, so h is the parity of the thread.
    for (int k0 = threadIdx.x * 8; k0 < J.K; k0 += blockDim.x * 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + k0);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        acc[i] += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xFFFF0000u);
    }
    __shared__ float red[kClasses][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = acc[i];
#pragma unroll
      for (int o = 16; o > 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);  // same parity
      const int lane = threadIdx.x & 31;
      if (lane < 2) red[4 * lane + i][threadIdx.x >> 5] = v;
    }
    __syncthreads();
    if (threadIdx.x < kClasses) {
      float v = 0.f;
      for (int w8 = 0; w8 < (int)(blockDim.x >> 5); ++w8) v += red[threadIdx.x][w8];
      J.psum[m * kClasses + threadIdx.x] = v;
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
      if (L.perm02) {
        const uint32_t a = __byte_perm(v.x, v.y, 0x5410), b = __byte_perm(v.x, v.y, 0x7632);
        const uint32_t c = __byte_perm(v.z, v.w, 0x5410), d = __byte_perm(v.z, v.w, 0x7632);
        v = make_uint4(a, b, c, d);
      }
      const int s = grp / (4 * L.w8);
      const int rem = grp % (4 * L.w8);
      const int t = rem / L.w8, q = rem % L.w8;
      const int64_t off = int64_t(kc) * M * L.kc * 2 +
                          ((int64_t(s * L.w8 + q) * M + m) * 4 + t) * 16;
      if (MQ_IN_BOUNDS(off + 16 <= int64_t(L.n_kc) * M * L.kc * 2, p.err))
        *reinterpret_cast<uint4*>(L.xf + off) = v;
    }
  }
  // (4) Extra Precision sums: one warp per (job, row). With M' the next power
  // of two >= M, lane l takes batch row l % M' and every (32 / M')-th listed
  // position; lanes of one batch row then add up with shuffles.
  if (p.n_ep > 0) {
    int mp = 1;
    while (mp < M) mp <<= 1;
    const int lane = threadIdx.x & 31;
    const int m = lane & (mp - 1), jo = lane / mp, P = 32 / mp;
    const int64_t warps = stride / 32;
    int64_t total_rows = 0;
    for (int i = 0; i < p.n_ep; ++i) total_rows += p.ep[i].N;
    for (int64_t w = tid / 32; w < total_rows; w += warps) {
      int job = 0;
      int64_t n = w;
      while (n >= p.ep[job].N) { n -= p.ep[job].N; ++job; }
      const PrepEp& E = p.ep[job];
      const int beg = E.rows[n], end = E.rows[n + 1];
      float acc = 0.f;
      if (m < M) {
        const __nv_bfloat16* xr = E.x + int64_t(m) * E.K;
#pragma unroll 4
        for (int j = beg + jo; j < end; j += P) {
          const int k = E.cols[j];
          if (MQ_IN_BOUNDS(k < E.K, p.err)) acc += __bfloat162float(xr[k]);
        }
      }
      for (int o = mp; o < 32; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (jo == 0 && m < M) E.out[int64_t(m) * E.N + n] = acc;
    }
  }
  // (3) zero the shared output row blocks
  const int64_t zt = int64_t(p.n_zero) * M * p.rows;
  for (int64_t i = tid; i < zt; i += stride) {
    const PrepZero& Z = p.zero[i / (int64_t(M) * p.rows)];
    const int rem = static_cast<int>(i % (int64_t(M) * p.rows));
    const int m = rem / p.rows;
    const int n = Z.rb * p.rows + rem % p.rows;
    if (n < Z.N) Z.y[int64_t(m) * Z.N + n] = 0.f;
  }
}

// Per-(device, kernel instantiation) launch facts, computed once: the
// dynamic shared-memory limit is raised to the largest stage plan and the
// occupancy of each shared-memory size is remembered.
struct KernelCache {
  bool attr_set = false;
  std::map<size_t, int> occ;
};
std::mutex g_cache_mutex;

// Persistent grid for `units` work units at `smem` bytes of shared memory:
// every resident CTA slot of the device, at most one CTA per unit.
template <int NT, int CAP>
cudaError_t gemv_grid(size_t smem, int sms, int units, int* grid_out) {
  auto kern = gemv_streamk_kernel<NT, CAP>;
  static std::map<int, KernelCache> caches;
  int dev = 0;
  cudaGetDevice(&dev);
  int occ = 1;
  {
    std::lock_guard<std::mutex> lk(g_cache_mutex);
    KernelCache& kc = caches[dev];
    if (!kc.attr_set) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kMaxDynSmem);
      if (e != cudaSuccess) return e;
      kc.attr_set = true;
    }
    auto it = kc.occ.find(smem);
    if (it == kc.occ.end()) {
      int blocks = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kGemvThreads, smem) != cudaSuccess ||
          blocks < 1)
        blocks = 1;
      it = kc.occ.emplace(smem, blocks).first;
    }
    occ = it->second;
  }
  *grid_out = std::max(1, std::min(std::min(units, sms * occ), kMaxCtas));
  return cudaSuccess;
}

template <int NT, int CAP>
cudaError_t launch_gemv(const GemvParams<CAP>& gp, size_t smem, int grid, cudaStream_t stream) {
  auto kern = gemv_streamk_kernel<NT, CAP>;
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

// Device tables of tensor maps for large launches, one per distinct list of
// (planes address, N, K, r) and box width. Built with a synchronous copy the
// first time a stack is served (so the first call must not be captured),
// then reused by every later identical call.
std::map<std::pair<int, std::vector<uint64_t>>, CUtensorMap*> g_map_tables;

cudaError_t encode_plane_maps(const LinearJob& j, int P0, CUtensorMap* out2) {
  int b0, b1;
  job_planes(j, b0, b1);
  // 128-byte plane-0 rows go with 256-row units and the 128-byte swizzle
  const uint32_t rows = P0 == 128 ? 256u : 128u;
  cudaError_t e = encode_map_2d(&out2[0], j.packed, uint64_t(j.N), uint64_t(j.K) * b0 / 8,
                                static_cast<uint32_t>(P0), rows, 1, P0 == 128 ? 128 : 0);
  if (e != cudaSuccess || !b1) return e;
  return encode_map_2d(&out2[1], j.packed + j.N * j.K * b0 / 8, uint64_t(j.N),
                       uint64_t(j.K) * b1 / 8, static_cast<uint32_t>(P0 / 2), rows, 1);
}

cudaError_t get_map_table(const LinearJob* jobs, int n_jobs, int P0, const CUtensorMap** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::vector<uint64_t> key;
  key.reserve(size_t(n_jobs) * 4 + 1);
  key.push_back(uint64_t(P0));
  for (int i = 0; i < n_jobs; ++i) {
    key.push_back(reinterpret_cast<uint64_t>(jobs[i].packed));
    key.push_back(uint64_t(jobs[i].N));
    key.push_back(uint64_t(jobs[i].K));
    key.push_back(uint64_t(jobs[i].r) | (uint64_t(jobs[i].src) << 8));
  }
  std::lock_guard<std::mutex> lk(g_cache_mutex);
  auto k2 = std::make_pair(dev, std::move(key));
  auto it = g_map_tables.find(k2);
  if (it != g_map_tables.end()) {
    *out = it->second;
    return cudaSuccess;
  }
  std::vector<CUtensorMap> host(size_t(n_jobs) * 2);
  std::memset(host.data(), 0, host.size() * sizeof(CUtensorMap));
  for (int i = 0; i < n_jobs; ++i) {
    e = encode_plane_maps(jobs[i], P0, &host[size_t(2) * i]);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap* dptr = nullptr;
  e = cudaMalloc(&dptr, host.size() * sizeof(CUtensorMap));
  if (e != cudaSuccess) return e;
  e = cudaMemcpy(dptr, host.data(), host.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) { cudaFree(dptr); return e; }
  g_map_tables.emplace(std::move(k2), dptr);
  *out = dptr;
  return cudaSuccess;
}

// Relative cost of one unit of each width, for cutting the CTA ranges. A unit
// always holds the same plane bytes per row (two planes hold 1.5x), while the
// decode and MMA work grows with the codes in it: per-unit times of
// single-width stacks on B200 at M = 1 put r = 4 at about 1.26x and r = 2 at
// about 1.88x an r = 8 unit; r = 3 and 6 are scaled from their planes.
int64_t unit_cost(const LinearJob& j) {
  switch (decode_kind(j)) {
    case 8: return 100;
    case 4: return 126;
    case 2: return 188;
    case 6: return 183;
    case 10: case 11: return 110;  // one 8-bit plane, one MMA per 16 codes, more decode work
    default: return 301;  // 3
  }
}

template <int CAP>
cudaError_t run_gemv_cap(const LinearJob* jobs, int n_jobs, int M, cudaStream_t stream,
                         const FixedScratch* fixed = nullptr) {
  // Plane-0 bytes per row per unit and rows per unit (Tiling): 128 bytes in
  // 256-row units up to 8 batch rows, 64 bytes in 128-row units above.
  const int P0 = tiling_p0(M);
  const int RU = tiling_rows(M);
  const int NT = (M + 7) / 8;

  static thread_local GemvParams<CAP> gp;
  static thread_local PrepParams<CAP> pp;

  // Distinct inputs (class sums) and distinct (input, layout) pairs. Few
  // entries: linear scans are cheaper than maps here.
  struct LayoutInfo { const void* x; int b0, K, kc, w8, n_kc; size_t off; };
  LayoutInfo layouts[CAP];
  const void* sum_x[CAP];
  int sum_k[CAP];
  int n_layouts = 0, n_sums = 0;
  int lay_of[CAP], sum_of[CAP];
  bool two_planes = false;
  int units = 0;
  size_t xf_bytes = 0;
  for (int i = 0; i < n_jobs; ++i) {
    const LinearJob& j = jobs[i];
    int b0, b1;
    job_planes(j, b0, b1);
    if (b1) two_planes = true;
    const int kc = P0 * 8 / b0;
    const int n_kc = static_cast<int>((j.K + kc - 1) / kc);
    int si = 0;
    while (si < n_sums && sum_x[si] != j.x) ++si;
    if (si == n_sums) { sum_x[n_sums] = j.x; sum_k[n_sums] = static_cast<int>(j.K); ++n_sums; }
    sum_of[i] = si;
    int li = 0;
    while (li < n_layouts && !(layouts[li].x == j.x && layouts[li].b0 == b0)) ++li;
    if (li == n_layouts) {
      layouts[n_layouts++] = {j.x, b0, static_cast<int>(j.K), kc, (128 / b0) / 8, n_kc, xf_bytes};
      xf_bytes += size_t(n_kc) * M * kc * 2;
      xf_bytes = (xf_bytes + 255) & ~size_t(255);
    }
    lay_of[i] = li;
    const int nrb = static_cast<int>((j.N + RU - 1) / RU);
    LinDesc& d = gp.lin[i];
    d.plane0 = j.packed;
    d.plane1 = b1 ? j.packed + j.N * j.K * b0 / 8 : nullptr;
    d.alpha = j.alpha;
    d.zero = j.zero;
    d.y = j.y;
    d.N = static_cast<int>(j.N);
    d.K = static_cast<int>(j.K);
    d.r = j.r;
    d.dk = decode_kind(j);
    d.epc = nullptr;  // set with the workspace below
    d.kc = kc;
    d.n_kc = n_kc;
    d.unit_begin = units;
    units += nrb * n_kc;
  }
  if constexpr (CAP <= 8) {
    for (int i = 0; i < n_jobs; ++i) {
      cudaError_t em = encode_plane_maps(jobs[i], P0, &gp.maps[2 * i]);
      if (em != cudaSuccess) return em;
    }
    gp.map_table = nullptr;
  } else {
    cudaError_t em = get_map_table(jobs, n_jobs, P0, &gp.map_table);
    if (em != cudaSuccess) return em;
  }
  const size_t psum_off = xf_bytes;
  // Extra Precision sums (M x N fp32 per linear that has a list) follow the class sums.
  size_t ep_off = (psum_off + size_t(n_sums) * M * kClasses * sizeof(float) + 255) & ~size_t(255);
  const size_t ep_begin = ep_off;
  int n_ep = 0;
  for (int i = 0; i < n_jobs; ++i) {
    if (!jobs[i].ep_rows) continue;
    if (++n_ep > kMaxEpJobs) return cudaErrorNotSupported;
    ep_off += (size_t(M) * jobs[i].N * sizeof(float) + 255) & ~size_t(255);
  }
  const size_t ws_bytes = ep_off + 256;
  void* ws = nullptr;
  cudaError_t e = cudaSuccess;
  if (fixed) {
    if (ws_bytes > fixed->bytes) return cudaErrorMemoryAllocation;
    ws = fixed->ptr;
  } else {
    e = get_workspace(stream, ws_bytes, &ws);
    if (e != cudaSuccess) return e;
  }
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* psum_base = reinterpret_cast<float*>(wsb + psum_off);
  for (int i = 0; i < n_jobs; ++i) {
    gp.lin[i].xf = wsb + layouts[lay_of[i]].off;
    gp.lin[i].psum = psum_base + size_t(sum_of[i]) * M * kClasses;
  }
  {
    size_t off = ep_begin;
    int k = 0;
    for (int i = 0; i < n_jobs; ++i) {
      const LinearJob& j = jobs[i];
      if (!j.ep_rows) continue;
      float* out = reinterpret_cast<float*>(wsb + off);
      gp.lin[i].epc = out;
      pp.ep[k++] = {j.ep_rows, j.ep_cols, static_cast<const __nv_bfloat16*>(j.x), out,
                    static_cast<int>(j.N), static_cast<int>(j.K)};
      off += (size_t(M) * j.N * sizeof(float) + 255) & ~size_t(255);
    }
    pp.n_ep = k;
  }

  // Stage layout: [128 rows x P0][128 rows x P1][M x KC bf16 activations].
  const int P1 = two_planes ? P0 / 2 : 0;
  const uint32_t off_plane1 = static_cast<uint32_t>(RU * P0);
  const uint32_t off_x = off_plane1 + static_cast<uint32_t>(RU * P1);
  const uint32_t x_bytes = static_cast<uint32_t>(M * (P0 * 8 / 2) * 2);  // largest KC (b0 = 2)
  uint32_t stage_bytes = off_x + x_bytes;
  stage_bytes = (stage_bytes + 1023) & ~1023u;  // swizzled boxes start 1024-aligned
  int stages = static_cast<int>(kStageBudget / stage_bytes);
  stages = std::max(2, std::min(stages, kMaxStages));
  const size_t smem = 1024 /* alignment slack */ + kHeaderBytes + size_t(stages) * stage_bytes;
  const int sms = sm_count();
  int grid = 1;
  switch (NT) {
    case 1: e = gemv_grid<1, CAP>(smem, sms, units, &grid); break;
    case 2: e = gemv_grid<2, CAP>(smem, sms, units, &grid); break;
    case 3: e = gemv_grid<3, CAP>(smem, sms, units, &grid); break;
    default: e = gemv_grid<4, CAP>(smem, sms, units, &grid); break;
  }
  if (e != cudaSuccess) return e;

  // CTA ranges of equal estimated cost, and the row blocks they share.
  int64_t total_cost = 0;
  for (int i = 0; i < n_jobs; ++i) {
    const int64_t lin_units = (i + 1 < n_jobs ? gp.lin[i + 1].unit_begin : units) - gp.lin[i].unit_begin;
    total_cost += lin_units * unit_cost(jobs[i]);
  }
  int n_zero = 0;
  {
    int li = 0;
    int64_t cost_before = 0;  // cost of the units before linear li
    for (int c = 0; c <= grid; ++c) {
      const int64_t target = (total_cost * c + grid - 1) / grid;  // ceil(c T / G)
      // first unit whose preceding cost reaches the target
      while (li < n_jobs) {
        const int64_t lin_units = (li + 1 < n_jobs ? gp.lin[li + 1].unit_begin : units) - gp.lin[li].unit_begin;
        const int64_t lin_cost = lin_units * unit_cost(jobs[li]);
        if (target <= cost_before + lin_cost) break;
        cost_before += lin_cost;
        ++li;
      }
      int u;
      if (li >= n_jobs) {
        u = units;
      } else {
        const int64_t w = unit_cost(jobs[li]);
        u = gp.lin[li].unit_begin + static_cast<int>((target - cost_before + w - 1) / w);
      }
      if (c == 0) u = 0;
      if (c == grid) u = units;
      gp.cta_begin[c] = u;
      if (c > 0 && c < grid && u < units && li < n_jobs) {
        const LinDesc& L = gp.lin[li];
        const int local = u - L.unit_begin;
        if (local % L.n_kc != 0) {
          const int rb = local / L.n_kc;
          if (n_zero == 0 || pp.zero[n_zero - 1].y != L.y || pp.zero[n_zero - 1].rb != rb)
            pp.zero[n_zero++] = {L.y, L.N, rb};
        }
      }
    }
  }

  // Prep launch.
  uint32_t* err = nullptr;
  if (fixed) {
    err = fixed->err;
  } else {
    e = get_error_word(&err);
    if (e != cudaSuccess) return e;
  }
  pp.M = M;
  pp.err = err;
  pp.n_layout = n_layouts;
  pp.n_sum = n_sums;
  pp.n_zero = n_zero;
  pp.rows = RU;
  for (int i = 0; i < n_layouts; ++i) {
    pp.lay[i] = {static_cast<const __nv_bfloat16*>(layouts[i].x), wsb + layouts[i].off,
                 layouts[i].K, layouts[i].kc, layouts[i].w8, layouts[i].n_kc,
                 layouts[i].b0 == 8 ? 1 : 0};
  }
  for (int i = 0; i < n_sums; ++i) {
    pp.sum[i] = {static_cast<const __nv_bfloat16*>(sum_x[i]),
                 psum_base + size_t(i) * M * kClasses, sum_k[i]};
  }
  int prep_grid = std::max(n_sums * M, sms);
  if (pp.n_ep > 0) prep_grid = 4 * sms;  // the Extra Precision gathers want many warps in flight
  prep_grid = std::min(prep_grid, 4 * sms);
  e = launch_pdl(gemv_prep_kernel<CAP>, dim3(prep_grid), dim3(256), 0, stream, pp);
  if (e != cudaSuccess) return e;

  gp.n_lin = n_jobs;
  gp.M = M;
  gp.total_units = units;
  gp.stages = stages;
  gp.stage_bytes = stage_bytes;
  gp.off_plane1 = off_plane1;
  gp.off_x = off_x;
  gp.pitch0 = P0;
  gp.pitch1 = P1;
  gp.err = err;
  gp.wait_ns = wait_limit_ns();

  switch (NT) {
    case 1: return launch_gemv<1, CAP>(gp, smem, grid, stream);
    case 2: return launch_gemv<2, CAP>(gp, smem, grid, stream);
    case 3: return launch_gemv<3, CAP>(gp, smem, grid, stream);
    default: return launch_gemv<4, CAP>(gp, smem, grid, stream);
  }
}

}  // namespace

cudaError_t run_gemv(const LinearJob* jobs, int n_jobs, int M, cudaStream_t stream) {
  if (n_jobs < 1 || n_jobs > kGemvMaxLinears || M < 1 || M > 32) return cudaErrorInvalidValue;
  if (n_jobs == 1) return run_gemv_cap<1>(jobs, n_jobs, M, stream);
  if (n_jobs <= 8) return run_gemv_cap<8>(jobs, n_jobs, M, stream);
  return run_gemv_cap<kGemvMaxLinears>(jobs, n_jobs, M, stream);
}

size_t gemv_scratch_bytes(const LinearJob& job, int M) {
  // Same arithmetic as the planner in run_gemv_cap for one linear.
  const int P0 = tiling_p0(M);
  int b0, b1;
  job_planes(job, b0, b1);
  const int kc = P0 * 8 / b0;
  const int64_t n_kc = (job.K + kc - 1) / kc;
  size_t xf = size_t(n_kc) * M * kc * 2;
  xf = (xf + 255) & ~size_t(255);
  return xf + size_t(M) * kClasses * sizeof(float) + 256;
}

cudaError_t run_gemv_fixed_n(const LinearJob* jobs, int n_jobs, int M, cudaStream_t stream,
                             const FixedScratch& scratch) {
  if (n_jobs < 1 || n_jobs > 8 || M < 1 || M > 32) return cudaErrorInvalidValue;
  if (n_jobs == 1) return run_gemv_cap<1>(jobs, 1, M, stream, &scratch);
  return run_gemv_cap<8>(jobs, n_jobs, M, stream, &scratch);
}

cudaError_t run_gemv_fixed(const LinearJob& job, int M, cudaStream_t stream,
                           const FixedScratch& scratch) {
  if (M < 1 || M > 32) return cudaErrorInvalidValue;
  return run_gemv_cap<1>(&job, 1, M, stream, &scratch);
}

}  // namespace mq
