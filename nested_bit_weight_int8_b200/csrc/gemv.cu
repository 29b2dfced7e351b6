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
// kernel zeroes exactly those shared row blocks first (a short integer launch
// without a prep kernel zeroes them itself, before a grid barrier).
//
// CTA = 8 consumer warps + 1 producer warp. The producer stages each unit in
// shared memory with one 2-D TMA box per plane (cp.async.bulk.tensor; rows
// past N and bytes past K read as zero) plus one bulk copy of the unit's
// activation block from the prep kernel's layout, or, without a prep kernel,
// the block computed from x by the producer warp itself; either signals an
// mbarrier. Up to 8 batch rows each consumer warp owns two 16-row tiles
// (128-byte plane rows in the 128-byte swizzle, 256-row units); above 8 it
// owns one tile (64-byte rows, 128-row units). It runs mma.sync m16n8k16
// (bf16 in, fp32 accumulate) with the weights as the A operand and the batch
// (n8 tiles) as B.
//
// One batch row at r = 8, 4, 2 runs on the integer tensor cores instead
// (mma.sync m16n8k32, u8 x s8 -> s32): the codes are the A operand as plain
// bytes, with no offset, so r = 8 needs no decode at all, r = 4 one shift and
// two ANDs per 8 codes, r = 2 three shifts and four ANDs per 16 codes, and one
// instruction covers 512 weights. A bf16 input is not an integer, so the prep
// kernel writes each input of a unit exactly as an integer X = x 2^sigma of up
// to 49 bits, sigma = 48 - E from the unit's largest exponent E, in seven
// signed 7-bit digits, digit g in batch column g of the MMA (columns free at
// one batch row). Accumulation is exact in int32; the epilogue weighs column
// g by 2^(7g - sigma) when it folds the unit. Inputs more than 41 octaves
// below the unit's largest (or non-finite ones, or a scale outside the fp32
// range) mark the unit for the bf16 path instead, so the product is exact for
// every input up to fp32 rounding.
//
// Exactness of the operands. A code c (0 <= c < 2^b, b <= 4) is OR-ed into
// the mantissa of a bf16 power of two 2^e at a bit position p, which yields
// exactly 2^e + c * 2^(e-7+p); choosing p and e so that the code weight is 1
// (or 4, 16 for the high plane of r = 3, 6) gives the integer value
// 2^e + weight*c, exact in bf16. One bf16x2 subtract then takes out the magic
// 2^e and, on the low plane, the centre code 2^(r-1): the MMA sums
// x (c - 2^(r-1)) with no offset, so an fp32 partial sum never carries a
// magic (up to 256 per code) that the epilogue would have to cancel again, and
// a row whose zero point sits near the middle of the codes keeps small sums.
// A byte (r = 8) has one significant bit too many for the magic; it goes
// through fp32 instead (below), with the same centring. The epilogue is
//   y = A_n acc - alpha_n (z_n - 128) Sx_m,  A_n = alpha_n 2^(8-r),
// since 2^(r-1) 2^(8-r) = 128 at every width.
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
#include <list>
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
// Header: barriers and flags from byte 0, each consumer warp's output and
// Extra Precision pointers (16 bytes a warp) from byte 256, a 64-byte zero
// block ending at byte 1024, then each consumer warp's row scales (alpha and
// z of its 32 rows, 256 bytes a warp) up to byte 3072, where the stages start.
constexpr int kHeaderBytes = 3072;
constexpr int kPtrsOff = 256;
constexpr int kScalesOff = 1024;
static_assert(kScalesOff + kConsumerWarps * 64 * 4 <= kHeaderBytes, "row scales overflow the header");
static_assert(kPtrsOff + kConsumerWarps * 16 <= kScalesOff - 64, "pointer slots overlap the zero block");
constexpr int kMaxDynSmem = 227 * 1024;
constexpr size_t kStageBudget = 108 * 1024;  // two CTAs per SM with the header and alignment slack
constexpr int kMaxCtas = 320;       // persistent grid cap (2 CTAs on each of 148 SMs fit)
constexpr int kClasses = 8;         // activation classes (k >> 1) & 7
constexpr int kFuseUnitsPerCta = 8; // integer launches up to this many units per CTA skip the prep kernel
static_assert(kMaxStages <= kConsumerWarps, "one consumer warp stages each of the first stages' blocks");

// Decode kinds of the planes at one batch row on the integer tensor cores:
// kDkI8 + r for r = 8, 4, 2. A unit is 256 rows x 128 plane bytes (1024 / r
// codes). Its staged activation block is a 64-byte header (int mode: 0 digits,
// 1 bf16 fragments; int E, the unit's largest exponent; float Sxu, the input
// sum of a bf16 unit) and then slot (s, jj, t, g) of 16 bytes at
// 64 + (((s * J / 2 + jj) * kI8Digits + g) * 4 + t) * 16, J = 16 / r MMAs per
// 16-byte chunk: digit g of the 16 inputs of MMAs 2 jj and 2 jj + 1 of chunk
// 4s + t, in their k-slot order (b0, b1 of each); lane 4g + t reads slot
// (g, t), so each 8-lane phase of the 16-byte load reads 128 contiguous bytes.
// A mode-1 unit holds the width's bf16 fragments there instead.
constexpr int kDkI8 = 20;
constexpr int kI8Digits = 7;
constexpr int kI8Header = 64;
__host__ __device__ constexpr uint32_t i8_unit_bytes(int r) {
  return kI8Header + 2u * static_cast<uint32_t>(16 / r / 2) * 4u * kI8Digits * 16u;  // 960, 1856, 3648
}
__host__ __device__ constexpr bool is_i8(int dk) { return dk == kDkI8 + 8 || dk == kDkI8 + 4 || dk == kDkI8 + 2; }

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
  // Unit row (within a 16-row tile, before + 8h) of MMA fragment row g. With
  // the 128-byte swizzle (chunk c of row w at c ^ (w % 8)) the two rows that
  // one 8-lane phase of a 16-byte load reads (g = 2p, 2p + 1) are made to
  // differ in bit 2, which puts their chunks in different bank groups.
  static __device__ __forceinline__ int frag_row(int g) { return SWZ ? (((g & 1) << 2) | (g >> 1)) : g; }
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
  const uint8_t* xf;   // activations in fragment order, n_kc blocks of M*KC bf16; in a
                       // launch without a prep kernel, the input row x itself (bf16)
  const float* psum;   // [M][8] activation sums per class (k >> 1) & 7
  int N, K, r, kc, n_kc, unit_begin;
  int dk;  // decode kind: r for planes, 10 / 11 for the container sliced by Eq. 6 / Eq. 8,
           // kDkI8 + r for the planes on the integer tensor cores
  uint32_t xunit;  // bytes of one unit's staged activation block
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
  // Launches without a prep kernel: grid-barrier words {arrivals, generation}
  // of the stream, zero between launches.
  uint32_t* sync;
  unsigned long long wait_ns;
  // 4, 16, 64: left shifts of the integer decode done as multiplies (the FMA
  // pipe) instead of shifts (the ALU pipe, its busiest); as kernel
  // parameters the compiler cannot turn them back into shifts
  uint32_t shl[3];
  int cta_begin[kMaxCtas + 1];  // unit range of CTA c: [cta_begin[c], cta_begin[c + 1])
  LinDesc lin[CAP];
};
// kernel parameters are limited to 32764 bytes
static_assert(sizeof(GemvParams<kGemvMaxLinears>) <= 32764, "decode kernel parameters too large");

// Geometry of one width: the high plane's width (b1, 0 for one plane), and
// the 8-code activation groups per 16-byte low-plane chunk (W8).
template <int R> struct Geo;
template <> struct Geo<2> { static constexpr int b1 = 0, W8 = 8; };
template <> struct Geo<4> { static constexpr int b1 = 0, W8 = 4; };
template <> struct Geo<8> { static constexpr int b1 = 0, W8 = 2; };
template <> struct Geo<3> { static constexpr int b1 = 1, W8 = 8; };
template <> struct Geo<6> { static constexpr int b1 = 2, W8 = 4; };
// The container sliced on load (Eq. 6: kind 10, Eq. 8: kind 11) streams the
// 8-bit plane.
template <> struct Geo<10> { static constexpr int b1 = 0, W8 = 2; };
template <> struct Geo<11> { static constexpr int b1 = 0, W8 = 2; };

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
  // 10, 11: the container; kDkI8 + r: planes of width r
  b0 = (r == 8 || r == 10 || r == 11 || r == kDkI8 + 8) ? 8 : (r == 4 || r == 6 || r == kDkI8 + 4) ? 4 : 2;
  b1 = (r == 3) ? 1 : (r == 6) ? 2 : 0;
}

template <int SIG>
__device__ __forceinline__ uint32_t shift_to(uint32_t w) {
  if constexpr (SIG < 0) return w << (-SIG);
  else if constexpr (SIG == 0) return w;
  else return w >> SIG;
}

// a - b on bf16x2 pairs. The decode uses it on exact small integers (a code
// under its magic, minus the magic and the centre code), where it is exact.
__device__ __forceinline__ uint32_t bsub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The centre code of a row: the code nearest to z / 2^(8-r), clamped to
// [0, cmax]. The bf16 decode subtracts it from every code of the row and the
// epilogue adds alpha c0 2^(8-r) back through the zero-point term, so the
// MMA sums x (c - c0), small wherever the dequantized weights are small.
__device__ __forceinline__ int centre_code(float z, int rw, int cmax) {
  const float zc = rintf(z * (1.0f / static_cast<float>(1 << (8 - rw))));
  return zc <= 0.f ? 0 : zc >= static_cast<float>(cmax) ? cmax : static_cast<int>(zc);
}

// What the bf16 decode subtracts from one weight row's registers: s[i] =
// bf16x2 of magic_i + c0 for the low plane's magics (at most three classes),
// f = 2^23 + c0 for bytes through fp32; c0 itself for the epilogue.
struct RowSub {
  uint32_t s[3];
  float f;
  float c0;
};

template <int R>
__device__ __forceinline__ RowSub make_rowsub(float zero, int r) {
  const int rw = (R == 10 || R == 11) ? r : R;
  const int cmax = R == 11 ? (1 << rw) : (1 << rw) - 1;
  const int c0 = centre_code(zero, rw, cmax);  // rows past N: z = 0, c0 = 0
  // the low plane's magics: r = 2 by bit position 1, 3, 5; r = 3 by 3, 5;
  // r = 4 and 6 one; the container the power of two 2^r (Eq. 6) or 2^(r+1)
  const int m0 = R == 2 ? 64 : (R == 3 || R == 4 || R == 6) ? 16 : (R == 10 ? (1 << rw) : (2 << rw));
  const int m1 = R == 2 ? 16 : 4;
  const int m2 = 4;
  auto pair = [](int v) {
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(static_cast<float>(v)));  // exact: v < 256
    return b * 0x10001u;
  };
  RowSub rs;
  rs.s[0] = pair(m0 + c0);
  rs.s[1] = pair(m1 + c0);
  rs.s[2] = pair(m2 + c0);
  rs.f = 8388608.0f + static_cast<float>(c0);
  rs.c0 = static_cast<float>(c0);
  return rs;
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
// the exponent of 2^23) minus the row's centre code c0 (subf = 2^23 + c0), as
// an exact bf16x2 pair of integers -255..255.
__device__ __forceinline__ uint32_t bytes_bf16x2(uint32_t w, uint32_t sel_lo, uint32_t sel_hi, float subf) {
  const float lo = __uint_as_float(__byte_perm(w, 0x4B000000u, sel_lo)) - subf;
  const float hi = __uint_as_float(__byte_perm(w, 0x4B000000u, sel_hi)) - subf;
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// The pair of 2-bit codes at half-word position P (0, 2, ..., 14) of a plane
// word as bf16x2 c - c0. A left shift by 1 puts positions 0-4 at bits 1, 3, 5
// of each half, right shifts by 5 and 11 do the same for 6-10 and 12-14, so a
// word costs three shifts and eight LOP3s. The code sits under the magic
// 2^(7-p) that gives it weight 1 (the bits shifted in from the other half
// fall outside the mask); one bf16x2 subtract of the magic plus the row's
// centre code c0 leaves c - c0.
template <int P>
__device__ __forceinline__ uint32_t pick2(uint32_t w, const RowSub& rs) {
  constexpr int sh = P <= 4 ? -1 : (P <= 10 ? 5 : 11);
  constexpr int p = P - sh;
  constexpr uint32_t mask = 0x00030003u << p;
  return bsub(and_or(shift_to<sh>(w), mask, p == 1 ? kMag64 : p == 3 ? kMag16 : kMag4),
              rs.s[p == 1 ? 0 : p == 3 ? 1 : 2]);
}

// Decoded A registers of one MMA for one weight row: x0 fills k-slots
// {2t, 2t+1}, x1 fills {2t+8, 2t+9}. PLANE 0 is the low plane, 1 the high
// plane; Q is the 8-code group of the chunk, HF the 4-code half of it. Every
// register holds exact integers with no offset: plane 0 its code minus the
// row's centre code c0, plane 1 its weighted code, so the MMA sums x (c - c0)
// and never carries the magics through fp32.
template <int R, int PLANE, int Q, int HF>
__device__ __forceinline__ void decode_quad(const uint32_t (&lo)[4], const uint32_t (&hi)[2],
                                            const Cdec& cd, const RowSub& rs, uint32_t& x0, uint32_t& x1) {
  if constexpr (R == 10 || R == 11) {
    // container bytes c0..c3 of one word, registers pair (c0, c2) and (c1, c3)
    // as the r = 8 plane does; q + h never leaves its 16-bit half
    const uint32_t w = lo[2 * Q + HF];
    const uint32_t ev = w & 0x00FF00FFu;
    const uint32_t od = __byte_perm(w, 0u, 0x4341);
    if constexpr (R == 10) {
      x0 = bsub(and_or(__viaddmin_u16x2(ev, cd.h2, 0x00FF00FFu) >> 1, cd.kmask, cd.mag), rs.s[0]);
      x1 = bsub(and_or(__viaddmin_u16x2(od, cd.h2, 0x00FF00FFu) >> 1, cd.kmask, cd.mag), rs.s[0]);
    } else {
      x0 = bsub(and_or((ev + cd.h2) >> 2, cd.kmask, cd.mag), rs.s[0]);
      x1 = bsub(and_or((od + cd.h2) >> 2, cd.kmask, cd.mag), rs.s[0]);
    }
  } else if constexpr (R == 2) {
    // 2-bit codes, word = 16 codes; x0 holds codes 4j, 4j+1 (half-word
    // position 4j), x1 codes 4j+2, 4j+3 (position 4j+2), j = 2(Q%2)+HF.
    constexpr int j = 2 * (Q % 2) + HF;
    x0 = pick2<4 * j>(lo[Q / 2], rs);
    x1 = pick2<4 * j + 2>(lo[Q / 2], rs);
  } else if constexpr (R == 3 && PLANE == 0) {
    // 2-bit codes, word = 16 codes; pairs 2j, 2j+1 (j = 2(Q%2)+HF) at half-bits
    // 4j, 4j+2 -> bits 3-4 (16 + c) and bits 5-6 (4 + c) after one shift.
    constexpr int j = 2 * (Q % 2) + HF;
    const uint32_t sh = shift_to<4 * j - 3>(lo[Q / 2]);
    x0 = bsub(and_or(sh, kMaskP3b2, kMag16), rs.s[0]);
    x1 = bsub(and_or(sh, kMaskP5b2, kMag4), rs.s[1]);
  } else if constexpr (R == 4 || (R == 6 && PLANE == 0)) {
    // 4-bit codes, word = 8 codes; pairs 2HF, 2HF+1 at half-bits 8HF, 8HF+4 -> bits 3-6 (16 + c)
    const uint32_t w = lo[Q];
    x0 = bsub(and_or(shift_to<8 * HF - 3>(w), kMaskP3b4, kMag16), rs.s[0]);
    x1 = bsub(and_or(shift_to<8 * HF + 1>(w), kMaskP3b4, kMag16), rs.s[0]);
  } else if constexpr (R == 8) {
    // bytes c0..c3 of one word; registers pair (c0, c2) and (c1, c3). A byte
    // has 8 significant bits, one more than a bf16 mantissa holds under a
    // magic exponent, so it goes through fp32: 2^23 + c minus 2^23 + c0 is
    // c - c0, and its conversion to bf16 is exact.
    const uint32_t w = lo[2 * Q + HF];
    x0 = bytes_bf16x2(w, 0x7440u, 0x7442u, rs.f);
    x1 = bytes_bf16x2(w, 0x7441u, 0x7443u, rs.f);
  } else if constexpr (R == 3) {
    // high 1-bit plane (weight 4), word = 32 codes; pairs P = 4(Q%4)+2HF, +1 at
    // half-bit P; one shift puts the group's 4 pairs at bits 3..6 (64/32/16/8 + 4h)
    const uint32_t sh = shift_to<4 * (Q % 4) - 3>(hi[Q / 4]);
    constexpr int p0 = 3 + 2 * HF;
    constexpr uint32_t m0 = (1u << p0) | (1u << (16 + p0));
    constexpr uint32_t m1 = (1u << (p0 + 1)) | (1u << (17 + p0));
    x0 = bsub(and_or(sh, m0, HF == 0 ? kMag64 : kMag16), HF == 0 ? kMag64 : kMag16);
    x1 = bsub(and_or(sh, m1, HF == 0 ? kMag32 : kMag8), HF == 0 ? kMag32 : kMag8);
  } else {  // R == 6, high 2-bit plane (weight 16), word = 16 codes
    constexpr int j = 2 * (Q % 2) + HF;
    const uint32_t sh = shift_to<4 * j - 3>(hi[Q / 2]);
    x0 = bsub(and_or(sh, kMaskP3b2, kMag256), kMag256);
    x1 = bsub(and_or(sh, kMaskP5b2, kMag64), kMag64);
  }
}

// All MMAs of one 8-code activation group: for each 4-code half and each
// plane, one m16n8k16 per batch tile, the B registers shared by the planes.
template <int R, int NT, int TW, int Q>
__device__ __forceinline__ void group_mmas(const uint32_t (&lo)[TW][2][4], const uint32_t (&hi)[TW][2][2],
                                           const uint32_t (&xaddr)[NT], const uint32_t (&xstep)[NT],
                                           int gbase, const Cdec& cd, const RowSub (&rs)[TW][2],
                                           uint32_t* errp, float (&ch)[TW][NT][2][4]) {
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
        if (hf == 0 && pl == 0) { decode_quad<R, 0, Q, 0>(lo[T][0], hi[T][0], cd, rs[T][0], a0, a2); decode_quad<R, 0, Q, 0>(lo[T][1], hi[T][1], cd, rs[T][1], a1, a3); }
        if (hf == 0 && pl == 1) { decode_quad<R, 1, Q, 0>(lo[T][0], hi[T][0], cd, rs[T][0], a0, a2); decode_quad<R, 1, Q, 0>(lo[T][1], hi[T][1], cd, rs[T][1], a1, a3); }
        if (hf == 1 && pl == 0) { decode_quad<R, 0, Q, 1>(lo[T][0], hi[T][0], cd, rs[T][0], a0, a2); decode_quad<R, 0, Q, 1>(lo[T][1], hi[T][1], cd, rs[T][1], a1, a3); }
        if (hf == 1 && pl == 1) { decode_quad<R, 1, Q, 1>(lo[T][0], hi[T][0], cd, rs[T][0], a0, a2); decode_quad<R, 1, Q, 1>(lo[T][1], hi[T][1], cd, rs[T][1], a1, a3); }
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
                                           int gbase, const Cdec& cd, const RowSub (&rs)[TW][2],
                                           uint32_t* errp, float (&ch)[TW][NT][2][4],
                                           std::integer_sequence<int, Qs...>) {
  (group_mmas<R, NT, TW, Qs>(lo, hi, xaddr, xstep, gbase, cd, rs, errp, ch), ...);
}

// One staged unit for this warp's 16-row tiles, sub-step by sub-step.
// Sub-steps past the unit's valid codes read zero-filled planes and zero
// activations and add nothing. Activation
// group q of chunk 4s+t for batch row m sits at ((((s*W8 + q)*M + m)*4 + t)
// * 16) bytes of the staged block; lanes whose batch row is past M read a
// zero block instead (step 0). With 128-byte plane rows the box is stored in
// 128-byte swizzled atoms: chunk c of row r at chunk c ^ (r % 8).
template <int R, int NT>
__device__ __forceinline__ void process_unit(const uint8_t* st0, const uint8_t* st1,
                                             const uint32_t (&xaddr)[NT],
                                             const uint32_t (&xstep)[NT], int warp, int lane,
                                             const Cdec& cd, const RowSub (&rs)[Tiling<NT>::TW][2],
                                             uint32_t* errp, float (&ch)[Tiling<NT>::TW][NT][2][4]) {
  using G = Geo<R>;
  using TL = Tiling<NT>;
  constexpr int TW = TL::TW, NSUB = TL::NSUB, P0 = TL::P0, P1 = TL::P0 / 2;
  const int g = lane >> 2, t = lane & 3;
  // one sub-step's planes at a time (the row subtrahends take the registers
  // a whole unit's words would)
#pragma unroll
  for (int s = 0; s < NSUB; ++s) {
    uint32_t lo[TW][2][4];
    uint32_t hi[TW][2][2];
    const int ci = 4 * s + t;  // this thread's 16-byte chunk of the low plane
#pragma unroll
    for (int T = 0; T < TW; ++T) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = warp * TL::RPW + 16 * T + TL::frag_row(g) + 8 * h;
        const int cs = TL::SWZ ? (ci ^ (row & 7)) : ci;
        const uint4 v = *reinterpret_cast<const uint4*>(st0 + row * P0 + cs * 16);
        lo[T][h][0] = v.x; lo[T][h][1] = v.y; lo[T][h][2] = v.z; lo[T][h][3] = v.w;
        if constexpr (G::b1 != 0) {
          const uint2 u = *reinterpret_cast<const uint2*>(st1 + row * P1 + ci * 8);
          hi[T][h][0] = u.x; hi[T][h][1] = u.y;
        } else {
          hi[T][h][0] = 0; hi[T][h][1] = 0;
        }
      }
    }
    chunk_mmas<R, NT, TW>(lo, hi, xaddr, xstep, s * G::W8, cd, rs, errp, ch,
                          std::make_integer_sequence<int, G::W8>{});
  }
}

// The current linear of a CTA's walk over its unit range, cached in registers.
struct Cursor {
  int l, rb, kc;          // linear, row block, k-chunk of the current unit
  int nrb, n_kc, r, N;    // of linear l
  int dk;                 // its decode kind (width, 10 / 11 for the container, or kDkI8 + r)
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

// Copies alpha and z of this warp's rows of row block rb of linear l into
// its shared slots sc[0..31] (alpha) and sc[32..63] (z), asynchronously
// (cp.async, waited for before their first use); rows past N read as zero.
// The scales do not change during a launch, so the first copy is issued
// before the wait for the previous grid.
//
// Lane 0 also keeps the linear's y and Extra Precision pointers in the
// warp's slot `ptrs`: read here, at the start of the row block, their load
// from the kernel parameters (a cold line on every call) is off the flush's
// path.
template <int NT, int CAP>
__device__ __forceinline__ void stage_scales(const GemvParams<CAP>& p, int l, int rb, int warp, int lane,
                                             float* sc, const void** ptrs) {
  const LinDesc& L = p.lin[l];
  const int n = rb * Tiling<NT>::RPU + warp * Tiling<NT>::RPW + lane;
  const bool in = lane < Tiling<NT>::RPW && n < L.N;
  cp_async_4(sc + lane, in ? L.alpha + n : L.alpha, in ? 4u : 0u);
  cp_async_4(sc + 32 + lane, in ? L.zero + n : L.zero, in ? 4u : 0u);
  cp_async_commit();
  if (lane == 0) {
    ptrs[0] = L.y;
    ptrs[1] = L.epc;
  }
}

// Epilogue of one row block of this warp's 16 rows: scales the raw sums,
// removes the zero point and writes y. The bf16 decode sums x (c - c0), so
// its zero point is taken relative to the row's centre code:
// y = A acc - alpha (z - c0 2^(8-r)) Sx, once per row by the part that starts
// at k-chunk 0 (Sx from the class sums). The integer kinds sum x c and each
// part removes its own share, y = A acc - alpha z sxs, with sxs the input sum
// of the part's units. A row block this CTA owns whole is stored; a shared one
// is added atomically into y, zeroed first (by the prep kernel, or inside a
// launch without one).
//
// Everything it reads is at hand (the cursor's N, r and kind, the staged
// scales and pointers): no kernel-parameter load on the flush's path.
template <int NT, int CAP>
__device__ void flush_rows(const GemvParams<CAP>& p, int l, int rb, int kc0, bool whole, int warp,
                           int lane, const float (&tot)[Tiling<NT>::TW][NT][4], float sxs, const float* sc,
                           const void* const* ptrs, int N, int r, int dk, int M) {
  constexpr int TW = Tiling<NT>::TW;
  float* const y = static_cast<float*>(const_cast<void*>(ptrs[0]));  // L.y, staged
  const float* const epc = static_cast<const float*>(ptrs[1]);       // L.epc, staged
  const int g = lane >> 2, t = lane & 3;
  const float scale = static_cast<float>(1 << (8 - r));
  const int cmax = dk == 11 ? (1 << r) : (1 << r) - 1;
  // the row scales, staged in shared memory (stage_scales)
  float av[TW][2], zv[TW][2];
#pragma unroll
  for (int T = 0; T < TW; ++T)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 16 * T + Tiling<NT>::frag_row(g) + 8 * h;
      av[T][h] = sc[i];
      zv[T][h] = sc[32 + i];
    }
#pragma unroll
  for (int T = 0; T < TW; ++T) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = rb * Tiling<NT>::RPU + warp * Tiling<NT>::RPW + 16 * T + Tiling<NT>::frag_row(g) + 8 * h;
      if (n >= N) continue;
      const float a = av[T][h], z = zv[T][h];
      // the same centre code the decode subtracted (make_rowsub)
      const float c0 = is_i8(dk) ? 0.f : static_cast<float>(centre_code(z, r, cmax));
      const float A = a * scale, B = a * (z - c0 * scale);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int m = nt * 8 + 2 * t + e;
          if (m >= M) continue;
          float v = tot[T][nt][2 * h + e];
          if (is_i8(dk)) {
            if (kc0 == 0 && epc) v += epc[static_cast<int64_t>(m) * N + n];
            v = A * v - B * sxs;
          } else if (kc0 == 0) {
            // Extra Precision: each listed position adds one code step
            if (epc) v += epc[static_cast<int64_t>(m) * N + n];
            const float* P = p.lin[l].psum + m * kClasses;
            float Sx = 0.f;
#pragma unroll
            for (int i = 0; i < kClasses; ++i) Sx += P[i];
            v = A * v - B * Sx;
          } else {
            v = A * v;
          }
          float* dst = y + static_cast<int64_t>(m) * N + n;
          if (whole) *dst = v;
          else atomicAdd(dst, v);
        }
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
                                            const Cdec& cd, int l, int rb,
                                            float (&tot)[Tiling<NT>::TW][NT][4], const float* sc) {
  constexpr int TW = Tiling<NT>::TW;
  // the centre codes of this thread's rows (rows g and g + 8 of each tile),
  // from the row scales staged in shared memory
  RowSub rs[TW][2];
  {
    const LinDesc& L = p.lin[l];
    const int g = lane >> 2;
    cp_async_wait_all();
    __syncwarp();
#pragma unroll
    for (int T = 0; T < TW; ++T)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        rs[T][h] = make_rowsub<R>(sc[32 + 16 * T + Tiling<NT>::frag_row(g) + 8 * h], L.r);
  }
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
      process_unit<R, NT>(st, st + Tiling<NT>::RPU * Tiling<NT>::P0, xa, xstep, warp, lane, cd, rs, p.err, ch);
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

// The A registers of MMA j of a 16-byte chunk for one weight row (words
// w[0..3] of the chunk) on the integer path: codes as bytes, in k-slot order
// k 4t + i (a0) and 16 + 4t + i (a2), each code in the top bits of its byte
// (a power-of-two multiple, taken out when the unit is folded).
//  r = 8: the bytes themselves; a0 = word 2j, a2 = word 2j + 1.
//  r = 4: word j holds codes u at bit 16 (u % 2) + 4 (u / 2);
//         (w << 4) & 0xF0F0F0F0 gives 16 x codes 0, 4, 1, 5 and
//         w & 0xF0F0F0F0 16 x codes 2, 6, 3, 7.
//  r = 2: word j / 2 holds 16 codes at bit 16 (u % 2) + 2 (u / 2);
//         (w << (6 - 2i)) & 0xC0C0C0C0 gives 64 x codes 2i, 2i + 8, 2i + 1,
//         2i + 9, and MMA j takes i = 2 (j % 2) (a0) and i = 2 (j % 2) + 1 (a2).
// The left shifts are multiplies by the kernel parameters shl = {4, 16, 64}.
template <int R, int J>
__device__ __forceinline__ void i8_regs(const uint32_t (&w)[4], const uint32_t (&shl)[3], uint32_t& a0,
                                        uint32_t& a2) {
  if constexpr (R == 8) {
    a0 = w[2 * J];
    a2 = w[2 * J + 1];
  } else if constexpr (R == 4) {
    a0 = (w[J] * shl[1]) & 0xF0F0F0F0u;
    a2 = w[J] & 0xF0F0F0F0u;
  } else if constexpr (J % 2 == 0) {
    a0 = (w[J / 2] * shl[2]) & 0xC0C0C0C0u;  // i = 0: << 6
    a2 = (w[J / 2] * shl[1]) & 0xC0C0C0C0u;  // i = 1: << 4
  } else {
    a0 = (w[J / 2] * shl[0]) & 0xC0C0C0C0u;  // i = 2: << 2
    a2 = w[J / 2] & 0xC0C0C0C0u;             // i = 3
  }
}
// log2 of the code multiple that i8_regs leaves at each width
template <int R> constexpr int kI8CodeShift = R == 8 ? 0 : R == 4 ? 4 : 6;

// One staged unit at width R on the integer path (one batch row, Tiling<1>):
// the planes are loaded as for the bf16 path (128-byte swizzle); per chunk
// J = 16 / R MMAs of 16 rows x 32 k, the digits of MMAs 2jj, 2jj + 1 in one
// 16-byte load at xaddr + (s * J / 2 + jj) * xstep. MMA j accumulates into
// chain j % 2.
template <int R, int... Js>
__device__ __forceinline__ void i8_chunk(const uint32_t (&lo)[2][2][4], const uint32_t (&shl)[3],
                                         const uint8_t* smem_base, uint32_t xaddr, uint32_t xstep, int s,
                                         uint32_t* errp, int (&ch)[2][2][4], std::integer_sequence<int, Js...>) {
  // the chunk's digit loads first, then its MMAs
  uint4 xbs[16 / R / 2];
#pragma unroll
  for (int jj = 0; jj < 16 / R / 2; ++jj) {
    const uint32_t a = xaddr + static_cast<uint32_t>(s * (16 / R / 2) + jj) * xstep;
    xbs[jj] = make_uint4(0u, 0u, 0u, 0u);
    if (MQ_IN_BOUNDS(a + 16u <= dynamic_smem_bytes(), errp)) xbs[jj] = *reinterpret_cast<const uint4*>(smem_base + a);
  }
  auto mma_j = [&](auto jc) {
    constexpr int J = decltype(jc)::value;
    const uint4& xb = xbs[J / 2];
#pragma unroll
    for (int T = 0; T < 2; ++T) {
      uint32_t a0, a1, a2, a3;
      i8_regs<R, J>(lo[T][0], shl, a0, a2);
      i8_regs<R, J>(lo[T][1], shl, a1, a3);
      mma_u8s8_16832(ch[T][J % 2], a0, a1, a2, a3, (J % 2) ? xb.z : xb.x, (J % 2) ? xb.w : xb.y);
    }
  };
  (mma_j(std::integral_constant<int, Js>{}), ...);
}

template <int R>
__device__ __forceinline__ void process_unit_i8(const uint8_t* st0, uint32_t xaddr, uint32_t xstep,
                                                int warp, int lane, const uint32_t (&shl)[3], uint32_t* errp,
                                                int (&ch)[2][2][4]) {
  using TL = Tiling<1>;
  constexpr int TW = TL::TW, NSUB = TL::NSUB, P0 = TL::P0;
  const int g = lane >> 2, t = lane & 3;
  uint32_t lo[NSUB][TW][2][4];
#pragma unroll
  for (int s = 0; s < NSUB; ++s) {
    const int ci = 4 * s + t;
#pragma unroll
    for (int T = 0; T < TW; ++T) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = warp * TL::RPW + 16 * T + TL::frag_row(g) + 8 * h;
        const int cs = ci ^ (row & 7);  // 128-byte swizzle
        const uint4 v = *reinterpret_cast<const uint4*>(st0 + row * P0 + cs * 16);
        lo[s][T][h][0] = v.x; lo[s][T][h][1] = v.y; lo[s][T][h][2] = v.z; lo[s][T][h][3] = v.w;
      }
    }
  }
  extern __shared__ __align__(128) uint8_t smem[];
#pragma unroll
  for (int s = 0; s < NSUB; ++s)
    i8_chunk<R>(lo[s], shl, smem, xaddr, xstep, s, errp, ch, std::make_integer_sequence<int, 16 / R>{});
}

// run_segment for the integer kinds (one batch row). Each unit's header says
// whether its activation block holds digits (mode 0) or, for inputs that the
// digits cannot hold exactly, the bf16 fragments of the width's bf16 path
// (mode 1), and gives the unit's input sum Sxu, which adds into sxs for the
// zero-point term. Thread (g, t) of a digit unit holds the int32 sums of
// columns 2t and 2t + 1, digits 2t and 2t + 1 (column 7 is zero): it weighs
// them by 2^(7 digit - sigma), sigma = 48 - E. A bf16 unit sums x (c - c0)
// per row; thread t = 0 adds c0 Sxu back. The partials stay in tot[T][0][0]
// (row g) and tot[T][0][2] (row g + 8) until the row block is flushed.
template <int R, int CAP>
__device__ __forceinline__ bool run_segment_i8(const GemvParams<CAP>& p, const uint8_t* stages,
                                               uint64_t* full, uint64_t* empty, volatile int* s_abort,
                                               int seg, int& s, uint32_t& ph, bool active,
                                               uint32_t zero_addr, int warp, int lane, int l, int rb,
                                               float (&tot)[2][1][4], float& sxs, const float* sc) {
  const int g = lane >> 2, t = lane & 3;
  for (int i = 0; i < seg; ++i) {
    if (*s_abort || !mbar_wait_bounded(&full[s], ph, p.wait_ns)) {
      if (lane == 0) { atomicOr(p.err, kErrWaitFull); *s_abort = 1; }
      return false;
    }
    if (active) {
      const uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
      extern __shared__ __align__(128) uint8_t smem[];
      const uint8_t* hdr = st + p.off_x;
      const uint32_t xs = static_cast<uint32_t>(hdr - smem) + kI8Header;  // data, shared offset
      const int mode = reinterpret_cast<const int*>(hdr)[0];
      sxs += reinterpret_cast<const float*>(hdr)[2];
      if (mode == 0) {
        const int E = reinterpret_cast<const int*>(hdr)[1];
        int ch[2][2][4];
#pragma unroll
        for (int T = 0; T < 2; ++T)
#pragma unroll
          for (int j = 0; j < 4; ++j) { ch[T][0][j] = 0; ch[T][1][j] = 0; }
        const bool live = g < kI8Digits;
        process_unit_i8<R>(st, live ? xs + static_cast<uint32_t>(g * 4 + t) * 16u : zero_addr,
                           live ? 4u * kI8Digits * 16u : 0u, warp, lane, p.shl, p.err, ch);
        // digit 2t weighs 2^(14t + E - 48), digit 2t + 1 2^(14t + 7 + E - 48);
        // the codes came 2^kI8CodeShift times their value
        const float w0 = __int_as_float((127 + 14 * t + E - 48 - kI8CodeShift<R>) << 23);
        const float w1 = __int_as_float((127 + 14 * t + 7 + E - 48 - kI8CodeShift<R>) << 23);
#pragma unroll
        for (int T = 0; T < 2; ++T) {
          tot[T][0][0] = fmaf(static_cast<float>(ch[T][0][0] + ch[T][1][0]), w0,
                              fmaf(static_cast<float>(ch[T][0][1] + ch[T][1][1]), w1, tot[T][0][0]));
          tot[T][0][2] = fmaf(static_cast<float>(ch[T][0][2] + ch[T][1][2]), w0,
                              fmaf(static_cast<float>(ch[T][0][3] + ch[T][1][3]), w1, tot[T][0][2]));
        }
      } else {
        // bf16 fragments of batch row 0 (lanes g = 0), the width's bf16 decode,
        // which sums x (c - c0): thread t = 0 adds c0 Sxu back (Sxu = the
        // unit's input sum from the header)
        const float Sxu = t == 0 ? reinterpret_cast<const float*>(hdr)[2] : 0.f;
        float ch[2][1][2][4];
#pragma unroll
        for (int T = 0; T < 2; ++T)
#pragma unroll
          for (int j = 0; j < 4; ++j) { ch[T][0][0][j] = 0.f; ch[T][0][1][j] = 0.f; }
        const uint32_t xa[1] = {g == 0 ? xs + static_cast<uint32_t>(t) * 16u : zero_addr};
        const uint32_t xstep[1] = {g == 0 ? 64u : 0u};
        // the centre codes of this thread's rows, made here (a rare path)
        // rather than held in registers across the unit loop
        RowSub rs[2][2];
        const LinDesc& L = p.lin[l];
        cp_async_wait_all();
        __syncwarp();
#pragma unroll
        for (int T = 0; T < 2; ++T)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            rs[T][h] = make_rowsub<R>(sc[32 + 16 * T + Tiling<1>::frag_row(g) + 8 * h], L.r);
        process_unit<R, 1>(st, st + Tiling<1>::RPU * Tiling<1>::P0, xa, xstep, warp, lane, Cdec{0u, 0u, 0u},
                           rs, p.err, ch);
#pragma unroll
        for (int T = 0; T < 2; ++T) {
          tot[T][0][0] += fmaf(rs[T][0].c0, Sxu, ch[T][0][0][0] + ch[T][0][1][0]);
          tot[T][0][2] += fmaf(rs[T][1].c0, Sxu, ch[T][0][0][2] + ch[T][0][1][2]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == p.stages) { s = 0; ph ^= 1u; }
  }
  return true;
}

// Stages the activation block of one integer-kind unit (one batch row,
// inputs kc KC .. kc KC + KC - 1 of the row xr, KC = 1024 / R) in shared
// memory at blk, in the layout the prep kernel writes to global memory: the
// header (mode, E, Sxu) and either the seven digit slots or, for inputs the
// digits cannot hold exactly, the width's bf16 fragments. Run by one whole
// warp. Used by launches without a prep kernel: the producer warp stages each
// unit while the unit's weight box is in flight.
template <int R>
__device__ __forceinline__ void stage_i8_unit(const uint16_t* __restrict__ xr, int K, int kc, uint8_t* blk,
                                              int lane) {
  constexpr int KC = 1024 / R, EPT = KC / 32, CPC = 128 / R, J2 = 16 / R / 2;
  constexpr int kNone = -100000;
  const int kbase = kc * KC;
  // (a) the unit's largest exponent E, smallest exponent f, non-finite
  // inputs and input sum: lane l holds inputs kbase + EPT l .. + EPT - 1
  // (all inside K or all past it: K % 32 at r = 8, 4 and K % 64 at r = 2)
  uint32_t xe[EPT / 2];
#pragma unroll
  for (int i = 0; i < EPT / 2; ++i) xe[i] = 0u;
  const int k0 = kbase + lane * EPT;
  if (k0 < K) {
    if constexpr (EPT == 16) {
      const uint4 va = *reinterpret_cast<const uint4*>(xr + k0);
      const uint4 vb = *reinterpret_cast<const uint4*>(xr + k0 + 8);
      xe[0] = va.x; xe[1] = va.y; xe[2] = va.z; xe[3] = va.w;
      xe[4] = vb.x; xe[5] = vb.y; xe[6] = vb.z; xe[7] = vb.w;
    } else if constexpr (EPT == 8) {
      const uint4 va = *reinterpret_cast<const uint4*>(xr + k0);
      xe[0] = va.x; xe[1] = va.y; xe[2] = va.z; xe[3] = va.w;
    } else {
      const uint2 va = *reinterpret_cast<const uint2*>(xr + k0);
      xe[0] = va.x; xe[1] = va.y;
    }
  }
  // (b)'s inputs too, before anything waits on (a): slot group (s, jj, t)
  // of 16 inputs (MMAs 2 jj, 2 jj + 1 of chunk 4s + t) goes to 4 / J2 lanes,
  // each writing every (4 / J2)-th digit g
  constexpr int LPG = 4 / J2;
  const int grp = lane / LPG, sub = lane % LPG;
  const int s = grp / (4 * J2), jj = (grp / 4) % J2, t = grp % 4;
  const int k16 = kbase + (4 * s + t) * CPC + 16 * jj;
  uint32_t xw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  if (k16 < K) {
    const uint4 va = *reinterpret_cast<const uint4*>(xr + k16);
    const uint4 vb = *reinterpret_cast<const uint4*>(xr + k16 + 8);
    xw[0] = va.x; xw[1] = va.y; xw[2] = va.z; xw[3] = va.w;
    xw[4] = vb.x; xw[5] = vb.y; xw[6] = vb.z; xw[7] = vb.w;
  }
  int emax = kNone, fmin = 1 << 30;
  bool bad = false;
  float xsum = 0.f;
#pragma unroll
  for (int u = 0; u < EPT; ++u) {
    const uint32_t bits = (u & 1) ? (xe[u >> 1] >> 16) : (xe[u >> 1] & 0xFFFFu);
    const uint32_t ef = (bits >> 7) & 0xFFu, mf = bits & 0x7Fu;
    if (ef == 0xFFu) bad = true;
    xsum += __uint_as_float(bits << 16);
    if (ef == 0u && mf == 0u) continue;
    const uint32_t m = ef ? (0x80u | mf) : mf;
    const int f = static_cast<int>(ef ? ef : 1u) - 134;
    emax = max(emax, f + 31 - __clz(static_cast<int>(m)));
    fmin = min(fmin, f);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
    fmin = min(fmin, __shfl_xor_sync(0xffffffffu, fmin, o));
    xsum += __shfl_xor_sync(0xffffffffu, xsum, o);
  }
  const int E = emax == kNone ? 0 : emax;
  if (emax != kNone && (fmin < E - 48 || E > 100 || E < -72)) bad = true;
  const bool fallback = __any_sync(0xffffffffu, bad);
  if (!fallback) {
    // (b) X = |x| 2^(48 - E) (an integer below 2^49) of each input in k-slot
    // order b, and the signs
    uint64_t X[16];
    uint32_t neg = 0u;
#pragma unroll
    for (int b = 0; b < 16; ++b) {
      const int h = b / 8, bb = b % 8;
      // the input's index among the 16: r = 8 bytes in order; r = 4 codes
      // 0, 4, 1, 5, 2, 6, 3, 7 of word 2 jj + h; r = 2 codes 4h + (0, 8, 1,
      // 9, 2, 10, 3, 11) of word jj
      const int u = R == 8 ? 8 * h + bb
                  : R == 4 ? 8 * h + ((bb & 1) ? 4 : 0) + (bb >> 1)
                           : 4 * h + ((bb & 1) ? 8 : 0) + (bb >> 1);
      const uint32_t bits = (u & 1) ? (xw[u >> 1] >> 16) : (xw[u >> 1] & 0xFFFFu);
      const uint32_t ef = (bits >> 7) & 0xFFu, mf = bits & 0x7Fu;
      const uint32_t m = ef ? (0x80u | mf) : mf;
      const int sh = static_cast<int>(ef ? ef : 1u) - 134 + 48 - E;  // >= 0 wherever m != 0
      X[b] = m ? (static_cast<uint64_t>(m) << sh) : 0ull;
      neg |= ((bits >> 15) & 1u) << b;
    }
    for (int g = sub; g < kI8Digits; g += LPG) {
      uint32_t out[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t word = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int b = 4 * w + i;
          uint32_t d = static_cast<uint32_t>(X[b] >> (7 * g)) & 127u;
          if ((neg >> b) & 1u) d = (0u - d) & 0xFFu;
          word |= d << (8 * i);
        }
        out[w] = word;
      }
      *reinterpret_cast<uint4*>(blk + kI8Header + (((s * J2 + jj) * kI8Digits + g) * 4 + t) * 16) =
          make_uint4(out[0], out[1], out[2], out[3]);
    }
  } else {
    // (c) the width's bf16 fragments: group q of 8 inputs of chunk 4s + t at
    // ((s W8 + q) 4 + t) 16, byte planes (r = 8) pairing codes (c0, c2), (c1, c3)
    constexpr int W8 = 16 / R;
    for (int gq = lane; gq < KC / 8; gq += 32) {
      const int sq = gq / (4 * W8), tq = (gq / W8) % 4, q = gq % W8;
      const int kg = kbase + (4 * sq + tq) * CPC + 8 * q;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (kg < K) v = *reinterpret_cast<const uint4*>(xr + kg);
      if constexpr (R == 8) {
        const uint32_t a = __byte_perm(v.x, v.y, 0x5410), b = __byte_perm(v.x, v.y, 0x7632);
        const uint32_t c = __byte_perm(v.z, v.w, 0x5410), d = __byte_perm(v.z, v.w, 0x7632);
        v = make_uint4(a, b, c, d);
      }
      *reinterpret_cast<uint4*>(blk + kI8Header + ((sq * W8 + q) * 4 + tq) * 16) = v;
    }
  }
  if (lane == 0) {
    reinterpret_cast<int*>(blk)[0] = fallback ? 1 : 0;
    reinterpret_cast<int*>(blk)[1] = E;
    reinterpret_cast<float*>(blk)[2] = xsum;
  }
}

// The stream's grid barrier for launches without a prep kernel. Every CTA
// arrives once, after zeroing the shared row blocks it starts in; the last
// arrival resets the count and advances the generation. Called by one thread
// per CTA after its zeroing stores (a CTA barrier orders them before the
// fence); returns the generation the CTA arrived in.
__device__ __forceinline__ uint32_t grid_arrive(uint32_t* sync) {
  __threadfence();
  const uint32_t gen = *reinterpret_cast<volatile uint32_t*>(sync + 1);
  const uint32_t old = atomicAdd(sync, 1u);
  if (old == gridDim.x - 1) {
    atomicExch(sync, 0u);
    __threadfence();
    atomicAdd(sync + 1, 1u);
  }
  return gen;
}

// Waits (at most limit_ns) until every CTA of the grid has arrived: the
// generation moved past gen. Returns false if it gave up.
__device__ __forceinline__ bool grid_wait(const uint32_t* sync, uint32_t gen, uint64_t limit_ns) {
  const volatile uint32_t* g = reinterpret_cast<const volatile uint32_t*>(sync + 1);
  bool ok = *g != gen;
  if (!ok && limit_ns > 0) {
    const uint64_t t0 = globaltimer_ns();
    while (!(ok = (*g != gen)) && globaltimer_ns() - t0 <= limit_ns) __nanosleep(64);
  }
  __threadfence();
  return ok;
}

// I8: a launch whose linears all take the integer kinds (one batch row,
// planes of width 8, 4, 2): its instantiation holds only their code paths, so
// the registers of the bf16 decodes do not press on the integer loop.
// FUSE (with I8): a launch without a prep kernel. The producer warp stages
// each unit's activation block from x itself, the consumers zero the shared
// row blocks, and a grid barrier orders that zeroing before any atomic add.
template <int NT, int CAP, bool I8 = false, bool FUSE = false>
__global__ void __launch_bounds__(kGemvThreads, (NT <= 2 ? 2 : 1))
gemv_streamk_kernel(const __grid_constant__ GemvParams<CAP> p) {
  static_assert(!FUSE || (I8 && NT == 1), "launches without a prep kernel are integer-only, one batch row");
  using TL = Tiling<NT>;
  extern __shared__ __align__(128) uint8_t smem[];
  // 1024-byte aligned header and stages: the swizzled plane boxes need it
  const uint32_t raw = smem_u32(smem);
  uint8_t* base = smem + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base);
  uint64_t* empty = full + kMaxStages;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kMaxStages);
  volatile uint32_t* s_gen = reinterpret_cast<volatile uint32_t*>(s_abort + 1);  // grid barrier (FUSE)
  uint8_t* zero_block = base + kScalesOff - 64;  // 64 zero bytes read by lanes past M
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
  if (u0 >= u1) {
    if constexpr (FUSE) {
      // every CTA arrives at the grid barrier, after the previous grid ended
      if (threadIdx.x == 0) {
        pdl_wait_primary();
        grid_arrive(p.sync);
      }
    }
    return;
  }

  if constexpr (FUSE) {
    if (warp == kConsumerWarps) {
      // -------------------------------------------------- producer (FUSE)
      // Lane 0 requests each unit's weight box (counted in the stage's
      // transaction bytes, with no arrival); the warp then writes the unit's
      // activation block from x and lane 0 arrives, which completes the stage
      // once the box has landed. Weight boxes do not depend on the previous
      // grid, so the first stages' boxes go out before waiting for it.
      Cursor c;
      cursor_init<TL::RPU>(p, u0, c);
      Cursor pre_c = c;
      // weights are read once: first out of L2, ahead of code and small data
      const uint64_t pol = l2_policy_evict_first();
      auto issue_weights = [&](const Cursor& cc, int s) {
        uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
        const CUtensorMap* tm = p.map_table ? p.map_table + 2 * cc.l : &p.maps[2 * cc.l];
        mbar_expect_tx(&full[s], TL::RPU * p.pitch0);
        tma_load_2d_hint(st, tm, cc.kc * p.pitch0, cc.rb * TL::RPU, &full[s], pol);
      };
      auto stage_x = [&](const Cursor& cc, int s) {
        const LinDesc& L = p.lin[cc.l];
        const uint16_t* xr = reinterpret_cast<const uint16_t*>(L.xf);  // the input row itself
        uint8_t* blk = stages + static_cast<size_t>(s) * p.stage_bytes + p.off_x;
        if (cc.dk == kDkI8 + 8) stage_i8_unit<8>(xr, L.K, cc.kc, blk, lane);
        else if (cc.dk == kDkI8 + 4) stage_i8_unit<4>(xr, L.K, cc.kc, blk, lane);
        else stage_i8_unit<2>(xr, L.K, cc.kc, blk, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      };
      const int pre = min(S, u1 - u0);
      if (lane == 0)
        for (int i = 0; i < pre; ++i) { issue_weights(c, i); cursor_next<TL::RPU>(p, c); }
      // the first stages' transaction counts are set before any warp arrives
      // on their barriers: the producer stages unit 0 at once, consumer warp
      // i the block of unit i for the other first stages (the producer only
      // signals; the consumers wait). Named barriers are warp-aligned: the
      // warp reconverges after lane 0's loop first.
      __syncwarp();
      named_bar_arrive(2, kGemvThreads);
      c = pre_c;
      for (int i = 0; i < pre; ++i) cursor_next<TL::RPU>(p, c);
      pdl_wait_primary();
      {
        // the inputs of this CTA's first units, into L1 ahead of their staging
        // (after the wait: the previous grid may have written them)
        Cursor pc = pre_c;
        const int n_pf = min(u1 - u0, kFuseUnitsPerCta);
        for (int i = 0; i < n_pf; ++i) {
          const LinDesc& L = p.lin[pc.l];
          const int unit_bytes = (1024 / (pc.dk - kDkI8)) * 2;  // KC bf16 inputs
          const int64_t first = int64_t(pc.kc) * unit_bytes, end = int64_t(L.K) * 2;
          for (int off = lane * 128; off < unit_bytes && first + off < end; off += 32 * 128)
            prefetch_l1(L.xf + first + off);
          cursor_next<TL::RPU>(p, pc);
        }
      }
      stage_x(pre_c, 0);  // unit 0 (pre >= 1 in a CTA with units)
      for (int i = 0; i < pre; ++i) cursor_next<TL::RPU>(p, pre_c);
      int issued = pre;
      for (int u = u0 + pre; u < u1; ++u, ++issued) {
        const int s = issued % S;
        int st = 0;  // 0: go on, 1: the wait gave up, 2: the consumers stopped
        if (lane == 0) {
          if (!mbar_wait_bounded(&empty[s], ((issued / S) - 1) & 1, p.wait_ns)) st = 1;
          else if (*s_abort) st = 2;
        }
        st = __shfl_sync(0xffffffffu, st, 0);
        if (st != 0) {
          if (st == 1 && lane == 0) { atomicOr(p.err, kErrWaitEmpty); *s_abort = 1; }
          break;
        }
        if (lane == 0) issue_weights(c, s);
        stage_x(c, s);
        cursor_next<TL::RPU>(p, c);
      }
      // no bulk copy may be in flight when this warp exits
      if (lane == 0) {
        const int first = issued > S ? issued - S : 0;
        for (int j = first; j < issued; ++j)
          if (!mbar_wait_bounded(&full[j % S], (j / S) & 1, 1000000000ull)) atomicOr(p.err, kErrDrain);
      }
      return;
    }
  }

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
      // weights are read once: first out of L2, ahead of code and small data
      const uint64_t pol = l2_policy_evict_first();
      auto issue_weights = [&](const Cursor& cc, int s) {
        int b0, b1;
        plane_widths_dev(cc.dk, b0, b1);
        uint8_t* st = stages + static_cast<size_t>(s) * p.stage_bytes;
        const CUtensorMap* tm = p.map_table ? p.map_table + 2 * cc.l : &p.maps[2 * cc.l];
        const uint32_t box = TL::RPU * (p.pitch0 + (b1 ? p.pitch1 : 0));
        const uint32_t bytesx = p.lin[cc.l].xunit;
        // One 2-D box per plane (128 rows x the unit's bytes; rows past N and
        // bytes past K read as zero) plus the unit's activation block.
        mbar_arrive_expect_tx(&full[s], box + bytesx);
        tma_load_2d_hint(st, tm, cc.kc * p.pitch0, cc.rb * TL::RPU, &full[s], pol);
        if (b1) tma_load_2d_hint(st + p.off_plane1, tm + 1, cc.kc * p.pitch1, cc.rb * TL::RPU, &full[s], pol);
      };
      auto issue_x = [&](const Cursor& cc, int s) {
        const LinDesc& L = p.lin[cc.l];
        const uint32_t bytesx = L.xunit;
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
  // This warp's row scales slots; the first segment's copy goes out before
  // the wait for the previous grid (the scales are constant).
  float* sc = reinterpret_cast<float*>(base + kScalesOff) + warp * 64;
  const void** ptrs = reinterpret_cast<const void**>(base + kPtrsOff) + 2 * warp;
  {
    Cursor c1;
    cursor_init<TL::RPU>(p, u0, c1);
    stage_scales<NT>(p, c1.l, c1.rb, warp, lane, sc, ptrs);
  }
  // Class sums and the zeroed outputs come from the prep kernel; without one
  // (FUSE), the consumers zero the row block this CTA starts inside (the CTA
  // before adds into it too) and arrive at the grid barrier.
  pdl_wait_primary();
  bool grid_passed = !FUSE;
  if constexpr (FUSE) {
    Cursor c0c;
    cursor_init<TL::RPU>(p, u0, c0c);
    if (c0c.kc != 0) {
      const int n = c0c.rb * TL::RPU + static_cast<int>(threadIdx.x);  // one row per consumer thread
      if (n < c0c.N) p.lin[c0c.l].y[n] = 0.f;
    }
    __syncwarp();  // named barriers are warp-aligned
    named_bar_sync(1, kConsumerWarps * 32);
    if (threadIdx.x == 0) *s_gen = grid_arrive(p.sync);
    __syncwarp();
    named_bar_sync(1, kConsumerWarps * 32);
    // Consumer warp i (i >= 1) stages the activation block of the CTA's unit
    // i into stage i for the first min(stages, units) units, all at once
    // (the producer, which stages unit 0, would stage them one after
    // another), and arrives on its full barrier; the producer set the stage's
    // transaction count before the barrier below.
    named_bar_sync(2, kGemvThreads);
    if (warp >= 1 && warp < min(S, u1 - u0)) {
      Cursor cw;
      cursor_init<TL::RPU>(p, u0 + warp, cw);
      const LinDesc& L = p.lin[cw.l];
      const uint16_t* xr = reinterpret_cast<const uint16_t*>(L.xf);  // the input row itself
      uint8_t* blk = stages + static_cast<size_t>(warp) * p.stage_bytes + p.off_x;
      if (cw.dk == kDkI8 + 8) stage_i8_unit<8>(xr, L.K, cw.kc, blk, lane);
      else if (cw.dk == kDkI8 + 4) stage_i8_unit<4>(xr, L.K, cw.kc, blk, lane);
      else stage_i8_unit<2>(xr, L.K, cw.kc, blk, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[warp]);
    }
  }
  const int g = lane >> 2, t = lane & 3;
  const int M_rows = p.M;
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
  bool first_seg = true;
  for (int u = u0; u < u1;) {
    // One row block: units kc0 .. kc0 + seg - 1 of (linear c.l, row block c.rb).
    if (!first_seg) {
      // the previous copy has landed (and the flush read it) before the slots are reused
      cp_async_wait_all();
      __syncwarp();
      stage_scales<NT>(p, c.l, c.rb, warp, lane, sc, ptrs);
    }
    first_seg = false;
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
    float sxs = 0.f;  // input sum of the segment's units (integer kinds)
    const Cdec cd = make_cdec(c.dk, c.r);
    if constexpr (I8) {
      switch (c.dk) {
        case kDkI8 + 8: ok = run_segment_i8<8>(p, stages, full, empty, s_abort, seg, s, ph, active, zero_addr, warp, lane, c.l, c.rb, tot, sxs, sc); break;
        case kDkI8 + 4: ok = run_segment_i8<4>(p, stages, full, empty, s_abort, seg, s, ph, active, zero_addr, warp, lane, c.l, c.rb, tot, sxs, sc); break;
        default: ok = run_segment_i8<2>(p, stages, full, empty, s_abort, seg, s, ph, active, zero_addr, warp, lane, c.l, c.rb, tot, sxs, sc); break;
      }
    } else {
      switch (c.dk) {
        case 2: ok = run_segment<2, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, c.l, c.rb, tot, sc); break;
        case 4: ok = run_segment<4, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, c.l, c.rb, tot, sc); break;
        case 8: ok = run_segment<8, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, c.l, c.rb, tot, sc); break;
        case 3: ok = run_segment<3, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, c.l, c.rb, tot, sc); break;
        case 10: ok = run_segment<10, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, c.l, c.rb, tot, sc); break;
        case 11: ok = run_segment<11, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, c.l, c.rb, tot, sc); break;
        // the host plans the integer kinds only for one batch row
        case kDkI8 + 8:
          if constexpr (NT == 1) ok = run_segment_i8<8>(p, stages, full, empty, s_abort, seg, s, ph, active, zero_addr, warp, lane, c.l, c.rb, tot, sxs, sc);
          else ok = false;
          break;
        case kDkI8 + 4:
          if constexpr (NT == 1) ok = run_segment_i8<4>(p, stages, full, empty, s_abort, seg, s, ph, active, zero_addr, warp, lane, c.l, c.rb, tot, sxs, sc);
          else ok = false;
          break;
        case kDkI8 + 2:
          if constexpr (NT == 1) ok = run_segment_i8<2>(p, stages, full, empty, s_abort, seg, s, ph, active, zero_addr, warp, lane, c.l, c.rb, tot, sxs, sc);
          else ok = false;
          break;
        default: ok = run_segment<6, NT>(p, stages, full, empty, s_abort, seg, s, ph, active, xaddr, xstep, warp, lane, cd, c.l, c.rb, tot, sc); break;
      }
    }
    if (!ok) break;  // outputs are undefined after a give-up; the flag says so
    if (active) {
      if (is_i8(c.dk)) {
        // add up the digit partials of the quad: thread t = 0 then holds
        // batch row 0 of rows g and g + 8, as flush_rows expects
#pragma unroll
        for (int T = 0; T < TL::TW; ++T) {
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            float v = tot[T][0][j];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            tot[T][0][j] = v;
          }
        }
      }
      if (!whole && !grid_passed) {
        // the first add into a shared row block waits until every CTA has
        // zeroed its own (at most the wait limit; past it the flag is set)
        if (lane == 0 && !grid_wait(p.sync, *s_gen, p.wait_ns)) atomicOr(p.err, kErrWaitGrid);
        __syncwarp();
        grid_passed = true;
      }
      cp_async_wait_all();  // the row scales (bf16 segments waited already)
      __syncwarp();
      flush_rows<NT>(p, c.l, c.rb, kc0, whole, warp, lane, tot, sxs, sc, ptrs, c.N, c.r, c.dk, M_rows);
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
  cp_async_wait_all();  // no copy into shared memory outlives the thread
}

// ------------------------------------------------------------------ prep
struct PrepLayout {
  const __nv_bfloat16* x;
  uint8_t* xf;
  int K, kc, w8, n_kc;
  int perm02;  // byte planes pair codes (c0, c2), (c1, c3): store x0, x2, x1, x3
  int i8;      // width r of a digit layout (integer kinds, one batch row), else 0
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
  int n_i8;  // units of all digit layouts (phase 2b)
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
    // eight loads in flight per thread before any add (the row is read once,
    // from L2 or HBM, and this CTA is on the decode kernel's critical path)
    for (int kb = threadIdx.x * 8; kb < J.K; kb += blockDim.x * 64) {
      uint4 u[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k0 = kb + j * blockDim.x * 8;
        u[j] = k0 < J.K ? *reinterpret_cast<const uint4*>(row + k0) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          acc[i] += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xFFFF0000u);
      }
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
    if (L.i8) continue;  // phase (2b)
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
  // (2b) digit blocks of the integer kinds (one batch row): one warp per
  // (unit, digit g). Every warp of a unit reads all its inputs to find the
  // largest top exponent E and whether the digits hold every input exactly;
  // lane l then writes digit g of the 16 inputs of slot group l = (s, jj, t).
  // An input x = +-m 2^f (m < 256 an integer, f = e - 134 for a normal bf16 of
  // biased exponent e, -133 for a subnormal) becomes X = m 2^(f + 48 - E),
  // below 2^49, an integer when f >= E - 48; digit g is (X >> 7g) & 127 with
  // x's sign. A unit with f < E - 48 somewhere, a non-finite input or E
  // outside [-72, 100] gets the width's bf16 fragments and input sum instead
  // (written by the digit-0 warp).
  if (p.n_i8 > 0) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = stride / 32;
    constexpr int kNone = -100000;
    for (int64_t wi = tid / 32; wi < int64_t(p.n_i8) * kI8Digits; wi += warps) {
      const int g = static_cast<int>(wi % kI8Digits);
      int64_t rem = wi / kI8Digits;
      int li = 0;
      while (!p.lay[li].i8 || rem >= p.lay[li].n_kc) {
        if (p.lay[li].i8) rem -= p.lay[li].n_kc;
        ++li;
      }
      const PrepLayout& L = p.lay[li];
      const int r = L.i8, KC = L.kc, cpc = 128 / r;  // codes per unit, per 16-byte chunk
      const int kc = static_cast<int>(rem);
      const int64_t kbase = int64_t(kc) * KC;
      const uint16_t* xr = reinterpret_cast<const uint16_t*>(L.x);  // one batch row
      // (a) E, the smallest exponent f and non-finite inputs over the unit
      // (b)'s inputs are loaded with (a)'s, before anything waits on them:
      // lane < 8 J2 takes slot group (s, jj, t), the 16 inputs of MMAs
      // 2 jj, 2 jj + 1 of chunk 4s + t
      const int J2 = 16 / r / 2;
      const int s_b = lane / (4 * J2), jj_b = (lane / 4) % J2, t_b = lane % 4;
      const int64_t k16 = kbase + int64_t(4 * s_b + t_b) * cpc + 16 * jj_b;
      uint32_t xw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      if (lane < 8 * J2 && k16 < L.K) {  // the 16 inputs lie wholly inside or outside K
        const uint4 va = *reinterpret_cast<const uint4*>(xr + k16);
        const uint4 vb = *reinterpret_cast<const uint4*>(xr + k16 + 8);
        xw[0] = va.x; xw[1] = va.y; xw[2] = va.z; xw[3] = va.w;
        xw[4] = vb.x; xw[5] = vb.y; xw[6] = vb.z; xw[7] = vb.w;
      }
      int emax = kNone, fmin = 1 << 30;
      bool bad = false;
      float xsum = 0.f;  // the unit's input sum (the zero-point term)
      const int ept = KC / 32;  // 4, 8 or 16 consecutive inputs per lane (all in or all out: K % 32
                                // at r = 8 and 4, K % 64 at r = 2)
      const int64_t k0 = kbase + int64_t(lane) * ept;
      uint32_t xe[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      if (k0 < L.K) {  // all loads first
        if (ept == 16) {
          const uint4 va = *reinterpret_cast<const uint4*>(xr + k0);
          const uint4 vb = *reinterpret_cast<const uint4*>(xr + k0 + 8);
          xe[0] = va.x; xe[1] = va.y; xe[2] = va.z; xe[3] = va.w;
          xe[4] = vb.x; xe[5] = vb.y; xe[6] = vb.z; xe[7] = vb.w;
        } else if (ept == 8) {
          const uint4 va = *reinterpret_cast<const uint4*>(xr + k0);
          xe[0] = va.x; xe[1] = va.y; xe[2] = va.z; xe[3] = va.w;
        } else {
          const uint2 va = *reinterpret_cast<const uint2*>(xr + k0);
          xe[0] = va.x; xe[1] = va.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {  // zero words (past ept or past K) add nothing
        const uint32_t bits = (u & 1) ? (xe[u >> 1] >> 16) : (xe[u >> 1] & 0xFFFFu);
        const uint32_t ef = (bits >> 7) & 0xFFu, mf = bits & 0x7Fu;
        if (ef == 0xFFu) bad = true;
        xsum += __uint_as_float(bits << 16);
        if (ef == 0u && mf == 0u) continue;
        const uint32_t m = ef ? (0x80u | mf) : mf;
        const int f = static_cast<int>(ef ? ef : 1u) - 134;
        emax = max(emax, f + 31 - __clz(static_cast<int>(m)));
        fmin = min(fmin, f);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
        fmin = min(fmin, __shfl_xor_sync(0xffffffffu, fmin, o));
        xsum += __shfl_xor_sync(0xffffffffu, xsum, o);
      }
      const int E = emax == kNone ? 0 : emax;
      if (emax != kNone && (fmin < E - 48 || E > 100 || E < -72)) bad = true;
      const bool fallback = __any_sync(0xffffffffu, bad);
      uint8_t* blk = L.xf + int64_t(kc) * i8_unit_bytes(r);
      const int64_t blk_end = int64_t(L.n_kc) * i8_unit_bytes(r);  // bytes of the layout
      if (!fallback) {
        // (b) digit g of slot group (s, jj, t): MMAs j = 2 jj, 2 jj + 1 of chunk
        // 4s + t, whose 16 inputs are the chunk's codes 16 jj .. 16 jj + 15
        // (loaded above), in the k-slot order of i8_regs
        if (lane < 8 * J2) {
          const int s = s_b, jj = jj_b, t = t_b;
          uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int b = 0; b < 16; ++b) {
            const int h = b / 8, bb = b % 8;  // MMA 2 jj + h, k-slot byte bb
            // the input's index among the 16: r = 8 bytes in order; r = 4
            // codes 0, 4, 1, 5, 2, 6, 3, 7 of word 2 jj + h; r = 2 codes
            // 4h + (0, 8, 1, 9, 2, 10, 3, 11) of word jj
            const int u = r == 8 ? 8 * h + bb
                        : r == 4 ? 8 * h + ((bb & 1) ? 4 : 0) + (bb >> 1)
                                 : 4 * h + ((bb & 1) ? 8 : 0) + (bb >> 1);
            const uint32_t bits = (u & 1) ? (xw[u >> 1] >> 16) : (xw[u >> 1] & 0xFFFFu);
            const uint32_t ef = (bits >> 7) & 0xFFu, mf = bits & 0x7Fu;
            const uint32_t m = ef ? (0x80u | mf) : mf;
            const int sh = static_cast<int>(ef ? ef : 1u) - 134 + 48 - E - 7 * g;  // X >> 7g = m 2^sh
            // m < 2^8: digit g = (m 2^sh) & 127 for sh in (-8, 7), else 0
            uint32_t d = 0u;
            if (sh >= 0) d = sh < 7 ? ((m << sh) & 127u) : 0u;
            else d = sh > -8 ? ((m >> -sh) & 127u) : 0u;
            const uint32_t sd = (bits & 0x8000u) ? (0u - d) & 0xFFu : d;
            out[b >> 2] |= sd << (8 * (b & 3));
          }
          const int64_t off = kI8Header + (int64_t((s * J2 + jj) * kI8Digits + g) * 4 + t) * 16;
          if (MQ_IN_BOUNDS(int64_t(kc) * i8_unit_bytes(r) + off + 16 <= blk_end, p.err))
            *reinterpret_cast<uint4*>(blk + off) = make_uint4(out[0], out[1], out[2], out[3]);
        }
        if (g == 0 && lane == 0) {
          reinterpret_cast<int*>(blk)[0] = 0;
          reinterpret_cast<int*>(blk)[1] = E;
          reinterpret_cast<float*>(blk)[2] = xsum;
        }
      } else if (g == 0) {
        // (c) the width's bf16 fragments: group q of 8 inputs of chunk 4s + t at
        // ((s W8 + q) 4 + t) 16, byte planes (r = 8) pairing codes (c0, c2), (c1, c3)
        const int W8 = 16 / r;
        float part = 0.f;
        for (int grp = lane; grp < KC / 8; grp += 32) {
          const int s = grp / (4 * W8), t = (grp / W8) % 4, q = grp % W8;
          const int64_t kg = kbase + int64_t(4 * s + t) * cpc + 8 * q;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (kg < L.K) v = *reinterpret_cast<const uint4*>(xr + kg);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int u = 0; u < 8; ++u)  // the unit's input sum: the fold adds c0 times it back
            part += __uint_as_float(((u & 1) ? (w4[u >> 1] >> 16) : (w4[u >> 1] & 0xFFFFu)) << 16);
          if (r == 8) {
            const uint32_t a = __byte_perm(v.x, v.y, 0x5410), b = __byte_perm(v.x, v.y, 0x7632);
            const uint32_t c = __byte_perm(v.z, v.w, 0x5410), d = __byte_perm(v.z, v.w, 0x7632);
            v = make_uint4(a, b, c, d);
          }
          const int64_t off = kI8Header + int64_t((s * W8 + q) * 4 + t) * 16;
          if (MQ_IN_BOUNDS(int64_t(kc) * i8_unit_bytes(r) + off + 16 <= blk_end, p.err))
            *reinterpret_cast<uint4*>(blk + off) = v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) {
          reinterpret_cast<int*>(blk)[0] = 1;
          reinterpret_cast<int*>(blk)[1] = E;
          reinterpret_cast<float*>(blk)[2] = part;
        }
      }
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
template <int NT, int CAP, bool I8 = false, bool FUSE = false>
cudaError_t gemv_grid(size_t smem, int sms, int units, int* grid_out) {
  auto kern = gemv_streamk_kernel<NT, CAP, I8, FUSE>;
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

template <int NT, int CAP, bool I8 = false, bool FUSE = false>
cudaError_t launch_gemv(const GemvParams<CAP>& gp, size_t smem, int grid, cudaStream_t stream) {
  auto kern = gemv_streamk_kernel<NT, CAP, I8, FUSE>;
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

// Device tables of tensor maps for launches with more linears than fit in
// the kernel parameters: one table per distinct (device, box width, list of
// planes address, N, K, r), uploaded on the call's stream the first time that
// list is served and reused by every later identical call.
//
// The cache is bounded: at most kMaxMapTables tables and kMaxMapBytes bytes.
// A new table evicts the least recently used ones; since an evicted table may
// still be read by a launch in flight, eviction synchronizes that table's
// device before freeing it. A table served to a call that is being captured
// into a CUDA graph is pinned (the graph holds its address) and stays until
// mq_release_workspace. A list first seen during a capture is refused: its
// upload would have to become part of the graph.
constexpr size_t kMaxMapTables = 64;
constexpr size_t kMaxMapBytes = size_t(16) << 20;

using MapKey = std::pair<int, std::vector<uint64_t>>;
struct MapTable {
  CUtensorMap* dptr;
  size_t bytes;
  bool pinned;
  std::list<const MapKey*>::iterator lru;  // position in g_map_lru (front: most recent)
};
std::map<MapKey, MapTable> g_map_tables;
std::list<const MapKey*> g_map_lru;
size_t g_map_bytes = 0;

// Frees one table after its device has finished all work. Caller holds
// g_cache_mutex.
void free_map_table(std::map<MapKey, MapTable>::iterator it) {
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != it->first.first) cudaSetDevice(it->first.first);
  cudaDeviceSynchronize();
  cudaFree(it->second.dptr);
  if (cur != it->first.first) cudaSetDevice(cur);
  g_map_bytes -= it->second.bytes;
  g_map_lru.erase(it->second.lru);
  g_map_tables.erase(it);
}

cudaError_t get_map_table(const LinearJob* jobs, int n_jobs, int P0, cudaStream_t stream,
                          const CUtensorMap** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cap);
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
  MapKey k2(dev, std::move(key));
  auto it = g_map_tables.find(k2);
  if (it != g_map_tables.end()) {
    g_map_lru.splice(g_map_lru.begin(), g_map_lru, it->second.lru);
    if (cap != cudaStreamCaptureStatusNone) it->second.pinned = true;
    *out = it->second.dptr;
    return cudaSuccess;
  }
  if (cap != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;

  const size_t bytes = size_t(n_jobs) * 2 * sizeof(CUtensorMap);
  std::vector<CUtensorMap> host(size_t(n_jobs) * 2);
  std::memset(host.data(), 0, bytes);
  for (int i = 0; i < n_jobs; ++i) {
    e = encode_plane_maps(jobs[i], P0, &host[size_t(2) * i]);
    if (e != cudaSuccess) return e;
  }
  // evict from the least recent end, passing over pinned tables
  auto victim = g_map_lru.end();
  while ((g_map_tables.size() >= kMaxMapTables || g_map_bytes + bytes > kMaxMapBytes) &&
         victim != g_map_lru.begin()) {
    --victim;
    auto vt = g_map_tables.find(**victim);
    if (vt->second.pinned) continue;
    auto next = std::next(victim);
    free_map_table(vt);
    victim = next;
  }
  CUtensorMap* dptr = nullptr;
  e = cudaMalloc(&dptr, bytes);
  if (e != cudaSuccess) return e;
  // from pageable memory: the call returns once `host` has been staged
  e = cudaMemcpyAsync(dptr, host.data(), bytes, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) {
    cudaFree(dptr);
    return e;
  }
  auto ins = g_map_tables.emplace(std::move(k2), MapTable{dptr, bytes, false, {}}).first;
  g_map_lru.push_front(&ins->first);
  ins->second.lru = g_map_lru.begin();
  g_map_bytes += bytes;
  *out = dptr;
  return cudaSuccess;
}

}  // namespace

// Frees every tensor-map table (all devices), after their devices finish.
void release_map_tables() {
  std::lock_guard<std::mutex> lk(g_cache_mutex);
  while (!g_map_tables.empty()) free_map_table(g_map_tables.begin());
}

size_t map_table_count() {
  std::lock_guard<std::mutex> lk(g_cache_mutex);
  return g_map_tables.size();
}

namespace {

// Relative cost of one unit of each width, for cutting the CTA ranges. A unit
// always holds the same plane bytes per row (two planes hold 1.5x), while the
// decode and MMA work grows with the codes in it: per-unit times of
// single-width stacks on B200 at M = 1 put r = 4 at about 1.26x and r = 2 at
// about 1.88x an r = 8 unit; r = 3 and 6 are scaled from their planes.
int64_t unit_cost(int dk) {
  switch (dk) {
    case 8: return 100;
    case 4: return 126;
    case 2: return 188;
    case 6: return 183;
    case 10: case 11: return 110;  // one 8-bit plane, one MMA per 16 codes, more decode work
    // the integer kinds, from per-unit times of single-width stacks at one
    // batch row on B200 (r = 8 streams near the HBM peak; r = 4 1.09x,
    // r = 2 1.24x its unit time)
    case kDkI8 + 8: return 100;
    case kDkI8 + 4: return 109;
    case kDkI8 + 2: return 124;
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
  struct LayoutInfo { const void* x; int b0, i8, K, kc, w8, n_kc; uint32_t xunit; size_t off; };
  LayoutInfo layouts[CAP];
  const void* sum_x[CAP];
  int sum_k[CAP];
  int n_layouts = 0, n_sums = 0;
  int lay_of[CAP], sum_of[CAP];
  bool two_planes = false;
  int units = 0;
  size_t xf_bytes = 0;
  uint32_t x_unit_max = 0;
  for (int i = 0; i < n_jobs; ++i) {
    const LinearJob& j = jobs[i];
    int b0, b1;
    job_planes(j, b0, b1);
    if (b1) two_planes = true;
    const int kc = P0 * 8 / b0;
    const int n_kc = static_cast<int>((j.K + kc - 1) / kc);
    // planes of width 8, 4, 2 at one batch row run on the integer tensor cores
    const int dk0 = decode_kind(j);
    const int i8 = (M == 1 && (dk0 == 8 || dk0 == 4 || dk0 == 2)) ? dk0 : 0;
    int si = 0;
    while (si < n_sums && sum_x[si] != j.x) ++si;
    if (si == n_sums) { sum_x[n_sums] = j.x; sum_k[n_sums] = static_cast<int>(j.K); ++n_sums; }
    sum_of[i] = si;
    int li = 0;
    while (li < n_layouts && !(layouts[li].x == j.x && layouts[li].b0 == b0 && layouts[li].i8 == i8)) ++li;
    if (li == n_layouts) {
      const uint32_t xunit = i8 ? i8_unit_bytes(i8) : static_cast<uint32_t>(M * kc * 2);
      layouts[n_layouts++] = {j.x, b0, i8, static_cast<int>(j.K), kc, (128 / b0) / 8, n_kc, xunit, xf_bytes};
      xf_bytes += size_t(n_kc) * xunit;
      xf_bytes = (xf_bytes + 255) & ~size_t(255);
      if (xunit > x_unit_max) x_unit_max = xunit;
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
    d.dk = i8 ? kDkI8 + i8 : dk0;
    d.xunit = layouts[li].xunit;
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
    cudaError_t em = get_map_table(jobs, n_jobs, P0, stream, &gp.map_table);
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
  // Stage layout: [128 rows x P0][128 rows x P1][M x KC bf16 activations].
  const int P1 = two_planes ? P0 / 2 : 0;
  const uint32_t off_plane1 = static_cast<uint32_t>(RU * P0);
  const uint32_t off_x = off_plane1 + static_cast<uint32_t>(RU * P1);
  uint32_t stage_bytes = off_x + x_unit_max;
  stage_bytes = (stage_bytes + 1023) & ~1023u;  // swizzled boxes start 1024-aligned
  int stages = static_cast<int>(kStageBudget / stage_bytes);
  stages = std::max(2, std::min(stages, kMaxStages));
  const size_t smem = 1024 /* alignment slack */ + kHeaderBytes + size_t(stages) * stage_bytes;
  const int sms = sm_count();
  bool i8_only = true;
  for (int i = 0; i < n_jobs; ++i) i8_only = i8_only && is_i8(gp.lin[i].dk);
  cudaError_t e = cudaSuccess;
  int grid = 1;
  // A short integer launch (at most kFuseUnitsPerCta units per CTA) runs
  // without the prep kernel: its producer warps stage the activation blocks
  // themselves, which takes the prep grid and its wait off the call's path.
  // Longer launches keep the prep kernel, which stages every block once.
  bool fuse = false;
  if (NT == 1 && i8_only && n_ep == 0 && (!fixed || fixed->sync)) {
    e = gemv_grid<1, CAP, true, true>(smem, sms, units, &grid);
    if (e != cudaSuccess) return e;
    fuse = int64_t(units) <= int64_t(kFuseUnitsPerCta) * grid;
  }
  if (!fuse) {
    switch (NT) {
      case 1: e = i8_only ? gemv_grid<1, CAP, true>(smem, sms, units, &grid) : gemv_grid<1, CAP>(smem, sms, units, &grid); break;
      case 2: e = gemv_grid<2, CAP>(smem, sms, units, &grid); break;
      case 3: e = gemv_grid<3, CAP>(smem, sms, units, &grid); break;
      default: e = gemv_grid<4, CAP>(smem, sms, units, &grid); break;
    }
    if (e != cudaSuccess) return e;
  }

  const size_t ws_bytes = fuse ? 0 : ep_off + 256;
  void* ws = nullptr;
  uint32_t* sync = nullptr;
  if (fixed) {
    if (ws_bytes > fixed->bytes) return cudaErrorMemoryAllocation;
    ws = fixed->ptr;
    sync = fixed->sync;
  } else {
    e = get_workspace(stream, ws_bytes, &ws, &sync);
    if (e != cudaSuccess) return e;
  }
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* psum_base = reinterpret_cast<float*>(wsb + psum_off);
  for (int i = 0; i < n_jobs; ++i) {
    if (fuse) {
      gp.lin[i].xf = static_cast<const uint8_t*>(jobs[i].x);  // the producers read x itself
      gp.lin[i].psum = nullptr;
    } else {
      gp.lin[i].xf = wsb + layouts[lay_of[i]].off;
      gp.lin[i].psum = psum_base + size_t(sum_of[i]) * M * kClasses;
    }
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

  // CTA ranges of equal estimated cost, and the row blocks they share.
  int64_t total_cost = 0;
  for (int i = 0; i < n_jobs; ++i) {
    const int64_t lin_units = (i + 1 < n_jobs ? gp.lin[i + 1].unit_begin : units) - gp.lin[i].unit_begin;
    total_cost += lin_units * unit_cost(gp.lin[i].dk);
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
        const int64_t lin_cost = lin_units * unit_cost(gp.lin[li].dk);
        if (target <= cost_before + lin_cost) break;
        cost_before += lin_cost;
        ++li;
      }
      int u;
      if (li >= n_jobs) {
        u = units;
      } else {
        const int64_t w = unit_cost(gp.lin[li].dk);
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
  pp.n_i8 = 0;
  for (int i = 0; i < n_layouts; ++i) {
    pp.lay[i] = {static_cast<const __nv_bfloat16*>(layouts[i].x), wsb + layouts[i].off,
                 layouts[i].K, layouts[i].kc, layouts[i].w8, layouts[i].n_kc,
                 layouts[i].b0 == 8 ? 1 : 0, layouts[i].i8};
    if (layouts[i].i8) pp.n_i8 += layouts[i].n_kc;
  }
  for (int i = 0; i < n_sums; ++i) {
    pp.sum[i] = {static_cast<const __nv_bfloat16*>(sum_x[i]),
                 psum_base + size_t(i) * M * kClasses, sum_k[i]};
  }
  if (!fuse) {
    int prep_grid = std::max(n_sums * M, sms);
    if (pp.n_ep > 0) prep_grid = 4 * sms;  // the Extra Precision gathers want many warps in flight
    // one warp per (unit, digit) of the digit layouts, all in one round
    prep_grid = std::max(prep_grid, (pp.n_i8 * kI8Digits + 7) / 8);
    prep_grid = std::min(prep_grid, 4 * sms);
    e = launch_pdl(gemv_prep_kernel<CAP>, dim3(prep_grid), dim3(256), 0, stream, pp);
    if (e != cudaSuccess) return e;
  }

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
  gp.sync = sync;
  gp.wait_ns = wait_limit_ns();
  gp.shl[0] = 4u;
  gp.shl[1] = 16u;
  gp.shl[2] = 64u;

  if (fuse) return launch_gemv<1, CAP, true, true>(gp, smem, grid, stream);
  switch (NT) {
    case 1: return i8_only ? launch_gemv<1, CAP, true>(gp, smem, grid, stream) : launch_gemv<1, CAP>(gp, smem, grid, stream);
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
  // Same arithmetic as the planner in run_gemv_cap for one linear (without an
  // Extra Precision list): activation blocks, class sums, the trailing 256.
  const int P0 = tiling_p0(M);
  int b0, b1;
  job_planes(job, b0, b1);
  const int kc = P0 * 8 / b0;
  const int64_t n_kc = (job.K + kc - 1) / kc;
  const int dk = decode_kind(job);
  const bool i8 = M == 1 && (dk == 8 || dk == 4 || dk == 2);
  size_t xf = size_t(n_kc) * (i8 ? size_t(i8_unit_bytes(dk)) : size_t(M) * kc * 2);
  xf = (xf + 255) & ~size_t(255);
  const size_t sums = (size_t(M) * kClasses * sizeof(float) + 255) & ~size_t(255);
  return xf + sums + 256;
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
