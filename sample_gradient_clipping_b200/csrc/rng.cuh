// Counter-based Gaussian noise: Philox4x32-10 followed by Box-Muller in fp64.
//
// Philox4x32-10 is written from Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
// easy as 1, 2, 3" (SC'11).  Each of the ten rounds multiplies words 0 and 2 by two fixed
// odd constants, keeping both halves of the 64-bit products.  It then mixes the high halves
// with words 1 and 3 and with the key, and permutes the words.  The key is bumped by two Weyl
// constants between rounds.
//
// Box-Muller (Box and Muller, Ann. Math. Stat. 1958) maps a pair (x_even, x_odd) to two
// standard normals:
//   u1 = (x_even + 1) 2^-32 lies in (0, 1], so the logarithm is finite;
//   u2 = x_odd 2^-32;
//   z_even = sqrt(-2 ln u1) cos(2 pi u2) and z_odd = sqrt(-2 ln u1) sin(2 pi u2).
// The transform is evaluated in fp64.  A value in fp32 would be off by several 1e-7 near
// |z| = 6.7, because 2 pi u2 and ln u1 then lose bits.  The logarithm and the sine/cosine take
// their arguments straight from the 32-bit words, so the range reduction is exact integer
// work, and each is a table lookup plus a short polynomial (box_muller_f64 below).
//
// Counter layout: (j, layer_id, step mod 2^32, stream); key: (seed mod 2^32, seed >> 32).
#pragma once
#include <cstdint>

#include "noise_tables.cuh"

namespace dpclip {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

constexpr uint32_t kStreamNoise = 0u;
constexpr uint32_t kStreamProjection = 1u;

struct PhiloxKey {
  uint32_t k0, k1;
};

// The step number of the noise counter: fixed at launch, or read from device memory when the
// kernel runs, so that one CUDA graph captured once serves every training step.
struct StepRef {
  uint32_t lo;                      // step mod 2^32, used when dev is null
  const unsigned long long* dev;    // DEVICE address of the step, or null
  __device__ __forceinline__ uint32_t get() const {
    return dev ? static_cast<uint32_t>(*dev & 0xFFFFFFFFull) : lo;
  }
};

inline StepRef step_value(unsigned long long step) {
  return StepRef{static_cast<uint32_t>(step & 0xFFFFFFFFull), nullptr};
}

__host__ __device__ inline PhiloxKey philox_key_from_seed(unsigned long long seed) {
  return PhiloxKey{static_cast<uint32_t>(seed & 0xFFFFFFFFull), static_cast<uint32_t>(seed >> 32)};
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, PhiloxKey k) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    if (round) {
      k.k0 += kPhiloxW0;
      k.k1 += kPhiloxW1;
    }
    const uint32_t hi_a = __umulhi(kPhiloxM0, c.x);
    const uint32_t lo_a = kPhiloxM0 * c.x;
    const uint32_t hi_b = __umulhi(kPhiloxM1, c.z);
    const uint32_t lo_b = kPhiloxM1 * c.z;
    c = make_uint4(hi_b ^ c.y ^ k.k0, lo_b, hi_a ^ c.w ^ k.k1, lo_a);
  }
  return c;
}

// Table-driven Box-Muller (Tang, "Table-driven implementation of the logarithm function in
// IEEE floating-point arithmetic", ACM TOMS 1990; sine and cosine by the addition formula
// around tabulated angles).  Every breakpoint value is the double nearest its exact value
// (gen_noise_tables.py), so each piece is a short polynomial on a small interval.  The noise is
// issue-bound where it is generated, so the form is cut to about 30 fp64 operations a pair:
// polynomial degrees only as high as a 1e-12 result needs, the factor -2 of -2 ln u1 and the
// angle unit 2 pi 2^-32 folded into the tables and coefficients, one Newton step for the square
// root, and the caller's scale (the noise std) folded into the radius.  Against CUDA's
// full-precision log, sqrt and sincospi, |z - z_ref| stayed below 2.1e-12 on all edge words
// (every table breakpoint of both words and its neighbours, u1 = 1, u1 = 2^-32) and on 2^30
// random pairs; the largest errors come at u1 just below 1, where the radius is ~2e-5.

// Where the transform reads its tables.  Global: the module's arrays through the read-only
// cache.  Shared: eight copies, entry j of copy c at [8 j + c], each thread reading copy
// threadIdx.x mod 8.  A 128-bit shared load serves 8 threads per pass, so the 8 threads of a
// pass always read 8 different bank groups, whatever entries they want.
struct NoiseTablesGlobal {
  __device__ __forceinline__ double2 ln(uint32_t j) const { return __ldg(&kLnTable[j]); }
  __device__ __forceinline__ double2 sincos(uint32_t j) const { return __ldg(&kSinCosTable[j]); }
};

constexpr int kNoiseTableCopies = 8;
constexpr int kNoiseSharedEntries = 2 * kNoiseTableSize * kNoiseTableCopies;
constexpr int kNoiseSharedBytes = kNoiseSharedEntries * 16;  // 32 KB

struct NoiseTablesShared {
  const double2* s;  // kNoiseSharedEntries entries, filled by stage_noise_tables
  __device__ __forceinline__ double2 ln(uint32_t j) const {
    return s[j * kNoiseTableCopies + (threadIdx.x & (kNoiseTableCopies - 1))];
  }
  __device__ __forceinline__ double2 sincos(uint32_t j) const {
    return s[(kNoiseTableSize + j) * kNoiseTableCopies + (threadIdx.x & (kNoiseTableCopies - 1))];
  }
};

// Fills the shared copies; the caller synchronises the block before the first read.
__device__ __forceinline__ void stage_noise_tables(double2* s) {
  for (int i = threadIdx.x; i < kNoiseSharedEntries; i += blockDim.x) {
    const int j = (i / kNoiseTableCopies) % kNoiseTableSize;
    s[i] = i < kNoiseTableSize * kNoiseTableCopies ? kLnTable[j] : kSinCosTable[j];
  }
}

__device__ __forceinline__ float rsqrt_approx(float a) {
  float r;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}

// Integer -> double without a conversion instruction: the double with high word 0x43300000
// and low word u is exactly 2^52 + u, so one subtraction gives u - offset exactly.  Where the
// noise is generated, conversions share a narrow pipe that would otherwise be the bound.
constexpr double kTwo52 = 4503599627370496.0;
__device__ __forceinline__ double u32_minus(uint32_t u, double offset) {
  return __hiloint2double(0x43300000, static_cast<int>(u)) - (kTwo52 + offset);
}

// -2 ln(u1), u1 = (x + 1) 2^-32.  x + 1 = 2^k m exactly, m in [1, 2).  With (F, L) the table
// entry of m's top 7 fraction bits, ln m = L + ln(1 + r), r = m F - 1, |r| <= 2^-8.  The table
// holds (-2F, -2L), so one fused multiply-add gives r' = -2r exactly as -2 times the rounded r,
// and -2 ln(1 + r) = r' + r'^2/4 + r'^3/12 + r'^4/32 + r'^5/80 (the next term is below 2e-15).
// ln 2 is split so that (k - 32)(-2 ln 2) adds without rounding error.
template <class Tab>
__device__ __forceinline__ double minus_two_ln_u1(uint32_t x, const Tab& tab) {
  const double d = u32_minus(x, -1.0);             // x + 1, exact
  const int hi = __double2hiint(d);                // biased exponent 1023 + k, k = 0 .. 32
  const double m = __hiloint2double((hi & 0x000FFFFF) | 0x3FF00000, __double2loint(d));
  const double2 GH = tab.ln((static_cast<uint32_t>(hi) >> 13) & (kNoiseTableSize - 1));
  const double rp = fma(m, GH.x, 2.0);
  double q = fma(rp, 1.0 / 80.0, 1.0 / 32.0);
  q = fma(rp, q, 1.0 / 12.0);
  q = fma(rp, q, 0.25);
  const double p = fma(rp * rp, q, rp);
  const double kk = u32_minus(static_cast<uint32_t>(hi) >> 20, 1055.0);  // k - 32
  return fma(kk, kMinus2Ln2Hi, GH.y) + fma(kk, kMinus2Ln2Lo, p);
}

// sqrt(y) for 2^-126 <= y < 2^128: an fp32 reciprocal-square-root seed r0 (relative error
// e ~ 2^-22) moved into fp64 by bit manipulation, s = y r0, then one Newton step on the
// residual, s + (y - s^2) r0 / 2, whose relative error is about e^2.
__device__ __forceinline__ double sqrt_pos_f64(double y) {
  const int yh = __double2hiint(y);
  const uint32_t yl = static_cast<uint32_t>(__double2loint(y));
  // y truncated to fp32: exponent rebased from 1023 to 127, 23 fraction bits.
  const float f = __int_as_float(static_cast<int>(__funnelshift_l(yl, static_cast<uint32_t>(yh), 3)) - (896 << 23));
  const int rb = __float_as_int(rsqrt_approx(f));
  const int rl = rb << 29;
  const double r0 = __hiloint2double((rb >> 3) + (896 << 20), rl);
  const double half_r0 = __hiloint2double((rb >> 3) + (895 << 20), rl);
  const double s = y * r0;
  return fma(fma(-s, s, y), half_r0, s);
}

// (cos, sin) of 2 pi x 2^-32.  The top 7 bits of x pick the sector centre a_j = 2 pi (j + 1/2)
// / 128; the other 25 bits, centred, give the integer k with angle - a_j = k a, a = 2 pi 2^-32,
// |k a| <= pi/128.  sin(k a) to (k a)^5 and 1 - cos(k a) to (k a)^4 are polynomials in the
// exact k^2 (next terms below 6e-16 and 3e-13), and enter the addition formulas as
// S (1 - (1 - cos)) + C sin and C (1 - (1 - cos)) - S sin.
template <class Tab>
__device__ __forceinline__ void sincos_turn(uint32_t x, const Tab& tab, double& c, double& s) {
  const double k = u32_minus(x & 0x1FFFFFFu, 16777216.0);
  const double k2 = k * k;                          // exact: |k| <= 2^24
  double t = fma(k2, kSinK5, kSinK3);
  t = fma(k2, t, kSinK1);
  const double sin_d = k * t;
  const double one_minus_cos_d = k2 * fma(k2, kCosK4, kCosK2);
  const double2 SC = tab.sincos(x >> 25);
  s = fma(SC.y, sin_d, fma(-SC.x, one_minus_cos_d, SC.x));
  c = fma(-SC.x, sin_d, fma(-SC.y, one_minus_cos_d, SC.y));
}

// (z_even, z_odd) times `scale`.
template <class Tab>
__device__ __forceinline__ void box_muller_f64(uint32_t x_even, uint32_t x_odd, const Tab& tab, double scale,
                                               double& z_even, double& z_odd) {
  // Every word but x_even = 2^32 - 1 gives y >= 4.6e-10; there u1 = 1, the radius is 0 and y
  // is a rounding residue, which the clamp turns into a radius of 2^-50 instead.
  const double y = fmax(minus_two_ln_u1(x_even, tab), 0x1p-100);
  const double radius = sqrt_pos_f64(y) * scale;
  double c, s;
  sincos_turn(x_odd, tab, c, s);
  z_even = radius * c;
  z_odd = radius * s;
}

// Full-precision Box-Muller (CUDA's log, sqrt and sincospi, ~1e-16).  Used where the normals
// are rounded to a storage type and that rounding must agree with an exact reference bit for
// bit: the projection matrix P.  A 1e-11 error would move a few P entries across a rounding
// boundary.
__device__ __forceinline__ void box_muller_f64_precise(uint32_t x_even, uint32_t x_odd, double& z_even,
                                                       double& z_odd) {
  const double u1 = (static_cast<double>(x_even) + 1.0) * 0x1p-32;
  const double u2 = static_cast<double>(x_odd) * 0x1p-32;
  const double radius = sqrt(-2.0 * log(u1));
  double s, c;
  sincospi(2.0 * u2, &s, &c);
  z_even = radius * c;
  z_odd = radius * s;
}

__device__ __forceinline__ void normals4_precise(uint32_t j, uint32_t layer_id, uint32_t step_lo,
                                                 uint32_t stream, PhiloxKey key, double (&z)[4]) {
  const uint4 x = philox4x32_10(make_uint4(j, layer_id, step_lo, stream), key);
  box_muller_f64_precise(x.x, x.y, z[0], z[1]);
  box_muller_f64_precise(x.z, x.w, z[2], z[3]);
}

// The four standard normals of Philox block j (elements 4j .. 4j+3 of the stream), times
// `scale`.
template <class Tab = NoiseTablesGlobal>
__device__ __forceinline__ void normals4(uint32_t j, uint32_t layer_id, uint32_t step_lo,
                                         uint32_t stream, PhiloxKey key, double (&z)[4],
                                         const Tab& tab = Tab{}, double scale = 1.0) {
  const uint4 x = philox4x32_10(make_uint4(j, layer_id, step_lo, stream), key);
  box_muller_f64(x.x, x.y, tab, scale, z[0], z[1]);
  box_muller_f64(x.z, x.w, tab, scale, z[2], z[3]);
}

}  // namespace dpclip
