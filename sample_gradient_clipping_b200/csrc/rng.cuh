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
// their arguments straight from the 32-bit words.  So the range reduction is exact integer
// work, and each is a short textbook series (log_u1_from_word, sincos_turn_from_word), with
// errors near 1e-16.
//
// Counter layout: (j, layer_id, step mod 2^32, stream); key: (seed mod 2^32, seed >> 32).
#pragma once
#include <cstdint>

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

// ln(u1) for u1 = (x + 1) 2^-32, in fp64, straight from the integer.
// y = x + 1 = 2^e f with f in [sqrt(2)/2, sqrt(2)) found exactly from the leading bit, so
// ln u1 = (e - 32) ln 2 + ln f, and ln f = 2 atanh(s) = 2 (s + s^3/3 + s^5/5 + ...) with
// s = (f - 1) / (f + 1), |s| <= 0.1716 (the classical atanh series for the logarithm).  Nine
// terms leave a truncation error below 0.1716^19 / 19 < 3e-16 relative.
__device__ __forceinline__ double log_u1_from_word(uint32_t x) {
  const unsigned long long y = static_cast<unsigned long long>(x) + 1ull;  // 1 .. 2^32
  int e = 63 - __clzll(static_cast<long long>(y));                         // y in [2^e, 2^(e+1))
  // f = y 2^-e, exact: y < 2^53 and the scale is a power of two.
  double f = static_cast<double>(y) * __longlong_as_double(static_cast<long long>(1023 - e) << 52);
  if (f > 1.4142135623730951) {
    f *= 0.5;
    ++e;
  }
  const double s = (f - 1.0) / (f + 1.0);
  const double s2 = s * s;
  double p = 1.0 / 19.0;
  p = fma(p, s2, 1.0 / 17.0);
  p = fma(p, s2, 1.0 / 15.0);
  p = fma(p, s2, 1.0 / 13.0);
  p = fma(p, s2, 1.0 / 11.0);
  p = fma(p, s2, 1.0 / 9.0);
  p = fma(p, s2, 1.0 / 7.0);
  p = fma(p, s2, 1.0 / 5.0);
  p = fma(p, s2, 1.0 / 3.0);
  const double ln_f = 2.0 * s * fma(p, s2, 1.0);
  return fma(static_cast<double>(e - 32), 0.6931471805599453, ln_f);
}

// (cos, sin) of the angle 2 pi x 2^-32, in fp64, from the integer.
// The quadrant is the top two bits of x.  Within it, the angle fraction f < 2^30 is reflected
// to f' = 2^30 - f when f > 2^29, so that the reduced angle t = f' 2 pi 2^-32 lies in
// [0, pi/4]; the reflection swaps sine and cosine, and each quadrant rotates the pair by 90
// degrees.  All of this is exact integer work.  sin t and cos t are then the Taylor series to
// t^15 and t^16: the next terms are below (pi/4)^17/17! < 2e-16.
__device__ __forceinline__ void sincos_turn_from_word(uint32_t x, double& c, double& s) {
  const uint32_t quadrant = x >> 30;
  uint32_t f = x & 0x3FFFFFFFu;
  const bool reflect = f > 0x20000000u;
  if (reflect) f = 0x40000000u - f;
  const double t = static_cast<double>(f) * 1.4629180792671596e-09;  // 2 pi / 2^32
  const double t2 = t * t;
  double sp = -1.0 / 1307674368000.0;          // -1/15!
  sp = fma(sp, t2, 1.0 / 6227020800.0);         //  1/13!
  sp = fma(sp, t2, -1.0 / 39916800.0);          // -1/11!
  sp = fma(sp, t2, 1.0 / 362880.0);             //  1/9!
  sp = fma(sp, t2, -1.0 / 5040.0);              // -1/7!
  sp = fma(sp, t2, 1.0 / 120.0);                //  1/5!
  sp = fma(sp, t2, -1.0 / 6.0);                 // -1/3!
  const double sin_t = fma(sp * t2, t, t);
  double cp = 1.0 / 20922789888000.0;           //  1/16!
  cp = fma(cp, t2, -1.0 / 87178291200.0);       // -1/14!
  cp = fma(cp, t2, 1.0 / 479001600.0);          //  1/12!
  cp = fma(cp, t2, -1.0 / 3628800.0);           // -1/10!
  cp = fma(cp, t2, 1.0 / 40320.0);              //  1/8!
  cp = fma(cp, t2, -1.0 / 720.0);               // -1/6!
  cp = fma(cp, t2, 1.0 / 24.0);                 //  1/4!
  cp = fma(cp, t2, -0.5);                       // -1/2!
  const double cos_t = fma(cp, t2, 1.0);
  const double cq = reflect ? sin_t : cos_t;    // cos and sin of the angle within the quadrant
  const double sq = reflect ? cos_t : sin_t;
  // Rotate by quadrant * 90 degrees without branches: odd quadrants swap the pair, and the
  // cosine is negative in quadrants 1 and 2, the sine in quadrants 2 and 3.
  const bool odd = quadrant & 1u;
  const double c0 = odd ? sq : cq;
  const double s0 = odd ? cq : sq;
  c = (quadrant == 1u || quadrant == 2u) ? -c0 : c0;
  s = (quadrant >= 2u) ? -s0 : s0;
}

__device__ __forceinline__ void box_muller_f64(uint32_t x_even, uint32_t x_odd, double& z_even,
                                               double& z_odd) {
  const double radius = sqrt(-2.0 * log_u1_from_word(x_even));
  double c, s;
  sincos_turn_from_word(x_odd, c, s);
  z_even = radius * c;
  z_odd = radius * s;
}

// The four standard normals of Philox block j: elements 4j .. 4j+3 of the stream.
__device__ __forceinline__ void normals4(uint32_t j, uint32_t layer_id, uint32_t step_lo,
                                         uint32_t stream, PhiloxKey key, double (&z)[4]) {
  const uint4 x = philox4x32_10(make_uint4(j, layer_id, step_lo, stream), key);
  box_muller_f64(x.x, x.y, z[0], z[1]);
  box_muller_f64(x.z, x.w, z[2], z[3]);
}

}  // namespace dpclip
