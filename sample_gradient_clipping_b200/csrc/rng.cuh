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
// The transform is evaluated in fp64 with CUDA's log and sincospi.  A value in fp32 would
// be off by several 1e-7 near |z| = 6.7, because 2 pi u2 and ln u1 then lose bits.
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

__device__ __forceinline__ void box_muller_f64(uint32_t x_even, uint32_t x_odd, double& z_even,
                                               double& z_odd) {
  const double u1 = (static_cast<double>(x_even) + 1.0) * 0x1p-32;
  const double u2 = static_cast<double>(x_odd) * 0x1p-32;
  const double radius = sqrt(-2.0 * log(u1));
  double s, c;
  sincospi(2.0 * u2, &s, &c);
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
