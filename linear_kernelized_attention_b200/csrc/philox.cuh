// philox.cuh - counter-based Gaussian draws for redrawing ORF Omega on the device.
//
// The generator is Philox4x64 with 10 rounds, from its published definition (Salmon, Moraes,
// Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011): a 4-word counter and a
// 2-word key; each round maps (x0, x1, x2, x3) to
//   (hi(M1 x2) ^ x1 ^ k0, lo(M1 x2), hi(M0 x0) ^ x3 ^ k1, lo(M0 x0)),
// and the key gains (W0, W1) between rounds. Normal draws: group g is the block of counter
// (g, 0, 0, 0) under key (seed, 0); each word w gives u = (floor(w / 2^11) + 1/2) 2^-53 in (0, 1)
// and the pairs (u0, u1), (u2, u3) go through Box-Muller, sqrt(-2 ln u_a) (cos, sin)(2 pi u_b),
// in double. Draw n is normal n % 4 of group n / 4.
//
// The ORF draws of a seed (the directions' Gaussian blocks and the chi lengths' Gaussians,
// "Masked Language Modeling for Proteins via Linearly Scalable Long-Context Transformers",
// 方法详解) use one stream: G[h, b, i, j] is draw ((h nb + b) d + i) d + j and R[h, r, j] is
// draw NG + (h M + r) d + j, NG being the size of G rounded up to a multiple of 4.
#pragma once
#include <cstdint>

namespace favor {
namespace rng {

constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ull, kM1 = 0xCA5A826395121157ull;  // round multipliers
constexpr uint64_t kW0 = 0x9E3779B97F4A7C15ull, kW1 = 0xBB67AE8584CAA73Bull;  // key increments

__device__ __forceinline__ void philox4x64_10(uint64_t (&x)[4], uint64_t k0, uint64_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint64_t hi0 = __umul64hi(kM0, x[0]), lo0 = kM0 * x[0];
    const uint64_t hi1 = __umul64hi(kM1, x[2]), lo1 = kM1 * x[2];
    const uint64_t y0 = hi1 ^ x[1] ^ k0, y2 = hi0 ^ x[3] ^ k1;
    x[0] = y0;
    x[1] = lo1;
    x[2] = y2;
    x[3] = lo0;
  }
}

// The four normal draws of group g.
__device__ __forceinline__ void normals4(uint64_t seed, uint64_t g, double (&z)[4]) {
  uint64_t x[4] = {g, 0ull, 0ull, 0ull};
  philox4x64_10(x, seed, 0ull);
  double u[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) u[i] = (static_cast<double>(x[i] >> 11) + 0.5) * 0x1p-53;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const double r = sqrt(-2.0 * log(u[2 * p]));
    const double t = (2.0 * 3.141592653589793) * u[2 * p + 1];
    double s, c;
    sincos(t, &s, &c);
    z[2 * p] = r * c;
    z[2 * p + 1] = r * s;
  }
}

// Raw blocks: out[4 i .. 4 i + 3] = Philox4x64-10 of counter (first + i, 0, 0, 0), key (key, 0).
__global__ void k_philox_raw(uint64_t key, uint64_t first, uint64_t n, uint64_t* __restrict__ out) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    uint64_t x[4] = {first + i, 0ull, 0ull, 0ull};
    philox4x64_10(x, key, 0ull);
#pragma unroll
    for (int w = 0; w < 4; ++w) out[4 * i + w] = x[w];
  }
}

// The ORF draws of a seed, written out: G [H, nb, d, d] and R [H, M, d] (layout above).
__global__ void k_orf_gaussians(uint64_t seed, double* __restrict__ G, double* __restrict__ R, long long ng,
                                long long NG, long long nr) {
  const long long total = NG + nr, groups = (total + 3) / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
    double z[4];
    normals4(seed, (uint64_t)g, z);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const long long n = 4 * g + p;
      if (n < ng)
        G[n] = z[p];
      else if (n >= NG && n < total)
        R[n - NG] = z[p];
    }
  }
}

}  // namespace rng
}  // namespace favor
