// kernels_f32.cuh - fp32 FAVOR forward on CUDA cores (the accuracy path), plus the ORF builder.
//
// The arithmetic follows the explainer page "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？",
// section 核心机制：FAVOR+:
//   - features phi(x) (cos/sin random features or ReLU generalized-attention features);
//   - chunk states dS_c = sum_{j in chunk c} phi(k_j) [v_j | 1]^T;
//   - a scan over chunks: exclusive prefix for causal, total for bidirectional;
//   - out_i = (phi(q_i) S_i)[:d] / (phi(q_i) S_i)[d].
//     Causal: S_i = (prefix before the chunk) + sum_{j in chunk, j <= i} phi(k_j)[v_j|1]^T.
// Cancelling factors: 1/sqrt(M) and exp(|q|^2/2) are dropped, and the key factor is
// exp(|k|^2/2 - c_h) with c_h = max_j |k_j|^2/2 of the head.
// sin, cos and exp are evaluated in double and rounded to fp32: the library is built with fast
// single-precision intrinsics, whose error grows with the angle.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "philox.cuh"
#include "ptx.cuh"

namespace favor {
namespace f32 {

constexpr int kChunk = 64;   // tokens per chunk
constexpr int kFeatTile = 32;  // features per tile
constexpr int kThreads = 256;
constexpr int kMaxD = 128;

// Feature f of token x (length d) with projection u = omega_a . x:
//   trig: f <  M -> w cos(u_f),  f >= M -> w sin(u_{f-M})
//   relu: max(u_f, 0)
__device__ __forceinline__ float feature_value(int kind, int M, int f, const float* x,
                                              const float* __restrict__ omega, int d, float w) {
  const int a = (kind == 0 && f >= M) ? f - M : f;
  const float* om = omega + (size_t)a * d;
  float u = 0.f;
  for (int t = 0; t < d; ++t) u = fmaf(om[t], x[t], u);
  if (kind == 0) {
    double s, c;
    sincos(static_cast<double>(u), &s, &c);
    return w * static_cast<float>(f < M ? c : s);
  }
  return fmaxf(u, 0.f);
}

// c_h = max_j |k_j|^2 / 2 for each head (trig stabiliser).
__global__ void __launch_bounds__(kThreads) k_key_halfnorm_max(const float* __restrict__ k,
                                                                float* __restrict__ cmax, int L,
                                                                int d) {
  const int bh = blockIdx.x;
  const float* kh = k + (size_t)bh * L * d;
  float m = -INFINITY;
  for (int j = threadIdx.x; j < L; j += blockDim.x) {
    float s = 0.f;
    for (int t = 0; t < d; ++t) s = fmaf(kh[(size_t)j * d + t], kh[(size_t)j * d + t], s);
    m = fmaxf(m, 0.5f * s);
  }
  __shared__ float red[kThreads / 32];
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
    for (int i = 1; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
    cmax[bh] = r;
  }
}

// dS[bh][c][f][n] = sum_{j in chunk c} phi_f(k_j) vv_j[n], vv_j = [v_j | 1], for one tile of
// kFeatTile features. grid = (nfeat_tiles, nchunks, BH).
__global__ void __launch_bounds__(kThreads)
    k_chunk_state(const float* __restrict__ k, const float* __restrict__ v,
                  const float* __restrict__ omega, const float* __restrict__ cmax,
                  float* __restrict__ dS, int H, int L, int d, int M, int F, int kind) {
  extern __shared__ float sm[];
  float* sk = sm;                             // [kChunk][d]
  float* sv = sk + kChunk * d;                // [kChunk][d]
  float* sw = sv + kChunk * d;                // [kChunk]
  float* sphi = sw + kChunk;                  // [kChunk][kFeatTile]
  const int ft = blockIdx.x, c = blockIdx.y, bh = blockIdx.z, h = bh % H;
  const int j0 = c * kChunk, nj = min(kChunk, L - j0);
  const float* kh = k + ((size_t)bh * L + j0) * d;
  const float* vh = v + ((size_t)bh * L + j0) * d;
  const float* om = omega + (size_t)h * M * d;
  for (int i = threadIdx.x; i < kChunk * d; i += blockDim.x) {
    const bool ok = i < nj * d;
    sk[i] = ok ? kh[i] : 0.f;
    sv[i] = ok ? vh[i] : 0.f;
  }
  __syncthreads();
  if (threadIdx.x < kChunk) {
    const int j = threadIdx.x;
    float w = 0.f;
    if (j < nj) {
      if (kind == 0) {
        float s = 0.f;
        for (int t = 0; t < d; ++t) s = fmaf(sk[j * d + t], sk[j * d + t], s);
        w = static_cast<float>(exp(0.5 * static_cast<double>(s) - cmax[bh]));
      } else {
        w = 1.f;
      }
    }
    sw[j] = w;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
    const int j = p / kFeatTile, fl = p % kFeatTile, f = ft * kFeatTile + fl;
    float val = 0.f;
    if (j < nj && f < F) val = feature_value(kind, M, f, sk + j * d, om, d, sw[j]);
    sphi[j * kFeatTile + fl] = (j < nj) ? val : 0.f;
  }
  __syncthreads();
  const int dv = d + 1;
  float* out = dS + (((size_t)bh * gridDim.y + c) * F) * dv;
  for (int p = threadIdx.x; p < kFeatTile * dv; p += blockDim.x) {
    const int fl = p / dv, n = p % dv, f = ft * kFeatTile + fl;
    if (f >= F) continue;
    float acc = 0.f;
    for (int j = 0; j < nj; ++j) acc = fmaf(sphi[j * kFeatTile + fl], n < d ? sv[j * d + n] : 1.f, acc);
    out[(size_t)f * dv + n] = acc;
  }
}

// In-place scan over chunks for every (bh, f, n): exclusive prefix (causal) or the total,
// written into chunk 0 (bidirectional).
__global__ void k_scan_chunks(float* __restrict__ dS, int nchunks, long long per_chunk, long long total,
                              int causal) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const long long bh = e / per_chunk, r = e % per_chunk;
  float* p = dS + bh * nchunks * per_chunk + r;
  float run = 0.f;
  for (int c = 0; c < nchunks; ++c) {
    const float x = p[c * per_chunk];
    if (causal) p[c * per_chunk] = run;
    run += x;
  }
  if (!causal) p[0] = run;
}

// Output for one chunk of queries: grid = (nchunks, BH).
__global__ void __launch_bounds__(kThreads)
    k_output(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
             const float* __restrict__ omega, const float* __restrict__ cmax,
             const float* __restrict__ S, float* __restrict__ out, int H, int L, int d, int M,
             int F, int kind, int causal) {
  extern __shared__ float sm[];
  const int dv = d + 1;
  float* sq = sm;                           // [kChunk][d]
  float* sk = sq + kChunk * d;              // [kChunk][d]
  float* sv = sk + kChunk * d;              // [kChunk][d]
  float* sw = sv + kChunk * d;              // [kChunk]
  float* pq = sw + kChunk;                  // [kChunk][kFeatTile]
  float* pk = pq + kChunk * kFeatTile;      // [kChunk][kFeatTile]
  float* sS = pk + kChunk * kFeatTile;      // [kFeatTile][dv]
  float* A = sS + kFeatTile * dv;           // [kChunk][kChunk]
  const int c = blockIdx.x, bh = blockIdx.y, h = bh % H;
  const int i0 = c * kChunk, ni = min(kChunk, L - i0);
  const size_t base = ((size_t)bh * L + i0) * d;
  const float* om = omega + (size_t)h * M * d;
  const float* Sc = S + (((size_t)bh * gridDim.x + (causal ? c : 0)) * F) * dv;
  for (int i = threadIdx.x; i < kChunk * d; i += blockDim.x) {
    const bool ok = i < ni * d;
    sq[i] = ok ? q[base + i] : 0.f;
    sk[i] = (ok && causal) ? k[base + i] : 0.f;
    sv[i] = (ok && causal) ? v[base + i] : 0.f;
  }
  for (int i = threadIdx.x; i < kChunk * kChunk; i += blockDim.x) A[i] = 0.f;
  __syncthreads();
  if (causal && threadIdx.x < kChunk) {
    const int j = threadIdx.x;
    float w = 0.f;
    if (j < ni) {
      if (kind == 0) {
        float s = 0.f;
        for (int t = 0; t < d; ++t) s = fmaf(sk[j * d + t], sk[j * d + t], s);
        w = static_cast<float>(exp(0.5 * static_cast<double>(s) - cmax[bh]));
      } else {
        w = 1.f;
      }
    }
    sw[j] = w;
  }
  // Thread mapping for the numerator: token i = tid / 4, columns n = tid % 4 + 4 m.
  const int ti = threadIdx.x >> 2, tn = threadIdx.x & 3;
  constexpr int kMaxCols = (kMaxD + 1 + 3) / 4;
  float acc[kMaxCols];
#pragma unroll
  for (int m = 0; m < kMaxCols; ++m) acc[m] = 0.f;
  const int nft = (F + kFeatTile - 1) / kFeatTile;
  for (int ft = 0; ft < nft; ++ft) {
    __syncthreads();
    for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
      const int j = p / kFeatTile, fl = p % kFeatTile, f = ft * kFeatTile + fl;
      float a = 0.f, b = 0.f;
      if (j < ni && f < F) {
        a = feature_value(kind, M, f, sq + j * d, om, d, 1.f);
        if (causal) b = feature_value(kind, M, f, sk + j * d, om, d, sw[j]);
      }
      pq[p] = a;
      pk[p] = b;
    }
    for (int p = threadIdx.x; p < kFeatTile * dv; p += blockDim.x) {
      const int fl = p / dv, f = ft * kFeatTile + fl;
      sS[p] = (f < F) ? Sc[(size_t)f * dv + (p % dv)] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
      const int n = tn + 4 * m;
      if (n < dv) {
        float s = acc[m];
        for (int fl = 0; fl < kFeatTile; ++fl) s = fmaf(pq[ti * kFeatTile + fl], sS[fl * dv + n], s);
        acc[m] = s;
      }
    }
    if (causal) {
      for (int p = threadIdx.x; p < kChunk * kChunk; p += blockDim.x) {
        const int i = p / kChunk, j = p % kChunk;
        if (j <= i) {
          float s = A[p];
          for (int fl = 0; fl < kFeatTile; ++fl) s = fmaf(pq[i * kFeatTile + fl], pk[j * kFeatTile + fl], s);
          A[p] = s;
        }
      }
    }
  }
  __syncthreads();
  if (causal) {
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
      const int n = tn + 4 * m;
      if (n < dv) {
        float s = acc[m];
        for (int j = 0; j <= ti; ++j) s = fmaf(A[ti * kChunk + j], n < d ? sv[j * d + n] : 1.f, s);
        acc[m] = s;
      }
    }
  }
  // den lives in column d, held by thread tn == d % 4 at m = d / 4.
  __shared__ float sden[kChunk];
  if (tn == (d & 3)) sden[ti] = acc[d >> 2];
  __syncthreads();
  if (ti < ni) {
    const float den = sden[ti];
    const float inv = den != 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
      const int n = tn + 4 * m;
      if (n < d) out[base + (size_t)ti * d + n] = den != 0.f ? acc[m] * inv : 0.f;
    }
  }
}

}  // namespace f32

// ------------------------------------------------------------------ ORF builder
// One block per (head, d x d Gaussian block). The block's rows are orthonormalised in order:
// the Q factor of G^T = Q R with a positive diagonal R, which is what Gram-Schmidt in order
// produces. Row r is then scaled by |gauss_norms[h, r, :]|. With `seeded`, the block's Gaussians
// and its rows' chi draws are generated here from `seed` (philox.cuh: the same draws
// k_orf_gaussians writes out) instead of being read from G and R.
// "Masked Language Modeling for Proteins via Linearly Scalable Long-Context Transformers"
// (方法详解) calls these orthogonal random features. The explainer's 核心机制 section
// constrains the directions to a random subsample of an orthogonal matrix.
//
// Rows go in panels of kOrfPanel. A panel is first made orthogonal to every finished row by two
// passes of block classical Gram-Schmidt (8x8x4 fp64 tensor-core products), then
// orthonormalised within itself by two passes of Cholesky QR on its Gram matrix (the lower
// Cholesky factor L of V V^T gives V <- L^-1 V). Both are exact reformulations of Gram-Schmidt in
// order (the same Q), in fp64; the serial chain is a few dozen small steps per panel instead of a
// block-wide reduction per row.
// D = A B + D on the fp64 tensor cores, 8x8x4: lane l holds A[l/4][l%4], B[l%4][l/4] and
// D[l/4][2(l%4)], D[l/4][2(l%4)+1].
__device__ __forceinline__ void mma_f64_m8n8k4(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

constexpr int kOrfThreads = 512;
constexpr int kOrfPanel = 8;  // rows per panel: one warp each

// Row stride of the block in shared memory (doubles): 4 modulo 16, so the 8x4 and 4x8 operand
// fragments of the fp64 MMAs (lane l reads row l/4, column l%4, or the transpose) fall on distinct
// banks within each half-warp.
__host__ __device__ constexpr int orf_ld(int d) { return (d + 11) / 16 * 16 + 4; }
constexpr int kOrfCoefLd = 132;  // coefficient rows, 4 modulo 16 for the same reason
__host__ __device__ constexpr size_t orf_smem_bytes(int d) {
  return ((size_t)d * orf_ld(d) + kOrfPanel * kOrfCoefLd + kOrfPanel * kOrfPanel + kOrfPanel + 128) * sizeof(double);
}

__global__ void __launch_bounds__(kOrfThreads)
    k_orf(const double* __restrict__ G, const double* __restrict__ R, void* __restrict__ omega,
          int H, int M, int d, int out_bf16, uint64_t seed, int seeded) {
  extern __shared__ double orf_sm[];
  const int ld = orf_ld(d);
  double* sq = orf_sm;                            // [d][ld] rows being orthonormalised
  double* coef = sq + (size_t)d * ld;             // [kOrfPanel][kOrfCoefLd] coefficients against finished rows
  double* gram = coef + kOrfPanel * kOrfCoefLd;   // [kOrfPanel][kOrfPanel] Gram matrix -> Cholesky factor
  double* rdiag = gram + kOrfPanel * kOrfPanel;   // [kOrfPanel] 1 / L_kk
  double* chi = rdiag + kOrfPanel;                // [128] row lengths
  const int h = blockIdx.y, blk = blockIdx.x, nb = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long n0 = (((long long)h * nb + blk) * d) * d;  // first draw of this block
  const long long NG = ((long long)H * nb * d * d + 3) / 4 * 4;
  if (seeded) {
    for (long long gq = n0 / 4 + tid; gq <= (n0 + d * d - 1) / 4; gq += blockDim.x) {
      double z[4];
      rng::normals4(seed, (uint64_t)gq, z);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const long long e = 4 * gq + p - n0;
        if (e >= 0 && e < (long long)d * d) sq[(e / d) * ld + e % d] = z[p];
      }
    }
  } else {
    const double* g = G + n0;
    for (int e = tid; e < d * d; e += blockDim.x) sq[(e / d) * ld + e % d] = g[e];
  }
  // chi lengths: tpr threads per output row (a power of two <= 32), each summing every tpr-th
  // group of four draws of the row
  {
    int lg = 0;
    while ((1 << (lg + 1)) <= 32 && (d << (lg + 1)) <= (int)blockDim.x) ++lg;
    const int tpr = 1 << lg, i = tid >> lg, part = tid & (tpr - 1);
    const int r = blk * d + i;
    double s = 0.0;
    if (i < d && r < M) {
      if (seeded) {
        const long long nr = NG + ((long long)h * M + r) * d;
        const long long g0 = nr / 4, g1 = (nr + d - 1) / 4;
        for (long long gq = g0 + part; gq <= g1; gq += tpr) {
          double z[4];
          rng::normals4(seed, (uint64_t)gq, z);
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const long long n = 4 * gq + p;
            if (n >= nr && n < nr + d) s = fma(z[p], z[p], s);
          }
        }
      } else {
        const double* rr = R + ((size_t)h * M + r) * d;
        for (int t = part; t < d; t += tpr) s = fma(rr[t], rr[t], s);
      }
    }
    for (int o = 1; o < tpr; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (part == 0 && i < d) chi[i] = sqrt(s);
  }
  __syncthreads();

  for (int r0 = 0; r0 < d; r0 += kOrfPanel) {
    const int nr = min(kOrfPanel, d - r0);
    const bool act = warp < nr;
    double* vi = sq + (size_t)(r0 + warp) * ld;
    // (1) two passes of block classical Gram-Schmidt of the panel against rows 0 .. r0-1, on the
    // fp64 tensor cores (mma m8n8k4: the panel is the 8-row side): C = V Q^T over 8-row blocks of
    // Q, one block per warp, then V -= C Q over 8-column blocks of V, one block per warp
    if (r0 > 0) {
      const int gi = lane >> 2, gk = lane & 3, nw = blockDim.x >> 5;
      const double* arow = sq + (size_t)(r0 + min(gi, nr - 1)) * ld;
      for (int pass = 0; pass < 2; ++pass) {
        for (int jb = warp; jb < (r0 >> 3); jb += nw) {
          double c0 = 0.0, c1 = 0.0;
          const double* brow = sq + (size_t)(jb * 8 + gi) * ld;
          for (int t0 = 0; t0 < d; t0 += 4) {
            const int t = t0 + gk;
            const double a = (gi < nr && t < d) ? arow[t] : 0.0;
            const double b = t < d ? brow[t] : 0.0;
            mma_f64_m8n8k4(c0, c1, a, b);
          }
          if (gi < nr) {
            coef[gi * kOrfCoefLd + jb * 8 + 2 * gk] = c0;
            coef[gi * kOrfCoefLd + jb * 8 + 2 * gk + 1] = c1;
          }
        }
        __syncthreads();
        for (int tb = warp; tb < ((d + 7) >> 3); tb += nw) {
          double d0 = 0.0, d1 = 0.0;
          const int tn = tb * 8 + gi;
          for (int j0 = 0; j0 < r0; j0 += 4) {
            const double a = gi < nr ? coef[gi * kOrfCoefLd + j0 + gk] : 0.0;
            const double b = tn < d ? sq[(size_t)(j0 + gk) * ld + tn] : 0.0;
            mma_f64_m8n8k4(d0, d1, a, b);
          }
          const int t = tb * 8 + 2 * gk;
          if (gi < nr) {
            double* v = sq + (size_t)(r0 + gi) * ld;
            if (t < d) v[t] -= d0;
            if (t + 1 < d) v[t + 1] -= d1;
          }
        }
        __syncthreads();
      }
    }
    __syncthreads();
    // (2) two passes of Cholesky QR within the panel
    for (int pass = 0; pass < 2; ++pass) {
      if (act) {  // Gram row warp: <v_warp, v_k> for k <= warp
        double g[kOrfPanel];
#pragma unroll
        for (int k = 0; k < kOrfPanel; ++k) g[k] = 0.0;
        for (int t = lane; t < d; t += 32) {
          const double x = vi[t];
#pragma unroll
          for (int k = 0; k < kOrfPanel; ++k)
            if (k <= warp) g[k] = fma(x, sq[(size_t)(r0 + k) * ld + t], g[k]);
        }
#pragma unroll
        for (int k = 0; k < kOrfPanel; ++k) {
#pragma unroll
          for (int o = 16; o; o >>= 1) g[k] += __shfl_xor_sync(0xffffffffu, g[k], o);
        }
        if (lane == 0) {
#pragma unroll
          for (int k = 0; k < kOrfPanel; ++k)
            if (k <= warp) gram[warp * kOrfPanel + k] = g[k];
        }
      }
      __syncthreads();
      if (tid == 0) {  // lower Cholesky factor, in registers; rows past nr are the identity
        double L[kOrfPanel][kOrfPanel];
#pragma unroll
        for (int a = 0; a < kOrfPanel; ++a)
#pragma unroll
          for (int b = 0; b <= a; ++b) L[a][b] = (a < nr) ? gram[a * kOrfPanel + b] : (a == b ? 1.0 : 0.0);
        // right-looking: column c is scaled by 1/sqrt(pivot), then the trailing block loses its
        // outer product, so the next pivot is ready after one update
#pragma unroll
        for (int c = 0; c < kOrfPanel; ++c) {
          const double il = rsqrt(L[c][c]);
          rdiag[c] = il;
#pragma unroll
          for (int a = c + 1; a < kOrfPanel; ++a) L[a][c] *= il;
#pragma unroll
          for (int a = c + 1; a < kOrfPanel; ++a)
#pragma unroll
            for (int b = c + 1; b <= a; ++b) L[a][b] = fma(-L[a][c], L[b][c], L[a][b]);
        }
#pragma unroll
        for (int a = 0; a < kOrfPanel; ++a)
#pragma unroll
          for (int b = 0; b < a; ++b) gram[a * kOrfPanel + b] = L[a][b];
      }
      __syncthreads();
      // V <- L^-1 V by forward substitution, one thread per column
      for (int t = tid; t < d; t += blockDim.x) {
        double q[kOrfPanel];
#pragma unroll
        for (int k = 0; k < kOrfPanel; ++k) {
          if (k < nr) {
            double x = sq[(size_t)(r0 + k) * ld + t];
#pragma unroll
            for (int j = 0; j < k; ++j) x = fma(-gram[k * kOrfPanel + j], q[j], x);
            q[k] = x * rdiag[k];
            sq[(size_t)(r0 + k) * ld + t] = q[k];
          }
        }
      }
      __syncthreads();
    }
  }
  for (int e = tid; e < d * d; e += blockDim.x) {
    const int i = e / d, t = e % d, r = blk * d + i;
    if (r >= M) continue;
    const double val = sq[(size_t)i * ld + t] * chi[i];
    const size_t o = ((size_t)h * M + r) * d + t;
    if (out_bf16)
      reinterpret_cast<__nv_bfloat16*>(omega)[o] = __double2bfloat16(val);
    else
      reinterpret_cast<float*>(omega)[o] = (float)val;
  }
}

}  // namespace favor
