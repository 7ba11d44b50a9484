// kernels_bwd_f32.cuh - FAVOR backward (dq, dk, dv) in fp32 on CUDA cores.
//
// What it computes: the gradients of sum(dout * out) for out = D^-1 A V, A = phi(Q) phi(K)^T
// (masked to j <= i when causal), the quantity the explainer page
// "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？" (核心机制：FAVOR+) computes in linear
// time. Omega is a fixed random draw and gets no gradient.
//
// Scaled quantities. With the forward's stabilised features psi(q) = [cos u, sin u] (or
// max(u, 0)), psi(k) = w [cos u, sin u] (w = exp(|k|^2/2 - c), c = max |k|^2/2 of the head), the
// kernels form S = sum_j psi(k_j) [v_j | 1]^T and, per query row, N~ = psi(q) S, D~ = its last
// column and out = N~ / D~. Every factor dropped from the features (exp(|q|^2/2), e^c, 1/sqrt(M))
// cancels in the gradients too, which become, with e_i = [dout_i / D~_i | -(dout_i . out_i) / D~_i]:
//   g_i  = S_i e_i                     (S_i: all keys, or keys j <= i when causal)
//   R_j  = sum_i psi(q_i) e_i^T         (all queries, or queries i >= j when causal)
//   h_j  = R_j [v_j | 1],   dv_j = R_j[:, :d]^T psi(k_j)
//   dq_i = q_i (g_i . psi(q_i)) + Omega^T (g_i * psi'(q_i))          (trig)
//        = Omega^T (g_i * [u_i > 0])                                   (ReLU)
//   dk_j = k_j (h_j . psi(k_j)) + Omega^T (h_j * psi'(k_j))           (trig; psi' carries w_j)
//        = Omega^T (h_j * [u_j > 0])                                   (ReLU)
// where psi' is the partner derivative: -w sin u for a cos feature, w cos u for a sin feature.
//
// Work: 64-token chunks, features in tiles of 32. S comes from the forward's chunk states and
// scan (exclusive prefix when causal, the total otherwise). k_bwd_query recomputes the forward
// for its chunk, forms e, dq and its chunk's share of R. A reverse scan turns the shares into
// exclusive suffixes (causal) or the total. k_bwd_key forms dk and dv. Inside a chunk, causal
// terms use the masked 64 x 64 matrices A_ij = psi(q_i) . psi(k_j) and B_ij = [v_j | 1] . e_i.
#pragma once
#include <cstdint>

#include "kernels_f32.cuh"

namespace favor {
namespace bwd {

constexpr int kChunk = f32::kChunk;        // 64 tokens
constexpr int kFeatTile = f32::kFeatTile;  // 32 features
constexpr int kThreads = 256;
constexpr int kMaxD = 64;
constexpr int kCols = kMaxD / 4;  // dq / dk / dv columns per thread (token tid / 4, columns tid % 4 + 4 m)

// Feature f of token x with weight w: its value and its partner derivative (see the header).
__device__ __forceinline__ void feature_pair(int kind, int M, int f, const float* x, const float* __restrict__ om,
                                             int d, float w, float& val, float& der) {
  const int a = (kind == 0 && f >= M) ? f - M : f;
  const float* row = om + (size_t)a * d;
  float u = 0.f;
  for (int t = 0; t < d; ++t) u = fmaf(row[t], x[t], u);
  if (kind == 0) {
    double s, c;
    sincos(static_cast<double>(u), &s, &c);
    const bool is_cos = f < M;
    val = w * static_cast<float>(is_cos ? c : s);
    der = w * static_cast<float>(is_cos ? -s : c);
  } else {
    val = fmaxf(u, 0.f);
    der = u > 0.f ? 1.f : 0.f;
  }
}

// Stabiliser weight of key row j: exp(|k|^2/2 - c) (trig), 1 (ReLU).
__device__ __forceinline__ float key_weight(int kind, const float* kj, int d, float c) {
  if (kind != 0) return 1.f;
  float s = 0.f;
  for (int t = 0; t < d; ++t) s = fmaf(kj[t], kj[t], s);
  return static_cast<float>(exp(0.5 * static_cast<double>(s) - c));
}

struct BwdSmem {
  // offsets in floats from the start of dynamic shared memory
  int sq, sk, sv, sdo, sw, pq, dq_, pk, dk_, sS, sOm, A, Bm, se, sg, sden, total;
};
__host__ __device__ inline BwdSmem bwd_smem(int d) {
  const int dv = d + 1;
  BwdSmem o{};
  int p = 0;
  o.sq = p; p += kChunk * d;
  o.sk = p; p += kChunk * d;
  o.sv = p; p += kChunk * d;
  o.sdo = p; p += kChunk * d;
  o.sw = p; p += kChunk;
  o.pq = p; p += kChunk * kFeatTile;
  o.dq_ = p; p += kChunk * kFeatTile;
  o.pk = p; p += kChunk * kFeatTile;
  o.dk_ = p; p += kChunk * kFeatTile;
  o.sS = p; p += kFeatTile * dv;
  o.sOm = p; p += kFeatTile * d;
  o.A = p; p += kChunk * kChunk;
  o.Bm = p; p += kChunk * kChunk;
  o.se = p; p += kChunk * dv;
  o.sg = p; p += kChunk * kFeatTile;
  o.sden = p; p += kChunk;
  o.total = p;
  return o;
}

// Rows of Omega behind the features of tile ft: sOm[fl][t] = omega[angle(f)][t].
__device__ __forceinline__ void load_omega_tile(float* sOm, const float* __restrict__ om, int ft, int F, int M,
                                                int d, int kind) {
  for (int p = threadIdx.x; p < kFeatTile * d; p += blockDim.x) {
    const int fl = p / d, t = p % d, f = ft * kFeatTile + fl;
    const int a = (kind == 0 && f >= M) ? f - M : f;
    sOm[p] = f < F ? om[(size_t)a * d + t] : 0.f;
  }
}

// Query chunk c of head bh: forward recompute, e, dq, and R's share sum_{i in c} psi(q_i) e_i^T.
// grid = (nchunks, BH).
__global__ void __launch_bounds__(kThreads)
    k_bwd_query(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                const float* __restrict__ omega, const float* __restrict__ cmax, const float* __restrict__ S,
                const float* __restrict__ dout, float* __restrict__ dq, float* __restrict__ E,
                float* __restrict__ Rc, int H, int L, int d, int M, int F, int kind, int causal) {
  extern __shared__ float sm[];
  const BwdSmem o = bwd_smem(d);
  const int dv = d + 1;
  float *sq = sm + o.sq, *sk = sm + o.sk, *sv = sm + o.sv, *sdo = sm + o.sdo, *sw = sm + o.sw;
  float *pq = sm + o.pq, *dqd = sm + o.dq_, *pk = sm + o.pk, *sS = sm + o.sS, *sOm = sm + o.sOm;
  float *A = sm + o.A, *Bm = sm + o.Bm, *se = sm + o.se, *sg = sm + o.sg, *sden = sm + o.sden;
  const int c = blockIdx.x, nch = gridDim.x, bh = blockIdx.y, h = bh % H;
  const int i0 = c * kChunk, ni = min(kChunk, L - i0);
  const size_t base = ((size_t)bh * L + i0) * d;
  const float* om = omega + (size_t)h * M * d;
  const float* Sc = S + (((size_t)bh * nch + (causal ? c : 0)) * F) * dv;
  for (int i = threadIdx.x; i < kChunk * d; i += blockDim.x) {
    const bool ok = i < ni * d;
    sq[i] = ok ? q[base + i] : 0.f;
    sdo[i] = ok ? dout[base + i] : 0.f;
    sk[i] = (ok && causal) ? k[base + i] : 0.f;
    sv[i] = (ok && causal) ? v[base + i] : 0.f;
  }
  for (int i = threadIdx.x; i < kChunk * kChunk; i += blockDim.x) A[i] = 0.f;
  __syncthreads();
  if (threadIdx.x < kChunk) {
    const int j = threadIdx.x;
    sw[j] = (causal && j < ni) ? key_weight(kind, sk + j * d, d, cmax[bh]) : 0.f;
  }
  const int ti = threadIdx.x >> 2, tn = threadIdx.x & 3;
  constexpr int kAcc = (kMaxD + 1 + 3) / 4;
  float acc[kAcc];
#pragma unroll
  for (int m = 0; m < kAcc; ++m) acc[m] = 0.f;
  const int nft = (F + kFeatTile - 1) / kFeatTile;

  // Pass 1: N~ and D~ of the chunk's rows (and the masked A when causal).
  for (int ft = 0; ft < nft; ++ft) {
    __syncthreads();
    for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
      const int j = p / kFeatTile, f = ft * kFeatTile + p % kFeatTile;
      float a = 0.f, b = 0.f, da, db;
      if (j < ni && f < F) {
        feature_pair(kind, M, f, sq + j * d, om, d, 1.f, a, da);
        if (causal) feature_pair(kind, M, f, sk + j * d, om, d, sw[j], b, db);
      }
      pq[p] = a;
      pk[p] = b;
    }
    for (int p = threadIdx.x; p < kFeatTile * dv; p += blockDim.x) {
      const int f = ft * kFeatTile + p / dv;
      sS[p] = f < F ? Sc[(size_t)f * dv + p % dv] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < kAcc; ++m) {
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
    for (int m = 0; m < kAcc; ++m) {
      const int n = tn + 4 * m;
      if (n < dv) {
        float s = acc[m];
        for (int j = 0; j <= ti; ++j) s = fmaf(A[ti * kChunk + j], n < d ? sv[j * d + n] : 1.f, s);
        acc[m] = s;
      }
    }
  }
  // e_i = [dout_i / D~ | -(dout_i . out_i) / D~] (zero when D~ = 0)
  if (tn == (d & 3)) sden[ti] = acc[d >> 2];
  __syncthreads();
  {
    const float den = sden[ti];
    const float inv = den != 0.f ? 1.f / den : 0.f;
    float dot = 0.f;
#pragma unroll
    for (int m = 0; m < kAcc; ++m) {
      const int n = tn + 4 * m;
      if (n < d) dot = fmaf(sdo[ti * d + n], acc[m] * inv, dot);
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    const bool live = ti < ni && den != 0.f;
#pragma unroll
    for (int m = 0; m < kAcc; ++m) {
      const int n = tn + 4 * m;
      if (n < d) se[ti * dv + n] = live ? sdo[ti * d + n] * inv : 0.f;
    }
    if (tn == 0) se[ti * dv + d] = live ? -dot * inv : 0.f;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < ni * dv; p += blockDim.x) E[((size_t)bh * L + i0) * dv + p] = se[p];
  if (causal) {  // B_ij = [v_j | 1] . e_i for j <= i
    for (int p = threadIdx.x; p < kChunk * kChunk; p += blockDim.x) {
      const int i = p / kChunk, j = p % kChunk;
      float s = 0.f;
      if (j <= i) {
        s = se[i * dv + d];
        for (int n = 0; n < d; ++n) s = fmaf(sv[j * d + n], se[i * dv + n], s);
      }
      Bm[p] = s;
    }
  }

  // Pass 2: g tile by tile; dq and R's share.
  float dacc[kCols];
#pragma unroll
  for (int m = 0; m < kCols; ++m) dacc[m] = 0.f;
  float scal = 0.f;  // sum_f g_if psi_f(q_i), held by the 4 threads of row ti in parts
  float* Rout = Rc + (((size_t)bh * nch + c) * F) * dv;
  for (int ft = 0; ft < nft; ++ft) {
    __syncthreads();
    for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
      const int j = p / kFeatTile, f = ft * kFeatTile + p % kFeatTile;
      float a = 0.f, da = 0.f, b = 0.f, db;
      if (j < ni && f < F) {
        feature_pair(kind, M, f, sq + j * d, om, d, 1.f, a, da);
        if (causal) feature_pair(kind, M, f, sk + j * d, om, d, sw[j], b, db);
      }
      pq[p] = a;
      dqd[p] = da;
      pk[p] = b;
    }
    for (int p = threadIdx.x; p < kFeatTile * dv; p += blockDim.x) {
      const int f = ft * kFeatTile + p / dv;
      sS[p] = f < F ? Sc[(size_t)f * dv + p % dv] : 0.f;
    }
    load_omega_tile(sOm, om, ft, F, M, d, kind);
    __syncthreads();
    // g[i][fl] = S_tile[fl] . e_i  (+ sum_{j <= i} B_ij psi_fl(k_j))
    for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
      const int i = p / kFeatTile, fl = p % kFeatTile;
      float s = 0.f;
      for (int n = 0; n < dv; ++n) s = fmaf(sS[fl * dv + n], se[i * dv + n], s);
      if (causal)
        for (int j = 0; j <= i; ++j) s = fmaf(Bm[i * kChunk + j], pk[j * kFeatTile + fl], s);
      sg[p] = s;
    }
    // R share: Rout[f][n] = sum_i psi_f(q_i) e_i[n]
    for (int p = threadIdx.x; p < kFeatTile * dv; p += blockDim.x) {
      const int fl = p / dv, n = p % dv, f = ft * kFeatTile + fl;
      if (f >= F) continue;
      float s = 0.f;
      for (int i = 0; i < ni; ++i) s = fmaf(pq[i * kFeatTile + fl], se[i * dv + n], s);
      Rout[(size_t)f * dv + n] = s;
    }
    __syncthreads();
    // dq_i += sum_fl g * psi'(q_i) * omega_row(fl); the radial sum g . psi(q_i)
    for (int fl = tn; fl < kFeatTile; fl += 4) scal = fmaf(sg[ti * kFeatTile + fl], pq[ti * kFeatTile + fl], scal);
#pragma unroll
    for (int m = 0; m < kCols; ++m) {
      const int t = tn + 4 * m;
      if (t < d) {
        float s = dacc[m];
        for (int fl = 0; fl < kFeatTile; ++fl)
          s = fmaf(sg[ti * kFeatTile + fl] * dqd[ti * kFeatTile + fl], sOm[fl * d + t], s);
        dacc[m] = s;
      }
    }
  }
  scal += __shfl_xor_sync(0xffffffffu, scal, 1);
  scal += __shfl_xor_sync(0xffffffffu, scal, 2);
  if (ti < ni) {
#pragma unroll
    for (int m = 0; m < kCols; ++m) {
      const int t = tn + 4 * m;
      if (t < d) dq[base + (size_t)ti * d + t] = (kind == 0 ? sq[ti * d + t] * scal : 0.f) + dacc[m];
    }
  }
}

// In-place reverse scan over chunks: exclusive suffix (causal) or the total into chunk 0.
__global__ void k_scan_chunks_rev(float* __restrict__ R, int nchunks, long long per_chunk, long long total,
                                  int causal) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const long long bh = e / per_chunk, r = e % per_chunk;
  float* p = R + bh * nchunks * per_chunk + r;
  float run = 0.f;
  for (int c = nchunks - 1; c >= 0; --c) {
    const float x = p[c * per_chunk];
    if (causal) p[c * per_chunk] = run;
    run += x;
  }
  if (!causal) p[0] = run;
}

// Key chunk c of head bh: dk and dv. grid = (nchunks, BH).
__global__ void __launch_bounds__(kThreads)
    k_bwd_key(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
              const float* __restrict__ omega, const float* __restrict__ cmax, const float* __restrict__ R,
              const float* __restrict__ E, float* __restrict__ dk, float* __restrict__ dvout, int H, int L,
              int d, int M, int F, int kind, int causal) {
  extern __shared__ float sm[];
  const BwdSmem o = bwd_smem(d);
  const int dv = d + 1;
  float *sq = sm + o.sq, *sk = sm + o.sk, *sv = sm + o.sv, *sw = sm + o.sw;
  float *pq = sm + o.pq, *pk = sm + o.pk, *dkd = sm + o.dk_, *sR = sm + o.sS, *sOm = sm + o.sOm;
  float *A = sm + o.A, *Bm = sm + o.Bm, *se = sm + o.se, *sh = sm + o.sg;
  const int c = blockIdx.x, nch = gridDim.x, bh = blockIdx.y, h = bh % H;
  const int j0 = c * kChunk, nj = min(kChunk, L - j0);
  const size_t base = ((size_t)bh * L + j0) * d;
  const float* om = omega + (size_t)h * M * d;
  const float* Rn = R + (((size_t)bh * nch + (causal ? c : 0)) * F) * dv;
  for (int i = threadIdx.x; i < kChunk * d; i += blockDim.x) {
    const bool ok = i < nj * d;
    sk[i] = ok ? k[base + i] : 0.f;
    sv[i] = ok ? v[base + i] : 0.f;
    sq[i] = (ok && causal) ? q[base + i] : 0.f;
  }
  for (int p = threadIdx.x; p < kChunk * dv; p += blockDim.x)
    se[p] = (causal && p < nj * dv) ? E[((size_t)bh * L + j0) * dv + p] : 0.f;
  for (int i = threadIdx.x; i < kChunk * kChunk; i += blockDim.x) A[i] = 0.f;
  __syncthreads();
  if (threadIdx.x < kChunk) {
    const int j = threadIdx.x;
    sw[j] = j < nj ? key_weight(kind, sk + j * d, d, cmax[bh]) : 0.f;
  }
  __syncthreads();
  const int nft = (F + kFeatTile - 1) / kFeatTile;
  if (causal) {
    // B_ij = [v_j | 1] . e_i (j <= i), and A_ij = psi(q_i) . psi(k_j) over all features
    for (int p = threadIdx.x; p < kChunk * kChunk; p += blockDim.x) {
      const int i = p / kChunk, j = p % kChunk;
      float s = 0.f;
      if (j <= i) {
        s = se[i * dv + d];
        for (int n = 0; n < d; ++n) s = fmaf(sv[j * d + n], se[i * dv + n], s);
      }
      Bm[p] = s;
    }
    for (int ft = 0; ft < nft; ++ft) {
      __syncthreads();
      for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
        const int j = p / kFeatTile, f = ft * kFeatTile + p % kFeatTile;
        float a = 0.f, b = 0.f, da, db;
        if (j < nj && f < F) {
          feature_pair(kind, M, f, sq + j * d, om, d, 1.f, a, da);
          feature_pair(kind, M, f, sk + j * d, om, d, sw[j], b, db);
        }
        pq[p] = a;
        pk[p] = b;
      }
      __syncthreads();
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
  const int tj = threadIdx.x >> 2, tn = threadIdx.x & 3;
  float kacc[kCols], vacc[kCols];
#pragma unroll
  for (int m = 0; m < kCols; ++m) kacc[m] = vacc[m] = 0.f;
  float scal = 0.f;
  for (int ft = 0; ft < nft; ++ft) {
    __syncthreads();
    for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
      const int j = p / kFeatTile, f = ft * kFeatTile + p % kFeatTile;
      float a = 0.f, b = 0.f, db = 0.f, da;
      if (j < nj && f < F) {
        feature_pair(kind, M, f, sk + j * d, om, d, sw[j], b, db);
        if (causal) feature_pair(kind, M, f, sq + j * d, om, d, 1.f, a, da);
      }
      pk[p] = b;
      dkd[p] = db;
      pq[p] = a;
    }
    for (int p = threadIdx.x; p < kFeatTile * dv; p += blockDim.x) {
      const int f = ft * kFeatTile + p / dv;
      sR[p] = f < F ? Rn[(size_t)f * dv + p % dv] : 0.f;
    }
    load_omega_tile(sOm, om, ft, F, M, d, kind);
    __syncthreads();
    // h[j][fl] = R_tile[fl] . [v_j | 1]  (+ sum_{i >= j} B_ij psi_fl(q_i))
    for (int p = threadIdx.x; p < kChunk * kFeatTile; p += blockDim.x) {
      const int j = p / kFeatTile, fl = p % kFeatTile;
      float s = sR[fl * dv + d];
      for (int n = 0; n < d; ++n) s = fmaf(sR[fl * dv + n], sv[j * d + n], s);
      if (causal)
        for (int i = j; i < kChunk; ++i) s = fmaf(Bm[i * kChunk + j], pq[i * kFeatTile + fl], s);
      sh[p] = s;
    }
    __syncthreads();
    for (int fl = tn; fl < kFeatTile; fl += 4) scal = fmaf(sh[tj * kFeatTile + fl], pk[tj * kFeatTile + fl], scal);
#pragma unroll
    for (int m = 0; m < kCols; ++m) {
      const int t = tn + 4 * m;
      if (t < d) {
        float sk_ = kacc[m], sv_ = vacc[m];
        for (int fl = 0; fl < kFeatTile; ++fl) {
          sk_ = fmaf(sh[tj * kFeatTile + fl] * dkd[tj * kFeatTile + fl], sOm[fl * d + t], sk_);
          sv_ = fmaf(sR[fl * dv + t], pk[tj * kFeatTile + fl], sv_);
        }
        kacc[m] = sk_;
        vacc[m] = sv_;
      }
    }
  }
  if (causal) {  // dv_j += sum_{i >= j} A_ij e_i[:d]
#pragma unroll
    for (int m = 0; m < kCols; ++m) {
      const int t = tn + 4 * m;
      if (t < d) {
        float s = vacc[m];
        for (int i = tj; i < kChunk; ++i) s = fmaf(A[i * kChunk + tj], se[i * dv + t], s);
        vacc[m] = s;
      }
    }
  }
  scal += __shfl_xor_sync(0xffffffffu, scal, 1);
  scal += __shfl_xor_sync(0xffffffffu, scal, 2);
  if (tj < nj) {
#pragma unroll
    for (int m = 0; m < kCols; ++m) {
      const int t = tn + 4 * m;
      if (t < d) {
        dk[base + (size_t)tj * d + t] = (kind == 0 ? sk[tj * d + t] * scal : 0.f) + kacc[m];
        dvout[base + (size_t)tj * d + t] = vacc[m];
      }
    }
  }
}

}  // namespace bwd
}  // namespace favor
