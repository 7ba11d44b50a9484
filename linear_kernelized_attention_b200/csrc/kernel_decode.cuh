// kernel_decode.cuh - one causal FAVOR decode step with a carried state.
//
// What it computes. The explainer page "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？",
// section 核心机制：FAVOR+: the causal prefix sums S_t = S_{t-1} + phi(k_t) v_t^T and
// z_t = z_{t-1} + phi(k_t), read by the query of the same token: out_t = phi(q_t) S_t / phi(q_t) z_t.
// One launch advances every (batch, head) by one token. From an empty state, calls on tokens
// 0 .. L-1 return the causal rows 0 .. L-1.
//
// State, per head h of BH: S_h [F, d] fp32, z_h [F] fp32 and a reference c_h (fp32). The three
// live in three consecutive regions: all S, then all z, then all c. Trig features carry the
// weight exp(|k|^2/2 - c) with c the running max of |k|^2/2 (-inf for an empty state), and S, z
// are rescaled by exp(c_old - c_new) when c grows. Factors that cancel between numerator and
// denominator (1/sqrt(M), exp(|q|^2/2)) are dropped. ReLU features have unit weight and c is
// left untouched. sin, cos and exp are evaluated in double and rounded to fp32 (the library is
// built with fast single-precision intrinsics, which lose accuracy on large angles).
//
// Work split. A cluster of G CTAs serves one head; CTA r owns the angles [r*na, (r+1)*na) and
// with them the state rows m (cos / ReLU) and M + m (sin): two contiguous row ranges, cut into
// chunks of 16 KB. The step is a matrix-vector product over the state, so it is HBM-bound and
// runs on CUDA cores; what decides its speed is keeping the state's reads in flight:
//   1. At entry, one thread starts bulk copies (cp.async.bulk) of the first kStages chunks
//      into a ring of shared-memory stages. They fly while the CTA loads the token, projects
//      its angles and builds its features.
//   2. Chunk by chunk, every thread rescales and adds its rows (S = rho S + w phi(k) v^T),
//      stores them to HBM with 16-byte stores and accumulates phi(q).S. Thread t holds
//      columns [4(t mod d/4), +4) of rows t div (d/4), + 256/(d/4), ... of the chunk. Once every
//      thread is past a stage, the next chunk's copy is started into it.
//   3. Rank 0 sums the G partial numerators and denominators through distributed shared memory
//      and writes the row.
// Every wait on a stage is bounded; on a timeout the CTA stops streaming, records
// FAVOR_ERR_TIMEOUT, lets the copies it started land (again bounded) and finishes.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace favor {
namespace dec {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxD = 128;
constexpr int kMaxRows = 1024;  // state rows one CTA holds (2 * 512 trig angles)
constexpr int kMaxG = 8;
constexpr int kZPerThread = kMaxRows / kThreads;
constexpr int kGroups = kThreads / 8;  // angles per projection pass
constexpr int kProjBatch = 4;          // projection passes whose omega loads are issued together
constexpr int kStages = 3;             // shared-memory ring for the state rows
constexpr int kStageBytes = 16384;
constexpr int kSmemBytes = kStages * kStageBytes;  // dynamic shared memory per CTA

// State row of local row i: the CTA's cos (or ReLU) rows m0 .. m0+na-1, then its sin rows.
__device__ __forceinline__ int local_row(int i, int na, int m0, int M) {
  return i < na ? m0 + i : M + m0 + (i - na);
}

struct DecodeParams {
  long long z_off;  // float offset of the z region (BH * F * d)
  long long c_off;  // float offset of the references (BH * F * (d + 1))
  int BH, H, d, M, kind, G, na;
};

// Chunk c of a CTA's rows: local rows [lrow, lrow + cnt), state rows [grow, grow + cnt).
struct Chunk {
  int lrow, grow, cnt;
};
template <int CR>
__device__ __forceinline__ Chunk chunk_of(int c, int ncos, int na, int m0, int M) {
  const bool sin_rows = c >= ncos;
  const int kk = sin_rows ? c - ncos : c;
  Chunk ch;
  ch.cnt = min(CR, na - kk * CR);
  ch.lrow = (sin_rows ? na : 0) + kk * CR;
  ch.grow = (sin_rows ? M : 0) + m0 + kk * CR;
  return ch;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 3) k_decode_step(const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            const __nv_bfloat16* __restrict__ v,
                                                            const __nv_bfloat16* __restrict__ omega,
                                                            float* __restrict__ state,
                                                            __nv_bfloat16* __restrict__ out,
                                                            const DecodeParams p) {
  static_assert(D == 16 || D == 32 || D == 64 || D == 128, "d must be 16, 32, 64 or 128");
  constexpr int d = D, d4 = D / 4, RP = kThreads / d4, kSlots = (D + 63) / 64;
  constexpr int CR = kStageBytes / (D * 4);  // rows per chunk
  constexpr int PB = D == 128 ? kProjBatch / 2 : kProjBatch;  // keeps d = 128 within registers
  extern __shared__ __align__(128) float ring[];  // kStages x kStageBytes
  __shared__ __align__(16) float sq[kMaxD], sk[kMaxD], sv[kMaxD];
  __shared__ float sa[kMaxRows], sb[kMaxRows];       // local row i: key coefficient, query feature
  __shared__ __align__(16) float red[kThreads * 4];  // [rows per pass][d] partial numerators
  __shared__ __align__(16) float part[kMaxD + 4];    // this CTA's numerator; [d] = denominator
  __shared__ __align__(16) float tot[kMaxD + 4];
  __shared__ float wden[kWarps];
  __shared__ float sc[3];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G, M = p.M;
  const int rank = static_cast<int>(cluster_ctarank());
  const int bh = blockIdx.x / G, h = bh % p.H;
  const bool trig = p.kind == 0;
  const int F = trig ? 2 * M : M;
  const int m0 = rank * p.na;
  const int na = max(0, min(M, m0 + p.na) - m0);
  const int nrows = trig ? 2 * na : na;
  const int ncos = (na + CR - 1) / CR;
  const int nch = trig ? 2 * ncos : ncos;
  float* __restrict__ S = state + (size_t)bh * F * d;
  float* __restrict__ z = state + p.z_off + (size_t)bh * F;
  float* cref = state + p.c_off + bh;

  auto issue = [&](int c) {  // one thread: bulk copy of chunk c into stage c % kStages
    const Chunk ch = chunk_of<CR>(c, ncos, na, m0, M);
    const uint32_t bar = smem_u32(&full[c % kStages]);
    const uint32_t bytes = static_cast<uint32_t>(ch.cnt * d * 4);
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(smem_u32(ring + (c % kStages) * (kStageBytes / 4)), S + (size_t)ch.grow * d, bytes, bar);
  };
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&full[s]), 1);
    abort_flag = 0;
    fence_mbar_init();
    for (int c = 0; c < min(kStages, nch); ++c) issue(c);
  }
  float zr[kZPerThread];
#pragma unroll
  for (int u = 0; u < kZPerThread; ++u) {
    const int i = tid + u * kThreads;
    zr[u] = i < nrows ? z[local_row(i, na, m0, M)] : 0.f;
  }
  for (int i = tid; i < d; i += kThreads) {
    const size_t o = (size_t)bh * d + i;
    sq[i] = __bfloat162float(q[o]);
    sk[i] = __bfloat162float(k[o]);
    sv[i] = __bfloat162float(v[o]);
  }
  __syncthreads();
  if (warp == 0) {
    float a = 0.f;
    for (int i = lane; i < d; i += 32) a = fmaf(sk[i], sk[i], a);
#pragma unroll
    for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) {
      float wk = 1.f, rho = 1.f, cnew = 0.f;
      if (trig) {
        const float n2 = 0.5f * a, cold = *cref;
        cnew = fmaxf(cold, n2);
        wk = static_cast<float>(exp(static_cast<double>(n2) - cnew));
        rho = static_cast<float>(exp(static_cast<double>(cold) - cnew));  // 0 for an empty state
      }
      sc[0] = wk;
      sc[1] = rho;
      sc[2] = cnew;
    }
  }
  // Projections: 8 lanes per angle (kGroups angles per pass), 8 bf16 of omega per lane and load,
  // PB passes' loads in flight at once.
  {
    const int sub = lane & 7, grp = tid >> 3;
    const __nv_bfloat16* om = omega + ((size_t)h * M + m0) * d;
    const int npass = (na + kGroups - 1) / kGroups;
    for (int p0 = 0; p0 < npass; p0 += PB) {
      uint4 w[PB][kSlots];
#pragma unroll
      for (int pp = 0; pp < PB; ++pp) {
        const int j = (p0 + pp) * kGroups + grp;
#pragma unroll
        for (int es = 0; es < kSlots; ++es) {
          const int e = 8 * sub + 64 * es;
          w[pp][es] = (j < na && e < d) ? *reinterpret_cast<const uint4*>(om + (size_t)j * d + e)
                                        : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // After the group's reduction every lane holds each pass's two projections; lane `sub`
      // keeps value sub of the 2 * PB (pass sub / 2; k if sub is even, q if odd) and turns it into
      // features, so the group's sin/cos run in parallel.
      float mine = 0.f;
#pragma unroll
      for (int pp = 0; pp < PB; ++pp) {
        float uk = 0.f, uq = 0.f;
#pragma unroll
        for (int es = 0; es < kSlots; ++es) {
          const int e = 8 * sub + 64 * es;
          if (e < d) {
            const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&w[pp][es]);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 x = __bfloat1622float2(w2[t]);
              uk = fmaf(x.x, sk[e + 2 * t], fmaf(x.y, sk[e + 2 * t + 1], uk));
              uq = fmaf(x.x, sq[e + 2 * t], fmaf(x.y, sq[e + 2 * t + 1], uq));
            }
          }
        }
#pragma unroll
        for (int o = 4; o; o >>= 1) {
          uk += __shfl_xor_sync(0xffffffffu, uk, o);
          uq += __shfl_xor_sync(0xffffffffu, uq, o);
        }
        if (sub == 2 * pp) mine = uk;
        if (sub == 2 * pp + 1) mine = uq;
      }
      const int j = (p0 + (sub >> 1)) * kGroups + grp;
      if ((sub >> 1) < PB && j < na) {
        float* dst = (sub & 1) ? sb : sa;
        if (trig) {
          double sn, cs;
          sincos(static_cast<double>(mine), &sn, &cs);
          dst[j] = static_cast<float>(cs);
          dst[na + j] = static_cast<float>(sn);
        } else {
          dst[j] = fmaxf(mine, 0.f);
        }
      }
    }
  }
  __syncthreads();
  const float wk = sc[0], rho = sc[1];

  // Stream the chunks through the ring.
  const int c4 = tid % d4, r0 = tid / d4;
  const float4 v4 = reinterpret_cast<const float4*>(sv)[c4];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int c = 0;
  for (; c < nch; ++c) {
    const int s = c % kStages;
    const bool ok = mbar_wait(smem_u32(&full[s]), (c / kStages) & 1, &abort_flag);
    if (ok) {
      const Chunk ch = chunk_of<CR>(c, ncos, na, m0, M);
      const float* st = ring + s * (kStageBytes / 4);
#pragma unroll 4
      for (int r = r0; r < ch.cnt; r += RP) {
        const int i = ch.lrow + r;
        const float a = wk * sa[i], b = sb[i];
        float4 t = reinterpret_cast<const float4*>(st + r * d)[c4];
        t.x = fmaf(t.x, rho, a * v4.x);
        t.y = fmaf(t.y, rho, a * v4.y);
        t.z = fmaf(t.z, rho, a * v4.z);
        t.w = fmaf(t.w, rho, a * v4.w);
        reinterpret_cast<float4*>(S + (size_t)(ch.grow + r) * d)[c4] = t;
        acc.x = fmaf(b, t.x, acc.x);
        acc.y = fmaf(b, t.y, acc.y);
        acc.z = fmaf(b, t.z, acc.z);
        acc.w = fmaf(b, t.w, acc.w);
      }
    }
    // Every thread is past stage s (or a wait gave up, and all stop together).
    if (__syncthreads_or(!ok)) break;
    if (tid == 0 && c + kStages < nch) issue(c + kStages);
  }
  if (c < nch && tid == 0) {
    // Stopped early: let the copies already started land before the CTA can exit.
    for (int cc = c; cc < min(nch, c + kStages); ++cc)
      mbar_wait(smem_u32(&full[cc % kStages]), (cc / kStages) & 1, nullptr, kWaitLimitCycles / 8);
  }

  // z rows, and phi(q).z
  float dz = 0.f;
#pragma unroll
  for (int u = 0; u < kZPerThread; ++u) {
    const int i = tid + u * kThreads;
    if (i < nrows) {
      const float t = fmaf(zr[u], rho, wk * sa[i]);
      z[local_row(i, na, m0, M)] = t;
      dz = fmaf(sb[i], t, dz);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) dz += __shfl_xor_sync(0xffffffffu, dz, o);
  if (lane == 0) wden[warp] = dz;
  reinterpret_cast<float4*>(red)[r0 * d4 + c4] = acc;
  __syncthreads();
  for (int n = tid; n < d + 4; n += kThreads) {
    float t = 0.f;
    if (n < d) {
      for (int r = 0; r < RP; ++r) t += red[r * d + n];
    } else if (n == d) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) t += wden[w];
    }
    part[n] = t;
  }
  // Every CTA's partial is in its shared memory; rank 0 sums them. A cluster barrier (its release
  // waits for this CTA's HBM stores) is taken only when there is another CTA to read from.
  if (G > 1)
    cluster_sync();
  else
    __syncthreads();
  if (rank == 0) {
    if (tid <= d4) {
      float4 t = reinterpret_cast<const float4*>(part)[tid];
      const uint32_t a = smem_u32(&part[4 * tid]);
      for (int r = 1; r < G; ++r) {
        const float4 x = ld_dsmem_f4(mapa_shared(a, r));
        t.x += x.x;
        t.y += x.y;
        t.z += x.z;
        t.w += x.w;
      }
      reinterpret_cast<float4*>(tot)[tid] = t;
    }
    __syncthreads();
    const float den = tot[d];
    const float inv = den != 0.f ? 1.f / den : 0.f;
    for (int n = tid; n < d; n += kThreads)
      out[(size_t)bh * d + n] = __float2bfloat16_rn(den != 0.f ? tot[n] * inv : 0.f);
    if (tid == 0 && trig) *cref = sc[2];  // every CTA of the cluster read c before the barrier
  }
  // The other CTAs keep their shared memory until rank 0 has read it.
  if (G > 1) cluster_sync();
}

// Empty state: S = 0, z = 0 and every reference -inf.
__global__ void k_decode_init(float* __restrict__ state, long long n_sz, long long BH) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_sz + BH; i += stride)
    state[i] = i < n_sz ? 0.f : -INFINITY;
}

}  // namespace dec
}  // namespace favor
