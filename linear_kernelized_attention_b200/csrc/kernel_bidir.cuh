// kernel_bidir.cuh - fused bidirectional FAVOR forward on sm_100a tensor cores.
//
// What it computes. The explainer page "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？",
// section 核心机制：FAVOR+, gives out = D_hat^-1 phi(Q) (phi(K)^T [V|1]). The state
// S = phi(K)^T [V|1] is aggregated first, then left-multiplied by phi(Q). No L x L matrix is
// formed.
//
// Structure. One thread-block cluster of P CTAs per (batch, head). CTA r of the cluster owns a
// contiguous run of 128-token tiles.
//   Key phase. Per tile and per 128-angle block a, and per 64-token half:
//     MMA1  U^T = Omega_a . K_half^T   (M=128 angles, N=64 tokens, K=64; bf16 in, fp32 in TMEM)
//     epilogue: w_j cos(U), w_j sin(U) (trig) or max(U, 0) (relu) -> bf16 -> TMEM, in place
//     MMA2  S_blk += phi^T . [V_half | 1]  (A from TMEM, B = V tile MN-major + a constant ones
//           column; M=128 features, N=80, K=64 tokens; fp32 in TMEM)
//     w_j = exp(|k_j|^2/2 - c). c is a running per-CTA reference kept 16 nats above the
//     largest |k|^2/2 seen. If a tile exceeds it, S is rescaled in TMEM before that tile.
//   Reduction. Each CTA writes its fp32 partial state and its c to scratch. After a cluster
//     barrier, CTA r sums feature rows [r F/P, (r+1) F/P) over the P partials in fixed order,
//     rescaled to the largest c. It writes them as an fp16 image under a power-of-two scale,
//     in the swizzled K-major layout the query phase's MMA reads. After a second barrier,
//     every CTA bulk-copies the whole image into shared memory. P = 1 skips the round trip.
//   Query phase. Per tile and per 64-angle chunk c:
//     MMA1  U = Q_tile . Omega_c^T  (M=128 tokens, N=64 angles)
//     epilogue: cos(U), sin(U) (trig) or max(U, 0) (relu) -> fp16 -> TMEM, in place. The
//     exp(|q|^2/2) and 1/sqrt(M) factors cancel.
//     MMA2  num += phi_c . S_c  (A from TMEM, B = image from shared memory; N=80)
//   then out = num[:, :64] / num[:, 64] -> bf16 -> swizzled staging -> TMA store.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer,
// warps 2-3 key norms (trig), warps 4-11 epilogue (two warpgroups; warp w reads TMEM lanes
// 32 (w % 4) .. +31, and warpgroup (w - 4) / 4 takes half of the columns).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace favor {
namespace tc {

constexpr int kTile = 128;               // tokens per tile
constexpr int kD = 64;                   // head dimension of this path
constexpr int kRowB = 128;               // bytes of one 64-element 16-bit row
constexpr int kTileB = kTile * kRowB;    // 16 KB
constexpr int kStagesK = 3;              // key-phase K+V stages
constexpr int kStagesQ = 2;              // query-phase Q stages
constexpr int kNumU = 3;                 // U ring buffers (64 TMEM columns each)
constexpr int kUBase = 320;              // first TMEM column of the U ring
constexpr int kNPad = 80;                // d + 1 padded to a multiple of 16
constexpr int kNV = kD + 1;              // value columns plus the normaliser column
constexpr int kImgAtomB = kNPad * kRowB; // bytes of one 64-feature atom of the state image
constexpr int kRegionB = 112 * 1024;     // shared region: key stages / image + Q stages
constexpr int kImgMaxB = 80 * 1024;
constexpr float kMargin = 16.f;          // stabiliser head-room, in nats
constexpr int kThreads = 384;

struct BidirParams {
  int BH, H, L, M;      // heads (B*H), heads per batch, tokens, random features
  int Mpad;             // M rounded up to a multiple of 128
  int P;                // CTAs per head (cluster size)
  int ntiles;           // ceil(L / 128)
  float* part;          // [BH][P][65][Fpad] fp32 partial states (P > 1)
  float* pmeta;         // [BH][P][2]: stabiliser reference, max |partial|
  uint8_t* image;       // [BH][natoms][80][128 B] fp16 state image (P > 1)
};

struct alignas(16) Misc {
  float wbuf[kStagesK][kTile];
  float rescale[4];
  float red[16];
  float cfinal;
  int abort_flag;
  uint32_t tmem_base;
  float pad0;
  uint64_t om_full;
  uint64_t kv_full[kStagesK], kv_empty[kStagesK], w_full[kStagesK];
  uint64_t u_full[kNumU], u_empty[kNumU], phi_full[kNumU];
  uint64_t s_done, img_full, mma_drain;
  uint64_t q_full[kStagesQ], q_empty[kStagesQ];
  uint64_t uq_full[kNumU], uq_empty[kNumU], phiq_full[kNumU];
  uint64_t num_full[2], num_empty[2];
  uint64_t epi_sync, help_sync;  // bounded group barriers (256 epilogue / 64 helper threads)
};
static_assert(sizeof(Misc) <= 4096, "misc block too large");

__host__ __device__ constexpr uint32_t bidir_smem_bytes(int Mpad) {
  return uint32_t(Mpad) * kRowB + kRegionB + 2 * kTileB + 2048 + 4096 + 1024;
}

// Feature row f of the key-phase state (TMEM block f / 128, lane f % 128) -> (atom, k) in the
// query-phase image. Trig: block 2a is cos and 2a+1 is sin of angles 128a..128a+127. The query
// phase orders chunk c (64 angles) as [cos 32 | sin 32 | cos 32 | sin 32].
template <int KIND>
__device__ __forceinline__ void feature_to_image(int f, int& atom, int& k) {
  if (KIND == 0) {
    const int blk = f >> 7, lane = f & 127, a = blk >> 1, s = blk & 1;
    const int r = a * 128 + lane;
    atom = 2 * (r >> 6) + ((r >> 5) & 1);
    k = s * 32 + (r & 31);
  } else {
    atom = f >> 6;
    k = f & 63;
  }
}
__device__ __forceinline__ uint32_t image_byte(int atom, int n, int k) {
  return uint32_t(atom) * kImgAtomB + uint32_t(n) * kRowB + ((uint32_t((k >> 3) ^ (n & 7))) << 4) +
         uint32_t(k & 7) * 2;
}

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    favor_bidir_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_om,
                   const __grid_constant__ CUtensorMap tm_out, const BidirParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t s_om = base;
  const uint32_t s_reg = base + uint32_t(p.Mpad) * kRowB;
  const uint32_t s_stage = s_reg + kRegionB;
  const uint32_t s_ones = s_stage + 2 * kTileB;
  Misc* ms = reinterpret_cast<Misc*>(gbase + (s_ones + 2048 - base));
  volatile int* abort_flag = &ms->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = p.P;
  const int rank = blockIdx.x % P;
  const int bh = blockIdx.x / P;
  const int h = bh % p.H;
  const int t_begin = rank * p.ntiles / P;
  const int my_tiles = (rank + 1) * p.ntiles / P - t_begin;
  const int nblk = p.Mpad / 128;               // key-phase angle blocks
  const int nsb = KIND == 0 ? 2 * nblk : nblk; // state blocks of 128 feature rows
  const int Fpad = nsb * 128;
  const int natoms = Fpad / 64;
  const int ipt = nblk * 2;                    // key-phase items per tile
  const int nchq = p.Mpad / 64;                // query-phase chunks per tile
  auto bar = [](uint64_t& b) { return smem_u32(&b); };

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    ms->abort_flag = 0;
    mbar_init(bar(ms->om_full), 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(bar(ms->kv_full[s]), 1);
      mbar_init(bar(ms->kv_empty[s]), KIND == 0 ? 3 : 1);
      mbar_init(bar(ms->w_full[s]), 64);
    }
    for (int b = 0; b < kNumU; ++b) {
      mbar_init(bar(ms->u_full[b]), 1);
      mbar_init(bar(ms->u_empty[b]), 1);
      mbar_init(bar(ms->phi_full[b]), 8);
      mbar_init(bar(ms->uq_full[b]), 1);
      mbar_init(bar(ms->uq_empty[b]), 1);
      mbar_init(bar(ms->phiq_full[b]), 8);
    }
    mbar_init(bar(ms->s_done), 1);
    mbar_init(bar(ms->img_full), 1);
    mbar_init(bar(ms->mma_drain), 1);
    for (int s = 0; s < kStagesQ; ++s) {
      mbar_init(bar(ms->q_full[s]), 1);
      mbar_init(bar(ms->q_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ms->num_full[s]), 1);
      mbar_init(bar(ms->num_empty[s]), 8);
    }
    mbar_init(bar(ms->epi_sync), 256);
    mbar_init(bar(ms->help_sync), 64);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish();
  }
  {  // ones column for [V | 1]: rows of 128 B, column 64 (first element of atom 1) = 1.0
    uint32_t* ones = reinterpret_cast<uint32_t*>(gbase + (s_ones - base));
    for (int i = tid; i < 512; i += kThreads) ones[i] = 0u;
    __syncthreads();
    if (tid < 16) {
      const int r = tid;
      reinterpret_cast<uint16_t*>(gbase + (s_ones - base) + r * kRowB + ((r & 7) << 4))[0] = 0x3F80u;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  // ================================================================ key phase
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(bar(ms->om_full), uint32_t(p.Mpad) * kRowB);
      for (int blk = 0; blk < nblk; ++blk)
        tma_load_3d(s_om + blk * kTileB, &tm_om, bar(ms->om_full), 0, blk * 128, h);
      for (int t = 0; t < my_tiles; ++t) {
        const int s = t % kStagesK, k = t / kStagesK;
        if (!mbar_wait(bar(ms->kv_empty[s]), (k & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(ms->kv_full[s]), 2 * kTileB);
        const int row = (t_begin + t) * kTile;
        tma_load_3d(s_reg + s * 2 * kTileB, &tm_k, bar(ms->kv_full[s]), 0, row, bh);
        tma_load_3d(s_reg + s * 2 * kTileB + kTileB, &tm_v, bar(ms->kv_full[s]), 0, row, bh);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id1 = idesc_f16(128, 64, 1, 1, 0, 0);
      const uint32_t id2 = idesc_f16(128, kNPad, 1, 1, 0, 1);
      const int n = my_tiles * ipt;
      bool ok = mbar_wait(bar(ms->om_full), 0, abort_flag);
      auto issue1 = [&](int j) -> bool {
        const int t = j / ipt, rem = j % ipt, a = rem >> 1, hh = rem & 1;
        const int s = t % kStagesK, b = j % kNumU;
        if (rem == 0 && !mbar_wait(bar(ms->kv_full[s]), (t / kStagesK) & 1, abort_flag)) return false;
        if (j >= kNumU && !mbar_wait(bar(ms->u_empty[b]), ((j / kNumU) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kUBase + b * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = sdesc_sw128(s_om + a * kTileB + kk * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(s_reg + s * 2 * kTileB + hh * 64 * kRowB + kk * 32, 16, 1024);
          mma_ss(d, ad, bd, id1, kk > 0);
        }
        mma_commit(bar(ms->u_full[b]));
        return true;
      };
      for (int j = 0; ok && j < n && j < kNumU; ++j) ok = issue1(j);
      for (int i = 0; ok && i < n; ++i) {
        const int t = i / ipt, rem = i % ipt, a = rem >> 1, hh = rem & 1;
        const int s = t % kStagesK, b = i % kNumU;
        if (!mbar_wait(bar(ms->phi_full[b]), (i / kNumU) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t vrow0 = s_reg + s * 2 * kTileB + kTileB + hh * 64 * kRowB;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t bstart = vrow0 + kk * 16 * kRowB;
          const uint64_t bd = sdesc_sw128(bstart, s_ones - bstart, 1024);
          const uint32_t acc = (t == 0 && hh == 0 && kk == 0) ? 0u : 1u;
          const uint32_t acol = kUBase + b * 64 + (kk < 2 ? kk * 8 : 32 + (kk - 2) * 8);
          if (KIND == 0) {
            mma_ts(tmem + (2 * a) * kNPad, tmem + acol, bd, id2, acc);
            mma_ts(tmem + (2 * a + 1) * kNPad, tmem + acol + 16, bd, id2, acc);
          } else {
            mma_ts(tmem + a * kNPad, tmem + acol, bd, id2, acc);
          }
        }
        mma_commit(bar(ms->u_empty[b]));
        if (rem == ipt - 1) mma_commit(bar(ms->kv_empty[s]));
        if (i + kNumU < n) ok = issue1(i + kNumU);
      }
      mma_commit(bar(ms->s_done));
    }
    __syncwarp();
  } else if (warp < 4) {
    if (KIND == 0) {  // key norms, tile maxima and the running stabiliser reference
      const int ht = tid - 64;
      uint32_t hph = 0;
      float cr = 0.f;
      for (int t = 0; t < my_tiles; ++t) {
        const int s = t % kStagesK;
        if (!mbar_wait(bar(ms->kv_full[s]), (t / kStagesK) & 1, abort_flag)) break;
        const uint8_t* kt = gbase + (s_reg - base) + s * 2 * kTileB;
        const int row0 = (t_begin + t) * kTile;
        float n2[2];
        bool valid[2];
        float m = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = ht + 64 * jj;
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 x = *reinterpret_cast<const uint4*>(kt + j * kRowB + ((c ^ (j & 7)) << 4));
            const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xFFFF0000u);
              acc = fmaf(lo, lo, acc);
              acc = fmaf(hi, hi, acc);
            }
          }
          n2[jj] = 0.5f * acc;
          valid[jj] = row0 + j < p.L;
          if (valid[jj]) m = fmaxf(m, n2[jj]);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) ms->red[warp - 2] = m;
        group_sync(bar(ms->help_sync), hph, abort_flag);
        m = fmaxf(ms->red[0], ms->red[1]);
        float f = 1.f;
        if (t == 0) {
          cr = m + kMargin;
        } else if (m > cr) {
          const float nc = m + kMargin;
          f = __expf(cr - nc);
          cr = nc;
        }
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
          ms->wbuf[s][ht + 64 * jj] = valid[jj] ? __expf(n2[jj] - cr) : 0.f;
        if (ht == 0) {
          ms->rescale[s] = f;
          if (t == my_tiles - 1) ms->cfinal = cr;
        }
        group_sync(bar(ms->help_sync), hph, abort_flag);
        mbar_arrive(bar(ms->w_full[s]));
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->kv_empty[s]));
      }
    }
  } else {
    // ------------------------------------------------------------ key-phase epilogue
    const int q4 = warp & 3, ch = (warp - 4) >> 2, row = q4 * 32 + lane;
    const uint32_t lane_addr = uint32_t(q4 * 32) << 16;
    const int n = my_tiles * ipt;
    for (int i = 0; i < n; ++i) {
      const int t = i / ipt, rem = i % ipt, a = rem >> 1, hh = rem & 1;
      const int s = t % kStagesK, b = i % kNumU;
      if (!mbar_wait(bar(ms->u_full[b]), (i / kNumU) & 1, abort_flag)) break;
      tc_fence_after();
      if (KIND == 0 && rem == 0) {
        if (!mbar_wait(bar(ms->w_full[s]), (t / kStagesK) & 1, abort_flag)) break;
        const float f = ms->rescale[s];
        if (f != 1.f) {  // the reference grew: rescale the accumulated state first
          if (i > 0 && !mbar_wait(bar(ms->u_empty[(i - 1) % kNumU]), ((i - 1) / kNumU) & 1, abort_flag))
            break;
          tc_fence_after();
          const int half = nsb * kNPad / 2;
          for (int c0 = ch * half; c0 < (ch + 1) * half; c0 += 8) {
            uint32_t r[8];
            tmem_ld8(tmem + lane_addr + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
            tmem_st8(tmem + lane_addr + c0, r);
          }
          tmem_wait_st();
        }
      }
      const uint32_t taddr = tmem + lane_addr + kUBase + b * 64 + ch * 32;
      uint32_t u[32];
      tmem_ld32(taddr, u);
      tmem_wait_ld();
      if (KIND == 0) {
        const bool valid = a * 128 + row < p.M;
        const float* wv = &ms->wbuf[s][hh * 64 + ch * 32];
        uint32_t cp[16], sp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float s0, c0, s1, c1;
          __sincosf(__uint_as_float(u[2 * j]), &s0, &c0);
          __sincosf(__uint_as_float(u[2 * j + 1]), &s1, &c1);
          const float w0 = valid ? wv[2 * j] : 0.f, w1 = valid ? wv[2 * j + 1] : 0.f;
          cp[j] = pack_bf16x2(w0 * c0, w1 * c1);
          sp[j] = pack_bf16x2(w0 * s0, w1 * s1);
        }
        tmem_st16(taddr, cp);
        tmem_st16(taddr + 16, sp);
      } else {
        uint32_t rp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          rp[j] = pack_bf16x2(fmaxf(__uint_as_float(u[2 * j]), 0.f), fmaxf(__uint_as_float(u[2 * j + 1]), 0.f));
        tmem_st16(taddr, rp);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->phi_full[b]));
    }
  }

  // ================================================================ state reduction
  const bool epi = warp >= 4;
  const int q4 = warp & 3, ch = (warp - 4) >> 2, row = q4 * 32 + lane;
  const uint32_t lane_addr = uint32_t(q4 * 32) << 16;
  const int etid = tid - 128;  // 0..255 for epilogue threads
  uint32_t eph = 0;            // phase of the epilogue group barrier
  if (epi) {
    if (mbar_wait(bar(ms->s_done), 0, abort_flag)) tc_fence_after();
  }
  if (P == 1) {
    if (epi) {
      float mx = 0.f;
      for (int blk = 0; blk < nsb; ++blk)
        for (int cc = 0; cc < 5; ++cc) {
          uint32_t r[8];
          tmem_ld8(tmem + lane_addr + blk * kNPad + ch * 40 + cc * 8, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (ch * 40 + cc * 8 + e < kNV) mx = fmaxf(mx, fabsf(__uint_as_float(r[e])));
        }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) ms->red[warp - 4] = mx;
      group_sync(bar(ms->epi_sync), eph, abort_flag);
      mx = 0.f;
      for (int w = 0; w < 8; ++w) mx = fmaxf(mx, ms->red[w]);
      const float scale = mx > 0.f ? ldexpf(1.f, 15 - (int)ceilf(log2f(mx))) : 1.f;
      uint8_t* img = gbase + (s_reg - base);
      for (int blk = 0; blk < nsb; ++blk) {
        int atom, k;
        feature_to_image<KIND>(blk * 128 + row, atom, k);
        for (int cc = 0; cc < 5; ++cc) {
          uint32_t r[8];
          tmem_ld8(tmem + lane_addr + blk * kNPad + ch * 40 + cc * 8, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int nn = ch * 40 + cc * 8 + e;
            const float v = nn < kNV ? __uint_as_float(r[e]) * scale : 0.f;
            *reinterpret_cast<__half*>(img + image_byte(atom, nn, k)) = __float2half_rn(v);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      group_sync(bar(ms->epi_sync), eph, abort_flag);
      if (etid == 0) mbar_arrive(bar(ms->img_full));
    }
  } else {
    float* part = p.part + (size_t)bh * P * kNV * Fpad;
    float* pmeta = p.pmeta + (size_t)bh * P * 2;
    if (epi) {
      float mx = 0.f;
      float* mine = part + (size_t)rank * kNV * Fpad;
      for (int blk = 0; blk < nsb; ++blk)
        for (int cc = 0; cc < 5; ++cc) {
          uint32_t r[8];
          tmem_ld8(tmem + lane_addr + blk * kNPad + ch * 40 + cc * 8, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int nn = ch * 40 + cc * 8 + e;
            if (nn < kNV) {
              const float v = __uint_as_float(r[e]);
              mine[(size_t)nn * Fpad + blk * 128 + row] = v;
              mx = fmaxf(mx, fabsf(v));
            }
          }
        }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) ms->red[warp - 4] = mx;
      tc_fence_before();
      group_sync(bar(ms->epi_sync), eph, abort_flag);
      if (etid == 0) {
        float m = 0.f;
        for (int w = 0; w < 8; ++w) m = fmaxf(m, ms->red[w]);
        pmeta[rank * 2 + 0] = KIND == 0 ? ms->cfinal : 0.f;
        pmeta[rank * 2 + 1] = m;
      }
    }
    cluster_sync();
    {  // owner reduction of feature rows [rank Fc, (rank + 1) Fc), all 384 threads
      float cmax = -INFINITY;
      for (int q = 0; q < P; ++q) cmax = fmaxf(cmax, pmeta[q * 2]);
      float bound = 0.f;
      for (int q = 0; q < P; ++q) bound += pmeta[q * 2 + 1] * (KIND == 0 ? __expf(pmeta[q * 2] - cmax) : 1.f);
      const float scale = bound > 0.f ? ldexpf(1.f, 15 - (int)ceilf(log2f(bound))) : 1.f;
      const int Fc = Fpad / P, f0 = rank * Fc;
      uint8_t* gimg = p.image + (size_t)bh * natoms * kImgAtomB;
      for (int idx = tid; idx < kNPad * Fc; idx += kThreads) {
        const int nn = idx / Fc, f = f0 + idx % Fc;
        float acc = 0.f;
        if (nn < kNV) {
          for (int q = 0; q < P; ++q) {
            const float sq = KIND == 0 ? __expf(pmeta[q * 2] - cmax) : 1.f;
            acc = fmaf(sq, part[((size_t)q * kNV + nn) * Fpad + f], acc);
          }
        }
        int atom, k;
        feature_to_image<KIND>(f, atom, k);
        *reinterpret_cast<__half*>(gimg + image_byte(atom, nn, k)) = __float2half_rn(acc * scale);
      }
      fence_proxy_async_global();
    }
    cluster_sync();
    if (warp == 0 && lane == 0 && !*abort_flag) {
      const uint32_t bytes = uint32_t(natoms) * kImgAtomB;
      mbar_arrive_expect_tx(bar(ms->img_full), bytes);
      bulk_load(s_reg, p.image + (size_t)bh * natoms * kImgAtomB, bytes, bar(ms->img_full));
    }
  }

  // ================================================================ query phase
  if (warp == 0) {
    if (lane == 0) {
      if (mbar_wait(bar(ms->s_done), 0, abort_flag)) {
        for (int t = 0; t < my_tiles; ++t) {
          const int s = t % kStagesQ, k = t / kStagesQ;
          if (!mbar_wait(bar(ms->q_empty[s]), (k & 1) ^ 1, abort_flag)) break;
          mbar_arrive_expect_tx(bar(ms->q_full[s]), kTileB);
          tma_load_3d(s_reg + kImgMaxB + s * kTileB, &tm_q, bar(ms->q_full[s]), 0,
                      (t_begin + t) * kTile, bh);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id1 = idesc_f16(128, 64, 1, 1, 0, 0);
      const uint32_t id2 = idesc_f16(128, kNPad, 0, 0, 0, 0);
      const int n = my_tiles * nchq;
      bool ok = mbar_wait(bar(ms->s_done), 0, abort_flag);
      auto issue1 = [&](int j) -> bool {
        const int t = j / nchq, c = j % nchq, s = t % kStagesQ, b = j % kNumU;
        if (c == 0 && !mbar_wait(bar(ms->q_full[s]), (t / kStagesQ) & 1, abort_flag)) return false;
        if (j >= kNumU && !mbar_wait(bar(ms->uq_empty[b]), ((j / kNumU) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = sdesc_sw128(s_reg + kImgMaxB + s * kTileB + kk * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(s_om + c * 64 * kRowB + kk * 32, 16, 1024);
          mma_ss(tmem + kUBase + b * 64, ad, bd, id1, kk > 0);
        }
        mma_commit(bar(ms->uq_full[b]));
        if (c == nchq - 1) mma_commit(bar(ms->q_empty[s]));
        return true;
      };
      for (int j = 0; ok && j < n && j < kNumU; ++j) ok = issue1(j);
      if (ok) ok = mbar_wait(bar(ms->img_full), 0, abort_flag);
      for (int i = 0; ok && i < n; ++i) {
        const int t = i / nchq, c = i % nchq, b = i % kNumU, nb = t & 1;
        if (!mbar_wait(bar(ms->phiq_full[b]), (i / kNumU) & 1, abort_flag)) { ok = false; break; }
        if (c == 0 && !mbar_wait(bar(ms->num_empty[nb]), ((t >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int ksteps = KIND == 0 ? 8 : 4;
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint32_t acol = KIND == 0 ? kk * 8 : (kk < 2 ? kk * 8 : 32 + (kk - 2) * 8);
          const int atom = KIND == 0 ? 2 * c + (kk >> 2) : c;
          const uint32_t koff = KIND == 0 ? (kk & 3) * 32 : kk * 32;
          const uint64_t bd = sdesc_sw128(s_reg + atom * kImgAtomB + koff, 16, 1024);
          mma_ts(tmem + nb * kNPad, tmem + kUBase + b * 64 + acol, bd, id2, (c > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(ms->uq_empty[b]));
        if (c == nchq - 1) mma_commit(bar(ms->num_full[nb]));
        if (i + kNumU < n) ok = issue1(i + kNumU);
      }
      mma_commit(bar(ms->mma_drain));
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int n = my_tiles * nchq;
    const bool issuer = (etid == 0);
    for (int i = 0; i < n; ++i) {
      const int t = i / nchq, c = i % nchq, b = i % kNumU;
      if (!mbar_wait(bar(ms->uq_full[b]), (i / kNumU) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + lane_addr + kUBase + b * 64 + ch * 32;
      uint32_t u[32];
      tmem_ld32(taddr, u);
      tmem_wait_ld();
      if (KIND == 0) {
        const int a0 = c * 64 + ch * 32;
        uint32_t cp[16], sp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float s0, c0, s1, c1;
          __sincosf(__uint_as_float(u[2 * j]), &s0, &c0);
          __sincosf(__uint_as_float(u[2 * j + 1]), &s1, &c1);
          const bool v0 = a0 + 2 * j < p.M, v1 = a0 + 2 * j + 1 < p.M;
          cp[j] = pack_f16x2(v0 ? c0 : 0.f, v1 ? c1 : 0.f);
          sp[j] = pack_f16x2(v0 ? s0 : 0.f, v1 ? s1 : 0.f);
        }
        tmem_st16(taddr, cp);
        tmem_st16(taddr + 16, sp);
      } else {
        uint32_t rp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          rp[j] = pack_f16x2(fmaxf(__uint_as_float(u[2 * j]), 0.f), fmaxf(__uint_as_float(u[2 * j + 1]), 0.f));
        tmem_st16(taddr, rp);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->phiq_full[b]));

      if (c == nchq - 1) {  // the tile's numerator is complete: normalise and store
        const int nb = t & 1;
        if (!mbar_wait(bar(ms->num_full[nb]), (t >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        uint32_t nv[32], dv;
        tmem_ld32(tmem + lane_addr + nb * kNPad + ch * 32, nv);
        tmem_ld1(tmem + lane_addr + nb * kNPad + 64, dv);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->num_empty[nb]));
        const float den = __uint_as_float(dv);
        const float inv = den != 0.f ? 1.f / den : 0.f;
        uint32_t o[16];
#pragma unroll
        for (int m = 0; m < 16; ++m)
          o[m] = pack_bf16x2(__uint_as_float(nv[2 * m]) * inv, __uint_as_float(nv[2 * m + 1]) * inv);
        const int sb = t & 1;
        if (issuer && t >= 2) bulk_wait_read1();
        group_sync(bar(ms->epi_sync), eph, abort_flag);
        uint8_t* stg = gbase + (s_stage - base) + sb * kTileB + row * kRowB;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int chunk = ch * 4 + m;
          *reinterpret_cast<uint4*>(stg + ((chunk ^ (row & 7)) << 4)) =
              make_uint4(o[4 * m], o[4 * m + 1], o[4 * m + 2], o[4 * m + 3]);
        }
        fence_proxy_async_smem();
        group_sync(bar(ms->epi_sync), eph, abort_flag);
        if (issuer) {
          tma_store_3d(&tm_out, s_stage + sb * kTileB, 0, (t_begin + t) * kTile, bh);
          bulk_commit();
        }
      }
    }
    if (issuer) bulk_wait0();
  }

  // ================================================================ teardown
  if (warp == 1) mbar_wait(bar(ms->mma_drain), 0, nullptr, 200000000ll);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace favor
