// kernel_bidir_split.cuh - bidirectional FAVOR forward on sm_100a tensor cores, as three
// launches that spread the work over every SM.
//
// What it computes. The explainer page "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？",
// section 核心机制：FAVOR+: out = D_hat^-1 phi(Q) (phi(K)^T [V|1]). The state S = phi(K)^T [V|1]
// is aggregated first and then left-multiplied by phi(Q); no L x L matrix is formed.
//
// 1. k_bidir_state: key-side partial states. The work is the list of units (pair, tile) with
//    pair = (head, 128-angle block) and tile = 128 keys, cut into one contiguous run per CTA
//    (one CTA per SM), so every SM gets the same number of tiles whatever B*H is. Per 64-key
//    item of a tile:
//      MMA1  U^T = Omega_a K_item^T    (M = 128 angles, N = 64 keys, K = head dim; bf16 -> fp32 TMEM)
//      epilogue: cos/sin (trig) or max(., 0) (ReLU) of U^T -> bf16, in place in TMEM
//      MMA2  S_blk += phi^T [w o V | w]  (A = phi^T from TMEM, B = the V tile plus a column
//            buffer, MN-major; M = 128 feature rows, N = d_pad + 16, K = 16 keys per instruction)
//    Trig keys carry w_j = exp(|k_j|^2/2 - c), the exp(|x|^2/2) factor of the trig map with a
//    running reference c kept 16 nats above the largest |k|^2/2 seen in the run; four warps
//    compute the norms and fold w_j into row j of the V tile. When c grows, S is rescaled in
//    TMEM first. At the end of a run of tiles of one pair, S (fp32) and (c, max |S|) go to a
//    workspace slot.
// 2. k_bidir_merge: per pair and 32 state rows, the slots are summed at the head's largest
//    reference and rounded to the query-side operand type: fp16 under a power-of-two scale
//    taken from the slots' bounds (trig), or bf16 (ReLU). The result is written in the
//    swizzled K-major layout the query kernel's MMA reads, so one bulk copy places it.
// 3. k_bidir_query: units (head, tile) cut into one run per CTA. Per 128-angle block of a
//    128-query tile:
//      MMA1  U = Q_tile Omega_ab^T      (M = 128 queries, N = 128 angles)
//      epilogue: cos/sin or max(., 0) -> fp16/bf16 in place in TMEM (the exp(|q|^2/2) and
//            1/sqrt(M) factors cancel between numerator and denominator)
//      MMA2  num += phi_ab S_ab          (A from TMEM, B = the state image; N = d_pad + 16)
//    then out = num[:, :d] / num[:, d_pad] -> bf16 -> swizzled staging -> TMA store.
//
// Head sizes d = 16, 32, 64 are carried in 64-column boxes (the TMA box reads zeros past d and
// the output store clips them); d = 128 uses two boxes.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "sincos_poly.cuh"

namespace favor {
namespace bs {

constexpr int kTile = 128;          // tokens per tile
constexpr int kRowB = 128;          // one 64-element 16-bit row
constexpr int kBoxB = 128 * kRowB;  // one TMA box: 128 rows x 64 elements
constexpr float kMargin = 16.f;     // stabiliser head-room above the largest |k|^2/2 seen (nats)
constexpr int kThreads = 512;

// Angles of 8 consecutive ones evaluated on the FMA pipe (bit j set: angle j of the group);
// the rest go to the SFU. With the projections issued by their own warp the feature warps are
// busy enough for the SFU to matter: 0x11 (two angles in eight on the FMA pipe) measured fastest,
// ahead of 0x00, 0x01, 0x15, 0x41 and 0x55.
#ifndef FAVOR_POLY_MASK
#define FAVOR_POLY_MASK 0x11u
#endif
constexpr uint32_t kPolyMask = FAVOR_POLY_MASK;

// Contiguous runs of units: CTA i owns units [floor(i U / P), floor((i + 1) U / P)).
__host__ __device__ inline long long run_begin(long long i, long long U, long long P) { return i * U / P; }
__host__ __device__ inline long long cta_of_unit(long long x, long long U, long long P) {
  return ((x + 1) * P - 1) / U;
}

// Position of a tile in a CTA's run: the run starts tt0 tiles into its first pair (or head); the
// walker advances tile by tile with no division, so the issuing warps never evaluate 64-bit
// quotients in their loops.
struct RunWalker {
  int t, k, tt;   // tile of the run, pair (head) index within the run, tile within that pair
  int n, nt;      // tiles in the run, tiles per pair
  __device__ __forceinline__ RunWalker(int tt0, int n_, int nt_) : t(0), k(0), tt(tt0), n(n_), nt(nt_) {}
  __device__ __forceinline__ void advance_to(int t_new) {
    while (t < t_new) {
      ++t;
      if (++tt == nt) {
        tt = 0;
        ++k;
      }
    }
  }
  __device__ __forceinline__ bool first() const { return t == 0 || tt == 0; }
  __device__ __forceinline__ bool last() const { return t == n - 1 || tt == nt - 1; }
};

// ============================================================================ key states
template <int KIND, int DP>
struct StateCfg {
  static constexpr int NCB = DP / 64;                        // 64-column boxes of a row
  static constexpr int NV = DP + 16;                         // MMA2 N: values, normaliser (column DP), pad
  static constexpr int NSB = KIND == 0 ? 2 : 1;              // 128-row state blocks (trig: cos, sin)
  static constexpr int R = 128 * NSB;                        // state rows of a pair
  static constexpr int NBUF = (KIND == 0 && DP == 128) ? 3 : 5;  // 64-key U/phi buffers
  static constexpr int NS = DP == 64 ? 4 : 2;                // K/V stages
  static constexpr int NG = KIND == 0 ? 3 : 2;               // feature groups of four warps (trig: SFU-heavy)
  static constexpr int kThreads = 256 + 128 * NG;             // warps 0-7, then the feature groups
  static constexpr int kStageB = (2 * NCB + 1) * kBoxB;      // V boxes | column box | K boxes
  static constexpr int kOmB = NCB * kBoxB;                   // one Omega block
  static constexpr int kUcol = (NSB * NV + 31) / 32 * 32;    // TMEM column of the U ring
  static constexpr int kMiscOff = 2 * kOmB + NS * kStageB;
  static constexpr int kSmem = kMiscOff + 1024 + 1024;       // misc block + alignment slack
  static_assert(kUcol + NBUF * 64 <= 512, "TMEM budget");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct StateParams {
  int H, L, M;
  int nab;        // 128-angle blocks
  int ntiles;     // 128-key tiles per head
  long long units;  // B * H * nab * ntiles
  int smax;       // workspace slots per pair
  float* part;    // [pair * smax + slot][d_pad + 1][R] fp32
  float* meta;    // [pair * smax + slot][2]: reference c (trig), max |entry|
};

struct alignas(16) StateMisc {
  int abort_flag;
  uint32_t tmem_base;
  float tmax[2][4];
  float frescale[4];  // by stage
  float redmax[2][8];
  uint64_t om_full[2], om_free[2];
  uint64_t kv_full[4], kv_empty[4], w_full[4];
  uint64_t u_full[5], p_full[5], buf_free[5];
  uint64_t s_done, s_free, drain;
  uint64_t norm_sync;  // bounded barrier among the 128 norm threads
};
static_assert(sizeof(StateMisc) <= 1024, "misc block");

template <int KIND, int DP>
__global__ void __launch_bounds__(StateCfg<KIND, DP>::kThreads, 1)
    k_bidir_state(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_om, const StateParams p) {
  using C = StateCfg<KIND, DP>;
  constexpr int NCB = C::NCB, NV = C::NV, NSB = C::NSB, R = C::R, NBUF = C::NBUF, NS = C::NS, NG = C::NG;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (base - raw);
  const uint32_t s_om = base, s_stage = base + 2 * C::kOmB;
  StateMisc* ms = reinterpret_cast<StateMisc*>(gb + C::kMiscOff);
  volatile int* abort_flag = &ms->abort_flag;
  auto bar = [](uint64_t& b) { return smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long P = gridDim.x, U = p.units;
  const long long u0 = run_begin(blockIdx.x, U, P), u1 = run_begin(blockIdx.x + 1, U, P);
  const int n = (int)(u1 - u0);  // tiles of this CTA
  const int nt = p.ntiles;
  const long long p0 = u0 / nt;  // first pair of the run
  const int tt0 = (int)(u0 - p0 * nt);
  auto slot_of = [&](long long pr) {
    return pr * p.smax + (blockIdx.x - cta_of_unit(pr * nt, U, P));
  };

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    ms->abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(ms->om_full[i]), 1);
      mbar_init(bar(ms->om_free[i]), 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(ms->kv_full[s]), 1);
      mbar_init(bar(ms->kv_empty[s]), 1);
      mbar_init(bar(ms->w_full[s]), 4);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(bar(ms->u_full[b]), 1);
      mbar_init(bar(ms->p_full[b]), 4);
      mbar_init(bar(ms->buf_free[b]), 1);
    }
    mbar_init(bar(ms->s_done), 1);
    mbar_init(bar(ms->s_free), 8);
    mbar_init(bar(ms->drain), 1);
    mbar_init(bar(ms->norm_sync), 128);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish();
  }
  {  // column boxes: zero, with the normaliser column (element 0 of each row) 1.0 for ReLU
    for (int s = 0; s < NS; ++s) {
      uint4* col = reinterpret_cast<uint4*>(gb + (s_stage - base) + s * C::kStageB + NCB * kBoxB);
      for (int i = tid; i < kBoxB / 16; i += C::kThreads) col[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    if (KIND == 1 && tid < kTile)
      for (int s = 0; s < NS; ++s)
        *reinterpret_cast<uint16_t*>(gb + (s_stage - base) + s * C::kStageB + NCB * kBoxB + tid * kRowB +
                                     ((tid & 7) << 4)) = 0x3F80u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  pdl_launch_dependents();  // the merge may be scheduled; it waits for this grid's results

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (whole warp; the
    // elected lane issues the copies)
    if (n > 0) {
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_om);
      }
      int issued = 0, pk_issued = 0;
      RunWalker w(tt0, n, nt);
      int bh = 0, ab = 0, h = 0;
      for (int t = 0; t < n; ++t) {
        w.advance_to(t);
        const int pk = w.k;
        if (w.first()) {
          const int pr = (int)(p0 + pk);
          bh = pr / p.nab;
          ab = pr - bh * p.nab;
          h = bh % p.H;
          if (pk >= 2 && !mbar_wait(bar(ms->om_free[pk & 1]), ((pk >> 1) - 1) & 1, abort_flag)) break;
          if (leader) {
            mbar_arrive_expect_tx(bar(ms->om_full[pk & 1]), C::kOmB);
            for (int kb = 0; kb < NCB; ++kb)
              tma_load_3d(s_om + (pk & 1) * C::kOmB + kb * kBoxB, &tm_om, bar(ms->om_full[pk & 1]), kb * 64, ab * 128,
                          h);
          }
          pk_issued = pk + 1;
        }
        const int s = t % NS;
        if (t >= NS && !mbar_wait(bar(ms->kv_empty[s]), ((t / NS) - 1) & 1, abort_flag)) break;
        const uint32_t st = s_stage + s * C::kStageB;
        const int row = w.tt * kTile;
        if (leader) {
          mbar_arrive_expect_tx(bar(ms->kv_full[s]), 2 * NCB * kBoxB);
          for (int kb = 0; kb < NCB; ++kb) {
            tma_load_3d(st + kb * kBoxB, &tm_v, bar(ms->kv_full[s]), kb * 64, row, bh);
            tma_load_3d(st + (NCB + 1 + kb) * kBoxB, &tm_k, bar(ms->kv_full[s]), kb * 64, row, bh);
          }
        }
        issued = t + 1;
      }
      if (*abort_flag) {  // let the copies already issued land before the CTA can exit
        constexpr long long kDrain = kWaitLimitCycles / 8;
        for (int t = issued > NS ? issued - NS : 0; t < issued; ++t)
          mbar_wait(bar(ms->kv_full[t % NS]), (t / NS) & 1, nullptr, kDrain);
        for (int pk = pk_issued > 2 ? pk_issued - 2 : 0; pk < pk_issued; ++pk)
          mbar_wait(bar(ms->om_full[pk & 1]), (pk >> 1) & 1, nullptr, kDrain);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ projection issuer (whole warp;
    // the elected lane issues): U^T = Omega_a K_item^T into buffer it % NBUF as soon as the state
    // product of item it - NBUF has released that buffer, so the epilogue warps find the next
    // item's angles ready instead of waiting for the state products in between
    if (n > 0) {
      const bool leader = elect_one();
      const uint32_t id1 = idesc_f16(128, 64, 1, 1, 0, 0);
      const int nitems = 2 * n;
      RunWalker w1(tt0, n, nt);
      for (int it = 0; it < nitems; ++it) {
        const int t = it >> 1, hf = it & 1, s = t % NS, b = it % NBUF;
        w1.advance_to(t);
        const int pk = w1.k;
        if (hf == 0) {
          if (w1.first() && !mbar_wait(bar(ms->om_full[pk & 1]), (pk >> 1) & 1, abort_flag)) break;
          if (!mbar_wait(bar(ms->kv_full[s]), (t / NS) & 1, abort_flag)) break;
        }
        if (it >= NBUF && !mbar_wait(bar(ms->buf_free[b]), ((it - NBUF) / NBUF) & 1, abort_flag)) break;
        tc_fence_after();
        const uint64_t a0 = sdesc_sw128(s_om + (pk & 1) * C::kOmB, 16, 1024);
        const uint64_t b0 = sdesc_sw128(s_stage + s * C::kStageB + (NCB + 1) * kBoxB + hf * 64 * kRowB, 16, 1024);
        const uint32_t d = tmem + C::kUcol + b * 64;
        if (leader) {
#pragma unroll
          for (int kb = 0; kb < NCB; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t off = uint64_t((kb * kBoxB + kk * 32) >> 4);
              mma_ss(d, a0 + off, b0 + off, id1, (kb | kk) ? 1u : 0u);
            }
          mma_commit(bar(ms->u_full[b]));
          if (hf == 1 && w1.last()) mma_commit(bar(ms->om_free[pk & 1]));
        }
        __syncwarp();
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ state-product issuer (whole
    // warp; the elected lane issues the MMAs and commits)
    if (n > 0) {
      const bool leader = elect_one();
      const uint32_t id2 = idesc_f16(128, NV, 1, 1, 0, 1);
      const int nitems = 2 * n;
      bool ok = true;
      RunWalker w2(tt0, n, nt);
      auto write_meta_max = [&](int pk) {
        float mx = 0.f;
        for (int w = 0; w < 8; ++w) mx = fmaxf(mx, ms->redmax[pk & 1][w]);
        const long long sl = slot_of(p0 + pk);
        if (leader) {
          p.meta[sl * 2 + 1] = mx;
          if (KIND == 1) p.meta[sl * 2] = 0.f;
        }
      };
      for (int it = 0; ok && it < nitems; ++it) {
        const int t = it >> 1, hf = it & 1, s = t % NS, b = it % NBUF;
        w2.advance_to(t);
        const int pk = w2.k;
        const bool fresh = hf == 0 && w2.first();
        if (!(ok = mbar_wait(bar(ms->p_full[b]), (it / NBUF) & 1, abort_flag))) break;
        if (KIND == 0 && hf == 0 && !(ok = mbar_wait(bar(ms->w_full[s]), (t / NS) & 1, abort_flag))) break;
        if (fresh && pk > 0) {
          if (!(ok = mbar_wait(bar(ms->s_free), (pk - 1) & 1, abort_flag))) break;
          write_meta_max(pk - 1);
        }
        tc_fence_after();
        const uint64_t vd =
            sdesc_sw128(s_stage + s * C::kStageB, kBoxB, 1024) + uint64_t((hf * 64 * kRowB) >> 4);
        const uint32_t ub = tmem + C::kUcol + b * 64;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = vd + uint64_t((kk * 16 * kRowB) >> 4);
            const uint32_t acc = (fresh && kk == 0) ? 0u : 1u;
            const uint32_t col = 32 * (kk >> 1) + 8 * (kk & 1);
            mma_ts(tmem, ub + col, bd, id2, acc);
            if (KIND == 0) mma_ts(tmem + NV, ub + 16 + col, bd, id2, acc);
          }
          mma_commit(bar(ms->buf_free[b]));
          if (hf == 1) {
            mma_commit(bar(ms->kv_empty[s]));
            if (w2.last()) mma_commit(bar(ms->s_done));
          }
        }
        __syncwarp();
      }
      if (ok) {
        w2.advance_to(n - 1);
        const int pk_last = w2.k;
        if (mbar_wait(bar(ms->s_free), pk_last & 1, abort_flag)) write_meta_max(pk_last);
      }
      if (leader) mma_commit(bar(ms->drain));
      __syncwarp();
      mbar_wait(bar(ms->drain), 0, nullptr, kWaitLimitCycles / 8);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ key norms (trig)
    if (KIND == 0 && n > 0) {
      const int j = (warp - 4) * 32 + lane;  // key row of the tile
      float c = 0.f;
      uint32_t nph = 0;
      RunWalker rw(tt0, n, nt);
      for (int t = 0; t < n; ++t) {
        rw.advance_to(t);
        const int s = t % NS;
        if (!mbar_wait(bar(ms->kv_full[s]), (t / NS) & 1, abort_flag)) break;
        uint8_t* st = gb + (s_stage - base) + s * C::kStageB;
        float acc = 0.f;
#pragma unroll
        for (int kb = 0; kb < NCB; ++kb)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 xv =
                *reinterpret_cast<const uint4*>(st + (NCB + 1 + kb) * kBoxB + j * kRowB + ((ch ^ (j & 7)) << 4));
            const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xFFFF0000u);
              acc = fmaf(lo, lo, acc);
              acc = fmaf(hi, hi, acc);
            }
          }
        const bool valid = rw.tt * kTile + j < p.L;
        const float n2 = valid ? 0.5f * acc : -INFINITY;
        float m = n2;
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) ms->tmax[t & 1][warp - 4] = m;
        if (!group_sync(bar(ms->norm_sync), nph, abort_flag)) break;
        m = fmaxf(fmaxf(ms->tmax[t & 1][0], ms->tmax[t & 1][1]), fmaxf(ms->tmax[t & 1][2], ms->tmax[t & 1][3]));
        float f = 1.f;
        if (rw.first()) {
          c = m + kMargin;
        } else if (m > c) {
          const float cn = m + kMargin;
          f = __expf(c - cn);
          c = cn;
        }
        const float w = valid ? __expf(n2 - c) : 0.f;
#pragma unroll
        for (int kb = 0; kb < NCB; ++kb)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint4* px = reinterpret_cast<uint4*>(st + kb * kBoxB + j * kRowB + ((ch ^ (j & 7)) << 4));
            const uint4 xv = *px;
            const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o4[e] = pack_bf16x2(__uint_as_float(w4[e] << 16) * w, __uint_as_float(w4[e] & 0xFFFF0000u) * w);
            *px = make_uint4(o4[0], o4[1], o4[2], o4[3]);
          }
        *reinterpret_cast<__nv_bfloat16*>(st + NCB * kBoxB + j * kRowB + ((j & 7) << 4)) = __float2bfloat16_rn(w);
        if (j == 0) {
          ms->frescale[s] = f;
          if (rw.last()) p.meta[slot_of(p0 + rw.k) * 2] = c;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->w_full[s]));
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ features and state flushes
    const int g = (warp - 8) >> 2, q = warp & 3;
    const uint32_t la = uint32_t(q * 32) << 16;
    const int nitems = 2 * n;
    bool ok = true;
    RunWalker w(tt0, n, nt);
    // Groups 0 and 1 flush share 0 and share 1 of every pair of the run, in pair order: a pair
    // when the group first reaches an item past it, the last pair after the loop. (Waiting on
    // s_done for every pair in order keeps each wait within one phase of the barrier.)
    int flushed = 0;
    auto flush = [&](int pk) -> bool {
      const long long pr = p0 + pk;
      if (!mbar_wait(bar(ms->s_done), pk & 1, abort_flag)) return false;
      tc_fence_after();
      float* dst = p.part + slot_of(pr) * (long long)(DP + 1) * R;
      float mx = 0.f;
      // trig: group g writes state block g (rows g*128 ..); ReLU: group g writes value
      // columns [g*DP/2, (g+1)*DP/2) and group 1 the normaliser column
      const int row = (KIND == 0 ? g * 128 : 0) + q * 32 + lane;
      const uint32_t sa = tmem + la + (KIND == 0 ? g * NV : 0);
      const int c_lo = KIND == 0 ? 0 : g * (DP / 2), c_hi = KIND == 0 ? DP : (g + 1) * (DP / 2);
#pragma unroll 1
      for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(sa + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = __uint_as_float(v[e]);
          dst[(long long)(c0 + e) * R + row] = x;
          mx = fmaxf(mx, fabsf(x));
        }
      }
      if (KIND == 0 || g == 1) {
        uint32_t zc;
        tmem_ld1(sa + DP, zc);
        tmem_wait_ld();
        const float x = __uint_as_float(zc);
        dst[(long long)DP * R + row] = x;
        mx = fmaxf(mx, fabsf(x));
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) ms->redmax[pk & 1][g * 4 + q] = mx;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->s_free));
      return true;
    };
    for (int it = g; ok && it < nitems; it += NG) {
      const int t = it >> 1, hf = it & 1, s = t % NS, b = it % NBUF;
      w.advance_to(t);
      if (g < 2)
        while (ok && flushed < w.k) ok = flush(flushed++);
      if (!ok) break;
      if (!(ok = mbar_wait(bar(ms->u_full[b]), (it / NBUF) & 1, abort_flag))) break;
      if (KIND == 0 && hf == 0 && !w.first()) {
        // the tile raised the reference: rescale S once every earlier state MMA has completed
        if (!(ok = mbar_wait(bar(ms->w_full[s]), (t / NS) & 1, abort_flag))) break;
        const float f = ms->frescale[s];
        if (f != 1.f) {
          if (!(ok = mbar_wait(bar(ms->buf_free[(it - 1) % NBUF]), ((it - 1) / NBUF) & 1, abort_flag))) break;
          tc_fence_after();
          for (int c0 = 0; c0 < NSB * NV; c0 += 8) {
            uint32_t r8[8];
            tmem_ld8(tmem + la + c0, r8);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) r8[e] = __float_as_uint(__uint_as_float(r8[e]) * f);
            tmem_st8(tmem + la + c0, r8);
          }
          tmem_wait_st();
        }
      }
      tc_fence_after();
      const uint32_t ub = tmem + la + C::kUcol + b * 64;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t u[32];
        tmem_ld32(ub + 32 * c, u);
        tmem_wait_ld();
        if (KIND == 0) {
          uint32_t cp[16], sp[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float s0, c0, s1, c1;
            sincos_mixed<kPolyMask>(2 * e, __uint_as_float(u[2 * e]), s0, c0);
            sincos_mixed<kPolyMask>(2 * e + 1, __uint_as_float(u[2 * e + 1]), s1, c1);
#ifdef FAVOR_PACK_TRUNC
            cp[e] = pack_hi16(c0, c1);
            sp[e] = pack_hi16(s0, s1);
#else
            cp[e] = pack_bf16x2(c0, c1);
            sp[e] = pack_bf16x2(s0, s1);
#endif
          }
          tmem_st16(ub + 32 * c, cp);
          tmem_st16(ub + 32 * c + 16, sp);
        } else {
          uint32_t rp[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            rp[e] = pack_bf16x2(fmaxf(__uint_as_float(u[2 * e]), 0.f), fmaxf(__uint_as_float(u[2 * e + 1]), 0.f));
          tmem_st16(ub + 32 * c, rp);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->p_full[b]));
    }
    if (g < 2 && ok && n > 0) {
      w.advance_to(n - 1);
      while (ok && flushed <= w.k) ok = flush(flushed++);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================================ merge
struct MergeParams {
  int nab, ntiles, smax, M;
  long long units, P;   // the state kernel's unit count and grid size
  const float* part;
  const float* meta;
  uint8_t* img;         // [B*H][image bytes]
  long long img_bytes;  // per head
};

__device__ __forceinline__ int nslots(long long pr, const MergeParams& p) {
  return (int)(cta_of_unit((pr + 1) * p.ntiles - 1, p.units, p.P) - cta_of_unit(pr * p.ntiles, p.units, p.P) + 1);
}

// Byte of (feature f, value row n) in a K-major 128-byte-swizzled image of NV rows per
// 64-feature atom.
template <int NV>
__device__ __forceinline__ uint32_t img_byte(int f, int n) {
  return uint32_t(f >> 6) * (NV * kRowB) + uint32_t(n) * kRowB + ((uint32_t(((f & 63) >> 3) ^ (n & 7))) << 4) +
         uint32_t(f & 7) * 2;
}

// One block per (pair, 32 state rows), one thread per 8-row work item (4 (d_pad + 16) threads).
// Trig feature order within a 128-angle block: 32-angle groups of [cos 32 | sin 32], matching the
// query kernel's packing. The first warp turns the head's slot metadata into per-slot weights in
// shared memory while every thread's loads of its first slots are in flight; then every thread
// sums its item over the pair's slots.
constexpr int kMergeMaxSlots = 64;  // slots of one head (nab * smax) the merge can weight

template <int KIND, int DP>
__host__ __device__ constexpr int merge_threads() { return 4 * (DP + 16); }  // one 8-row work item per thread

// Blocks per SM the merge is compiled for, and the slots of a work item whose loads are issued
// before the weights are known: trig has twice the blocks of ReLU (256 state rows per pair, not
// 128), so it keeps fewer loads in flight per thread to fit four blocks per SM (one wave at the
// usual shapes); ReLU fits two blocks per SM with four.
template <int KIND>
__host__ __device__ constexpr int merge_min_blocks() { return KIND == 0 ? 4 : 2; }
template <int KIND>
__host__ __device__ constexpr int merge_pre() { return KIND == 0 ? 2 : 4; }

template <int KIND, int DP>
__global__ void __launch_bounds__(merge_threads<KIND, DP>(), merge_min_blocks<KIND>())
    k_bidir_merge(const MergeParams p) {
  constexpr int NV = DP + 16, R = KIND == 0 ? 256 : 128, FB = R;
  constexpr int kMergePre = merge_pre<KIND>();
  __shared__ float wts[kMergeMaxSlots];
  __shared__ float scale_s;
  pdl_launch_dependents();  // the query kernel may start its projections
  pdl_wait();               // the key-state partials are complete
  const long long pr = blockIdx.x;
  const int rb = blockIdx.y;
  const long long bh = pr / p.nab;
  const int ab = (int)(pr % p.nab);
  // slot counts of the head's (at most 4) angle blocks: lane a of every warp evaluates block a's
  // (two 64-bit divisions), and the warp shares them
  const int nsl = (threadIdx.x & 31) < p.nab ? nslots(bh * p.nab + (threadIdx.x & 31), p) : 0;
  const int ns = min(__shfl_sync(0xffffffffu, nsl, ab), kMergeMaxSlots);
  uint8_t* img = p.img + bh * p.img_bytes;
  const float* part = p.part + pr * p.smax * (long long)(DP + 1) * R;
  const long long sstride = (long long)(DP + 1) * R;
  // Work item of this thread: 8 consecutive state rows of value row nn (two float4 loads per
  // slot), i.e. 8 consecutive features of the image, one 16-byte chunk. The partial states do not
  // depend on the weights: the loads of the first kMergePre slots are issued before the first
  // warp has turned the metadata into weights, so they are in flight together with its loads.
  const int w = threadIdx.x, oct = w & 3, nn = w >> 2;
  const int r0 = rb * 32 + oct * 8;
  const bool live = nn <= DP;
  const float* src = part + (long long)nn * R + r0;
  float4 pre[kMergePre][2];
#pragma unroll
  for (int s = 0; s < kMergePre; ++s) {
    pre[s][0] = make_float4(0.f, 0.f, 0.f, 0.f);
    pre[s][1] = pre[s][0];
    if (live && s < ns) {
      pre[s][0] = *reinterpret_cast<const float4*>(src + s * sstride);
      pre[s][1] = *reinterpret_cast<const float4*>(src + s * sstride + 4);
    }
  }
  if (threadIdx.x < 32) {
    // the head's reference (max over its slots) and the bound of its merged state; a lane holds
    // slots lane and lane + 32 of each of the head's (at most 4) angle blocks
    const int lane = threadIdx.x;
    float mc[8], mb[8];
    float cmax = -INFINITY;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int a2 = e >> 1, sl = lane + 32 * (e & 1);
      mc[e] = -INFINITY;
      mb[e] = 0.f;
      const int ns2 = __shfl_sync(0xffffffffu, nsl, a2 & 3);
      if (a2 < p.nab) {
        const long long q2 = bh * p.nab + a2;
        if (sl < ns2) {
          const float* m = p.meta + (q2 * p.smax + sl) * 2;
          mc[e] = KIND == 0 ? m[0] : 0.f;
          mb[e] = m[1];
        }
      }
      cmax = fmaxf(cmax, mc[e]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    float bound = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int a2 = e >> 1, sl = lane + 32 * (e & 1);
      if (mc[e] == -INFINITY) continue;
      const float wt = KIND == 0 ? __expf(mc[e] - cmax) : 1.f;
      bound += wt * mb[e];
      if (a2 == ab) wts[sl] = wt;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) bound += __shfl_xor_sync(0xffffffffu, bound, o);
    if (lane == 0) scale_s = (KIND == 0 && bound > 0.f) ? exp2f(14.f - ceilf(log2f(bound))) : 1.f;
  }
  __syncthreads();
  const float scale = scale_s;
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (live) {
#pragma unroll
    for (int s = 0; s < kMergePre; ++s) {
      if (s < ns) {
        const float wa = wts[s];
        v[0] = fmaf(wa, pre[s][0].x, v[0]);
        v[1] = fmaf(wa, pre[s][0].y, v[1]);
        v[2] = fmaf(wa, pre[s][0].z, v[2]);
        v[3] = fmaf(wa, pre[s][0].w, v[3]);
        v[4] = fmaf(wa, pre[s][1].x, v[4]);
        v[5] = fmaf(wa, pre[s][1].y, v[5]);
        v[6] = fmaf(wa, pre[s][1].z, v[6]);
        v[7] = fmaf(wa, pre[s][1].w, v[7]);
      }
    }
    for (int s = kMergePre; s < ns; ++s) {
      const float4 a0 = *reinterpret_cast<const float4*>(src + s * sstride);
      const float4 a1 = *reinterpret_cast<const float4*>(src + s * sstride + 4);
      const float wa = wts[s];
      v[0] = fmaf(wa, a0.x, v[0]);
      v[1] = fmaf(wa, a0.y, v[1]);
      v[2] = fmaf(wa, a0.z, v[2]);
      v[3] = fmaf(wa, a0.w, v[3]);
      v[4] = fmaf(wa, a1.x, v[4]);
      v[5] = fmaf(wa, a1.y, v[5]);
      v[6] = fmaf(wa, a1.z, v[6]);
      v[7] = fmaf(wa, a1.w, v[7]);
    }
  }
  const int a0 = KIND == 0 ? (r0 & 127) : r0;  // first angle of the octet (same sin/cos block)
  uint32_t pk[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float x0 = ab * 128 + a0 + 2 * e < p.M ? v[2 * e] : 0.f;      // padded angles read as zero
    const float x1 = ab * 128 + a0 + 2 * e + 1 < p.M ? v[2 * e + 1] : 0.f;
    pk[e] = KIND == 0 ? pack_f16x2(x0 * scale, x1 * scale) : pack_bf16x2(x0, x1);
  }
  const int f0 = KIND == 0 ? ab * FB + (a0 >> 5) * 64 + (r0 >> 7) * 32 + (a0 & 31) : ab * FB + r0;
  *reinterpret_cast<uint4*>(img + img_byte<NV>(f0, nn)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

// ============================================================================ queries
template <int KIND, int DP>
struct QueryCfg {
  static constexpr int NCB = DP / 64, NV = DP + 16;
  static constexpr int FB = KIND == 0 ? 256 : 128;   // features of a 128-angle block
  static constexpr int NBQ = DP == 64 ? 3 : 2;       // 128-angle U/phi buffers
  static constexpr int NBN = 1;                      // numerator buffers
  static constexpr int NOS = DP == 64 ? 2 : 1;       // output staging buffers
  static constexpr int kNumCol = NBQ * 128;          // TMEM: U ring, then the numerator
  static_assert(kNumCol + NBN * NV <= 512, "TMEM budget");
};

struct QueryParams {
  int H, L, M, nab, ntiles;
  long long units;          // B * H * ntiles
  const uint8_t* img;       // [B*H][img_bytes]
  int img_bytes;
  int om_bytes;             // nab * NCB boxes
  int off_img, off_q, off_out, off_misc;  // shared-memory layout (bytes from the aligned base)
};

struct alignas(16) QueryMisc {
  int abort_flag;
  uint32_t tmem_base;
  uint64_t om_full;    // a head's Omega blocks (the projections)
  uint64_t head_full;  // a head's state image (the state products)
  uint64_t head_free;  // both buffers may take the next head
  uint64_t q_full[2], q_empty[2];
  uint64_t u_full[3], p_full[3], buf_free[3];
  uint64_t num_full[2], num_empty[2];
  uint64_t drain;
  uint64_t out_sync;  // bounded barrier among the 128 output threads
};
static_assert(sizeof(QueryMisc) <= 1024, "misc block");

template <int KIND, int DP>
__global__ void __launch_bounds__(kThreads, 1)
    k_bidir_query(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_om,
                  const __grid_constant__ CUtensorMap tm_out, const QueryParams p) {
  using C = QueryCfg<KIND, DP>;
  constexpr int NCB = C::NCB, NV = C::NV, FB = C::FB, NBN = C::NBN, NOS = C::NOS, NBQ = C::NBQ;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (base - raw);
  const uint32_t s_om = base, s_img = base + p.off_img, s_q = base + p.off_q, s_out = base + p.off_out;
  QueryMisc* ms = reinterpret_cast<QueryMisc*>(gb + p.off_misc);
  volatile int* abort_flag = &ms->abort_flag;
  auto bar = [](uint64_t& b) { return smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long P = gridDim.x, U = p.units;
  const long long u0 = run_begin(blockIdx.x, U, P), u1 = run_begin(blockIdx.x + 1, U, P);
  const int n = (int)(u1 - u0);
  const int nt = p.ntiles, nab = p.nab;
  const long long h0 = u0 / nt;
  const int tt0 = (int)(u0 - h0 * nt);

  if (tid == 0) {
    ms->abort_flag = 0;
    mbar_init(bar(ms->om_full), 1);
    mbar_init(bar(ms->head_full), 1);
    mbar_init(bar(ms->head_free), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(ms->q_full[i]), 1);
      mbar_init(bar(ms->q_empty[i]), 1);
      mbar_init(bar(ms->num_full[i]), 1);
      mbar_init(bar(ms->num_empty[i]), 4);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(bar(ms->u_full[i]), 1);
      mbar_init(bar(ms->p_full[i]), 8);
      mbar_init(bar(ms->buf_free[i]), 1);
    }
    mbar_init(bar(ms->drain), 1);
    mbar_init(bar(ms->out_sync), 128);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (whole warp; the
    // elected lane issues the copies)
    if (n > 0) {
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_om);
        tma_prefetch_desc(&tm_out);
      }
      int issued = 0, heads = 0;
      RunWalker w(tt0, n, nt);
      for (int t = 0; t < n; ++t) {
        w.advance_to(t);
        const long long bh = h0 + w.k;
        const int s = t & 1;
        if (t >= 2 && !mbar_wait(bar(ms->q_empty[s]), ((t >> 1) - 1) & 1, abort_flag)) break;
        if (leader) {
          mbar_arrive_expect_tx(bar(ms->q_full[s]), NCB * kBoxB);
          for (int kb = 0; kb < NCB; ++kb)
            tma_load_3d(s_q + (s * NCB + kb) * kBoxB, &tm_q, bar(ms->q_full[s]), kb * 64, w.tt * kTile, (int)bh);
        }
        issued = t + 1;
        if (w.first()) {
          const int hk = w.k;
          if (hk >= 1 && !mbar_wait(bar(ms->head_free), (hk - 1) & 1, abort_flag)) break;
          const int h = (int)(bh % p.H);
          const uint8_t* src = p.img + bh * p.img_bytes;
          if (leader) {  // Omega does not come from the merge: the projections may start now
            mbar_arrive_expect_tx(bar(ms->om_full), p.om_bytes);
            for (int ab = 0; ab < nab; ++ab)
              for (int kb = 0; kb < NCB; ++kb)
                tma_load_3d(s_om + (ab * NCB + kb) * kBoxB, &tm_om, bar(ms->om_full), kb * 64, ab * 128, h);
          }
          if (hk == 0) pdl_wait();  // the merge has written the state images
          if (leader) {
            mbar_arrive_expect_tx(bar(ms->head_full), p.img_bytes);
            for (int off = 0; off < p.img_bytes; off += 32768) {
              const int sz = min(32768, p.img_bytes - off);
              bulk_load(s_img + off, src + off, sz, bar(ms->head_full));
            }
          }
          heads = hk + 1;
        }
      }
      if (*abort_flag) {
        constexpr long long kDrain = kWaitLimitCycles / 8;
        for (int t = issued > 2 ? issued - 2 : 0; t < issued; ++t)
          mbar_wait(bar(ms->q_full[t & 1]), (t >> 1) & 1, nullptr, kDrain);
        if (heads > 0) {
          mbar_wait(bar(ms->om_full), (heads - 1) & 1, nullptr, kDrain);
          mbar_wait(bar(ms->head_full), (heads - 1) & 1, nullptr, kDrain);
        }
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ projection issuer (whole warp;
    // the elected lane issues): U = Q_tile Omega_ab^T into buffer j % NBQ once the state product
    // of item j - NBQ has released it; a new head's first projection waits for its Omega
    if (n > 0) {
      const bool leader = elect_one();
      const uint32_t id1 = idesc_f16(128, 128, 1, 1, 0, 0);
      const int nit = n * nab;
      const uint64_t om0 = sdesc_sw128(s_om, 16, 1024);
      RunWalker w1(tt0, n, nt);
      for (int j = 0; j < nit; ++j) {
        const int t = j / nab, ab = j - t * nab, b = j % NBQ, s = t & 1;
        w1.advance_to(t);
        if (ab == 0) {
          if (!mbar_wait(bar(ms->q_full[s]), (t >> 1) & 1, abort_flag)) break;
          if (w1.first() && !mbar_wait(bar(ms->om_full), w1.k & 1, abort_flag)) break;
        }
        if (j >= NBQ && !mbar_wait(bar(ms->buf_free[b]), ((j - NBQ) / NBQ) & 1, abort_flag)) break;
        tc_fence_after();
        const uint64_t q0 = sdesc_sw128(s_q + s * NCB * kBoxB, 16, 1024);
        if (leader) {
#pragma unroll
          for (int kb = 0; kb < NCB; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem + b * 128, q0 + uint64_t((kb * kBoxB + kk * 32) >> 4),
                     om0 + uint64_t(((ab * NCB + kb) * kBoxB + kk * 32) >> 4), id1, (kb | kk) ? 1u : 0u);
          mma_commit(bar(ms->u_full[b]));
          if (ab == nab - 1) mma_commit(bar(ms->q_empty[s]));
        }
        __syncwarp();
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ state-product issuer (whole
    // warp; the elected lane issues the MMAs and commits)
    if (n > 0) {
      const bool leader = elect_one();
      const uint32_t fmt = KIND == 0 ? 0u : 1u;  // fp16 (trig) or bf16 (ReLU) state operands
      const uint32_t id2 = idesc_f16(128, NV, fmt, fmt, 0, 0);
      const int nit = n * nab;
      const uint64_t img0 = sdesc_sw128(s_img, 16, 1024);
      bool ok = true;
      RunWalker w2(tt0, n, nt);
      for (int j = 0; ok && j < nit; ++j) {
        const int t = j / nab, ab = j - t * nab, b = j % NBQ, nb = t % NBN;
        w2.advance_to(t);
        if (!(ok = mbar_wait(bar(ms->p_full[b]), (j / NBQ) & 1, abort_flag))) break;
        if (ab == 0 && w2.first() && !(ok = mbar_wait(bar(ms->head_full), w2.k & 1, abort_flag))) break;
        if (ab == 0 && t >= NBN && !(ok = mbar_wait(bar(ms->num_empty[nb]), ((t / NBN) - 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t dn = tmem + C::kNumCol + nb * NV;
        const bool head_end = ab == nab - 1 && w2.last();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < FB / 16; ++kk) {
            const int f = ab * FB + 16 * kk;
            const uint64_t bd = img0 + uint64_t(((f >> 6) * (NV * kRowB) + ((f & 63) >> 4) * 32) >> 4);
            const uint32_t acol = KIND == 0 ? 8 * kk : 64 * (kk >> 2) + 8 * (kk & 3);
            mma_ts(dn, tmem + b * 128 + acol, bd, id2, (ab | kk) ? 1u : 0u);
          }
          mma_commit(bar(ms->buf_free[b]));
          if (ab == nab - 1) mma_commit(bar(ms->num_full[nb]));
          if (head_end) mma_commit(bar(ms->head_free));
        }
        __syncwarp();
      }
      if (leader) mma_commit(bar(ms->drain));
      __syncwarp();
      mbar_wait(bar(ms->drain), 0, nullptr, kWaitLimitCycles / 8);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ normalise and store
    const int q = warp & 3, row = q * 32 + lane;
    const uint32_t la = uint32_t(q * 32) << 16;
    const bool issuer = warp == 4 && lane == 0;
    uint32_t oph = 0;
    RunWalker w(tt0, n, nt);
    for (int t = 0; t < n; ++t) {
      w.advance_to(t);
      const int nb = t % NBN, sb = t % NOS;
      if (!mbar_wait(bar(ms->num_full[nb]), (t / NBN) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t dn = tmem + la + C::kNumCol + nb * NV;
      uint32_t dv;
      tmem_ld1(dn + DP, dv);
      tmem_wait_ld();
      const float den = __uint_as_float(dv);
      const float inv = den != 0.f ? 1.f / den : 0.f;
      if (issuer && t >= NOS) {
        if (NOS == 2)
          bulk_wait_read1();
        else
          bulk_wait_read0();
      }
      if (!group_sync(bar(ms->out_sync), oph, abort_flag)) break;
      uint8_t* stg = gb + (s_out - base) + sb * NCB * kBoxB + row * kRowB;
#pragma unroll 1
      for (int kb = 0; kb < NCB; ++kb) {
        uint32_t v[32], w[32];
        tmem_ld32(dn + kb * 64, v);
        tmem_ld32(dn + kb * 64 + 32, w);
        tmem_wait_ld();
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t* src = m < 4 ? v + 8 * m : w + 8 * (m - 4);
          *reinterpret_cast<uint4*>(stg + kb * kBoxB + ((m ^ (row & 7)) << 4)) = make_uint4(
              pack_bf16x2(__uint_as_float(src[0]) * inv, __uint_as_float(src[1]) * inv),
              pack_bf16x2(__uint_as_float(src[2]) * inv, __uint_as_float(src[3]) * inv),
              pack_bf16x2(__uint_as_float(src[4]) * inv, __uint_as_float(src[5]) * inv),
              pack_bf16x2(__uint_as_float(src[6]) * inv, __uint_as_float(src[7]) * inv));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->num_empty[nb]));
      fence_proxy_async_smem();
      if (!group_sync(bar(ms->out_sync), oph, abort_flag)) break;
      if (issuer) {
        for (int kb = 0; kb < NCB; ++kb)
          tma_store_3d(&tm_out, s_out + (sb * NCB + kb) * kBoxB, kb * 64, w.tt * kTile, (int)(h0 + w.k));
        bulk_commit();
      }
    }
    if (issuer) bulk_wait0();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ query features
    const int q = warp & 3, hcol = (warp - 8) >> 2;
    const uint32_t la = uint32_t(q * 32) << 16;
    const int nit = n * nab;
    for (int j = 0; j < nit; ++j) {
      const int b = j % NBQ;
      if (!mbar_wait(bar(ms->u_full[b]), (j / NBQ) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t ub = tmem + la + b * 128 + 64 * hcol;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t u[32];
        tmem_ld32(ub + 32 * c, u);
        tmem_wait_ld();
        if (KIND == 0) {
          uint32_t cp[16], sp[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float s0, c0, s1, c1;
            sincos_mixed<kPolyMask>(2 * e, __uint_as_float(u[2 * e]), s0, c0);
            sincos_mixed<kPolyMask>(2 * e + 1, __uint_as_float(u[2 * e + 1]), s1, c1);
            cp[e] = pack_f16x2(c0, c1);
            sp[e] = pack_f16x2(s0, s1);
          }
          tmem_st16(ub + 32 * c, cp);
          tmem_st16(ub + 32 * c + 16, sp);
        } else {
          uint32_t rp[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            rp[e] = pack_bf16x2(fmaxf(__uint_as_float(u[2 * e]), 0.f), fmaxf(__uint_as_float(u[2 * e + 1]), 0.f));
          tmem_st16(ub + 16 * c, rp);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->p_full[b]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bs
}  // namespace favor
