// kernel_bidir.cuh - fused bidirectional FAVOR forward on sm_100a tensor cores.
//
// What it computes. The explainer page "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？",
// section 核心机制：FAVOR+, gives out = D_hat^-1 phi(Q) (phi(K)^T [V|1]). The state
// S = phi(K)^T [V|1] is aggregated first, then left-multiplied by phi(Q). No L x L matrix is
// formed.
//
// Structure. One thread-block cluster of P CTAs per (batch, head). CTA r of the cluster owns a
// contiguous run of 128-token tiles.
//   Key phase. Per tile, per 128-angle block a and per IW-token slice (IW = 32 or 64):
//     MMA1  U^T = Omega_a . K_slice^T   (M=128 angles, N=IW tokens, K=64; bf16, fp32 in TMEM)
//     epilogue: cos(U), sin(U) (trig) or max(U, 0) (relu) -> bf16 -> a separate TMEM phi slot
//     MMA2  S_blk += phi^T . [w o V | w]  (A from TMEM; B = the V tile, MN-major, plus a
//           column held in a per-stage buffer reached through the descriptor's leading-byte
//           offset; M=128 features, N=80, K=16 tokens per instruction; fp32 in TMEM)
//     Trig key features carry w_j = exp(|k_j|^2/2 - c) (the exp(|x|^2/2) factor of the feature
//     map, stabilised). The norm warp folds w_j into row j of the V tile and into the extra
//     column, so the epilogue only computes cos and sin. c is a running per-CTA reference kept
//     16 nats above the largest |k|^2/2 seen. If a tile exceeds it, S is rescaled in TMEM first.
//     ReLU features use w_j = 1 (a constant ones column).
//   Reduction, through distributed shared memory (no global scratch). Each CTA stages its fp32
//     partial state and its c. CTA r sums feature rows [r F / P, (r+1) F / P) over the P
//     partials in rank order, rescaled to the largest c, and rounds them to fp16 under a
//     power-of-two scale shared by the cluster. It writes them into every CTA's state image,
//     in the swizzled K-major layout the query phase's MMA reads. P = 1 converts in place.
//     Rows of padded features (angle >= M) are written as zero.
//   Query phase. Per tile and per 64-angle chunk c:
//     MMA1  U = Q_tile . Omega_c^T  (M=128 tokens, N=64 angles)
//     epilogue: cos(U), sin(U) (trig) or max(U, 0) (relu) -> fp16 -> a TMEM phi slot. The
//     exp(|q|^2/2) and 1/sqrt(M) factors cancel.
//     MMA2  num += phi_c . S_c  (A from TMEM, B = image from shared memory; N=80)
//   then out = num[:, :64] / num[:, 64] -> bf16 -> swizzled staging -> TMA store.
//
// Warp roles (384 threads): warp 0 TMA producer; warp 1 TMEM allocator and projection-MMA
// issuer; warp 2 state/numerator-MMA issuer; warp 3 key norms and V scaling (trig); warps 4-11
// epilogue in two warpgroups that take alternate items (warp w reads TMEM lanes 32 (w % 4) ..
// +31). The epilogue loads the next 32-column sub-item from TMEM while it computes the current.
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
constexpr int kNU = 3;                   // U ring depth (both phases)
constexpr int kNPK = 3;                  // key-phase phi ring depth
constexpr int kNPQ = 2;                  // query-phase phi ring depth
constexpr int kUQ = 160, kPQ = 352;      // query-phase TMEM ring bases (64-column slots)
constexpr int kNPad = 80;                // d + 1 padded to a multiple of 16
constexpr int kNV = kD + 1;              // value columns plus the normaliser column
constexpr int kImgAtomB = kNPad * kRowB; // bytes of one 64-feature atom of the state image
constexpr int kRegionB = 144 * 1024;     // shared region reused by every phase (see below)
constexpr int kColOff = 96 * 1024;       // key phase: w / ones column buffers after 3 stages
constexpr int kImgMaxB = 80 * 1024;      // query phase: state image, then Q stages, then output
constexpr int kQOff = kImgMaxB, kOutOff = kImgMaxB + kStagesQ * kTileB;
constexpr float kMargin = 16.f;          // stabiliser head-room, in nats
constexpr int kThreads = 384;
static_assert(kOutOff + 2 * kTileB == kRegionB, "query-phase layout");
static_assert(kColOff + kStagesK * kTileB == kRegionB, "key-phase layout");

struct BidirParams {
  int BH, H, L, M;      // heads (B*H), heads per batch, tokens, random features
  int Mpad;             // M rounded up to a multiple of 128
  int P;                // CTAs per head (cluster size, a power of two)
  int ntiles;           // ceil(L / 128)
};

struct alignas(16) Misc {
  float rescale[4];
  float red[16];
  float meta[2];                  // stabiliser reference and max |partial| for the cluster
  float cfinal;
  int abort_flag;
  uint32_t tmem_base;
  uint32_t pad[3];
  uint64_t om_full;
  uint64_t kv_full[kStagesK], kv_empty[kStagesK], w_full[kStagesK];
  uint64_t u_full[kNU], u_free[kNU], p_full[kNPK], p_free[kNPK];
  uint64_t s_done, img_full, mma_drain, mma_drain1;
  uint64_t q_full[kStagesQ], q_empty[kStagesQ];
  uint64_t uq_full[kNU], uq_free[kNU], pq_full[kNPQ], pq_free[kNPQ];
  uint64_t num_full[2], num_empty[2];
  uint64_t epi_sync;              // bounded barrier among the 256 epilogue threads
  uint64_t out_sync[2];           // per-warpgroup barrier around the output staging
};
static_assert(sizeof(Misc) <= 1024, "misc block too large");

// Shared memory: Omega (Mpad rows of 128 B) | 144 KB region | 1 KB misc | 1 KB alignment slack.
// The region holds, in turn: key stages (K, V) x 3 and the w / ones column buffers; the fp32
// partial state (cluster reduction); the state image, Q stages and output staging.
__host__ __device__ constexpr uint32_t bidir_smem_bytes(int Mpad) {
  return uint32_t(Mpad) * kRowB + kRegionB + 1024 + 1024;
}

// Angle of key-phase state row f (TMEM block f / 128, lane f % 128).
template <int KIND>
__device__ __forceinline__ int feature_angle(int f) {
  return KIND == 0 ? ((f >> 8) << 7) + (f & 127) : f;
}
// Feature row f -> (atom, k) in the query-phase image. Trig: block 2a is cos and 2a+1 is sin of
// angles 128a .. 128a+127. The query phase orders chunk c (64 angles) as
// [cos 32 | sin 32 | cos 32 | sin 32], one atom per 32 angles.
template <int KIND>
__device__ __forceinline__ void feature_to_image(int f, int& atom, int& k) {
  if (KIND == 0) {
    const int s = (f >> 7) & 1, r = feature_angle<0>(f);
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

// 32 columns of one lane -> cos/sin as 16-bit pairs, stored as [cos 16 columns | sin 16].
template <bool F16>
__device__ __forceinline__ void trig_cols(const uint32_t (&u)[32], uint32_t taddr) {
  uint32_t cp[16], sp[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float s0, c0, s1, c1;
    __sincosf(__uint_as_float(u[2 * j]), &s0, &c0);
    __sincosf(__uint_as_float(u[2 * j + 1]), &s1, &c1);
    cp[j] = F16 ? pack_f16x2(c0, c1) : pack_bf16x2(c0, c1);
    sp[j] = F16 ? pack_f16x2(s0, s1) : pack_bf16x2(s0, s1);
  }
  tmem_st16(taddr, cp);
  tmem_st16(taddr + 16, sp);
}
// 32 columns of one lane -> max(u, 0) as 16-bit pairs in 16 columns.
template <bool F16>
__device__ __forceinline__ void relu_cols(const uint32_t (&u)[32], uint32_t taddr) {
  uint32_t rp[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float x0 = fmaxf(__uint_as_float(u[2 * j]), 0.f), x1 = fmaxf(__uint_as_float(u[2 * j + 1]), 0.f);
    rp[j] = F16 ? pack_f16x2(x0, x1) : pack_bf16x2(x0, x1);
  }
  tmem_st16(taddr, rp);
}

// 40 consecutive fp32 TMEM columns of this thread's lane (one half of an 80-column state block).
__device__ __forceinline__ void load_state_cols(uint32_t taddr, float (&v)[40]) {
  uint32_t a[32], b[8];
  tmem_ld32(taddr, a);
  tmem_ld8(taddr + 32, b);
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(a[e]);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[32 + e] = __uint_as_float(b[e]);
}

// Everything the key phase needs from its kernel.
struct KeyCtx {
  uint8_t* gbase;                 // generic pointer to the 1024-aligned shared base
  uint32_t base, s_om, s_reg;     // shared-space addresses
  uint32_t tmem;                  // TMEM base (512 columns)
  int tid, warp, lane;
  int h, bh, t_begin, my_tiles, L, Mpad;
  int nblk, nsb, ipt, kUK, kPK;
};

// Key phase (see the file comment): accumulates the CTA's partial state in TMEM columns
// [0, nsb * 80) and commits ms->s_done when the last state MMA completes. Trig also leaves the
// final stabiliser reference in ms->cfinal. Every warp of the CTA calls this.
template <int KIND, int IW>
__device__ __forceinline__ void key_phase(const KeyCtx& kc, Misc* ms, const CUtensorMap* tm_k,
                                          const CUtensorMap* tm_v, const CUtensorMap* tm_q,
                                          const CUtensorMap* tm_om) {
  constexpr int NH = IW / 32;
  constexpr int PW = KIND == 0 ? IW : IW / 2;
  constexpr int SPT = kTile / IW;
  uint8_t* const gbase = kc.gbase;
  const uint32_t base = kc.base, s_om = kc.s_om, s_reg = kc.s_reg, tmem = kc.tmem;
  const int warp = kc.warp, lane = kc.lane;
  const int h = kc.h, bh = kc.bh, t_begin = kc.t_begin, my_tiles = kc.my_tiles;
  const int nblk = kc.nblk, nsb = kc.nsb, ipt = kc.ipt, kUK = kc.kUK, kPK = kc.kPK;
  volatile int* abort_flag = &ms->abort_flag;
  auto bar = [](uint64_t& b) { return smem_u32(&b); };
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(tm_k);
      tma_prefetch_desc(tm_v);
      tma_prefetch_desc(tm_q);
      mbar_arrive_expect_tx(bar(ms->om_full), uint32_t(kc.Mpad) * kRowB);
      for (int blk = 0; blk < nblk; ++blk)
        tma_load_3d(s_om + blk * kTileB, tm_om, bar(ms->om_full), 0, blk * 128, h);
      for (int t = 0; t < my_tiles; ++t) {
        const int s = t % kStagesK, k = t / kStagesK;
        if (!mbar_wait(bar(ms->kv_empty[s]), (k & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(ms->kv_full[s]), 2 * kTileB);
        const int row = (t_begin + t) * kTile;
        tma_load_3d(s_reg + s * 2 * kTileB, tm_k, bar(ms->kv_full[s]), 0, row, bh);
        tma_load_3d(s_reg + s * 2 * kTileB + kTileB, tm_v, bar(ms->kv_full[s]), 0, row, bh);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // Key-phase projection issuer: MMA1 of every item, U^T = Omega_a . K_slice^T into an
    // IW-column U slot. Descriptors are built once; each instruction adds a constant offset to
    // the start-address field (16-byte units).
    if (lane == 0) {
      const uint32_t id1 = idesc_f16(128, IW, 1, 1, 0, 0);
      const uint64_t a0 = sdesc_sw128(s_om, 16, 1024);
      const uint64_t k0 = sdesc_sw128(s_reg, 16, 1024);
      const int n = my_tiles * ipt;
      bool ok = mbar_wait(bar(ms->om_full), 0, abort_flag);
      int rem = 0, s = 0, b = 0;
      uint32_t kv_ph = 0, u_ph = 0;  // parity of the next kv_full / u_free completion to wait for
      for (int i = 0; ok && i < n; ++i) {
        if (rem == 0 && !(ok = mbar_wait(bar(ms->kv_full[s]), kv_ph, abort_flag))) break;
        if (i >= kNU && !(ok = mbar_wait(bar(ms->u_free[b]), u_ph, abort_flag))) break;
        tc_fence_after();
        const int a = rem / SPT, sl = rem % SPT;
        const uint64_t ad = a0 + uint64_t((a * kTileB) >> 4);
        const uint64_t bd = k0 + uint64_t((s * 2 * kTileB + sl * IW * kRowB) >> 4);
        const uint32_t d = tmem + kUK + b * IW;
        mma_ss(d, ad, bd, id1, 0u);
        mma_ss(d, ad + 2, bd + 2, id1, 1u);
        mma_ss(d, ad + 4, bd + 4, id1, 1u);
        mma_ss(d, ad + 6, bd + 6, id1, 1u);
        mma_commit(bar(ms->u_full[b]));
        if (++b == kNU) { b = 0; if (i >= 2 * kNU - 1) u_ph ^= 1u; }
        if (++rem == ipt) {
          rem = 0;
          if (++s == kStagesK) { s = 0; kv_ph ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // Key-phase state issuer: MMA2 of every item, S_blk += phi^T . [w o V_slice | w]. The B
    // descriptor's leading-byte offset reaches the stage's column buffer, which has the V
    // tile's layout, so it is the same for every instruction of a stage.
    if (lane == 0) {
      const uint32_t id2 = idesc_f16(128, kNPad, 1, 1, 0, 1);
      uint64_t vd[kStagesK];
#pragma unroll
      for (int s = 0; s < kStagesK; ++s) {
        const uint32_t vt = s_reg + s * 2 * kTileB + kTileB;
        const uint32_t ct = s_reg + kColOff + (KIND == 0 ? s * kTileB : 0);
        vd[s] = sdesc_sw128(vt, ct - vt, 1024);
      }
      const int n = my_tiles * ipt;
      int rem = 0, s = 0, pb = 0, t = 0;
      uint32_t p_ph = 0, w_ph = 0;
      bool ok = true;
      for (int i = 0; i < n; ++i) {
        if (KIND == 0 && rem == 0 && !(ok = mbar_wait(bar(ms->w_full[s]), w_ph, abort_flag))) break;
        if (!(ok = mbar_wait(bar(ms->p_full[pb]), p_ph, abort_flag))) break;
        tc_fence_after();
        const int a = rem / SPT, sl = rem % SPT;
        const uint32_t pcol = tmem + kPK + pb * PW;
#pragma unroll
        for (int kk = 0; kk < IW / 16; ++kk) {
          const uint64_t bd = vd[s] + uint64_t(((sl * IW + kk * 16) * kRowB) >> 4);
          const uint32_t acc = (t == 0 && sl == 0 && kk == 0) ? 0u : 1u;
          if (KIND == 0) {
            mma_ts(tmem + (2 * a) * kNPad, pcol + kk * 8, bd, id2, acc);
            mma_ts(tmem + (2 * a + 1) * kNPad, pcol + 16 + kk * 8, bd, id2, acc);
          } else {
            mma_ts(tmem + a * kNPad, pcol + kk * 8, bd, id2, acc);
          }
        }
        mma_commit(bar(ms->p_free[pb]));
        if (++pb == kNPK) { pb = 0; p_ph ^= 1u; }
        if (++rem == ipt) {
          mma_commit(bar(ms->kv_empty[s]));
          rem = 0;
          ++t;
          if (++s == kStagesK) { s = 0; w_ph ^= 1u; }
        }
      }
      mma_commit(bar(ms->s_done));
    }
    __syncwarp();
  } else if (warp == 3) {
    if (KIND == 0) {
      // Key norms and the running stabiliser reference c. w_j = exp(|k_j|^2/2 - c) is folded
      // into V row j and written to column 64 of the stage's column buffer.
      float cr = 0.f;
      for (int t = 0; t < my_tiles; ++t) {
        const int s = t % kStagesK;
        if (!mbar_wait(bar(ms->kv_full[s]), (t / kStagesK) & 1, abort_flag)) break;
        const uint8_t* kt = gbase + (s_reg - base) + s * 2 * kTileB;
        uint8_t* vt = gbase + (s_reg - base) + s * 2 * kTileB + kTileB;
        uint8_t* ct = gbase + (s_reg - base) + kColOff + s * kTileB;
        const int row0 = (t_begin + t) * kTile;
        float n2[4];
        float m = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = lane + 32 * jj;
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
          n2[jj] = row0 + j < kc.L ? 0.5f * acc : -INFINITY;
          m = fmaxf(m, n2[jj]);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float f = 1.f;
        if (t == 0) {
          cr = m + kMargin;
        } else if (m > cr) {
          const float nc = m + kMargin;
          f = __expf(cr - nc);
          cr = nc;
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = lane + 32 * jj;
          const float w = __expf(n2[jj] - cr);  // 0 for rows past L
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4* px = reinterpret_cast<uint4*>(vt + j * kRowB + ((c ^ (j & 7)) << 4));
            const uint4 x = *px;
            const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o4[e] = pack_bf16x2(__uint_as_float(w4[e] << 16) * w, __uint_as_float(w4[e] & 0xFFFF0000u) * w);
            *px = make_uint4(o4[0], o4[1], o4[2], o4[3]);
          }
          *reinterpret_cast<__nv_bfloat16*>(ct + j * kRowB + ((j & 7) << 4)) = __float2bfloat16_rn(w);
        }
        if (lane == 0) {
          ms->rescale[s] = f;
          if (t == my_tiles - 1) ms->cfinal = cr;
        }
        fence_proxy_async_smem();
        __syncwarp();
        mbar_arrive(bar(ms->w_full[s]));
        if (lane == 0) mbar_arrive(bar(ms->kv_empty[s]));
      }
    }
  } else {
    // ------------------------------------------------------------ key-phase epilogue
    // Items alternate between the two warpgroups. Warp w owns TMEM lanes 32 (w % 4) .. +31,
    // i.e. 32 angles of the block. An item is NH sub-items of 32 token columns. The U slot is
    // released once all of it is in registers, and the next sub-item's load is issued before
    // the current one is computed.
    const int q4 = warp & 3, grp = (warp - 4) >> 2;
    const uint32_t lane_addr = uint32_t(q4 * 32) << 16;
    const int n = my_tiles * ipt;
    int i = grp, hs = 0;
    uint32_t ua[32], ub[32];
    bool have = i < n, loaded = false;  // loaded: the current sub-item's TMEM load is issued
    // Issue the load of sub-item (i, hs). A sub-item that starts a new item first needs that
    // item's projection: wait for it only if `block`, else leave the load for later.
    auto issue = [&](int ii, int hh, uint32_t (&dst)[32], bool block) -> bool {
      if (hh == 0) {
        const uint32_t bb = bar(ms->u_full[ii % kNU]), ph = (ii / kNU) & 1;
        if (!(block ? mbar_wait(bb, ph, abort_flag) : mbar_test(bb, ph))) return false;
      }
      tc_fence_after();
      tmem_ld32(tmem + lane_addr + kUK + (ii % kNU) * IW + hh * 32, dst);
      return true;
    };
    auto step = [&](uint32_t (&cur)[32], uint32_t (&nxt)[32]) -> bool {
      if (!loaded && !issue(i, hs, cur, true)) return false;
      tmem_wait_ld();
      const int b = i % kNU, pb = i % kNPK;
      int i2 = i, h2 = hs + 1;
      if (h2 == NH) { h2 = 0; i2 = i + 2; }
      if (hs == NH - 1) {  // U(i) is in registers
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->u_free[b]));
      }
      const bool more = i2 < n;
      loaded = more && issue(i2, h2, nxt, false);
      if (hs == 0) {
        const int t = i / ipt, rem = i % ipt;
        if (KIND == 0 && rem == 0) {  // first item of the tile: grow the reference if needed
          const int s = t % kStagesK;
          if (!mbar_wait(bar(ms->w_full[s]), (t / kStagesK) & 1, abort_flag)) return false;
          const float f = ms->rescale[s];
          if (f != 1.f) {
            if (i > 0 && !mbar_wait(bar(ms->p_free[(i - 1) % kNPK]), ((i - 1) / kNPK) & 1, abort_flag))
              return false;
            tc_fence_after();
            for (int c0 = 0; c0 < nsb * kNPad; c0 += 8) {
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
        if (i >= kNPK && !mbar_wait(bar(ms->p_free[pb]), ((i / kNPK) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
      }
      const uint32_t paddr = tmem + lane_addr + kPK + pb * PW;
      if (KIND == 0) {
        trig_cols<false>(cur, paddr);
      } else {
        relu_cols<false>(cur, paddr + hs * 16);
      }
      if (hs == NH - 1) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->p_full[pb]));
      }
      i = i2;
      hs = h2;
      return more;
    };
    while (have) {
      if (!(have = step(ua, ub))) break;
      have = step(ub, ua);
    }
  }

}

// KIND: 0 trig, 1 ReLU. IW: key-phase slice width in tokens (32 or 64).
template <int KIND, int IW>
__global__ void __launch_bounds__(kThreads, 1)
    favor_bidir_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_om,
                   const __grid_constant__ CUtensorMap tm_out, const BidirParams p) {
  static_assert(IW == 32 || IW == 64, "key slice width");
  static_assert(KIND == 1 || IW == 32, "trig uses 32-token key slices");
  constexpr int NH = IW / 32;                       // 32-column sub-items per key item
  constexpr int PW = KIND == 0 ? IW : IW / 2;       // key phi slot width (packed 16-bit)
  constexpr int PWQ = KIND == 0 ? 64 : 32;          // query phi slot width
  constexpr int SPT = kTile / IW;                   // key slices per tile

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t s_om = base;
  const uint32_t s_reg = base + uint32_t(p.Mpad) * kRowB;
  Misc* ms = reinterpret_cast<Misc*>(gbase + (s_reg + kRegionB - base));
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
  const int ipt = nblk * SPT;                  // key-phase items per tile
  const int nchq = p.Mpad / 64;                // query-phase chunks per tile (even)
  const int kUK = nsb * kNPad;                 // key-phase U ring base, then the phi ring
  const int kPK = kUK + kNU * IW;
  auto bar = [](uint64_t& b) { return smem_u32(&b); };

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    ms->abort_flag = 0;
    mbar_init(bar(ms->om_full), 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(bar(ms->kv_full[s]), 1);
      mbar_init(bar(ms->kv_empty[s]), KIND == 0 ? 2 : 1);
      mbar_init(bar(ms->w_full[s]), 32);
    }
    for (int b = 0; b < kNU; ++b) {
      mbar_init(bar(ms->u_full[b]), 1);
      mbar_init(bar(ms->u_free[b]), 4);
      mbar_init(bar(ms->uq_full[b]), 1);
      mbar_init(bar(ms->uq_free[b]), 4);
    }
    for (int b = 0; b < kNPK; ++b) {
      mbar_init(bar(ms->p_full[b]), 4);
      mbar_init(bar(ms->p_free[b]), 1);
    }
    for (int b = 0; b < kNPQ; ++b) {
      mbar_init(bar(ms->pq_full[b]), 4);
      mbar_init(bar(ms->pq_free[b]), 1);
    }
    mbar_init(bar(ms->s_done), 1);
    mbar_init(bar(ms->img_full), 1);
    mbar_init(bar(ms->mma_drain), 1);
    mbar_init(bar(ms->mma_drain1), 1);
    for (int s = 0; s < kStagesQ; ++s) {
      mbar_init(bar(ms->q_full[s]), 1);
      mbar_init(bar(ms->q_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ms->num_full[s]), 1);
      mbar_init(bar(ms->num_empty[s]), 4);
      mbar_init(bar(ms->out_sync[s]), 128);
    }
    mbar_init(bar(ms->epi_sync), 256);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish();
  }
  {  // column buffers for [V | w]: zero, and for ReLU a constant 1.0 in column 64 of every row
    uint4* col = reinterpret_cast<uint4*>(gbase + (s_reg + kColOff - base));
    const int n16 = (KIND == 0 ? kStagesK : 1) * kTileB / 16;
    for (int i = tid; i < n16; i += kThreads) col[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    if (KIND == 1 && tid < kTile)
      reinterpret_cast<uint16_t*>(gbase + (s_reg + kColOff - base) + tid * kRowB + ((tid & 7) << 4))[0] = 0x3F80u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  // ================================================================ key phase
  {
    KeyCtx kc;
    kc.gbase = gbase;
    kc.base = base;
    kc.s_om = s_om;
    kc.s_reg = s_reg;
    kc.tmem = tmem;
    kc.tid = tid;
    kc.warp = warp;
    kc.lane = lane;
    kc.h = h;
    kc.bh = bh;
    kc.t_begin = t_begin;
    kc.my_tiles = my_tiles;
    kc.L = p.L;
    kc.Mpad = p.Mpad;
    kc.nblk = nblk;
    kc.nsb = nsb;
    kc.ipt = ipt;
    kc.kUK = kUK;
    kc.kPK = kPK;
    key_phase<KIND, IW>(kc, ms, &tm_k, &tm_v, &tm_q, &tm_om);
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
    if (epi) {  // convert the state straight from TMEM into the shared-memory image
      float mx = 0.f;
      for (int blk = 0; blk < nsb; ++blk) {
        float v[40];
        load_state_cols(tmem + lane_addr + blk * kNPad + ch * 40, v);
#pragma unroll
        for (int e = 0; e < 40; ++e)
          if (ch * 40 + e < kNV) mx = fmaxf(mx, fabsf(v[e]));
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
        const int f = blk * 128 + row;
        const float sf = feature_angle<KIND>(f) < p.M ? scale : 0.f;
        int atom, k;
        feature_to_image<KIND>(f, atom, k);
        float v[40];
        load_state_cols(tmem + lane_addr + blk * kNPad + ch * 40, v);
#pragma unroll
        for (int e = 0; e < 40; ++e) {
          const int nn = ch * 40 + e;
          *reinterpret_cast<__half*>(img + image_byte(atom, nn, k)) =
              __float2half_rn(nn < kNV ? v[e] * sf : 0.f);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      group_sync(bar(ms->epi_sync), eph, abort_flag);
      if (etid == 0) mbar_arrive(bar(ms->img_full));
    }
  } else {
    // Cross-CTA reduction through distributed shared memory. Each CTA stages its fp32 partial
    // state owner-major, as [owner][value column][feature % Fc] with Fc = Fpad / P, in the
    // shared region. After a cluster barrier, CTA r ("owner" of feature rows [r Fc, (r+1) Fc))
    // reads its slice from every CTA, sums the P partials in rank order (each rescaled to the
    // largest stabiliser reference), and rounds to fp16 under a power-of-two scale shared by
    // the cluster. After a second barrier, nobody reads the staging any more: the owner writes
    // its slice of the image into every CTA's image region (which overlaps the staging), and a
    // third barrier publishes it.
    const int Fc = Fpad / P;
    float* stg = reinterpret_cast<float*>(gbase + (s_reg - base));
    if (epi) {
      float mx = 0.f;
      for (int blk = 0; blk < nsb; ++blk) {
        float v[40];
        load_state_cols(tmem + lane_addr + blk * kNPad + ch * 40, v);
        const int f = blk * 128 + row, owner = f / Fc, fl = f - owner * Fc;
#pragma unroll
        for (int e = 0; e < 40; ++e) {
          const int nn = ch * 40 + e;
          if (nn < kNV) {
            stg[(owner * kNV + nn) * Fc + fl] = v[e];
            mx = fmaxf(mx, fabsf(v[e]));
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
        ms->meta[0] = KIND == 0 ? ms->cfinal : 0.f;
        ms->meta[1] = m;
      }
    }
    cluster_sync();
    // every thread: cluster-wide stabiliser reference and image scale (same in every CTA)
    float sc[8];
    float cmax = -INFINITY, bound = 0.f;
    {
      float2 mt[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        mt[q] = q < P ? ld_dsmem_f2(mapa_shared(smem_u32(&ms->meta[0]), q)) : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) cmax = fmaxf(cmax, mt[q].x);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        sc[q] = q < P ? (KIND == 0 ? __expf(mt[q].x - cmax) : 1.f) : 0.f;
        bound += mt[q].y * sc[q];
      }
    }
    const float scale = bound > 0.f ? ldexpf(1.f, 15 - (int)ceilf(log2f(bound))) : 1.f;
    // owner sums: groups of 4 consecutive features, (value column, group) spread over threads
    const int ngrp = kNV * (Fc / 4);
    constexpr int kMaxG = 12;  // groups per thread: ceil(65 * 256 / 4 / 384) = 11 for P = 2
    uint32_t packed[kMaxG][2];
    const uint32_t stg_addr = s_reg + uint32_t(rank * kNV * Fc) * 4u;
#pragma unroll
    for (int gi = 0; gi < kMaxG; ++gi) {
      const int g = tid + gi * kThreads;
      packed[gi][0] = packed[gi][1] = 0u;
      if (g < ngrp) {
        const int nn = g / (Fc / 4), f4 = g - nn * (Fc / 4);
        const uint32_t off = stg_addr + uint32_t(nn * Fc + f4 * 4) * 4u;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < P) {
            const float4 x = ld_dsmem_f4(mapa_shared(off, q));
            acc.x = fmaf(sc[q], x.x, acc.x);
            acc.y = fmaf(sc[q], x.y, acc.y);
            acc.z = fmaf(sc[q], x.z, acc.z);
            acc.w = fmaf(sc[q], x.w, acc.w);
          }
        }
        // zero the rows of padded angles
        const int f = rank * Fc + f4 * 4;
        const float s0 = feature_angle<KIND>(f) < p.M ? scale : 0.f;
        const float s1 = feature_angle<KIND>(f + 1) < p.M ? scale : 0.f;
        const float s2 = feature_angle<KIND>(f + 2) < p.M ? scale : 0.f;
        const float s3 = feature_angle<KIND>(f + 3) < p.M ? scale : 0.f;
        packed[gi][0] = pack_f16x2(acc.x * s0, acc.y * s1);
        packed[gi][1] = pack_f16x2(acc.z * s2, acc.w * s3);
      }
    }
    cluster_sync();
    {
      // rows 65..79 of every atom are zero (the image region overlapped the staging)
      uint8_t* img = gbase + (s_reg - base);
      for (int i = tid; i < natoms * (kNPad - kNV) * 8; i += kThreads) {
        const int atom = i / ((kNPad - kNV) * 8), rem = i - atom * ((kNPad - kNV) * 8);
        *reinterpret_cast<uint4*>(img + atom * kImgAtomB + (kNV + rem / 8) * kRowB + (rem % 8) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int gi = 0; gi < kMaxG; ++gi) {
        const int g = tid + gi * kThreads;
        if (g < ngrp) {
          const int nn = g / (Fc / 4), f4 = g - nn * (Fc / 4);
          int atom, k;
          feature_to_image<KIND>(rank * Fc + f4 * 4, atom, k);
          const uint32_t dst = s_reg + image_byte(atom, nn, k);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q < P) st_dsmem_u2(mapa_shared(dst, q), packed[gi][0], packed[gi][1]);
        }
      }
      fence_proxy_async_cluster();
    }
    cluster_sync();
    if (warp == 0 && lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive(bar(ms->img_full));
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
          tma_load_3d(s_reg + kQOff + s * kTileB, &tm_q, bar(ms->q_full[s]), 0, (t_begin + t) * kTile, bh);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // Query-phase projection issuer: U = Q_tile . Omega_c^T into a 64-column U slot. TMEM
    // columns [0, 320) held the key-phase state until the reduction read it, so nothing is
    // issued before the image is in.
    if (lane == 0) {
      const uint32_t id1 = idesc_f16(128, 64, 1, 1, 0, 0);
      const uint64_t q0 = sdesc_sw128(s_reg + kQOff, 16, 1024);
      const uint64_t o0 = sdesc_sw128(s_om, 16, 1024);
      const int n = my_tiles * nchq;
      bool ok = mbar_wait(bar(ms->s_done), 0, abort_flag) && mbar_wait(bar(ms->img_full), 0, abort_flag);
      int c = 0, s = 0, b = 0;
      uint32_t q_ph = 0, u_ph = 0;
      for (int i = 0; ok && i < n; ++i) {
        if (c == 0 && !(ok = mbar_wait(bar(ms->q_full[s]), q_ph, abort_flag))) break;
        if (i >= kNU && !(ok = mbar_wait(bar(ms->uq_free[b]), u_ph, abort_flag))) break;
        tc_fence_after();
        const uint64_t ad = q0 + uint64_t((s * kTileB) >> 4);
        const uint64_t bd = o0 + uint64_t((c * 64 * kRowB) >> 4);
        const uint32_t d = tmem + kUQ + b * 64;
        mma_ss(d, ad, bd, id1, 0u);
        mma_ss(d, ad + 2, bd + 2, id1, 1u);
        mma_ss(d, ad + 4, bd + 4, id1, 1u);
        mma_ss(d, ad + 6, bd + 6, id1, 1u);
        mma_commit(bar(ms->uq_full[b]));
        if (++b == kNU) { b = 0; if (i >= 2 * kNU - 1) u_ph ^= 1u; }
        if (++c == nchq) {
          mma_commit(bar(ms->q_empty[s]));
          c = 0;
          if (++s == kStagesQ) { s = 0; q_ph ^= 1u; }
        }
      }
      mma_commit(bar(ms->mma_drain1));
    }
    __syncwarp();
  } else if (warp == 2) {
    // Query-phase numerator issuer: num += phi_c . S_c, A from TMEM, B = state image.
    if (lane == 0) {
      const uint32_t id2 = idesc_f16(128, kNPad, 0, 0, 0, 0);
      const uint64_t g0 = sdesc_sw128(s_reg, 16, 1024);
      const int n = my_tiles * nchq;
      bool ok = mbar_wait(bar(ms->img_full), 0, abort_flag);
      int c = 0, pb = 0, nb = 0;
      uint32_t p_ph = 0, n_ph = 1;  // the first wait on an empty numerator passes at once
      for (int i = 0; ok && i < n; ++i) {
        if (!(ok = mbar_wait(bar(ms->pq_full[pb]), p_ph, abort_flag))) break;
        if (c == 0 && !(ok = mbar_wait(bar(ms->num_empty[nb]), n_ph, abort_flag))) break;
        tc_fence_after();
        const uint32_t acol = tmem + kPQ + pb * PWQ;
        const uint32_t dn = tmem + nb * kNPad;
        if (KIND == 0) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bd = g0 + uint64_t(((2 * c + (kk >> 2)) * kImgAtomB + (kk & 3) * 32) >> 4);
            mma_ts(dn, acol + kk * 8, bd, id2, (c > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = g0 + uint64_t((c * kImgAtomB + kk * 32) >> 4);
            mma_ts(dn, acol + kk * 8, bd, id2, (c > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(bar(ms->pq_free[pb]));
        if (++pb == kNPQ) { pb = 0; p_ph ^= 1u; }
        if (++c == nchq) {
          mma_commit(bar(ms->num_full[nb]));
          c = 0;
          if (++nb == 2) { nb = 0; n_ph ^= 1u; }
        }
      }
      mma_commit(bar(ms->mma_drain));
    }
    __syncwarp();
  } else if (warp >= 4) {
    // Query-phase epilogue: items alternate between the warpgroups; an item is two sub-items
    // of 32 angle columns, and the next sub-item's load overlaps the current compute. The
    // group holding a tile's last chunk (always warpgroup 1: nchq is even) normalises the
    // tile and stores it.
    const int grp = ch;
    const int n = my_tiles * nchq;
    uint32_t oph = 0;                              // phase of this group's output barrier
    const bool issuer = (q4 == 0 && lane == 0);    // first thread of the group
    int i = grp, hs = 0;
    uint32_t ua[32], ub[32];
    bool have = i < n, loaded = false;
    auto issue = [&](int ii, int hh, uint32_t (&dst)[32], bool block) -> bool {
      if (hh == 0) {
        const uint32_t bb = bar(ms->uq_full[ii % kNU]), ph = (ii / kNU) & 1;
        if (!(block ? mbar_wait(bb, ph, abort_flag) : mbar_test(bb, ph))) return false;
      }
      tc_fence_after();
      tmem_ld32(tmem + lane_addr + kUQ + (ii % kNU) * 64 + hh * 32, dst);
      return true;
    };
    auto step = [&](uint32_t (&cur)[32], uint32_t (&nxt)[32]) -> bool {
      if (!loaded && !issue(i, hs, cur, true)) return false;
      tmem_wait_ld();
      const int b = i % kNU, pb = i % kNPQ;
      int i2 = i, h2 = hs + 1;
      if (h2 == 2) { h2 = 0; i2 = i + 2; }
      if (hs == 1) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->uq_free[b]));
      }
      const bool more = i2 < n;
      loaded = more && issue(i2, h2, nxt, false);
      if (hs == 0) {
        if (i >= kNPQ && !mbar_wait(bar(ms->pq_free[pb]), ((i / kNPQ) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
      }
      const uint32_t paddr = tmem + lane_addr + kPQ + pb * PWQ;
      if (KIND == 0) {
        trig_cols<true>(cur, paddr + hs * 32);
      } else {
        relu_cols<true>(cur, paddr + hs * 16);
      }
      if (hs == 1) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->pq_full[pb]));
        const int t = i / nchq, c = i % nchq;
        if (c == nchq - 1) {  // this group owns the tile's last chunk: normalise and store
          const int nb = t & 1;
          if (!mbar_wait(bar(ms->num_full[nb]), (t >> 1) & 1, abort_flag)) return false;
          tc_fence_after();
          uint32_t nv[32], dv;
          tmem_ld1(tmem + lane_addr + nb * kNPad + 64, dv);
          const int sb = t & 1;
          if (issuer && t >= 2) bulk_wait_read1();
          group_sync(bar(ms->out_sync[grp]), oph, abort_flag);
          uint8_t* stg = gbase + (s_reg + kOutOff - base) + sb * kTileB + row * kRowB;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld32(tmem + lane_addr + nb * kNPad + half * 32, nv);
            tmem_wait_ld();
            const float den = __uint_as_float(dv);
            const float inv = den != 0.f ? 1.f / den : 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m)
              *reinterpret_cast<uint4*>(stg + (((half * 4 + m) ^ (row & 7)) << 4)) = make_uint4(
                  pack_bf16x2(__uint_as_float(nv[8 * m]) * inv, __uint_as_float(nv[8 * m + 1]) * inv),
                  pack_bf16x2(__uint_as_float(nv[8 * m + 2]) * inv, __uint_as_float(nv[8 * m + 3]) * inv),
                  pack_bf16x2(__uint_as_float(nv[8 * m + 4]) * inv, __uint_as_float(nv[8 * m + 5]) * inv),
                  pack_bf16x2(__uint_as_float(nv[8 * m + 6]) * inv, __uint_as_float(nv[8 * m + 7]) * inv));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(ms->num_empty[nb]));
          fence_proxy_async_smem();
          group_sync(bar(ms->out_sync[grp]), oph, abort_flag);
          if (issuer) {
            tma_store_3d(&tm_out, s_reg + kOutOff + sb * kTileB, 0, (t_begin + t) * kTile, bh);
            bulk_commit();
          }
        }
      }
      i = i2;
      hs = h2;
      return more;
    };
    while (have) {
      if (!(have = step(ua, ub))) break;
      have = step(ub, ua);
    }
    if (issuer) bulk_wait0();
  }

  // ================================================================ teardown
  if (warp == 1) mbar_wait(bar(ms->mma_drain1), 0, nullptr, 200000000ll);
  if (warp == 2) mbar_wait(bar(ms->mma_drain), 0, nullptr, 200000000ll);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace favor
