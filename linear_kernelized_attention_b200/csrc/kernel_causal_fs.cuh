// kernel_causal_fs.cuh - causal FAVOR forward on sm_100a tensor cores: a chunked prefix scan
// with the features split across a thread-block cluster.
//
// What it computes. The explainer page "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？",
// section 核心机制：FAVOR+: the causal variant keeps the prefix sum
// S_i = sum_{j <= i} phi(k_j) [v_j | 1]^T, and out_i = (phi(q_i) S_i)[:d] / (phi(q_i) S_i)[d].
//
// Blocking. Tokens are taken in 128-token chunks c. With S_{<c} the state of all earlier chunks,
//   out_c = phi(Q_c) S_{<c} + tril(phi(Q_c) phi(K_c)^T) [V_c | 1]   (keys j <= i of the chunk)
//   S_{<c+1} = S_{<c} + phi(K_c)^T [V_c | 1].
// The first term ("inter") reads the state; the second ("intra") is a masked 128 x 128 product.
//
// Parallel split. One thread-block cluster of G CTAs per (batch, head); CTA g owns 64 angles
// (trig: 128 features as interleaved cos/sin pairs; ReLU: 64 features), so every CTA walks the
// whole sequence with its own state slab in TMEM. num and den are sums over features, so the G
// partial rows add: the rows of a chunk are cut into eight 16-row blocks, block b belongs to CTA
// b % G, every CTA deposits its partial rows (numerators in bf16, the denominator in fp32; two
// deposit buffers by chunk parity) with the block's owner, and a combiner warp there sums them
// in CTA order, divides and stores.
//
// Stabiliser (trig). Key features carry exp(|k_j|^2/2). The state S_{<c} is kept relative to the
// running reference cref_c = max |k_j|^2/2 over earlier chunks; row i of chunk c uses its own
// reference R_i = max(cref_c, max_{j <= i in c} |k_j|^2/2), so every weight is <= 1 and no row's
// terms vanish under another row's larger keys:
//   intra_ij = P_ij exp(|k_j|^2/2 - R_i), inter_i scaled by exp(cref_c - R_i).
// The key weight is folded into the stored key features, phi'(k_j) = a_j phi(k_j):
//   usual chunks: a_j = exp(|k_j|^2/2 - cnew_c), cnew_c = max(cref_c, chunk max). Then
//     P' = phi(Q) phi'(K)^T needs only the causal mask, the row factor rho_i = exp(cnew_c - R_i)
//     is applied to the intra sums once, and S += phi'(K)^T [V | 1] reads the V tile as it is.
//   chunks whose keys rise more than 2^80 above R_0 (e.g. the first large key of a sequence):
//     a_j = exp(|k_j|^2/2 - R_j), P16_ij = P'_ij exp(R_j - R_i) per element, and the state update
//     uses [u o V | u] with u_j = exp(R_j - cnew_c). A weight that underflows there is below 2^-46
//     of its row's largest weight.
// After chunk c the state is rescaled from cref_c to cnew_c before the chunk's keys are added.
// Factors that cancel in the ratio (1/sqrt(M), exp(|q|^2/2)) are dropped. ReLU uses unit weights.
//
// Per chunk (bf16 operands, fp32 accumulation in TMEM):
//   issuer A:  U_K = K_c Omega_g^T (N = 64)                    -> phi'(K) in smem (2 buffers)
//              S += phi'(K)^T V  (M = 128 feature rows, N = 64)  z += phi'(K)^T 1  (N = 16)
//   issuer B:  U_Q = Q_c Omega_g^T (N = 64)                    -> phi(Q) in TMEM (2 slots, in place)
//              P' = phi(Q) phi'(K)^T (N = 128), inter = phi(Q) S_img (bf16 image of S_{<c}),
//              phi(Q).z with z split into bf16 hi and lo rows, intra = P16 V_c
// The intra denominator sum_j P16_ij is accumulated in fp32 registers.
//
// Warp roles (640 threads): 0 TMA; 1 TMEM allocator and issuer A (U_K(c + 1) is issued before
// the state update of chunk c); 2 issuer B; 3 key norms and references; 4-7 phi'(K) (thread =
// key row); 8-11 the state image, then phi(Q) (thread = feature row, then query row; two phi(Q)
// slots, so the next chunk's features overlap this chunk's products); 12-15 P16 and partial rows
// (thread = query row); 16-19 combiner of the owned rows (thread = a quarter of a row).
// Head sizes 16 and 32 ride in the 64-column boxes (zeros past d).
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "sincos_poly.cuh"

namespace favor {
namespace cf {

constexpr int kTile = 128;
constexpr int kRowB = 128;
constexpr int kTileB = kTile * kRowB;  // 16 KB
constexpr int kThreads = 640;
#ifndef FAVOR_POLY_MASK_CAUSAL
#define FAVOR_POLY_MASK_CAUSAL 0x00u
#endif
constexpr uint32_t kPolyMask = FAVOR_POLY_MASK_CAUSAL;
// Shared memory (offsets from the 1024-aligned base).
constexpr int kC_OM = 0;              // Omega rows of this CTA's angles (one 128-row box)
constexpr int kC_K = 16 * 1024;       // K tile
constexpr int kC_V = 32 * 1024;       // V stages, 2 x 16 KB (V_c stays until its intra MMA)
constexpr int kC_Q = 64 * 1024;       // Q tile
constexpr int kC_PHK = 80 * 1024;     // phi(K): 2 buffers x 2 atoms of 64 features x 128 keys
constexpr int kPhkB = 2 * kTileB;     // one phi(K) buffer
constexpr int kC_VW = 144 * 1024;     // [u o V] bf16 (trig, large-rise chunks), the V tile's layout
constexpr int kC_WROW = 160 * 1024;   // 1 (or u) as row 0 of a 16 x 128 K-major operand (2 x 2 KB)
constexpr int kC_ZROW = 164 * 1024;   // z of S_{<c} (hi, lo) as rows 0, 1 of a 16 x 128 operand
constexpr int kC_IMG = 168 * 1024;    // state image bf16: 128 feature rows x 64 values
constexpr int kC_RECV = 184 * 1024;   // partial rows deposited for the rows this CTA owns
constexpr int kRecvRowB = 144;        // one partial row: 64 bf16 numerators, fp32 denominator, pad
constexpr int kRecvBufB = 128 * kRecvRowB;  // 128 row slots (owned blocks x senders x 16 rows)
constexpr int kRecvB = 2 * kRecvBufB;       // two buffers, by chunk parity
constexpr int kC_SMALL = kC_RECV + kRecvB;  // per-chunk scalars and vectors (CausalSmall)
constexpr int kC_MISC = kC_SMALL + 5120;    // barriers (CausalMisc)
constexpr int kMeta = 4;                     // chunks of key metadata in flight
// TMEM columns.
constexpr uint32_t kT_S = 0;          // state slab: 64 value columns + 16 (column 64 = z)
constexpr uint32_t kT_PR = 80;        // P (128 fp32) -> P16 [80, 144) + intra [144, 208)
constexpr uint32_t kT_IN = 208;       // inter accumulator (64 columns) + phi(Q).z (16; column 64)
constexpr uint32_t kT_A = 288;        // phi(Q) slots: U_Q (64 columns) -> phi(Q) packed bf16, 2 x 64
constexpr uint32_t kT_B = 416;        // U_K, 64 columns

struct CausalParams {
  int BH, H, L, M;   // heads (B*H), heads per batch, tokens, random features
  int G;             // CTAs per head (64-angle blocks): 1, 2, 4 or 8
  int nch;           // ceil(L / 128)
  int d;             // head dimension (16, 32 or 64)
};

struct CausalSmall {
  float rl[kMeta][128];      // row references R_i * log2(e), by chunk % kMeta
  float wk[kMeta][128];      // key feature weights a_j, by chunk % kMeta
  float crefl[kMeta], cnewl[kMeta];  // references of S_{<c} and S_{<=c} (log2 units)
  int fb[kMeta];             // 1: the chunk takes the large-rise weights
};
static_assert(sizeof(CausalSmall) <= 5120, "causal small block");

struct alignas(16) CausalMisc {
  int abort_flag;
  uint32_t tmem_base;
  int pad[2];
  uint64_t om_full, k_full, k_empty, v_full[2], v_empty[2], q_full, q_empty;
  uint64_t meta_full[kMeta], meta_free[kMeta], vw_full;
  uint64_t uk_full, uk_free, uq_full[2], slot_free[2], phiq_full[2];
  uint64_t p_full, s_done, o_full, drain_a, drain_b;
  uint64_t img_full, img_free, s_ready, p16_full, pr_free;
  uint64_t phik_full[2], phik_free[2];  // per phi(K) buffer
  uint64_t recv_full[2], recv_free[2];  // per deposit buffer
  uint64_t comb_sync;                   // bounded barrier among the 128 combiner threads
};
static_assert(sizeof(CausalMisc) <= 1024, "causal misc block");

__host__ __device__ constexpr uint32_t causal_smem_bytes() { return kC_MISC + 1024 + 1024; }

// Store one output row of d (16, 32 or 64) values, scaled by inv, as bf16.
__device__ __forceinline__ void store_row(__nv_bfloat16* dst, const float* nm, float inv, int d) {
  uint4* o = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (8 * q < d)
      o[q] = make_uint4(pack_bf16x2(nm[8 * q] * inv, nm[8 * q + 1] * inv),
                        pack_bf16x2(nm[8 * q + 2] * inv, nm[8 * q + 3] * inv),
                        pack_bf16x2(nm[8 * q + 4] * inv, nm[8 * q + 5] * inv),
                        pack_bf16x2(nm[8 * q + 6] * inv, nm[8 * q + 7] * inv));
}

// KIND: 0 trig, 1 ReLU. Every CTA owns 64 angles.
template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    k_causal_fs(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_om,
                const CausalParams p, __nv_bfloat16* __restrict__ out) {
  constexpr int NA = 64;
  constexpr int NKS = KIND == 0 ? 8 : 4;        // 16-feature steps of the feature contractions
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kNegBig = -1.0e30f;           // reference before any key; weight of padded keys
  constexpr float kSplitMax = 80.f;             // largest reference jump (log2) for w_j rho_i

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (base - raw);
  CausalMisc* ms = reinterpret_cast<CausalMisc*>(gb + kC_MISC);
  CausalSmall* sm = reinterpret_cast<CausalSmall*>(gb + kC_SMALL);
  volatile int* abort_flag = &ms->abort_flag;
  auto bar = [](uint64_t& b) { return smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G, L = p.L, nch = p.nch;
  const int g = blockIdx.x % G;
  const int bh = blockIdx.x / G;
  const int h = bh % p.H;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    ms->abort_flag = 0;
    mbar_init(bar(ms->om_full), 1);
    mbar_init(bar(ms->k_full), 1);
    mbar_init(bar(ms->k_empty), 2);        // key-norm warp + issuer A (U_K)
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ms->v_full[s]), 1);
      mbar_init(bar(ms->v_empty[s]), 3);   // key-norm warp + issuer A (S) + issuer B (intra)
      mbar_init(bar(ms->uq_full[s]), 1);
      mbar_init(bar(ms->slot_free[s]), 1);
      mbar_init(bar(ms->phiq_full[s]), 4);
      mbar_init(bar(ms->phik_full[s]), 4);
      mbar_init(bar(ms->phik_free[s]), 1);  // issuer B's commit after P
      mbar_init(bar(ms->recv_full[s]), 128);  // every deposited row of every CTA of the cluster
      mbar_init(bar(ms->recv_free[s]), G);    // one release from every owner
    }
    for (int b = 0; b < kMeta; ++b) {
      mbar_init(bar(ms->meta_full[b]), 32);
      mbar_init(bar(ms->meta_free[b]), 4);
    }
    mbar_init(bar(ms->q_full), 1);
    mbar_init(bar(ms->q_empty), 1);
    mbar_init(bar(ms->vw_full), 32);
    mbar_init(bar(ms->uk_full), 1);
    mbar_init(bar(ms->uk_free), 4);
    mbar_init(bar(ms->p_full), 1);
    mbar_init(bar(ms->s_done), 1);
    mbar_init(bar(ms->o_full), 1);
    mbar_init(bar(ms->drain_a), 1);
    mbar_init(bar(ms->drain_b), 1);
    mbar_init(bar(ms->img_full), 4);
    mbar_init(bar(ms->img_free), 1);      // issuer B's commit after the inter and z MMAs
    mbar_init(bar(ms->s_ready), 4);
    mbar_init(bar(ms->p16_full), 4);
    mbar_init(bar(ms->pr_free), 4);
    mbar_init(bar(ms->comb_sync), 128);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish();
  }
  {  // phi(K) buffers zero (ReLU keeps features 64..127 of a block zero); the w row operand zero
     // except row 0, which is 1 (trig large-rise chunks rewrite it); the z operand zero
    uint4* phk = reinterpret_cast<uint4*>(gb + kC_PHK);
    for (int i = tid; i < 2 * kPhkB / 16; i += kThreads) phk[i] = make_uint4(0u, 0u, 0u, 0u);
    uint4* wr = reinterpret_cast<uint4*>(gb + kC_WROW);  // the w and z operands, 8 KB
    for (int i = tid; i < 8192 / 16; i += kThreads) wr[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    if (tid < kTile) *reinterpret_cast<uint16_t*>(gb + kC_WROW + (tid >> 6) * 2048 + (tid & 63) * 2) = 0x3F80u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (G > 1) cluster_sync();  // the partners' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  const uint32_t id_uk = idesc_f16(128, 64, 1, 1, 0, 0);
  const uint32_t id_p = idesc_f16(128, 128, 1, 1, 0, 0);
  const uint32_t id_in = idesc_f16(128, 64, 1, 1, 0, 1);
  const uint32_t id_s = idesc_f16(128, 64, 1, 1, 1, 1);
  const uint32_t id_z = idesc_f16(128, 16, 1, 1, 1, 0);
  const uint32_t id_qz = idesc_f16(128, 16, 1, 1, 0, 0);
  const uint32_t id_it = idesc_f16(128, 64, 1, 1, 0, 1);
  constexpr uint64_t kKStep = (16 * kRowB) >> 4;  // 16 rows of an MN-major operand

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (whole warp; the
    // elected lane issues the copies)
    {
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_q);
        mbar_arrive_expect_tx(bar(ms->om_full), kTileB);
        tma_load_3d(base + kC_OM, &tm_om, bar(ms->om_full), 0, g * NA, h);
      }
      int k_issued = 0, v_issued = 0, q_issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        if (c >= 1 && !mbar_wait(bar(ms->k_empty), (c - 1) & 1, abort_flag)) break;
        if (leader) {
          mbar_arrive_expect_tx(bar(ms->k_full), kTileB);
          tma_load_3d(base + kC_K, &tm_k, bar(ms->k_full), 0, c * kTile, bh);
        }
        k_issued = c + 1;
        if (c >= 2 && !mbar_wait(bar(ms->v_empty[s]), ((c >> 1) - 1) & 1, abort_flag)) break;
        if (leader) {
          mbar_arrive_expect_tx(bar(ms->v_full[s]), kTileB);
          tma_load_3d(base + kC_V + s * kTileB, &tm_v, bar(ms->v_full[s]), 0, c * kTile, bh);
        }
        v_issued = c + 1;
        if (c >= 1 && !mbar_wait(bar(ms->q_empty), (c - 1) & 1, abort_flag)) break;
        if (leader) {
          mbar_arrive_expect_tx(bar(ms->q_full), kTileB);
          tma_load_3d(base + kC_Q, &tm_q, bar(ms->q_full), 0, c * kTile, bh);
        }
        q_issued = c + 1;
      }
      // On an abort, let the copies already issued land before the CTA can exit.
      if (*abort_flag) {
        constexpr long long kDrain = kWaitLimitCycles / 8;
        mbar_wait(bar(ms->om_full), 0, nullptr, kDrain);
        if (k_issued > 0) mbar_wait(bar(ms->k_full), (k_issued - 1) & 1, nullptr, kDrain);
        for (int c = v_issued > 2 ? v_issued - 2 : 0; c < v_issued; ++c)
          mbar_wait(bar(ms->v_full[c & 1]), (c >> 1) & 1, nullptr, kDrain);
        if (q_issued > 0) mbar_wait(bar(ms->q_full), (q_issued - 1) & 1, nullptr, kDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ issuer A: U_K, S and z (whole
    // warp; the elected lane issues)
    {
      const bool leader = elect_one();
      const uint64_t d_om = sdesc_sw128(base + kC_OM, 16, 1024);
      const uint64_t d_k = sdesc_sw128(base + kC_K, 16, 1024);
      const uint64_t d_phk_a = sdesc_sw128(base + kC_PHK, kTileB, 1024);  // MN-major A of S, z
      const uint64_t d_vw = sdesc_sw128(base + kC_VW, kTileB, 1024);
      const uint64_t d_v0 = sdesc_sw128(base + kC_V, kTileB, 1024);
      const uint64_t d_wr = sdesc_sw128(base + kC_WROW, 16, 1024);        // K-major B of z
      auto uk = [&](int c) -> bool {
        if (!mbar_wait(bar(ms->k_full), c & 1, abort_flag)) return false;
        if (c > 0 && !mbar_wait(bar(ms->uk_free), (c - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + kT_B, d_k + 2 * kk, d_om + 2 * kk, id_uk, kk > 0 ? 1u : 0u);
          mma_commit(bar(ms->uk_full));
          mma_commit(bar(ms->k_empty));  // the K tile has been read
        }
        __syncwarp();
        return true;
      };
      bool ok = mbar_wait(bar(ms->om_full), 0, abort_flag) && (nch == 0 || uk(0));
      for (int c = 0; ok && c < nch; ++c) {
        // U_K(c + 1) first: it needs only the next K tile and the phi(K) warps' copy of U_K(c), so
        // their next chunk does not wait for this chunk's state image and update
        if (c + 1 < nch && !(ok = uk(c + 1))) break;
        // S += phi(K)^T [w o V], z += phi(K)^T w
        if (!(ok = mbar_wait(bar(ms->phik_full[c & 1]), (c >> 1) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(bar(ms->s_ready), c & 1, abort_flag))) break;
        if (!(ok = mbar_wait(bar(ms->vw_full), c & 1, abort_flag))) break;
        tc_fence_after();
        const uint64_t a = d_phk_a + uint64_t(((c & 1) * kPhkB) >> 4);
        const bool use_vw = KIND == 0 && sm->fb[c & (kMeta - 1)];
        const uint64_t bvw = use_vw ? d_vw : d_v0 + uint64_t(((c & 1) * kTileB) >> 4);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
            mma_ss(tmem + kT_S, a + kk * kKStep, bvw + kk * kKStep, id_s, acc);
            mma_ss(tmem + kT_S + 64, a + kk * kKStep, d_wr + uint64_t(((kk >> 2) * 2048 + (kk & 3) * 32) >> 4),
                   id_z, acc);
          }
          mma_commit(bar(ms->s_done));
          mma_commit(bar(ms->v_empty[c & 1]));  // the V tile has been read
        }
        __syncwarp();
      }
      if (leader) mma_commit(bar(ms->drain_a));
      __syncwarp();
      mbar_wait(bar(ms->drain_a), 0, nullptr, kWaitLimitCycles / 8);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ issuer B: U_Q, P, inter, intra
    // (whole warp; the elected lane issues)
    {
      const bool leader = elect_one();
      const uint64_t d_om = sdesc_sw128(base + kC_OM, 16, 1024);
      const uint64_t d_q = sdesc_sw128(base + kC_Q, 16, 1024);
      const uint64_t d_v0 = sdesc_sw128(base + kC_V, kTileB, 1024);
      const uint64_t d_phk_b = sdesc_sw128(base + kC_PHK, 16, 1024);  // K-major B of P
      const uint64_t d_img = sdesc_sw128(base + kC_IMG, kTileB, 1024);
      const uint64_t d_zr = sdesc_sw128(base + kC_ZROW, 16, 1024);  // K-major B of phi(Q).z
      // U_Q(c) into phi(Q) slot c & 1, once P(c - 2) and inter(c - 2) have read that slot
      auto uq = [&](int c) -> bool {
        if (!mbar_wait(bar(ms->q_full), c & 1, abort_flag)) return false;
        if (c >= 2 && !mbar_wait(bar(ms->slot_free[c & 1]), ((c >> 1) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + kT_A + (c & 1) * 64, d_q + 2 * kk, d_om + 2 * kk, id_uk, kk > 0 ? 1u : 0u);
          mma_commit(bar(ms->uq_full[c & 1]));
          mma_commit(bar(ms->q_empty));
        }
        __syncwarp();
        return true;
      };
      bool ok = mbar_wait(bar(ms->om_full), 0, abort_flag) && (nch == 0 || uq(0)) && (nch < 2 || uq(1));
      for (int c = 0; ok && c < nch; ++c) {
        const uint32_t slot = tmem + kT_A + (c & 1) * 64;
        // P(c) = phi(Q) phi(K)^T
        if (!(ok = mbar_wait(bar(ms->phik_full[c & 1]), (c >> 1) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(bar(ms->phiq_full[c & 1]), (c >> 1) & 1, abort_flag))) break;
        if (c >= 1 && !(ok = mbar_wait(bar(ms->pr_free), (c - 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint64_t bk = d_phk_b + uint64_t(((c & 1) * kPhkB) >> 4);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < NKS; ++kk)
            mma_ts(tmem + kT_PR, slot + 8 * kk, bk + uint64_t(((kk >> 2) * kTileB + (kk & 3) * 32) >> 4), id_p,
                   kk > 0 ? 1u : 0u);
          mma_commit(bar(ms->p_full));
          mma_commit(bar(ms->phik_free[c & 1]));
        }
        __syncwarp();
        // inter(c) = phi(Q) S_img and phi(Q).z
        if (!(ok = mbar_wait(bar(ms->img_full), c & 1, abort_flag))) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < NKS; ++kk) {
            mma_ts(tmem + kT_IN, slot + 8 * kk, d_img + kk * kKStep, id_in, kk > 0 ? 1u : 0u);
            mma_ts(tmem + kT_IN + 64, slot + 8 * kk, d_zr + uint64_t(((kk >> 2) * 2048 + (kk & 3) * 32) >> 4),
                   id_qz, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(ms->img_free));
          mma_commit(bar(ms->slot_free[c & 1]));
        }
        __syncwarp();
        // intra(c) = P16 V_c
        if (!(ok = mbar_wait(bar(ms->p16_full), c & 1, abort_flag))) break;
        if (!(ok = mbar_wait(bar(ms->v_full[c & 1]), (c >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint64_t bv = d_v0 + uint64_t(((c & 1) * kTileB) >> 4);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kT_PR + 64, tmem + kT_PR + 8 * kk, bv + kk * kKStep, id_it, kk > 0 ? 1u : 0u);
          mma_commit(bar(ms->o_full));
          mma_commit(bar(ms->v_empty[c & 1]));  // the V tile has been read
        }
        __syncwarp();
        // U_Q(c + 2) into this chunk's slot
        if (c + 2 < nch && !(ok = uq(c + 2))) break;
      }
      if (leader) mma_commit(bar(ms->drain_b));
      __syncwarp();
      mbar_wait(bar(ms->drain_b), 0, nullptr, kWaitLimitCycles / 8);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ key norms and references
    float crefl = kNegBig;
    bool prev_fb = false;
    for (int c = 0; c < nch; ++c) {
      const int s = c & 1, mb = c & (kMeta - 1);
      if (!mbar_wait(bar(ms->k_full), c & 1, abort_flag)) break;
      if (c >= kMeta && !mbar_wait(bar(ms->meta_free[mb]), ((c / kMeta) - 1) & 1, abort_flag)) break;
      const int row0 = c * kTile;
      float cnewl = 0.f;
      bool fb = false;
      if (KIND == 0) {
        // |k_j|^2/2 (log2 units; kept in wk until the weights are known) and R_j, the
        // inclusive prefix max over the chunk's keys in order, seeded with cref
        float run = crefl;
#pragma unroll 1
        for (int jj = 0; jj < 4; ++jj) {
          const int j = lane + 32 * jj;
          float acc = 0.f;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 x = *reinterpret_cast<const uint4*>(gb + kC_K + j * kRowB + ((ch ^ (j & 7)) << 4));
            const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xFFFF0000u);
              acc = fmaf(lo, lo, acc);
              acc = fmaf(hi, hi, acc);
            }
          }
          const float nl = row0 + j < L ? 0.5f * acc * kLog2e : kNegBig;
          float x = nl;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x = fmaxf(x, y);
          }
          x = fmaxf(x, run);
          sm->rl[mb][j] = x;
          sm->wk[mb][j] = nl;
          run = __shfl_sync(0xffffffffu, x, 31);
        }
        cnewl = run;
        __syncwarp();
        // every R_i >= R_0, so rho_i = 2^(cnewl - rl_i) <= 2^(cnewl - R_0)
        fb = cnewl - sm->rl[mb][0] > kSplitMax;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = lane + 32 * jj;
          sm->wk[mb][j] = ex2_approx(sm->wk[mb][j] - (fb ? sm->rl[mb][j] : cnewl));
        }
      }
      if (lane == 0) {
        sm->crefl[mb] = crefl;
        sm->cnewl[mb] = cnewl;
        sm->fb[mb] = fb ? 1 : 0;
      }
      mbar_arrive(bar(ms->meta_full[mb]));
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->k_empty));
      if (!mbar_wait(bar(ms->v_full[s]), (c >> 1) & 1, abort_flag)) break;
      // the previous state update has read [u o V] and the w row (this also keeps vw_full at
      // most one phase ahead of its waiter)
      if (c >= 1 && !mbar_wait(bar(ms->s_done), (c - 1) & 1, abort_flag)) break;
      if (KIND == 0 && (fb || prev_fb)) {
        // large-rise chunk: [u o V] and u in row 0 of the w operand; the next chunk restores 1
        const uint8_t* vt = gb + kC_V + s * kTileB;
#pragma unroll 1
        for (int jj = 0; jj < 4; ++jj) {
          const int j = lane + 32 * jj;
          const float u = fb ? ex2_approx(sm->rl[mb][j] - cnewl) : 1.f;
          if (fb) {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const uint32_t off = j * kRowB + ((ch ^ (j & 7)) << 4);
              const uint4 x = *reinterpret_cast<const uint4*>(vt + off);
              const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
              uint32_t o4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                o4[e] = pack_bf16x2(__uint_as_float(w4[e] << 16) * u, __uint_as_float(w4[e] & 0xFFFF0000u) * u);
              *reinterpret_cast<uint4*>(gb + kC_VW + off) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
          }
          *reinterpret_cast<__nv_bfloat16*>(gb + kC_WROW + (j >> 6) * 2048 + (j & 63) * 2) = __float2bfloat16_rn(u);
        }
        fence_proxy_async_smem();
      }
      prev_fb = fb;
      mbar_arrive(bar(ms->vw_full));
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->v_empty[s]));
      crefl = cnewl;
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ phi(K)
    const int q4 = warp & 3, row = q4 * 32 + lane;
    const uint32_t la = uint32_t(q4 * 32) << 16;
    // phi'(K_c) = a_j phi(k_j) into buffer c & 1, once P(c-2) and S(c-2) have read that buffer
    // (S(c-2) is complete: the state image of chunk c-1 waited for it)
    auto phi_k = [&](int c) -> bool {
      if (c >= 2 && !mbar_wait(bar(ms->phik_free[c & 1]), ((c >> 1) - 1) & 1, abort_flag)) return false;
      float aw = 1.f;
      if (KIND == 0) {
        if (!mbar_wait(bar(ms->meta_full[c & (kMeta - 1)]), (c / kMeta) & 1, abort_flag)) return false;
        aw = sm->wk[c & (kMeta - 1)][row];
      }
      uint8_t* dstb = gb + kC_PHK + (c & 1) * kPhkB + row * kRowB;
      if (!mbar_wait(bar(ms->uk_full), c & 1, abort_flag)) return false;
      tc_fence_after();
#pragma unroll 1
      for (int gi = 0; gi < 4; ++gi) {
        uint32_t u[16];
        tmem_ld16(tmem + la + kT_B + 16 * gi, u);
        tmem_wait_ld();
        if (gi == 3) {
          tc_fence_before();  // U_K is in registers: the next chunk's projection may overwrite it
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(ms->uk_free));
        }
        if (KIND == 0) {
          // angle a -> features (2a, 2a+1) = (cos, sin): atom a / 32, 4 angles per 16 bytes
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int a = 16 * gi + 4 * q + e;
              float sn, cs;
              sincos_mixed<kPolyMask>(4 * q + e, __uint_as_float(u[4 * q + e]), sn, cs);
              pk[e] = g * NA + a < p.M ? pack_bf16x2(cs * aw, sn * aw) : 0u;
            }
            const int ch = (gi & 1) * 4 + q;
            *reinterpret_cast<uint4*>(dstb + (gi >> 1) * kTileB + ((ch ^ (row & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
          // angle a -> feature a: 8 features per 16 bytes (padded angles give max(0, 0) = 0)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              pk[e] = pack_bf16x2(fmaxf(__uint_as_float(u[8 * q + 2 * e]), 0.f),
                                  fmaxf(__uint_as_float(u[8 * q + 2 * e + 1]), 0.f));
            const int ch = 2 * gi + q;
            *reinterpret_cast<uint4*>(dstb + ((ch ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->phik_full[c & 1]));
      return true;
    };
    for (int c = 0; c < nch; ++c)
      if (!phi_k(c)) break;
  } else if (warp < 12) {
    // ------------------------------------------------------------ state image and phi(Q)
    // (thread = feature row for the image, query row for phi(Q); two phi(Q) slots)
    const int q4 = warp & 3, row = q4 * 32 + lane;
    const uint32_t la = uint32_t(q4 * 32) << 16;
    // z_f as bf16 hi + lo parts in rows 0 and 1 of the K-major z operand (128-byte swizzle)
    auto zrow_store = [&](float z) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(z);
      const __nv_bfloat16 lo = __float2bfloat16_rn(z - __bfloat162float(hi));
      uint8_t* zb = gb + kC_ZROW + (row >> 6) * 2048 + (row & 7) * 2;
      const int ch = (row & 63) >> 3;
      *reinterpret_cast<__nv_bfloat16*>(zb + (ch << 4)) = hi;
      *reinterpret_cast<__nv_bfloat16*>(zb + kRowB + ((ch ^ 1) << 4)) = lo;
    };
    bool ok = true;
    for (int c = 0; ok && c < nch; ++c) {
      const int mb = c & (kMeta - 1);
      // image of S_{<c} at reference cref_c, then S rescaled to cnew_c
      if (c >= 1 && !(ok = mbar_wait(bar(ms->s_done), (c - 1) & 1, abort_flag))) break;
      if (!(ok = mbar_wait(bar(ms->meta_full[mb]), (c / kMeta) & 1, abort_flag))) break;
      if (c >= 1 && !(ok = mbar_wait(bar(ms->img_free), (c - 1) & 1, abort_flag))) break;
      tc_fence_after();
      uint8_t* img = gb + kC_IMG + row * kRowB;
      if (c == 0) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(img + (ch << 4)) = make_uint4(0u, 0u, 0u, 0u);
        zrow_store(0.f);
      } else {
        uint32_t a[32], b[32], zz[16];
        tmem_ld32(tmem + la + kT_S, a);
        tmem_ld32(tmem + la + kT_S + 32, b);
        tmem_ld16(tmem + la + kT_S + 64, zz);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t* src = ch < 4 ? a + 8 * ch : b + 8 * (ch - 4);
          uint4 o;
          o.x = pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1]));
          o.y = pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3]));
          o.z = pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5]));
          o.w = pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7]));
          *reinterpret_cast<uint4*>(img + ((ch ^ (row & 7)) << 4)) = o;
        }
        zrow_store(__uint_as_float(zz[0]));
        if (KIND == 0) {
          const float rho = ex2_approx(sm->crefl[mb] - sm->cnewl[mb]);
          if (rho != 1.f) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              a[e] = __float_as_uint(__uint_as_float(a[e]) * rho);
              b[e] = __float_as_uint(__uint_as_float(b[e]) * rho);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) zz[e] = __float_as_uint(__uint_as_float(zz[e]) * rho);
            tmem_st32(tmem + la + kT_S, a);
            tmem_st32(tmem + la + kT_S + 32, b);
            tmem_st16(tmem + la + kT_S + 64, zz);
            tmem_wait_st();
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(ms->img_full));
        mbar_arrive(bar(ms->s_ready));
      }
      const uint32_t slot = tmem + la + kT_A + (c & 1) * 64;
      if (!mbar_wait(bar(ms->uq_full[c & 1]), (c >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      if (KIND == 0) {
        // 4 groups of 16 angles; angle a -> packed (cos, sin) in column a, in place
#pragma unroll 1
        for (int gi = 0; gi < 4; ++gi) {
          uint32_t u[16];
          tmem_ld16(slot + 16 * gi, u);
          tmem_wait_ld();
#pragma unroll
          for (int a = 0; a < 16; ++a) {
            float sn, cs;
            sincos_mixed<kPolyMask>(a, __uint_as_float(u[a]), sn, cs);
            u[a] = pack_bf16x2(cs, sn);
          }
          tmem_st16(slot + 16 * gi, u);
        }
      } else {
#pragma unroll 1
        for (int pc = 0; pc < 2; ++pc) {
          uint32_t u[32], pk[16];
          tmem_ld32(slot + 32 * pc, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(fmaxf(__uint_as_float(u[2 * e]), 0.f), fmaxf(__uint_as_float(u[2 * e + 1]), 0.f));
          tmem_st16(slot + 16 * pc, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->phiq_full[c & 1]));
    }
  } else if (warp < 16) {
    // ------------------------------------------------------------ P16 and partial rows
    const int q4 = warp & 3, row = q4 * 32 + lane;
    const uint32_t la = uint32_t(q4 * 32) << 16;
    const int blk = row >> 4;             // 16-row block of the chunk
    const int owner = blk % G;
    const int slot_row = ((blk / G) * G + g) * 16 + (row & 15);
    int pend = -1;  // chunk whose deposit is stored but not yet signalled
    bool ok = true;
    for (int c = 0; ok && c < nch; ++c) {
      const int mb = c & (kMeta - 1);
      // P16 = masked P' in bf16 (in place; large-rise chunks also weight it), and sum_j P16_ij
      if (!(ok = mbar_wait(bar(ms->p_full), c & 1, abort_flag))) break;
      if (!(ok = mbar_wait(bar(ms->meta_full[mb]), (c / kMeta) & 1, abort_flag))) break;
      tc_fence_after();
      const bool fb = KIND == 0 && sm->fb[mb];
      const float ri = sm->rl[mb][row];
      const int rmax = q4 * 32 + 31;
      float di = 0.f;
      // one 32-key piece per iteration, in place: piece pc (columns 32 pc ..) becomes 16 packed
      // columns at 16 pc, which the earlier pieces have already read
#pragma unroll 1
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t pk[16];
        if (32 * pc > rmax) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        } else {
          uint32_t u[32];
          tmem_ld32(tmem + la + kT_PR + 32 * pc, u);
          tmem_wait_ld();
          if (KIND == 0 && fb) {  // large-rise chunk: exact weights exp(R_j - R_i)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              u[e] = __float_as_uint(__uint_as_float(u[e]) * ex2_approx(sm->rl[mb][32 * pc + e] - ri));
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j0 = 32 * pc + 2 * e;
            const float x0 = j0 <= row ? __uint_as_float(u[2 * e]) : 0.f;
            const float x1 = j0 + 1 <= row ? __uint_as_float(u[2 * e + 1]) : 0.f;
            pk[e] = pack_bf16x2(x0, x1);
            di += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xFFFF0000u);
          }
        }
        tmem_st16(tmem + la + kT_PR + 16 * pc, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->p16_full));
      // the partial row of chunk c: inter and intra combined at the row's reference; stored
      // directly (G = 1) or deposited with the owner of the row. TMEM is released before the
      // wait for the deposit slot, so the next chunk's P does not wait on the combiner.
      if (!(ok = mbar_wait(bar(ms->o_full), c & 1, abort_flag))) break;
      tc_fence_after();
      const float gfac = KIND == 0 ? ex2_approx(sm->crefl[mb] - ri) : 1.f;
      const float rho = KIND == 0 && !fb ? ex2_approx(sm->cnewl[mb] - ri) : 1.f;
      uint32_t dzh, dzl;
      tmem_ld1(tmem + la + kT_IN + 64, dzh);
      tmem_ld1(tmem + la + kT_IN + 65, dzl);
      tmem_wait_ld();
      const float den = fmaf(__uint_as_float(dzh) + __uint_as_float(dzl), gfac, di * rho);
      // G = 1 stores the normalised row; otherwise the partial numerators go out unscaled
      const float inv = G == 1 ? (den != 0.f ? 1.f / den : 0.f) : 1.f;
      const float fi = gfac * inv, fr = rho * inv;
      uint32_t pkd[32];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t in[32], it[32];
        tmem_ld32(tmem + la + kT_IN + 32 * hf, in);
        tmem_ld32(tmem + la + kT_PR + 64 + 32 * hf, it);
        tmem_wait_ld();
        if (hf == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(bar(ms->pr_free));
            mbar_arrive(bar(ms->meta_free[mb]));
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pkd[16 * hf + e] =
              pack_bf16x2(fmaf(__uint_as_float(in[2 * e]), fi, __uint_as_float(it[2 * e]) * fr),
                          fmaf(__uint_as_float(in[2 * e + 1]), fi, __uint_as_float(it[2 * e + 1]) * fr));
      }
      if (G == 1) {
        const int token = c * kTile + row;
        if (token < L) {
          uint4* o = reinterpret_cast<uint4*>(out + ((size_t)bh * L + token) * p.d);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (8 * q < p.d) o[q] = make_uint4(pkd[4 * q], pkd[4 * q + 1], pkd[4 * q + 2], pkd[4 * q + 3]);
        }
        continue;
      }
      // the previous chunk's deposit: its release no longer waits for stores in flight
      if (pend >= 0) {
        mbar_arrive_remote(mapa_shared(smem_u32(&ms->recv_full[pend & 1]), owner));
        pend = -1;
      }
      // deposit buffer c & 1: free once every owner has combined chunk c - 2
      const int pb = c & 1;
      if (c >= 2 && !(ok = mbar_wait(bar(ms->recv_free[pb]), ((c >> 1) - 1) & 1, abort_flag))) break;
      const uint32_t dst = mapa_shared(base + kC_RECV + pb * kRecvBufB + slot_row * kRecvRowB, owner);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        st_dsmem_f4(dst + 16 * e, make_float4(__uint_as_float(pkd[4 * e]), __uint_as_float(pkd[4 * e + 1]),
                                              __uint_as_float(pkd[4 * e + 2]), __uint_as_float(pkd[4 * e + 3])));
      st_dsmem_f4(dst + 128, make_float4(den, 0.f, 0.f, 0.f));
      pend = c;  // signalled at the next deposit (or after the last), once the stores have landed
    }
    if (G > 1 && pend >= 0) mbar_arrive_remote(mapa_shared(smem_u32(&ms->recv_full[pend & 1]), owner));
  } else if (G > 1) {
    // ------------------------------------------------------------ combiner (warps 16-19)
    // The owned rows of every chunk (16-row blocks b with b % G == g): the G partial rows,
    // summed in CTA order, divided and stored; every depositor may reuse its buffer once all
    // owners have read it. Thread t takes 16 of the 64 columns of owned row t / 4 (G = 2 owns 64
    // rows and takes them in two passes; G = 8 owns 16). The buffer is released as soon as every
    // owned row is in registers, before the output stores.
    const int t = tid - 16 * 32;
    const int qq = t & 3, nown = kTile / G;
    const bool cols = 16 * qq < p.d;
    uint32_t cph = 0;  // phase of comb_sync
    bool ok = true;
    for (int c = 0; ok && c < nch; ++c) {
      const int pb = c & 1;
      if (!(ok = mbar_wait_cluster(bar(ms->recv_full[pb]), (c >> 1) & 1, abort_flag))) break;
      float acc[2][16], den[2] = {0.f, 0.f};
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[ps][e] = 0.f;
        const int ro = 32 * ps + (t >> 2);
        if (ro < nown && cols) {
          const int bi = ro >> 4, rr = ro & 15;
          for (int s = 0; s < G; ++s) {
            const uint8_t* src = gb + kC_RECV + pb * kRecvBufB + ((bi * G + s) * 16 + rr) * kRecvRowB;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint4 x = *reinterpret_cast<const uint4*>(src + 32 * qq + 16 * e);
              const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                acc[ps][8 * e + 2 * u] += __uint_as_float(w4[u] << 16);
                acc[ps][8 * e + 2 * u + 1] += __uint_as_float(w4[u] & 0xFFFF0000u);
              }
            }
            den[ps] += *reinterpret_cast<const float*>(src + 128);
          }
        }
      }
      // every owned row is read: release the buffer in every depositor (one fence per releasing
      // thread, then relaxed arrives that do not wait for one another)
      if (!(ok = group_sync(bar(ms->comb_sync), cph, abort_flag))) break;
      if (t < G) {
        fence_acq_rel_cluster();
        mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&ms->recv_free[pb]), t));
      }
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
        const int ro = 32 * ps + (t >> 2);
        if (ro >= nown || !cols) continue;
        const int bi = ro >> 4, rr = ro & 15;
        const int token = c * kTile + (bi * G + g) * 16 + rr;
        if (token >= L) continue;
        const float inv = den[ps] != 0.f ? 1.f / den[ps] : 0.f;
        uint4* o = reinterpret_cast<uint4*>(out + ((size_t)bh * L + token) * p.d + 16 * qq);
#pragma unroll
        for (int e = 0; e < 2; ++e)
          o[e] = make_uint4(pack_bf16x2(acc[ps][8 * e] * inv, acc[ps][8 * e + 1] * inv),
                            pack_bf16x2(acc[ps][8 * e + 2] * inv, acc[ps][8 * e + 3] * inv),
                            pack_bf16x2(acc[ps][8 * e + 4] * inv, acc[ps][8 * e + 5] * inv),
                            pack_bf16x2(acc[ps][8 * e + 6] * inv, acc[ps][8 * e + 7] * inv));
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (G > 1) cluster_sync();  // no partner still writes into this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace cf
}  // namespace favor
