// kernel_causal.cuh - causal FAVOR forward on sm_100a tensor cores (chunked prefix scan).
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
// Parallel split. One thread-block cluster of G CTAs per (batch, head); CTA g owns a block of
// 128 features (trig: 64 angles as interleaved cos/sin pairs; ReLU: 128 angles), so every CTA
// walks the whole sequence with a 128 x 80 state slab in TMEM. num and den are sums over
// features, so the G partial rows add; CTA (q4 % G) owns rows 32 q4 .. 32 q4 + 31 of a chunk
// and receives the other CTAs' partials through distributed shared memory.
//
// Stabiliser (trig). Key features carry exp(|k_j|^2/2). The state S_{<c} is kept relative to
// the running reference cref_c = max |k_j|^2/2 over earlier chunks; row i of chunk c uses its
// own reference R_i = max(cref_c, max_{j <= i in c} |k_j|^2/2), so every weight is <= 1 and no
// row's terms vanish under another row's larger keys:
//   intra_ij = P_ij exp(|k_j|^2/2 - R_i), inter_i scaled by exp(cref_c - R_i).
// After chunk c the state is rescaled to cnew_c = max(cref_c, chunk max) before the chunk's keys
// (weighted exp(|k_j|^2/2 - cnew_c)) are added. Factors that cancel in the ratio (1/sqrt(M),
// exp(|q|^2/2)) are dropped. ReLU uses unit weights.
//
// Per chunk (MMAs issued by one thread; fp32 accumulation in TMEM):
//   U_K = K_c Omega_g^T      bf16, M=128 keys, N=64 angles per slice  -> phi(K) fp16 in smem
//   U_Q = Q_c Omega_g^T      bf16, M=128 queries, N=64/128           -> phi(Q) fp16 in TMEM
//   P = phi(Q) phi(K)^T      fp16, N=128 keys
//   inter = phi(Q) S_img     fp16 image of S_{<c} (power-of-two scale), N=64
//   S += phi(K)^T [w o V | w]  fp16, M=128 features, N=80
//   intra = P16 V_c          P16 = weighted, masked P in bf16 (TMEM), V_c the bf16 tile, N=64
// Denominators are accumulated in fp32 registers: phi(q_i).z (z = the state's normaliser
// column, kept in fp32) and sum_j P16_ij.
//
// Warp roles (384 threads): 0 TMA; 1 TMEM allocator and MMA issuer; 3 key norms, references
// and [w o V | w]; 4-7 key features and the state image (thread = key / feature row);
// 8-11 query features, P16, output and the cluster exchange (thread = query row).
#pragma once
#include "kernel_bidir.cuh"

namespace favor {
namespace tc {

// Shared memory (offsets from the 1024-aligned base).
constexpr int kC_OM = 0;              // Omega rows of this CTA's angles (one 128-row box)
constexpr int kC_K = 16 * 1024;       // K stages, 2 x 16 KB
constexpr int kC_V = 48 * 1024;       // V stages, 2 x 16 KB (V_c stays until its intra MMA)
constexpr int kC_Q = 80 * 1024;       // Q stage
constexpr int kC_PHK = 96 * 1024;     // phi(K) fp16: 2 atoms of 64 features x 128 keys
constexpr int kC_VW = 128 * 1024;     // [w o V] fp16, the V tile's layout
constexpr int kC_COL = 144 * 1024;    // column buffer: w (trig) or 1 (ReLU) as column 64
constexpr int kC_IMG = 160 * 1024;    // state image fp16: 128 feature rows x 64 values
constexpr int kC_RECV = 176 * 1024;   // partial rows received from the cluster (<= 26 KB)
constexpr int kC_SMALL = 202 * 1024;  // per-chunk scalars and vectors (CausalSmall)
constexpr int kC_MISC = 206 * 1024;   // barriers (CausalMisc)
constexpr int kRecvRowB = 68 * 4;     // one partial row: 64 numerators, the denominator, pad
// TMEM columns.
constexpr uint32_t kT_S = 0;          // state slab, 80 columns (lanes = features)
constexpr uint32_t kT_PR = 80;        // P (128 fp32) -> P16 [80, 144) + intra [144, 208)
constexpr uint32_t kT_IN = 208;       // inter accumulator, 64 columns
constexpr uint32_t kT_A = 272;        // U_Q (64 / 128 columns) -> phi(Q) packed fp16 (64)
constexpr uint32_t kT_B = 400;        // U_K slice, 64 columns

struct CausalParams {
  int BH, H, L, M;   // heads (B*H), heads per batch, tokens, random features
  int G;             // CTAs per head (feature blocks): 1, 2 or 4
  int nch;           // ceil(L / 128)
};

struct CausalSmall {
  float z[128];           // normaliser column of S_{<c}, fp32
  float n2l[2][128];      // |k_j|^2/2 * log2(e) of the chunk's keys, by chunk parity
  float rl[2][128];       // row references R_i * log2(e), by chunk parity
  float crefl[2], cnewl[2];  // references of S_{<c} and S_{<=c} (log2 units)
  float imgexp[2];        // image scale exponent of S_{<c}
  float red[2][4];        // per-warp max |S| for the image scale
};
static_assert(sizeof(CausalSmall) <= 4096, "causal small block");
static_assert(kC_RECV + 3 * 32 * kRecvRowB <= kC_SMALL, "receive buffer");

struct alignas(16) CausalMisc {
  int abort_flag;
  uint32_t tmem_base;
  int pad[2];
  uint64_t om_full, kv_full[2], kv_empty[2], q_full, q_empty;
  uint64_t meta_full[2], meta_free[2], vw_full;
  uint64_t uk_full, uk_free, uq_full, p_full, inter_done, s_done, o_full, drain;
  uint64_t img_full, img_free, s_ready, phik_full, phiq_full, p16_full, pr_free;
  uint64_t ksync;
  uint64_t recv_full[4], recv_free[4];
};
static_assert(sizeof(CausalMisc) <= 1024, "causal misc block");

__host__ __device__ constexpr uint32_t causal_smem_bytes() { return kC_MISC + 1024 + 1024; }

// KIND: 0 trig, 1 ReLU.
template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    favor_causal_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_om,
                    const CausalParams p, __nv_bfloat16* __restrict__ out) {
  constexpr int NA = KIND == 0 ? 64 : 128;  // angles per CTA
  constexpr int NSL = NA / 64;              // 64-angle slices of the key projection
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kNegBig = -1.0e30f;       // reference before any key; weight of padded keys

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
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ms->kv_full[s]), 1);
      mbar_init(bar(ms->kv_empty[s]), 2);  // key-norm warp + the intra MMA's commit
      mbar_init(bar(ms->meta_full[s]), 32);
      mbar_init(bar(ms->meta_free[s]), 4);
    }
    mbar_init(bar(ms->q_full), 1);
    mbar_init(bar(ms->q_empty), 1);
    mbar_init(bar(ms->vw_full), 32);
    mbar_init(bar(ms->uk_full), 1);
    mbar_init(bar(ms->uk_free), 4);
    mbar_init(bar(ms->uq_full), 1);
    mbar_init(bar(ms->p_full), 1);
    mbar_init(bar(ms->inter_done), 1);
    mbar_init(bar(ms->s_done), 1);
    mbar_init(bar(ms->o_full), 1);
    mbar_init(bar(ms->drain), 1);
    mbar_init(bar(ms->img_full), 4);
    mbar_init(bar(ms->img_free), 1 + 4);  // inter MMA commit + the 4 query warps (z read)
    mbar_init(bar(ms->s_ready), 4);
    mbar_init(bar(ms->phik_full), 4);
    mbar_init(bar(ms->phiq_full), 4);
    mbar_init(bar(ms->p16_full), 4);
    mbar_init(bar(ms->pr_free), 4);
    mbar_init(bar(ms->ksync), 128);
    for (int q = 0; q < 4; ++q) {
      mbar_init(bar(ms->recv_full[q]), G > 1 ? 32 * (G - 1) : 1);
      mbar_init(bar(ms->recv_free[q]), 32);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ms->tmem_base), 512);
    tmem_relinquish();
  }
  {  // column buffer: zero; ReLU: fp16 1.0 in column 64 of every key row
    uint4* col = reinterpret_cast<uint4*>(gb + kC_COL);
    for (int i = tid; i < kTileB / 16; i += kThreads) col[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    if (KIND == 1 && tid < kTile)
      reinterpret_cast<uint16_t*>(gb + kC_COL + tid * kRowB + ((tid & 7) << 4))[0] = 0x3C00u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (G > 1) cluster_sync();  // the partners' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(bar(ms->om_full), kTileB);
      tma_load_3d(base + kC_OM, &tm_om, bar(ms->om_full), 0, g * NA, h);
      int kv_issued = 0, q_issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        if (c >= 2 && !mbar_wait(bar(ms->kv_empty[s]), ((c >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(ms->kv_full[s]), 2 * kTileB);
        tma_load_3d(base + kC_K + s * kTileB, &tm_k, bar(ms->kv_full[s]), 0, c * kTile, bh);
        tma_load_3d(base + kC_V + s * kTileB, &tm_v, bar(ms->kv_full[s]), 0, c * kTile, bh);
        kv_issued = c + 1;
        if (c >= 1 && !mbar_wait(bar(ms->q_empty), (c - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(ms->q_full), kTileB);
        tma_load_3d(base + kC_Q, &tm_q, bar(ms->q_full), 0, c * kTile, bh);
        q_issued = c + 1;
      }
      // On an abort, let the copies already issued land before the CTA can exit.
      if (*abort_flag) {
        mbar_wait(bar(ms->om_full), 0, nullptr, kWaitLimitCycles / 8);
        for (int c = kv_issued > 2 ? kv_issued - 2 : 0; c < kv_issued; ++c)
          mbar_wait(bar(ms->kv_full[c & 1]), (c >> 1) & 1, nullptr, kWaitLimitCycles / 8);
        if (q_issued > 0) mbar_wait(bar(ms->q_full), (q_issued - 1) & 1, nullptr, kWaitLimitCycles / 8);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_uk = idesc_f16(128, 64, 1, 1, 0, 0);
      const uint32_t id_uq = idesc_f16(128, NA, 1, 1, 0, 0);
      const uint32_t id_p = idesc_f16(128, 128, 0, 0, 0, 0);
      const uint32_t id_in = idesc_f16(128, 64, 0, 0, 0, 1);
      const uint32_t id_s = idesc_f16(128, kNPad, 0, 0, 1, 1);
      const uint32_t id_it = idesc_f16(128, 64, 1, 1, 0, 1);
      const uint64_t d_om = sdesc_sw128(base + kC_OM, 16, 1024);
      const uint64_t d_q = sdesc_sw128(base + kC_Q, 16, 1024);
      const uint64_t d_k0 = sdesc_sw128(base + kC_K, 16, 1024);
      const uint64_t d_v0 = sdesc_sw128(base + kC_V, kTileB, 1024);
      const uint64_t d_phk_b = sdesc_sw128(base + kC_PHK, 16, 1024);      // K-major B of P
      const uint64_t d_phk_a = sdesc_sw128(base + kC_PHK, kTileB, 1024);  // MN-major A of S
      const uint64_t d_img = sdesc_sw128(base + kC_IMG, kTileB, 1024);
      const uint64_t d_vw = sdesc_sw128(base + kC_VW, kC_COL - kC_VW, 1024);
      constexpr uint64_t kKStep = (16 * kRowB) >> 4;  // 16 rows of an MN-major operand
      auto intra = [&](int cc) -> bool {
        if (!mbar_wait(bar(ms->p16_full), cc & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t bv = d_v0 + uint64_t(((cc & 1) * kTileB) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + kT_PR + 64, tmem + kT_PR + 8 * kk, bv + kk * kKStep, id_it, kk > 0 ? 1u : 0u);
        mma_commit(bar(ms->o_full));
        mma_commit(bar(ms->kv_empty[cc & 1]));
        return true;
      };
      bool ok = mbar_wait(bar(ms->om_full), 0, abort_flag);
      uint32_t ukc = 0;
      for (int c = 0; ok && c < nch; ++c) {
        const int s = c & 1;
        // U_K(c), one 64-angle slice at a time
        if (!(ok = mbar_wait(bar(ms->kv_full[s]), (c >> 1) & 1, abort_flag))) break;
        for (int sl = 0; sl < NSL; ++sl) {
          if (ukc > 0 && !(ok = mbar_wait(bar(ms->uk_free), (ukc - 1) & 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t a = d_k0 + uint64_t((s * kTileB) >> 4);
          const uint64_t b = d_om + uint64_t((sl * 64 * kRowB) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + kT_B, a + 2 * kk, b + 2 * kk, id_uk, kk > 0 ? 1u : 0u);
          mma_commit(bar(ms->uk_full));
          ++ukc;
        }
        if (!ok) break;
        // U_Q(c) into the phi(Q) region, once P(c-1) and inter(c-1) have read phi(Q_{c-1})
        if (!(ok = mbar_wait(bar(ms->q_full), c & 1, abort_flag))) break;
        if (c >= 1 && !(ok = mbar_wait(bar(ms->inter_done), (c - 1) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + kT_A, d_q + 2 * kk, d_om + 2 * kk, id_uq, kk > 0 ? 1u : 0u);
        mma_commit(bar(ms->uq_full));
        mma_commit(bar(ms->q_empty));
        // intra(c-1)
        if (c >= 1 && !(ok = intra(c - 1))) break;
        // P(c) = phi(Q) phi(K)^T
        if (!(ok = mbar_wait(bar(ms->phik_full), c & 1, abort_flag))) break;
        if (!(ok = mbar_wait(bar(ms->phiq_full), c & 1, abort_flag))) break;
        if (c >= 1 && !(ok = mbar_wait(bar(ms->pr_free), (c - 1) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + kT_PR, tmem + kT_A + 8 * kk, d_phk_b + uint64_t(((kk >> 2) * kTileB + (kk & 3) * 32) >> 4),
                 id_p, kk > 0 ? 1u : 0u);
        mma_commit(bar(ms->p_full));
        // inter(c) = phi(Q) S_img
        if (!(ok = mbar_wait(bar(ms->img_full), c & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + kT_IN, tmem + kT_A + 8 * kk, d_img + kk * kKStep, id_in, kk > 0 ? 1u : 0u);
        mma_commit(bar(ms->inter_done));
        mma_commit(bar(ms->img_free));
        // S += phi(K)^T [w o V | w]
        if (!(ok = mbar_wait(bar(ms->s_ready), c & 1, abort_flag))) break;
        if (!(ok = mbar_wait(bar(ms->vw_full), c & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + kT_S, d_phk_a + kk * kKStep, d_vw + kk * kKStep, id_s, (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(ms->s_done));
      }
      if (ok && nch > 0) intra(nch - 1);
      // every MMA issued has completed before TMEM can be released
      mma_commit(bar(ms->drain));
      mbar_wait(bar(ms->drain), 0, nullptr, kWaitLimitCycles / 8);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ key norms, references, [w o V | w]
    float crefl = kNegBig;
    for (int c = 0; c < nch; ++c) {
      const int s = c & 1, pz = c & 1;
      if (!mbar_wait(bar(ms->kv_full[s]), (c >> 1) & 1, abort_flag)) break;
      if (c >= 2 && !mbar_wait(bar(ms->meta_free[pz]), ((c >> 1) - 1) & 1, abort_flag)) break;
      const uint8_t* kt = gb + kC_K + s * kTileB;
      const int row0 = c * kTile;
      float nl[4];
      float cnewl = 0.f;
      if (KIND == 0) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = lane + 32 * jj;
          float acc = 0.f;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 x = *reinterpret_cast<const uint4*>(kt + j * kRowB + ((ch ^ (j & 7)) << 4));
            const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xFFFF0000u);
              acc = fmaf(lo, lo, acc);
              acc = fmaf(hi, hi, acc);
            }
          }
          nl[jj] = row0 + j < L ? 0.5f * acc * kLog2e : kNegBig;
        }
        // R_i: inclusive prefix max over the chunk's keys in order, seeded with cref
        float run = crefl;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float x = nl[jj];
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x = fmaxf(x, y);
          }
          x = fmaxf(x, run);
          sm->n2l[pz][lane + 32 * jj] = nl[jj];
          sm->rl[pz][lane + 32 * jj] = x;
          run = __shfl_sync(0xffffffffu, x, 31);
        }
        cnewl = run;
      } else {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) nl[jj] = 0.f;
      }
      if (lane == 0) {
        sm->crefl[pz] = crefl;
        sm->cnewl[pz] = cnewl;
      }
      mbar_arrive(bar(ms->meta_full[pz]));
      // [w o V] and w, once the previous state update has read the buffers
      if (c >= 1 && !mbar_wait(bar(ms->s_done), (c - 1) & 1, abort_flag)) break;
      const uint8_t* vt = gb + kC_V + s * kTileB;
      uint8_t* vw = gb + kC_VW;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = lane + 32 * jj;
        const float w = KIND == 0 ? ex2_approx(nl[jj] - cnewl) : 1.f;  // 0 for padded keys
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t off = j * kRowB + ((ch ^ (j & 7)) << 4);
          const uint4 x = *reinterpret_cast<const uint4*>(vt + off);
          const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
          uint32_t o4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o4[e] = pack_f16x2(__uint_as_float(w4[e] << 16) * w, __uint_as_float(w4[e] & 0xFFFF0000u) * w);
          *reinterpret_cast<uint4*>(vw + off) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        if (KIND == 0)
          *reinterpret_cast<__half*>(gb + kC_COL + j * kRowB + ((j & 7) << 4)) = __float2half_rn(w);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(ms->vw_full));
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->kv_empty[s]));
      crefl = cnewl;
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ state image and phi(K)
    const int q4 = warp & 3, row = q4 * 32 + lane;
    const uint32_t la = uint32_t(q4 * 32) << 16;
    uint32_t kph = 0, ukc = 0;
    for (int c = 0; c < nch; ++c) {
      const int pz = c & 1;
      // (1) image of S_{<c} at reference cref_c, then S rescaled to cnew_c
      if (c >= 1 && !mbar_wait(bar(ms->s_done), (c - 1) & 1, abort_flag)) break;
      if (!mbar_wait(bar(ms->meta_full[pz]), (c >> 1) & 1, abort_flag)) break;
      if (c >= 1 && !mbar_wait(bar(ms->img_free), (c - 1) & 1, abort_flag)) break;
      tc_fence_after();
      uint8_t* img = gb + kC_IMG + row * kRowB;
      if (c == 0) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(img + (ch << 4)) = make_uint4(0u, 0u, 0u, 0u);
        sm->z[row] = 0.f;
        if (row == 0) sm->imgexp[pz] = 0.f;
      } else {
        uint32_t a[32], b[32], zz[16];
        tmem_ld32(tmem + la + kT_S, a);
        tmem_ld32(tmem + la + kT_S + 32, b);
        tmem_ld16(tmem + la + kT_S + 64, zz);
        tmem_wait_ld();
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(a[e])), fabsf(__uint_as_float(b[e]))));
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) sm->red[pz][q4] = mx;
        if (!group_sync(bar(ms->ksync), kph, abort_flag)) break;
        mx = fmaxf(fmaxf(sm->red[pz][0], sm->red[pz][1]), fmaxf(sm->red[pz][2], sm->red[pz][3]));
        // power-of-two scale putting the largest |S| in [2^13, 2^14)
        int e2 = 0;
        if (mx > 1e-30f) {
          const int ex = int((__float_as_uint(mx) >> 23) & 0xFF) - 127;
          e2 = min(max(13 - ex, -120), 120);
        }
        const float sc = pow2i(e2);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t* src = ch < 4 ? a + 8 * ch : b + 8 * (ch - 4);
          uint4 o;
          o.x = pack_f16x2(__uint_as_float(src[0]) * sc, __uint_as_float(src[1]) * sc);
          o.y = pack_f16x2(__uint_as_float(src[2]) * sc, __uint_as_float(src[3]) * sc);
          o.z = pack_f16x2(__uint_as_float(src[4]) * sc, __uint_as_float(src[5]) * sc);
          o.w = pack_f16x2(__uint_as_float(src[6]) * sc, __uint_as_float(src[7]) * sc);
          *reinterpret_cast<uint4*>(img + ((ch ^ (row & 7)) << 4)) = o;
        }
        sm->z[row] = __uint_as_float(zz[0]);
        if (row == 0) sm->imgexp[pz] = float(e2);
        const float rho = ex2_approx(sm->crefl[pz] - sm->cnewl[pz]);
        if (KIND == 0 && rho != 1.f) {
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
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(ms->img_full));
        mbar_arrive(bar(ms->s_ready));
      }
      // (2) phi(K_c) into shared memory (the buffer is free: S(c-1) has completed)
      bool ok = true;
      for (int sl = 0; sl < NSL; ++sl) {
        if (!(ok = mbar_wait(bar(ms->uk_full), ukc & 1, abort_flag))) break;
        ++ukc;
        tc_fence_after();
        uint32_t u0[32], u1[32];
        tmem_ld32(tmem + la + kT_B, u0);
        tmem_ld32(tmem + la + kT_B + 32, u1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ms->uk_free));
        if (KIND == 0) {
          // angle a -> features (2a, 2a+1) = (cos, sin); atom a / 32, 4 angles per 16 bytes
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int a = 4 * q + e;
              const float x = __uint_as_float(a < 32 ? u0[a] : u1[a - 32]);
              float sn, cs;
              __sincosf(x, &sn, &cs);
              const bool live = g * NA + a < p.M;
              pk[e] = live ? pack_f16x2(cs, sn) : 0u;
            }
            const int atom = q >> 3, ch = q & 7;
            *reinterpret_cast<uint4*>(gb + kC_PHK + atom * kTileB + row * kRowB + ((ch ^ (row & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int a = 8 * q + 2 * e;
              const float x0 = __uint_as_float(a < 32 ? u0[a] : u1[a - 32]);
              const float x1 = __uint_as_float(a + 1 < 32 ? u0[a + 1] : u1[a + 1 - 32]);
              pk[e] = pack_f16x2(fmaxf(x0, 0.f), fmaxf(x1, 0.f));
            }
            *reinterpret_cast<uint4*>(gb + kC_PHK + sl * kTileB + row * kRowB + ((q ^ (row & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ms->phik_full));
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ phi(Q), P16, output
    const int q4 = warp & 3, row = q4 * 32 + lane;
    const uint32_t la = uint32_t(q4 * 32) << 16;
    const int owner = q4 % G;
    float dz_cur = 0.f, dz_prev = 0.f, di_cur = 0.f, di_prev = 0.f;
    // phi(Q_c): features into TMEM (in place over U_Q), and phi(q_i).z
    auto phi_q = [&](int c) -> bool {
      if (!mbar_wait(bar(ms->uq_full), c & 1, abort_flag)) return false;
      if (!mbar_wait(bar(ms->img_full), c & 1, abort_flag)) return false;
      tc_fence_after();
      float dz = 0.f;
      if (KIND == 0) {
        uint32_t u0[32], u1[32];
        tmem_ld32(tmem + la + kT_A, u0);
        tmem_ld32(tmem + la + kT_A + 32, u1);
        tmem_wait_ld();
#pragma unroll
        for (int a = 0; a < 32; ++a) {
          float sn, cs;
          __sincosf(__uint_as_float(u0[a]), &sn, &cs);
          const float2 zf = *reinterpret_cast<const float2*>(&sm->z[2 * a]);
          dz = fmaf(cs, zf.x, fmaf(sn, zf.y, dz));
          u0[a] = pack_f16x2(cs, sn);
        }
#pragma unroll
        for (int a = 0; a < 32; ++a) {
          float sn, cs;
          __sincosf(__uint_as_float(u1[a]), &sn, &cs);
          const float2 zf = *reinterpret_cast<const float2*>(&sm->z[64 + 2 * a]);
          dz = fmaf(cs, zf.x, fmaf(sn, zf.y, dz));
          u1[a] = pack_f16x2(cs, sn);
        }
        tmem_st32(tmem + la + kT_A, u0);
        tmem_st32(tmem + la + kT_A + 32, u1);
      } else {
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          uint32_t u[32], pk[16];
          tmem_ld32(tmem + la + kT_A + 32 * pc, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = fmaxf(__uint_as_float(u[2 * e]), 0.f), x1 = fmaxf(__uint_as_float(u[2 * e + 1]), 0.f);
            const float2 zf = *reinterpret_cast<const float2*>(&sm->z[32 * pc + 2 * e]);
            dz = fmaf(x0, zf.x, fmaf(x1, zf.y, dz));
            pk[e] = pack_f16x2(x0, x1);
          }
          tmem_st16(tmem + la + kT_A + 16 * pc, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(ms->phiq_full));
        mbar_arrive(bar(ms->img_free));
      }
      dz_cur = dz;
      return true;
    };
    // P16 = weighted, masked P in bf16 (in place), and sum_j P16_ij
    auto p16 = [&](int c) -> bool {
      const int pz = c & 1;
      if (!mbar_wait(bar(ms->p_full), c & 1, abort_flag)) return false;
      if (!mbar_wait(bar(ms->meta_full[pz]), (c >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const float ri = sm->rl[pz][row];
      const int rmax = q4 * 32 + 31;
      float di = 0.f;
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
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j0 = 32 * pc + 2 * e;
            float x0 = __uint_as_float(u[2 * e]), x1 = __uint_as_float(u[2 * e + 1]);
            if (KIND == 0) {
              const float2 nn = *reinterpret_cast<const float2*>(&sm->n2l[pz][j0]);
              x0 *= ex2_approx(nn.x - ri);
              x1 *= ex2_approx(nn.y - ri);
            }
            x0 = j0 <= row ? x0 : 0.f;
            x1 = j0 + 1 <= row ? x1 : 0.f;
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
      di_cur = di;
      return true;
    };
    // output of chunk c: combine inter and intra, exchange partials, divide, store
    auto output = [&](int c, float dz, float di) -> bool {
      const int pz = c & 1;
      if (!mbar_wait(bar(ms->o_full), c & 1, abort_flag)) return false;
      tc_fence_after();
      uint32_t in0[32], in1[32], it0[32], it1[32];
      tmem_ld32(tmem + la + kT_IN, in0);
      tmem_ld32(tmem + la + kT_IN + 32, in1);
      tmem_ld32(tmem + la + kT_PR + 64, it0);
      tmem_ld32(tmem + la + kT_PR + 96, it1);
      tmem_wait_ld();
      const float gfac = KIND == 0 ? ex2_approx(sm->crefl[pz] - sm->rl[pz][row]) : 1.f;
      const float ffac = gfac * pow2i(-int(sm->imgexp[pz]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(ms->pr_free));
        mbar_arrive(bar(ms->meta_free[pz]));
      }
      float num[64];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        num[e] = fmaf(__uint_as_float(in0[e]), ffac, __uint_as_float(it0[e]));
        num[32 + e] = fmaf(__uint_as_float(in1[e]), ffac, __uint_as_float(it1[e]));
      }
      float den = fmaf(dz, gfac, di);
      if (G > 1) {
        if (owner != g) {
          // send this CTA's partial row to the owner of the rows
          if (c >= 1 && !mbar_wait(bar(ms->recv_free[q4]), (c - 1) & 1, abort_flag)) return false;
          const int qo = q4 / G, sidx = (g - owner + G) % G - 1;
          const uint32_t dst =
              mapa_shared(base + kC_RECV + ((qo * (G - 1) + sidx) * 32 + lane) * kRecvRowB, owner);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            st_dsmem_f4(dst + 16 * e, make_float4(num[4 * e], num[4 * e + 1], num[4 * e + 2], num[4 * e + 3]));
          st_dsmem_f4(dst + 256, make_float4(den, 0.f, 0.f, 0.f));
          mbar_arrive_remote(mapa_shared(smem_u32(&ms->recv_full[q4]), owner));
          return true;
        }
        if (!mbar_wait_cluster(bar(ms->recv_full[q4]), c & 1, abort_flag)) return false;
        const int qo = q4 / G;
        for (int sidx = 0; sidx < G - 1; ++sidx) {
          const float* src =
              reinterpret_cast<const float*>(gb + kC_RECV + ((qo * (G - 1) + sidx) * 32 + lane) * kRecvRowB);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float4 x = *reinterpret_cast<const float4*>(src + 4 * e);
            num[4 * e] += x.x;
            num[4 * e + 1] += x.y;
            num[4 * e + 2] += x.z;
            num[4 * e + 3] += x.w;
          }
          den += src[64];
        }
        // the received rows are consumed: let each sender reuse its slot
        for (int sidx = 0; sidx < G - 1; ++sidx) {
          const int sender = (owner + 1 + sidx) % G;
          mbar_arrive_remote(mapa_shared(smem_u32(&ms->recv_free[q4]), sender));
        }
      }
      const int token = c * kTile + row;
      if (token < L) {
        const float inv = den != 0.f ? 1.f / den : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)bh * L + token) * kD);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4 o;
          o.x = pack_bf16x2(num[8 * q] * inv, num[8 * q + 1] * inv);
          o.y = pack_bf16x2(num[8 * q + 2] * inv, num[8 * q + 3] * inv);
          o.z = pack_bf16x2(num[8 * q + 4] * inv, num[8 * q + 5] * inv);
          o.w = pack_bf16x2(num[8 * q + 6] * inv, num[8 * q + 7] * inv);
          dst[q] = o;
        }
      }
      return true;
    };
    bool ok = true;
    for (int c = 0; ok && c < nch; ++c) {
      if (!(ok = phi_q(c))) break;
      if (c >= 1 && !(ok = output(c - 1, dz_prev, di_prev))) break;
      if (!(ok = p16(c))) break;
      dz_prev = dz_cur;
      di_prev = di_cur;
    }
    if (ok && nch > 0) output(nch - 1, dz_prev, di_prev);
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

}  // namespace tc
}  // namespace favor
