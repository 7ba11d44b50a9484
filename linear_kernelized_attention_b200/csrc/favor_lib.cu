// favor_lib.cu - host side of libfavor.so: argument validation, TMA descriptors, scratch,
// launches and the C ABI declared in include/favor.h. All device code is included here, so
// the library is one translation unit with one device status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/favor.h"
#include "ptx.cuh"
#include "kernels_f32.cuh"
#include "kernel_bidir_split.cuh"
#include "kernel_causal_fs.cuh"
#include "kernel_decode.cuh"
#include "kernels_bwd_f32.cuh"

namespace favor {

// A kernel whose only job is a bounded wait on an mbarrier nobody arrives on. It checks that
// the timeout path records FAVOR_ERR_TIMEOUT and returns, leaving the context usable.
__global__ void k_selftest_timeout(long long limit_cycles) {
  __shared__ uint64_t b;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&b), 1);
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(smem_u32(&b), 0, nullptr, limit_cycles);
  __syncthreads();
}

// The FMA-pipe sine and cosine (sincos_poly.cuh) of n angles, one per thread, so that tests can
// hold the device evaluation against the mathematics and the kernels' SFU alternative.
__global__ void k_selftest_sincos(const float* __restrict__ u, float* __restrict__ s, float* __restrict__ c,
                                  int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float sv, cv;
  sincos_fma(u[i], sv, cv);
  s[i] = sv;
  c[i] = cv;
}
}  // namespace favor

namespace {

using namespace favor;

#define FAVOR_TRY(expr)                          \
  do {                                           \
    if ((expr) != cudaSuccess) return FAVOR_ERR_CUDA; \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FAVOR_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return FAVOR_ERR_CUDA;
  return major == 10 ? FAVOR_OK : FAVOR_ERR_DEVICE;
}

int sm_count() {
  static int cache[64] = {};
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device): the attribute
// persists, and setting it on every call costs host time on the launch path.
int ensure_smem_attr(const void* kern, int bytes) {
  struct Entry {
    const void* k;
    int dev, bytes;
  };
  static Entry done[64];
  static int n = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FAVOR_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  for (int i = 0; i < n; ++i)
    if (done[i].k == kern && done[i].dev == dev && done[i].bytes >= bytes) return FAVOR_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return FAVOR_ERR_CUDA;
  if (n < 64) done[n++] = Entry{kern, dev, bytes};
  return FAVOR_OK;
}

// Common shape/pointer checks shared by every entry point.
int check_common(const void* q, const void* k, const void* v, const void* omega, const void* out,
                 int B, int H, int L, int d, int M, int kind) {
  if (!q || !k || !v || !omega || !out) return FAVOR_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(omega) || !aligned16(out))
    return FAVOR_ERR_ALIGN;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || M <= 0) return FAVOR_ERR_SHAPE;
  if ((long long)B * H > INT_MAX / 2 || (long long)B * H * L > (1ll << 40) ||
      (long long)B * H * L * d > (1ll << 40))
    return FAVOR_ERR_SHAPE;
  if (kind != FAVOR_TRIG && kind != FAVOR_RELU) return FAVOR_ERR_KIND;
  return FAVOR_OK;
}

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 tensor [n2][n1][d] (d = 16, 32, 64 or 128 elements per row) read in boxes of
// {64, 128, 1} with 128-byte swizzle. Columns past d and rows past n1 read as zero and are not
// written; a row of d = 128 takes two boxes (columns 0 and 64).
bool make_map_rows(CUtensorMap* m, const void* ptr, int d, uint64_t n1, uint64_t n2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, n1, n2};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * n1};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ scratch
// Scratch comes from a library-owned stream-ordered pool (per device) that keeps its memory
// between calls, so repeated calls do not return memory to the driver.
cudaMemPool_t pool_for_device() {
  static cudaMemPool_t pools[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> g(mu);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    if (cudaMemPoolCreate(&pools[dev], &props) != cudaSuccess) return nullptr;
    uint64_t thr = UINT64_MAX;
    cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &thr);
  }
  return pools[dev];
}

int scratch_alloc(void** p, size_t bytes, cudaStream_t st) {
  *p = nullptr;
  if (bytes == 0) return FAVOR_OK;
  cudaMemPool_t pool = pool_for_device();
  if (!pool) return FAVOR_ERR_CUDA;
  return cudaMallocFromPoolAsync(p, bytes, pool, st) == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

// Two non-blocking streams per device for the host-buffer entry's copies in and out, created on
// first use and kept for the life of the process.
constexpr int kHostSlices = 4;  // batch slices of the host-buffer entry's copy/compute pipeline
int copy_streams(cudaStream_t* s_in, cudaStream_t* s_out) {
  static cudaStream_t streams[64][2] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FAVOR_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FAVOR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(mu);
  for (int i = 0; i < 2; ++i)
    if (!streams[dev][i] && cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking) != cudaSuccess)
      return FAVOR_ERR_CUDA;
  *s_in = streams[dev][0];
  *s_out = streams[dev][1];
  return FAVOR_OK;
}

int check_tc_shape(int d, int M, int kind, int causal) {
  if (d != 16 && d != 32 && d != 64 && d != 128) return FAVOR_ERR_UNSUPPORTED;
  if (kind == FAVOR_TRIG && M > 256) return FAVOR_ERR_UNSUPPORTED;
  if (kind == FAVOR_RELU && M > 512) return FAVOR_ERR_UNSUPPORTED;
  if (causal && d > 64) return FAVOR_ERR_UNSUPPORTED;
  return FAVOR_OK;
}

// ------------------------------------------------------------------ bf16 bidirectional, split
// Shapes of the three-launch bidirectional path: key states over (pair, tile) units, the merge,
// and queries over (head, tile) units. Every CTA takes a contiguous run of units; the grids are
// the SM count (one CTA per SM) or the unit count if smaller.
struct SplitPlan {
  int dp, nab, ntiles, smax, Pk, Pq;
  long long units_k, units_q, npairs;
  size_t part_bytes, meta_bytes, img_bytes_head, ws_bytes;
  int q_off_img, q_off_q, q_off_out, q_off_misc, q_smem, k_smem;
};

template <int KIND, int DP>
void plan_split_t(SplitPlan& pl, int BH, int L, int M) {
  using SC = bs::StateCfg<KIND, DP>;
  using QC = bs::QueryCfg<KIND, DP>;
  pl.dp = DP;
  pl.nab = (M + 127) / 128;
  pl.ntiles = (L + bs::kTile - 1) / bs::kTile;
  pl.npairs = (long long)BH * pl.nab;
  pl.units_k = pl.npairs * pl.ntiles;
  pl.units_q = (long long)BH * pl.ntiles;
  const int sms = sm_count();
  // a pair's tiles spread over at most Pk / npairs + 2 runs; the merge weights at most
  // bs::kMergeMaxSlots of them
  pl.Pk = (int)std::min<long long>(std::min<long long>(sms, pl.units_k), (bs::kMergeMaxSlots - 2) * pl.npairs);
  pl.Pq = (int)std::min<long long>(sms, pl.units_q);
  const long long per = pl.units_k / pl.Pk;  // >= 1
  pl.smax = (int)std::min<long long>(pl.Pk, (pl.ntiles + per - 1) / per + 1);
  pl.part_bytes = (size_t)pl.npairs * pl.smax * (DP + 1) * SC::R * sizeof(float);
  pl.meta_bytes = ((size_t)pl.npairs * pl.smax * 2 * sizeof(float) + 255) / 256 * 256;
  pl.img_bytes_head = (size_t)pl.nab * (QC::FB / 64) * QC::NV * bs::kRowB;
  pl.ws_bytes = pl.part_bytes + pl.meta_bytes + (size_t)BH * pl.img_bytes_head;
  const int om_bytes = pl.nab * QC::NCB * bs::kBoxB;
  pl.q_off_img = om_bytes;
  pl.q_off_q = (int)((pl.q_off_img + pl.img_bytes_head + 1023) / 1024 * 1024);
  pl.q_off_out = pl.q_off_q + 2 * QC::NCB * bs::kBoxB;
  pl.q_off_misc = pl.q_off_out + QC::NOS * QC::NCB * bs::kBoxB;
  pl.q_smem = pl.q_off_misc + 1024 + 1024;
  pl.k_smem = SC::kSmem;
}

bool plan_split(SplitPlan& pl, int BH, int L, int d, int M, int kind) {
  const int dp = d <= 64 ? 64 : 128;
  if (kind == FAVOR_TRIG) {
    if (dp == 64) plan_split_t<0, 64>(pl, BH, L, M); else plan_split_t<0, 128>(pl, BH, L, M);
  } else {
    if (dp == 64) plan_split_t<1, 64>(pl, BH, L, M); else plan_split_t<1, 128>(pl, BH, L, M);
  }
  return pl.q_smem <= 232448 && pl.smax <= bs::kMergeMaxSlots;
}

template <int KIND, int DP>
int launch_split_t(const SplitPlan& pl, const void* q, const void* k, const void* v, const void* omega, void* out,
                   int BH, int H, int L, int d, int M, void* ws, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mo, mom;
  if (!make_map_rows(&mq, q, d, L, BH) || !make_map_rows(&mk, k, d, L, BH) || !make_map_rows(&mv, v, d, L, BH) ||
      !make_map_rows(&mo, out, d, L, BH) || !make_map_rows(&mom, omega, d, M, H))
    return FAVOR_ERR_CUDA;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  float* part = reinterpret_cast<float*>(w8);
  float* meta = reinterpret_cast<float*>(w8 + pl.part_bytes);
  uint8_t* img = w8 + pl.part_bytes + pl.meta_bytes;

  bs::StateParams sp{};
  sp.H = H;
  sp.L = L;
  sp.M = M;
  sp.nab = pl.nab;
  sp.ntiles = pl.ntiles;
  sp.units = pl.units_k;
  sp.smax = pl.smax;
  sp.part = part;
  sp.meta = meta;
  auto ks = bs::k_bidir_state<KIND, DP>;
  if (ensure_smem_attr(reinterpret_cast<const void*>(ks), pl.k_smem) != FAVOR_OK) return FAVOR_ERR_CUDA;
  ks<<<pl.Pk, bs::StateCfg<KIND, DP>::kThreads, pl.k_smem, st>>>(mk, mv, mom, sp);

  bs::MergeParams mp{};
  mp.nab = pl.nab;
  mp.ntiles = pl.ntiles;
  mp.smax = pl.smax;
  mp.M = M;
  mp.units = pl.units_k;
  mp.P = pl.Pk;
  mp.part = part;
  mp.meta = meta;
  mp.img = img;
  mp.img_bytes = (long long)pl.img_bytes_head;
  // the merge and the query kernel are launched with programmatic stream serialization: each may
  // start while the kernel before it drains, and waits (griddepcontrol.wait) before reading its
  // results
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.npairs, bs::StateCfg<KIND, DP>::R / 32, 1);
    cfg.blockDim = dim3(bs::merge_threads<KIND, DP>(), 1, 1);
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, bs::k_bidir_merge<KIND, DP>, mp) != cudaSuccess) return FAVOR_ERR_CUDA;
  }

  bs::QueryParams qp{};
  qp.H = H;
  qp.L = L;
  qp.M = M;
  qp.nab = pl.nab;
  qp.ntiles = pl.ntiles;
  qp.units = pl.units_q;
  qp.img = img;
  qp.img_bytes = (int)pl.img_bytes_head;
  qp.om_bytes = pl.nab * bs::QueryCfg<KIND, DP>::NCB * bs::kBoxB;
  qp.off_img = pl.q_off_img;
  qp.off_q = pl.q_off_q;
  qp.off_out = pl.q_off_out;
  qp.off_misc = pl.q_off_misc;
  auto kq = bs::k_bidir_query<KIND, DP>;
  if (ensure_smem_attr(reinterpret_cast<const void*>(kq), pl.q_smem) != FAVOR_OK) return FAVOR_ERR_CUDA;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.Pq, 1, 1);
    cfg.blockDim = dim3(bs::kThreads, 1, 1);
    cfg.dynamicSmemBytes = pl.q_smem;
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kq, mq, mom, mo, qp) != cudaSuccess) return FAVOR_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

int launch_bidir_split(const void* q, const void* k, const void* v, const void* omega, void* out, int B, int H,
                       int L, int d, int M, int kind, cudaStream_t st) {
  const int BH = B * H;
  SplitPlan pl{};
  if (!plan_split(pl, BH, L, d, M, kind)) return FAVOR_ERR_UNSUPPORTED;
  if (pl.npairs > INT_MAX) return FAVOR_ERR_UNSUPPORTED;
  void* ws = nullptr;
  int rc = scratch_alloc(&ws, pl.ws_bytes, st);
  if (rc != FAVOR_OK) return rc;
  if (kind == FAVOR_TRIG)
    rc = pl.dp == 64 ? launch_split_t<0, 64>(pl, q, k, v, omega, out, BH, H, L, d, M, ws, st)
                     : launch_split_t<0, 128>(pl, q, k, v, omega, out, BH, H, L, d, M, ws, st);
  else
    rc = pl.dp == 64 ? launch_split_t<1, 64>(pl, q, k, v, omega, out, BH, H, L, d, M, ws, st)
                     : launch_split_t<1, 128>(pl, q, k, v, omega, out, BH, H, L, d, M, ws, st);
  cudaFreeAsync(ws, st);
  return rc;
}

// ------------------------------------------------------------------ bf16 causal, feature split
// One cluster of G CTAs per head, each owning 64 angles: G = ceil(M / 64) (<= 4 trig, <= 8 ReLU).
int launch_causal_fs(const void* q, const void* k, const void* v, const void* omega, void* out, int B, int H,
                     int L, int d, int M, int kind, cudaStream_t st) {
  const int BH = B * H;
  const int G0 = (M + 63) / 64;
  const int G = G0 <= 1 ? 1 : G0 <= 2 ? 2 : G0 <= 4 ? 4 : 8;
  if (G0 > 8 || (kind == FAVOR_TRIG && G0 > 4)) return FAVOR_ERR_UNSUPPORTED;
  if ((long long)BH * G > INT_MAX) return FAVOR_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv, mom;
  if (!make_map_rows(&mq, q, d, L, BH) || !make_map_rows(&mk, k, d, L, BH) || !make_map_rows(&mv, v, d, L, BH) ||
      !make_map_rows(&mom, omega, d, M, H))
    return FAVOR_ERR_CUDA;
  cf::CausalParams prm{};
  prm.BH = BH;
  prm.H = H;
  prm.L = L;
  prm.M = M;
  prm.G = G;
  prm.nch = (L + cf::kTile - 1) / cf::kTile;
  prm.d = d;
  const uint32_t smem = cf::causal_smem_bytes();
  auto kern = kind == FAVOR_TRIG ? cf::k_causal_fs<0> : cf::k_causal_fs<1>;
  if (ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)smem) != FAVOR_OK) return FAVOR_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(BH * G, 1, 1);
  cfg.blockDim = dim3(cf::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mom, prm, static_cast<__nv_bfloat16*>(out)) == cudaSuccess
             ? FAVOR_OK
             : FAVOR_ERR_CUDA;
}

// ------------------------------------------------------------------ fp32 path
}  // namespace

namespace favor {
namespace cvt {
// bf16 -> fp32 (exact) and fp32 -> bf16 (round to nearest even) over a flat array; x and y are
// 16-byte aligned, eight elements per step, then the tail one by one.
__global__ void __launch_bounds__(256) k_widen(const __nv_bfloat16* __restrict__ x, float* __restrict__ y,
                                               long long n) {
  const long long n8 = n / 8, stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long i = t0; i < n8; i += stride) {
    const uint4 w = reinterpret_cast<const uint4*>(x)[i];
    const float4 a = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                                 __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u));
    const float4 b = make_float4(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u),
                                 __uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u));
    reinterpret_cast<float4*>(y)[2 * i] = a;
    reinterpret_cast<float4*>(y)[2 * i + 1] = b;
  }
  for (long long i = 8 * n8 + t0; i < n; i += stride) y[i] = __bfloat162float(x[i]);
}

__global__ void __launch_bounds__(256) k_narrow(const float* __restrict__ y, __nv_bfloat16* __restrict__ x,
                                                long long n) {
  const long long n8 = n / 8, stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long i = t0; i < n8; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(y)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(y)[2 * i + 1];
    reinterpret_cast<uint4*>(x)[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                                                pack_bf16x2(b.z, b.w));
  }
  for (long long i = 8 * n8 + t0; i < n; i += stride) x[i] = __float2bfloat16_rn(y[i]);
}
}  // namespace cvt
}  // namespace favor

namespace {
using namespace favor;

size_t f32_workspace(int BH, int L, int d, int M, int kind) {
  const int F = kind == FAVOR_TRIG ? 2 * M : M;
  const int nch = (L + f32::kChunk - 1) / f32::kChunk;
  return (size_t)BH * nch * F * (d + 1) * sizeof(float) + (size_t)BH * sizeof(float);
}

int launch_f32(const float* q, const float* k, const float* v, const float* omega, float* out,
               int B, int H, int L, int d, int M, int kind, int causal, cudaStream_t st) {
  const int BH = B * H;
  const int F = kind == FAVOR_TRIG ? 2 * M : M;
  const int nch = (L + f32::kChunk - 1) / f32::kChunk;
  const int nft = (F + f32::kFeatTile - 1) / f32::kFeatTile;
  if (BH > 65535 || nch > 65535) return FAVOR_ERR_UNSUPPORTED;
  void* ws = nullptr;
  int rc = scratch_alloc(&ws, f32_workspace(BH, L, d, M, kind), st);
  if (rc != FAVOR_OK) return rc;
  float* dS = static_cast<float*>(ws);
  float* cmax = dS + (size_t)BH * nch * F * (d + 1);
  const size_t sm_state = (size_t)(2 * f32::kChunk * d + f32::kChunk + f32::kChunk * f32::kFeatTile) * 4;
  const size_t sm_out = (size_t)(3 * f32::kChunk * d + f32::kChunk + 2 * f32::kChunk * f32::kFeatTile +
                                 f32::kFeatTile * (d + 1) + f32::kChunk * f32::kChunk) * 4;
  if (cudaFuncSetAttribute(f32::k_chunk_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_state) != cudaSuccess ||
      cudaFuncSetAttribute(f32::k_output, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_out) != cudaSuccess)
    rc = FAVOR_ERR_CUDA;
  if (rc == FAVOR_OK) {
    if (kind == FAVOR_TRIG) f32::k_key_halfnorm_max<<<BH, f32::kThreads, 0, st>>>(k, cmax, L, d);
    f32::k_chunk_state<<<dim3(nft, nch, BH), f32::kThreads, sm_state, st>>>(k, v, omega, cmax, dS, H, L,
                                                                             d, M, F, kind);
    const long long per_chunk = (long long)F * (d + 1);
    const long long total = (long long)BH * per_chunk;
    f32::k_scan_chunks<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(dS, nch, per_chunk, total, causal);
    f32::k_output<<<dim3(nch, BH), f32::kThreads, sm_out, st>>>(q, k, v, omega, cmax, dS, out, H, L, d, M,
                                                                F, kind, causal);
    if (cudaGetLastError() != cudaSuccess) rc = FAVOR_ERR_CUDA;
  }
  cudaFreeAsync(ws, st);
  return rc;
}

// ------------------------------------------------------------------ bf16 shapes the tensor-core kernels leave out
// Causal d > 64, bidirectional trig d = 128 with M > 128, d outside {16, 32, 64, 128} and trig
// 256 < M <= 512 run the fp32 CUDA-core kernels on fp32 copies of the bf16 inputs (the widening is
// exact) and round the result to bf16 once. Scratch: the four fp32 copies and the fp32 output, then
// the fp32 path's own scratch, both from the stream-ordered pool.
size_t round_up256(size_t b) { return (b + 255) / 256 * 256; }

bool cuda_core_route_ok(long long BH, int L, int d, int M) {
  return d <= f32::kMaxD && M <= 512 && BH <= 65535 && (L + f32::kChunk - 1) / f32::kChunk <= 65535;
}

size_t cuda_core_route_bytes(long long BH, int H, int L, int d, int M) {
  const size_t n = (size_t)BH * L * d;
  return 4 * round_up256(n * sizeof(float)) + round_up256((size_t)H * M * d * sizeof(float));
}

int launch_bf16_cuda_cores(const void* q, const void* k, const void* v, const void* omega, void* out, int B, int H,
                           int L, int d, int M, int kind, int causal, cudaStream_t st) {
  const long long BH = (long long)B * H;
  if (!cuda_core_route_ok(BH, L, d, M)) return FAVOR_ERR_UNSUPPORTED;
  const long long n = BH * L * d, nom = (long long)H * M * d;
  void* ws = nullptr;
  int rc = scratch_alloc(&ws, cuda_core_route_bytes(BH, H, L, d, M), st);
  if (rc != FAVOR_OK) return rc;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const size_t nb = round_up256((size_t)n * sizeof(float));
  float* qf = reinterpret_cast<float*>(w8);
  float* kf = reinterpret_cast<float*>(w8 + nb);
  float* vf = reinterpret_cast<float*>(w8 + 2 * nb);
  float* of = reinterpret_cast<float*>(w8 + 3 * nb);
  float* omf = reinterpret_cast<float*>(w8 + 4 * nb);
  const long long max_blocks = 16ll * sm_count();  // grid-stride loops: up to 16 blocks per SM
  auto grid = [max_blocks](long long m) {
    return (unsigned)std::max<long long>(1, std::min<long long>((m / 8 + 255) / 256, max_blocks));
  };
  cvt::k_widen<<<grid(n), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), qf, n);
  cvt::k_widen<<<grid(n), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(k), kf, n);
  cvt::k_widen<<<grid(n), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(v), vf, n);
  cvt::k_widen<<<grid(nom), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(omega), omf, nom);
  rc = cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
  if (rc == FAVOR_OK) rc = launch_f32(qf, kf, vf, omf, of, B, H, L, d, M, kind, causal, st);
  if (rc == FAVOR_OK) {
    cvt::k_narrow<<<grid(n), 256, 0, st>>>(of, static_cast<__nv_bfloat16*>(out), n);
    if (cudaGetLastError() != cudaSuccess) rc = FAVOR_ERR_CUDA;
  }
  cudaFreeAsync(ws, st);
  return rc;
}

}  // namespace

// ------------------------------------------------------------------ allocation-free fp32 entry
namespace favor {
// Scratch of favor_attention_f32_noalloc: a static device array, so that entry point needs no
// allocation. One array per device, shared by every call on that device.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
}  // namespace favor

namespace {

// Device address of the static scratch on the current device. The address belongs to the
// device's current context, which a device reset replaces, so it is looked up again on every
// call that is not being captured into a graph. A call under stream capture cannot make that
// runtime call; it takes the address the last uncaptured call on the device found.
int noalloc_scratch(void** p, cudaStream_t st) {
  static void* addr[64] = {};
  static std::mutex mu;
  *p = nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FAVOR_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FAVOR_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return FAVOR_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, favor::g_noalloc_scratch) != cudaSuccess || !a) return FAVOR_ERR_CUDA;
    addr[dev] = a;
  } else if (!addr[dev]) {
    return FAVOR_ERR_UNSUPPORTED;  // the first call on a device must not be captured
  }
  *p = addr[dev];
  return FAVOR_OK;
}

// The fp32 path's launch sequence with its workspace in the static scratch.
int launch_f32_static(const float* q, const float* k, const float* v, const float* omega, float* out,
                      int B, int H, int L, int d, int M, int kind, int causal, cudaStream_t st) {
  const int BH = B * H;
  const int F = kind == FAVOR_TRIG ? 2 * M : M;
  const int nch = (L + f32::kChunk - 1) / f32::kChunk;
  const int nft = (F + f32::kFeatTile - 1) / f32::kFeatTile;
  if (BH > 65535 || nch > 65535) return FAVOR_ERR_UNSUPPORTED;
  if (f32_workspace(BH, L, d, M, kind) > favor::kNoAllocScratchBytes) return FAVOR_ERR_UNSUPPORTED;
  void* ws = nullptr;
  int rc = noalloc_scratch(&ws, st);
  if (rc != FAVOR_OK) return rc;
  float* dS = static_cast<float*>(ws);
  float* cmax = dS + (size_t)BH * nch * F * (d + 1);
  const size_t sm_state = (size_t)(2 * f32::kChunk * d + f32::kChunk + f32::kChunk * f32::kFeatTile) * 4;
  const size_t sm_out = (size_t)(3 * f32::kChunk * d + f32::kChunk + 2 * f32::kChunk * f32::kFeatTile +
                                 f32::kFeatTile * (d + 1) + f32::kChunk * f32::kChunk) * 4;
  if (cudaFuncSetAttribute(f32::k_chunk_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_state) != cudaSuccess ||
      cudaFuncSetAttribute(f32::k_output, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_out) != cudaSuccess)
    return FAVOR_ERR_CUDA;
  if (kind == FAVOR_TRIG) f32::k_key_halfnorm_max<<<BH, f32::kThreads, 0, st>>>(k, cmax, L, d);
  f32::k_chunk_state<<<dim3(nft, nch, BH), f32::kThreads, sm_state, st>>>(k, v, omega, cmax, dS, H, L, d, M, F,
                                                                           kind);
  const long long per_chunk = (long long)F * (d + 1);
  const long long total = (long long)BH * per_chunk;
  f32::k_scan_chunks<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(dS, nch, per_chunk, total, causal);
  f32::k_output<<<dim3(nch, BH), f32::kThreads, sm_out, st>>>(q, k, v, omega, cmax, dS, out, H, L, d, M, F, kind,
                                                              causal);
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

}  // namespace

// ------------------------------------------------------------------ decode step
int check_decode(const void* state, int B, int H, int d, int M, int kind) {
  if (B <= 0 || H <= 0 || d <= 0 || M <= 0) return FAVOR_ERR_SHAPE;
  if ((long long)B * H * dec::kMaxG > INT_MAX) return FAVOR_ERR_SHAPE;
  if (kind != FAVOR_TRIG && kind != FAVOR_RELU) return FAVOR_ERR_KIND;
  if (d != 16 && d != 32 && d != 64 && d != 128) return FAVOR_ERR_UNSUPPORTED;
  if (M > (kind == FAVOR_TRIG ? dec::kMaxRows / 2 : dec::kMaxRows)) return FAVOR_ERR_UNSUPPORTED;
  (void)state;
  return FAVOR_OK;
}

long long decode_rows(int M, int kind) { return kind == FAVOR_TRIG ? 2ll * M : M; }

// Cluster size: double G (<= 8) while B*H*G CTAs fill at most half the SMs and every CTA
// keeps at least 16 angles. Large batches take G = 1 (no cluster exchange); a few heads
// (B*H = 32) take G = 4.
int decode_cluster(long long BH, int M) {
  int G = 1;
  while (G < dec::kMaxG && BH * G * 2 <= sm_count() && (M + 2 * G - 1) / (2 * G) >= 16) G *= 2;
  return G;
}

// ------------------------------------------------------------------ ORF
// One CTA per (d x d block, head): panel-blocked Gram-Schmidt in fp64 shared memory, rows scaled
// by chi lengths. The Gaussians come from G and R, or (seeded) from the Philox stream of `seed`.
int launch_orf(const double* G, const double* R, void* omega, int H, int M, int d, int omega_dtype, uint64_t seed,
               int seeded, cudaStream_t st) {
  if (H <= 0 || M <= 0 || d <= 0) return FAVOR_ERR_SHAPE;
  if (d > 128 || H > 65535) return FAVOR_ERR_UNSUPPORTED;
  if (omega_dtype != 0 && omega_dtype != 1) return FAVOR_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != FAVOR_OK) return rc;
  const int nb = (M + d - 1) / d;
  const size_t smem = orf_smem_bytes(d);
  if ((rc = ensure_smem_attr(reinterpret_cast<const void*>(k_orf), (int)smem)) != FAVOR_OK) return rc;
  k_orf<<<dim3(nb, H), kOrfThreads, smem, st>>>(G, R, omega, H, M, d, omega_dtype, seed, seeded);
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

// ------------------------------------------------------------------ fp32 backward
size_t bwd_workspace(int BH, int L, int d, int M, int kind) {
  const size_t F = kind == FAVOR_TRIG ? 2 * (size_t)M : (size_t)M;
  const size_t nch = (L + f32::kChunk - 1) / f32::kChunk;
  return (2 * (size_t)BH * nch * F * (d + 1) + (size_t)BH * L * (d + 1) + BH) * sizeof(float);
}

// cmax (trig) -> chunk states of phi(K)[V|1] and their scan (S) -> k_bwd_query (dq, e, R shares)
// -> reverse scan of R -> k_bwd_key (dk, dv). Scratch from the stream-ordered pool.
int launch_bwd_f32(const float* q, const float* k, const float* v, const float* omega, const float* dout,
                   float* dq, float* dk, float* dv, int B, int H, int L, int d, int M, int kind, int causal,
                   cudaStream_t st) {
  const int BH = B * H;
  const int F = kind == FAVOR_TRIG ? 2 * M : M;
  const int nch = (L + f32::kChunk - 1) / f32::kChunk;
  const int nft = (F + f32::kFeatTile - 1) / f32::kFeatTile;
  if (BH > 65535 || nch > 65535) return FAVOR_ERR_UNSUPPORTED;
  void* ws = nullptr;
  int rc = scratch_alloc(&ws, bwd_workspace(BH, L, d, M, kind), st);
  if (rc != FAVOR_OK) return rc;
  const size_t per = (size_t)BH * nch * F * (d + 1);
  float* dS = static_cast<float*>(ws);
  float* Rc = dS + per;
  float* E = Rc + per;
  float* cmax = E + (size_t)BH * L * (d + 1);
  const size_t sm_state = (size_t)(2 * f32::kChunk * d + f32::kChunk + f32::kChunk * f32::kFeatTile) * 4;
  const size_t sm_bwd = (size_t)bwd::bwd_smem(d).total * 4;
  if (ensure_smem_attr(reinterpret_cast<const void*>(f32::k_chunk_state), (int)sm_state) != FAVOR_OK ||
      ensure_smem_attr(reinterpret_cast<const void*>(bwd::k_bwd_query), (int)sm_bwd) != FAVOR_OK ||
      ensure_smem_attr(reinterpret_cast<const void*>(bwd::k_bwd_key), (int)sm_bwd) != FAVOR_OK)
    rc = FAVOR_ERR_CUDA;
  if (rc == FAVOR_OK) {
    if (kind == FAVOR_TRIG) f32::k_key_halfnorm_max<<<BH, f32::kThreads, 0, st>>>(k, cmax, L, d);
    f32::k_chunk_state<<<dim3(nft, nch, BH), f32::kThreads, sm_state, st>>>(k, v, omega, cmax, dS, H, L, d, M,
                                                                             F, kind);
    const long long per_chunk = (long long)F * (d + 1);
    const long long total = (long long)BH * per_chunk;
    const unsigned sblocks = (unsigned)((total + 255) / 256);
    f32::k_scan_chunks<<<sblocks, 256, 0, st>>>(dS, nch, per_chunk, total, causal);
    bwd::k_bwd_query<<<dim3(nch, BH), bwd::kThreads, sm_bwd, st>>>(q, k, v, omega, cmax, dS, dout, dq, E, Rc, H,
                                                                   L, d, M, F, kind, causal);
    bwd::k_scan_chunks_rev<<<sblocks, 256, 0, st>>>(Rc, nch, per_chunk, total, causal);
    bwd::k_bwd_key<<<dim3(nch, BH), bwd::kThreads, sm_bwd, st>>>(q, k, v, omega, cmax, Rc, E, dk, dv, H, L, d,
                                                                 M, F, kind, causal);
    if (cudaGetLastError() != cudaSuccess) rc = FAVOR_ERR_CUDA;
  }
  cudaFreeAsync(ws, st);
  return rc;
}

// ====================================================================== C ABI
extern "C" {

const char* favor_status_string(int status) {
  switch (status) {
    case FAVOR_OK: return "ok";
    case FAVOR_ERR_NULL: return "a required pointer is NULL";
    case FAVOR_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case FAVOR_ERR_SHAPE: return "a size is non-positive or too large";
    case FAVOR_ERR_KIND: return "feature_kind must be FAVOR_TRIG (0) or FAVOR_RELU (1)";
    case FAVOR_ERR_UNSUPPORTED: return "shape not supported by the library";
    case FAVOR_ERR_CUDA: return "a CUDA runtime call failed";
    case FAVOR_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case FAVOR_ERR_DEVICE: return "the current device is not sm_100";
    default: return "unknown favor status";
  }
}

int favor_sync_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FAVOR_ERR_CUDA;
  int s = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&s, favor::g_status, sizeof(int)) != cudaSuccess) return FAVOR_ERR_CUDA;
  if (cudaMemcpyToSymbol(favor::g_status, &zero, sizeof(int)) != cudaSuccess) return FAVOR_ERR_CUDA;
  return s;
}

size_t favor_workspace_bytes(int B, int H, int L, int d, int M, int feature_kind, int causal) {
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || M <= 0) return 0;
  if ((long long)B * H > INT_MAX) return 0;
  if (feature_kind != FAVOR_TRIG && feature_kind != FAVOR_RELU) return 0;
  const long long BH = (long long)B * H;
  if (check_tc_shape(d, M, feature_kind, causal) == FAVOR_OK) {
    // causal: the state stays in TMEM and partial rows cross the cluster in shared memory
    if (causal) return 0;
    SplitPlan pl{};
    if (plan_split(pl, (int)BH, L, d, M, feature_kind)) return pl.ws_bytes;
  }
  if (!cuda_core_route_ok(BH, L, d, M)) return 0;
  // the CUDA-core route: fp32 copies and output, then (not at the same time) the fp32 path's scratch
  return cuda_core_route_bytes(BH, H, L, d, M) + f32_workspace((int)BH, L, d, M, feature_kind);
}

int favor_attention_chunked(const void* q, const void* k, const void* v, const void* omega,
                            void* out, int B, int H, int L, int d, int M, int feature_kind,
                            int causal, int chunk, void* stream) {
  int rc = check_common(q, k, v, omega, out, B, H, L, d, M, feature_kind);
  if (rc != FAVOR_OK) return rc;
  if ((rc = check_device()) != FAVOR_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (check_tc_shape(d, M, feature_kind, causal) == FAVOR_OK) {
    if (causal) {
      if (chunk != 0 && chunk != cf::kTile) return FAVOR_ERR_UNSUPPORTED;
      return launch_causal_fs(q, k, v, omega, out, B, H, L, d, M, feature_kind, st);
    }
    rc = launch_bidir_split(q, k, v, omega, out, B, H, L, d, M, feature_kind, st);
    if (rc != FAVOR_ERR_UNSUPPORTED) return rc;  // unsupported: no shared-memory plan, nothing launched
  }
  // shapes the tensor-core kernels leave out: the fp32 CUDA-core kernels on widened copies
  if (causal && chunk != 0) return FAVOR_ERR_UNSUPPORTED;
  return launch_bf16_cuda_cores(q, k, v, omega, out, B, H, L, d, M, feature_kind, causal, st);
}

int favor_attention(const void* q, const void* k, const void* v, const void* omega, void* out,
                    int B, int H, int L, int d, int M, int feature_kind, int causal, void* stream) {
  return favor_attention_chunked(q, k, v, omega, out, B, H, L, d, M, feature_kind, causal, 0, stream);
}

int favor_attention_f32(const float* q, const float* k, const float* v, const float* omega,
                        float* out, int B, int H, int L, int d, int M, int feature_kind,
                        int causal, void* stream) {
  int rc = check_common(q, k, v, omega, out, B, H, L, d, M, feature_kind);
  if (rc != FAVOR_OK) return rc;
  if ((rc = check_device()) != FAVOR_OK) return rc;
  if (d > f32::kMaxD || M > 512) return FAVOR_ERR_UNSUPPORTED;
  return launch_f32(q, k, v, omega, out, B, H, L, d, M, feature_kind, causal,
                    static_cast<cudaStream_t>(stream));
}

int favor_orf_omega(const double* gauss_blocks, const double* gauss_norms, void* omega, int H, int M,
                    int d, int omega_dtype, void* stream) {
  if (!gauss_blocks || !gauss_norms || !omega) return FAVOR_ERR_NULL;
  if (!aligned16(gauss_blocks) || !aligned16(gauss_norms) || !aligned16(omega)) return FAVOR_ERR_ALIGN;
  return launch_orf(gauss_blocks, gauss_norms, omega, H, M, d, omega_dtype, 0, 0,
                    static_cast<cudaStream_t>(stream));
}

int favor_orf_omega_seeded(uint64_t seed, void* omega, int H, int M, int d, int omega_dtype, void* stream) {
  if (!omega) return FAVOR_ERR_NULL;
  if (!aligned16(omega)) return FAVOR_ERR_ALIGN;
  return launch_orf(nullptr, nullptr, omega, H, M, d, omega_dtype, seed, 1, static_cast<cudaStream_t>(stream));
}

int favor_orf_gaussians_seeded(uint64_t seed, double* gauss_blocks, double* gauss_norms, int H, int M, int d,
                               void* stream) {
  if (!gauss_blocks || !gauss_norms) return FAVOR_ERR_NULL;
  if (!aligned16(gauss_blocks) || !aligned16(gauss_norms)) return FAVOR_ERR_ALIGN;
  if (H <= 0 || M <= 0 || d <= 0) return FAVOR_ERR_SHAPE;
  if (d > 128 || H > 65535) return FAVOR_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != FAVOR_OK) return rc;
  const long long nb = (M + d - 1) / d, ng = H * nb * d * d, NG = (ng + 3) / 4 * 4, nr = (long long)H * M * d;
  const long long groups = (NG + nr + 3) / 4;
  const long long blocks = std::min<long long>((groups + 255) / 256, 8ll * sm_count());
  rng::k_orf_gaussians<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(seed, gauss_blocks,
                                                                                         gauss_norms, ng, NG, nr);
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

int favor_philox4x64(uint64_t key, uint64_t first_counter, uint64_t n_blocks, uint64_t* out, void* stream) {
  if (!out) return FAVOR_ERR_NULL;
  if (!aligned16(out)) return FAVOR_ERR_ALIGN;
  if (n_blocks == 0 || n_blocks > (1ull << 40)) return FAVOR_ERR_SHAPE;
  int rc = check_device();
  if (rc != FAVOR_OK) return rc;
  const unsigned long long blocks = std::min<unsigned long long>((n_blocks + 255) / 256, 8ull * sm_count());
  rng::k_philox_raw<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(key, first_counter, n_blocks,
                                                                                      out);
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

int favor_attention_host(const void* q, const void* k, const void* v, const void* omega, void* out,
                         int B, int H, int L, int d, int M, int feature_kind, int causal,
                         int dtype_code, void* stream) {
  int rc = check_common(q, k, v, omega, out, B, H, L, d, M, feature_kind);
  if (rc != FAVOR_OK) return rc;
  if (dtype_code != 0 && dtype_code != 1) return FAVOR_ERR_UNSUPPORTED;
  if ((rc = check_device()) != FAVOR_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  if ((rc = copy_streams(&s_in, &s_out)) != FAVOR_OK) return rc;
  const size_t es = dtype_code == 1 ? 2 : 4;
  const size_t per_b = (size_t)H * L * d * es;  // one batch entry of q, k, v or out
  const size_t nx = (size_t)B * per_b, nom = (size_t)H * M * d * es;
  // Batch slices: slice i's copy in, its forward pass and its copy out run on three streams, so
  // one slice's compute and copy out overlap the next slice's copy in.
  // (slices start at whole batch entries; they need the 16-byte alignment every entry point checks)
  const int S = per_b % 16 == 0 ? std::min(B, kHostSlices) : 1;
  void *dq = nullptr, *dk = nullptr, *dv = nullptr, *dom = nullptr, *dout = nullptr;
  cudaEvent_t ev[2 * kHostSlices + 2] = {};
  const int nev = 2 * S + 2;
  for (int e = 0; e < nev; ++e)
    if (cudaEventCreateWithFlags(&ev[e], cudaEventDisableTiming) != cudaSuccess) rc = FAVOR_ERR_CUDA;
  if (rc == FAVOR_OK && (rc = scratch_alloc(&dq, nx, st)) == FAVOR_OK) {
    scratch_alloc(&dk, nx, st);
    scratch_alloc(&dv, nx, st);
    scratch_alloc(&dom, nom, st);
    scratch_alloc(&dout, nx, st);
    if (!dk || !dv || !dom || !dout) rc = FAVOR_ERR_CUDA;
  }
  cudaEvent_t ev_alloc = ev[2 * S], ev_done = ev[2 * S + 1];
  // the copy streams may touch the buffers only after their allocation on `stream`
  if (rc == FAVOR_OK && (cudaEventRecord(ev_alloc, st) != cudaSuccess || cudaStreamWaitEvent(s_in, ev_alloc, 0) != cudaSuccess ||
                         cudaStreamWaitEvent(s_out, ev_alloc, 0) != cudaSuccess))
    rc = FAVOR_ERR_CUDA;
  if (rc == FAVOR_OK && cudaMemcpyAsync(dom, omega, nom, cudaMemcpyHostToDevice, s_in) != cudaSuccess) rc = FAVOR_ERR_CUDA;
  int issued = 0;  // slices whose compute was launched
  for (int i = 0; rc == FAVOR_OK && i < S; ++i) {
    const int b0 = (int)((long long)B * i / S), b1 = (int)((long long)B * (i + 1) / S);
    const size_t off = (size_t)b0 * per_b, len = (size_t)(b1 - b0) * per_b;
    uint8_t *q8 = static_cast<uint8_t*>(dq) + off, *k8 = static_cast<uint8_t*>(dk) + off,
            *v8 = static_cast<uint8_t*>(dv) + off, *o8 = static_cast<uint8_t*>(dout) + off;
    if (cudaMemcpyAsync(q8, static_cast<const uint8_t*>(q) + off, len, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(k8, static_cast<const uint8_t*>(k) + off, len, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(v8, static_cast<const uint8_t*>(v) + off, len, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(ev[2 * i], s_in) != cudaSuccess || cudaStreamWaitEvent(st, ev[2 * i], 0) != cudaSuccess) {
      rc = FAVOR_ERR_CUDA;
      break;
    }
    rc = dtype_code == 1
             ? favor_attention(q8, k8, v8, dom, o8, b1 - b0, H, L, d, M, feature_kind, causal, stream)
             : favor_attention_f32(reinterpret_cast<float*>(q8), reinterpret_cast<float*>(k8),
                                   reinterpret_cast<float*>(v8), static_cast<float*>(dom),
                                   reinterpret_cast<float*>(o8), b1 - b0, H, L, d, M, feature_kind, causal, stream);
    if (rc != FAVOR_OK) break;
    issued = i + 1;
    if (cudaEventRecord(ev[2 * i + 1], st) != cudaSuccess || cudaStreamWaitEvent(s_out, ev[2 * i + 1], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(out) + off, o8, len, cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
      rc = FAVOR_ERR_CUDA;
  }
  (void)issued;
  // `stream` takes over both copy streams' work before the buffers are released on it
  if (ev_alloc && ev_done) {
    if (cudaEventRecord(ev_done, s_in) == cudaSuccess) cudaStreamWaitEvent(st, ev_done, 0);
    if (cudaEventRecord(ev_done, s_out) == cudaSuccess) cudaStreamWaitEvent(st, ev_done, 0);
  }
  for (void* p : {dq, dk, dv, dom, dout})
    if (p) cudaFreeAsync(p, st);
  if (cudaStreamSynchronize(st) != cudaSuccess && rc == FAVOR_OK) rc = FAVOR_ERR_CUDA;
  for (int e = 0; e < nev; ++e)
    if (ev[e]) cudaEventDestroy(ev[e]);
  return rc;
}

int favor_attention_f32_noalloc(const float* q, const float* k, const float* v, const float* omega,
                                float* out, int B, int H, int L, int d, int M, int feature_kind,
                                int causal, void* stream) {
  int rc = check_common(q, k, v, omega, out, B, H, L, d, M, feature_kind);
  if (rc != FAVOR_OK) return rc;
  if ((rc = check_device()) != FAVOR_OK) return rc;
  if (d > f32::kMaxD || M > 512) return FAVOR_ERR_UNSUPPORTED;
  return launch_f32_static(q, k, v, omega, out, B, H, L, d, M, feature_kind, causal,
                           static_cast<cudaStream_t>(stream));
}

size_t favor_noalloc_scratch_bytes(void) { return favor::kNoAllocScratchBytes; }

int favor_attention_backward_f32(const float* q, const float* k, const float* v, const float* omega,
                                 const float* dout, float* dq, float* dk, float* dv, int B, int H, int L, int d,
                                 int M, int feature_kind, int causal, void* stream) {
  int rc = check_common(q, k, v, omega, dout, B, H, L, d, M, feature_kind);
  if (rc != FAVOR_OK) return rc;
  if (!dq || !dk || !dv) return FAVOR_ERR_NULL;
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return FAVOR_ERR_ALIGN;
  if (d > bwd::kMaxD || M > 512) return FAVOR_ERR_UNSUPPORTED;
  if ((rc = check_device()) != FAVOR_OK) return rc;
  return launch_bwd_f32(q, k, v, omega, dout, dq, dk, dv, B, H, L, d, M, feature_kind, causal,
                        static_cast<cudaStream_t>(stream));
}

size_t favor_decode_state_bytes(int B, int H, int d, int M, int feature_kind) {
  if (check_decode(nullptr, B, H, d, M, feature_kind) != FAVOR_OK) return 0;
  const long long BH = (long long)B * H;
  return (size_t)(BH * decode_rows(M, feature_kind) * (d + 1) + BH) * sizeof(float);
}

int favor_decode_init(void* state, int B, int H, int d, int M, int feature_kind, void* stream) {
  if (!state) return FAVOR_ERR_NULL;
  if (!aligned16(state)) return FAVOR_ERR_ALIGN;
  int rc = check_decode(state, B, H, d, M, feature_kind);
  if (rc != FAVOR_OK) return rc;
  if ((rc = check_device()) != FAVOR_OK) return rc;
  const long long BH = (long long)B * H;
  const long long n_sz = BH * decode_rows(M, feature_kind) * (d + 1);
  const long long blocks = std::min<long long>((n_sz + BH + 255) / 256, 8ll * sm_count());
  dec::k_decode_init<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<float*>(state), n_sz, BH);
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

int favor_decode_step(const void* q, const void* k, const void* v, const void* omega, void* state,
                      void* out, int B, int H, int d, int M, int feature_kind, void* stream) {
  if (!q || !k || !v || !omega || !state || !out) return FAVOR_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(omega) || !aligned16(state) ||
      !aligned16(out))
    return FAVOR_ERR_ALIGN;
  int rc = check_decode(state, B, H, d, M, feature_kind);
  if (rc != FAVOR_OK) return rc;
  if ((rc = check_device()) != FAVOR_OK) return rc;
  const long long BH = (long long)B * H, F = decode_rows(M, feature_kind);
  dec::DecodeParams prm{};
  prm.z_off = BH * F * d;
  prm.c_off = BH * F * (d + 1);
  prm.BH = (int)BH;
  prm.H = H;
  prm.d = d;
  prm.M = M;
  prm.kind = feature_kind;
  prm.G = decode_cluster(BH, M);
  prm.na = (M + prm.G - 1) / prm.G;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(BH * prm.G));
  cfg.blockDim = dim3(dec::kThreads);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = prm.G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void (*kern)(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, float*,
               __nv_bfloat16*, const dec::DecodeParams) = d == 16   ? dec::k_decode_step<16>
                                                         : d == 32 ? dec::k_decode_step<32>
                                                         : d == 64 ? dec::k_decode_step<64>
                                                                   : dec::k_decode_step<128>;
  if ((rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), dec::kSmemBytes)) != FAVOR_OK) return rc;
  cfg.dynamicSmemBytes = dec::kSmemBytes;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(q),
                            static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                            static_cast<const __nv_bfloat16*>(omega), static_cast<float*>(state),
                            static_cast<__nv_bfloat16*>(out), prm) == cudaSuccess
             ? FAVOR_OK
             : FAVOR_ERR_CUDA;
}

// Launch the bounded-wait self-test: a wait that nothing satisfies, limited to `limit_cycles`.
// favor_sync_status() afterwards must report FAVOR_ERR_TIMEOUT.
int favor_selftest_timeout(long long limit_cycles, void* stream) {
  int rc = check_device();
  if (rc != FAVOR_OK) return rc;
  if (limit_cycles <= 0 || limit_cycles > 4000000000ll) return FAVOR_ERR_SHAPE;
  favor::k_selftest_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

int favor_selftest_sincos(const float* u, float* sin_out, float* cos_out, int n, void* stream) {
  if (!u || !sin_out || !cos_out) return FAVOR_ERR_NULL;
  if (n <= 0) return FAVOR_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(u) | reinterpret_cast<uintptr_t>(sin_out) | reinterpret_cast<uintptr_t>(cos_out)) &
      3u)
    return FAVOR_ERR_ALIGN;
  int rc = check_device();
  if (rc != FAVOR_OK) return rc;
  favor::k_selftest_sincos<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(u, sin_out, cos_out, n);
  return cudaGetLastError() == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

}  // extern "C"
