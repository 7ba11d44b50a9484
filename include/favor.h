/*
 * favor.h - C ABI of libfavor.so: B200 (sm_100a) FAVOR attention.
 *
 * The operation. For each head h and batch b, with Q, K, V in R^{L x d} and Omega_h in R^{M x d}:
 *   out = D_hat^-1 (phi(Q) (phi(K)^T [V | 1]))
 * This is softmax attention D^-1 A V, A = exp(Q K^T / sqrt(d)), with the kernel factored as
 * exp(q.k) ~ phi(q).phi(k). phi(K)^T [V|1] (an F x (d+1) state) is formed first, then
 * left-multiplied by phi(Q), so no L x L matrix is formed. Source: the explainer page
 * "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？" (arXiv 2009.14794), section
 * "核心机制：FAVOR+". The feature maps:
 *   FAVOR_TRIG: phi(x) = exp(|x|^2/2)/sqrt(M) [cos(Omega x), sin(Omega x)], F = 2M.
 *               The random Fourier features of the Gaussian kernel ("Masked Language
 *               Modeling for Proteins via Linearly Scalable Long-Context Transformers",
 *               Methodology / 方法详解).
 *   FAVOR_RELU: phi(x) = max(Omega x, 0)/sqrt(M), F = M. A generalized-attention kernel
 *               (the same paper, 核心创新).
 * causal != 0 sums over keys j <= i only. This is the prefix sum of phi(k_j)[v_j|1]^T
 * from the explainer's 核心机制 section.
 *
 * Scaling. The library computes exp(q.k) of q and k as passed. The 1/sqrt(d) temperature is
 * the caller's d^-1/4 pre-scale of Q and K. Constant factors that cancel between numerator
 * and denominator are dropped: 1/sqrt(M), exp(|q|^2/2), and a per-head max of |k|^2/2
 * (the stabiliser). They do not change the result.
 *
 * Layout. Everything is row-major and contiguous:
 *   q, k, v, out: [B, H, L, d], d contiguous.
 *   omega:        [H, M, d], one matrix per head, shared across the batch.
 *
 * Ownership. Every pointer is owned by the caller. The library frees nothing and keeps no
 * pointer after a call returns. Device pointers must be on the current device.
 *
 * Streams. Calls are asynchronous and ordered on `stream`, passed as a cudaStream_t
 * (NULL means the legacy default stream). The return value reports argument validation and
 * launch errors. Errors from inside a kernel surface at the next synchronisation.
 * favor_sync_status() synchronises the stream and returns the device-side status word.
 *
 * Scratch. The bf16 causal path needs none (its cross-CTA sums travel through distributed
 * shared memory). The bf16 bidirectional path, favor_attention_f32,
 * favor_attention_backward_f32 and favor_attention_host take scratch from a library-owned
 * stream-ordered pool on `stream` and release it on the same stream;
 * favor_attention_f32_noalloc uses a static device array instead. The decode step keeps its
 * state in caller-owned memory and needs no scratch; so does favor_orf_omega_seeded.
 *
 * Beyond the forward pass: a causal decode step against a carried state
 * (favor_decode_*), the fp32 backward pass (favor_attention_backward_f32) and ORF redrawn on
 * the device from a seed (favor_orf_omega_seeded).
 *
 * Errors. Negative favor_status codes. On an error nothing is launched and no output is
 * written.
 */
#ifndef FAVOR_H_
#define FAVOR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FAVOR_TRIG = 0, /* cos/sin softmax-kernel random features, F = 2M */
  FAVOR_RELU = 1  /* ReLU generalized-attention features, F = M */
} favor_feature_kind;

typedef enum {
  FAVOR_OK = 0,
  FAVOR_ERR_NULL = -1,        /* a required pointer is NULL */
  FAVOR_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
  FAVOR_ERR_SHAPE = -3,       /* a size is non-positive or the total overflows */
  FAVOR_ERR_KIND = -4,        /* feature_kind is not FAVOR_TRIG / FAVOR_RELU */
  FAVOR_ERR_UNSUPPORTED = -5, /* a valid shape the library has no kernel for */
  FAVOR_ERR_CUDA = -6,        /* a CUDA runtime call failed (launch, allocation, copy) */
  FAVOR_ERR_TIMEOUT = -7,     /* a bounded device-side wait gave up */
  FAVOR_ERR_DEVICE = -8       /* the current device is not sm_100 */
} favor_status;

/*
 * bf16 forward pass: the tensor-core path.
 * q, k, v, omega, out: device pointers to __nv_bfloat16, 16-byte aligned, layouts above.
 * Tensor-core kernels: d in {16, 32, 64, 128}; 1 <= M <= 256 (trig) or <= 512 (relu); L >= 1
 * (ragged tails are masked). Bidirectional with d = 128 needs M <= 128 (shared memory of the
 * query kernel). Causal needs d <= 64 and B*H*ceil(M/64) < 2^31.
 * Other shapes with 1 <= d <= 128, M <= 512, B*H <= 65535 and ceil(L/64) <= 65535 (for
 * example causal d = 128, or d = 48) run the fp32 CUDA-core kernels of favor_attention_f32 on
 * fp32 copies of q, k, v and omega (an exact widening on the device) and round the result to
 * bf16 once; their scratch (the copies, the fp32 output and the fp32 path's chunk states) comes
 * from the same pool (favor_workspace_bytes). Shapes beyond that return FAVOR_ERR_UNSUPPORTED
 * and launch nothing.
 * Launches: bidirectional is three kernels on `stream` (key-side partial states over every SM,
 * their merge into per-head state images, then the queries); its scratch comes from the
 * library's stream-ordered pool and is released on the same stream (favor_workspace_bytes gives
 * the size). Causal is one kernel (one thread-block cluster per head) and takes no scratch.
 * Arithmetic: Q Omega^T and K Omega^T on tensor cores (bf16 in, fp32 accumulate); features in
 * fp32 registers; every product on tensor cores accumulates in fp32.
 *   Bidirectional: phi(K) and the stabiliser-weighted values are rounded to bf16 for
 *   phi(K)^T [V|1]; the merged state is rounded to fp16 under a power-of-two scale and phi(Q) to
 *   fp16 for phi(Q) S.
 *   Causal (128-token chunks): phi(K) (carrying its stabiliser weight), phi(Q), the masked
 *   intra-chunk scores and the state image are rounded to bf16; the state's normaliser column
 *   enters phi(Q).z as a bf16 hi + lo pair; the intra-chunk denominator is summed in fp32.
 * The normaliser division is in fp32, and the result is rounded once to bf16.
 * A zero denominator gives a zero output row.
 */
int favor_attention(const void* q, const void* k, const void* v, const void* omega, void* out,
                    int B, int H, int L, int d, int M, int feature_kind, int causal,
                    void* stream);

/*
 * As favor_attention, with an explicit causal chunk length. The chunk changes how the prefix
 * sum is blocked, not its value. The tensor-core kernel scans 128-token chunks: chunk 0 (the
 * default) or 128; any other value returns FAVOR_ERR_UNSUPPORTED when causal != 0, and so does
 * any chunk but 0 for a shape on the CUDA-core route (which blocks by 64 tokens). Ignored when
 * causal == 0.
 */
int favor_attention_chunked(const void* q, const void* k, const void* v, const void* omega,
                            void* out, int B, int H, int L, int d, int M, int feature_kind,
                            int causal, int chunk, void* stream);

/*
 * fp32 forward pass: the accuracy path (CUDA cores, fp32 throughout, accurate sin/cos/exp).
 * q, k, v, omega, out: device pointers to float, 16-byte aligned, same layouts.
 * Supported: 1 <= d <= 128, 1 <= M <= 512, L >= 1.
 */
int favor_attention_f32(const float* q, const float* k, const float* v, const float* omega,
                        float* out, int B, int H, int L, int d, int M, int feature_kind,
                        int causal, void* stream);

/*
 * Orthogonal random features (ORF) Omega, built on the device from Gaussian draws.
 * "Masked Language Modeling for Proteins via Linearly Scalable Long-Context Transformers"
 * (方法详解; 实验设计 ablation) and the explainer's 核心机制 section: random directions
 * constrained to a random subsample of an orthogonal matrix.
 *   gauss_blocks: device double [H, ceil(M/d), d, d], i.i.d. N(0,1). Each d x d block's rows
 *                 are orthonormalised in order (Gram-Schmidt, fp64).
 *   gauss_norms:  device double [H, M, d], i.i.d. N(0,1). Row r of Omega_h is scaled by
 *                 |gauss_norms[h, r, :]|, a chi_d length.
 *   omega:        device output [H, M, d], dtype per omega_dtype (0 = float, 1 = bf16).
 * Blocks are stacked and cut to M rows. Supported: 1 <= d <= 128, 1 <= M.
 */
int favor_orf_omega(const double* gauss_blocks, const double* gauss_norms, void* omega,
                    int H, int M, int d, int omega_dtype, void* stream);

/*
 * ORF Omega redrawn on the device from a seed: as favor_orf_omega, with the Gaussian draws
 * generated in the kernel instead of read from memory (no scratch). A new seed per call gives a
 * new draw of the orthogonal random features (the pages' ORF: "Masked Language Modeling for
 * Proteins via Linearly Scalable Long-Context Transformers", 方法详解 and 实验设计; the explainer's
 * 核心机制 section).
 * The draws: Philox4x64 with 10 rounds (Salmon, Moraes, Dror and Shaw, SC 2011), counter
 * (g, 0, 0, 0) and key (seed, 0) for group g. Each 64-bit word w gives
 * u = (floor(w / 2^11) + 1/2) 2^-53, and Box-Muller turns (u0, u1) and (u2, u3) into
 * sqrt(-2 ln u_a) (cos, sin)(2 pi u_b) in double. Draw n is normal n % 4 of group n / 4.
 * gauss_blocks[h, b, i, j] is draw ((h nb + b) d + i) d + j, with nb = ceil(M/d). gauss_norms[h, r, j]
 * is draw NG + (h M + r) d + j, with NG = H nb d d rounded up to a multiple of 4. Those are
 * exactly the arrays favor_orf_gaussians_seeded writes.
 * omega: device output [H, M, d], 16-byte aligned, dtype per omega_dtype (0 = float, 1 = bf16).
 * Supported: 1 <= d <= 128, 1 <= M, 1 <= H <= 65535.
 */
int favor_orf_omega_seeded(uint64_t seed, void* omega, int H, int M, int d, int omega_dtype, void* stream);

/*
 * The Gaussian draws behind favor_orf_omega_seeded, written out. gauss_blocks: device double
 * [H, ceil(M/d), d, d]; gauss_norms: device double [H, M, d]; both 16-byte aligned.
 * favor_orf_omega on these arrays gives the same Omega as favor_orf_omega_seeded(seed).
 */
int favor_orf_gaussians_seeded(uint64_t seed, double* gauss_blocks, double* gauss_norms, int H, int M, int d,
                               void* stream);

/*
 * The raw generator: out[4 i + w] = word w of Philox4x64-10 applied to counter
 * (first_counter + i, 0, 0, 0) with key (key, 0), for i < n_blocks (1 <= n_blocks <= 2^40).
 * out is device memory, 16-byte aligned, 4 n_blocks uint64 words.
 */
int favor_philox4x64(uint64_t key, uint64_t first_counter, uint64_t n_blocks, uint64_t* out, void* stream);

/*
 * Host-buffer convenience entry: q, k, v, omega, out are HOST pointers (pinned memory
 * makes the copies asynchronous). Allocates device buffers from the pool on `stream`, copies
 * in, runs favor_attention (dtype_code 1 = bf16) or favor_attention_f32 (dtype_code 0 =
 * float), copies out and frees. The batch is cut into up to four slices of whole batch entries
 * (slice i = entries [B i / S, B (i+1) / S); one slice when an entry's H L d elements are not a
 * multiple of 16 bytes, since every device entry needs 16-byte aligned pointers): slice i's
 * copies in run on a library-owned
 * stream, its forward pass on `stream` and its copy out on a second library stream, so one
 * slice's compute and copy out overlap the next slice's copies in; each slice's result equals
 * the device entry run on that slice alone. It synchronises `stream` before returning, so
 * `out` is ready when it returns FAVOR_OK.
 */
int favor_attention_host(const void* q, const void* k, const void* v, const void* omega,
                         void* out, int B, int H, int L, int d, int M, int feature_kind,
                         int causal, int dtype_code, void* stream);

/*
 * fp32 forward pass that allocates nothing (no counterpart on the pages: an interface for
 * callers that cannot allocate device memory). Same arguments, arithmetic and results as
 * favor_attention_f32, whose kernels it launches, but the workspace lives in a static
 * device array of favor_noalloc_scratch_bytes() bytes (32 MiB) that belongs to the library,
 * one per device. No cudaMalloc, cudaMallocAsync, cudaFree or allocating library routine is
 * called.
 *   Size limit: the workspace is B*H*ceil(L/64)*F*(d+1)*4 + B*H*4 bytes (F = 2M for trig,
 *   M for ReLU). A call whose workspace exceeds the array returns FAVOR_ERR_UNSUPPORTED and
 *   launches nothing.
 *   Overlap: every call on a device uses the same array. Calls whose executions overlap (on
 *   different streams, or from different host threads without ordering between their streams)
 *   race on it and give undefined results. Order them on one stream or with events.
 *   Address: every call that is not under stream capture looks up the array's device address
 *   with cudaGetSymbolAddress (FAVOR_ERR_CUDA if that fails), so a device reset between calls,
 *   which replaces the context the address belongs to, leaves no stale pointer behind. A call
 *   under stream capture reuses the address the last uncaptured call on the device found, and
 *   returns FAVOR_ERR_UNSUPPORTED if there was none: make a first call on each device before any
 *   stream capture begins, and again after a device reset.
 */
int favor_attention_f32_noalloc(const float* q, const float* k, const float* v, const float* omega,
                                float* out, int B, int H, int L, int d, int M, int feature_kind,
                                int causal, void* stream);

/* Size in bytes of the static workspace of favor_attention_f32_noalloc. */
size_t favor_noalloc_scratch_bytes(void);

/*
 * fp32 backward pass: the gradients dq, dk, dv of sum(dout * out), out = favor_attention_f32 of
 * the same arguments. The differentiated quantity is D^-1 A V with A = phi(Q) phi(K)^T (masked
 * to j <= i when causal), as the explainer's 核心机制 section defines it; it is computed in
 * linear time, with the causal gradients as reverse prefix sums over 64-token chunks. Omega is
 * a fixed random draw and gets no gradient. Rows whose denominator is zero (output zero) pass no
 * gradient.
 * q, k, v, dout, dq, dk, dv: device float [B, H, L, d]; omega: device float [H, M, d]; all
 * 16-byte aligned. dq, dk, dv are written in full.
 * Arithmetic: fp32 on CUDA cores, sin/cos/exp in double rounded to fp32. Feature scale
 * factors that cancel (exp(|q|^2/2), the key stabiliser, 1/sqrt(M)) are dropped.
 * Scratch: 2 B H ceil(L/64) F (d+1) + B H L (d+1) + B H floats from the library's stream-ordered
 * pool on `stream`.
 * Supported: 1 <= d <= 64, 1 <= M <= 512, L >= 1, B*H <= 65535, ceil(L/64) <= 65535.
 */
int favor_attention_backward_f32(const float* q, const float* k, const float* v, const float* omega,
                                 const float* dout, float* dq, float* dk, float* dv, int B, int H, int L, int d,
                                 int M, int feature_kind, int causal, void* stream);

/*
 * Causal decode: one token per (batch, head) per call, against a carried state.
 * The explainer's 核心机制 section: the causal prefix sums S_t = S_{t-1} + phi(k_t) v_t^T and
 * z_t = z_{t-1} + phi(k_t), read by the same token's query: out_t = phi(q_t) S_t / phi(q_t) z_t.
 * From a state set by favor_decode_init, calls on tokens 0 .. t return causal rows 0 .. t of
 * favor_attention(causal = 1) on the same sequence. Each call streams the state once (an
 * HBM-bound matrix-vector product on CUDA cores); the cost per token does not grow with t.
 *
 * State (owned by the caller, device memory, 16-byte aligned, favor_decode_state_bytes() bytes),
 * fp32, three regions one after another, heads numbered bh = b*H + h:
 *   S [B*H, F, d]   the state rows; F = 2M (trig: M cos rows, then M sin rows) or M (ReLU)
 *   z [B*H, F]      the normaliser column
 *   c [B*H]         the stabiliser reference: -inf when empty, then the running max of |k|^2/2
 * Trig rows are stored as the sum of exp(|k_j|^2/2 - c) [cos(Omega k_j), sin(Omega k_j)] [v_j | 1];
 * ReLU rows as the sum of max(Omega k_j, 0) [v_j | 1]; the factor 1/sqrt(M) is dropped (it
 * cancels). Where c grows, S and z are rescaled by exp(c_old - c_new) in the same pass.
 *
 * favor_decode_step: q, k, v, out [B, H, d] bf16 (this token of every head); omega [H, M, d] bf16.
 * Device pointers, 16-byte aligned. Reads and rewrites `state` in place; calls on one state must
 * be ordered (one stream, or events). Arithmetic: projections, features (sincosf, expf) and the
 * state in fp32; the row is divided in fp32 and rounded once to bf16. A zero denominator gives a
 * zero row. Supported: d in {16, 32, 64, 128}; 1 <= M <= 512 (trig) or <= 1024 (ReLU);
 * B*H*8 <= INT_MAX. Other shapes return FAVOR_ERR_UNSUPPORTED (or FAVOR_ERR_SHAPE for sizes
 * that are non-positive or too large) and launch nothing.
 */
size_t favor_decode_state_bytes(int B, int H, int d, int M, int feature_kind); /* 0: unsupported */
int favor_decode_init(void* state, int B, int H, int d, int M, int feature_kind, void* stream);
int favor_decode_step(const void* q, const void* k, const void* v, const void* omega, void* state,
                      void* out, int B, int H, int d, int M, int feature_kind, void* stream);

/* Synchronise `stream`, then read and clear the device status word (FAVOR_OK or a code). */
int favor_sync_status(void* stream);

/* Static description of a status code. Never NULL. */
const char* favor_status_string(int status);

/*
 * Self-test of the bounded device-side waits (no counterpart on the pages). Launches one block
 * that waits on a barrier nothing completes, for at most `limit_cycles` SM clock cycles
 * (0 < limit_cycles <= 4e9). favor_sync_status() afterwards returns FAVOR_ERR_TIMEOUT, and the
 * context stays usable.
 */
int favor_selftest_timeout(long long limit_cycles, void* stream);

/*
 * Self-test of the FMA-pipe sine and cosine the trig kernels can use in place of the SFU's (no
 * counterpart on the pages; the method is a Cody-Waite reduction by pi and minimax polynomials on
 * [-pi/2, pi/2], coefficients derived in csrc/sincos_coeffs.py). u, sin_out, cos_out: device
 * pointers to n floats, 4-byte aligned; sin_out[i] and cos_out[i] receive sin(u[i]) and cos(u[i]).
 * Accurate to 1e-6 (sin) and 2e-7 (cos) absolute for |u| <= 400. Errors: FAVOR_ERR_NULL,
 * FAVOR_ERR_SHAPE (n <= 0), FAVOR_ERR_ALIGN, FAVOR_ERR_DEVICE, FAVOR_ERR_CUDA.
 */
int favor_selftest_sincos(const float* u, float* sin_out, float* cos_out, int n, void* stream);

/*
 * Bytes of scratch one favor_attention call takes from the library's stream-ordered pool (host
 * only; no launch). Bidirectional: the key kernel's partial states (fp32) and their references,
 * and the merged state images the query kernel reads; the run split follows the current
 * device's SM count. Causal: 0 (the state stays in TMEM, partial rows cross the cluster in
 * shared memory). Shapes on the CUDA-core route: the fp32 copies of q, k, v, out and omega plus
 * the fp32 path's chunk states. 0 for non-positive sizes and for shapes without a kernel.
 */
size_t favor_workspace_bytes(int B, int H, int L, int d, int M, int feature_kind, int causal);

#ifdef __cplusplus
}
#endif
#endif /* FAVOR_H_ */
