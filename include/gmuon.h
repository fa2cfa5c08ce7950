/*
 * libgmuon -- one 4-bit-Muon-GRASP optimizer step on an NVIDIA B200 (sm_100a).
 *
 * C ABI. Every pointer argument is a DEVICE pointer unless marked "host".
 * All matrices are row-major and batch-contiguous: a call operates on B
 * same-shape matrices stored back to back (batch stride = rows * cols).
 * Shapes: batch 1 <= B <= 65535; m, n multiples of 16, 16 <= m, n <= 65536;
 * top rank 1 <= k <= 32. An empty batch or matrix (B, m or n = 0) is an
 * argument error (GM_E_ARG), not a no-op: a caller skips empty groups itself.
 * Every device array pointer must be 16-byte aligned (the kernels move
 * 16-byte vectors); a misaligned pointer returns GM_E_ARG.
 * The 4-bit grid uses fixed 128 x 128 blocks (ragged edge blocks allowed).
 *
 * Ownership: the caller allocates every buffer (typically torch tensors) and
 * keeps it alive until the stream work completes. The library never
 * allocates or frees device memory (gm_ipc_open only maps another process's
 * allocation, which gm_ipc_close unmaps) and keeps no per-call device state.
 * Library-wide device state is limited to two file-scope arrays that every
 * GPU loading the library holds: one int32 error word (see
 * gm_device_errors) and the scratch of gm_newton_schulz_noalloc.
 *
 * Devices: one process may drive several GPUs; each call works on the
 * current device. Kernel attributes and looked-up device addresses are set
 * up once per device on first use (thread-safe). These caches do not survive
 * cudaDeviceReset (or any other primary-context reset): do not reset a
 * device between calls into the library.
 *
 * Execution: every call enqueues work on `stream` and returns without
 * synchronising. Argument errors are detected on the host before any launch
 * and return GM_E_ARG (nothing is enqueued). A CUDA launch error returns
 * GM_E_CUDA. Device-side conditions (non-finite input, a bounded wait that
 * ran out) are reported through `dev_status` words or gm_device_errors().
 *
 * Sources (cited per entry point):
 *  [GRASP]  "Achieving low-bit Muon through subspace preservation and grid
 *           quantization" (ICLR 2026 paper note)
 *  [LiMuon] "LiMuon: Light and Fast Muon Optimizer for Large Models" (note)
 *  [GramNS] "优化器 (3)（Gram Newton-Schulz）" (blog post on Gram NS)
 */
#ifndef GMUON_H
#define GMUON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GMUON_VERSION 1
#define GM_GRID_BLOCK 128
#define GM_MAX_K 32
#define GM_MAX_T 16

/* Same underlying type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* gm_stream_t;

typedef int gm_status;
enum {
  GM_OK = 0,
  GM_E_ARG = -1,          /* bad shape, pointer, dtype or parameter */
  GM_E_CUDA = -2,         /* a CUDA runtime call or launch failed */
  GM_E_NONFINITE = -3,    /* NaN/Inf in G or in the rebuilt momentum (device) */
  GM_E_WORKSPACE = -4,    /* workspace pointer NULL or smaller than required */
  GM_E_UNSUPPORTED = -5,  /* device is not sm_100 */
  GM_E_TIMEOUT = -6       /* a kernel's bounded wait ran out (device) */
};

typedef enum { GM_F32 = 0, GM_BF16 = 1, GM_F16 = 2 } gm_dtype;
typedef enum { GM_NS_STANDARD = 0, GM_NS_GRAM = 1 } gm_ns_mode;
typedef enum {
  GM_OP_MOMENTUM_POWERIT = 1,
  GM_OP_NEWTON_SCHULZ = 2,
  GM_OP_GRAM_NS = 3,
  GM_OP_GRASP_STEP = 4
} gm_op;

/* Human-readable name of a status code (static string). */
const char* gm_status_string(gm_status s);
/* Detail of the last host-side error on the calling thread (static per thread). */
const char* gm_last_error(void);
int gm_version(void);

/*
 * Workspace bytes needed by `op` for B matrices of m x n with top rank k.
 * `ns_mode` matters for GM_OP_GRASP_STEP only. Returns 0 on bad arguments.
 * The workspace must be 256-byte aligned.
 */
size_t gm_workspace_bytes(int op, int B, int m, int n, int k, int ns_mode);

/*
 * Rebuild the previous momentum from the stored low-bit state
 * [GRASP, worked step, step 1]:
 *   M[i][j] = (q4_ij / 7) * s_ij + sum_l (p_il / 127 * Pscale_l)(r_jl / 127 * Rscale_l)
 * with s_ij = min(rscale[i][j/128], cscale[i/128][j]).
 *   codes4  uint8 [B][m][n/2]  two's-complement nibbles, low nibble = even col
 *   rscale  f32   [B][m][ceil(n/128)]   cscale f32 [B][ceil(m/128)][n]
 *   P8 int8 [B][m][k], Pscale f32 [B][k], R8 int8 [B][n][k], Rscale f32 [B][k]
 *   M_out   f32   [B][m][n]
 * k = 0 rebuilds the residual only (P8..Rscale may be NULL).
 */
gm_status gm_dequant_rebuild(int B, int m, int n, int k,
                             const uint8_t* codes4, const float* rscale, const float* cscale,
                             const int8_t* P8, const float* Pscale,
                             const int8_t* R8, const float* Rscale,
                             float* M_out, gm_stream_t stream);

/*
 * Momentum update and one warm-started power iteration
 * [GRASP, key design 1; worked step, steps 2-4]:
 *   M = mu * M_prev + G
 *   Q[:, l] = R_prev[:, l] / |R_prev[:, l]|   (Rademacher +-1/sqrt(n) column when
 *             R_prev is NULL or the column is zero; sign = top bit of
 *             splitmix64(seed ^ b<<48 ^ j<<16 ^ l), b = index in the batch)
 *   P = orth(M Q)  (thin QR, positive diagonal; a column whose residual is
 *                   <= 1e-6 * max column norm of M Q is zero)
 *   R = M^T P
 *   M_prev f32 [B][m][n] (NULL: zero), G [B][m][n] of dtype gdt (f32/bf16/f16),
 *   R_prev f32 [B][n][k] or NULL, M_out f32 [B][m][n], P_out f32 [B][m][k],
 *   R_out f32 [B][n][k]; ws >= gm_workspace_bytes(GM_OP_MOMENTUM_POWERIT, ...).
 */
gm_status gm_momentum_powerit(int B, int m, int n, int k, float mu,
                              const float* M_prev, const void* G, gm_dtype gdt,
                              const float* R_prev, uint64_t seed,
                              float* M_out, float* P_out, float* R_out,
                              void* ws, size_t ws_bytes, gm_stream_t stream);

/*
 * 4-bit grid quantization of X - P R^T [GRASP, key design 2, N_grid;
 * worked step 5]. Per 128 x 128 block: r_i = max_j |x_ij|, c_j = max_i |x_ij|,
 * s_ij = min(r_i, c_j), q = clamp(rint(fp32(x / s) * 7), -7, 7) (IEEE fp32
 * division, ties to even), s = 0 -> q = 0.
 *   X f32 [B][m][n]; P f32 [B][m][k] and R f32 [B][n][k] both NULL (quantize X)
 *   or both non-NULL (quantize the residual, fp32 FMA); codes4/rscale/cscale as
 *   in gm_dequant_rebuild (outputs). block is the grid block side: 128, the
 *   size the method uses and the only one built (anything else: GM_E_INVALID);
 *   k is ignored when P and R are NULL.
 */
gm_status gm_grid_quant4(int B, int m, int n, int block, int k, const float* X,
                         const float* P, const float* R,
                         uint8_t* codes4, float* rscale, float* cscale, gm_stream_t stream);

/*
 * 8-bit per-column absmax quantization of P or R [GRASP, worked step 5;
 * training strategy: INT8 factors]:
 *   s_l = max_i |x_il|; q = clamp(rint(fp32(x / s_l) * 127), -127, 127); s = 0 -> 0.
 *   X f32 [B][rows][k] -> codes int8 [B][rows][k], colscale f32 [B][k];
 *   1 <= rows <= 2^20 (any count, not only multiples of 16).
 */
gm_status gm_quant8(int B, int rows, int k, const float* X,
                    int8_t* codes, float* colscale, gm_stream_t stream);

/*
 * The 4bit-Muon-base codec: direct 4-bit quantization of the whole momentum,
 * the baseline [GRASP] compares its codec with (research background: the
 * error NS amplifies; the results tables' "4bit-Muon-base" rows). The page
 * does not describe its grouping; this library's reading: one absmax scale per
 * group of 128 consecutive row-major elements (m n is a multiple of 256, so no
 * group is ragged or spans two matrices):
 *   s_g = max |x| over the group; q = clamp(rint(fp32(x / s_g) * 7), -7, 7);
 *   s_g = 0 -> q = 0; a NaN in a group makes s_g NaN and its codes 0.
 *   X f32 [B][m][n] -> codes4 uint8 [B][m][n/2] (nibbles as in
 *   gm_dequant_rebuild), gscale f32 [B][m*n/128].
 */
gm_status gm_group_quant4(int B, int m, int n, const float* X, uint8_t* codes4, float* gscale,
                          gm_stream_t stream);
/* The inverse: X_out[e] = fp32(q_e / 7) * s_g (f32 [B][m][n]). */
gm_status gm_group_dequant4(int B, int m, int n, const uint8_t* codes4, const float* gscale,
                            float* X_out, gm_stream_t stream);

/*
 * MuonQ's mu-law companding 4-bit codec ("MuonQ: Enhancing Low-Bit Muon
 * Quantization via Directional Fidelity Optimization", abstract: mu-law
 * companding gives finer steps where the momentum values are dense). The
 * abstract states neither mu nor the pre-quantization normalisation; this
 * library's reading: the groups, absmax scales and code layout of the
 * 4bit-Muon-base codec above, and
 *   F(y) = sign(y) ln(1 + mu |y|) / ln(1 + mu),  q = clamp(rint(7 F(x / s_g)), -7, 7)
 * (s_g = 0 or NaN -> q = 0); decided exactly: |q| >= j iff |x| / s_g >=
 * F^-1((j - 1/2) / 7) (ties of the rounding, which have measure zero, go up).
 * Decode: X_out = s_g F^-1(|q| / 7) sign(q), the level F^-1(|q| / 7) in fp32.
 * 0 < mu <= 1e6 (255 is the telephony value).
 */
gm_status gm_mulaw_quant4(int B, int m, int n, float mu, const float* X, uint8_t* codes4,
                          float* gscale, gm_stream_t stream);
gm_status gm_mulaw_dequant4(int B, int m, int n, float mu, const uint8_t* codes4,
                            const float* gscale, float* X_out, gm_stream_t stream);

/*
 * Standard quintic Newton-Schulz [GramNS §1.2, eq. (2); Algorithm 1 first
 * line for the normalisation; LiMuon key design 3 for the coefficients]:
 *   wide form Y = X (m <= n) or X^T (m > n); Y <- Y / (|Y|_F + eps);
 *   T times: A = Y Y^T; B = b A + c A^2; Y <- a Y + B Y;  O = Y (or Y^T).
 * Operands are bf16 with fp32 accumulation on the tensor cores; X^T-products
 * that produce a symmetric matrix compute one triangle and mirror it.
 *   X [B][m][n] of dtype xdt (f32/bf16/f16); abc host f32 [3T] (a_t, b_t, c_t)
 *   per step, NULL = the constant quintic (3.4445, -4.7750, 2.0315);
 *   1 <= T <= 16; O [B][m][n] of dtype odt.
 */
gm_status gm_newton_schulz(int B, int m, int n, const void* X, gm_dtype xdt,
                           const float* abc, int T, float eps,
                           void* O, gm_dtype odt,
                           void* ws, size_t ws_bytes, gm_stream_t stream);

/*
 * gm_newton_schulz without any device allocation (the paper has no counterpart:
 * this is a deployment convenience of this library).
 *
 * For callers that cannot allocate GPU memory where they need the update --
 * code running inside a framework that owns every allocation through its own
 * pool, plugins that may not call the device allocator, or paths where an
 * allocation would synchronise the device. Same arguments and result as
 * gm_newton_schulz, minus the workspace: the scratch is a fixed device array of
 * GM_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits. The call makes no cudaMalloc,
 * cudaFree or other allocating call.
 *  - Shapes whose workspace (gm_workspace_bytes(GM_OP_NEWTON_SCHULZ, ...))
 *    exceeds GM_NOALLOC_SCRATCH_BYTES are rejected with GM_E_WORKSPACE before
 *    any launch; gm_last_error() states the bytes needed.
 *  - The first call on a device looks up the scratch array's device address
 *    (cudaGetSymbolAddress) with that device current and caches it; make that
 *    first call before any stream capture. The cached address does not survive
 *    cudaDeviceReset: do not reset the device between calls.
 *  - All calls share the one scratch array and it keeps the last call's
 *    contents (nothing in it needs to start at zero: every byte a call reads,
 *    it first writes). Calls that overlap on the GPU -- different streams, or
 *    threads enqueueing concurrently -- race on it: serialise them.
 */
#define GM_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
gm_status gm_newton_schulz_noalloc(int B, int m, int n, const void* X, gm_dtype xdt,
                                   const float* abc, int T, float eps,
                                   void* O, gm_dtype odt, gm_stream_t stream);

/*
 * Stabilized Gram Newton-Schulz [GramNS Algorithm 2; Algorithm 1 with
 * n_restart = 0]: fp16 operands, fp32 accumulation, a_t added in fp32
 * epilogues:
 *   Y <- fp16(Y / (|Y|_F + eps)); R = Y Y^T; Q = I;
 *   per step: Z = b R + c R^2; Q <- Q Z + a Q; RZ = R Z + a R; R <- Z RZ + a RZ;
 *   after each step listed in restart_after (host int[n_restart], 1-based,
 *   < T): Y <- Q Y, R <- Y Y^T, Q <- I.  O = Q Y (transposed back if tall).
 * Products whose result is not used again are skipped (Q_1 = Z + a I; no R
 * update on the last step of a block).
 */
gm_status gm_gram_ns(int B, int m, int n, const void* X, gm_dtype xdt,
                     const float* abc, int T, const int* restart_after, int n_restart,
                     float eps, void* O, gm_dtype odt,
                     void* ws, size_t ws_bytes, gm_stream_t stream);

/*
 * gm_gram_ns, also copying the chain's fp16 Gram and transform matrices after
 * every step, for checking the restart bounds [GramNS §3.2: with a restart
 * after step 2, the smallest eigenvalue of R_t stays above -0.4 and the
 * condition number of Q_t below about 100]. Rtrace and Qtrace are fp16
 * [T][B][Np][Np], Np = min(m, n) rounded up to a multiple of 64 (the chain's
 * zero-padded size; the valid block is the leading min(m, n) square):
 *   Qtrace[t-1] = Q_t after step t (before a restart resets it);
 *   Rtrace[t-1] = R_t after step t when the chain computes it (not on the last
 *     step of a block, whose R update is skipped); after a restart at step t,
 *     the restarted Gram X_t X_t^T; untouched for t = T.
 */
gm_status gm_gram_ns_trace(int B, int m, int n, const void* X, gm_dtype xdt, const float* abc,
                           int T, const int* restart_after, int n_restart, float eps, void* O,
                           gm_dtype odt, uint16_t* Rtrace, uint16_t* Qtrace, void* ws,
                           size_t ws_bytes, gm_stream_t stream);

/* Hyper-parameters of one GRASP step (host struct). */
typedef struct {
  float mu;                  /* momentum coefficient */
  float eta;                 /* learning rate */
  float wd;                  /* decoupled weight decay lambda */
  int k;                     /* top rank, 1..32 */
  int T;                     /* NS steps, 1..16 */
  gm_ns_mode ns;             /* standard (bf16) or Gram (fp16) NS */
  const float* abc;          /* host f32 [3T] or NULL for the constant quintic */
  const int* restart_after;  /* host, Gram NS only (NULL with n_restart = 0) */
  int n_restart;
  float eps;                 /* Frobenius normalisation epsilon (1e-7) */
  uint64_t seed;             /* Rademacher start vectors */
  /* The fields below may be left zero (their defaults): */
  int power_steps;           /* power-iteration steps per GRASP step, 1..3 (0 = 1). Each
                                step after the first restarts from Q = column-normalised R
                                of the one before ([GRASP] ablation table: 1/2/3 steps) */
  int residual_from_codes;   /* 0: residual M_t - P R^T with the unquantized P, R
                                ([GRASP] worked step 5); 1: M_t - P^ R^T with P^, R^ the
                                dequantized 8-bit codes of this step */
  const int64_t* matrix_ids; /* device int64 [B] or NULL: the index b that the Rademacher
                                counter uses for each matrix (NULL: 0 .. B-1). Giving each
                                matrix its index in the whole parameter set makes the start
                                vectors independent of how a set is split into calls (e.g.
                                across ranks); ids lie in [0, 65536) */
  int block;                 /* grid block side of the 4-bit residual: 0 or 128 (the only
                                size built; anything else: GM_E_INVALID) */
} gm_grasp_params;

/* The quantized momentum state [GRASP, worked step, last paragraph];
 * all device pointers, layouts as in gm_dequant_rebuild. A zero state (all
 * codes and scales 0, *step = 0) is the state before the first step. */
typedef struct {
  uint8_t* codes4;
  float* rscale;
  float* cscale;
  int8_t* P8;
  float* Pscale;
  int8_t* R8;
  float* Rscale;
  int64_t* step;        /* [1] incremented on device by every completed step */
  int32_t* dev_status;  /* [1] written by every step: GM_OK, GM_E_NONFINITE or GM_E_TIMEOUT */
} gm_grasp_state;

/*
 * One full GRASP step for B same-shape matrices [GRASP, overall framework;
 * worked step 1-6]:
 *   rebuild M_{t-1}; warm start Q; M_t = mu M_{t-1} + G; P, R = PowerIter(M_t, Q);
 *   residual M_t - P R^T -> 4-bit grid codes; P, R -> 8-bit codes (state updated
 *   in place); O = NS(M_t) (standard or Gram); W <- W - eta (O + wd W).
 * The Rademacher start column of matrix b (step 1, or a zero column of the
 * stored R) takes its sign from splitmix64(seed ^ id<<48 ^ j<<16 ^ l), id =
 * matrix_ids[b] or b.
 *   W f32 [B][m][n] (in place), G [B][m][n] of dtype gdt.
 * If G or M_t holds a NaN/Inf, *dev_status = GM_E_NONFINITE and W and the
 * state are left unchanged (the step counter too).
 */
gm_status gm_grasp_step(int B, int m, int n, const gm_grasp_params* params,
                        const gm_grasp_state* state, float* W, const void* G, gm_dtype gdt,
                        void* ws, size_t ws_bytes, gm_stream_t stream);

/*
 * gm_grasp_step in its two halves, on the same arguments and workspace
 * (gm_grasp_step = gm_grasp_state_update, then gm_grasp_apply):
 *  - gm_grasp_state_update: worked steps 1-5 (rebuild, warm start, momentum,
 *    power iteration, re-quantization into `state`); it resets and then writes
 *    *dev_status and leaves M_t, P, R and the normalised NS input X in `ws`.
 *  - gm_grasp_apply: worked step 6 on the X that the state update left in
 *    `ws`: O = NS(X), W <- W - eta (O + wd W); nothing happens (W unchanged)
 *    when *dev_status is non-zero. The NS chain overwrites X.
 * A caller may run other work between the halves on the same stream, as long
 * as it leaves `ws` and the state alone.
 */
gm_status gm_grasp_state_update(int B, int m, int n, const gm_grasp_params* params,
                                const gm_grasp_state* state, const void* G, gm_dtype gdt,
                                void* ws, size_t ws_bytes, gm_stream_t stream);
gm_status gm_grasp_apply(int B, int m, int n, const gm_grasp_params* params,
                         const gm_grasp_state* state, float* W,
                         void* ws, size_t ws_bytes, gm_stream_t stream);

/*
 * Worked step 6 split at O, for callers that move O before applying it (a
 * parameter set split across ranks by ownership exchanges the owners' 16-bit
 * O: half the bytes of their fp32 weights):
 *  - gm_grasp_orth: O = NS(X) on the X that gm_grasp_state_update left in
 *    `ws` (the NS form, table and restarts of `params`), written to O
 *    [B][m][n] in odt (GM_F32, GM_BF16 or GM_F16; device, 16-byte aligned,
 *    owned by the caller). When *dev_status is non-zero nothing is written.
 *    The NS chain overwrites X.
 *  - gm_weight_update: W <- W - eta (O + wd W), elementwise in fp32 with O
 *    widened from odt; W f32 [B][m][n] (device, 16-byte aligned, in place).
 *    skip (device int32, nullable): matrix b keeps its weights when
 *    skip[b * skip_stride] is non-zero (skip_stride 0: one flag for the whole
 *    batch, e.g. a state's dev_status; 1: one flag per matrix).
 * gm_grasp_state_update, gm_grasp_orth (O in GM_F32) and gm_weight_update
 * give W within fp32 rounding of gm_grasp_step's (whose last NS product
 * applies the same update to its fp32 accumulators); with O in 16 bits, within
 * eta times O's rounding. Every rank that applies the same O to the same W gets
 * the same bits.
 */
gm_status gm_grasp_orth(int B, int m, int n, const gm_grasp_params* params,
                        const gm_grasp_state* state, void* O, gm_dtype odt,
                        void* ws, size_t ws_bytes, gm_stream_t stream);
gm_status gm_weight_update(int B, int m, int n, float eta, float wd, const void* O, gm_dtype odt,
                           float* W, const int32_t* skip, int skip_stride, gm_stream_t stream);

/*
 * gm_grasp_orth with O delivered to several receive buffers at once, for a set
 * split by ownership across the GPUs of a node: the last NS product's epilogue
 * stores each element of O into every peer_O[r] (r < npeers <= 8: device
 * pointers, other GPUs' memory mapped through gm_ipc_open included; plain
 * stores, over NVLink for a peer) at matrix dst_index[b] (device int64 [B];
 * NULL: b) of that [.][m][n] buffer in odt; then peer_flags[r][dst_index[b]]
 * (int32) = *dev_status for every r and b. The compute step and the exchange
 * are one pass: no separate all-gather. When *dev_status is non-zero no O is
 * written, only the flags. The caller orders the receivers' reads after every
 * sender's call has completed (e.g. a stream synchronize and a host barrier)
 * and keeps a receive buffer alive while senders may write it.
 */
gm_status gm_grasp_orth_peers(int B, int m, int n, const gm_grasp_params* params,
                              const gm_grasp_state* state, void* const* peer_O,
                              int32_t* const* peer_flags, int npeers, const int64_t* dst_index,
                              gm_dtype odt, void* ws, size_t ws_bytes, gm_stream_t stream);

/*
 * Device buffers shared between the processes of one node (CUDA IPC), for the
 * receive buffers of gm_grasp_orth_peers.
 *  - gm_ipc_export: the handle of the allocation that holds dev_ptr and the
 *    offset of dev_ptr in it.
 *  - gm_ipc_open (in another process): maps that allocation, *base its start
 *    (add the exporter's offset); peer access is enabled on first use.
 *  - gm_ipc_close: unmaps a base returned by gm_ipc_open.
 * The exporter keeps the allocation alive until every importer has closed it.
 */
typedef struct {
  unsigned char bytes[64];
} gm_ipc_handle;
gm_status gm_ipc_export(const void* dev_ptr, gm_ipc_handle* handle, size_t* offset);
gm_status gm_ipc_open(const gm_ipc_handle* handle, void** base);
gm_status gm_ipc_close(void* base);

/* Byte offsets of the stage buffers inside the gm_grasp_step workspace, for
 * inspection by tests: M f32 [B][m][n]; Q f32 [B][n][k]; P, R f32; X the NS
 * input (bf16 or fp16, wide form); scale f32 [B] = 1/(|M|_F + eps). */
typedef struct {
  size_t M, Q, P, R, X, scale, total;
} gm_grasp_ws_layout;
gm_status gm_grasp_workspace_layout(int B, int m, int n, int k, int ns_mode,
                                    gm_grasp_ws_layout* out);

/* Algorithmic FLOPs (symmetric products counted once) and product count of
 * the NS schedule this library issues for one matrix [GramNS §1.2, §2.4, §3.4]. */
gm_status gm_ns_flops(int ns_mode, int m, int n, int T, const int* restart_after,
                      int n_restart, double* flops, int* products);

/* Synchronises `stream`, then reads and clears the current device's error
 * word, which the standalone NS entry points' kernels set when a bounded wait
 * ran out (gm_grasp_step reports through its state's dev_status instead).
 * The word is shared by every stream and thread on that device: a timeout is
 * reported to whichever caller reads the word first. Returns GM_OK or
 * GM_E_TIMEOUT (or GM_E_CUDA). */
gm_status gm_device_errors(gm_stream_t stream);

/*
 * Test hook of the failure path (not part of the method): launches the NS
 * product kernel on one 256 x 256 tile with its operand copies withheld, so
 * that the bounded wait for the first operand stage runs out after limit_ns
 * (1 ms .. 1 s). The kernel then records GM_E_TIMEOUT in the current device's
 * error word, every role leaves its loop, and the tensor memory is released;
 * gm_device_errors() then returns GM_E_TIMEOUT (and clears the word), and the
 * device stays usable. X, D: bf16 [256][256] device buffers, never read or
 * written (the operand and output maps need real addresses).
 */
gm_status gm_test_wait_timeout(const uint16_t* X, uint16_t* D, int64_t limit_ns,
                               gm_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* GMUON_H */
