// Internal launcher interface between the libgmuon translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cudaTypedefs.h>

namespace gm {

// The driver's cuTensorMapEncodeTiled (NULL if the driver does not provide it).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

// Column / row split counts of the power-iteration reductions. They depend
// only on the problem shape, so the workspace layout is a pure function of it.
int rebuild_row_blocks(int m);   // 64-row tiles of the fused rebuild / projection
int backproject_row_splits(int B, int m, int n);
int gram_row_splits(int B, int m);
// The factor width k rounded up to 8, 16 or 32: the depth of the codec kernels'
// warp MMA fragments (components beyond k are zero).
__host__ __device__ inline int factor_width(int k) { return k <= 8 ? 8 : (k <= 16 ? 16 : 32); }

// 32-bit words of the fragment-ordered factor copies of B matrices (layouts in
// gm_codec.cu): QF, RF, PF feed the rebuild / projection, PA, RB the residual,
// PB the back-projection.
struct FactorFrags {
  long long QF, RF, PF, PA, RB, PB;
};
FactorFrags factor_frag_words(int B, int m, int n, int k);

// ---- codec / power-iteration kernels (gm_codec.cu) ------------------------
// Q from the stored 8-bit R (norm2_int: scratch int [3][B][k], zeroed here: the
// column norms, then the P and R column maxima of launch_orth / launch_backproject)
// or from fp32 Rprev,
// with its fragments QF; from the stored state also the R and P code fragments
// RF, PF (P8, Pscale needed then).
// ids (nullable, device int64 [B]): the matrices' indices in the Rademacher counter.
cudaError_t launch_warm_start(int B, int m, int n, int k, const int8_t* R8, const float* Rscale,
                              const int8_t* P8, const float* Pscale, const float* Rprev,
                              uint64_t seed, const int64_t* ids, float* Q, int* norm2_int,
                              uint32_t* QF, uint32_t* RF, uint32_t* PF, const int32_t* skip,
                              cudaStream_t s);

// M = mu * Mprev + G where Mprev is either the rebuilt state (codes4 != NULL)
// or a dense fp32 matrix (Mprev32 != NULL) or zero; with Q != NULL also the
// projection partials Ppart f32 [B][ceil(n/128)][m][k] (sum over one 128-column
// block each). norm2_part gets one fp64 partial |M|^2 per warp of a 64 x 128 tile
// ([B][ceil(m/64)][ceil(n/128)][8]); status (nullable) gets GM_E_NONFINITE.
// Data pointers are 16-byte aligned; m and n are multiples of 16. The fused pass
// takes the ready-made fragments QF (with Q) and RF, PF (with the state); the
// rebuild alone (state, no G, no Q, no fragments) builds its fragments in each
// CTA from R8, P8.
cudaError_t launch_rebuild(int B, int m, int n, int k, const uint8_t* codes4,
                           const float* rscale, const float* cscale, const int8_t* P8,
                           const float* Pscale, const int8_t* R8, const float* Rscale,
                           const float* Mprev32, float mu, const void* G, int gdt, const float* Q,
                           const uint32_t* QF, const uint32_t* RF, const uint32_t* PF, float* M,
                           double* norm2_part, float* Ppart, int32_t* status, cudaStream_t s);

// P = orth(P~) (fp32 [B][m][k]) with its fragments PB (back-projection) and PA
// (residual, nullable) and the tensor-core residual's operand rows PT (nullable:
// [2][B][m][32] fp32, tf32 hi then lo, columns beyond k zero).
// Pmax (nullable): the column absolute maxima of P (fp32 bits, atomicMax into zeroed words).
cudaError_t launch_orth(int B, int m, int k, int csplit, const float* Ppart, double* Ptil,
                        double* gram_part, double* Lmat, const double* norm2_part, int ntiles,
                        float eps, float* scale, float* P, uint32_t* PB, uint32_t* PA, float* PT,
                        unsigned* Pmax, const int32_t* skip, cudaStream_t s);

// R = M^T P from PB, with its residual fragments RB (nullable) and operand rows RT
// (nullable, [2][B][n][32] as PT).
cudaError_t launch_backproject(int B, int m, int n, int k, const float* M, const uint32_t* PB,
                               const float* scale, void* X16, bool f16, double* Rpart,
                               float* R, uint32_t* RB, float* RT, unsigned* Rmax,
                               const int32_t* skip, cudaStream_t s);

// The step's residual pass on the tensor cores (tcgen05, kind::tf32), persistent and
// warp-specialized (one CTA per SM streaming M through a TMA ring): the same outputs
// as launch_residual_quant4 with ready-made operand rows PT, RT; status gets
// GM_E_TIMEOUT when a bounded wait runs out.
cudaError_t launch_residual_ws(int B, int m, int n, int k, const float* X, const float* P,
                               const float* R, const float* PT, const float* RT, uint8_t* codes4,
                               float* rscale, float* cscale, const unsigned* PRmax, int8_t* P8,
                               float* Pscale, int8_t* R8, float* Rscale, int64_t* step,
                               const int32_t* skip, int32_t* status, cudaStream_t s);

// flags[r][dst_index[b]] = *status for every destination r < npeers (<= kMaxPeers)
// and matrix b < B (dst_index NULL: b).
cudaError_t launch_put_status(int B, int npeers, int32_t* const* flags, const int64_t* dst_index,
                              const int32_t* status, cudaStream_t s);

// W <- W - eta (O + wd W) (O in odt: GM_F32, GM_BF16 or GM_F16); matrix b is
// left alone when skip && skip[b * skip_stride].
cudaError_t launch_weight_update(int B, int m, int n, float eta, float wd, const void* O, int odt,
                                 float* W, const int32_t* skip, int skip_stride, cudaStream_t s);

// PA, RB: ready-made fragments of -P and R (both or neither; NULL stages P, R).
// PRmax (nullable): the P then R column maxima; with it the kernel also writes the
// 8-bit state P8, Pscale, R8, Rscale and increments step.
cudaError_t launch_residual_quant4(int B, int m, int n, int k, const float* X, const float* P,
                                   const float* R, const uint32_t* PA, const uint32_t* RB,
                                   uint8_t* codes4, float* rscale, float* cscale,
                                   const unsigned* PRmax, int8_t* P8, float* Pscale, int8_t* R8,
                                   float* Rscale, int64_t* step, const int32_t* skip,
                                   cudaStream_t s);

// Residual-from-codes variant: PA, RB from the dequantized 8-bit codes of P, R
// (Pmax, Rmax: their complete column absolute maxima).
cudaError_t launch_codes_frags(int B, int m, int n, int k, const float* P, const float* R,
                               const unsigned* Pmax, const unsigned* Rmax, uint32_t* PA,
                               uint32_t* RB, float* PT, float* RT, const int32_t* skip,
                               cudaStream_t s);

cudaError_t launch_quant8(int B, int rows0, int rows1, int k, const float* X0, int8_t* c0,
                          float* s0, const float* X1, int8_t* c1, float* s1,
                          int64_t* step, const int32_t* skip, cudaStream_t s);

// The 4bit-Muon-base group codec (gm_base4.cu): 128 consecutive elements per
// absmax scale, codes packed as in the grid codec.
cudaError_t launch_group_quant4(int B, int m, int n, const float* X, uint8_t* codes4,
                                float* gscale, cudaStream_t s);
cudaError_t launch_group_dequant4(int B, int m, int n, const uint8_t* codes4, const float* gscale,
                                  float* X, cudaStream_t s);

// MuonQ's mu-law companding codec (gm_base4.cu): the same groups and layout.
cudaError_t launch_mulaw_quant4(int B, int m, int n, float mu, const float* X, uint8_t* codes4,
                                float* gscale, cudaStream_t s);
cudaError_t launch_mulaw_dequant4(int B, int m, int n, float mu, const uint8_t* codes4,
                                  const float* gscale, float* X, cudaStream_t s);

// Standalone NS input: scale = 1/(|X|_F + eps) per matrix, then the wide
// 16-bit copy Y = round(scale * X) (transposed when m > n).
cudaError_t launch_ns_prep(int B, int m, int n, const void* X, int xdt, float eps,
                           double* norm2_part, int nparts, float* scale, void* Y16, bool f16,
                           cudaStream_t s);
int ns_prep_parts(int m, int n);

// ---- tensor-core Newton-Schulz chains (gm_gemm.cu) --------------------------
constexpr int kMaxPeers = 8;   // destinations of one O store (ranks of a node)
struct NsOutput {
  int mode;            // 0: write O (dtype odt), 1: W -= eta (O + wd W)
  void* O;
  int odt;
  float* W;
  float eta, wd;
  // mode 0 only: with npeers > 0, O goes to every peer[r] (device pointers, other
  // GPUs' memory included) instead of O, matrix b of the batch at index
  // dst_index[b] (device int64) of each [.][m][n] destination
  int npeers;
  void* peer[kMaxPeers];
  const int64_t* dst_index;
};

size_t ns_standard_ws_bytes(int B, int m, int n);
size_t ns_gram_ws_bytes(int B, int m, int n);

// X16: wide-form normalised input [B][N][M'] (bf16 for standard, fp16 for
// Gram); it is overwritten. ws: scratch of the sizes above.
cudaError_t run_ns_standard(int B, int m, int n, uint16_t* X16, const float* abc, int T,
                            const NsOutput& out, void* ws, const int32_t* skip, int32_t* err,
                            cudaStream_t s);
// Rtrace, Qtrace (nullable): fp16 [T][B][Np][Np] (Np = N rounded up to 64) per-step
// copies of R_t (when the chain computes it: not on the last step of a block,
// whose R update is skipped; after a restart, the restarted Gram X X^T) and Q_t.
cudaError_t run_ns_gram(int B, int m, int n, uint16_t* X16, const float* abc, int T,
                        const int* restart_after, int n_restart, const NsOutput& out, void* ws,
                        const int32_t* skip, int32_t* err, cudaStream_t s,
                        uint16_t* Rtrace = nullptr, uint16_t* Qtrace = nullptr);

// Test hook of the bounded waits: a one-tile product that never gets its
// operands; X, D: bf16 [256][256] (never read or written).
cudaError_t run_wait_timeout_probe(const uint16_t* X, uint16_t* D, uint64_t limit_ns, cudaStream_t s);

void ns_schedule_flops(int ns_mode, int m, int n, int T, const int* restart_after,
                       int n_restart, double* flops, int* products);
int32_t* device_error_word();

}  // namespace gm
