// extern "C" entry points of libgmuon: argument validation, workspace
// layout and the enqueueing of the step's kernels on the caller's stream.

#include <stdarg.h>
#include <atomic>
#include <cmath>
#include <stdio.h>
#include <string.h>

#include "gm_common.cuh"
#include "gm_internal.h"

namespace gm {

namespace {

thread_local char g_last_error[512] = "";

size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

const float kQuintic[3] = {3.4445f, -4.7750f, 2.0315f};

// The current device is an sm_100 part (checked once per device).
bool device_ok() {
  static std::atomic<int> verdict[kMaxDevices];   // 0 unknown, 1 sm_100, 2 other
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  int v = verdict[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return false;
    v = (major == 10 && minor == 0) ? 1 : 2;
    verdict[dev].store(v, std::memory_order_relaxed);
  }
  return v == 1;
}

bool shape_ok(int B, int m, int n) {
  return B >= 1 && B <= 65535 && m >= 16 && n >= 16 && m <= 65536 && n <= 65536 &&
         m % 16 == 0 && n % 16 == 0;
}

// Expand an (a, b, c) table: NULL -> the constant quintic T times.
void expand_abc(const float* abc, int T, float* out) {
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < 3; ++j) out[3 * t + j] = abc ? abc[3 * t + j] : kQuintic[j];
}

struct StepLayout {
  size_t M, Q, P, R, X, scale, norm2, Ppart, Ptil, gram, Tm, Rpart, qnorm, QF, RF, PF, PA, RB, PB,
      PT, RT, ns, total;
  int csplit, rsplit_b, rsplit_g, ntiles;
};

StepLayout step_layout(int B, int m, int n, int k, int ns_mode, bool with_ns) {
  StepLayout L;
  memset(&L, 0, sizeof(L));
  L.csplit = cdiv(n, kGrid);                        // projection partials: one per 128-column block
  L.rsplit_b = backproject_row_splits(B, m, n);
  L.rsplit_g = gram_row_splits(B, m);
  L.ntiles = rebuild_row_blocks(m) * cdiv(n, kGrid) * 8;  // |M|^2 partials: one per warp of a tile
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += al256(bytes); return o; };
  const size_t Bz = (size_t)B, mz = (size_t)m, nz = (size_t)n, kz = (size_t)k;
  L.M = take(Bz * mz * nz * 4);
  L.Q = take(Bz * nz * kz * 4);
  L.P = take(Bz * mz * kz * 4);
  L.R = take(Bz * nz * kz * 4);
  L.X = with_ns ? take(Bz * mz * nz * 2) : 0;
  L.scale = take(Bz * 4);
  L.norm2 = take(Bz * L.ntiles * 8);
  L.Ppart = take(Bz * L.csplit * mz * kz * 4);
  L.Ptil = take(Bz * mz * kz * 8);
  L.gram = take(Bz * L.rsplit_g * kz * kz * 8);
  L.Tm = take(Bz * kz * kz * 8);
  L.Rpart = take(Bz * L.rsplit_b * nz * kz * 8);
  L.qnorm = take(Bz * kz * 4 * 3);   // column norms of R8, then the P and R column maxima
  const FactorFrags fw = factor_frag_words(B, m, n, k);
  L.QF = take((size_t)fw.QF * 4);
  L.RF = take((size_t)fw.RF * 4);
  L.PF = take((size_t)fw.PF * 4);
  L.PA = take((size_t)fw.PA * 4);
  L.RB = take((size_t)fw.RB * 4);
  L.PB = take((size_t)fw.PB * 4);
  L.PT = take(Bz * mz * 32 * 4 * 2);   // tensor-core residual operand rows: tf32 hi, lo
  L.RT = take(Bz * nz * 32 * 4 * 2);
  if (with_ns)
    L.ns = take(ns_mode == GM_NS_GRAM ? ns_gram_ws_bytes(B, m, n) : ns_standard_ws_bytes(B, m, n));
  L.total = off;
  return L;
}

struct NsLayout {
  size_t Y, parts, scale, ns, total;
  int nparts;
};
NsLayout ns_layout(int B, int m, int n, bool gram) {
  NsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += al256(bytes); return o; };
  L.nparts = ns_prep_parts(m, n);
  L.Y = take((size_t)B * m * n * 2);
  L.parts = take((size_t)B * L.nparts * 8);
  L.scale = take((size_t)B * 4);
  L.ns = take(gram ? ns_gram_ws_bytes(B, m, n) : ns_standard_ws_bytes(B, m, n));
  L.total = off;
  return L;
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }
// NULL counts as aligned (optional arguments are checked for presence separately).
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

gm_status set_error(gm_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace gm

using namespace gm;

#define GM_CHECK_ARG(cond, ...) \
  do {                          \
    if (!(cond)) return set_error(GM_E_ARG, __VA_ARGS__); \
  } while (0)

#define GM_CUDA(call)                                                                    \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return set_error(GM_E_CUDA, "%s: %s", #call, cudaGetErrorString(e_));              \
  } while (0)

#define GM_DEVICE()                                                                      \
  do {                                                                                   \
    if (!device_ok()) return set_error(GM_E_UNSUPPORTED, "current device is not sm_100"); \
  } while (0)

extern "C" {

const char* gm_status_string(gm_status s) {
  switch (s) {
    case GM_OK: return "GM_OK";
    case GM_E_ARG: return "GM_E_ARG";
    case GM_E_CUDA: return "GM_E_CUDA";
    case GM_E_NONFINITE: return "GM_E_NONFINITE";
    case GM_E_WORKSPACE: return "GM_E_WORKSPACE";
    case GM_E_UNSUPPORTED: return "GM_E_UNSUPPORTED";
    case GM_E_TIMEOUT: return "GM_E_TIMEOUT";
  }
  return "GM_E_UNKNOWN";
}

const char* gm_last_error(void) { return g_last_error; }

int gm_version(void) { return GMUON_VERSION; }

size_t gm_workspace_bytes(int op, int B, int m, int n, int k, int ns_mode) {
  if (!shape_ok(B, m, n)) return 0;
  switch (op) {
    case GM_OP_MOMENTUM_POWERIT:
      if (k < 1 || k > kMaxK) return 0;
      return step_layout(B, m, n, k, GM_NS_STANDARD, false).total;
    case GM_OP_NEWTON_SCHULZ: return ns_layout(B, m, n, false).total;
    case GM_OP_GRAM_NS: return ns_layout(B, m, n, true).total;
    case GM_OP_GRASP_STEP:
      if (k < 1 || k > kMaxK || (ns_mode != GM_NS_STANDARD && ns_mode != GM_NS_GRAM)) return 0;
      return step_layout(B, m, n, k, ns_mode, true).total;
  }
  return 0;
}

gm_status gm_grasp_workspace_layout(int B, int m, int n, int k, int ns_mode,
                                    gm_grasp_ws_layout* out) {
  GM_CHECK_ARG(out, "out is NULL");
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(k >= 1 && k <= kMaxK, "k=%d out of [1, %d]", k, kMaxK);
  StepLayout L = step_layout(B, m, n, k, ns_mode, true);
  out->M = L.M; out->Q = L.Q; out->P = L.P; out->R = L.R; out->X = L.X;
  out->scale = L.scale; out->total = L.total;
  return GM_OK;
}

gm_status gm_ns_flops(int ns_mode, int m, int n, int T, const int* restart_after, int n_restart,
                      double* flops, int* products) {
  GM_CHECK_ARG(m >= 1 && n >= 1 && T >= 1 && T <= GM_MAX_T, "bad m/n/T");
  GM_CHECK_ARG(n_restart == 0 || restart_after, "restart_after is NULL");
  ns_schedule_flops(ns_mode, m, n, T, restart_after, n_restart, flops, products);
  return GM_OK;
}

gm_status gm_device_errors(gm_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  GM_CUDA(cudaStreamSynchronize(s));
  int32_t* w = device_error_word();
  if (!w) return set_error(GM_E_CUDA, "device error word unavailable");
  int32_t v = 0;
  GM_CUDA(cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost));
  if (v != 0) {
    const int32_t zero = 0;
    GM_CUDA(cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice));
    return set_error((gm_status)v, "a kernel reported %s", gm_status_string(v));
  }
  return GM_OK;
}

gm_status gm_test_wait_timeout(const uint16_t* X, uint16_t* D, int64_t limit_ns,
                               gm_stream_t stream) {
  GM_CHECK_ARG(X && D, "NULL buffer");
  GM_CHECK_ARG(al16(X) && al16(D), "device arrays must be 16-byte aligned");
  GM_CHECK_ARG(limit_ns >= 1000000 && limit_ns <= 1000000000, "limit_ns out of [1 ms, 1 s]");
  GM_DEVICE();
  GM_CUDA(run_wait_timeout_probe(X, D, (uint64_t)limit_ns, reinterpret_cast<cudaStream_t>(stream)));
  return GM_OK;
}

gm_status gm_dequant_rebuild(int B, int m, int n, int k, const uint8_t* codes4,
                             const float* rscale, const float* cscale, const int8_t* P8,
                             const float* Pscale, const int8_t* R8, const float* Rscale,
                             float* M_out, gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(k >= 0 && k <= kMaxK, "k=%d out of [0, %d]", k, kMaxK);
  GM_CHECK_ARG(codes4 && rscale && cscale && M_out, "NULL state or output pointer");
  GM_CHECK_ARG(k == 0 || (P8 && Pscale && R8 && Rscale), "k > 0 needs P8, Pscale, R8, Rscale");
  GM_CHECK_ARG(al16(codes4) && al16(rscale) && al16(cscale) && al16(P8) && al16(Pscale) &&
                   al16(R8) && al16(Rscale) && al16(M_out),
               "device arrays must be 16-byte aligned");
  GM_DEVICE();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  GM_CUDA(launch_rebuild(B, m, n, k, codes4, rscale, cscale, P8, Pscale, R8, Rscale, nullptr, 1.0f,
                         nullptr, GM_F32, nullptr, nullptr, nullptr, nullptr, M_out, nullptr, nullptr,
                         nullptr, s));
  return GM_OK;
}

gm_status gm_momentum_powerit(int B, int m, int n, int k, float mu, const float* M_prev,
                              const void* G, gm_dtype gdt, const float* R_prev, uint64_t seed,
                              float* M_out, float* P_out, float* R_out, void* ws, size_t ws_bytes,
                              gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(k >= 1 && k <= kMaxK, "k=%d out of [1, %d]", k, kMaxK);
  GM_CHECK_ARG(G && M_out && P_out && R_out, "NULL G or output pointer");
  GM_CHECK_ARG(gdt == GM_F32 || gdt == GM_BF16 || gdt == GM_F16, "bad gdt %d", (int)gdt);
  GM_CHECK_ARG(al16(M_prev) && al16(G) && al16(R_prev) && al16(M_out) && al16(P_out) && al16(R_out),
               "device arrays must be 16-byte aligned");
  StepLayout L = step_layout(B, m, n, k, GM_NS_STANDARD, false);
  if (!ws || ws_bytes < L.total || !aligned256(ws))
    return set_error(GM_E_WORKSPACE, "workspace needs %zu bytes, 256-aligned", L.total);
  GM_DEVICE();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* Q = reinterpret_cast<float*>(w + L.Q);
  double* norm2 = reinterpret_cast<double*>(w + L.norm2);
  float* Ppart = reinterpret_cast<float*>(w + L.Ppart);
  double* Ptil = reinterpret_cast<double*>(w + L.Ptil);
  double* gram = reinterpret_cast<double*>(w + L.gram);
  double* Tm = reinterpret_cast<double*>(w + L.Tm);
  double* Rpart = reinterpret_cast<double*>(w + L.Rpart);
  float* scale = reinterpret_cast<float*>(w + L.scale);
  uint32_t* QF = reinterpret_cast<uint32_t*>(w + L.QF);
  uint32_t* PB = reinterpret_cast<uint32_t*>(w + L.PB);
  GM_CUDA(launch_warm_start(B, m, n, k, nullptr, nullptr, nullptr, nullptr, R_prev, seed, nullptr, Q,
                            nullptr, QF, nullptr, nullptr, nullptr, s));
  GM_CUDA(launch_rebuild(B, m, n, k, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                         M_prev, mu, G, gdt, Q, QF, nullptr, nullptr, M_out, norm2, Ppart, nullptr, s));
  GM_CUDA(launch_orth(B, m, k, L.csplit, Ppart, Ptil, gram, Tm, norm2, L.ntiles, 1e-7f, scale,
                      P_out, PB, nullptr, nullptr, nullptr, nullptr, s));
  GM_CUDA(launch_backproject(B, m, n, k, M_out, PB, nullptr, nullptr, false, Rpart, R_out, nullptr,
                             nullptr, nullptr, nullptr, s));
  return GM_OK;
}

gm_status gm_grid_quant4(int B, int m, int n, int block, int k, const float* X, const float* P,
                         const float* R, uint8_t* codes4, float* rscale, float* cscale,
                         gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(block == kGrid, "block=%d: only %d x %d grid blocks are built", block, kGrid, kGrid);
  GM_CHECK_ARG(X && codes4 && rscale && cscale, "NULL input or output pointer");
  GM_CHECK_ARG((P == nullptr) == (R == nullptr), "P and R must both be NULL or both set");
  GM_CHECK_ARG(!P || (k >= 1 && k <= kMaxK), "k=%d out of [1, %d]", k, kMaxK);
  GM_CHECK_ARG(al16(X) && al16(P) && al16(R) && al16(codes4) && al16(rscale) && al16(cscale),
               "device arrays must be 16-byte aligned");
  GM_DEVICE();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  GM_CUDA(launch_residual_quant4(B, m, n, P ? k : 0, X, P, R, nullptr, nullptr, codes4, rscale,
                                 cscale, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                 nullptr, s));
  return GM_OK;
}

gm_status gm_quant8(int B, int rows, int k, const float* X, int8_t* codes, float* colscale,
                    gm_stream_t stream) {
  GM_CHECK_ARG(B >= 1 && B <= 65535 && rows >= 1 && rows <= (1 << 20), "bad B=%d rows=%d", B, rows);
  GM_CHECK_ARG(k >= 1 && k <= kMaxK, "k=%d out of [1, %d]", k, kMaxK);
  GM_CHECK_ARG(X && codes && colscale, "NULL pointer");
  GM_CHECK_ARG(al16(X) && al16(codes) && al16(colscale), "device arrays must be 16-byte aligned");
  GM_DEVICE();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  GM_CUDA(launch_quant8(B, rows, 0, k, X, codes, colscale, nullptr, nullptr, nullptr, nullptr,
                        nullptr, s));
  return GM_OK;
}

gm_status gm_group_quant4(int B, int m, int n, const float* X, uint8_t* codes4, float* gscale,
                          gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(X && codes4 && gscale, "NULL pointer");
  GM_CHECK_ARG(al16(X) && al16(codes4) && al16(gscale), "device arrays must be 16-byte aligned");
  GM_DEVICE();
  GM_CUDA(launch_group_quant4(B, m, n, X, codes4, gscale, reinterpret_cast<cudaStream_t>(stream)));
  return GM_OK;
}

gm_status gm_group_dequant4(int B, int m, int n, const uint8_t* codes4, const float* gscale,
                            float* X_out, gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(codes4 && gscale && X_out, "NULL pointer");
  GM_CHECK_ARG(al16(codes4) && al16(gscale) && al16(X_out), "device arrays must be 16-byte aligned");
  GM_DEVICE();
  GM_CUDA(launch_group_dequant4(B, m, n, codes4, gscale, X_out,
                                reinterpret_cast<cudaStream_t>(stream)));
  return GM_OK;
}

gm_status gm_mulaw_quant4(int B, int m, int n, float mu, const float* X, uint8_t* codes4,
                          float* gscale, gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(mu > 0.f && mu <= 1e6f, "mu=%g out of (0, 1e6]", (double)mu);
  GM_CHECK_ARG(X && codes4 && gscale, "NULL pointer");
  GM_CHECK_ARG(al16(X) && al16(codes4) && al16(gscale), "device arrays must be 16-byte aligned");
  GM_DEVICE();
  GM_CUDA(launch_mulaw_quant4(B, m, n, mu, X, codes4, gscale, reinterpret_cast<cudaStream_t>(stream)));
  return GM_OK;
}

gm_status gm_mulaw_dequant4(int B, int m, int n, float mu, const uint8_t* codes4,
                            const float* gscale, float* X_out, gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(mu > 0.f && mu <= 1e6f, "mu=%g out of (0, 1e6]", (double)mu);
  GM_CHECK_ARG(codes4 && gscale && X_out, "NULL pointer");
  GM_CHECK_ARG(al16(codes4) && al16(gscale) && al16(X_out), "device arrays must be 16-byte aligned");
  GM_DEVICE();
  GM_CUDA(launch_mulaw_dequant4(B, m, n, mu, codes4, gscale, X_out,
                                reinterpret_cast<cudaStream_t>(stream)));
  return GM_OK;
}

static gm_status ns_common(int B, int m, int n, const void* X, gm_dtype xdt, const float* abc,
                           int T, const int* restart_after, int n_restart, float eps, void* O,
                           gm_dtype odt, void* ws, size_t ws_bytes, gm_stream_t stream, bool gram,
                           uint16_t* Rtrace = nullptr, uint16_t* Qtrace = nullptr) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(X && O, "NULL X or O");
  GM_CHECK_ARG(al16(X) && al16(O), "device arrays must be 16-byte aligned");
  GM_CHECK_ARG(xdt == GM_F32 || xdt == GM_BF16 || xdt == GM_F16, "bad xdt");
  GM_CHECK_ARG(odt == GM_F32 || odt == GM_BF16 || odt == GM_F16, "bad odt");
  GM_CHECK_ARG(T >= 1 && T <= GM_MAX_T, "T=%d out of [1, %d]", T, GM_MAX_T);
  GM_CHECK_ARG(eps >= 0.f, "eps < 0");
  GM_CHECK_ARG(n_restart >= 0 && (n_restart == 0 || restart_after), "bad restart list");
  NsLayout L = ns_layout(B, m, n, gram);
  if (!ws || ws_bytes < L.total || !aligned256(ws))
    return set_error(GM_E_WORKSPACE, "workspace needs %zu bytes, 256-aligned", L.total);
  GM_DEVICE();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float tab[3 * GM_MAX_T];
  expand_abc(abc, T, tab);
  uint16_t* Y = reinterpret_cast<uint16_t*>(w + L.Y);
  GM_CUDA(launch_ns_prep(B, m, n, X, xdt, eps, reinterpret_cast<double*>(w + L.parts), L.nparts,
                         reinterpret_cast<float*>(w + L.scale), Y, gram, s));
  NsOutput out{0, O, (int)odt, nullptr, 0.f, 0.f};
  if (gram)
    GM_CUDA(run_ns_gram(B, m, n, Y, tab, T, restart_after, n_restart, out, w + L.ns, nullptr,
                        nullptr, s, Rtrace, Qtrace));
  else
    GM_CUDA(run_ns_standard(B, m, n, Y, tab, T, out, w + L.ns, nullptr, nullptr, s));
  return GM_OK;
}

gm_status gm_newton_schulz(int B, int m, int n, const void* X, gm_dtype xdt, const float* abc,
                           int T, float eps, void* O, gm_dtype odt, void* ws, size_t ws_bytes,
                           gm_stream_t stream) {
  return ns_common(B, m, n, X, xdt, abc, T, nullptr, 0, eps, O, odt, ws, ws_bytes, stream, false);
}

gm_status gm_gram_ns(int B, int m, int n, const void* X, gm_dtype xdt, const float* abc, int T,
                     const int* restart_after, int n_restart, float eps, void* O, gm_dtype odt,
                     void* ws, size_t ws_bytes, gm_stream_t stream) {
  return ns_common(B, m, n, X, xdt, abc, T, restart_after, n_restart, eps, O, odt, ws, ws_bytes,
                   stream, true);
}

gm_status gm_gram_ns_trace(int B, int m, int n, const void* X, gm_dtype xdt, const float* abc,
                           int T, const int* restart_after, int n_restart, float eps, void* O,
                           gm_dtype odt, uint16_t* Rtrace, uint16_t* Qtrace, void* ws,
                           size_t ws_bytes, gm_stream_t stream) {
  GM_CHECK_ARG(Rtrace && Qtrace, "NULL trace buffer");
  GM_CHECK_ARG(al16(Rtrace) && al16(Qtrace), "trace buffers must be 16-byte aligned");
  return ns_common(B, m, n, X, xdt, abc, T, restart_after, n_restart, eps, O, odt, ws, ws_bytes,
                   stream, true, Rtrace, Qtrace);
}

// Argument checks shared by the step and its two halves (W, G: NULL where the
// half does not take them).
static gm_status step_checks(int B, int m, int n, const gm_grasp_params* prm, const gm_grasp_state* st,
                             const float* W, bool need_w, const void* G, bool need_g, gm_dtype gdt,
                             void* ws, size_t ws_bytes, StepLayout* L) {
  GM_CHECK_ARG(prm && st, "NULL params or state");
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  const int k = prm->k;
  GM_CHECK_ARG(k >= 1 && k <= kMaxK, "k=%d out of [1, %d]", k, kMaxK);
  GM_CHECK_ARG(prm->T >= 1 && prm->T <= GM_MAX_T, "T=%d out of [1, %d]", prm->T, GM_MAX_T);
  GM_CHECK_ARG(prm->ns == GM_NS_STANDARD || prm->ns == GM_NS_GRAM, "bad ns mode");
  GM_CHECK_ARG(prm->n_restart >= 0 && (prm->n_restart == 0 || prm->restart_after),
               "bad restart list");
  GM_CHECK_ARG(prm->eps >= 0.f, "eps < 0");
  GM_CHECK_ARG(prm->power_steps >= 0 && prm->power_steps <= 3, "power_steps=%d out of [0, 3]",
               prm->power_steps);
  GM_CHECK_ARG(prm->residual_from_codes == 0 || prm->residual_from_codes == 1,
               "residual_from_codes must be 0 or 1");
  GM_CHECK_ARG(al16(prm->matrix_ids), "matrix_ids must be 16-byte aligned");
  GM_CHECK_ARG(prm->block == 0 || prm->block == kGrid, "block=%d: only %d x %d grid blocks are built",
               prm->block, kGrid, kGrid);
  GM_CHECK_ARG(st->codes4 && st->rscale && st->cscale && st->P8 && st->Pscale && st->R8 &&
                   st->Rscale && st->step && st->dev_status,
               "NULL state pointer");
  GM_CHECK_ARG(!need_w || W, "NULL W");
  GM_CHECK_ARG(!need_g || G, "NULL G");
  GM_CHECK_ARG(al16(W) && al16(G) && al16(st->codes4) && al16(st->rscale) && al16(st->cscale) &&
                   al16(st->P8) && al16(st->Pscale) && al16(st->R8) && al16(st->Rscale),
               "device arrays must be 16-byte aligned");
  GM_CHECK_ARG(!need_g || gdt == GM_F32 || gdt == GM_BF16 || gdt == GM_F16, "bad gdt");
  *L = step_layout(B, m, n, k, prm->ns, true);
  if (!ws || ws_bytes < L->total || !aligned256(ws))
    return set_error(GM_E_WORKSPACE, "workspace needs %zu bytes, 256-aligned", L->total);
  GM_DEVICE();
  return GM_OK;
}

gm_status gm_grasp_state_update(int B, int m, int n, const gm_grasp_params* prm,
                                const gm_grasp_state* st, const void* G, gm_dtype gdt, void* ws,
                                size_t ws_bytes, gm_stream_t stream) {
  StepLayout L;
  const gm_status chk = step_checks(B, m, n, prm, st, nullptr, false, G, true, gdt, ws, ws_bytes, &L);
  if (chk != GM_OK) return chk;
  const int k = prm->k;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* M = reinterpret_cast<float*>(w + L.M);
  float* Q = reinterpret_cast<float*>(w + L.Q);
  float* P = reinterpret_cast<float*>(w + L.P);
  float* R = reinterpret_cast<float*>(w + L.R);
  uint16_t* X = reinterpret_cast<uint16_t*>(w + L.X);
  float* scale = reinterpret_cast<float*>(w + L.scale);
  double* norm2 = reinterpret_cast<double*>(w + L.norm2);
  float* Ppart = reinterpret_cast<float*>(w + L.Ppart);
  double* Ptil = reinterpret_cast<double*>(w + L.Ptil);
  double* gram = reinterpret_cast<double*>(w + L.gram);
  double* Tm = reinterpret_cast<double*>(w + L.Tm);
  double* Rpart = reinterpret_cast<double*>(w + L.Rpart);
  uint32_t* QF = reinterpret_cast<uint32_t*>(w + L.QF);
  uint32_t* RF = reinterpret_cast<uint32_t*>(w + L.RF);
  uint32_t* PF = reinterpret_cast<uint32_t*>(w + L.PF);
  uint32_t* PA = reinterpret_cast<uint32_t*>(w + L.PA);
  uint32_t* RB = reinterpret_cast<uint32_t*>(w + L.RB);
  uint32_t* PB = reinterpret_cast<uint32_t*>(w + L.PB);
  float* PT = reinterpret_cast<float*>(w + L.PT);
  float* RT = reinterpret_cast<float*>(w + L.RT);
  int32_t* status = st->dev_status;
  const bool gramns = prm->ns == GM_NS_GRAM;
  const int psteps = prm->power_steps < 1 ? 1 : prm->power_steps;
  unsigned* PRmax = reinterpret_cast<unsigned*>(w + L.qnorm) + (size_t)B * k;

  GM_CUDA(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
  // worked step 2: warm start from the stored R (read before it is overwritten)
  // (with the fragment copies of Q, R and P that the rebuild reads)
  GM_CUDA(launch_warm_start(B, m, n, k, st->R8, st->Rscale, st->P8, st->Pscale, nullptr, prm->seed,
                            prm->matrix_ids, Q, reinterpret_cast<int*>(w + L.qnorm), QF, RF, PF,
                            status, s));
  // worked steps 1 and 3: rebuild M_{t-1}, M_t = mu M_{t-1} + G
  // (with the projection P~ = M Q of worked step 4 fused in)
  GM_CUDA(launch_rebuild(B, m, n, k, st->codes4, st->rscale, st->cscale, st->P8, st->Pscale,
                         st->R8, st->Rscale, nullptr, prm->mu, G, gdt, Q, QF, RF, PF, M, norm2, Ppart,
                         status, s));
  // worked step 4: P = orth(P~), R = M^T P (and the normalised NS input X)
  GM_CUDA(launch_orth(B, m, k, L.csplit, Ppart, Ptil, gram, Tm, norm2, L.ntiles, prm->eps, scale,
                      P, PB, PA, PT, PRmax, status, s));
  GM_CUDA(launch_backproject(B, m, n, k, M, PB, scale, X, gramns, Rpart, R, RB, RT,
                             PRmax + (size_t)B * k, status, s));
  // further power-iteration steps: Q = column-normalised R, P~ = M Q (a projection
  // pass over the stored M_t), P = orth(P~), R = M^T P
  for (int it = 1; it < psteps; ++it) {
    GM_CUDA(launch_warm_start(B, m, n, k, nullptr, nullptr, nullptr, nullptr, R, prm->seed,
                              prm->matrix_ids, Q, nullptr, QF, nullptr, nullptr, status, s));
    GM_CUDA(launch_rebuild(B, m, n, k, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                           nullptr, M, 1.0f, nullptr, GM_F32, Q, QF, nullptr, nullptr, nullptr,
                           nullptr, Ppart, status, s));
    GM_CUDA(cudaMemsetAsync(PRmax, 0, sizeof(unsigned) * 2 * (size_t)B * k, s));
    GM_CUDA(launch_orth(B, m, k, L.csplit, Ppart, Ptil, gram, Tm, norm2, L.ntiles, prm->eps, scale,
                        P, PB, PA, PT, PRmax, status, s));
    GM_CUDA(launch_backproject(B, m, n, k, M, PB, nullptr, nullptr, gramns, Rpart, R, RB, RT,
                               PRmax + (size_t)B * k, status, s));
  }
  // worked step 5 variant: the residual from the dequantized 8-bit factors
  if (prm->residual_from_codes)
    GM_CUDA(launch_codes_frags(B, m, n, k, P, R, PRmax, PRmax + (size_t)B * k, PA, RB, PT, RT, status,
                               s));
  // worked step 5: residual -> 4-bit grid codes (tensor cores); P, R -> 8-bit codes
  // (state in place)
  GM_CUDA(launch_residual_ws(B, m, n, k, M, P, R, PT, RT, st->codes4, st->rscale, st->cscale, PRmax,
                             st->P8, st->Pscale, st->R8, st->Rscale, st->step, status, status, s));
  return GM_OK;
}

gm_status gm_grasp_apply(int B, int m, int n, const gm_grasp_params* prm, const gm_grasp_state* st,
                         float* W, void* ws, size_t ws_bytes, gm_stream_t stream) {
  StepLayout L;
  const gm_status chk = step_checks(B, m, n, prm, st, W, true, nullptr, false, GM_F32, ws, ws_bytes, &L);
  if (chk != GM_OK) return chk;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* X = reinterpret_cast<uint16_t*>(w + L.X);
  int32_t* status = st->dev_status;
  float tab[3 * GM_MAX_T];
  expand_abc(prm->abc, prm->T, tab);
  // worked step 6: O = NS(M_t); W <- W - eta (O + wd W) in the last product's epilogue
  NsOutput out{1, nullptr, 0, W, prm->eta, prm->wd};
  if (prm->ns == GM_NS_GRAM)
    GM_CUDA(run_ns_gram(B, m, n, X, tab, prm->T, prm->restart_after, prm->n_restart, out,
                        w + L.ns, status, status, s));
  else
    GM_CUDA(run_ns_standard(B, m, n, X, tab, prm->T, out, w + L.ns, status, status, s));
  return GM_OK;
}

gm_status gm_grasp_orth(int B, int m, int n, const gm_grasp_params* prm, const gm_grasp_state* st,
                        void* O, gm_dtype odt, void* ws, size_t ws_bytes, gm_stream_t stream) {
  GM_CHECK_ARG(odt == GM_F32 || odt == GM_BF16 || odt == GM_F16, "bad odt");
  GM_CHECK_ARG(O, "NULL O");
  GM_CHECK_ARG(al16(O), "device arrays must be 16-byte aligned");
  StepLayout L;
  const gm_status chk =
      step_checks(B, m, n, prm, st, nullptr, false, nullptr, false, GM_F32, ws, ws_bytes, &L);
  if (chk != GM_OK) return chk;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* X = reinterpret_cast<uint16_t*>(w + L.X);
  int32_t* status = st->dev_status;
  float tab[3 * GM_MAX_T];
  expand_abc(prm->abc, prm->T, tab);
  // worked step 6 up to O = NS(M_t)
  NsOutput out{0, O, (int)odt, nullptr, 0.f, 0.f};
  if (prm->ns == GM_NS_GRAM)
    GM_CUDA(run_ns_gram(B, m, n, X, tab, prm->T, prm->restart_after, prm->n_restart, out,
                        w + L.ns, status, status, s));
  else
    GM_CUDA(run_ns_standard(B, m, n, X, tab, prm->T, out, w + L.ns, status, status, s));
  return GM_OK;
}

gm_status gm_grasp_orth_peers(int B, int m, int n, const gm_grasp_params* prm,
                              const gm_grasp_state* st, void* const* peer_O,
                              int32_t* const* peer_flags, int npeers, const int64_t* dst_index,
                              gm_dtype odt, void* ws, size_t ws_bytes, gm_stream_t stream) {
  GM_CHECK_ARG(odt == GM_F32 || odt == GM_BF16 || odt == GM_F16, "bad odt");
  GM_CHECK_ARG(npeers >= 1 && npeers <= kMaxPeers, "npeers=%d out of [1, %d]", npeers, kMaxPeers);
  GM_CHECK_ARG(peer_O && peer_flags, "NULL peer arrays");
  for (int r = 0; r < npeers; ++r) {
    GM_CHECK_ARG(peer_O[r] && peer_flags[r], "NULL receive buffer of peer %d", r);
    GM_CHECK_ARG(al16(peer_O[r]) && al16(peer_flags[r]), "device arrays must be 16-byte aligned");
  }
  GM_CHECK_ARG(al16(dst_index), "device arrays must be 16-byte aligned");
  StepLayout L;
  const gm_status chk =
      step_checks(B, m, n, prm, st, nullptr, false, nullptr, false, GM_F32, ws, ws_bytes, &L);
  if (chk != GM_OK) return chk;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* X = reinterpret_cast<uint16_t*>(w + L.X);
  int32_t* status = st->dev_status;
  float tab[3 * GM_MAX_T];
  expand_abc(prm->abc, prm->T, tab);
  // worked step 6 up to O = NS(M_t), stored straight into every receive buffer
  NsOutput out{0, nullptr, (int)odt, nullptr, 0.f, 0.f};
  out.npeers = npeers;
  for (int r = 0; r < npeers; ++r) out.peer[r] = peer_O[r];
  out.dst_index = dst_index;
  if (prm->ns == GM_NS_GRAM)
    GM_CUDA(run_ns_gram(B, m, n, X, tab, prm->T, prm->restart_after, prm->n_restart, out,
                        w + L.ns, status, status, s));
  else
    GM_CUDA(run_ns_standard(B, m, n, X, tab, prm->T, out, w + L.ns, status, status, s));
  GM_CUDA(launch_put_status(B, npeers, peer_flags, dst_index, status, s));
  return GM_OK;
}

static_assert(sizeof(gm_ipc_handle) >= sizeof(cudaIpcMemHandle_t), "IPC handle size");

gm_status gm_ipc_export(const void* dev_ptr, gm_ipc_handle* handle, size_t* offset) {
  GM_CHECK_ARG(dev_ptr && handle && offset, "NULL argument");
  using AddrRange = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
  static std::atomic<AddrRange> fn{nullptr};
  AddrRange f = fn.load(std::memory_order_acquire);
  if (!f) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return set_error(GM_E_UNSUPPORTED, "cuMemGetAddressRange is not available");
    f = reinterpret_cast<AddrRange>(p);
    fn.store(f, std::memory_order_release);
  }
  CUdeviceptr base = 0;
  size_t size = 0;
  if (f(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return set_error(GM_E_ARG, "not a device allocation");
  cudaIpcMemHandle_t h;
  GM_CUDA(cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)));
  memset(handle, 0, sizeof(*handle));
  memcpy(handle->bytes, &h, sizeof(h));
  *offset = (size_t)(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return GM_OK;
}

gm_status gm_ipc_open(const gm_ipc_handle* handle, void** base) {
  GM_CHECK_ARG(handle && base, "NULL argument");
  cudaIpcMemHandle_t h;
  memcpy(&h, handle->bytes, sizeof(h));
  GM_CUDA(cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess));
  return GM_OK;
}

gm_status gm_ipc_close(void* base) {
  GM_CHECK_ARG(base, "NULL argument");
  GM_CUDA(cudaIpcCloseMemHandle(base));
  return GM_OK;
}

gm_status gm_weight_update(int B, int m, int n, float eta, float wd, const void* O, gm_dtype odt,
                           float* W, const int32_t* skip, int skip_stride, gm_stream_t stream) {
  GM_CHECK_ARG(shape_ok(B, m, n), "bad shape B=%d m=%d n=%d", B, m, n);
  GM_CHECK_ARG(O && W, "NULL O or W");
  GM_CHECK_ARG(odt == GM_F32 || odt == GM_BF16 || odt == GM_F16, "bad odt");
  GM_CHECK_ARG(al16(O) && al16(W) && al16(skip), "device arrays must be 16-byte aligned");
  GM_CHECK_ARG(skip_stride == 0 || skip_stride == 1, "skip_stride must be 0 or 1");
  GM_CHECK_ARG(std::isfinite(eta) && std::isfinite(wd), "eta and wd must be finite");
  GM_DEVICE();
  GM_CUDA(launch_weight_update(B, m, n, eta, wd, O, (int)odt, W, skip, skip_stride,
                               reinterpret_cast<cudaStream_t>(stream)));
  return GM_OK;
}

gm_status gm_grasp_step(int B, int m, int n, const gm_grasp_params* prm, const gm_grasp_state* st,
                        float* W, const void* G, gm_dtype gdt, void* ws, size_t ws_bytes,
                        gm_stream_t stream) {
  StepLayout L;
  const gm_status chk = step_checks(B, m, n, prm, st, W, true, G, true, gdt, ws, ws_bytes, &L);
  if (chk != GM_OK) return chk;
  const gm_status a = gm_grasp_state_update(B, m, n, prm, st, G, gdt, ws, ws_bytes, stream);
  if (a != GM_OK) return a;
  return gm_grasp_apply(B, m, n, prm, st, W, ws, ws_bytes, stream);
}

}  // extern "C"
