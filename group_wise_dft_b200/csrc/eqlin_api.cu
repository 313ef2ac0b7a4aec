// Host side of the C ABI: argument validation, transform tables, buffer
// layouts and kernel selection.  Every check happens here, before a launch.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "eqlin_internal.cuh"

namespace eqlin {

static thread_local char g_msg[512] = "";

void clear_error() { g_msg[0] = 0; }

int set_error(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return code;
}

int check_launch(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(EQLIN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return EQLIN_OK;
}

void unit_root(int j, int N, double *c, double *s) {
  j %= N;
  if (j < 0) j += N;
  if ((4 * j) % N == 0) {   // a whole number of quarter turns: exactly 0 and +-1
    static const double cq[4] = {1.0, 0.0, -1.0, 0.0}, sq[4] = {0.0, 1.0, 0.0, -1.0};
    const int q = 4 * j / N;
    *c = cq[q];
    *s = sq[q];
    return;
  }
  const double a = 2.0 * M_PI * (double)j / (double)N;
  *c = cos(a);
  *s = sin(a);
}

// Half-spectrum real-coordinate transforms (see DftTables).  Twiddles come
// from unit_root (double, exact at quarter turns), rounded once to fp32: for
// N = 4 (p4) every entry is 0, +-1 or +-2, as the Flash EQ-Linear page's
// "Specialization for p4" has it, so these transforms are exact.
void make_dft_tables(int N, DftTables *t) {
  memset(t, 0, sizeof *t);
  for (int h = 0; h < N; ++h) {
    t->fwd[0][h] = 1.0f;
    for (int k = 1; 2 * k < N; ++k) {
      double c, s;
      unit_root(k * h, N, &c, &s);
      t->fwd[2 * k - 1][h] = (float)c;
      t->fwd[2 * k][h] = (float)(-s);
    }
    if (N % 2 == 0 && N > 1) t->fwd[N - 1][h] = (h % 2) ? -1.0f : 1.0f;
  }
  for (int g = 0; g < N; ++g) {
    t->inv[g][0] = 1.0f;
    for (int k = 1; 2 * k < N; ++k) {
      double c, s;
      unit_root(k * g, N, &c, &s);
      t->inv[g][2 * k - 1] = (float)(2.0 * c);
      t->inv[g][2 * k] = (float)(-2.0 * s);
    }
    if (N % 2 == 0 && N > 1) t->inv[g][N - 1] = (g % 2) ? -1.0f : 1.0f;
  }
}

// D8 = <r, s | r^4 = s^2 = 1, s r s = r^-1>; slot j <-> r^j, slot 4+j <-> r^j s.
// Q rows: the four 1-D characters / sqrt 8, then rho_E(g)[a][b] / 2 for
// (a,b) = 00, 01, 10, 11 with rho_E(r) = [[0,-1],[1,0]], rho_E(s) = diag(1,-1).
void make_d8_tables(D8Tables *t) {
  const double inv_sqrt8 = 1.0 / sqrt(8.0);
  for (int slot = 0; slot < 8; ++slot) {
    const int j = slot & 3, f = slot >> 2;
    const double chi[4] = {1.0, f ? -1.0 : 1.0, (j & 1) ? -1.0 : 1.0,
                           ((j + f) & 1) ? -1.0 : 1.0};
    for (int c = 0; c < 4; ++c) t->q[c][slot] = (float)(chi[c] * inv_sqrt8);
    // rho_E(r^j) is rotation by j quarter turns; rho_E(s) flips the sign of column 1.
    int R[2][2] = {{1, 0}, {0, 1}};
    for (int n = 0; n < j; ++n) {
      const int a00 = -R[1][0], a01 = -R[1][1], a10 = R[0][0], a11 = R[0][1];
      R[0][0] = a00; R[0][1] = a01; R[1][0] = a10; R[1][1] = a11;
    }
    if (f) { R[0][1] = -R[0][1]; R[1][1] = -R[1][1]; }
    for (int a = 0; a < 2; ++a)
      for (int b = 0; b < 2; ++b) t->q[4 + 2 * a + b][slot] = (float)(0.5 * R[a][b]);
  }
}

static size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

CyclicSpecLayout cyclic_spec_layout(int N, int Cin, int Cout, int dtype) {
  CyclicSpecLayout L{};
  L.simt_offset = 0;
  L.simt_bytes = (size_t)Cin * N * Cout * sizeof(float);
  L.tc_offset = round_up(L.simt_bytes, 256);
  L.tc_bytes = cyclic_tc_supported(N, Cin, Cout, dtype) || cyclic_tc_f16_supported(N, Cin, Cout, dtype)
                   ? cyclic_tc_bytes(N, Cin, Cout)
               : cyclic4_tc_supported(N, Cin, Cout, dtype) ? cyclic4_tc_bytes(Cin, Cout)
               : cyclic_tc_f32_supported(N, Cin, Cout, dtype) ? cyclic_tc_f32_bytes(Cin, Cout)
                   : (N == 16 && cyclic16_tc_supported(Cin, Cout, dtype) ? cyclic16_tc_bytes(Cin, Cout) : 0);
  L.total = L.tc_offset + L.tc_bytes;
  return L;
}

D8PackLayout d8_pack_layout(int C, int dtype) {
  D8PackLayout L{};
  const size_t F = (size_t)C / 8;
  L.simt_offset = 0;
  L.simt_bytes = 8 * F * F * sizeof(float);
  L.tc_offset = round_up(L.simt_bytes, 256);
  L.tc_bytes = d8_tc_supported(C, dtype) ? d8_tc_bytes(C) : 0;
  L.total = L.tc_offset + L.tc_bytes;
  return L;
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
// The tensor-core path writes y in 32-byte pieces; AUTO falls back otherwise.
static bool aligned32(const void *p) { return ((uintptr_t)p & 31u) == 0; }

int check_cyclic_shape(int N, int Cin, int Cout, int dtype) {
  if (dtype != EQLIN_F32 && dtype != EQLIN_BF16 && dtype != EQLIN_F16)
    return set_error(EQLIN_ERR_UNSUPPORTED, "dtype %d is not EQLIN_F32, EQLIN_BF16 or EQLIN_F16", dtype);
  if (N < 1 || N > kMaxN) return set_error(EQLIN_ERR_UNSUPPORTED, "N=%d not in 1..16", N);
  if (Cin < 1 || Cout < 1)
    return set_error(EQLIN_ERR_INVALID_ARG, "Cin=%d, Cout=%d must be >= 1", Cin, Cout);
  if ((int64_t)Cin * N > (1 << 24) || (int64_t)Cout * N > (1 << 24))
    return set_error(EQLIN_ERR_UNSUPPORTED, "channel count too large");
  return EQLIN_OK;
}

static int check_d8_shape(int C, int dtype) {
  if (dtype != EQLIN_F32 && dtype != EQLIN_BF16 && dtype != EQLIN_F16)
    return set_error(EQLIN_ERR_UNSUPPORTED, "dtype %d is not EQLIN_F32, EQLIN_BF16 or EQLIN_F16", dtype);
  if (C < 8 || C % 8) return set_error(EQLIN_ERR_UNSUPPORTED, "C=%d must be a positive multiple of 8", C);
  if (C > (1 << 20)) return set_error(EQLIN_ERR_UNSUPPORTED, "C=%d too large", C);
  return EQLIN_OK;
}

}  // namespace eqlin

using namespace eqlin;

extern "C" {

const char *eqlin_last_error(void) { return g_msg; }

int eqlin_version(void) { return 102; }

int eqlin_device_fault(int reset) { return read_device_fault(reset); }

int eqlin_selftest_wait_timeout(uint64_t limit_ns, int arrive, void *elapsed_ns, eqlin_stream_t stream) {
  g_msg[0] = 0;
  if (limit_ns < 1000ull || limit_ns > 10000000000ull)
    return set_error(EQLIN_ERR_INVALID_ARG, "limit_ns=%llu not in 1000..1e10", (unsigned long long)limit_ns);
  if (arrive != 0 && arrive != 1) return set_error(EQLIN_ERR_INVALID_ARG, "arrive must be 0 or 1");
  if (elapsed_ns && ((uintptr_t)elapsed_ns & 7u))
    return set_error(EQLIN_ERR_ALIGN, "elapsed_ns must be 8-byte aligned");
  return launch_bounded_wait_selftest(limit_ns, arrive, static_cast<unsigned long long *>(elapsed_ns),
                                      (cudaStream_t)stream);
}

size_t eqlin_cyclic_spectrum_bytes(int N, int Cin, int Cout, int dtype) {
  if (check_cyclic_shape(N, Cin, Cout, dtype) != EQLIN_OK) return 0;
  return cyclic_spec_layout(N, Cin, Cout, dtype).total;
}

int eqlin_cyclic_weight_spectrum(const void *W, int N, int Cin, int Cout, int dtype, void *Wspec,
                                 size_t Wspec_bytes, eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_cyclic_shape(N, Cin, Cout, dtype);
  if (rc) return rc;
  if (!W || !Wspec) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(Wspec))
    return set_error(EQLIN_ERR_ALIGN, "W and Wspec must be 16-byte aligned");
  const CyclicSpecLayout L = cyclic_spec_layout(N, Cin, Cout, dtype);
  if (Wspec_bytes < L.total)
    return set_error(EQLIN_ERR_SIZE, "Wspec_bytes=%zu < required %zu", Wspec_bytes, L.total);
  return launch_cyclic_spectrum(W, N, Cin, Cout, dtype, 0, Wspec, L, (cudaStream_t)stream);
}

int eqlin_cyclic_weight_spectrum_adjoint(const void *W, int N, int Cin, int Cout, int dtype,
                                         void *Wspec, size_t Wspec_bytes, eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_cyclic_shape(N, Cin, Cout, dtype);
  if (rc) return rc;
  if (!W || !Wspec) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(Wspec))
    return set_error(EQLIN_ERR_ALIGN, "W and Wspec must be 16-byte aligned");
  // the backward data pass is the layer Cout -> Cin with weight W[i][o][(-m) mod N]
  const CyclicSpecLayout L = cyclic_spec_layout(N, Cout, Cin, dtype);
  if (Wspec_bytes < L.total)
    return set_error(EQLIN_ERR_SIZE, "Wspec_bytes=%zu < required %zu", Wspec_bytes, L.total);
  return launch_cyclic_spectrum(W, N, Cout, Cin, dtype, 1, Wspec, L, (cudaStream_t)stream);
}

int eqlin_cyclic_auto_path(int N, int Cin, int Cout, int dtype) {
  if (check_cyclic_shape(N, Cin, Cout, dtype) != EQLIN_OK) return -1;
  return cyclic_tc_supported(N, Cin, Cout, dtype) ? EQLIN_PATH_TC : EQLIN_PATH_SIMT;
}

int eqlin_cyclic_forward_ex(const void *x, const void *Wspec, void *y, int64_t T, int N, int Cin,
                            int Cout, int dtype, int path, eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_cyclic_shape(N, Cin, Cout, dtype);
  if (rc) return rc;
  if (T < 0) return set_error(EQLIN_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
  if (path != EQLIN_PATH_AUTO && path != EQLIN_PATH_SIMT && path != EQLIN_PATH_TC)
    return set_error(EQLIN_ERR_INVALID_ARG, "unknown path %d", path);
  if (T == 0) return EQLIN_OK;
  if (!x || !Wspec || !y) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(y) || !aligned16(Wspec))
    return set_error(EQLIN_ERR_ALIGN, "x, y and Wspec must be 16-byte aligned");
  const bool tc_ok = cyclic_tc_supported(N, Cin, Cout, dtype);
  // fp16 and p4 reach the tensor cores only when asked for
  const bool tc_f16 = path == EQLIN_PATH_TC && cyclic_tc_f16_supported(N, Cin, Cout, dtype);
  const bool tc_c4 = path == EQLIN_PATH_TC && cyclic4_tc_supported(N, Cin, Cout, dtype);
  if (path == EQLIN_PATH_TC && !tc_ok && !tc_f16 && !tc_c4)
    return set_error(EQLIN_ERR_UNSUPPORTED,
                     "tensor-core path needs bf16 or fp16, N=8, Cin%%16==0 (16..160), Cout%%32==0 "
                     "(or bf16, N=4, Cin%%32==0 (32..320), Cout%%32==0)");
  const CyclicSpecLayout L = cyclic_spec_layout(N, Cin, Cout, dtype);
  if (tc_c4)
    return launch_cyclic4_tc(x, static_cast<const char *>(Wspec) + L.tc_offset, y, T, Cin, Cout,
                             (cudaStream_t)stream);
  if ((tc_ok || tc_f16) && (path == EQLIN_PATH_TC || (path == EQLIN_PATH_AUTO && aligned32(y))))
    return launch_cyclic_tc(x, static_cast<const char *>(Wspec) + L.tc_offset, y, T, Cin, Cout, dtype,
                            (cudaStream_t)stream);
  return launch_cyclic_simt(x, Wspec, y, T, N, Cin, Cout, dtype, L, (cudaStream_t)stream);
}

int eqlin_cyclic_forward(const void *x, const void *Wspec, void *y, int64_t T, int N, int Cin,
                         int Cout, int dtype, eqlin_stream_t stream) {
  return eqlin_cyclic_forward_ex(x, Wspec, y, T, N, Cin, Cout, dtype, EQLIN_PATH_AUTO, stream);
}

size_t eqlin_cyclic_forward_workspace_bytes(int64_t T, int N, int Cin, int Cout, int dtype) {
  if (check_cyclic_shape(N, Cin, Cout, dtype) != EQLIN_OK || T < 0) return 0;
  if (N == 16 && cyclic16_tc_supported(Cin, Cout, dtype)) return cyclic16_tc_workspace_bytes(T, Cin, Cout);
  if (cyclic_tc_f32_supported(N, Cin, Cout, dtype)) return cyclic_tc_f32_workspace_bytes(T, Cin, Cout);
  return 0;
}

int eqlin_cyclic_forward_ws(const void *x, const void *Wspec, void *y, int64_t T, int N, int Cin,
                            int Cout, int dtype, int path, void *workspace, size_t workspace_bytes,
                            eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_cyclic_shape(N, Cin, Cout, dtype);
  if (rc) return rc;
  const bool tc16 = N == 16 && cyclic16_tc_supported(Cin, Cout, dtype);
  // fp32 on the tensor cores (split spectra) only when asked for
  const bool tcf32 = path == EQLIN_PATH_TC && cyclic_tc_f32_supported(N, Cin, Cout, dtype);
  if (!tc16 && !tcf32) return eqlin_cyclic_forward_ex(x, Wspec, y, T, N, Cin, Cout, dtype, path, stream);
  if (T < 0) return set_error(EQLIN_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
  if (path != EQLIN_PATH_AUTO && path != EQLIN_PATH_SIMT && path != EQLIN_PATH_TC)
    return set_error(EQLIN_ERR_INVALID_ARG, "unknown path %d", path);
  if (T == 0) return EQLIN_OK;
  if (!x || !Wspec || !y) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(y) || !aligned16(Wspec))
    return set_error(EQLIN_ERR_ALIGN, "x, y and Wspec must be 16-byte aligned");
  const size_t need = tc16 ? cyclic16_tc_workspace_bytes(T, Cin, Cout) : cyclic_tc_f32_workspace_bytes(T, Cin, Cout);
  const bool ws_ok = workspace && workspace_bytes >= need && ((uintptr_t)workspace & 255u) == 0;
  if (path == EQLIN_PATH_TC && !ws_ok)
    return set_error(EQLIN_ERR_SIZE, "this tensor-core path needs a 256-byte aligned workspace of %zu bytes",
                     need);
  if (path == EQLIN_PATH_SIMT || (path == EQLIN_PATH_AUTO && !ws_ok))
    return eqlin_cyclic_forward_ex(x, Wspec, y, T, N, Cin, Cout, dtype, EQLIN_PATH_SIMT, stream);
  if (!aligned32(y)) {
    if (path == EQLIN_PATH_TC) return set_error(EQLIN_ERR_ALIGN, "tensor-core path needs y 32-byte aligned");
    return eqlin_cyclic_forward_ex(x, Wspec, y, T, N, Cin, Cout, dtype, EQLIN_PATH_SIMT, stream);
  }
  const CyclicSpecLayout L = cyclic_spec_layout(N, Cin, Cout, dtype);
  if (tcf32)
    return launch_cyclic_tc_f32(x, static_cast<const char *>(Wspec) + L.tc_offset, y, T, Cin, Cout, workspace,
                                (cudaStream_t)stream);
  return launch_cyclic16_tc(x, static_cast<const char *>(Wspec) + L.tc_offset, y, T, Cin, Cout, workspace,
                            (cudaStream_t)stream);
}

int eqlin_cyclic_backward_data_ex(const void *dy, const void *Wspec_adj, void *dx, int64_t T, int N,
                                  int Cin, int Cout, int dtype, int path, eqlin_stream_t stream) {
  return eqlin_cyclic_forward_ex(dy, Wspec_adj, dx, T, N, Cout, Cin, dtype, path, stream);
}

int eqlin_cyclic_backward_data(const void *dy, const void *Wspec_adj, void *dx, int64_t T, int N,
                               int Cin, int Cout, int dtype, eqlin_stream_t stream) {
  return eqlin_cyclic_forward_ex(dy, Wspec_adj, dx, T, N, Cout, Cin, dtype, EQLIN_PATH_AUTO, stream);
}

size_t eqlin_cyclic_weight_grad_workspace_bytes(int64_t T, int N, int Cin, int Cout, int dtype) {
  if (check_cyclic_shape(N, Cin, Cout, dtype) != EQLIN_OK || T < 0) return 0;
  size_t need = cyclic_wgrad_part_bytes(cyclic_wgrad_splits(T, Cin, Cout), N, Cin, Cout);
  if (cyclic_wgrad_tc_supported(T, N, Cin, Cout, dtype)) {
    const size_t tc = cyclic_wgrad_part_bytes(cyclic_wgrad_tc_plan(T, Cin, Cout).splits, N, Cin, Cout);
    if (tc > need) need = tc;
  }
  return need;
}

int eqlin_cyclic_weight_grad_ex(const void *x, const void *dy, void *dW, int64_t T, int N, int Cin,
                                int Cout, int dtype, void *workspace, size_t workspace_bytes, int path,
                                eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_cyclic_shape(N, Cin, Cout, dtype);
  if (rc) return rc;
  if (T < 0) return set_error(EQLIN_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
  if (path != EQLIN_PATH_AUTO && path != EQLIN_PATH_SIMT && path != EQLIN_PATH_TC)
    return set_error(EQLIN_ERR_INVALID_ARG, "unknown path %d", path);
  const bool tc_ok = cyclic_wgrad_tc_supported(T, N, Cin, Cout, dtype);
  if (path == EQLIN_PATH_TC && !tc_ok)
    return set_error(EQLIN_ERR_UNSUPPORTED, "tensor-core weight gradient needs bf16 and N=8");
  if (!dW || (T > 0 && (!x || !dy))) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(dW) || (T > 0 && (!aligned16(x) || !aligned16(dy))))
    return set_error(EQLIN_ERR_ALIGN, "x, dy and dW must be 16-byte aligned");
  const size_t need = eqlin_cyclic_weight_grad_workspace_bytes(T, N, Cin, Cout, dtype);
  if (need > 0 && !workspace) return set_error(EQLIN_ERR_INVALID_ARG, "null workspace");
  if (workspace_bytes < need)
    return set_error(EQLIN_ERR_SIZE, "workspace_bytes=%zu < required %zu", workspace_bytes, need);
  if (workspace && !aligned16(workspace))
    return set_error(EQLIN_ERR_ALIGN, "workspace must be 16-byte aligned");
  float *part = static_cast<float *>(workspace);
  if (tc_ok && path != EQLIN_PATH_SIMT) {
    const WgradTcPlan plan = cyclic_wgrad_tc_plan(T, Cin, Cout);
    rc = launch_cyclic_wgrad_tc_partials(x, dy, part, T, Cin, Cout, plan, (cudaStream_t)stream);
    if (rc) return rc;
    return launch_cyclic_wgrad_finish(part, plan.splits, N, Cin, Cout, dtype, dW, (cudaStream_t)stream);
  }
  return launch_cyclic_wgrad(x, dy, dW, T, N, Cin, Cout, dtype, part, cyclic_wgrad_splits(T, Cin, Cout),
                             (cudaStream_t)stream);
}

int eqlin_cyclic_weight_grad(const void *x, const void *dy, void *dW, int64_t T, int N, int Cin,
                             int Cout, int dtype, void *workspace, size_t workspace_bytes,
                             eqlin_stream_t stream) {
  return eqlin_cyclic_weight_grad_ex(x, dy, dW, T, N, Cin, Cout, dtype, workspace, workspace_bytes,
                                     EQLIN_PATH_AUTO, stream);
}

size_t eqlin_d8_weight_bytes(int C, int dtype) {
  if (check_d8_shape(C, dtype) != EQLIN_OK) return 0;
  return d8_pack_layout(C, dtype).total;
}

int eqlin_d8_pack_weights(const void *wA1, const void *wA2, const void *wB1, const void *wB2,
                          const void *wE, int C, int dtype, void *Wpack, size_t Wpack_bytes,
                          eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_d8_shape(C, dtype);
  if (rc) return rc;
  const void *w[5] = {wA1, wA2, wB1, wB2, wE};
  for (int k = 0; k < 5; ++k) {
    if (!w[k]) return set_error(EQLIN_ERR_INVALID_ARG, "null weight pointer");
    if (!aligned16(w[k])) return set_error(EQLIN_ERR_ALIGN, "weights must be 16-byte aligned");
  }
  if (!Wpack) return set_error(EQLIN_ERR_INVALID_ARG, "null Wpack");
  if (!aligned16(Wpack)) return set_error(EQLIN_ERR_ALIGN, "Wpack must be 16-byte aligned");
  const D8PackLayout L = d8_pack_layout(C, dtype);
  if (Wpack_bytes < L.total)
    return set_error(EQLIN_ERR_SIZE, "Wpack_bytes=%zu < required %zu", Wpack_bytes, L.total);
  return launch_d8_pack(w, C, dtype, Wpack, L, (cudaStream_t)stream);
}

int eqlin_d8_auto_path(int C, int dtype) {
  if (check_d8_shape(C, dtype) != EQLIN_OK) return -1;
  return d8_tc_supported(C, dtype) ? EQLIN_PATH_TC : EQLIN_PATH_SIMT;
}

int eqlin_d8_forward_ex(const void *x, const void *Wpack, void *y, int64_t T, int C, int fuse_gelu,
                        int dtype, int path, eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_d8_shape(C, dtype);
  if (rc) return rc;
  if (T < 0) return set_error(EQLIN_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
  if (fuse_gelu != 0 && fuse_gelu != 1)
    return set_error(EQLIN_ERR_INVALID_ARG, "fuse_gelu must be 0 or 1");
  if (path != EQLIN_PATH_AUTO && path != EQLIN_PATH_SIMT && path != EQLIN_PATH_TC)
    return set_error(EQLIN_ERR_INVALID_ARG, "unknown path %d", path);
  if (T == 0) return EQLIN_OK;
  if (!x || !Wpack || !y) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(y) || !aligned16(Wpack))
    return set_error(EQLIN_ERR_ALIGN, "x, y and Wpack must be 16-byte aligned");
  const bool tc_ok = d8_tc_supported(C, dtype);
  if (path == EQLIN_PATH_TC && !tc_ok)
    return set_error(EQLIN_ERR_UNSUPPORTED, "tensor-core D8 path needs bf16 and C%%256==0, 256<=C<=1280");
  const D8PackLayout L = d8_pack_layout(C, dtype);
  if (tc_ok && (path == EQLIN_PATH_TC || (path == EQLIN_PATH_AUTO && aligned32(y))))
    return launch_d8_tc(x, static_cast<const char *>(Wpack) + L.tc_offset, y, T, C, fuse_gelu,
                        (cudaStream_t)stream);
  return launch_d8_simt(x, Wpack, y, T, C, fuse_gelu, dtype, L, (cudaStream_t)stream);
}

int eqlin_d8_forward(const void *x, const void *Wpack, void *y, int64_t T, int C, int fuse_gelu,
                     int dtype, eqlin_stream_t stream) {
  return eqlin_d8_forward_ex(x, Wpack, y, T, C, fuse_gelu, dtype, EQLIN_PATH_AUTO, stream);
}

static int check_d8_fourier(int F_in, int F_out, int dtype) {
  if (dtype != EQLIN_F32 && dtype != EQLIN_BF16 && dtype != EQLIN_F16)
    return set_error(EQLIN_ERR_UNSUPPORTED, "dtype %d is not EQLIN_F32, EQLIN_BF16 or EQLIN_F16", dtype);
  if (F_in < 1 || F_out < 1 || F_in > (1 << 17) || F_out > (1 << 17))
    return set_error(EQLIN_ERR_UNSUPPORTED, "F_in=%d, F_out=%d must be in 1..131072", F_in, F_out);
  return EQLIN_OK;
}

// Fourier-domain D8 pack: the fp32 CUDA-core section, then, for bf16 layers
// the fused kernel takes, its packed weight stages on 256-byte boundaries: one
// section, or for F_in > 160 one per column slice of at most 160 input fields
// (slices run as separate layers whose bf16 partial outputs are summed).
constexpr int kD8SliceMax = 160;
struct D8FourierLayout {
  size_t simt_bytes, tc_offset, tc_bytes, total;
  int nslices;                       // 0: no tensor-core section
  size_t slice_off[8];               // from the pack's start
};
static int d8_slice_width(int F_in, int sl) {
  const int w = F_in - sl * kD8SliceMax;
  return w < kD8SliceMax ? w : kD8SliceMax;
}
static D8FourierLayout d8_fourier_layout(int F_in, int F_out, int dtype) {
  D8FourierLayout L{};
  L.simt_bytes = d8_fourier_pack_bytes(F_in, F_out);
  L.tc_offset = round_up(L.simt_bytes, 256);
  const int ns = (F_in + kD8SliceMax - 1) / kD8SliceMax;
  const bool ok = dtype == EQLIN_BF16 && F_in % 16 == 0 && ns <= 8 &&
                  d8_fourier_tc_supported(d8_slice_width(F_in, 0), F_out, dtype) &&
                  d8_fourier_tc_supported(d8_slice_width(F_in, ns - 1), F_out, dtype);
  size_t off = L.tc_offset;
  if (ok) {
    L.nslices = ns;
    for (int sl = 0; sl < ns; ++sl) {
      L.slice_off[sl] = off;
      off += round_up(d8_fourier_tc_bytes(d8_slice_width(F_in, sl), F_out), 256);
    }
  }
  L.tc_bytes = ok ? off - L.tc_offset : 0;
  L.total = ok ? off : L.simt_bytes;
  return L;
}

size_t eqlin_d8_fourier_weight_bytes(int F_in, int F_out, int dtype) {
  if (check_d8_fourier(F_in, F_out, dtype) != EQLIN_OK) return 0;
  return d8_fourier_layout(F_in, F_out, dtype).total;
}

size_t eqlin_d8_fourier_workspace_bytes(int64_t T, int F_in, int F_out, int dtype) {
  if (check_d8_fourier(F_in, F_out, dtype) != EQLIN_OK || T < 0) return 0;
  const D8FourierLayout L = d8_fourier_layout(F_in, F_out, dtype);
  if (L.nslices < 2) return 0;
  return (size_t)L.nslices * (size_t)T * (size_t)F_out * 8 * sizeof(__nv_bfloat16);
}

int eqlin_d8_fourier_pack_weights(const void *wA1, const void *wA2, const void *wB1, const void *wB2,
                                  const void *wE, int F_in, int F_out, int dtype, void *Wpack,
                                  size_t Wpack_bytes, eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_d8_fourier(F_in, F_out, dtype);
  if (rc) return rc;
  const void *w[5] = {wA1, wA2, wB1, wB2, wE};
  for (int k = 0; k < 5; ++k) {
    if (!w[k]) return set_error(EQLIN_ERR_INVALID_ARG, "null weight pointer");
    if (!aligned16(w[k])) return set_error(EQLIN_ERR_ALIGN, "weights must be 16-byte aligned");
  }
  if (!Wpack) return set_error(EQLIN_ERR_INVALID_ARG, "null Wpack");
  if (!aligned16(Wpack)) return set_error(EQLIN_ERR_ALIGN, "Wpack must be 16-byte aligned");
  const D8FourierLayout L = d8_fourier_layout(F_in, F_out, dtype);
  if (Wpack_bytes < L.total)
    return set_error(EQLIN_ERR_SIZE, "Wpack_bytes=%zu < required %zu", Wpack_bytes, L.total);
  rc = launch_d8_fourier_pack(w, F_in, F_out, dtype, Wpack, (cudaStream_t)stream);
  for (int sl = 0; rc == EQLIN_OK && sl < L.nslices; ++sl)
    rc = launch_d8_fourier_tc_pack(w, F_in, sl * kD8SliceMax, d8_slice_width(F_in, sl), F_out,
                                   static_cast<char *>(Wpack) + L.slice_off[sl], (cudaStream_t)stream);
  return rc;
}

static const char *kD8TcNeeds =
    "tensor-core Fourier-domain D8 layer needs bf16, F_in%%16==0 and F_out%%32==0 (F_in > 160: a workspace)";

static int d8_fourier_run(const void *z, const void *Wpack, void *y, int64_t T, int F_in, int F_out,
                          int roundtrip_gelu, int dtype, int path, void *ws, size_t ws_bytes,
                          cudaStream_t s) {
  const D8FourierLayout L = d8_fourier_layout(F_in, F_out, dtype);
  const char *pk = static_cast<const char *>(Wpack);
  const bool one = L.nslices == 1;
  const size_t need = L.nslices > 1 ? (size_t)L.nslices * (size_t)T * F_out * 16 : 0;
  // slice partials are the fused kernel's outputs: 32-byte aligned
  const bool sliced = L.nslices > 1 && ws && ws_bytes >= need && aligned32(ws);
  if (path == EQLIN_PATH_TC && !one && !sliced) return set_error(EQLIN_ERR_UNSUPPORTED, kD8TcNeeds);
  if (one && (path == EQLIN_PATH_TC || (path == EQLIN_PATH_AUTO && aligned32(y))))
    return launch_d8_fourier_tc(z, pk + L.slice_off[0], y, T, F_in, F_out, roundtrip_gelu, F_in, s);
  if (sliced && path != EQLIN_PATH_SIMT) {
    // each slice: its F_in columns of z (rows F_in fields apart) -> a bf16
    // partial output; then the partials are summed in slice order
    char *parts = static_cast<char *>(ws);
    const size_t part_bytes = (size_t)T * F_out * 16;
    for (int sl = 0; sl < L.nslices; ++sl) {
      const int rc = launch_d8_fourier_tc(static_cast<const __nv_bfloat16 *>(z) + (size_t)sl * kD8SliceMax * 8,
                                          pk + L.slice_off[sl], parts + sl * part_bytes, T,
                                          d8_slice_width(F_in, sl), F_out, 0, F_in, s);
      if (rc) return rc;
    }
    return launch_d8_slice_sum(parts, L.nslices, T, F_out, roundtrip_gelu, y, s);
  }
  return launch_d8_fourier_linear(z, Wpack, y, T, F_in, F_out, roundtrip_gelu, dtype, s);
}

static int d8_fourier_check_io(const void *z, const void *Wpack, const void *y, int64_t T, int F_in,
                               int F_out, int roundtrip_gelu, int dtype, int path) {
  int rc = check_d8_fourier(F_in, F_out, dtype);
  if (rc) return rc;
  if (T < 0) return set_error(EQLIN_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
  if (roundtrip_gelu != 0 && roundtrip_gelu != 1)
    return set_error(EQLIN_ERR_INVALID_ARG, "roundtrip_gelu must be 0 or 1");
  if (path != EQLIN_PATH_AUTO && path != EQLIN_PATH_SIMT && path != EQLIN_PATH_TC)
    return set_error(EQLIN_ERR_INVALID_ARG, "unknown path %d", path);
  if (path == EQLIN_PATH_TC && d8_fourier_layout(F_in, F_out, dtype).nslices == 0)
    return set_error(EQLIN_ERR_UNSUPPORTED, kD8TcNeeds);
  if (T == 0) return EQLIN_OK;
  if (!z || !Wpack || !y) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(z) || !aligned16(y) || !aligned16(Wpack))
    return set_error(EQLIN_ERR_ALIGN, "z, y and Wpack must be 16-byte aligned");
  return EQLIN_OK;
}

int eqlin_d8_fourier_linear_ws(const void *z, const void *Wpack, void *y, int64_t T, int F_in, int F_out,
                               int roundtrip_gelu, int dtype, int path, void *workspace,
                               size_t workspace_bytes, eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = d8_fourier_check_io(z, Wpack, y, T, F_in, F_out, roundtrip_gelu, dtype, path);
  if (rc || T == 0) return rc;
  const size_t need = eqlin_d8_fourier_workspace_bytes(T, F_in, F_out, dtype);
  if (workspace && !aligned16(workspace))
    return set_error(EQLIN_ERR_ALIGN, "workspace must be 16-byte aligned");
  if (path == EQLIN_PATH_TC && need && (!workspace || workspace_bytes < need))
    return set_error(EQLIN_ERR_SIZE, "workspace_bytes=%zu < required %zu", workspace_bytes, need);
  if (path == EQLIN_PATH_TC && need && !aligned32(workspace))
    return set_error(EQLIN_ERR_ALIGN, "the tensor-core path's workspace must be 32-byte aligned");
  return d8_fourier_run(z, Wpack, y, T, F_in, F_out, roundtrip_gelu, dtype, path, workspace,
                        workspace_bytes, (cudaStream_t)stream);
}

int eqlin_d8_fourier_linear_ex(const void *z, const void *Wpack, void *y, int64_t T, int F_in, int F_out,
                               int roundtrip_gelu, int dtype, int path, eqlin_stream_t stream) {
  return eqlin_d8_fourier_linear_ws(z, Wpack, y, T, F_in, F_out, roundtrip_gelu, dtype, path, nullptr, 0,
                                    stream);
}

int eqlin_d8_fourier_linear(const void *z, const void *Wpack, void *y, int64_t T, int F_in, int F_out,
                            int roundtrip_gelu, int dtype, eqlin_stream_t stream) {
  return eqlin_d8_fourier_linear_ws(z, Wpack, y, T, F_in, F_out, roundtrip_gelu, dtype, EQLIN_PATH_AUTO,
                                    nullptr, 0, stream);
}

size_t eqlin_d8_fourier_mlp_workspace_bytes(int64_t T, int F, int F_hidden, int dtype) {
  return eqlin_d8_fourier_workspace_bytes(T, F_hidden, F, dtype);
}

int eqlin_d8_fourier_mlp_ws(const void *z, const void *W1pack, const void *W2pack, void *hidden, void *y,
                            int64_t T, int F, int F_hidden, int dtype, void *workspace,
                            size_t workspace_bytes, eqlin_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_d8_fourier(F, F_hidden, dtype);
  if (rc) return rc;
  if (T < 0) return set_error(EQLIN_ERR_INVALID_ARG, "T=%lld < 0", (long long)T);
  if (T == 0) return EQLIN_OK;
  if (!z || !W1pack || !W2pack || !hidden || !y) return set_error(EQLIN_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(z) || !aligned16(y) || !aligned16(hidden) || !aligned16(W1pack) || !aligned16(W2pack))
    return set_error(EQLIN_ERR_ALIGN, "z, hidden, y and the packs must be 16-byte aligned");
  if (workspace && !aligned16(workspace))
    return set_error(EQLIN_ERR_ALIGN, "workspace must be 16-byte aligned");
  rc = d8_fourier_run(z, W1pack, hidden, T, F, F_hidden, 1, dtype, EQLIN_PATH_AUTO, nullptr, 0,
                      (cudaStream_t)stream);
  if (rc) return rc;
  return d8_fourier_run(hidden, W2pack, y, T, F_hidden, F, 0, dtype, EQLIN_PATH_AUTO, workspace,
                        workspace_bytes, (cudaStream_t)stream);
}

int eqlin_d8_fourier_mlp(const void *z, const void *W1pack, const void *W2pack, void *hidden, void *y,
                         int64_t T, int F, int F_hidden, int dtype, eqlin_stream_t stream) {
  return eqlin_d8_fourier_mlp_ws(z, W1pack, W2pack, hidden, y, T, F, F_hidden, dtype, nullptr, 0, stream);
}

}  // extern "C"
