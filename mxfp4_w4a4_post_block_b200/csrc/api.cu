// extern "C" boundary of libbatq: argument checks, host-side preparation and launches.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/batq.h"
#include "host_util.h"
#include "kernels.h"

namespace {

// Device error word, one per device (set by kernels whose bounded waits gave up).
__device__ unsigned int g_batq_error_word;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device must be sm_100 (B200 class).  Cached per device.
batq_status check_arch() {
  static int state[kMaxDevices] = {0};  // 0 unknown, 1 ok, 2 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BATQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BATQ_ERR_ARCH;
  if (state[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return BATQ_ERR_CUDA;
    state[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return state[dev] == 1 ? BATQ_OK : BATQ_ERR_ARCH;
}

unsigned* error_word() {
  static unsigned* cached[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (cached[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_batq_error_word) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<unsigned*>(p);
  }
  return cached[dev];
}

size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }

size_t scale_bytes_for(int rows, int N, batq_scale_layout layout) {
  const size_t k = (size_t)N / 32;
  if (layout == BATQ_SCALES_MMA) return round_up((size_t)rows, 128) * round_up(k, 4);
  return (size_t)rows * k;
}

// rows x N/32 below 2^31 keeps every tile index, scale offset and scale
// buffer inside the kernels' 32-bit arithmetic (N = 4096: up to 16.7 M rows).
batq_status check_mn(int rows, int N) {
  if (rows < 1 || N < 64 || (N % 64) != 0) return BATQ_ERR_SHAPE;
  if ((long long)rows * (N / 32) >= (1LL << 31)) return BATQ_ERR_SHAPE;
  return BATQ_OK;
}

// Inverse of an n x n matrix (row-major, double) by Gauss-Jordan elimination
// with partial pivoting; returns false if singular or if the 1-norm condition
// number exceeds 1e8.
bool invert(const double* a, double* inv, int n) {
  std::vector<double> m((size_t)n * 2 * n);
  double norm_a = 0.0;
  for (int c = 0; c < n; ++c) {
    double col = 0.0;
    for (int r = 0; r < n; ++r) col += std::fabs(a[r * n + c]);
    norm_a = col > norm_a ? col : norm_a;
  }
  for (int r = 0; r < n; ++r) {
    for (int c = 0; c < n; ++c) {
      m[(size_t)r * 2 * n + c] = a[r * n + c];
      m[(size_t)r * 2 * n + n + c] = (r == c) ? 1.0 : 0.0;
    }
  }
  for (int col = 0; col < n; ++col) {
    int piv = col;
    for (int r = col + 1; r < n; ++r)
      if (std::fabs(m[(size_t)r * 2 * n + col]) > std::fabs(m[(size_t)piv * 2 * n + col])) piv = r;
    const double pv = m[(size_t)piv * 2 * n + col];
    if (!(std::fabs(pv) > 0.0) || !std::isfinite(pv)) return false;
    if (piv != col)
      for (int c = 0; c < 2 * n; ++c) std::swap(m[(size_t)piv * 2 * n + c], m[(size_t)col * 2 * n + c]);
    for (int c = 0; c < 2 * n; ++c) m[(size_t)col * 2 * n + c] /= pv;
    for (int r = 0; r < n; ++r) {
      if (r == col) continue;
      const double f = m[(size_t)r * 2 * n + col];
      if (f == 0.0) continue;
      for (int c = 0; c < 2 * n; ++c) m[(size_t)r * 2 * n + c] -= f * m[(size_t)col * 2 * n + c];
    }
  }
  double norm_inv = 0.0;
  for (int c = 0; c < n; ++c) {
    double col = 0.0;
    for (int r = 0; r < n; ++r) {
      inv[r * n + c] = m[(size_t)r * 2 * n + n + c];
      col += std::fabs(inv[r * n + c]);
    }
    norm_inv = col > norm_inv ? col : norm_inv;
  }
  const double cond = norm_a * norm_inv;
  return std::isfinite(cond) && cond <= 1e8;
}

// gs / gs_amax / gs_out / amax_out: the NVFP4 per-tensor scale sources and
// outputs of batq::QuantLaunch (nullptr for the MX formats).
batq_status launch_quant(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                         const float* B_dev, const float* ratios_dev, uint8_t* codes, uint8_t* scales,
                         batq_scale_layout layout, float* y_debug, int fmt, cudaStream_t stream,
                         const float* gs = nullptr, const unsigned* gs_amax = nullptr, float* gs_out = nullptr,
                         unsigned* amax_out = nullptr, const float* A_blocks = nullptr,
                         const float* gamma = nullptr, const float* row_scale = nullptr) {
  batq::QuantLaunch L;
  L.X = X;
  L.bf16 = (x_dtype == BATQ_BF16);
  L.S = S;
  L.N = N;
  L.ldx = ldx;
  std::memcpy(L.A, A_host, sizeof(L.A));
  L.B = B_dev;
  L.ratios = ratios_dev;
  L.codes = codes;
  L.scales = scales;
  L.mma_layout = (layout == BATQ_SCALES_MMA);
  L.y_debug = y_debug;
  L.err = error_word();
  L.stream = stream;
  L.fmt = fmt;
  L.gs = gs;
  L.gs_amax = gs_amax;
  L.gs_out = gs_out;
  L.amax_out = amax_out;
  L.A_blocks = A_blocks;
  L.gamma = gamma;
  L.row_scale = row_scale;
  cudaError_t e = batq::launch_quant_act(L);
  if (e == cudaErrorInvalidValue) return BATQ_ERR_ALIGNMENT;
  return e == cudaSuccess ? BATQ_OK : BATQ_ERR_CUDA;
}

batq_status check_quant_args(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                             const float* B_dev, const float* ratios_dev, const uint8_t* codes,
                             const uint8_t* scales, batq_scale_layout layout, const float* y_debug) {
  if (!X || !A_host || !B_dev || !codes || !scales) return BATQ_ERR_INVALID_ARG;
  if (x_dtype != BATQ_F32 && x_dtype != BATQ_BF16) return BATQ_ERR_INVALID_ARG;
  if (layout != BATQ_SCALES_LINEAR && layout != BATQ_SCALES_MMA) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(S, N);
  if (st != BATQ_OK) return st;
  if (ldx < N) return BATQ_ERR_SHAPE;
  const size_t esz = x_dtype == BATQ_BF16 ? 2 : 4;
  if (!aligned16(X) || ((size_t)ldx * esz) % 16 != 0 || !aligned16(codes) || !aligned16(B_dev))
    return BATQ_ERR_ALIGNMENT;
  if (ratios_dev && !aligned16(ratios_dev)) return BATQ_ERR_ALIGNMENT;
  if (y_debug && !aligned16(y_debug)) return BATQ_ERR_ALIGNMENT;
  if (layout == BATQ_SCALES_MMA && !aligned16(scales)) return BATQ_ERR_ALIGNMENT;
  return BATQ_OK;
}

batq_status check_gemm_args(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                            const uint8_t* w_scales, int S, int M, int N, batq_dtype out_dtype, const void* out,
                            int ldo) {
  if (!a_codes || !a_scales || !w_codes || !w_scales || !out) return BATQ_ERR_INVALID_ARG;
  if (out_dtype != BATQ_F32 && out_dtype != BATQ_BF16) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(S, N);
  if (st != BATQ_OK) return st;
  if (M < 16 || (M % 16) != 0 || ldo < M) return BATQ_ERR_SHAPE;
  const size_t esz = out_dtype == BATQ_BF16 ? 2 : 4;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(out) || ((size_t)ldo * esz) % 16 != 0)
    return BATQ_ERR_ALIGNMENT;
  return BATQ_OK;
}

batq_status launch_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                        const uint8_t* w_scales, int S, int M, int N, batq_dtype out_dtype, void* out, int ldo,
                        bool weights_ready, int fmt, cudaStream_t stream, const float* gs_a = nullptr,
                        const float* gs_w = nullptr) {
  batq::GemmLaunch L;
  L.a_codes = a_codes;
  L.a_scales = a_scales;
  L.w_codes = w_codes;
  L.w_scales = w_scales;
  L.S = S;
  L.M = M;
  L.N = N;
  L.out_bf16 = (out_dtype == BATQ_BF16);
  L.out = out;
  L.ldo = ldo;
  L.err = error_word();
  L.stream = stream;
  L.weights_ready = weights_ready;
  L.fmt = fmt;
  L.gs_a = gs_a;
  L.gs_w = gs_w;
  cudaError_t e = batq::launch_gemm_mxfp4(L);
  if (e == cudaErrorInvalidValue) return BATQ_ERR_ALIGNMENT;
  return e == cudaSuccess ? BATQ_OK : BATQ_ERR_CUDA;
}

// Transform of the fused weights: W'_mat = B_i^-1 W_mat A^-T, and the
// activation kernel computes B'^T X A', so A' = A^-T (to a_fused, host) and
// B'_i = B_i^-T (k x 16 floats copied to the start of `workspace`, device).
batq_status fused_transform(const float* A_host, const float* B_host, int N, void* workspace, float a_fused[64],
                            cudaStream_t s) {
  const int k = N / 32;
  double a[64], ainv[64];
  for (int i = 0; i < 64; ++i) a[i] = A_host[i];
  if (!invert(a, ainv, 8)) return BATQ_ERR_SINGULAR;
  for (int r = 0; r < 8; ++r)
    for (int c = 0; c < 8; ++c) a_fused[r * 8 + c] = (float)ainv[c * 8 + r];
  std::vector<float> b_fused((size_t)k * 16);
  for (int i = 0; i < k; ++i) {
    double b[16], binv[16];
    for (int j = 0; j < 16; ++j) b[j] = B_host[(size_t)i * 16 + j];
    if (!invert(b, binv, 4)) return BATQ_ERR_SINGULAR;
    for (int r = 0; r < 4; ++r)
      for (int c = 0; c < 4; ++c) b_fused[(size_t)i * 16 + r * 4 + c] = (float)binv[c * 4 + r];
  }
  if (cudaMemcpyAsync(workspace, b_fused.data(), b_fused.size() * sizeof(float), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return BATQ_ERR_CUDA;
  // cudaMemcpyAsync from pageable memory has staged the bytes when it returns,
  // so b_fused may be released.
  return BATQ_OK;
}

size_t nv_scale_bytes_for(int rows, int N, batq_scale_layout layout) {
  const size_t cols = (size_t)N / 16;  // a multiple of 4 for N % 64 == 0
  if (layout == BATQ_SCALES_MMA) return round_up((size_t)rows, 128) * cols;
  return (size_t)rows * cols;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Stand-in for the shared A where the naive Kronecker calls pass one A_i per block instead.
const float kUnusedA[64] = {};

// Naive Kronecker weight side: A'_i = A_i^-T (k x 64 floats) for every block, and B'_i as in
// fused_transform, both copied into the workspace: B' at 0, A' at a_offset.
batq_status fused_transform_kron(const float* A_blocks_host, const float* B_host, int N, void* workspace,
                                 size_t a_offset, cudaStream_t s) {
  const int k = N / 32;
  float unused[64];
  // B'_i and the transfer to the workspace's start: the shared-A routine with an identity A.
  float eye[64] = {};
  for (int i = 0; i < 8; ++i) eye[i * 9] = 1.0f;
  batq_status st = fused_transform(eye, B_host, N, workspace, unused, s);
  if (st != BATQ_OK) return st;
  std::vector<float> a_fused((size_t)k * 64);
  for (int i = 0; i < k; ++i) {
    double a[64], ainv[64];
    for (int j = 0; j < 64; ++j) a[j] = A_blocks_host[(size_t)i * 64 + j];
    if (!invert(a, ainv, 8)) return BATQ_ERR_SINGULAR;
    for (int r = 0; r < 8; ++r)
      for (int c = 0; c < 8; ++c) a_fused[(size_t)i * 64 + r * 8 + c] = (float)ainv[c * 8 + r];
  }
  if (cudaMemcpyAsync(static_cast<uint8_t*>(workspace) + a_offset, a_fused.data(), a_fused.size() * sizeof(float),
                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return BATQ_ERR_CUDA;
  return BATQ_OK;
}

size_t rms_bytes_for(int S) { return round_up((size_t)S * sizeof(float), 256); }

// Checks of the RMSNorm arguments beyond the quantiser's own.
batq_status check_rmsnorm_args(const float* gamma_dev, float eps) {
  if (!gamma_dev) return BATQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return BATQ_ERR_INVALID_ARG;
  if (!aligned16(gamma_dev)) return BATQ_ERR_ALIGNMENT;
  return BATQ_OK;
}

// RMSNorm factors of every token into rms (device, S floats), then the
// quantiser with gamma and those factors, on one stream.
batq_status launch_rmsnorm_quant(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* gamma_dev,
                                 float eps, const float* A_host, const float* B_dev, const float* ratios_dev,
                                 uint8_t* codes, uint8_t* scales, batq_scale_layout layout, float* rms,
                                 float* y_debug, cudaStream_t s) {
  if (batq::launch_row_rms(X, x_dtype == BATQ_BF16, S, N, ldx, eps, rms, s) != cudaSuccess) return BATQ_ERR_CUDA;
  return launch_quant(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout, y_debug,
                      batq::kFmtMxfp4, s, nullptr, nullptr, nullptr, nullptr, nullptr, gamma_dev, rms);
}

}  // namespace

extern "C" {

const char* batq_status_string(batq_status status) {
  switch (status) {
    case BATQ_OK: return "ok";
    case BATQ_ERR_INVALID_ARG: return "invalid argument";
    case BATQ_ERR_SHAPE: return "unsupported shape";
    case BATQ_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case BATQ_ERR_SINGULAR: return "transform factor singular or ill-conditioned";
    case BATQ_ERR_ARCH: return "device is not sm_100";
    case BATQ_ERR_CUDA: return "CUDA error";
    case BATQ_ERR_TIMEOUT: return "kernel barrier wait timed out";
    case BATQ_ERR_WORKSPACE: return "workspace too small";
    case BATQ_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the fixed no-allocation array holds";
  }
  return "unknown status";
}

int batq_version(void) { return 100; }

batq_status batq_act_buffer_sizes(int rows, int N, batq_scale_layout layout, size_t* code_bytes,
                                  size_t* scale_bytes) {
  if (!code_bytes || !scale_bytes) return BATQ_ERR_INVALID_ARG;
  if (layout != BATQ_SCALES_LINEAR && layout != BATQ_SCALES_MMA) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(rows, N);
  if (st != BATQ_OK) return st;
  *code_bytes = (size_t)rows * (size_t)(N / 2);
  *scale_bytes = scale_bytes_for(rows, N, layout);
  return BATQ_OK;
}

batq_status batq_clip_ratios(const float* alpha_min_host, const float* alpha_max_host, int k,
                             float* ratios_out_host) {
  if (!alpha_min_host || !alpha_max_host || !ratios_out_host || k < 1) return BATQ_ERR_INVALID_ARG;
  for (int i = 0; i < k; ++i) {
    ratios_out_host[2 * i] = (float)(1.0 / (1.0 + std::exp(-(double)alpha_min_host[i])));
    ratios_out_host[2 * i + 1] = (float)(1.0 / (1.0 + std::exp(-(double)alpha_max_host[i])));
  }
  return BATQ_OK;
}

batq_status batq_quant_act(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                           const float* B_dev, const float* ratios_dev, uint8_t* codes, uint8_t* scales,
                           batq_scale_layout layout, float* y_debug, void* stream) {
  batq_status st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout,
                                    y_debug);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  return launch_quant(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout, y_debug,
                      batq::kFmtMxfp4, static_cast<cudaStream_t>(stream));
}

batq_status batq_prepare_workspace_size(int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  if (N < 64 || N % 64 != 0) return BATQ_ERR_SHAPE;
  *bytes = round_up((size_t)(N / 32) * 16 * sizeof(float), 256);
  return BATQ_OK;
}

batq_status batq_prepare_weights(const void* W, batq_dtype w_dtype, int M, int N, int ldw, const float* A_host,
                                 const float* B_host, uint8_t* w_codes, uint8_t* w_scales,
                                 batq_scale_layout layout, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!B_host || !workspace) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_quant_args(W, w_dtype, M, N, ldw, A_host, reinterpret_cast<const float*>(workspace),
                                    nullptr, w_codes, w_scales, layout, nullptr);
  if (st != BATQ_OK) return st;
  size_t need = 0;
  batq_prepare_workspace_size(N, &need);
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  st = check_arch();
  if (st != BATQ_OK) return st;

  float a_fused[64];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = fused_transform(A_host, B_host, N, workspace, a_fused, s);
  if (st != BATQ_OK) return st;
  return launch_quant(W, w_dtype, M, N, ldw, a_fused, reinterpret_cast<const float*>(workspace), nullptr, w_codes,
                      w_scales, layout, nullptr, batq::kFmtMxfp4, s);
}

batq_status batq_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                            const uint8_t* w_scales, int S, int M, int N, batq_dtype out_dtype, void* out, int ldo,
                            void* stream) {
  batq_status st = check_gemm_args(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  // The preceding grid may be anything (e.g. the weight quantiser of
  // batq_prepare_weights): wait for it before reading any operand.
  return launch_gemm(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo, false, batq::kFmtMxfp4,
                     static_cast<cudaStream_t>(stream));
}

batq_status batq_linear_workspace_size(int S, int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(S, N);
  if (st != BATQ_OK) return st;
  *bytes = round_up((size_t)S * (N / 2), 256) + scale_bytes_for(S, N, BATQ_SCALES_MMA);
  return BATQ_OK;
}

batq_status batq_linear(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                        const float* B_dev, const float* ratios_dev, const uint8_t* w_codes,
                        const uint8_t* w_scales, int M, void* workspace, size_t workspace_bytes,
                        batq_dtype out_dtype, void* out, int ldo, void* stream) {
  if (!workspace) return BATQ_ERR_INVALID_ARG;
  size_t need = 0;
  batq_status st = batq_linear_workspace_size(S, N, &need);
  if (st != BATQ_OK) return st;
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BATQ_ERR_ALIGNMENT;
  uint8_t* a_codes = static_cast<uint8_t*>(workspace);
  uint8_t* a_scales = a_codes + round_up((size_t)S * (N / 2), 256);
  st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA,
                        nullptr);
  if (st != BATQ_OK) return st;
  st = check_gemm_args(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_quant(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA, nullptr,
                    batq::kFmtMxfp4, s);
  if (st != BATQ_OK) return st;
  // The quantiser just launched writes only the workspace and starts its
  // dependents after every earlier grid has finished, so the GEMM may fetch
  // weights while the quantiser runs.
  return launch_gemm(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo, true, batq::kFmtMxfp4, s);
}

// ------------------------------------------------------------------ groups of linears

// Launch an already checked quantiser group.  Each activation takes the
// kernel its own batq_quant_act call would take, so the codes are the same:
// those for the tensor-core kernel (bf16, six or more 128 x 128 tiles per SM)
// share one launch of it, the others one launch of the CUDA-core kernel per
// input type.
batq_status quant_group_checked(const batq_quant_args* q, int count, cudaStream_t s) {
  batq::QuantLaunch Q[BATQ_MAX_LINEAR_GROUP];
  for (int i = 0; i < count; ++i) {
    batq::QuantLaunch& L = Q[i];
    L.X = q[i].X;
    L.bf16 = (q[i].x_dtype == BATQ_BF16);
    L.S = q[i].S;
    L.N = q[i].N;
    L.ldx = q[i].ldx;
    std::memcpy(L.A, q[i].A_host, sizeof(L.A));
    L.B = q[i].B_dev;
    L.ratios = q[i].ratios_dev;
    L.codes = q[i].codes;
    L.scales = q[i].scales;
    L.mma_layout = (q[i].layout == BATQ_SCALES_MMA);
    L.y_debug = nullptr;
    L.err = error_word();
    L.stream = s;
    L.fmt = batq::kFmtMxfp4;
  }
  cudaError_t e = batq::launch_quant_act_group(Q, count);
  if (e == cudaErrorInvalidValue) return BATQ_ERR_ALIGNMENT;
  return e == cudaSuccess ? BATQ_OK : BATQ_ERR_CUDA;
}

// Tile configuration of the single-CTA GEMM for S <= 128 tokens.
int small_bucket(int S) { return S <= 16 ? 0 : S <= 32 ? 1 : S <= 64 ? 2 : 3; }

// Launch an already checked GEMM group: one CTA-pair launch when every S > 128,
// one single-CTA launch when every S <= 128 falls in the same tile
// configuration (S <= 16 / 32 / 64 / 128), in both cases with one output
// type; else one launch per product.  weights_ready: the grid before this
// call writes no weights.
batq_status gemm_group_checked(const batq_gemm_args* g, int count, bool weights_ready, cudaStream_t s) {
  bool all_pair = true, all_small = true;
  for (int i = 0; i < count; ++i) {
    const bool same_out = g[i].out_dtype == g[0].out_dtype;
    all_pair = all_pair && g[i].S > 128 && same_out;
    all_small = all_small && g[i].S <= 128 && small_bucket(g[i].S) == small_bucket(g[0].S) && same_out;
  }
  if (!all_pair && !all_small) {
    for (int i = 0; i < count; ++i) {
      // After the first, the grid before each launch is an earlier GEMM of the
      // group, whose output overlaps no input.
      batq_status st = launch_gemm(g[i].a_codes, g[i].a_scales, g[i].w_codes, g[i].w_scales, g[i].S, g[i].M, g[i].N,
                                   g[i].out_dtype, g[i].out, g[i].ldo, weights_ready || i > 0, batq::kFmtMxfp4, s);
      if (st != BATQ_OK) return st;
    }
    return BATQ_OK;
  }
  batq::GemmLaunch G[BATQ_MAX_LINEAR_GROUP];
  for (int i = 0; i < count; ++i) {
    batq::GemmLaunch& L = G[i];
    L.a_codes = g[i].a_codes;
    L.a_scales = g[i].a_scales;
    L.w_codes = g[i].w_codes;
    L.w_scales = g[i].w_scales;
    L.S = g[i].S;
    L.M = g[i].M;
    L.N = g[i].N;
    L.out_bf16 = (g[i].out_dtype == BATQ_BF16);
    L.out = g[i].out;
    L.ldo = g[i].ldo;
    L.err = error_word();
    L.stream = s;
    L.weights_ready = weights_ready;
    L.fmt = batq::kFmtMxfp4;
    L.gs_a = nullptr;
    L.gs_w = nullptr;
  }
  cudaError_t e = all_pair ? batq::launch_gemm_pair_group(G, count) : batq::launch_gemm_mxfp4_small_group(G, count);
  if (e == cudaErrorInvalidValue) return BATQ_ERR_ALIGNMENT;
  return e == cudaSuccess ? BATQ_OK : BATQ_ERR_CUDA;
}

batq_status batq_quant_act_grouped(const batq_quant_args* acts, int count, void* stream) {
  if (!acts || count < 1 || count > BATQ_MAX_LINEAR_GROUP) return BATQ_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const batq_quant_args& q = acts[i];
    batq_status st = check_quant_args(q.X, q.x_dtype, q.S, q.N, q.ldx, q.A_host, q.B_dev, q.ratios_dev, q.codes,
                                      q.scales, q.layout, nullptr);
    if (st != BATQ_OK) return st;
  }
  batq_status st = check_arch();
  if (st != BATQ_OK) return st;
  return quant_group_checked(acts, count, static_cast<cudaStream_t>(stream));
}

batq_status batq_gemm_mxfp4_grouped(const batq_gemm_args* gemms, int count, void* stream) {
  if (!gemms || count < 1 || count > BATQ_MAX_LINEAR_GROUP) return BATQ_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const batq_gemm_args& g = gemms[i];
    batq_status st = check_gemm_args(g.a_codes, g.a_scales, g.w_codes, g.w_scales, g.S, g.M, g.N, g.out_dtype,
                                     g.out, g.ldo);
    if (st != BATQ_OK) return st;
  }
  batq_status st = check_arch();
  if (st != BATQ_OK) return st;
  return gemm_group_checked(gemms, count, false, static_cast<cudaStream_t>(stream));
}

batq_status batq_linear_grouped_workspace_size(const batq_linear_args* linears, int count, size_t* bytes) {
  if (!linears || !bytes || count < 1 || count > BATQ_MAX_LINEAR_GROUP) return BATQ_ERR_INVALID_ARG;
  size_t total = 0;
  for (int i = 0; i < count; ++i) {
    size_t need = 0;
    batq_status st = batq_linear_workspace_size(linears[i].S, linears[i].N, &need);
    if (st != BATQ_OK) return st;
    total += round_up(need, 256);
  }
  *bytes = total;
  return BATQ_OK;
}

batq_status batq_linear_grouped(const batq_linear_args* linears, int count, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!linears || !workspace || count < 1 || count > BATQ_MAX_LINEAR_GROUP) return BATQ_ERR_INVALID_ARG;
  size_t need = 0;
  batq_status st = batq_linear_grouped_workspace_size(linears, count, &need);
  if (st != BATQ_OK) return st;
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BATQ_ERR_ALIGNMENT;
  // Every check before any launch; linear i's codes and MMA scales in its
  // 256-byte-aligned part of the workspace.
  batq_quant_args q[BATQ_MAX_LINEAR_GROUP];
  batq_gemm_args g[BATQ_MAX_LINEAR_GROUP];
  uint8_t* at = static_cast<uint8_t*>(workspace);
  for (int i = 0; i < count; ++i) {
    const batq_linear_args& l = linears[i];
    uint8_t* codes = at;
    uint8_t* scales = at + round_up((size_t)l.S * (l.N / 2), 256);
    size_t one = 0;
    batq_linear_workspace_size(l.S, l.N, &one);
    at += round_up(one, 256);
    q[i] = batq_quant_args{l.X, l.x_dtype, l.S, l.N, l.ldx, l.A_host, l.B_dev, l.ratios_dev, codes, scales,
                           BATQ_SCALES_MMA};
    g[i] = batq_gemm_args{codes, scales, l.w_codes, l.w_scales, l.S, l.M, l.N, l.out_dtype, l.out, l.ldo};
    st = check_quant_args(l.X, l.x_dtype, l.S, l.N, l.ldx, l.A_host, l.B_dev, l.ratios_dev, codes, scales,
                          BATQ_SCALES_MMA, nullptr);
    if (st != BATQ_OK) return st;
    st = check_gemm_args(codes, scales, l.w_codes, l.w_scales, l.S, l.M, l.N, l.out_dtype, l.out, l.ldo);
    if (st != BATQ_OK) return st;
  }
  st = check_arch();
  if (st != BATQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = quant_group_checked(q, count, s);
  if (st != BATQ_OK) return st;
  // The quantiser grid(s) just launched write only the workspace, so the GEMM
  // may fetch weights before they finish.
  return gemm_group_checked(g, count, true, s);
}

// ------------------------------------------------------------------ W4A8 variant

batq_status batq_mxfp8_buffer_sizes(int rows, int N, batq_scale_layout layout, size_t* code_bytes,
                                    size_t* scale_bytes) {
  if (!code_bytes || !scale_bytes) return BATQ_ERR_INVALID_ARG;
  if (layout != BATQ_SCALES_LINEAR && layout != BATQ_SCALES_MMA) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(rows, N);
  if (st != BATQ_OK) return st;
  *code_bytes = (size_t)rows * (size_t)N;
  *scale_bytes = scale_bytes_for(rows, N, layout);
  return BATQ_OK;
}

batq_status batq_quant_act_mxfp8(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                                 const float* B_dev, const float* ratios_dev, uint8_t* codes, uint8_t* scales,
                                 batq_scale_layout layout, float* y_debug, void* stream) {
  batq_status st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout,
                                    y_debug);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  return launch_quant(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout, y_debug,
                      batq::kFmtMxfp8, static_cast<cudaStream_t>(stream));
}

batq_status batq_prepare_weights_w4a8_workspace_size(int M, int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(M, N);
  if (st != BATQ_OK) return st;
  size_t base = 0;
  batq_prepare_workspace_size(N, &base);
  *bytes = base + round_up((size_t)M * (size_t)(N / 2), 256);
  return BATQ_OK;
}

batq_status batq_prepare_weights_w4a8(const void* W, batq_dtype w_dtype, int M, int N, int ldw,
                                      const float* A_host, const float* B_host, uint8_t* w_codes8,
                                      uint8_t* w_scales, batq_scale_layout layout, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!workspace || !w_codes8) return BATQ_ERR_INVALID_ARG;
  size_t need = 0, base = 0;
  batq_status st = batq_prepare_weights_w4a8_workspace_size(M, N, &need);
  if (st != BATQ_OK) return st;
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace) || !aligned16(w_codes8)) return BATQ_ERR_ALIGNMENT;
  batq_prepare_workspace_size(N, &base);
  // The MXFP4 weights go to the workspace first (packed), then are widened
  // into the caller's E4M3 containers.
  uint8_t* packed = static_cast<uint8_t*>(workspace) + base;
  st = batq_prepare_weights(W, w_dtype, M, N, ldw, A_host, B_host, packed, w_scales, layout, workspace, base,
                            stream);
  if (st != BATQ_OK) return st;
  cudaError_t e = batq::launch_e2m1_to_e4m3(packed, w_codes8, (size_t)M * (size_t)(N / 2),
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BATQ_OK : BATQ_ERR_CUDA;
}

batq_status batq_gemm_w4a8(const uint8_t* a_codes8, const uint8_t* a_scales, const uint8_t* w_codes8,
                           const uint8_t* w_scales, int S, int M, int N, batq_dtype out_dtype, void* out, int ldo,
                           void* stream) {
  batq_status st = check_gemm_args(a_codes8, a_scales, w_codes8, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  return launch_gemm(a_codes8, a_scales, w_codes8, w_scales, S, M, N, out_dtype, out, ldo, false, batq::kFmtMxfp8,
                     static_cast<cudaStream_t>(stream));
}

batq_status batq_linear_w4a8_workspace_size(int S, int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(S, N);
  if (st != BATQ_OK) return st;
  *bytes = round_up((size_t)S * (size_t)N, 256) + scale_bytes_for(S, N, BATQ_SCALES_MMA);
  return BATQ_OK;
}

batq_status batq_linear_w4a8(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                             const float* B_dev, const float* ratios_dev, const uint8_t* w_codes8,
                             const uint8_t* w_scales, int M, void* workspace, size_t workspace_bytes,
                             batq_dtype out_dtype, void* out, int ldo, void* stream) {
  if (!workspace) return BATQ_ERR_INVALID_ARG;
  size_t need = 0;
  batq_status st = batq_linear_w4a8_workspace_size(S, N, &need);
  if (st != BATQ_OK) return st;
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BATQ_ERR_ALIGNMENT;
  uint8_t* a_codes = static_cast<uint8_t*>(workspace);
  uint8_t* a_scales = a_codes + round_up((size_t)S * (size_t)N, 256);
  st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA,
                        nullptr);
  if (st != BATQ_OK) return st;
  st = check_gemm_args(a_codes, a_scales, w_codes8, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_quant(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA, nullptr,
                    batq::kFmtMxfp8, s);
  if (st != BATQ_OK) return st;
  return launch_gemm(a_codes, a_scales, w_codes8, w_scales, S, M, N, out_dtype, out, ldo, true, batq::kFmtMxfp8, s);
}

// ------------------------------------------------------------------ NVFP4 output variant

batq_status batq_nvfp4_buffer_sizes(int rows, int N, batq_scale_layout layout, size_t* code_bytes,
                                    size_t* scale_bytes) {
  if (!code_bytes || !scale_bytes) return BATQ_ERR_INVALID_ARG;
  if (layout != BATQ_SCALES_LINEAR && layout != BATQ_SCALES_MMA) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(rows, N);
  if (st != BATQ_OK) return st;
  *code_bytes = (size_t)rows * (size_t)(N / 2);
  *scale_bytes = nv_scale_bytes_for(rows, N, layout);
  return BATQ_OK;
}

batq_status batq_quant_act_nvfp4(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                                 const float* B_dev, const float* ratios_dev, const float* gs_dev, uint8_t* codes,
                                 uint8_t* scales, batq_scale_layout layout, float* y_debug, void* stream) {
  batq_status st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout,
                                    y_debug);
  if (st != BATQ_OK) return st;
  if (!aligned16(scales) || (gs_dev && !aligned4(gs_dev))) return BATQ_ERR_ALIGNMENT;
  st = check_arch();
  if (st != BATQ_OK) return st;
  return launch_quant(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout, y_debug,
                      batq::kFmtNvfp4, static_cast<cudaStream_t>(stream), gs_dev);
}

batq_status batq_prepare_weights_nvfp4_workspace_size(int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  size_t base = 0;
  batq_status st = batq_prepare_workspace_size(N, &base);
  if (st != BATQ_OK) return st;
  *bytes = base + 256;  // + the amax word of the measuring pass
  return BATQ_OK;
}

batq_status batq_prepare_weights_nvfp4(const void* W, batq_dtype w_dtype, int M, int N, int ldw, const float* A_host,
                                       const float* B_host, uint8_t* w_codes, uint8_t* w_scales,
                                       batq_scale_layout layout, float* gs_out_dev, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (!B_host || !workspace || !gs_out_dev) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_quant_args(W, w_dtype, M, N, ldw, A_host, reinterpret_cast<const float*>(workspace),
                                    nullptr, w_codes, w_scales, layout, nullptr);
  if (st != BATQ_OK) return st;
  if (!aligned16(w_scales) || !aligned4(gs_out_dev)) return BATQ_ERR_ALIGNMENT;
  size_t need = 0, base = 0;
  batq_prepare_weights_nvfp4_workspace_size(N, &need);
  batq_prepare_workspace_size(N, &base);
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  st = check_arch();
  if (st != BATQ_OK) return st;
  float a_fused[64];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = fused_transform(A_host, B_host, N, workspace, a_fused, s);
  if (st != BATQ_OK) return st;
  // Pass 1 measures the amax of the fused weights, pass 2 quantises them with
  // gs = 448 * 6 / amax and publishes gs.
  unsigned* amax_word = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + base);
  if (cudaMemsetAsync(amax_word, 0, sizeof(unsigned), s) != cudaSuccess) return BATQ_ERR_CUDA;
  const float* b_fused = reinterpret_cast<const float*>(workspace);
  st = launch_quant(W, w_dtype, M, N, ldw, a_fused, b_fused, nullptr, w_codes, w_scales, layout, nullptr,
                    batq::kFmtNvfp4, s, nullptr, nullptr, nullptr, amax_word);
  if (st != BATQ_OK) return st;
  return launch_quant(W, w_dtype, M, N, ldw, a_fused, b_fused, nullptr, w_codes, w_scales, layout, nullptr,
                      batq::kFmtNvfp4, s, nullptr, amax_word, gs_out_dev, nullptr);
}

batq_status batq_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_gs_dev,
                            const uint8_t* w_codes, const uint8_t* w_scales, const float* w_gs_dev, int S, int M,
                            int N, batq_dtype out_dtype, void* out, int ldo, void* stream) {
  batq_status st = check_gemm_args(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  if ((a_gs_dev && !aligned4(a_gs_dev)) || (w_gs_dev && !aligned4(w_gs_dev))) return BATQ_ERR_ALIGNMENT;
  st = check_arch();
  if (st != BATQ_OK) return st;
  return launch_gemm(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo, false, batq::kFmtNvfp4,
                     static_cast<cudaStream_t>(stream), a_gs_dev, w_gs_dev);
}

batq_status batq_linear_nvfp4_workspace_size(int S, int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_mn(S, N);
  if (st != BATQ_OK) return st;
  *bytes = round_up((size_t)S * (size_t)(N / 2), 256) + nv_scale_bytes_for(S, N, BATQ_SCALES_MMA);
  return BATQ_OK;
}

batq_status batq_linear_nvfp4(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                              const float* B_dev, const float* ratios_dev, const float* a_gs_dev,
                              const uint8_t* w_codes, const uint8_t* w_scales, const float* w_gs_dev, int M,
                              void* workspace, size_t workspace_bytes, batq_dtype out_dtype, void* out, int ldo,
                              void* stream) {
  if (!workspace) return BATQ_ERR_INVALID_ARG;
  size_t need = 0;
  batq_status st = batq_linear_nvfp4_workspace_size(S, N, &need);
  if (st != BATQ_OK) return st;
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BATQ_ERR_ALIGNMENT;
  uint8_t* a_codes = static_cast<uint8_t*>(workspace);
  uint8_t* a_scales = a_codes + round_up((size_t)S * (size_t)(N / 2), 256);
  st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA,
                        nullptr);
  if (st != BATQ_OK) return st;
  st = check_gemm_args(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  if ((a_gs_dev && !aligned4(a_gs_dev)) || (w_gs_dev && !aligned4(w_gs_dev))) return BATQ_ERR_ALIGNMENT;
  st = check_arch();
  if (st != BATQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_quant(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA, nullptr,
                    batq::kFmtNvfp4, s, a_gs_dev);
  if (st != BATQ_OK) return st;
  return launch_gemm(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo, true, batq::kFmtNvfp4, s,
                     a_gs_dev, w_gs_dev);
}

// ------------------------------------------------------------------ naive Kronecker (per-block A_i)

batq_status batq_quant_act_kron(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_blocks_dev,
                                const float* B_dev, const float* ratios_dev, uint8_t* codes, uint8_t* scales,
                                batq_scale_layout layout, float* y_debug, void* stream) {
  if (!A_blocks_dev) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_quant_args(X, x_dtype, S, N, ldx, kUnusedA, B_dev, ratios_dev, codes, scales, layout,
                                    y_debug);
  if (st != BATQ_OK) return st;
  if (!aligned16(A_blocks_dev)) return BATQ_ERR_ALIGNMENT;
  st = check_arch();
  if (st != BATQ_OK) return st;
  return launch_quant(X, x_dtype, S, N, ldx, kUnusedA, B_dev, ratios_dev, codes, scales, layout, y_debug,
                      batq::kFmtMxfp4, static_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, nullptr,
                      A_blocks_dev);
}

batq_status batq_prepare_weights_kron_workspace_size(int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  size_t base = 0;
  batq_status st = batq_prepare_workspace_size(N, &base);
  if (st != BATQ_OK) return st;
  *bytes = base + round_up((size_t)(N / 32) * 64 * sizeof(float), 256);
  return BATQ_OK;
}

batq_status batq_prepare_weights_kron(const void* W, batq_dtype w_dtype, int M, int N, int ldw,
                                      const float* A_blocks_host, const float* B_host, uint8_t* w_codes,
                                      uint8_t* w_scales, batq_scale_layout layout, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!A_blocks_host || !B_host || !workspace) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_quant_args(W, w_dtype, M, N, ldw, kUnusedA, reinterpret_cast<const float*>(workspace),
                                    nullptr, w_codes, w_scales, layout, nullptr);
  if (st != BATQ_OK) return st;
  size_t need = 0, base = 0;
  batq_prepare_weights_kron_workspace_size(N, &need);
  batq_prepare_workspace_size(N, &base);
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  st = check_arch();
  if (st != BATQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = fused_transform_kron(A_blocks_host, B_host, N, workspace, base, s);
  if (st != BATQ_OK) return st;
  const float* a_fused = reinterpret_cast<const float*>(static_cast<uint8_t*>(workspace) + base);
  return launch_quant(W, w_dtype, M, N, ldw, kUnusedA, reinterpret_cast<const float*>(workspace), nullptr, w_codes,
                      w_scales, layout, nullptr, batq::kFmtMxfp4, s, nullptr, nullptr, nullptr, nullptr, a_fused);
}

batq_status batq_linear_kron(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_blocks_dev,
                             const float* B_dev, const float* ratios_dev, const uint8_t* w_codes,
                             const uint8_t* w_scales, int M, void* workspace, size_t workspace_bytes,
                             batq_dtype out_dtype, void* out, int ldo, void* stream) {
  if (!workspace || !A_blocks_dev) return BATQ_ERR_INVALID_ARG;
  size_t need = 0;
  batq_status st = batq_linear_workspace_size(S, N, &need);
  if (st != BATQ_OK) return st;
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace) || !aligned16(A_blocks_dev)) return BATQ_ERR_ALIGNMENT;
  uint8_t* a_codes = static_cast<uint8_t*>(workspace);
  uint8_t* a_scales = a_codes + round_up((size_t)S * (N / 2), 256);
  st = check_quant_args(X, x_dtype, S, N, ldx, kUnusedA, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA,
                        nullptr);
  if (st != BATQ_OK) return st;
  st = check_gemm_args(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_quant(X, x_dtype, S, N, ldx, kUnusedA, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA, nullptr,
                    batq::kFmtMxfp4, s, nullptr, nullptr, nullptr, nullptr, A_blocks_dev);
  if (st != BATQ_OK) return st;
  return launch_gemm(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo, true, batq::kFmtMxfp4, s);
}

// ------------------------------------------------------------------ KV cache

batq_status batq_quant_kv_cache(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* A_host,
                                const float* B_dev, const float* ratios_dev, const int* slot_mapping_dev,
                                int num_slots, batq_kv_format kv_format, uint8_t* cache_codes,
                                uint8_t* cache_scales, void* stream) {
  if (!slot_mapping_dev || num_slots < 1) return BATQ_ERR_INVALID_ARG;
  if (kv_format != BATQ_KV_MXFP4 && kv_format != BATQ_KV_MXFP8) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, cache_codes, cache_scales,
                                    BATQ_SCALES_LINEAR, nullptr);
  if (st != BATQ_OK) return st;
  if (!aligned4(slot_mapping_dev)) return BATQ_ERR_ALIGNMENT;
  st = check_arch();
  if (st != BATQ_OK) return st;
  batq::QuantLaunch L;
  L.X = X;
  L.bf16 = (x_dtype == BATQ_BF16);
  L.S = S;
  L.N = N;
  L.ldx = ldx;
  std::memcpy(L.A, A_host, sizeof(L.A));
  L.B = B_dev;
  L.ratios = ratios_dev;
  L.codes = cache_codes;
  L.scales = cache_scales;
  L.mma_layout = false;
  L.y_debug = nullptr;
  L.err = error_word();
  L.stream = static_cast<cudaStream_t>(stream);
  L.fmt = kv_format == BATQ_KV_MXFP8 ? batq::kFmtMxfp8 : batq::kFmtMxfp4;
  L.row_map = slot_mapping_dev;
  L.num_slots = num_slots;
  cudaError_t e = batq::launch_quant_act(L);
  if (e == cudaErrorInvalidValue) return BATQ_ERR_ALIGNMENT;
  return e == cudaSuccess ? BATQ_OK : BATQ_ERR_CUDA;
}

batq_status batq_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000u) return BATQ_ERR_INVALID_ARG;
  batq_status st = check_arch();
  if (st != BATQ_OK) return st;
  unsigned* err = error_word();
  if (!err) return BATQ_ERR_CUDA;
  cudaError_t e = batq::launch_wait_selftest((uint64_t)limit_us * 1000ull, err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BATQ_OK : BATQ_ERR_CUDA;
}

batq_status batq_device_error(void* stream, unsigned int* flags_out) {
  if (!flags_out) return BATQ_ERR_INVALID_ARG;
  unsigned* word = error_word();
  if (!word) return BATQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BATQ_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return BATQ_ERR_CUDA;
  if (v != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return BATQ_ERR_CUDA;
  }
  *flags_out = v;
  return v ? BATQ_ERR_TIMEOUT : BATQ_OK;
}

}  // extern "C"

// ------------------------------------------------------ RMSNorm ahead of the transform

extern "C" {

batq_status batq_rmsnorm_workspace_size(int S, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  if (S < 1) return BATQ_ERR_SHAPE;
  *bytes = rms_bytes_for(S);
  return BATQ_OK;
}

batq_status batq_rmsnorm_quant_act(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* gamma_dev,
                                   float eps, const float* A_host, const float* B_dev, const float* ratios_dev,
                                   uint8_t* codes, uint8_t* scales, batq_scale_layout layout, void* workspace,
                                   size_t workspace_bytes, float* y_debug, void* stream) {
  batq_status st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, codes, scales, layout,
                                    y_debug);
  if (st != BATQ_OK) return st;
  st = check_rmsnorm_args(gamma_dev, eps);
  if (st != BATQ_OK) return st;
  if (!workspace) return BATQ_ERR_INVALID_ARG;
  if (workspace_bytes < rms_bytes_for(S)) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BATQ_ERR_ALIGNMENT;
  st = check_arch();
  if (st != BATQ_OK) return st;
  return launch_rmsnorm_quant(X, x_dtype, S, N, ldx, gamma_dev, eps, A_host, B_dev, ratios_dev, codes, scales,
                              layout, static_cast<float*>(workspace), y_debug, static_cast<cudaStream_t>(stream));
}

batq_status batq_rmsnorm_linear_workspace_size(int S, int N, size_t* bytes) {
  if (!bytes) return BATQ_ERR_INVALID_ARG;
  size_t lin = 0;
  batq_status st = batq_linear_workspace_size(S, N, &lin);
  if (st != BATQ_OK) return st;
  *bytes = round_up(lin, 256) + rms_bytes_for(S);
  return BATQ_OK;
}

batq_status batq_rmsnorm_linear(const void* X, batq_dtype x_dtype, int S, int N, int ldx, const float* gamma_dev,
                                float eps, const float* A_host, const float* B_dev, const float* ratios_dev,
                                const uint8_t* w_codes, const uint8_t* w_scales, int M, void* workspace,
                                size_t workspace_bytes, batq_dtype out_dtype, void* out, int ldo, void* stream) {
  if (!workspace) return BATQ_ERR_INVALID_ARG;
  size_t need = 0, lin = 0;
  batq_status st = batq_rmsnorm_linear_workspace_size(S, N, &need);
  if (st != BATQ_OK) return st;
  batq_linear_workspace_size(S, N, &lin);
  if (workspace_bytes < need) return BATQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BATQ_ERR_ALIGNMENT;
  uint8_t* a_codes = static_cast<uint8_t*>(workspace);
  uint8_t* a_scales = a_codes + round_up((size_t)S * (N / 2), 256);
  float* rms = reinterpret_cast<float*>(a_codes + round_up(lin, 256));
  st = check_quant_args(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, a_codes, a_scales, BATQ_SCALES_MMA,
                        nullptr);
  if (st != BATQ_OK) return st;
  st = check_rmsnorm_args(gamma_dev, eps);
  if (st != BATQ_OK) return st;
  st = check_gemm_args(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo);
  if (st != BATQ_OK) return st;
  st = check_arch();
  if (st != BATQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_rmsnorm_quant(X, x_dtype, S, N, ldx, gamma_dev, eps, A_host, B_dev, ratios_dev, a_codes, a_scales,
                            BATQ_SCALES_MMA, rms, nullptr, s);
  if (st != BATQ_OK) return st;
  // As in batq_linear: the quantiser writes only the workspace, so the GEMM
  // may fetch weights while it runs.
  return launch_gemm(a_codes, a_scales, w_codes, w_scales, S, M, N, out_dtype, out, ldo, true, batq::kFmtMxfp4, s);
}

}  // extern "C"
