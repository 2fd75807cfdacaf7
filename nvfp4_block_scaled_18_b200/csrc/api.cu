// C-ABI entry points declared in include/nvfp4.h: argument validation on the
// host, then kernel launches on the caller's stream.  No allocation, no
// global state beyond a per-device SM-count cache and the bounded-wait test
// setting.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4.h"

using namespace nvfp4;

namespace {

std::atomic<uint64_t> g_wait_limit_ns{tc_wait_default_ns()};
std::atomic<int> g_wait_hold{0};

int num_sms_current_device() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cache[dev] = n;
  return n;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dt_size(nvfp4_dtype dt) { return dt == NVFP4_BF16 ? 2 : 4; }
inline bool dt_ok(nvfp4_dtype dt) { return dt == NVFP4_BF16 || dt == NVFP4_F32; }

nvfp4_status check_input(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx) {
  if (x == nullptr || !dt_ok(dt) || M <= 0 || K <= 0 || ldx < K) return NVFP4_ERR_INVALID_ARG;
  if (K % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || ((size_t)ldx * dt_size(dt)) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

nvfp4_status check_tensor(const nvfp4_tensor* t, int64_t rows, int64_t cols) {
  if (t == nullptr || t->codes == nullptr || t->scales == nullptr || t->tensor_scale == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (t->rows != rows || t->cols != cols || cols % 16 != 0 || rows <= 0) return NVFP4_ERR_INVALID_ARG;
  if (t->sf_layout != NVFP4_SF_ROWMAJOR && t->sf_layout != NVFP4_SF_TILED) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(t->codes) || !aligned16(t->scales) || (reinterpret_cast<uintptr_t>(t->tensor_scale) & 3u))
    return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

QOut qout(const nvfp4_tensor* t) {
  return QOut{t->codes, t->scales, t->tensor_scale, t->cols, t->sf_layout == NVFP4_SF_TILED};
}

nvfp4_status check_ws(const void* ws, size_t ws_bytes, int64_t M, int64_t K) {
  if (ws == nullptr || ws_bytes < nvfp4_workspace_size(M, K)) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(ws)) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

inline nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

#define NVFP4_TRY(expr)                       \
  do {                                        \
    nvfp4_status _s = (expr);                 \
    if (_s != NVFP4_OK) return _s;            \
  } while (0)

nvfp4_status check_gemm_operands(const nvfp4_tensor* a, const nvfp4_tensor* r, const nvfp4_tensor* w,
                                 const void* y, nvfp4_dtype out_dt, int64_t ldy) {
  if (a == nullptr || w == nullptr || y == nullptr || !dt_ok(out_dt)) return NVFP4_ERR_INVALID_ARG;
  const int64_t M = a->rows, K = a->cols, N = w->rows;
  NVFP4_TRY(check_tensor(a, M, K));
  NVFP4_TRY(check_tensor(w, N, K));
  if (r != nullptr) {
    NVFP4_TRY(check_tensor(r, M, K));
    if (r->sf_layout != a->sf_layout) return NVFP4_ERR_UNSUPPORTED;
  }
  if (ldy < N) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(y) % dt_size(out_dt)) != 0) return NVFP4_ERR_ALIGNMENT;
  if (K % 64 != 0) return NVFP4_ERR_UNSUPPORTED;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return NVFP4_ERR_UNSUPPORTED;  // 32-bit in the kernels
  return NVFP4_OK;
}

nvfp4_status run_gemm(const nvfp4_tensor* a, const nvfp4_tensor* r, const nvfp4_tensor* w, void* y,
                      nvfp4_dtype out_dt, int64_t ldy, int* dev_status, void* stream) {
  NVFP4_TRY(check_gemm_operands(a, r, w, y, out_dt, ldy));
  GemmArgs g{};
  g.a_codes = a->codes; g.a_scales = a->scales; g.a_s = a->tensor_scale;
  if (r) { g.r_codes = r->codes; g.r_scales = r->scales; g.r_s = r->tensor_scale; }
  g.w_codes = w->codes; g.w_scales = w->scales; g.w_s = w->tensor_scale;
  g.y = y; g.ldy = ldy; g.y_bf16 = out_dt == NVFP4_BF16;
  g.M = a->rows; g.N = w->rows; g.K = a->cols; g.st = dev_status;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tiled = a->sf_layout == NVFP4_SF_TILED && w->sf_layout == NVFP4_SF_TILED;
  const bool rowmajor = a->sf_layout == NVFP4_SF_ROWMAJOR && w->sf_layout == NVFP4_SF_ROWMAJOR;
  cudaError_t e;
  if (rowmajor && g.M <= 16) {
    e = launch_gemv(g, num_sms_current_device(), s);              // CUDA-core decode GEMV
  } else if (w->sf_layout == NVFP4_SF_TILED && g.M <= 16) {
    DecodeArgs d{};                                               // tensor-core decode kernel
    d.x_codes = a->codes; d.x_scales = a->scales; d.x_s = a->tensor_scale;
    if (r) { d.r_codes = r->codes; d.r_scales = r->scales; d.r_s = r->tensor_scale; }
    d.x_tiled = a->sf_layout == NVFP4_SF_TILED;
    d.w_codes = w->codes; d.w_scales = w->scales; d.w_s = w->tensor_scale;
    d.y = y; d.ldy = ldy; d.y_bf16 = out_dt == NVFP4_BF16;
    d.M = g.M; d.N = g.N; d.K = g.K; d.st = dev_status;
    e = launch_decode_tc(d, num_sms_current_device(), s);
  } else if (tiled && g.M <= 128) {
    e = launch_gemv_tc(g, num_sms_current_device(), s);           // tensor cores, operands swapped
  } else if (tiled) {
    e = launch_gemm_tc(g, num_sms_current_device(), s);           // tensor cores, 128x256 tiles
  } else {
    return NVFP4_ERR_UNSUPPORTED;
  }
  if (e == cudaErrorNotSupported) return NVFP4_ERR_UNSUPPORTED;
  return cuda_status(e);
}

nvfp4_status run_mx_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* r_codes,
                         const uint8_t* r_scales, const uint8_t* w_codes, const uint8_t* w_scales, int64_t M,
                         int64_t N, int64_t K, void* y, nvfp4_dtype out_dt, int64_t ldy, int* dev_status,
                         void* stream) {
  if (a_codes == nullptr || a_scales == nullptr || w_codes == nullptr || w_scales == nullptr || y == nullptr ||
      !dt_ok(out_dt))
    return NVFP4_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || ldy < N || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
    return NVFP4_ERR_INVALID_ARG;
  if (K % 128 != 0 || K < 256) return NVFP4_ERR_UNSUPPORTED;
  if (!aligned16(a_codes) || !aligned16(w_codes) || !aligned16(a_scales) || !aligned16(w_scales))
    return NVFP4_ERR_ALIGNMENT;
  if (r_codes != nullptr && (!aligned16(r_codes) || !aligned16(r_scales))) return NVFP4_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(y) % dt_size(out_dt)) != 0) return NVFP4_ERR_ALIGNMENT;
  GemmArgs g{};
  g.a_codes = a_codes; g.a_scales = a_scales;
  g.r_codes = r_codes; g.r_scales = r_scales;
  g.w_codes = w_codes; g.w_scales = w_scales;
  g.y = y; g.ldy = ldy; g.y_bf16 = out_dt == NVFP4_BF16;
  g.M = M; g.N = N; g.K = K; g.st = dev_status;
  const cudaError_t e = launch_gemm_mx(g, num_sms_current_device(), static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return NVFP4_ERR_UNSUPPORTED;
  return cuda_status(e);
}

}  // namespace

namespace nvfp4 {
WaitTest wait_test() { return WaitTest{g_wait_limit_ns.load(), g_wait_hold.load()}; }
}  // namespace nvfp4

extern "C" {

void nvfp4_test_wait_fault(uint64_t limit_ns, int withhold) {
  g_wait_limit_ns.store(limit_ns == 0 ? tc_wait_default_ns() : limit_ns);
  g_wait_hold.store(withhold != 0 ? 1 : 0);
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout) {
  if (rows <= 0 || cols <= 0) return 0;
  if (layout == NVFP4_SF_TILED) return (size_t)((rows + 127) / 128) * (size_t)((cols + 63) / 64) * 512;
  return (size_t)rows * (size_t)((cols + 15) / 16);
}

size_t nvfp4_workspace_size(int64_t M, int64_t K) {
  (void)K;
  if (M <= 0) return kWsHeaderBytes;
  return kWsHeaderBytes + (((size_t)M * 4 + 255) / 256) * 256;
}

nvfp4_status nvfp4_quantize(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                            const float* scale_in, nvfp4_tensor* q, void* workspace,
                            size_t ws_bytes, int* dev_status, void* stream) {
  NVFP4_TRY(check_input(x, dt, M, K, ldx));
  NVFP4_TRY(check_tensor(q, M, K));
  if (scale_in == nullptr) NVFP4_TRY(check_ws(workspace, ws_bytes, M, K));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms_current_device();
  WsHeader* ws = static_cast<WsHeader*>(workspace);
  const QOut qo = qout(q);
  if (M * (K / 8) <= quant_small_max_units(dt))   // decode-sized: one launch, no workspace traffic
    return cuda_status(launch_quant_small(false, x, dt, M, K, ldx, scale_in, nullptr, qo, qo, dev_status, s));
  const float* s_ptr = scale_in;
  if (s_ptr == nullptr) {
    NVFP4_TRY(cuda_status(launch_amax(x, dt, M, K, ldx, ws, 0, q->tensor_scale, dev_status, sms, s)));
    s_ptr = q->tensor_scale;
  }
  return cuda_status(launch_quant(Q_PLAIN, x, dt, M, K, ldx, s_ptr, nullptr, qo, qo, ws, dev_status, sms, s,
                                  scale_in == nullptr));
}

nvfp4_status nvfp4_quantize_residue(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                    const float* scale_in, const float* rscale_in, nvfp4_tensor* q,
                                    nvfp4_tensor* r, void* workspace, size_t ws_bytes,
                                    int* dev_status, void* stream) {
  NVFP4_TRY(check_input(x, dt, M, K, ldx));
  NVFP4_TRY(check_tensor(q, M, K));
  NVFP4_TRY(check_tensor(r, M, K));
  if (scale_in == nullptr || rscale_in == nullptr) NVFP4_TRY(check_ws(workspace, ws_bytes, M, K));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms_current_device();
  WsHeader* ws = static_cast<WsHeader*>(workspace);
  const QOut qo = qout(q), ro = qout(r);
  if (M * (K / 8) <= quant_small_max_units(dt))
    return cuda_status(launch_quant_small(true, x, dt, M, K, ldx, scale_in, rscale_in, qo, ro, dev_status, s));
  const float* s_ptr = scale_in;
  if (s_ptr == nullptr) {
    NVFP4_TRY(cuda_status(launch_amax(x, dt, M, K, ldx, ws, 0, q->tensor_scale, dev_status, sms, s)));
    s_ptr = q->tensor_scale;
  }
  if (rscale_in != nullptr)
    return cuda_status(launch_quant(Q_BOTH, x, dt, M, K, ldx, s_ptr, rscale_in, qo, ro, ws, dev_status, sms, s,
                                    scale_in == nullptr));
  NVFP4_TRY(cuda_status(launch_quant(Q_MAIN_AMAXR, x, dt, M, K, ldx, s_ptr, nullptr, qo, ro, ws, dev_status, sms,
                                     s, scale_in == nullptr)));
  return cuda_status(launch_quant(Q_RES_ONLY, x, dt, M, K, ldx, s_ptr, r->tensor_scale, qo, ro, ws, dev_status, sms, s));
}

nvfp4_status nvfp4_rmsnorm_reorder_quantize(const void* x, nvfp4_dtype dt, int64_t M, int64_t K,
                                            int64_t ldx, const void* gamma, float eps,
                                            const int32_t* perm, int64_t S, const float* scale_in,
                                            nvfp4_tensor* x_aug, void* workspace, size_t ws_bytes,
                                            int* dev_status, void* stream) {
  NVFP4_TRY(check_input(x, dt, M, K, ldx));
  if (S < 0 || S > K || S % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  NVFP4_TRY(check_tensor(x_aug, M, K + S));
  if (gamma != nullptr && !aligned16(gamma)) return NVFP4_ERR_ALIGNMENT;
  if (gamma != nullptr && !(eps >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (gamma != nullptr || scale_in == nullptr) NVFP4_TRY(check_ws(workspace, ws_bytes, M, K));
  if (reorder_smem_bytes(dt, K, gamma != nullptr) > 200 * 1024) return NVFP4_ERR_UNSUPPORTED;
  if (K > 65536) return NVFP4_ERR_UNSUPPORTED;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms_current_device();
  WsHeader* ws = static_cast<WsHeader*>(workspace);
  float* rinv = workspace ? reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsHeaderBytes) : nullptr;
  if (gamma != nullptr || scale_in == nullptr) {
    // small enough for one launch: X read once, no second pass
    const cudaError_t e = launch_reorder_onepass(x, dt, M, K, ldx, gamma, eps, perm, S, scale_in, qout(x_aug), ws,
                                                 dev_status, sms, s);
    if (e != cudaErrorNotSupported) return cuda_status(e);
  }
  if (gamma != nullptr) {
    NVFP4_TRY(cuda_status(launch_rms_stats(x, dt, M, K, ldx, gamma, eps, ws, rinv, x_aug->tensor_scale,
                                           scale_in == nullptr, dev_status, sms, s)));
  } else if (scale_in == nullptr) {
    NVFP4_TRY(cuda_status(launch_amax(x, dt, M, K, ldx, ws, 0, x_aug->tensor_scale, dev_status, sms, s)));
  }
  const float* s_ptr = scale_in ? scale_in : x_aug->tensor_scale;
  // a programmatic dependent of the statistics pass, when there is one
  return cuda_status(launch_reorder_quant(x, dt, M, K, ldx, gamma, rinv, perm, S, s_ptr, qout(x_aug),
                                          dev_status, sms, s, gamma != nullptr || scale_in == nullptr));
}

nvfp4_status nvfp4_quantize_weight(const void* w, nvfp4_dtype dt, int64_t N, int64_t K, int64_t ldw,
                                   const float* sigma, const int32_t* perm, int64_t S, const float* scale_in,
                                   nvfp4_tensor* w_aug, void* workspace, size_t ws_bytes, int* dev_status,
                                   void* stream) {
  if (w == nullptr || !dt_ok(dt) || N <= 0 || K <= 0 || ldw < K || K % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(w) % dt_size(dt)) != 0) return NVFP4_ERR_ALIGNMENT;
  if (S < 0 || S > K || S % 16 != 0) return NVFP4_ERR_INVALID_ARG;
  if ((sigma != nullptr && (reinterpret_cast<uintptr_t>(sigma) & 3u)) ||
      (perm != nullptr && (reinterpret_cast<uintptr_t>(perm) & 3u)))
    return NVFP4_ERR_ALIGNMENT;
  NVFP4_TRY(check_tensor(w_aug, N, K + S));
  if (scale_in == nullptr) NVFP4_TRY(check_ws(workspace, ws_bytes, N, K));
  return cuda_status(launch_weight_quant(w, dt, N, K, ldw, sigma, perm, S, scale_in, qout(w_aug),
                                         static_cast<WsHeader*>(workspace), dev_status, num_sms_current_device(),
                                         static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor* a, const nvfp4_tensor* w, void* y, nvfp4_dtype out_dt,
                        int64_t ldy, int* dev_status, void* stream) {
  return run_gemm(a, nullptr, w, y, out_dt, ldy, dev_status, stream);
}

nvfp4_status nvfp4_gemm_residue(const nvfp4_tensor* a, const nvfp4_tensor* r, const nvfp4_tensor* w,
                                void* y, nvfp4_dtype out_dt, int64_t ldy, int* dev_status,
                                void* stream) {
  if (r == nullptr) return NVFP4_ERR_INVALID_ARG;
  return run_gemm(a, r, w, y, out_dt, ldy, dev_status, stream);
}

nvfp4_status nvfp4_quantize_residue_gemm(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                         const float* scale_in, const float* rscale_in, nvfp4_tensor* q,
                                         nvfp4_tensor* r, const nvfp4_tensor* w, void* y, nvfp4_dtype out_dt,
                                         int64_t ldy, int* dev_status, void* stream) {
  NVFP4_TRY(check_input(x, dt, M, K, ldx));
  NVFP4_TRY(check_tensor(q, M, K));
  if (r != nullptr) {
    NVFP4_TRY(check_tensor(r, M, K));
    if (r->sf_layout != q->sf_layout) return NVFP4_ERR_UNSUPPORTED;
  }
  NVFP4_TRY(check_gemm_operands(q, r, w, y, out_dt, ldy));
  if (M > 16 || w->sf_layout != NVFP4_SF_TILED || K < 256) return NVFP4_ERR_UNSUPPORTED;
  if (M * (K / 8) > quant_small_max_units(dt)) return NVFP4_ERR_UNSUPPORTED;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms_current_device();
  DecodeArgs d{};
  d.x = x; d.x_bf16 = dt == NVFP4_BF16; d.ldx = ldx;
  d.s_in = scale_in; d.sr_in = r ? rscale_in : nullptr;
  d.q_out = qout(q);
  if (r) d.r_out = qout(r);
  d.w_codes = w->codes; d.w_scales = w->scales; d.w_s = w->tensor_scale;
  d.y = y; d.ldy = ldy; d.y_bf16 = out_dt == NVFP4_BF16;
  d.M = M; d.N = w->rows; d.K = K; d.st = dev_status;
  cudaError_t e = launch_decode_tc(d, sms, s);
  if (e != cudaErrorNotSupported) return cuda_status(e);
  // the activation slice does not fit the fused kernel's registers: quantize
  // in one launch, then run the same kernel on the NVFP4 operands
  const QOut qo = qout(q), ro = r ? qout(r) : qout(q);
  NVFP4_TRY(cuda_status(launch_quant_small(r != nullptr, x, dt, M, K, ldx, scale_in, d.sr_in, qo, ro,
                                           dev_status, s)));
  return run_gemm(q, r, w, y, out_dt, ldy, dev_status, stream);
}

int nvfp4_quantize_gemm_plan(int64_t M, int64_t N, int64_t K, nvfp4_dtype dt, int residue, nvfp4_dtype out_dt) {
  if (M < 1 || M > 16 || N < 1 || N > INT32_MAX || K < 256 || K > INT32_MAX || K % 64 != 0 || !dt_ok(dt) ||
      !dt_ok(out_dt))
    return 0;
  if (M * (K / 8) > quant_small_max_units(dt)) return 0;
  static const uint8_t dummy[16] = {0};
  DecodeArgs d{};
  d.x = dummy; d.x_bf16 = dt == NVFP4_BF16; d.ldx = K;
  d.q_out = QOut{const_cast<uint8_t*>(dummy), const_cast<uint8_t*>(dummy), nullptr, K, true};
  if (residue) d.r_out = d.q_out;
  d.w_codes = dummy; d.w_scales = dummy;
  d.y_bf16 = out_dt == NVFP4_BF16;
  d.M = M; d.N = N; d.K = K; d.dry_run = true;
  const cudaError_t e = launch_decode_tc(d, num_sms_current_device(), nullptr);
  if (e == cudaSuccess) return 1;
  if (e != cudaErrorNotSupported) return 0;
  d.x = nullptr;                       // quantize, then the decode kernel on NVFP4 operands
  d.x_codes = dummy; d.x_scales = dummy; d.x_tiled = true;
  if (residue) { d.r_codes = dummy; d.r_scales = dummy; }
  d.r_out = QOut{};
  return launch_decode_tc(d, num_sms_current_device(), nullptr) == cudaSuccess ? 2 : 0;
}

nvfp4_status nvfp4_quantize_gemm(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                 const float* scale_in, nvfp4_tensor* q, const nvfp4_tensor* w, void* y,
                                 nvfp4_dtype out_dt, int64_t ldy, int* dev_status, void* stream) {
  return nvfp4_quantize_residue_gemm(x, dt, M, K, ldx, scale_in, nullptr, q, nullptr, w, y, out_dt, ldy,
                                     dev_status, stream);
}

nvfp4_status nvfp4_quantize_gemm_host(const void* x_host, void* x_dev, nvfp4_dtype dt, int64_t M, int64_t K,
                                      int64_t ldx, const float* scale_in, nvfp4_tensor* q,
                                      const nvfp4_tensor* w, void* y_dev, void* y_host, nvfp4_dtype out_dt,
                                      int64_t ldy, int* dev_status, void* stream) {
  if (x_host == nullptr || y_host == nullptr) return NVFP4_ERR_INVALID_ARG;
  NVFP4_TRY(check_input(x_dev, dt, M, K, ldx));
  NVFP4_TRY(check_tensor(q, M, K));
  NVFP4_TRY(check_gemm_operands(q, nullptr, w, y_dev, out_dt, ldy));
  if (M > 16 || w->sf_layout != NVFP4_SF_TILED || K < 256) return NVFP4_ERR_UNSUPPORTED;
  if (M * (K / 8) > quant_small_max_units(dt)) return NVFP4_ERR_UNSUPPORTED;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t es = dt_size(dt), oes = dt_size(out_dt), N = (size_t)w->rows;
  NVFP4_TRY(cuda_status(cudaMemcpy2DAsync(x_dev, (size_t)ldx * es, x_host, (size_t)K * es, (size_t)K * es,
                                          (size_t)M, cudaMemcpyHostToDevice, s)));
  NVFP4_TRY(nvfp4_quantize_gemm(x_dev, dt, M, K, ldx, scale_in, q, w, y_dev, out_dt, ldy, dev_status, stream));
  return cuda_status(cudaMemcpy2DAsync(y_host, N * oes, y_dev, (size_t)ldy * oes, N * oes, (size_t)M,
                                       cudaMemcpyDeviceToHost, s));
}

size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout) {
  if (rows <= 0 || cols <= 0) return 0;
  const int64_t nb = (cols + 31) / 32;
  if (layout == NVFP4_SF_TILED) return (size_t)((rows + 127) / 128) * (size_t)((nb + 3) / 4) * 512;
  return (size_t)rows * (size_t)nb;
}

nvfp4_status nvfp4_mx_quantize(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                               uint8_t* codes, uint8_t* scales, uint8_t* r_codes, uint8_t* r_scales,
                               nvfp4_sf_layout sf_layout, int* dev_status, void* stream) {
  NVFP4_TRY(check_input(x, dt, M, K, ldx));
  if (K % 32 != 0 || codes == nullptr || scales == nullptr) return NVFP4_ERR_INVALID_ARG;
  if ((r_codes == nullptr) != (r_scales == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_TILED) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(codes) || (r_codes != nullptr && !aligned16(r_codes))) return NVFP4_ERR_ALIGNMENT;
  return cuda_status(launch_mx_quant(x, dt, M, K, ldx, codes, scales, r_codes, r_scales,
                                     sf_layout == NVFP4_SF_TILED, dev_status, num_sms_current_device(),
                                     static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_mx_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                           const uint8_t* w_scales, int64_t M, int64_t N, int64_t K, void* y,
                           nvfp4_dtype out_dt, int64_t ldy, int* dev_status, void* stream) {
  return run_mx_gemm(a_codes, a_scales, nullptr, nullptr, w_codes, w_scales, M, N, K, y, out_dt, ldy, dev_status,
                     stream);
}

nvfp4_status nvfp4_mx_gemm_residue(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* r_codes,
                                   const uint8_t* r_scales, const uint8_t* w_codes, const uint8_t* w_scales,
                                   int64_t M, int64_t N, int64_t K, void* y, nvfp4_dtype out_dt, int64_t ldy,
                                   int* dev_status, void* stream) {
  if (r_codes == nullptr || r_scales == nullptr) return NVFP4_ERR_INVALID_ARG;
  return run_mx_gemm(a_codes, a_scales, r_codes, r_scales, w_codes, w_scales, M, N, K, y, out_dt, ldy, dev_status,
                     stream);
}

const char* nvfp4_status_string(nvfp4_status st) {
  switch (st) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported shape or layout";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_NONFINITE: return "non-finite input";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* nvfp4_version(void) { return "nvfp4 0.1 sm_100a"; }

}  // extern "C"
