// api.cu -- the extern "C" entry points declared in include/awq_w4a16.h.
//
// Every entry point validates its arguments on the host and returns a status without launching
// anything when they are out of range; otherwise it enqueues the kernels on the caller's stream and
// returns.  No entry point allocates device memory.  The device status word (set by kernels whose
// bounded waits run out) is a file-scope __device__ variable; its address is looked up once per device.
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace awq {

__device__ unsigned g_device_status = 0u;

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = v > 0 ? v : 1;
  }
  return cached[dev];
}

unsigned* device_status_ptr() {
  static unsigned* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (cached[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<unsigned*>(p);
  }
  return cached[dev];
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxN = 1 << 21;   // sanity bounds on the sizes (a split linear further needs N / 32 <= 16384)
constexpr int kMaxK = 1 << 20;

static bool group_supported(int g) { return g == 64 || g == 128 || g == 256; }

awq_status check_linear(const uint16_t* x, const uint32_t* qw, const uint16_t* sc, const uint32_t* qz,
                               const uint16_t* y, int M, int N, int K, int g) {
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (M < 1 || N < 1 || K < g || K % g != 0 || N % 8 != 0 || N > kMaxN || K > kMaxK)
    return AWQ_ERR_INVALID_ARG;
  if (!x || !qw || !sc || !qz || !y) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(qw) || !aligned16(sc) || !aligned16(qz) || !aligned16(y))
    return AWQ_ERR_MISALIGNED;
  return AWQ_OK;
}

}  // namespace awq

using namespace awq;

extern "C" {

const char* awq_status_string(awq_status st) {
  switch (st) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG";
    case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED";
    case AWQ_ERR_MISALIGNED: return "AWQ_ERR_MISALIGNED";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA";
    case AWQ_ERR_DEVICE_TIMEOUT: return "AWQ_ERR_DEVICE_TIMEOUT";
    case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE";
    case AWQ_ERR_NUMERIC: return "AWQ_ERR_NUMERIC";
  }
  return "AWQ_ERR_UNKNOWN";
}

int awq_version(void) { return 100; }

awq_status awq_packed_sizes(int N, int K, int g, size_t* qweight_bytes, size_t* scales_bytes,
                            size_t* qzeros_bytes) {
  if (!qweight_bytes || !scales_bytes || !qzeros_bytes) return AWQ_ERR_INVALID_ARG;
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (N < 1 || K < 1 || K % g != 0 || N > kMaxN || K > kMaxK) return AWQ_ERR_INVALID_ARG;
  const size_t Np = (size_t)(N + 31) / 32 * 32;
  const size_t G = (size_t)K / (size_t)g;
  *qweight_bytes = Np * (size_t)K / 2;
  *scales_bytes = G * Np * 2;
  *qzeros_bytes = G * Np / 2;
  return AWQ_OK;
}

awq_status awq_act_scale(const uint16_t* d_xcal, int R, int K, uint16_t* d_s, awq_stream_t stream) {
  if (R < 1 || R > 8192 || K < 1 || K > kMaxK || !d_xcal || !d_s) return AWQ_ERR_INVALID_ARG;
  return prep_act_scale_launch(d_xcal, R, K, d_s, reinterpret_cast<cudaStream_t>(stream));
}

awq_status awq_apply_inv_scale(const uint16_t* d_x, const uint16_t* d_s, int M, int K, uint16_t* d_xp,
                               awq_stream_t stream) {
  if (M < 1 || K < 1 || K > kMaxK || !d_x || !d_s || !d_xp) return AWQ_ERR_INVALID_ARG;
  return prep_inv_scale_launch(d_x, d_s, M, K, d_xp, reinterpret_cast<cudaStream_t>(stream));
}

awq_status awq_pack(const uint16_t* d_W, const uint16_t* d_s, int N, int K, int g, uint32_t* d_qweight,
                    uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream) {
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (N < 1 || K < g || K % g != 0 || N > kMaxN || K > kMaxK) return AWQ_ERR_INVALID_ARG;
  if (!d_W || !d_qweight || !d_scales || !d_qzeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(d_W) || (d_s && !aligned16(d_s)) || !aligned16(d_qweight) || !aligned16(d_scales) ||
      !aligned16(d_qzeros))
    return AWQ_ERR_MISALIGNED;
  return pack_launch(d_W, nullptr, d_s, N, K, g, d_qweight, d_scales, d_qzeros, reinterpret_cast<cudaStream_t>(stream));
}

awq_status awq_pack_bits(const uint16_t* d_W, const uint16_t* d_s, int N, int K, int g, int w_bit, uint32_t* d_qweight,
                         uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream) {
  if (w_bit != 3 && w_bit != 4) return AWQ_ERR_UNSUPPORTED;
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (N < 1 || K < g || K % g != 0 || N > kMaxN || K > kMaxK) return AWQ_ERR_INVALID_ARG;
  if (!d_W || !d_qweight || !d_scales || !d_qzeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(d_W) || (d_s && !aligned16(d_s)) || !aligned16(d_qweight) || !aligned16(d_scales) ||
      !aligned16(d_qzeros))
    return AWQ_ERR_MISALIGNED;
  return pack_launch(d_W, nullptr, d_s, N, K, g, d_qweight, d_scales, d_qzeros, reinterpret_cast<cudaStream_t>(stream),
                     w_bit);
}

awq_status awq_packed3_sizes(int N, int K, int g, size_t* qweight_bytes, size_t* scales_bytes, size_t* qzeros_bytes) {
  awq_status st = awq_packed_sizes(N, K, g, qweight_bytes, scales_bytes, qzeros_bytes);
  if (st != AWQ_OK) return st;
  if (K % 32 != 0) return AWQ_ERR_INVALID_ARG;
  *qweight_bytes = *qweight_bytes / 4 * 3;  // 12 bytes per row per 32 channels instead of 16
  return AWQ_OK;
}

awq_status awq_pack3(const uint16_t* d_W, const uint16_t* d_s, int N, int K, int g, uint32_t* d_qweight,
                     uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream) {
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (N < 1 || K < g || K % g != 0 || N > kMaxN || K > kMaxK) return AWQ_ERR_INVALID_ARG;
  if (!d_W || !d_qweight || !d_scales || !d_qzeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(d_W) || (d_s && !aligned16(d_s)) || !aligned16(d_qweight) || !aligned16(d_scales) ||
      !aligned16(d_qzeros))
    return AWQ_ERR_MISALIGNED;
  return pack_launch(d_W, nullptr, d_s, N, K, g, d_qweight, d_scales, d_qzeros, reinterpret_cast<cudaStream_t>(stream),
                     3, 3);
}

awq_status awq_pack_gate_up(const uint16_t* d_Wgate, const uint16_t* d_Wup, const uint16_t* d_s, int NI, int K, int g,
                            uint32_t* d_qweight, uint16_t* d_scales, uint32_t* d_qzeros, awq_stream_t stream) {
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (NI < 16 || NI % 16 != 0 || 2 * (size_t)NI > (size_t)kMaxN || K < g || K % g != 0 || K > kMaxK)
    return AWQ_ERR_INVALID_ARG;
  if (!d_Wgate || !d_Wup || !d_qweight || !d_scales || !d_qzeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(d_Wgate) || !aligned16(d_Wup) || (d_s && !aligned16(d_s)) || !aligned16(d_qweight) ||
      !aligned16(d_scales) || !aligned16(d_qzeros))
    return AWQ_ERR_MISALIGNED;
  return pack_launch(d_Wgate, d_Wup, d_s, 2 * NI, K, g, d_qweight, d_scales, d_qzeros,
                     reinterpret_cast<cudaStream_t>(stream));
}

size_t w4a16_workspace_bytes(int mode, int M, int N, int K, int g) {
  if (!group_supported(g) || M < 1 || N < 1 || K < g || K % g != 0 || N % 8 != 0 || N > kMaxN || K > kMaxK)
    return SIZE_MAX;
  switch (mode) {
    case AWQ_MODE_GEMV: return gemv_workspace_bytes(M, N, K, g);
    case AWQ_MODE_GEMM: return gemm_workspace_bytes(M, N, K, g);
    case AWQ_MODE_LINEAR:
      return M <= w4a16_gemv_max_m(N, K) ? gemv_workspace_bytes(M, N, K, g) : gemm_workspace_bytes(M, N, K, g);
    default: return SIZE_MAX;
  }
}

static LinearArgs linear_args(const uint16_t* x, const uint32_t* qw, const uint16_t* sc, const uint32_t* qz,
                              uint16_t* y, int M, int N, int K, int g, void* ws, size_t ws_bytes, unsigned* status,
                              awq_stream_t stream) {
  LinearArgs a;
  a.x = x;
  a.qw = qw;
  a.scales = sc;
  a.qzeros = qz;
  a.y = y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.g = g;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.status = status;
  a.st = reinterpret_cast<cudaStream_t>(stream);
  return a;
}

awq_status w4a16_gemv(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                      const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g, void* d_workspace,
                      size_t workspace_bytes, awq_stream_t stream) {
  awq_status st = check_linear(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g);
  if (st != AWQ_OK) return st;
  if (d_workspace && !aligned16(d_workspace)) return AWQ_ERR_MISALIGNED;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  return gemv_launch(linear_args(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes,
                                 status, stream));
}

awq_status w4a16_gemv_s(const uint16_t* d_x, const uint16_t* d_s, const uint32_t* d_qweight,
                        const uint16_t* d_scales, const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g,
                        void* d_workspace, size_t workspace_bytes, awq_stream_t stream) {
  awq_status st = check_linear(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g);
  if (st != AWQ_OK) return st;
  if (d_s == nullptr) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(d_s) || (d_workspace && !aligned16(d_workspace))) return AWQ_ERR_MISALIGNED;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  LinearArgs a = linear_args(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes,
                             status, stream);
  a.inv_s = d_s;
  return gemv_launch(a);
}

awq_status w4a16_gemm(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                      const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g, void* d_workspace,
                      size_t workspace_bytes, awq_stream_t stream) {
  awq_status st = check_linear(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g);
  if (st != AWQ_OK) return st;
  if (d_workspace && !aligned16(d_workspace)) return AWQ_ERR_MISALIGNED;
  if (workspace_bytes < gemm_workspace_bytes(M, N, K, g)) return AWQ_ERR_WORKSPACE;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  return gemm_launch(linear_args(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes,
                                 status, stream));
}

// Crossover measured on B200 over the 70B-class shapes (M = 1 .. 256): the weight-streaming GEMV costs
// almost the same from M = 1 to 8 (one pass), 1.35x at M = 16 (two 8-row tiles per pass) and 2.7x at M = 32
// (two passes), and is faster than the tcgen05 GEMM through M = 32; from M = 64 the GEMM is faster.
int w4a16_gemv_max_m(int N, int K) {
  (void)N;
  (void)K;
  return 32;
}

awq_status w4a16_linear(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                        const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g, void* d_workspace,
                        size_t workspace_bytes, awq_stream_t stream) {
  if (M >= 1 && M <= w4a16_gemv_max_m(N, K))
    return w4a16_gemv(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes, stream);
  return w4a16_gemm(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes, stream);
}

awq_status w4a16_linear_pf(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                           const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g, void* d_workspace,
                           size_t workspace_bytes, const void* d_next, size_t next_bytes, awq_stream_t stream) {
  if (d_next == nullptr || next_bytes == 0 || M > w4a16_gemv_max_m(N, K))
    return w4a16_linear(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes, stream);
  if (!aligned16(d_next)) return AWQ_ERR_MISALIGNED;
  if (next_bytes % 16 != 0) return AWQ_ERR_INVALID_ARG;
  awq_status st = check_linear(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g);
  if (st != AWQ_OK) return st;
  if (d_workspace && !aligned16(d_workspace)) return AWQ_ERR_MISALIGNED;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  LinearArgs a = linear_args(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes,
                             status, stream);
  a.pf = d_next;
  a.pf_bytes = next_bytes;
  return gemv_launch(a);
}

awq_status w4a16_gate_up_silu(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                              const uint32_t* d_qzeros, uint16_t* d_h, int M, int NI, int K, int g, void* d_workspace,
                              size_t workspace_bytes, awq_stream_t stream) {
  if (NI < 16 || NI % 16 != 0 || 2 * (size_t)NI > (size_t)kMaxN) return AWQ_ERR_INVALID_ARG;
  const int N = 2 * NI;
  awq_status st = check_linear(d_x, d_qweight, d_scales, d_qzeros, d_h, M, N, K, g);
  if (st != AWQ_OK) return st;
  if (d_workspace && !aligned16(d_workspace)) return AWQ_ERR_MISALIGNED;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  LinearArgs a = linear_args(d_x, d_qweight, d_scales, d_qzeros, d_h, M, N, K, g, d_workspace, workspace_bytes,
                             status, stream);
  a.epi = 1;
  if (M <= w4a16_gemv_max_m(N, K)) return gemv_launch(a);
  if (workspace_bytes < gemm_workspace_bytes(M, N, K, g)) return AWQ_ERR_WORKSPACE;
  return gemm_launch(a);
}

awq_status w3a16_gemv(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                      const uint32_t* d_qzeros, uint16_t* d_y, int M, int N, int K, int g, void* d_workspace,
                      size_t workspace_bytes, awq_stream_t stream) {
  awq_status st = check_linear(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g);
  if (st != AWQ_OK) return st;
  if (d_workspace && !aligned16(d_workspace)) return AWQ_ERR_MISALIGNED;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  LinearArgs a = linear_args(d_x, d_qweight, d_scales, d_qzeros, d_y, M, N, K, g, d_workspace, workspace_bytes,
                             status, stream);
  a.bits = 3;
  return gemv_launch(a);
}

static bool gptq_args_ok(int N, int K, int R, int g, double damp) {
  return N >= 1 && N % 8 == 0 && N <= kMaxN && K >= 128 && K % 128 == 0 && K % g == 0 && K <= 65536 && R >= 1 &&
         R <= (1 << 24) && damp >= 0.0;
}

size_t gptq_workspace_bytes(int N, int K, int R, int g) {
  if (!group_supported(g) || !gptq_args_ok(N, K, R, g, 0.0)) return SIZE_MAX;
  return awq::gptq_workspace_bytes(N, K);
}

awq_status gptq_quantize(const uint16_t* d_W, const uint16_t* d_xcal, int N, int K, int R, int g, double damp,
                         uint32_t* d_qweight, uint16_t* d_scales, uint32_t* d_qzeros, void* d_workspace,
                         size_t workspace_bytes, awq_stream_t stream) {
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (!gptq_args_ok(N, K, R, g, damp)) return AWQ_ERR_INVALID_ARG;
  if (!d_W || !d_xcal || !d_qweight || !d_scales || !d_qzeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(d_W) || !aligned16(d_xcal) || !aligned16(d_qweight) || !aligned16(d_scales) ||
      !aligned16(d_qzeros) || (d_workspace && !aligned16(d_workspace)))
    return AWQ_ERR_MISALIGNED;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  return gptq_launch(d_W, d_xcal, N, K, R, g, damp, d_qweight, d_scales, d_qzeros, d_workspace, workspace_bytes,
                     status, reinterpret_cast<cudaStream_t>(stream));
}

static bool search_args_ok(int N, int K, int R, int g, int n_grid) {
  return N >= 1 && N % 8 == 0 && N <= kMaxN && K >= g && K % g == 0 && K <= kMaxK && R >= 1 && R <= 8192 &&
         n_grid >= 1 && n_grid <= 1000;
}

size_t awq_search_workspace_bytes(int N, int K, int R, int g, int n_grid) {
  if (!group_supported(g) || !search_args_ok(N, K, R, g, n_grid)) return SIZE_MAX;
  return search_workspace_bytes(N, K, R, g);
}

awq_status awq_search_scale(const uint16_t* d_W, const uint16_t* d_xcal, int N, int K, int R, int g, int n_grid,
                            double* d_losses, uint16_t* d_s, int32_t* d_best, void* d_workspace,
                            size_t workspace_bytes, awq_stream_t stream) {
  if (!group_supported(g)) return AWQ_ERR_UNSUPPORTED;
  if (!search_args_ok(N, K, R, g, n_grid)) return AWQ_ERR_INVALID_ARG;
  if (!d_W || !d_xcal || !d_losses || !d_s || !d_best) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(d_W) || !aligned16(d_xcal) || !aligned16(d_losses) || !aligned16(d_s) || !aligned16(d_best) ||
      (d_workspace && !aligned16(d_workspace)))
    return AWQ_ERR_MISALIGNED;
  unsigned* status = device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  return search_launch(d_W, d_xcal, N, K, R, g, n_grid, d_losses, d_s, d_best, d_workspace, workspace_bytes, status,
                       reinterpret_cast<cudaStream_t>(stream));
}

awq_status awq_last_device_status(awq_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return AWQ_ERR_CUDA;
  unsigned* p = device_status_ptr();
  if (p == nullptr) return AWQ_ERR_CUDA;
  unsigned v = 0u;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return AWQ_ERR_CUDA;
  if (v != 0u) {
    const unsigned zero = 0u;
    if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return AWQ_ERR_CUDA;
    return v == 2u ? AWQ_ERR_NUMERIC : AWQ_ERR_DEVICE_TIMEOUT;
  }
  return AWQ_OK;
}

}  // extern "C"
