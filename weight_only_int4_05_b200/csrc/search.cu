// search.cu -- awq_search_scale: the AWQ scale search run on the GPU with the library's own kernels.
//
// "AWQ and GPTQ algorithms" (jsqmd.com), section 2.1 (3): the per-channel scale s is chosen to minimise the
// layer's output error after quantization, || Q(W diag(s)) (diag(s)^-1 X) - W X ||^2, over calibration
// activations X; "LLM-AWQ academic impact" (CSDN mirror), "quantization flow": a search stage whose result
// the real-quantization stage then uses.  This library's reading: s = fp16((mean_r |X_rj|)^alpha) on the
// grid alpha_i = i / n_grid (i = 0 .. n_grid), the quantized layer as deployed (x' = fp16(x / s), packed
// weight, fp16 output), the error summed in fp64 over every calibration row and output against the exact
// unquantized X W^T, and the first grid point of least error wins.
//
// Per grid point, on the caller's stream and with no host synchronisation:
//   act_pow_kernel (s_i) -> pack_kernel (W, s_i) -> inv_scale_kernel (X / s_i) -> the linear (GEMV or GEMM
//   by the calibration row count) -> sq_err_kernel (fp64 partial sums per block) -> loss_finish_kernel
//   (the partials summed in block order: deterministic).
// Once: ref_matmul_kernel (X W^T in fp32 from exact fp16 x fp16 products) before the loop, and
// pick_best_kernel (argmin, then s of the winner) after it.
#include "common.cuh"
#include "internal.h"

namespace awq {

namespace {

bool use_gemv(int M, int N, int K) { return M <= w4a16_gemv_max_m(N, K); }

constexpr int kLossBlocks = 256;  // fp64 partials per loss (one per block of sq_err_kernel)

__device__ __forceinline__ uint16_t f64_to_f16_rn(double v) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return h;
}

// mean_r |x_rj|^alpha in fp64, rounded once to fp16.  The fp64 sum of up to 8192 fp16 magnitudes is exact,
// so the mean is the correctly rounded quotient whatever the order.  alpha = 0 gives 1; 0.5 the correctly
// rounded square root (as awq_act_scale); 1 the mean itself; anything else pow().
__device__ __forceinline__ uint16_t act_pow_one(const __half* xcal, int R, int K, int j, double alpha) {
  double sum = 0.0;
  for (int r = 0; r < R; ++r) sum += fabs((double)__half2float(xcal[(size_t)r * K + j]));
  const double mean = __ddiv_rn(sum, (double)R);
  double v;
  if (alpha == 0.0) v = 1.0;
  else if (alpha == 0.5) v = __dsqrt_rn(mean);
  else if (alpha == 1.0) v = mean;
  else v = pow(mean, alpha);
  return f64_to_f16_rn(v);
}

__global__ void __launch_bounds__(256) act_pow_kernel(const __half* __restrict__ xcal, int R, int K, double alpha,
                                                       uint16_t* __restrict__ s) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < K) s[j] = act_pow_one(xcal, R, K, j, alpha);
}

// yref[r][n] = sum_k x[r][k] W[n][k] in fp32: 64 x 64 output tile per 256-thread block, 4 x 4 per thread,
// K in steps of 32 through shared memory.  Every product of two fp16 values is exact in fp32.
constexpr int kRefTile = 64, kRefK = 32;
__global__ void __launch_bounds__(256) ref_matmul_kernel(const __half* __restrict__ x, const __half* __restrict__ W,
                                                          int R, int N, int K, float* __restrict__ yref) {
  __shared__ float xs[kRefK][kRefTile + 1];
  __shared__ float ws[kRefK][kRefTile + 1];
  const int r0 = blockIdx.y * kRefTile, n0 = blockIdx.x * kRefTile;
  const int tr = threadIdx.x / 16, tn = threadIdx.x % 16;  // rows r0 + tr + 16 i, columns n0 + tn + 16 j
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kRefK) {
    for (int e = threadIdx.x; e < kRefTile * kRefK; e += 256) {
      const int row = e / kRefK, kk = e % kRefK;
      const int k = k0 + kk;
      xs[kk][row] = (r0 + row < R && k < K) ? __half2float(x[(size_t)(r0 + row) * K + k]) : 0.f;
      ws[kk][row] = (n0 + row < N && k < K) ? __half2float(W[(size_t)(n0 + row) * K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRefK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][tr + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tn + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + tr + 16 * i, n = n0 + tn + 16 * j;
      if (r < R && n < N) yref[(size_t)r * N + n] = acc[i][j];
    }
}

// partial[b] = sum over block b's share of (y - yref)^2 in fp64 (fixed order: per-thread strided sums, then a
// fixed tree in shared memory).
__global__ void __launch_bounds__(256) sq_err_kernel(const __half* __restrict__ y, const float* __restrict__ yref,
                                                      long long count, double* __restrict__ partial) {
  __shared__ double red[256];
  double acc = 0.0;
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < count; i += (long long)gridDim.x * 256) {
    const double d = (double)__half2float(y[i]) - (double)yref[i];
    acc += d * d;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

__global__ void loss_finish_kernel(const double* __restrict__ partial, int n, double* __restrict__ loss) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double sum = 0.0;
  for (int b = 0; b < n; ++b) sum += partial[b];
  *loss = sum;
}

// Every thread finds the first least loss (n_grid + 1 values), then writes s of that alpha for its channel.
__global__ void __launch_bounds__(256) pick_best_kernel(const __half* __restrict__ xcal, int R, int K, int n_grid,
                                                         const double* __restrict__ losses, uint16_t* __restrict__ s,
                                                         int* __restrict__ best_out) {
  int best = 0;
  for (int i = 1; i <= n_grid; ++i)
    if (losses[i] < losses[best]) best = i;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j == 0) *best_out = best;
  if (j < K) s[j] = act_pow_one(xcal, R, K, j, (double)best / (double)n_grid);
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct SearchLayout {
  size_t lin, s, xp, qw, sc, qz, y, yref, part, total;
};

SearchLayout search_layout(int N, int K, int R, int g) {
  SearchLayout L{};
  const size_t Np = (size_t)(N + 31) / 32 * 32, G = (size_t)K / (size_t)g;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  const size_t lin_bytes = use_gemv(R, N, K) ? gemv_workspace_bytes(R, N, K, g) : gemm_workspace_bytes(R, N, K, g);
  L.lin = take(lin_bytes > 0 ? lin_bytes : 256);
  L.s = take((size_t)K * 2);
  L.xp = take((size_t)R * K * 2);
  L.qw = take(Np * (size_t)K / 2);
  L.sc = take(G * Np * 2);
  L.qz = take(G * Np / 2);
  L.y = take((size_t)R * N * 2);
  L.yref = take((size_t)R * N * 4);
  L.part = take(kLossBlocks * sizeof(double));
  L.total = off;
  return L;
}

}  // namespace

size_t search_workspace_bytes(int N, int K, int R, int g) { return search_layout(N, K, R, g).total; }

awq_status search_launch(const uint16_t* W, const uint16_t* xcal, int N, int K, int R, int g, int n_grid,
                         double* losses, uint16_t* s_out, int* best_out, void* ws, size_t ws_bytes,
                         unsigned* status, cudaStream_t st) {
  const SearchLayout L = search_layout(N, K, R, g);
  if (ws == nullptr || ws_bytes < L.total) return AWQ_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  uint16_t* s = reinterpret_cast<uint16_t*>(base + L.s);
  uint16_t* xp = reinterpret_cast<uint16_t*>(base + L.xp);
  uint32_t* qw = reinterpret_cast<uint32_t*>(base + L.qw);
  uint16_t* sc = reinterpret_cast<uint16_t*>(base + L.sc);
  uint32_t* qz = reinterpret_cast<uint32_t*>(base + L.qz);
  uint16_t* y = reinterpret_cast<uint16_t*>(base + L.y);
  float* yref = reinterpret_cast<float*>(base + L.yref);
  double* part = reinterpret_cast<double*>(base + L.part);
  const __half* xh = reinterpret_cast<const __half*>(xcal);
  // the linear's counters start at zero (the workspace carries no state between searches)
  if (cudaMemsetAsync(base + L.lin, 0, L.s - L.lin, st) != cudaSuccess) return AWQ_ERR_CUDA;
  {
    const dim3 grid((unsigned)((N + kRefTile - 1) / kRefTile), (unsigned)((R + kRefTile - 1) / kRefTile));
    ref_matmul_kernel<<<grid, 256, 0, st>>>(xh, reinterpret_cast<const __half*>(W), R, N, K, yref);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
  }
  const unsigned kgrid = (unsigned)((K + 255) / 256);
  const long long count = (long long)R * N;
  LinearArgs a;
  a.x = xp;
  a.qw = qw;
  a.scales = sc;
  a.qzeros = qz;
  a.y = y;
  a.M = R;
  a.N = N;
  a.K = K;
  a.g = g;
  a.ws = base + L.lin;
  a.ws_bytes = L.s - L.lin;
  a.status = status;
  a.st = st;
  const bool gemv = use_gemv(R, N, K);
  for (int i = 0; i <= n_grid; ++i) {
    act_pow_kernel<<<kgrid, 256, 0, st>>>(xh, R, K, (double)i / (double)n_grid, s);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
    awq_status e = pack_launch(W, nullptr, s, N, K, g, qw, sc, qz, st);
    if (e == AWQ_OK) e = prep_inv_scale_launch(xcal, s, R, K, xp, st);
    if (e == AWQ_OK) e = gemv ? gemv_launch(a) : gemm_launch(a);
    if (e != AWQ_OK) return e;
    sq_err_kernel<<<kLossBlocks, 256, 0, st>>>(reinterpret_cast<const __half*>(y), yref, count, part);
    loss_finish_kernel<<<1, 32, 0, st>>>(part, kLossBlocks, losses + i);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
  }
  pick_best_kernel<<<kgrid, 256, 0, st>>>(xh, R, K, n_grid, losses, s_out, best_out);
  return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
