// prep.cu -- the two activation-side steps of AWQ that surround the quantized linear layer.
//
//  awq_act_scale:       s_j = fp16(sqrt(mean_r |xcal_rj|))     "AWQ and GPTQ algorithms" (jsqmd.com),
//                       section 2.1 (2): channel importance is the mean absolute calibration activation;
//                       the exponent 0.5 is this library's fixed reading of the scale.
//  awq_apply_inv_scale: x'_mk = fp16(x_mk / s_k)               same page, section 2.1 (3): activations
//                       are divided by s at inference, undoing the factor folded into the weights.
// Both run in IEEE fp64 (correctly rounded add, divide and square root) and round once to fp16, so
// the results are bit-exact and independent of summation order (the fp64 sum of fp16 magnitudes is
// exact for up to 8192 rows).
#include "common.cuh"
#include "internal.h"

namespace awq {

__device__ __forceinline__ uint16_t f64_to_f16_rn(double v) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return h;
}

__global__ void __launch_bounds__(256) act_scale_kernel(const __half* __restrict__ xcal, int R, int K,
                                                         uint16_t* __restrict__ s) {
  pdl_launch_dependents();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait_prior_grids();
  if (j >= K) return;
  double sum = 0.0;
  for (int r = 0; r < R; ++r) sum += fabs((double)__half2float(xcal[(size_t)r * K + j]));
  s[j] = f64_to_f16_rn(__dsqrt_rn(__ddiv_rn(sum, (double)R)));
}

__global__ void __launch_bounds__(256) inv_scale_kernel(const __half* __restrict__ x, const __half* __restrict__ s,
                                                         long long total, int K, uint16_t* xp) {
  pdl_launch_dependents();
  pdl_wait_prior_grids();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int k = (int)(i % K);
    const double q = __ddiv_rn((double)__half2float(x[i]), (double)__half2float(s[k]));
    xp[i] = f64_to_f16_rn(q);
  }
}

awq_status prep_act_scale_launch(const uint16_t* xcal, int R, int K, uint16_t* s, cudaStream_t st) {
  const unsigned grid = (unsigned)((K + 255) / 256);
  cudaError_t e = launch_pdl(act_scale_kernel, dim3(grid), dim3(256), 0, st,
                             reinterpret_cast<const __half*>(xcal), R, K, s);
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status prep_inv_scale_launch(const uint16_t* x, const uint16_t* s, int M, int K, uint16_t* xp,
                                 cudaStream_t st) {
  const long long total = (long long)M * K;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  cudaError_t e = launch_pdl(inv_scale_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                             reinterpret_cast<const __half*>(x), reinterpret_cast<const __half*>(s), total, K, xp);
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
