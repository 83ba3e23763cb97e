// pack.cu -- awq_pack: fold the AWQ scale into W, quantize each (row, 128-channel group) with the
// asymmetric 4-bit min/max grid and write the packed layout of the public header.  Bit-exact.
//
// Sources: "AWQ and GPTQ algorithms" (jsqmd.com), section 2.1 (3) (multiply the weight channels by s);
// "LLM-AWQ academic impact" (CSDN mirror), "quantization flow" (w_bit 4, q_group_size 128, the real
// quantization stage); "LLM quantization speed-up" (bjdmk.com.cn), "quantization parameters" (zero point).
// Grid, in IEEE fp32 with correctly rounded operations and no contraction:
//   w' = W*s; sc32 = max((max-min)/15, 1e-5); S = float(fp16(sc32)); z = clamp(rint(-min/S), 0, 15);
//   q = clamp(rint(w'/S) + z, 0, 15).
//
// One CTA per packed unit (32-row block rb, group g): 8 warps x 4 rows, lane l holds channels
// 4l..4l+3 of the group (one 8-byte load per row), min/max by warp shuffles, codes assembled into the
// nibble order of the layout with one shuffle, and the 2 KB unit written from shared memory with
// coalesced 16-byte stores (the unit's 32 scales and 4 zero words are contiguous too).  The kernel streams 2 bytes in and 0.52 bytes out per weight.
#include "common.cuh"
#include "internal.h"

namespace awq {

__device__ __forceinline__ float clamp015(float v) { return fminf(fmaxf(v, 0.0f), 15.0f); }

__global__ void __launch_bounds__(256) pack_kernel(const __half* __restrict__ W, const __half* __restrict__ s,
                                                    int N, int K, int Np, int G, uint4* __restrict__ qw,
                                                    uint16_t* __restrict__ scales, uint32_t* __restrict__ qz) {
  pdl_launch_dependents();
  __shared__ __align__(16) uint32_t s_words[512];
  __shared__ uint16_t s_sc[32];
  __shared__ uint32_t s_z[32];
  const int g = blockIdx.x, rb = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = g * 128 + lane * 4;
  pdl_wait_prior_grids();

  float sv[4] = {1.f, 1.f, 1.f, 1.f};
  if (s != nullptr) {
    const uint2 sr = *reinterpret_cast<const uint2*>(s + k0);
    sv[0] = __half2float(__ushort_as_half((unsigned short)(sr.x & 0xFFFF)));
    sv[1] = __half2float(__ushort_as_half((unsigned short)(sr.x >> 16)));
    sv[2] = __half2float(__ushort_as_half((unsigned short)(sr.y & 0xFFFF)));
    sv[3] = __half2float(__ushort_as_half((unsigned short)(sr.y >> 16)));
  }
  uint2 raw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = rb * 32 + warp * 4 + i;
    raw[i] = n < N ? *reinterpret_cast<const uint2*>(W + (size_t)n * K + k0) : make_uint2(0u, 0u);
  }
  // nibble position of this lane's 4 channels (offsets e = 4*(lane&1) + i inside an 8-channel word):
  // even e -> e/2, odd e -> 4 + e/2
  const int odd = lane & 1;
  const int pos0 = odd ? 2 : 0, pos1 = odd ? 6 : 4, pos2 = odd ? 3 : 1, pos3 = odd ? 7 : 5;

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = warp * 4 + i;
    const int n = rb * 32 + r;
    uint32_t word = 0u;
    uint16_t sch_bits = 0;
    uint32_t zi = 0u;
    if (n < N) {  // warp-uniform
      float wp[4];
      wp[0] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(raw[i].x & 0xFFFF))), sv[0]);
      wp[1] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(raw[i].x >> 16))), sv[1]);
      wp[2] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(raw[i].y & 0xFFFF))), sv[2]);
      wp[3] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(raw[i].y >> 16))), sv[3]);
      float mn = fminf(fminf(wp[0], wp[1]), fminf(wp[2], wp[3]));
      float mx = fmaxf(fmaxf(wp[0], wp[1]), fmaxf(wp[2], wp[3]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
      }
      const float sc32 = fmaxf(__fdiv_rn(__fsub_rn(mx, mn), 15.0f), 1e-5f);
      const __half sch = __float2half_rn(sc32);
      const float S = __half2float(sch);
      const float zf = clamp015(rintf(__fdiv_rn(-mn, S)));
      zi = (uint32_t)(int)zf;
      uint32_t c[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) c[e] = (uint32_t)(int)clamp015(__fadd_rn(rintf(__fdiv_rn(wp[e], S)), zf));
      const uint32_t part = (c[0] << (4 * pos0)) | (c[1] << (4 * pos1)) | (c[2] << (4 * pos2)) |
                            (c[3] << (4 * pos3));
      word = part | __shfl_xor_sync(0xFFFFFFFFu, part, 1);
      sch_bits = __half_as_ushort(sch);
    }
    if (!odd) s_words[(lane >> 3) * 128 + r * 4 + ((lane & 7) >> 1)] = word;
    if (lane == 0) {
      s_sc[r] = sch_bits;
      s_z[r] = zi;
    }
  }
  __syncthreads();
  if (threadIdx.x < 128)
    qw[((size_t)rb * G + g) * 128 + threadIdx.x] = reinterpret_cast<const uint4*>(s_words)[threadIdx.x];
  const size_t unit = (size_t)rb * G + g;  // scales and zeros are unit major
  if (threadIdx.x < 32) scales[unit * 32 + threadIdx.x] = s_sc[threadIdx.x];
  if (threadIdx.x < 4) {
    uint32_t zw = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) zw |= s_z[threadIdx.x * 8 + i] << (4 * i);
    qz[unit * 4 + threadIdx.x] = zw;
  }
}

awq_status pack_launch(const uint16_t* W, const uint16_t* s, int N, int K, uint32_t* qw, uint16_t* scales,
                       uint32_t* qz, cudaStream_t st) {
  const int Np = (N + 31) / 32 * 32;
  const int G = K / 128;
  cudaError_t e = launch_pdl(pack_kernel, dim3((unsigned)G, (unsigned)(Np / 32)), dim3(256), 0, st,
                             reinterpret_cast<const __half*>(W), reinterpret_cast<const __half*>(s), N, K, Np, G,
                             reinterpret_cast<uint4*>(qw), scales, qz);
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
