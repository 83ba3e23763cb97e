// pack.cu -- awq_pack: fold the AWQ scale into W, quantize each (row, 128-channel group) with the
// asymmetric 4-bit min/max grid and write the packed layout of the public header.  Bit-exact.
//
// Sources: "AWQ and GPTQ algorithms" (jsqmd.com), section 2.1 (3) (multiply the weight channels by s);
// "LLM-AWQ academic impact" (CSDN mirror), "quantization flow" (w_bit 4, q_group_size 128, the real
// quantization stage); "LLM quantization speed-up" (bjdmk.com.cn), "quantization parameters" (zero point).
// Grid, in IEEE fp32 with correctly rounded operations and no contraction (qmax = 2^w_bit - 1: 15 for the
// pages' 4 bits, 7 for the 3-bit grid, whose codes are stored in the same 4-bit layout):
//   w' = W*s; sc32 = max((max-min)/qmax, 1e-5); S = float(fp16(sc32)); z = clamp(rint(-min/S), 0, qmax);
//   q = clamp(rint(w'/S) + z, 0, qmax).
//
// One CTA per run of kPackGroups units of one row block (the units (rb, g0 .. g0+3) are consecutive in all
// three packed arrays).  LPG = GS / 8 lanes take one (row, group): lane h of them holds channels 8h..8h+7
// (one 16-byte load), which are exactly the 8 codes of one packed word, so no lane exchange is needed to
// assemble it.  Min and max come from log2(LPG) shuffles inside those lanes.  The units are assembled in
// shared memory and written with coalesced 16-byte stores.  The kernel streams 2 bytes in and 0.52 bytes out
// per weight.
//
// 3-bit storage (BITS = 3): the 3-bit grid (qmax = 7) written in the packed 3-bit layout of the public header --
// per row and 32-channel chunk, a word of low 2-bit fields for channels 0..15, one for 16..31, and a word of
// high bits -- with scales and zeros exactly as at 4 bits.
//
// Gate|up packing (W2 != NULL): row 32j + i of the packed weight comes from W row 16j + i (i < 16) or W2 row
// 16j + i - 16 (i >= 16), so the decode and prefill kernels find each gate row and its up row in the same
// row block, 16 rows apart.
#include "common.cuh"
#include "internal.h"

namespace awq {

constexpr int kPackGroups = 4;  // units per CTA

__device__ __forceinline__ float clamp0q(float v, float qmax) { return fminf(fmaxf(v, 0.0f), qmax); }
__device__ __forceinline__ float h2f_bits(uint32_t bits) { return __half2float(__ushort_as_half((unsigned short)bits)); }

template <int GS, int BITS>
__global__ void __launch_bounds__(256) pack_kernel(const __half* __restrict__ W, const __half* __restrict__ W2,
                                                    const __half* __restrict__ s, int N, int K, int G, float qmax,
                                                    uint8_t* __restrict__ qw, uint16_t* __restrict__ scales,
                                                    uint32_t* __restrict__ qz) {
  // No griddepcontrol.launch_dependents here: the linear kernels read packed weights before their own
  // dependency wait, so a kernel launched after this one must not start until every packed byte is
  // written.  Without an explicit trigger the dependents start only when this grid has completed.
  constexpr int LPG = GS / 8;           // lanes per (row, group)
  constexpr int IPW = 32 / LPG;         // (row, group) items per warp at a time
  constexpr int NP = 32 / (8 * IPW);    // passes over the 32 rows of the block (8 warps)
  constexpr int UW = BITS * GS;         // 32-bit code words per unit (16 GS bytes at 4 bits, 12 GS at 3)
  __shared__ __align__(16) uint32_t s_words[kPackGroups * UW];
  __shared__ __align__(16) uint16_t s_sc[kPackGroups * 32];
  __shared__ uint8_t s_zb[kPackGroups * 32];
  const int rb = blockIdx.x, g0 = blockIdx.y * kPackGroups;
  const int ng = min(kPackGroups, G - g0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPG, hl = lane % LPG;
  pdl_wait_prior_grids();

  // rows (8 * pass + warp) * IPW + sub of the row block; all loads first
  uint4 raw[NP][kPackGroups];
  uint4 sraw[kPackGroups];
#pragma unroll
  for (int gi = 0; gi < kPackGroups; ++gi) {
    const int k0 = (g0 + gi) * GS + 8 * hl;
    sraw[gi] = make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);  // s = 1
    if (gi < ng && s != nullptr) sraw[gi] = *reinterpret_cast<const uint4*>(s + k0);
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int r = (8 * i + warp) * IPW + sub;
      const int n = rb * 32 + r;
      const __half* src = W + (size_t)n * K;
      if (W2 != nullptr) src = (r < 16 ? W : W2) + (size_t)(rb * 16 + (r & 15)) * K;
      raw[i][gi] = (gi < ng && n < N) ? *reinterpret_cast<const uint4*>(src + k0) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // nibble position of channel offset e in a word: even e -> e/2, odd e -> 4 + e/2
#pragma unroll
  for (int gi = 0; gi < kPackGroups; ++gi) {
    if (gi >= ng) break;  // CTA-uniform
    const uint32_t sw[4] = {sraw[gi].x, sraw[gi].y, sraw[gi].z, sraw[gi].w};
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int r = (8 * i + warp) * IPW + sub;
      const bool valid = rb * 32 + r < N;
      const uint32_t ww[4] = {raw[i][gi].x, raw[i][gi].y, raw[i][gi].z, raw[i][gi].w};
      float wp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        wp[e] = __fmul_rn(h2f_bits(ww[e >> 1] >> (16 * (e & 1))), h2f_bits(sw[e >> 1] >> (16 * (e & 1))));
      float mn = wp[0], mx = wp[0];
#pragma unroll
      for (int e = 1; e < 8; ++e) {
        mn = fminf(mn, wp[e]);
        mx = fmaxf(mx, wp[e]);
      }
#pragma unroll
      for (int off = LPG / 2; off > 0; off >>= 1) {  // inside the LPG lanes of this (row, group)
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
      }
      const float sc32 = fmaxf(__fdiv_rn(__fsub_rn(mx, mn), qmax), 1e-5f);
      const __half sch = __float2half_rn(sc32);
      const float S = __half2float(sch);
      const float zf = clamp0q(rintf(__fdiv_rn(-mn, S)), qmax);
      if (BITS == 4) {
        uint32_t word = 0u;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t code = (uint32_t)(int)clamp0q(__fadd_rn(rintf(__fdiv_rn(wp[e], S)), zf), qmax);
          word |= code << (4 * ((e & 1) ? 4 + (e >> 1) : (e >> 1)));
        }
        // word hl & 3 of row r in the unit's chunk hl >> 2 (chunk = 512 B = 128 words, row = 4 words)
        s_words[gi * UW + (hl >> 2) * 128 + r * 4 + (hl & 3)] = valid ? word : 0u;
      } else {
        // 3-bit layout: this lane's 8 channels are group j = hl & 3 of chunk hl >> 2; channel 8j + 2p + h puts
        // its low 2 bits at bit 8 (j % 2) + 2p + 16h of word j / 2 and its high bit at bit 4j + p + 16h of
        // word 2 (chunk = 384 B = 96 words, row = 3 words).  The four lanes of a chunk are adjacent lanes.
        const int j = hl & 3;
        uint32_t lo = 0u, hi = 0u;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t code = (uint32_t)(int)clamp0q(__fadd_rn(rintf(__fdiv_rn(wp[e], S)), zf), qmax);
          const int pp = e >> 1, hh = e & 1;
          lo |= (code & 3u) << (8 * (j & 1) + 2 * pp + 16 * hh);
          hi |= (code >> 2) << (4 * j + pp + 16 * hh);
        }
        lo |= __shfl_xor_sync(0xFFFFFFFFu, lo, 1);  // groups 0 | 1 -> word 0, groups 2 | 3 -> word 1
        hi |= __shfl_xor_sync(0xFFFFFFFFu, hi, 1);
        hi |= __shfl_xor_sync(0xFFFFFFFFu, hi, 2);  // all four groups -> word 2
        uint32_t* row3 = s_words + gi * UW + (hl >> 2) * 96 + r * 3;
        if (j == 0) row3[0] = valid ? lo : 0u;
        if (j == 2) row3[1] = valid ? lo : 0u;
        if (j == 1) row3[2] = valid ? hi : 0u;
      }
      if (hl == 0) {
        s_sc[gi * 32 + r] = valid ? __half_as_ushort(sch) : (uint16_t)0;
        s_zb[gi * 32 + r] = valid ? (uint8_t)(int)zf : (uint8_t)0;
      }
    }
  }
  __syncthreads();
  const size_t u0 = (size_t)rb * G + g0;  // first unit of this CTA; its ng units are consecutive
  uint4* dst = reinterpret_cast<uint4*>(qw + u0 * (size_t)(4 * BITS * GS));
  for (int idx = threadIdx.x; idx < ng * UW / 4; idx += 256) dst[idx] = reinterpret_cast<const uint4*>(s_words)[idx];
  if (threadIdx.x < ng * 4) {
    reinterpret_cast<uint4*>(scales + u0 * 32)[threadIdx.x] = reinterpret_cast<const uint4*>(s_sc)[threadIdx.x];
    uint32_t zw = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) zw |= (uint32_t)s_zb[threadIdx.x * 8 + i] << (4 * i);
    qz[u0 * 4 + threadIdx.x] = zw;
  }
  __threadfence();  // the packed units are performed at device scope before this CTA exits
}

awq_status pack_launch(const uint16_t* W, const uint16_t* W2, const uint16_t* s, int N, int K, int g, uint32_t* qw,
                       uint16_t* scales, uint32_t* qz, cudaStream_t st, int w_bit, int storage_bits) {
  const float qmax = (float)((1 << (storage_bits == 3 ? 3 : w_bit)) - 1);
  const int RB = (N + 31) / 32;
  const int G = K / g;
  const dim3 grid((unsigned)RB, (unsigned)((G + kPackGroups - 1) / kPackGroups));  // x: row blocks (no 65535 cap)
  const __half* w = reinterpret_cast<const __half*>(W);
  const __half* w2 = reinterpret_cast<const __half*>(W2);
  const __half* sh = reinterpret_cast<const __half*>(s);
  uint8_t* q = reinterpret_cast<uint8_t*>(qw);
  cudaError_t e;
  if (storage_bits == 3) {
    switch (g) {
      case 64: e = launch_pdl(pack_kernel<64, 3>, grid, dim3(256), 0, st, w, w2, sh, N, K, G, qmax, q, scales, qz); break;
      case 256: e = launch_pdl(pack_kernel<256, 3>, grid, dim3(256), 0, st, w, w2, sh, N, K, G, qmax, q, scales, qz); break;
      default: e = launch_pdl(pack_kernel<128, 3>, grid, dim3(256), 0, st, w, w2, sh, N, K, G, qmax, q, scales, qz); break;
    }
  } else {
    switch (g) {
      case 64: e = launch_pdl(pack_kernel<64, 4>, grid, dim3(256), 0, st, w, w2, sh, N, K, G, qmax, q, scales, qz); break;
      case 256: e = launch_pdl(pack_kernel<256, 4>, grid, dim3(256), 0, st, w, w2, sh, N, K, G, qmax, q, scales, qz); break;
      default: e = launch_pdl(pack_kernel<128, 4>, grid, dim3(256), 0, st, w, w2, sh, N, K, G, qmax, q, scales, qz); break;
    }
  }
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
