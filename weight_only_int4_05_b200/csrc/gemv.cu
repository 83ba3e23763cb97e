// gemv.cu -- W4A16 decode kernel ("GEMV mode" of the AutoAWQ page: single batch, top speed).
//
// y[m][n] = sum_g S[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x'[m][k]   for up to MT rows of x' per pass.
//
// Work decomposition.  The packed layout stores each (32-row block rb, 128-channel group g) as 2048
// contiguous bytes, so a "unit" u = rb * G + g is one 2 KB stretch of memory and the whole weight is
// U = (N_pad / 32) * G consecutive units.  T warps share them evenly: warp t owns units
// [U*t/T, U*(t+1)/T) -- one contiguous range, so every SM streams the same number of bytes and the
// kernel has no wave-quantization tail.  Inside a warp, lane r owns row 32*rb + r: each unit is four
// coalesced 128-bit loads per lane (512 contiguous bytes per warp-instruction), dequantized in
// registers with the int4->fp16 bit trick, multiplied with x' in packed half2 FMAs (partials of 16
// products, flushed to fp32 every 32 channels), scaled by the group's fp16 scale and accumulated in
// fp32.  No cross-lane reduction is needed because the layout gives each lane a whole row.
//
// Split-K combine.  A row block whose G units are spread over several warps gets one fp32 partial per
// warp in the workspace slot (rb, t - first_warp(rb)); the warp that brings the per-row-block counter
// to its final value sums the slots in slot order (deterministic) and writes fp16 y, then resets the
// counter to 0 for the next call.  Row blocks owned entirely by one warp are written directly.
//
// Programmatic dependent launch: the first unit's weights are loaded before griddepcontrol.wait, so
// the weight stream of this kernel overlaps the tail of the kernel before it on the stream.
#include "common.cuh"
#include "internal.h"

namespace awq {

struct GemvParams {
  const uint16_t* x;
  const uint4* qw;
  const __half* scales;
  const uint32_t* qzeros;
  uint16_t* y;
  float* ws_part;
  unsigned* ws_cnt;
  long long U;   // units = RB * G
  long long T;   // warps sharing the units
  int M, N, Np, K, G, RB, S, m0;
};

__device__ __forceinline__ long long warp_of_unit(long long u, long long U, long long T) {
  return ((u + 1) * T - 1) / U;
}

__device__ __forceinline__ void load_unit(uint4 (&w)[4], const uint4* qw, long long u, int lane) {
  const uint4* p = qw + u * 128 + lane;  // unit u = 2048 B = 128 x 16 B; chunk c at +32*c
#pragma unroll
  for (int c = 0; c < 4; ++c) w[c] = ldg_stream(p + 32 * c);
}

template <int MT>
__global__ void __launch_bounds__(256) gemv_kernel(const GemvParams p) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= p.T) return;  // writes nothing
  const int mcount = min(MT, p.M - p.m0);
  long long u = p.U * t / p.T;
  const long long u_end = p.U * (t + 1) / p.T;
  const int G = p.G;

  uint4 w[4];
  load_unit(w, p.qw, u, lane);
  pdl_wait_prior_grids();  // activations, outputs and workspace belong to the stream order

  // Row pointers of x' for this pass; rows beyond M repeat the last row (computed, never stored).
  const uint16_t* xrow[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) xrow[m] = p.x + (size_t)(p.m0 + min(m, mcount - 1)) * p.K;

  while (u < u_end) {
    const int rb = (int)(u / G);
    const int g0 = (int)(u - (long long)rb * G);
    const long long seg_end = min(u_end, (long long)(rb + 1) * G);
    const int n = rb * 32 + lane;
    float yacc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) yacc[m] = 0.f;

    for (; u < seg_end; ++u) {
      const int g = (int)(u - (long long)rb * G);
      uint4 wn[4];
      const bool more = (u + 1 < u_end);
      if (more) load_unit(wn, p.qw, u + 1, lane);
      const float scf = __half2float(p.scales[(size_t)g * p.Np + n]);
      const uint32_t zw = p.qzeros[(size_t)g * (p.Np >> 3) + rb * 4 + (lane >> 3)];
      const uint32_t z = (zw >> (4 * (lane & 7))) & 0xFu;
      const __half2 z1024 = zero_1024(z), nz64 = neg_zero_64(z);
      float part[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) part[m] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t ww[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
        __half2 acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = __float2half2_rn(0.f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __half2 d[4];
          word_minus_zero(ww[j], z1024, nz64, d);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 xv = ldg_cached(xrow[m] + g * 128 + c * 32 + j * 8);
            acc[m] = __hfma2(d[0], u32_as_h2(xv.x), acc[m]);
            acc[m] = __hfma2(d[1], u32_as_h2(xv.y), acc[m]);
            acc[m] = __hfma2(d[2], u32_as_h2(xv.z), acc[m]);
            acc[m] = __hfma2(d[3], u32_as_h2(xv.w), acc[m]);
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) part[m] += __low2float(acc[m]) + __high2float(acc[m]);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) yacc[m] = fmaf(scf, part[m], yacc[m]);
      if (more) {
#pragma unroll
        for (int c = 0; c < 4; ++c) w[c] = wn[c];
      }
    }

    const bool whole = (g0 == 0) && (seg_end == (long long)(rb + 1) * G);
    if (whole) {
      if (n < p.N) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < mcount) p.y[(size_t)(p.m0 + m) * p.N + n] = __half_as_ushort(__float2half_rn(yacc[m]));
      }
      continue;
    }
    // ---- split-K combine through the workspace
    const long long tf = warp_of_unit((long long)rb * G, p.U, p.T);
    const long long tl = warp_of_unit((long long)rb * G + G - 1, p.U, p.T);
    const int nc = (int)(tl - tf + 1);
    const int slot = (int)(t - tf);
    float* base = p.ws_part + (size_t)rb * p.S * 32 * MT;
#pragma unroll
    for (int m = 0; m < MT; ++m) base[(size_t)(slot * MT + m) * 32 + lane] = yacc[m];
    __threadfence();
    __syncwarp();
    unsigned old = 0;
    if (lane == 0) old = atomicAdd(&p.ws_cnt[rb], 1u);
    old = __shfl_sync(0xFFFFFFFFu, old, 0);
    if (old == (unsigned)(nc - 1)) {
      __threadfence();
      float sum[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) sum[m] = 0.f;
      for (int j = 0; j < nc; ++j) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
          sum[m] += (j == slot) ? yacc[m] : __ldcg(&base[(size_t)(j * MT + m) * 32 + lane]);
      }
      if (n < p.N) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < mcount) p.y[(size_t)(p.m0 + m) * p.N + n] = __half_as_ushort(__float2half_rn(sum[m]));
      }
      if (lane == 0) p.ws_cnt[rb] = 0u;
    }
  }
}

// ------------------------------------------------------------------------------------------ host
namespace {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

int pick_mt(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

template <int MT>
int gemv_ctas_per_sm() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_kernel<MT>, kGemvThreads, 0);
    cached[dev] = occ > 0 ? occ : 1;
  }
  return cached[dev];
}

int ctas_per_sm(int MT) {
  switch (MT) {
    case 1: return gemv_ctas_per_sm<1>();
    case 2: return gemv_ctas_per_sm<2>();
    case 4: return gemv_ctas_per_sm<4>();
    default: return gemv_ctas_per_sm<8>();
  }
}

struct GemvPlan {
  int MT, RB, G, S, Np;
  long long U, T;
  size_t part_bytes;
};

GemvPlan plan_gemv(int M, int N, int K) {
  GemvPlan pl{};
  pl.MT = pick_mt(M);
  pl.Np = (N + 31) / 32 * 32;
  pl.RB = pl.Np / 32;
  pl.G = K / 128;
  pl.U = (long long)pl.RB * pl.G;
  const long long slots = (long long)num_sms() * ctas_per_sm(pl.MT) * kGemvWarps;
  pl.T = pl.U < slots ? pl.U : slots;
  const long long L = pl.U / pl.T;  // >= 1
  pl.S = pl.G >= 2 ? (int)((pl.G - 2) / L + 2) : 1;
  pl.part_bytes = (size_t)pl.RB * pl.S * 32 * pl.MT * sizeof(float);
  return pl;
}

}  // namespace

size_t gemv_workspace_bytes(int M, int N, int K) {
  const GemvPlan pl = plan_gemv(M, N, K);
  return kWorkspaceCounterBytes + pl.part_bytes;
}

awq_status gemv_launch(const uint16_t* x, const uint32_t* qw, const uint16_t* scales, const uint32_t* qzeros,
                       uint16_t* y, int M, int N, int K, void* ws, size_t ws_bytes, cudaStream_t st) {
  const GemvPlan pl = plan_gemv(M, N, K);
  if (pl.RB * 4 > (int)(kWorkspaceCounterBytes)) return AWQ_ERR_UNSUPPORTED;
  if (ws == nullptr || ws_bytes < kWorkspaceCounterBytes + pl.part_bytes) return AWQ_ERR_WORKSPACE;
  GemvParams p;
  p.x = x;
  p.qw = reinterpret_cast<const uint4*>(qw);
  p.scales = reinterpret_cast<const __half*>(scales);
  p.qzeros = qzeros;
  p.y = y;
  p.ws_cnt = static_cast<unsigned*>(ws);
  p.ws_part = reinterpret_cast<float*>(static_cast<char*>(ws) + kWorkspaceCounterBytes);
  p.U = pl.U;
  p.T = pl.T;
  p.M = M;
  p.N = N;
  p.Np = pl.Np;
  p.K = K;
  p.G = pl.G;
  p.RB = pl.RB;
  p.S = pl.S;
  const unsigned grid = (unsigned)((pl.T + kGemvWarps - 1) / kGemvWarps);
  // passes of MT rows run one after the other on the stream and share the workspace
  for (int m0 = 0; m0 < M; m0 += pl.MT) {
    p.m0 = m0;
    cudaError_t e;
    switch (pl.MT) {
      case 1: e = launch_pdl(gemv_kernel<1>, dim3(grid), dim3(kGemvThreads), 0, st, p); break;
      case 2: e = launch_pdl(gemv_kernel<2>, dim3(grid), dim3(kGemvThreads), 0, st, p); break;
      case 4: e = launch_pdl(gemv_kernel<4>, dim3(grid), dim3(kGemvThreads), 0, st, p); break;
      default: e = launch_pdl(gemv_kernel<8>, dim3(grid), dim3(kGemvThreads), 0, st, p); break;
    }
    if (e != cudaSuccess) return AWQ_ERR_CUDA;
  }
  return AWQ_OK;
}

}  // namespace awq
