// gptq.cu -- gptq_quantize: GPTQ on the GPU, writing the W4A16 packed layout of the public header.
//
// "AWQ and GPTQ algorithms" (jsqmd.com), section 3.1: minimise ||W X - W_hat X||_F^2 over calibration
// activations X with the Hessian H = X^T X; the columns are quantized in blocks of 128, each column's
// quantization error compensated in the columns not yet quantized through the inverse Hessian (obtained via
// Cholesky), with lazy batch updates of the columns after the block; section 3.3: a small term (1e-6 by
// default) on the diagonal keeps H non-singular.  The grid is awq_pack's asymmetric fp32 min/max grid (s = 1)
// applied, at each group's first column, to the group's current weights rounded to fp32.
//
// Everything except the grid is fp64:
//   gram_rev_kernel     H = X^T X + damp I in index-reversed order (Hr[i][j] = H[K-1-i][K-1-j]); every
//                       element sums its products over the rows in row order (each product is exact).
//   chol_panel_kernel,  blocked right-looking Cholesky Hr = L L^T (64 x 64 tiles): each step factors the
//   chol_update_kernel  diagonal tile, solves the panel below it, and updates the trailing lower triangle.
//   trtri_solve_kernel, Xi = L^-1, right-looking: solve one block row (the diagonal tile's forward substitution),
//   trtri_update_kernel then add its contribution to every later block row at once.
//   Then U = J Xi J (J the index reversal) is upper triangular with H^-1 = U^T U -- the factor GPTQ's
//   error compensation uses -- without a second factorisation.
//   gptq_block_kernel   one 128-column block: a CTA per 32-row block quantizes the columns in order, spreads
//                       each column's error over the block's later columns, writes codes, scales and zeros.
//   gptq_lazy_kernel    the block's errors applied to every later column at once (W -= E U_block,rest).
#include "common.cuh"
#include "internal.h"

namespace awq {

namespace {

constexpr int kT = 64;    // fp64 tile edge of the Gram, Cholesky and inverse kernels
constexpr int kGB = 128;  // GPTQ column block
constexpr unsigned kDevNotPositive = 2u;  // status word: a Cholesky pivot was not positive

__device__ __forceinline__ void tri_index(int t, int& a, int& b) {  // t -> (a, b), a >= b >= 0, row-major lower
  a = (int)((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
  while ((a + 1) * (a + 2) / 2 <= t) ++a;
  while (a * (a + 1) / 2 > t) --a;
  b = t - a * (a + 1) / 2;
}

__global__ void __launch_bounds__(256) to_f64_kernel(const __half* __restrict__ W, long long count,
                                                      double* __restrict__ Wc) {
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < count; i += (long long)gridDim.x * 256)
    Wc[i] = (double)__half2float(W[i]);
}

// Hr[i][j] for the lower-triangle tiles (ti >= tj); thread (ty, tx) owns rows ty + 16u, columns tx + 16v.
__global__ void __launch_bounds__(256) gram_rev_kernel(const __half* __restrict__ x, int R, int K, double damp,
                                                        double* __restrict__ Hr) {
  __shared__ double xa[16][kT + 1];
  __shared__ double xb[16][kT + 1];
  int ti, tj;
  tri_index(blockIdx.x, ti, tj);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
  for (int r0 = 0; r0 < R; r0 += 16) {
    for (int e = threadIdx.x; e < 16 * kT; e += 256) {
      const int rr = e / kT, a = e % kT, r = r0 + rr;
      xa[rr][a] = r < R ? (double)__half2float(x[(size_t)r * K + (K - 1 - (ti * kT + a))]) : 0.0;
      xb[rr][a] = r < R ? (double)__half2float(x[(size_t)r * K + (K - 1 - (tj * kT + a))]) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int rr = 0; rr < 16; ++rr)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(xa[rr][ty + 16 * u], xb[rr][tx + 16 * v], acc[u][v]);
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int i = ti * kT + ty + 16 * u, j = tj * kT + tx + 16 * v;
      Hr[(size_t)i * K + j] = acc[u][v] + (i == j ? damp : 0.0);
    }
}

// Step c of the Cholesky: every CTA factors the diagonal tile (c, c) in shared memory; CTA 0 stores it in the
// scratch tile D (lower, zero above: the other CTAs may still be reading the tile from A, so chol_update_kernel
// copies D into place), CTA q > 0 solves the panel tile (c + q, c):  X L_cc^T = A  ->  X.
__global__ void __launch_bounds__(256) chol_panel_kernel(double* __restrict__ A, int K, int c, double* __restrict__ D,
                                                          unsigned* status) {
  extern __shared__ double csm[];
  double* L = csm;                  // [64][65]
  double* P = csm + kT * (kT + 1);  // [64][65]
  const int tid = threadIdx.x;
  const size_t base = (size_t)c * kT * K + (size_t)c * kT;
  for (int e = tid; e < kT * kT; e += 256) L[(e / kT) * (kT + 1) + e % kT] = A[base + (size_t)(e / kT) * K + e % kT];
  __syncthreads();
  for (int j = 0; j < kT; ++j) {
    if (tid == 0) {
      double d = L[j * (kT + 1) + j];
      if (!(d > 0.0)) {
        atomicExch(status, kDevNotPositive);
        d = 1.0;
      }
      L[j * (kT + 1) + j] = sqrt(d);
    }
    __syncthreads();
    for (int i = j + 1 + tid; i < kT; i += 256) L[i * (kT + 1) + j] /= L[j * (kT + 1) + j];
    __syncthreads();
    const int m = kT - 1 - j;
    for (int e = tid; e < m * m; e += 256) {
      const int i = j + 1 + e / m, k = j + 1 + e % m;
      if (k <= i) L[i * (kT + 1) + k] -= L[i * (kT + 1) + j] * L[k * (kT + 1) + j];
    }
    __syncthreads();
  }
  if (blockIdx.x == 0) {
    for (int e = tid; e < kT * kT; e += 256) {
      const int i = e / kT, k = e % kT;
      D[e] = k <= i ? L[i * (kT + 1) + k] : 0.0;
    }
    return;
  }
  const size_t pb = (size_t)(c + blockIdx.x) * kT * K + (size_t)c * kT;
  for (int e = tid; e < kT * kT; e += 256) P[(e / kT) * (kT + 1) + e % kT] = A[pb + (size_t)(e / kT) * K + e % kT];
  __syncthreads();
  if (tid < kT) {  // row tid of the panel tile, columns in order
    double* pr = P + tid * (kT + 1);
    for (int j = 0; j < kT; ++j) {
      double v = pr[j];
      for (int k = 0; k < j; ++k) v -= pr[k] * L[j * (kT + 1) + k];
      pr[j] = v / L[j * (kT + 1) + j];
    }
  }
  __syncthreads();
  for (int e = tid; e < kT * kT; e += 256) A[pb + (size_t)(e / kT) * K + e % kT] = P[(e / kT) * (kT + 1) + e % kT];
}

// Trailing update of step c: A[ti][tj] -= P_ti P_tj^T for c < tj <= ti (P = the panel column c just solved).
// The last CTA copies the factored diagonal tile D into A[c][c] (no CTA of this kernel reads that tile).
__global__ void __launch_bounds__(256) chol_update_kernel(double* __restrict__ A, int K, int c,
                                                           const double* __restrict__ D) {
  __shared__ double Pi[kT][33];
  __shared__ double Pj[kT][33];
  if (blockIdx.x == gridDim.x - 1) {
    for (int e = threadIdx.x; e < kT * kT; e += 256) A[(size_t)(c * kT + e / kT) * K + c * kT + e % kT] = D[e];
    return;
  }
  int a, b;
  tri_index(blockIdx.x, a, b);
  const int ti = c + 1 + a, tj = c + 1 + b;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
  for (int k0 = 0; k0 < kT; k0 += 32) {  // the panel's 64 columns in two halves (static shared memory)
    for (int e = threadIdx.x; e < kT * 32; e += 256) {
      const int r = e / 32, k = e % 32;
      Pi[r][k] = A[(size_t)(ti * kT + r) * K + c * kT + k0 + k];
      Pj[r][k] = A[(size_t)(tj * kT + r) * K + c * kT + k0 + k];
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < 32; ++k)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(Pi[ty + 16 * u][k], Pj[tx + 16 * v][k], acc[u][v]);
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) A[(size_t)(ti * kT + ty + 16 * u) * K + tj * kT + tx + 16 * v] -= acc[u][v];
}

// Xi = L^-1 (L lower, the factored Hr), right-looking over block rows; Xi starts at zero and its rows below the
// current one accumulate T[i][c] = sum_{k < i} L[i][k] Xi[k][c].
// Row k: CTA c (0 .. k) solves L[k][k] Xi[k][c] = (c == k ? I : -T[k][c]) by forward substitution.
__global__ void __launch_bounds__(256) trtri_solve_kernel(const double* __restrict__ L, double* __restrict__ Xi, int K,
                                                           int k) {
  extern __shared__ double tsm[];
  double* La = tsm;                 // [64][65] the diagonal tile L[k][k]
  double* T = La + kT * (kT + 1);   // [64][65] right-hand side, then the solution
  const int c = blockIdx.x, tid = threadIdx.x;
  for (int e = tid; e < kT * kT; e += 256) {
    const int r = e / kT, q = e % kT;
    La[r * (kT + 1) + q] = L[(size_t)(k * kT + r) * K + k * kT + q];
    T[r * (kT + 1) + q] = (c == k) ? (r == q ? 1.0 : 0.0) : -Xi[(size_t)(k * kT + r) * K + c * kT + q];
  }
  __syncthreads();
  if (tid < kT) {  // column tid of the right-hand side, down the rows
    for (int r = 0; r < kT; ++r) {
      double v = T[r * (kT + 1) + tid];
      for (int q = 0; q < r; ++q) v -= La[r * (kT + 1) + q] * T[q * (kT + 1) + tid];
      T[r * (kT + 1) + tid] = v / La[r * (kT + 1) + r];
    }
  }
  __syncthreads();
  for (int e = tid; e < kT * kT; e += 256)
    Xi[(size_t)(k * kT + e / kT) * K + c * kT + e % kT] = T[(e / kT) * (kT + 1) + e % kT];
}

// After row k: T[i][c] += L[i][k] Xi[k][c] for every later row block i > k and column block c <= k (one tile per
// CTA; the later rows' accumulators live in Xi until their own solve).
__global__ void __launch_bounds__(256) trtri_update_kernel(const double* __restrict__ L, double* __restrict__ Xi, int K,
                                                            int k) {
  __shared__ double La[kT][33];
  __shared__ double Xb[32][kT + 1];
  const int cols = k + 1;
  const int i = k + 1 + blockIdx.x / cols, c = blockIdx.x % cols;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
  for (int q0 = 0; q0 < kT; q0 += 32) {
    for (int e = threadIdx.x; e < kT * 32; e += 256) {
      const int r = e / 32, q = e % 32;
      La[r][q] = L[(size_t)(i * kT + r) * K + k * kT + q0 + q];
    }
    for (int e = threadIdx.x; e < 32 * kT; e += 256) {
      const int q = e / kT, col = e % kT;
      Xb[q][col] = Xi[(size_t)(k * kT + q0 + q) * K + c * kT + col];
    }
    __syncthreads();
#pragma unroll 4
    for (int q = 0; q < 32; ++q)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(La[ty + 16 * u][q], Xb[q][tx + 16 * v], acc[u][v]);
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) Xi[(size_t)(i * kT + ty + 16 * u) * K + c * kT + tx + 16 * v] += acc[u][v];
}

struct GptqParams {
  const double* Xi;  // L^-1; U[i][j] = Xi[K-1-i][K-1-j] for i <= j
  double* Wc;        // [N][K] current weights
  double* E;         // [N_pad][128] errors of the current block
  uint32_t* qw;
  uint16_t* scales;
  uint32_t* qz;
  int N, K, g, G;
};

// Quantize columns b0 .. b0 + 127.  CTA = row block rb (32 rows), thread (r = tid / 4, quarter qd = tid % 4)
// owns columns 32 qd .. 32 qd + 31 of the block for row r; the owner of column i quantizes it and hands its
// error to the row's other three threads (same warp).
constexpr int kGptqThreads = 128;
constexpr int kUbStride = kGB + 1, kWbStride = kGB + 1;
__host__ __device__ constexpr size_t gptq_block_smem() {
  return ((size_t)kGB * kUbStride + 32 * kWbStride) * sizeof(double) + 32 * (sizeof(float) + sizeof(int));
}

__global__ void __launch_bounds__(kGptqThreads) gptq_block_kernel(const GptqParams p, int b0) {
  extern __shared__ double gsm[];
  double* Ub = gsm;                                 // [128][129]  U[b0 + i][b0 + j], j >= i
  double* Wb = Ub + kGB * kUbStride;                // [32][129]   current weights of the block
  float* Ss = reinterpret_cast<float*>(Wb + 32 * kWbStride);  // [32] scale of the row's current group
  int* Zs = reinterpret_cast<int*>(Ss + 32);                  // [32] zero of the row's current group
  const int tid = threadIdx.x, lane = tid & 31;
  const int rb = blockIdx.x, r = tid >> 2, qd = tid & 3;
  const int n = rb * 32 + r;
  const bool valid = n < p.N;
  const int K = p.K;
  for (int e = tid; e < kGB * kGB; e += kGptqThreads) {
    const int i = e / kGB, j = e % kGB;
    Ub[i * kUbStride + j] = j >= i ? p.Xi[(size_t)(K - 1 - b0 - i) * K + (K - 1 - b0 - j)] : 0.0;
  }
  for (int e = tid; e < 32 * kGB; e += kGptqThreads) {
    const int rr = e / kGB, j = e % kGB;
    Wb[rr * kWbStride + j] = (rb * 32 + rr < p.N) ? p.Wc[(size_t)(rb * 32 + rr) * K + b0 + j] : 0.0;
  }
  if (b0 % p.g != 0 && qd == 0) {  // the group began in the previous block: its grid is in the outputs
    const size_t unit = (size_t)rb * p.G + b0 / p.g;
    Ss[r] = valid ? __half2float(__ushort_as_half(p.scales[unit * 32 + r])) : 1.0f;
    Zs[r] = valid ? (int)((p.qz[unit * 4 + r / 8] >> (4 * (r % 8))) & 0xFu) : 0;
  }
  __syncthreads();
  double* wr = Wb + r * kWbStride;
  uint32_t words[4] = {0u, 0u, 0u, 0u};
  for (int i = 0; i < kGB; ++i) {
    const int col = b0 + i;
    if (col % p.g == 0) {  // a group starts (block-uniform): its grid from the current weights
      float mn = INFINITY, mx = -INFINITY;
      const int hi = min(i + p.g, kGB);
      for (int j = max(i, 32 * qd); j < min(hi, 32 * qd + 32); ++j) {  // this thread's own in-block columns
        const float f = (float)wr[j];
        mn = fminf(mn, f);
        mx = fmaxf(mx, f);
      }
      for (int e = kGB - i + qd; e < p.g; e += 4) {  // columns past the block (g = 256), as stored
        const float f = valid ? (float)p.Wc[(size_t)n * K + col + e] : 0.f;
        mn = fminf(mn, f);
        mx = fmaxf(mx, f);
      }
      mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      const float sc32 = fmaxf(__fdiv_rn(__fsub_rn(mx, mn), 15.0f), 1e-5f);
      const __half sch = __float2half_rn(sc32);
      const float S = __half2float(sch);
      const float zf = fminf(fmaxf(rintf(__fdiv_rn(-mn, S)), 0.f), 15.f);
      const size_t unit = (size_t)rb * p.G + col / p.g;
      if (qd == 0) {
        Ss[r] = valid ? S : 1.0f;
        Zs[r] = (int)zf;
        p.scales[unit * 32 + r] = valid ? __half_as_ushort(sch) : (uint16_t)0;
      }
      __syncthreads();
      if (tid < 4) {
        uint32_t zw = 0u;
        for (int q = 0; q < 8; ++q)
          if (rb * 32 + 8 * tid + q < p.N) zw |= (uint32_t)Zs[8 * tid + q] << (4 * q);
        p.qz[unit * 4 + tid] = zw;
      }
    }
    const int owner = i >> 5;
    double err = 0.0;
    if (qd == owner) {
      const float S = Ss[r];
      const int z = Zs[r];
      const double w = wr[i];
      const float v = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn((float)w, S)), (float)z), 0.f), 15.f);
      const int code = (int)v;
      const int e = i & 7;  // nibble of channel offset e: even e -> e / 2, odd e -> 4 + e / 2
      words[(i & 31) >> 3] |= (uint32_t)code << (4 * ((e & 1) ? 4 + (e >> 1) : (e >> 1)));
      err = __ddiv_rn(__dsub_rn(w, __dmul_rn((double)(code - z), (double)S)), Ub[i * kUbStride + i]);
      if (valid) p.E[(size_t)n * kGB + i] = err;
    }
    err = __shfl_sync(0xFFFFFFFFu, err, (lane & ~3) | owner);
    const double* ui = Ub + i * kUbStride;
    for (int j = max(i + 1, 32 * qd); j < 32 * qd + 32; ++j) wr[j] = __dsub_rn(wr[j], __dmul_rn(err, ui[j]));
  }
  // packed words: this thread's 32 columns are chunk (b0 / 32 + qd) of row r
  const size_t tile = (size_t)rb * (K / 32) + b0 / 32 + qd;
#pragma unroll
  for (int j = 0; j < 4; ++j) p.qw[tile * 128 + r * 4 + j] = valid ? words[j] : 0u;
}

// Wc[n][j] -= sum_t E[n][t] U[b0 + t][j] for j >= b0 + 128: 64 x 64 output tile per CTA, t in chunks of 16; the
// sum is formed in t order with separately rounded products, then subtracted once.
__global__ void __launch_bounds__(256) gptq_lazy_kernel(const GptqParams p, int b0) {
  __shared__ double Es[16][kT + 1];
  __shared__ double Us[16][kT + 1];
  const int K = p.K;
  const int j0 = b0 + kGB + blockIdx.x * kT, n0 = blockIdx.y * kT;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
  for (int t0 = 0; t0 < kGB; t0 += 16) {
    for (int e = threadIdx.x; e < 16 * kT; e += 256) {
      const int tt = e / kT, a = e % kT;
      Es[tt][a] = (n0 + a < p.N) ? p.E[(size_t)(n0 + a) * kGB + t0 + tt] : 0.0;
      Us[tt][a] = p.Xi[(size_t)(K - 1 - b0 - t0 - tt) * K + (K - 1 - (j0 + a))];
    }
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < 16; ++tt)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v)
          acc[u][v] = __dadd_rn(acc[u][v], __dmul_rn(Es[tt][ty + 16 * u], Us[tt][tx + 16 * v]));
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int nn = n0 + ty + 16 * u;
    if (nn >= p.N) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      double* w = p.Wc + (size_t)nn * K + j0 + tx + 16 * v;
      *w = __dsub_rn(*w, acc[u][v]);
    }
  }
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct GptqLayout {
  size_t hr, xi, wc, e, d, total;
};
GptqLayout gptq_layout(int N, int K) {
  GptqLayout L{};
  const size_t Np = (size_t)(N + 31) / 32 * 32;
  L.hr = 0;
  L.xi = L.hr + align256((size_t)K * K * 8);
  L.wc = L.xi + align256((size_t)K * K * 8);
  L.e = L.wc + align256((size_t)N * K * 8);
  L.d = L.e + align256(Np * kGB * 8);
  L.total = L.d + align256((size_t)kT * kT * 8);
  return L;
}

bool attrs_set() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(gptq_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)gptq_block_smem()) != cudaSuccess)
      return false;
    if (cudaFuncSetAttribute(trtri_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(2 * kT * (kT + 1) * sizeof(double))) != cudaSuccess)
      return false;
    if (cudaFuncSetAttribute(chol_panel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(2 * kT * (kT + 1) * sizeof(double))) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

}  // namespace

size_t gptq_workspace_bytes(int N, int K) { return gptq_layout(N, K).total; }

awq_status gptq_launch(const uint16_t* W, const uint16_t* xcal, int N, int K, int R, int g, double damp,
                       uint32_t* qw, uint16_t* scales, uint32_t* qz, void* ws, size_t ws_bytes, unsigned* status,
                       cudaStream_t st) {
  const GptqLayout L = gptq_layout(N, K);
  if (ws == nullptr || ws_bytes < L.total) return AWQ_ERR_WORKSPACE;
  if (!attrs_set()) return AWQ_ERR_CUDA;
  char* base = static_cast<char*>(ws);
  double* Hr = reinterpret_cast<double*>(base + L.hr);
  double* Xi = reinterpret_cast<double*>(base + L.xi);
  double* D = reinterpret_cast<double*>(base + L.d);
  GptqParams p;
  p.Xi = Xi;
  p.Wc = reinterpret_cast<double*>(base + L.wc);
  p.E = reinterpret_cast<double*>(base + L.e);
  p.qw = qw;
  p.scales = scales;
  p.qz = qz;
  p.N = N;
  p.K = K;
  p.g = g;
  p.G = K / g;
  const int nb = K / kT;
  const int RB = (N + 31) / 32;
  // padding rows N .. N_pad - 1 of the packed arrays are written by the block kernel (code, scale, zero 0)
  to_f64_kernel<<<num_sms() * 8, 256, 0, st>>>(reinterpret_cast<const __half*>(W), (long long)N * K, p.Wc);
  gram_rev_kernel<<<nb * (nb + 1) / 2, 256, 0, st>>>(reinterpret_cast<const __half*>(xcal), R, K, damp, Hr);
  if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
  const size_t panel_smem = 2 * kT * (kT + 1) * sizeof(double);
  for (int c = 0; c < nb; ++c) {
    chol_panel_kernel<<<nb - c, 256, panel_smem, st>>>(Hr, K, c, D, status);
    const int m = nb - c - 1;
    chol_update_kernel<<<m * (m + 1) / 2 + 1, 256, 0, st>>>(Hr, K, c, D);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
  }
  const size_t tri_smem = 2 * kT * (kT + 1) * sizeof(double);
  if (cudaMemsetAsync(Xi, 0, (size_t)K * K * sizeof(double), st) != cudaSuccess) return AWQ_ERR_CUDA;
  for (int k = 0; k < nb; ++k) {
    trtri_solve_kernel<<<k + 1, 256, tri_smem, st>>>(Hr, Xi, K, k);
    if (k + 1 < nb) trtri_update_kernel<<<(nb - k - 1) * (k + 1), 256, 0, st>>>(Hr, Xi, K, k);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
  }
  for (int b0 = 0; b0 < K; b0 += kGB) {
    gptq_block_kernel<<<RB, kGptqThreads, gptq_block_smem(), st>>>(p, b0);
    if (b0 + kGB < K) {
      const dim3 grid((unsigned)((K - b0 - kGB) / kT), (unsigned)((N + kT - 1) / kT));
      gptq_lazy_kernel<<<grid, 256, 0, st>>>(p, b0);
    }
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
  }
  return AWQ_OK;
}

}  // namespace awq
