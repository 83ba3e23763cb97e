// gemv.cu -- W4A16 decode kernel ("GEMV mode" of the AutoAWQ page: single batch, top speed).
//
// y[m][n] = sum_g S[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x'[m][k]   for up to MT rows of x' per pass.
//
// Units.  The packed layout stores each (32-row block rb, 128-channel group g) as 2048 contiguous
// bytes, so unit u = rb * G + g is one 2 KB stretch and the weight is U = RB * G consecutive units.
// Each of the P CTAs owns a balanced contiguous range (q = U / P units, one more for the first U % P
// CTAs); its NW warps split that range into NW balanced contiguous sub-ranges.  Inside a warp, lane r owns row 32*rb + r: a unit is four
// coalesced 128-bit loads per lane (512 contiguous bytes per warp-instruction), dequantized in registers
// with the int4->fp16 bit trick, multiplied with x' in packed half2 FMAs (two independent accumulators,
// 16 products each, flushed to fp32 every 64 channels), scaled by the group's fp16 scale and
// accumulated in fp32.  No cross-lane reduction is needed: the layout gives each lane a whole row.
//
// Streaming.  Each warp owns a contiguous sub-range and streams its codes through its own
// shared-memory ring of kRing 2 KB unit slots with TMA bulk copies, so the bytes in flight cost no
// registers; the lanes read each unit's scales and zeros themselves, two units ahead.  As many 8-warp
// CTAs per SM as the launch's shared memory allows (3 at K = 4096) keep up to 24 warps issuing.  Before
// griddepcontrol.wait a kernel touches only its weights -- every warp issues one bulk L2 prefetch of its
// whole sub-range and fills its ring -- so with programmatic dependent launch the weight stream of the
// next kernel on the stream starts while this one drains.
//
// Combining split row blocks.  A row block wholly inside one warp's sub-range is written directly.  A
// row block split between warps of one CTA is summed in shared memory, in warp order.  A row block
// split between CTAs gets one fp32 partial per CTA in the workspace slot (rb, c - first_cta(rb)); the
// CTA that brings the row block's counter to its final value sums the slots in slot order
// (deterministic), writes fp16 y and resets the counter to 0 for the next call.
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
  unsigned* status;  // device status word (bounded waits)
  const uint8_t* pf;              // optional: bytes to prefetch into L2 for a later call (NULL: none)
  unsigned long long pf_bytes;    // their size (a multiple of 16)
  unsigned long long pf_share;    // bytes per CTA (a multiple of 16)
  int U;   // units = RB * G
  int P;   // CTAs sharing the units: CTA c owns q units, plus one more if c < r
  int q, r;
  int M, N, Np, K, G, RB, S, m0;
};

__device__ __forceinline__ int cta_first_unit(const GemvParams& p, int c) { return p.q * c + min(c, p.r); }
__device__ __forceinline__ int cta_of_unit(const GemvParams& p, int u) {
  const int b = p.r * (p.q + 1);
  return u < b ? u / (p.q + 1) : p.r + (u - b) / p.q;
}

// One shared-memory ring slot per unit: its 2048 B of codes (one TMA bulk copy).  The unit's 64 B of
// scales and 16 B of zeros are read by the lanes themselves, one unit ahead.
constexpr int kSlotBytes = 2048;
constexpr int kSlotStride = 2048;
#ifndef AWQ_GEMV_RING
#define AWQ_GEMV_RING 4
#endif
constexpr int kRing = AWQ_GEMV_RING;  // units in flight per warp
__host__ __device__ constexpr int ring_bytes(int nw) { return nw * kRing * kSlotStride; }
// Activations staged in shared memory (one TMA copy per row after the dependency wait) when they fit.
constexpr int kXsMaxBytes = 32 * 1024;

// Copies the codes of unit u into a ring slot; completion is counted on `bar`.
__device__ __forceinline__ void issue_unit(const GemvParams& p, int u, uint8_t* slot, uint64_t* bar) {
  mbar_arrive_expect_tx(bar, kSlotBytes);
  bulk_g2s(slot, p.qw + (size_t)u * 128, 2048u, bar);
}

// Scale (as float) and zero point of this lane's row in unit u (coalesced across the warp).
__device__ __forceinline__ void load_meta(const GemvParams& p, int u, int lane, float& sc, uint32_t& z) {
  sc = __half2float(p.scales[(size_t)u * 32 + lane]);
  z = (p.qzeros[(size_t)u * 4 + (lane >> 3)] >> (4 * (lane & 7))) & 0xFu;
}

template <int MT>
__device__ __forceinline__ void unit_dot(const uint4 (&w)[4], float sc, uint32_t z,
                                         const uint16_t* __restrict__ const (&xg)[MT],
                                         float (&yacc)[MT]) {
  const __half2 z1024 = zero_1024(z), nz64 = neg_zero_64(z);
  const uint32_t magic = magic_1024x2();
  float part[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) part[m] = 0.f;
#pragma unroll(MT >= 4 ? 1 : 2)
  for (int cp = 0; cp < 2; ++cp) {  // pairs of 32-channel chunks
    __half2 acc[2][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[0][m] = acc[1][m] = u32_as_h2(0u);
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      const int c = cp * 2 + c2;
      const uint32_t ww[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __half2 d[4];
        word_minus_zero(ww[j], z1024, nz64, magic, d);
        const int a = j & 1;  // two independent accumulator chains
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint4 xv = ldg_cached(xg[m] + c * 32 + j * 8);
          acc[a][m] = __hfma2(d[0], u32_as_h2(xv.x), acc[a][m]);
          acc[a][m] = __hfma2(d[1], u32_as_h2(xv.y), acc[a][m]);
          acc[a][m] = __hfma2(d[2], u32_as_h2(xv.z), acc[a][m]);
          acc[a][m] = __hfma2(d[3], u32_as_h2(xv.w), acc[a][m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m)
      part[m] += (__low2float(acc[0][m]) + __high2float(acc[0][m])) +
                 (__low2float(acc[1][m]) + __high2float(acc[1][m]));
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) yacc[m] = fmaf(sc, part[m], yacc[m]);
}

template <int MT>
__device__ __forceinline__ void store_y(const GemvParams& p, int rb, int lane, const float (&v)[MT]) {
  const int n = rb * 32 + lane;
  const int mcount = min(MT, p.M - p.m0);
  if (n < p.N) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (m < mcount) p.y[(size_t)(p.m0 + m) * p.N + n] = __half_as_ushort(__float2half_rn(v[m]));
  }
}

// Sum over the CTAs that share row block r (called by the one warp per CTA that combines r).
template <int MT>
__device__ __forceinline__ void cross_cta_combine(const GemvParams& p, int r, int lane, const float (&part)[MT]) {
  const int cf = cta_of_unit(p, r * p.G);
  const int cl = cta_of_unit(p, r * p.G + p.G - 1);
  const int nc = cl - cf + 1;
  const int slot = (int)blockIdx.x - cf;
  float* base = p.ws_part + (size_t)r * p.S * 32 * MT;  // slots of row block r
#pragma unroll
  for (int m = 0; m < MT; ++m) base[(size_t)(slot * MT + m) * 32 + lane] = part[m];
  __threadfence();
  __syncwarp();
  unsigned old = 0;
  if (lane == 0) old = atomicAdd(&p.ws_cnt[r], 1u);
  old = __shfl_sync(0xFFFFFFFFu, old, 0);
  if (old != (unsigned)(nc - 1)) return;
  __threadfence();
  float sum[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) sum[m] = 0.f;
  for (int j = 0; j < nc; ++j) {
#pragma unroll
    for (int m = 0; m < MT; ++m) sum[m] += (j == slot) ? part[m] : __ldcg(&base[(size_t)(j * MT + m) * 32 + lane]);
  }
  store_y<MT>(p, r, lane, sum);
  if (lane == 0) p.ws_cnt[r] = 0u;
}

#ifndef AWQ_GEMV_MINB_MT1
#define AWQ_GEMV_MINB_MT1 3
#endif
#ifndef AWQ_GEMV_META_AHEAD
#define AWQ_GEMV_META_AHEAD 2
#endif
// NW warps per CTA: 8, 16 or 32.  A 16-warp CTA takes half an SM (64 registers per thread), so the
// next kernel's CTAs can already be resident beside it; a 32-warp CTA takes a whole SM.
template <int MT, int NW, bool XS>
__global__ void __launch_bounds__(NW * 32, (NW == 32 ? 1 : NW == 16 ? 2 : MT == 1 ? AWQ_GEMV_MINB_MT1 : MT == 2 ? 2 : 1))
    gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(128) uint8_t ring_smem[];
  __shared__ __align__(8) uint64_t full[NW][kRing];
  __shared__ __align__(8) uint64_t xbar;
  __shared__ float s_part[NW][2][MT * 32];
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = p.G;
  const int c = blockIdx.x;
  const int cu0 = cta_first_unit(p, c), n = p.q + (c < p.r ? 1 : 0), cu1 = cu0 + n;
  const int wq = n / NW, wr = n % NW;  // NW is a power of two
  const int wu0 = cu0 + wq * warp + min(warp, wr), nw = wq + (warp < wr ? 1 : 0), wu1 = wu0 + nw;
  const bool active = nw > 0;
  uint8_t* ring = ring_smem + (size_t)warp * kRing * kSlotStride;

  // Before the dependency wait: only weights.  The warp's whole sub-range goes towards L2, and the
  // first kRing units into this warp's shared-memory ring.
  if (XS && threadIdx.x == 0) {
    mbar_init(&xbar, 1);
    fence_mbar_init();
  }
  if (XS) __syncthreads();
  if (active && lane == 0) {
#pragma unroll
    for (int i = 0; i < kRing; ++i) mbar_init(&full[warp][i], 1);
    fence_mbar_init();
    const char* base = reinterpret_cast<const char*>(p.qw + (size_t)wu0 * 128);
    for (int off = 0; off < nw * 2048; off += 32768)
      prefetch_l2_bulk(base + off, (unsigned)min(32768, nw * 2048 - off));
    prefetch_l2_bulk(p.scales + (size_t)wu0 * 32, (unsigned)(nw * 64));
    prefetch_l2_bulk(p.qzeros + (size_t)wu0 * 4, (unsigned)(nw * 16));
    for (int i = 0; i < kRing && i < nw; ++i) issue_unit(p, wu0 + i, ring + i * kSlotStride, &full[warp][i]);
  }
  // L2 prefetch of a later call's weights (a caller's hint), spread over the CTAs; weights only.
  if (p.pf != nullptr && p.m0 == 0 && threadIdx.x == (NW - 1) * 32) {
    const unsigned long long a = (unsigned long long)c * p.pf_share;
    const unsigned long long e = a + p.pf_share < p.pf_bytes ? a + p.pf_share : p.pf_bytes;
    for (unsigned long long o = a; o < e; o += 32768ull)
      prefetch_l2_bulk(p.pf + o, (unsigned)(e - o < 32768ull ? e - o : 32768ull));
  }
  __syncwarp();
  float sc = 0.f, sc1 = 0.f;
  uint32_t z = 0u, z1 = 0u;
  if (active) load_meta(p, wu0, lane, sc, z);  // weights only: no dependency on earlier kernels
  if (AWQ_GEMV_META_AHEAD == 2 && nw > 1) load_meta(p, wu0 + 1, lane, sc1, z1);
  pdl_wait_prior_grids();  // activations, outputs and workspace follow the stream order

  const int mcount = min(MT, p.M - p.m0);
  const uint16_t* xrow[MT];
  if (XS) {  // x' rows of this pass -> shared memory, one bulk copy per row
    uint16_t* xs = reinterpret_cast<uint16_t*>(ring_smem + ring_bytes(NW));
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(&xbar, (unsigned)(mcount * p.K * 2));
      for (int m = 0; m < mcount; ++m) bulk_g2s(xs + m * p.K, p.x + (size_t)(p.m0 + m) * p.K, (unsigned)(p.K * 2), &xbar);
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) xrow[m] = xs + min(m, mcount - 1) * p.K;
  } else {
#pragma unroll
    for (int m = 0; m < MT; ++m) xrow[m] = p.x + (size_t)(p.m0 + min(m, mcount - 1)) * p.K;
  }
  const int rb_f = active ? wu0 / G : -1;  // the only division of the main path
  const int g0 = active ? wu0 - rb_f * G : 0;

  bool ok = true;
  if (XS && active) ok = __all_sync(0xFFFFFFFFu, mbar_wait_backoff(&xbar, 0u, p.status));
  int rb = rb_f, g = g0, rb_l = rb_f;
  int t = 0;  // units of this warp consumed so far
  while (t < nw && ok) {  // segments: the units of one row block inside this warp's range
    const int seg = min(nw - t, G - g);
    const bool whole = (g == 0) && (seg == G);
    float yacc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) yacc[m] = 0.f;
    for (int i = 0; i < seg; ++i, ++t) {
      const int si = t & (kRing - 1);
      uint8_t* slot = ring + si * kSlotStride;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait_backoff(&full[warp][si], (unsigned)(t / kRing) & 1u, p.status));
      if (!ok) break;  // warp-uniform
      float scn = 0.f;
      uint32_t zn = 0u;
      // scale and zero of a later unit: the next one, or the one after it (two in flight)
      if (t + AWQ_GEMV_META_AHEAD < nw) load_meta(p, wu0 + t + AWQ_GEMV_META_AHEAD, lane, scn, zn);
      uint4 w[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) w[cc] = *reinterpret_cast<const uint4*>(slot + cc * 512 + lane * 16);
      const uint16_t* xg[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) xg[m] = xrow[m] + (g + i) * 128;
      unit_dot<MT>(w, sc, z, xg, yacc);
      __syncwarp();  // every lane has consumed the slot
      if (lane == 0 && t + kRing < nw) {
        fence_proxy_async_smem();  // our generic reads of the slot before the async-proxy refill
        issue_unit(p, wu0 + t + kRing, slot, &full[warp][si]);
      }
      if (AWQ_GEMV_META_AHEAD == 2) {
        sc = sc1;
        z = z1;
        sc1 = scn;
        z1 = zn;
      } else {
        sc = scn;
        z = zn;
      }
    }
    if (!ok) break;
    if (whole) {
      store_y<MT>(p, rb, lane, yacc);
    } else {
      const int slot = (rb == rb_f) ? 0 : 1;
#pragma unroll
      for (int m = 0; m < MT; ++m) s_part[warp][slot][m * 32 + lane] = yacc[m];
    }
    rb_l = rb;
    ++rb;
    g = 0;
  }
  if (!ok && lane == 0) {  // give up: wait (bounded) for this warp's copies still in flight
    for (int j = t; j < nw && j < t + kRing; ++j)
      mbar_wait(&full[warp][j & (kRing - 1)], (unsigned)(j / kRing) & 1u, p.status);
  }
  __syncthreads();
  if (!active || !ok) return;

  // A split row block r is combined by the warp holding its first unit inside this CTA.
  auto combine = [&](int r) {
    const int a = max(r * G, cu0), b = min((r + 1) * G, cu1);
    float sum[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) sum[m] = 0.f;
    for (int j = warp; j < NW; ++j) {
      const int j0 = cu0 + wq * j + min(j, wr), jn = wq + (j < wr ? 1 : 0);
      if (j0 >= b) break;
      if (jn == 0) continue;
      const int slot = (j0 >= r * G) ? 0 : 1;  // r is warp j's first row block iff it starts at or before j0
#pragma unroll
      for (int m = 0; m < MT; ++m) sum[m] += s_part[j][slot][m * 32 + lane];
    }
    if (a == r * G && b == (r + 1) * G) store_y<MT>(p, r, lane, sum);
    else cross_cta_combine<MT>(p, r, lane, sum);
  };
  const bool whole_f = (g0 == 0) && (nw >= G);
  const bool owner_f = (g0 == 0) || (wu0 == cu0);
  if (owner_f && !whole_f) combine(rb_f);
  if (rb_l != rb_f && wu1 - rb_l * G < G) combine(rb_l);
}

// ------------------------------------------------------------------------------------------ host
#ifndef AWQ_GEMV_CTAS_PER_SM
#define AWQ_GEMV_CTAS_PER_SM 4
#endif
#ifndef AWQ_GEMV_WHOLE_RB_MAX_UNITS
#define AWQ_GEMV_WHOLE_RB_MAX_UNITS 48
#endif
#ifndef AWQ_GEMV_BIG_CTA_WARPS  // warps of the one-row-block-per-CTA plan: 16 or 32
#define AWQ_GEMV_BIG_CTA_WARPS 16
#endif
#ifndef AWQ_GEMV_STAGE_X  // stage activations in shared memory when they fit
#define AWQ_GEMV_STAGE_X 1
#endif

namespace {

int pick_mt(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

template <int MT, int NW, bool XS>
bool gemv_smem_attr() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(gemv_kernel<MT, NW, XS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ring_bytes(NW) + (XS ? kXsMaxBytes : 0)) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

#ifndef AWQ_GEMV_OCC_EXACT
#define AWQ_GEMV_OCC_EXACT 1
#endif
// 8-warp CTAs of one launch resident per SM (at most AWQ_GEMV_CTAS_PER_SM), for the shared memory the
// launch really uses: the rings plus xs_bytes of staged activations (0: not staged).
template <int MT>
int resident_ctas_mt(int xs_bytes) {
  static int cached[64][kXsMaxBytes / 256 + 1] = {{0}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!AWQ_GEMV_OCC_EXACT) xs_bytes = kXsMaxBytes;  // sized for the largest staging
  const int i = (xs_bytes + 255) / 256;
  if (cached[dev][i] == 0) {
    int occ = 0;
    cudaError_t e;
    if (xs_bytes > 0) {
      gemv_smem_attr<MT, 8, true>();
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_kernel<MT, 8, true>, 8 * 32,
                                                        ring_bytes(8) + i * 256);
    } else {
      gemv_smem_attr<MT, 8, false>();
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_kernel<MT, 8, false>, 8 * 32, ring_bytes(8));
    }
    if (e != cudaSuccess || occ < 1) occ = 1;
    cached[dev][i] = occ < AWQ_GEMV_CTAS_PER_SM ? occ : AWQ_GEMV_CTAS_PER_SM;
  }
  return cached[dev][i];
}

int resident_ctas(int MT, int xs_bytes) {
  switch (MT) {
    case 1: return resident_ctas_mt<1>(xs_bytes);
    default: return resident_ctas_mt<2>(xs_bytes);
  }
}
int resident_ctas_big(int MT) {  // MT 4 and 8 never stage activations
  static int cached[64][2] = {{0}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  const int i = MT == 4 ? 0 : 1;
  if (cached[dev][i] == 0) {
    int occ = 0;
    cudaError_t e;
    if (MT == 4) {
      gemv_smem_attr<4, 8, false>();
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_kernel<4, 8, false>, 256, ring_bytes(8));
    } else {
      gemv_smem_attr<8, 8, false>();
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_kernel<8, 8, false>, 256, ring_bytes(8));
    }
    if (e != cudaSuccess || occ < 1) occ = 1;
    cached[dev][i] = occ < AWQ_GEMV_CTAS_PER_SM ? occ : AWQ_GEMV_CTAS_PER_SM;
  }
  return cached[dev][i];
}

struct GemvPlan {
  int MT, NW, RB, G, S, Np, P;
  bool xs;  // activations staged in shared memory
  int U, q, r;
  size_t part_bytes;
};

// Three shapes of work, chosen so that all CTAs of a launch are resident at once:
//  - at most one row block per SM (and M <= 2): one 16-warp CTA per row block; its warps split the
//    row block's groups and combine in shared memory -- no partial sum leaves a CTA;
//  - short row blocks (G <= 48) that fit the 8-warp CTAs resident on all SMs: one 8-warp CTA per row
//    block, likewise self-contained;
//  - otherwise the units are spread evenly over all resident 8-warp CTAs and the row blocks cut by CTA
//    boundaries are combined in the workspace.
GemvPlan plan_gemv(int M, int N, int K) {
  GemvPlan pl{};
  pl.MT = pick_mt(M);
  pl.Np = (N + 31) / 32 * 32;
  pl.RB = pl.Np / 32;
  pl.G = K / 128;
  pl.U = pl.RB * pl.G;
  const int sms = num_sms();
  pl.S = 1;
  pl.part_bytes = 0;
  if (pl.MT <= 2 && pl.RB <= sms) {
    pl.NW = AWQ_GEMV_BIG_CTA_WARPS;
    pl.P = pl.RB;
  } else {
    pl.NW = 8;
    const int xs_bytes = (AWQ_GEMV_STAGE_X && pl.MT <= 2 && pl.MT * K * 2 <= kXsMaxBytes) ? pl.MT * K * 2 : 0;
    int p_bal = sms * (pl.MT <= 2 ? resident_ctas(pl.MT, xs_bytes) : resident_ctas_big(pl.MT));
    const int by_units = pl.U / 8 > 0 ? pl.U / 8 : 1;
    if (p_bal > by_units) p_bal = by_units;
    if (pl.RB <= p_bal && pl.G <= AWQ_GEMV_WHOLE_RB_MAX_UNITS) {
      pl.P = pl.RB;
    } else {
      pl.P = p_bal;
      const int L = pl.U / pl.P;  // >= 1 units per CTA
      pl.S = pl.G >= 2 ? (pl.G - 2) / L + 2 : 1;
      pl.part_bytes = (size_t)pl.RB * pl.S * 32 * pl.MT * sizeof(float);
    }
  }
  pl.q = pl.U / pl.P;
  pl.r = pl.U % pl.P;
  pl.xs = AWQ_GEMV_STAGE_X && pl.MT <= 2 && pl.MT * K * 2 <= kXsMaxBytes;
  return pl;
}

template <int MT, int NW, bool XS>
cudaError_t launch_mt(const GemvParams& p, cudaStream_t st) {
  if (!gemv_smem_attr<MT, NW, XS>()) return cudaErrorInvalidValue;
  const size_t smem = (size_t)ring_bytes(NW) + (XS ? (size_t)MT * p.K * 2 : 0);
  return launch_pdl(gemv_kernel<MT, NW, XS>, dim3((unsigned)p.P), dim3(NW * 32), smem, st, p);
}

}  // namespace

size_t gemv_workspace_bytes(int M, int N, int K) {
  const GemvPlan pl = plan_gemv(M, N, K);
  return pl.part_bytes == 0 ? 0 : kWorkspaceCounterBytes + pl.part_bytes;
}

awq_status gemv_launch(const uint16_t* x, const uint32_t* qw, const uint16_t* scales, const uint32_t* qzeros,
                       uint16_t* y, int M, int N, int K, void* ws, size_t ws_bytes, unsigned* dev_status,
                       cudaStream_t st, const void* pf, size_t pf_bytes) {
  const GemvPlan pl = plan_gemv(M, N, K);
  if ((size_t)pl.RB * 4 > kWorkspaceCounterBytes) return AWQ_ERR_UNSUPPORTED;
  if (pl.part_bytes > 0 && (ws == nullptr || ws_bytes < kWorkspaceCounterBytes + pl.part_bytes))
    return AWQ_ERR_WORKSPACE;
  GemvParams p;
  p.x = x;
  p.qw = reinterpret_cast<const uint4*>(qw);
  p.scales = reinterpret_cast<const __half*>(scales);
  p.qzeros = qzeros;
  p.y = y;
  p.ws_cnt = static_cast<unsigned*>(ws);
  p.ws_part = ws ? reinterpret_cast<float*>(static_cast<char*>(ws) + kWorkspaceCounterBytes) : nullptr;
  p.status = dev_status;
  p.pf = pf_bytes > 0 ? static_cast<const uint8_t*>(pf) : nullptr;
  p.pf_bytes = pf_bytes;
  p.pf_share = ((pf_bytes + (size_t)pl.P - 1) / (size_t)pl.P + 15) / 16 * 16;
  p.U = pl.U;
  p.P = pl.P;
  p.q = pl.q;
  p.r = pl.r;
  p.M = M;
  p.N = N;
  p.Np = pl.Np;
  p.K = K;
  p.G = pl.G;
  p.RB = pl.RB;
  p.S = pl.S;
  // passes of MT rows run one after the other on the stream and share the workspace
  for (int m0 = 0; m0 < M; m0 += pl.MT) {
    p.m0 = m0;
    cudaError_t e;
    if (pl.NW == 16 || pl.NW == 32) {
      constexpr int BW = AWQ_GEMV_BIG_CTA_WARPS;
      static_assert(ring_bytes(BW) + kXsMaxBytes <= 227 * 1024, "GEMV shared memory over the per-CTA limit");
      if (pl.MT == 1) e = pl.xs ? launch_mt<1, BW, true>(p, st) : launch_mt<1, BW, false>(p, st);
      else e = pl.xs ? launch_mt<2, BW, true>(p, st) : launch_mt<2, BW, false>(p, st);
    } else {
      switch (pl.MT) {
        case 1: e = pl.xs ? launch_mt<1, 8, true>(p, st) : launch_mt<1, 8, false>(p, st); break;
        case 2: e = pl.xs ? launch_mt<2, 8, true>(p, st) : launch_mt<2, 8, false>(p, st); break;
        case 4: e = launch_mt<4, 8, false>(p, st); break;
        default: e = launch_mt<8, 8, false>(p, st); break;
      }
    }
    if (e != cudaSuccess) return AWQ_ERR_CUDA;
  }
  return AWQ_OK;
}

}  // namespace awq
