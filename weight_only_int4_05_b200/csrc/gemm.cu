// gemm.cu -- W4A16 prefill kernel ("GEMM mode" of the AutoAWQ page: long context, many tokens).
//
// y^T tile [128 weight rows][BT tokens] = dequant(W)[128][K] . x'[BT][K]^T on the tcgen05 tensor cores.
// Weights are the UMMA A operand (M = 128 rows of N), activations the B operand (N = BT tokens), so a
// small token count still maps onto a full-height MMA.
//
// Per CTA (64 + 128 * kDequantWG threads, one output tile, k-blocks of 64 channels through an ST-stage ring):
//   warp 0, lane 0  producer: four TMA tensor copies per stage -- the codes of the tile's 4 row blocks, their
//                   fp16 scales and their packed zeros, and a 2-D tensor copy of the x' tile in the 128-byte swizzle
//                   layout; all complete on full[s].  Weight copies for the first ring are issued before
//                   griddepcontrol.wait, so they overlap the previous kernel on the stream.
//   warps 2..       kDequantWG (4) dequant warpgroups take k-blocks round robin, so one warpgroup's latency
//                   overlaps the others'.  Thread r of a warpgroup owns weight row r of the tile; it turns 64 packed codes into
//                   fp16 (q - z) * S (exact q - z by the int4->fp16 bit trick, one rounding for the
//                   scale) and writes them in the 128-byte swizzle K-major layout the MMA reads, then
//                   fence.proxy.async + arrive on afull[s].  After the main loop the same warps are
//                   the epilogue (the warpgroups split the columns): tcgen05.ld of their 32-lane TMEM
//                   quarter, fp16 convert, store y.
//   warp 1          allocates TMEM (fp32 accumulator, BT columns); lane 0 issues 4 x
//                   tcgen05.mma.kind::f16 (128 x BT x 16) per k-block and tcgen05.commit -> empty[s].
// Every mbarrier wait is bounded (see common.cuh); a timeout is recorded in the status word, the CTA
// drains its own copies and MMAs, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace awq {

constexpr int kBN = 128;  // weight rows per tile (UMMA M)
constexpr int kBK = 64;   // channels per k-block (one 128-byte swizzle row of fp16)
#ifndef AWQ_GEMM_DEQUANT_WG
#define AWQ_GEMM_DEQUANT_WG 4
#endif
constexpr int kDequantWG = AWQ_GEMM_DEQUANT_WG;            // dequant warpgroups, k-blocks round robin
constexpr int kGemmThreads = 64 + 128 * kDequantWG;
constexpr int kMaxSmem = 232448;  // opt-in dynamic shared memory per block on sm_100

// byte offsets inside one pipeline stage
constexpr int kOffA = 0;                       // 128 x 64 fp16, swizzled: 16 KB
constexpr int kOffB = kBN * kBK * 2;           // BT x 64 fp16, swizzled: BT * 128 B
__host__ __device__ constexpr int off_pk(int BT) { return kOffB + BT * 128; }  // 4 x 1 KB packed codes
__host__ __device__ constexpr int off_sc(int BT) { return off_pk(BT) + 4096; } // 128 fp16 scales
__host__ __device__ constexpr int off_z(int BT) { return off_sc(BT) + 256; }   // 128 packed zeros
__host__ __device__ constexpr int stage_bytes(int BT) { return (off_z(BT) + 256 + 1023) / 1024 * 1024; }

struct GemmParams {
  const uint4* qw;
  const uint16_t* scales;
  const uint32_t* qzeros;
  uint16_t* y;
  unsigned* status;
  int epi;     // 0: y [M][N]; 1: gate|up, y [M][N/2] = silu(row 32j + i) * row 32j + 16 + i (i < 16)
  int gshift;  // group of k-block kb: kb >> gshift (group size 64 << gshift)
  float* ws_part;    // split-K partial tiles [tile][split][BT][128] fp32 (splits > 1 only)
  unsigned* ws_cnt;  // per-tile arrival counters (zero between calls)
  int M, N, Np, K, KB, BT, ST, tmem_cols;
  int splits, kb_per_split;  // k-blocks [split * kb_per_split, ...) per CTA
  int tile_base, n_tiles;    // CTA x handles output tile tile_base + x (n-tile = tile % n_tiles, t-tile = tile / n_tiles)
  uint32_t idesc;
};

// Producer (lane 0 of warp 0).  Four TMA copies per stage: a 3-D box of the codes of the tile's 4 row
// blocks (2 chunks of 512 B each), 2-D boxes of their scales (4 x 64 B) and zeros (4 x 16 B) of the group
// the k-block falls in (a k-block of 64 channels never straddles a group of 64, 128 or 256), and the
// x' tile in the 128-byte swizzle layout.  Row blocks past the end of the weight come back zero-filled.
struct GemmMaps {
  CUtensorMap x, codes, scales, zeros;
};

__device__ __forceinline__ void gemm_producer(const GemmMaps* maps, const GemmParams& p, uint8_t* smem,
                                              uint64_t* full, uint64_t* empty, volatile int* abort_flag,
                                              int n0, int t0, int kb0, int nkb) {
  const unsigned tx = (unsigned)p.BT * 128u + 4096u + 256u + 64u;
  const int rb0 = n0 / 32;
  auto issue_w = [&](int kk, int s) {  // kk: k-block index within this CTA's range
    const int kb = kb0 + kk, g = kb >> p.gshift;
    uint8_t* st = smem + (size_t)s * stage_bytes(p.BT);
    mbar_arrive_expect_tx(&full[s], tx);
    tma_load_3d(st + off_pk(p.BT), &maps->codes, 0, kb * 2, rb0, &full[s]);
    tma_load_2d(st + off_sc(p.BT), &maps->scales, g * 32, rb0, &full[s]);
    tma_load_2d(st + off_z(p.BT), &maps->zeros, g * 4, rb0, &full[s]);
  };
  auto issue_x = [&](int kk, int s) {
    tma_load_2d(smem + (size_t)s * stage_bytes(p.BT) + kOffB, &maps->x, (kb0 + kk) * kBK, t0, &full[s]);
  };
  const int pre = nkb < p.ST ? nkb : p.ST;
  for (int kk = 0; kk < pre; ++kk) issue_w(kk, kk);
  pdl_wait_prior_grids();
  for (int kk = 0; kk < pre; ++kk) issue_x(kk, kk);
  int issued = pre;
  for (int kk = pre; kk < nkb; ++kk) {
    const int s = kk % p.ST, use = kk / p.ST;
    if (*abort_flag || !mbar_wait(&empty[s], (use - 1) & 1, p.status)) {
      *abort_flag = 1;
      break;
    }
    issue_w(kk, s);
    issue_x(kk, s);
    issued = kk + 1;
  }
  if (*abort_flag) {  // wait (bounded) until every copy this thread issued has landed
    for (int kk = issued > p.ST ? issued - p.ST : 0; kk < issued; ++kk)
      mbar_wait(&full[kk % p.ST], (kk / p.ST) & 1, p.status);
  }
}

__device__ __forceinline__ void gemm_mma(const GemmParams& p, uint8_t* smem, uint64_t* full, uint64_t* afull,
                                         uint64_t* empty, uint64_t* accf, volatile int* abort_flag,
                                         uint32_t tmem, int nkb) {
  for (int kb = 0; kb < nkb; ++kb) {
    const int s = kb % p.ST;
    const unsigned par = (kb / p.ST) & 1;
    if (*abort_flag || !mbar_wait(&full[s], par, p.status) || !mbar_wait(&afull[s], par, p.status)) {
      *abort_flag = 1;
      break;
    }
    tc_fence_after_sync();
    const uint32_t a = smem_u32(smem + (size_t)s * stage_bytes(p.BT) + kOffA);
    const uint32_t b = smem_u32(smem + (size_t)s * stage_bytes(p.BT) + kOffB);
#pragma unroll
    for (int kk = 0; kk < kBK / 16; ++kk)
      umma_f16(tmem, umma_desc_sw128(a + kk * 32), umma_desc_sw128(b + kk * 32), p.idesc, (kb | kk) != 0);
    umma_commit(&empty[s]);
  }
  umma_commit(accf);  // also on abort: lets the CTA wait for in-flight MMAs before freeing TMEM
}

__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + expf(-a)); }

// Store 16 output columns (tokens t0 + c0 + i) of weight row n (= n0 + 32 q + lane).  Called by all 32 lanes
// of a warp with a warp-uniform row block: the gate|up epilogue pairs lane l (< 16, gate row) with lane
// l + 16 (the matching up row) and writes h[t][16 (n / 32) + l].
__device__ __forceinline__ void epi_store16(const GemmParams& p, int n, int lane, int tbase, const float (&v)[16]) {
  if (p.epi) {
    const int j = n >> 5;  // row block (N is a multiple of 32 for gate|up)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float up = __shfl_down_sync(0xFFFFFFFFu, v[i], 16);
      const int t = tbase + i;
      if (lane < 16 && n < p.N && t < p.M)
        p.y[(size_t)t * (p.N / 2) + 16 * j + lane] = __half_as_ushort(__float2half_rn(silu_f32(v[i]) * up));
    }
    return;
  }
  if (n < p.N) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int t = tbase + i;
      if (t < p.M) p.y[(size_t)t * p.N + n] = __half_as_ushort(__float2half_rn(v[i]));
    }
  }
}

// Dequant role then epilogue; r = 0..127 is the weight row of the tile this thread owns.
__device__ __forceinline__ void gemm_dequant_epilogue(const GemmParams& p, uint8_t* smem, uint64_t* full,
                                                      uint64_t* afull, uint64_t* accf, volatile int* abort_flag,
                                                      uint32_t tmem, int n0, int t0, int rb_avail, int r,
                                                      int wg, int warp, int lane, int nkb) {
  const int rbl = r >> 5, rr = r & 31;
  const bool row_ok = rbl < rb_avail;
  const uint32_t swz = (uint32_t)(r & 7);
  for (int kb = wg; kb < nkb; kb += kDequantWG) {  // this warpgroup's k-blocks
    const int s = kb % p.ST;
    if (*abort_flag || !mbar_wait(&full[s], (kb / p.ST) & 1, p.status)) {
      *abort_flag = 1;
      break;
    }
    uint8_t* st = smem + (size_t)s * stage_bytes(p.BT);
    uint8_t* arow = st + kOffA + r * 128;
    if (row_ok) {
      const uint16_t scb = reinterpret_cast<const uint16_t*>(st + off_sc(p.BT))[r];
      const uint32_t zw = reinterpret_cast<const uint32_t*>(st + off_z(p.BT))[r >> 3];
      const uint32_t z = (zw >> (4 * (r & 7))) & 0xFu;
      const __half2 sc2 = u32_as_h2((uint32_t)scb * 0x00010001u);
      const __half2 z1024 = zero_1024(z), nz64 = neg_zero_64(z);
      const uint32_t magic = magic_1024x2();
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint4 pk = *reinterpret_cast<const uint4*>(st + off_pk(p.BT) + rbl * 1024 + j * 512 + rr * 16);
        const uint32_t ww[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          __half2 d[4];
          word_minus_zero(ww[wi], z1024, nz64, magic, d);
          uint4 v;
          v.x = h2_as_u32(__hmul2(d[0], sc2));
          v.y = h2_as_u32(__hmul2(d[1], sc2));
          v.z = h2_as_u32(__hmul2(d[2], sc2));
          v.w = h2_as_u32(__hmul2(d[3], sc2));
          const uint32_t c = (uint32_t)(j * 4 + wi);  // 16-byte chunk (8 channels) within the 128-B row
          *reinterpret_cast<uint4*>(arow + ((c ^ swz) << 4)) = v;
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(arow + (c << 4)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();  // this thread's generic writes -> visible to the MMA (async proxy)
    __syncwarp();
    if (lane == 0) mbar_arrive(&afull[s]);  // one arrival per warp
  }

  // ---- epilogue: TMEM lanes 32*q .. 32*q+31 hold weight rows 32*q + lane of the tile
  pdl_wait_prior_grids();
  if (!mbar_wait(accf, 0, p.status)) *abort_flag = 1;
  tc_fence_after_sync();
  // Every epilogue thread reaches this barrier (its wait is bounded); after it the abort flag is final
  // (the producer and MMA roles are done), so all epilogue warps take the same decision.
  named_barrier_sync(1, 128 * kDequantWG);
  const bool aborted = *abort_flag != 0;
  if (aborted && p.splits == 1) return;
  const int q = warp & 3;
  const int row = 32 * q + lane;
  const int n = n0 + row;
  const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
  if (p.splits == 1) {
    for (int c0 = 16 * wg; c0 < p.BT; c0 += 16 * kDequantWG) {  // warpgroups split the columns
      uint32_t v[16];
      tmem_ld_32x32b_x16(tq + (uint32_t)c0, v);
      tmem_wait_ld();
      float f[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]);
      epi_store16(p, n, lane, t0 + c0, f);
    }
    return;
  }
  // ---- split-K: fp32 partial tile to the workspace; the last split to arrive sums them in order
  const int tile = blockIdx.x;  // this launch's tile slot in the workspace and the counters
  float* tile_ws = p.ws_part + (size_t)tile * p.splits * p.BT * 128;
  float* mine = tile_ws + (size_t)blockIdx.z * p.BT * 128;  // [column][row]
  if (!aborted) {  // an aborted CTA has no valid accumulator, but still arrives on the tile counter below
    for (int c0 = 16 * wg; c0 < p.BT; c0 += 16 * kDequantWG) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(tq + (uint32_t)c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) mine[(size_t)(c0 + i) * 128 + row] = __uint_as_float(v[i]);
    }
  }
  __threadfence();
  named_barrier_sync(1, 128 * kDequantWG);
  volatile unsigned* s_last = reinterpret_cast<volatile unsigned*>(abort_flag) + 1;
  if (threadIdx.x == 64) *s_last = atomicAdd(&p.ws_cnt[tile], 1u) == (unsigned)(p.splits - 1);
  named_barrier_sync(1, 128 * kDequantWG);
  if (!*s_last) return;
  // Every split of the tile has arrived: the counter goes back to zero for the next call whatever
  // happened (after a timeout the output is invalid and the status word says so).
  if (aborted) {
    if (threadIdx.x == 64) p.ws_cnt[tile] = 0u;
    return;
  }
  __threadfence();
  for (int c0 = 16 * wg; c0 < p.BT; c0 += 16 * kDequantWG) {
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    for (int sp = 0; sp < p.splits; ++sp) {
      const float* src = tile_ws + (size_t)sp * p.BT * 128;
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] += __ldcg(src + (size_t)(c0 + i) * 128 + row);
    }
    epi_store16(p, n, lane, t0 + c0, acc);
  }
  if (threadIdx.x == 64) p.ws_cnt[tile] = 0u;
}

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmMaps maps,
                                                               const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)p.ST * stage_bytes(p.BT));
  uint64_t* full = bars;
  uint64_t* afull = bars + p.ST;
  uint64_t* empty = bars + 2 * p.ST;
  uint64_t* accf = bars + 3 * p.ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = p.tile_base + (int)blockIdx.x;
  const int n0 = (tile % p.n_tiles) * kBN, t0 = (tile / p.n_tiles) * p.BT;
  const int rb_avail = min(4, (p.Np - n0) / 32);
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int nkb = min(p.kb_per_split, p.KB - kb0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);  // the 4 warps of the dequant warpgroup that owns the stage
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&maps.x);
    prefetch_tensormap(&maps.codes);
    prefetch_tensormap(&maps.scales);
    prefetch_tensormap(&maps.zeros);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, (unsigned)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) gemm_producer(&maps, p, smem, full, empty, abort_flag, n0, t0, kb0, nkb);
  } else if (warp == 1) {
    if (lane == 0) gemm_mma(p, smem, full, afull, empty, accf, abort_flag, tmem, nkb);
  } else {
    const int wg = (threadIdx.x - 64) >> 7;
    gemm_dequant_epilogue(p, smem, full, afull, accf, abort_flag, tmem, n0, t0, rb_avail, (threadIdx.x - 64) & 127, wg,
                          warp, lane, nkb);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag) mbar_wait(accf, 0, p.status);  // in-flight MMAs finish before TMEM is released
    tc_fence_after_sync();
    tmem_dealloc(tmem, (unsigned)p.tmem_cols);
  }
}

// ------------------------------------------------------------------------------------------ host
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

int pick_bt(int M) {
  if (M >= 256) return 256;
  return (M + 15) / 16 * 16;
}

int pow2_at_least(int v, int lo) {
  int c = lo;
  while (c < v) c <<= 1;
  return c;
}

bool smem_attr_set(int smem) {
  static int done_for[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (done_for[dev] >= smem) return true;
  if (cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem) != cudaSuccess)
    return false;
  done_for[dev] = kMaxSmem;
  return true;
}

}  // namespace

struct GemmPlan {
  int BT, n_tiles, t_tiles, KB, splits, kb_per_split;
  int main_tiles;                        // tiles of the first launch (all of them unless there is a tail)
  int tail_tiles, tail_splits, tail_kbs;  // a short last wave, run as a second launch with K split
  size_t part_bytes;
};

// Split K when the output tiles alone cannot occupy the SMs: as many splits as fit in one wave, each with at
// least 4 k-blocks.  When the tiles fill the SMs but leave a short last wave (at most a quarter of the SMs,
// e.g. 896 tiles = 6 waves + 8), the whole waves run as one launch and the last few tiles as a second
// launch with K split over the SMs, so the last wave takes a fraction of a tile's time instead of a whole one.
GemmPlan plan_gemm(int M, int N, int K) {  // the same plan for every group size
  GemmPlan g{};
  g.BT = pick_bt(M);
  g.n_tiles = ((N + 31) / 32 * 32 + kBN - 1) / kBN;
  g.t_tiles = (M + g.BT - 1) / g.BT;
  g.KB = K / kBK;
  const int tiles = g.n_tiles * g.t_tiles;
  const int sms = num_sms();
  const int max_by_k = g.KB / 4 > 0 ? g.KB / 4 : 1;
  auto split_for = [&](int count, int& splits, int& kbs) {
    int s = count >= sms ? 1 : sms / count;
    if (s > max_by_k) s = max_by_k;
    if (s < 1) s = 1;
    kbs = (g.KB + s - 1) / s;
    splits = (g.KB + kbs - 1) / kbs;  // no empty split
  };
#ifndef AWQ_GEMM_TAIL_SPLITS  // cap on the splits of the last-wave launch (measured on 4096 -> 14336 at M = 2048:
#define AWQ_GEMM_TAIL_SPLITS 8  // 292.6 us as one launch, 280.6 / 282.1 / 278.6 us with 2 / 4 / 8 splits)
#endif
  const int tail = tiles > sms ? tiles % sms : 0;
  if (AWQ_GEMM_TAIL_SPLITS > 1 && tail > 0 && tail * 4 <= sms) {
    g.main_tiles = tiles - tail;
    g.splits = 1;
    g.kb_per_split = g.KB;
    g.tail_tiles = tail;
    split_for(tail, g.tail_splits, g.tail_kbs);
    if (g.tail_splits > AWQ_GEMM_TAIL_SPLITS) {  // fewer, longer splits: the last arriver sums fewer partials
      g.tail_kbs = (g.KB + AWQ_GEMM_TAIL_SPLITS - 1) / AWQ_GEMM_TAIL_SPLITS;
      g.tail_splits = (g.KB + g.tail_kbs - 1) / g.tail_kbs;
    }
    g.part_bytes = g.tail_splits > 1 ? (size_t)tail * g.tail_splits * g.BT * 128 * sizeof(float) : 0;
  } else {
    g.main_tiles = tiles;
    split_for(tiles, g.splits, g.kb_per_split);
    g.part_bytes = g.splits > 1 ? (size_t)tiles * g.splits * g.BT * 128 * sizeof(float) : 0;
  }
  return g;
}

size_t gemm_workspace_bytes(int M, int N, int K, int gs) {
  (void)gs;
  const GemmPlan g = plan_gemm(M, N, K);
  return g.part_bytes == 0 ? 0 : kWorkspaceCounterBytes + g.part_bytes;
}

awq_status gemm_launch(const LinearArgs& a) {
  EncodeTiledFn encode = encode_fn();
  if (encode == nullptr) return AWQ_ERR_CUDA;
  const int M = a.M, N = a.N, K = a.K;
  void* ws = a.ws;
  const size_t ws_bytes = a.ws_bytes;
  const uint16_t* x = a.x;
  const uint32_t* qw = a.qw;
  const uint16_t* scales = a.scales;
  const uint32_t* qzeros = a.qzeros;
  GemmParams p;
  p.qw = reinterpret_cast<const uint4*>(qw);
  p.scales = scales;
  p.qzeros = qzeros;
  p.y = a.y;
  p.status = a.status;
  p.epi = a.epi;
  p.gshift = a.g == 64 ? 0 : a.g == 128 ? 1 : 2;
  p.M = M;
  p.N = N;
  p.Np = (N + 31) / 32 * 32;
  p.K = K;
  p.KB = K / kBK;
  const GemmPlan g = plan_gemm(M, N, K);
  if ((size_t)g.n_tiles * g.t_tiles * 4 > kWorkspaceCounterBytes) return AWQ_ERR_UNSUPPORTED;
  if (g.part_bytes > 0 && (ws == nullptr || ws_bytes < kWorkspaceCounterBytes + g.part_bytes))
    return AWQ_ERR_WORKSPACE;
  p.ws_cnt = static_cast<unsigned*>(ws);
  p.ws_part = ws ? reinterpret_cast<float*>(static_cast<char*>(ws) + kWorkspaceCounterBytes) : nullptr;
  p.splits = g.splits;
  p.kb_per_split = g.kb_per_split;
  p.tile_base = 0;
  p.n_tiles = g.n_tiles;
  p.BT = g.BT;
  const int sb = stage_bytes(p.BT);
  p.ST = (kMaxSmem - 2048) / sb;
  if (p.ST > 8) p.ST = 8;
  // The dequant warpgroups take k-blocks round robin (kb % kDequantWG) and stage s = kb % ST.  With ST a
  // multiple of kDequantWG every stage always belongs to the same warpgroup, which then waits for the stage's
  // phases strictly in order.  Otherwise two warpgroups alternate on a stage, and when copies land out of
  // order one of them can reach phase P + 2 of full[s] while P + 1 is still in flight: its parity wait then
  // matches phase P and it reads a stage that is still being filled (and its early arrival shifts afull[s]
  // one phase ahead of the MMA thread, which then waits until its bounded wait gives up).
  p.ST = p.ST / kDequantWG * kDequantWG;
  if (p.ST < kDequantWG) return AWQ_ERR_UNSUPPORTED;
  p.tmem_cols = pow2_at_least(p.BT, 32);
  p.idesc = umma_idesc_f16(kBN, p.BT);
  const int smem = p.ST * sb + 1024 + 256;
  if (!smem_attr_set(smem)) return AWQ_ERR_CUDA;

  GemmMaps maps;
  const cuuint32_t estr[3] = {1, 1, 1};
  const cuuint64_t RB = (cuuint64_t)p.Np / 32, G = (cuuint64_t)K / (cuuint64_t)a.g;
  {  // x' [M][K] fp16, 64 x BT boxes in the 128-byte swizzle layout
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)p.BT};
    if (encode(&maps.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  {  // codes: [RB][K/32 chunks][128 words]; box = 2 chunks x 4 row blocks
    const cuuint64_t dims[3] = {128, (cuuint64_t)K / 32, RB};
    const cuuint64_t strides[2] = {512, (cuuint64_t)K / 32 * 512};
    const cuuint32_t box[3] = {128, 2, 4};
    if (encode(&maps.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(qw), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  {  // scales: [RB][G * 32] fp16; box = 32 x 4 row blocks
    const cuuint64_t dims[2] = {G * 32, RB};
    const cuuint64_t strides[1] = {G * 64};
    const cuuint32_t box[2] = {32, 4};
    if (encode(&maps.scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(scales), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  {  // zeros: [RB][G * 4] u32; box = 4 x 4 row blocks
    const cuuint64_t dims[2] = {G * 4, RB};
    const cuuint64_t strides[1] = {G * 16};
    const cuuint32_t box[2] = {4, 4};
    if (encode(&maps.zeros, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(qzeros), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  cudaError_t e = launch_pdl(gemm_kernel, dim3((unsigned)g.main_tiles, 1u, (unsigned)g.splits), dim3(kGemmThreads),
                             (size_t)smem, a.st, maps, p);
  if (e == cudaSuccess && g.tail_tiles > 0) {  // the short last wave, K split over the SMs
    p.tile_base = g.main_tiles;
    p.splits = g.tail_splits;
    p.kb_per_split = g.tail_kbs;
    e = launch_pdl(gemm_kernel, dim3((unsigned)g.tail_tiles, 1u, (unsigned)g.tail_splits), dim3(kGemmThreads),
                   (size_t)smem, a.st, maps, p);
  }
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
