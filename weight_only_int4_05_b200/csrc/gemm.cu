// gemm.cu -- W4A16 prefill kernel ("GEMM mode" of the AutoAWQ page: long context, many tokens).
//
// y^T tile [128 weight rows][BT tokens] = dequant(W)[128][K] . x'[BT][K]^T on the tcgen05 tensor cores.
// Weights are the UMMA A operand (M = 128 rows of N), activations the B operand (N = BT tokens), so a
// small token count still maps onto a full-height MMA.
//
// Per CTA (192 threads, one output tile, k-blocks of 64 channels through an ST-stage ring):
//   warp 0, lane 0  producer: TMA bulk copies of the packed tile (4 row blocks x 1 KB), its fp16 scales
//                   and packed zeros, and a 2-D tensor copy of the x' tile in the 128-byte swizzle
//                   layout; all complete on full[s].  Weight copies for the first ring are issued before
//                   griddepcontrol.wait, so they overlap the previous kernel on the stream.
//   warps 2..5      dequant: thread r owns weight row r of the tile; it turns 64 packed codes into
//                   fp16 (q - z) * S (exact q - z by the int4->fp16 bit trick, one rounding for the
//                   scale) and writes them in the 128-byte swizzle K-major layout the MMA reads, then
//                   fence.proxy.async + arrive on afull[s].  After the main loop the same warps are
//                   the epilogue: tcgen05.ld of their 32-lane TMEM quarter, fp16 convert, store y.
//   warp 1          allocates TMEM (fp32 accumulator, BT columns); lane 0 issues 4 x
//                   tcgen05.mma.kind::f16 (128 x BT x 16) per k-block and tcgen05.commit -> empty[s].
// Every mbarrier wait is bounded (see common.cuh); a timeout is recorded in the status word, the CTA
// drains its own copies and MMAs, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace awq {

constexpr int kBN = 128;  // weight rows per tile (UMMA M)
constexpr int kBK = 64;   // channels per k-block (one 128-byte swizzle row of fp16)
constexpr int kGemmThreads = 192;
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
  int M, N, Np, K, KB, BT, ST, tmem_cols;
  uint32_t idesc;
};

__device__ __forceinline__ void gemm_producer(const CUtensorMap* xmap, const GemmParams& p, uint8_t* smem,
                                              uint64_t* full, uint64_t* empty, volatile int* abort_flag,
                                              int n0, int t0, int rb_avail) {
  const unsigned pk_bytes = 1024u * rb_avail, sc_bytes = 64u * rb_avail, z_bytes = 16u * rb_avail;
  const unsigned tx = (unsigned)p.BT * 128u + pk_bytes + sc_bytes + z_bytes;
  const int KC = p.K / 32;
  auto issue_w = [&](int kb, int s) {
    uint8_t* st = smem + (size_t)s * stage_bytes(p.BT);
    mbar_arrive_expect_tx(&full[s], tx);
    for (int i = 0; i < rb_avail; ++i)
      bulk_g2s(st + off_pk(p.BT) + i * 1024, p.qw + ((size_t)(n0 / 32 + i) * KC + kb * 2) * 32, 1024u, &full[s]);
    const int g = kb >> 1;
    bulk_g2s(st + off_sc(p.BT), p.scales + (size_t)g * p.Np + n0, sc_bytes, &full[s]);
    bulk_g2s(st + off_z(p.BT), p.qzeros + (size_t)g * (p.Np / 8) + n0 / 8, z_bytes, &full[s]);
  };
  auto issue_x = [&](int kb, int s) {
    tma_load_2d(smem + (size_t)s * stage_bytes(p.BT) + kOffB, xmap, kb * kBK, t0, &full[s]);
  };
  const int pre = p.KB < p.ST ? p.KB : p.ST;
  for (int kb = 0; kb < pre; ++kb) issue_w(kb, kb);
  pdl_wait_prior_grids();
  for (int kb = 0; kb < pre; ++kb) issue_x(kb, kb);
  int issued = pre;
  for (int kb = pre; kb < p.KB; ++kb) {
    const int s = kb % p.ST, use = kb / p.ST;
    if (*abort_flag || !mbar_wait(&empty[s], (use - 1) & 1, p.status)) {
      *abort_flag = 1;
      break;
    }
    issue_w(kb, s);
    issue_x(kb, s);
    issued = kb + 1;
  }
  if (*abort_flag) {  // wait (bounded) until every copy this thread issued has landed
    for (int kb = issued > p.ST ? issued - p.ST : 0; kb < issued; ++kb)
      mbar_wait(&full[kb % p.ST], (kb / p.ST) & 1, p.status);
  }
}

__device__ __forceinline__ void gemm_mma(const GemmParams& p, uint8_t* smem, uint64_t* full, uint64_t* afull,
                                         uint64_t* empty, uint64_t* accf, volatile int* abort_flag,
                                         uint32_t tmem) {
  for (int kb = 0; kb < p.KB; ++kb) {
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

// Dequant role then epilogue; r = 0..127 is the weight row of the tile this thread owns.
__device__ __forceinline__ void gemm_dequant_epilogue(const GemmParams& p, uint8_t* smem, uint64_t* full,
                                                      uint64_t* afull, uint64_t* accf, volatile int* abort_flag,
                                                      uint32_t tmem, int n0, int t0, int rb_avail, int r,
                                                      int warp, int lane) {
  const int rbl = r >> 5, rr = r & 31;
  const bool row_ok = rbl < rb_avail;
  const uint32_t swz = (uint32_t)(r & 7);
  for (int kb = 0; kb < p.KB; ++kb) {
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
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint4 pk = *reinterpret_cast<const uint4*>(st + off_pk(p.BT) + rbl * 1024 + j * 512 + rr * 16);
        const uint32_t ww[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          __half2 d[4];
          word_minus_zero(ww[wi], z1024, nz64, d);
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
    fence_proxy_async_smem();
    mbar_arrive(&afull[s]);
  }

  // ---- epilogue: TMEM lanes 32*q .. 32*q+31 hold weight rows 32*q + lane of the tile
  pdl_wait_prior_grids();
  const bool acc_ok = mbar_wait(accf, 0, p.status);
  tc_fence_after_sync();
  // tcgen05.ld is warp-collective: the whole warp takes the same decision
  if (!__all_sync(0xFFFFFFFFu, acc_ok && !*abort_flag)) {
    *abort_flag = 1;
    return;
  }
  const int q = warp & 3;
  const int n = n0 + 32 * q + lane;
  for (int c0 = 0; c0 < p.BT; c0 += 16) {
    uint32_t v[16];
    tmem_ld_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    if (n < p.N) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = t0 + c0 + i;
        if (t < p.M) p.y[(size_t)t * p.N + n] = __half_as_ushort(__float2half_rn(__uint_as_float(v[i])));
      }
    }
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap xmap,
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
  const int n0 = blockIdx.x * kBN, t0 = blockIdx.y * p.BT;
  const int rb_avail = min(4, (p.Np - n0) / 32);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&xmap);
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
    if (lane == 0) gemm_producer(&xmap, p, smem, full, empty, abort_flag, n0, t0, rb_avail);
  } else if (warp == 1) {
    if (lane == 0) gemm_mma(p, smem, full, afull, empty, accf, abort_flag, tmem);
  } else {
    gemm_dequant_epilogue(p, smem, full, afull, accf, abort_flag, tmem, n0, t0, rb_avail, threadIdx.x - 64, warp,
                          lane);
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

size_t gemm_workspace_bytes(int, int, int) { return 0; }

awq_status gemm_launch(const uint16_t* x, const uint32_t* qw, const uint16_t* scales, const uint32_t* qzeros,
                       uint16_t* y, int M, int N, int K, void*, size_t, unsigned* dev_status, cudaStream_t st) {
  EncodeTiledFn encode = encode_fn();
  if (encode == nullptr) return AWQ_ERR_CUDA;
  GemmParams p;
  p.qw = reinterpret_cast<const uint4*>(qw);
  p.scales = scales;
  p.qzeros = qzeros;
  p.y = y;
  p.status = dev_status;
  p.M = M;
  p.N = N;
  p.Np = (N + 31) / 32 * 32;
  p.K = K;
  p.KB = K / kBK;
  p.BT = pick_bt(M);
  const int sb = stage_bytes(p.BT);
  p.ST = (kMaxSmem - 2048) / sb;
  if (p.ST > 8) p.ST = 8;
  p.tmem_cols = pow2_at_least(p.BT, 32);
  p.idesc = umma_idesc_f16(kBN, p.BT);
  const int smem = p.ST * sb + 1024 + 256;
  if (!smem_attr_set(smem)) return AWQ_ERR_CUDA;

  CUtensorMap xmap;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)p.BT};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return AWQ_ERR_CUDA;
  const dim3 grid((unsigned)((p.Np + kBN - 1) / kBN), (unsigned)((M + p.BT - 1) / p.BT));
  cudaError_t e = launch_pdl(gemm_kernel, grid, dim3(kGemmThreads), (size_t)smem, st, xmap, p);
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
