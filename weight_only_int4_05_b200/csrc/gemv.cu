// gemv.cu -- W4A16 decode kernel ("GEMV mode" of the AutoAWQ page: single batch, top speed).
//
// y[m][n] = sum_g S[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x'[m][k]   for up to 8 * NT rows of x' per pass.
//
// Units.  The packed layout stores each (32-row block rb, group g of GS = 64, 128 or 256 channels) as 16 * GS
// contiguous bytes of codes (GS / 32 tiles of 32 rows x 32 channels), and its 32 scales (64 B) and 32 zero
// nibbles (16 B) contiguously in the unit-major scale and zero arrays, so unit u = rb * G + g is one stretch
// of each.  Each of the P CTAs owns a balanced contiguous range
// of units (q = U / P, one more for the first U % P CTAs); its kNW consumer warps split that range into
// contiguous sub-ranges, and each consumer warp has its own ring of kRing shared-memory slots.
//
// Warp roles.  One producer warp per CTA fills every slot with TMA bulk copies -- the codes, scales and zeros
// of the 8 KB of consecutive units a slot holds, three copies completing on the slot's "full" mbarrier -- and
// refills a slot when its consumer has released it on the slot's "empty" mbarrier (the first fill of a warp's
// second slot is held back a little; see gemv_producer).  Slot j of the CTA (warp j / kRing, ring index j % kRing) is
// served by producer lane j % 32: a thread completes about one bulk copy per ~770 cycles whatever its size,
// and a copy waiting behind another one stalls its thread, so spreading the slots over the lanes keeps the
// copies in parallel and keeps every issue stall off the consumer warps.
//
// Arithmetic: the tensor cores, fp32 accumulation.  One unit is two 16-row halves x GS / 16 steps of
// mma.sync m16n8k16 (A = weights, 16 rows x 16 channels; B = x', 16 channels x 8 rows of x'; C = fp32).
// Lane (g = lane / 4, t = lane % 4) reads word t of rows g and g + 8 of each 32-channel chunk c (conflict-
// free 4-byte shared loads).  The nibble order of a word makes (w & 0x000F000F) | 0x64006400 the fp16 pair
// (1024 + q) for channels (8t, 8t+1) and (w & 0x00F000F0) | 0x54005400 the pair (64 + q) for (8t+2, 8t+3);
// the word shifted right by 8 gives channels 8t+4 .. 8t+7 the same way.  One fp16 subtraction of
// (1024 + z) or (64 + z) turns each pair into the exact integers q - z.  Those four pairs are the thread's
// A fragment for one MMA: its k slots {2t, 2t+1} and {2t+8, 2t+9} stand for channels 32c + 8t + {0, 1}
// and + {2, 3} (or + {4..7}), and the B fragment holds x' at the same channels, so every product
// (q - z) * x' is formed exactly in fp32 and summed in fp32.  Each half runs two independent MMA chains
// (even and odd chunks).  After the steps of a group the fp32 sum of each row is multiplied by the row's
// scale and added to the row's fp32 output accumulator.  Nothing is summed in fp16.
//
// 3-bit codes (BITS = 3, the packed 3-bit layout): the same kernel with 384-B tiles and unit_mma3 building the
// fp16 pairs from a 2-bit plane and a 1-bit plane.
//
// Epilogue.  Plain: y = fp16(sum).  Gate|up (epi = 1, the weight packed by awq_pack_gate_up, rows 0..15 of
// row block j the gate rows 16j..16j+15 and rows 16..31 the up rows 16j..16j+15): the output has N / 2
// columns, h[m][16j + i] = fp16(silu(sum of row i) * sum of row 16 + i), silu(a) = a / (1 + e^-a), in fp32
// on the final sums, so the gate and up products never round to fp16 in between.
//
// Before griddepcontrol.wait a kernel touches only its weights: the producer fills the first kRing slots of
// every consumer before the wait, so with programmatic dependent launch the next kernel's weight stream
// starts while the previous kernel still runs.  After the wait, x' (the rows of this pass) is staged in
// shared memory by one TMA copy per row when it fits, with a row pitch padded so that rows fall in different
// banks; otherwise each lane reads its B fragments (64 bytes per unit) from global memory one unit ahead.
//
// Combining split row blocks.  A row block wholly inside one warp's sub-range is written directly.  A row
// block split between warps of one CTA is summed in shared memory, in warp order.  A row block split between
// CTAs gets one fp32 partial per CTA in the workspace slot (rb, c - first_cta(rb)); the CTA that brings the
// row block's counter to its final value sums the slots in slot order (deterministic), writes fp16 y and
// resets the counter to 0 for the next call.  A CTA whose bounded wait ran out still takes part in this
// protocol (with invalid values), so the counters are zero again after every call.
#include "common.cuh"
#include "internal.h"

namespace awq {

// ------------------------------------------------------------------------------------------ constants
// A ring slot holds kSlotCodeBytes of codes of consecutive units of a warp's range, then their scales
// (64 B per unit) and zeros (16 B per unit) -- three copies per slot, since consecutive units are contiguous
// in all three arrays.  Few large copies keep the bytes in flight high: a thread gets only about one bulk
// copy serviced at a time, and under load a copy takes the full memory latency.
constexpr int kSlotCodeBytes = 8192;
#ifndef AWQ_GEMV_RING
#define AWQ_GEMV_RING 2
#endif
constexpr int kRing = AWQ_GEMV_RING;  // slots per consumer warp (power of two)
static_assert((kRing & (kRing - 1)) == 0, "ring depth must be a power of two");
#ifndef AWQ_GEMV_WARPS
#define AWQ_GEMV_WARPS 8
#endif
constexpr int kNW = AWQ_GEMV_WARPS;  // consumer warps per CTA (power of two); one producer warp besides
#ifndef AWQ_GEMV_L2_PREFETCH  // bulk L2 prefetch of each warp's range before the wait (measured slower: off)
#define AWQ_GEMV_L2_PREFETCH 0
#endif
static_assert((kNW & (kNW - 1)) == 0 && kNW >= 2 && kNW <= 16, "consumer warps per CTA: 2, 4, 8 or 16");
constexpr int kSlots = kNW * kRing;
constexpr int kThreads = (kNW + 1) * 32;

// Geometry of a unit and a slot for group size GS and code width BITS (4: the 4-bit layout, 512-B tiles of 32 rows
// x 32 channels; 3: the packed 3-bit layout, 384-B tiles).  A slot holds 8 KB (6 KB at 3 bits) of codes: the
// same number of units either way.
template <int GS, int BITS = 4>
struct Geo {
  static_assert(GS == 64 || GS == 128 || GS == 256, "group size 64, 128 or 256");
  static_assert(BITS == 3 || BITS == 4, "3- or 4-bit codes");
  static constexpr int CH = GS / 32;                    // 32-channel chunks per unit
  static constexpr int TB = BITS == 4 ? 512 : 384;      // bytes per 32-row x 32-channel tile
  static constexpr int UB = CH * TB;                    // code bytes per unit
  static constexpr int SLOT = kSlotCodeBytes / 4 * BITS;
  static constexpr int SU = SLOT / UB;                  // units per slot: 8, 4, 2
  static constexpr int SCO = SLOT;                      // scales offset in a slot
  static constexpr int ZO = SCO + SU * 64;              // zeros offset in a slot
  static constexpr int STRIDE = (ZO + SU * 16 + 127) / 128 * 128;
  static constexpr int RING = kSlots * STRIDE;          // ring bytes per CTA
  static_assert(RING <= 160 * 1024, "rings too large for shared memory");
};
constexpr int kXsMaxBytes = 36 * 1024;  // x' of one pass staged in shared memory when it fits
constexpr int kXPad = 32;                // halves of padding per staged row: rows 64 B apart fall in other banks
constexpr int kMaxDynSmem = 232448 - 2048;  // opt-in shared memory per block, less the static barriers

struct GemvParams {
  const uint16_t* x;
  const uint16_t* s;  // AWQ per-channel scale, divided out of the staged x (DIVS kernels), else NULL
  const uint8_t* qw;
  const uint16_t* scales;
  const uint32_t* qzeros;
  uint16_t* y;
  int epi;  // 0: y[m][n] (ny = N); 1: gate|up SiLU product (ny = N / 2)
  int ny;   // columns of y
  float* ws_part;
  unsigned* ws_cnt;
  unsigned* status;             // device status word (bounded waits)
  const uint8_t* pf;            // optional: bytes to prefetch into L2 for a later call (NULL: none)
  unsigned long long pf_bytes;  // their size (a multiple of 16)
  unsigned long long pf_share;  // bytes per CTA (a multiple of 16)
  int U;                        // units = RB * G (G = K / GS)
  int P;                        // CTAs sharing the units: CTA c owns q granules, plus one more if c < r
  int q, r;
  int gran;                     // units per granule: 1, or G when CTA ranges are whole row blocks
  int M, N, K, G, RB, S, m0;
  int mts;     // rows of x' per workspace slot: min(M, 8 * NT)
  int xpitch;  // staged x' row pitch in halves (XS kernels)
};

__device__ __forceinline__ int cta_first_unit(const GemvParams& p, int c) { return p.gran * (p.q * c + min(c, p.r)); }
__device__ __forceinline__ int cta_units(const GemvParams& p, int c) { return p.gran * (p.q + (c < p.r ? 1 : 0)); }
// CTA owning unit u (only used when row blocks are split between CTAs, i.e. gran == 1)
__device__ __forceinline__ int cta_of_unit(const GemvParams& p, int u) {
  const int b = p.r * (p.q + 1);
  return u < b ? u / (p.q + 1) : p.r + (u - b) / p.q;
}

// Sub-range of consumer warp w inside the CTA's units [cu0, cu0 + n): first unit and count.
__device__ __forceinline__ void warp_range(int cu0, int n, int w, int& wu0, int& nw) {
  const int wq = n / kNW, wr = n % kNW;
  wu0 = cu0 + wq * w + min(w, wr);
  nw = wq + (w < wr ? 1 : 0);
}

// Copies of the c consecutive units from unit u into a ring slot, completion counted on `bar`.  The codes
// copy (with the barrier's expected byte count) and the scales + zeros copies can come from different lanes,
// which proceed in parallel; the barrier's phase cannot complete before the arming arrival, so the order in
// which the lanes' bytes land does not matter.
template <int GS, int BITS>
__device__ __forceinline__ void issue_codes(const GemvParams& p, int u, int c, uint8_t* slot, uint64_t* bar) {
  using Ge = Geo<GS, BITS>;
  mbar_arrive_expect_tx(bar, (unsigned)c * (unsigned)(Ge::UB + 80));
  bulk_g2s(slot, p.qw + (size_t)u * Ge::UB, (unsigned)(c * Ge::UB), bar);
}
template <int GS, int BITS>
__device__ __forceinline__ void issue_meta(const GemvParams& p, int u, int c, uint8_t* slot, uint64_t* bar) {
  using Ge = Geo<GS, BITS>;
  bulk_g2s(slot + Ge::SCO, p.scales + (size_t)u * 32, (unsigned)(c * 64), bar);
  bulk_g2s(slot + Ge::ZO, p.qzeros + (size_t)u * 4, (unsigned)(c * 16), bar);
}

// One unit: y rows (g + 8i, i = 0..3) x columns (8 nt + 2t + j) += S_row * sum_k (q - z) x'.
// codes / scl / zer: 32-bit shared addresses of the unit's codes, scales and zeros; xb[nt][c]: x' row 8 nt + g
// (clamped to the pass), channels GS grp + 32c + 8t .. + 7, as 16 bytes; CH = GS / 32 chunks.
template <int NT, int CH>
__device__ __forceinline__ void unit_mma(uint32_t codes, uint32_t scl, uint32_t zer, int g, int t,
                                         const uint4 (&xb)[NT][CH], float (&yacc)[NT][4][2]) {
  uint32_t w[2][2][CH];  // [half][row g / g + 8][chunk]
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int cc = 0; cc < CH; ++cc) {
      w[h][0][cc] = ld_shared_u32(codes + 512 * cc + 16 * (16 * h + g) + 4 * t);
      w[h][1][cc] = ld_shared_u32(codes + 512 * cc + 16 * (16 * h + g + 8) + 4 * t);
    }
  const uint4 zw = ld_shared_v4(zer);  // word i: zero nibbles of rows 8i .. 8i+7
  float S[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    S[i] = __half2float(__ushort_as_half(ld_shared_u16(scl + 2 * (g + 8 * i))));
  const uint32_t zws[4] = {zw.x, zw.y, zw.z, zw.w};
  __half2 zlo[4], zhi[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t z = (zws[i] >> (4 * g)) & 0xFu;
    zlo[i] = zero_1024(z);
    zhi[i] = zero_64(z);
  }
  const uint32_t m1024 = magic_1024x2(), m64 = magic_64x2();
  float c[NT][2][2][4];  // [n-tile][half][chunk parity][fragment]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) c[nt][h][pr][0] = c[nt][h][pr][1] = c[nt][h][pr][2] = c[nt][h][pr][3] = 0.f;
#pragma unroll
  for (int cc = 0; cc < CH; ++cc)
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t ua = s ? (w[h][0][cc] >> 8) : w[h][0][cc], ub = s ? (w[h][1][cc] >> 8) : w[h][1][cc];
        const uint32_t a0 = h2_as_u32(__hsub2(u32_as_h2(and_or<0x000F000Fu>(ua, m1024)), zlo[2 * h]));
        const uint32_t a1 = h2_as_u32(__hsub2(u32_as_h2(and_or<0x000F000Fu>(ub, m1024)), zlo[2 * h + 1]));
        const uint32_t a2 = h2_as_u32(__hsub2(u32_as_h2(and_or<0x00F000F0u>(ua, m64)), zhi[2 * h]));
        const uint32_t a3 = h2_as_u32(__hsub2(u32_as_h2(and_or<0x00F000F0u>(ub, m64)), zhi[2 * h + 1]));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816_f32(c[nt][h][cc & 1], a0, a1, a2, a3, s ? xb[nt][cc].z : xb[nt][cc].x,
                        s ? xb[nt][cc].w : xb[nt][cc].y);
      }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      yacc[nt][2 * h][0] = fmaf(S[2 * h], c[nt][h][0][0] + c[nt][h][1][0], yacc[nt][2 * h][0]);
      yacc[nt][2 * h][1] = fmaf(S[2 * h], c[nt][h][0][1] + c[nt][h][1][1], yacc[nt][2 * h][1]);
      yacc[nt][2 * h + 1][0] = fmaf(S[2 * h + 1], c[nt][h][0][2] + c[nt][h][1][2], yacc[nt][2 * h + 1][0]);
      yacc[nt][2 * h + 1][1] = fmaf(S[2 * h + 1], c[nt][h][0][3] + c[nt][h][1][3], yacc[nt][2 * h + 1][1]);
    }
}

// The same unit for the packed 3-bit layout.  Lane (g, t) reads, for rows g and g + 8 of each half and each
// chunk, the word holding the low 2-bit fields of its channel group t (word t / 2 of the row, the group's fields
// at bit 8 (t % 2) on) and the row's high-bit word (word 2; pair p of group t at bits 4t + p and 4t + p + 16).
// For each channel pair, (lo >> 2p) & 0x00030003 brought together with the high bits moved to bits 2 and 18 and
// the exponent bits 0x6400 is the fp16 pair 1024 + q; one subtraction of (1024 + z) makes q - z exact, and the
// MMA steps, B fragments and epilogue are those of the 4-bit unit.
template <int NT, int CH>
__device__ __forceinline__ void unit_mma3(uint32_t codes, uint32_t scl, uint32_t zer, int g, int t,
                                          const uint4 (&xb)[NT][CH], float (&yacc)[NT][4][2]) {
  uint32_t lo[2][2][CH], hl[2][2][CH], hh[2][2][CH];  // [half][row g / g + 8][chunk]
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int cc = 0; cc < CH; ++cc)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const uint32_t row = codes + 384 * cc + 12 * (16 * h + g + 8 * rr);
        lo[h][rr][cc] = ld_shared_u32(row + 4 * (t >> 1)) >> (8 * (t & 1));
        const uint32_t w2 = ld_shared_u32(row + 8);
        hl[h][rr][cc] = w2 << 2;  // the 64-bit value (w2 << 2), whose bits 4t + p + 2 and 4t + p + 18 ...
        hh[h][rr][cc] = w2 >> 30;
      }
  const uint4 zw = ld_shared_v4(zer);
  float S[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    S[i] = __half2float(__ushort_as_half(ld_shared_u16(scl + 2 * (g + 8 * i))));
  const uint32_t zws[4] = {zw.x, zw.y, zw.z, zw.w};
  __half2 z1024[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) z1024[i] = zero_1024((zws[i] >> (4 * g)) & 0xFu);
  const uint32_t m1024 = magic_1024x2();
  float c[NT][2][2][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) c[nt][h][pr][0] = c[nt][h][pr][1] = c[nt][h][pr][2] = c[nt][h][pr][3] = 0.f;
  // fp16 pair (1024 + q) of channel pair p of this lane's group, for one row
  auto pair = [&](int h, int rr, int cc, int p) -> uint32_t {
    const uint32_t hb = __funnelshift_r(hl[h][rr][cc], hh[h][rr][cc], 4 * t + p);  // ... land at bits 2 and 18
    return and_or<0x00030003u>(lo[h][rr][cc] >> (2 * p), and_or<0x00040004u>(hb, m1024));
  };
#pragma unroll
  for (int cc = 0; cc < CH; ++cc)
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t a0 = h2_as_u32(__hsub2(u32_as_h2(pair(h, 0, cc, 2 * s)), z1024[2 * h]));
        const uint32_t a1 = h2_as_u32(__hsub2(u32_as_h2(pair(h, 1, cc, 2 * s)), z1024[2 * h + 1]));
        const uint32_t a2 = h2_as_u32(__hsub2(u32_as_h2(pair(h, 0, cc, 2 * s + 1)), z1024[2 * h]));
        const uint32_t a3 = h2_as_u32(__hsub2(u32_as_h2(pair(h, 1, cc, 2 * s + 1)), z1024[2 * h + 1]));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816_f32(c[nt][h][cc & 1], a0, a1, a2, a3, s ? xb[nt][cc].z : xb[nt][cc].x,
                        s ? xb[nt][cc].w : xb[nt][cc].y);
      }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      yacc[nt][2 * h][0] = fmaf(S[2 * h], c[nt][h][0][0] + c[nt][h][1][0], yacc[nt][2 * h][0]);
      yacc[nt][2 * h][1] = fmaf(S[2 * h], c[nt][h][0][1] + c[nt][h][1][1], yacc[nt][2 * h][1]);
      yacc[nt][2 * h + 1][0] = fmaf(S[2 * h + 1], c[nt][h][0][2] + c[nt][h][1][2], yacc[nt][2 * h + 1][0]);
      yacc[nt][2 * h + 1][1] = fmaf(S[2 * h + 1], c[nt][h][0][3] + c[nt][h][1][3], yacc[nt][2 * h + 1][1]);
    }
}

template <int NT, int GS>
__device__ __forceinline__ void load_xb(const uint16_t* const (&xrow)[NT], int grp, int t,
                                        uint4 (&xb)[NT][Geo<GS>::CH]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int cc = 0; cc < Geo<GS>::CH; ++cc) xb[nt][cc] = ldg_cached(xrow[nt] + grp * GS + cc * 32 + t * 8);
}

__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + expf(-a)); }

// Row block r written directly from a warp's fragments.
template <int NT>
__device__ __forceinline__ void store_frag(const GemvParams& p, int r, int g, int t, int mcount,
                                           const float (&yacc)[NT][4][2]) {
  if (p.epi) {  // rows g + 8i (i = 0, 1) are gate rows, g + 8i + 16 the matching up rows
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int m = 8 * nt + 2 * t + j;
          if (m < mcount)
            p.y[(size_t)(p.m0 + m) * p.ny + r * 16 + g + 8 * i] =
                __half_as_ushort(__float2half_rn(silu_f32(yacc[nt][i][j]) * yacc[nt][i + 2][j]));
        }
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = r * 32 + g + 8 * i;
    if (n >= p.N) continue;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int m = 8 * nt + 2 * t + j;
        if (m < mcount) p.y[(size_t)(p.m0 + m) * p.N + n] = __half_as_ushort(__float2half_rn(yacc[nt][i][j]));
      }
  }
}

// A warp's partial of one row block into its shared-memory slot, [m][32 rows].
template <int NT>
__device__ __forceinline__ void stash_frag(float* part, int g, int t, int mcount, const float (&yacc)[NT][4][2]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int m = 8 * nt + 2 * t + j;
      if (m < mcount) {
#pragma unroll
        for (int i = 0; i < 4; ++i) part[m * 32 + g + 8 * i] = yacc[nt][i][j];
      }
    }
}

// lane = row of row block r: y[m][32 r + lane] for m < mcount.  (Fixed-size, fully unrolled arrays keep the
// values in registers: a dynamically indexed array would live in local memory.)
// Called by all 32 lanes of a warp (the gate|up epilogue exchanges values between lanes l and l + 16).
template <int NT>
__device__ __forceinline__ void store_row(const GemvParams& p, int r, int lane, int mcount, const float (&v)[8 * NT]) {
  if (p.epi) {
#pragma unroll
    for (int m = 0; m < 8 * NT; ++m) {
      const float up = __shfl_down_sync(0xFFFFFFFFu, v[m], 16);
      if (lane < 16 && m < mcount)
        p.y[(size_t)(p.m0 + m) * p.ny + r * 16 + lane] = __half_as_ushort(__float2half_rn(silu_f32(v[m]) * up));
    }
    return;
  }
  const int n = r * 32 + lane;
  if (n >= p.N) return;
#pragma unroll
  for (int m = 0; m < 8 * NT; ++m)
    if (m < mcount) p.y[(size_t)(p.m0 + m) * p.N + n] = __half_as_ushort(__float2half_rn(v[m]));
}

// Sum over the CTAs that share row block r (called by the one warp per CTA that combines r; lane = row).
template <int NT>
__device__ __forceinline__ void cross_cta_combine(const GemvParams& p, int r, int lane, int mcount,
                                                  const float (&part)[8 * NT]) {
  const int cf = cta_of_unit(p, r * p.G);
  const int cl = cta_of_unit(p, r * p.G + p.G - 1);
  const int nc = cl - cf + 1;
  const int slot = (int)blockIdx.x - cf;
  float* base = p.ws_part + (size_t)r * p.S * 32 * p.mts;  // slots of row block r
#pragma unroll
  for (int m = 0; m < 8 * NT; ++m)
    if (m < mcount) base[(size_t)(slot * p.mts + m) * 32 + lane] = part[m];
  __threadfence();
  __syncwarp();
  unsigned old = 0;
  if (lane == 0) old = atomicAdd(&p.ws_cnt[r], 1u);
  old = __shfl_sync(0xFFFFFFFFu, old, 0);
  if (old != (unsigned)(nc - 1)) return;
  __threadfence();
  float sum[8 * NT];
#pragma unroll
  for (int m = 0; m < 8 * NT; ++m) sum[m] = 0.f;
  for (int j = 0; j < nc; ++j) {
#pragma unroll
    for (int m = 0; m < 8 * NT; ++m)
      if (m < mcount) sum[m] += (j == slot) ? part[m] : __ldcg(&base[(size_t)(j * p.mts + m) * 32 + lane]);
  }
  store_row<NT>(p, r, lane, mcount, sum);
  if (lane == 0) p.ws_cnt[r] = 0u;
}

// Dynamic shared memory: [rings][staged x' (XS): rows x xpitch halves][partials: kNW x 2 slots x mcount x 32 fp32].
__host__ __device__ constexpr int gemv_part_bytes(int rows) { return kNW * 2 * rows * 32 * 4; }
__host__ __device__ constexpr int gemv_xs_bytes(int rows, int xpitch) { return (rows * xpitch * 2 + 127) / 128 * 128; }

// Producer warp.  Lane L serves CTA slot j = L % kSlotLanes (consumer warp j / kRing, ring index j % kRing):
// lanes below kSlotLanes issue the slot's codes copy (and arm its barrier), lanes from kSlotLanes on issue its
// scales and zeros when there are enough lanes, so the big and small copies of a slot are serviced in
// parallel.  The warp's slot sequence number sq = 0, 1, ... covers its units [sq * kSU, sq * kSU + kSU) (kSU
// units per slot); ring index si takes the sequence numbers si, si + kRing, ...  The first fill of ring index 0
// is issued at once (before any dependency wait), the first fill of ring index si > 0 after si * kStaggerCycles
// cycles, and every later fill when the consumer has released the slot.
//
// Why the stagger: at a kernel's start every CTA asks for all its slots at once (about 20 MB over the GPU), and
// DRAM serves the outstanding copies side by side, so the slot each warp needs first lands only near the end of
// the whole burst.  Holding back the second slots lets the first ones land sooner.  Measured on one B200 (µs
// per call at M = 1, programmatic dependent launch between calls): the 224-linear decode stack 1621 -> 1589 per
// token, 14336 -> 4096 10.83 -> 10.34, 4096 -> 14336 10.66 -> 10.86, q/o and k/v unchanged.  Issuing the second
// slot as soon as the first has landed instead was slower on the single linears (14336 -> 4096 11.42).
constexpr int kSlotLanes = kSlots <= 16 ? kSlots : 32;  // lanes that issue codes; kSlots <= 16: one more lane for meta
static_assert(kSlots <= 32, "one producer warp serves at most 32 slots");
#ifndef AWQ_GEMV_STAGGER_CYCLES
#define AWQ_GEMV_STAGGER_CYCLES 4000  // about 2 us at the 1965 MHz boost clock
#endif
constexpr long long kStaggerCycles = AWQ_GEMV_STAGGER_CYCLES;

// Bounded pause of the calling thread (SM clock cycles).
__device__ __forceinline__ void pause_cycles(long long cycles) {
  const long long c0 = clock64();
  while (clock64() - c0 < cycles) __nanosleep(32);
}

template <int GS, int BITS>
__device__ __forceinline__ void gemv_producer(const GemvParams& p, uint8_t* ring, uint64_t* full, uint64_t* empty,
                                              int cu0, int n, int lane) {
  constexpr int kSU = Geo<GS, BITS>::SU;
  const bool split = kSlots <= 16;
  const int j = split ? lane % 16 : lane;
  const bool does_codes = lane < kSlotLanes, does_meta = split ? (lane >= 16 && j < kSlots) : does_codes;
  if (j >= kSlots || !(does_codes || does_meta)) return;
  int wu0, nw;
  warp_range(cu0, n, j / kRing, wu0, nw);
  const int si = j % kRing;
  uint8_t* slot = ring + (size_t)j * Geo<GS, BITS>::STRIDE;
  auto issue = [&](int sq) {
    const int u = wu0 + sq * kSU, c = min(kSU, nw - sq * kSU);
    if (does_codes) issue_codes<GS, BITS>(p, u, c, slot, &full[j]);
    if (does_meta) issue_meta<GS, BITS>(p, u, c, slot, &full[j]);
  };
  int next = si;  // next slot sequence number to issue
  if (next * kSU < nw) {
    if (si > 0 && kStaggerCycles > 0) pause_cycles(kStaggerCycles * si);
    issue(next);
    next += kRing;
  }
  // Refills once the consumer has released the slot (bounded: on a timeout the lane records it, stops issuing
  // and drains what it issued).
  bool ok = true;
  while (next * kSU < nw) {
    const int use = next / kRing;  // uses of this slot so far; the consumer's release of use - 1 frees it
    if (!mbar_wait_backoff(&empty[j], (unsigned)(use - 1) & 1u, p.status)) {
      ok = false;
      break;
    }
    issue(next);
    next += kRing;
  }
  if (!ok) {  // drain: every copy this lane issued lands before the CTA can exit
    const int last = next - kRing;
    if (last >= 0 && last * kSU < nw) mbar_wait(&full[j], (unsigned)(last / kRing) & 1u, p.status);
  }
}

template <int NT, bool XS, bool DIVS, int GS, int BITS>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(const GemvParams p) {
  using Ge = Geo<GS, BITS>;
  constexpr int kSU = Ge::SU, CH = Ge::CH;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kSlots];
  __shared__ __align__(8) uint64_t empty[kSlots];
  __shared__ __align__(8) uint64_t xbar;
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = p.G;
  const int c = blockIdx.x;
  const int cu0 = cta_first_unit(p, c), n = cta_units(p, c), cu1 = cu0 + n;
  const int mcount = min(8 * NT, p.M - p.m0);
  uint8_t* ring = smem;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + Ge::RING);
  float* s_part = reinterpret_cast<float*>(smem + Ge::RING + (XS ? gemv_xs_bytes(mcount, p.xpitch) : 0));

  for (int j = threadIdx.x; j < kSlots; j += kThreads) {
    mbar_init(&full[j], 1);
    mbar_init(&empty[j], 1);
  }
  if (XS && threadIdx.x == 0) mbar_init(&xbar, 1);
  fence_mbar_init();
  __syncthreads();

  if (warp == kNW) {  // ---------------------------------------------------------------- producer warp
    // L2 prefetch of a later call's weights (a caller's hint), spread over the CTAs; weights only.
    if (p.pf != nullptr && p.m0 == 0 && lane == 31) {
      const unsigned long long a = (unsigned long long)c * p.pf_share;
      const unsigned long long e = a + p.pf_share < p.pf_bytes ? a + p.pf_share : p.pf_bytes;
      for (unsigned long long o = a; o < e; o += 32768ull)
        prefetch_l2_bulk(p.pf + o, (unsigned)(e - o < 32768ull ? e - o : 32768ull));
    }
    gemv_producer<GS, BITS>(p, ring, full, empty, cu0, n, lane);
    return;
  }

  // ------------------------------------------------------------------------------------ consumer warps
  const int g4 = lane >> 2, t4 = lane & 3;
  int wu0, nw;
  warp_range(cu0, n, warp, wu0, nw);
  const int wu1 = wu0 + nw;
  const bool active = nw > 0;
  const uint32_t ring_addr = smem_u32(ring) + (uint32_t)(warp * kRing * Ge::STRIDE);
  const uint32_t empty_addr = smem_u32(&empty[warp * kRing]);
#if AWQ_GEMV_L2_PREFETCH
  // Before the dependency wait the consumers are idle: each asks for its whole range of codes (32 KB per
  // lane, lanes in parallel) and of scales and zeros to be brought towards L2, so HBM streams at full rate
  // from the kernel's start and the producer's ring copies mostly hit L2.
  if (active) {
    const int chunks = (nw * Ge::UB + 32767) / 32768;
    for (int ch = lane; ch < chunks; ch += 30) {
      const int off = ch * 32768;
      prefetch_l2_bulk(p.qw + (size_t)wu0 * Ge::UB + off, (unsigned)min(32768, nw * Ge::UB - off));
    }
    if (lane == 30) prefetch_l2_bulk(p.scales + (size_t)wu0 * 32, (unsigned)(nw * 64));
    if (lane == 31) prefetch_l2_bulk(p.qzeros + (size_t)wu0 * 4, (unsigned)(nw * 16));
  }
#endif
  pdl_wait_prior_grids();  // activations, outputs and workspace follow the stream order

  const uint16_t* xrow[NT];  // this lane's B column (row 8 nt + g4 of the pass, clamped) per n-tile
  if (XS) {  // x' rows of this pass -> shared memory, one bulk copy per row (padded pitch)
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(&xbar, (unsigned)(mcount * p.K * 2));
      for (int m = 0; m < mcount; ++m)
        bulk_g2s(xs + m * p.xpitch, p.x + (size_t)(p.m0 + m) * p.K, (unsigned)(p.K * 2), &xbar);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) xrow[nt] = xs + min(8 * nt + g4, mcount - 1) * p.xpitch;
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) xrow[nt] = p.x + (size_t)(p.m0 + min(8 * nt + g4, mcount - 1)) * p.K;
  }
  const int rb_f = active ? wu0 / G : -1;
  const int g0 = active ? wu0 - rb_f * G : 0;
  const int rb_l = active ? (wu1 - 1) / G : -1;  // the warp's last row block

  bool ok = true;
  if (XS && (active || DIVS)) ok = __all_sync(0xFFFFFFFFu, mbar_wait_backoff(&xbar, 0u, p.status));
  if (DIVS) {
    // x' = fp16(x / s) in place, every consumer thread taking 8 channels at a time.  The correctly rounded
    // fp32 quotient rounds to the same fp16 as the exact quotient of two fp16 values (it never lands on an
    // fp16 rounding midpoint unless the exact quotient is that midpoint), so x' is bit-identical to
    // awq_apply_inv_scale's fp64 result.
    if (ok) {
      const int ct = threadIdx.x;  // 0 .. kNW * 32 - 1
      for (int m = 0; m < mcount; ++m)
        for (int k = ct * 8; k < p.K; k += kNW * 32 * 8) {
          uint4 xv = *reinterpret_cast<const uint4*>(xs + m * p.xpitch + k);
          const uint4 sv = ldg_cached(p.s + k);
          uint32_t* xw = reinterpret_cast<uint32_t*>(&xv);
          const uint32_t* sw = reinterpret_cast<const uint32_t*>(&sv);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __half2 xh = u32_as_h2(xw[i]), sh = u32_as_h2(sw[i]);
            const __half lo = __float2half_rn(__fdiv_rn(__low2float(xh), __low2float(sh)));
            const __half hi = __float2half_rn(__fdiv_rn(__high2float(xh), __high2float(sh)));
            xw[i] = h2_as_u32(__halves2half2(lo, hi));
          }
          *reinterpret_cast<uint4*>(xs + m * p.xpitch + k) = xv;
        }
    }
    named_barrier_sync(3, kNW * 32);  // every consumer sees the divided x'
  }
  uint4 xb[NT][CH];
  if (!XS && active) load_xb<NT, GS>(xrow, g0, t4, xb);
  int rb = rb_f, g = g0;
  int t = 0;  // units of this warp consumed so far
  while (t < nw && ok) {  // segments: the units of one row block inside this warp's range
    const int seg = min(nw - t, G - g);
    const bool whole = (g == 0) && (seg == G);
    float yacc[NT][4][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) yacc[nt][i][0] = yacc[nt][i][1] = 0.f;
    for (int i = 0; i < seg; ++i, ++t) {
      const int sq = t / kSU, ui = t & (kSU - 1);  // slot sequence number and unit within the slot
      const int si = sq & (kRing - 1);
      const uint32_t slot = ring_addr + (uint32_t)(si * Ge::STRIDE);
      uint4 xcur[NT][CH];
      if (XS) {  // B fragments from the staged x'
        load_xb<NT, GS>(xrow, g + i, t4, xcur);
      } else {  // loaded one unit ahead from global memory; start the next unit's loads
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int cc = 0; cc < CH; ++cc) xcur[nt][cc] = xb[nt][cc];
        if (t + 1 < nw) load_xb<NT, GS>(xrow, (g + i + 1 == G) ? 0 : g + i + 1, t4, xb);
      }
      if (ui == 0) {  // first unit of the slot: wait for its copies
        ok = __all_sync(0xFFFFFFFFu, mbar_wait_backoff(&full[warp * kRing + si], (unsigned)(sq / kRing) & 1u, p.status));
        if (!ok) break;  // warp-uniform
      }
      if (BITS == 4)
        unit_mma<NT, CH>(slot + (uint32_t)(ui * Ge::UB), slot + (uint32_t)(Ge::SCO + ui * 64),
                         slot + (uint32_t)(Ge::ZO + ui * 16), g4, t4, xcur, yacc);
      else
        unit_mma3<NT, CH>(slot + (uint32_t)(ui * Ge::UB), slot + (uint32_t)(Ge::SCO + ui * 64),
                          slot + (uint32_t)(Ge::ZO + ui * 16), g4, t4, xcur, yacc);
      if (ui == kSU - 1 || t == nw - 1) {  // last unit of the slot: every lane has read it; release it
        __syncwarp();
        if (lane == 0) mbar_arrive_addr(empty_addr + 8u * (uint32_t)si);
      }
    }
    if (!ok) break;
    if (whole) {
      store_frag<NT>(p, rb, g4, t4, mcount, yacc);
    } else {
      const int sl = (rb == rb_f) ? 0 : 1;
      stash_frag<NT>(s_part + (size_t)(warp * 2 + sl) * mcount * 32, g4, t4, mcount, yacc);
    }
    ++rb;
    g = 0;
  }
  // A consumer that gave up leaves the producer's remaining refills unreleased; the producer's bounded
  // waits run out and it drains its own copies.
  if (XS && threadIdx.x == 0 && !mbar_try_wait(&xbar, 0u)) mbar_wait(&xbar, 0u, p.status);  // x' copy landed
  named_barrier_sync(1, kNW * 32);  // consumer warps only: their partials are in shared memory
  if (!active) return;
  // A split row block r is combined by the warp holding its first unit inside this CTA.  This runs
  // whether or not a wait gave up, so that every counter returns to zero.
  const int wq = n / kNW, wr = n % kNW;
  // The partial of warp j for row block r sits in its slot 0 when r is warp j's first row block, else in slot 1.
  // All warps' loads are issued together (unrolled, predicated), so the reduction costs one load latency.
  auto combine = [&](int r) {
    const int a = max(r * G, cu0), b = min((r + 1) * G, cu1);
    float sum[8 * NT];
#pragma unroll
    for (int m = 0; m < 8 * NT; ++m) sum[m] = 0.f;
#pragma unroll
    for (int j = 0; j < kNW; ++j) {
      const int j0 = cu0 + wq * j + min(j, wr), jn = wq + (j < wr ? 1 : 0);
      // warp j holds units [j0, j0 + jn); it has a partial of r iff that range meets [a, b)
      const bool has = jn > 0 && j0 < b && j0 + jn > a;
      const float* src = s_part + (size_t)(j * 2 + ((j0 >= r * G) ? 0 : 1)) * mcount * 32 + lane;
#pragma unroll
      for (int m = 0; m < 8 * NT; ++m)
        if (has && m < mcount) sum[m] += src[m * 32];
    }
    if (a == r * G && b == (r + 1) * G) store_row<NT>(p, r, lane, mcount, sum);
    else cross_cta_combine<NT>(p, r, lane, mcount, sum);
  };
  const bool whole_f = (g0 == 0) && (nw >= G);
  const bool owner_f = (g0 == 0) || (wu0 == cu0);
  if (owner_f && !whole_f) combine(rb_f);
  if (rb_l != rb_f && wu1 - rb_l * G < G) combine(rb_l);
}

// ------------------------------------------------------------------------------------------ host
#ifndef AWQ_GEMV_CTAS_PER_SM
#define AWQ_GEMV_CTAS_PER_SM 1
#endif


namespace {

template <int NT, bool XS, bool DIVS, int GS, int BITS>
bool gemv_smem_attr() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(gemv_kernel<NT, XS, DIVS, GS, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMaxDynSmem) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

int ring_bytes(int gs, int bits) {
  if (bits == 3) return gs == 64 ? Geo<64, 3>::RING : gs == 128 ? Geo<128, 3>::RING : Geo<256, 3>::RING;
  return gs == 64 ? Geo<64>::RING : gs == 128 ? Geo<128>::RING : Geo<256>::RING;
}

struct GemvPlan {
  int NT, mts, RB, G, U, P, q, r, S, gran;
  bool xs;     // x' staged in shared memory
  int xpitch;  // its row pitch in halves
  size_t part_bytes;
};

// Three shapes of work, at most AWQ_GEMV_CTAS_PER_SM CTAs per SM:
//  - at most that many row blocks: one CTA per row block; its warps split the row block's groups and
//    combine in shared memory -- no partial sum leaves a CTA;
//  - more row blocks, evenly enough divisible: each CTA takes a balanced run of whole row blocks;
//  - otherwise (a few row blocks more than CTAs) the units are spread evenly over the CTAs and the row
//    blocks cut by CTA boundaries are combined in the workspace.
GemvPlan plan_gemv(int M, int N, int K, int gs, bool divide = false, int bits = 4) {
  GemvPlan pl{};
  pl.NT = M <= 8 ? 1 : 2;
  pl.mts = M < 8 * pl.NT ? M : 8 * pl.NT;
  pl.RB = (N + 31) / 32;
  pl.G = K / gs;
  pl.U = pl.RB * pl.G;
  pl.xpitch = K + kXPad;
  const int p_max = num_sms() * AWQ_GEMV_CTAS_PER_SM;
  pl.S = 1;
  pl.part_bytes = 0;
  pl.gran = pl.G;
  if (pl.RB <= p_max) {
    pl.P = pl.RB;
  } else if ((pl.RB + p_max - 1) / p_max * p_max <= pl.RB * 3 / 2) {
    // Whole row blocks per CTA (3 or 4 per CTA for 448 row blocks on 148 SMs): no partial sum leaves a CTA.
    // Measured on the 4096 -> 14336 linear at M = 1: 10.9 us, against 12.5 us with balanced units and the
    // workspace combine.  Kept while the busiest CTA has at most 1.5x the average work.
    pl.P = p_max;
  } else {
    pl.P = p_max;
    pl.gran = 1;
    const int L = pl.U / pl.P;  // >= 1 units per CTA
    pl.S = pl.G >= 2 ? (pl.G - 2) / L + 2 : 1;
    pl.part_bytes = (size_t)pl.RB * pl.S * 32 * pl.mts * sizeof(float);
  }
  pl.q = pl.U / pl.gran / pl.P;
  pl.r = pl.U / pl.gran % pl.P;
  // x' staged in shared memory when it fits and each warp's range covers at least a third of the groups (a
  // warp with few units reads only its own groups' x' more cheaply from global memory: measured on the M = 1
  // decode shapes, q/o 4.83 -> 4.51 us and down 11.08 -> 10.96 us unstaged, gate/up 10.64 vs 10.96 staged).
  // The fused 1/s variant divides the staged copy, so it stages whatever fits beside the rings and partials.
  const int units_per_warp = pl.U / pl.P / kNW;
  pl.xs = (divide || (pl.mts * pl.xpitch * 2 <= kXsMaxBytes && 3 * units_per_warp >= pl.G)) &&
          ring_bytes(gs, bits) + gemv_xs_bytes(pl.mts, pl.xpitch) + gemv_part_bytes(pl.mts) <= kMaxDynSmem;
  return pl;
}

template <int NT, bool XS, bool DIVS, int GS, int BITS>
cudaError_t launch_nt(const GemvParams& p, int mcount, cudaStream_t st) {
  if (!gemv_smem_attr<NT, XS, DIVS, GS, BITS>()) return cudaErrorInvalidValue;
  const size_t smem =
      (size_t)Geo<GS, BITS>::RING + (XS ? gemv_xs_bytes(mcount, p.xpitch) : 0) + gemv_part_bytes(mcount);
  return launch_pdl(gemv_kernel<NT, XS, DIVS, GS, BITS>, dim3((unsigned)p.P), dim3(kThreads), smem, st, p);
}

template <int GS>
cudaError_t launch_gs(const GemvParams& p, int NT, bool xs, bool divide, int mcount, cudaStream_t st, int bits) {
  if (bits == 3) {  // the 3-bit layout: plain x' only
    if (NT == 1) return xs ? launch_nt<1, true, false, GS, 3>(p, mcount, st) : launch_nt<1, false, false, GS, 3>(p, mcount, st);
    return xs ? launch_nt<2, true, false, GS, 3>(p, mcount, st) : launch_nt<2, false, false, GS, 3>(p, mcount, st);
  }
  if (divide)
    return NT == 1 ? launch_nt<1, true, true, GS, 4>(p, mcount, st) : launch_nt<2, true, true, GS, 4>(p, mcount, st);
  if (NT == 1) return xs ? launch_nt<1, true, false, GS, 4>(p, mcount, st) : launch_nt<1, false, false, GS, 4>(p, mcount, st);
  return xs ? launch_nt<2, true, false, GS, 4>(p, mcount, st) : launch_nt<2, false, false, GS, 4>(p, mcount, st);
}

}  // namespace

size_t gemv_workspace_bytes(int M, int N, int K, int g) {
  const GemvPlan pl = plan_gemv(M, N, K, g);  // the fused 1/s variant has the same plan (same split)
  return pl.part_bytes == 0 ? 0 : kWorkspaceCounterBytes + pl.part_bytes;
}

awq_status gemv_launch(const LinearArgs& a) {
  const bool divide = a.inv_s != nullptr;
  if (a.bits == 3 && (divide || a.epi)) return AWQ_ERR_UNSUPPORTED;
  const GemvPlan pl = plan_gemv(a.M, a.N, a.K, a.g, divide, a.bits);
  if (divide && !pl.xs) return AWQ_ERR_UNSUPPORTED;  // x / s needs the staged copy
  if ((size_t)pl.RB * 4 > kWorkspaceCounterBytes) return AWQ_ERR_UNSUPPORTED;
  if (pl.part_bytes > 0 && (a.ws == nullptr || a.ws_bytes < kWorkspaceCounterBytes + pl.part_bytes))
    return AWQ_ERR_WORKSPACE;
  GemvParams p;
  p.x = a.x;
  p.s = a.inv_s;
  p.qw = reinterpret_cast<const uint8_t*>(a.qw);
  p.scales = a.scales;
  p.qzeros = a.qzeros;
  p.y = a.y;
  p.epi = a.epi;
  p.ny = a.epi ? a.N / 2 : a.N;
  p.ws_cnt = static_cast<unsigned*>(a.ws);
  p.ws_part = a.ws ? reinterpret_cast<float*>(static_cast<char*>(a.ws) + kWorkspaceCounterBytes) : nullptr;
  p.status = a.status;
  p.pf = a.pf_bytes > 0 ? static_cast<const uint8_t*>(a.pf) : nullptr;
  p.pf_bytes = a.pf_bytes;
  p.pf_share = ((a.pf_bytes + (size_t)pl.P - 1) / (size_t)pl.P + 15) / 16 * 16;
  p.U = pl.U;
  p.P = pl.P;
  p.q = pl.q;
  p.r = pl.r;
  p.gran = pl.gran;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.G = pl.G;
  p.RB = pl.RB;
  p.S = pl.S;
  p.mts = pl.mts;
  p.xpitch = pl.xpitch;
  // passes of 8 * NT rows run one after the other on the stream and share the workspace
  const int rows = 8 * pl.NT;
  for (int m0 = 0; m0 < a.M; m0 += rows) {
    p.m0 = m0;
    const int mcount = a.M - m0 < rows ? a.M - m0 : rows;
    cudaError_t e;
    switch (a.g) {
      case 64: e = launch_gs<64>(p, pl.NT, pl.xs, divide, mcount, a.st, a.bits); break;
      case 256: e = launch_gs<256>(p, pl.NT, pl.xs, divide, mcount, a.st, a.bits); break;
      default: e = launch_gs<128>(p, pl.NT, pl.xs, divide, mcount, a.st, a.bits); break;
    }
    if (e != cudaSuccess) return AWQ_ERR_CUDA;
  }
  return AWQ_OK;
}

}  // namespace awq
