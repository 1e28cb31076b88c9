// ta_attn_common.cuh -- pieces shared by the fused attention kernels: the
// tile walk of a row's compacted list, exponentials and number-format packing
// of P', and the TMEM / shared-memory layout of NVFP4 block scales.
#pragma once

#include "ta_common.cuh"
#include "ta_kernels.cuh"

namespace ta {
namespace tile {

enum TileKind { KIND_FULL = 0, KIND_LOW = 1, KIND_SKIP = 2, KIND_RES = 3 };

struct RowPlan {
  int n_full, n_res, n_low, n_skip;
  int T;             // number of tiles (skip blocks chunked by BK)
  const int* list;   // this row's list
};

// Tile t of a row: its kind and the position of its (first) key block in the
// row's list.  Kept tiles come in list order (full, residual, low); skipped
// blocks follow in chunks of BK.
template <int BK>
__device__ __forceinline__ void tile_of(const RowPlan& rp, int t, int& kind, int& first) {
  const int kept = rp.n_full + rp.n_res + rp.n_low;
  if (t < kept) {
    kind = t < rp.n_full ? KIND_FULL : (t < rp.n_full + rp.n_res ? KIND_RES : KIND_LOW);
    first = t;
  } else {
    kind = KIND_SKIP;
    first = kept + (t - kept) * BK;
  }
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for two floats on the FMA pipe, leaving the MUFU unit to ex2.approx:
// x = j + f with j = rint(x) from the magic-number addition (x + 1.5 * 2^23
// rounds to an integer in the low mantissa bits), 2^f for f in [-1/2, 1/2]
// by the cubic 1 + f (c1 + f (c2 + f c3)), and j added into the exponent
// field of the result.  The coefficients are a minimax fit of our own
// (Lawson's iteratively reweighted least squares on the relative error, with
// p(0) = 1 so that integer arguments give exact powers of two): relative
// error <= 1.02e-4 in fp32.  x is clamped below at -125 (masked columns
// arrive as -inf and come out as 2^-125, which no sum or rounding of P'
// against a row maximum of 2^o notices).
__device__ __forceinline__ void exp2_poly2(float a0, float a1, float& y0, float& y1) {
  constexpr float kMagic = 12582912.0f;
  const float x0 = fmaxf(a0, -125.0f), x1 = fmaxf(a1, -125.0f);
  const uint64_t x = pack2(x0, x1);
  const uint64_t t = add2(x, pack2(kMagic, kMagic));
  const uint64_t j = add2(t, pack2(-kMagic, -kMagic));
  const uint64_t f = fma2(j, pack2(-1.0f, -1.0f), x);
  uint64_t p = fma2(f, pack2(0.055008940398693085f, 0.055008940398693085f),
                    pack2(0.2422109991312027f, 0.2422109991312027f));
  p = fma2(f, p, pack2(0.6932829022407532f, 0.6932829022407532f));
  p = fma2(f, p, pack2(1.0f, 1.0f));
  float p0, p1, t0, t1;
  unpack2(p, p0, p1);
  unpack2(t, t0, t1);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Low-tier execution mode of a kernel instance.
enum LowMode { LM_IMAGE = 0, LM_NVFP4 = 1, LM_NVFP4_RES = 2, LM_FP8 = 3 };

// TMEM columns of one CTA: S of even and of odd tiles, the O accumulator, the
// block scales of the narrow MMAs, and bf16 P (the A operand of the TMEM x
// shared-memory PV product).  Block scales (4 columns per 64-element K chunk,
// 2 chunks per operand) have one slot per operand: the thread that issues the
// MMAs reading a slot also refills it, and its tcgen05 operations run in issue
// order.
template <int D, int BK, int LM>
struct TmemMap {
  static constexpr bool FP4 = (LM == LM_NVFP4 || LM == LM_NVFP4_RES);
  static constexpr bool F8 = (LM == LM_FP8);
  static constexpr uint32_t NC = (LM == LM_NVFP4_RES) ? 2 : 1;   // NVFP4 copies
  static constexpr uint32_t kS0 = 0, kS1 = BK, kO = 2 * BK, kSf = 2 * BK + D;
  // NVFP4: query copy c, key copy c, V copy c, P copy c
  static constexpr __device__ uint32_t sfaQ(int c) { return kSf + 8 * c; }
  static constexpr __device__ uint32_t sfbK(int c) { return kSf + 8 * NC + 8 * c; }
  static constexpr __device__ uint32_t sfbV(int c) { return kSf + 16 * NC + 8 * c; }
  static constexpr __device__ uint32_t sfaP(int c) { return kSf + 24 * NC + 8 * c; }
  // FP8: UE8M0 scale factors of P (constant 2^0) and of V
  static constexpr __device__ uint32_t sfaP8() { return kSf; }
  static constexpr __device__ uint32_t sfbV8() { return kSf + 4; }
  static constexpr uint32_t kSfEnd = FP4 ? kSf + 32 * NC : (F8 ? kSf + 8 : kSf);
  static constexpr uint32_t kP = kSfEnd;            // bf16 P: BK/2 columns
  static constexpr uint32_t kEnd = kP + BK / 2;
  static constexpr uint32_t kCols = kEnd <= 256 ? 256u : 512u;
  static_assert(kEnd <= 512, "TMEM columns");
};

// NVFP4 tiles in shared memory: codes [rows][64 B] with 64-byte swizzle, then
// the two [32][16 B] scale-factor blocks at +kFp4Sf.
constexpr int kFp4Sf = 128 * 64;

// Gather the ue4m3 scales of `nrows` rows (row-major, 8 bytes = 8 groups of 16
// along d = 128) into the two [32][16 B] blocks at `dst`: row 32*m1 + m0 of K
// chunk c (groups 4c..4c+3) at dst + c*512 + m0*16 + m1*4.  Rows past
// `nrows` get zero scales.
__device__ __forceinline__ void gather_row_sf(unsigned char* dst, const uint8_t* src, int nrows,
                                              int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = lane * 4 + i;
    uint2 v = make_uint2(0u, 0u);
    if (rr < nrows) v = *reinterpret_cast<const uint2*>(src + (int64_t)rr * 8);
    const int off = (rr & 31) * 16 + (rr >> 5) * 4;
    *reinterpret_cast<uint32_t*>(dst + off) = v.x;
    *reinterpret_cast<uint32_t*>(dst + 512 + off) = v.y;
  }
}

// NVFP4 of 32 non-negative P' values, two groups of 16 keys: sc =
// ue4m3_rn(fp32(amax / 6)), code = e2m1_rn_satfinite(fp32(x * fp32(1 / sc)))
// (code 0 when sc = 0).  Codes go to p[0..3] (element i of a word in nibble
// i); the two scale codes come back in the low 16 bits.  `sc_tab[c]` holds
// (value, correctly rounded reciprocal) of ue4m3 code c.
__device__ __forceinline__ uint32_t nvfp4_quant32(const float* x, const float2* sc_tab,
                                                  uint32_t* p) {
  uint32_t scw = 0u;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < 16; ++i) am[i & 3] = fmaxf(am[i & 3], x[g * 16 + i]);
    const float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
    const uint32_t scc = cvt_e4m3x2(div6(amax), 0.0f) & 0xFFu;
    const float inv = sc_tab[scc].y;
    scw |= scc << (8 * g);
    const uint64_t inv2 = pack2(inv, inv);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2)
        unpack2(mul2(pack2(x[g * 16 + w * 8 + i], x[g * 16 + w * 8 + i + 1]), inv2), y[i], y[i + 1]);
      p[g * 2 + w] = cvt_e2m1x8(y);
    }
  }
  return scw;
}

// The same, with each group's amax given (the P' of its largest S, taken
// from the maximum pass): no maximum over the 16 values here.
__device__ __forceinline__ uint32_t nvfp4_quant32_am(const float* x, float am0, float am1,
                                                     const float2* sc_tab, uint32_t* p) {
  uint32_t scw = 0u;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const uint32_t scc = cvt_e4m3x2(div6(g ? am1 : am0), 0.0f) & 0xFFu;
    const float inv = sc_tab[scc].y;
    scw |= scc << (8 * g);
    const uint64_t inv2 = pack2(inv, inv);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2)
        unpack2(mul2(pack2(x[g * 16 + w * 8 + i], x[g * 16 + w * 8 + i + 1]), inv2), y[i], y[i + 1]);
      p[g * 2 + w] = cvt_e2m1x8(y);
    }
  }
  return scw;
}

// The residual copy of the same 32 values: r = fp32(x - deq(first copy)),
// quantised by the same rule on |r| (codes keep the sign).
__device__ __forceinline__ uint32_t nvfp4_residual32(const float* x, const uint32_t* p,
                                                     uint32_t scw, const float2* sc_tab,
                                                     uint32_t* p2) {
  uint32_t scw2 = 0u;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const float sc1 = sc_tab[(scw >> (8 * g)) & 0xFFu].x;
    // x - code * sc1 in one rounding: code * sc1 is exact in fp32 (at most
    // 2 + 4 significant bits), so a fused multiply-add rounds like the
    // subtraction of that exact product
    const uint64_t nsc1 = pack2(-sc1, -sc1);
    float rr[16];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const float2 f = __half22float2(e2m1x2_to_half2(p[g * 2 + w] >> (8 * bb)));
        const int c = w * 8 + 2 * bb;
        unpack2(fma2(pack2(f.x, f.y), nsc1, pack2(x[g * 16 + c], x[g * 16 + c + 1])), rr[c], rr[c + 1]);
      }
    }
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(rr[i]));
    const uint32_t scc2 = cvt_e4m3x2(div6(am), 0.0f) & 0xFFu;
    const float inv2 = sc_tab[scc2].y;
    scw2 |= scc2 << (8 * g);
    const uint64_t inv22 = pack2(inv2, inv2);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2)
        unpack2(mul2(pack2(rr[w * 8 + i], rr[w * 8 + i + 1]), inv22), y[i], y[i + 1]);
      p2[g * 2 + w] = cvt_e2m1x8(y);
    }
  }
  return scw2;
}

}  // namespace tile
}  // namespace ta
