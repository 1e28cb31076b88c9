// ta_prep.cu -- one pass over Q, K, V: block means for the router and the
// low-precision copies for the low / refine tiers.
//
// "Triage" (zhuanzhiai paper page, abstract) routes tiles from block
// statistics and runs them in NVFP4 (skim) or NVFP4 plus a residual term
// (refine); the skip tier replaces a tile by its block means.  Every one of
// those needs a full read of Q, K and V, so this kernel reads each token row
// exactly once and produces all of them:
//   * fp64 block sums -> qbar (per query block), kbar (per key block), and the
//     bf16 (round-to-nearest-even) kbar_b / vbar_b used by the skip tier;
//     for the price router also each query and key block's coordinate
//     variances;
//   * FP8 e4m3: one power-of-two scale per tile (the smallest 2^k with
//     amax <= 448 * 2^k), codes = e4m3_rn_satfinite(x * 2^-k);
//   * NVFP4: per 16 elements along d (Q, K rows) or along tokens (V columns,
//     groups aligned to token 0) a ue4m3 scale sc = e4m3_rn(amax / 6), codes
//     e2m1_rn_satfinite(x * rcp_rn(sc)); residual copies quantise
//     fp32(x - dequant(x)) the same way.
// One CTA per (chunk of R = max(bq, bk) tokens, head, operand Q / K / V); the
// chunk is staged in shared memory with 16-byte coalesced loads and written
// back coalesced.
#include "ta_common.cuh"
#include "ta_kernels.cuh"

namespace ta {
namespace {

constexpr int kThreads = 256;

// The two bf16 values of a 32-bit word as fp32 (exact), element 0 in the low half.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16 bytes global -> shared without a register round trip; src_bytes = 0
// writes zeros (and reads nothing).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Smallest power of two s with amax <= 448 s (1 when amax == 0).
__device__ __forceinline__ float fp8_pow2_scale(float amax) {
  if (amax == 0.0f) return 1.0f;
  int e;
  const float m = frexpf(amax, &e);  // amax = m * 2^e, m in [0.5, 1); 448 = 0.875 * 2^9
  const int k = (m <= 0.875f) ? e - 9 : e - 8;
  return ldexpf(1.0f, k);
}

// NVFP4 of one group of 16 values: returns the ue4m3 scale code
// sc = e4m3_rn(amax / 6); the codes e2m1_rn_satfinite(x * rcp_rn(sc)) go to
// `packed`, element i in nibble i (a zero scale gives zero codes).
// `tab[c]` = (value, correctly rounded 1 / value) of ue4m3 code c.
__device__ __forceinline__ uint32_t nvfp4_group(const float (&x)[16], uint32_t (&packed)[2],
                                                const float2* tab) {
  // amax of |x| with three-input maxima: 8 instructions for 16 values
  float am[3];
#pragma unroll
  for (int u = 0; u < 3; ++u)
    am[u] = fmax3(fabsf(x[5 * u]), fabsf(x[5 * u + 1]), fmax3(fabsf(x[5 * u + 2]), fabsf(x[5 * u + 3]),
                                                               fabsf(x[5 * u + 4])));
  const float amax = fmax3(am[0], fmax3(am[1], am[2], fabsf(x[15])), 0.0f);
  const uint32_t scc = cvt_e4m3x2(div6(amax), 0.0f) & 0xFFu;
  const float inv = tab[scc].y;
  const uint64_t inv2 = pack2(inv, inv);
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2)
      unpack2(mul2(pack2(x[w * 8 + i], x[w * 8 + i + 1]), inv2), y[i], y[i + 1]);
    const uint32_t c = cvt_e2m1x8(y);
    packed[w] = scc ? c : 0u;
  }
  return scc;
}

// The residual of a quantised group, r = fp32(x - code * sc).  code * sc is
// exact in fp32 (at most 2 + 4 significant bits), so one fused multiply-add
// per pair rounds like the subtraction of that exact product.
__device__ __forceinline__ void nvfp4_residual(const float (&x)[16], const uint32_t (&packed)[2],
                                               float sc, float (&r)[16]) {
  const uint64_t nsc = pack2(-sc, -sc);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f = __half22float2(e2m1x2_to_half2(packed[i >> 2] >> (8 * (i & 3))));
    unpack2(fma2(pack2(f.x, f.y), nsc, pack2(x[2 * i], x[2 * i + 1])), r[2 * i], r[2 * i + 1]);
  }
}

// Shared memory of one CTA: the staged chunk [R][D] bf16, then a region that
// first holds the partial column sums (fp64) and maxima (fp32) [SEG][D] and
// later the V codes in transit [2 copies][R / 16][D + 2] uint2, then the FP8
// tile scales.
template <int D, int R>
struct PrepSmem {
  static constexpr int CP = D / 2;            // column pairs
  static constexpr int SEG = kThreads / CP;   // row segments of the column sums
  static constexpr int RS = R / SEG;          // rows per segment
  static constexpr int G = R / 16;            // 16-token groups of a V column
  static constexpr int VP = D + 2;            // uint2 pitch of a group's V codes
  static constexpr size_t oTile = 0;
  static constexpr size_t oPsum = oTile + (size_t)R * D * 2;
  static constexpr size_t oRed = oPsum + (size_t)SEG * D * 8;
  static constexpr size_t oVst = oPsum;
  static constexpr size_t kSums = (size_t)SEG * D * 12, kVst = (size_t)2 * G * VP * 8;
  static constexpr size_t oScale = oPsum + (kSums > kVst ? kSums : kVst);
  static constexpr size_t kBytes = oScale + 8 * sizeof(float);
  static_assert(kThreads % CP == 0 && R % SEG == 0 && 32 % RS == 0,
                "a row segment must lie inside one block (blocks of 32, 64 or 128 rows)");
  static_assert(SEG >= R / 32, "the column maxima of every block fit the reduction area");
};

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 4) prep_kernel(const PlanArgs a) {
  using L = PrepSmem<D, R>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(smem_raw + L::oTile);
  const uint32_t* tile32 = reinterpret_cast<const uint32_t*>(tile);
  double* psum = reinterpret_cast<double*>(smem_raw + L::oPsum);
  float* red = reinterpret_cast<float*>(smem_raw + L::oRed);
  uint2* vst = reinterpret_cast<uint2*>(smem_raw + L::oVst);
  float* tile_scale = reinterpret_cast<float*>(smem_raw + L::oScale);

  __shared__ float2 sc_tab[128];   // ue4m3 code -> (value, correctly rounded 1 / value)
  const int tid = threadIdx.x;
  if (tid < 128) {
    const float v = (tid == 0x7F) ? 0.0f : e4m3_to_float(tid);
    sc_tab[tid] = make_float2(v, v > 0.0f ? __frcp_rn(v) : 0.0f);
  }
  const int which = blockIdx.z;
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int r0 = blockIdx.x * R;
  const int nrows = min(R, a.N - r0);
  const int64_t bhN = (int64_t)bh * a.N;
  const __nv_bfloat16* src =
      (which == 0 ? a.Q : which == 1 ? a.K : a.V) + (int64_t)b * a.sb + (int64_t)h * a.sh;

  // ---- stage the chunk; rows past N are zeros ----
  for (int idx = tid; idx < R * (D / 8); idx += kThreads) {
    const int r = idx / (D / 8), c8 = idx % (D / 8);
    const bool in = r < nrows;
    cp_async16(tile + r * D + c8 * 8, src + (int64_t)(r0 + (in ? r : 0)) * a.sn + c8 * 8,
               in ? 16u : 0u);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  // ---- block sums in fp64 and column maxima.  A sum of bf16 values is exact
  // in fp64 while a block's values span at most 38 binades (53 - 8 - 7 bits),
  // and then the order of the additions does not matter.  Each thread takes
  // two adjacent columns over one segment of RS rows (zero rows add nothing) ----
  // block sizes are powers of two (32, 64 or 128 rows): shifts, not divisions
  const int blk = (which == 0) ? a.bq : a.bk;
  const int lb = __ffs(blk) - 1;            // log2(blk)
  const int nb = R >> lb;
  {
    const int cp = tid % L::CP, seg = tid / L::CP;
    const uint32_t* col = tile32 + seg * L::RS * L::CP + cp;
    double s0 = 0.0, s1 = 0.0;
    float m0 = 0.0f, m1 = 0.0f;
    if (a.low == TA_LOW_FP8_E4M3) {
      // column maxima: only the FP8 tile scale needs them
#pragma unroll 8
      for (int r = 0; r < L::RS; ++r) {
        const uint32_t w = col[r * L::CP];
        const float lo = bf_lo(w), hi = bf_hi(w);
        s0 += (double)lo;
        s1 += (double)hi;
        m0 = fmaxf(m0, fabsf(lo));
        m1 = fmaxf(m1, fabsf(hi));
      }
    } else {
#pragma unroll 8
      for (int r = 0; r < L::RS; ++r) {
        const uint32_t w = col[r * L::CP];
        s0 += (double)bf_lo(w);
        s1 += (double)bf_hi(w);
      }
    }
    *reinterpret_cast<double2*>(psum + seg * D + 2 * cp) = make_double2(s0, s1);
    *reinterpret_cast<float2*>(red + seg * D + 2 * cp) = make_float2(m0, m1);
  }
  __syncthreads();
  // nb * D (block, column) pairs, at most kPer per thread
  constexpr int kPer = (R / 32) * D / kThreads > 0 ? (R / 32) * D / kThreads : 1;
  double s[kPer];
  float amax_c[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int w = tid + u * kThreads;
    s[u] = 0.0;
    amax_c[u] = 0.0f;
    if (w < nb * D) {
      const int jb = w / D, c = w % D;
      const int spb = L::SEG >> (__ffs(nb) - 1);   // segments per block
      for (int k = 0; k < spb; ++k) {
        s[u] += psum[(jb * spb + k) * D + c];
        amax_c[u] = fmaxf(amax_c[u], red[(jb * spb + k) * D + c]);
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int w = tid + u * kThreads;
    if (w >= nb * D) continue;
    const int jb = w / D, c = w % D;
    const int rs = jb * blk, re = min(rs + blk, nrows);
    red[w] = amax_c[u];
    if (re > rs) {
      const int gb = (r0 >> lb) + jb;
      const double mean = s[u] / (double)(re - rs);
      if (which == 0) {
        a.qbar[((int64_t)bh * a.nQb + gb) * D + c] = mean;
        if (a.qvar) {
          // variance of coordinate c over the block's queries (second pass)
          double ss = 0.0;
          for (int r = rs; r < re; ++r) {
            const double dv = (double)__bfloat162float(tile[r * D + c]) - mean;
            ss += dv * dv;
          }
          a.qvar[((int64_t)bh * a.nQb + gb) * D + c] = ss / (double)(re - rs);
        }
      } else if (which == 1) {
        a.kbar[((int64_t)bh * a.nKb + gb) * D + c] = mean;
        a.kbar_b[((int64_t)bh * a.nKb + gb) * D + c] = bf16_from_double(mean);
        if (bh == 0 && c == 0) a.n_k[gb] = re - rs;
        if (a.kvar) {
          // variance of coordinate c over the block's keys (second pass over
          // the staged rows, deviations from the fp64 mean)
          double ss = 0.0;
          for (int r = rs; r < re; ++r) {
            const double dv = (double)__bfloat162float(tile[r * D + c]) - mean;
            ss += dv * dv;
          }
          a.kvar[((int64_t)bh * a.nKb + gb) * D + c] = ss / (double)(re - rs);
        }
      } else {
        a.vbar_b[((int64_t)bh * a.nKb + gb) * D + c] = bf16_from_double(mean);
      }
    }
  }
  __syncthreads();
  if (a.low == TA_LOW_NONE) return;

  uint8_t* codes = which == 0 ? a.q_codes : which == 1 ? a.k_codes : a.v_codes;

  if (a.low == TA_LOW_FP8_E4M3) {
    // ---- FP8: one power-of-two scale per tile of `blk` rows ----
    if (tid < nb) {
      float amax = 0.0f;
      for (int c = 0; c < D; ++c) amax = fmaxf(amax, red[tid * D + c]);
      const float sc = fp8_pow2_scale(amax);
      tile_scale[tid] = sc;
      const int gb = (r0 >> lb) + tid;
      if (tid * blk < nrows) {
        float* scp = reinterpret_cast<float*>(which == 0 ? a.q_scales
                                              : which == 1 ? a.k_scales
                                                           : a.v_scales);
        scp[(int64_t)bh * (which == 0 ? a.nQb : a.nKb) + gb] = sc;
      }
    }
    __syncthreads();
    for (int idx = tid; idx < R * (D / 16); idx += kThreads) {
      const int r = idx / (D / 16), g = idx % (D / 16);
      if (r >= nrows) continue;
      const float sc = tile_scale[r >> lb];
      const float inv = 1.0f / sc;  // exact: sc is a power of two
      const __nv_bfloat16* px = tile + r * D + g * 16;
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t c2 = cvt_e4m3x2(__bfloat162float(px[2 * i]) * inv,
                                       __bfloat162float(px[2 * i + 1]) * inv);
        if (i & 1)
          w[i >> 1] |= c2 << 16;
        else
          w[i >> 1] = c2;
      }
      *reinterpret_cast<uint4*>(codes + (bhN + r0 + r) * D + g * 16) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    // ---- NVFP4 (+ residual) ----
    const bool res = (a.low == TA_LOW_NVFP4_RES);
    uint8_t* rcodes = which == 0 ? a.rq_codes : which == 1 ? a.rk_codes : a.rv_codes;
    uint8_t* scales = reinterpret_cast<uint8_t*>(which == 0 ? a.q_scales
                                                 : which == 1 ? a.k_scales
                                                              : a.v_scales);
    uint8_t* rscales = which == 0 ? a.rq_scales : which == 1 ? a.rk_scales : a.rv_scales;
    if (which < 2) {
      // groups of 16 along d; codes [BH, N, D/2], scales [BH, N, D/16]
      for (int idx = tid; idx < R * (D / 16); idx += kThreads) {
        const int r = idx / (D / 16), g = idx % (D / 16);
        if (r >= nrows) continue;
        const uint4* pv = reinterpret_cast<const uint4*>(tile + r * D + g * 16);
        float x[16];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const uint4 q = pv[v];
          const uint32_t ws[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x[v * 8 + e * 2] = bf_lo(ws[e]);
            x[v * 8 + e * 2 + 1] = bf_hi(ws[e]);
          }
        }
        uint32_t pk[2];
        const uint32_t scc = nvfp4_group(x, pk, sc_tab);
        const int64_t row = bhN + r0 + r;
        *reinterpret_cast<uint2*>(codes + row * (D / 2) + g * 8) = make_uint2(pk[0], pk[1]);
        scales[row * (D / 16) + g] = (uint8_t)scc;
        if (res) {
          float rr[16];
          nvfp4_residual(x, pk, sc_tab[scc].x, rr);
          const uint32_t scc2 = nvfp4_group(rr, pk, sc_tab);
          *reinterpret_cast<uint2*>(rcodes + row * (D / 2) + g * 8) = make_uint2(pk[0], pk[1]);
          rscales[row * (D / 16) + g] = (uint8_t)scc2;
        }
      }
    } else {
      // V: groups of 16 tokens per column; codes [BH, D, Np/2] (transposed),
      // scales [BH, Np/16, D].  A thread takes two adjacent columns of one
      // group (a warp reads 128 contiguous bytes of a staged row per token);
      // the codes go to shared memory group-major and leave 64 bytes per
      // column.  Groups past N come out as zero codes with a zero scale, up to
      // the pitch Np.
      for (int idx = tid; idx < L::CP * L::G; idx += kThreads) {
        const int cp = idx % L::CP, g = idx / L::CP;
        if (r0 + g * 16 >= a.Np) continue;
        float x0[16], x1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t w = tile32[(g * 16 + i) * L::CP + cp];
          x0[i] = bf_lo(w);
          x1[i] = bf_hi(w);
        }
        uint32_t p0[2], p1[2];
        const uint32_t s0 = nvfp4_group(x0, p0, sc_tab);
        const uint32_t s1 = nvfp4_group(x1, p1, sc_tab);
        const int64_t srow = ((int64_t)bh * (a.Np / 16) + (r0 + g * 16) / 16) * D + 2 * cp;
        *reinterpret_cast<uint4*>(vst + g * L::VP + 2 * cp) = make_uint4(p0[0], p0[1], p1[0], p1[1]);
        *reinterpret_cast<uint16_t*>(scales + srow) = (uint16_t)(s0 | (s1 << 8));
        if (res) {
          float rr[16];
          nvfp4_residual(x0, p0, sc_tab[s0].x, rr);
          const uint32_t t0 = nvfp4_group(rr, p0, sc_tab);
          nvfp4_residual(x1, p1, sc_tab[s1].x, rr);
          const uint32_t t1 = nvfp4_group(rr, p1, sc_tab);
          *reinterpret_cast<uint4*>(vst + (L::G + g) * L::VP + 2 * cp) =
              make_uint4(p0[0], p0[1], p1[0], p1[1]);
          *reinterpret_cast<uint16_t*>(rscales + srow) = (uint16_t)(t0 | (t1 << 8));
        }
      }
      __syncthreads();
      const int gv = min(L::G, (a.Np - r0) / 16);   // groups below the pitch
      const int copies = res ? 2 : 1;
      // 8 bytes (group g of column c) of one copy's codes
      auto put = [&](int copy, int c, int g) {
        uint8_t* dst = (copy ? rcodes : codes) + ((int64_t)bh * D + c) * (a.Np / 2) + r0 / 2 + g * 8;
        *reinterpret_cast<uint2*>(dst) = vst[(copy * L::G + g) * L::VP + c];
      };
      if (gv == L::G) {
        // every chunk but the sequence's last: compile-time index arithmetic
        for (int idx = tid; idx < copies * D * L::G; idx += kThreads)
          put(idx / (D * L::G), (idx / L::G) % D, idx % L::G);
      } else {
        for (int idx = tid; idx < copies * D * gv; idx += kThreads) {
          const int copy = idx / (D * gv), rem = idx % (D * gv);
          put(copy, rem / gv, rem % gv);
        }
      }
    }
  }
}

template <int D, int R>
cudaError_t launch_prep_dr(const PlanArgs& a, cudaStream_t s) {
  using L = PrepSmem<D, R>;
  const int chunks = (a.N + R - 1) / R;
  auto k = prep_kernel<D, R>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(chunks, a.B * a.H, 3);
  k<<<grid, kThreads, L::kBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prep(const PlanArgs& a, cudaStream_t s) {
  // R = max(bq, bk), which the parameter check keeps to 64 or 128
  if (a.d == 64) return a.R == 64 ? launch_prep_dr<64, 64>(a, s) : launch_prep_dr<64, 128>(a, s);
  return a.R == 64 ? launch_prep_dr<128, 64>(a, s) : launch_prep_dr<128, 128>(a, s);
}

}  // namespace ta
