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
//     fp32(x - dequant(x)) the same way;
//   * for an FP8 low tier that the attention kernel runs on bf16 images (d =
//     64 or 64-row tiles), the dequantised values in bf16 (exact: at most 4
//     significant bits), row-major like the input.
// One CTA per (chunk of R = max(bq, bk) tokens, head, operand Q / K / V); the
// chunk is staged in shared memory with 16-byte coalesced loads and written
// back coalesced.
#include "ta_common.cuh"
#include "ta_kernels.cuh"

namespace ta {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Smallest power of two s with amax <= 448 s (1 when amax == 0).
__device__ __forceinline__ float fp8_pow2_scale(float amax) {
  if (amax == 0.0f) return 1.0f;
  int e;
  const float m = frexpf(amax, &e);  // amax = m * 2^e, m in [0.5, 1); 448 = 0.875 * 2^9
  const int k = (m <= 0.875f) ? e - 9 : e - 8;
  return ldexpf(1.0f, k);
}

// NVFP4 of one group of 16 values: packed codes (element 2i in the low nibble
// of byte i) and the ue4m3 scale code; the scale value comes back in `sc`.
// `inv_tab[c]` is the correctly rounded reciprocal of ue4m3 code c's value.
__device__ __forceinline__ void nvfp4_group(const float (&x)[16], uint32_t (&packed)[2],
                                            uint32_t& sc_code, float& sc, const float* inv_tab) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  sc_code = cvt_e4m3x2(div6(amax), 0.0f) & 0xFFu;
  sc = e4m3_to_float(sc_code);
  packed[0] = packed[1] = 0u;
  if (sc == 0.0f) return;
  const float inv = inv_tab[sc_code];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = cvt_e2m1x2(__fmul_rn(x[2 * i], inv), __fmul_rn(x[2 * i + 1], inv));
    packed[i >> 2] |= c << (8 * (i & 3));
  }
}

// The values a packed group stands for: code value times the scale (exact in
// fp32: at most 3 + 4 significant bits).
__device__ __forceinline__ void nvfp4_dequant(const uint32_t (&packed)[2], float sc,
                                              float (&deq)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = (packed[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    deq[2 * i] = e2m1_value(c & 0xFu) * sc;
    deq[2 * i + 1] = e2m1_value(c >> 4) * sc;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 3) prep_kernel(const PlanArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int LD = D + 8;  // padded row stride (elements)
  const int R = a.R;
  __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* rtile = tile + R * LD;  // staging of the transposed NVFP4 V codes
  float* red = reinterpret_cast<float*>(rtile + R * LD);
  float* tile_scale = red + kThreads;

  __shared__ float inv_tab[128];   // ue4m3 code -> correctly rounded 1 / value
  const int tid = threadIdx.x;
  if (tid < 128) {
    const float v = (tid == 0x7F) ? 0.0f : e4m3_to_float(tid);
    inv_tab[tid] = v > 0.0f ? __frcp_rn(v) : 0.0f;
  }
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int r0 = blockIdx.x * R;
  const int nrows = min(R, a.N - r0);
  const int64_t in_off = (int64_t)b * a.sb + (int64_t)h * a.sh;
  const int64_t bhN = (int64_t)bh * a.N;
  double* psum = reinterpret_cast<double*>(tile_scale + 8);   // [kThreads] partial block sums

  {
    const int which = blockIdx.z;
    const __nv_bfloat16* src = (which == 0 ? a.Q : which == 1 ? a.K : a.V) + in_off;
    // ---- stage the chunk (rows past N read as zero) ----
    for (int idx = tid; idx < R * (D / 8); idx += kThreads) {
      const int r = idx / (D / 8), c8 = idx % (D / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nrows) v = *reinterpret_cast<const uint4*>(src + (int64_t)(r0 + r) * a.sn + c8 * 8);
      *reinterpret_cast<uint4*>(tile + r * LD + c8 * 8) = v;
    }
    __syncthreads();

    // ---- block sums (fp64: exact for bf16 inputs, so the order of the
    // additions does not matter) and per-column amax; kSeg threads share a
    // (block, column) and each sums a run of its rows ----
    const int blk = (which == 0) ? a.bq : a.bk;
    const int nb = R / blk;
    const int kSeg = kThreads / (nb * D) > 0 ? kThreads / (nb * D) : 1;
    for (int w0 = tid; w0 < nb * D * kSeg; w0 += kThreads) {
      const int w = w0 % (nb * D), seg = w0 / (nb * D);
      const int jb = w / D, c = w % D;
      const int rs = jb * blk, re = min(rs + blk, nrows);
      const int len = (blk + kSeg - 1) / kSeg;
      const int s0 = rs + seg * len, s1 = min(s0 + len, re);
      double sum = 0.0;
      float amax = 0.0f;
      for (int r = s0; r < s1; ++r) {
        const float x = bf2f(tile[r * LD + c]);
        sum += (double)x;
        amax = fmaxf(amax, fabsf(x));
      }
      psum[w0] = sum;
      red[w0] = amax;
    }
    __syncthreads();
    // nb * D <= 256 = kThreads: one (block, column) per thread
    const bool mine = tid < nb * D;
    double s = 0.0;
    float amax_c = 0.0f;
    if (mine) {
      for (int seg = 0; seg < kSeg; ++seg) {
        s += psum[seg * nb * D + tid];
        amax_c = fmaxf(amax_c, red[seg * nb * D + tid]);
      }
    }
    __syncthreads();
    if (mine) {
      const int w = tid;
      const int jb = w / D, c = w % D;
      const int rs = jb * blk, re = min(rs + blk, nrows);
      red[w] = amax_c;
      if (re > rs) {
        const int gb = r0 / blk + jb;
        const double mean = s / (double)(re - rs);
        if (which == 0) {
          a.qbar[((int64_t)bh * a.nQb + gb) * D + c] = mean;
          if (a.qvar) {
            // variance of coordinate c over the block's queries (second pass)
            double ss = 0.0;
            for (int r = rs; r < re; ++r) {
              const double dv = (double)bf2f(tile[r * LD + c]) - mean;
              ss += dv * dv;
            }
            a.qvar[((int64_t)bh * a.nQb + gb) * D + c] = ss / (double)(re - rs);
          }
        } else if (which == 1) {
          a.kbar[((int64_t)bh * a.nKb + gb) * D + c] = mean;
          a.kbar_b[((int64_t)bh * a.nKb + gb) * D + c] = bf16_from_double(mean);
          if (bh == 0 && c == 0) a.n_k[gb] = re - rs;
          if (a.kvar) {
            // variance of coordinate c over the block's keys (second pass
            // over the staged rows, deviations from the fp64 mean)
            double ss = 0.0;
            for (int r = rs; r < re; ++r) {
              const double dv = (double)bf2f(tile[r * LD + c]) - mean;
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
    __nv_bfloat16* deq_out = which == 0 ? a.dq : which == 1 ? a.dk : a.dv;

    if (a.low == TA_LOW_FP8_E4M3) {
      // ---- FP8: one power-of-two scale per tile of `blk` rows ----
      if (tid < nb) {
        float amax = 0.0f;
        for (int c = 0; c < D; ++c) amax = fmaxf(amax, red[tid * D + c]);
        const float s = fp8_pow2_scale(amax);
        tile_scale[tid] = s;
        const int gb = r0 / blk + tid;
        if (tid * blk < nrows) {
          float* sc = reinterpret_cast<float*>(which == 0 ? a.q_scales
                                               : which == 1 ? a.k_scales
                                                            : a.v_scales);
          sc[(int64_t)bh * (which == 0 ? a.nQb : a.nKb) + gb] = s;
        }
      }
      __syncthreads();
      for (int idx = tid; idx < R * (D / 16); idx += kThreads) {
        const int r = idx / (D / 16), g = idx % (D / 16);
        if (r >= nrows) continue;
        const float s = tile_scale[r / blk];
        const float inv = 1.0f / s;  // exact: s is a power of two
        __nv_bfloat16* px = tile + r * LD + g * 16;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t c2 = cvt_e4m3x2(bf2f(px[2 * i]) * inv, bf2f(px[2 * i + 1]) * inv);
          if (i & 1)
            w[i >> 1] |= c2 << 16;
          else
            w[i >> 1] = c2;
          const float2 f = e4m3x2_to_float2(c2);
          px[2 * i] = __float2bfloat16_rn(f.x * s);
          px[2 * i + 1] = __float2bfloat16_rn(f.y * s);
        }
        *reinterpret_cast<uint4*>(codes + (bhN + r0 + r) * D + g * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      // ---- NVFP4 (+ residual); no bf16 images of these copies are kept ----
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
          const uint4* pv = reinterpret_cast<const uint4*>(tile + r * LD + g * 16);
          float x[16], dqv[16], sc;
          uint32_t pk[2], scc;
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const uint4 w = pv[v];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              x[v * 8 + e * 2] = __uint_as_float(ws[e] << 16);
              x[v * 8 + e * 2 + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
            }
          }
          nvfp4_group(x, pk, scc, sc, inv_tab);
          const int64_t row = bhN + r0 + r;
          *reinterpret_cast<uint2*>(codes + row * (D / 2) + g * 8) = make_uint2(pk[0], pk[1]);
          scales[row * (D / 16) + g] = (uint8_t)scc;
          if (res) {
            float rr[16], rsc;
            nvfp4_dequant(pk, sc, dqv);
#pragma unroll
            for (int i = 0; i < 16; ++i) rr[i] = __fsub_rn(x[i], dqv[i]);
            nvfp4_group(rr, pk, scc, rsc, inv_tab);
            *reinterpret_cast<uint2*>(rcodes + row * (D / 2) + g * 8) = make_uint2(pk[0], pk[1]);
            rscales[row * (D / 16) + g] = (uint8_t)scc;
          }
        }
      } else {
        // V: groups of 16 tokens per column; codes [BH, D, Np/2] (transposed),
        // scales [BH, Np/16, D].  Threads walk the columns fastest, so that a
        // warp reads one 64-byte run of a staged row at a time (no bank
        // conflicts); the codes go column-major to shared memory (the residual
        // tile area, unused here; group-major with a padded row of D + 1, so
        // that both the writes here and the reads below avoid bank conflicts)
        // and leave 64 bytes per column.  Groups past
        // N come out as zero codes with a zero scale, up to the pitch Np.
        const int G = R / 16;
        uint2* vst = reinterpret_cast<uint2*>(rtile);   // [copy][G][D + 1]
        for (int idx = tid; idx < D * G; idx += kThreads) {
          const int c = idx % D, g = idx / D;
          if (r0 + g * 16 >= a.Np) continue;
          float x[16], dqv[16], sc;
          uint32_t pk[2], scc;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int r = g * 16 + i;
            x[i] = (r < nrows) ? bf2f(tile[r * LD + c]) : 0.0f;
          }
          nvfp4_group(x, pk, scc, sc, inv_tab);
          const int64_t tok = r0 + g * 16;
          vst[g * (D + 1) + c] = make_uint2(pk[0], pk[1]);
          scales[((int64_t)bh * (a.Np / 16) + tok / 16) * D + c] = (uint8_t)scc;
          if (res) {
            float rr[16], rsc;
            nvfp4_dequant(pk, sc, dqv);
#pragma unroll
            for (int i = 0; i < 16; ++i) rr[i] = __fsub_rn(x[i], dqv[i]);
            nvfp4_group(rr, pk, scc, rsc, inv_tab);
            vst[(G + g) * (D + 1) + c] = make_uint2(pk[0], pk[1]);
            rscales[((int64_t)bh * (a.Np / 16) + tok / 16) * D + c] = (uint8_t)scc;
          }
        }
        __syncthreads();
        const int gv = min(G, (a.Np - r0) / 16);   // groups below the pitch
        const int copies = res ? 2 : 1;
        for (int idx = tid; idx < copies * D * gv; idx += kThreads) {
          const int copy = idx / (D * gv), rem = idx % (D * gv);
          const int c = rem / gv, g = rem % gv;
          uint8_t* dst = (copy ? rcodes : codes) + ((int64_t)bh * D + c) * (a.Np / 2) + r0 / 2 + g * 8;
          *reinterpret_cast<uint2*>(dst) = vst[(copy * G + g) * (D + 1) + c];
        }
      }
    }
    __syncthreads();
    // ---- dequantised copy, coalesced (only where a tile path reads it) ----
    if (deq_out != nullptr)
    for (int idx = tid; idx < R * (D / 8); idx += kThreads) {
      const int r = idx / (D / 8), c8 = idx % (D / 8);
      if (r < nrows)
        *reinterpret_cast<uint4*>(deq_out + (bhN + r0 + r) * D + c8 * 8) =
            *reinterpret_cast<const uint4*>(tile + r * LD + c8 * 8);
    }
    __syncthreads();
  }
}

template <int D>
cudaError_t launch_prep_d(const PlanArgs& a, cudaStream_t s) {
  const int chunks = (a.N + a.R - 1) / a.R;
  const size_t smem = (size_t)2 * a.R * (D + 8) * sizeof(__nv_bfloat16) +
                      (size_t)(kThreads + 8) * sizeof(float) + (size_t)kThreads * sizeof(double);
  auto k = prep_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(chunks, a.B * a.H, 3);
  k<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prep(const PlanArgs& a, cudaStream_t s) {
  if (a.d == 64) return launch_prep_d<64>(a, s);
  return launch_prep_d<128>(a, s);
}

}  // namespace ta
