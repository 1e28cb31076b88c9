// ta_attn.cu -- the fused one-pass tiered attention kernel (sm_100a).
//
// "Triage" (zhuanzhiai paper page, abstract) runs all tiers of a query block
// in a single fused pass: full tiles in bf16, low tiles in reduced precision,
// and skipped tiles replaced by their block means, so that block j of n_j keys
// adds n_j exp(q . kbar_j * scale) to the softmax denominator and that weight
// times vbar_j to the numerator.  One CTA owns one (head, query block) and
// walks the block's compacted tile list (full tiles, then low tiles, each by
// descending pooled mass, then the skipped blocks) with an online softmax:
//
//   warps 4S, 4S+1  producers of K and of V: TMA loads of the kept tiles
//               (bf16, or the low copies) into two two-stage rings; a K stage
//               is released as soon as its S = Q K^T is done, a V stage after
//               its PV.  For skipped blocks they gather up to BK pooled rows
//               kbar_b / vbar_b into a "pseudo-key" tile, so a skip chunk costs
//               one tile of MMA for up to BK skipped blocks and never touches
//               their K / V;
//   warp 4S+2   S issuer: S = Q K^T into a double-buffered TMEM accumulator,
//               as soon as the softmax has read the buffer's previous S;
//   warp 4S+3   PV issuer: O += P V into a TMEM accumulator.  One thread each
//               issues tcgen05.mma: kind::f16 for full and skip tiles;
//               kind::mxf4nvf4.block16 for NVFP4 tiles (ue4m3 scales copied
//               to TMEM with tcgen05.cp; three MMAs per product on residual
//               tiles); kind::f8f6f4 for FP8 S and kind::mxf8f6f4 for FP8 PV
//               (V's power-of-two tile scale as a UE8M0 block scale; d = 64
//               or 64-key tiles use 64-byte-swizzled FP8 rows).  Two
//               threads, because one thread issues an N <= 128 MMA only every
//               ~100 cycles.  Completion is signalled with tcgen05.commit on
//               mbarriers;
//   warps 0..4S-1 softmax (S = min(d, BK)/32 column parts): the S warps with
//               equal w%4 share TMEM lanes 32(w%4).. (query rows) and split
//               each row's columns into S parts of 32; they swap their part
//               maxima through shared memory and a named barrier.  Each thread
//               loads its part of an S row, keeps the running max m and its
//               part of the sum l, and hands the rest of the tile to a tail
//               specialised for the tile's P format: P' = 2^o exp(s - m'),
//               rounded as the tier demands (bf16; e4m3; NVFP4 per 16 keys,
//               plus its residual), O rescaled in TMEM when m grew, and P'
//               handed to the PV MMA: bf16 P' is stored into TMEM columns of
//               its own (the A operand of a TMEM x shared-memory MMA), NVFP4 /
//               FP8 P' into one of two shared-memory buffers.
//               The epilogue writes O = acc / l in bf16.
//
// All waits are bounded: a wait that runs out sets the CTA's abort flag and
// the workspace status word, every role leaves its loop, in-flight copies and
// MMAs are drained (bounded), and TMEM is freed before return.
#include "ta_common.cuh"
#include "ta_kernels.cuh"
#include "ta_attn_common.cuh"

namespace ta {
namespace {

using namespace tile;

// Softmax warps: warp w owns TMEM lanes 32*(w%4).. (query rows) and column
// part w/4 of those rows; kSplit parts per row (32 columns of S and of O each).
template <int D, int BK>
struct Roles {
  static constexpr int kSplit = (D < BK ? D : BK) / 32;
  static constexpr int kSoftmaxWarps = 4 * kSplit;
  static constexpr int kProducerKWarp = kSoftmaxWarps;      // Q and K tiles
  static constexpr int kProducerVWarp = kSoftmaxWarps + 1;  // V tiles
  static constexpr int kMmaWarp = kSoftmaxWarps + 2;        // S = Q K^T issuer
  static constexpr int kPvWarp = kSoftmaxWarps + 3;         // O += P V issuer
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 4);
};

// Named barrier over `count` threads that also ANDs a predicate across them:
// the warps of a softmax pair leave their loop together or not at all.
__device__ __forceinline__ bool bar_and(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}

// Shared-memory layout (offsets from a 1024-aligned base).
template <int D, int BK, int LM>
struct Smem {
  static constexpr bool FP4 = (LM == LM_NVFP4 || LM == LM_NVFP4_RES);
  static constexpr bool RES = (LM == LM_NVFP4_RES);
  static constexpr bool F8 = (LM == LM_FP8);
  static constexpr int NC = RES ? 2 : 1;      // NVFP4 copies per operand
  static constexpr int kQ = 128 * D * 2;      // one query tile, 128 rows
  static constexpr int kKV = BK * D * 2;      // one K or V tile
  static constexpr int kPfp4 = 128 * 64 + 1024;  // one NVFP4 tile: codes + scales
  static constexpr int kF8 = 128 * 128;                // an FP8 Q or P buffer (128 rows x up to 128 B)
  static constexpr int kF8KV = BK * D;                 // an FP8 K or V tile; V's scales follow it
  static constexpr int kQlow = FP4 ? NC * kPfp4 : (F8 ? kF8 : kQ);  // low query copies
  // P: bf16 P lives in TMEM; NVFP4 / FP8 P in two shared-memory buffers
  static constexpr int kP = FP4 ? 2 * NC * kPfp4 : (F8 ? 2 * kF8 + 1024 : 0);
  static constexpr int oQ = 0;
  static constexpr int oDQ = oQ + kQ;
  static constexpr int oK0 = oDQ + kQlow;
  static constexpr int oV0 = oK0 + kKV;
  static constexpr int oK1 = oV0 + kKV;
  static constexpr int oV1 = oK1 + kKV;
  static constexpr int oP = oV1 + kKV;
  static constexpr int oBar = oP + kP;
  static constexpr int kBars = 24;
  static constexpr int oMisc = oBar + kBars * 8;
  static constexpr int oXchg = oMisc + 64;           // float [2 slots][4 parts][128 rows]
  static constexpr int oScTab = oXchg + 2 * 4 * 128 * 4;  // float2 [128]: ue4m3 value, 1/value
  static constexpr int kTotal = oScTab + 128 * 8;
  static constexpr int kAlloc = kTotal;  // the base is checked for 1024-byte alignment
};

// mbarriers; pairs are indexed by the parity of the tile
//   S   S of the tile is in TMEM (S issuer)      SC  the softmax has read that S
//   P   the tile's P is written (softmax)        PD  the tile's PV is done (PV issuer)
enum {
  BAR_Q = 0, BAR_K0 = 1, BAR_K1 = 2, BAR_V0 = 3, BAR_V1 = 4, BAR_KE0 = 5, BAR_KE1 = 6,
  BAR_S0 = 7, BAR_S1 = 8, BAR_P0 = 9, BAR_P1 = 10, BAR_PD0 = 11, BAR_PD1 = 12,
  BAR_DRAIN_S = 13, BAR_DRAIN_PV = 14, BAR_VE0 = 15, BAR_VE1 = 16, BAR_SC0 = 17, BAR_SC1 = 18
};

// Formats of P' in the softmax's tile tail.
enum { PK_BF16 = 0, PK_SKIP = 1, PK_FP4 = 2, PK_RES = 3, PK_F8 = 4 };

// What the tail of one tile's softmax needs (one thread: one query row, one
// column part of HB keys).
struct SoftmaxTail {
  float* x;                 // the part's S values (masked to -inf past nv)
  int nv;                   // valid columns of this part
  float c2t, mc;            // P' = 2^(s * c2t - mc)
  float alpha;              // exp(m - m') of this row
  int t;                    // tile index in the row
  const int* list;          // list entries of this part's columns
  int N;
  uint64_t* bars;
  AbortCtx ctx;
  int row_bar;
  unsigned char* sm;
  uint32_t tP, tO;          // this lane's bf16 P columns and O accumulator
  int part, quarter, lane, r;
  const float2* sc_tab;     // ue4m3 code -> (value, 1 / value)
};

// Tail of one tile's softmax for one P format, in straight-line code:
// P' = 2^o exp(s - m') and its part row sum, P' rounded as the tier demands,
// O rescaled when the maximum grew (after the previous PV), and P' handed to
// the PV MMA (bf16 in the TMEM P columns, once the previous PV has read
// them; NVFP4 / FP8 in a shared-memory buffer, once the PV two tiles back has
// read it).  False when the CTA aborts; the warp then leaves at the row
// group's next named barrier.
template <int PK, int D, int BK, int LM>
__device__ __forceinline__ bool softmax_tail(const SoftmaxTail q, float& psum) {
  using L = Smem<D, BK, LM>;
  constexpr int kSplit = Roles<D, BK>::kSplit;
  constexpr int HB = BK / kSplit, HD = D / kSplit;
  constexpr bool smem_p = (PK == PK_FP4 || PK == PK_RES || PK == PK_F8);
  const int s = q.t & 1;
  float* x = q.x;
  {
    // arguments two at a time (packed fp32 FMA), then the exponentials
    const uint64_t c2t2 = pack2(q.c2t, q.c2t), nmc2 = pack2(-q.mc, -q.mc);
#pragma unroll
    for (int c = 0; c < HB; c += 2) {
      float a0, a1;
      unpack2(fma2(pack2(x[c], x[c + 1]), c2t2, nmc2), a0, a1);
      x[c] = fast_exp2(a0);
      x[c + 1] = fast_exp2(a1);
    }
  }
  if constexpr (PK == PK_SKIP) {
    // pooled keys weigh n_j
#pragma unroll
    for (int c = 0; c < HB; ++c) {
      if (c < q.nv) {
        const int j = q.list[c];
        x[c] *= (float)min(BK, q.N - j * BK);
      }
    }
  }
  {
    // four running sums (keys c = 0, 1, 2, 3 mod 4) as two packed pairs
    uint64_t sa = pack2(0.0f, 0.0f), sb = pack2(0.0f, 0.0f);
#pragma unroll
    for (int c = 0; c < HB; c += 4) {
      sa = add2(sa, pack2(x[c], x[c + 1]));
      sb = add2(sb, pack2(x[c + 2], x[c + 3]));
    }
    float s0, s1, s2, s3;
    unpack2(sa, s0, s1);
    unpack2(sb, s2, s3);
    psum = (s0 + s1) + (s2 + s3);
  }

  // round P' as the tier demands
  uint32_t p[(PK == PK_RES) ? 13 : (HB / 2)];
  if constexpr (PK == PK_FP4 || PK == PK_RES) {
    // codes of this part (HB = 32 keys, half an MMA K chunk) in p[0..3], its
    // two ue4m3 scales in p[4]; the residual copy in p[8..12]
    static_assert(HB == 32, "NVFP4 parts are 32 keys");
    p[4] = nvfp4_quant32(x, q.sc_tab, p);
    if constexpr (PK == PK_RES) p[12] = nvfp4_residual32(x, p, p[4], q.sc_tab, p + 8);
  } else if constexpr (PK == PK_F8) {
    // e4m3 codes of P' (scale 1), four per word
#pragma unroll
    for (int c = 0; c < HB; c += 4)
      p[c / 4] = cvt_e4m3x2(x[c], x[c + 1]) | (cvt_e4m3x2(x[c + 2], x[c + 3]) << 16);
  } else {
#pragma unroll
    for (int c = 0; c < HB; c += 2) p[c / 2] = pack_bf16(x[c], x[c + 1]);
  }

  // O may be rescaled, and the TMEM P columns rewritten, only once the
  // previous tile's PV is done; a shared-memory P buffer may be rewritten
  // once the PV two tiles back is done.  Each warp decides and waits for
  // itself (it rescales and writes only its own columns).
  const bool rescale = (q.t > 0) && __any_sync(0xffffffffu, q.alpha != 1.0f);
  const bool prev = (q.t > 0) && (rescale || !smem_p);
  const bool reuse = smem_p && q.t >= 2;
  if (prev || reuse) {
    bool ok2 = true;
    if (reuse) ok2 = mbar_wait(&q.bars[BAR_PD0 + s], ((q.t >> 1) - 1) & 1, q.ctx, 7);
    if (prev && ok2) ok2 = mbar_wait(&q.bars[BAR_PD0 + (s ^ 1)], ((q.t - 1) >> 1) & 1, q.ctx, 9);
    if (!__all_sync(0xffffffffu, ok2)) return false;
  }
  if (rescale) {
    tc_fence_after();
#pragma unroll
    for (int c0 = 0; c0 < HD; c0 += 32) {
      uint32_t raw[32];
      tmem_ld32(q.tO + q.part * HD + c0, raw);
      const uint64_t al2 = pack2(q.alpha, q.alpha);
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float o0, o1;
        unpack2(mul2(pack2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), al2), o0, o1);
        raw[c] = __float_as_uint(o0);
        raw[c + 1] = __float_as_uint(o1);
      }
      tmem_st32(q.tO + q.part * HD + c0, raw);
    }
  }
  if constexpr (PK == PK_FP4 || PK == PK_RES) {
    // NVFP4 P part: 16 bytes of codes into the 64-byte-swizzled tile, 2
    // scale bytes into the scale-factor block of K chunk part/2 (and the same
    // for the residual copy on residual tiles)
    unsigned char* pbuf = q.sm + L::oP + s * L::NC * L::kPfp4;
    const uint32_t off = q.r * 64 + ((q.part ^ ((q.r >> 1) & 3)) * 16);
    const uint32_t soff = kFp4Sf + (q.part >> 1) * 512 + q.lane * 16 + q.quarter * 4 + (q.part & 1) * 2;
    *reinterpret_cast<uint4*>(pbuf + off) = make_uint4(p[0], p[1], p[2], p[3]);
    *reinterpret_cast<uint16_t*>(pbuf + soff) = (uint16_t)p[4];
    if constexpr (PK == PK_RES) {
      *reinterpret_cast<uint4*>(pbuf + L::kPfp4 + off) = make_uint4(p[8], p[9], p[10], p[11]);
      *reinterpret_cast<uint16_t*>(pbuf + L::kPfp4 + soff) = (uint16_t)p[12];
    }
  } else if constexpr (PK == PK_F8) {
    // FP8 P part: HB codes into the tile of buffer s, rows of BK bytes,
    // 128-byte swizzle (BK = 128) or 64-byte swizzle (BK = 64)
    unsigned char* pbuf = q.sm + L::oP + s * L::kF8;
#pragma unroll
    for (int h = 0; h < HB / 16; ++h) {
      const int ch = q.part * (HB / 16) + h;
      const uint32_t off = (BK == 128) ? q.r * 128 + ((ch ^ (q.r & 7)) * 16)
                                       : q.r * 64 + ((ch ^ ((q.r >> 1) & 3)) * 16);
      *reinterpret_cast<uint4*>(pbuf + off) = make_uint4(p[h * 4 + 0], p[h * 4 + 1], p[h * 4 + 2], p[h * 4 + 3]);
    }
  } else {
    // bf16 P' of this part into the TMEM P columns
#pragma unroll
    for (int h = 0; h < HB / 2; h += 16) tmem_st16(q.tP + q.part * (HB / 2) + h, p + h);
  }
  if constexpr (smem_p) fence_proxy_async_smem();
  tmem_wait_st();
  tc_fence_before();
  mbar_arrive(&q.bars[BAR_P0 + s]);
  return true;
}

template <int D, int BK, int LM>
__global__ void __launch_bounds__(Roles<D, BK>::kThreads, 1)
    attn_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tmQ,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                const __grid_constant__ CUtensorMap tmDV, const __grid_constant__ CUtensorMap tmRQ,
                const __grid_constant__ CUtensorMap tmRK, const __grid_constant__ CUtensorMap tmRV) {
  using L = Smem<D, BK, LM>;
  constexpr bool FP4 = L::FP4, RES = L::RES, F8 = L::F8;
  using TS = TmemMap<D, BK, LM>;
  using RL = Roles<D, BK>;
  constexpr int kSplit = RL::kSplit, kSoftmaxWarps = RL::kSoftmaxWarps;
  constexpr int kProducerKWarp = RL::kProducerKWarp, kProducerVWarp = RL::kProducerVWarp;
  constexpr int kMmaWarp = RL::kMmaWarp, kPvWarp = RL::kPvWarp;
  static_assert(!FP4 || (D == 128 && BK == 128), "native NVFP4 tiles need d = 128, 128-key tiles");
  constexpr uint32_t kTmemCols = TS::kCols;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw;
  if (smem_u32(sm) & 1023u) {
    // the 128-byte-swizzled tiles need a 1024-byte-aligned base: refuse cleanly
    if (threadIdx.x == 0 && a.status) atomicCAS(a.status + ST_CODE, 0, (int)TA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::oBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::oMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::oMisc + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qb = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int q0 = qb * a.bq;
  const int64_t row_id = (int64_t)bh * a.nQb + qb;

  RowPlan rp;
  rp.n_full = a.row_counts[row_id * 4 + 0];
  rp.n_res = a.row_counts[row_id * 4 + 1];
  rp.n_low = a.row_counts[row_id * 4 + 2];
  rp.n_skip = a.row_counts[row_id * 4 + 3];
  rp.list = a.row_lists + row_id * a.nKb;
  rp.T = rp.n_full + rp.n_res + rp.n_low + (rp.n_skip + BK - 1) / BK;
  const bool has_low = rp.n_low > 0 || rp.n_res > 0;  // tiles reading the first low copy
  const int nq = rp.n_res > 0 ? 2 : (has_low ? 1 : 0);  // NVFP4 query copies to load

  AbortCtx ctx{abort_flag, a.status};

  // ---- set-up: barriers, zero padding rows, TMEM ----
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bars[BAR_Q], 1);
    mbar_init(&bars[BAR_K0], 1);
    mbar_init(&bars[BAR_K1], 1);
    mbar_init(&bars[BAR_V0], 1);
    mbar_init(&bars[BAR_V1], 1);
    mbar_init(&bars[BAR_KE0], 1);
    mbar_init(&bars[BAR_KE1], 1);
    mbar_init(&bars[BAR_VE0], 1);
    mbar_init(&bars[BAR_VE1], 1);
    mbar_init(&bars[BAR_S0], 1);
    mbar_init(&bars[BAR_S1], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[BAR_P0 + i], kSplit * a.bq);   // every column part of every live row
      mbar_init(&bars[BAR_SC0 + i], kSplit * a.bq);
    }
    mbar_init(&bars[BAR_PD0], 1);
    mbar_init(&bars[BAR_PD1], 1);
    mbar_init(&bars[BAR_DRAIN_S], 1);
    mbar_init(&bars[BAR_DRAIN_PV], 1);
    fence_mbar_init();
  }
  if (F8 && threadIdx.x < 128) {
    // UE8M0 scale factors of the FP8 P operand: all 2^0
    *reinterpret_cast<uint32_t*>(sm + L::oP + 2 * L::kF8 + threadIdx.x * 4) = 0x7F7F7F7Fu;
    fence_proxy_async_smem();
  }
  if (FP4 && threadIdx.x < 128) {
    // ue4m3 code -> (value, correctly rounded reciprocal) for P' quantisation
    const float v = (threadIdx.x == 0x7F) ? 0.0f : e4m3_to_float(threadIdx.x);
    reinterpret_cast<float2*>(sm + L::oScTab)[threadIdx.x] =
        make_float2(v, v > 0.0f ? __frcp_rn(v) : 0.0f);
  }
  if (warp < 4) {
    // Rows >= bq of the query tiles stay zero for the whole kernel.
    const int r = threadIdx.x;
    if (r >= a.bq) {
      for (int c = 0; c < (D * 2) / 16; ++c) {
        const int box = c / 8, ch = c % 8;
        const uint32_t off = box * (128 * 128) + r * 128 + ((ch ^ (r & 7)) * 16);
        *reinterpret_cast<uint4*>(sm + L::oQ + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sm + L::oDQ + off) = make_uint4(0, 0, 0, 0);
      }
      // (rows >= bq of S are exact zeros; rows >= bq of P and O are never
      // read back: a product's row depends on its own row of P only)
      fence_proxy_async_smem();
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem + TS::kS0, tS1 = tmem + TS::kS1, tO = tmem + TS::kO;
  const uint32_t tP = tmem + TS::kP;

  bool aborted = false;

  if (warp == kProducerKWarp || warp == kProducerVWarp) {
    // ===================== producers (K ring / V ring) =====================
    const bool isK = (warp == kProducerKWarp);
    int issued[2] = {0, 0};   // loads (or gathers) signalled per stage barrier
    uint64_t* full = &bars[isK ? BAR_K0 : BAR_V0];
    uint64_t* empty = &bars[isK ? BAR_KE0 : BAR_VE0];
    if (isK) {
      if (FP4 && nq > 0) {
        // scales of the NVFP4 query copies, ready for tcgen05.cp
        for (int c = 0; c < nq; ++c)
          gather_row_sf(sm + L::oDQ + c * L::kPfp4 + kFp4Sf,
                        (c ? a.rq_sf : a.q_sf) + ((int64_t)bh * a.N + q0) * 8, min(128, a.N - q0),
                        lane);
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        const uint32_t qbytes = (uint32_t)a.bq * D * 2;
        const uint32_t lbytes = FP4 ? (uint32_t)(nq * a.bq * 64)
                                : (has_low ? (F8 ? (uint32_t)a.bq * D : qbytes) : 0u);
        mbar_arrive_expect_tx(&bars[BAR_Q], qbytes + lbytes);
        for (int x = 0; x < D / 64; ++x)
          tma_load_4d(sm + L::oQ + x * (128 * 128), &tmQ, &bars[BAR_Q], x * 64, q0, h, b);
        if (has_low) {
          if (FP4) {
            tma_load_3d(sm + L::oDQ, &tmDQ, &bars[BAR_Q], 0, q0, bh);
            if (nq > 1) tma_load_3d(sm + L::oDQ + L::kPfp4, &tmRQ, &bars[BAR_Q], 0, q0, bh);
          } else if (F8) {
            tma_load_3d(sm + L::oDQ, &tmDQ, &bars[BAR_Q], 0, q0, bh);
          } else {
            for (int x = 0; x < D / 64; ++x)
              tma_load_4d(sm + L::oDQ + x * (128 * 128), &tmDQ, &bars[BAR_Q], x * 64, q0, h, b);
          }
        }
      }
    } else if (lane == 0) {
      tma_prefetch_desc(&tmV);
    }
    // pooled rows for skip chunks: kbar_b for the K ring, vbar_b for the V ring
    const __nv_bfloat16* pooled = (isK ? a.kbar_b : a.vbar_b) + (int64_t)bh * a.nKb * D;
    for (int t = 0; t < rp.T; ++t) {
      const int s = t & 1;
      if (t >= 2) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], ((t >> 1) - 1) & 1, ctx, isK ? 1 : 10);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { aborted = true; break; }
      }
      int kind, first;
      tile_of<BK>(rp, t, kind, first);
      unsigned char* st = sm + (isK ? (s ? L::oK1 : L::oK0) : (s ? L::oV1 : L::oV0));
      if (FP4 && (kind == KIND_LOW || kind == KIND_RES)) {
        const int j = rp.list[first];
        const int ncopy = (RES && kind == KIND_RES) ? 2 : 1;   // first copy [+ residual]
        for (int c = 0; c < ncopy; ++c) {
          unsigned char* cst = st + c * L::kPfp4;
          if (isK) {
            // K scales (rows of the key tile) in the tcgen05.cp block layout
            gather_row_sf(cst + kFp4Sf, (c ? a.rk_sf : a.k_sf) + ((int64_t)bh * a.N + j * BK) * 8,
                          min(BK, a.N - j * BK), lane);
          } else {
            // V scales: groups of 16 keys of each d row of V^T
            const uint8_t* vsf = c ? a.rv_sf : a.v_sf;
            const int ng = a.Np / 16;
#pragma unroll
            for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int g = j * 8 + kc * 4 + k;   // group of 16 keys
                uint32_t w = 0u;
                if (g < ng)
                  w = *reinterpret_cast<const uint32_t*>(vsf + ((int64_t)bh * ng + g) * D + lane * 4);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int m = lane * 4 + i;        // d row of V^T
                  cst[kFp4Sf + kc * 512 + (m & 31) * 16 + (m >> 5) * 4 + k] = (unsigned char)(w >> (8 * i));
                }
              }
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const bool drop = isK && (t == 0) && (a.debug_flags & TA_DEBUG_DROP_FIRST_K);
          if (!drop) {
            mbar_arrive_expect_tx(&full[s], ncopy * (isK ? BK : D) * 64);
            for (int c = 0; c < ncopy; ++c) {
              if (isK)
                tma_load_3d(st + c * L::kPfp4, c ? &tmRK : &tmDK, &full[s], 0, j * BK, bh);
              else
                tma_load_3d(st + c * L::kPfp4, c ? &tmRV : &tmDV, &full[s], j * 64, 0, bh);
            }
            issued[s]++;
          }
        }
      } else if (F8 && kind == KIND_LOW) {
        const int j = rp.list[first];
        if (!isK) {
          // UE8M0 scale factor of this V tile: the exponent of its power-of-two scale
          const uint32_t e = (__float_as_uint(a.v_s8[(int64_t)bh * a.nKb + j]) >> 23) & 0xFFu;
          reinterpret_cast<uint32_t*>(st + L::kF8KV)[lane * 4 + 0] = e * 0x01010101u;
          reinterpret_cast<uint32_t*>(st + L::kF8KV)[lane * 4 + 1] = e * 0x01010101u;
          reinterpret_cast<uint32_t*>(st + L::kF8KV)[lane * 4 + 2] = e * 0x01010101u;
          reinterpret_cast<uint32_t*>(st + L::kF8KV)[lane * 4 + 3] = e * 0x01010101u;
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          const bool drop = isK && (t == 0) && (a.debug_flags & TA_DEBUG_DROP_FIRST_K);
          if (!drop) {
            mbar_arrive_expect_tx(&full[s], BK * D);
            tma_load_3d(st, isK ? &tmDK : &tmDV, &full[s], 0, j * BK, bh);
            issued[s]++;
          }
        }
      } else if (kind != KIND_SKIP) {
        if (lane == 0) {
          const int j = rp.list[first];
          const CUtensorMap* mp = isK ? ((kind == KIND_LOW) ? &tmDK : &tmK)
                                      : ((kind == KIND_LOW) ? &tmDV : &tmV);
          const bool drop = isK && (t == 0) && (a.debug_flags & TA_DEBUG_DROP_FIRST_K);
          if (!drop) {
            mbar_arrive_expect_tx(&full[s], BK * D * 2);
            for (int x = 0; x < D / 64; ++x)
              tma_load_4d(st + x * (BK * 128), mp, &full[s], x * 64, j * BK, h, b);
            issued[s]++;
          }
        }
      } else {
        // gather pooled rows of the skipped blocks into a pseudo K (or V)
        // tile: the chunk's list entries once (lane l holds columns l, l+32,
        // ...), then every 16-byte piece as an asynchronous copy, all in
        // flight together (zero fill past the chunk's last column)
        const int cnt = min(BK, rp.n_skip - (first - rp.n_full - rp.n_res - rp.n_low));
        constexpr int kCh = D / 8;             // 16-byte pieces per pooled row
        constexpr int kCols = 32 / kCh;        // rows per warp-wide step
        int jl[BK / 32];
#pragma unroll
        for (int i = 0; i < BK / 32; ++i) {
          const int c = lane + 32 * i;
          jl[i] = (c < cnt) ? rp.list[first + c] : 0;
        }
#pragma unroll
        for (int c0 = 0; c0 < BK; c0 += kCols) {
          const int c = c0 + lane / kCh, ch = lane % kCh;
          const int j = __shfl_sync(0xffffffffu, jl[c0 / 32], c % 32);
          const uint32_t off = (ch >> 3) * (BK * 128) + c * 128 + (((ch & 7) ^ (c & 7)) * 16);
          cp_async16(st + off, pooled + (int64_t)j * D + ch * 8, c < cnt ? 16u : 0u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full[s]);
          issued[s]++;
        }
      }
    }
    if (aborted && lane == 0) {
      // let copies already in flight land before the CTA goes away
      for (int s = 0; s < 2; ++s)
        if (issued[s] > 0) mbar_wait_drain(&full[s], (issued[s] - 1) & 1);
      if (isK) mbar_wait_drain(&bars[BAR_Q], 0);
    }
  } else if (warp == kMmaWarp) {
    // ===================== S issuer: S = Q K^T =====================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, BK, false);
      const uint32_t sQ = smem_u32(sm + L::oQ), sDQ = smem_u32(sm + L::oDQ);
      bool ok = mbar_wait(&bars[BAR_Q], 0, ctx, 3);
      if (ok) {
        tc_fence_after();
        if (FP4) {
          for (int c = 0; c < nq; ++c) {
            tc_cp_sf(tmem + TS::sfaQ(c), smem_desc_rows16(sDQ + c * L::kPfp4 + kFp4Sf));
            tc_cp_sf(tmem + TS::sfaQ(c) + 4, smem_desc_rows16(sDQ + c * L::kPfp4 + kFp4Sf + 512));
          }
        }
      }
      for (int t = 0; ok && t < rp.T; ++t) {
        const int s = t & 1;
        // the S buffer is free once the softmax has read S of tile t-2
        if (t >= 2 && !mbar_wait(&bars[BAR_SC0 + s], ((t - 2) >> 1) & 1, ctx, 10)) { ok = false; break; }
        if (!mbar_wait(&bars[BAR_K0 + s], (t >> 1) & 1, ctx, 2)) { ok = false; break; }
        tc_fence_after();
        int kind, first;
        tile_of<BK>(rp, t, kind, first);
        const uint32_t aq = (kind == KIND_LOW || kind == KIND_RES) ? sDQ : sQ;
        const uint32_t sk = smem_u32(sm + (s ? L::oK1 : L::oK0));
        const uint32_t d = s ? tS1 : tS0;
        if (FP4 && (kind == KIND_LOW || kind == KIND_RES)) {
          // NVFP4: Q1 K1 (+ Q1 K2 + Q2 K1 on residual tiles), block scales in TMEM
          const int ncopy = (RES && kind == KIND_RES) ? 2 : 1;
          for (int c = 0; c < ncopy; ++c) {
            const uint32_t sfb = tmem + TS::sfbK(c);
            tc_cp_sf(sfb, smem_desc_rows16(sk + c * L::kPfp4 + kFp4Sf));
            tc_cp_sf(sfb + 4, smem_desc_rows16(sk + c * L::kPfp4 + kFp4Sf + 512));
          }
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            mma_nvfp4_ss(d, smem_desc_sw64(aq + kk * 32), smem_desc_sw64(sk + kk * 32),
                         idesc_nvfp4(128, BK), tmem + TS::sfaQ(0) + kk * 4,
                         tmem + TS::sfbK(0) + kk * 4, kk > 0 ? 1u : 0u);
            if (RES && kind == KIND_RES) {
              mma_nvfp4_ss(d, smem_desc_sw64(aq + kk * 32), smem_desc_sw64(sk + L::kPfp4 + kk * 32),
                           idesc_nvfp4(128, BK), tmem + TS::sfaQ(0) + kk * 4,
                           tmem + TS::sfbK(1) + kk * 4, 1u);
              mma_nvfp4_ss(d, smem_desc_sw64(aq + L::kPfp4 + kk * 32), smem_desc_sw64(sk + kk * 32),
                           idesc_nvfp4(128, BK), tmem + TS::sfaQ(1) + kk * 4,
                           tmem + TS::sfbK(0) + kk * 4, 1u);
            }
          }
        } else if (F8 && kind == KIND_LOW) {
          // FP8 codes: D / 32 MMAs of K = 32 over the D-byte rows, 128- or
          // 64-byte swizzled (scales applied in the softmax)
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            if constexpr (D == 128)
              mma_f8_ss(d, smem_desc_sw128(aq + kk * 32, 16, 1024),
                        smem_desc_sw128(sk + kk * 32, 16, 1024), idesc_f8(128, BK), kk > 0 ? 1u : 0u);
            else
              mma_f8_ss(d, smem_desc_sw64(aq + kk * 32), smem_desc_sw64(sk + kk * 32), idesc_f8(128, BK),
                        kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(aq + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sk + (kk >> 2) * (BK * 128) + (kk & 3) * 32, 16, 1024);
            mma_f16_ss(d, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit(&bars[BAR_S0 + s]);
        tc_commit(&bars[BAR_KE0 + s]);   // the K stage is free once S is done
      }
      if (!ok) {
        aborted = true;
        tc_commit(&bars[BAR_DRAIN_S]);
        mbar_wait_drain(&bars[BAR_DRAIN_S], 0);
      }
    }
  } else if (warp == kPvWarp) {
    // ===================== PV issuer: O += P V =====================
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, true);
      const uint32_t sP = smem_u32(sm + L::oP);  // NVFP4 / FP8 P buffers
      if (F8) tc_cp_sf(tmem + TS::sfaP8(), smem_desc_rows16(sP + 2 * L::kF8));
      bool ok = true;
      for (int t = 0; t < rp.T; ++t) {
        const int s = t & 1;
        if (!mbar_wait(&bars[BAR_P0 + s], (t >> 1) & 1, ctx, 4)) { ok = false; break; }
        if (!mbar_wait(&bars[BAR_V0 + s], (t >> 1) & 1, ctx, 5)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sv = smem_u32(sm + (s ? L::oV1 : L::oV0));
        int kind_t, first_t;
        tile_of<BK>(rp, t, kind_t, first_t);
        if (FP4 && (kind_t == KIND_LOW || kind_t == KIND_RES)) {
          // NVFP4: P1 V1 (+ P1 V2 + P2 V1 on residual tiles)
          const int ncopy = (RES && kind_t == KIND_RES) ? 2 : 1;
          const uint32_t pb = sP + s * L::NC * L::kPfp4;
          for (int c = 0; c < ncopy; ++c) {
            const uint32_t sfa = tmem + TS::sfaP(c), sfb = tmem + TS::sfbV(c);
            tc_cp_sf(sfa, smem_desc_rows16(pb + c * L::kPfp4 + kFp4Sf));
            tc_cp_sf(sfa + 4, smem_desc_rows16(pb + c * L::kPfp4 + kFp4Sf + 512));
            tc_cp_sf(sfb, smem_desc_rows16(sv + c * L::kPfp4 + kFp4Sf));
            tc_cp_sf(sfb + 4, smem_desc_rows16(sv + c * L::kPfp4 + kFp4Sf + 512));
          }
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            mma_nvfp4_ss(tO, smem_desc_sw64(pb + kk * 32), smem_desc_sw64(sv + kk * 32),
                         idesc_nvfp4(128, D), tmem + TS::sfaP(0) + kk * 4,
                         tmem + TS::sfbV(0) + kk * 4, (t > 0 || kk > 0) ? 1u : 0u);
            if (RES && kind_t == KIND_RES) {
              mma_nvfp4_ss(tO, smem_desc_sw64(pb + kk * 32), smem_desc_sw64(sv + L::kPfp4 + kk * 32),
                           idesc_nvfp4(128, D), tmem + TS::sfaP(0) + kk * 4,
                           tmem + TS::sfbV(1) + kk * 4, 1u);
              mma_nvfp4_ss(tO, smem_desc_sw64(pb + L::kPfp4 + kk * 32), smem_desc_sw64(sv + kk * 32),
                           idesc_nvfp4(128, D), tmem + TS::sfaP(1) + kk * 4,
                           tmem + TS::sfbV(0) + kk * 4, 1u);
            }
          }
        } else if (F8 && kind_t == KIND_LOW) {
          // FP8 P codes (scale 2^0) x FP8 V codes (MN-major) with V's power-of-two
          // tile scale as the UE8M0 block scale
          const uint32_t pb = sP + s * L::kF8;
          tc_cp_sf(tmem + TS::sfbV8(), smem_desc_rows16(sv + L::kF8KV));
          // BK / 32 MMAs of K = 32 keys: P rows of BK bytes (K-major), V rows
          // of D bytes (MN-major), each 128- or 64-byte swizzled
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t ad = (BK == 128) ? smem_desc_sw128(pb + kk * 32, 16, 1024) : smem_desc_sw64(pb + kk * 32);
            const uint64_t bd = (D == 128) ? smem_desc_sw128(sv + kk * 32 * 128, 16, 1024)
                                           : smem_desc_sw64(sv + kk * 32 * 64);
            mma_mxf8_ss(tO, ad, bd, idesc_mxf8_bmn(128, D), tmem + TS::sfaP8(), tmem + TS::sfbV8(),
                        (t > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
          // A = bf16 P' in the TMEM P columns
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(sv + kk * 16 * 128, BK * 128, 1024);
            mma_f16_ts(tO, tP + kk * 8, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&bars[BAR_PD0 + s]);
        tc_commit(&bars[BAR_VE0 + s]);   // the V stage is free once PV is done
      }
      if (!ok) {
        aborted = true;
        tc_commit(&bars[BAR_DRAIN_PV]);
        mbar_wait_drain(&bars[BAR_DRAIN_PV], 0);
      }
    }
  } else if (warp < kSoftmaxWarps && (warp & 3) * 32 < a.bq) {
    // ===================== softmax warps =====================
    constexpr int HB = BK / kSplit;         // S columns per thread
    constexpr int HD = D / kSplit;          // O columns per thread
    const int quarter = warp & 3, part = warp >> 2;
    const int r = quarter * 32 + lane;      // query row within the tile == TMEM lane
    const int row_bar = 1 + quarter;        // named barrier of the warps sharing these rows
    constexpr int kBarThreads = 32 * kSplit;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float* xchg = reinterpret_cast<float*>(sm + L::oXchg);  // [slot][part][row]
    const float2* sc_tab = reinterpret_cast<const float2*>(sm + L::oScTab);
    const float c2 = a.scale_log2;           // S -> log2 units
    const float o_off = (float)a.p_offset;
    // FP8 tiles hold the dot products of the codes: their true S is S * s_q * s_k
    const float s_q8 = F8 ? a.q_s8[(int64_t)bh * a.nQb + qb] : 1.0f;
    float m = -INFINITY, l = 0.0f;           // running max (S units), part row sum
    bool tail_ok = true;   // false once a wait in a tile's tail failed (abort)
    for (int t = 0; t < rp.T; ++t) {
      const int s = t & 1;
      bool ok = tail_ok && mbar_wait(&bars[BAR_S0 + s], (t >> 1) & 1, ctx, 6);
      ok = __all_sync(0xffffffffu, ok);
      int kind, first;
      tile_of<BK>(rp, t, kind, first);
      int nvalid;
      if (kind == KIND_SKIP) {
        nvalid = min(BK, rp.n_skip - (first - rp.n_full - rp.n_res - rp.n_low));
      } else {
        nvalid = min(BK, a.N - rp.list[first] * BK);
      }
      const int nv = min(max(nvalid - part * HB, 0), HB);  // valid columns of this part
      const float sqk = (F8 && kind == KIND_LOW) ? s_q8 * a.k_s8[(int64_t)bh * a.nKb + rp.list[first]]
                                                 : 1.0f;   // exact: powers of two
      float x[HB];
      float tmax = -INFINITY;
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < HB; c0 += 32) {
          uint32_t raw[32];
          tmem_ld32((s ? tS1 : tS0) + lane_off + part * HB + c0, raw);
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c0 + c] = __uint_as_float(raw[c]);
        }
        // this part of S is in registers: the S buffer may take tile t+2
        tc_fence_before();
        mbar_arrive(&bars[BAR_SC0 + s]);
        if (nv < HB) {
#pragma unroll
          for (int c = 0; c < HB; ++c)
            if (c >= nv) x[c] = -INFINITY;
        }
        float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < HB; ++c) pm[c & 3] = fmaxf(pm[c & 3], x[c]);
        tmax = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])) * sqk;
        xchg[(s * 4 + part) * 128 + r] = tmax;
      }
      // swap part maxima with the warps sharing these rows; leave together on abort
      ok = bar_and(row_bar, kBarThreads, ok);
      if (!ok) { aborted = true; break; }
      float m_new = m;
#pragma unroll
      for (int q = 0; q < kSplit; ++q) m_new = fmaxf(m_new, xchg[(s * 4 + q) * 128 + r]);
      const float alpha = fast_exp2((m - m_new) * c2);  // 0 on the first tile
      const float mc = m_new * c2 - o_off;              // P' = 2^(s*c2 - mc)
      const float c2t = c2 * sqk;                       // this tile's S -> log2 units
      SoftmaxTail q;
      q.x = x;
      q.nv = nv;
      q.c2t = c2t;
      q.mc = mc;
      q.alpha = alpha;
      q.t = t;
      q.list = rp.list + first + part * HB;
      q.N = a.N;
      q.bars = bars;
      q.ctx = ctx;
      q.row_bar = row_bar;
      q.sm = sm;
      q.tP = tP + lane_off;
      q.tO = tO + lane_off;
      q.part = part;
      q.quarter = quarter;
      q.lane = lane;
      q.r = r;
      q.sc_tab = sc_tab;
      float psum = 0.0f;
      bool ok3;
      if (kind == KIND_SKIP) {
        ok3 = softmax_tail<PK_SKIP, D, BK, LM>(q, psum);
      } else if (kind == KIND_FULL) {
        ok3 = softmax_tail<PK_BF16, D, BK, LM>(q, psum);
      } else {
        if constexpr (RES) {
          ok3 = (kind == KIND_RES) ? softmax_tail<PK_RES, D, BK, LM>(q, psum)
                                   : softmax_tail<PK_FP4, D, BK, LM>(q, psum);
        } else if constexpr (FP4) {
          ok3 = softmax_tail<PK_FP4, D, BK, LM>(q, psum);
        } else if constexpr (F8) {
          ok3 = softmax_tail<PK_F8, D, BK, LM>(q, psum);
        } else {
          ok3 = false;   // no low tier in this instance: not reached
        }
      }
      // a failed wait leaves the loop at the next row barrier, with the other
      // warps of these rows
      if (!ok3) tail_ok = false;
      l = l * alpha + psum;
      m = m_new;
    }
    if (!aborted) {
      bool ok = tail_ok && mbar_wait(&bars[BAR_PD0 + ((rp.T - 1) & 1)], ((rp.T - 1) >> 1) & 1, ctx, 8);
      ok = __all_sync(0xffffffffu, ok);
      // row sums through the exchange slot the last tile did not use (its
      // last readers passed the last tile's row barrier)
      const int ls = rp.T & 1;
      xchg[(ls * 4 + part) * 128 + r] = l;
      ok = bar_and(row_bar, kBarThreads, ok);
      if (ok) {
        tc_fence_after();
        float lt = 0.0f;
#pragma unroll
        for (int q = 0; q < kSplit; ++q) lt += xchg[(ls * 4 + q) * 128 + r];
        const float inv_l = 1.0f / lt;
        const bool valid = (q0 + r) < a.N;
        __nv_bfloat16* orow = a.O + (int64_t)b * a.sb + (int64_t)h * a.sh + (int64_t)(q0 + r) * a.sn +
                              part * HD;
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t raw[32];
          tmem_ld32(tO + lane_off + part * HD + c0, raw);
          uint32_t w[16];
          const uint64_t il2 = pack2(inv_l, inv_l);
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float o0, o1;
            unpack2(mul2(pack2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), il2), o0, o1);
            w[c / 2] = pack_bf16(o0, o1);
          }
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              *reinterpret_cast<uint4*>(orow + c0 + v * 8) =
                  make_uint4(w[v * 4 + 0], w[v * 4 + 1], w[v * 4 + 2], w[v * 4 + 3]);
          }
        }
      } else {
        aborted = true;
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int D, int BK, int LM>
cudaError_t launch_d(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t s) {
  using L = Smem<D, BK, LM>;
  auto k = attn_kernel<D, BK, LM>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nQb, a.B * a.H);
  k<<<grid, Roles<D, BK>::kThreads, L::kAlloc, s>>>(a, maps[0], maps[1], maps[2], maps[3], maps[4],
                                                   maps[5], maps[6], maps[7], maps[8]);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t s) {
  // d = 128 with 128 x 128 tiles runs on the two-group kernel (ta_attn2.cu)
  const cudaError_t e2 = launch_attn2(a, maps, s);
  if (e2 != cudaErrorNotSupported) return e2;
  // FP8 low tiles run natively on the FP8 tensor pipe at every shape
  if (a.low == TA_LOW_FP8_E4M3) {
    if (a.d == 64 && a.bk == 64) return launch_d<64, 64, LM_FP8>(a, maps, s);
    if (a.d == 64 && a.bk == 128) return launch_d<64, 128, LM_FP8>(a, maps, s);
    if (a.d == 128 && a.bk == 64) return launch_d<128, 64, LM_FP8>(a, maps, s);
    return launch_d<128, 128, LM_FP8>(a, maps, s);
  }
  if (a.d == 64 && a.bk == 64) return launch_d<64, 64, LM_IMAGE>(a, maps, s);
  if (a.d == 64 && a.bk == 128) return launch_d<64, 128, LM_IMAGE>(a, maps, s);
  if (a.d == 128 && a.bk == 64) return launch_d<128, 64, LM_IMAGE>(a, maps, s);
  if (a.low == TA_LOW_NVFP4) return launch_d<128, 128, LM_NVFP4>(a, maps, s);
  if (a.low == TA_LOW_NVFP4_RES) return launch_d<128, 128, LM_NVFP4_RES>(a, maps, s);
  return launch_d<128, 128, LM_IMAGE>(a, maps, s);
}

}  // namespace ta
