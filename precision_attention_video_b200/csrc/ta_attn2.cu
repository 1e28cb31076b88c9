// ta_attn2.cu -- the fused one-pass tiered attention kernel for d = 128 and
// 128 x 128 tiles (sm_100a): two softmax warpgroups on alternating tiles.
//
// "Triage" (zhuanzhiai paper page, abstract) runs every tier of a query block
// in one fused pass: full tiles in bf16, low tiles in reduced precision (here
// NVFP4, NVFP4 + residual, or FP8), and skipped blocks replaced by their
// block means, so that block j of n_j keys adds n_j exp(q . kbar_j * scale) to
// the softmax denominator and that weight times vbar_j to the numerator.  One
// CTA owns one (head, query block) and walks the block's compacted tile list
// (full, residual, low tiles, each by descending pooled mass, then the skipped
// blocks in chunks of 128) with an online softmax.
//
// Roles (12 warps; warp 11 idles):
//   warps 0-3, 4-7  softmax groups A and B.  Group A takes the even tiles of
//               the row, group B the odd ones; a thread owns one query row
//               (TMEM lane) and all 128 columns of the tile.  While one group
//               runs its exponentials the tensor pipe works on the other
//               group's S and PV.  The running maximum is handed from group to
//               group through shared memory (tile t's maximum is published as
//               soon as it is known, before tile t's exponentials).
//   warp 8, 9   producers of K and of V: TMA loads of the kept tiles into two
//               rings of 32 KB stages (bf16 tiles, or the low copies with
//               their block scales gathered for tcgen05.cp), and for skip
//               chunks a gather of up to 128 pooled rows kbar_b / vbar_b.
//   warp 10     issues every MMA (the whole warp runs the loop, one elected
//               lane issues), in this order: S(0), S(1), then PV(t), S(t+2)
//               for t = 0, 1, ...  Issue order is execution order on the
//               tensor pipe, which lets bf16 P(t) live in the TMEM columns of
//               its own S(t): S(t+2), which overwrites them, runs after PV(t)
//               has read them.
// TMEM (512 columns): O [0,128), S of group A [128,256), S of group B
// [256,384), Q as the bf16 A operand of S = Q K^T [384,448) (so that S reads
// only K from shared memory), block scales [448,512).
// NVFP4 / FP8 P goes to shared memory, into the half of its tile's V stage
// that the low V copy leaves free: the PV that last read that stage finished
// before S(t) (issued after it) did.
// O is rescaled by exp(m_old - m_new) only in warps where the maximum grew,
// after the previous tile's PV; the two groups keep their own row sums and
// combine them at the end.  Every wait is bounded: a wait that runs out sets
// the CTA's abort flag and the workspace status word, all roles leave their
// loops, issued copies and MMAs are drained (bounded), TMEM is freed.
#include "ta_common.cuh"
#include "ta_kernels.cuh"
#include "ta_attn_common.cuh"

namespace ta {
namespace {

using namespace tile;

constexpr int kD = 128, kBK = 128;

// Shared-memory layout (offsets from a 1024-aligned base) of one instance.
template <int LM>
struct Lay {
  static constexpr bool FP4 = (LM == LM_NVFP4 || LM == LM_NVFP4_RES);
  static constexpr bool RES = (LM == LM_NVFP4_RES);
  static constexpr bool F8 = (LM == LM_FP8);
  static constexpr int NC = RES ? 2 : 1;         // NVFP4 copies per operand
  static constexpr int NK = 3;                   // K ring stages
  static constexpr int NV = RES ? 2 : 3;         // V ring stages
  static constexpr int kStage = 32768;           // one bf16 128 x 128 tile
  static constexpr int kCodes = 8192;            // one NVFP4 copy: [128 rows][64 B]
  static constexpr int kSfBlk = 1024;            // its scales: two [32][16 B] blocks
  static constexpr int kKSide = FP4 ? NC * kSfBlk : 512;
  static constexpr int kVSide = FP4 ? 2 * NC * kSfBlk : (F8 ? 512 : 0);
  static constexpr int kQlow = FP4 ? NC * (kCodes + kSfBlk) : (F8 ? 16384 : 0);
  static constexpr int oK = 0;
  static constexpr int oV = oK + NK * kStage;
  static constexpr int oKS = oV + NV * kStage;   // per K stage: NVFP4 K scales
  static constexpr int oVS = oKS + NK * kKSide;  // per V stage: V scales, then P scales
  static constexpr int oQL = oVS + NV * kVSide;  // the query block's low copy (+ scales)
  static constexpr int oP8 = oQL + kQlow;        // FP8: UE8M0 scales of P (all 2^0)
  static constexpr int oBar = oP8 + (F8 ? 512 : 0);
  static constexpr int kBars = 32;
  static constexpr int oMisc = oBar + kBars * 8;
  static constexpr int oM = oMisc + 64;          // float [2][128]: running max, by tile parity
  static constexpr int oX = oM + 2 * 128 * 4;    // float [2 groups][2][128]: final (l, m)
  static constexpr int oSc = oX + 4 * 128 * 4;   // float2 [128]: ue4m3 value, 1 / value
  static constexpr int kTotal = oSc + 128 * 8;
  static constexpr int oPinV = 16384;            // low P inside its V stage
  static_assert(kQlow == 0 || oQL % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kTotal <= 227 * 1024, "shared memory");
  static_assert(NK <= 3 && NV <= 3, "the mbarrier slots below hold at most three stages per ring");
};

// TMEM columns.
template <int LM>
struct Tm {
  static constexpr int NC = Lay<LM>::NC;
  static constexpr uint32_t kO = 0, kS0 = 128, kQ = 384, kSf = 448;
  static constexpr uint32_t sfaQ(int c) { return kSf + 8 * c; }
  static constexpr uint32_t sfbK(int c) { return kSf + 8 * NC + 8 * c; }
  static constexpr uint32_t sfbV(int c) { return kSf + 16 * NC + 8 * c; }
  static constexpr uint32_t sfaP(int c) { return kSf + 24 * NC + 8 * c; }
  static constexpr uint32_t kSfaP8 = kSf, kSfbV8 = kSf + 4;
  static_assert(kSf + 32 * NC <= 512, "TMEM columns");
};

constexpr int kSoftWarps = 8, kProdKWarp = 8, kProdVWarp = 9, kMmaWarp = 10;
constexpr int kThreads2 = 32 * 12;   // warp 11 only completes the third warpgroup
// Register split (setmaxnreg): the launch gives every thread 168; the two
// softmax warpgroups take 192 each (an S row of 128 floats lives in
// registers), the producer / MMA warpgroup gives back down to 112:
// 256 * 192 + 128 * 112 = 63488 <= 384 * 168 = 64512.
constexpr int kRegSoft = 192, kRegOther = 112;
static_assert(256 * kRegSoft + 128 * kRegOther <= kThreads2 * 168, "register split");

// mbarriers
enum {
  B_QR = 0,      // Q rows written into TMEM (group A, one arrival per warp)
  B_QL = 1,      // the query block's low copy landed (TMA)
  B_KF = 2,      // K stage full  [NK]
  B_KE = 5,      // K stage empty [NK] (S of its tile done)
  B_VF = 8,      // V stage full  [NV]
  B_VE = 11,     // V stage empty [NV] (PV of its tile done)
  B_SR = 14,     // S of group g's tile in TMEM [2]
  B_PR = 16,     // P of group g's tile written [2] (one arrival per warp)
  B_MX = 18,     // running max after group g's tile published [2] (one per warp)
  B_PD = 20,     // PV of group g's tile done [2]
  B_DRAIN = 22
};

// Named barrier over `count` threads that also ANDs a predicate across them.
__device__ __forceinline__ bool bar_and2(int id, int count, bool pred) {
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

// Tile t of a row whose kept key blocks are KB keys wide, PK = 128 / KB of
// them (consecutive in the list, one tier) to a 128-key tile: its kind, the
// list position of its first block and how many blocks it holds (for a skip
// chunk: how many skipped blocks, up to 128).  Skipped blocks follow the kept
// tiles in chunks of 128.
template <int PK>
__device__ __forceinline__ void tile_of_packed(const RowPlan& rp, int t, int& kind, int& first, int& cnt) {
  const int nf = (rp.n_full + PK - 1) / PK, nr = (rp.n_res + PK - 1) / PK;
  const int nl = (rp.n_low + PK - 1) / PK;
  if (t < nf) {
    kind = KIND_FULL;
    first = t * PK;
    cnt = min(PK, rp.n_full - first);
  } else if (t < nf + nr) {
    const int u = (t - nf) * PK;
    kind = KIND_RES;
    first = rp.n_full + u;
    cnt = min(PK, rp.n_res - u);
  } else if (t < nf + nr + nl) {
    const int u = (t - nf - nr) * PK;
    kind = KIND_LOW;
    first = rp.n_full + rp.n_res + u;
    cnt = min(PK, rp.n_low - u);
  } else {
    const int kept = rp.n_full + rp.n_res + rp.n_low;
    kind = KIND_SKIP;
    first = kept + (t - nf - nr - nl) * 128;
    cnt = min(128, rp.n_skip - (first - kept));
  }
}

// Key blocks of a packed tile: slot i holds list entry first + i; slots past
// cnt repeat the last real block (their columns are masked, their values
// only need to be finite).
template <int PK>
__device__ __forceinline__ void pack_blocks(const RowPlan& rp, int first, int cnt, int (&jsl)[PK]) {
#pragma unroll
  for (int i = 0; i < PK; ++i) jsl[i] = rp.list[first + min(i, cnt - 1)];
}

// NVFP4 block scales of the 128 key rows of a packed tile (row rr = slot
// rr / KB, key (rr % KB) of that slot's block) into the two [32][16 B] blocks
// at dst: row 32*m1 + m0 of K chunk c at dst + c*512 + m0*16 + m1*4.  Keys
// past N get zero scales.  `src` points at the head's [N][8] scales.
template <int KB, int PK>
__device__ __forceinline__ void gather_key_sf(unsigned char* dst, const uint8_t* src, const int (&jsl)[PK],
                                              int N, int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = lane * 4 + i, slot = rr / KB;
    int j = jsl[0];
#pragma unroll
    for (int u = 1; u < PK; ++u) j = (slot == u) ? jsl[u] : j;
    const int key = j * KB + rr % KB;
    uint2 v = make_uint2(0u, 0u);
    if (key < N) v = *reinterpret_cast<const uint2*>(src + (int64_t)key * 8);
    const int off = (rr & 31) * 16 + (rr >> 5) * 4;
    *reinterpret_cast<uint32_t*>(dst + off) = v.x;
    *reinterpret_cast<uint32_t*>(dst + 512 + off) = v.y;
  }
}

// Formats of P' in a tile's softmax tail.
enum { T_BF16 = 0, T_SKIP = 1, T_FP4 = 2, T_RES = 3, T_F8 = 4 };

// Pairs of columns (of every 8) whose exponentials run on the FMA pipe
// (exp2_poly2) instead of ex2 on the MUFU unit.  Measured on whole 480p
// layers, 2 of 8 pairs made the forward 13 % slower and 3 of 8 slower still:
// the softmax is bound by latency, not by the MUFU pipe, and the polynomial
// lengthens each thread's chain.  Kept at 0; the path stays for tuning.
template <int K>
constexpr int kEmuPairs() {
  return 0;
}

// What one thread's tail of a tile needs (one query row, 128 columns).
struct Tail {
  float c2t, mc;            // P' = 2^(s * c2t - mc)
  float alpha;              // exp(m_old - m_new) of this row
  int t;                    // tile index
  int last_col;             // skip chunks: column of the last key block, or -1
  float w_last;             // its key count
  float w_blk;              // the key count of every other block
  uint64_t* bars;
  AbortCtx ctx;
  unsigned char* sm;
  uint32_t tS, tO;          // this lane's S columns of the group, O accumulator
  int r;                    // query row == TMEM lane
  int g;                    // softmax group
  const float2* sc_tab;
};

// Tail of one tile's softmax: P' = 2^o exp(s - m') from the S row in x, its
// row sum, P' rounded as the tier demands, O rescaled when the maximum grew
// (after the previous tile's PV), and P' handed to the PV MMA: bf16 over the
// group's own S columns in TMEM, NVFP4 / FP8 into the tile's V stage.  False
// when the CTA aborts.
template <int K, int LM>
__device__ __forceinline__ bool tail(float (&x)[128], const float (&gm)[8], const Tail& q, float& psum) {
  using L = Lay<LM>;
  {
    // exponent arguments two at a time (packed fp32 FMA); in every 8 pairs of
    // columns, kEmu pairs take the FMA-pipe exponential and the rest ex2 on
    // the MUFU unit, so that neither pipe bounds the tile alone
    constexpr int kEmu = kEmuPairs<K>();
    const uint64_t c2t2 = pack2(q.c2t, q.c2t), nmc2 = pack2(-q.mc, -q.mc);
#pragma unroll
    for (int c = 0; c < 128; c += 2) {
      float a0, a1;
      unpack2(fma2(pack2(x[c], x[c + 1]), c2t2, nmc2), a0, a1);
      if (((c / 2) % 8) < kEmu) {
        exp2_poly2(a0, a1, x[c], x[c + 1]);
      } else {
        x[c] = fast_exp2(a0);
        x[c + 1] = fast_exp2(a1);
      }
    }
  }
  if constexpr (K == T_SKIP) {
    // pooled keys weigh n_j: KB for every block but the sequence's ragged
    // last one, which sits in column q.last_col (or nowhere: -1); columns
    // past nv are exp(-inf) = 0 already
#pragma unroll
    for (int c = 0; c < 128; ++c) x[c] *= (c == q.last_col) ? q.w_last : q.w_blk;
  }
  {
    uint64_t sa = pack2(0.0f, 0.0f), sb = pack2(0.0f, 0.0f);
#pragma unroll
    for (int c = 0; c < 128; c += 4) {
      sa = add2(sa, pack2(x[c], x[c + 1]));
      sb = add2(sb, pack2(x[c + 2], x[c + 3]));
    }
    float s0, s1, s2, s3;
    unpack2(sa, s0, s1);
    unpack2(sb, s2, s3);
    psum = (s0 + s1) + (s2 + s3);
  }

  // P' rounded as the tier demands
  constexpr int kWords = (K == T_RES) ? 40 : (K == T_FP4 ? 20 : (K == T_F8 ? 32 : 64));
  uint32_t p[kWords];
  if constexpr (K == T_FP4 || K == T_RES) {
    // codes of 32 keys in p[4q .. 4q+3], their two ue4m3 scales in p[16 + q]
    // (residual copy: codes in p[20 + 4q ..], scales in p[36 + q])
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      // each group's amax is P' of its largest S (exp2 is increasing)
      const float am0 = fast_exp2(fmaf(gm[2 * c], q.c2t, -q.mc));
      const float am1 = fast_exp2(fmaf(gm[2 * c + 1], q.c2t, -q.mc));
      p[16 + c] = nvfp4_quant32_am(x + 32 * c, am0, am1, q.sc_tab, p + 4 * c);
      if constexpr (K == T_RES)
        p[36 + c] = nvfp4_residual32(x + 32 * c, p + 4 * c, p[16 + c], q.sc_tab, p + 20 + 4 * c);
    }
  } else if constexpr (K == T_F8) {
#pragma unroll
    for (int c = 0; c < 128; c += 4)
      p[c / 4] = cvt_e4m3x2(x[c], x[c + 1]) | (cvt_e4m3x2(x[c + 2], x[c + 3]) << 16);
  } else {
#pragma unroll
    for (int c = 0; c < 128; c += 2) p[c / 2] = pack_bf16(x[c], x[c + 1]);
  }

  const int vs = q.t % L::NV;
  unsigned char* vst = q.sm + L::oV + vs * L::kStage + L::oPinV;
  unsigned char* vside = q.sm + L::oVS + vs * L::kVSide + L::NC * L::kSfBlk;
  if constexpr (K == T_FP4 || K == T_RES) {
    // codes: row r of a [128][64 B] 64-byte-swizzled tile; scales: byte
    // (group) of K chunk kc at kc * 512 + (r % 32) * 16 + (r / 32) * 4
    constexpr int ncopy = (K == T_RES) ? 2 : 1;
    const int r = q.r;
#pragma unroll
    for (int cp = 0; cp < ncopy; ++cp) {
      const uint32_t* pc = p + 20 * cp;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(vst + cp * L::kCodes + r * 64 + ((c ^ ((r >> 1) & 3)) * 16)) =
            make_uint4(pc[4 * c], pc[4 * c + 1], pc[4 * c + 2], pc[4 * c + 3]);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
        *reinterpret_cast<uint32_t*>(vside + cp * L::kSfBlk + kc * 512 + (r & 31) * 16 + (r >> 5) * 4) =
            (pc[16 + 2 * kc] & 0xFFFFu) | (pc[17 + 2 * kc] << 16);
    }
    fence_proxy_async_smem();
  } else if constexpr (K == T_F8) {
    const int r = q.r;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch)
      *reinterpret_cast<uint4*>(vst + r * 128 + ((ch ^ (r & 7)) * 16)) =
          make_uint4(p[ch * 4 + 0], p[ch * 4 + 1], p[ch * 4 + 2], p[ch * 4 + 3]);
    fence_proxy_async_smem();
  } else {
    tmem_st32(q.tS, *reinterpret_cast<const uint32_t(*)[32]>(p));
    tmem_st32(q.tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(p + 32));
  }
  // O rescale: only where the maximum grew, once the previous tile's PV
  // (the other group's) is done; P(t) is written already, but PV(t) is
  // issued only after the arrival below
  if (q.t > 0 && __any_sync(0xffffffffu, q.alpha != 1.0f)) {
    bool ok = mbar_wait(&q.bars[B_PD + (q.g ^ 1)], ((q.t - 1) >> 1) & 1, q.ctx, 21);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    const uint64_t al2 = pack2(q.alpha, q.alpha);
#pragma unroll
    for (int c0 = 0; c0 < kD; c0 += 32) {
      uint32_t raw[32];
      tmem_ld32(q.tO + c0, raw);
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float o0, o1;
        unpack2(mul2(pack2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), al2), o0, o1);
        raw[c] = __float_as_uint(o0);
        raw[c + 1] = __float_as_uint(o1);
      }
      tmem_st32(q.tO + c0, raw);
    }
  }

  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if ((q.r & 31) == 0) mbar_arrive(&q.bars[B_PR + q.g]);   // one arrival per warp
  return true;
}

template <int LM, int KB>
__global__ void __launch_bounds__(kThreads2, 1)
    attn2_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                 const __grid_constant__ CUtensorMap tmDV, const __grid_constant__ CUtensorMap tmRQ,
                 const __grid_constant__ CUtensorMap tmRK, const __grid_constant__ CUtensorMap tmRV) {
  using L = Lay<LM>;
  using TM = Tm<LM>;
  constexpr bool FP4 = L::FP4, RES = L::RES, F8 = L::F8;
  constexpr int NK = L::NK, NV = L::NV;
  constexpr int PK = kBK / KB;   // key blocks per tile
  static_assert(PK == 1 || (PK == 4 && !F8), "32-key blocks: bf16 and NVFP4 tiers");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw;
  if (smem_u32(sm) & 1023u) {
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
  rp.T = (rp.n_full + PK - 1) / PK + (rp.n_res + PK - 1) / PK + (rp.n_low + PK - 1) / PK +
         (rp.n_skip + kBK - 1) / kBK;
  const int kept = rp.n_full + rp.n_res + rp.n_low;
  const bool has_low = (FP4 || F8) && (rp.n_low > 0 || rp.n_res > 0);
  const int nq = rp.n_res > 0 ? 2 : (has_low ? 1 : 0);   // query low copies to load
  const int T = rp.T;

  AbortCtx ctx{abort_flag, a.status};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bars[B_QR], 4);
    mbar_init(&bars[B_QL], 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&bars[B_KF + i], 1);
      mbar_init(&bars[B_KE + i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&bars[B_VF + i], 1);
      mbar_init(&bars[B_VE + i], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bars[B_SR + g], 1);
      mbar_init(&bars[B_PR + g], 4);   // one arrival per warp of the group
      mbar_init(&bars[B_MX + g], 4);
      mbar_init(&bars[B_PD + g], 1);
    }
    mbar_init(&bars[B_DRAIN], 1);
    fence_mbar_init();
  }
  if (F8 && threadIdx.x < 128) {
    *reinterpret_cast<uint32_t*>(sm + L::oP8 + threadIdx.x * 4) = 0x7F7F7F7Fu;
    fence_proxy_async_smem();
  }
  if (FP4 && threadIdx.x < 128) {
    const float v = (threadIdx.x == 0x7F) ? 0.0f : e4m3_to_float(threadIdx.x);
    reinterpret_cast<float2*>(sm + L::oSc)[threadIdx.x] = make_float2(v, v > 0.0f ? __frcp_rn(v) : 0.0f);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + TM::kO, tQ = tmem + TM::kQ;

  if (warp >= kSoftWarps) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegOther));
  if (warp == kProdKWarp || warp == kProdVWarp) {
    // ===================== producers =====================
    const bool isK = (warp == kProdKWarp);
    const int depth = isK ? NK : NV;
    int issued[3] = {0, 0, 0};
    uint64_t* full = &bars[isK ? B_KF : B_VF];
    uint64_t* empty = &bars[isK ? B_KE : B_VE];
    bool aborted = false;
    if (isK && has_low) {
      if (FP4) {
        for (int c = 0; c < nq; ++c)
          gather_row_sf(sm + L::oQL + L::NC * L::kCodes + c * L::kSfBlk,
                        (c ? a.rq_sf : a.q_sf) + ((int64_t)bh * a.N + q0) * 8, min(128, a.N - q0), lane);
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        tma_prefetch_desc(&tmDQ);
        if (FP4) {
          mbar_arrive_expect_tx(&bars[B_QL], (uint32_t)(nq * a.bq * 64));
          tma_load_3d(sm + L::oQL, &tmDQ, &bars[B_QL], 0, q0, bh);
          if (nq > 1) tma_load_3d(sm + L::oQL + L::kCodes, &tmRQ, &bars[B_QL], 0, q0, bh);
        } else {
          mbar_arrive_expect_tx(&bars[B_QL], (uint32_t)(a.bq * 128));
          tma_load_3d(sm + L::oQL, &tmDQ, &bars[B_QL], 0, q0, bh);
        }
      }
    }
    if (lane == 0) tma_prefetch_desc(isK ? &tmK : &tmV);
    const __nv_bfloat16* pooled = (isK ? a.kbar_b : a.vbar_b) + (int64_t)bh * a.nKb * kD;
    for (int t = 0; t < T; ++t) {
      const int s = t % depth;
      if (t >= depth) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], ((t / depth) - 1) & 1, ctx, isK ? 1 : 10);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { aborted = true; break; }
      }
      int kind, first, cnt = 0;
      if constexpr (PK == 1)
        tile_of<kBK>(rp, t, kind, first);
      else
        tile_of_packed<PK>(rp, t, kind, first, cnt);
      unsigned char* st = sm + (isK ? L::oK : L::oV) + s * L::kStage;
      unsigned char* side = sm + (isK ? L::oKS + s * L::kKSide : L::oVS + s * L::kVSide);
      const bool drop = isK && (t == 0) && (a.debug_flags & TA_DEBUG_DROP_FIRST_K);
      if (kind != KIND_SKIP && PK > 1) {
        // packed tile: PK key blocks of KB keys side by side
        int jsl[PK];
        pack_blocks<PK>(rp, first, cnt, jsl);
        if (FP4 && (kind == KIND_LOW || kind == KIND_RES)) {
          const int ncopy = (RES && kind == KIND_RES) ? 2 : 1;
          for (int c = 0; c < ncopy; ++c) {
            if (isK) {
              gather_key_sf<KB, PK>(side + c * L::kSfBlk, (c ? a.rk_sf : a.k_sf) + (int64_t)bh * a.N * 8, jsl,
                                    a.N, lane);
            } else {
              // V scales: groups of 16 keys of each d row of V^T; group k of K
              // chunk kc covers keys 64 kc + 16 k .. of the tile, in block
              // (4 kc + k) / (KB / 16)
              const uint8_t* vsf = c ? a.rv_sf : a.v_sf;
              const int ng = a.Np / 16;
#pragma unroll
              for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  constexpr int kGroups = KB / 16;   // scale groups per key block
                  const int gi = jsl[(kc * 4 + k) / kGroups] * kGroups + (kc * 4 + k) % kGroups;
                  uint32_t w = 0u;
                  if (gi < ng)
                    w = *reinterpret_cast<const uint32_t*>(vsf + ((int64_t)bh * ng + gi) * kD + lane * 4);
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    const int m = lane * 4 + i;
                    side[c * L::kSfBlk + kc * 512 + (m & 31) * 16 + (m >> 5) * 4 + k] = (unsigned char)(w >> (8 * i));
                  }
                }
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && !drop) {
            mbar_arrive_expect_tx(&full[s], ncopy * 128 * 64);
            for (int c = 0; c < ncopy; ++c) {
#pragma unroll
              for (int i = 0; i < PK; ++i) {
                // K: KB rows of 64 bytes; V^T: 128 rows of KB / 2 bytes
                if (isK)
                  tma_load_3d(st + c * L::kCodes + i * (KB * 64), c ? &tmRK : &tmDK, &full[s], 0, jsl[i] * KB, bh);
                else
                  tma_load_3d(st + c * L::kCodes + i * (KB * 64), c ? &tmRV : &tmDV, &full[s], jsl[i] * (KB / 2),
                              0, bh);
              }
            }
            issued[s]++;
          }
        } else {
          if (lane == 0 && !drop) {
            mbar_arrive_expect_tx(&full[s], kBK * kD * 2);
#pragma unroll
            for (int i = 0; i < PK; ++i)
              for (int x = 0; x < 2; ++x)
                tma_load_4d(st + x * (kBK * 128) + i * (KB * 128), isK ? &tmK : &tmV, &full[s], x * 64,
                            jsl[i] * KB, h, b);
            issued[s]++;
          }
        }
      } else if (FP4 && (kind == KIND_LOW || kind == KIND_RES)) {
        const int j = rp.list[first];
        const int ncopy = (RES && kind == KIND_RES) ? 2 : 1;
        for (int c = 0; c < ncopy; ++c) {
          if (isK) {
            gather_row_sf(side + c * L::kSfBlk, (c ? a.rk_sf : a.k_sf) + ((int64_t)bh * a.N + j * kBK) * 8,
                          min(kBK, a.N - j * kBK), lane);
          } else {
            // V scales: groups of 16 keys of each d row of V^T
            const uint8_t* vsf = c ? a.rv_sf : a.v_sf;
            const int ng = a.Np / 16;
#pragma unroll
            for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int gi = j * 8 + kc * 4 + k;
                uint32_t w = 0u;
                if (gi < ng)
                  w = *reinterpret_cast<const uint32_t*>(vsf + ((int64_t)bh * ng + gi) * kD + lane * 4);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int m = lane * 4 + i;
                  side[c * L::kSfBlk + kc * 512 + (m & 31) * 16 + (m >> 5) * 4 + k] = (unsigned char)(w >> (8 * i));
                }
              }
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && !drop) {
          mbar_arrive_expect_tx(&full[s], ncopy * 128 * 64);
          for (int c = 0; c < ncopy; ++c) {
            if (isK)
              tma_load_3d(st + c * L::kCodes, c ? &tmRK : &tmDK, &full[s], 0, j * kBK, bh);
            else
              tma_load_3d(st + c * L::kCodes, c ? &tmRV : &tmDV, &full[s], j * 64, 0, bh);
          }
          issued[s]++;
        }
      } else if (F8 && kind == KIND_LOW) {
        const int j = rp.list[first];
        if (!isK) {
          // UE8M0 scale factor of this V tile: the exponent of its power-of-two scale
          const uint32_t e = (__float_as_uint(a.v_s8[(int64_t)bh * a.nKb + j]) >> 23) & 0xFFu;
#pragma unroll
          for (int i = 0; i < 4; ++i) reinterpret_cast<uint32_t*>(side)[lane * 4 + i] = e * 0x01010101u;
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0 && !drop) {
          mbar_arrive_expect_tx(&full[s], kBK * 128);
          tma_load_3d(st, isK ? &tmDK : &tmDV, &full[s], 0, j * kBK, bh);
          issued[s]++;
        }
      } else if (kind != KIND_SKIP) {
        if (lane == 0 && !drop) {
          const int j = rp.list[first];
          mbar_arrive_expect_tx(&full[s], kBK * kD * 2);
          for (int x = 0; x < 2; ++x)
            tma_load_4d(st + x * (kBK * 128), isK ? &tmK : &tmV, &full[s], x * 64, j * kBK, h, b);
          issued[s]++;
        }
      } else {
        // pooled rows of the chunk's skipped blocks as a pseudo tile: the
        // list entries once (lane l holds columns l, l+32, ...), then every
        // 16-byte piece as an asynchronous copy (zero past the chunk's end)
        if constexpr (PK == 1) cnt = min(kBK, rp.n_skip - (first - kept));
        int jl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = lane + 32 * i;
          jl[i] = (c < cnt) ? rp.list[first + c] : 0;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll 4
          for (int c1 = 0; c1 < 32; c1 += 2) {
            const int c = 32 * i + c1 + lane / 16, ch = lane % 16;
            const int j = __shfl_sync(0xffffffffu, jl[i], c % 32);
            const uint32_t off = (ch >> 3) * (kBK * 128) + c * 128 + (((ch & 7) ^ (c & 7)) * 16);
            cp_async16(st + off, pooled + (int64_t)j * kD + ch * 8, c < cnt ? 16u : 0u);
          }
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
      for (int s = 0; s < depth; ++s)
        if (issued[s] > 0) mbar_wait_drain(&full[s], (issued[s] - 1) & 1);
      if (isK && has_low) mbar_wait_drain(&bars[B_QL], 0);
    }
  } else if (warp == kMmaWarp) {
    // ===================== MMA issuer =====================
    // the whole warp runs the issue loop (converged, warp-uniform values);
    // elect.sync picks the lane that issues each tcgen05 instruction
    {
      const uint32_t tS0 = tmem + TM::kS0;
      const uint32_t sQL = smem_u32(sm + L::oQL);
      constexpr uint32_t idesc_qk = idesc_bf16(128, kBK, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, kD, true);
      // waits agreed by the whole warp, so that it stays converged
      auto wait_all = [&](uint64_t* bar, uint32_t parity, int site) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, ctx, site));
      };
      bool ok = wait_all(&bars[B_QR], 0, 3);
      if (ok && has_low) ok = wait_all(&bars[B_QL], 0, 3);
      if (ok) {
        tc_fence_after();
        if (FP4) {
          for (int c = 0; c < nq; ++c) {
            const uint32_t sf = sQL + L::NC * L::kCodes + c * L::kSfBlk;
            tc_cp_sf_w(tmem + TM::sfaQ(c), smem_desc_rows16(sf));
            tc_cp_sf_w(tmem + TM::sfaQ(c) + 4, smem_desc_rows16(sf + 512));
          }
        }
        if (F8) tc_cp_sf_w(tmem + TM::kSfaP8, smem_desc_rows16(smem_u32(sm + L::oP8)));
      }
      // S(t) = Q K(t)^T into the S columns of group t % 2
      auto issue_s = [&](int t) -> bool {
        const int s = t % NK;
        if (!wait_all(&bars[B_KF + s], (t / NK) & 1, 2)) return false;
        tc_fence_after();
        int kind, first, cnt;
        if constexpr (PK == 1)
          tile_of<kBK>(rp, t, kind, first);
        else
          tile_of_packed<PK>(rp, t, kind, first, cnt);
        const uint32_t sk = smem_u32(sm + L::oK + s * L::kStage);
        const uint32_t d = tS0 + 128 * (t & 1);
        if (FP4 && (kind == KIND_LOW || kind == KIND_RES)) {
          const int ncopy = (RES && kind == KIND_RES) ? 2 : 1;
          const uint32_t ksf = smem_u32(sm + L::oKS + s * L::kKSide);
          for (int c = 0; c < ncopy; ++c) {
            tc_cp_sf_w(tmem + TM::sfbK(c), smem_desc_rows16(ksf + c * L::kSfBlk));
            tc_cp_sf_w(tmem + TM::sfbK(c) + 4, smem_desc_rows16(ksf + c * L::kSfBlk + 512));
          }
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            mma_nvfp4_ss_w(d, smem_desc_sw64(sQL + kk * 32), smem_desc_sw64(sk + kk * 32),
                           idesc_nvfp4(128, kBK), tmem + TM::sfaQ(0) + kk * 4,
                           tmem + TM::sfbK(0) + kk * 4, kk > 0 ? 1u : 0u);
            if (RES && kind == KIND_RES) {
              mma_nvfp4_ss_w(d, smem_desc_sw64(sQL + kk * 32), smem_desc_sw64(sk + L::kCodes + kk * 32),
                             idesc_nvfp4(128, kBK), tmem + TM::sfaQ(0) + kk * 4,
                             tmem + TM::sfbK(1) + kk * 4, 1u);
              mma_nvfp4_ss_w(d, smem_desc_sw64(sQL + L::kCodes + kk * 32), smem_desc_sw64(sk + kk * 32),
                             idesc_nvfp4(128, kBK), tmem + TM::sfaQ(1) + kk * 4,
                             tmem + TM::sfbK(0) + kk * 4, 1u);
            }
          }
        } else if (F8 && kind == KIND_LOW) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ss_w(d, smem_desc_sw128(sQL + kk * 32, 16, 1024), smem_desc_sw128(sk + kk * 32, 16, 1024),
                        idesc_f8(128, kBK), kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(sk + (kk >> 2) * (kBK * 128) + (kk & 3) * 32, 16, 1024);
            mma_f16_ts_w(d, tQ + kk * 8, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit_w(&bars[B_SR + (t & 1)]);
        tc_commit_w(&bars[B_KE + s]);
        return true;
      };
      // O += P(t) V(t)
      auto issue_pv = [&](int t) -> bool {
        const int g = t & 1, s = t % NV;
        if (!wait_all(&bars[B_PR + g], (t >> 1) & 1, 4)) return false;
        if (!wait_all(&bars[B_VF + s], (t / NV) & 1, 5)) return false;
        tc_fence_after();
        int kind, first, cnt;
        if constexpr (PK == 1)
          tile_of<kBK>(rp, t, kind, first);
        else
          tile_of_packed<PK>(rp, t, kind, first, cnt);
        const uint32_t sv = smem_u32(sm + L::oV + s * L::kStage);
        const uint32_t acc0 = t > 0 ? 1u : 0u;
        if (FP4 && (kind == KIND_LOW || kind == KIND_RES)) {
          const int ncopy = (RES && kind == KIND_RES) ? 2 : 1;
          const uint32_t pb = sv + L::oPinV;
          const uint32_t vside = smem_u32(sm + L::oVS + s * L::kVSide);
          for (int c = 0; c < ncopy; ++c) {
            const uint32_t psf = vside + L::NC * L::kSfBlk + c * L::kSfBlk, vsf = vside + c * L::kSfBlk;
            tc_cp_sf_w(tmem + TM::sfaP(c), smem_desc_rows16(psf));
            tc_cp_sf_w(tmem + TM::sfaP(c) + 4, smem_desc_rows16(psf + 512));
            tc_cp_sf_w(tmem + TM::sfbV(c), smem_desc_rows16(vsf));
            tc_cp_sf_w(tmem + TM::sfbV(c) + 4, smem_desc_rows16(vsf + 512));
          }
          // V^T copy c, keys 64 kk ..: 64-byte-swizzled rows of one 128-key
          // block, or (32-key blocks) the unswizzled 16-byte columns of two
          // blocks, 2048 bytes apart
          auto vdesc = [&](int c, int kk) -> uint64_t {
            if constexpr (PK == 1)
              return smem_desc_sw64(sv + c * L::kCodes + kk * 32);
            else
              return smem_desc_kmajor_noswz(sv + c * L::kCodes + kk * 4096, 2048, 128);
          };
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            mma_nvfp4_ss_w(tO, smem_desc_sw64(pb + kk * 32), vdesc(0, kk),
                         idesc_nvfp4(128, kD), tmem + TM::sfaP(0) + kk * 4,
                         tmem + TM::sfbV(0) + kk * 4, (acc0 || kk > 0) ? 1u : 0u);
            if (RES && kind == KIND_RES) {
              mma_nvfp4_ss_w(tO, smem_desc_sw64(pb + kk * 32), vdesc(1, kk),
                           idesc_nvfp4(128, kD), tmem + TM::sfaP(0) + kk * 4,
                           tmem + TM::sfbV(1) + kk * 4, 1u);
              mma_nvfp4_ss_w(tO, smem_desc_sw64(pb + L::kCodes + kk * 32), vdesc(0, kk),
                           idesc_nvfp4(128, kD), tmem + TM::sfaP(1) + kk * 4,
                           tmem + TM::sfbV(0) + kk * 4, 1u);
            }
          }
        } else if (F8 && kind == KIND_LOW) {
          const uint32_t pb = sv + L::oPinV;
          tc_cp_sf_w(tmem + TM::kSfbV8, smem_desc_rows16(smem_u32(sm + L::oVS + s * L::kVSide)));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_mxf8_ss_w(tO, smem_desc_sw128(pb + kk * 32, 16, 1024),
                        smem_desc_sw128(sv + kk * 32 * 128, 16, 1024), idesc_mxf8_bmn(128, kD),
                        tmem + TM::kSfaP8, tmem + TM::kSfbV8, (acc0 || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(sv + kk * 16 * 128, kBK * 128, 1024);
            mma_f16_ts_w(tO, tS0 + 128 * g + kk * 8, bd, idesc_pv, (acc0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit_w(&bars[B_PD + g]);
        tc_commit_w(&bars[B_VE + s]);
        return true;
      };
      // Issue order: S(0), S(1), then for each t: PV(t), S(t+2).  S(t+2)
      // writes the columns of S(t), where bf16 P(t) lives until PV(t) has
      // read it; issue order is execution order on the tensor pipe.  (Issuing
      // S(t+2) of NVFP4 / FP8 tiles early, as soon as the softmax holds S(t),
      // measured slower on whole layers: it delays the other group's PV.)
      for (int t = 0; ok && t < 2 && t < T; ++t) ok = issue_s(t);
      for (int t = 0; ok && t < T; ++t) {
        ok = issue_pv(t);
        if (ok && t + 2 < T) ok = issue_s(t + 2);
      }
      if (!ok) {
        tc_commit_w(&bars[B_DRAIN]);
        mbar_wait_drain(&bars[B_DRAIN], 0);
      }
    }
  } else if (warp < kSoftWarps) {
    // ===================== softmax groups =====================
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoft));
    const int g = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;                  // query row == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + TM::kS0 + 128 * g + lane_off;
    float* mrow = reinterpret_cast<float*>(sm + L::oM);  // [tile parity][row]
    float* xl = reinterpret_cast<float*>(sm + L::oX);    // [group][l, m][row]
    const float c2 = a.scale_log2;
    const float o_off = (float)a.p_offset;
    const float s_q8 = F8 ? a.q_s8[(int64_t)bh * a.nQb + qb] : 1.0f;
    const int nrows = min(a.bq, a.N - q0);
    if (g == 0) {
      // Q row r into TMEM columns [384, 448): the bf16 A operand of S = Q K^T
      uint32_t w[64];
      if (r < nrows) {
        const uint4* src = reinterpret_cast<const uint4*>(a.Q + (int64_t)b * a.sb + (int64_t)h * a.sh +
                                                          (int64_t)(q0 + r) * a.sn);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint4 v = src[i];
          w[4 * i] = v.x;
          w[4 * i + 1] = v.y;
          w[4 * i + 2] = v.z;
          w[4 * i + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) w[i] = 0u;
      }
      tmem_st32(tQ + lane_off, *reinterpret_cast<const uint32_t(*)[32]>(w));
      tmem_st32(tQ + lane_off + 32, *reinterpret_cast<const uint32_t(*)[32]>(w + 32));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_QR]);
    }
    // the ragged last key block (n < KB keys) and its position in the row's
    // list: the only skipped block whose pooled key does not weigh KB
    const int n_last = a.N - (a.nKb - 1) * KB;
    const float w_last = (float)n_last;
    // (only a skipped ragged block needs it, so only the skip segment of the
    // list is searched, 128 entries per round of loads; rows of 32-key blocks
    // keep the plain scan over the whole list, which measured faster there)
    int pos_last = -1000000;
    if (PK > 1 && n_last < KB) {
      for (int i0 = 0; i0 < a.nKb; i0 += 32) {
        const int i = i0 + lane;
        const unsigned bal = __ballot_sync(0xffffffffu, i < a.nKb && rp.list[i] == a.nKb - 1);
        if (bal) pos_last = i0 + __ffs(bal) - 1;
      }
    } else if (n_last < KB && rp.n_skip > 0) {
      const int s0 = rp.n_full + rp.n_res + rp.n_low, s1 = s0 + rp.n_skip;
      for (int i0 = s0; i0 < s1; i0 += 128) {
        int v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + 32 * u + lane;
          v[u] = i < s1 ? rp.list[i] : -1;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const unsigned bal = __ballot_sync(0xffffffffu, v[u] == a.nKb - 1);
          if (bal) pos_last = i0 + 32 * u + __ffs(bal) - 1;
        }
      }
    }
    float m_own = -INFINITY, l_own = 0.0f;   // this group's last max and its row sum
    bool ok = true;
    for (int t = g; t < T; t += 2) {
      ok = ok && mbar_wait(&bars[B_SR + g], (t >> 1) & 1, ctx, 6);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      int kind, first, cnt;
      float sqk = 1.0f;
      float x[128];
      if constexpr (PK == 1) {
        tile_of<kBK>(rp, t, kind, first);
        const int j = (kind == KIND_SKIP) ? 0 : rp.list[first];
        const int nv = (kind == KIND_SKIP) ? min(kBK, rp.n_skip - (first - kept)) : min(kBK, a.N - j * kBK);
        if (F8 && kind == KIND_LOW) sqk = s_q8 * a.k_s8[(int64_t)bh * a.nKb + j];
        tc_fence_after();
        {
          uint32_t raw[128];
#pragma unroll
          for (int c0 = 0; c0 < 128; c0 += 32) tmem_ld32_nw(tS + c0, raw + c0);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(raw[c]);
        }
        // columns past the skip chunk's end or past N in the ragged last block
        if (nv < 128) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= nv) x[c] = -INFINITY;
        }
      } else {
        tile_of_packed<PK>(rp, t, kind, first, cnt);
        int jsl[PK];
        if (kind != KIND_SKIP) pack_blocks<PK>(rp, first, cnt, jsl);
        tc_fence_after();
        {
          uint32_t raw[128];
#pragma unroll
          for (int c0 = 0; c0 < 128; c0 += 32) tmem_ld32_nw(tS + c0, raw + c0);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(raw[c]);
        }
        // columns without a real key: past the skip chunk's end, past N in
        // the ragged last block, and in slots past the tile's blocks
        if (kind == KIND_SKIP) {
          if (cnt < 128) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= cnt) x[c] = -INFINITY;
          }
        } else {
          int vs[PK];
          bool ragged = false;
#pragma unroll
          for (int i = 0; i < PK; ++i) {
            vs[i] = (i < cnt) ? min(KB, a.N - jsl[i] * KB) : 0;
            ragged |= vs[i] < KB;
          }
          if (ragged) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c % KB >= vs[c / KB]) x[c] = -INFINITY;
          }
        }
      }
      // maxima of the 8 groups of 16 columns (the NVFP4 scale groups), then of the row
      float gm[8];
#pragma unroll
      for (int gi = 0; gi < 8; ++gi) {
        const float* v = x + 16 * gi;
        const float a0 = fmax3(v[0], v[1], v[2]), a1 = fmax3(v[3], v[4], v[5]);
        const float a2 = fmax3(v[6], v[7], v[8]), a3 = fmax3(v[9], v[10], v[11]);
        const float a4 = fmax3(v[12], v[13], v[14]);
        gm[gi] = fmax3(fmax3(a0, a1, a2), fmax3(a3, a4, v[15]), -INFINITY);
      }
      const float tmax =
          fmaxf(fmax3(gm[0], gm[1], gm[2]), fmax3(fmax3(gm[3], gm[4], gm[5]), gm[6], gm[7])) * sqk;
      float m_in = -INFINITY;
      if (t > 0) {
        ok = mbar_wait(&bars[B_MX + (g ^ 1)], ((t - 1) >> 1) & 1, ctx, 7);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        m_in = mrow[(g ^ 1) * 128 + r];
      }
      const float m_new = fmaxf(m_in, tmax);
      mrow[g * 128 + r] = m_new;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_MX + g]);
      Tail q;
      q.c2t = c2 * sqk;
      q.mc = m_new * c2 - o_off;
      q.alpha = fast_exp2((m_in - m_new) * c2);
      q.t = t;
      q.last_col = (kind == KIND_SKIP) ? pos_last - first : -1;
      q.w_last = w_last;
      q.w_blk = (float)KB;
      q.bars = bars;
      q.ctx = ctx;
      q.sm = sm;
      q.tS = tS;
      q.tO = tO + lane_off;
      q.r = r;
      q.g = g;
      q.sc_tab = reinterpret_cast<const float2*>(sm + L::oSc);
      float psum = 0.0f;
      bool ok3;
      if (kind == KIND_SKIP) {
        ok3 = tail<T_SKIP, LM>(x, gm, q, psum);
      } else if (kind == KIND_FULL) {
        ok3 = tail<T_BF16, LM>(x, gm, q, psum);
      } else if constexpr (RES) {
        ok3 = (kind == KIND_RES) ? tail<T_RES, LM>(x, gm, q, psum) : tail<T_FP4, LM>(x, gm, q, psum);
      } else if constexpr (FP4) {
        ok3 = tail<T_FP4, LM>(x, gm, q, psum);
      } else if constexpr (F8) {
        ok3 = tail<T_F8, LM>(x, gm, q, psum);
      } else {
        ok3 = false;   // no low tier in this instance: not reached
      }
      l_own = l_own * fast_exp2((m_own - m_new) * c2) + psum;
      m_own = m_new;
      ok = ok3;
      if (!ok) break;
    }
    // epilogue: the group that ran the last tile waits for its PV; the row
    // sums of both groups are brought to the final maximum and combined;
    // group g writes O columns [64 g, 64 g + 64) of its row
    if (ok && T > 0 && g == ((T - 1) & 1)) {
      ok = mbar_wait(&bars[B_PD + g], ((T - 1) >> 1) & 1, ctx, 8);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    xl[(g * 2 + 0) * 128 + r] = l_own;
    xl[(g * 2 + 1) * 128 + r] = m_own;
    tc_fence_before();
    ok = bar_and2(1, 256, ok);
    tc_fence_after();
    if (ok) {
      const float la = xl[0 * 128 + r], ma = xl[1 * 128 + r];
      const float lb = xl[2 * 128 + r], mb = xl[3 * 128 + r];
      const float mf = fmaxf(ma, mb);
      const float lt = (la > 0.0f ? la * fast_exp2((ma - mf) * c2) : 0.0f) +
                       (lb > 0.0f ? lb * fast_exp2((mb - mf) * c2) : 0.0f);
      const float inv_l = 1.0f / lt;
      uint32_t raw[64];
      tmem_ld32_nw(tO + lane_off + 64 * g, raw);
      tmem_ld32_nw(tO + lane_off + 64 * g + 32, raw + 32);
      tmem_wait_ld();
      uint32_t w[32];
      const uint64_t il2 = pack2(inv_l, inv_l);
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float o0, o1;
        unpack2(mul2(pack2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), il2), o0, o1);
        w[c / 2] = pack_bf16(o0, o1);
      }
      if (r < nrows) {
        __nv_bfloat16* orow = a.O + (int64_t)b * a.sb + (int64_t)h * a.sh + (int64_t)(q0 + r) * a.sn + 64 * g;
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(orow + v * 8) = make_uint4(w[v * 4], w[v * 4 + 1], w[v * 4 + 2], w[v * 4 + 3]);
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

template <int LM, int KB>
cudaError_t launch2(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t s) {
  using L = Lay<LM>;
  auto k = attn2_kernel<LM, KB>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nQb, a.B * a.H);
  k<<<grid, kThreads2, L::kTotal, s>>>(a, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6],
                                       maps[7], maps[8]);
  return cudaGetLastError();
}

}  // namespace

// d = 128 with 128-query blocks and 128-key tiles: every low format this
// kernel has a tail for; 32-key blocks (four to a tile) for the bf16 and
// NVFP4 tiers.  Returns cudaErrorNotSupported for shapes it does not cover.
cudaError_t launch_attn2(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t s) {
  if (a.d != 128 || a.bq != 128) return cudaErrorNotSupported;
  if (a.bk == 32) {
    if (a.low == TA_LOW_NONE) return launch2<LM_IMAGE, 32>(a, maps, s);
    if (a.low == TA_LOW_NVFP4) return launch2<LM_NVFP4, 32>(a, maps, s);
    if (a.low == TA_LOW_NVFP4_RES) return launch2<LM_NVFP4_RES, 32>(a, maps, s);
    return cudaErrorInvalidValue;   // no other kernel takes 32-key blocks   // no other kernel takes 32-key blocks
  }
  if (a.bk != 128) return cudaErrorNotSupported;
  // NVFP4 + residual layers tiered by thresholds (mass or entropy router) mix
  // full, residual, NVFP4 and skipped blocks in every row; there the 16-warp
  // kernel measured faster (720p layer 120 vs 139 ms; the 480p shape with the
  // same four tiers 13.6 vs 17.2 ms), while this kernel wins on each tier
  // alone, on mixes without skipped blocks and on the price router's rows
  // (480p price layer 11.6 vs 12.3 ms)
  if (a.low == TA_LOW_NVFP4_RES && a.router != TA_ROUTER_PRICE) return cudaErrorNotSupported;
  if (a.low == TA_LOW_NONE) return launch2<LM_IMAGE, 128>(a, maps, s);
  if (a.low == TA_LOW_NVFP4) return launch2<LM_NVFP4, 128>(a, maps, s);
  if (a.low == TA_LOW_NVFP4_RES) return launch2<LM_NVFP4_RES, 128>(a, maps, s);
  if (a.low == TA_LOW_FP8_E4M3) return launch2<LM_FP8, 128>(a, maps, s);
  return cudaErrorNotSupported;
}

}  // namespace ta
