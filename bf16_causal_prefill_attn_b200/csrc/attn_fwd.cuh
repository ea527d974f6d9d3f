// Forward causal (prefill) attention on sm_100a: TMA-fed tcgen05 MMAs with TMEM
// accumulators, warp-specialised, two query tiles per CTA in ping-pong.
//
// Computes O = softmax(mask(Q K^T * scale)) V (the forward causal attention of the
// prefill phase, [ZYFA-fr] "Ce que couvrent les noyaux") in two precisions:
//   BF16  S = Q K^T (kind::f16, fp32 accumulate); P = exp2((S - M) * scale * log2 e) in
//         fp32 (three quarters on the MUFU, one quarter by a polynomial on the FMA pipe),
//         rounded to bf16 for O += P V; the row sum is accumulated in fp32.
//   FP8   S = Q K^T on e4m3 codes (kind::f8f6f4); P is produced without an exponential by
//         the lean-P encoding ([ZYFA-mb] "Como o motor de atenção FP8 da Zyphra
//         funciona": a multiply-add and an integer conversion write the e4m3 bit pattern);
//         each 64-key block carries a power-of-two shift that the block-scaled MMA
//         (kind::mxf8f6f4.block_scale, UE8M0 scale per 32 keys) removes, and the row
//         normaliser is the sum of the rounded probabilities, formed by one extra MMA per
//         key tile against a matrix of ones.
//
// A work unit is two 128-row query tiles (slots t = 0, 1) that share every K/V tile in
// shared memory: rows [256 p + 128 t, +128) of query-tile pair p of one (batch, head), or
// (head pairs) one query tile of two query heads of one kv group.  Units are numbered
// longest first.  A CTA runs a sequence of units, which its K/V producer publishes to the
// other roles through a small queue in shared memory: unit blockIdx.x, then either a static
// list (rounds of gridDim.x units, alternate rounds in reverse CTA order) or, with one CTA
// launched per unit, the units of CTAs that have not started yet, taken over with cluster
// launch control (clusterlaunchcontrol.try_cancel) -- dynamic longest-first scheduling.
// When a CTA runs several units, its setup is paid once and each slot's epilogue overlaps
// the other slot's work and the next unit's first S.  All barrier phases are running counts.
// Roles (384 threads, 12 warps):
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1: thread r of the group owns
//               query row r (TMEM lane r); reads S, updates the reference max (lazily:
//               only when the tile max exceeds it by more than the headroom), rescales O
//               in TMEM when it does, writes P (BF16: into TMEM, over the S columns it has
//               consumed or, S-ahead, into columns of its own; FP8: into shared memory,
//               with its scale factors in TMEM), and finally writes O and lse;
//   warp 8      TMA producer of K and V (NK / NV stages, continuing across units) and the
//               CTA's scheduler (publishes each unit to the other roles);
//   warp 9      MMA issuer (warp-wide control flow, one elected lane issues).  One tile's
//               softmax overlaps the other tile's MMAs (ping-pong).  Two pipelines:
//                 S-ahead (FP8; BF16 with BSA): warp 9 issues S_t(j+1) as soon as both
//                       slots have read their latest S (S_t(j+1) only needs S_t(j) read into
//                       registers, so it runs during the softmax of S_t(j): each softmax
//                       group has a whole period, not half, for its tile), warp 10 PV_t(j);
//                 P over S (BF16 without BSA): warp 9 issues PV_0(j), S_0(j+1), PV_1(j),
//                       S_1(j+1) (P_t aliases S_t, so S_t(j+1) must follow PV_t(j));
//   warp 10     S-ahead: PV MMA issuer; otherwise idle;
//   warp 11     TMEM allocator, then the Q loader: slot t's Q tile of the next unit as soon
//               as the slot's last S MMA of the current unit has completed (q_empty).
// TMEM (512 columns x 128 lanes, see TmemMap):
//   BF16  P over S: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512); P_t (bf16,
//         64 columns) overwrites the first columns of S_t.  S-ahead: S [0,128) shared by
//         both slots in turn, P_0 [128,192), P_1 [192,256), O_0 [256,384), O_1 [384,512).
//   FP8   O_0 [0,144), O_1 [160,304): the PV MMA has N = 144, V extended by a 16-column
//         block of ones, so columns 128..143 accumulate the row sum of the rounded P with
//         the same block scales (the "extra matrix instruction" costs no extra issue);
//         scale factors of P_0, P_1 at [144,148), [148,152), the constant scale factors
//         of V at [152,160); S_0 [320,448), S_1 [384,512) overlap in [384,448), so an S
//         MMA is issued only after both softmax groups have read their latest S (s_read
//         barriers).  P_t (128 x 128 e4m3) is in shared memory in the K-major 128-byte
//         swizzled layout of an MMA A operand.
//
// Every wait is bounded (mbar_wait): on expiry the CTA records DEV_TIMEOUT and unwinds.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace attn {

constexpr int BLOCK_M = 128;
constexpr int BLOCK_N = 128;
constexpr int DV = 128;
constexpr int NUM_THREADS = 384;
// Registers per thread after setmaxnreg: warps 0-7 (softmax) and warps 8-11 (producer, MMA
// issuers, Q loader), per pipeline -- SAHEAD (the S MMAs a key tile ahead of the PV MMAs,
// on an issuing warp of their own: FP8, and BF16 with BSA) needs more in the issuing warps
// for their unit-loop state; the other (BF16: one warp issues PV_t(j) then S_t(j+1)) gives
// the BF16 softmax more for its exponentials.
template <bool SAHEAD> struct RegSplit {
  static constexpr int SOFTMAX = SAHEAD ? 200 : 208;
  static constexpr int OTHER = SAHEAD ? 104 : 88;
};
// registers per thread the launch must provide at least for either split
constexpr int regs_needed_at_launch(int softmax, int other) {
  return (2 * 128 * softmax + 128 * other + NUM_THREADS - 1) / NUM_THREADS;
}
constexpr int REGS_NEEDED_AT_LAUNCH =
    regs_needed_at_launch(RegSplit<true>::SOFTMAX, RegSplit<true>::OTHER) >
            regs_needed_at_launch(RegSplit<false>::SOFTMAX, RegSplit<false>::OTHER)
        ? regs_needed_at_launch(RegSplit<true>::SOFTMAX, RegSplit<true>::OTHER)
        : regs_needed_at_launch(RegSplit<false>::SOFTMAX, RegSplit<false>::OTHER);
static_assert(REGS_NEEDED_AT_LAUNCH * NUM_THREADS <= 65536, "register split exceeds the SM");
// TMEM column map per precision (see the layout above)
template <bool FP8, bool SAHEAD>
struct TmemMap {
  // BF16 with SAHEAD: one S buffer for both slots (S_0 and S_1 alternate in it), P_t of its
  // own; BF16 otherwise: S_t of its own, P_t written over the first 64 columns of S_t
  __host__ __device__ static constexpr uint32_t S(int t) {
    return FP8 ? 320u + 64u * t : (SAHEAD ? 0u : 128u * t);
  }
  __host__ __device__ static constexpr uint32_t O(int t) { return FP8 ? 160u * t : 256u + 128u * t; }
  __host__ __device__ static constexpr uint32_t P(int t) {  // BF16 only
    return SAHEAD ? 128u + 64u * t : 128u * t;
  }
  __host__ __device__ static constexpr uint32_t SFA(int t) { return 144u + 4u * t; }  // FP8, 4 columns
  static constexpr uint32_t SFB = 152;                         // FP8, 8 columns
  static constexpr uint32_t RS = 128;                          // row-sum column of O(t)
  static constexpr uint32_t PV_N = FP8 ? 144 : 128;
};
constexpr int UQ = 4;  // depth of a CTA's queue of work units (producer -> other roles)
constexpr float LEANP_MAGIC = 12582912.0f;  // 1.5 * 2^23
constexpr int LEANP_KMAX = 16;
constexpr int LEANP_TOP = 112;       // code of a block maximum at the reference
constexpr int LEANP_HEADROOM = 14;   // 126 - LEANP_TOP
constexpr float BF16_HEADROOM = 24.0f;  // log2 units the reference max may lag the true max

// 2^f on [-0.5, 0.5], degree 3, coefficients fitted here to minimise the relative error
// (max 7.5e-5, well under the bf16 rounding of P)
constexpr float EXP2_C0 = 0.99992817640304565f;
constexpr float EXP2_C1 = 0.69326096773147583f;
constexpr float EXP2_C2 = 0.24260970950126648f;
constexpr float EXP2_C3 = 0.05517097562551498f;

struct FwdParams {
  int B, S, Hq, Hkv, G;
  int n_q_tiles, n_pairs;  // VARLEN: of the longest sequence (max_seqlen); n_pairs = units
                           // along the queries (query-tile pairs, or query tiles with head_pairs)
  int n_units;             // n_pairs * B * (head_pairs ? Hq / 2 : Hq)
  int dynamic;             // 1: one CTA launched per unit, running CTAs take the units of
                           // CTAs not yet started (cluster launch control); 0: static list
  int head_pairs;          // 1: a CTA's two slots are two query heads of one kv group at the
                           // same query tile (Hq / Hkv even); 0: two query tiles of one head
  int causal;
  // VARLEN: sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1]) of the packed tensors
  // (null: every sequence has S tokens, sequence b starting at token b S), at most
  // max_seqlen long; total_tokens bounds every token index written
  const int* cu_seqlens;
  int max_seqlen;
  int64_t total_tokens;
  __nv_bfloat16* o;   // [B, S, Hq, DV]
  float* lse;         // [B, Hq, S] or null
  float c1;           // BF16: scale * log2(e)
  double leanp_c;     // FP8: 8 * log2(e) * scale  (slope a = c * dq * dk)
  const float* descale_q;
  const float* descale_k;
  const float* descale_v;
  int unrotate;       // apply x H / sqrt(128) to each output row (Hadamard-rotated V)
  uint32_t* err;
  uint64_t timeout_ns;
  int stall_tile;        // test-only: the producer stops before this key tile (-1: never)
  float* dump_s;         // FP8 debug: raw scores [B, Hq, S, S]
  uint8_t* dump_codes;   // FP8 debug: P codes   [B, Hq, S, S]
  uint8_t* dump_kshift;  // FP8 debug: shifts    [B, Hq, S, S/64]
};

template <bool FP8, int DQK>
struct FwdCfg {
  static constexpr int E = FP8 ? 1 : 2;                         // bytes per element
  static constexpr int BOX_COLS = 128 / E;                      // elements per 128-B row
  static constexpr int Q_BOXES = (DQK * E + 127) / 128;         // 128-B column boxes
  static constexpr int V_BOXES = DV * E / 128;
  static constexpr int BOX_BYTES = 128 * 128;                   // 128 rows x 128 B
  static constexpr int Q_BYTES = Q_BOXES * BOX_BYTES;
  static constexpr int K_BYTES = Q_BYTES;
  static constexpr int V_BYTES = V_BOXES * BOX_BYTES;
  static constexpr int NK = FP8 ? (DQK == 128 ? 4 : 2) : 2;     // K ring depth
  static constexpr int NV = FP8 ? (DQK == 128 ? 4 : 2) : (DQK == 128 ? 2 : 1);
  static constexpr int KSTEP = FP8 ? 32 : 16;                   // MMA K per instruction
  static constexpr int QK_STEPS = DQK / KSTEP;
  static constexpr int PV_STEPS = BLOCK_N / KSTEP;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * K_BYTES;
  static constexpr int OFF_ONES = OFF_V + NV * V_BYTES;  // FP8: 128 keys x 128 B of 1.0
  static constexpr int OFF_P = OFF_ONES + (FP8 ? BOX_BYTES : 0);  // FP8: P_0, P_1
  // O leaves through shared memory and a TMA store (64 columns, 16 KB per slot at a time):
  // FP8 stages in P_t (free once the slot's last PV has completed); BF16 with d_qk = 128
  // has a staging area of its own; BF16 with d_qk = 192 has no room and stores rows directly
  static constexpr bool TMA_O = FP8 || DQK == 128;
  // BF16: each softmax warp stores its own 32 rows (no warp waits for another; measured
  // faster); FP8: one thread per slot stores 128 rows (the per-warp form measured slower
  // there: the FP8 softmax sits at its register limit)
  static constexpr bool WARP_O = !FP8;
  static constexpr int O_BOX_ROWS = WARP_O ? 32 : 128;
  static constexpr int OFF_OST = OFF_P;                        // slot t at OFF_OST + t BOX_BYTES
  static constexpr int OFF_BAR = OFF_P + (TMA_O ? 2 * BOX_BYTES : 0);
  // barriers: k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], per slot q_full, q_empty,
  //           s_full, p_full, pv_done, s_read, mma_done, then unit_full[UQ],
  //           unit_empty[UQ], the launch-control barrier and per slot the O-staging
  //           barrier
  static constexpr int NUM_BARS = 2 * NK + 2 * NV + 2 * 7 + 2 * UQ + 1 + 2;
  // unit queue: UQ entries of 12 ints (the unit, its status, the decoded Unit)
  static constexpr int UQ_INTS = 12;
  static constexpr int OFF_UNITQ = (OFF_BAR + NUM_BARS * 8 + 15) / 16 * 16;
  static constexpr int OFF_CLC = OFF_UNITQ + UQ * UQ_INTS * 4;         // 16-byte response
  static constexpr int OFF_TMEMPTR = OFF_CLC + 16;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;           // 1024-B alignment slack
  static_assert(SMEM_ALLOC <= 232448, "shared memory per block exceeded");
  static constexpr uint32_t IDESC_S =
      idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, 0u, 0u, BLOCK_M, BLOCK_N);
  static constexpr uint32_t IDESC_PV_BF16 = idesc_dense(1u, 1u, 0u, 1u, BLOCK_M, DV);
};

// k_b: power-of-two shift of one 64-key block (block max mu, reference m in code units)
__device__ __forceinline__ int leanp_kshift(float mu, float a, int m) {
  float t = __fmaf_rn(mu, a, -__int2float_rn(m));
  float g = -t * 0.125f;
  int k = __float2int_rd(g);  // saturating: +inf -> INT_MAX
  return min(max(k, 0), LEANP_KMAX);
}

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for x <= BF16_HEADROOM on the FMA pipe: x = n + f, f in [-0.5, 0.5], 2^f by the polynomial,
// 2^n added to the exponent field.  Inputs below -125 give 2^-125.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float j = __fadd_rn(x, LEANP_MAGIC);   // round to the nearest integer n
  const float n = __fsub_rn(j, LEANP_MAGIC);
  const float f = __fsub_rn(x, n);
  float p = __fmaf_rn(EXP2_C3, f, EXP2_C2);
  p = __fmaf_rn(p, f, EXP2_C1);
  p = __fmaf_rn(p, f, EXP2_C0);
  // low bits of j hold n (two's complement); n << 23 added to the exponent of p
  return __int_as_float(__float_as_int(j) * (1 << 23) + __float_as_int(p));
}

// Two lanes of exp2_poly with the packed two-wide fp32 instructions of sm_100 (per lane the
// same operations and roundings as exp2_poly, so the same results bit for bit).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 j = __fadd2_rn(x, make_float2(LEANP_MAGIC, LEANP_MAGIC));
  const float2 n = __fadd2_rn(j, make_float2(-LEANP_MAGIC, -LEANP_MAGIC));
  const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
  float2 q = __ffma2_rn(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
  q = __ffma2_rn(q, f, make_float2(EXP2_C1, EXP2_C1));
  q = __ffma2_rn(q, f, make_float2(EXP2_C0, EXP2_C0));
  return make_float2(__int_as_float(__float_as_int(j.x) * (1 << 23) + __float_as_int(q.x)),
                     __int_as_float(__float_as_int(j.y) * (1 << 23) + __float_as_int(q.y)));
}

// One work unit: its sequence and the query tiles / heads of its two slots.
struct Unit {
  int b, h, g;        // batch, query head of slot 0 (slot 1: h + 1 with head pairs), kv head
  int tok0, seq_len;  // first token and length of the sequence
  int qt0, qt1;       // query tile of each slot
  int n_t0, n_t1;     // key tiles of each slot (0: the slot has no query tile in this unit)
};

// Unit u (0 = the longest).  Returns 1, 0 if the unit has no query tile in its sequence
// (packed sequences shorter than the longest), -1 if the sequence bounds are invalid.
template <bool VARLEN>
__device__ __forceinline__ int unit_info(const FwdParams& p, int u, Unit& U) {
  const bool hp = p.head_pairs != 0;
  const int heads_per_unit = hp ? p.Hq / 2 : p.Hq;
  const int nbh = p.B * heads_per_unit;
  const int pr = p.n_pairs - 1 - u / nbh;
  const int bh = u % nbh;
  U.b = bh / heads_per_unit;
  U.h = hp ? 2 * (bh % heads_per_unit) : bh % heads_per_unit;
  U.g = U.h / p.G;
  U.tok0 = U.b * p.S;
  U.seq_len = p.S;
  int n_q_tiles = p.n_q_tiles;
  if constexpr (VARLEN) {
    if (p.cu_seqlens != nullptr) {
      const int c0 = __ldg(p.cu_seqlens + U.b), c1 = __ldg(p.cu_seqlens + U.b + 1);
      if (c0 < 0 || c1 < c0 || static_cast<int64_t>(c1) > p.total_tokens ||
          c1 - c0 > p.max_seqlen)
        return -1;
      U.tok0 = c0;
      U.seq_len = c1 - c0;
    }
    n_q_tiles = (U.seq_len + BLOCK_M - 1) / BLOCK_M;
    if ((hp ? pr : 2 * pr) >= n_q_tiles) return 0;
  }
  U.qt0 = hp ? pr : 2 * pr;
  U.qt1 = hp ? pr : 2 * pr + 1;
  const bool has1 = U.qt1 < n_q_tiles;
  U.n_t0 = p.causal ? U.qt0 + 1 : n_q_tiles;
  U.n_t1 = has1 ? (p.causal ? U.qt1 + 1 : n_q_tiles) : 0;
  return 1;
}

// The k-th unit of this CTA: round k holds units [k G, (k+1) G) (G = gridDim.x), taken in
// CTA order in even rounds and in reverse CTA order in odd rounds, which evens out the
// decreasing unit lengths.  Every role of the CTA walks the same list.
__device__ __forceinline__ int cta_unit(int k) {
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// EXACT (FP8 only): the exact-P ablation -- P = e4m3_rn(2^((a s - m)/8 + 7 + k_b)) by the
// MUFU exponential and the hardware e4m3 conversion, instead of the lean-P multiply-add and
// integer conversion; everything else (reference max, block shifts, block-scaled PV, row
// sum) is shared.
// VARLEN: sequences of any length (packed, or a fixed S not a multiple of 128): keys past
// the end of the sequence are masked, rows past it are not written.
// tm_o: O [tokens, Hq, 128] bf16, boxes of 64 columns x C::O_BOX_ROWS rows (FP8 128, BF16
// 32) with the 128-byte swizzle
// (used when C::TMA_O and not VARLEN).
// BSA (BF16 only): the S-ahead pipeline of FP8 -- warp 9 issues S_t(j+1) as soon as both
// slots have read their latest S (they alternate in one S buffer), warp 10 issues PV_t(j)
// from P_t in TMEM columns of its own.  Without it one warp issues PV_t(j) then S_t(j+1)
// (P_t is written over S_t).  Results are the same bits either way.
template <bool FP8, int DQK, bool DUMP, bool EXACT = false, bool VARLEN = false, bool BSA = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using C = FwdCfg<FP8, DQK>;
  constexpr bool SAHEAD = FP8 || BSA;
  using TM = TmemMap<FP8, SAHEAD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + C::NK;
  uint64_t* v_full = k_empty + C::NK;
  uint64_t* v_empty = v_full + C::NV;
  uint64_t* tbar = v_empty + C::NV;  // per slot: 7 barriers
  auto q_full = [&](int t) { return tbar + 7 * t + 0; };
  auto q_empty = [&](int t) { return tbar + 7 * t + 1; };
  auto s_full = [&](int t) { return tbar + 7 * t + 2; };
  auto p_full = [&](int t) { return tbar + 7 * t + 3; };
  auto pv_done = [&](int t) { return tbar + 7 * t + 4; };
  auto s_read = [&](int t) { return tbar + 7 * t + 5; };
  auto mma_done = [&](int t) { return tbar + 7 * t + 6; };
  uint64_t* unit_full = tbar + 14;       // [UQ] unit index published by the producer
  uint64_t* unit_empty = unit_full + UQ;  // [UQ] read by every consumer warp
  uint64_t* clc_bar = unit_empty + UQ;   // launch-control response landed
  uint64_t* o_sync = clc_bar + 1;        // [2] the four warps of slot t at the O staging
  int* unit_q = reinterpret_cast<int*>(smem + C::OFF_UNITQ);
  void* clc_resp = smem + C::OFF_CLC;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEMPTR);
  // warps that read the unit queue: the Q loader, the MMA warps and the softmax warps
  constexpr int UNIT_CONSUMERS = 1 + (SAHEAD ? 2 : 1) + 8;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool hp = p.head_pairs != 0;

  if (tid == 0) {
    for (int i = 0; i < C::NK; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < C::NV; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(q_full(t), 1);
      mbar_init(q_empty(t), 1);
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 128);
      mbar_init(pv_done(t), 1);
      mbar_init(s_read(t), 128);
      mbar_init(mma_done(t), 1);
    }
    for (int i = 0; i < UQ; ++i) {
      mbar_init(unit_full + i, 1);
      mbar_init(unit_empty + i, UNIT_CONSUMERS);
    }
    mbar_init(clc_bar, 1);
    mbar_init(o_sync + 0, 4);  // FP8 only
    mbar_init(o_sync + 1, 4);
    fence_barrier_init();
  }
  if (warp == 11) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (C::TMA_O && !VARLEN) tma_prefetch_desc(&tm_o);
  }
  if constexpr (FP8) {
    // the ones block (e4m3 1.0 = 0x38) that extends every V tile to N = 144 for the row
    // sum; written once, visible to the async proxy
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::OFF_ONES);
    for (int i = tid; i < C::BOX_BYTES / 4; i += NUM_THREADS) ones[i] = 0x38383838u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  // the k-th unit of this CTA from the queue (warp-wide; u = -1: no more units), decoded
  // once by the producer: st is unit_info's result, U its unit; false if the wait ran out.
  // Without `release` the caller keeps the entry (and may read it again) until
  // release_unit(k).
  auto take_unit = [&](int k, int& u, int& st, Unit& U, bool release = true) -> bool {
    const int slot = k % UQ;
    const bool r = mbar_wait(unit_full + slot, (k / UQ) & 1, p.err, p.timeout_ns);
    if (!__all_sync(0xffffffffu, r)) return false;
    // scalar loads: a role's unused fields are never loaded
    const int* e = unit_q + slot * C::UQ_INTS;
    u = e[0];
    st = e[1];
    U.b = e[2];
    U.h = e[3];
    U.g = e[4];
    U.tok0 = e[5];
    U.seq_len = e[6];
    U.qt0 = e[7];
    U.qt1 = e[8];
    U.n_t0 = e[9];
    U.n_t1 = e[10];
    __syncwarp();
    if (release && lane == 0) mbar_arrive(unit_empty + slot);
    return true;
  };
  auto release_unit = [&](int k) {
    __syncwarp();
    if (lane == 0) mbar_arrive(unit_empty + k % UQ);
  };

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<SAHEAD>::OTHER));
    // Q is read once (evicted first); K and V are read by every CTA of the kv group and
    // of later query tiles (kept in L2 longest)
    if (warp == 8) {
      // ----------------------------------------------------------- K/V producer (warp-wide,
      // one elected lane issues); gk / gv count the tiles issued by this CTA.  It also
      // schedules the CTA: it publishes each unit in the queue before loading its tiles.
      // The first unit is the CTA's own; the next one comes from the static list, or
      // (dynamic) from a CTA of the launch that has not started yet, requested once this
      // unit's last tiles are being loaded (so units are taken longest first, as late as
      // possible).
      const uint64_t pol_keep = l2_policy_evict_last();
      bool ok = true;
      int gk = 0, gv = 0;
      int n_req = 0;         // launch-control responses received
      bool pending = false;  // a request whose response has not been waited for
      auto request = [&]() {
        if (elect_one()) {
          mbar_arrive_expect_tx(clc_bar, 16);
          clc_try_cancel(clc_resp, clc_bar);
        }
        __syncwarp();
        pending = true;
      };
      int u = cta_unit(0);
      for (int k = 0; ok; ++k) {
        if (u >= p.n_units) u = -1;
        const int slot = k % UQ;
        if (k >= UQ) ok = mbar_wait(unit_empty + slot, ((k / UQ) - 1) & 1, p.err, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
        Unit U = {};
        const int st = u >= 0 ? unit_info<VARLEN>(p, u, U) : 0;
        if (lane == 0) {
          int4* e = reinterpret_cast<int4*>(unit_q + slot * C::UQ_INTS);
          e[0] = make_int4(u, st, U.b, U.h);
          e[1] = make_int4(U.g, U.tok0, U.seq_len, U.qt0);
          e[2] = make_int4(U.qt1, U.n_t0, U.n_t1, 0);
          mbar_arrive(unit_full + slot);
        }
        __syncwarp();
        if (u < 0) break;
        const int n_max = st > 0 ? max(U.n_t0, U.n_t1) : 0;
        if constexpr (FP8 || !BSA) {
          for (int j = 0; j < n_max; ++j) {
            if (j == p.stall_tile) {  // test-only: the waits on this tile must run out
              ok = false;
              break;
            }
            const int sk = gk % C::NK;
            if (gk >= C::NK) ok = mbar_wait(k_empty + sk, ((gk / C::NK) - 1) & 1, p.err, p.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (elect_one()) {
              mbar_arrive_expect_tx(k_full + sk, C::K_BYTES);
              for (int i = 0; i < C::Q_BOXES; ++i)
                tma_load_3d_hint(smem + C::OFF_K + sk * C::K_BYTES + i * C::BOX_BYTES, &tm_k,
                                 k_full + sk, i * C::BOX_COLS, U.g, U.tok0 + j * BLOCK_N, pol_keep);
            }
            __syncwarp();
            ++gk;
            const int sv = gv % C::NV;
            if (gv >= C::NV) ok = mbar_wait(v_empty + sv, ((gv / C::NV) - 1) & 1, p.err, p.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (elect_one()) {
              mbar_arrive_expect_tx(v_full + sv, C::V_BYTES);
              for (int i = 0; i < C::V_BOXES; ++i)
                tma_load_3d_hint(smem + C::OFF_V + sv * C::V_BYTES + i * C::BOX_BYTES, &tm_v,
                                 v_full + sv, i * C::BOX_COLS, U.g, U.tok0 + j * BLOCK_N, pol_keep);
            }
            __syncwarp();
            ++gv;
            if (p.dynamic && j == n_max - 1) request();
          }
        } else {
          // BF16 S-ahead: K leads V by a tile.  S_t(j+1) needs K(j+1) about a tile
          // before PV_t(j) needs V(j), and with two-stage rings a V load waiting for its slot
          // would otherwise hold the next K load back
          constexpr int KLEAD = 1;
          for (int i = 0; i < n_max + KLEAD; ++i) {
            if (i < n_max) {
              const int j = i;
              if (j == p.stall_tile) {  // test-only: the waits on this tile must run out
                ok = false;
                break;
              }
              const int sk = gk % C::NK;
              if (gk >= C::NK) ok = mbar_wait(k_empty + sk, ((gk / C::NK) - 1) & 1, p.err, p.timeout_ns);
              if (!__all_sync(0xffffffffu, ok)) break;
              if (elect_one()) {
                mbar_arrive_expect_tx(k_full + sk, C::K_BYTES);
                for (int b = 0; b < C::Q_BOXES; ++b)
                  tma_load_3d_hint(smem + C::OFF_K + sk * C::K_BYTES + b * C::BOX_BYTES, &tm_k,
                                   k_full + sk, b * C::BOX_COLS, U.g, U.tok0 + j * BLOCK_N, pol_keep);
              }
              __syncwarp();
              ++gk;
            }
            if (i >= KLEAD) {
              const int j = i - KLEAD;
              const int sv = gv % C::NV;
              if (gv >= C::NV) ok = mbar_wait(v_empty + sv, ((gv / C::NV) - 1) & 1, p.err, p.timeout_ns);
              if (!__all_sync(0xffffffffu, ok)) break;
              if (elect_one()) {
                mbar_arrive_expect_tx(v_full + sv, C::V_BYTES);
                for (int b = 0; b < C::V_BOXES; ++b)
                  tma_load_3d_hint(smem + C::OFF_V + sv * C::V_BYTES + b * C::BOX_BYTES, &tm_v,
                                   v_full + sv, b * C::BOX_COLS, U.g, U.tok0 + j * BLOCK_N, pol_keep);
              }
              __syncwarp();
              ++gv;
            }
          }
        }
        if (!ok) break;
        if (p.dynamic) {
          if (!pending) request();
          ok = mbar_wait(clc_bar, n_req & 1, p.err, p.timeout_ns);
          if (!__all_sync(0xffffffffu, ok)) break;
          ++n_req;
          pending = false;
          int x = -1;
          u = clc_query(clc_resp, &x) ? x : -1;  // -1: no CTA left to take; no more requests
        } else {
          u = cta_unit(k + 1);
        }
      }
      // a request in flight writes shared memory: its response must land before exit
      if (pending) mbar_wait(clc_bar, n_req & 1, p.err, DRAIN_TIMEOUT_NS, false);
      // drain: no copy issued by this CTA may still be in flight at exit
      for (int i = (gk > C::NK ? gk - C::NK : 0); i < gk; ++i)
        mbar_wait(k_full + i % C::NK, (i / C::NK) & 1, p.err, DRAIN_TIMEOUT_NS, false);
      for (int i = (gv > C::NV ? gv - C::NV : 0); i < gv; ++i)
        mbar_wait(v_full + i % C::NV, (i / C::NV) & 1, p.err, DRAIN_TIMEOUT_NS, false);
    } else if (warp == 11) {
      // ----------------------------------------------------------- Q loader: slot t's tile
      // of each unit once the slot's last S MMA of its previous unit has completed
      const uint64_t pol_once = l2_policy_evict_first();
      bool ok = true;
      int nq[2] = {0, 0};  // Q tiles loaded per slot
      for (int k = 0; ok; ++k) {
        int u = -1, st = 0;
        Unit U;
        ok = take_unit(k, u, st, U);
        if (!ok || u < 0) break;
        if (st <= 0) continue;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if ((t ? U.n_t1 : U.n_t0) == 0) continue;
          if (nq[t] > 0) ok = mbar_wait(q_empty(t), (nq[t] - 1) & 1, p.err, p.timeout_ns);
          if (!__all_sync(0xffffffffu, ok)) break;
          if (elect_one()) {
            mbar_arrive_expect_tx(q_full(t), C::Q_BYTES);
            for (int i = 0; i < C::Q_BOXES; ++i)
              tma_load_3d_hint(smem + C::OFF_Q + t * C::Q_BYTES + i * C::BOX_BYTES, &tm_q,
                               q_full(t), i * C::BOX_COLS, hp ? U.h + t : U.h,
                               U.tok0 + (t ? U.qt1 : U.qt0) * BLOCK_M, pol_once);
          }
          __syncwarp();
          ++nq[t];
        }
      }
      for (int t = 0; t < 2; ++t)
        if (nq[t] > 0) mbar_wait(q_full(t), (nq[t] - 1) & 1, p.err, DRAIN_TIMEOUT_NS, false);
    } else if (warp == 9 || (SAHEAD && warp == 10)) {
      // ----------------------------------------------------------- MMA issuers (warp-wide
      // control flow, one elected lane issues); the order per key tile is in the header.
      // FP8: warp 9 issues the S MMAs, warp 10 the PV MMAs (they touch disjoint TMEM
      // columns and P is in shared memory, so only mbarriers order them), so that one
      // warp's waits and control flow overlap the other warp's issue.  BF16: warp 9 issues
      // both (P_t aliases S_t, so S_t(j+1) must follow PV_t(j) in one issue stream).
      // Descriptors are built once; advancing an operand by `off` bytes adds off >> 4 to
      // the start-address field (shared-memory addresses stay below 2^18, so the 14-bit
      // field never carries into its neighbours).
      const uint64_t dq0 = smem_desc_sw128(smem_addr(smem + C::OFF_Q), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_addr(smem + C::OFF_K), 16, 1024);
      const uint64_t dp0 = smem_desc_sw128(smem_addr(smem + C::OFF_P), 16, 1024);  // FP8
      auto v_desc = [&](int sv) -> uint64_t {
        const uint32_t va = smem_addr(smem + C::OFF_V + sv * C::V_BYTES);
        if constexpr (FP8) {
          // N = 144: the 128 d-columns of V, then the ones block one leading offset away
          return smem_desc_sw128(va, smem_addr(smem + C::OFF_ONES) - va, 1024);
        } else {
          return smem_desc_sw128(va, C::BOX_BYTES, 1024);  // two 64-column atoms of V
        }
      };
      // S_t(j) of a unit whose key tiles start at ring position g0; commits s_full, q_empty
      // after the slot's last S of the unit, and k_empty after the tile's last S (slot 1's,
      // or slot 0's where slot 1 does not use the tile)
      auto issue_s = [&](int t, int j, int g0, const Unit& U) {
        const int sk = (g0 + j) % C::NK;
        const uint64_t qd = dq0 + static_cast<uint32_t>((t * C::Q_BYTES) >> 4);
        const uint64_t kd = dk0 + static_cast<uint32_t>((sk * C::K_BYTES) >> 4);
        const uint32_t tm_s = tmem + TM::S(t);
        if (elect_one()) {
          // unrolled per 128-byte box: fully unrolled, d_qk = 192 runs out of the issuing
          // warps' registers
#pragma unroll 4
          for (int s = 0; s < C::QK_STEPS; ++s) {
            const uint32_t off = ((s / 4) * C::BOX_BYTES + (s % 4) * 32) >> 4;
            mma_ss<FP8 ? 1 : 0>(tm_s, qd + off, kd + off, C::IDESC_S, s > 0 ? 1u : 0u);
          }
          tc_commit(s_full(t));
          if (j == (t ? U.n_t1 : U.n_t0) - 1) tc_commit(q_empty(t));
          if (t == 1 || j >= U.n_t1) tc_commit(k_empty + sk);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int j, int g0, const Unit& U) {
        const int sv = (g0 + j) % C::NV;
        const uint64_t vd = v_desc(sv);
        const uint32_t tm_o = tmem + TM::O(t);
        if (elect_one()) {
          if constexpr (!FP8) {
            const uint32_t tm_p = tmem + TM::P(t);
#pragma unroll
            for (int s = 0; s < C::PV_STEPS; ++s) {
              // V is [keys x d] with d contiguous: B operand MN-major; 8-key groups 1 KB
              // apart (16 keys per step), 64-column atoms 16 KB apart (LBO)
              mma_ts_f16(tm_o, tm_p + s * 8, vd + ((s * 2048) >> 4), C::IDESC_PV_BF16,
                         (j > 0 || s > 0) ? 1u : 0u);
            }
          } else {
            const uint64_t pd = dp0 + static_cast<uint32_t>((t * C::BOX_BYTES) >> 4);
#pragma unroll
            for (int s = 0; s < C::PV_STEPS; ++s) {
              // [O | row sum] += (P * 2^-(7+k)) x [V | 1]; 32 keys (32 B of P) per step
              const uint32_t sfa = (tmem + TM::SFA(t)) | (static_cast<uint32_t>(s) << 30);
              const uint32_t sfb = (tmem + TM::SFB) | (static_cast<uint32_t>(s) << 30);
              mma_ss_mxf8(tm_o, pd + ((s * 32) >> 4), vd + ((s * 4096) >> 4),
                          idesc_mxf8(0, 1, BLOCK_M, TM::PV_N, s, s), sfa, sfb,
                          (j > 0 || s > 0) ? 1u : 0u);
            }
          }
          tc_commit(pv_done(t));
          if (t == 1 || j >= U.n_t1) tc_commit(v_empty + sv);
        }
        __syncwarp();
      };
      const bool s_issuer = warp == 9;  // S MMAs (warp 10: PV MMAs)
      bool ok = true;
      int cs[2] = {0, 0};  // S MMAs issued per slot
      int cp[2] = {0, 0};  // PV MMAs issued per slot
      int nq[2] = {0, 0};  // units begun per slot (Q tiles consumed)
      int g0 = 0;          // ring position of the current unit's key tile 0
      // the Q tile of slot t for its current unit has landed
      auto wait_q = [&](int t) { return mbar_wait(q_full(t), nq[t] & 1, p.err, p.timeout_ns); };
      auto wait_k = [&](int g) {
        return mbar_wait(k_full + g % C::NK, (g / C::NK) & 1, p.err, p.timeout_ns);
      };
      // before writing S_t, both slots must have read every S issued to them (S_0 and S_1
      // share TMEM columns: 64 for FP8, all 128 for BF16)
      auto wait_reads = [&]() {
        bool r = true;
#pragma unroll
        for (int x = 0; x < 2; ++x)
          if (r && cs[x] > 0) r = mbar_wait(s_read(x), (cs[x] - 1) & 1, p.err, p.timeout_ns);
        return r;
      };
      for (int k = 0; ok; ++k) {
        int u = -1, st = 0;
        Unit U;
        ok = take_unit(k, u, st, U);
        if (!ok || u < 0) break;
        if (st <= 0) continue;
        const int n_max = max(U.n_t0, U.n_t1);
        auto nt = [&](int t) { return t == 0 ? U.n_t0 : U.n_t1; };
        if constexpr (SAHEAD) {
          if (s_issuer) {
            // S_0(0), S_1(0), then S_t(j+1) in iteration j (this loop shape measured ~12%
            // faster than issuing S_t(j) in iteration j, with the same waits)
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!ok || nt(t) == 0) continue;
              ok = wait_reads();
              if (ok) ok = wait_q(t);
              if (ok) ok = wait_k(g0);
              if (!__all_sync(0xffffffffu, ok)) break;
              tc_fence_after();
              issue_s(t, 0, g0, U);
              ++cs[t];
            }
            for (int j = 0; j < n_max && ok; ++j) {
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                if (j + 1 >= nt(t)) continue;
                // S_t(j+1) once this slot has read S_t(j) and the other slot its latest S
                ok = mbar_wait(s_read(t), (cs[t] - 1) & 1, p.err, p.timeout_ns);
                if (ok && cs[1 - t] > 0)
                  ok = mbar_wait(s_read(1 - t), (cs[1 - t] - 1) & 1, p.err, p.timeout_ns);
                if (ok) ok = wait_k(g0 + j + 1);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                issue_s(t, j + 1, g0, U);
                ++cs[t];
              }
            }
          } else {
            // PV_t(j) once P_t(j) is written (FP8: shared memory; BF16: TMEM) and V(j) has
            // landed
            for (int j = 0; j < n_max && ok; ++j) {
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                if (j >= nt(t)) continue;
                ok = mbar_wait(p_full(t), cp[t] & 1, p.err, p.timeout_ns);
                if (ok) ok = mbar_wait(v_full + (g0 + j) % C::NV, ((g0 + j) / C::NV) & 1, p.err, p.timeout_ns);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                issue_pv(t, j, g0, U);
                ++cp[t];
              }
            }
          }
        } else {
          // S_0(0), S_1(0); then per key tile j and slot t: PV_t(j), S_t(j+1).  S_t(0) of a
          // unit follows the slot's last PV of the previous unit in this issue stream, so it
          // overwrites P_t only after that PV has read it.
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!ok || nt(t) == 0) continue;
            ok = wait_q(t);
            if (ok) ok = wait_k(g0);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            issue_s(t, 0, g0, U);
            ++cs[t];
          }
          for (int j = 0; j < n_max && ok; ++j) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (j >= nt(t)) continue;
              const bool next = j + 1 < nt(t);
              // prerequisites of S_t(j+1), normally met long before P_t(j) is ready
              if (next) ok = wait_k(g0 + j + 1);
              if (ok) ok = mbar_wait(p_full(t), cp[t] & 1, p.err, p.timeout_ns);
              if (ok) ok = mbar_wait(v_full + (g0 + j) % C::NV, ((g0 + j) / C::NV) & 1, p.err, p.timeout_ns);
              if (!__all_sync(0xffffffffu, ok)) break;
              tc_fence_after();
              issue_pv(t, j, g0, U);
              ++cp[t];
              if (next) {
                issue_s(t, j + 1, g0, U);
                ++cs[t];
              }
            }
          }
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) nq[t] += nt(t) > 0 ? 1 : 0;
        g0 += n_max;
      }
      // every MMA issued by this warp completes before TMEM is released
      const int mine = s_issuer ? 0 : 1;
      if (elect_one()) tc_commit(mma_done(mine));
      __syncwarp();
      mbar_wait(mma_done(mine), 0, p.err, DRAIN_TIMEOUT_NS, false);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<SAHEAD>::SOFTMAX));
    // ------------------------------------------------------------- softmax of slot t
    const int t = warp >> 2;
    const int r = tid & 127;                      // row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t ts = lane_base + TM::S(t);     // S_t columns of this lane
    const uint32_t tp = lane_base + TM::P(t);     // BF16: P_t columns
    const uint32_t to = lane_base + TM::O(t);     // O_t (FP8: and the row sum) columns
    float a = 0.0f, a256 = 0.0f;  // FP8 slope in code units per raw score (and / 256)
    if constexpr (FP8) {
      a = static_cast<float>(p.leanp_c * static_cast<double>(*p.descale_q) *
                             static_cast<double>(*p.descale_k));
      a256 = a * 0.00390625f;
      // scale factors of the B operand [V | 1]: 2^0, for every PV of this CTA
      const uint32_t sfb = lane_base + TM::SFB;
      tmem_st4(sfb, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_st4(sfb + 4, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    }
    bool ok = true;
    int c = 0;  // key tiles of this slot processed so far (all units)
    constexpr bool TMA_O = C::TMA_O && !VARLEN;
    constexpr bool WARP_O = C::WARP_O;
    // issues this slot's O stores (BF16: this warp's)
    const bool o_issuer = WARP_O ? lane == 0 : (tid & 127) == 0;
    bool o_pending = false;  // FP8: a store from P_t may still be reading it
    int o_phase = 0;         // completed phases of o_sync(t)
    // the slot's four warps meet (bounded, so that a warp that has given up cannot leave the
    // others waiting for ever); orders the issuer's and the other threads' shared-memory
    // accesses through the barrier's release / acquire
    auto slot_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(o_sync + t);
      const bool r = mbar_wait(o_sync + t, o_phase & 1, p.err, p.timeout_ns);
      ++o_phase;
      return __all_sync(0xffffffffu, r);
    };
    for (int k = 0; ok; ++k) {
      // the unit's queue entry is kept until the end of its epilogue, which reads the
      // head, batch and first token from it again (fewer values live through the tiles)
      int u = -1, st = 0;
      Unit U;
      ok = take_unit(k, u, st, U, false);
      if (!ok || u < 0) break;
      if (st < 0 && tid == 0) atomicCAS(p.err, DEV_OK, DEV_BAD_SEQLENS);
      const int n_t = t == 0 ? U.n_t0 : U.n_t1;
      if (st <= 0 || n_t == 0) {
        release_unit(k);
        continue;
      }
      const int qt = t ? U.qt1 : U.qt0;
      const int q_pos = qt * BLOCK_M + r;           // query position in the sequence
      float ms = -INFINITY;  // BF16 reference max, scaled to log2 units
      int m_i = 0;           // FP8 reference max, code units
      float l = 0.0f;        // running row sum
      for (int j = 0; j < n_t; ++j, ++c) {
        ok = mbar_wait(s_full(t), c & 1, p.err, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        uint32_t sraw[BLOCK_N];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld32(ts + cc * 32, sraw + cc * 32);
        tmem_wait_ld();
        if constexpr (SAHEAD) {
          // S_t is in registers: the next S (of either slot) may now overwrite the columns
          tc_fence_before();
          mbar_arrive(s_read(t));
        }
        float s[BLOCK_N];
#pragma unroll
        for (int cc = 0; cc < BLOCK_N; ++cc) s[cc] = __uint_as_float(sraw[cc]);
        const bool diag = p.causal && j == qt;
        if (diag) {
#pragma unroll
          for (int cc = 0; cc < BLOCK_N; ++cc)
            if (cc > r) s[cc] = -INFINITY;
        }
        if constexpr (VARLEN) {
          // keys past the end of the sequence (the next sequence's, or zero fill)
          const int kvalid = U.seq_len - j * BLOCK_N;
          if (kvalid < BLOCK_N) {
#pragma unroll
            for (int cc = 0; cc < BLOCK_N; ++cc)
              if (cc >= kvalid) s[cc] = -INFINITY;
          }
        }
        // block maxima with two independent chains per 64-key block
        float mx[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = s[i * 32];
#pragma unroll
        for (int cc = 1; cc < 31; cc += 2) {
#pragma unroll
          for (int i = 0; i < 4; ++i) mx[i] = fmax3(mx[i], s[i * 32 + cc], s[i * 32 + cc + 1]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], s[i * 32 + 31]);
        const float mu0 = fmaxf(mx[0], mx[1]);
        const float mu1 = fmaxf(mx[2], mx[3]);

        uint32_t pw[FP8 ? 32 : 64];
        float alpha = 1.0f;
        uint32_t sf_w = 0;
        if constexpr (!FP8) {
          const float cand = fmaxf(mu0, mu1) * p.c1;
          const float ms_new = (j == 0 || cand > ms + BF16_HEADROOM) ? cand : ms;
          if (j > 0) alpha = ex2_approx(ms - ms_new);
          ms = ms_new;
          // element pairs in packed two-wide fp32 (the even and odd sums are the two lanes)
          const float2 c1x2 = make_float2(p.c1, p.c1);
          const float2 nms2 = make_float2(-ms, -ms);
          float2 lsum = make_float2(0.0f, 0.0f);
          // one loop for every tile, the diagonal one included (a second copy for it cost
          // 1-4% in instruction fetch): a masked score (-inf) gives 0 on the MUFU and 2^-125
          // on the polynomial, against a row sum of at least 1 (the row's maximum gives 1)
          {
#pragma unroll
            for (int cc = 0; cc < BLOCK_N; cc += 2) {
              const float2 x = __ffma2_rn(make_float2(s[cc], s[cc + 1]), c1x2, nms2);
              // one element pair in four on the FMA pipe, the rest on the MUFU
              const bool poly = (cc & 7) == 6;
              const float2 pp = poly ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
              lsum = __fadd2_rn(lsum, pp);
              pw[cc >> 1] = pack_bf16x2(pp.x, pp.y);
            }
          }
          l = l * alpha + (lsum.x + lsum.y);
        } else {
          const float mu = fmaxf(mu0, mu1);
          const int cand = __float2int_ru(__fmul_rn(a, mu));
          const int m_new = (j == 0 || cand > m_i + LEANP_HEADROOM) ? cand : m_i;
          if (j > 0) alpha = ex2_approx(static_cast<float>(m_i - m_new) * 0.125f);
          m_i = m_new;
          const int k0 = leanp_kshift(mu0, a, m_new);
          const int k1 = leanp_kshift(mu1, a, m_new);
          if constexpr (EXACT) {
            // x = fmaf(s, a/8, (8 (7 + k_b) - m)/8); P code = e4m3_rn(2^x)
            const float a8 = a * 0.125f;
            const float cx0 = __int2float_rn(8 * (7 + k0) - m_new) * 0.125f;
            const float cx1 = __int2float_rn(8 * (7 + k1) - m_new) * 0.125f;
#pragma unroll
            for (int cc = 0; cc < BLOCK_N; cc += 4) {
              const float cx = cc < 64 ? cx0 : cx1;
              const float p0 = ex2_approx(__fmaf_rn(s[cc + 0], a8, cx));
              const float p1 = ex2_approx(__fmaf_rn(s[cc + 1], a8, cx));
              const float p2 = ex2_approx(__fmaf_rn(s[cc + 2], a8, cx));
              const float p3 = ex2_approx(__fmaf_rn(s[cc + 3], a8, cx));
              pw[cc >> 2] = f32_to_e4m3x2(p0, p1) | (f32_to_e4m3x2(p2, p3) << 16);
            }
          } else {
            const float cb0 = __int2float_rn(LEANP_TOP + 8 * k0 - m_new) * 0.00390625f;
            const float cb1 = __int2float_rn(LEANP_TOP + 8 * k1 - m_new) * 0.00390625f;
            const float2 s256 = make_float2(256.0f, 256.0f);
            const float2 magic = make_float2(LEANP_MAGIC, LEANP_MAGIC);
#pragma unroll
            for (int cc = 0; cc < BLOCK_N; cc += 4) {
              const float cb = cc < 64 ? cb0 : cb1;
              // multiply-add (saturating to [0,1]), then the integer conversion by a magic
              // fma, two lanes at a time
              const float2 u01 = make_float2(fma_sat(s[cc + 0], a256, cb), fma_sat(s[cc + 1], a256, cb));
              const float2 u23 = make_float2(fma_sat(s[cc + 2], a256, cb), fma_sat(s[cc + 3], a256, cb));
              const float2 r01 = __ffma2_rn(u01, s256, magic);
              const float2 r23 = __ffma2_rn(u23, s256, magic);
              pw[cc >> 2] = pack_low_bytes(__float_as_uint(r01.x), __float_as_uint(r01.y),
                                           __float_as_uint(r23.x), __float_as_uint(r23.y));
            }
          }
          const uint32_t e0 = static_cast<uint32_t>(120 - k0), e1 = static_cast<uint32_t>(120 - k1);
          const uint32_t sf_word = e0 | (e0 << 8) | (e1 << 16) | (e1 << 24);  // UE8M0 2^-(7+k)
          if constexpr (DUMP) {
            const int* ue = unit_q + (k % UQ) * C::UQ_INTS;
            const size_t row = (static_cast<size_t>(ue[2]) * p.Hq + (hp ? ue[3] + t : ue[3])) * p.S + q_pos;
            float* ds = p.dump_s + row * p.S + static_cast<size_t>(j) * BLOCK_N;
            uint8_t* dc = p.dump_codes + row * p.S + static_cast<size_t>(j) * BLOCK_N;
            for (int cc = 0; cc < BLOCK_N; ++cc) ds[cc] = s[cc];
            for (int cc = 0; cc < BLOCK_N / 4; ++cc) reinterpret_cast<uint32_t*>(dc)[cc] = pw[cc];
            uint8_t* dk = p.dump_kshift + row * (p.S / 64) + j * 2;
            dk[0] = static_cast<uint8_t>(k0);
            dk[1] = static_cast<uint8_t>(k1);
          }
          sf_w = sf_word;
        }
        if constexpr (SAHEAD) {
          // S_t(j) may have been issued before PV_t(j-1): that PV must be complete before
          // O_t is rescaled and before P_t (FP8: and its scale factors) is overwritten (the
          // previous unit's last PV was waited for by its epilogue)
          if (j > 0) {
            ok = mbar_wait(pv_done(t), (c - 1) & 1, p.err, p.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
          }
        }
        // O_t (and the FP8 row sum) may be rescaled (without SAHEAD, PV_t(j-1) has completed:
        // S_t(j) was issued after it and has completed)
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            tmem_ld32(to + cc * 32, o);
            tmem_wait_ld();
            const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 rr = __fmul2_rn(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2);
              o[i] = __float_as_uint(rr.x);
              o[i + 1] = __float_as_uint(rr.y);
            }
            tmem_st32(to + cc * 32, o);
          }
          if constexpr (FP8) {
            uint32_t rs;
            tmem_ld1(to + TM::RS, rs);
            tmem_wait_ld();
            tmem_st1(to + TM::RS, __float_as_uint(__uint_as_float(rs) * alpha));
          }
        }
        if constexpr (!FP8) {
          tmem_st32(tp, pw);
          tmem_st32(tp + 32, pw + 32);
        } else {
          // row r of P_t: 128 codes = 8 chunks of 16 B; chunk cc sits at chunk position
          // cc ^ (r mod 8) of the row (128-byte swizzle, rows 128 B apart)
          if (o_pending) {
            // P_t held the previous unit's O on its way out: that store must have read it
            if (o_issuer) bulk_wait_read_all();
            o_pending = false;
            ok = slot_sync();
            if (!ok) break;
          }
          const uint32_t prow = smem_addr(smem + C::OFF_P + t * C::BOX_BYTES) + r * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            st_shared_v4(prow + ((cc ^ (r & 7)) << 4), pw[4 * cc], pw[4 * cc + 1], pw[4 * cc + 2],
                         pw[4 * cc + 3]);
          fence_proxy_async_smem();
          // scale factors of P: row R's word (byte k = 32-key block k of the tile) at lane R,
          // column SFA + R/32 -- the quadrant of the MMA datapath that computes row R
          tmem_st1(lane_base + TM::SFA(t) + (warp & 3), sf_w);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(t));
      }
      tmem_wait_st();  // nothing of this thread may still be writing TMEM on any exit path
      if (!ok) break;
      // ----------------------------------------------------------- epilogue of the unit
      ok = mbar_wait(pv_done(t), (c - 1) & 1, p.err, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      if constexpr (TMA_O && !FP8) {
        // this warp's previous store from the staging buffer (the previous unit's second
        // half) must have read its rows; waited for here, before O occupies the registers
        if (o_issuer) bulk_wait_read_all();
        __syncwarp();
      }
      tc_fence_after();
      uint32_t oraw[DV];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(to + cc * 32, oraw + cc * 32);
      if constexpr (FP8) {
        uint32_t rs;
        tmem_ld1(to + TM::RS, rs);
        tmem_wait_ld();
        l = __uint_as_float(rs);  // sum of the rounded probabilities, 2^-(7+k) scaled
      }
      tmem_wait_ld();
      // O_t is in registers: the next unit's first PV may overwrite it once this slot
      // signals P_t(0) of that unit (after its own fence and arrive)
      float o[DV];
#pragma unroll
      for (int cc = 0; cc < DV; ++cc) o[cc] = __uint_as_float(oraw[cc]);
      float inv = 1.0f / l;
      if constexpr (FP8) inv *= *p.descale_v;
      if (p.unrotate) {
        // x -> x H_128 / sqrt(128), butterfly stages h = 1, 2, ..., 64
#pragma unroll
        for (int hh = 1; hh < DV; hh <<= 1) {
#pragma unroll
          for (int i = 0; i < DV; ++i) {
            if ((i & hh) == 0) {
              const float x0 = o[i], x1 = o[i + hh];
              o[i] = x0 + x1;
              o[i + hh] = x0 - x1;
            }
          }
        }
        inv *= 0.08838834764831845f;
      }
      // VARLEN: rows past the end of the sequence hold another sequence's queries (or zero
      // fill) and are not written
      const int* ue = unit_q + (k % UQ) * C::UQ_INTS;
      const int hs = hp ? ue[3] + t : ue[3];  // this slot's query head
      U.b = ue[2];
      U.tok0 = ue[5];
      const bool row_in = !VARLEN || q_pos < U.seq_len;
      const uint64_t pol_once = l2_policy_evict_first();  // O is written once
      const float2 inv2 = make_float2(inv, inv);
      if constexpr (TMA_O) {
        // 64 columns at a time: row r's 128 bytes as 8 chunks at positions cc ^ (r mod 8) of
        // the slot's staging buffer (the tensor map's swizzle), then one thread stores the
        // 128 x 64 box (BF16: lane 0 of each warp its 32 x 64 box, 4 KB and 1 KB aligned);
        // rows of O are 8 KB apart, so per-thread row stores would touch a separate line
        // per lane
        const int wr = WARP_O ? (warp & 3) * 32 : 0;  // first row of the stored box
        uint8_t* ost = smem + C::OFF_OST + t * C::BOX_BYTES;
        const uint32_t srow = smem_addr(ost) + r * 128;
        auto staging_sync = [&]() -> bool {
          if constexpr (WARP_O) {
            __syncwarp();
            return true;
          } else {
            return slot_sync();
          }
        };
#pragma unroll
        for (int h = 0; h < 2 && ok; ++h) {
          if (h == 1) {
            // the buffer's previous store (this unit's first half) must have read it
            if (o_issuer) bulk_wait_read_all();
            ok = staging_sync();
            if (!ok) break;
          }
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const int col = 64 * h + 8 * cc;
            const float2 a0 = __fmul2_rn(make_float2(o[col + 0], o[col + 1]), inv2);
            const float2 a1 = __fmul2_rn(make_float2(o[col + 2], o[col + 3]), inv2);
            const float2 a2 = __fmul2_rn(make_float2(o[col + 4], o[col + 5]), inv2);
            const float2 a3 = __fmul2_rn(make_float2(o[col + 6], o[col + 7]), inv2);
            st_shared_v4(srow + ((cc ^ (r & 7)) << 4), pack_bf16x2(a0.x, a0.y), pack_bf16x2(a1.x, a1.y),
                         pack_bf16x2(a2.x, a2.y), pack_bf16x2(a3.x, a3.y));
          }
          fence_proxy_async_smem();
          ok = staging_sync();
          if (!ok) break;
          if (o_issuer) {
            tma_store_3d_hint(&tm_o, ost + wr * 128, 64 * h, hs, U.tok0 + qt * BLOCK_M + wr, pol_once);
            bulk_commit_group();
          }
        }
        o_pending = FP8;
        if (!ok) break;
      } else {
        __nv_bfloat16* orow = p.o + ((static_cast<size_t>(U.tok0) + q_pos) * p.Hq + hs) * DV;
#pragma unroll
        for (int cc = 0; cc < DV; cc += 8) {
          const float2 a0 = __fmul2_rn(make_float2(o[cc + 0], o[cc + 1]), inv2);
          const float2 a1 = __fmul2_rn(make_float2(o[cc + 2], o[cc + 3]), inv2);
          const float2 a2 = __fmul2_rn(make_float2(o[cc + 4], o[cc + 5]), inv2);
          const float2 a3 = __fmul2_rn(make_float2(o[cc + 6], o[cc + 7]), inv2);
          uint4 v;
          v.x = pack_bf16x2(a0.x, a0.y);
          v.y = pack_bf16x2(a1.x, a1.y);
          v.z = pack_bf16x2(a2.x, a2.y);
          v.w = pack_bf16x2(a3.x, a3.y);
          if (row_in) st_global_v4_hint(orow + cc, v, pol_once);
        }
      }
      if (p.lse != nullptr && row_in) {
        float lse_v;
        if constexpr (FP8)
          lse_v = 0.69314718055994531f * (static_cast<float>(m_i) * 0.125f + __log2f(l));
        else
          lse_v = 0.69314718055994531f * (ms + __log2f(l));
        // lse [B, Hq, S], or [Hq, total tokens] for packed sequences
        const size_t li = (VARLEN && p.cu_seqlens != nullptr)
                              ? static_cast<size_t>(hs) * p.total_tokens + U.tok0 + q_pos
                              : (static_cast<size_t>(U.b) * p.Hq + hs) * p.S + q_pos;
        p.lse[li] = lse_v;
      }
      release_unit(k);
    }
    // the O stores complete before the CTA exits (their source is this CTA's shared memory)
    if (TMA_O && o_issuer) bulk_wait_all();
  }
  __syncthreads();
  if (warp == 11) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
