// Forward causal (prefill) attention on sm_100a over CTA pairs: every MMA is a
// tcgen05.mma.cta_group::2 of M = 256 rows, 128 in each CTA of a two-CTA cluster, so one
// instruction issued by the leader CTA does the work of two single-CTA instructions.
//
// Computes O = softmax(mask(Q K^T * scale)) V (the forward causal attention of the
// prefill phase, [ZYFA-fr] "Ce que couvrent les noyaux") in BF16 and in FP8 e4m3 with the
// lean-P probabilities of [ZYFA-mb] "Como o motor de atenção FP8 da Zyphra funciona" (one
// multiply-add and one integer conversion write the e4m3 bit pattern; a power of two per
// 64-key block removed by the block-scaled MMA; the row normaliser is the tensor-core sum
// of the rounded probabilities).  The softmax arithmetic is the single-CTA kernel's
// (attn_fwd.cuh); what changes is the work unit, the operand split and the signalling.
//
// Work unit (one cluster): two CTAs c = 0, 1, each with two 128-row query slots t = 0, 1
// in ping-pong, all four slots against the same K/V tiles:
//   heads mode (Hq / Hkv even): CTA c takes query head 2 hp + c -- two heads of one
//     grouped-query kv group -- at query tiles 2 p + t, so every K/V tile in shared memory
//     serves two heads and both CTAs have the same causal extent;
//   rows mode (otherwise, e.g. Hq == Hkv): CTA c takes query tiles 4 p + 2 t + c of one
//     head; the pair runs to CTA 1's causal extent, where CTA 0 sees one fully masked key
//     tile per slot.
// Operands of the pair MMAs, at the same shared-memory offsets in both CTAs:
//   S_t = Q_t K^T   A = Q_t (each CTA its own 128 rows), B = K tile (CTA c holds keys
//                   64 c .. 64 c + 63, K-major), N = 128: each CTA's TMEM gets its rows x
//                   all 128 keys;
//   O_t += P_t V    A = P_t (each CTA its own rows, in shared memory; BF16 with d_qk = 192:
//                   in TMEM over S_t),
//                   B = V tile (CTA c holds value columns 64 c .. 64 c + 63, MN-major);
//                   FP8 extends each half by 16 columns of ones (64-byte swizzled atoms,
//                   the ones one leading-byte offset away), so N = 160 and TMEM columns
//                   [0,64) = O[:, 0:64], [64,80) = row sum, [80,144) = O[:, 64:128].  (A
//                   pair MMA with an MN-major B takes N in multiples of 32, 16 per CTA; the
//                   single-CTA kernel's N = 144 is not one.)
// Roles (384 threads per CTA, 12 warps):
//   warps 0-7   softmax of slots 0 and 1 (thread r = query row r = TMEM lane r), both CTAs;
//   warp 8      TMA producer of this CTA's operands (its Q rows, its K and V halves);
//   warp 9      leader: the MMA issuer (S and PV of both slots); peer: idle;
//   warp 10     idle;
//   warp 11     TMEM allocator (cta_group::2) and forwarder: each CTA's copies complete on
//               its own barriers (so each CTA can drain its own copies on any exit path);
//               the forwarder relays each completion to the leader's ready barriers
//               (count 2: both CTAs' halves landed).
// Barriers: the leader waits on q_ready, k_ready, v_ready (forwarded), p_full and s_read
// (one arrival per softmax warp of both CTAs: 8); the MMA completions (s_full, pv_done,
// k_empty, v_empty) are committed with multicast to the same barriers in both CTAs.
//
// Every wait is bounded (mbar_wait): on expiry the CTA records DEV_TIMEOUT and unwinds; both
// CTAs meet at a final cluster barrier before the TMEM is released.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_fwd.cuh"
#include "ptx.cuh"

namespace attn {

// Register split after setmaxnreg: the pair kernel's MMA warp issues for both CTAs from
// precomputed descriptors (more live registers than the single-CTA kernel's), so it takes
// 104 per thread and the softmax warps 200; the launch needs 168 either way.
constexpr int PAIR_REGS_SOFTMAX = 200;
constexpr int PAIR_REGS_OTHER = 104;
static_assert((2 * 128 * PAIR_REGS_SOFTMAX + 128 * PAIR_REGS_OTHER + NUM_THREADS - 1) /
                      NUM_THREADS <= REGS_NEEDED_AT_LAUNCH,
              "the pair split must fit the registers the launch checks for");

template <bool FP8, int DQK>
struct PairCfg {
  static constexpr int E = FP8 ? 1 : 2;                    // bytes per element
  static constexpr int BOX_COLS = 128 / E;                 // elements per 128-B box row
  static constexpr int Q_BOXES = (DQK * E + 127) / 128;    // 128-B column boxes of Q and K
  static constexpr int Q_BOX_BYTES = 128 * 128;            // 128 rows x 128 B
  static constexpr int K_BOX_BYTES = 64 * 128;             // 64 keys x 128 B
  static constexpr int Q_BYTES = Q_BOXES * Q_BOX_BYTES;    // one slot
  static constexpr int K_BYTES = Q_BOXES * K_BOX_BYTES;    // this CTA's half of a K tile
  // this CTA's half of a V tile: 128 keys x 64 columns (FP8: 64 B rows, 64-B swizzle;
  // BF16: 128 B rows, 128-B swizzle)
  static constexpr int V_BYTES = 128 * 64 * E;
  static constexpr int V_ROW = 64 * E;
  // P_t in shared memory (the A operand of PV, K-major, 128-B swizzle): always for FP8
  // (e4m3 codes), for BF16 with d_qk = 128 (with d_qk = 192 the bf16 P stays over S_t in
  // TMEM: shared memory holds Q, the K/V ring and no more)
  static constexpr bool PSMEM = FP8 || DQK == 128;
  static constexpr int P_BYTES = FP8 ? 128 * 128 : (PSMEM ? 2 * 128 * 128 : 0);  // per slot
  static constexpr int NK = FP8 ? (DQK == 128 ? 6 : 4) : (DQK == 128 ? 3 : 2);
  static constexpr int NV = NK;
  static constexpr int KSTEP = FP8 ? 32 : 16;
  static constexpr int QK_STEPS = DQK / KSTEP;
  static constexpr int PV_STEPS = BLOCK_N / KSTEP;
  static constexpr int PV_N = FP8 ? 160 : 128;
  static constexpr int OV1 = PV_N / 2;       // TMEM column of O[:, 64] within O_t
  static constexpr int RS = 64;              // FP8: row-sum column within O_t
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * K_BYTES;
  static constexpr int OFF_ONES = OFF_V + NV * V_BYTES;           // FP8: 128 keys x 64 B
  static constexpr int OFF_P = OFF_ONES + (FP8 ? 128 * 64 : 0);   // P_0, P_1 (PSMEM)
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  // barriers, per CTA: q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV] (this
  // CTA's copies / the pair's MMAs), q_ready, k_ready[NK], v_ready[NV] (leader: both
  // halves landed), and per slot: s_full, p_full, pv_done, s_read, mma_done
  static constexpr int NUM_BARS = 1 + 2 * NK + 2 * NV + 1 + NK + NV + 2 * 5;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static_assert(SMEM_ALLOC <= 232448, "shared memory per block exceeded");
  // one CTA per SM: the pair's 512-column TMEM allocations never wait on another CTA
  static_assert(SMEM_ALLOC > 232448 / 2, "a pair CTA must hold more than half of the SM");
  static constexpr uint32_t IDESC_S =
      idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, 0u, 0u, 2 * BLOCK_M, BLOCK_N);
  static constexpr uint32_t IDESC_PV_BF16 = idesc_dense(1u, 1u, 0u, 1u, 2 * BLOCK_M, DV);
};

// TMEM columns per CTA (every MMA accumulator at a multiple of 32 columns).  FP8: O_0
// [0,160), O_1 [160,320) (value columns and row sum as above); scale factors of P at
// [320,336): slot t, 64-key block b at 320 + 8 t + 4 b, one column per 32-row quadrant of the
// datapath (row R's factor in byte 0 of lane R, column + R / 32); scale factors of [V | 1] at
// [336,344); S_0 [352,480), S_1 [384,512) (overlapping in [384,480): an S MMA waits until
// both slots have read their latest S).  BF16: S_0 [0,128), S_1 [128,256), O_0 [256,384),
// O_1 [384,512); with d_qk = 192 P_t (bf16) over the first columns of S_t.
template <bool FP8>
struct PairTmem {
  __host__ __device__ static constexpr uint32_t S(int t) { return FP8 ? 352u + 32u * t : 128u * t; }
  __host__ __device__ static constexpr uint32_t O(int t) { return FP8 ? 160u * t : 256u + 128u * t; }
  __host__ __device__ static constexpr uint32_t P(int t) { return 128u * t; }       // BF16 only
  __host__ __device__ static constexpr uint32_t SFA(int t, int b) { return 320u + 8u * t + 4u * b; }
  static constexpr uint32_t SFB = 336;
};
static_assert(PairTmem<true>::S(0) % 32 == 0 && PairTmem<true>::S(1) + 128 == 512, "TMEM");

template <bool FP8, int DQK, bool DUMP, bool EXACT = false, bool VARLEN = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = PairCfg<FP8, DQK>;
  using TM = PairTmem<FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::NK;
  uint64_t* v_full = k_empty + C::NK;
  uint64_t* v_empty = v_full + C::NV;
  uint64_t* q_ready = v_empty + C::NV;
  uint64_t* k_ready = q_ready + 1;
  uint64_t* v_ready = k_ready + C::NK;
  uint64_t* tbar = v_ready + C::NV;  // per slot: 5 barriers
  auto s_full = [&](int t) { return tbar + 5 * t + 0; };
  auto p_full = [&](int t) { return tbar + 5 * t + 1; };
  auto pv_done = [&](int t) { return tbar + 5 * t + 2; };
  auto s_read = [&](int t) { return tbar + 5 * t + 3; };
  auto mma_done = [&](int t) { return tbar + 5 * t + 4; };
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEMPTR);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t cta = cluster_ctarank();  // 0: leader, 1: peer
  const bool leader = cta == 0;
  // a barrier of the leader, as seen from this CTA (its own address when this is the leader)
  auto at_leader = [&](uint64_t* bar) { return mapa_shared(smem_addr(bar), 0); };

  // ---- work unit: longest-processing-time order over units of the pair
  const bool heads_mode = (p.G % 2) == 0;
  const int u = static_cast<int>(blockIdx.x) >> 1;
  const int heads_per_unit = heads_mode ? p.Hq / 2 : p.Hq;
  const int nbh = p.B * heads_per_unit;
  const int pos = p.n_pairs - 1 - u / nbh;  // n_pairs counts units along the queries
  const int bh = u % nbh;
  const int b = bh / heads_per_unit;
  const int h = heads_mode ? 2 * (bh % heads_per_unit) + static_cast<int>(cta) : bh % heads_per_unit;
  const int g = h / p.G;
  int tok0 = b * p.S;
  int seq_len = p.S;
  int n_q_tiles = p.n_q_tiles;
  if constexpr (VARLEN) {
    if (p.cu_seqlens != nullptr) {
      const int c0 = p.cu_seqlens[b], c1 = p.cu_seqlens[b + 1];
      if (c0 < 0 || c1 < c0 || static_cast<int64_t>(c1) > p.total_tokens ||
          c1 - c0 > p.max_seqlen) {
        if (threadIdx.x == 0) atomicCAS(p.err, DEV_OK, DEV_BAD_SEQLENS);
        return;  // both CTAs of the pair, before any barrier or allocation
      }
      tok0 = c0;
      seq_len = c1 - c0;
    }
    n_q_tiles = (seq_len + BLOCK_M - 1) / BLOCK_M;
  }
  // query tile of slot t in CTA c, and the pair's key-tile extent of slot t
  auto qtile = [&](int t, int c) { return heads_mode ? 2 * pos + t : 4 * pos + 2 * t + c; };
  if constexpr (VARLEN) {
    if (qtile(0, 0) >= n_q_tiles) return;  // this sequence has fewer units (both CTAs)
  }
  auto extent = [&](int t) {
    const int lo = qtile(t, 0), hi = qtile(t, 1);
    if (lo >= n_q_tiles) return 0;                  // slot empty in both CTAs
    if (!p.causal) return n_q_tiles;
    return min(hi, n_q_tiles - 1) + 1;
  };
  const int n_t0 = extent(0);
  const int n_t1 = extent(1);
  const int n_max = n_t1 > n_t0 ? n_t1 : n_t0;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, 2);
    for (int i = 0; i < C::NK; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(k_ready + i, 2);
    }
    for (int i = 0; i < C::NV; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
      mbar_init(v_ready + i, 2);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 8);   // one arrival per softmax warp of the slot, both CTAs
      mbar_init(pv_done(t), 1);
      mbar_init(s_read(t), 8);
      mbar_init(mma_done(t), 1);
    }
    fence_barrier_init();
  }
  if (warp == 11) {
    tmem_alloc2(tmem_ptr, 512);
    tmem_relinquish2();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if constexpr (FP8) {
    // the ones block (e4m3 1.0 = 0x38) after each V half, for the row sum
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::OFF_ONES);
    for (int i = tid; i < 128 * 64 / 4; i += NUM_THREADS) ones[i] = 0x38383838u;
    fence_proxy_async_smem();
  }
  __syncthreads();
  cluster_sync();  // both CTAs' barriers, ones and TMEM exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(PAIR_REGS_OTHER));
    if (warp == 8) {
      // ------------------------------------------------- TMA producer of this CTA's operands
      bool ok = true;
      const int nslots = n_t1 > 0 ? 2 : (n_t0 > 0 ? 1 : 0);
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full, nslots * C::Q_BYTES);
        for (int t = 0; t < nslots; ++t)
          for (int i = 0; i < C::Q_BOXES; ++i)
            tma_load_3d(smem + C::OFF_Q + t * C::Q_BYTES + i * C::Q_BOX_BYTES, &tm_q, q_full,
                        i * C::BOX_COLS, h, tok0 + qtile(t, static_cast<int>(cta)) * BLOCK_M);
      }
      __syncwarp();
      int jk = 0, jv = 0;
      for (int j = 0; j < n_max && ok; ++j) {
        if (j == p.stall_tile) break;  // test-only: the waits on this tile must run out
        const int sk = j % C::NK;
        if (j >= C::NK) ok = mbar_wait(k_empty + sk, ((j / C::NK) - 1) & 1, p.err, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(k_full + sk, C::K_BYTES);
          for (int i = 0; i < C::Q_BOXES; ++i)
            tma_load_3d(smem + C::OFF_K + sk * C::K_BYTES + i * C::K_BOX_BYTES, &tm_k,
                        k_full + sk, i * C::BOX_COLS, g, tok0 + j * BLOCK_N + 64 * static_cast<int>(cta));
        }
        __syncwarp();
        jk = j + 1;
        const int sv = j % C::NV;
        if (j >= C::NV) ok = mbar_wait(v_empty + sv, ((j / C::NV) - 1) & 1, p.err, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(v_full + sv, C::V_BYTES);
          tma_load_3d(smem + C::OFF_V + sv * C::V_BYTES, &tm_v, v_full + sv,
                      64 * static_cast<int>(cta), g, tok0 + j * BLOCK_N);
        }
        __syncwarp();
        jv = j + 1;
      }
      // drain: no copy issued by this CTA may still be in flight at exit
      if (nslots > 0) mbar_wait(q_full, 0, p.err, DRAIN_TIMEOUT_NS, false);
      for (int jj = (jk > C::NK ? jk - C::NK : 0); jj < jk; ++jj)
        mbar_wait(k_full + jj % C::NK, (jj / C::NK) & 1, p.err, DRAIN_TIMEOUT_NS, false);
      for (int jj = (jv > C::NV ? jv - C::NV : 0); jj < jv; ++jj)
        mbar_wait(v_full + jj % C::NV, (jj / C::NV) & 1, p.err, DRAIN_TIMEOUT_NS, false);
    } else if (warp == 11) {
      // ------------------------------------------------- forwarder: this CTA's copies have
      // landed -> one arrival on the leader's ready barrier of the same stage
      if (lane == 0 && n_max > 0) {
        bool ok = mbar_wait(q_full, 0, p.err, p.timeout_ns);
        if (ok) mbar_arrive_cluster(at_leader(q_ready));
        for (int j = 0; j < n_max && ok; ++j) {
          ok = mbar_wait(k_full + j % C::NK, (j / C::NK) & 1, p.err, p.timeout_ns);
          if (!ok) break;
          mbar_arrive_cluster(at_leader(k_ready + j % C::NK));
          ok = mbar_wait(v_full + j % C::NV, (j / C::NV) & 1, p.err, p.timeout_ns);
          if (!ok) break;
          mbar_arrive_cluster(at_leader(v_ready + j % C::NV));
        }
      }
      __syncwarp();
    } else if (leader && warp == 9) {
      // ------------------------------------------------- pair MMA issuer (leader only; one
      // warp issues every MMA of the pair, S and PV)
      auto nt = [&](int t) { return t == 0 ? n_t0 : n_t1; };
      const uint64_t dq0 = smem_desc_sw128(smem_addr(smem + C::OFF_Q), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_addr(smem + C::OFF_K), 16, 1024);
      const uint64_t dp0 = smem_desc_sw128(smem_addr(smem + C::OFF_P), 16, 1024);  // PSMEM
      auto v_desc = [&](int sv) -> uint64_t {
        const uint32_t va = smem_addr(smem + C::OFF_V + sv * C::V_BYTES);
        if constexpr (FP8) {
          // 72 columns per CTA: its 64 value columns, then 8 of the ones block one leading
          // offset away; 8-key groups 512 B apart
          return smem_desc_sw64(va, smem_addr(smem + C::OFF_ONES) - va, 512);
        } else {
          return smem_desc_sw128(va, C::V_BYTES, 1024);  // one 64-column atom per CTA
        }
      };
      constexpr uint16_t BOTH = 3;
      auto issue_s = [&](int t, int j) {
        const int sk = j % C::NK;
        const uint64_t qd = dq0 + static_cast<uint32_t>((t * C::Q_BYTES) >> 4);
        const uint64_t kd = dk0 + static_cast<uint32_t>((sk * C::K_BYTES) >> 4);
        const uint32_t tm_s = tmem + TM::S(t);
        if (elect_one()) {
#pragma unroll
          for (int s = 0; s < C::QK_STEPS; ++s) {
            const uint32_t oq = ((s / 4) * C::Q_BOX_BYTES + (s % 4) * 32) >> 4;
            const uint32_t ok_ = ((s / 4) * C::K_BOX_BYTES + (s % 4) * 32) >> 4;
            mma2_ss<FP8 ? 1 : 0>(tm_s, qd + oq, kd + ok_, C::IDESC_S, s > 0 ? 1u : 0u);
          }
          tc_commit2(s_full(t), BOTH);
          // K(j) is free once its last S has run: slot 1's, or slot 0's if slot 1 skips j
          if (t == 1 || j >= n_t1) tc_commit2(k_empty + sk, BOTH);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int j) {
        const int sv = j % C::NV;
        const uint64_t vd = v_desc(sv);
        const uint32_t tm_o = tmem + TM::O(t);
        if (elect_one()) {
          if constexpr (!FP8 && C::PSMEM) {
            // bf16 P_t from shared memory: 16 keys (32 B) per step, 64 keys per 128-B box
            const uint64_t pd = dp0 + static_cast<uint32_t>((t * C::P_BYTES) >> 4);
#pragma unroll
            for (int s = 0; s < C::PV_STEPS; ++s)
              mma2_ss<0>(tm_o, pd + (((s / 4) * C::Q_BOX_BYTES + (s % 4) * 32) >> 4),
                         vd + ((s * 16 * C::V_ROW) >> 4), C::IDESC_PV_BF16,
                         (j > 0 || s > 0) ? 1u : 0u);
          } else if constexpr (!FP8) {
            const uint32_t tm_p = tmem + TM::P(t);
#pragma unroll
            for (int s = 0; s < C::PV_STEPS; ++s)
              mma2_ts_f16(tm_o, tm_p + s * 8, vd + ((s * 16 * C::V_ROW) >> 4), C::IDESC_PV_BF16,
                          (j > 0 || s > 0) ? 1u : 0u);
          } else {
            const uint64_t pd = dp0 + static_cast<uint32_t>((t * C::P_BYTES) >> 4);
#pragma unroll
            for (int s = 0; s < C::PV_STEPS; ++s) {
              // 32 keys per step: block b = s / 2 of the tile; scale-factor id 0 (byte 0)
              const uint32_t sfa = tmem + TM::SFA(t, s / 2);
              const uint32_t sfb = tmem + TM::SFB;
              mma2_ss_mxf8(tm_o, pd + ((s * 32) >> 4), vd + ((s * 32 * C::V_ROW) >> 4),
                           idesc_mxf8(0, 1, 2 * BLOCK_M, C::PV_N, 0, 0), sfa, sfb,
                           (j > 0 || s > 0) ? 1u : 0u);
            }
          }
          tc_commit2(pv_done(t), BOTH);
          if (t == 1 || j >= n_t1) tc_commit2(v_empty + sv, BOTH);
        }
        __syncwarp();
      };
      // FP8: S_0 and S_1 share 64 TMEM columns; before writing S_t, the other slot's
      // softmax warps (both CTAs) must have read its latest S
      auto wait_other_read = [&](int t, int jo) -> bool {
        if constexpr (!FP8) return true;
        if (jo < 0) return true;
        return mbar_wait<true>(s_read(1 - t), jo & 1, p.err, p.timeout_ns);
      };
      bool ok = true;
      {
        ok = mbar_wait<true>(q_ready, 0, p.err, p.timeout_ns);
        if (__all_sync(0xffffffffu, ok)) {
          ok = n_max > 0 ? mbar_wait<true>(k_ready, 0, p.err, p.timeout_ns) : true;
          if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            if (n_t0 > 0) issue_s(0, 0);
            if (n_t1 > 0) {
              ok = wait_other_read(1, n_t0 > 0 ? 0 : -1);
              if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                issue_s(1, 0);
              }
            }
          }
        }
      }
      for (int j = 0; j < n_max && __all_sync(0xffffffffu, ok); ++j) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (j >= nt(t)) continue;
          const bool next = j + 1 < nt(t);
          if constexpr (C::PSMEM) {
            // S_t(j+1) as soon as S_t(j) and the other slot's latest S have been read (P is
            // in shared memory, so S_t(j+1) need not wait for PV_t(j)), then PV_t(j)
            if (next) {
              const int jo = t == 0 ? min(j, n_t1 - 1) : min(j + 1, n_t0 - 1);
              ok = mbar_wait<true>(s_read(t), j & 1, p.err, p.timeout_ns);
              if (ok) ok = wait_other_read(t, jo);
              if (ok) ok = mbar_wait<true>(k_ready + (j + 1) % C::NK, ((j + 1) / C::NK) & 1, p.err, p.timeout_ns);
              if (!__all_sync(0xffffffffu, ok)) break;
              tc_fence_after();
              issue_s(t, j + 1);
            }
            ok = mbar_wait<true>(p_full(t), j & 1, p.err, p.timeout_ns);
            if (ok) ok = mbar_wait<true>(v_ready + j % C::NV, (j / C::NV) & 1, p.err, p.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            issue_pv(t, j);
          } else {
            if (next) ok = mbar_wait<true>(k_ready + (j + 1) % C::NK, ((j + 1) / C::NK) & 1, p.err, p.timeout_ns);
            if (ok) ok = mbar_wait<true>(p_full(t), j & 1, p.err, p.timeout_ns);
            if (ok) ok = mbar_wait<true>(v_ready + j % C::NV, (j / C::NV) & 1, p.err, p.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            issue_pv(t, j);
            if (next) issue_s(t, j + 1);
          }
        }
      }
      // every MMA issued by this warp completes before the pair's TMEM is released
      if (elect_one()) tc_commit2(mma_done(0), 1);
      __syncwarp();
      mbar_wait(mma_done(0), 0, p.err, DRAIN_TIMEOUT_NS, false);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(PAIR_REGS_SOFTMAX));
    // ------------------------------------------------------------- softmax of slot t
    const int t = warp >> 2;
    const int n_t = t == 0 ? n_t0 : n_t1;
    const int qt = qtile(t, static_cast<int>(cta));
    const bool slot_in = qt < n_q_tiles;          // rows of a tile past the sequence: no output
    const int r = tid & 127;
    const int q_pos = qt * BLOCK_M + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t ts = lane_base + TM::S(t);
    const uint32_t tp = lane_base + TM::P(t);
    const uint32_t to = lane_base + TM::O(t);
    const uint32_t s_read_l = at_leader(s_read(t));
    const uint32_t p_full_l = at_leader(p_full(t));
    float a = 0.0f, a256 = 0.0f;
    if constexpr (FP8) {
      a = static_cast<float>(p.leanp_c * static_cast<double>(*p.descale_q) *
                             static_cast<double>(*p.descale_k));
      a256 = a * 0.00390625f;
    }
    float ms = -INFINITY;
    int m_i = 0;
    float l = 0.0f;
    if constexpr (FP8) {
      const uint32_t sfb = lane_base + TM::SFB;
      tmem_st4(sfb, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_st4(sfb + 4, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    }
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      ok = mbar_wait(s_full(t), j & 1, p.err, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sraw[BLOCK_N];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(ts + c * 32, sraw + c * 32);
      tmem_wait_ld();
      if constexpr (C::PSMEM) {
        // S_t is in registers: the leader may now issue the next S into these columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(s_read_l);
      }
      float s[BLOCK_N];
#pragma unroll
      for (int c = 0; c < BLOCK_N; ++c) s[c] = __uint_as_float(sraw[c]);
      // causal: keys past this row's position (the diagonal tile, and in rows mode CTA 0's
      // fully masked last tile)
      const int lim = q_pos - j * BLOCK_N;
      const bool diag = p.causal && lim < BLOCK_N - 1;
      if (diag) {
#pragma unroll
        for (int c = 0; c < BLOCK_N; ++c)
          if (c > lim) s[c] = -INFINITY;
      }
      if constexpr (VARLEN) {
        const int kvalid = seq_len - j * BLOCK_N;
        if (kvalid < BLOCK_N) {
#pragma unroll
          for (int c = 0; c < BLOCK_N; ++c)
            if (c >= kvalid) s[c] = -INFINITY;
        }
      }
      float mx[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = s[i * 32];
#pragma unroll
      for (int c = 1; c < 31; c += 2) {
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmax3(mx[i], s[i * 32 + c], s[i * 32 + c + 1]);
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
        float lsum0 = 0.0f, lsum1 = 0.0f;
        if (diag) {
#pragma unroll
          for (int c = 0; c < BLOCK_N; c += 2) {
            const float p0 = ex2_approx(__fmaf_rn(s[c], p.c1, -ms));
            const float p1 = ex2_approx(__fmaf_rn(s[c + 1], p.c1, -ms));
            lsum0 += p0;
            lsum1 += p1;
            pw[c >> 1] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < BLOCK_N; c += 2) {
            const float x0 = __fmaf_rn(s[c], p.c1, -ms);
            const float x1 = __fmaf_rn(s[c + 1], p.c1, -ms);
            const bool poly = (c & 7) == 6;
            const float p0 = poly ? exp2_poly(x0) : ex2_approx(x0);
            const float p1 = poly ? exp2_poly(x1) : ex2_approx(x1);
            lsum0 += p0;
            lsum1 += p1;
            pw[c >> 1] = pack_bf16x2(p0, p1);
          }
        }
        l = l * alpha + (lsum0 + lsum1);
      } else {
        const float mu = fmaxf(mu0, mu1);
        const int cand = __float2int_ru(__fmul_rn(a, mu));
        const int m_new = (j == 0 || cand > m_i + LEANP_HEADROOM) ? cand : m_i;
        if (j > 0) alpha = ex2_approx(static_cast<float>(m_i - m_new) * 0.125f);
        m_i = m_new;
        const int k0 = leanp_kshift(mu0, a, m_new);
        const int k1 = leanp_kshift(mu1, a, m_new);
        if constexpr (EXACT) {
          const float a8 = a * 0.125f;
          const float cx0 = __int2float_rn(8 * (7 + k0) - m_new) * 0.125f;
          const float cx1 = __int2float_rn(8 * (7 + k1) - m_new) * 0.125f;
#pragma unroll
          for (int c = 0; c < BLOCK_N; c += 4) {
            const float cx = c < 64 ? cx0 : cx1;
            const float p0 = ex2_approx(__fmaf_rn(s[c + 0], a8, cx));
            const float p1 = ex2_approx(__fmaf_rn(s[c + 1], a8, cx));
            const float p2 = ex2_approx(__fmaf_rn(s[c + 2], a8, cx));
            const float p3 = ex2_approx(__fmaf_rn(s[c + 3], a8, cx));
            pw[c >> 2] = f32_to_e4m3x2(p0, p1) | (f32_to_e4m3x2(p2, p3) << 16);
          }
        } else {
          const float cb0 = __int2float_rn(LEANP_TOP + 8 * k0 - m_new) * 0.00390625f;
          const float cb1 = __int2float_rn(LEANP_TOP + 8 * k1 - m_new) * 0.00390625f;
#pragma unroll
          for (int c = 0; c < BLOCK_N; c += 4) {
            const float cb = c < 64 ? cb0 : cb1;
            const uint32_t b0 = __float_as_uint(__fmaf_rn(fma_sat(s[c + 0], a256, cb), 256.0f, LEANP_MAGIC));
            const uint32_t b1 = __float_as_uint(__fmaf_rn(fma_sat(s[c + 1], a256, cb), 256.0f, LEANP_MAGIC));
            const uint32_t b2 = __float_as_uint(__fmaf_rn(fma_sat(s[c + 2], a256, cb), 256.0f, LEANP_MAGIC));
            const uint32_t b3 = __float_as_uint(__fmaf_rn(fma_sat(s[c + 3], a256, cb), 256.0f, LEANP_MAGIC));
            pw[c >> 2] = pack_low_bytes(b0, b1, b2, b3);
          }
        }
        const uint32_t e0 = static_cast<uint32_t>(120 - k0), e1 = static_cast<uint32_t>(120 - k1);
        // UE8M0 2^-(7+k) of the two 64-key blocks (byte 0 of each block's column)
        const uint32_t sf_word = e0 | (e1 << 16);
        if constexpr (DUMP) {
          // key tiles past the row's causal extent (rows mode) are not part of its row
          if (slot_in && (!p.causal || j <= qt)) {
            const size_t row = (static_cast<size_t>(b) * p.Hq + h) * p.S + q_pos;
            float* ds = p.dump_s + row * p.S + static_cast<size_t>(j) * BLOCK_N;
            uint8_t* dc = p.dump_codes + row * p.S + static_cast<size_t>(j) * BLOCK_N;
            for (int c = 0; c < BLOCK_N; ++c) ds[c] = s[c];
            for (int c = 0; c < BLOCK_N / 4; ++c) reinterpret_cast<uint32_t*>(dc)[c] = pw[c];
            uint8_t* dk = p.dump_kshift + row * (p.S / 64) + j * 2;
            dk[0] = static_cast<uint8_t>(k0);
            dk[1] = static_cast<uint8_t>(k1);
          }
        }
        sf_w = sf_word;
      }
      if constexpr (C::PSMEM) {
        // S_t(j) may have been issued before PV_t(j-1): that PV must be complete before O_t
        // is rescaled and before P_t (and its scale factors) are overwritten
        if (j > 0) {
          ok = mbar_wait(pv_done(t), (j - 1) & 1, p.err, p.timeout_ns);
          if (!__all_sync(0xffffffffu, ok)) break;
          tc_fence_after();
        }
      }
      if (__any_sync(0xffffffffu, alpha != 1.0f)) {
        // O_t (and the FP8 row sum) x alpha: FP8 columns [0,64) and [OV1, OV1 + 64)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t col = FP8 ? (c < 2 ? c * 32 : C::OV1 + (c - 2) * 32) : c * 32;
          uint32_t o[32];
          tmem_ld32(to + col, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(to + col, o);
        }
        if constexpr (FP8) {
          uint32_t rs;
          tmem_ld1(to + C::RS, rs);
          tmem_wait_ld();
          tmem_st1(to + C::RS, __float_as_uint(__uint_as_float(rs) * alpha));
        }
      }
      if constexpr (!FP8 && C::PSMEM) {
        // row r of P_t: 128 bf16 = 16 chunks of 16 B; chunk c in 128-B box c / 8 at chunk
        // position (c mod 8) ^ (r mod 8) of the row
        const uint32_t prow = smem_addr(smem + C::OFF_P + t * C::P_BYTES) + r * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c)
          st_shared_v4(prow + (c / 8) * C::Q_BOX_BYTES + (((c % 8) ^ (r & 7)) << 4), pw[4 * c],
                       pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
        fence_proxy_async_smem();
      } else if constexpr (!FP8) {
        tmem_st32(tp, pw);
        tmem_st32(tp + 32, pw + 32);
      } else {
        const uint32_t prow = smem_addr(smem + C::OFF_P + t * C::P_BYTES) + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(prow + ((c ^ (r & 7)) << 4), pw[4 * c], pw[4 * c + 1], pw[4 * c + 2],
                       pw[4 * c + 3]);
        fence_proxy_async_smem();
        tmem_st1(lane_base + TM::SFA(t, 0) + (warp & 3), sf_w & 0xFFu);
        tmem_st1(lane_base + TM::SFA(t, 1) + (warp & 3), sf_w >> 16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_full_l);
    }
    tmem_wait_st();
    // ------------------------------------------------------------- epilogue
    if (ok && n_t > 0) ok = mbar_wait(pv_done(t), (n_t - 1) & 1, p.err, p.timeout_ns);
    if (ok && n_t > 0 && slot_in) {
      tc_fence_after();
      uint32_t oraw[DV];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(to + (FP8 ? (c < 2 ? c * 32 : C::OV1 + (c - 2) * 32) : c * 32), oraw + c * 32);
      if constexpr (FP8) {
        uint32_t rs;
        tmem_ld1(to + C::RS, rs);
        tmem_wait_ld();
        l = __uint_as_float(rs);
      }
      tmem_wait_ld();
      float o[DV];
#pragma unroll
      for (int c = 0; c < DV; ++c) o[c] = __uint_as_float(oraw[c]);
      float inv = 1.0f / l;
      if constexpr (FP8) inv *= *p.descale_v;
      if (p.unrotate) {
#pragma unroll
        for (int hh = 1; hh < DV; hh <<= 1) {
#pragma unroll
          for (int i = 0; i < DV; ++i) {
            if ((i & hh) == 0) {
              const float u_ = o[i], w = o[i + hh];
              o[i] = u_ + w;
              o[i + hh] = u_ - w;
            }
          }
        }
        inv *= 0.08838834764831845f;
      }
      const bool row_in = !VARLEN || q_pos < seq_len;
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(tok0) + q_pos) * p.Hq + h) * DV;
#pragma unroll
      for (int c = 0; c < DV; c += 8) {
        uint4 v;
        v.x = pack_bf16x2(o[c + 0] * inv, o[c + 1] * inv);
        v.y = pack_bf16x2(o[c + 2] * inv, o[c + 3] * inv);
        v.z = pack_bf16x2(o[c + 4] * inv, o[c + 5] * inv);
        v.w = pack_bf16x2(o[c + 6] * inv, o[c + 7] * inv);
        if (row_in) *reinterpret_cast<uint4*>(orow + c) = v;
      }
      if (p.lse != nullptr && row_in) {
        float lse_v;
        if constexpr (FP8)
          lse_v = 0.69314718055994531f * (static_cast<float>(m_i) * 0.125f + __log2f(l));
        else
          lse_v = 0.69314718055994531f * (ms + __log2f(l));
        const size_t li = (VARLEN && p.cu_seqlens != nullptr)
                              ? static_cast<size_t>(h) * p.total_tokens + tok0 + q_pos
                              : (static_cast<size_t>(b) * p.Hq + h) * p.S + q_pos;
        p.lse[li] = lse_v;
      }
    }
  }
  __syncthreads();
  cluster_sync();  // the leader's MMAs into this CTA's TMEM and reads of its smem are done
  if (warp == 11) {
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
}

}  // namespace attn
