// Forward causal (prefill) attention on sm_100a with 64-key tiles: the same computation,
// roles and precisions as attn_fwd.cuh (two 128-row query slots per CTA in ping-pong,
// TMA-fed tcgen05 MMAs with TMEM accumulators, lean-P FP8 or BF16 probabilities), with key
// tiles of 64 instead of 128 so that every TMEM buffer fits without sharing columns:
//   FP8   O_0 [0,144) (value columns, row sum at 128), P scale factors of slot 0 [144,152)
//         (two buffers of 4 columns), V scale factors [152,160), O_1 [160,304), P scale
//         factors of slot 1 [304,312), S_0 [320,384), S_1 [384,448);
//   BF16  O_0 [0,128), O_1 [128,256), S_0 [256,320), S_1 [320,384), P of slot t in two
//         buffers [384 + 64 t + 32 h, +32) (bf16 pairs).
// With 128-key tiles the two slots' S accumulators overlap in TMEM (FP8) or P overwrites S
// (BF16), so a slot's next S must wait for the other slot's softmax (FP8) or for its own PV
// (BF16).  Here S_t(j+1) waits only for slot t to have read S_t(j): the S MMAs of a slot run
// while its softmax works, the PV MMAs of a tile run while the next tile's softmax works,
// and P (codes in shared memory, or bf16 in TMEM) is double-buffered, its buffer h = j mod 2
// reused two tiles later.
//
// The lean-P reading is the same with a 64-key tile: the reference max is updated per tile
// (lazily, 14-code headroom), and the tile is one 64-key block with one power-of-two shift
// ([ZYFA-mb] "Como o motor de atenção FP8 da Zyphra funciona").
//
// Roles (384 threads): warps 0-3 / 4-7 softmax of slot 0 / 1 (thread r = row r = TMEM lane
// r); warp 8 TMA producer (Q once, then K and V tiles of 64 keys through NK / NV stages);
// warp 9 issues the S MMAs; warp 10 issues the PV MMAs; warp 11 allocates TMEM.  Barriers
// that a fast producer could complete twice before the consumer waits (p_full, pv_done) are
// kept per P buffer, so every wait is on the phase just after the last one it saw.  Every
// wait is bounded (mbar_wait): on expiry the CTA records DEV_TIMEOUT and unwinds.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_fwd.cuh"
#include "ptx.cuh"

namespace attn {

constexpr int KT = 64;  // keys per tile

template <bool FP8>
struct TmemMap64 {
  __host__ __device__ static constexpr uint32_t O(int t) { return FP8 ? 160u * t : 128u * t; }
  __host__ __device__ static constexpr uint32_t S(int t) { return FP8 ? 320u + 64u * t : 256u + 64u * t; }
  __host__ __device__ static constexpr uint32_t SFA(int t, int h) { return (t ? 304u : 144u) + 4u * h; }
  static constexpr uint32_t SFB = 152;
  __host__ __device__ static constexpr uint32_t P(int t, int h) { return 384u + 64u * t + 32u * h; }
  static constexpr uint32_t RS = 128;
  static constexpr uint32_t PV_N = FP8 ? 144 : 128;
};
static_assert(TmemMap64<true>::S(1) + 64 <= 512 && TmemMap64<true>::SFA(1, 1) + 4 <= TmemMap64<true>::S(0),
              "FP8 TMEM map");
static_assert(TmemMap64<false>::P(1, 1) + 32 == 512, "BF16 TMEM map");

template <bool FP8, int DQK>
struct Cfg64 {
  static constexpr int E = FP8 ? 1 : 2;
  static constexpr int BOX_COLS = 128 / E;                 // elements per 128-B box row
  static constexpr int Q_BOXES = (DQK * E + 127) / 128;    // 128-B column boxes of Q and K
  static constexpr int V_BOXES = DV * E / 128;
  static constexpr int Q_BOX_BYTES = 128 * 128;            // 128 rows x 128 B
  static constexpr int KV_BOX_BYTES = KT * 128;            // 64 keys x 128 B
  static constexpr int Q_BYTES = Q_BOXES * Q_BOX_BYTES;
  static constexpr int K_BYTES = Q_BOXES * KV_BOX_BYTES;
  static constexpr int V_BYTES = V_BOXES * KV_BOX_BYTES;
  static constexpr int NK = FP8 ? (DQK == 128 ? 8 : 4) : (DQK == 128 ? 4 : 3);
  static constexpr int NV = NK;
  static constexpr int KSTEP = FP8 ? 32 : 16;
  static constexpr int QK_STEPS = DQK / KSTEP;
  static constexpr int PV_STEPS = KT / KSTEP;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * K_BYTES;
  static constexpr int OFF_ONES = OFF_V + NV * V_BYTES;            // FP8: 64 keys x 128 B of 1.0
  static constexpr int OFF_P = OFF_ONES + (FP8 ? KV_BOX_BYTES : 0);  // FP8: P_0, P_1
  static constexpr int OFF_BAR = OFF_P + (FP8 ? 2 * Q_BOX_BYTES : 0);
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV]; per slot: s_full, s_read,
  // p_full[2], pv_done[2]; mma_done[2]
  static constexpr int NUM_BARS = 1 + 2 * NK + 2 * NV + 2 * 6 + 2;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static_assert(SMEM_ALLOC <= 232448, "shared memory per block exceeded");
  static constexpr uint32_t IDESC_S = idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, 0u, 0u, BLOCK_M, KT);
  static constexpr uint32_t IDESC_PV_BF16 = idesc_dense(1u, 1u, 0u, 1u, BLOCK_M, DV);
};

template <bool FP8, int DQK, bool DUMP, bool EXACT = false, bool VARLEN = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_k64_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg64<FP8, DQK>;
  using TM = TmemMap64<FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::NK;
  uint64_t* v_full = k_empty + C::NK;
  uint64_t* v_empty = v_full + C::NV;
  uint64_t* tbar = v_empty + C::NV;  // per slot: 6 barriers
  auto s_full = [&](int t) { return tbar + 6 * t + 0; };
  auto s_read = [&](int t) { return tbar + 6 * t + 1; };
  auto p_full = [&](int t, int h) { return tbar + 6 * t + 2 + h; };
  auto pv_done = [&](int t, int h) { return tbar + 6 * t + 4 + h; };
  uint64_t* mma_done = tbar + 12;  // [2]
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEMPTR);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // units as in attn_fwd.cuh: two query tiles of one head, or one query tile of two heads
  // of one kv group; longest first
  const bool hp = p.head_pairs != 0;
  const int heads_per_unit = hp ? p.Hq / 2 : p.Hq;
  const int nbh = p.B * heads_per_unit;
  const int pr = p.n_pairs - 1 - static_cast<int>(blockIdx.x) / nbh;
  const int bh = static_cast<int>(blockIdx.x) % nbh;
  const int b = bh / heads_per_unit;
  const int h = hp ? 2 * (bh % heads_per_unit) : bh % heads_per_unit;  // head of slot 0
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
        return;
      }
      tok0 = c0;
      seq_len = c1 - c0;
    }
    n_q_tiles = (seq_len + BLOCK_M - 1) / BLOCK_M;
    if ((hp ? pr : 2 * pr) >= n_q_tiles) return;
  }
  const int n_k_tiles = (seq_len + KT - 1) / KT;       // key tiles of the sequence
  const int qt0 = hp ? pr : 2 * pr;
  const int qt1 = hp ? pr : 2 * pr + 1;
  const bool has1 = qt1 < n_q_tiles;
  // key tiles of each slot: causal, the query tile's rows see keys up to 128 qt + 127
  const int n_t0 = p.causal ? min(2 * qt0 + 2, n_k_tiles) : n_k_tiles;
  const int n_t1 = has1 ? (p.causal ? min(2 * qt1 + 2, n_k_tiles) : n_k_tiles) : 0;
  const int n_max = n_t1 > n_t0 ? n_t1 : n_t0;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::NK; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < C::NV; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(s_read(t), 128);
      for (int hh = 0; hh < 2; ++hh) {
        mbar_init(p_full(t, hh), 128);
        mbar_init(pv_done(t, hh), 1);
      }
    }
    mbar_init(mma_done + 0, 1);
    mbar_init(mma_done + 1, 1);
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
  }
  if constexpr (FP8) {
    // the ones block (e4m3 1.0) that extends every V tile to N = 144 for the row sum
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::OFF_ONES);
    for (int i = tid; i < C::KV_BOX_BYTES / 4; i += NUM_THREADS) ones[i] = 0x38383838u;
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
    if (warp == 8) {
      // ----------------------------------------------------------- TMA producer
      bool ok = true;
      const uint64_t pol_once = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      if (elect_one()) {
        mbar_arrive_expect_tx(q_full, (has1 ? 2 : 1) * C::Q_BYTES);
        for (int t = 0; t < (has1 ? 2 : 1); ++t)
          for (int i = 0; i < C::Q_BOXES; ++i)
            tma_load_3d_hint(smem + C::OFF_Q + t * C::Q_BYTES + i * C::Q_BOX_BYTES, &tm_q,
                             q_full, i * C::BOX_COLS, hp ? h + t : h,
                             tok0 + (t ? qt1 : qt0) * BLOCK_M, pol_once);
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
            tma_load_3d_hint(smem + C::OFF_K + sk * C::K_BYTES + i * C::KV_BOX_BYTES, &tm_k,
                             k_full + sk, i * C::BOX_COLS, g, tok0 + j * KT, pol_keep);
        }
        __syncwarp();
        jk = j + 1;
        const int sv = j % C::NV;
        if (j >= C::NV) ok = mbar_wait(v_empty + sv, ((j / C::NV) - 1) & 1, p.err, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(v_full + sv, C::V_BYTES);
          for (int i = 0; i < C::V_BOXES; ++i)
            tma_load_3d_hint(smem + C::OFF_V + sv * C::V_BYTES + i * C::KV_BOX_BYTES, &tm_v,
                             v_full + sv, i * C::BOX_COLS, g, tok0 + j * KT, pol_keep);
        }
        __syncwarp();
        jv = j + 1;
      }
      mbar_wait(q_full, 0, p.err, DRAIN_TIMEOUT_NS, false);
      for (int jj = (jk > C::NK ? jk - C::NK : 0); jj < jk; ++jj)
        mbar_wait(k_full + jj % C::NK, (jj / C::NK) & 1, p.err, DRAIN_TIMEOUT_NS, false);
      for (int jj = (jv > C::NV ? jv - C::NV : 0); jj < jv; ++jj)
        mbar_wait(v_full + jj % C::NV, (jj / C::NV) & 1, p.err, DRAIN_TIMEOUT_NS, false);
    } else if (warp == 9 || warp == 10) {
      // ----------------------------------------------------------- MMA issuers: warp 9 the
      // S MMAs, warp 10 the PV MMAs (disjoint TMEM columns; mbarriers order them)
      auto nt = [&](int t) { return t == 0 ? n_t0 : n_t1; };
      const uint64_t dq0 = smem_desc_sw128(smem_addr(smem + C::OFF_Q), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_addr(smem + C::OFF_K), 16, 1024);
      const uint64_t dp0 = smem_desc_sw128(smem_addr(smem + C::OFF_P), 16, 1024);  // FP8
      bool ok = true;
      if (warp == 9) {
        ok = mbar_wait(q_full, 0, p.err, p.timeout_ns);
        for (int j = 0; j < n_max && __all_sync(0xffffffffu, ok); ++j) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (j >= nt(t)) continue;
            // S_t(j) once slot t has read S_t(j-1) and K(j) has landed
            if (j > 0) ok = mbar_wait(s_read(t), (j - 1) & 1, p.err, p.timeout_ns);
            if (ok) ok = mbar_wait(k_full + j % C::NK, (j / C::NK) & 1, p.err, p.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint64_t qd = dq0 + static_cast<uint32_t>((t * C::Q_BYTES) >> 4);
            const uint64_t kd = dk0 + static_cast<uint32_t>(((j % C::NK) * C::K_BYTES) >> 4);
            if (elect_one()) {
#pragma unroll
              for (int s = 0; s < C::QK_STEPS; ++s) {
                const uint32_t oq = ((s / 4) * C::Q_BOX_BYTES + (s % 4) * 32) >> 4;
                const uint32_t ok_ = ((s / 4) * C::KV_BOX_BYTES + (s % 4) * 32) >> 4;
                mma_ss<FP8 ? 1 : 0>(tmem + TM::S(t), qd + oq, kd + ok_, C::IDESC_S, s > 0 ? 1u : 0u);
              }
              tc_commit(s_full(t));
              if (t == 1 || j >= n_t1) tc_commit(k_empty + j % C::NK);
            }
            __syncwarp();
          }
        }
        if (elect_one()) tc_commit(mma_done + 0);
        __syncwarp();
        mbar_wait(mma_done + 0, 0, p.err, DRAIN_TIMEOUT_NS, false);
      } else {
        for (int j = 0; j < n_max && __all_sync(0xffffffffu, ok); ++j) {
          const int hb = j & 1;  // P buffer of tile j
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (j >= nt(t)) continue;
            // PV_t(j) once P_t(j) is written and V(j) has landed
            ok = mbar_wait(p_full(t, hb), (j >> 1) & 1, p.err, p.timeout_ns);
            if (ok) ok = mbar_wait(v_full + j % C::NV, (j / C::NV) & 1, p.err, p.timeout_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t va = smem_addr(smem + C::OFF_V + (j % C::NV) * C::V_BYTES);
            const uint32_t tm_o = tmem + TM::O(t);
            if (elect_one()) {
              if constexpr (!FP8) {
                // V is [64 keys x 128 d] bf16, d contiguous: two 64-column atoms 8 KB apart
                const uint64_t vd = smem_desc_sw128(va, C::KV_BOX_BYTES, 1024);
                const uint32_t tm_p = tmem + TM::P(t, hb);
#pragma unroll
                for (int s = 0; s < C::PV_STEPS; ++s)
                  mma_ts_f16(tm_o, tm_p + s * 8, vd + ((s * 16 * 128) >> 4), C::IDESC_PV_BF16,
                             (j > 0 || s > 0) ? 1u : 0u);
              } else {
                // [O | row sum] += (P * 2^-(7+k)) x [V | 1]: the ones block one leading
                // offset away; P_t(j) is the half hb of each 128-B row of P_t
                const uint64_t vd = smem_desc_sw128(va, smem_addr(smem + C::OFF_ONES) - va, 1024);
                const uint64_t pd = dp0 + static_cast<uint32_t>((t * C::Q_BOX_BYTES + hb * 64) >> 4);
#pragma unroll
                for (int s = 0; s < C::PV_STEPS; ++s) {
                  const uint32_t sfa = (tmem + TM::SFA(t, hb)) | (static_cast<uint32_t>(s) << 30);
                  const uint32_t sfb = (tmem + TM::SFB) | (static_cast<uint32_t>(s) << 30);
                  mma_ss_mxf8(tm_o, pd + ((s * 32) >> 4), vd + ((s * 32 * 128) >> 4),
                              idesc_mxf8(0, 1, BLOCK_M, TM::PV_N, s, s), sfa, sfb,
                              (j > 0 || s > 0) ? 1u : 0u);
                }
              }
              tc_commit(pv_done(t, hb));
              if (t == 1 || j >= n_t1) tc_commit(v_empty + j % C::NV);
            }
            __syncwarp();
          }
        }
        if (elect_one()) tc_commit(mma_done + 1);
        __syncwarp();
        mbar_wait(mma_done + 1, 0, p.err, DRAIN_TIMEOUT_NS, false);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // ------------------------------------------------------------- softmax of slot t
    const int t = warp >> 2;
    const int n_t = t == 0 ? n_t0 : n_t1;
    const int qt = t ? qt1 : qt0;
    const int hs = hp ? h + t : h;
    const int r = tid & 127;
    const int q_pos = qt * BLOCK_M + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t ts = lane_base + TM::S(t);
    const uint32_t to = lane_base + TM::O(t);
    float a = 0.0f, a256 = 0.0f;
    if constexpr (FP8) {
      a = static_cast<float>(p.leanp_c * static_cast<double>(*p.descale_q) *
                             static_cast<double>(*p.descale_k));
      a256 = a * 0.00390625f;
      const uint32_t sfb = lane_base + TM::SFB;
      tmem_st4(sfb, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_st4(sfb + 4, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    }
    float ms = -INFINITY;
    int m_i = 0;
    float l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      const int hb = j & 1;
      ok = mbar_wait(s_full(t), j & 1, p.err, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sraw[KT];
      tmem_ld32(ts, sraw);
      tmem_ld32(ts + 32, sraw + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_read(t));  // S_t may now be overwritten by S_t(j+1)
      float s[KT];
#pragma unroll
      for (int c = 0; c < KT; ++c) s[c] = __uint_as_float(sraw[c]);
      // causal: keys past this row's position; VARLEN: keys past the end of the sequence
      const int lim = q_pos - j * KT;
      const bool diag = p.causal && lim < KT - 1;
      if (diag) {
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (c > lim) s[c] = -INFINITY;
      }
      if constexpr (VARLEN) {
        const int kvalid = seq_len - j * KT;
        if (kvalid < KT) {
#pragma unroll
          for (int c = 0; c < KT; ++c)
            if (c >= kvalid) s[c] = -INFINITY;
        }
      }
      float mx0 = s[0], mx1 = s[32];
#pragma unroll
      for (int c = 1; c < 31; c += 2) {
        mx0 = fmax3(mx0, s[c], s[c + 1]);
        mx1 = fmax3(mx1, s[32 + c], s[32 + c + 1]);
      }
      const float mu = fmaxf(fmaxf(mx0, s[31]), fmaxf(mx1, s[63]));

      uint32_t pw[FP8 ? KT / 4 : KT / 2];
      float alpha = 1.0f;
      uint32_t sf_w = 0;
      if constexpr (!FP8) {
        const float cand = mu * p.c1;
        const float ms_new = (j == 0 || cand > ms + BF16_HEADROOM) ? cand : ms;
        if (j > 0) alpha = ex2_approx(ms - ms_new);
        ms = ms_new;
        const float2 c1x2 = make_float2(p.c1, p.c1);
        const float2 nms2 = make_float2(-ms, -ms);
        float2 lsum = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int c = 0; c < KT; c += 2) {
          const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), c1x2, nms2);
          // one element pair in four on the FMA pipe, the rest on the MUFU (all on the MUFU
          // in tiles with masked keys, where x can be -inf)
          const bool poly = !diag && (c & 7) == 6;
          const float2 pp = poly ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
          lsum = __fadd2_rn(lsum, pp);
          pw[c >> 1] = pack_bf16x2(pp.x, pp.y);
        }
        l = l * alpha + (lsum.x + lsum.y);
      } else {
        const int cand = __float2int_ru(__fmul_rn(a, mu));
        const int m_new = (j == 0 || cand > m_i + LEANP_HEADROOM) ? cand : m_i;
        if (j > 0) alpha = ex2_approx(static_cast<float>(m_i - m_new) * 0.125f);
        m_i = m_new;
        const int k0 = leanp_kshift(mu, a, m_new);
        if constexpr (EXACT) {
          const float a8 = a * 0.125f;
          const float cx = __int2float_rn(8 * (7 + k0) - m_new) * 0.125f;
#pragma unroll
          for (int c = 0; c < KT; c += 4) {
            const float p0 = ex2_approx(__fmaf_rn(s[c + 0], a8, cx));
            const float p1 = ex2_approx(__fmaf_rn(s[c + 1], a8, cx));
            const float p2 = ex2_approx(__fmaf_rn(s[c + 2], a8, cx));
            const float p3 = ex2_approx(__fmaf_rn(s[c + 3], a8, cx));
            pw[c >> 2] = f32_to_e4m3x2(p0, p1) | (f32_to_e4m3x2(p2, p3) << 16);
          }
        } else {
          const float cb = __int2float_rn(LEANP_TOP + 8 * k0 - m_new) * 0.00390625f;
          const float2 s256 = make_float2(256.0f, 256.0f);
          const float2 magic = make_float2(LEANP_MAGIC, LEANP_MAGIC);
#pragma unroll
          for (int c = 0; c < KT; c += 4) {
            const float2 u01 = make_float2(fma_sat(s[c + 0], a256, cb), fma_sat(s[c + 1], a256, cb));
            const float2 u23 = make_float2(fma_sat(s[c + 2], a256, cb), fma_sat(s[c + 3], a256, cb));
            const float2 r01 = __ffma2_rn(u01, s256, magic);
            const float2 r23 = __ffma2_rn(u23, s256, magic);
            pw[c >> 2] = pack_low_bytes(__float_as_uint(r01.x), __float_as_uint(r01.y),
                                        __float_as_uint(r23.x), __float_as_uint(r23.y));
          }
        }
        const uint32_t e0 = static_cast<uint32_t>(120 - k0);
        sf_w = e0 | (e0 << 8);  // UE8M0 2^-(7+k) for both 32-key steps of the tile
        if constexpr (DUMP) {
          if (!p.causal || j <= 2 * qt + 1) {
            const size_t row = (static_cast<size_t>(b) * p.Hq + hs) * p.S + q_pos;
            float* ds = p.dump_s + row * p.S + static_cast<size_t>(j) * KT;
            uint8_t* dc = p.dump_codes + row * p.S + static_cast<size_t>(j) * KT;
            for (int c = 0; c < KT; ++c) ds[c] = s[c];
            for (int c = 0; c < KT / 4; ++c) reinterpret_cast<uint32_t*>(dc)[c] = pw[c];
            p.dump_kshift[row * (p.S / 64) + j] = static_cast<uint8_t>(k0);
          }
        }
      }
      // P buffer hb (and its scale factors) was last read by PV_t(j-2)
      if (j >= 2) {
        ok = mbar_wait(pv_done(t, hb), ((j - 2) >> 1) & 1, p.err, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      if (__any_sync(0xffffffffu, alpha != 1.0f)) {
        // O_t is rescaled once PV_t(j-1) (the last PV into it) is complete
        if (j >= 1) {
          ok = mbar_wait(pv_done(t, hb ^ 1), ((j - 1) >> 1) & 1, p.err, p.timeout_ns);
          if (!__all_sync(0xffffffffu, ok)) break;
        }
        tc_fence_after();
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(to + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 rr = __fmul2_rn(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2);
            o[i] = __float_as_uint(rr.x);
            o[i + 1] = __float_as_uint(rr.y);
          }
          tmem_st32(to + c * 32, o);
        }
        if constexpr (FP8) {
          uint32_t rs;
          tmem_ld1(to + TM::RS, rs);
          tmem_wait_ld();
          tmem_st1(to + TM::RS, __float_as_uint(__uint_as_float(rs) * alpha));
        }
      } else {
        tc_fence_after();
      }
      if constexpr (!FP8) {
        tmem_st32(lane_base + TM::P(t, hb), pw);
      } else {
        // row r of P_t(j): 64 codes = 4 chunks of 16 B at chunk positions (4 hb + c) ^ (r mod 8)
        const uint32_t prow = smem_addr(smem + C::OFF_P + t * C::Q_BOX_BYTES) + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(prow + (((4 * hb + c) ^ (r & 7)) << 4), pw[4 * c], pw[4 * c + 1],
                       pw[4 * c + 2], pw[4 * c + 3]);
        fence_proxy_async_smem();
        tmem_st1(lane_base + TM::SFA(t, hb) + (warp & 3), sf_w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(t, hb));
    }
    tmem_wait_st();
    // ------------------------------------------------------------- epilogue
    if (ok && n_t > 0)
      ok = mbar_wait(pv_done(t, (n_t - 1) & 1), ((n_t - 1) >> 1) & 1, p.err, p.timeout_ns);
    if (ok && n_t > 0) {
      tc_fence_after();
      uint32_t oraw[DV];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(to + c * 32, oraw + c * 32);
      if constexpr (FP8) {
        uint32_t rs;
        tmem_ld1(to + TM::RS, rs);
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
              const float u = o[i], w = o[i + hh];
              o[i] = u + w;
              o[i + hh] = u - w;
            }
          }
        }
        inv *= 0.08838834764831845f;
      }
      const bool row_in = !VARLEN || q_pos < seq_len;
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(tok0) + q_pos) * p.Hq + hs) * DV;
      const uint64_t pol_once = l2_policy_evict_first();
      const float2 inv2 = make_float2(inv, inv);
#pragma unroll
      for (int c = 0; c < DV; c += 8) {
        const float2 a0 = __fmul2_rn(make_float2(o[c + 0], o[c + 1]), inv2);
        const float2 a1 = __fmul2_rn(make_float2(o[c + 2], o[c + 3]), inv2);
        const float2 a2 = __fmul2_rn(make_float2(o[c + 4], o[c + 5]), inv2);
        const float2 a3 = __fmul2_rn(make_float2(o[c + 6], o[c + 7]), inv2);
        uint4 v;
        v.x = pack_bf16x2(a0.x, a0.y);
        v.y = pack_bf16x2(a1.x, a1.y);
        v.z = pack_bf16x2(a2.x, a2.y);
        v.w = pack_bf16x2(a3.x, a3.y);
        if (row_in) st_global_v4_hint(orow + c, v, pol_once);
      }
      if (p.lse != nullptr && row_in) {
        float lse_v;
        if constexpr (FP8)
          lse_v = 0.69314718055994531f * (static_cast<float>(m_i) * 0.125f + __log2f(l));
        else
          lse_v = 0.69314718055994531f * (ms + __log2f(l));
        const size_t li = (VARLEN && p.cu_seqlens != nullptr)
                              ? static_cast<size_t>(hs) * p.total_tokens + tok0 + q_pos
                              : (static_cast<size_t>(b) * p.Hq + hs) * p.S + q_pos;
        p.lse[li] = lse_v;
      }
    }
  }
  __syncthreads();
  if (warp == 11) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
