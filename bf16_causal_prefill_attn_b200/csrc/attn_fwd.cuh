// Forward causal (prefill) attention on sm_100a: TMA-fed tcgen05 MMAs with TMEM
// accumulators, warp-specialised.
//
// Computes O = softmax(mask(Q K^T * scale)) V for one 128-row query tile per CTA
// (the forward causal attention of the prefill phase, [ZYFA-fr] "Ce que couvrent les
// noyaux"), in two precisions:
//   BF16  S = Q K^T (kind::f16, fp32 accumulate); P = exp2((S - M) * scale * log2 e) in
//         fp32, rounded to bf16 for O += P V; the row sum is accumulated in fp32.
//   FP8   S = Q K^T on e4m3 codes (kind::f8f6f4); P is produced without an exponential by
//         the lean-P encoding ([ZYFA-mb] "Como o motor de atenção FP8 da Zyphra
//         funciona": one multiply-add and an integer conversion write the e4m3 bit
//         pattern), each 64-key block carries a power-of-two shift that the block-scaled
//         MMA (kind::mxf8f6f4.block_scale, UE8M0 scale per 32 keys) removes, and the row
//         normaliser is the sum of the rounded probabilities formed by one extra MMA per
//         key tile against a matrix of ones.
//
// Roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r of the tile (TMEM lane r); reads S,
//              updates the running max, rescales O in TMEM when the max grows, writes P
//              (and the FP8 scale factors) to TMEM, and finally writes O and lse.
//   warp 4     TMA producer: Q once, then K and V tiles through an NST-stage ring.
//   warp 5     TMEM allocator and MMA issuer (one thread): S(j+1) is issued before
//              PV(j) so the tensor core computes the next scores while the softmax warps
//              turn S(j) into P(j).
// TMEM (512 columns x 128 lanes, fp32): S double buffer [0,256), O [256,384), P at 384
// (bf16: 64 columns, e4m3: 32), and for FP8 the row-sum accumulator at 448 (16 columns),
// scale factors of P at 464 (4 columns) and of V / ones at 468 (4 columns).
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
constexpr int NUM_THREADS = 192;
constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_P = 384, TM_RS = 448, TM_SFA = 464, TM_SFB = 468;
constexpr float LEANP_MAGIC = 12582912.0f;  // 1.5 * 2^23
constexpr int LEANP_KMAX = 16;

struct FwdParams {
  int B, S, Hq, Hkv, G;
  int n_q_tiles;
  int causal;
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
  float* dump_s;      // FP8 debug: raw scores [B, Hq, S, S]
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
  static constexpr int NST = FP8 ? 3 : 2;                       // K/V ring depth
  static constexpr int KSTEP = FP8 ? 32 : 16;                   // MMA K per instruction
  static constexpr int QK_STEPS = DQK / KSTEP;
  static constexpr int PV_STEPS = BLOCK_N / KSTEP;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NST * K_BYTES;
  static constexpr int OFF_ONES = OFF_V + NST * V_BYTES;        // FP8: 16 x 128 B of 1.0
  static constexpr int OFF_BAR = OFF_ONES + (FP8 ? 2048 : 0);
  // barriers: q_full, k_full[NST], k_empty[NST], v_full[NST], v_empty[NST], s_full[2],
  //           s_empty[2], p_full, o_done, sf_bar, mma_done
  static constexpr int NUM_BARS = 1 + 4 * NST + 4 + 4;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_SF = (OFF_TMEMPTR + 4 + 15) / 16 * 16;  // [2][128] u32
  static constexpr int SMEM_BYTES = OFF_SF + 2 * 128 * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;           // 1024-B alignment slack
  static constexpr uint32_t IDESC_S =
      idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, 0u, 0u, BLOCK_M, BLOCK_N);
  static constexpr uint32_t IDESC_PV_BF16 = idesc_dense(1u, 1u, 0u, 1u, BLOCK_M, DV);
};

// k'_b: power-of-two shift of one 64-key block (block max mu, reference m in byte units)
__device__ __forceinline__ int leanp_kshift(float mu, float a, int m) {
  float t = __fmaf_rn(mu, a, -__int2float_rn(m));
  float g = -t * 0.125f;
  int k = __float2int_rd(g);  // saturating: +inf -> INT_MAX
  return min(max(k, 0), LEANP_KMAX);
}

template <bool FP8, int DQK, bool DUMP>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<FP8, DQK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::NST;
  uint64_t* v_full = k_empty + C::NST;
  uint64_t* v_empty = v_full + C::NST;
  uint64_t* s_full = v_empty + C::NST;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* sf_bar = o_done + 1;
  uint64_t* mma_done = sf_bar + 1;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEMPTR);
  uint32_t* sf_x = reinterpret_cast<uint32_t*>(smem + C::OFF_SF);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // longest-processing-time order: the longest query tiles (largest causal extent) first
  const int nbh = p.B * p.Hq;
  const int qt = p.n_q_tiles - 1 - static_cast<int>(blockIdx.x) / nbh;
  const int bh = static_cast<int>(blockIdx.x) % nbh;
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int g = h / p.G;
  const int n_kv = p.causal ? qt + 1 : p.n_q_tiles;
  const int tok0 = b * p.S;  // first token of this batch entry

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_empty + i, 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(sf_bar, 128);
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if constexpr (FP8) {
    // ones matrix (e4m3 1.0 = 0x38) for the row-sum MMA, visible to the async proxy
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::OFF_ONES);
    for (int i = tid; i < 512; i += NUM_THREADS) ones[i] = 0x38383838u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;

  if (warp == 4) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int i = 0; i < C::Q_BOXES; ++i)
        tma_load_3d(smem + C::OFF_Q + i * C::BOX_BYTES, &tm_q, q_full, i * C::BOX_COLS, h,
                    tok0 + qt * BLOCK_M);
      int j = 0;
      bool v_issued_last = true;  // whether the V load of tile j-1 was issued
      for (; j < n_kv && ok; ++j) {
        const int st = j % C::NST;
        const uint32_t use = j / C::NST;
        if (j >= C::NST) ok = mbar_wait(k_empty + st, (use - 1) & 1, p.err, p.timeout_ns);
        if (!ok) break;
        mbar_arrive_expect_tx(k_full + st, C::K_BYTES);
        for (int i = 0; i < C::Q_BOXES; ++i)
          tma_load_3d(smem + C::OFF_K + st * C::K_BYTES + i * C::BOX_BYTES, &tm_k, k_full + st,
                      i * C::BOX_COLS, g, tok0 + j * BLOCK_N);
        if (j >= C::NST) ok = mbar_wait(v_empty + st, (use - 1) & 1, p.err, p.timeout_ns);
        if (!ok) {
          ++j;  // the K load of this tile is in flight, its V load is not
          v_issued_last = false;
          break;
        }
        mbar_arrive_expect_tx(v_full + st, C::V_BYTES);
        for (int i = 0; i < C::V_BOXES; ++i)
          tma_load_3d(smem + C::OFF_V + st * C::V_BYTES + i * C::BOX_BYTES, &tm_v, v_full + st,
                      i * C::BOX_COLS, g, tok0 + j * BLOCK_N);
      }
      // drain: make sure no copy issued by this CTA is still in flight at exit
      mbar_wait(q_full, 0, p.err, DRAIN_TIMEOUT_NS, false);
      for (int jj = (j > C::NST ? j - C::NST : 0); jj < j; ++jj) {
        const int st = jj % C::NST;
        mbar_wait(k_full + st, (jj / C::NST) & 1, p.err, DRAIN_TIMEOUT_NS, false);
        if (jj < j - 1 || v_issued_last)
          mbar_wait(v_full + st, (jj / C::NST) & 1, p.err, DRAIN_TIMEOUT_NS, false);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, p.err, p.timeout_ns);
      const uint32_t q_base = smem_addr(smem + C::OFF_Q);
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj % C::NST;
        if (!mbar_wait(p_full, jj & 1, p.err, p.timeout_ns)) return false;
        if (!mbar_wait(v_full + st, (jj / C::NST) & 1, p.err, p.timeout_ns)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_addr(smem + C::OFF_V + st * C::V_BYTES);
        if constexpr (!FP8) {
#pragma unroll
          for (int s = 0; s < C::PV_STEPS; ++s) {
            // V is [keys x d] with d contiguous: B operand MN-major; 8-key groups 1 KB apart,
            // 64-column atoms 16 KB apart
            const uint64_t bdesc = smem_desc_sw128(v_base + s * 2048, C::BOX_BYTES, 1024);
            mma_ts_f16(tmem + TM_O, tmem + TM_P + s * 8, bdesc, C::IDESC_PV_BF16,
                       (jj > 0 || s > 0) ? 1u : 0u);
          }
        } else {
          const uint32_t ones_base = smem_addr(smem + C::OFF_ONES);
#pragma unroll
          for (int s = 0; s < C::PV_STEPS; ++s) {
            const uint64_t bdesc = smem_desc_sw128(v_base + s * 4096, C::BOX_BYTES, 1024);
            const uint32_t sfa = (tmem + TM_SFA) | (static_cast<uint32_t>(s) << 30);
            const uint32_t sfb = (tmem + TM_SFB) | (static_cast<uint32_t>(s) << 30);
            mma_ts_mxf8(tmem + TM_O, tmem + TM_P + s * 8, bdesc, idesc_mxf8(0, 1, BLOCK_M, DV, s, s),
                        sfa, sfb, (jj > 0 || s > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int s = 0; s < C::PV_STEPS; ++s) {
            // row sum of the rounded probabilities: P x ones (16 x 128 keys, K-major)
            const uint64_t odesc = smem_desc_sw128(ones_base + s * 32, 16, 1024);
            const uint32_t sfa = (tmem + TM_SFA) | (static_cast<uint32_t>(s) << 30);
            const uint32_t sfb = (tmem + TM_SFB) | (static_cast<uint32_t>(s) << 30);
            mma_ts_mxf8(tmem + TM_RS, tmem + TM_P + s * 8, odesc, idesc_mxf8(0, 0, BLOCK_M, 16, s, s),
                        sfa, sfb, (jj > 0 || s > 0) ? 1u : 0u);
          }
        }
        tc_commit(o_done);
        tc_commit(v_empty + st);
        return true;
      };
      int j = 0;
      for (; j < n_kv && ok; ++j) {
        const int st = j % C::NST;
        const int sb = j & 1;
        ok = mbar_wait(k_full + st, (j / C::NST) & 1, p.err, p.timeout_ns);
        if (ok && j >= 2) ok = mbar_wait(s_empty + sb, ((j >> 1) - 1) & 1, p.err, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t k_base = smem_addr(smem + C::OFF_K + st * C::K_BYTES);
#pragma unroll
        for (int s = 0; s < C::QK_STEPS; ++s) {
          const uint32_t off = (s / 4) * C::BOX_BYTES + (s % 4) * 32;
          const uint64_t adesc = smem_desc_sw128(q_base + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(k_base + off, 16, 1024);
          mma_ss<FP8 ? 1 : 0>(tmem + TM_S0 + sb * 128, adesc, bdesc, C::IDESC_S, s > 0 ? 1u : 0u);
        }
        tc_commit(s_full + sb);
        tc_commit(k_empty + st);
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok && j == n_kv) issue_pv(n_kv - 1);
      // all MMAs issued by this thread complete before TMEM is released
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, p.err, DRAIN_TIMEOUT_NS, false);
    }
  } else {
    // ------------------------------------------------------------- softmax warps 0-3
    const int r = tid;                       // row within the tile == TMEM lane
    const int q_pos = qt * BLOCK_M + r;      // query position in the sequence
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float a = 0.0f;  // FP8 slope, byte units per raw score
    if constexpr (FP8) {
      a = static_cast<float>(p.leanp_c * static_cast<double>(*p.descale_q) *
                             static_cast<double>(*p.descale_k));
      // B-operand scale factors: 2^0 everywhere (V and the ones matrix)
      tmem_st4(lane_base + TM_SFB, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_wait_st();
    }
    float m_f = -INFINITY;  // BF16 running max (raw scores)
    int m_i = 0;            // FP8 running max (byte units)
    float l = 0.0f;         // BF16 running row sum
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      ok = mbar_wait(s_full + sb, (j >> 1) & 1, p.err, p.timeout_ns);
      if (!ok) break;
      tc_fence_after();
      uint32_t sraw[BLOCK_N];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + TM_S0 + sb * 128 + c * 32, sraw + c * 32);
      tmem_wait_ld();
      float s[BLOCK_N];
#pragma unroll
      for (int c = 0; c < BLOCK_N; ++c) s[c] = __uint_as_float(sraw[c]);
      tc_fence_before();
      mbar_arrive(s_empty + sb);
      if (p.causal && j == qt) {
#pragma unroll
        for (int c = 0; c < BLOCK_N; ++c)
          if (c > r) s[c] = -INFINITY;
      }
      float mu0 = s[0], mu1 = s[64];
#pragma unroll
      for (int c = 1; c < 63; c += 2) {
        mu0 = fmax3(mu0, s[c], s[c + 1]);
        mu1 = fmax3(mu1, s[64 + c], s[64 + c + 1]);
      }
      mu0 = fmaxf(mu0, s[63]);
      mu1 = fmaxf(mu1, s[127]);

      uint32_t pw[FP8 ? 32 : 64];
      float alpha;
      uint32_t sf_word = 0;
      if constexpr (!FP8) {
        const float m_new = fmaxf(m_f, fmaxf(mu0, mu1));
        alpha = ex2_approx((m_f - m_new) * p.c1);
        const float mc = m_new * p.c1;
        float lsum = 0.0f;
#pragma unroll
        for (int c = 0; c < BLOCK_N; c += 2) {
          const float p0 = ex2_approx(__fmaf_rn(s[c], p.c1, -mc));
          const float p1 = ex2_approx(__fmaf_rn(s[c + 1], p.c1, -mc));
          lsum += p0 + p1;
          pw[c >> 1] = pack_bf16x2(p0, p1);
        }
        l = l * alpha + lsum;
        m_f = m_new;
      } else {
        const float mu = fmaxf(mu0, mu1);
        const int cand = __float2int_ru(__fmul_rn(a, mu));
        const int m_new = (j == 0) ? cand : max(m_i, cand);
        alpha = (j == 0) ? 0.0f : ex2_approx(static_cast<float>(m_i - m_new) * 0.125f);
        const int k0 = leanp_kshift(mu0, a, m_new);
        const int k1 = leanp_kshift(mu1, a, m_new);
        const float cb0 = LEANP_MAGIC + __int2float_rn(120 + 8 * k0 - m_new);
        const float cb1 = LEANP_MAGIC + __int2float_rn(120 + 8 * k1 - m_new);
#pragma unroll
        for (int c = 0; c < BLOCK_N; c += 4) {
          const float cb = c < 64 ? cb0 : cb1;
          const uint32_t b0 = __float_as_uint(fmaxf(__fmaf_rn(s[c + 0], a, cb), LEANP_MAGIC));
          const uint32_t b1 = __float_as_uint(fmaxf(__fmaf_rn(s[c + 1], a, cb), LEANP_MAGIC));
          const uint32_t b2 = __float_as_uint(fmaxf(__fmaf_rn(s[c + 2], a, cb), LEANP_MAGIC));
          const uint32_t b3 = __float_as_uint(fmaxf(__fmaf_rn(s[c + 3], a, cb), LEANP_MAGIC));
          pw[c >> 2] = pack_low_bytes(b0, b1, b2, b3);
        }
        const uint32_t e0 = static_cast<uint32_t>(119 - k0), e1 = static_cast<uint32_t>(119 - k1);
        sf_word = e0 | (e0 << 8) | (e1 << 16) | (e1 << 24);
        m_i = m_new;
        if constexpr (DUMP) {
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
      if constexpr (FP8) {
        // scale factors of P: the word for row R lives in column TM_SFA + R/32 at lane R%32
        // of every 32-lane quadrant (byte k = 32-key block k of the tile), so each warp
        // writes the words of all 128 rows for its own quadrant: exchange through smem
        sf_x[(j & 1) * 128 + r] = sf_word;
        mbar_arrive(sf_bar);
      }
      if (j >= 1) {
        // PV(j-1) must be complete before P, its scale factors and O are touched again
        ok = mbar_wait(o_done, (j - 1) & 1, p.err, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + TM_O + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(lane_base + TM_O + c * 32, o);
          }
          if constexpr (FP8) {
            uint32_t rs;
            tmem_ld1(lane_base + TM_RS, rs);
            tmem_wait_ld();
            tmem_st1(lane_base + TM_RS, __float_as_uint(__uint_as_float(rs) * alpha));
          }
        }
      }
      if constexpr (!FP8) {
        tmem_st32(lane_base + TM_P, pw);
        tmem_st32(lane_base + TM_P + 32, pw + 32);
      } else {
        tmem_st32(lane_base + TM_P, pw);
        ok = mbar_wait(sf_bar, j & 1, p.err, p.timeout_ns);
        if (!ok) break;
        const uint32_t* x = sf_x + (j & 1) * 128;
        tmem_st4(lane_base + TM_SFA, x[lane], x[32 + lane], x[64 + lane], x[96 + lane]);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    tmem_wait_st();  // nothing of this thread may still be writing TMEM on any exit path
    // ------------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait(o_done, (n_kv - 1) & 1, p.err, p.timeout_ns);
    if (ok) {
      tc_fence_after();
      uint32_t oraw[DV];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + TM_O + c * 32, oraw + c * 32);
      float lrow = l;
      if constexpr (FP8) {
        uint32_t rs;
        tmem_ld1(lane_base + TM_RS, rs);
        tmem_wait_ld();
        lrow = __uint_as_float(rs);
      } else {
        tmem_wait_ld();
      }
      float o[DV];
#pragma unroll
      for (int c = 0; c < DV; ++c) o[c] = __uint_as_float(oraw[c]);
      float inv = 1.0f / lrow;
      if constexpr (FP8) inv *= *p.descale_v;
      if (p.unrotate) {
        // x -> x H_128 / sqrt(128), butterfly stages h = 1, 2, ..., 64
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
      __nv_bfloat16* orow =
          p.o + ((static_cast<size_t>(tok0) + q_pos) * p.Hq + h) * DV;
#pragma unroll
      for (int c = 0; c < DV; c += 8) {
        uint4 v;
        v.x = pack_bf16x2(o[c + 0] * inv, o[c + 1] * inv);
        v.y = pack_bf16x2(o[c + 2] * inv, o[c + 3] * inv);
        v.z = pack_bf16x2(o[c + 4] * inv, o[c + 5] * inv);
        v.w = pack_bf16x2(o[c + 6] * inv, o[c + 7] * inv);
        *reinterpret_cast<uint4*>(orow + c) = v;
      }
      if (p.lse != nullptr) {
        float lse_v;
        if constexpr (FP8)
          lse_v = 0.69314718055994531f * (static_cast<float>(m_i) * 0.125f + __log2f(lrow));
        else
          lse_v = 0.69314718055994531f * (m_f * p.c1 + __log2f(lrow));
        p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.S + q_pos] = lse_v;
      }
    }
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
