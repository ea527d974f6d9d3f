// Decode attention over a paged KV cache on sm_100a: one query token per sequence against
// every cached token of its sequence (the pages list decode and paged KV caches as work
// their kernels do not cover yet, [ZYFA-fr] "Ce que couvrent les noyaux").
//
//   o[b,h]   = sum_j softmax_j(scale <q[b,h], k_j>) v_j,  j < seq_lens[b]
//   token j of sequence b: page block_table[b][j / page_size], slot j % page_size of
//   k_cache / v_cache [num_pages, page_size, Hkv, 128]; query head h reads kv head h / G.
//
// The operation reads every cached K and V byte once and does ~2 G flops per byte (G =
// Hq / Hkv query heads share a kv head): HBM-bound, so it runs on the CUDA cores, with the
// cache streamed through shared memory by 16-byte asynchronous copies; no tensor cores.
//
// Split-KV: CTA (split, g, b) takes one kv head g of sequence b, all G query heads that read
// it, and a contiguous range of its tokens; it writes the unnormalised partial output and
// the (max, sum) of its range, and decode_combine_kernel merges the ranges.  Per 64-token
// tile (double-buffered):
//   A  scores: TPT threads per token, each with a DPT-element slice of the G queries in
//      registers (already scaled by scale * log2 e, and for FP8 by the Q and K descales),
//      reduce their partial dot products by shuffles;
//   B  per head: the tile max, the running max, alpha = 2^(m_old - m_new), p = 2^(s - m_new)
//      and the running sum (one warp per head, shuffles);
//   C  O += p V: each thread owns two value columns of all G heads.
// Page ids and sequence lengths are read on the device: entries outside the cache make the
// CTA record DEV_BAD_SEQLENS and write an empty partial instead of reading out of bounds.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace attn {

constexpr int DEC_D = 128;        // head dim of q, k and v
constexpr int DEC_TT = 64;        // tokens per tile
constexpr int DEC_THREADS = 128;

struct DecodeParams {
  const void* q;            // [B, Hq, 128] bf16 or e4m3 codes
  const uint8_t* k_cache;   // [num_pages, page_size, Hkv, 128]
  const uint8_t* v_cache;
  const int* block_table;   // [B, max_blocks]
  const int* seq_lens;      // [B]
  int B, Hq, Hkv, G;
  int num_pages, page_shift, max_blocks, max_seqlen;
  int n_splits, split_tokens;  // tokens per split: a multiple of DEC_TT
  float qk_scale;              // scale * log2(e) (FP8: times the Q and K descales later)
  const float* descale_q;
  const float* descale_k;
  const float* descale_v;
  float* part_o;    // [B, Hq, n_splits, 128] unnormalised
  float* part_ml;   // [B, Hq, n_splits, 2] (max in log2 units, sum)
  __nv_bfloat16* o; // [B, Hq, 128]
  float* lse;       // [B, Hq] or null
  uint32_t* err;
};

template <bool FP8>
struct DecCfg {
  static constexpr int E = FP8 ? 1 : 2;
  static constexpr int ROW = DEC_D * E;          // bytes of one token's K (or V) row
  static constexpr int CHUNKS = ROW / 16;        // 16-byte chunks per row
  static constexpr int TILE_BYTES = DEC_TT * ROW;
};

// dynamic shared memory of decode_split_kernel<FP8, G>: K and V tiles (double-buffered),
// the queries, the scores / probabilities, per-head state and the half-sum exchange
template <bool FP8, int G>
constexpr int dec_smem_bytes() {
  return 4 * DecCfg<FP8>::TILE_BYTES + (G * DEC_D + DEC_TT * G + 3 * G + G * DEC_D) * 4;
}

// split-KV policy: about four CTAs per SM of a 148-SM B200 over B x Hkv (sequence, kv head)
// pairs, each split at least two tiles; tokens per split a multiple of the tile
inline int dec_n_splits(int B, int Hkv, int max_seqlen) {
  const int tiles = (max_seqlen + DEC_TT - 1) / DEC_TT;
  const long long pairs = static_cast<long long>(B) * Hkv;
  long long want = pairs > 0 ? (4 * 148 + pairs - 1) / pairs : 1;
  const long long cap = tiles / 2 > 1 ? tiles / 2 : 1;
  if (want > cap) want = cap;
  return static_cast<int>(want < 1 ? 1 : want);
}
inline int dec_split_tokens(int max_seqlen, int n_splits) {
  const int tiles = (max_seqlen + DEC_TT - 1) / DEC_TT;
  return ((tiles + n_splits - 1) / n_splits) * DEC_TT;
}

// 16-byte chunk c of token row j of a tile, XOR-swizzled so that the reads of phase A (8 or
// more tokens x consecutive chunks) and C (one row, consecutive words) spread over banks
template <bool FP8>
__device__ __forceinline__ int dec_chunk_off(int j, int c) {
  using C = DecCfg<FP8>;
  return j * C::ROW + ((c ^ (j & (C::CHUNKS - 1))) << 4);
}

__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 8 elements of a 16-byte chunk (bf16 x8, or the low 8 bytes as e4m3 x8) to float
template <bool FP8>
__device__ __forceinline__ void dec_unpack8(const uint4& w, float* f) {
  if constexpr (!FP8) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(u[i] << 16);
      f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
  } else {
    const uint32_t u[2] = {w.x, w.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const uint16_t pair = static_cast<uint16_t>(u[i] >> (16 * hlf));
        uint32_t h2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
        const __half2 hv = *reinterpret_cast<const __half2*>(&h2);
        f[4 * i + 2 * hlf] = __low2float(hv);
        f[4 * i + 2 * hlf + 1] = __high2float(hv);
      }
    }
  }
}

// G query heads per kv head; DPT elements of d per thread in phase A
template <bool FP8, int G>
__global__ void __launch_bounds__(DEC_THREADS)
    decode_split_kernel(const DecodeParams p) {
  using C = DecCfg<FP8>;
  constexpr int DPT = G <= 4 ? 32 : (G == 8 ? 16 : 8);
  constexpr int TPT = DEC_D / DPT;               // threads per token in phase A
  constexpr int TOK_PER_PASS = DEC_THREADS / TPT;
  constexpr int PASSES = DEC_TT / TOK_PER_PASS;
  constexpr int SLICE_BYTES = DPT * C::E;        // bytes of a token row per thread in phase A
  constexpr int LOAD_BYTES = SLICE_BYTES < 16 ? SLICE_BYTES : 16;
  constexpr int LOAD_ELEMS = LOAD_BYTES / C::E;

  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t* kbuf = dsm;                                   // [2][TILE_BYTES]
  uint8_t* vbuf = dsm + 2 * C::TILE_BYTES;               // [2][TILE_BYTES]
  float* q_s = reinterpret_cast<float*>(dsm + 4 * C::TILE_BYTES);   // [G][128]
  float* s_s = q_s + G * DEC_D;                          // [DEC_TT][G] scores, then p
  float* hm = s_s + DEC_TT * G;                          // [G] running max (log2 units)
  float* hl = hm + G;                                    // [G] running sum
  float* ha = hl + G;                                    // [G] alpha of this tile
  float* ored = ha + G;                                  // [G][128] half-sum exchange

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = p.seq_lens[b];
  const int t_begin = split * p.split_tokens;
  const int t_end = min(len, t_begin + p.split_tokens);
  const size_t pidx = (static_cast<size_t>(b) * p.Hq + g * G) * p.n_splits + split;

  // ---- validate this CTA's sequence length and pages before any cache read
  bool bad = len < 0 || len > p.max_seqlen || len > (p.max_blocks << p.page_shift);
  const int* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
  if (!bad && t_begin < t_end) {
    const int blk0 = t_begin >> p.page_shift, blk1 = (t_end - 1) >> p.page_shift;
    for (int i = blk0 + tid; i <= blk1; i += DEC_THREADS) {
      const int pg = table[i];
      if (pg < 0 || pg >= p.num_pages) bad = true;
    }
  }
  bad = __syncthreads_or(bad);
  if (bad || t_begin >= t_end) {
    // an empty partial: max -inf, sum 0, o 0
    for (int i = tid; i < G * DEC_D; i += DEC_THREADS)
      p.part_o[(pidx + static_cast<size_t>(i / DEC_D) * p.n_splits) * DEC_D + i % DEC_D] = 0.0f;
    if (tid < G) {
      float* ml = p.part_ml + (pidx + static_cast<size_t>(tid) * p.n_splits) * 2;
      ml[0] = -INFINITY;
      ml[1] = 0.0f;
    }
    if (bad && tid == 0) atomicCAS(p.err, DEV_OK, DEV_BAD_SEQLENS);
    return;
  }

  // ---- queries of the G heads, scaled into log2 units
  float qs = p.qk_scale;
  if constexpr (FP8) qs *= *p.descale_q * *p.descale_k;
  for (int i = tid; i < G * DEC_D; i += DEC_THREADS) {
    const size_t qi = (static_cast<size_t>(b) * p.Hq + g * G) * DEC_D + i;
    float x;
    if constexpr (FP8) {
      uint32_t h2;
      const uint16_t pair = static_cast<const uint8_t*>(p.q)[qi];
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
      x = __low2float(*reinterpret_cast<const __half2*>(&h2));
    } else {
      x = __bfloat162float(static_cast<const __nv_bfloat16*>(p.q)[qi]);
    }
    q_s[i] = x * qs;
  }
  if (tid < G) {
    hm[tid] = -INFINITY;
    hl[tid] = 0.0f;
  }

  // ---- tile loader: rows of tokens [t0, t0 + 64) of kv head g, 16-byte chunks
  const uint32_t kbuf_a = smem_addr(kbuf), vbuf_a = smem_addr(vbuf);
  const size_t head_off = static_cast<size_t>(g) * C::ROW;
  const size_t tok_stride = static_cast<size_t>(p.Hkv) * C::ROW;
  const int pmask = (1 << p.page_shift) - 1;
  auto load_tile = [&](int t0, int buf) {
    for (int i = tid; i < DEC_TT * C::CHUNKS; i += DEC_THREADS) {
      const int j = i / C::CHUNKS, c = i % C::CHUNKS;
      int t = t0 + j;
      if (t >= t_end) t = t_end - 1;  // tail rows: a valid row, masked in phase A
      const size_t row = (static_cast<size_t>(table[t >> p.page_shift]) << p.page_shift) + (t & pmask);
      const size_t go = row * tok_stride + head_off + c * 16;
      const uint32_t so = buf * C::TILE_BYTES + dec_chunk_off<FP8>(j, c);
      cp_async16(kbuf_a + so, p.k_cache + go);
      cp_async16(vbuf_a + so, p.v_cache + go);
    }
    cp_async_commit();
  };

  const int n_tiles = (t_end - t_begin + DEC_TT - 1) / DEC_TT;
  load_tile(t_begin, 0);
  __syncthreads();  // q_s, hm, hl

  // phase A mapping and the query slice in registers
  const int a_tok = tid / TPT, a_part = tid % TPT;
  float qr[G][DPT];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPT; ++e) qr[h][e] = q_s[h * DEC_D + a_part * DPT + e];
  // phase C mapping: value columns 2 ce, 2 ce + 1, tokens of parity cpar
  const int ce = tid & 63, cpar = tid >> 6;
  float acc[G][2];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = 0.0f;

  for (int it = 0; it < n_tiles; ++it) {
    const int buf = it & 1;
    const int t0 = t_begin + it * DEC_TT;
    if (it + 1 < n_tiles) {
      load_tile(t0 + DEC_TT, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint8_t* kt = kbuf + buf * C::TILE_BYTES;
    const uint8_t* vt = vbuf + buf * C::TILE_BYTES;

    // ---- A: scores of the tile
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int j = ps * TOK_PER_PASS + a_tok;
      float part[G];
#pragma unroll
      for (int h = 0; h < G; ++h) part[h] = 0.0f;
#pragma unroll
      for (int lb = 0; lb < SLICE_BYTES; lb += LOAD_BYTES) {
        // bytes [a_part * SLICE_BYTES + lb, + LOAD_BYTES) of row j
        const int byte = a_part * SLICE_BYTES + lb;
        const uint8_t* src = kt + dec_chunk_off<FP8>(j, byte >> 4) + (byte & 15);
        float kf[16];
        if constexpr (LOAD_BYTES == 16) {
          const uint4 w = *reinterpret_cast<const uint4*>(src);
          if constexpr (FP8) {
            dec_unpack8<true>(w, kf);
            dec_unpack8<true>(make_uint4(w.z, w.w, 0, 0), kf + 8);
          } else {
            dec_unpack8<false>(w, kf);
          }
        } else {
          const uint2 w = *reinterpret_cast<const uint2*>(src);  // FP8, 8 elements
          dec_unpack8<true>(make_uint4(w.x, w.y, 0, 0), kf);
        }
#pragma unroll
        for (int e = 0; e < LOAD_ELEMS; ++e)
#pragma unroll
          for (int h = 0; h < G; ++h)
            part[h] = __fmaf_rn(qr[h][lb / C::E + e], kf[e], part[h]);
      }
#pragma unroll
      for (int off = 1; off < TPT; off <<= 1)
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] += __shfl_xor_sync(0xffffffffu, part[h], off);
      if (a_part == 0) {
        const bool in = t0 + j < t_end;
#pragma unroll
        for (int h = 0; h < G; ++h) s_s[j * G + h] = in ? part[h] : -INFINITY;
      }
    }
    __syncthreads();

    // ---- B: per-head tile softmax in log2 units
    for (int h = warp; h < G; h += DEC_THREADS / 32) {
      const float s0 = s_s[lane * G + h], s1 = s_s[(lane + 32) * G + h];
      float mt = fmaxf(s0, s1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_old = hm[h];
      const float m_new = fmaxf(m_old, mt);
      const float p0 = ex2_approx(s0 - m_new), p1 = ex2_approx(s1 - m_new);
      s_s[lane * G + h] = p0;
      s_s[(lane + 32) * G + h] = p1;
      float ls = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
      __syncwarp();
      if (lane == 0) {
        const float alpha = ex2_approx(m_old - m_new);  // 0 on the first tile
        ha[h] = alpha;
        hl[h] = hl[h] * alpha + ls;
        hm[h] = m_new;
      }
    }
    __syncthreads();

    // ---- C: O += p V over the tokens of this thread's parity
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float a = ha[h];
      acc[h][0] *= a;
      acc[h][1] *= a;
    }
#pragma unroll 4
    for (int j = cpar; j < DEC_TT; j += 2) {
      float v0, v1;
      if constexpr (FP8) {
        const uint16_t pair = *reinterpret_cast<const uint16_t*>(
            vt + dec_chunk_off<true>(j, (2 * ce) >> 4) + ((2 * ce) & 15));
        uint32_t h2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
        const __half2 hv = *reinterpret_cast<const __half2*>(&h2);
        v0 = __low2float(hv);
        v1 = __high2float(hv);
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(
            vt + dec_chunk_off<false>(j, (4 * ce) >> 4) + ((4 * ce) & 15));
        v0 = __uint_as_float(w << 16);
        v1 = __uint_as_float(w & 0xffff0000u);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pj = s_s[j * G + h];
        acc[h][0] = __fmaf_rn(pj, v0, acc[h][0]);
        acc[h][1] = __fmaf_rn(pj, v1, acc[h][1]);
      }
    }
    __syncthreads();  // this buffer is refilled two tiles later; s_s is rewritten
  }

  // ---- the two token parities, then the partial output of this range
  if (cpar == 1) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      ored[h * DEC_D + 2 * ce] = acc[h][0];
      ored[h * DEC_D + 2 * ce + 1] = acc[h][1];
    }
  }
  __syncthreads();
  if (cpar == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float* po = p.part_o + (pidx + static_cast<size_t>(h) * p.n_splits) * DEC_D + 2 * ce;
      po[0] = acc[h][0] + ored[h * DEC_D + 2 * ce];
      po[1] = acc[h][1] + ored[h * DEC_D + 2 * ce + 1];
    }
  }
  if (tid < G) {
    float* ml = p.part_ml + (pidx + static_cast<size_t>(tid) * p.n_splits) * 2;
    ml[0] = hm[tid];
    ml[1] = hl[tid];
  }
}

// o[b,h] = sum_s 2^(m_s - m) o_s / sum_s 2^(m_s - m) l_s  (times the V descale for FP8);
// lse = ln 2 (m + log2 sum_s 2^(m_s - m) l_s).  An empty sequence gives o = 0, lse = -inf.
template <bool FP8>
__global__ void __launch_bounds__(DEC_D) decode_combine_kernel(const DecodeParams p) {
  const int bh = blockIdx.x;
  const int e = threadIdx.x;
  const float* ml = p.part_ml + static_cast<size_t>(bh) * p.n_splits * 2;
  float m = -INFINITY;
  for (int s = 0; s < p.n_splits; ++s) m = fmaxf(m, ml[2 * s]);
  float o = 0.0f, l = 0.0f;
  if (m != -INFINITY) {
    for (int s = 0; s < p.n_splits; ++s) {
      const float w = ex2_approx(ml[2 * s] - m);
      l = __fmaf_rn(w, ml[2 * s + 1], l);
      o = __fmaf_rn(w, p.part_o[(static_cast<size_t>(bh) * p.n_splits + s) * DEC_D + e], o);
    }
    o /= l;
    if constexpr (FP8) o *= *p.descale_v;
  }
  p.o[static_cast<size_t>(bh) * DEC_D + e] = __float2bfloat16_rn(o);
  if (e == 0 && p.lse != nullptr)
    p.lse[bh] = m == -INFINITY ? -INFINITY : 0.69314718055994531f * (m + __log2f(l));
}

}  // namespace attn
