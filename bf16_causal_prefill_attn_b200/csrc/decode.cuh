// Decode attention over a paged KV cache on sm_100a: one query token per sequence against
// every cached token of its sequence (the pages list decode and paged KV caches as work
// their kernels do not cover yet, [ZYFA-fr] "Ce que couvrent les noyaux").
//
//   o[b,h]   = sum_j softmax_j(scale <q[b,h], k_j>) v_j,  j < seq_lens[b]
//   token j of sequence b: page block_table[b][j / page_size], slot j % page_size of
//   k_cache / v_cache [num_pages, page_size, Hkv, 128]; query head h reads kv head h / G.
//
// The operation reads every cached K and V byte once and does ~2 G flops per byte (G =
// Hq / Hkv query heads share a kv head): HBM-bound, with the cache streamed through shared
// memory by 16-byte asynchronous copies.  What has to keep up with the copies is the
// instruction issue of the two contractions: a CUDA-core loop needs one fma per product
// (plus conversions for e4m3), which held e4m3 caches to ~3 TB/s, so both contractions are
// warp-level tensor-core MMAs (mma.sync: scores m16n8k32 e4m3 or m16n8k16 bf16, PV
// m16n8k16 f16 or bf16; each replaces 64-128 fma instructions of a warp).  The tiles are
// thin (the G heads are the MMA's 8 or 16 rows or columns): issue slots are the point,
// not the tensor throughput.
//
// Split-KV: CTA (g, split, b) takes one kv head g of sequence b, all G query heads that read
// it, and a contiguous range of its tokens; it writes the unnormalised partial output and
// the (max, sum) of its range, and decode_combine_kernel merges the ranges.  Per tile of TT
// tokens (NST tiles in flight):
//   A  scores: warp w multiplies tokens 64 m + 16 w .. + 15 (the MMA's rows) by the G
//      queries (its 8-wide columns, query fragments in registers), fp32 accumulators,
//      scaled by scale * log2 e (FP8: times the Q and K descales);
//   B  per head: the tile max, the running max, alpha = 2^(m_old - m_new), p = 2^(s - m_new)
//      and the running sum (one warp per head, shuffles);
//   C  O += p V with p rounded to 16 bits (f16 for FP8 caches, bf16 for BF16 ones; the
//      running sum adds the same rounded values): warp w owns value columns 32 w .. 32 w +
//      31 of all G heads (the heads are the MMA's rows) and all TT tokens; e4m3 values are
//      converted to f16 (exact) in registers.
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
constexpr int DEC_TT = 64;        // split unit (tokens); the kernels' tiles are multiples of it
constexpr int DEC_THREADS = 128;

struct DecodeParams {
  const void* q;            // [B, Hq, 128] bf16 or e4m3 codes
  const uint8_t* k_cache;   // [num_pages, page_size, Hkv, 128]
  const uint8_t* v_cache;
  const int* block_table;   // [B, max_blocks]
  const int* seq_lens;      // [B]
  int B, Hq, Hkv, G;
  int num_pages, page_shift, max_blocks, max_seqlen;
  int n_splits, split_tokens;  // tokens per split: a multiple of the kernel's tile
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
  static constexpr int TT = DEC_TT;              // tokens per tile
  static constexpr int PST = TT + 8;             // row stride (16-bit elements) of p [G][PST]
  static constexpr int ROW = DEC_D * E;          // bytes of one token's K (or V) row
  static constexpr int CHUNKS = ROW / 16;        // 16-byte chunks per row
  static constexpr int TILE_BYTES = TT * ROW;
  // tiles in flight per CTA (a third cost the e4m3 kernel 7%: fewer CTAs fit on an SM)
  static constexpr int NST = 2;
};

// dynamic shared memory of decode_split_kernel<FP8, G>: K and V tiles (double-buffered),
// the scores, per-head state and p in 16 bits
// (the row stride of p is padded so that the eight heads of one MMA fragment read fall in
// different banks)
template <bool FP8, int G>
constexpr int dec_smem_bytes() {
  using C = DecCfg<FP8>;
  return 2 * C::NST * C::TILE_BYTES + (C::TT * G + 3 * G) * 4 + G * C::PST * 2;
}

// split-KV policy: about sixteen CTAs per SM of a 148-SM B200 (several full waves at the
// kernel's occupancy, so the last wave's tail is small) over B x Hkv (sequence, kv head)
// pairs, each split at least two tiles; tokens per split a multiple of the tile
inline int dec_n_splits(int B, int Hkv, int max_seqlen) {
  const int tiles = (max_seqlen + DEC_TT - 1) / DEC_TT;
  const long long pairs = static_cast<long long>(B) * Hkv;
  long long want = pairs > 0 ? (16 * 148 + pairs - 1) / pairs : 1;
  const long long cap = tiles / 2 > 1 ? tiles / 2 : 1;
  if (want > cap) want = cap;
  return static_cast<int>(want < 1 ? 1 : want);
}
// tokens per split: the split of max_seqlen into n_splits ranges of whole 64-token units,
// rounded up to whole kernel tiles (trailing splits may then be empty)
template <bool FP8>
inline int dec_split_tokens(int max_seqlen, int n_splits) {
  const int tiles = (max_seqlen + DEC_TT - 1) / DEC_TT;
  const int tok = ((tiles + n_splits - 1) / n_splits) * DEC_TT;
  return (tok + DecCfg<FP8>::TT - 1) / DecCfg<FP8>::TT * DecCfg<FP8>::TT;
}

// 16-byte chunk c of token row j of a tile, XOR-swizzled so that the MMA fragment reads
// spread over the banks: phase A reads one chunk of eight consecutive rows, phase C the same
// one or two chunks of four rows two apart
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

// two e4m3 codes (low 16 bits) -> f16x2, exact
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(pair)));
  return h2;
}

// d += a b for one warp: a 16 x 32 e4m3 (row-major fragments), b 32 x 8 e4m3 (column-major),
// d 16 x 8 fp32.  Fragments (r = lane / 4, c = lane % 4): a[0] row r, elements 4c .. 4c+3;
// a[1] row r + 8, same; a[2], a[3] the same rows, elements 16 + 4c ..; b0 column r,
// elements 4c .. 4c+3, b1 column r, 16 + 4c ..; d[0], d[1] row r, columns 2c, 2c+1;
// d[2], d[3] row r + 8
__device__ __forceinline__ void mma_16832_e4m3(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
      " {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += a b for one warp: a 16 x 16 f16, or bf16 with BF (a[0] row r, elements 2c, 2c+1;
// a[1] row r + 8; a[2], a[3] the same rows, elements 2c + 8, 2c + 9), b 16 x 8 of the same
// type (b0 column r, elements 2c, 2c+1; b1 elements 2c + 8, 2c + 9), d as for
// mma_16832_e4m3
template <bool BF>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (BF) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// G query heads per kv head
template <bool FP8, int G>
__global__ void __launch_bounds__(DEC_THREADS)
    decode_split_kernel(const DecodeParams p) {
  using C = DecCfg<FP8>;
  constexpr int QNT = (G + 7) / 8;   // 8-wide MMA column tiles of heads in phase A
  constexpr int KS = FP8 ? 4 : 8;    // phase A steps of d: 32 e4m3 or 16 bf16 elements (32 bytes)
  constexpr int TT = C::TT, PST = C::PST;
  static_assert(DEC_THREADS == 128 && TT % 64 == 0, "phases A and C: four warps of 16-token MMA rows / 32 columns");

  extern __shared__ __align__(16) uint8_t dsm[];
  uint8_t* kbuf = dsm;                                   // [NST][TILE_BYTES]
  uint8_t* vbuf = dsm + C::NST * C::TILE_BYTES;          // [NST][TILE_BYTES]
  float* s_s = reinterpret_cast<float*>(dsm + 2 * C::NST * C::TILE_BYTES);  // [TT][G]
  float* hm = s_s + TT * G;                          // [G] running max (log2 units)
  float* hl = hm + G;                                    // [G] running sum
  float* ha = hl + G;                                    // [G] alpha of this tile
  uint16_t* p16 = reinterpret_cast<uint16_t*>(ha + G);   // [G][PST] p, 16-bit

  // kv head fastest: the CTAs of one (sequence, split) read the same pages (their head's
  // slice of every token row) at about the same time, which keeps DRAM rows open
  const int g = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int fr = lane >> 2, fc = lane & 3;  // MMA fragment row group and column pair
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

  // ---- the queries as the score MMA's column fragments, in registers: head 8 nt + fr,
  // bytes 32 ks + 4 fc .. + 3 and 32 ks + 16 + 4 fc .. + 3 of its row (zero for heads >= G).
  // The scale into log2 units is applied to each finished dot product.
  float qs = p.qk_scale;
  if constexpr (FP8) qs *= *p.descale_q * *p.descale_k;
  uint32_t qb[QNT][KS][2];
  {
    const uint8_t* qrow = static_cast<const uint8_t*>(p.q) + (static_cast<size_t>(b) * p.Hq + g * G) * C::ROW;
#pragma unroll
    for (int nt = 0; nt < QNT; ++nt) {
      const int h = 8 * nt + fr;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t w = 0;
          if (h < G) {
            const uint8_t* src = qrow + h * C::ROW + 32 * ks + 16 * hf + 4 * fc;
            w = static_cast<uint32_t>(src[0]) | (static_cast<uint32_t>(src[1]) << 8) |
                (static_cast<uint32_t>(src[2]) << 16) | (static_cast<uint32_t>(src[3]) << 24);
          }
          qb[nt][ks][hf] = w;
        }
    }
  }
  if (tid < G) {
    hm[tid] = -INFINITY;
    hl[tid] = 0.0f;
  }

  // ---- tile loader: rows of tokens [t0, t0 + TT) of kv head g, 16-byte chunks; thread tid
  // copies chunk lc = tid % CHUNKS of rows lj + k RSTEP.  Rows past the end of the range
  // repeat its last row (a valid one; phase A masks them).  Tiles start at multiples of TT,
  // so with pages of TT tokens or more a tile lies in one page: one page-table read per tile
  // instead of one per row.
  constexpr int RSTEP = DEC_THREADS / C::CHUNKS;
  constexpr int LK = TT / RSTEP;
  const int lc = tid % C::CHUNKS, lj = tid / C::CHUNKS;
  const uint32_t kbuf_a = smem_addr(kbuf), vbuf_a = smem_addr(vbuf);
  const size_t col_off = static_cast<size_t>(g) * C::ROW + lc * 16;
  const size_t tok_stride = static_cast<size_t>(p.Hkv) * C::ROW;
  const int pmask = (1 << p.page_shift) - 1;
  const bool one_page = (1 << p.page_shift) >= TT;
  auto load_tile = [&](int t0, int buf) {
    const int last = t_end - 1 - t0;
    if (one_page) {
      const size_t row0 = (static_cast<size_t>(table[t0 >> p.page_shift]) << p.page_shift) + (t0 & pmask);
      const uint8_t* kg = p.k_cache + row0 * tok_stride + col_off;
      const uint8_t* vg = p.v_cache + row0 * tok_stride + col_off;
#pragma unroll
      for (int k = 0; k < LK; ++k) {
        const int j = lj + k * RSTEP;
        const size_t off = static_cast<size_t>(min(j, last)) * tok_stride;
        const uint32_t so = buf * C::TILE_BYTES + dec_chunk_off<FP8>(j, lc);
        cp_async16(kbuf_a + so, kg + off);
        cp_async16(vbuf_a + so, vg + off);
      }
    } else {
#pragma unroll
      for (int k = 0; k < LK; ++k) {
        const int j = lj + k * RSTEP;
        const int t = t0 + min(j, last);
        const size_t go = ((static_cast<size_t>(table[t >> p.page_shift]) << p.page_shift) + (t & pmask)) * tok_stride + col_off;
        const uint32_t so = buf * C::TILE_BYTES + dec_chunk_off<FP8>(j, lc);
        cp_async16(kbuf_a + so, p.k_cache + go);
        cp_async16(vbuf_a + so, p.v_cache + go);
      }
    }
    cp_async_commit();
  };

  const int n_tiles = (t_end - t_begin + TT - 1) / TT;
  // prologue: the first NST - 1 tiles (an empty group where there is no tile keeps the
  // count of committed groups uniform)
#pragma unroll
  for (int st = 0; st < C::NST - 1; ++st) {
    if (st < n_tiles) load_tile(t_begin + st * TT, st);
    else cp_async_commit();
  }
  __syncthreads();  // hm, hl

  // phase C accumulators: MMA tile i (of four) of warp w, fragment element e: head
  // fr + 8 (e >> 1), value column 32 w + 8 fc + 4 (e & 1) + i
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

  for (int it = 0; it < n_tiles; ++it) {
    const int buf = it % C::NST;
    const int t0 = t_begin + it * TT;
    // tile it + NST - 1 into the buffer tile it - 1 used (every thread is past it)
    if (it + C::NST - 1 < n_tiles) load_tile(t0 + (C::NST - 1) * TT, (it + C::NST - 1) % C::NST);
    else cp_async_commit();
    cp_async_wait<C::NST - 1>();  // tile it has landed
    __syncthreads();
    const uint8_t* kt = kbuf + buf * C::TILE_BYTES;
    const uint8_t* vt = vbuf + buf * C::TILE_BYTES;

    // ---- A: scores of the tile; warp w: tokens 64 mt + 16 w .. + 15 as the MMA's rows,
    // the heads as its columns; step ks covers bytes 32 ks .. 32 ks + 31 of the rows
#pragma unroll
    for (int mt = 0; mt < TT / 64; ++mt) {
      const int j0 = 64 * mt + 16 * warp;
      float sc[QNT][4];
#pragma unroll
      for (int nt = 0; nt < QNT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t af[4];
        af[0] = *reinterpret_cast<const uint32_t*>(kt + dec_chunk_off<FP8>(j0 + fr, 2 * ks) + 4 * fc);
        af[1] = *reinterpret_cast<const uint32_t*>(kt + dec_chunk_off<FP8>(j0 + fr + 8, 2 * ks) + 4 * fc);
        af[2] = *reinterpret_cast<const uint32_t*>(kt + dec_chunk_off<FP8>(j0 + fr, 2 * ks + 1) + 4 * fc);
        af[3] = *reinterpret_cast<const uint32_t*>(kt + dec_chunk_off<FP8>(j0 + fr + 8, 2 * ks + 1) + 4 * fc);
#pragma unroll
        for (int nt = 0; nt < QNT; ++nt) {
          if constexpr (FP8) mma_16832_e4m3(sc[nt], af, qb[nt][ks][0], qb[nt][ks][1]);
          else mma_16816<true>(sc[nt], af, qb[nt][ks][0], qb[nt][ks][1]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < QNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j0 + fr + 8 * (e >> 1), h = 8 * nt + 2 * fc + (e & 1);
          if (h < G) s_s[j * G + h] = t0 + j < t_end ? sc[nt][e] * qs : -INFINITY;
        }
    }
    __syncthreads();

    // ---- B: per-head tile softmax in log2 units
    for (int h = warp; h < G; h += DEC_THREADS / 32) {
      constexpr int U = TT / 32;  // tokens lane + 32 u of the tile
      float sv[U];
      float mx = -INFINITY;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        sv[u] = s_s[(lane + 32 * u) * G + h];
        mx = fmaxf(mx, sv[u]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = hm[h];
      const float m_new = fmaxf(m_old, mx);
      // p rounded to the 16-bit type of the cached values (FP8: f16, BF16: bf16), the
      // form O += p V multiplies; the row sum adds the same rounded values
      float ls = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float pf = ex2_approx(sv[u] - m_new);
        uint16_t r;
        float pr;
        if constexpr (FP8) {
          r = __half_as_ushort(__float2half_rn(pf));
          pr = __half2float(__ushort_as_half(r));
        } else {
          r = __bfloat16_as_ushort(__float2bfloat16_rn(pf));
          pr = __bfloat162float(__ushort_as_bfloat16(r));
        }
        p16[h * PST + lane + 32 * u] = r;
        ls += pr;
      }
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

    // ---- C: O += p V.  Warp w: value columns 32 w .. 32 w + 31 as four 8-wide MMA tiles
    // (column n of tile i = value column 32 w + 4 n + i, so one read of four columns of a
    // token row feeds all four tiles), the heads as the MMA's rows, the tile's tokens in
    // 16-token steps
    {
      const float a_lo = fr < G ? ha[fr] : 1.0f, a_hi = fr + 8 < G ? ha[fr + 8] : 1.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[i][0] *= a_lo;
        acc[i][1] *= a_lo;
        acc[i][2] *= a_hi;
        acc[i][3] *= a_hi;
      }
      const int vb = (32 * warp + 4 * fr) * C::E;  // byte of this lane's four value columns
      const uint8_t* vcol = vt + (vb & 15);
      const uint32_t* pw = reinterpret_cast<const uint32_t*>(p16);
#pragma unroll
      for (int ks = 0; ks < TT / 16; ++ks) {
        const int k0 = 16 * ks + 2 * fc;  // this lane's tokens k0, k0 + 1, k0 + 8, k0 + 9
        uint32_t af[4];
        af[0] = fr < G ? pw[(fr * PST + k0) >> 1] : 0u;
        af[1] = fr + 8 < G ? pw[((fr + 8) * PST + k0) >> 1] : 0u;
        af[2] = fr < G ? pw[(fr * PST + k0 + 8) >> 1] : 0u;
        af[3] = fr + 8 < G ? pw[((fr + 8) * PST + k0 + 8) >> 1] : 0u;
        // bf[i][0]: column i of tokens (k0, k0 + 1), bf[i][1]: of tokens (k0 + 8, k0 + 9)
        uint32_t bf[4][2];
        if constexpr (FP8) {
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(vcol + dec_chunk_off<true>(k0, vb >> 4));
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(vcol + dec_chunk_off<true>(k0 + 1, vb >> 4));
          const uint32_t w2 = *reinterpret_cast<const uint32_t*>(vcol + dec_chunk_off<true>(k0 + 8, vb >> 4));
          const uint32_t w3 = *reinterpret_cast<const uint32_t*>(vcol + dec_chunk_off<true>(k0 + 9, vb >> 4));
          // byte i of the two tokens of a pair side by side, then e4m3 -> f16 (exact)
          const uint32_t lo01 = __byte_perm(w0, w1, 0x5140), hi01 = __byte_perm(w0, w1, 0x7362);
          const uint32_t lo89 = __byte_perm(w2, w3, 0x5140), hi89 = __byte_perm(w2, w3, 0x7362);
          bf[0][0] = e4m3x2_to_f16x2(lo01);
          bf[1][0] = e4m3x2_to_f16x2(lo01 >> 16);
          bf[2][0] = e4m3x2_to_f16x2(hi01);
          bf[3][0] = e4m3x2_to_f16x2(hi01 >> 16);
          bf[0][1] = e4m3x2_to_f16x2(lo89);
          bf[1][1] = e4m3x2_to_f16x2(lo89 >> 16);
          bf[2][1] = e4m3x2_to_f16x2(hi89);
          bf[3][1] = e4m3x2_to_f16x2(hi89 >> 16);
        } else {
          const uint2 w0 = *reinterpret_cast<const uint2*>(vcol + dec_chunk_off<false>(k0, vb >> 4));
          const uint2 w1 = *reinterpret_cast<const uint2*>(vcol + dec_chunk_off<false>(k0 + 1, vb >> 4));
          const uint2 w2 = *reinterpret_cast<const uint2*>(vcol + dec_chunk_off<false>(k0 + 8, vb >> 4));
          const uint2 w3 = *reinterpret_cast<const uint2*>(vcol + dec_chunk_off<false>(k0 + 9, vb >> 4));
          // bf16 column i of the two tokens of a pair side by side
          bf[0][0] = __byte_perm(w0.x, w1.x, 0x5410);
          bf[1][0] = __byte_perm(w0.x, w1.x, 0x7632);
          bf[2][0] = __byte_perm(w0.y, w1.y, 0x5410);
          bf[3][0] = __byte_perm(w0.y, w1.y, 0x7632);
          bf[0][1] = __byte_perm(w2.x, w3.x, 0x5410);
          bf[1][1] = __byte_perm(w2.x, w3.x, 0x7632);
          bf[2][1] = __byte_perm(w2.y, w3.y, 0x5410);
          bf[3][1] = __byte_perm(w2.y, w3.y, 0x7632);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) mma_16816<!FP8>(acc[i], af, bf[i][0], bf[i][1]);
      }
    }
    __syncthreads();  // this buffer is refilled next iteration; s_s and p16 are rewritten
  }

  // ---- the partial output of this range: lane (fr, fc) of warp w holds value columns
  // 32 w + 8 fc .. + 7 of heads fr and fr + 8
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int h = fr + 8 * hh;
    if (h < G) {
      float* po = p.part_o + (pidx + static_cast<size_t>(h) * p.n_splits) * DEC_D + 32 * warp + 8 * fc;
      *reinterpret_cast<float4*>(po) = make_float4(acc[0][2 * hh], acc[1][2 * hh], acc[2][2 * hh], acc[3][2 * hh]);
      *reinterpret_cast<float4*>(po + 4) =
          make_float4(acc[0][2 * hh + 1], acc[1][2 * hh + 1], acc[2][2 * hh + 1], acc[3][2 * hh + 1]);
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
