// Per-tensor e4m3 quantisation of bf16 activations, optionally after a 128-point
// Hadamard rotation along the head dimension ([ZYFA-mb] "Precisão, estabilidade e efeito
// na prática": most FP8 error comes from quantising Q, K and V; a Hadamard rotation of
// those tensors halves it).
//
// Two HBM-bound passes over x [rows, d] (rows = tokens * heads, d contiguous):
//   1. amax = max |y| with y = x or y = (x H_128) * float32(1/sqrt(128)), the rotation done
//      in float32 by the butterfly stages h = 1, 2, ..., 64, (u, w) -> (u + w, u - w).
//      Reduced with an integer atomicMax on the bit pattern (exact and order-free for
//      non-negative floats, so the result is deterministic).
//   2. scale = 448 / amax (float32, correctly rounded); code = e4m3 RNE-satfinite of
//      float32(y * scale); descale = amax / 448 written once.
// The rounding of every step is fixed, so the codes are a defined function of x.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace attn {

constexpr float HAD_R = 0.08838834764831845f;  // float32(1/sqrt(128))

// ---- rotated rows: one warp per 128-element row, 4 consecutive elements per lane
__device__ __forceinline__ void load_row4(const __nv_bfloat16* x, int64_t row, int lane,
                                          float v[4]) {
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + row * 128) + lane);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  v[0] = __low2float(a);
  v[1] = __high2float(a);
  v[2] = __low2float(b);
  v[3] = __high2float(b);
}

__device__ __forceinline__ void hadamard_row4(float v[4], int lane) {
  // stages h = 1, 2 inside the lane
  float u, w;
  u = v[0]; w = v[1]; v[0] = __fadd_rn(u, w); v[1] = __fsub_rn(u, w);
  u = v[2]; w = v[3]; v[2] = __fadd_rn(u, w); v[3] = __fsub_rn(u, w);
  u = v[0]; w = v[2]; v[0] = __fadd_rn(u, w); v[2] = __fsub_rn(u, w);
  u = v[1]; w = v[3]; v[1] = __fadd_rn(u, w); v[3] = __fsub_rn(u, w);
  // stages h = 4 .. 64 across lanes (partner lane = lane ^ (h / 4))
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? __fsub_rn(other, v[i]) : __fadd_rn(v[i], other);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __fmul_rn(v[i], HAD_R);
}

__device__ __forceinline__ void block_amax_atomic(float m, uint32_t* amax_bits) {
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < (blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) atomicMax(amax_bits, __float_as_uint(m));
  }
}

__device__ __forceinline__ float quant_scale(uint32_t amax_bits) {
  const float amax = __uint_as_float(amax_bits);
  return amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
}

// descale of an empty tensor (amax 0): 1, written on the device so the call stays
// stream-ordered and capturable (no host-to-device copy)
__global__ void descale_one_kernel(float* descale_out) { *descale_out = 1.0f; }

// ---- several tensors in one launch per pass (Q, K and V of one attention call): block b
// works on job j for block_end[j-1] <= b < block_end[j], grid-striding over that job's
// range only, so each block reads one tensor and its own amax word.  Same arithmetic and
// results as one launch per tensor.
constexpr int QUANT_MAX_JOBS = 3;
struct QuantJob {
  const __nv_bfloat16* x;
  uint8_t* y;
  int64_t n;          // 16-byte chunks (flat) or 128-element rows (rotated)
  uint32_t* amax;     // this tensor's amax word (cleared before the amax pass)
  float* descale;
};
struct QuantBatch {
  QuantJob job[QUANT_MAX_JOBS];
  int block_end[QUANT_MAX_JOBS];
  int njobs;
};

__device__ __forceinline__ int batch_job(const QuantBatch& b, int& first_block) {
  int j = 0;
  first_block = 0;
  while (j + 1 < b.njobs && static_cast<int>(blockIdx.x) >= b.block_end[j]) {
    first_block = b.block_end[j];
    ++j;
  }
  return j;
}

__device__ __forceinline__ float absmax8(const uint4 raw, float m) {
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    m = fmaxf(m, fmaxf(fabsf(__low2float(h2[k])), fabsf(__high2float(h2[k]))));
  return m;
}

// Four independent 16-byte loads (or rows) in flight per thread, then one per step for the
// remainder: the passes are HBM-bound and need the bytes in flight.
template <bool ROT>
__global__ void amax_batch_kernel(const QuantBatch b) {
  int first = 0;
  const int j = batch_job(b, first);
  const QuantJob& jb = b.job[j];
  const int nblk = b.block_end[j] - first;
  const int64_t tid = static_cast<int64_t>(blockIdx.x - first) * blockDim.x + threadIdx.x;
  float m = 0.0f;
  if constexpr (ROT) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (static_cast<int64_t>(nblk) * blockDim.x) >> 5;
    int64_t row = tid >> 5;
    for (; row + nwarps < jb.n; row += 2 * nwarps) {
      float v[4], w[4];
      load_row4(jb.x, row, lane, v);
      load_row4(jb.x, row + nwarps, lane, w);
      hadamard_row4(v, lane);
      hadamard_row4(w, lane);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
      m = fmaxf(m, fmaxf(fmaxf(fabsf(w[0]), fabsf(w[1])), fmaxf(fabsf(w[2]), fabsf(w[3]))));
    }
    for (; row < jb.n; row += nwarps) {
      float v[4];
      load_row4(jb.x, row, lane, v);
      hadamard_row4(v, lane);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
    }
  } else {
    const int64_t st = static_cast<int64_t>(nblk) * blockDim.x;
    const uint4* x = reinterpret_cast<const uint4*>(jb.x);
    int64_t i = tid;
    for (; i + 3 * st < jb.n; i += 4 * st) {
      const uint4 r0 = __ldg(x + i), r1 = __ldg(x + i + st), r2 = __ldg(x + i + 2 * st),
                  r3 = __ldg(x + i + 3 * st);
      m = absmax8(r3, absmax8(r2, absmax8(r1, absmax8(r0, m))));
    }
    for (; i < jb.n; i += st) m = absmax8(__ldg(x + i), m);
  }
  block_amax_atomic(m, jb.amax);
}

__device__ __forceinline__ uint2 e4m3x8(const uint4 raw, float sc) {
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    w[k] = f32_to_e4m3x2(__fmul_rn(__low2float(h2[k]), sc), __fmul_rn(__high2float(h2[k]), sc));
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

__device__ __forceinline__ void convert_row(const QuantJob& jb, int64_t row, int lane, float sc) {
  float v[4];
  load_row4(jb.x, row, lane, v);
  hadamard_row4(v, lane);
  const uint32_t lo = f32_to_e4m3x2(__fmul_rn(v[0], sc), __fmul_rn(v[1], sc));
  const uint32_t hi = f32_to_e4m3x2(__fmul_rn(v[2], sc), __fmul_rn(v[3], sc));
  reinterpret_cast<uint32_t*>(jb.y + row * 128)[lane] = lo | (hi << 16);
}

template <bool ROT>
__global__ void convert_batch_kernel(const QuantBatch b) {
  int first = 0;
  const int j = batch_job(b, first);
  const QuantJob& jb = b.job[j];
  const int nblk = b.block_end[j] - first;
  const uint32_t ab = *jb.amax;
  const float sc = quant_scale(ab);
  if (blockIdx.x == first && threadIdx.x == 0) {
    const float amax = __uint_as_float(ab);
    *jb.descale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  }
  const int64_t tid = static_cast<int64_t>(blockIdx.x - first) * blockDim.x + threadIdx.x;
  if constexpr (ROT) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (static_cast<int64_t>(nblk) * blockDim.x) >> 5;
    int64_t row = tid >> 5;
    for (; row + nwarps < jb.n; row += 2 * nwarps) {
      convert_row(jb, row, lane, sc);
      convert_row(jb, row + nwarps, lane, sc);
    }
    for (; row < jb.n; row += nwarps) convert_row(jb, row, lane, sc);
  } else {
    const int64_t st = static_cast<int64_t>(nblk) * blockDim.x;
    const uint4* x = reinterpret_cast<const uint4*>(jb.x);
    uint2* y = reinterpret_cast<uint2*>(jb.y);
    int64_t i = tid;
    for (; i + 3 * st < jb.n; i += 4 * st) {
      const uint4 r0 = __ldg(x + i), r1 = __ldg(x + i + st), r2 = __ldg(x + i + 2 * st),
                  r3 = __ldg(x + i + 3 * st);
      y[i] = e4m3x8(r0, sc);
      y[i + st] = e4m3x8(r1, sc);
      y[i + 2 * st] = e4m3x8(r2, sc);
      y[i + 3 * st] = e4m3x8(r3, sc);
    }
    for (; i < jb.n; i += st) y[i] = e4m3x8(__ldg(x + i), sc);
  }
}

}  // namespace attn
