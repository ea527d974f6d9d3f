// Issue-rate microbenchmark of tcgen05.mma on sm_100a: how many SM cycles one MMA
// instruction occupies, back to back from one issuing thread, for the instruction shapes
// the attention kernels use (S = Q K^T: A and B K-major from shared memory; P V: B MN-major,
// A from shared or tensor memory; block-scaled e4m3) with one CTA (M = 128) or a CTA pair
// (M = 256 over two SMs).  Every SM runs one CTA (or half a pair); operands are zeros (the
// rate does not depend on the values).  Prints one JSON line per shape.
//
// Also: the round trip of a dependent MMA group (issue, commit, wait for the commit).
//
// Build and run: python -m bf16_causal_prefill_attn_b200.microbench.umma_rate
#include <cuda_runtime.h>

#include <cstdio>
#include <vector>

#include "../csrc/ptx.cuh"

using namespace attn;

namespace {

constexpr int SMEM_A = 0;           // 16 KB: 128 rows x 128 B, K-major, 128-B swizzle
constexpr int SMEM_B = 32768;       // 64 KB
constexpr int SMEM_BAR = 32768 + 65536;
// more than half of an SM's shared memory: never two CTAs (nor both CTAs of a pair) on one
// SM, so every 512-column TMEM allocation succeeds at once
constexpr int SMEM_BYTES = 160 * 1024;

__device__ __forceinline__ uint64_t desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return smem_desc_sw128(saddr, lbo, sbo);
}

// CG: CTAs per MMA (1 or 2); KIND: 0 bf16 (kind::f16), 1 e4m3 (kind::f8f6f4),
// 2 block-scaled e4m3 (kind::mxf8f6f4.block_scale); ATM: A from tensor memory (bf16 only);
// BL: B layout -- 0 K-major, 128-B swizzle (the K operand of Q K^T); 1 MN-major, 128-B
// swizzle, atoms 16 KB apart (the V operand of the single-CTA P V); 2 MN-major, 64-B swizzle,
// a 64-column atom then a second atom 8 KB away (the pair kernel's V half + ones block).
// A pair MMA with an MN-major B takes N in multiples of 32.
template <int CG, int KIND, bool ATM, int N, int BL>
__global__ void __launch_bounds__(128, 1) rate_kernel(long long* cycles, int ni) {
  extern __shared__ uint8_t raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SMEM_BAR);
  uint32_t* tptr = reinterpret_cast<uint32_t*>(smem + SMEM_BAR + 16);
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < SMEM_BAR / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    if constexpr (CG == 2) {
      tmem_alloc2(tptr, 512);
      tmem_relinquish2();
    } else {
      tmem_alloc(tptr, 512);
      tmem_relinquish();
    }
  }
  __syncthreads();
  if constexpr (CG == 2) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tptr;
  const bool leader = CG == 1 || cluster_ctarank() == 0;
  constexpr int M = 128 * CG;
  constexpr uint32_t D1 = N <= 128 ? 128 : 256;
  static_assert(!ATM || N <= 128, "A in TMEM at column 384");
  static_assert(KIND != 2 || N <= 192, "scale factors at columns 448..463");
  static_assert(CG == 1 || BL == 0 || N % 32 == 0, "pair MMA, MN-major B: N % 32");
  constexpr uint32_t BMN = BL != 0 ? 1u : 0u;
  constexpr uint32_t IDESC = KIND == 2 ? idesc_mxf8(0, BMN, M, N, 0, 0)
                                       : idesc_dense(KIND == 0 ? 1 : 0, KIND == 0 ? 1 : 0, 0,
                                                     BMN, M, N);
  const uint64_t ad = desc(smem_addr(smem + SMEM_A), 16, 1024);
  const uint64_t bd = BL == 1   ? desc(smem_addr(smem + SMEM_B), 16384, 1024)
                      : BL == 2 ? smem_desc_sw64(smem_addr(smem + SMEM_B), 8192, 512)
                                : desc(smem_addr(smem + SMEM_B), 16, 1024);
  long long t = 0;
  bool ok = true;
  if (warp == 0) {
    if (leader) {
      long long t0 = 0;
      if (threadIdx.x == 0) {
        t0 = clock64();
        for (int i = 0; i < ni; ++i) {
          const uint32_t d = tmem + ((i & 1) ? D1 : 0u);
          if constexpr (CG == 1) {
            if constexpr (KIND == 2)
              mma_ss_mxf8(d, ad, bd, IDESC, tmem + 448, tmem + 456, 1u);
            else if constexpr (ATM)
              mma_ts_f16(d, tmem + 384, bd, IDESC, 1u);
            else
              mma_ss<KIND>(d, ad, bd, IDESC, 1u);
          } else {
            if constexpr (KIND == 2)
              mma2_ss_mxf8(d, ad, bd, IDESC, tmem + 448, tmem + 456, 1u);
            else if constexpr (ATM)
              mma2_ts_f16(d, tmem + 384, bd, IDESC, 1u);
            else
              mma2_ss<KIND>(d, ad, bd, IDESC, 1u);
          }
        }
        if constexpr (CG == 1)
          tc_commit(bar);
        else
          tc_commit2(bar, 3);
      }
      __syncwarp();
      // bounded wait (a second at most) for the MMAs to finish
      uint64_t g0 = globaltimer_ns();
      while (!mbar_try_wait(bar, 0)) {
        if (globaltimer_ns() - g0 > 1000000000ull) {
          ok = false;
          break;
        }
      }
      if (threadIdx.x == 0) t = clock64() - t0;
    } else {
      uint64_t g0 = globaltimer_ns();
      while (!mbar_try_wait(bar, 0)) {
        if (globaltimer_ns() - g0 > 1000000000ull) {
          ok = false;
          break;
        }
      }
    }
  }
  __syncthreads();
  if constexpr (CG == 2) cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    if constexpr (CG == 2)
      tmem_dealloc2(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) cycles[blockIdx.x] = ok ? t : -1;
}

// Round trip of a dependent group: one thread issues G MMAs (K-major A and B from shared
// memory) and a commit, waits for the commit's arrival, and repeats -- the latency an S MMA
// group pays between its issue and the softmax seeing it.  Every wait is bounded (a second
// in all); after a timeout the thread stops issuing and the MMAs in flight drain (again
// bounded) before TMEM is released.
template <int KIND, int N, int G>
__global__ void __launch_bounds__(128, 1) lat_kernel(long long* cycles, int ni) {
  extern __shared__ uint8_t raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SMEM_BAR);
  uint32_t* tptr = reinterpret_cast<uint32_t*>(smem + SMEM_BAR + 16);
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < SMEM_BAR / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tptr, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tptr;
  constexpr uint32_t IDESC = idesc_dense(KIND == 0 ? 1 : 0, KIND == 0 ? 1 : 0, 0, 0, 128, N);
  const uint64_t ad = desc(smem_addr(smem + SMEM_A), 16, 1024);
  const uint64_t bd = desc(smem_addr(smem + SMEM_B), 16, 1024);
  long long t = 0;
  bool ok = true;
  if (threadIdx.x == 0) {
    const uint64_t g0 = globaltimer_ns();
    const long long t0 = clock64();
    for (int i = 0; i < ni && ok; ++i) {
      for (int g = 0; g < G; ++g) mma_ss<KIND>(tmem, ad, bd, IDESC, g > 0 ? 1u : 0u);
      tc_commit(bar);
      while (!mbar_try_wait(bar, static_cast<uint32_t>(i & 1))) {
        if (globaltimer_ns() - g0 > 1000000000ull) {
          ok = false;
          break;
        }
      }
    }
    t = clock64() - t0;
    tc_commit(bar + 1);
    const uint64_t g1 = globaltimer_ns();
    while (!mbar_try_wait(bar + 1, 0))
      if (globaltimer_ns() - g1 > 1000000000ull) break;
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) cycles[blockIdx.x] = ok ? t : -1;
}

template <int KIND, int N, int G>
void run_lat(const char* name, int sms, int ni) {
  auto k = lat_kernel<KIND, N, G>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES + 1024);
  long long* d = nullptr;
  cudaMalloc(&d, sms * sizeof(long long));
  for (int rep = 0; rep < 3; ++rep) k<<<sms, 128, SMEM_BYTES + 1024>>>(d, ni);
  cudaDeviceSynchronize();
  cudaError_t err = cudaGetLastError();
  std::vector<long long> h(sms);
  cudaMemcpy(h.data(), d, sms * sizeof(long long), cudaMemcpyDeviceToHost);
  cudaFree(d);
  double sum = 0;
  int n = 0, bad = 0;
  for (long long v : h) {
    if (v > 0) {
      sum += double(v);
      ++n;
    } else if (v < 0) {
      ++bad;
    }
  }
  const double cyc = n ? sum / n / ni : 0.0;
  std::printf(
      "{\"latency\": \"%s\", \"N\": %d, \"mmas_per_group\": %d, \"cycles_per_round_trip\": %.1f, "
      "\"timeouts\": %d, \"error\": \"%s\"}\n",
      name, N, G, cyc, bad, cudaGetErrorString(err));
  std::fflush(stdout);
}

template <int CG, int KIND, bool ATM, int N, int BL>
void run(const char* name, int sms, int ni) {
  auto k = rate_kernel<CG, KIND, ATM, N, BL>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES + 1024);
  const int grid = sms / CG * CG;
  long long* d = nullptr;
  cudaMalloc(&d, grid * sizeof(long long));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = SMEM_BYTES + 1024;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  float ms = 0.0f;
  for (int rep = 0; rep < 3; ++rep) {
    cudaEventRecord(e0);
    cudaLaunchKernelEx(&cfg, k, d, ni);
    cudaEventRecord(e1);
    cudaEventSynchronize(e1);
    cudaEventElapsedTime(&ms, e0, e1);
  }
  cudaError_t err = cudaGetLastError();
  std::vector<long long> h(grid);
  cudaMemcpy(h.data(), d, grid * sizeof(long long), cudaMemcpyDeviceToHost);
  cudaFree(d);
  double sum = 0;
  int n = 0, bad = 0;
  for (long long v : h) {
    if (v > 0) {
      sum += double(v);
      ++n;
    } else if (v < 0) {
      ++bad;
    }
  }
  const double cyc = n ? sum / n / ni : 0.0;
  const int K = KIND == 0 ? 16 : 32;
  const double flop_per_sm = 2.0 * 128 * N * K;  // per instruction, per SM
  const double peak = KIND == 0 ? 8192.0 : 16384.0;  // dense flop per SM per cycle
  std::printf(
      "{\"shape\": \"%s\", \"cta_group\": %d, \"M\": %d, \"N\": %d, \"K\": %d, \"cycles_per_mma\": "
      "%.1f, \"flop_per_sm_cycle\": %.0f, \"frac_of_dense_rate\": %.3f, \"kernel_ms\": %.4f, "
      "\"timeouts\": %d, \"error\": \"%s\"}\n",
      name, CG, 128 * CG, N, K, cyc, cyc > 0 ? flop_per_sm / cyc : 0.0,
      cyc > 0 ? flop_per_sm / cyc / peak : 0.0, ms, bad, cudaGetErrorString(err));
  std::fflush(stdout);
}

}  // namespace

int main() {
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  const int ni = 4096;
  // S = Q K^T shapes (A, B K-major in shared memory)
  // below N = 128: where the instruction stops being bound by its own work
  run<1, 0, false, 16, 0>("bf16 QK^T", sms, ni);
  run<1, 0, false, 32, 0>("bf16 QK^T", sms, ni);
  run<1, 0, false, 64, 0>("bf16 QK^T", sms, ni);
  run<1, 0, false, 128, 0>("bf16 QK^T", sms, ni);
  run<1, 0, false, 256, 0>("bf16 QK^T", sms, ni);
  run<2, 0, false, 128, 0>("bf16 QK^T", sms, ni);
  run<2, 0, false, 256, 0>("bf16 QK^T", sms, ni);
  run<1, 1, false, 16, 0>("e4m3 QK^T", sms, ni);
  run<1, 1, false, 32, 0>("e4m3 QK^T", sms, ni);
  run<1, 1, false, 64, 0>("e4m3 QK^T", sms, ni);
  run<1, 1, false, 128, 0>("e4m3 QK^T", sms, ni);
  run<1, 1, false, 256, 0>("e4m3 QK^T", sms, ni);
  run<2, 1, false, 128, 0>("e4m3 QK^T", sms, ni);
  run<2, 1, false, 256, 0>("e4m3 QK^T", sms, ni);
  // P V shapes (B MN-major)
  run<1, 0, true, 128, 1>("bf16 PV, P in TMEM", sms, ni);
  run<2, 0, true, 128, 1>("bf16 PV, P in TMEM", sms, ni);
  run<1, 0, false, 128, 1>("bf16 PV, P in smem", sms, ni);
  run<2, 0, false, 128, 1>("bf16 PV, P in smem", sms, ni);
  run<1, 1, false, 128, 1>("e4m3 PV (no scales)", sms, ni);
  run<2, 1, false, 128, 1>("e4m3 PV (no scales)", sms, ni);
  run<1, 2, false, 128, 1>("e4m3 block-scaled PV", sms, ni);
  run<1, 2, false, 144, 1>("e4m3 block-scaled PV + row sum (single-CTA kernel)", sms, ni);
  run<2, 2, false, 128, 1>("e4m3 block-scaled PV", sms, ni);
  run<2, 2, false, 160, 2>("e4m3 block-scaled PV + row sum (pair kernel, 64-B swizzle)", sms, ni);
  // dependent round trips: the S group of each kernel (d = 128) and its key halves
  run_lat<0, 128, 8>("bf16 S group", sms, 1024);
  run_lat<0, 64, 8>("bf16 S key half", sms, 1024);
  run_lat<1, 128, 4>("e4m3 S group", sms, 1024);
  run_lat<1, 64, 4>("e4m3 S key half", sms, 1024);
  run_lat<0, 128, 1>("bf16 one MMA", sms, 1024);
  return 0;
}
