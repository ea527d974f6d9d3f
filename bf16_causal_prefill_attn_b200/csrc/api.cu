// C ABI of libattn_b200.so (declared in include/attn.h): argument validation, TMA tensor
// maps, kernel selection and launch.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "attn_fwd.cuh"
#include "decode.cuh"
#include "quantize.cuh"

namespace {

constexpr int kVersion = 1;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait

// Device error word of every GPU that loads the library (set by bounded waits).
__device__ uint32_t g_dev_err = 0;

uint64_t g_timeout_ns = kDefaultTimeoutNs;
int g_stall_tile = -1;  // test-only (attn_selftest_stall_tile)
int g_kernel = ATTN_KERNEL_AUTO;  // prefill unit and schedule (attn_select_prefill_kernel)
int g_max_ctas = 0;  // test-only cap on the persistent grid (attn_selftest_max_ctas; 0: none)

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

unsigned long long current_context_id();

// Device address of the error word in the current context, looked up once per context by
// this host thread (the last few contexts are kept, by their unique ids).
bool dev_err_ptr(uint32_t** out) {
  constexpr int kSlots = 4;
  thread_local unsigned long long ctxs[kSlots] = {};
  thread_local uint32_t* ptrs[kSlots] = {};
  thread_local int next = 0;
  const unsigned long long c = current_context_id();
  if (c != 0)
    for (int i = 0; i < kSlots; ++i)
      if (ctxs[i] == c) {
        *out = ptrs[i];
        return true;
      }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess) return false;
  *out = static_cast<uint32_t*>(p);
  if (c != 0) {
    ctxs[next] = c;
    ptrs[next] = *out;
    next = (next + 1) % kSlots;
  }
  return true;
}

// 3-D tiled map over [T, H, d] (d innermost), box = (box_cols, 1, box_rows).  An encoded map
// is a pure function of these arguments, so the last few are kept per host thread and
// reused when the same tensor is passed again (no lock: the cache is thread-local).
struct MapKey {
  const void* base;
  uint64_t d, H, T;
  uint32_t box_cols, box_rows;
  int dt, esize, swz;
  bool operator==(const MapKey& o) const {
    return base == o.base && d == o.d && H == o.H && T == o.T && box_cols == o.box_cols &&
           box_rows == o.box_rows && dt == o.dt && esize == o.esize && swz == o.swz;
  }
};

bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t d,
              uint64_t H, uint64_t T, uint32_t box_cols, uint32_t box_rows = 128,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  constexpr int kSlots = 8;
  thread_local MapKey keys[kSlots] = {};
  thread_local CUtensorMap maps[kSlots];
  thread_local int next = 0;
  const MapKey key{base, d, H, T, box_cols, box_rows, static_cast<int>(dt), esize,
                   static_cast<int>(swz)};
  for (int i = 0; i < kSlots; ++i) {
    if (keys[i] == key && keys[i].base != nullptr) {
      *m = maps[i];
      return true;
    }
  }
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d, H, T};
  cuuint64_t strides[2] = {d * esize, H * d * esize};
  cuuint32_t box[3] = {box_cols, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  keys[next] = key;
  maps[next] = *m;
  next = (next + 1) % kSlots;
  return true;
}

// The unique id of the current context (driver API through the runtime's entry-point
// query), to key state that belongs to a context.  Ids are never reused, unlike context
// handles: after cudaDeviceReset the new primary context may have the old handle.  0: no
// context, or the driver offers no id (callers then cache nothing).
using PFN_ctxGetCurrent = CUresult (*)(CUcontext*);
using PFN_ctxGetId = CUresult (*)(CUcontext, unsigned long long*);
unsigned long long current_context_id() {
  static PFN_ctxGetCurrent get_current = nullptr;
  static PFN_ctxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_ctxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_ctxGetId>(p);
  });
  CUcontext c = nullptr;
  if (get_current == nullptr || get_id == nullptr || get_current(&c) != CUDA_SUCCESS ||
      c == nullptr)
    return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// cudaFuncSetAttribute(max dynamic shared memory) for kernel KERN, skipped when it was
// already done for the current context by this host thread.  The cache is per kernel (a
// template on the kernel's address: the prefill kernels all share one function type).
template <auto KERN>
bool set_smem_attr(int bytes) {
  thread_local unsigned long long done_ctx[4] = {};
  thread_local int next = 0;
  const unsigned long long c = current_context_id();
  if (c != 0)
    for (unsigned long long d : done_ctx)
      if (d == c) return true;
  if (cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  if (c != 0) {
    done_ctx[next] = c;
    next = (next + 1) % 4;
  }
  return true;
}

// The prefill kernels move registers from their producer/MMA warps to their softmax warps
// (setmaxnreg); the increase only succeeds if the block was launched with at least
// REGS_NEEDED_AT_LAUNCH registers per thread, so never launch one with fewer.  The count
// is a property of the compiled kernel: checked once per kernel (a template on its
// address), then remembered.
template <auto KERN>
attn_status_t register_split_ok() {
  static std::atomic<int> known{0};  // 0 not yet checked, 1 ok, 2 too few registers
  const int k = known.load(std::memory_order_relaxed);
  if (k != 0) return k == 1 ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, KERN) != cudaSuccess) return ATTN_ERR_CUDA;  // not cached
  const bool ok = fa.numRegs >= attn::REGS_NEEDED_AT_LAUNCH &&
                  fa.numRegs * attn::NUM_THREADS <= 65536;
  known.store(ok ? 1 : 2, std::memory_order_relaxed);
  return ok ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

// Multiprocessors of the current device (cached per device; devices are few).
int sm_count() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < kMaxDev) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < kMaxDev) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <bool FP8, int DQK, bool DUMP, bool EXACT, bool VARLEN, bool BSA>
attn_status_t launch_fwd(const void* q, const void* k, const void* v, attn::FwdParams& prm,
                         cudaStream_t stream) {
  using C = attn::FwdCfg<FP8, DQK>;
  const CUtensorMapDataType dt =
      FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t T = static_cast<uint64_t>(prm.total_tokens);
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, dt, C::E, DQK, prm.Hq, T, C::BOX_COLS) ||
      !make_map(&mk, k, dt, C::E, DQK, prm.Hkv, T, C::BOX_COLS) ||
      !make_map(&mv, v, dt, C::E, attn::DV, prm.Hkv, T, C::BOX_COLS))
    return ATTN_ERR_CUDA;
  // O [T, Hq, 128] bf16 in boxes of 64 columns x 128 rows (FP8) or 32 rows (BF16: one box
  // per softmax warp), stored through shared memory
  if (C::TMA_O && !VARLEN) {
    if (!make_map(&mo, prm.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, attn::DV, prm.Hq, T, 64, C::O_BOX_ROWS))
      return ATTN_ERR_CUDA;
  } else {
    mo = mq;  // unused
  }
  constexpr auto kern = attn::attn_fwd_kernel<FP8, DQK, DUMP, EXACT, VARLEN, BSA>;
  if (!set_smem_attr<kern>(C::SMEM_ALLOC)) return ATTN_ERR_CUDA;
  const attn_status_t rs = register_split_ok<kern>();
  if (rs != ATTN_OK) return rs;
  // units: two query tiles of one head, or (ATTN_KERNEL_HEADS, Hq / Hkv even) one query
  // tile of two heads of one kv group; one CTA per unit (ATTN_KERNEL_DYNAMIC: running CTAs
  // take over the units of CTAs not yet started), or (ATTN_KERNEL_PERSISTENT) one CTA per
  // SM running a static list of units
  attn::FwdParams pp = prm;
  const int kernel =
      g_kernel == ATTN_KERNEL_AUTO ? (ATTN_KERNEL_DYNAMIC | (FP8 ? ATTN_KERNEL_HEADS : 0)) : g_kernel;
  pp.head_pairs = ((kernel & ATTN_KERNEL_HEADS) && prm.G % 2 == 0) ? 1 : 0;
  pp.n_pairs = pp.head_pairs ? prm.n_q_tiles : (prm.n_q_tiles + 1) / 2;
  const int64_t units = static_cast<int64_t>(pp.n_pairs) * prm.B *
                        (pp.head_pairs ? prm.Hq / 2 : prm.Hq);
  if (units <= 0 || units > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  pp.n_units = static_cast<int>(units);
  unsigned grid = static_cast<unsigned>(units);
  pp.dynamic = (kernel & ATTN_KERNEL_DYNAMIC) ? 1 : 0;
  if (kernel & ATTN_KERNEL_PERSISTENT) {
    const int sms = sm_count();
    if (sms <= 0) return ATTN_ERR_CUDA;
    grid = static_cast<unsigned>(std::min<int64_t>(units, sms));
    if (g_max_ctas > 0) grid = std::min(grid, static_cast<unsigned>(g_max_ctas));
  }
  kern<<<grid, attn::NUM_THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv, mo, pp);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// BF16 pipeline: the S-ahead one when selected, or by default with grouped-query heads
// (Hq > Hkv: its earlier K loads are mostly L2 hits there; with as many kv heads as query
// heads every CTA streams its own K and V, and the P-over-S pipeline measured faster)
bool bf16_s_ahead(const attn::FwdParams& prm) {
  if (g_kernel != ATTN_KERNEL_AUTO && (g_kernel & ATTN_KERNEL_BF16_S_AHEAD)) return true;
  if (g_kernel != ATTN_KERNEL_AUTO && (g_kernel & ATTN_KERNEL_BF16_P_OVER_S)) return false;
  return prm.Hq > prm.Hkv;
}

// The prefill kernel for one instantiation.
template <bool FP8, int DQK, bool DUMP, bool EXACT = false, bool VARLEN = false>
attn_status_t launch_prefill(const void* q, const void* k, const void* v, attn::FwdParams& prm,
                             cudaStream_t stream) {
  if constexpr (!FP8) {
    if (bf16_s_ahead(prm)) return launch_fwd<FP8, DQK, DUMP, EXACT, VARLEN, true>(q, k, v, prm, stream);
  }
  return launch_fwd<FP8, DQK, DUMP, EXACT, VARLEN, false>(q, k, v, prm, stream);
}

// Checks shared by the fixed-length and packed entry points; fills the parameters that
// do not depend on the sequence layout.
attn_status_t common_args(void* o, float* lse, int Hq, int Hkv, int d_qk, int d_v,
                          attn_dtype_t dtype, const float* dq, const float* dk,
                          const float* dv, int causal, unsigned flags, attn::FwdParams* prm) {
  if (Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if ((flags & ~static_cast<unsigned>(ATTN_FLAG_UNROTATE_O | ATTN_FLAG_EXACT_P)) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP8_E4M3) return ATTN_ERR_INVALID_ARG;
  if ((flags & ATTN_FLAG_EXACT_P) && dtype != ATTN_FP8_E4M3) return ATTN_ERR_INVALID_ARG;
  if ((d_qk != 128 && d_qk != 192) || d_v != 128) return ATTN_ERR_UNSUPPORTED;
  prm->Hq = Hq;
  prm->Hkv = Hkv;
  prm->G = Hq / Hkv;
  prm->causal = causal;
  prm->o = static_cast<__nv_bfloat16*>(o);
  prm->lse = lse;
  const double scale = 1.0 / std::sqrt(static_cast<double>(d_qk));
  const double log2e = 1.4426950408889634;
  prm->c1 = static_cast<float>(scale * log2e);
  prm->leanp_c = 8.0 * log2e * scale;
  prm->descale_q = dq;
  prm->descale_k = dk;
  prm->descale_v = dv;
  prm->unrotate = (flags & ATTN_FLAG_UNROTATE_O) ? 1 : 0;
  prm->timeout_ns = g_timeout_ns;
  prm->stall_tile = g_stall_tile;
  return ATTN_OK;
}

attn_status_t pointer_args(const void* q, const void* k, const void* v, void* o, float* lse,
                           attn_dtype_t dtype, const float* dq, const float* dk,
                           const float* dv) {
  if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
  if (dtype == ATTN_FP8_E4M3 && (!dq || !dk || !dv)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_ALIGNMENT;
  return ATTN_OK;
}

attn_status_t dispatch(const void* q, const void* k, const void* v, int d_qk, attn_dtype_t dtype,
                       unsigned flags, bool dump, bool varlen, attn::FwdParams& prm,
                       cudaStream_t st) {
  const bool exact = (flags & ATTN_FLAG_EXACT_P) != 0;
  if (varlen) {
    // sequences of any length: lean-P FP8 and BF16 (not the exact-P ablation, not the
    // test-only dump)
    if (exact || dump) return ATTN_ERR_UNSUPPORTED;
    if (dtype == ATTN_BF16) {
      if (d_qk == 128) return launch_prefill<false, 128, false, false, true>(q, k, v, prm, st);
      return launch_prefill<false, 192, false, false, true>(q, k, v, prm, st);
    }
    if (d_qk == 128) return launch_prefill<true, 128, false, false, true>(q, k, v, prm, st);
    return launch_prefill<true, 192, false, false, true>(q, k, v, prm, st);
  }
  if (dtype == ATTN_BF16) {
    if (d_qk == 128) return launch_prefill<false, 128, false>(q, k, v, prm, st);
    return launch_prefill<false, 192, false>(q, k, v, prm, st);
  }
  if (dump) {
    if (exact) {
      if (d_qk == 128) return launch_prefill<true, 128, true, true>(q, k, v, prm, st);
      return launch_prefill<true, 192, true, true>(q, k, v, prm, st);
    }
    if (d_qk == 128) return launch_prefill<true, 128, true>(q, k, v, prm, st);
    return launch_prefill<true, 192, true>(q, k, v, prm, st);
  }
  if (exact) {
    if (d_qk == 128) return launch_prefill<true, 128, false, true>(q, k, v, prm, st);
    return launch_prefill<true, 192, false, true>(q, k, v, prm, st);
  }
  if (d_qk == 128) return launch_prefill<true, 128, false>(q, k, v, prm, st);
  return launch_prefill<true, 192, false>(q, k, v, prm, st);
}

attn_status_t fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int S, int d_qk, int d_v, attn_dtype_t dtype,
                       const float* dq, const float* dk, const float* dv, int causal,
                       unsigned flags, float* dump_s, uint8_t* dump_codes,
                       uint8_t* dump_kshift, bool dump, void* stream) {
  attn::FwdParams prm{};
  if (B < 0 || S < 0) return ATTN_ERR_INVALID_ARG;
  attn_status_t e = common_args(o, lse, Hq, Hkv, d_qk, d_v, dtype, dq, dk, dv, causal, flags,
                                &prm);
  if (e != ATTN_OK) return e;
  if (B == 0 || S == 0) return ATTN_OK;
  if (dump && (dtype != ATTN_FP8_E4M3 || !dump_s || !dump_codes || !dump_kshift))
    return ATTN_ERR_INVALID_ARG;
  // the tail-masking variant covers lean-P FP8 and BF16 only
  if ((S % 128) != 0 && (dump || (flags & ATTN_FLAG_EXACT_P))) return ATTN_ERR_UNSUPPORTED;
  const int n_q_tiles = (S + 127) / 128;
  if (static_cast<int64_t>(B) * S > INT32_MAX ||
      static_cast<int64_t>(n_q_tiles) * B * Hq > INT32_MAX)
    return ATTN_ERR_UNSUPPORTED;
  e = pointer_args(q, k, v, o, lse, dtype, dq, dk, dv);
  if (e != ATTN_OK) return e;
  prm.B = B;
  prm.S = S;
  prm.n_q_tiles = n_q_tiles;
  prm.n_pairs = (n_q_tiles + 1) / 2;
  prm.cu_seqlens = nullptr;
  prm.max_seqlen = S;
  prm.total_tokens = static_cast<int64_t>(B) * S;
  prm.dump_s = dump_s;
  prm.dump_codes = dump_codes;
  prm.dump_kshift = dump_kshift;
  if (!dev_err_ptr(&prm.err)) return ATTN_ERR_CUDA;
  // S not a multiple of 128: the kernel variant that masks the tail of each sequence
  return dispatch(q, k, v, d_qk, dtype, flags, dump, (S % 128) != 0, prm,
                  static_cast<cudaStream_t>(stream));
}

attn_status_t varlen_impl(const void* q, const void* k, const void* v, void* o, float* lse,
                          const int32_t* cu_seqlens, int B, int max_seqlen,
                          int64_t total_tokens, int Hq, int Hkv, int d_qk, int d_v,
                          attn_dtype_t dtype, const float* dq, const float* dk,
                          const float* dv, int causal, unsigned flags, void* stream) {
  attn::FwdParams prm{};
  if (B < 0 || max_seqlen < 0 || total_tokens < 0) return ATTN_ERR_INVALID_ARG;
  attn_status_t e = common_args(o, lse, Hq, Hkv, d_qk, d_v, dtype, dq, dk, dv, causal, flags,
                                &prm);
  if (e != ATTN_OK) return e;
  if (B == 0 || max_seqlen == 0 || total_tokens == 0) return ATTN_OK;
  if (flags & ATTN_FLAG_EXACT_P) return ATTN_ERR_UNSUPPORTED;
  if (!cu_seqlens) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) return ATTN_ERR_ALIGNMENT;
  const int n_q_tiles = (max_seqlen + 127) / 128;
  if (total_tokens > INT32_MAX || max_seqlen > total_tokens ||
      static_cast<int64_t>(n_q_tiles) * B * Hq > INT32_MAX)
    return ATTN_ERR_UNSUPPORTED;
  e = pointer_args(q, k, v, o, lse, dtype, dq, dk, dv);
  if (e != ATTN_OK) return e;
  prm.B = B;
  prm.S = 0;  // unused with cu_seqlens
  prm.n_q_tiles = n_q_tiles;
  prm.n_pairs = (n_q_tiles + 1) / 2;
  prm.cu_seqlens = cu_seqlens;
  prm.max_seqlen = max_seqlen;
  prm.total_tokens = total_tokens;
  if (!dev_err_ptr(&prm.err)) return ATTN_ERR_CUDA;
  return dispatch(q, k, v, d_qk, dtype, flags, false, true, prm, static_cast<cudaStream_t>(stream));
}

template <bool FP8, int G>
attn_status_t launch_decode(attn::DecodeParams& prm, cudaStream_t st) {
  constexpr auto k1 = attn::decode_split_kernel<FP8, G>;
  constexpr int smem = attn::dec_smem_bytes<FP8, G>();
  if (!set_smem_attr<k1>(smem)) return ATTN_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>(prm.Hkv), static_cast<unsigned>(prm.n_splits),
                  static_cast<unsigned>(prm.B));
  k1<<<grid, attn::DEC_THREADS, smem, st>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  attn::decode_combine_kernel<FP8><<<static_cast<unsigned>(prm.B) * prm.Hq, attn::DEC_D, 0, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <bool FP8>
attn_status_t dispatch_decode(attn::DecodeParams& prm, cudaStream_t st) {
  switch (prm.G) {
    case 1: return launch_decode<FP8, 1>(prm, st);
    case 2: return launch_decode<FP8, 2>(prm, st);
    case 4: return launch_decode<FP8, 4>(prm, st);
    case 8: return launch_decode<FP8, 8>(prm, st);
    case 16: return launch_decode<FP8, 16>(prm, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

// A wait that nothing ever satisfies: one thread waits (bounded) on an mbarrier no one
// arrives at, records DEV_TIMEOUT and returns.
__global__ void selftest_wait_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  attn::mbar_init(&bar, 1);
  attn::fence_barrier_init();
  attn::mbar_wait(&bar, 0, err, timeout_ns);
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// One amax launch and one conversion launch over n tensors (n <= 3): x[i] bf16 [el[i]
// elements] -> y[i] e4m3 codes, ds[i] its descale, amax[i] a cleared word.  Blocks are split
// among the tensors in proportion to their sizes; the conversion visits the tensors in the
// reverse order, so those the amax pass read last are re-read first, while they may still
// be in L2.
attn_status_t launch_quantize(int n, const void* const* x, void* const* y, float* const* ds,
                              const int64_t* el, int hadamard, uint32_t* amax,
                              cudaStream_t st) {
  const int threads = 256;
  const int64_t per_block_items = hadamard ? threads / 32 : threads * 4;  // rows or chunks
  const int64_t budget = int64_t(num_sms()) * 16;  // blocks per pass, split by size
  int64_t total = 0;
  for (int i = 0; i < n; ++i) total += el[i];
  attn::QuantBatch fwd{}, rev{};
  fwd.njobs = rev.njobs = n;
  int end_f = 0, end_r = 0;
  for (int o = 0; o < n; ++o) {
    for (int pass = 0; pass < 2; ++pass) {
      const int i = pass == 0 ? o : n - 1 - o;
      const int64_t items = hadamard ? el[i] / 128 : el[i] / 8;
      const int64_t want = (items + per_block_items - 1) / per_block_items;
      const int64_t share = std::max<int64_t>(1, (budget * el[i] + total - 1) / total);
      const int nb = static_cast<int>(std::max<int64_t>(1, std::min(want, share)));
      attn::QuantJob jb{static_cast<const __nv_bfloat16*>(x[i]), static_cast<uint8_t*>(y[i]),
                        items, amax + i, ds[i]};
      if (pass == 0) {
        fwd.job[o] = jb;
        end_f += nb;
        fwd.block_end[o] = end_f;
      } else {
        rev.job[o] = jb;
        end_r += nb;
        rev.block_end[o] = end_r;
      }
    }
  }
  if (cudaMemsetAsync(amax, 0, n * sizeof(uint32_t), st) != cudaSuccess) return ATTN_ERR_CUDA;
  if (hadamard) {
    attn::amax_batch_kernel<true><<<end_f, threads, 0, st>>>(fwd);
    attn::convert_batch_kernel<true><<<end_r, threads, 0, st>>>(rev);
  } else {
    attn::amax_batch_kernel<false><<<end_f, threads, 0, st>>>(fwd);
    attn::convert_batch_kernel<false><<<end_r, threads, 0, st>>>(rev);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int S, int d_qk, int d_v, attn_dtype_t dtype,
                       const float* descale_q, const float* descale_k, const float* descale_v,
                       int causal, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, S, d_qk, d_v, dtype, descale_q, descale_k,
                  descale_v, causal, 0u, nullptr, nullptr, nullptr, false, stream);
}

attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int S, int d_qk, int d_v, attn_dtype_t dtype,
                          const float* descale_q, const float* descale_k,
                          const float* descale_v, int causal, unsigned flags, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, S, d_qk, d_v, dtype, descale_q, descale_k,
                  descale_v, causal, flags, nullptr, nullptr, nullptr, false, stream);
}

attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                              const int32_t* cu_seqlens, int B, int max_seqlen,
                              int64_t total_tokens, int Hq, int Hkv, int d_qk, int d_v,
                              attn_dtype_t dtype, const float* descale_q, const float* descale_k,
                              const float* descale_v, int causal, unsigned flags, void* stream) {
  return varlen_impl(q, k, v, o, lse, cu_seqlens, B, max_seqlen, total_tokens, Hq, Hkv, d_qk,
                     d_v, dtype, descale_q, descale_k, descale_v, causal, flags, stream);
}

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int max_seqlen) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || max_seqlen <= 0) return 0;
  const int ns = attn::dec_n_splits(B, Hkv, max_seqlen);
  return static_cast<size_t>(B) * Hq * ns * (attn::DEC_D + 2) * sizeof(float);
}

attn_status_t attn_decode_paged(const void* q, const void* k_cache, const void* v_cache, void* o,
                                float* lse, const int32_t* block_table, const int32_t* seq_lens,
                                int B, int Hq, int Hkv, int d_qk, int d_v, int num_pages,
                                int page_size, int max_blocks_per_seq, int max_seqlen,
                                attn_dtype_t dtype, const float* descale_q,
                                const float* descale_k, const float* descale_v, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || max_seqlen < 0 || num_pages < 0 ||
      max_blocks_per_seq < 0 || page_size <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP8_E4M3) return ATTN_ERR_INVALID_ARG;
  if ((page_size & (page_size - 1)) != 0 || page_size > 65536) return ATTN_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (d_qk != 128 || d_v != 128 || (G != 1 && G != 2 && G != 4 && G != 8 && G != 16))
    return ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(max_blocks_per_seq) * page_size > INT32_MAX || B > 65535 ||
      attn::dec_n_splits(B, Hkv, max_seqlen > 0 ? max_seqlen : 1) > 65535)
    return ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(max_seqlen) > static_cast<int64_t>(max_blocks_per_seq) * page_size)
    return ATTN_ERR_INVALID_ARG;
  if (B == 0) return ATTN_OK;
  if (!q || !o || !seq_lens) return ATTN_ERR_INVALID_ARG;
  if (dtype == ATTN_FP8_E4M3 && (!descale_q || !descale_k || !descale_v))
    return ATTN_ERR_INVALID_ARG;
  if (!workspace) return ATTN_ERR_INVALID_ARG;  // the partial results always go there
  if (max_seqlen > 0 && (!k_cache || !v_cache || !block_table || num_pages == 0 ||
                         max_blocks_per_seq == 0))
    return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 1u) || (reinterpret_cast<uintptr_t>(o) & 1u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(workspace) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return ATTN_ERR_ALIGNMENT;
  const int msl = max_seqlen > 0 ? max_seqlen : 1;
  if (workspace_bytes < attn_decode_workspace_size(B, Hq, Hkv, msl)) return ATTN_ERR_INVALID_ARG;
  attn::DecodeParams prm{};
  prm.q = q;
  prm.k_cache = static_cast<const uint8_t*>(k_cache);
  prm.v_cache = static_cast<const uint8_t*>(v_cache);
  prm.block_table = block_table;
  prm.seq_lens = seq_lens;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = G;
  prm.num_pages = num_pages;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  prm.page_shift = shift;
  prm.max_blocks = max_blocks_per_seq;
  prm.max_seqlen = max_seqlen;
  prm.n_splits = attn::dec_n_splits(B, Hkv, msl);
  prm.split_tokens = dtype == ATTN_FP8_E4M3 ? attn::dec_split_tokens<true>(msl, prm.n_splits)
                                          : attn::dec_split_tokens<false>(msl, prm.n_splits);
  prm.qk_scale = static_cast<float>((1.0 / std::sqrt(128.0)) * 1.4426950408889634);
  prm.descale_q = descale_q;
  prm.descale_k = descale_k;
  prm.descale_v = descale_v;
  prm.part_o = static_cast<float*>(workspace);
  prm.part_ml = prm.part_o + static_cast<size_t>(B) * Hq * prm.n_splits * attn::DEC_D;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  if (!dev_err_ptr(&prm.err)) return ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == ATTN_FP8_E4M3 ? dispatch_decode<true>(prm, st) : dispatch_decode<false>(prm, st);
}

attn_status_t attn_fwd_fp8_dump(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int Hq, int Hkv, int S, int d_qk, int d_v,
                                const float* descale_q, const float* descale_k,
                                const float* descale_v, int causal, unsigned flags,
                                float* dump_s, uint8_t* dump_codes, uint8_t* dump_kshift,
                                void* stream) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, S, d_qk, d_v, ATTN_FP8_E4M3, descale_q, descale_k,
                  descale_v, causal, flags, dump_s, dump_codes, dump_kshift, true, stream);
}

size_t attn_quantize_workspace_size(int64_t tokens, int H, int d) {
  (void)tokens;
  (void)H;
  (void)d;
  return 16;
}

attn_status_t attn_quantize_e4m3(const void* x_bf16, void* x_e4m3, float* descale_out,
                                 int64_t tokens, int H, int d, int hadamard, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (tokens < 0 || H <= 0 || d <= 0 || (d % 8) != 0) return ATTN_ERR_INVALID_ARG;
  if (hadamard != 0 && hadamard != 1) return ATTN_ERR_INVALID_ARG;
  if (hadamard && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!descale_out || !workspace) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < attn_quantize_workspace_size(tokens, H, d)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 3u) ||
      (reinterpret_cast<uintptr_t>(descale_out) & 3u))
    return ATTN_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows = tokens * H;
  uint32_t* amax = static_cast<uint32_t*>(workspace);
  if (rows == 0) {
    attn::descale_one_kernel<<<1, 1, 0, st>>>(descale_out);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (!x_bf16 || !x_e4m3) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(x_e4m3)) return ATTN_ERR_ALIGNMENT;
  const void* xs[1] = {x_bf16};
  void* ys[1] = {x_e4m3};
  float* dss[1] = {descale_out};
  const int64_t el[1] = {rows * d};
  return launch_quantize(1, xs, ys, dss, el, hadamard, amax, st);
}

size_t attn_quantize_qkv_workspace_size(void) { return 16; }

attn_status_t attn_quantize_qkv_e4m3(const void* q, const void* k, const void* v, void* q8,
                                     void* k8, void* v8, float* descale_q, float* descale_k,
                                     float* descale_v, int64_t tokens, int Hq, int Hkv, int d_qk,
                                     int d_v, int hadamard, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (tokens < 0 || Hq <= 0 || Hkv <= 0 || d_qk <= 0 || d_v <= 0 || (d_qk % 8) != 0 ||
      (d_v % 8) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (hadamard != 0 && hadamard != 1) return ATTN_ERR_INVALID_ARG;
  if (hadamard && (d_qk != 128 || d_v != 128)) return ATTN_ERR_UNSUPPORTED;
  if (!descale_q || !descale_k || !descale_v || !workspace) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < attn_quantize_qkv_workspace_size()) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 3u) ||
      (reinterpret_cast<uintptr_t>(descale_q) & 3u) ||
      (reinterpret_cast<uintptr_t>(descale_k) & 3u) ||
      (reinterpret_cast<uintptr_t>(descale_v) & 3u))
    return ATTN_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tokens == 0) {
    for (float* d : {descale_q, descale_k, descale_v}) {
      attn::descale_one_kernel<<<1, 1, 0, st>>>(d);
      if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  }
  if (!q || !k || !v || !q8 || !k8 || !v8) return ATTN_ERR_INVALID_ARG;
  for (const void* p : {q, k, v, static_cast<const void*>(q8), static_cast<const void*>(k8),
                        static_cast<const void*>(v8)})
    if (!aligned16(p)) return ATTN_ERR_ALIGNMENT;
  const int64_t el[3] = {tokens * Hq * d_qk, tokens * Hkv * d_qk, tokens * Hkv * d_v};
  const void* xs[3] = {q, k, v};
  void* ys[3] = {q8, k8, v8};
  float* dss[3] = {descale_q, descale_k, descale_v};
  return launch_quantize(3, xs, ys, dss, el, hadamard, static_cast<uint32_t*>(workspace), st);
}

attn_status_t attn_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ERR_CUDA;
  uint32_t host = 0;
  if (cudaMemcpyFromSymbol(&host, g_dev_err, sizeof(host)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (host != attn::DEV_OK) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
    return host == attn::DEV_BAD_SEQLENS ? ATTN_ERR_INVALID_ARG : ATTN_ERR_TIMEOUT;
  }
  return ATTN_OK;
}

void attn_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns ? ns : kDefaultTimeoutNs; }

void attn_selftest_stall_tile(int tile) { g_stall_tile = tile < 0 ? -1 : tile; }

void attn_selftest_max_ctas(int n) { g_max_ctas = n > 0 ? n : 0; }

attn_status_t attn_select_prefill_kernel(int kernel) {
  if (kernel != ATTN_KERNEL_AUTO &&
      ((kernel & ~(ATTN_KERNEL_HEADS | ATTN_KERNEL_PERSISTENT | ATTN_KERNEL_DYNAMIC |
                   ATTN_KERNEL_BF16_S_AHEAD | ATTN_KERNEL_BF16_P_OVER_S)) != 0 ||
       ((kernel & ATTN_KERNEL_PERSISTENT) && (kernel & ATTN_KERNEL_DYNAMIC)) ||
       ((kernel & ATTN_KERNEL_BF16_S_AHEAD) && (kernel & ATTN_KERNEL_BF16_P_OVER_S))))
    return ATTN_ERR_INVALID_ARG;
  g_kernel = kernel;
  return ATTN_OK;
}

attn_status_t attn_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  uint32_t* err = nullptr;
  if (!dev_err_ptr(&err)) return ATTN_ERR_CUDA;
  selftest_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(err, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape or option";
    case ATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int attn_version(void) { return kVersion; }

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Quantiser entry point for callers that cannot allocate device memory.
//
// attn_quantize_e4m3 needs a few bytes of device scratch (the running amax).  Some callers
// cannot provide it: a plugin running inside an engine whose device memory is planned and
// owned entirely by the host framework, or a latency-critical loop where a cudaMalloc
// (which may synchronise the device) is not allowed.  attn_quantize_e4m3_static takes the
// scratch from a fixed array compiled into this library instead.  Every GPU that loads the
// library holds the array until the process exits.
namespace {

constexpr size_t kStaticScratchBytes = 256;  // maximum scratch this entry point can use
static __device__ __align__(256) uint32_t g_static_scratch[kStaticScratchBytes / 4];

// Device address of g_static_scratch in the current context.  In host code the array's
// name only stands in for the symbol; the runtime translates it for the device (and
// context) current at the call.  It is looked up on every call -- a lookup allocates
// nothing -- so the address stays right after cudaDeviceReset or in another context.  The
// first call on a device loads this library's device code there if it is not yet loaded,
// which must not happen during a stream capture.
attn_status_t static_scratch(uint32_t** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
    return ATTN_ERR_CUDA;
  *out = static_cast<uint32_t*>(p);
  return ATTN_OK;
}

}  // namespace

extern "C" attn_status_t attn_quantize_e4m3_static(const void* x_bf16, void* x_e4m3,
                                                   float* descale_out, int64_t tokens, int H,
                                                   int d, int hadamard, void* stream) {
  if (tokens < 0 || H <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (attn_quantize_workspace_size(tokens, H, d) > kStaticScratchBytes)
    return ATTN_ERR_UNSUPPORTED;  // would need more scratch than the fixed array holds
  uint32_t* scratch = nullptr;
  const attn_status_t st = static_scratch(&scratch);
  if (st != ATTN_OK) return st;
  // same kernels as attn_quantize_e4m3; the amax word is cleared at the start of every call
  return attn_quantize_e4m3(x_bf16, x_e4m3, descale_out, tokens, H, d, hadamard, scratch,
                            kStaticScratchBytes, stream);
}
