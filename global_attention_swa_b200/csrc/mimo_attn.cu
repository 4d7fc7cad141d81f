// Host side of the C ABI declared in include/mimo_attn.h: argument checks,
// TMA descriptor encoding, the decode split plan, and kernel launches.
// All kernels of the library live in this one translation unit so that the
// device status word is shared without relocatable device code.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>

#ifndef MIMO_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

#include "../../include/mimo_attn.h"
#include "common.cuh"
#include "decode_kernel.cuh"
#include "decode_fp8_kernel.cuh"
#include "rope_append_kernel.cuh"
#include "decode_merge_kernel.cuh"
#include "backward_kernel.cuh"
#include "backward_tc_kernel.cuh"
#include "backward_dq_tc_kernel.cuh"
#include "prefill_kernel.cuh"
#include "prefill_swa_kernel.cuh"

#undef MIMO_FILE_ID
#define MIMO_FILE_ID 10  // site numbers of the checked build

namespace {
// An NVTX range around each compute entry point, named after it, so that a
// profiler's timeline groups each call's launches (header-only NVTX v3: with
// no tool attached a push / pop costs a check of a function pointer).
// -DMIMO_NO_NVTX builds without it.
struct NvtxRange {
#ifndef MIMO_NO_NVTX
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
#else
  explicit NvtxRange(const char*) {}
#endif
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace

namespace mimo {
__device__ __align__(16) unsigned char g_wait_selftest_src[16];

// A real time-out, for the failure-path test: one thread copies 16 bytes in
// with a bulk copy; another waits on a barrier nothing ever arrives at, gives
// up after the bound, records MIMO_ERR_TIMEOUT and raises the CTA's abort
// flag; the teardown then waits for the armed copy, as the kernels do.
__global__ void __launch_bounds__(64) wait_selftest_kernel() {
  __shared__ __align__(16) unsigned char buf[16];
  __shared__ __align__(8) uint64_t bars[2];  // [0] the copy, [1] never arrived at
  __shared__ int abort_flag, never;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    never = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars[0], 16);
    bulk_load(buf, g_wait_selftest_src, 16, &bars[0]);
  }
  if (threadIdx.x == 32) wait_bounded(&bars[1], 0, &abort_flag);
  __syncthreads();
  if (*reinterpret_cast<volatile int*>(&abort_flag) && threadIdx.x == 0) drain_armed(&bars[0], 1, &never);
}
}  // namespace mimo

#ifdef MIMO_CHECKED
namespace mimo {
// One row index past a 4-row buffer, checked and not used for any access.
__global__ void checked_selftest_kernel() {
  const volatile int row = 4;
  if (MIMO_ROW_OK(row, 4)) record_status(3 /* not reached: the check fails */);
}
}  // namespace mimo
#endif

namespace {

thread_local std::string g_last_error;

mimo_status_t fail(mimo_status_t st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
mimo_status_t fail(mimo_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

mimo_status_t ok() {
  g_last_error.clear();
  return MIMO_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor with `rank` dims (innermost first), byte strides of dims 1.., box sizes.
mimo_status_t make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MIMO_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t gd[5], gs[4];
  cuuint32_t bd[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bd[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, rank, const_cast<void*>(base), gd, gs, bd,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MIMO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MIMO_OK;
}

// ---------------------------------------------------------------- common checks

mimo_status_t check_dims(const mimo_attn_dims_t* d) {
  if (!d) return fail(MIMO_ERR_INVALID_ARG, "dims is NULL");
  if (d->num_heads_q <= 0 || d->num_heads_kv <= 0)
    return fail(MIMO_ERR_INVALID_ARG, "head counts must be positive (Hq=%d, Hkv=%d)",
                d->num_heads_q, d->num_heads_kv);
  if (d->num_heads_q % d->num_heads_kv)
    return fail(MIMO_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", d->num_heads_q,
                d->num_heads_kv);
  if (d->head_dim_qk != 192 || d->head_dim_v != 128)
    return fail(MIMO_ERR_UNSUPPORTED, "only head_dim_qk=192, head_dim_v=128 are built (got %d, %d)",
                d->head_dim_qk, d->head_dim_v);
  if (d->out_dtype != MIMO_DTYPE_BF16 && d->out_dtype != MIMO_DTYPE_F32)
    return fail(MIMO_ERR_INVALID_ARG, "out_dtype must be MIMO_DTYPE_BF16 or MIMO_DTYPE_F32");
  if (!std::isfinite(d->softmax_scale) || !std::isfinite(d->v_scale))
    return fail(MIMO_ERR_INVALID_ARG, "softmax_scale and v_scale must be finite");
  return MIMO_OK;
}

float scale_log2_of(const mimo_attn_dims_t* d) {
  const float s = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / std::sqrt((float)d->head_dim_qk);
  return s * 1.4426950408889634f;
}

float v_scale_of(const mimo_attn_dims_t* d) { return d->v_scale != 0.f ? d->v_scale : 1.0f; }

mimo_status_t cuda_check(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(MIMO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MIMO_OK;
}

// Opt every kernel into its dynamic shared memory once per device.
mimo_status_t ensure_attributes() {
  static std::mutex mu;
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(MIMO_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(mu);
  if (done[dev]) return MIMO_OK;
  mimo_status_t st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::prefill_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kPfSmemBytes),
                       "prefill smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::prefill_swa_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kSwSmemBytes),
                       "sliding-window prefill smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::decode_split_kernel<mimo::kDecStages, 1, mimo::kDecTileKeys>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kDecSmemBytes),
                       "decode smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::decode_split_kernel<mimo::kDecShortStages, 2, mimo::kDecTileKeys>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::dec_smem_bytes(mimo::kDecShortStages)),
                       "short-cache decode smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::decode_split_kernel<mimo::kDecRingStages, 2, mimo::kDecRingRows>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::dec_smem_bytes(mimo::kDecRingStages, mimo::kDecRingRows)),
                       "ring decode smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::bwd_dq_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kBqSmemBytes),
                       "backward dq smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::bwd_dkv_kernel<true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kBkSmemBytes),
                       "backward dv smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::bwd_dkv_tc_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kBtSmemBytes),
                       "backward dk/dv (tcgen05) smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::bwd_dq_tc_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kBdSmemBytes),
                       "backward dq (tcgen05) smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::bwd_dkv_kernel<false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kBkSmemBytes),
                       "backward dk smem attribute")))
    return st;
  if ((st = cuda_check(cudaFuncSetAttribute(mimo::decode_split_fp8_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            mimo::kD8SmemBytes),
                       "FP8 decode smem attribute")))
    return st;
  done[dev] = true;
  return MIMO_OK;
}

// SMs of the current device (148 on B200; also the answer without a device,
// so that host-only size queries match the launches on B200).
int sm_count() {
  static std::atomic<int> counts[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int c = counts[dev].load(std::memory_order_relaxed);
  if (c <= 0) {
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
      c = 148;
    counts[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

// ---------------------------------------------------------------- decode plan

struct DecodePlan {
  int ring, cap_eff, chunk, nsplit;
};

int env_chunk() {
  static int v = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    const char* s = std::getenv("MIMO_DECODE_CHUNK");
    v = s ? std::atoi(s) : 0;
  });
  return v;
}

DecodePlan decode_plan(int batch, int hkv, int capacity, int window) {
  DecodePlan pl;
  pl.ring = (window > 0 && capacity == window) ? 1 : 0;
  pl.cap_eff = (!pl.ring && window > 0) ? std::min(window, capacity) : capacity;
  const int tile = mimo::kDecTileKeys;
  // Aim for >= 2 resident work units per SM across the grid, splits of
  // 256..16384 keys (a split's fixed costs -- query fragments, the warp merge,
  // its partial and the combine -- fall behind its streaming from ~8K keys on:
  // at batch 64 x 262144 slots, 16384-key splits run 9 % faster than 2048);
  // a single split needs no workspace and no combine.
  int chunk = env_chunk();
  if (chunk <= 0) {
    const long units = (long)batch * hkv;
    const long want = 2L * sm_count();
    long nsplit = (want + units - 1) / units;
    long max_split = std::max(1L, ((long)pl.cap_eff + 255) / 256);
    nsplit = std::max(1L, std::min(nsplit, max_split));
    long c = ((long)pl.cap_eff + nsplit - 1) / nsplit;
    chunk = (int)std::min<long>(c, 16384);
  }
  chunk = std::max(tile, ((chunk + tile - 1) / tile) * tile);
  pl.chunk = chunk;
  pl.nsplit = std::max(1, (pl.cap_eff + chunk - 1) / chunk);
  return pl;
}

size_t workspace_bytes_of(int batch, int hkv, const DecodePlan& pl) {
  if (pl.nsplit <= 1) return 0;
  const size_t units = (size_t)batch * hkv * pl.nsplit;
  // partial O [units][16][128], then (max, sum, rounded-P sum, unused) [units][16][4]
  return units * 16 * 128 * sizeof(float) + units * 16 * 4 * sizeof(float);
}

}  // namespace

extern "C" {

const char* mimo_attn_last_error(void) { return g_last_error.c_str(); }

mimo_status_t mimo_attn_prefill(const mimo_attn_dims_t* dims, const void* q, const void* k,
                                const void* v, const float* sinks, int window,
                                const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                                int max_seqlen, void* out, float* lse, void* stream) {
  NvtxRange nvtx_range("mimo_attn_prefill");
  mimo_status_t st = check_dims(dims);
  if (st) return st;
  if (window < 0) return fail(MIMO_ERR_INVALID_ARG, "window must be >= 0 (got %d)", window);
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0)
    return fail(MIMO_ERR_INVALID_ARG, "sizes must be non-negative");
  if (!cu_seqlens) return fail(MIMO_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (total_tokens == 0 || num_seqs == 0 || max_seqlen == 0) return ok();  // nothing to do
  if (!q || !k || !v || !out) return fail(MIMO_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (lse && ((uintptr_t)lse & 3u)) || (sinks && ((uintptr_t)sinks & 3u)))
    return fail(MIMO_ERR_INVALID_ARG, "q, k, v, out must be 16-byte aligned");
  if (max_seqlen > total_tokens)
    return fail(MIMO_ERR_INVALID_ARG, "max_seqlen (%d) > total_tokens (%d)", max_seqlen, total_tokens);
  if (num_seqs > 65535) return fail(MIMO_ERR_UNSUPPORTED, "num_seqs > 65535");
  const int Hq = dims->num_heads_q, Hkv = dims->num_heads_kv, G = Hq / Hkv;
  if ((st = ensure_attributes())) return st;

  // Sliding window with the key/value group packed into one 128-row tile:
  // 128 / G queries x G heads per block, one score tile of N keys per block.
  const int QB = (G >= 8 && 128 % G == 0) ? 128 / G : 0;
  const int Nsw = QB ? ((window + 2 * QB - 1 + 15) / 16) * 16 : 0;  // window of a block pair
  if (window > 0 && QB > 0 && Nsw <= mimo::kSwNMax) {
    CUtensorMap tq, tk, tv;
    {
      const uint64_t d[3] = {192, (uint64_t)Hq, (uint64_t)total_tokens};
      const uint64_t s[2] = {192 * 2, (uint64_t)Hq * 192 * 2};
      const uint32_t b[3] = {64, (uint32_t)G, (uint32_t)QB};
      if ((st = make_map(&tq, q, 3, d, s, b))) return st;
    }
    {
      const uint64_t d[3] = {192, (uint64_t)Hkv, (uint64_t)total_tokens};
      const uint64_t s[2] = {192 * 2, (uint64_t)Hkv * 192 * 2};
      const uint32_t b[3] = {64, 1, (uint32_t)Nsw};
      if ((st = make_map(&tk, k, 3, d, s, b))) return st;
    }
    {
      const uint64_t d[3] = {128, (uint64_t)Hkv, (uint64_t)total_tokens};
      const uint64_t s[2] = {128 * 2, (uint64_t)Hkv * 128 * 2};
      const uint32_t b[3] = {64, 1, (uint32_t)Nsw};
      if ((st = make_map(&tv, v, 3, d, s, b))) return st;
    }
    mimo::SwaParams sp;
    sp.cu_seqlens = cu_seqlens;
    sp.sinks = sinks;
    sp.out = out;
    sp.lse = lse;
    sp.total = total_tokens;
    sp.Hq = Hq;
    sp.Hkv = Hkv;
    sp.G = G;
    sp.QB = QB;
    sp.N = Nsw;
    sp.window = window;
    sp.num_seqs = num_seqs;
    sp.max_seqlen = max_seqlen;
    sp.num_pairs = (max_seqlen + 2 * QB - 1) / (2 * QB);
    const long items = (long)sp.num_pairs * Hkv * num_seqs;
    if (items > 0x7fffffffL) return fail(MIMO_ERR_UNSUPPORTED, "too many work items (%ld)", items);
    sp.num_items = (int)items;
    sp.scale_log2 = scale_log2_of(dims);
    sp.v_scale = v_scale_of(dims);
    sp.out_f32 = dims->out_dtype == MIMO_DTYPE_F32;
    sp.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    const int grid = (int)std::min<long>(items, sm_count());
    mimo::prefill_swa_kernel<<<grid, mimo::kSwThreads, mimo::kSwSmemBytes, (cudaStream_t)stream>>>(
        tq, tk, tv, sp);
    if ((st = cuda_check(cudaGetLastError(), "sliding-window prefill launch"))) return st;
    return ok();
  }

  CUtensorMap tq, tk, tv;
  {
    const uint64_t d[3] = {192, (uint64_t)Hq, (uint64_t)total_tokens};
    const uint64_t s[2] = {192 * 2, (uint64_t)Hq * 192 * 2};
    const uint32_t b[3] = {64, 1, 128};
    if ((st = make_map(&tq, q, 3, d, s, b))) return st;
  }
  {
    const uint64_t d[3] = {192, (uint64_t)Hkv, (uint64_t)total_tokens};
    const uint64_t s[2] = {192 * 2, (uint64_t)Hkv * 192 * 2};
    const uint32_t b[3] = {64, 1, 128};
    if ((st = make_map(&tk, k, 3, d, s, b))) return st;
  }
  {
    const uint64_t d[3] = {128, (uint64_t)Hkv, (uint64_t)total_tokens};
    const uint64_t s[2] = {128 * 2, (uint64_t)Hkv * 128 * 2};
    const uint32_t b[3] = {64, 1, 128};
    if ((st = make_map(&tv, v, 3, d, s, b))) return st;
  }
  mimo::PrefillParams p;
  p.cu_seqlens = cu_seqlens;
  p.sinks = sinks;
  p.out = out;
  p.lse = lse;
  p.total = total_tokens;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.window = window;
  p.pairs_per_group = (G + 1) / 2;
  p.scale_log2 = scale_log2_of(dims);
  p.v_scale = v_scale_of(dims);
  p.out_f32 = dims->out_dtype == MIMO_DTYPE_F32;
  p.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
  p.num_seqs = num_seqs;
  p.max_seqlen = max_seqlen;
  p.num_qtiles = (max_seqlen + mimo::kPfTile - 1) / mimo::kPfTile;
  const long items = (long)p.num_qtiles * Hkv * p.pairs_per_group * num_seqs;
  if (items > 0x7fffffffL) return fail(MIMO_ERR_UNSUPPORTED, "too many work items (%ld)", items);
  p.num_items = (int)items;
  // persistent: one CTA per SM (225 KB of shared memory and all of TMEM each)
  const int grid = (int)std::min<long>(items, sm_count());
  mimo::prefill_kernel<<<grid, mimo::kPfThreads, mimo::kPfSmemBytes, (cudaStream_t)stream>>>(
      tq, tk, tv, p);
  if ((st = cuda_check(cudaGetLastError(), "prefill launch"))) return st;
  return ok();
}

size_t mimo_attn_decode_workspace_size(const mimo_attn_dims_t* dims, int batch, int capacity,
                                       int window) {
  if (!dims || dims->num_heads_kv <= 0 || batch <= 0 || capacity <= 0 || window < 0) return 0;
  return workspace_bytes_of(batch, dims->num_heads_kv,
                            decode_plan(batch, dims->num_heads_kv, capacity, window));
}

}  // extern "C"

namespace {

// Decode over a bf16 cache (fp8 = false) or an e4m3 cache with per-KV-head
// scales (fp8 = true); both entry points validate and launch here.
mimo_status_t decode_impl(const mimo_attn_dims_t* dims, const void* q, const void* k_cache,
                          const void* v_cache, bool fp8, const float* k_scale,
                          const float* v_scale_kv, const int32_t* seqlens, int batch,
                          int capacity, int window, const float* sinks, void* out, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream) {
  mimo_status_t st = check_dims(dims);
  if (st) return st;
  if (window < 0) return fail(MIMO_ERR_INVALID_ARG, "window must be >= 0 (got %d)", window);
  if (batch < 0 || capacity < 0) return fail(MIMO_ERR_INVALID_ARG, "sizes must be non-negative");
  if (batch == 0) return ok();
  if (capacity == 0) return fail(MIMO_ERR_INVALID_ARG, "capacity must be positive");
  if (!q || !k_cache || !v_cache || !seqlens || !out)
    return fail(MIMO_ERR_INVALID_ARG, "q, k_cache, v_cache, seqlens and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (lse && ((uintptr_t)lse & 3u)) || (sinks && ((uintptr_t)sinks & 3u)))
    return fail(MIMO_ERR_INVALID_ARG, "q, caches and out must be 16-byte aligned");
  if (fp8 && (!k_scale || !v_scale_kv))
    return fail(MIMO_ERR_INVALID_ARG, "an FP8 cache needs k_scale and v_scale_kv");
  if (fp8 && (((uintptr_t)k_scale & 3u) || ((uintptr_t)v_scale_kv & 3u)))
    return fail(MIMO_ERR_INVALID_ARG, "k_scale and v_scale_kv must be 4-byte aligned");
  const int Hq = dims->num_heads_q, Hkv = dims->num_heads_kv, G = Hq / Hkv;
  if (G > 16) return fail(MIMO_ERR_UNSUPPORTED, "decode packs at most 16 query heads per KV head (got %d)", G);
  if ((long)batch * capacity > 0x7fffffffL)
    return fail(MIMO_ERR_UNSUPPORTED, "batch * capacity must fit in int32");
  if (batch > 65535 || Hkv > 65535) return fail(MIMO_ERR_UNSUPPORTED, "batch or Hkv > 65535");
  const DecodePlan pl = decode_plan(batch, Hkv, capacity, window);
  const size_t need = workspace_bytes_of(batch, Hkv, pl);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(MIMO_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, workspace_bytes);
  if (need > 0 && !aligned16(workspace))
    return fail(MIMO_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((st = ensure_attributes())) return st;

  // A small ring (at most 3 x 48 slots, e.g. the 129-slot sliding-window cache)
  // is streamed whole in three equal tiles (43 rows for 129 slots), issued
  // before the sequence length is known.
  const bool small_ring = !fp8 && pl.ring && pl.nsplit == 1 &&
                          capacity <= mimo::kDecRingStages * mimo::kDecRingRows;
  int tile = mimo::kDecTileKeys, spec_tiles = 0;
  if (small_ring) {
    spec_tiles = (capacity + mimo::kDecRingRows - 1) / mimo::kDecRingRows;
    tile = (capacity + spec_tiles - 1) / spec_tiles;
  }
  CUtensorMap tk, tv;
  {
    // bf16: boxes of 64 elements (128 B, 128-byte swizzle); e4m3: 64 bytes, 64-byte swizzle
    const int eb = fp8 ? 1 : 2;
    const CUtensorMapDataType dt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = fp8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    const uint32_t rows = fp8 ? (uint32_t)mimo::kD8TileKeys : (uint32_t)tile;
    {
      const uint64_t d[2] = {(uint64_t)Hkv * 192, (uint64_t)batch * capacity};
      const uint64_t s[1] = {(uint64_t)Hkv * 192 * eb};
      const uint32_t b[2] = {64, rows};
      if ((st = make_map(&tk, k_cache, 2, d, s, b, dt, sw))) return st;
    }
    {
      const uint64_t d[2] = {(uint64_t)Hkv * 128, (uint64_t)batch * capacity};
      const uint64_t s[1] = {(uint64_t)Hkv * 128 * eb};
      const uint32_t b[2] = {64, rows};
      if ((st = make_map(&tv, v_cache, 2, d, s, b, dt, sw))) return st;
    }
  }
  mimo::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.seqlens = seqlens;
  p.sinks = sinks;
  p.out = out;
  p.lse = lse;
  const size_t units = (size_t)batch * Hkv * pl.nsplit;
  p.ws_o = need ? static_cast<float*>(workspace) : nullptr;
  p.ws_ml = need ? static_cast<float*>(workspace) + units * 16 * 128 : nullptr;
  p.B = batch;
  p.C = capacity;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.window = window;
  p.ring = pl.ring;
  p.chunk = pl.chunk;
  p.nsplit = pl.nsplit;
  p.tile = tile;
  p.spec_tiles = spec_tiles;
  p.scale_log2 = scale_log2_of(dims);
  p.v_scale = v_scale_of(dims);
  p.out_f32 = dims->out_dtype == MIMO_DTYPE_F32;
  p.k_scale = fp8 ? k_scale : nullptr;
  p.kv_v_scale = fp8 ? v_scale_kv : nullptr;
  dim3 grid(pl.nsplit, Hkv, batch);
  if (fp8)
    mimo::decode_split_fp8_kernel<<<grid, mimo::kD8Threads, mimo::kD8SmemBytes, (cudaStream_t)stream>>>(
        tk, tv, p);
  else if (small_ring)
    mimo::decode_split_kernel<mimo::kDecRingStages, 2, mimo::kDecRingRows>
        <<<grid, mimo::kDecThreads, mimo::dec_smem_bytes(mimo::kDecRingStages, mimo::kDecRingRows),
           (cudaStream_t)stream>>>(tk, tv, p);
  else if (pl.cap_eff <= mimo::kDecShortKeys)
    mimo::decode_split_kernel<mimo::kDecShortStages, 2, mimo::kDecTileKeys>
        <<<grid, mimo::kDecThreads, mimo::dec_smem_bytes(mimo::kDecShortStages), (cudaStream_t)stream>>>(tk, tv, p);
  else
    mimo::decode_split_kernel<mimo::kDecStages, 1, mimo::kDecTileKeys>
        <<<grid, mimo::kDecThreads, mimo::kDecSmemBytes, (cudaStream_t)stream>>>(tk, tv, p);
  if ((st = cuda_check(cudaGetLastError(), "decode launch"))) return st;
  if (pl.nsplit > 1) {
    const int warps = batch * Hq;
    const int blocks = (warps * 32 + 255) / 256;
    mimo::decode_combine_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(p);
    if ((st = cuda_check(cudaGetLastError(), "decode combine launch"))) return st;
  }
  return ok();
}

}  // namespace

extern "C" {

mimo_status_t mimo_attn_decode(const mimo_attn_dims_t* dims, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* seqlens, int batch,
                               int capacity, int window, const float* sinks, void* out,
                               float* lse, void* workspace, size_t workspace_bytes,
                               void* stream) {
  NvtxRange nvtx_range("mimo_attn_decode");
  return decode_impl(dims, q, k_cache, v_cache, false, nullptr, nullptr, seqlens, batch, capacity,
                     window, sinks, out, lse, workspace, workspace_bytes, stream);
}

size_t mimo_attn_decode_fp8_workspace_size(const mimo_attn_dims_t* dims, int batch, int capacity,
                                           int window) {
  return mimo_attn_decode_workspace_size(dims, batch, capacity, window);
}

mimo_status_t mimo_attn_decode_fp8(const mimo_attn_dims_t* dims, const void* q,
                                   const void* k_cache, const void* v_cache,
                                   const float* k_scale, const float* v_scale_kv,
                                   const int32_t* seqlens, int batch, int capacity, int window,
                                   const float* sinks, void* out, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("mimo_attn_decode_fp8");
  return decode_impl(dims, q, k_cache, v_cache, true, k_scale, v_scale_kv, seqlens, batch,
                     capacity, window, sinks, out, lse, workspace, workspace_bytes, stream);
}

mimo_status_t mimo_attn_rope_append(const mimo_attn_dims_t* dims, void* q, const void* k_new,
                                    const void* v_new, void* k_cache, void* v_cache,
                                    const int32_t* seqlens, int batch, int capacity, int window,
                                    float rope_theta, int rotary_dim, void* stream) {
  NvtxRange nvtx_range("mimo_attn_rope_append");
  mimo_status_t st = check_dims(dims);
  if (st) return st;
  if (window < 0) return fail(MIMO_ERR_INVALID_ARG, "window must be >= 0 (got %d)", window);
  if (batch < 0 || capacity < 0) return fail(MIMO_ERR_INVALID_ARG, "sizes must be non-negative");
  if (batch == 0) return ok();
  if (capacity == 0) return fail(MIMO_ERR_INVALID_ARG, "capacity must be positive");
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta))
    return fail(MIMO_ERR_INVALID_ARG, "rope_theta must be positive and finite");
  if (rotary_dim < 0 || rotary_dim > dims->head_dim_qk || (rotary_dim & 1))
    return fail(MIMO_ERR_INVALID_ARG, "rotary_dim must be even and in [0, %d] (got %d)",
                dims->head_dim_qk, rotary_dim);
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !seqlens)
    return fail(MIMO_ERR_INVALID_ARG, "q, k_new, v_new, caches and seqlens must be non-NULL");
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache))
    return fail(MIMO_ERR_INVALID_ARG, "q, k_new, v_new and the caches must be 16-byte aligned");
  if ((long)batch * capacity > 0x7fffffffL)
    return fail(MIMO_ERR_UNSUPPORTED, "batch * capacity must fit in int32");
  mimo::RopeAppendParams p;
  p.q = static_cast<__nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  p.seqlens = seqlens;
  p.B = batch;
  p.C = capacity;
  p.Hq = dims->num_heads_q;
  p.Hkv = dims->num_heads_kv;
  p.ring = (window > 0 && capacity == window) ? 1 : 0;
  p.rotary_dim = rotary_dim;
  for (int i = 0; i < mimo::kRaMaxHalf; ++i)
    p.inv_freq[i] = (rotary_dim > 0 && i < rotary_dim / 2)
                        ? std::pow((double)rope_theta, -2.0 * i / (double)rotary_dim)
                        : 0.0;
  if (batch > 0x7fffffff || p.Hq > 65535 * mimo::kRaHeadsPerCta)
    return fail(MIMO_ERR_UNSUPPORTED, "batch or Hq too large");
  const dim3 grid(batch, (p.Hq + mimo::kRaHeadsPerCta - 1) / mimo::kRaHeadsPerCta + 1);
  mimo::rope_append_kernel<<<grid, mimo::kRaThreads, 0, (cudaStream_t)stream>>>(p);
  if ((st = cuda_check(cudaGetLastError(), "rope/append launch"))) return st;
  return ok();
}

mimo_status_t mimo_attn_decode_merge(const mimo_attn_dims_t* dims, const float* part_out,
                                     const float* part_lse, int num_parts, int batch,
                                     const float* sinks, void* out, float* lse, void* stream) {
  NvtxRange nvtx_range("mimo_attn_decode_merge");
  mimo_status_t st = check_dims(dims);
  if (st) return st;
  if (num_parts < 1) return fail(MIMO_ERR_INVALID_ARG, "num_parts must be >= 1 (got %d)", num_parts);
  if (batch < 0) return fail(MIMO_ERR_INVALID_ARG, "batch must be non-negative");
  if (batch == 0) return ok();
  if (!part_out || !part_lse || !out)
    return fail(MIMO_ERR_INVALID_ARG, "part_out, part_lse and out must be non-NULL");
  if (!aligned16(part_out) || !aligned16(out) || ((uintptr_t)part_lse & 3u) ||
      (lse && ((uintptr_t)lse & 3u)) || (sinks && ((uintptr_t)sinks & 3u)))
    return fail(MIMO_ERR_INVALID_ARG, "part_out and out must be 16-byte aligned");
  const long warps = (long)batch * dims->num_heads_q;
  if (warps * 32 > 0x7fffffffL) return fail(MIMO_ERR_UNSUPPORTED, "batch * Hq too large");
  mimo::DecodeMergeParams p;
  p.part_out = part_out;
  p.part_lse = part_lse;
  p.sinks = sinks;
  p.out = out;
  p.lse = lse;
  p.R = num_parts;
  p.B = batch;
  p.Hq = dims->num_heads_q;
  p.v_scale = v_scale_of(dims);
  p.out_f32 = dims->out_dtype == MIMO_DTYPE_F32;
  const int blocks = (int)((warps * 32 + 255) / 256);
  mimo::decode_merge_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(p);
  if ((st = cuda_check(cudaGetLastError(), "decode merge launch"))) return st;
  return ok();
}

size_t mimo_attn_prefill_backward_workspace_size(const mimo_attn_dims_t* dims, int total_tokens) {
  if (!dims || dims->num_heads_q <= 0 || total_tokens <= 0) return 0;
  return (size_t)2 * dims->num_heads_q * total_tokens * sizeof(float);
}

mimo_status_t mimo_attn_prefill_backward(const mimo_attn_dims_t* dims, const void* q, const void* k,
                                         const void* v, const void* out, const float* lse,
                                         const void* dout, const float* sinks, int window,
                                         const int32_t* cu_seqlens, int num_seqs,
                                         int total_tokens, int max_seqlen, float* dq, float* dk,
                                         float* dv, float* dsinks, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("mimo_attn_prefill_backward");
  mimo_status_t st = check_dims(dims);
  if (st) return st;
  if (window < 0) return fail(MIMO_ERR_INVALID_ARG, "window must be >= 0 (got %d)", window);
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0)
    return fail(MIMO_ERR_INVALID_ARG, "sizes must be non-negative");
  if (!cu_seqlens) return fail(MIMO_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (total_tokens == 0 || num_seqs == 0 || max_seqlen == 0) return ok();
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)
    return fail(MIMO_ERR_INVALID_ARG, "q, k, v, out, lse, dout, dq, dk and dv must be non-NULL");
  if (sinks && !dsinks) return fail(MIMO_ERR_INVALID_ARG, "dsinks is NULL while sinks is given");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || ((uintptr_t)lse & 3u) ||
      (sinks && ((uintptr_t)sinks & 3u)) || (dsinks && ((uintptr_t)dsinks & 3u)))
    return fail(MIMO_ERR_INVALID_ARG, "tensors must be 16-byte aligned (lse, sinks, dsinks 4-byte)");
  if (max_seqlen > total_tokens)
    return fail(MIMO_ERR_INVALID_ARG, "max_seqlen (%d) exceeds total_tokens (%d)", max_seqlen,
                total_tokens);
  if (num_seqs > 65535) return fail(MIMO_ERR_UNSUPPORTED, "num_seqs > 65535");
  const size_t need = mimo_attn_prefill_backward_workspace_size(dims, total_tokens);
  if (!workspace || workspace_bytes < need)
    return fail(MIMO_ERR_WORKSPACE, "backward workspace of %zu bytes needed (got %zu)", need,
                workspace_bytes);
  if ((uintptr_t)workspace & 15u) return fail(MIMO_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((long)total_tokens * dims->num_heads_q * 32 > 0x7fffffffL * 255L)
    return fail(MIMO_ERR_UNSUPPORTED, "total_tokens * Hq too large");
  if ((st = ensure_attributes())) return st;
  mimo::BackwardParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.out = out;
  p.dout = dout;
  p.lse = lse;
  p.sinks = sinks;
  p.cu_seqlens = cu_seqlens;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dsinks = dsinks;
  p.D = static_cast<float*>(workspace);
  p.psd = p.D + (size_t)dims->num_heads_q * total_tokens;
  p.total = total_tokens;
  p.Hq = dims->num_heads_q;
  p.Hkv = dims->num_heads_kv;
  p.G = p.Hq / p.Hkv;
  p.window = window;
  p.num_seqs = num_seqs;
  p.max_seqlen = max_seqlen;
  p.scale = dims->softmax_scale > 0.f ? dims->softmax_scale : 1.0f / std::sqrt((float)dims->head_dim_qk);
  p.scale_log2 = scale_log2_of(dims);
  p.v_scale = v_scale_of(dims);
  p.io_f32 = dims->out_dtype == MIMO_DTYPE_F32;
  cudaStream_t s = (cudaStream_t)stream;
  const long pre_threads = (long)total_tokens * p.Hq * 32;
  mimo::bwd_preprocess_kernel<<<(unsigned)((pre_threads + 255) / 256), 256, 0, s>>>(p);
  if ((st = cuda_check(cudaGetLastError(), "backward preprocess launch"))) return st;
  if (sinks) {
    mimo::bwd_sink_kernel<<<p.Hq, 256, 0, s>>>(p);
    if ((st = cuda_check(cudaGetLastError(), "backward sink launch"))) return st;
  }
  const int tiles = (max_seqlen + mimo::kBwTile - 1) / mimo::kBwTile;
  const int qtiles = (max_seqlen + mimo::kBqRows - 1) / mimo::kBqRows;
  if (p.io_f32) {
    mimo::bwd_dq_kernel<<<dim3(qtiles, p.Hq, num_seqs), mimo::kBkThreads, mimo::kBqSmemBytes, s>>>(p);
    if ((st = cuda_check(cudaGetLastError(), "backward dq launch"))) return st;
  }
  if (!p.io_f32) {
    // bf16 out / dout: dQ, then dK and dV, on tcgen05 over 128-key tiles
    CUtensorMap tq, tk, tv, tdo, tq128, tdo128;
    const int Hq = p.Hq, Hkv = p.Hkv;
    {
      const uint64_t d[3] = {192, (uint64_t)Hq, (uint64_t)total_tokens};
      const uint64_t st2[2] = {192 * 2, (uint64_t)Hq * 192 * 2};
      const uint32_t b[3] = {64, 1, mimo::kBtQ};
      if ((st = make_map(&tq, q, 3, d, st2, b))) return st;
      const uint32_t b128[3] = {64, 1, mimo::kBdRows};
      if ((st = make_map(&tq128, q, 3, d, st2, b128))) return st;
    }
    {
      const uint64_t d[3] = {128, (uint64_t)Hq, (uint64_t)total_tokens};
      const uint64_t st2[2] = {128 * 2, (uint64_t)Hq * 128 * 2};
      const uint32_t b[3] = {64, 1, mimo::kBtQ};
      if ((st = make_map(&tdo, dout, 3, d, st2, b))) return st;
      const uint32_t b128[3] = {64, 1, mimo::kBdRows};
      if ((st = make_map(&tdo128, dout, 3, d, st2, b128))) return st;
    }
    {
      const uint64_t d[3] = {192, (uint64_t)Hkv, (uint64_t)total_tokens};
      const uint64_t st2[2] = {192 * 2, (uint64_t)Hkv * 192 * 2};
      const uint32_t b[3] = {64, 1, mimo::kBtKeys};
      if ((st = make_map(&tk, k, 3, d, st2, b))) return st;
    }
    {
      const uint64_t d[3] = {128, (uint64_t)Hkv, (uint64_t)total_tokens};
      const uint64_t st2[2] = {128 * 2, (uint64_t)Hkv * 128 * 2};
      const uint32_t b[3] = {64, 1, mimo::kBtKeys};
      if ((st = make_map(&tv, v, 3, d, st2, b))) return st;
    }
    static_assert(mimo::kBtKeys == mimo::kBdKeys, "the K / V maps serve both tcgen05 kernels");
    const int dq_tiles = (max_seqlen + mimo::kBdRows - 1) / mimo::kBdRows;
    mimo::bwd_dq_tc_kernel<<<dim3(dq_tiles, p.Hq, num_seqs), mimo::kBdThreads, mimo::kBdSmemBytes, s>>>(
        tq128, tk, tv, tdo128, p);
    if ((st = cuda_check(cudaGetLastError(), "backward dq launch"))) return st;
    const int ktiles = (max_seqlen + mimo::kBtKeys - 1) / mimo::kBtKeys;
    mimo::bwd_dkv_tc_kernel<<<dim3((unsigned)ktiles * Hkv, num_seqs), mimo::kBtThreads, mimo::kBtSmemBytes,
                              s>>>(tq, tk, tv, tdo, p);
    if ((st = cuda_check(cudaGetLastError(), "backward dk/dv launch"))) return st;
    return ok();
  }
  // fp32 out / dout: two warp-level passes (dV, then dK)
  const dim3 kv_grid((unsigned)tiles * p.Hkv, num_seqs);  // (key tile, KV head) per CTA
  mimo::bwd_dkv_kernel<true><<<kv_grid, mimo::kBkThreads, mimo::kBkSmemBytes, s>>>(p);
  if ((st = cuda_check(cudaGetLastError(), "backward dv launch"))) return st;
  mimo::bwd_dkv_kernel<false><<<kv_grid, mimo::kBkThreads, mimo::kBkSmemBytes, s>>>(p);
  if ((st = cuda_check(cudaGetLastError(), "backward dk launch"))) return st;
  return ok();
}

mimo_status_t mimo_attn_device_status(void* stream) {
  mimo_status_t st;
  if ((st = cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "stream synchronize"))) return st;
  int v = 0;
  if ((st = cuda_check(cudaMemcpyFromSymbol(&v, mimo::g_device_status, sizeof(int)), "read status")))
    return st;
  const int zero = 0;
  if ((st = cuda_check(cudaMemcpyToSymbol(mimo::g_device_status, &zero, sizeof(int)), "clear status")))
    return st;
  if (v == 0) return ok();
  return fail(static_cast<mimo_status_t>(v), "device status %d recorded by a kernel", v);
}

int mimo_attn_is_checked_build(void) {
#ifdef MIMO_CHECKED
  return 1;
#else
  return 0;
#endif
}

int mimo_attn_checked_site(void* stream) {
  int v = 0;
  const int zero = 0;
  if (cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "stream synchronize") ||
      cuda_check(cudaMemcpyFromSymbol(&v, mimo::g_checked_site, sizeof(int)), "read checked site") ||
      cuda_check(cudaMemcpyToSymbol(mimo::g_checked_site, &zero, sizeof(int)), "clear checked site"))
    return -1;
  return v;
}

mimo_status_t mimo_attn_wait_selftest(void* stream) {
  mimo::wait_selftest_kernel<<<1, 64, 0, (cudaStream_t)stream>>>();
  mimo_status_t st;
  if ((st = cuda_check(cudaGetLastError(), "wait self-test launch"))) return st;
  return ok();
}

mimo_status_t mimo_attn_checked_selftest(void* stream) {
#ifdef MIMO_CHECKED
  mimo::checked_selftest_kernel<<<1, 1, 0, (cudaStream_t)stream>>>();
  mimo_status_t st;
  if ((st = cuda_check(cudaGetLastError(), "checked self-test launch"))) return st;
  return ok();
#else
  (void)stream;
  return fail(MIMO_ERR_UNSUPPORTED, "not the checked build");
#endif
}

mimo_status_t mimo_attn_set_device_status(int code, void* stream) {
  if (code < MIMO_OK || code > MIMO_ERR_TIMEOUT)
    return fail(MIMO_ERR_INVALID_ARG, "status code %d is not a mimo_status_t", code);
  // pageable source: the value is captured before the call returns
  mimo_status_t st;
  if ((st = cuda_check(cudaMemcpyToSymbolAsync(mimo::g_device_status, &code, sizeof(int), 0,
                                               cudaMemcpyHostToDevice, (cudaStream_t)stream),
                       "write status")))
    return st;
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without allocation.
//
// Some callers cannot call cudaMalloc: code that runs inside a host process
// whose device memory belongs to another allocator (a serving runtime or a
// framework's memory pool that forbids raw allocations), and latency-critical
// loops that cannot afford the implicit device synchronisation cudaMalloc and
// cudaFree may bring.  For them the split-KV partial results live in this
// file-scope device array instead of a caller-provided workspace.  Every GPU
// that loads the library reserves it until the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
}  // namespace

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_decode_scratch on the current device.  In host code the
// array's name is only a host-side stand-in; the real address is looked up once
// per device, with that device current, and cached.
void* noalloc_scratch(mimo_status_t* st) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = fail(MIMO_ERR_CUDA, "cudaGetDevice failed");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      *st = fail(MIMO_ERR_CUDA, "cudaGetSymbolAddress(decode scratch): %s", cudaGetErrorString(e));
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" mimo_status_t mimo_attn_decode_noalloc(const mimo_attn_dims_t* dims, const void* q,
                                                  const void* k_cache, const void* v_cache,
                                                  const int32_t* seqlens, int batch, int capacity,
                                                  int window, const float* sinks, void* out,
                                                  float* lse, void* stream) {
  NvtxRange nvtx_range("mimo_attn_decode_noalloc");
  mimo_status_t st = check_dims(dims);
  if (st) return st;
  const size_t need = mimo_attn_decode_workspace_size(dims, batch, capacity, window);
  if (need > kNoAllocScratchBytes)
    return fail(MIMO_ERR_WORKSPACE,
                "decode needs %zu bytes of scratch but the built-in scratch holds %zu; use fewer "
                "sequences or a smaller capacity, or mimo_attn_decode with a workspace",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (need > 0 && !(scratch = noalloc_scratch(&st))) return st;
  // The split kernel writes every partial the combine kernel reads, so nothing
  // in the scratch has to start at zero.
  return mimo_attn_decode(dims, q, k_cache, v_cache, seqlens, batch, capacity, window, sinks, out,
                          lse, scratch, need > 0 ? kNoAllocScratchBytes : 0, stream);
}
