// C ABI of libpa.so: argument validation, launch configuration and the
// device-status word.  All kernels live in this one translation unit (the
// status word is a plain __device__ variable, no relocatable device code).
// The host allocator is in pa_alloc.cpp.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/pa.h"
#include "pa_cache.cuh"
#include "pa_common.cuh"
#include "pa_decode.cuh"
#include "pa_prefill.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxBatch = 8192;  // decode: one int per sequence of shared memory per CTA

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int smem_optin = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Measured on B200 (LLaMA-7B batch-64 decode): 8 warps x 2 pages in flight
// (128 KiB per SM) beat 3+ stages by ~10%; deeper rings only add contention.
struct Tuning {
  int warps = 0;  // 0: by group size (default_warps)
  int stages = 2;
  int ctas_per_sm = 1;
};
Tuning g_tuning;

// Measured on B200: one kv head per warp streams best with 8 warps x 2
// pages in flight; grouped heads (G = 2, 4) do more math per page and need
// 12 warps to hide it (+15% on the GQA workload); G = 8 is capped at 8 by
// registers.
// An FP8 cache doubles the dequantization and math per byte and takes 16
// warps up to G = 4 (at G = 1 the scalar page math in 126 registers, at
// G = 2 and 4 the tensor-core page math with the query in shared memory);
// G = 8 keeps 8.
int default_warps(int G, bool fp8 = false) { return (fp8 && G <= 4) ? 16 : (G == 2 || G == 4 || fp8) ? 12 : 8; }

// Cache elements per 16-byte vector (dims per lane) of a cache dtype.
int epv_of(int32_t kv_dtype) { return kv_dtype == PA_F32 ? 4 : kv_dtype == PA_FP8_E4M3 ? 16 : 8; }

int warps_for(int G, int32_t kv_dtype) {
  const int w = g_tuning.warps ? g_tuning.warps : default_warps(G, kv_dtype == PA_FP8_E4M3);
  const int cap = pa::max_warps_for(G, epv_of(kv_dtype));
  return w < cap ? w : cap;
}

pa_status device_info(DeviceInfo* out, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return PA_ERR_CUDA;
    d.ready = true;
  }
  *out = d;
  if (dev_out) *dev_out = dev;
  return PA_OK;
}

inline cudaStream_t stream_of(const pa_opts* o) {
  return o ? reinterpret_cast<cudaStream_t>(o->stream) : nullptr;
}

inline uint64_t timeout_of(const pa_opts* o) {
  const int ms = (o && o->timeout_ms > 0) ? o->timeout_ms : 1000;
  return uint64_t(ms) * 1000000ull;
}

inline int esize(int32_t dt) {
  return dt == PA_F32 ? 4 : dt == PA_BF16 ? 2 : dt == PA_I32 ? 4 : dt == PA_I64 ? 8 : dt == PA_FP8_E4M3 ? 1 : 0;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The cache: [NB, Hkv, 16, D] contiguous, 16-byte aligned.
pa_status check_cache(const pa_tensor* t) {
  if (t == nullptr || t->ndim != 4 || (t->dtype != PA_F32 && t->dtype != PA_BF16 && t->dtype != PA_FP8_E4M3))
    return PA_ERR_INVALID_ARG;
  const int64_t* s = t->shape;
  if (s[0] <= 0 || s[1] <= 0 || s[2] <= 0 || s[3] <= 0) return PA_ERR_INVALID_ARG;
  if (t->stride[3] != 1 || t->stride[2] != s[3] || t->stride[1] != s[2] * s[3] || t->stride[0] != s[1] * s[2] * s[3])
    return PA_ERR_INVALID_ARG;
  if (t->data == nullptr || !aligned16(t->data)) return PA_ERR_INVALID_ARG;
  if (s[2] != 16) return PA_ERR_UNSUPPORTED;
  if (s[3] != 64 && s[3] != 128) return PA_ERR_UNSUPPORTED;
  if (t->dtype == PA_FP8_E4M3 && s[3] != 128) return PA_ERR_UNSUPPORTED;
  if (s[0] > INT32_MAX || s[1] > 1024) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

pa_status check_pair(const pa_tensor* k, const pa_tensor* v) {
  pa_status st = check_cache(k);
  if (st != PA_OK) return st;
  st = check_cache(v);
  if (st != PA_OK) return st;
  if (k->dtype != v->dtype) return PA_ERR_INVALID_ARG;
  for (int d = 0; d < 4; ++d)
    if (k->shape[d] != v->shape[d]) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

// [n0, n1, D] rows: last dim contiguous, other strides multiples of 16 bytes.
// An empty tensor (n0 or n1 zero) is never read or written, so its strides
// and pointer are not checked (frameworks give empty tensors any strides).
pa_status check_rows3(const pa_tensor* t, int32_t dtype, int64_t n0, int64_t n1, int64_t D) {
  if (t == nullptr || t->ndim != 3 || t->dtype != dtype) return PA_ERR_INVALID_ARG;
  if (t->shape[0] != n0 || t->shape[1] != n1 || t->shape[2] != D) return PA_ERR_INVALID_ARG;
  if (n0 == 0 || n1 == 0) return PA_OK;
  if (t->stride[2] != 1) return PA_ERR_INVALID_ARG;
  const int e = esize(dtype);
  if (t->stride[0] < 0 || t->stride[1] < 0 || (t->stride[0] * e) % 16 || (t->stride[1] * e) % 16)
    return PA_ERR_INVALID_ARG;
  if (n0 > 0 && (t->data == nullptr || !aligned16(t->data))) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

// Per-kv-head FP8 scales: [Hkv] fp32, contiguous, every value finite and > 0
// (the values are not checked on the host: they live on the device).
pa_status check_scale(const pa_tensor* t, int64_t Hkv) {
  if (t == nullptr || t->ndim != 1 || t->dtype != PA_F32 || t->shape[0] != Hkv || t->data == nullptr)
    return PA_ERR_INVALID_ARG;
  if (Hkv > 1 && t->stride[0] != 1) return PA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t->data) & 3u) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

pa_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Raise a kernel's dynamic shared-memory limit on the current device to at
// least `bytes` (limit[dev] remembers what was set).  The limit only grows and
// the check-and-set is serialised, so host threads launching the same kernel
// cannot lower it under one another.  False if the runtime refused.
std::mutex g_attr_mu;

template <typename Kern>
bool raise_smem_limit(Kern kern, size_t bytes, int dev, std::atomic<size_t>* limit) {
  if (limit[dev].load(std::memory_order_acquire) >= bytes) return true;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (limit[dev].load(std::memory_order_relaxed) >= bytes) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  limit[dev].store(bytes, std::memory_order_release);
  return true;
}

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---------------------------------------------------------------------------
// decode launch plumbing
// ---------------------------------------------------------------------------
struct DecodePlan {
  int mode;
  int grid;
  int warps;
  int stages;
  size_t smem;
  int part_pages;
  int P_max;
  size_t ws_need;
};

// Shared-memory bytes of a decode launch: the row-sequence prefix (U row
// sequences, X extra ints) and one ring per warp, with the deepest ring (at
// most `want` stages) that fits.
template <typename Tkv, typename Tq, int D, int G>
size_t stage_fit(int U, int X, int warps, int want, int optin, int* stages_out) {
  using C = pa::DecodeCfg<Tkv, Tq, D, G>;
  for (int st = want; st >= 1; --st) {
    const size_t bytes = pa::decode_prefix_bytes(U, X) + size_t(warps) * C::warp_bytes(st);
    if (bytes <= size_t(optin)) {
      *stages_out = st;
      return bytes;
    }
  }
  return 0;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Every decode workspace starts with the same header: one 32-bit merge
// counter per worker of the balanced split (PA_DECODE_WS_HEADER_BYTES,
// enough for kMaxWorkers).  Every mode leaves it alone or leaves it zero, so
// one zero-filled workspace serves every mode and launch shape in turn.
constexpr size_t kWsHeader = PA_DECODE_WS_HEADER_BYTES;
constexpr int64_t kMaxWorkers = int64_t(PA_DECODE_WS_HEADER_BYTES / 4);

// Fixed mode, after the header: the documented per-partition partials
// (o, then lse); the shares of partitions cut between workers follow.
size_t fixed_partials_bytes(int64_t B, int64_t H, int64_t D, int64_t P) {
  return align_up(size_t(B * H * P * D) * 4, 256) + align_up(size_t(B * H * P) * 4, 256);
}

// Shares of units cut between workers: per worker two slots ([G][D]
// outputs + [G] lse): one for a cut unit its range begins in, one for a cut
// unit it ends in.
size_t shares_bytes(int64_t workers, int64_t G, int64_t D) {
  return align_up(size_t(2 * workers * G * D) * 4, 256) + align_up(size_t(2 * workers * G) * 4, 256);
}

size_t fixed_ws_bytes(int64_t B, int64_t H, int64_t D, int64_t P, int64_t workers, int64_t G) {
  return kWsHeader + fixed_partials_bytes(B, H, D, P) + shares_bytes(workers, G, D);
}

size_t balanced_ws_bytes(int64_t workers, int64_t G, int64_t D) { return kWsHeader + shares_bytes(workers, G, D); }

template <typename Tkv, typename Tq, int D, int G, int CK>
pa_status run_decode(const pa::DecodeArgs& base, const DecodePlan& p, cudaStream_t st, int dev) {
  static std::atomic<size_t> smem_limit[kMaxDevices];
  auto kern = pa::decode_kernel<Tkv, Tq, D, G, CK>;
  if (!raise_smem_limit(kern, p.smem, dev, smem_limit)) return PA_ERR_CUDA;
  pa::DecodeArgs a = base;
  a.stages = p.stages;
  a.mode = p.mode;
  a.part_pages = p.part_pages;
  a.P_max = p.P_max;
  if (launch_pdl(kern, dim3(p.grid), dim3(p.warps * 32), p.smem, st, true, a) != cudaSuccess) return launch_status();
  if (p.mode == pa::kFixed) {
    const int64_t rows = int64_t(a.B) * a.H;  // one CTA per (sequence, query head)
    if (launch_pdl(pa::merge_fixed_kernel<Tq, D>, dim3(unsigned(rows)), dim3(pa::kMergeWarps * 32), 0, st, true, a,
                   p.part_pages * pa::kBS) != cudaSuccess)
      return launch_status();
  }
  return launch_status();
}

template <typename Tkv, typename Tq, int D, int CK>
pa_status dispatch_group(int G, const pa::DecodeArgs& a, const DecodePlan& p, cudaStream_t st, int dev) {
  switch (G) {
    case 1:
      return run_decode<Tkv, Tq, D, 1, CK>(a, p, st, dev);
    case 2:
      return run_decode<Tkv, Tq, D, 2, CK>(a, p, st, dev);
    case 4:
      return run_decode<Tkv, Tq, D, 4, CK>(a, p, st, dev);
    case 8:
      return run_decode<Tkv, Tq, D, 8, CK>(a, p, st, dev);
    default:
      return PA_ERR_UNSUPPORTED;
  }
}

template <typename Tkv, typename Tq, int D>
size_t fit_for_group(int G, int U, int X, int warps, int want, int optin, int* stages) {
  switch (G) {
    case 1:
      return stage_fit<Tkv, Tq, D, 1>(U, X, warps, want, optin, stages);
    case 2:
      return stage_fit<Tkv, Tq, D, 2>(U, X, warps, want, optin, stages);
    case 4:
      return stage_fit<Tkv, Tq, D, 4>(U, X, warps, want, optin, stages);
    case 8:
      return stage_fit<Tkv, Tq, D, 8>(U, X, warps, want, optin, stages);
    default:
      return 0;
  }
}

// The (cache type, query/output type, head size) combinations built.
size_t fit_stages(int32_t kv_dtype, int D, int G, int U, int X, int warps, int want, int optin, int* stages) {
  if (kv_dtype == PA_BF16 && D == 128)
    return fit_for_group<__nv_bfloat16, __nv_bfloat16, 128>(G, U, X, warps, want, optin, stages);
  if (kv_dtype == PA_BF16 && D == 64)
    return fit_for_group<__nv_bfloat16, __nv_bfloat16, 64>(G, U, X, warps, want, optin, stages);
  if (kv_dtype == PA_F32 && D == 64) return fit_for_group<float, float, 64>(G, U, X, warps, want, optin, stages);
  if (kv_dtype == PA_F32 && D == 128) return fit_for_group<float, float, 128>(G, U, X, warps, want, optin, stages);
  if (kv_dtype == PA_FP8_E4M3 && D == 128)
    return fit_for_group<__nv_fp8_e4m3, __nv_bfloat16, 128>(G, U, X, warps, want, optin, stages);
  return 0;
}

// Mode, grid and smem of one decode launch whose rows carry G query rows
// each, over U row sequences (X extra prefix ints); ws_need = the workspace
// bytes its split uses (header included).  Shares of a balanced split need
// share_room bytes after the header.
pa_status plan_decode(int32_t dtype, int G, int64_t U, int64_t X, int64_t B, int64_t H, int64_t D, int64_t max_nb,
                      int32_t part_tokens, size_t share_room, bool ws_given, DecodePlan* p) {
  DeviceInfo di;
  int dev = 0;
  pa_status s = device_info(&di, &dev);
  if (s != PA_OK) return s;
  p->warps = warps_for(G, dtype);
  p->grid = di.sms * g_tuning.ctas_per_sm;
  p->smem = fit_stages(dtype, int(D), G, int(U), int(X), p->warps, g_tuning.stages, di.smem_optin, &p->stages);
  if (p->smem == 0) return PA_ERR_UNSUPPORTED;
  p->part_pages = 0;
  p->P_max = 0;
  p->ws_need = 0;
  const int64_t nworkers = int64_t(p->grid) * p->warps;
  if (part_tokens > 0) {
    if (part_tokens % pa::kBS) return PA_ERR_INVALID_ARG;
    p->mode = pa::kFixed;
    p->part_pages = part_tokens / pa::kBS;
    p->P_max = int((max_nb + p->part_pages - 1) / p->part_pages);
    if (p->P_max < 1) p->P_max = 1;
    if (nworkers > kMaxWorkers) return PA_ERR_UNSUPPORTED;
    p->ws_need = fixed_ws_bytes(B, H, D, p->P_max, nworkers, G);
  } else if (part_tokens == 0) {
    const size_t need = shares_bytes(nworkers, G, D);
    if (ws_given && share_room >= need && nworkers <= kMaxWorkers) {
      p->mode = pa::kBalanced;
      p->ws_need = kWsHeader + need;
    } else {
      p->mode = pa::kNoSplit;
    }
  } else if (part_tokens == -1) {
    p->mode = pa::kNoSplit;
  } else {
    return PA_ERR_INVALID_ARG;
  }
  return PA_OK;
}

// ---------------------------------------------------------------------------
// prefill launch plumbing: tensor maps for the tiled TMA loads
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims innermost first, strides in
// bytes for dims 1.. (each a multiple of 16), out-of-range elements read 0.
pa_status bf16_map(CUtensorMap* m, void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                   const cuuint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return PA_ERR_CUDA;
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), ptr, dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_INVALID_ARG;
}

template <int G>
pa_status run_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const pa::PrefillArgs& a,
                      int max_query_len, int Hkv, cudaStream_t st, int dev) {
  static std::atomic<size_t> smem_limit[kMaxDevices];
  auto kern = pa::prefill_kernel<G>;
  if (!raise_smem_limit(kern, size_t(pa::kPfSmemBytes), dev, smem_limit)) return PA_ERR_CUDA;
  constexpr int TOK = pa::kPfRows / G;  // new tokens per CTA
  const dim3 grid(unsigned((max_query_len + TOK - 1) / TOK), unsigned(Hkv), unsigned(a.B));
  if (launch_pdl(kern, grid, dim3(pa::kPfThreads), pa::kPfSmemBytes, st, true, tq, tk, tv, a) != cudaSuccess)
    return launch_status();
  return PA_OK;
}

}  // namespace

extern "C" {

int32_t pa_version(void) { return 1; }

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK:
      return "ok";
    case PA_ERR_INVALID_ARG:
      return "invalid argument";
    case PA_ERR_UNSUPPORTED:
      return "unsupported shape or dtype";
    case PA_ERR_OUT_OF_BLOCKS:
      return "out of free blocks";
    case PA_ERR_CUDA:
      return "CUDA runtime error";
    case PA_ERR_DEVICE_TIMEOUT:
      return "device wait timed out";
    case PA_ERR_DEVICE_BOUNDS:
      return "device index check failed";
    case PA_ERR_SCRATCH_LIMIT:
      return "needs more split scratch than the library's fixed no-alloc buffer holds";
    case PA_ERR_HOST_ALLOC:
      return "host memory allocation failed";
  }
  return "unknown status";
}

pa_status pa_set_decode_tuning(int32_t warps_per_cta, int32_t stages, int32_t ctas_per_sm) {
  if (warps_per_cta < 0 || warps_per_cta > pa::kMaxWarps || stages < 0 || stages > 16 || ctas_per_sm < 0 || ctas_per_sm > 8)
    return PA_ERR_INVALID_ARG;
  g_tuning.warps = warps_per_cta;
  g_tuning.stages = stages ? stages : 2;
  g_tuning.ctas_per_sm = ctas_per_sm ? ctas_per_sm : 1;
  return PA_OK;
}

pa_status pa_reshape_and_cache(const pa_tensor* key, const pa_tensor* value, pa_tensor* k_cache, pa_tensor* v_cache,
                               const pa_tensor* slot_mapping, const pa_opts* opts) {
  pa_status st = check_pair(k_cache, v_cache);
  if (st != PA_OK) return st;
  const int64_t NB = k_cache->shape[0], Hkv = k_cache->shape[1], D = k_cache->shape[3];
  if (slot_mapping == nullptr || slot_mapping->ndim != 1 || slot_mapping->dtype != PA_I64) return PA_ERR_INVALID_ARG;
  const int64_t T = slot_mapping->shape[0];
  if (T < 0 || (T > 0 && (slot_mapping->stride[0] != 1 || slot_mapping->data == nullptr))) return PA_ERR_INVALID_ARG;
  st = check_rows3(key, k_cache->dtype, T, Hkv, D);
  if (st != PA_OK) return st;
  st = check_rows3(value, k_cache->dtype, T, Hkv, D);
  if (st != PA_OK) return st;
  if (T == 0) return PA_OK;
  const int e = esize(k_cache->dtype);
  const int vpr = int(D * e / 16);
  const int64_t vec = 16 / e;  // elements per 16-byte vector
  const int64_t total = T * Hkv * vpr;
  DeviceInfo di;
  st = device_info(&di, nullptr);
  if (st != PA_OK) return st;
  const int64_t want = (total + 255) / 256;
  const int blocks = int(want < int64_t(di.sms) * 16 ? want : int64_t(di.sms) * 16);
  cudaStream_t s = stream_of(opts);
  const uint4* kp = static_cast<const uint4*>(key->data);
  const uint4* vp = static_cast<const uint4*>(value->data);
  uint4* kc = static_cast<uint4*>(k_cache->data);
  uint4* vc = static_cast<uint4*>(v_cache->data);
  const int64_t* sl = static_cast<const int64_t*>(slot_mapping->data);
  const int64_t ks0 = key->stride[0] / vec, ks1 = key->stride[1] / vec;
  const int64_t vs0 = value->stride[0] / vec, vs1 = value->stride[1] / vec;
  const int64_t nslots = NB * 16;
  cudaError_t err;
  switch (vpr) {
    case 8:
      err = launch_pdl(pa::reshape_and_cache_kernel<8>, dim3(blocks), dim3(256), 0, s, false, kp, vp, kc, vc, sl, T,
                       int(Hkv), ks0, ks1, vs0, vs1, nslots);
      break;
    case 16:
      err = launch_pdl(pa::reshape_and_cache_kernel<16>, dim3(blocks), dim3(256), 0, s, false, kp, vp, kc, vc, sl, T,
                       int(Hkv), ks0, ks1, vs0, vs1, nslots);
      break;
    case 32:
      err = launch_pdl(pa::reshape_and_cache_kernel<32>, dim3(blocks), dim3(256), 0, s, false, kp, vp, kc, vc, sl, T,
                       int(Hkv), ks0, ks1, vs0, vs1, nslots);
      break;
    default:
      return PA_ERR_UNSUPPORTED;
  }
  return err == cudaSuccess ? PA_OK : launch_status();
}

pa_status pa_reshape_and_cache_fp8(const pa_tensor* key, const pa_tensor* value, pa_tensor* k_cache,
                                   pa_tensor* v_cache, const pa_tensor* slot_mapping, const pa_tensor* k_scale,
                                   const pa_tensor* v_scale, const pa_opts* opts) {
  pa_status st = check_pair(k_cache, v_cache);
  if (st != PA_OK) return st;
  if (k_cache->dtype != PA_FP8_E4M3) return PA_ERR_INVALID_ARG;
  const int64_t NB = k_cache->shape[0], Hkv = k_cache->shape[1], D = k_cache->shape[3];
  if (slot_mapping == nullptr || slot_mapping->ndim != 1 || slot_mapping->dtype != PA_I64) return PA_ERR_INVALID_ARG;
  const int64_t T = slot_mapping->shape[0];
  if (T < 0 || (T > 0 && (slot_mapping->stride[0] != 1 || slot_mapping->data == nullptr))) return PA_ERR_INVALID_ARG;
  if (key == nullptr || (key->dtype != PA_BF16 && key->dtype != PA_F32)) return PA_ERR_INVALID_ARG;
  const int32_t in_dt = key->dtype;
  st = check_rows3(key, in_dt, T, Hkv, D);
  if (st != PA_OK) return st;
  st = check_rows3(value, in_dt, T, Hkv, D);
  if (st != PA_OK) return st;
  st = check_scale(k_scale, Hkv);
  if (st != PA_OK) return st;
  st = check_scale(v_scale, Hkv);
  if (st != PA_OK) return st;
  if (T == 0) return PA_OK;
  constexpr int OPR = 128 / 16;  // e4m3 codes of one 128-element row: 8 vectors
  const int64_t total = T * Hkv * OPR;
  DeviceInfo di;
  st = device_info(&di, nullptr);
  if (st != PA_OK) return st;
  const int64_t want = (total + 255) / 256;
  const int blocks = int(want < int64_t(di.sms) * 16 ? want : int64_t(di.sms) * 16);
  cudaStream_t s = stream_of(opts);
  uint4* kc = static_cast<uint4*>(k_cache->data);
  uint4* vc = static_cast<uint4*>(v_cache->data);
  const int64_t* sl = static_cast<const int64_t*>(slot_mapping->data);
  const float* ks = static_cast<const float*>(k_scale->data);
  const float* vs = static_cast<const float*>(v_scale->data);
  cudaError_t err;
  if (in_dt == PA_BF16) {
    err = launch_pdl(pa::reshape_and_cache_fp8_kernel<__nv_bfloat16, OPR>, dim3(blocks), dim3(256), 0, s, false,
                     static_cast<const __nv_bfloat16*>(key->data), static_cast<const __nv_bfloat16*>(value->data),
                     kc, vc, sl, T, int(Hkv), key->stride[0], key->stride[1], value->stride[0], value->stride[1],
                     NB * 16, ks, vs);
  } else {
    err = launch_pdl(pa::reshape_and_cache_fp8_kernel<float, OPR>, dim3(blocks), dim3(256), 0, s, false,
                     static_cast<const float*>(key->data), static_cast<const float*>(value->data), kc, vc, sl, T,
                     int(Hkv), key->stride[0], key->stride[1], value->stride[0], value->stride[1], NB * 16, ks, vs);
  }
  return err == cudaSuccess ? PA_OK : launch_status();
}

pa_status pa_copy_blocks(pa_tensor* k_cache, pa_tensor* v_cache, const pa_tensor* pairs, const pa_opts* opts) {
  pa_status st = check_pair(k_cache, v_cache);
  if (st != PA_OK) return st;
  if (pairs == nullptr || pairs->ndim != 2 || pairs->dtype != PA_I64 || pairs->shape[1] != 2) return PA_ERR_INVALID_ARG;
  const int64_t n = pairs->shape[0];
  if (n < 0) return PA_ERR_INVALID_ARG;
  if (n == 0) return PA_OK;
  if (pairs->stride[1] != 1 || pairs->stride[0] != 2 || pairs->data == nullptr) return PA_ERR_INVALID_ARG;
  const int64_t NB = k_cache->shape[0];
  const int e = esize(k_cache->dtype);
  const int64_t block_vecs = k_cache->shape[1] * 16 * k_cache->shape[3] * e / 16;
  const int gx = int((block_vecs + 1023) / 1024);
  const int gy = int(n < 65535 ? n : 65535);
  const cudaError_t err = launch_pdl(pa::copy_blocks_kernel, dim3(gx, gy), dim3(256), 0, stream_of(opts), false,
                                     static_cast<uint4*>(k_cache->data), static_cast<uint4*>(v_cache->data),
                                     static_cast<const int64_t*>(pairs->data), n, block_vecs, NB);
  return err == cudaSuccess ? PA_OK : launch_status();
}

// Device address of one pool of a swap: device memory of the current device,
// or page-locked host memory the device can reach (else the kernel would
// fault on it).
static pa_status swap_pool_ptr(const pa_tensor* t, void** dptr) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, t->data) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (at.type == cudaMemoryTypeDevice && at.device == dev) {
    *dptr = t->data;
    return PA_OK;
  }
  if (at.type == cudaMemoryTypeHost && at.devicePointer != nullptr) {
    *dptr = at.devicePointer;
    return PA_OK;
  }
  return PA_ERR_INVALID_ARG;  // pageable host memory, managed memory or another device's memory
}

pa_status pa_swap_blocks(const pa_tensor* src_k, const pa_tensor* src_v, pa_tensor* dst_k, pa_tensor* dst_v,
                         const pa_tensor* pairs, const pa_opts* opts) {
  pa_status st = check_pair(src_k, src_v);
  if (st != PA_OK) return st;
  st = check_pair(dst_k, dst_v);
  if (st != PA_OK) return st;
  if (src_k->dtype != dst_k->dtype) return PA_ERR_INVALID_ARG;
  for (int d = 1; d < 4; ++d)
    if (src_k->shape[d] != dst_k->shape[d]) return PA_ERR_INVALID_ARG;
  if (pairs == nullptr || pairs->ndim != 2 || pairs->dtype != PA_I64 || pairs->shape[1] != 2) return PA_ERR_INVALID_ARG;
  const int64_t n = pairs->shape[0];
  if (n < 0) return PA_ERR_INVALID_ARG;
  if (n == 0) return PA_OK;
  if (pairs->stride[1] != 1 || pairs->stride[0] != 2 || pairs->data == nullptr) return PA_ERR_INVALID_ARG;
  void *sk, *sv, *dk, *dv, *pp;
  if ((st = swap_pool_ptr(src_k, &sk)) != PA_OK || (st = swap_pool_ptr(src_v, &sv)) != PA_OK ||
      (st = swap_pool_ptr(dst_k, &dk)) != PA_OK || (st = swap_pool_ptr(dst_v, &dv)) != PA_OK ||
      (st = swap_pool_ptr(pairs, &pp)) != PA_OK)
    return st;
  const int e = esize(src_k->dtype);
  const int64_t block_vecs = src_k->shape[1] * 16 * src_k->shape[3] * e / 16;
  const int gx = int((block_vecs + 1023) / 1024);
  const int gy = int(n < 65535 ? n : 65535);
  const cudaError_t err = launch_pdl(pa::swap_blocks_kernel, dim3(gx, gy), dim3(256), 0, stream_of(opts), false,
                                     static_cast<const uint4*>(sk), static_cast<const uint4*>(sv),
                                     static_cast<uint4*>(dk), static_cast<uint4*>(dv),
                                     static_cast<const int64_t*>(pp), n, block_vecs, src_k->shape[0],
                                     dst_k->shape[0]);
  return err == cudaSuccess ? PA_OK : launch_status();
}

pa_status pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_size,
                                    int32_t max_blocks_per_seq, int32_t partition_tokens, size_t* bytes_out) {
  if (bytes_out == nullptr || num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_size <= 0 ||
      max_blocks_per_seq < 0 || num_heads % num_kv_heads)
    return PA_ERR_INVALID_ARG;
  *bytes_out = 0;
  if (partition_tokens == -1) return PA_OK;
  if (partition_tokens < -1 || (partition_tokens > 0 && partition_tokens % pa::kBS)) return PA_ERR_INVALID_ARG;
  DeviceInfo di;
  pa_status st = device_info(&di, nullptr);
  if (st != PA_OK) return st;
  const int G = num_heads / num_kv_heads;
  // an upper bound over cache types (the warps per CTA differ by cache type)
  const int64_t workers = int64_t(di.sms) * g_tuning.ctas_per_sm *
                          (g_tuning.warps ? g_tuning.warps : std::max(default_warps(G, false), default_warps(G, true)));
  if (partition_tokens > 0) {
    const int64_t pp = partition_tokens / pa::kBS;
    int64_t P = (max_blocks_per_seq + pp - 1) / pp;
    if (P < 1) P = 1;
    *bytes_out = fixed_ws_bytes(num_seqs, num_heads, head_size, P, workers, G);
    return PA_OK;
  }
  *bytes_out = balanced_ws_bytes(workers, G, head_size);
  return PA_OK;
}

}  // extern "C"

namespace {

// What every decode entry point checks and passes on: sizes, layouts and the
// kernel arguments that do not depend on the launch plan.
struct DecodeCall {
  int64_t B, H, Hkv, D, G, max_nb;
  int32_t dt;
  pa::DecodeArgs a;
};

// k_scale/v_scale are null unless the cache is FP8.
static pa_status decode_prepare(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache,
                                const pa_tensor* v_cache, const pa_tensor* block_tables,
                                const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                                const pa_tensor* k_scale, const pa_tensor* v_scale, const pa_opts* opts,
                                DecodeCall* dc) {
  pa_status st = check_pair(k_cache, v_cache);
  if (st != PA_OK) return st;
  const int64_t NB = k_cache->shape[0], Hkv = k_cache->shape[1], D = k_cache->shape[3];
  const int32_t dt = k_cache->dtype;
  const int32_t qdt = dt == PA_FP8_E4M3 ? PA_BF16 : dt;  // query/output type
  if (num_kv_heads != Hkv) return PA_ERR_INVALID_ARG;
  if (query == nullptr || query->ndim != 3) return PA_ERR_INVALID_ARG;
  const int64_t B = query->shape[0], H = query->shape[1];
  if (B < 0 || H <= 0 || H % Hkv) return PA_ERR_INVALID_ARG;
  st = check_rows3(query, qdt, B, H, D);
  if (st != PA_OK) return st;
  st = check_rows3(out, qdt, B, H, D);
  if (st != PA_OK) return st;
  if (dt == PA_FP8_E4M3) {
    st = check_scale(k_scale, Hkv);
    if (st != PA_OK) return st;
    st = check_scale(v_scale, Hkv);
    if (st != PA_OK) return st;
  }
  if (block_tables == nullptr || block_tables->ndim != 2 || block_tables->dtype != PA_I32 ||
      block_tables->shape[0] != B || block_tables->shape[1] < 0)
    return PA_ERR_INVALID_ARG;
  const int64_t max_nb = block_tables->shape[1];
  if (B > 0 && max_nb > 0 && (block_tables->stride[1] != 1 || block_tables->stride[0] < max_nb ||
                              block_tables->data == nullptr))
    return PA_ERR_INVALID_ARG;
  if (context_lens == nullptr || context_lens->ndim != 1 || context_lens->dtype != PA_I32 ||
      context_lens->shape[0] != B || (B > 0 && (context_lens->stride[0] != 1 || context_lens->data == nullptr)))
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  const int64_t G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (B >= (int64_t(1) << 20) || B > kMaxBatch) return PA_ERR_UNSUPPORTED;
  if (B * Hkv * max_nb >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  if (max_nb * 16 > INT32_MAX) return PA_ERR_UNSUPPORTED;
  const int32_t part = opts ? opts->partition_tokens : 0;
  if (part < -1 || (part > 0 && part % pa::kBS)) return PA_ERR_INVALID_ARG;
  if (opts && opts->workspace != nullptr && (reinterpret_cast<uintptr_t>(opts->workspace) & 255u))
    return PA_ERR_INVALID_ARG;

  dc->B = B, dc->H = H, dc->Hkv = Hkv, dc->D = D, dc->G = G, dc->max_nb = max_nb, dc->dt = dt;
  pa::DecodeArgs& a = dc->a;
  std::memset(&a, 0, sizeof(a));
  a.out = out->data;
  a.q = query->data;
  a.kc = k_cache->data;
  a.vc = v_cache->data;
  a.bt = static_cast<const int32_t*>(block_tables->data);
  a.ctx = static_cast<const int32_t*>(context_lens->data);
  a.q_sb = query->stride[0];
  a.q_sh = query->stride[1];
  a.o_sb = out->stride[0];
  a.o_sh = out->stride[1];
  a.bt_stride = block_tables->stride[0];
  a.B = int32_t(B);
  a.H = int32_t(H);
  a.Hkv = int32_t(Hkv);
  a.max_nb = int32_t(max_nb);
  a.num_blocks = int32_t(NB);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = timeout_of(opts);
  if (dt == PA_FP8_E4M3) {
    a.k_scale = static_cast<const float*>(k_scale->data);
    a.v_scale = static_cast<const float*>(v_scale->data);
  }
  return PA_OK;
}

// Points a launch's counters (the header) and shares (at byte offset
// shares_off) into the workspace.
static void place_shares(pa::DecodeArgs* a, void* workspace, size_t shares_off, const DecodePlan& plan, int64_t G,
                         int64_t D) {
  const int64_t workers = int64_t(plan.grid) * plan.warps;
  char* w = static_cast<char*>(workspace);
  a->ws_cnt = reinterpret_cast<unsigned int*>(w);
  w += shares_off;
  a->sh_o = reinterpret_cast<float*>(w);
  a->sh_lse = reinterpret_cast<float*>(w + align_up(size_t(2 * workers * G * D) * 4, 256));
}

template <int CK>
static pa_status launch_kind(const DecodeCall& dc, int G, const pa::DecodeArgs& a, const DecodePlan& plan,
                             cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  const int32_t dt = dc.dt;
  const int64_t D = dc.D;
  if constexpr (CK == pa::kPlain) {
    if (dt == PA_BF16 && D == 128) return dispatch_group<__nv_bfloat16, __nv_bfloat16, 128, CK>(G, a, plan, s, dev);
    if (dt == PA_BF16 && D == 64) return dispatch_group<__nv_bfloat16, __nv_bfloat16, 64, CK>(G, a, plan, s, dev);
    if (dt == PA_F32 && D == 64) return dispatch_group<float, float, 64, CK>(G, a, plan, s, dev);
    if (dt == PA_F32 && D == 128) return dispatch_group<float, float, 128, CK>(G, a, plan, s, dev);
    if (dt == PA_FP8_E4M3 && D == 128)
      return dispatch_group<__nv_fp8_e4m3, __nv_bfloat16, 128, CK>(G, a, plan, s, dev);
  } else {
    // shared-prefix decode: bf16 head size 128 and fp32 head size 64
    if (dt == PA_BF16 && D == 128) return dispatch_group<__nv_bfloat16, __nv_bfloat16, 128, CK>(G, a, plan, s, dev);
    if (dt == PA_F32 && D == 64) return dispatch_group<float, float, 64, CK>(G, a, plan, s, dev);
  }
  return PA_ERR_UNSUPPORTED;
}

static pa_status decode_impl(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache,
                             const pa_tensor* v_cache, const pa_tensor* block_tables, const pa_tensor* context_lens,
                             float scale, int32_t num_kv_heads, const pa_tensor* k_scale, const pa_tensor* v_scale,
                             const pa_opts* opts) {
  DecodeCall dc;
  pa_status st = decode_prepare(out, query, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads,
                                k_scale, v_scale, opts, &dc);
  if (st != PA_OK) return st;
  if (dc.B == 0) return PA_OK;
  const int32_t part = opts ? opts->partition_tokens : 0;
  const bool ws_given = opts && opts->workspace != nullptr;
  const size_t ws_bytes = ws_given ? opts->workspace_bytes : 0;
  DecodePlan plan;
  st = plan_decode(dc.dt, int(dc.G), dc.B, 0, dc.B, dc.H, dc.D, dc.max_nb, part,
                   ws_bytes > kWsHeader ? ws_bytes - kWsHeader : 0, ws_given, &plan);
  if (st != PA_OK) return st;
  if (plan.mode != pa::kNoSplit && (!ws_given || ws_bytes < plan.ws_need)) return PA_ERR_INVALID_ARG;
  pa::DecodeArgs a = dc.a;
  if (plan.mode == pa::kFixed) {
    char* w = static_cast<char*>(opts->workspace) + kWsHeader;
    a.ws_o = reinterpret_cast<float*>(w);
    a.ws_lse = reinterpret_cast<float*>(w + align_up(size_t(dc.B * dc.H * plan.P_max * dc.D) * 4, 256));
    place_shares(&a, opts->workspace, kWsHeader + fixed_partials_bytes(dc.B, dc.H, dc.D, plan.P_max), plan, dc.G,
                 dc.D);
  } else if (plan.mode == pa::kBalanced) {
    place_shares(&a, opts->workspace, kWsHeader, plan, dc.G, dc.D);
  }
  return launch_kind<pa::kPlain>(dc, int(dc.G), a, plan, stream_of(opts));
}

// ---------------------------------------------------------------------------
// shared-prefix (cascade) decode
// ---------------------------------------------------------------------------
// Workspace: [header][shares of the group rows' launch] (the balanced split);
// none without a split.
static pa_status cascade_ws_bytes(int32_t dt, int64_t gp, int64_t D, size_t* out) {
  DeviceInfo di;
  pa_status st = device_info(&di, nullptr);
  if (st != PA_OK) return st;
  const int64_t workers = int64_t(di.sms) * g_tuning.ctas_per_sm * warps_for(int(gp), dt);
  *out = balanced_ws_bytes(workers, gp, D);
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache, const pa_tensor* v_cache,
                    const pa_tensor* block_tables, const pa_tensor* context_lens, float scale, int32_t num_kv_heads,
                    const pa_opts* opts) {
  if (k_cache != nullptr && k_cache->dtype == PA_FP8_E4M3) return PA_ERR_INVALID_ARG;  // needs scales
  return decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, nullptr, nullptr,
                     opts);
}

pa_status pa_decode_fp8(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache, const pa_tensor* v_cache,
                        const pa_tensor* block_tables, const pa_tensor* context_lens, float scale,
                        int32_t num_kv_heads, const pa_tensor* k_scale, const pa_tensor* v_scale,
                        const pa_opts* opts) {
  if (k_cache == nullptr || k_cache->dtype != PA_FP8_E4M3) return PA_ERR_INVALID_ARG;
  return decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, k_scale, v_scale,
                     opts);
}

}  // extern "C"

namespace {

// Checks the group tensors and the group width of a shared-prefix decode.
static pa_status cascade_groups(const pa_tensor* group_start, const pa_tensor* group_blocks, int64_t G,
                                int32_t max_group_size, int64_t* n_groups) {
  if (group_blocks == nullptr || group_blocks->ndim != 1 || group_blocks->dtype != PA_I32 ||
      group_start == nullptr || group_start->ndim != 1 || group_start->dtype != PA_I32)
    return PA_ERR_INVALID_ARG;
  const int64_t n = group_blocks->shape[0];
  if (n < 1 || n > kMaxBatch || group_start->shape[0] != n + 1) return PA_ERR_INVALID_ARG;
  if (group_start->stride[0] != 1 || group_blocks->stride[0] != 1 || group_start->data == nullptr ||
      group_blocks->data == nullptr)
    return PA_ERR_INVALID_ARG;
  if (max_group_size < 1) return PA_ERR_INVALID_ARG;
  const int64_t gp = G * max_group_size;
  if (gp != 1 && gp != 2 && gp != 4 && gp != 8) return PA_ERR_UNSUPPORTED;
  *n_groups = n;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode_cascade_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                            int32_t head_size, int32_t max_group_size, int32_t partition_tokens,
                                            size_t* bytes_out) {
  if (bytes_out == nullptr || num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_size <= 0 ||
      num_heads % num_kv_heads || max_group_size < 1)
    return PA_ERR_INVALID_ARG;
  if (partition_tokens != 0 && partition_tokens != -1) return PA_ERR_UNSUPPORTED;
  const int64_t G = num_heads / num_kv_heads;
  const int64_t gp = G * max_group_size;
  if (gp != 1 && gp != 2 && gp != 4 && gp != 8) return PA_ERR_UNSUPPORTED;
  *bytes_out = 0;
  if (partition_tokens == -1) return PA_OK;
  // an upper bound over the cache types built
  size_t a = 0, b = 0;
  pa_status st = cascade_ws_bytes(PA_BF16, gp, head_size, &a);
  if (st != PA_OK) return st;
  if ((st = cascade_ws_bytes(PA_F32, gp, head_size, &b)) != PA_OK) return st;
  *bytes_out = a > b ? a : b;
  return PA_OK;
}

pa_status pa_decode_cascade(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache,
                            const pa_tensor* v_cache, const pa_tensor* block_tables, const pa_tensor* context_lens,
                            const pa_tensor* group_start, const pa_tensor* group_blocks, int32_t max_group_size,
                            float scale, int32_t num_kv_heads, const pa_opts* opts) {
  if (k_cache != nullptr && k_cache->dtype == PA_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  DecodeCall dc;
  pa_status st = decode_prepare(out, query, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads,
                                nullptr, nullptr, opts, &dc);
  if (st != PA_OK) return st;
  if (!((dc.dt == PA_BF16 && dc.D == 128) || (dc.dt == PA_F32 && dc.D == 64))) return PA_ERR_UNSUPPORTED;
  int64_t n_groups = 0;
  if ((st = cascade_groups(group_start, group_blocks, dc.G, max_group_size, &n_groups)) != PA_OK) return st;
  const int32_t part = opts ? opts->partition_tokens : 0;
  if (part != 0 && part != -1) return PA_ERR_UNSUPPORTED;
  if (dc.B == 0) return PA_OK;
  const int64_t gp = dc.G * max_group_size;
  const bool ws_given = opts && opts->workspace != nullptr;
  const size_t ws_bytes = ws_given ? opts->workspace_bytes : 0;
  // one launch over the group rows; the row sequences are the groups, or
  // the sequences when the groups turn out malformed on the device
  const int64_t umax = n_groups > dc.B ? n_groups : dc.B;
  DecodePlan plan;
  st = plan_decode(dc.dt, int(gp), umax, umax, dc.B, dc.H, dc.D, dc.max_nb, part,
                   ws_bytes > kWsHeader ? ws_bytes - kWsHeader : 0, ws_given, &plan);
  if (st != PA_OK) return st;
  if (part == 0 && plan.mode != pa::kBalanced) return PA_ERR_INVALID_ARG;  // the workspace is too small
  pa::DecodeArgs a = dc.a;
  a.grp_start = static_cast<const int32_t*>(group_start->data);
  a.grp_blocks = static_cast<const int32_t*>(group_blocks->data);
  a.n_groups = int32_t(n_groups);
  a.grp_members = max_group_size;
  a.g_real = int32_t(dc.G);
  if (plan.mode == pa::kBalanced) place_shares(&a, opts->workspace, kWsHeader, plan, gp, dc.D);
  return launch_kind<pa::kGroup>(dc, int(gp), a, plan, stream_of(opts));
}

pa_status pa_prefill(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache, const pa_tensor* v_cache,
                     const pa_tensor* block_tables, const pa_tensor* context_lens, const pa_tensor* query_start,
                     int32_t max_query_len, float scale, int32_t num_kv_heads, const pa_opts* opts) {
  pa_status st = check_pair(k_cache, v_cache);
  if (st != PA_OK) return st;
  const int64_t NB = k_cache->shape[0], Hkv = k_cache->shape[1], D = k_cache->shape[3];
  if (k_cache->dtype != PA_BF16 || D != 128) return PA_ERR_UNSUPPORTED;
  if (num_kv_heads != Hkv) return PA_ERR_INVALID_ARG;
  if (query == nullptr || query->ndim != 3) return PA_ERR_INVALID_ARG;
  const int64_t T = query->shape[0], H = query->shape[1];
  if (T < 0 || H <= 0 || H % Hkv) return PA_ERR_INVALID_ARG;
  if ((st = check_rows3(query, PA_BF16, T, H, D)) != PA_OK) return st;
  if ((st = check_rows3(out, PA_BF16, T, H, D)) != PA_OK) return st;
  if (context_lens == nullptr || context_lens->ndim != 1 || context_lens->dtype != PA_I32) return PA_ERR_INVALID_ARG;
  const int64_t B = context_lens->shape[0];
  if (B < 0 || (B > 0 && (context_lens->stride[0] != 1 || context_lens->data == nullptr))) return PA_ERR_INVALID_ARG;
  if (query_start == nullptr || query_start->ndim != 1 || query_start->dtype != PA_I32 ||
      query_start->shape[0] != B + 1 || query_start->stride[0] != 1 || query_start->data == nullptr)
    return PA_ERR_INVALID_ARG;
  if (block_tables == nullptr || block_tables->ndim != 2 || block_tables->dtype != PA_I32 ||
      block_tables->shape[0] != B || block_tables->shape[1] < 0)
    return PA_ERR_INVALID_ARG;
  const int64_t max_nb = block_tables->shape[1];
  if (B > 0 && max_nb > 0 &&
      (block_tables->stride[1] != 1 || block_tables->stride[0] < max_nb || block_tables->data == nullptr))
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return PA_ERR_INVALID_ARG;
  if (max_query_len < 0 || (T > 0 && max_query_len == 0) || max_query_len > T) return PA_ERR_INVALID_ARG;
  const int64_t G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (B > 65535 || T >= (int64_t(1) << 31) || max_nb * 16 > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return PA_OK;

  DeviceInfo di;
  int dev = 0;
  if ((st = device_info(&di, &dev)) != PA_OK) return st;
  if (di.smem_optin < int(pa::kPfSmemBytes)) return PA_ERR_UNSUPPORTED;

  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T)};
    const cuuint64_t strides[2] = {cuuint64_t(query->stride[1]) * 2, cuuint64_t(query->stride[0]) * 2};
    const cuuint32_t box[3] = {64, cuuint32_t(G), cuuint32_t(128 / G)};
    if ((st = bf16_map(&tq, query->data, 3, dims, strides, box)) != PA_OK) return st;
  }
  {
    const cuuint64_t dims[4] = {cuuint64_t(D), 16, cuuint64_t(Hkv), cuuint64_t(NB)};
    const cuuint64_t strides[3] = {cuuint64_t(D) * 2, cuuint64_t(16 * D) * 2, cuuint64_t(Hkv * 16 * D) * 2};
    const cuuint32_t box[4] = {64, 16, 1, 1};
    if ((st = bf16_map(&tk, k_cache->data, 4, dims, strides, box)) != PA_OK) return st;
    if ((st = bf16_map(&tv, v_cache->data, 4, dims, strides, box)) != PA_OK) return st;
  }
  pa::PrefillArgs a;
  std::memset(&a, 0, sizeof(a));
  a.out = static_cast<__nv_bfloat16*>(out->data);
  a.o_st = out->stride[0];
  a.o_sh = out->stride[1];
  a.bt = static_cast<const int32_t*>(block_tables->data);
  a.bt_stride = block_tables->stride[0];
  a.ctx = static_cast<const int32_t*>(context_lens->data);
  a.query_start = static_cast<const int32_t*>(query_start->data);
  a.B = int32_t(B);
  a.T = int32_t(T);
  a.max_nb = int32_t(max_nb);
  a.num_blocks = int32_t(NB);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = timeout_of(opts);
  cudaStream_t s = stream_of(opts);
  switch (G) {
    case 1:
      return run_prefill<1>(tq, tk, tv, a, max_query_len, int(Hkv), s, dev);
    case 2:
      return run_prefill<2>(tq, tk, tv, a, max_query_len, int(Hkv), s, dev);
    case 4:
      return run_prefill<4>(tq, tk, tv, a, max_query_len, int(Hkv), s, dev);
    default:
      return run_prefill<8>(tq, tk, tv, a, max_query_len, int(Hkv), s, dev);
  }
}

pa_status pa_get_device_status(const pa_opts* opts, uint32_t* bits_out) {
  cudaStream_t s = stream_of(opts);
  unsigned int bits = 0;
  const unsigned int zero = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyFromSymbolAsync(&bits, pa::g_status, sizeof(bits), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(pa::g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  if (bits & PA_DEV_TIMEOUT) return PA_ERR_DEVICE_TIMEOUT;
  if (bits) return PA_ERR_DEVICE_BOUNDS;
  return PA_OK;
}

// ---------------------------------------------------------------------------
// pa_decode_no_alloc: pa_decode with its split scratch in a fixed device
// array of this library instead of a caller workspace.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

static __device__ __align__(256) unsigned char g_no_alloc_scratch[PA_NO_ALLOC_SCRATCH_BYTES];

// In host code g_no_alloc_scratch names a host-side stand-in, not device
// memory; the kernels must be given the address cudaGetSymbolAddress returns,
// looked up once per device with that device current.
void* g_no_alloc_ptr[kMaxDevices] = {};
std::mutex g_no_alloc_mu;

pa_status no_alloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_no_alloc_mu);
  if (g_no_alloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || p == nullptr) return PA_ERR_CUDA;
    g_no_alloc_ptr[dev] = p;
  }
  *out = g_no_alloc_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode_no_alloc(pa_tensor* out, const pa_tensor* query, const pa_tensor* k_cache,
                             const pa_tensor* v_cache, const pa_tensor* block_tables, const pa_tensor* context_lens,
                             float scale, int32_t num_kv_heads, const pa_opts* opts) {
  if (query == nullptr || query->ndim != 3 || k_cache == nullptr || k_cache->ndim != 4 || block_tables == nullptr ||
      block_tables->ndim != 2)
    return PA_ERR_INVALID_ARG;
  const int32_t part = opts ? opts->partition_tokens : 0;
  if (part < -1 || (part > 0 && part % pa::kBS)) return PA_ERR_INVALID_ARG;
  const int64_t B = query->shape[0], H = query->shape[1], D = query->shape[2];
  const int64_t max_nb = block_tables->shape[1];
  if (B < 0 || H <= 0 || num_kv_heads <= 0 || H % num_kv_heads || B > INT32_MAX || max_nb < 0 || max_nb > INT32_MAX ||
      D <= 0 || D > INT32_MAX || H > INT32_MAX)
    return PA_ERR_INVALID_ARG;
  // Fixed partitions need their whole layout; the auto mode, like pa_decode
  // given too small a workspace, falls back to no split by itself.
  if (part > 0 && B > 0) {
    size_t need = 0;
    const pa_status st = pa_decode_workspace_bytes(int32_t(B), int32_t(H), num_kv_heads, int32_t(D),
                                                   int32_t(max_nb), part, &need);
    if (st != PA_OK) return st;
    if (need > PA_NO_ALLOC_SCRATCH_BYTES) return PA_ERR_SCRATCH_LIMIT;
  }
  pa_opts o;
  std::memset(&o, 0, sizeof(o));
  if (opts) o = *opts;
  o.workspace = nullptr;
  o.workspace_bytes = 0;
  if (part != -1 && B > 0) {
    void* p = nullptr;
    const pa_status st = no_alloc_scratch(&p);
    if (st != PA_OK) return st;
    o.workspace = p;
    o.workspace_bytes = PA_NO_ALLOC_SCRATCH_BYTES;
  }
  return pa_decode(out, query, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, &o);
}

pa_status pa_debug_wait_selftest(const pa_opts* opts) {
  const uint64_t t = timeout_of(opts);
  pa::wait_selftest_kernel<<<1, 32, 0, stream_of(opts)>>>(t);
  return launch_status();
}

}  // extern "C"
