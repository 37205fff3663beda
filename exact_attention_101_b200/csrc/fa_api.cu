// fa_api.cu -- host side of the C ABI declared in include/fa_b200.h: argument
// validation, TMA tensor-map encoding, kernel-instance selection and launch.
//
// Every call validates its arguments on the host before any CUDA call is made, so an
// invalid request never reaches the GPU.  Buffers are then checked to be device (or
// managed) memory of the current device whose allocation covers the bytes the shape
// implies; only then are the three TMA descriptors encoded and one persistent kernel
// launched on the caller's stream.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <atomic>
#include <mutex>
#include <type_traits>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_b200.h"
#include "fa_bwd_kernel.cuh"
#include "fa_fwd_kernel.cuh"
#include "fa_fwd_pair.cuh"
#include "fa_quant.cuh"

namespace {

constexpr int kMaxDevices = 64;

using PFN_encodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
using PFN_pointerAttrs = CUresult (*)(unsigned int, CUpointer_attribute *, void **, CUdeviceptr);

struct DriverFns {
  PFN_encodeTiled encode = nullptr;
  PFN_pointerAttrs attrs = nullptr;
  bool ok = false;
};

const DriverFns &driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.encode = reinterpret_cast<PFN_encodeTiled>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuPointerGetAttributes", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.attrs = reinterpret_cast<PFN_pointerAttrs>(fn);
    fns.ok = fns.encode && fns.attrs;
  });
  return fns;
}

struct DeviceInfo {
  int sms = 0;
  int major = 0, minor = 0;
  int max_smem_optin = 0;
};

std::mutex g_dev_mu;
DeviceInfo g_dev_info[kMaxDevices];
bool g_dev_known[kMaxDevices] = {};

fa_status device_info(int dev, DeviceInfo *out) {
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev_known[dev]) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return FA_ERR_CUDA;
    g_dev_info[dev] = d;
    g_dev_known[dev] = true;
  }
  *out = g_dev_info[dev];
  return FA_OK;
}

// Device memory of device `dev` (or managed memory), and the allocation holding `p`
// extends at least `bytes` past it.  One driver query per buffer: memory type, managed
// flag, device and the allocation's address range together.  (A pointer the driver does
// not know gets zeroed attributes and is refused.)
bool buffer_ok(const void *p, size_t bytes, int dev) {
  CUpointer_attribute which[5] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE, CU_POINTER_ATTRIBUTE_IS_MANAGED,
                                  CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL,
                                  CU_POINTER_ATTRIBUTE_RANGE_START_ADDR,
                                  CU_POINTER_ATTRIBUTE_RANGE_SIZE};
  unsigned int type = 0;
  uint64_t managed = 0;  // written as a boolean of at most 4 bytes
  int ordinal = -1;
  CUdeviceptr start = 0;
  size_t size = 0;
  void *data[5] = {&type, &managed, &ordinal, &start, &size};
  if (driver_fns().attrs(5, which, data, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS)
    return false;
  const bool is_managed = (managed & 0xffffffffull) != 0;
  if (!is_managed && (type != CU_MEMORYTYPE_DEVICE || ordinal != dev)) return false;
  if (size == 0) return false;
  const uint64_t end = static_cast<uint64_t>(reinterpret_cast<uintptr_t>(p)) + bytes;
  return end <= static_cast<uint64_t>(start) + size;
}

// Tensor maps are pure functions of (address, shape, box, format): a call looks them up in
// a small per-thread cache before encoding one, so repeated calls on the same buffers skip
// the encoding.  The buffer checks above still run on every call.
struct TmapKey {
  const void *base;
  uint64_t d, rows, heads;
  uint32_t box_rows, kind;  // kind: 0 bf16 [heads, rows, d], 1 e4m3, 2 packed bf16, 3 fp32 dQ
  bool operator==(const TmapKey &o) const {
    return base == o.base && d == o.d && rows == o.rows && heads == o.heads &&
           box_rows == o.box_rows && kind == o.kind;
  }
};
struct TmapEntry {
  CUtensorMap map;
  TmapKey key;
  bool valid;
};
constexpr int kTmapCache = 32;
thread_local TmapEntry t_tmap_cache[kTmapCache];
thread_local unsigned t_tmap_next = 0;

template <class Encode>
bool cached_tmap(CUtensorMap *m, const TmapKey &key, Encode encode) {
  for (int i = 0; i < kTmapCache; ++i) {
    if (t_tmap_cache[i].valid && t_tmap_cache[i].key == key) {
      *m = t_tmap_cache[i].map;
      return true;
    }
  }
  if (!encode(m)) return false;
  TmapEntry &e = t_tmap_cache[t_tmap_next++ % kTmapCache];
  e.map = *m;
  e.key = key;
  e.valid = true;
  return true;
}

// 3-D tensor map over a [heads, rows, d] tensor, box = [1, box_rows, 128 bytes of d],
// 128-byte swizzle, out-of-bounds elements read as zero.
bool encode_tmap_now(CUtensorMap *m, const void *base, bool fp8, uint64_t d, uint64_t rows,
                     uint64_t heads, uint32_t box_rows) {
  const uint64_t eb = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {d, rows, heads};
  cuuint64_t strides[2] = {d * eb, rows * d * eb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = driver_fns().encode(
      m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
      const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap(CUtensorMap *m, const void *base, bool fp8, uint64_t d, uint64_t rows,
                 uint64_t heads, uint32_t box_rows) {
  const TmapKey key{base, d, rows, heads, box_rows, fp8 ? 1u : 0u};
  return cached_tmap(m, key, [&](CUtensorMap *out) {
    return encode_tmap_now(out, base, fp8, d, rows, heads, box_rows);
  });
}

// The next slot of the forward kernel's work counters (fa::g_fa_sched) on device `dev`,
// round-robin over the slots: launches in flight at the same time get different slots as
// long as fewer than SCHED_SLOTS of them are.  The slots start at zero (static device
// memory) and every launch leaves its slot at zero.
fa_status sched_slot(int dev, unsigned int **out) {
  static std::once_flag once[kMaxDevices];
  static unsigned int *base[kMaxDevices];
  static fa_status st[kMaxDevices];
  static std::atomic<uint32_t> cursor[kMaxDevices];
  std::call_once(once[dev], [&] {
    void *a = nullptr;
    st[dev] = cudaGetSymbolAddress(&a, fa::g_fa_sched) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    if (st[dev] != FA_OK) cudaGetLastError();
    base[dev] = static_cast<unsigned int *>(a);
  });
  if (st[dev] != FA_OK) return st[dev];
  *out = base[dev] + 2 * (cursor[dev].fetch_add(1u) % fa::SCHED_SLOTS);
  return FA_OK;
}

template <int D, bool CAUSAL, bool OUT_F32, bool FP8, bool VARLEN = false, bool DROPOUT = false>
fa_status launch(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                 const fa::FwdParams &params, int grid, int dev, cudaStream_t stream) {
  fa::FwdParams p = params;
  if (sched_slot(dev, &p.sched) != FA_OK) return FA_ERR_CUDA;
  using C = fa::TileCfg<D, FP8>;
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, OUT_F32, FP8, VARLEN, DROPOUT>;
  static std::once_flag attr_once[kMaxDevices];
  static fa_status attr_st[kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    attr_st[dev] = FA_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess) {
      attr_st[dev] = FA_ERR_CUDA;
      return;
    }
    // The warpgroups re-split the launch register pool with setmaxnreg; a build that
    // launches with fewer registers per thread than the split assumes would wait forever
    // in setmaxnreg.inc, so it is never launched.
    cudaFuncAttributes fa_attr;
    if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess) {
      attr_st[dev] = FA_ERR_CUDA;
      return;
    }
    if (fa_attr.numRegs * fa::NUM_THREADS < 256 * fa::SOFTMAX_REGS + 128 * fa::OTHER_REGS)
      attr_st[dev] = FA_ERR_UNSUPPORTED;
  });
  if (attr_st[dev] != FA_OK) return attr_st[dev];
  kern<<<grid, fa::NUM_THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// The bf16 forward without dropout runs on CTA pairs (fa_fwd_pair.cuh) at head dimension
// 256, and at 128 without the causal mask, unless the library is built with
// FA_NO_PAIR_KERNEL.  Under the causal mask at 128 the one-CTA kernel measured faster on
// B200 (GQA causal B4 Hq32 Hkv8 N8192: 1 205 against 1 167 TFLOP/s; long causal level), so
// that work stays there unless the library is built with FA_PAIR_CAUSAL.  At 256 the pair
// wins either way (long d256: 1 465 against 1 190, causal 1 409 against 1 168).
bool pair_path(int d, bool fp8, int drop_thr, bool causal) {
#ifdef FA_NO_PAIR_KERNEL
  (void)d; (void)fp8; (void)drop_thr; (void)causal;
  return false;
#else
#ifdef FA_PAIR_CAUSAL
  (void)causal;
  return (d == 128 || d == 256) && !fp8 && drop_thr == 0;
#else
  return (d == 256 || (d == 128 && !causal)) && !fp8 && drop_thr == 0;
#endif
#endif
}

// Query rows per work unit, and CTAs per unit, of the forward instance for (d, path).
int fwd_unit_rows(int d, bool pair) {
  return pair ? fa::pair::UNIT_ROWS : (d > 128 ? fa::BM : fa::UNIT_ROWS);
}

// Clusters of the pair kernel that fit on device `dev` at once (0 if none), asked once per
// device and instance.
template <int D, bool CAUSAL, bool OUT_F32>
fa_status pair_setup(int dev, int sms, int *clusters) {
  auto kern = fa::pair::fa_fwd_pair_kernel<D, CAUSAL, OUT_F32>;
  constexpr int SMEM = fa::pair::PCfg<D>::SMEM_BYTES;
  static std::once_flag once[kMaxDevices];
  static fa_status st[kMaxDevices];
  static int n[kMaxDevices];
  std::call_once(once[dev], [&] {
    st[dev] = FA_ERR_CUDA;
    n[dev] = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    cudaFuncAttributes fa_attr;
    if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    // setmaxnreg.inc would wait forever if the launch pool could not cover the split
    if (fa_attr.numRegs * fa::pair::NUM_THREADS <
        256 * fa::pair::SOFTMAX_REGS + 128 * fa::pair::OTHER_REGS) {
      st[dev] = FA_ERR_UNSUPPORTED;
      return;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sms / 2 * 2), 1, 1);
    cfg.blockDim = dim3(fa::pair::NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    n[dev] = c;
    st[dev] = FA_OK;
  });
  *clusters = n[dev];
  return st[dev];
}

template <int D, bool CAUSAL, bool OUT_F32>
fa_status launch_pair(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                      const fa::FwdParams &params, int clusters, int dev, cudaStream_t stream) {
  fa::FwdParams p = params;
  if (sched_slot(dev, &p.sched) != FA_OK) return FA_ERR_CUDA;
  const int n = p.num_units < clusters ? p.num_units : clusters;
  fa::pair::fa_fwd_pair_kernel<D, CAUSAL, OUT_F32>
      <<<2 * n, fa::pair::NUM_THREADS, fa::pair::PCfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool CAUSAL, bool OUT_F32>
fa_status run_pair(const void *q, const void *k, const void *v, int B, int Hq, int Hkv, int Nq,
                   int Nk, fa::FwdParams &p, const DeviceInfo &info, int dev, cudaStream_t stream,
                   bool *ran) {
  *ran = false;
  int clusters = 0;
  const fa_status st = pair_setup<D, CAUSAL, OUT_F32>(dev, info.sms, &clusters);
  if (st != FA_OK || clusters < 1) return FA_OK;  // not resident here: the one-CTA kernel runs
  CUtensorMap tq, tk, tv;
  if (!encode_tmap(&tq, q, false, D, Nq, static_cast<uint64_t>(B) * Hq, fa::pair::BM) ||
      !encode_tmap(&tk, k, false, D, Nk, static_cast<uint64_t>(B) * Hkv, 64) ||
      !encode_tmap(&tv, v, false, D, Nk, static_cast<uint64_t>(B) * Hkv, fa::pair::BN))
    return FA_ERR_INVALID_ARG;
  p.num_qb = (Nq + fa::pair::UNIT_ROWS - 1) / fa::pair::UNIT_ROWS;
  p.num_units = B * Hq * p.num_qb;
  *ran = true;
  return launch_pair<D, CAUSAL, OUT_F32>(tq, tk, tv, p, clusters, dev, stream);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Pure host-side checks; no CUDA call.  Returns FA_OK or the error to report.
fa_status check_args(const void *q, const void *k, const void *v, const void *o,
                     const float *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                     float scale, int causal, bool fp8, const float *dq, const float *dk,
                     const float *dv) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (fp8 && (!dq || !dk || !dv)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_INVALID_ARG;
  if (fp8 && ((reinterpret_cast<uintptr_t>(dq) | reinterpret_cast<uintptr_t>(dk) |
               reinterpret_cast<uintptr_t>(dv)) & 3u))
    return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  // Index ranges: work-unit and row counts must fit the kernel's 32-bit arithmetic.
  const int64_t bh = static_cast<int64_t>(B) * Hq;
  const int64_t unit_rows = d > 128 ? fa::BM : fa::UNIT_ROWS;
  const int64_t units = bh * ((static_cast<int64_t>(Nq) + unit_rows - 1) / unit_rows);
  if (bh > INT32_MAX || static_cast<int64_t>(B) * Hkv > INT32_MAX || units > INT32_MAX)
    return FA_ERR_INVALID_ARG;
  if (Nk > INT32_MAX - 2 * fa::BN || Nq > INT32_MAX - 2 * fa::UNIT_ROWS) return FA_ERR_INVALID_ARG;
  if (fp8 ? d != 128 : (d != 64 && d != 128 && d != 256)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Dropout threshold for probability p (the nearest multiple of 1/256), -1 if p is not in
// [0, 1).
int dropout_threshold(float p) {
  if (!(p >= 0.f) || !(p < 1.f)) return -1;
  const int thr = static_cast<int>(std::lrint(static_cast<double>(p) * 256.0));
  return thr > 255 ? 255 : thr;
}

fa_status fwd_common(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                     int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     bool out_f32, bool fp8, const float *dq, const float *dk, const float *dv,
                     cudaStream_t stream, int drop_thr = 0, uint64_t seed = 0,
                     uint64_t offset = 0) {
  fa_status st = check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, fp8, dq, dk, dv);
  if (st != FA_OK) return st;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  DeviceInfo info;
  st = device_info(dev, &info);
  if (st != FA_OK) return st;
  if (info.major != 10 || info.minor != 0) return FA_ERR_UNSUPPORTED;
  if (!driver_fns().ok) return FA_ERR_CUDA;

  const uint64_t eb = fp8 ? 1 : 2;
  const uint64_t q_bytes = static_cast<uint64_t>(B) * Hq * Nq * d * eb;
  const uint64_t kv_bytes = static_cast<uint64_t>(B) * Hkv * Nk * d * eb;
  const uint64_t o_bytes = static_cast<uint64_t>(B) * Hq * Nq * d * (out_f32 ? 4 : 2);
  const uint64_t lse_bytes = static_cast<uint64_t>(B) * Hq * Nq * 4;
  if (!buffer_ok(q, q_bytes, dev) || !buffer_ok(k, kv_bytes, dev) || !buffer_ok(v, kv_bytes, dev) ||
      !buffer_ok(o, o_bytes, dev) || !buffer_ok(lse, lse_bytes, dev))
    return FA_ERR_INVALID_ARG;
  if (fp8 && (!buffer_ok(dq, static_cast<size_t>(B) * Hq * 4, dev) ||
              !buffer_ok(dk, static_cast<size_t>(B) * Hkv * 4, dev) ||
              !buffer_ok(dv, static_cast<size_t>(B) * Hkv * 4, dev)))
    return FA_ERR_INVALID_ARG;

  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.descale_q = dq;
  p.descale_k = dk;
  p.descale_v = dv;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.seed = seed;
  p.offset = offset;
  p.drop_thr4 = static_cast<uint32_t>(drop_thr) * 0x01010101u;
  p.keep_scale = static_cast<float>(256.0 / (256.0 - drop_thr));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = Hq / Hkv;
  const int unit_rows = d > 128 ? fa::BM : fa::UNIT_ROWS;  // one Q tile per unit at d = 256
  p.num_qb = (Nq + unit_rows - 1) / unit_rows;
  p.num_units = B * Hq * p.num_qb;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);

  if (pair_path(d, fp8, drop_thr, causal)) {
    bool ran = false;
#ifdef FA_PAIR_CAUSAL
    auto run = [&](auto dd) {
      constexpr int DD = decltype(dd)::value;
      return causal ? (out_f32 ? run_pair<DD, true, true>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran)
                               : run_pair<DD, true, false>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran))
                    : (out_f32 ? run_pair<DD, false, true>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran)
                               : run_pair<DD, false, false>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran));
    };
#else
    // head dim 128: without the mask only; head dim 256: both
    auto run = [&](auto dd) {
      constexpr int DD = decltype(dd)::value;
      if (DD == 256 && causal)
        return out_f32 ? run_pair<256, true, true>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran)
                       : run_pair<256, true, false>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran);
      return out_f32 ? run_pair<DD, false, true>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran)
                     : run_pair<DD, false, false>(q, k, v, B, Hq, Hkv, Nq, Nk, p, info, dev, stream, &ran);
    };
#endif
    const fa_status ps = d == 128 ? run(std::integral_constant<int, 128>())
                                  : run(std::integral_constant<int, 256>());
    if (ran || ps != FA_OK) return ps;
    p.num_qb = (Nq + unit_rows - 1) / unit_rows;
    p.num_units = B * Hq * p.num_qb;
  }

  CUtensorMap tq, tk, tv;
  if (!encode_tmap(&tq, q, fp8, d, Nq, static_cast<uint64_t>(B) * Hq, fa::BM) ||
      !encode_tmap(&tk, k, fp8, d, Nk, static_cast<uint64_t>(B) * Hkv, fa::BN) ||
      !encode_tmap(&tv, v, fp8, d, Nk, static_cast<uint64_t>(B) * Hkv, fa::BN))
    return FA_ERR_INVALID_ARG;
  const int grid = p.num_units < info.sms ? p.num_units : info.sms;

  if (fp8) {
    if (causal) return launch<128, true, false, true>(tq, tk, tv, p, grid, dev, stream);
    return launch<128, false, false, true>(tq, tk, tv, p, grid, dev, stream);
  }
  if (drop_thr > 0) {
#define FA_DROP(DD)                                                                           \
  if (d == DD) {                                                                              \
    if (causal)                                                                               \
      return out_f32 ? launch<DD, true, true, false, false, true>(tq, tk, tv, p, grid, dev, stream) \
                     : launch<DD, true, false, false, false, true>(tq, tk, tv, p, grid, dev, stream); \
    return out_f32 ? launch<DD, false, true, false, false, true>(tq, tk, tv, p, grid, dev, stream) \
                   : launch<DD, false, false, false, false, true>(tq, tk, tv, p, grid, dev, stream); \
  }
    FA_DROP(64)
    FA_DROP(128)
    FA_DROP(256)
#undef FA_DROP
    return FA_ERR_UNSUPPORTED;
  }
  if (d == 64) {
    if (causal)
      return out_f32 ? launch<64, true, true, false>(tq, tk, tv, p, grid, dev, stream)
                     : launch<64, true, false, false>(tq, tk, tv, p, grid, dev, stream);
    return out_f32 ? launch<64, false, true, false>(tq, tk, tv, p, grid, dev, stream)
                   : launch<64, false, false, false>(tq, tk, tv, p, grid, dev, stream);
  }
  if (d == 256) {
    if (causal)
      return out_f32 ? launch<256, true, true, false>(tq, tk, tv, p, grid, dev, stream)
                     : launch<256, true, false, false>(tq, tk, tv, p, grid, dev, stream);
    return out_f32 ? launch<256, false, true, false>(tq, tk, tv, p, grid, dev, stream)
                   : launch<256, false, false, false>(tq, tk, tv, p, grid, dev, stream);
  }
  if (causal)
    return out_f32 ? launch<128, true, true, false>(tq, tk, tv, p, grid, dev, stream)
                   : launch<128, true, false, false>(tq, tk, tv, p, grid, dev, stream);
  return out_f32 ? launch<128, false, true, false>(tq, tk, tv, p, grid, dev, stream)
                 : launch<128, false, false, false>(tq, tk, tv, p, grid, dev, stream);
}

// 3-D tensor map over a packed [tokens, heads, d] bf16 tensor, box = [128 bytes of d,
// 1 head, box_rows tokens], 128-byte swizzle: the same shared-memory tile as encode_tmap.
bool encode_tmap_packed_now(CUtensorMap *m, const void *base, uint64_t d, uint64_t heads,
                            uint64_t tokens, uint32_t box_rows) {
  cuuint64_t dims[3] = {d, heads, tokens};
  cuuint64_t strides[2] = {d * 2, heads * d * 2};
  cuuint32_t box[3] = {64, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = driver_fns().encode(
      m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_packed(CUtensorMap *m, const void *base, uint64_t d, uint64_t heads,
                        uint64_t tokens, uint32_t box_rows) {
  const TmapKey key{base, d, tokens, heads, box_rows, 2u};
  return cached_tmap(m, key, [&](CUtensorMap *out) {
    return encode_tmap_packed_now(out, base, d, heads, tokens, box_rows);
  });
}

fa_status fwd_varlen_common(const void *q, const void *k, const void *v, void *o, float *lse,
                            const int *cu_q, const int *cu_k, int B, int Hq, int Hkv,
                            int total_q, int total_k, int max_q, int d, float scale,
                            int causal, fa_dtype dtype, cudaStream_t stream) {
  // Pure host checks first.
  if (!q || !k || !v || !o || !lse || !cu_q || !cu_k) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      ((reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(cu_q) |
        reinterpret_cast<uintptr_t>(cu_k)) & 3u))
    return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || total_q < 1 || total_k < 1 || max_q < 1 || d < 1)
    return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_BF16_OUT_F32) return FA_ERR_INVALID_ARG;
  const int64_t unit_rows = d > 128 ? fa::BM : fa::UNIT_ROWS;  // one Q tile per unit at d = 256
  const int64_t num_qb = (static_cast<int64_t>(max_q) + unit_rows - 1) / unit_rows;
  if (static_cast<int64_t>(B) * Hq * num_qb > INT32_MAX || max_q > INT32_MAX - 2 * fa::UNIT_ROWS ||
      total_k > INT32_MAX - 2 * fa::BN || total_q > INT32_MAX - 2 * fa::UNIT_ROWS)
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  DeviceInfo info;
  fa_status st = device_info(dev, &info);
  if (st != FA_OK) return st;
  if (info.major != 10 || info.minor != 0) return FA_ERR_UNSUPPORTED;
  if (!driver_fns().ok) return FA_ERR_CUDA;
  const bool out_f32 = dtype == FA_BF16_OUT_F32;
  const uint64_t q_bytes = static_cast<uint64_t>(total_q) * Hq * d * 2;
  const uint64_t kv_bytes = static_cast<uint64_t>(total_k) * Hkv * d * 2;
  const uint64_t o_bytes = static_cast<uint64_t>(total_q) * Hq * d * (out_f32 ? 4 : 2);
  if (!buffer_ok(q, q_bytes, dev) || !buffer_ok(k, kv_bytes, dev) || !buffer_ok(v, kv_bytes, dev) ||
      !buffer_ok(o, o_bytes, dev) || !buffer_ok(lse, static_cast<uint64_t>(total_q) * Hq * 4, dev) ||
      !buffer_ok(cu_q, static_cast<uint64_t>(B + 1) * 4, dev) ||
      !buffer_ok(cu_k, static_cast<uint64_t>(B + 1) * 4, dev))
    return FA_ERR_INVALID_ARG;

  CUtensorMap tq, tk, tv;
  if (!encode_tmap_packed(&tq, q, d, Hq, total_q, fa::BM) ||
      !encode_tmap_packed(&tk, k, d, Hkv, total_k, fa::BN) ||
      !encode_tmap_packed(&tv, v, d, Hkv, total_k, fa::BN))
    return FA_ERR_INVALID_ARG;

  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.descale_q = p.descale_k = p.descale_v = nullptr;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.seed = p.offset = 0;
  p.drop_thr4 = 0;
  p.keep_scale = 1.f;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = total_q;
  p.Nk = total_k;
  p.group = Hq / Hkv;
  p.num_qb = static_cast<int>(num_qb);
  p.num_units = static_cast<int>(B * Hq * num_qb);
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  const int grid = p.num_units < info.sms ? p.num_units : info.sms;
  if (d == 64) {
    if (causal)
      return out_f32 ? launch<64, true, true, false, true>(tq, tk, tv, p, grid, dev, stream)
                     : launch<64, true, false, false, true>(tq, tk, tv, p, grid, dev, stream);
    return out_f32 ? launch<64, false, true, false, true>(tq, tk, tv, p, grid, dev, stream)
                   : launch<64, false, false, false, true>(tq, tk, tv, p, grid, dev, stream);
  }
  if (d == 256) {
    if (causal)
      return out_f32 ? launch<256, true, true, false, true>(tq, tk, tv, p, grid, dev, stream)
                     : launch<256, true, false, false, true>(tq, tk, tv, p, grid, dev, stream);
    return out_f32 ? launch<256, false, true, false, true>(tq, tk, tv, p, grid, dev, stream)
                   : launch<256, false, false, false, true>(tq, tk, tv, p, grid, dev, stream);
  }
  if (causal)
    return out_f32 ? launch<128, true, true, false, true>(tq, tk, tv, p, grid, dev, stream)
                   : launch<128, true, false, false, true>(tq, tk, tv, p, grid, dev, stream);
  return out_f32 ? launch<128, false, true, false, true>(tq, tk, tv, p, grid, dev, stream)
                 : launch<128, false, false, false, true>(tq, tk, tv, p, grid, dev, stream);
}

// Shared-memory quantisation kernel: the smallest power-of-two cluster (<= 8 CTAs) that
// keeps a CTA at <= MAX_SMEM_ROWS rows.  Returns false if the slice is longer than that.
bool quant_smem_shape(int N, int *cs, int *cta_rows) {
  int c = 1;
  auto rows_for = [&](int cc) { return ((N + cc - 1) / cc + 7) / 8 * 8; };
  while (c < fa::quant::MAX_CLUSTER && rows_for(c) > fa::quant::MAX_SMEM_ROWS) c *= 2;
  *cs = c;
  *cta_rows = rows_for(c);
  return *cta_rows <= fa::quant::MAX_SMEM_ROWS;
}

// Whether a cluster of `cs` CTAs with `smem` bytes of dynamic shared memory each can be
// resident on this device (asked once per device, kernel and shape).
template <bool ROTATE>
bool quant_smem_fits(int dev, int cs, int smem, int grid) {
  static std::mutex mu;
  static std::map<long long, bool> known;
  auto kern = fa::quant::fa_quant_smem_kernel<ROTATE>;
  static std::once_flag attr_once[kMaxDevices];
  static bool attr_ok[kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    attr_ok[dev] =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::quant::MAX_SMEM_ROWS * fa::quant::ROW_BYTES) == cudaSuccess;
  });
  if (!attr_ok[dev]) {
    cudaGetLastError();
    return false;
  }
  const long long key = (static_cast<long long>(dev) << 40) | (static_cast<long long>(cs) << 32) | smem;
  std::lock_guard<std::mutex> lk(mu);
  auto it = known.find(key);
  if (it != known.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = cs;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(fa::quant::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  const bool ok =
      cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0;
  if (!ok) cudaGetLastError();
  known[key] = ok;
  return ok;
}

template <bool ROTATE>
fa_status quant_launch(fa::quant::QuantParams qp, long long slices, int dev,
                       cudaStream_t stream) {
  int cs = 1, cta_rows = 0;
  if (quant_smem_shape(qp.rows, &cs, &cta_rows)) {
    const long long grid = slices * cs;
    const int smem = cta_rows * fa::quant::ROW_BYTES;
    if (grid <= INT32_MAX && quant_smem_fits<ROTATE>(dev, cs, smem, static_cast<int>(grid))) {
      qp.cta_rows = cta_rows;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = cs;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
      cfg.blockDim = dim3(fa::quant::THREADS, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = stream;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, fa::quant::fa_quant_smem_kernel<ROTATE>, qp) != cudaSuccess)
        return FA_ERR_CUDA;
      return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
  }
  const long long grid = slices * fa::quant::CLUSTER;
  if (grid > INT32_MAX) return FA_ERR_INVALID_ARG;
  fa::quant::fa_quant_kernel<ROTATE>
      <<<static_cast<unsigned>(grid), fa::quant::THREADS, 0, stream>>>(qp);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status quantize_common(const void *x, const int8_t *signs, void *x8, float *descale, int B,
                          int H, int N, int d, cudaStream_t stream) {
  if (!x || !x8 || !descale) return FA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || (reinterpret_cast<uintptr_t>(descale) & 3u))
    return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (d != fa::quant::D) return FA_ERR_UNSUPPORTED;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  DeviceInfo info;
  fa_status st = device_info(dev, &info);
  if (st != FA_OK) return st;
  if (info.major != 10 || info.minor != 0) return FA_ERR_UNSUPPORTED;
  if (!driver_fns().ok) return FA_ERR_CUDA;

  const uint64_t slices = static_cast<uint64_t>(B) * H;
  const uint64_t elems = slices * N * d;
  if (!buffer_ok(x, elems * 2, dev) || !buffer_ok(x8, elems, dev) ||
      !buffer_ok(descale, slices * 4, dev) || (signs && !buffer_ok(signs, d, dev)))
    return FA_ERR_INVALID_ARG;

  fa::quant::QuantParams qp;
  qp.x = static_cast<const uint16_t *>(x);
  qp.signs = signs;
  qp.codes = static_cast<uint8_t *>(x8);
  qp.descale = descale;
  qp.rows = N;
  qp.cta_rows = 0;
  const long long s = static_cast<long long>(slices);
  if (signs) {
    qp.norm_over_max = static_cast<float>(1.0 / (448.0 * std::sqrt(static_cast<double>(d))));
    return quant_launch<true>(qp, s, dev, stream);
  }
  qp.norm_over_max = static_cast<float>(1.0 / 448.0);
  return quant_launch<false>(qp, s, dev, stream);
}

// 3-D tensor map over the fp32 dQ accumulator [heads, rows, d], box = [1, 64 rows, 32
// floats], no swizzle: the target of the backward kernel's bulk reduce-adds.
bool encode_tmap_dq(CUtensorMap *m, void *base, uint64_t d, uint64_t rows, uint64_t heads) {
  cuuint64_t dims[3] = {d, rows, heads};
  cuuint64_t strides[2] = {d * 4, rows * d * 4};
  cuuint32_t box[3] = {32, static_cast<cuuint32_t>(fa::bwd::BM), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = driver_fns().encode(
      m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool CAUSAL>
fa_status bwd_launch(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     const CUtensorMap &tdo, const CUtensorMap &tdq,
                     const fa::bwd::BwdParams &p, int grid, int dev, cudaStream_t stream) {
  auto kern = fa::bwd::fa_bwd_kernel<D, CAUSAL>;
  constexpr int smem_bytes = fa::bwd::BCfg<D>::SMEM_BYTES;
  static std::once_flag attr_once[kMaxDevices];
  static fa_status attr_st[kMaxDevices];
  std::call_once(attr_once[dev], [&] {
    attr_st[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        smem_bytes) == cudaSuccess
                       ? FA_OK
                       : FA_ERR_CUDA;
  });
  if (attr_st[dev] != FA_OK) return attr_st[dev];
  kern<<<grid, fa::bwd::NUM_THREADS, smem_bytes, stream>>>(tq, tk, tv, tdo, tdq, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Pure host-side checks of fa_bwd; no CUDA call.
fa_status check_bwd_args(const void *q, const void *k, const void *v, const void *o,
                         const void *dout, const float *lse, const void *dq, const void *dk,
                         const void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         float scale, int causal) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  const int64_t bh = static_cast<int64_t>(B) * Hq;
  const int64_t units = static_cast<int64_t>(B) * Hkv * ((static_cast<int64_t>(Nk) + fa::bwd::BN - 1) / fa::bwd::BN);
  if (bh > INT32_MAX || units > INT32_MAX || Nq > INT32_MAX - 2 * fa::bwd::BM ||
      Nk > INT32_MAX - 2 * fa::bwd::BN)
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Bytes of backward scratch: the fp32 dQ accumulator and two padded per-row vectors,
// each rounded up to 256 bytes.  *acc_used is the accumulator's own size (before the
// rounding): the bytes every call clears.
uint64_t bwd_scratch_bytes(int B, int Hq, int Nq, int d, uint64_t *acc_bytes, uint64_t *vec_bytes,
                           uint64_t *acc_used = nullptr) {
  const uint64_t npad = (static_cast<uint64_t>(Nq) + fa::bwd::BM - 1) / fa::bwd::BM * fa::bwd::BM;
  const uint64_t used = static_cast<uint64_t>(B) * Hq * Nq * d * 4;
  if (acc_used) *acc_used = used;
  *acc_bytes = (used + 255) / 256 * 256;
  *vec_bytes = (static_cast<uint64_t>(B) * Hq * npad * 4 + 255) / 256 * 256;
  return *acc_bytes + 2 * *vec_bytes;
}

// Stream-ordered memory pool of the backward's scratch, one per device, created on first
// use and kept for the life of the process.  Freed scratch stays in the pool up to
// kScratchKeepBytes across synchronisations, so repeated calls of similar size take it
// back without asking the driver for memory again (the device's default pool hands
// everything back at each synchronisation, and the next call then waits on the driver).
constexpr uint64_t kScratchKeepBytes = 4ull << 30;

fa_status scratch_pool(int dev, cudaMemPool_t *out) {
  static std::once_flag once[kMaxDevices];
  static cudaMemPool_t pool[kMaxDevices];
  static fa_status st[kMaxDevices];
  std::call_once(once[dev], [&] {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    uint64_t keep = kScratchKeepBytes;
    st[dev] = cudaMemPoolCreate(&pool[dev], &props) == cudaSuccess &&
                      cudaMemPoolSetAttribute(pool[dev], cudaMemPoolAttrReleaseThreshold,
                                              &keep) == cudaSuccess
                  ? FA_OK
                  : FA_ERR_CUDA;
    if (st[dev] != FA_OK) cudaGetLastError();
  });
  *out = pool[dev];
  return st[dev];
}

// fixed_ws == nullptr: scratch is taken from and returned to the library's pool on
// `stream` (stream-ordered); otherwise fixed_ws (large enough, checked by the caller) is
// used.
fa_status bwd_common(const void *q, const void *k, const void *v, const void *o,
                     const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                     int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     cudaStream_t stream, void *fixed_ws = nullptr) {
  fa_status st = check_bwd_args(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale,
                                causal);
  if (st != FA_OK) return st;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  DeviceInfo info;
  st = device_info(dev, &info);
  if (st != FA_OK) return st;
  if (info.major != 10 || info.minor != 0) return FA_ERR_UNSUPPORTED;
  if (!driver_fns().ok) return FA_ERR_CUDA;

  const uint64_t q_bytes = static_cast<uint64_t>(B) * Hq * Nq * d * 2;
  const uint64_t kv_bytes = static_cast<uint64_t>(B) * Hkv * Nk * d * 2;
  const uint64_t lse_bytes = static_cast<uint64_t>(B) * Hq * Nq * 4;
  if (!buffer_ok(q, q_bytes, dev) || !buffer_ok(k, kv_bytes, dev) || !buffer_ok(v, kv_bytes, dev) ||
      !buffer_ok(o, q_bytes, dev) || !buffer_ok(dout, q_bytes, dev) ||
      !buffer_ok(lse, lse_bytes, dev) || !buffer_ok(dq, q_bytes, dev) ||
      !buffer_ok(dk, kv_bytes, dev) || !buffer_ok(dv, kv_bytes, dev))
    return FA_ERR_INVALID_ARG;

  fa::bwd::BwdParams p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = Hq / Hkv;
  p.diag = Nk - Nq;
  p.num_qb = (Nq + fa::bwd::BM - 1) / fa::bwd::BM;
  p.Npad = p.num_qb * fa::bwd::BM;
  p.num_kb = (Nk + fa::bwd::BN - 1) / fa::bwd::BN;
  p.num_units = B * Hkv * p.num_kb;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
  p.dk = static_cast<uint16_t *>(dk);
  p.dv = static_cast<uint16_t *>(dv);

  CUtensorMap tq, tk, tv, tdo;
  if (!encode_tmap(&tq, q, false, d, Nq, static_cast<uint64_t>(B) * Hq, fa::bwd::BM) ||
      !encode_tmap(&tdo, dout, false, d, Nq, static_cast<uint64_t>(B) * Hq, fa::bwd::BM) ||
      !encode_tmap(&tk, k, false, d, Nk, static_cast<uint64_t>(B) * Hkv, fa::bwd::BN) ||
      !encode_tmap(&tv, v, false, d, Nk, static_cast<uint64_t>(B) * Hkv, fa::bwd::BN))
    return FA_ERR_INVALID_ARG;

  // Scratch, stream-ordered: the fp32 dQ accumulator and the padded per-row LSE * log2(e)
  // and D arrays.
  const uint64_t rows_padded = static_cast<uint64_t>(B) * Hq * p.Npad;
  uint64_t acc_bytes = 0, vec_bytes = 0, acc_used = 0;
  const uint64_t ws_bytes = bwd_scratch_bytes(B, Hq, Nq, d, &acc_bytes, &vec_bytes, &acc_used);
  void *ws = fixed_ws;
  if (ws == nullptr) {
    cudaMemPool_t pool;
    if (scratch_pool(dev, &pool) != FA_OK) return FA_ERR_CUDA;
    if (cudaMallocFromPoolAsync(&ws, ws_bytes, pool, stream) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
  }
  float *dq_acc = static_cast<float *>(ws);
  p.l2 = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + acc_bytes);
  p.dd = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + acc_bytes + vec_bytes);
  CUtensorMap tdq;
  st = encode_tmap_dq(&tdq, dq_acc, d, Nq, static_cast<uint64_t>(B) * Hq) ? FA_OK
                                                                           : FA_ERR_INVALID_ARG;
  if (st == FA_OK && cudaMemsetAsync(dq_acc, 0, acc_used, stream) != cudaSuccess)
    st = FA_ERR_CUDA;
  if (st == FA_OK) {
    const unsigned blocks = static_cast<unsigned>((rows_padded + 7) / 8);
    auto prep = d == 64 ? fa::bwd::fa_bwd_prep_kernel<64> : fa::bwd::fa_bwd_prep_kernel<128>;
    prep<<<blocks, 256, 0, stream>>>(static_cast<const uint16_t *>(o),
                                     static_cast<const uint16_t *>(dout), lse,
                                     const_cast<float *>(p.l2), const_cast<float *>(p.dd),
                                     static_cast<long long>(rows_padded), Nq, p.Npad);
    if (cudaGetLastError() != cudaSuccess) st = FA_ERR_CUDA;
  }
  if (st == FA_OK && sched_slot(dev, &p.sched) != FA_OK) st = FA_ERR_CUDA;
  if (st == FA_OK) {
    const int grid = p.num_units < info.sms ? p.num_units : info.sms;
    if (d == 64)
      st = causal ? bwd_launch<64, true>(tq, tk, tv, tdo, tdq, p, grid, dev, stream)
                  : bwd_launch<64, false>(tq, tk, tv, tdo, tdq, p, grid, dev, stream);
    else
      st = causal ? bwd_launch<128, true>(tq, tk, tv, tdo, tdq, p, grid, dev, stream)
                  : bwd_launch<128, false>(tq, tk, tv, tdo, tdq, p, grid, dev, stream);
  }
  if (st == FA_OK) {
    const long long n4 = static_cast<long long>(acc_used / 16);  // float4 groups of dQ
    fa::bwd::fa_bwd_dq_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, stream>>>(
        dq_acc, static_cast<uint16_t *>(dq), n4, scale);
    if (cudaGetLastError() != cudaSuccess) st = FA_ERR_CUDA;
  }
  if (fixed_ws == nullptr && cudaFreeAsync(ws, stream) != cudaSuccess && st == FA_OK)
    st = FA_ERR_CUDA;
  return st;
}

// Scratch of fa_bwd_noalloc.  Some callers cannot let the library allocate device memory
// per call: a framework whose own caching allocator has reserved (nearly) all of the
// device's memory, so that a stream-ordered allocation outside it can fail, or a service
// that must keep a fixed, known memory footprint.  For them the backward pass runs in this
// statically sized buffer, which exists once per device as part of the loaded library
// (no allocation at call time).  One buffer per device means calls that overlap in time on
// the same device (other streams, other host threads) would share it and race; such calls
// must be serialised by the caller.
constexpr uint64_t kNoAllocScratchBytes = 64ull << 20;
static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the fixed scratch on device `dev` (looked up once per device).
fa_status noalloc_scratch(int dev, void **out) {
  static std::once_flag once[kMaxDevices];
  static void *addr[kMaxDevices];
  static fa_status st[kMaxDevices];
  std::call_once(once[dev], [&] {
    st[dev] = cudaGetSymbolAddress(&addr[dev], g_bwd_noalloc_scratch) == cudaSuccess
                  ? FA_OK
                  : FA_ERR_CUDA;
    if (st[dev] != FA_OK) cudaGetLastError();
  });
  *out = addr[dev];
  return st[dev];
}

fa_status bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                      const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                      int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                      cudaStream_t stream) {
  fa_status st = check_bwd_args(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale,
                                causal);
  if (st != FA_OK) return st;
  uint64_t acc_bytes = 0, vec_bytes = 0;
  if (bwd_scratch_bytes(B, Hq, Nq, d, &acc_bytes, &vec_bytes) > kNoAllocScratchBytes)
    return FA_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  void *ws = nullptr;
  st = noalloc_scratch(dev, &ws);
  if (st != FA_OK) return st;
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                    stream, ws);
}

// ---------------------------------------------------------------- host-memory forward

// Per device: a stream for host-to-device copies, one for device-to-host copies, and the
// events that order them against the caller's stream.  Created on first use, kept for
// the life of the process; the mutex serialises the enqueueing of calls that share them.
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, in_done = nullptr, chunk_done = nullptr, out_done = nullptr;
  std::mutex mu;
  fa_status st = FA_ERR_CUDA;
};

HostPipe &host_pipe(int dev) {
  static HostPipe pipes[kMaxDevices];
  static std::once_flag once[kMaxDevices];
  HostPipe &hp = pipes[dev];
  std::call_once(once[dev], [&] {
    const unsigned ef = cudaEventDisableTiming;
    const bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.start, ef) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.in_done, ef) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.chunk_done, ef) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.out_done, ef) == cudaSuccess;
    if (!ok) cudaGetLastError();
    hp.st = ok ? FA_OK : FA_ERR_CUDA;
  });
  return hp;
}

// The forward for Q, K, V, O and LSE in host memory, pipelined by chunks of heads.  A
// chunk is a run of consecutive K/V heads (flattened over the batch) with the query heads
// that read them: for every tensor that is one contiguous byte range, and on the device
// it is an ordinary problem with B = 1.  Chunk c's inputs are copied on the input stream
// while the kernel of chunk c-1 runs on `stream` and the outputs of chunk c-2 go back on
// the output stream.
fa_status fwd_host(const void *qh, const void *kh, const void *vh, void *oh, float *lseh,
                   void *qd, void *kd, void *vd, void *od, float *lsed, int B, int Hq, int Hkv,
                   int Nq, int Nk, int d, float scale, int causal, bool out_f32, int chunks,
                   cudaStream_t stream) {
  if (!qh || !kh || !vh || !oh || !lseh || chunks < 0) return FA_ERR_INVALID_ARG;
  // the whole problem first, so that nothing is enqueued for an invalid request
  fa_status st = check_args(qd, kd, vd, od, lsed, B, Hq, Hkv, Nq, Nk, d, scale, causal, false,
                            nullptr, nullptr, nullptr);
  if (st != FA_OK) return st;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  const uint64_t groups = static_cast<uint64_t>(B) * Hkv;  // K/V heads, flattened
  const uint64_t g = static_cast<uint64_t>(Hq / Hkv);      // query heads per K/V head
  const uint64_t q_head = static_cast<uint64_t>(Nq) * d * 2;
  const uint64_t kv_head = static_cast<uint64_t>(Nk) * d * 2;
  const uint64_t o_head = static_cast<uint64_t>(Nq) * d * (out_f32 ? 4 : 2);
  const uint64_t lse_head = static_cast<uint64_t>(Nq) * 4;
  if (!buffer_ok(qd, groups * g * q_head, dev) || !buffer_ok(kd, groups * kv_head, dev) ||
      !buffer_ok(vd, groups * kv_head, dev) || !buffer_ok(od, groups * g * o_head, dev) ||
      !buffer_ok(lsed, groups * g * lse_head, dev))
    return FA_ERR_INVALID_ARG;
  // Chunk plan: chunk c covers K/V heads [c * per, min(groups, (c + 1) * per)) when the
  // library picks the size (chunks == 0), else an even split into `chunks` pieces.  The
  // library's size is as many K/V heads as fit one wave of work units (one CTA per SM),
  // at least one: a chunk's kernel then takes about as long as its copies, and a chunk
  // just over a wave, which would take two wave-times, never occurs.
  uint64_t n = static_cast<uint64_t>(chunks), per = 0;
  if (chunks == 0) {
    DeviceInfo info;
    st = device_info(dev, &info);
    if (st != FA_OK) return st;
    const bool pair = pair_path(d, false, 0, causal != 0);
    const uint64_t unit_rows = static_cast<uint64_t>(fwd_unit_rows(d, pair));
    const uint64_t group_units = g * ((static_cast<uint64_t>(Nq) + unit_rows - 1) / unit_rows);
    per = static_cast<uint64_t>(pair ? info.sms / 2 : info.sms) / group_units;
    if (per < 1) per = 1;
    n = (groups + per - 1) / per;
  }
  if (n > groups) n = groups;
  HostPipe &hp = host_pipe(dev);
  if (hp.st != FA_OK) return hp.st;
  std::lock_guard<std::mutex> lk(hp.mu);
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  auto bytes = [](const void *p, uint64_t off) {
    return static_cast<const uint8_t *>(p) + off;
  };
  auto wbytes = [](void *p, uint64_t off) { return static_cast<uint8_t *>(p) + off; };
  // nothing may overwrite the device buffers before the caller's earlier work is done
  if (!ok(cudaEventRecord(hp.start, stream)) || !ok(cudaStreamWaitEvent(hp.in, hp.start, 0)) ||
      !ok(cudaStreamWaitEvent(hp.out, hp.start, 0)))
    st = FA_ERR_CUDA;
  for (uint64_t c = 0; c < n && st == FA_OK; ++c) {
    // K/V heads [c0, c1)
    const uint64_t c0 = per ? c * per : groups * c / n;
    const uint64_t c1 = per ? (c0 + per < groups ? c0 + per : groups) : groups * (c + 1) / n;
    const uint64_t qo = c0 * g * q_head, qn = (c1 - c0) * g * q_head;
    const uint64_t ko = c0 * kv_head, kn = (c1 - c0) * kv_head;
    const uint64_t oo = c0 * g * o_head, on = (c1 - c0) * g * o_head;
    const uint64_t lo = c0 * g * lse_head, ln = (c1 - c0) * g * lse_head;
    if (!ok(cudaMemcpyAsync(wbytes(qd, qo), bytes(qh, qo), qn, cudaMemcpyHostToDevice, hp.in)) ||
        !ok(cudaMemcpyAsync(wbytes(kd, ko), bytes(kh, ko), kn, cudaMemcpyHostToDevice, hp.in)) ||
        !ok(cudaMemcpyAsync(wbytes(vd, ko), bytes(vh, ko), kn, cudaMemcpyHostToDevice, hp.in)) ||
        !ok(cudaEventRecord(hp.in_done, hp.in)) ||
        !ok(cudaStreamWaitEvent(stream, hp.in_done, 0))) {
      st = FA_ERR_CUDA;
      break;
    }
    st = fwd_common(bytes(qd, qo), bytes(kd, ko), bytes(vd, ko), wbytes(od, oo),
                    reinterpret_cast<float *>(wbytes(lsed, lo)), 1,
                    static_cast<int>((c1 - c0) * g), static_cast<int>(c1 - c0), Nq, Nk, d, scale,
                    causal, out_f32, false, nullptr, nullptr, nullptr, stream);
    if (st != FA_OK) break;
    if (!ok(cudaEventRecord(hp.chunk_done, stream)) ||
        !ok(cudaStreamWaitEvent(hp.out, hp.chunk_done, 0)) ||
        !ok(cudaMemcpyAsync(wbytes(oh, oo), bytes(od, oo), on, cudaMemcpyDeviceToHost, hp.out)) ||
        !ok(cudaMemcpyAsync(wbytes(lseh, lo), bytes(lsed, lo), ln, cudaMemcpyDeviceToHost,
                            hp.out)))
      st = FA_ERR_CUDA;
  }
  // whatever was enqueued, the caller's stream ends after all of it
  if (!ok(cudaEventRecord(hp.in_done, hp.in)) || !ok(cudaStreamWaitEvent(stream, hp.in_done, 0)) ||
      !ok(cudaEventRecord(hp.out_done, hp.out)) ||
      !ok(cudaStreamWaitEvent(stream, hp.out_done, 0))) {
    cudaGetLastError();
    if (st == FA_OK) st = FA_ERR_CUDA;
  }
  if (st == FA_ERR_CUDA) cudaGetLastError();
  return st;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                 int Hkv, int Nq, int Nk, int d, float scale, int causal, fa_dtype dtype,
                 fa_stream_t stream) {
  if (dtype != FA_BF16 && dtype != FA_BF16_OUT_F32) return FA_ERR_INVALID_ARG;
  return fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                    dtype == FA_BF16_OUT_F32, false, nullptr, nullptr, nullptr,
                    reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                     int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     const float *descale_q, const float *descale_k, const float *descale_v,
                     fa_stream_t stream) {
  return fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, false, true,
                    descale_q, descale_k, descale_v, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_quantize_e4m3(const void *x, const int8_t *signs, void *x8, float *descale, int B,
                           int H, int N, int d, fa_stream_t stream) {
  return quantize_common(x, signs, x8, descale, B, H, N, d,
                         reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_host(const void *q_host, const void *k_host, const void *v_host, void *o_host,
                      float *lse_host, void *q_dev, void *k_dev, void *v_dev, void *o_dev,
                      float *lse_dev, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                      int causal, fa_dtype dtype, int chunks, fa_stream_t stream) {
  if (dtype != FA_BF16 && dtype != FA_BF16_OUT_F32) return FA_ERR_INVALID_ARG;
  return fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev, lse_dev,
                  B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype == FA_BF16_OUT_F32, chunks,
                  reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         float dropout_p, uint64_t seed, uint64_t offset, fa_dtype dtype,
                         fa_stream_t stream) {
  if (dtype != FA_BF16 && dtype != FA_BF16_OUT_F32) return FA_ERR_INVALID_ARG;
  const int thr = dropout_threshold(dropout_p);
  if (thr < 0) return FA_ERR_INVALID_ARG;
  return fwd_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                    dtype == FA_BF16_OUT_F32, false, nullptr, nullptr, nullptr,
                    reinterpret_cast<cudaStream_t>(stream), thr, seed, offset);
}

fa_status fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                        const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int Hq, int Hkv,
                        int total_q, int total_k, int max_seqlen_q, int d, float scale,
                        int causal, fa_dtype dtype, fa_stream_t stream) {
  return fwd_varlen_common(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, total_q,
                           total_k, max_seqlen_q, d, scale, causal, dtype,
                           reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                 const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq,
                 int Nk, int d, float scale, int causal, fa_stream_t stream) {
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                    reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                         const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         fa_stream_t stream) {
  return bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                     reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_check_device_error(fa_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, fa::g_fa_error, sizeof(word)) != cudaSuccess) return FA_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_fa_error, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

fa_status fa_rescale_stats(fa_stream_t stream, unsigned long long *steps,
                           unsigned long long *lazy, unsigned long long *eager, int reset) {
  if (!steps || !lazy || !eager) return FA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  unsigned long long v[3] = {0, 0, 0};
  if (cudaMemcpyFromSymbol(v, fa::g_fa_rescale_stats, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  *steps = v[0];
  *lazy = v[1];
  *eager = v[2];
  if (reset) {
    const unsigned long long zero[3] = {0, 0, 0};
    if (cudaMemcpyToSymbol(fa::g_fa_rescale_stats, zero, sizeof(zero)) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  return FA_OK;
}

fa_status fa_selftest_bounded_wait(int timeout_us, fa_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return FA_ERR_INVALID_ARG;
  fa::fa_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

const char *fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "success";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int fa_version(void) { return 100; }

}  // extern "C"
