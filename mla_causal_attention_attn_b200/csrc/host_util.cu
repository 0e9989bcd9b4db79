// host_util.cu -- see host_util.h.
#include "host_util.h"

#include <mutex>

namespace mla {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
int g_cc[kMaxDevices] = {0};
std::mutex g_dev_mu;

void fill_device_info(int dev) {
  int sms = 0, major = 0, minor = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  g_sm_count[dev] = sms;
  g_cc[dev] = major * 10 + minor;
}

}  // namespace

namespace {

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 bool swizzle128) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t bdim[5];
  cuuint32_t estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank),
                  const_cast<void*>(base), gdim, gstride, bdim, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box,
                     swizzle128);
}

bool encode_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides_bytes, box,
                     swizzle128);
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> g(g_dev_mu);
  if (g_sm_count[dev] == 0) fill_device_info(dev);
  return g_sm_count[dev];
}

int device_cc() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> g(g_dev_mu);
  if (g_cc[dev] == 0) fill_device_info(dev);
  return g_cc[dev];
}

}  // namespace mla

namespace mla {

namespace {

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn get_ctx_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

std::mutex g_cache_mu;

}  // namespace

void* current_context() {
  CtxGetCurrentFn fn = get_ctx_fn();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return static_cast<void*>(c);
}

void* symbol_address_cached(ContextCache* cache, const void* symbol) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= ContextCache::kMaxDevices)
    return nullptr;
  std::lock_guard<std::mutex> g(g_cache_mu);
  void* ctx = current_context();
  if (ctx && cache->ctx[dev] == ctx && cache->value[dev]) return cache->value[dev];
  void* a = nullptr;
  if (cudaGetSymbolAddress(&a, symbol) != cudaSuccess || a == nullptr) return nullptr;
  // the lookup makes the device's primary context current if none was
  cache->ctx[dev] = current_context();
  cache->value[dev] = a;
  return a;
}

cudaError_t ensure_smem_attr(const void* func, int bytes, ContextCache* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < ContextCache::kMaxDevices;
  if (cacheable) {
    std::lock_guard<std::mutex> g(g_cache_mu);
    void* ctx = current_context();
    if (ctx && done->ctx[dev] == ctx) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cacheable) {
    std::lock_guard<std::mutex> g(g_cache_mu);
    done->ctx[dev] = current_context();
  }
  return e;
}

}  // namespace mla
