// host_util.h -- host-side helpers shared by the launchers: TMA tensor-map
// encoding through the driver entry point, per-device SM count cache and
// kernel-attribute setup.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mla {

// Encode a row-major bf16 tensor of `rank` dims (dims[0] innermost, in
// elements; strides_bytes[i] is the byte stride of dim i+1) as a TMA tiled map
// with 128-byte swizzle and zero fill out of bounds. Returns false when the
// driver rejects the map.
bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);

// Same for a tensor of bytes (e4m3 codes): dims and box in elements = bytes.
bool encode_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);

// Number of SMs of the current device (cached per device ordinal).
int device_sm_count();

// Compute capability major*10+minor of the current device (cached).
int device_cc();

// Opaque handle of the calling thread's current CUDA context (the driver's
// CUcontext), or null if none is current or the driver entry point is missing.
void* current_context();

// Per-device cache of values that belong to one CUDA context (device
// addresses of module variables, function attributes already set). An entry
// is valid only for the context it was filled in: after a device reset, or
// when another context of the same device is current, it is filled again.
struct ContextCache {
  static constexpr int kMaxDevices = 64;
  void* ctx[kMaxDevices] = {};
  void* value[kMaxDevices] = {};
};

// Device address of the module variable `symbol` on the current device and
// context (cudaGetSymbolAddress), cached in `cache`; null if the lookup fails.
void* symbol_address_cached(ContextCache* cache, const void* symbol);

// Sets the max-dynamic-shared-memory attribute of `func` once per device and
// context.
cudaError_t ensure_smem_attr(const void* func, int bytes, ContextCache* done);

}  // namespace mla
