// noalloc.cu -- mla_attn_oproj_noalloc: the whole path (attention, head
// merge, o_proj) for callers that cannot allocate device memory at all, e.g.
// code that runs inside a host framework which owns every device allocation,
// or a plugin that is handed its inputs and outputs and nothing else. Its
// scratch (the merged attention output and the mask-tile classes) lives in a
// fixed, file-scope device array instead of a caller workspace.
#include "../../include/mla.h"
#include "abi_internal.h"
#include "attn_prefill.h"
#include "host_util.h"
#include "oproj_gemm.h"

namespace mla {
namespace {

// Merged attention output for up to MLA_NOALLOC_MAX_TOKENS tokens (64 MiB),
// then the mask-tile classes (64 KiB: B * ceil(T/128)^2 bytes fits for every
// B*T <= MLA_NOALLOC_MAX_TOKENS).
constexpr size_t kAttnBytes = size_t(MLA_NOALLOC_MAX_TOKENS) * MLA_OPROJ_IN * 2;
constexpr size_t kClassBytes = size_t(64) << 10;
constexpr size_t kScratchBytes = kAttnBytes + kClassBytes;
static_assert(kAttnBytes % 256 == 0, "class region alignment");

// Every GPU that loads this library holds this array until the process exits.
// Host code must not use the name as an address: it is a host-side stand-in;
// the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up with
// that device current (cudaGetSymbolAddress) and cached per device and
// context: after a device reset, or under another context of the device, it
// is looked up again. Null if the lookup fails.
ContextCache g_scratch_cache;

uint8_t* scratch_on_current_device() {
  return static_cast<uint8_t*>(symbol_address_cached(
      &g_scratch_cache, reinterpret_cast<const void*>(&g_noalloc_scratch)));
}

}  // namespace
}  // namespace mla

using namespace mla;
using namespace mla::abi;

extern "C" mla_status_t mla_attn_oproj_noalloc(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                               const mla_bf16* k_nope,
                                               const mla_bf16* k_pe_shared, const mla_bf16* v,
                                               const mla_bf16* mask, int64_t mask_ld, int B,
                                               int T, float softmax_scale, const mla_bf16* W_o,
                                               mla_bf16* out, mla_stream_t stream) {
  CallRange range("mla_attn_oproj_noalloc");
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if (!W_o) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W_o)) return MLA_ERR_MISALIGNED;
  // The fixed scratch bounds the problem size.
  if (int64_t(B) * int64_t(T) > MLA_NOALLOC_MAX_TOKENS) return MLA_ERR_WORKSPACE;
  if (mask && attn_class_bytes(B, T) > kClassBytes) return MLA_ERR_WORKSPACE;
  s = check_device();
  if (s != MLA_OK) return s;
  uint8_t* scratch = scratch_on_current_device();
  if (!scratch) return MLA_ERR_CUDA;
  // Nothing in the scratch has to start at zero: the attention kernel writes
  // every merged-output row it covers and the classifier every class byte
  // before either is read.
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* attn = scratch;
  void* cls = mask ? scratch + kAttnBytes : nullptr;
  s = run_attention(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T, softmax_scale, cls,
                    attn, st, device_error_word());
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_gemm(attn, W_o, out, int64_t(B) * T, MLA_HIDDEN, MLA_OPROJ_IN,
                                     device_sm_count(), wait_limit_ns(), 0, device_error_word(),
                                     st));
}
