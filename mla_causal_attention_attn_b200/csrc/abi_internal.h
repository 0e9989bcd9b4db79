// abi_internal.h -- host-side helpers shared by the C entry points
// (argument checks, device checks, the device status word, the attention
// launch sequence). Defined in mla_abi.cu.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/mla.h"

namespace mla {
namespace abi {

// NVTX range named after the entry point, open for the call's duration, so a
// profiler's timeline shows which library call enqueued which kernels. With
// no tool attached the push and pop do nothing.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

constexpr int kMaxB = 65535;
constexpr int kMaxT = 65535 * 128;
constexpr int64_t kMaxM = (int64_t(1) << 31) - 129;

// Device address of the device-wide status word on the current device and
// context (looked up once per context), or null. Calls without a workspace
// report bounded-wait timeouts there.
unsigned int* device_error_word();

// The status word a call reports timeouts to: the first word of its workspace
// (cleared on `stream` first, so it describes this call alone) or, without a
// workspace, the device-wide word. *st is MLA_ERR_CUDA if the clear could not
// be enqueued.
unsigned int* call_status_word(void* workspace, cudaStream_t stream, mla_status_t* st);

// Per-wait limit of the kernels' bounded waits (MLA_WAIT_LIMIT_NS, else 1 s).
unsigned long long wait_limit_ns();

// MLA_TEST_STALL_WAIT (failure-detection tests only): 1 stalls the attention
// kernel, 2 the small-M o_proj, 3 the attention kernel of masked calls only;
// 0 when unset.
int test_stall_wait();

bool aligned16(const void* p);
bool aligned4(const void* p);
size_t round_up(size_t x, size_t a);

// MLA_ERR_UNSUPPORTED_DEVICE unless the current device is CC 10.0.
mla_status_t check_device();

// Pointer, shape, scale and alignment checks shared by the attention calls.
mla_status_t check_attn_args(const void* q_nope, const void* q_pe, const void* k_nope,
                             const void* k_pe, const void* v, const void* mask, int64_t mask_ld,
                             int B, int T, float softmax_scale, const void* out);

mla_status_t from_cuda(cudaError_t e);

// Mask-tile classification (when mask is given, into `cls`) followed by the
// attention kernel writing the merged heads to `out`; timeouts go to
// err_word. valid_len (device [B], only without mask) selects causal
// attention with key padding; rope_cs (the rotary pre-pass's cos / sin
// table) makes the kernel rotate q_pe, with k_pe already rotated.
mla_status_t run_attention(const void* q_nope, const void* q_pe, const void* k_nope,
                           const void* k_pe, const void* v, const void* mask, int64_t mask_ld,
                           int B, int T, float softmax_scale, void* cls, void* out,
                           cudaStream_t stream, unsigned int* err_word,
                           const int* valid_len = nullptr, const void* rope_cs = nullptr);

}  // namespace abi
}  // namespace mla
