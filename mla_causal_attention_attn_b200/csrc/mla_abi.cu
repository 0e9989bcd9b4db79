// mla_abi.cu -- the extern "C" entry points declared in include/mla.h:
// argument validation, workspace carving, then kernel launches on the
// caller's stream.
#include <cmath>
#include <cstdlib>
#include <mutex>

#include "../../include/mla.h"
#include "abi_internal.h"
#include "attn_prefill.h"
#include "fp8_oproj.h"
#include "host_util.h"
#include "oproj_gemm.h"
#include "rope.h"
#include "sm100.cuh"

namespace mla {

// The device-wide status word (one per device that loads the library), used by
// the calls that take no workspace; and the mailbox mla_device_status reads it
// through.
__device__ unsigned int g_device_error = 0;
__device__ unsigned int g_status_mailbox = 0;

namespace {

// Takes the device-wide word and clears it in one atomic step, so that a
// timeout recorded by a kernel on another stream meanwhile is never lost.
__global__ void take_status_kernel(unsigned int* word, unsigned int* mailbox) {
  *mailbox = atomicExch(word, 0u);
}

ContextCache g_error_word_cache, g_mailbox_cache;
std::mutex g_status_mu;

}  // namespace

namespace abi {

unsigned int* device_error_word() {
  return static_cast<unsigned int*>(
      symbol_address_cached(&g_error_word_cache, reinterpret_cast<const void*>(&g_device_error)));
}

unsigned int* call_status_word(void* workspace, cudaStream_t stream, mla_status_t* st) {
  *st = MLA_OK;
  if (!workspace) return device_error_word();
  if (cudaMemsetAsync(workspace, 0, sizeof(unsigned int), stream) != cudaSuccess)
    *st = MLA_ERR_CUDA;
  return static_cast<unsigned int*>(workspace);
}

unsigned long long wait_limit_ns() {
  // MLA_WAIT_LIMIT_NS overrides the per-wait limit (read once).
  static const unsigned long long v = [] {
    const char* s = std::getenv("MLA_WAIT_LIMIT_NS");
    if (s && *s) {
      char* end = nullptr;
      unsigned long long x = std::strtoull(s, &end, 10);
      if (end && *end == '\0' && x > 0) return x;
    }
    return kDefaultWaitLimitNs;
  }();
  return v;
}

// MLA_TEST_STALL_WAIT (read once) lets tests make one bounded wait run out,
// to check that the kernel gives up cleanly and MLA_ERR_TIMEOUT is reported:
// 1 = the attention kernel's first CTA waits on a barrier that nothing
// completes; 2 = in the first cluster of the small-M o_proj, the rank-1 CTA
// never reports its partial sum; 3 = as 1, but only in attention calls given
// an explicit mask. Never set in normal use.
int test_stall_wait() {
  static const int v = [] {
    const char* s = std::getenv("MLA_TEST_STALL_WAIT");
    if (s && s[0] >= '1' && s[0] <= '3' && s[1] == '\0') return s[0] - '0';
    return 0;
  }();
  return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

mla_status_t check_device() {
  const int cc = device_cc();
  if (cc == 0) return MLA_ERR_CUDA;
  if (cc != 100) return MLA_ERR_UNSUPPORTED_DEVICE;
  if (!device_error_word()) return MLA_ERR_CUDA;
  return MLA_OK;
}

mla_status_t check_attn_args(const void* q_nope, const void* q_pe, const void* k_nope,
                             const void* k_pe, const void* v, const void* mask, int64_t mask_ld,
                             int B, int T, float softmax_scale, const void* out) {
  if (!q_nope || !q_pe || !k_nope || !k_pe || !v || !out) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT) return MLA_ERR_SHAPE;
  if (mask && mask_ld < T) return MLA_ERR_SHAPE;
  if (!aligned16(q_nope) || !aligned16(q_pe) || !aligned16(k_nope) || !aligned16(k_pe) ||
      !aligned16(v) || !aligned16(out))
    return MLA_ERR_MISALIGNED;
  if (mask && (reinterpret_cast<uintptr_t>(mask) & 1u) != 0) return MLA_ERR_MISALIGNED;
  return MLA_OK;
}

mla_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

mla_status_t run_attention(const void* q_nope, const void* q_pe, const void* k_nope,
                           const void* k_pe, const void* v, const void* mask, int64_t mask_ld,
                           int B, int T, float softmax_scale, void* cls, void* out,
                           cudaStream_t stream, unsigned int* err_word, const int* valid_len,
                           const void* rope_cs) {
  if (mask) {
    mla_status_t s = from_cuda(launch_mask_classify(mask, mask_ld, B, T, cls, stream));
    if (s != MLA_OK) return s;
  }
  const int stall = test_stall_wait();
  return from_cuda(launch_attn_prefill(q_nope, q_pe, k_nope, k_pe, v, mask, mask_ld,
                                       mask ? cls : nullptr, B, T, softmax_scale, out,
                                       wait_limit_ns(), err_word,
                                       (stall == 1 || (stall == 3 && mask)) ? 1 : 0, stream,
                                       valid_len, rope_cs));
}

mla_status_t rope_freqs(const mla_yarn_rope_t* rope, RopeFreqs* f) {
  if (!rope) return MLA_ERR_INVALID_ARG;
  return yarn_frequencies(rope->rope_theta, rope->factor, rope->original_max_position_embeddings,
                          rope->beta_fast, rope->beta_slow, rope->mscale, rope->mscale_all_dim, f)
             ? MLA_OK
             : MLA_ERR_INVALID_ARG;
}

// Workspace regions of the rotary calls after the status block: the rotated
// key, then the cos / sin table.
size_t rope_region_bytes(int B, int T) {
  return round_up(rope_krot_bytes(B, T), 256) + round_up(rope_cs_bytes(B, T), 256);
}

}  // namespace abi
}  // namespace mla

using namespace mla;
using namespace mla::abi;

extern "C" {

size_t mla_attn_prefill_workspace_bytes(int B, int T, int has_mask) {
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT) return 0;
  return MLA_WORKSPACE_STATUS_BYTES + (has_mask ? attn_class_bytes(B, T) : 0);
}

mla_status_t mla_attn_prefill(const mla_bf16* q_nope, const mla_bf16* q_pe,
                              const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                              const mla_bf16* v, const mla_bf16* mask, int64_t mask_ld, int B,
                              int T, float softmax_scale, void* workspace,
                              size_t workspace_bytes, mla_bf16* out, mla_stream_t stream) {
  CallRange range("mla_attn_prefill");
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if (mask && !workspace) return MLA_ERR_WORKSPACE;
  if (workspace) {
    if (workspace_bytes < mla_attn_prefill_workspace_bytes(B, T, mask != nullptr))
      return MLA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  }
  s = check_device();
  if (s != MLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = call_status_word(workspace, st, &s);
  if (s != MLA_OK) return s;
  void* cls = workspace ? static_cast<uint8_t*>(workspace) + MLA_WORKSPACE_STATUS_BYTES : nullptr;
  return run_attention(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T, softmax_scale,
                       cls, out, st, err);
}

mla_status_t mla_o_proj(const mla_bf16* attn, const mla_bf16* W_o, int64_t M, mla_bf16* out,
                        mla_stream_t stream) {
  CallRange range("mla_o_proj");
  if (!attn || !W_o || !out) return MLA_ERR_INVALID_ARG;
  if (M < 1 || M > kMaxM) return MLA_ERR_SHAPE;
  if (!aligned16(attn) || !aligned16(W_o) || !aligned16(out)) return MLA_ERR_MISALIGNED;
  mla_status_t s = check_device();
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_gemm(attn, W_o, out, M, MLA_HIDDEN, MLA_OPROJ_IN,
                                     device_sm_count(), wait_limit_ns(), 0, device_error_word(),
                                     reinterpret_cast<cudaStream_t>(stream),
                                     test_stall_wait() == 2 ? 1 : 0));
}

size_t mla_attn_oproj_workspace_bytes(int B, int T, int has_mask) {
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT) return 0;
  size_t bytes = MLA_WORKSPACE_STATUS_BYTES + round_up(size_t(B) * size_t(T) * MLA_OPROJ_IN * 2, 256);
  if (has_mask) bytes += round_up(attn_class_bytes(B, T), 256);
  return bytes;
}

mla_status_t mla_attn_oproj(const mla_bf16* q_nope, const mla_bf16* q_pe,
                            const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                            const mla_bf16* v, const mla_bf16* mask, int64_t mask_ld, int B,
                            int T, float softmax_scale, const mla_bf16* W_o, void* workspace,
                            size_t workspace_bytes, mla_bf16* out, mla_stream_t stream) {
  CallRange range("mla_attn_oproj");
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if (!W_o) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W_o)) return MLA_ERR_MISALIGNED;
  if (int64_t(B) * int64_t(T) > kMaxM) return MLA_ERR_SHAPE;
  const size_t need = mla_attn_oproj_workspace_bytes(B, T, mask != nullptr);
  if (!workspace || workspace_bytes < need) return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  s = check_device();
  if (s != MLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = call_status_word(workspace, st, &s);
  if (s != MLA_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace) + MLA_WORKSPACE_STATUS_BYTES;
  const size_t attn_bytes = round_up(size_t(B) * size_t(T) * MLA_OPROJ_IN * 2, 256);
  void* attn = ws;
  void* cls = mask ? ws + attn_bytes : nullptr;
  s = run_attention(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T, softmax_scale, cls,
                    attn, st, err);
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_gemm(attn, W_o, out, int64_t(B) * T, MLA_HIDDEN, MLA_OPROJ_IN,
                                     device_sm_count(), wait_limit_ns(), 0, err, st));
}

mla_status_t mla_attn_prefill_varlen(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                     const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                                     const mla_bf16* v, const int32_t* valid_len, int B, int T,
                                     float softmax_scale, mla_bf16* out, mla_stream_t stream) {
  CallRange range("mla_attn_prefill_varlen");
  if (!valid_len) return MLA_ERR_INVALID_ARG;
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe_shared, v, nullptr, 0, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if ((reinterpret_cast<uintptr_t>(valid_len) & 3u) != 0) return MLA_ERR_MISALIGNED;
  s = check_device();
  if (s != MLA_OK) return s;
  return run_attention(q_nope, q_pe, k_nope, k_pe_shared, v, nullptr, 0, B, T, softmax_scale,
                       nullptr, out, reinterpret_cast<cudaStream_t>(stream), device_error_word(),
                       valid_len);
}

mla_status_t mla_attn_oproj_varlen(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                   const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                                   const mla_bf16* v, const int32_t* valid_len, int B, int T,
                                   float softmax_scale, const mla_bf16* W_o, void* workspace,
                                   size_t workspace_bytes, mla_bf16* out, mla_stream_t stream) {
  CallRange range("mla_attn_oproj_varlen");
  if (!valid_len || !W_o) return MLA_ERR_INVALID_ARG;
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe_shared, v, nullptr, 0, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if ((reinterpret_cast<uintptr_t>(valid_len) & 3u) != 0 || !aligned16(W_o))
    return MLA_ERR_MISALIGNED;
  if (int64_t(B) * int64_t(T) > kMaxM) return MLA_ERR_SHAPE;
  const size_t need = mla_attn_oproj_workspace_bytes(B, T, 0);
  if (!workspace || workspace_bytes < need) return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  s = check_device();
  if (s != MLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = call_status_word(workspace, st, &s);
  if (s != MLA_OK) return s;
  void* attn = static_cast<uint8_t*>(workspace) + MLA_WORKSPACE_STATUS_BYTES;
  s = run_attention(q_nope, q_pe, k_nope, k_pe_shared, v, nullptr, 0, B, T, softmax_scale, nullptr,
                    attn, st, err, valid_len);
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_gemm(attn, W_o, out, int64_t(B) * T, MLA_HIDDEN, MLA_OPROJ_IN,
                                     device_sm_count(), wait_limit_ns(), 0, err, st));
}

size_t mla_attn_prefill_rope_workspace_bytes(int B, int T, int has_mask) {
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT) return 0;
  size_t bytes = MLA_WORKSPACE_STATUS_BYTES + rope_region_bytes(B, T);
  if (has_mask) bytes += round_up(attn_class_bytes(B, T), 256);
  return bytes;
}

mla_status_t mla_attn_prefill_rope(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                   const mla_bf16* k_nope, const mla_bf16* k_pe,
                                   const mla_bf16* v, const int32_t* position_ids,
                                   const mla_yarn_rope_t* rope, const mla_bf16* mask,
                                   int64_t mask_ld, int B, int T, float softmax_scale,
                                   void* workspace, size_t workspace_bytes, mla_bf16* out,
                                   mla_stream_t stream) {
  CallRange range("mla_attn_prefill_rope");
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe, v, mask, mask_ld, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  RopeFreqs f;
  s = rope_freqs(rope, &f);
  if (s != MLA_OK) return s;
  if (position_ids && !aligned4(position_ids)) return MLA_ERR_MISALIGNED;
  if (!workspace ||
      workspace_bytes < mla_attn_prefill_rope_workspace_bytes(B, T, mask != nullptr))
    return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  s = check_device();
  if (s != MLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = call_status_word(workspace, st, &s);
  if (s != MLA_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace) + MLA_WORKSPACE_STATUS_BYTES;
  uint8_t* k_rot = ws;
  uint8_t* cs = k_rot + round_up(rope_krot_bytes(B, T), 256);
  void* cls = mask ? ws + rope_region_bytes(B, T) : nullptr;
  s = from_cuda(launch_rope_prepass(k_pe, position_ids, B, T, f, cs, k_rot, st));
  if (s != MLA_OK) return s;
  return run_attention(q_nope, q_pe, k_nope, k_rot, v, mask, mask_ld, B, T, softmax_scale, cls,
                       out, st, err, nullptr, cs);
}

size_t mla_attn_oproj_rope_workspace_bytes(int B, int T, int has_mask) {
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT) return 0;
  return mla_attn_prefill_rope_workspace_bytes(B, T, has_mask) +
         round_up(size_t(B) * size_t(T) * MLA_OPROJ_IN * 2, 256);
}

mla_status_t mla_attn_oproj_rope(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                 const mla_bf16* k_nope, const mla_bf16* k_pe, const mla_bf16* v,
                                 const int32_t* position_ids, const mla_yarn_rope_t* rope,
                                 const mla_bf16* mask, int64_t mask_ld, int B, int T,
                                 float softmax_scale, const mla_bf16* W_o, void* workspace,
                                 size_t workspace_bytes, mla_bf16* out, mla_stream_t stream) {
  CallRange range("mla_attn_oproj_rope");
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe, v, mask, mask_ld, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if (!W_o) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W_o)) return MLA_ERR_MISALIGNED;
  if (int64_t(B) * int64_t(T) > kMaxM) return MLA_ERR_SHAPE;
  RopeFreqs f;
  s = rope_freqs(rope, &f);
  if (s != MLA_OK) return s;
  if (position_ids && !aligned4(position_ids)) return MLA_ERR_MISALIGNED;
  if (!workspace ||
      workspace_bytes < mla_attn_oproj_rope_workspace_bytes(B, T, mask != nullptr))
    return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  s = check_device();
  if (s != MLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = call_status_word(workspace, st, &s);
  if (s != MLA_OK) return s;
  // status | rotated key | cos/sin table | merged attention | mask classes
  uint8_t* ws = static_cast<uint8_t*>(workspace) + MLA_WORKSPACE_STATUS_BYTES;
  uint8_t* k_rot = ws;
  uint8_t* cs = k_rot + round_up(rope_krot_bytes(B, T), 256);
  uint8_t* attn = ws + rope_region_bytes(B, T);
  void* cls = mask ? attn + round_up(size_t(B) * size_t(T) * MLA_OPROJ_IN * 2, 256) : nullptr;
  s = from_cuda(launch_rope_prepass(k_pe, position_ids, B, T, f, cs, k_rot, st));
  if (s != MLA_OK) return s;
  s = run_attention(q_nope, q_pe, k_nope, k_rot, v, mask, mask_ld, B, T, softmax_scale, cls,
                    attn, st, err, nullptr, cs);
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_gemm(attn, W_o, out, int64_t(B) * T, MLA_HIDDEN, MLA_OPROJ_IN,
                                     device_sm_count(), wait_limit_ns(), 0, err, st));
}

mla_status_t mla_kv_up_proj(const mla_bf16* c_kv, const mla_bf16* W_kv_b, int B, int T,
                            mla_bf16* k_nope, mla_bf16* v, mla_stream_t stream) {
  CallRange range("mla_kv_up_proj");
  if (!c_kv || !W_kv_b || !k_nope || !v) return MLA_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT || int64_t(B) * int64_t(T) > kMaxM)
    return MLA_ERR_SHAPE;
  if (!aligned16(c_kv) || !aligned16(W_kv_b) || !aligned16(k_nope) || !aligned16(v))
    return MLA_ERR_MISALIGNED;
  mla_status_t s = check_device();
  if (s != MLA_OK) return s;
  return from_cuda(launch_kv_up(c_kv, W_kv_b, k_nope, v, B, T, MLA_KV_RANK, device_sm_count(),
                                wait_limit_ns(), device_error_word(),
                                reinterpret_cast<cudaStream_t>(stream)));
}

size_t mla_attn_oproj_latent_workspace_bytes(int B, int T, int has_mask) {
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT) return 0;
  // status | k_nope | v | merged attention | mask classes
  const size_t kv = round_up(size_t(B) * MLA_NUM_HEADS * size_t(T) * MLA_QK_NOPE_DIM * 2, 256);
  return mla_attn_oproj_workspace_bytes(B, T, has_mask) + 2 * kv;
}

mla_status_t mla_attn_oproj_latent(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                   const mla_bf16* c_kv, const mla_bf16* k_pe_shared,
                                   const mla_bf16* W_kv_b, const mla_bf16* mask, int64_t mask_ld,
                                   int B, int T, float softmax_scale, const mla_bf16* W_o,
                                   void* workspace, size_t workspace_bytes, mla_bf16* out,
                                   mla_stream_t stream) {
  CallRange range("mla_attn_oproj_latent");
  // the up-projection's outputs stand in for k_nope and v in the checks
  mla_status_t s = check_attn_args(q_nope, q_pe, c_kv, k_pe_shared, W_kv_b, mask, mask_ld, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if (!W_o) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W_o)) return MLA_ERR_MISALIGNED;
  if (int64_t(B) * int64_t(T) > kMaxM) return MLA_ERR_SHAPE;
  const size_t need = mla_attn_oproj_latent_workspace_bytes(B, T, mask != nullptr);
  if (!workspace || workspace_bytes < need) return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  s = check_device();
  if (s != MLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = call_status_word(workspace, st, &s);
  if (s != MLA_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace) + MLA_WORKSPACE_STATUS_BYTES;
  const size_t kv = round_up(size_t(B) * MLA_NUM_HEADS * size_t(T) * MLA_QK_NOPE_DIM * 2, 256);
  const size_t attn_bytes = round_up(size_t(B) * size_t(T) * MLA_OPROJ_IN * 2, 256);
  uint8_t* k_nope = ws;
  uint8_t* v = ws + kv;
  uint8_t* attn = ws + 2 * kv;
  void* cls = mask ? attn + attn_bytes : nullptr;
  s = from_cuda(launch_kv_up(c_kv, W_kv_b, k_nope, v, B, T, MLA_KV_RANK, device_sm_count(),
                             wait_limit_ns(), err, st));
  if (s != MLA_OK) return s;
  s = run_attention(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T, softmax_scale,
                    cls, attn, st, err);
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_gemm(attn, W_o, out, int64_t(B) * T, MLA_HIDDEN, MLA_OPROJ_IN,
                                     device_sm_count(), wait_limit_ns(), 0, err, st));
}

mla_status_t mla_quantize_act_fp8(const mla_bf16* x, int64_t M, uint8_t* q, float* scale,
                                  mla_stream_t stream) {
  CallRange range("mla_quantize_act_fp8");
  if (!x || !q || !scale) return MLA_ERR_INVALID_ARG;
  if (M < 1 || M > kMaxM) return MLA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(q) || !aligned4(scale)) return MLA_ERR_MISALIGNED;
  mla_status_t s = check_device();
  if (s != MLA_OK) return s;
  return from_cuda(launch_quant_rows_fp8(x, MLA_OPROJ_IN, M, MLA_OPROJ_IN, q, scale,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

mla_status_t mla_quantize_weight_fp8(const mla_bf16* W, uint8_t* q, float* scale,
                                     mla_stream_t stream) {
  CallRange range("mla_quantize_weight_fp8");
  if (!W || !q || !scale) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(q) || !aligned4(scale)) return MLA_ERR_MISALIGNED;
  mla_status_t s = check_device();
  if (s != MLA_OK) return s;
  return from_cuda(launch_quant_weight_fp8(W, MLA_HIDDEN, MLA_OPROJ_IN, q, scale,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

mla_status_t mla_o_proj_fp8(const uint8_t* attn_q, const float* attn_scale, const uint8_t* W_q,
                            const float* W_scale, int64_t M, mla_bf16* out,
                            mla_stream_t stream) {
  CallRange range("mla_o_proj_fp8");
  if (!attn_q || !attn_scale || !W_q || !W_scale || !out) return MLA_ERR_INVALID_ARG;
  if (M < 1 || M > kMaxM) return MLA_ERR_SHAPE;
  if (!aligned16(attn_q) || !aligned16(W_q) || !aligned16(out) || !aligned4(attn_scale) ||
      !aligned4(W_scale))
    return MLA_ERR_MISALIGNED;
  mla_status_t s = check_device();
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_fp8(attn_q, attn_scale, W_q, W_scale, out, M, MLA_HIDDEN,
                                    MLA_OPROJ_IN, device_sm_count(), wait_limit_ns(),
                                    device_error_word(), reinterpret_cast<cudaStream_t>(stream)));
}

size_t mla_attn_oproj_fp8_workspace_bytes(int B, int T, int has_mask) {
  if (B < 1 || T < 1 || B > kMaxB || T > kMaxT) return 0;
  const size_t M = size_t(B) * size_t(T);
  size_t bytes = MLA_WORKSPACE_STATUS_BYTES + round_up(M * MLA_OPROJ_IN * 2, 256) +
                 round_up(M * MLA_OPROJ_IN, 256) +
                 round_up(M * MLA_FP8_K_GROUPS * 4, 256);
  if (has_mask) bytes += round_up(attn_class_bytes(B, T), 256);
  return bytes;
}

mla_status_t mla_attn_oproj_fp8(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                                const mla_bf16* v, const mla_bf16* mask, int64_t mask_ld, int B,
                                int T, float softmax_scale, const uint8_t* W_q,
                                const float* W_scale, void* workspace, size_t workspace_bytes,
                                mla_bf16* out, mla_stream_t stream) {
  CallRange range("mla_attn_oproj_fp8");
  mla_status_t s = check_attn_args(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T,
                                   softmax_scale, out);
  if (s != MLA_OK) return s;
  if (!W_q || !W_scale) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W_q) || !aligned4(W_scale)) return MLA_ERR_MISALIGNED;
  if (int64_t(B) * int64_t(T) > kMaxM) return MLA_ERR_SHAPE;
  const size_t need = mla_attn_oproj_fp8_workspace_bytes(B, T, mask != nullptr);
  if (!workspace || workspace_bytes < need) return MLA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  s = check_device();
  if (s != MLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = call_status_word(workspace, st, &s);
  if (s != MLA_OK) return s;
  const int64_t M = int64_t(B) * T;
  uint8_t* ws = static_cast<uint8_t*>(workspace) + MLA_WORKSPACE_STATUS_BYTES;
  uint8_t* attn = ws;
  uint8_t* attn_q = attn + round_up(size_t(M) * MLA_OPROJ_IN * 2, 256);
  float* attn_scale =
      reinterpret_cast<float*>(attn_q + round_up(size_t(M) * MLA_OPROJ_IN, 256));
  void* cls = mask ? reinterpret_cast<uint8_t*>(attn_scale) +
                         round_up(size_t(M) * MLA_FP8_K_GROUPS * 4, 256)
                   : nullptr;
  s = run_attention(q_nope, q_pe, k_nope, k_pe_shared, v, mask, mask_ld, B, T, softmax_scale, cls,
                    attn, st, err);
  if (s != MLA_OK) return s;
  s = from_cuda(launch_quant_rows_fp8(attn, MLA_OPROJ_IN, M, MLA_OPROJ_IN, attn_q, attn_scale,
                                      st));
  if (s != MLA_OK) return s;
  return from_cuda(launch_oproj_fp8(attn_q, attn_scale, W_q, W_scale, out, M, MLA_HIDDEN,
                                    MLA_OPROJ_IN, device_sm_count(), wait_limit_ns(), err, st));
}

mla_status_t mla_device_status(mla_stream_t stream, uint32_t* detail) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (detail) *detail = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_status_mu);  // one mailbox per device
  unsigned int* word = device_error_word();
  unsigned int* box = static_cast<unsigned int*>(
      symbol_address_cached(&g_mailbox_cache, reinterpret_cast<const void*>(&g_status_mailbox)));
  if (!word || !box) return MLA_ERR_CUDA;
  take_status_kernel<<<1, 1, 0, st>>>(word, box);
  if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, box, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (detail) *detail = v;
  return (v & kErrTimeoutFlag) ? MLA_ERR_TIMEOUT : MLA_OK;
}

mla_status_t mla_last_device_status(const void* workspace, mla_stream_t stream,
                                    uint32_t* detail) {
  if (detail) *detail = 0;
  if (!workspace) return MLA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return MLA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (detail) *detail = v;
  return (v & kErrTimeoutFlag) ? MLA_ERR_TIMEOUT : MLA_OK;
}

const char* mla_status_string(mla_status_t status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_SHAPE: return "MLA_ERR_SHAPE";
    case MLA_ERR_MISALIGNED: return "MLA_ERR_MISALIGNED";
    case MLA_ERR_UNSUPPORTED_DEVICE: return "MLA_ERR_UNSUPPORTED_DEVICE";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
  }
  return "MLA_ERR_UNKNOWN";
}

int mla_abi_version(void) { return MLA_ABI_VERSION; }

}  // extern "C"
