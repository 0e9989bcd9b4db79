/*
 * mla.h -- C ABI of the B200 (sm_100a) MLA prefill attention + o_proj library
 * (libmla_b200.so).
 *
 * What it computes is the attention core and output projection of one Kimi K2
 * multi-head latent attention block during prefill, as defined on the page
 * "Kimi K2 · Mix and project" (code excerpts modeling_deepseek.py 799-840 and
 * 848-852) with the dimensions of the model configuration printed on
 * "Kimi K2 · Block input" (num_attention_heads 64, qk_nope_head_dim 128,
 * qk_rope_head_dim 64, v_head_dim 128, hidden_size 7168):
 *
 *   s[b,h,i,j] = softmax_scale * ( q_nope[b,h,i,:] . k_nope[b,h,j,:]
 *                                + q_pe[b,h,i,:]   . k_pe[b,0,j,:] ) + M[b,0,i,j]
 *   p[b,h,i,:] = softmax over j of s[b,h,i,:]     (fp32)
 *   attn[b,i,h*128+e] = sum_j p[b,h,i,j] v[b,h,j,e]     (heads merged)
 *   out[b,i,n] = sum_k attn[b,i,k] W_o[n,k]             (o_proj, no bias)
 *
 * Conventions shared by every call:
 *  - Element type: bf16, passed as its 16-bit pattern (mla_bf16). All tensors
 *    are dense, row-major, in the layouts stated per argument.
 *  - Memory: every pointer is a device pointer on the current CUDA device.
 *    The caller allocates and frees everything, workspaces included; the
 *    library never allocates device memory.
 *  - Alignment: every tensor pointer and the workspace must be 16-byte
 *    aligned (TMA), the mask 2-byte aligned; otherwise MLA_ERR_MISALIGNED.
 *  - Streams: work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and the call returns without synchronising. Only
 *    mla_last_device_status() and mla_device_status() synchronise.
 *  - Errors: every argument is checked before anything is launched; errors
 *    are returned, never thrown or printed. A kernel that gives up on an
 *    internal bounded wait records MLA_ERR_TIMEOUT in a status word instead of
 *    trapping:
 *      - calls given a workspace use the first word of it (the workspace
 *        starts with MLA_WORKSPACE_STATUS_BYTES reserved for this). The call
 *        clears that word on its stream before its kernels run, so it holds
 *        this call's outcome alone; read it with mla_last_device_status();
 *      - calls without a workspace (mla_o_proj, mla_attn_prefill with
 *        workspace NULL, mla_attn_prefill_varlen, mla_kv_up_proj, the FP8
 *        quantisers and GEMM, mla_attn_oproj_noalloc) use one device-wide
 *        word per device, read and cleared atomically by mla_device_status().
 *  - Device: compute capability 10.0 (B200, sm_100a) only; otherwise
 *    MLA_ERR_UNSUPPORTED_DEVICE.
 *  - Threads: calls are thread-safe. Mutable state shared between calls: the
 *    device-wide status word above (calls without a workspace on different
 *    streams report into the same word) and the no-alloc call's fixed
 *    scratch. Cached per device and context: the SM count, device addresses
 *    of the library's module variables, kernel attributes.
 *  - Environment (each read once per process): MLA_WAIT_LIMIT_NS sets the
 *    bounded waits' limit in nanoseconds; MLA_ATTN_KERNEL selects the
 *    attention kernel: unset, the one-SM kernel with 64-key score halves
 *    (under an explicit mask, 128-key tiles for the CTAs whose query tiles
 *    skip a key tile before a used one);
 *    "tile", 128-key tiles for every call; "pair", the CTA-pair kernel for
 *    every call. The choice changes rounding order only: every setting
 *    meets the same tolerance. MLA_ATTN_PV_ISSUER ("1" or "0") overrides
 *    which thread issues the 64-key halves' PV products (a thread of their
 *    own from T = 4096 on, else each query tile's MMA issuer); both give
 *    bit-identical results. MLA_TEST_STALL_WAIT makes
 *    one bounded wait never complete, for failure-detection tests.
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 4

/* Model dimensions (fixed at compile time; no other values are accepted). */
#define MLA_NUM_HEADS 64
#define MLA_QK_NOPE_DIM 128
#define MLA_QK_ROPE_DIM 64
#define MLA_V_DIM 128
#define MLA_OPROJ_IN 8192 /* MLA_NUM_HEADS * MLA_V_DIM */
#define MLA_HIDDEN 7168

/* Bytes at the start of every workspace reserved for the call's status word. */
#define MLA_WORKSPACE_STATUS_BYTES 256

typedef uint16_t mla_bf16; /* bit pattern of a bfloat16 value */
struct CUstream_st;
typedef struct CUstream_st* mla_stream_t; /* same type as cudaStream_t */

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,        /* a required pointer is NULL, or a scalar is not finite */
  MLA_ERR_SHAPE = -2,              /* B, T or M out of range, or mask_ld < T */
  MLA_ERR_MISALIGNED = -3,         /* a tensor pointer not 16-byte aligned (mask: 2-byte) */
  MLA_ERR_UNSUPPORTED_DEVICE = -4, /* current device is not compute capability 10.0 */
  MLA_ERR_WORKSPACE = -5,          /* workspace missing or smaller than required */
  MLA_ERR_CUDA = -6,               /* a CUDA runtime/driver call or kernel launch failed */
  MLA_ERR_TIMEOUT = -7             /* a kernel gave up on a bounded internal wait */
} mla_status_t;

/*
 * Workspace bytes of mla_attn_prefill: MLA_WORKSPACE_STATUS_BYTES for the
 * call's status word, plus B * ceil(T/128)^2 bytes for the per-tile mask
 * classes when has_mask != 0. Returns 0 for B < 1 or T < 1.
 */
size_t mla_attn_prefill_workspace_bytes(int B, int T, int has_mask);

/*
 * MLA prefill attention for all 64 heads, heads merged
 * (page "Kimi K2 · Mix and project", excerpt modeling_deepseek.py 799-840:
 * query/key assembly from the non-rotary and rotary parts, scores scaled by
 * softmax_scale, additive mask, fp32 softmax over keys, value mix; plus the
 * transpose/reshape of excerpt 848-852).
 *
 *   q_nope       [B, 64, T, 128]  non-rotary query parts
 *   q_pe         [B, 64, T, 64]   rotary query parts (already rotated)
 *   k_nope       [B, 64, T, 128]  non-rotary key parts
 *   k_pe_shared  [B, 1,  T, 64]   rotary key, one tensor shared by all heads
 *   v            [B, 64, T, 128]  values
 *   mask         [B, 1,  T, mask_ld] additive bf16 mask (entries j < T used),
 *                or NULL for the implicit causal mask (key j allowed iff j <= i).
 *                A non-NULL mask is applied exactly as given, with no extra
 *                causal term; -inf entries exclude a key. A row with no
 *                allowed key produces zeros.
 *   mask_ld      row stride of mask in elements (>= T); ignored when mask is
 *                NULL. Rows are read with 16-byte loads when mask is 16-byte
 *                aligned and mask_ld % 8 == 0, with 2-byte loads otherwise.
 *   B, T         batch (1..65535) and sequence length (1..8388480); keys = queries = T
 *   softmax_scale  multiplies Q.K^T before the mask is added (finite)
 *   workspace    device scratch of mla_attn_prefill_workspace_bytes(B,T,mask!=NULL)
 *                bytes; required with a mask, optional (NULL) without one.
 *                Contents on entry are ignored; the call must not overlap
 *                another call using it. With a workspace, timeouts are
 *                reported in it (mla_last_device_status), without one in the
 *                device-wide word (mla_device_status).
 *   out          [B, T, 8192]: out[b,i,h*128+e], bf16
 */
mla_status_t mla_attn_prefill(const mla_bf16* q_nope, const mla_bf16* q_pe,
                              const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                              const mla_bf16* v, const mla_bf16* mask, int64_t mask_ld, int B,
                              int T, float softmax_scale, void* workspace,
                              size_t workspace_bytes, mla_bf16* out, mla_stream_t stream);

/*
 * Output projection, nn.Linear(8192 -> 7168, bias=False)
 * (page "Kimi K2 · Mix and project", excerpt modeling_deepseek.py 848-852 and
 * the page's parameter table: 8,192 x 7,168 = 58,720,256 weights):
 *
 *   attn  [M, 8192] bf16 (merged heads, row = token)
 *   W_o   [7168, 8192] bf16 (out_features, in_features)
 *   M     rows, 1 .. 2^31 - 129
 *   out   [M, 7168] bf16 = attn . W_o^T, fp32 accumulation, rounded once
 */
mla_status_t mla_o_proj(const mla_bf16* attn, const mla_bf16* W_o, int64_t M, mla_bf16* out,
                        mla_stream_t stream);

/*
 * Workspace bytes mla_attn_oproj needs: MLA_WORKSPACE_STATUS_BYTES for the
 * call's status word, B*T*8192*2 bytes for the merged attention output,
 * rounded up to 256, plus the mask-class bytes when has_mask != 0. Returns 0
 * for B < 1 or T < 1.
 */
size_t mla_attn_oproj_workspace_bytes(int B, int T, int has_mask);

/*
 * Attention followed by o_proj: the whole path of the page
 * "Kimi K2 · Mix and project" from the per-head inputs to Delta_attn.
 * Arguments as in mla_attn_prefill and mla_o_proj; the merged attention output
 * lives in `workspace` (mla_attn_oproj_workspace_bytes bytes, required), and
 *   out   [B, T, 7168] bf16.
 */
mla_status_t mla_attn_oproj(const mla_bf16* q_nope, const mla_bf16* q_pe,
                            const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                            const mla_bf16* v, const mla_bf16* mask, int64_t mask_ld, int B,
                            int T, float softmax_scale, const mla_bf16* W_o, void* workspace,
                            size_t workspace_bytes, mla_bf16* out, mla_stream_t stream);

/*
 * Causal attention with key padding given compactly, as one valid length per
 * sequence instead of a [B,1,T,T] mask (page "Kimi K2 · Transformer blocks",
 * excerpt modeling_deepseek.py 1443-1457: the flash path keeps the 2-D padding
 * mask, the other paths expand it with the causal mask into the 4-D additive
 * form). For right-padded sequences the two forms agree: key j is allowed for
 * query i iff j <= i and j < valid_len[b]. Query rows i >= valid_len[b] still
 * attend to the sequence's valid keys and are written like any other row.
 *
 *   valid_len  device array of B int32 (4-byte aligned), read by the kernel;
 *              values are clamped to [0, T]. A sequence with valid_len 0 has
 *              no allowed key: its rows are zeros.
 * Every other argument as in mla_attn_prefill with mask == NULL (no workspace
 * is needed). NULL valid_len -> MLA_ERR_INVALID_ARG.
 */
mla_status_t mla_attn_prefill_varlen(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                     const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                                     const mla_bf16* v, const int32_t* valid_len, int B, int T,
                                     float softmax_scale, mla_bf16* out, mla_stream_t stream);

/*
 * mla_attn_prefill_varlen followed by o_proj, as mla_attn_oproj; workspace of
 * mla_attn_oproj_workspace_bytes(B, T, 0) bytes.
 */
mla_status_t mla_attn_oproj_varlen(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                   const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                                   const mla_bf16* v, const int32_t* valid_len, int B, int T,
                                   float softmax_scale, const mla_bf16* W_o, void* workspace,
                                   size_t workspace_bytes, mla_bf16* out, mla_stream_t stream);

/*
 * ------------------------------------------------------------ rotary inputs
 * The excerpt rotates the rotary parts right before assembling query and key
 * (page "Kimi K2 · Mix and project", excerpt modeling_deepseek.py 799-840:
 * cos, sin = self.rotary_emb(value_states, ...); q_pe, k_pe =
 * apply_rotary_pos_emb(q_pe, k_pe, cos, sin, position_ids)). The calls below
 * take q_pe and k_pe unrotated and do that step themselves, with the YaRN
 * rotary embedding whose parameters config.json prints (page "Kimi K2 · Block
 * input": rope_theta and rope_scaling). The pages print neither function's
 * body; the library reads them as:
 *  - pair i (i < 32) of a rotary vector, elements 2i and 2i+1, turns as one
 *    complex number by the angle position * inv_freq[i], and both elements
 *    are multiplied by the attention factor f;
 *  - inv_freq[i] = theta^(-i/32) * ((1 - r_i) + r_i / factor), r_i =
 *    clamp((i - lo) / (hi - lo), 0, 1), with lo = floor(d(beta_fast)),
 *    hi = ceil(d(beta_slow)) clamped to [0, 63], d(n) = 64 ln(L / (2 pi n)) /
 *    (2 ln theta), L = original_max_position_embeddings (YaRN's NTK-by-parts
 *    interpolation; hi = lo + 0.001 when they meet). The printed values give
 *    lo = 19, hi = 20: pairs 0..19 keep theta^(-i/32), pairs 20..31 divide it
 *    by 32;
 *  - f = m(factor, mscale) / m(factor, mscale_all_dim), m(s, k) = 1 for
 *    s <= 1, else 0.1 k ln(s) + 1 (exactly 1 for the printed values);
 *  - query and key use the same position_ids.
 * Angles, cos and sin are computed in double precision; the rotated values
 * are rounded once to bf16 before the score MMAs.
 */
typedef struct mla_yarn_rope {
  double rope_theta;                       /* > 1 */
  double factor;                           /* > 0 */
  double original_max_position_embeddings; /* > 0 */
  double beta_fast;                        /* > 0 */
  double beta_slow;                        /* > 0 */
  double mscale;
  double mscale_all_dim;
} mla_yarn_rope_t;

/* The printed configuration's values, as an initializer of mla_yarn_rope_t. */
#define MLA_KIMI_K2_YARN_ROPE {50000.0, 32.0, 4096.0, 1.0, 1.0, 1.0, 1.0}

/*
 * Workspace bytes of mla_attn_prefill_rope: MLA_WORKSPACE_STATUS_BYTES, the
 * rotated key (B*T*64*2) and the cos/sin table (B*T*32*8), each rounded up to
 * 256, plus the mask-class bytes (rounded up to 256) when has_mask != 0.
 * Returns 0 for B < 1 or T < 1.
 */
size_t mla_attn_prefill_rope_workspace_bytes(int B, int T, int has_mask);

/*
 * mla_attn_prefill with unrotated rotary parts:
 *   q_pe          [B, 64, T, 64] rotary query parts before rotation
 *   k_pe          [B, 1, T, 64]  shared rotary key before rotation
 *   position_ids  [B, T] int32 device array (4-byte aligned), the position of
 *                 every token; NULL means 0..T-1 in every sequence. Any int32
 *                 value is used as given.
 *   rope          host pointer to the rotary parameters (read during the
 *                 call only); NULL, a non-finite value or one out of range
 *                 -> MLA_ERR_INVALID_ARG.
 *   workspace     mla_attn_prefill_rope_workspace_bytes(B, T, mask != NULL)
 *                 bytes, required (it holds the rotated key and the table).
 * Every other argument, the layouts and the errors as in mla_attn_prefill.
 * The shared key is rotated once per call by a small pre-pass kernel; each
 * query tile's q_pe is rotated by the attention kernel in shared memory right
 * after its load. With all positions 0 the result equals mla_attn_prefill's
 * on the same inputs, bit for bit.
 */
mla_status_t mla_attn_prefill_rope(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                   const mla_bf16* k_nope, const mla_bf16* k_pe,
                                   const mla_bf16* v, const int32_t* position_ids,
                                   const mla_yarn_rope_t* rope, const mla_bf16* mask,
                                   int64_t mask_ld, int B, int T, float softmax_scale,
                                   void* workspace, size_t workspace_bytes, mla_bf16* out,
                                   mla_stream_t stream);

/*
 * Workspace bytes of mla_attn_oproj_rope: mla_attn_prefill_rope_workspace_bytes
 * plus the merged attention output (B*T*8192*2, rounded up to 256).
 */
size_t mla_attn_oproj_rope_workspace_bytes(int B, int T, int has_mask);

/*
 * mla_attn_prefill_rope followed by o_proj, as mla_attn_oproj:
 *   out [B, T, 7168] bf16.
 */
mla_status_t mla_attn_oproj_rope(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                 const mla_bf16* k_nope, const mla_bf16* k_pe, const mla_bf16* v,
                                 const int32_t* position_ids, const mla_yarn_rope_t* rope,
                                 const mla_bf16* mask, int64_t mask_ld, int B, int T,
                                 float softmax_scale, const mla_bf16* W_o, void* workspace,
                                 size_t workspace_bytes, mla_bf16* out, mla_stream_t stream);

/*
 * ------------------------------------------------------------ KV latent
 * The non-rotary key parts and the values come from each token's compressed
 * KV latent of kv_lora_rank = 512 values (config.json on page "Kimi K2 · Block
 * input"). The pages print only the rank; the library reads the step as one
 * bias-free linear map (attention_bias false) per token,
 *   kv[b,t,:] = c_kv[b,t,:] . W_kv_b^T,   W_kv_b [64 * 256, 512],
 * whose 256 outputs per head h (rows h*256 .. h*256+255 of W_kv_b) are the
 * head's 128 non-rotary key parts followed by its 128 values.
 */
#define MLA_KV_RANK 512

/*
 * Up-projection of the latent into the attention's key and value layouts:
 *   c_kv    [B, T, 512] bf16
 *   W_kv_b  [16384, 512] bf16
 *   k_nope  [B, 64, T, 128] bf16: k_nope[b,h,t,e] = kv[b,t,h*256 + e]
 *   v       [B, 64, T, 128] bf16: v[b,h,t,e]      = kv[b,t,h*256 + 128 + e]
 * fp32 accumulation, each output rounded once. A tcgen05 GEMM with 128 x 256
 * tiles, one head per column tile, whose epilogue writes the two halves of a
 * tile straight into k_nope and v. All pointers 16-byte aligned; B, T as in
 * mla_attn_prefill with B*T <= 2^31 - 129. Timeouts go to the device-wide
 * word (mla_device_status).
 */
mla_status_t mla_kv_up_proj(const mla_bf16* c_kv, const mla_bf16* W_kv_b, int B, int T,
                            mla_bf16* k_nope, mla_bf16* v, mla_stream_t stream);

/*
 * Workspace bytes of mla_attn_oproj_latent: mla_attn_oproj_workspace_bytes
 * plus k_nope and v (B*64*T*128*2 each, rounded up to 256).
 */
size_t mla_attn_oproj_latent_workspace_bytes(int B, int T, int has_mask);

/*
 * The whole path from the latent: mla_kv_up_proj into the workspace, then
 * mla_attn_oproj on its k_nope and v. Arguments as in mla_attn_oproj with
 * c_kv [B, T, 512] and W_kv_b [16384, 512] in place of k_nope and v (same
 * pointer checks), and workspace of mla_attn_oproj_latent_workspace_bytes.
 */
mla_status_t mla_attn_oproj_latent(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                   const mla_bf16* c_kv, const mla_bf16* k_pe_shared,
                                   const mla_bf16* W_kv_b, const mla_bf16* mask, int64_t mask_ld,
                                   int B, int T, float softmax_scale, const mla_bf16* W_o,
                                   void* workspace, size_t workspace_bytes, mla_bf16* out,
                                   mla_stream_t stream);

/* Largest B*T mla_attn_oproj_noalloc accepts (its fixed scratch holds the
 * merged attention output of this many tokens: 64 MiB). */
#define MLA_NOALLOC_MAX_TOKENS 4096

/*
 * mla_attn_oproj without a workspace argument, for callers that cannot
 * allocate device memory at all (for example code running inside a host
 * framework that owns every device allocation, or a plugin that is handed its
 * inputs and outputs and nothing else). The pages have no counterpart of
 * this call; it exists only because of how such callers are built.
 *
 * Arguments, layouts and results are those of mla_attn_oproj minus
 * `workspace`/`workspace_bytes`. The scratch is one fixed device array inside
 * the library (64 MiB + 64 KiB) that every GPU which loads the library holds
 * until the process exits; this call allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine).
 *  - B*T above MLA_NOALLOC_MAX_TOKENS -> MLA_ERR_WORKSPACE (the fixed scratch
 *    is too small); every other error as in mla_attn_oproj.
 *  - The first call on a device looks up the scratch's device address on that
 *    device (cudaGetSymbolAddress, which may load the library's module there):
 *    make that first call before any stream capture.
 *  - All calls share the one scratch array, which keeps the previous call's
 *    contents (nothing in it needs to start at zero). Calls whose GPU work can
 *    overlap -- different streams, or different host threads, on one device --
 *    race on it and must be serialised by the caller.
 */
mla_status_t mla_attn_oproj_noalloc(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                    const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                                    const mla_bf16* v, const mla_bf16* mask, int64_t mask_ld,
                                    int B, int T, float softmax_scale, const mla_bf16* W_o,
                                    mla_bf16* out, mla_stream_t stream);

/*
 * ------------------------------------------------------------ FP8 o_proj
 * The checkpoint stores o_proj as 8-bit floats (page "Kimi K2 · Transformer
 * blocks", configuration excerpt config.json, quantization_config:
 * quant_method fp8, fmt e4m3, activation_scheme dynamic, weight_block_size
 * [128, 128]). The calls below use that format, read as follows:
 *  - codes: e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 *    infinities, largest finite value 448), one byte per element;
 *  - weights: one fp32 scale per 128 x 128 block, W_o ~= value(code) * scale;
 *  - activations ("dynamic"): scales computed at run time, one per token and
 *    per 128-wide group of the 8192 input features;
 *  - a group's scale is amax / 448 in fp32 (1 for a group of zeros) and each
 *    code is the e4m3 value nearest to x / scale computed in fp32, ties to
 *    the even code, saturating at +-448;
 *  - the product: out[m,n] = sum_g a_scale[g][m] * W_scale[n/128][g] *
 *    sum over the group's 128 features of value(a) * value(W), accumulated in
 *    fp32 and rounded once to bf16.
 * Inputs must be finite.
 */

/* Quantisation groups along the 8192 input features, and weight blocks along
 * the 7168 outputs. */
#define MLA_FP8_GROUP 128
#define MLA_FP8_K_GROUPS 64  /* MLA_OPROJ_IN / MLA_FP8_GROUP */
#define MLA_FP8_N_BLOCKS 56  /* MLA_HIDDEN / MLA_FP8_GROUP */

/*
 * Dynamic activation quantisation:
 *   x      [M, 8192] bf16 (row-major, contiguous)
 *   M      rows, 1 .. 2^31 - 129
 *   q      [M, 8192] e4m3 codes (uint8)
 *   scale  [64, M] fp32, group-major: scale[g * M + m] for features
 *          128g .. 128g+127 of row m
 */
mla_status_t mla_quantize_act_fp8(const mla_bf16* x, int64_t M, uint8_t* q, float* scale,
                                  mla_stream_t stream);

/*
 * Block weight quantisation of W_o (done once, like loading a checkpoint):
 *   W      [7168, 8192] bf16 (out_features, in_features)
 *   q      [7168, 8192] e4m3 codes
 *   scale  [56, 64] fp32: scale[nb * 64 + g] for rows 128nb.. and features 128g..
 */
mla_status_t mla_quantize_weight_fp8(const mla_bf16* W, uint8_t* q, float* scale,
                                     mla_stream_t stream);

/*
 * o_proj on e4m3 operands (the product above):
 *   attn_q      [M, 8192] codes, attn_scale [64, M] (from mla_quantize_act_fp8)
 *   W_q         [7168, 8192] codes, W_scale [56, 64] (from mla_quantize_weight_fp8
 *               or a checkpoint in that layout)
 *   M           rows, 1 .. 2^31 - 129
 *   out         [M, 7168] bf16
 * Code pointers and out 16-byte aligned; scale pointers 4-byte aligned.
 */
mla_status_t mla_o_proj_fp8(const uint8_t* attn_q, const float* attn_scale, const uint8_t* W_q,
                            const float* W_scale, int64_t M, mla_bf16* out, mla_stream_t stream);

/*
 * Workspace bytes mla_attn_oproj_fp8 needs: MLA_WORKSPACE_STATUS_BYTES for the
 * call's status word, the merged bf16 attention output (B*T*8192*2), its codes
 * (B*T*8192) and scales (64*B*T*4), each rounded up to 256, plus the
 * mask-class bytes when has_mask != 0. Returns 0 for B < 1 or T < 1.
 */
size_t mla_attn_oproj_fp8_workspace_bytes(int B, int T, int has_mask);

/*
 * mla_attn_oproj with an FP8 o_proj: attention, dynamic quantisation of its
 * merged output, then mla_o_proj_fp8 with the quantised W_o. Arguments as in
 * mla_attn_oproj, with W_q / W_scale in place of W_o.
 */
mla_status_t mla_attn_oproj_fp8(const mla_bf16* q_nope, const mla_bf16* q_pe,
                                const mla_bf16* k_nope, const mla_bf16* k_pe_shared,
                                const mla_bf16* v, const mla_bf16* mask, int64_t mask_ld, int B,
                                int T, float softmax_scale, const uint8_t* W_q,
                                const float* W_scale, void* workspace, size_t workspace_bytes,
                                mla_bf16* out, mla_stream_t stream);

/*
 * Outcome of the last call that used `workspace` (a workspace given to
 * mla_attn_prefill, mla_attn_oproj, mla_attn_oproj_varlen,
 * mla_attn_prefill_rope, mla_attn_oproj_rope, mla_attn_oproj_latent or
 * mla_attn_oproj_fp8; that call
 * must have been enqueued on `stream` or be complete). Synchronises `stream`, then reads the call's status word.
 * Returns MLA_ERR_TIMEOUT if one of that call's kernels gave up on a bounded
 * wait, MLA_ERR_CUDA if the stream reports an error, MLA_ERR_INVALID_ARG for
 * a NULL workspace, MLA_ERR_MISALIGNED for one not 16-byte aligned, else
 * MLA_OK. The word is not cleared (the next call using the workspace clears
 * it). If `detail` is not NULL it receives the raw word (kernel id << 8 | wait
 * site, timeout flag in bit 16; 0 when nothing was recorded).
 */
mla_status_t mla_last_device_status(const void* workspace, mla_stream_t stream,
                                    uint32_t* detail);

/*
 * Synchronises `stream`, then takes the device-wide status word of the
 * current device (the one the calls without a workspace report to): reads and
 * clears it in one atomic step on the device, so a timeout recorded meanwhile
 * by a kernel on another stream is kept for the next read, never lost.
 * Returns MLA_ERR_TIMEOUT if such a kernel gave up on a bounded wait since the
 * word was last taken, MLA_ERR_CUDA if the stream reports an error, else
 * MLA_OK. If `detail` is not NULL it receives the raw word, as above.
 */
mla_status_t mla_device_status(mla_stream_t stream, uint32_t* detail);

/* Static, human-readable name of a status code. */
const char* mla_status_string(mla_status_t status);

/* MLA_ABI_VERSION of the loaded library. */
int mla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H_ */
