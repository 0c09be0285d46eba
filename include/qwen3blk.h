/*
 * libqwen3blk -- forward pass of the Qwen3 decoder block on NVIDIA B200 (sm_100a).
 *
 * The operations follow these pages (title, site; sections named as on the page):
 *   [P-Mini] "从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构" (quarkcode.cn)
 *   [P-MoE]  "从零构建 Qwen-3 MoE" (adg.csdn.net)
 *   [P-Hand] "手搓一个Qwen3" (news.43b.com.cn)
 *   [P-SGL]  "从0实现SGLang 3: Qwen3-0.6B" (wmrh.cn)
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers, allocated and owned by the caller, unless a
 *     parameter says "host". The library never allocates device memory; scratch
 *     space is a caller buffer of qwen3_workspace_size() bytes.
 *   - Every device pointer must be 16-byte aligned (tensor-memory-accelerator
 *     copies); violations return QWEN3_EALIGN before anything is launched.
 *   - bf16 tensors are stored as their 16-bit patterns (qwen3_bf16). Matrices are
 *     row-major. Linear weights are [out_features, in_features] (nn.Linear).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work on it and return; they never synchronise, so they
 *     can be captured in a CUDA graph (argument checks happen at enqueue time).
 *   - Return value: QWEN3_OK (0) or a negative qwen3_status; on error nothing
 *     has been enqueued and qwen3_last_error() names the offending argument.
 *   - Batch and token counts (B, T, rows, n_new) must be at least 1: an empty batch
 *     returns QWEN3_EINVAL rather than doing nothing, and qwen3_workspace_size()
 *     returns 0 for it.
 *   - Conditions only visible on the device (a position beyond the cache, a
 *     token id outside the vocabulary, an expired bounded wait) are recorded in
 *     a device error word; qwen3_check_device_error() reads and clears it.
 *   - Kernels are launched with programmatic dependent launch (each kernel's set-up
 *     overlaps the end of the previous one on the stream) and large prefill GEMMs run
 *     on pairs of CTAs (clusters of 2). The environment variables QWEN3_PDL=0 and
 *     QWEN3_GEMM_PAIR=0, read once per process, turn either off.
 */
#ifndef QWEN3BLK_H
#define QWEN3BLK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t qwen3_bf16;
typedef uint16_t qwen3_f16; /* IEEE binary16 bit pattern */

typedef enum {
  QWEN3_OK = 0,
  QWEN3_EINVAL = -1,     /* null pointer, bad enum, non-positive size */
  QWEN3_ESHAPE = -2,     /* configuration or shape the kernels do not support */
  QWEN3_EALIGN = -3,     /* pointer or leading dimension not 16-byte aligned */
  QWEN3_ECAPACITY = -4,  /* position beyond max_pos or the cache capacity */
  QWEN3_EWORKSPACE = -5, /* workspace smaller than qwen3_workspace_size() */
  QWEN3_ECUDA = -6,      /* CUDA runtime / driver error */
  QWEN3_ETIMEOUT = -7,   /* a device-side bounded wait expired */
  QWEN3_EDEVICE = -8     /* current device is not an sm_100 GPU */
} qwen3_status;

/* Model hyper-parameters ([P-Mini] section 配置文件, table; [P-SGL] section 一). */
typedef struct {
  int hidden;           /* H: 1024 for Qwen3-0.6B; multiple of 256, at most 2048 */
  int n_q_heads;        /* Hq: 16 */
  int n_kv_heads;       /* Hkv: 8; Hq % Hkv == 0 and Hq/Hkv in {1, 2, 4, 8, 16} */
  int head_dim;         /* D: must be 128 */
  int intermediate;     /* I: 3072 (dense SwiGLU); multiple of 64 */
  int vocab;            /* V: 151936; multiple of 32 */
  int n_layers;         /* 28 */
  int max_pos;          /* 40960: RoPE table rows */
  int n_experts;        /* E: MoE experts (0 = dense model) */
  int top_k;            /* experts per token (top_k <= n_experts <= 256) */
  int moe_intermediate; /* Im: per-expert SwiGLU width; multiple of 64 */
  int norm_topk_prob;   /* 1: renormalise the top-k probabilities to sum 1 */
  float rms_eps;        /* 1e-6 */
  double rope_theta;    /* 1e6 */
  /* Operand type of the linear layers (projections, router, experts, tied LM head):
   *   0: bf16, the pages' model dtype ([P-Mini] section RMSNorm: the model body is bf16);
   *   1: fp16. Every bf16 weight converts to fp16 exactly for magnitudes in
   *      [2^-17, 65504] (qwen3_convert_to_f16; below, within 2^-25), so the weights keep
   *      their values, while the activations fed to the projections round to 11
   *      significant bits instead of 8 -- at the same tensor-core rate. The linear
   *      weights (w_qkv, w_o, w_gate_up, w_down, router, moe_gate_up, moe_down) and the
   *      embedding / LM head must then hold fp16; norm weights stay bf16. Activations
   *      entering a projection must stay within +-65504 (larger ones become inf).
   * The KV cache, q and the softmax probabilities stay bf16 in both modes. */
  int gemm_f16;
} qwen3_config;

/* One layer's weights in the library's packed layouts (see the pack helpers).
 * Unused members (the FFN kind not present) may be NULL. */
typedef struct {
  const qwen3_bf16* in_norm;     /* [H] input_layernorm */
  const qwen3_bf16* w_qkv;       /* [(Hq+2*Hkv)*D, H]: q_proj rows, then k_proj, then v_proj */
  const qwen3_bf16* q_norm;      /* [D] per-head RMSNorm of q, shared by all heads */
  const qwen3_bf16* k_norm;      /* [D] per-head RMSNorm of k */
  const qwen3_bf16* w_o;         /* [H, Hq*D] o_proj */
  const qwen3_bf16* post_norm;   /* [H] post_attention_layernorm */
  const qwen3_bf16* w_gate_up;   /* [2I, H] gate/up interleaved in 16-row blocks */
  const qwen3_bf16* w_down;      /* [H, I] down_proj */
  const qwen3_bf16* router;      /* [E, H] MoE gate (router) */
  const qwen3_bf16* moe_gate_up; /* [E, 2Im, H], each expert interleaved in 16-row blocks */
  const qwen3_bf16* moe_down;    /* [E, H, Im] */
} qwen3_layer_weights;

/* One layer's KV cache: k and v are [B][Hkv][s_max][D] bf16. Keys are stored
 * after the per-head QK RMSNorm and RoPE ([P-Mini] section GQA). */
typedef struct {
  qwen3_bf16* k;
  qwen3_bf16* v;
  int s_max;
} qwen3_kv_layer;

typedef enum {
  QWEN3_OP_BLOCK_PREFILL = 1,
  QWEN3_OP_BLOCK_DECODE = 2,
  QWEN3_OP_MOE_BLOCK = 3,
  QWEN3_OP_STACK_PREFILL = 4,
  QWEN3_OP_STACK_DECODE = 5,
  QWEN3_OP_GENERATE = 6  /* qwen3_generate_greedy: T = prompt length */
} qwen3_op;

typedef enum { QWEN3_MODE_PREFILL = 0, QWEN3_MODE_DECODE = 1 } qwen3_mode;

/* ---------------------------------------------------------------- utilities */

/* Thread-local message describing the last error of this thread ("" if none). */
const char* qwen3_last_error(void);
const char* qwen3_status_string(int status);

/* Fills *cfg (host) with the Qwen3-0.6B dense configuration ([P-Mini] table). */
int qwen3_config_qwen3_0_6b(qwen3_config* cfg);

/* Checks a configuration against what the kernels support (QWEN3_ESHAPE otherwise). */
int qwen3_validate_config(const qwen3_config* cfg);

/* Bytes of the RoPE table: max_pos * 64 * 2 floats. */
size_t qwen3_rope_table_bytes(const qwen3_config* cfg);

/* RoPE table ([P-Mini] section RoPE: theta_i = theta^(-2i/D), angle = m * theta_i,
 * dimension i paired with i + D/2). Computed on the host in double precision and
 * rounded to fp32, layout [max_pos][D/2][2] = (cos, sin). Copies into the device
 * buffer `rope` on `stream` and waits for that copy (a set-up call: not for capture). */
int qwen3_rope_table(const qwen3_config* cfg, float* rope, void* stream);

/* Scratch bytes needed by `op` for B sequences of T new tokens each, with KV
 * caches of capacity s_max (decode: T is ignored and taken as 1). */
size_t qwen3_workspace_size(const qwen3_config* cfg, int op, int B, int T, int s_max);

/* Converts n bf16 values to fp16 (round to nearest even; exact for magnitudes in
 * [2^-17, 65504]), e.g. a packed weight matrix for the gemm_f16 mode. in == out converts
 * in place. Asynchronous on `stream`. */
int qwen3_convert_to_f16(const qwen3_bf16* in, qwen3_f16* out, size_t n, void* stream);

/* Packs q/k/v_proj ([Hq*D,H], [Hkv*D,H], [Hkv*D,H]) into w_qkv (concatenated rows). */
int qwen3_pack_qkv(const qwen3_config* cfg, const qwen3_bf16* wq, const qwen3_bf16* wk, const qwen3_bf16* wv,
                   qwen3_bf16* w_qkv, void* stream);

/* Packs gate_proj and up_proj (each [I, H]) into w_gate_up [2I, H]: rows 32j..32j+15 are
 * gate rows 16j..16j+15 and rows 32j+16..32j+31 the matching up rows. */
int qwen3_pack_gate_up(int I, int H, const qwen3_bf16* w_gate, const qwen3_bf16* w_up, qwen3_bf16* w_gate_up,
                       void* stream);

/* Packs the fused expert weights gate_up_proj [E, 2Im, H] ([P-Mini] section MoE: chunk(2)
 * gives gate first, then up) into the same 16-row interleave per expert. */
int qwen3_pack_moe_gate_up(int E, int Im, int H, const qwen3_bf16* gate_up_proj, qwen3_bf16* out, void* stream);

/* Block kinds for qwen3_check_layer_weights. */
typedef enum { QWEN3_LAYER_DENSE = 0, QWEN3_LAYER_MOE = 1 } qwen3_layer_kind;

/* Two-way check of one layer's weight pointers for a block kind, on the host (reads no
 * device memory; a set-up call). It restates for raw pointers the two-way check the
 * pages run when they load weights ("从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构",
 * section 加载官方权重：名字映射与双重校验: every expected tensor present with its
 * shape, every model parameter covered):
 *   - every member the kind reads is non-NULL (QWEN3_EINVAL) and 16-byte aligned
 *     (QWEN3_EALIGN);
 *   - every member the kind does not read is NULL (QWEN3_ESHAPE), so that a layer built
 *     for the other kind, or a config of the wrong kind, is reported;
 *   - with each member's size from cfg, no two members overlap (QWEN3_EINVAL), which is
 *     what an offset into one weight arena computed with a wrong dimension produces;
 *     the same pointer for two members of equal size (a shared read-only buffer) is
 *     allowed.
 * qwen3_last_error() names the member(s). The block calls check only the first
 * point, so a struct that also carries the other kind's members stays usable there. */
int qwen3_check_layer_weights(const qwen3_config* cfg, const qwen3_layer_weights* w, int kind);

/* Synchronises `stream`, then returns and clears the device error word
 * (QWEN3_OK, QWEN3_ECAPACITY, QWEN3_EINVAL or QWEN3_ETIMEOUT). */
int qwen3_check_device_error(void* stream);

/* Per-launch timing of the block and stack calls. After qwen3_profile_begin(n), each
 * kernel launch (up to n) is bracketed by two CUDA events on the call's stream;
 * qwen3_profile_end(stream) stops recording, synchronises the stream and returns the
 * number of records; qwen3_profile_record(i, ...) gives the i-th launch's role name
 * (e.g. "gemm_qkv", "attn_prefill", "lm_head") and its device time in ms.
 * The recorder is process-global: profile one thread's calls at a time. */
int qwen3_profile_begin(int max_records);
int qwen3_profile_end(void* stream);
int qwen3_profile_record(int i, char* name, int name_cap, float* ms);

/* -------------------------------------------------------------- block calls */

/* Dense decoder block, prefill ([P-Mini] section TransformerBlock: pre-norm, GQA with
 * QK-norm and RoPE, o_proj + residual, norm, SwiGLU FFN + residual).
 *   x          [B*T, H] bf16, updated in place (sequence b occupies rows b*T..b*T+T-1)
 *   start_pos  [B] int32 (device): token t of sequence b is at position start_pos[b]+t;
 *              it attends to cache positions 0..start_pos[b]+t, which must already hold
 *              the earlier tokens (chunked prefill) -- this call writes positions
 *              start_pos[b]..start_pos[b]+T-1 of kv.
 *   kv         host pointer to the layer's cache descriptor
 *   rope       qwen3_rope_table() output
 *   ws         workspace of qwen3_workspace_size(cfg, QWEN3_OP_BLOCK_PREFILL, B, T, kv->s_max) */
int qwen3_block_prefill(const qwen3_config* cfg, const qwen3_layer_weights* w, qwen3_bf16* x, int B, int T,
                        const int* start_pos, const qwen3_kv_layer* kv, const float* rope, void* ws,
                        size_t ws_bytes, void* stream);

/* Dense decoder block, one decode step per sequence ([P-Mini] section prefill 与 decode):
 *   x          [B, H] bf16, updated in place
 *   cache_len  [B] int32 (device): the new token is at position cache_len[b], is appended to
 *              kv at that position and attends to positions 0..cache_len[b] (itself included).
 *              cache_len is not modified (qwen3_stack_forward advances it). */
int qwen3_block_decode(const qwen3_config* cfg, const qwen3_layer_weights* w, qwen3_bf16* x, int B,
                       const int* cache_len, const qwen3_kv_layer* kv, const float* rope, void* ws,
                       size_t ws_bytes, void* stream);

/* MoE decoder block, prefill: attention half as qwen3_block_prefill, then the top-k
 * router FFN ([P-Mini] section MoE: fp32 softmax over the router logits, top-k by
 * descending probability (ties: lower expert index first), renormalised when
 * norm_topk_prob; each selected expert's SwiGLU output scaled by its weight and summed
 * in slot order). Optional outputs (may be NULL):
 *   topk_idx [B*T, k] int32, topk_w [B*T, k] fp32,
 *   expert_offsets [E+1] int32 (rows of each expert in the permuted order),
 *   perm_token [B*T*k] int32 (token of each permuted row: expert ascending, then token). */
int qwen3_moe_block(const qwen3_config* cfg, const qwen3_layer_weights* w, qwen3_bf16* x, int B, int T,
                    const int* start_pos, const qwen3_kv_layer* kv, const float* rope, int* topk_idx,
                    float* topk_w, int* expert_offsets, int* perm_token, void* ws, size_t ws_bytes, void* stream);

/* The n_layers-deep dense stack with final RMSNorm and tied LM head ([P-Mini] section
 * 骨架; [P-SGL] section 一: tie_word_embeddings).
 *   embed       [V, H] bf16, also the LM head
 *   layers      host array of n_layers weight descriptors
 *   ids         [B*T] int32 (decode: [B])
 *   mode        QWEN3_MODE_PREFILL: pos_or_len = start positions [B] (as block_prefill);
 *               QWEN3_MODE_DECODE: T must be 1, pos_or_len = cache lengths [B] (as
 *               block_decode) and is advanced by one on the device after the step.
 *   kv          host array of n_layers cache descriptors
 *   logits      fp32: [B*T, V], or [B, V] (last position of each sequence) if last_only
 *   The residual stream between layers is kept in fp32 inside the workspace. */
int qwen3_stack_forward(const qwen3_config* cfg, const qwen3_bf16* embed, const qwen3_layer_weights* layers,
                        const qwen3_bf16* final_norm, const int* ids, int B, int T, int mode, int* pos_or_len,
                        const qwen3_kv_layer* kv, const float* rope, float* logits, int last_only, void* ws,
                        size_t ws_bytes, void* stream);

/* Greedy generation: the prompt runs as one prefill of the stack, then one decode step
 * per further token ([P-Mini] section prefill 与 decode; [P-MoE] last-position logits),
 * every token chosen as the argmax of the fp32 logits (ties: lower id).
 *   prompt_ids  [B*T] int32 (device), sequence b at rows b*T..b*T+T-1, positions 0..T-1
 *   n_new       new tokens per sequence (>= 1): token 0 from the prompt's last logits,
 *               token s (s >= 1) from a decode step at position T+s-1 fed token s-1
 *   kv          host array of n_layers cache descriptors, s_max >= T + n_new - 1;
 *               positions 0..T+n_new-2 are written
 *   out_ids     [B, n_new] int32 (device)
 *   ws          qwen3_workspace_size(cfg, QWEN3_OP_GENERATE, B, T, s_max) bytes; it also holds
 *               the [B, V] fp32 logits of the current step and the cache lengths.
 * Everything is enqueued on `stream` (one stack prefill, n_new - 1 stack decode steps and
 * an argmax after each); the caller may capture the whole call in a CUDA graph. */
int qwen3_generate_greedy(const qwen3_config* cfg, const qwen3_bf16* embed, const qwen3_layer_weights* layers,
                          const qwen3_bf16* final_norm, const int* prompt_ids, int B, int T, int n_new,
                          const qwen3_kv_layer* kv, const float* rope, int* out_ids, void* ws, size_t ws_bytes,
                          void* stream);

/* ------------------------------------------------ single kernels (ops) */

/* out[r] = x[r] * rsqrt(mean(x[r]^2) + eps) * w  ([P-Mini] section RMSNorm formula).
 * x bf16 or fp32 (x_f32 = 1), row stride ldx elements; out bf16 (out_f16 = 0) or fp16
 * (out_f16 = 1, the projections' operand type of the gemm_f16 mode) with stride ldo;
 * n % 256 == 0 and n <= 2048. */
int qwen3_op_rmsnorm(const void* x, int x_f32, long long ldx, const qwen3_bf16* w, qwen3_bf16* out, long long ldo,
                     int rows, int n, float eps, int out_f16, void* stream);

/* Linear layer on the tensor cores: out = epilogue(A . W^T), A [M, K] (lda), W [N, K] (ldw).
 *   epilogue 0: out = acc;  1: out = resid + acc (resid may alias out);
 *            2: SwiGLU -- W rows interleaved as qwen3_pack_gate_up, out [M, N/2] bf16.
 *   out_f32 / resid_f32 select fp32 (else bf16). swap: 1 = weight rows on the MMA's 128-row
 *   side (small M), 0 = activations there, 2 = weight rows on the 128-row side with K split
 *   over the CTAs of a thread-block cluster and summed in the same kernel (M <= 64,
 *   N % 128 == 0; ws unused), 3 = as 2 with A holding 2M rows: row t = hi(a_t) and row M + t
 *   = lo(a_t) = a_t - hi(a_t) rounded to the operand type, the product taken on hi + lo
 *   (about twice the operand type's significant bits; the decode path's operand form),
 *   -1 = automatic (2 when it applies, else 1 when M <= 256).
 *   ws (may be NULL): scratch for split-K when the output has too few tiles to fill the GPU;
 *   it holds fp32 partials, up to ws_bytes (split count = largest that fits).
 *   ab_f16: A and W hold fp16 (1) or bf16 (0); the SwiGLU output takes the same type.
 *   K % 64 == 0, N % 32 == 0, leading dimensions multiples of 8 elements. */
int qwen3_op_gemm(const qwen3_bf16* A, long long lda, const qwen3_bf16* W, long long ldw, void* out, long long ldo,
                  int M, int N, int K, int epilogue, const void* resid, long long ldr, int resid_f32, int out_f32,
                  int swap, int ab_f16, void* ws, size_t ws_bytes, void* stream);

/* Per-head QK RMSNorm + rotate-half RoPE + KV-cache write (see qwen3_block_prefill for
 * positions). qkv [B*T, (Hq+2Hkv)*D] (row stride ldqkv): q heads are normalised and rotated
 * in place; k heads (normalised, rotated) and v heads are written to kv at their positions. */
int qwen3_op_qk_norm_rope(const qwen3_config* cfg, qwen3_bf16* qkv, long long ldqkv, int B, int T,
                          const int* pos_base, const qwen3_bf16* q_norm, const qwen3_bf16* k_norm,
                          const qwen3_kv_layer* kv, const float* rope, void* stream);

/* The prefill QKV projection with the QK-norm/RoPE/KV-write step fused into its epilogue
 * (the form qwen3_block_prefill uses): acc = h . w_qkv^T in fp32; q heads are normalised,
 * rotated and written to qkv [B*T, (Hq+2Hkv)*D] (bf16, same columns); k heads (normalised,
 * rotated) and v heads go straight to kv at their positions. The k/v columns of qkv are not
 * written. h [B*T, H] bf16; positions as qwen3_op_qk_norm_rope. */
int qwen3_op_gemm_qkv_rope(const qwen3_config* cfg, const qwen3_bf16* h, const qwen3_bf16* w_qkv, qwen3_bf16* qkv,
                           int B, int T, const int* pos_base, const qwen3_bf16* q_norm, const qwen3_bf16* k_norm,
                           const qwen3_kv_layer* kv, const float* rope, void* stream);

/* Causal GQA prefill attention: queries from qkv (already normed/rotated q heads), keys and
 * values from kv positions 0..start_pos[b]+t; o [B*T, Hq*D] (stride ldo), head-major columns,
 * bf16 (fp16 when cfg->gemm_f16: o is the input of the o_proj projection). */
int qwen3_op_attention_prefill(const qwen3_config* cfg, const qwen3_bf16* qkv, long long ldqkv, int B, int T,
                               const int* start_pos, const qwen3_kv_layer* kv, qwen3_bf16* o, long long ldo,
                               void* stream);

/* Decode attention for one query per sequence at position cache_len[b] over kv positions
 * 0..cache_len[b] ("从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构", sections GQA and
 * prefill 与 decode). qkv: [B][ldqkv] bf16 with the Hq query heads (post-norm, post-RoPE)
 * at its start; ldqkv a multiple of 8 and >= Hq*128. The 128-key tiles of all (sequence,
 * KV group) rows are divided evenly among the SMs; a row shared by several SMs leaves
 * (max, sum, unnormalised output) partials in ws that the row's first SM merges with
 * log-sum-exp weights. ws also holds the call's tile plan and per-row merge counters
 * (qwen3_workspace_size(cfg, QWEN3_OP_BLOCK_DECODE, B, 1, s_max) suffices; the size does
 * not depend on s_max). Hq / Hkv must be 1, 2, 4, 8 or 16. A position past the cache
 * (cache_len[b] >= s_max) is reported by the device as QWEN3_ECAPACITY, a negative one as
 * QWEN3_EINVAL; that sequence's output row is not written. o is bf16, or fp16 when
 * cfg->gemm_f16 (as qwen3_op_attention_prefill); ldo a multiple of 8 and >= Hq*128. */
int qwen3_op_attention_decode(const qwen3_config* cfg, const qwen3_bf16* qkv, long long ldqkv, int B,
                              const int* cache_len, const qwen3_kv_layer* kv, qwen3_bf16* o, long long ldo,
                              void* ws, size_t ws_bytes, void* stream);

/* Decode attention exactly as qwen3_op_attention_decode, for callers that cannot allocate
 * device memory (for example a host application given a fixed memory budget, or a plugin
 * that is handed tensors but no allocator or workspace). The pages have no counterpart:
 * this entry point exists for such callers only.
 * Instead of a caller workspace, the partials, tile plan and merge counters live in a static
 * device array of this library, 12 MiB on every GPU that loads the library (held until
 * the process exits). Limit: (B * Hkv + 256) * G * 130 * 4 bytes of partials plus
 * (B + 4 + B * Hkv) * 4 bytes must fit (G = Hq / Hkv; B up to 1250 for 16 query heads in
 * 8 groups, whatever s_max); larger sizes return QWEN3_EWORKSPACE with the numbers in
 * qwen3_last_error().
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture. The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 * All calls share the one array: calls that overlap on the GPU (other streams, other
 * threads) race and must be serialised by the caller. Each call writes its plan and clears
 * its merge counters before use, and every partial it reads is written by that same call, so
 * nothing needs clearing between calls. */
int qwen3_op_attention_decode_noalloc(const qwen3_config* cfg, const qwen3_bf16* qkv, long long ldqkv, int B,
                                      const int* cache_len, const qwen3_kv_layer* kv, qwen3_bf16* o, long long ldo,
                                      void* stream);

/* out[r * ld_out] = argmax_j x[r * ldx + j], j < V (fp32 logits; ties: lower index; NaN
 * never chosen). V % 4 == 0, x and ldx 16-byte aligned in bytes. */
int qwen3_op_argmax(const float* x, long long ldx, int rows, int V, int* out, long long ld_out, void* stream);

/* out[m] = embed[ids[m]] ([P-MoE] section 5). embed holds bf16, or fp16 (embed_f16 = 1, the
 * gemm_f16 mode's tied embedding); out is fp32 (out_f32 = 1, exact widening) or a copy in
 * embed's own type. */
int qwen3_op_embed(const int* ids, int n, const qwen3_bf16* embed, int vocab, int H, void* out, int out_f32,
                   int embed_f16, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QWEN3BLK_H */
