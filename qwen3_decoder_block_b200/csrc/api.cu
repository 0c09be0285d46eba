// C ABI of libqwen3blk: argument validation, workspace carving and the kernel
// sequences of the block, MoE block and stack calls. Host code only launches
// kernels on the caller's stream; it never allocates device memory.
//
// Pages cited:
//   [P-Mini] "从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构" (quarkcode.cn)
//   [P-Hand] "手搓一个Qwen3" (news.43b.com.cn)
//   [P-SGL]  "从0实现SGLang 3: Qwen3-0.6B" (wmrh.cn)
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>
#include "../../include/qwen3blk.h"
#include "common.cuh"
#include "internal.h"

namespace q3 {

int launch_rmsnorm(const void* x, bool x_f32, long long ldx, const uint16_t* w, uint16_t* out, long long ldo,
                   int rows, int n, float eps, cudaStream_t s, int* zero_word = nullptr, bool out_f16 = false,
                   long long out_lo = 0, float* r_out = nullptr);
int launch_qk_norm_rope(uint16_t* qkv, long long ldqkv, int B, int T, int Hq, int Hkv, const int* pos_base,
                        const uint16_t* qw, const uint16_t* kw, const float* rope, uint16_t* ck, uint16_t* cv,
                        int s_max, int max_pos, float eps, int* err, cudaStream_t s);
int launch_embed(const int* ids, int n, const uint16_t* E, int vocab, int H, void* out, bool out_f32, int* err,
                 cudaStream_t s, int* zero_word = nullptr, bool e_f16 = false);
int launch_convert_to_f16(const uint16_t* in, uint16_t* out, long long n, cudaStream_t s);
int launch_pack_gate_up(const uint16_t* gate, const uint16_t* up, long long mat_stride, int n_mats, int I, int H,
                        uint16_t* out, cudaStream_t s);
int launch_advance_lengths(int* len, int B, cudaStream_t s);
int launch_argmax_rows(const float* x, long long ldx, int rows, int V, int* out, long long ld_out, int* next,
                       cudaStream_t s);
int launch_fill_lengths(int* len, int B, int value, cudaStream_t s);
int launch_attention_prefill(const uint16_t* qkv, long long ldqkv, int B, int T, int Hq, int Hkv,
                             const int* start_pos, const uint16_t* ck, const uint16_t* cv, int s_max, uint16_t* out,
                             long long ldo, int* err, cudaStream_t s, bool o_f16 = false);
int launch_attention_decode(const uint16_t* qkv, long long ldqkv, int B, int Hq, int Hkv, const int* cache_len,
                            const uint16_t* ck, const uint16_t* cv, int s_max, float* scratch, uint16_t* out,
                            long long ldo, int* err, cudaStream_t s, bool o_f16 = false, bool q_hilo = false,
                            long long o_lo = 0, bool plan_ready = false);
size_t decode_partial_bytes(int B, int Hq, int Hkv);
int launch_attention_decode_static(const uint16_t* qkv, long long ldqkv, int B, int Hq, int Hkv,
                                   const int* cache_len, const uint16_t* ck, const uint16_t* cv, int s_max,
                                   uint16_t* out, long long ldo, int* err, cudaStream_t s, bool o_f16 = false);
int launch_moe_route(const float* logits, int T, int E, int k, int renorm, int* idx, float* w, int* counts,
                     cudaStream_t s);
int launch_moe_permute(const int* idx, int T, int k, int E, const int* counts, int* offsets, int* perm_token,
                       int* perm_slot, int* inv_pos, const uint16_t* h, int H, uint16_t* a_perm, cudaStream_t s);
int launch_moe_combine(const float* x1, const uint16_t* Y, const float* w, const int* inv_pos, int T, int k, int H,
                       void* out, bool out_f32, cudaStream_t s);

// ----------------------------------------------------------------------------- errors
static thread_local std::string g_last_error;

void set_last_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

// The device error word (first failure wins; cleared by qwen3_check_device_error).
__device__ int g_device_error;

static int g_sm_count[64];
static int* g_err_ptr[64];
static std::mutex g_dev_mu;

static int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d < 0 || d >= 64 ? 0 : d;
}

int num_sms() {
  const int d = current_device();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_sm_count[d] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    g_sm_count[d] = n > 0 ? n : 148;
  }
  return g_sm_count[d];
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("QWEN3_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Large plain GEMMs on CTA pairs; QWEN3_GEMM_PAIR=0 keeps every GEMM on single CTAs.
bool gemm_pair_enabled() {
  static const bool on = [] {
    const char* e = getenv("QWEN3_GEMM_PAIR");
    return !(e && e[0] == '0');
  }();
  return on;
}

// The dynamic shared-memory limit of a kernel is a per-device setting: raise it once
// per (kernel, device), under the lock, and report a failure instead of launching.
int ensure_smem_attr(const void* func, int bytes, bool* first) {
  const int d = current_device();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  static std::vector<std::pair<const void*, int>> done;
  if (first) *first = false;
  for (const auto& e : done)
    if (e.first == func && e.second == d) return 0;
  const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    set_last_error("cannot raise a kernel's shared memory to %d bytes on device %d: %s", bytes, d,
                   cudaGetErrorString(e));
    return -6;
  }
  done.emplace_back(func, d);
  if (first) *first = true;
  return 0;
}

int* device_error_word() {
  const int d = current_device();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_err_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) g_err_ptr[d] = static_cast<int*>(p);
  }
  return g_err_ptr[d];
}

// ----------------------------------------------------------------------------- profiling
// Optional per-launch timing: while enabled, every kernel launch made by the
// block/stack calls is bracketed by two CUDA events on the caller's stream.
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
static std::vector<ProfRec> g_prof;
static size_t g_prof_used = 0;
static bool g_prof_on = false;

struct ProfScope {
  ProfRec* r = nullptr;
  cudaStream_t s;
  ProfScope(const char* name, cudaStream_t st) : s(st) {
    if (!g_prof_on || g_prof_used >= g_prof.size()) return;
    r = &g_prof[g_prof_used++];
    r->name = name;
    cudaEventRecord(r->a, s);
  }
  ~ProfScope() {
    if (r) cudaEventRecord(r->b, s);
  }
};

// ----------------------------------------------------------------------------- validation
#define Q3_CHECK(cond, code, ...)  \
  do {                             \
    if (!(cond)) {                 \
      set_last_error(__VA_ARGS__); \
      return (code);               \
    }                              \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_device() {
  static bool ok[64] = {false};
  const int d = current_device();
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (ok[d]) return 0;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, d) != cudaSuccess) {
    set_last_error("no CUDA device available");
    return QWEN3_EDEVICE;
  }
  if (prop.major != 10) {
    set_last_error("device %d is sm_%d%d; libqwen3blk needs an sm_100 (B200) GPU", d, prop.major, prop.minor);
    return QWEN3_EDEVICE;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  ok[d] = true;
  return 0;
}

static int validate_cfg(const qwen3_config* c) {
  Q3_CHECK(c, QWEN3_EINVAL, "cfg is NULL");
  Q3_CHECK(c->head_dim == 128, QWEN3_ESHAPE, "head_dim must be 128 (got %d)", c->head_dim);
  Q3_CHECK(c->n_q_heads > 0 && c->n_kv_heads > 0, QWEN3_ESHAPE, "head counts must be positive");
  // [P-Hand] section GroupedQueryAttention: num_heads must be divisible by the number of KV groups
  Q3_CHECK(c->n_q_heads % c->n_kv_heads == 0, QWEN3_ESHAPE, "n_q_heads (%d) %% n_kv_heads (%d) != 0", c->n_q_heads,
           c->n_kv_heads);
  // a 128-row attention tile packs 128 / G tokens of one KV group; the decode kernel is
  // instantiated for G up to 16, the largest group of the Qwen3 family's GQA configs
  const int G = c->n_q_heads / c->n_kv_heads;
  Q3_CHECK(G == 1 || G == 2 || G == 4 || G == 8 || G == 16, QWEN3_ESHAPE,
           "query heads per KV group (%d) must be 1, 2, 4, 8 or 16", G);
  Q3_CHECK(c->hidden > 0 && c->hidden % 256 == 0 && c->hidden <= 2048, QWEN3_ESHAPE,
           "hidden (%d) must be a multiple of 256 and at most 2048", c->hidden);
  Q3_CHECK(c->max_pos > 0, QWEN3_ESHAPE, "max_pos must be positive");
  Q3_CHECK(c->rms_eps >= 0.f, QWEN3_ESHAPE, "rms_eps must be non-negative");
  if (c->intermediate > 0)
    Q3_CHECK(c->intermediate % 64 == 0, QWEN3_ESHAPE, "intermediate (%d) must be a multiple of 64", c->intermediate);
  if (c->vocab > 0) Q3_CHECK(c->vocab % 32 == 0, QWEN3_ESHAPE, "vocab (%d) must be a multiple of 32", c->vocab);
  Q3_CHECK(c->gemm_f16 == 0 || c->gemm_f16 == 1, QWEN3_ESHAPE, "gemm_f16 must be 0 or 1 (got %d)", c->gemm_f16);
  if (c->n_experts > 0) {
    Q3_CHECK(c->n_experts <= 256 && c->n_experts % 32 == 0, QWEN3_ESHAPE,
             "n_experts (%d) must be a multiple of 32 and at most 256", c->n_experts);
    Q3_CHECK(c->top_k >= 1 && c->top_k <= c->n_experts && c->top_k <= 32, QWEN3_ESHAPE,
             "top_k (%d) must be in [1, min(n_experts, 32)]", c->top_k);
    Q3_CHECK(c->moe_intermediate > 0 && c->moe_intermediate % 64 == 0, QWEN3_ESHAPE,
             "moe_intermediate (%d) must be a positive multiple of 64", c->moe_intermediate);
  }
  return 0;
}

// ----------------------------------------------------------------------------- workspace
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t count) {
    used = (used + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
};

struct Buffers {
  uint16_t* h = nullptr;     // [M, H] normed activations
  uint16_t* qkv = nullptr;   // [M, Nqkv]
  uint16_t* q2 = nullptr;    // [M, 2*Hq*D] decode: q as hi/lo bf16 rows per KV group
  uint16_t* o = nullptr;     // [M, Hq*D]
  float* x1 = nullptr;       // [M, H] residual after attention (fp32)
  uint16_t* act = nullptr;   // [M, I] SwiGLU output
  float* part = nullptr;     // decode attention scratch (partials, tile plan, merge counters)
  bool plan_ready = false;   // part holds this call's decode tile plan (same lengths for every layer)
  float* gpart = nullptr;    // split-K partials of small-M GEMMs
  // MoE
  float* logits = nullptr;   // [M, E]
  int* idx = nullptr;        // [M, k]
  float* w = nullptr;        // [M, k]
  int* counts = nullptr;     // [E]
  int* offsets = nullptr;    // [E+1]
  int* perm_token = nullptr; // [M*k]
  int* perm_slot = nullptr;  // [M*k]
  int* inv_pos = nullptr;    // [M*k]
  uint16_t* a_perm = nullptr;   // [M*k, H]
  uint16_t* act_perm = nullptr; // [M*k, Im]
  uint16_t* y = nullptr;        // [M*k, H]
  // stack
  float* xs = nullptr;       // [M, H] fp32 residual stream
  uint16_t* hf = nullptr;    // [rows, H] final-normed
  // grid barrier of the decode-sized projections' fused RMSNorm: [0] zeroed by the first
  // kernel of every call and left at zero by every launch that uses it, [1] a generation
  int* ticket = nullptr;
  float* ssq = nullptr;      // the fused RMSNorm's per-tile sums of squares [H / 128][64]
  // decode-sized calls: 1/rms per token of the residual stream before (rs_x) and after
  // (rs_x1) the attention sub-block, and whether b.h holds a deferred norm's output
  // (y = x * w * s_t, to be rescaled by the projection that reads it)
  float* rs_x = nullptr;     // [64]
  float* rs_x1 = nullptr;    // [64]
  bool h_deferred = false;   // b.h as the block's input norm (QKV side)
  bool h2_deferred = false;  // b.h as the post-attention norm (gate/up side)
};

static size_t carve(const qwen3_config& c, int op, int B, int T, int s_max, void* ws, Buffers* out) {
  Carver cv(ws);
  Buffers b;
  const bool decode = op == QWEN3_OP_BLOCK_DECODE || op == QWEN3_OP_STACK_DECODE;
  const long long M = (long long)B * (decode ? 1 : T);
  const int D = c.head_dim, H = c.hidden;
  const long long nqkv = (long long)(c.n_q_heads + 2 * c.n_kv_heads) * D;
  // decode-sized calls carry projection inputs as hi/lo rows: twice the rows
  const long long Mh = M <= 64 ? 2 * M : M;
  b.h = cv.take<uint16_t>(Mh * H);
  b.qkv = cv.take<uint16_t>(M * nqkv);
  b.o = cv.take<uint16_t>(Mh * c.n_q_heads * D);
  b.x1 = cv.take<float>(M * H);
  // one new token per sequence (decode, or a prefill of T = 1) runs the decode attention
  if (decode || T == 1) {
    b.part = cv.take<float>(decode_partial_bytes(B, c.n_q_heads, c.n_kv_heads) / sizeof(float));
    b.q2 = cv.take<uint16_t>(M * 2 * c.n_q_heads * D);
  }
  if (M <= 256) b.gpart = cv.take<float>(kSplitKBytes / sizeof(float));
  if (op == QWEN3_OP_MOE_BLOCK) {
    const int E = c.n_experts, k = c.top_k;
    b.logits = cv.take<float>(M * E);
    b.idx = cv.take<int>(M * k);
    b.w = cv.take<float>(M * k);
    b.counts = cv.take<int>(E);
    b.offsets = cv.take<int>(E + 1);
    b.perm_token = cv.take<int>(M * k);
    b.perm_slot = cv.take<int>(M * k);
    b.inv_pos = cv.take<int>(M * k);
    b.a_perm = cv.take<uint16_t>(M * k * H);
    b.act_perm = cv.take<uint16_t>(M * k * c.moe_intermediate);
    b.y = cv.take<uint16_t>(M * k * H);
  } else {
    b.act = cv.take<uint16_t>(Mh * c.intermediate);
  }
  if (op == QWEN3_OP_STACK_PREFILL || op == QWEN3_OP_STACK_DECODE) {
    b.xs = cv.take<float>(M * H);
    b.hf = cv.take<uint16_t>(M * H);
  }
  b.ticket = cv.take<int>(64);
  if (M <= 64) {
    b.ssq = cv.take<float>((size_t)(H / 128 + 1) * 64);
    b.rs_x = cv.take<float>(64);
    b.rs_x1 = cv.take<float>(64);
  }
  if (out) *out = b;
  return cv.used + 256;
}

// ----------------------------------------------------------------------------- layer pieces
struct Ctx {
  const qwen3_config& c;
  cudaStream_t s;
  int* err;
};

static inline bool swap_for(long long M) { return M <= 256; }

// Every projection of a dense block runs on the decode-sized cluster GEMM (at most 64
// tokens): the RMSNorms after o_proj and down can then be deferred into the projection
// that reads them.
static bool decode_sized_block(const qwen3_config& c, long long M) {
  const int H = c.hidden, I = c.intermediate, D = c.head_dim;
  const int nqkv = (c.n_q_heads + 2 * c.n_kv_heads) * D;
  return skinny_supported((int)M, nqkv, H, kEpiQKRope) && skinny_supported((int)M, H, c.n_q_heads * D, kEpiResid) &&
         skinny_supported((int)M, 2 * I, H, kEpiSwiglu) && skinny_supported((int)M, H, I, kEpiResid);
}

// x1 = x + o_proj(attn(norm1(x)))   ([P-Mini] section TransformerBlock, first half)
// h_ready: b.h already holds norm1(x) (written by the previous layer's last GEMM).
// *h2_ready is set when the o_proj GEMM also left norm2(x1) in b.h.
static int attention_half(const Ctx& k, const qwen3_layer_weights& w, const void* x, bool x_f32, int B, int T,
                          bool decode, const int* pos, const qwen3_kv_layer& kv, const float* rope, Buffers& b,
                          bool h_ready, bool* h2_ready, bool defer2 = false) {
  const qwen3_config& c = k.c;
  const int H = c.hidden, D = c.head_dim;
  const long long M = (long long)B * T;
  const int nqkv = (c.n_q_heads + 2 * c.n_kv_heads) * D;
  const bool f16 = c.gemm_f16 != 0;  // projections' operand type (q and the cache stay bf16)
  // one token per sequence at position pos[b], attending 0..pos[b]: the decode attention
  // computes exactly that, for a prefill of T = 1 as well
  decode = decode || T == 1;
  // decode-sized (at most 64 tokens): every projection is one cluster split-K launch, and
  // its activation operand is carried as hi/lo halves (2M rows: the weight stream bounds
  // these GEMMs, so the doubled N costs nothing measurable)
  const bool skinny = skinny_supported((int)M, nqkv, H, kEpiQKRope) &&
                      skinny_supported((int)M, H, c.n_q_heads * D, kEpiResid);
  int rc = 0;
  if (!h_ready) {
    ProfScope ps("rmsnorm", k.s);
    rc = launch_rmsnorm(x, x_f32, H, w.in_norm, b.h, H, (int)M, H, c.rms_eps, k.s, b.ticket, f16,
                        skinny ? M * H : 0, skinny ? b.rs_x : nullptr);
    b.h_deferred = false;
  }
  if (rc) return rc;
  QKRopeArgs qa;
  qa.T = T;
  qa.Hq = c.n_q_heads;
  qa.Hkv = c.n_kv_heads;
  qa.s_max = kv.s_max;
  qa.max_pos = c.max_pos;
  qa.pos_base = pos;
  qa.q_norm = w.q_norm;
  qa.k_norm = w.k_norm;
  qa.rope = rope;
  qa.ck = kv.k;
  qa.cv = kv.v;
  qa.eps = c.rms_eps;
  if (skinny) {
    SkinnyDesc q;
    q.A = b.h; q.lda = H; q.W = w.w_qkv; q.ldw = H;
    q.M = (int)M; q.N = nqkv; q.K = H;
    q.a_hilo = true;  // b.h: M hi rows, then M lo rows
    q.epi = kEpiQKRope;
    q.out = b.qkv; q.ldo = nqkv;
    q.w_early = true;  // weights; a library kernel of this call runs before this GEMM
    q.qk = qa;
    // one token per sequence: q as hi/lo halves for the decode attention (G <= 8)
    const bool hilo = decode && c.n_q_heads / c.n_kv_heads <= 8;
    if (hilo) {
      q.qk.q2 = b.q2;
      q.qk.ldq2 = 2LL * c.n_q_heads * D;
    }
    q.f16 = f16;
    if (h_ready && b.h_deferred) {  // b.h = x * in_norm * s_t: scale by r_t / s_t, keep r_t
      q.row_ssq = b.ssq; q.ssq_tiles = H / 128; q.ssq_n = H; q.ssq_eps = c.rms_eps;
      q.row_s_in = b.rs_x1; q.row_r_out = b.rs_x;
    }
    {
      ProfScope ps("gemm_qkv", k.s);
      rc = launch_gemm_skinny(q, k.s, k.err);
    }
    if (rc) return rc;
    {
      ProfScope ps(decode ? "attn_decode" : "attn_prefill", k.s);
      if (decode) {
        rc = launch_attention_decode(hilo ? b.q2 : b.qkv, hilo ? 2LL * c.n_q_heads * D : nqkv, B, c.n_q_heads,
                                     c.n_kv_heads, pos, kv.k, kv.v, kv.s_max, b.part, b.o,
                                     (long long)c.n_q_heads * D, k.err, k.s, f16, hilo,
                                     M * c.n_q_heads * D,  // o as hi/lo rows for o_proj
                                     b.plan_ready);
        b.plan_ready = rc == 0;
      } else
        rc = launch_attention_prefill(b.qkv, nqkv, B, T, c.n_q_heads, c.n_kv_heads, pos, kv.k, kv.v, kv.s_max, b.o,
                                      (long long)c.n_q_heads * D, k.err, k.s, f16);
    }
    if (rc) return rc;
    SkinnyDesc o;
    o.A = b.o; o.lda = c.n_q_heads * D; o.W = w.w_o; o.ldw = c.n_q_heads * D;
    o.M = (int)M; o.N = H; o.K = c.n_q_heads * D;
    o.a_hilo = decode;  // the decode merge writes o as hi/lo rows; the prefill attention does not
    o.epi = kEpiResid;
    o.resid = x; o.resid_f32 = x_f32; o.ldr = H;
    o.out = b.x1; o.out_f32 = true; o.ldo = H;
    o.w_early = true;
    // the post-attention RMSNorm of x1 goes to b.h (hi/lo rows) in the same launch
    o.norm_w = w.post_norm; o.norm_out = b.h; o.ld_norm = H; o.norm_eps = c.rms_eps; o.ticket = b.ticket; o.ssq = b.ssq;
    o.norm_lo = M * H;
    if (defer2) {  // the gate/up projection applies it: y = x1 * post_norm * r(x)_t
      o.norm_deferred = true;
      o.pre_scale = b.rs_x;
    } else {
      o.row_r_out = b.rs_x1;
    }
    o.f16 = f16;
    if (defer2) {
      // a dense FFN follows: leave the SMs of its gate/up projection free, so that all of
      // its CTAs start beside this one and prefetch their weights
      SkinnyDesc gu;
      gu.M = (int)M; gu.N = 2 * c.intermediate; gu.K = H; gu.epi = kEpiSwiglu; gu.a_hilo = true;
      const int n_gu = skinny_ctas(gu);
      if (n_gu > 0 && n_gu < num_sms()) o.max_ctas = num_sms() - n_gu;
    }
    ProfScope ps("gemm_o", k.s);
    rc = launch_gemm_skinny(o, k.s, k.err);
    *h2_ready = rc == 0;
    b.h2_deferred = rc == 0 && defer2;
    return rc;
  }
  GemmDesc g;
  g.swap = swap_for(M);
  g.K = H;
  const void* act = b.h;
  if (g.swap) { g.P = w.w_qkv; g.p_rows = nqkv; g.ldp = H; g.Q = act; g.q_rows = (int)M; g.ldq = H; }
  else        { g.P = act; g.p_rows = (int)M; g.ldp = H; g.Q = w.w_qkv; g.q_rows = nqkv; g.ldq = H; }
  g.p_early = g.swap;  // weights; a library kernel of this call runs before this GEMM
  g.f16 = f16;
  g.epi = kEpiStore;
  g.out = b.qkv;
  g.ldo = nqkv;
  g.partial = b.gpart;
  g.partial_bytes = b.gpart ? kSplitKBytes : 0;
  int qk_done = 0;
  {
    // QK-norm, RoPE and the KV-cache write run on the fp32 accumulators (no bf16 round
    // trip of q/k/v): in the GEMM's epilogue for prefill, in the split-K completion
    // for small token counts
    if (!g.swap) {
      g.epi = kEpiQKRope;
      g.force_bn = 256;
    } else {
      g.qk_in_reduce = true;
      g.fused = &qk_done;
    }
    g.qk.T = T;
    g.qk.Hq = c.n_q_heads;
    g.qk.Hkv = c.n_kv_heads;
    g.qk.s_max = kv.s_max;
    g.qk.max_pos = c.max_pos;
    g.qk.pos_base = pos;
    g.qk.q_norm = w.q_norm;
    g.qk.k_norm = w.k_norm;
    g.qk.rope = rope;
    g.qk.ck = kv.k;
    g.qk.cv = kv.v;
    g.qk.eps = c.rms_eps;
  }
  {
    ProfScope ps("gemm_qkv", k.s);
    rc = launch_gemm(g, k.s, k.err);
  }
  if (rc) return rc;
  if (g.swap && !qk_done) {
    ProfScope ps("qk_norm_rope", k.s);
    rc = launch_qk_norm_rope(b.qkv, nqkv, B, T, c.n_q_heads, c.n_kv_heads, pos, w.q_norm, w.k_norm, rope, kv.k,
                             kv.v, kv.s_max, c.max_pos, c.rms_eps, k.err, k.s);
  }
  if (rc) return rc;
  {
    ProfScope ps(decode ? "attn_decode" : "attn_prefill", k.s);
    if (decode)
      rc = launch_attention_decode(b.qkv, nqkv, B, c.n_q_heads, c.n_kv_heads, pos, kv.k, kv.v, kv.s_max, b.part,
                                   b.o, (long long)c.n_q_heads * D, k.err, k.s, f16, false, 0, b.plan_ready);
    if (decode) b.plan_ready = rc == 0;
    else
      rc = launch_attention_prefill(b.qkv, nqkv, B, T, c.n_q_heads, c.n_kv_heads, pos, kv.k, kv.v, kv.s_max, b.o,
                                    (long long)c.n_q_heads * D, k.err, k.s, f16);
  }
  if (rc) return rc;
  GemmDesc o;
  o.swap = swap_for(M);
  o.K = c.n_q_heads * D;
  if (o.swap) { o.P = w.w_o; o.p_rows = H; o.ldp = o.K; o.Q = b.o; o.q_rows = (int)M; o.ldq = o.K; }
  else        { o.P = b.o; o.p_rows = (int)M; o.ldp = o.K; o.Q = w.w_o; o.q_rows = H; o.ldq = o.K; }
  o.p_early = o.swap;  // weights; a library kernel of this call runs before this GEMM
  o.f16 = f16;
  o.epi = kEpiResid;
  o.resid = x;
  o.resid_f32 = x_f32;
  o.ldr = H;
  o.out = b.x1;
  o.out_f32 = true;
  o.ldo = H;
  o.partial = b.gpart;
  o.partial_bytes = b.gpart ? kSplitKBytes : 0;
  // with split K, the completion kernel also writes norm2(x1) into b.h
  int h2 = 0;
  o.norm_w = w.post_norm;
  o.norm_out = b.h;
  o.norm_eps = c.rms_eps;
  o.fused = &h2;
  ProfScope ps("gemm_o", k.s);
  rc = launch_gemm(o, k.s, k.err);
  *h2_ready = h2 != 0;
  return rc;
}

// out = x1 + down(silu(gate(norm2(x1))) * up(norm2(x1)))   ([P-Mini] sections SwiGLU FFN, TransformerBlock)
// h2_ready: b.h already holds norm2(x1). With next_norm set, the down GEMM's split-K
// completion may also write norm(out) * next_norm into next_out (*next_ready set then).
// next_hilo: next_out feeds a decode-sized projection (it then also gets the lo rows).
static int dense_ffn(const Ctx& k, const qwen3_layer_weights& w, long long M, void* out, bool out_f32, Buffers& b,
                     bool h2_ready, const uint16_t* next_norm = nullptr, uint16_t* next_out = nullptr,
                     bool* next_ready = nullptr, bool next_hilo = false, bool next_defer = false) {
  const qwen3_config& c = k.c;
  const int H = c.hidden, I = c.intermediate;
  const bool f16 = c.gemm_f16 != 0;
  const bool skinny = skinny_supported((int)M, 2 * I, H, kEpiSwiglu) && skinny_supported((int)M, H, I, kEpiResid);
  int rc = 0;
  if (!h2_ready) {
    ProfScope ps("rmsnorm", k.s);
    rc = launch_rmsnorm(b.x1, true, H, w.post_norm, b.h, H, (int)M, H, c.rms_eps, k.s, nullptr, f16,
                        skinny ? M * H : 0, skinny ? b.rs_x1 : nullptr);
    b.h2_deferred = false;
  }
  if (rc) return rc;
  if (skinny) {
    SkinnyDesc g;
    g.A = b.h; g.lda = H; g.W = w.w_gate_up; g.ldw = H;
    g.M = (int)M; g.N = 2 * I; g.K = H;
    g.a_hilo = true;  // b.h: hi rows then lo rows
    g.epi = kEpiSwiglu;
    g.out = b.act; g.ldo = I;
    g.out_lo = M * I;  // act as hi/lo rows for the down projection
    g.w_early = true;  // weights; a library kernel of this call runs before this GEMM
    g.f16 = f16;
    if (h2_ready && b.h2_deferred) {  // b.h = x1 * post_norm * r(x)_t: scale by r(x1)_t / r(x)_t
      g.row_ssq = b.ssq; g.ssq_tiles = H / 128; g.ssq_n = H; g.ssq_eps = c.rms_eps;
      g.row_s_in = b.rs_x; g.row_r_out = b.rs_x1;
    }
    {
      ProfScope ps("gemm_gate_up", k.s);
      rc = launch_gemm_skinny(g, k.s, k.err);
    }
    if (rc) return rc;
    SkinnyDesc d;
    d.A = b.act; d.lda = I; d.W = w.w_down; d.ldw = I;
    d.M = (int)M; d.N = H; d.K = I;
    d.a_hilo = true;
    d.epi = kEpiResid;
    d.resid = b.x1; d.resid_f32 = true; d.ldr = H;
    d.out = out; d.out_f32 = out_f32; d.ldo = H;
    d.w_early = true;
    d.f16 = f16;
    if (next_norm && next_out) {
      d.norm_w = next_norm; d.norm_out = next_out; d.ld_norm = H; d.norm_eps = c.rms_eps; d.ticket = b.ticket; d.ssq = b.ssq;
      d.norm_lo = next_hilo ? M * H : 0;
      if (next_defer) {  // the next layer's QKV projection applies it: y = x * in_norm * r(x1)_t
        d.norm_deferred = true;
        d.pre_scale = b.rs_x1;
      } else {
        d.row_r_out = b.rs_x;
      }
    }
    {
      // fit beside the gate/up projection, so that all of this launch's CTAs start early
      const int n_gu = skinny_ctas(g);
      if (n_gu > 0 && n_gu < num_sms()) d.max_ctas = num_sms() - n_gu;
    }
    ProfScope ps("gemm_down", k.s);
    rc = launch_gemm_skinny(d, k.s, k.err);
    if (next_ready) *next_ready = rc == 0 && next_norm && next_out;
    b.h_deferred = rc == 0 && next_norm && next_out && next_defer;
    return rc;
  }
  GemmDesc g;
  g.swap = swap_for(M);
  g.K = H;
  if (g.swap) { g.P = w.w_gate_up; g.p_rows = 2 * I; g.ldp = H; g.Q = b.h; g.q_rows = (int)M; g.ldq = H; }
  else        { g.P = b.h; g.p_rows = (int)M; g.ldp = H; g.Q = w.w_gate_up; g.q_rows = 2 * I; g.ldq = H; }
  g.p_early = g.swap;  // weights; a library kernel of this call runs before this GEMM
  g.f16 = f16;
  g.epi = kEpiSwiglu;
  g.out = b.act;
  g.ldo = I;
  g.partial = b.gpart;
  g.partial_bytes = b.gpart ? kSplitKBytes : 0;
  {
    ProfScope ps("gemm_gate_up", k.s);
    rc = launch_gemm(g, k.s, k.err);
  }
  if (rc) return rc;
  GemmDesc d;
  d.swap = swap_for(M);
  d.K = I;
  if (d.swap) { d.P = w.w_down; d.p_rows = H; d.ldp = I; d.Q = b.act; d.q_rows = (int)M; d.ldq = I; }
  else        { d.P = b.act; d.p_rows = (int)M; d.ldp = I; d.Q = w.w_down; d.q_rows = H; d.ldq = I; }
  d.p_early = d.swap;  // weights; a library kernel of this call runs before this GEMM
  d.f16 = f16;
  d.epi = kEpiResid;
  d.resid = b.x1;
  d.resid_f32 = true;
  d.ldr = H;
  d.out = out;
  d.out_f32 = out_f32;
  d.ldo = H;
  d.partial = b.gpart;
  d.partial_bytes = b.gpart ? kSplitKBytes : 0;
  int nr = 0;
  if (next_norm && next_out) {
    d.norm_w = next_norm;
    d.norm_out = next_out;
    d.norm_eps = c.rms_eps;
    d.fused = &nr;
  }
  ProfScope ps("gemm_down", k.s);
  rc = launch_gemm(d, k.s, k.err);
  if (next_ready) *next_ready = nr != 0;
  return rc;
}

// out = x1 + sum_j w_j Expert_{e_j}(norm2(x1))   ([P-Mini] section MoE)
static int moe_ffn(const Ctx& k, const qwen3_layer_weights& w, long long M, void* out, bool out_f32, Buffers& b,
                   bool h2_ready) {
  const qwen3_config& c = k.c;
  const int H = c.hidden, E = c.n_experts, kk = c.top_k, Im = c.moe_intermediate;
  const bool f16 = c.gemm_f16 != 0;
  int rc = 0;
  if (!h2_ready) {
    ProfScope ps("rmsnorm", k.s);
    rc = launch_rmsnorm(b.x1, true, H, w.post_norm, b.h, H, (int)M, H, c.rms_eps, k.s, nullptr, f16);
  }
  if (rc) return rc;
  // router logits in fp32 (no bf16 rounding before the softmax)
  if (skinny_supported((int)M, E, H, kEpiStore)) {
    SkinnyDesc r;
    r.A = b.h; r.lda = H; r.W = w.router; r.ldw = H;
    r.M = (int)M; r.N = E; r.K = H;
    r.a_hilo = h2_ready;  // the decode-sized o_proj left norm2(x1) as hi/lo rows
    r.epi = kEpiStore;
    r.out = b.logits; r.out_f32 = true; r.ldo = E;
    r.w_early = true;  // weights; a library kernel of this call runs before this GEMM
    r.f16 = f16;
    ProfScope ps("gemm_router", k.s);
    rc = launch_gemm_skinny(r, k.s, k.err);
  } else {
  GemmDesc r;
  r.swap = swap_for(M);
  r.K = H;
  if (r.swap) { r.P = w.router; r.p_rows = E; r.ldp = H; r.Q = b.h; r.q_rows = (int)M; r.ldq = H; }
  else        { r.P = b.h; r.p_rows = (int)M; r.ldp = H; r.Q = w.router; r.q_rows = E; r.ldq = H; r.force_bn = 128; }
  r.p_early = r.swap;  // weights; a library kernel of this call runs before this GEMM
  r.f16 = f16;
  r.epi = kEpiStore;
  r.out = b.logits;
  r.out_f32 = true;
  r.ldo = E;
  r.partial = b.gpart;
  r.partial_bytes = b.gpart ? kSplitKBytes : 0;
  {
    ProfScope ps("gemm_router", k.s);
    rc = launch_gemm(r, k.s, k.err);
  }
  }
  if (rc) return rc;
  {
    ProfScope ps("moe_route", k.s);
    rc = launch_moe_route(b.logits, (int)M, E, kk, c.norm_topk_prob, b.idx, b.w, b.counts, k.s);
  }
  if (rc) return rc;
  {
    ProfScope ps("moe_permute", k.s);
    rc = launch_moe_permute(b.idx, (int)M, kk, E, b.counts, b.offsets, b.perm_token, b.perm_slot, b.inv_pos, b.h, H,
                            b.a_perm, k.s);
  }
  if (rc) return rc;
  const long long rows = M * kk;
  // few routed rows per expert (decode-sized batches): each expert's weights on the MMA's
  // 128-row side and its rows as N, so that every hit expert's weights stream once
  const bool per_expert_swap = rows <= 32LL * E;
  GemmDesc gu;
  if (per_expert_swap) {
    gu.swap = true;
    gu.P = w.moe_gate_up; gu.p_rows = 2 * Im; gu.ldp = H; gu.p_rows_total = (long long)E * 2 * Im;
    gu.Q = b.a_perm; gu.q_rows = (int)rows; gu.ldq = H;
    gu.force_bn = 64;
  } else {
    gu.P = b.a_perm; gu.p_rows = (int)rows; gu.ldp = H;
    gu.Q = w.moe_gate_up; gu.q_rows = 2 * Im; gu.ldq = H; gu.q_rows_total = (long long)E * 2 * Im;
  }
  gu.K = H;
  gu.f16 = f16;
  gu.epi = kEpiSwiglu;
  gu.out = b.act_perm; gu.ldo = Im;
  gu.n_groups = E; gu.group_offsets = b.offsets;
  {
    ProfScope ps("moe_gemm_gate_up", k.s);
    rc = launch_gemm(gu, k.s, k.err);
  }
  if (rc) return rc;
  GemmDesc dn;
  if (per_expert_swap) {
    dn.swap = true;
    dn.P = w.moe_down; dn.p_rows = H; dn.ldp = Im; dn.p_rows_total = (long long)E * H;
    dn.Q = b.act_perm; dn.q_rows = (int)rows; dn.ldq = Im;
    dn.force_bn = 64;
  } else {
    dn.P = b.act_perm; dn.p_rows = (int)rows; dn.ldp = Im;
    dn.Q = w.moe_down; dn.q_rows = H; dn.ldq = Im; dn.q_rows_total = (long long)E * H;
  }
  dn.K = Im;
  dn.f16 = f16;
  dn.epi = kEpiStore;
  dn.out = b.y; dn.ldo = H;
  dn.n_groups = E; dn.group_offsets = b.offsets;
  {
    ProfScope ps("moe_gemm_down", k.s);
    rc = launch_gemm(dn, k.s, k.err);
  }
  if (rc) return rc;
  ProfScope ps("moe_combine", k.s);
  return launch_moe_combine(b.x1, b.y, b.w, b.inv_pos, (int)M, kk, H, out, out_f32, k.s);
}

static int check_weights(const qwen3_config& c, const qwen3_layer_weights* w, bool moe) {
  Q3_CHECK(w, QWEN3_EINVAL, "layer weights pointer is NULL");
  const void* need[] = {w->in_norm, w->w_qkv, w->q_norm, w->k_norm, w->w_o, w->post_norm};
  const char* names[] = {"in_norm", "w_qkv", "q_norm", "k_norm", "w_o", "post_norm"};
  for (int i = 0; i < 6; ++i) {
    Q3_CHECK(need[i], QWEN3_EINVAL, "weights.%s is NULL", names[i]);
    Q3_CHECK(aligned16(need[i]), QWEN3_EALIGN, "weights.%s is not 16-byte aligned", names[i]);
  }
  if (moe) {
    Q3_CHECK(c.n_experts > 0, QWEN3_ESHAPE, "MoE block needs n_experts > 0");
    const void* m[] = {w->router, w->moe_gate_up, w->moe_down};
    const char* mn[] = {"router", "moe_gate_up", "moe_down"};
    for (int i = 0; i < 3; ++i) {
      Q3_CHECK(m[i], QWEN3_EINVAL, "weights.%s is NULL", mn[i]);
      Q3_CHECK(aligned16(m[i]), QWEN3_EALIGN, "weights.%s is not 16-byte aligned", mn[i]);
    }
  } else {
    Q3_CHECK(c.intermediate > 0, QWEN3_ESHAPE, "dense block needs intermediate > 0");
    Q3_CHECK(w->w_gate_up && w->w_down, QWEN3_EINVAL, "weights.w_gate_up / w_down is NULL");
    Q3_CHECK(aligned16(w->w_gate_up) && aligned16(w->w_down), QWEN3_EALIGN, "FFN weights not 16-byte aligned");
  }
  return 0;
}

static int check_kv(const qwen3_config& c, const qwen3_kv_layer* kv, int T) {
  Q3_CHECK(kv, QWEN3_EINVAL, "kv descriptor is NULL");
  Q3_CHECK(kv->k && kv->v, QWEN3_EINVAL, "kv->k / kv->v is NULL");
  Q3_CHECK(aligned16(kv->k) && aligned16(kv->v), QWEN3_EALIGN, "kv buffers are not 16-byte aligned");
  Q3_CHECK(kv->s_max > 0, QWEN3_EINVAL, "kv->s_max must be positive");
  Q3_CHECK(T <= kv->s_max && T <= c.max_pos, QWEN3_ECAPACITY, "T (%d) exceeds the cache capacity (%d) or max_pos (%d)",
           T, kv->s_max, c.max_pos);
  return 0;
}

static int finish(int rc) {
  if (rc == -6 && g_last_error.empty()) set_last_error("CUDA error: %s", cudaGetErrorString(cudaGetLastError()));
  return rc;
}

}  // namespace q3

using namespace q3;

// ============================================================================= C ABI
extern "C" {

const char* qwen3_last_error(void) { return g_last_error.c_str(); }

const char* qwen3_status_string(int s) {
  switch (s) {
    case QWEN3_OK: return "ok";
    case QWEN3_EINVAL: return "invalid argument";
    case QWEN3_ESHAPE: return "unsupported shape";
    case QWEN3_EALIGN: return "misaligned pointer";
    case QWEN3_ECAPACITY: return "capacity exceeded";
    case QWEN3_EWORKSPACE: return "workspace too small";
    case QWEN3_ECUDA: return "CUDA error";
    case QWEN3_ETIMEOUT: return "device wait timed out";
    case QWEN3_EDEVICE: return "unsupported device";
    default: return "unknown status";
  }
}

int qwen3_config_qwen3_0_6b(qwen3_config* c) {
  Q3_CHECK(c, QWEN3_EINVAL, "cfg is NULL");
  memset(c, 0, sizeof(*c));
  c->hidden = 1024;
  c->n_q_heads = 16;
  c->n_kv_heads = 8;
  c->head_dim = 128;
  c->intermediate = 3072;
  c->vocab = 151936;
  c->n_layers = 28;
  c->max_pos = 40960;
  c->norm_topk_prob = 1;
  c->rms_eps = 1e-6f;
  c->rope_theta = 1e6;
  return 0;
}

int qwen3_validate_config(const qwen3_config* c) {
  g_last_error.clear();
  return validate_cfg(c);
}

size_t qwen3_rope_table_bytes(const qwen3_config* c) {
  if (!c || c->max_pos <= 0 || c->head_dim <= 0) return 0;
  return (size_t)c->max_pos * (c->head_dim / 2) * 2 * sizeof(float);
}

int qwen3_rope_table(const qwen3_config* c, float* rope, void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(rope && aligned16(rope), rope ? QWEN3_EALIGN : QWEN3_EINVAL, "rope table pointer NULL or misaligned");
  if ((rc = check_device())) return rc;
  const int half = c->head_dim / 2;
  std::vector<float> host((size_t)c->max_pos * half * 2);
  std::vector<double> inv_freq(half);
  // theta_i = theta^(-2i/D)   ([P-Mini] section RoPE)
  for (int i = 0; i < half; ++i) inv_freq[i] = std::pow(c->rope_theta, -2.0 * i / c->head_dim);
  for (int m = 0; m < c->max_pos; ++m)
    for (int i = 0; i < half; ++i) {
      const double a = (double)m * inv_freq[i];
      host[((size_t)m * half + i) * 2 + 0] = (float)std::cos(a);
      host[((size_t)m * half + i) * 2 + 1] = (float)std::sin(a);
    }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(rope, host.data(), host.size() * sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    set_last_error("rope table copy failed: %s", cudaGetErrorString(cudaGetLastError()));
    return QWEN3_ECUDA;
  }
  return 0;
}

// Greedy generation: the stack's workspace (the larger of prefill and decode) followed
// by the step's logits [B, V] fp32, the cache lengths [B] and the next ids [B].
static size_t generate_stack_bytes(const qwen3_config& c, int B, int T, int s_max) {
  const size_t a = carve(c, QWEN3_OP_STACK_PREFILL, B, T, s_max, nullptr, nullptr);
  const size_t d = carve(c, QWEN3_OP_STACK_DECODE, B, 1, s_max, nullptr, nullptr);
  return ((a > d ? a : d) + 255) & ~(size_t)255;
}
static size_t generate_extra_bytes(const qwen3_config& c, int B) {
  return (((size_t)B * c.vocab * sizeof(float) + 255) & ~(size_t)255) + 2 * (((size_t)B * sizeof(int) + 255) & ~(size_t)255);
}

size_t qwen3_workspace_size(const qwen3_config* c, int op, int B, int T, int s_max) {
  if (!c || validate_cfg(c) != 0 || B <= 0 || s_max <= 0) return 0;
  if (op == QWEN3_OP_GENERATE)
    return T > 0 ? generate_stack_bytes(*c, B, T, s_max) + generate_extra_bytes(*c, B) : 0;
  if (op < QWEN3_OP_BLOCK_PREFILL || op > QWEN3_OP_STACK_DECODE) return 0;
  if (op != QWEN3_OP_BLOCK_DECODE && op != QWEN3_OP_STACK_DECODE && T <= 0) return 0;
  return carve(*c, op, B, T, s_max, nullptr, nullptr);
}

int qwen3_pack_qkv(const qwen3_config* c, const qwen3_bf16* wq, const qwen3_bf16* wk, const qwen3_bf16* wv,
                   qwen3_bf16* out, void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(wq && wk && wv && out, QWEN3_EINVAL, "pack_qkv: NULL pointer");
  const size_t H = c->hidden, D = c->head_dim;
  const size_t nq = (size_t)c->n_q_heads * D * H, nk = (size_t)c->n_kv_heads * D * H;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(out, wq, nq * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(out + nq, wk, nk * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(out + nq + nk, wv, nk * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
    set_last_error("pack_qkv copy failed: %s", cudaGetErrorString(cudaGetLastError()));
    return QWEN3_ECUDA;
  }
  return 0;
}

int qwen3_pack_gate_up(int I, int H, const qwen3_bf16* gate, const qwen3_bf16* up, qwen3_bf16* out, void* stream) {
  g_last_error.clear();
  Q3_CHECK(gate && up && out, QWEN3_EINVAL, "pack_gate_up: NULL pointer");
  Q3_CHECK(I > 0 && I % 16 == 0 && H > 0 && H % 8 == 0, QWEN3_ESHAPE, "pack_gate_up: I %% 16 and H %% 8 required");
  Q3_CHECK(aligned16(gate) && aligned16(up) && aligned16(out), QWEN3_EALIGN, "pack_gate_up: misaligned pointer");
  return finish(launch_pack_gate_up(gate, up, (long long)I * H, 1, I, H, out, static_cast<cudaStream_t>(stream)));
}

int qwen3_pack_moe_gate_up(int E, int Im, int H, const qwen3_bf16* gate_up, qwen3_bf16* out, void* stream) {
  g_last_error.clear();
  Q3_CHECK(gate_up && out, QWEN3_EINVAL, "pack_moe_gate_up: NULL pointer");
  Q3_CHECK(E > 0 && Im > 0 && Im % 16 == 0 && H > 0 && H % 8 == 0, QWEN3_ESHAPE,
           "pack_moe_gate_up: Im %% 16 and H %% 8 required");
  Q3_CHECK(aligned16(gate_up) && aligned16(out), QWEN3_EALIGN, "pack_moe_gate_up: misaligned pointer");
  return finish(launch_pack_gate_up(gate_up, gate_up + (size_t)Im * H, (long long)2 * Im * H, E, Im, H, out,
                                    static_cast<cudaStream_t>(stream)));
}

// Two-way check of a layer's weight pointers (a set-up call; reads no device memory).
// Forward: every member the block kind reads is set and 16-byte aligned. Reverse: every
// member it does not read is NULL, so that weights built for the other kind (or a config
// of the wrong kind) are reported instead of silently ignored. With the byte size of
// each member taken from the config, no two members may overlap: an offset into one
// weight arena computed with a wrong dimension shows up here. One read-only buffer may
// serve two members of the same size (the same pointer), e.g. shared norm weights.
int qwen3_check_layer_weights(const qwen3_config* c, const qwen3_layer_weights* w, int kind) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(w, QWEN3_EINVAL, "check_layer_weights: weights pointer is NULL");
  Q3_CHECK(kind == QWEN3_LAYER_DENSE || kind == QWEN3_LAYER_MOE, QWEN3_EINVAL,
           "check_layer_weights: kind %d is neither QWEN3_LAYER_DENSE nor QWEN3_LAYER_MOE", kind);
  const bool moe = kind == QWEN3_LAYER_MOE;
  const char* kname = moe ? "MoE" : "dense";
  if (moe)
    Q3_CHECK(c->n_experts > 0 && c->moe_intermediate > 0, QWEN3_ESHAPE,
             "check_layer_weights: a MoE layer needs n_experts > 0 and moe_intermediate > 0");
  else
    Q3_CHECK(c->intermediate > 0, QWEN3_ESHAPE, "check_layer_weights: a dense layer needs intermediate > 0");
  const size_t H = c->hidden, D = c->head_dim, Hq = c->n_q_heads, Hkv = c->n_kv_heads;
  const size_t I = moe ? 0 : c->intermediate, E = moe ? c->n_experts : 0, Im = moe ? c->moe_intermediate : 0;
  struct Member {
    const char* name;
    const void* p;
    size_t bytes;
    bool read;
  } m[] = {
      {"in_norm", w->in_norm, H * 2, true},
      {"w_qkv", w->w_qkv, (Hq + 2 * Hkv) * D * H * 2, true},
      {"q_norm", w->q_norm, D * 2, true},
      {"k_norm", w->k_norm, D * 2, true},
      {"w_o", w->w_o, H * Hq * D * 2, true},
      {"post_norm", w->post_norm, H * 2, true},
      {"w_gate_up", w->w_gate_up, 2 * I * H * 2, !moe},
      {"w_down", w->w_down, H * I * 2, !moe},
      {"router", w->router, E * H * 2, moe},
      {"moe_gate_up", w->moe_gate_up, E * 2 * Im * H * 2, moe},
      {"moe_down", w->moe_down, E * H * Im * 2, moe},
  };
  const int n = (int)(sizeof(m) / sizeof(m[0]));
  for (int i = 0; i < n; ++i) {
    if (m[i].read) {
      Q3_CHECK(m[i].p, QWEN3_EINVAL, "weights.%s is NULL but a %s layer reads it", m[i].name, kname);
      Q3_CHECK(aligned16(m[i].p), QWEN3_EALIGN, "weights.%s is not 16-byte aligned", m[i].name);
    } else {
      Q3_CHECK(!m[i].p, QWEN3_ESHAPE, "weights.%s is set but a %s layer does not read it (wrong kind or config)",
               m[i].name, kname);
    }
  }
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j) {
      if (!m[i].p || !m[j].p) continue;
      if (m[i].p == m[j].p && m[i].bytes == m[j].bytes) continue;
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(m[i].p), b0 = reinterpret_cast<uintptr_t>(m[j].p);
      Q3_CHECK(a0 + m[i].bytes <= b0 || b0 + m[j].bytes <= a0, QWEN3_EINVAL,
               "weights.%s (%zu bytes at %p) overlaps weights.%s (%zu bytes at %p)", m[i].name, m[i].bytes, m[i].p,
               m[j].name, m[j].bytes, m[j].p);
    }
  return 0;
}

int qwen3_check_device_error(void* stream) {
  g_last_error.clear();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_last_error("stream error: %s", cudaGetErrorString(e));
    return QWEN3_ECUDA;
  }
  int* p = device_error_word();
  if (!p) {
    set_last_error("device error word unavailable");
    return QWEN3_ECUDA;
  }
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QWEN3_ECUDA;
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    set_last_error("device reported: %s", qwen3_status_string(v));
  }
  return v;
}

static int common_block_checks(const qwen3_config* c, const qwen3_layer_weights* w, const void* x, int B, int T,
                               const int* pos, const qwen3_kv_layer* kv, const float* rope, void* ws, size_t ws_bytes,
                               int op, bool moe) {
  int rc = validate_cfg(c);
  if (rc) return rc;
  if ((rc = check_weights(*c, w, moe))) return rc;
  Q3_CHECK(x && pos && rope && ws, QWEN3_EINVAL, "x, positions, rope and ws must be non-NULL");
  Q3_CHECK(aligned16(x) && aligned16(rope) && aligned16(ws), QWEN3_EALIGN, "x, rope or ws not 16-byte aligned");
  Q3_CHECK(B > 0 && T > 0, QWEN3_EINVAL, "B (%d) and T (%d) must be positive", B, T);
  if ((rc = check_kv(*c, kv, T))) return rc;
  const size_t need = qwen3_workspace_size(c, op, B, T, kv->s_max);
  Q3_CHECK(ws_bytes >= need, QWEN3_EWORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return check_device();
}

int qwen3_block_prefill(const qwen3_config* c, const qwen3_layer_weights* w, qwen3_bf16* x, int B, int T,
                        const int* start_pos, const qwen3_kv_layer* kv, const float* rope, void* ws, size_t ws_bytes,
                        void* stream) {
  g_last_error.clear();
  int rc = common_block_checks(c, w, x, B, T, start_pos, kv, rope, ws, ws_bytes, QWEN3_OP_BLOCK_PREFILL, false);
  if (rc) return rc;
  Buffers b;
  carve(*c, QWEN3_OP_BLOCK_PREFILL, B, T, kv->s_max, ws, &b);
  Ctx k{*c, static_cast<cudaStream_t>(stream), device_error_word()};
  bool h2 = false;
  if ((rc = attention_half(k, *w, x, false, B, T, false, start_pos, *kv, rope, b, false, &h2,
                           decode_sized_block(*c, (long long)B * T))))
    return finish(rc);
  return finish(dense_ffn(k, *w, (long long)B * T, x, false, b, h2));
}

int qwen3_block_decode(const qwen3_config* c, const qwen3_layer_weights* w, qwen3_bf16* x, int B,
                       const int* cache_len, const qwen3_kv_layer* kv, const float* rope, void* ws, size_t ws_bytes,
                       void* stream) {
  g_last_error.clear();
  int rc = common_block_checks(c, w, x, B, 1, cache_len, kv, rope, ws, ws_bytes, QWEN3_OP_BLOCK_DECODE, false);
  if (rc) return rc;
  Buffers b;
  carve(*c, QWEN3_OP_BLOCK_DECODE, B, 1, kv->s_max, ws, &b);
  Ctx k{*c, static_cast<cudaStream_t>(stream), device_error_word()};
  bool h2 = false;
  if ((rc = attention_half(k, *w, x, false, B, 1, true, cache_len, *kv, rope, b, false, &h2,
                           decode_sized_block(*c, B))))
    return finish(rc);
  return finish(dense_ffn(k, *w, B, x, false, b, h2));
}

int qwen3_moe_block(const qwen3_config* c, const qwen3_layer_weights* w, qwen3_bf16* x, int B, int T,
                    const int* start_pos, const qwen3_kv_layer* kv, const float* rope, int* topk_idx, float* topk_w,
                    int* expert_offsets, int* perm_token, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  int rc = common_block_checks(c, w, x, B, T, start_pos, kv, rope, ws, ws_bytes, QWEN3_OP_MOE_BLOCK, true);
  if (rc) return rc;
  Buffers b;
  carve(*c, QWEN3_OP_MOE_BLOCK, B, T, kv->s_max, ws, &b);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Ctx k{*c, s, device_error_word()};
  const long long M = (long long)B * T;
  bool h2 = false;
  if ((rc = attention_half(k, *w, x, false, B, T, false, start_pos, *kv, rope, b, false, &h2))) return finish(rc);
  if ((rc = moe_ffn(k, *w, M, x, false, b, h2))) return finish(rc);
  const size_t mk = (size_t)M * c->top_k;
  if (topk_idx && cudaMemcpyAsync(topk_idx, b.idx, mk * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess) rc = -6;
  if (topk_w && cudaMemcpyAsync(topk_w, b.w, mk * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess) rc = -6;
  if (expert_offsets &&
      cudaMemcpyAsync(expert_offsets, b.offsets, (c->n_experts + 1) * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    rc = -6;
  if (perm_token && cudaMemcpyAsync(perm_token, b.perm_token, mk * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    rc = -6;
  return finish(rc);
}

int qwen3_stack_forward(const qwen3_config* c, const qwen3_bf16* embed, const qwen3_layer_weights* layers,
                        const qwen3_bf16* final_norm, const int* ids, int B, int T, int mode, int* pos_or_len,
                        const qwen3_kv_layer* kv, const float* rope, float* logits, int last_only, void* ws,
                        size_t ws_bytes, void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(c->n_layers > 0 && c->vocab > 0, QWEN3_ESHAPE, "stack needs n_layers > 0 and vocab > 0");
  Q3_CHECK(mode == QWEN3_MODE_PREFILL || mode == QWEN3_MODE_DECODE, QWEN3_EINVAL, "mode must be PREFILL or DECODE");
  const bool decode = mode == QWEN3_MODE_DECODE;
  Q3_CHECK(!decode || T == 1, QWEN3_EINVAL, "decode mode needs T == 1 (got %d)", T);
  Q3_CHECK(embed && layers && final_norm && ids && pos_or_len && kv && rope && logits && ws, QWEN3_EINVAL,
           "stack_forward: NULL argument");
  Q3_CHECK(aligned16(embed) && aligned16(final_norm) && aligned16(rope) && aligned16(logits) && aligned16(ws),
           QWEN3_EALIGN, "stack_forward: misaligned pointer");
  Q3_CHECK(B > 0 && T > 0, QWEN3_EINVAL, "B (%d) and T (%d) must be positive", B, T);
  for (int l = 0; l < c->n_layers; ++l) {
    if ((rc = check_weights(*c, &layers[l], false))) {
      set_last_error("layer %d: %s", l, g_last_error.c_str());
      return rc;
    }
    if ((rc = check_kv(*c, &kv[l], T))) {
      set_last_error("layer %d: %s", l, g_last_error.c_str());
      return rc;
    }
    Q3_CHECK(kv[l].s_max == kv[0].s_max, QWEN3_EINVAL, "all layers' caches must share s_max");
  }
  const int op = decode ? QWEN3_OP_STACK_DECODE : QWEN3_OP_STACK_PREFILL;
  const size_t need = qwen3_workspace_size(c, op, B, T, kv[0].s_max);
  Q3_CHECK(ws_bytes >= need, QWEN3_EWORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  if ((rc = check_device())) return rc;
  Buffers b;
  carve(*c, op, B, T, kv[0].s_max, ws, &b);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Ctx k{*c, s, device_error_word()};
  const int H = c->hidden;
  const long long M = (long long)B * T;
  {
    ProfScope ps("embed", s);
    rc = launch_embed(ids, (int)M, embed, c->vocab, H, b.xs, true, k.err, s, b.ticket, c->gemm_f16 != 0);
  }
  if (rc) return finish(rc);
  // With split K (small token counts), each layer's down projection also leaves the
  // next layer's norm1 (or, after the last layer, the final norm when every row is
  // kept) in b.h / b.hf, and the o_proj leaves norm2.
  bool h_ready = false;
  const bool fuse_final = !last_only || T == 1;
  // decode-sized: the RMSNorms after o_proj and down are deferred into the next projection
  const bool defer = decode_sized_block(*c, M);
  for (int l = 0; l < c->n_layers; ++l) {
    bool h2 = false;
    if ((rc = attention_half(k, layers[l], b.xs, true, B, T, decode, pos_or_len, kv[l], rope, b, h_ready, &h2,
                             defer)))
      return finish(rc);
    const bool last = l + 1 == c->n_layers;
    const uint16_t* nn = last ? (fuse_final ? final_norm : nullptr) : layers[l + 1].in_norm;
    if ((rc = dense_ffn(k, layers[l], M, b.xs, true, b, h2, nn, last ? b.hf : b.h, &h_ready, !last, defer && !last)))
      return finish(rc);
  }
  // final RMSNorm and tied LM head ([P-Mini] section 骨架; [P-SGL] section 一)
  const int rows = last_only ? B : (int)M;
  const float* xf = last_only ? b.xs + (long long)(T - 1) * H : b.xs;
  const long long ldx = last_only ? (long long)T * H : H;
  if (!h_ready) {
    ProfScope ps("rmsnorm", s);
    rc = launch_rmsnorm(xf, true, ldx, final_norm, b.hf, H, rows, H, c->rms_eps, s, nullptr, c->gemm_f16 != 0);
  }
  if (rc) return finish(rc);
  GemmDesc g;
  g.swap = swap_for(rows);
  g.K = H;
  if (g.swap) { g.P = embed; g.p_rows = c->vocab; g.ldp = H; g.Q = b.hf; g.q_rows = rows; g.ldq = H; }
  else        { g.P = b.hf; g.p_rows = rows; g.ldp = H; g.Q = embed; g.q_rows = c->vocab; g.ldq = H; }
  g.p_early = g.swap;  // weights; a library kernel of this call runs before this GEMM
  g.f16 = c->gemm_f16 != 0;
  g.epi = kEpiStore;
  g.out = logits;
  g.out_f32 = true;
  g.ldo = c->vocab;
  {
    ProfScope ps("lm_head", s);
    rc = launch_gemm(g, s, k.err);
  }
  if (rc) return finish(rc);
  if (decode) {
    ProfScope ps("advance_lengths", s);
    rc = launch_advance_lengths(pos_or_len, B, s);
  }
  return finish(rc);
}


int qwen3_profile_begin(int max_records) {
  g_last_error.clear();
  Q3_CHECK(max_records > 0, QWEN3_EINVAL, "profile_begin: max_records must be positive");
  if ((int)g_prof.size() < max_records) {
    const size_t old = g_prof.size();
    g_prof.resize(max_records);
    for (size_t i = old; i < g_prof.size(); ++i) {
      if (cudaEventCreate(&g_prof[i].a) != cudaSuccess || cudaEventCreate(&g_prof[i].b) != cudaSuccess) {
        g_prof.resize(i);
        set_last_error("profile_begin: cudaEventCreate failed");
        return QWEN3_ECUDA;
      }
    }
  }
  g_prof_used = 0;
  g_prof_on = true;
  return 0;
}

int qwen3_profile_end(void* stream) {
  g_prof_on = false;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    set_last_error("profile_end: stream error");
    return QWEN3_ECUDA;
  }
  return (int)g_prof_used;
}

int qwen3_profile_record(int i, char* name, int name_cap, float* ms) {
  Q3_CHECK(i >= 0 && (size_t)i < g_prof_used, QWEN3_EINVAL, "profile_record: index %d out of range", i);
  if (name && name_cap > 0) {
    strncpy(name, g_prof[i].name, name_cap - 1);
    name[name_cap - 1] = 0;
  }
  if (ms && cudaEventElapsedTime(ms, g_prof[i].a, g_prof[i].b) != cudaSuccess) return QWEN3_ECUDA;
  return 0;
}

// ----------------------------------------------------------------------------- ops
int qwen3_op_rmsnorm(const void* x, int x_f32, long long ldx, const qwen3_bf16* w, qwen3_bf16* out, long long ldo,
                     int rows, int n, float eps, int out_f16, void* stream) {
  g_last_error.clear();
  Q3_CHECK(x && w && out, QWEN3_EINVAL, "rmsnorm: NULL pointer");
  Q3_CHECK(aligned16(x) && aligned16(w) && aligned16(out), QWEN3_EALIGN, "rmsnorm: misaligned pointer");
  Q3_CHECK(n > 0 && n % 256 == 0 && n <= 2048, QWEN3_ESHAPE, "rmsnorm: n (%d) must be a multiple of 256, <= 2048", n);
  Q3_CHECK(rows >= 0 && ldx >= n && ldo >= n && ldx % 8 == 0 && ldo % 8 == 0, QWEN3_ESHAPE,
           "rmsnorm: bad rows or leading dimensions");
  int rc = check_device();
  if (rc) return rc;
  return finish(launch_rmsnorm(x, x_f32 != 0, ldx, w, out, ldo, rows, n, eps, static_cast<cudaStream_t>(stream),
                               nullptr, out_f16 != 0));
}

int qwen3_op_gemm(const qwen3_bf16* A, long long lda, const qwen3_bf16* W, long long ldw, void* out, long long ldo,
                  int M, int N, int K, int epilogue, const void* resid, long long ldr, int resid_f32, int out_f32,
                  int swap, int ab_f16, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  Q3_CHECK(A && W && out, QWEN3_EINVAL, "gemm: NULL operand");
  Q3_CHECK(aligned16(A) && aligned16(W) && aligned16(out), QWEN3_EALIGN, "gemm: misaligned operand");
  Q3_CHECK(M > 0 && N > 0 && K > 0, QWEN3_EINVAL, "gemm: M, N, K must be positive");
  Q3_CHECK(K % 64 == 0 && N % 32 == 0, QWEN3_ESHAPE, "gemm: K %% 64 == 0 and N %% 32 == 0 required");
  Q3_CHECK(lda >= K && ldw >= K && lda % 8 == 0 && ldw % 8 == 0 && ldo % 8 == 0, QWEN3_EALIGN,
           "gemm: leading dimensions must be >= K and multiples of 8");
  Q3_CHECK(epilogue >= 0 && epilogue <= 2, QWEN3_EINVAL, "gemm: epilogue must be 0, 1 or 2");
  if (epilogue == kEpiResid) {
    Q3_CHECK(resid && aligned16(resid) && ldr % 8 == 0 && ldr >= N, QWEN3_EINVAL, "gemm: residual missing or misaligned");
  }
  Q3_CHECK(ab_f16 == 0 || ab_f16 == 1, QWEN3_EINVAL, "gemm: ab_f16 must be 0 or 1");
  if (epilogue == kEpiSwiglu) {
    Q3_CHECK(!out_f32, QWEN3_EINVAL, "gemm: SwiGLU output is 16-bit (the operand type)");
    Q3_CHECK(ldo >= N / 2, QWEN3_EINVAL, "gemm: ldo too small for N/2 outputs");
  } else {
    Q3_CHECK(ldo >= N, QWEN3_EINVAL, "gemm: ldo (%lld) < N (%d)", ldo, N);
  }
  Q3_CHECK(swap >= -1 && swap <= 3, QWEN3_EINVAL, "gemm: swap must be -1, 0, 1, 2 or 3 (got %d)", swap);
  if (swap >= 2)
    Q3_CHECK(skinny_supported(M, N, K, epilogue), QWEN3_ESHAPE,
             "gemm: the cluster split-K form needs M <= 64 and N %% 128 == 0 (M %d, N %d)", M, N);
  int rc = check_device();
  if (rc) return rc;
  if (swap >= 2 || (swap < 0 && skinny_supported(M, N, K, epilogue))) {
    SkinnyDesc d;
    d.A = A; d.lda = lda; d.W = W; d.ldw = ldw;
    d.M = M; d.N = N; d.K = K;
    d.a_hilo = swap == 3;
    d.epi = epilogue;
    d.out = out; d.ldo = ldo; d.out_f32 = out_f32 != 0;
    d.resid = resid; d.ldr = ldr; d.resid_f32 = resid_f32 != 0;
    d.f16 = ab_f16 != 0;
    return finish(launch_gemm_skinny(d, static_cast<cudaStream_t>(stream), device_error_word()));
  }
  GemmDesc g;
  g.swap = swap < 0 ? swap_for(M) : swap != 0;
  g.K = K;
  if (g.swap) { g.P = W; g.p_rows = N; g.ldp = ldw; g.Q = A; g.q_rows = M; g.ldq = lda; }
  else        { g.P = A; g.p_rows = M; g.ldp = lda; g.Q = W; g.q_rows = N; g.ldq = ldw; }
  g.epi = epilogue;
  g.resid = resid;
  g.ldr = ldr;
  g.resid_f32 = resid_f32 != 0;
  g.out = out;
  g.ldo = ldo;
  g.out_f32 = out_f32 != 0;
  g.f16 = ab_f16 != 0;
  if (ws && aligned16(ws)) {
    g.partial = static_cast<float*>(ws);
    g.partial_bytes = ws_bytes;
  }
  return finish(launch_gemm(g, static_cast<cudaStream_t>(stream), device_error_word()));
}

int qwen3_op_qk_norm_rope(const qwen3_config* c, qwen3_bf16* qkv, long long ldqkv, int B, int T, const int* pos_base,
                          const qwen3_bf16* q_norm, const qwen3_bf16* k_norm, const qwen3_kv_layer* kv,
                          const float* rope, void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(qkv && pos_base && q_norm && k_norm && rope, QWEN3_EINVAL, "qk_norm_rope: NULL pointer");
  Q3_CHECK(B > 0 && T > 0, QWEN3_EINVAL, "qk_norm_rope: B and T must be positive");
  if ((rc = check_kv(*c, kv, T))) return rc;
  Q3_CHECK(ldqkv % 8 == 0 && ldqkv >= (long long)(c->n_q_heads + 2 * c->n_kv_heads) * c->head_dim, QWEN3_EALIGN,
           "qk_norm_rope: bad ldqkv");
  if ((rc = check_device())) return rc;
  return finish(launch_qk_norm_rope(qkv, ldqkv, B, T, c->n_q_heads, c->n_kv_heads, pos_base, q_norm, k_norm, rope,
                                    kv->k, kv->v, kv->s_max, c->max_pos, c->rms_eps, device_error_word(),
                                    static_cast<cudaStream_t>(stream)));
}

int qwen3_op_gemm_qkv_rope(const qwen3_config* c, const qwen3_bf16* h, const qwen3_bf16* w_qkv, qwen3_bf16* qkv,
                           int B, int T, const int* pos_base, const qwen3_bf16* q_norm, const qwen3_bf16* k_norm,
                           const qwen3_kv_layer* kv, const float* rope, void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(h && w_qkv && qkv && pos_base && q_norm && k_norm && rope, QWEN3_EINVAL, "gemm_qkv_rope: NULL pointer");
  Q3_CHECK(aligned16(h) && aligned16(w_qkv) && aligned16(qkv) && aligned16(q_norm) && aligned16(k_norm) &&
               aligned16(rope),
           QWEN3_EALIGN, "gemm_qkv_rope: misaligned pointer");
  Q3_CHECK(B > 0 && T > 0, QWEN3_EINVAL, "gemm_qkv_rope: B and T must be positive");
  if ((rc = check_kv(*c, kv, T))) return rc;
  if ((rc = check_device())) return rc;
  const int H = c->hidden, nqkv = (c->n_q_heads + 2 * c->n_kv_heads) * c->head_dim;
  GemmDesc g;
  g.swap = false;
  g.K = H;
  g.P = h; g.p_rows = B * T; g.ldp = H;
  g.Q = w_qkv; g.q_rows = nqkv; g.ldq = H;
  g.epi = kEpiQKRope;
  g.force_bn = 256;
  g.f16 = c->gemm_f16 != 0;
  g.out = qkv;
  g.ldo = nqkv;
  g.qk.T = T;
  g.qk.Hq = c->n_q_heads;
  g.qk.Hkv = c->n_kv_heads;
  g.qk.s_max = kv->s_max;
  g.qk.max_pos = c->max_pos;
  g.qk.pos_base = pos_base;
  g.qk.q_norm = q_norm;
  g.qk.k_norm = k_norm;
  g.qk.rope = rope;
  g.qk.ck = kv->k;
  g.qk.cv = kv->v;
  g.qk.eps = c->rms_eps;
  return finish(launch_gemm(g, static_cast<cudaStream_t>(stream), device_error_word()));
}

int qwen3_op_attention_prefill(const qwen3_config* c, const qwen3_bf16* qkv, long long ldqkv, int B, int T,
                               const int* start_pos, const qwen3_kv_layer* kv, qwen3_bf16* o, long long ldo,
                               void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(qkv && start_pos && o, QWEN3_EINVAL, "attention_prefill: NULL pointer");
  Q3_CHECK(aligned16(qkv) && aligned16(o), QWEN3_EALIGN, "attention_prefill: misaligned pointer");
  Q3_CHECK(B > 0 && T > 0, QWEN3_EINVAL, "attention_prefill: B and T must be positive");
  Q3_CHECK(ldqkv % 8 == 0 && ldo % 8 == 0 && ldo >= (long long)c->n_q_heads * c->head_dim, QWEN3_EALIGN,
           "attention_prefill: bad leading dimension");
  if ((rc = check_kv(*c, kv, T))) return rc;
  if ((rc = check_device())) return rc;
  return finish(launch_attention_prefill(qkv, ldqkv, B, T, c->n_q_heads, c->n_kv_heads, start_pos, kv->k, kv->v,
                                         kv->s_max, o, ldo, device_error_word(), static_cast<cudaStream_t>(stream),
                                         c->gemm_f16 != 0));
}

int qwen3_op_attention_decode(const qwen3_config* c, const qwen3_bf16* qkv, long long ldqkv, int B,
                              const int* cache_len, const qwen3_kv_layer* kv, qwen3_bf16* o, long long ldo, void* ws,
                              size_t ws_bytes, void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(qkv && cache_len && o && ws, QWEN3_EINVAL, "attention_decode: NULL pointer");
  Q3_CHECK(aligned16(qkv) && aligned16(o) && aligned16(ws), QWEN3_EALIGN, "attention_decode: misaligned pointer");
  Q3_CHECK(B > 0, QWEN3_EINVAL, "attention_decode: B must be positive");
  Q3_CHECK(ldqkv % 8 == 0 && ldqkv >= (long long)c->n_q_heads * c->head_dim, QWEN3_EALIGN,
           "attention_decode: ldqkv (%lld) must be a multiple of 8 and cover the query heads", ldqkv);
  Q3_CHECK(ldo % 8 == 0 && ldo >= (long long)c->n_q_heads * c->head_dim, QWEN3_EALIGN,
           "attention_decode: ldo (%lld) must be a multiple of 8 and at least n_q_heads * head_dim (%d)", ldo,
           c->n_q_heads * c->head_dim);
  if ((rc = check_kv(*c, kv, 1))) return rc;
  const size_t need = decode_partial_bytes(B, c->n_q_heads, c->n_kv_heads);
  Q3_CHECK(ws_bytes >= need, QWEN3_EWORKSPACE, "attention_decode: workspace has %zu bytes, needs %zu", ws_bytes, need);
  if ((rc = check_device())) return rc;
  return finish(launch_attention_decode(qkv, ldqkv, B, c->n_q_heads, c->n_kv_heads, cache_len, kv->k, kv->v,
                                        kv->s_max, static_cast<float*>(ws), o, ldo, device_error_word(),
                                        static_cast<cudaStream_t>(stream), c->gemm_f16 != 0));
}

int qwen3_op_attention_decode_noalloc(const qwen3_config* c, const qwen3_bf16* qkv, long long ldqkv, int B,
                                      const int* cache_len, const qwen3_kv_layer* kv, qwen3_bf16* o, long long ldo,
                                      void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(qkv && cache_len && o, QWEN3_EINVAL, "attention_decode_noalloc: NULL pointer");
  Q3_CHECK(aligned16(qkv) && aligned16(o), QWEN3_EALIGN, "attention_decode_noalloc: misaligned pointer");
  Q3_CHECK(B > 0, QWEN3_EINVAL, "attention_decode_noalloc: B must be positive");
  Q3_CHECK(ldqkv % 8 == 0 && ldqkv >= (long long)c->n_q_heads * c->head_dim, QWEN3_EALIGN,
           "attention_decode_noalloc: ldqkv (%lld) must be a multiple of 8 and cover the query heads", ldqkv);
  Q3_CHECK(ldo % 8 == 0 && ldo >= (long long)c->n_q_heads * c->head_dim, QWEN3_EALIGN,
           "attention_decode_noalloc: ldo (%lld) must be a multiple of 8 and at least n_q_heads * head_dim (%d)",
           ldo, c->n_q_heads * c->head_dim);
  if ((rc = check_kv(*c, kv, 1))) return rc;
  if ((rc = check_device())) return rc;
  return finish(launch_attention_decode_static(qkv, ldqkv, B, c->n_q_heads, c->n_kv_heads, cache_len, kv->k, kv->v,
                                               kv->s_max, o, ldo, device_error_word(),
                                               static_cast<cudaStream_t>(stream), c->gemm_f16 != 0));
}

int qwen3_op_argmax(const float* x, long long ldx, int rows, int V, int* out, long long ld_out, void* stream) {
  g_last_error.clear();
  Q3_CHECK(x && out, QWEN3_EINVAL, "argmax: NULL pointer");
  Q3_CHECK(rows > 0 && V > 0 && ld_out > 0, QWEN3_EINVAL, "argmax: rows, V and ld_out must be positive");
  Q3_CHECK(V % 4 == 0 && aligned16(x) && ldx % 4 == 0 && ldx >= V, QWEN3_EALIGN,
           "argmax: V and ldx must be multiples of 4 (16-byte rows), ldx >= V");
  int rc;
  if ((rc = check_device())) return rc;
  return finish(launch_argmax_rows(x, ldx, rows, V, out, ld_out, nullptr, static_cast<cudaStream_t>(stream)));
}

int qwen3_generate_greedy(const qwen3_config* c, const qwen3_bf16* embed, const qwen3_layer_weights* layers,
                          const qwen3_bf16* final_norm, const int* prompt_ids, int B, int T, int n_new,
                          const qwen3_kv_layer* kv, const float* rope, int* out_ids, void* ws, size_t ws_bytes,
                          void* stream) {
  g_last_error.clear();
  int rc = validate_cfg(c);
  if (rc) return rc;
  Q3_CHECK(prompt_ids && out_ids && kv && ws && layers, QWEN3_EINVAL, "generate: NULL argument");
  Q3_CHECK(aligned16(ws), QWEN3_EALIGN, "generate: workspace not 16-byte aligned");
  Q3_CHECK(B > 0 && T > 0 && n_new > 0, QWEN3_EINVAL, "generate: B (%d), T (%d) and n_new (%d) must be positive", B,
           T, n_new);
  const long long last_pos = (long long)T + n_new - 1;  // positions 0..last_pos-1 are written
  Q3_CHECK(last_pos - 1 < kv[0].s_max && last_pos - 1 < c->max_pos, QWEN3_ECAPACITY,
           "generate: positions up to %lld exceed the cache capacity (%d) or max_pos (%d)", last_pos - 1, kv[0].s_max,
           c->max_pos);
  const size_t need = qwen3_workspace_size(c, QWEN3_OP_GENERATE, B, T, kv[0].s_max);
  Q3_CHECK(need > 0 && ws_bytes >= need, QWEN3_EWORKSPACE, "generate: workspace has %zu bytes, needs %zu", ws_bytes,
           need);
  const size_t stack_bytes = generate_stack_bytes(*c, B, T, kv[0].s_max);
  char* base = static_cast<char*>(ws);
  float* logits = reinterpret_cast<float*>(base + stack_bytes);
  int* lens = reinterpret_cast<int*>(base + stack_bytes + (((size_t)B * c->vocab * sizeof(float) + 255) & ~(size_t)255));
  int* next = lens + ((((size_t)B * sizeof(int) + 255) & ~(size_t)255) / sizeof(int));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // prefill the prompt at positions 0..T-1, logits of each sequence's last position
  if ((rc = finish(launch_fill_lengths(lens, B, 0, s)))) return rc;
  if ((rc = qwen3_stack_forward(c, embed, layers, final_norm, prompt_ids, B, T, QWEN3_MODE_PREFILL, lens, kv, rope,
                                logits, 1, ws, stack_bytes, stream)))
    return rc;
  if ((rc = finish(launch_argmax_rows(logits, c->vocab, B, c->vocab, out_ids, n_new, next, s)))) return rc;
  if ((rc = finish(launch_fill_lengths(lens, B, T, s)))) return rc;
  // one decode step per further token; the stack advances lens on the device
  for (int t = 1; t < n_new; ++t) {
    if ((rc = qwen3_stack_forward(c, embed, layers, final_norm, next, B, 1, QWEN3_MODE_DECODE, lens, kv, rope,
                                  logits, 1, ws, stack_bytes, stream)))
      return rc;
    if ((rc = finish(launch_argmax_rows(logits, c->vocab, B, c->vocab, out_ids + t, n_new, next, s)))) return rc;
  }
  return 0;
}

int qwen3_op_embed(const int* ids, int n, const qwen3_bf16* embed, int vocab, int H, void* out, int out_f32,
                   int embed_f16, void* stream) {
  g_last_error.clear();
  Q3_CHECK(ids && embed && out, QWEN3_EINVAL, "embed: NULL pointer");
  Q3_CHECK(aligned16(embed) && aligned16(out), QWEN3_EALIGN, "embed: misaligned pointer");
  Q3_CHECK(n >= 0 && vocab > 0 && H > 0 && H % 8 == 0, QWEN3_ESHAPE, "embed: bad sizes");
  int rc = check_device();
  if (rc) return rc;
  return finish(launch_embed(ids, n, embed, vocab, H, out, out_f32 != 0, device_error_word(),
                             static_cast<cudaStream_t>(stream), nullptr, embed_f16 != 0));
}

int qwen3_convert_to_f16(const qwen3_bf16* in, qwen3_f16* out, size_t n, void* stream) {
  g_last_error.clear();
  Q3_CHECK(in && out, QWEN3_EINVAL, "convert_to_f16: NULL pointer");
  Q3_CHECK(aligned16(in) && aligned16(out), QWEN3_EALIGN, "convert_to_f16: misaligned pointer");
  Q3_CHECK(n > 0, QWEN3_EINVAL, "convert_to_f16: n must be positive");
  Q3_CHECK(in == out || reinterpret_cast<uintptr_t>(in) + 2 * n <= reinterpret_cast<uintptr_t>(out) ||
               reinterpret_cast<uintptr_t>(out) + 2 * n <= reinterpret_cast<uintptr_t>(in),
           QWEN3_EINVAL, "convert_to_f16: in and out overlap without being the same buffer");
  int rc = check_device();
  if (rc) return rc;
  return finish(launch_convert_to_f16(in, out, (long long)n, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
