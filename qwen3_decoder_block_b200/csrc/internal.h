// Host-side declarations shared by the library's translation units.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace q3 {

enum Epilogue : int {
  kEpiStore = 0,   // out = acc (bf16 or f32)
  kEpiResid = 1,   // out = resid + acc (resid bf16 or f32; out bf16 or f32); may alias
  kEpiSwiglu = 2,  // operand rows interleaved in 16-row gate/up blocks: out = silu(g) * u, bf16
  kEpiQKRope = 3,  // fused QKV epilogue: per-head QK RMSNorm + RoPE (q in place), k/v to the cache
};

// Arguments of the fused QKV epilogue (non-swap GEMM over [q heads | k heads | v heads]).
struct QKRopeArgs {
  int T = 1, Hq = 0, Hkv = 0, s_max = 0, max_pos = 0;
  const int* pos_base = nullptr;  // [B]: token t of sequence b is at pos_base[b] + t
  const uint16_t* q_norm = nullptr;
  const uint16_t* k_norm = nullptr;
  const float* rope = nullptr;    // [max_pos][64][2] (cos, sin)
  uint16_t* ck = nullptr;         // [B][Hkv][s_max][128]
  uint16_t* cv = nullptr;
  float eps = 1e-6f;
  // decode-sized QKV only (optional): the q heads go to q2 [tokens][ldq2] instead of the
  // output, split as q_hi = bf16(q) and q_lo = bf16(q - q_hi): for KV group g the G hi
  // rows, then the G lo rows (the decode attention's hi/lo layout)
  uint16_t* q2 = nullptr;
  long long ldq2 = 0;
};

// D[p][q] = sum_k P[p][k] * Q[q][k]; both operands bf16, K-major (row-major [rows, K]).
// Non-swap: P = activations [M, K], Q = weights [N, K]; out[p][q].
// Swap:     P = weights [N, K], Q = activations [M, K]; out[q][p]  (for small M).
// Grouped, non-swap: P rows [off[g], off[g+1]) use Q rows g*q_rows_per_group + [0, q_rows_per_group).
// Grouped, swap (few activation rows per group): P = weights, group g's rows
// [g*p_rows, (g+1)*p_rows) (p_rows_total = n_groups * p_rows); Q = activations, group g's rows
// [off[g], off[g+1]) of q_rows; out[q][p - g*p_rows].
struct GemmDesc {
  const void* P = nullptr;
  int p_rows = 0;
  long long ldp = 0;  // elements
  const void* Q = nullptr;
  int q_rows = 0;     // non-grouped: rows of Q; grouped: rows per group
  long long ldq = 0;
  long long q_rows_total = 0;  // rows of the Q tensor map (grouped non-swap: n_groups * q_rows)
  long long p_rows_total = 0;  // rows of the P tensor map (grouped swap: n_groups * p_rows)
  int K = 0;
  bool swap = false;
  int epi = kEpiStore;
  bool resid_f32 = false, out_f32 = false;
  void* out = nullptr;
  long long ldo = 0;
  const void* resid = nullptr;
  long long ldr = 0;
  int n_groups = 0;
  const int* group_offsets = nullptr;  // device, n_groups + 1 entries
  int force_bn = 0;                    // 0 = automatic
  // operands fp16 (else bf16); the SwiGLU output and the fused RMSNorm output (norm_out),
  // which feed the next projection, then hold fp16 as well
  bool f16 = false;
  // P is final before the kernel launched just before this GEMM on the stream started
  // (a weight matrix, when a library kernel of the same call precedes the GEMM; every
  // library kernel waits for its predecessor before it lets its dependents launch):
  // the first tile's P loads may then precede the grid-dependency wait.
  bool p_early = false;
  QKRopeArgs qk;                       // kEpiQKRope only
  float* partial = nullptr;            // optional split-K scratch (fp32)
  size_t partial_bytes = 0;
  // When K is split, the kernel that sums the partials can also finish the next step:
  //  qk_in_reduce (store epilogue of the fused QKV projection): per-head QK-norm, RoPE
  //    and the KV-cache write, with the qk arguments (q written back to out);
  //  norm_out (residual epilogue): norm_out = RMSNorm(out) * norm_w for every token row
  //    (row stride ldo).
  // *fused is set to 1 when that happened, else left as it is.
  bool qk_in_reduce = false;
  const uint16_t* norm_w = nullptr;
  uint16_t* norm_out = nullptr;
  float norm_eps = 1e-6f;
  int* fused = nullptr;
};

// Decode-sized projection (M <= 64 tokens, N % 128 == 0, K % 64 == 0): out[t][n] =
// epilogue(sum_k A[t][k] W[n][k]) with K split over the CTAs of a cluster and summed
// in-kernel (gemm_skinny.cu). Epilogues: kEpiStore, kEpiResid (optionally followed by
// norm_out = RMSNorm(out) * norm_w over all N features, computed by the cluster that
// finishes last; `ticket` is an int that is 0 before the launch and 0 after it),
// kEpiSwiglu (out [M][N/2]), kEpiQKRope (q heads written back to out, k/v to the cache).
struct SkinnyDesc {
  const void* A = nullptr;  // activations [M][K] bf16
  long long lda = 0;
  const void* W = nullptr;  // weights [N][K] bf16
  long long ldw = 0;
  int M = 0, N = 0, K = 0;
  int epi = kEpiStore;
  void* out = nullptr;
  long long ldo = 0;
  bool out_f32 = false;
  const void* resid = nullptr;
  long long ldr = 0;
  bool resid_f32 = false;
  bool w_early = false;  // W is final before the previous kernel started (see GemmDesc::p_early)
  // residual epilogue only: norm_out = RMSNorm(out rows) * norm_w (N features per row),
  // through a grid-wide barrier on ticket[0..1] (ticket[0] zero before the launch) and
  // per-tile sums of squares in ssq ([N / 128][64] floats)
  const uint16_t* norm_w = nullptr;
  uint16_t* norm_out = nullptr;
  long long ld_norm = 0;
  float norm_eps = 1e-6f;
  int* ticket = nullptr;
  float* ssq = nullptr;
  // deferred norm (the next projection is one of these kernels): norm_out gets
  // y = out * norm_w * pre_scale[t] and ssq the per-tile sums of squares; no barrier
  bool norm_deferred = false;
  const float* pre_scale = nullptr;
  // the A rows are a deferred norm's y: scale token t's accumulators by r_t / row_s_in[t],
  // r_t = rsqrt(sum over ssq_tiles tiles of row_ssq[q * 64 + t] / ssq_n + ssq_eps); r_t is
  // written to row_r_out (also written by the grid-mode norm: r_t of its output rows)
  const float* row_ssq = nullptr;
  int ssq_tiles = 0, ssq_n = 0;
  float ssq_eps = 1e-6f;
  const float* row_s_in = nullptr;
  float* row_r_out = nullptr;
  QKRopeArgs qk;
  bool f16 = false;  // as GemmDesc::f16
  // a_hilo: A holds 2M rows, row t = hi(a_t), row M + t = lo(a_t) = round(a_t - hi), both in
  // the operand type; the product uses hi + lo (twice the precision of one 16-bit value)
  bool a_hilo = false;
  // optional lo copies for a following hi/lo consumer, written this many elements after
  // each hi value: norm_lo for norm_out, out_lo for the SwiGLU output
  long long norm_lo = 0;
  long long out_lo = 0;
  // at most this many CTAs (0: as many K splits as fit one wave), so that this launch and
  // the next projection's fit the SMs together and the next one's CTAs all start early
  int max_ctas = 0;
};

bool skinny_supported(int M, int N, int K, int epi);
int launch_gemm_skinny(const SkinnyDesc& d, cudaStream_t s, int* err);
// The CTAs launch_gemm_skinny would launch for d (feature tiles x K splits), 0 when the
// shape is unsupported. Host only.
int skinny_ctas(const SkinnyDesc& d);

// Scratch the block calls reserve for split-K partials of small-M GEMMs.
constexpr size_t kSplitKBytes = (size_t)2 * 148 * 128 * 256 * sizeof(float);

int launch_gemm(const GemmDesc& d, cudaStream_t s, int* err);

int num_sms();

// Every library kernel is launched with programmatic stream serialisation (its prologue
// may overlap the tail of the previous kernel; the kernel waits with griddepcontrol.wait
// before reading or writing global data). QWEN3_PDL=0 in the environment turns it off.
bool pdl_enabled();
bool gemm_pair_enabled();

template <typename... KArgs, typename... Args>
inline cudaError_t q3_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Same, launched as clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t q3_launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                     unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

int* device_error_word();  // device pointer of the library's error word

// Raises `func`'s dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device); *first (optional) tells whether this call set it. Returns 0 or -6
// (with the CUDA error in the last-error message).
int ensure_smem_attr(const void* func, int bytes, bool* first = nullptr);
void set_last_error(const char* fmt, ...);

}  // namespace q3
