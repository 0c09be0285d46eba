// K1 RMSNorm, K5 per-head QK-RMSNorm + rotate-half RoPE + KV-cache write, the
// embedding gather and the weight-interleave pack. All are HBM-bound: one warp
// per row (or per head), 16-byte (RMSNorm) or 4-byte coalesced accesses, fp32
// arithmetic, one bf16 rounding per output.
//
// Pages cited:
//   [P-Mini] "从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构" (quarkcode.cn)
//   [P-MoE]  "从零构建 Qwen-3 MoE" (adg.csdn.net)
#include "common.cuh"
#include "internal.h"

namespace q3 {

// ---------------------------------------------------------------------------
// K1: out = x * rsqrt(mean(x^2) + eps) * w  ([P-Mini] section RMSNorm, the
// x-hat formula: computed in fp32, cast back once). x is bf16 or fp32.
// One warp per row; each lane owns 8 consecutive elements of every 256-wide
// slice (n <= 2048, n % 256 == 0).
// ---------------------------------------------------------------------------
// A row of up to 1024 features is read once into registers (32 values per lane), then
// scaled and stored; longer rows take two passes (the second read hits L1).
template <bool IN_F32>
__device__ __forceinline__ void rms_load8(const void* x, long long off, float (&v)[8]) {
  if (IN_F32) {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + off);
    const float4 a = src[0], b = src[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + off);
    v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x); v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
    v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z); v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
  }
}

// zero_word (optional): an int this kernel sets to 0 (the fused-norm ticket of the
// call's decode-sized projections; see launch_gemm_skinny).
// OUT_F16: the output feeds an fp16-operand projection (bf16 otherwise).
// out_lo > 0: a lo copy lo = round(v - hi) of every output value, out_lo elements after it
// (the hi/lo operand of a decode-sized projection).
// r_out (optional): the row's 1/rms (the scale a deferred norm after the next projection
// starts from).
constexpr int kNormRegChunks = 4;  // rows of up to 4 x 256 features are read once, into registers

template <bool IN_F32, bool OUT_F16>
__global__ void __launch_bounds__(256, 4) rmsnorm_kernel(const void* __restrict__ x, long long ldx,
                                                         const uint16_t* __restrict__ w, uint16_t* __restrict__ out,
                                                         long long ldo, int rows, int n, float eps, int* zero_word,
                                                         long long out_lo, float* r_out) {
  pdl_wait();
  pdl_trigger();
  if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0;
  const int lane = threadIdx.x & 31;
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int n_warps = (gridDim.x * blockDim.x) >> 5;
  // the weighted, rounded output of 8 values at column col (hi, and lo when out_lo > 0)
  auto emit8 = [&](int row, int col, const float(&v)[8], float r) {
    const uint4 wv = *reinterpret_cast<const uint4*>(w + col);
    const float wf[8] = {bf16_lo(wv.x), bf16_hi(wv.x), bf16_lo(wv.y), bf16_hi(wv.y),
                         bf16_lo(wv.z), bf16_hi(wv.z), bf16_lo(wv.w), bf16_hi(wv.w)};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a0 = v[2 * j] * r * wf[2 * j], a1 = v[2 * j + 1] * r * wf[2 * j + 1];
      hi[j] = pack_op_x2(OUT_F16, a0, a1);
      lo[j] = pack_op_x2(OUT_F16, a0 - op_bits_to_f32(OUT_F16, (uint16_t)(hi[j] & 0xFFFFu)),
                         a1 - op_bits_to_f32(OUT_F16, (uint16_t)(hi[j] >> 16)));
    }
    uint16_t* dst = out + (long long)row * ldo + col;
    *reinterpret_cast<uint4*>(dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    if (out_lo) *reinterpret_cast<uint4*>(dst + out_lo) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  };
  for (int row = warp_global; row < rows; row += n_warps) {
    if (n <= 256 * kNormRegChunks) {
      // the whole row in registers: one read of x
      float v[kNormRegChunks][8];
#pragma unroll
      for (int c = 0; c < kNormRegChunks; ++c)
        if (c * 256 + lane * 8 < n) rms_load8<IN_F32>(x, (long long)row * ldx + c * 256 + lane * 8, v[c]);
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < kNormRegChunks; ++c)
        if (c * 256 + lane * 8 < n)
#pragma unroll
          for (int j = 0; j < 8; ++j) ss += v[c][j] * v[c][j];
      ss = warp_sum(ss);
      const float r = rsqrtf(ss / (float)n + eps);
      if (r_out && lane == 0) r_out[row] = r;
#pragma unroll
      for (int c = 0; c < kNormRegChunks; ++c)
        if (c * 256 + lane * 8 < n) emit8(row, c * 256 + lane * 8, v[c], r);
      continue;
    }
    float ss = 0.f;
    for (int col = lane * 8; col < n; col += 256) {
      float v[8];
      rms_load8<IN_F32>(x, (long long)row * ldx + col, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss += v[j] * v[j];
    }
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / (float)n + eps);
    if (r_out && lane == 0) r_out[row] = r;
    for (int col = lane * 8; col < n; col += 256) {
      float v[8];
      rms_load8<IN_F32>(x, (long long)row * ldx + col, v);
      emit8(row, col, v, r);
    }
  }
}

int launch_rmsnorm(const void* x, bool x_f32, long long ldx, const uint16_t* w, uint16_t* out, long long ldo,
                   int rows, int n, float eps, cudaStream_t s, int* zero_word, bool out_f16, long long out_lo,
                   float* r_out) {
  if (rows <= 0) return 0;
  const int warps_per_block = 8;
  long long blocks = (rows + warps_per_block - 1) / warps_per_block;
  if (blocks > (long long)num_sms() * 16) blocks = (long long)num_sms() * 16;
  auto k = x_f32 ? (out_f16 ? rmsnorm_kernel<true, true> : rmsnorm_kernel<true, false>)
                 : (out_f16 ? rmsnorm_kernel<false, true> : rmsnorm_kernel<false, false>);
  q3_launch(k, (int)blocks, 256, 0, s, x, ldx, w, out, ldo, rows, n, eps, zero_word, out_lo, r_out);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// ---------------------------------------------------------------------------
// K5: for every token m = b*T + t at absolute position pos = pos_base[b] + t and
// every head slot of the fused QKV row:
//   q heads: RMSNorm over the 128 dims with q_norm weights, then RoPE, written
//            back in place ([P-Mini] section GQA: q_norm / k_norm before RoPE);
//   k heads: the same with k_norm, written to the cache at [b][g][pos][:];
//   v heads: copied to the cache at [b][g][pos][:].
// RoPE pairs dimension i with i + 64 ([P-Mini] section RoPE):
//   (a, b) -> (a cos(pos theta_i) - b sin(pos theta_i), a sin(pos theta_i) + b cos(pos theta_i)),
// with cos/sin read from the fp32 table [max_pos][64][2] (cos, sin).
// One warp per (token, head slot); lane l owns dims {2l, 2l+1} and {64+2l, 65+2l}.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qk_norm_rope_kernel(uint16_t* __restrict__ qkv, long long ldqkv, int B, int T,
                                                           int Hq, int Hkv, const int* __restrict__ pos_base,
                                                           const uint16_t* __restrict__ qw,
                                                           const uint16_t* __restrict__ kw,
                                                           const float* __restrict__ rope, uint16_t* __restrict__ ck,
                                                           uint16_t* __restrict__ cv, int s_max, int max_pos,
                                                           float eps, int* err) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long item = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int slots = Hq + 2 * Hkv;
  const long long total = (long long)B * T * slots;
  if (item >= total) return;
  const int slot = (int)(item % slots);
  const long long m = item / slots;
  const int b = (int)(m / T), t = (int)(m % T);
  const int pos = pos_base[b] + t;
  if (pos < 0 || pos >= s_max || pos >= max_pos) {
    if (lane == 0) record_error(err, kErrCapacity);
    return;
  }
  uint16_t* row = qkv + m * ldqkv + (long long)slot * 128;
  const uint32_t x0 = *reinterpret_cast<const uint32_t*>(row + 2 * lane);
  const uint32_t x1 = *reinterpret_cast<const uint32_t*>(row + 64 + 2 * lane);
  if (slot >= Hq + Hkv) {  // value head: copy into the cache
    const int g = slot - Hq - Hkv;
    uint16_t* dst = cv + (((long long)b * Hkv + g) * s_max + pos) * 128;
    *reinterpret_cast<uint32_t*>(dst + 2 * lane) = x0;
    *reinterpret_cast<uint32_t*>(dst + 64 + 2 * lane) = x1;
    return;
  }
  const bool is_q = slot < Hq;
  const uint16_t* wn = is_q ? qw : kw;
  float a0 = bf16_lo(x0), a1 = bf16_hi(x0), b0 = bf16_lo(x1), b1 = bf16_hi(x1);
  const float ss = warp_sum(a0 * a0 + a1 * a1 + b0 * b0 + b1 * b1);
  const float r = rsqrtf(ss * (1.0f / 128.0f) + eps);
  const uint32_t wa = *reinterpret_cast<const uint32_t*>(wn + 2 * lane);
  const uint32_t wb = *reinterpret_cast<const uint32_t*>(wn + 64 + 2 * lane);
  a0 *= r * bf16_lo(wa); a1 *= r * bf16_hi(wa);
  b0 *= r * bf16_lo(wb); b1 *= r * bf16_hi(wb);
  const float4 cs = *reinterpret_cast<const float4*>(rope + ((long long)pos * 64 + 2 * lane) * 2);  // (c0, s0, c1, s1)
  const float o_a0 = a0 * cs.x - b0 * cs.y, o_b0 = a0 * cs.y + b0 * cs.x;
  const float o_a1 = a1 * cs.z - b1 * cs.w, o_b1 = a1 * cs.w + b1 * cs.z;
  uint16_t* dst;
  if (is_q) {
    dst = row;
  } else {
    const int g = slot - Hq;
    dst = ck + (((long long)b * Hkv + g) * s_max + pos) * 128;
  }
  *reinterpret_cast<uint32_t*>(dst + 2 * lane) = pack_bf16x2(o_a0, o_a1);
  *reinterpret_cast<uint32_t*>(dst + 64 + 2 * lane) = pack_bf16x2(o_b0, o_b1);
}

int launch_qk_norm_rope(uint16_t* qkv, long long ldqkv, int B, int T, int Hq, int Hkv, const int* pos_base,
                        const uint16_t* qw, const uint16_t* kw, const float* rope, uint16_t* ck, uint16_t* cv,
                        int s_max, int max_pos, float eps, int* err, cudaStream_t s) {
  const long long warps = (long long)B * T * (Hq + 2 * Hkv);
  if (warps == 0) return 0;
  const long long blocks = (warps * 32 + 255) / 256;
  q3_launch(qk_norm_rope_kernel, (unsigned)blocks, 256, 0, s, qkv, ldqkv, B, T, Hq, Hkv, pos_base, qw, kw, rope, ck, cv,
                                                       s_max, max_pos, eps, err);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// ---------------------------------------------------------------------------
// Embedding gather ([P-MoE] section 5; [P-Mini] section 骨架): out[m] = E[ids[m]],
// widened to fp32 when the residual stream is kept in fp32.
// ---------------------------------------------------------------------------
// E holds bf16, or fp16 (e_f16) in the fp16 operand mode; the fp32 output widens
// either exactly, a 16-bit output copies E's values unchanged.
__global__ void embed_kernel(const int* __restrict__ ids, int n, const uint16_t* __restrict__ E, int vocab, int H,
                             void* __restrict__ out, int out_f32, int e_f16, int* err, int* zero_word) {
  pdl_wait();
  pdl_trigger();
  if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0;
  const int m = blockIdx.x;
  if (m >= n) return;
  const int id = ids[m];
  if (id < 0 || id >= vocab) {
    if (threadIdx.x == 0) record_error(err, kErrInvalid);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(E + (long long)id * H);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    uint4 a = src[c];
    if (out_f32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + (long long)m * H + c * 8);
      if (e_f16) {
        const uint16_t* h = reinterpret_cast<const uint16_t*>(&a);
        dst[0] = make_float4(f16_bits_to_f32(h[0]), f16_bits_to_f32(h[1]), f16_bits_to_f32(h[2]), f16_bits_to_f32(h[3]));
        dst[1] = make_float4(f16_bits_to_f32(h[4]), f16_bits_to_f32(h[5]), f16_bits_to_f32(h[6]), f16_bits_to_f32(h[7]));
      } else {
        dst[0] = make_float4(bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y));
        dst[1] = make_float4(bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w));
      }
    } else {
      reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + (long long)m * H)[c] = a;
    }
  }
}

int launch_embed(const int* ids, int n, const uint16_t* E, int vocab, int H, void* out, bool out_f32, int* err,
                 cudaStream_t s, int* zero_word, bool e_f16) {
  if (n <= 0) return 0;
  q3_launch(embed_kernel, n, 128, 0, s, ids, n, E, vocab, H, out, out_f32 ? 1 : 0, e_f16 ? 1 : 0, err, zero_word);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// ---------------------------------------------------------------------------
// Gate/up interleave: packed rows [32j, 32j+16) = gate rows [16j, 16j+16),
// rows [32j+16, 32j+32) = up rows [16j, 16j+16), for n_mats matrices of I rows
// (dense FFN: separate gate and up; MoE: fused [E, 2I, H] split by chunk(2)).
// ---------------------------------------------------------------------------
__global__ void pack_gate_up_kernel(const uint16_t* __restrict__ gate, const uint16_t* __restrict__ up,
                                    long long mat_stride, int n_mats, int I, int H, uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const long long R = blockIdx.x;  // output row
  const long long rows = (long long)n_mats * 2 * I;
  if (R >= rows) return;
  const int mat = (int)(R / (2 * I));
  const int rr = (int)(R % (2 * I));
  const int blk = rr / 32, half = (rr / 16) & 1, r = rr % 16;
  const uint16_t* src = (half ? up : gate) + mat * mat_stride + (long long)(blk * 16 + r) * H;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(out + R * H);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) d4[c] = s4[c];
}

int launch_pack_gate_up(const uint16_t* gate, const uint16_t* up, long long mat_stride, int n_mats, int I, int H,
                        uint16_t* out, cudaStream_t s) {
  const long long rows = (long long)n_mats * 2 * I;
  if (rows == 0) return 0;
  q3_launch(pack_gate_up_kernel, (unsigned)rows, 128, 0, s, gate, up, mat_stride, n_mats, I, H, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// Decode bookkeeping: every sequence's cached length grows by one token.
__global__ void advance_lengths_kernel(int* len, int B) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] += 1;
}

int launch_advance_lengths(int* len, int B, cudaStream_t s) {
  if (B <= 0) return 0;
  q3_launch(advance_lengths_kernel, (B + 127) / 128, 128, 0, s, len, B);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// ---------------------------------------------------------------------------
// Greedy token choice: out[r * ld_out] = next[r] = argmax_j x[r][j] over the V fp32
// logits of row r, ties toward the lower id ([P-Mini] section prefill 与 decode: the
// next token comes from the last position's logits). One CTA of 1024 threads per row,
// 16-byte loads (V % 4 == 0); NaN never wins a comparison.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) argmax_rows_kernel(const float* __restrict__ x, long long ldx, int V,
                                                           int* __restrict__ out, long long ld_out,
                                                           int* __restrict__ next) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_v[32];
  __shared__ int s_i[32];
  const int r = blockIdx.x;
  const float4* row = reinterpret_cast<const float4*>(x + (long long)r * ldx);
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int c = threadIdx.x; c < V / 4; c += blockDim.x) {  // ascending ids per thread: strict > keeps the lower id
    const float4 v = row[c];
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (e[k] > best || (e[k] == best && 4 * c + k < bi)) { best = e[k]; bi = 4 * c + k; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) { s_v[warp] = best; s_i[warp] = bi; }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    best = lane < nw ? s_v[lane] : -INFINITY;
    bi = lane < nw ? s_i[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    if (lane == 0) {
      const int id = bi == 0x7fffffff ? 0 : bi;  // a row of NaN picks id 0
      out[(long long)r * ld_out] = id;
      if (next) next[r] = id;
    }
  }
}

int launch_argmax_rows(const float* x, long long ldx, int rows, int V, int* out, long long ld_out, int* next,
                       cudaStream_t s) {
  if (rows <= 0) return 0;
  q3_launch(argmax_rows_kernel, rows, 1024, 0, s, x, ldx, V, out, ld_out, next);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// len[b] = value for every sequence.
__global__ void fill_lengths_kernel(int* len, int B, int value) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] = value;
}

int launch_fill_lengths(int* len, int B, int value, cudaStream_t s) {
  if (B <= 0) return 0;
  q3_launch(fill_lengths_kernel, (B + 127) / 128, 128, 0, s, len, B, value);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}


// ---------------------------------------------------------------------------
// bf16 -> fp16 conversion (round to nearest even), 8 elements per thread where the
// buffers allow; in == out converts in place (each element is read before it is
// written, by the same thread).
// ---------------------------------------------------------------------------
__global__ void convert_to_f16_kernel(const uint16_t* in, uint16_t* out, long long n) {
  pdl_wait();
  pdl_trigger();
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long n8 = n / 8;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 a = reinterpret_cast<const uint4*>(in)[i];
    uint4 o;
    o.x = pack_f16x2(bf16_lo(a.x), bf16_hi(a.x));
    o.y = pack_f16x2(bf16_lo(a.y), bf16_hi(a.y));
    o.z = pack_f16x2(bf16_lo(a.z), bf16_hi(a.z));
    o.w = pack_f16x2(bf16_lo(a.w), bf16_hi(a.w));
    reinterpret_cast<uint4*>(out)[i] = o;
  }
  for (long long i = n8 * 8 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = to_f16_bits(__uint_as_float((uint32_t)in[i] << 16));
}

int launch_convert_to_f16(const uint16_t* in, uint16_t* out, long long n, cudaStream_t s) {
  if (n <= 0) return 0;
  long long blocks = (n / 8 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > (long long)num_sms() * 8) blocks = (long long)num_sms() * 8;
  q3_launch(convert_to_f16_kernel, (int)blocks, 256, 0, s, in, out, n);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

}  // namespace q3
