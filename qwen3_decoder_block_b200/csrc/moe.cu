// MoE FFN kernels: K6 router softmax / top-k / renormalise, K7 deterministic
// permutation (expert ascending, then token ascending) with the row gather,
// K9 weighted combine + residual in slot order. The expert SwiGLU GEMMs run on
// the grouped mode of the tcgen05 GEMM (K8).
//
// Routing follows "从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构" (quarkcode.cn),
// section MoE: router logits from a linear layer, probabilities by a float softmax,
// top-k, renormalised inside the top-k when norm_topk_prob, each selected expert's
// output scaled by its weight and accumulated into the token's row.
#include "common.cuh"
#include "internal.h"

namespace q3 {

// ---------------------------------------------------------------------------
// K6: one warp per token. logits fp32 [T, E] (E <= 256). Top-k by descending
// probability, ties toward the lower expert index. counts[e] += 1 per selection
// (counts must be zero on entry).
// ---------------------------------------------------------------------------
__global__ void moe_route_kernel(const float* __restrict__ logits, int T, int E, int k, int renorm,
                                 int* __restrict__ idx, float* __restrict__ w, int* __restrict__ counts) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  constexpr int kMaxPer = 8;  // E <= 256
  float p[kMaxPer];
  const int per = (E + 31) / 32;
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const int e = i * 32 + lane;
    p[i] = (i < per && e < E) ? logits[(long long)t * E + e] : -INFINITY;
    mx = fmaxf(mx, p[i]);
  }
  mx = warp_max(mx);
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) {
    const int e = i * 32 + lane;
    p[i] = (i < per && e < E) ? expf(p[i] - mx) : 0.f;
    sum += p[i];
  }
  sum = warp_sum(sum);
  const float inv = 1.f / sum;
#pragma unroll
  for (int i = 0; i < kMaxPer; ++i) p[i] *= inv;
  unsigned taken = 0;  // bit i: p[i] already selected
  float sel_sum = 0.f;
  float my_w = 0.f;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    float best = -1.f;
    int best_e = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
      const int e = i * 32 + lane;
      if (i < per && e < E && !(taken >> i & 1u) && p[i] > best) { best = p[i]; best_e = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oe = __shfl_xor_sync(0xffffffffu, best_e, o);
      if (ob > best || (ob == best && oe < best_e)) { best = ob; best_e = oe; }
    }
    if ((best_e & 31) == lane) taken |= 1u << (best_e >> 5);
    sel_sum += best;
    if (lane == j) { my_w = best; my_e = best_e; }
  }
  if (lane < k) {
    idx[(long long)t * k + lane] = my_e;
    w[(long long)t * k + lane] = renorm ? my_w / sel_sum : my_w;
    atomicAdd(&counts[my_e], 1);
  }
}

// ---------------------------------------------------------------------------
// K7: one CTA per expert e. offsets[e] = sum of counts below e; the CTA walks the
// tokens in order, and each token that picked e (at slot j) gets the next row of
// e's range: perm_token[row] = t, perm_slot[row] = j, inv_pos[t*k + j] = row.
// ---------------------------------------------------------------------------
constexpr int kPermThreads = 256;

__global__ void __launch_bounds__(kPermThreads) moe_permute_kernel(const int* __restrict__ idx, int T, int k, int E,
                                                                   const int* __restrict__ counts,
                                                                   int* __restrict__ offsets,
                                                                   int* __restrict__ perm_token,
                                                                   int* __restrict__ perm_slot,
                                                                   int* __restrict__ inv_pos) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  __shared__ int s_warp[kPermThreads / 32];
  __shared__ int s_base;
  // offset of expert e
  int part = 0;
  for (int i = threadIdx.x; i < e; i += blockDim.x) part += counts[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane == 0) s_warp[warp] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = 0;
    for (int i = 0; i < kPermThreads / 32; ++i) off += s_warp[i];
    s_base = off;
    offsets[e] = off;
    if (e == E - 1) offsets[E] = off + counts[e];
  }
  __syncthreads();
  int base = s_base;
  for (int t0 = 0; t0 < T; t0 += kPermThreads) {
    const int t = t0 + threadIdx.x;
    int slot = -1;
    if (t < T)
      for (int j = 0; j < k; ++j)
        if (idx[(long long)t * k + j] == e) { slot = j; break; }
    const unsigned bal = __ballot_sync(0xffffffffu, slot >= 0);
    __syncthreads();  // s_warp reuse
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < kPermThreads / 32; ++i) {
      const int c = s_warp[i];
      if (i < warp) before += c;
      total += c;
    }
    if (slot >= 0) {
      const int row = base + before + __popc(bal & ((1u << lane) - 1u));
      perm_token[row] = t;
      perm_slot[row] = slot;
      inv_pos[(long long)t * k + slot] = row;
    }
    base += total;
  }
}

// A_perm[row] = h[perm_token[row]]   (H % 8 == 0)
__global__ void moe_gather_kernel(const uint16_t* __restrict__ h, int H, const int* __restrict__ perm_token,
                                  int n_rows, uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  if (row >= n_rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(h + (long long)perm_token[row] * H);
  uint4* dst = reinterpret_cast<uint4*>(out + (long long)row * H);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) dst[c] = src[c];
}

// ---------------------------------------------------------------------------
// K9: out[t] = x1[t] + sum_{j=0..k-1} w[t][j] * Y[inv_pos[t][j]], summed in slot order
// in fp32. x1 fp32; out bf16 or fp32.
// ---------------------------------------------------------------------------
__global__ void moe_combine_kernel(const float* __restrict__ x1, const uint16_t* __restrict__ Y,
                                   const float* __restrict__ w, const int* __restrict__ inv_pos, int k, int H,
                                   void* __restrict__ out, int out_f32) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const float4* xs = reinterpret_cast<const float4*>(x1 + (long long)t * H + c * 8);
    float4 a = xs[0], b = xs[1];
    float acc[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    for (int j = 0; j < k; ++j) {
      const float wj = w[(long long)t * k + j];
      const uint4 y = *reinterpret_cast<const uint4*>(Y + (long long)inv_pos[(long long)t * k + j] * H + c * 8);
      acc[0] += wj * bf16_lo(y.x); acc[1] += wj * bf16_hi(y.x);
      acc[2] += wj * bf16_lo(y.y); acc[3] += wj * bf16_hi(y.y);
      acc[4] += wj * bf16_lo(y.z); acc[5] += wj * bf16_hi(y.z);
      acc[6] += wj * bf16_lo(y.w); acc[7] += wj * bf16_hi(y.w);
    }
    if (out_f32) {
      float4* d = reinterpret_cast<float4*>(static_cast<float*>(out) + (long long)t * H + c * 8);
      d[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      d[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint4 o = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + (long long)t * H + c * 8) = o;
    }
  }
}

int launch_moe_route(const float* logits, int T, int E, int k, int renorm, int* idx, float* w, int* counts,
                     cudaStream_t s) {
  if (T <= 0) return 0;
  if (cudaMemsetAsync(counts, 0, sizeof(int) * E, s) != cudaSuccess) return -6;
  const int warps_per_block = 8;
  q3_launch(moe_route_kernel, (T + warps_per_block - 1) / warps_per_block, 32 * warps_per_block, 0, s, logits, T, E, k,
                                                                                             renorm, idx, w, counts);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int launch_moe_permute(const int* idx, int T, int k, int E, const int* counts, int* offsets, int* perm_token,
                       int* perm_slot, int* inv_pos, const uint16_t* h, int H, uint16_t* a_perm, cudaStream_t s) {
  if (T <= 0) return 0;
  q3_launch(moe_permute_kernel, E, kPermThreads, 0, s, idx, T, k, E, counts, offsets, perm_token, perm_slot, inv_pos);
  q3_launch(moe_gather_kernel, T * k, 128, 0, s, h, H, perm_token, T * k, a_perm);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int launch_moe_combine(const float* x1, const uint16_t* Y, const float* w, const int* inv_pos, int T, int k, int H,
                       void* out, bool out_f32, cudaStream_t s) {
  if (T <= 0) return 0;
  q3_launch(moe_combine_kernel, T, 256, 0, s, x1, Y, w, inv_pos, k, H, out, out_f32 ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

}  // namespace q3
