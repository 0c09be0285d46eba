// K3: causal grouped-query prefill attention on tcgen05 tensor cores.
// K4: split-KV decode attention (memory bound, CUDA cores) + log-sum-exp merge.
//
// Both compute, for query head h at absolute position m and its KV group
// g = h / (Hq / Hkv),  o = softmax(q k^T / sqrt(128) + M) v  with M = -inf for keys
// after m ("从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构", section GQA, the
// attention formula; section prefill 与 decode: a decoded token sees every cached
// position and itself). Keys and values are read from the KV cache, which already
// holds this call's tokens (written by the QK-norm/RoPE kernel).
//
// Prefill design: one CTA per (q tile, kv group, sequence). The 128-row MMA tile
// packs 128/G tokens x the G query heads of one KV group, so every K/V tile is
// loaded once for the whole group. S = Q K^T goes to tensor memory (double
// buffered), 4 softmax warps (one row per thread) read it with tcgen05.ld, apply
// the causal mask and an online softmax in the exp2 domain with lazy rescaling
// of O (only when the running max grows by more than 2^8), write P as bf16 into a
// 128-byte swizzled shared tile, and O += P V accumulates in tensor memory with V
// as an MN-major operand. Causal tiles beyond the diagonal are skipped and the
// heaviest q tiles are scheduled first.
#include <mutex>
#include "common.cuh"
#include "internal.h"

namespace q3 {

int make_tmap_2d(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld, int box_rows);
int make_tmap_3d(CUtensorMap* map, const void* base, long long inner, long long mid, long long outer,
                 long long mid_stride_bytes, long long outer_stride_bytes, int box_inner, int box_mid, int box_outer);

namespace {

constexpr int kHeadDim = 128;
constexpr int kTileQ = 128;   // rows of one MMA tile (tokens x heads of one KV group)
constexpr int kTileK = 128;   // keys per KV tile
constexpr uint32_t kHalf = 128 * 64 * 2;  // one [128 rows][64] bf16 swizzled half tile: 16 KB
// shared memory (1024-aligned): Q tiles 0 and 1 (2 halves each), 2 stages x (K 2 halves, V 2 halves)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = 4 * kHalf;
constexpr uint32_t kStageBytes = 4 * kHalf;
constexpr uint32_t kOffBar = kOffKV + 2 * kStageBytes;
constexpr uint32_t kPrefillSmem = kOffBar + 256 + 1024;
constexpr int kPrefillThreads = 320;  // TMA warp, MMA warp, 2 softmax warpgroups
// log2(e) / sqrt(128)
constexpr float kScaleLog2 = 0.12751743074380304f;
constexpr float kRescaleThreshold = 8.0f;

struct PrefillParams {
  int B, T, Hq, Hkv, G, s_max, n_cta_q;
  const int* start_pos;
  uint16_t* out;
  long long ldo;
  int* err;
};

}  // namespace

// Tensor memory (512 columns): tile X in {0, 1} owns columns [256X, 256X+256):
// S_X = [256X, 256X+128) (fp32 scores; its first 64 columns are reused for the bf16
// probabilities P_X), O_X = [256X+128, 256X+256) (fp32 output accumulator).
__global__ void __launch_bounds__(kPrefillThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2] per stage
  uint64_t* v_full = bars + 3;    // [2] per stage
  uint64_t* kv_empty = bars + 5;  // [2] per stage
  uint64_t* s_full = bars + 7;    // [2] per Q tile
  uint64_t* p_full = bars + 9;    // [2] per Q tile
  uint64_t* pv_done = bars + 11;  // [2] per Q tile
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cq = p.n_cta_q - 1 - (int)blockIdx.x;  // heavy CTAs first
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = p.G, TQ = kTileQ / G;
  const int t0 = cq * 2 * TQ;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&v_full[i], 1); mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 128); mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // barrier set-up and the tensor-memory allocation overlap the previous kernel;
  // global data (positions, Q, the cache) is read only after the wait
  pdl_wait();
  pdl_trigger();
  const int start = p.start_pos[b];
  const int kv_limit = start + p.T;  // keys [0, kv_limit) are in the cache
  // KV tiles each Q tile needs (tile 1 holds the later tokens)
  const int nk0 = t0 < p.T ? (start + min(t0 + TQ, p.T) - 1) / kTileK + 1 : 0;
  const int nk1 = t0 + TQ < p.T ? (start + min(t0 + 2 * TQ, p.T) - 1) / kTileK + 1 : 0;
  const int n_kv = max(nk0, nk1);
  const long long kv_row0 = ((long long)b * p.Hkv + g) * p.s_max;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- TMA producer
      bool ok = true;
      long long issued = 0;
      mbar_arrive_expect_tx(q_full, 4 * kHalf);
      for (int X = 0; X < 2; ++X)
        for (int h = 0; h < 2; ++h)
          tma_load_3d(smem + kOffQ + (2 * X + h) * kHalf, &tmQ, q_full, 64 * h, g * G, b * p.T + t0 + X * TQ);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (*s_abort || !mbar_wait(&kv_empty[st], par ^ 1, p.err)) { ok = false; break; }
        uint8_t* base = smem + kOffKV + st * kStageBytes;
        const int row = (int)(kv_row0 + (long long)j * kTileK);
        mbar_arrive_expect_tx(&k_full[st], 2 * kHalf);
        tma_load_2d(base, &tmK, &k_full[st], 0, row);
        tma_load_2d(base + kHalf, &tmK, &k_full[st], 64, row);
        mbar_arrive_expect_tx(&v_full[st], 2 * kHalf);
        tma_load_2d(base + 2 * kHalf, &tmV, &v_full[st], 0, row);
        tma_load_2d(base + 3 * kHalf, &tmV, &v_full[st], 64, row);
        ++issued;
      }
      mbar_wait(q_full, 0, p.err);
      if (!ok) {
        *s_abort = 1;
        for (long long i = issued > 2 ? issued - 2 : 0; i < issued; ++i) {
          mbar_wait(&k_full[i & 1], (uint32_t)((i >> 1) & 1), p.err);
          mbar_wait(&v_full[i & 1], (uint32_t)((i >> 1) & 1), p.err);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTileK, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, kHeadDim, 0, 1);  // V is MN-major
      bool ok = mbar_wait(q_full, 0, p.err);
      const uint32_t sq = smem_u32(smem + kOffQ);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (*s_abort || !mbar_wait(&k_full[st], par, p.err)) { ok = false; break; }
        const uint32_t sk = smem_u32(smem + kOffKV + st * kStageBytes);
        for (int X = 0; X < 2 && ok; ++X) {
          if (j >= (X ? nk1 : nk0)) continue;
          // S_X reuses the columns of P_X of the previous tile: wait until that P.V is done
          if (j > 0 && (*s_abort || !mbar_wait(&pv_done[X], (j - 1) & 1, p.err))) { ok = false; break; }
          tc_fence_after();
          const uint32_t qa = sq + 2 * X * kHalf;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = sdesc_kmajor_sw128(qa + (kk >> 2) * kHalf) + 2 * (kk & 3);
            const uint64_t bd = sdesc_kmajor_sw128(sk + (kk >> 2) * kHalf) + 2 * (kk & 3);
            mma_bf16_ss(tmem + 256 * X, a, bd, idesc_s, kk ? 1u : 0u);
          }
          mma_commit(&s_full[X]);
        }
        if (!ok) break;
        if (*s_abort || !mbar_wait(&v_full[st], par, p.err)) { ok = false; break; }
        const uint32_t sv = sk + 2 * kHalf;
        for (int X = 0; X < 2 && ok; ++X) {
          if (j >= (X ? nk1 : nk0)) continue;
          if (*s_abort || !mbar_wait(&p_full[X], j & 1, p.err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bd = sdesc_mnmajor_sw128(sv + kk * 16 * 128, kHalf, 1024);
            mma_bf16_ts(tmem + 256 * X + 128, tmem + 256 * X + kk * 8, bd, idesc_o, (j | kk) ? 1u : 0u);
          }
          mma_commit(&pv_done[X]);
        }
        if (!ok) break;
        mma_commit(&kv_empty[st]);
      }
      if (!ok) {
        *s_abort = 1;
        mma_commit(drain);
        mbar_wait(drain, 0, p.err);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int X = (warp - 2) >> 2;  // which Q tile this warpgroup owns
    const int quad = warp & 3;      // tensor-memory lanes [32 quad, 32 quad + 32)
    const int r = quad * 32 + lane;
    const int t = t0 + X * TQ + r / G;
    const int qpos = start + t;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + 256 * X + lane_base;
    const uint32_t tO = tS + 128;
    const int nkx = X ? nk1 : nk0;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkx; ++j) {
      const int st = j & 1;
      bool w_ok = !*s_abort && mbar_wait(&s_full[X], j & 1, p.err);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      const int kv0 = j * kTileK;
      // only tiles touching the diagonal or the end of the cache need the mask
      const bool need_mask = __any_sync(0xffffffffu, kv0 + kTileK - 1 > qpos || kv0 + kTileK > kv_limit);
      // pass 1: row max, two 32-column chunks per tensor-memory round trip
      float mx = -INFINITY;
#pragma unroll
      for (int c2 = 0; c2 < 4; c2 += 2) {
        uint32_t v[2][32];
        tmem_ld32(tS + c2 * 32, v[0]);
        tmem_ld32(tS + c2 * 32 + 32, v[1]);
        tmem_wait_ld_regs(v[0]);
        tmem_wait_ld_regs(v[1]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int kp = kv0 + (c2 + h) * 32 + i;
              if (kp > qpos || kp >= kv_limit) v[h][i] = __float_as_uint(-INFINITY);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) mx = fmax3(mx, __uint_as_float(v[h][i]), __uint_as_float(v[h][i + 1]));
        }
      }
      const float mxs = mx * kScaleLog2;
      float alpha = 1.f;
      if (mxs > m_run + kRescaleThreshold || m_run == -INFINITY) {
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mxs);
        m_run = mxs;
      }
      // pass 2: p = 2^(s*scale - m) (packed fp32x2 FMA), row sums (packed adds), bf16 pairs
      // written over the columns already consumed
      const uint64_t scale2 = f2_pack(__float_as_uint(kScaleLog2), __float_as_uint(kScaleLog2));
      const uint64_t neg2 = f2_pack(__float_as_uint(-m_run), __float_as_uint(-m_run));
      uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
      for (int c2 = 0; c2 < 4; c2 += 2) {
        uint32_t v[2][32];
        tmem_ld32(tS + c2 * 32, v[0]);
        tmem_ld32(tS + c2 * 32 + 32, v[1]);
        tmem_wait_ld_regs(v[0]);
        tmem_wait_ld_regs(v[1]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int kp = kv0 + (c2 + h) * 32 + i;
              if (kp > qpos || kp >= kv_limit) v[h][i] = __float_as_uint(-INFINITY);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const uint64_t e = f2_fma(f2_pack(v[h][i], v[h][i + 1]), scale2, neg2);
            const float p0 = ex2_approx(f2_lo(e));
            const float p1 = ex2_approx(f2_hi(e));
            acc2[(i >> 1) & 1] = f2_add(acc2[(i >> 1) & 1], f2_pack(__float_as_uint(p0), __float_as_uint(p1)));
            v[h][i >> 1] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + (c2 + h) * 16, v[h]);  // columns [16c, 16c+16) were read already
        }
      }
      const uint64_t acc = f2_add(acc2[0], acc2[1]);
      const float sum_tile = f2_lo(acc) + f2_hi(acc);
      l_run = l_run * alpha + sum_tile;
      // O_X is stable here: S_X of this tile was issued only after the previous P.V completed
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld_regs(v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tmem_st32(tO + c * 32, v);
        }
      }
      // The last KV tile may extend past the written cache: zero those V rows so that
      // 0-probability keys cannot inject NaN/Inf through P.V. One warpgroup does it:
      // tile 0's if tile 0 takes part in this KV tile (its P.V is issued first).
      if (kv0 + kTileK > kv_limit && (X == 0 || j >= nk0)) {
        w_ok = !*s_abort && mbar_wait(&v_full[st], (j >> 1) & 1, p.err);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        if (kv0 + r >= kv_limit) {
          uint4* v0 = reinterpret_cast<uint4*>(smem + kOffKV + st * kStageBytes + 2 * kHalf + r * 128);
          uint4* v1 = reinterpret_cast<uint4*>(smem + kOffKV + st * kStageBytes + 3 * kHalf + r * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) { v0[c] = make_uint4(0, 0, 0, 0); v1[c] = make_uint4(0, 0, 0, 0); }
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[X]);
    }
    // epilogue: O / l -> bf16
    if (ok && nkx > 0) {
      bool w_ok = !*s_abort && mbar_wait(&pv_done[X], (nkx - 1) & 1, p.err);
      if (__all_sync(0xffffffffu, w_ok)) {
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        const int h = g * G + (r % G);
        uint16_t* dst = p.out + ((long long)b * p.T + t) * p.ldo + (long long)h * kHeadDim;
        const bool store = t < p.T;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld_regs(v);
          if (store) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]) * inv_l, __uint_as_float(v[8 * i + 1]) * inv_l);
              o.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]) * inv_l, __uint_as_float(v[8 * i + 3]) * inv_l);
              o.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]) * inv_l, __uint_as_float(v[8 * i + 5]) * inv_l);
              o.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]) * inv_l, __uint_as_float(v[8 * i + 7]) * inv_l);
              *reinterpret_cast<uint4*>(dst + c * 32 + i * 8) = o;
            }
          }
        }
      } else {
        *s_abort = 1;
      }
    } else if (!ok) {
      *s_abort = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int launch_attention_prefill(const uint16_t* qkv, long long ldqkv, int B, int T, int Hq, int Hkv,
                             const int* start_pos, const uint16_t* ck, const uint16_t* cv, int s_max, uint16_t* out,
                             long long ldo, int* err, cudaStream_t s) {
  if (B <= 0 || T <= 0) return 0;
  const int G = Hq / Hkv;
  const int TQ = kTileQ / G;
  CUtensorMap tmQ, tmK, tmV;
  // Q: (dim, head, token) with the G heads of one group and TQ tokens per box
  if (make_tmap_3d(&tmQ, qkv, kHeadDim, Hq, (long long)B * T, kHeadDim * 2, ldqkv * 2, 64, G, TQ) != 0) {
    set_last_error("attention: cannot encode the query tensor map");
    return -6;
  }
  const long long kv_rows = (long long)B * Hkv * s_max;
  if (make_tmap_2d(&tmK, ck, kv_rows, kHeadDim, kHeadDim, kTileK) != 0 ||
      make_tmap_2d(&tmV, cv, kv_rows, kHeadDim, kHeadDim, kTileK) != 0) {
    set_last_error("attention: cannot encode the KV-cache tensor maps");
    return -6;
  }
  PrefillParams p;
  p.B = B; p.T = T; p.Hq = Hq; p.Hkv = Hkv; p.G = G; p.s_max = s_max;
  p.n_cta_q = (T + 2 * TQ - 1) / (2 * TQ);
  p.start_pos = start_pos;
  p.out = out;
  p.ldo = ldo;
  p.err = err;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPrefillSmem);
    attr = true;
  }
  dim3 grid(p.n_cta_q, Hkv, B);
  q3_launch(attn_prefill_kernel, grid, kPrefillThreads, kPrefillSmem, s, tmQ, tmK, tmV, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("attention prefill launch failed: %s", cudaGetErrorString(e));
    return -6;
  }
  return 0;
}

// ============================================================================
// K4: split-KV decode attention. CTA (split, group, sequence) handles keys
// [split*256, split*256+256) of one sequence's KV group for all G query heads of
// the group, so each K/V line is read once. Warp w owns 32 consecutive keys:
//   scores: lane = key; the lane reads its key's 256-byte row straight from HBM
//           (16 x 16-byte loads in flight) and dots it with the G queries, which
//           sit pre-scaled in shared memory (broadcast reads);
//   softmax: per head over the warp's 32 keys (warp max / sum);
//   P V:    lane = 4 head dims; each key's V row is one coalesced 256-byte warp read.
// The 8 warps merge in shared memory; the split's (max, sum, unnormalised o) goes
// to the workspace and a second kernel merges the splits with log-sum-exp weights.
// ============================================================================
constexpr int kDecChunk = 256;
constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

template <int G>
__global__ void __launch_bounds__(kDecThreads) attn_decode_split_kernel(
    const uint16_t* __restrict__ qkv, long long ldqkv, int Hq, int Hkv, const int* __restrict__ cache_len,
    const uint16_t* __restrict__ ck, const uint16_t* __restrict__ cv, int s_max, int n_splits,
    float* __restrict__ part, int* err) {
  __shared__ __align__(16) float sQ[G][kHeadDim];
  __shared__ float sP[kDecWarps][G][32];
  __shared__ float sM[kDecWarps][G], sL[kDecWarps][G];
  __shared__ __align__(16) float sO[kDecWarps][G][kHeadDim];
  pdl_wait();
  pdl_trigger();

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_keys_total = cache_len[b] + 1;  // cached tokens + the new one
  const int k0 = split * kDecChunk;
  float* my_part = part + (((long long)b * Hq + g * G) * n_splits + split) * (kHeadDim + 2);
  const long long head_stride = (long long)n_splits * (kHeadDim + 2);
  if (k0 >= n_keys_total || n_keys_total > s_max) {
    if (n_keys_total > s_max && split == 0 && g == 0 && threadIdx.x == 0) record_error(err, kErrCapacity);
    if (threadIdx.x < G) {
      my_part[threadIdx.x * head_stride + kHeadDim] = -INFINITY;
      my_part[threadIdx.x * head_stride + kHeadDim + 1] = 0.f;
    }
    return;
  }
  for (int i = threadIdx.x; i < G * kHeadDim; i += kDecThreads) {
    const int j = i / kHeadDim, d = i % kHeadDim;
    sQ[j][d] = __uint_as_float((uint32_t)qkv[(long long)b * ldqkv + (long long)(g * G + j) * kHeadDim + d] << 16) *
               kScaleLog2;
  }
  __syncthreads();

  const long long row0 = ((long long)b * Hkv + g) * s_max;
  const int kw0 = k0 + warp * 32;  // first key of this warp
  const int key = kw0 + lane;
  const bool valid = key < n_keys_total;
  // ---- scores: one key per lane
  float s[G];
#pragma unroll
  for (int j = 0; j < G; ++j) s[j] = 0.f;
  if (valid) {
    const uint4* kr = reinterpret_cast<const uint4*>(ck + (row0 + key) * kHeadDim);
    uint4 kv[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) kv[c] = __ldg(kr + c);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float k8[8] = {bf16_lo(kv[c].x), bf16_hi(kv[c].x), bf16_lo(kv[c].y), bf16_hi(kv[c].y),
                           bf16_lo(kv[c].z), bf16_hi(kv[c].z), bf16_lo(kv[c].w), bf16_hi(kv[c].w)};
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float4 qa = *reinterpret_cast<const float4*>(&sQ[j][8 * c]);
        const float4 qb = *reinterpret_cast<const float4*>(&sQ[j][8 * c + 4]);
        s[j] += qa.x * k8[0] + qa.y * k8[1] + qa.z * k8[2] + qa.w * k8[3] + qb.x * k8[4] + qb.y * k8[5] +
                qb.z * k8[6] + qb.w * k8[7];
      }
    }
  }
  // ---- softmax over the warp's keys
  float m[G], l[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const float sj = valid ? s[j] : -INFINITY;
    m[j] = warp_max(sj);
    const float p = valid ? exp2f(sj - m[j]) : 0.f;
    l[j] = warp_sum(p);
    sP[warp][j][lane] = p;
  }
  __syncwarp();
  // ---- o = P V over the warp's keys, lane owns dims [4*lane, 4*lane+4)
  float o[G][4];
#pragma unroll
  for (int j = 0; j < G; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  const int nk = min(32, n_keys_total - kw0);
  const uint16_t* vbase = cv + (row0 + kw0) * kHeadDim + 4 * lane;
#pragma unroll 4
  for (int kk0 = 0; kk0 < 32; kk0 += 8) {
    uint2 vv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (kk0 + u < nk) vv[u] = __ldg(reinterpret_cast<const uint2*>(vbase + (long long)(kk0 + u) * kHeadDim));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (kk0 + u < nk) {
        const float v0 = bf16_lo(vv[u].x), v1 = bf16_hi(vv[u].x), v2 = bf16_lo(vv[u].y), v3 = bf16_hi(vv[u].y);
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const float p = sP[warp][j][kk0 + u];
          o[j][0] += p * v0; o[j][1] += p * v1; o[j][2] += p * v2; o[j][3] += p * v3;
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < G; ++j) {
    *reinterpret_cast<float4*>(&sO[warp][j][4 * lane]) = make_float4(o[j][0], o[j][1], o[j][2], o[j][3]);
    if (lane == 0) { sM[warp][j] = nk > 0 ? m[j] : -INFINITY; sL[warp][j] = nk > 0 ? l[j] : 0.f; }
  }
  __syncthreads();
  // ---- merge the warps into this split's partial
  for (int i = threadIdx.x; i < G * kHeadDim; i += kDecThreads) {
    const int j = i / kHeadDim, d = i % kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sM[w][j]);
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      if (sM[w][j] == -INFINITY) continue;
      const float sc = exp2f(sM[w][j] - M);
      acc += sO[w][j][d] * sc;
      L += sL[w][j] * sc;
    }
    my_part[j * head_stride + d] = acc;
    if (d == 0) {
      my_part[j * head_stride + kHeadDim] = M;
      my_part[j * head_stride + kHeadDim + 1] = L;
    }
  }
}

// ============================================================================
// K4, pipelined form (1, 2 or 4 query heads per KV group). Persistent: one CTA per
// SM walks the (sequence, group, 256-key split) items in a fixed order. A producer
// warp streams each split's K and V rows as two 128-key halves into a 3-stage ring
// of shared-memory buffers with bulk copies (the DMA engine, whole lines); 16 compute
// warps take 8 keys each. Scores: lane l holds 4 head dims of the G queries, partial
// dot products of the warp's 8 keys x G heads are reduced across lanes with a
// transposing butterfly (lane l ends with value l). Softmax is online across the two
// halves; P.V puts lane l on dims [4l, 4l+4). The 16 warps merge in shared memory and
// the split's (max, sum, unnormalised o) goes to the workspace, as in the form above.
// ============================================================================
constexpr int kD3Warps = 16;             // compute warps
constexpr int kD3Threads = 32 * (kD3Warps + 1);
constexpr int kD3Half = 128;             // keys per stage
constexpr int kD3Stages = 3;
constexpr uint32_t kD3StageBytes = 2u * kD3Half * kHeadDim * 2;  // K then V: 64 KB

template <int G>
struct D3Smem {
  static constexpr uint32_t kO = kD3Stages * kD3StageBytes;           // [16][G][128] fp32
  static constexpr uint32_t kM = kO + kD3Warps * G * kHeadDim * 4;    // [16][G]
  static constexpr uint32_t kL = kM + kD3Warps * G * 4;               // [16][G]
  static constexpr uint32_t kBar = (kL + kD3Warps * G * 4 + 7) & ~7u;  // full[3], empty[3]
  static constexpr uint32_t kAbort = kBar + 2 * kD3Stages * 8;
  static constexpr uint32_t kBytes = kAbort + 16 + 128;
};

// Butterfly that reduces NV (power of two, <= 32) per-lane values across the warp:
// afterwards lane l holds the full sum of value (l & (NV - 1)).
template <int NV>
__device__ __forceinline__ float transpose_reduce(float (&a)[NV], int lane) {
#pragma unroll
  for (int o = NV / 2; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float keep = upper ? a[i + o] : a[i];
      const float send = upper ? a[i] : a[i + o];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float v = a[0];
#pragma unroll
  for (int o = NV; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void named_bar_compute() {
  asm volatile("bar.sync 1, %0;" ::"n"(kD3Warps * 32) : "memory");
}

template <int G>
__global__ void __launch_bounds__(kD3Threads, 1) attn_decode_tma_kernel(
    const uint16_t* __restrict__ qkv, long long ldqkv, int B, int Hq, int Hkv, const int* __restrict__ cache_len,
    const uint16_t* __restrict__ ck, const uint16_t* __restrict__ cv, int s_max, int n_splits,
    float* __restrict__ part, int* err) {
  using L = D3Smem<G>;
  constexpr int NV = 8 * G;  // 8 keys x G heads per warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  float* sO = reinterpret_cast<float*>(smem + L::kO);
  float* sM = reinterpret_cast<float*>(smem + L::kM);
  float* sL = reinterpret_cast<float*>(smem + L::kL);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + kD3Stages;
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = B * Hkv * n_splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kD3Stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kD3Warps); }
    *s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  if (warp == kD3Warps) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0;
      long long issued = 0;
      for (int it = blockIdx.x; it < n_items && !*s_abort; it += gridDim.x) {
        const int split = it % n_splits, bg = it / n_splits, b = bg / Hkv;
        const int n_total = cache_len[b] + 1;
        if (n_total > s_max) continue;  // reported by the compute warps
        const long long row0 = (long long)bg * s_max;
        for (int h = 0; h < 2; ++h) {
          const int k0 = split * 2 * kD3Half + h * kD3Half;
          const int nk = min(kD3Half, n_total - k0);
          if (nk <= 0) continue;
          if (!mbar_wait(&empty[st], ph ^ 1, err)) { *s_abort = 1; break; }
          uint8_t* base = smem + st * kD3StageBytes;
          mbar_arrive_expect_tx(&full[st], 2u * nk * kHeadDim * 2);
          bulk_load(base, ck + (row0 + k0) * kHeadDim, nk * kHeadDim * 2, &full[st]);
          bulk_load(base + kD3StageBytes / 2, cv + (row0 + k0) * kHeadDim, nk * kHeadDim * 2, &full[st]);
          ++issued;
          if (++st == kD3Stages) { st = 0; ph ^= 1; }
        }
      }
      // every copy issued lands before the CTA exits (normally all were consumed already)
      for (long long i = issued > kD3Stages ? issued - kD3Stages : 0; i < issued; ++i)
        mbar_wait(&full[i % kD3Stages], (uint32_t)((i / kD3Stages) & 1), err);
    }
    return;  // the producer warp takes no part in the compute warps' named barrier
  }

  // -------------------------------------------------------------------- compute
  int st = 0;
  uint32_t ph = 0;
  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
    const int split = it % n_splits, bg = it / n_splits, b = bg / Hkv, g = bg % Hkv;
    const int n_total = cache_len[b] + 1;
    const bool over = n_total > s_max;
    if (over && split == 0 && g == 0 && threadIdx.x == 0) record_error(err, kErrCapacity);
    // this lane's 4 dims of the G queries, pre-scaled into the exp2 domain
    float qv[G][4];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const uint2 q2 = *reinterpret_cast<const uint2*>(qkv + (long long)b * ldqkv + (long long)(g * G + j) * kHeadDim +
                                                      4 * lane);
      qv[j][0] = bf16_lo(q2.x) * kScaleLog2; qv[j][1] = bf16_hi(q2.x) * kScaleLog2;
      qv[j][2] = bf16_lo(q2.y) * kScaleLog2; qv[j][3] = bf16_hi(q2.y) * kScaleLog2;
    }
    float m[G], l[G], o[G][4];
#pragma unroll
    for (int j = 0; j < G; ++j) { m[j] = -INFINITY; l[j] = 0.f; o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f; }
    for (int h = 0; h < 2 && !over; ++h) {
      const int k0 = split * 2 * kD3Half + h * kD3Half;
      const int nk = min(kD3Half, n_total - k0);
      if (nk <= 0) continue;
      const bool ok = !*s_abort && mbar_wait(&full[st], ph, err);
      if (!__all_sync(0xffffffffu, ok)) { *s_abort = 1; }
      const uint16_t* sK = reinterpret_cast<const uint16_t*>(smem + st * kD3StageBytes);
      const uint16_t* sV = sK + kD3Half * kHeadDim;
      const int kw = warp * 8;  // this warp's first key in the half
      if (!*s_abort) {
        // partial dot products: value index kk*G + j
        float a[NV];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          float k4[4] = {0.f, 0.f, 0.f, 0.f};
          if (kw + kk < nk) {
            const uint2 kr = *reinterpret_cast<const uint2*>(sK + (kw + kk) * kHeadDim + 4 * lane);
            k4[0] = bf16_lo(kr.x); k4[1] = bf16_hi(kr.x); k4[2] = bf16_lo(kr.y); k4[3] = bf16_hi(kr.y);
          }
#pragma unroll
          for (int j = 0; j < G; ++j)
            a[kk * G + j] = qv[j][0] * k4[0] + qv[j][1] * k4[1] + qv[j][2] * k4[2] + qv[j][3] * k4[3];
        }
        const float s = transpose_reduce<NV>(a, lane);
        const int vidx = lane & (NV - 1);
        const int my_key = vidx / G, my_j = vidx % G;
        const bool valid = kw + my_key < nk;
        // per-head max over the first NV lanes (lanes with the same head differ in bits >= log2 G)
        float mh = valid ? s : -INFINITY;
#pragma unroll
        for (int off = G; off < NV; off <<= 1) mh = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, off));
        float m_new[G], alpha[G];
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const float mj = __shfl_sync(0xffffffffu, mh, j);
          m_new[j] = fmaxf(m[j], mj);
          alpha[j] = (m[j] == -INFINITY) ? 0.f : exp2f(m[j] - m_new[j]);
        }
        float my_m = m_new[0];
#pragma unroll
        for (int j = 1; j < G; ++j) my_m = (my_j == j) ? m_new[j] : my_m;
        const float p = (valid && my_m != -INFINITY) ? exp2f(s - my_m) : 0.f;
        float ps = p;
#pragma unroll
        for (int off = G; off < NV; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
#pragma unroll
        for (int j = 0; j < G; ++j) {
          l[j] = l[j] * alpha[j] + __shfl_sync(0xffffffffu, ps, j);
          m[j] = m_new[j];
#pragma unroll
          for (int c = 0; c < 4; ++c) o[j][c] *= alpha[j];
        }
        // P.V: lane owns dims [4*lane, 4*lane+4)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          float pj[G];
#pragma unroll
          for (int j = 0; j < G; ++j) pj[j] = __shfl_sync(0xffffffffu, p, kk * G + j);
          if (kw + kk < nk) {
            const uint2 vr = *reinterpret_cast<const uint2*>(sV + (kw + kk) * kHeadDim + 4 * lane);
            const float v0 = bf16_lo(vr.x), v1 = bf16_hi(vr.x), v2 = bf16_lo(vr.y), v3 = bf16_hi(vr.y);
#pragma unroll
            for (int j = 0; j < G; ++j) {
              o[j][0] += pj[j] * v0; o[j][1] += pj[j] * v1; o[j][2] += pj[j] * v2; o[j][3] += pj[j] * v3;
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == kD3Stages) { st = 0; ph ^= 1; }
    }
    // merge the 16 warps into this split's partial
#pragma unroll
    for (int j = 0; j < G; ++j) {
      *reinterpret_cast<float4*>(&sO[(warp * G + j) * kHeadDim + 4 * lane]) = make_float4(o[j][0], o[j][1], o[j][2], o[j][3]);
      if (lane == 0) { sM[warp * G + j] = m[j]; sL[warp * G + j] = l[j]; }
    }
    named_bar_compute();
    float* my_part = part + ((long long)(b * Hq + g * G) * n_splits + split) * (kHeadDim + 2);
    const long long head_stride = (long long)n_splits * (kHeadDim + 2);
    for (int i = threadIdx.x; i < G * kHeadDim; i += kD3Warps * 32) {
      const int j = i / kHeadDim, d = i % kHeadDim;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kD3Warps; ++w) M = fmaxf(M, sM[w * G + j]);
      float acc = 0.f, Lsum = 0.f;
#pragma unroll
      for (int w = 0; w < kD3Warps; ++w) {
        const float mw = sM[w * G + j];
        if (mw == -INFINITY) continue;
        const float sc = exp2f(mw - M);
        acc += sO[(w * G + j) * kHeadDim + d] * sc;
        Lsum += sL[w * G + j] * sc;
      }
      my_part[j * head_stride + d] = acc;
      if (d == 0) {
        my_part[j * head_stride + kHeadDim] = M;
        my_part[j * head_stride + kHeadDim + 1] = Lsum;
      }
    }
    named_bar_compute();  // the next item overwrites sO / sM / sL
  }
}

__global__ void attn_decode_merge_kernel(const float* __restrict__ part, int Hq, int n_splits,
                                         uint16_t* __restrict__ out, long long ldo) {
  pdl_wait();
  pdl_trigger();
  const int bh = blockIdx.x;  // b * Hq + h
  const int b = bh / Hq, h = bh % Hq;
  const float* pp = part + (long long)bh * n_splits * (kHeadDim + 2);
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, pp[s * (kHeadDim + 2) + kHeadDim]);
  const int d = threadIdx.x;
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float* q = pp + s * (kHeadDim + 2);
    const float m = q[kHeadDim];
    if (m == -INFINITY) continue;
    const float w = exp2f(m - M);
    L += q[kHeadDim + 1] * w;
    acc += q[d] * w;
  }
  out[(long long)b * ldo + (long long)h * kHeadDim + d] = to_bf16_bits(acc / L);
}

int decode_splits(int s_max) { return (s_max + kDecChunk - 1) / kDecChunk; }

size_t decode_partial_bytes(int B, int Hq, int s_max) {
  return (size_t)B * Hq * decode_splits(s_max) * (kHeadDim + 2) * sizeof(float);
}

int launch_attention_decode(const uint16_t* qkv, long long ldqkv, int B, int Hq, int Hkv, const int* cache_len,
                            const uint16_t* ck, const uint16_t* cv, int s_max, float* part, uint16_t* out,
                            long long ldo, int* err, cudaStream_t s) {
  if (B <= 0) return 0;
  const int G = Hq / Hkv;
  const int n_splits = decode_splits(s_max);
  if (G == 1 || G == 2 || G == 4) {
    // pipelined form: persistent CTAs, bulk copies into a 3-stage shared-memory ring
    const long long items = (long long)B * Hkv * n_splits;
    const int grid = (int)(items < num_sms() ? items : num_sms());
    static bool attr[3] = {false, false, false};
#define Q3_D3_CASE(GG, SLOT)                                                                                     \
  case GG:                                                                                                       \
    if (!attr[SLOT]) {                                                                                           \
      cudaFuncSetAttribute(attn_decode_tma_kernel<GG>, cudaFuncAttributeMaxDynamicSharedMemorySize,              \
                           D3Smem<GG>::kBytes);                                                                  \
      attr[SLOT] = true;                                                                                         \
    }                                                                                                            \
    q3_launch(attn_decode_tma_kernel<GG>, grid, kD3Threads, D3Smem<GG>::kBytes, s, qkv, ldqkv, B, Hq, Hkv, cache_len, ck, \
                                                                           cv, s_max, n_splits, part, err);     \
    break;
    switch (G) {
      Q3_D3_CASE(1, 0)
      Q3_D3_CASE(2, 1)
      Q3_D3_CASE(4, 2)
    }
#undef Q3_D3_CASE
    q3_launch(attn_decode_merge_kernel, B * Hq, kHeadDim, 0, s, part, Hq, n_splits, out, ldo);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      set_last_error("attention decode launch failed: %s", cudaGetErrorString(e));
      return -6;
    }
    return 0;
  }
  dim3 grid(n_splits, Hkv, B);
  switch (G) {
#define Q3_DEC_CASE(GG)                                                                                         \
  case GG:                                                                                                      \
    q3_launch(attn_decode_split_kernel<GG>, grid, kDecThreads, 0, s, qkv, ldqkv, Hq, Hkv, cache_len, ck, cv, s_max,    \
                                                              n_splits, part, err);                            \
    break;
    Q3_DEC_CASE(1)
    Q3_DEC_CASE(2)
    Q3_DEC_CASE(4)
    Q3_DEC_CASE(8)
#undef Q3_DEC_CASE
    default:
      set_last_error("attention decode: %d query heads per KV group is not supported (1, 2, 4 or 8)", G);
      return -2;
  }
  q3_launch(attn_decode_merge_kernel, B * Hq, kHeadDim, 0, s, part, Hq, n_splits, out, ldo);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("attention decode launch failed: %s", cudaGetErrorString(e));
    return -6;
  }
  return 0;
}

// ----------------------------------------------------------------------------
// Decode attention without caller scratch. The split partials live in a fixed
// device array of this library instead of a caller workspace, for callers that
// cannot allocate device memory. Its capacity is kStaticDecodeFloats floats
// (12 MiB): B * Hq * ceil(s_max / 256) * 130 floats must fit. The array's device
// address is looked up on the host once per device (with that device current);
// every call shares the array, so calls that overlap on the GPU race. Each call
// rewrites every partial it reads, so nothing has to be cleared between calls.
// ----------------------------------------------------------------------------
constexpr size_t kStaticDecodeFloats = (size_t)3 << 20;
static __device__ __align__(256) float g_decode_scratch[kStaticDecodeFloats];

static std::mutex g_static_mu;
static float* g_static_ptr[64];

size_t static_decode_scratch_bytes() { return kStaticDecodeFloats * sizeof(float); }

int launch_attention_decode_static(const uint16_t* qkv, long long ldqkv, int B, int Hq, int Hkv,
                                   const int* cache_len, const uint16_t* ck, const uint16_t* cv, int s_max,
                                   uint16_t* out, long long ldo, int* err, cudaStream_t s) {
  const size_t need = decode_partial_bytes(B, Hq, s_max);
  if (need > kStaticDecodeFloats * sizeof(float)) {
    set_last_error("attention_decode_noalloc: B=%d, Hq=%d, s_max=%d need %zu bytes of split scratch; the "
                   "static scratch holds %zu bytes (B * Hq * ceil(s_max/256) must be <= %zu)",
                   B, Hq, s_max, need, kStaticDecodeFloats * sizeof(float), kStaticDecodeFloats / (kHeadDim + 2));
    return -5;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    set_last_error("attention_decode_noalloc: no current CUDA device");
    return -6;
  }
  float* ptr;
  {
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_ptr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess || !p) {
        set_last_error("attention_decode_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return -6;
      }
      g_static_ptr[dev] = static_cast<float*>(p);
    }
    ptr = g_static_ptr[dev];
  }
  return launch_attention_decode(qkv, ldqkv, B, Hq, Hkv, cache_len, ck, cv, s_max, ptr, out, ldo, err, s);
}

}  // namespace q3
