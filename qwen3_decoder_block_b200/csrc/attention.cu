// K3: causal grouped-query prefill attention on tcgen05 tensor cores.
// K4: decode attention (memory bound; both products on tcgen05): the cache tiles of
//     all (sequence, KV group) rows are divided evenly among persistent CTAs, and a
//     row shared by several CTAs is merged (log-sum-exp) by the last of them.
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
// heaviest q tiles of all (group, sequence) pairs are scheduled first.
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
constexpr int kPrefillThreads = 384;  // softmax warpgroups (warps 0-3, 4-7), TMA warp 8, MMA warps 9-10
// Register split after the prologue: the softmax warpgroups hold a whole 128-column
// score row per thread; the third warpgroup (TMA, MMA, two idle warps) needs few.
// (2 x 200 + 88) x 128 registers must fit the launch allocation (384 x regs/thread).
constexpr int kPrefillRegsSoftmax = 200;
constexpr int kPrefillRegsCtl = 88;
constexpr int kPrefillRegBudget = (2 * kPrefillRegsSoftmax + kPrefillRegsCtl) * 128;
// log2(e) / sqrt(128)
constexpr float kScaleLog2 = 0.12751743074380304f;
constexpr float kRescaleThreshold = 8.0f;

struct PrefillParams {
  int B, T, Hq, Hkv, G, s_max, n_cta_q;
  int o_f16;  // o feeds an fp16-operand projection (bf16 otherwise)
  const int* start_pos;
  uint16_t* out;
  long long ldo;
  int* err;
};

}  // namespace

// Tensor memory (512 columns): tile X in {0, 1} owns columns [256X, 256X+256):
// S_X = [256X, 256X+128) (fp32 scores; columns [64, 128) are reused for the bf16
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
  uint64_t* s_read = bars + 13;   // [2] per Q tile: scores loaded into registers
  uint64_t* drain = bars + 15;    // [2] per MMA issuer
  uint64_t* mufu_tok = bars + 17; // [2] softmax X may start its exponentials
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Linear order, heaviest q tiles of every (group, sequence) first: the causal
  // work of a CTA grows with cq, so the block scheduler fills the SMs longest-first.
  const int gb = (int)(blockIdx.x % (unsigned)(p.Hkv * p.B));
  const int cq = p.n_cta_q - 1 - (int)(blockIdx.x / (unsigned)(p.Hkv * p.B));
  const int g = gb % p.Hkv, b = gb / p.Hkv;
  const int G = p.G, TQ = kTileQ / G;
  const int t0 = cq * 2 * TQ;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&v_full[i], 1); mbar_init(&kv_empty[i], 2);
      mbar_init(&s_read[i], 128); mbar_init(&drain[i], 1); mbar_init(&mufu_tok[i], 128);
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 128); mbar_init(&pv_done[i], 1);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
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

  if (warp >= 8) {
    regs_decrease<kPrefillRegsCtl>();
  if (warp == 8) {
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
  } else if (warp == 9 || warp == 10) {
    if (lane == 0) {
      // ------------------------------------------------- MMA issuers, one per Q tile
      // Each Q tile's chain S(j) -> softmax -> P.V(j) -> S(j+1) is issued by its own
      // thread, so neither chain waits behind the other's softmax.
      const int X = warp - 9;
      const int nkx = X ? nk1 : nk0;
      const int nk_other = X ? nk0 : nk1;
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);        // one 64-key half of S
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, kHeadDim, 0, 1);  // V is MN-major
      const uint32_t qa = smem_u32(smem + kOffQ) + 2 * X * kHalf;
      // S_X(j) in two N = 64 halves: keys [0, 64) into columns [0, 64) of S_X, keys
      // [64, 128) into [64, 128). P_X occupies columns [64, 128): the first half of
      // S_X(j+1) only needs the softmax to have read S_X(j), the second half needs
      // P.V(j) to be complete.
      auto issue_s_half = [&](int j, int h) -> bool {
        const int st = j & 1;
        if (*s_abort || !mbar_wait(&k_full[st], (j >> 1) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + kOffKV + st * kStageBytes) + h * 64 * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sdesc_kmajor_sw128(qa + (kk >> 2) * kHalf) + 2 * (kk & 3);
          const uint64_t bd = sdesc_kmajor_sw128(sk + (kk >> 2) * kHalf) + 2 * (kk & 3);
          mma_bf16_ss(tmem + 256 * X + 64 * h, a, bd, idesc_s, kk ? 1u : 0u);
        }
        if (h == 1) mma_commit(&s_full[X]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int st = j & 1;
        if (*s_abort || !mbar_wait(&v_full[st], (j >> 1) & 1, p.err)) return false;
        if (*s_abort || !mbar_wait(&p_full[X], j & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t sv = smem_u32(smem + kOffKV + st * kStageBytes + 2 * kHalf);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = sdesc_mnmajor_sw128(sv + kk * 16 * 128, kHalf, 1024);
          mma_bf16_ts(tmem + 256 * X + 128, tmem + 256 * X + 64 + kk * 8, bd, idesc_o, (j | kk) ? 1u : 0u);
        }
        mma_commit(&pv_done[X]);
        // the stage takes one arrival per Q tile; this chain also stands in for the
        // other tile when that tile does not use KV tile j
        mma_commit(&kv_empty[st]);
        if (j >= nk_other) mma_commit(&kv_empty[st]);
        return true;
      };
      bool ok = nkx > 0 ? mbar_wait(q_full, 0, p.err) : true;
      if (ok && nkx > 0) ok = issue_s_half(0, 0) && issue_s_half(0, 1);
      for (int j = 0; j < nkx && ok; ++j) {
        if (j + 1 < nkx) {
          if (*s_abort || !mbar_wait(&s_read[X], j & 1, p.err)) { ok = false; break; }
          tc_fence_after();
          if (!issue_s_half(j + 1, 0)) { ok = false; break; }
        }
        if (!issue_pv(j)) { ok = false; break; }
        if (j + 1 < nkx) {
          if (*s_abort || !mbar_wait(&pv_done[X], j & 1, p.err)) { ok = false; break; }
          tc_fence_after();
          if (!issue_s_half(j + 1, 1)) { ok = false; break; }
        }
      }
      if (!ok) {
        *s_abort = 1;
        mma_commit(&drain[X]);
        mbar_wait(&drain[X], 0, p.err);
      }
    }
  }
  } else {
    regs_increase<kPrefillRegsSoftmax>();
    // ---------------------------------------------------------------- softmax
    const int X = warp >> 2;        // which Q tile this warpgroup owns
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
      // the whole 128-column score row of this thread in one tensor-memory round trip
      uint32_t v[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, v[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_wait_ld_regs(v[c]);
      tc_fence_before();
      mbar_arrive(&s_read[X]);  // columns [0, 64) of S_X may now take the next tile's scores
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kp = kv0 + c * 32 + i;
            if (kp > qpos || kp >= kv_limit) v[c][i] = __float_as_uint(-INFINITY);
          }
      }
      // row max: four independent 3-input max chains
      float mc[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        mc[c] = __uint_as_float(v[c][0]);
#pragma unroll
        for (int i = 1; i < 31; i += 2) mc[c] = fmax3(mc[c], __uint_as_float(v[c][i]), __uint_as_float(v[c][i + 1]));
        mc[c] = fmaxf(mc[c], __uint_as_float(v[c][31]));
      }
      const float mxs = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])) * kScaleLog2;
      float alpha = 1.f;
      if (mxs > m_run + kRescaleThreshold || m_run == -INFINITY) {
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mxs);
        m_run = mxs;
      }
      // p = 2^(s*scale - m) (packed fp32x2 FMA), row sums (packed adds), bf16 pairs
      // written over columns [64, 128) (all scores are in registers already)
      const uint64_t scale2 = f2_pack(__float_as_uint(kScaleLog2), __float_as_uint(kScaleLog2));
      const uint64_t neg2 = f2_pack(__float_as_uint(-m_run), __float_as_uint(-m_run));
      uint64_t acc2[2] = {0ull, 0ull};
      // The two softmax warpgroups take turns on the exponentials (the special-function
      // unit is the bottleneck of the softmax): tile 0 of KV tile j goes after tile 1 of
      // KV tile j-1, tile 1 of KV tile j after tile 0 of KV tile j. Each turn overlaps
      // the tensor core's work on the other Q tile. A turn is only awaited while the
      // other warpgroup still has KV tiles.
      if (X == 0 ? (j >= 1 && j - 1 < nk1) : (j < nk0)) {
        w_ok = !*s_abort && mbar_wait(&mufu_tok[X], (uint32_t)((X == 0 ? j - 1 : j) & 1), p.err);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const uint64_t e = f2_fma(f2_pack(v[c][i], v[c][i + 1]), scale2, neg2);
          const float p0 = ex2_approx(f2_lo(e));
          const float p1 = ex2_approx(f2_hi(e));
          acc2[(i >> 1) & 1] = f2_add(acc2[(i >> 1) & 1], f2_pack(__float_as_uint(p0), __float_as_uint(p1)));
          v[c][i >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + 64 + c * 16, v[c]);
      }
      mbar_arrive(&mufu_tok[X ^ 1]);
      const uint64_t acc = f2_add(acc2[0], acc2[1]);
      const float sum_tile = f2_lo(acc) + f2_hi(acc);
      l_run = l_run * alpha + sum_tile;
      // O_X is stable here: the second half of S_X(j) was issued only after P.V of tile j-1 completed
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
      // 0-probability keys cannot inject NaN/Inf through P.V. Both Q tiles' P.V of
      // this KV tile are issued independently, so each warpgroup zeroes the rows
      // before releasing its own P (the second writes zeros over zeros).
      if (kv0 + kTileK > kv_limit) {
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
              const bool f16 = p.o_f16 != 0;
              o.x = pack_op_x2(f16, __uint_as_float(v[8 * i + 0]) * inv_l, __uint_as_float(v[8 * i + 1]) * inv_l);
              o.y = pack_op_x2(f16, __uint_as_float(v[8 * i + 2]) * inv_l, __uint_as_float(v[8 * i + 3]) * inv_l);
              o.z = pack_op_x2(f16, __uint_as_float(v[8 * i + 4]) * inv_l, __uint_as_float(v[8 * i + 5]) * inv_l);
              o.w = pack_op_x2(f16, __uint_as_float(v[8 * i + 6]) * inv_l, __uint_as_float(v[8 * i + 7]) * inv_l);
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int launch_attention_prefill(const uint16_t* qkv, long long ldqkv, int B, int T, int Hq, int Hkv,
                             const int* start_pos, const uint16_t* ck, const uint16_t* cv, int s_max, uint16_t* out,
                             long long ldo, int* err, cudaStream_t s, bool o_f16) {
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
  p.o_f16 = o_f16 ? 1 : 0;
  p.start_pos = start_pos;
  p.out = out;
  p.ldo = ldo;
  p.err = err;
  bool first = false;
  if (ensure_smem_attr(reinterpret_cast<const void*>(attn_prefill_kernel), kPrefillSmem, &first)) return -6;
  if (first) {
    // the register split must fit what the block is launched with, or the increase never returns
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_prefill_kernel) != cudaSuccess ||
        fa.numRegs * kPrefillThreads < kPrefillRegBudget) {
      set_last_error("attention prefill: kernel built with too few registers for its warpgroup split");
      return -6;
    }
  }
  const long long n_cta = (long long)p.n_cta_q * Hkv * B;
  if (n_cta >= (1ll << 31)) {
    set_last_error("attention prefill: %lld CTAs exceed the grid limit", n_cta);
    return -2;
  }
  dim3 grid((unsigned)n_cta);
  q3_launch(attn_prefill_kernel, grid, kPrefillThreads, kPrefillSmem, s, tmQ, tmK, tmV, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("attention prefill launch failed: %s", cudaGetErrorString(e));
    return -6;
  }
  return 0;
}

// ============================================================================
// K4, tensor-core form (any G in {1, 2, 4, 8, 16}). Persistent: the 128-key tiles of
// every (sequence b, KV group g) row, rows in order, form one list of T tiles, and CTA
// c of n takes tiles [c T / n, (c + 1) T / n) -- the same number of tiles per CTA
// whatever the lengths, and only a few row boundaries per CTA. A small plan kernel
// turns the lengths into the per-sequence tile prefix the CTAs search. Both products
// of a tile are tcgen05 MMAs with keys or head dims on the 128-row side and the G
// query heads of the group (padded to 16) as N:
//   S^T[key][j]  = sum_d K[key][d] q_j[d]      A = K tile (K-major), B = Q (K-major)
//   O^T[d][j]   += sum_key V[key][d] P[j][key]  A = V tile (MN-major), B = P (K-major)
// so the CUDA cores only run the softmax. A TMA warp streams Q, K and V of each tile
// into a 3-stage shared-memory ring (128-byte swizzle, whole 256-byte rows); one warp
// issues the scores of each tile as it lands (S double-buffered in tensor memory),
// another P.V and the stage's release; 8 softmax warps (4 for G = 1), two per
// tensor-memory lane quarter, own one key each (S) and one head dim each (O) for half
// of the group's heads: the tile maximum per head is a warp reduction plus a 4-quarter
// exchange, the online softmax rescales O only when the running maximum grows by more
// than 2^8, and P is written as bf16 into a swizzled K-major tile. A row that lies in
// one CTA is normalised and written at once; otherwise the CTAs after the row's first
// write their partial (unnormalised O, running maximum, sum) to the scratch and count
// it with a release add, and the row's first CTA, which reaches the row last, merges
// its own values with theirs in CTA order.
// ============================================================================
constexpr int kD4Stages = 3;
constexpr int kD4MaxCtas = 256;                    // grid bound (partial slots per call: rows + CTAs)
constexpr int kD4PartFloats = kHeadDim + 2;        // one head's partial: o[128], running max, sum
constexpr uint32_t kD4Half = 128 * 128;            // [128 rows][64] bf16, swizzled: 16 KB
constexpr uint32_t kD4QHalf = 16 * 128;            // [16 rows][64] bf16, swizzled: 2 KB
constexpr uint32_t kD4OffK = 0;
constexpr uint32_t kD4OffV = 2 * kD4Half;
constexpr uint32_t kD4OffQ = 4 * kD4Half;
constexpr uint32_t kD4StageBytes = 4 * kD4Half + 2 * kD4QHalf;  // 68 KB
constexpr uint32_t kD4OffP = kD4Stages * kD4StageBytes;         // P [2 buffers][16][128] as two K halves each
constexpr uint32_t kD4OffRed = kD4OffP + 4 * kD4QHalf;          // maxima [2][4][16], sums [4][16]
constexpr uint32_t kD4OffBar = kD4OffRed + (2 * 4 * 16 + 4 * 16) * 4;
constexpr uint32_t kD4Smem = kD4OffBar + 16 * 8 + 16 + 1024;
// softmax warps: two per tensor-memory lane quarter, each owning half of the group's
// heads (G >= 2), or one per quarter (G = 1); then the TMA warp and the MMA warp
// softmax warps per tensor-memory lane quarter, each owning G / that many of the heads
__host__ __device__ constexpr int d4_head_warps(int G) { return G >= 8 ? 4 : (G >= 2 ? 2 : 1); }
__host__ __device__ constexpr int d4_softmax_warps(int G) { return 4 * d4_head_warps(G); }
// softmax warps, then the TMA warp, the S-issuing warp and the P.V-issuing warp
__host__ __device__ constexpr int d4_threads(int G) { return 32 * (d4_softmax_warps(G) + 3); }
constexpr uint32_t kD4TmemCols = 64;  // S0 [0,16), S1 [16,32), O [32,48)

template <int SW>
__device__ __forceinline__ void named_bar_softmax() { asm volatile("bar.sync 1, %0;" ::"n"(32 * SW) : "memory"); }

// Log-sum-exp merge of one query head's partials (unnormalised o, running max in the
// exp2 domain, sum) for head dim d: o = sum_s o_s 2^(m_s - M) / sum_s l_s 2^(m_s - M),
// M = max_s m_s, partials in CTA order, read from L2 (other SMs wrote them). Written as
// bf16 or fp16, with an optional lo copy o_lo elements after it (the hi/lo operand of
// the decode-sized o_proj).
struct DecodeMergeOut {
  uint16_t* out;
  long long ldo;
  int o_f16;
  long long o_lo;
};
__device__ __forceinline__ void store_head_dim(float o, int d, uint16_t* dst, const DecodeMergeOut& mo) {
  const uint16_t hi = to_op_bits(mo.o_f16 != 0, o);
  dst[d] = hi;
  if (mo.o_lo) dst[mo.o_lo + d] = to_op_bits(mo.o_f16 != 0, o - op_bits_to_f32(mo.o_f16 != 0, hi));
}
// CTA c's tile range [c T / n, (c + 1) T / n) is empty (only when T < n).
__device__ __forceinline__ bool d4_cta_empty(int c, long long T, int n) {
  return T * c / n == T * (c + 1) / n;
}

// Merge of one head's partials of a row, by the row's first CTA: its own (m, l, o_d) are
// in registers and come first in the (deterministic) order; then the CTAs c_first + 1 ..
// c_last with a non-empty range, which wrote slot (row + c), `stride` floats apart from
// row_base's slot 0 numbering.
__device__ __forceinline__ void merge_row_dim_own(const float* row_base, int c_first, int c_last, long long T, int n,
                                                  long long stride, int d, float m_own, float l_own, float o_own,
                                                  uint16_t* dst, const DecodeMergeOut& mo) {
  float M = m_own;
  for (int c = c_first + 1; c <= c_last; ++c)
    if (!d4_cta_empty(c, T, n)) M = fmaxf(M, __ldcg(row_base + c * stride + kHeadDim));
  float L = 0.f, acc = 0.f;
  if (m_own != -INFINITY) {
    const float w = exp2f(m_own - M);
    L = l_own * w;
    acc = o_own * w;
  }
  for (int c = c_first + 1; c <= c_last; ++c) {
    if (d4_cta_empty(c, T, n)) continue;
    const float* q = row_base + c * stride;
    const float m = __ldcg(q + kHeadDim);
    if (m == -INFINITY) continue;
    const float w = exp2f(m - M);
    L += __ldcg(q + kHeadDim + 1) * w;
    acc += __ldcg(q + d) * w;
  }
  store_head_dim(acc / L, d, dst, mo);
}

// Maximum (MAX) or sum over the 32 lanes of each of G per-lane values, with log2(G) halving
// exchanges (each leaves a lane the half of the heads its lane bit selects) and then a
// plain butterfly over the remaining lane bits: G - 1 + 5 - log2(G) shuffles instead of
// 5 G. Lane l ends with head hd = l >> (5 - log2 G).
template <int G, bool MAX>
__device__ __forceinline__ float warp_reduce_heads(const float (&x)[G], int lane) {
  float a[G];
#pragma unroll
  for (int j = 0; j < G; ++j) a[j] = x[j];
#pragma unroll
  for (int half = G / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float send = upper ? a[k] : a[k + half];
      const float keep = upper ? a[k + half] : a[k];
      const float got = __shfl_xor_sync(0xffffffffu, send, bit);
      a[k] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
#pragma unroll
  for (int o = 16 / G; o > 0; o >>= 1) {
    const float got = __shfl_xor_sync(0xffffffffu, a[0], o);
    a[0] = MAX ? fmaxf(a[0], got) : a[0] + got;
  }
  return a[0];
}

// CTA holding global tile t when T tiles are divided among n CTAs as [c T / n, (c+1) T / n).
__device__ __forceinline__ int d4_cta_of(long long t, long long T, int n) { return (int)(((t + 1) * n - 1) / T); }

// Walk over the (sequence, group) rows that meet this CTA's tile range. plan[b] is the
// index of the first tile of sequence b's rows (Hkv rows of plan[b+1]-plan[b] tiles in
// all); rows of an over-capacity sequence hold no tiles.
struct D4Walk {
  const int* plan;
  int B, Hkv, b, g, nt;
  long long rs, t_begin, t_end;  // rs: global index of the current row's first tile
  __device__ D4Walk(const int* p, int B_, int Hkv_, int b0, long long tb, long long te)
      : plan(p), B(B_), Hkv(Hkv_), b(b0), g(0), nt(0), rs(te), t_begin(tb), t_end(te) {
    if (tb < te) {
      nt = (plan[b + 1] - plan[b]) / Hkv;
      g = (int)((tb - plan[b]) / nt);
      rs = plan[b] + (long long)g * nt;
    }
  }
  __device__ bool valid() const { return rs < t_end; }
  __device__ int j0() const { return (int)((t_begin > rs ? t_begin : rs) - rs); }
  __device__ int j1() const { return (int)((t_end < rs + nt ? t_end : rs + nt) - rs); }
  __device__ void next() {
    rs += nt;
    if (++g == Hkv) {
      g = 0;
      do { ++b; } while (b < B && plan[b + 1] == plan[b]);
      if (b < B) nt = (plan[b + 1] - plan[b]) / Hkv;
      else rs = t_end;
    }
  }
};

// HILO (G <= 8): q arrives as 2G rows per group, q_hi = bf16(q) in rows 0..G-1 and
// q_lo = bf16(q - q_hi) in rows G..2G-1, and P is written the same way, so the N = 16
// columns of both MMAs carry the hi and lo halves: S = K q_hi + K q_lo and
// O = V P_hi + V P_lo, summed in fp32 -- about 16 significant bits for q and P at no
// extra MMA instruction (the kernel is bound by the K/V stream).
// Element base + hh * GH + jj of a register array for the warp's head group hh (run
// time, < HW) and head jj (a constant after unrolling): only constant indices, so the
// array stays in registers.
template <int HW, int GH, int N>
__device__ __forceinline__ uint32_t pick_head(const uint32_t (&a)[N], int base, int hh, int jj) {
  uint32_t v = a[base + jj];
#pragma unroll
  for (int h = 1; h < HW; ++h)
    if (hh == h) v = a[base + h * GH + jj];
  return v;
}

template <int G, bool HILO>
__global__ void __launch_bounds__(d4_threads(G), 1)
    attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK16,
                          const __grid_constant__ CUtensorMap tmV16, int B, int Hq, int Hkv,
                          const int* __restrict__ cache_len, int s_max, const int* __restrict__ plan,
                          float* __restrict__ part, int* __restrict__ counters, const DecodeMergeOut mo, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kD4OffBar);
  uint64_t* full = bars;         // [3] stage loaded
  uint64_t* empty = bars + 3;    // [3] stage consumed
  uint64_t* s_full = bars + 6;   // [2] scores ready
  uint64_t* s_empty = bars + 8;  // [2] scores read
  uint64_t* p_full = bars + 10;  // [2] P buffer written (and O rescaled)
  uint64_t* pv_done = bars + 12; // [2] P.V of a tile using that buffer complete
  uint64_t* drain = bars + 14;     // the S issuer's MMAs complete
  uint64_t* drain_pv = bars + 15;  // the P.V issuer's MMAs complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_b0 = s_abort + 1;   // sequence holding this CTA's first tile
  volatile int* s_fix = s_abort + 2;  // 1 + first CTA of a row this CTA merges, else 0
  float* red_max = reinterpret_cast<float*>(smem + kD4OffRed);  // [2][4][16]
  float* red_sum = red_max + 2 * 4 * 16;                         // [4][16]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int SW = d4_softmax_warps(G);   // softmax warps; then the TMA warp SW, the MMA warps SW + 1 (S), SW + 2 (P.V)
  constexpr int HW = d4_head_warps(G);      // softmax warps per lane quarter
  constexpr int GH = G / HW;                 // heads per softmax warp

  if (threadIdx.x == 0) {
    for (int i = 0; i < kD4Stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 32 * SW); }
    for (int i = 0; i < 2; ++i) { mbar_init(&p_full[i], 32 * SW); mbar_init(&pv_done[i], 1); }
    mbar_init(drain, 1);
    mbar_init(drain_pv, 1);
    *s_abort = 0;
    *s_b0 = 0;
    fence_barrier_init();
  }
  // Rows G..15 of the Q and P operand tiles are never written: clear all of them once.
  for (int i = threadIdx.x; i < (2 * kD4Stages + 4) * (int)(kD4QHalf / 16); i += blockDim.x) {
    const int buf = i / (int)(kD4QHalf / 16), off = i % (int)(kD4QHalf / 16);
    uint8_t* base = buf < 2 * kD4Stages ? smem + (buf >> 1) * kD4StageBytes + kD4OffQ + (buf & 1) * kD4QHalf
                                        : smem + kD4OffP + (buf - 2 * kD4Stages) * kD4QHalf;
    reinterpret_cast<uint4*>(base)[off] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 32 * SW) {
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmK16); tma_prefetch_desc(&tmV16);
  }
  if (warp == SW + 1) { tmem_alloc(tmem_slot, kD4TmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();
  // this CTA's tiles [t_begin, t_end) of the T in the call; the sequence holding t_begin
  const long long T = plan[B];
  const int n_cta = (int)gridDim.x;
  const long long t_begin = T * blockIdx.x / n_cta, t_end = T * (blockIdx.x + 1) / n_cta;
  for (int b = threadIdx.x; b < B; b += blockDim.x)
    if (plan[b] <= t_begin && t_begin < plan[b + 1]) *s_b0 = b;
  __syncthreads();
  const int b0 = *s_b0;

  if (warp == SW) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      long long tc = 0;
      bool ok = true;
      for (D4Walk w(plan, B, Hkv, b0, t_begin, t_end); w.valid() && ok; w.next()) {
        const int b = w.b, g = w.g, bg = b * Hkv + g;
        const int row0 = bg * s_max;
        const int n_total = cache_len[b] + 1;
        for (int j = w.j0(); j < w.j1(); ++j) {
          const int k0 = j * 128;
          const int st = (int)(tc % kD4Stages);
          if (*s_abort || !mbar_wait(&empty[st], (uint32_t)((tc / kD4Stages) & 1) ^ 1u, err)) { ok = false; break; }
          uint8_t* base = smem + st * kD4StageBytes;
          constexpr int QR = HILO ? 2 * G : G;  // query rows of a group in the tile
          // a row's last tile: only the boxes of 16 keys that hold visible keys (the other
          // rows keep stale data; their scores are masked and their V rows zeroed)
          const int nb = n_total - k0 >= 128 ? 0 : (n_total - k0 + 15) / 16;
          mbar_arrive_expect_tx(&full[st], (nb ? nb * 4 * 16 * 128 : 4 * kD4Half) + 2 * QR * 128);
          tma_load_3d(base + kD4OffQ, &tmQ, &full[st], 0, g * QR, b);
          tma_load_3d(base + kD4OffQ + kD4QHalf, &tmQ, &full[st], 64, g * QR, b);
          if (nb == 0) {
            tma_load_2d(base + kD4OffK, &tmK, &full[st], 0, row0 + k0);
            tma_load_2d(base + kD4OffK + kD4Half, &tmK, &full[st], 64, row0 + k0);
            tma_load_2d(base + kD4OffV, &tmV, &full[st], 0, row0 + k0);
            tma_load_2d(base + kD4OffV + kD4Half, &tmV, &full[st], 64, row0 + k0);
          } else {
            for (int i = 0; i < nb; ++i) {  // 16 rows of 128 bytes per box: 2 KB, swizzle phase kept
              const int r = row0 + k0 + 16 * i;
              tma_load_2d(base + kD4OffK + i * 2048, &tmK16, &full[st], 0, r);
              tma_load_2d(base + kD4OffK + kD4Half + i * 2048, &tmK16, &full[st], 64, r);
              tma_load_2d(base + kD4OffV + i * 2048, &tmV16, &full[st], 0, r);
              tma_load_2d(base + kD4OffV + kD4Half + i * 2048, &tmV16, &full[st], 64, r);
            }
          }
          ++tc;
        }
      }
      if (!ok) {
        *s_abort = 1;
        // let the copies still in flight land before the CTA exits
        for (long long i = tc > kD4Stages ? tc - kD4Stages : 0; i < tc; ++i)
          mbar_wait(&full[i % kD4Stages], (uint32_t)((i / kD4Stages) & 1), err);
      }
    }
  } else if (warp == SW + 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ S issuer: S = K q
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 16, 0, 0);
      long long tc = 0;
      bool ok = true;
      for (D4Walk w(plan, B, Hkv, b0, t_begin, t_end); w.valid() && ok; w.next()) {
        const int jb = w.j0(), je = w.j1();
        for (int j = jb; j < je; ++j) {
          const int st = (int)(tc % kD4Stages), sb = (int)(tc & 1);
          if (*s_abort || !mbar_wait(&full[st], (uint32_t)((tc / kD4Stages) & 1), err)) { ok = false; break; }
          if (tc >= 2 && (*s_abort || !mbar_wait(&s_empty[sb], (uint32_t)(((tc - 2) >> 1) & 1), err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + st * kD4StageBytes + kD4OffK);
          const uint32_t sQ = smem_u32(smem + st * kD4StageBytes + kD4OffQ);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = sdesc_kmajor_sw128(sK + (kk >> 2) * kD4Half) + 2 * (kk & 3);
            const uint64_t bq = sdesc_kmajor_sw128(sQ + (kk >> 2) * kD4QHalf) + 2 * (kk & 3);
            mma_bf16_ss(tmem + 16 * sb, a, bq, idesc_s, kk ? 1u : 0u);
          }
          mma_commit(&s_full[sb]);
          ++tc;
        }
      }
      if (!ok) *s_abort = 1;
      // every MMA completes before the tensor memory is released
      mma_commit(drain);
      mbar_wait(drain, 0, err);
    }
  } else if (warp == SW + 2) {
    if (lane == 0) {
      // -------------------------------------------- P.V issuer: O^T += V^T P^T, stage release
      // Its own warp, so that a stage is released as soon as its P is written, whether or
      // not the next tile's data has landed. P of tile u is in buffer u & 1, whose barriers
      // advance once every second tile; the first tile of a split overwrites O. S of tile u
      // completed before its P was written, so this warp's commit also frees the stage's K.
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 16, 1, 0);  // V^T: MN-major A
      const uint32_t sP = smem_u32(smem + kD4OffP);
      long long tc = 0;
      bool ok = true;
      for (D4Walk w(plan, B, Hkv, b0, t_begin, t_end); w.valid() && ok; w.next()) {
        const int jb = w.j0(), je = w.j1();
        for (int j = jb; j < je; ++j) {
          const int st = (int)(tc % kD4Stages), pb = (int)(tc & 1);
          // the stage's copies (V), observed here too, then the tile's P
          if (*s_abort || !mbar_wait(&full[st], (uint32_t)((tc / kD4Stages) & 1), err) ||
              !mbar_wait(&p_full[pb], (uint32_t)((tc >> 1) & 1), err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sV = smem_u32(smem + st * kD4StageBytes + kD4OffV);
          const uint32_t sPb = sP + pb * 2 * kD4QHalf;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = sdesc_mnmajor_sw128(sV + kk * 16 * 128, kD4Half, 1024);
            const uint64_t bp = sdesc_kmajor_sw128(sPb + (kk >> 2) * kD4QHalf) + 2 * (kk & 3);
            mma_bf16_ss(tmem + 32, a, bp, idesc_o, (j == jb && kk == 0) ? 0u : 1u);
          }
          mma_commit(&pv_done[pb]);
          mma_commit(&empty[st]);
          ++tc;
        }
      }
      if (!ok) *s_abort = 1;
      mma_commit(drain_pv);
      mbar_wait(drain_pv, 0, err);
    }
  } else {
    // -------------------------------------------------------------------- softmax
    // warp (quarter q, half hh): key / head dim t of lanes [32 q, 32 q + 32), heads
    // [j0, j0 + GH) of the group
    const int q = warp & 3, hh = warp >> 2, j0 = hh * GH;
    const int t = q * 32 + lane;  // key of the tile (S) / head dim (O)
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    long long tc = 0;
    bool ok = true;
    for (D4Walk w(plan, B, Hkv, b0, t_begin, t_end); w.valid(); w.next()) {
      const int b = w.b, g = w.g, bg = b * Hkv + g;
      const int n_total = cache_len[b] + 1;
      const int jb = w.j0(), je = w.j1();
      float m_run[GH], l_part[GH];
#pragma unroll
      for (int j = 0; j < GH; ++j) { m_run[j] = -INFINITY; l_part[j] = 0.f; }
      int n_tiles = 0;
      for (int j = jb; j < je; ++j) {
        const int k0 = j * 128;
        const int nk = min(128, n_total - k0);
        const int sb = (int)(tc & 1);
        ok = ok && !*s_abort && mbar_wait(&s_full[sb], (uint32_t)((tc >> 1) & 1), err);
        ok = __all_sync(0xffffffffu, ok);
        uint32_t sv[16];
        if (ok) {
          tc_fence_after();
          tmem_ld16(tl + 16 * sb, sv);
          tmem_wait_ld_regs16(sv);
        }
        tc_fence_before();
        mbar_arrive(&s_empty[sb]);
        float s[GH];
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          const float sj = HILO ? __uint_as_float(pick_head<HW, GH>(sv, 0, hh, jj)) + __uint_as_float(pick_head<HW, GH>(sv, G, hh, jj)) : __uint_as_float(pick_head<HW, GH>(sv, 0, hh, jj));
          s[jj] = (ok && t < nk) ? sj * kScaleLog2 : -INFINITY;
        }
        // tile maximum per head: the warp's 32 keys, then the 4 quarters
        float* rm = red_max + (tc & 1) * 64;
        {
          const float wm = warp_reduce_heads<GH, true>(s, lane);
          if ((lane & (32 / GH - 1)) == 0) rm[q * 16 + j0 + lane / (32 / GH)] = wm;
        }
        named_bar_softmax<SW>();
        float alpha[GH];
        bool rescale = false;
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          const int hd = j0 + jj;
          const float mt = fmaxf(fmaxf(rm[hd], rm[16 + hd]), fmaxf(rm[32 + hd], rm[48 + hd]));
          alpha[jj] = 1.f;
          if (mt > m_run[jj] + kRescaleThreshold || m_run[jj] == -INFINITY) {
            alpha[jj] = (m_run[jj] == -INFINITY) ? 0.f : ex2_approx(m_run[jj] - mt);
            m_run[jj] = mt;
            rescale = true;
          }
        }
        float p[GH];
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          p[jj] = (t < nk && m_run[jj] != -INFINITY) ? ex2_approx(s[jj] - m_run[jj]) : 0.f;
          l_part[jj] = l_part[jj] * alpha[jj] + p[jj];
        }
        // P is double-buffered: buffer tc & 1 was last read by the P.V of tile tc - 2. A
        // rescale of O (below) needs the P.V of tile tc - 1 complete as well.
        const int pbuf = (int)(tc & 1);
        if (tc >= 2) {
          ok = ok && !*s_abort && mbar_wait(&pv_done[pbuf], (uint32_t)(((tc - 2) >> 1) & 1), err);
          ok = __all_sync(0xffffffffu, ok);
        }
        if (n_tiles > 0 && rescale) {  // uniform within the warp: its lanes hold the same maxima
          ok = ok && !*s_abort && mbar_wait(&pv_done[pbuf ^ 1], (uint32_t)(((tc - 1) >> 1) & 1), err);
          ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
          tc_fence_after();
          if (n_tiles > 0 && rescale) {
            // this warp's own O columns only (head hd: column hd, and G + hd for the lo half)
            uint32_t ov[16];
            tmem_ld16(tl + 32, ov);
            tmem_wait_ld_regs16(ov);
#pragma unroll
            for (int jj = 0; jj < GH; ++jj) {
              const int hd = j0 + jj;
              tmem_st1(tl + 32 + hd, __float_as_uint(__uint_as_float(pick_head<HW, GH>(ov, 0, hh, jj)) * alpha[jj]));
              if (HILO) tmem_st1(tl + 32 + G + hd, __float_as_uint(__uint_as_float(pick_head<HW, GH>(ov, G, hh, jj)) * alpha[jj]));
            }
            tmem_wait_st();
          }
          // P[j][t] into the K-major B tile of buffer pbuf: row j, key t, 128-byte swizzle
          uint8_t* pb = smem + kD4OffP + pbuf * 2 * kD4QHalf + (t >> 6) * kD4QHalf + (t & 7) * 2;
          const int chunk = (t & 63) >> 3;
#pragma unroll
          for (int jj = 0; jj < GH; ++jj) {
            const int hd = j0 + jj;
            const uint16_t hi = to_bf16_bits(p[jj]);
            *reinterpret_cast<uint16_t*>(pb + hd * 128 + ((chunk ^ (hd & 7)) << 4)) = hi;
            if (HILO) {
              const int jl = G + hd;
              *reinterpret_cast<uint16_t*>(pb + jl * 128 + ((chunk ^ (jl & 7)) << 4)) =
                  to_bf16_bits(p[jj] - __uint_as_float((uint32_t)hi << 16));
            }
          }
          // keys past the written cache: zero their V rows (0 * NaN would poison O)
          if (hh == 0 && t >= nk) {
            uint4* v0 = reinterpret_cast<uint4*>(smem + (int)(tc % kD4Stages) * kD4StageBytes + kD4OffV + t * 128);
            uint4* v1 = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(v0) + kD4Half);
#pragma unroll
            for (int c = 0; c < 8; ++c) { v0[c] = make_uint4(0, 0, 0, 0); v1[c] = make_uint4(0, 0, 0, 0); }
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&p_full[pbuf]);
        ++n_tiles;
        ++tc;
      }
      // end of the row's tiles in this CTA: O from tensor memory, the sums of the quarters
      uint32_t ov[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) ov[j] = 0u;
      if (n_tiles > 0) {
        ok = ok && !*s_abort && mbar_wait(&pv_done[(tc - 1) & 1], (uint32_t)(((tc - 1) >> 1) & 1), err);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          tmem_ld16(tl + 32, ov);
          tmem_wait_ld_regs16(ov);
        }
        {
          const float ws = warp_reduce_heads<GH, false>(l_part, lane);
          if ((lane & (32 / GH - 1)) == 0) red_sum[q * 16 + j0 + lane / (32 / GH)] = ws;
        }
        named_bar_softmax<SW>();
      }
      uint16_t* out_row = mo.out + (long long)b * mo.ldo + (long long)g * G * kHeadDim;
      if (jb == 0 && je == w.nt) {
        // the whole row is here: normalise and write the output
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          const int hd = j0 + jj;
          const float L = red_sum[hd] + red_sum[16 + hd] + red_sum[32 + hd] + red_sum[48 + hd];
          const float o = HILO ? __uint_as_float(pick_head<HW, GH>(ov, 0, hh, jj)) + __uint_as_float(pick_head<HW, GH>(ov, G, hh, jj)) : __uint_as_float(pick_head<HW, GH>(ov, 0, hh, jj));
          store_head_dim(o / L, t, out_row + hd * kHeadDim, mo);
        }
      } else {
        // a row shared by several CTAs: the row's first CTA merges, at the end of its range
        // (where it reaches the row); the others leave a partial in slot row + CTA (unique:
        // the rows and the CTA ranges are both in tile order) and publish it with one
        // release add, without waiting
        const int c_first = d4_cta_of(w.rs, T, n_cta), c_last = d4_cta_of(w.rs + w.nt - 1, T, n_cta);
        if ((int)blockIdx.x != c_first) {
          float* my_part = part + ((long long)bg + blockIdx.x) * G * kD4PartFloats;
#pragma unroll
          for (int jj = 0; jj < GH; ++jj) {
            const int hd = j0 + jj;
            my_part[hd * kD4PartFloats + t] =
                HILO ? __uint_as_float(pick_head<HW, GH>(ov, 0, hh, jj)) + __uint_as_float(pick_head<HW, GH>(ov, G, hh, jj)) : __uint_as_float(pick_head<HW, GH>(ov, 0, hh, jj));
            if (t == hd) {
              my_part[hd * kD4PartFloats + kHeadDim] = m_run[jj];
              my_part[hd * kD4PartFloats + kHeadDim + 1] =
                  red_sum[hd] + red_sum[16 + hd] + red_sum[32 + hd] + red_sum[48 + hd];
            }
          }
          named_bar_softmax<SW>();  // every thread's partial stores precede the release
          if (threadIdx.x == 0) red_release_gpu_add(&counters[bg], 1);
        } else {
          if (threadIdx.x == 0) {
            // the row's other CTAs (those of (c_first, c_last] whose range is not empty:
            // fewer tiles than CTAs leaves some empty) have all published (bounded wait)
            int n_other = 0;
            for (int c = c_first + 1; c <= c_last; ++c) n_other += d4_cta_empty(c, T, n_cta) ? 0 : 1;
            bool done = true;
            const unsigned long long t0 = global_ns();
            while (ld_acquire_gpu_s32(&counters[bg]) < n_other) {
              if (global_ns() - t0 > kWaitLimitNs) {
                record_error(err, kErrTimeout);
                done = false;
                break;
              }
            }
            counters[bg] = 0;  // ready for the next call
            *s_fix = done ? 1 : 0;
          }
          named_bar_softmax<SW>();  // the acquire above precedes every thread's reads
          if (*s_fix) {
#pragma unroll
            for (int jj = 0; jj < GH; ++jj) {
              const int hd = j0 + jj;
              const float o_own = HILO ? __uint_as_float(pick_head<HW, GH>(ov, 0, hh, jj)) + __uint_as_float(pick_head<HW, GH>(ov, G, hh, jj)) : __uint_as_float(pick_head<HW, GH>(ov, 0, hh, jj));
              merge_row_dim_own(part + ((long long)bg * G + hd) * kD4PartFloats, c_first, c_last, T, n_cta,
                                (long long)G * kD4PartFloats, t, m_run[jj],
                                red_sum[hd] + red_sum[16 + hd] + red_sum[32 + hd] + red_sum[48 + hd], o_own,
                                out_row + hd * kHeadDim, mo);
            }
          }
        }
      }
    }
    if (!ok) *s_abort = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == SW + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kD4TmemCols);
  }
}

// Tile prefix of the decode call: plan[b] = index of the first tile of sequence b's rows
// (Hkv rows of ceil((cache_len[b] + 1) / 128) tiles each; none for a sequence whose
// new position is past the cache, which is reported), plan[B] = all tiles. Clears the
// rows' merge counters. One block.
__global__ void __launch_bounds__(1024) attn_decode_plan_kernel(const int* __restrict__ cache_len, int B, int Hkv,
                                                                int s_max, int* __restrict__ plan,
                                                                int* __restrict__ counters, int* err) {
  __shared__ int wsum[32];
  __shared__ int carry;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < B; base += blockDim.x) {
    const int b = base + (int)threadIdx.x;
    int v = 0;
    if (b < B) {
      const int len = cache_len[b];
      if (len < 0) record_error(err, kErrInvalid);
      else if (len >= s_max) record_error(err, kErrCapacity);
      else v = Hkv * ((len + 1 + 127) / 128);
    }
    int x = v;  // inclusive scan within the warp, then over the warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int u = lane < nw ? wsum[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, u, o);
        if (lane >= o) u += y;
      }
      wsum[lane] = u;
    }
    __syncthreads();
    if (b < B) plan[b] = carry + (wid > 0 ? wsum[wid - 1] : 0) + x - v;
    __syncthreads();
    if (threadIdx.x == 0) carry += wsum[nw - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) plan[B] = carry;
  for (int i = threadIdx.x; i < B * Hkv; i += blockDim.x) counters[i] = 0;
}

// Scratch of one decode call: partial slots (rows + CTAs, G heads each), the tile plan,
// the rows' merge counters.
static size_t d4_part_floats(int B, int Hq) { return ((size_t)B * Hq + (size_t)kD4MaxCtas * 16) * kD4PartFloats; }
static size_t d4_plan_ints(int B) { return ((size_t)B + 1 + 3) & ~(size_t)3; }

size_t decode_partial_bytes(int B, int Hq, int Hkv) {
  return d4_part_floats(B, Hq) * sizeof(float) + (d4_plan_ints(B) + (size_t)B * Hkv) * sizeof(int) + 256;
}

// qkv: [B][ldqkv] with the Hq query heads at the start of each row; with q_hilo the row
// holds 2 * Hq heads instead, for group g the G rows q_hi then the G rows q_lo
// (G <= 8 only).
// scratch: decode_partial_bytes(B, Hq, Hkv) bytes, 16-byte aligned. plan_ready: the
// scratch already holds this call's tile plan (same cache_len, B, Hkv, s_max and scratch,
// written by an earlier launch on the stream), so the plan kernel is skipped.
int launch_attention_decode(const uint16_t* qkv, long long ldqkv, int B, int Hq, int Hkv, const int* cache_len,
                            const uint16_t* ck, const uint16_t* cv, int s_max, float* scratch, uint16_t* out,
                            long long ldo, int* err, cudaStream_t s, bool o_f16, bool q_hilo, long long o_lo,
                            bool plan_ready) {
  if (B <= 0) return 0;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) {
    set_last_error("attention decode: %d query heads per KV group is not supported (1, 2, 4, 8 or 16)", G);
    return -2;
  }
  if ((long long)B * Hkv * s_max + 128 >= (1ll << 31)) {
    set_last_error("attention decode: B * Hkv * s_max = %lld cache rows exceed the 2^31 tensor-map range",
                   (long long)B * Hkv * s_max);
    return -2;
  }
  if (q_hilo && G > 8) {
    set_last_error("attention decode: the hi/lo query layout needs at most 8 query heads per KV group");
    return -2;
  }
  CUtensorMap tmQ, tmK, tmV;
  // Q: (dim, head, token), box = the G heads of one group (2G rows: hi and lo)
  const int qr = q_hilo ? 2 * G : G;
  if (make_tmap_3d(&tmQ, qkv, kHeadDim, (long long)qr * Hkv, B, kHeadDim * 2, ldqkv * 2, 64, qr, 1) != 0) {
    set_last_error("attention decode: cannot encode the query tensor map");
    return -6;
  }
  const long long kv_rows = (long long)B * Hkv * s_max;
  CUtensorMap tmK16, tmV16;  // 16-row boxes for the last tile of a row
  if (make_tmap_2d(&tmK, ck, kv_rows, kHeadDim, kHeadDim, 128) != 0 ||
      make_tmap_2d(&tmV, cv, kv_rows, kHeadDim, kHeadDim, 128) != 0 ||
      make_tmap_2d(&tmK16, ck, kv_rows, kHeadDim, kHeadDim, 16) != 0 ||
      make_tmap_2d(&tmV16, cv, kv_rows, kHeadDim, kHeadDim, 16) != 0) {
    set_last_error("attention decode: cannot encode the KV-cache tensor maps");
    return -6;
  }
  const int grid = num_sms() < kD4MaxCtas ? num_sms() : kD4MaxCtas;
  float* part = scratch;
  int* plan = reinterpret_cast<int*>(scratch + d4_part_floats(B, Hq));
  int* counters = plan + d4_plan_ints(B);
  if (!plan_ready) q3_launch(attn_decode_plan_kernel, 1, 1024, 0, s, cache_len, B, Hkv, s_max, plan, counters, err);
  DecodeMergeOut mo;
  mo.out = out;
  mo.ldo = ldo;
  mo.o_f16 = o_f16 ? 1 : 0;
  mo.o_lo = o_lo;
  const int variant = G * 2 + (q_hilo ? 1 : 0);
  switch (variant) {
#define Q3_D4_CASE(GG, HL)                                                                                        \
  case GG * 2 + HL:                                                                                               \
    if (ensure_smem_attr(reinterpret_cast<const void*>(attn_decode_tc_kernel<GG, HL>), kD4Smem)) return -6;       \
    q3_launch(attn_decode_tc_kernel<GG, HL>, grid, d4_threads(GG), kD4Smem, s, tmQ, tmK, tmV, tmK16, tmV16, B, Hq, \
              Hkv, cache_len, s_max, plan, part, counters, mo, err);                                              \
    break;
    Q3_D4_CASE(1, false)
    Q3_D4_CASE(2, false)
    Q3_D4_CASE(4, false)
    Q3_D4_CASE(8, false)
    Q3_D4_CASE(16, false)
    Q3_D4_CASE(1, true)
    Q3_D4_CASE(2, true)
    Q3_D4_CASE(4, true)
    Q3_D4_CASE(8, true)
#undef Q3_D4_CASE
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("attention decode launch failed: %s", cudaGetErrorString(e));
    return -6;
  }
  return 0;
}

// ----------------------------------------------------------------------------
// Decode attention without caller scratch. The partials, the tile plan and the merge
// counters live in a fixed device array of this library instead of a caller workspace,
// for callers that cannot allocate device memory. Its capacity is kStaticDecodeFloats
// floats (12 MiB): decode_partial_bytes(B, Hq, Hkv) must fit (B * Hq up to about 20000).
// The array's device address is looked up on the host once per device (with that device
// current); every call shares the array, so calls that overlap on the GPU race. Each
// call writes its plan and clears its merge counters before use, and every partial it reads is
// written by that same call, so nothing has to be cleared between calls.
// ----------------------------------------------------------------------------
constexpr size_t kStaticDecodeFloats = (size_t)3 << 20;
static __device__ __align__(256) float g_decode_scratch[kStaticDecodeFloats];

static std::mutex g_static_mu;
static float* g_static_ptr[64];

size_t static_decode_scratch_bytes() { return kStaticDecodeFloats * sizeof(float); }

int launch_attention_decode_static(const uint16_t* qkv, long long ldqkv, int B, int Hq, int Hkv,
                                   const int* cache_len, const uint16_t* ck, const uint16_t* cv, int s_max,
                                   uint16_t* out, long long ldo, int* err, cudaStream_t s, bool o_f16) {
  const size_t need = decode_partial_bytes(B, Hq, Hkv);
  if (need > kStaticDecodeFloats * sizeof(float)) {
    set_last_error("attention_decode_noalloc: B=%d, Hq=%d, Hkv=%d need %zu bytes of scratch; the static scratch "
                   "holds %zu bytes", B, Hq, Hkv, need, kStaticDecodeFloats * sizeof(float));
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
  return launch_attention_decode(qkv, ldqkv, B, Hq, Hkv, cache_len, ck, cv, s_max, ptr, out, ldo, err, s, o_f16,
                                 false, 0, false);
}

}  // namespace q3
