// Decode-sized projections (at most 64 tokens): a tcgen05 GEMM whose K dimension is
// split over the CTAs of one thread-block cluster and summed through distributed
// shared memory, so that the split-K reduction and the step that follows the
// projection run in the same kernel.
//
// Shapes and formulas are the block's linear layers ("从零实现 Qwen3：拆解 mini-qwen3
// 的 0.6B Dense 架构", sections GQA, SwiGLU FFN and TransformerBlock): out = x W^T with
// W stored [out_features, in_features]. With few tokens the weights are the operand
// on the MMA's 128-row side (swap form): tile = 128 output features x BN tokens.
//
// Design (sm_100a):
//   * grid = feature tiles x S; the S CTAs of one feature tile form a cluster (up to 16)
//     and each takes a contiguous range of the K blocks (64 wide); one CTA per SM;
//   * warp 0: TMA producer (weights 128 x 64 and tokens BN x 64 per K block, 128-byte
//     swizzle; the weight loads of the first stages precede the grid-dependency
//     wait, since no kernel of the call writes weights); warp 1: one thread issues
//     tcgen05.mma (M = 128, N = BN, K = 16) into one fp32 accumulator in tensor memory;
//     warps 2-5 read the accumulator; all 8 warps then share the tokens' epilogues;
//   * after the last MMA each CTA copies its accumulator to shared memory as
//     [token][feature]; after a cluster barrier, token t is finished by one warp of the
//     cluster, which adds the S partials in split order (deterministic) with
//     ld.shared::cluster and applies the epilogue: plain store, residual add, SwiGLU, or
//     per-head QK RMSNorm + rotate-half RoPE + KV-cache write;
//   * residual projections can also produce the RMSNorm of their whole output (the
//     norm that follows them in the block): every warp writes the sum of squares of
//     its token's 128 features, all CTAs (co-resident: one wave) meet at a grid-wide
//     barrier, and each warp then adds the tiles' sums of its token in tile order and
//     normalises the features it still holds in registers ("grid" mode); or, when the
//     next projection is one of these kernels too, the norm is deferred: this kernel
//     writes y = x * w * s_t (s_t = 1/rms of the residual stream before this projection,
//     which keeps y at the normalised magnitude) and the sums of squares, and the next
//     projection, which is linear in its input row, multiplies its accumulators of
//     token t by r_t / s_t (r_t = 1/rms of x_t from the sums, in tile order) -- the same
//     result as normalising first, without the barrier;
//   * every mbarrier wait is bounded; cluster barriers are executed by every thread on
//     every path, so an expired wait cannot leave a peer CTA waiting.
#include <cstdio>
#include <mutex>
#include <vector>
#include "common.cuh"
#include "internal.h"

namespace q3 {

int make_tmap_2d(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld, int box_rows);

namespace {

constexpr int kSkThreads = 512;  // TMA warp, MMA warp, 4 accumulator warps, 10 more epilogue warps
constexpr int kSkMaxSplits = 16;  // cluster size: 16 is the non-portable maximum on sm_100
constexpr int kSkPre = 2;        // tokens per epilogue warp whose side operands are prefetched
constexpr uint32_t kSkPBytes = 128 * 64 * 2;  // weight tile: 128 features x 64 of K, bf16

// HILO: the activation operand holds 2M rows, row t = hi(a_t) and row M + t = lo(a_t)
// (a = hi + lo to about twice the type's precision). Two TMA boxes of BN rows put the hi
// rows at tile rows [0, BN) and the lo rows at [BN, 2 BN), so the MMA's N = 2 BN covers
// both and accumulator columns t and BN + t (32-aligned chunks) are added in registers.
// A kernel that allocates tensor memory runs one CTA per SM, so the ring takes up to
// 200 KB: deep enough that a split's weight blocks (at most 8) are all requested before
// the grid-dependency wait.
template <int BN, bool HILO>
struct SkCfg {
  static constexpr int NQ = HILO ? 2 * BN : BN;  // activation rows per tile = MMA N
  static constexpr uint32_t Q_BYTES = NQ * 64 * 2;
  static constexpr uint32_t STAGE = kSkPBytes + Q_BYTES;
  static constexpr int STAGES = (int)(((200u << 10) - 1280u) / STAGE) > 8 ? 8 : (int)(((200u << 10) - 1280u) / STAGE);
  static constexpr uint32_t TMEM_COLS = NQ < 32 ? 32 : NQ;
  // + barriers, flags and the TMA and MMA warps' row scales
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 256;
  static_assert((2 * STAGES + 1) * 8 + 16 + 2 * kSkPre * 3 * 4 <= 256, "barrier area too small");
  static_assert(STAGES >= 3, "ring too shallow");
  static_assert((size_t)BN * 128 * 4 <= (size_t)STAGES * STAGE, "the split partial must fit over the ring");
};

struct SkParams {
  int M;         // tokens (<= BN)
  int k_blocks;  // K / 64
  int kpb;       // K blocks per split
  int S;         // splits = cluster size
  int epi;
  int out_f32, resid_f32;
  int p_early;
  void* out;
  long long ldo;
  const void* resid;
  long long ldr;
  // residual epilogue: RMSNorm of the whole output (N features) by the last cluster
  const uint16_t* norm_w;
  uint16_t* norm_out;
  long long ld_norm;
  long long norm_lo;  // > 0: also write lo(norm_out) this many elements after each hi value
  long long out_lo;   // SwiGLU: > 0: also write lo(out) this many elements after each hi value
  int N;
  float norm_eps;
  int* ticket;  // grid barrier of the fused norm: [0] arrivals (0 between launches), [1] generation
  float* ssq;   // fused norm: per-tile sums of squares [N / 128][64]
  int norm_deferred;       // fused norm deferred to the next projection (no barrier)
  const float* pre_scale;  // deferred norm: s_t, written as y = x * w * s_t ([64]; null: 1)
  // this projection's input is a deferred norm's output: scale token t's accumulators by
  // r_t / s_in[t], r_t = rsqrt(sum_q row_ssq[q * 64 + t] / ssq_n + eps) (q < ssq_tiles)
  const float* row_ssq;
  int ssq_tiles, ssq_n;
  float ssq_eps;
  const float* row_s_in;  // [64] (null: 1)
  float* row_r_out;       // [64] r_t of the input rows (feature tile 0 writes it), or null
  QKRopeArgs qk;
  int f16;  // operands fp16 (else bf16); the SwiGLU and fused-norm outputs are fp16 too
  int* err;
};

}  // namespace

// Barrier of all n CTAs of the grid, called by one thread per CTA after a CTA-level
// barrier (every CTA of the grid is resident: the launch is one wave). The arrival is a
// release at GPU scope (cumulative over the writes the CTA barrier ordered before it),
// the wait an acquire. bar[0] counts arrivals and is back at 0 after each use; bar[1] is
// a generation that the last arrival advances. Bounded wait: false (and kErrTimeout).
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ bool grid_barrier(int* bar, int n, int* err) {
  const int g0 = ld_acquire_gpu(bar + 1);  // cannot advance before this CTA arrives
  if (atom_add_acq_rel_gpu(bar, 1) == n - 1) {
    bar[0] = 0;
    atom_add_acq_rel_gpu(bar + 1, 1);  // releases the reset and everything before it
    return true;
  }
  const unsigned long long t0 = global_ns();
  while (ld_acquire_gpu(bar + 1) == g0) {
    if (global_ns() - t0 > kWaitLimitNs) {
      record_error(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

// All warps of the CTA, on the epilogue path.
__device__ __forceinline__ void epi_bar_sync() { asm volatile("bar.sync 2, %0;" ::"n"(kSkThreads) : "memory"); }

template <int BN, bool HILO>
__global__ void __launch_bounds__(kSkThreads, 1)
    gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                       const SkParams g) {
  using C = SkCfg<BN, HILO>;
  constexpr int kSkStages = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSkStages * C::STAGE);
  uint64_t* empty = full + kSkStages;
  uint64_t* done = empty + kSkStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = s_abort + 1;  // the fused norm's grid barrier completed
  float* s_scale = reinterpret_cast<float*>(tmem_slot + 4);  // [2 warps][kSkPre tokens][k, r, s]
  float* red = reinterpret_cast<float*>(smem);  // [BN][128] partial sums, over the stages once the MMAs are done

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int tile = (int)(blockIdx.x / (unsigned)g.S);
  const int kb0 = (int)rank * g.kpb;
  const int nkb = min(g.k_blocks, kb0 + g.kpb) - kb0;  // >= 1 by the host's choice of S

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSkStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(done, 1);
    *s_abort = 0;
    *s_last = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == 32) { tma_prefetch_desc(&tmP); tma_prefetch_desc(&tmQ); }
  if (warp == 1) { tmem_alloc(tmem_slot, C::TMEM_COLS); tmem_relinquish(); }
  // weight loads of the first stages before the wait (weights are final before the call)
  int p_pre = 0;
  if (g.p_early && threadIdx.x == 0) {
    p_pre = min(kSkStages, nkb);
    for (int i = 0; i < p_pre; ++i) {
      mbar_arrive_expect_tx(&full[i], C::STAGE);
      tma_load_2d(smem + i * C::STAGE, &tmP, &full[i], (kb0 + i) * 64, tile * 128);
    }
    // the split's remaining weight blocks into L2, so that their ring loads hit L2
    for (int i = p_pre; i < nkb; ++i) tma_prefetch_l2_2d(&tmP, (kb0 + i) * 64, tile * 128);
  }
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // warp ew = 8 rank + warp of the cluster finishes tokens ew + i enw; the side operands
  // of its first kSkPre tokens are loaded ahead (npre)
  const int ew = (int)rank * (kSkThreads / 32) + warp;
  const int enw = (kSkThreads / 32) * g.S;
  constexpr int npre = kSkPre;
  float pre_a[kSkPre][4] = {};
  float2 pre_c0[kSkPre] = {}, pre_c1[kSkPre] = {};
  int pre_pos[kSkPre] = {};
  float pre_k[kSkPre], pre_r[kSkPre], pre_s[kSkPre];  // input-row scale, its r_t; deferred norm's s_t
  float wn[4] = {0.f, 0.f, 0.f, 0.f};  // QK-norm weights (kEpiQKRope), fused-norm weights (norm_out)
  float keep[kSkPre][4] = {};          // fused norm: the output values of the prefetched tokens
  // residual values (kEpiResid), or position and rotary factors (kEpiQKRope) of token t
  auto load_side = [&](int t, float(&a)[4], float2& c0, float2& c1, int& pos) {
    if (g.epi == kEpiResid) {
      const long long base = (long long)t * g.ldr + (long long)tile * 128 + lane;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        a[j] = g.resid_f32 ? static_cast<const float*>(g.resid)[base + 32 * j]
                           : __uint_as_float((uint32_t)static_cast<const uint16_t*>(g.resid)[base + 32 * j] << 16);
    } else if (g.epi == kEpiQKRope) {
      const QKRopeArgs& q = g.qk;
      const int b = t / q.T;
      pos = q.pos_base[b] + (t - b * q.T);
      c0 = c1 = make_float2(0.f, 0.f);
      if (tile < q.Hq + q.Hkv && pos >= 0 && pos < q.s_max && pos < q.max_pos) {
        c0 = *reinterpret_cast<const float2*>(q.rope + ((long long)pos * 64 + lane) * 2);
        c1 = *reinterpret_cast<const float2*>(q.rope + ((long long)pos * 64 + 32 + lane) * 2);
      }
    }
  };

  // the deferred-norm factors of token t: input-row scale k = r / s_in (and r), and the
  // s_t this kernel's own deferred norm writes with
  auto load_scales = [&](int t, float& k, float& r, float& sp) {
    k = 1.f;
    r = 1.f;
    if (g.row_ssq) {
      float ss = 0.f;
#pragma unroll 8
      for (int q = 0; q < g.ssq_tiles; ++q) ss += __ldcg(g.row_ssq + q * 64 + t);  // tile order
      r = rsqrtf(ss / (float)g.ssq_n + g.ssq_eps);
      k = r / (g.row_s_in ? g.row_s_in[t] : 1.f);
    }
    sp = g.pre_scale ? g.pre_scale[t] : 1.f;
  };
  // epilogue operands that do not depend on the product (residual rows, positions,
  // rotary factors), requested by every warp before its role: the loads complete while
  // the weights stream and the MMAs run
#pragma unroll
  for (int i = 0; i < kSkPre; ++i) {
    const int t = ew + i * enw;
    if (t < g.M) load_side(t, pre_a[i], pre_c0[i], pre_c1[i], pre_pos[i]);
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nkb && ok; ++i) {
        const int st = i % kSkStages;
        const uint32_t ph = (uint32_t)(i / kSkStages) & 1u;
        uint8_t* sp = smem + st * C::STAGE;
        if (i >= p_pre) {  // else the weights are on their way; the stage expects all boxes
          if (*s_abort || !mbar_wait(&empty[st], ph ^ 1u, g.err)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], C::STAGE);
          tma_load_2d(sp, &tmP, &full[st], (kb0 + i) * 64, tile * 128);
        }
        tma_load_2d(sp + kSkPBytes, &tmQ, &full[st], (kb0 + i) * 64, 0);
        if (HILO) tma_load_2d(sp + kSkPBytes + BN * 128, &tmQ, &full[st], (kb0 + i) * 64, g.M);
        ++issued;
      }
      if (!ok) {
        *s_abort = 1;
        for (int i = issued > kSkStages ? issued - kSkStages : 0; i < issued; ++i)
          mbar_wait(&full[i % kSkStages], (uint32_t)(i / kSkStages) & 1u, g.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t idesc = g.f16 ? idesc_f16_f32(128, C::NQ) : idesc_bf16_f32(128, C::NQ);
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int st = i % kSkStages;
        const uint32_t ph = (uint32_t)(i / kSkStages) & 1u;
        if (*s_abort || !mbar_wait(&full[st], ph, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + st * C::STAGE);
        const uint64_t adesc = sdesc_kmajor_sw128(sa);
        const uint64_t bdesc = sdesc_kmajor_sw128(sa + kSkPBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (i | kk) ? 1u : 0u);
        mma_commit(&empty[st]);
      }
      if (!ok) *s_abort = 1;
      // arrives once every MMA issued above has completed (at once if none was issued)
      mma_commit(done);
    }
  }
  // per-feature weights of the epilogue (QK-norm, or the fused RMSNorm), every warp
  if (g.epi == kEpiQKRope && tile < g.qk.Hq + g.qk.Hkv) {
    const uint16_t* wsrc = tile < g.qk.Hq ? g.qk.q_norm : g.qk.k_norm;
#pragma unroll
    for (int j = 0; j < 4; ++j) wn[j] = __uint_as_float((uint32_t)wsrc[32 * j + lane] << 16);
  }
  if (g.norm_out) {
#pragma unroll
    for (int j = 0; j < 4; ++j) wn[j] = __uint_as_float((uint32_t)g.norm_w[tile * 128 + 32 * j + lane] << 16);
  }
  // the scales use their loads at once, so the warps that wait for the MMAs compute
  // them: their own, and (warps 2 and 3) those of warps 0 and 1 into shared memory, read
  // after the cluster barrier
  if (warp >= 2) {
#pragma unroll
    for (int i = 0; i < kSkPre; ++i) {
      const int t = ew + i * enw;
      if (t < g.M) load_scales(t, pre_k[i], pre_r[i], pre_s[i]);
    }
    if (warp < 4) {
#pragma unroll
      for (int i = 0; i < kSkPre; ++i) {
        const int t = ew - 2 + i * enw;  // token i of warp (warp - 2)
        float k = 1.f, r = 1.f, sp = 1.f;
        if (t < g.M) load_scales(t, k, r, sp);
        if (lane == 0) {
          s_scale[((warp - 2) * kSkPre + i) * 3] = k;
          s_scale[((warp - 2) * kSkPre + i) * 3 + 1] = r;
          s_scale[((warp - 2) * kSkPre + i) * 3 + 2] = sp;
        }
      }
    }
  }
  if (warp >= 2 && warp < 6) {
    // ---------------------------------------------------------- accumulator -> smem
    const int quad = warp & 3;  // tensor-memory lanes [32 quad, 32 quad + 32)
    bool ok = mbar_wait(done, 0, g.err);
    ok = __all_sync(0xffffffffu, ok) && !*s_abort;
    tc_fence_after();
    const int f = quad * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
    // column j < M: token j (its hi half with HILO); with HILO, column BN + j: its lo half
    const int M = g.M;
    if constexpr (BN == 16) {
      uint32_t r[16], rl[16];
      tmem_ld16(taddr, r);
      if constexpr (HILO) tmem_ld16(taddr + 16, rl);
      tmem_wait_ld_regs16(r);
      if constexpr (HILO) tmem_wait_ld_regs16(rl);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float v = HILO ? __uint_as_float(r[j]) + __uint_as_float(rl[j]) : __uint_as_float(r[j]);
        if (j < M) red[j * 128 + f] = ok ? v : 0.f;
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        if (c * 32 >= M) break;  // warp-uniform
        uint32_t r[32], rl[32];
        tmem_ld32(taddr + c * 32, r);
        if constexpr (HILO) tmem_ld32(taddr + BN + c * 32, rl);
        tmem_wait_ld_regs(r);
        if constexpr (HILO) tmem_wait_ld_regs(rl);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float v = HILO ? __uint_as_float(r[j]) + __uint_as_float(rl[j]) : __uint_as_float(r[j]);
          if (c * 32 + j < M) red[(c * 32 + j) * 128 + f] = ok ? v : 0.f;
        }
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // every split's partial is in its CTA's shared memory

  if (!*s_abort) {
    // -------------------------------------------------- split sum + epilogue, one warp per token
    // split s's partial of (token t, feature f) in CTA s: the mapa (a volatile asm after
    // the barrier) keeps the loads, which no longer change, below the barrier
    const uint32_t red0 = smem_u32(red);
    auto sum_token = [&](int t, float(&v)[4]) {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = 0.f;
#pragma unroll 4
      for (int s = 0; s < g.S; ++s) {
        const uint32_t base = mapa_shared_addr(red0 + (uint32_t)((t * 128 + lane) * 4), (uint32_t)s);
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] += ld_cluster_f32_ro(base + 128u * j);  // split order: deterministic
      }
    };
    // v: the token's sums in, and (residual epilogue) the values the fused norm sees out
    auto finish = [&](int t, float(&v)[4], const float(&a)[4], float2 c0, float2 c1, int pos, float kin, float rin,
                      float sp) {
      if (g.row_ssq) {  // the input rows were a deferred norm's output
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] *= kin;
        if (g.row_r_out && tile == 0 && lane == 0) g.row_r_out[t] = rin;
      }
      if (g.epi == kEpiQKRope) {
        // slot = head of the fused QKV row: q heads, then k heads, then v heads
        const QKRopeArgs& q = g.qk;
        const int slot = tile;
        const int b = t / q.T;
        if (pos < 0 || pos >= q.s_max || pos >= q.max_pos) {
          if (lane == 0) record_error(g.err, kErrCapacity);
          return;
        }
        if (slot >= q.Hq + q.Hkv) {  // value head: straight to the cache
          uint16_t* dst = q.cv + (((long long)b * q.Hkv + (slot - q.Hq - q.Hkv)) * q.s_max + pos) * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[32 * j + lane] = to_bf16_bits(v[j]);
          return;
        }
        const bool is_q = slot < q.Hq;
        const float ss = warp_sum(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
        const float r = rsqrtf(ss * (1.0f / 128.0f) + q.eps);
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] *= r * wn[j];
        // rotation pairs (d, d + 64): d = lane (v[0], v[2]) and d = 32 + lane (v[1], v[3])
        const float o[4] = {v[0] * c0.x - v[2] * c0.y, v[1] * c1.x - v[3] * c1.y, v[0] * c0.y + v[2] * c0.x,
                            v[1] * c1.y + v[3] * c1.x};  // dims lane, 32 + lane, 64 + lane, 96 + lane
        if (is_q && q.q2) {
          // hi/lo rows of the decode attention: group grp, head j of the group
          const int G = q.Hq / q.Hkv, grp = slot / G, jh = slot - grp * G;
          uint16_t* hi = q.q2 + (long long)t * q.ldq2 + ((long long)grp * 2 * G + jh) * 128;
          uint16_t* lo = hi + (long long)G * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint16_t h = to_bf16_bits(o[i]);
            hi[32 * i + lane] = h;
            lo[32 * i + lane] = to_bf16_bits(o[i] - __uint_as_float((uint32_t)h << 16));
          }
          return;
        }
        uint16_t* dst = is_q ? static_cast<uint16_t*>(g.out) + (long long)t * g.ldo + (long long)slot * 128
                             : q.ck + (((long long)b * q.Hkv + (slot - q.Hq)) * q.s_max + pos) * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[32 * i + lane] = to_bf16_bits(o[i]);
      } else if (g.epi == kEpiSwiglu) {
        // 32-feature block j: lanes 0-15 hold gate features, lanes 16-31 the matching up
        uint16_t* dst = static_cast<uint16_t*>(g.out) + (long long)t * g.ldo + tile * 64;
        const bool f16 = g.f16 != 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float u = __shfl_down_sync(0xffffffffu, v[j], 16);
          if (lane < 16) {
            const float h = silu_f(v[j]) * u;
            const uint16_t hi = to_op_bits(f16, h);
            dst[16 * j + lane] = hi;
            if (g.out_lo) dst[g.out_lo + 16 * j + lane] = to_op_bits(f16, h - op_bits_to_f32(f16, hi));
          }
        }
      } else {
        const long long col = (long long)tile * 128 + lane;
        if (g.epi == kEpiResid) {
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] += a[j];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (g.out_f32) {
            static_cast<float*>(g.out)[(long long)t * g.ldo + col + 32 * j] = v[j];
          } else {
            const uint16_t h = to_bf16_bits(v[j]);
            static_cast<uint16_t*>(g.out)[(long long)t * g.ldo + col + 32 * j] = h;
            v[j] = __uint_as_float((uint32_t)h << 16);  // the norm sees the stored value
          }
        }
        if (g.norm_out) {
          const float ss = warp_sum(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
          if (lane == 0) g.ssq[tile * 64 + t] = ss;
          if (g.norm_deferred) {
            // y = x * w * s_t as hi/lo operand rows; the next projection applies r_t / s_t
            uint16_t* dst = g.norm_out + (long long)t * g.ld_norm + col;
            const bool f16 = g.f16 != 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float y = v[j] * wn[j] * sp;
              const uint16_t hi = to_op_bits(f16, y);
              dst[32 * j] = hi;
              if (g.norm_lo) dst[g.norm_lo + 32 * j] = to_op_bits(f16, y - op_bits_to_f32(f16, hi));
            }
          }
        }
      }
    };
    // the TMA and MMA warps' scales, computed by warps 2 and 3 while the MMAs ran
    if (warp < 2) {
#pragma unroll
      for (int i = 0; i < kSkPre; ++i) {
        pre_k[i] = s_scale[(warp * kSkPre + i) * 3];
        pre_r[i] = s_scale[(warp * kSkPre + i) * 3 + 1];
        pre_s[i] = s_scale[(warp * kSkPre + i) * 3 + 2];
      }
    }
    // one copy of the token code, run as a loop: a launch executes it from a cold
    // instruction cache, so an unrolled copy per token would pay the fetches once per
    // token. The prefetched operands rotate down to slot 0 (registers, fixed indices);
    // the fused norm's values rotate in at the end of keep.
#pragma unroll 1
    for (int i = 0; i < kSkPre; ++i) {
      const int t = ew + i * enw;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (t < g.M) {
        sum_token(t, v);
        finish(t, v, pre_a[0], pre_c0[0], pre_c1[0], pre_pos[0], pre_k[0], pre_r[0], pre_s[0]);
      }
#pragma unroll
      for (int k = 0; k + 1 < kSkPre; ++k) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          pre_a[k][j] = pre_a[k + 1][j];
          keep[k][j] = keep[k + 1][j];
        }
        pre_c0[k] = pre_c0[k + 1];
        pre_c1[k] = pre_c1[k + 1];
        pre_pos[k] = pre_pos[k + 1];
        pre_k[k] = pre_k[k + 1];
        pre_r[k] = pre_r[k + 1];
        pre_s[k] = pre_s[k + 1];
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) keep[kSkPre - 1][j] = v[j];
    }
    for (int t = ew + npre * enw; t < g.M; t += enw) {  // tokens beyond the prefetched ones
      float a[4], v[4];
      float2 c0, c1;
      int pos = 0;
      float kin, rin, sp;
      load_side(t, a, c0, c1, pos);
      load_scales(t, kin, rin, sp);
      sum_token(t, v);
      finish(t, v, a, c0, c1, pos, kin, rin, sp);
    }
  }

  if (g.norm_out && !g.norm_deferred) {
    // ------------------------------------------------ RMSNorm of the whole output rows
    epi_bar_sync();  // the epilogue warps' output and sum-of-squares stores precede the arrival
    if (threadIdx.x == 64) *s_last = grid_barrier(g.ticket, (int)gridDim.x, g.err) ? 1 : 0;
    epi_bar_sync();
    if (*s_last && !*s_abort) {
      const int n_tiles = (int)(gridDim.x / (unsigned)g.S);
      const bool f16 = g.f16 != 0;
      const long long col = (long long)tile * 128 + lane;
      // sum over the tiles in tile order (L2 reads: other SMs wrote them)
      auto tiles_ss = [&](int t) {
        float ss = 0.f;
#pragma unroll 8
        for (int q = 0; q < n_tiles; ++q) ss += __ldcg(g.ssq + q * 64 + t);
        return ss;
      };
      auto normalise = [&](int t, float ss, const float(&x)[4]) {
        const float r = rsqrtf(ss / (float)g.N + g.norm_eps);
        if (g.row_r_out && tile == 0 && lane == 0) g.row_r_out[t] = r;  // the next stage's s_t
        uint16_t* dst = g.norm_out + (long long)t * g.ld_norm + col;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a = x[j] * r * wn[j];
          const uint16_t hi = to_op_bits(f16, a);
          dst[32 * j] = hi;
          if (g.norm_lo) dst[g.norm_lo + 32 * j] = to_op_bits(f16, a - op_bits_to_f32(f16, hi));
        }
      };
      float ssk[kSkPre];
#pragma unroll
      for (int i = 0; i < kSkPre; ++i) ssk[i] = i < npre && ew + i * enw < g.M ? tiles_ss(ew + i * enw) : 0.f;
#pragma unroll
      for (int i = 0; i < kSkPre; ++i) {
        const int t = ew + i * enw;
        if (i < npre && t < g.M) normalise(t, ssk[i], keep[i]);
      }
      for (int t = ew + npre * enw; t < g.M; t += enw) {  // tokens past the kept ones: re-read
        float x[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          x[j] = g.out_f32 ? static_cast<const float*>(g.out)[(long long)t * g.ldo + col + 32 * j]
                           : __uint_as_float((uint32_t)static_cast<const uint16_t*>(g.out)[(long long)t * g.ldo + col + 32 * j] << 16);
        normalise(t, tiles_ss(t), x);
      }
    }
  }
  __syncwarp();
  cluster_sync();  // no CTA leaves while a peer may still read its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------- host
namespace {

struct SkChoice {
  const void* func;
  int dev, S, smem, ok;
};
std::mutex g_sk_mu;
std::vector<SkChoice> g_sk_fit;

// Can n_clusters clusters of S CTAs all be resident at once (one wave)?
template <int BN, bool HILO>
bool clusters_fit(int S, int n_clusters) {
  int dev = 0;
  cudaGetDevice(&dev);
  const void* func = reinterpret_cast<const void*>(gemm_skinny_kernel<BN, HILO>);
  {
    std::lock_guard<std::mutex> lk(g_sk_mu);
    for (const auto& c : g_sk_fit)
      if (c.func == func && c.dev == dev && c.S == S) return c.ok >= n_clusters;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S * n_clusters);
  cfg.blockDim = dim3(kSkThreads);
  cfg.dynamicSmemBytes = SkCfg<BN, HILO>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_skinny_kernel<BN, HILO>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(g_sk_mu);
  g_sk_fit.push_back({func, dev, S, (int)SkCfg<BN, HILO>::SMEM, n});
  return n >= n_clusters;
}

// K splits of d: as many as fit one wave of co-resident clusters (one CTA per SM;
// clusters above 8 CTAs need the non-portable size, allowed once per kernel and device),
// within d.max_ctas; every split gets at least one K block.
template <int BN, bool HILO>
int choose_splits(const SkinnyDesc& d) {
  const int n_tiles = d.N / 128, k_blocks = d.K / 64;
  // the occupancy answers below assume the kernel's shared-memory limit is raised (a
  // grid computed before the first launch of this instantiation included)
  if (ensure_smem_attr(reinterpret_cast<const void*>(gemm_skinny_kernel<BN, HILO>), (int)SkCfg<BN, HILO>::SMEM))
    return 1;
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> wide;  // (kernel, device) allowed 16-CTA clusters
  int max_c = 8;
  {
    const void* func = reinterpret_cast<const void*>(gemm_skinny_kernel<BN, HILO>);
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    bool ok = false;
    for (const auto& e : wide) ok = ok || (e.first == func && e.second == dev);
    if (!ok && cudaFuncSetAttribute(gemm_skinny_kernel<BN, HILO>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                   cudaSuccess) {
      wide.emplace_back(func, dev);
      ok = true;
    }
    cudaGetLastError();
    if (ok) max_c = kSkMaxSplits;
  }
  int S = 1;
  if (d.max_ctas > 0 && d.max_ctas / n_tiles < max_c) max_c = d.max_ctas / n_tiles > 1 ? d.max_ctas / n_tiles : 1;
  for (int c = max_c; c >= 1; --c) {
    if ((long long)n_tiles * c > num_sms() || c > k_blocks) continue;
    if (c > 1 && !clusters_fit<BN, HILO>(c, n_tiles)) continue;
    S = c;
    break;
  }
  const int kpb = (k_blocks + S - 1) / S;
  return (k_blocks + kpb - 1) / kpb;
}

template <int BN, bool HILO>
int launch_bn(const SkinnyDesc& d, cudaStream_t s, int* err) {
  using C = SkCfg<BN, HILO>;
  if (ensure_smem_attr(reinterpret_cast<const void*>(gemm_skinny_kernel<BN, HILO>), (int)C::SMEM)) return -6;
  const int n_tiles = d.N / 128, k_blocks = d.K / 64;
  const int S = choose_splits<BN, HILO>(d);
  const int kpb = (k_blocks + S - 1) / S;
  CUtensorMap tmP, tmQ;
  if (make_tmap_2d(&tmP, d.W, d.N, d.K, d.ldw, 128) != 0 ||
      make_tmap_2d(&tmQ, d.A, HILO ? 2LL * d.M : d.M, d.K, d.lda, BN) != 0) {
    set_last_error("skinny gemm: cannot encode the operand tensor maps");
    return -6;
  }
  SkParams g;
  g.M = d.M;
  g.k_blocks = k_blocks;
  g.kpb = kpb;
  g.S = S;
  g.epi = d.epi;
  g.out_f32 = d.out_f32 ? 1 : 0;
  g.resid_f32 = d.resid_f32 ? 1 : 0;
  g.p_early = d.w_early ? 1 : 0;
  g.out = d.out;
  g.ldo = d.ldo;
  g.resid = d.resid;
  g.ldr = d.ldr;
  g.norm_w = d.norm_w;
  g.norm_out = d.norm_out;
  g.ld_norm = d.ld_norm;
  g.norm_lo = d.norm_lo;
  g.out_lo = d.out_lo;
  g.N = d.N;
  g.norm_eps = d.norm_eps;
  g.ticket = d.ticket;
  g.ssq = d.ssq;
  g.norm_deferred = d.norm_deferred ? 1 : 0;
  g.pre_scale = d.pre_scale;
  g.row_ssq = d.row_ssq;
  g.ssq_tiles = d.ssq_tiles;
  g.ssq_n = d.ssq_n;
  g.ssq_eps = d.ssq_eps;
  g.row_s_in = d.row_s_in;
  g.row_r_out = d.row_r_out;
  g.qk = d.qk;
  g.f16 = d.f16 ? 1 : 0;
  g.err = err;
  q3_launch_cluster(gemm_skinny_kernel<BN, HILO>, dim3(n_tiles * S), dim3(kSkThreads), C::SMEM, s, (unsigned)S,
                    tmP, tmQ, g);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("skinny gemm launch failed: %s", cudaGetErrorString(e));
    return -6;
  }
  return 0;
}

}  // namespace

bool skinny_supported(int M, int N, int K, int epi) {
  if (M < 1 || M > 64 || N % 128 != 0 || K % 64 != 0 || K < 64) return false;
  return epi == kEpiStore || epi == kEpiResid || epi == kEpiSwiglu || epi == kEpiQKRope;
}

int skinny_ctas(const SkinnyDesc& d) {
  if (!skinny_supported(d.M, d.N, d.K, d.epi)) return 0;
  const int n_tiles = d.N / 128;
  if (d.a_hilo) {
    if (d.M <= 16) return n_tiles * choose_splits<16, true>(d);
    if (d.M <= 32) return n_tiles * choose_splits<32, true>(d);
    return n_tiles * choose_splits<64, true>(d);
  }
  if (d.M <= 16) return n_tiles * choose_splits<16, false>(d);
  if (d.M <= 32) return n_tiles * choose_splits<32, false>(d);
  return n_tiles * choose_splits<64, false>(d);
}

int launch_gemm_skinny(const SkinnyDesc& d, cudaStream_t s, int* err) {
  if (!skinny_supported(d.M, d.N, d.K, d.epi)) {
    set_last_error("skinny gemm: unsupported shape M %d N %d K %d", d.M, d.N, d.K);
    return -2;
  }
  if (d.row_ssq && (d.ssq_tiles < 1 || d.ssq_tiles > 64 || d.ssq_n < 1)) {
    set_last_error("skinny gemm: bad deferred-norm input (%d sum-of-squares tiles, row length %d)", d.ssq_tiles,
                   d.ssq_n);
    return -1;
  }
  if (d.norm_out && (d.epi != kEpiResid || !d.norm_w || !d.ssq || (!d.norm_deferred && !d.ticket) ||
                     d.N / 128 > num_sms())) {
    set_last_error("skinny gemm: the fused RMSNorm needs the residual epilogue, weights, a barrier word pair, the "
                   "sum-of-squares scratch and at most one feature tile per SM");
    return -1;
  }
  if (d.epi == kEpiSwiglu ? false : d.out_lo != 0) {
    set_last_error("skinny gemm: a lo copy of the output is only written by the SwiGLU epilogue");
    return -1;
  }
  if (d.a_hilo) {
    if (d.M <= 16) return launch_bn<16, true>(d, s, err);
    if (d.M <= 32) return launch_bn<32, true>(d, s, err);
    return launch_bn<64, true>(d, s, err);
  }
  if (d.M <= 16) return launch_bn<16, false>(d, s, err);
  if (d.M <= 32) return launch_bn<32, false>(d, s, err);
  return launch_bn<64, false>(d, s, err);
}

}  // namespace q3
