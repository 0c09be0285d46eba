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
//   * grid = feature tiles x S; the S CTAs of one feature tile form a cluster and each
//     takes a contiguous range of the K blocks (64 wide);
//   * warp 0: TMA producer (weights 128 x 64 and tokens BN x 64 per K block, 128-byte
//     swizzle; the weight loads of the first stages precede the grid-dependency
//     wait, since no kernel of the call writes weights); warp 1: one thread issues
//     tcgen05.mma (M = 128, N = BN, K = 16) into one fp32 accumulator in tensor memory;
//     warps 2-5: epilogue;
//   * after the last MMA each CTA copies its accumulator to shared memory as
//     [token][feature]; after a cluster barrier, token t is finished by one warp of the
//     cluster, which adds the S partials in split order (deterministic) with
//     ld.shared::cluster and applies the epilogue: plain store, residual add, SwiGLU, or
//     per-head QK RMSNorm + rotate-half RoPE + KV-cache write;
//   * residual projections can also produce the RMSNorm of their whole output (the
//     norm that follows them in the block): every cluster stores its tile, takes a
//     ticket, and the cluster holding the last ticket normalises all token rows;
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

constexpr int kSkThreads = 192;
constexpr int kSkMaxSplits = 8;
constexpr uint32_t kSkPBytes = 128 * 64 * 2;  // weight tile: 128 features x 64 of K, bf16

// HILO: the activation operand holds 2M rows, row t = hi(a_t) and row M + t = lo(a_t)
// (a = hi + lo to about twice the type's precision); the MMA's N covers both and the
// accumulator columns t and M + t are added before the split sum.
// The ring is sized so that two CTAs fit on an SM (at most ~110 KB each): a CTA keeps
// its shared memory through the split reduction at its end, and the next projection's
// CTAs, which prefetch their weights before the grid-dependency wait, can then start
// beside it instead of after it.
template <int BN, bool HILO>
struct SkCfg {
  static constexpr int NQ = HILO ? 2 * BN : BN;  // activation rows per tile = MMA N
  static constexpr uint32_t Q_BYTES = NQ * 64 * 2;
  static constexpr uint32_t STAGE = kSkPBytes + Q_BYTES;
  static constexpr int STAGES = (int)(((110u << 10) - 1280u) / STAGE) > 8 ? 8 : (int)(((110u << 10) - 1280u) / STAGE);
  static constexpr uint32_t TMEM_COLS = NQ < 32 ? 32 : NQ;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 256;  // + barriers and flags
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
  int* ticket;
  QKRopeArgs qk;
  int f16;  // operands fp16 (else bf16); the SwiGLU and fused-norm outputs are fp16 too
  int* err;
};

}  // namespace

template <int BN, bool HILO>
__global__ void __launch_bounds__(kSkThreads, 2)
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
  volatile int* s_last = s_abort + 1;
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
  }
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nkb && ok; ++i) {
        const int st = i % kSkStages;
        const uint32_t ph = (uint32_t)(i / kSkStages) & 1u;
        uint8_t* sp = smem + st * C::STAGE;
        if (i < p_pre) {  // weights already on their way; the stage expects both halves
          tma_load_2d(sp + kSkPBytes, &tmQ, &full[st], (kb0 + i) * 64, 0);
          ++issued;
          continue;
        }
        if (*s_abort || !mbar_wait(&empty[st], ph ^ 1u, g.err)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[st], C::STAGE);
        tma_load_2d(sp, &tmP, &full[st], (kb0 + i) * 64, tile * 128);
        tma_load_2d(sp + kSkPBytes, &tmQ, &full[st], (kb0 + i) * 64, 0);
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
  } else {
    // ---------------------------------------------------------- accumulator -> smem
    const int quad = warp & 3;  // tensor-memory lanes [32 quad, 32 quad + 32)
    bool ok = mbar_wait(done, 0, g.err);
    ok = __all_sync(0xffffffffu, ok) && !*s_abort;
    tc_fence_after();
    const int f = quad * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
    // column j < M: token j (its hi half with HILO); column M + t: token t's lo half,
    // added after its hi value (columns are visited in increasing order)
    const int M = g.M;
    auto put = [&](int j, uint32_t r) {
      const float v = ok ? __uint_as_float(r) : 0.f;
      if (j < M) red[j * 128 + f] = v;
      else if (HILO && j < 2 * M) red[(j - M) * 128 + f] += v;
    };
    if constexpr (C::NQ == 16) {
      uint32_t r[16];
      tmem_ld16(taddr, r);
      tmem_wait_ld_regs16(r);
#pragma unroll
      for (int j = 0; j < 16; ++j) put(j, r[j]);
    } else {
      const int used = HILO ? 2 * M : M;
#pragma unroll 1
      for (int c = 0; c < C::NQ / 32; ++c) {
        if (c * 32 >= used) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_wait_ld_regs(r);
#pragma unroll
        for (int j = 0; j < 32; ++j) put(c * 32 + j, r[j]);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // every split's partial is in its CTA's shared memory

  if (warp >= 2 && !*s_abort) {
    // -------------------------------------------------- split sum + epilogue, one warp per token
    const int ew = (int)rank * 4 + (warp - 2);
    uint32_t rbase[kSkMaxSplits];
#pragma unroll
    for (int s = 0; s < kSkMaxSplits; ++s) rbase[s] = s < g.S ? mapa_shared(red, (uint32_t)s) : 0u;
    for (int t = ew; t < g.M; t += 4 * g.S) {
      float part[kSkMaxSplits][4];
#pragma unroll
      for (int s = 0; s < kSkMaxSplits; ++s)
        if (s < g.S)
#pragma unroll
          for (int j = 0; j < 4; ++j) part[s][j] = ld_cluster_f32(rbase[s] + (uint32_t)((t * 128 + 32 * j + lane) * 4));
      float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < kSkMaxSplits; ++s)
        if (s < g.S)
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] += part[s][j];
      if (g.epi == kEpiQKRope) {
        // slot = head of the fused QKV row: q heads, then k heads, then v heads
        const QKRopeArgs& a = g.qk;
        const int slot = tile;
        const int b = t / a.T;
        const int pos = a.pos_base[b] + (t - b * a.T);
        if (pos < 0 || pos >= a.s_max || pos >= a.max_pos) {
          if (lane == 0) record_error(g.err, kErrCapacity);
          continue;
        }
        if (slot >= a.Hq + a.Hkv) {  // value head: straight to the cache
          uint16_t* dst = a.cv + (((long long)b * a.Hkv + (slot - a.Hq - a.Hkv)) * a.s_max + pos) * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[32 * j + lane] = to_bf16_bits(v[j]);
          continue;
        }
        const bool is_q = slot < a.Hq;
        const uint16_t* wn = is_q ? a.q_norm : a.k_norm;
        const float ss = warp_sum(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
        const float r = rsqrtf(ss * (1.0f / 128.0f) + a.eps);
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] *= r * __uint_as_float((uint32_t)wn[32 * j + lane] << 16);
        // rotation pairs (d, d + 64): d = lane (v[0], v[2]) and d = 32 + lane (v[1], v[3])
        const float2 c0 = *reinterpret_cast<const float2*>(a.rope + ((long long)pos * 64 + lane) * 2);
        const float2 c1 = *reinterpret_cast<const float2*>(a.rope + ((long long)pos * 64 + 32 + lane) * 2);
        const float o[4] = {v[0] * c0.x - v[2] * c0.y, v[1] * c1.x - v[3] * c1.y, v[0] * c0.y + v[2] * c0.x,
                            v[1] * c1.y + v[3] * c1.x};  // dims lane, 32 + lane, 64 + lane, 96 + lane
        if (is_q && a.q2) {
          // hi/lo rows of the decode attention: group grp, head j of the group
          const int G = a.Hq / a.Hkv, grp = slot / G, j = slot - grp * G;
          uint16_t* hi = a.q2 + (long long)t * a.ldq2 + ((long long)grp * 2 * G + j) * 128;
          uint16_t* lo = hi + (long long)G * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint16_t h = to_bf16_bits(o[i]);
            hi[32 * i + lane] = h;
            lo[32 * i + lane] = to_bf16_bits(o[i] - __uint_as_float((uint32_t)h << 16));
          }
          continue;
        }
        uint16_t* dst = is_q ? static_cast<uint16_t*>(g.out) + (long long)t * g.ldo + (long long)slot * 128
                             : a.ck + (((long long)b * a.Hkv + (slot - a.Hq)) * a.s_max + pos) * 128;
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
            const float a = silu_f(v[j]) * u;
            const uint16_t hi = to_op_bits(f16, a);
            dst[16 * j + lane] = hi;
            if (g.out_lo) dst[g.out_lo + 16 * j + lane] = to_op_bits(f16, a - op_bits_to_f32(f16, hi));
          }
        }
      } else {
        const long long col = (long long)tile * 128 + lane;
        if (g.epi == kEpiResid) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            v[j] += g.resid_f32 ? static_cast<const float*>(g.resid)[(long long)t * g.ldr + col + 32 * j]
                                : __uint_as_float((uint32_t)static_cast<const uint16_t*>(
                                                      g.resid)[(long long)t * g.ldr + col + 32 * j]
                                                  << 16);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (g.out_f32) static_cast<float*>(g.out)[(long long)t * g.ldo + col + 32 * j] = v[j];
          else static_cast<uint16_t*>(g.out)[(long long)t * g.ldo + col + 32 * j] = to_bf16_bits(v[j]);
        }
      }
    }
  }

  if (g.norm_out) {
    // ------------------------------------------ RMSNorm of the whole output, last cluster
    __threadfence();  // this thread's output stores, visible to the whole GPU
    __syncwarp();
    cluster_sync();
    if (rank == 0 && threadIdx.x == 0) {
      const int prev = atomicAdd(g.ticket, 1);
      const uint32_t last = prev == (int)(gridDim.x / (unsigned)g.S) - 1 ? 1u : 0u;
      for (int s = 0; s < g.S; ++s) st_cluster_u32(mapa_shared((const void*)s_last, (uint32_t)s), last);
    }
    __syncwarp();
    cluster_sync();
    if (*s_last) {
      __threadfence();  // the other clusters' stores (their fences precede their tickets)
      const int gw = (int)rank * (kSkThreads / 32) + warp;
      const int nw = g.S * (kSkThreads / 32);
      const int N = g.N;
      for (int t = gw; t < g.M; t += nw) {
        float ss = 0.f;
        for (int col = lane * 8; col < N; col += 256) {
          float x[8];
          if (g.out_f32) {
            const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(g.out) + (long long)t * g.ldo + col);
            const float4 a = p[0], b = p[1];
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
          } else {
            const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g.out) + (long long)t * g.ldo + col);
            x[0] = bf16_lo(a.x); x[1] = bf16_hi(a.x); x[2] = bf16_lo(a.y); x[3] = bf16_hi(a.y);
            x[4] = bf16_lo(a.z); x[5] = bf16_hi(a.z); x[6] = bf16_lo(a.w); x[7] = bf16_hi(a.w);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) ss += x[j] * x[j];
        }
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)N + g.norm_eps);
        for (int col = lane * 8; col < N; col += 256) {
          float x[8];
          if (g.out_f32) {
            const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(g.out) + (long long)t * g.ldo + col);
            const float4 a = p[0], b = p[1];
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
          } else {
            const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g.out) + (long long)t * g.ldo + col);
            x[0] = bf16_lo(a.x); x[1] = bf16_hi(a.x); x[2] = bf16_lo(a.y); x[3] = bf16_hi(a.y);
            x[4] = bf16_lo(a.z); x[5] = bf16_hi(a.z); x[6] = bf16_lo(a.w); x[7] = bf16_hi(a.w);
          }
          const uint4 w = *reinterpret_cast<const uint4*>(g.norm_w + col);
          const bool f16 = g.f16 != 0;
          const float wv[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                               bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float a0 = x[2 * j] * r * wv[2 * j], a1 = x[2 * j + 1] * r * wv[2 * j + 1];
            hi[j] = pack_op_x2(f16, a0, a1);
            lo[j] = pack_op_x2(f16, a0 - op_bits_to_f32(f16, (uint16_t)(hi[j] & 0xFFFFu)),
                               a1 - op_bits_to_f32(f16, (uint16_t)(hi[j] >> 16)));
          }
          uint16_t* dst = g.norm_out + (long long)t * g.ld_norm + col;
          *reinterpret_cast<uint4*>(dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          if (g.norm_lo) *reinterpret_cast<uint4*>(dst + g.norm_lo) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // every cluster has taken its ticket: reset it for the next launch
      if (rank == 0 && threadIdx.x == 0) atomicExch(g.ticket, 0);
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

template <int BN, bool HILO>
int launch_bn(const SkinnyDesc& d, cudaStream_t s, int* err) {
  using C = SkCfg<BN, HILO>;
  if (ensure_smem_attr(reinterpret_cast<const void*>(gemm_skinny_kernel<BN, HILO>), (int)C::SMEM)) return -6;
  const int n_tiles = d.N / 128, k_blocks = d.K / 64;
  // splits: as many as fill the SMs in one wave of co-resident clusters
  int S = 1;
  for (int c = kSkMaxSplits; c >= 1; --c) {
    if ((long long)n_tiles * c > num_sms() || c > k_blocks) continue;
    if (c > 1 && !clusters_fit<BN, HILO>(c, n_tiles)) continue;
    S = c;
    break;
  }
  const int kpb = (k_blocks + S - 1) / S;
  S = (k_blocks + kpb - 1) / kpb;  // every split gets at least one K block
  CUtensorMap tmP, tmQ;
  if (make_tmap_2d(&tmP, d.W, d.N, d.K, d.ldw, 128) != 0 ||
      make_tmap_2d(&tmQ, d.A, HILO ? 2LL * d.M : d.M, d.K, d.lda, C::NQ) != 0) {
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

int launch_gemm_skinny(const SkinnyDesc& d, cudaStream_t s, int* err) {
  if (!skinny_supported(d.M, d.N, d.K, d.epi)) {
    set_last_error("skinny gemm: unsupported shape M %d N %d K %d", d.M, d.N, d.K);
    return -2;
  }
  if (d.norm_out && (d.epi != kEpiResid || !d.norm_w || !d.ticket || d.N % 256 != 0)) {
    set_last_error("skinny gemm: the fused RMSNorm needs the residual epilogue, weights, a ticket and N %% 256 == 0");
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
