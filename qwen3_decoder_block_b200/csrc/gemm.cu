// K2: persistent tcgen05 GEMM for the block's projections (QKV, o_proj, gate/up,
// down), the tied LM head, the MoE router and the grouped expert GEMMs.
//
// Every projection on the pages is an nn.Linear without bias, x @ W^T with W
// stored [out, in] ("从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构", section GQA;
// section SwiGLU FFN), so both operands are K-major and the kernel computes
// D[p][q] = sum_k P[p][k] Q[q][k].
//
// Design (sm_100a):
//   * one CTA per SM, persistent over output tiles of 128 x BN;
//   * warp 0: TMA producer (128-byte swizzled 128x64 and BNx64 tiles, mbarrier
//     ring of STAGES); warp 1: one thread issues tcgen05.mma (M=128, N=BN, K=16)
//     into a double-buffered fp32 accumulator in tensor memory; warps 2-5:
//     epilogue, tcgen05.ld of the accumulator, fused epilogue, global stores;
//   * swap mode for small M: the weight rows fill the MMA's 128-row side and the
//     tokens become N, so decode-sized GEMMs still stream the weights;
//   * grouped mode for MoE: per-expert row ranges of the permuted activations.
// Every wait is bounded (1 s of %globaltimer); on expiry the kernel records
// QWEN3_ETIMEOUT in the device error word, drains its copies and MMAs, frees
// its tensor memory and returns.
#include <cstdio>
#include <mutex>
#include <cudaTypedefs.h>
#include "common.cuh"
#include "internal.h"

namespace q3 {

constexpr int BM = 128;
constexpr int BK = 64;

// PAIR: the CTA is one half of a 2-CTA pair computing a 256 x BN tile with M = 256
// MMAs; it loads its 128 rows of A and BN/2 rows of B per stage.
// ROPE: the fused QK-norm + RoPE epilogue, which keeps RoPE rows 0..127 in the
// (otherwise unused) staging area, grown to 64 KB at the cost of one stage.
template <int BN, bool PAIR = false, bool ROPE = false>
struct GemmCfg {
  static constexpr int STAGES = PAIR ? (BN == 256 ? (ROPE ? 5 : 6) : 8) : (BN == 256 ? (ROPE ? 3 : 4) : (BN == 128 ? 6 : 8));
  static constexpr uint32_t P_BYTES = BM * BK * 2;
  static constexpr uint32_t Q_BYTES = (PAIR ? BN / 2 : BN) * BK * 2;
  static constexpr uint32_t STAGE_BYTES = P_BYTES + Q_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  // 4 epilogue warps x 2 buffers x 32x32 fp32, or the 128 x 128 fp32 RoPE rows
  static constexpr uint32_t STAGING_BYTES = ROPE ? 128 * 128 * 4 : 4 * 2 * 4096;
  static constexpr uint32_t BAR_BYTES = 256;
  static size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + STAGING_BYTES + BAR_BYTES + 8 * (size_t)(n_groups + 2);
  }
};

struct GemmParams {
  int p_rows, q_rows, k_blocks;
  int p_tiles, q_tiles, q_fast;
  int k_splits, kb_per_split;  // split-K: tile t covers k-blocks [ks*kb_per_split, ...)
  float* partial;              // split-K partials [k_splits][tokens][features] (fp32)
  int epi, resid_f32, out_f32, swap;
  int tma_store;  // non-swap store/residual epilogues: stage in shared memory, TMA tile store
  int f16;        // operands fp16 (else bf16); the SwiGLU output is fp16 too
  int p_early;    // P is final before this grid launches: its first tile's loads precede the grid-dependency wait
  void* out;
  long long ldo;
  const void* resid;
  long long ldr;
  int n_groups;
  const int* group_offsets;
  int* err;
  QKRopeArgs qk;
};

struct Tile {
  int p0, p_end, q0, q_end, q_load, kb0, kb1, ks;
  int p_out;  // output column of row p0 of the tile (grouped swap: p0 minus the group's first weight row)
};

__device__ __forceinline__ int total_tiles(const GemmParams& g, const int* s_prefix) {
  return g.n_groups > 0 ? s_prefix[g.n_groups] : g.p_tiles * g.q_tiles * g.k_splits;
}

// BMT: output rows per tile (128, or 256 for a CTA pair)
template <int BN, int BMT = BM>
__device__ __forceinline__ Tile decode_tile(int t, const GemmParams& g, const int* s_prefix, const int* s_off) {
  Tile r;
  r.kb0 = 0;
  r.kb1 = g.k_blocks;
  r.ks = 0;
  if (g.n_groups > 0) {
    int lo = 0, hi = g.n_groups - 1;  // largest grp with s_prefix[grp] <= t
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int grp = lo, local = t - s_prefix[grp];
    if (g.swap) {
      // weights of group grp on the 128-row side ([grp * p_rows, (grp + 1) * p_rows)), the
      // group's activation rows [off[grp], off[grp + 1]) as N; weight tiles fastest
      const int pt = local % g.p_tiles, qt = local / g.p_tiles;
      r.p0 = grp * g.p_rows + pt * BM;
      r.p_end = (grp + 1) * g.p_rows;
      r.p_out = pt * BM;
      r.q0 = s_off[grp] + qt * BN;
      r.q_end = s_off[grp + 1];
      r.q_load = r.q0;
      return r;
    }
    const int pt = local / g.q_tiles, qt = local % g.q_tiles;
    r.p0 = s_off[grp] + pt * BM;
    r.p_end = s_off[grp + 1];
    r.p_out = r.p0;
    r.q0 = qt * BN;
    r.q_end = g.q_rows;
    r.q_load = grp * g.q_rows + r.q0;
  } else {
    if (g.k_splits > 1) {
      r.ks = t % g.k_splits;
      t /= g.k_splits;
      r.kb0 = r.ks * g.kb_per_split;
      r.kb1 = min(g.k_blocks, r.kb0 + g.kb_per_split);
    }
    int pt, qt;
    if (g.q_fast) { pt = t / g.q_tiles; qt = t % g.q_tiles; }
    else          { qt = t / g.p_tiles; pt = t % g.p_tiles; }
    r.p0 = pt * BMT;
    r.p_end = g.p_rows;
    r.p_out = r.p0;
    r.q0 = qt * BN;
    r.q_end = g.q_rows;
    r.q_load = r.q0;
  }
  return r;
}

// --------------------------------------------------------------------------- epilogues
__device__ __forceinline__ void store_row_chunk(const GemmParams& g, int p, int q, const uint32_t (&r)[32]) {
  // non-swap: 32 accumulators of output row p, columns [q, q+32)
  if (g.epi == kEpiSwiglu) {
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float g0 = __uint_as_float(r[2 * j]), g1 = __uint_as_float(r[2 * j + 1]);
      float u0 = __uint_as_float(r[16 + 2 * j]), u1 = __uint_as_float(r[16 + 2 * j + 1]);
      o[j] = pack_op_x2(g.f16, silu_f(g0) * u0, silu_f(g1) * u1);
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(g.out) + (long long)p * g.ldo + (q >> 1));
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    return;
  }
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  if (g.epi == kEpiResid) {
    if (g.resid_f32) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(g.resid) + (long long)p * g.ldr + q);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 a = src[j];
        v[4 * j] += a.x; v[4 * j + 1] += a.y; v[4 * j + 2] += a.z; v[4 * j + 3] += a.w;
      }
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g.resid) + (long long)p * g.ldr + q);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 a = src[j];
        v[8 * j + 0] += bf16_lo(a.x); v[8 * j + 1] += bf16_hi(a.x);
        v[8 * j + 2] += bf16_lo(a.y); v[8 * j + 3] += bf16_hi(a.y);
        v[8 * j + 4] += bf16_lo(a.z); v[8 * j + 5] += bf16_hi(a.z);
        v[8 * j + 6] += bf16_lo(a.w); v[8 * j + 7] += bf16_hi(a.w);
      }
    }
  }
  if (g.out_f32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out) + (long long)p * g.ldo + q);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(g.out) + (long long)p * g.ldo + q);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                          pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
  }
}

// TMA-store epilogue: this thread's row (p < 0: outside the output, values unused) of a
// 32 x 32 chunk goes into a swizzled staging tile (128-byte swizzle for fp32 rows of
// 128 bytes, 64-byte swizzle for bf16 rows of 64 bytes) that one TMA store writes out.
__device__ __forceinline__ void stage_row_chunk(const GemmParams& g, int p, int q, const uint32_t (&r)[32],
                                                uint8_t* stg, int lane) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  if (g.epi == kEpiResid && p >= 0) {
    if (g.resid_f32) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(g.resid) + (long long)p * g.ldr + q);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 a = src[j];
        v[4 * j] += a.x; v[4 * j + 1] += a.y; v[4 * j + 2] += a.z; v[4 * j + 3] += a.w;
      }
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g.resid) + (long long)p * g.ldr + q);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 a = src[j];
        v[8 * j + 0] += bf16_lo(a.x); v[8 * j + 1] += bf16_hi(a.x);
        v[8 * j + 2] += bf16_lo(a.y); v[8 * j + 3] += bf16_hi(a.y);
        v[8 * j + 4] += bf16_lo(a.z); v[8 * j + 5] += bf16_hi(a.z);
        v[8 * j + 6] += bf16_lo(a.w); v[8 * j + 7] += bf16_hi(a.w);
      }
    }
  }
  if (g.out_f32) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4*>(stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
          make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                     pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
  }
}

// Residual values of row p (p < 0: outside the output, zeros), columns [q, q+32), as fp32.
__device__ __forceinline__ void load_resid_chunk(const GemmParams& g, int p, int q, float (&v)[32]) {
  if (p < 0) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = 0.f;
    return;
  }
  if (g.resid_f32) {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(g.resid) + (long long)p * g.ldr + q);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 a = src[j];
      v[4 * j] = a.x; v[4 * j + 1] = a.y; v[4 * j + 2] = a.z; v[4 * j + 3] = a.w;
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g.resid) + (long long)p * g.ldr + q);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 a = src[j];
      v[8 * j + 0] = bf16_lo(a.x); v[8 * j + 1] = bf16_hi(a.x);
      v[8 * j + 2] = bf16_lo(a.y); v[8 * j + 3] = bf16_hi(a.y);
      v[8 * j + 4] = bf16_lo(a.z); v[8 * j + 5] = bf16_hi(a.z);
      v[8 * j + 6] = bf16_lo(a.w); v[8 * j + 7] = bf16_hi(a.w);
    }
  }
}

// TMA-store staging of acc + res (see stage_row_chunk), the residual already loaded.
__device__ __forceinline__ void stage_row_chunk_res(const GemmParams& g, const uint32_t (&r)[32],
                                                    const float (&res)[32], uint8_t* stg, int lane) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + res[j];
  if (g.out_f32) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4*>(stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
          make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                     pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
  }
}

// swap: this thread owns feature p (one TMEM lane) and tokens [q, q+32)
__device__ __forceinline__ void store_col_chunk(const GemmParams& g, int p, int p_valid, int q, int q_end,
                                                int lane, int feat_block, const uint32_t (&r)[32]) {
  if (g.epi == kEpiSwiglu) {
    // lanes 0..15 hold gate features, lanes 16..31 the matching up features
    const int f = (feat_block >> 1) + lane;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float a = __uint_as_float(r[j]);
      float u = __shfl_down_sync(0xffffffffu, a, 16);
      if (lane < 16 && p_valid && q + j < q_end)
        static_cast<uint16_t*>(g.out)[(long long)(q + j) * g.ldo + f] = to_op_bits(g.f16, silu_f(a) * u);
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (!p_valid || q + j >= q_end) continue;
    float v = __uint_as_float(r[j]);
    const long long row = q + j;
    if (g.epi == kEpiResid) {
      if (g.resid_f32) v += static_cast<const float*>(g.resid)[row * g.ldr + p];
      else v += __uint_as_float((uint32_t)static_cast<const uint16_t*>(g.resid)[row * g.ldr + p] << 16);
    }
    if (g.out_f32) static_cast<float*>(g.out)[row * g.ldo + p] = v;
    else static_cast<uint16_t*>(g.out)[row * g.ldo + p] = to_bf16_bits(v);
  }
}

// Fused QKV epilogue for the two 128-column heads of a non-swap 256-column tile (one
// token row per thread): per-head RMSNorm over the 128 fp32 accumulators, weights,
// rotate-half RoPE at the token's absolute position, one bf16 rounding; q heads are
// written back in place (row p of out), k and v heads go to the KV cache at
// [b][g][pos][:] ("从零实现 Qwen3：拆解 mini-qwen3 的 0.6B Dense 架构", sections GQA and
// RoPE). The row's cos/sin values are read once for both heads. All 32 lanes execute
// the tensor-memory loads; only valid rows store.
// rope_lo: RoPE rows 0..127 in shared memory, row r's 16-byte chunk k stored at chunk
// k ^ (r & 31). The angle of position pos splits as (pos & ~127) + (pos & 127): its
// cos/sin follow from the two rows by the angle-addition formulas, so every thread
// reads one row shared by its warp (L1) and one row from shared memory, instead of a
// 512-byte row of its own.
__device__ __forceinline__ void qk_rope_tile(const GemmParams& g, uint32_t taddr, int slot0, int n_heads, int p,
                                             bool valid, const float* rope_lo) {
  const QKRopeArgs& a = g.qk;
  int b = 0, pos = 0;
  if (valid) {
    b = p / a.T;
    pos = a.pos_base[b] + (p - b * a.T);
    if (pos < 0 || pos >= a.s_max || pos >= a.max_pos) {
      record_error(g.err, kErrCapacity);
      valid = false;
    }
  }
  // pass 1: per-head sum of squares (value heads skip the norm)
  float rinv[2] = {0.f, 0.f};
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    if (hh >= n_heads || slot0 + hh >= a.Hq + a.Hkv) continue;  // warp-uniform
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 4; c += 2) {  // two loads in flight per wait
      uint32_t v[32], w[32];
      tmem_ld32(taddr + hh * 128 + c * 32, v);
      tmem_ld32(taddr + hh * 128 + c * 32 + 32, w);
      tmem_wait_ld_regs(v);
      tmem_wait_ld_regs(w);
#pragma unroll
      for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(v[i]), __uint_as_float(v[i]), ss);
#pragma unroll
      for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(w[i]), __uint_as_float(w[i]), ss);
    }
    rinv[hh] = rsqrtf(ss * (1.0f / 128.0f) + a.eps);
  }
  const float* rph = a.rope + (long long)(pos & ~127) * 128;
  const int lo = pos & 127;
  const float4* rpl = reinterpret_cast<const float4*>(rope_lo + lo * 128);
  // pass 2: dims d (first half) and d + 64 (second half) form one rotation pair
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    float4 cs[16];  // (cos_d, sin_d, cos_d+1, sin_d+1) for d = 32c .. 32c+31
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int k = c * 16 + i;
      if (valid) {
        const float4 h = *reinterpret_cast<const float4*>(rph + k * 4);
        const float4 l = rpl[k ^ (lo & 31)];
        cs[i] = make_float4(h.x * l.x - h.y * l.y, h.y * l.x + h.x * l.y, h.z * l.z - h.w * l.w,
                            h.w * l.z + h.z * l.w);
      } else {
        cs[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      if (hh >= n_heads) break;
      const int slot = slot0 + hh;
      uint32_t lo[32], hi[32];
      tmem_ld32(taddr + hh * 128 + c * 32, lo);
      tmem_ld32(taddr + hh * 128 + 64 + c * 32, hi);
      tmem_wait_ld_regs(lo);
      tmem_wait_ld_regs(hi);
      if (!valid) continue;
      uint32_t olo[16], ohi[16];
      uint16_t* dst;
      if (slot >= a.Hq + a.Hkv) {  // value head: straight to the cache
        dst = a.cv + (((long long)b * a.Hkv + (slot - a.Hq - a.Hkv)) * a.s_max + pos) * 128;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          olo[i] = pack_bf16x2(__uint_as_float(lo[2 * i]), __uint_as_float(lo[2 * i + 1]));
          ohi[i] = pack_bf16x2(__uint_as_float(hi[2 * i]), __uint_as_float(hi[2 * i + 1]));
        }
      } else {
        const bool is_q = slot < a.Hq;
        const uint16_t* wn = is_q ? a.q_norm : a.k_norm;
        dst = is_q ? static_cast<uint16_t*>(g.out) + (long long)p * g.ldo + (long long)slot * 128
                   : a.ck + (((long long)b * a.Hkv + (slot - a.Hq)) * a.s_max + pos) * 128;
        const float r = hh ? rinv[1] : rinv[0];
#pragma unroll
        for (int i8 = 0; i8 < 4; ++i8) {
          const uint4 wa = *reinterpret_cast<const uint4*>(wn + c * 32 + i8 * 8);
          const uint4 wb = *reinterpret_cast<const uint4*>(wn + 64 + c * 32 + i8 * 8);
          const uint32_t wa_[4] = {wa.x, wa.y, wa.z, wa.w}, wb_[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int i = i8 * 8 + e;
            const float4 t = cs[i / 2];
            const float a0 = __uint_as_float(lo[i]) * r * bf16_lo(wa_[e / 2]);
            const float a1 = __uint_as_float(lo[i + 1]) * r * bf16_hi(wa_[e / 2]);
            const float b0 = __uint_as_float(hi[i]) * r * bf16_lo(wb_[e / 2]);
            const float b1 = __uint_as_float(hi[i + 1]) * r * bf16_hi(wb_[e / 2]);
            olo[i / 2] = pack_bf16x2(a0 * t.x - b0 * t.y, a1 * t.z - b1 * t.w);
            ohi[i / 2] = pack_bf16x2(a0 * t.y + b0 * t.x, a1 * t.w + b1 * t.z);
          }
        }
      }
      uint4* dlo = reinterpret_cast<uint4*>(dst + c * 32);
      uint4* dhi = reinterpret_cast<uint4*>(dst + 64 + c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dlo[i] = make_uint4(olo[4 * i], olo[4 * i + 1], olo[4 * i + 2], olo[4 * i + 3]);
        dhi[i] = make_uint4(ohi[4 * i], ohi[4 * i + 1], ohi[4 * i + 2], ohi[4 * i + 3]);
      }
    }
  }
}

// --------------------------------------------------------------------------- kernel
template <int BN, bool PAIR, bool ROPE>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmO, const GemmParams g) {
  using C = GemmCfg<BN, PAIR, ROPE>;
  constexpr int BMT = PAIR ? 2 * BM : BM;  // output rows per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::STAGING_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(staging + C::STAGING_BYTES + C::BAR_BYTES);
  int* s_off = s_prefix + (g.n_groups + 1);  // only used in grouped mode (aliases past prefix)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // PAIR: rank 0 issues the MMAs for both CTAs; the tile loop runs over pairs
  const uint32_t rank = PAIR ? cluster_ctarank() : 0;
  const int t_first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int t_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    // PAIR: the 4 epilogue warps of both CTAs release an accumulator (one arrival each)
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], PAIR ? 8 : 128); }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == 32) { tma_prefetch_desc(&tmP); tma_prefetch_desc(&tmQ); }
  if (warp == 1) {
    if (PAIR) { tmem_alloc_pair(tmem_slot, C::TMEM_COLS); tmem_relinquish_pair(); }
    else      { tmem_alloc(tmem_slot, C::TMEM_COLS); tmem_relinquish(); }
  }
  // P loads of the first tile issued before the wait (producer thread only): when P is
  // a weight matrix that no kernel of this call writes, its stream from HBM overlaps
  // the previous kernel, and only the Q (activation) halves of these stages wait.
  int p_pre = 0;
  if constexpr (!PAIR) {
    if (g.p_early && g.n_groups == 0 && threadIdx.x == 0 && t_first < g.p_tiles * g.q_tiles * g.k_splits) {
      const Tile tl = decode_tile<BN, BMT>(t_first, g, nullptr, nullptr);
      p_pre = min(C::STAGES, tl.kb1 - tl.kb0);
      for (int i = 0; i < p_pre; ++i) {
        mbar_arrive_expect_tx(&full[i], C::STAGE_BYTES);
        tma_load_2d(smem + i * C::STAGE_BYTES, &tmP, &full[i], (tl.kb0 + i) * BK, tl.p0);
      }
    }
  }
  // Everything above touches only this CTA's own resources (and, with p_early,
  // memory no kernel of this call writes), so it overlaps the tail of the previous
  // kernel on the stream; all other global data is read after the wait.
  pdl_wait();
  pdl_trigger();
  if (g.n_groups > 0) {
    // per-group tile counts -> prefix (offsets are stored right after the prefix)
    for (int i = threadIdx.x; i <= g.n_groups; i += blockDim.x) s_off[i] = g.group_offsets[i];
    __syncthreads();
    if (threadIdx.x == 0) {
      int acc = 0;
      for (int i = 0; i < g.n_groups; ++i) {
        s_prefix[i] = acc;
        const int m = s_off[i + 1] - s_off[i];
        acc += g.swap ? ((m + BN - 1) / BN) * g.p_tiles : ((m + BM - 1) / BM) * g.q_tiles;
      }
      s_prefix[g.n_groups] = acc;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = total_tiles(g, s_prefix);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const uint32_t full_leader = PAIR ? mapa_shared(full, 0) : 0;
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = t_first; t < ntiles && ok; t += t_step) {
        const Tile tl = decode_tile<BN, BMT>(t, g, s_prefix, s_off);
        // PAIR: this CTA's 128 rows of A and BN/2 rows of B; both CTAs' copies complete
        // on the even CTA's full barrier, which expects the bytes of both
        const int a_row = tl.p0 + (int)rank * BM;
        const int b_row = tl.q_load + (int)rank * (BN / 2);
        for (int kb = tl.kb0; kb < tl.kb1; ++kb) {
          uint8_t* sp = smem + stage * C::STAGE_BYTES;
          if (issued < p_pre) {
            // P already on its way to this (fresh) stage, whose barrier expects both
            // halves: always add Q, so that every armed stage completes
            tma_load_2d(sp + C::P_BYTES, &tmQ, &full[stage], kb * BK, b_row);
            ++issued;
            if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
            continue;
          }
          if (*s_abort || !mbar_wait(&empty[stage], phase ^ 1, g.err)) { ok = false; break; }
          if (PAIR) {
            const uint32_t fb = full_leader + stage * 8;
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            tma_load_2d_pair(sp, &tmP, fb, kb * BK, a_row);
            tma_load_2d_pair(sp + C::P_BYTES, &tmQ, fb, kb * BK, b_row);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
            tma_load_2d(sp, &tmP, &full[stage], kb * BK, a_row);
            tma_load_2d(sp + C::P_BYTES, &tmQ, &full[stage], kb * BK, b_row);
          }
          ++issued;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        *s_abort = 1;
        // let every copy still in flight land before the CTA exits (PAIR: the even
        // CTA's barrier also counts the odd CTA's copies; neither CTA leaves before
        // the final cluster barrier)
        if (!PAIR || rank == 0)
          for (long long i = issued > C::STAGES ? issued - C::STAGES : 0; i < issued; ++i)
            mbar_wait(&full[i % C::STAGES], (uint32_t)((i / C::STAGES) & 1), g.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && (!PAIR || rank == 0)) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = g.f16 ? idesc_f16_f32(BMT, BN) : idesc_bf16_f32(BMT, BN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = t_first; t < ntiles && ok; t += t_step, ++local) {
        const Tile tl = decode_tile<BN, BMT>(t, g, s_prefix, s_off);
        const int buf = local & 1;
        const uint32_t use_par = (local >> 1) & 1;
        if (*s_abort || !mbar_wait(&tempty[buf], use_par ^ 1, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = tl.kb0; kb < tl.kb1; ++kb) {
          if (*s_abort || !mbar_wait(&full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint64_t adesc = sdesc_kmajor_sw128(sa);
          const uint64_t bdesc = sdesc_kmajor_sw128(sa + C::P_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            if (PAIR) mma_bf16_ss_pair(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb > tl.kb0 || kk) ? 1u : 0u);
            else      mma_bf16_ss(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb > tl.kb0 || kk) ? 1u : 0u);
          }
          if (PAIR) mma_commit_pair_mc(&empty[stage], 3);  // frees the stage in both CTAs
          else      mma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (PAIR) mma_commit_pair_mc(&tfull[buf], 3);
        else      mma_commit(&tfull[buf]);
      }
      if (!ok) {
        *s_abort = 1;
        // completes once every issued MMA has finished
        if (PAIR) mma_commit_pair(drain);
        else      mma_commit(drain);
        mbar_wait(drain, 0, g.err);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32) are reachable from this warp
    int local = 0;
    int sbuf = 0;
    // PAIR: this CTA's accumulator rows are rows [128 rank, 128 rank + 128) of the tile;
    // each warp releases the accumulator on the even CTA's barrier
    const uint32_t tempty_addr0 = PAIR ? mapa_shared(&tempty[0], 0) : 0;
    auto release_acc = [&](int b) {
      tc_fence_before();
      if (PAIR) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_addr0 + b * 8);
      } else {
        mbar_arrive(&tempty[b]);
      }
    };
    const float* rope_lo = reinterpret_cast<const float*>(staging);
    if (ROPE) {
      // RoPE rows 0..127 into shared memory (coalesced: a warp reads 512 contiguous bytes)
      const int et = threadIdx.x - 64;  // 0..127
      for (int i = et; i < 128 * 32; i += 128) {
        const int r = i >> 5, k = i & 31;
        const float4 v = r < g.qk.max_pos ? reinterpret_cast<const float4*>(g.qk.rope)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(staging)[r * 32 + (k ^ (r & 31))] = v;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");  // the 4 epilogue warps only
    }
    // residual epilogue with the TMA store: the residual (an input, final since the
    // grid-dependency wait) is read two 32-column chunks ahead of the accumulator, the
    // first two before the accumulator is waited for
    const bool res_path = !ROPE && g.tma_store && g.epi == kEpiResid;
    for (int t = t_first; t < ntiles; t += t_step, ++local) {
      Tile tl = decode_tile<BN, BMT>(t, g, s_prefix, s_off);
      if (PAIR) tl.p0 += (int)rank * BM;
      const int buf = local & 1;
      const uint32_t use_par = (local >> 1) & 1;
      const int row = quad * 32 + lane;
      float res[32], nxt[32];
      const int pr = tl.p0 + row < tl.p_end ? tl.p0 + row : -1;
      if (res_path) {
        load_resid_chunk(g, pr, tl.q0, res);
        if (BN > 32 && tl.q0 + 32 < tl.q_end) load_resid_chunk(g, pr, tl.q0 + 32, nxt);
      }
      bool ok = !*s_abort && mbar_wait(&tfull[buf], use_par, g.err);
      if (!__all_sync(0xffffffffu, ok)) { *s_abort = 1; break; }  // keep the warp converged
      tc_fence_after();
      if constexpr (ROPE) {
        // non-swap only: the tile's BN columns are BN/128 whole heads
        const int p = tl.p0 + row;
        const int heads = min(BN / 128, (tl.q_end - tl.q0) / 128);
        if (heads > 0)
          qk_rope_tile(g, tmem_base + ((uint32_t)(quad * 32) << 16) + buf * BN, tl.q0 / 128, heads, p,
                       p < tl.p_end, rope_lo);
      } else if (res_path) {
        // software-pipelined: the residual loads of chunk c + 2 are in flight while chunk
        // c is read from tensor memory, added and staged
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int q = tl.q0 + c * 32;
          if (q >= tl.q_end) break;  // warp-uniform
          const bool more = c + 1 < BN / 32 && q + 32 < tl.q_end;
          const bool more2 = c + 2 < BN / 32 && q + 64 < tl.q_end;
          float nxt2[32];
          if (more2) load_resid_chunk(g, pr, q + 64, nxt2);
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(quad * 32) << 16) + buf * BN + c * 32, r);
          tmem_wait_ld_regs(r);
          uint8_t* stg = staging + ((warp - 2) * 2 + sbuf) * 4096;
          if (lane == 0) bulk_wait_read<1>();  // the store that used this buffer has read it
          __syncwarp();
          stage_row_chunk_res(g, r, res, stg, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmO, stg, q, tl.p0 + quad * 32);
            bulk_commit();
          }
          sbuf ^= 1;
          if (more) {
#pragma unroll
            for (int j = 0; j < 32; ++j) res[j] = nxt[j];
          }
          if (more2) {
#pragma unroll
            for (int j = 0; j < 32; ++j) nxt[j] = nxt2[j];
          }
        }
      } else {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(quad * 32) << 16) + buf * BN + c * 32, r);
        tmem_wait_ld_regs(r);
        if (g.partial) {
          // split-K: raw fp32 partial sums, [ks][token][feature]
          if (!g.swap) {
            const int p = tl.p0 + row, q = tl.q0 + c * 32;
            if (p < tl.p_end && q < tl.q_end) {
              float4* dst = reinterpret_cast<float4*>(g.partial + ((long long)tl.ks * g.p_rows + p) * g.q_rows + q);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                     __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
            }
          } else {
            const int p = tl.p0 + row;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int q = tl.q0 + c * 32 + j;
              if (p < tl.p_end && q < tl.q_end)
                g.partial[((long long)tl.ks * g.q_rows + q) * g.p_rows + p] = __uint_as_float(r[j]);
            }
          }
        } else if (g.tma_store) {
          const int q = tl.q0 + c * 32;
          if (q < tl.q_end) {  // warp-uniform
            const int p = tl.p0 + row;
            uint8_t* stg = staging + ((warp - 2) * 2 + sbuf) * 4096;
            if (lane == 0) bulk_wait_read<1>();  // the store that used this buffer has read it
            __syncwarp();
            stage_row_chunk(g, p < tl.p_end ? p : -1, q, r, stg, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmO, stg, q, tl.p0 + quad * 32);
              bulk_commit();
            }
            sbuf ^= 1;
          }
        } else if (!g.swap) {
          const int p = tl.p0 + row, q = tl.q0 + c * 32;
          if (p < tl.p_end && q < tl.q_end) store_row_chunk(g, p, q, r);
        } else {
          // feature p_out + row of the output; grouped: the group's weight row p0 + row
          store_col_chunk(g, tl.p_out + row, tl.p0 + row < tl.p_end, tl.q0 + c * 32, tl.q_end, lane,
                          tl.p_out + quad * 32, r);
        }
      }
      }
      release_acc(buf);
    }
    if (g.tma_store && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  // PAIR: the even CTA's MMAs read the odd CTA's shared memory and write its tensor
  // memory; neither leaves before both are done
  if (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else      tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// --------------------------------------------------------------------------- split-K reduce
// out[m][n] = epilogue(sum_s part[s][m][n']) over tokens m and output features n;
// SwiGLU reads the packed gate column (n/16)*32 + n%16 and the up column 16 after it.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int S, int M, int N, int epi, int resid_f32,
                                     int out_f32, const void* __restrict__ resid, long long ldr,
                                     void* __restrict__ out, long long ldo, int f16) {
  pdl_wait();
  pdl_trigger();
  const int n_out = epi == kEpiSwiglu ? N / 2 : N;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)M * n_out) return;
  const int m = (int)(idx / n_out), n = (int)(idx % n_out);
  const long long plane = (long long)M * N;
  if (epi == kEpiSwiglu) {
    const int pg = (n / 16) * 32 + (n % 16);
    float gsum = 0.f, usum = 0.f;
    for (int s = 0; s < S; ++s) {
      gsum += part[s * plane + (long long)m * N + pg];
      usum += part[s * plane + (long long)m * N + pg + 16];
    }
    static_cast<uint16_t*>(out)[(long long)m * ldo + n] = to_op_bits(f16 != 0, silu_f(gsum) * usum);
    return;
  }
  float acc = 0.f;
  for (int s = 0; s < S; ++s) acc += part[s * plane + (long long)m * N + n];
  if (epi == kEpiResid) {
    if (resid_f32) acc += static_cast<const float*>(resid)[(long long)m * ldr + n];
    else acc += __uint_as_float((uint32_t)static_cast<const uint16_t*>(resid)[(long long)m * ldr + n] << 16);
  }
  if (out_f32) static_cast<float*>(out)[(long long)m * ldo + n] = acc;
  else static_cast<uint16_t*>(out)[(long long)m * ldo + n] = to_bf16_bits(acc);
}

// Split-K completion fused with the QK-norm + RoPE + KV-cache write (swap layout:
// part[s][token][feature]). One warp per (token m, head slot); lane l owns dims
// {2l, 2l+1} and {64+2l, 65+2l} of the slot. Token m of sequence b = m / T sits at
// position pos_base[b] + m % T. Sums in split order, then the same arithmetic as
// qk_norm_rope_kernel on the fp32 sums (q/k/v are not rounded before the norm).
__global__ void __launch_bounds__(256) splitk_qkrope_kernel(const float* __restrict__ part, int S, int M, int N,
                                                            uint16_t* __restrict__ qkv, long long ldqkv,
                                                            const QKRopeArgs a, int* err) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int slots = a.Hq + 2 * a.Hkv;
  const long long item = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (item >= (long long)M * slots) return;
  const int slot = (int)(item % slots);
  const int m = (int)(item / slots);
  const int b = m / a.T, t = m % a.T;
  const int pos = a.pos_base[b] + t;
  if (pos < 0 || pos >= a.s_max || pos >= a.max_pos) {
    if (lane == 0) record_error(err, kErrCapacity);
    return;
  }
  const long long plane = (long long)M * N;
  const float* src = part + (long long)m * N + slot * 128;
  float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
  int s = 0;
  for (; s + 4 <= S; s += 4) {  // four splits' loads in flight, added in split order
    float2 x0[4], x1[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x0[u] = *reinterpret_cast<const float2*>(src + (s + u) * plane + 2 * lane);
      x1[u] = *reinterpret_cast<const float2*>(src + (s + u) * plane + 64 + 2 * lane);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) { a0 += x0[u].x; a1 += x0[u].y; b0 += x1[u].x; b1 += x1[u].y; }
  }
  for (; s < S; ++s) {
    const float2 x0 = *reinterpret_cast<const float2*>(src + s * plane + 2 * lane);
    const float2 x1 = *reinterpret_cast<const float2*>(src + s * plane + 64 + 2 * lane);
    a0 += x0.x; a1 += x0.y; b0 += x1.x; b1 += x1.y;
  }
  if (slot >= a.Hq + a.Hkv) {  // value head: to the cache
    uint16_t* dst = a.cv + (((long long)b * a.Hkv + (slot - a.Hq - a.Hkv)) * a.s_max + pos) * 128;
    *reinterpret_cast<uint32_t*>(dst + 2 * lane) = pack_bf16x2(a0, a1);
    *reinterpret_cast<uint32_t*>(dst + 64 + 2 * lane) = pack_bf16x2(b0, b1);
    return;
  }
  const bool is_q = slot < a.Hq;
  const uint16_t* wn = is_q ? a.q_norm : a.k_norm;
  const float ss = warp_sum(a0 * a0 + a1 * a1 + b0 * b0 + b1 * b1);
  const float r = rsqrtf(ss * (1.0f / 128.0f) + a.eps);
  const uint32_t wa = *reinterpret_cast<const uint32_t*>(wn + 2 * lane);
  const uint32_t wb = *reinterpret_cast<const uint32_t*>(wn + 64 + 2 * lane);
  a0 *= r * bf16_lo(wa); a1 *= r * bf16_hi(wa);
  b0 *= r * bf16_lo(wb); b1 *= r * bf16_hi(wb);
  const float4 cs = *reinterpret_cast<const float4*>(a.rope + ((long long)pos * 64 + 2 * lane) * 2);
  const float o_a0 = a0 * cs.x - b0 * cs.y, o_b0 = a0 * cs.y + b0 * cs.x;
  const float o_a1 = a1 * cs.z - b1 * cs.w, o_b1 = a1 * cs.w + b1 * cs.z;
  uint16_t* dst = is_q ? qkv + (long long)m * ldqkv + (long long)slot * 128
                       : a.ck + (((long long)b * a.Hkv + (slot - a.Hq)) * a.s_max + pos) * 128;
  *reinterpret_cast<uint32_t*>(dst + 2 * lane) = pack_bf16x2(o_a0, o_a1);
  *reinterpret_cast<uint32_t*>(dst + 64 + 2 * lane) = pack_bf16x2(o_b0, o_b1);
}

// Split-K completion of a residual GEMM fused with the RMSNorm that follows it: one
// CTA of 1024 threads per token row m, PER = N / 1024 features per thread; out[m] =
// resid[m] + sum_s part[s][m] (summed in split order), then norm_out[m] =
// out[m] * rsqrt(mean(out[m]^2) + eps) * w on the fp32 values.
template <int PER>
__global__ void __launch_bounds__(1024) splitk_resid_norm_kernel(const float* __restrict__ part, int S, int M, int N,
                                                                 int resid_f32, int out_f32,
                                                                 const void* __restrict__ resid, long long ldr,
                                                                 void* __restrict__ out, long long ldo,
                                                                 const uint16_t* __restrict__ w,
                                                                 uint16_t* __restrict__ norm_out, float eps, int f16) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_red[32];
  const int m = blockIdx.x;
  const long long plane = (long long)M * N;
  const float* src = part + (long long)m * N + threadIdx.x;
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) v[i] = 0.f;
  int s = 0;
  for (; s + 8 <= S; s += 8) {  // eight splits' loads in flight, added in split order
    float x[8][PER];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int i = 0; i < PER; ++i) x[u][i] = src[(s + u) * plane + i * 1024];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int i = 0; i < PER; ++i) v[i] += x[u][i];
  }
  for (; s < S; ++s)
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] += src[s * plane + i * 1024];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int n = i * 1024 + threadIdx.x;
    v[i] += resid_f32 ? static_cast<const float*>(resid)[(long long)m * ldr + n]
                      : __uint_as_float((uint32_t)static_cast<const uint16_t*>(resid)[(long long)m * ldr + n] << 16);
    if (out_f32) static_cast<float*>(out)[(long long)m * ldo + n] = v[i];
    else static_cast<uint16_t*>(out)[(long long)m * ldo + n] = to_bf16_bits(v[i]);
    ss += v[i] * v[i];
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) tot += s_red[i];
  const float r = rsqrtf(tot / (float)N + eps);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int n = i * 1024 + threadIdx.x;
    norm_out[(long long)m * ldo + n] = to_op_bits(f16 != 0, v[i] * r * bf16_lo((uint32_t)w[n]));
  }
}

// --------------------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A tensor map is a function of its encode arguments only, and repeated calls (a decode
// step, a small layer) encode the same maps every time: they come from a hash table keyed
// by those arguments (open addressing over a short probe window, the window's first
// slot replaced when it is full; under a lock).
namespace {
struct TmapKey {
  int kind, rank;
  const void* base;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3];
};
constexpr int kTmapCache = 1024;  // a power of two
constexpr int kTmapProbe = 8;
struct TmapEntry {
  TmapKey key;
  CUtensorMap map;
  bool used;
};
std::mutex g_tmap_mu;
TmapEntry g_tmap[kTmapCache];

size_t key_hash(const TmapKey& k) {
  size_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
  auto mix = [&](unsigned long long v) { h = (h ^ v) * 0x100000001B3ull; };
  mix((unsigned long long)k.kind * 8 + (unsigned long long)k.rank);
  for (int i = 0; i < k.rank; ++i) {
    mix(k.dims[i]);
    mix(k.box[i]);
  }
  for (int i = 0; i + 1 < k.rank; ++i) mix(k.strides[i]);
  return h ^ (h >> 29);
}

bool same_key(const TmapKey& a, const TmapKey& b) {
  if (a.kind != b.kind || a.rank != b.rank || a.base != b.base) return false;
  for (int i = 0; i < a.rank; ++i)
    if (a.dims[i] != b.dims[i] || a.box[i] != b.box[i]) return false;
  for (int i = 0; i + 1 < a.rank; ++i)
    if (a.strides[i] != b.strides[i]) return false;
  return true;
}

// kind 0: bf16 operand, 128-byte swizzle, L2 256-byte promotion; 1: fp32 output, 128-byte
// swizzle; 2: bf16 output, 64-byte swizzle (the epilogue staging layouts)
int encode_cached(CUtensorMap* map, const TmapKey& k) {
  const size_t h0 = key_hash(k);
  {
    std::lock_guard<std::mutex> lk(g_tmap_mu);
    for (int i = 0; i < kTmapProbe; ++i) {
      const TmapEntry& e = g_tmap[(h0 + i) & (kTmapCache - 1)];
      if (!e.used) break;
      if (same_key(e.key, k)) {
        *map = e.map;
        return 0;
      }
    }
  }
  auto enc = get_encode();
  if (!enc) return -1;
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      enc(map, k.kind == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k.rank,
          const_cast<void*>(k.base), k.dims, k.strides, k.box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          k.kind == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
          k.kind == 0 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return -2;
  std::lock_guard<std::mutex> lk(g_tmap_mu);
  int slot = (int)(h0 & (kTmapCache - 1));  // replaced when the window is full
  for (int i = 0; i < kTmapProbe; ++i) {
    const int j = (int)((h0 + i) & (kTmapCache - 1));
    if (!g_tmap[j].used) {
      slot = j;
      break;
    }
  }
  TmapEntry& e = g_tmap[slot];
  e.key = k;
  e.map = *map;
  e.used = true;
  return 0;
}
}  // namespace

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with row stride ld
// (elements), box = box_rows x 64 columns, 128-byte swizzle, zero fill out of bounds.
int make_tmap_2d(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld, int box_rows) {
  TmapKey k = {};
  k.kind = 0;
  k.rank = 2;
  k.base = base;
  k.dims[0] = (cuuint64_t)cols;
  k.dims[1] = (cuuint64_t)rows;
  k.strides[0] = (cuuint64_t)(ld * 2);
  k.box[0] = 64;
  k.box[1] = (cuuint32_t)box_rows;
  return encode_cached(map, k);
}

// 3-D bf16 tensor map: dims (inner, mid, outer) with byte strides for mid and outer.
int make_tmap_3d(CUtensorMap* map, const void* base, long long inner, long long mid, long long outer,
                 long long mid_stride_bytes, long long outer_stride_bytes, int box_inner, int box_mid, int box_outer) {
  TmapKey k = {};
  k.kind = 0;
  k.rank = 3;
  k.base = base;
  k.dims[0] = (cuuint64_t)inner;
  k.dims[1] = (cuuint64_t)mid;
  k.dims[2] = (cuuint64_t)outer;
  k.strides[0] = (cuuint64_t)mid_stride_bytes;
  k.strides[1] = (cuuint64_t)outer_stride_bytes;
  k.box[0] = (cuuint32_t)box_inner;
  k.box[1] = (cuuint32_t)box_mid;
  k.box[2] = (cuuint32_t)box_outer;
  return encode_cached(map, k);
}

// Output tensor map for the TMA-store epilogue: [rows, cols] fp32 or bf16, box 32 x 32,
// 128-byte (fp32) or 64-byte (bf16) swizzle matching stage_row_chunk.
static int make_tmap_out(CUtensorMap* map, void* base, long long rows, long long cols, long long ld, bool f32) {
  TmapKey k = {};
  k.kind = f32 ? 1 : 2;
  k.rank = 2;
  k.base = base;
  k.dims[0] = (cuuint64_t)cols;
  k.dims[1] = (cuuint64_t)rows;
  k.strides[0] = (cuuint64_t)(ld * (f32 ? 4 : 2));
  k.box[0] = 32;
  k.box[1] = 32;
  return encode_cached(map, k);
}

// One kernel instantiation: shared-memory attribute (once per device), launch (CTA pairs as
// clusters of 2), launch-error check.
template <int BN, bool PAIR, bool ROPE>
static int launch_variant(const GemmParams& g, const CUtensorMap& tmP, const CUtensorMap& tmQ,
                          const CUtensorMap& tmO, cudaStream_t s) {
  using C = GemmCfg<BN, PAIR, ROPE>;
  if (ensure_smem_attr(reinterpret_cast<const void*>(gemm_tc_kernel<BN, PAIR, ROPE>), 227 * 1024)) return -6;
  const size_t smem = C::smem_bytes(g.n_groups);
  if (PAIR) {
    const long long tiles = (long long)g.p_tiles * g.q_tiles;
    const int pairs = (int)(tiles < num_sms() / 2 ? tiles : num_sms() / 2);
    if (pairs <= 0) return 0;
    q3_launch_cluster(gemm_tc_kernel<BN, PAIR, ROPE>, 2 * pairs, 192, smem, s, 2, tmP, tmQ, tmO, g);
  } else {
    int grid;
    if (g.n_groups > 0) {
      grid = num_sms();
    } else {
      const long long tiles = (long long)g.p_tiles * g.q_tiles * g.k_splits;
      grid = (int)(tiles < num_sms() ? tiles : num_sms());
    }
    if (grid <= 0) return 0;
    q3_launch(gemm_tc_kernel<BN, PAIR, ROPE>, grid, 192, smem, s, tmP, tmQ, tmO, g);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("gemm launch failed: %s", cudaGetErrorString(e));
    return -6;
  }
  return 0;
}

template <int BN>
static int launch_bn(const GemmDesc& d, cudaStream_t s, int* err) {
  using C = GemmCfg<BN>;
  CUtensorMap tmP, tmQ;
  // grouped: the weight operand holds every group's rows (P when swapped, else Q)
  const long long p_total = d.n_groups > 0 && d.swap ? d.p_rows_total : d.p_rows;
  if (make_tmap_2d(&tmP, d.P, p_total, d.K, d.ldp, BM) != 0) {
    set_last_error("gemm: cannot encode the tensor map of operand P");
    return -6;
  }
  // Large plain GEMMs run on CTA pairs (M = 256 MMAs; each CTA loads half of B)
  const bool pair = BN == 256 && !d.swap && d.n_groups == 0 && d.p_rows >= 2 * BM && gemm_pair_enabled();
  const long long q_total = d.n_groups > 0 && !d.swap ? d.q_rows_total : d.q_rows;
  if (make_tmap_2d(&tmQ, d.Q, q_total, d.K, d.ldq, pair ? BN / 2 : BN) != 0) {
    set_last_error("gemm: cannot encode the tensor map of operand Q");
    return -6;
  }
  GemmParams g;
  g.p_rows = d.p_rows;
  g.q_rows = d.q_rows;
  g.k_blocks = d.K / BK;
  g.p_tiles = (d.p_rows + (pair ? 2 * BM : BM) - 1) / (pair ? 2 * BM : BM);
  g.q_tiles = (d.q_rows + BN - 1) / BN;
  // Keep the smaller operand cache-resident: sweep fastest over the tiles of the
  // operand that is re-read, so that the larger operand streams from HBM once.
  g.q_fast = (long long)d.q_rows <= (long long)d.p_rows ? 1 : 0;
  g.epi = d.epi;
  g.resid_f32 = d.resid_f32;
  g.out_f32 = d.out_f32;
  g.swap = d.swap;
  g.out = d.out;
  g.ldo = d.ldo;
  g.resid = d.resid;
  g.ldr = d.ldr;
  g.n_groups = d.n_groups;
  g.group_offsets = d.group_offsets;
  g.err = err;
  g.qk = d.qk;
  g.f16 = d.f16 ? 1 : 0;
  g.k_splits = 1;
  g.kb_per_split = g.k_blocks;
  g.partial = nullptr;
  g.p_early = d.p_early && !pair && d.n_groups == 0 ? 1 : 0;
  // Split K when the output has too few tiles to keep the SMs streaming: each split
  // writes fp32 partials, and a reduce kernel applies the epilogue.
  const long long out_tiles = (long long)g.p_tiles * g.q_tiles;
  if (!pair && d.n_groups == 0 && d.epi != kEpiQKRope && d.partial && out_tiles * 2 <= num_sms() && g.k_blocks > 1) {
    int S = (int)(num_sms() / out_tiles);
    if (S > g.k_blocks) S = g.k_blocks;
    const size_t per_split = (size_t)d.p_rows * d.q_rows * sizeof(float);
    while (S > 1 && (size_t)S * per_split > d.partial_bytes) --S;
    if (S > 1) {
      g.kb_per_split = (g.k_blocks + S - 1) / S;
      g.k_splits = (g.k_blocks + g.kb_per_split - 1) / g.kb_per_split;
      g.partial = d.partial;
    }
  }
  // TMA-store epilogue for the plain non-swap store / residual epilogues
  CUtensorMap tmO = tmP;
  g.tma_store = 0;
  if (!d.swap && d.n_groups == 0 && g.k_splits == 1 && (d.epi == kEpiStore || d.epi == kEpiResid) &&
      (reinterpret_cast<uintptr_t>(d.out) & 15) == 0 && (d.ldo * (d.out_f32 ? 4 : 2)) % 16 == 0) {
    if (make_tmap_out(&tmO, d.out, d.p_rows, d.q_rows, d.ldo, d.out_f32) == 0) g.tma_store = 1;
  }
  if constexpr (BN == 256) {
    if (d.epi == kEpiQKRope)
      return pair ? launch_variant<BN, true, true>(g, tmP, tmQ, tmO, s) : launch_variant<BN, false, true>(g, tmP, tmQ, tmO, s);
    if (pair) return launch_variant<BN, true, false>(g, tmP, tmQ, tmO, s);
  } else {
    if (d.epi == kEpiQKRope) {
      set_last_error("gemm: the fused QK-norm/RoPE epilogue needs 256-column tiles");
      return -1;
    }
  }
  int rc = launch_variant<BN, false, false>(g, tmP, tmQ, tmO, s);
  if (rc) return rc;
  if (g.k_splits > 1) {
    const int M = d.swap ? d.q_rows : d.p_rows, N = d.swap ? d.p_rows : d.q_rows;
    const long long n_out = (long long)M * (d.epi == kEpiSwiglu ? N / 2 : N);
    if (d.qk_in_reduce && d.swap && d.epi == kEpiStore) {
      const long long warps = (long long)M * (d.qk.Hq + 2 * d.qk.Hkv);
      q3_launch(splitk_qkrope_kernel, (unsigned)((warps * 32 + 255) / 256), 256, 0, s, g.partial, g.k_splits, M, N,
                static_cast<uint16_t*>(d.out), d.ldo, d.qk, err);
      if (d.fused) *d.fused = 1;
    } else if (d.norm_out && d.norm_w && d.epi == kEpiResid && (N == 1024 || N == 2048)) {
      if (N == 1024)
        q3_launch(splitk_resid_norm_kernel<1>, (unsigned)M, 1024, 0, s, g.partial, g.k_splits, M, N,
                  d.resid_f32 ? 1 : 0, d.out_f32 ? 1 : 0, d.resid, d.ldr, d.out, d.ldo, d.norm_w, d.norm_out,
                  d.norm_eps, g.f16);
      else
        q3_launch(splitk_resid_norm_kernel<2>, (unsigned)M, 1024, 0, s, g.partial, g.k_splits, M, N,
                  d.resid_f32 ? 1 : 0, d.out_f32 ? 1 : 0, d.resid, d.ldr, d.out, d.ldo, d.norm_w, d.norm_out,
                  d.norm_eps, g.f16);
      if (d.fused) *d.fused = 1;
    } else {
      q3_launch(splitk_reduce_kernel, (unsigned)((n_out + 255) / 256), 256, 0, s, g.partial, g.k_splits, M, N,
                d.epi, d.resid_f32, d.out_f32, d.resid, d.ldr, d.out, d.ldo, g.f16);
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("gemm launch failed: %s", cudaGetErrorString(e));
    return -6;
  }
  return 0;
}

int launch_gemm(const GemmDesc& d, cudaStream_t s, int* err) {
  int bn = d.force_bn;
  if (bn == 0) {
    if (d.swap) bn = d.q_rows <= 64 ? 64 : (d.q_rows <= 128 ? 128 : 256);
    else bn = 256;
  }
  switch (bn) {
    case 64: return launch_bn<64>(d, s, err);
    case 128: return launch_bn<128>(d, s, err);
    case 256: return launch_bn<256>(d, s, err);
    default:
      set_last_error("gemm: unsupported tile width %d", bn);
      return -1;
  }
}

}  // namespace q3
