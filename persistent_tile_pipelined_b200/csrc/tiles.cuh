// Tile micro-kernels of the persistent engine: warp-level compute on one shared-memory
// ring stage.  The stage layouts here must match stage_desc() in engine.cu.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "tre_internal.h"

namespace tre {

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// acc + sum_k W[k] x[k] over 8 bf16 weights; x split in planes a = x[0:4], b = x[4:8].
__device__ __forceinline__ float dot8(const uint4 w, const float4 a, const float4 b, float acc) {
  acc = fmaf(bf_lo(w.x), a.x, acc);
  acc = fmaf(bf_hi(w.x), a.y, acc);
  acc = fmaf(bf_lo(w.y), a.z, acc);
  acc = fmaf(bf_hi(w.y), a.w, acc);
  acc = fmaf(bf_lo(w.z), b.x, acc);
  acc = fmaf(bf_hi(w.z), b.y, acc);
  acc = fmaf(bf_lo(w.w), b.z, acc);
  acc = fmaf(bf_hi(w.w), b.w, acc);
  return acc;
}

// Sum four per-lane partials across the warp with 6 shuffles (transpose-reduce).
// Lane l ends with the total of value (l >> 4 & 1) * 2 + (l >> 3 & 1).
__device__ __forceinline__ float reduce4(float a0, float a1, float a2, float a3, int lane) {
  const bool b4 = lane & 16;
  float s0 = b4 ? a0 : a2, s1 = b4 ? a1 : a3;
  float k0 = b4 ? a2 : a0, k1 = b4 ? a3 : a1;
  k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
  const bool b3 = lane & 8;
  float s = b3 ? k0 : k1;
  float k = b3 ? k1 : k0;
  k += __shfl_xor_sync(0xffffffffu, s, 8);
  k += __shfl_xor_sync(0xffffffffu, k, 4);
  k += __shfl_xor_sync(0xffffffffu, k, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

// Sum 32 per-lane values across the warp with 31 shuffles; lane l ends with the total
// of value l.
__device__ __forceinline__ float reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool up = lane & half;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      float send = up ? v[i] : v[i + half];
      float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}

// ---- GEMV on one stage ------------------------------------------------------------------
// The stage holds rows [n0, n0 + nr) of the op's matrix (and, for the gate/up op, the same
// rows of the second matrix at byte offset seg1).  x is the input vector in two planes:
// xl[j] = x[8j : 8j+4], xh[j] = x[8j+4 : 8j+8].  `emit(row, value)` is called by one lane
// per row with the full dot product (gate/up: emit2(row, gate, up)).
template <class Emit>
__device__ __forceinline__ void gemv_stage_rows(const uint8_t* slot, int K8, int nr,
                                                const float4* __restrict__ xl,
                                                const float4* __restrict__ xh, int lane,
                                                Emit&& emit) {
  const uint4* base = reinterpret_cast<const uint4*>(slot);
  for (int r = 0; r < nr; r += 4) {
    const uint4* w0 = base + (size_t)r * K8;
    const uint4* w1 = base + (size_t)min(r + 1, nr - 1) * K8;
    const uint4* w2 = base + (size_t)min(r + 2, nr - 1) * K8;
    const uint4* w3 = base + (size_t)min(r + 3, nr - 1) * K8;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 2
    for (int j = lane; j < K8; j += 32) {
      const float4 x0 = xl[j], x1 = xh[j];
      a0 = dot8(w0[j], x0, x1, a0);
      a1 = dot8(w1[j], x0, x1, a1);
      a2 = dot8(w2[j], x0, x1, a2);
      a3 = dot8(w3[j], x0, x1, a3);
    }
    const float v = reduce4(a0, a1, a2, a3, lane);
    const int row = r + ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
    if ((lane & 7) == 0 && row < nr) emit(row, v);
  }
}

template <class Emit2>
__device__ __forceinline__ void gemv_stage_pairs(const uint8_t* slot, size_t seg1, int K8, int nr,
                                                 const float4* __restrict__ xl,
                                                 const float4* __restrict__ xh, int lane,
                                                 Emit2&& emit2) {
  const uint4* g = reinterpret_cast<const uint4*>(slot);
  const uint4* u = reinterpret_cast<const uint4*>(slot + seg1);
  for (int r = 0; r < nr; r += 2) {
    const int rb = min(r + 1, nr - 1);
    const uint4* g0 = g + (size_t)r * K8;
    const uint4* g1 = g + (size_t)rb * K8;
    const uint4* u0 = u + (size_t)r * K8;
    const uint4* u1 = u + (size_t)rb * K8;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 2
    for (int j = lane; j < K8; j += 32) {
      const float4 x0 = xl[j], x1 = xh[j];
      a0 = dot8(g0[j], x0, x1, a0);
      a1 = dot8(g1[j], x0, x1, a1);
      a2 = dot8(u0[j], x0, x1, a2);
      a3 = dot8(u1[j], x0, x1, a3);
    }
    // lanes 0 / 8 hold gate(r) / gate(r+1); lanes 16 / 24 hold up(r) / up(r+1)
    const float v = reduce4(a0, a1, a2, a3, lane);
    const float up = __shfl_xor_sync(0xffffffffu, v, 16);
    const int row = r + ((lane >> 3) & 1);
    if ((lane & 23) == 0 && row < nr) emit2(row, v, up);
  }
}

// ---- split-KV decode attention on one stage -----------------------------------------------
// G query heads share one kv head; lane owns dims [lane*DPL, lane*DPL + DPL) of D = 32*DPL.
// q is pre-scaled by log2(e)/sqrt(D) so scores are in log2 units.  Running state per warp:
// m[h] (max), l[h] (sum of 2^(s-m)), o[h][:] (sum of 2^(s-m) v).  kb / vb hold n <= 64
// consecutive positions of K and V rows (bf16, D each).
template <int DPL>
__device__ __forceinline__ void load_bf16_row(const uint8_t* p, float (&f)[DPL]) {
  if constexpr (DPL == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    f[0] = bf_lo(w.x); f[1] = bf_hi(w.x); f[2] = bf_lo(w.y); f[3] = bf_hi(w.y);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    f[0] = bf_lo(w); f[1] = bf_hi(w);
  }
}

template <int G, int DPL>
__device__ __forceinline__ void attn_stage(const uint8_t* kb, const uint8_t* vb, int n,
                                           const float (&q)[G][DPL], float (&m)[G], float (&l)[G],
                                           float (&o)[G][DPL], int lane) {
  constexpr int D = 32 * DPL;
  constexpr int CP = 32 / G;                 // positions per 32-score chunk
  constexpr int NCH = kMaxPosPerStage / CP;  // chunks per stage (max)
  float sc[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    sc[c] = -INFINITY;
    if (c * CP < n) {
      float v[32];
#pragma unroll
      for (int pp = 0; pp < CP; ++pp) {
        const int t = min(c * CP + pp, n - 1);
        float kf[DPL];
        load_bf16_row<DPL>(kb + ((size_t)t * D + lane * DPL) * 2, kf);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float a = 0.f;
#pragma unroll
          for (int j = 0; j < DPL; ++j) a = fmaf(q[h][j], kf[j], a);
          v[pp * G + h] = a;
        }
      }
      const float s = reduce32(v, lane);  // score of position c*CP + lane/G, head lane%G
      if (c * CP + lane / G < n) sc[c] = s;
    }
  }
  // stage max per head (lanes with equal lane % G)
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < NCH; ++c) mx = fmaxf(mx, sc[c]);
#pragma unroll
  for (int off = G; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float mnew[G], corr[G];
  float my_m = 0.f;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float mh = __shfl_sync(0xffffffffu, mx, h);
    mnew[h] = fmaxf(m[h], mh);
    corr[h] = exp2f(m[h] - mnew[h]);  // m = -inf before the first stage: corr = 0
    if ((lane % G) == h) my_m = mnew[h];
  }
  float ps = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    sc[c] = exp2f(sc[c] - my_m);  // -inf (padding) -> 0
    ps += sc[c];
  }
#pragma unroll
  for (int off = G; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    l[h] = l[h] * corr[h] + __shfl_sync(0xffffffffu, ps, h);
    m[h] = mnew[h];
#pragma unroll
    for (int j = 0; j < DPL; ++j) o[h][j] *= corr[h];
  }
  // o += p V
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c * CP < n) {
#pragma unroll
      for (int pp = 0; pp < CP; ++pp) {
        const int t = c * CP + pp;
        if (t < n) {
          float vf[DPL];
          load_bf16_row<DPL>(vb + ((size_t)t * D + lane * DPL) * 2, vf);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pr = __shfl_sync(0xffffffffu, sc[c], pp * G + h);
#pragma unroll
            for (int j = 0; j < DPL; ++j) o[h][j] = fmaf(pr, vf[j], o[h][j]);
          }
        }
      }
    }
  }
}

}  // namespace tre
