// Tile micro-kernels of the persistent engine: per-warp compute on one shared-memory ring
// stage.  Every consumer warp processes every stage (its own rows, or its own positions);
// the stage layouts here must match the producer's stage_copy() in engine.cu.
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

// ---- GEMV: one warp computes NR (<= 4) whole rows of a stage ------------------------------
// rows[r] points at row r's K8 16-byte vectors in shared memory; x planes xl[j] = x[8j:8j+4],
// xh[j] = x[8j+4:8j+8].  NACC independent accumulators per row keep enough FMA chains in
// flight when a stage holds only one or two (long) rows.
template <int NR, int NACC>
__device__ __forceinline__ void gemv_rows(const uint4* r0, const uint4* r1, const uint4* r2,
                                          const uint4* r3, int K8, const float4* __restrict__ xl,
                                          const float4* __restrict__ xh, int lane, float& o0,
                                          float& o1, float& o2, float& o3) {
  const uint4* rp[4] = {r0, r1, r2, r3};
  float acc[NR][NACC];
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int a = 0; a < NACC; ++a) acc[r][a] = 0.f;
  int j = lane;
#pragma unroll 2
  for (; j + 32 * (NACC - 1) < K8; j += 32 * NACC) {
#pragma unroll
    for (int a = 0; a < NACC; ++a) {
      const float4 x0 = xl[j + 32 * a], x1 = xh[j + 32 * a];
#pragma unroll
      for (int r = 0; r < NR; ++r) acc[r][a] = dot8(rp[r][j + 32 * a], x0, x1, acc[r][a]);
    }
  }
  for (; j < K8; j += 32) {
    const float4 x0 = xl[j], x1 = xh[j];
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r][0] = dot8(rp[r][j], x0, x1, acc[r][0]);
  }
  float out[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float v = 0.f;
    if (r < NR) {
#pragma unroll
      for (int a = 0; a < NACC; ++a) v += acc[r][a];
    }
    out[r] = v;
  }
  o0 = out[0];
  o1 = out[1];
  o2 = out[2];
  o3 = out[3];
}

__device__ __forceinline__ void gemv_rows_n(int nr, const uint4* r0, const uint4* r1,
                                            const uint4* r2, const uint4* r3, int K8,
                                            const float4* xl, const float4* xh, int lane,
                                            float& o0, float& o1, float& o2, float& o3) {
  switch (nr) {
    case 4: gemv_rows<4, 1>(r0, r1, r2, r3, K8, xl, xh, lane, o0, o1, o2, o3); break;
    case 3: gemv_rows<3, 1>(r0, r1, r2, r3, K8, xl, xh, lane, o0, o1, o2, o3); break;
    case 2: gemv_rows<2, 2>(r0, r1, r2, r3, K8, xl, xh, lane, o0, o1, o2, o3); break;
    default: gemv_rows<1, 4>(r0, r1, r2, r3, K8, xl, xh, lane, o0, o1, o2, o3); break;
  }
}

// ---- split-KV decode attention: a warp's positions of one stage ----------------------------
// G query heads share one kv head; lane owns dims [lane*DPL, lane*DPL + DPL) of D = 32*DPL.
// q is pre-scaled by log2(e)/sqrt(D) so scores are in log2 units.  Running state per warp:
// m[h] (max), l[h] (sum of 2^(s-m)), o[h][:] (sum of 2^(s-m) v).  kb / vb point at this
// warp's first position's K and V rows (bf16, D each); nw <= kPosPerWarp positions.
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
__device__ __forceinline__ void attn_warp_positions(const uint8_t* kb, const uint8_t* vb, int nw,
                                                    const float (&q)[G][DPL], float (&m)[G],
                                                    float (&l)[G], float (&o)[G][DPL], int lane) {
  constexpr int D = 32 * DPL;
  constexpr int CP = 32 / G;                                   // positions per 32 scores
  constexpr int PPC = CP < kPosPerWarp ? CP : kPosPerWarp;     // positions per chunk
  constexpr int NCH = kPosPerWarp / PPC;                       // chunks per warp
  float sc[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    sc[c] = -INFINITY;
    if (c * PPC < nw) {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
#pragma unroll
      for (int pp = 0; pp < PPC; ++pp) {
        const int t = min(c * PPC + pp, nw - 1);
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
      const float s = reduce32(v, lane);  // score of position c*PPC + lane/G, head lane%G
      const int pp = lane / G;
      if (pp < PPC && c * PPC + pp < nw) sc[c] = s;
    }
  }
  // this stage's max per head (lanes with equal lane % G)
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
#pragma unroll
    for (int pp = 0; pp < PPC; ++pp) {
      const int t = c * PPC + pp;
      if (t < nw) {
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

}  // namespace tre
