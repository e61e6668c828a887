// GEMV tile micro-kernels of the persistent engine: one consumer warp computes whole rows
// of one shared-memory ring stage (the stage layout matches issue_stage() in engine.cu).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
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

// ---- E4M3 weights on the tensor cores ---------------------------------------------------------
// f32 -> E4M3 (nearest, saturating) for two values, the first in the low byte; and back.
__device__ __forceinline__ uint32_t f2_to_e4m3x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t v) {
  const __half2_raw h =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v & 0xffffu), __NV_E4M3);
  __half2 hh;
  *reinterpret_cast<__half2_raw*>(&hh) = h;
  return __half22float2(hh);
}

// ---- MXFP4 rows (FP4 routed experts) --------------------------------------------------------
// Two E2M1 codes (the low byte of v: the first in the low nibble) -> their values.
__device__ __forceinline__ float2 e2m1x2_to_f2(uint32_t v) {
  const __half2_raw h =
      __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(v & 0xffu), __NV_E2M1);
  __half2 hh;
  *reinterpret_cast<__half2_raw*>(&hh) = h;
  return __half22float2(hh);
}

// E8M0 scale byte -> 2^(s - 127) (s = 0: 2^-127, a subnormal; s = 255: NaN).
__device__ __forceinline__ float e8m0_to_f(uint32_t s) {
  return __uint_as_float(s == 0u ? 0x00400000u : s == 255u ? 0x7fc00000u : s << 23);
}

// sum_k W[k] x[k] over 8 E2M1 weights (one 32-bit word: weight 2i in the low nibble of
// byte i) against the x planes a = x[0:4], b = x[4:8] (the bf16 rows' planes).
__device__ __forceinline__ float dot8_e2m1(uint32_t w, const float4 a, const float4 b) {
  const float2 p0 = e2m1x2_to_f2(w), p1 = e2m1x2_to_f2(w >> 8);
  const float2 p2 = e2m1x2_to_f2(w >> 16), p3 = e2m1x2_to_f2(w >> 24);
  float s = p0.x * a.x;
  s = fmaf(p0.y, a.y, s);
  s = fmaf(p1.x, a.z, s);
  s = fmaf(p1.y, a.w, s);
  s = fmaf(p2.x, b.x, s);
  s = fmaf(p2.y, b.y, s);
  s = fmaf(p3.x, b.z, s);
  s = fmaf(p3.y, b.w, s);
  return s;
}

// One warp computes NR (<= 4) whole MXFP4 rows of Kp weights (Kp a multiple of 32) of a
// stage: row r's codes are Kp / 2 bytes at rows[r], its scales the Kp / 32 bytes after
// them.  Lane l takes the 8-weight groups j = l, l + 32, ...: a 32-bit code word, the x
// planes of the bf16 rows (xl[j] = x[8j:8j+4], xh[j] = x[8j+4:8j+8]) and the scale of
// group j / 4; each group's 8 products are summed before its scale multiplies them.
template <int NR>
__device__ __forceinline__ void gemv_rows_e2m1(const uint8_t* r0, const uint8_t* r1,
                                               const uint8_t* r2, const uint8_t* r3, int Kp,
                                               const float4* __restrict__ xl,
                                               const float4* __restrict__ xh, int lane,
                                               float& o0, float& o1, float& o2, float& o3) {
  const uint8_t* rp[4] = {r0, r1, r2, r3};
  const int K8 = Kp >> 3, half = Kp >> 1;
  float acc[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) acc[r] = 0.f;
#pragma unroll 2
  for (int j = lane; j < K8; j += 32) {
    const float4 x0 = xl[j], x1 = xh[j];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const uint32_t w = reinterpret_cast<const uint32_t*>(rp[r])[j];
      const float sc = e8m0_to_f(rp[r][half + (j >> 2)]);
      acc[r] = fmaf(dot8_e2m1(w, x0, x1), sc, acc[r]);
    }
  }
  float out[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) out[r] = r < NR ? acc[r] : 0.f;
  o0 = out[0];
  o1 = out[1];
  o2 = out[2];
  o3 = out[3];
}

__device__ __forceinline__ void gemv_rows_e2m1_n(int nr, const uint8_t* r0, const uint8_t* r1,
                                                 const uint8_t* r2, const uint8_t* r3, int Kp,
                                                 const float4* xl, const float4* xh, int lane,
                                                 float& o0, float& o1, float& o2, float& o3) {
  switch (nr) {
    case 4: gemv_rows_e2m1<4>(r0, r1, r2, r3, Kp, xl, xh, lane, o0, o1, o2, o3); break;
    case 3: gemv_rows_e2m1<3>(r0, r1, r2, r3, Kp, xl, xh, lane, o0, o1, o2, o3); break;
    case 2: gemv_rows_e2m1<2>(r0, r1, r2, r3, Kp, xl, xh, lane, o0, o1, o2, o3); break;
    default: gemv_rows_e2m1<1>(r0, r1, r2, r3, Kp, xl, xh, lane, o0, o1, o2, o3); break;
  }
}

// ---- GEMV for MT tokens: one warp computes NR (<= 4) whole rows against MT input vectors -----
// Token v's planes start vs float4s after token 0's.  Each weight vector is loaded once and
// used for every token (the MT tokens give the FMA chains their independence).
template <int NR, int MT>
__device__ __forceinline__ void gemv_rows_mt(const uint4* r0, const uint4* r1, const uint4* r2,
                                             const uint4* r3, int K8, const float4* __restrict__ xl,
                                             const float4* __restrict__ xh, int vs, int lane,
                                             float (&out)[MT][4]) {
  const uint4* rp[4] = {r0, r1, r2, r3};
  float acc[MT][NR];
#pragma unroll
  for (int v = 0; v < MT; ++v)
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[v][r] = 0.f;
  for (int j = lane; j < K8; j += 32) {
    uint4 w[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) w[r] = rp[r][j];
#pragma unroll
    for (int v = 0; v < MT; ++v) {
      const float4 x0 = xl[v * vs + j], x1 = xh[v * vs + j];
#pragma unroll
      for (int r = 0; r < NR; ++r) acc[v][r] = dot8(w[r], x0, x1, acc[v][r]);
    }
  }
#pragma unroll
  for (int v = 0; v < MT; ++v)
#pragma unroll
    for (int r = 0; r < 4; ++r) out[v][r] = r < NR ? acc[v][r] : 0.f;
}

template <int MT>
__device__ __forceinline__ void gemv_rows_mt_n(int nr, const uint4* r0, const uint4* r1,
                                               const uint4* r2, const uint4* r3, int K8,
                                               const float4* xl, const float4* xh, int vs,
                                               int lane, float (&out)[MT][4]) {
  switch (nr) {
    case 4: gemv_rows_mt<4, MT>(r0, r1, r2, r3, K8, xl, xh, vs, lane, out); break;
    case 3: gemv_rows_mt<3, MT>(r0, r1, r2, r3, K8, xl, xh, vs, lane, out); break;
    case 2: gemv_rows_mt<2, MT>(r0, r1, r2, r3, K8, xl, xh, vs, lane, out); break;
    default: gemv_rows_mt<1, MT>(r0, r1, r2, r3, K8, xl, xh, vs, lane, out); break;
  }
}

}  // namespace tre
