// Tensor-core helpers of the persistent engine (mma.sync, ldmatrix, swizzled tensor-map
// tiles) used by the GQA flash-decode tile and the absorbed-MLA latent attention.
//
// Absorbed MLA (DeepSeek-V2's; the pages name the fused kernel FlashSparseMLA with
// batch == 1 — TileRT code audit, blog-vs-code table — and fold the query heads of a
// latent tile together — Speed is intelligence talk, section on the attention kernel) is
// multi-query attention of H heads over one latent row per position: query head h is
// [W_uk,h^T q_nope,h | RoPE(q_pe,h)] (KL + R wide), every key is the cached latent row
// [c_kv | k_pe] and every value its first KL columns.  That is a dense contraction per
// position tile (16 heads x (KL + R) x 32 positions), so it runs on the tensor cores with
// mma.sync m16n8k16 (bf16 in, fp32 accumulate).  Keys and values are bf16 already; the
// fp32 query and probabilities are split into bf16 hi + lo parts and both parts go
// through the product, which keeps about 16 significand bits of them.
//
// A latent stage is 32 cached rows brought in by 2-D tensor copies of 64-column boxes
// with the 128-byte swizzle, so ldmatrix reads rows 1152 bytes apart without bank
// conflicts: chunk c (16 bytes) of row r of box b lives at b * 4096 + r * 128 + ((c ^ (r & 7)) << 4).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"
#include "tre_internal.h"

namespace tre {

// ---- tensor-core helpers ------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// d += a * b for one 16x8x16 tile (A row-major 16x16, B column-major 16x8, fp32 C).
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d = a * b for one 16x8x32 tile of E4M3 operands (A row-major 16x32, B column-major 32x8,
// fp32 D): thread (g, t4) holds A bytes (row g, k 4 t4 .. + 3), (row g + 8, same k),
// (row g, k 16 + 4 t4 ..), (row g + 8, ...) and B bytes (k 4 t4 .., n = g), (k 16 + 4 t4 ..).
__device__ __forceinline__ void mma_e4m3(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

// x0, x1 -> packed bf16 pairs hi = rn(x), lo = rn(x - hi); the lower column in the low half.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  hi = bf2_bits(h);
  lo = bf2_bits(__floats2bfloat162_rn(x0 - hf.x, x1 - hf.y));
}

// Byte offset of 16-byte chunk c (0..7) of row r of box b in a stage of `rows`-row boxes
// of 64 bf16 columns, as the 128-byte swizzle lays them out (boxes 1024-byte aligned).
__device__ __forceinline__ uint32_t swz_off(int b, int r, int c, int rows) {
  return (uint32_t)(b * rows * 128 + r * 128 + ((c ^ (r & 7)) << 4));
}

// Byte offset of 16-byte chunk `ch` (columns 8 ch .. 8 ch + 7) of row r of a latent stage.
__device__ __forceinline__ uint32_t lat_off(int r, int ch) {
  return swz_off(ch >> 3, r, ch & 7, kMlaPosPerStage);
}

// 2-D tensor copy of one box into shared memory, completing on `bar`.
// Order this thread's later tensor copies through `map` (a 128-byte tensor map in global
// memory) after generic-proxy writes of it, such as a host copy that rewrote the map at
// the same address before this launch.
__device__ __forceinline__ void tensormap_acquire(const void* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(map) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace tre
