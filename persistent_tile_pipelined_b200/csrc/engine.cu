// The persistent engine kernel: one CTA per SM runs that SM's static task queue for one
// whole decode step.
//
// Roles inside a CTA (Static Compilation for LLM Inference, §5.2: a TMA copy warp group
// stands in for the DMA engine, a compute group with the activation fused in):
//   * warp 8 (one elected lane) is the PRODUCER: it walks the queue and streams every
//     task's weight rows (or KV rows) into a ring of shared-memory stages with 1-D bulk
//     copies that complete on the stage's "full" mbarrier.  Weights and cached KV never
//     depend on this step's activations, so the producer never waits for a dependency:
//     it runs ahead across op boundaries as far as the ring allows — the cross-op
//     overlap of compute and HBM traffic the pages describe (§1; tile pipeline §5.1).
//   * warps 0-7 are CONSUMERS: per task they wait for the task's dependency counter,
//     stage the input vector (RMSNorm folded in) in shared memory, consume the ring
//     stages round-robin (one warp per stage), run the epilogue, and publish by bumping
//     the task's output counter with release semantics.
// Every wait is bounded; on expiry the first error is recorded, an abort flag makes every
// CTA drain, and the kernel returns (no trap, no hang).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "mla.cuh"
#include "ptx.cuh"
#include "tiles.cuh"
#include "tre_internal.h"

namespace tre {

// ---- errors -------------------------------------------------------------------------------
__device__ __noinline__ void record_error(const Params& p, int code, int detail) {
  if (atomicCAS(p.err, 0, code) == 0) {
    p.status_host[1] = detail;
    __threadfence_system();
    p.status_host[0] = code;
    __threadfence_system();
  }
  *p.abort_flag = 1;
  __threadfence();
}

__device__ __forceinline__ bool aborted(const Params& p) { return *p.abort_flag != 0; }

// Poll loops look at the abort flag and their time budget once per ~16 us of SM clock: the
// flag is a global-memory read, and a waiter stalled on it notices its own event late.
constexpr long long kCheckCycles = 1 << 15;

// GEMV input staging: items each thread fetches before storing any (tensor-core fragments;
// fp32 planes).
constexpr int kLoadBatch = 2;
#ifndef TRE_PLANE_BATCH
#define TRE_PLANE_BATCH 2
#endif
constexpr int kPlaneBatch = TRE_PLANE_BATCH;

// Wait until counter `idx` reaches epoch * count (wrap-safe).  Bounded; on expiry the
// error names `detail` (a task index).  A kernel-per-op launch never waits: the launches
// before it in the stream met every dependency of its tasks.
__device__ bool wait_counter(const Params& p, int idx, uint32_t count, int detail) {
  if (p.op_group >= 0) return true;
  const uint32_t target = p.epoch * count;
  const uint32_t* c = p.counters + (size_t)idx * kCtrStride;
  if ((int32_t)(ld_acquire_gpu(c) - target) >= 0) return true;
  const uint64_t t0 = globaltimer_ns();
  long long c0 = clock64();
  for (;;) {
    if ((int32_t)(ld_acquire_gpu(c) - target) >= 0) return true;
    if (clock64() - c0 > kCheckCycles) {
      if (aborted(p)) return false;
      if ((long long)(globaltimer_ns() - t0) > p.timeout_ns) {
        record_error(p, TRE_ERR_DEP_TIMEOUT, detail);
        return false;
      }
      c0 = clock64();
    }
  }
}

// Wait until the task's dependency counter reaches epoch * t.dep_count.
__device__ __forceinline__ bool wait_dep(const Params& p, const Task& t) {
  if (t.dep < 0) return true;
  return wait_counter(p, t.dep, t.dep_count, t.id);
}

// Bounded wait on an mbarrier phase; `slack` scales the time budget (ring waits get
// twice the dependency budget so that a dependency timeout is reported first).
__device__ bool mbar_wait(const Params& p, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  long long c0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - c0 > kCheckCycles) {
      if (aborted(p)) return false;
      if ((long long)(globaltimer_ns() - t0) > 2 * p.timeout_ns) {
        record_error(p, TRE_ERR_DEP_TIMEOUT, -1);
        return false;
      }
      c0 = clock64();
    }
  }
}

// Wait for ring stage `sidx` to land.  GEMV stages are taken round-robin by single warps,
// so a warp can reach a slot before the slot's previous stage (sidx - NS) was even
// issued; a parity wait there would match the previous phase.  The producer therefore
// tags each slot with the stage it claimed (after that slot's previous stage was
// consumed, which implies its full-barrier phase completed); waiting for the tag first
// keeps every parity wait at most one phase ahead.
__device__ bool stage_wait_at(const Params& p, uint64_t* full, const uint32_t* tags, uint32_t sidx,
                              uint32_t slot, uint32_t parity);

__device__ bool stage_wait(const Params& p, uint64_t* full, const uint32_t* tags, uint32_t sidx) {
  const uint32_t NS = (uint32_t)p.ring_stages;
  return stage_wait_at(p, full, tags, sidx, sidx % NS, (sidx / NS) & 1u);
}

// The ring slot and phase parity of the next stage.
__device__ __forceinline__ void ring_next(uint32_t& slot, uint32_t& par, uint32_t NS) {
  if (++slot == NS) {
    slot = 0;
    par ^= 1u;
  }
}

// The same with the slot and phase parity of stage sidx known to the caller.
__device__ bool stage_wait_at(const Params& p, uint64_t* full, const uint32_t* tags, uint32_t sidx,
                              uint32_t slot, uint32_t parity) {
  const volatile uint32_t* tag = tags + slot;
  if (*tag != sidx) {
    const uint64_t t0 = globaltimer_ns();
    long long c0 = clock64();
    while (*tag != sidx) {
      __nanosleep(64);  // yield issue slots to the warps that are computing
      if (clock64() - c0 > kCheckCycles) {
        if (aborted(p)) return false;
        if ((long long)(globaltimer_ns() - t0) > 2 * p.timeout_ns) {
          record_error(p, TRE_ERR_DEP_TIMEOUT, -2);
          return false;
        }
        c0 = clock64();
      }
    }
  }
  return mbar_wait(p, &full[slot], parity);
}

// ---- task geometry (shared by producer and consumers) ---------------------------------------
// GEMV task: rows [r0, r1) of the op's matrix (gate/up: the same rows of both matrices),
// streamed as stages of whole contiguous rows (one bulk copy per contiguous run of rows).
__device__ __forceinline__ int gemv_K(const Params& p, int op) {
  switch (op) {
    case OP_O: return p.Hq * p.D;
    case OP_DOWN: return p.F;
    case OP_MDOWN: return (p.nshared + p.topk) * p.Fe;
    case OP_UQ: return p.QL;
    case OP_UK: case OP_UV: return p.KL;   // W_uk / W_uv rows are KL wide
    case OP_MO: case OP_MOS: return p.Hq * p.VD;
    default: return p.d;
  }
}

// Tasks whose weight addresses depend on this step's routing (the selected experts).
__device__ __forceinline__ bool needs_route(const Params& p, const Task& t) {
  return t.type == T_GEMV && (t.op == OP_RGU || (t.op == OP_MDOWN && (t.aux & 0xff) >= p.nshared));
}

// The expert selected in slot j of `layer` (valid once the layer's route counter is met);
// an id outside [0, E) records a bounds error and is clamped so no access leaves the
// expert tensors.
__device__ __forceinline__ int routed_expert(const Params& p, int layer, int j, int detail) {
  const int e = __ldcg(p.route_idx + layer * p.topk + j);
  if (e < 0 || e >= p.E) {
    record_error(p, TRE_ERR_BOUNDS, detail);
    return 0;
  }
  return e;
}
struct GemvGeom {
  int K;        // full row length (inputs)
  int nseg;     // 2 for gate/up (a row of each matrix), else 1
  int np, part; // K-parts of the op and this task's part
  int k0, Kp;   // this part's input columns [k0, k0 + Kp)
  int rps;      // rows per ring stage
  int nstages;
  int nkk;      // tiles (multi-token plans): stages per row tile and segment (k-chunks)
  int esz;      // bytes per weight: 2 (bf16), 1 (E4M3 projections)
  int rowb;     // bytes of one row of the K-part as stored and copied (MXFP4: the pitch)
  bool f4;      // MXFP4 rows (FP4 routed experts)
};

// F4: the FP4-expert kernel (only its tasks can be MXFP4 rows; the other kernels fold f4 away)
template <bool TILED, bool F4 = false>
__device__ __forceinline__ GemvGeom gemv_geom(const Params& p, const Task& t) {
  GemvGeom g;
  g.K = gemv_K(p, t.op);
  g.nseg = (t.op == OP_GU || t.op == OP_SGU || t.op == OP_RGU) ? 2 : 1;
  g.esz = (p.wfp8 && (t.op == OP_QKV || t.op == OP_O || t.op == OP_GU || t.op == OP_DOWN)) ? 1 : 2;
  if (t.op == OP_LM || t.op == OP_ROUTER) {
    g.np = 1;
    g.part = 0;
  } else if (t.op == OP_MDOWN) {  // aux = slot | block << 8
    g.part = t.aux & 0xff;
    g.np = p.nshared + p.topk;
  } else if (t.op == OP_MOS) {    // aux = slice | block << 8 | slices << 16
    g.part = t.aux & 0xff;
    g.np = (t.aux >> 16) & 0xff;
  } else {
    g.part = t.aux & 0xff;
    g.np = max(1, t.aux >> 8);
  }
  const int len = g.np == 1 ? g.K : gemv_part_len(g.K, g.np, gemv_part_align(TILED, g.esz == 1));
  g.k0 = g.part * len;
  g.Kp = min(len, g.K - g.k0);
  g.f4 = F4 && p.wfp4 && (t.op == OP_RGU || (t.op == OP_MDOWN && g.part >= p.nshared));
  g.rowb = g.f4 ? fp4_row_pitch(g.Kp) : g.Kp * g.esz;
  if (TILED) {  // row tiles of 16; per tile and segment, k-chunks of kTileK columns
    g.rps = kTileRows;
    g.nkk = (g.Kp + kTileK - 1) / kTileK;
    g.nstages = (t.r1 - t.r0 + kTileRows - 1) / kTileRows * g.nseg * g.nkk;
  } else {
    // E4M3: one tensor-core tile of 8 rows (gate / up: 4 of each) per stage at most
    g.rps = g.esz == 1 ? min(8 / g.nseg, fp8_rows_per_stage(g.Kp, g.nseg, p.stage_bytes))
            : g.f4     ? max(1, p.stage_bytes / (g.nseg * g.rowb))
                       : gemv_rows_per_stage(g.Kp, g.nseg, p.stage_bytes, g.esz);
    g.nkk = 1;
    g.nstages = (t.r1 - t.r0 + g.rps - 1) / g.rps;
  }
  return g;
}

// Source (byte address) of this task's K-part of row n of segment `seg`; *contig receives
// how many rows from n on follow it contiguously in memory (same matrix, row stride = the
// part length): QKV rows cross from Wq into Wk into Wv, routed rows end at their expert's
// last row, K-parts of a wider matrix are one row each.  Offsets count weights of g.esz
// bytes (E4M3 projections: 1); MXFP4 expert rows count whole rows of their pitch.
__device__ __forceinline__ const uint8_t* wbytes(const uint16_t* w) {
  return reinterpret_cast<const uint8_t*>(w);
}

__device__ __forceinline__ const uint8_t* part_row(const Params& p, const Task& t,
                                                   const GemvGeom& g, int seg, int n,
                                                   int* contig) {
  *contig = 0x7fffffff;
  const size_t e = (size_t)g.esz;
  if (t.op == OP_LM) return wbytes(p.lm_head) + (size_t)n * g.K * 2;
  const LayerPtrs& L = p.layers[t.layer];
  const size_t K = (size_t)g.K;
  switch (t.op) {
    case OP_QKV: {
      const int nq = p.Hq * p.D, nk = p.Hkv * p.D;
      if (n < nq) { *contig = nq - n; return wbytes(L.w[TRE_W_Q]) + (size_t)n * K * e; }
      if (n < nq + nk) { *contig = nq + nk - n; return wbytes(L.w[TRE_W_K]) + (size_t)(n - nq) * K * e; }
      return wbytes(L.w[TRE_W_V]) + (size_t)(n - nq - nk) * K * e;
    }
    case OP_O:
    case OP_DOWN:
      if (g.np > 1) *contig = 1;
      return wbytes(L.w[t.op == OP_O ? TRE_W_O : TRE_W_DOWN]) + ((size_t)n * K + g.k0) * e;
    case OP_GU: return wbytes(L.w[seg ? TRE_W_UP : TRE_W_GATE]) + (size_t)n * K * e;
    case OP_ROUTER: return wbytes(L.w[TRE_W_ROUTER]) + (size_t)n * K * 2;
    case OP_MDQKV: {  // W_dq, W_dkv, then (sparse) W_ik
      const int C = p.KL + p.R;
      if (n < p.QL) { *contig = p.QL - n; return wbytes(L.w[TRE_W_DQ]) + (size_t)n * K * 2; }
      if (n < p.QL + C) {
        *contig = p.QL + C - n;
        return wbytes(L.w[TRE_W_DKV]) + (size_t)(n - p.QL) * K * 2;
      }
      return wbytes(L.w[TRE_W_INDEX_K]) + (size_t)(n - p.QL - C) * K * 2;
    }
    case OP_UQ: {  // W_uq, then (sparse) W_iq
      const int nq = p.Hq * (p.NP + p.R);
      if (n < nq) { *contig = nq - n; return wbytes(L.w[TRE_W_UQ]) + (size_t)n * K * 2; }
      return wbytes(L.w[TRE_W_INDEX_Q]) + (size_t)(n - nq) * K * 2;
    }
    case OP_UK: return wbytes(L.w[TRE_W_UK]) + (size_t)n * K * 2;
    case OP_UV: return wbytes(L.w[TRE_W_UV]) + (size_t)n * K * 2;
    case OP_MO:
    case OP_MOS:
      if (g.np > 1) *contig = 1;
      return wbytes(L.w[TRE_W_MLA_O]) + ((size_t)n * K + g.k0) * 2;
    case OP_SGU: return wbytes(L.w[seg ? TRE_W_SHARED_UP : TRE_W_SHARED_GATE]) + (size_t)n * K * 2;
    case OP_RGU: {
      const int j = n / p.Fe, r = n - j * p.Fe;
      const int ex = routed_expert(p, t.layer, j, t.id);
      *contig = p.Fe - r;
      return wbytes(L.w[seg ? TRE_W_EXPERT_UP : TRE_W_EXPERT_GATE]) +
             ((size_t)ex * p.Fe + r) * (g.f4 ? (size_t)g.rowb : K * 2);
    }
    default: {  // OP_MDOWN: part < nshared is a column slice of the shared down matrix
      if (g.part < p.nshared) {
        if (p.nshared > 1) *contig = 1;
        return wbytes(L.w[TRE_W_SHARED_DOWN]) +
               ((size_t)n * p.nshared * p.Fe + (size_t)g.part * p.Fe) * 2;
      }
      const int ex = routed_expert(p, t.layer, g.part - p.nshared, t.id);
      return wbytes(L.w[TRE_W_EXPERT_DOWN]) +
             ((size_t)ex * p.d + n) * (g.f4 ? (size_t)g.rowb : (size_t)p.Fe * 2);
    }
  }
}

// Block scales of an E4M3 GEMV task, resolved once per task: row n of segment seg uses the
// scale row base[...] + (row within its matrix / 128) * KB, where KB = ceil(K / 128); QKV
// rows cross from Wq's scales into Wk's into Wv's at split[0], split[1].
struct Fp8Scales {
  const float* base[3];
  int split[2];
  int KB;
};

__device__ __forceinline__ Fp8Scales fp8_scales(const Params& p, const Task& t, const GemvGeom& g) {
  const LayerPtrs& L = p.layers[t.layer];
  auto sc = [&](int slot) { return reinterpret_cast<const float*>(L.w[slot]); };
  Fp8Scales f;
  f.KB = (g.K + 127) >> 7;
  f.split[0] = f.split[1] = 0x7fffffff;
  f.base[1] = f.base[2] = nullptr;
  switch (t.op) {
    case OP_QKV:
      f.base[0] = sc(TRE_W_SCALE_Q);
      f.base[1] = sc(TRE_W_SCALE_K);
      f.base[2] = sc(TRE_W_SCALE_V);
      f.split[0] = p.Hq * p.D;
      f.split[1] = (p.Hq + p.Hkv) * p.D;
      break;
    case OP_O: f.base[0] = sc(TRE_W_SCALE_O); break;
    case OP_GU:
      f.base[0] = sc(TRE_W_SCALE_GATE);
      f.base[1] = sc(TRE_W_SCALE_UP);
      break;
    default: f.base[0] = sc(TRE_W_SCALE_DOWN); break;
  }
  return f;
}

__device__ __forceinline__ const float* fp8_scale_row(const Fp8Scales& f, int seg, int n) {
  if (seg) return f.base[1] + (size_t)(n >> 7) * f.KB;                 // gate/up: up rows
  if (n < f.split[0]) return f.base[0] + (size_t)(n >> 7) * f.KB;
  if (n < f.split[1]) return f.base[1] + (size_t)((n - f.split[0]) >> 7) * f.KB;
  return f.base[2] + (size_t)((n - f.split[1]) >> 7) * f.KB;
}

// ---- sparse MLA ----------------------------------------------------------------------------------
// A sparse plan's step attends to chosen positions once pos + 1 > K (before that, to all).
__device__ __forceinline__ bool sparse_step(const Params& p) { return p.KI > 0 && p.pos + 1 > p.KI; }
__device__ __forceinline__ uint32_t* index_meta(const Params& p, int layer) {
  return p.ix_meta + (size_t)layer * IM_WORDS;
}
// Order key of a float: larger floats have larger keys (one key for -0 and +0 is the
// caller's business).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Positions of a task's stages.  GQA attention: split sp of [0, pos) (the last split a
// half share: it also takes the new positions); MLA attention: split sp of [0, pos), or
// in a sparse step entries [t0, t1) of the layer's chosen positions (read once the
// selection is published); index scoring: split sp of the cached positions [0, pos).
__device__ __forceinline__ void attn_range(const Params& p, const Task& t, int& t0, int& t1) {
  long long P = p.pos;
  const long long S = t.aux, sp = t.r1;
  if (t.type == T_MLA_ATTN && sparse_step(p))
    P = min(__ldcg(index_meta(p, t.layer) + IM_NSEL), (uint32_t)p.KI);
  if (t.type == T_ATTN) {
    t0 = (int)(P * 2 * sp / (2 * S - 1));
    t1 = sp + 1 == S ? (int)P : (int)(P * 2 * (sp + 1) / (2 * S - 1));
    return;
  }
  t0 = (int)(P * sp / S);
  t1 = (int)(P * (sp + 1) / S);
}

template <bool TILED, bool F4 = false>
__device__ __forceinline__ int task_nstages(const Params& p, const Task& t) {
  if (t.type == T_GEMV) return gemv_geom<TILED, F4>(p, t).nstages;
  if (t.type == T_ISEL) return 0;
  int t0, t1;
  attn_range(p, t, t0, t1);
  const int rows = t.type == T_INDEX ? kIndexRows : p.pps;
  return (t1 - t0 + rows - 1) / rows;
}

// Where a GEMV task's rows come from, resolved once per task (expert ids and layer
// pointers are looked up here, not per stage): row n of segment s of the task's K-part
// starts at base[s] + (n - r0) * stride.  QKV rows cross from Wq into Wk into Wv, so QKV
// whole-row stages are resolved per stage instead (lookup = true); for those ops base[]
// holds the matrices themselves, row n from base[0] below split[0], base[1] below
// split[1], else base[2] (used by the tile stages).
struct RowSrc {
  const uint8_t* base[3];
  long long stride;   // bytes between consecutive rows in memory
  int split[2];
  bool lookup;        // whole-row stages: resolve every stage with part_row
};

__device__ __forceinline__ RowSrc row_src(const Params& p, const Task& t, const GemvGeom& g) {
  RowSrc r;
  r.lookup = t.op == OP_QKV || t.op == OP_MDQKV || (t.op == OP_UQ && p.KI > 0);
  r.stride = (long long)g.K * g.esz;
  if (t.op == OP_RGU) r.stride = g.f4 ? (long long)g.rowb : 2LL * p.d;
  else if (t.op == OP_MDOWN)
    r.stride = g.f4 ? (long long)g.rowb : 2LL * (g.part < p.nshared ? (long long)p.nshared * p.Fe : p.Fe);
  int contig;
  r.base[2] = nullptr;
  r.split[0] = r.split[1] = 0x7fffffff;
  if (r.lookup) {
    const LayerPtrs& L = p.layers[t.layer];
    if (t.op == OP_QKV) {
      r.base[0] = wbytes(L.w[TRE_W_Q]);
      r.base[1] = wbytes(L.w[TRE_W_K]);
      r.base[2] = wbytes(L.w[TRE_W_V]);
      r.split[0] = p.Hq * p.D;
      r.split[1] = (p.Hq + p.Hkv) * p.D;
    } else if (t.op == OP_MDQKV) {
      r.base[0] = wbytes(L.w[TRE_W_DQ]);
      r.base[1] = wbytes(L.w[TRE_W_DKV]);
      r.base[2] = wbytes(L.w[TRE_W_INDEX_K]);  // sparse only (rows past QL + C)
      r.split[0] = p.QL;
      r.split[1] = p.QL + p.KL + p.R;
    } else {  // sparse q up-projection: W_uq rows, then W_iq rows
      r.base[0] = wbytes(L.w[TRE_W_UQ]);
      r.base[1] = wbytes(L.w[TRE_W_INDEX_Q]);
      r.split[0] = p.Hq * (p.NP + p.R);
    }
    return r;
  }
  r.base[0] = part_row(p, t, g, 0, t.r0, &contig);
  r.base[1] = g.nseg < 2 ? nullptr : part_row(p, t, g, 1, t.r0, &contig);
  return r;
}

// Row n of segment seg of a GEMV task's K-part, from its resolved row source.
__device__ __forceinline__ const uint8_t* src_row(const RowSrc& rs, int seg, int n, int r0) {
  if (!rs.lookup) return (seg ? rs.base[1] : rs.base[0]) + (long long)(n - r0) * rs.stride;
  if (n < rs.split[0]) return rs.base[0] + (long long)n * rs.stride;
  if (n < rs.split[1]) return rs.base[1] + (long long)(n - rs.split[0]) * rs.stride;
  return rs.base[2] + (long long)(n - rs.split[1]) * rs.stride;
}

// ---- producer -------------------------------------------------------------------------------
// Bytes of stage i of task t.  GEMV stages are whole rows of the task's K-part (gate/up:
// the rows of both matrices); attention stages are the K and V rows of up to `pps`
// consecutive cached positions of one kv head.
// Tile stages of a multi-token GEMV task in order: row tile, then segment, then k-chunk.
// A cursor walks them with additions only (the producer and consumers advance it per stage).
struct TileStage {
  int n0, nr;    // rows [n0, n0 + nr), nr <= 16
  int seg;
  int c0, kw;    // columns [c0, c0 + kw) of the task's K-part, kw <= kTileK
  bool last;     // last stage of the row tile
};

__device__ __forceinline__ void tile_set(TileStage& ts, const Task& t, const GemvGeom& g) {
  ts.nr = min(kTileRows, t.r1 - ts.n0);
  ts.kw = min(kTileK, g.Kp - ts.c0);
  ts.last = ts.seg == g.nseg - 1 && ts.c0 + ts.kw == g.Kp;
}

__device__ __forceinline__ TileStage tile_first(const Task& t, const GemvGeom& g) {
  TileStage ts;
  ts.n0 = t.r0;
  ts.seg = 0;
  ts.c0 = 0;
  tile_set(ts, t, g);
  return ts;
}

__device__ __forceinline__ void tile_next(TileStage& ts, const Task& t, const GemvGeom& g) {
  ts.c0 += kTileK;
  if (ts.c0 >= g.Kp) {
    ts.c0 = 0;
    if (++ts.seg == g.nseg) {
      ts.seg = 0;
      ts.n0 += kTileRows;
    }
  }
  tile_set(ts, t, g);
}

template <bool MLA, bool SP>
__device__ __forceinline__ uint32_t stage_total(const Params& p, const Task& t, const GemvGeom& g,
                                                int t0, int t1, int i) {
  if (t.type == T_GEMV) {
    const int nr = min(g.rps, t.r1 - (t.r0 + i * g.rps));
    return (uint32_t)(g.nseg * nr * g.rowb);
  }
  if constexpr (SP) {
    if (t.type == T_INDEX) return (uint32_t)(p.DI * 2 * kIndexRows);  // whole boxes
    // sparse: every row of the stage is gathered (rows past the split repeat its first)
    if (t.type == T_MLA_ATTN && sparse_step(p)) return (uint32_t)(kMlaPosPerStage * (p.KL + p.R) * 2);
  }
  if constexpr (MLA) {
    // whole boxes (rows past the cache are zero-filled)
    if (t.type == T_MLA_ATTN) return (uint32_t)((p.KL + p.R) / kMlaBox * kMlaPosPerStage * 128);
  }
  return (uint32_t)(2 * (p.D / 64) * p.pps * 128);  // K and V boxes of pps rows
}

// Issue the bulk copies of stage i into `dst`: one copy per contiguous run of rows (per
// segment; gate rows at the stage's start, up rows after `rps` rows), spread over the
// producer lanes; attention: the K rows then the V rows (lanes 0 and 1).
template <bool MLA, bool SP>
__device__ __forceinline__ void issue_stage(const Params& p, const Task& t, const GemvGeom& g,
                                            const RowSrc& rs, int t0, int t1, int i, int lane,
                                            uint8_t* dst, uint64_t* bar, uint64_t pol) {
  if (t.type == T_GEMV) {
    const int n0 = t.r0 + i * g.rps, n1 = min(t.r1, n0 + g.rps);
    const uint32_t rowb = (uint32_t)g.rowb;
    if (g.esz == 1) {  // E4M3 rows: one copy per row, rows at the padded pitch
      const uint32_t pitch = (uint32_t)fp8_row_pitch(g.Kp);
      for (int k = lane; k < g.nseg * (n1 - n0); k += 32) {
        const int seg = k / (n1 - n0), r = k % (n1 - n0);
        bulk_g2s(dst + (size_t)(seg * g.rps + r) * pitch, src_row(rs, seg, n0 + r, t.r0), rowb,
                 bar, pol);
      }
      return;
    }
    if (!rs.lookup) {
      if (rs.stride == (long long)rowb) {  // rows adjacent in memory: one copy per segment
        if (lane < g.nseg)
          bulk_g2s(dst + (size_t)lane * g.rps * rowb, rs.base[lane] + (n0 - t.r0) * rs.stride,
                   (uint32_t)(n1 - n0) * rowb, bar, pol);
      } else {                  // strided rows (K-parts): one copy per row
        for (int k = lane; k < g.nseg * (n1 - n0); k += 32) {
          const int seg = k / (n1 - n0), r = k % (n1 - n0);
          bulk_g2s(dst + (size_t)(seg * g.rps + r) * rowb,
                   rs.base[seg] + (n0 - t.r0 + r) * rs.stride, rowb, bar, pol);
        }
      }
      return;
    }
    // QKV: each segment's rows of the stage in at most three runs
    int contig = 0;
    const uint8_t* w0 = lane < g.nseg ? part_row(p, t, g, lane, n0, &contig) : nullptr;
    if (__all_sync(0xffffffffu, lane >= g.nseg || contig >= n1 - n0)) {
      if (lane < g.nseg)
        bulk_g2s(dst + (size_t)lane * g.rps * rowb, w0, (uint32_t)(n1 - n0) * rowb, bar, pol);
      return;
    }
    int piece = 0;
    for (int seg = 0; seg < g.nseg; ++seg) {
      for (int n = n0; n < n1;) {
        int contig;
        const uint8_t* w = part_row(p, t, g, seg, n, &contig);
        const int take = min(n1 - n, contig);
        if ((piece & 31) == lane)
          bulk_g2s(dst + (size_t)(seg * g.rps + (n - n0)) * rowb, w, (uint32_t)take * rowb, bar, pol);
        ++piece;
        n += take;
      }
    }
  } else if (SP && t.type == T_INDEX) {
    // 64-column boxes of kIndexRows index keys, 128-byte swizzled
    if (lane < p.DI / 64) {
      const uint8_t* map = static_cast<const uint8_t*>(p.ix_maps) + (size_t)t.layer * 128;
      tma_load_2d(dst + (size_t)lane * kIndexRows * 128, map, lane * 64, t0 + i * kIndexRows, bar);
    }
  } else if (SP && t.type == T_MLA_ATTN && sparse_step(p)) {
    // gather: lane r copies the latent row of chosen entry t0 + 32 i + r (past the split:
    // entry t0 again, so that the masked rows hold finite values) at the padded pitch
    const int C = p.KL + p.R;
    int j = t0 + i * kMlaPosPerStage + lane;
    if (j >= t1) j = t0;
    int pos = __ldcg(p.ix_sel + (size_t)t.layer * p.KI + j);
    if (pos < 0 || pos >= p.pos) {
      record_error(p, TRE_ERR_BOUNDS, t.id);
      pos = 0;
    }
    bulk_g2s(dst + (size_t)lane * sparse_lat_pitch(C),
             reinterpret_cast<const uint8_t*>(p.layers[t.layer].k_cache) + (size_t)pos * C * 2,
             (uint32_t)C * 2u, bar, pol);
  } else if (MLA && t.type == T_MLA_ATTN) {
    // 64-column boxes of 32 latent rows, 128-byte swizzled (see mla.cuh)
    if (lane < (p.KL + p.R) / kMlaBox) {
      const uint8_t* map = static_cast<const uint8_t*>(p.kv_maps) + (size_t)t.layer * 128;
      tma_load_2d(dst + (size_t)lane * kMlaPosPerStage * 128, map, lane * kMlaBox,
                  t0 + i * kMlaPosPerStage, bar);
    }
  } else {
    // K then V: 64-column boxes of pps rows of kv head r0 (rows of the caches viewed as
    // [Hkv * capacity][D]; rows past the split are masked by the consumer)
    const int kb = p.D / 64;
    if (lane < 2 * kb) {
      const uint8_t* map = static_cast<const uint8_t*>(p.kv_maps) +
                           ((size_t)t.layer * 2 + (lane >= kb)) * 128;
      tma_load_2d(dst + (size_t)lane * p.pps * 128, map, (lane % kb) * 64,
                  t.r0 * p.cap + t0 + i * p.pps, bar);
    }
  }
}

// L2 prefetch of a whole GEMV task ahead of its stages: the contiguous byte ranges task t
// will stream (its rows of each matrix), as a few large
// requests — a bulk request costs the same fixed time whatever its size, so one request
// per range rather than one per stage.  At most `budget` bytes; K-part tasks (strided rows)
// are skipped.
__device__ __forceinline__ void task_prefetch(const Params& p, const Task& t, int lane,
                                              long long budget) {
  const uint8_t* src[3] = {nullptr, nullptr, nullptr};
  long long bytes[3] = {0, 0, 0};
  if (t.type != T_GEMV) return;  // KV tiles come through the tensor maps
  {
    const GemvGeom g = gemv_geom<false>(p, t);
    if (g.np > 1 || needs_route(p, t)) return;  // strided rows, or addresses not known yet
    const size_t rowb = (size_t)g.K * g.esz;
    if (g.nseg == 2) {
      for (int s = 0; s < 2; ++s) {
        int run;
        src[s] = part_row(p, t, g, s, t.r0, &run);
        bytes[s] = (long long)(t.r1 - t.r0) * rowb;
      }
    } else {
      int n = t.r0, left = t.r1 - t.r0;
      for (int piece = 0; left > 0 && piece < 3; ++piece) {
        int run;
        src[piece] = part_row(p, t, g, 0, n, &run);
        const int take = min(left, run);
        bytes[piece] = (long long)take * rowb;
        n += take;
        left -= take;
      }
    }
  }
  if (lane < 3 && src[lane]) {
    long long before = 0;  // budget left after the pieces of lower lanes
    for (int k = 0; k < lane; ++k) before += bytes[k];
    long long n = min(bytes[lane], budget - before);
    const uint8_t* a = src[lane];
    while (n >= 16) {
      const uint32_t chunk = (uint32_t)min(n, 1LL << 20) & ~15u;
      bulk_prefetch_l2(a, chunk);
      a += chunk;
      n -= chunk;
    }
  }
}

// The whole producer warp issues a stage: lane 0 claims the slot (waits for its "empty"
// phase) and announces the stage's byte count on the "full" barrier; each lane then copies
// its piece.  When it starts a task it first asks L2 for the next task's bytes (up to
// pf_window): weights and cached KV never depend on this step's activations, so HBM keeps
// streaming through op boundaries even while the shared-memory ring is full.
// A new op starts at task b (a different op, layer or task type than task a).
__device__ __forceinline__ bool op_boundary(const Task& a, const Task& b) {
  return a.type != b.type || a.op != b.op || a.layer != b.layer;
}

// Producer: wait (bounded) until this SM's consumers have finished task ti - 1.
__device__ __forceinline__ bool hold_for_consumers(const Params& p, const volatile int* done, int ti, int detail,
                                   int lane) {
  bool r = true;
  if (lane == 0) {
    const uint64_t w0 = globaltimer_ns();
    long long c0 = clock64();
    while (*done < ti) {
      __nanosleep(32);
      if (clock64() - c0 > kCheckCycles) {
        if (aborted(p) || (long long)(globaltimer_ns() - w0) > 2 * p.timeout_ns) {
          if (!aborted(p)) record_error(p, TRE_ERR_DEP_TIMEOUT, detail);
          r = false;
          break;
        }
        c0 = clock64();
      }
    }
  }
  return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
}

template <bool TILED, bool MLA, bool SP, bool F4 = false>
__device__ void producer(const Params& p, const Task* my, int ntask, uint8_t* ring,
                         uint64_t* full, uint64_t* empty, uint32_t* tags,
                         const volatile int* done, int lane) {
  const uint64_t pol = l2_policy_evict_first();
  const uint32_t NS = (uint32_t)p.ring_stages;
  const uint32_t SB = (uint32_t)p.stage_bytes;
  const bool no_overlap = (p.flags & TRE_DEBUG_NO_OVERLAP) != 0;
  const long long window = no_overlap ? 0 : p.pf_window;
  uint32_t gs = 0, slot = 0, ph = 0;  // stage count, its ring slot and phase parity (tiles)
  bool ok = true;
  for (int ti = 0; ti < ntask && ok; ++ti) {
    const Task t = my[ti];
    if (no_overlap) {
      bool r = true;
      if (lane == 0) r = wait_dep(p, t);
      ok = __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
      if (!ok) break;
    }
    // at an op boundary, hold the next op's tiles (all of them, or those after its first
    // hold_next_op - 1 stages) until this SM's consumers have finished (and published) the
    // previous task, so that their publish does not wait behind queued copies
    int hold_at = -1;
    if (p.hold_next_op > 0 && ti > 0 && op_boundary(my[ti - 1], t)) hold_at = p.hold_next_op - 1;
    if (hold_at == 0 && !hold_for_consumers(p, done, ti, t.id, lane)) {
      ok = false;
      break;
    }
    if (needs_route(p, t)) {  // the expert ids pick the addresses: wait for the routing
      bool r = true;
      if (lane == 0) r = wait_counter(p, t.layer * C_PER_LAYER + C_ROUTE, 1u, t.id);
      ok = __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
      if (!ok) break;
    }
    if (SP && t.type == T_MLA_ATTN && sparse_step(p)) {  // the chosen positions pick the rows
      bool r = true;
      if (lane == 0) r = wait_dep(p, t);
      ok = __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
      if (!ok) break;
      __syncwarp();  // orders the other lanes' reads of the selection after lane 0's acquire
    }
    if (window > 0 && ti + 1 < ntask) task_prefetch(p, my[ti + 1], lane, window);
    const int ns = task_nstages<TILED, F4>(p, t);
    GemvGeom g{};
    RowSrc rs{};
    int t0 = 0, t1 = 0;
    if (t.type == T_GEMV) {
      g = gemv_geom<TILED, F4>(p, t);
      rs = row_src(p, t, g);
    } else {
      attn_range(p, t, t0, t1);
      // each lane that copies through a cache's tensor map acquires the map first (the
      // allocation-free entry point rewrites its maps in place between launches)
      const uint8_t* maps = static_cast<const uint8_t*>(p.kv_maps);
      if (SP && t.type == T_INDEX) {
        if (lane < p.DI / 64)
          tensormap_acquire(static_cast<const uint8_t*>(p.ix_maps) + (size_t)t.layer * 128);
      } else if (SP && t.type == T_ISEL) {
      } else if (MLA && t.type == T_MLA_ATTN) {
        if (lane < (p.KL + p.R) / kMlaBox) tensormap_acquire(maps + (size_t)t.layer * 128);
      } else if (lane < 2 * (p.D / 64)) {
        tensormap_acquire(maps + ((size_t)t.layer * 2 + (lane >= p.D / 64)) * 128);
      }
    }
    const bool tiled = TILED && t.type == T_GEMV;
    TileStage ts{};
    if (tiled) ts = tile_first(t, g);
    for (int i = 0; i < ns; ++i, ++gs) {
      if (i > 0 && i == hold_at && !hold_for_consumers(p, done, ti, t.id, lane)) {
        ok = false;
        break;
      }
      if (!TILED) {  // whole-row kernels: from the stage count (measured faster there)
        slot = gs % NS;
        ph = (gs / NS) & 1u;
      }
      bool r = true;
      if (lane == 0) r = mbar_wait(p, &empty[slot], ph ^ 1u);
      if (__shfl_sync(0xffffffffu, r ? 1 : 0, 0) == 0) {
        ok = false;
        break;
      }
      if (lane == 0) {
        *reinterpret_cast<volatile uint32_t*>(tags + slot) = gs;
        mbar_arrive_expect_tx(&full[slot], tiled ? (uint32_t)(ts.nr * ts.kw * 2)
                                                 : stage_total<MLA, SP>(p, t, g, t0, t1, i));
      }
      __syncwarp();
      if (tiled) {
        // one copy per row of the tile: columns [c0, c0 + kw) into a padded row slot
        if (lane < ts.nr)
          bulk_g2s(ring + (size_t)slot * SB + (size_t)lane * kTilePitch,
                   src_row(rs, ts.seg, ts.n0 + lane, t.r0) + 2 * ts.c0, (uint32_t)ts.kw * 2u,
                   &full[slot], pol);
        tile_next(ts, t, g);
      } else {
        issue_stage<MLA, SP>(p, t, g, rs, t0, t1, i, lane, ring + (size_t)slot * SB, &full[slot], pol);
      }
      if (TILED) ring_next(slot, ph, NS);
    }
  }
  if (!ok && lane == 0) {
    // Abort: let the copies still in flight land before the CTA can exit.
    const uint32_t first = gs > NS ? gs - NS : 0u;
    for (uint32_t k = first; k < gs; ++k) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&full[k % NS], (k / NS) & 1u))
        if ((long long)(globaltimer_ns() - t0) > p.timeout_ns) break;
    }
  }
}

// ---- consumer helpers -----------------------------------------------------------------------
struct Best {
  float v;
  int i;
};

__device__ __forceinline__ void best_update(Best& b, float v, int i) {
  if (v > b.v || (v == b.v && i < b.i)) {
    b.v = v;
    b.i = i;
  }
}

__device__ __forceinline__ unsigned long long pack_best(const Best& b) {
  const uint32_t u = __float_as_uint(b.v);
  const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)key << 32) | (uint32_t)(0xffffffffu - (uint32_t)b.i);
}

// Token v of this step: a kernel argument, or (greedy loop) token 0 read from the device
// word the previous step's argmax wrote.  An id outside [0, V) records a bounds error and
// is clamped, so that no access leaves the embedding.
__device__ __forceinline__ int step_token(const Params& p, int v) {
  if (v > 0 || !p.token_in) return p.tokens[v];
  const int tok = __ldcg(p.token_in);
  if (tok < 0 || tok >= p.V) {
    record_error(p, TRE_ERR_BOUNDS, -4);
    return 0;
  }
  return tok;
}

// Row n of token v's residual stream entering `layer` (layer 0: the embedding row or the
// layer-only input).
__device__ __forceinline__ float resid_in(const Params& p, int layer, int n, int v = 0) {
  if (layer > 0) return __ldcg(p.x + (size_t)v * p.d + n);
  if (p.x_in) return __ldcg(p.x_in + (size_t)v * p.d + n);
  return bf_lo(p.embed[(size_t)step_token(p, v) * p.d + n]);
}

// Input-vector identity for reuse across consecutive tasks (same layer, same source,
// same K-part).  The router, shared and routed gate/up all read RMSNorm(h1).  -1: the
// input depends on the task's rows (MLA per-head ops): always staged again.
__device__ __forceinline__ int input_key(const Task& t) {
  int cls;
  switch (t.op) {
    case OP_QKV: case OP_MDQKV: cls = 0; break;
    case OP_O: case OP_MO: case OP_MOS: cls = 1; break;
    case OP_GU: case OP_ROUTER: case OP_SGU: case OP_RGU: cls = 2; break;
    case OP_DOWN: case OP_MDOWN: cls = 3; break;
    case OP_UQ: cls = 5; break;
    case OP_UK: case OP_UV: return -1;
    default: cls = 4; break;
  }
  const int part = (t.op == OP_LM || t.op == OP_ROUTER) ? 0 : (t.aux & 0xff);
  return (((int)t.layer * 8 + cls) << 8) | part;
}

// The input of a GEMV over E4M3 rows (one token) as the B operand of mma.sync m16n8k32
// E4M3.  Each input x (times its gain) becomes 4 E4M3 terms: with 2^sg the power of two
// that brings the largest |x| of its 32-column chunk into [128, 256),
// x 2^sg ~ t0 + t1 / 16 + t2 / 256 + t3 / 4096, each term the nearest E4M3 number to what
// the earlier ones left, times 16 (about 16 significand bits in all).  Fragment order:
// column c of the K-part lies in row segment q = c / Ls, 32-column chunk cc = (c % Ls) / 32,
// half h and column group t4 (c % 32 = 16 h + 4 t4 + i), and the 4 bytes of term tau for
// (q, cc, h, t4) sit at byte q 4 Ls + cc 128 + tau 32 + t4 8 + h 4 (a lane reads its term's
// two halves as one 8-byte word, a warp's 32 words two 128-byte rows).  After the 4
// segments: 2^-sg per chunk (span / 32 floats).  Columns past Kp are zero.  rn receives
// the RMSNorm scale (1 when the op has no norm).
__device__ void load_input_e4m3(const Params& p, const Task& t, const GemvGeom& gg, float* ub,
                                float* red, int ctid, float* rn) {
  const int K = gg.Kp, Ls = fp8_half_len(K), span = 2 * Ls, NG = span / 4;  // 4-column groups
  const float* src = nullptr;
  const uint16_t* src_bf = nullptr;
  const uint16_t* gain = nullptr;
  switch (t.op) {
    case OP_QKV:
      gain = p.layers[t.layer].w[TRE_W_ATTN_NORM];
      if (t.layer > 0) src = p.x;
      else if (p.x_in) src = p.x_in;
      else src_bf = p.embed + (size_t)step_token(p, 0) * p.d;
      break;
    case OP_O: src = p.attn; break;
    case OP_GU: src = p.h1; gain = p.layers[t.layer].w[TRE_W_FFN_NORM]; break;
    default: src = p.u; break;  // OP_DOWN
  }
  if (src) src += gg.k0;
  uint8_t* fr = reinterpret_cast<uint8_t*>(ub);
  float* cs = ub + span;
  float ss = 0.f;
  constexpr int B = 4;  // groups a thread fetches before it stores any
  // the loop runs from the warp's first group, so every lane of a warp takes the same number
  // of trips (the shuffles below need all 32); groups past NG only skip their stores
  const int lane = ctid & 31;
  for (int q0 = ctid - lane; q0 < NG; q0 += B * kConsumerThreads) {
    float4 xv[B];
    uint2 gv[B];
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int q = q0 + lane + u * kConsumerThreads, c = min(4 * q, K - 4);  // clamped fetch
      if (src_bf) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(src_bf + c));
        xv[u] = make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
      } else {
        xv[u] = __ldcg(reinterpret_cast<const float4*>(src + c));
      }
      if (gain) gv[u] = __ldg(reinterpret_cast<const uint2*>(gain + c));
    }
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int q = q0 + lane + u * kConsumerThreads, col = 4 * q;
      const bool live = col < K;  // (all lanes run the shuffles below)
      float e[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
      if (!live) {
        e[0] = e[1] = e[2] = e[3] = 0.f;
      } else if (gain) {
#pragma unroll
        for (int k = 0; k < 4; ++k) ss = fmaf(e[k], e[k], ss);
        e[0] *= bf_lo(gv[u].x); e[1] *= bf_hi(gv[u].x);
        e[2] *= bf_lo(gv[u].y); e[3] *= bf_hi(gv[u].y);
      }
      // the chunk's largest |x| (its 8 groups sit on 8 consecutive lanes)
      float am = fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3])));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
      int sg = 0;
      if (am > 0.f && am < INFINITY)
        sg = min(100, max(-100, 7 - (((int)(__float_as_uint(am) >> 23) & 0xff) - 127)));
      const float up = __int_as_float((127 + sg) << 23);  // 2^sg, exact
      float y[4] = {e[0] * up, e[1] * up, e[2] * up, e[3] * up};
      if (q < NG) {
        const int sgm = col / Ls, cl = col - sgm * Ls;
        uint8_t* dst = fr + sgm * 4 * Ls + (cl >> 5) * 128 + ((cl >> 2) & 3) * 8 + ((cl >> 4) & 1) * 4;
#pragma unroll
        for (int tau = 0; tau < 4; ++tau) {
          const uint32_t w01 = f2_to_e4m3x2(y[0], y[1]), w23 = f2_to_e4m3x2(y[2], y[3]);
          *reinterpret_cast<uint32_t*>(dst + tau * 32) = w01 | (w23 << 16);
          const float2 b01 = e4m3x2_to_f2(w01), b23 = e4m3x2_to_f2(w23);
          y[0] = (y[0] - b01.x) * 16.f; y[1] = (y[1] - b01.y) * 16.f;
          y[2] = (y[2] - b23.x) * 16.f; y[3] = (y[3] - b23.y) * 16.f;
        }
        if ((col & 31) == 0) cs[col >> 5] = __int_as_float((127 - sg) << 23);  // 2^-sg
      }
    }
  }
  if (gain) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((ctid & 31) == 0) red[ctid >> 5] = ss;
  }
  consumer_sync(kConsumerThreads);
  float r = 1.f;
  if (gain) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += red[w];
    r = 1.f / sqrtf(tot / (float)K + p.eps);
  }
  rn[0] = r;
}

// Stage the GEMV input of each of the MT tokens into its two planes (token v's at
// ub + v Kp); rn[v] receives token v's RMSNorm scale (1 when the op has no norm).
// FRAG (tensor-core tiles): the inputs are written as the mma B operand instead, split
// into bf16 hi and lo parts once here (one 8-column group of one token per thread, the
// tokens interleaved across lanes so that the stores spread over the banks): for k-step s (columns 16 s .. 16 s + 15) and
// fragment lane c = (part * MT + v) * 4 + tig (part 0 hi, 1 lo), the 32-bit pair at
// 2 (8 MT s + c) holds columns 16 s + 2 tig, + 1 and the one after it columns
// 16 s + 8 + 2 tig, + 1 of token v.  A warp reads a k-step's operand as 8 MT consecutive
// 8-byte words, with no bank conflicts.  Same size as the planes: MT Kp floats.
template <int MT, bool FRAG = false>
__device__ void load_input(const Params& p, const Task& t, const GemvGeom& gg, float* ub,
                           float* red, int ctid, float* rn) {
  const int K = gg.Kp;  // this K-part's slice of the input vector
  const float* src = nullptr;
  const uint16_t* src_bf = nullptr;
  const uint16_t* gain = nullptr;
  size_t vstride = 0;   // floats between consecutive tokens' vectors
  switch (t.op) {
    case OP_QKV:
    case OP_MDQKV:
      gain = p.layers[t.layer].w[TRE_W_ATTN_NORM];
      vstride = p.d;
      if (t.layer > 0) src = p.x;
      else if (p.x_in) src = p.x_in;
      else src_bf = p.embed;
      break;
    case OP_O: src = p.attn; vstride = (size_t)p.Hq * p.D; break;
    case OP_GU: case OP_ROUTER: case OP_SGU: case OP_RGU:
      src = p.h1; vstride = p.d; gain = p.layers[t.layer].w[TRE_W_FFN_NORM]; break;
    case OP_DOWN: case OP_MDOWN: src = p.u; vstride = p.F; break;
    case OP_UQ: src = p.cqkv; gain = p.layers[t.layer].w[TRE_W_Q_NORM]; break;
    case OP_UV: src = p.o_lat + (size_t)(t.r0 / p.VD) * p.KL; break;
    case OP_MO: case OP_MOS: src = p.mla_o; break;
    default: src = p.x; vstride = p.d; gain = p.final_norm; break;
  }
  if (src) src += gg.k0;        // normalised inputs are single-part (k0 = 0)
  const int K8 = K >> 3;
  float ss[MT];
#pragma unroll
  for (int v = 0; v < MT; ++v) ss[v] = 0.f;
  // Fragments: work item w is one 8-column group j of token v, the tokens interleaved
  // across lanes (so that the fragment stores spread over the banks).  Each thread fetches
  // a batch of items before it stores any, so that the global reads overlap; indices are
  // clamped, so the fetches need no guard.
  const int nitems = MT * K8;
  for (int w0 = ctid; FRAG && w0 < nitems; w0 += kLoadBatch * kConsumerThreads) {
    float4 ra[kLoadBatch], rb[kLoadBatch];
    uint4 gw[kLoadBatch];
    if (src_bf) {
#pragma unroll
      for (int u = 0; u < kLoadBatch; ++u) {
        const int w = min(w0 + u * kConsumerThreads, nitems - 1);
        const int v = w % MT, j = w / MT;
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(src_bf + (size_t)step_token(p, v) * p.d) + j);
        ra[u] = make_float4(__uint_as_float(x.x), __uint_as_float(x.y), __uint_as_float(x.z),
                            __uint_as_float(x.w));
      }
    } else {
#pragma unroll
      for (int u = 0; u < kLoadBatch; ++u) {
        const int w = min(w0 + u * kConsumerThreads, nitems - 1);
        const int v = w % MT, j = w / MT;
        const float4* sv = reinterpret_cast<const float4*>(src + v * vstride) + 2 * j;
        ra[u] = __ldcg(sv);
        rb[u] = __ldcg(sv + 1);
      }
    }
    if (gain) {
#pragma unroll
      for (int u = 0; u < kLoadBatch; ++u) {
        const int w = min(w0 + u * kConsumerThreads, nitems - 1);
        const int j = w / MT;
        gw[u] = __ldg(reinterpret_cast<const uint4*>(gain) + j);
      }
    }
#pragma unroll
    for (int u = 0; u < kLoadBatch; ++u) {
      const int w = w0 + u * kConsumerThreads;
      if (w >= nitems) break;
      const int v = w % MT, j = w / MT;
      float e[8];
      if (src_bf) {
        const uint32_t x0 = __float_as_uint(ra[u].x), x1 = __float_as_uint(ra[u].y);
        const uint32_t x2 = __float_as_uint(ra[u].z), x3 = __float_as_uint(ra[u].w);
        e[0] = bf_lo(x0); e[1] = bf_hi(x0); e[2] = bf_lo(x1); e[3] = bf_hi(x1);
        e[4] = bf_lo(x2); e[5] = bf_hi(x2); e[6] = bf_lo(x3); e[7] = bf_hi(x3);
      } else {
        e[0] = ra[u].x; e[1] = ra[u].y; e[2] = ra[u].z; e[3] = ra[u].w;
        e[4] = rb[u].x; e[5] = rb[u].y; e[6] = rb[u].z; e[7] = rb[u].w;
      }
      if (gain) {
        float s2 = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) s2 = fmaf(e[k], e[k], s2);
#pragma unroll
        for (int vv = 0; vv < MT; ++vv)
          if (vv == v) ss[vv] += s2;
        const uint4 g = gw[u];
        e[0] *= bf_lo(g.x); e[1] *= bf_hi(g.x); e[2] *= bf_lo(g.y); e[3] *= bf_hi(g.y);
        e[4] *= bf_lo(g.z); e[5] *= bf_hi(g.z); e[6] *= bf_lo(g.w); e[7] *= bf_hi(g.w);
      }
      uint32_t* fr = reinterpret_cast<uint32_t*>(ub) + 2 * (8 * MT * (j >> 1)) + (j & 1);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t hi, lo;
        split_pair(e[2 * q], e[2 * q + 1], hi, lo);
        fr[2 * (v * 4 + q)] = hi;
        fr[2 * ((MT + v) * 4 + q)] = lo;
      }
    }
  }
#pragma unroll
  for (int v = 0; v < (FRAG ? 0 : MT); ++v) {
    float* xlo = ub + (size_t)v * K;
    float* xhi = xlo + K / 2;
    const float* sv = src ? src + v * vstride : nullptr;
    const uint16_t* bv = src_bf ? src_bf + (size_t)step_token(p, v) * p.d : nullptr;
    // each thread fetches kPlaneBatch 8-column groups (and their gains) before it stores
    // any, so that the global reads overlap instead of costing one round trip per group;
    // indices are clamped, so the fetches need no guard
    constexpr int PB = MT == 1 ? kPlaneBatch : 1;  // (more tokens: registers are short)
    for (int j0 = ctid; j0 < K8; j0 += PB * kConsumerThreads) {
      float4 ra[PB], rb[PB];
      uint4 gw[PB];
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const int j = min(j0 + u * kConsumerThreads, K8 - 1);
        if (bv) {
          const uint4 w = __ldg(reinterpret_cast<const uint4*>(bv) + j);
          ra[u] = make_float4(__uint_as_float(w.x), __uint_as_float(w.y), __uint_as_float(w.z),
                              __uint_as_float(w.w));
        } else {
          ra[u] = __ldcg(reinterpret_cast<const float4*>(sv) + 2 * j);
          rb[u] = __ldcg(reinterpret_cast<const float4*>(sv) + 2 * j + 1);
        }
        if (gain) gw[u] = __ldg(reinterpret_cast<const uint4*>(gain) + j);
      }
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const int j = j0 + u * kConsumerThreads;
        if (j >= K8) break;
        float e[8];
        if (bv) {
          const uint32_t x0 = __float_as_uint(ra[u].x), x1 = __float_as_uint(ra[u].y);
          const uint32_t x2 = __float_as_uint(ra[u].z), x3 = __float_as_uint(ra[u].w);
          e[0] = bf_lo(x0); e[1] = bf_hi(x0); e[2] = bf_lo(x1); e[3] = bf_hi(x1);
          e[4] = bf_lo(x2); e[5] = bf_hi(x2); e[6] = bf_lo(x3); e[7] = bf_hi(x3);
        } else {
          e[0] = ra[u].x; e[1] = ra[u].y; e[2] = ra[u].z; e[3] = ra[u].w;
          e[4] = rb[u].x; e[5] = rb[u].y; e[6] = rb[u].z; e[7] = rb[u].w;
        }
        if (gain) {
#pragma unroll
          for (int k = 0; k < 8; ++k) ss[v] = fmaf(e[k], e[k], ss[v]);
          const uint4 g = gw[u];
          e[0] *= bf_lo(g.x); e[1] *= bf_hi(g.x); e[2] *= bf_lo(g.y); e[3] *= bf_hi(g.y);
          e[4] *= bf_lo(g.z); e[5] *= bf_hi(g.z); e[6] *= bf_lo(g.w); e[7] *= bf_hi(g.w);
        }
        reinterpret_cast<float4*>(xlo)[j] = make_float4(e[0], e[1], e[2], e[3]);
        reinterpret_cast<float4*>(xhi)[j] = make_float4(e[4], e[5], e[6], e[7]);
      }
    }
  }
  if (gain) {
#pragma unroll
    for (int v = 0; v < MT; ++v) {
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ss[v] += __shfl_xor_sync(0xffffffffu, ss[v], off);
      if ((ctid & 31) == 0) red[(ctid >> 5) * MT + v] = ss[v];
    }
  }
  consumer_sync(kConsumerThreads);
#pragma unroll
  for (int v = 0; v < MT; ++v) {
    float r = 1.f;
    if (gain) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) tot += red[w * MT + v];
      r = 1.f / sqrtf(tot / (float)K + p.eps);
    }
    rn[v] = r;
  }
}

// ---- attention task ----------------------------------------------------------------------------
__device__ __forceinline__ void rope_cs(const Params& p, int i, float& c, float& s,
                                        const double* inv_freq = nullptr, int dpos = 0) {
  const double ang = (double)(p.pos + dpos) * (inv_freq ? inv_freq : p.rope_inv_freq)[i];
  const double two_pi = 6.283185307179586476925286766559;
  const double red = ang - two_pi * rint(ang / two_pi);
  sincosf((float)red, &s, &c);
}

// One split of the split-KV decode attention for kv head g = t.r0 (split t.r1 of t.aux):
// the G query heads of the group attend to cached positions [t0, t1) streamed through the
// ring; the last split also takes the new position pos from this step's k / v, appends
// them to the caches and merges its partial.  Every split writes its partial (m, l, O) and
// takes an arrival ticket; the last split of the group to arrive combines all splits —
// the fused combine — and publishes the group.
template <int G, int D, int MT>
__device__ void attn_task(const Params& p, const Task& t, uint32_t gs, int ns, uint8_t* ring,
                          uint64_t* full, uint64_t* empty, const uint32_t* tags, float* ub,
                          int* flag, int warp, int lane, int ctid, bool& abort_out) {
  // query rows r = v G + h: token v (position pos + v) of head g G + h
  constexpr int ROWS = MT * G;
  constexpr bool PACK = ROWS <= 8;  // hi / lo packed into rows r and r + 8 of one tile
  const int g = t.r0, split = t.r1, S = t.aux;
  const bool last = (split == S - 1);
  const int qkv_n = (p.Hq + 2 * p.Hkv) * D;
  float* q_s = ub;                            // [ROWS][D] roped, scaled
  float* kn_s = q_s + ROWS * D;               // [MT][D] new k (bf16 values)
  float* vn_s = kn_s + MT * D;                // [MT][D] new v (bf16 values)
  float* mw = vn_s + MT * D;                  // [warps][ROWS]
  float* lw = mw + kConsumerWarps * ROWS;     // [warps][ROWS]
  float* ow = lw + kConsumerWarps * ROWS;     // [warps][ROWS][D]
  float* sn = ow + kConsumerWarps * ROWS * D; // [ROWS][MT] scores of the new positions
  const float qscale = 1.4426950408889634f / sqrtf((float)D);

  for (int idx = ctid; idx < ROWS * (D / 2); idx += kConsumerThreads) {
    const int r = idx / (D / 2), i = idx % (D / 2), v = r / G, h = r % G;
    const float* qsrc = p.qkv + (size_t)v * qkv_n + (size_t)(g * G + h) * D;
    const float x0 = __ldcg(qsrc + i), x1 = __ldcg(qsrc + i + D / 2);
    float c, s;
    rope_cs(p, i, c, s, nullptr, v);
    q_s[r * D + i] = (x0 * c - x1 * s) * qscale;
    q_s[r * D + i + D / 2] = (x0 * s + x1 * c) * qscale;
  }
  if (last) {  // this step's MT keys and values: RoPE, round to bf16, append at pos + v
    const LayerPtrs& L = p.layers[t.layer];
    for (int idx = ctid; idx < MT * (D / 2); idx += kConsumerThreads) {
      const int v = idx / (D / 2), i = idx % (D / 2);
      const float* ksrc = p.qkv + (size_t)v * qkv_n + (size_t)p.Hq * D + (size_t)g * D;
      __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(L.k_cache) +
                          ((size_t)g * p.cap + p.pos + v) * D;
      const float x0 = __ldcg(ksrc + i), x1 = __ldcg(ksrc + i + D / 2);
      float c, s;
      rope_cs(p, i, c, s, nullptr, v);
      const __nv_bfloat16 k0 = __float2bfloat16_rn(x0 * c - x1 * s);
      const __nv_bfloat16 k1 = __float2bfloat16_rn(x0 * s + x1 * c);
      kc[i] = k0;
      kc[i + D / 2] = k1;
      kn_s[v * D + i] = __bfloat162float(k0);
      kn_s[v * D + i + D / 2] = __bfloat162float(k1);
    }
    for (int idx = ctid; idx < MT * D; idx += kConsumerThreads) {
      const int v = idx / D, i = idx % D;
      const float* vsrc = p.qkv + (size_t)v * qkv_n + (size_t)(p.Hq + p.Hkv) * D + (size_t)g * D;
      __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(L.v_cache) +
                          ((size_t)g * p.cap + p.pos + v) * D;
      const __nv_bfloat16 val = __float2bfloat16_rn(__ldcg(vsrc + i));
      vc[i] = val;
      vn_s[v * D + i] = __bfloat162float(val);
    }
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 4] = (long long)globaltimer_ns();

  if (last) {  // scores of the new positions; token v sees new positions j <= v
    for (int idx = warp; idx < ROWS * MT; idx += kConsumerWarps) {
      const int r = idx / MT, j = idx % MT;
      float a = 0.f;
      for (int i = lane; i < D; i += 32) a = fmaf(q_s[r * D + i], kn_s[j * D + i], a);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0) sn[idx] = j <= r / G ? a : -INFINITY;
    }
  }

  // ---- tensor-core flash-decode over the split's cached positions
  // The query rows form one 16-row A tile.  With ROWS <= 8 each row's bf16 hi part sits in
  // row r and its lo part in row r + 8, so one mma.sync computes both and the thread adds
  // its two accumulator rows (c0 + c2, c1 + c3); with more rows the hi and lo tiles are
  // separate and every tile takes two mma.  A stage holds 64 positions of K then V as
  // 64-column swizzled boxes; the 8 warps form two groups taking alternate stages, and warp
  // (group, quarter) owns positions 16 quarter .. 16 quarter + 15 of its stages with its own
  // running (m, l, O) per row.  P goes from the score registers straight into the A operand
  // of O += P V (the m16n8 accumulator layout of two n-tiles is the m16k16 A layout).
  // Positions past the split are masked (score -inf, value rows zeroed).
  constexpr int KS = D / 16, NT = D / 8, KB = D / 64;  // k-steps, output n-tiles, boxes
  constexpr int NST = PACK ? 1 : 2;                     // running states per thread
  const int g8 = lane >> 2, t4 = lane & 3;
  const bool real0 = g8 < ROWS, real1 = !PACK && g8 + 8 < ROWS;
  uint32_t qh[KS][4], ql[PACK ? 1 : KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int k0 = ks * 16 + 2 * t4;
    const float* q0 = q_s + (real0 ? g8 : 0) * D;
    const float* q1 = q_s + (real1 ? g8 + 8 : 0) * D;
    if constexpr (PACK) {
      split_pair(real0 ? q0[k0] : 0.f, real0 ? q0[k0 + 1] : 0.f, qh[ks][0], qh[ks][1]);
      split_pair(real0 ? q0[k0 + 8] : 0.f, real0 ? q0[k0 + 9] : 0.f, qh[ks][2], qh[ks][3]);
    } else {
      split_pair(real0 ? q0[k0] : 0.f, real0 ? q0[k0 + 1] : 0.f, qh[ks][0], ql[ks][0]);
      split_pair(real1 ? q1[k0] : 0.f, real1 ? q1[k0 + 1] : 0.f, qh[ks][1], ql[ks][1]);
      split_pair(real0 ? q0[k0 + 8] : 0.f, real0 ? q0[k0 + 9] : 0.f, qh[ks][2], ql[ks][2]);
      split_pair(real1 ? q1[k0 + 8] : 0.f, real1 ? q1[k0 + 9] : 0.f, qh[ks][3], ql[ks][3]);
    }
  }
  float mrow[NST], lrow[NST];
#pragma unroll
  for (int k = 0; k < NST; ++k) {
    mrow[k] = -INFINITY;
    lrow[k] = 0.f;
  }
  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  const uint32_t NS = (uint32_t)p.ring_stages;
  int t0, t1;
  attn_range(p, t, t0, t1);
  const int grp = warp >> 2, r0 = (warp & 3) * 16;
  long long waited = 0;  // trace: ns thread 0 spent waiting for its stages to land
  for (int i = grp; i < ns; i += 2) {
    const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
    const long long w0 = (p.trace && ctid == 0) ? (long long)globaltimer_ns() : 0;
    if (!stage_wait(p, full, tags, sidx)) {
      abort_out = true;
      break;
    }
    if (p.trace && ctid == 0) waited += (long long)globaltimer_ns() - w0;
    const int valid = min(16, t1 - (t0 + i * p.pps) - r0);
    if (valid > 0) {
      const uint32_t tb = smem_u32(ring + (size_t)slot * p.stage_bytes);
      const int m = lane >> 3;
      float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int r = r0 + (m >> 1) * 8 + (lane & 7), ch = ks * 2 + (m & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tb + swz_off(ch >> 3, r, ch & 7, 64), b0, b1, b2, b3);
        mma_bf16(c[0], qh[ks], b0, b1);
        mma_bf16(c[1], qh[ks], b2, b3);
        if constexpr (!PACK) {
          mma_bf16(c[0], ql[ks], b0, b1);
          mma_bf16(c[1], ql[ks], b2, b3);
        }
      }
      // scores per state (row g8; unpacked: also row g8 + 8); mask positions past the split
      float sc[NST][2][2];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const bool in = n * 8 + 2 * t4 + j < valid;
          if constexpr (PACK) {
            sc[0][n][j] = in ? c[n][j] + c[n][j + 2] : -INFINITY;
          } else {
            sc[0][n][j] = in ? c[n][j] : -INFINITY;
            sc[NST - 1][n][j] = in ? c[n][j + 2] : -INFINITY;
          }
        }
      float alpha[NST], pv[NST][2][2];
#pragma unroll
      for (int k = 0; k < NST; ++k) {
        float mx = fmaxf(fmaxf(sc[k][0][0], sc[k][0][1]), fmaxf(sc[k][1][0], sc[k][1][1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(mrow[k], mx);   // finite: valid > 0
        alpha[k] = exp2f(mrow[k] - mn);        // 0 while the row had no position yet
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int j = 0; j < 2; ++j) pv[k][n][j] = exp2f(sc[k][n][j] - mn);
        lrow[k] = lrow[k] * alpha[k] + (pv[k][0][0] + pv[k][0][1] + pv[k][1][0] + pv[k][1][1]);
        mrow[k] = mn;
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[NST - 1];
        o[n][3] *= alpha[NST - 1];
      }
      uint32_t ph[4], pl[4];
      if constexpr (PACK) {
        split_pair(pv[0][0][0], pv[0][0][1], ph[0], ph[1]);
        split_pair(pv[0][1][0], pv[0][1][1], ph[2], ph[3]);
      } else {
        split_pair(pv[0][0][0], pv[0][0][1], ph[0], pl[0]);
        split_pair(pv[1][0][0], pv[1][0][1], ph[1], pl[1]);
        split_pair(pv[0][1][0], pv[0][1][1], ph[2], pl[2]);
        split_pair(pv[1][1][0], pv[1][1][1], ph[3], pl[3]);
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        const int r = r0 + (m & 1) * 8 + (lane & 7), ch = np * 2 + (m >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(tb + swz_off(KB + (ch >> 3), r, ch & 7, 64), b0, b1, b2, b3);
        if (valid < 16) {  // value rows past the split may hold anything: zero them
          const int pa0 = 2 * t4, pb0 = 8 + 2 * t4;
          if (pa0 >= valid) { b0 &= 0xffff0000u; b2 &= 0xffff0000u; }
          if (pa0 + 1 >= valid) { b0 &= 0x0000ffffu; b2 &= 0x0000ffffu; }
          if (pb0 >= valid) { b1 &= 0xffff0000u; b3 &= 0xffff0000u; }
          if (pb0 + 1 >= valid) { b1 &= 0x0000ffffu; b3 &= 0x0000ffffu; }
        }
        mma_bf16(o[2 * np], ph, b0, b1);
        mma_bf16(o[2 * np + 1], ph, b2, b3);
        if constexpr (!PACK) {
          mma_bf16(o[2 * np], pl, b0, b1);
          mma_bf16(o[2 * np + 1], pl, b2, b3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_n(&empty[slot], 2u);  // 4 warps per stage, 8 arrivals
  }
#pragma unroll
  for (int k = 0; k < NST; ++k) {
    lrow[k] += __shfl_xor_sync(0xffffffffu, lrow[k], 1);
    lrow[k] += __shfl_xor_sync(0xffffffffu, lrow[k], 2);
  }
  if (real0) {
    if (t4 == 0) {
      mw[warp * ROWS + g8] = mrow[0];
      lw[warp * ROWS + g8] = lrow[0];
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float* d0 = ow + (warp * ROWS + g8) * D + n * 8 + 2 * t4;
      if constexpr (PACK) {  // hi rows + lo rows
        d0[0] = o[n][0] + o[n][2];
        d0[1] = o[n][1] + o[n][3];
      } else {
        d0[0] = o[n][0];
        d0[1] = o[n][1];
      }
    }
  }
  if (real1) {
    if (t4 == 0) {
      mw[warp * ROWS + g8 + 8] = mrow[NST - 1];
      lw[warp * ROWS + g8 + 8] = lrow[NST - 1];
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float* d1 = ow + (warp * ROWS + g8 + 8) * D + n * 8 + 2 * t4;
      d1[0] = o[n][2];
      d1[1] = o[n][3];
    }
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) {
    p.trace[(size_t)t.id * kTraceCols + 5] = (long long)globaltimer_ns();
    p.trace[(size_t)t.id * kTraceCols + 7] = waited;
  }

  // merge the warps (and, in the last split, the new positions) into this split's partial
  const size_t pstride = (size_t)gqa_pstride(D);
  for (int idx = ctid; idx < ROWS * D; idx += kConsumerThreads) {
    const int r = idx / D, dd = idx % D, v = r / G, h = r % G;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mw[w * ROWS + r]);
    if (last)
#pragma unroll
      for (int j = 0; j < MT; ++j) M = fmaxf(M, sn[r * MT + j]);
    float O = 0.f, Ls = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mv = mw[w * ROWS + r];
        if (mv != -INFINITY) {
          const float sc = exp2f(mv - M);
          O = fmaf(sc, ow[(w * ROWS + r) * D + dd], O);
          Ls = fmaf(sc, lw[w * ROWS + r], Ls);
        }
      }
      if (last)
#pragma unroll
        for (int j = 0; j < MT; ++j) {
          const float pn = exp2f(sn[r * MT + j] - M);   // 0 for positions after token v
          O = fmaf(pn, vn_s[j * D + dd], O);
          Ls += pn;
        }
    }
    float* dst = p.part + ((size_t)(v * p.Hq + g * G + h) * S + split) * pstride;
    dst[dd] = O;
    if (dd == 0) {
      dst[D] = M;
      dst[D + 1] = Ls;
    }
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0) {
    const uint32_t old = ticket_add(p.tickets + g, 1u);
    *flag = ((old + 1u) % (uint32_t)S) == 0u;
    if (p.trace) p.trace[(size_t)t.id * kTraceCols + 6] = (long long)globaltimer_ns();
  }
  consumer_sync(kConsumerThreads);
  if (!*flag) return;
  // The last split of this kv head to finish combines all splits (the fused combine):
  // attn = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s (splits that saw no
  // position have m_s = -inf and weigh 0).  Two threads share each group of 4 output
  // columns and take alternate splits; each fetches its splits' (m, l) and 4 O values
  // before it sums them (one round trip for up to 18 splits), the pair merges with
  // shuffles.
  constexpr int CH = 9;      // splits a thread fetches at once
  const int sub = ctid & 1;
  constexpr int NIT = ROWS * D / 4;
  for (int it0 = 0; it0 < NIT; it0 += kConsumerThreads / 2) {
    const int it = it0 + (ctid >> 1);
    const bool act = it < NIT;
    const int r = act ? it / (D / 4) : 0, dd = act ? (it % (D / 4)) * 4 : 0;
    const int v = r / G, h = r % G;
    const size_t q = (size_t)v * p.Hq + g * G + h;
    const float* base = p.part + q * S * pstride;
    float M = -INFINITY, L = 0.f, O0 = 0.f, O1 = 0.f, O2 = 0.f, O3 = 0.f;
    for (int s0 = sub; act && s0 < S; s0 += 2 * CH) {
      float2 ml[CH];
      float4 ov[CH];
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int sp = s0 + 2 * u;
        if (sp < S) {
          ml[u] = __ldcg(reinterpret_cast<const float2*>(base + (size_t)sp * pstride + D));
          ov[u] = __ldcg(reinterpret_cast<const float4*>(base + (size_t)sp * pstride + dd));
        } else {
          ml[u] = make_float2(-INFINITY, 0.f);
          ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float Mn = M;
#pragma unroll
      for (int u = 0; u < CH; ++u) Mn = fmaxf(Mn, ml[u].x);
      if (Mn == -INFINITY) continue;
      const float a = M == -INFINITY ? 0.f : exp2f(M - Mn);
      L *= a; O0 *= a; O1 *= a; O2 *= a; O3 *= a;
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const float w = ml[u].x == -INFINITY ? 0.f : exp2f(ml[u].x - Mn);
        L = fmaf(w, ml[u].y, L);
        O0 = fmaf(w, ov[u].x, O0); O1 = fmaf(w, ov[u].y, O1);
        O2 = fmaf(w, ov[u].z, O2); O3 = fmaf(w, ov[u].w, O3);
      }
      M = Mn;
    }
    const float Mo = __shfl_xor_sync(0xffffffffu, M, 1), Lo = __shfl_xor_sync(0xffffffffu, L, 1);
    const float P0 = __shfl_xor_sync(0xffffffffu, O0, 1), P1 = __shfl_xor_sync(0xffffffffu, O1, 1);
    const float P2 = __shfl_xor_sync(0xffffffffu, O2, 1), P3 = __shfl_xor_sync(0xffffffffu, O3, 1);
    if (act && sub == 0) {  // the last split holds the new position: M is finite
      const float Mm = fmaxf(M, Mo);
      const float a0 = M == -INFINITY ? 0.f : exp2f(M - Mm);
      const float a1 = Mo == -INFINITY ? 0.f : exp2f(Mo - Mm);
      const float inv = 1.f / fmaf(L, a0, Lo * a1);
      *reinterpret_cast<float4*>(p.attn + q * D + dd) =
          make_float4(fmaf(O0, a0, P0 * a1) * inv, fmaf(O1, a0, P1 * a1) * inv,
                      fmaf(O2, a0, P2 * a1) * inv, fmaf(O3, a0, P3 * a1) * inv);
    }
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0) publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);
}

template <int MT>
__device__ __forceinline__ void run_attn(const Params& p, const Task& t, uint32_t gs, int ns,
                                         uint8_t* ring, uint64_t* full, uint64_t* empty,
                                         const uint32_t* tags, float* ub, int* flag, int warp,
                                         int lane, int ctid, bool& ab) {
  const int G = p.Hq / p.Hkv;
#define TRE_ATTN(GG, DD) \
  attn_task<GG, DD, MT>(p, t, gs, ns, ring, full, empty, tags, ub, flag, warp, lane, ctid, ab)
  if (p.D == 128) {
    switch (G) {
      case 1: TRE_ATTN(1, 128); break;
      case 2: TRE_ATTN(2, 128); break;
      case 4: if constexpr (MT <= 4) TRE_ATTN(4, 128); break;
      default: if constexpr (MT <= 2) TRE_ATTN(8, 128); break;
    }
  } else {
    switch (G) {
      case 1: TRE_ATTN(1, 64); break;
      case 2: TRE_ATTN(2, 64); break;
      case 4: if constexpr (MT <= 4) TRE_ATTN(4, 64); break;
      default: if constexpr (MT <= 2) TRE_ATTN(8, 64); break;
    }
  }
#undef TRE_ATTN
}

// ---- absorbed MLA: per-head W_uk contraction ----------------------------------------------------
// Task = one head h: rows [h NP, (h + 1) NP) of W_uk ([H NP][KL]) stream through the ring,
// and q_lat[c] = sum_i q_nope[i] W_uk[h NP + i][c] accumulates per warp (lane owns columns
// 8 lane .. 8 lane + 7 of every 256-column block); the warps' sums are added in warp order.
// The task also writes RoPE(q_pe) after q_lat, and head 0 appends this token's latent row
// [RMSNorm(c_kv; kv_norm) | RoPE(k_pe)] (bf16) to the cache and keeps its values for the
// attention's new position.
__device__ void uk_task(const Params& p, const Task& t, const GemvGeom& g, uint32_t gs, int ns,
                        uint8_t* ring, uint64_t* full, uint64_t* empty, const uint32_t* tags,
                        float* ub, float* red1, int warp, int lane, int ctid, bool& ab) {
  const int h = t.r0 / p.NP, KL = p.KL, C = KL + p.R;
  float* qn = ub;                                  // [NP] q_nope of this head
  float* red = ub + ((p.NP + 63) / 64) * 64;       // [8][KL] per-warp sums
  const float* qh = p.qkv + (size_t)h * (p.NP + p.R);
  for (int i = ctid; i < p.NP; i += kConsumerThreads) qn[i] = __ldcg(qh + i);
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 4] = (long long)globaltimer_ns();
  const uint32_t NS = (uint32_t)p.ring_stages;
  const int nblk = KL / 256 + ((KL % 256) ? 1 : 0);   // 256-column blocks (lane: 8 columns each)
  float acc[3][8];
#pragma unroll
  for (int b = 0; b < 3; ++b)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[b][k] = 0.f;
  const int first = (int)((warp - (int)(gs % kConsumerWarps) + kConsumerWarps) % kConsumerWarps);
  for (int i = first; i < ns; i += kConsumerWarps) {
    const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
    if (!stage_wait(p, full, tags, sidx)) {
      ab = true;
      break;
    }
    const int n0 = t.r0 + i * g.rps, nr = min(g.rps, t.r1 - n0);
    const uint8_t* sp = ring + (size_t)slot * p.stage_bytes;
    for (int r = 0; r < nr; ++r) {
      const float qv = qn[n0 - t.r0 + r];
      const uint8_t* row = sp + (size_t)r * KL * 2;
#pragma unroll
      for (int b = 0; b < 3; ++b) {
        const int c0 = b * 256 + lane * 8;
        if (b < nblk && c0 < KL) {
          const uint4 w = *reinterpret_cast<const uint4*>(row + (size_t)c0 * 2);
          acc[b][0] = fmaf(qv, bf_lo(w.x), acc[b][0]);
          acc[b][1] = fmaf(qv, bf_hi(w.x), acc[b][1]);
          acc[b][2] = fmaf(qv, bf_lo(w.y), acc[b][2]);
          acc[b][3] = fmaf(qv, bf_hi(w.y), acc[b][3]);
          acc[b][4] = fmaf(qv, bf_lo(w.z), acc[b][4]);
          acc[b][5] = fmaf(qv, bf_hi(w.z), acc[b][5]);
          acc[b][6] = fmaf(qv, bf_lo(w.w), acc[b][6]);
          acc[b][7] = fmaf(qv, bf_hi(w.w), acc[b][7]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_n(&empty[slot], kConsumerWarps);
  }
#pragma unroll
  for (int b = 0; b < 3; ++b) {
    const int c0 = b * 256 + lane * 8;
    if (b < nblk && c0 < KL)
#pragma unroll
      for (int k = 0; k < 8; ++k) red[warp * KL + c0 + k] = acc[b][k];
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 5] = (long long)globaltimer_ns();
  float* qf = p.qf + (size_t)h * C;
  for (int c = ctid; c < KL; c += kConsumerThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) v += red[w * KL + c];
    qf[c] = v;
  }
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 7] = (long long)globaltimer_ns();
  const int R2 = p.R / 2;
  for (int i = ctid; i < R2; i += kConsumerThreads) {
    const float x0 = __ldcg(qh + p.NP + i), x1 = __ldcg(qh + p.NP + i + R2);
    float cs, sn;
    rope_cs(p, i, cs, sn, p.rope_inv_freq_r);
    qf[KL + i] = x0 * cs - x1 * sn;
    qf[KL + i + R2] = x0 * sn + x1 * cs;
  }
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 6] = (long long)globaltimer_ns();
  if (h == 0) {  // this token's latent row
    const float* kv = p.cqkv + p.QL;
    const uint16_t* gain = p.layers[t.layer].w[TRE_W_KV_NORM];
    float ss = 0.f;
    for (int c = ctid; c < KL; c += kConsumerThreads) ss = fmaf(__ldcg(kv + c), __ldcg(kv + c), ss);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) red1[warp] = ss;
    consumer_sync(kConsumerThreads);
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += red1[w];
    const float rn = 1.f / sqrtf(tot / (float)KL + p.eps);
    __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(p.layers[t.layer].k_cache) + (size_t)p.pos * C;
    for (int c = ctid; c < KL; c += kConsumerThreads) {
      const __nv_bfloat16 v = __float2bfloat16_rn(__ldcg(kv + c) * rn * bf_lo(gain[c]));
      row[c] = v;
      p.lat_new[c] = __bfloat162float(v);
    }
    for (int i = ctid; i < R2; i += kConsumerThreads) {
      const float x0 = __ldcg(kv + KL + i), x1 = __ldcg(kv + KL + i + R2);
      float cs, sn;
      rope_cs(p, i, cs, sn, p.rope_inv_freq_r);
      const __nv_bfloat16 a = __float2bfloat16_rn(x0 * cs - x1 * sn);
      const __nv_bfloat16 b = __float2bfloat16_rn(x0 * sn + x1 * cs);
      row[KL + i] = a;
      row[KL + i + R2] = b;
      p.lat_new[KL + i] = __bfloat162float(a);
      p.lat_new[KL + i + R2] = __bfloat162float(b);
    }
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0) publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);
}

// ---- absorbed MLA: latent attention on tensor cores ---------------------------------------------
// Task = (head group hg of 16 heads, split s of the cached positions [0, pos)); the last
// split also takes the new position from lat_new.  Per 32-row latent stage:
//   scores: warp w multiplies the group's queries (A, hi + lo, held in registers for the
//           warp's k-steps of the KL + R columns) by the stage's rows (B, ldmatrix from the
//           swizzled tile); the 8 warps' partial scores are summed through shared memory;
//   softmax: thread (head, 2 positions) scales to log2 units, masks rows past the split,
//           updates the head's running max / sum and writes P as bf16 hi + lo;
//   values: warp w accumulates O[16][KL / 8 columns] += P (hi + lo) x rows (ldmatrix.trans).
// The split's (m, l, O) go to the partial buffer and the split publishes; each head's
// W_uv task merges the head's splits while it stages its input (mla_combine_input).
__device__ void mla_attn_task(const Params& p, const Task& t, uint32_t gs, int ns, uint8_t* ring,
                              uint64_t* full, uint64_t* empty, const uint32_t* tags, float* ub,
                              int warp, int lane, int ctid, bool& ab) {
  constexpr int HG = kMlaHeadGroup, PS = kMlaPosPerStage, RP = 36;  // score row pitch (floats)
  const int KL = p.KL, C = KL + p.R, hg = t.r0, split = t.r1, S = t.aux;
  // sparse step: the stage rows are the chosen positions' latent rows at a padded pitch,
  // and the new position joins only when the indexer chose it
  const bool sp = sparse_step(p);
  const uint32_t LP = (uint32_t)sparse_lat_pitch(C);
  const bool last = (split == S - 1) && (!sp || __ldcg(index_meta(p, t.layer) + IM_HASPOS) != 0u);
  auto row_off = [&](int r, int ch) { return sp ? (uint32_t)r * LP + (uint32_t)ch * 16u : lat_off(r, ch); };
  float* red = ub;                                        // [8][16][RP] partial scores
  __nv_bfloat16* phi = reinterpret_cast<__nv_bfloat16*>(ub + kConsumerWarps * HG * RP);  // [16][40]
  __nv_bfloat16* plo = phi + HG * 40;                                                    // [16][40]
  float* mst = reinterpret_cast<float*>(plo + HG * 40);   // [16] running max (log2 units)
  float* lst = mst + HG;                                  // [16] running sum
  float* alp = lst + HG;                                  // [16] rescale of this stage
  float* snw = alp + HG;                                  // [16] score of the new position
  const float scale = 1.4426950408889634f / sqrtf((float)(p.NP + p.R));
  const int g8 = lane >> 2, t4 = lane & 3;

  // this warp's k-steps of the score product, and its query fragments (hi, lo)
  const int KS = C / 16, kb = KS / kConsumerWarps, kr = KS % kConsumerWarps;
  const int k_begin = warp * kb + min(warp, kr), k_count = kb + (warp < kr ? 1 : 0);
  uint32_t ahi[kMlaMaxKSteps][4], alo[kMlaMaxKSteps][4];
  const float* q0 = p.qf + (size_t)(hg * HG + g8) * C;
  const float* q8 = q0 + (size_t)8 * C;
#pragma unroll
  for (int j = 0; j < kMlaMaxKSteps; ++j) {
    if (j < k_count) {
      const int k0 = (k_begin + j) * 16 + 2 * t4;
      split_pair(__ldcg(q0 + k0), __ldcg(q0 + k0 + 1), ahi[j][0], alo[j][0]);
      split_pair(__ldcg(q8 + k0), __ldcg(q8 + k0 + 1), ahi[j][1], alo[j][1]);
      split_pair(__ldcg(q0 + k0 + 8), __ldcg(q0 + k0 + 9), ahi[j][2], alo[j][2]);
      split_pair(__ldcg(q8 + k0 + 8), __ldcg(q8 + k0 + 9), ahi[j][3], alo[j][3]);
    }
  }
  if (ctid < HG) {
    mst[ctid] = -INFINITY;
    lst[ctid] = 0.f;
  }
  // output accumulators: this warp's KL / 8 columns = KL / 64 n-tiles of 8
  const int ncol = KL / kConsumerWarps, nt_count = ncol / 8, col0 = warp * ncol;
  float o[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int k = 0; k < 4; ++k) o[n][k] = 0.f;
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 4] = (long long)globaltimer_ns();

  int t0, t1;
  attn_range(p, t, t0, t1);
  const uint32_t NS = (uint32_t)p.ring_stages;
  long long waited = 0;  // trace: ns warp 0 spent waiting for stages to land
  for (int i = 0; i < ns; ++i) {
    const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
    const long long w0 = p.trace ? (long long)globaltimer_ns() : 0;
    const bool landed = stage_wait(p, full, tags, sidx);
    if (p.trace) waited += (long long)globaltimer_ns() - w0;
    const uint8_t* tile = ring + (size_t)slot * p.stage_bytes;
    const uint32_t tb = smem_u32(tile);
    // ---- partial scores over this warp's k-steps, 4 n-tiles of 8 rows
    float c[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int k = 0; k < 4; ++k) c[n][k] = 0.f;
#pragma unroll
    for (int j = 0; j < kMlaMaxKSteps; ++j) {
      if (landed && j < k_count) {
        const int ch = (k_begin + j) * 2;  // 16-byte chunk of the step's first 8 columns
#pragma unroll
        for (int np = 0; np < 2; ++np) {   // n-tile pairs (rows 16 np .. 16 np + 15)
          const int m = lane >> 3, r = np * 16 + (m >> 1) * 8 + (lane & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(tb + row_off(r, ch + (m & 1)), b0, b1, b2, b3);
          mma_bf16(c[2 * np], ahi[j], b0, b1);
          mma_bf16(c[2 * np], alo[j], b0, b1);
          mma_bf16(c[2 * np + 1], ahi[j], b2, b3);
          mma_bf16(c[2 * np + 1], alo[j], b2, b3);
        }
      }
    }
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      float* r0 = red + (warp * HG + g8) * RP + n * 8 + 2 * t4;
      r0[0] = c[n][0];
      r0[1] = c[n][1];
      r0[8 * RP] = c[n][2];
      r0[8 * RP + 1] = c[n][3];
    }
    // every warp takes part in every stage: the barrier also agrees on an abort
    if (consumer_sync_or(!landed, kConsumerThreads)) {
      ab = true;
      break;
    }
    // ---- softmax: thread = (head hh, rows pp, pp + 1)
    {
      const int hh = ctid >> 4, pp = (ctid & 15) * 2;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        s0 += red[(w * HG + hh) * RP + pp];
        s1 += red[(w * HG + hh) * RP + pp + 1];
      }
      const int tt = t0 + i * PS + pp;
      s0 = tt < t1 ? s0 * scale : -INFINITY;
      s1 = tt + 1 < t1 ? s1 * scale : -INFINITY;
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = mst[hh], m_new = fmaxf(m_old, mx);
      float p0 = 0.f, p1 = 0.f, a = 1.f;
      if (m_new != -INFINITY) {
        p0 = exp2f(s0 - m_new);
        p1 = exp2f(s1 - m_new);
        a = exp2f(m_old - m_new);
      }
      float ps = p0 + p1;
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      uint32_t hi, lo;
      split_pair(p0, p1, hi, lo);
      *reinterpret_cast<uint32_t*>(phi + hh * 40 + pp) = hi;
      *reinterpret_cast<uint32_t*>(plo + hh * 40 + pp) = lo;
      __syncwarp();
      if ((ctid & 15) == 0) {
        mst[hh] = m_new;
        lst[hh] = lst[hh] * a + ps;
        alp[hh] = a;
      }
    }
    consumer_sync(kConsumerThreads);
    // ---- O += P x rows, this warp's columns
    {
      const float a0 = alp[g8], a8 = alp[g8 + 8];
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        o[n][0] *= a0;
        o[n][1] *= a0;
        o[n][2] *= a8;
        o[n][3] *= a8;
      }
      const uint32_t ph = smem_u32(phi), pl = smem_u32(plo);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {   // rows 16 ks .. 16 ks + 15
        const int m = lane >> 3;
        const uint32_t aoff = (uint32_t)(((m & 1) * 8 + (lane & 7)) * 80 + (ks * 2 + (m >> 1)) * 16);
        uint32_t ah[4], al[4];
        ldsm_x4(ph + aoff, ah[0], ah[1], ah[2], ah[3]);
        ldsm_x4(pl + aoff, al[0], al[1], al[2], al[3]);
#pragma unroll
        for (int n = 0; n < 8; n += 2) {
          if (n < nt_count) {
            const int r = ks * 16 + (m & 1) * 8 + (lane & 7);
            const int ch = (col0 + n * 8) / 8 + (m >> 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(tb + row_off(r, ch), b0, b1, b2, b3);
            mma_bf16(o[n], ah, b0, b1);
            mma_bf16(o[n], al, b0, b1);
            mma_bf16(o[n + 1], ah, b2, b3);
            mma_bf16(o[n + 1], al, b2, b3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_n(&empty[slot], 1u);
  }
  if (ab) return;
  if (ctid == 0 && p.trace) {
    p.trace[(size_t)t.id * kTraceCols + 5] = (long long)globaltimer_ns();
    p.trace[(size_t)t.id * kTraceCols + 7] = waited;
  }

  // ---- the new position (last split): score from lat_new, merged into (m, l, O)
  if (last) {
    for (int hh = warp * 2; hh < warp * 2 + 2; ++hh) {
      const float* q = p.qf + (size_t)(hg * HG + hh) * C;
      float a = 0.f;
      for (int k = lane; k < C; k += 32) a = fmaf(__ldcg(q + k), __ldcg(p.lat_new + k), a);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0) snw[hh] = a * scale;
    }
    consumer_sync(kConsumerThreads);
    float mn[2], an[2], pn[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int hh = g8 + 8 * half;
      const float mo = mst[hh], sv = snw[hh];
      mn[half] = fmaxf(mo, sv);
      an[half] = mo == -INFINITY ? 0.f : exp2f(mo - mn[half]);
      pn[half] = exp2f(sv - mn[half]);
    }
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      if (n < nt_count) {
        const int cc = col0 + n * 8 + 2 * t4;
        const float v0 = __ldcg(p.lat_new + cc), v1 = __ldcg(p.lat_new + cc + 1);
        o[n][0] = o[n][0] * an[0] + pn[0] * v0;
        o[n][1] = o[n][1] * an[0] + pn[0] * v1;
        o[n][2] = o[n][2] * an[1] + pn[1] * v0;
        o[n][3] = o[n][3] * an[1] + pn[1] * v1;
      }
    }
    consumer_sync(kConsumerThreads);
    if (ctid < HG) {
      const float mo = mst[ctid], sv = snw[ctid], m2 = fmaxf(mo, sv);
      const float a = mo == -INFINITY ? 0.f : exp2f(mo - m2);
      lst[ctid] = lst[ctid] * a + exp2f(sv - m2);
      mst[ctid] = m2;
    }
    consumer_sync(kConsumerThreads);
  }

  // ---- this split's partial: O (KL), m, l per head
  const size_t pstride = (size_t)mla_pstride(KL);
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    if (n < nt_count) {
      const int cc = col0 + n * 8 + 2 * t4;
      float* d0 = p.part + ((size_t)(hg * HG + g8) * S + split) * pstride + cc;
      float* d8 = p.part + ((size_t)(hg * HG + g8 + 8) * S + split) * pstride + cc;
      d0[0] = o[n][0];
      d0[1] = o[n][1];
      d8[0] = o[n][2];
      d8[1] = o[n][3];
    }
  }
  if (ctid < HG) {
    float* d = p.part + ((size_t)(hg * HG + ctid) * S + split) * pstride + KL;
    d[0] = mst[ctid];
    d[1] = lst[ctid];
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0) {
    if (p.trace) p.trace[(size_t)t.id * kTraceCols + 6] = (long long)globaltimer_ns();
    publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);
  }
}

// ---- sparse MLA: index scoring and top-K selection ----------------------------------------------
// Index scoring task = split sp of the cached positions [0, pos).  Per stage of kIndexRows
// index keys: S[j][t] = q_I[j] . k_I[t] on the tensor cores (mma.sync m16n8k16, fp32
// accumulation; the queries, rounded to bf16, as A from shared memory, 16 heads per
// m-tile; the bf16 keys as B straight from the swizzled tile), then
// I[t] = sum_j w'_j ReLU(S[j][t]) with w' = w_I / sqrt(H_I D_I).  Warp w takes the
// stage's positions 16 w .. 16 w + 15 against every head, so ReLU, weights and the sum
// over heads stay in the warp (per thread, then shuffles).  The scores go to
// iscore[layer]; a shared histogram of their order keys' top bits is added into the
// layer's global histogram, and every split publishes the layer's index counter (split 0
// first resets the chosen counts).  The last split also scores the new position from its
// on-chip key (rounded to bf16 as the cache holds it).

// Byte offset of 16-byte chunk c of row r of the [H_I][D_I] bf16 query tile (rows of
// 2 D_I bytes, chunks XOR-swizzled by r & 7 so that ldmatrix reads 8 rows conflict-free).
__device__ __forceinline__ uint32_t qtile_off(int r, int c, int DI) {
  return (uint32_t)(r * DI * 2 + ((c ^ (r & 7)) << 4));
}

__device__ void index_task(const Params& p, const Task& t, uint32_t gs, int ns, uint8_t* ring,
                           uint64_t* full, uint64_t* empty, const uint32_t* tags, float* ub,
                           int* tk, int warp, int lane, int ctid, bool& ab) {
  const int HI = p.HI, DI = p.DI, MTI = HI / 16, KS = DI / 16;
  const int g8 = lane >> 2, t4 = lane & 3;
  uint32_t* hist = reinterpret_cast<uint32_t*>(ub);                   // [kIndexBins]
  uint8_t* qt = reinterpret_cast<uint8_t*>(ub + kIndexBins);          // [H_I][D_I] bf16
  float* wsc = ub + kIndexBins + kIndexMaxHeads * 128 / 2;            // [kIndexMaxHeads]
  float* nsum = wsc + kIndexMaxHeads;                                 // [kConsumerWarps]
  const int C = p.KL + p.R;
  const float* qi = p.qkv + (size_t)p.Hq * (p.NP + p.R);  // q_I [H_I][D_I]
  const float* kin = p.cqkv + p.QL + C;                    // k_I of this position [D_I]
  const float* win = kin + DI;                             // w_I [H_I]
  for (int b = ctid; b < kIndexBins; b += kConsumerThreads) hist[b] = 0u;
  for (int e = ctid; e < HI * DI / 8; e += kConsumerThreads) {  // 8 columns per item
    const int r = e / (DI / 8), c = e % (DI / 8);
    const float4 x0 = __ldcg(reinterpret_cast<const float4*>(qi + (size_t)r * DI + 8 * c));
    const float4 x1 = __ldcg(reinterpret_cast<const float4*>(qi + (size_t)r * DI + 8 * c + 4));
    uint4 v;
    v.x = bf2_bits(__floats2bfloat162_rn(x0.x, x0.y));
    v.y = bf2_bits(__floats2bfloat162_rn(x0.z, x0.w));
    v.z = bf2_bits(__floats2bfloat162_rn(x1.x, x1.y));
    v.w = bf2_bits(__floats2bfloat162_rn(x1.z, x1.w));
    *reinterpret_cast<uint4*>(qt + qtile_off(r, c, DI)) = v;
  }
  const float wnorm = 1.f / sqrtf((float)(HI * DI));
  if (ctid < HI) wsc[ctid] = __ldcg(win + ctid) * wnorm;
  consumer_sync(kConsumerThreads);
  float wt[4][2];  // this thread's head weights: rows g8, g8 + 8 of every m-tile
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    wt[mt][0] = mt < MTI ? wsc[mt * 16 + g8] : 0.f;
    wt[mt][1] = mt < MTI ? wsc[mt * 16 + g8 + 8] : 0.f;
  }
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 4] = (long long)globaltimer_ns();
  float* score = p.iscore + (size_t)t.layer * p.cap;
  int t0, t1;
  attn_range(p, t, t0, t1);
  const uint32_t NS = (uint32_t)p.ring_stages;
  const uint32_t qb = smem_u32(qt);
  const int m = lane >> 3;
  const int rb = warp * 16 + (m >> 1) * 8 + (lane & 7);   // this lane's key row (ldmatrix)
  const int ra = (m & 1) * 8 + (lane & 7);                // this lane's query row in an m-tile
  long long waited = 0;  // trace: ns warp 0 spent waiting for stages to land
  for (int i = 0; i < ns; ++i) {
    const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
    const long long w0 = p.trace ? (long long)globaltimer_ns() : 0;
    const bool landed = stage_wait(p, full, tags, sidx);
    if (p.trace) waited += (long long)globaltimer_ns() - w0;
    const uint32_t tb = smem_u32(ring + (size_t)slot * p.stage_bytes);
    float c[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int k = 0; k < 4; ++k) c[mt][n][k] = 0.f;
    if (landed) {
#pragma unroll 2
      for (int j = 0; j < KS; ++j) {
        uint32_t b0, b1, b2, b3;
        const int chb = 2 * j + (m & 1);  // key chunk: k 0-7 (even) or 8-15 of the step
        ldsm_x4(tb + swz_off(chb >> 3, rb, chb & 7, kIndexRows), b0, b1, b2, b3);
        const int cha = 2 * j + (m >> 1);  // query chunk of matrices 2, 3: k 8-15
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          if (mt < MTI) {
            uint32_t a[4];
            ldsm_x4(qb + qtile_off(mt * 16 + ra, cha, DI), a[0], a[1], a[2], a[3]);
            mma_bf16(c[mt][0], a, b0, b1);
            mma_bf16(c[mt][1], a, b2, b3);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_n(&empty[slot], 1u);
    }
    if (__any_sync(0xffffffffu, !landed)) {  // one warp's view is enough to stop
      ab = true;
      break;
    }
    // ReLU, head weights, sum over the heads: positions 16 warp + 8 n + 2 t4 (+ 1)
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      float v0 = 0.f, v1 = 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        v0 = fmaf(fmaxf(c[mt][n][0], 0.f), wt[mt][0], v0);
        v0 = fmaf(fmaxf(c[mt][n][2], 0.f), wt[mt][1], v0);
        v1 = fmaf(fmaxf(c[mt][n][1], 0.f), wt[mt][0], v1);
        v1 = fmaf(fmaxf(c[mt][n][3], 0.f), wt[mt][1], v1);
      }
#pragma unroll
      for (int off = 4; off <= 16; off <<= 1) {
        v0 += __shfl_xor_sync(0xffffffffu, v0, off);
        v1 += __shfl_xor_sync(0xffffffffu, v1, off);
      }
      if (g8 == 0) {
        const int tt = t0 + i * kIndexRows + warp * 16 + 8 * n + 2 * t4;
        if (tt < t1) {
          const float sc = v0 == 0.f ? 0.f : v0;  // -0 and +0 are one score
          score[tt] = sc;
          atomicAdd(hist + (order_key(sc) >> (32 - kIndexBinBits)), 1u);
        }
        if (tt + 1 < t1) {
          const float sc = v1 == 0.f ? 0.f : v1;
          score[tt + 1] = sc;
          atomicAdd(hist + (order_key(sc) >> (32 - kIndexBinBits)), 1u);
        }
      }
    }
  }
  // every warp must agree on an abort before the barriers below
  if (consumer_sync_or(ab, kConsumerThreads)) {
    ab = true;
    return;
  }
  if (ctid == 0 && p.trace) {
    p.trace[(size_t)t.id * kTraceCols + 5] = (long long)globaltimer_ns();
    p.trace[(size_t)t.id * kTraceCols + 7] = waited;
  }
  if (t.r1 == t.aux - 1) {  // the new position, from its key on chip (rounded to bf16)
    // warp w takes heads w, w + 8, ...; lane l columns 4 l .. 4 l + 3 (D_I <= 128), the
    // queries from the bf16 tile the stages used
    float part = 0.f;
    const int k0 = 4 * lane;
    float kv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      kv[k] = k0 + k < DI ? __bfloat162float(__float2bfloat16_rn(__ldcg(kin + k0 + k))) : 0.f;
    for (int h = warp; h < HI; h += kConsumerWarps) {
      float d = 0.f;
      if (k0 < DI) {
        const __nv_bfloat16* qr =
            reinterpret_cast<const __nv_bfloat16*>(qt + qtile_off(h, k0 >> 3, DI)) + (k0 & 7);
#pragma unroll
        for (int k = 0; k < 4; ++k) d = fmaf(__bfloat162float(qr[k]), kv[k], d);
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      part = fmaf(fmaxf(d, 0.f), wsc[h], part);
    }
    if (lane == 0) nsum[warp] = part;
    consumer_sync(kConsumerThreads);
    if (ctid == 0) {
      float sc = 0.f;
      for (int w = 0; w < kConsumerWarps; ++w) sc += nsum[w];
      if (sc == 0.f) sc = 0.f;
      score[p.pos] = sc;
      atomicAdd(hist + (order_key(sc) >> (32 - kIndexBinBits)), 1u);
    }
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 6] = (long long)globaltimer_ns();
  uint32_t* gh = p.ix_hist + (size_t)t.layer * kIndexBins;
  for (int b = ctid; b < kIndexBins; b += kConsumerThreads) {
    const uint32_t v = hist[b];
    if (v) atomicAdd(gh + b, v);
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0) {
    if (t.r1 == 0) {  // this step's selection starts from no chosen positions
      uint32_t* meta = index_meta(p, t.layer);
      meta[IM_NSEL] = 0u;
      meta[IM_NCAND] = 0u;
      meta[IM_HASPOS] = 0u;
    }
    publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);  // after the CTA's histogram adds (barrier above)
  }
}

// The bin of the K-th largest score of the layer's complete histogram, found by every
// selection task: thread j holds bins kIndexBins - 1 - (16 j + k), k < 16 (descending); a
// scan over the threads finds the bin b where the count above it is below K and the count
// from it on reaches K.  thr[0..2] receive b, how many of b are still to take, b's count.
__device__ void index_threshold(const Params& p, int layer, uint32_t* thr, uint32_t* wt,
                                int warp, int lane, int ctid) {
  static_assert(kIndexBins == 16 * kConsumerThreads, "16 bins per consumer thread");
  const uint32_t* gh = p.ix_hist + (size_t)layer * kIndexBins;
  const uint32_t K = (uint32_t)p.KI;
  uint32_t cnt[16], sum = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    cnt[k] = __ldcg(gh + kIndexBins - 1 - (16 * ctid + k));
    sum += cnt[k];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) wt[warp] = incl;
  consumer_sync(kConsumerThreads);
  uint32_t excl = incl - sum;
  for (int w = 0; w < warp; ++w) excl += wt[w];
  if (excl < K && excl + sum >= K) {
    uint32_t run = excl;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (run < K && run + cnt[k] >= K) {
        thr[0] = (uint32_t)(kIndexBins - 1 - (16 * ctid + k));
        thr[1] = K - run;
        thr[2] = cnt[k];
      }
      run += cnt[k];
    }
  }
  consumer_sync(kConsumerThreads);
}

// Append `take` lanes' values to list[] at the counter *ctr (one atomic per warp); an
// index at or past `cap` records a bounds error instead.
__device__ __forceinline__ void warp_append(const Params& p, bool take, uint32_t* ctr, int32_t* list,
                                            int32_t val, int cap, int lane, int detail) {
  const uint32_t mask = __ballot_sync(0xffffffffu, take);
  if (!mask) return;
  const int leader = __ffs(mask) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(ctr, (uint32_t)__popc(mask));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (take) {
    const uint32_t idx = base + (uint32_t)__popc(mask & ((1u << lane) - 1u));
    if (idx < (uint32_t)cap) list[idx] = val;
    else record_error(p, TRE_ERR_BOUNDS, detail);
  }
}

// Run by the selection task that arrives last when the threshold bin holds more than are
// still to take: the `need` largest (score, then lower position) of its candidates, by an
// MSD radix select on keys (low 20 bits of the order key << pb) | (2^pb - 1 - position),
// pb = bits of a position (all candidates share the top 12 bits); the keys are unique, so
// exactly `need` of them reach the selected one.
__device__ void index_pick(const Params& p, const Task& t, float* scratch, uint32_t need, int warp,
                           int lane, int ctid) {
  uint32_t* meta = index_meta(p, t.layer);
  const unsigned long long* cand = p.ix_cand + (size_t)t.layer * p.cap;
  int32_t* sel = p.ix_sel + (size_t)t.layer * p.KI;
  const uint32_t n = min(__ldcg(meta + IM_NCAND), (uint32_t)p.cap);
  uint32_t* h = reinterpret_cast<uint32_t*>(scratch);  // [256]
  uint32_t* sh = h + 256;                               // digit, still to take
  // the candidates' keys in shared memory when they fit (the usual case: the threshold
  // bin holds a small share of the positions), else read from L2 on every pass
  unsigned long long* ks = reinterpret_cast<unsigned long long*>(scratch + 512);
  const bool in_smem = n <= kPickSmemKeys;
  const int pb = 32 - __clz(max(p.cap - 1, 1));
  const unsigned long long pmask = (1ull << pb) - 1ull;
  auto keyof = [&](unsigned long long c) {
    const unsigned long long k20 = (c >> 32) & 0xFFFFFull;
    const unsigned long long pos = 0xffffffffull - (c & 0xffffffffull);
    return (k20 << pb) | (pmask - pos);
  };
  auto key_at = [&](uint32_t i) { return in_smem ? ks[i] : keyof(__ldcg(cand + i)); };
  if (in_smem)
    for (uint32_t i = ctid; i < n; i += kConsumerThreads) ks[i] = keyof(__ldcg(cand + i));
  const int bits = 20 + pb;
  unsigned long long prefix = 0;
  uint32_t rem = need;
  for (int sft = (bits + 7) / 8 * 8 - 8; sft >= 0; sft -= 8) {
    for (int i = ctid; i < 256; i += kConsumerThreads) h[i] = 0u;
    consumer_sync(kConsumerThreads);
    for (uint32_t i = ctid; i < n; i += kConsumerThreads) {
      const unsigned long long k = key_at(i);
      if ((k >> (sft + 8)) == prefix) atomicAdd(h + ((k >> sft) & 255u), 1u);
    }
    consumer_sync(kConsumerThreads);
    if (warp == 0) {  // lane l holds digits 255 - 8 l - k, k < 8 (descending)
      uint32_t c8[8], s8 = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        c8[k] = h[255 - 8 * lane - k];
        s8 += c8[k];
      }
      uint32_t incl = s8;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      uint32_t run = incl - s8;
      if (run < rem && run + s8 >= rem) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (run < rem && run + c8[k] >= rem) {
            sh[0] = (uint32_t)(255 - 8 * lane - k);
            sh[1] = rem - run;
          }
          run += c8[k];
        }
      }
    }
    consumer_sync(kConsumerThreads);
    prefix = (prefix << 8) | sh[0];
    rem = sh[1];
    consumer_sync(kConsumerThreads);  // sh and h are rewritten by the next pass
  }
  // every candidate whose key reaches the selected one
  for (uint32_t i0 = 0; i0 < n; i0 += kConsumerThreads) {
    const uint32_t i = i0 + ctid;
    bool take = false;
    int pos = 0;
    if (i < n) {
      const unsigned long long k = key_at(i);
      take = k >= prefix;
      pos = (int)(pmask - (k & pmask));
    }
    if (take && pos == p.pos) {
      meta[IM_HASPOS] = 1u;
      take = false;
    }
    warp_append(p, take, meta + IM_NSEL, sel, pos, p.KI, lane, t.id);
  }
}

// Selection task = split sp of the positions [0, pos]: it finds the threshold bin in the
// complete histogram (index_threshold), then positions whose bin is above it are chosen
// (the whole threshold bin when all of it is to take) and the threshold bin's others
// become candidates; the new position is flagged instead of listed (its latent row comes
// from on chip).  The task that arrives last clears the histogram, runs index_pick when
// needed, then (the attention also reads this layer's W_uk contraction) waits for the
// W_uk tasks and publishes the layer's selection counter.  Steps with pos + 1 <= K only
// do the last part.
__device__ void isel_task(const Params& p, const Task& t, float* ub, int* tk, int warp, int lane,
                          int ctid, bool& ab) {
  uint32_t* meta = index_meta(p, t.layer);
  const bool sparse = sparse_step(p);
  uint32_t* th = reinterpret_cast<uint32_t*>(ub);  // threshold bin, still to take, its count
  uint32_t need = 0, bincnt = 0;
  if (sparse) {
    index_threshold(p, t.layer, th, th + 4, warp, lane, ctid);
    const uint32_t thr = th[0];
    need = th[1];
    bincnt = th[2];
    const bool whole_bin = need == bincnt;
    const long long P = p.pos + 1;
    const int t0 = (int)(P * t.r1 / t.aux), t1 = (int)(P * (t.r1 + 1) / t.aux);
    const float* score = p.iscore + (size_t)t.layer * p.cap;
    int32_t* sel = p.ix_sel + (size_t)t.layer * p.KI;
    unsigned long long* cand = p.ix_cand + (size_t)t.layer * p.cap;
    for (int b0 = t0; b0 < t1; b0 += kConsumerThreads) {
      const int tt = b0 + ctid;
      const bool live = tt < t1;
      const float sc = live ? __ldcg(score + tt) : 0.f;
      const uint32_t key = order_key(sc), bin = key >> (32 - kIndexBinBits);
      bool above = live && (bin > thr || (whole_bin && bin == thr));
      const bool cnd = live && !whole_bin && bin == thr;
      if (above && tt == p.pos) {
        meta[IM_HASPOS] = 1u;
        above = false;
      }
      warp_append(p, above, meta + IM_NSEL, sel, tt, p.KI, lane, t.id);
      const uint32_t mask = __ballot_sync(0xffffffffu, cnd);
      if (mask) {
        const int leader = __ffs(mask) - 1;
        uint32_t base = 0;
        if (lane == leader) base = atomicAdd(meta + IM_NCAND, (uint32_t)__popc(mask));
        base = __shfl_sync(0xffffffffu, base, leader);
        if (cnd) {
          const uint32_t idx = base + (uint32_t)__popc(mask & ((1u << lane) - 1u));
          if (idx < (uint32_t)p.cap)
            cand[idx] = ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)tt);
          else
            record_error(p, TRE_ERR_BOUNDS, t.id);
        }
      }
    }
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 4] = (long long)globaltimer_ns();
  if (ctid == 0) *tk = ((ticket_add(meta + IM_TICK_B, 1u) + 1u) % (uint32_t)t.aux) == 0u;
  consumer_sync(kConsumerThreads);
  if (!*tk) return;
  // every selection task has read the histogram: clear it for the next step
  {
    uint32_t* gh = p.ix_hist + (size_t)t.layer * kIndexBins;
    for (int b = ctid; b < kIndexBins; b += kConsumerThreads) gh[b] = 0u;
  }
  if (sparse && need != bincnt) index_pick(p, t, ub + 16, need, warp, lane, ctid);
  consumer_sync(kConsumerThreads);
  if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 5] = (long long)globaltimer_ns();
  if (ctid == 0) {
    const bool ok = wait_counter(p, t.layer * C_PER_LAYER + C_MLA_UK, (uint32_t)p.Hq, t.id);
    if (ok) publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);
    *tk = ok ? 0 : 1;
  }
  consumer_sync(kConsumerThreads);
  if (*tk) ab = true;
}

// The W_uv task of head h stages o_lat_h, merging the head's KV splits on the way:
// o_lat_h = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s (splits that saw no position
// have m_s = -inf and weigh 0).  128 heads merge on 128 SMs at once.
__device__ __noinline__ void mla_combine_input(const Params& p, const Task& t, float* ub, float* scratch,
                                  int ctid) {
  const int h = t.r0 / p.VD, KL = p.KL, S = p.nsplit;
  const size_t pstride = (size_t)mla_pstride(KL);
  const float* base = p.part + (size_t)h * S * pstride;
  float* ms = scratch;       // [S] split maxima, then weights 2^(m_s - M)
  float* lsum = scratch + S; // [S] split sums
  float* ls = lsum + S;      // [1] 1 / sum_s w_s l_s
  // Every load is issued before the weights are known: (m, l) of each split, and this
  // thread's two columns of the first kPre splits' partials (the loads of one thread are
  // independent, so they overlap: one L2 round trip instead of one per phase).
  constexpr int kPre = 16;
  const int c = 2 * ctid;
  float2 pv[kPre];
#pragma unroll
  for (int s2 = 0; s2 < kPre; ++s2)
    if (s2 < S && c < KL)
      pv[s2] = __ldcg(reinterpret_cast<const float2*>(base + s2 * pstride + c));
  for (int s2 = ctid; s2 < S; s2 += kConsumerThreads) {
    ms[s2] = __ldcg(base + s2 * pstride + KL);
    lsum[s2] = __ldcg(base + s2 * pstride + KL + 1);
  }
  consumer_sync(kConsumerThreads);
  if (ctid < 32) {
    float M = -INFINITY;
    for (int s2 = ctid; s2 < S; s2 += 32) M = fmaxf(M, ms[s2]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
    for (int s2 = ctid; s2 < S; s2 += 32) {
      const float w = ms[s2] == -INFINITY ? 0.f : exp2f(ms[s2] - M);
      L = fmaf(w, lsum[s2], L);
      ms[s2] = w;
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (ctid == 0) ls[0] = 1.f / L;
  }
  consumer_sync(kConsumerThreads);
  const float inv = ls[0];
  float* xlo = ub;
  float* xhi = ub + KL / 2;
  // columns c, c + 1 of the input planes (plane lo holds x[8j .. 8j + 3], hi x[8j + 4 ..])
  auto put = [&](int col, float v) {
    const int j = col >> 3, w = col & 7;
    (w < 4 ? xlo : xhi)[4 * j + (w & 3)] = v * inv;
  };
  for (int cc = c; cc < KL; cc += 2 * kConsumerThreads) {
    float v0 = 0.f, v1 = 0.f;
    if (cc == c) {
#pragma unroll
      for (int s2 = 0; s2 < kPre; ++s2)
        if (s2 < S) {
          v0 = fmaf(ms[s2], pv[s2].x, v0);
          v1 = fmaf(ms[s2], pv[s2].y, v1);
        }
    }
    for (int s2 = cc == c ? kPre : 0; s2 < S; ++s2) {
      const float2 a = __ldcg(reinterpret_cast<const float2*>(base + s2 * pstride + cc));
      v0 = fmaf(ms[s2], a.x, v0);
      v1 = fmaf(ms[s2], a.y, v1);
    }
    put(cc, v0);
    put(cc + 1, v1);
  }
  consumer_sync(kConsumerThreads);
}

// ---- GEMV epilogue ---------------------------------------------------------------------------------
// Residual rows of an O-proj / down task, staged before its stages: part 0 reads the
// residual stream (x, or for layer 0 the embedding row / layer input; h1 for down), later
// K-parts read the partial sum the previous part left in the output.
template <int MT>
__device__ __forceinline__ void prefetch_resid(const Params& p, const Task& t, const GemvGeom& g,
                                               float* resid, int ctid) {
  const int nr = t.r1 - t.r0;
  for (int idx = ctid; idx < MT * nr; idx += kConsumerThreads) {
    const int v = idx / nr, r = idx % nr, n = t.r0 + r;
    const size_t off = (size_t)v * p.d + n;
    float val;
    if (t.op == OP_O) val = g.part == 0 ? resid_in(p, t.layer, n, v) : __ldcg(p.h1 + off);
    else if (t.op == OP_MO) val = g.part == 0 ? resid_in(p, t.layer, n, v) : __ldcg(p.x + off);
    else val = g.part == 0 ? __ldcg(p.h1 + off) : __ldcg(p.x + off);
    resid[v * kMaxResidRows + r] = val;
  }
}

// One output row of a GEMV task (MLA: the absorbed-MLA ops' epilogues; else GQA / MoE),
// specialised per stack so that each kernel dispatches over its own ops only.
template <bool MLA>
__device__ __forceinline__ void gemv_emit(const Params& p, const Task& t, const GemvGeom& g, int n,
                                          float v, float rn, const float* resid, Best& best,
                                          int tok = 0) {
  if constexpr (MLA) {
    switch (t.op) {
      case OP_UQ: p.qkv[n] = v * rn; break;
      case OP_MDQKV: {
        const float y = v * rn;
        p.cqkv[n] = y;
        const int ki = n - (p.QL + p.KL + p.R);  // sparse: this position's index key
        if (ki >= 0 && ki < p.DI)
          reinterpret_cast<__nv_bfloat16*>(p.layers[t.layer].v_cache)[(size_t)p.pos * p.DI + ki] =
              __float2bfloat16_rn(y);
      } break;
      case OP_UV: p.mla_o[n] = v; break;
      case OP_MOS: p.mpart[(size_t)g.part * p.d + n] = v; break;
      case OP_MO: {
        const float y = resid[n - t.r0] + v;
        p.x[n] = y;
        if (g.part == g.np - 1) {
          if (p.hidden) p.hidden[(size_t)t.layer * p.d + n] = y;
          if (p.x_out && t.layer == p.L - 1) p.x_out[n] = y;
        }
      } break;
      default: {
        const float y = v * rn;
        p.logits[n] = y;
        best_update(best, y, n);
      } break;
    }
  } else {
    switch (t.op) {
      case OP_QKV: p.qkv[(size_t)tok * (p.Hq + 2 * p.Hkv) * p.D + n] = v * rn; break;
      case OP_O: p.h1[(size_t)tok * p.d + n] = resid[n - t.r0] + v; break;
      case OP_ROUTER: p.scores[n] = 1.f / (1.f + expf(-v * rn)); break;
      case OP_MDOWN: p.mpart[(size_t)g.part * p.d + n] = v; break;
      case OP_DOWN: {
        const float y = resid[n - t.r0] + v;
        p.x[(size_t)tok * p.d + n] = y;
        if (g.part == g.np - 1) {
          if (p.hidden) p.hidden[((size_t)t.layer * p.m + tok) * p.d + n] = y;
          if (p.x_out && t.layer == p.L - 1) p.x_out[(size_t)tok * p.d + n] = y;
        }
      } break;
      default: {
        const float y = v * rn;
        p.logits[(size_t)tok * p.V + n] = y;
        best_update(best, y, n);
      } break;
    }
  }
}

// ---- MoE routing -----------------------------------------------------------------------------------
// Run by the router task that finishes last (arrival ticket): the top_k experts by score,
// ties to the lower expert index, in descending order, and their weights normalised over
// the selection (DeepSeek-style sigmoid routing; the pages name the fused op
// ExpertSelectUpGateSiLU — TileRT code audit, MoE paragraph).  Warp 0 selects: each lane
// holds the scores of experts lane, lane + 32, ...; every round is one warp arg-max.
// Then the layer's route counter is bumped with release semantics.
__device__ void route_topk(const Params& p, int layer, float* sc, int warp, int lane, int ctid) {
  for (int e = ctid; e < p.E; e += kConsumerThreads) sc[e] = __ldcg(p.scores + e);
  consumer_sync(kConsumerThreads);
  if (warp != 0) return;
  uint32_t taken = 0;  // bit i: expert lane + 32 i already selected
  float tot = 0.f, mine = 0.f;
  for (int j = 0; j < p.topk; ++j) {
    Best b{-INFINITY, 0x7fffffff};
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const int e = lane + 32 * i;
      if (e < p.E && !((taken >> i) & 1u)) best_update(b, sc[e], e);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      Best o;
      o.v = __shfl_xor_sync(0xffffffffu, b.v, off);
      o.i = __shfl_xor_sync(0xffffffffu, b.i, off);
      best_update(b, o.v, o.i);
    }
    if (b.i != 0x7fffffff && (b.i & 31) == lane) taken |= 1u << (b.i >> 5);
    tot += b.v;
    if (lane == j) mine = b.v;
    if (lane == 0) p.route_idx[layer * p.topk + j] = b.i;
  }
  if (lane < p.topk) p.route_w[layer * p.topk + lane] = mine / tot;
  __syncwarp();
  if (lane == 0) publish_add(p.counters + (size_t)(layer * C_PER_LAYER + C_ROUTE) * kCtrStride, 1u);
}

// The last slot of a MoE-down row block to finish: x = h1 + sum of the slots' partial rows
// in slot order (deterministic), then the block is published.
// The last K-slice of an MLA output row block to finish: x = x + sum_j partial_j (slice
// order, deterministic), then the layer's output counter.
__device__ void mo_slices_combine(const Params& p, const Task& t, int np, int ctid) {
  for (int n = t.r0 + ctid; n < t.r1; n += kConsumerThreads) {
    float y = resid_in(p, t.layer, n);
    for (int j = 0; j < np; ++j) y += __ldcg(p.mpart + (size_t)j * p.d + n);
    p.x[n] = y;
    if (p.hidden) p.hidden[(size_t)t.layer * p.d + n] = y;
    if (p.x_out && t.layer == p.L - 1) p.x_out[n] = y;
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0) publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);
}

__device__ void moe_down_combine(const Params& p, const Task& t, int ctid) {
  const int np = p.nshared + p.topk;
  for (int n = t.r0 + ctid; n < t.r1; n += kConsumerThreads) {
    float y = __ldcg(p.h1 + n);
    for (int j = 0; j < np; ++j) y += __ldcg(p.mpart + (size_t)j * p.d + n);
    p.x[n] = y;
    if (p.hidden) p.hidden[(size_t)t.layer * p.d + n] = y;
    if (p.x_out && t.layer == p.L - 1) p.x_out[n] = y;
  }
  consumer_sync(kConsumerThreads);
  if (ctid == 0) publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);
}


// ---- multi-token GEMV on the tensor cores ---------------------------------------------------------
// With m tokens per step a GEMV row is dotted with m input vectors, which makes the stage a
// small dense contraction (16 rows x kw columns x m tokens): mma.sync m16n8k16 with A = the
// tile's 16 weight rows (bf16, ldmatrix from the padded row slots) and B = the tokens' input
// columns split into bf16 hi parts (column v) and lo parts (column 4 + v), so that
// D[r][v] + D[r][4 + v] is row r . x_v with about 16 significand bits of x (the input
// staging writes that operand in fragment order).  Every consumer
// warp takes every stage and a 1/8 share of its 16-column k-steps; the warps' accumulators
// are summed once per row tile through a double-buffered shared-memory area.
template <int MT>
__device__ __forceinline__ void gemv_tile_task(const Params& p, const Task& t, const GemvGeom& g,
                                               uint32_t gs, int ns, uint8_t* ring, uint64_t* full,
                                               uint64_t* empty, const uint32_t* tags,
                                               const float* xs, float* tred, const float* resid,
                                               const float (&rnt)[MT], float wsel, int uoff,
                                               Best (&best)[MT], int warp, int lane, int ctid,
                                               bool& ab) {
  const uint32_t NS = (uint32_t)p.ring_stages;
  const int gq = lane >> 2, tig = lane & 3;
  // B fragment of this lane (mma column gq: token gq & 3, hi part for gq < 4, else lo), as
  // the input staging laid it out: 8 MT words of 8 bytes per k-step
  const int bv = gq & 3;
  const bool bact = bv < MT;
  const uint2* xb = reinterpret_cast<const uint2*>(xs) + ((gq >> 2) * MT + (bact ? bv : 0)) * 4 + tig;
  float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
  int buf = 0;
  bool bad = false;
  uint32_t slot = gs % NS, par = (gs / NS) & 1u;
  TileStage ts = tile_first(t, g);
  for (int i = 0; i < ns; ++i, tile_next(ts, t, g), ring_next(slot, par, NS)) {
    const uint32_t sidx = gs + (uint32_t)i;
    if (!bad) bad = !stage_wait_at(p, full, tags, sidx, slot, par);
    if (!bad) {
      const uint32_t sa = smem_u32(ring + (size_t)slot * p.stage_bytes) +
                          (uint32_t)((lane & 15) * kTilePitch + (lane >> 4) * 16);
      const int nks = ts.kw >> 4;
      for (int k = warp; k < nks; k += kConsumerWarps) {
        uint32_t a[4];
        ldsm_x4(sa + (uint32_t)k * 32u, a[0], a[1], a[2], a[3]);
        uint2 b = make_uint2(0u, 0u);
        if (bact) b = xb[(size_t)((ts.c0 >> 4) + k) * (8 * MT)];
        const uint32_t b0 = b.x, b1 = b.y;
        if (ts.seg == 0) mma_bf16(acc0, a, b0, b1);
        else mma_bf16(acc1, a, b0, b1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_n(&empty[slot], 1u);
    }
    if (!ts.last) continue;
    // row tile done: hi + lo (columns v and 4 + v are lanes tig and tig ^ 2), then the
    // lanes tig < 2 store tokens 2 tig, 2 tig + 1 of rows gq and gq + 8
    float* tb = tred + buf * (2 * kConsumerWarps * kTileRows * kMaxTokens);
#pragma unroll
    for (int sg = 0; sg < 2; ++sg) {
      if (sg == 1 && g.nseg < 2) break;
      float* acc = sg == 0 ? acc0 : acc1;
      float d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        d[e] = acc[e] + __shfl_xor_sync(0xffffffffu, acc[e], 2);
        acc[e] = 0.f;
      }
      if (tig < 2) {
        float* w = tb + (sg * kConsumerWarps + warp) * (kTileRows * kMaxTokens);
        *reinterpret_cast<float2*>(w + gq * kMaxTokens + 2 * tig) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(w + (gq + 8) * kMaxTokens + 2 * tig) = make_float2(d[2], d[3]);
      }
    }
    if (consumer_sync_or(bad, kConsumerThreads)) {  // uniform: all warps leave together
      ab = true;
      return;
    }
    const int r = ctid & (kTileRows - 1), v = ctid >> 4;
    if (v < MT && r < ts.nr) {
      float y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        y0 += tb[w * (kTileRows * kMaxTokens) + r * kMaxTokens + v];
        if (g.nseg == 2) y1 += tb[(kConsumerWarps + w) * (kTileRows * kMaxTokens) + r * kMaxTokens + v];
      }
      const int n = ts.n0 + r;
#pragma unroll
      for (int vv = 0; vv < MT; ++vv) {
        if (vv != v) continue;
        if (g.nseg == 2) {
          const float a = y0 * rnt[vv], bb = y1 * rnt[vv];
          p.u[(size_t)vv * p.F + uoff + n] = wsel * (a / (1.f + expf(-a)) * bb);
        } else {
          gemv_emit<false>(p, t, g, n, y0, rnt[vv], resid + vv * kMaxResidRows, best[vv], vv);
        }
      }
    }
    buf ^= 1;
  }
  if (bad) ab = true;
}

// ---- consumers -----------------------------------------------------------------------------------
// ---- E4M3 GEMV on the tensor cores ------------------------------------------------------------
// A stage holds up to 8 weight rows (gate / up: up to 4 rows of each) of the task's K-part at
// a pitch of span + 16 bytes, span = 2 Lh (Lh: half the K-part, rounded up to 32 columns).
// One mma.sync m16n8k32 E4M3 x E4M3 -> fp32 tile covers 32 columns of both halves of the 8
// rows, the weights as stored: tile row r < 8 is weight row r at columns [c, c + 32), tile
// row 8 + r the same row at [Lh + c, Lh + c + 32), so an ldmatrix.x4 is exactly the A
// fragment.  The B operand holds the input's 4 E4M3 terms of those columns (load_input_e4m3):
// columns 0-3 the terms of half 0, 4-7 those of half 1.  Of the 16 x 8 products a lane keeps
// its row g's pair of terms of its half (lanes t4 < 2: half 0, t4 >= 2: half 1), weighed by
// 16^-tau, the chunk's 2^-sg and the weight block scale (32 columns never straddle a
// 128-column block).  All 8 warps share each stage, warp w taking the chunks w, w + 8, ...;
// the lanes of a row and then the warps are summed (shuffles, shared memory), and one thread
// per row finishes it.
__device__ void fp8_task(const Params& p, const Task& t, const GemvGeom& g, uint32_t gs, int ns,
                         uint8_t* ring, uint64_t* full, uint64_t* empty, const uint32_t* tags,
                         float* ub, const float* resid, float rn, float wsel, int uoff, int warp,
                         int lane, int ctid, bool& ab, Best& best) {
  const int Lh = fp8_half_len(g.Kp), P = fp8_row_pitch(g.Kp), nch = Lh / 32;
  const uint8_t* frag = reinterpret_cast<const uint8_t*>(ub);
  const float* csc = ub + 2 * Lh;            // 2^-sg per 32 columns of the span
  float* red = ub + fp8_frag_floats(g.Kp);   // [2][kConsumerWarps][8]
  const Fp8Scales fs = fp8_scales(p, t, g);
  const bool two = g.nseg == 2;
  const int gq = lane >> 2, t4 = lane & 3, half = t4 >> 1;
  const float wa = (t4 & 1) ? 1.f / 256.f : 1.f, wb = wa * (1.f / 16.f);
  // B: this lane's 8 bytes are term gq & 3 of half gq >> 2, column group t4 (+ 128 per chunk)
  const uint8_t* bp = frag + (gq >> 2) * 4 * Lh + (gq & 3) * 32 + t4 * 8;
  const int mat = lane >> 3, trow = lane & 7;  // ldmatrix: this lane's matrix and row
  const uint32_t NS = (uint32_t)p.ring_stages;
  for (int i = 0; i < ns; ++i) {
    const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
    const bool landed = stage_wait(p, full, tags, sidx);
    const int n0 = t.r0 + i * g.rps, nr = min(g.rps, t.r1 - n0);
    // tile row trow's stage row (gate / up: rows 0-3 gate, 4-7 up), clamped to a loaded row
    const int sr = two ? ((trow >> 2) ? g.rps : 0) + min(trow & 3, nr - 1) : min(trow, nr - 1);
    const uint32_t arow = smem_u32(ring + (size_t)slot * p.stage_bytes) +
                          (uint32_t)(sr * P + (mat & 1) * Lh + (mat >> 1) * 16);
    // the weight row of this lane's output row gq, for its block scales
    const float* srow = two ? fp8_scale_row(fs, gq >> 2, n0 + min(gq & 3, nr - 1))
                            : fp8_scale_row(fs, 0, n0 + min(gq, nr - 1));
    float acc = 0.f;
    if (landed) {
      // kU chunks at a time (chunks w, w + 8, ...), every load issued before the products,
      // so that a warp keeps several ldmatrix / scale loads and mma in flight
      constexpr int kU = 4;
      float accu[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) accu[u] = 0.f;
      for (int cb = warp; cb < nch; cb += kU * kConsumerWarps) {
        uint32_t a[kU][4];
        uint2 b[kU];
        float sc[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int cc = min(cb + u * kConsumerWarps, nch - 1);  // clamped: in-range reads
          ldsm_x4(arow + (uint32_t)(cc * 32), a[u][0], a[u][1], a[u][2], a[u][3]);
          b[u] = *reinterpret_cast<const uint2*>(bp + cc * 128);
          const int col = half * Lh + cc * 32;
          sc[u] = __ldg(srow + ((g.k0 + col) >> 7)) * csc[col >> 5];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int cc = cb + u * kConsumerWarps;
          // columns past Kp are stale shared memory: zero them (the input is zero there); a
          // chunk past the last one (clamped above) counts nothing
          const int c0 = cc * 32 + 4 * t4, c1 = Lh + c0;
          const bool live = cc < nch;
          if (!live || c0 >= g.Kp) a[u][0] = 0u;
          if (!live || c0 + 16 >= g.Kp) a[u][2] = 0u;
          if (!live || c1 >= g.Kp) a[u][1] = 0u;
          if (!live || c1 + 16 >= g.Kp) a[u][3] = 0u;
          float d[4];
          mma_e4m3(d, a[u], b[u].x, b[u].y);
          const float v = half ? fmaf(d[3], wb, d[2] * wa) : fmaf(d[1], wb, d[0] * wa);
          accu[u] = fmaf(v, sc[u], accu[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) acc += accu[u];
      __syncwarp();
      if (lane == 0) mbar_arrive_n(&empty[slot], 1u);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    float* rb = red + (i & 1) * kConsumerWarps * 8;
    if (t4 == 0) rb[warp * 8 + gq] = acc;
    if (consumer_sync_or(!landed, kConsumerThreads)) {
      ab = true;
      return;
    }
    if (ctid < nr && (!two || ctid < 4)) {
      float v = 0.f, u = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        v += rb[w * 8 + ctid];
        if (two) u += rb[w * 8 + 4 + ctid];
      }
      if (two) {  // gate row ctid (v), up row ctid (u)
        const float aa = v * rn, bb = u * rn;
        p.u[uoff + n0 + ctid] = wsel * (aa / (1.f + expf(-aa)) * bb);
      } else {
        gemv_emit<false>(p, t, g, n0 + ctid, v, rn, resid, best);
      }
    }
  }
}

// MLA = true: the absorbed-MLA stack's kernel (MLA tiles, no GQA attention); false: GQA /
// MoE.  Separate instantiations keep each kernel's register allocation to its own tiles.
// TILED: GEMV stages are 16-row tensor-core tiles (multi-token plans).
template <bool MLA, int MT, bool TILED, bool F8, bool SP, bool F4>
__device__ void consumer(const Params& p, const Task* my, int ntask, uint8_t* ring,
                         uint64_t* full, uint64_t* empty, const uint32_t* tags, float* ub,
                         float* misc) {
  const int ctid = threadIdx.x, warp = ctid >> 5, lane = ctid & 31;
  float* red = misc;                                      // [64] reductions
  int* flags = reinterpret_cast<int*>(misc + 64);         // [0] abort, [1] ticket
  float* rn_s = misc + 72;                                // [MT] RMSNorm scales
  const uint32_t NS = (uint32_t)p.ring_stages;
  uint32_t gs = 0;
  int cur_key = -1;
  bool ab = false;
  for (int ti = 0; ti < ntask; ++ti) {
    const Task t = my[ti];
    // stage count before the dependency wait (off the hand-off's critical path), except for
    // tasks whose stages follow this step's sparse selection
    const int ns_early = (MLA && t.type == T_MLA_ATTN) ? -1 : task_nstages<TILED, F4>(p, t);
    if (ctid == 0) {
      long long* tr = p.trace ? p.trace + (size_t)t.id * kTraceCols : nullptr;
      if (tr) tr[0] = (long long)globaltimer_ns();
      const bool ok = !ab && wait_dep(p, t);
      if (ok) fence_acq_rel_gpu();
      flags[0] = ok ? 0 : 1;
      if (tr) {
        tr[1] = (long long)globaltimer_ns();
        tr[3] = (long long)smid();
      }
    }
    consumer_sync(kConsumerThreads);
    if (flags[0]) break;  // uniform: every consumer thread read the same flag
    const int ns = ns_early >= 0 ? ns_early : task_nstages<TILED, F4>(p, t);

    if (!MLA && t.type == T_ATTN) {
      cur_key = -1;  // the attention scratch aliases the input-vector planes
      if constexpr (!MLA)
        run_attn<MT>(p, t, gs, ns, ring, full, empty, tags, ub, flags + 1, warp, lane, ctid, ab);
    } else if (MLA && t.type == T_MLA_ATTN) {
      cur_key = -1;
      if constexpr (MLA)
        mla_attn_task(p, t, gs, ns, ring, full, empty, tags, ub, warp, lane, ctid, ab);
    } else if (SP && t.type == T_INDEX) {
      cur_key = -1;
      if constexpr (SP)
        index_task(p, t, gs, ns, ring, full, empty, tags, ub, flags + 1, warp, lane, ctid, ab);
    } else if (SP && t.type == T_ISEL) {
      cur_key = -1;
      if constexpr (SP) isel_task(p, t, ub, flags + 1, warp, lane, ctid, ab);
    } else if (MLA && t.op == OP_UK) {
      cur_key = -1;
      if constexpr (MLA)
        uk_task(p, t, gemv_geom<false>(p, t), gs, ns, ring, full, empty, tags, ub, red, warp, lane, ctid, ab);
    } else {
      const GemvGeom g = gemv_geom<TILED, F4>(p, t);
      const int key = input_key(t);
      float* resid = ub + p.xs_floats;  // residual rows of this task (O-proj, down)
      const bool has_resid = t.op == OP_O || t.op == OP_DOWN || t.op == OP_MO;
      if (has_resid) prefetch_resid<MT>(p, t, g, resid, ctid);
      if (MLA && t.op == OP_UV) {
        if constexpr (MLA) mla_combine_input(p, t, ub, ub + p.xs_floats, ctid);
        if (ctid == 0) *rn_s = 1.f;
        cur_key = -1;
      } else if (F8 && g.esz == 1 && (key != cur_key || key < 0)) {
        if constexpr (F8) {
          float rnv[1];
          load_input_e4m3(p, t, g, ub, red, ctid, rnv);
          if (ctid == 0) rn_s[0] = rnv[0];
        }
        cur_key = key;
      } else if (key != cur_key || key < 0) {
        float rnv[MT];
        load_input<MT, TILED>(p, t, g, ub, red, ctid, rnv);
        if (ctid == 0)
#pragma unroll
          for (int v = 0; v < MT; ++v) rn_s[v] = rnv[v];
        cur_key = key;
      }
      consumer_sync(kConsumerThreads);
      if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 4] = (long long)globaltimer_ns();
      float rnt[MT];
#pragma unroll
      for (int v = 0; v < MT; ++v) rnt[v] = rn_s[v];
      const float rn = rnt[0];
      const int K8 = g.Kp >> 3;
      const float4* xl = reinterpret_cast<const float4*>(ub);
      const float4* xh = reinterpret_cast<const float4*>(ub + g.Kp / 2);
      Best best[MT];
#pragma unroll
      for (int v = 0; v < MT; ++v) best[v] = Best{-INFINITY, 0x7fffffff};
      // routed experts: the slot's weight folds into u; u holds the shared slices first
      float wsel = 1.f;
      int uoff = 0;
      if (t.op == OP_RGU) {
        wsel = __ldcg(p.route_w + t.layer * p.topk + t.r0 / p.Fe);
        uoff = p.nshared * p.Fe;
      }
      if constexpr (TILED) {
        gemv_tile_task<MT>(p, t, g, gs, ns, ring, full, empty, tags, ub,
                           ub + p.ub_floats - kTileRedFloats, resid, rnt, wsel, uoff, best, warp,
                           lane, ctid, ab);
      }
      const bool coop = F8 && g.esz == 1;  // E4M3 stages: every warp takes part in each
      if constexpr (F8) {
        if (coop)
          fp8_task(p, t, g, gs, ns, ring, full, empty, tags, ub, resid, rn, wsel, uoff, warp,
                   lane, ctid, ab, best[0]);
      }
      // stage gs + i belongs to warp (gs + i) % 8; each warp takes its stages in order
      const int first = (int)((warp - (int)(gs % kConsumerWarps) + kConsumerWarps) % kConsumerWarps);
      for (int i = first; i < (TILED || coop ? 0 : ns); i += kConsumerWarps) {
        const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
        if (!stage_wait(p, full, tags, sidx)) {
          ab = true;
          break;
        }
        const int n0 = t.r0 + i * g.rps, nr = min(g.rps, t.r1 - n0);
        const uint4* sp = reinterpret_cast<const uint4*>(ring + (size_t)slot * p.stage_bytes);
        if (F4 && g.f4) {  // MXFP4 expert rows at their pitch (as the bf16 rows below)
          const uint8_t* sb = ring + (size_t)slot * p.stage_bytes;
          const size_t rb = (size_t)g.rowb;
          if (g.nseg == 2) {  // gate rows [0, nr), up rows at +rps rows
            for (int r = 0; r < nr; r += 2) {
              const int np = min(2, nr - r);
              const uint8_t* g0 = sb + (size_t)r * rb;
              const uint8_t* u0 = sb + (size_t)(g.rps + r) * rb;
              float o0, o1, o2, o3;
              if (np == 2) gemv_rows_e2m1<4>(g0, g0 + rb, u0, u0 + rb, g.Kp, xl, xh, lane, o0, o1, o2, o3);
              else gemv_rows_e2m1<2>(g0, u0, u0, u0, g.Kp, xl, xh, lane, o0, o1, o2, o3);
              const float v = reduce4(o0, o1, o2, o3, lane);
              const float upv = __shfl_xor_sync(0xffffffffu, v, np == 2 ? 16 : 8);
              const int k = (lane >> 3) & 1;
              if ((np == 2 && (lane & 23) == 0) || (np == 1 && lane == 0)) {
                const float a = v * rn, bb = upv * rn;
                p.u[uoff + n0 + r + k] = wsel * (a / (1.f + expf(-a)) * bb);
              }
            }
          } else {
            for (int r = 0; r < nr; r += 4) {
              const int nv = min(4, nr - r);
              const uint8_t* r0 = sb + (size_t)r * rb;
              float o0, o1, o2, o3;
              gemv_rows_e2m1_n(nv, r0, r0 + (size_t)min(1, nv - 1) * rb, r0 + (size_t)min(2, nv - 1) * rb,
                               r0 + (size_t)min(3, nv - 1) * rb, g.Kp, xl, xh, lane, o0, o1, o2, o3);
              const float v = reduce4(o0, o1, o2, o3, lane);
              const int idx = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
              if ((lane & 7) == 0 && idx < nv) gemv_emit<MLA>(p, t, g, n0 + r + idx, v, rn, resid, best[0]);
            }
          }
        } else if (MT == 1 && g.nseg == 2) {  // gate rows [0, nr), up rows at +rps rows
          const uint4* up = sp + (size_t)g.rps * K8;
          for (int r = 0; r < nr; r += 2) {
            const int np = min(2, nr - r);
            float o0, o1, o2, o3;
            const uint4* g0 = sp + (size_t)r * K8;
            const uint4* u0 = up + (size_t)r * K8;
            if (np == 2) {
              gemv_rows<4, 1>(g0, g0 + K8, u0, u0 + K8, K8, xl, xh, lane, o0, o1, o2, o3);
            } else {
              gemv_rows<2, 2>(g0, u0, u0, u0, K8, xl, xh, lane, o0, o1, o2, o3);
            }
            const float v = reduce4(o0, o1, o2, o3, lane);
            // np == 2: lanes 0 / 8 hold gate r / r+1, lanes 16 / 24 up r / r+1
            // np == 1: lane 0 holds gate r, lane 8 up r
            const float upv = __shfl_xor_sync(0xffffffffu, v, np == 2 ? 16 : 8);
            const int k = (lane >> 3) & 1;
            if ((np == 2 && (lane & 23) == 0) || (np == 1 && lane == 0)) {
              const float a = v * rn, bb = upv * rn;
              p.u[uoff + n0 + r + k] = wsel * (a / (1.f + expf(-a)) * bb);
            }
          }
        } else if (MT == 1) {
          for (int r = 0; r < nr; r += 4) {
            const int nv = min(4, nr - r);
            const uint4* r0 = sp + (size_t)r * K8;
            float o0, o1, o2, o3;
            gemv_rows_n(nv, r0, r0 + (size_t)min(1, nv - 1) * K8, r0 + (size_t)min(2, nv - 1) * K8,
                        r0 + (size_t)min(3, nv - 1) * K8, K8, xl, xh, lane, o0, o1, o2, o3);
            const float v = reduce4(o0, o1, o2, o3, lane);
            const int idx = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
            if ((lane & 7) == 0 && idx < nv) gemv_emit<MLA>(p, t, g, n0 + r + idx, v, rn, resid, best[0]);
          }
        } else if (TILED) {
        } else if (g.nseg == 2) {  // MT tokens: gate / up rows as above, per token
          const uint4* up = sp + (size_t)g.rps * K8;
          const int vs = g.Kp / 4;  // float4 stride between the tokens' planes
          for (int r = 0; r < nr; r += 2) {
            const int np = min(2, nr - r);
            float out[MT][4];
            const uint4* g0 = sp + (size_t)r * K8;
            const uint4* u0 = up + (size_t)r * K8;
            if (np == 2) gemv_rows_mt<4, MT>(g0, g0 + K8, u0, u0 + K8, K8, xl, xh, vs, lane, out);
            else gemv_rows_mt<2, MT>(g0, u0, u0, u0, K8, xl, xh, vs, lane, out);
#pragma unroll
            for (int v = 0; v < MT; ++v) {
              const float val = reduce4(out[v][0], out[v][1], out[v][2], out[v][3], lane);
              const float upv = __shfl_xor_sync(0xffffffffu, val, np == 2 ? 16 : 8);
              const int k = (lane >> 3) & 1;
              if ((np == 2 && (lane & 23) == 0) || (np == 1 && lane == 0)) {
                const float a = val * rnt[v], bb = upv * rnt[v];
                p.u[(size_t)v * p.F + uoff + n0 + r + k] = wsel * (a / (1.f + expf(-a)) * bb);
              }
            }
          }
        } else {
          const int vs = g.Kp / 4;
          for (int r = 0; r < nr; r += 4) {
            const int nv = min(4, nr - r);
            const uint4* r0 = sp + (size_t)r * K8;
            float out[MT][4];
            gemv_rows_mt_n<MT>(nv, r0, r0 + (size_t)min(1, nv - 1) * K8, r0 + (size_t)min(2, nv - 1) * K8,
                               r0 + (size_t)min(3, nv - 1) * K8, K8, xl, xh, vs, lane, out);
            const int idx = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
#pragma unroll
            for (int v = 0; v < MT; ++v) {
              const float val = reduce4(out[v][0], out[v][1], out[v][2], out[v][3], lane);
              if ((lane & 7) == 0 && idx < nv)
                gemv_emit<MLA>(p, t, g, n0 + r + idx, val, rnt[v], resid + v * kMaxResidRows, best[v], v);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_n(&empty[slot], kConsumerWarps);
      }
      if (t.op == OP_LM) {
#pragma unroll
        for (int v = 0; v < MT; ++v) {
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) {
            Best o;
            o.v = __shfl_xor_sync(0xffffffffu, best[v].v, off);
            o.i = __shfl_xor_sync(0xffffffffu, best[v].i, off);
            best_update(best[v], o.v, o.i);
          }
          if (lane == 0) {
            red[warp * MT + v] = best[v].v;
            reinterpret_cast<int*>(red)[32 + warp * MT + v] = best[v].i;
          }
        }
      }
      consumer_sync(kConsumerThreads);
      if (ctid == 0 && p.trace) p.trace[(size_t)t.id * kTraceCols + 5] = (long long)globaltimer_ns();
      if (t.op == OP_LM && ctid == 0) {  // per token: this task's best, then the last task
#pragma unroll
        for (int v = 0; v < MT; ++v) {
          Best bb{-INFINITY, 0x7fffffff};
          for (int w = 0; w < kConsumerWarps; ++w)
            best_update(bb, red[w * MT + v], reinterpret_cast<int*>(red)[32 + w * MT + v]);
          atomicMax(p.argmax_slot + v, pack_best(bb));
        }
        const uint32_t old = ticket_add(p.lm_ticket, 1u);
        if (((old + 1u) % (uint32_t)t.aux) == 0u) {
#pragma unroll
          for (int v = 0; v < MT; ++v) {
            const unsigned long long w = atomicExch(p.argmax_slot + v, 0ull);
            if (p.token_out) p.token_out[v] = (int32_t)(0xffffffffu - (uint32_t)(w & 0xffffffffull));
          }
        }
      }
      if (t.op == OP_ROUTER) {  // the last router task of the layer selects the experts
        if (ctid == 0) {
          const uint32_t old = ticket_add(p.router_ticket, 1u);
          flags[1] = ((old + 1u) % (uint32_t)t.aux) == 0u;
        }
        consumer_sync(kConsumerThreads);
        if (flags[1]) route_topk(p, t.layer, ub + p.xs_floats, warp, lane, ctid);
      } else if (t.op == OP_MOS) {  // the block's last slice sums the partial rows
        const int np = (t.aux >> 16) & 0xff;
        if (ctid == 0) {
          const uint32_t old = ticket_add(p.down_tickets + ((t.aux >> 8) & 0xff), 1u);
          flags[1] = ((old + 1u) % (uint32_t)np) == 0u;
        }
        consumer_sync(kConsumerThreads);
        if (flags[1]) mo_slices_combine(p, t, np, ctid);
      } else if (t.op == OP_MDOWN) {  // the block's last slot sums the partial rows
        if (ctid == 0) {
          const uint32_t old = ticket_add(p.down_tickets + (t.aux >> 8), 1u);
          flags[1] = ((old + 1u) % (uint32_t)(p.nshared + p.topk)) == 0u;
        }
        consumer_sync(kConsumerThreads);
        if (flags[1]) moe_down_combine(p, t, ctid);
      } else if (ctid == 0 && t.out >= 0) {
        publish_add(p.counters + (size_t)t.out * kCtrStride, 1u);
      }
    }
    if (ctid == 0) {
      if (p.trace) p.trace[(size_t)t.id * kTraceCols + 2] = (long long)globaltimer_ns();
      *reinterpret_cast<volatile int*>(misc + 80) = ti + 1;  // tasks finished (producer reads)
    }
    gs += (uint32_t)ns;
  }
}

// ---- the kernel ----------------------------------------------------------------------------------
template <bool MLA, int MT, bool TILED, bool F8 = false, bool SP = false, bool F4 = false>
__global__ void __launch_bounds__(kThreads, 1) engine_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t NS = (uint32_t)p.ring_stages;
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)NS * p.stage_bytes);
  uint64_t* empty = full + NS;
  uint32_t* tags = reinterpret_cast<uint32_t*>(empty + NS);
  const size_t bar_bytes = ((2 * NS * 8 + NS * 4 + 127) / 128) * 128;
  float* ub = reinterpret_cast<float*>(smem + (size_t)NS * p.stage_bytes + bar_bytes);
  float* misc = ub + p.ub_floats;  // the union buffer covers the input planes and attention scratch

  const int b = blockIdx.x;
  const Task* my;
  int ntask;
  if (p.op_group >= 0) {  // kernel-per-op form: this CTA's tasks of one op
    const int32_t* r = p.op_ranges + 2 * ((size_t)p.op_group * gridDim.x + b);
    my = p.tasks + r[0];
    ntask = r[1] - r[0];
    if (ntask == 0) return;
  } else {
    my = p.tasks + p.sm_begin[b];
    ntask = p.sm_begin[b + 1] - p.sm_begin[b];
  }
  // the swizzled latent tiles assume 1024-byte aligned ring slots
  if (p.KL > 0 && (smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) record_error(p, TRE_ERR_BOUNDS, -3);
    return;
  }

  if (threadIdx.x == 0) {
    *reinterpret_cast<volatile int*>(misc + 80) = 0;
    for (uint32_t i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);                 // the producer's arrive + the copies' bytes
      mbar_init(&empty[i], kConsumerWarps);   // 8 arrivals: all warps, or one warp's 8
      tags[i] = 0xffffffffu;
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) {
    producer<TILED, MLA, SP, F4>(p, my, ntask, ring, full, empty, tags,
             reinterpret_cast<const volatile int*>(misc + 80), threadIdx.x & 31);
    return;
  }
  consumer<MLA, MT, TILED, F8, SP, F4>(p, my, ntask, ring, full, empty, tags, ub, misc);
}

// ---- host-side launch helpers ------------------------------------------------------------------
// The kernel instantiation for a stack kind, a number of tokens per step, the GEMV stage
// form (tiled: multi-token tensor-core tiles) and the weight format (fp8: E4M3 projections
// on the tensor cores; fp4: MXFP4 routed experts; their own instantiations keep the bf16
// kernel's code and registers as they are).
static const void* kernel_for(bool mla, int m, bool tiled, bool fp8 = false, bool sparse = false,
                              bool fp4 = false) {
  if (mla && sparse) return reinterpret_cast<const void*>(engine_kernel<true, 1, false, false, true>);
  if (mla) return reinterpret_cast<const void*>(engine_kernel<true, 1, false>);
  if (fp8) return reinterpret_cast<const void*>(engine_kernel<false, 1, false, true>);
  if (fp4) return reinterpret_cast<const void*>(engine_kernel<false, 1, false, false, false, true>);
  if (tiled) {
    switch (m) {
      case 2: return reinterpret_cast<const void*>(engine_kernel<false, 2, true>);
      case 3: return reinterpret_cast<const void*>(engine_kernel<false, 3, true>);
      case 4: return reinterpret_cast<const void*>(engine_kernel<false, 4, true>);
      default: return reinterpret_cast<const void*>(engine_kernel<false, 1, true>);
    }
  }
  switch (m) {
    case 2: return reinterpret_cast<const void*>(engine_kernel<false, 2, false>);
    case 3: return reinterpret_cast<const void*>(engine_kernel<false, 3, false>);
    case 4: return reinterpret_cast<const void*>(engine_kernel<false, 4, false>);
    default: return reinterpret_cast<const void*>(engine_kernel<false, 1, false>);
  }
}

// Configure the instantiations a plan can launch (m = 1 .. max_m) and report how many
// CTAs of `smem_bytes` fit on an SM.  The shared-memory limit is a property of the kernel
// function shared by every engine in the process, so it is raised to the device maximum
// (never lowered to this plan's need: an engine created later must not shrink what an
// earlier one launches with).
cudaError_t engine_configure(int smem_bytes, int* blocks_per_sm, bool mla, int max_m, bool tiled,
                             bool fp8, bool sparse, bool fp4) {
  *blocks_per_sm = 1 << 30;
  int dev = 0, optin = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 == cudaSuccess)
    e0 = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e0 != cudaSuccess) return e0;
  const int limit = optin > smem_bytes ? optin : smem_bytes;
  for (int m = 1; m <= (mla || fp8 || fp4 ? 1 : max_m); ++m) {
    const void* k = kernel_for(mla, m, tiled, fp8, sparse, fp4);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
    if (e != cudaSuccess) return e;
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k, kThreads, smem_bytes);
    if (e != cudaSuccess) return e;
    *blocks_per_sm = b < *blocks_per_sm ? b : *blocks_per_sm;
  }
  return cudaSuccess;
}

// The persistent form is a cooperative launch (every CTA resident: tasks wait on other
// CTAs' counters); a kernel-per-op launch (p.op_group >= 0) is a plain one, since every
// dependency of its tasks was met by the launches before it.
cudaError_t engine_launch(const Params& p, int grid, int smem_bytes, cudaStream_t stream, bool mla) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.op_group >= 0 ? 0 : 1;
  void* args[] = {const_cast<Params*>(&p)};
  const cudaError_t e =
      cudaLaunchKernelExC(&cfg, kernel_for(mla, p.m, p.gemv_tiles != 0, p.wfp8 != 0, p.KI > 0, p.wfp4 != 0),
                          args);
  if (e != cudaSuccess) cudaGetLastError();  // returned here: do not leave it to the caller
  return e;
}

}  // namespace tre
