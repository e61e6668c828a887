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

// Wait until counter `t.dep` reaches epoch * t.dep_count (wrap-safe).  Bounded.
__device__ bool wait_dep(const Params& p, const Task& t) {
  if (t.dep < 0) return true;
  const uint32_t target = p.epoch * t.dep_count;
  const uint32_t* c = p.counters + t.dep;
  if ((int32_t)(ld_acquire_gpu(c) - target) >= 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if ((int32_t)(ld_acquire_gpu(c) - target) >= 0) return true;
    if ((it & 31) == 0) {
      if (aborted(p)) return false;
      if ((long long)(globaltimer_ns() - t0) > p.timeout_ns) {
        record_error(p, TRE_ERR_DEP_TIMEOUT, t.id);
        return false;
      }
    }
  }
}

// Bounded wait on an mbarrier phase; `slack` scales the time budget (ring waits get
// twice the dependency budget so that a dependency timeout is reported first).
__device__ bool mbar_wait(const Params& p, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15) == 0) {
      if (aborted(p)) return false;
      if ((long long)(globaltimer_ns() - t0) > 2 * p.timeout_ns) {
        record_error(p, TRE_ERR_DEP_TIMEOUT, -1);
        return false;
      }
    }
  }
}

// Wait for ring stage `sidx` to land.  Consumer warps take stages round-robin, so a warp
// can reach a slot before the slot's previous stage (sidx - NS) was even issued; a parity
// wait there would match the previous phase.  The producer therefore tags each slot with
// the stage it claimed (after that slot's previous stage was consumed, which implies its
// full-barrier phase completed); waiting for the tag first keeps every parity wait at most
// one phase ahead.
__device__ bool stage_wait(const Params& p, uint64_t* full, const uint32_t* tags, uint32_t sidx) {
  const uint32_t NS = (uint32_t)p.ring_stages, slot = sidx % NS;
  const volatile uint32_t* tag = tags + slot;
  if (*tag != sidx) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1; *tag != sidx; ++it) {
      if ((it & 63) == 0) {
        if (aborted(p)) return false;
        if ((long long)(globaltimer_ns() - t0) > 2 * p.timeout_ns) {
          record_error(p, TRE_ERR_DEP_TIMEOUT, -2);
          return false;
        }
      }
    }
  }
  return mbar_wait(p, &full[slot], (sidx / NS) & 1u);
}

// ---- task geometry (shared by producer and consumers) ---------------------------------------
__device__ __forceinline__ int gemv_K(const Params& p, int op) {
  return op == OP_O ? p.Hq * p.D : (op == OP_DOWN ? p.F : p.d);
}
__device__ __forceinline__ int gemv_nseg(int op) { return op == OP_GU ? 2 : 1; }
__device__ __forceinline__ int gemv_rps(const Params& p, int op) {
  const int r = p.stage_bytes / (gemv_nseg(op) * gemv_K(p, op) * 2);
  return r < 1 ? 1 : r;
}
__device__ __forceinline__ const uint16_t* gemv_w(const Params& p, int op, int layer, int seg) {
  if (op == OP_LM) return p.lm_head;
  const LayerPtrs& L = p.layers[layer];
  switch (op) {
    case OP_Q: return L.w[TRE_W_Q];
    case OP_K: return L.w[TRE_W_K];
    case OP_V: return L.w[TRE_W_V];
    case OP_O: return L.w[TRE_W_O];
    case OP_GU: return seg ? L.w[TRE_W_UP] : L.w[TRE_W_GATE];
    default: return L.w[TRE_W_DOWN];
  }
}

__device__ __forceinline__ void attn_range(const Params& p, const Task& t, int& t0, int& t1) {
  const long long P = p.pos;  // cached positions [0, pos); the new one comes from qkv
  t0 = (int)(P * t.r1 / t.aux);
  t1 = (int)(P * (t.r1 + 1) / t.aux);
}

__device__ __forceinline__ int task_nstages(const Params& p, const Task& t) {
  if (t.type == T_GEMV) {
    const int rps = gemv_rps(p, t.op);
    return (t.r1 - t.r0 + rps - 1) / rps;
  }
  int t0, t1;
  attn_range(p, t, t0, t1);
  return (t1 - t0 + p.pps - 1) / p.pps;
}

struct StageSrc {
  const uint8_t* src0;
  const uint8_t* src1;
  uint32_t bytes0, bytes1, off1;
};

__device__ __forceinline__ StageSrc stage_desc(const Params& p, const Task& t, int i) {
  StageSrc s;
  if (t.type == T_GEMV) {
    const int K = gemv_K(p, t.op), rps = gemv_rps(p, t.op);
    const int n0 = t.r0 + i * rps, nr = min(rps, t.r1 - n0);
    const size_t rowb = (size_t)K * 2;
    s.src0 = reinterpret_cast<const uint8_t*>(gemv_w(p, t.op, t.layer, 0)) + (size_t)n0 * rowb;
    s.bytes0 = (uint32_t)(nr * rowb);
    if (t.op == OP_GU) {
      s.src1 = reinterpret_cast<const uint8_t*>(gemv_w(p, t.op, t.layer, 1)) + (size_t)n0 * rowb;
      s.bytes1 = s.bytes0;
      s.off1 = (uint32_t)(rps * rowb);
    } else {
      s.src1 = nullptr;
      s.bytes1 = 0;
      s.off1 = 0;
    }
  } else {
    int t0, t1;
    attn_range(p, t, t0, t1);
    const int tt = t0 + i * p.pps, n = min(p.pps, t1 - tt);
    const size_t rowb = (size_t)p.D * 2;
    const LayerPtrs& L = p.layers[t.layer];
    const size_t off = ((size_t)t.r0 * p.cap + tt) * rowb;
    s.src0 = reinterpret_cast<const uint8_t*>(L.k_cache) + off;
    s.src1 = reinterpret_cast<const uint8_t*>(L.v_cache) + off;
    s.bytes0 = s.bytes1 = (uint32_t)(n * rowb);
    s.off1 = (uint32_t)(p.pps * rowb);
  }
  return s;
}

// ---- producer -------------------------------------------------------------------------------
__device__ void producer(const Params& p, const Task* my, int ntask, uint8_t* ring,
                         uint64_t* full, uint64_t* empty, uint32_t* tags) {
  const uint64_t pol = l2_policy_evict_first();
  const uint32_t NS = (uint32_t)p.ring_stages;
  const uint32_t SB = (uint32_t)p.stage_bytes;
  uint32_t gs = 0;
  bool ok = true;
  for (int ti = 0; ti < ntask && ok; ++ti) {
    const Task t = my[ti];
    if ((p.flags & TRE_DEBUG_NO_OVERLAP) && !wait_dep(p, t)) {
      ok = false;
      break;
    }
    const int ns = task_nstages(p, t);
    for (int i = 0; i < ns; ++i, ++gs) {
      const uint32_t slot = gs % NS, ph = (gs / NS) & 1u;
      if (!mbar_wait(p, &empty[slot], ph ^ 1u)) {
        ok = false;
        break;
      }
      const StageSrc s = stage_desc(p, t, i);
      *reinterpret_cast<volatile uint32_t*>(tags + slot) = gs;
      mbar_arrive_expect_tx(&full[slot], s.bytes0 + s.bytes1);
      bulk_g2s(ring + (size_t)slot * SB, s.src0, s.bytes0, &full[slot], pol);
      if (s.bytes1) bulk_g2s(ring + (size_t)slot * SB + s.off1, s.src1, s.bytes1, &full[slot], pol);
    }
  }
  if (!ok) {
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

__device__ __forceinline__ float resid_in(const Params& p, int layer, int n) {
  if (layer > 0) return __ldcg(p.x + n);
  if (p.x_in) return __ldcg(p.x_in + n);
  return bf_lo(p.embed[(size_t)p.token * p.d + n]);
}

// Input-vector identity for reuse across consecutive tasks (same layer, same source).
__device__ __forceinline__ int input_key(const Task& t) {
  int cls;
  switch (t.op) {
    case OP_Q: case OP_K: case OP_V: cls = 0; break;
    case OP_O: cls = 1; break;
    case OP_GU: cls = 2; break;
    case OP_DOWN: cls = 3; break;
    default: cls = 4; break;
  }
  return (int)t.layer * 8 + cls;
}

// Stage the GEMV input into the two planes; returns the RMSNorm scale (1 when none).
__device__ float load_input(const Params& p, const Task& t, float* xlo, float* xhi, float* red,
                            int ctid) {
  const int K = gemv_K(p, t.op);
  const float* src = nullptr;
  const uint16_t* src_bf = nullptr;
  const uint16_t* gain = nullptr;
  switch (t.op) {
    case OP_Q: case OP_K: case OP_V:
      gain = p.layers[t.layer].w[TRE_W_ATTN_NORM];
      if (t.layer > 0) src = p.x;
      else if (p.x_in) src = p.x_in;
      else src_bf = p.embed + (size_t)p.token * p.d;
      break;
    case OP_O: src = p.attn; break;
    case OP_GU: src = p.h1; gain = p.layers[t.layer].w[TRE_W_FFN_NORM]; break;
    case OP_DOWN: src = p.u; break;
    default: src = p.x; gain = p.final_norm; break;
  }
  float ss = 0.f;
  const int K8 = K >> 3;
  for (int j = ctid; j < K8; j += kConsumerThreads) {
    float v[8];
    if (src_bf) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(src_bf) + j);
      v[0] = bf_lo(w.x); v[1] = bf_hi(w.x); v[2] = bf_lo(w.y); v[3] = bf_hi(w.y);
      v[4] = bf_lo(w.z); v[5] = bf_hi(w.z); v[6] = bf_lo(w.w); v[7] = bf_hi(w.w);
    } else {
      const float4 a = __ldcg(reinterpret_cast<const float4*>(src) + 2 * j);
      const float4 b = __ldcg(reinterpret_cast<const float4*>(src) + 2 * j + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    if (gain) {
#pragma unroll
      for (int k = 0; k < 8; ++k) ss = fmaf(v[k], v[k], ss);
      const uint4 g = __ldg(reinterpret_cast<const uint4*>(gain) + j);
      v[0] *= bf_lo(g.x); v[1] *= bf_hi(g.x); v[2] *= bf_lo(g.y); v[3] *= bf_hi(g.y);
      v[4] *= bf_lo(g.z); v[5] *= bf_hi(g.z); v[6] *= bf_lo(g.w); v[7] *= bf_hi(g.w);
    }
    reinterpret_cast<float4*>(xlo)[j] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(xhi)[j] = make_float4(v[4], v[5], v[6], v[7]);
  }
  float rn = 1.f;
  if (gain) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((ctid & 31) == 0) red[ctid >> 5] = ss;
  }
  consumer_sync(kConsumerThreads);
  if (gain) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += red[w];
    rn = 1.f / sqrtf(tot / (float)K + p.eps);
  }
  return rn;
}

// ---- attention task ----------------------------------------------------------------------------
__device__ __forceinline__ void rope_cs(const Params& p, int i, float& c, float& s) {
  const double ang = (double)p.pos * p.rope_inv_freq[i];
  const double two_pi = 6.283185307179586476925286766559;
  const double red = ang - two_pi * rint(ang / two_pi);
  sincosf((float)red, &s, &c);
}

template <int G, int DPL>
__device__ void attn_task(const Params& p, const Task& t, uint32_t gs, int ns, uint8_t* ring,
                          uint64_t* full, uint64_t* empty, const uint32_t* tags, float* ub,
                          float* red, int* flag, int warp, int lane, int ctid, bool& abort_out) {
  constexpr int D = 32 * DPL;
  const int g = t.r0, split = t.r1, S = t.aux;
  const bool last = (split == S - 1);
  float* q_s = ub;                            // [G][D] roped, scaled
  float* kn_s = q_s + G * D;                  // [D]   new k (bf16 value)
  float* vn_s = kn_s + D;                     // [D]   new v (bf16 value)
  float* mw = vn_s + D;                       // [warps][G]
  float* lw = mw + kConsumerWarps * G;        // [warps][G]
  float* ow = lw + kConsumerWarps * G;        // [warps][G][D]
  float* sn = ow + kConsumerWarps * G * D;    // [G] score of the new position
  const float qscale = 1.4426950408889634f / sqrtf((float)D);

  const float* qsrc = p.qkv + (size_t)g * G * D;
  for (int idx = ctid; idx < G * (D / 2); idx += kConsumerThreads) {
    const int h = idx / (D / 2), i = idx % (D / 2);
    const float x0 = __ldcg(qsrc + h * D + i), x1 = __ldcg(qsrc + h * D + i + D / 2);
    float c, s;
    rope_cs(p, i, c, s);
    q_s[h * D + i] = (x0 * c - x1 * s) * qscale;
    q_s[h * D + i + D / 2] = (x0 * s + x1 * c) * qscale;
  }
  if (last) {
    const float* ksrc = p.qkv + (size_t)p.Hq * D + (size_t)g * D;
    const float* vsrc = ksrc + (size_t)p.Hkv * D;
    const LayerPtrs& L = p.layers[t.layer];
    __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(L.k_cache) + ((size_t)g * p.cap + p.pos) * D;
    __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(L.v_cache) + ((size_t)g * p.cap + p.pos) * D;
    for (int i = ctid; i < D / 2; i += kConsumerThreads) {
      const float x0 = __ldcg(ksrc + i), x1 = __ldcg(ksrc + i + D / 2);
      float c, s;
      rope_cs(p, i, c, s);
      const __nv_bfloat16 k0 = __float2bfloat16_rn(x0 * c - x1 * s);
      const __nv_bfloat16 k1 = __float2bfloat16_rn(x0 * s + x1 * c);
      kc[i] = k0;
      kc[i + D / 2] = k1;
      kn_s[i] = __bfloat162float(k0);
      kn_s[i + D / 2] = __bfloat162float(k1);
    }
    for (int i = ctid; i < D; i += kConsumerThreads) {
      const __nv_bfloat16 v = __float2bfloat16_rn(__ldcg(vsrc + i));
      vc[i] = v;
      vn_s[i] = __bfloat162float(v);
    }
  }
  consumer_sync(kConsumerThreads);

  if (last && warp < G) {  // score of the new position for head `warp`
    float a = 0.f;
    for (int i = lane; i < D; i += 32) a = fmaf(q_s[warp * D + i], kn_s[i], a);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (lane == 0) sn[warp] = a;
  }

  float q[G][DPL], m[G], l[G], o[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      q[h][j] = q_s[h * D + lane * DPL + j];
      o[h][j] = 0.f;
    }
  }
  const uint32_t NS = (uint32_t)p.ring_stages;
  int t0, t1;
  attn_range(p, t, t0, t1);
  const int first = (int)((warp - (int)(gs % kConsumerWarps) + kConsumerWarps) % kConsumerWarps);
  for (int i = first; i < ns; i += kConsumerWarps) {
    const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
    if (!stage_wait(p, full, tags, sidx)) {
      abort_out = true;
      break;
    }
    const int tt = t0 + i * p.pps, n = min(p.pps, t1 - tt);
    const uint8_t* kb = ring + (size_t)slot * p.stage_bytes;
    attn_stage<G, DPL>(kb, kb + (size_t)p.pps * D * 2, n, q, m, l, o, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (lane == 0) {
      mw[warp * G + h] = m[h];
      lw[warp * G + h] = l[h];
    }
#pragma unroll
    for (int j = 0; j < DPL; ++j) ow[(warp * G + h) * D + lane * DPL + j] = o[h][j];
  }
  consumer_sync(kConsumerThreads);

  // merge the warps (and the new position) into this split's partial
  const size_t pstride = (size_t)D + 2;
  for (int idx = ctid; idx < G * D; idx += kConsumerThreads) {
    const int h = idx / D, dd = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mw[w * G + h]);
    const float snew = last ? sn[h] : -INFINITY;
    M = fmaxf(M, snew);
    float O = 0.f, Ls = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mv = mw[w * G + h];
        if (mv != -INFINITY) {
          const float sc = exp2f(mv - M);
          O = fmaf(sc, ow[(w * G + h) * D + dd], O);
          Ls = fmaf(sc, lw[w * G + h], Ls);
        }
      }
      if (last) {
        const float pn = exp2f(snew - M);
        O = fmaf(pn, vn_s[dd], O);
        Ls += pn;
      }
    }
    float* dst = p.part + ((size_t)(g * G + h) * S + split) * pstride;
    dst[dd] = O;
    if (dd == 0) {
      dst[D] = M;
      dst[D + 1] = Ls;
    }
  }
  __threadfence();
  consumer_sync(kConsumerThreads);
  if (ctid == 0) {
    const uint32_t old = atom_acq_rel_gpu_add(p.tickets + g, 1u);
    *flag = ((old + 1u) % (uint32_t)S) == 0u;
  }
  consumer_sync(kConsumerThreads);
  if (*flag) {  // last split of this kv head to finish: combine all splits
    for (int idx = ctid; idx < G * D; idx += kConsumerThreads) {
      const int h = idx / D, dd = idx % D;
      const float* src = p.part + (size_t)(g * G + h) * S * pstride;
      float M = -INFINITY;
      for (int s2 = 0; s2 < S; ++s2) M = fmaxf(M, __ldcg(src + s2 * pstride + D));
      float O = 0.f, Ls = 0.f;
      for (int s2 = 0; s2 < S; ++s2) {
        const float ms = __ldcg(src + s2 * pstride + D);
        if (ms != -INFINITY) {
          const float sc = exp2f(ms - M);
          O = fmaf(sc, __ldcg(src + s2 * pstride + dd), O);
          Ls = fmaf(sc, __ldcg(src + s2 * pstride + D + 1), Ls);
        }
      }
      p.attn[(size_t)(g * G + h) * D + dd] = O / Ls;
    }
    __threadfence();
    consumer_sync(kConsumerThreads);
    if (ctid == 0) red_release_gpu_add(p.counters + t.out, 1u);
  }
}

__device__ __forceinline__ void run_attn(const Params& p, const Task& t, uint32_t gs, int ns,
                                         uint8_t* ring, uint64_t* full, uint64_t* empty,
                                         const uint32_t* tags, float* ub, float* red, int* flag,
                                         int warp, int lane, int ctid, bool& ab) {
  const int G = p.Hq / p.Hkv;
  if (p.D == 128) {
    switch (G) {
      case 1: attn_task<1, 4>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
      case 2: attn_task<2, 4>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
      case 4: attn_task<4, 4>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
      default: attn_task<8, 4>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
    }
  } else {
    switch (G) {
      case 1: attn_task<1, 2>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
      case 2: attn_task<2, 2>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
      case 4: attn_task<4, 2>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
      default: attn_task<8, 2>(p, t, gs, ns, ring, full, empty, tags, ub, red, flag, warp, lane, ctid, ab); break;
    }
  }
}

// ---- consumers -----------------------------------------------------------------------------------
__device__ void consumer(const Params& p, const Task* my, int ntask, uint8_t* ring,
                         uint64_t* full, uint64_t* empty, const uint32_t* tags, float* ub,
                         float* misc) {
  const int ctid = threadIdx.x, warp = ctid >> 5, lane = ctid & 31;
  float* red = misc;                                      // [32] reductions
  int* flags = reinterpret_cast<int*>(misc + 32);         // [0] abort, [1] ticket
  float* rn_s = misc + 40;
  const uint32_t NS = (uint32_t)p.ring_stages;
  const int half = p.xs_floats / 2;
  float* xlo = ub;
  float* xhi = ub + half;
  uint32_t gs = 0;
  int cur_key = -1;
  bool ab = false;
  for (int ti = 0; ti < ntask; ++ti) {
    const Task t = my[ti];
    const int ns = task_nstages(p, t);
    if (ctid == 0) {
      long long* tr = p.trace ? p.trace + (size_t)t.id * 4 : nullptr;
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

    if (t.type == T_ATTN) {
      cur_key = -1;  // the attention scratch aliases the input-vector planes
      run_attn(p, t, gs, ns, ring, full, empty, tags, ub, red, flags + 1, warp, lane, ctid, ab);
    } else {
      const int key = input_key(t);
      if (key != cur_key) {
        const float rn = load_input(p, t, xlo, xhi, red, ctid);
        if (ctid == 0) *rn_s = rn;
        consumer_sync(kConsumerThreads);
        cur_key = key;
      }
      const float rn = *rn_s;
      const int op = t.op, K = gemv_K(p, op), K8 = K >> 3, rps = gemv_rps(p, op);
      const float4* xl = reinterpret_cast<const float4*>(xlo);
      const float4* xh = reinterpret_cast<const float4*>(xhi);
      Best best{-INFINITY, 0x7fffffff};
      const int first = (int)((warp - (int)(gs % kConsumerWarps) + kConsumerWarps) % kConsumerWarps);
      for (int i = first; i < ns; i += kConsumerWarps) {
        const uint32_t sidx = gs + (uint32_t)i, slot = sidx % NS;
        if (!stage_wait(p, full, tags, sidx)) {
          ab = true;
          break;
        }
        const uint8_t* sp = ring + (size_t)slot * p.stage_bytes;
        const int n0 = t.r0 + i * rps, nr = min(rps, t.r1 - n0);
        if (op == OP_GU) {
          gemv_stage_pairs(sp, (size_t)rps * K * 2, K8, nr, xl, xh, lane,
                           [&](int r, float gt, float up) {
                             const float a = gt * rn, b = up * rn;
                             p.u[n0 + r] = a / (1.f + expf(-a)) * b;
                           });
        } else {
          gemv_stage_rows(sp, K8, nr, xl, xh, lane, [&](int r, float v) {
            const int n = n0 + r;
            switch (op) {
              case OP_Q: p.qkv[n] = v * rn; break;
              case OP_K: p.qkv[(size_t)p.Hq * p.D + n] = v * rn; break;
              case OP_V: p.qkv[(size_t)(p.Hq + p.Hkv) * p.D + n] = v * rn; break;
              case OP_O: p.h1[n] = resid_in(p, t.layer, n) + v; break;
              case OP_DOWN: {
                const float y = __ldcg(p.h1 + n) + v;
                p.x[n] = y;
                if (p.hidden) p.hidden[(size_t)t.layer * p.d + n] = y;
                if (p.x_out && t.layer == p.L - 1) p.x_out[n] = y;
              } break;
              default: {
                const float y = v * rn;
                p.logits[n] = y;
                best_update(best, y, n);
              } break;
            }
          });
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      if (op == OP_LM) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          Best o;
          o.v = __shfl_xor_sync(0xffffffffu, best.v, off);
          o.i = __shfl_xor_sync(0xffffffffu, best.i, off);
          best_update(best, o.v, o.i);
        }
        if (lane == 0) {
          red[warp] = best.v;
          reinterpret_cast<int*>(red)[16 + warp] = best.i;
        }
      }
      __threadfence();
      consumer_sync(kConsumerThreads);
      if (op == OP_LM && ctid == 0) {
        Best b{-INFINITY, 0x7fffffff};
        for (int w = 0; w < kConsumerWarps; ++w) best_update(b, red[w], reinterpret_cast<int*>(red)[16 + w]);
        atomicMax(p.argmax_slot, pack_best(b));
        __threadfence();
        const uint32_t old = atom_acq_rel_gpu_add(p.lm_ticket, 1u);
        if (((old + 1u) % (uint32_t)t.aux) == 0u) {
          const unsigned long long w = atomicExch(p.argmax_slot, 0ull);
          if (p.token_out) *p.token_out = (int32_t)(0xffffffffu - (uint32_t)(w & 0xffffffffull));
        }
      }
      if (ctid == 0 && t.out >= 0) red_release_gpu_add(p.counters + t.out, 1u);
    }
    if (ctid == 0 && p.trace) p.trace[(size_t)t.id * 4 + 2] = (long long)globaltimer_ns();
    gs += (uint32_t)ns;
  }
}

// ---- the kernel ----------------------------------------------------------------------------------
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
  const Task* my = p.tasks + p.sm_begin[b];
  const int ntask = p.sm_begin[b + 1] - p.sm_begin[b];

  if (threadIdx.x == 0) {
    for (uint32_t i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      tags[i] = 0xffffffffu;
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) {
    if (threadIdx.x == kConsumerThreads) producer(p, my, ntask, ring, full, empty, tags);
    return;
  }
  consumer(p, my, ntask, ring, full, empty, tags, ub, misc);
}

// ---- host-side launch helpers ------------------------------------------------------------------
cudaError_t engine_configure(int smem_bytes, int* blocks_per_sm) {
  cudaError_t e = cudaFuncSetAttribute(engine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_bytes);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, engine_kernel, kThreads,
                                                       smem_bytes);
}

cudaError_t engine_launch(const Params& p, int grid, int smem_bytes, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, engine_kernel, p);
}

}  // namespace tre
