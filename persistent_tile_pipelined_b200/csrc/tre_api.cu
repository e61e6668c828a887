// C ABI of the engine (declared in include/tre.h): create / step / status / destroy.
//
// The caller owns weights, KV caches and streams (the pages' inject_cache() likewise
// takes an external KV cache as raw tensors — TileRT code audit, KV-cache section); the
// engine owns its plan, counters and activation scratch.  One decode step is one
// cooperative launch of the persistent kernel (Static Compilation for LLM Inference, §1).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "tre_internal.h"

namespace tre {
cudaError_t engine_configure(int smem_bytes, int* blocks_per_sm, bool mla, int max_m, bool tiled,
                             bool fp8 = false, bool sparse = false, bool fp4 = false);
cudaError_t engine_launch(const Params& p, int grid, int smem_bytes, cudaStream_t stream,
                          bool mla = false);
const char* last_error_cstr();
}  // namespace tre

using namespace tre;

struct tre_engine {
  tre_config cfg;
  int device = 0;
  PlanShape shape{};
  int n_tasks = 0;
  uint32_t epoch = 0;
  cudaStream_t last_stream = nullptr;
  void* block = nullptr;         // one device allocation for all engine-owned state
  size_t block_bytes = 0;
  int32_t* status_host = nullptr;  // mapped pinned [4]
  int32_t* status_dev = nullptr;
  Params base{};
  int32_t* token_buf = nullptr;
  int last_m = 1;                // tokens of the last step (debug hidden layout)
  float* logits_buf = nullptr;
  int n_groups = 0;              // op groups of the plan (kernel-per-op form)
  uint32_t* op_counters = nullptr;  // counters the kernel-per-op launches bump
  int launch_mode = TRE_LAUNCH_PERSISTENT;
  std::vector<uint32_t> expected;  // per counter: increments per step (0: no task waits on it)
  std::vector<size_t> guards;      // offsets of the guard words after every owned buffer
};

#define TRE_EXPORT extern "C" __attribute__((visibility("default")))

static tre_status cuda_fail(cudaError_t e, const char* what) {
  set_error(std::string(what) + ": " + cudaGetErrorString(e));
  return TRE_ERR_CUDA;
}

#define CK(call)                                          \
  do {                                                    \
    cudaError_t _e = (call);                              \
    if (_e != cudaSuccess) return cuda_fail(_e, #call);   \
  } while (0)

static bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

// cuTensorMapEncodeTiled from the driver, looked up through the runtime (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// A cache [rows][C] bf16 as a 2-D tensor; boxes of 64 columns x box_rows rows with the
// 128-byte swizzle the attention tiles read (rows past the cache read as zero).
namespace tre {
tre_status encode_cache_map(void* cache, int C, long long rows, int box_rows, void* out128) {
  CUtensorMap* out = static_cast<CUtensorMap*>(out128);
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f) {
      set_error("cuTensorMapEncodeTiled is not available");
      return TRE_ERR_CUDA;
    }
    fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)C * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kMlaBox, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cache, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")");
    return TRE_ERR_CUDA;
  }
  return TRE_OK;
}
}  // namespace tre

namespace {
constexpr size_t kGuardBytes = 64;       // guard words after every engine-owned buffer
constexpr unsigned char kGuardFill = 0x5A;

struct Carve {  // bump allocator over the engine's single device block
  size_t off = 0;
  std::vector<size_t> guards;
  template <class T>
  size_t take(size_t count) {
    off = (off + 255) & ~size_t(255);
    size_t at = off;
    off += count * sizeof(T);
    guards.push_back(off);  // kGuardBytes of fill pattern right after the buffer
    off += kGuardBytes;
    return at;
  }
};
}  // namespace

TRE_EXPORT const char* tre_last_error(void) { return last_error_cstr(); }

TRE_EXPORT tre_status tre_plan_inspect(const tre_config* cfg, int32_t num_sms,
                                       int32_t smem_per_block, tre_plan_info* info) {
  if (!cfg || !info) {
    set_error("tre_plan_inspect: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  PlanShape s;
  std::vector<Task> tasks;
  std::vector<int32_t> begin;
  std::vector<int64_t> bytes;
  int nsm = cfg->num_sms ? std::min<int>(cfg->num_sms, num_sms) : num_sms;
  tre_status st = plan_build(*cfg, nsm, smem_per_block, &s, &tasks, &begin, &bytes);
  if (st != TRE_OK) return st;
  std::memset(info, 0, sizeof(*info));
  info->num_sms = s.nsm;
  info->num_tasks = (int32_t)tasks.size();
  info->num_counters = s.n_counters;
  info->kv_splits = s.kv_splits;
  info->ring_stages = s.ring_stages;
  info->stage_bytes = s.stage_bytes;
  info->smem_bytes = s.smem_bytes;
  int mx = 0;
  for (int i = 0; i < s.nsm; ++i) mx = std::max(mx, begin[i + 1] - begin[i]);
  info->max_tasks_per_sm = mx;
  info->gemv_tiles = s.tiles;
  info->index_splits = s.isplits;
  const int64_t row_new = s.kind == TRE_LAYER_MLA ? (int64_t)(s.KL + s.R) * 2 : (int64_t)s.Hkv * s.D * 4;
  const int64_t row_read = s.kind == TRE_LAYER_MLA ? (int64_t)(s.KL + s.R) * 2 : (int64_t)s.Hkv * s.D * 4;
  info->weight_bytes = step_bytes(s, 0) - (int64_t)s.L * (row_new + (int64_t)s.DI * 2) -
                       (s.has_lm ? (int64_t)s.V * 4 + 2LL * s.d : 0);
  info->kv_bytes_at_capacity = (int64_t)s.L * (int64_t)(s.cap - s.M) * row_read;
  if (s.KI)  // sparse MLA: every index key, and only the K chosen latent rows
    info->kv_bytes_at_capacity = (int64_t)s.L * ((int64_t)(s.cap - 1) * s.DI * 2 +
                                                 (int64_t)std::min(s.KI, s.cap - 1) * row_read);
  int64_t lo = INT64_MAX, hi = 0;
  for (int64_t b : bytes) {
    lo = std::min(lo, b);
    hi = std::max(hi, b);
  }
  info->max_sm_bytes = hi;
  info->min_sm_bytes = lo;
  return TRE_OK;
}

// Dump the planned task descriptors (8 int32 per task, the Task layout) and the per-SM
// queue offsets; returns the task count (or a negative tre_status).  Host only.
TRE_EXPORT int32_t tre_plan_tasks(const tre_config* cfg, int32_t num_sms, int32_t smem_per_block,
                       int32_t* out_tasks, int32_t max_tasks, int32_t* out_sm_begin) {
  if (!cfg) return TRE_ERR_INVALID_ARG;
  PlanShape s;
  std::vector<Task> tasks;
  std::vector<int32_t> begin;
  int nsm = cfg->num_sms ? std::min<int>(cfg->num_sms, num_sms) : num_sms;
  tre_status st = plan_build(*cfg, nsm, smem_per_block, &s, &tasks, &begin, nullptr);
  if (st != TRE_OK) return st;
  if (out_tasks && max_tasks >= (int32_t)tasks.size())
    std::memcpy(out_tasks, tasks.data(), tasks.size() * sizeof(Task));
  if (out_sm_begin) std::memcpy(out_sm_begin, begin.data(), begin.size() * sizeof(int32_t));
  return (int32_t)tasks.size();
}

TRE_EXPORT int32_t tre_plan_op_groups(const tre_config* cfg, int32_t num_sms,
                                      int32_t smem_per_block, int32_t* out_ranges,
                                      int32_t max_groups) {
  if (!cfg) return TRE_ERR_INVALID_ARG;
  PlanShape s;
  std::vector<Task> tasks;
  std::vector<int32_t> begin, ranges;
  int nsm = cfg->num_sms ? std::min<int>(cfg->num_sms, num_sms) : num_sms;
  tre_status st = plan_build(*cfg, nsm, smem_per_block, &s, &tasks, &begin, nullptr);
  if (st != TRE_OK) return st;
  const int G = plan_op_groups(tasks, begin, nsm, &ranges);
  if (G < 0) {
    set_error("tre_plan_op_groups: an op's tasks are not contiguous in an SM queue");
    return TRE_ERR_UNSUPPORTED;
  }
  if (out_ranges && max_groups >= G)
    std::memcpy(out_ranges, ranges.data(), ranges.size() * sizeof(int32_t));
  return G;
}

TRE_EXPORT void tre_destroy(tre_engine* e) {
  if (!e) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(e->device);
  if (e->last_stream) cudaStreamSynchronize(e->last_stream);
  cudaDeviceSynchronize();
  if (e->block) cudaFree(e->block);
  if (e->status_host) cudaFreeHost(e->status_host);
  cudaSetDevice(prev);
  delete e;
}

TRE_EXPORT tre_status tre_create(const tre_config* cfg, const tre_weights* w, int device,
                                 tre_engine** out) {
  if (!cfg || !w || !out) {
    set_error("tre_create: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  *out = nullptr;
  int ndev = 0;
  CK(cudaGetDeviceCount(&ndev));
  if (device < 0 || device >= ndev) {
    set_error("tre_create: no such device");
    return TRE_ERR_INVALID_ARG;
  }
  CK(cudaSetDevice(device));
  int sms = 0, smem_optin = 0, coop = 0;
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device));
  CK(cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device));
  CK(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, device));
  if (!coop) {
    set_error("tre_create: device lacks cooperative launch");
    return TRE_ERR_UNSUPPORTED;
  }
  const int nsm = cfg->num_sms ? std::min(cfg->num_sms, sms) : sms;

  PlanShape s;
  std::vector<Task> tasks;
  std::vector<int32_t> begin;
  tre_status st = plan_build(*cfg, nsm, smem_optin, &s, &tasks, &begin, nullptr);
  if (st != TRE_OK) return st;

  // ---- pointer validation: everything the plan reads must be present and 16B-aligned.
  if (!w->layer_w || !w->k_cache || (!w->v_cache && (s.kind != TRE_LAYER_MLA || s.KI))) {
    set_error("tre_create: layer_w / k_cache / v_cache tables must be non-NULL");
    return TRE_ERR_INVALID_ARG;
  }
  static const int gqa_slots[] = {TRE_W_ATTN_NORM, TRE_W_Q,        TRE_W_K,  TRE_W_V,   TRE_W_O,
                                  TRE_W_FFN_NORM,  TRE_W_GATE,     TRE_W_UP, TRE_W_DOWN};
  std::vector<int> slots(gqa_slots, gqa_slots + 9);
  if (s.wfp8)  // the E4M3 projections' block scales
    slots.insert(slots.end(), {TRE_W_SCALE_Q, TRE_W_SCALE_K, TRE_W_SCALE_V, TRE_W_SCALE_O,
                               TRE_W_SCALE_GATE, TRE_W_SCALE_UP, TRE_W_SCALE_DOWN});
  const bool mla = s.kind == TRE_LAYER_MLA;
  if (mla) {
    slots = {TRE_W_ATTN_NORM, TRE_W_DQ, TRE_W_Q_NORM, TRE_W_UQ, TRE_W_DKV, TRE_W_KV_NORM,
             TRE_W_UK, TRE_W_UV, TRE_W_MLA_O};
    if (s.KI) slots.insert(slots.end(), {TRE_W_INDEX_Q, TRE_W_INDEX_K});
  } else if (s.kind == TRE_LAYER_MOE) {
    slots = {TRE_W_ATTN_NORM, TRE_W_Q, TRE_W_K, TRE_W_V, TRE_W_O, TRE_W_FFN_NORM, TRE_W_ROUTER,
             TRE_W_EXPERT_GATE, TRE_W_EXPERT_UP, TRE_W_EXPERT_DOWN};
    if (s.nshared > 0)
      slots.insert(slots.end(), {TRE_W_SHARED_GATE, TRE_W_SHARED_UP, TRE_W_SHARED_DOWN});
  }
  std::vector<LayerPtrs> lp(s.L);
  for (int l = 0; l < s.L; ++l) {
    std::memset(&lp[l], 0, sizeof(LayerPtrs));
    for (int slot : slots) {
      const void* p = w->layer_w[(size_t)l * TRE_W_SLOTS + slot];
      if (!aligned16(p)) {
        set_error("tre_create: layer " + std::to_string(l) + " slot " + std::to_string(slot) +
                  " is NULL or not 16-byte aligned");
        return TRE_ERR_INVALID_ARG;
      }
      lp[l].w[slot] = static_cast<const uint16_t*>(p);
    }
    const bool has_v = !mla || s.KI;  // sparse MLA: v_cache holds the index keys
    if (!aligned16(w->k_cache[l]) || (has_v && (!w->v_cache || !aligned16(w->v_cache[l])))) {
      set_error("tre_create: KV (or index-key) cache of layer " + std::to_string(l) +
                " NULL or misaligned");
      return TRE_ERR_INVALID_ARG;
    }
    lp[l].k_cache = static_cast<uint16_t*>(w->k_cache[l]);
    lp[l].v_cache = has_v ? static_cast<uint16_t*>(w->v_cache[l]) : nullptr;
  }
  if (s.has_lm && (!aligned16(w->embed) || !aligned16(w->final_norm) || !aligned16(w->lm_head))) {
    set_error("tre_create: embed / final_norm / lm_head NULL or not 16-byte aligned");
    return TRE_ERR_INVALID_ARG;
  }

  std::vector<int32_t> ranges;
  const int n_groups = plan_op_groups(tasks, begin, nsm, &ranges);
  if (n_groups < 0) {
    set_error("tre_create: an op's tasks are not contiguous in an SM queue");
    return TRE_ERR_UNSUPPORTED;
  }

  int bps = 0;
  CK(engine_configure(s.smem_bytes, &bps, s.kind == TRE_LAYER_MLA, s.M, s.tiles != 0,
                      s.wfp8 != 0, s.KI > 0, s.wfp4 != 0));
  if (bps < 1) {
    set_error("tre_create: the persistent CTA does not fit on an SM");
    return TRE_ERR_OCCUPANCY;
  }

  tre_engine* e = new tre_engine();
  e->cfg = *cfg;
  e->device = device;
  e->shape = s;
  e->n_tasks = (int)tasks.size();
  e->n_groups = n_groups;

  // ---- one device block for all engine-owned state
  const int qkv_n = mla ? s.Hq * (s.NP + s.R) + s.HI * s.DI : (s.Hq + 2 * s.Hkv) * s.D;
  const int C = s.KL + s.R;
  // MLA: one map per layer over the latent cache; GQA / MoE: K and V maps per layer over
  // the caches viewed as [Hkv * capacity][D]
  std::vector<CUtensorMap> maps(mla ? s.L : 2 * s.L);
  for (int l = 0; l < s.L; ++l) {
    tre_status ms = mla ? encode_cache_map(w->k_cache[l], C, s.cap, kMlaPosPerStage, &maps[l])
                        : encode_cache_map(w->k_cache[l], s.D, (long long)s.Hkv * s.cap,
                                           s.pos_per_stage, &maps[2 * l]);
    if (ms == TRE_OK && !mla)
      ms = encode_cache_map(w->v_cache[l], s.D, (long long)s.Hkv * s.cap, s.pos_per_stage,
                            &maps[2 * l + 1]);
    if (ms != TRE_OK) return ms;
  }
  // sparse MLA: one map per layer over the index-key cache, boxes of kIndexRows keys
  std::vector<CUtensorMap> imaps(s.KI ? s.L : 0);
  for (int l = 0; l < (int)imaps.size(); ++l) {
    const tre_status ms = encode_cache_map(w->v_cache[l], s.DI, s.cap, kIndexRows, &imaps[l]);
    if (ms != TRE_OK) return ms;
  }
  Carve cv;
  size_t o_tasks = cv.take<Task>(tasks.size());
  size_t o_begin = cv.take<int32_t>(begin.size());
  size_t o_ranges = cv.take<int32_t>(ranges.size());
  size_t o_layers = cv.take<LayerPtrs>(s.L);
  size_t o_ctr = cv.take<uint32_t>((size_t)s.n_counters * kCtrStride);
  size_t o_ctr_op = cv.take<uint32_t>((size_t)s.n_counters * kCtrStride);  // bumped by kernel-per-op launches only
  size_t o_tick = cv.take<uint32_t>(std::max(s.Hkv, mla ? s.Hq / kMlaHeadGroup : 1));
  size_t o_lmt = cv.take<uint32_t>(1);
  size_t o_arg = cv.take<unsigned long long>(kMaxTokens);
  size_t o_err = cv.take<int32_t>(2);
  const size_t M = (size_t)s.M;  // per-token buffers: [M][...]
  size_t o_x = cv.take<float>(M * s.d);
  size_t o_h1 = cv.take<float>(M * s.d);
  size_t o_qkv = cv.take<float>(M * qkv_n);
  size_t o_attn = cv.take<float>(M * s.Hq * s.D);
  size_t o_u = cv.take<float>(M * s.u_floats);
  const bool moe = s.kind == TRE_LAYER_MOE;
  size_t o_scores = cv.take<float>(moe ? s.E : 1);
  size_t o_ridx = cv.take<int32_t>(moe ? (size_t)s.L * s.topk : 1);
  size_t o_rw = cv.take<float>(moe ? (size_t)s.L * s.topk : 1);
  size_t o_rtick = cv.take<uint32_t>(1);
  size_t o_mpart = cv.take<float>(moe ? (size_t)(s.nshared + s.topk) * s.d
                                       : s.mo_slices ? (size_t)s.mo_slices * s.d : 1);
  size_t o_dtick = cv.take<uint32_t>(s.down_blocks ? s.down_blocks : 1);
  size_t o_part = cv.take<float>(M * s.Hq * s.kv_splits * (mla ? mla_pstride(s.KL) : gqa_pstride(s.D)));
  size_t o_logits = cv.take<float>(s.V > 0 ? M * s.V : 1);
  size_t o_tok = cv.take<int32_t>(kMaxTokens);
  size_t o_inv = cv.take<double>(std::max(1, s.D / 2));
  size_t o_invr = cv.take<double>(std::max(1, s.R / 2));
  size_t o_cqkv = cv.take<float>(mla ? s.QL + C + s.DI + s.HI : 1);
  size_t o_qf = cv.take<float>(mla ? (size_t)s.Hq * C : 1);
  size_t o_latn = cv.take<float>(mla ? C : 1);
  size_t o_olat = cv.take<float>(mla ? (size_t)s.Hq * s.KL : 1);
  size_t o_mlao = cv.take<float>(mla ? (size_t)s.Hq * s.VD : 1);
  const bool sp = s.KI > 0;
  size_t o_isc = cv.take<float>(sp ? (size_t)s.L * s.cap : 1);
  size_t o_isel = cv.take<int32_t>(sp ? (size_t)s.L * s.KI : 1);
  size_t o_icand = cv.take<unsigned long long>(sp ? (size_t)s.L * s.cap : 1);
  size_t o_ihist = cv.take<uint32_t>(sp ? (size_t)s.L * kIndexBins : 1);
  size_t o_imeta = cv.take<uint32_t>(sp ? (size_t)s.L * IM_WORDS : 1);
  cv.off = (cv.off + 127) & ~size_t(127);
  size_t o_maps = cv.take<CUtensorMap>(maps.size() ? maps.size() : 1);
  size_t o_imaps = cv.take<CUtensorMap>(imaps.size() ? imaps.size() : 1);
  const bool dbg_hidden = cfg->debug_flags & TRE_DEBUG_HIDDEN;
  const bool dbg_trace = cfg->debug_flags & TRE_DEBUG_TRACE;
  size_t o_hidden = dbg_hidden ? cv.take<float>((size_t)s.L * M * s.d) : 0;
  size_t o_trace = dbg_trace ? cv.take<long long>((size_t)tasks.size() * kTraceCols) : 0;
  e->block_bytes = cv.off;
  cudaError_t ce = cudaMalloc(&e->block, e->block_bytes);
  if (ce != cudaSuccess) {
    delete e;
    return cuda_fail(ce, "cudaMalloc(engine state)");
  }
  uint8_t* B = static_cast<uint8_t*>(e->block);
  auto fail_free = [&](cudaError_t err, const char* what) {
    tre_status r = cuda_fail(err, what);
    tre_destroy(e);
    return r;
  };
  if ((ce = cudaMemset(e->block, 0, e->block_bytes)) != cudaSuccess)
    return fail_free(ce, "cudaMemset(engine state)");
  e->guards = cv.guards;
  for (size_t g : e->guards)
    if ((ce = cudaMemset(B + g, kGuardFill, kGuardBytes)) != cudaSuccess)
      return fail_free(ce, "cudaMemset(guards)");
  e->expected.assign(s.n_counters, 0u);
  for (const Task& t : tasks)
    if (t.dep >= 0) e->expected[t.dep] = t.dep_count;
  if ((ce = cudaMemcpy(B + o_tasks, tasks.data(), tasks.size() * sizeof(Task),
                       cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail_free(ce, "upload tasks");
  if ((ce = cudaMemcpy(B + o_begin, begin.data(), begin.size() * sizeof(int32_t),
                       cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail_free(ce, "upload queues");
  if ((ce = cudaMemcpy(B + o_ranges, ranges.data(), ranges.size() * sizeof(int32_t),
                       cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail_free(ce, "upload op groups");
  if ((ce = cudaMemcpy(B + o_layers, lp.data(), lp.size() * sizeof(LayerPtrs),
                       cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail_free(ce, "upload layer table");
  // RoPE frequencies theta^(-2i/D) of the head dim (GQA / MoE) or the rope dim (MLA)
  for (int which = 0; which < 2; ++which) {
    const int D = which ? s.R : s.D;
    if (D < 2) continue;
    std::vector<double> inv(D / 2);
    for (int i = 0; i < D / 2; ++i) inv[i] = std::pow((double)cfg->rope_theta, -2.0 * i / (double)D);
    if ((ce = cudaMemcpy(B + (which ? o_invr : o_inv), inv.data(), inv.size() * sizeof(double),
                         cudaMemcpyHostToDevice)) != cudaSuccess)
      return fail_free(ce, "upload rope table");
  }
  if (!maps.empty() &&
      (ce = cudaMemcpy(B + o_maps, maps.data(), maps.size() * sizeof(CUtensorMap),
                       cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail_free(ce, "upload tensor maps");
  if (!imaps.empty() &&
      (ce = cudaMemcpy(B + o_imaps, imaps.data(), imaps.size() * sizeof(CUtensorMap),
                       cudaMemcpyHostToDevice)) != cudaSuccess)
    return fail_free(ce, "upload index tensor maps");
  if ((ce = cudaHostAlloc(reinterpret_cast<void**>(&e->status_host), 4 * sizeof(int32_t),
                          cudaHostAllocMapped)) != cudaSuccess)
    return fail_free(ce, "cudaHostAlloc(status)");
  std::memset(e->status_host, 0, 4 * sizeof(int32_t));
  if ((ce = cudaHostGetDevicePointer(reinterpret_cast<void**>(&e->status_dev), e->status_host,
                                     0)) != cudaSuccess)
    return fail_free(ce, "cudaHostGetDevicePointer(status)");

  Params& p = e->base;
  p.tasks = reinterpret_cast<const Task*>(B + o_tasks);
  p.sm_begin = reinterpret_cast<const int32_t*>(B + o_begin);
  p.op_ranges = reinterpret_cast<const int32_t*>(B + o_ranges);
  p.op_group = -1;
  p.token_in = nullptr;
  p.counters = reinterpret_cast<uint32_t*>(B + o_ctr);
  e->op_counters = reinterpret_cast<uint32_t*>(B + o_ctr_op);
  p.tickets = reinterpret_cast<uint32_t*>(B + o_tick);
  p.lm_ticket = reinterpret_cast<uint32_t*>(B + o_lmt);
  p.argmax_slot = reinterpret_cast<unsigned long long*>(B + o_arg);
  p.layers = reinterpret_cast<const LayerPtrs*>(B + o_layers);
  p.embed = static_cast<const uint16_t*>(w->embed);
  p.final_norm = static_cast<const uint16_t*>(w->final_norm);
  p.lm_head = static_cast<const uint16_t*>(w->lm_head);
  p.x = reinterpret_cast<float*>(B + o_x);
  p.h1 = reinterpret_cast<float*>(B + o_h1);
  p.qkv = reinterpret_cast<float*>(B + o_qkv);
  p.attn = reinterpret_cast<float*>(B + o_attn);
  p.u = reinterpret_cast<float*>(B + o_u);
  p.scores = reinterpret_cast<float*>(B + o_scores);
  p.route_idx = reinterpret_cast<int32_t*>(B + o_ridx);
  p.route_w = reinterpret_cast<float*>(B + o_rw);
  p.router_ticket = reinterpret_cast<uint32_t*>(B + o_rtick);
  p.mpart = reinterpret_cast<float*>(B + o_mpart);
  p.down_tickets = reinterpret_cast<uint32_t*>(B + o_dtick);
  p.E = s.E; p.topk = s.topk; p.nshared = s.nshared; p.Fe = s.Fe;
  p.part = reinterpret_cast<float*>(B + o_part);
  p.logits = reinterpret_cast<float*>(B + o_logits);
  e->logits_buf = p.logits;
  e->token_buf = reinterpret_cast<int32_t*>(B + o_tok);
  p.hidden = dbg_hidden ? reinterpret_cast<float*>(B + o_hidden) : nullptr;
  p.trace = dbg_trace ? reinterpret_cast<long long*>(B + o_trace) : nullptr;
  p.rope_inv_freq = reinterpret_cast<const double*>(B + o_inv);
  p.rope_inv_freq_r = reinterpret_cast<const double*>(B + o_invr);
  p.cqkv = reinterpret_cast<float*>(B + o_cqkv);
  p.qf = reinterpret_cast<float*>(B + o_qf);
  p.lat_new = reinterpret_cast<float*>(B + o_latn);
  p.o_lat = reinterpret_cast<float*>(B + o_olat);
  p.mla_o = reinterpret_cast<float*>(B + o_mlao);
  p.kv_maps = B + o_maps;
  p.QL = s.QL; p.KL = s.KL; p.R = s.R; p.NP = s.NP; p.VD = s.VD;
  p.HI = s.HI; p.DI = s.DI; p.KI = s.KI; p.isplits = s.isplits;
  p.iscore = reinterpret_cast<float*>(B + o_isc);
  p.ix_sel = reinterpret_cast<int32_t*>(B + o_isel);
  p.ix_cand = reinterpret_cast<unsigned long long*>(B + o_icand);
  p.ix_hist = reinterpret_cast<uint32_t*>(B + o_ihist);
  p.ix_meta = reinterpret_cast<uint32_t*>(B + o_imeta);
  p.ix_maps = B + o_imaps;
  p.kpart_max = s.kpart_max;
  p.m = 1;
  // default: hold (measured faster on the 8B-shaped stack: 0.683 vs 0.665 of peak)
  p.hold_next_op = cfg->stream_policy == 1 ? 0 : cfg->stream_policy >= 3 ? cfg->stream_policy - 1 : 1;
  p.gemv_tiles = s.tiles;
  p.wfp8 = s.wfp8;
  p.wfp4 = s.wfp4;
  p.err = reinterpret_cast<int32_t*>(B + o_err);
  p.abort_flag = reinterpret_cast<volatile int32_t*>(B + o_err + 4);
  p.status_host = e->status_dev;
  p.d = s.d; p.Hq = s.Hq; p.Hkv = s.Hkv; p.D = s.D; p.F = s.F; p.V = s.V; p.L = s.L;
  p.cap = s.cap;
  p.nsplit = s.kv_splits;
  p.pps = s.pos_per_stage;
  p.stage_bytes = s.stage_bytes;
  p.ring_stages = s.ring_stages;
  p.xs_floats = s.xs_floats;
  p.ub_floats = s.ub_floats;
  p.eps = cfg->norm_eps;
  p.flags = cfg->debug_flags;
  p.timeout_ns = 1000LL * (cfg->dep_timeout_us ? cfg->dep_timeout_us : 1000000);
  p.pf_window = cfg->l2_prefetch_kb > 0 ? 1024LL * cfg->l2_prefetch_kb : 1024LL * kDefaultPrefetchKB;
  *out = e;
  return TRE_OK;
}

static tre_status pending_device_error(tre_engine* e) {
  const int32_t code = *reinterpret_cast<volatile int32_t*>(e->status_host);
  if (code == 0) return TRE_OK;
  set_error("a previous step recorded device error " + std::to_string(code) + " (task " +
            std::to_string(reinterpret_cast<volatile int32_t*>(e->status_host)[1]) +
            "); call tre_reset");
  return (tre_status)code;
}

// Enqueue one step: one persistent launch, or (kernel-per-op form) one plain launch per
// op group.  token_in (device, or NULL): token 0 is read there by the kernel.
static tre_status launch_step(tre_engine* e, const int32_t* tokens, int m, int32_t pos,
                              cudaStream_t stream, float* logits_dev, int32_t* token_dev,
                              const float* x_in, float* x_out, const int32_t* token_in = nullptr) {
  tre_status st = pending_device_error(e);
  if (st != TRE_OK) return st;
  if (pos < 0 || pos + m > e->shape.cap) {
    set_error("pos .. pos + tokens - 1 outside [0, kv_capacity)");
    return TRE_ERR_POS_RANGE;
  }
  CK(cudaSetDevice(e->device));
  const bool per_op = e->launch_mode == TRE_LAUNCH_PER_OP;
  if (!per_op) {
    // A persistent step waits for its counters to reach epoch * count; a replayed capture
    // would carry a stale epoch and not wait at all, so it is refused.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    CK(cudaStreamIsCapturing(stream, &cap));
    if (cap != cudaStreamCaptureStatusNone) {
      set_error("a persistent step cannot be captured in a CUDA graph (each step waits for a "
                "new epoch of its counters); capture TRE_LAUNCH_PER_OP steps instead");
      return TRE_ERR_UNSUPPORTED;
    }
  }
  Params p = e->base;
  p.m = m;
  for (int v = 0; v < kMaxTokens; ++v) p.tokens[v] = v < m ? tokens[v] : tokens[0];
  p.token = tokens[0];
  p.token_in = token_in;
  p.pos = pos;
  p.epoch = per_op ? e->epoch : ++e->epoch;
  if (per_op) p.counters = e->op_counters;
  if (logits_dev) p.logits = logits_dev;
  p.token_out = token_dev ? token_dev : e->token_buf;
  p.x_in = x_in;
  p.x_out = x_out;
  const bool mla = e->shape.kind == TRE_LAYER_MLA;
  cudaError_t ce = cudaSuccess;
  if (per_op) {
    for (int g = 0; g < e->n_groups && ce == cudaSuccess; ++g) {
      p.op_group = g;
      ce = engine_launch(p, e->shape.nsm, e->shape.smem_bytes, stream, mla);
    }
  } else {
    ce = engine_launch(p, e->shape.nsm, e->shape.smem_bytes, stream, mla);
  }
  if (ce != cudaSuccess) {
    if (!per_op) --e->epoch;
    return cuda_fail(ce, "launch of the engine kernel");
  }
  e->last_m = m;
  e->last_stream = stream;
  return TRE_OK;
}

TRE_EXPORT tre_status tre_set_launch_mode(tre_engine* e, int32_t mode,
                                          int32_t* launches_per_step) {
  if (!e) {
    set_error("tre_set_launch_mode: NULL engine");
    return TRE_ERR_INVALID_ARG;
  }
  if (mode != TRE_LAUNCH_PERSISTENT && mode != TRE_LAUNCH_PER_OP) {
    set_error("tre_set_launch_mode: unknown mode");
    return TRE_ERR_INVALID_ARG;
  }
  e->launch_mode = mode;
  if (launches_per_step) *launches_per_step = mode == TRE_LAUNCH_PER_OP ? e->n_groups : 1;
  return TRE_OK;
}

TRE_EXPORT tre_status tre_decode_loop(tre_engine* e, int32_t token, int32_t pos, int32_t n_steps,
                                      tre_stream stream, int32_t* tokens_dev, float* logits_dev) {
  if (!e || !tokens_dev) {
    set_error("tre_decode_loop: NULL engine or tokens_dev");
    return TRE_ERR_INVALID_ARG;
  }
  if (!e->shape.has_lm) {
    set_error("tre_decode_loop: engine has no embedding / LM head");
    return TRE_ERR_UNSUPPORTED;
  }
  if (n_steps < 1) {
    set_error("tre_decode_loop: n_steps must be >= 1");
    return TRE_ERR_INVALID_ARG;
  }
  if (token < 0 || token >= e->shape.V) {
    set_error("tre_decode_loop: token outside [0, vocab)");
    return TRE_ERR_INVALID_ARG;
  }
  if (((uintptr_t)tokens_dev & 3u) || (logits_dev && ((uintptr_t)logits_dev & 15u))) {
    set_error("tre_decode_loop: tokens_dev must be 4-byte and logits_dev 16-byte aligned");
    return TRE_ERR_INVALID_ARG;
  }
  if (pos < 0 || (int64_t)pos + n_steps > e->shape.cap) {
    set_error("tre_decode_loop: pos .. pos + n_steps - 1 outside [0, kv_capacity)");
    return TRE_ERR_POS_RANGE;
  }
  for (int i = 0; i < n_steps; ++i) {
    tre_status st = launch_step(e, &token, 1, pos + i, (cudaStream_t)stream, logits_dev,
                                tokens_dev + i, nullptr, nullptr,
                                i == 0 ? nullptr : tokens_dev + i - 1);
    if (st != TRE_OK) return st;
  }
  return TRE_OK;
}

TRE_EXPORT tre_status tre_decode_step(tre_engine* e, int32_t token, int32_t pos, tre_stream stream,
                                      float* logits_dev, int32_t* token_dev) {
  if (!e) {
    set_error("tre_decode_step: NULL engine");
    return TRE_ERR_INVALID_ARG;
  }
  if (!e->shape.has_lm) {
    set_error("tre_decode_step: engine has no embedding / LM head (use a layers step)");
    return TRE_ERR_UNSUPPORTED;
  }
  if (token < 0 || token >= e->shape.V) {
    set_error("tre_decode_step: token outside [0, vocab)");
    return TRE_ERR_INVALID_ARG;
  }
  if (logits_dev && ((uintptr_t)logits_dev & 15u)) {
    set_error("tre_decode_step: logits_dev must be 16-byte aligned");
    return TRE_ERR_INVALID_ARG;
  }
  return launch_step(e, &token, 1, pos, (cudaStream_t)stream, logits_dev, token_dev, nullptr,
                     nullptr);
}

TRE_EXPORT tre_status tre_decode_tokens(tre_engine* e, const int32_t* tokens_host, int32_t m,
                                        int32_t pos, tre_stream stream, float* logits_dev,
                                        int32_t* tokens_dev) {
  if (!e || !tokens_host) {
    set_error("tre_decode_tokens: NULL engine or tokens");
    return TRE_ERR_INVALID_ARG;
  }
  if (!e->shape.has_lm) {
    set_error("tre_decode_tokens: engine has no embedding / LM head");
    return TRE_ERR_UNSUPPORTED;
  }
  if (m < 1 || m > e->shape.M) {
    set_error("tre_decode_tokens: m outside [1, max_tokens_per_step]");
    return TRE_ERR_INVALID_ARG;
  }
  for (int v = 0; v < m; ++v)
    if (tokens_host[v] < 0 || tokens_host[v] >= e->shape.V) {
      set_error("tre_decode_tokens: token outside [0, vocab)");
      return TRE_ERR_INVALID_ARG;
    }
  if (logits_dev && ((uintptr_t)logits_dev & 15u)) {
    set_error("tre_decode_tokens: logits_dev must be 16-byte aligned");
    return TRE_ERR_INVALID_ARG;
  }
  return launch_step(e, tokens_host, m, pos, (cudaStream_t)stream, logits_dev, tokens_dev,
                     nullptr, nullptr);
}

TRE_EXPORT tre_status tre_decode_step_host(tre_engine* e, int32_t token, int32_t pos,
                                           tre_stream stream, float* logits_host,
                                           int32_t* token_host) {
  if (!e || !token_host) {
    set_error("tre_decode_step_host: NULL engine or token_host");
    return TRE_ERR_INVALID_ARG;
  }
  tre_status st = tre_decode_step(e, token, pos, stream, nullptr, nullptr);
  if (st != TRE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  CK(cudaMemcpyAsync(token_host, e->token_buf, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  if (logits_host)
    CK(cudaMemcpyAsync(logits_host, e->logits_buf, (size_t)e->shape.V * sizeof(float),
                       cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return pending_device_error(e);
}

TRE_EXPORT tre_status tre_layers_step(tre_engine* e, const float* x_in_dev, float* x_out_dev,
                                      int32_t pos, tre_stream stream) {
  if (!e || !x_in_dev || !x_out_dev) {
    set_error("tre_layers_step: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  if (e->shape.has_lm) {
    set_error("tre_layers_step: engine has an embedding / LM head (use tre_decode_step)");
    return TRE_ERR_UNSUPPORTED;
  }
  if (!aligned16(x_in_dev) || !aligned16(x_out_dev)) {
    set_error("tre_layers_step: x_in_dev / x_out_dev must be 16-byte aligned");
    return TRE_ERR_INVALID_ARG;
  }
  const size_t bytes = (size_t)e->shape.d * sizeof(float);
  const uintptr_t a = (uintptr_t)x_in_dev, b = (uintptr_t)x_out_dev;
  if (a < b + bytes && b < a + bytes) {
    set_error("tre_layers_step: x_out_dev overlaps x_in_dev");
    return TRE_ERR_INVALID_ARG;
  }
  const int32_t none = 0;
  return launch_step(e, &none, 1, pos, (cudaStream_t)stream, nullptr, nullptr, x_in_dev,
                     x_out_dev);
}

TRE_EXPORT tre_status tre_debug_routing(tre_engine* e, int32_t* idx_host, float* w_host) {
  if (!e) {
    set_error("tre_debug_routing: NULL engine");
    return TRE_ERR_INVALID_ARG;
  }
  if (e->shape.kind != TRE_LAYER_MOE) {
    set_error("tre_debug_routing: not a MoE engine");
    return TRE_ERR_UNSUPPORTED;
  }
  CK(cudaSetDevice(e->device));
  if (e->last_stream) CK(cudaStreamSynchronize(e->last_stream));
  const size_t n = (size_t)e->shape.L * e->shape.topk;
  if (idx_host) CK(cudaMemcpy(idx_host, e->base.route_idx, n * 4, cudaMemcpyDeviceToHost));
  if (w_host) CK(cudaMemcpy(w_host, e->base.route_w, n * 4, cudaMemcpyDeviceToHost));
  return TRE_OK;
}

TRE_EXPORT tre_status tre_debug_check(tre_engine* e, int32_t* bad_counter_out,
                                      int32_t* bad_guard_out) {
  if (!e || !bad_counter_out || !bad_guard_out) {
    set_error("tre_debug_check: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  CK(cudaSetDevice(e->device));
  if (e->last_stream) CK(cudaStreamSynchronize(e->last_stream));
  CK(cudaDeviceSynchronize());
  const int n = e->shape.n_counters;
  std::vector<uint32_t> c((size_t)n * kCtrStride);
  CK(cudaMemcpy(c.data(), e->base.counters, c.size() * 4, cudaMemcpyDeviceToHost));
  *bad_counter_out = -1;
  for (int i = 0; i < n; ++i)
    if (e->expected[i] && c[(size_t)i * kCtrStride] != e->epoch * e->expected[i]) {
      *bad_counter_out = i;
      break;
    }
  *bad_guard_out = -1;
  std::vector<unsigned char> g(kGuardBytes);
  const uint8_t* B = static_cast<const uint8_t*>(e->block);
  for (size_t k = 0; k < e->guards.size() && *bad_guard_out < 0; ++k) {
    CK(cudaMemcpy(g.data(), B + e->guards[k], kGuardBytes, cudaMemcpyDeviceToHost));
    for (unsigned char b : g)
      if (b != kGuardFill) {
        *bad_guard_out = (int32_t)k;
        break;
      }
  }
  return TRE_OK;
}

TRE_EXPORT tre_status tre_debug_index(tre_engine* e, int32_t layer, int32_t pos, float* score_host,
                                      int32_t* sel_host, int32_t* n_sel_out) {
  if (!e || !n_sel_out) {
    set_error("tre_debug_index: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  const PlanShape& s = e->shape;
  if (!s.KI || layer < 0 || layer >= s.L || pos < 0 || pos >= s.cap) {
    set_error("tre_debug_index: not a sparse MLA engine, or layer / pos out of range");
    return TRE_ERR_INVALID_ARG;
  }
  CK(cudaSetDevice(e->device));
  if (e->last_stream) CK(cudaStreamSynchronize(e->last_stream));
  CK(cudaDeviceSynchronize());
  const Params& p = e->base;
  if (score_host)
    CK(cudaMemcpy(score_host, p.iscore + (size_t)layer * s.cap, (size_t)(pos + 1) * 4,
                  cudaMemcpyDeviceToHost));
  if (pos + 1 <= s.KI) {  // every position
    *n_sel_out = pos + 1;
    if (sel_host)
      for (int i = 0; i <= pos; ++i) sel_host[i] = i;
    return TRE_OK;
  }
  uint32_t meta[IM_WORDS];
  CK(cudaMemcpy(meta, p.ix_meta + (size_t)layer * IM_WORDS, sizeof(meta), cudaMemcpyDeviceToHost));
  const int n = (int)std::min<uint32_t>(meta[IM_NSEL], (uint32_t)s.KI);
  if (sel_host) {
    CK(cudaMemcpy(sel_host, p.ix_sel + (size_t)layer * s.KI, (size_t)n * 4, cudaMemcpyDeviceToHost));
    if (meta[IM_HASPOS] && n < s.KI) sel_host[n] = pos;
  }
  *n_sel_out = n + (meta[IM_HASPOS] && n < s.KI ? 1 : 0);
  return TRE_OK;
}

TRE_EXPORT tre_status tre_get_status(tre_engine* e, int32_t* device_status, int32_t* detail_out) {
  if (!e || !device_status) {
    set_error("tre_get_status: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  CK(cudaSetDevice(e->device));
  if (e->last_stream) CK(cudaStreamSynchronize(e->last_stream));
  CK(cudaDeviceSynchronize());
  volatile int32_t* sh = e->status_host;
  *device_status = sh[0];
  if (detail_out) *detail_out = sh[1];
  return TRE_OK;
}

TRE_EXPORT tre_status tre_reset(tre_engine* e, tre_stream stream) {
  if (!e) {
    set_error("tre_reset: NULL engine");
    return TRE_ERR_INVALID_ARG;
  }
  CK(cudaSetDevice(e->device));
  cudaStream_t s = (cudaStream_t)stream;
  CK(cudaDeviceSynchronize());
  const Params& p = e->base;
  CK(cudaMemsetAsync(p.counters, 0, (size_t)e->shape.n_counters * kCtrStride * 4, s));
  CK(cudaMemsetAsync(e->op_counters, 0, (size_t)e->shape.n_counters * kCtrStride * 4, s));
  CK(cudaMemsetAsync(p.tickets, 0,
                     (size_t)std::max(e->shape.Hkv, e->shape.kind == TRE_LAYER_MLA
                                                        ? e->shape.Hq / kMlaHeadGroup : 1) * 4,
                     s));
  CK(cudaMemsetAsync(p.lm_ticket, 0, 4, s));
  CK(cudaMemsetAsync(p.router_ticket, 0, 4, s));
  if (e->shape.down_blocks)
    CK(cudaMemsetAsync(p.down_tickets, 0, (size_t)e->shape.down_blocks * 4, s));
  CK(cudaMemsetAsync(p.argmax_slot, 0, 8 * kMaxTokens, s));
  CK(cudaMemsetAsync(p.err, 0, 8, s));  // error word + abort flag
  if (e->shape.KI) {  // sparse MLA: histograms and selection state (tickets included)
    CK(cudaMemsetAsync(p.ix_hist, 0, (size_t)e->shape.L * kIndexBins * 4, s));
    CK(cudaMemsetAsync(p.ix_meta, 0, (size_t)e->shape.L * IM_WORDS * 4, s));
  }
  CK(cudaStreamSynchronize(s));
  std::memset(e->status_host, 0, 4 * sizeof(int32_t));
  e->epoch = 0;
  return TRE_OK;
}

TRE_EXPORT tre_status tre_debug_hidden(tre_engine* e, float* hidden_dev, tre_stream stream) {
  if (!e || !hidden_dev) {
    set_error("tre_debug_hidden: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  if (!e->base.hidden) {
    set_error("tre_debug_hidden: engine created without TRE_DEBUG_HIDDEN");
    return TRE_ERR_INVALID_ARG;
  }
  CK(cudaSetDevice(e->device));
  CK(cudaMemcpyAsync(hidden_dev, e->base.hidden,
                     (size_t)e->shape.L * e->last_m * e->shape.d * sizeof(float),
                     cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return TRE_OK;
}

TRE_EXPORT tre_status tre_debug_trace(tre_engine* e, int64_t* trace_host, int32_t* n_tasks) {
  if (!e || !n_tasks) {
    set_error("tre_debug_trace: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  *n_tasks = e->n_tasks;
  if (!trace_host) return TRE_OK;
  if (!e->base.trace) {
    set_error("tre_debug_trace: engine created without TRE_DEBUG_TRACE");
    return TRE_ERR_INVALID_ARG;
  }
  CK(cudaSetDevice(e->device));
  CK(cudaDeviceSynchronize());
  CK(cudaMemcpy(trace_host, e->base.trace, (size_t)e->n_tasks * kTraceCols * sizeof(long long),
                cudaMemcpyDeviceToHost));
  return TRE_OK;
}

TRE_EXPORT tre_status tre_step_bytes(const tre_engine* e, int32_t pos, int32_t m, int64_t* bytes) {
  if (!e || !bytes) {
    set_error("tre_step_bytes: NULL argument");
    return TRE_ERR_INVALID_ARG;
  }
  if (m < 1 || m > e->shape.M) {
    set_error("tre_step_bytes: m outside [1, max_tokens_per_step]");
    return TRE_ERR_INVALID_ARG;
  }
  *bytes = step_bytes(e->shape, pos, m);
  return TRE_OK;
}
