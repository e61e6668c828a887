// tre_decode_step_static: one decode step for callers that cannot allocate GPU memory.
//
// The regular path (tre_create + tre_decode_step) cudaMallocs the engine's plan, counters
// and activation scratch once, at create time.  Some callers cannot do that: code that runs
// under an allocator it does not own (a framework whose caching allocator must see every
// byte), real-time loops where any allocation is forbidden, or plug-ins handed only raw
// input / output pointers.  This entry point serves them: every byte the engine kernel
// needs beyond the caller's weights, caches and outputs lives in one file-scope device
// array of fixed size, so the call itself allocates no GPU memory.
//
// The same persistent kernel runs; only where its scratch lives differs.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "tre_internal.h"

namespace tre {
cudaError_t engine_configure(int smem_bytes, int* blocks_per_sm, bool mla, int max_m, bool tiled,
                             bool fp8 = false, bool sparse = false, bool fp4 = false);
cudaError_t engine_launch(const Params& p, int grid, int smem_bytes, cudaStream_t stream,
                          bool mla = false);
}  // namespace tre

using namespace tre;

// Upper bound on the scratch one call may use (plan + counters + activations + split-KV
// partials).  4 MiB holds the 32-layer, 4096-wide stack with room to spare.
static constexpr size_t kStaticScratchBytes = size_t(4) << 20;

// Every GPU that loads this library holds this array until the process exits.  In host
// code the name is only a stand-in for the device address: never pass it to a kernel;
// use the address cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_tre_static_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_dev[kMaxDevices] = {};  // device address of the array, per device

tre_status fail(tre_status st, const std::string& m) {
  set_error(m);
  return st;
}

tre_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TRE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Once per device, with that device current: resolve the array's device address.  Every
// call also makes sure the kernel's shared-memory limit is the device maximum (a host-side
// attribute, not an allocation).
tre_status setup_device(int dev, void** scratch) {
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_dev[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_tre_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_scratch_dev[dev] = ptr;
  }
  int bps = 0;
  cudaError_t e = engine_configure(kSmemLimit, &bps, false, 1, false);
  if (e != cudaSuccess) return cuda_fail(e, "engine_configure");
  if (bps < 1) return fail(TRE_ERR_OCCUPANCY, "the persistent CTA does not fit on an SM");
  *scratch = g_scratch_dev[dev];
  return TRE_OK;
}

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

struct Carve {
  size_t off = 0;
  template <class T>
  size_t take(size_t count) {
    off = (off + 255) & ~size_t(255);
    const size_t at = off;
    off += count * sizeof(T);
    return at;
  }
};

}  // namespace

extern "C" __attribute__((visibility("default"))) tre_status tre_decode_step_static(
    const tre_config* cfg, const tre_weights* w, int32_t token, int32_t pos, tre_stream stream,
    float* logits_dev, int32_t* token_dev, int32_t* status_dev) {
  if (!cfg || !w || !logits_dev)
    return fail(TRE_ERR_INVALID_ARG, "tre_decode_step_static: cfg, w and logits_dev are required");
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TRE_ERR_UNSUPPORTED, "device index above 63");
  int sms = 0, smem_optin = 0;
  if ((ce = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return cuda_fail(ce, "cudaDeviceGetAttribute");
  if ((ce = cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
      cudaSuccess)
    return cuda_fail(ce, "cudaDeviceGetAttribute");
  const int nsm = cfg->num_sms ? std::min(cfg->num_sms, sms) : sms;

  PlanShape s;
  std::vector<Task> tasks;
  std::vector<int32_t> begin;
  tre_status st = plan_build(*cfg, nsm, smem_optin, &s, &tasks, &begin, nullptr);
  if (st != TRE_OK) return st;
  if (!s.has_lm)
    return fail(TRE_ERR_UNSUPPORTED, "tre_decode_step_static: needs an embedding and LM head");
  if (s.kind != TRE_LAYER_GQA || s.M != 1)
    return fail(TRE_ERR_UNSUPPORTED, "tre_decode_step_static: GQA stacks, one token per step");
  if (cfg->debug_flags & (TRE_DEBUG_HIDDEN | TRE_DEBUG_TRACE))
    return fail(TRE_ERR_UNSUPPORTED, "tre_decode_step_static: debug buffers are not available");
  if (s.wfp8)
    return fail(TRE_ERR_UNSUPPORTED, "tre_decode_step_static: bf16 weights only");

  // ---- scratch layout inside the static array; reject plans that do not fit
  const int qkv_n = (s.Hq + 2 * s.Hkv) * s.D;
  Carve cv;
  const size_t o_tasks = cv.take<Task>(tasks.size());
  const size_t o_begin = cv.take<int32_t>(begin.size());
  const size_t o_layers = cv.take<LayerPtrs>(s.L);
  const size_t o_zero = cv.take<uint32_t>(0);  // everything from here to o_zero_end starts at 0
  const size_t o_ctr = cv.take<uint32_t>((size_t)s.n_counters * kCtrStride);
  const size_t o_tick = cv.take<uint32_t>(s.Hkv);
  const size_t o_lmt = cv.take<uint32_t>(1);
  const size_t o_arg = cv.take<unsigned long long>(kMaxTokens);
  const size_t o_err = cv.take<int32_t>(4);  // error word, abort flag, status fallback [2]
  const size_t o_zero_end = cv.off;
  const size_t o_x = cv.take<float>(s.d);
  const size_t o_h1 = cv.take<float>(s.d);
  const size_t o_qkv = cv.take<float>(qkv_n);
  const size_t o_attn = cv.take<float>((size_t)s.Hq * s.D);
  const size_t o_u = cv.take<float>(s.F);
  const size_t o_part = cv.take<float>((size_t)s.Hq * s.kv_splits * gqa_pstride(s.D));
  const size_t o_inv = cv.take<double>(s.D / 2);
  cv.off = (cv.off + 127) & ~size_t(127);
  const size_t o_maps = cv.take<uint8_t>((size_t)2 * s.L * 128);  // K and V tensor maps
  if (cv.off > kStaticScratchBytes)
    return fail(TRE_ERR_UNSUPPORTED,
                "tre_decode_step_static: this model needs " + std::to_string(cv.off) +
                    " bytes of scratch, above the static maximum of " +
                    std::to_string(kStaticScratchBytes));

  // ---- argument checks (nothing is enqueued before they pass)
  if (token < 0 || token >= s.V) return fail(TRE_ERR_INVALID_ARG, "token outside [0, vocab)");
  if (pos < 0 || pos >= s.cap) return fail(TRE_ERR_POS_RANGE, "pos outside [0, kv_capacity)");
  if ((uintptr_t)logits_dev & 15u)
    return fail(TRE_ERR_INVALID_ARG, "logits_dev must be 16-byte aligned");
  if (status_dev && ((uintptr_t)status_dev & 3u))
    return fail(TRE_ERR_INVALID_ARG, "status_dev must be 4-byte aligned");
  if (!w->layer_w || !w->k_cache || !w->v_cache || !aligned16(w->embed) ||
      !aligned16(w->final_norm) || !aligned16(w->lm_head))
    return fail(TRE_ERR_INVALID_ARG, "weights: NULL or misaligned pointer");
  static const int slots[] = {TRE_W_ATTN_NORM, TRE_W_Q,    TRE_W_K,  TRE_W_V,   TRE_W_O,
                              TRE_W_FFN_NORM,  TRE_W_GATE, TRE_W_UP, TRE_W_DOWN};
  std::vector<LayerPtrs> lp(s.L);
  for (int l = 0; l < s.L; ++l) {
    std::memset(&lp[l], 0, sizeof(LayerPtrs));
    for (int slot : slots) {
      const void* p = w->layer_w[(size_t)l * TRE_W_SLOTS + slot];
      if (!aligned16(p)) return fail(TRE_ERR_INVALID_ARG, "weights: NULL or misaligned layer tensor");
      lp[l].w[slot] = static_cast<const uint16_t*>(p);
    }
    if (!aligned16(w->k_cache[l]) || !aligned16(w->v_cache[l]))
      return fail(TRE_ERR_INVALID_ARG, "weights: NULL or misaligned KV cache");
    lp[l].k_cache = static_cast<uint16_t*>(w->k_cache[l]);
    lp[l].v_cache = static_cast<uint16_t*>(w->v_cache[l]);
  }

  // tensor maps over the K and V caches, built on the host (no allocation)
  std::vector<uint8_t> maps((size_t)2 * s.L * 128);
  for (int l = 0; l < s.L; ++l) {
    st = encode_cache_map(w->k_cache[l], s.D, (long long)s.Hkv * s.cap, s.pos_per_stage,
                          maps.data() + (size_t)2 * l * 128);
    if (st == TRE_OK)
      st = encode_cache_map(w->v_cache[l], s.D, (long long)s.Hkv * s.cap, s.pos_per_stage,
                            maps.data() + (size_t)(2 * l + 1) * 128);
    if (st != TRE_OK) return st;
  }

  // Every call copies its plan from ordinary host memory that is gone once it returns, so
  // a captured call could never be replayed: refuse capture before enqueuing anything.
  cudaStream_t sm = (cudaStream_t)stream;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if ((ce = cudaStreamIsCapturing(sm, &cap)) != cudaSuccess)
    return cuda_fail(ce, "cudaStreamIsCapturing");
  if (cap != cudaStreamCaptureStatusNone)
    return fail(TRE_ERR_UNSUPPORTED,
                "tre_decode_step_static cannot be captured in a CUDA graph (it copies the "
                "plan from host memory on every call)");

  void* scratch = nullptr;
  st = setup_device(dev, &scratch);
  if (st != TRE_OK) return st;
  uint8_t* B = static_cast<uint8_t*>(scratch);

  // ---- fill the array for this call (copies and a memset: no allocation)
  std::vector<double> inv(s.D / 2);
  for (int i = 0; i < s.D / 2; ++i) inv[i] = std::pow((double)cfg->rope_theta, -2.0 * i / (double)s.D);
  if ((ce = cudaMemcpyAsync(B + o_tasks, tasks.data(), tasks.size() * sizeof(Task),
                            cudaMemcpyHostToDevice, sm)) != cudaSuccess ||
      (ce = cudaMemcpyAsync(B + o_begin, begin.data(), begin.size() * sizeof(int32_t),
                            cudaMemcpyHostToDevice, sm)) != cudaSuccess ||
      (ce = cudaMemcpyAsync(B + o_layers, lp.data(), lp.size() * sizeof(LayerPtrs),
                            cudaMemcpyHostToDevice, sm)) != cudaSuccess ||
      (ce = cudaMemcpyAsync(B + o_inv, inv.data(), inv.size() * sizeof(double),
                            cudaMemcpyHostToDevice, sm)) != cudaSuccess ||
      (ce = cudaMemcpyAsync(B + o_maps, maps.data(), maps.size(), cudaMemcpyHostToDevice, sm)) !=
          cudaSuccess ||
      (ce = cudaMemsetAsync(B + o_zero, 0, o_zero_end - o_zero, sm)) != cudaSuccess)
    return cuda_fail(ce, "filling the static scratch");
  if (status_dev && (ce = cudaMemsetAsync(status_dev, 0, 2 * sizeof(int32_t), sm)) != cudaSuccess)
    return cuda_fail(ce, "clearing status_dev");
  // The host buffers above are pageable, so each copy has staged them before returning and
  // they may go out of scope; the copies and the launch below are ordered on `stream`.

  Params p{};
  p.tasks = reinterpret_cast<const Task*>(B + o_tasks);
  p.sm_begin = reinterpret_cast<const int32_t*>(B + o_begin);
  p.op_group = -1;  // the whole step in one persistent launch
  p.counters = reinterpret_cast<uint32_t*>(B + o_ctr);
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
  p.part = reinterpret_cast<float*>(B + o_part);
  p.logits = logits_dev;
  p.token_out = token_dev;
  p.rope_inv_freq = reinterpret_cast<const double*>(B + o_inv);
  p.kv_maps = B + o_maps;
  p.err = reinterpret_cast<int32_t*>(B + o_err);
  p.abort_flag = reinterpret_cast<volatile int32_t*>(B + o_err + 4);
  p.status_host = status_dev ? status_dev : reinterpret_cast<int32_t*>(B + o_err + 8);
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
  p.token = token;
  p.m = 1;
  p.hold_next_op = cfg->stream_policy == 1 ? 0 : cfg->stream_policy >= 3 ? cfg->stream_policy - 1 : 1;
  for (int v = 0; v < kMaxTokens; ++v) p.tokens[v] = token;
  p.pos = pos;
  p.epoch = 1;  // counters were just cleared
  if ((ce = engine_launch(p, s.nsm, s.smem_bytes, sm)) != cudaSuccess)
    return cuda_fail(ce, "launch of the persistent engine");
  return TRE_OK;
}
