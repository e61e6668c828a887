// Host AOT planner: flattens the decoder stack into a static list of tile tasks.
//
// The pages' engine is compiled ahead of time: the whole model is unrolled into one
// persistent kernel whose scheduling unit is the tile (Static Compilation for LLM
// Inference, §1 and §5.1), and the dataflow graph is lowered to tile micro-kernels plus
// an engine that maps tasks onto hardware units (Speed is intelligence talk, section on
// breaking the kernel boundary).  This planner is that step for one GPU:
//
//   * every GEMV op (Q, K, V, O, gate/up, down, LM head, MoE router and experts) is cut
//     into one contiguous row range per SM of equal size (the SMs then finish the op
//     together: every op ends at a dependency the next one waits for);
//   * the attention of each layer is cut into (kv head, KV split) tasks, and the MoE down
//     into (expert slot, row block) tasks, dealt round robin to the SMs (at most one more
//     on any SM than on another; the extras to the SMs with the least streamed bytes);
//   * each task waits on one counter (the op it reads from, all of its tasks) and bumps
//     one counter; counters only grow, so step e waits for e * count;
//   * each SM's queue is in global topological order, so with every CTA resident the
//     lowest unfinished task always has its inputs ready (no deadlock).
#include <algorithm>
#include <cmath>
#include <numeric>
#include <string>
#include <vector>

#include "tre_internal.h"

namespace tre {

static thread_local std::string g_err;
void set_error(const std::string& m) { g_err = m; }
const char* last_error_cstr() { return g_err.c_str(); }

static tre_status fail(tre_status s, const std::string& m) {
  set_error(m);
  return s;
}

static inline int counter_of(int layer, int kind) { return layer * C_PER_LAYER + kind; }

// Split N rows of `row_bytes` each over the SMs: every SM gets floor(N / n) rows and the
// remainder goes one row each to the SMs with the least streamed bytes so far.  Each op
// ends at a dependency every later op waits for, so it is the op's own balance that sets
// its time; `cum` (cumulative bytes) only breaks ties.
static std::vector<std::pair<int, int>> assign_rows(int N, int64_t row_bytes,
                                                    std::vector<int64_t>& cum) {
  const int n = (int)cum.size();
  std::vector<int> rows(n, N / n);
  std::vector<int> idx(n);
  std::iota(idx.begin(), idx.end(), 0);
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return cum[a] < cum[b]; });
  for (int k = 0; k < N % n; ++k) rows[idx[k]]++;
  std::vector<std::pair<int, int>> ranges(n);
  int r = 0;
  for (int i = 0; i < n; ++i) {
    ranges[i] = {r, r + rows[i]};
    r += rows[i];
    cum[i] += (int64_t)rows[i] * row_bytes;
  }
  return ranges;
}

struct Builder {
  int nsm;
  std::vector<std::vector<Task>> q;  // per SM
  std::vector<int64_t> cum;          // streamed bytes per SM
  int next_id = 0;
  int kpart_max = kMaxKPart;

  explicit Builder(int n) : nsm(n), q(n), cum(n, 0) {}

  Task make(uint8_t type, uint8_t op, int layer, int dep, uint32_t dep_count, int out) {
    Task t{};
    t.type = type;
    t.op = op;
    t.layer = (uint16_t)layer;
    t.dep = dep;
    t.dep_count = dep_count;
    t.out = out;
    t.id = next_id++;
    return t;
  }

  // Cut N rows (K inputs each, nseg matrices) into per-SM ranges; a range longer than
  // `cap` rows becomes several sub-ranges, a range is also cut at every multiple of
  // `cut` (> 0: rows of different experts never share a task), and each sub-range is one
  // task per K-part (only the last part bumps `out`).  `np` > 0 fixes the number of
  // K-parts (else they follow from K).  Returns the number of tasks that bump `out`.
  int esz_proj = 2;  // bytes per weight of the GQA projections (1: E4M3)
  bool fp4 = false;  // routed experts are MXFP4 rows

  int gemv(uint8_t op, int layer, int N, int K, int nseg, int dep, uint32_t dep_count, int out,
           int cap, int np = 0, int cut = 0) {
    if (np <= 0) np = (op == OP_LM || op == OP_ROUTER) ? 1 : gemv_nparts(K, kpart_max);
    const int esz = (op == OP_QKV || op == OP_O || op == OP_GU || op == OP_DOWN) ? esz_proj : 2;
    const int64_t rowb = (fp4 && op == OP_RGU) ? fp4_row_pitch(K) : (int64_t)K * esz;
    auto ranges = assign_rows(N, (int64_t)nseg * rowb, cum);
    int n = 0;
    for (int s = 0; s < nsm; ++s) {
      for (int r = ranges[s].first; r < ranges[s].second;) {
        int e = std::min(ranges[s].second, r + cap);
        if (cut > 0) e = std::min(e, (r / cut + 1) * cut);
        for (int part = 0; part < np; ++part) {
          Task t = make(T_GEMV, op, layer, dep, dep_count, part == np - 1 ? out : -1);
          t.r0 = r;
          t.r1 = e;
          t.aux = part | (np << 8);
          q[s].push_back(t);
          if (part == np - 1) ++n;
        }
        r = e;
      }
    }
    return n;
  }

  // SMs for `count` equal tasks of one op: every SM takes floor or ceil(count / nsm) of
  // them (round robin), in order of the least streamed bytes so far.
  std::vector<int> spread(int count) const {
    std::vector<int> idx(nsm);
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return cum[a] < cum[b]; });
    std::vector<int> out(count);
    for (int k = 0; k < count; ++k) out[k] = idx[k % nsm];
    return out;
  }

  // One GEMV task per unit (an MLA head): rows [u * rows, (u + 1) * rows), dealt round
  // robin to the SMs.  Returns the task count.
  int per_unit(uint8_t op, int layer, int units, int rows, int64_t bytes_per_unit, int dep,
               uint32_t dep_count, int out) {
    const std::vector<int> sms = spread(units);
    for (int u = 0; u < units; ++u) {
      Task t = make(T_GEMV, op, layer, dep, dep_count, out);
      t.r0 = u * rows;
      t.r1 = (u + 1) * rows;
      t.aux = 0 | (1 << 8);
      q[sms[u]].push_back(t);
      cum[sms[u]] += bytes_per_unit;
    }
    return units;
  }

  // MLA attention: (head group, KV split) tasks dealt round robin; aux = splits.
  void mla_attention(int layer, int groups, int S, int64_t bytes_per_task, int dep,
                     uint32_t dep_count, int out) {
    const std::vector<int> sms = spread(groups * S);
    for (int g = 0; g < groups; ++g)
      for (int sp = 0; sp < S; ++sp) {
        const int best = sms[g * S + sp];
        Task t = make(T_MLA_ATTN, 0, layer, dep, dep_count, out);
        t.r0 = g;
        t.r1 = sp;
        t.aux = S;
        q[best].push_back(t);
        cum[best] += bytes_per_task;
      }
  }

  // Sparse MLA: `n` tasks of one type (index scoring or selection), split sp = r1 of n
  // (aux = n), each on the SM with the least streamed bytes so far.
  void splits(uint8_t type, int layer, int n, int64_t bytes_per_task, int dep,
              uint32_t dep_count, int out) {
    const std::vector<int> sms = spread(n);
    for (int sp = 0; sp < n; ++sp) {
      Task t = make(type, 0, layer, dep, dep_count, out);
      t.r0 = 0;
      t.r1 = sp;
      t.aux = n;
      q[sms[sp]].push_back(t);
      cum[sms[sp]] += bytes_per_task;
    }
  }

  // MLA output projection in K-slices on different SMs: nb row blocks x np slices, each
  // placed on the SM with the least streamed bytes so far; aux = slice | block << 8 |
  // np << 16.  Returns nb (one bump per block, by its last slice).
  int mo_slices(int layer, int d, int K, int np, int nb, int dep, uint32_t dep_count, int out) {
    const std::vector<int> sms = spread(np * nb);
    const int len = gemv_part_len(K, np, 8);
    for (int bl = 0; bl < nb; ++bl) {
      const int r0 = (int)((int64_t)d * bl / nb), r1 = (int)((int64_t)d * (bl + 1) / nb);
      for (int j = 0; j < np; ++j) {
        const int best = sms[bl * np + j];
        Task t = make(T_GEMV, OP_MOS, layer, dep, dep_count, out);
        t.r0 = r0;
        t.r1 = r1;
        t.aux = j | (bl << 8) | (np << 16);
        q[best].push_back(t);
        cum[best] += (int64_t)(r1 - r0) * std::min(len, K - j * len) * 2;
      }
    }
    return nb;
  }

  // Set aux = count on every task of `op` created since task id `first`.
  void set_count(int first, uint8_t op, int count) {
    for (auto& qq : q)
      for (auto& t : qq)
        if (t.id >= first && t.type == T_GEMV && t.op == op) t.aux = count;
  }

  // MoE down: np slots x nb row blocks of d rows, each placed on the SM with the least
  // streamed bytes so far; aux = slot | block << 8.  Returns nb (one bump per block).
  int nshared = 0;   // MoE: slots below nshared are the shared experts (bf16)
  int moe_down(int layer, int d, int np, int Fe, int nb, int dep, uint32_t dep_count, int out) {
    const std::vector<int> sms = spread(np * nb);
    // MXFP4 routed slots stream fewer bytes than the bf16 shared ones: the shared slots'
    // tasks take the least loaded SMs first
    const bool cheap_routed = fp4 && nshared > 0;
    for (int bl = 0; bl < nb; ++bl) {
      const int r0 = (int)((int64_t)d * bl / nb), r1 = (int)((int64_t)d * (bl + 1) / nb);
      for (int j = 0; j < np; ++j) {
        const int k = !cheap_routed ? bl * np + j
                      : j < nshared ? bl * nshared + j
                                    : nb * nshared + bl * (np - nshared) + (j - nshared);
        const int best = sms[k];
        Task t = make(T_GEMV, OP_MDOWN, layer, dep, dep_count, out);
        t.r0 = r0;
        t.r1 = r1;
        t.aux = j | (bl << 8);
        q[best].push_back(t);
        cum[best] += (int64_t)(r1 - r0) * (fp4 && j >= nshared ? fp4_row_pitch(Fe) : Fe * 2);
      }
    }
    return nb;
  }

  void attention(int layer, int Hkv, int S, int64_t bytes_per_task, int dep, uint32_t dep_count,
                 int out) {
    const std::vector<int> sms = spread(Hkv * S);
    for (int g = 0; g < Hkv; ++g)
      for (int s = 0; s < S; ++s) {
        const int best = sms[g * S + s];
        Task t = make(T_ATTN, 0, layer, dep, dep_count, out);
        t.r0 = g;
        t.r1 = s;
        t.aux = S;
        q[best].push_back(t);
        cum[best] += bytes_per_task;
      }
  }
};

static tre_status validate_mla(const tre_config& c) {
  if (c.n_q_heads < kMlaHeadGroup || c.n_q_heads % kMlaHeadGroup)
    return fail(TRE_ERR_UNSUPPORTED, "MLA heads must be a positive multiple of 16");
  if (c.kv_lora < 128 || c.kv_lora % 128)
    return fail(TRE_ERR_UNSUPPORTED, "MLA kv_lora must be a positive multiple of 128");
  if (c.rope_dim < 16 || c.rope_dim % 16)
    return fail(TRE_ERR_UNSUPPORTED, "MLA rope_dim must be a positive multiple of 16");
  const int C = c.kv_lora + c.rope_dim;
  if (C % kMlaBox || C > 16 * kMlaMaxKSteps * kConsumerWarps)
    return fail(TRE_ERR_UNSUPPORTED, "MLA kv_lora + rope_dim must be a multiple of 64, <= 768");
  if (c.q_lora < 8 || c.q_lora % 8 || c.nope_dim < 8 || c.nope_dim % 8 || c.v_dim < 8 ||
      c.v_dim % 8)
    return fail(TRE_ERR_INVALID_ARG, "MLA q_lora, nope_dim and v_dim must be positive multiples of 8");
  if (c.q_lora > kMaxKPart) return fail(TRE_ERR_UNSUPPORTED, "MLA q_lora above 16384");
  if (c.nope_dim > kMaxResidRows) return fail(TRE_ERR_UNSUPPORTED, "MLA nope_dim above 512");
  if (c.index_topk < 0) return fail(TRE_ERR_INVALID_ARG, "index_topk must be >= 0");
  if (c.index_topk > 0) {
    if (c.index_heads != 16 && c.index_heads != 32 && c.index_heads != 64)
      return fail(TRE_ERR_UNSUPPORTED, "index_heads must be 16, 32 or 64");
    if (c.index_dim != 64 && c.index_dim != 128)
      return fail(TRE_ERR_UNSUPPORTED, "index_dim must be 64 or 128");
    if (c.index_topk > c.kv_capacity)
      return fail(TRE_ERR_INVALID_ARG, "index_topk above kv_capacity");
  } else if (c.index_heads || c.index_dim) {
    return fail(TRE_ERR_INVALID_ARG, "index_heads / index_dim set without index_topk");
  }
  return TRE_OK;
}

static tre_status validate(const tre_config& c) {
  if (c.kind != TRE_LAYER_GQA && c.kind != TRE_LAYER_MOE && c.kind != TRE_LAYER_MLA)
    return fail(TRE_ERR_INVALID_ARG, "unknown layer kind");
  if (c.kind == TRE_LAYER_MLA) {
    tre_status st = validate_mla(c);
    if (st != TRE_OK) return st;
  }
  if (c.kind == TRE_LAYER_MOE) {
    if (c.n_experts < 1 || c.n_experts > kMaxExperts)
      return fail(TRE_ERR_UNSUPPORTED, "n_experts must be in [1, 512]");
    if (c.top_k < 1 || c.top_k > c.n_experts || c.top_k > kMaxTopK)
      return fail(TRE_ERR_INVALID_ARG, "top_k must be in [1, min(n_experts, 32)]");
    if (c.n_shared < 0 || c.n_shared > 16)
      return fail(TRE_ERR_INVALID_ARG, "n_shared must be in [0, 16]");
    if (c.expert_ffn < 8 || c.expert_ffn % 8)
      return fail(TRE_ERR_INVALID_ARG, "expert_ffn must be a positive multiple of 8");
  }
  if (c.kind != TRE_LAYER_MLA && (c.index_heads || c.index_dim || c.index_topk))
    return fail(TRE_ERR_INVALID_ARG, "index_heads / index_dim / index_topk are MLA fields");
  if (c.n_layers < 1 || c.n_layers > 1024) return fail(TRE_ERR_INVALID_ARG, "n_layers out of range");
  if (c.hidden < 8 || c.hidden % 8) return fail(TRE_ERR_INVALID_ARG, "hidden must be a positive multiple of 8");
  if (c.kind != TRE_LAYER_MLA) {
    if (c.n_q_heads < 1 || c.n_kv_heads < 1 || c.n_q_heads % c.n_kv_heads)
      return fail(TRE_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
    int G = c.n_q_heads / c.n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8)
      return fail(TRE_ERR_UNSUPPORTED, "q heads per kv head must be 1, 2, 4 or 8");
    if (c.head_dim != 64 && c.head_dim != 128)
      return fail(TRE_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  }
  if (c.kind == TRE_LAYER_GQA && (c.ffn < 8 || c.ffn % 8))
    return fail(TRE_ERR_INVALID_ARG, "ffn must be a positive multiple of 8");
  if (c.has_embed_lm_head != 0 && c.has_embed_lm_head != 1)
    return fail(TRE_ERR_INVALID_ARG, "has_embed_lm_head must be 0 or 1");
  if (c.has_embed_lm_head && c.vocab < 1) return fail(TRE_ERR_INVALID_ARG, "vocab must be >= 1");
  if (c.kv_capacity < 1) return fail(TRE_ERR_INVALID_ARG, "kv_capacity must be >= 1");
  if (c.max_tokens_per_step < 0 || c.max_tokens_per_step > kMaxTokens)
    return fail(TRE_ERR_INVALID_ARG, "max_tokens_per_step must be in [0, 4]");
  if (c.max_tokens_per_step > 1) {
    if (c.kind != TRE_LAYER_GQA)
      return fail(TRE_ERR_UNSUPPORTED, "multi-token steps are implemented for GQA stacks only");
    if (c.multi_token_gemv == 2 && (c.hidden % 16 || c.ffn % 16))
      return fail(TRE_ERR_UNSUPPORTED, "multi-token tensor-core tiles need hidden and ffn multiples of 16");
    if (c.max_tokens_per_step * (c.n_q_heads / c.n_kv_heads) > 16)
      return fail(TRE_ERR_UNSUPPORTED, "tokens x (q heads per kv head) above 16");
  }
  if (c.weight_format != TRE_WEIGHTS_BF16 && c.weight_format != TRE_WEIGHTS_FP8_BLOCK128 &&
      c.weight_format != TRE_WEIGHTS_FP4_EXPERTS)
    return fail(TRE_ERR_INVALID_ARG, "unknown weight_format");
  if (c.weight_format == TRE_WEIGHTS_FP4_EXPERTS) {
    if (c.kind != TRE_LAYER_MOE)
      return fail(TRE_ERR_UNSUPPORTED, "FP4 weights are implemented for the routed experts of MoE stacks");
    if (c.max_tokens_per_step > 1)
      return fail(TRE_ERR_UNSUPPORTED, "FP4 experts are implemented for one token per step");
    if (c.hidden % 32 || c.expert_ffn % 32)
      return fail(TRE_ERR_UNSUPPORTED, "FP4 experts need hidden and expert_ffn multiples of 32");
  }
  if (c.weight_format == TRE_WEIGHTS_FP8_BLOCK128) {
    if (c.kind != TRE_LAYER_GQA)
      return fail(TRE_ERR_UNSUPPORTED, "FP8 weights are implemented for GQA stacks only");
    if (c.max_tokens_per_step > 1)
      return fail(TRE_ERR_UNSUPPORTED, "FP8 weights are implemented for one token per step");
    if (c.hidden % 16 || c.ffn % 16)
      return fail(TRE_ERR_UNSUPPORTED, "FP8 weights need hidden and ffn multiples of 16");
  }
  if (!(c.rope_theta > 0.f)) return fail(TRE_ERR_INVALID_ARG, "rope_theta must be > 0");
  if (!(c.norm_eps >= 0.f)) return fail(TRE_ERR_INVALID_ARG, "norm_eps must be >= 0");
  if (c.dep_timeout_us < 0) return fail(TRE_ERR_INVALID_ARG, "dep_timeout_us < 0");
  if (c.multi_token_gemv < 0 || c.multi_token_gemv > 2)
    return fail(TRE_ERR_INVALID_ARG, "multi_token_gemv must be 0, 1 or 2");
  if (c.stream_policy < 0 || c.stream_policy > 6)
    return fail(TRE_ERR_INVALID_ARG, "stream_policy must be in [0, 6]");
  if (c.gemv_kpart_max < 0 || (c.gemv_kpart_max > 0 && c.gemv_kpart_max < 512))
    return fail(TRE_ERR_INVALID_ARG, "gemv_kpart_max must be 0 or >= 512");
  if (c.num_sms < 0 || c.kv_splits < 0 || c.stage_bytes < 0 || c.ring_stages < 0)
    return fail(TRE_ERR_INVALID_ARG, "negative launch-shape field");
  if (c.stage_bytes && (c.stage_bytes % 1024 || c.stage_bytes > kMaxStageBytes))
    return fail(TRE_ERR_INVALID_ARG, "stage_bytes must be a multiple of 1024, <= 65536");
  return TRE_OK;
}

tre_status plan_build(const tre_config& c, int nsm, int smem_limit, PlanShape* shape,
                      std::vector<Task>* tasks_out, std::vector<int32_t>* sm_begin,
                      std::vector<int64_t>* sm_bytes) {
  tre_status st = validate(c);
  if (st != TRE_OK) return st;
  if (nsm < 1) return fail(TRE_ERR_INVALID_ARG, "no SMs to plan for");
  if (smem_limit > kSmemLimit) smem_limit = kSmemLimit;

  PlanShape s{};
  s.kind = c.kind;
  const bool mla = c.kind == TRE_LAYER_MLA;
  s.d = c.hidden;
  s.Hq = c.n_q_heads;
  s.Hkv = mla ? 1 : c.n_kv_heads;
  s.D = mla ? 0 : c.head_dim;
  if (mla) {
    s.QL = c.q_lora;
    s.KL = c.kv_lora;
    s.R = c.rope_dim;
    s.NP = c.nope_dim;
    s.VD = c.v_dim;
    if (c.index_topk > 0) {
      s.HI = c.index_heads;
      s.DI = c.index_dim;
      s.KI = c.index_topk;
      s.isplits = nsm;
    }
  }
  // an MLA output projection (K = H * v_dim) is staged in halves of at most 8192 inputs,
  // so that the input planes leave room for a 5-deep ring of 36 KB stages; with M tokens
  // per step the M input vectors share the planes
  s.M = c.max_tokens_per_step < 1 ? 1 : c.max_tokens_per_step;
  // E4M3 plans: K-parts of at most 8192 columns, so that a long row (the down projection)
  // leaves 4 rows to a stage and its input operand leaves room for the ring
  s.kpart_max = mla || c.weight_format == TRE_WEIGHTS_FP8_BLOCK128
                    ? 8192 : (kMaxKPart / s.M) / 16 * 16;  // 16: tile k-steps
  // multi-token GEMV form: tensor-core tiles cost the same per stage whatever the token
  // count, CUDA-core rows grow with it (measured on the 8B-shaped stack: rows faster at 2
  // and 3 tokens, tiles at 4)
  const bool tiles_fit = c.hidden % 16 == 0 && c.ffn % 16 == 0;
  s.tiles = s.M > 1 && (c.multi_token_gemv == 2 ||
                        (c.multi_token_gemv == 0 && s.M >= kTileMinTokens && tiles_fit));
  if (c.gemv_kpart_max > 0) s.kpart_max = std::min(s.kpart_max, c.gemv_kpart_max / 16 * 16);
  s.F = c.ffn;
  s.V = c.has_embed_lm_head ? c.vocab : 0;
  s.L = c.n_layers;
  s.cap = c.kv_capacity;
  s.nsm = nsm;
  s.has_lm = c.has_embed_lm_head;
  const bool moe = c.kind == TRE_LAYER_MOE;
  if (moe) {
    s.F = 0;
    s.E = c.n_experts;
    s.topk = c.top_k;
    s.nshared = c.n_shared;
    s.Fe = c.expert_ffn;
  }
  s.u_floats = moe ? (s.nshared + s.topk) * s.Fe : s.F;
  // MoE down row blocks: enough (slot, block) tasks to cover the SMs once
  if (moe) s.down_blocks = std::max(1, std::min(s.d / 8, nsm / (s.nshared + s.topk)));
  // MLA output projection: its K-parts as slices on different SMs, row blocks to cover the
  // SMs once (up to 255 blocks and slices: the task's aux fields)
  if (mla) {
    const int np = gemv_nparts(s.Hq * s.VD, s.kpart_max);
    if (np > 1 && np <= 255) {
      s.mo_slices = np;
      s.down_blocks = std::max(1, std::min({s.d / 8, nsm / np, 255}));
    }
  }
  const int G = s.Hq / s.Hkv;

  // Inputs longer than kMaxKPart are staged in K-parts; ops that normalise their input
  // (QKV, gate/up, LM head) need the whole vector at once.
  if (s.d > s.kpart_max)
    return fail(TRE_ERR_UNSUPPORTED, "hidden above 16384 / tokens per step (normalised inputs are staged whole)");
  // (input length, segments, K-part length) of every op the stack uses
  // E4M3 projections (GQA): QKV, O, gate/up and down rows are 1 byte per weight
  s.wfp8 = c.weight_format == TRE_WEIGHTS_FP8_BLOCK128;
  s.wfp4 = c.weight_format == TRE_WEIGHTS_FP4_EXPERTS;
  const int pesz = s.wfp8 ? 1 : 2;  // bytes per weight of the layer projections
  struct OpShape { int K, nseg, kp, esz; };
  std::vector<OpShape> ops = {{s.d, 1, 0, pesz}, {s.Hq * s.D, 1, 0, pesz}, {s.d, 1, s.d, 2}};
  if (mla) {
    ops = {{s.d, 1, s.d, 2}, {s.QL, 1, s.QL, 2}, {s.KL, 1, s.KL, 2}, {s.Hq * s.VD, 1, 0, 2},
           {s.NP, 1, s.NP, 2}};
    if (s.has_lm) ops.push_back({s.d, 1, s.d, 2});
  } else if (moe) {
    ops.push_back({s.d, 2, 0, 2});                               // shared / routed gate-up
    ops.push_back({(s.nshared + s.topk) * s.Fe, 1, s.Fe, 2});    // MoE down: one part per expert
  } else {
    ops.push_back({s.d, 2, 0, pesz});
    ops.push_back({s.F, 1, 0, pesz});
  }
  // a stage holds one attention tile: 64 K and V rows (GQA) or 32 latent rows (MLA; sparse:
  // 32 gathered rows at a padded pitch, or kIndexRows index keys)
  int xs = 8, need = mla ? (s.KL + s.R) * kMlaPosPerStage * 2 : 4 * s.D * kMaxPosPerStage;
  if (s.KI) need = std::max({need, kMlaPosPerStage * sparse_lat_pitch(s.KL + s.R),
                             kIndexRows * s.DI * 2});
  for (auto& o : ops) {
    const int kp = o.kp ? o.kp : gemv_part_len(o.K, gemv_nparts(o.K, s.kpart_max),
                                               gemv_part_align(s.tiles, o.esz == 1));
    // E4M3 rows: the tensor-core operand of the input covers the 4 row segments
    xs = std::max(xs, o.esz == 1 ? fp8_frag_floats(kp) + kFp8RedFloats : kp);
    need = std::max(need, s.tiles ? kTileRows * kTilePitch
                                  : o.esz == 1 ? o.nseg * fp8_row_pitch(kp) : o.nseg * kp * o.esz);
  }
  // A ring stage holds whole rows of one K-part (gate/up: a row of each matrix), or the K
  // and V rows of 8-64 cached positions.
  int sb = c.stage_bytes ? c.stage_bytes : std::max(kDefaultStageBytes, (need + 1023) / 1024 * 1024);
  // E4M3 plans: a stage of 8 hidden-wide rows (one full tensor-core tile; gate / up: 4 row
  // pairs) when that is at least the default
  if (!c.stage_bytes && s.wfp8 && 8 * fp8_row_pitch(s.d) >= sb)
    sb = (8 * fp8_row_pitch(s.d) + 1023) / 1024 * 1024;  // ring slots stay 1024-byte aligned
  if (!c.stage_bytes)
    while (sb < need && sb < kMaxStageBytes) sb += 1024;
  if (sb < need)
    return fail(TRE_ERR_UNSUPPORTED, "a weight row part (or gate/up row pair) is wider than a ring stage");
  s.stage_bytes = sb;
  // positions per attention stage: MLA 32 latent rows; GQA 64 (four warps x 16 rows)
  s.pos_per_stage = mla ? kMlaPosPerStage : kMaxPosPerStage;

  // KV splits: enough (kv head, split) tasks to cover the SMs, but no split shorter than
  // one stage of positions at full capacity.  MLA: (head group, split) tasks.
  const int units = mla ? s.Hq / kMlaHeadGroup : s.Hkv;
  int S = c.kv_splits;
  if (!S) {
    S = std::max(1, nsm / units);
    int max_s = std::max(1, (s.cap - 1 + s.pos_per_stage - 1) / s.pos_per_stage);  // >= 1 stage each
    S = std::min(S, max_s);
  }
  if (!mla && S > 4 * s.D) return fail(TRE_ERR_UNSUPPORTED, "kv_splits above 4 * head_dim");

  s.xs_floats = (s.M * xs + 7) / 8 * 8;
  s.resid_floats = s.M * kMaxResidRows;

  // attention scratch: q rows (M tokens x G heads), the M new k / v rows, per-warp
  // (m, l, O) per row, scores of the new positions
  const int rows = s.M * G;
  s.attn_floats = rows * s.D + 2 * s.M * s.D + kConsumerWarps * (2 * rows + rows * s.D) +
                  rows * s.M + 16;
  if (mla) {
    // score partials [8 warps][16][32] + P hi / lo (16 x 40 bf16 each) + head state; the
    // combine stages (m, l) of every split; the W_uk contraction sums [8][KL]
    const int Smax = std::max(1, nsm / (s.Hq / kMlaHeadGroup));
    s.attn_floats = std::max(kConsumerWarps * kMlaHeadGroup * 36 + 640 + 128,
                             2 * kMlaHeadGroup * Smax);
    s.attn_floats = std::max(s.attn_floats, kConsumerWarps * s.KL + s.NP + 64);
    // index scoring: the score histogram, the bf16 query tile [H_I][D_I], the head weights,
    // the new position's per-warp sums
    if (s.KI)
      s.attn_floats = std::max({s.attn_floats, kIndexBins + kIndexMaxHeads * 128 / 2 +
                                                   kIndexMaxHeads + 64,
                                16 + 512 + 2 * kPickSmemKeys});  // the pick's keys
  }
  const int ubuf_floats = (std::max(s.xs_floats + s.resid_floats + (s.tiles ? kTileRedFloats : 0),
                                     s.attn_floats) + 7) / 8 * 8;
  s.ub_floats = ubuf_floats;
  const int misc_bytes = 1024;
  const int fixed = ubuf_floats * 4 + misc_bytes;
  int ns = c.ring_stages;
  if (!ns) ns = std::min(16, (smem_limit - fixed - 1024) / (sb + 20));
  if (ns < 2) return fail(TRE_ERR_UNSUPPORTED, "shared memory too small for a 2-stage ring");
  s.ring_stages = ns;
  s.smem_bytes = ns * sb + ((2 * ns * 8 + ns * 4 + 127) / 128) * 128 + fixed;
  if (s.smem_bytes > smem_limit)
    return fail(TRE_ERR_UNSUPPORTED, "ring + buffers exceed the shared memory per block");

  if (mla && 2 * kMlaHeadGroup * S > s.attn_floats)
    return fail(TRE_ERR_UNSUPPORTED, "kv_splits too large for the MLA combine");
  s.kv_splits = S;

  Builder b(nsm);
  b.kpart_max = s.kpart_max;
  b.esz_proj = pesz;
  b.fp4 = s.wfp4 != 0;
  b.nshared = s.nshared;
  int prev_down = -1;
  uint32_t prev_down_count = 0;
  for (int l = 0; l < s.L && mla; ++l) {
    // absorbed MLA: down-projections -> q up-projection -> per-head W_uk contraction (+ the
    // latent append) -> attention over the latent cache -> per-head W_uv -> W_o + residual
    const int cdq = counter_of(l, C_QKV), cuq = counter_of(l, C_MLA_UQ),
              cuk = counter_of(l, C_MLA_UK), ca = counter_of(l, C_ATTN),
              cuv = counter_of(l, C_MLA_UV), co = counter_of(l, C_O);
    const int big = 1 << 30, C = s.KL + s.R, H = s.Hq, groups = H / kMlaHeadGroup;
    // sparse: the down-projection also yields the index key and head weights, the q
    // up-projection the index queries; index scoring tasks (after the q up-projection)
    // score every cached position, selection tasks keep the top K, and the attention
    // waits for the selection (whose last task also waits for the W_uk contraction)
    const int n1 = b.gemv(OP_MDQKV, l, s.QL + C + (s.KI ? s.DI + s.HI : 0), s.d, 1, prev_down,
                          prev_down_count, cdq, big);
    const int n2 = b.gemv(OP_UQ, l, H * (s.NP + s.R) + s.HI * s.DI, s.QL, 1, cdq, (uint32_t)n1,
                          cuq, big);
    const int cix = counter_of(l, C_MLA_IDX), csel = counter_of(l, C_MLA_SEL);
    if (s.KI)
      b.splits(T_INDEX, l, s.isplits, (int64_t)s.cap / s.isplits * s.DI * 2, cuq, (uint32_t)n2,
               cix);
    const int n3 = b.per_unit(OP_UK, l, H, s.NP, (int64_t)s.NP * s.KL * 2, cuq, (uint32_t)n2, cuk);
    if (s.KI) b.splits(T_ISEL, l, s.isplits, 0, cix, (uint32_t)s.isplits, csel);
    const int64_t lat_task =
        (int64_t)((s.KI ? std::min(s.KI, s.cap) : s.cap) - s.M) / S * C * 2;
    if (s.KI) b.mla_attention(l, groups, S, lat_task, csel, 1u, ca);
    else b.mla_attention(l, groups, S, lat_task, cuk, (uint32_t)n3, ca);
    const int n5 = b.per_unit(OP_UV, l, H, s.VD, (int64_t)s.VD * s.KL * 2, ca,
                              (uint32_t)(groups * S), cuv);
    // W_o (K = H v_dim) in K-slices: the slices of a row block run on different SMs and the
    // last to finish adds them to the residual (one K-part per SM instead of two in a row)
    const int n6 = s.mo_slices > 1
                       ? b.mo_slices(l, s.d, H * s.VD, s.mo_slices, s.down_blocks, cuv,
                                     (uint32_t)n5, co)
                       : b.gemv(OP_MO, l, s.d, H * s.VD, 1, cuv, (uint32_t)n5, co, kMaxResidRows);
    prev_down = co;
    prev_down_count = (uint32_t)n6;
  }
  for (int l = 0; l < s.L && !mla; ++l) {
    const int cq = counter_of(l, C_QKV), ca = counter_of(l, C_ATTN), co = counter_of(l, C_O),
              cg = counter_of(l, C_GU), cd = counter_of(l, C_DOWN);
    // Q, K and V as one op over the stacked matrix [Wq; Wk; Wv]
    const int big = 1 << 30;
    const int nqkv = b.gemv(OP_QKV, l, (s.Hq + 2 * s.Hkv) * s.D, s.d, 1, prev_down,
                            prev_down_count, cq, big);
    const int64_t kv_task_bytes = (int64_t)(s.cap - s.M) / S * s.D * 2 * 2;
    b.attention(l, s.Hkv, S, kv_task_bytes, cq, (uint32_t)nqkv, ca);
    // the last split of each kv head to finish combines the head's splits and publishes
    int no = b.gemv(OP_O, l, s.d, s.Hq * s.D, 1, ca, (uint32_t)s.Hkv, co, kMaxResidRows);
    int nd;
    if (!moe) {
      int ng = b.gemv(OP_GU, l, s.F, s.d, 2, co, (uint32_t)no, cg, big);
      nd = b.gemv(OP_DOWN, l, s.d, s.F, 1, cg, (uint32_t)ng, cd, kMaxResidRows);
    } else {
      // Router rows first, then the shared expert (which needs no routing, so its weights
      // stream while the top-k is decided), then the selected experts' gate/up rows: their
      // producer waits for the route counter, since the expert ids pick the addresses.
      const int cr = counter_of(l, C_ROUTE);
      const int first = b.next_id;
      const int nr = b.gemv(OP_ROUTER, l, s.E, s.d, 1, co, (uint32_t)no, cr, big);
      b.set_count(first, OP_ROUTER, nr);
      int ng = 0;
      if (s.nshared > 0) ng += b.gemv(OP_SGU, l, s.nshared * s.Fe, s.d, 2, co, (uint32_t)no, cg, big);
      ng += b.gemv(OP_RGU, l, s.topk * s.Fe, s.d, 2, cr, 1u, cg, big, 0, s.Fe);
      // down: one task per (expert slot j, row block); slot j reads the j-th Fe-slice of u
      // (shared slices first, then the selected experts).  Each task writes its partial
      // rows; the last of a block's slots to finish sums them (fixed slot order) with h1
      // into x and bumps the down counter once per block.
      nd = b.moe_down(l, s.d, s.nshared + s.topk, s.Fe, s.down_blocks, cg, (uint32_t)ng, cd);
    }
    prev_down = cd;
    prev_down_count = (uint32_t)nd;
  }
  const int c_lm = s.L * C_PER_LAYER, c_fault = c_lm + 1;
  s.n_counters = c_lm + 2;
  if (s.has_lm) {
    int first = b.next_id;
    int nlm = b.gemv(OP_LM, s.L - 1, s.V, s.d, 1, prev_down, prev_down_count, c_lm, 1 << 30);
    s.n_lm_tasks = nlm;
    b.set_count(first, OP_LM, nlm);
  }
  if (c.debug_flags & TRE_DEBUG_FAULT_INJECT) {
    // the first O-projection task of layer 0 waits on a counter nothing bumps
    for (auto& qq : b.q) {
      bool done = false;
      for (auto& t : qq)
        if (t.type == T_GEMV && t.op == OP_O && t.layer == 0) {
          t.dep = c_fault;
          t.dep_count = 1;
          done = true;
          break;
        }
      if (done) break;
    }
  }

  tasks_out->clear();
  sm_begin->assign(nsm + 1, 0);
  size_t mx = 0;
  for (int i = 0; i < nsm; ++i) {
    (*sm_begin)[i] = (int32_t)tasks_out->size();
    tasks_out->insert(tasks_out->end(), b.q[i].begin(), b.q[i].end());
    mx = std::max(mx, b.q[i].size());
  }
  (*sm_begin)[nsm] = (int32_t)tasks_out->size();
  if (sm_bytes) *sm_bytes = b.cum;
  *shape = s;
  (void)mx;
  return TRE_OK;
}

// Kernel-per-op form of a plan: the op groups (maximal runs of tasks, in global task
// order, of one layer, task type and op) and, per group and SM, the contiguous range of
// that SM's queue holding the group's tasks ([G][nsm][2] into the task array; empty
// ranges where an SM has none).  Returns G, or -1 if some SM's tasks of a group are not
// contiguous in its queue (the planner never builds such a plan).
int plan_op_groups(const std::vector<Task>& tasks, const std::vector<int32_t>& sm_begin, int nsm,
                   std::vector<int32_t>* ranges) {
  const int n = (int)tasks.size();
  std::vector<int> at(n, -1);  // queue index of each task id
  for (int i = 0; i < n; ++i) {
    if (tasks[i].id < 0 || tasks[i].id >= n || at[tasks[i].id] >= 0) return -1;
    at[tasks[i].id] = i;
  }
  std::vector<int> group(n, 0);  // by queue index
  int G = 0;
  for (int id = 0; id < n; ++id) {
    const Task& t = tasks[at[id]];
    if (id == 0) {
      G = 1;
    } else {
      const Task& u = tasks[at[id - 1]];
      if (t.layer != u.layer || t.type != u.type || t.op != u.op) ++G;
    }
    group[at[id]] = G - 1;
  }
  ranges->assign((size_t)G * nsm * 2, 0);
  for (int s = 0; s < nsm; ++s) {
    for (int g = 0; g < G; ++g) {
      (*ranges)[2 * ((size_t)g * nsm + s)] = sm_begin[s];
      (*ranges)[2 * ((size_t)g * nsm + s) + 1] = sm_begin[s];
    }
    int prev = -1;
    for (int i = sm_begin[s]; i < sm_begin[s + 1]; ++i) {
      const int g = group[i];
      int32_t* r = ranges->data() + 2 * ((size_t)g * nsm + s);
      if (g != prev) {
        if (g < prev) return -1;
        r[0] = i;
        prev = g;
      }
      r[1] = i + 1;
    }
  }
  return G;
}

int64_t step_bytes(const PlanShape& s, int pos, int m) {
  const int64_t d = s.d, D = s.D;
  if (s.kind == TRE_LAYER_MLA) {
    const int64_t H = s.Hq, C = s.KL + s.R;
    const int64_t w = (s.QL + C) * d + H * (s.NP + s.R) * s.QL +
                      H * s.NP * s.KL + H * s.VD * s.KL + d * H * s.VD;
    const int64_t wi = s.KI ? (int64_t)s.HI * s.DI * s.QL + (int64_t)(s.DI + s.HI) * d : 0;
    int64_t bytes = ((w + wi) * 2 + (d + s.QL + s.KL) * 2) * s.L;   // weights and norm gains
    if (s.KI && pos + 1 > s.KI) {
      // sparse: the index keys read + this one written, the K chosen latent rows read (the
      // new one from on chip when chosen) + this position's written
      bytes += (int64_t)s.L * ((int64_t)(pos + 1) * s.DI * 2 + (int64_t)(s.KI + 1) * C * 2);
    } else {
      bytes += (int64_t)s.L * (pos + 1) * C * 2;              // latent rows read + written
      if (s.KI) bytes += (int64_t)s.L * (pos + 1) * s.DI * 2;  // the index keys too
    }
    if (s.has_lm) bytes += (int64_t)s.V * d * 2 + d * 2 + d * 2 + (int64_t)s.V * 4;
    return bytes;
  }
  // MoE: the router, the shared experts and the selected experts only (what one token reads)
  const int64_t mlp = s.kind == TRE_LAYER_MOE
                          ? (int64_t)s.E * d + 3LL * (s.nshared + s.topk) * s.Fe * d
                          : 3LL * s.F * d;
  const int64_t proj = (int64_t)(s.Hq + 2 * s.Hkv) * D * d + d * s.Hq * D + mlp;
  int64_t per_layer = proj * 2 + 2 * d * 2;
  if (s.wfp4)  // the selected experts' rows are MXFP4 rows instead of bf16
    per_layer += (int64_t)s.topk * (2LL * s.Fe * fp4_row_pitch(d) + (int64_t)d * fp4_row_pitch(s.Fe) -
                                    3LL * s.Fe * d * 2);
  if (s.wfp8) {  // E4M3 bytes plus one fp32 scale per 128 x 128 block of every matrix
    auto blocks = [](int64_t N, int64_t K) { return ((N + 127) / 128) * ((K + 127) / 128); };
    const int64_t nq = (int64_t)s.Hq * D, nk = (int64_t)s.Hkv * D;
    per_layer = proj + 4 * (blocks(nq, d) + 2 * blocks(nk, d) + blocks(d, nq) +
                            2 * blocks(s.F, d) + blocks(d, s.F)) + 2 * d * 2;
  }
  int64_t bytes = per_layer * s.L;
  bytes += (int64_t)s.L * s.Hkv * (int64_t)pos * D * 2 * 2;  // K and V read
  bytes += (int64_t)s.L * s.Hkv * D * 2 * 2 * m;             // the m tokens' K and V written
  if (s.has_lm) bytes += (int64_t)s.V * d * 2 + d * 2 + m * (d * 2 + (int64_t)s.V * 4);
  return bytes;
}

}  // namespace tre
