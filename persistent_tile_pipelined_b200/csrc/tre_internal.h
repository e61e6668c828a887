// Internal types of the engine shared by the host planner (planner.cpp), the C ABI
// (tre_api.cu) and the persistent kernel (engine.cu).
#pragma once
#include <stdint.h>

#include "tre.h"

namespace tre {

// ---- compile-time shape of the persistent CTA -------------------------------------
constexpr int kConsumerWarps = 8;                      // compute warps
constexpr int kConsumerThreads = kConsumerWarps * 32;  // 256
constexpr int kThreads = kConsumerThreads + 32;        // + one producer warp
constexpr int kMaxGroup = 8;                           // q heads per kv head (GQA)
constexpr int kMaxPosPerStage = 64;                    // GQA attention stage: 4 warps x 16 rows
constexpr int kDefaultStageBytes = 32768;  // a bulk-copy stage costs ~0.4 us per SM: keep them large
constexpr int kMaxKPart = 16384;         // longest input slice one GEMV task stages (floats)
constexpr int kMaxResidRows = 512;       // rows per task of ops that add a residual
constexpr int kTraceCols = 8;          // int64 per task in the debug trace
constexpr int kMaxExperts = 512;         // routed experts per MoE layer (scores fit the
                                         // residual-row buffer for the top-k)
constexpr int kMaxTopK = 32;
constexpr int kDefaultPrefetchKB = 0;    // next-task L2 prefetch: opt-in (measured 4% slower)
constexpr int kMaxStageBytes = 65536;
constexpr int kMaxTokens = 4;            // tokens per step (multi-token verify tiles)
// Dependency counters sit kCtrStride words apart (packed: padding them to 128 bytes each
// measured no different)
constexpr int kCtrStride = 1;
// Multi-token GEMV on tensor cores: a stage is one tile of 16 weight rows x up to 1024
// input columns, each row copied into a 16-byte-padded slot (conflict-free ldmatrix).
constexpr int kTileRows = 16;
constexpr int kTileMinTokens = 4;                      // the planner's choice of tiles from here
constexpr int kTileK = 1024;
constexpr int kTilePitch = kTileK * 2 + 16;            // bytes per row slot
constexpr int kTileRedFloats = 2 * 2 * kConsumerWarps * kTileRows * kMaxTokens;  // [2 bufs][2 segs]...
constexpr int kSmemLimit = 232448;                     // sm_100 opt-in max per block

#ifdef __CUDACC__
#define TRE_HD __host__ __device__
#else
#define TRE_HD
#endif

// ---- GEMV stage geometry ----------------------------------------------------------------
// A GEMV stage holds `rows per stage` whole contiguous rows of the op's matrix (gate/up:
// the same rows of both matrices); one consumer warp computes the whole stage.
// Rows longer than kMaxKPart are cut into K-parts: part j of a task covers input columns
// [j * len, min(K, (j + 1) * len)); the parts of one row range are consecutive tasks on
// one SM, the first adds the residual and later parts accumulate into the output.
TRE_HD inline int gemv_nparts(int K, int kmax = kMaxKPart) { return (K + kmax - 1) / kmax; }
TRE_HD inline int gemv_part_len(int K, int nparts, int align = 8) {
  const int l = (K + nparts - 1) / nparts;
  return (l + align - 1) / align * align;
}
// esz: bytes per weight element (2 bf16, 1 E4M3)
TRE_HD inline int gemv_rows_per_stage(int K, int nseg, int stage_bytes, int esz = 2) {
  const int r = stage_bytes / (nseg * K * esz);
  return r < 1 ? 1 : r;
}
// K-part boundaries: multiples of 8 columns (16 bytes of bf16), of 16 for tensor-core
// tiles, of 128 for E4M3 rows (a K-part then covers whole 128-column scale blocks)
TRE_HD inline int gemv_part_align(bool tiles, bool fp8) { return fp8 ? 128 : tiles ? 16 : 8; }
// E4M3 rows on the tensor cores are read as 2 halves of fp8_half_len(Kp) columns (a
// multiple of 32: the tiles take 32 columns of both halves at a time); the input operand
// covers both (fp8_span columns, zero past Kp).  Rows sit at a pitch of span + 16 bytes, an
// odd number of 16-byte units, so that an ldmatrix's 8 rows hit 8 different bank groups.
TRE_HD inline int fp8_half_len(int Kp) { return (Kp + 63) / 64 * 32; }
TRE_HD inline int fp8_span(int Kp) { return 2 * fp8_half_len(Kp); }
TRE_HD inline int fp8_row_pitch(int Kp) { return fp8_span(Kp) + 16; }
// The input operand of an E4M3 GEMV: 4 E4M3 terms per input (4 bytes) in fragment order,
// then one scale per 32 columns: its size in floats (the cross-warp sums follow it)
TRE_HD inline int fp8_frag_floats(int Kp) { return fp8_span(Kp) + fp8_span(Kp) / 32; }
constexpr int kFp8RedFloats = 2 * kConsumerWarps * 8;
// MXFP4 rows (FP4 routed experts): K/2 bytes of E2M1 codes, then K/32 E8M0 scale bytes,
// padded to a multiple of 16 bytes; rows are stored, copied and staged at this pitch
TRE_HD inline int fp4_row_pitch(int K) { return (K / 2 + K / 32 + 15) / 16 * 16; }
TRE_HD inline int fp8_rows_per_stage(int Kp, int nseg, int stage_bytes) {
  const int r = stage_bytes / (nseg * fp8_row_pitch(Kp));
  return r < 1 ? 1 : r;
}

// ---- tasks --------------------------------------------------------------------------
enum TaskType : uint8_t { T_GEMV = 0, T_ATTN = 1, T_MLA_ATTN = 2, T_INDEX = 3, T_ISEL = 4 };

// GEMV ops: which matrix, which input vector, which epilogue.
enum GemvOp : uint8_t {
  OP_QKV = 0,     // in: RMSNorm(x; attn_norm)  -> qkv = [Wq; Wk; Wv] xn  (rows of the stacked matrix)
  OP_O = 1,       // in: attn                   -> h1 = x + Wo attn
  OP_GU = 2,      // in: RMSNorm(h1; ffn_norm)  -> u = silu(Wg hn) * (Wu hn)   (2 segments)
  OP_DOWN = 3,    // in: u                      -> x = h1 + Wd u
  OP_LM = 4,      // in: RMSNorm(x; final_norm) -> logits, greedy argmax
  OP_ROUTER = 5,  // in: hn                     -> scores = sigmoid(Wr hn); last task: top-k
  OP_SGU = 6,     // in: hn                     -> u[0, Fs) = shared expert silu(g) * u
  OP_RGU = 7,     // in: hn                     -> u[Fs + j Fe + r] = w_j silu(g) * u of the
                  //                               j-th selected expert (virtual row j Fe + r)
  OP_MDOWN = 8,   // in: u slice j              -> partial rows of slot j (a shared-expert
                  //                               slice or a selected expert); the block's
                  //                               last slot sums x = h1 + sum_j partial_j
  // absorbed MLA (attention-only layers)
  OP_MDQKV = 9,   // in: RMSNorm(x; attn_norm)  -> cqkv = [Wdq; Wdkv] xn  (c_q, then c_kv | k_pe)
  OP_UQ = 10,     // in: RMSNorm(c_q; q_norm)   -> q = Wuq c_q  (per head: nope, rope)
  OP_UK = 11,     // in: q_nope of one head     -> q_lat = Wuk_h^T q_nope (rows contracted);
                  //                               also RoPE(q_pe); head 0 appends the latent
  OP_UV = 12,     // in: o_lat of one head      -> o = Wuv_h o_lat
  OP_MO = 13,     // in: o                      -> x = x + Wo o
  OP_MOS = 14,    // in: o, K-slice j           -> partial rows of slice j of a row block
                  //                               (aux = j | block << 8 | slices << 16); the
                  //                               block's last slice sums x = x + sum_j partial_j
  OP_COUNT = 15
};

// MLA counters reuse the per-layer slots: QKV = down-projections, ATTN, O = output
// projection, and these three.
enum MlaCounter { C_MLA_UQ = 3, C_MLA_UK = 4, C_MLA_UV = 5, C_MLA_IDX = 6, C_MLA_SEL = 7 };
// Sparse MLA (the lightning-indexer reading): index scoring tasks stream the index-key
// cache in stages of kIndexRows positions (64-column swizzled boxes, like the latent
// stages) and histogram the scores on the top kIndexBinBits bits of their order key; the
// chosen positions' latent rows are gathered by per-row bulk copies into stages of
// kMlaPosPerStage rows at a padded pitch (conflict-free ldmatrix without the swizzle).
constexpr int kIndexRows = 128;
constexpr int kIndexBinBits = 12;
constexpr int kIndexBins = 1 << kIndexBinBits;
constexpr int kIndexMaxHeads = 64;
constexpr int kPickSmemKeys = 3840;  // threshold-bin candidates the pick keeps in shared memory
TRE_HD inline int sparse_lat_pitch(int C) { return C * 2 + 16; }  // bytes per gathered row
// Per-layer selection state (uint32 words): the chosen-position count, the candidate
// count, whether the new position was chosen, and the selection tasks' arrival ticket.
enum IndexMeta { IM_NSEL = 4, IM_NCAND = 5, IM_HASPOS = 6, IM_TICK_B = 8, IM_WORDS = 16 };
constexpr int kMlaHeadGroup = 16;     // query heads per MLA attention tile (the mma M)
constexpr int kMlaPosPerStage = 32;   // latent rows per MLA attention stage
constexpr int kMlaBox = 64;           // latent columns per tensor-map box (128 B, swizzled)
constexpr int kMlaMaxKSteps = 6;      // 16-column k-steps of the score product per warp
// floats per MLA split partial: O (KL), m, l, 2 pad -> every row starts on 16 bytes
TRE_HD inline int mla_pstride(int KL) { return KL + 4; }
// floats per GQA split partial: O (D), m, l, 2 pad -> every row starts on 16 bytes (the O
// projection reads the partials with 16-byte loads while it combines them)
TRE_HD inline int gqa_pstride(int D) { return D + 4; }

// Dependency counters: one per (layer, stage of the layer), then the LM head and a
// counter nothing ever bumps (used only by the fault-injection debug plan).
// C_ROUTE (MoE) is bumped once per step by the router task that finishes last, after it
// has written the layer's selected experts and weights.
enum CounterKind { C_QKV = 0, C_ATTN = 1, C_O = 2, C_GU = 3, C_DOWN = 4, C_ROUTE = 5,
                   C_PER_LAYER = 8 };

struct Task {          // 32 bytes, 16-byte aligned array
  uint8_t type;        // TaskType
  uint8_t op;          // GemvOp (T_GEMV)
  uint16_t layer;
  int32_t dep;         // counter to wait on, -1 = none
  uint32_t dep_count;  // increments of `dep` per step
  int32_t out;         // counter to bump when done, -1 = none
  int32_t r0, r1;      // GEMV: output rows [r0, r1).  ATTN: kv head, split index.
                       // INDEX / ISEL: -, split index
  int32_t aux;         // ATTN / INDEX / ISEL: number of splits.  LM / ROUTER: number of
                       // tasks of the op.
                       // other GEMV: K-part index | (number of K-parts << 8)
  int32_t id;          // global task index (trace rows, error detail)
};
static_assert(sizeof(Task) == 32, "task descriptor is 32 bytes");

struct LayerPtrs {     // device-side per-layer pointer table
  const uint16_t* w[TRE_W_SLOTS];
  uint16_t* k_cache;
  uint16_t* v_cache;   // MLA sparse: the index-key cache [cap][D_I]
};

// ---- the plan (host side) -----------------------------------------------------------
struct PlanShape {
  int kind;
  int d, Hq, Hkv, D, F, V, L, cap, M;
  int E, topk, nshared, Fe;  // MoE: experts, selected per token, shared, expert FFN
  int QL, KL, R, NP, VD;  // MLA: q_lora, kv_lora, rope, nope, v dims
  int HI, DI, KI;         // MLA sparse: index heads, index dim, positions kept (0: dense)
  int isplits;            // MLA sparse: index scoring tasks = selection tasks per layer
  int kpart_max;       // longest input slice of a GEMV task (floats)
  int tiles;           // multi-token plan: GEMV stages are 16-row tensor-core tiles
  int wfp8;            // GQA projections are E4M3 with 128 x 128 block scales
  int wfp4;            // MoE routed experts are MXFP4 rows
  int u_floats;        // the SwiGLU activation buffer (MoE: shared then routed slices)
  int down_blocks;     // MoE down / MLA output slices: row blocks (each summed by its last
                       // slot or slice to finish)
  int mo_slices;       // MLA output projection: K-slices on different SMs (0: one K-part)
  int nsm;
  int stage_bytes, ring_stages;
  int kv_splits, pos_per_stage;
  int xs_floats;       // input-vector buffer (floats): the longest K-part
  int resid_floats;    // residual rows staged per task (floats)
  int attn_floats;     // attention scratch (floats), aliases the input-vector buffer
  int ub_floats;       // the shared union buffer: input planes, or attention scratch
  int smem_bytes;
  int n_counters;
  int n_lm_tasks;
  int has_lm;
};

// ---- kernel parameters ----------------------------------------------------------------
struct Params {
  const Task* tasks;
  const int32_t* sm_begin;         // [nsm + 1] offsets into tasks
  // Kernel-per-op launches (the measurement form with the kernel boundary put back): this
  // launch runs op group `op_group` only, CTA b the tasks [op_ranges[2 (g nsm + b)],
  // op_ranges[2 (g nsm + b) + 1]) of p.tasks; op_group < 0: the whole step (the
  // persistent form).  Per-op launches wait on no counter (stream order meets every
  // dependency) and bump a counter array of their own, so that the persistent form's
  // counters always stand at epoch * count between steps.
  const int32_t* op_ranges;
  int op_group;
  uint32_t* counters;
  uint32_t* tickets;               // [Hkv] split-KV arrival tickets
  uint32_t* lm_ticket;
  unsigned long long* argmax_slot;  // [kMaxTokens]
  const LayerPtrs* layers;
  const uint16_t* embed;
  const uint16_t* final_norm;
  const uint16_t* lm_head;
  const float* x_in;               // layer-only input (NULL: embedding row)
  float* x_out;                    // layer-only output (NULL: none)
  // per-token buffers are [m][...] (token v's vector at v * length)
  float* x;                        // residual stream [d]
  float* h1;                       // after attention [d]
  float* qkv;                      // [(Hq + 2 Hkv) D]
  float* attn;                     // [Hq D]
  float* u;                        // [F] (MoE: [nshared Fe + topk Fe])
  float* scores;                   // MoE router scores [E]
  int32_t* route_idx;              // MoE selected experts [L][topk]
  float* route_w;                  // MoE normalised weights [L][topk]
  uint32_t* router_ticket;         // MoE: arrival ticket of the router tasks
  float* mpart;                    // MoE down partial rows [nshared + topk][d]
  // absorbed MLA
  float* cqkv;                     // [QL + KL + R]: c_q, then c_kv | k_pe (before norm / rope)
  float* qf;                       // [H][KL + R]: q_lat | RoPE(q_pe), per head
  float* lat_new;                  // [KL + R]: this token's latent row (bf16 values)
  float* o_lat;                    // [H][KL]
  float* mla_o;                    // [H * VD]
  // sparse MLA (HI > 0): per layer scores [L][cap], chosen positions [L][KI], threshold-bin
  // candidates [L][cap] (order key << 32 | ~position), score histograms [L][kIndexBins],
  // selection state [L][IM_WORDS]; index-cache tensor maps [L] (128 B each)
  float* iscore;
  int32_t* ix_sel;
  unsigned long long* ix_cand;
  uint32_t* ix_hist;
  uint32_t* ix_meta;
  const void* ix_maps;
  const void* kv_maps;             // tensor maps (128 B each): GQA / MoE [L][K, V] caches,
                                   // MLA [L] latent caches
  const double* rope_inv_freq_r;   // [R / 2]
  uint32_t* down_tickets;          // MoE down: arrival ticket per row block
  float* part;                     // [m][Hq][splits][gqa_pstride(D)] (MLA: mla_pstride)
  float* logits;                   // [V]
  int32_t* token_out;              // [1] or NULL
  float* hidden;                   // debug [L][d] or NULL
  long long* trace;                // debug [n_tasks][4] or NULL
  const double* rope_inv_freq;     // [D/2]
  int32_t* err;                    // device word: first error wins
  volatile int32_t* abort_flag;    // device word
  volatile int32_t* status_host;   // host-mapped [2]: code, detail
  int d, Hq, Hkv, D, F, V, L, cap;
  int E, topk, nshared, Fe;
  int QL, KL, R, NP, VD, kpart_max;
  int HI, DI, KI, isplits;
  int nsplit, pps, stage_bytes, ring_stages, xs_floats, ub_floats;
  float eps;
  int token, pos;
  const int32_t* token_in;         // device word holding token 0 (greedy loop), or NULL
  int m;                           // tokens this step (1 .. kMaxTokens): positions pos .. pos + m - 1
  int32_t tokens[kMaxTokens];
  uint32_t epoch;
  int flags;
  int hold_next_op;                // > 0: at op boundaries the producer issues hold_next_op - 1
                                   // stages, then waits for this SM's publish; 0: no wait
  int gemv_tiles;                  // GEMV stages are 16-row tiles (multi-token plans)
  int wfp8;                        // QKV / O / gate-up / down weights are E4M3 + block scales
  int wfp4;                        // routed experts' gate / up / down rows are MXFP4
  long long timeout_ns;
  long long pf_window;             // L2 prefetch bytes allowed beyond the ring (0 = off)
};

}  // namespace tre

// Planner entry (planner.cpp).  Fills shape, tasks (grouped per SM, topological order
// within each SM) and sm_begin.  Returns TRE_OK or an error with tre_set_error text.
#ifdef __cplusplus
#include <string>
#include <vector>
namespace tre {
tre_status plan_build(const tre_config& cfg, int nsm, int smem_limit, PlanShape* shape,
                      std::vector<Task>* tasks, std::vector<int32_t>* sm_begin,
                      std::vector<int64_t>* sm_bytes);
int64_t step_bytes(const PlanShape& s, int pos, int m = 1);
int plan_op_groups(const std::vector<Task>& tasks, const std::vector<int32_t>& sm_begin, int nsm,
                   std::vector<int32_t>* ranges);
void set_error(const std::string& msg);
// Host only, allocates nothing: a 2-D tensor map (128 bytes at out128) over a bf16 cache
// [rows][C] with 64-column x box_rows boxes and the 128-byte swizzle (tre_api.cu).
tre_status encode_cache_map(void* cache, int C, long long rows, int box_rows, void* out128);
}  // namespace tre
#endif
