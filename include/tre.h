/*
 * tre.h — C ABI of the persistent tile engine for batch-1 LLM decode (sm_100a).
 *
 * One decode step of a whole decoder stack runs as ONE persistent kernel launch that
 * executes a static, host-planned list of tile tasks.  Each task waits on a dependency
 * counter in global memory, streams its weight (or KV) tiles through a shared-memory
 * ring filled by a bulk-copy producer warp, computes, publishes its outputs and bumps
 * its output counter, so later tiles start as soon as the tiles they read are done.
 *
 * Sources (the pages describe the method only in prose; they print no formula):
 *   [SC]  "Static Compilation for LLM Inference: from ASIC Graph Compile to Persistent
 *         Engine Kernel" — §1 (the whole model is statically unrolled ahead of time into
 *         one Persistent Engine Kernel; the tile is the scheduling unit), §5.1 (tile
 *         pipeline: shared memory holds one tile at a time), §5.2 (warp-group roles:
 *         a TMA copy group stands in for the DMA engine, a compute group with the
 *         activation fused in), §5.4 table (bs=1 GEMM is memory bound, fuse norm+GEMM),
 *         §6 (launch overhead dominates bs=1 decode).
 *   [TA]  "TileRT code audit" (tile-ai-tilert page) — blog-vs-code table (host launches
 *         once; fused ops RMSNormProjxWqkvia, UnProjOAllReduce, ExpertSelectUpGateSiLU,
 *         ExpertDownAllReduce, FlashSparseMLA with batch == 1; inject_cache() takes an
 *         external KV cache as raw tensors).
 *   [SI]  "Speed is intelligence" talk transcript (TileRT team) — section on breaking
 *         the kernel boundary: tasks whose dependencies are met start early; the model
 *         is a dataflow graph lowered to tile micro-kernels and an execution engine.
 *
 * Conventions for every call:
 *   - All pointers named *_dev are device pointers on the engine's device; *_host are
 *     host pointers.  Weight and KV memory is OWNED BY THE CALLER and must outlive the
 *     engine; the engine never frees it.  The engine owns its plan, task list,
 *     counters, activation scratch and split-KV partial buffers.
 *   - Every call returns a tre_status.  Errors detectable on the host are returned
 *     before anything is enqueued.  Errors found on the device (a dependency wait that
 *     ran out of time, a bounds check) are recorded in a device status word: they are
 *     returned by the next tre_decode_step / tre_layers_step (which then launches
 *     nothing) and by tre_get_status; tre_reset clears them.
 *   - An engine is not thread safe: calls on one engine must not overlap.
 *   - Weights, embedding, norm gains and KV caches are bf16 (raw 16-bit words,
 *     round-to-nearest-even).  Activations, the residual stream, attention partials and
 *     logits are fp32.  Matrices are row-major W[N][K] (N outputs, K inputs), the
 *     layout of torch.nn.Linear.weight; every K must be a multiple of 8 (16-byte rows)
 *     and every pointer 16-byte aligned.
 */
#ifndef TRE_H
#define TRE_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tre_engine tre_engine;          /* opaque, library owned */
typedef struct CUstream_st* tre_stream;        /* a cudaStream_t (NULL = legacy default) */

typedef enum {
  TRE_OK = 0,
  TRE_ERR_INVALID_ARG = -1,   /* bad config value, NULL or misaligned pointer        */
  TRE_ERR_CUDA = -2,          /* a CUDA runtime call failed (see tre_last_error)     */
  TRE_ERR_OCCUPANCY = -3,     /* one CTA per SM cannot be co-resident                */
  TRE_ERR_DEP_TIMEOUT = -4,   /* a device wait ran out of time (device status word)  */
  TRE_ERR_POS_RANGE = -5,     /* pos (+ tokens) beyond the KV capacity               */
  TRE_ERR_UNSUPPORTED = -6,   /* config outside what the engine implements          */
  TRE_ERR_BOUNDS = -7,        /* device bounds check fired (device status word)      */
  TRE_ERR_STATE = -8          /* previous device error not yet cleared by tre_reset  */
} tre_status;

/* Layer kinds.  GQA: Llama-style pre-norm attention + SwiGLU MLP.  MOE: the same
 * attention with a routed mixture-of-experts MLP.  MLA: absorbed multi-head latent
 * attention only (pre-norm -> MLA -> residual, no MLP); the pages name the fused MLA
 * kernel FlashSparseMLA with batch == 1 (TileRT code audit, blog-vs-code table) and fold
 * query heads into one tile (Speed is intelligence talk, section on the attention
 * kernel); absorbed MLA is read as DeepSeek-V2's. */
enum { TRE_LAYER_GQA = 0, TRE_LAYER_MLA = 1, TRE_LAYER_MOE = 2 };

/* debug_flags bits */
enum {
  TRE_DEBUG_HIDDEN = 1,        /* keep the residual stream after every layer          */
  TRE_DEBUG_TRACE = 2,         /* record per-task start / ready / end timestamps      */
  TRE_DEBUG_FAULT_INJECT = 4,  /* plan one dependency that can never be met (tests the
                                  bounded-wait error path; the step returns
                                  TRE_ERR_DEP_TIMEOUT and the context stays usable)   */
  TRE_DEBUG_NO_OVERLAP = 8     /* producer waits for each task's dependency before
                                  streaming its tiles (removes cross-op prefetch; for
                                  measurement only)                                   */
};

typedef struct {
  int32_t kind;                 /* TRE_LAYER_*  (one kind for the whole stack)          */
  int32_t n_layers;
  int32_t hidden;               /* d                                                    */
  int32_t n_q_heads;            /* Hq (MLA: heads H, a multiple of 16)                  */
  int32_t n_kv_heads;           /* Hkv (GQA/MOE); Hq % Hkv == 0                         */
  int32_t head_dim;             /* D (GQA/MOE): 64 or 128                               */
  int32_t ffn;                  /* F, SwiGLU hidden (GQA)                               */
  int32_t vocab;                /* V (0 when has_embed_lm_head == 0)                    */
  int32_t q_lora, kv_lora, rope_dim, nope_dim, v_dim;          /* MLA: kv_lora a multiple
                                   of 128, rope_dim of 16, kv_lora + rope_dim of 64 and
                                   <= 768, q_lora / nope_dim / v_dim of 8               */
  int32_t n_experts, top_k, n_shared, expert_ffn;              /* MOE                   */
  int32_t kv_capacity;          /* positions allocated in each KV cache                 */
  int32_t max_tokens_per_step;  /* M, 0..4 (0 = 1): tokens tre_decode_tokens may take;
                                   GQA stacks with M x (q heads per kv head) <= 16      */
  float rope_theta;
  float norm_eps;
  int32_t has_embed_lm_head;    /* 1: token in, logits out; 0: hidden in, hidden out    */
  int32_t debug_flags;          /* TRE_DEBUG_*                                          */
  int32_t dep_timeout_us;       /* bound on every device wait; 0 = 1,000,000 us         */
  int32_t num_sms;              /* CTAs of the persistent grid; 0 = every SM            */
  int32_t kv_splits;            /* split-KV chunks per kv head; 0 = planner's choice    */
  int32_t stage_bytes;          /* bytes per ring stage; 0 = 32768                      */
  int32_t ring_stages;          /* ring depth; 0 = as many as shared memory allows      */
  int32_t l2_prefetch_kb;       /* per-SM budget (KiB) for asking L2 for the next task's
                                   bytes when a task starts; <= 0 = off (the default:
                                   measured slower on the 8B-shaped stack)              */
  int32_t gemv_kpart_max;       /* longest input slice (floats) a GEMV task stages; longer
                                   inputs (not the normalised ones) run in K-parts;
                                   0 = the planner's choice (16384 / tokens per step;
                                   8192 for MLA)                                         */
  int32_t stream_policy;        /* when the producer streams the next op's tiles:
                                   1 = as soon as ring slots free up; 2 = once this SM
                                   has published the current op (its publish then does
                                   not wait behind in-flight copies); 3..6 = its first
                                   1..4 stages at once, the rest as 2; 0 = default (2)   */
  int32_t multi_token_gemv;     /* GEMV form of a plan with max_tokens_per_step > 1:
                                   1 = CUDA-core rows; 2 = tensor-core tiles of 16 rows
                                   (hidden and ffn multiples of 16); 0 = the planner's
                                   choice: tiles at 4 tokens per step when the sizes
                                   allow, else rows                                     */
  int32_t weight_format;        /* TRE_WEIGHTS_*: storage of the GQA projections (FP8)
                                   or of the MoE routed experts (FP4)                   */
  int32_t index_heads;          /* MLA sparse attention (index_topk > 0): H_I index heads,
                                   16, 32 or 64                                         */
  int32_t index_dim;            /* D_I, the index key width: 64 or 128                  */
  int32_t index_topk;           /* K: positions each step attends to (0 = dense MLA)    */
} tre_config;

/* Sparse MLA (index_topk > 0; one token per step).  The pages give the sparse attention of
 * a DeepSeek-V3.2-class model as 64 index heads that choose the top-2048 cached positions
 * of a 160K context for the attention kernel (TileRT code audit, sparse-index paragraph)
 * and print no formula; the indexer is read as DeepSeek-V3.2's lightning indexer with
 * plain projections.  At position pos, with xn = RMSNorm(x) and c_q = RMSNorm(W_dq xn):
 *   k_I = W_ik[0:D_I] xn (this position's index key, appended to the index cache as bf16),
 *   w_I = W_ik[D_I:D_I+H_I] xn,  q_I = W_iq c_q (H_I heads of D_I),
 *   I[t] = sum_j (w_I[j] / sqrt(H_I)) * ReLU(q_I[j] . k_I[t] / sqrt(D_I)),  t in [0, pos];
 * the attention then runs over the K positions of largest I (ties to the lower position);
 * when pos + 1 <= K that is every position.  The score of every position and the chosen
 * set are kept per layer for tre_debug_index. */

/* Weight formats (tre_config.weight_format).  BF16: every matrix bf16.  FP8_BLOCK128 (GQA
 * stacks, one token per step): the seven projection matrices of every layer (Q, K, V, O,
 * gate, up, down) are E4M3 bytes (the OCP 8-bit float with 4 exponent and 3 mantissa
 * bits) with one fp32 scale per 128 x 128 block, element W[n][k] standing for
 * e4m3(W[n][k]) * SCALE[n / 128][k / 128]; the embedding, the norm gains and the LM head
 * stay bf16.  The dequantisation is fused into the weight-streaming GEMV ("RMSNorm + QKV
 * + FP8 dequant", TileRT code audit, fused-op list; fewer bytes per token is the pages'
 * "tokens per byte" lever, Speed is intelligence talk).  Every K must then be a multiple
 * of 16 (16-byte rows).  The E4M3 NaN bytes (S.1111.111) are not decoded as NaN.
 * FP4_EXPERTS (MoE stacks, one token per step): the routed experts' gate, up and down
 * matrices are MXFP4 rows (the OCP Microscaling MXFP4 format): a row of K weights is K/2
 * bytes of E2M1 codes (weight k in the low nibble of byte k/2 when k is even, in the high
 * nibble when odd; E2M1 = sign, 2 exponent bits of bias 1, 1 mantissa bit), then K/32 E8M0
 * scale bytes (weights [32b, 32b + 32) are scaled by 2^(byte b - 127); byte 255 is NaN),
 * zero-padded to a pitch of round_up(K/2 + K/32, 16) bytes.  Attention, router and shared
 * experts stay bf16.  The pages quantise only the MoE experts to FP4 (Speed is intelligence
 * talk, the MiMo co-design passage).  hidden and expert_ffn must be multiples of 32. */
enum { TRE_WEIGHTS_BF16 = 0, TRE_WEIGHTS_FP8_BLOCK128 = 1, TRE_WEIGHTS_FP4_EXPERTS = 2 };

/* Per-layer tensor slots.  layer_w[l * TRE_W_SLOTS + slot] is the device pointer of
 * tensor `slot` of layer l (NULL for slots the layer kind does not use).
 *   GQA : ATTN_NORM[d], WQ[Hq*D][d], WK[Hkv*D][d], WV[Hkv*D][d], WO[d][Hq*D],
 *         FFN_NORM[d], WGATE[F][d], WUP[F][d], WDOWN[d][F]
 *   MOE : slots 0-5 as GQA, then (Fe = expert_ffn, Fs = n_shared * Fe, E = n_experts)
 *         ROUTER[E][d], SHARED_GATE[Fs][d], SHARED_UP[Fs][d], SHARED_DOWN[d][Fs]
 *         (NULL when n_shared == 0), and the routed experts stacked expert-major:
 *         EXPERT_GATE[E][Fe][d], EXPERT_UP[E][Fe][d], EXPERT_DOWN[E][d][Fe]
 *         (the layout of a fused-MoE weight: expert e's matrix starts at e * Fe * d);
 *         FP4_EXPERTS: the same matrices as MXFP4 rows, [E][Fe] rows of pitch(d) bytes
 *         (gate, up) and [E][d] rows of pitch(Fe) bytes (down).
 *   MLA : ATTN_NORM[d], DQ[QL][d], Q_NORM[QL], UQ[H*(NP+R)][QL] (per head: NP nope rows
 *         then R rope rows), DKV[KL+R][d] (KL latent rows then R rope rows),
 *         KV_NORM[KL], UK[H*NP][KL], UV[H*VD][KL], MLA_O[d][H*VD]
 *         (QL = q_lora, KL = kv_lora, R = rope_dim, NP = nope_dim, VD = v_dim)
 *   MLA sparse (index_topk > 0), also: INDEX_Q[H_I*D_I][QL] (the index queries W_iq),
 *         INDEX_K[D_I+H_I][d] (D_I index-key rows, then H_I head-weight rows: W_ik)
 *   GQA with weight_format FP8_BLOCK128: slots 1-4 and 6-8 hold E4M3 bytes of the same
 *         shapes, and their fp32 block scales [ceil(N/128)][ceil(K/128)] sit in
 *         SCALE_Q .. SCALE_DOWN (slots 9-15)
 * KV caches (bf16, written at pos by every step, caller owned):
 *   GQA/MOE : k_cache[l], v_cache[l] = [Hkv][kv_capacity][D]
 *   MLA     : k_cache[l] = latent [kv_capacity][KL + R]: RMSNorm(c_kv) then RoPE(k_pe);
 *             v_cache unused (may be NULL); sparse: v_cache[l] = the index-key cache
             [kv_capacity][D_I] bf16
 */
enum {
  TRE_W_ATTN_NORM = 0, TRE_W_Q = 1, TRE_W_K = 2, TRE_W_V = 3, TRE_W_O = 4,
  TRE_W_FFN_NORM = 5, TRE_W_GATE = 6, TRE_W_UP = 7, TRE_W_DOWN = 8,
  TRE_W_ROUTER = 6, TRE_W_SHARED_GATE = 7, TRE_W_SHARED_UP = 8, TRE_W_SHARED_DOWN = 9,
  TRE_W_EXPERT_GATE = 10, TRE_W_EXPERT_UP = 11, TRE_W_EXPERT_DOWN = 12,
  TRE_W_DQ = 1, TRE_W_Q_NORM = 2, TRE_W_UQ = 3, TRE_W_DKV = 4, TRE_W_KV_NORM = 5,
  TRE_W_UK = 6, TRE_W_UV = 7, TRE_W_MLA_O = 8,
  TRE_W_SCALE_Q = 9, TRE_W_SCALE_K = 10, TRE_W_SCALE_V = 11, TRE_W_SCALE_O = 12,
  TRE_W_SCALE_GATE = 13, TRE_W_SCALE_UP = 14, TRE_W_SCALE_DOWN = 15,
  TRE_W_INDEX_Q = 9, TRE_W_INDEX_K = 10,
  TRE_W_SLOTS = 16
};

typedef struct {
  const void* embed;              /* [V][d] bf16                                        */
  const void* final_norm;         /* [d] bf16                                           */
  const void* lm_head;            /* [V][d] bf16                                        */
  const void* const* layer_w;     /* host array of n_layers * TRE_W_SLOTS device ptrs   */
  void* const* k_cache;           /* host array of n_layers device ptrs                 */
  void* const* v_cache;           /* host array of n_layers device ptrs (MLA: unused)   */
} tre_weights;

/* Summary of a plan, filled by tre_plan_inspect (host only, needs no GPU). */
typedef struct {
  int32_t num_sms;                /* CTAs planned                                       */
  int32_t num_tasks;              /* tasks in the whole step                            */
  int32_t num_counters;
  int32_t kv_splits;
  int32_t ring_stages, stage_bytes, smem_bytes;
  int32_t max_tasks_per_sm;
  int32_t gemv_tiles;             /* 1: multi-token GEMV stages are 16-row tensor-core tiles */
  int32_t index_splits;           /* sparse MLA: index scoring (= selection) tasks per layer */
  int64_t weight_bytes;           /* weight bytes streamed per step                     */
  int64_t kv_bytes_at_capacity;   /* KV bytes streamed per step at pos = capacity - M   */
  int64_t max_sm_bytes, min_sm_bytes;  /* per-CTA streamed bytes (balance)              */
} tre_plan_info;

/* ---- lifecycle ---------------------------------------------------------------- */

/* Validate cfg and the weight pointers, build the static tile task list (the "AOT
 * compile" of [SC] §1 / [SI] dataflow-graph-to-engine section), allocate the engine's
 * device state on `device` and check that one CTA per SM is co-resident.  On success
 * *out receives the engine.  Ownership: the engine copies cfg and the pointer tables;
 * the pointed-to device memory stays the caller's. */
tre_status tre_create(const tre_config* cfg, const tre_weights* w, int device,
                      tre_engine** out);

/* Free everything the engine owns (not the caller's weights / caches).  NULL is a no-op. */
void tre_destroy(tre_engine* e);

/* ---- the hot path ------------------------------------------------------------- */

/* One batch-1 decode step of the whole stack as ONE persistent launch on `stream`
 * ([SC] §1; [TA] blog-vs-code table: the host launches once per token).
 *   token        input token id, 0 <= token < vocab (kernel argument, no copy)
 *   pos          position of this token; the KV caches hold positions [0, pos) on
 *                entry and [0, pos] on return; 0 <= pos < kv_capacity
 *   logits_dev   device fp32[vocab] or NULL (then only token_dev is produced)
 *   token_dev    device int32[1] or NULL: greedy argmax of the logits (lowest index
 *                on ties)
 * Enqueues asynchronously; returns the previous step's device error, if any, without
 * launching.  Requires has_embed_lm_head == 1. */
tre_status tre_decode_step(tre_engine* e, int32_t token, int32_t pos, tre_stream stream,
                           float* logits_dev, int32_t* token_dev);

/* One step over m consecutive tokens of one sequence (speculative-style verification:
 * the pages' multi-token prediction, Speed is intelligence talk, section on tokens per
 * byte): token v sits at position pos + v and attends to the cached positions [0, pos) and
 * to the step's own positions pos .. pos + v (causal).  Every weight byte is read once for
 * all m tokens.  Results equal m successive tre_decode_step calls with the same tokens.
 *   tokens_host  host int32[m], each in [0, vocab) (kernel arguments, no copy)
 *   m            1 <= m <= max_tokens_per_step
 *   pos          the caches hold [0, pos) on entry and [0, pos + m) on return;
 *                pos + m <= kv_capacity
 *   logits_dev   device fp32[m][vocab] or NULL
 *   tokens_dev   device int32[m] or NULL: the greedy argmax of each row of logits
 * Enqueues asynchronously; returns a previous step's device error without launching.
 * Requires has_embed_lm_head == 1. */
tre_status tre_decode_tokens(tre_engine* e, const int32_t* tokens_host, int32_t m, int32_t pos,
                             tre_stream stream, float* logits_dev, int32_t* tokens_dev);

/* The same step driven from host memory: copies nothing in (the token is a kernel
 * argument), runs the step, copies the argmax token (and the logits when logits_host
 * is not NULL) back into host memory and waits for them.  This is the call a greedy
 * generation loop makes once per token. */
tre_status tre_decode_step_host(tre_engine* e, int32_t token, int32_t pos, tre_stream stream,
                                float* logits_host, int32_t* token_host);

/* One decode step, like tre_decode_step, for callers that cannot allocate GPU memory
 * (the pages have no counterpart: it exists for this library's users).  Some callers
 * cannot call cudaMalloc — code running under a framework allocator that must own every
 * byte, real-time loops where allocation is forbidden, plug-ins handed only raw
 * pointers — so no engine is created: each call plans the step on the host (ordinary CPU
 * memory) and keeps everything the kernel needs beyond the caller's tensors (task list,
 * tensor maps of the KV caches, counters, activations, split-KV partials) in one fixed
 * device array built into the
 * library, 4 MiB per GPU, held by every GPU that loads the library until the process exits.
 * The call allocates no GPU memory: no cudaMalloc / cudaMallocAsync / cudaHostAlloc and no
 * cudaFree.
 *   cfg, w       as for tre_create (weights and caches caller owned); no debug flags
 *   token, pos   as for tre_decode_step; the step runs on the CURRENT device
 *   logits_dev   device fp32[vocab], required;  token_dev  device int32[1] or NULL
 *   status_dev   device int32[2] or NULL (4-byte aligned): set to {0, 0}, then on a
 *                device error to {TRE_ERR_DEP_TIMEOUT or TRE_ERR_BOUNDS, task index}.
 *                With NULL a device error is NOT reported to the caller: the kernel
 *                records it in a word of the shared array, which the next call clears.
 * Returns TRE_ERR_UNSUPPORTED, before enqueuing anything, when the model's plan needs
 * more than the 4 MiB array, and when `stream` is capturing a CUDA graph: every call
 * copies its plan from host memory that is gone once the call returns, so the call
 * cannot be captured.  Every call shares the array and leaves the previous call's
 * contents in it (the call clears what must start at zero): calls whose work overlaps on
 * the GPU — two streams, two threads — race and give undefined results; calls in one
 * stream are ordered. */
tre_status tre_decode_step_static(const tre_config* cfg, const tre_weights* w, int32_t token,
                                  int32_t pos, tre_stream stream, float* logits_dev,
                                  int32_t* token_dev, int32_t* status_dev);

/* n_steps greedy decode steps with no host round trip between them ([SC] §1: the host
 * launches once per token and never waits for the model; [TA] blog-vs-code table).  Step
 * i runs at position pos + i; its input token is `token` for i = 0 and, for i > 0, the
 * greedy argmax of step i - 1, which the kernel reads from tokens_dev[i - 1] on the
 * device.  Every step is enqueued on `stream` before the call returns; nothing waits.
 *   tokens_dev   device int32[n_steps] (4-byte aligned): the argmax token of every step
 *   logits_dev   device fp32[vocab] or NULL (16-byte aligned): the last step's logits
 * The caches hold [0, pos) on entry and [0, pos + n_steps) once the steps have run;
 * pos + n_steps <= kv_capacity.  Each step is one launch in the engine's launch mode.
 * Requires has_embed_lm_head == 1.  Enqueues asynchronously; returns a previous step's
 * device error without launching. */
tre_status tre_decode_loop(tre_engine* e, int32_t token, int32_t pos, int32_t n_steps,
                           tre_stream stream, int32_t* tokens_dev, float* logits_dev);

/* Launch modes.  PERSISTENT (the default): a step is ONE cooperative launch of the
 * persistent kernel, in which a task starts as soon as the tasks it reads are done
 * ([SI] section on breaking the kernel boundary).  PER_OP: the same tasks on the same
 * plan, with the kernel boundary put back — one plain launch per op group (the tasks of
 * one layer's op: QKV, attention, O, gate/up, down, ...; ~9 per layer plus the LM head),
 * each launch starting after the previous one has finished.  PER_OP exists to measure
 * what the persistent form removes (the launch cost and the drain / ramp at every op
 * boundary that [SC] §6 names); it computes the same results.
 * Stream capture: PER_OP steps may be captured in a CUDA graph and replayed (their
 * launches wait on nothing but stream order); a PERSISTENT step returns
 * TRE_ERR_UNSUPPORTED on a capturing stream (it waits for a new epoch of its dependency
 * counters, which a replay would not have). */
enum { TRE_LAUNCH_PERSISTENT = 0, TRE_LAUNCH_PER_OP = 1 };

/* Set the launch mode of every later step call on `e`.  *launches_per_step (may be NULL)
 * receives the number of kernel launches one step then takes (1, or the op groups). */
tre_status tre_set_launch_mode(tre_engine* e, int32_t mode, int32_t* launches_per_step);

/* One step of a layers-only stack (has_embed_lm_head == 0): the residual stream after
 * the last layer for one token at `pos`, from the hidden vector entering layer 0.
 *   x_in_dev    device fp32[hidden], read only (16-byte aligned)
 *   x_out_dev   device fp32[hidden], written (16-byte aligned; may not alias x_in_dev)
 *   pos         as for tre_decode_step: the caches hold [0, pos) on entry, [0, pos] after
 * MoE layers route the token on the device (sigmoid scores, top_k by score with ties to
 * the lower expert index, weights normalised over the selection; the pages name the
 * fused op ExpertSelectUpGateSiLU — TileRT code audit, MoE paragraph — and print no
 * formula): only the selected experts' weights are read.  Enqueues asynchronously and
 * returns a previous step's device error without launching, like tre_decode_step. */
tre_status tre_layers_step(tre_engine* e, const float* x_in_dev, float* x_out_dev, int32_t pos,
                           tre_stream stream);

/* ---- status / debug ----------------------------------------------------------- */

/* MoE engines: copy the routing of the last step to host memory — idx_host int32
 * [n_layers][top_k] (selected experts in descending score order) and w_host fp32
 * [n_layers][top_k] (their normalised weights); either may be NULL.  Waits for the
 * engine's last stream.  TRE_ERR_UNSUPPORTED for other kinds. */
tre_status tre_debug_routing(tre_engine* e, int32_t* idx_host, float* w_host);

/* Per-step invariants, a debug check that stands in for a memory checker: wait for the
 * engine's last stream, then check that every dependency counter some task waits on stands
 * at (persistent steps run since create / tre_reset) x (its increments per step), and that
 * the guard words the engine keeps after every buffer it owns still hold their fill
 * pattern.  *bad_counter_out receives the first counter that does not (or -1),
 * *bad_guard_out the index of the first overwritten guard (or -1).  The counters of
 * kernel-per-op launches (their own array) are not checked.  Host copies only. */
tre_status tre_debug_check(tre_engine* e, int32_t* bad_counter_out, int32_t* bad_guard_out);

/* Sparse MLA: wait for the engine's last stream, then copy layer `layer`'s index scores
 * of the last step (score_host: float[pos + 1], I[0 .. pos] as defined above, may be
 * NULL) and its chosen positions (sel_host: int32[index_topk], in no particular order,
 * may be NULL); *n_sel_out receives how many were chosen (min(pos + 1, K)).  pos is the
 * position of that step.  TRE_ERR_INVALID_ARG for a dense engine or a layer or pos out
 * of range. */
tre_status tre_debug_index(tre_engine* e, int32_t layer, int32_t pos, float* score_host,
                           int32_t* sel_host, int32_t* n_sel_out);

/* Wait for the engine's last stream, then report the device status word: 0, or a
 * negative tre_status (TRE_ERR_DEP_TIMEOUT / TRE_ERR_BOUNDS).  *detail_out (may be
 * NULL) receives the global index of the task that recorded it. */
tre_status tre_get_status(tre_engine* e, int32_t* device_status, int32_t* detail_out);

/* Clear the device status word, the dependency counters and the epoch so that the
 * engine can step again after a device error.  Enqueued on `stream`. */
tre_status tre_reset(tre_engine* e, tre_stream stream);

/* Copy the residual stream after every layer of the last step ([n_layers][m][d] fp32,
 * device; m = the last step's tokens, 1 for tre_decode_step) — requires TRE_DEBUG_HIDDEN. */
tre_status tre_debug_hidden(tre_engine* e, float* hidden_dev, tre_stream stream);

/* Copy the per-task trace of the last step to host memory: 8 int64 per task, in global
 * task order: start ns (dependency wait begins), dependency met ns, end ns, SM id, then
 * phase marks — GEMV: input vector staged, last stage consumed; attention: q ready,
 * stages consumed, partial written and published, ns spent waiting for stages to land
 * (0 where a mark does not apply).
 * Requires TRE_DEBUG_TRACE.  *n_tasks receives the task count; trace_host may be NULL to
 * query. */
tre_status tre_debug_trace(tre_engine* e, int64_t* trace_host, int32_t* n_tasks);

/* Bytes a step of m tokens at `pos` streams from HBM (weights + KV read + the m tokens' KV
 * rows written + embedding rows + logits); m = 1 for tre_decode_step / tre_layers_step. */
tre_status tre_step_bytes(const tre_engine* e, int32_t pos, int32_t m, int64_t* bytes);

/* Plan without a GPU: run the planner for cfg on a hypothetical device with `num_sms`
 * SMs and `smem_per_block` bytes of opt-in shared memory, and summarise the plan. */
tre_status tre_plan_inspect(const tre_config* cfg, int32_t num_sms, int32_t smem_per_block,
                            tre_plan_info* info);

/* Plan without a GPU and dump the task descriptors: 8 int32 per task in per-SM queue
 * order — word 0 packs type (bits 0-7), op (8-15) and layer (16-31); then dep, dep_count,
 * out, r0, r1, aux, id — and the per-SM queue offsets (num_sms + 1 int32).  Returns the
 * task count or a negative tre_status; out_tasks is written only when max_tasks is at
 * least the task count, out_sm_begin whenever it is not NULL. */
int32_t tre_plan_tasks(const tre_config* cfg, int32_t num_sms, int32_t smem_per_block,
                       int32_t* out_tasks, int32_t max_tasks, int32_t* out_sm_begin);

/* Plan without a GPU and dump the kernel-per-op form (TRE_LAUNCH_PER_OP): the op groups
 * are the maximal runs of tasks, in global task order, of one layer, task type and op;
 * for group g and SM s, out_ranges[2 (g num_sms + s)] .. [+1] is the half-open range of
 * task indices (into the tre_plan_tasks array) that CTA s runs in launch g.  Returns the
 * number of groups or a negative tre_status; out_ranges ([groups][num_sms][2] int32) is
 * written only when max_groups is at least the group count. */
int32_t tre_plan_op_groups(const tre_config* cfg, int32_t num_sms, int32_t smem_per_block,
                           int32_t* out_ranges, int32_t max_groups);

/* Human-readable text of the last host-side error of this thread. */
const char* tre_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* TRE_H */
