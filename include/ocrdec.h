/*
 * ocrdec - greedy-verified speculative decode step of a mixture-of-experts
 * decoder with a FastMTP draft block, as hand-written CUDA for B200 (sm_100a).
 *
 * What the step computes (jina-ocr-v1 pages; news article "jina-ocr-v1: faster
 * document parsing on low-budget GPUs" and the jina-ocr-v1 model page):
 *   - the verifier is a pre-norm MoE decoder (specification table: 12 layers,
 *     d = 1280, 64 routed + 2 shared experts, top-6, vocabulary 129,280, RoPE
 *     theta = 10^6);
 *   - the draft is FastMTP: ONE shared dense block applied recursively for up
 *     to K = 3 steps, each step fed with its own previous hidden state
 *     (sections "Model and training" and "Getting started");
 *   - one verifier pass over the k+1 positions [bonus, d_1..d_k] checks the
 *     proposals greedily, commits the longest agreeing prefix plus one bonus
 *     token and discards the rest, so the committed text equals plain greedy
 *     decoding (model page: bit-identical to autoregressive decoding).
 * This library makes that claim checkable: every kernel reduces each output in
 * an order fixed by the model shape alone (never by the number of rows in a
 * pass), so a run at any k commits exactly the tokens of the same library at
 * k = 0.
 *
 * Conventions
 *   - Every entry point returns an ocrdec_status (0 = OCRDEC_OK).  Nothing
 *     aborts or throws across the ABI.
 *   - "dev_" pointers are device pointers, "host_" pointers are host memory.
 *   - Device work is enqueued on the caller's stream and is asynchronous; a
 *     failure detected on the device (KV capacity exceeded, a stuck wait) is
 *     recorded in a sticky status word read by ocrdec_get_status.  Once it is
 *     set, device work of later calls does nothing until ocrdec_clear_status.
 *   - The caller owns all device memory: the weights (borrowed, must outlive
 *     the context) and one workspace buffer (KV caches, activations, sequence
 *     state).  The library owns only the context object and its CUDA graphs.
 *   - Layouts are row-major; a matrix "[out][in]" maps an input vector of
 *     length in to out outputs.  Weights are bfloat16, 16-byte aligned.
 *   - Sequences live in slots 0..max_batch-1.  Batched calls operate on
 *     slots 0..batch-1.
 *
 * Names against the planned interface of this step (create / workspace /
 * load_weights / prefill / draft / verify_commit / step graph / status /
 * debug taps): the captured whole-step call is ocrdec_step (planned name
 * ocrdec_step_graph); the parity taps are set with ocrdec_set_debug_taps
 * (planned ocrdec_debug_taps) and ocrdec_set_draft_taps; batched calls take
 * the slot range 0..batch-1 instead of a device array of slot ids, because
 * every pass is laid out slot-major on the device; the expert path has one
 * mode (the weight-streaming GEMV of up to 8 rows per pass), so the config
 * has no expert-path field.
 */
#ifndef OCRDEC_H
#define OCRDEC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define OCRDEC_API __attribute__((visibility("default")))
#else
#define OCRDEC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ocrdec_stream; /* = cudaStream_t; NULL = legacy default stream */

typedef enum {
  OCRDEC_OK = 0,
  OCRDEC_EINVAL = 1,    /* bad argument (null pointer, size, alignment, k, slot) */
  OCRDEC_ENOMEM = 2,    /* workspace smaller than ocrdec_workspace_bytes */
  OCRDEC_ECUDA = 3,     /* a CUDA runtime call failed */
  OCRDEC_ECAPACITY = 4, /* a step would write past kv_capacity (device-detected) */
  OCRDEC_ETIMEOUT = 5,  /* a bounded device wait gave up (device-detected) */
  OCRDEC_ESTATE = 6     /* call order violated (no weights, no workspace, slot empty) */
} ocrdec_status;

/* Model and capacity.  The tensor manifest (ocrdec_weight_info) follows from it. */
typedef struct {
  int32_t d_model, n_layers, n_heads, head_dim;
  int32_t n_dense_first; /* leading layers with a dense SwiGLU FFN instead of MoE */
  int32_t n_experts, n_shared, top_k;
  int32_t expert_ffn, shared_ffn, dense_ffn, draft_ffn, vocab;
  int32_t max_k;       /* largest number of draft tokens per step, 0..3 */
  int32_t max_batch;   /* number of sequence slots */
  int32_t kv_capacity; /* positions per slot (context + generated + max_k), <= 8192 */
  float rope_theta, rms_eps;
} ocrdec_config;

typedef struct ocrdec_ctx ocrdec_ctx;

/* Counters of one slot, accumulated on the device. */
typedef struct {
  int32_t kv_len;       /* verified positions in the KV cache (= next verify position) */
  int32_t n_context;    /* prompt rows (visual + text) of the sequence */
  int32_t n_generated;  /* committed generated tokens, including the first one */
  int32_t bonus;        /* latest committed token, not yet in the KV cache */
  int32_t steps;        /* speculative steps run */
  int32_t tau_sum;      /* tokens committed by those steps (tau = tau_sum / steps) */
  int32_t accepted_hist[4]; /* steps that accepted exactly 0..3 draft tokens */
} ocrdec_slot_stats;

/* ---- setup ---------------------------------------------------------------- */

/* The model: the specification table of the news article "jina-ocr-v1:
 * faster document parsing on low-budget GPUs" (and the tahou.com item's
 * "model core parameters" table): 12 layers, d = 1280, 64 routed + 2 shared
 * experts, top-6, vocabulary 129,280, RoPE theta = 10^6; the head layout and
 * FFN widths are free parameters of the config.
 * Validates the config (positive sizes, n_heads*head_dim == d_model, head_dim
 * 64 or 128, n_heads <= 16, d_model <= 1280 (each attention CTA keeps its
 * 3 * head_dim / 8 rows of W_qkv in shared memory) and a multiple of 128, the FFN
 * widths multiples of 64,
 * vocab a multiple of 8, top_k <= min(n_experts, 8), n_experts <= 64,
 * n_shared <= 8, max_k <= 3, kv_capacity <= 8192).
 * *out receives a context that must be released with ocrdec_destroy. */
OCRDEC_API int ocrdec_create(const ocrdec_config* cfg, ocrdec_ctx** out);
OCRDEC_API void ocrdec_destroy(ocrdec_ctx* ctx);

/* The tensors of the decoder and its draft block (news article, "Model and
 * training": a DeepSeek-style MoE decoder and one FastMTP dense block; model
 * page "jina-ocr-v1", architecture paragraph).
 * Number of weight tensors and the shape of tensor `index` in manifest order:
 * embed[V][d]; per layer: attn_norm[d], wqkv[3d][d] (rows q | k | v, head-major),
 * wo[d][d], ffn_norm[d], then for a dense layer w_gate_up[2F][d] (gate rows then
 * up rows), w_down[d][F], and for a MoE layer router[E][d],
 * exp_gate_up[E][2f][d], exp_down[E][d][f], sh_gate_up[S][2fs][d],
 * sh_down[S][d][fs]; final_norm[d], lm_head[V][d]; draft: norm_h[d], norm_e[d],
 * fc[d][2d], attn_norm[d], wqkv[3d][d], wo[d][d], ffn_norm[d],
 * w_gate_up[2Fd][d], w_down[d][Fd], final_norm[d].  The draft uses the
 * verifier's embedding and LM head (tied).  dims gets up to 3 extents. */
OCRDEC_API int ocrdec_weight_count(const ocrdec_config* cfg);
OCRDEC_API int ocrdec_weight_info(const ocrdec_config* cfg, int index, int64_t dims[3], int32_t* ndim);

/* Bytes of the caller-allocated workspace (256-byte aligned device buffer). */
OCRDEC_API size_t ocrdec_workspace_bytes(const ocrdec_config* cfg);

/* Binds the workspace, fills the RoPE table (float64 math, float32 values) and
 * clears every slot.  The buffer must stay valid for the context's lifetime. */
OCRDEC_API int ocrdec_bind_workspace(ocrdec_ctx* ctx, void* dev_workspace, size_t bytes, ocrdec_stream stream);

/* Registers the weights: host array of n device pointers in manifest order,
 * each to a bfloat16 tensor of the manifest's shape, 16-byte aligned.  The
 * tensors are borrowed and must outlive the context. */
OCRDEC_API int ocrdec_load_weights(ocrdec_ctx* ctx, const void* const* host_dev_ptrs, int n);

/* ---- the decode path -------------------------------------------------------- */

/* Prefill (news article, figure caption of the architecture and "Model and
 * training": the decoder reads 256 + 100n visual tokens from the vision
 * encoder, then the text prompt; model page: up to 1,156 visual tokens per
 * page in Gundam mode).
 * Context of one sequence: n_visual visual embeddings (float32 [n_visual][d],
 * standing in for the vision encoder output) then n_prompt tokens, at
 * positions 0..C-1.  Runs the verifier over the context and the draft block
 * over the context pairs, writes the first generated token (argmax at C-1) to
 * dev_first_token[0], and resets the slot's counters.  Requires C >= 1 and
 * C + max_k + 2 <= kv_capacity. */
OCRDEC_API int ocrdec_prefill(ocrdec_ctx* ctx, int slot, const float* dev_visual, int n_visual,
                   const int32_t* dev_prompt, int n_prompt, int32_t* dev_first_token,
                   ocrdec_stream stream);

/* The FastMTP draft (news article, "Model and training": ONE shared dense
 * block applied recursively for K = 3 prediction steps; "Getting started":
 * recursive hidden-state feedback, mtp_recursive=True; model page, FastMTP
 * paragraph).
 * Draft for slots 0..batch-1: recursion 1 runs the shared block on the
 * pairs committed by the previous verify (verifier hidden at p, token at p+1),
 * recursions 2..k feed the block's own output hidden with the previous draft
 * token; each recursion ends with the tied LM head's argmax.  Writes
 * dev_proposals[batch][k].  1 <= k <= max_k. */
OCRDEC_API int ocrdec_draft(ocrdec_ctx* ctx, int batch, int k, int32_t* dev_proposals, ocrdec_stream stream);

/* Greedy verification (news article, "Model and training": the verifier
 * checks the proposals greedily and keeps the longest prefix on which draft
 * and verifier agree, plus the verifier's own next token; model page: the
 * output is bit-identical to plain autoregressive decoding; "L4 speculative
 * decoding" analysis: tau counts the committed tokens including that bonus).
 * Verifier pass over [bonus, proposals[b][0..k-1]] at positions kv_len..kv_len+k
 * for slots 0..batch-1, then greedy acceptance: a = length of the longest prefix
 * with proposals[b][j] == argmax at row j; commits rows' argmax 0..a (a+1 tokens),
 * sets kv_len += a+1 (the rejected rows' KV entries become dead), and stores
 * the hidden states the next draft needs.  dev_committed[batch][k+1] gets the
 * committed tokens (entries past n_committed are -1), dev_n_committed[batch]
 * their count.  k = 0 is plain greedy decoding (dev_proposals may be NULL). */
OCRDEC_API int ocrdec_verify_commit(ocrdec_ctx* ctx, int batch, int k, const int32_t* dev_proposals,
                         int32_t* dev_committed, int32_t* dev_n_committed, ocrdec_stream stream);

/* The step as one replayed CUDA graph (news article, "L4 speculative
 * decoding" table: graph mode against eager mode, 158.3 against 42.7 tokens/s
 * at k = 0 - launch overhead is the lever at batch 1).
 * One whole step (draft when k > 0, the forced-acceptance override when set,
 * verify and commit), launched as a CUDA graph captured on first use for each
 * (batch, k, output pointers).  Same outputs as ocrdec_verify_commit. */
OCRDEC_API int ocrdec_step(ocrdec_ctx* ctx, int batch, int k, int32_t* dev_committed,
                int32_t* dev_n_committed, ocrdec_stream stream);

/* The same passage as ocrdec_step.
 * Same step for callers holding host buffers: copies the results back into
 * host_committed[batch][k+1] / host_n_committed[batch] and synchronises the
 * stream before returning. */
OCRDEC_API int ocrdec_step_host(ocrdec_ctx* ctx, int batch, int k, int32_t* host_committed,
                     int32_t* host_n_committed, ocrdec_stream stream);

/* Benchmark acceptance model (not part of the method; its per-depth hit
 * probabilities 0.83 / 0.69 / 0.58 reproduce the acceptance and tau columns of
 * the news article's "L4 speculative decoding" table, and 0.83 is the
 * mubeitech.com interpretation's first-draft hit rate): after the draft runs,
 * its proposal for target position t at depth j (1-based) is replaced by
 * dev_ref[t] when dev_u[t*max_k + j-1] < p[j-1], and otherwise by the token
 * dev_alt[t*max_k + j-1] of the vocabulary with dev_ref[t] removed.  dev_ref
 * holds tokens by absolute position (n_pos entries); dev_u float32 and dev_alt
 * int32 are [n_pos][max_k].  Pass dev_ref = NULL to switch it off. */
OCRDEC_API int ocrdec_set_forced_acceptance(ocrdec_ctx* ctx, const int32_t* dev_ref, const float* dev_u,
                                 const int32_t* dev_alt, int n_pos, const float* host_p);

/* ---- state, errors, diagnostics --------------------------------------------- */

/* Sticky device status (ocrdec_status); synchronises `stream` to read it. */
OCRDEC_API int ocrdec_get_status(ocrdec_ctx* ctx, int32_t* host_status, ocrdec_stream stream);
/* Clears the sticky status and the device's internal arrival counters (which
 * a launch that gave up part-way may leave inconsistent), on `stream`. */
OCRDEC_API int ocrdec_clear_status(ocrdec_ctx* ctx, ocrdec_stream stream);
/* Synchronises `stream` and copies the slot's counters. */
OCRDEC_API int ocrdec_get_slot_stats(ocrdec_ctx* ctx, int slot, ocrdec_slot_stats* host_stats, ocrdec_stream stream);
/* Device pointer to the committed-token history of a slot, indexed by absolute
 * position (entries for positions >= n_context are generated tokens). */
OCRDEC_API int ocrdec_token_history(ocrdec_ctx* ctx, int slot, const int32_t** dev_tokens);

/* Device counters (synchronises `stream`): host[0] = routed experts touched,
 * summed over the MoE layers of every verifier pass since the last reset (the
 * per-step byte model of the benchmark needs it); host[1] = number of such
 * layer passes.  n = 1 or 2. */
OCRDEC_API int ocrdec_get_counters(ocrdec_ctx* ctx, int32_t* host, int n, ocrdec_stream stream);
OCRDEC_API int ocrdec_reset_counters(ocrdec_ctx* ctx, ocrdec_stream stream);

/* Number of kernel launches in the step graph that ocrdec_step captured for
 * (batch, k, dev_committed, dev_n_committed); OCRDEC_ESTATE if none yet. */
OCRDEC_API int ocrdec_step_kernel_count(ocrdec_ctx* ctx, int batch, int k, int32_t* dev_committed,
                                        int32_t* dev_n_committed, int32_t* count);

/* Parity taps for tests (not used by the timed path).  When set, every
 * verifier pass run by ocrdec_prefill / ocrdec_verify_commit also writes the
 * residual stream after each layer to dev_hidden[layer][row][d] and the logits
 * to dev_logits[row][V] (float32; rows of that pass, at most
 * max_batch*(max_k+1) or the prefill chunk of 8).  NULL switches a tap off. */
OCRDEC_API int ocrdec_set_debug_taps(ocrdec_ctx* ctx, float* dev_hidden, float* dev_logits);

/* Timeline tracer (diagnostics).  While enabled, every CTA of the library's
 * kernels appends one 24-byte record {uint64 t0_ns (%globaltimer, when the CTA
 * passed its dependency wait), uint32 ns to the end of phase 1, phase 2 and
 * phase 3 (= CTA end), uint16 kernel tag, uint16 SM id} to a device buffer of
 * 524,288 records; enabling clears it.  GEMV phases: activation prologue,
 * main loop, epilogue/finish; MoE FFN (recorded by its epilogue warp): dependency wait
 * returned, routing tables first needed, end; attention block: q and the new
 * K/V rows broadcast in the cluster (RMSNorm + QKV projection + RoPE done),
 * the first K/V group's softmax done, end (after the cluster merge, the output
 * projection and, in MoE layers, the router partials).  ocrdec_read_trace
 * copies up to max_records records to host memory and sets *n to the number
 * recorded (synchronises `stream`).  Tags: 1 QKV (draft KV append of
 * prefill pairs), 6 dense gate/up, 7 dense
 * down, 8 verify LM head + acceptance, 9 draft LM head, 10 draft input fc,
 * 11 MoE FFN (routing, experts, combine), 40 attention block (RMSNorm,
 * QKV + RoPE + KV append, attention, output projection; 41 for cluster rank 0), 42 verify setup, 43 draft setup. */
OCRDEC_API int ocrdec_set_trace(ocrdec_ctx* ctx, int enable, ocrdec_stream stream);
OCRDEC_API int ocrdec_read_trace(ocrdec_ctx* ctx, void* host_records, int max_records, int32_t* n,
                                 ocrdec_stream stream);

/* Timing hook (diagnostics, not part of the decode path): enqueues again the
 * MoE FFN sub-layer - routing, shared and routed experts, combine - of
 * verifier layers first_layer .. first_layer + n_layers - 1, with the launches
 * of a (batch, k) verify pass, on the pass rows and router partials the last
 * verifier pass (which must have been a (batch, k) pass) left in the
 * workspace, so that the MoE kernels can be timed alone (CUDA events, graph
 * capture) on their real routing.  The workspace's residual rows are updated in place: call it
 * only between steps; the next step recomputes everything it reads.  The
 * routed experts touched are added to the ocrdec_get_counters counters.
 * first_layer must be a MoE layer (>= n_dense_first). */
OCRDEC_API int ocrdec_replay_moe_ffn(ocrdec_ctx* ctx, int batch, int k, int first_layer, int n_layers,
                                     ocrdec_stream stream);

/* Variant not on the pages: a cheaper draft argmax.  Every draft recursion
 * ends with a full-vocabulary argmax over the LM head (V x d bf16, 331 MB at
 * the full size); this call makes the draft read an e4m3 copy instead (half
 * the bytes), with the activations as e4m3 high and low parts and the logits
 * scaled back per row.  Verification keeps the bf16 head and greedy
 * acceptance, so the committed tokens stay exactly those of plain greedy
 * decoding (model page: verification is greedy); only which proposals get
 * accepted can change.
 * dev_buf: caller-owned device memory of ocrdec_draft_head_fp8_bytes(cfg)
 * bytes, 256-byte aligned, kept alive while the variant is on; the call fills
 * it on `stream` (row n of the head scaled by 448 / max_k |W[n][k]|, rounded
 * to nearest even; then the V float32 inverse scales).  NULL switches back to
 * the bf16 head.  Requires the weights (OCRDEC_ESTATE otherwise) and d_model a
 * multiple of 128; OCRDEC_EINVAL for a short or misaligned buffer. */
OCRDEC_API size_t ocrdec_draft_head_fp8_bytes(const ocrdec_config* cfg);
OCRDEC_API int ocrdec_set_draft_head_fp8(ocrdec_ctx* ctx, void* dev_buf, size_t bytes, ocrdec_stream stream);

/* Parity tap for the draft: when set, recursion j (1-based) of every draft
 * also writes its LM-head logits to dev_logits[j-1][slot][V] (float32,
 * max_k * max_batch * V entries).  NULL switches it off. */
OCRDEC_API int ocrdec_set_draft_taps(ocrdec_ctx* ctx, float* dev_logits);

OCRDEC_API const char* ocrdec_strerror(int status);

/* ---- single-kernel entry points (kernel-level parity tests) ----------------- */

/* RMSNorm followed by a linear map, the first step of every sub-layer of the
 * decoder (pre-norm transformer block; the MoE router, Q/K/V and FFN inputs):
 *   y[r][n] = sum_k W[n][k] * bf16(x[r][k] * rsqrt(mean_k x[r][k]^2 + eps) * g[k])
 * for r < R, accumulated in float32 (bfloat16 operands, float32 products).
 * Layouts (device pointers, owned by the caller): W bfloat16 [N][K] row-major
 * (16-byte aligned), x float32 [R][K], g bfloat16 [K], y float32 [R][N].
 * Sizes: 1 <= R <= 8, N >= 1, K a multiple of 64 with 64 <= K <= 2048.
 * dev_scratch: ocrdec_op_scratch_bytes() bytes, 256-byte aligned; the call
 * clears what it needs.  Asynchronous on `stream`.  Returns OCRDEC_OK,
 * OCRDEC_EINVAL (sizes, alignment, NULL pointers) or OCRDEC_ECUDA (tensor
 * map or launch failure); a device wait that gives up stores
 * OCRDEC_ETIMEOUT in the first int of dev_scratch. */
OCRDEC_API int ocrdec_op_norm_gemv(const void* dev_W, const float* dev_x, const void* dev_g, float eps,
                        int R, int N, int K, float* dev_y, void* dev_scratch, ocrdec_stream stream);

/* Final RMSNorm, LM head and greedy argmax - the verifier's token choice in
 * greedy speculative decoding: tok[r] = argmax_n (W[n] . bf16(RMSNorm(x[r]) * g))
 * with ties to the lower index; if dev_logits is not NULL it also receives
 * the float32 logits [R][N].  Layouts, sizes, scratch, stream and errors as
 * for ocrdec_op_norm_gemv; dev_tok is int32 [R]. */
OCRDEC_API int ocrdec_op_lm_argmax(const void* dev_W, const float* dev_x, const void* dev_g, float eps,
                        int R, int N, int K, int32_t* dev_tok, float* dev_logits,
                        void* dev_scratch, ocrdec_stream stream);

/* Bytes of scratch the two single-kernel entry points need on the current device. */
OCRDEC_API size_t ocrdec_op_scratch_bytes(void);

/* The same final norm + LM head + greedy argmax as ocrdec_op_lm_argmax, for
 * callers that may not allocate device memory and hold no scratch buffer of
 * their own: for example a serving runtime whose memory pool owns all free
 * device memory, or a caller inside an allocator callback, where a cudaMalloc
 * would fail or re-enter the allocator.  It allocates nothing: its scratch is a
 * fixed array of ocrdec_op_static_scratch_bytes() (64 KiB) in the library's own
 * device image, one per device.
 *
 * The method's published description has no counterpart for this call; it is
 * a deployment convenience around the kernel of ocrdec_op_lm_argmax.
 *
 * Arguments, layouts and results are those of ocrdec_op_lm_argmax (all device
 * pointers, owned by the caller; the call only enqueues work on `stream`).
 * The first call on a device, made with that device current, looks up the
 * scratch's address (cudaGetSymbolAddress) and may load the module; make it
 * before capturing any stream.  The scratch status words and counters are
 * cleared on `stream` at every call.  The scratch is shared by every caller on
 * a device: calls that overlap in time (other streams, other threads) race
 * and give undefined results; serialise them.
 *
 * Returns OCRDEC_OK, OCRDEC_EINVAL (the argument checks of
 * ocrdec_op_lm_argmax), OCRDEC_ENOMEM if this device needs more scratch than
 * the fixed array holds (more than 510 SMs: 256 + 128 bytes per SM must fit
 * in 64 KiB), or OCRDEC_ECUDA (no current
 * device, symbol lookup or launch failed). */
OCRDEC_API int ocrdec_op_lm_argmax_static(const void* dev_W, const float* dev_x, const void* dev_g, float eps,
                                          int R, int N, int K, int32_t* dev_tok, float* dev_logits,
                                          ocrdec_stream stream);
OCRDEC_API size_t ocrdec_op_static_scratch_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* OCRDEC_H */
