/*
 * smdm.h — C ABI of the sparse masked-diffusion sampling library (B200, sm_100a).
 *
 * Method: Sparse-LaViDa (arXiv 2512.14008).  At sampling step k a masked discrete diffusion
 * model runs only a sparse row set through the transformer: the prompt and earlier decoded
 * tokens live in an incrementally appended KV cache; the tokens decoded at step k-1 are
 * computed once more and appended; the masked positions of the step-k decode set C get logits;
 * n_reg register tokens with position ids L+1..L+n_reg close the sequence.  A step-causal
 * attention mask ties the rows together.  (papernotes.org CVPR-2026 notes, "Key design 1-3"
 * and the Figure-3 example; paperlayer.ai Sec. 3.1-3.3 and Appendix 7.2-7.3.)
 *
 * Conventions shared by every entry point
 *  - All pointers named d_* are DEVICE pointers, h_* are HOST pointers.  The caller owns every
 *    buffer (weights, workspace, inputs, outputs); the library never allocates device memory.
 *    The handle borrows the weights and the workspace: both must outlive it.
 *  - Every call that takes a cudaStream_t is asynchronous on that stream.  Calls on one handle
 *    must be ordered by the caller (use one stream).  The handle's host-side bookkeeping
 *    (cache lengths, step counters) advances when the call is made, so a sequence of calls
 *    can be captured into a CUDA graph and replayed as a whole.
 *  - Argument errors are detected on the host before anything is launched: the call returns a
 *    non-zero smdm_status, leaves the state unchanged and smdm_last_error() explains why.
 *    Device-side problems (a bounded wait that timed out, a failed bounds check) are OR-ed
 *    into a status word that smdm_device_status() reads (it synchronises the stream).
 *  - Positions are 1-based: prompt 1..P, generated tokens P+1..P+Lgen, registers
 *    L+1..L+n_reg with L = P + Lgen.
 *  - Token ids: content ids 0..vocab-1, [MASK] = vocab, [LEN] = vocab+1, register j =
 *    vocab+2+j.  The embedding table has vocab+2+max(n_reg, 0) rows; the LM head covers content ids
 *    only.  A grid (the generated part of a sequence) is int32 [Lgen], -1 = still masked.
 *  - Weight layout: every linear weight is [out_features][in_features], input features
 *    contiguous; dtype per smdm_config.dtype (float32 or bfloat16).
 */
#ifndef SMDM_H_
#define SMDM_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SMDM_OK = 0,
  SMDM_EINVAL = 1,   /* bad argument (null pointer, out-of-range value, bad plan) */
  SMDM_ESHAPE = 2,   /* shape not supported or beyond the configured maxima */
  SMDM_ENOMEM = 3,   /* workspace too small */
  SMDM_ECUDA = 4,    /* a CUDA runtime/driver call failed */
  SMDM_ESTATE = 5,   /* call out of order (e.g. step before prefill) */
  SMDM_ETIMEOUT = 6, /* a device-side bounded wait gave up (see smdm_device_status) */
  SMDM_EDEVICE = 7   /* a device-side bounds check failed */
} smdm_status;

enum { SMDM_F32 = 0, SMDM_BF16 = 1 };
enum { SMDM_POLICY_ALL = 0, SMDM_POLICY_TOPN = 1 };
enum { SMDM_MODE_SPARSE = 0, SMDM_MODE_DENSE = 1 };
/* Row types of a step-labelled sequence.  PROMPT/CLEAN rows are clean tokens; MASK and REG
 * rows belong to a masked block (registers share their block's number). */
enum { SMDM_TYPE_PROMPT = 0, SMDM_TYPE_CLEAN = 1, SMDM_TYPE_MASK = 2, SMDM_TYPE_REG = 3 };
enum { SMDM_PLAN_ORDER = 0, SMDM_PLAN_SEMIAR = 1 };
#define SMDM_MAX_BATCH 8
/* smdm_config.n_reg value of the length-token variant: no registers, and a single [LEN] row
 * (id vocab+1, position L+1, the registers' attention rule) closes every step's rows.  It is
 * the 0-register setting of the register-count ablation (papernotes' Table 7), read with
 * "Key design 2" (one length token standing for the truncated masks). */
#define SMDM_REG_LEN (-1)

/* Model and capacity.  The pages do not describe the base network; the library implements a
 * pre-RMSNorm transformer (multi-head attention with 1-D rotate-half RoPE on the original
 * position ids, SwiGLU MLP, untied LM head).
 * bf16 models need d_model % 128 == 0, d_head in {64, 128}, d_ffn % 64 == 0 and vocab % 4 == 0
 * (logit rows are written with 16-byte-aligned bulk copies; logit buffers passed to the
 * library must be 16-byte aligned).
 * Arithmetic of bf16 models: the weights are given in bf16; smdm_create keeps an fp16 copy of
 * every weight matrix in the workspace, and the GEMMs and the attention multiply fp16 operands
 * (weights, normalised rows, q/K/V, P, attention and SwiGLU outputs) with fp32 accumulation,
 * around an fp32 residual stream, fp32 RMSNorm statistics, fp32 softmax and fp32 logits.  fp16
 * keeps three more mantissa bits than bf16 at the same width and MMA rate; its range ends at
 * 65504, so a model whose weights or activations go beyond it is not served in this mode (a
 * weight beyond it fails smdm_create with SMDM_EINVAL). */
typedef struct {
  int n_layers, d_model, n_heads, d_head, d_ffn;
  int vocab;         /* content vocabulary V */
  int n_reg;         /* register tokens per step (64 in the method; >= 0), or SMDM_REG_LEN */
  int dtype;         /* SMDM_F32 or SMDM_BF16 (weights and activations) */
  float rope_theta;  /* e.g. 10000 */
  float rms_eps;     /* e.g. 1e-6 */
  int max_batch;     /* sequences held at once, <= SMDM_MAX_BATCH */
  int max_len;       /* max P + Lgen of one sequence */
  int max_step_rows; /* max rows of one sequence in one sampling step: n_new + n_query + n_reg
                        (+ 1 for the [LEN] row of the length-token variant) */
  int max_rows;      /* max rows of any single forward: a batched step (sum over sequences),
                        a prefill (P), a dense step (P + Lgen, per sequence) or a
                        training-form forward (n) */
} smdm_config;

/* Device pointers to the weights (borrowed).  Per-layer fields are HOST arrays of n_layers
 * device pointers; the library copies the pointer arrays at create. */
typedef struct {
  const void* emb;        /* [vocab + 2 + max(n_reg, 0)][d] */
  const void* final_norm; /* [d] */
  const void* lm_head;    /* [vocab][d] */
  const void* const* attn_norm; /* [d] */
  const void* const* w_qkv;     /* [3d][d]: rows 0..d-1 -> q, d..2d-1 -> k, 2d..3d-1 -> v;
                                   head h owns rows h*d_head .. h*d_head + d_head - 1 of each */
  const void* const* w_o;       /* [d][d] */
  const void* const* mlp_norm;  /* [d] */
  const void* const* w_gate;    /* [d_ffn][d] */
  const void* const* w_up;      /* [d_ffn][d] */
  const void* const* w_down;    /* [d][d_ffn] */
} smdm_weights;

typedef struct smdm_handle smdm_handle;

/* Bytes of device workspace the handle needs (KV caches for max_batch sequences, activations,
 * RoPE table, reduction scratch and, for bf16 models, the fp16 copies of the weight matrices).
 * Returns 0 for an invalid config. */
size_t smdm_workspace_bytes(const smdm_config* cfg);

/* Create a handle.  d_workspace: caller-allocated device memory of >= smdm_workspace_bytes,
 * 256-byte aligned; it is initialised here (synchronously, on the legacy default stream).
 * Fails with SMDM_ENOMEM if `bytes` is too small, SMDM_ESHAPE for unsupported shapes,
 * SMDM_EINVAL for a null `out`, null weights or a misaligned workspace (checked on the host,
 * before any CUDA call) or for a bf16 weight beyond the fp16 range (found while making the fp16
 * copies), SMDM_ECUDA if a CUDA call fails.  *out is null after any failure.
 * Every other call returns SMDM_EINVAL for a null handle; smdm_destroy(NULL) does nothing. */
smdm_status smdm_create(const smdm_config* cfg, const smdm_weights* w, void* d_workspace,
                        size_t bytes, smdm_handle** out);
void smdm_destroy(smdm_handle* h);
const char* smdm_last_error(const smdm_handle* h);

/* Prefill (Sec. 3.2: the prompt is prefetched into the KV cache).  Starts sequence slot `seq`:
 * runs the P prompt rows (block 0, bidirectional among themselves) through every layer and
 * stores their K/V; no logits.  d_grid: caller-owned int32 [Lgen] that the library fills with
 * -1 and then updates at every step; it must stay valid while the sequence is in use.
 * P may be 0. */
smdm_status smdm_prefill(smdm_handle* h, int seq, const int32_t* d_prompt, int P, int Lgen,
                         int32_t* d_grid, cudaStream_t stream);

/* Prefill with given generation tokens, for bidirectional-context tasks (inpainting,
 * outpainting, infilling: the paper page's sec. 4.5, Figure 6).  As smdm_prefill, and the
 * n_given tokens d_given_tok[i] at 1-based absolute positions d_given_pos[i] (distinct, in
 * P+1..P+Lgen) are clean rows of block 0: computed with the prompt (label 0, bidirectional with
 * it), cached, and written into d_grid.  Later steps must query only the other positions.
 * d_given_pos / d_given_tok: device int32 [n_given], read during the call.  A position outside
 * the generation region or a token id outside the vocabulary sets the device status word
 * (SMDM_EDEVICE at the next synchronising call); duplicate positions are not detected. */
smdm_status smdm_prefill_given(smdm_handle* h, int seq, const int32_t* d_prompt, int P, int Lgen,
                               const int32_t* d_given_pos, const int32_t* d_given_tok,
                               int n_given, int32_t* d_grid, cudaStream_t stream);

/* One sampling step for one sequence (Figure-3 example; Sec. 3.2; Appendix 7.2).
 * Rows, in this order: the tokens decoded at the previous step of this sequence (new cache:
 * their ids from the grid, label k-1), the decode set C (id [MASK], label k), n_reg registers
 * (or the one [LEN] row when n_reg = SMDM_REG_LEN).
 *  - d_query_pos != NULL: C is this explicit list of n_query 1-based positions, each in the
 *    generated region and still masked (checked on the device: a violation sets the status
 *    word, SMDM_EDEVICE at the next synchronising call); duplicates are not detected.
 *  - d_query_pos == NULL: C is every still-masked position in [block_lo, block_hi) in
 *    position order (semi-autoregressive block decoding); n_query must equal their number.
 * After the forward: tok = argmax of the row's logits (ties -> lowest id), conf = max softmax
 * probability.  policy SMDM_POLICY_ALL commits every row of C; SMDM_POLICY_TOPN commits the
 * n_commit most confident rows (ties -> lowest position).  Committed tokens are written into
 * the grid and become the next step's new-cache rows (in row order). */
typedef struct {
  int seq;                  /* sequence slot */
  const int32_t* d_query_pos;
  int n_query;
  int block_lo, block_hi;
  int policy;
  int n_commit;
} smdm_step_desc;

/* Advance n_seq sequences by one step in ONE batched forward (the weights are streamed once
 * for all of them).  h_desc: host array [n_seq].  d_logits: optional fp32
 * [sum of n_query][vocab] (descriptor order), written when non-NULL.  d_tok / d_conf:
 * optional int32 / fp32 [sum of n_query] argmax and confidence per query row. */
smdm_status smdm_step(smdm_handle* h, int n_seq, const smdm_step_desc* h_desc, float* d_logits,
                      int32_t* d_tok, float* d_conf, cudaStream_t stream);

/* Speed switches of the paper notes' Table 6 ablation (cache the prompt, cache decoded
 * responses, truncate the masked responses); SMDM_SW_ALL is the method's own step. */
enum { SMDM_SW_CACHE_PROMPT = 1, SMDM_SW_CACHE_RES = 2, SMDM_SW_TRUNCATE = 4, SMDM_SW_ALL = 7 };

/* One sampling step of one sequence with some of the method's speed switches off.  Off states
 * (the pages name the switches but do not define them; reading): without CACHE_PROMPT the
 * prompt rows (label 0) are computed again every step; without CACHE_RES every decoded token
 * is computed again every step (its label = the step it was decoded at) instead of staying in
 * the cache; without TRUNCATE every other still-masked position joins the step as a [MASK] row
 * of label k (the decode set sees it, so its logits change).  Logits, tokens and the commit are
 * for the decode set only, as in smdm_step.
 * Rows: [prompt?][decoded tokens][decode set][other masks?][registers], each row seeing a key
 * prefix of the sequence's cache, which holds the prompt at slots [0, P) and decoded tokens in
 * decode order after it.  The step needs max_step_rows and max_rows >= P (prompt not cached)
 * + decoded tokens (responses not cached; else the previous step's commits) + n_query + the
 * other masks (not truncated) + registers.
 * The sequence must come from smdm_prefill (no given tokens), take explicit query positions,
 * and keep one value of `switches` for its whole run; smdm_step and smdm_dense_step refuse a
 * sequence that ran switched steps (SMDM_ESTATE). */
smdm_status smdm_step_switched(smdm_handle* h, const smdm_step_desc* h_desc, int switches,
                               float* d_logits, int32_t* d_tok, float* d_conf,
                               cudaStream_t stream);

/* The dense comparator (the standard MDM step the pages argue against, papernotes
 * "Key design 1"): all P+Lgen rows of sequence `seq`, [MASK] ids at undecoded positions, no
 * registers, no cache, full bidirectional attention, logits for every generated position
 * (Lgen x V).  The decode set / commit policy are as in smdm_step; the grid is updated the
 * same way.  d_logits (optional) receives fp32 logits for every generated position,
 * [Lgen][vocab]; d_tok / d_conf (optional) are per decode-set row as in smdm_step. */
smdm_status smdm_dense_step(smdm_handle* h, const smdm_step_desc* h_desc, float* d_logits,
                            int32_t* d_tok, float* d_conf, cudaStream_t stream);

/* A whole sampling plan: the decode set of every step (paperlayer.ai Sec. 3.2).  ORDER plans
 * give the positions in decode order and the count per step: image generation and editing
 * follow a pre-generated 2-D unmasking order with no confidence scores.  SEMIAR plans decode
 * blocks one after another (left to right, or in any order for infilling), querying every
 * masked position of the current block and committing the most confident. */
typedef struct {
  int kind;                   /* SMDM_PLAN_ORDER or SMDM_PLAN_SEMIAR */
  int n_steps;                /* K */
  const int32_t* h_n_per_step;/* ORDER: host [K], tokens decoded per step (sum = Lgen) */
  const int32_t* d_order;     /* ORDER: device [Lgen], 1-based positions in decode order */
  int block;                  /* SEMIAR: block length (Lgen % block == 0) */
  int steps_per_block;        /* SEMIAR */
  int commit;                 /* SEMIAR: tokens committed per step (block == steps * commit) */
  const int32_t* h_block_order; /* SEMIAR, optional: host [Lgen / block], the order in which the
                                   blocks are decoded (a permutation of 0 .. Lgen/block - 1;
                                   NULL = left to right) */
} smdm_plan;

/* Full generation of `batch` sequences (slots 0..batch-1) with the same P, Lgen and step
 * count: prefill (the prompt cached once, Sec. 3.2), then K sparse steps, each one forward
 * over the step's new-cache rows, decode set and registers (the Figure-3 example,
 * papernotes "a complete example"; paperlayer.ai Sec. 3.2 and Appendix 7.2).  d_prompts: int32 [batch][P]; plans: host [batch];
 * d_grids: int32 [batch][Lgen] (output).  mode SMDM_MODE_SPARSE batches the sequences into
 * one forward per step; SMDM_MODE_DENSE runs the dense comparator step per sequence.
 * The whole plan is checked on the host before any work (step sizes, their sum, P + Lgen
 * against max_len and, in sparse mode, every step's rows against max_step_rows and the
 * batched rows against max_rows): a bad plan returns SMDM_EINVAL / SMDM_ESHAPE with no
 * sequence changed. */
smdm_status smdm_generate(smdm_handle* h, int batch, const int32_t* d_prompts, int P, int Lgen,
                          const smdm_plan* plans, int mode, int32_t* d_grids,
                          cudaStream_t stream);

/* Training (parallel) form (Sec. 3.3, Appendix 7.3): one forward over an arbitrary
 * step-labelled sequence of n rows under the step-causal mask — clean rows (PROMPT label 0,
 * CLEAN label = the step they were decoded at) see clean rows with label <= theirs; MASK and
 * REG rows of label s see clean rows with label < s and the MASK/REG rows of label s.
 * Writes fp32 logits [n_rows][vocab] for the rows listed in d_logit_rows.  Does not touch any
 * sequence's generation state.  Any row order is allowed.  Ids must lie in the embedding
 * table, positions in [0, max_len + tail rows + 2), types in 0..3, labels in [0, n] and logit
 * rows in [0, n): an id, position or logit row outside its range sets the device status word
 * (SMDM_EDEVICE at the next smdm_device_status) and is replaced by 0.  For bf16 models the
 * attention skips the 128-key tiles that hold no key visible to a 128-row query tile (same
 * result): rows laid out as the prompt, the clean tokens by step, then each step's masks and
 * registers skip most of them. */
smdm_status smdm_forward_stepcausal(smdm_handle* h, const int32_t* d_ids, const int32_t* d_pos,
                                    const int32_t* d_type, const int32_t* d_label, int n,
                                    const int32_t* d_logit_rows, int n_rows, float* d_logits,
                                    cudaStream_t stream);

/* Test hook: evaluate the device's step-causal predicate for n rows into a bitmap
 * uint32 [n][(n+31)/32] (bit j of row i = row i may attend to row j). */
smdm_status smdm_debug_mask(smdm_handle* h, const int32_t* d_type, const int32_t* d_label, int n,
                            uint32_t* d_bitmap, cudaStream_t stream);

/* Test hook: copy the row arrays of the most recent forward (pack output) into caller
 * buffers of >= *h_n int32 each (any may be NULL).  *h_n receives the row count. */
smdm_status smdm_debug_rows(smdm_handle* h, int32_t* d_ids, int32_t* d_pos, int32_t* d_type,
                            int32_t* d_label, int* h_n, cudaStream_t stream);

/* Cache length (prompt + cached clean tokens) of a sequence slot, host bookkeeping. */
int smdm_context_length(const smdm_handle* h, int seq);

/* Kernel classes for profiling. */
enum {
  SMDM_K_PACK = 0, SMDM_K_NORM = 1, SMDM_K_GEMM_QKV = 2, SMDM_K_ATTN = 3, SMDM_K_GEMM_O = 4,
  SMDM_K_GEMM_GATEUP = 5, SMDM_K_GEMM_DOWN = 6, SMDM_K_GEMM_LMHEAD = 7, SMDM_K_UNMASK = 8,
  SMDM_K_OTHER = 9, SMDM_K_CLASSES = 10
};

typedef struct {
  unsigned long long launches;                      /* kernels launched since profile_begin */
  unsigned long long class_launches[SMDM_K_CLASSES];
  double class_ms[SMDM_K_CLASSES];  /* device time per class from CUDA events recorded on the
                                       launching stream around every launch (timed mode only) */
} smdm_profile;

/* Start counting kernel launches.  timed != 0 also records a CUDA event pair around every
 * launch.  Resets the counters.  Timed profiling may stay on while a CUDA graph is captured:
 * the event records become nodes of the graph, and smdm_profile_end reads the times of the
 * graph's latest replay (replay it before calling smdm_profile_end). */
smdm_status smdm_profile_begin(smdm_handle* h, int timed);
/* Synchronise `stream`, fill *out and stop profiling. */
smdm_status smdm_profile_end(smdm_handle* h, smdm_profile* out, cudaStream_t stream);

/* Allocation-free training-form forward (no counterpart in the paper; it exists for callers
 * that cannot allocate device memory when they need a forward — code under an allocator that
 * is frozen after start-up, a plug-in that is only handed pointers by its host application).
 * Same computation and arguments as smdm_forward_stepcausal, but without a handle: the caller
 * passes the model config, the weights and the inputs/outputs, and every byte of scratch
 * (activations, KV rows, split-K partial sums and tile counters, LM-head statistics, RoPE
 * table and, for bf16 models, the fp16 copies of the weight matrices, remade on every call)
 * lives in one 16 MiB static device array inside the library, which every GPU that
 * loads the library holds until the process exits.  It calls no cudaMalloc/cudaFree.
 *  - Size limit: the scratch this call needs (a one-sequence workspace for max(n, n_rows) rows
 *    with the config's max_len, split-K over 32 CTAs, the weight copies) must fit in 16 MiB;
 *    otherwise the call
 *    returns SMDM_ESHAPE before launching anything.  A 2-layer d=256 model with a few hundred
 *    rows fits.
 *  - The first call on each device looks up the array's device address and sets kernel
 *    attributes; make that first call before any stream capture.
 *  - Every call shares the array and overwrites it (the call clears it first); calls that
 *    overlap on the GPU — on different streams, or from different host threads — race.
 *    Serialise them.
 *  - There is no status word to read back: SMDM_OK means the arguments passed the host checks
 *    and the launches were accepted, NOT that the logits are valid.  A device-side wait that
 *    timed out, or an id outside the embedding table or a position outside
 *    [0, max_len + tail rows + 2) (replaced by 0 on the device), leaves wrong logits and no
 *    error, and so does a bf16 weight beyond the fp16 range.  Check the inputs on the host
 *    before the call: ids and positions in those ranges, types in 0..3, labels in [0, n],
 *    logit rows in [0, n). */
smdm_status smdm_forward_stepcausal_noalloc(const smdm_config* cfg, const smdm_weights* w,
                                            const int32_t* d_ids, const int32_t* d_pos,
                                            const int32_t* d_type, const int32_t* d_label, int n,
                                            const int32_t* d_logit_rows, int n_rows,
                                            float* d_logits, cudaStream_t stream);

/* Synchronise `stream` and return the device status word (0 = no device-side error) and clear
 * it.  Returns SMDM_ETIMEOUT / SMDM_EDEVICE when a bit is set. */
smdm_status smdm_device_status(smdm_handle* h, unsigned* h_bits, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SMDM_H_ */
