/*
 * dllm.h - C ABI of the token-skipping denoising step for masked diffusion LMs.
 *
 * One denoising iteration of a masked diffusion LM in which only a set of
 * active token rows is recomputed, while skipped or locked rows keep their
 * K/V (and hidden state) in a cache and active queries still attend over the
 * whole sequence.  The calls follow the iteration as the source pages state
 * it: choose the rows to compute, compute them, unmask:
 *   - "ES-dLLM: Efficient Inference for Diffusion Large Language Models by
 *     Early-Skipping", sec. 2.1 (Eq. 1 importance; top-k early skip; partial
 *     in-place cache update) and sec. 2.2 (periodic refresh);
 *   - "SureLock: Stopping Computation for Converged Tokens", sec. 2.1 (lock
 *     when KL(p_t || p_t-1) < eps; locked rows skip Q projection and FFN and
 *     keep frozen K/V; active rows still attend to them);
 *   - the dLLM-Cache explainer, sec. 3 (long-interval prompt cache; response
 *     rows recomputed when their features move, at most a ratio rho);
 *   - "Plan for Speed: Dilated Scheduling for Masked Diffusion Language
 *     Models", sec. 2 (R = ceil(log2 B) rounds of non-adjacent positions).
 *
 * Conventions (every call):
 *   - Returns an int status: DLLM_OK or one of DLLM_ERR_*.  No call exits,
 *     aborts or throws.  dllm_last_error() gives a message for the last
 *     failure on this thread.
 *   - Device pointers are plain CUDA device addresses on the current device;
 *     the caller allocates and owns all of them (weights, tokens, state,
 *     workspace) and keeps them alive for the life of a handle.  A handle
 *     owns host metadata only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on it unless stated otherwise; a
 *     device-side failure (a bounded wait that ran out) is reported by
 *     dllm_device_status() at the caller's next synchronisation.
 *   - Layouts: weights bf16 row-major [out, in]; tokens int32 [B, N];
 *     positions and indices int32; scores fp32; hidden states fp32.
 */
#ifndef DLLM_H_
#define DLLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
enum {
  DLLM_OK = 0,
  DLLM_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum value */
  DLLM_ERR_SHAPE = 2,       /* sizes that do not fit the layout */
  DLLM_ERR_UNSUPPORTED = 3, /* a valid request the library does not implement */
  DLLM_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  DLLM_ERR_TIMEOUT = 5,     /* a bounded device wait ran out */
  DLLM_ERR_DEVICE = 6,      /* the device status word was set */
  DLLM_ERR_STATE = 7        /* call out of order (e.g. generation finished) */
};

enum { DLLM_POLICY_VANILLA = 0, DLLM_POLICY_ES = 1, DLLM_POLICY_SURELOCK = 2, DLLM_POLICY_DLLM_CACHE = 3 };
/* TOPCONF: the tokens_per_step masked positions of the block with the highest confidence.
   DUS: the dilated round of the step (Plan for Speed summary sec. 2).
   CB_DUS: confidence-bounded with the dilation rule as a post-filter (the same summary, sec. 3):
   positions with confidence >= cb_tau in confidence order (the first one always), none next to
   another taken in the step, at most tokens_per_step; a block ends when nothing in it is masked
   (the step count is data-dependent: the host reads B counts after each step). */
enum { DLLM_UNMASK_TOPCONF = 0, DLLM_UNMASK_DUS = 1, DLLM_UNMASK_CB_DUS = 2 };
enum { DLLM_SCOPE_BLOCK = 0, DLLM_SCOPE_ALL = 1 };
/* How a layer over a small row set runs: AUTO lets the library choose, SPLIT launches one
   kernel per step of the layer, FUSED runs the whole layer as one persistent kernel whenever
   at most 64 rows are recomputed (larger row sets always take SPLIT). */
enum { DLLM_LAYER_AUTO = 0, DLLM_LAYER_SPLIT = 1, DLLM_LAYER_FUSED = 2 };
enum { DLLM_STEP_FULL = 0, DLLM_STEP_SKIP = 1, DLLM_STEP_LOCKED = 2, DLLM_STEP_PARTIAL = 3 };

/* Model shape, generation schedule and row-selection policy. */
typedef struct dllm_config {
  /* model */
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab, mask_id;
  float rope_theta, rms_eps;
  /* generation: B sequences of N = prompt_len + gen_len positions, blocks of block_len */
  int32_t batch, prompt_len, gen_len, block_len;
  /* policy */
  int32_t policy;          /* DLLM_POLICY_* */
  int32_t cand_scope;      /* DLLM_SCOPE_*: candidate rows = current block or all rows */
  /* ES-dLLM: select at layer skip_layer, keep k = ceil(keep_ratio * n_cand), Eq. 1 weight alpha;
     refresh at the first step of each block and every refresh_period steps (0 = never else) */
  int32_t skip_layer;
  float keep_ratio, alpha;
  int32_t refresh_period;
  /* SureLock: lock when KL < kl_eps and confidence > conf_tau (unmasked rows only) */
  float kl_eps, conf_tau;
  /* dLLM-Cache: full refresh every prompt_interval steps; recompute response rows whose value
     cosine < sim_tau, at most ceil(rho_cap * n_resp); forced_rho != 0 keeps exactly that many */
  float sim_tau, rho_cap;
  int32_t prompt_interval, forced_rho;
  /* unmasking */
  int32_t unmask;          /* DLLM_UNMASK_* */
  int32_t tokens_per_step; /* TOPCONF: n committed per step and sequence */
  int32_t layer_kernel;    /* DLLM_LAYER_* */
  /* SureLock lock scope: 0 = unmasked positions only (prompt and decoded tokens); 1 = every
     position, masked ones included (a locked masked position is still unmasked later from the
     confidence and argmax stored when it locked) */
  int32_t lock_masked;
  float cb_tau;            /* CB_DUS confidence bound */
  /* ES-dLLM: 0 = one top-k choice at skip_layer for the rest of the step; 1 = the choice is
     made again at the start of every layer from skip_layer on (ES-dLLM sec. 2.1, item 2),
     Eq. 1 on that layer's input; needs skip_layer < n_layers */
  int32_t es_per_layer;
} dllm_config;

/* Device pointers to the weights (bf16 unless noted), all row-major [out, in]. */
typedef struct dllm_weights {
  const void* embed;   /* [V, d] */
  const void* lm_head; /* [V, d] */
  const void* w_qkv;   /* [L, Hq*hd + 2*Hkv*hd, d]: q rows, then k rows, then v rows */
  const void* w_o;     /* [L, d, Hq*hd] */
  const void* w_gu;    /* [L, 2F, d]: gate rows, then up rows */
  const void* w_down;  /* [L, d, F] */
  const float* g_attn; /* fp32 [L, d] */
  const float* g_ffn;  /* fp32 [L, d] */
  const float* g_final;/* fp32 [d] */
} dllm_weights;

typedef struct dllm_step_info {
  int32_t kind;          /* DLLM_STEP_* */
  int32_t step;          /* index of the step just run */
  int32_t block;         /* block it belonged to */
  int32_t step_in_block;
  int32_t rows_first;    /* rows recomputed below the skip layer (host bound) */
  int32_t rows_last;     /* rows recomputed at the last layer (device count) */
  int32_t lm_rows;       /* rows through the vocabulary projection */
  int32_t n_locked;      /* SureLock: locked positions over the batch */
  int32_t done;          /* 1 when every block is finished */
} dllm_step_info;

typedef struct dllm_handle dllm_handle;

const char* dllm_status_string(int status);
/* Message of the last failing call on this thread ("" if none). */
const char* dllm_last_error(void);
/* Device status word values: the first failure a kernel records is kept until read. */
enum {
  DLLM_DEV_OK = 0,
  DLLM_DEV_TIMEOUT = 1,    /* a bounded wait ran out (the kernel stopped its work and returned) */
  DLLM_DEV_BAD_INDEX = 2   /* an index outside its table (a token id, an argmax of no finite logit) */
};
/* Reads (and with reset != 0 clears) the device status word; synchronises the device. */
int dllm_device_status(int32_t* status, int32_t reset);

/* Bytes of caller-allocated device memory a configuration needs: `state`
 * persists across steps (K/V cache, hidden snapshots, confidences, locks,
 * stored distributions, per-layer output cache), `workspace` is scratch for
 * one step.  Both must be 256-byte aligned.  Validates the configuration.
 * What persists follows what each policy keeps between iterations: ES-dLLM
 * sec. 2.1 (the skip layer's hidden state and confidence of the previous
 * iteration, the partially updated K/V cache), SureLock sec. 2.1 (the lock
 * flags and the previous step's distribution of every lock-eligible row, the
 * frozen K/V), the dLLM-Cache explainer sec. 3 (per-layer cached outputs).
 * state_bytes / workspace_bytes must be non-null; returns
 * DLLM_ERR_INVALID_ARG / _SHAPE / _UNSUPPORTED for a configuration the
 * library cannot serve.  Host only: launches nothing. */
int dllm_state_bytes(const dllm_config* cfg, size_t* state_bytes, size_t* workspace_bytes);

/* Creates a handle over caller memory and zero-initialises the caches.
 * tokens: device int32 [B, N], the prompt followed by mask ids; updated in
 * place by every step.  Enqueued on `stream`.
 * The start of a generation as the pages describe it: the prompt is followed
 * by masked positions that the iterations unmask (ES-dLLM sec. 1; Plan for
 * Speed sec. 2, blocks generated in order).  state / workspace must hold the
 * sizes dllm_state_bytes gives, 256-byte aligned, every weight pointer 16-byte
 * aligned and tokens 4-byte aligned, else DLLM_ERR_INVALID_ARG (checked before
 * anything is enqueued); every pointer must stay valid until dllm_destroy.  Synchronises `stream`
 * once (the host copy of the DUS round masks must outlive its upload). */
int dllm_step_init(dllm_handle** out, const dllm_config* cfg, const dllm_weights* w, void* state, void* workspace,
                   int32_t* tokens, void* stream);

/* Starts one denoising step: decides from the schedule whether it is a full
 * refresh (ES-dLLM sec. 2.2; dLLM-Cache prompt interval), chooses the rows
 * that enter layer 0 (all rows; the current block; SureLock's unlocked rows)
 * and gathers their embeddings.  *kind_out (nullable) gets DLLM_STEP_*.
 * DLLM_ERR_STATE once every block is finished.  Asynchronous on `stream`. */
int dllm_begin_step(dllm_handle* h, int32_t* kind_out, void* stream);

/* Runs one transformer layer for the current row set, in place: new K/V rows
 * are written into the cache before attention, attention reads all N cached
 * rows of the sequence.  Under dLLM-Cache the layer first scores the response
 * rows by value-vector cosine and recomputes only the selected ones.
 * Follows ES-dLLM sec. 2.1 item 3 (the computed rows' K/V are updated in
 * place in the cache, the skipped rows' entries are kept), SureLock sec. 2.1
 * item 3 (active queries attend over all positions, locked ones through their
 * frozen K/V) and the dLLM-Cache explainer sec. 3 (per-layer partial update of
 * the response rows).  layer in [0, n_layers) else DLLM_ERR_INVALID_ARG;
 * DLLM_ERR_STATE before dllm_begin_step or out of the per-layer selection
 * order.  Asynchronous on `stream`; reads and writes only caller memory. */
int dllm_layer_forward(dllm_handle* h, int32_t layer, void* stream);

/* Runs layers l0 .. l1-1 for the current row set, with the same result as
 * dllm_layer_forward on each in turn.  When at most 64 rows are recomputed (and
 * layer_kernel allows it) the whole run is one persistent kernel whose weight
 * stream continues across the layer boundaries.  Same algorithm and page
 * passages as dllm_layer_forward; l0 == l1 is a no-op; DLLM_ERR_INVALID_ARG when
 * the range is outside [0, n_layers]. */
int dllm_layers_forward(dllm_handle* h, int32_t l0, int32_t l1, void* stream);

/* ES-dLLM early skip at the skip layer: scores the candidates by Eq. 1 (or
 * uses `scores_or_null`, fp32 [B, n_cand] device, for teacher forcing), keeps
 * the top k per sequence (ties to the lower position) and makes them the row
 * set of the remaining layers.  active_idx (device int32 [B, k], ascending
 * positions) and active_count (device int32 [B]) are optional outputs.
 * On a refresh step it only snapshots the candidates' hidden states.
 *
 * With es_per_layer the call is made before every layer from skip_layer on
 * (the first call applies to skip_layer, each next one to the following
 * layer) and the layer then runs alone (dllm_layer_forward, or
 * dllm_layers_forward over that one layer).  Eq. 1 compares each candidate's
 * input of that layer with its input of the previous iteration; a row the
 * previous layer skipped enters with its cached output of that layer and a
 * zero variation term, and the chosen rows become the layer's row set.
 * Calls out of this order return DLLM_ERR_STATE, as does dllm_unmask before
 * the last layer's call. */
int dllm_select_active(dllm_handle* h, const float* scores_or_null, int32_t* active_idx, int32_t* active_count,
                       void* stream);

/* ES-dLLM: the choice and layers skip_layer .. n_layers-1 of the step, with the same
 * result as dllm_select_active -> dllm_layers_forward(skip_layer, n_layers), or with
 * es_per_layer as dllm_select_active -> dllm_layer_forward for each layer in turn.
 * On a skip step whose kept rows fit the fused layer kernel (B * k <= 64,
 * n_cand <= 512, layer_kernel not SPLIT) the whole run is one persistent launch
 * that scores (Eq. 1; per layer with the carry of skipped rows) and chooses the
 * rows itself, at the skip layer or at the start of every layer.
 * `scores_or_null`: fp32 device [S, B, n_cand], S = 1 (or n_layers - skip_layer
 * with es_per_layer), the scores each choice uses (teacher forcing), or NULL for
 * Eq. 1.  Call after dllm_layers_forward(0, skip_layer) and before dllm_unmask;
 * DLLM_ERR_STATE outside the ES policy or when the step's choice was already made. */
int dllm_select_layers_forward(dllm_handle* h, const float* scores_or_null, void* stream);

/* Ends the step: final RMSNorm and vocabulary projection of the recomputed
 * masked rows of the current block (DUS: of this round), confidence and
 * argmax (mask id excluded), SureLock's KL and locking, and unmasking
 * (top-n confidence, or the DUS round).  pos_out / tok_out (device int32
 * [B, max(n, round size)]) and n_out (device int32 [B]) are optional.
 * Advances the schedule.
 * Follows ES-dLLM sec. 1 (a few tokens of highest confidence are unmasked per
 * iteration; the confidences are stored for the next iteration's Eq. 1),
 * SureLock sec. 2.1 items 1-2 (KL(p_t || p_t-1) per position from the step's
 * logits and the stored ones; lock when KL < eps and the confidence > tau) and
 * Plan for Speed sec. 2 (the round's dilated group is unmasked together).
 * DLLM_ERR_STATE before dllm_begin_step or with per-layer choices left; with
 * the CB_DUS unmasking the call reads B ints back and synchronises `stream`,
 * otherwise it is asynchronous. */
int dllm_unmask(dllm_handle* h, int32_t* pos_out, int32_t* tok_out, int32_t* n_out, void* stream);

/* One whole denoising step (begin, layers, selection, unmask).  With `info`
 * non-null the call synchronises the stream and fills it.
 * The iteration of the pages: choose the rows to compute (ES-dLLM sec. 2.1
 * Eq. 1 and early skip; SureLock sec. 2.1 locks; dLLM-Cache sec. 3 similarity
 * gate), compute them over the cached K/V, unmask; refresh steps per ES-dLLM
 * sec. 2.2 and the dLLM-Cache prompt interval.  DLLM_ERR_STATE once
 * dllm_done() is 1; a failing call leaves the step unfinished (the handle
 * stays valid; dllm_reset starts over). */
int dllm_step(dllm_handle* h, dllm_step_info* info_or_null, void* stream);

/* Host-side schedule: 1 when every block is finished. */
int dllm_done(const dllm_handle* h);

/* SureLock measurement mode: with a device uint8 [B, N] pattern, a row locks as soon
 * as it is unmasked and has a previous distribution and pattern[b, pos] != 0,
 * instead of by the KL / confidence rule (random weights never reach the
 * confidence threshold).  NULL restores the rule.  The pattern must outlive
 * the handle's steps. */
int dllm_set_lock_pattern(dllm_handle* h, const uint8_t* pattern);

/* Starts a new generation on the same handle: zeroes the caches and rewinds
 * the schedule, asynchronously on `stream` (the caller rewrites `tokens`).
 * It also clears the GEMM tile and attention split counters of the workspace:
 * every launch leaves them at zero except one that gave up a wait, so after
 * dllm_device_status reports DLLM_DEV_TIMEOUT call dllm_reset (or destroy the
 * handle) before further steps. */
int dllm_reset(dllm_handle* h, void* stream);

/* Per-kernel timing of the fused GEMMs and the attention, for roofline
 * reporting: with enable = n > 0 every n-th launch of each kind is bracketed by
 * CUDA events on its stream, and its algorithmic bytes and flops are recorded
 * (sampling keeps the event overhead off the timed stream); 0 turns it off.
 * dllm_profile_read synchronises, sums the records since the last read and
 * clears them. */
typedef struct dllm_profile {
  int64_t gemm_launches;   /* kernel-per-step path: each GEMM launch */
  double gemm_ms, gemm_bytes, gemm_flops, gemm_roofline_ms;
  int64_t attn_launches;   /* kernel-per-step path: each attention launch (with its merge) */
  double attn_ms, attn_bytes, attn_flops;
  int64_t fused_launches;  /* fused runs of layers (one persistent kernel each) */
  int64_t fused_layers;    /* layers those launches ran */
  double fused_ms, fused_bytes, fused_flops;   /* bytes: weights + K/V read + row traffic */
} dllm_profile;
int dllm_profile_enable(dllm_handle* h, int32_t enable, double hbm_gbs, double tensor_tflops);
int dllm_profile_read(dllm_handle* h, dllm_profile* out);

/* Position of the generation schedule (host state of a handle).  Together with the
 * caller-owned `state` buffer and the token buffer it is the whole generation state:
 * copying state and tokens to a fresh handle of the same configuration and setting
 * its progress resumes the generation exactly (checkpoint / resume).  The pages have
 * no counterpart; this is a facility of this library. */
typedef struct dllm_progress {
  int32_t step;           /* steps run so far */
  int32_t block;          /* current block */
  int32_t step_in_block;  /* steps run in it */
} dllm_progress;
/* Reads the schedule position; valid between steps. */
int dllm_get_progress(const dllm_handle* h, dllm_progress* out);
/* Sets it (between steps): DLLM_ERR_INVALID_ARG for a position outside the schedule of
 * the configuration, DLLM_ERR_STATE in the middle of a step. */
int dllm_set_progress(dllm_handle* h, const dllm_progress* p);

/* dLLM-Cache teacher forcing: with a device fp32 [L, B, n_resp] array the partial
 * steps choose each layer's rows from these similarities instead of the cosine of
 * the value vectors (n_resp = gen_len, or prompt_len + gen_len over all rows); the
 * cosine is still computed and left in DLLM_BUF_SCORES.  The threshold, the cap and
 * the tie rule are those of the dLLM-Cache explainer sec. 3 as configured.  NULL
 * restores the cosine; the array must outlive the handle's steps.
 * DLLM_ERR_STATE outside the dLLM-Cache policy. */
int dllm_set_forced_similarities(dllm_handle* h, const float* sims);

/* Poll limit of the grid-wide waits of the fused layer kernel (0: the default, about
 * 0.4 s).  Failure-detection tests lower it so that a wait they make unsatisfiable
 * (DLLM_BUF_FUSED_SYNC) runs out quickly: the kernel then records DLLM_DEV_TIMEOUT,
 * stops its work, waits for its own copies in flight, frees its tensor memory and
 * returns, and the next launch starts clean.  The pages have no counterpart. */
int dllm_set_wait_limit(dllm_handle* h, uint32_t polls);

/* Number of CUDA kernels this library has launched in the process so far. */
int64_t dllm_kernel_launches(void);

/* Internal device buffers, for inspection and teacher forcing in tests. */
enum {
  DLLM_BUF_KCACHE = 0,   /* bf16 [L, B, Hkv, N, hd] */
  DLLM_BUF_VCACHE = 1,
  DLLM_BUF_HIDDEN = 2,   /* fp32 [B*N, d] residual stream of the recomputed rows */
  DLLM_BUF_HPREV = 3,    /* fp32 [B*N, d] ES-dLLM snapshot at the skip layer */
  DLLM_BUF_CONF = 4,     /* fp32 [B*N] latest confidence */
  DLLM_BUF_ARGMAX = 5,   /* int32 [B*N] latest argmax */
  DLLM_BUF_ROWS = 6,     /* int32 [B*N] current row set (flat b*N + pos) */
  DLLM_BUF_NROWS = 7,    /* int32 [1] its size */
  DLLM_BUF_SCORES = 8,   /* fp32 [B*N] last selection scores */
  DLLM_BUF_LOCK = 9,     /* uint8 [B*N] SureLock lock flags */
  DLLM_BUF_MASKED_PREV = 10, /* uint8 [B*N] */
  DLLM_BUF_LMROWS = 11,  /* int32 [B*N] rows of the last vocabulary projection */
  DLLM_BUF_NLMROWS = 12, /* int32 [1] */
  DLLM_BUF_KL = 13,      /* fp32 [B*N] SureLock divergences of the LM rows (NaN: no previous p) */
  DLLM_BUF_HCACHE = 14,  /* fp32 [L, B*N, d] dLLM-Cache per-layer outputs */
  DLLM_BUF_LSE = 15,     /* fp32 [B*N] log-sum-exp of the last logits per position */
  DLLM_BUF_SELROWS = 16, /* int32 [B*N] rows picked by the last selection (ES top-k; dLLM-Cache per layer) */
  DLLM_BUF_NSEL = 17,    /* int32 [1] their number */
  /* workspace views of the last layer's intermediates (row j = j-th recomputed row; valid
     until the next call that runs a layer) */
  DLLM_BUF_LAYER_Z = 18,    /* bf16 [rows, d] gate/up operand: RMSNorm before the FFN (the fused
                               layer keeps g * h there and scales the sums by 1/rms instead) */
  DLLM_BUF_LAYER_Q = 19,    /* bf16 [rows, Hq*hd] rotated queries */
  DLLM_BUF_LAYER_ATTN = 20, /* bf16 [rows, Hq*hd] attention output */
  DLLM_BUF_LAYER_ACT = 21,  /* bf16 [rows, F] SwiGLU activation */
  DLLM_BUF_ES_IN = 22,      /* fp32 [L - skip_layer - 1, B*N, d] per-layer ES: each candidate's input
                               of layer skip_layer + 1 + i in the last iteration that scored it */
  DLLM_BUF_ZSTORE = 23,     /* bf16 [2, B*N, V] SureLock: stored logits, buffer (step & 1) written
                               by step `step` */
  DLLM_BUF_LSE_STORE = 24,  /* fp32 [2, B*N] their log-sum-exp */
  DLLM_BUF_STAMP = 25,      /* int32 [B*N] step + 1 of the last stored distribution per position */
  DLLM_BUF_VNEW = 26,       /* fp32 [B*n_resp, Hkv*hd] dLLM-Cache: value vectors of the last layer's probe */
  DLLM_BUF_FUSED_SYNC = 27  /* int32 [16] phase counters of the fused layer kernel, zero between launches;
                               element 0 gates every CTA's first QKV step of a launch */
};
int dllm_get_buffer(dllm_handle* h, int32_t which, void** ptr, size_t* bytes);

/* Frees the handle's host metadata (the pages have no counterpart: ownership
 * rule of this library).  Caller memory (weights, tokens, state, workspace)
 * is not touched and stays owned by the caller; NULL is a no-op.  Kernels
 * already enqueued keep running: synchronise the stream first if the caller
 * frees its buffers next. */
void dllm_destroy(dllm_handle* h);

/* ------------------------------------------------------------------ ops
 * Single kernels of the path on caller buffers (parity tests, the
 * single-layer microbenchmark).  Device pointers, stream as above.
 * `workspace` (where taken) is caller scratch: zero it before its first use;
 * its first 256 KB hold GEMM tile counters that every call leaves at zero, so
 * calls on one stream may share it; calls that overlap on the GPU may not.
 * After dllm_device_status reports DLLM_DEV_TIMEOUT, zero it again.
 * Alignment (the kernels move 16-byte vectors): workspaces 256-byte aligned;
 * embedding tables, fp32 rows (h, h_prev, gains), caches, q and attention
 * outputs and RoPE tables 16-byte aligned; bf16 outputs written 4 values at a
 * time (RMSNorm z, q and cache rows of the QKV op) 8-byte aligned.  A pointer
 * that misses its alignment is refused with DLLM_ERR_INVALID_ARG before
 * anything is launched.  Device-resident index arrays (rows, rows_map, seq_off)
 * are read by the kernels as given: each index must lie inside the buffer it
 * addresses (device counts are clamped to rows_cap, token ids are checked).  */

/* RoPE tables cos/sin fp32 [N, hd/2] with angle pos * theta^(-2i/hd). */
int dllm_op_rope_table(float* cos_t, float* sin_t, int32_t N, int32_t head_dim, double theta, void* stream);

/* h[rows[j]] = float(E[tokens[rows[j]]]) for j < *count (count nullable: rows_cap), E bf16 [vocab, d].
 * A token id outside [0, vocab) is never read: its row is zeroed and the device status word
 * records DLLM_DEV_BAD_INDEX (dllm_device_status). */
int dllm_op_embed_rows(const void* embed, int32_t vocab, const int32_t* tokens, const int32_t* rows,
                       const int32_t* count, int32_t rows_cap, int32_t d, float* h, void* stream);

/* z[j] = bf16(x / sqrt(mean(x^2) + eps) * g), x = h[rows[j]] (rows nullable: j). */
int dllm_op_rmsnorm_rows(const float* h, const int32_t* rows, const int32_t* count, int32_t rows_cap, int32_t d,
                         const float* g, float eps, void* z, void* stream);

/* C = X W^T with X bf16 [rows_cap, K] (first *count rows valid), W bf16 [n_out, K].
 * kind 0: out fp32 [rows, n_out]; 1: out bf16; 3: residual h[rows_map[j]] += C (fp32, ld n_out).
 * splits / bn: 0 = automatic (tests force them to cover the split-K and tile paths). */
int dllm_op_gemm(int32_t kind, const void* W, int32_t n_out, const void* X, int32_t rows_cap, const int32_t* count,
                 int32_t K, void* out, const int32_t* rows_map, int32_t splits, int32_t bn, void* workspace,
                 size_t workspace_bytes, void* stream);

/* The same GEMM as dllm_op_gemm for callers that cannot allocate device memory:
 * a host framework that owns all device memory and hands a plugin only its
 * input and output buffers, or a hot path that must not call cudaMalloc (it
 * synchronises the device and can fail under memory pressure).  The paper has
 * no counterpart; this is a deployment convenience of this library.
 * Its scratch (tile counters and split-tile partial sums, ~4.9 MB) is a fixed
 * array in the library's device image, held on every device that loads the
 * library until the process exits.  The call allocates nothing: no cudaMalloc,
 * no cudaFree, no allocating library routine.  Limits: rows_cap <= 32 and
 * n_out <= 524288 (4096 tiles of 128); larger problems return DLLM_ERR_SHAPE
 * and belong to dllm_op_gemm.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current, so
 * make that first call before any stream capture.  All calls on a device share
 * its one array, which keeps what the last call left; each call clears the tile
 * counters it needs on `stream`.  Calls that can overlap on the GPU (issued on
 * different streams of one device without ordering between them) race on the
 * array and must be serialised by the caller. */
int dllm_op_gemm_noalloc(int32_t kind, const void* W, int32_t n_out, const void* X, int32_t rows_cap,
                         const int32_t* count, int32_t K, void* out, const int32_t* rows_map, void* stream);

/* QKV projection with RoPE on q and k: q -> q_out bf16 [rows, Hq*hd], k and v -> the cache
 * rows (b, :, pos) of rows_map[j] = b * N + pos.  W = one layer of w_qkv.  The products are
 * kept in fp32 in the workspace (rows_cap * (Hq + 2 Hkv) * hd * 4 bytes after the GEMM
 * scratch; DLLM_ERR_SHAPE when it does not fit) and one coalesced pass rotates and
 * scatters them; head_dim a power of two.  rope_cos / rope_sin 16-byte aligned, q_out and
 * the caches 8-byte aligned, else DLLM_ERR_INVALID_ARG. */
int dllm_op_qkv_rope(const void* W, const void* X, int32_t rows_cap, const int32_t* count, int32_t d,
                     int32_t n_heads, int32_t n_kv_heads, int32_t head_dim, int32_t N, const int32_t* rows_map,
                     const float* rope_cos, const float* rope_sin, void* q_out, void* kcache, void* vcache,
                     int32_t splits, void* workspace, size_t workspace_bytes, void* stream);

/* Fused gate/up projection + SwiGLU: act bf16 [rows, F] = silu(X Wg^T) * (X Wu^T), W = [2F, d]. */
int dllm_op_gate_up(const void* W, int32_t F, const void* X, int32_t rows_cap, const int32_t* count, int32_t d,
                    void* act, int32_t splits, void* workspace, size_t workspace_bytes, void* stream);

/* Attention of the rows of each sequence (seq_off device int32 [B+1]) over all N cached keys.
 * q, out bf16 [rows, Hq*hd]; caches bf16 [B, Hkv, N, hd] (16-byte aligned); splits 0 = automatic
 * (key splits, merged afterwards).  Head dim 128 with at least 64 query units per sequence and
 * KV head (a unit is a (row, query head) pair) runs on the tensor cores, else on CUDA cores. */
int dllm_op_attention(const void* q, const void* kcache, const void* vcache, void* out, const int32_t* seq_off,
                      int32_t B, int32_t rows_cap, int32_t rows_per_seq_cap, int32_t N, int32_t n_heads,
                      int32_t n_kv_heads, int32_t head_dim, int32_t splits, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Vocabulary projection + confidence: for X bf16 [rows, d] (already normalised), conf / argmax / lse
 * per row written at out_index[j] (nullable: j); argmax excludes mask_id; conf = p(argmax). */
int dllm_op_lm_head(const void* W, int32_t V, const void* X, int32_t rows_cap, const int32_t* count, int32_t d,
                    int32_t mask_id, const int32_t* out_index, float* conf, int32_t* argmax, float* lse,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ES-dLLM Eq. 1 on rows[j] (rows nullable: j); with update != 0 also h_prev := h, masked_prev := (tok == mask). */
int dllm_op_score_es(const float* h, float* h_prev, const float* conf, uint8_t* masked_prev, const int32_t* tokens,
                     int32_t mask_id, const int32_t* rows, int32_t n_rows, int32_t d, float alpha, int32_t update,
                     float* score, void* stream);

/* dLLM-Cache cosine of v_new fp32 [rows, Hkv*hd] against the V cache rows of rows[j]. */
int dllm_op_score_cos(const float* vnew, const void* vcache, const int32_t* rows, const int32_t* count,
                      int32_t rows_cap, int32_t N, int32_t n_kv_heads, int32_t head_dim, float* sim, void* stream);

/* SureLock: from bf16 logits [rows, V], lse / conf / argmax at rows[j], and KL(p_t || p_prev)
 * against the stored bf16 logits zp_store[rows[j]] and lse_prev when has_prev[rows[j]] (else NaN). */
int dllm_op_kl_conf(const void* logits, const void* zp_store, const float* lse_prev, const int32_t* has_prev,
                    const int32_t* rows, const int32_t* count, int32_t rows_cap, int32_t V, int32_t mask_id,
                    float* conf, int32_t* argmax, float* lse, float* kl, void* stream);

/* Row selection over B sequences of n candidates (positions cand_start + i):
 * mode 0 top-k by score desc; 1 score < tau capped at the k lowest; 2 the k lowest;
 * 3 every row with lock[b*N + pos] == 0.  Ties go to the lower position.  Outputs
 * (all optional): act_pos [B, k_max] ascending, count [B], rows flat b*N+pos (b-major),
 * seq_off [B+1].  n <= 8192. */
int dllm_op_select(const float* scores, int32_t B, int32_t n, int32_t mode, int32_t k, float tau, int32_t cand_start,
                   int32_t N, const uint8_t* lock, int32_t* act_pos, int32_t k_max, int32_t* count, int32_t* rows,
                   int32_t* seq_off, void* stream);

/* Unmask within [blk_s, blk_s + blk_len) of each sequence.  mode DLLM_UNMASK_TOPCONF: the
 * n_commit masked positions with the highest conf (round_mask null), or every masked position
 * of the round (round_mask uint8 [blk_len], DUS); mode DLLM_UNMASK_CB_DUS: at most n_commit
 * positions with conf >= cb_tau (the best one always), none adjacent to another taken, in
 * confidence order (ties to the lower position).  tokens[b, pos] = argmax[b*N + pos].
 * remain (nullable): masked positions left in the block of each sequence afterwards. */
int dllm_op_unmask(int32_t* tokens, const float* conf, const int32_t* argmax, int32_t B, int32_t N, int32_t blk_s,
                   int32_t blk_len, int32_t mask_id, int32_t mode, int32_t n_commit, float cb_tau,
                   const uint8_t* round_mask, int32_t* pos_out, int32_t* tok_out, int32_t* n_out, int32_t max_out,
                   int32_t* remain, void* stream);

/* One transformer layer for the rows rows[j] (j < *count) of the hidden buffer h fp32 [B*N, d],
 * in place, with the layer's weights (pointers to layer l of w_qkv, w_o, w_gu, w_down, g_attn,
 * g_ffn) and caches (layer l, [B, Hkv, N, hd]).  seq_off [B+1] groups rows by sequence. */
int dllm_op_layer(const dllm_config* cfg, const void* w_qkv, const void* w_o, const void* w_gu, const void* w_down,
                  const float* g_attn, const float* g_ffn, void* kcache, void* vcache, const float* rope_cos,
                  const float* rope_sin, float* h, const int32_t* rows, const int32_t* count, const int32_t* seq_off,
                  int32_t rows_cap, int32_t rows_per_seq_cap, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes dllm_op_layer needs for rows_cap rows (zero it before its first use;
 * the GEMM tile counters at its start are left at zero by every call).  dllm_op_layer
 * takes its weights, gains, caches, RoPE tables and h 16-byte aligned and the workspace
 * 256-byte aligned, else DLLM_ERR_INVALID_ARG. */
int dllm_op_layer_workspace(const dllm_config* cfg, int32_t rows_cap, int32_t rows_per_seq_cap, size_t* bytes);

#ifdef __cplusplus
}
#endif
#endif /* DLLM_H_ */
