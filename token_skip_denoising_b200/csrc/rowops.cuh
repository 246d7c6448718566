// Host launchers of the row-wise kernels (rowops.cu) and the attention (attention.cu).
#pragma once
#include "common.cuh"

namespace dllm {

enum SelMode : int {
  SEL_TOPK_DESC = 0,       // keep the k highest scores (ties: lower index)
  SEL_BELOW_CAP_ASC = 1,   // rows with score < tau (NaN counts), at most k lowest
  SEL_FORCED_ASC = 2,      // exactly min(k, n) lowest scores
  SEL_ALL_ELIGIBLE = 3,    // every row whose lock flag is 0
};

struct SelectParams {
  const float* scores = nullptr;   // [B, n]
  int B = 0, n = 0;
  int mode = SEL_TOPK_DESC;
  int k = 0;
  float tau = 0.f;
  int cand_start = 0;              // candidate i is position cand_start + i
  int seq_n = 0;                   // sequence length N
  const uint8_t* lock = nullptr;   // [B, N] (SEL_ALL_ELIGIBLE)
  int* act_pos = nullptr;          // [B, k_max] ascending positions
  int k_max = 0;
  int* count = nullptr;            // [B]
  int* row_map = nullptr;          // flat rows, b-major
  int* seq_off = nullptr;          // [B + 1]
  int* total = nullptr;
  uint8_t* flag = nullptr;         // [B, seq_n]: 1 where a candidate is chosen, 0 where not
};

int rope_table_launch(float* cos_t, float* sin_t, int N, int hd, double theta, cudaStream_t st);
int embed_rows_launch(const __nv_bfloat16* E, int V, const int* tokens, const int* row_map, const int* count_dev,
                      int rows_cap, int d, float* h, cudaStream_t st);
// RoPE and K/V scatter of the rows' fp32 QKV products y [rows_cap, qkvd] (row j at position
// row_map[j] = b N + pos): q rotated to q_out [rows, qd], k rotated and v into the caches.
int rope_scatter_launch(const float* y, int rows_cap, const int* count_dev, const int* row_map, int qkvd, int qd,
                        int kvd, int hd, int N, int Hkv, const float* rope_cos, const float* rope_sin,
                        __nv_bfloat16* q_out, __nv_bfloat16* kc, __nv_bfloat16* vc, cudaStream_t st);
int rmsnorm_rows_launch(const float* h, const int* row_map, const int* count_dev, int rows_cap, int d, const float* g,
                        float eps, __nv_bfloat16* z, int64_t ldz, cudaStream_t st);
int score_es_launch(float* h, float* h_prev, const float* conf, uint8_t* masked_prev, const int* tokens,
                    int mask_id, const int* rows, int n_rows, int d, float alpha, int update,
                    const uint8_t* act_prev, float* score, cudaStream_t st);
int score_cos_launch(const float* vnew, int64_t ldv, const __nv_bfloat16* vc, const int* rows, const int* count_dev,
                     int rows_cap, int N, int Hkv, int hd, float* sim, cudaStream_t st);
// SureLock: statistics of the stored logits of each LM row, its divergence from the
// previous step's distribution and the lock decision (see KlStep in rowops.cu).
struct KlStep {
  const __nv_bfloat16* z_cur = nullptr;   // logits of this step, position-indexed [B*N, V]
  const __nv_bfloat16* z_prev = nullptr;  // previous step's logits, same layout
  const float* lse_prev = nullptr;        // [B*N]
  float* lse_cur = nullptr;               // [B*N]
  int* stamp = nullptr;                   // [B*N]: step + 1 at which a position's logits were stored
  int step = 0;
  const int* rows = nullptr;              // LM rows (flat) and their device count
  const int* count = nullptr;
  int rows_cap = 0;
  int V = 0, mask_id = 0;
  const int* tokens = nullptr;            // eligibility: token != mask at the start of the step
  uint8_t* lock = nullptr;
  const uint8_t* pattern = nullptr;       // forced locks (measurement mode) instead of the KL rule
  int lock_masked = 0;                    // masked positions are lock-eligible too
  float kl_eps = 0.f, conf_tau = 0.f;
  float* conf = nullptr;
  int* amax = nullptr;
  float* kl_out = nullptr;                // [rows]: divergence, NaN without a previous distribution
};
int kl_step_launch(const KlStep& k, cudaStream_t st);
int copy_rows_launch(const float* src, float* dst, const int* rows, const int* count_dev, int rows_cap, int d,
                     cudaStream_t st);

int kl_conf_launch(const __nv_bfloat16* z, int64_t ldz, const __nv_bfloat16* zp_store, int64_t ldp,
                   const float* lse_prev, const int* has_prev, const int* rows, const int* count_dev, int rows_cap,
                   int V, int mask_id, float* conf, int* amax, float* lse_out, float* kl_out, cudaStream_t st);
int select_launch(const SelectParams& p, cudaStream_t st);
int range_rows_launch(int B, int N, int start, int len, int* row_map, int* seq_off, int* total, cudaStream_t st);
// include_unmasked: also keep every recomputed row that is already unmasked (SureLock's
// lock-eligible rows need their distribution every step).
int lm_rows_launch(const int* rows, const int* count_dev, int rows_cap, const int* tokens, int mask_id, int N,
                   int blk_s, int blk_e, const uint8_t* round_mask, int include_unmasked, int* lm_rows, int* lm_count,
                   cudaStream_t st);
int snapshot_rows_launch(const float* h, float* h_prev, const int* tokens, uint8_t* masked_prev, int mask_id,
                         const int* rows, int n_rows, int d, cudaStream_t st);
// cb_mode: confidence-bounded, dilation-filtered choice (at most n_commit, conf >= cb_tau after the
// first, none adjacent); remain (nullable): masked positions left in the block per sequence.
int unmask_launch(int* tokens, const float* conf, const int* amax, int B, int N, int blk_s, int blk_len, int mask_id,
                  int n_commit, const uint8_t* round_mask, int cb_mode, float cb_tau, int* pos_out, int* tok_out,
                  int* n_out, int max_out, int* remain, cudaStream_t st);

size_t attn_partial_floats(int rows_cap, int Hq, int hd, int splits);
// Key splits attn_launch uses when given none (the tensor-core or the CUDA-core path).
int attn_pick_splits(int B, int Hkv, int G, int rows_per_seq, int N, int hd);
// Query units per (sequence, KV head) from which head dimension 128 runs on tcgen05 (attn_tc.cu).
constexpr int kAttnTcMinUnits = 64;
bool attn_use_tc(int hd, int G, int rows_per_seq);
int attn_tc_pick_splits(int B, int Hkv, int G, int rows_per_seq, int N);
int attn_counters_needed(int B, int Hkv, int G, int rows_per_seq);
// counters: zero on entry, left at zero.
int attn_launch(const __nv_bfloat16* q, const __nv_bfloat16* kc, const __nv_bfloat16* vc, __nv_bfloat16* out,
                const int* seq_off, int B, int rows_cap, int rows_per_seq_cap, int N, int Hq, int Hkv, int hd,
                int splits, float* opart, float2* ml, size_t partial_floats, int* counters, int n_counters,
                cudaStream_t st);

// A run of layers over at most kFusedMaxRows rows as one persistent kernel (fused_layer.cu).
constexpr int kFusedSyncInts = 16;
constexpr int kFusedMaxRows = 64;   // row sets the fused kernel serves (its sum buffers' rows)
// ES-dLLM choice inside the fused layer run: the first n_scored layers of the run are scored
// and the rows re-chosen at their start (1: the per-step choice at the skip layer; all: the
// per-layer re-selection).  Same definition as the score and select kernels:
// Eq. 1 on each candidate's layer input with the carry of skipped rows, the top k of each
// sequence (ties to the lower position) in ascending position order.
struct FusedEs {
  int on = 0;
  int n_scored = 0;                  // layers of the run, from its first, that choose (1: per step)
  int ls = 0, L = 0;                 // skip layer, layers of the model
  int B = 0, n_cand = 0, cand_start = 0, k = 0;
  float alpha = 0.f;
  int mask_id = 0;
  float* h_prev = nullptr;           // inputs of layer ls last iteration, position-indexed [B*N, d]
  float* es_in = nullptr;            // the same for layers ls+1 .. L-1: [L - ls - 1, B*N, d]
  const float* conf = nullptr;       // [B*N]
  uint8_t* masked_prev = nullptr;    // [B*N], rolled forward at the last layer
  const int* tokens = nullptr;       // [B*N]
  uint8_t* flag = nullptr;           // [B*N] chosen at the previous layer
  int* rows = nullptr;               // [B*k] the chosen rows (the run's row map)
  float* scores = nullptr;           // [B*n_cand] the latest layer's Eq. 1 scores
  const float* forced = nullptr;     // [n_layers, B, n_cand] scores used for the choice, or null
};
constexpr int kFusedEsMaxCand = 512;  // candidates per sequence the in-kernel choice ranks

struct FusedLayerArgs {
  int B, N, d, qd, kvd, qkvd, F, hd, Hq, Hkv;
  int L, l0, n_layers;              // layers l0 .. l0 + n_layers - 1 of L
  float eps;
  const __nv_bfloat16 *Wqkv, *Wo, *Wgu, *Wdn;   // weight stacks [L, rows, K] (layer 0)
  const float *g_attn, *g_ffn;                  // [L, d]
  __nv_bfloat16 *kc, *vc;                       // caches [L, B, Hkv, N, hd]
  const float *rope_cos, *rope_sin;
  float* h;
  const int* rows;
  const int* n_rows;
  const int* seq_off;
  int rows_cap, rows_per_seq;
  __nv_bfloat16 *z1, *z2, *q, *attn, *act;
  float* attn_opart;
  float2* attn_ml;
  size_t attn_floats;
  int* attn_ctr;           // fused_attn_counters(...) ints, zero before the launch; left zero
  int n_attn_ctr;
  float* scratch;          // fused_scratch_floats(qkvd, F): fp32 QKV and gate/up sums, per-CTA partial
                           // sums of squares, the ES choice's row sums; zero before the first launch,
                           // the kernel leaves it zero
  int* sync;               // kFusedSyncInts counters, zero before the launch; the kernel leaves them zero
  FusedEs es;              // per-layer re-selection (es.on = 0: the row map is fixed)
  int max_ctas = 0;        // grid bound the scratch was sized for (fused_scratch_floats)
  uint32_t spin_limit = 0; // polls of a grid-phase wait (0: the default)
};
size_t fused_scratch_floats(int qkvd, int F, int max_ctas);
int fused_attn_counters(int B, int Hq, int Hkv, int rows_cap);
int fused_layer_launch(const FusedLayerArgs& a, cudaStream_t st);

}  // namespace dllm
