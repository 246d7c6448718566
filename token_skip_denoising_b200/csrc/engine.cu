// The step engine behind the C ABI: validation, carving of caller memory,
// the generation schedule and the kernel sequence of one denoising step.
//
// Step kinds (the pages' denoising iteration with its four row policies):
//   FULL    every row through every layer: the vanilla step, ES-dLLM's
//           periodic refresh (ES-dLLM summary sec. 2.2), dLLM-Cache's prompt
//           refresh (dLLM-Cache explainer sec. 3).
//   SKIP    ES-dLLM (sec. 2.1): the candidates run the layers below the skip
//           layer, Eq. 1 scores them, the top k run the remaining layers.
//   LOCKED  SureLock (sec. 2.1): the unlocked rows run every layer; locked
//           rows keep their frozen K/V; unmasked rows are checked for locking.
//   PARTIAL dLLM-Cache: per layer, response rows whose value vectors moved
//           (cosine < tau, at most ceil(rho * n)) are recomputed; the rest
//           keep their cached layer output and K/V.
// No step synchronises the host: row counts live in device memory and the
// schedule (block, round) is known on the host in advance.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <set>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace dllm {

static thread_local std::string g_last_error;

void set_last_error(const char* msg, const char* file, int line) {
  char buf[512];
  snprintf(buf, sizeof buf, "%s (%s:%d)", msg, file, line);
  g_last_error = buf;
}

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_sms[kMaxDevices] = {};
std::set<std::pair<const void*, int>> g_attr_done;
}  // namespace

int num_sms() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return kDefaultSMs;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (g_sms[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return kDefaultSMs;
    }
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

int ensure_smem_attr(const void* fn, int bytes) {
  int dev = -1;
  DLLM_CUDA_TRY(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_attr_done.count({fn, dev})) return DLLM_OK;
  }
  DLLM_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  std::lock_guard<std::mutex> lock(g_dev_mu);
  g_attr_done.insert({fn, dev});
  return DLLM_OK;
}

#define DLLM_FAIL(code, msg)                              \
  do {                                                    \
    dllm::set_last_error((msg), __FILE__, __LINE__);      \
    return (code);                                        \
  } while (0)

#define DLLM_TRY(expr)             \
  do {                             \
    int _rc = (expr);              \
    if (_rc != DLLM_OK) return _rc; \
  } while (0)

namespace {

// Bump allocator over caller memory (256-byte aligned pieces).
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

int ceil_div(int a, int b) { return (a + b - 1) / b; }

int dus_rounds_for(int block) {
  if (block <= 1) return 1;
  int r = 0;
  while ((1 << r) < block) ++r;
  return r;
}

int keep_count(float ratio, int n) {
  if (n <= 0) return 0;
  const double k = std::ceil(static_cast<double>(ratio) * n - 1e-9);
  return std::max(1, std::min(n, static_cast<int>(k)));
}

int rho_cap_count(float rho, int n) {
  if (rho >= 1.f) return n;
  const double k = std::ceil(static_cast<double>(rho) * n - 1e-9);
  return std::max(0, std::min(n, static_cast<int>(k)));
}

int validate(const dllm_config* c) {
  if (!c) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null config");
  if (c->n_layers <= 0 || c->d_model <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
      c->ffn_dim <= 0 || c->vocab <= 1 || c->batch <= 0 || c->prompt_len < 0 || c->gen_len <= 0 ||
      c->block_len <= 0)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "non-positive dimension");
  if (c->mask_id < 0 || c->mask_id >= c->vocab) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "mask_id outside the vocabulary");
  if (c->gen_len % c->block_len) DLLM_FAIL(DLLM_ERR_SHAPE, "gen_len must be a multiple of block_len");
  if (c->n_heads % c->n_kv_heads) DLLM_FAIL(DLLM_ERR_SHAPE, "n_heads must be a multiple of n_kv_heads");
  if (c->head_dim != 64 && c->head_dim != 128) DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  const int qd = c->n_heads * c->head_dim, kvd = c->n_kv_heads * c->head_dim;
  if (qd % 128 || kvd % 128) DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "q and kv widths must be multiples of 128");
  if (c->d_model % 128) DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "d_model must be a multiple of 128");
  if (c->ffn_dim % 64) DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "ffn_dim must be a multiple of 64");
  if (c->vocab % 128) DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "vocab must be a multiple of 128");
  if (c->policy < DLLM_POLICY_VANILLA || c->policy > DLLM_POLICY_DLLM_CACHE)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "unknown policy");
  if (c->unmask != DLLM_UNMASK_TOPCONF && c->unmask != DLLM_UNMASK_DUS && c->unmask != DLLM_UNMASK_CB_DUS)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "unknown unmask");
  if (c->cand_scope != DLLM_SCOPE_BLOCK && c->cand_scope != DLLM_SCOPE_ALL)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "unknown candidate scope");
  if ((c->unmask == DLLM_UNMASK_TOPCONF || c->unmask == DLLM_UNMASK_CB_DUS) && c->tokens_per_step <= 0)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "tokens_per_step must be positive");
  if (c->unmask == DLLM_UNMASK_DUS && c->block_len == 2)
    DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "DUS: a block of 2 has no single-round non-adjacent schedule");
  if (c->block_len > 8192) DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "block_len above 8192");
  if (c->layer_kernel < DLLM_LAYER_AUTO || c->layer_kernel > DLLM_LAYER_FUSED)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "unknown layer_kernel");
  if (c->lock_masked != 0 && c->lock_masked != 1) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "lock_masked must be 0 or 1");
  if (c->es_per_layer != 0 && c->es_per_layer != 1) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "es_per_layer must be 0 or 1");
  if (c->policy == DLLM_POLICY_ES && c->es_per_layer && c->skip_layer >= c->n_layers)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "per-layer selection needs skip_layer < n_layers");
  if (c->policy == DLLM_POLICY_ES && (c->skip_layer < 0 || c->skip_layer > c->n_layers))
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "skip_layer outside [0, n_layers]");
  if (c->policy == DLLM_POLICY_ES && !(c->keep_ratio > 0.f && c->keep_ratio <= 1.f))
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "keep_ratio must be in (0, 1]");
  if (c->policy == DLLM_POLICY_DLLM_CACHE && c->prompt_interval <= 0)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "prompt_interval must be positive");
  const int N = c->prompt_len + c->gen_len;
  const int n_cand = c->cand_scope == DLLM_SCOPE_ALL ? N : c->block_len;
  if (n_cand > 8192 || N > 65536) DLLM_FAIL(DLLM_ERR_UNSUPPORTED, "sequence too long for the selection kernel");
  return DLLM_OK;
}

}  // namespace
}  // namespace dllm

using namespace dllm;

std::atomic<int64_t> dllm::g_kernel_launches{0};

// CUDA-event brackets around the fused GEMMs and the attention (roofline reporting).
struct Prof {
  struct Rec {
    cudaEvent_t a, b;
    int cls;            // 0 GEMM, 1 attention, 2 fused run of layers
    double bytes, flops;
    int layers;
  };
  bool on = false;
  int every = 1;                // bracket every n-th launch of each class
  int64_t seen[3] = {0, 0, 0};
  double hbm_gbs = 0, tflops = 0;
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e;
    cudaEventCreate(&e);
    return e;
  }
  void begin(cudaStream_t st, cudaEvent_t* a, int cls) {
    *a = nullptr;
    if (!on || (seen[cls]++ % every) != 0) return;
    *a = get();
    cudaEventRecord(*a, st);
  }
  void end(cudaStream_t st, cudaEvent_t a, int cls, double bytes, double flops, int layers = 0) {
    if (!on || !a) return;
    cudaEvent_t b = get();
    cudaEventRecord(b, st);
    recs.push_back({a, b, cls, bytes, flops, layers});
  }
  ~Prof() {
    for (auto& r : recs) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
    for (auto e : pool) cudaEventDestroy(e);
  }
};

struct dllm_handle {
  dllm_config c;
  dllm_weights w;
  int32_t* tokens;
  int N, B, L, d, qd, kvd, qkvd, F, V, hd;
  int n_cand, cand_start, k_keep, steps_per_block, n_rounds, n_resp, resp_start, resp_cap;
  // state
  __nv_bfloat16 *kcache, *vcache;
  float *h, *h_prev, *conf, *lse, *rope_cos, *rope_sin, *hcache;
  int* amax;
  uint8_t *masked_prev, *lock;
  __nv_bfloat16* zstore;   // SureLock: position-indexed bf16 logits, 2 buffers
  float* lse_store;        // 2 x [B*N]
  int* has_prev;           // [B*N] step + 1 at which the stored logits were written
  const uint8_t* lock_pattern = nullptr;   // SureLock forced-lock mode (measurement), caller-owned
  // workspace
  int *rows, *rows2, *nrows, *nrows2, *seq_off, *seq_off2, *lm_rows, *n_lm, *act_idx, *act_count;
  float *scores, *kl;
  uint8_t* round_masks;    // [R, block_len] (state constants)
  size_t const_bytes = 0, state_total = 0;
  Prof prof;
  __nv_bfloat16 *z, *q, *attn, *act;
  float* yqkv;             // [rows, qkvd] fp32 QKV products of the kernel-per-step layer
  float* vnew;
  float4* lm_part;
  GemmScratch gs;
  float* attn_opart;
  float2* attn_ml;
  size_t attn_floats;
  int* attn_ctr;
  int n_attn_ctr;
  __nv_bfloat16* z2;
  float* fused_scratch;
  int* fused_sync;         // state: phase counters of the fused layer kernel (zero between launches)
  int* fused_attn_ctr;     // state: split arrival counters of its attention step (zero between uses)
  int n_fused_attn_ctr;
  int n_sms = kDefaultSMs;          // SMs the fused kernel's per-CTA scratch was sized for
  uint32_t spin_limit = 0;          // fused kernel grid-phase wait limit (0: default)
  const float* forced_sims = nullptr;   // dLLM-Cache teacher forcing: [L, B, n_resp] (caller-owned)
  float* fused_opart;
  float2* fused_ml;
  size_t fused_attn_floats;
  // schedule
  int block = 0, step_in_block = 0, n_steps = 0;
  // current step
  int kind = DLLM_STEP_FULL;
  int cur_rows_cap = 0, cur_rows_per_seq = 0;
  int* cur_rows = nullptr;
  int* cur_n = nullptr;
  int* cur_seq_off = nullptr;
  int rows_first = 0;
  bool began = false;
  int* blk_remain = nullptr;   // workspace: masked positions left in the block per sequence (CB_DUS)
  // ES per-layer re-selection: the input of layer l seen last iteration for l > skip_layer
  // (layer skip_layer uses h_prev), the rows chosen at the previous layer, the next layer
  // select_active applies to
  float* es_in = nullptr;
  uint8_t* act_flag = nullptr;
  int es_layer = 0;
  std::vector<uint8_t> round_host;
};

namespace {

bool es_per_layer(const dllm_handle* x) { return x->c.policy == DLLM_POLICY_ES && x->c.es_per_layer; }

int lm_cap_of(const dllm_handle* hd) {
  const auto& c = hd->c;
  if (c.policy == DLLM_POLICY_SURELOCK) return hd->B * hd->N;
  return hd->B * c.block_len;
}

// Carve state (persistent) and workspace pieces; with null bases only sizes are computed.
void carve(dllm_handle* x, void* state, void* ws, size_t* state_bytes, size_t* ws_bytes) {
  const auto& c = x->c;
  const int64_t BN = static_cast<int64_t>(x->B) * x->N;
  Carver s(state);
  // constants (kept by dllm_reset): RoPE tables and DUS round masks
  x->rope_cos = s.take<float>(static_cast<size_t>(x->N) * x->hd / 2);
  x->rope_sin = s.take<float>(static_cast<size_t>(x->N) * x->hd / 2);
  x->round_masks = s.take<uint8_t>(static_cast<size_t>(x->n_rounds) * c.block_len);
  x->const_bytes = (s.off + 255) & ~size_t(255);
  const size_t kv = static_cast<size_t>(x->L) * x->B * c.n_kv_heads * x->N * x->hd;
  x->kcache = s.take<__nv_bfloat16>(kv);
  x->vcache = s.take<__nv_bfloat16>(kv);
  x->h = s.take<float>(BN * x->d);
  x->h_prev = c.policy == DLLM_POLICY_ES ? s.take<float>(BN * x->d) : nullptr;
  x->conf = s.take<float>(BN);
  x->lse = s.take<float>(BN);
  x->amax = s.take<int>(BN);
  x->masked_prev = s.take<uint8_t>(BN);
  x->lock = s.take<uint8_t>(BN);
  x->has_prev = s.take<int>(BN);
  x->fused_sync = s.take<int>(kFusedSyncInts);
  x->n_fused_attn_ctr = fused_attn_counters(x->B, c.n_heads, c.n_kv_heads, kFusedMaxRows);
  x->fused_attn_ctr = s.take<int>(x->n_fused_attn_ctr);
  if (c.policy == DLLM_POLICY_SURELOCK) {
    x->zstore = s.take<__nv_bfloat16>(2 * BN * x->V);
    x->lse_store = s.take<float>(2 * BN);
  } else {
    x->zstore = nullptr;
    x->lse_store = nullptr;
  }
  x->hcache = c.policy == DLLM_POLICY_DLLM_CACHE ? s.take<float>(static_cast<size_t>(x->L) * BN * x->d) : nullptr;
  const int n_es_in = es_per_layer(x) ? x->L - c.skip_layer - 1 : 0;
  x->es_in = n_es_in > 0 ? s.take<float>(static_cast<size_t>(n_es_in) * BN * x->d) : nullptr;
  x->state_total = (s.off + 255) & ~size_t(255);
  if (state_bytes) *state_bytes = x->state_total;

  Carver w(ws);
  x->rows = w.take<int>(BN);
  x->rows2 = w.take<int>(BN);
  x->nrows = w.take<int>(1);
  x->nrows2 = w.take<int>(1);
  x->seq_off = w.take<int>(x->B + 1);
  x->seq_off2 = w.take<int>(x->B + 1);
  x->lm_rows = w.take<int>(BN);
  x->n_lm = w.take<int>(1);
  x->act_idx = w.take<int>(BN);
  x->act_count = w.take<int>(x->B);
  x->blk_remain = w.take<int>(x->B);
  x->act_flag = c.policy == DLLM_POLICY_ES ? w.take<uint8_t>(BN) : nullptr;
  x->scores = w.take<float>(BN);
  x->kl = w.take<float>(BN);
  const int64_t R = BN;   // row bound of any step
  x->z = w.take<__nv_bfloat16>(R * x->d);
  x->q = w.take<__nv_bfloat16>(R * x->qd);
  x->attn = w.take<__nv_bfloat16>(R * x->qd);
  x->act = w.take<__nv_bfloat16>(R * x->F);
  x->yqkv = w.take<float>(R * x->qkvd);
  x->vnew = c.policy == DLLM_POLICY_DLLM_CACHE ? w.take<float>(static_cast<size_t>(x->B) * x->n_resp * x->kvd) : nullptr;
  const int lm_cap = lm_cap_of(x);
  x->lm_part = w.take<float4>(c.policy == DLLM_POLICY_SURELOCK ? 0 : static_cast<size_t>(lm_cap) * (x->V / 128));
  // split-K scratch: the largest need over the row counts a step can use
  std::vector<int> caps = {static_cast<int>(BN), x->B * x->n_cand, x->B * x->k_keep, x->B * x->n_resp, lm_cap};
  size_t pf = 0;
  int ctr = 0;
  for (int cap : caps) {
    if (cap <= 0) continue;
    const int tiles[5] = {x->qkvd / 128, x->d / 128, x->F / 64, x->kvd / 128, x->V / 128};
    const int Ks[5] = {x->d, x->qd, x->d, x->d, x->d};
    for (int i = 0; i < 5; ++i) {
      pf = std::max(pf, gemm_partial_floats(cap, tiles[i], Ks[i]));
      ctr = std::max(ctr, gemm_counters_needed(cap, tiles[i]));
    }
    pf = std::max(pf, gemm_partial_floats(cap, x->d / 128, x->F));
  }
  x->gs.partial = w.take<float>(pf);
  x->gs.partial_floats = pf;
  x->gs.counters = w.take<int>(ctr);
  x->gs.n_counters = ctr;
  size_t af = 0;
  const int G = c.n_heads / c.n_kv_heads;
  for (int cap_seq : {x->N, x->n_cand, x->k_keep, x->n_resp}) {
    if (cap_seq <= 0) continue;
    const int sp = attn_pick_splits(x->B, c.n_kv_heads, G, cap_seq, x->N, x->hd);
    if (sp > 1) af = std::max(af, attn_partial_floats(x->B * cap_seq, c.n_heads, x->hd, sp));
  }
  x->attn_opart = w.take<float>(af);
  x->attn_floats = af;
  size_t ml = af / std::max(1, x->hd);
  x->attn_ml = w.take<float2>(ml);
  // fused small-row layer scratch
  x->z2 = w.take<__nv_bfloat16>(static_cast<size_t>(kFusedMaxRows) * x->d);
  x->n_sms = num_sms();
  x->fused_scratch = w.take<float>(fused_scratch_floats(x->qkvd, x->F, x->n_sms));
  x->fused_attn_floats = static_cast<size_t>((x->N + 63) / 64) * kFusedMaxRows * c.n_heads * x->hd;
  x->fused_opart = w.take<float>(x->fused_attn_floats);
  x->fused_ml = w.take<float2>(x->fused_attn_floats / x->hd);
  int actr = 0;
  for (int cap_seq : {x->N, x->n_cand, x->k_keep, x->n_resp})
    if (cap_seq > 0) actr = std::max(actr, attn_counters_needed(x->B, c.n_kv_heads, G, cap_seq));
  x->attn_ctr = w.take<int>(actr);
  x->n_attn_ctr = actr;
  if (ws_bytes) *ws_bytes = (w.off + 255) & ~size_t(255);
}

void fill_dims(dllm_handle* x, const dllm_config* c) {
  x->c = *c;
  x->N = c->prompt_len + c->gen_len;
  x->B = c->batch;
  x->L = c->n_layers;
  x->d = c->d_model;
  x->hd = c->head_dim;
  x->qd = c->n_heads * c->head_dim;
  x->kvd = c->n_kv_heads * c->head_dim;
  x->qkvd = x->qd + 2 * x->kvd;
  x->F = c->ffn_dim;
  x->V = c->vocab;
  x->cand_start = c->cand_scope == DLLM_SCOPE_ALL ? 0 : c->prompt_len;   // plus block offset at run time
  x->n_cand = c->cand_scope == DLLM_SCOPE_ALL ? x->N : c->block_len;
  x->k_keep = c->policy == DLLM_POLICY_ES ? keep_count(c->keep_ratio, x->n_cand) : x->n_cand;
  x->n_rounds = dus_rounds_for(c->block_len);
  x->steps_per_block = c->unmask == DLLM_UNMASK_DUS      ? x->n_rounds
                       : c->unmask == DLLM_UNMASK_CB_DUS ? c->block_len   // an upper bound: the block ends when done
                                                         : ceil_div(c->block_len, c->tokens_per_step);
  x->resp_start = c->cand_scope == DLLM_SCOPE_ALL ? 0 : c->prompt_len;
  x->n_resp = x->N - x->resp_start;
  x->resp_cap = rho_cap_count(c->rho_cap, x->n_resp);
}

int blk_start(const dllm_handle* x) { return x->c.prompt_len + x->block * x->c.block_len; }

int cand_first(const dllm_handle* x) {
  return x->c.cand_scope == DLLM_SCOPE_ALL ? 0 : blk_start(x);
}

// Everything one transformer layer needs (weights of the layer, its caches, scratch).
struct LayerCtx {
  int B, N, d, qd, kvd, qkvd, F, hd, Hq, Hkv;
  float eps;
  const __nv_bfloat16 *Wqkv, *Wo, *Wgu, *Wdn;
  const float *g_attn, *g_ffn;
  __nv_bfloat16 *kc, *vc;
  const float *rope_cos, *rope_sin;
  __nv_bfloat16 *z, *q, *attn, *act;
  float* yqkv;             // [rows, qkvd] fp32 QKV products of the kernel-per-step layer
  GemmScratch gs;
  float* attn_opart;
  float2* attn_ml;
  size_t attn_floats;
  int* attn_ctr = nullptr;
  int n_attn_ctr = 0;
  Prof* prof = nullptr;
  // fused small-row layers (used when `fused` is set and the scratch below is present): the
  // kernel addresses whole weight stacks and caches, so the context also holds layer 0's pointers
  bool fused = false;
  int layer = 0, n_layers_total = 1;
  const __nv_bfloat16 *Wqkv0 = nullptr, *Wo0 = nullptr, *Wgu0 = nullptr, *Wdn0 = nullptr;
  const float *g_attn0 = nullptr, *g_ffn0 = nullptr;
  __nv_bfloat16 *kc0 = nullptr, *vc0 = nullptr;
  __nv_bfloat16* z2 = nullptr;
  float* fused_scratch = nullptr;
  int* fused_sync = nullptr;
  int* fused_attn_ctr = nullptr;
  int n_fused_attn_ctr = 0;
  float* fused_opart = nullptr;
  float2* fused_ml = nullptr;
  size_t fused_attn_floats = 0;
  int max_ctas = kDefaultSMs;       // grid bound its per-CTA scratch was sized for
  uint32_t spin_limit = 0;
};

// GEMM launch with optional event bracketing; bytes / flops are the algorithmic figures
// (weights + activation rows + outputs) for rows_cap rows.
int timed_gemm(Prof* prof, const GemmArgs& g, const GemmScratch& gs, cudaStream_t st, double out_bytes_per_row) {
  cudaEvent_t a = nullptr;
  if (prof) prof->begin(st, &a, 0);
  const int rc = gemm_launch(g, gs, st);
  if (prof && a) {
    const double wrows = g.swiglu ? 2.0 * g.epi.ffn : 128.0 * g.n_tiles_w;
    const double bytes = wrows * g.K * 2.0 + static_cast<double>(g.rows_cap) * (g.K * 2.0 + out_bytes_per_row);
    prof->end(st, a, 0, bytes, 2.0 * g.rows_cap * wrows * g.K);
  }
  return rc;
}

// The fused persistent kernel serves row sets of at most kFusedMaxRows rows.
bool fused_applies(const LayerCtx& x, int rows_cap) { return x.fused && x.fused_sync && rows_cap <= kFusedMaxRows; }

// Layers x.layer .. x.layer + n_layers - 1 as one fused persistent kernel (DLLM_ERR_UNSUPPORTED
// when the shapes do not allow it).
int run_fused_layers(const LayerCtx& x, int n_layers, float* hbuf, const int* rows, const int* n, const int* seq_off,
                     int rows_cap, int rows_per_seq, cudaStream_t st, const FusedEs* es = nullptr) {
  FusedLayerArgs a;
  if (es) a.es = *es;
  a.B = x.B; a.N = x.N; a.d = x.d; a.qd = x.qd; a.kvd = x.kvd; a.qkvd = x.qkvd; a.F = x.F; a.hd = x.hd;
  a.Hq = x.Hq; a.Hkv = x.Hkv; a.eps = x.eps;
  a.L = x.n_layers_total; a.l0 = x.layer; a.n_layers = n_layers;
  a.Wqkv = x.Wqkv0; a.Wo = x.Wo0; a.Wgu = x.Wgu0; a.Wdn = x.Wdn0; a.g_attn = x.g_attn0; a.g_ffn = x.g_ffn0;
  a.kc = x.kc0; a.vc = x.vc0; a.rope_cos = x.rope_cos; a.rope_sin = x.rope_sin;
  a.h = hbuf; a.rows = rows; a.n_rows = n; a.seq_off = seq_off; a.rows_cap = rows_cap; a.rows_per_seq = rows_per_seq;
  a.z1 = x.z2; a.z2 = x.z; a.q = x.q; a.attn = x.attn; a.act = x.act;   // x.z ends with the FFN RMSNorm, as below
  a.attn_opart = x.fused_opart; a.attn_ml = x.fused_ml; a.attn_floats = x.fused_attn_floats;
  a.attn_ctr = x.fused_attn_ctr; a.n_attn_ctr = x.n_fused_attn_ctr;
  a.scratch = x.fused_scratch;
  a.sync = x.fused_sync;
  a.max_ctas = x.max_ctas;
  a.spin_limit = x.spin_limit;
  cudaEvent_t ev = nullptr;
  if (x.prof) x.prof->begin(st, &ev, 2);
  const int rc = fused_layer_launch(a, st);
  if (x.prof && ev) {
    // algorithmic traffic per layer: the four weight matrices, this layer's K and V cache (read by
    // attention), and the rows' hidden state, operands and sums (bound: rows_cap rows)
    const double P = static_cast<double>(x.qkvd) * x.d + static_cast<double>(x.d) * x.qd + 3.0 * x.d * x.F;
    const double kv = 2.0 * x.B * x.Hkv * static_cast<double>(x.N) * x.hd * 2.0;
    const double rowb = static_cast<double>(rows_cap) * (8.0 * x.d + 4.0 * (x.qkvd + 2.0 * x.F) + 2.0 * x.F);
    const double fl = 2.0 * rows_cap * P + 4.0 * rows_cap * static_cast<double>(x.N) * x.Hq * x.hd;
    x.prof->end(st, ev, 2, n_layers * (2.0 * P + kv + rowb), n_layers * fl, n_layers);
  }
  return rc;
}

// One transformer layer on rows[j] (j < *n) of the position-indexed hidden buffer hbuf:
// RMSNorm gather -> QKV (+RoPE, K/V scatter) -> attention over all cached keys ->
// O (+residual) -> RMSNorm -> gate/up (+SwiGLU) -> down (+residual).
int run_layer(const LayerCtx& x, float* hbuf, const int* rows, const int* n, const int* seq_off, int rows_cap,
              int rows_per_seq, cudaStream_t st) {
  if (fused_applies(x, rows_cap)) {
    const int rc = run_fused_layers(x, 1, hbuf, rows, n, seq_off, rows_cap, rows_per_seq, st);
    if (rc != DLLM_ERR_UNSUPPORTED) return rc;
  }
  DLLM_TRY(rmsnorm_rows_launch(hbuf, rows, n, rows_cap, x.d, x.g_attn, x.eps, x.z, x.d, st));
  GemmArgs g;
  g.W = x.Wqkv; g.w_rows_total = x.qkvd; g.X = x.z; g.rows_cap = rows_cap; g.rows_dev = n; g.K = x.d;
  g.n_tiles_w = x.qkvd / 128;
  // fp32 products, then RoPE and the K/V scatter as one coalesced pass (a rotation inside the
  // GEMM epilogue waits on the row map and the cos/sin table in every 16-column chunk)
  g.epi.kind = EPI_STORE_F32; g.epi.out = x.yqkv; g.epi.ldo = x.qkvd; g.wide_ok = true;
  DLLM_TRY(timed_gemm(x.prof, g, x.gs, st, 4.0 * x.qkvd));
  DLLM_TRY(rope_scatter_launch(x.yqkv, rows_cap, n, rows, x.qkvd, x.qd, x.kvd, x.hd, x.N, x.Hkv, x.rope_cos,
                               x.rope_sin, x.q, x.kc, x.vc, st));
  {
    cudaEvent_t a = nullptr;
    if (x.prof) x.prof->begin(st, &a, 1);
    DLLM_TRY(attn_launch(x.q, x.kc, x.vc, x.attn, seq_off, x.B, rows_cap, rows_per_seq, x.N, x.Hq, x.Hkv, x.hd, 0,
                         x.attn_opart, x.attn_ml, x.attn_floats, x.attn_ctr, x.n_attn_ctr, st));
    if (x.prof && a) {
      const double kvb = 2.0 * x.B * x.Hkv * static_cast<double>(x.N) * x.hd * 2.0;
      x.prof->end(st, a, 1, kvb + 4.0 * rows_cap * x.qd, 4.0 * rows_cap * x.Hq * static_cast<double>(x.N) * x.hd);
    }
  }
  GemmArgs o;
  o.W = x.Wo; o.w_rows_total = x.d; o.X = x.attn; o.rows_cap = rows_cap; o.rows_dev = n; o.K = x.qd;
  o.n_tiles_w = x.d / 128;
  o.epi.kind = EPI_RESID_ADD; o.epi.h = hbuf; o.epi.ldh = x.d; o.epi.row_map = rows;
  DLLM_TRY(timed_gemm(x.prof, o, x.gs, st, 8.0 * x.d));
  DLLM_TRY(rmsnorm_rows_launch(hbuf, rows, n, rows_cap, x.d, x.g_ffn, x.eps, x.z, x.d, st));
  GemmArgs gu;
  gu.W = x.Wgu; gu.w_rows_total = 2 * x.F; gu.X = x.z; gu.rows_cap = rows_cap; gu.rows_dev = n; gu.K = x.d;
  gu.n_tiles_w = x.F / 64; gu.swiglu = true;
  gu.epi.kind = EPI_SWIGLU; gu.epi.act = x.act; gu.epi.ffn = x.F;
  DLLM_TRY(timed_gemm(x.prof, gu, x.gs, st, 2.0 * x.F));
  GemmArgs dn;
  dn.W = x.Wdn; dn.w_rows_total = x.d; dn.X = x.act; dn.rows_cap = rows_cap; dn.rows_dev = n; dn.K = x.F;
  dn.n_tiles_w = x.d / 128;
  dn.epi.kind = EPI_RESID_ADD; dn.epi.h = hbuf; dn.epi.ldh = x.d; dn.epi.row_map = rows;
  DLLM_TRY(timed_gemm(x.prof, dn, x.gs, st, 8.0 * x.d));
  return DLLM_OK;
}

LayerCtx layer_ctx(const dllm_handle* x, int l) {
  LayerCtx L;
  const auto& c = x->c;
  L.B = x->B; L.N = x->N; L.d = x->d; L.qd = x->qd; L.kvd = x->kvd; L.qkvd = x->qkvd; L.F = x->F; L.hd = x->hd;
  L.Hq = c.n_heads; L.Hkv = c.n_kv_heads; L.eps = c.rms_eps;
  L.Wqkv = static_cast<const __nv_bfloat16*>(x->w.w_qkv) + static_cast<size_t>(l) * x->qkvd * x->d;
  L.Wo = static_cast<const __nv_bfloat16*>(x->w.w_o) + static_cast<size_t>(l) * x->d * x->qd;
  L.Wgu = static_cast<const __nv_bfloat16*>(x->w.w_gu) + static_cast<size_t>(l) * 2 * x->F * x->d;
  L.Wdn = static_cast<const __nv_bfloat16*>(x->w.w_down) + static_cast<size_t>(l) * x->d * x->F;
  L.g_attn = x->w.g_attn + static_cast<size_t>(l) * x->d;
  L.g_ffn = x->w.g_ffn + static_cast<size_t>(l) * x->d;
  const size_t kvl = static_cast<size_t>(x->B) * c.n_kv_heads * x->N * x->hd;
  L.kc = x->kcache + l * kvl;
  L.vc = x->vcache + l * kvl;
  L.rope_cos = x->rope_cos; L.rope_sin = x->rope_sin;
  L.z = x->z; L.q = x->q; L.attn = x->attn; L.act = x->act; L.yqkv = x->yqkv;
  L.gs = x->gs;
  L.attn_opart = x->attn_opart; L.attn_ml = x->attn_ml; L.attn_floats = x->attn_floats;
  L.attn_ctr = x->attn_ctr; L.n_attn_ctr = x->n_attn_ctr;
  L.fused = c.layer_kernel != DLLM_LAYER_SPLIT;   // AUTO: the fused layer whenever it applies
  L.layer = l;
  L.n_layers_total = x->L;
  L.Wqkv0 = static_cast<const __nv_bfloat16*>(x->w.w_qkv);
  L.Wo0 = static_cast<const __nv_bfloat16*>(x->w.w_o);
  L.Wgu0 = static_cast<const __nv_bfloat16*>(x->w.w_gu);
  L.Wdn0 = static_cast<const __nv_bfloat16*>(x->w.w_down);
  L.g_attn0 = x->w.g_attn;
  L.g_ffn0 = x->w.g_ffn;
  L.kc0 = x->kcache;
  L.vc0 = x->vcache;
  L.z2 = x->z2; L.fused_scratch = x->fused_scratch; L.fused_sync = x->fused_sync;
  L.fused_attn_ctr = x->fused_attn_ctr; L.n_fused_attn_ctr = x->n_fused_attn_ctr;
  L.fused_opart = x->fused_opart; L.fused_ml = x->fused_ml; L.fused_attn_floats = x->fused_attn_floats;
  L.max_ctas = x->n_sms;
  L.spin_limit = x->spin_limit;
  L.prof = const_cast<Prof*>(&x->prof);
  return L;
}

// The single-layer op's share of the fused kernel's buffers (row sets of at most
// kFusedMaxRows rows, unless the configuration asks for the kernel-per-step layer); with a
// null context only sizes are taken.  Its counters rely on the op workspace being zeroed once.
void carve_fused_op(Carver& w, const dllm_config* cfg, int rows_cap, LayerCtx* L) {
  if (rows_cap > kFusedMaxRows || cfg->layer_kernel == DLLM_LAYER_SPLIT) return;
  const int d = cfg->d_model, qd = cfg->n_heads * cfg->head_dim, kvd = cfg->n_kv_heads * cfg->head_dim;
  const int N = cfg->prompt_len + cfg->gen_len;
  int* sync = w.take<int>(kFusedSyncInts);
  const int n_ctr = fused_attn_counters(cfg->batch, cfg->n_heads, cfg->n_kv_heads, kFusedMaxRows);
  int* ctr = w.take<int>(n_ctr);
  __nv_bfloat16* z2 = w.take<__nv_bfloat16>(static_cast<size_t>(kFusedMaxRows) * d);
  const int sms = num_sms();
  float* scratch = w.take<float>(fused_scratch_floats(qd + 2 * kvd, cfg->ffn_dim, sms));
  const size_t af = static_cast<size_t>((N + 63) / 64) * kFusedMaxRows * cfg->n_heads * cfg->head_dim;
  float* opart = w.take<float>(af);
  float2* ml = w.take<float2>(af / cfg->head_dim);
  if (!L) return;
  L->fused = true;
  L->layer = 0;
  L->n_layers_total = 1;
  L->Wqkv0 = L->Wqkv; L->Wo0 = L->Wo; L->Wgu0 = L->Wgu; L->Wdn0 = L->Wdn;
  L->g_attn0 = L->g_attn; L->g_ffn0 = L->g_ffn;
  L->kc0 = L->kc; L->vc0 = L->vc;
  L->z2 = z2;
  L->fused_scratch = scratch;
  L->fused_sync = sync;
  L->fused_attn_ctr = ctr;
  L->n_fused_attn_ctr = n_ctr;
  L->fused_opart = opart;
  L->fused_ml = ml;
  L->fused_attn_floats = af;
  L->max_ctas = sms;
}

// Per-layer ES selection: from the skip layer on, each layer runs alone and right after
// its select_active call.
int per_layer_order(const dllm_handle* x, int l0, int l1) {
  if (!es_per_layer(x) || l1 <= x->c.skip_layer) return DLLM_OK;
  if (l1 - l0 == 1 && l0 >= x->c.skip_layer && x->es_layer == l0 + 1) return DLLM_OK;
  DLLM_FAIL(DLLM_ERR_STATE, "per-layer selection: each layer from skip_layer on runs alone, after select_active");
}

// ES-dLLM sec. 2.1 item 2, per layer: the top k chosen at the start of layer es_layer.
// Refresh steps snapshot each candidate's input of the layer instead.
int select_layer(dllm_handle* x, const float* forced, int32_t* active_idx, int32_t* active_count, cudaStream_t st) {
  const auto& c = x->c;
  const int l = x->es_layer, ls = c.skip_layer;
  if (l >= x->L) DLLM_FAIL(DLLM_ERR_STATE, "select_active after the last layer");
  const int64_t BNd = static_cast<int64_t>(x->B) * x->N * x->d;
  float* prev = l == ls ? x->h_prev : x->es_in + (l - ls - 1) * BNd;
  const int ncand = x->B * x->n_cand;
  if (x->kind == DLLM_STEP_FULL) {
    if (l == ls) {
      DLLM_TRY(range_rows_launch(x->B, x->N, cand_first(x), x->n_cand, x->rows2, x->seq_off2, x->nrows2, st));
      DLLM_TRY(snapshot_rows_launch(x->h, x->h_prev, x->tokens, x->masked_prev, c.mask_id, x->rows2, ncand, x->d, st));
    } else {
      DLLM_TRY(copy_rows_launch(x->h, prev, x->rows2, x->nrows2, ncand, x->d, st));
    }
    x->es_layer += 1;
    return DLLM_OK;
  }
  if (x->kind != DLLM_STEP_SKIP) DLLM_FAIL(DLLM_ERR_STATE, "select_active outside an ES step");
  // Eq. 1 on this layer's input; rows the previous layer skipped take their cached output
  // (their input last iteration) and score the confidence term alone.  masked_prev rolls
  // forward at the last layer, after every layer has read it.
  DLLM_TRY(score_es_launch(x->h, prev, x->conf, x->masked_prev, l == x->L - 1 ? x->tokens : nullptr, c.mask_id,
                           x->rows, ncand, x->d, c.alpha, 1, l > ls ? x->act_flag : nullptr, x->scores, st));
  SelectParams sp;
  sp.scores = forced ? forced : x->scores;
  sp.B = x->B; sp.n = x->n_cand; sp.mode = SEL_TOPK_DESC; sp.k = x->k_keep; sp.cand_start = cand_first(x);
  sp.seq_n = x->N; sp.act_pos = active_idx ? active_idx : x->act_idx; sp.k_max = x->k_keep;
  sp.count = active_count ? active_count : x->act_count; sp.row_map = x->rows2; sp.seq_off = x->seq_off2;
  sp.total = x->nrows2; sp.flag = x->act_flag;
  DLLM_TRY(select_launch(sp, st));
  x->cur_rows = x->rows2;
  x->cur_n = x->nrows2;
  x->cur_seq_off = x->seq_off2;
  x->cur_rows_cap = x->B * x->k_keep;
  x->cur_rows_per_seq = x->k_keep;
  x->es_layer += 1;
  return DLLM_OK;
}

// Layers skip_layer .. L-1 of an ES skip step as one fused launch that scores and chooses the
// rows itself: at the skip layer, or at the start of every layer with es_per_layer
// (DLLM_ERR_UNSUPPORTED when it does not apply).
int fused_es_run(dllm_handle* x, const float* forced, cudaStream_t st) {
  const auto& c = x->c;
  const int ls = c.skip_layer;
  const LayerCtx L0 = layer_ctx(x, ls);
  const int cap = x->B * x->k_keep;
  if (!fused_applies(L0, cap) || x->n_cand > kFusedEsMaxCand) return DLLM_ERR_UNSUPPORTED;
  // the row counts and sequence offsets of k rows per sequence (the kernel fills the rows)
  DLLM_TRY(range_rows_launch(x->B, x->N, cand_first(x), x->k_keep, x->rows2, x->seq_off2, x->nrows2, st));
  FusedEs e;
  e.on = 1;
  e.n_scored = c.es_per_layer ? x->L - ls : 1;
  e.ls = ls; e.L = x->L;
  e.B = x->B; e.n_cand = x->n_cand; e.cand_start = cand_first(x); e.k = x->k_keep;
  e.alpha = c.alpha; e.mask_id = c.mask_id;
  e.h_prev = x->h_prev; e.es_in = x->es_in;
  e.conf = x->conf; e.masked_prev = x->masked_prev; e.tokens = x->tokens;
  e.flag = x->act_flag; e.rows = x->rows2; e.scores = x->scores; e.forced = forced;
  const int rc = run_fused_layers(L0, x->L - ls, x->h, x->rows2, x->nrows2, x->seq_off2, cap, x->k_keep, st, &e);
  if (rc) return rc;
  x->cur_rows = x->rows2;
  x->cur_n = x->nrows2;
  x->cur_seq_off = x->seq_off2;
  x->cur_rows_cap = cap;
  x->cur_rows_per_seq = x->k_keep;
  x->es_layer = x->L;
  return DLLM_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* dllm_status_string(int s) {
  switch (s) {
    case DLLM_OK: return "ok";
    case DLLM_ERR_INVALID_ARG: return "invalid argument";
    case DLLM_ERR_SHAPE: return "shape mismatch";
    case DLLM_ERR_UNSUPPORTED: return "unsupported";
    case DLLM_ERR_CUDA: return "CUDA error";
    case DLLM_ERR_TIMEOUT: return "device wait timed out";
    case DLLM_ERR_DEVICE: return "device status set";
    case DLLM_ERR_STATE: return "call out of order";
    default: return "unknown status";
  }
}

const char* dllm_last_error(void) { return g_last_error.c_str(); }

int dllm_state_bytes(const dllm_config* cfg, size_t* state_bytes, size_t* workspace_bytes) {
  DLLM_TRY(validate(cfg));
  dllm_handle x{};
  fill_dims(&x, cfg);
  carve(&x, nullptr, nullptr, state_bytes, workspace_bytes);
  return DLLM_OK;
}

int dllm_step_init(dllm_handle** out, const dllm_config* cfg, const dllm_weights* w, void* state, void* workspace,
                   int32_t* tokens, void* stream) {
  if (!out || !w || !state || !workspace || !tokens) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null argument");
  DLLM_TRY(validate(cfg));
  if (!w->embed || !w->lm_head || !w->w_qkv || !w->w_o || !w->w_gu || !w->w_down || !w->g_attn || !w->g_ffn ||
      !w->g_final)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null weight pointer");
  if ((reinterpret_cast<uintptr_t>(state) | reinterpret_cast<uintptr_t>(workspace)) & 255)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "state and workspace must be 256-byte aligned");
  // the kernels read weights and gains as 16-byte vectors (and through TMA)
  const void* wp[9] = {w->embed, w->lm_head, w->w_qkv, w->w_o, w->w_gu, w->w_down, w->g_attn, w->g_ffn, w->g_final};
  for (const void* p : wp)
    if (reinterpret_cast<uintptr_t>(p) & 15) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "weights must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(tokens) & 3) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "tokens must be 4-byte aligned");
  dllm_handle* x = new (std::nothrow) dllm_handle();
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "out of host memory");
  fill_dims(x, cfg);
  x->w = *w;
  x->tokens = tokens;
  size_t sb = 0, wb = 0;
  carve(x, state, workspace, &sb, &wb);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto fail = [&](int rc) { delete x; return rc; };
  if (cudaMemsetAsync(state, 0, sb, st) != cudaSuccess) { set_last_error("memset state", __FILE__, __LINE__); return fail(DLLM_ERR_CUDA); }
  if (cudaMemsetAsync(workspace, 0, wb, st) != cudaSuccess) { set_last_error("memset workspace", __FILE__, __LINE__); return fail(DLLM_ERR_CUDA); }
  int rc = rope_table_launch(x->rope_cos, x->rope_sin, x->N, x->hd, cfg->rope_theta, st);
  if (rc) return fail(rc);
  // DUS round masks: round r takes positions divisible by 2^(R-1-r) not taken earlier
  x->round_host.assign(static_cast<size_t>(x->n_rounds) * cfg->block_len, 0);
  std::vector<uint8_t> taken(cfg->block_len, 0);
  for (int r = 0; r < x->n_rounds; ++r) {
    const int stride = 1 << (x->n_rounds - 1 - r);
    for (int p = 0; p < cfg->block_len; ++p)
      if (p % stride == 0 && !taken[p]) { taken[p] = 1; x->round_host[static_cast<size_t>(r) * cfg->block_len + p] = 1; }
  }
  if (cudaMemcpyAsync(x->round_masks, x->round_host.data(), x->round_host.size(), cudaMemcpyHostToDevice, st) !=
      cudaSuccess) { set_last_error("round masks", __FILE__, __LINE__); return fail(DLLM_ERR_CUDA); }
  // the host vector must outlive the copy
  if (cudaStreamSynchronize(st) != cudaSuccess) { set_last_error("init sync", __FILE__, __LINE__); return fail(DLLM_ERR_CUDA); }
  *out = x;
  return DLLM_OK;
}

int dllm_done(const dllm_handle* h) { return (!h || h->block >= h->c.gen_len / h->c.block_len) ? 1 : 0; }

int dllm_begin_step(dllm_handle* x, int32_t* kind_out, void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (dllm_done(x)) DLLM_FAIL(DLLM_ERR_STATE, "generation finished");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto& c = x->c;
  const int BN = x->B * x->N;
  int kind = DLLM_STEP_FULL;
  switch (c.policy) {
    case DLLM_POLICY_VANILLA: kind = DLLM_STEP_FULL; break;
    case DLLM_POLICY_ES: {
      const bool refresh = x->step_in_block == 0 || (c.refresh_period > 0 && x->step_in_block % c.refresh_period == 0);
      kind = refresh ? DLLM_STEP_FULL : DLLM_STEP_SKIP;
      break;
    }
    case DLLM_POLICY_SURELOCK: kind = DLLM_STEP_LOCKED; break;
    case DLLM_POLICY_DLLM_CACHE: kind = (x->n_steps % c.prompt_interval == 0) ? DLLM_STEP_FULL : DLLM_STEP_PARTIAL; break;
  }
  x->kind = kind;
  if (kind == DLLM_STEP_FULL) {
    DLLM_TRY(range_rows_launch(x->B, x->N, 0, x->N, x->rows, x->seq_off, x->nrows, st));
    x->cur_rows_cap = BN;
    x->cur_rows_per_seq = x->N;
  } else if (kind == DLLM_STEP_SKIP) {
    DLLM_TRY(range_rows_launch(x->B, x->N, cand_first(x), x->n_cand, x->rows, x->seq_off, x->nrows, st));
    x->cur_rows_cap = x->B * x->n_cand;
    x->cur_rows_per_seq = x->n_cand;
  } else if (kind == DLLM_STEP_LOCKED) {
    SelectParams sp;
    sp.B = x->B; sp.n = x->N; sp.mode = SEL_ALL_ELIGIBLE; sp.cand_start = 0; sp.seq_n = x->N; sp.lock = x->lock;
    sp.row_map = x->rows; sp.seq_off = x->seq_off; sp.total = x->nrows;
    DLLM_TRY(select_launch(sp, st));
    x->cur_rows_cap = BN;
    x->cur_rows_per_seq = x->N;
  } else {   // PARTIAL: the response rows enter layer 0
    DLLM_TRY(range_rows_launch(x->B, x->N, x->resp_start, x->n_resp, x->rows, x->seq_off, x->nrows, st));
    x->cur_rows_cap = x->B * x->n_resp;
    x->cur_rows_per_seq = x->n_resp;
  }
  x->cur_rows = x->rows;
  x->cur_n = x->nrows;
  x->cur_seq_off = x->seq_off;
  x->rows_first = x->cur_rows_cap;
  DLLM_TRY(embed_rows_launch(static_cast<const __nv_bfloat16*>(x->w.embed), x->V, x->tokens, x->rows, x->nrows,
                             x->cur_rows_cap, x->d, x->h, st));
  x->began = true;
  x->es_layer = c.skip_layer;
  if (kind_out) *kind_out = kind;
  return DLLM_OK;
}

int dllm_layer_forward(dllm_handle* x, int32_t layer, void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (!x->began) DLLM_FAIL(DLLM_ERR_STATE, "layer_forward before begin_step");
  if (layer < 0 || layer >= x->L) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "layer out of range");
  DLLM_TRY(per_layer_order(x, layer, layer + 1));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto& c = x->c;
  const int64_t BNd = static_cast<int64_t>(x->B) * x->N * x->d;
  if (c.policy == DLLM_POLICY_DLLM_CACHE) {
    float* out_l = x->hcache + layer * BNd;
    if (x->kind == DLLM_STEP_FULL) {
      DLLM_TRY(run_layer(layer_ctx(x, layer), x->h, x->cur_rows, x->cur_n, x->cur_seq_off, x->cur_rows_cap,
                         x->cur_rows_per_seq, st));
      DLLM_CUDA_TRY(cudaMemcpyAsync(out_l, x->h, BNd * sizeof(float), cudaMemcpyDeviceToDevice, st));
      return DLLM_OK;
    }
    // partial step (dLLM-Cache explainer sec. 3): score the response rows by the cosine of their new
    // value vectors to the cached ones, recompute only the selected rows, keep the rest cached
    const float* in_l = layer == 0 ? x->h : x->hcache + (layer - 1) * BNd;
    const LayerCtx L = layer_ctx(x, layer);
    const int cap = x->B * x->n_resp;
    DLLM_TRY(rmsnorm_rows_launch(in_l, x->rows, x->nrows, cap, x->d, L.g_attn, c.rms_eps, x->z, x->d, st));
    GemmArgs v;
    v.W = L.Wqkv + static_cast<size_t>(x->qd + x->kvd) * x->d; v.w_rows_total = x->kvd; v.X = x->z;
    v.rows_cap = cap; v.rows_dev = x->nrows; v.K = x->d; v.n_tiles_w = x->kvd / 128;
    v.epi.kind = EPI_STORE_F32; v.epi.out = x->vnew; v.epi.ldo = x->kvd;
    DLLM_TRY(timed_gemm(&x->prof, v, x->gs, st, 4.0 * x->kvd));
    DLLM_TRY(score_cos_launch(x->vnew, x->kvd, L.vc, x->rows, x->nrows, cap, x->N, c.n_kv_heads, x->hd, x->scores, st));
    SelectParams sp;
    sp.scores = x->forced_sims ? x->forced_sims + static_cast<int64_t>(layer) * x->B * x->n_resp : x->scores;
    sp.B = x->B; sp.n = x->n_resp; sp.mode = c.forced_rho ? SEL_FORCED_ASC : SEL_BELOW_CAP_ASC;
    sp.k = x->resp_cap; sp.tau = c.sim_tau; sp.cand_start = x->resp_start; sp.seq_n = x->N;
    sp.act_pos = x->act_idx; sp.k_max = std::max(1, x->resp_cap); sp.count = x->act_count;
    sp.row_map = x->rows2; sp.seq_off = x->seq_off2; sp.total = x->nrows2;
    DLLM_TRY(select_launch(sp, st));
    const int cap2 = x->B * std::max(1, x->resp_cap);
    DLLM_TRY(copy_rows_launch(in_l, out_l, x->rows2, x->nrows2, cap2, x->d, st));
    return run_layer(L, out_l, x->rows2, x->nrows2, x->seq_off2, cap2, std::max(1, x->resp_cap), st);
  }
  return run_layer(layer_ctx(x, layer), x->h, x->cur_rows, x->cur_n, x->cur_seq_off, x->cur_rows_cap,
                   x->cur_rows_per_seq, st);
}

int dllm_layers_forward(dllm_handle* x, int32_t l0, int32_t l1, void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (!x->began) DLLM_FAIL(DLLM_ERR_STATE, "layers_forward before begin_step");
  if (l0 < 0 || l1 > x->L || l0 > l1) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "layer range out of bounds");
  if (l0 == l1) return DLLM_OK;
  DLLM_TRY(per_layer_order(x, l0, l1));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (x->c.policy != DLLM_POLICY_DLLM_CACHE) {   // dLLM-Cache picks its rows per layer
    const LayerCtx L0 = layer_ctx(x, l0);
    if (fused_applies(L0, x->cur_rows_cap)) {
      const int rc = run_fused_layers(L0, l1 - l0, x->h, x->cur_rows, x->cur_n, x->cur_seq_off, x->cur_rows_cap,
                                      x->cur_rows_per_seq, st);
      if (rc != DLLM_ERR_UNSUPPORTED) return rc;
    }
  }
  for (int l = l0; l < l1; ++l) DLLM_TRY(dllm_layer_forward(x, l, stream));
  return DLLM_OK;
}

int dllm_select_active(dllm_handle* x, const float* scores_or_null, int32_t* active_idx, int32_t* active_count,
                       void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (!x->began) DLLM_FAIL(DLLM_ERR_STATE, "select_active before begin_step");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto& c = x->c;
  if (c.policy != DLLM_POLICY_ES) return DLLM_OK;
  if (c.es_per_layer) return select_layer(x, scores_or_null, active_idx, active_count, st);
  const int mask = c.mask_id;
  if (x->kind == DLLM_STEP_FULL) {
    // refresh: snapshot the candidates' hidden state at the skip layer
    DLLM_TRY(range_rows_launch(x->B, x->N, cand_first(x), x->n_cand, x->rows2, x->seq_off2, x->nrows2, st));
    DLLM_TRY(snapshot_rows_launch(x->h, x->h_prev, x->tokens, x->masked_prev, mask, x->rows2, x->B * x->n_cand, x->d, st));
    x->es_layer = x->L;
    return DLLM_OK;
  }
  if (x->kind != DLLM_STEP_SKIP) DLLM_FAIL(DLLM_ERR_STATE, "select_active outside an ES step");
  // Eq. 1 (always evaluated: it also rolls h_prev and masked_prev forward)
  DLLM_TRY(score_es_launch(x->h, x->h_prev, x->conf, x->masked_prev, x->tokens, mask, x->rows, x->B * x->n_cand, x->d,
                           c.alpha, 1, nullptr, x->scores, st));
  SelectParams sp;
  sp.scores = scores_or_null ? scores_or_null : x->scores;
  sp.B = x->B; sp.n = x->n_cand; sp.mode = SEL_TOPK_DESC; sp.k = x->k_keep; sp.cand_start = cand_first(x);
  sp.seq_n = x->N; sp.act_pos = active_idx ? active_idx : x->act_idx; sp.k_max = x->k_keep;
  sp.count = active_count ? active_count : x->act_count; sp.row_map = x->rows2; sp.seq_off = x->seq_off2;
  sp.total = x->nrows2;
  DLLM_TRY(select_launch(sp, st));
  x->cur_rows = x->rows2;
  x->cur_n = x->nrows2;
  x->cur_seq_off = x->seq_off2;
  x->cur_rows_cap = x->B * x->k_keep;
  x->cur_rows_per_seq = x->k_keep;
  x->es_layer = x->L;
  return DLLM_OK;
}

int dllm_select_layers_forward(dllm_handle* x, const float* scores_or_null, void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (!x->began) DLLM_FAIL(DLLM_ERR_STATE, "select_layers_forward before begin_step");
  if (x->c.policy != DLLM_POLICY_ES) DLLM_FAIL(DLLM_ERR_STATE, "select_layers_forward needs the ES policy");
  if (x->es_layer != x->c.skip_layer) DLLM_FAIL(DLLM_ERR_STATE, "select_layers_forward starts at skip_layer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int ls = x->c.skip_layer;
  if (x->kind == DLLM_STEP_SKIP && ls < x->L) {
    const int rc = fused_es_run(x, scores_or_null, st);
    if (rc != DLLM_ERR_UNSUPPORTED) return rc;
  }
  if (!x->c.es_per_layer) {
    DLLM_TRY(dllm_select_active(x, scores_or_null, nullptr, nullptr, stream));
    return dllm_layers_forward(x, ls, x->L, stream);
  }
  const int64_t per = static_cast<int64_t>(x->B) * x->n_cand;
  for (int l = ls; l < x->L; ++l) {
    DLLM_TRY(select_layer(x, scores_or_null ? scores_or_null + (l - ls) * per : nullptr, nullptr, nullptr, st));
    DLLM_TRY(dllm_layers_forward(x, l, l + 1, stream));
  }
  return DLLM_OK;
}

int dllm_unmask(dllm_handle* x, int32_t* pos_out, int32_t* tok_out, int32_t* n_out, void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (!x->began) DLLM_FAIL(DLLM_ERR_STATE, "unmask before begin_step");
  if (es_per_layer(x) && x->es_layer != x->L)
    DLLM_FAIL(DLLM_ERR_STATE, "per-layer selection: select_active before every layer from skip_layer on");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto& c = x->c;
  const int bs = blk_start(x);
  const uint8_t* rmask = nullptr;
  if (c.unmask == DLLM_UNMASK_DUS)
    rmask = x->round_masks + static_cast<size_t>(std::min(x->step_in_block, x->n_rounds - 1)) * c.block_len;
  const float* hsrc = (c.policy == DLLM_POLICY_DLLM_CACHE) ? x->hcache + static_cast<int64_t>(x->L - 1) * x->B * x->N * x->d
                                                          : x->h;
  const int lm_cap = std::min(lm_cap_of(x), x->cur_rows_cap);
  const bool surelock = c.policy == DLLM_POLICY_SURELOCK;
  // SureLock needs the distribution of every lock-eligible row (with lock_masked: every row)
  const bool all_rows = surelock && c.lock_masked;
  DLLM_TRY(lm_rows_launch(x->cur_rows, x->cur_n, x->cur_rows_cap, x->tokens, c.mask_id, x->N, all_rows ? 0 : bs,
                          all_rows ? x->N : bs + c.block_len, all_rows ? nullptr : rmask, surelock ? 1 : 0,
                          x->lm_rows, x->n_lm, st));
  DLLM_TRY(rmsnorm_rows_launch(hsrc, x->lm_rows, x->n_lm, lm_cap, x->d, x->w.g_final, c.rms_eps, x->z, x->d, st));
  GemmArgs g;
  g.W = x->w.lm_head; g.w_rows_total = x->V; g.X = x->z; g.rows_cap = lm_cap; g.rows_dev = x->n_lm; g.K = x->d;
  g.n_tiles_w = x->V / 128;
  if (surelock) {
    // SureLock: every recomputed unmasked row needs its full distribution (stored, position-indexed,
    // in the buffer of this step's parity) to compare with the previous step's
    const int64_t BN = static_cast<int64_t>(x->B) * x->N;
    __nv_bfloat16* zcur = x->zstore + (x->n_steps & 1) * BN * x->V;
    __nv_bfloat16* zprev = x->zstore + ((x->n_steps + 1) & 1) * BN * x->V;
    float* lcur = x->lse_store + (x->n_steps & 1) * BN;
    float* lprev = x->lse_store + ((x->n_steps + 1) & 1) * BN;
    g.epi.kind = EPI_STORE_BF16; g.epi.out = zcur; g.epi.ldo = x->V; g.epi.row_map = x->lm_rows;
    DLLM_TRY(timed_gemm(&x->prof, g, x->gs, st, 2.0 * x->V));
    KlStep k;
    k.z_cur = zcur; k.z_prev = zprev; k.lse_prev = lprev; k.lse_cur = lcur; k.stamp = x->has_prev;
    k.step = x->n_steps; k.rows = x->lm_rows; k.count = x->n_lm; k.rows_cap = lm_cap; k.V = x->V;
    k.mask_id = c.mask_id; k.tokens = x->tokens; k.lock = x->lock; k.pattern = x->lock_pattern;
    k.lock_masked = c.lock_masked;
    k.kl_eps = c.kl_eps; k.conf_tau = c.conf_tau; k.conf = x->conf; k.amax = x->amax; k.kl_out = x->kl;
    DLLM_TRY(kl_step_launch(k, st));
  } else {
    g.epi.kind = EPI_LMHEAD; g.epi.lm_part = x->lm_part; g.epi.n_vtiles = x->V / 128; g.epi.mask_id = c.mask_id;
    DLLM_TRY(timed_gemm(&x->prof, g, x->gs, st, 16.0 * (x->V / 128)));
    DLLM_TRY(lmhead_combine_launch(x->lm_part, x->V / 128, lm_cap, x->n_lm, x->lm_rows, x->conf, x->amax, x->lse, st));
  }
  const int max_out = c.unmask == DLLM_UNMASK_DUS ? c.block_len : c.tokens_per_step;
  const bool cb = c.unmask == DLLM_UNMASK_CB_DUS;
  DLLM_TRY(unmask_launch(x->tokens, x->conf, x->amax, x->B, x->N, bs, c.block_len, c.mask_id, c.tokens_per_step, rmask,
                         cb ? 1 : 0, c.cb_tau, pos_out, tok_out, n_out, max_out, cb ? x->blk_remain : nullptr, st));
  // schedule: a confidence-bounded step unmasks a data-dependent number of positions, so the host
  // reads how many are left in the block (B ints, the one synchronisation of such a step)
  bool block_done = false;
  if (cb) {
    std::vector<int> left(x->B);
    DLLM_CUDA_TRY(cudaMemcpyAsync(left.data(), x->blk_remain, x->B * sizeof(int), cudaMemcpyDeviceToHost, st));
    DLLM_CUDA_TRY(cudaStreamSynchronize(st));
    block_done = true;
    for (int v : left) block_done = block_done && v == 0;
  }
  x->n_steps += 1;
  x->step_in_block += 1;
  if (block_done || x->step_in_block >= x->steps_per_block) {
    x->block += 1;
    x->step_in_block = 0;
  }
  x->began = false;
  return DLLM_OK;
}

int dllm_step(dllm_handle* x, dllm_step_info* info, void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  const int step = x->n_steps, block = x->block, sib = x->step_in_block;
  int32_t kind = 0;
  DLLM_TRY(dllm_begin_step(x, &kind, stream));
  const auto& c = x->c;
  const int ls = c.policy == DLLM_POLICY_ES ? c.skip_layer : x->L;
  DLLM_TRY(dllm_layers_forward(x, 0, ls, stream));
  if (c.policy == DLLM_POLICY_ES) DLLM_TRY(dllm_select_layers_forward(x, nullptr, stream));
  else DLLM_TRY(dllm_layers_forward(x, ls, x->L, stream));
  DLLM_TRY(dllm_unmask(x, nullptr, nullptr, nullptr, stream));
  if (info) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DLLM_CUDA_TRY(cudaStreamSynchronize(st));
    int nl = 0, nlm = 0;
    DLLM_CUDA_TRY(cudaMemcpy(&nl, x->cur_n, sizeof(int), cudaMemcpyDeviceToHost));
    DLLM_CUDA_TRY(cudaMemcpy(&nlm, x->n_lm, sizeof(int), cudaMemcpyDeviceToHost));
    info->kind = kind;
    info->step = step;
    info->block = block;
    info->step_in_block = sib;
    info->rows_first = x->rows_first;
    info->rows_last = nl;
    info->lm_rows = nlm;
    info->n_locked = 0;
    info->done = dllm_done(x);
  }
  return DLLM_OK;
}

int dllm_get_buffer(dllm_handle* x, int32_t which, void** ptr, size_t* bytes) {
  if (!x || !ptr) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null argument");
  const size_t BN = static_cast<size_t>(x->B) * x->N;
  const size_t kv = static_cast<size_t>(x->L) * x->B * x->c.n_kv_heads * x->N * x->hd;
  void* p = nullptr;
  size_t b = 0;
  switch (which) {
    case DLLM_BUF_KCACHE: p = x->kcache; b = kv * 2; break;
    case DLLM_BUF_VCACHE: p = x->vcache; b = kv * 2; break;
    case DLLM_BUF_HIDDEN: p = x->h; b = BN * x->d * 4; break;
    case DLLM_BUF_HPREV: p = x->h_prev; b = x->h_prev ? BN * x->d * 4 : 0; break;
    case DLLM_BUF_CONF: p = x->conf; b = BN * 4; break;
    case DLLM_BUF_ARGMAX: p = x->amax; b = BN * 4; break;
    case DLLM_BUF_ROWS: p = x->cur_rows ? x->cur_rows : x->rows; b = BN * 4; break;
    case DLLM_BUF_NROWS: p = x->cur_n ? x->cur_n : x->nrows; b = 4; break;
    case DLLM_BUF_SCORES: p = x->scores; b = BN * 4; break;
    case DLLM_BUF_LOCK: p = x->lock; b = BN; break;
    case DLLM_BUF_MASKED_PREV: p = x->masked_prev; b = BN; break;
    case DLLM_BUF_LMROWS: p = x->lm_rows; b = BN * 4; break;
    case DLLM_BUF_NLMROWS: p = x->n_lm; b = 4; break;
    case DLLM_BUF_KL: p = x->kl; b = BN * 4; break;
    case DLLM_BUF_HCACHE: p = x->hcache; b = x->hcache ? static_cast<size_t>(x->L) * BN * x->d * 4 : 0; break;
    case DLLM_BUF_LSE: p = x->lse; b = BN * 4; break;
    case DLLM_BUF_SELROWS: p = x->rows2; b = BN * 4; break;
    case DLLM_BUF_NSEL: p = x->nrows2; b = 4; break;
    case DLLM_BUF_LAYER_Z: p = x->z; b = BN * x->d * 2; break;
    case DLLM_BUF_LAYER_Q: p = x->q; b = BN * x->qd * 2; break;
    case DLLM_BUF_LAYER_ATTN: p = x->attn; b = BN * x->qd * 2; break;
    case DLLM_BUF_LAYER_ACT: p = x->act; b = BN * x->F * 2; break;
    case DLLM_BUF_ES_IN:
      p = x->es_in;
      b = x->es_in ? static_cast<size_t>(x->L - x->c.skip_layer - 1) * BN * x->d * 4 : 0;
      break;
    case DLLM_BUF_ZSTORE: p = x->zstore; b = x->zstore ? 2 * BN * static_cast<size_t>(x->V) * 2 : 0; break;
    case DLLM_BUF_LSE_STORE: p = x->lse_store; b = x->lse_store ? 2 * BN * 4 : 0; break;
    case DLLM_BUF_STAMP: p = x->has_prev; b = BN * 4; break;
    case DLLM_BUF_VNEW: p = x->vnew; b = x->vnew ? static_cast<size_t>(x->B) * x->n_resp * x->kvd * 4 : 0; break;
    case DLLM_BUF_FUSED_SYNC: p = x->fused_sync; b = kFusedSyncInts * 4; break;
    default: DLLM_FAIL(DLLM_ERR_INVALID_ARG, "unknown buffer");
  }
  *ptr = p;
  if (bytes) *bytes = b;
  return DLLM_OK;
}

void dllm_destroy(dllm_handle* x) { delete x; }

int dllm_set_lock_pattern(dllm_handle* x, const uint8_t* pattern) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (x->c.policy != DLLM_POLICY_SURELOCK) DLLM_FAIL(DLLM_ERR_STATE, "lock patterns apply to the SureLock policy");
  x->lock_pattern = pattern;
  return DLLM_OK;
}

int dllm_reset(dllm_handle* x, void* stream) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = reinterpret_cast<uint8_t*>(x->rope_cos);
  DLLM_CUDA_TRY(cudaMemsetAsync(base + x->const_bytes, 0, x->state_total - x->const_bytes, st));
  // GEMM tile and attention split counters of the workspace: every launch leaves them at
  // zero, except one that gave up a wait (DLLM_DEV_TIMEOUT)
  if (x->gs.n_counters) DLLM_CUDA_TRY(cudaMemsetAsync(x->gs.counters, 0, x->gs.n_counters * sizeof(int), st));
  if (x->n_attn_ctr) DLLM_CUDA_TRY(cudaMemsetAsync(x->attn_ctr, 0, x->n_attn_ctr * sizeof(int), st));
  x->block = 0;
  x->step_in_block = 0;
  x->n_steps = 0;
  x->began = false;
  return DLLM_OK;
}

int dllm_get_progress(const dllm_handle* x, dllm_progress* out) {
  if (!x || !out) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null argument");
  out->step = x->n_steps;
  out->block = x->block;
  out->step_in_block = x->step_in_block;
  return DLLM_OK;
}

int dllm_set_progress(dllm_handle* x, const dllm_progress* p) {
  if (!x || !p) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null argument");
  if (x->began) DLLM_FAIL(DLLM_ERR_STATE, "set_progress in the middle of a step");
  const int n_blocks = x->c.gen_len / x->c.block_len;
  if (p->step < 0 || p->block < 0 || p->block > n_blocks || p->step_in_block < 0 ||
      p->step_in_block >= x->steps_per_block || (p->block == n_blocks && p->step_in_block != 0))
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "progress outside the schedule");
  x->n_steps = p->step;
  x->block = p->block;
  x->step_in_block = p->step_in_block;
  return DLLM_OK;
}

int dllm_set_forced_similarities(dllm_handle* x, const float* sims) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  if (x->c.policy != DLLM_POLICY_DLLM_CACHE) DLLM_FAIL(DLLM_ERR_STATE, "forced similarities apply to dLLM-Cache");
  x->forced_sims = sims;
  return DLLM_OK;
}

int dllm_set_wait_limit(dllm_handle* x, uint32_t polls) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  x->spin_limit = polls;
  return DLLM_OK;
}

int dllm_profile_enable(dllm_handle* x, int32_t enable, double hbm_gbs, double tensor_tflops) {
  if (!x) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null handle");
  x->prof.on = enable > 0;
  x->prof.every = enable > 0 ? enable : 1;
  x->prof.seen[0] = x->prof.seen[1] = 0;
  x->prof.hbm_gbs = hbm_gbs;
  x->prof.tflops = tensor_tflops;
  return DLLM_OK;
}

int dllm_profile_read(dllm_handle* x, dllm_profile* out) {
  if (!x || !out) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null argument");
  std::memset(out, 0, sizeof(*out));
  for (auto& r : x->prof.recs) {
    DLLM_CUDA_TRY(cudaEventSynchronize(r.b));
    float ms = 0.f;
    DLLM_CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
    if (r.cls == 0) {
      out->gemm_launches += 1;
      out->gemm_ms += ms;
      out->gemm_bytes += r.bytes;
      out->gemm_flops += r.flops;
      if (x->prof.hbm_gbs > 0 && x->prof.tflops > 0)
        out->gemm_roofline_ms += std::max(r.bytes / (x->prof.hbm_gbs * 1e6), r.flops / (x->prof.tflops * 1e9));
    } else if (r.cls == 1) {
      out->attn_launches += 1;
      out->attn_ms += ms;
      out->attn_bytes += r.bytes;
      out->attn_flops += r.flops;
    } else {
      out->fused_launches += 1;
      out->fused_layers += r.layers;
      out->fused_ms += ms;
      out->fused_bytes += r.bytes;
      out->fused_flops += r.flops;
    }
    x->prof.pool.push_back(r.a);
    x->prof.pool.push_back(r.b);
  }
  x->prof.recs.clear();
  return DLLM_OK;
}

int64_t dllm_kernel_launches(void) { return dllm::g_kernel_launches.load(); }

int dllm_op_layer_workspace(const dllm_config* cfg, int32_t rows_cap, int32_t rows_per_seq_cap, size_t* bytes) {
  DLLM_TRY(validate(cfg));
  if (!cfg || !bytes || rows_cap <= 0) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "bad layer workspace args");
  const int d = cfg->d_model, qd = cfg->n_heads * cfg->head_dim, kvd = cfg->n_kv_heads * cfg->head_dim;
  const int qkvd = qd + 2 * kvd, F = cfg->ffn_dim;
  Carver w(nullptr);
  int ctr = std::max({gemm_counters_needed(rows_cap, qkvd / 128), gemm_counters_needed(rows_cap, d / 128),
                      gemm_counters_needed(rows_cap, F / 64)});
  w.take<int>(ctr);
  const int N0 = cfg->prompt_len + cfg->gen_len;
  w.take<int>(attn_counters_needed(cfg->batch, cfg->n_kv_heads, cfg->n_heads / cfg->n_kv_heads, rows_per_seq_cap));
  (void)N0;
  w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * d);
  w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * qd);
  w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * qd);
  w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * F);
  w.take<float>(static_cast<size_t>(rows_cap) * qkvd);
  size_t pf = std::max({gemm_partial_floats(rows_cap, qkvd / 128, d), gemm_partial_floats(rows_cap, d / 128, qd),
                        gemm_partial_floats(rows_cap, F / 64, d), gemm_partial_floats(rows_cap, d / 128, F)});
  w.take<float>(pf);
  const int B = cfg->batch, N = cfg->prompt_len + cfg->gen_len;
  const int sp = attn_pick_splits(B, cfg->n_kv_heads, cfg->n_heads / cfg->n_kv_heads, rows_per_seq_cap, N, cfg->head_dim);
  const size_t af = sp > 1 ? attn_partial_floats(rows_cap, cfg->n_heads, cfg->head_dim, sp) : 0;
  w.take<float>(af);
  w.take<float2>(af / cfg->head_dim);
  carve_fused_op(w, cfg, rows_cap, nullptr);
  *bytes = (w.off + 255) & ~size_t(255);
  return DLLM_OK;
}

int dllm_op_layer(const dllm_config* cfg, const void* w_qkv, const void* w_o, const void* w_gu, const void* w_down,
                  const float* g_attn, const float* g_ffn, void* kcache, void* vcache, const float* rope_cos,
                  const float* rope_sin, float* h, const int32_t* rows, const int32_t* count, const int32_t* seq_off,
                  int32_t rows_cap, int32_t rows_per_seq_cap, void* workspace, size_t workspace_bytes, void* stream) {
  DLLM_TRY(validate(cfg));
  if (!w_qkv || !w_o || !w_gu || !w_down || !g_attn || !g_ffn || !kcache || !vcache || !rope_cos || !rope_sin || !h ||
      !rows || !seq_off || !workspace)
    DLLM_FAIL(DLLM_ERR_INVALID_ARG, "null argument");
  {
    // 16-byte vector and TMA access to the weights, gains, caches, tables and h
    const void* ap[11] = {w_qkv, w_o, w_gu, w_down, g_attn, g_ffn, kcache, vcache, rope_cos, rope_sin, h};
    for (const void* p : ap)
      if (reinterpret_cast<uintptr_t>(p) & 15) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "layer operands must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(workspace) & 255) DLLM_FAIL(DLLM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  size_t need = 0;
  DLLM_TRY(dllm_op_layer_workspace(cfg, rows_cap, rows_per_seq_cap, &need));
  if (workspace_bytes < need) DLLM_FAIL(DLLM_ERR_SHAPE, "workspace too small for the layer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LayerCtx L;
  L.B = cfg->batch; L.N = cfg->prompt_len + cfg->gen_len; L.d = cfg->d_model; L.hd = cfg->head_dim;
  L.Hq = cfg->n_heads; L.Hkv = cfg->n_kv_heads; L.qd = L.Hq * L.hd; L.kvd = L.Hkv * L.hd; L.qkvd = L.qd + 2 * L.kvd;
  L.F = cfg->ffn_dim; L.eps = cfg->rms_eps;
  L.Wqkv = static_cast<const __nv_bfloat16*>(w_qkv); L.Wo = static_cast<const __nv_bfloat16*>(w_o);
  L.Wgu = static_cast<const __nv_bfloat16*>(w_gu); L.Wdn = static_cast<const __nv_bfloat16*>(w_down);
  L.g_attn = g_attn; L.g_ffn = g_ffn;
  L.kc = static_cast<__nv_bfloat16*>(kcache); L.vc = static_cast<__nv_bfloat16*>(vcache);
  L.rope_cos = rope_cos; L.rope_sin = rope_sin;
  Carver w(workspace);
  int ctr = std::max({gemm_counters_needed(rows_cap, L.qkvd / 128), gemm_counters_needed(rows_cap, L.d / 128),
                      gemm_counters_needed(rows_cap, L.F / 64)});
  L.gs.counters = w.take<int>(ctr);
  L.gs.n_counters = ctr;
  L.n_attn_ctr = attn_counters_needed(L.B, L.Hkv, L.Hq / L.Hkv, rows_per_seq_cap);
  L.attn_ctr = w.take<int>(L.n_attn_ctr);
  L.z = w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * L.d);
  L.q = w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * L.qd);
  L.attn = w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * L.qd);
  L.act = w.take<__nv_bfloat16>(static_cast<size_t>(rows_cap) * L.F);
  L.yqkv = w.take<float>(static_cast<size_t>(rows_cap) * L.qkvd);
  size_t pf = std::max({gemm_partial_floats(rows_cap, L.qkvd / 128, L.d), gemm_partial_floats(rows_cap, L.d / 128, L.qd),
                        gemm_partial_floats(rows_cap, L.F / 64, L.d), gemm_partial_floats(rows_cap, L.d / 128, L.F)});
  L.gs.partial = w.take<float>(pf);
  L.gs.partial_floats = pf;
  const int sp = attn_pick_splits(L.B, L.Hkv, L.Hq / L.Hkv, rows_per_seq_cap, L.N, L.hd);
  L.attn_floats = sp > 1 ? attn_partial_floats(rows_cap, L.Hq, L.hd, sp) : 0;
  L.attn_opart = w.take<float>(L.attn_floats);
  L.attn_ml = w.take<float2>(L.attn_floats / L.hd);
  carve_fused_op(w, cfg, rows_cap, &L);
  return run_layer(L, h, rows, count, seq_off, rows_cap, rows_per_seq_cap, st);
}

}  // extern "C"
