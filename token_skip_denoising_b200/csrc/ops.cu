// C ABI of single kernels (dllm_op_*): argument checks, workspace carving and
// one launch each.  Used by the parity tests and the single-layer benchmark.
#include <algorithm>
#include <cstdint>
#include <initializer_list>
#include <vector>

#include "common.cuh"
#include "rowops.cuh"

using namespace dllm;

#define OP_FAIL(code, msg)                         \
  do {                                             \
    dllm::set_last_error((msg), __FILE__, __LINE__); \
    return (code);                                 \
  } while (0)

namespace {

struct OpCarver {
  uint8_t* base;
  size_t cap, off = 0;
  bool ok = true;
  OpCarver(void* b, size_t c) : base(static_cast<uint8_t*>(b)), cap(c) {}
  template <class T>
  T* take(size_t n) {
    off = (off + 255) & ~size_t(255);
    if (!base || off + n * sizeof(T) > cap) { ok = false; return nullptr; }
    T* p = reinterpret_cast<T*>(base + off);
    off += n * sizeof(T);
    return p;
  }
};

// Scratch of one GEMM launched through an op: the tile counters live at the start of the
// workspace (the caller zeroes the workspace once; every GEMM leaves its counters at zero),
// the partial tiles of split work follow.
// Whether every pointer is a multiple of `a` bytes: the kernels move 16-byte (and 8-byte) vectors.
bool aligned_to(size_t a, std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs)
    if (reinterpret_cast<uintptr_t>(q) % a) return false;
  return true;
}

constexpr int kOpCounters = 65536;

int gemm_scratch(OpCarver& cv, int rows_cap, int tiles, int K, GemmScratch& gs) {
  const int b = rows_cap <= 16 ? 16 : rows_cap <= 32 ? 32 : rows_cap <= 64 ? 64 : rows_cap <= 128 ? 128 : 256;
  const int nc = tiles * ((rows_cap + b - 1) / b);
  if (nc > kOpCounters) OP_FAIL(DLLM_ERR_SHAPE, "too many output tiles for the op workspace");
  gs.counters = cv.take<int>(kOpCounters);
  const size_t pf = gemm_partial_floats(rows_cap, tiles, K);
  gs.partial = cv.take<float>(pf);
  if (!cv.ok) OP_FAIL(DLLM_ERR_SHAPE, "workspace too small for the GEMM scratch");
  gs.partial_floats = pf;
  gs.n_counters = nc;
  return DLLM_OK;
}

}  // namespace

extern "C" {

int dllm_op_rope_table(float* cos_t, float* sin_t, int32_t N, int32_t head_dim, double theta, void* stream) {
  if (!cos_t || !sin_t || N <= 0 || head_dim <= 0 || head_dim % 2) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad rope args");
  return rope_table_launch(cos_t, sin_t, N, head_dim, theta, static_cast<cudaStream_t>(stream));
}

int dllm_op_embed_rows(const void* embed, int32_t vocab, const int32_t* tokens, const int32_t* rows,
                       const int32_t* count, int32_t rows_cap, int32_t d, float* h, void* stream) {
  if (!embed || !tokens || !rows || !h || rows_cap < 0 || d <= 0 || vocab <= 0)
    OP_FAIL(DLLM_ERR_INVALID_ARG, "bad embed args");
  if (!aligned_to(16, {embed, h})) OP_FAIL(DLLM_ERR_INVALID_ARG, "embedding table and h must be 16-byte aligned");
  return embed_rows_launch(static_cast<const __nv_bfloat16*>(embed), vocab, tokens, rows, count, rows_cap, d, h,
                           static_cast<cudaStream_t>(stream));
}

int dllm_op_rmsnorm_rows(const float* h, const int32_t* rows, const int32_t* count, int32_t rows_cap, int32_t d,
                         const float* g, float eps, void* z, void* stream) {
  if (!h || !g || !z || rows_cap < 0 || d <= 0) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad rmsnorm args");
  if (!aligned_to(16, {h, g}) || !aligned_to(8, {z}))
    OP_FAIL(DLLM_ERR_INVALID_ARG, "h and g must be 16-byte aligned, z 8-byte aligned");
  return rmsnorm_rows_launch(h, rows, count, rows_cap, d, g, eps, static_cast<__nv_bfloat16*>(z), d,
                             static_cast<cudaStream_t>(stream));
}

int dllm_op_gemm(int32_t kind, const void* W, int32_t n_out, const void* X, int32_t rows_cap, const int32_t* count,
                 int32_t K, void* out, const int32_t* rows_map, int32_t splits, int32_t bn, void* workspace,
                 size_t workspace_bytes, void* stream) {
  if (!W || !X || !out || rows_cap <= 0 || K <= 0 || n_out <= 0) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad gemm args");
  if (n_out % 128 || K % 64) OP_FAIL(DLLM_ERR_SHAPE, "n_out must be a multiple of 128 and K of 64");
  if (kind != EPI_STORE_F32 && kind != EPI_STORE_BF16 && kind != EPI_RESID_ADD)
    OP_FAIL(DLLM_ERR_INVALID_ARG, "kind must be 0, 1 or 3");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!aligned_to(256, {workspace})) OP_FAIL(DLLM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  OpCarver cv(workspace, workspace_bytes);
  GemmScratch gs;
  const int rc = gemm_scratch(cv, rows_cap, n_out / 128, K, gs);
  if (rc) return rc;
  GemmArgs a;
  a.W = W; a.w_rows_total = n_out; a.X = X; a.rows_cap = rows_cap; a.rows_dev = count; a.K = K;
  a.n_tiles_w = n_out / 128;
  a.epi.kind = kind;
  if (kind == EPI_RESID_ADD) {
    a.epi.h = static_cast<float*>(out); a.epi.ldh = n_out; a.epi.row_map = rows_map;
  } else {
    a.epi.out = out; a.epi.ldo = n_out;
  }
  return gemm_launch(a, gs, st, splits, bn);
}

int dllm_op_qkv_rope(const void* W, const void* X, int32_t rows_cap, const int32_t* count, int32_t d,
                     int32_t n_heads, int32_t n_kv_heads, int32_t head_dim, int32_t N, const int32_t* rows_map,
                     const float* rope_cos, const float* rope_sin, void* q_out, void* kcache, void* vcache,
                     int32_t splits, void* workspace, size_t workspace_bytes, void* stream) {
  if (!W || !X || !rows_map || !rope_cos || !rope_sin || !q_out || !kcache || !vcache || rows_cap <= 0)
    OP_FAIL(DLLM_ERR_INVALID_ARG, "bad qkv args");
  if (head_dim != 64 && head_dim != 128) OP_FAIL(DLLM_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  const int qd = n_heads * head_dim, kvd = n_kv_heads * head_dim;
  if (qd % 128 || kvd % 128 || d % 64) OP_FAIL(DLLM_ERR_SHAPE, "q / kv widths must be multiples of 128");
  if (!aligned_to(16, {rope_cos, rope_sin}) || !aligned_to(8, {q_out, kcache, vcache}))
    OP_FAIL(DLLM_ERR_INVALID_ARG, "cos/sin tables must be 16-byte aligned, q and the caches 8-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int qkvd = qd + 2 * kvd;
  if (!aligned_to(256, {workspace})) OP_FAIL(DLLM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  OpCarver cv(workspace, workspace_bytes);
  GemmScratch gs;
  const int rc = gemm_scratch(cv, rows_cap, qkvd / 128, d, gs);
  if (rc) return rc;
  float* y = cv.take<float>(static_cast<size_t>(rows_cap) * qkvd);
  if (!cv.ok) OP_FAIL(DLLM_ERR_SHAPE, "workspace too small for the fp32 QKV products");
  GemmArgs g;
  g.W = W; g.w_rows_total = qkvd; g.X = X; g.rows_cap = rows_cap; g.rows_dev = count; g.K = d;
  g.n_tiles_w = qkvd / 128;
  g.epi.kind = EPI_STORE_F32; g.epi.out = y; g.epi.ldo = qkvd; g.wide_ok = true;
  const int rc2 = gemm_launch(g, gs, st, splits, 0);
  if (rc2) return rc2;
  return rope_scatter_launch(y, rows_cap, count, rows_map, qkvd, qd, kvd, head_dim, N, n_kv_heads, rope_cos,
                             rope_sin, static_cast<__nv_bfloat16*>(q_out), static_cast<__nv_bfloat16*>(kcache),
                             static_cast<__nv_bfloat16*>(vcache), st);
}

int dllm_op_gate_up(const void* W, int32_t F, const void* X, int32_t rows_cap, const int32_t* count, int32_t d,
                    void* act, int32_t splits, void* workspace, size_t workspace_bytes, void* stream) {
  if (!W || !X || !act || rows_cap <= 0 || F <= 0) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad gate_up args");
  if (F % 64 || d % 64) OP_FAIL(DLLM_ERR_SHAPE, "F and d must be multiples of 64");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!aligned_to(256, {workspace})) OP_FAIL(DLLM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  OpCarver cv(workspace, workspace_bytes);
  GemmScratch gs;
  const int rc = gemm_scratch(cv, rows_cap, F / 64, d, gs);
  if (rc) return rc;
  GemmArgs g;
  g.W = W; g.w_rows_total = 2 * F; g.X = X; g.rows_cap = rows_cap; g.rows_dev = count; g.K = d;
  g.n_tiles_w = F / 64; g.swiglu = true;
  g.epi.kind = EPI_SWIGLU; g.epi.act = static_cast<__nv_bfloat16*>(act); g.epi.ffn = F;
  return gemm_launch(g, gs, st, splits, 0);
}

int dllm_op_attention(const void* q, const void* kcache, const void* vcache, void* out, const int32_t* seq_off,
                      int32_t B, int32_t rows_cap, int32_t rows_per_seq_cap, int32_t N, int32_t n_heads,
                      int32_t n_kv_heads, int32_t head_dim, int32_t splits, void* workspace, size_t workspace_bytes,
                      void* stream) {
  if (!q || !kcache || !vcache || !out || !seq_off) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad attention args");
  if (!aligned_to(16, {q, kcache, vcache, out}))
    OP_FAIL(DLLM_ERR_INVALID_ARG, "q, the caches and out must be 16-byte aligned");
  if (n_kv_heads <= 0 || n_heads % n_kv_heads) OP_FAIL(DLLM_ERR_SHAPE, "n_heads must be a multiple of n_kv_heads");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = n_heads / n_kv_heads;
  int sp = splits > 0 ? splits : attn_pick_splits(B, n_kv_heads, G, rows_per_seq_cap, N, head_dim);
  float* opart = nullptr;
  float2* ml = nullptr;
  int* ctr = nullptr;
  int nctr = 0;
  size_t pf = 0;
  if (sp > 1) {
    if (!aligned_to(256, {workspace})) OP_FAIL(DLLM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    OpCarver cv(workspace, workspace_bytes);
    nctr = attn_counters_needed(B, n_kv_heads, G, rows_per_seq_cap);
    ctr = cv.take<int>(kOpCounters);        // the zeroed counter region at the workspace start
    if (nctr > kOpCounters) OP_FAIL(DLLM_ERR_SHAPE, "too many attention groups for the op workspace");
    pf = attn_partial_floats(rows_cap, n_heads, head_dim, sp);
    opart = cv.take<float>(pf);
    ml = cv.take<float2>(pf / head_dim);
    if (!cv.ok) OP_FAIL(DLLM_ERR_SHAPE, "workspace too small for attention partials");
  }
  return attn_launch(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(kcache),
                     static_cast<const __nv_bfloat16*>(vcache), static_cast<__nv_bfloat16*>(out), seq_off, B, rows_cap,
                     rows_per_seq_cap, N, n_heads, n_kv_heads, head_dim, sp, opart, ml, pf, ctr, nctr, st);
}

int dllm_op_lm_head(const void* W, int32_t V, const void* X, int32_t rows_cap, const int32_t* count, int32_t d,
                    int32_t mask_id, const int32_t* out_index, float* conf, int32_t* argmax, float* lse,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!W || !X || rows_cap <= 0 || V <= 0) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad lm_head args");
  if (V % 128 || d % 64) OP_FAIL(DLLM_ERR_SHAPE, "V must be a multiple of 128 and d of 64");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!aligned_to(256, {workspace})) OP_FAIL(DLLM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  OpCarver cv(workspace, workspace_bytes);
  GemmScratch gs;
  const int rc = gemm_scratch(cv, rows_cap, V / 128, d, gs);
  if (rc) return rc;
  float4* part = cv.take<float4>(static_cast<size_t>(rows_cap) * (V / 128));
  if (!cv.ok) OP_FAIL(DLLM_ERR_SHAPE, "workspace too small for LM-head partials");
  GemmArgs g;
  g.W = W; g.w_rows_total = V; g.X = X; g.rows_cap = rows_cap; g.rows_dev = count; g.K = d; g.n_tiles_w = V / 128;
  g.epi.kind = EPI_LMHEAD; g.epi.lm_part = part; g.epi.n_vtiles = V / 128; g.epi.mask_id = mask_id;
  int r = gemm_launch(g, gs, st, 0, 0);
  if (r) return r;
  return lmhead_combine_launch(part, V / 128, rows_cap, count, out_index, conf, argmax, lse, st);
}

int dllm_op_score_es(const float* h, float* h_prev, const float* conf, uint8_t* masked_prev, const int32_t* tokens,
                     int32_t mask_id, const int32_t* rows, int32_t n_rows, int32_t d, float alpha, int32_t update,
                     float* score, void* stream) {
  if (!h || !h_prev || !conf || !score || n_rows < 0 || d <= 0) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad score_es args");
  if (update && (!masked_prev || !tokens)) OP_FAIL(DLLM_ERR_INVALID_ARG, "update needs masked_prev and tokens");
  if (!aligned_to(16, {h, h_prev})) OP_FAIL(DLLM_ERR_INVALID_ARG, "h and h_prev must be 16-byte aligned");
  // without a previous-layer choice (act_prev null) the kernel only reads h
  return score_es_launch(const_cast<float*>(h), h_prev, conf, masked_prev, tokens, mask_id, rows, n_rows, d, alpha,
                         update, nullptr, score, static_cast<cudaStream_t>(stream));
}

int dllm_op_score_cos(const float* vnew, const void* vcache, const int32_t* rows, const int32_t* count,
                      int32_t rows_cap, int32_t N, int32_t n_kv_heads, int32_t head_dim, float* sim, void* stream) {
  if (!vnew || !vcache || !rows || !sim) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad score_cos args");
  return score_cos_launch(vnew, static_cast<int64_t>(n_kv_heads) * head_dim, static_cast<const __nv_bfloat16*>(vcache),
                          rows, count, rows_cap, N, n_kv_heads, head_dim, sim, static_cast<cudaStream_t>(stream));
}

int dllm_op_kl_conf(const void* logits, const void* zp_store, const float* lse_prev, const int32_t* has_prev,
                    const int32_t* rows, const int32_t* count, int32_t rows_cap, int32_t V, int32_t mask_id,
                    float* conf, int32_t* argmax, float* lse, float* kl, void* stream) {
  if (!logits || !conf || !argmax || rows_cap < 0 || V <= 0) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad kl_conf args");
  if (has_prev && (!zp_store || !lse_prev)) OP_FAIL(DLLM_ERR_INVALID_ARG, "has_prev needs the stored logits");
  return kl_conf_launch(static_cast<const __nv_bfloat16*>(logits), V, static_cast<const __nv_bfloat16*>(zp_store), V,
                        lse_prev, has_prev, rows, count, rows_cap, V, mask_id, conf, argmax, lse, kl,
                        static_cast<cudaStream_t>(stream));
}

int dllm_op_select(const float* scores, int32_t B, int32_t n, int32_t mode, int32_t k, float tau, int32_t cand_start,
                   int32_t N, const uint8_t* lock, int32_t* act_pos, int32_t k_max, int32_t* count, int32_t* rows,
                   int32_t* seq_off, void* stream) {
  if (B < 0 || n < 0 || k < 0 || mode < 0 || mode > 3) OP_FAIL(DLLM_ERR_INVALID_ARG, "bad select args");
  if (mode != SEL_ALL_ELIGIBLE && !scores) OP_FAIL(DLLM_ERR_INVALID_ARG, "scores required");
  if (mode == SEL_ALL_ELIGIBLE && !lock) OP_FAIL(DLLM_ERR_INVALID_ARG, "lock flags required");
  if (act_pos && k_max < std::min(k, n) && mode != SEL_ALL_ELIGIBLE) OP_FAIL(DLLM_ERR_SHAPE, "k_max below k");
  SelectParams p;
  p.scores = scores; p.B = B; p.n = n; p.mode = mode; p.k = k; p.tau = tau; p.cand_start = cand_start; p.seq_n = N;
  p.lock = lock; p.act_pos = act_pos; p.k_max = k_max; p.count = count; p.row_map = rows; p.seq_off = seq_off;
  return select_launch(p, static_cast<cudaStream_t>(stream));
}

int dllm_op_unmask(int32_t* tokens, const float* conf, const int32_t* argmax, int32_t B, int32_t N, int32_t blk_s,
                   int32_t blk_len, int32_t mask_id, int32_t mode, int32_t n_commit, float cb_tau,
                   const uint8_t* round_mask, int32_t* pos_out, int32_t* tok_out, int32_t* n_out, int32_t max_out,
                   int32_t* remain, void* stream) {
  if (!tokens || !conf || !argmax || B <= 0 || blk_s < 0 || blk_s + blk_len > N)
    OP_FAIL(DLLM_ERR_INVALID_ARG, "bad unmask args");
  if (mode != DLLM_UNMASK_TOPCONF && mode != DLLM_UNMASK_CB_DUS) OP_FAIL(DLLM_ERR_INVALID_ARG, "unknown unmask mode");
  if (mode == DLLM_UNMASK_CB_DUS && (round_mask || n_commit <= 0))
    OP_FAIL(DLLM_ERR_INVALID_ARG, "the confidence-bounded mode takes no round mask and n_commit >= 1");
  if (pos_out && (!tok_out || max_out <= 0)) OP_FAIL(DLLM_ERR_INVALID_ARG, "pos_out needs tok_out and max_out");
  return unmask_launch(tokens, conf, argmax, B, N, blk_s, blk_len, mask_id, n_commit, round_mask,
                       mode == DLLM_UNMASK_CB_DUS ? 1 : 0, cb_tau, pos_out, tok_out, n_out, max_out, remain,
                       static_cast<cudaStream_t>(stream));
}

}  // extern "C"
