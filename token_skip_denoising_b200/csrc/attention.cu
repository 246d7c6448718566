// Active-query attention over the full cached K/V (bidirectional, no mask).
//
// SureLock summary sec. 2.1 items 3-4: the recomputed (active) rows attend to
// every position through the cached K/V, so the cost is O(M_t * N * d)
// instead of O(N^2 d).  ES-dLLM summary sec. 2.1 item 2: skipped rows reuse
// their cached K/V.  The new K/V rows of the active set were written into the
// cache by the QKV epilogue before this kernel runs.
//
// Flash-style: a CTA owns up to 64 (query row, head) units of one KV head of
// one sequence and streams a range of 64-key blocks of that head's K and V
// through double-buffered, XOR-swizzled shared memory (cp.async), with an
// online softmax in fp32 (mma.sync bf16 tiles for Q K^T and P V).  When the
// query tiles alone cannot fill the GPU (few active rows), the key range is
// split across CTAs and a combine kernel merges the partial (O, max, sum).
#include <algorithm>

#include "attn_dev.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace dllm {
namespace {

using namespace attn;

struct CtaBar {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

template <int HD>
__global__ void __launch_bounds__(128) attn_kernel(AttnParams p) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(128) uint8_t smem[];
  const int b = blockIdx.y / p.Hkv;
  const int kvh = blockIdx.y % p.Hkv;
  attn_item<HD>(p, blockIdx.x, b, kvh, blockIdx.z, smem, threadIdx.x, CtaBar{});
}

// One warp per (row, head): merge the split partials.
template <int HD>
__global__ void attn_combine_kernel(AttnParams p) {
  pdl_trigger();
  pdl_wait();
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int total = p.seq_off[p.B];
  const int row = wid / p.Hq, h = wid % p.Hq;
  if (row >= total) return;
  attn_merge<HD>(p, row, h, lane);
}

// Merge of the split partials: one warp per (row, head).
int combine_launch(const AttnParams& p, int rows_cap, int hd, cudaStream_t st) {
  const int warps = rows_cap * p.Hq;
  const int blocks = (warps * 32 + 255) / 256;
  return hd == 128 ? launch_pdl(attn_combine_kernel<128>, dim3(blocks), dim3(256), 0, st, p)
                   : launch_pdl(attn_combine_kernel<64>, dim3(blocks), dim3(256), 0, st, p);
}

}  // namespace

int attn_tc_run(const attn::AttnParams& p, int rows_per_seq_cap, cudaStream_t st);

size_t attn_partial_floats(int rows_cap, int Hq, int hd, int splits) {
  return static_cast<size_t>(splits) * rows_cap * Hq * hd;
}

int attn_pick_splits(int B, int Hkv, int G, int rows_per_seq, int N, int hd) {
  if (attn_use_tc(hd, G, rows_per_seq)) return attn_tc_pick_splits(B, Hkv, G, rows_per_seq, N);
  const int qtiles = (rows_per_seq * G + kUnitsPerCta - 1) / kUnitsPerCta;
  const int ctas = qtiles * B * Hkv;
  const int n_blocks = (N + kKeysPerBlock - 1) / kKeysPerBlock;
  const int sms = num_sms();
  if (ctas >= sms) return 1;
  int s = (2 * sms + ctas - 1) / ctas;
  s = std::min(s, n_blocks);
  return std::max(1, s);
}

int attn_counters_needed(int B, int Hkv, int G, int rows_per_seq) {
  (void)B; (void)Hkv; (void)G; (void)rows_per_seq;
  return 0;
}

int attn_launch(const __nv_bfloat16* q, const __nv_bfloat16* kc, const __nv_bfloat16* vc, __nv_bfloat16* out,
                const int* seq_off, int B, int rows_cap, int rows_per_seq_cap, int N, int Hq, int Hkv, int hd,
                int splits, float* opart, float2* ml, size_t partial_floats, int* counters, int n_counters,
                cudaStream_t st) {
  (void)counters;
  (void)n_counters;
  if (B <= 0 || N <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return DLLM_ERR_SHAPE;
  if (hd != 64 && hd != 128) return DLLM_ERR_UNSUPPORTED;
  if (rows_cap <= 0 || rows_per_seq_cap <= 0) return DLLM_OK;
  const int G = Hq / Hkv;
  const bool tc = attn_use_tc(hd, G, rows_per_seq_cap);
  // key blocks of the chosen path: 128 keys on the tensor cores, 64 on the CUDA cores
  const int kblk = tc ? 128 : kKeysPerBlock;
  const int n_blocks = (N + kblk - 1) / kblk;
  if (splits <= 0) splits = attn_pick_splits(B, Hkv, G, rows_per_seq_cap, N, hd);
  splits = std::min(splits, n_blocks);
  if (splits > 1 && (!opart || !ml || partial_floats < attn_partial_floats(rows_cap, Hq, hd, splits))) splits = 1;
  const int bps = (n_blocks + splits - 1) / splits;
  splits = (n_blocks + bps - 1) / bps;
  AttnParams p;
  p.q = q; p.kc = kc; p.vc = vc; p.out = out; p.seq_off = seq_off;
  p.B = B; p.N = N; p.Hq = Hq; p.Hkv = Hkv; p.rows_cap = rows_cap;
  p.splits = splits; p.blocks_per_split = bps;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(hd));
  p.opart = opart; p.ml = ml;
  if (tc) {
    const int rc = attn_tc_run(p, rows_per_seq_cap, st);
    if (rc) return rc;
    return splits > 1 ? combine_launch(p, rows_cap, hd, st) : DLLM_OK;
  }
  const int qtiles = (rows_per_seq_cap * G + kUnitsPerCta - 1) / kUnitsPerCta;
  dim3 grid(qtiles, B * Hkv, splits);
  const size_t smem = 4 * kKeysPerBlock * hd * 2;
  {
    const int rc = hd == 128 ? ensure_smem_attr(reinterpret_cast<const void*>(attn_kernel<128>),
                                                static_cast<int>(4 * kKeysPerBlock * 128 * 2))
                             : ensure_smem_attr(reinterpret_cast<const void*>(attn_kernel<64>),
                                                static_cast<int>(4 * kKeysPerBlock * 64 * 2));
    if (rc) return rc;
  }
  if (hd == 128) {
    const int rc = launch_pdl(attn_kernel<128>, grid, dim3(128), smem, st, p);
    if (rc) return rc;
  } else {
    const int rc = launch_pdl(attn_kernel<64>, grid, dim3(128), smem, st, p);
    if (rc) return rc;
  }
  return splits > 1 ? combine_launch(p, rows_cap, hd, st) : DLLM_OK;
}

}  // namespace dllm
