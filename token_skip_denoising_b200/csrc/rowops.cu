// Row-wise kernels of the step: embedding gather, RMSNorm gather, the three
// row scores (ES-dLLM Eq. 1, SureLock KL, dLLM-Cache cosine), radix top-k /
// threshold selection with compaction, vocabulary-row lists and unmasking.
// All of them are HBM- or latency-bound; none is a contraction.
#include <algorithm>

#include "common.cuh"
#include "es_dev.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace dllm {
namespace {

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------------ RoPE table
__global__ void rope_table_kernel(float* cos_t, float* sin_t, int N, int half, double theta, int hd) {
  pdl_trigger();
  pdl_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * half) return;
  const int pos = idx / half, i = idx % half;
  const double inv = pow(theta, -2.0 * i / static_cast<double>(hd));
  const double ang = static_cast<double>(pos) * inv;
  double s, c;
  sincos(ang, &s, &c);
  cos_t[idx] = static_cast<float>(c);
  sin_t[idx] = static_cast<float>(s);
}

// ------------------------------------------------------------------ embedding
// h[row_map[j]] = E[tokens[row_map[j]]] (bf16 -> fp32), j < count
__global__ void embed_rows_kernel(const __nv_bfloat16* __restrict__ E, const int* __restrict__ tokens,
                                  const int* __restrict__ row_map, const int* count_dev, int rows_cap, int d, int V,
                                  float* __restrict__ h) {
  pdl_trigger();
  pdl_wait();
  const int m = count_dev ? min(*count_dev, rows_cap) : rows_cap;
  const int j = blockIdx.x;
  if (j >= m) return;
  const int flat = row_map[j];
  const int tok = tokens[flat];
  float* dst = h + static_cast<int64_t>(flat) * d;
  if (tok < 0 || tok >= V) {   // a token id outside the vocabulary is reported, never read
    if (threadIdx.x == 0) set_dev_status(DLLM_DEV_BAD_INDEX);
    for (int i = threadIdx.x; i < d; i += blockDim.x) dst[i] = 0.f;
    return;
  }
  const __nv_bfloat16* src = E + static_cast<int64_t>(tok) * d;
  for (int i = threadIdx.x * 8; i < d; i += blockDim.x * 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(src + i);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float4 a, b;
    float2 f0 = __bfloat1622float2(p2[0]), f1 = __bfloat1622float2(p2[1]);
    float2 f2 = __bfloat1622float2(p2[2]), f3 = __bfloat1622float2(p2[3]);
    a = make_float4(f0.x, f0.y, f1.x, f1.y);
    b = make_float4(f2.x, f2.y, f3.x, f3.y);
    *reinterpret_cast<float4*>(dst + i) = a;
    *reinterpret_cast<float4*>(dst + i + 4) = b;
  }
}

// ------------------------------------------------------------------ RMSNorm gather
// z[j] = bf16(h[src(j)] / sqrt(mean(h^2) + eps) * g); src(j) = row_map[j] (or j).
// One CTA of 256 threads per row.
__global__ void rmsnorm_rows_kernel(const float* __restrict__ h, const int* __restrict__ row_map,
                                    const int* count_dev, int rows_cap, int d, const float* __restrict__ g,
                                    float eps, __nv_bfloat16* __restrict__ z, int64_t ldz) {
  pdl_trigger();
  pdl_wait();
  const int m = count_dev ? min(*count_dev, rows_cap) : rows_cap;
  const int j = blockIdx.x;
  if (j >= m) return;
  const int src = row_map ? row_map[j] : j;
  const float* x = h + static_cast<int64_t>(src) * d;
  float ss = 0.f;
  for (int i = threadIdx.x * 4; i < d; i += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(x + i);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  __shared__ float red[32];
  ss = warp_sum_f(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum_f(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float r = rsqrtf(red[0] / static_cast<float>(d) + eps);
  __nv_bfloat16* out = z + static_cast<int64_t>(j) * ldz;
  for (int i = threadIdx.x * 4; i < d; i += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(x + i);
    const float4 gg = *reinterpret_cast<const float4*>(g + i);
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x * r * gg.x, v.y * r * gg.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z * r * gg.z, v.w * r * gg.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&a);
    pk.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(out + i) = pk;
  }
}

// ------------------------------------------------------------------ ES-dLLM Eq. 1
// For candidate row j (flat = rows[j]):
//   c   = masked_prev[flat] ? conf[flat] : 0
//   var = ||h - h_prev||_1 / (sqrt(d) ||h_prev||_2)   (0 when ||h_prev|| = 0)
//   score[j] = alpha c + (1 - alpha) var
// then h_prev[flat] := h[flat] and masked_prev[flat] := (tokens[flat] == mask_id)
// (tokens null: masked_prev is read but not rolled).
// Per-layer re-selection: with act_prev non-null, a row whose act_prev[flat] is 0 was
// skipped by the previous layer, so its input here is its cached output of that layer,
// h_prev[flat] itself: var = 0 and the row of h is overwritten with h_prev (the carry of
// the cached state into this layer), h_prev unchanged.
// One warp per row.
__global__ void score_es_kernel(float* __restrict__ h, float* __restrict__ h_prev,
                                const float* __restrict__ conf, uint8_t* __restrict__ masked_prev,
                                const int* __restrict__ tokens, int mask_id, const int* __restrict__ rows,
                                int n_rows, int d, float alpha, int update, const uint8_t* __restrict__ act_prev,
                                float* __restrict__ score) {
  pdl_trigger();
  pdl_wait();
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= n_rows) return;
  const int flat = rows ? rows[wid] : wid;
  const bool carried = act_prev && !act_prev[flat];
  const float c = (masked_prev && masked_prev[flat]) ? conf[flat] : 0.f;
  const float s = es_eq1_row(h + static_cast<int64_t>(flat) * d, h_prev + static_cast<int64_t>(flat) * d, d, c,
                             alpha, update, carried, lane);
  if (lane == 0) {
    score[wid] = s;
    if (update && masked_prev && tokens) masked_prev[flat] = tokens[flat] == mask_id ? 1 : 0;
  }
}

// ------------------------------------------------------------------ dLLM-Cache cosine
// s[j] = <v_new[j], v_cache(rows[j])> / (|v_new| |v_cache|); 1 if both zero, 0 if one is.
// v_cache for flat = b * N + pos is the concatenation over KV heads of cache[b, kvh, pos, :].
__global__ void score_cos_kernel(const float* __restrict__ vnew, int64_t ldv, const __nv_bfloat16* __restrict__ vc,
                                 const int* __restrict__ rows, const int* count_dev, int rows_cap, int N, int Hkv,
                                 int hd, float* __restrict__ sim) {
  pdl_trigger();
  pdl_wait();
  const int m = count_dev ? min(*count_dev, rows_cap) : rows_cap;
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= m) return;
  const int flat = rows[wid];
  const int b = flat / N, pos = flat % N;
  // one warp per row, 8 elements per lane and step: 16 bytes of the cached V row, 32 of v_new
  const int chunks = Hkv * hd / 8;
  const int per_head = hd / 8;
  const float* nv = vnew + static_cast<int64_t>(wid) * ldv;
  float dot = 0.f, na = 0.f, nb = 0.f;
#pragma unroll 4
  for (int c = lane; c < chunks; c += 32) {
    const int kvh = c / per_head, off = (c - kvh * per_head) * 8;
    const uint4 cv = __ldg(reinterpret_cast<const uint4*>(vc + ((static_cast<int64_t>(b) * Hkv + kvh) * N + pos) * hd + off));
    const float4 a0 = __ldg(reinterpret_cast<const float4*>(nv + c * 8));
    const float4 a1 = __ldg(reinterpret_cast<const float4*>(nv + c * 8 + 4));
    const __nv_bfloat162* cp = reinterpret_cast<const __nv_bfloat162*>(&cv);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 cf = __bfloat1622float2(cp[e]);
      dot += av[2 * e] * cf.x + av[2 * e + 1] * cf.y;
      na += av[2 * e] * av[2 * e] + av[2 * e + 1] * av[2 * e + 1];
      nb += cf.x * cf.x + cf.y * cf.y;
    }
  }
  dot = warp_sum_f(dot);
  na = warp_sum_f(na);
  nb = warp_sum_f(nb);
  if (lane == 0) {
    float s;
    if (na > 0.f && nb > 0.f) s = dot / (sqrtf(na) * sqrtf(nb));
    else s = (na == 0.f && nb == 0.f) ? 1.f : 0.f;
    sim[wid] = s;
  }
}

// ------------------------------------------------------------------ SureLock KL + confidence
// Statistics of one logit row z [V] (bf16), by the whole CTA in one pass of 16-byte loads:
// M = max z, S = sum exp(z - M), the argmax over v != mask_id (ties to the lower id), and with
// a previous row zp: T = sum exp(z - M) (z - zp).  The running (M, S, T) of a thread is
// rescaled by exp(M_old - M_new) whenever its maximum grows (online softmax).  Then
// lse = M + log S, p(v) = exp(z - lse), and KL(p || p_prev) = sum p (z - lse - zp + lse_p)
// = T / S - (lse - lse_p).  V % 8 == 0 and 16-byte aligned rows.
struct RowStats {
  float M, S, T, BV;
  int BI;
};
__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}
__device__ __forceinline__ RowStats row_stats(const __nv_bfloat16* __restrict__ z, const __nv_bfloat16* __restrict__ zp,
                                              int V, int mask_id, float* s_f, int* s_i) {
  float m = -INFINITY, sum = 0.f, tt = 0.f, bv = -INFINITY;
  int bi = 0x7fffffff;
  const uint4* z4 = reinterpret_cast<const uint4*>(z);
  const uint4* p4 = reinterpret_cast<const uint4*>(zp);
  const int n8 = V >> 3;
#pragma unroll 2
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    float x[8];
    unpack8(__ldg(z4 + i), x);
    float y[8];
    if (zp) unpack8(__ldg(p4 + i), y);
    float lm = x[0];
#pragma unroll
    for (int e = 1; e < 8; ++e) lm = fmaxf(lm, x[e]);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int v = i * 8 + e;
      if (v != mask_id && (x[e] > bv || (x[e] == bv && v < bi))) { bv = x[e]; bi = v; }
    }
    if (lm > m) {
      const float r = __expf(m - lm);
      sum *= r;
      tt *= r;
      m = lm;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float ex = __expf(x[e] - m);
      sum += ex;
      if (zp) tt += ex * (x[e] - y[e]);
    }
  }
  // combine the threads: warps by shuffles, then the warps through shared memory
  auto combine = [](float& m1, float& s1, float& t1, float& b1, int& i1, float m2, float s2, float t2, float b2, int i2) {
    const float mn = fmaxf(m1, m2);
    const float r1 = m1 == -INFINITY ? 0.f : __expf(m1 - mn), r2 = m2 == -INFINITY ? 0.f : __expf(m2 - mn);
    s1 = s1 * r1 + s2 * r2;
    t1 = t1 * r1 + t2 * r2;
    m1 = mn;
    if (b2 > b1 || (b2 == b1 && i2 < i1)) { b1 = b2; i1 = i2; }
  };
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, sum, o);
    const float t2 = __shfl_xor_sync(0xffffffffu, tt, o), b2 = __shfl_xor_sync(0xffffffffu, bv, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
    combine(m, sum, tt, bv, bi, m2, s2, t2, b2, i2);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (l == 0) {
    s_f[4 * w] = m; s_f[4 * w + 1] = sum; s_f[4 * w + 2] = tt; s_f[4 * w + 3] = bv;
    s_i[w] = bi;
  }
  __syncthreads();
  RowStats r;
  r.M = s_f[0]; r.S = s_f[1]; r.T = s_f[2]; r.BV = s_f[3]; r.BI = s_i[0];
  for (int q = 1; q < nw; ++q)
    combine(r.M, r.S, r.T, r.BV, r.BI, s_f[4 * q], s_f[4 * q + 1], s_f[4 * q + 2], s_f[4 * q + 3], s_i[q]);
  __syncthreads();
  return r;
}
// For LM row j with logits z[j, :] (bf16): lse, conf = p(argmax over v != mask), argmax,
// and when has_prev: D = sum_v p_t (z_t - lse_t - z_p + lse_p), clamped at 0.
// One CTA (256 threads) per row.
__global__ void kl_conf_kernel(const __nv_bfloat16* __restrict__ z, int64_t ldz, const __nv_bfloat16* __restrict__ zp_store,
                               int64_t ldp, const float* __restrict__ lse_prev, const int* __restrict__ has_prev,
                               const int* __restrict__ rows, const int* count_dev, int rows_cap, int V, int mask_id,
                               float* __restrict__ conf, int* __restrict__ amax, float* __restrict__ lse_out,
                               float* __restrict__ kl_out) {
  pdl_trigger();
  pdl_wait();
  const int m = count_dev ? min(*count_dev, rows_cap) : rows_cap;
  const int j = blockIdx.x;
  if (j >= m) return;
  const int flat = rows ? rows[j] : j;
  __shared__ float s_f[4 * 32];
  __shared__ int s_i[32];
  const bool hp = has_prev && has_prev[flat];
  const RowStats r = row_stats(z + static_cast<int64_t>(j) * ldz, hp ? zp_store + static_cast<int64_t>(flat) * ldp : nullptr,
                               V, mask_id, s_f, s_i);
  if (threadIdx.x == 0) {
    const float L = r.M + logf(r.S);
    int BI = r.BI;
    if (BI == 0x7fffffff) {   // no finite logit: report it, and never hand on an invalid token id
      set_dev_status(DLLM_DEV_BAD_INDEX);
      BI = 0;
    }
    conf[flat] = __expf(r.BV - L);
    amax[flat] = BI;
    if (lse_out) lse_out[flat] = L;
    if (kl_out) kl_out[j] = hp ? fmaxf(r.T / r.S - (L - lse_prev[flat]), 0.f) : NAN;
  }
}

// ------------------------------------------------------------------ selection
constexpr int kSelThreads = 1024;
constexpr int kSelMaxN = 8192;

// exclusive block scan for 1024 threads; returns the exclusive prefix, total via ref
__device__ __forceinline__ int block_scan_excl(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    s_warp[lane] = t;   // inclusive
  }
  __syncthreads();
  const int base = w ? s_warp[w - 1] : 0;
  total = s_warp[31];
  __syncthreads();
  return base + x - v;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ uint32_t keys[kSelMaxN];
  __shared__ uint8_t elig[kSelMaxN];
  __shared__ int hist[256];
  __shared__ int s_warp[32];
  __shared__ int s_misc[4];
  const int tid = threadIdx.x;
  int off = 0;
  for (int b = 0; b < p.B; ++b) {
    const float* sc = p.scores ? p.scores + static_cast<int64_t>(b) * p.n : nullptr;
    int local_elig = 0;
    for (int i = tid; i < p.n; i += kSelThreads) {
      const float s = sc ? sc[i] : 0.f;
      uint32_t k;
      bool e;
      switch (p.mode) {
        case SEL_TOPK_DESC: k = order_key(s); e = true; break;
        case SEL_BELOW_CAP_ASC: k = (s != s) ? 0xffffffffu : ~order_key(s); e = (s != s) || (s < p.tau); break;
        case SEL_FORCED_ASC: k = (s != s) ? 0xffffffffu : ~order_key(s); e = true; break;
        default: k = 0; e = p.lock ? (p.lock[static_cast<int64_t>(b) * p.seq_n + p.cand_start + i] == 0) : true; break;
      }
      keys[i] = k;
      elig[i] = e ? 1 : 0;
      local_elig += e ? 1 : 0;
    }
    __syncthreads();
    int n_elig;
    block_scan_excl(local_elig, s_warp, n_elig);
    const int kk = (p.mode == SEL_ALL_ELIGIBLE) ? n_elig : min(p.k, n_elig);
    uint32_t T = 0;
    int need_eq = 0;
    const bool take_all = (kk == n_elig);
    if (!take_all && kk > 0) {
      uint32_t prefix = 0, mask = 0;
      int remaining = kk;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < p.n; i += kSelThreads)
          if (elig[i] && (keys[i] & mask) == prefix) atomicAdd(&hist[(keys[i] >> shift) & 255], 1);
        __syncthreads();
        if (tid == 0) {
          int above = 0, dg = 255;
          for (; dg >= 0; --dg) {
            if (above + hist[dg] >= remaining) break;
            above += hist[dg];
          }
          s_misc[0] = dg;
          s_misc[1] = remaining - above;
        }
        __syncthreads();
        prefix |= static_cast<uint32_t>(s_misc[0]) << shift;
        mask |= 255u << shift;
        remaining = s_misc[1];
        __syncthreads();
      }
      T = prefix;
      need_eq = remaining;
    }
    // flags in index order: eq-rank among keys == T, then compaction
    int carry_eq = 0, carry_sel = 0;
    for (int base = 0; base < p.n; base += kSelThreads) {
      const int i = base + tid;
      const bool in = i < p.n;
      const bool e = in && elig[i];
      const bool eq = e && !take_all && keys[i] == T;
      int tot_eq;
      const int eqr = block_scan_excl(eq ? 1 : 0, s_warp, tot_eq) + carry_eq;
      const bool sel = e && (take_all || keys[i] > T || (eq && eqr < need_eq));
      int tot_sel;
      const int o = block_scan_excl(sel ? 1 : 0, s_warp, tot_sel) + carry_sel;
      if (p.flag && in) p.flag[static_cast<int64_t>(b) * p.seq_n + p.cand_start + i] = (sel && kk > 0) ? 1 : 0;
      if (sel && kk > 0) {
        const int pos = p.cand_start + i;
        if (p.act_pos) p.act_pos[static_cast<int64_t>(b) * p.k_max + o] = pos;
        if (p.row_map) p.row_map[off + o] = b * p.seq_n + pos;
      }
      carry_eq += tot_eq;
      carry_sel += tot_sel;
    }
    const int cnt = kk > 0 ? carry_sel : 0;
    if (tid == 0) {
      if (p.count) p.count[b] = cnt;
      if (p.seq_off) p.seq_off[b] = off;
    }
    off += cnt;
    __syncthreads();
  }
  if (tid == 0) {
    if (p.seq_off) p.seq_off[p.B] = off;
    if (p.total) *p.total = off;
  }
}

// ------------------------------------------------------------------ row lists
// Rows of a contiguous position range per sequence: row_map = b * N + start + i.
__global__ void range_rows_kernel(int B, int N, int start, int len, int* row_map, int* seq_off, int* total) {
  pdl_trigger();
  pdl_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < B * len) row_map[idx] = (idx / len) * N + start + (idx % len);
  if (idx <= B && seq_off) seq_off[idx] = idx * len;
  if (idx == 0 && total) *total = B * len;
}

// LM rows: the recomputed rows that are masked and inside [blk_s, blk_e) (and, with
// a round mask, inside this round).  Single CTA, order-preserving compaction.
__global__ void __launch_bounds__(kSelThreads) lm_rows_kernel(const int* __restrict__ rows, const int* count_dev,
                                                              int rows_cap, const int* __restrict__ tokens, int mask_id,
                                                              int N, int blk_s, int blk_e,
                                                              const uint8_t* __restrict__ round_mask,
                                                              int include_unmasked, int* __restrict__ lm_rows,
                                                              int* lm_count) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_warp[32];
  const int m = count_dev ? min(*count_dev, rows_cap) : rows_cap;
  int carry = 0;
  for (int base = 0; base < m; base += kSelThreads) {
    const int j = base + threadIdx.x;
    bool keep = false;
    int flat = 0;
    if (j < m) {
      flat = rows[j];
      const int pos = flat % N;
      const bool masked = tokens[flat] == mask_id;
      keep = (masked && pos >= blk_s && pos < blk_e && (!round_mask || round_mask[pos - blk_s])) ||
             (include_unmasked && !masked);
    }
    int tot;
    const int o = block_scan_excl(keep ? 1 : 0, s_warp, tot) + carry;
    if (keep) lm_rows[o] = flat;
    carry += tot;
  }
  if (threadIdx.x == 0) *lm_count = carry;
}

// h_prev[flat] = h[flat], masked_prev[flat] = (tokens[flat] == mask) for the given rows.
__global__ void snapshot_rows_kernel(const float* __restrict__ h, float* __restrict__ h_prev,
                                     const int* __restrict__ tokens, uint8_t* __restrict__ masked_prev, int mask_id,
                                     const int* __restrict__ rows, int n_rows, int d) {
  pdl_trigger();
  pdl_wait();
  const int j = blockIdx.x;
  if (j >= n_rows) return;
  const int flat = rows[j];
  for (int i = threadIdx.x * 4; i < d; i += blockDim.x * 4)
    *reinterpret_cast<float4*>(h_prev + static_cast<int64_t>(flat) * d + i) =
        *reinterpret_cast<const float4*>(h + static_cast<int64_t>(flat) * d + i);
  if (threadIdx.x == 0 && masked_prev) masked_prev[flat] = tokens[flat] == mask_id ? 1 : 0;
}

// ------------------------------------------------------------------ unmask
// One CTA per sequence; threads stride over the block positions blk_s + i.
// TOPCONF: commit the n masked positions with the highest conf (ties: lower position).
// round_mask (DUS): commit every masked position of this round.
__global__ void unmask_kernel(int* __restrict__ tokens, const float* __restrict__ conf, const int* __restrict__ amax,
                              int N, int blk_s, int blk_len, int mask_id, int n_commit,
                              const uint8_t* __restrict__ round_mask, int cb_mode, float cb_tau,
                              int* __restrict__ pos_out, int* __restrict__ tok_out, int* __restrict__ n_out,
                              int max_out, int* __restrict__ remain) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float s_conf[];
  uint8_t* s_masked = reinterpret_cast<uint8_t*>(s_conf + blk_len);
  __shared__ int s_cnt;
  const int b = blockIdx.x;
  if (threadIdx.x == 0) s_cnt = 0;
  const int64_t base = static_cast<int64_t>(b) * N + blk_s;
  for (int i = threadIdx.x; i < blk_len; i += blockDim.x) {
    s_masked[i] = tokens[base + i] == mask_id ? 1 : 0;
    float c = conf[base + i];
    c = (c != c) ? -INFINITY : c + 0.0f;
    s_conf[i] = c;
  }
  __syncthreads();
  if (cb_mode) {
    // confidence-bounded, dilation-filtered: take the best eligible position (confidence
    // descending, ties to the lower position) while it reaches cb_tau (the first always),
    // making its neighbours ineligible, at most n_commit times.  s_masked: 1 eligible,
    // 2 taken, 3 masked but next to a taken position.
    __shared__ float s_bv[32];
    __shared__ int s_bi[32];
    __shared__ int s_stop;
    for (int k = 0; k < n_commit; ++k) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      for (int i = threadIdx.x; i < blk_len; i += blockDim.x)
        if (s_masked[i] == 1 && (s_conf[i] > bv || (s_conf[i] == bv && i < bi))) { bv = s_conf[i]; bi = i; }
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if ((threadIdx.x & 31) == 0) { s_bv[threadIdx.x >> 5] = bv; s_bi[threadIdx.x >> 5] = bi; }
      __syncthreads();
      if (threadIdx.x == 0) {
        for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w)
          if (s_bv[w] > bv || (s_bv[w] == bv && s_bi[w] < bi)) { bv = s_bv[w]; bi = s_bi[w]; }
        s_stop = (bi == 0x7fffffff || (k > 0 && !(bv >= cb_tau))) ? 1 : 0;
        if (!s_stop) {
          s_masked[bi] = 2;
          if (bi > 0 && s_masked[bi - 1] == 1) s_masked[bi - 1] = 3;
          if (bi + 1 < blk_len && s_masked[bi + 1] == 1) s_masked[bi + 1] = 3;
        }
      }
      __syncthreads();
      if (s_stop) break;
    }
  }
  for (int i = threadIdx.x; i < blk_len; i += blockDim.x) {
    bool commit = false;
    if (cb_mode) {
      commit = s_masked[i] == 2;
    } else if (s_masked[i]) {
      if (round_mask) {
        commit = round_mask[i] != 0;
      } else {
        int rank = 0;
        const float ci = s_conf[i];
        for (int q = 0; q < blk_len && rank < n_commit; ++q)
          if (s_masked[q] && (s_conf[q] > ci || (s_conf[q] == ci && q < i))) ++rank;
        commit = rank < n_commit;
      }
    }
    if (commit) {
      const int tok = amax[base + i];
      tokens[base + i] = tok;
      if (pos_out) {
        const int slot = atomicAdd(&s_cnt, 1);
        if (slot < max_out) {
          pos_out[static_cast<int64_t>(b) * max_out + slot] = blk_s + i;
          tok_out[static_cast<int64_t>(b) * max_out + slot] = tok;
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && n_out) n_out[b] = min(s_cnt, max_out);
  if (remain) {   // masked positions of the block left after this step
    __shared__ int s_left;
    if (threadIdx.x == 0) s_left = 0;
    __syncthreads();
    int left = 0;
    for (int i = threadIdx.x; i < blk_len; i += blockDim.x) left += tokens[base + i] == mask_id;
    atomicAdd(&s_left, left);
    __syncthreads();
    if (threadIdx.x == 0) remain[b] = s_left;
  }
}

// SureLock per LM row (one CTA): lse, argmax (mask id excluded), conf = p(argmax) of this
// step's stored logits; when the position's logits were also stored at the previous step,
// D = KL(p_t || p_t-1) clamped at 0; the lock rule for rows unmasked at the start of the
// step: D < eps and conf > tau (or a forced pattern); finally the position's stamp is set.
__global__ void kl_step_kernel(KlStep k) {
  pdl_trigger();
  pdl_wait();
  const int m = k.count ? min(*k.count, k.rows_cap) : k.rows_cap;
  const int j = blockIdx.x;
  if (j >= m) return;
  const int flat = k.rows[j];
  const int V = k.V;
  __shared__ float s_f[4 * 32];
  __shared__ int s_i[32];
  // stamps hold step + 1 of the last store, so a store at the previous step reads k.step
  const bool has_prev = k.stamp && k.z_prev && k.step > 0 && k.stamp[flat] == k.step;
  const RowStats r = row_stats(k.z_cur + static_cast<int64_t>(flat) * V,
                               has_prev ? k.z_prev + static_cast<int64_t>(flat) * V : nullptr, V, k.mask_id, s_f, s_i);
  if (threadIdx.x == 0) {
    const float L = r.M + logf(r.S);
    int BI = r.BI;
    if (BI == 0x7fffffff) {   // no finite logit: report it, and never hand on an invalid token id
      set_dev_status(DLLM_DEV_BAD_INDEX);
      BI = 0;
    }
    const float kl = has_prev ? fmaxf(r.T / r.S - (L - k.lse_prev[flat]), 0.f) : NAN;
    const float conf = __expf(r.BV - L);
    k.conf[flat] = conf;
    k.amax[flat] = BI;
    k.lse_cur[flat] = L;
    if (k.kl_out) k.kl_out[j] = kl;
    const bool eligible = k.lock_masked || k.tokens[flat] != k.mask_id;
    if (k.lock && eligible && has_prev) {
      const bool lock_now = k.pattern ? (k.pattern[flat] != 0) : (kl < k.kl_eps && conf > k.conf_tau);
      if (lock_now) k.lock[flat] = 1;
    }
    if (k.stamp) k.stamp[flat] = k.step + 1;
  }
}

// dst[rows[j]] = src[rows[j]] (d floats) for j < *count.
__global__ void copy_rows_kernel(const float* __restrict__ src, float* __restrict__ dst, const int* __restrict__ rows,
                                 const int* count_dev, int rows_cap, int d) {
  pdl_trigger();
  pdl_wait();
  const int m = count_dev ? min(*count_dev, rows_cap) : rows_cap;
  const int j = blockIdx.x;
  if (j >= m) return;
  const int64_t off = static_cast<int64_t>(rows[j]) * d;
  for (int i = threadIdx.x * 4; i < d; i += blockDim.x * 4)
    *reinterpret_cast<float4*>(dst + off + i) = *reinterpret_cast<const float4*>(src + off + i);
}

}  // namespace

// ------------------------------------------------------------------ launchers
int rope_table_launch(float* cos_t, float* sin_t, int N, int hd, double theta, cudaStream_t st) {
  const int half = hd / 2;
  const int n = N * half;
{
    const int rc_ = launch_pdl(  rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, st, cos_t, sin_t, N, half, theta, hd);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int embed_rows_launch(const __nv_bfloat16* E, int V, const int* tokens, const int* row_map, const int* count_dev,
                      int rows_cap, int d, float* h, cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
  if (d % 8) return DLLM_ERR_SHAPE;
{
    const int rc_ = launch_pdl(  embed_rows_kernel, dim3(rows_cap), dim3(128), 0, st, E, tokens, row_map, count_dev, rows_cap, d, V, h);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

namespace {
// RoPE (rotate-half pairs i, i + hd/2 of every q and k head, by pos theta^(-2i/hd) from the
// cos/sin table) on the rows' fp32 QKV products, rounded once to bf16: q to its row of q_out,
// k and v into the cache rows of their positions.  A thread takes four consecutive i of one
// head (16-byte loads of both halves and of the table) in the rows of its grid row.
__global__ void rope_scatter_kernel(const float* __restrict__ y, int rows_cap, const int* count_dev,
                                    const int* __restrict__ row_map, int qkvd, int qd, int kvd, int hd_log2, int N,
                                    int Hkv, const float* __restrict__ rope_cos, const float* __restrict__ rope_sin,
                                    __nv_bfloat16* q_out, __nv_bfloat16* kc, __nv_bfloat16* vc) {
  pdl_trigger();
  pdl_wait();
  const int m_rows = count_dev ? min(*count_dev, rows_cap) : rows_cap;
  const int hd = 1 << hd_log2, half = hd >> 1;
  const int r = blockIdx.x * blockDim.x + threadIdx.x;      // 4-pair group within a row
  if (r >= (qkvd >> 3)) return;
  const int head = r >> (hd_log2 - 3);                      // head slot over q, k, v heads (hd / 8 groups each)
  const int i = (r - (head << (hd_log2 - 3))) * 4;
  const int n_lo = (head << hd_log2) + i;                   // feature of the low half
  const bool rotate = n_lo < qd + kvd;
  int nn = n_lo - qd;                                       // feature within K (or V) when not a q feature
  __nv_bfloat16* cache = kc;
  if (nn >= kvd) {
    nn -= kvd;
    cache = vc;
  }
  const int kvh = nn >> hd_log2;
  for (int j = blockIdx.y; j < m_rows; j += gridDim.y) {    // rows
    const float* yr = y + static_cast<int64_t>(j) * qkvd;
    const float4 a = __ldg(reinterpret_cast<const float4*>(yr + n_lo));
    const float4 bq = __ldg(reinterpret_cast<const float4*>(yr + n_lo + half));
    const int flat = __ldg(row_map + j);
    const int b = flat / N, pos = flat - b * N;
    float lo[4] = {a.x, a.y, a.z, a.w}, hi[4] = {bq.x, bq.y, bq.z, bq.w};
    if (rotate) {
      const float4 c4 = __ldg(reinterpret_cast<const float4*>(rope_cos + static_cast<int64_t>(pos) * half + i));
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(rope_sin + static_cast<int64_t>(pos) * half + i));
      const float cs[4] = {c4.x, c4.y, c4.z, c4.w}, sn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = lo[e], z = hi[e];
        lo[e] = x * cs[e] - z * sn[e];
        hi[e] = z * cs[e] + x * sn[e];
      }
    }
    __nv_bfloat16* dst = n_lo < qd ? q_out + static_cast<int64_t>(j) * qd + n_lo
                                   : cache + ((static_cast<int64_t>(b) * Hkv + kvh) * N + pos) * hd +
                                         (nn - (kvh << hd_log2));
    uint2 w0, w1;
    __nv_bfloat162 t0 = __floats2bfloat162_rn(lo[0], lo[1]), t1 = __floats2bfloat162_rn(lo[2], lo[3]);
    __nv_bfloat162 t2 = __floats2bfloat162_rn(hi[0], hi[1]), t3 = __floats2bfloat162_rn(hi[2], hi[3]);
    w0.x = *reinterpret_cast<uint32_t*>(&t0);
    w0.y = *reinterpret_cast<uint32_t*>(&t1);
    w1.x = *reinterpret_cast<uint32_t*>(&t2);
    w1.y = *reinterpret_cast<uint32_t*>(&t3);
    *reinterpret_cast<uint2*>(dst) = w0;
    *reinterpret_cast<uint2*>(dst + half) = w1;
  }
}
}  // namespace

int rope_scatter_launch(const float* y, int rows_cap, const int* count_dev, const int* row_map, int qkvd, int qd,
                        int kvd, int hd, int N, int Hkv, const float* rope_cos, const float* rope_sin,
                        __nv_bfloat16* q_out, __nv_bfloat16* kc, __nv_bfloat16* vc, cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
  int hd_log2 = 0;
  while ((1 << hd_log2) < hd) ++hd_log2;
  if (hd < 8 || (1 << hd_log2) != hd || qd % hd || kvd % hd || qkvd != qd + 2 * kvd) {
    set_last_error("rope_scatter: head_dim a power of two >= 8, q/kv widths whole heads", __FILE__, __LINE__);
    return DLLM_ERR_SHAPE;
  }
  // 16-byte loads of the fp32 products and of the cos/sin rows, 8-byte stores of 4 bf16 values
  if ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(rope_cos) |
       reinterpret_cast<uintptr_t>(rope_sin)) % 16 ||
      (reinterpret_cast<uintptr_t>(q_out) | reinterpret_cast<uintptr_t>(kc) | reinterpret_cast<uintptr_t>(vc)) % 8) {
    set_last_error("rope_scatter: products and cos/sin tables 16-byte aligned, q and caches 8-byte aligned",
                   __FILE__, __LINE__);
    return DLLM_ERR_INVALID_ARG;
  }
  const int per_row = qkvd >> 3;
  return launch_pdl(rope_scatter_kernel, dim3((per_row + 255) / 256, std::min(rows_cap, 65535)), dim3(256), 0, st, y, rows_cap,
                    count_dev, row_map, qkvd, qd, kvd, hd_log2, N, Hkv, rope_cos, rope_sin, q_out, kc, vc);
}

int rmsnorm_rows_launch(const float* h, const int* row_map, const int* count_dev, int rows_cap, int d, const float* g,
                        float eps, __nv_bfloat16* z, int64_t ldz, cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
  if (d % 4) return DLLM_ERR_SHAPE;
{
    const int rc_ = launch_pdl(  rmsnorm_rows_kernel, dim3(rows_cap), dim3(256), 0, st, h, row_map, count_dev, rows_cap, d, g, eps, z, ldz);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int score_es_launch(float* h, float* h_prev, const float* conf, uint8_t* masked_prev, const int* tokens,
                    int mask_id, const int* rows, int n_rows, int d, float alpha, int update,
                    const uint8_t* act_prev, float* score, cudaStream_t st) {
  if (n_rows <= 0) return DLLM_OK;
  if (d % 4) return DLLM_ERR_SHAPE;
  const int blocks = (n_rows * 32 + 255) / 256;
{
    const int rc_ = launch_pdl(  score_es_kernel, dim3(blocks), dim3(256), 0, st, h, h_prev, conf, masked_prev, tokens, mask_id, rows, n_rows, d, alpha,
                                          update, act_prev, score);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int score_cos_launch(const float* vnew, int64_t ldv, const __nv_bfloat16* vc, const int* rows, const int* count_dev,
                     int rows_cap, int N, int Hkv, int hd, float* sim, cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
  // 16-byte vector loads: rows of 8-element multiples on 16-byte boundaries
  if (hd % 8 || ldv % 4 || (reinterpret_cast<uintptr_t>(vnew) | reinterpret_cast<uintptr_t>(vc)) % 16) {
    set_last_error("score_cos: head_dim a multiple of 8, 16-byte aligned rows", __FILE__, __LINE__);
    return DLLM_ERR_SHAPE;
  }
  const int blocks = (rows_cap * 32 + 255) / 256;
{
    const int rc_ = launch_pdl(  score_cos_kernel, dim3(blocks), dim3(256), 0, st, vnew, ldv, vc, rows, count_dev, rows_cap, N, Hkv, hd, sim);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int kl_conf_launch(const __nv_bfloat16* z, int64_t ldz, const __nv_bfloat16* zp_store, int64_t ldp,
                   const float* lse_prev, const int* has_prev, const int* rows, const int* count_dev, int rows_cap,
                   int V, int mask_id, float* conf, int* amax, float* lse_out, float* kl_out, cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
  // 16-byte vector loads: rows of 8-element multiples on 16-byte boundaries
  if (V % 8 || ldz % 8 || ldp % 8 ||
      (reinterpret_cast<uintptr_t>(z) | reinterpret_cast<uintptr_t>(zp_store)) % 16) {
    set_last_error("kl_conf: vocabulary and row strides multiples of 8, 16-byte aligned rows", __FILE__, __LINE__);
    return DLLM_ERR_SHAPE;
  }
{
    const int rc_ = launch_pdl(  kl_conf_kernel, dim3(rows_cap), dim3(256), 0, st, z, ldz, zp_store, ldp, lse_prev, has_prev, rows, count_dev, rows_cap, V,
                                           mask_id, conf, amax, lse_out, kl_out);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int select_launch(const SelectParams& p, cudaStream_t st) {
  if (p.B <= 0) return DLLM_OK;
  if (p.n < 0 || p.n > kSelMaxN) return DLLM_ERR_UNSUPPORTED;
{
    const int rc_ = launch_pdl(  select_kernel, dim3(1), dim3(kSelThreads), 0, st, p);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int range_rows_launch(int B, int N, int start, int len, int* row_map, int* seq_off, int* total, cudaStream_t st) {
  const int n = std::max(B * len, B + 1);
{
    const int rc_ = launch_pdl(  range_rows_kernel, dim3((n + 255) / 256), dim3(256), 0, st, B, N, start, len, row_map, seq_off, total);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int lm_rows_launch(const int* rows, const int* count_dev, int rows_cap, const int* tokens, int mask_id, int N,
                   int blk_s, int blk_e, const uint8_t* round_mask, int include_unmasked, int* lm_rows, int* lm_count,
                   cudaStream_t st) {
{
    const int rc_ = launch_pdl(  lm_rows_kernel, dim3(1), dim3(kSelThreads), 0, st, rows, count_dev, rows_cap, tokens, mask_id, N, blk_s, blk_e, round_mask, include_unmasked,
                                            lm_rows, lm_count);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int snapshot_rows_launch(const float* h, float* h_prev, const int* tokens, uint8_t* masked_prev, int mask_id,
                         const int* rows, int n_rows, int d, cudaStream_t st) {
  if (n_rows <= 0) return DLLM_OK;
{
    const int rc_ = launch_pdl(  snapshot_rows_kernel, dim3(n_rows), dim3(256), 0, st, h, h_prev, tokens, masked_prev, mask_id, rows, n_rows, d);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

int unmask_launch(int* tokens, const float* conf, const int* amax, int B, int N, int blk_s, int blk_len, int mask_id,
                  int n_commit, const uint8_t* round_mask, int cb_mode, float cb_tau, int* pos_out, int* tok_out,
                  int* n_out, int max_out, int* remain, cudaStream_t st) {
  if (blk_len <= 0 || blk_len > 8192) return DLLM_ERR_UNSUPPORTED;
  const int threads = std::min(1024, ((blk_len + 31) / 32) * 32);
  const size_t smem = blk_len * sizeof(float) + blk_len;
{
    const int rc_ = launch_pdl(  unmask_kernel, dim3(B), dim3(threads), smem, st, tokens, conf, amax, N, blk_s, blk_len, mask_id, n_commit, round_mask,
                                          cb_mode, cb_tau, pos_out, tok_out, n_out, max_out, remain);
    if (rc_) return rc_;
  }
  return DLLM_OK;
}

}  // namespace dllm

namespace dllm {

int kl_step_launch(const KlStep& k, cudaStream_t st) {
  if (k.rows_cap <= 0) return DLLM_OK;
  if (k.V % 8 || (reinterpret_cast<uintptr_t>(k.z_cur) | reinterpret_cast<uintptr_t>(k.z_prev)) % 16) return DLLM_ERR_SHAPE;
  return launch_pdl(kl_step_kernel, dim3(k.rows_cap), dim3(256), 0, st, k);
}

int copy_rows_launch(const float* src, float* dst, const int* rows, const int* count_dev, int rows_cap, int d,
                     cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
  if (d % 4) return DLLM_ERR_SHAPE;
  return launch_pdl(copy_rows_kernel, dim3(rows_cap), dim3(256), 0, st, src, dst, rows, count_dev, rows_cap, d);
}

}  // namespace dllm
