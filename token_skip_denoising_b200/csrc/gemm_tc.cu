// Active-row GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// The recomputed rows of a token-skipping step are few (7..32 per sequence in
// the block-cached regime, ES-dLLM summary sec. 2.1 item 2: "the size of the
// matrix multiplications in later layers shrinks"), so the kernel is laid out
// swap-AB: the weight matrix supplies the 128-row MMA operand A, the active
// rows the N = BN operand B (BN in {16, 32, 64, 128, 256}).  Small row counts
// are weight-streaming (HBM-bound): enough CTAs are launched, with split-K, to
// keep every SM's TMA engine busy, and the last CTA of a split group reduces
// the partial tiles in a fixed order (deterministic).  Epilogues fuse RoPE +
// K/V cache scatter, the residual add, SwiGLU and the LM-head softmax
// statistics.
//
// Roles (128 threads): warp 0 lane 0 issues TMA loads, warp 1 lane 0 issues
// MMAs, warp 1 owns the TMEM allocation; all four warps run the epilogue, one
// thread per TMEM lane (= one weight row of the tile).
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace dllm {

__device__ int g_dev_status = 0;

namespace {

constexpr int kBK = 64;                      // K elements per stage (128 B rows, one swizzle span)
constexpr int kTileM = 128;                  // weight rows per tile
constexpr uint32_t kABytes = kTileM * kBK * 2;

template <int BN>
struct Cfg {
  static constexpr int kStages = (BN >= 256) ? 4 : 4;
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
  static constexpr int kXPitch = 17;         // epilogue exchange buffer pitch (floats)
  static constexpr size_t kSmem = 1024 /*align slack*/ + kStages * kStageBytes + 128 * kXPitch * 4 +
                                  (2 * kStages + 2) * 8 + 64;
};

struct KParams {
  int K;
  int rows_cap;
  const int* rows_dev;
  int n_tiles_w;
  int tiles_act;
  int splits;
  int kb_per_split;
  int swiglu;
  int ffn;
  float* partial;
  int* counters;
  EpiParams epi;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// (value desc, id asc) argmax across the warp
__device__ __forceinline__ void warp_argmax(float& v, int& id) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, v, o);
    int oi = __shfl_xor_sync(0xffffffffu, id, o);
    if (ov > v || (ov == v && oi < id)) { v = ov; id = oi; }
  }
}

template <int BN>
__global__ void __launch_bounds__(128, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, KParams p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* xbuf = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(xbuf + 128 * C::kXPitch);
  uint64_t* empty_bar = full_bar + C::kStages;
  uint64_t* done_bar = empty_bar + C::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tw = blockIdx.x;             // weight tile
  const int ta = blockIdx.y;             // activation-row tile
  const int z = blockIdx.z;              // K split
  const int act0 = ta * BN;
  const int m_rows = p.rows_dev ? min(*p.rows_dev, p.rows_cap) : p.rows_cap;
  if (act0 >= m_rows) return;            // uniform: no valid rows in this tile

  const int KB = p.K / kBK;
  const int kb0 = z * p.kb_per_split;
  const int kb1 = min(KB, kb0 + p.kb_per_split);
  const int row0 = p.swiglu ? tw * 64 : tw * kTileM;
  const int row1 = p.swiglu ? p.ffn + tw * 64 : tw * kTileM + 64;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(done_bar, 1);
    s_flag[0] = 0;   // abort flag
    s_flag[1] = 0;   // split-K "last CTA" flag
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_x = policy_evict_last();
    for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
      const int s = i % C::kStages;
      const uint32_t ph = (i / C::kStages) & 1;
      if (!mbar_wait(&empty_bar[s], ph ^ 1)) { s_flag[0] = 1; break; }
      if (s_flag[0]) break;
      uint8_t* a = stage_base + s * C::kStageBytes;
      uint8_t* b = a + kABytes;
      mbar_arrive_expect_tx(&full_bar[s], C::kStageBytes);
      tma_load_2d(a, &tmW, &full_bar[s], kb * kBK, row0, pol_w);
      tma_load_2d(a + kABytes / 2, &tmW, &full_bar[s], kb * kBK, row1, pol_w);
      tma_load_2d(b, &tmX, &full_bar[s], kb * kBK, act0, pol_x);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = make_idesc_bf16(kTileM, BN);
    bool ok = true;
    for (int kb = kb0, i = 0; kb < kb1; ++kb, ++i) {
      const int s = i % C::kStages;
      const uint32_t ph = (i / C::kStages) & 1;
      if (!mbar_wait(&full_bar[s], ph)) { s_flag[0] = 1; ok = false; break; }
      tc_fence_after();
      const uint32_t a = smem_u32(stage_base + s * C::kStageBytes);
      const uint32_t b = a + kABytes;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
        tc_mma_f16(tmem, make_desc_k_sw128(a + k * 32), make_desc_k_sw128(b + k * 32), idesc,
                   (kb > kb0 || k > 0) ? 1u : 0u);
      }
      tc_commit(&empty_bar[s]);
    }
    (void)ok;
    tc_commit(done_bar);
  }
  __syncwarp();

  // ---------------- epilogue (all 128 threads)
  const int t = threadIdx.x;
  if (!mbar_wait(done_bar, 0)) s_flag[0] = 1;
  tc_fence_after();
  const uint32_t tbase = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const EpiParams& e = p.epi;
  __syncthreads();
  bool do_epi = !s_flag[0];   // uniform across the CTA

  const int tile_lin = tw * p.tiles_act + ta;
  if (do_epi && p.splits > 1) {
    float* mine = p.partial + (static_cast<size_t>(tile_lin) * p.splits + z) * (BN * 128);
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(tbase + c, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) mine[(c + i) * 128 + t] = v[i];
    }
    __threadfence();
    __syncthreads();
    if (t == 0) {
      const int old = atomicAdd(&p.counters[tile_lin], 1);
      s_flag[1] = (old == p.splits - 1) ? 1 : 0;
    }
    __syncthreads();
    do_epi = s_flag[1] != 0;
    __threadfence();
  }

  if (do_epi) {
    const int hd = e.head_dim;
    const int n = row0 + (t < 64 ? t : (row1 - row0) + t - 64);   // global weight row of this lane
    float* xb = xbuf;
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      if (p.splits > 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
        for (int zz = 0; zz < p.splits; ++zz) {
          if (zz == z) {
            float w[16];
            tmem_ld16(tbase + c, w);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] += w[i];
          } else {
            const float* src = p.partial + (static_cast<size_t>(tile_lin) * p.splits + zz) * (BN * 128);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] += __ldcg(src + (c + i) * 128 + t);
          }
        }
      } else {
        tmem_ld16(tbase + c, v);
      }
      const int jbase = act0 + c;
      switch (e.kind) {
        case EPI_STORE_F32: {
          float* o = static_cast<float*>(e.out);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (jbase + i < m_rows) o[static_cast<int64_t>(jbase + i) * e.ldo + n] = v[i];
          break;
        }
        case EPI_STORE_BF16: {
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(e.out);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (jbase + i < m_rows) o[static_cast<int64_t>(jbase + i) * e.ldo + n] = __float2bfloat16(v[i]);
          break;
        }
        case EPI_RESID_ADD: {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (jbase + i < m_rows) {
              const int r = e.row_map ? __ldg(e.row_map + jbase + i) : jbase + i;
              float* dst = e.h + static_cast<int64_t>(r) * e.ldh + n;
              *dst = *dst + v[i];
            }
          }
          break;
        }
        case EPI_QKV_ROPE: {
          // exchange with the rotate-half partner lane (same head, offset hd/2)
#pragma unroll
          for (int i = 0; i < 16; ++i) xb[t * C::kXPitch + i] = v[i];
          __syncthreads();
          const int half = hd >> 1;
          const int partner = t ^ half;
          const int i_in_head = n % hd;
          const int fi = i_in_head % half;
          const bool lo = i_in_head < half;
          const int region = n < e.q_dim ? 0 : (n < e.q_dim + e.kv_dim ? 1 : 2);
#pragma unroll 4
          for (int i = 0; i < 16; ++i) {
            const int j = jbase + i;
            if (j < m_rows) {
              const int flat = __ldg(e.row_map + j);
              const int b = flat / e.seq_n;
              const int pos = flat - b * e.seq_n;
              float x = v[i];
              if (region < 2) {
                const float y = xb[partner * C::kXPitch + i];
                const float cs = __ldg(e.rope_cos + static_cast<int64_t>(pos) * half + fi);
                const float sn = __ldg(e.rope_sin + static_cast<int64_t>(pos) * half + fi);
                x = lo ? (x * cs - y * sn) : (x * cs + y * sn);
              }
              const __nv_bfloat16 xv = __float2bfloat16(x);
              if (region == 0) {
                e.q_out[static_cast<int64_t>(j) * e.q_dim + n] = xv;
              } else {
                const int nn = n - e.q_dim - (region == 2 ? e.kv_dim : 0);
                const int kvh = nn / hd;
                const int64_t off = ((static_cast<int64_t>(b) * e.n_kv + kvh) * e.seq_n + pos) * hd + (nn % hd);
                (region == 1 ? e.kcache : e.vcache)[off] = xv;
              }
            }
          }
          __syncthreads();
          break;
        }
        case EPI_SWIGLU: {
#pragma unroll
          for (int i = 0; i < 16; ++i) xb[t * C::kXPitch + i] = v[i];
          __syncthreads();
          if (t < 64) {
            const int f = tw * 64 + t;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int j = jbase + i;
              if (j < m_rows) {
                const float g = v[i];
                const float u = xb[(t + 64) * C::kXPitch + i];
                const float a = g / (1.f + __expf(-g)) * u;
                e.act[static_cast<int64_t>(j) * e.ffn + f] = __float2bfloat16(a);
              }
            }
          }
          __syncthreads();
          break;
        }
        case EPI_LMHEAD: {
          // per row j: max, sum exp(x - max), argmax over this tile's 128 vocab ids
          float4* red = reinterpret_cast<float4*>(xb);   // [4 warps][16 cols]
#pragma unroll 1
          for (int i = 0; i < 16; ++i) {
            const float x = v[i];
            const float mx = warp_max(x);
            const float se = warp_sum(__expf(x - mx));
            float bv = (n == e.mask_id) ? -INFINITY : x;
            int bi = (n == e.mask_id) ? 0x7fffffff : n;
            warp_argmax(bv, bi);
            if (lane == 0) red[warp * 16 + i] = make_float4(mx, se, bv, __int_as_float(bi));
          }
          __syncthreads();
          if (t < 16 && jbase + t < m_rows) {
            float M = -INFINITY, S = 0.f, BV = -INFINITY;
            int BI = 0x7fffffff;
            for (int w = 0; w < 4; ++w) {
              const float4 r = red[w * 16 + t];
              const float nm = fmaxf(M, r.x);
              S = S * __expf(M - nm) + r.y * __expf(r.x - nm);
              M = nm;
              const int ri = __float_as_int(r.w);
              if (r.z > BV || (r.z == BV && ri < BI)) { BV = r.z; BI = ri; }
            }
            e.lm_part[static_cast<int64_t>(jbase + t) * e.n_vtiles + tw] = make_float4(M, S, BV, __int_as_float(BI));
          }
          __syncthreads();
          break;
        }
        default:
          break;
      }
    }
    if (p.splits > 1 && t == 0) p.counters[tile_lin] = 0;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

__global__ void lmhead_combine_kernel(const float4* __restrict__ part, int n_vtiles, int rows_cap,
                                      const int* rows_dev, const int* out_index, float* conf, int* amax,
                                      float* lse) {
  const int m_rows = rows_dev ? min(*rows_dev, rows_cap) : rows_cap;
  const int j = blockIdx.x;
  if (j >= m_rows) return;
  __shared__ float4 red[32];
  float M = -INFINITY, S = 0.f, BV = -INFINITY;
  int BI = 0x7fffffff;
  for (int tt = threadIdx.x; tt < n_vtiles; tt += blockDim.x) {
    const float4 r = part[static_cast<int64_t>(j) * n_vtiles + tt];
    const float nm = fmaxf(M, r.x);
    S = (M == -INFINITY ? 0.f : S * __expf(M - nm)) + r.y * __expf(r.x - nm);
    M = nm;
    const int ri = __float_as_int(r.w);
    if (r.z > BV || (r.z == BV && ri < BI)) { BV = r.z; BI = ri; }
  }
  // block reduce: 32 lanes per warp, then warps
  for (int o = 16; o; o >>= 1) {
    const float oM = __shfl_xor_sync(0xffffffffu, M, o);
    const float oS = __shfl_xor_sync(0xffffffffu, S, o);
    const float oB = __shfl_xor_sync(0xffffffffu, BV, o);
    const int oI = __shfl_xor_sync(0xffffffffu, BI, o);
    const float nm = fmaxf(M, oM);
    S = (M == -INFINITY ? 0.f : S * __expf(M - nm)) + (oM == -INFINITY ? 0.f : oS * __expf(oM - nm));
    M = nm;
    if (oB > BV || (oB == BV && oI < BI)) { BV = oB; BI = oI; }
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = make_float4(M, S, BV, __int_as_float(BI));
  __syncthreads();
  if (threadIdx.x == 0) {
    M = -INFINITY; S = 0.f; BV = -INFINITY; BI = 0x7fffffff;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      const float4 r = red[i];
      const float nm = fmaxf(M, r.x);
      S = (M == -INFINITY ? 0.f : S * __expf(M - nm)) + (r.x == -INFINITY ? 0.f : r.y * __expf(r.x - nm));
      M = nm;
      const int ri = __float_as_int(r.w);
      if (r.z > BV || (r.z == BV && ri < BI)) { BV = r.z; BI = ri; }
    }
    const int o = out_index ? out_index[j] : j;
    const float L = M + logf(S);
    if (conf) conf[o] = expf(BV - L);
    if (amax) amax[o] = BI;
    if (lse) lse[o] = L;
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2D bf16 tensor map over a row-major [rows, cols] matrix, box [box_rows, 64], 128 B swizzle.
int make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  auto enc = get_encode();
  if (!enc) { set_last_error("cuTensorMapEncodeTiled unavailable", __FILE__, __LINE__); return DLLM_ERR_CUDA; }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d): rows %lld cols %lld box %d", (int)r,
             (long long)rows, (long long)cols, box_rows);
    set_last_error(buf, __FILE__, __LINE__);
    return DLLM_ERR_CUDA;
  }
  return DLLM_OK;
}

int pick_bn(int rows) {
  if (rows <= 16) return 16;
  if (rows <= 32) return 32;
  if (rows <= 64) return 64;
  if (rows <= 128) return 128;
  return 256;
}

int pick_splits(int tiles, int KB) {
  if (tiles >= kNumSMs) return 1;
  // aim for about two resident CTAs per SM, at least 4 K blocks per split
  int best = 1;
  double best_eff = 0;
  const int max_s = std::max(1, KB / 4);
  for (int s = 1; s <= max_s && s <= 32; ++s) {
    const int total = tiles * s;
    const int slots = 2 * kNumSMs;
    const int waves = (total + slots - 1) / slots;
    const double eff = static_cast<double>(total) / (waves * slots) - 0.01 * s;
    if (eff > best_eff) { best_eff = eff; best = s; }
  }
  return best;
}

template <int BN>
int launch_bn(const CUtensorMap& tmW, const CUtensorMap& tmX, KParams& kp, cudaStream_t st) {
  using C = Cfg<BN>;
  static bool attr_done = false;
  if (!attr_done) {
    DLLM_CUDA_TRY(cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem)));
    attr_done = true;
  }
  dim3 grid(kp.n_tiles_w, kp.tiles_act, kp.splits);
  gemm_tc_kernel<BN><<<grid, 128, C::kSmem, st>>>(tmW, tmX, kp);
  count_launch();
  DLLM_CUDA_TRY(cudaGetLastError());
  return DLLM_OK;
}

}  // namespace

size_t gemm_partial_floats(int rows_cap, int n_tiles_w, int K) {
  const int bn = pick_bn(rows_cap);
  const int tiles_act = (rows_cap + bn - 1) / bn;
  const int s = pick_splits(n_tiles_w * tiles_act, K / kBK);
  if (s <= 1) return 0;
  return static_cast<size_t>(n_tiles_w) * tiles_act * s * bn * 128;
}

int gemm_counters_needed(int rows_cap, int n_tiles_w) {
  const int bn = pick_bn(rows_cap);
  return n_tiles_w * ((rows_cap + bn - 1) / bn);
}

int gemm_launch(const GemmArgs& a, const GemmScratch& s, cudaStream_t st, int force_splits, int force_bn) {
  if (a.K <= 0 || a.K % kBK != 0 || a.rows_cap <= 0 || a.n_tiles_w <= 0) return DLLM_ERR_SHAPE;
  const int bn = force_bn ? force_bn : pick_bn(a.rows_cap);
  if (bn != 16 && bn != 32 && bn != 64 && bn != 128 && bn != 256) return DLLM_ERR_INVALID_ARG;
  const int tiles_act = (a.rows_cap + bn - 1) / bn;
  const int KB = a.K / kBK;
  int splits = force_splits ? force_splits : pick_splits(a.n_tiles_w * tiles_act, KB);
  splits = std::max(1, std::min(splits, KB));
  const int kbps = (KB + splits - 1) / splits;
  splits = (KB + kbps - 1) / kbps;   // no empty split
  if (splits > 1) {
    const size_t need = static_cast<size_t>(a.n_tiles_w) * tiles_act * splits * bn * 128;
    if (!s.partial || s.partial_floats < need || !s.counters || s.n_counters < a.n_tiles_w * tiles_act) {
      // not enough scratch for split-K: run unsplit
      splits = 1;
    }
  }
  CUtensorMap tmW, tmX;
  int rc = make_tmap(&tmW, a.W, a.w_rows_total, a.K, 64);
  if (rc) return rc;
  rc = make_tmap(&tmX, a.X, a.rows_cap, a.K, bn);
  if (rc) return rc;
  KParams kp;
  kp.K = a.K;
  kp.rows_cap = a.rows_cap;
  kp.rows_dev = a.rows_dev;
  kp.n_tiles_w = a.n_tiles_w;
  kp.tiles_act = tiles_act;
  kp.splits = splits;
  kp.kb_per_split = (KB + splits - 1) / splits;
  kp.swiglu = a.swiglu ? 1 : 0;
  kp.ffn = a.epi.ffn;
  kp.partial = s.partial;
  kp.counters = s.counters;
  kp.epi = a.epi;
  switch (bn) {
    case 16: return launch_bn<16>(tmW, tmX, kp, st);
    case 32: return launch_bn<32>(tmW, tmX, kp, st);
    case 64: return launch_bn<64>(tmW, tmX, kp, st);
    case 128: return launch_bn<128>(tmW, tmX, kp, st);
    default: return launch_bn<256>(tmW, tmX, kp, st);
  }
}

int lmhead_combine_launch(const float4* part, int n_vtiles, int rows_cap, const int* rows_dev,
                          const int* out_index, float* conf, int* amax, float* lse, cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
  lmhead_combine_kernel<<<rows_cap, 256, 0, st>>>(part, n_vtiles, rows_cap, rows_dev, out_index, conf, amax, lse);
  count_launch();
  DLLM_CUDA_TRY(cudaGetLastError());
  return DLLM_OK;
}

}  // namespace dllm

extern "C" int dllm_device_status(int32_t* status, int32_t reset) {
  if (!status) {
    dllm::set_last_error("null status", __FILE__, __LINE__);
    return DLLM_ERR_INVALID_ARG;
  }
  int v = 0;
  DLLM_CUDA_TRY(cudaDeviceSynchronize());
  DLLM_CUDA_TRY(cudaMemcpyFromSymbol(&v, dllm::g_dev_status, sizeof(int)));
  if (reset) {
    int z = 0;
    DLLM_CUDA_TRY(cudaMemcpyToSymbol(dllm::g_dev_status, &z, sizeof(int)));
  }
  *status = v;
  return DLLM_OK;
}
