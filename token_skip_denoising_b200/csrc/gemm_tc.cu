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
#include <cstdlib>
#include <mutex>
#include <unordered_map>

#include "common.cuh"
#include "gemm_dev.cuh"
#include "ptx.cuh"

namespace dllm {

__device__ int g_dev_status = 0;

namespace {

using namespace gemm;

// Pipeline depth and shared memory per tile width.  Weight-streaming widths (BN <= 64)
// use ~100 KB so a CTA of the next GEMM fits beside the current one on an SM and starts
// streaming its weights during this kernel's tail (programmatic dependent launch);
// compute-bound widths take ~200 KB for a deeper ring.  Two TMEM accumulators let the
// epilogue of one work segment overlap the MMAs of the next.
template <int BN, int KSUB, bool BIG = false>
struct Cfg {
  static constexpr uint32_t kBBytes = BN * kBK * 2;                // one 64-wide k block of X
  static constexpr uint32_t kStageBytes = KSUB * (kABytes + kBBytes);
  static constexpr uint32_t kBudget = (BN <= 64 && !BIG ? 100u : 200u) * 1024u;
  static constexpr int kStagesFit = static_cast<int>(kBudget / kStageBytes);
  static constexpr int kStages = kStagesFit > 12 ? 12 : (kStagesFit < 2 ? 2 : kStagesFit);
  static constexpr uint32_t kAccCols = BN < 32 ? 32 : BN;          // TMEM columns per accumulator
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static constexpr int kXPitch = 17;                                 // epilogue exchange pitch (floats)
  // Epilogue warps: one group of four (one thread per TMEM lane) drains a tile, or, from
  // 128-wide tiles on, two groups that split its columns (a wide tile's epilogue would
  // otherwise take longer than the next tile's MMAs); then the TMA producer warp and the
  // MMA issuer warp (TMEM owner).
  static constexpr int kGroups = BN >= 128 ? 2 : 1;
  static constexpr int kEpiThreads = 128 * kGroups;
  static constexpr int kThreads = kEpiThreads + 64;
  static constexpr int kProducerWarp = kEpiThreads / 32, kMmaWarp = kProducerWarp + 1;
  static constexpr size_t kSmem = 1024 /*align slack*/ + kStages * kStageBytes + kGroups * 128 * kXPitch * 4 +
                                  (2 * kStages + 4) * 8 + 64;
  static_assert(kSmem <= 227 * 1024, "GEMM stage ring does not fit shared memory");
};
constexpr int kEpiAllBar = 3;        // named barrier of every epilogue thread (groups use 1 and 2)

struct KParams {
  int K;
  int rows_cap;
  const int* rows_dev;
  int n_tiles_w;
  int tiles_act;
  int wt_fastest;      // tile numbering: 1 weight tile fastest, 0 activation tile fastest
  int add_pieces;      // the epilogue adds into its target: a split tile's piece adds its own partial
  int swiglu;
  int ffn;
  float* partial;      // [gridDim.x][2][BN * 128]
  int* counters;       // [tiles]
  EpiParams epi;
};

// Persistent stream-K GEMM: grid = one CTA per SM (or fewer), each CTA walks its
// contiguous share of the (tile, k-block) iterations; a tile split across CTAs is
// summed by the last CTA to finish its piece, in k order.  The tile numbering decides
// which operand the concurrently running CTAs share, since CTA c works on tiles near
// c * tiles / grid:
//   weight tile fastest (tile = ta * n_tiles_w + tw), for a few activation tiles (a
//     refresh): the CTAs of the ~grid / tiles_act groups, one per activation tile, stream
//     the same weight tile at about the same time, so each weight k-block comes from DRAM
//     once (numbered the other way, a CTA would reread its whole weight tile once per
//     activation tile, a reuse distance of K x 256 B per CTA, beyond L2 across the grid);
//   activation tile fastest (tile = tw * tiles_act + ta), for many activation tiles (a
//     batch of long sequences): each CTA keeps one weight tile and passes every
//     activation tile under it, so a weight matrix larger than L2 (the vocabulary) is
//     read once; the activations are shared by all CTAs.
template <int BN, int KSUB, bool BIG>
__global__ void __launch_bounds__(Cfg<BN, KSUB, BIG>::kThreads, BN >= 128 ? 1 : 2)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, KParams p) {
  using C = Cfg<BN, KSUB, BIG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* xbuf = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(xbuf + C::kGroups * 128 * C::kXPitch);
  uint64_t* empty_bar = full_bar + C::kStages;
  uint64_t* acc_full = empty_bar + C::kStages;     // [2]
  uint64_t* acc_empty = acc_full + 2;              // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);   // [0] abort, [1] last-piece

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int c = blockIdx.x;
  const int KB = p.K / (kBK * KSUB);                    // k chunks of KSUB x 64
  const int tiles = p.n_tiles_w * p.tiles_act;
  const int64_t T = static_cast<int64_t>(tiles) * KB;
  const int64_t lo = sk_lo(T, G, c), hi = sk_lo(T, G, c + 1);
  pdl_trigger();
  if (lo >= hi) return;                                  // uniform: no work for this CTA
  const int first_tile = static_cast<int>(lo / KB);
  // With one activation tile every segment is processed (rows past the device count are
  // masked in the epilogue), so weights can stream before the previous kernel finishes.
  const bool single = p.tiles_act == 1;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::kEpiThreads);
    }
    s_flag[0] = 0;
    s_flag[1] = 0;
    fence_barrier_init();
  }
  if (warp == C::kMmaWarp) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::kProducerWarp) {
    if (lane == 0) {
      // ---------------- TMA producer: one continuous ring over every segment
      // one activation tile: every weight tile is read once (evict first); several: each weight
      // tile is read once per activation tile by neighbouring CTAs, so it should stay in L2
      const uint64_t pol_w = p.tiles_act > 1 ? policy_evict_normal() : policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int m_rows = p.rows_cap;
      // stages whose weight tiles were requested before the grid dependency resolved
      int pend_x[C::kStages], pend_a[C::kStages], n_pend = 0;
      bool waited = false;
      if (!single) {
        pdl_wait();
        waited = true;
        m_rows = p.rows_dev ? min(*p.rows_dev, p.rows_cap) : p.rows_cap;
      }
      int i = 0;
      for (int64_t it = lo; it < hi && !s_flag[0];) {
        const int tile = static_cast<int>(it / KB);
        const int kb0 = static_cast<int>(it % KB);
        const int kb1 = (hi - it < KB - kb0) ? kb0 + static_cast<int>(hi - it) : KB;
        it += kb1 - kb0;
        const int tw = p.wt_fastest ? tile % p.n_tiles_w : tile / p.tiles_act;
        const int ta = p.wt_fastest ? tile / p.n_tiles_w : tile % p.tiles_act;
        const int act0 = ta * BN;
        if (!single && act0 >= m_rows) continue;     // tile without valid rows: skipped by every role
        const int row0 = p.swiglu ? tw * 64 : tw * kTileM;
        const int row1 = p.swiglu ? p.ffn + tw * 64 : tw * kTileM + 64;
        for (int kb = kb0; kb < kb1; ++kb, ++i) {
          const int s = i % C::kStages;
          const uint32_t ph = (i / C::kStages) & 1;
          if (!waited && i >= C::kStages) {
            // the ring is full of weight tiles: now the activations are needed
            pdl_wait();
            waited = true;
            for (int q = 0; q < n_pend; ++q) {
              uint8_t* bx = stage_base + q * C::kStageBytes + KSUB * kABytes;
#pragma unroll
              for (int sub = 0; sub < KSUB; ++sub)
                tma_load_2d(bx + sub * C::kBBytes, &tmX, &full_bar[q], pend_x[q] + sub * kBK, pend_a[q], pol_x);
            }
            n_pend = 0;
          }
          if (!mbar_wait(&empty_bar[s], ph ^ 1)) { s_flag[0] = 1; break; }
          uint8_t* a = stage_base + s * C::kStageBytes;
          uint8_t* bx = a + KSUB * kABytes;
          mbar_arrive_expect_tx(&full_bar[s], C::kStageBytes);
#pragma unroll
          for (int sub = 0; sub < KSUB; ++sub) {
            const int x = (kb * KSUB + sub) * kBK;
            if (p.swiglu) {   // 64 gate rows and the matching 64 up rows: two boxes
              tma_load_2d(a + sub * kABytes, &tmW, &full_bar[s], x, row0, pol_w);
              tma_load_2d(a + sub * kABytes + kABytes / 2, &tmW, &full_bar[s], x, row1, pol_w);
            } else {          // one 128-row box (fewer, larger TMA requests stream faster)
              tma_load_2d(a + sub * kABytes, &tmW, &full_bar[s], x, row0, pol_w);
            }
          }
          if (waited) {
#pragma unroll
            for (int sub = 0; sub < KSUB; ++sub)
              tma_load_2d(bx + sub * C::kBBytes, &tmX, &full_bar[s], (kb * KSUB + sub) * kBK, act0, pol_x);
          } else {
            pend_x[n_pend] = kb * KSUB * kBK;
            pend_a[n_pend] = act0;
            ++n_pend;
          }
        }
      }
      if (!waited) {
        pdl_wait();
        for (int q = 0; q < n_pend; ++q) {
          uint8_t* bx = stage_base + q * C::kStageBytes + KSUB * kABytes;
#pragma unroll
          for (int sub = 0; sub < KSUB; ++sub)
            tma_load_2d(bx + sub * C::kBBytes, &tmX, &full_bar[q], pend_x[q] + sub * kBK, pend_a[q], pol_x);
        }
      }
    }
  } else if (warp == C::kMmaWarp) {
    if (lane == 0) {
      // ---------------- MMA issuer: alternates between the two TMEM accumulators
      constexpr uint32_t idesc = make_idesc_bf16(kTileM, BN);
      int m_rows = p.rows_cap;
      if (!single) {
        pdl_wait();
        m_rows = p.rows_dev ? min(*p.rows_dev, p.rows_cap) : p.rows_cap;
      }
      int i = 0, j = 0;
      for (int64_t it = lo; it < hi && !s_flag[0];) {
        const int tile = static_cast<int>(it / KB);
        const int kb0 = static_cast<int>(it % KB);
        const int kb1 = (hi - it < KB - kb0) ? kb0 + static_cast<int>(hi - it) : KB;
        it += kb1 - kb0;
        if (!single && (p.wt_fastest ? tile / p.n_tiles_w : tile % p.tiles_act) * BN >= m_rows) continue;
        const int b = j & 1;
        const uint32_t u = static_cast<uint32_t>(j >> 1);
        ++j;
        if (!mbar_wait(&acc_empty[b], (u & 1) ^ 1)) { s_flag[0] = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + b * C::kAccCols;
        for (int kb = kb0; kb < kb1; ++kb, ++i) {
          const int s = i % C::kStages;
          const uint32_t ph = (i / C::kStages) & 1;
          if (!mbar_wait(&full_bar[s], ph)) { s_flag[0] = 1; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(stage_base + s * C::kStageBytes);
          const uint32_t bb = a + KSUB * kABytes;
#pragma unroll
          for (int sub = 0; sub < KSUB; ++sub)
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              tc_mma_f16(d, make_desc_k_sw128(a + sub * kABytes + k * 32),
                         make_desc_k_sw128(bb + sub * C::kBBytes + k * 32), idesc,
                         (kb > kb0 || sub > 0 || k > 0) ? 1u : 0u);
          tc_commit(&empty_bar[s]);
        }
        tc_commit(&acc_full[b]);
      }
    }
  } else {
    // ---------------- epilogue warps (one or two groups of four)
    const EpiParams& e = p.epi;
    pdl_wait();
    const int m_rows = p.rows_dev ? min(*p.rows_dev, p.rows_cap) : p.rows_cap;
    // group grp drains columns [c0, c1) of every tile; thread t holds TMEM lane t (weight row)
    const int grp = warp >> 2, wq = warp & 3;
    const int t = threadIdx.x & 127;
    const int gbar = 1 + grp;
    constexpr int kCols = BN / C::kGroups;
    const int c0 = grp * kCols, c1 = c0 + kCols;
    float* const xg = xbuf + grp * 128 * C::kXPitch;
    int j = 0;
    for (int64_t it = lo; it < hi;) {
      const int tile = static_cast<int>(it / KB);
      const int kb0 = static_cast<int>(it % KB);
      const int kb1 = (hi - it < KB - kb0) ? kb0 + static_cast<int>(hi - it) : KB;
      it += kb1 - kb0;
      const int tw = p.wt_fastest ? tile % p.n_tiles_w : tile / p.tiles_act;
      const int ta = p.wt_fastest ? tile / p.n_tiles_w : tile % p.tiles_act;
      const int act0 = ta * BN;
      if (!single && act0 >= m_rows) continue;
      const int b = j & 1;
      const uint32_t u = static_cast<uint32_t>(j >> 1);
      ++j;
      const bool late = !mbar_wait(&acc_full[b], u & 1);
      if (bar_any(late || s_flag[0], kEpiAllBar, C::kEpiThreads)) {   // one decision for all epilogue threads
        s_flag[0] = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(wq * 32) << 16) + b * C::kAccCols;
      const int row0 = p.swiglu ? tw * 64 : tw * kTileM;
      const int row1 = p.swiglu ? p.ffn + tw * 64 : tw * kTileM + 64;
      const int n = t < 64 ? row0 + t : row1 + (t - 64);
      const bool whole = (kb0 == 0 && kb1 == KB) || p.add_pieces;
      if (whole) {
        for (int cc = c0; cc < c1; cc += 16) {
          float v[16];
          tmem_ld16(tb + cc, v);
          if (cc + 16 >= c1) {                         // this group's columns drained: hand them back
            tc_fence_before();
            mbar_arrive(&acc_empty[b]);
          }
          epi_chunk<C::kXPitch>(e, v, t, lane, wq, n, act0 + cc, m_rows, tw, xg, gbar);
        }
      } else {
        // a piece of a split tile: store it, then the last piece to arrive sums all of them
        const int which = (tile == first_tile) ? 0 : 1;
        float* mine = p.partial + (static_cast<size_t>(c) * 2 + which) * (BN * 128);
        for (int cc = c0; cc < c1; cc += 16) {
          float v[16];
          tmem_ld16(tb + cc, v);
#pragma unroll
          for (int q = 0; q < 16; ++q) mine[(cc + q) * 128 + t] = v[q];
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
        __threadfence();
        bar_any(false, kEpiAllBar, C::kEpiThreads);
        const int64_t x0 = static_cast<int64_t>(tile) * KB;
        const int c_first = sk_first_cta(x0, T, G);
        const int c_last = sk_first_cta(x0 + KB - 1, T, G);
        if (threadIdx.x == 0) {
          const int old = atomicAdd(&p.counters[tile], 1);
          s_flag[1] = (old == c_last - c_first) ? 1 : 0;
        }
        bar_any(false, kEpiAllBar, C::kEpiThreads);
        if (s_flag[1]) {
          __threadfence();
          for (int cc = c0; cc < c1; cc += 16) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = 0.f;
            for (int cp = c_first; cp <= c_last; ++cp) {
              const int wp = (tile == static_cast<int>(sk_lo(T, G, cp) / KB)) ? 0 : 1;
              const float* src = p.partial + (static_cast<size_t>(cp) * 2 + wp) * (BN * 128);
#pragma unroll
              for (int q = 0; q < 16; ++q) v[q] += __ldcg(src + (cc + q) * 128 + t);
            }
            epi_chunk<C::kXPitch>(e, v, t, lane, wq, n, act0 + cc, m_rows, tw, xg, gbar);
          }
          if (threadIdx.x == 0) p.counters[tile] = 0;
        }
        bar_any(false, kEpiAllBar, C::kEpiThreads);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) tmem_dealloc(tmem, C::kTmemCols);
}

__global__ void lmhead_combine_kernel(const float4* __restrict__ part, int n_vtiles, int rows_cap,
                                      const int* rows_dev, const int* out_index, float* conf, int* amax,
                                      float* lse) {
  pdl_trigger();
  pdl_wait();
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
    if (BI == 0x7fffffff) {   // no finite logit: report it, and never hand on an invalid token id
      set_dev_status(DLLM_DEV_BAD_INDEX);
      BI = 0;
    }
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
int encode_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
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

// Tensor maps are pure functions of (address, shape, box); the step issues the same few
// hundred of them every denoising step, so they are encoded once and reused.
struct TmapKey {
  const void* base;
  int64_t rows, cols;
  int box;
  bool operator==(const TmapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && box == o.box;
  }
};
struct TmapKeyHash {
  size_t operator()(const TmapKey& k) const {
    size_t h = reinterpret_cast<size_t>(k.base);
    h ^= static_cast<size_t>(k.rows) * 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
    h ^= static_cast<size_t>(k.cols) * 0xc2b2ae3d27d4eb4full + (h << 6) + (h >> 2);
    h ^= static_cast<size_t>(k.box) + (h << 6) + (h >> 2);
    return h;
  }
};

}  // namespace

// Cached tensor-map encoding (also used by the fused layer kernel).
int make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  static std::mutex mu;
  static std::unordered_map<TmapKey, CUtensorMap, TmapKeyHash> cache;
  const TmapKey key{base, rows, cols, box_rows};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *m = it->second;
      return DLLM_OK;
    }
  }
  const int rc = encode_tmap(m, base, rows, cols, box_rows);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() > 8192) cache.clear();
  cache.emplace(key, *m);
  return DLLM_OK;
}

namespace {

// Activation-tile width.  Up to 512 rows the 128-wide tile: it keeps twice the weight bytes
// in flight per stage (two 64-column k-blocks: 96 KB of weights in the ring against 64 KB at
// 256 wide) and fills more SMs with whole tiles.  Above, the 256-wide tile halves the weight
// tile rereads and the shared-memory operand traffic per MMA (LLaDA-8B shapes, 128 vs 256 wide:
// QKV 84 vs 71 us at 640 rows, 88 vs 75 us at 768; gate/up + SwiGLU 147 vs 126 and 156 vs 131 us;
// the 768-row layer over 2048 positions 452 -> 408 us).  Gate/up goes wide from 385 rows (below).
int pick_bn(int rows) {
  static const int wide = [] {
    const char* e = getenv("DLLM_GEMM_WIDE_BN");   // A/B switch for measurements: width above 64 rows
    return e ? atoi(e) : 0;
  }();
  if (rows <= 16) return 16;
  if (rows <= 32) return 32;
  if (rows <= 64) return 64;
  if (wide == 128 || wide == 256) return wide;
  if (rows <= 512) return 128;
  return 256;
}
// Weight tile fastest up to 8 activation tiles (whole 768-row layers: 583 us against 638 us
// activation tile fastest; 2048 rows: 1.68 -> 1.57 ms), activation tile fastest above
// (batch-8 SureLock steps, 12288 rows: the vocabulary projection reads its 1.09 GB once).
constexpr int kMaxActTilesWtFastest = 8;

// Grid of the persistent kernel: one CTA per SM, never more CTAs than k-block iterations.
int pick_grid(int tiles, int KB) {
  const int64_t T = static_cast<int64_t>(tiles) * KB;
  return static_cast<int>(std::min<int64_t>(num_sms(), T));
}

// Grid for 128- and 256-wide activation tiles: every CTA takes whole tiles, or one of p equal
// pieces of a tile (p divides the k blocks, a piece at least 32 of them), never the uneven
// stream-K share, whose split tiles cost a partial-sum round trip and a serial fix-up at the
// end.  Measured (LLaDA-8B shapes): at 65-128 rows QKV 39.7 -> 24.7 us (96 tiles, 96 CTAs),
// O 29.7 -> 20.3 us (32 CTAs), down 40.8 -> 33.5 us (3 pieces of 32 tiles), gate/up 54.1 ->
// 46.3 us (2 of 192 tiles per CTA); a whole 768-row layer 507 -> 441 us; O at 1536 rows 101 ->
// 69 us.
// Above kMaxWholePerCta tiles per CTA the stream-K share wins (0 returned) unless rounding up
// to whole tiles costs under a quarter tile per CTA: its two split tiles per CTA cost little
// against many whole ones, while the rounding idles SMs (Dream-7B O at 12288 rows: 1344 tiles
// on 135 CTAs of 10; batch-8 SureLock step 223 -> 244 ms with whole tiles at any count).
constexpr int kMaxWholePerCta = 4;
int whole_piece_grid(int tiles, int KB) {
  const int sms = num_sms();
  if (tiles >= sms) {
    const int per = (tiles + sms - 1) / sms;
    if (per > kMaxWholePerCta && 4 * (static_cast<int64_t>(per) * sms - tiles) >= sms) return 0;
    return (tiles + per - 1) / per;
  }
  int p = std::max(1, std::min(sms / tiles, KB / 32));
  while (p > 1 && KB % p) --p;
  return tiles * p;
}

template <int BN, int KSUB, bool BIG>
int launch_cfg2(const CUtensorMap& tmW, const CUtensorMap& tmX, KParams& kp, int grid, cudaStream_t st) {
  using C = Cfg<BN, KSUB, BIG>;
  const int rc = ensure_smem_attr(reinterpret_cast<const void*>(gemm_tc_kernel<BN, KSUB, BIG>),
                                  static_cast<int>(C::kSmem));
  if (rc) return rc;
  return launch_pdl(gemm_tc_kernel<BN, KSUB, BIG>, dim3(grid), dim3(C::kThreads), C::kSmem, st, tmW, tmX, kp);
}

template <int BN, int KSUB>
int launch_cfg(const CUtensorMap& tmW, const CUtensorMap& tmX, KParams& kp, int grid, cudaStream_t st) {
  static const bool big = getenv("DLLM_GEMM_BIGRING") != nullptr;   // A/B switch for measurements
  if constexpr (BN <= 64) {
    if (big) return launch_cfg2<BN, KSUB, true>(tmW, tmX, kp, grid, st);
  }
  return launch_cfg2<BN, KSUB, false>(tmW, tmX, kp, grid, st);
}

// Widest KSUB whose two-stage ring still fits shared memory for this tile width.
constexpr int max_ksub(int bn) { return bn <= 64 ? 4 : (bn <= 128 ? 2 : 1); }

template <int BN>
int launch_bn(const CUtensorMap& tmW, const CUtensorMap& tmX, KParams& kp, int grid, int ksub, cudaStream_t st) {
  if constexpr (max_ksub(BN) >= 4) {
    if (ksub >= 4) return launch_cfg<BN, 4>(tmW, tmX, kp, grid, st);
  }
  if constexpr (max_ksub(BN) >= 2) {
    if (ksub >= 2) return launch_cfg<BN, 2>(tmW, tmX, kp, grid, st);
  }
  return launch_cfg<BN, 1>(tmW, tmX, kp, grid, st);
}

// k blocks fetched per pipeline stage: consecutive 128-byte pieces of every weight row are
// requested together, so each DRAM page opened for a row serves several of them.
int pick_ksub(int K, int bn) {
  const char* env = getenv("DLLM_GEMM_KSUB");
  const int KB = K / kBK;
  int want = std::min(env ? atoi(env) : 4, max_ksub(bn));
  for (int k : {4, 2, 1})
    if (k <= want && KB % k == 0) return k;
  return 1;
}

}  // namespace

size_t gemm_partial_floats(int rows_cap, int n_tiles_w, int K) {
  (void)n_tiles_w;
  (void)K;
  const int bn = pick_bn(rows_cap);
  return static_cast<size_t>(num_sms()) * 2 * bn * 128;
}

int gemm_counters_needed(int rows_cap, int n_tiles_w) {
  const int bn = pick_bn(rows_cap);
  return n_tiles_w * ((rows_cap + bn - 1) / bn);
}

int gemm_launch(const GemmArgs& a, const GemmScratch& s, cudaStream_t st, int force_grid, int force_bn) {
  if (a.K <= 0 || a.K % kBK != 0 || a.rows_cap <= 0 || a.n_tiles_w <= 0) return DLLM_ERR_SHAPE;
  int bn = force_bn ? force_bn : pick_bn(a.rows_cap);
  // 129-256 rows as one 256-wide activation tile when the caller allows it (QKV at 205 rows:
  // 41.6 -> 32.3 us; gate/up, O and down are not faster that way)
  if (!force_bn && a.wide_ok && bn == 128 && a.rows_cap > 128 && a.rows_cap <= 256) bn = 256;
  // gate/up + SwiGLU at 385-512 rows: two 256-wide tiles beat three or four 128-wide ones
  // (512 rows: 115.6 -> 98.3 us; at 384 rows 85.3 against 93.7 us the narrow tile still wins)
  if (!force_bn && a.swiglu && bn == 128 && a.rows_cap > 384) bn = 256;
  // O and down (residual add): when 128-wide tiles outnumber the SMs, so that a CTA takes two
  // or more of them anyway, one 256-wide tile per weight tile instead (768 rows: O 44.6 ->
  // 40.4 us, down 106 -> 90 us; at 384-512 rows the 128-wide tiles fill more SMs and win)
  if (!force_bn && a.epi.kind == EPI_RESID_ADD && bn == 128 &&
      static_cast<int64_t>(a.n_tiles_w) * ((a.rows_cap + 127) / 128) > num_sms())
    bn = 256;
  if (bn != 16 && bn != 32 && bn != 64 && bn != 128 && bn != 256) return DLLM_ERR_INVALID_ARG;
  const int tiles_act = (a.rows_cap + bn - 1) / bn;
  const int tiles = a.n_tiles_w * tiles_act;
  const int ksub = pick_ksub(a.K, bn);
  const int KB = a.K / (kBK * ksub);
  int grid = force_grid > 0 ? force_grid : pick_grid(tiles, KB);
  // The residual add is a reduction: when whole tiles would leave more than half the SMs idle
  // (O and down at 65-256 rows: 32 or 64 tiles), each piece of a split tile adds its own partial
  // sums into h, so the stream-K share over every SM needs no partial buffer and no fix-up
  // (layers over 2048 positions: 65 rows 179 -> 161 us, 205 rows 240 -> 228 us; with 96 or 512
  // tiles the extra reductions cost more than they gain: 384 rows 288 -> 298 us).  Narrower
  // tiles keep the fixed-order fix-up, so layers of up to 64 rows stay bit-reproducible.
  const bool add_pieces = a.epi.kind == EPI_RESID_ADD && bn >= 128 && 2 * tiles <= num_sms();
  if (force_grid <= 0 && bn >= 128 && !add_pieces) {
    const int wg = whole_piece_grid(tiles, KB);
    if (wg > 0) grid = wg;
  }
  grid = static_cast<int>(std::min<int64_t>(grid, static_cast<int64_t>(tiles) * KB));
  // split tiles need the partial buffer and one counter per tile; without them every
  // CTA takes whole tiles only (grid = number of tiles divides the work exactly)
  const size_t need = static_cast<size_t>(grid) * 2 * bn * 128;
  if (!add_pieces && (!s.partial || s.partial_floats < need || !s.counters || s.n_counters < tiles)) {
    if (static_cast<int64_t>(tiles) * KB % grid != 0 || tiles % grid != 0) grid = std::min(grid, tiles);
    while (grid > 1 && tiles % grid != 0) --grid;
  }
  CUtensorMap tmW, tmX;
  int rc = make_tmap(&tmW, a.W, a.w_rows_total, a.K, a.swiglu ? 64 : 128);
  if (rc) return rc;
  rc = make_tmap(&tmX, a.X, a.rows_cap, a.K, bn);
  if (rc) return rc;
  KParams kp;
  kp.K = a.K;
  kp.rows_cap = a.rows_cap;
  kp.rows_dev = a.rows_dev;
  kp.n_tiles_w = a.n_tiles_w;
  kp.tiles_act = tiles_act;
  static const int order_env = [] {
    const char* e = getenv("DLLM_GEMM_ORDER");   // A/B switch for measurements: 0 activation, 1 weight tile fastest
    return e ? atoi(e) : -1;
  }();
  kp.wt_fastest = order_env >= 0 ? order_env : (tiles_act <= kMaxActTilesWtFastest ? 1 : 0);
  kp.add_pieces = add_pieces ? 1 : 0;
  kp.swiglu = a.swiglu ? 1 : 0;
  kp.ffn = a.epi.ffn;
  kp.partial = s.partial;
  kp.counters = s.counters;
  kp.epi = a.epi;
  switch (bn) {
    case 16: return launch_bn<16>(tmW, tmX, kp, grid, ksub, st);
    case 32: return launch_bn<32>(tmW, tmX, kp, grid, ksub, st);
    case 64: return launch_bn<64>(tmW, tmX, kp, grid, ksub, st);
    case 128: return launch_bn<128>(tmW, tmX, kp, grid, ksub, st);
    default: return launch_bn<256>(tmW, tmX, kp, grid, ksub, st);
  }
}

int lmhead_combine_launch(const float4* part, int n_vtiles, int rows_cap, const int* rows_dev,
                          const int* out_index, float* conf, int* amax, float* lse, cudaStream_t st) {
  if (rows_cap <= 0) return DLLM_OK;
{
    const int rc_ = launch_pdl(  lmhead_combine_kernel, dim3(rows_cap), dim3(256), 0, st, part, n_vtiles, rows_cap, rows_dev, out_index, conf, amax, lse);
    if (rc_) return rc_;
  }
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
