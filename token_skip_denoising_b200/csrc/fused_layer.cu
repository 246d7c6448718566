// One transformer layer for a few recomputed rows as a single persistent kernel.
//
// With at most 32 active rows (the ES-dLLM skip step: the block's rows below the
// skip layer, the kept rows above it) a layer is four weight streams (QKV, O,
// gate/up, down: 436 MB for the LLaDA-8B shape) separated by small dependent
// steps (RMSNorm, attention over the cached K/V, the merge of split attention
// partials).  As separate kernels each weight stream pays a pipeline fill and
// drain.  Here one CTA per SM runs the whole layer:
//   warp 4 (TMA producer) streams the weight tiles of all four GEMMs through one
//     ring without draining between them; the activation tiles of a GEMM are
//     requested only once its input is complete (grid-wide counters);
//   warp 5 (MMA issuer) accumulates into two TMEM buffers;
//   warps 0-3 run the GEMM epilogues and, between GEMMs, the RMSNorm rows, the
//     attention items and the split merge, signalling each phase on a counter.
// Every cross-CTA wait is bounded; on expiry the kernel records a timeout in the
// device status word and every role stops.
#include <algorithm>

#include "attn_dev.cuh"
#include "common.cuh"
#include "gemm_dev.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace dllm {

int make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows);

namespace {

using namespace gemm;

constexpr int kThreads = 192;
constexpr uint32_t kSpinLimit = 1u << 22;

enum Phase : int { S_NORM1 = 0, S_QKV, S_ATTN, S_COMB, S_O, S_NORM2, S_GU, S_DOWN, S_COUNT };

template <int BN, int KSUB>
struct FCfg {
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStageBytes = KSUB * (kABytes + kBBytes);
  static constexpr int kFit = static_cast<int>((144u * 1024u) / kStageBytes);
  static constexpr int kStages = kFit > 12 ? 12 : (kFit < 2 ? 2 : kFit);
  static constexpr uint32_t kAccCols = BN < 32 ? 32 : BN;
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static constexpr int kXPitch = 17;
  static constexpr size_t kAttnBytes = 4 * 64 * 128 * 2;   // K/V double buffer for hd <= 128
  static constexpr size_t kSmem = 1024 + kStages * kStageBytes + kAttnBytes + 128 * kXPitch * 4 +
                                  (2 * kStages + 4) * 8 + 64;
  static_assert(kSmem <= 227 * 1024, "fused layer does not fit shared memory");
};

struct FGemm {
  int K;
  int n_tiles;            // output tiles (SwiGLU: F / 64)
  int swiglu, ffn;
  int wait_slot;          // phase whose completion the activation operand needs
  int done_slot;          // phase signalled when this GEMM's tiles are final
  EpiParams epi;
  float* partial;         // [gridDim.x][2][BN * 128]
  int* counters;          // [n_tiles], zero between launches
};

struct FParams {
  FGemm gm[4];
  int rows_cap;
  const int* n_rows;      // device count of the rows
  const int* rows;        // row j -> flat b * N + pos
  int d;
  float eps;
  const float* g_attn;
  const float* g_ffn;
  float* h;               // position-indexed fp32 hidden
  __nv_bfloat16* z1;      // [rows_cap, d]  RMSNorm before attention (QKV operand)
  __nv_bfloat16* z2;      // [rows_cap, d]  RMSNorm before the FFN (gate/up operand)
  attn::AttnParams ap;    // q, caches, out (O operand), seq_off, split partials
  int attn_qtiles;
  int attn_items;
  int* sync;              // [S_COUNT] phase counters + [S_COUNT] exit counter, zero at launch
  int target;             // gridDim.x: every CTA signals each phase once
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Bounded wait until counter >= target.
__device__ __forceinline__ bool wait_count(const int* ctr, int target, volatile int* abort) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (ld_acquire(ctr) >= target) return true;
    if (*abort) return false;
    __nanosleep(64);
  }
  set_dev_status(DLLM_DEV_TIMEOUT);
  *abort = 1;
  return false;
}

// The 128 epilogue threads wait for a phase of every CTA: thread 0 polls, the barrier
// vote hands the outcome to all of them (true: go on).
__device__ __forceinline__ bool epi_wait_phase(const int* ctr, int target, volatile int* abort, int tid) {
  const bool ok = tid == 0 ? wait_count(ctr, target, abort) : true;
  const bool stop = epi_any(!ok || *abort);
  if (!stop) __threadfence();
  return !stop;
}

// The 128 epilogue threads publish a finished phase: every thread's writes are made
// visible, then one thread bumps the counter.
__device__ __forceinline__ void signal_phase(int* ctr, int tid) {
  __threadfence();
  fence_proxy_async();
  epi_bar();
  if (tid == 0) atomicAdd(ctr, 1);
}

// RMSNorm of one row by the 128 epilogue threads.
__device__ __forceinline__ void norm_row(const float* __restrict__ x, const float* __restrict__ g, float eps, int d,
                                         __nv_bfloat16* __restrict__ out, int tid, float* red) {
  float ss = 0.f;
  for (int i = tid * 4; i < d; i += 512) {
    const float4 v = *reinterpret_cast<const float4*>(x + i);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  if ((tid & 31) == 0) red[tid >> 5] = ss;
  epi_bar();
  const float r = rsqrtf((red[0] + red[1] + red[2] + red[3]) / static_cast<float>(d) + eps);
  for (int i = tid * 4; i < d; i += 512) {
    const float4 v = *reinterpret_cast<const float4*>(x + i);
    const float4 gg = *reinterpret_cast<const float4*>(g + i);
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x * r * gg.x, v.y * r * gg.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z * r * gg.z, v.w * r * gg.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&a);
    pk.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(out + i) = pk;
  }
  epi_bar();
}

struct NamedBar {
  __device__ __forceinline__ void operator()() const { epi_bar(); }
};

template <int BN, int KSUB>
__global__ void __launch_bounds__(kThreads, 1)
fused_layer_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                   const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmW3,
                   const __grid_constant__ CUtensorMap tmX0, const __grid_constant__ CUtensorMap tmX1,
                   const __grid_constant__ CUtensorMap tmX2, const __grid_constant__ CUtensorMap tmX3, FParams p) {
  using C = FCfg<BN, KSUB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* attn_smem = smem + C::kStages * C::kStageBytes;
  float* xbuf = reinterpret_cast<float*>(attn_smem + C::kAttnBytes);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(xbuf + 128 * C::kXPitch);
  uint64_t* empty_bar = full_bar + C::kStages;
  uint64_t* acc_full = empty_bar + C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);   // [0] abort, [1] last piece

  const CUtensorMap* tmW[4] = {&tmW0, &tmW1, &tmW2, &tmW3};
  const CUtensorMap* tmX[4] = {&tmX0, &tmX1, &tmX2, &tmX3};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int c = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int q = 0; q < 4; ++q) {
      tma_prefetch_desc(tmW[q]);
      tma_prefetch_desc(tmX[q]);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    s_flag[0] = 0;
    s_flag[1] = 0;
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- producer: every GEMM's weight tiles through one ring
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int i = 0;
      for (int g = 0; g < 4 && !s_flag[0]; ++g) {
        const FGemm& gm = p.gm[g];
        const int KB = gm.K / (kBK * KSUB);
        const int64_t T = static_cast<int64_t>(gm.n_tiles) * KB;
        const int64_t lo = sk_lo(T, G, c), hi = sk_lo(T, G, c + 1);
        bool ready = false;
        int pend_s[C::kStages], pend_x[C::kStages], n_pend = 0, pend_first = 0;
        auto flush = [&]() {
          fence_proxy_async();
          for (int q = 0; q < n_pend; ++q) {
            uint8_t* bx = stage_base + pend_s[q] * C::kStageBytes + KSUB * kABytes;
#pragma unroll
            for (int sub = 0; sub < KSUB; ++sub)
              tma_load_2d(bx + sub * C::kBBytes, tmX[g], &full_bar[pend_s[q]], pend_x[q] + sub * kBK, 0, pol_x);
          }
          n_pend = 0;
          ready = true;
        };
        for (int64_t it = lo; it < hi && !s_flag[0];) {
          const int tile = static_cast<int>(it / KB);
          const int kb0 = static_cast<int>(it % KB);
          const int kb1 = (hi - it < KB - kb0) ? kb0 + static_cast<int>(hi - it) : KB;
          it += kb1 - kb0;
          const int row0 = gm.swiglu ? tile * 64 : tile * kTileM;
          const int row1 = gm.swiglu ? gm.ffn + tile * 64 : tile * kTileM + 64;
          for (int kb = kb0; kb < kb1; ++kb, ++i) {
            const int s = i % C::kStages;
            const uint32_t ph = (i / C::kStages) & 1;
            if (!ready && n_pend > 0 && i - C::kStages >= pend_first) {
              // the stage to reuse still waits for its activation tile
              if (!wait_count(p.sync + gm.wait_slot, p.target, s_flag)) break;
              flush();
            }
            if (!mbar_wait(&empty_bar[s], ph ^ 1)) { s_flag[0] = 1; break; }
            uint8_t* a = stage_base + s * C::kStageBytes;
            mbar_arrive_expect_tx(&full_bar[s], C::kStageBytes);
#pragma unroll
            for (int sub = 0; sub < KSUB; ++sub) {
              const int x = (kb * KSUB + sub) * kBK;
              tma_load_2d(a + sub * kABytes, tmW[g], &full_bar[s], x, row0, pol_w);
              tma_load_2d(a + sub * kABytes + kABytes / 2, tmW[g], &full_bar[s], x, row1, pol_w);
            }
            if (!ready && ld_acquire(p.sync + gm.wait_slot) >= p.target) flush();
            if (ready) {
              uint8_t* bx = a + KSUB * kABytes;
#pragma unroll
              for (int sub = 0; sub < KSUB; ++sub)
                tma_load_2d(bx + sub * C::kBBytes, tmX[g], &full_bar[s], (kb * KSUB + sub) * kBK, 0, pol_x);
            } else {
              if (n_pend == 0) pend_first = i;
              pend_s[n_pend] = s;
              pend_x[n_pend] = kb * KSUB * kBK;
              ++n_pend;
            }
          }
        }
        if (!ready && n_pend > 0 && !s_flag[0]) {
          if (wait_count(p.sync + gm.wait_slot, p.target, s_flag)) flush();
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = make_idesc_bf16(kTileM, BN);
      int i = 0, j = 0;
      for (int g = 0; g < 4 && !s_flag[0]; ++g) {
        const FGemm& gm = p.gm[g];
        const int KB = gm.K / (kBK * KSUB);
        const int64_t T = static_cast<int64_t>(gm.n_tiles) * KB;
        const int64_t lo = sk_lo(T, G, c), hi = sk_lo(T, G, c + 1);
        for (int64_t it = lo; it < hi && !s_flag[0];) {
          const int kb0 = static_cast<int>(it % KB);
          const int kb1 = (hi - it < KB - kb0) ? kb0 + static_cast<int>(hi - it) : KB;
          it += kb1 - kb0;
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
    }
  } else {
    // ---------------- warps 0-3: epilogues and the steps between GEMMs
    const int t = threadIdx.x;
    const int m_rows = min(*p.n_rows, p.rows_cap);
    float* red = xbuf;
    int j = 0;
    auto gemm_epilogues = [&](int g) {
      const FGemm& gm = p.gm[g];
      const EpiParams& e = gm.epi;
      const int KB = gm.K / (kBK * KSUB);
      const int64_t T = static_cast<int64_t>(gm.n_tiles) * KB;
      const int64_t lo = sk_lo(T, G, c), hi = sk_lo(T, G, c + 1);
      const int first_tile = static_cast<int>(lo / KB);
      for (int64_t it = lo; it < hi;) {
        const int tile = static_cast<int>(it / KB);
        const int kb0 = static_cast<int>(it % KB);
        const int kb1 = (hi - it < KB - kb0) ? kb0 + static_cast<int>(hi - it) : KB;
        it += kb1 - kb0;
        const int b = j & 1;
        const uint32_t u = static_cast<uint32_t>(j >> 1);
        ++j;
        const bool late = !mbar_wait(&acc_full[b], u & 1);
        if (epi_any(late || s_flag[0])) {              // one decision for all epilogue threads
          s_flag[0] = 1;
          return;
        }
        tc_fence_after();
        const uint32_t tb = tmem + (static_cast<uint32_t>(warp * 32) << 16) + b * C::kAccCols;
        const int row0 = gm.swiglu ? tile * 64 : tile * kTileM;
        const int row1 = gm.swiglu ? gm.ffn + tile * 64 : tile * kTileM + 64;
        const int n = t < 64 ? row0 + t : row1 + (t - 64);
        if (kb0 == 0 && kb1 == KB) {
          for (int cc = 0; cc < BN; cc += 16) {
            float v[16];
            tmem_ld16(tb + cc, v);
            if (cc + 16 >= BN) {
              tc_fence_before();
              mbar_arrive(&acc_empty[b]);
            }
            epi_chunk<C::kXPitch>(e, v, t, lane, warp, n, cc, m_rows, tile, xbuf);
          }
        } else {
          const int which = (tile == first_tile) ? 0 : 1;
          float* mine = gm.partial + (static_cast<size_t>(c) * 2 + which) * (BN * 128);
          for (int cc = 0; cc < BN; cc += 16) {
            float v[16];
            tmem_ld16(tb + cc, v);
#pragma unroll
            for (int q = 0; q < 16; ++q) mine[(cc + q) * 128 + t] = v[q];
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[b]);
          __threadfence();
          epi_bar();
          const int64_t x0 = static_cast<int64_t>(tile) * KB;
          const int c_first = sk_first_cta(x0, T, G);
          const int c_last = sk_first_cta(x0 + KB - 1, T, G);
          if (t == 0) s_flag[1] = (atomicAdd(&gm.counters[tile], 1) == c_last - c_first) ? 1 : 0;
          epi_bar();
          if (s_flag[1]) {
            __threadfence();
            for (int cc = 0; cc < BN; cc += 16) {
              float v[16];
#pragma unroll
              for (int q = 0; q < 16; ++q) v[q] = 0.f;
              for (int cp = c_first; cp <= c_last; ++cp) {
                const int wp = (tile == static_cast<int>(sk_lo(T, G, cp) / KB)) ? 0 : 1;
                const float* src = gm.partial + (static_cast<size_t>(cp) * 2 + wp) * (BN * 128);
#pragma unroll
                for (int q = 0; q < 16; ++q) v[q] += __ldcg(src + (cc + q) * 128 + t);
              }
              epi_chunk<C::kXPitch>(e, v, t, lane, warp, n, cc, m_rows, tile, xbuf);
            }
            if (t == 0) gm.counters[tile] = 0;
          }
          epi_bar();
        }
      }
    };

    // RMSNorm before attention
    for (int r = c; r < m_rows; r += G) norm_row(p.h + static_cast<int64_t>(p.rows[r]) * p.d, p.g_attn, p.eps, p.d,
                                                 p.z1 + static_cast<int64_t>(r) * p.d, t, red);
    signal_phase(p.sync + S_NORM1, t);
    gemm_epilogues(0);                                             // QKV (+RoPE, K/V scatter)
    signal_phase(p.sync + S_QKV, t);
    // attention items over the cached K/V (the new rows are in the cache now)
    if (epi_wait_phase(p.sync + S_QKV, p.target, s_flag, t)) {
      for (int it = c; it < p.attn_items; it += G) {
        int rem = it;
        const int split = rem % p.ap.splits;
        rem /= p.ap.splits;
        const int qt = rem % p.attn_qtiles;
        rem /= p.attn_qtiles;
        const int kvh = rem % p.ap.Hkv;
        const int b = rem / p.ap.Hkv;
        if (p.gm[0].epi.head_dim == 128) attn::attn_item<128>(p.ap, qt, b, kvh, split, attn_smem, t, NamedBar{});
        else attn::attn_item<64>(p.ap, qt, b, kvh, split, attn_smem, t, NamedBar{});
        epi_bar();
      }
    }
    signal_phase(p.sync + S_ATTN, t);
    // merge of the split partials: one warp per (row, head)
    if (p.ap.splits > 1 && epi_wait_phase(p.sync + S_ATTN, p.target, s_flag, t)) {
      const int units = m_rows * p.ap.Hq;
      for (int uu = c * 4 + warp; uu < units; uu += G * 4) {
        if (p.gm[0].epi.head_dim == 128) attn::attn_merge<128>(p.ap, uu / p.ap.Hq, uu % p.ap.Hq, lane);
        else attn::attn_merge<64>(p.ap, uu / p.ap.Hq, uu % p.ap.Hq, lane);
      }
    }
    signal_phase(p.sync + S_COMB, t);
    gemm_epilogues(1);                                             // O (+residual)
    signal_phase(p.sync + S_O, t);
    // RMSNorm before the FFN
    if (epi_wait_phase(p.sync + S_O, p.target, s_flag, t)) {
      for (int r = c; r < m_rows; r += G) norm_row(p.h + static_cast<int64_t>(p.rows[r]) * p.d, p.g_ffn, p.eps, p.d,
                                                   p.z2 + static_cast<int64_t>(r) * p.d, t, red);
    }
    signal_phase(p.sync + S_NORM2, t);
    gemm_epilogues(2);                                             // gate/up (+SwiGLU)
    signal_phase(p.sync + S_GU, t);
    gemm_epilogues(3);                                             // down (+residual)
    signal_phase(p.sync + S_DOWN, t);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, C::kTmemCols);
  // the last CTA out clears the counters, so every launch (a graph replay too) starts from zero
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sync + S_COUNT, 1) == G - 1) {
      for (int q = 0; q <= S_COUNT; ++q) atomicExch(p.sync + q, 0);
      __threadfence();
    }
  }
}

template <int BN, int KSUB>
int launch_fused(const CUtensorMap (&tw)[4], const CUtensorMap (&tx)[4], const FParams& p, int grid, cudaStream_t st) {
  using C = FCfg<BN, KSUB>;
  static bool attr_done = false;
  if (!attr_done) {
    DLLM_CUDA_TRY(cudaFuncSetAttribute(fused_layer_kernel<BN, KSUB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem)));
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the phase counters are grid-wide
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fused_layer_kernel<BN, KSUB>, tw[0], tw[1], tw[2], tw[3], tx[0],
                                           tx[1], tx[2], tx[3], p);
  count_launch();
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e), __FILE__, __LINE__);
    return DLLM_ERR_CUDA;
  }
  return DLLM_OK;
}

}  // namespace

size_t fused_partial_floats(int rows_cap) {
  const int bn = rows_cap <= 16 ? 16 : 32;
  return static_cast<size_t>(4) * kNumSMs * 2 * bn * 128;
}

int fused_layer_launch(const FusedLayerArgs& a, cudaStream_t st) {
  if (a.rows_cap <= 0 || a.rows_cap > 32) return DLLM_ERR_UNSUPPORTED;
  const int bn = a.rows_cap <= 16 ? 16 : 32;
  const int ksub = bn == 16 ? 4 : 2;
  if (a.d % (64 * ksub) || a.qd % (64 * ksub) || a.F % (64 * ksub) || a.hd > 128) return DLLM_ERR_UNSUPPORTED;
  const int grid = kNumSMs;
  CUtensorMap tw[4], tx[4];
  const void* W[4] = {a.Wqkv, a.Wo, a.Wgu, a.Wdn};
  const int64_t wrows[4] = {a.qkvd, a.d, 2LL * a.F, a.d};
  const int K[4] = {a.d, a.qd, a.d, a.F};
  const void* X[4] = {a.z1, a.attn, a.z2, a.act};
  for (int q = 0; q < 4; ++q) {
    int rc = make_tmap(&tw[q], W[q], wrows[q], K[q], 64);
    if (rc) return rc;
    rc = make_tmap(&tx[q], X[q], a.rows_cap, K[q], bn);
    if (rc) return rc;
  }
  FParams p;
  const int n_tiles[4] = {a.qkvd / 128, a.d / 128, a.F / 64, a.d / 128};
  const int waits[4] = {S_NORM1, S_COMB, S_NORM2, S_GU};
  const int dones[4] = {S_QKV, S_O, S_GU, S_DOWN};
  for (int q = 0; q < 4; ++q) {
    FGemm& g = p.gm[q];
    g.K = K[q];
    g.n_tiles = n_tiles[q];
    g.swiglu = q == 2;
    g.ffn = a.F;
    g.wait_slot = waits[q];
    g.done_slot = dones[q];
    g.partial = a.partial + static_cast<size_t>(q) * kNumSMs * 2 * bn * 128;
    g.counters = a.tile_counters + q * a.max_tiles;
  }
  EpiParams& e0 = p.gm[0].epi;
  e0.kind = EPI_QKV_ROPE; e0.q_out = a.q; e0.kcache = a.kc; e0.vcache = a.vc; e0.row_map = a.rows;
  e0.seq_n = a.N; e0.n_kv = a.Hkv; e0.head_dim = a.hd; e0.q_dim = a.qd; e0.kv_dim = a.kvd;
  e0.rope_cos = a.rope_cos; e0.rope_sin = a.rope_sin;
  EpiParams& e1 = p.gm[1].epi;
  e1.kind = EPI_RESID_ADD; e1.h = a.h; e1.ldh = a.d; e1.row_map = a.rows; e1.head_dim = a.hd;
  EpiParams& e2 = p.gm[2].epi;
  e2.kind = EPI_SWIGLU; e2.act = a.act; e2.ffn = a.F; e2.head_dim = a.hd;
  EpiParams& e3 = p.gm[3].epi;
  e3.kind = EPI_RESID_ADD; e3.h = a.h; e3.ldh = a.d; e3.row_map = a.rows; e3.head_dim = a.hd;
  p.rows_cap = a.rows_cap;
  p.n_rows = a.n_rows;
  p.rows = a.rows;
  p.d = a.d;
  p.eps = a.eps;
  p.g_attn = a.g_attn;
  p.g_ffn = a.g_ffn;
  p.h = a.h;
  p.z1 = a.z1;
  p.z2 = a.z2;
  // attention work: every (sequence, KV head, query tile, key split) item
  const int Gq = a.Hq / a.Hkv;
  const int units = a.rows_per_seq * Gq;
  const int qtiles = (units + 63) / 64;
  const int n_blocks = (a.N + 63) / 64;
  int splits = std::max(1, std::min(n_blocks, (2 * kNumSMs + a.B * a.Hkv * qtiles - 1) / (a.B * a.Hkv * qtiles)));
  const int bps = (n_blocks + splits - 1) / splits;
  splits = (n_blocks + bps - 1) / bps;
  if (static_cast<size_t>(splits) * a.rows_cap * a.Hq * a.hd > a.attn_floats) return DLLM_ERR_SHAPE;
  attn::AttnParams& ap = p.ap;
  ap.q = a.q; ap.kc = a.kc; ap.vc = a.vc; ap.out = a.attn; ap.seq_off = a.seq_off;
  ap.B = a.B; ap.N = a.N; ap.Hq = a.Hq; ap.Hkv = a.Hkv; ap.rows_cap = a.rows_cap;
  ap.splits = splits; ap.blocks_per_split = bps;
  ap.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.hd));
  ap.opart = a.attn_opart; ap.ml = a.attn_ml;
  p.attn_qtiles = qtiles;
  p.attn_items = a.B * a.Hkv * qtiles * splits;
  p.sync = a.sync;
  p.target = grid;
  if (bn == 16) return launch_fused<16, 4>(tw, tx, p, grid, st);
  return launch_fused<32, 2>(tw, tx, p, grid, st);
}

}  // namespace dllm
