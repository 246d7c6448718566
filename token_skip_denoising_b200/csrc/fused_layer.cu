// A run of transformer layers for a few recomputed rows as a single persistent kernel.
//
// With at most 64 active rows (the ES-dLLM skip step: the block's rows below the
// skip layer, the kept rows above it) a layer is four weight streams (QKV, O,
// gate/up, down: 436 MB for the LLaDA-8B shape) separated by small dependent
// steps (RMSNorm, RoPE, attention over the cached K/V, the split merge, SwiGLU).
// One CTA per SM runs every layer of the run, so the weight stream never stops at
// a layer boundary:
//   warp 4 (TMA producer) streams the weight tiles of all four GEMMs through one
//     ring; the activation tiles of a GEMM are requested once its input is
//     complete (grid-wide phase counters).  At the start of each layer it
//     prefetches that layer's K/V cache into L2 for the attention step;
//   warp 5 (MMA issuer) accumulates each (weight tile, k range) piece into one of
//     two TMEM buffers;
//   warps 0-3 add every piece into an fp32 target with global reductions (the
//     residual stream h for O and down, row-major sums for QKV and gate/up), so no
//     piece waits for another, and between GEMMs run the elementwise steps spread
//     over the whole grid.  RMSNorm is a per-row scale, so the QKV and gate/up
//     operands are bf16(g * h) (each CTA also leaves its partial sums of h^2) and the
//     GEMM sums are multiplied by 1/rms afterwards, in the RoPE and SwiGLU steps.
//     Phases per layer, each a counter that grows by the grid size: operand g * h ->
//     QKV sums -> RoPE and K/V scatter -> attention (the last split of a query tile
//     merges the partials) -> O in h -> operand g * h -> gate/up sums -> SwiGLU ->
//     down in h.
//   With the ES-dLLM choice in the run (the top k at the skip layer, or again at the start
//   of every layer) two phases open each choosing layer: Eq. 1 for every candidate (one warp per row; a row the
//   previous layer skipped first takes its cached output) and the top k of each sequence
//   (one CTA per sequence, rank counting), which rewrites the row map the layer then uses.
// Every cross-CTA wait is bounded; on expiry the kernel records a timeout in the
// device status word and every role stops.
#include <algorithm>
#include <cstdlib>

#include "attn_dev.cuh"
#include "common.cuh"
#include "es_dev.cuh"
#include "gemm_dev.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace dllm {

int make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows);

namespace {

using namespace gemm;

constexpr int kThreads = 192;
constexpr int kKsub = 2;                          // 64-column k-blocks per ring stage
constexpr int kMaxRows = kFusedMaxRows;           // rows of the fp32 sum buffers (any launch's row count)
constexpr uint32_t kSpinLimit = 1u << 22;          // default polls of a grid-phase wait (~0.4 s)
constexpr size_t kMaxKvPrefetch = 64ull << 20;    // larger caches are not prefetched

enum Phase : int { S_X1 = 0, S_QKV, S_ROPE, S_COMB, S_O, S_X2, S_GU, S_SWIGLU, S_DOWN, S_SCORE, S_PICK, S_COUNT };
constexpr int S_ABORT = S_COUNT + 1;              // set by a CTA that gave up a wait
static_assert(S_ABORT + 1 <= kFusedSyncInts, "phase counters + exit counter + abort word");
static_assert(kMaxRows <= 128 && 128 % kMaxRows == 0, "rows are handled by the 128 step threads");

template <int BN>
struct FCfg {
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStageBytes = kKsub * (kABytes + kBBytes);
  static constexpr int kFit = static_cast<int>((160u * 1024u) / kStageBytes);
  static constexpr int kStages = kFit > 8 ? 8 : (kFit < 2 ? 2 : kFit);
  static constexpr uint32_t kAccCols = BN < 32 ? 32 : BN;
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static constexpr size_t kAttnBytes = 4 * 64 * 128 * 2;   // K/V double buffer for hd <= 128
  static constexpr size_t kMiscBytes = 4 * kMaxRows * 4;    // row map, 1/rms before attention and FFN, partial sums
  static constexpr size_t kSmem = 1024 + kStages * kStageBytes + kAttnBytes + kMiscBytes + (2 * kStages + 5) * 8 + 64;
  static_assert(kSmem <= 227 * 1024, "fused layer does not fit shared memory");
};

struct FGemm {
  int K;
  int n_tiles;            // 128-row weight tiles of one layer (the tensor map stacks every layer)
  int wait_slot;          // phase whose completion the activation operand needs
  float* out;             // out[row(j) * ldo + n] += (W X^T)[n][j]
  int ldo;
  int use_rows;           // row(j) = rows[j] (position-indexed h) or j
};

struct FParams {
  FGemm gm[4];
  int l0, n_layers;       // layers l0 .. l0 + n_layers - 1 of the stacks
  int rows_cap;
  const int* n_rows;      // device count of the rows
  const int* rows;        // row j -> flat b * N + pos
  int d;
  float eps;
  const float* g_attn;     // [L, d] (layer 0 of the stack)
  const float* g_ffn;
  float* h;               // position-indexed fp32 hidden
  __nv_bfloat16* z1;      // [rows_cap, d]  g_attn * h (QKV operand; 1/rms applied to the sums)
  __nv_bfloat16* z2;      // [rows_cap, d]  g_ffn * h (gate/up operand)
  float* s_qkv;           // [kMaxRows, qkvd] fp32 QKV sums
  float* s_gu;            // [kMaxRows, 2F]   fp32 gate/up sums
  float* ss1;             // [kMaxRows] sums of h^2 per row before attention (RMSNorm); zero
                          // between uses: CTA 0 clears it once every CTA has read it
  float* ss2;             // [kMaxRows] the same before the FFN
  int qkvd, qd, kvd, hd, Hkv, N, F;
  const float* rope_cos;
  const float* rope_sin;
  __nv_bfloat16* q;       // [rows_cap, qd] rotated queries (attention operand)
  __nv_bfloat16* kc;      // caches [L, B, Hkv, N, hd] (layer 0 of the stack)
  __nv_bfloat16* vc;
  int64_t kv_layer;       // elements of one layer's cache
  __nv_bfloat16* act;     // [rows_cap, F] SwiGLU output (down operand)
  size_t kv_bytes;        // bytes of each cache prefetched into L2 at a layer's start (0: none)
  attn::AttnParams ap;    // q, out (O operand), seq_off, split partials (caches set per layer)
  int attn_qtiles;
  int attn_items;
  int attn_group_merge;   // every item in one round: the splits of a group merge together
  int* attn_ctr;          // [B * Hkv * attn_qtiles] split arrivals, zero between uses
  int* sync;              // [S_COUNT] phase counters + exit counter + abort word, zero at launch
  FusedEs es;             // per-layer re-selection at the start of every layer (es.on)
  float* es_acc;          // [2 * B * n_cand] Eq. 1 sums of the candidates, zero between layers
  int n_attn_ctr;         // attention split counters (cleared after an aborted launch)
  uint32_t spin_limit;    // polls of a grid-phase wait before it gives up
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
               : "memory");
}

// The (tile, k-block) items of a GEMM that CTA c owns: a contiguous range of the
// tile-major item order, split evenly over min(items, grid) CTAs.
struct Items {
  int64_t lo, hi;
  int KB;
};
__device__ __forceinline__ Items items_of(int K, int n_tiles, int G, int c) {
  Items r;
  r.KB = K / (kBK * kKsub);
  const int64_t T = static_cast<int64_t>(n_tiles) * r.KB;
  const int Gg = static_cast<int>(T < G ? T : G);
  r.lo = c < Gg ? T * c / Gg : 0;
  r.hi = c < Gg ? T * (c + 1) / Gg : 0;
  return r;
}

// Bounded wait until counter >= target.  On expiry the CTA records the timeout, raises its
// abort flag and marks the launch aborted (the last CTA out then clears what an unfinished
// layer leaves behind).
__device__ __forceinline__ bool wait_count(const int* ctr, int target, volatile int* abort, uint32_t limit,
                                           int* abort_word) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (ld_acquire(ctr) >= target) return true;
    if (*abort) return false;
    __nanosleep(64);
  }
  set_dev_status(DLLM_DEV_TIMEOUT);
  *abort = 1;
  atomicExch(abort_word, 1);
  return false;
}

// Bounded wait on an mbarrier phase that also gives up as soon as the CTA's abort flag is up.
__device__ __forceinline__ bool mbar_wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31) == 31 && *abort) return false;
  }
  set_dev_status(DLLM_DEV_TIMEOUT);
  return false;
}

// The 128 epilogue threads wait for a phase of every CTA: thread 0 polls, the barrier
// vote hands the outcome to all of them (true: go on).
__device__ __forceinline__ bool epi_wait_phase(const int* ctr, int target, volatile int* abort, int tid,
                                               uint32_t limit, int* abort_word) {
  bool ok = true;
  if (tid == 0) {
    ok = wait_count(ctr, target, abort, limit, abort_word);
    __threadfence();
  }
  return !epi_any(!ok || *abort);   // the barrier orders the other threads' reads after the acquire
}

// The 128 epilogue threads publish a finished phase: their writes (for the TMA loads
// of other CTAs, through the async proxy too) are ordered before the barrier, and one
// thread's fence after it makes all of them visible before the counter moves.
__device__ __forceinline__ void signal_phase(int* ctr, int tid) {
  fence_proxy_async();
  epi_bar();
  if (tid == 0) {
    __threadfence();
    atomicAdd(ctr, 1);
  }
}

struct NamedBar {
  __device__ __forceinline__ void operator()() const { epi_bar(); }
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
fused_layer_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                   const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmW3,
                   const __grid_constant__ CUtensorMap tmX0, const __grid_constant__ CUtensorMap tmX1,
                   const __grid_constant__ CUtensorMap tmX2, const __grid_constant__ CUtensorMap tmX3, FParams p) {
  using C = FCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* attn_smem = smem + C::kStages * C::kStageBytes;
  int* s_rows = reinterpret_cast<int*>(attn_smem + C::kAttnBytes);   // [kMaxRows]
  float* s_rinv1 = reinterpret_cast<float*>(s_rows + kMaxRows);       // 1/rms before attention
  float* s_rinv2 = s_rinv1 + kMaxRows;                                // 1/rms before the FFN
  float* s_ss = s_rinv2 + kMaxRows;                                   // partial sums of squares
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(attn_smem + C::kAttnBytes + C::kMiscBytes);
  uint64_t* empty_bar = full_bar + C::kStages;
  uint64_t* acc_full = empty_bar + C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;                                 // every MMA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);   // [0] abort, [1] last split

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
    mbar_init(mma_done, 1);
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
      // ---------------- producer: every GEMM's weight tiles of every layer through one ring
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      Items R[4];
      for (int g = 0; g < 4; ++g) R[g] = items_of(p.gm[g].K, p.gm[g].n_tiles, G, c);
      int i = 0;
      for (int li = 0; li < p.n_layers && !s_flag[0]; ++li) {
        const int target = (li + 1) * G;
        // this layer's K/V cache into L2: its attention step reads all of it
        if (p.kv_bytes) {
          const size_t slice = ((p.kv_bytes + G - 1) / G + 15) & ~size_t(15);
          const size_t a0 = slice * c;
          const size_t a1 = a0 + slice < p.kv_bytes ? a0 + slice : p.kv_bytes;
          const size_t lo = static_cast<size_t>(p.l0 + li) * p.kv_layer * 2;
          for (size_t o = a0; o < a1; o += 32768) {
            const uint32_t n = static_cast<uint32_t>(a1 - o < 32768 ? a1 - o : 32768);
            prefetch_l2(reinterpret_cast<const uint8_t*>(p.kc) + lo + o, n);
            prefetch_l2(reinterpret_cast<const uint8_t*>(p.vc) + lo + o, n);
          }
        }
        // bounded wait for the activation operand of GEMM g of this layer (a grid phase)
        auto x_ready = [&](int g) -> bool { return ld_acquire(p.sync + p.gm[g].wait_slot) >= target; };
        auto wait_x = [&](int g) -> bool {
          return wait_count(p.sync + p.gm[g].wait_slot, target, s_flag, p.spin_limit, p.sync + S_ABORT);
        };
        for (int g = 0; g < 4 && !s_flag[0]; ++g) {
          const FGemm& gm = p.gm[g];
          const int KB = R[g].KB;
          const int wrow0 = (p.l0 + li) * gm.n_tiles * kTileM;
          bool ready = false;
          int pend_s[C::kStages], pend_x[C::kStages], n_pend = 0, pend_first = 0;
          auto flush = [&]() {
            fence_proxy_async();
            for (int q = 0; q < n_pend; ++q) {
              uint8_t* bx = stage_base + pend_s[q] * C::kStageBytes + kKsub * kABytes;
#pragma unroll
              for (int sub = 0; sub < kKsub; ++sub)
                tma_load_2d(bx + sub * C::kBBytes, tmX[g], &full_bar[pend_s[q]], pend_x[q] + sub * kBK, 0, pol_x);
            }
            n_pend = 0;
            ready = true;
          };
          for (int64_t it = R[g].lo; it < R[g].hi && !s_flag[0];) {
            const int tile = static_cast<int>(it / KB);
            const int kb0 = static_cast<int>(it % KB);
            const int kb1 = (R[g].hi - it < KB - kb0) ? kb0 + static_cast<int>(R[g].hi - it) : KB;
            it += kb1 - kb0;
            for (int kb = kb0; kb < kb1; ++kb, ++i) {
              const int s = i % C::kStages;
              const uint32_t ph = (i / C::kStages) & 1;
              if (!ready && n_pend > 0 && i - C::kStages >= pend_first) {
                // the stage to reuse still waits for its activation tile
                if (!wait_x(g)) break;
                flush();
              }
              if (!mbar_wait_ab(&empty_bar[s], ph ^ 1, s_flag)) { s_flag[0] = 1; break; }
              uint8_t* a = stage_base + s * C::kStageBytes;
              mbar_arrive_expect_tx(&full_bar[s], C::kStageBytes);
#pragma unroll
              for (int sub = 0; sub < kKsub; ++sub) {
                const int x = (kb * kKsub + sub) * kBK;
                tma_load_2d(a + sub * kABytes, tmW[g], &full_bar[s], x, wrow0 + tile * kTileM, pol_w);
                tma_load_2d(a + sub * kABytes + kABytes / 2, tmW[g], &full_bar[s], x, wrow0 + tile * kTileM + 64,
                            pol_w);
              }
              if (!ready && x_ready(g)) flush();
              if (ready) {
                uint8_t* bx = a + kKsub * kABytes;
#pragma unroll
                for (int sub = 0; sub < kKsub; ++sub)
                  tma_load_2d(bx + sub * C::kBBytes, tmX[g], &full_bar[s], (kb * kKsub + sub) * kBK, 0, pol_x);
              } else {
                if (n_pend == 0) pend_first = i;
                pend_s[n_pend] = s;
                pend_x[n_pend] = kb * kKsub * kBK;
                ++n_pend;
              }
            }
          }
          if (!ready && n_pend > 0 && !s_flag[0]) {
            if (wait_x(g)) flush();
          }
          if (s_flag[0] && n_pend > 0) flush();   // aborting: complete the stages already requested
        }
      }
      if (s_flag[0]) {
        // aborting: wait (bounded) until the copies of the last stages requested have landed
        for (int q = i > C::kStages ? i - C::kStages : 0; q < i; ++q)
          mbar_wait(&full_bar[q % C::kStages], (q / C::kStages) & 1);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = make_idesc_bf16(kTileM, BN);
      int i = 0, j = 0;
      for (int li = 0; li < p.n_layers && !s_flag[0]; ++li) {
        for (int g = 0; g < 4 && !s_flag[0]; ++g) {
          const Items r = items_of(p.gm[g].K, p.gm[g].n_tiles, G, c);
          const int KB = r.KB;
          for (int64_t it = r.lo; it < r.hi && !s_flag[0];) {
            const int kb0 = static_cast<int>(it % KB);
            const int kb1 = (r.hi - it < KB - kb0) ? kb0 + static_cast<int>(r.hi - it) : KB;
            it += kb1 - kb0;
            const int b = j & 1;
            const uint32_t u = static_cast<uint32_t>(j >> 1);
            ++j;
            if (!mbar_wait_ab(&acc_empty[b], (u & 1) ^ 1, s_flag)) { s_flag[0] = 1; break; }
            tc_fence_after();
            const uint32_t d = tmem + b * C::kAccCols;
            for (int kb = kb0; kb < kb1; ++kb, ++i) {
              const int s = i % C::kStages;
              const uint32_t ph = (i / C::kStages) & 1;
              if (!mbar_wait_ab(&full_bar[s], ph, s_flag)) { s_flag[0] = 1; break; }
              tc_fence_after();
              const uint32_t a = smem_u32(stage_base + s * C::kStageBytes);
              const uint32_t bb = a + kKsub * kABytes;
#pragma unroll
              for (int sub = 0; sub < kKsub; ++sub)
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
      // every MMA issued has completed before the tensor memory is freed
      tc_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else {
    // ---------------- warps 0-3: reductions of the GEMM pieces and the steps between GEMMs
    const int t = threadIdx.x;
    const int m_rows = min(*p.n_rows, p.rows_cap);
    if (t < kMaxRows) s_rows[t] = t < m_rows ? p.rows[t] : 0;
    epi_bar();
    const int64_t gt = static_cast<int64_t>(c) * 128 + t;   // grid-wide epilogue thread index
    const int64_t gstride = static_cast<int64_t>(G) * 128;
    const int half = p.hd >> 1;
    int j = 0;
    auto gemm_epilogues = [&](int g, int li) {
      const FGemm& gm = p.gm[g];
      float* const out = gm.out;
      const Items r = items_of(gm.K, gm.n_tiles, G, c);
      const int KB = r.KB;
      for (int64_t it = r.lo; it < r.hi;) {
        const int tile = static_cast<int>(it / KB);
        const int kb0 = static_cast<int>(it % KB);
        const int kb1 = (r.hi - it < KB - kb0) ? kb0 + static_cast<int>(r.hi - it) : KB;
        it += kb1 - kb0;
        const int b = j & 1;
        const uint32_t u = static_cast<uint32_t>(j >> 1);
        ++j;
        const bool late = !mbar_wait_ab(&acc_full[b], u & 1, s_flag);
        if (epi_any(late || s_flag[0])) {              // one decision for all epilogue threads
          s_flag[0] = 1;
          return;
        }
        tc_fence_after();
        const uint32_t tb = tmem + (static_cast<uint32_t>(warp * 32) << 16) + b * C::kAccCols;
        float* col = out + tile * kTileM + t;           // output feature n = tile * 128 + t
#pragma unroll
        for (int cc = 0; cc < BN; cc += 16) {
          float v[16];
          tmem_ld16(tb + cc, v);
          if (cc + 16 >= BN) {
            tc_fence_before();
            mbar_arrive(&acc_empty[b]);
          }
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int jj = cc + q;
            if (jj < m_rows) atomicAdd(col + static_cast<int64_t>(gm.use_rows ? s_rows[jj] : jj) * gm.ldo, v[q]);
          }
        }
      }
    };

    // GEMM operand X = bf16(gain * h) over every row, each CTA a slice of the columns, and
    // the CTA's partial sums of h^2 per row added into ss[j] (RMSNorm is a per-row scale: the
    // GEMM sums are multiplied by 1/rms afterwards)
    auto gain_operand = [&](const float* gain, __nv_bfloat16* X, float* ss) {
      const int n4 = p.d >> 2;
      const int q0 = static_cast<int>(static_cast<int64_t>(n4) * c / G);
      const int q1 = static_cast<int>(static_cast<int64_t>(n4) * (c + 1) / G);
      const int w4 = q1 - q0;
      if (t < kMaxRows) s_ss[t] = 0.f;
      epi_bar();
      for (int u = t; u < m_rows * w4; u += 128) {
        const int jj = u / w4;
        const int k = (q0 + u - jj * w4) * 4;
        const float4 v = __ldcg(reinterpret_cast<const float4*>(p.h + static_cast<int64_t>(s_rows[jj]) * p.d + k));
        const float4 g4 = __ldg(reinterpret_cast<const float4*>(gain + k));
        __nv_bfloat162 lo = __floats2bfloat162_rn(g4.x * v.x, g4.y * v.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(g4.z * v.z, g4.w * v.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(X + static_cast<int64_t>(jj) * p.d + k) = pk;
        atomicAdd(&s_ss[jj], v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w);
      }
      epi_bar();
      if (t < m_rows) atomicAdd(ss + t, s_ss[t]);
    };
    // 1/rms of every row from the sums all CTAs added (after the phase that added them): one
    // L2 round trip, where summing 148 per-CTA partials was a chain of dependent loads
    auto rinv_from = [&](const float* ss, float* rinv) {
      if (t < m_rows) rinv[t] = rsqrtf(__ldcg(ss + t) / static_cast<float>(p.d) + p.eps);
      epi_bar();
    };

    for (int li = 0; li < p.n_layers; ++li) {
      const int l = p.l0 + li;
      const int target = (li + 1) * G;
      __nv_bfloat16* kc = p.kc + static_cast<int64_t>(l) * p.kv_layer;
      __nv_bfloat16* vc = p.vc + static_cast<int64_t>(l) * p.kv_layer;
      // the previous layer's down sums are complete in h (and its sums have been read)
      if (li > 0 && !epi_wait_phase(p.sync + S_DOWN, li * G, s_flag, t, p.spin_limit, p.sync + S_ABORT)) s_flag[0] = 1;
      if (p.es.on && li < p.es.n_scored) {
        // ES-dLLM Eq. 1 on every candidate's input of this layer: each row split into column
        // slices over the grid's warps, whose partial sums meet in es_acc[2 u .. 2 u + 1]
        const FusedEs& es = p.es;
        const int n = es.n_cand;
        const int nrow = es.B * n;
        if (!s_flag[0]) {
          const int64_t BNd = static_cast<int64_t>(es.B) * p.N * p.d;
          float* prev = l == es.ls ? es.h_prev : es.es_in + static_cast<int64_t>(l - es.ls - 1) * BNd;
          const int nch = p.d >> 7;                                  // 128-column chunks of a row
          const int S = max(1, min(nch, (G * 4) / nrow));            // slices per row
          for (int w = c * 4 + warp; w < nrow * S; w += G * 4) {
            const int u = w / S, sl = w - (w / S) * S;
            const int b = u / n;
            const int flat = b * p.N + es.cand_start + (u - b * n);
            const bool carried = l > es.ls && __ldcg(es.flag + flat) == 0;
            float l1 = 0.f, l2 = 0.f;
            es_eq1_part(p.h + static_cast<int64_t>(flat) * p.d, prev + static_cast<int64_t>(flat) * p.d,
                        (nch * sl / S) << 7, min(p.d, (nch * (sl + 1) / S) << 7), 1, carried, lane, l1, l2);
            l1 = es_warp_sum(l1);
            l2 = es_warp_sum(l2);
            if (lane == 0) {
              atomicAdd(p.es_acc + 2 * u, l1);
              atomicAdd(p.es_acc + 2 * u + 1, l2);
            }
          }
        }
        signal_phase(p.sync + S_SCORE, t);
        // the top k of sequence b by CTA b: a candidate is chosen when fewer than k others
        // rank above it (higher key, or an equal key at a lower position)
        if (epi_wait_phase(p.sync + S_SCORE, target, s_flag, t, p.spin_limit, p.sync + S_ABORT) && c < es.B) {
          const int b = c;
          const bool last = li == es.n_scored - 1;
          uint8_t* s_pick = attn_smem;                                         // idle outside attention
          uint32_t* s_key = reinterpret_cast<uint32_t*>(attn_smem + kFusedEsMaxCand);
          const float* fv = es.forced ? es.forced + (static_cast<int64_t>(li) * es.B + b) * n : nullptr;
          for (int i = t; i < n; i += 128) {
            const int u = b * n + i;
            const int flat = b * p.N + es.cand_start + i;
            const float l1 = __ldcg(p.es_acc + 2 * u), l2 = __ldcg(p.es_acc + 2 * u + 1);
            p.es_acc[2 * u] = 0.f;                                           // zero for the next layer
            p.es_acc[2 * u + 1] = 0.f;
            const float cf = __ldcg(es.masked_prev + flat) ? __ldcg(es.conf + flat) : 0.f;
            const float sc = es_eq1_score(l1, l2, p.d, cf, es.alpha);
            es.scores[u] = sc;
            // masked_prev rolls forward once every layer has read it
            if (last) es.masked_prev[flat] = __ldcg(es.tokens + flat) == es.mask_id ? 1 : 0;
            s_key[i] = order_key(fv ? __ldcg(fv + i) : sc);
          }
          epi_bar();
          for (int i = t; i < n; i += 128) {
            const uint32_t ki = s_key[i];
            int rank = 0;
            for (int jn = 0; jn < n; ++jn) {
              const uint32_t kj = s_key[jn];
              rank += (kj > ki || (kj == ki && jn < i)) ? 1 : 0;
            }
            const uint8_t ch = rank < es.k ? 1 : 0;
            s_pick[i] = ch;
            es.flag[b * p.N + es.cand_start + i] = ch;
          }
          epi_bar();
          for (int i = t; i < n; i += 128) {
            if (!s_pick[i]) continue;
            int o = 0;
            for (int jn = 0; jn < i; ++jn) o += s_pick[jn];
            es.rows[b * es.k + o] = b * p.N + es.cand_start + i;
          }
        }
        signal_phase(p.sync + S_PICK, t);
        if (epi_wait_phase(p.sync + S_PICK, target, s_flag, t, p.spin_limit, p.sync + S_ABORT) && t < kMaxRows)
          s_rows[t] = t < m_rows ? __ldcg(es.rows + t) : 0;
        epi_bar();
      }
      if (!s_flag[0]) {
        // zero this layer's sums (every CTA passes this phase before any adds into them)
        const int64_t nq = static_cast<int64_t>(m_rows) * p.qkvd / 4;
        const int64_t ng = static_cast<int64_t>(m_rows) * 2 * p.F / 4;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int64_t x = gt; x < nq; x += gstride) reinterpret_cast<float4*>(p.s_qkv)[x] = z;
        for (int64_t x = gt; x < ng; x += gstride) reinterpret_cast<float4*>(p.s_gu)[x] = z;
        gain_operand(p.g_attn + static_cast<int64_t>(l) * p.d, p.z1, p.ss1);    // QKV operand
      }
      signal_phase(p.sync + S_X1, t);
      if (epi_wait_phase(p.sync + S_X1, target, s_flag, t, p.spin_limit, p.sync + S_ABORT)) rinv_from(p.ss1, s_rinv1);   // while QKV streams
      gemm_epilogues(0, li);                                       // QKV sums
      signal_phase(p.sync + S_QKV, t);
      // RMSNorm scale and RoPE (rotate-half pairs i, i + hd/2) on q and k; q to the attention
      // operand, k and v scattered into the cache rows of their positions
      if (epi_wait_phase(p.sync + S_QKV, target, s_flag, t, p.spin_limit, p.sync + S_ABORT)) {
        if (c == 0 && t < kMaxRows) p.ss1[t] = 0.f;    // every CTA has read this layer's sums
        // an item is 4 consecutive pairs of one head of one row: 16-byte loads of both halves
        // and of the cos/sin table, 8-byte stores
        const int groups = p.qkvd >> 3;         // items per row
        const int gph = half >> 2;              // items per head
        const int64_t total = static_cast<int64_t>(m_rows) * groups;
        constexpr int U = 4;                    // items per thread in flight: their loads go out together
        for (int64_t u0 = gt; u0 < total; u0 += U * gstride) {
          float4 xl[U], xh[U], cs[U], sn[U];
          int jrs[U], nlo[U], pis[U];
#pragma unroll
          for (int e = 0; e < U; ++e) {
            const int64_t uu = u0 + e * gstride < total ? u0 + e * gstride : 0;   // in bounds either way
            const int jr = static_cast<int>(uu / groups);
            const int rr = static_cast<int>(uu - static_cast<int64_t>(jr) * groups);
            const int head = rr / gph;
            pis[e] = (rr - head * gph) * 4;
            nlo[e] = head * p.hd + pis[e];
            jrs[e] = jr;
            const float* srow = p.s_qkv + static_cast<int64_t>(jr) * p.qkvd;
            xl[e] = __ldcg(reinterpret_cast<const float4*>(srow + nlo[e]));
            xh[e] = __ldcg(reinterpret_cast<const float4*>(srow + nlo[e] + half));
            const int flat = s_rows[jr];
            const int pos = flat - (flat / p.N) * p.N;
            cs[e] = __ldg(reinterpret_cast<const float4*>(p.rope_cos + static_cast<int64_t>(pos) * half + pis[e]));
            sn[e] = __ldg(reinterpret_cast<const float4*>(p.rope_sin + static_cast<int64_t>(pos) * half + pis[e]));
          }
#pragma unroll
          for (int e = 0; e < U; ++e) {
            if (u0 + e * gstride >= total) break;
            const int jr = jrs[e], n_lo = nlo[e], pi = pis[e];
            const float ri = s_rinv1[jr];
            float lo[4] = {xl[e].x * ri, xl[e].y * ri, xl[e].z * ri, xl[e].w * ri};
            float hi[4] = {xh[e].x * ri, xh[e].y * ri, xh[e].z * ri, xh[e].w * ri};
            if (n_lo < p.qd + p.kvd) {
              const float c4[4] = {cs[e].x, cs[e].y, cs[e].z, cs[e].w};
              const float s4[4] = {sn[e].x, sn[e].y, sn[e].z, sn[e].w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float x_l = lo[k], x_h = hi[k];
                lo[k] = x_l * c4[k] - x_h * s4[k];
                hi[k] = x_h * c4[k] + x_l * s4[k];
              }
            }
            const int flat = s_rows[jr];
            const int b = flat / p.N;
            const int pos = flat - b * p.N;
            __nv_bfloat16* dst;
            if (n_lo < p.qd) {
              dst = p.q + static_cast<int64_t>(jr) * p.qd + n_lo;
            } else {
              int nn = n_lo - p.qd;
              __nv_bfloat16* cache = kc;
              if (nn >= p.kvd) {
                nn -= p.kvd;
                cache = vc;
              }
              const int kvh = nn / p.hd;
              dst = cache + ((static_cast<int64_t>(b) * p.Hkv + kvh) * p.N + pos) * p.hd + pi;
            }
            __nv_bfloat162 t0 = __floats2bfloat162_rn(lo[0], lo[1]), t1 = __floats2bfloat162_rn(lo[2], lo[3]);
            __nv_bfloat162 t2 = __floats2bfloat162_rn(hi[0], hi[1]), t3 = __floats2bfloat162_rn(hi[2], hi[3]);
            uint2 w0, w1;
            w0.x = *reinterpret_cast<uint32_t*>(&t0);
            w0.y = *reinterpret_cast<uint32_t*>(&t1);
            w1.x = *reinterpret_cast<uint32_t*>(&t2);
            w1.y = *reinterpret_cast<uint32_t*>(&t3);
            *reinterpret_cast<uint2*>(dst) = w0;
            *reinterpret_cast<uint2*>(dst + half) = w1;
          }
        }
      }
      signal_phase(p.sync + S_ROPE, t);
      // attention items over the cached K/V (the new rows are in the cache now); the last
      // split of a (sequence, KV head, query tile) to finish merges the partials
      if (epi_wait_phase(p.sync + S_ROPE, target, s_flag, t, p.spin_limit, p.sync + S_ABORT)) {
        attn::AttnParams ap = p.ap;
        ap.kc = kc;
        ap.vc = vc;
        const int Gq = ap.Hq / ap.Hkv;
        for (int it = c; it < p.attn_items; it += G) {
          int rem = it;
          const int split = rem % ap.splits;
          rem /= ap.splits;
          const int qt = rem % p.attn_qtiles;
          rem /= p.attn_qtiles;
          const int kvh = rem % ap.Hkv;
          const int b = rem / ap.Hkv;
          if (p.hd == 128) attn::attn_item<128>(ap, qt, b, kvh, split, attn_smem, t, NamedBar{});
          else attn::attn_item<64>(ap, qt, b, kvh, split, attn_smem, t, NamedBar{});
          if (ap.splits > 1 && p.attn_group_merge) {
            // every split of the group is another CTA's item of this same round, all resident:
            // each waits for all of them, then merges its share of the query tile's units
            __threadfence();
            epi_bar();
            const int grp = (b * ap.Hkv + kvh) * p.attn_qtiles + qt;
            if (t == 0) atomicAdd(p.attn_ctr + grp, 1);
            if (epi_wait_phase(p.attn_ctr + grp, ap.splits, s_flag, t, p.spin_limit, p.sync + S_ABORT)) {
              const int off = ap.seq_off[b];
              const int n_units = (ap.seq_off[b + 1] - off) * Gq;
              const int u1 = min(n_units, (qt + 1) * 64);
              for (int uu = qt * 64 + split + ap.splits * warp; uu < u1; uu += 4 * ap.splits) {
                const int row = off + uu / Gq, hh = kvh * Gq + uu % Gq;
                if (p.hd == 128) attn::attn_merge<128>(ap, row, hh, lane);
                else attn::attn_merge<64>(ap, row, hh, lane);
              }
            }
            // a second arrival once the partials are read: the last one re-arms the counter
            epi_bar();
            if (t == 0 && atomicAdd(p.attn_ctr + grp, 1) == 2 * ap.splits - 1) p.attn_ctr[grp] = 0;
          } else if (ap.splits > 1) {
            __threadfence();
            epi_bar();
            const int grp = (b * ap.Hkv + kvh) * p.attn_qtiles + qt;
            if (t == 0) s_flag[1] = atomicAdd(p.attn_ctr + grp, 1) == ap.splits - 1 ? 1 : 0;
            epi_bar();
            if (s_flag[1]) {
              __threadfence();
              const int off = ap.seq_off[b];
              const int n_units = (ap.seq_off[b + 1] - off) * Gq;
              const int u1 = min(n_units, (qt + 1) * 64);
              for (int uu = qt * 64 + warp; uu < u1; uu += 4) {
                const int row = off + uu / Gq, hh = kvh * Gq + uu % Gq;
                if (p.hd == 128) attn::attn_merge<128>(ap, row, hh, lane);
                else attn::attn_merge<64>(ap, row, hh, lane);
              }
              if (t == 0) p.attn_ctr[grp] = 0;
            }
          }
          epi_bar();
        }
      }
      signal_phase(p.sync + S_COMB, t);
      gemm_epilogues(1, li);                                       // O, added into h
      signal_phase(p.sync + S_O, t);
      // gate/up operand g_ffn * h once every O sum is in h
      if (epi_wait_phase(p.sync + S_O, target, s_flag, t, p.spin_limit, p.sync + S_ABORT))
        gain_operand(p.g_ffn + static_cast<int64_t>(l) * p.d, p.z2, p.ss2);
      signal_phase(p.sync + S_X2, t);
      if (epi_wait_phase(p.sync + S_X2, target, s_flag, t, p.spin_limit, p.sync + S_ABORT)) rinv_from(p.ss2, s_rinv2);   // while gate/up streams
      gemm_epilogues(2, li);                                       // gate/up sums
      signal_phase(p.sync + S_GU, t);
      // SwiGLU on the RMSNorm-scaled sums: act = silu(gate) * up
      if (epi_wait_phase(p.sync + S_GU, target, s_flag, t, p.spin_limit, p.sync + S_ABORT)) {
        if (c == 0 && t < kMaxRows) p.ss2[t] = 0.f;
        const int f4 = p.F >> 2;
        const int64_t total = static_cast<int64_t>(m_rows) * f4;
        constexpr int U = 8;                    // groups per thread in flight: their loads go out together
        for (int64_t u0 = gt; u0 < total; u0 += U * gstride) {
          float4 g4s[U], u4s[U];
#pragma unroll
          for (int e = 0; e < U; ++e) {
            const int64_t uu = u0 + e * gstride < total ? u0 + e * gstride : 0;   // in bounds either way
            const int jr = static_cast<int>(uu / f4);
            const int f = static_cast<int>(uu - static_cast<int64_t>(jr) * f4) * 4;
            const float* srow = p.s_gu + static_cast<int64_t>(jr) * 2 * p.F;
            g4s[e] = __ldcg(reinterpret_cast<const float4*>(srow + f));
            u4s[e] = __ldcg(reinterpret_cast<const float4*>(srow + p.F + f));
          }
#pragma unroll
          for (int e = 0; e < U; ++e) {
          const int64_t uu = u0 + e * gstride;
          if (uu >= total) break;
          const int jr = static_cast<int>(uu / f4);
          const int f = static_cast<int>(uu - static_cast<int64_t>(jr) * f4) * 4;
          const float ri = s_rinv2[jr];
          const float4 g4 = g4s[e], u4 = u4s[e];
          const float g[4] = {g4.x * ri, g4.y * ri, g4.z * ri, g4.w * ri};
          const float u[4] = {u4.x * ri, u4.y * ri, u4.z * ri, u4.w * ri};
          float a[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) a[e] = g[e] / (1.f + __expf(-g[e])) * u[e];
          __nv_bfloat162 lo = __floats2bfloat162_rn(a[0], a[1]);
          __nv_bfloat162 hi = __floats2bfloat162_rn(a[2], a[3]);
          uint2 pk;
          pk.x = *reinterpret_cast<uint32_t*>(&lo);
          pk.y = *reinterpret_cast<uint32_t*>(&hi);
          *reinterpret_cast<uint2*>(p.act + static_cast<int64_t>(jr) * p.F + f) = pk;
          }
        }
      }
      signal_phase(p.sync + S_SWIGLU, t);
      gemm_epilogues(3, li);                                       // down, added into h
      signal_phase(p.sync + S_DOWN, t);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tmem, C::kTmemCols);
  // the last CTA out clears the counters, so every launch (a graph replay too) starts from zero;
  // after an aborted launch it also clears what an unfinished layer can leave behind (attention
  // split arrivals, the ES choice's row sums)
  if (threadIdx.x == 0) {
    if (s_flag[0]) atomicExch(p.sync + S_ABORT, 1);
    __threadfence();
    if (atomicAdd(p.sync + S_COUNT, 1) == G - 1) {
      if (atomicAdd(p.sync + S_ABORT, 0) != 0) {
        for (int q = 0; q < p.n_attn_ctr; ++q) p.attn_ctr[q] = 0;
        if (p.es.on)
          for (int q = 0; q < 2 * p.es.B * p.es.n_cand; ++q) p.es_acc[q] = 0.f;
        for (int q = 0; q < kMaxRows; ++q) p.ss1[q] = p.ss2[q] = 0.f;
      }
      for (int q = 0; q <= S_ABORT; ++q) atomicExch(p.sync + q, 0);
      __threadfence();
    }
  }
}

template <int BN>
int launch_fused(const CUtensorMap (&tw)[4], const CUtensorMap (&tx)[4], const FParams& p, int grid,
                 cudaStream_t st) {
  using C = FCfg<BN>;
  const int rc = ensure_smem_attr(reinterpret_cast<const void*>(fused_layer_kernel<BN>), static_cast<int>(C::kSmem));
  if (rc) return rc;
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fused_layer_kernel<BN>, tw[0], tw[1], tw[2], tw[3], tx[0], tx[1],
                                           tx[2], tx[3], p);
  count_launch();
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e), __FILE__, __LINE__);
    return DLLM_ERR_CUDA;
  }
  return DLLM_OK;
}

}  // namespace

size_t fused_scratch_floats(int qkvd, int F, int max_ctas) {
  return static_cast<size_t>(kMaxRows) * (static_cast<size_t>(qkvd) + 2 * static_cast<size_t>(F)) +
         2 * static_cast<size_t>(max_ctas) * kMaxRows + 2 * static_cast<size_t>(kMaxRows) * kFusedEsMaxCand;
}

int fused_attn_counters(int B, int Hq, int Hkv, int rows_cap) {
  const int qtiles = (rows_cap * (Hq / Hkv) + 63) / 64;
  return B * Hkv * qtiles;
}

int fused_layer_launch(const FusedLayerArgs& a, cudaStream_t st) {
  if (a.rows_cap <= 0 || a.rows_cap > kMaxRows) return DLLM_ERR_UNSUPPORTED;
  if (a.d % 128 || a.qd % 128 || a.F % 128 || a.qkvd % 128 || a.hd > 128) return DLLM_ERR_UNSUPPORTED;
  // the RoPE phase moves 4 pairs per item: 16-byte table loads, 8-byte operand and cache stores
  if (a.hd % 8 || reinterpret_cast<uintptr_t>(a.rope_cos) % 16 || reinterpret_cast<uintptr_t>(a.rope_sin) % 16 ||
      reinterpret_cast<uintptr_t>(a.kc) % 8 || reinterpret_cast<uintptr_t>(a.vc) % 8)
    return DLLM_ERR_UNSUPPORTED;
  if (a.n_layers <= 0 || a.l0 < 0 || a.l0 + a.n_layers > a.L) return DLLM_ERR_INVALID_ARG;
  const int bn = a.rows_cap <= 16 ? 16 : (a.rows_cap <= 32 ? 32 : 64);
  if (a.max_ctas <= 0) return DLLM_ERR_INVALID_ARG;
  const int grid = std::min(num_sms(), a.max_ctas);   // one CTA per SM, all resident (cooperative)
  CUtensorMap tw[4], tx[4];
  // every layer of a weight stack in one map: layer l's tile rows start at l * rows per layer
  const void* W[4] = {a.Wqkv, a.Wo, a.Wgu, a.Wdn};
  const int64_t wrows[4] = {a.qkvd, a.d, 2LL * a.F, a.d};
  const int K[4] = {a.d, a.qd, a.d, a.F};
  const void* X[4] = {a.z1, a.attn, a.z2, a.act};
  for (int q = 0; q < 4; ++q) {
    int rc = make_tmap(&tw[q], W[q], wrows[q] * a.L, K[q], 64);
    if (rc) return rc;
    rc = make_tmap(&tx[q], X[q], a.rows_cap, K[q], bn);
    if (rc) return rc;
  }
  FParams p;
  p.l0 = a.l0;
  p.n_layers = a.n_layers;
  float* s_qkv = a.scratch;
  float* s_gu = s_qkv + static_cast<size_t>(kMaxRows) * a.qkvd;
  float* ssp = s_gu + static_cast<size_t>(kMaxRows) * 2 * a.F;
  const int waits[4] = {S_X1, S_COMB, S_X2, S_SWIGLU};
  float* outs[4] = {s_qkv, a.h, s_gu, a.h};
  const int ldos[4] = {a.qkvd, a.d, 2 * a.F, a.d};
  for (int q = 0; q < 4; ++q) {
    FGemm& g = p.gm[q];
    g.K = K[q];
    g.n_tiles = static_cast<int>(wrows[q] / 128);
    g.wait_slot = waits[q];
    g.out = outs[q];
    g.ldo = ldos[q];
    g.use_rows = (q == 1 || q == 3) ? 1 : 0;
  }
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
  p.s_qkv = s_qkv;
  p.s_gu = s_gu;
  p.ss1 = ssp;
  p.ss2 = ssp + kMaxRows;
  p.es_acc = ssp + 2 * static_cast<size_t>(a.max_ctas) * kMaxRows;
  p.n_attn_ctr = a.n_attn_ctr;
  p.spin_limit = a.spin_limit ? a.spin_limit : kSpinLimit;
  p.qkvd = a.qkvd; p.qd = a.qd; p.kvd = a.kvd; p.hd = a.hd; p.Hkv = a.Hkv; p.N = a.N; p.F = a.F;
  p.rope_cos = a.rope_cos;
  p.rope_sin = a.rope_sin;
  p.q = a.q;
  p.kc = a.kc;
  p.vc = a.vc;
  p.kv_layer = static_cast<int64_t>(a.B) * a.Hkv * a.N * a.hd;
  p.act = a.act;
  const size_t kv_bytes = static_cast<size_t>(p.kv_layer) * 2;
  p.kv_bytes = kv_bytes <= kMaxKvPrefetch ? kv_bytes : 0;
  // attention work: every (sequence, KV head, query tile, key split) item
  const int Gq = a.Hq / a.Hkv;
  const int units = a.rows_per_seq * Gq;
  const int qtiles = (units + 63) / 64;
  const int n_blocks = (a.N + 63) / 64;
  // key splits: enough items for about one round over the grid
  static const int splits_env = [] {
    const char* e = getenv("DLLM_FUSED_ATTN_SPLITS");   // tuning knob for measurements
    return e ? std::max(0, atoi(e)) : 0;
  }();
  const int groups = a.B * a.Hkv * qtiles;
  int splits = splits_env > 0 ? splits_env : std::max(1, grid / groups);
  splits = std::max(1, std::min(n_blocks, splits));
  const int bps = (n_blocks + splits - 1) / splits;
  splits = (n_blocks + bps - 1) / bps;
  if (static_cast<size_t>(splits) * a.rows_cap * a.Hq * a.hd > a.attn_floats) return DLLM_ERR_SHAPE;
  if (a.B * a.Hkv * qtiles > a.n_attn_ctr) return DLLM_ERR_SHAPE;
  attn::AttnParams& ap = p.ap;
  ap.q = a.q; ap.kc = a.kc; ap.vc = a.vc; ap.out = a.attn; ap.seq_off = a.seq_off;
  ap.B = a.B; ap.N = a.N; ap.Hq = a.Hq; ap.Hkv = a.Hkv; ap.rows_cap = a.rows_cap;
  ap.splits = splits; ap.blocks_per_split = bps;
  ap.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.hd));
  ap.opart = a.attn_opart; ap.ml = a.attn_ml;
  p.attn_qtiles = qtiles;
  p.attn_items = a.B * a.Hkv * qtiles * splits;
  p.attn_group_merge = p.attn_items <= grid ? 1 : 0;
  p.attn_ctr = a.attn_ctr;
  p.sync = a.sync;
  p.es = a.es;
  if (a.es.on) {
    const FusedEs& e = a.es;
    if (e.n_cand <= 0 || e.n_cand > kFusedEsMaxCand || e.k <= 0 || e.k > e.n_cand || e.B != a.B || e.B > grid ||
        e.B * e.k > a.rows_cap || e.ls < 0 || a.l0 < e.ls || a.l0 + a.n_layers > e.L || e.L != a.L ||
        e.n_scored < 1 || e.n_scored > a.n_layers)
      return DLLM_ERR_UNSUPPORTED;
    if (!e.h_prev || (a.l0 + e.n_scored - 1 > e.ls && !e.es_in) || !e.conf || !e.masked_prev || !e.tokens ||
        !e.flag || !e.rows || !e.scores || e.rows != a.rows)
      return DLLM_ERR_INVALID_ARG;
  }
  if (bn == 16) return launch_fused<16>(tw, tx, p, grid, st);
  if (bn == 32) return launch_fused<32>(tw, tx, p, grid, st);
  return launch_fused<64>(tw, tx, p, grid, st);
}

}  // namespace dllm
