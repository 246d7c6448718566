// Many-query attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// SureLock summary sec. 2.1 items 3-4: the recomputed rows attend to every position
// of their sequence through the cached K/V (bidirectional, no mask), O(M_t * N * d);
// ES-dLLM summary sec. 2.2: a refresh step recomputes every row, so there the query
// count equals the sequence length.  With many queries per (sequence, KV head) this
// is a pair of dense contractions, S = Q K^T and O = P V, so it runs on tcgen05:
//
//   one CTA per (sequence b, KV head, pair of 128-unit query tiles, key split), where a
//   unit is a (query row, query head of the KV head's group) pair, so the query heads
//   that share a KV head share its K/V tiles (grouped-query attention), and both query
//   tiles of the CTA share every K/V tile it loads;
//   warps 4 g .. 4 g + 3 load the q vectors of query tile g into a 128-byte-swizzled
//   K-major tile and run its softmax and output epilogue, one thread per unit (TMEM lane);
//   warp 8 lane 0 streams 128-key K and V tiles with TMA through a ring of five 32 KB
//   slots (a 3-D tensor map [B * Hkv][N][hd] per cache: keys past N are zero-filled);
//   warp 9 lane 0 issues the MMAs and owns the TMEM allocation: per query tile the S
//   tile (128 columns, P written over its first 64 as the A operand of P V) and the O
//   accumulator (128 columns).  The two query tiles alternate on the tensor pipe, so the
//   MMAs of one run while the other's softmax turns S into P.
//
// The softmax runs online over the key tiles with a lazily moved offset: for each tile
// the row maximum of S' = S log2(e) / sqrt(hd); while it stays within kSlack of the
// running offset m, P = 2^(S' - m) <= 2^kSlack is written in bf16 into TMEM (the A operand
// of the P V product) and l accumulates its fp32 row sum; when it exceeds m + kSlack, O
// (in TMEM) and l are first multiplied by 2^(m_old - m_new).  That rescale needs no wait:
// the MMAs of a CTA run in issue order, so when the tile's S is complete every earlier
// P V product is too.  The result is O / l in bf16, or, with the keys split over several
// CTAs, the unnormalised O with (m, l) per (row, head) for the split merge, in the format
// of the CUDA-core path.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>
#include <unordered_map>

#include "attn_dev.cuh"
#include "common.cuh"
#include "gemm_dev.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace dllm {
namespace {

using namespace attn;

constexpr int kHd = 128;                         // head dimension of this kernel
constexpr int kTq = 128;                         // query units per tile (MMA M, TMEM lanes)
constexpr int kTiles = 2;                        // query tiles per CTA, one softmax warpgroup each
constexpr int kTk = 128;                         // keys per tile (MMA N of S, K of P V)
constexpr uint32_t kPanel = 128 * 128;           // one 128-row x 64-column bf16 panel (128 B rows)
constexpr uint32_t kTileBytes = 2 * kPanel;      // 128 rows x 128 columns bf16: two panels
constexpr int kSlots = 5;                        // K/V ring of 32 KB tiles
constexpr int kThreadsTc = kTiles * 128 + 64;
constexpr int kProducerWarp = kTiles * 4, kMmaWarp = kProducerWarp + 1;
// TMEM per query tile g: S at 256 g (128 columns; P, bf16 two keys per 32-bit column, is
// written over its first 64 once S is in registers: the A operand of P V), O at 256 g + 128
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColTile = 256, kColO = 128;
static_assert(kTiles * kColTile <= kTmemCols, "TMEM columns");

// Shared memory: the Q tiles, the K/V ring, barriers.
constexpr size_t kOffQ = 0;
constexpr size_t kOffKV = kOffQ + kTiles * kTileBytes;
constexpr size_t kOffBar = kOffKV + static_cast<size_t>(kSlots) * kTileBytes;
constexpr size_t kSmemTc = 1024 + kOffBar + 256;
static_assert(kSmemTc <= 227 * 1024, "attention tiles do not fit shared memory");

// Shared-memory descriptor of an MN-major operand tile written with 128-byte swizzling:
// 64 contiguous elements (128 B) per row along MN, one row per K index, 8-row atoms of
// 1024 B along K (stride byte offset); the next 64 MN elements sit one panel further
// (leading byte offset).
__device__ __forceinline__ uint64_t make_desc_mn_sw128(uint32_t smem_addr, uint32_t panel_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFF) >> 4);
  d |= static_cast<uint64_t>((panel_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16, bf16 A K-major and bf16 B MN-major, fp32 D.
__host__ __device__ constexpr uint32_t make_idesc_bf16_bmn(int M, int N) {
  return make_idesc_bf16(M, N) | (1u << 16);
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y, int z,
                                            uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(cache_hint)
      : "memory");
}

__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Barrier of the 128 threads of softmax warpgroup g (named barrier 1 + g) that also returns
// whether any of them passed true.
__device__ __forceinline__ bool group_any(bool v, int g) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(1 + g)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void group_bar(int g) { asm volatile("bar.sync %0, 128;" ::"r"(1 + g) : "memory"); }

// 64 consecutive fp32 columns of this thread's TMEM lane, one load.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// 2^x by the MUFU instruction (relative error about 2^-22; the inputs here are at most the
// rescale slack, 8, and results below 2^-126 flush to 0; P is rounded to bf16 afterwards, 2^-9).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait of the softmax threads: between polls they sleep, so waiting softmax warps
// leave the issue slots of their SM sub-partitions to the TMA and MMA warps.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    __nanosleep(32);
  }
  set_dev_status(DLLM_DEV_TIMEOUT);
  return false;
}

// Largest of the first n of 64 values (tree order; n >= 64 takes the unpredicated path).
__device__ __forceinline__ float max64(const float (&v)[64], int n) {
  float r[32];
  if (n >= 64) {
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = fmaxf(v[i], v[i + 32]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      r[i] = fmaxf(i < n ? v[i] : -INFINITY, i + 32 < n ? v[i + 32] : -INFINITY);
  }
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) r[i] = fmaxf(r[i], r[i + w]);
  return r[0];
}

// P = 2^(S' - m), S' = S sc, for 64 S values of which the first n are valid keys (the rest
// give 0), packed as bf16 pairs; their fp32 sum is added to l.
__device__ __forceinline__ void p64(const float (&v)[64], int n, float sc, float nm, uint32_t (&pk)[32], float& l) {
  float lp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // independent partial sums
  if (n >= 64) {
#pragma unroll
    for (int q = 0; q < 64; q += 2) {
      const float p0 = ex2_approx(fmaf(v[q], sc, nm));
      const float p1 = ex2_approx(fmaf(v[q + 1], sc, nm));
      lp[(q >> 1) & 7] += p0 + p1;
      pk[q >> 1] = pack_bf16(p0, p1);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 64; q += 2) {
      const float p0 = q < n ? ex2_approx(fmaf(v[q], sc, nm)) : 0.f;
      const float p1 = q + 1 < n ? ex2_approx(fmaf(v[q + 1], sc, nm)) : 0.f;
      lp[(q >> 1) & 7] += p0 + p1;
      pk[q >> 1] = pack_bf16(p0, p1);
    }
  }
  l += ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
}

// Byte offset of 16-byte chunk `ch` (0..15) of row r in a two-panel 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int ch) {
  return static_cast<uint32_t>((ch >> 3) * kPanel + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

struct TcParams {
  AttnParams a;
  int qtiles;            // 128-unit query tiles per (sequence, KV head); a CTA takes two
  int blocks;            // 128-key tiles of N
  int blocks_per_split;
};

// S[d] = Q K^T over hd = 128: eight K = 16 steps, each inside one 64-column panel.
__device__ __forceinline__ void mma_qk(uint32_t d, uint32_t aq, uint32_t ak, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < kHd / 16; ++kk) {
    const uint32_t o = (kk >> 2) * kPanel + (kk & 3) * 32;
    tc_mma_f16(d, make_desc_k_sw128(aq + o), make_desc_k_sw128(ak + o), idesc, kk > 0 ? 1u : 0u);
  }
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16: A is 128 lanes x 16 bf16 (eight columns).
__device__ __forceinline__ void tc_mma_f16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// O[d] (+)= P V over 128 keys: P from TMEM (two keys per 32-bit column, eight columns per
// 16-key step), V MN-major (hd contiguous): a step is 16 key rows of V, 2048 B into each of
// its two hd panels.
__device__ __forceinline__ void mma_pv(uint32_t d, uint32_t ap_tmem, uint32_t av, uint32_t idesc, bool acc) {
#pragma unroll
  for (int kk = 0; kk < kTk / 16; ++kk)
    tc_mma_f16_ta(d, ap_tmem + kk * 8, make_desc_mn_sw128(av + kk * 2048, kPanel), idesc, (acc || kk > 0) ? 1u : 0u);
}

// 32 consecutive 32-bit columns of this thread's TMEM lane from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kThreadsTc, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, TcParams tp) {
  const AttnParams& p = tp.a;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;                       // [kTiles] Q tiles
  uint8_t* sKV = smem + kOffKV;                     // [kSlots] K or V tiles
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_empty = kv_full + kSlots;
  uint64_t* s_full = kv_empty + kSlots;             // [kTiles] S written
  uint64_t* p_full = s_full + kTiles;               // [kTiles] P written into TMEM (128 arrivals)
  uint64_t* q_full = p_full + kTiles;               // every Q tile written (kTiles x 128 arrivals)
  uint64_t* o_full = q_full + 1;                    // every P V product complete
  uint64_t* mma_done = o_full + 1;                  // every MMA issued complete (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int qp = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, kvh = blockIdx.y % p.Hkv;
  const int split = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  pdl_wait();                                       // q, the caches and seq_off come from earlier kernels
  const int off = p.seq_off[b];
  const int n_units = (p.seq_off[b + 1] - off) * G;
  const int u0 = qp * kTiles * kTq;
  const int blk0 = split * tp.blocks_per_split;
  const int blk1 = min(tp.blocks, blk0 + tp.blocks_per_split);
  if (u0 >= n_units || blk0 >= blk1) return;        // uniform over the CTA
  const int nb = blk1 - blk0;
  const int ng = min(kTiles, (n_units - u0 + kTq - 1) / kTq);   // query tiles with units
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int g = 0; g < kTiles; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], 128);
    }
    mbar_init(q_full, kTiles * 128);
    mbar_init(o_full, 1);
    mbar_init(mma_done, 1);
    s_abort[0] = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ---------------- TMA producer: one 32 KB tile per slot, in the order the MMAs use them:
      // K_j, V_j for every key tile j
      const uint64_t pol = policy_evict_last();      // reread by the other query tiles of the head
      const int z = b * p.Hkv + kvh;
      const int n_slots = 2 * nb;
      int i = 0;
      for (; i < n_slots && !s_abort[0]; ++i) {
        const int s = i % kSlots;
        if (!mbar_wait(&kv_empty[s], ((i / kSlots) & 1) ^ 1) || s_abort[0]) {
          s_abort[0] = 1;
          break;
        }
        const int j = i >> 1;
        const CUtensorMap* tm = (i & 1) ? &tmV : &tmK;
        const int key0 = (blk0 + j) * kTk;
        uint8_t* dst = sKV + s * kTileBytes;
        mbar_arrive_expect_tx(&kv_full[s], kTileBytes);
        tma_load_3d(dst, tm, &kv_full[s], 0, key0, z, pol);
        tma_load_3d(dst + kPanel, tm, &kv_full[s], 64, key0, z, pol);
      }
      if (s_abort[0]) {
        // the copies of the last slots requested land before the CTA leaves (bounded waits)
        for (int q = i > kSlots ? i - kSlots : 0; q < i; ++q) mbar_wait(&kv_full[q % kSlots], (q / kSlots) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ---------------- MMA issuer.  Per key tile j the tensor pipe runs S_0(j), S_1(j) (one
      // per query tile), then P_0(j) V_j, P_1(j) V_j as each softmax warpgroup hands over its P:
      // while one warpgroup turns its S into P, the MMAs of the other tile run.
      constexpr uint32_t idS = make_idesc_bf16(kTq, kTk);
      constexpr uint32_t idO = make_idesc_bf16_bmn(kTq, kHd);
      bool ok = mbar_wait(q_full, 0);
      auto slot_ready = [&](int i) -> bool {
        return mbar_wait(&kv_full[i % kSlots], (i / kSlots) & 1) && !s_abort[0];
      };
      const uint32_t aK = smem_u32(sKV);
      // S_g(0), then per key tile j: P_g(j) V_j once the softmax has written P_g(j), directly
      // followed by S_g(j + 1) into the same columns (the tensor pipe runs one CTA's MMAs in
      // issue order, so P_g(j) is read before S_g(j + 1) overwrites it, and S_g(j + 1) complete
      // means every P V product of the tile before it is complete)
      for (int g = 0; ok && g < ng; ++g) {
        if (!(ok = slot_ready(0))) break;
        tc_fence_after();
        mma_qk(tmem + g * kColTile, smem_u32(sQ + g * kTileBytes), aK, idS);
        tc_commit(&s_full[g]);
      }
      if (ok) tc_commit(&kv_empty[0]);
      for (int j = 0; ok && j < nb; ++j) {
        const int iV = 2 * j + 1, iK = iV + 1;
        const bool more = j + 1 < nb;
        if (!(ok = slot_ready(iV) && (!more || slot_ready(iK)))) break;
        for (int g = 0; g < ng; ++g) {
          if (!(ok = mbar_wait(&p_full[g], j & 1) && !s_abort[0])) break;
          tc_fence_after();
          mma_pv(tmem + g * kColTile + kColO, tmem + g * kColTile, aK + (iV % kSlots) * kTileBytes, idO, j > 0);
          if (more) {
            mma_qk(tmem + g * kColTile, smem_u32(sQ + g * kTileBytes), aK + (iK % kSlots) * kTileBytes, idS);
            tc_commit(&s_full[g]);
          }
        }
        if (!ok) break;
        tc_commit(&kv_empty[iV % kSlots]);
        if (more) tc_commit(&kv_empty[iK % kSlots]);
      }
      if (ok) tc_commit(o_full);
      else s_abort[0] = 1;
      tc_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else {
    // ---------------- warps 4 g .. 4 g + 3: softmax of query tile g; thread t owns unit
    // u0 + 128 g + t (TMEM lane t of the tile's columns)
    const int g = warp >> 2;
    const int t = threadIdx.x & 127;
    const int u = u0 + g * kTq + t;
    const bool valid = u < n_units;
    const int row = off + (valid ? u / G : 0);
    const int h = kvh * G + (valid ? u % G : 0);
    uint8_t* const qt = sQ + g * kTileBytes;
    // global element offset of unit ul's q / output row (any unit of the tile)
    auto unit_row = [&](int ul) -> int64_t {
      const int uu = u0 + g * kTq + ul;
      return static_cast<int64_t>(off + uu / G) * p.Hq + kvh * G + uu % G;
    };
    {
      // the tile's q vectors into the swizzled Q tile, zeros past the units: 16 consecutive
      // lanes read one unit's 256 B, so every load instruction covers two whole rows
      uint4 v[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int c = k * kTq + t, ul = c >> 4, ch = c & 15;
        v[k] = u0 + g * kTq + ul < n_units
                   ? __ldg(reinterpret_cast<const uint4*>(p.q + unit_row(ul) * kHd) + ch)
                   : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int c = k * kTq + t;
        *reinterpret_cast<uint4*>(qt + sw128_off(c >> 4, c & 15)) = v[k];
      }
      fence_async_shared();
      mbar_arrive(q_full);
    }
    if (g < ng) {
      const uint32_t lb = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + g * kColTile;
      const float sc = p.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      // per key tile: the tile's row maximum of S' = S log2(e) / sqrt(hd); the running
      // offset m moves up (O and l rescaled by 2^(m_old - m_new)) only when the tile's
      // maximum exceeds it by more than kSlack, so P = 2^(S' - m) <= 2^kSlack; then P in bf16
      // over the first 64 S columns and l += sum of P in fp32
      constexpr float kSlack = 8.f;
      for (int j = 0; ok && j < nb; ++j) {
        const bool late = !mbar_wait_sleep(&s_full[g], j & 1);
        if (group_any(late || s_abort[0], g)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int nvalid = min(kTk, p.N - (blk0 + j) * kTk);
        float mx;
        {
          float v[64];
          tmem_ld64(lb, v);
          mx = max64(v, nvalid);
          tmem_ld64(lb + 64, v);
          if (nvalid > 64) mx = fmaxf(mx, max64(v, nvalid - 64));
        }
        const float mt = mx * sc;                                  // sc > 0: the scale commutes with max
        const bool up = mt > m + kSlack;
        if (__any_sync(0xffffffffu, up) && j > 0) {
          // S_g(j) is complete, so every P V product before it is: O can be rescaled in place
          const float f = up ? ex2_approx(m - mt) : 1.f;
          l *= f;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            float o[64];
            tmem_ld64(lb + kColO + 64 * hf, o);
            uint32_t w[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) w[q] = __float_as_uint(o[q] * f);
            tmem_st32(lb + kColO + 64 * hf, w);
#pragma unroll
            for (int q = 0; q < 32; ++q) w[q] = __float_as_uint(o[32 + q] * f);
            tmem_st32(lb + kColO + 64 * hf + 32, w);
          }
        }
        if (up) m = mt;
        const float nm = -m;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          // keys 64 hf .. 64 hf + 63: read S columns 64 hf .., write P columns 32 hf .. (S
          // columns already read: 0 .. 63 by the first half)
          float v[64];
          tmem_ld64(lb + 64 * hf, v);
          uint32_t pk[32];
          p64(v, nvalid - 64 * hf, sc, nm, pk, l);
          tmem_st32(lb + 32 * hf, pk);
        }
        tc_fence_before();
        mbar_arrive(&p_full[g]);
      }
      // epilogue: O / l in bf16, or the unnormalised O and (m, l) of this key split
      if (ok) {
        const bool late = !mbar_wait_sleep(o_full, 0);
        ok = !group_any(late || s_abort[0], g);
      }
      if (ok) {
        tc_fence_after();
        const float inv = 1.f / l;
        // rows leave through the (now idle) Q tile: each thread writes its unit's row there,
        // then 16 consecutive lanes store one unit's 256 B, two whole rows per instruction.
        // One round for the bf16 row, two (64 columns each) for the fp32 split partial.
        const int64_t sbase = p.splits == 1 ? 0 : static_cast<int64_t>(split) * p.rows_cap * p.Hq;
        const int rounds = p.splits == 1 ? 1 : 2;
        for (int rd = 0; rd < rounds; ++rd) {
          uint4 w[16];
          if (p.splits == 1) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              float v[64];
              tmem_ld64(lb + kColO + 64 * hf, v);
#pragma unroll
              for (int c8 = 0; c8 < 8; ++c8)
                w[8 * hf + c8] = make_uint4(pack_bf16(v[8 * c8] * inv, v[8 * c8 + 1] * inv),
                                            pack_bf16(v[8 * c8 + 2] * inv, v[8 * c8 + 3] * inv),
                                            pack_bf16(v[8 * c8 + 4] * inv, v[8 * c8 + 5] * inv),
                                            pack_bf16(v[8 * c8 + 6] * inv, v[8 * c8 + 7] * inv));
            }
          } else {
            float v[64];
            tmem_ld64(lb + kColO + 64 * rd, v);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              w[e] = make_uint4(__float_as_uint(v[4 * e]), __float_as_uint(v[4 * e + 1]),
                                __float_as_uint(v[4 * e + 2]), __float_as_uint(v[4 * e + 3]));
          }
          group_bar(g);                                              // the previous round is out
#pragma unroll
          for (int ch = 0; ch < 16; ++ch)
            *reinterpret_cast<uint4*>(qt + t * 256 + ((ch ^ (t & 15)) << 4)) = w[ch];
          group_bar(g);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int c = k * kTq + t, ul = c >> 4, ch = c & 15;
            if (u0 + g * kTq + ul >= n_units) continue;
            const uint4 x = *reinterpret_cast<const uint4*>(qt + ul * 256 + ((ch ^ (ul & 15)) << 4));
            const int64_t r = sbase + unit_row(ul);
            if (p.splits == 1) reinterpret_cast<uint4*>(p.out + r * kHd)[ch] = x;
            else reinterpret_cast<uint4*>(p.opart + r * kHd + 64 * rd)[ch] = x;
          }
        }
        if (valid && p.splits > 1) p.ml[sbase + static_cast<int64_t>(row) * p.Hq + h] = make_float2(m, l);
      } else {
        s_abort[0] = 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 3-D map over a cache [B * Hkv][N][hd] (bf16), box 64 x 128 keys x 1 head, 128 B swizzle:
// a key tile that runs past N reads zeros instead of the next head's rows.  Cached: a step
// uses the same few caches in every layer.
int kv_tmap(CUtensorMap* m, const void* base, int BH, int N) {
  struct Key {
    const void* base;
    int BH, N;
    bool operator==(const Key& o) const { return base == o.base && BH == o.BH && N == o.N; }
  };
  struct Hash {
    size_t operator()(const Key& k) const {
      return reinterpret_cast<size_t>(k.base) ^ (static_cast<size_t>(k.BH) << 40) ^ (static_cast<size_t>(k.N) << 20);
    }
  };
  static std::mutex mu;
  static std::unordered_map<Key, CUtensorMap, Hash> cache;
  const Key key{base, BH, N};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *m = it->second;
      return DLLM_OK;
    }
  }
  auto enc = encode_fn();
  if (!enc) {
    set_last_error("cuTensorMapEncodeTiled unavailable", __FILE__, __LINE__);
    return DLLM_ERR_CUDA;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHd), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHd) * 2, static_cast<cuuint64_t>(N) * kHd * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTk), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[128];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d) for a K/V cache of %d heads x %d keys", (int)r, BH, N);
    set_last_error(buf, __FILE__, __LINE__);
    return DLLM_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() > 1024) cache.clear();
  cache.emplace(key, *m);
  return DLLM_OK;
}

}  // namespace

// Tensor-core path: head dimension 128 and at least kAttnTcMinUnits query units per
// (sequence, KV head); DLLM_ATTN_TC=0 / 1 forces the CUDA-core / tensor-core path where
// both apply (A/B measurements).
bool attn_use_tc(int hd, int G, int rows_per_seq) {
  static const int force = [] {
    const char* e = getenv("DLLM_ATTN_TC");
    return e ? atoi(e) : -1;
  }();
  if (hd != kHd || rows_per_seq <= 0) return false;
  if (force >= 0) return force != 0;
  return static_cast<int64_t>(rows_per_seq) * G >= kAttnTcMinUnits;
}

// Key splits of the tensor-core path: as many as keep the (sequence, KV head, query tile
// pair, split) CTAs within one wave over the SMs, never more than 128-key tiles.
int attn_tc_pick_splits(int B, int Hkv, int G, int rows_per_seq, int N) {
  const int64_t tiles = (static_cast<int64_t>(rows_per_seq) * G + kTq - 1) / kTq;
  const int64_t ctas = (tiles + kTiles - 1) / kTiles * B * Hkv;
  const int blocks = (N + kTk - 1) / kTk;
  const int sms = num_sms();
  if (ctas >= sms) return 1;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(sms / ctas, blocks)));   // at most one wave
}

// Launches the tensor-core kernel for p (p.splits key splits); the caller merges splits.
int attn_tc_run(const attn::AttnParams& p, int rows_per_seq_cap, cudaStream_t st) {
  if (p.Hq % p.Hkv) return DLLM_ERR_SHAPE;
  const int G = p.Hq / p.Hkv;
  TcParams tp;
  tp.a = p;
  tp.qtiles = static_cast<int>((static_cast<int64_t>(rows_per_seq_cap) * G + kTq - 1) / kTq);
  tp.blocks = (p.N + kTk - 1) / kTk;
  tp.blocks_per_split = (tp.blocks + p.splits - 1) / p.splits;
  if ((tp.blocks + tp.blocks_per_split - 1) / tp.blocks_per_split != p.splits) return DLLM_ERR_INVALID_ARG;
  CUtensorMap tk, tv;
  int rc = kv_tmap(&tk, p.kc, p.B * p.Hkv, p.N);
  if (rc) return rc;
  rc = kv_tmap(&tv, p.vc, p.B * p.Hkv, p.N);
  if (rc) return rc;
  rc = ensure_smem_attr(reinterpret_cast<const void*>(attn_tc_kernel), static_cast<int>(kSmemTc));
  if (rc) return rc;
  return launch_pdl(attn_tc_kernel, dim3((tp.qtiles + kTiles - 1) / kTiles, p.B * p.Hkv, p.splits), dim3(kThreadsTc),
                    kSmemTc, st, tk, tv, tp);
}

}  // namespace dllm
