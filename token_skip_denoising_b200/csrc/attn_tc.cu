// Many-query attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// SureLock summary sec. 2.1 items 3-4: the recomputed rows attend to every position
// of their sequence through the cached K/V (bidirectional, no mask), O(M_t * N * d);
// ES-dLLM summary sec. 2.2: a refresh step recomputes every row, so there the query
// count equals the sequence length.  With many queries per (sequence, KV head) this
// is a pair of dense contractions, S = Q K^T and O = P V, so it runs on tcgen05:
//
//   one CTA per (sequence b, KV head, tile of 128 query units, key split), where a
//   unit is a (query row, query head of the KV head's group) pair, so the query heads
//   that share a KV head share its K/V tiles (grouped-query attention);
//   warps 0-7 load the q vectors into a 128-byte-swizzled K-major tile and run the
//   softmax and the output epilogue: thread (g, t) owns unit t (TMEM lane t) and key
//   columns 64 g .. 64 g + 63 of every S tile (the two warpgroups meet only to combine
//   the row maximum and the row sum);
//   warp 8 lane 0 streams 128-key K and V tiles with TMA through a ring of four 32 KB
//   slots (a 3-D tensor map [B * Hkv][N][hd] per cache: keys past N are zero-filled);
//   warp 9 lane 0 issues the MMAs and owns the TMEM allocation (two S buffers of
//   128 columns and the O accumulator of hd columns).
//
// The softmax takes two passes over the keys: the first computes S tile by tile and
// keeps only the row maximum m; the second computes S again, P = 2^(S' - m) with
// S' = S log2(e) / sqrt(hd) (its row sum l in fp32), writes P to shared memory in
// bf16 and accumulates O += P V in TMEM.  Knowing m before any P V product, O never
// needs rescaling, which keeps TMEM read by the epilogue only, once; the price is a
// second Q K^T (half again the MMA work) and no extra exponentials.  The result is
// O / l in bf16, or, with the keys split over several CTAs, the unnormalised O with
// (m, l) per (row, head) for the split merge, in the format of the CUDA-core path.
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
constexpr int kTq = 128;                         // query units per CTA (MMA M, TMEM lanes)
constexpr int kTk = 128;                         // keys per tile (MMA N of S, K of P V)
constexpr uint32_t kPanel = 128 * 128;           // one 128-row x 64-column bf16 panel (128 B rows)
constexpr uint32_t kTileBytes = 2 * kPanel;      // 128 rows x 128 columns bf16: two panels
constexpr int kSlots = 4;                        // K/V ring of 32 KB tiles
constexpr int kSoftmax = 256;                   // two warpgroups: key columns 0-63 and 64-127 of S
constexpr int kThreadsTc = kSoftmax + 64;
constexpr int kProducerWarp = kSoftmax / 32, kMmaWarp = kProducerWarp + 1;
constexpr uint32_t kTmemCols = 512;              // S[2] (2 x 128) + O (128), rounded to a power of two
constexpr uint32_t kColS = 0, kColO = 2 * kTk;

// Shared memory: Q tile, two P tiles, the K/V ring, barriers, the softmax halves' exchange.
constexpr size_t kOffQ = 0;
constexpr size_t kOffP = kOffQ + kTileBytes;
constexpr size_t kOffKV = kOffP + 2 * kTileBytes;
constexpr size_t kOffBar = kOffKV + static_cast<size_t>(kSlots) * kTileBytes;
constexpr size_t kOffRed = kOffBar + 256;                 // [2][128] floats: the halves' m, then l
constexpr size_t kSmemTc = 1024 + kOffRed + 2 * 128 * 4;
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

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// Barrier of the softmax threads that also returns whether any of them passed true.
__device__ __forceinline__ bool softmax_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

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

// 2^x by the MUFU instruction (relative error about 2^-22, inputs <= 0 here; P is rounded to
// bf16 afterwards, 2^-9).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// Byte offset of 16-byte chunk `ch` (0..15) of row r in a two-panel 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int ch) {
  return static_cast<uint32_t>((ch >> 3) * kPanel + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

struct TcParams {
  AttnParams a;
  int qtiles;            // 128-unit tiles per (sequence, KV head)
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
// O[d] (+)= P V over 128 keys: P K-major (keys contiguous), V MN-major (hd contiguous);
// a K = 16 step is 16 key rows of V, 2048 B into each of its two hd panels.
__device__ __forceinline__ void mma_pv(uint32_t d, uint32_t ap, uint32_t av, uint32_t idesc, bool acc) {
#pragma unroll
  for (int kk = 0; kk < kTk / 16; ++kk) {
    const uint32_t o = (kk >> 2) * kPanel + (kk & 3) * 32;
    tc_mma_f16(d, make_desc_k_sw128(ap + o), make_desc_mn_sw128(av + kk * 2048, kPanel), idesc,
               (acc || kk > 0) ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(kThreadsTc, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, TcParams tp) {
  const AttnParams& p = tp.a;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sP = smem + kOffP;                       // [2] P tiles
  uint8_t* sKV = smem + kOffKV;                     // [kSlots] K or V tiles
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_empty = kv_full + kSlots;
  uint64_t* s_full = kv_empty + kSlots;            // [2] S buffer written
  uint64_t* s_empty = s_full + 2;                   // [2] S buffer read (128 arrivals)
  uint64_t* p_full = s_empty + 2;                   // [2] P tile written (128 arrivals)
  uint64_t* p_empty = p_full + 2;                   // [2] P tile consumed by its P V product
  uint64_t* q_full = p_empty + 2;                   // Q tile written (128 arrivals)
  uint64_t* o_full = q_full + 1;                    // every P V product complete
  uint64_t* mma_done = o_full + 1;                  // every MMA issued complete (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int qt = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, kvh = blockIdx.y % p.Hkv;
  const int split = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  pdl_wait();                                       // q, the caches and seq_off come from earlier kernels
  const int off = p.seq_off[b];
  const int n_units = (p.seq_off[b + 1] - off) * G;
  const int u0 = qt * kTq;
  const int blk0 = split * tp.blocks_per_split;
  const int blk1 = min(tp.blocks, blk0 + tp.blocks_per_split);
  if (u0 >= n_units || blk0 >= blk1) return;        // uniform over the CTA
  const int nb = blk1 - blk0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kSoftmax);
      mbar_init(&p_full[i], kSoftmax);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(q_full, kSoftmax);
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
      // K_0 .. K_{nb-1} for the first pass, then K_j, V_j for the second
      const uint64_t pol = policy_evict_last();      // reread by the second pass and the other query tiles
      const int z = b * p.Hkv + kvh;
      const int n_slots = 3 * nb;
      int i = 0;
      for (; i < n_slots && !s_abort[0]; ++i) {
        const int s = i % kSlots;
        if (!mbar_wait(&kv_empty[s], ((i / kSlots) & 1) ^ 1) || s_abort[0]) {
          s_abort[0] = 1;
          break;
        }
        const bool second = i >= nb;
        const int j = second ? (i - nb) >> 1 : i;
        const CUtensorMap* tm = (second && ((i - nb) & 1)) ? &tmV : &tmK;
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
      // ---------------- MMA issuer
      constexpr uint32_t idS = make_idesc_bf16(kTq, kTk);
      constexpr uint32_t idO = make_idesc_bf16_bmn(kTq, kHd);
      const uint32_t aq = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0);
      auto slot_ready = [&](int i) -> bool {
        return mbar_wait(&kv_full[i % kSlots], (i / kSlots) & 1) && !s_abort[0];
      };
      // S from the K tile in slot i into S buffer `sidx & 1`; the slot is released once S is done
      auto issue_s = [&](int i, int sidx) -> bool {
        const int sb = sidx & 1;
        if (!mbar_wait(&s_empty[sb], ((sidx >> 1) & 1) ^ 1)) return false;
        if (!slot_ready(i)) return false;
        tc_fence_after();
        mma_qk(tmem + kColS + sb * kTk, aq, smem_u32(sKV + (i % kSlots) * kTileBytes), idS);
        tc_commit(&s_full[sb]);
        tc_commit(&kv_empty[i % kSlots]);
        return true;
      };
      // first pass: S only
      for (int j = 0; ok && j < nb; ++j) ok = issue_s(j, j);
      // second pass: S of tile j + 1 goes ahead of P_j V_j, so the softmax of j + 1 overlaps it
      if (ok) ok = issue_s(nb, nb);
      for (int j = 0; ok && j < nb; ++j) {
        if (j + 1 < nb && !(ok = issue_s(nb + 2 * (j + 1), nb + j + 1))) break;
        const int pb = j & 1;
        const int iv = nb + 2 * j + 1;
        if (!(ok = mbar_wait(&p_full[pb], (j >> 1) & 1) && slot_ready(iv))) break;
        tc_fence_after();
        mma_pv(tmem + kColO, smem_u32(sP + pb * kTileBytes), smem_u32(sKV + (iv % kSlots) * kTileBytes), idO, j > 0);
        tc_commit(&kv_empty[iv % kSlots]);
        tc_commit(&p_empty[pb]);
      }
      if (ok) tc_commit(o_full);
      else s_abort[0] = 1;
      tc_commit(mma_done);
      mbar_wait(mma_done, 0);
    }
  } else {
    // ---------------- warps 0-7: thread (wg, t) owns query unit u0 + t (TMEM lane t) and key
    // columns 64 wg .. 64 wg + 63 of every S tile; the two halves meet twice, for m and for l
    const int t = threadIdx.x & 127;
    const int wg = threadIdx.x >> 7;
    const int u = u0 + t;
    const bool valid = u < n_units;
    const int row = off + (valid ? u / G : 0);
    const int h = kvh * G + (valid ? u % G : 0);
    float* red = reinterpret_cast<float*>(smem + kOffRed);   // [2][128]
    {
      // half wg of the unit's q vector (128 B) into panel wg of row t of the Q tile; zeros past the units
      const uint4* src = reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(row) * p.Hq + h) * kHd) + wg * 8;
      uint4 v[8];
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) v[ch] = valid ? __ldg(src + ch) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(sQ + sw128_off(t, wg * 8 + ch)) = v[ch];
      fence_async_shared();
      mbar_arrive(q_full);
    }
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int col0 = wg * 64;
    const float sc = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // first pass: the row maximum of S' = S log2(e) / sqrt(hd) over the valid keys
    for (int j = 0; j < nb; ++j) {
      const int sb = j & 1;
      const bool late = !mbar_wait(&s_full[sb], (j >> 1) & 1);
      if (softmax_any(late || s_abort[0])) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int nvalid = min(kTk, p.N - (blk0 + j) * kTk) - col0;   // valid columns of this half
      float v[64];
      tmem_ld64(lane_base + kColS + sb * kTk + col0, v);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);                                   // S is in registers: the buffer is free
      if (nvalid > 0) m = fmaxf(m, max64(v, nvalid) * sc);         // sc > 0: the scale commutes with max
    }
    if (ok) {
      red[wg * 128 + t] = m;
      softmax_bar();
      m = fmaxf(red[t], red[128 + t]);
      softmax_bar();
    }
    // second pass: P = 2^(S' - m) in bf16 into panel wg of the P tile, l = sum of P in fp32
    for (int j = 0; ok && j < nb; ++j) {
      const int sidx = nb + j;
      const int sb = sidx & 1, pb = j & 1;
      const bool late = !mbar_wait(&s_full[sb], (sidx >> 1) & 1);
      if (softmax_any(late || s_abort[0])) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int nvalid = min(kTk, p.N - (blk0 + j) * kTk) - col0;
      float v[64];
      tmem_ld64(lane_base + kColS + sb * kTk + col0, v);
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      uint32_t pk[32];
      float lp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // independent partial sums
      const float nm = -m;
      if (nvalid >= 64) {
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
          const float p0 = q < nvalid ? ex2_approx(fmaf(v[q], sc, nm)) : 0.f;
          const float p1 = q + 1 < nvalid ? ex2_approx(fmaf(v[q + 1], sc, nm)) : 0.f;
          lp[(q >> 1) & 7] += p0 + p1;
          pk[q >> 1] = pack_bf16(p0, p1);
        }
      }
      l += ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
      // the P tile is free once the P V product two tiles back has completed
      if (!mbar_wait(&p_empty[pb], ((j >> 1) & 1) ^ 1)) s_abort[0] = 1;
      uint8_t* pt = sP + pb * kTileBytes;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8)
        *reinterpret_cast<uint4*>(pt + sw128_off(t, wg * 8 + c8)) =
            make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
      fence_async_shared();
      mbar_arrive(&p_full[pb]);
    }
    // epilogue: O / l in bf16, or the unnormalised O and (m, l) of this key split; each half
    // of the threads drains its 64 of the hd columns
    if (ok) {
      const bool late = !mbar_wait(o_full, 0);
      ok = !softmax_any(late || s_abort[0]);
    }
    if (ok) {
      red[wg * 128 + t] = l;
      softmax_bar();
      l = red[t] + red[128 + t];
      tc_fence_after();
      const float inv = 1.f / l;
      const int64_t base = p.splits == 1 ? static_cast<int64_t>(row) * p.Hq + h
                                         : (static_cast<int64_t>(split) * p.rows_cap + row) * p.Hq + h;
      float v[64];
      tmem_ld64(lane_base + kColO + col0, v);
      if (valid) {
        if (p.splits == 1) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + base * kHd + col0);
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8)
            dst[c8] = make_uint4(pack_bf16(v[8 * c8] * inv, v[8 * c8 + 1] * inv),
                                 pack_bf16(v[8 * c8 + 2] * inv, v[8 * c8 + 3] * inv),
                                 pack_bf16(v[8 * c8 + 4] * inv, v[8 * c8 + 5] * inv),
                                 pack_bf16(v[8 * c8 + 6] * inv, v[8 * c8 + 7] * inv));
        } else {
          float4* dst = reinterpret_cast<float4*>(p.opart + base * kHd + col0);
#pragma unroll
          for (int e = 0; e < 16; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          if (wg == 0) p.ml[base] = make_float2(m, l);
        }
      }
    } else {
      s_abort[0] = 1;
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

// Key splits of the tensor-core path: enough (sequence, KV head, query tile, split) CTAs
// for one wave over the SMs, never more splits than 128-key tiles.
int attn_tc_pick_splits(int B, int Hkv, int G, int rows_per_seq, int N) {
  const int qtiles = static_cast<int>((static_cast<int64_t>(rows_per_seq) * G + kTq - 1) / kTq);
  const int ctas = qtiles * B * Hkv;
  const int blocks = (N + kTk - 1) / kTk;
  const int sms = num_sms();
  if (ctas >= sms) return 1;
  return std::max(1, std::min((sms + ctas - 1) / ctas, blocks));
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
  return launch_pdl(attn_tc_kernel, dim3(tp.qtiles, p.B * p.Hkv, p.splits), dim3(kThreadsTc), kSmemTc, st, tk, tv, tp);
}

}  // namespace dllm
