// Device code of the active-query attention, shared by the stand-alone kernels and
// the fused layer kernel: the flash-style block loop over one (sequence, KV head,
// query tile, key split) item, and the merge of split partials for one (row, head).
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace dllm {
namespace attn {

constexpr int kKeysPerBlock = 64;
constexpr int kUnitsPerCta = 64;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = smem_u32(smem);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct AttnParams {
  const __nv_bfloat16* q;      // [rows, Hq * hd]
  const __nv_bfloat16* kc;     // [B, Hkv, N, hd]
  const __nv_bfloat16* vc;
  __nv_bfloat16* out;          // [rows, Hq * hd]
  const int* seq_off;          // [B + 1] row offsets of each sequence (device)
  int B, N, Hq, Hkv;
  int rows_cap;
  int splits;
  int blocks_per_split;
  float scale_log2;            // log2(e) / sqrt(hd)
  float* opart;                // [splits, rows_cap, Hq, hd]
  float2* ml;                  // [splits, rows_cap, Hq]
};

// One work item with 128 threads (tid 0..127, four warps of 16 query units each).
// `bar` synchronises those 128 threads; `smem` holds 4 * 64 * HD * 2 bytes.
template <int HD, class Bar>
__device__ __forceinline__ void attn_item(const AttnParams& p, int qt, int b, int kvh, int split, uint8_t* smem,
                                          int tid, Bar bar) {

  constexpr int kChunks = HD / 8;                      // 16-byte chunks per key row
  constexpr int kTileBytes = kKeysPerBlock * HD * 2;
  uint8_t* kbuf[2] = {smem, smem + 2 * kTileBytes};
  uint8_t* vbuf[2] = {smem + kTileBytes, smem + 3 * kTileBytes};

  const int G = p.Hq / p.Hkv;
  const int off = p.seq_off[b];
  const int cnt = p.seq_off[b + 1] - off;
  const int n_units = cnt * G;
  const int u0 = qt * kUnitsPerCta;
  if (u0 >= n_units) return;

  const int n_blocks = (p.N + kKeysPerBlock - 1) / kKeysPerBlock;
  const int blk0 = split * p.blocks_per_split;
  const int blk1 = min(n_blocks, blk0 + p.blocks_per_split);
  if (blk0 >= blk1) return;

  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int wu0 = u0 + warp * 16;                      // first unit of this warp
  const bool warp_active = wu0 < n_units;

  const __nv_bfloat16* kbase = p.kc + (static_cast<int64_t>(b) * p.Hkv + kvh) * p.N * HD;
  const __nv_bfloat16* vbase = p.vc + (static_cast<int64_t>(b) * p.Hkv + kvh) * p.N * HD;

  auto load_block = [&](int blk, int buf) {
    const int key0 = blk * kKeysPerBlock;
    for (int i = tid; i < kKeysPerBlock * kChunks; i += 128) {
      const int r = i / kChunks, ch = i % kChunks;
      const int key = key0 + r;
      const bool ok = key < p.N;
      const int64_t go = static_cast<int64_t>(ok ? key : 0) * HD + ch * 8;
      const int so = r * (HD * 2) + ((ch ^ (r & 7)) * 16);
      cp_async16(kbuf[buf] + so, kbase + go, ok);
      cp_async16(vbuf[buf] + so, vbase + go, ok);
    }
    cp_async_commit();
  };

  // Q fragments of this warp's 16 units (rows g and g + 8)
  uint32_t qa[HD / 16][4];
  {
    const int ua = wu0 + g, ub = wu0 + g + 8;
    const bool va = ua < n_units, vb = ub < n_units;
    const __nv_bfloat16* qa_row = p.q + (static_cast<int64_t>(off + (va ? ua / G : 0)) * p.Hq + kvh * G + (va ? ua % G : 0)) * HD;
    const __nv_bfloat16* qb_row = p.q + (static_cast<int64_t>(off + (vb ? ub / G : 0)) * p.Hq + kvh * G + (vb ? ub % G : 0)) * HD;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const int d0 = kk * 16 + 2 * c;
      // read through L2: in the fused layer other SMs wrote q earlier in the same launch
      qa[kk][0] = va ? __ldcg(reinterpret_cast<const unsigned int*>(qa_row + d0)) : 0u;
      qa[kk][1] = vb ? __ldcg(reinterpret_cast<const unsigned int*>(qb_row + d0)) : 0u;
      qa[kk][2] = va ? __ldcg(reinterpret_cast<const unsigned int*>(qa_row + d0 + 8)) : 0u;
      qa[kk][3] = vb ? __ldcg(reinterpret_cast<const unsigned int*>(qb_row + d0 + 8)) : 0u;
    }
  }

  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  load_block(blk0, 0);
  for (int blk = blk0, it = 0; blk < blk1; ++blk, ++it) {
    const int buf = it & 1;
    if (blk + 1 < blk1) {
      load_block(blk + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    bar();
    if (warp_active) {
      const uint32_t ks = smem_u32(kbuf[buf]);
      const uint32_t vs = smem_u32(vbuf[buf]);
      float s[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          const int mi = lane >> 3;
          const int key = (nt + (mi >> 1)) * 8 + (lane & 7);
          const int ch = 2 * kk + (mi & 1);
          const uint32_t addr = ks + key * (HD * 2) + ((ch ^ (key & 7)) * 16);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_bf16(s[nt], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
          mma_bf16(s[nt + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
        }
      }
      // mask keys beyond N, scale to log2 domain, online softmax
      const int key0 = blk * kKeysPerBlock;
      float mx_a = m_a, mx_b = m_b;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + nt * 8 + 2 * c + (e & 1);
          s[nt][e] = key < p.N ? s[nt][e] * p.scale_log2 : -INFINITY;
        }
        mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
        mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
      }
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
      const float corr_a = exp2f(m_a - mx_a), corr_b = exp2f(m_b - mx_b);
      m_a = mx_a;
      m_b = mx_b;
      float rs_a = 0.f, rs_b = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = exp2f(s[nt][0] - m_a);
        s[nt][1] = exp2f(s[nt][1] - m_a);
        s[nt][2] = exp2f(s[nt][2] - m_b);
        s[nt][3] = exp2f(s[nt][3] - m_b);
        rs_a += s[nt][0] + s[nt][1];
        rs_b += s[nt][2] + s[nt][3];
      }
      l_a = l_a * corr_a + rs_a;
      l_b = l_b * corr_b + rs_b;
#pragma unroll
      for (int i = 0; i < HD / 8; ++i) {
        o[i][0] *= corr_a;
        o[i][1] *= corr_a;
        o[i][2] *= corr_b;
        o[i][3] *= corr_b;
      }
      // O += P V
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t a0 = pack_bf16(s[2 * t][0], s[2 * t][1]);
        const uint32_t a1 = pack_bf16(s[2 * t][2], s[2 * t][3]);
        const uint32_t a2 = pack_bf16(s[2 * t + 1][0], s[2 * t + 1][1]);
        const uint32_t a3 = pack_bf16(s[2 * t + 1][2], s[2 * t + 1][3]);
#pragma unroll
        for (int dn = 0; dn < HD / 8; dn += 2) {
          const int mi = lane >> 3;
          const int key = 16 * t + (mi & 1) * 8 + (lane & 7);
          const int ch = dn + (mi >> 1);
          const uint32_t addr = vs + key * (HD * 2) + ((ch ^ (key & 7)) * 16);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
          mma_bf16(o[dn], a0, a1, a2, a3, b0, b1);
          mma_bf16(o[dn + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    bar();
  }

  if (!warp_active) return;
  // full row sums across the quad
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int u = wu0 + g + half * 8;
    if (u >= n_units) continue;
    const int row = off + u / G;
    const int h = kvh * G + u % G;
    const float l = half ? l_b : l_a;
    const float m = half ? m_b : m_a;
    if (p.splits == 1) {
      const float inv = 1.f / l;
      __nv_bfloat16* dst = p.out + (static_cast<int64_t>(row) * p.Hq + h) * HD;
#pragma unroll
      for (int dn = 0; dn < HD / 8; ++dn) {
        const int d = dn * 8 + 2 * c;
        *reinterpret_cast<uint32_t*>(dst + d) = pack_bf16(o[dn][half * 2] * inv, o[dn][half * 2 + 1] * inv);
      }
    } else {
      const int64_t base = (static_cast<int64_t>(split) * p.rows_cap + row) * p.Hq + h;
      float* dst = p.opart + base * HD;
#pragma unroll
      for (int dn = 0; dn < HD / 8; ++dn) {
        const int d = dn * 8 + 2 * c;
        *reinterpret_cast<float2*>(dst + d) = make_float2(o[dn][half * 2], o[dn][half * 2 + 1]);
      }
      if (c == 0) p.ml[base] = make_float2(m, l);
    }
  }
}

// Merge of the split partials for one (row, head), one warp (lane 0..31).
template <int HD>
__device__ __forceinline__ void attn_merge(const AttnParams& p, int row, int h, int lane) {
  constexpr int PER = HD / 32;
  constexpr int kMaxUnrolled = 8;
  if (p.splits <= kMaxUnrolled) {
    // every split's (m, l) and partial row requested at once: two round trips in all
    float2 v[kMaxUnrolled];
#pragma unroll
    for (int s = 0; s < kMaxUnrolled; ++s)
      v[s] = s < p.splits ? __ldcg(&p.ml[(static_cast<int64_t>(s) * p.rows_cap + row) * p.Hq + h])
                          : make_float2(-INFINITY, 0.f);
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kMaxUnrolled; ++s) M = fmaxf(M, v[s].x);
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float L = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxUnrolled; ++s) {
      if (s < p.splits) {
        const int64_t base = (static_cast<int64_t>(s) * p.rows_cap + row) * p.Hq + h;
        const float w = (v[s].x == -INFINITY) ? 0.f : exp2f(v[s].x - M);
        L += w * v[s].y;
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] += w * __ldcg(p.opart + base * HD + lane + 32 * i);
      }
    }
    const float inv = 1.f / L;
    __nv_bfloat16* dst = p.out + (static_cast<int64_t>(row) * p.Hq + h) * HD;
#pragma unroll
    for (int i = 0; i < PER; ++i) dst[lane + 32 * i] = __float2bfloat16(acc[i] * inv);
    return;
  }
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) {
    const float2 v = __ldcg(&p.ml[(static_cast<int64_t>(s) * p.rows_cap + row) * p.Hq + h]);
    M = fmaxf(M, v.x);
  }
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float L = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const int64_t base = (static_cast<int64_t>(s) * p.rows_cap + row) * p.Hq + h;
    const float2 v = __ldcg(&p.ml[base]);
    const float w = (v.x == -INFINITY) ? 0.f : exp2f(v.x - M);
    L += w * v.y;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] += w * __ldcg(p.opart + base * HD + lane + 32 * i);
  }
  const float inv = 1.f / L;
  __nv_bfloat16* dst = p.out + (static_cast<int64_t>(row) * p.Hq + h) * HD;
#pragma unroll
  for (int i = 0; i < PER; ++i) dst[lane + 32 * i] = __float2bfloat16(acc[i] * inv);
}

}  // namespace attn
}  // namespace dllm
