// Device pieces shared by the GEMM kernels: tile constants, the stream-K partition,
// warp reductions and the fused epilogue of one 16-column chunk.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace dllm {
namespace gemm {

constexpr int kBK = 64;                      // K elements per stage (128 B rows, one swizzle span)
constexpr int kTileM = 128;                  // weight rows per tile
constexpr uint32_t kABytes = kTileM * kBK * 2;

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Barrier `id` of 128 threads (one epilogue group of four warps).
__device__ __forceinline__ void grp_bar(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
// Barrier `id` of `n` threads that also returns whether any of them passed true.
__device__ __forceinline__ bool bar_any(bool v, int id, int n) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Barrier of the 128 epilogue threads that also returns whether any of them passed true,
// so that every branch taken after it is the same for all of them.
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

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

// Stream-K partition: CTA c owns the k-block iterations [lo(c), lo(c + 1)) of the
// flattened (tile, k-block) space; first_cta(x) is the CTA whose range holds x.
__device__ __forceinline__ int64_t sk_lo(int64_t T, int G, int c) { return T * c / G; }
__device__ __forceinline__ int sk_first_cta(int64_t x, int64_t T, int G) {
  return static_cast<int>(((x + 1) * G + T - 1) / T - 1);
}

// Epilogue of one 16-column chunk (columns = activation rows jbase..jbase+15) for the
// weight row n held by TMEM lane t (warp = t / 32).  Exchange kinds synchronise the 128
// threads of the epilogue group through named barrier `bar` and its buffer xb.
template <int XP>
__device__ __forceinline__ void epi_chunk(const EpiParams& e, const float (&v)[16], int t, int lane, int warp, int n,
                                          int jbase, int m_rows, int tw, float* xb, int bar = 1) {
  switch (e.kind) {
    case EPI_STORE_F32: {
      float* o = static_cast<float*>(e.out);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (jbase + i < m_rows) o[static_cast<int64_t>(jbase + i) * e.ldo + n] = v[i];
      break;
    }
    case EPI_STORE_BF16: {
      // row j lands at row row_map[j] of the output when a map is given (scatter)
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(e.out);
      int rr[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        rr[i] = (jbase + i < m_rows) ? (e.row_map ? __ldg(e.row_map + jbase + i) : jbase + i) : -1;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (rr[i] >= 0) o[static_cast<int64_t>(rr[i]) * e.ldo + n] = __float2bfloat16(v[i]);
      break;
    }
    case EPI_RESID_ADD: {
      // a reduction, not a load and a store, so nothing waits for the load; the tile's owner
      // adds the whole sum, or (from 128-wide tiles on) each k piece of a split tile adds its own
      int rr[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        rr[i] = (jbase + i < m_rows) ? (e.row_map ? __ldg(e.row_map + jbase + i) : jbase + i) : -1;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (rr[i] >= 0) atomicAdd(e.h + static_cast<int64_t>(rr[i]) * e.ldh + n, v[i]);
      break;
    }
    case EPI_SWIGLU: {
      // lanes 0-63 hold gate rows, lanes 64-127 the matching up rows
#pragma unroll
      for (int i = 0; i < 16; ++i) xb[t * XP + i] = v[i];
      grp_bar(bar);
      if (t < 64) {
        const int f = tw * 64 + t;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int j = jbase + i;
          if (j < m_rows) {
            const float g = v[i];
            const float u = xb[(t + 64) * XP + i];
            e.act[static_cast<int64_t>(j) * e.ffn + f] = __float2bfloat16(g / (1.f + __expf(-g)) * u);
          }
        }
      }
      grp_bar(bar);
      break;
    }
    case EPI_LMHEAD: {
      // per row j: max, sum exp(x - max) and argmax over this tile's 128 vocabulary ids
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
      grp_bar(bar);
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
      grp_bar(bar);
      break;
    }
    default:
      break;
  }
}


}  // namespace gemm
}  // namespace dllm
