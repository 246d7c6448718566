// Shared declarations of the CUDA path: status codes, launch-side structs and
// the host entry points of each kernel family.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <utility>

#include "../../include/dllm.h"

namespace dllm {

// SMs of the current device, queried once per device (148 on a B200).  Grids and the
// scratch sized from them follow the device; with no device at all (a sizing call on a
// host without a GPU) it returns kDefaultSMs.
constexpr int kDefaultSMs = 148;
int num_sms();
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) for `fn`, once per device and function
// (thread-safe): a launch on a second device sets it there too.
int ensure_smem_attr(const void* fn, int bytes);

#define DLLM_CUDA_TRY(expr)                                                   \
  do {                                                                        \
    cudaError_t _e = (expr);                                                  \
    if (_e != cudaSuccess) {                                                  \
      dllm::set_last_error(cudaGetErrorString(_e), __FILE__, __LINE__);      \
      return DLLM_ERR_CUDA;                                                   \
    }                                                                         \
  } while (0)

void set_last_error(const char* msg, const char* file, int line);

// Kernels launched by this library in the process (reported by dllm_kernel_launches).
extern std::atomic<int64_t> g_kernel_launches;
inline void count_launch(int n = 1) { g_kernel_launches.fetch_add(n, std::memory_order_relaxed); }

// Launch with programmatic dependent launch: the kernel may be scheduled while the
// previous kernel on the stream is still running; every kernel of this library calls
// pdl_wait() before it touches memory an earlier kernel produced, and pdl_trigger()
// as soon as its own dependents may be scheduled.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  static const bool pdl_off = getenv("DLLM_NO_PDL") != nullptr;   // A/B switch for measurements
  cfg.numAttrs = pdl_off ? 0 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  count_launch();
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e), __FILE__, __LINE__);
    return DLLM_ERR_CUDA;
  }
  return DLLM_OK;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ GEMM
// C[j, n] = sum_k X[j, k] * W[n, k]: X holds the active rows (K-major), W the
// weight matrix [out, in] (K-major).  One CTA computes a 128 (W rows) x BN
// (rows of X) tile with tcgen05 into TMEM; the epilogue is fused.
enum EpiKind : int {
  EPI_STORE_F32 = 0,   // out_f32[j * ldo + n]
  EPI_STORE_BF16 = 1,  // out_bf16[r * ldo + n], r = row_map ? row_map[j] : j
  EPI_RESID_ADD = 3,   // h[row_map[j] * ldh + n] += C
  EPI_SWIGLU = 4,      // act[j * F + f] = silu(gate) * up   (W tile = 64 gate + 64 up rows)
  EPI_LMHEAD = 5,      // per (row, 128-vocab tile): max, sum exp, argmax (mask id excluded)
};

struct EpiParams {
  int kind = EPI_STORE_F32;
  void* out = nullptr;
  int64_t ldo = 0;
  const int* row_map = nullptr;     // row j -> output row (scatter kinds)
  // residual
  float* h = nullptr;
  int64_t ldh = 0;
  // SwiGLU
  __nv_bfloat16* act = nullptr;
  int ffn = 0;
  // LM head partials: [rows, n_vtiles] of {max, sumexp, best value, best id}
  float4* lm_part = nullptr;
  int n_vtiles = 0;
  int mask_id = -1;
};

struct GemmArgs {
  const void* W = nullptr;       // bf16 [w_rows_total, K]
  int64_t w_rows_total = 0;
  const void* X = nullptr;       // bf16 [rows_cap, K]
  int rows_cap = 0;              // host bound on the number of X rows
  const int* rows_dev = nullptr; // device count of valid rows (nullable: rows_cap)
  int K = 0;
  int n_tiles_w = 0;             // 128-row output tiles (SwiGLU: F / 64)
  bool swiglu = false;
  // the activation tile may be 256 wide for 129-256 rows (one tile instead of two): faster for
  // a weight matrix of many 128-row tiles whose epilogue is a plain store (QKV), not for the rest
  bool wide_ok = false;
  EpiParams epi;
};

struct GemmScratch {
  float* partial = nullptr;      // split-K partial tiles
  size_t partial_floats = 0;
  int* counters = nullptr;       // one per output tile, zero between launches
  int n_counters = 0;
};

// Launch one fused GEMM; returns a DLLM_* status.
int gemm_launch(const GemmArgs& a, const GemmScratch& s, cudaStream_t st, int force_splits = 0,
                int force_bn = 0);
// Scratch floats a launch with these sizes needs (upper bound over tile choices).
size_t gemm_partial_floats(int rows_cap, int n_tiles_w, int K);
int gemm_counters_needed(int rows_cap, int n_tiles_w);

// Combine LM-head partials into conf / argmax / lse per row; rows are written at
// out_index[j] (nullable: j).
int lmhead_combine_launch(const float4* part, int n_vtiles, int rows_cap, const int* rows_dev,
                          const int* out_index, float* conf, int* amax, float* lse, cudaStream_t st);

}  // namespace dllm
