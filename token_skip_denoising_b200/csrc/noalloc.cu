// An allocation-free variant of the active-row GEMM entry point.
//
// dllm_op_gemm takes a caller workspace for its split-tile scratch (tile
// counters and partial tiles).  Some callers have no workspace to give: a host
// framework that owns all device memory and hands a plugin only its input and
// output buffers, or a caller that must not call cudaMalloc on its hot path
// because it synchronises the device and can fail under memory pressure.  For
// them dllm_op_gemm_noalloc keeps that scratch in a fixed array in this
// library's device image, so the call itself allocates nothing.
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace dllm {
namespace {

// Largest problem the fixed scratch serves: up to 32 activation rows (one tile
// of the 32-wide MMA) and up to 4096 output tiles of 128 rows, with one partial
// tile pair per CTA of a grid of at most 148 CTAs (a device with more SMs runs
// this call on 148 of them).
constexpr int kNoAllocMaxRows = 32;
constexpr int kNoAllocMaxTiles = 4096;
constexpr int kNoAllocMaxGrid = 148;
constexpr size_t kNoAllocCounterBytes = kNoAllocMaxTiles * sizeof(int);
constexpr size_t kNoAllocPartialFloats = static_cast<size_t>(kNoAllocMaxGrid) * 2 * kNoAllocMaxRows * 128;
constexpr size_t kNoAllocBytes = kNoAllocCounterBytes + kNoAllocPartialFloats * sizeof(float);   // ~4.9 MB

// The scratch: one copy per device that loads the library, held until the process exits.
// Host code must not pass `g_noalloc_scratch` itself to a kernel (on the host it names a
// host-side stand-in); it uses the device address fetched below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device; the first call on a device looks
// it up (cudaGetSymbolAddress) with that device current.
int scratch_address(void** out) {
  int dev = -1;
  DLLM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) {
    set_last_error("device ordinal outside the no-alloc table", __FILE__, __LINE__);
    return DLLM_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      set_last_error(cudaGetErrorString(e), __FILE__, __LINE__);
      return DLLM_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DLLM_OK;
}

}  // namespace
}  // namespace dllm

using namespace dllm;

extern "C" int dllm_op_gemm_noalloc(int32_t kind, const void* W, int32_t n_out, const void* X, int32_t rows_cap,
                                    const int32_t* count, int32_t K, void* out, const int32_t* rows_map,
                                    void* stream) {
  if (!W || !X || !out || rows_cap <= 0 || K <= 0 || n_out <= 0) {
    set_last_error("bad gemm_noalloc args", __FILE__, __LINE__);
    return DLLM_ERR_INVALID_ARG;
  }
  if (kind != EPI_STORE_F32 && kind != EPI_STORE_BF16 && kind != EPI_RESID_ADD) {
    set_last_error("kind must be 0, 1 or 3", __FILE__, __LINE__);
    return DLLM_ERR_INVALID_ARG;
  }
  if (n_out % 128 || K % 64) {
    set_last_error("n_out must be a multiple of 128 and K of 64", __FILE__, __LINE__);
    return DLLM_ERR_SHAPE;
  }
  if (rows_cap > kNoAllocMaxRows || n_out / 128 > kNoAllocMaxTiles) {
    set_last_error("dllm_op_gemm_noalloc serves at most 32 rows and 4096 output tiles of 128 (n_out <= 524288); "
                   "use dllm_op_gemm with a workspace for larger problems",
                   __FILE__, __LINE__);
    return DLLM_ERR_SHAPE;
  }
  void* base = nullptr;
  const int rc = scratch_address(&base);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int tiles = n_out / 128;   // one activation tile: rows_cap <= 32
  GemmScratch gs;
  gs.counters = static_cast<int*>(base);
  gs.n_counters = tiles;
  gs.partial = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kNoAllocCounterBytes);
  gs.partial_floats = kNoAllocPartialFloats;
  // the array keeps whatever the last call left: the tile counters must start at zero
  DLLM_CUDA_TRY(cudaMemsetAsync(gs.counters, 0, tiles * sizeof(int), st));
  GemmArgs a;
  a.W = W; a.w_rows_total = n_out; a.X = X; a.rows_cap = rows_cap; a.rows_dev = count; a.K = K;
  a.n_tiles_w = tiles;
  a.epi.kind = kind;
  if (kind == EPI_RESID_ADD) {
    a.epi.h = static_cast<float*>(out); a.epi.ldh = n_out; a.epi.row_map = rows_map;
  } else {
    a.epi.out = out; a.epi.ldo = n_out;
  }
  return gemm_launch(a, gs, st, std::min(num_sms(), kNoAllocMaxGrid), 0);
}
