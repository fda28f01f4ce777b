// moe_permute_noalloc: the dispatch step (histogram, scan, stable scatter,
// row gather) for callers that cannot hand the library a workspace.
//
// Who needs it: a caller whose device memory is entirely owned by its own
// pool or arena (an inference server that plans every byte up front, where an
// extra cudaMalloc either fails or takes memory the plan relies on); a caller
// that enqueues work while another thread is capturing a CUDA graph (a
// cudaMalloc there is either refused or breaks the capture); and
// latency-critical callers that cannot accept the device-wide synchronisation
// a cudaMalloc may imply.  This entry point needs no workspace at all: its
// scratch lives in a fixed-size array in the library's own device memory.
//
// The scratch is one file-scope __device__ array, reserved on every GPU that
// loads the library until the process exits.  Its device address is looked
// up (cudaGetSymbolAddress, with that device current) on the first call made
// in each CUDA context -- once per device for the usual primary context, and
// again after a context has been torn down and rebuilt (cudaDeviceReset),
// when the array may sit elsewhere -- so the first call in a context must come
// before any stream capture.  Every call on a device shares the array and it
// keeps the last call's contents: the histogram is cleared at the start of
// each call, and calls whose work overlaps on the GPU (concurrent streams)
// race on it.
#include <cmath>
#include <mutex>

#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

// 2 MiB + 64 KiB of int32: the per-chunk histogram and rank bases
// (2 x ceil(T/256) x E_r) plus the counts (E_r) and the error word.
constexpr size_t kScratchInts = (size_t)(2u << 20) / 4 + 16384;
constexpr int kChunkTokens = 256;

static __device__ __align__(256) int g_permute_scratch[kScratchInts];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (false when no
// context is current yet or the driver cannot say).  Ids are never reused
// within a process, unlike context handles.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
    looked_up = true;
  }
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

struct ScratchSlot {
  int* ptr = nullptr;
  unsigned long long ctx_id = 0;
};

std::mutex g_mu;
ScratchSlot g_slot[64];

// Device address of the scratch array in the current context: looked up on
// the first call in each context, then served from the per-device cache as
// long as the same context is current.
cudaError_t scratch_address(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchSlot& slot = g_slot[dev];
  unsigned long long id = 0;
  const bool known = current_context_id(&id);
  if (!slot.ptr || !known || slot.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);   // also makes the primary context current
    if (e != cudaSuccess) return e;
    slot.ptr = static_cast<int*>(p);
    // a context the driver cannot identify is looked up again on every call
    slot.ctx_id = current_context_id(&id) ? id : 0;
    if (!slot.ctx_id) { *out = slot.ptr; slot.ptr = nullptr; return cudaSuccess; }
  }
  *out = slot.ptr;
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* idx,
                                          const float* gates, const void* h, int32_t* offsets,
                                          int32_t* perm_tok, int32_t* row_of, int32_t* kept,
                                          float* row_gate, void* x_perm, int32_t* dev_error,
                                          void* stream) {
  size_t unused = 0;
  moe_status st = moe_workspace_size(cfg, &unused);     // validates the config
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (!idx || !offsets || !perm_tok || !row_of || !kept) return MOE_ERR_INVALID_ARG;
  if (!aligned(idx, 4) || !aligned(offsets, 4) || !aligned(perm_tok, 4) || !aligned(row_of, 4) ||
      !aligned(kept, 4) || !aligned(gates, 4) || !aligned(row_gate, 4) || !aligned(dev_error, 4) ||
      !aligned(h, 16) || !aligned(x_perm, 16))
    return MOE_ERR_INVALID_ARG;
  if ((row_gate && !gates) || (x_perm && !h)) return MOE_ERR_INVALID_ARG;
  const int n_chunks = (c.T + kChunkTokens - 1) / kChunkTokens;
  const size_t need = (size_t)2 * n_chunks * c.E_r + c.E_r + 64;
  if (need > kScratchInts) return MOE_ERR_UNSUPPORTED;   // T * E_r too large for the array

  int* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
  int* hist = base;
  int* chunk_base = hist + (size_t)n_chunks * c.E_r;
  int* counts = chunk_base + (size_t)n_chunks * c.E_r;
  int* err = dev_error ? dev_error : counts + c.E_r;

  int64_t cap = (int64_t)c.T * c.K;
  if (c.capacity_factor > 0.0f) {
    double v = std::floor((double)c.T * (double)c.K * (double)c.capacity_factor / (double)c.E_r);
    if (v < (double)cap) cap = (int64_t)v;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(hist, 0, (size_t)n_chunks * c.E_r * sizeof(int), s);   // the one buffer that must start at 0
  moe::launch_hist(idx, hist, 8, c.T, c.K, c.E_r, err, s);
  moe::launch_scan(hist, n_chunks, c.E_r, (int)cap, counts, kept, offsets, chunk_base, s);
  moe::launch_scatter(idx, gates, offsets, chunk_base, (int)cap, c.T, c.K, c.E_r, perm_tok, row_of,
                      row_gate, err, s);
  if (x_perm)
    moe::launch_gather(h, perm_tok, offsets + c.E_r, x_perm, c.d_model,
                       c.dtype == MOE_DTYPE_F32 ? 4 : 2, c.T * c.K, c.T, err, s);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
