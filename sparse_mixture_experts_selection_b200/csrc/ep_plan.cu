// moe_ep_plan: the exchange plan of an expert-parallel layer, built on the
// device from the per-expert row offsets of every rank.
//
// Expert parallelism ("Sparse Mixture-of-Experts (MoE): Routing Math, Load
// Balancing & Expert Parallelism", section 3: dispatch, grouped GEMM over the
// local experts, combine; "Mixture-of-Experts: Expert Parallelism, All-to-All
// Routing, and Auxiliary-Loss-Free Load Balancing", all-to-all routing): rank r
// owns experts r*E_loc .. (r+1)*E_loc - 1.  Each rank's permuted rows are
// expert-major, so what rank src sends to rank r is one contiguous range of
// its rows.  The receiving rank gets its rows source by source (each source's
// rows expert-major) and regroups them expert by expert, sources ascending,
// each source's rows in their order -- the order in which its grouped GEMM
// wants them.
//
// One block does it all: the counts a rank receives (W x E_loc <= 1024 of
// them) sit in shared memory, the small prefix sums run serially, and the
// warps then write the two maps, one (source, expert) segment per warp.
#include "common.cuh"

namespace {

using moe::kWarp;
using moe::set_device_error;

constexpr int kMaxWorld = 64;
constexpr int kMaxExperts = 1024;
constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads) ep_plan_kernel(const int* __restrict__ offs_all, int W, int rank,
                                                           int E_r, int max_recv, int* __restrict__ splits,
                                                           int* __restrict__ local_off, int* __restrict__ regroup,
                                                           int* __restrict__ inverse, int* err) {
  __shared__ int mine[kMaxExperts];         // [src][e]: rows of local expert e that src sends here
  __shared__ int tgt_base[kMaxExperts];     // [src][e]: first regrouped row of that segment
  __shared__ int rcv_base[kMaxExperts];     // [src][e]: first received row of that segment
  __shared__ int recv[kMaxWorld];
  __shared__ int src_base[kMaxWorld + 1];
  __shared__ int loc[kMaxExperts + 1];
  __shared__ int bad;
  const int tid = threadIdx.x;
  const int E_loc = E_r / W;
  const int stride = E_r + 1;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int i = tid; i < W * E_loc; i += blockDim.x) {
    const int src = i / E_loc, g = rank * E_loc + i % E_loc;
    int c = offs_all[src * stride + g + 1] - offs_all[src * stride + g];
    if (c < 0) { bad = 1; c = 0; }        // offsets must not decrease
    mine[i] = c;
  }
  if (tid < W) {                            // rows this rank sends to rank tid
    const int* o = offs_all + rank * stride;
    const int c = o[(tid + 1) * E_loc] - o[tid * E_loc];
    splits[tid] = c < 0 ? 0 : c;
    if (c < 0) bad = 1;
  }
  __syncthreads();
  if (tid < W) {
    int s = 0;
    for (int e = 0; e < E_loc; ++e) s += mine[tid * E_loc + e];
    recv[tid] = s;
    splits[W + tid] = s;
  }
  if (tid < E_loc) {                        // this expert's rows over all sources (kept in loc for the scan)
    int s = 0;
    for (int src = 0; src < W; ++src) s += mine[src * E_loc + tid];
    loc[tid + 1] = s;
  }
  __syncthreads();
  if (tid == 0) {
    loc[0] = 0;
    for (int e = 0; e < E_loc; ++e) loc[e + 1] += loc[e];
    src_base[0] = 0;
    for (int src = 0; src < W; ++src) src_base[src + 1] = src_base[src] + recv[src];
  }
  __syncthreads();
  if (tid < E_loc) {                        // regrouped rows: expert-major, sources ascending
    int at = loc[tid];
    for (int src = 0; src < W; ++src) {
      tgt_base[src * E_loc + tid] = at;
      at += mine[src * E_loc + tid];
    }
  }
  if (tid < W) {                            // received rows: source-major, experts ascending
    int at = src_base[tid];
    for (int e = 0; e < E_loc; ++e) {
      rcv_base[tid * E_loc + e] = at;
      at += mine[tid * E_loc + e];
    }
  }
  for (int e = tid; e <= E_loc; e += blockDim.x) local_off[e] = loc[e];
  __syncthreads();
  if (bad || src_base[W] > max_recv) {      // maps would not fit (or the offsets are corrupt)
    if (tid == 0) set_device_error(err, MOE_DEVERR_INDEX);
    return;
  }
  const int warp = tid / kWarp, lane = tid % kWarp, n_warps = blockDim.x / kWarp;
  for (int seg = warp; seg < W * E_loc; seg += n_warps) {
    const int n = mine[seg], t = tgt_base[seg], r = rcv_base[seg];
    for (int i = lane; i < n; i += kWarp) {
      regroup[t + i] = r + i;
      inverse[r + i] = t + i;
    }
  }
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" moe_status moe_ep_plan(const int32_t* offsets_all, int32_t world, int32_t rank, int32_t E_r,
                                  int32_t max_recv, int32_t* splits, int32_t* local_offsets,
                                  int32_t* regroup, int32_t* inverse, int32_t* dev_error, void* stream) {
  if (world < 1 || world > kMaxWorld || rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
  if (E_r < 1 || E_r > kMaxExperts || E_r % world) return MOE_ERR_INVALID_ARG;
  if (max_recv < 0) return MOE_ERR_INVALID_ARG;
  if (!offsets_all || !splits || !local_offsets || (max_recv > 0 && (!regroup || !inverse)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned4(offsets_all) || !aligned4(splits) || !aligned4(local_offsets) || !aligned4(regroup) ||
      !aligned4(inverse) || !aligned4(dev_error))
    return MOE_ERR_INVALID_ARG;
  ep_plan_kernel<<<1, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      offsets_all, world, rank, E_r, max_recv, splits, local_offsets, regroup, inverse, dev_error);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
