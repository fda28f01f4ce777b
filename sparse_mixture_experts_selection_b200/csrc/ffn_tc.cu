// Grouped SwiGLU experts on the 5th-generation tensor cores (sm_100a):
// tcgen05.mma with bf16 operands staged in shared memory by TMA and fp32
// accumulators in tensor memory (TMEM), one persistent CTA per SM.
//
//   gate/up GEMM:  D = X W_gate^T | X W_up^T      epilogue: act = SiLU(gate) * up -> bf16
//   down GEMM:     D = act W_down^T                epilogue: out = g_{t,i} * D     -> bf16
//
// SwiGLU(h) = (SiLU(h W_gate^T) * (h W_up^T)) W_down^T and the gate-weighted
// routed sum follow "Sparse Mixture-of-Experts (MoE): Routing Math, Load
// Balancing & Expert Parallelism" (section 0 layer equation; section 3: all
// local experts run as one grouped GEMM over their variable-length row groups).
//
// Work unit = (group, 128-row tile, 256-column B tile).  Groups are the routed
// experts (expert-contiguous rows of the permuted activations) followed by the
// shared experts (all T tokens); the unit -> group map is a device-side prefix
// sum, so per-expert row counts never travel to the host.  Units are ordered
// row-tile fastest, so the CTAs running at the same time share weight tiles
// through L2 and each expert's weights stream from HBM about once.
//
// Warp roles (192 threads): warp 0 = TMA producer (+ TMEM allocation), warp 1 =
// MMA issuer (one thread), warps 2..5 = epilogue (TMEM -> registers -> global).
// Accumulators are double-buffered in TMEM (2 x 256 fp32 columns) so the
// epilogue of one unit overlaps the MMAs of the next.
//
// Short row tiles (an expert's last tile holding at most kSwapMaxRows rows) are
// computed transposed: the weight tile is the M = 128 operand and the n rows
// the N = round16(n) operand, D^T = W X^T, so the tensor cores do n/128 of a
// full tile's work instead of padding the rows up to 128.  A tail of at most
// kMergeMaxRows rows rides in the same unit as the full tile before it: each
// stage then holds the full tile's rows, the tail's rows and ONE copy of the
// weight tile, which feeds both the normal MMA and the transposed tail MMA.
// Experts of a little more than 128 tokens -- the common case when T*K/E_r is
// near 128 -- thus stream their weights through shared memory once, not twice,
// and spend no MMAs on padding.  Such a unit holds both TMEM accumulators; its
// epilogue drains the short tail first and the next unit takes the tail's
// buffer, so only the unit before it waits for a whole epilogue.
#include <algorithm>
#include <cuda.h>
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace tc {

constexpr int BM = 128;                         // rows per tile (MMA M)
constexpr int BN = 256;                         // B rows per tile (MMA N)
constexpr int BK = 64;                          // K per stage: one 128-byte swizzle atom of bf16
constexpr int UMMA_K = 16;
// Output tiles may leave through shared memory (kernel template TMA_OUT): each
// epilogue warp stages a 32-row x 64-column bf16 box (128-byte swizzle) and one
// TMA tensor store writes it as whole 128-byte lines, instead of 32 threads
// each storing 16 bytes of a different row.  The staging space (32 KB) costs
// one stage of the operand pipeline, which long reductions feel more than
// their stores: the launch picks it for the down GEMM when its units are short
// (at most kTmaOutMaxKb k-blocks), where the fine-grained stores of 128 x 256
// outputs per unit compete with the weight stream.
constexpr int kTmaOutMaxKb = 64;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int kSwapMaxRows = 96;                // tiles of <= this many rows run transposed
constexpr int kMergeMaxRows = 64;               // tails of <= this many rows join the tile before
constexpr int A_SUB_ROWS = 32;                  // row box of the transposed tiles' token loads
constexpr int A_SUB_BYTES = A_SUB_ROWS * BK * 2;
constexpr int T_BYTES = kMergeMaxRows * BK * 2; // 8 KB: a merged tail's rows per stage
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;                  // 2 accumulators x 256 columns
constexpr int OUT_BOX_ROWS = 32;                // one epilogue warp's rows
constexpr int OUT_BOX_BYTES = OUT_BOX_ROWS * 128;   // 32 rows x 64 bf16 columns
constexpr int CTRL_BYTES = 512;                  // barriers and the unit ring

enum { EPI_SWIGLU = 0, EPI_SCALE = 1, EPI_ROUTER = 2 };

// pipeline stages and shared memory with and without the output staging boxes
template <bool TMA_OUT> constexpr int stages_of() { return TMA_OUT ? 3 : 4; }
template <bool TMA_OUT> constexpr int out_bytes_of() { return TMA_OUT ? 4 * 2 * OUT_BOX_BYTES : 0; }
template <bool TMA_OUT> constexpr size_t smem_of() {
  return (size_t)stages_of<TMA_OUT>() * (STAGE_BYTES + T_BYTES) + out_bytes_of<TMA_OUT>() + 1024 + CTRL_BYTES;
}
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
constexpr uint32_t IDESC_Q8 = idesc_e4m3_f32(BM, BN);
static_assert(smem_of<true>() <= 232448 && smem_of<false>() <= 232448, "shared memory per CTA");

struct Params {
  CUtensorMap a_r, a_s;       // A: routed rows / shared rows
  CUtensorMap a32_r, a32_s;   // the same with a 32-row box (transposed tiles)
  CUtensorMap b0_r, b1_r;     // routed B: gate & up (SWIGLU) or down (b0 only)
  CUtensorMap b0_s, b1_s;     // shared B
  CUtensorMap o_r, o_s;       // outputs (routed / shared), boxes of 32 rows x 64 columns
  const int* grp_rows;
  const int* grp_row0;
  const int* prefix;          // [G + 1] unit prefix
  int G, E_r;
  int k_r, k_s;               // reduction length (routed / shared)
  int wrows_r, wrows_s;       // B rows per expert in the stacked weight tensors
  int ncols_r, ncols_s;       // output columns
  uint16_t* out_r;
  uint16_t* out_s;
  const float* row_scale;     // routed rows' gates (EPI_SCALE), may be null
  int* err;
  // EPI_ROUTER: z partial sums over split-K ranges of the virtual reduction
  // [h | h | h] . [e_hi | e_mid | e_lo]^T (no group table)
  int r_T, r_E, r_mtiles, r_ntiles, r_ks, r_nkd, r_per;
  int r_n;                    // MMA N of the router: round16(E) up to 256 (fewer experts: a narrower tile)
  float* zpart;               // [r_ks, r_T, r_E]
  // dynamic schedule: units are claimed from this zeroed counter (null: static
  // round-robin over the CTAs)
  int* tile_counter;
  // k-block length in elements: 64 bf16 or, with e4m3 operands (kernel
  // template Q8), 128 e4m3 -- 128 bytes either way; for e4m3, one power-of-two
  // scale per A row (xs) and per weight row (s0: gate or W_down, s1: up),
  // applied to the fp32 accumulators in the epilogue
  int bk;
  const float *xs_r, *xs_s;
  const float *s0_r, *s1_r, *s0_s, *s1_s;
  // training forward (EPI_SWIGLU): the pre-activations U | V of every row,
  // [rows, 2f] bf16 (U in columns 0..f-1, V in f..2f-1), for the backward
  uint16_t* uv_r;
  uint16_t* uv_s;
  // EPI_SCALE: 1 = outputs in fp16 (saturating, MOE_DEVERR_RANGE), else bf16
  int out_f16;
};

constexpr int UNIT_RING = 4;     // units handed from the producer to the MMA / epilogue warps

// One work unit: group g (routed / shared), row tile, column tile and the
// range of 64-wide k-blocks it reduces over; n16 > 0 marks a transposed tile
// (MMA N = n16); tail > 0 marks a full tile carrying the group's last tail
// rows (transposed, MMA N = t16) in the same unit.
struct Unit {
  int g, mt, nt, kb0, nk;
  int rows, n16, tail, t16;
  bool sh;
};

// Row units of a group of `rows` rows: one per 128-row tile, except that a
// last tile of at most kMergeMaxRows rows shares the unit of the tile before.
__device__ __forceinline__ int row_units(int rows, int merge_max) {
  const int mt = (rows + BM - 1) / BM;
  const int last = rows - (mt - 1) * BM;
  return mt - ((mt >= 2 && last <= merge_max) ? 1 : 0);
}

template <int EPI>
__device__ __forceinline__ int total_units(const Params& p) {
  if (EPI == EPI_ROUTER) return p.r_mtiles * p.r_ntiles * p.r_ks;
  return __ldg(p.prefix + p.G);
}

template <int EPI>
__device__ __forceinline__ Unit decode(const Params& p, int u) {
  Unit w;
  if (EPI == EPI_ROUTER) {
    // row tile fastest: CTAs running together read the same centroid tiles
    w.g = 0; w.sh = false;
    w.mt = u % p.r_mtiles;
    int rest = u / p.r_mtiles;
    const int ks = rest % p.r_ks;
    w.nt = rest / p.r_ks;
    w.kb0 = ks * p.r_per;
    w.nk = min(3 * p.r_nkd, w.kb0 + p.r_per) - w.kb0;
    w.nt = w.nt * p.r_ks + ks;          // packed (column tile, split) for the epilogue
    w.rows = p.r_T;
    w.n16 = w.tail = w.t16 = 0;
    return w;
  }
  int lo = 0, hi = p.G;                  // prefix[lo] <= u < prefix[lo + 1]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(p.prefix + mid) <= u) lo = mid; else hi = mid;
  }
  w.g = lo;
  w.sh = lo >= p.E_r;
  int local = u - __ldg(p.prefix + lo);
  w.rows = __ldg(p.grp_rows + lo);
  const int runits = row_units(w.rows, kMergeMaxRows);
  w.mt = local % runits;
  w.nt = local / runits;
  w.kb0 = 0;
  w.nk = ((w.sh ? p.k_s : p.k_r) + p.bk - 1) / p.bk;
  const int mtiles = (w.rows + BM - 1) / BM;
  w.tail = (runits < mtiles && w.mt == runits - 1) ? w.rows - (mtiles - 1) * BM : 0;
  w.t16 = (w.tail + 15) & ~15;
  const int rv = min(BM, w.rows - w.mt * BM);
  w.n16 = (w.tail == 0 && rv <= kSwapMaxRows) ? (rv + 15) & ~15 : 0;
  return w;
}

// Wait without giving up on *abort (used to drain copies and MMAs in flight
// before the CTA releases its shared and tensor memory).
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, int* err) {
  uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) { set_device_error(err, MOE_DEVERR_WAIT_TIMEOUT); return; }
  }
}

// One MMA of a k-step: 16 bf16 or 32 e4m3 elements of K (32 bytes of each row).
template <bool Q8>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if constexpr (Q8) tc_mma_e4m3(d, a, b, idesc, acc);
  else tc_mma_bf16(d, a, b, idesc, acc);
}

// Shared -> global tensor store of one box; completion is tracked per thread
// in bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tmap, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               :: "l"(tmap), "r"(smem_u32(smem_src)), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// all but the most recent bulk group of this thread have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every bulk group of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Write 16 bf16 pairs (32 columns) of this lane's row into the staging box:
// line `lane`, 16-byte chunks chunk0 .. chunk0 + 3, at chunk ^ (lane & 7) --
// the 128-byte swizzle of the store's tensor map (and bank-conflict free).
__device__ __forceinline__ void stage_row32(uint8_t* box, int lane, int chunk0, const uint32_t (&pk)[16]) {
  uint8_t* line = box + lane * 128;
#pragma unroll
  for (int v = 0; v < 4; ++v)
    *reinterpret_cast<uint4*>(line + (((chunk0 + v) ^ (lane & 7)) * 16)) =
        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
}

__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

__device__ __forceinline__ uint16_t bf16_bits(float a) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(a));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Down-GEMM outputs: bf16, or saturating fp16 for a layer's own slot rows
// (hit records a saturation, reported as MOE_DEVERR_RANGE).
__device__ __forceinline__ uint32_t pack_out(int f16, float a, float b, bool& hit) {
  return f16 ? pack_f16_sat(a, b, hit) : pack_bf16(a, b);
}
__device__ __forceinline__ uint16_t bits_out(int f16, float a, bool& hit) {
  return f16 ? f16_bits_sat(a, hit) : bf16_bits(a);
}

// Tensor-map coordinates of the A and B tiles of k-block i of unit w.
template <int EPI>
struct TileCoords {
  const CUtensorMap *am, *am32, *b0, *b1;
  int ax, ay, bx, by;
};

template <int EPI>
__device__ __forceinline__ TileCoords<EPI> tile_coords(const Params& p, const Unit& w, int i) {
  TileCoords<EPI> c;
  c.am = w.sh ? &p.a_s : &p.a_r;
  c.am32 = w.sh ? &p.a32_s : &p.a32_r;
  c.b0 = w.sh ? &p.b0_s : &p.b0_r;
  c.b1 = w.sh ? &p.b1_s : &p.b1_r;
  int brow;
  if (EPI == EPI_ROUTER) {
    c.ay = w.mt * BM;
    brow = (w.nt / p.r_ks) * BN;
    const int part = (w.kb0 + i) / p.r_nkd;     // virtual k-block -> (centroid part, k)
    c.ax = c.bx = ((w.kb0 + i) - part * p.r_nkd) * BK;
    c.by = part * p.r_E + brow;
  } else {
    const int e = w.sh ? w.g - p.E_r : w.g;
    c.ay = ((EPI == EPI_SWIGLU && w.sh) ? 0 : __ldg(p.grp_row0 + w.g)) + w.mt * BM;
    brow = e * (w.sh ? p.wrows_s : p.wrows_r) + w.nt * (EPI == EPI_SWIGLU ? BN / 2 : BN);
    c.ax = c.bx = (w.kb0 + i) * p.bk;
    c.by = brow;
  }
  return c;
}

// Epilogue of a transposed tile: the accumulator holds D^T, lane r = output
// column colA (gate or first W_down half, columns [0, n16)) and colB (up or
// second half, columns [128, 128 + n16)); accumulator column t = row row0 + t.
// out0 points at output row row0.
template <int EPI>
__device__ __noinline__ void epilogue_transposed(const Params& p, bool sh, uint16_t* out0, size_t row0,
                                                    int rv, int n16, int colA, int ncols, uint32_t tb,
                                                    const float* xs, const float* wsA, const float* wsB,
                                                    uint16_t* uv0) {
  // e4m3 operands: xs = scales of the tile's rows (row t at xs[t]); wsA = scales
  // of the expert's weight rows (gate, or W_down), wsB = up's (EPI_SWIGLU);
  // xs null: bf16 operands, no scaling
  const int colB = colA + BN / 2;                     // EPI_SCALE only
  float cA = 1.0f, cB = 1.0f;
  if (xs && colA < ncols) {
    cA = __ldg(wsA + colA);
    if (EPI == EPI_SWIGLU) cB = __ldg(wsB + colA);
  }
  if (EPI == EPI_SCALE && xs && colB < ncols) cB = __ldg(wsA + colB);
  bool hit = false;
#pragma unroll 1
  for (int c = 0; c < n16; c += 32) {
    float dv0[32], dv1[32];
    tmem_ld32(tb + c, dv0);
    tmem_ld32(tb + BN / 2 + c, dv1);
#pragma unroll
    for (int v = 0; v < 32; ++v) {
      const int t = c + v;
      if (t < rv) {
        uint16_t* orow_p = out0 + (size_t)t * ncols;
        const float rs = xs ? __ldg(xs + t) : 1.0f;
        if (EPI == EPI_SWIGLU) {
          if (colA < ncols) {
            const float g = dv0[v] * (rs * cA), u = dv1[v] * (rs * cB);
            orow_p[colA] = bf16_bits(silu(g) * u);
            if (uv0) {
              uv0[(size_t)t * 2 * ncols + colA] = bf16_bits(g);
              uv0[(size_t)t * 2 * ncols + ncols + colA] = bf16_bits(u);
            }
          }
        } else {
          const float sc = (!sh && p.row_scale) ? __ldg(p.row_scale + row0 + t) : 1.0f;
          if (colA < ncols) orow_p[colA] = bits_out(p.out_f16, dv0[v] * (rs * cA) * sc, hit);
          if (colB < ncols) orow_p[colB] = bits_out(p.out_f16, dv1[v] * (rs * cB) * sc, hit);
        }
      }
    }
  }
  if (hit) set_device_error(p.err, MOE_DEVERR_RANGE);
}

// The same for a down GEMM (EPI_SCALE) whose warps own staging boxes: 32 rows
// at a time, the warp writes its 32 columns x 32 rows of each half (lane =
// column) into a padded shared tile and reads them back by rows (lane = row),
// so every output row leaves as 16-byte vectors instead of one 2-byte store
// per value, and each row's gate is loaded once (lane = row) and broadcast.
// tile: two 32 x kTrLine halves (80-byte lines: no bank conflicts either way).
constexpr int kTrLine = 40;
static_assert(2 * 32 * kTrLine * 2 <= 2 * OUT_BOX_BYTES, "the tile fits a warp's two staging boxes");
__device__ __noinline__ void epilogue_transposed_staged(const Params& p, bool sh, uint16_t* out0, size_t row0,
                                                        int rv, int n16, int colA, int ncols, uint32_t tb,
                                                        const float* xs, const float* wsA, uint16_t* tile,
                                                        int lane) {
  const int colB = colA + BN / 2;
  float cA = 1.0f, cB = 1.0f;
  if (xs && colA < ncols) cA = __ldg(wsA + colA);
  if (xs && colB < ncols) cB = __ldg(wsA + colB);
  const int colA0 = colA - lane, colB0 = colB - lane;     // the warp's first column of each half
  uint16_t* tA = tile;
  uint16_t* tB = tile + 32 * kTrLine;
  bool hit = false;
#pragma unroll 1
  for (int c = 0; c < n16; c += 32) {
    float dv0[32], dv1[32];
    tmem_ld32(tb + c, dv0);
    tmem_ld32(tb + BN / 2 + c, dv1);
    const int tl = c + lane;                               // the row this lane loads for and stores
    float rs_l = 1.0f, sc_l = 1.0f;
    if (tl < rv) {
      if (xs) rs_l = __ldg(xs + tl);
      if (!sh && p.row_scale) sc_l = __ldg(p.row_scale + row0 + tl);
    }
    bool hA = false, hB = false;
#pragma unroll
    for (int v = 0; v < 32; ++v) {
      const float rs = xs ? __shfl_sync(0xffffffffu, rs_l, v) : 1.0f;
      const float sc = __shfl_sync(0xffffffffu, sc_l, v);
      uint16_t a = 0, b = 0;
      if (c + v < rv) {
        a = bits_out(p.out_f16, dv0[v] * (rs * cA) * sc, hA);
        b = bits_out(p.out_f16, dv1[v] * (rs * cB) * sc, hB);
      }
      tA[v * kTrLine + lane] = a;
      tB[v * kTrLine + lane] = b;
    }
    hit |= (hA && colA < ncols) || (hB && colB < ncols);
    __syncwarp();
    if (tl < rv) {
      uint16_t* orow = out0 + (size_t)tl * ncols;
      const uint16_t* sa = tA + lane * kTrLine;
      const uint16_t* sb = tB + lane * kTrLine;
      if (colA0 + 32 <= ncols) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(orow + colA0 + 8 * q) = *reinterpret_cast<const uint4*>(sa + 8 * q);
      } else {
        for (int j = 0; j < 32 && colA0 + j < ncols; ++j) orow[colA0 + j] = sa[j];
      }
      if (colB0 + 32 <= ncols) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(orow + colB0 + 8 * q) = *reinterpret_cast<const uint4*>(sb + 8 * q);
      } else {
        for (int j = 0; j < 32 && colB0 + j < ncols; ++j) orow[colB0 + j] = sb[j];
      }
    }
    __syncwarp();                                          // the tile is rewritten by the next 32 rows
  }
  if (hit) set_device_error(p.err, MOE_DEVERR_RANGE);
}

// Q8: e4m3 operands (kind::f8f6f4, epilogue scales); a template parameter so
// that the MMA issue loop carries no branch between the two MMA forms (a
// runtime choice there cost the bf16 kernel 15 % of its throughput).
template <int EPI, bool Q8, bool TMA_OUT = false>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_gemm_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int STAGES = stages_of<TMA_OUT>();
  constexpr bool kTmaStoreOut = TMA_OUT && EPI != EPI_ROUTER;
  constexpr int OUT_BYTES = out_bytes_of<TMA_OUT>();
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sT = smem + STAGES * STAGE_BYTES;     // merged tails' rows
  uint8_t* sOut = smem + STAGES * (STAGE_BYTES + T_BYTES);   // epilogue staging boxes (1024-aligned)
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + OUT_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* unit_full = drain + 1;
  uint64_t* unit_empty = unit_full + UNIT_RING;
  volatile int* unit_ring = reinterpret_cast<volatile int*>(unit_empty + UNIT_RING);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(unit_ring) + UNIT_RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], 4 * kWarp); }
    for (int s = 0; s < UNIT_RING; ++s) { mbar_init(&unit_full[s], 1); mbar_init(&unit_empty[s], 1 + 4 * kWarp); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&p.a_r); prefetch_tmap(&p.a_s); prefetch_tmap(&p.b0_r);
    prefetch_tmap(&p.b1_r); prefetch_tmap(&p.b0_s); prefetch_tmap(&p.b1_s);
    if (EPI != EPI_ROUTER) { prefetch_tmap(&p.a32_r); prefetch_tmap(&p.a32_s); }
    if (EPI != EPI_ROUTER && kTmaStoreOut) { prefetch_tmap(&p.o_r); prefetch_tmap(&p.o_s); }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the prologue above touches no global memory; everything below may read
  // what the previous kernels wrote
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_units<EPI>(p);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      int slot = 0;
      uint32_t uphase = 0;
      for (int k = 0;; ++k) {
        // claim the next unit and hand it to the MMA and epilogue warps (-1 = done)
        int u = p.tile_counter ? atomicAdd(p.tile_counter, 1) : (int)blockIdx.x + k * (int)gridDim.x;
        if (u >= total) u = -1;
        if (!mbar_wait(&unit_empty[slot], uphase ^ 1u, abort_flag, p.err)) goto producer_done;
        unit_ring[slot] = u;
        mbar_arrive(&unit_full[slot]);
        if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const Unit w = decode<EPI>(p, u);
        // a transposed tile (and a merged tail) loads only the 32-row slices
        // that hold its N rows
        const int n_sub = w.n16 ? (w.n16 + A_SUB_ROWS - 1) / A_SUB_ROWS : 0;
        const int t_sub = (w.t16 + A_SUB_ROWS - 1) / A_SUB_ROWS;
        const uint32_t b_bytes = EPI == EPI_ROUTER ? (uint32_t)p.r_n * BK * 2 : (uint32_t)B_BYTES;
        const uint32_t tx = (uint32_t)((n_sub ? n_sub * A_SUB_BYTES : A_BYTES) + t_sub * A_SUB_BYTES) + b_bytes;
        for (int i = 0; i < w.nk; ++i) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err)) goto producer_done;
          const TileCoords<EPI> c = tile_coords<EPI>(p, w, i);
          mbar_arrive_expect_tx(&full[stage], tx);
          // the weight tile first: it comes from HBM, the row tiles mostly from L2
          if (EPI == EPI_SWIGLU) {
            tma_load_2d(sB + stage * B_BYTES, c.b0, &full[stage], c.bx, c.by);
            tma_load_2d(sB + stage * B_BYTES + B_BYTES / 2, c.b1, &full[stage], c.bx, c.by);
          } else {
            tma_load_2d(sB + stage * B_BYTES, c.b0, &full[stage], c.bx, c.by);
          }
          if (n_sub == 0) {
            tma_load_2d(sA + stage * A_BYTES, c.am, &full[stage], c.ax, c.ay);
          } else {
            for (int q = 0; q < n_sub; ++q)
              tma_load_2d(sA + stage * A_BYTES + q * A_SUB_BYTES, c.am32, &full[stage], c.ax,
                          c.ay + q * A_SUB_ROWS);
          }
          for (int q = 0; q < t_sub; ++q)
            tma_load_2d(sT + stage * T_BYTES + q * A_SUB_BYTES, c.am32, &full[stage], c.ax,
                        c.ay + BM + q * A_SUB_ROWS);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    producer_done:
      // the last (up to STAGES) loads must have landed before shared memory is released
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (--stage < 0) { stage = STAGES - 1; phase ^= 1u; }
        wait_drain(&full[stage], phase, p.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int nb = 0;                           // accumulator buffer of the next one-buffer unit
      uint32_t ph_e = 0;                    // bit b: phase of acc_empty[b]
      int slot = 0;
      uint32_t uphase = 0;
      for (;;) {
        if (!mbar_wait(&unit_full[slot], uphase, abort_flag, p.err)) break;
        const int u = unit_ring[slot];
        mbar_arrive(&unit_empty[slot]);
        if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const Unit w = decode<EPI>(p, u);
        const int nk = w.nk;
        // transposed tile: two M = 128 halves of the weight tile (gate | up, or
        // the two 128-row halves of W_down's 256) against the N = n16 rows,
        // into accumulator columns [0, n16) and [128, 128 + n16)
        constexpr bool q8 = EPI != EPI_ROUTER && Q8;
        const uint32_t idesc_n = q8 ? IDESC_Q8 : EPI == EPI_ROUTER ? idesc_bf16_f32(BM, p.r_n) : IDESC;
        const uint32_t idesc_t = q8 ? idesc_e4m3_f32(BM, w.n16 ? w.n16 : 16) : idesc_bf16_f32(BM, w.n16 ? w.n16 : 16);
        const uint32_t idesc_tail = q8 ? idesc_e4m3_f32(BM, w.t16 ? w.t16 : 16) : idesc_bf16_f32(BM, w.t16 ? w.t16 : 16);
        // a unit with a merged tail holds buffer 0 (full tile) and buffer 1 (tail)
        const bool two = w.tail > 0;
        const int acc = two ? 0 : nb;
        if (!mbar_wait(&acc_empty[acc], ((ph_e >> acc) & 1u) ^ 1u, abort_flag, p.err)) break;
        ph_e ^= 1u << acc;
        if (two) {
          if (!mbar_wait(&acc_empty[1], ((ph_e >> 1) & 1u) ^ 1u, abort_flag, p.err)) break;
          ph_e ^= 2u;
        }
        nb = two ? 1 : nb ^ 1;              // after a merged unit, the tail's buffer frees first
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        const uint32_t d_tail = tmem_base + (uint32_t)BN;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {      // kb counts this unit's k-blocks
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
          if (w.n16 == 0) {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              tc_mma<q8>(d_tmem, sdesc_kmajor_sw128(a0 + k * UMMA_K * 2),
                     sdesc_kmajor_sw128(b0 + k * UMMA_K * 2), idesc_n, (kb | k) != 0);
            }
          } else {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              const uint64_t xd = sdesc_kmajor_sw128(a0 + k * UMMA_K * 2);
              tc_mma<q8>(d_tmem, sdesc_kmajor_sw128(b0 + k * UMMA_K * 2), xd, idesc_t, (kb | k) != 0);
              tc_mma<q8>(d_tmem + BN / 2, sdesc_kmajor_sw128(b0 + B_BYTES / 2 + k * UMMA_K * 2), xd,
                     idesc_t, (kb | k) != 0);
            }
          }
          if (two) {
            const uint32_t t0 = smem_u32(sT + stage * T_BYTES);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              const uint64_t xd = sdesc_kmajor_sw128(t0 + k * UMMA_K * 2);
              tc_mma<q8>(d_tail, sdesc_kmajor_sw128(b0 + k * UMMA_K * 2), xd, idesc_tail, (kb | k) != 0);
              tc_mma<q8>(d_tail + BN / 2, sdesc_kmajor_sw128(b0 + B_BYTES / 2 + k * UMMA_K * 2), xd,
                     idesc_tail, (kb | k) != 0);
            }
          }
          tc_commit(&empty[stage]);       // frees the stage once these MMAs are done
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);        // accumulator ready for the epilogue
        if (two) tc_commit(&acc_full[1]);
      }
      tc_commit(drain);                    // every MMA issued by this thread is done
      wait_drain(drain, 0, p.err);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int sub = warp & 3;              // TMEM lane quarter this warp may access
    const int r = sub * 32 + lane;         // row within the tile
    bool hit = false;                      // an fp16 output saturated
    int nb = 0;                            // same buffer sequence as the MMA issuer
    uint32_t ph_f = 0;                     // bit b: phase of acc_full[b]
    int slot = 0;
    uint32_t uphase = 0;
    uint8_t* my_boxes = sOut + sub * 2 * OUT_BOX_BYTES;   // this warp's two staging boxes
    int n_boxes = 0;                       // boxes this warp has staged (alternating buffers)
    for (;;) {
      if (!mbar_wait(&unit_full[slot], uphase, abort_flag, p.err)) break;
      const int u = unit_ring[slot];
      mbar_arrive(&unit_empty[slot]);
      if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
      if (u < 0) break;
      const Unit w = decode<EPI>(p, u);
      const int mt = w.mt, nt = w.nt;
      const bool sh = w.sh;
      const int rows = EPI == EPI_ROUTER ? p.r_T : __ldg(p.grp_rows + w.g);
      const int m = mt * BM + r;
      const bool valid = m < rows;
      const size_t orow = (EPI == EPI_ROUTER ? 0 : (size_t)__ldg(p.grp_row0 + w.g)) + m;
      const int ncols = sh ? p.ncols_s : p.ncols_r;
      uint16_t* out = (sh ? p.out_s : p.out_r) + orow * ncols;
      const bool two = w.tail > 0;
      const int acc = two ? 0 : nb;
      nb = two ? 1 : nb ^ 1;
      const uint32_t tb = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BN);
      // transposed tiles: this thread owns output column(s) r of the unit and
      // walks the rows along the accumulator columns
      const int colA = EPI == EPI_SWIGLU ? nt * (BN / 2) + r : nt * BN + r;
      const size_t row0 = orow - r;                       // output row of the tile's row 0
      uint16_t* out0 = (sh ? p.out_s : p.out_r) + row0 * ncols;
      // e4m3 operands: scales of the tile's A rows (xs[0] = tile row 0) and of
      // the expert's weight rows (wsA: gate or W_down, wsB: up)
      const float* xs = nullptr;
      const float* wsA = nullptr;
      const float* wsB = nullptr;
      if (EPI != EPI_ROUTER && Q8) {
        const int e = sh ? w.g - p.E_r : w.g;
        const size_t wr = (size_t)e * (sh ? p.wrows_s : p.wrows_r);
        wsA = (sh ? p.s0_s : p.s0_r) + wr;
        wsB = (sh ? p.s1_s : p.s1_r) + wr;
        xs = (sh ? p.xs_s : p.xs_r) + ((EPI == EPI_SWIGLU && sh) ? (size_t)mt * BM : row0);
      }
      // training forward: U | V rows of this tile (row 0 of the tile)
      uint16_t* uv0 = (EPI == EPI_SWIGLU && (sh ? p.uv_s : p.uv_r))
                          ? (sh ? p.uv_s : p.uv_r) + row0 * (size_t)(2 * ncols) : nullptr;
      if (EPI != EPI_ROUTER && two) {
        // the merged tail (rows (mt + 1) * 128 .. + tail, transposed, buffer 1)
        // first: its buffer is the one the next unit takes
        if (!mbar_wait(&acc_full[1], (ph_f >> 1) & 1u, abort_flag, p.err)) break;
        ph_f ^= 2u;
        tc_fence_after();
        if (EPI == EPI_SCALE && kTmaStoreOut) {
          if (lane == 0) bulk_wait_read_0();      // no store still reads this warp's boxes
          __syncwarp();
          epilogue_transposed_staged(p, sh, out0 + (size_t)BM * ncols, row0 + BM, w.tail, w.t16, colA, ncols,
                                     tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)BN,
                                     xs ? xs + BM : nullptr, wsA, reinterpret_cast<uint16_t*>(my_boxes), lane);
        } else {
          epilogue_transposed<EPI>(p, sh, out0 + (size_t)BM * ncols, row0 + BM, w.tail, w.t16, colA, ncols,
                                   tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)BN,
                                   xs ? xs + BM : nullptr, wsA, wsB, uv0 ? uv0 + (size_t)BM * 2 * ncols : nullptr);
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[1]);
      }
      if (!mbar_wait(&acc_full[acc], (ph_f >> acc) & 1u, abort_flag, p.err)) break;
      ph_f ^= 1u << acc;
      tc_fence_after();
      if (EPI == EPI_SCALE && kTmaStoreOut && w.n16) {
        if (lane == 0) bulk_wait_read_0();        // no store still reads this warp's boxes
        __syncwarp();
        epilogue_transposed_staged(p, sh, out0, row0, min(BM, rows - mt * BM), w.n16, colA, ncols, tb,
                                   xs, wsA, reinterpret_cast<uint16_t*>(my_boxes), lane);
      } else if (EPI != EPI_ROUTER && w.n16) {
        epilogue_transposed<EPI>(p, sh, out0, row0, min(BM, rows - mt * BM), w.n16, colA, ncols, tb,
                                 xs, wsA, wsB, uv0);
      } else if (EPI == EPI_ROUTER) {
        // fp32 partial logits of split (nt % ks) for experts of column tile nt / ks
        const int ks = nt % p.r_ks, ct = nt / p.r_ks;
        float* zrow = p.zpart + ((size_t)ks * p.r_T + m) * p.r_E;
#pragma unroll 1
        for (int c = 0; c < p.r_n; c += 32) {
          float dv[32];
          tmem_ld32(tb + c, dv);
          const int col0 = ct * BN + c;
          if (valid) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              if (col0 + 4 * v < p.r_E)
                *reinterpret_cast<float4*>(zrow + col0 + 4 * v) =
                    make_float4(dv[4 * v], dv[4 * v + 1], dv[4 * v + 2], dv[4 * v + 3]);
          }
        }
      } else if (EPI == EPI_SWIGLU && kTmaStoreOut && mt * BM + sub * 32 + 32 <= rows) {
        // every row of this warp is valid: stage 64 columns at a time, one TMA
        // store per box; the row stride of U | V is 2f, so those stay direct
        const float rs = xs ? __ldg(xs + r) : 1.0f;
        const CUtensorMap* om = sh ? &p.o_s : &p.o_r;
        const int orow0 = (int)(orow - (size_t)lane);
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 64) {
          uint8_t* box = my_boxes + (n_boxes & 1) * OUT_BOX_BYTES;
          if (lane == 0) bulk_wait_read_1();      // the store that last read this box is done reading
          __syncwarp();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float gv[32], uv[32];
            tmem_ld32(tb + c + 32 * half, gv);
            tmem_ld32(tb + BN / 2 + c + 32 * half, uv);
            const int col0 = nt * (BN / 2) + c + 32 * half;
            if (xs) {
#pragma unroll
              for (int v = 0; v < 32; ++v) {
                const bool in = col0 + v < ncols;
                gv[v] *= rs * (in ? __ldg(wsA + col0 + v) : 0.0f);
                uv[v] *= rs * (in ? __ldg(wsB + col0 + v) : 0.0f);
              }
            }
            if (uv0) {
              uint16_t* uvr = uv0 + (size_t)r * 2 * ncols;
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                if (col0 + 8 * v < ncols) {
                  *reinterpret_cast<uint4*>(uvr + col0 + 8 * v) =
                      make_uint4(pack_bf16(gv[8 * v], gv[8 * v + 1]), pack_bf16(gv[8 * v + 2], gv[8 * v + 3]),
                                 pack_bf16(gv[8 * v + 4], gv[8 * v + 5]), pack_bf16(gv[8 * v + 6], gv[8 * v + 7]));
                  *reinterpret_cast<uint4*>(uvr + ncols + col0 + 8 * v) =
                      make_uint4(pack_bf16(uv[8 * v], uv[8 * v + 1]), pack_bf16(uv[8 * v + 2], uv[8 * v + 3]),
                                 pack_bf16(uv[8 * v + 4], uv[8 * v + 5]), pack_bf16(uv[8 * v + 6], uv[8 * v + 7]));
                }
              }
            }
            uint32_t pk[16];
#pragma unroll
            for (int v = 0; v < 16; ++v) pk[v] = pack_bf16(silu(gv[2 * v]) * uv[2 * v], silu(gv[2 * v + 1]) * uv[2 * v + 1]);
            stage_row32(box, lane, 4 * half, pk);
          }
          fence_proxy_async_smem();               // the box is read by the async proxy
          __syncwarp();
          if (lane == 0) {
            const int x = nt * (BN / 2) + c;
            if (x < ncols) tma_store_2d(om, box, x, orow0);   // columns past ncols are clipped
            bulk_commit();                        // one group per box, even an empty one
          }
          ++n_boxes;
        }
      } else if (EPI == EPI_SWIGLU) {
        const float rs = (xs && valid) ? __ldg(xs + r) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          float gv[32], uv[32];
          tmem_ld32(tb + c, gv);
          tmem_ld32(tb + BN / 2 + c, uv);
          const int col0 = nt * (BN / 2) + c;
          if (xs && valid) {
#pragma unroll
            for (int v = 0; v < 32; ++v) {
              const bool in = col0 + v < ncols;
              gv[v] *= rs * (in ? __ldg(wsA + col0 + v) : 0.0f);
              uv[v] *= rs * (in ? __ldg(wsB + col0 + v) : 0.0f);
            }
          }
          if (valid && uv0) {
            uint16_t* uvr = uv0 + (size_t)r * 2 * ncols;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (col0 + 8 * v < ncols) {
                *reinterpret_cast<uint4*>(uvr + col0 + 8 * v) =
                    make_uint4(pack_bf16(gv[8 * v], gv[8 * v + 1]), pack_bf16(gv[8 * v + 2], gv[8 * v + 3]),
                               pack_bf16(gv[8 * v + 4], gv[8 * v + 5]), pack_bf16(gv[8 * v + 6], gv[8 * v + 7]));
                *reinterpret_cast<uint4*>(uvr + ncols + col0 + 8 * v) =
                    make_uint4(pack_bf16(uv[8 * v], uv[8 * v + 1]), pack_bf16(uv[8 * v + 2], uv[8 * v + 3]),
                               pack_bf16(uv[8 * v + 4], uv[8 * v + 5]), pack_bf16(uv[8 * v + 6], uv[8 * v + 7]));
              }
            }
          }
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (col0 + 8 * v < ncols) {
                uint4 pk;
                pk.x = pack_bf16(silu(gv[8 * v + 0]) * uv[8 * v + 0], silu(gv[8 * v + 1]) * uv[8 * v + 1]);
                pk.y = pack_bf16(silu(gv[8 * v + 2]) * uv[8 * v + 2], silu(gv[8 * v + 3]) * uv[8 * v + 3]);
                pk.z = pack_bf16(silu(gv[8 * v + 4]) * uv[8 * v + 4], silu(gv[8 * v + 5]) * uv[8 * v + 5]);
                pk.w = pack_bf16(silu(gv[8 * v + 6]) * uv[8 * v + 6], silu(gv[8 * v + 7]) * uv[8 * v + 7]);
                *reinterpret_cast<uint4*>(out + col0 + 8 * v) = pk;
              }
            }
          }
        }
      } else if (kTmaStoreOut && mt * BM + sub * 32 + 32 <= rows) {
        // every row of this warp is valid: stage 64 columns at a time, one TMA
        // store per box
        const float scale = (!sh && p.row_scale) ? __ldg(p.row_scale + orow) : 1.0f;
        const float rs = xs ? __ldg(xs + r) : 1.0f;
        const CUtensorMap* om = sh ? &p.o_s : &p.o_r;
        const int orow0 = (int)(orow - (size_t)lane);
#pragma unroll 1
        for (int c = 0; c < BN; c += 64) {
          uint8_t* box = my_boxes + (n_boxes & 1) * OUT_BOX_BYTES;
          if (lane == 0) bulk_wait_read_1();      // the store that last read this box is done reading
          __syncwarp();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float dv[32];
            tmem_ld32(tb + c + 32 * half, dv);
            const int col0 = nt * BN + c + 32 * half;
            if (xs) {
#pragma unroll
              for (int v = 0; v < 32; ++v) dv[v] *= rs * (col0 + v < ncols ? __ldg(wsA + col0 + v) : 0.0f);
            }
            uint32_t pk[16];
#pragma unroll
            for (int v = 0; v < 16; ++v) pk[v] = pack_out(p.out_f16, dv[2 * v] * scale, dv[2 * v + 1] * scale, hit);
            stage_row32(box, lane, 4 * half, pk);
          }
          fence_proxy_async_smem();               // the box is read by the async proxy
          __syncwarp();
          if (lane == 0) {
            const int x = nt * BN + c;
            if (x < ncols) tma_store_2d(om, box, x, orow0);   // columns past ncols are clipped
            bulk_commit();                        // one group per box, even an empty one
          }
          ++n_boxes;
        }
      } else {
        const float scale = (!sh && p.row_scale && valid) ? __ldg(p.row_scale + orow) : 1.0f;
        const float rs = (xs && valid) ? __ldg(xs + r) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float dv[32];
          tmem_ld32(tb + c, dv);
          const int col0 = nt * BN + c;
          if (xs && valid) {
#pragma unroll
            for (int v = 0; v < 32; ++v) dv[v] *= rs * (col0 + v < ncols ? __ldg(wsA + col0 + v) : 0.0f);
          }
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (col0 + 8 * v < ncols) {
                uint4 pk;
                pk.x = pack_out(p.out_f16, dv[8 * v + 0] * scale, dv[8 * v + 1] * scale, hit);
                pk.y = pack_out(p.out_f16, dv[8 * v + 2] * scale, dv[8 * v + 3] * scale, hit);
                pk.z = pack_out(p.out_f16, dv[8 * v + 4] * scale, dv[8 * v + 5] * scale, hit);
                pk.w = pack_out(p.out_f16, dv[8 * v + 6] * scale, dv[8 * v + 7] * scale, hit);
                *reinterpret_cast<uint4*>(out + col0 + 8 * v) = pk;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
    // the staging boxes must not be released while a store still reads them
    if (EPI != EPI_ROUTER && kTmaStoreOut && lane == 0) bulk_wait_all();
    if (hit) set_device_error(p.err, MOE_DEVERR_RANGE);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------
// CTA-pair grouped GEMM (tcgen05 cta_group::2) for experts with many rows.
//
// A cluster of two CTAs on neighbouring SMs computes 256-row x 256-column
// tiles: each CTA stages its own 128 rows of A and one half of the weight tile,
// and one thread of the even CTA issues M = 256 MMAs that read both CTAs'
// shared memory and accumulate each CTA's 128 rows in its own TMEM.  Per SM a
// k-block then costs 32 KB of operands for the same tensor work as a 48 KB
// stage of the single-CTA kernel, so six stages fit and each weight tile
// crosses L2 -> SM once per 256 rows instead of once per 128.
//
// Weight halves: for the down GEMM the even CTA holds rows 0..127 of W_down's
// 256-row tile and the odd CTA rows 128..255; for the gate/up GEMM each CTA
// holds 64 gate rows and the 64 up rows of the same output columns (the even
// CTA columns 0..63 of the 128-column tile, the odd CTA 64..127), so the
// accumulator columns are [gate 0..63 | up 0..63 | gate 64..127 | up 64..127].
//
// Merged tails: a group's last tile of at most kPairMergeMax rows rides in the
// unit of the full tile before it.  Each CTA stages half of the tail's rows,
// and one more MMA per k-step computes the tail transposed, D^T = W x^T with
// the two staged weight halves as the M = 256 operand and the tail rows as the
// N = round16(tail) operand, into the second accumulator: TMEM lane = weight
// row, column = tail row.  For the gate/up GEMM the gate rows land in lanes
// 0..63 and the up rows of the same columns in lanes 64..127 of the same CTA;
// the epilogue warps exchange them through shared memory.  Other short last
// tiles are padded to 256 rows, so the launch takes this kernel only when
// experts average many rows (kPairMinRows).  Units are claimed dynamically by
// the even CTA's producer (merged units cost more than plain ones, so a fixed
// round-robin leaves some pairs with more work) and handed to both CTAs through
// a unit ring mirrored in each CTA's shared memory.
//
// Barriers: full[s] lives in the even CTA and counts both CTAs' TMA bytes
// (the even CTA arms it with both halves; the odd CTA's loads complete on it
// through its cluster address); empty[s] and acc_full[a] exist in both CTAs
// and are signalled together by one multicast commit; acc_empty[a] lives in
// the even CTA and takes one arrival per epilogue warp of both CTAs.  Unit
// ring: the even CTA's producer writes each claimed unit into slot s of both
// CTAs (the odd CTA's by a remote store followed by a release arrive on its
// unit_full[s]); unit_empty[s] lives in the even CTA and takes one arrival
// from each reader: the MMA thread, the producer of the odd CTA and every
// epilogue warp of both CTAs.
// ---------------------------------------------------------------------------
constexpr int kPairMinRows = 512;               // routed rows per expert (mean) for the pair kernel
constexpr int kPairMergeMax = 64;               // tails of <= this many rows join the tile before
constexpr int P_M = 2 * BM;                     // 256 rows per pair tile
constexpr int P_B_BYTES = (BN / 2) * BK * 2;    // 16 KB: this CTA's half of the weight tile
constexpr int P_T_BYTES = A_SUB_BYTES;          // 4 KB: a 32-row box of this CTA's tail rows
constexpr int P_STAGE_BYTES = A_BYTES + P_B_BYTES + P_T_BYTES;
constexpr int P_XCHG_BYTES = 32 * 64 * 4;       // 8 KB: up values of 32 tail rows x 64 columns
// Down GEMMs with short units (at most kTmaOutMaxKb k-blocks) stage their
// outputs in shared memory for TMA stores, as the single-CTA down GEMM does:
// the 32 KB of boxes cost one of the six stages.
template <bool TMA_OUT> constexpr int p_stages() { return TMA_OUT ? 5 : 6; }
template <bool TMA_OUT> constexpr int p_extra_bytes() { return TMA_OUT ? 4 * 2 * OUT_BOX_BYTES : P_XCHG_BYTES; }
template <bool TMA_OUT> constexpr size_t p_smem() {
  return (size_t)p_stages<TMA_OUT>() * P_STAGE_BYTES + p_extra_bytes<TMA_OUT>() + 1024 + CTRL_BYTES;
}
constexpr size_t P_SMEM = p_smem<false>();
constexpr uint32_t P_IDESC = idesc_bf16_f32(P_M, BN);
static_assert(p_smem<false>() <= 232448 && p_smem<true>() <= 232448, "shared memory per CTA");
static_assert(kPairMergeMax <= 2 * A_SUB_ROWS, "a tail's half fits one 32-row box");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the same shared-memory location in cluster CTA `rank`
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ void st_remote_u32(uint32_t addr_cluster, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr_cluster), "r"(v) : "memory");
}
// the four epilogue warps of this CTA (named barrier 1; __syncthreads uses 0)
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// TMA load into this CTA's shared memory, its bytes counted on the barrier at
// cluster address bar_cluster (the even CTA's); no multicast
__device__ __forceinline__ void tma_load_2d_pair(void* sdst, const void* tmap, uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(sdst)), "l"(tmap), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// arrive on `bar` in both CTAs of the pair once this thread's MMAs are done
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      ::"r"(smem_u32(bar)), "h"((uint16_t)3) : "memory");
}
// arrive on `bar` in this CTA only
__device__ __forceinline__ void tc_commit_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(smem_slot)), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// One unit of the pair kernel: group g, 256-row tile mt, column tile nt; tail
// > 0 marks a full tile carrying the group's last `tail` rows (t16 rounded up
// to 16) as its merged tail.
struct PairUnit {
  int g, mt, nt, nk, rows, tail, t16;
  bool sh;
};

__device__ __forceinline__ PairUnit pair_decode(const Params& p, int u) {
  PairUnit w;
  int lo = 0, hi = p.G;                  // prefix[lo] <= u < prefix[lo + 1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p.prefix + mid) <= u) lo = mid; else hi = mid;
  }
  w.g = lo;
  w.sh = lo >= p.E_r;
  const int local = u - __ldg(p.prefix + lo);
  w.rows = __ldg(p.grp_rows + lo);
  const int mtiles = (w.rows + P_M - 1) / P_M;
  const int last = w.rows - (mtiles - 1) * P_M;
  const int runits = mtiles - ((mtiles >= 2 && last <= kPairMergeMax) ? 1 : 0);
  w.mt = local % runits;
  w.nt = local / runits;
  w.tail = (runits < mtiles && w.mt == runits - 1) ? last : 0;
  w.t16 = (w.tail + 15) & ~15;
  w.nk = ((w.sh ? p.k_s : p.k_r) + p.bk - 1) / p.bk;
  return w;
}

// A bounded wait that also tells the other CTA of the pair to give up.
__device__ __forceinline__ bool pair_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* err,
                                          uint32_t peer_abort) {
  if (mbar_wait(bar, parity, abort, err)) return true;
  st_remote_u32(peer_abort, 1u);
  return false;
}

// The same with acquire semantics at cluster scope: for the unit ring, whose
// slots the other CTA writes (remote store, then a release arrive).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool pair_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, int* err,
                                                  uint32_t peer_abort) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 63u) == 63u) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        set_device_error(err, MOE_DEVERR_WAIT_TIMEOUT);
        *abort = 1;
        st_remote_u32(peer_abort, 1u);
        return false;
      }
    }
  }
}

template <int EPI, bool TMA_OUT = false>
__global__ void __launch_bounds__(NUM_THREADS, 1) pair_gemm_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int P_STAGES = p_stages<TMA_OUT>();
  constexpr bool kTmaStoreOut = TMA_OUT && EPI == EPI_SCALE;
  uint8_t* sA = smem;
  uint8_t* sB = smem + P_STAGES * A_BYTES;
  uint8_t* sT = sB + P_STAGES * P_B_BYTES;
  float* xchg = reinterpret_cast<float*>(smem + P_STAGES * P_STAGE_BYTES);       // gate/up tails
  uint8_t* sOut = smem + P_STAGES * P_STAGE_BYTES;                               // staging boxes (TMA_OUT)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES + p_extra_bytes<TMA_OUT>());
  uint64_t* empty = full + P_STAGES;
  uint64_t* acc_full = empty + P_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* unit_full = drain + 1;
  uint64_t* unit_empty = unit_full + UNIT_RING;
  volatile int* unit_ring = reinterpret_cast<volatile int*>(unit_empty + UNIT_RING);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(unit_ring) + UNIT_RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr int kUnitReaders = 1 + 1 + 2 * 4;   // MMA thread, odd producer, epilogue warps

  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const uint32_t rank = cluster_rank();
  const uint32_t peer_abort = cluster_addr(const_cast<int*>(abort_flag), rank ^ 1u);
  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], 2 * 4); }
    for (int s = 0; s < UNIT_RING; ++s) { mbar_init(&unit_full[s], 1); mbar_init(&unit_empty[s], kUnitReaders); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&p.a_r); prefetch_tmap(&p.a_s); prefetch_tmap(&p.a32_r); prefetch_tmap(&p.a32_s);
    prefetch_tmap(&p.b0_r); prefetch_tmap(&p.b1_r); prefetch_tmap(&p.b0_s); prefetch_tmap(&p.b1_s);
    if (kTmaStoreOut) { prefetch_tmap(&p.o_r); prefetch_tmap(&p.o_s); }
  }
  __syncthreads();
  cluster_sync_all();          // both CTAs' barriers are initialised before either signals the other
  if (warp == 0) tmem_alloc_pair(tmem_slot, TMEM_COLS);   // the same warp in both CTAs
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem_base = *tmem_slot;
  const int total = __ldg(p.prefix + p.G);
  const int pair = (int)blockIdx.x >> 1, n_pairs = (int)gridDim.x >> 1;
  const uint32_t leader_unit_empty = cluster_addr(unit_empty, 0);   // slot s: + 8 s

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int slot = 0;
      uint32_t uphase = 0;
      int n_claims = 0;
      for (;;) {
        int u;
        if (rank == 0) {
          // claim the next unit and hand it to both CTAs (-1 = done)
          u = p.tile_counter ? atomicAdd(p.tile_counter, 1) : pair + n_claims * n_pairs;
          ++n_claims;
          if (u >= total) u = -1;
          if (!pair_wait_cluster(&unit_empty[slot], uphase ^ 1u, abort_flag, p.err, peer_abort)) goto producer_done;
          unit_ring[slot] = u;
          st_remote_u32(cluster_addr(const_cast<int*>(unit_ring + slot), 1), (uint32_t)u);
          mbar_arrive(&unit_full[slot]);
          mbar_arrive_remote(cluster_addr(&unit_full[slot], 1));
        } else {
          if (!pair_wait_cluster(&unit_full[slot], uphase, abort_flag, p.err, peer_abort)) goto producer_done;
          u = unit_ring[slot];
          mbar_arrive_remote(leader_unit_empty + 8u * slot);
        }
        if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const PairUnit w = pair_decode(p, u);
        const int e = w.sh ? w.g - p.E_r : w.g;
        const CUtensorMap* am = w.sh ? &p.a_s : &p.a_r;
        const CUtensorMap* am32 = w.sh ? &p.a32_s : &p.a32_r;
        const int row_base = (EPI == EPI_SWIGLU && w.sh) ? 0 : __ldg(p.grp_row0 + w.g);
        const int ay = row_base + w.mt * P_M + (int)rank * BM;
        // this CTA's half of the merged tail: rows rank * t16/2 .. of the tail
        const int ty = row_base + (w.mt + 1) * P_M + (int)rank * (w.t16 / 2);
        const int wrows = w.sh ? p.wrows_s : p.wrows_r;
        const CUtensorMap* b0 = w.sh ? &p.b0_s : &p.b0_r;
        const CUtensorMap* b1 = w.sh ? &p.b1_s : &p.b1_r;
        const int by = EPI == EPI_SWIGLU ? e * wrows + w.nt * (BN / 2) + (int)rank * (BN / 4)
                                         : e * wrows + w.nt * BN + (int)rank * (BN / 2);
        const uint32_t tx = 2u * (A_BYTES + P_B_BYTES + (w.tail ? P_T_BYTES : 0));
        for (int i = 0; i < w.nk; ++i) {
          if (!pair_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, peer_abort)) goto producer_done;
          const uint32_t bar = cluster_addr(&full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], tx);
          const int x = i * p.bk;
          if (EPI == EPI_SWIGLU) {
            // 64 gate rows, then the 64 up rows of the same columns
            tma_load_2d_pair(sB + stage * P_B_BYTES, b0, bar, x, by);
            tma_load_2d_pair(sB + stage * P_B_BYTES + P_B_BYTES / 2, b1, bar, x, by);
          } else {
            tma_load_2d_pair(sB + stage * P_B_BYTES, b0, bar, x, by);
          }
          tma_load_2d_pair(sA + stage * A_BYTES, am, bar, x, ay);
          if (w.tail) tma_load_2d_pair(sT + stage * P_T_BYTES, am32, bar, x, ty);
          if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // every stage's last release (the MMA commits reach both CTAs) has
      // arrived before this CTA may leave
      for (int i = 0; i < P_STAGES; ++i) {
        if (!pair_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, peer_abort)) break;
        if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (even CTA) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int nb = 0;                           // accumulator of the next one-buffer unit
      uint32_t ph_e = 0;                    // bit a: phase of acc_empty[a]
      bool ok = true;
      int slot = 0;
      uint32_t uphase = 0;
      for (;;) {
        if (!pair_wait(&unit_full[slot], uphase, abort_flag, p.err, peer_abort)) { ok = false; break; }
        const int u = unit_ring[slot];
        mbar_arrive(&unit_empty[slot]);
        if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const PairUnit w = pair_decode(p, u);
        // a unit with a merged tail holds accumulator 0 (full tile) and 1 (tail)
        const bool two = w.tail > 0;
        const int acc = two ? 0 : nb;
        if (!pair_wait(&acc_empty[acc], ((ph_e >> acc) & 1u) ^ 1u, abort_flag, p.err, peer_abort)) break;
        ph_e ^= 1u << acc;
        if (two) {
          if (!pair_wait(&acc_empty[1], ((ph_e >> 1) & 1u) ^ 1u, abort_flag, p.err, peer_abort)) break;
          ph_e ^= 2u;
        }
        nb = two ? 1 : nb ^ 1;              // after a merged unit, the tail's buffer frees first
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        const uint32_t d_tail = tmem_base + (uint32_t)BN;
        const uint32_t idesc_tail = idesc_bf16_f32(P_M, w.t16 ? w.t16 : 16);
        for (int kb = 0; kb < w.nk; ++kb) {
          if (!pair_wait(&full[stage], phase, abort_flag, p.err, peer_abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * P_B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k)
            tc_mma_pair(d_tmem, sdesc_kmajor_sw128(a0 + k * UMMA_K * 2), sdesc_kmajor_sw128(b0 + k * UMMA_K * 2),
                        P_IDESC, (kb | k) != 0);
          if (two) {
            const uint32_t t0 = smem_u32(sT + stage * P_T_BYTES);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              tc_mma_pair(d_tail, sdesc_kmajor_sw128(b0 + k * UMMA_K * 2), sdesc_kmajor_sw128(t0 + k * UMMA_K * 2),
                          idesc_tail, (kb | k) != 0);
          }
          tc_commit_pair(&empty[stage]);    // frees the stage in both CTAs once these MMAs are done
          if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[acc]);     // both CTAs' halves of the accumulator are ready
        if (two) tc_commit_pair(&acc_full[1]);
      }
      // the epilogues of both CTAs have released both accumulators
      for (int a = 0; a < 2 && ok; ++a)
        if (!pair_wait(&acc_empty[a], ((ph_e >> a) & 1u) ^ 1u, abort_flag, p.err, peer_abort)) break;
      tc_commit_local(drain);               // every MMA issued by this thread is done
      wait_drain(drain, 0, p.err);
    }
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
    const int sub = warp & 3;              // TMEM lane quarter this warp may access
    const int L = sub * 32 + lane;         // this thread's TMEM lane
    bool hit = false;                      // an fp16 output saturated
    uint8_t* my_boxes = sOut + sub * 2 * OUT_BOX_BYTES;   // this warp's two staging boxes (TMA_OUT)
    int n_boxes = 0;
    int nb = 0;
    uint32_t ph_f = 0;
    int slot = 0;
    uint32_t uphase = 0;
    for (;;) {
      if (!pair_wait_cluster(&unit_full[slot], uphase, abort_flag, p.err, peer_abort)) break;
      const int u = unit_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader_unit_empty + 8u * slot);
      if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
      if (u < 0) break;
      const PairUnit w = pair_decode(p, u);
      const bool two = w.tail > 0;
      const int acc = two ? 0 : nb;
      nb = two ? 1 : nb ^ 1;
      const int ncols = w.sh ? p.ncols_s : p.ncols_r;
      uint16_t* outb = w.sh ? p.out_s : p.out_r;
      const size_t grow0 = (size_t)__ldg(p.grp_row0 + w.g);      // output row of group row 0
      if (two) {
        // the merged tail (group rows (mt + 1) * 256 ..), transposed, accumulator 1
        // first: its buffer is the one the next unit takes
        if (!pair_wait(&acc_full[1], (ph_f >> 1) & 1u, abort_flag, p.err, peer_abort)) break;
        ph_f ^= 2u;
        tc_fence_after();
        const size_t trow0 = grow0 + (size_t)(w.mt + 1) * P_M;
        const uint32_t tt = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)BN;
        for (int c = 0; c < w.t16; c += 32) {
          float dv[32];
          if (EPI == EPI_SWIGLU) {
            // lanes 64..127 hold up; hand them to the gate lanes 0..63 of the same column
            if (sub >= 2) {
              tmem_ld32(tt + c, dv);
#pragma unroll
              for (int v = 0; v < 32; ++v) xchg[v * 64 + (L - 64)] = dv[v];
            }
            epilogue_bar();
            if (sub < 2) {
              tmem_ld32(tt + c, dv);
              const int col = w.nt * (BN / 2) + (int)rank * (BN / 4) + L;
              if (col < ncols) {
#pragma unroll
                for (int v = 0; v < 32; ++v)
                  if (c + v < w.tail)
                    outb[(trow0 + c + v) * ncols + col] = bf16_bits(silu(dv[v]) * xchg[v * 64 + L]);
              }
            }
            epilogue_bar();
          } else {
            tmem_ld32(tt + c, dv);
            const int col = w.nt * BN + (int)rank * (BN / 2) + L;
            if (col < ncols) {
#pragma unroll
              for (int v = 0; v < 32; ++v) {
                if (c + v < w.tail) {
                  const float sc = (!w.sh && p.row_scale) ? __ldg(p.row_scale + trow0 + c + v) : 1.0f;
                  outb[(trow0 + c + v) * ncols + col] = bits_out(p.out_f16, dv[v] * sc, hit);
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(cluster_addr(&acc_empty[1], 0));
      }
      if (!pair_wait(&acc_full[acc], (ph_f >> acc) & 1u, abort_flag, p.err, peer_abort)) break;
      ph_f ^= 1u << acc;
      tc_fence_after();
      const int m0 = w.mt * P_M + (int)rank * BM + sub * 32;   // group row of this warp's lane 0
      const int m = m0 + lane;
      const bool valid = m < w.rows;
      const size_t orow = grow0 + m;
      uint16_t* out = outb + orow * ncols;
      const uint32_t tb = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BN);
      if (m0 < w.rows) {                   // at least one valid row in this warp
        if (EPI == EPI_SWIGLU) {
#pragma unroll 1
          for (int c = 0; c < BN / 2; c += 32) {
            // output columns c .. c + 31 of the tile: gate in accumulator
            // column gc (c < 64: c; else c + 64), up 64 columns further
            const int gc = c < BN / 4 ? c : c + BN / 4;
            float gv[32], uv[32];
            tmem_ld32(tb + gc, gv);
            tmem_ld32(tb + gc + BN / 4, uv);
            const int col0 = w.nt * (BN / 2) + c;
            if (valid) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                if (col0 + 8 * v < ncols) {
                  uint4 pk;
                  pk.x = pack_bf16(silu(gv[8 * v + 0]) * uv[8 * v + 0], silu(gv[8 * v + 1]) * uv[8 * v + 1]);
                  pk.y = pack_bf16(silu(gv[8 * v + 2]) * uv[8 * v + 2], silu(gv[8 * v + 3]) * uv[8 * v + 3]);
                  pk.z = pack_bf16(silu(gv[8 * v + 4]) * uv[8 * v + 4], silu(gv[8 * v + 5]) * uv[8 * v + 5]);
                  pk.w = pack_bf16(silu(gv[8 * v + 6]) * uv[8 * v + 6], silu(gv[8 * v + 7]) * uv[8 * v + 7]);
                  *reinterpret_cast<uint4*>(out + col0 + 8 * v) = pk;
                }
              }
            }
          }
        } else if (kTmaStoreOut && m0 + 32 <= w.rows) {
          // every row of this warp is valid: 64 columns at a time through a
          // staging box and one TMA store (whole 128-byte lines)
          const float scale = (!w.sh && p.row_scale) ? __ldg(p.row_scale + orow) : 1.0f;
          const CUtensorMap* om = w.sh ? &p.o_s : &p.o_r;
          const int orow0 = (int)(orow - (size_t)lane);
#pragma unroll 1
          for (int c = 0; c < BN; c += 64) {
            uint8_t* box = my_boxes + (n_boxes & 1) * OUT_BOX_BYTES;
            if (lane == 0) bulk_wait_read_1();    // the store that last read this box is done reading
            __syncwarp();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              float dv[32];
              tmem_ld32(tb + c + 32 * half, dv);
              uint32_t pk[16];
#pragma unroll
              for (int v = 0; v < 16; ++v) pk[v] = pack_out(p.out_f16, dv[2 * v] * scale, dv[2 * v + 1] * scale, hit);
              stage_row32(box, lane, 4 * half, pk);
            }
            fence_proxy_async_smem();             // the box is read by the async proxy
            __syncwarp();
            if (lane == 0) {
              const int x = w.nt * BN + c;
              if (x < ncols) tma_store_2d(om, box, x, orow0);   // columns past ncols are clipped
              bulk_commit();                      // one group per box, even an empty one
            }
            ++n_boxes;
          }
        } else {
          const float scale = (!w.sh && p.row_scale && valid) ? __ldg(p.row_scale + orow) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < BN; c += 32) {
            float dv[32];
            tmem_ld32(tb + c, dv);
            const int col0 = w.nt * BN + c;
            if (valid) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                if (col0 + 8 * v < ncols) {
                  uint4 pk;
                  pk.x = pack_out(p.out_f16, dv[8 * v + 0] * scale, dv[8 * v + 1] * scale, hit);
                  pk.y = pack_out(p.out_f16, dv[8 * v + 2] * scale, dv[8 * v + 3] * scale, hit);
                  pk.z = pack_out(p.out_f16, dv[8 * v + 4] * scale, dv[8 * v + 5] * scale, hit);
                  pk.w = pack_out(p.out_f16, dv[8 * v + 6] * scale, dv[8 * v + 7] * scale, hit);
                  *reinterpret_cast<uint4*>(out + col0 + 8 * v) = pk;
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(cluster_addr(&acc_empty[acc], 0));
    }
    // the staging boxes must not be released while a store still reads them
    if (kTmaStoreOut && lane == 0) bulk_wait_all();
    if (hit) set_device_error(p.err, MOE_DEVERR_RANGE);
  }

  // after a wait gave up, loads may still be landing in this CTA's shared
  // memory (the odd CTA cannot observe its own: they complete on the even
  // CTA's barrier); they finish within microseconds, so wait a millisecond
  if (*abort_flag) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 1000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // neither CTA leaves while the other may still signal it
  tc_fence_after();
  if (warp == 0) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Matrix [rows, cols] row-major (cols contiguous) of bf16 (q8 = false) or e4m3
// bytes (q8 = true); box = one 128-byte row segment (64 bf16 / 128 e4m3) x box_rows
static bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                      bool q8 = false) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows < 1 ? 1 : rows};
  cuuint64_t strides[1] = {cols * (q8 ? 1 : 2)};
  cuuint32_t box[2] = {(cuuint32_t)(q8 ? 2 * BK : BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, q8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row scales of an e4m3 weight blob: n*rows*cols code bytes, then n*rows fp32.
static const float* blob_scales(const void* blob, uint64_t rows, uint64_t cols) {
  return reinterpret_cast<const float*>(static_cast<const uint8_t*>(blob) + rows * cols);
}

}  // namespace tc

int tc_bm() { return tc::BM; }
int tc_merge_rows() { return tc::kMergeMaxRows; }
int tc_cols_gateup() { return tc::BN / 2; }
int tc_cols_down() { return tc::BN; }

static int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

// e (fp32) = e_hi + e_mid + e_lo exactly, each term bf16: e_hi = RN_bf16(e),
// the residual e - e_hi is exact in fp32 (Sterbenz) and carries at most 16
// significant bits, e_mid takes 8 of them and the last residual fits in bf16.
__global__ void split_centroids_kernel(const float* __restrict__ e, __nv_bfloat16* __restrict__ e3,
                                       size_t n) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float x = e[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const float r1 = __fsub_rn(x, __bfloat162float(hi));
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = __fsub_rn(r1, __bfloat162float(mid));
    e3[i] = hi;
    e3[n + i] = mid;
    e3[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

// Split-K plan of the router GEMM: never more than kRouterMaxKbPerSplit
// k-blocks per split -- the tensor core's fp32 accumulation over long K drifts
// (observed 7e-6 in s at d = 7168 with 84 k-blocks per split), so long
// reductions are cut into short partial sums that the select kernel adds in
// fp32, in split order -- and at most router_max_splits(T) splits.  Within those
// bounds the split length minimises the modelled time, waves x (k-blocks per
// unit + a unit's fixed cost of about kRouterUnitCostKb k-blocks) on n_sms
// SMs; ties go to longer splits (fewer partials for the select kernel).
constexpr int kRouterUnitCostKb = 4;

void router_split_plan(int T, int d, int E, int n_sms, int* ks, int* per) {
  const int base = ((T + tc::BM - 1) / tc::BM) * ((E + tc::BN - 1) / tc::BN);
  const int total = 3 * ((d + tc::BK - 1) / tc::BK);
  const int max_splits = router_max_splits(T);
  int p_lo = (total + max_splits - 1) / max_splits;
  const int p_hi = std::max(p_lo, std::min(kRouterMaxKbPerSplit, total));
  long best = -1;
  int best_p = p_hi;
  for (int p = p_hi; p >= p_lo; --p) {
    const long units = (long)base * ((total + p - 1) / p);
    const long t = ((units + n_sms - 1) / n_sms) * (p + kRouterUnitCostKb);
    if (best < 0 || t < best) { best = t; best_p = p; }
  }
  *per = best_p;
  *ks = (total + best_p - 1) / best_p;   // every split non-empty
}

cudaError_t launch_router_tc(const void* h, const float* e, void* e3, float* zpart, int T, int d,
                             int E, int* err, int* ks_out, cudaStream_t st) {
  using namespace tc;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaFuncSetAttribute(grouped_gemm_kernel<EPI_ROUTER, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_of<false>());
    attr_done[dev] = true;
  }
  const size_t n = (size_t)E * d;
  launch_pdl(split_centroids_kernel, dim3((unsigned)std::min<size_t>((n + 255) / 256, 148 * 8)), dim3(256), 0, st,
             e, reinterpret_cast<__nv_bfloat16*>(e3), n);
  int ks, per;
  router_split_plan(T, d, E, num_sms(), &ks, &per);
  Params p{};
  bool ok = true;
  ok &= make_tmap(&p.a_r, h, (uint64_t)T, d, BM);
  ok &= make_tmap(&p.a_s, h, (uint64_t)T, d, BM);
  // fewer than 256 experts: an N = round16(E) tile (the box then holds only
  // this part's centroid rows, not the next part's)
  const int rn = E >= BN ? BN : ((E + 15) / 16) * 16;
  ok &= make_tmap(&p.b0_r, e3, (uint64_t)3 * E, d, rn);
  ok &= make_tmap(&p.b1_r, e3, (uint64_t)3 * E, d, rn);
  ok &= make_tmap(&p.b0_s, e3, (uint64_t)3 * E, d, rn);
  ok &= make_tmap(&p.b1_s, e3, (uint64_t)3 * E, d, rn);
  if (!ok) return cudaErrorInvalidValue;
  p.r_T = T; p.r_E = E; p.r_n = rn;
  p.r_mtiles = (T + BM - 1) / BM;
  p.r_ntiles = (E + BN - 1) / BN;
  p.r_ks = ks; p.r_per = per;
  p.r_nkd = (d + BK - 1) / BK;
  p.zpart = zpart;
  p.bk = BK;
  p.G = 1; p.E_r = 1;
  p.err = err;
  const int units = p.r_mtiles * p.r_ntiles * ks;
  const int grid = std::min(units, num_sms());
  launch_pdl(grouped_gemm_kernel<EPI_ROUTER, false>, dim3(grid), dim3(NUM_THREADS), smem_of<false>(), st, p);
  *ks_out = ks;
  return cudaGetLastError();
}

int tc_pair_min_rows() { return tc::kPairMinRows; }
int tc_pair_rows() { return tc::P_M; }
int tc_pair_merge_rows() { return tc::kPairMergeMax; }

// Largest grid of CTA pairs that is resident at once (the pair kernel is
// persistent: a pair that had to wait for another to finish would double the
// time of its units).
static int pair_grid(const void* kern, size_t smem) {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  cfg.blockDim = dim3(tc::NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 1;
  }
  const int grid = 2 * std::min(n, num_sms() / 2);
  if (dev < 64) cached[dev] = grid;
  return grid;
}

static void pair_attributes() {
  using namespace tc;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaFuncSetAttribute(pair_gemm_kernel<EPI_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM);
    cudaFuncSetAttribute(pair_gemm_kernel<EPI_SCALE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM);
    cudaFuncSetAttribute(pair_gemm_kernel<EPI_SCALE, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)p_smem<true>());
    attr_done[dev] = true;
  }
}

// The pair kernels are worth launching only if the device co-schedules pairs
// on at least three quarters of its SMs (a B200 holds 74 two-CTA clusters of
// this kernel at once).
bool tc_pair_available() {
  pair_attributes();
  const int g = pair_grid((const void*)tc::pair_gemm_kernel<tc::EPI_SWIGLU>, tc::P_SMEM);
  return g >= (3 * num_sms()) / 4;
}

static cudaError_t launch_ffn_pair(const FfnArgs& a, int which, cudaStream_t st) {
  using namespace tc;
  pair_attributes();
  const bool has_s = a.E_s > 0;
  Params p{};
  bool ok = true;
  p.grp_rows = a.grp_rows;
  p.grp_row0 = a.grp_row0;
  p.G = a.E_r + a.E_s;
  p.E_r = a.E_r;
  p.err = a.err;
  p.bk = BK;
  const uint32_t half = BN / 2, quarter = BN / 4;
  if (which == 0) {
    // gate/up: A = permuted tokens (routed) or h (shared); B = 64 gate rows and
    // the 64 up rows of the same columns per CTA
    const uint64_t wr_r = (uint64_t)a.E_r * a.f_r, wr_s = has_s ? (uint64_t)a.E_s * a.f_s : wr_r;
    const void* xs = has_s ? a.x_s : a.x_r;
    const uint64_t xs_rows = has_s ? (uint64_t)a.T : (uint64_t)a.max_rows_r;
    ok &= make_tmap(&p.a_r, a.x_r, (uint64_t)a.max_rows_r, a.d, BM);
    ok &= make_tmap(&p.a_s, xs, xs_rows, a.d, BM);
    ok &= make_tmap(&p.a32_r, a.x_r, (uint64_t)a.max_rows_r, a.d, A_SUB_ROWS);
    ok &= make_tmap(&p.a32_s, xs, xs_rows, a.d, A_SUB_ROWS);
    ok &= make_tmap(&p.b0_r, a.wg_r, wr_r, a.d, quarter);
    ok &= make_tmap(&p.b1_r, a.wu_r, wr_r, a.d, quarter);
    ok &= make_tmap(&p.b0_s, has_s ? a.wg_s : a.wg_r, wr_s, a.d, quarter);
    ok &= make_tmap(&p.b1_s, has_s ? a.wu_s : a.wu_r, wr_s, a.d, quarter);
    p.prefix = a.pre_gu;
    p.k_r = p.k_s = a.d;
    p.wrows_r = a.f_r; p.wrows_s = a.f_s;
    p.ncols_r = a.f_r; p.ncols_s = a.f_s;
    p.out_r = (uint16_t*)a.act_r; p.out_s = (uint16_t*)a.act_s;
    p.row_scale = nullptr;
  } else {
    // down: A = act (routed / shared); B = W_down, 128 of the tile's 256 rows per CTA
    const uint64_t rows_s = has_s ? (uint64_t)a.E_s * a.T : (uint64_t)a.max_rows_r;
    const int fs = has_s ? a.f_s : a.f_r;
    const uint64_t wd_rows_s = (uint64_t)(has_s ? a.E_s : a.E_r) * a.d;
    ok &= make_tmap(&p.a_r, a.act_r, (uint64_t)a.max_rows_r, a.f_r, BM);
    ok &= make_tmap(&p.a_s, has_s ? a.act_s : a.act_r, rows_s, fs, BM);
    ok &= make_tmap(&p.a32_r, a.act_r, (uint64_t)a.max_rows_r, a.f_r, A_SUB_ROWS);
    ok &= make_tmap(&p.a32_s, has_s ? a.act_s : a.act_r, rows_s, fs, A_SUB_ROWS);
    ok &= make_tmap(&p.b0_r, a.wd_r, (uint64_t)a.E_r * a.d, a.f_r, half);
    ok &= make_tmap(&p.b1_r, a.wd_r, (uint64_t)a.E_r * a.d, a.f_r, half);
    ok &= make_tmap(&p.b0_s, has_s ? a.wd_s : a.wd_r, wd_rows_s, fs, half);
    ok &= make_tmap(&p.b1_s, has_s ? a.wd_s : a.wd_r, wd_rows_s, fs, half);
    p.prefix = a.pre_dn;
    p.k_r = a.f_r; p.k_s = a.f_s;
    p.wrows_r = a.d; p.wrows_s = a.d;
    p.ncols_r = a.d; p.ncols_s = a.d;
    p.out_r = (uint16_t*)a.out_r; p.out_s = (uint16_t*)a.out_s;
    p.row_scale = a.row_scale;
    p.out_f16 = a.out_f16;
    ok &= make_tmap(&p.o_r, a.out_r, (uint64_t)a.max_rows_r, a.d, OUT_BOX_ROWS);
    ok &= make_tmap(&p.o_s, has_s ? a.out_s : a.out_r, rows_s, a.d, OUT_BOX_ROWS);
  }
  if (!ok) return cudaErrorInvalidValue;
  p.tile_counter = a.tile_counters ? a.tile_counters + which : nullptr;
  // down GEMM with short units: outputs through the staging boxes and TMA stores
  const int kb_r = (a.f_r + p.bk - 1) / p.bk, kb_s = (p.k_s + p.bk - 1) / p.bk;
  const bool tma_out = which == 1 && std::max(kb_r, has_s ? kb_s : 0) <= kTmaOutMaxKb;
  auto kern = which == 0 ? pair_gemm_kernel<EPI_SWIGLU>
            : tma_out ? pair_gemm_kernel<EPI_SCALE, true> : pair_gemm_kernel<EPI_SCALE>;
  const size_t smem = tma_out ? p_smem<true>() : P_SMEM;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pair_grid((const void*)kern, smem));
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kUsePdl ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_ffn_tc(const FfnArgs& a, int which, cudaStream_t st) {
  using namespace tc;
  if (a.pair) return launch_ffn_pair(a, which, st);
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SWIGLU, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_of<false>());
    cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SCALE, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_of<false>());
    cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SWIGLU, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_of<false>());
    cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SCALE, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_of<false>());
    cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SCALE, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_of<true>());
    cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SCALE, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_of<true>());
    attr_done[dev] = true;
  }
  const bool has_s = a.E_s > 0;
  const bool q8 = a.q8 != 0;
  Params p{};
  bool ok = true;
  p.grp_rows = a.grp_rows;
  p.grp_row0 = a.grp_row0;
  p.G = a.E_r + a.E_s;
  p.E_r = a.E_r;
  p.err = a.err;
  p.bk = q8 ? 2 * BK : BK;
  if (which == 0) {
    // gate/up: A = permuted tokens (routed) or h (shared); B = gate | up, 128 rows each
    const uint64_t wr_r = (uint64_t)a.E_r * a.f_r, wr_s = has_s ? (uint64_t)a.E_s * a.f_s : wr_r;
    const void* xr = a.x_r;
    const uint64_t xr_rows = (uint64_t)a.max_rows_r;
    ok &= make_tmap(&p.a_r, xr, xr_rows, a.d, BM, q8);
    ok &= make_tmap(&p.a_s, has_s ? a.x_s : xr, has_s ? (uint64_t)a.T : xr_rows, a.d, BM, q8);
    ok &= make_tmap(&p.a32_r, xr, xr_rows, a.d, A_SUB_ROWS, q8);
    ok &= make_tmap(&p.a32_s, has_s ? a.x_s : xr, has_s ? (uint64_t)a.T : xr_rows, a.d, A_SUB_ROWS, q8);
    ok &= make_tmap(&p.b0_r, a.wg_r, wr_r, a.d, BN / 2, q8);
    ok &= make_tmap(&p.b1_r, a.wu_r, wr_r, a.d, BN / 2, q8);
    ok &= make_tmap(&p.b0_s, has_s ? a.wg_s : a.wg_r, wr_s, a.d, BN / 2, q8);
    ok &= make_tmap(&p.b1_s, has_s ? a.wu_s : a.wu_r, wr_s, a.d, BN / 2, q8);
    if (q8) {
      p.xs_r = a.xs_r; p.xs_s = has_s ? a.xs_s : a.xs_r;
      p.s0_r = blob_scales(a.wg_r, wr_r, a.d); p.s1_r = blob_scales(a.wu_r, wr_r, a.d);
      p.s0_s = has_s ? blob_scales(a.wg_s, wr_s, a.d) : p.s0_r;
      p.s1_s = has_s ? blob_scales(a.wu_s, wr_s, a.d) : p.s1_r;
    }
    p.prefix = a.pre_gu;
    p.uv_r = (uint16_t*)a.uv_r; p.uv_s = (uint16_t*)(has_s ? a.uv_s : a.uv_r);
    p.k_r = p.k_s = a.d;
    p.wrows_r = a.f_r; p.wrows_s = a.f_s;
    p.ncols_r = a.f_r; p.ncols_s = a.f_s;
    p.out_r = (uint16_t*)a.act_r; p.out_s = (uint16_t*)a.act_s;
    p.row_scale = nullptr;
  } else {
    // down: A = act (routed / shared); B = W_down, 256 rows
    const uint64_t rows_s = has_s ? (uint64_t)a.E_s * a.T : (uint64_t)a.max_rows_r;
    const int fs = has_s ? a.f_s : a.f_r;
    const uint64_t wd_rows_s = (uint64_t)(has_s ? a.E_s : a.E_r) * a.d;
    // e4m3: the down GEMM reads the quantized copy of A (act_q) and its row scales
    const void* A_r = q8 ? a.actq_r : a.act_r;
    const void* A_s = q8 ? a.actq_s : a.act_s;
    ok &= make_tmap(&p.a_r, A_r, (uint64_t)a.max_rows_r, a.f_r, BM, q8);
    ok &= make_tmap(&p.a_s, has_s ? A_s : A_r, rows_s, fs, BM, q8);
    ok &= make_tmap(&p.a32_r, A_r, (uint64_t)a.max_rows_r, a.f_r, A_SUB_ROWS, q8);
    ok &= make_tmap(&p.a32_s, has_s ? A_s : A_r, rows_s, fs, A_SUB_ROWS, q8);
    ok &= make_tmap(&p.b0_r, a.wd_r, (uint64_t)a.E_r * a.d, a.f_r, BN, q8);
    ok &= make_tmap(&p.b1_r, a.wd_r, (uint64_t)a.E_r * a.d, a.f_r, BN, q8);
    ok &= make_tmap(&p.b0_s, has_s ? a.wd_s : a.wd_r, wd_rows_s, fs, BN, q8);
    ok &= make_tmap(&p.b1_s, has_s ? a.wd_s : a.wd_r, wd_rows_s, fs, BN, q8);
    if (q8) {
      p.xs_r = a.as_r; p.xs_s = has_s ? a.as_s : a.as_r;
      p.s0_r = p.s1_r = blob_scales(a.wd_r, (uint64_t)a.E_r * a.d, a.f_r);
      p.s0_s = p.s1_s = has_s ? blob_scales(a.wd_s, wd_rows_s, fs) : p.s0_r;
    }
    ok &= make_tmap(&p.o_r, a.out_r, (uint64_t)a.max_rows_r, a.d, OUT_BOX_ROWS);
    ok &= make_tmap(&p.o_s, has_s ? a.out_s : a.out_r, rows_s, a.d, OUT_BOX_ROWS);
    p.prefix = a.pre_dn;
    p.k_r = a.f_r; p.k_s = a.f_s;
    p.wrows_r = a.d; p.wrows_s = a.d;
    p.ncols_r = a.d; p.ncols_s = a.d;
    p.out_r = (uint16_t*)a.out_r; p.out_s = (uint16_t*)a.out_s;
    p.row_scale = a.row_scale;
    p.out_f16 = a.out_f16;
  }
  if (!ok) return cudaErrorInvalidValue;
  p.tile_counter = a.tile_counters ? a.tile_counters + which : nullptr;
  const int grid = num_sms();
  // down GEMM with short units: outputs through the staging boxes and TMA stores
  const int kb_r = (a.f_r + p.bk - 1) / p.bk, kb_s = (p.k_s + p.bk - 1) / p.bk;
  const bool tma_out = which == 1 && std::max(kb_r, has_s ? kb_s : 0) <= kTmaOutMaxKb;
  auto kern = which == 0 ? (q8 ? grouped_gemm_kernel<EPI_SWIGLU, true> : grouped_gemm_kernel<EPI_SWIGLU, false>)
            : tma_out ? (q8 ? grouped_gemm_kernel<EPI_SCALE, true, true> : grouped_gemm_kernel<EPI_SCALE, false, true>)
                      : (q8 ? grouped_gemm_kernel<EPI_SCALE, true> : grouped_gemm_kernel<EPI_SCALE, false>);
  const size_t smem = tma_out ? smem_of<true>() : smem_of<false>();
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(NUM_THREADS), smem, st, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
