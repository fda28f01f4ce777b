// Backward of the grouped SwiGLU experts on the 5th-generation tensor cores.
//
// For the rows X of one expert (permuted order), the saved pre-activations
// U = X W_g^T, V = X W_u^T and products A = SiLU(U) * V, and the output
// gradient dO (= g * dy for routed rows, dy for shared ones):
//   dA = dO W_d                      (EPI_DA; epilogue: dU = dA V SiLU'(U), dV = dA SiLU(U))
//   dX = dU W_g + dV W_u             (EPI_DX)
//   dW_d = dO^T A, dW_g = dU^T X, dW_u = dV^T X        (EPI_DW)
// -- the derivative of "Sparse Mixture-of-Experts (MoE): Routing Math, Load
// Balancing & Expert Parallelism", section 0 layer equation, per expert.
//
// The weights enter dA and dX untransposed, so B is an MN-major operand
// (TMA boxes of {64 MN-elements, 64 K-lines}, descriptor sdesc_mnmajor_sw128);
// the weight gradients reduce over an expert's rows, so both operands are
// MN-major there and K (the row count) ends inside a k-block: the lines past
// the expert's last row are zeroed in shared memory before the MMAs read them.
//
// Same persistent, warp-specialised structure as the forward GEMM: warp 0 =
// TMA producer + TMEM allocation, warp 1 = MMA issuer (lane 0 issues; the
// whole warp zeroes the K tail of EPI_DW), warps 2..5 = epilogue; 4 stages of
// 48 KB; two 256-column TMEM accumulators; every wait bounded.
#include <algorithm>
#include <cuda.h>
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace bwd {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int MN_BOX = 64;                      // MN-elements per MN-major box (128 bytes)
constexpr int MN_BOX_BYTES = MN_BOX * BK * 2;   // 8 KB
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int UNIT_RING = 4;
// EPI_DA / EPI_DX: a last row tile of <= MERGE_ROWS rows rides in the unit of
// the full tile before it (transposed: the stage's weight block is the M
// operand, the tail rows the N operand), so an expert of 129..192 rows stages
// each weight tile once; the tail rows take T_BYTES per stage (32-row boxes)
constexpr int MERGE_ROWS = 64;
constexpr int SUB_ROWS = 32;
constexpr int SUB_BYTES = SUB_ROWS * BK * 2;
constexpr int T_BYTES = MERGE_ROWS * BK * 2;
constexpr size_t SMEM_BYTES = (size_t)STAGES * (STAGE_BYTES + T_BYTES) + 1024 + 512;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
// EPI_DW: 3 stages (an expert has few k-blocks) and a 64 KB staging buffer for
// the output tile, written back by TMA stores (4 boxes of 64 columns x 128 rows)
constexpr int DW_STAGES = 3;
constexpr int DW_OUT_BYTES = BM * BN * 2;
constexpr size_t DW_SMEM_BYTES = (size_t)DW_STAGES * STAGE_BYTES + DW_OUT_BYTES + 1024 + 512;

enum { EPI_DA = 0, EPI_DX = 1, EPI_DW = 2 };

struct Params {
  CUtensorMap a_r, a_s;                  // A operand, routed / shared groups
  CUtensorMap a32_r, a32_s;              // EPI_DA / EPI_DX: the same rows with a 32-row box (tails)
  CUtensorMap b0_r, b1_r, b0_s, b1_s;    // B operand (EPI_DX: b0 = W_g for k < kb_split, b1 = W_u)
  const int* grp_rows;
  const int* grp_row0;
  const int* prefix;                     // EPI_DA / EPI_DX: unit prefix over the groups
  int G, E_r;
  int a_sh_zero, b_sh_zero;              // shared groups read A / B from row 0 (dy, h), not row0[g]
  // EPI_DA / EPI_DX
  int k_r, k_s, kb_split_r, kb_split_s, wrows_r, wrows_s, ncols_r, ncols_s, ld_r, ld_s;
  uint16_t* out_r;
  uint16_t* out_s;
  const uint16_t* uv_r;                  // EPI_DA: saved U | V rows [rows, 2f]
  const uint16_t* uv_s;
  int f_r, f_s;
  // EPI_DW
  int M_r, N_r, M_s, N_s, mt_r, nt_r, mt_s, nt_s;
  int a_x0_r, a_x0_s;                    // column offset into A's rows (dW_u: the V half, f)
  uint16_t* dw_r;                        // [E, M, N] bf16
  uint16_t* dw_s;
  CUtensorMap dws_r, dws_s;              // EPI_DW store maps over [E, M, N], box {64, 128, 1}
  int* err;
};

struct Unit {
  int g, mt, nt, nk, rows;
  int tail, t16;                         // EPI_DA / EPI_DX: merged tail rows, MMA N of the tail
  bool sh;
};

template <int EPI>
__device__ __forceinline__ int total_units(const Params& p) {
  if (EPI == EPI_DW) return p.E_r * p.mt_r * p.nt_r + (p.G - p.E_r) * p.mt_s * p.nt_s;
  return __ldg(p.prefix + p.G);
}

template <int EPI>
__device__ __forceinline__ Unit decode(const Params& p, int u) {
  Unit w;
  if (EPI == EPI_DW) {
    const int per_r = p.mt_r * p.nt_r;
    int local;
    if (u < p.E_r * per_r) {
      w.g = u / per_r; local = u - w.g * per_r; w.sh = false;
      w.mt = local % p.mt_r; w.nt = local / p.mt_r;
    } else {
      const int per_s = p.mt_s * p.nt_s, v = u - p.E_r * per_r;
      w.g = p.E_r + v / per_s; local = v % per_s; w.sh = true;
      w.mt = local % p.mt_s; w.nt = local / p.mt_s;
    }
    w.rows = __ldg(p.grp_rows + w.g);
    w.nk = (w.rows + BK - 1) / BK;
    w.tail = w.t16 = 0;
    return w;
  }
  int lo = 0, hi = p.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p.prefix + mid) <= u) lo = mid; else hi = mid;
  }
  w.g = lo;
  w.sh = lo >= p.E_r;
  w.rows = __ldg(p.grp_rows + lo);
  const int mtiles = (w.rows + BM - 1) / BM;
  const int last = w.rows - (mtiles - 1) * BM;
  const int runits = mtiles - ((mtiles >= 2 && last <= MERGE_ROWS) ? 1 : 0);
  const int local = u - __ldg(p.prefix + lo);
  w.mt = local % runits;
  w.nt = local / runits;
  w.nk = ((w.sh ? p.k_s : p.k_r) + BK - 1) / BK;
  w.tail = (runits < mtiles && w.mt == runits - 1) ? last : 0;
  w.t16 = (w.tail + 15) & ~15;
  return w;
}

__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, int* err) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) { set_device_error(err, MOE_DEVERR_WAIT_TIMEOUT); return; }
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void unpack8(uint4 q, float* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Loads of k-block i of unit w into stage buffers sa / sb.
template <int EPI>
__device__ __forceinline__ void load_stage(const Params& p, const Unit& w, int i, uint8_t* sa, uint8_t* sb,
                                           uint8_t* st, uint64_t* bar) {
  const CUtensorMap* am = w.sh ? &p.a_s : &p.a_r;
  const int row0 = __ldg(p.grp_row0 + w.g);
  const int e = w.sh ? w.g - p.E_r : w.g;
  if (EPI == EPI_DW) {
    // A: rows of the group (K) x 128 MN-columns (two boxes); B: 256 MN-columns (four boxes)
    const int ay = (w.sh && p.a_sh_zero ? 0 : row0) + i * BK;
    const int by = (w.sh && p.b_sh_zero ? 0 : row0) + i * BK;
    const CUtensorMap* bm = w.sh ? &p.b0_s : &p.b0_r;
#pragma unroll
    for (int j = 0; j < BM / MN_BOX; ++j)
      tma_load_2d(sa + j * MN_BOX_BYTES, am, bar, (w.sh ? p.a_x0_s : p.a_x0_r) + w.mt * BM + j * MN_BOX, ay);
#pragma unroll
    for (int j = 0; j < BN / MN_BOX; ++j) tma_load_2d(sb + j * MN_BOX_BYTES, bm, bar, w.nt * BN + j * MN_BOX, by);
  } else {
    // A: 128 rows of the group, K-major; B: K-lines of the expert's weight, 256 MN-columns
    const int ay = (EPI == EPI_DA && w.sh && p.a_sh_zero ? 0 : row0) + w.mt * BM;
    tma_load_2d(sa, am, bar, i * BK, ay);
    for (int q = 0; q * SUB_ROWS < w.t16; ++q)
      tma_load_2d(st + q * SUB_BYTES, w.sh ? &p.a32_s : &p.a32_r, bar, i * BK, ay + BM + q * SUB_ROWS);
    const int split = w.sh ? p.kb_split_s : p.kb_split_r;
    const bool second = EPI == EPI_DX && i >= split;
    const CUtensorMap* bm = w.sh ? (second ? &p.b1_s : &p.b0_s) : (second ? &p.b1_r : &p.b0_r);
    const int by = e * (w.sh ? p.wrows_s : p.wrows_r) + (second ? i - split : i) * BK;
#pragma unroll
    for (int j = 0; j < BN / MN_BOX; ++j) tma_load_2d(sb + j * MN_BOX_BYTES, bm, bar, w.nt * BN + j * MN_BOX, by);
  }
}

__device__ __forceinline__ void tma_store_3d(const void* tmap, const void* smem_src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
               :: "l"(tmap), "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// all but the most recent bulk group have read their shared memory
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }


// Epilogue of a merged tail (EPI_DA / EPI_DX): TMEM lane r of half h holds
// output column nt*256 + h*128 + r, accumulator column t the tail row t.
template <int EPI>
__device__ __noinline__ void epilogue_tail(const Params& p, const Unit& w, int r, uint32_t tb) {
  const size_t row0 = (size_t)__ldg(p.grp_row0 + w.g) + (size_t)(w.mt + 1) * BM;
  const int ncols = w.sh ? p.ncols_s : p.ncols_r;
  const int ld = w.sh ? p.ld_s : p.ld_r;
  const int f = w.sh ? p.f_s : p.f_r;
  uint16_t* out = w.sh ? p.out_s : p.out_r;
  const uint16_t* uv = EPI == EPI_DA ? (w.sh ? p.uv_s : p.uv_r) : nullptr;
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const int col = w.nt * BN + h * (BN / 2) + r;
#pragma unroll 1
    for (int c = 0; c < w.t16; c += 32) {
      float dv[32];
      tmem_ld32(tb + h * (BN / 2) + c, dv);
      if (col < ncols) {
#pragma unroll
        for (int v = 0; v < 32; ++v) {
          const int t = c + v;
          if (t < w.tail) {
            const size_t row = row0 + t;
            if (EPI == EPI_DA) {
              const float uu = __uint_as_float((uint32_t)uv[row * 2 * f + col] << 16);
              const float vv = __uint_as_float((uint32_t)uv[row * 2 * f + f + col] << 16);
              const float sg = 1.0f / (1.0f + __expf(-uu));
              out[row * ld + col] = __bfloat16_as_ushort(__float2bfloat16_rn(dv[v] * vv * sg * (1.0f + uu * (1.0f - sg))));
              out[row * ld + f + col] = __bfloat16_as_ushort(__float2bfloat16_rn(dv[v] * uu * sg));
            } else {
              out[row * ld + col] = __bfloat16_as_ushort(__float2bfloat16_rn(dv[v]));
            }
          }
        }
      }
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1) bwd_gemm_kernel(const __grid_constant__ Params p) {
  constexpr int STAGES = EPI == EPI_DW ? DW_STAGES : bwd::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sOut = smem + STAGES * STAGE_BYTES;                  // EPI_DW staging (1024-aligned)
  uint8_t* sT = sOut;                                            // EPI_DA / EPI_DX: merged tails' rows
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES +
                                               (EPI == EPI_DW ? DW_OUT_BYTES : STAGES * T_BYTES));
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* stg_full = drain + 1;        // EPI_DW [2]: a staged half tile is complete (128 arrivals)
  uint64_t* stg_free = stg_full + 2;     // EPI_DW [2]: that buffer's previous stores have read it
  uint64_t* unit_full = stg_free + 2;
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
    for (int q = 0; q < 2; ++q) { mbar_init(&stg_full[q], 4 * kWarp); mbar_init(&stg_free[q], 1); }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&p.a_r); prefetch_tmap(&p.a_s); prefetch_tmap(&p.b0_r);
    prefetch_tmap(&p.b1_r); prefetch_tmap(&p.b0_s); prefetch_tmap(&p.b1_s);
    if (EPI != EPI_DW) { prefetch_tmap(&p.a32_r); prefetch_tmap(&p.a32_s); }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_units<EPI>(p);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (static round-robin over the CTAs) ----------------
      int stage = 0, issued = 0, slot = 0;
      uint32_t phase = 0, uphase = 0;
      for (int k = 0;; ++k) {
        int u = (int)blockIdx.x + k * (int)gridDim.x;
        if (u >= total) u = -1;
        if (!mbar_wait(&unit_empty[slot], uphase ^ 1u, abort_flag, p.err)) goto producer_done;
        unit_ring[slot] = u;
        mbar_arrive(&unit_full[slot]);
        if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
        if (u < 0) break;
        const Unit w = decode<EPI>(p, u);
        const uint32_t tx = STAGE_BYTES + ((w.t16 + SUB_ROWS - 1) / SUB_ROWS) * SUB_BYTES;
        for (int i = 0; i < w.nk; ++i) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err)) goto producer_done;
          mbar_arrive_expect_tx(&full[stage], tx);
          load_stage<EPI>(p, w, i, sA + stage * A_BYTES, sB + stage * B_BYTES, sT + stage * T_BYTES,
                          &full[stage]);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    producer_done:
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (--stage < 0) { stage = STAGES - 1; phase ^= 1u; }
        wait_drain(&full[stage], phase, p.err);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (lane 0; the warp zeroes K tails) ----------------
    constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN) | kIdescBMnMajor | (EPI == EPI_DW ? kIdescAMnMajor : 0u);
    int stage = 0, slot = 0, nb = 0;
    uint32_t phase = 0, uphase = 0, ph_e = 0;      // ph_e bit b: phase of acc_empty[b]
    bool ok = true;
    for (;;) {
      if (!mbar_wait(&unit_full[slot], uphase, abort_flag, p.err)) { ok = false; break; }
      const int u = unit_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&unit_empty[slot]);
      if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
      if (u < 0) break;
      const Unit w = decode<EPI>(p, u);
      // a unit with a merged tail holds buffer 0 (full tile) and buffer 1 (tail, transposed)
      const bool two = w.tail > 0;
      const int acc = two ? 0 : nb;
      if (!mbar_wait(&acc_empty[acc], ((ph_e >> acc) & 1u) ^ 1u, abort_flag, p.err)) { ok = false; break; }
      ph_e ^= 1u << acc;
      if (two) {
        if (!mbar_wait(&acc_empty[1], ((ph_e >> 1) & 1u) ^ 1u, abort_flag, p.err)) { ok = false; break; }
        ph_e ^= 2u;
      }
      nb = two ? 0 : nb ^ 1;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      const uint32_t d_tail = tmem_base + (uint32_t)BN;
      // tail MMA: the weight block's two 128-column halves (MN-major, M = 128)
      // against the tail rows (K-major, N = t16)
      const uint32_t idesc_tail = idesc_bf16_f32(BM, w.t16 ? w.t16 : 16) | kIdescAMnMajor;
      for (int kb = 0; kb < w.nk; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
        uint8_t* a_st = sA + stage * A_BYTES;
        uint8_t* b_st = sB + stage * B_BYTES;
        if (EPI == EPI_DW) {
          const int valid = w.rows - kb * BK;           // K-lines that belong to the group
          if (valid < BK) {
            // zero lines valid..63 of A's two 64-element MN blocks: with those
            // lines zero, B's lines past the group (the next group's rows, the
            // zeroed rows after the last routed row, or TMA's zero fill) add nothing
            for (int line = valid + (lane >> 3); line < BK; line += kWarp / 8) {
              *reinterpret_cast<uint4*>(a_st + line * 128 + (lane & 7) * 16) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(a_st + MN_BOX_BYTES + line * 128 + (lane & 7) * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
        }
        if (lane == 0) {
          tc_fence_after();
          const uint32_t a0 = smem_u32(a_st), b0 = smem_u32(b_st);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t ad = EPI == EPI_DW ? sdesc_mnmajor_sw128(a0 + k * UMMA_K * 128)
                                              : sdesc_kmajor_sw128(a0 + k * UMMA_K * 2);
            tc_mma_bf16(d_tmem, ad, sdesc_mnmajor_sw128(b0 + k * UMMA_K * 128), IDESC, (kb | k) != 0);
          }
          if (EPI != EPI_DW && two) {
            const uint32_t t0 = smem_u32(sT + stage * T_BYTES);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              const uint64_t xd = sdesc_kmajor_sw128(t0 + k * UMMA_K * 2);
              tc_mma_bf16(d_tail, sdesc_mnmajor_sw128(b0 + k * UMMA_K * 128), xd, idesc_tail, (kb | k) != 0);
              tc_mma_bf16(d_tail + BN / 2, sdesc_mnmajor_sw128(b0 + 2 * MN_BOX_BYTES + k * UMMA_K * 128), xd,
                          idesc_tail, (kb | k) != 0);
            }
          }
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(&acc_full[acc]);                   // with no k-block: arrives at once
        if (two) tc_commit(&acc_full[1]);
      }
      __syncwarp();
    }
    if (lane == 0) {
      tc_commit(drain);
      wait_drain(drain, 0, p.err);
    }
    (void)ok;
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    int slot = 0, nb = 0;
    uint32_t uphase = 0, ph_f = 0;                 // ph_f bit b: phase of acc_full[b]
    uint32_t stg_count = 0;                        // EPI_DW: half tiles staged so far
    for (;;) {
      if (!mbar_wait(&unit_full[slot], uphase, abort_flag, p.err)) break;
      const int u = unit_ring[slot];
      mbar_arrive(&unit_empty[slot]);
      if (++slot == UNIT_RING) { slot = 0; uphase ^= 1u; }
      if (u < 0) break;
      const Unit w = decode<EPI>(p, u);
      const bool two = w.tail > 0;                  // same buffer sequence as the MMA issuer
      const int acc = two ? 0 : nb;
      nb = two ? 0 : nb ^ 1;
      if (!mbar_wait(&acc_full[acc], (ph_f >> acc) & 1u, abort_flag, p.err)) break;
      ph_f ^= 1u << acc;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BN);
      if (EPI == EPI_DW) {
        // weight-gradient tile, written as two halves of 128 columns through
        // two 32 KB staging buffers used in turn, so that one half's TMA stores
        // drain while the next half is staged.  A half is two 128-row x
        // 64-column boxes in the 128-byte swizzle layout of the store map
        // (16-byte chunk j of line r at chunk j ^ (r & 7)); each warp writes
        // lines sub*32.., one thread issues the stores, which clip at the
        // expert's M and N
        const bool leader = warp == 2 && lane == 0;
        bool aborted = false;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int bf = stg_count & 1;
          const uint32_t par = (stg_count >> 1) & 1u;
          uint8_t* buf = sOut + bf * (DW_OUT_BYTES / 2);
          if (leader) {
            bulk_wait_read_1();                       // the stores that last used buf have read it
            mbar_arrive(&stg_free[bf]);
          }
          if (!mbar_wait(&stg_free[bf], par, abort_flag, p.err)) { aborted = true; break; }
#pragma unroll 1
          for (int c = 0; c < BN / 2; c += 32) {
            float dv[32];
            tmem_ld32(tb + half * (BN / 2) + c, dv);
            uint8_t* line = buf + (c / 64) * (DW_OUT_BYTES / 4) + r * 128;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 pk;
              if (w.nk == 0) pk = make_uint4(0, 0, 0, 0);        // an expert without rows
              else {
                pk.x = pack_bf16(dv[8 * v + 0], dv[8 * v + 1]);
                pk.y = pack_bf16(dv[8 * v + 2], dv[8 * v + 3]);
                pk.z = pack_bf16(dv[8 * v + 4], dv[8 * v + 5]);
                pk.w = pack_bf16(dv[8 * v + 6], dv[8 * v + 7]);
              }
              const int chunk = ((c % 64) / 8 + v) ^ (r & 7);
              *reinterpret_cast<uint4*>(line + chunk * 16) = pk;
            }
          }
          if (half == 1) {
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);              // TMEM is free; the stores go on
          }
          fence_proxy_async_smem();
          mbar_arrive(&stg_full[bf]);
          if (leader) {
            if (!mbar_wait(&stg_full[bf], par, abort_flag, p.err)) { aborted = true; break; }
            const int e = w.sh ? w.g - p.E_r : w.g;
            const CUtensorMap* dm = w.sh ? &p.dws_s : &p.dws_r;
#pragma unroll
            for (int q = 0; q < 2; ++q)
              tma_store_3d(dm, buf + q * (DW_OUT_BYTES / 4), w.nt * BN + half * (BN / 2) + q * 64, w.mt * BM, e);
            bulk_commit();
          }
          ++stg_count;
        }
        if (aborted) break;
        continue;
      } else {
        const int m = w.mt * BM + r;
        const bool valid = m < w.rows;
        const size_t orow = (size_t)__ldg(p.grp_row0 + w.g) + m;
        const int ncols = w.sh ? p.ncols_s : p.ncols_r;
        const int ld = w.sh ? p.ld_s : p.ld_r;
        uint16_t* out = (w.sh ? p.out_s : p.out_r) + orow * ld;
        const int f = w.sh ? p.f_s : p.f_r;
        const uint16_t* uv = EPI == EPI_DA ? (w.sh ? p.uv_s : p.uv_r) + orow * (size_t)(2 * f) : nullptr;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float dv[32];
          tmem_ld32(tb + c, dv);
          const int col0 = w.nt * BN + c;
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int col = col0 + 8 * v;
              if (col < ncols) {
                if (EPI == EPI_DA) {
                  // dU = dA V SiLU'(U), dV = dA SiLU(U), SiLU'(u) = sig (1 + u (1 - sig))
                  float uu[8], vv[8];
                  unpack8(*reinterpret_cast<const uint4*>(uv + col), uu);
                  unpack8(*reinterpret_cast<const uint4*>(uv + f + col), vv);
                  float du[8], dvv[8];
#pragma unroll
                  for (int q = 0; q < 8; ++q) {
                    const float sg = 1.0f / (1.0f + __expf(-uu[q]));
                    const float da = dv[8 * v + q];
                    du[q] = da * vv[q] * sg * (1.0f + uu[q] * (1.0f - sg));
                    dvv[q] = da * uu[q] * sg;
                  }
                  *reinterpret_cast<uint4*>(out + col) =
                      make_uint4(pack_bf16(du[0], du[1]), pack_bf16(du[2], du[3]), pack_bf16(du[4], du[5]),
                                 pack_bf16(du[6], du[7]));
                  *reinterpret_cast<uint4*>(out + f + col) =
                      make_uint4(pack_bf16(dvv[0], dvv[1]), pack_bf16(dvv[2], dvv[3]), pack_bf16(dvv[4], dvv[5]),
                                 pack_bf16(dvv[6], dvv[7]));
                } else {
                  uint4 pk;
                  pk.x = pack_bf16(dv[8 * v + 0], dv[8 * v + 1]);
                  pk.y = pack_bf16(dv[8 * v + 2], dv[8 * v + 3]);
                  pk.z = pack_bf16(dv[8 * v + 4], dv[8 * v + 5]);
                  pk.w = pack_bf16(dv[8 * v + 6], dv[8 * v + 7]);
                  *reinterpret_cast<uint4*>(out + col) = pk;
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (EPI != EPI_DW && two) {
        // the merged tail (rows (mt + 1) * 128 ..), transposed in buffer 1
        if (!mbar_wait(&acc_full[1], (ph_f >> 1) & 1u, abort_flag, p.err)) break;
        ph_f ^= 2u;
        tc_fence_after();
        epilogue_tail<EPI>(p, w, r, tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)BN);
        tc_fence_before();
        mbar_arrive(&acc_empty[1]);
      }
    }
  }

  if (EPI == EPI_DW && warp == 2 && lane == 0) bulk_wait_all();   // every TMA store has landed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, TMEM_COLS);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 matrix [rows, cols] row-major; box = 64 columns x box_rows lines
static bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc || !base) return false;
  cuuint64_t dims[2] = {cols, rows < 1 ? 1 : rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor [n, rows, cols] for TMA stores; box = 64 columns x 128 rows x 1
static bool make_store_map(CUtensorMap* m, const void* base, uint64_t n, uint64_t rows, uint64_t cols) {
  EncodeTiledFn enc = get_encode();
  if (!enc || !base) return false;
  cuuint64_t dims[3] = {cols, rows, n < 1 ? 1 : n};
  cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

template <int EPI>
static cudaError_t launch(const Params& p, int units, cudaStream_t st) {
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = EPI == EPI_DW ? DW_SMEM_BYTES : SMEM_BYTES;
  if (dev < 64 && !attr_done[dev]) {
    cudaFuncSetAttribute(bwd_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr_done[dev] = true;
  }
  const int grid = std::max(1, std::min(units, num_sms()));
  bwd_gemm_kernel<EPI><<<grid, NUM_THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace bwd

int bwd_merge_rows() { return bwd::MERGE_ROWS; }

cudaError_t launch_bwd_tc(const BwdArgs& a, int which, cudaStream_t st) {
  using namespace bwd;
  Params p{};
  bool ok = true;
  const bool has_s = a.E_s > 0;
  const int fs = has_s ? a.f_s : a.f_r;
  const uint64_t R = (uint64_t)a.max_rows_r, RS = has_s ? (uint64_t)a.E_s * a.T : R;
  p.grp_rows = a.grp_rows; p.grp_row0 = a.grp_row0;
  p.G = a.E_r + a.E_s; p.E_r = a.E_r;
  p.err = a.err;
  p.f_r = a.f_r; p.f_s = fs;
  if (which == 0) {
    // dA = dO W_d -> dU | dV (routed rows: dO = g dy; shared rows: dy itself)
    ok &= make_tmap(&p.a_r, a.dO_r, R, a.d, BM);
    ok &= make_tmap(&p.a_s, has_s ? a.dy : a.dO_r, has_s ? (uint64_t)a.T : R, a.d, BM);
    ok &= make_tmap(&p.a32_r, a.dO_r, R, a.d, SUB_ROWS);
    ok &= make_tmap(&p.a32_s, has_s ? a.dy : a.dO_r, has_s ? (uint64_t)a.T : R, a.d, SUB_ROWS);
    ok &= make_tmap(&p.b0_r, a.wd_r, (uint64_t)a.E_r * a.d, a.f_r, BK);
    ok &= make_tmap(&p.b0_s, has_s ? a.wd_s : a.wd_r, (uint64_t)(has_s ? a.E_s : a.E_r) * a.d, fs, BK);
    p.b1_r = p.b0_r; p.b1_s = p.b0_s;
    p.a_sh_zero = 1;
    p.prefix = a.pre_da;
    p.k_r = p.k_s = a.d;
    p.kb_split_r = p.kb_split_s = 1 << 30;
    p.wrows_r = p.wrows_s = a.d;
    p.ncols_r = a.f_r; p.ncols_s = fs;
    p.ld_r = 2 * a.f_r; p.ld_s = 2 * fs;
    p.out_r = (uint16_t*)a.duv_r; p.out_s = (uint16_t*)(has_s ? a.duv_s : a.duv_r);
    p.uv_r = (const uint16_t*)a.uv_r; p.uv_s = (const uint16_t*)(has_s ? a.uv_s : a.uv_r);
    if (!ok) return cudaErrorInvalidValue;
    return launch<EPI_DA>(p, 148 * 64, st);
  }
  if (which == 1) {
    // dX = [dU | dV] [W_g ; W_u]
    ok &= make_tmap(&p.a_r, a.duv_r, R, 2 * (uint64_t)a.f_r, BM);
    ok &= make_tmap(&p.a_s, has_s ? a.duv_s : a.duv_r, RS, 2 * (uint64_t)fs, BM);
    ok &= make_tmap(&p.a32_r, a.duv_r, R, 2 * (uint64_t)a.f_r, SUB_ROWS);
    ok &= make_tmap(&p.a32_s, has_s ? a.duv_s : a.duv_r, RS, 2 * (uint64_t)fs, SUB_ROWS);
    ok &= make_tmap(&p.b0_r, a.wg_r, (uint64_t)a.E_r * a.f_r, a.d, BK);
    ok &= make_tmap(&p.b1_r, a.wu_r, (uint64_t)a.E_r * a.f_r, a.d, BK);
    ok &= make_tmap(&p.b0_s, has_s ? a.wg_s : a.wg_r, (uint64_t)(has_s ? a.E_s : a.E_r) * fs, a.d, BK);
    ok &= make_tmap(&p.b1_s, has_s ? a.wu_s : a.wu_r, (uint64_t)(has_s ? a.E_s : a.E_r) * fs, a.d, BK);
    p.prefix = a.pre_dx;
    p.k_r = 2 * a.f_r; p.k_s = 2 * fs;
    p.kb_split_r = a.f_r / BK; p.kb_split_s = fs / BK;
    p.wrows_r = a.f_r; p.wrows_s = fs;
    p.ncols_r = p.ncols_s = a.d;
    p.ld_r = p.ld_s = a.d;
    p.out_r = (uint16_t*)a.dx_r; p.out_s = (uint16_t*)(has_s ? a.dx_s : a.dx_r);
    if (!ok) return cudaErrorInvalidValue;
    return launch<EPI_DX>(p, 148 * 64, st);
  }
  // weight gradients: which 2 = W_d (dO^T A), 3 = W_g (dU^T X), 4 = W_u (dV^T X)
  if (which == 2) {
    ok &= make_tmap(&p.a_r, a.dO_r, R, a.d, BK);
    ok &= make_tmap(&p.a_s, has_s ? a.dy : a.dO_r, has_s ? (uint64_t)a.T : R, a.d, BK);
    ok &= make_tmap(&p.b0_r, a.act_r, R, a.f_r, BK);
    ok &= make_tmap(&p.b0_s, has_s ? a.act_s : a.act_r, RS, fs, BK);
    p.a_sh_zero = 1; p.b_sh_zero = 0;
    p.M_r = a.d; p.N_r = a.f_r; p.M_s = a.d; p.N_s = fs;
    p.dw_r = (uint16_t*)a.dwd_r; p.dw_s = (uint16_t*)a.dwd_s;
  } else {
    const bool up = which == 4;
    ok &= make_tmap(&p.a_r, a.duv_r, R, 2 * (uint64_t)a.f_r, BK);
    ok &= make_tmap(&p.a_s, has_s ? a.duv_s : a.duv_r, RS, 2 * (uint64_t)fs, BK);
    ok &= make_tmap(&p.b0_r, a.x_r, R, a.d, BK);
    ok &= make_tmap(&p.b0_s, has_s ? a.h : a.x_r, has_s ? (uint64_t)a.T : R, a.d, BK);
    p.a_sh_zero = 0; p.b_sh_zero = 1;
    p.M_r = a.f_r; p.N_r = a.d; p.M_s = fs; p.N_s = a.d;
    p.a_x0_r = up ? a.f_r : 0;
    p.a_x0_s = up ? fs : 0;
    p.dw_r = (uint16_t*)(up ? a.dwu_r : a.dwg_r); p.dw_s = (uint16_t*)(up ? a.dwu_s : a.dwg_s);
  }
  p.b1_r = p.b0_r; p.b1_s = p.b0_s;
  ok &= make_store_map(&p.dws_r, p.dw_r, (uint64_t)a.E_r, p.M_r, p.N_r);
  ok &= make_store_map(&p.dws_s, has_s ? (const void*)p.dw_s : (const void*)p.dw_r, (uint64_t)(has_s ? a.E_s : a.E_r),
                       has_s ? p.M_s : p.M_r, has_s ? p.N_s : p.N_r);
  p.mt_r = (p.M_r + BM - 1) / BM; p.nt_r = (p.N_r + BN - 1) / BN;
  p.mt_s = (p.M_s + BM - 1) / BM; p.nt_s = (p.N_s + BN - 1) / BN;
  if (!ok) return cudaErrorInvalidValue;
  const int units = a.E_r * p.mt_r * p.nt_r + a.E_s * p.mt_s * p.nt_s;
  return launch<EPI_DW>(p, units, st);
}

}  // namespace moe
