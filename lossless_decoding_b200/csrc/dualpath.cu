// Dual-pathway linear of a diffusion-augmented layer on sm_100a.
//
// Operation: "Unlocking Lossless Speedups in LLMs via Discrete Diffusion",
// picx.dev summary, "Methodology / Architecture" (each layer keeps frozen AR
// weights theta_AR and adds LoRA diffusion weights theta_Delta of rank 128,
// alpha 256; drafting uses theta_AR + theta_Delta, verification theta_AR
// alone) and the paperglide reader, "The Uno Framework":
//
//   y_ar    = x W^T
//   T       = (alpha / r) x A^T
//   y_draft = y_ar + T Bm^T
//
// Two launches:
//  1. T: a split-K tcgen05 GEMM writes float32 partial products of x A^T to
//     the workspace; a small kernel sums the splits in index order, scales by
//     alpha/r and rounds to the operand type.
//  2. The dual GEMM streams W once. Per output tile, a TMA producer warp feeds
//     a multi-stage shared-memory ring; one thread issues tcgen05.mma into a
//     TMEM accumulator D0 = x W^T over all of d_in, then r/64 more K-blocks
//     of T Bm^T into a second accumulator D1; four epilogue warps read both
//     with tcgen05.ld and store y_ar = D0 and y_draft = D0 + D1.
// For M <= 256 the operands swap roles (W rows fill the 128-row MMA side and
// the few activation rows are the N side), so small-batch decode still runs
// at full tile height while it is bound by the stream of W.
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "uno.h"
#include "uno_device.cuh"
#include "uno_host.h"

namespace {

constexpr int kBM = 128;              // MMA M (rows of the A operand per tile)
constexpr int kRowBytes = 128;        // bytes of K per tile row and stage (one swizzle row)
constexpr int kGemmThreads = 192;     // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kSmSplitTarget = 148;   // CTAs the T product aims to fill

enum : unsigned { kFaultProducer = 1u, kFaultMma = 2u, kFaultEpilogue = 4u };

__device__ unsigned int g_fault_flags;

struct GemmParams {
  int kb_total;      // K-blocks of the main product over the whole K extent
  int kb_per_split;  // K-blocks handled by one split (== kb_total without split)
  int nkb_adapt;     // K-blocks of the adapter product (0: none)
  int M;             // output rows
  int ncols;         // output columns (d_out, or r for the T product)
  void* y_ar;        // dual mode, may be null
  void* y_draft;     // dual mode, may be null
  float* partial;    // partial mode: [split][M][ncols]
};

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
}

template <int BN>
__host__ __device__ constexpr int stages_for() {
  return BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
}

template <int BN, int STAGES>
__host__ __device__ constexpr int smem_bytes() {
  return STAGES * (kBM + BN) * kRowBytes + 1024 /*align*/ + 256 /*barriers*/;
}

__device__ __forceinline__ void set_fault(unsigned bit, volatile int* abort_flag) {
  atomicOr(&g_fault_flags, bit);
  *abort_flag = 1;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Store 32 consecutive columns of one output row (non-swapped tiles).
template <typename T>
__device__ __forceinline__ void store_row32(T* dst, const float* v, int valid_cols) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g * 8 < valid_cols) {
        uint4 w;
        w.x = pack_bf16x2(v[g * 8 + 0], v[g * 8 + 1]);
        w.y = pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]);
        w.z = pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]);
        w.w = pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]);
        *reinterpret_cast<uint4*>(dst + g * 8) = w;
      }
    }
  } else {
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (g * 4 < valid_cols)
        *reinterpret_cast<float4*>(dst + g * 4) =
            make_float4(v[g * 4], v[g * 4 + 1], v[g * 4 + 2], v[g * 4 + 3]);
    }
  }
}

template <typename T>
__device__ __forceinline__ void store_one(T* dst, float v) {
  if constexpr (sizeof(T) == 2) {
    *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
  } else {
    *dst = v;
  }
}

// ---------------------------------------------------------------------------
// The tile GEMM. D[a, b] = sum_k A_op[a, k] * B_op[b, k] for a 128-row tile of
// the A operand and a BN-row tile of the B operand, both K-major in global
// memory and loaded by TMA with 128-byte swizzling.
//   PARTIAL = false: dual mode (main product + optional adapter product).
//   PARTIAL = true : float32 partial products of one K split.
//   SWAP    = false: output row = A row, output column = B row.
//   SWAP    = true : output row = B row, output column = A row.
// ---------------------------------------------------------------------------
template <typename T, int BN, bool SWAP, bool PARTIAL>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmA2,
                const __grid_constant__ CUtensorMap tmB2, const GemmParams p) {
  constexpr int STAGES = stages_for<BN>();
  constexpr int kAbytes = kBM * kRowBytes;
  constexpr int kStage = (kBM + BN) * kRowBytes;
  constexpr bool kTf32 = sizeof(T) == 4;
  constexpr int kElemsPerRow = kRowBytes / static_cast<int>(sizeof(T));
  constexpr uint32_t kIdesc = sm100::instr_desc(kTf32, kBM, BN);
  constexpr int kD1 = pow2_at_least(BN);                     // column of the adapter accumulator
  constexpr uint32_t kTmemCols = PARTIAL ? pow2_at_least(BN) : 2 * pow2_at_least(BN);
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert(kTmemCols <= 512, "TMEM");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * kStage);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* accum_bar = empty_bar + STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum_bar + 1);
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a_row0 = blockIdx.x * kBM;
  const int b_row0 = blockIdx.y * BN;
  const int split = blockIdx.z;
  const int kb_begin = split * p.kb_per_split;
  const int nkb = min(p.kb_per_split, p.kb_total - kb_begin);
  const int nadapt = PARTIAL ? 0 : p.nkb_adapt;
  const int total_it = nkb + nadapt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full_bar[s], 1);
      sm100::mbar_init(&empty_bar[s], 1);
    }
    sm100::mbar_init(accum_bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    sm100::tma_prefetch_desc(&tmA);
    sm100::tma_prefetch_desc(&tmB);
    if (nadapt) {
      sm100::tma_prefetch_desc(&tmA2);
      sm100::tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 1) sm100::tmem_alloc(tmem_holder, kTmemCols);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer ----
      int issued = 0;
      for (int it = 0; it < total_it; ++it) {
        const int s = it % STAGES;
        if (it >= STAGES && !sm100::mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1)) {
          set_fault(kFaultProducer, &abort_flag);
          break;
        }
        if (abort_flag) break;
        uint8_t* sa = smem + s * kStage;
        uint8_t* sb = sa + kAbytes;
        sm100::mbar_arrive_expect_tx(&full_bar[s], kStage);
        if (it < nkb) {
          const int kx = (kb_begin + it) * kElemsPerRow;
          sm100::tma_load_2d(sa, &tmA, &full_bar[s], kx, a_row0);
          sm100::tma_load_2d(sb, &tmB, &full_bar[s], kx, b_row0);
        } else {
          const int kx = (it - nkb) * kElemsPerRow;
          sm100::tma_load_2d(sa, &tmA2, &full_bar[s], kx, a_row0);
          sm100::tma_load_2d(sb, &tmB2, &full_bar[s], kx, b_row0);
        }
        issued = it + 1;
      }
      // Every issued load must land before the CTA may exit: wait for the
      // latest phase of each stage that received one (at most STAGES).
      for (int it = (issued > STAGES ? issued - STAGES : 0); it < issued; ++it) {
        if (!sm100::mbar_wait(&full_bar[it % STAGES], (it / STAGES) & 1))
          set_fault(kFaultProducer, &abort_flag);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      for (int it = 0; it < total_it; ++it) {
        const int s = it % STAGES;
        if (!sm100::mbar_wait(&full_bar[s], (it / STAGES) & 1)) {
          set_fault(kFaultMma, &abort_flag);
          break;
        }
        if (abort_flag) break;
        sm100::tc_fence_after();
        const uint32_t sa = sm100::smem_addr(smem + s * kStage);
        const uint64_t da = sm100::smem_desc_k_sw128(sa);
        const uint64_t db = sm100::smem_desc_k_sw128(sa + kAbytes);
        const bool main = it < nkb;
        const int kb_local = main ? it : it - nkb;
        const uint32_t d = tmem + (main ? 0u : static_cast<uint32_t>(kD1));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // 32 bytes of K per instruction: 16 bf16 or 8 tf32 elements.
          sm100::mma<kTf32>(d, da + 2 * k, db + 2 * k, kIdesc, (kb_local > 0) || (k > 0));
        }
        sm100::mma_commit(&empty_bar[s]);
      }
      sm100::mma_commit(accum_bar);  // fires when every issued MMA has completed
    }
  } else {
    // ---- epilogue: warps 2..5, TMEM lane quarter = warp % 4 ----
    // tcgen05.ld is warp-collective: decide for the whole warp at once.
    const bool ok = __all_sync(0xFFFFFFFFu, sm100::mbar_wait(accum_bar, 0));
    if (!ok && lane == 0) set_fault(kFaultEpilogue, &abort_flag);
    sm100::tc_fence_after();
    if (__all_sync(0xFFFFFFFFu, ok && !abort_flag)) {
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;
      const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      const int arow = a_row0 + r;
      const bool with_adapter = !PARTIAL && nadapt > 0;
      for (int c = 0; c < BN; c += 32) {
        uint32_t v0[32], v1[32];
        sm100::tmem_ld_32x32b_x32(tq + c, v0);
        if (with_adapter) sm100::tmem_ld_32x32b_x32(tq + kD1 + c, v1);
        sm100::tmem_ld_wait();
        float f0[32], f1[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          f0[e] = __uint_as_float(v0[e]);
          f1[e] = with_adapter ? f0[e] + __uint_as_float(v1[e]) : f0[e];
        }
        const int brow = b_row0 + c;  // first B row of this 32-column slice
        if constexpr (PARTIAL) {
          float* base = p.partial + static_cast<size_t>(split) * p.M * p.ncols;
          if constexpr (!SWAP) {
            // 32 consecutive columns of one row: 16-byte stores (ncols % 4 == 0)
            if (arow < p.M) {
              float* dst = base + static_cast<size_t>(arow) * p.ncols + brow;
#pragma unroll
              for (int g = 0; g < 8; ++g)
                if (brow + g * 4 < p.ncols)
                  *reinterpret_cast<float4*>(dst + g * 4) =
                      make_float4(f0[g * 4], f0[g * 4 + 1], f0[g * 4 + 2], f0[g * 4 + 3]);
            }
          } else {
            if (arow < p.ncols) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (brow + e < p.M) base[static_cast<size_t>(brow + e) * p.ncols + arow] = f0[e];
            }
          }
        } else {
          T* ya = static_cast<T*>(p.y_ar);
          T* yd = static_cast<T*>(p.y_draft);
          if constexpr (!SWAP) {
            if (arow < p.M) {
              const size_t off = static_cast<size_t>(arow) * p.ncols + brow;
              const int valid = p.ncols - brow;
              if (valid > 0) {
                if (ya) store_row32<T>(ya + off, f0, valid);
                if (yd) store_row32<T>(yd + off, f1, valid);
              }
            }
          } else {
            if (arow < p.ncols) {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                if (brow + e < p.M) {
                  const size_t off = static_cast<size_t>(brow + e) * p.ncols + arow;
                  if (ya) store_one<T>(ya + off, f0[e]);
                  if (yd) store_one<T>(yd + off, f1[e]);
                }
              }
            }
          }
        }
      }
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// The dual GEMM, persistent. Each CTA takes tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ... (the 128-row A tile index varies fastest, so
// neighbouring CTAs share a B tile in L2). TMEM holds two BN-column fp32
// accumulators, used by alternate tiles. Per tile the MMA thread accumulates
// x W^T over all K-blocks into the tile's accumulator; the epilogue drains it
// as y_ar and says so; the adapter product T Bm^T (two 64-wide K-blocks for
// r = 128) is then accumulated into the same accumulator, which the epilogue
// drains again as y_draft. The adapter K-blocks of tile i ride in the operand
// ring after the first kInsert K-blocks of tile i + 1, so the tensor pipe works
// on the next tile while the epilogue drains y_ar.
// ---------------------------------------------------------------------------
constexpr int kInsert = 6;

template <typename T, int BN, bool SWAP>
__global__ void __launch_bounds__(kGemmThreads, 1)
    dual_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                const GemmParams p, int rowsA, int rowsB) {
  constexpr int STAGES = stages_for<BN>();
  constexpr int kAbytes = kBM * kRowBytes;
  constexpr int kStage = (kBM + BN) * kRowBytes;
  constexpr bool kTf32 = sizeof(T) == 4;
  constexpr int kElemsPerRow = kRowBytes / static_cast<int>(sizeof(T));
  constexpr uint32_t kIdesc = sm100::instr_desc(kTf32, kBM, BN);
  constexpr int kAcc = pow2_at_least(BN);  // columns of one accumulator buffer
  constexpr uint32_t kTmemCols = 2 * kAcc;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256 && kTmemCols <= 512, "BN");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * kStage);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* acc_full = empty_bar + STAGES;   // [2] main product done
  uint64_t* ar_read = acc_full + 2;          // [2] epilogue drained y_ar
  uint64_t* draft_full = ar_read + 2;        // [2] adapter product done
  uint64_t* acc_empty = draft_full + 2;      // [2] epilogue drained the buffer
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_a = (rowsA + kBM - 1) / kBM;
  const int tiles_b = (rowsB + BN - 1) / BN;
  const int ntiles = tiles_a * tiles_b;
  const int nmine = (ntiles > static_cast<int>(blockIdx.x))
                        ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                        : 0;
  const int nkb = p.kb_total;
  const bool adapter = p.nkb_adapt > 0;
  const int nad = adapter ? p.nkb_adapt : 0;
  const int ins = min(kInsert, nkb);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full_bar[s], 1);
      sm100::mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(&acc_full[b], 1);
      sm100::mbar_init(&ar_read[b], 4);
      sm100::mbar_init(&draft_full[b], 1);
      sm100::mbar_init(&acc_empty[b], 4);
    }
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    sm100::tma_prefetch_desc(&tmA);
    sm100::tma_prefetch_desc(&tmB);
    if (adapter) {
      sm100::tma_prefetch_desc(&tmA2);
      sm100::tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 1) sm100::tmem_alloc(tmem_holder, kTmemCols);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // The operand stream of this CTA, in ring order: for local tile i, its main
  // K-blocks 0..ins-1, then the adapter K-blocks of tile i-1, then its main
  // K-blocks ins..nkb-1; after the last tile, that tile's adapter K-blocks.
  // Item q of local tile i (0 <= q < nkb + nad, nad only for i >= 1) maps to:
  //   q < ins            -> main block q of tile i
  //   ins <= q < ins+nad -> adapter block q-ins of tile i-1
  //   otherwise          -> main block q-nad of tile i
  auto tile_coords = [&](int li, int& a0, int& b0) {
    const int t = static_cast<int>(blockIdx.x) + li * static_cast<int>(gridDim.x);
    a0 = (t % tiles_a) * kBM;
    b0 = (t / tiles_a) * BN;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer ----
      int it = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* ma, const CUtensorMap* mb, int kx, int a0, int b0) {
        const int s = it % STAGES;
        if (it >= STAGES && !sm100::mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1)) {
          set_fault(kFaultProducer, &abort_flag);
          ok = false;
          return;
        }
        if (abort_flag) {
          ok = false;
          return;
        }
        uint8_t* sa = smem + s * kStage;
        sm100::mbar_arrive_expect_tx(&full_bar[s], kStage);
        sm100::tma_load_2d(sa, ma, &full_bar[s], kx, a0);
        sm100::tma_load_2d(sa + kAbytes, mb, &full_bar[s], kx, b0);
        ++it;
      };
      for (int li = 0; li <= nmine && ok; ++li) {
        int a0 = 0, b0 = 0, pa0 = 0, pb0 = 0;
        if (li < nmine) tile_coords(li, a0, b0);
        if (li > 0) tile_coords(li - 1, pa0, pb0);
        const int nmain = (li < nmine) ? nkb : 0;
        const int nadp = (li > 0) ? nad : 0;
        const int items = nmain + nadp;
        for (int q = 0; q < items && ok; ++q) {
          const int qa = q - min(ins, nmain);
          if (q < min(ins, nmain)) {
            load(&tmA, &tmB, q * kElemsPerRow, a0, b0);
          } else if (qa < nadp) {
            load(&tmA2, &tmB2, qa * kElemsPerRow, pa0, pb0);
          } else {
            load(&tmA, &tmB, (q - nadp) * kElemsPerRow, a0, b0);
          }
        }
      }
      for (int k = (it > STAGES ? it - STAGES : 0); k < it; ++k)
        if (!sm100::mbar_wait(&full_bar[k % STAGES], (k / STAGES) & 1))
          set_fault(kFaultProducer, &abort_flag);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      int it = 0;
      bool ok = true;
      auto consume = [&](uint32_t d, bool accumulate_first) {
        const int s = it % STAGES;
        if (!sm100::mbar_wait(&full_bar[s], (it / STAGES) & 1)) {
          set_fault(kFaultMma, &abort_flag);
          ok = false;
          return;
        }
        sm100::tc_fence_after();
        const uint32_t sa = sm100::smem_addr(smem + s * kStage);
        const uint64_t da = sm100::smem_desc_k_sw128(sa);
        const uint64_t db = sm100::smem_desc_k_sw128(sa + kAbytes);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          sm100::mma<kTf32>(d, da + 2 * k, db + 2 * k, kIdesc, accumulate_first || (k > 0));
        sm100::mma_commit(&empty_bar[s]);
        ++it;
      };
      for (int li = 0; li <= nmine && ok; ++li) {
        const int buf = li & 1, pbuf = (li - 1) & 1;
        const uint32_t d = tmem + static_cast<uint32_t>(buf * kAcc);
        const uint32_t pd = tmem + static_cast<uint32_t>(pbuf * kAcc);
        const int nmain = (li < nmine) ? nkb : 0;
        const int nadp = (li > 0) ? nad : 0;
        const int items = nmain + nadp;
        if (nmain && li >= 2 &&
            !sm100::mbar_wait(&acc_empty[buf], ((li >> 1) - 1) & 1)) {  // buffer drained
          set_fault(kFaultMma, &abort_flag);
          break;
        }
        sm100::tc_fence_after();
        for (int q = 0; q < items && ok; ++q) {
          const int qa = q - min(ins, nmain);
          if (q < min(ins, nmain)) {
            consume(d, q > 0);
            if (q == nmain - 1) sm100::mma_commit(&acc_full[buf]);
          } else if (qa < nadp) {
            if (qa == 0) {
              if (!sm100::mbar_wait(&ar_read[pbuf], ((li - 1) >> 1) & 1)) {
                set_fault(kFaultMma, &abort_flag);
                ok = false;
                break;
              }
              sm100::tc_fence_after();
            }
            consume(pd, true);  // adds T Bm^T onto y_ar of the previous tile
            if (qa == nadp - 1) sm100::mma_commit(&draft_full[pbuf]);
          } else {
            const int kb = q - nadp;
            consume(d, kb > 0);
            if (kb == nmain - 1) sm100::mma_commit(&acc_full[buf]);
          }
        }
      }
    }
  } else {
    // ---- epilogue: warps 2..5, TMEM lane quarter = warp % 4 ----
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    T* ya = static_cast<T*>(p.y_ar);
    T* yd = static_cast<T*>(p.y_draft);
    auto drain = [&](uint32_t acc, int a0, int b0, T* y) {
      if (!y) return;  // output not requested: nothing to read
      const uint32_t tq = acc + (static_cast<uint32_t>(quarter * 32) << 16);
      const int arow = a0 + r;
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        sm100::tmem_ld_32x32b_x32(tq + c, v);
        sm100::tmem_ld_wait();
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
        const int brow = b0 + c;
        if constexpr (!SWAP) {
          if (arow < p.M && brow < p.ncols)
            store_row32<T>(y + static_cast<size_t>(arow) * p.ncols + brow, f, p.ncols - brow);
        } else {
          if (arow < p.ncols) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (brow + e < p.M) store_one<T>(y + static_cast<size_t>(brow + e) * p.ncols + arow, f[e]);
          }
        }
      }
    };
    for (int li = 0; li < nmine; ++li) {
      const int buf = li & 1;
      const uint32_t acc = tmem + static_cast<uint32_t>(buf * kAcc);
      int a0, b0;
      tile_coords(li, a0, b0);
      const bool got = __all_sync(0xFFFFFFFFu, sm100::mbar_wait(&acc_full[buf], (li >> 1) & 1));
      if (!got || abort_flag) {
        if (lane == 0) set_fault(kFaultEpilogue, &abort_flag);
        break;
      }
      sm100::tc_fence_after();
      drain(acc, a0, b0, ya);
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(adapter ? &ar_read[buf] : &acc_empty[buf]);
      if (!adapter) continue;
      const bool got2 = __all_sync(0xFFFFFFFFu, sm100::mbar_wait(&draft_full[buf], (li >> 1) & 1));
      if (!got2 || abort_flag) {
        if (lane == 0) set_fault(kFaultEpilogue, &abort_flag);
        break;
      }
      sm100::tc_fence_after();
      drain(acc, a0, b0, yd);
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&acc_empty[buf]);
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// T = scale * sum_s partial[s]  (splits summed in index order), rounded to T.
// Four consecutive elements per thread (count is a multiple of 4).
template <typename T>
__global__ void reduce_t_kernel(const float* __restrict__ partial, int splits, size_t count,
                                float scale, T* __restrict__ out) {
  const size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i >= count) return;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < splits; ++k) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(partial + static_cast<size_t>(k) * count + i));
    s.x += v.x;
    s.y += v.y;
    s.z += v.z;
    s.w += v.w;
  }
  s.x *= scale;
  s.y *= scale;
  s.z *= scale;
  s.w *= scale;
  if constexpr (sizeof(T) == 2) {
    uint2 w;
    w.x = pack_bf16x2(s.x, s.y);
    w.y = pack_bf16x2(s.z, s.w);
    *reinterpret_cast<uint2*>(out + i) = w;
  } else {
    *reinterpret_cast<float4*>(out + i) = s;
  }
}

// ---- host side ------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D K-major map: inner dimension K (elements), outer dimension rows; box of
// 128 bytes of K by box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* map, const void* ptr, int dtype, int k_elems, int rows, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  const size_t esize = (dtype == UNO_BF16) ? 2 : 4;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k_elems), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k_elems) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kRowBytes / esize),
                       static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map,
                         dtype == UNO_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                         2, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename T, int BN, bool SWAP, bool PARTIAL>
int launch_gemm(dim3 grid, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                const CUtensorMap& b2, const GemmParams& p, cudaStream_t st) {
  constexpr int bytes = smem_bytes<BN, stages_for<BN>()>();
  auto kern = gemm_kernel<T, BN, SWAP, PARTIAL>;
  // The shared-memory opt-in is per device; remember which devices have it.
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return UNO_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (!bit || !(attr_done.load(std::memory_order_relaxed) & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return UNO_ERR_CUDA;
    attr_done.fetch_or(bit, std::memory_order_relaxed);
  }
  kern<<<grid, kGemmThreads, bytes, st>>>(a, b, a2, b2, p);
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

int sm_count_dual() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

template <typename T, int BN, bool SWAP>
int launch_dual(int rowsA, int rowsB, const CUtensorMap& a, const CUtensorMap& b,
                const CUtensorMap& a2, const CUtensorMap& b2, const GemmParams& p,
                cudaStream_t st) {
  constexpr int bytes = smem_bytes<BN, stages_for<BN>()>();
  auto kern = dual_kernel<T, BN, SWAP>;
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return UNO_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (!bit || !(attr_done.load(std::memory_order_relaxed) & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return UNO_ERR_CUDA;
    attr_done.fetch_or(bit, std::memory_order_relaxed);
  }
  const long long tiles =
      static_cast<long long>((rowsA + kBM - 1) / kBM) * ((rowsB + BN - 1) / BN);
  long long grid = sm_count_dual();
  if (grid > tiles) grid = tiles;
  kern<<<static_cast<unsigned>(grid), kGemmThreads, bytes, st>>>(a, b, a2, b2, p, rowsA, rowsB);
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

template <typename T, bool SWAP>
int launch_dual_bn(int bn, int rowsA, int rowsB, const CUtensorMap& a, const CUtensorMap& b,
                   const CUtensorMap& a2, const CUtensorMap& b2, const GemmParams& p,
                   cudaStream_t st) {
  switch (bn) {
    case 32: return launch_dual<T, 32, SWAP>(rowsA, rowsB, a, b, a2, b2, p, st);
    case 64: return launch_dual<T, 64, SWAP>(rowsA, rowsB, a, b, a2, b2, p, st);
    case 128: return launch_dual<T, 128, SWAP>(rowsA, rowsB, a, b, a2, b2, p, st);
    default: return launch_dual<T, 256, SWAP>(rowsA, rowsB, a, b, a2, b2, p, st);
  }
}

// Dispatch over the B-tile height (32, 64, 128 or 256 rows).
template <typename T, bool SWAP, bool PARTIAL>
int launch_bn(int bn, dim3 grid, const CUtensorMap& a, const CUtensorMap& b,
              const CUtensorMap& a2, const CUtensorMap& b2, const GemmParams& p,
              cudaStream_t st) {
  switch (bn) {
    case 32: return launch_gemm<T, 32, SWAP, PARTIAL>(grid, a, b, a2, b2, p, st);
    case 64: return launch_gemm<T, 64, SWAP, PARTIAL>(grid, a, b, a2, b2, p, st);
    case 128: return launch_gemm<T, 128, SWAP, PARTIAL>(grid, a, b, a2, b2, p, st);
    default: return launch_gemm<T, 256, SWAP, PARTIAL>(grid, a, b, a2, b2, p, st);
  }
}

int bn_for(int rows) { return rows <= 32 ? 32 : rows <= 64 ? 64 : rows <= 128 ? 128 : 256; }

struct Plan {
  bool swap;
  int esize;
  int kb_main;   // K-blocks over d_in
  int kb_adapt;  // K-blocks over r
  // T product
  int t_bn, t_grid_x, t_splits, t_per;
  size_t t_bytes, partial_bytes;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

bool dual_sizes_ok(int M, int d_in, int d_out, int r, int dtype) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return false;
  const int q = (dtype == UNO_BF16) ? 8 : 4;
  return M >= 0 && M <= (1 << 24) && d_in >= 1 && d_out >= 1 && r >= 1 && r <= 256 &&
         d_in % q == 0 && d_out % q == 0 && r % q == 0 && d_in <= (1 << 24) &&
         d_out <= (1 << 24);
}

Plan make_plan(int M, int d_in, int r, int dtype) {
  Plan pl{};
  pl.esize = (dtype == UNO_BF16) ? 2 : 4;
  pl.swap = M <= 256;
  pl.kb_main = (d_in * pl.esize + kRowBytes - 1) / kRowBytes;
  pl.kb_adapt = (r * pl.esize + kRowBytes - 1) / kRowBytes;
  if (pl.swap) {  // A op = A (r rows), B op = x (M rows)
    pl.t_bn = bn_for(M);
    pl.t_grid_x = (r + kBM - 1) / kBM;
  } else {        // A op = x (M rows), B op = A (r rows)
    pl.t_bn = bn_for(r);
    pl.t_grid_x = (M + kBM - 1) / kBM;
  }
  int splits = (kSmSplitTarget + pl.t_grid_x - 1) / pl.t_grid_x;
  if (splits > pl.kb_main) splits = pl.kb_main;
  if (splits < 1) splits = 1;
  pl.t_per = (pl.kb_main + splits - 1) / splits;
  pl.t_splits = (pl.kb_main + pl.t_per - 1) / pl.t_per;
  pl.t_bytes = align256(static_cast<size_t>(M) * r * pl.esize);
  pl.partial_bytes = align256(static_cast<size_t>(pl.t_splits) * M * r * sizeof(float));
  return pl;
}

template <typename T>
int run_dualpath(const void* x, const void* W, const void* A, const void* Bm, float scale,
                 void* y_ar, void* y_draft, int M, int d_in, int d_out, int r, int dtype,
                 void* workspace, cudaStream_t st) {
  const Plan pl = make_plan(M, d_in, r, dtype);
  const bool adapter = (y_draft != nullptr);
  T* Tbuf = static_cast<T*>(workspace);
  float* partial = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.t_bytes);
  CUtensorMap mx, mW, mBm, mT;
  const int xrows_box = pl.swap ? bn_for(M) : kBM;
  int st_code = UNO_OK;

  // 1. T = scale * x A^T (only when the draft output is wanted).
  if (adapter) {
    CUtensorMap ta, tb;
    bool ok;
    if (pl.swap) {
      ok = make_map(&ta, A, dtype, d_in, r, kBM) && make_map(&tb, x, dtype, d_in, M, pl.t_bn);
    } else {
      ok = make_map(&ta, x, dtype, d_in, M, kBM) && make_map(&tb, A, dtype, d_in, r, pl.t_bn);
    }
    if (!ok) return UNO_ERR_CUDA;
    GemmParams gp{};
    gp.kb_total = pl.kb_main;
    gp.kb_per_split = pl.t_per;
    gp.nkb_adapt = 0;
    gp.M = M;
    gp.ncols = r;
    gp.partial = partial;
    const dim3 grid(pl.t_grid_x, 1, pl.t_splits);
    st_code = pl.swap ? launch_bn<T, true, true>(pl.t_bn, grid, ta, tb, ta, tb, gp, st)
                      : launch_bn<T, false, true>(pl.t_bn, grid, ta, tb, ta, tb, gp, st);
    if (st_code != UNO_OK) return st_code;
    const size_t count = static_cast<size_t>(M) * r;
    reduce_t_kernel<T><<<static_cast<unsigned>((count / 4 + 255) / 256), 256, 0, st>>>(
        partial, pl.t_splits, count, scale, Tbuf);
    if (cudaGetLastError() != cudaSuccess) return UNO_ERR_CUDA;
  }

  // 2. dual GEMM over W.
  GemmParams gp{};
  gp.kb_total = pl.kb_main;
  gp.kb_per_split = pl.kb_main;
  gp.nkb_adapt = adapter ? pl.kb_adapt : 0;
  gp.M = M;
  gp.ncols = d_out;
  gp.y_ar = y_ar;
  gp.y_draft = y_draft;
  if (pl.swap) {
    const int bn = bn_for(M);
    bool ok = make_map(&mW, W, dtype, d_in, d_out, kBM) && make_map(&mx, x, dtype, d_in, M, bn);
    if (adapter) ok = ok && make_map(&mBm, Bm, dtype, r, d_out, kBM) &&
                      make_map(&mT, Tbuf, dtype, r, M, bn);
    if (!ok) return UNO_ERR_CUDA;
    return launch_dual_bn<T, true>(bn, d_out, M, mW, mx, adapter ? mBm : mW, adapter ? mT : mx,
                                   gp, st);
  }
  bool ok = make_map(&mx, x, dtype, d_in, M, xrows_box) && make_map(&mW, W, dtype, d_in, d_out, 256);
  if (adapter) ok = ok && make_map(&mT, Tbuf, dtype, r, M, kBM) &&
                    make_map(&mBm, Bm, dtype, r, d_out, 256);
  if (!ok) return UNO_ERR_CUDA;
  return launch_dual<T, 256, false>(M, d_out, mx, mW, adapter ? mT : mx, adapter ? mBm : mW, gp,
                                    st);
}

}  // namespace

extern "C" size_t uno_dualpath_workspace_bytes(int M, int d_in, int d_out, int r, int dtype) {
  if (!dual_sizes_ok(M, d_in, d_out, r, dtype)) return 0;
  const Plan pl = make_plan(M, d_in, r, dtype);
  return pl.t_bytes + pl.partial_bytes;
}

extern "C" int uno_dualpath_linear(const void* x, const void* W, const void* A, const void* Bm,
                                   float scale, void* y_ar, void* y_draft, int M, int d_in,
                                   int d_out, int r, int dtype, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (!dual_sizes_ok(M, d_in, d_out, r, dtype)) return UNO_ERR_SIZE;
  if (M == 0) return UNO_OK;
  if (!x || !W || (!y_ar && !y_draft)) return UNO_ERR_NULL;
  if (y_draft && (!A || !Bm)) return UNO_ERR_NULL;
  if (!workspace) return UNO_ERR_WORKSPACE;
  for (const void* ptr : {x, W, A, Bm, static_cast<const void*>(y_ar),
                          static_cast<const void*>(y_draft), static_cast<const void*>(workspace)})
    if (!uno_host::aligned(ptr, 16)) return UNO_ERR_ALIGN;
  if (workspace_bytes < uno_dualpath_workspace_bytes(M, d_in, d_out, r, dtype))
    return UNO_ERR_WORKSPACE;
  const int dev = uno_host::check_device();
  if (dev != UNO_OK) return dev;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == UNO_BF16)
    return run_dualpath<uint16_t>(x, W, A, Bm, scale, y_ar, y_draft, M, d_in, d_out, r, dtype,
                                  workspace, st);
  return run_dualpath<float>(x, W, A, Bm, scale, y_ar, y_draft, M, d_in, d_out, r, dtype,
                             workspace, st);
}

extern "C" int uno_device_fault_flags(int clear, unsigned int* flags) {
  if (!flags) return UNO_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return UNO_ERR_CUDA;
  if (cudaMemcpyFromSymbol(flags, g_fault_flags, sizeof(unsigned)) != cudaSuccess)
    return UNO_ERR_CUDA;
  if (clear) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_fault_flags, &zero, sizeof(unsigned)) != cudaSuccess)
      return UNO_ERR_CUDA;
  }
  return UNO_OK;
}
