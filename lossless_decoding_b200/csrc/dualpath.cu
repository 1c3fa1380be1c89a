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
// One persistent launch, one CTA per SM. Its tiles, in schedule order:
//  * T tiles: T = scale * x A^T for one 128-row block (or, with swapped
//    operands, one 128-column block of T), rounded to the operand type and
//    stored to the workspace; a release store of the call's epoch to the
//    tile's flag announces it.
//  * main tiles: a 128 x BN tile of x W^T over all of d_in, accumulated in
//    TMEM; the epilogue drains it as y_ar, then the adapter product T Bm^T is
//    accumulated onto the same accumulator and drained as y_draft.
// Warp roles: two producer warps issue TMA loads into a multi-stage
// shared-memory ring (a thread with copies in flight stalls at its next
// mbarrier operation until they land, so one producer would keep a single
// stage in flight); two issuer threads alternate K-blocks of tcgen05.mma (a thread that
// has committed stalls the same way until its MMAs finish); four epilogue
// warps drain TMEM with tcgen05.ld. Two accumulator buffers alternate between
// tiles, and the adapter K-blocks of a tile ride in the ring a few K-blocks
// into the next tile, so the tensor pipe keeps working while the epilogue
// drains.
//
// A main tile's producer reads T only after the T tile's flag holds the
// call's epoch (acquire, then an async-proxy fence before the TMA load). T
// tiles come first in the schedule, so the CTAs computing them started no
// later than any CTA that waits for them; the wait is bounded and reports
// through the fault flags.
//
// For M <= 256 the operands swap roles (W rows fill the 128-row MMA side, the
// few activation rows are the N side), so small-batch decode still runs at full
// tile height while it is bound by the stream of W.
#include <algorithm>
#include <atomic>
#include <chrono>
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

constexpr int kBM = 128;           // MMA M (rows of the A operand per tile)
constexpr int kRowBytes = 128;     // bytes of K per tile row and stage (one swizzle row)
// Warp roles: 0-3 epilogue (TMEM lane quarter = warp), 4-5 MMA issuers (4
// owns TMEM), kFirstProducer.. TMA producers.
constexpr int kMmaWarp0 = 4;
constexpr int kFirstProducer = 6;
constexpr int kProducers = 2;
constexpr int kGemmThreads = (kFirstProducer + kProducers) * 32;
constexpr int kInsert = 6;         // main K-blocks of the next tile before an adapter
constexpr int kPrefetch = 8;       // K-blocks of L2 prefetch ahead of the weight loads
constexpr int kMaxSplit = 4;       // K-pieces of a split tile, at most
constexpr uint64_t kWaitNs = 1000000000ull;  // default limit of every bounded wait

enum : unsigned { kFaultProducer = 1u, kFaultMma = 2u, kFaultEpilogue = 4u };

__device__ unsigned int g_fault_flags;

constexpr int kMaxGroups = 4;  // projections of one launch (they share x)

// One projection of a (grouped) launch.
struct GroupArgs {
  int ncols;          // its d_out
  int tiles_a;        // tiles along the A operand's rows
  int tiles;          // its main tiles
  int tile0;          // index of its first main tile among all main tiles
  float scale;        // alpha / r
  void* y_ar;         // may be null
  void* y_draft;      // may be null (then for every projection)
  void* t_buf;        // T [M][r]
  uint32_t* t_flags;  // [nT]
  float2* stats_ar;     // [M][stats_tiles] row softmax partials of y_ar (may be null)
  float2* stats_draft;  // [M][stats_tiles] the same for y_draft (may be null)
  int stats_tiles;      // column tiles of the projection: ceil(d_out / BN)
};

struct GemmParams {
  int kb_total;       // K-blocks over d_in
  int nkb_adapt;      // K-blocks over r (0: no adapter, no T tiles)
  int M;              // output rows
  int nT;             // T tiles per projection
  int ngroups;        // projections in this launch
  int r;              // adapter rank
  uint32_t idesc_t;   // instruction descriptor of the T tiles
  int t_brows;        // rows of the B box of a T-tile item (per CTA)
  uint32_t epoch;     // value a T tile's flag takes once T is stored
  uint32_t t_wait_epoch;  // value a producer waits for on a T flag (== epoch, except
                          // under the failure-path test hook: a value no tile writes)
  uint64_t wait_ns;   // limit of every bounded wait (1 s; shorter under the test hook)
  int main_tiles;     // main tiles over all projections
  // The last, partial round of main tiles may be split along K so that it
  // fills the GPU: units [split_start, split_start + n_split * split_k) are
  // piece (j % split_k) of main tile (split_start - nT * ngroups + j / split_k).
  // Piece 0 adds the fp32 partials of the other pieces (part_buf slots,
  // published through part_flags) before its epilogue.
  int split_start;    // first split unit (== total units when nothing is split)
  int split_k;        // pieces per split tile (1: no split)
  float* part_buf;    // [n_split][split_k - 1][CTAs per tile][128][BN] fp32
  uint32_t* part_flags;  // [n_split][split_k - 1]
  size_t part_capacity;  // bytes available at part_buf (host side: decides the split)
  const uint8_t* gate;   // [M] per-row adapter gate (0: AR only), or null (all on)
  GroupArgs g[kMaxGroups];
};

// Tensor maps of a launch: x is shared; the rest is per projection.
struct DualMaps {
  CUtensorMap x;               // activations [M][d_in]
  CUtensorMap w[kMaxGroups];   // W [d_out][d_in]
  CUtensorMap bm[kMaxGroups];  // Bm [d_out][r]
  CUtensorMap t[kMaxGroups];   // T [M][r] (workspace)
  CUtensorMap l[kMaxGroups];   // LoRA A [r][d_in]
  CUtensorMap ya[kMaxGroups];  // y_ar store map (TMA-store epilogue)
  CUtensorMap yd[kMaxGroups];  // y_draft store map
};

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
}

// Bytes of one K-block per CTA: a 128-row box of the A side and the B rows
// this CTA holds (all BN, or half of them with the CTA pair).
template <int BN, bool PAIR>
__host__ __device__ constexpr int kblock_bytes() {
  return (kBM + (PAIR ? BN / 2 : BN)) * kRowBytes;
}

// K-blocks per ring item. Every item costs its MMA issuer a wait on the
// item's data, a hand-over and a commit, and its producer a wait for the
// stage; the CTA pair moves two K-blocks per item (a 64 KB stage per CTA) so
// that these costs are paid once per 1024 cycles of tensor work, not 512.
template <bool PAIR>
__host__ __device__ constexpr int kblocks_per_item() {
  return PAIR ? 2 : 1;
}

template <int BN, bool PAIR>
__host__ __device__ constexpr int stage_bytes() {
  return kblocks_per_item<PAIR>() * kblock_bytes<BN, PAIR>();
}

template <int BN, bool PAIR>
__host__ __device__ constexpr int stages_for() {
  return PAIR ? 3 : (BN >= 256 ? 4 : (BN >= 128 ? 6 : 8));
}

// Barriers after the ring: full and empty per stage, 8 per-buffer barriers,
// t_stored, mma_done[2]; then the TMEM address and the issuers' hand-over word.
template <int BN, bool PAIR>
__host__ __device__ constexpr int barrier_bytes() {
  return (2 * stages_for<BN, PAIR>() + 8 + 1 + 2) * 8 + 4 + 4;
}

// One CTA's running row statistics in the swapped layout: per epilogue warp,
// y_ar and y_draft, BN rows of (m, z); then per epilogue warp a 32 x 33 float
// scratch for the transpose of a 32-row chunk.
template <int BN, bool PAIR>
__host__ __device__ constexpr int swap_stat_bytes() {
  return PAIR ? 0 : 4 * 2 * BN * 8 + 4 * 32 * 33 * 4;  // + the warps' transpose scratch
}

template <int BN, bool PAIR>
__host__ __device__ constexpr int smem_bytes() {
  static_assert(barrier_bytes<BN, PAIR>() <= 256, "barrier region");
  return stages_for<BN, PAIR>() * stage_bytes<BN, PAIR>() + 1024 /*align*/ + 256 /*barriers*/ +
         swap_stat_bytes<BN, PAIR>();
}
static_assert(smem_bytes<256, false>() <= 232448 && smem_bytes<128, false>() <= 232448 &&
                  smem_bytes<64, false>() <= 232448 && smem_bytes<32, false>() <= 232448 &&
                  smem_bytes<256, true>() <= 232448,
              "dynamic shared memory per CTA (227 KB)");

__device__ __forceinline__ void set_fault(unsigned bit, volatile int* abort_flag) {
  atomicOr(&g_fault_flags, bit);
  *abort_flag = 1;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Store 32 consecutive columns of one output row (valid_cols of them exist).
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

// Softmax statistics of one output row over a tile's columns, as the
// verifier merges them: m = the largest stored value times log2(e), z = the
// sum of 2^(value log2 e - m), over the values as stored (bfloat16-rounded
// for bfloat16 outputs). The reference m moves up only when a larger value
// arrives.
struct RowStats {
  float m, z;
  __device__ __forceinline__ void init() {
    m = -INFINITY;
    z = 0.f;
  }
  __device__ __forceinline__ void add(const float* v, int n) {  // the first n of 32 values
    constexpr float kL2e = 1.4426950408889634f;
    float mk = -INFINITY;
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (e < n) mk = fmaxf(mk, v[e]);
    mk *= kL2e;
    if (mk > m) {
      z *= uno::ex2(m - mk);
      m = mk;
    }
    if (m > -INFINITY) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (e < n) s += uno::ex2(fmaf(v[e], kL2e, -m));
      z += s;
    }
  }
};

// The value a store of v into T keeps.
template <typename T>
__device__ __forceinline__ float stored_value(float v) {
  if constexpr (sizeof(T) == 2) return __uint_as_float(pack_bf16x2(v, 0.f) << 16);
  else return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_release_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(sm100::smem_addr(p)), "r"(v)
               : "memory");
}

__device__ __forceinline__ int ld_acquire_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];"
               : "=r"(v)
               : "r"(sm100::smem_addr(p))
               : "memory");
  return v;
}

// Bounded wait until the other MMA issuer has handed over ring item `it`.
__device__ bool wait_order(const int* order, int it, volatile int* abort_flag, uint64_t limit_ns) {
  if (ld_acquire_shared(order) == it) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  for (uint32_t k = 1;; ++k) {
    if (ld_acquire_shared(order) == it) return true;
    if ((k & 255u) == 0 && (*abort_flag || sm100::globaltimer_ns() - t0 > limit_ns)) return false;
  }
}

// ---- two-SM (CTA pair) forms ----
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(sm100::smem_addr(p)), "r"(rank));
  return r;
}

// Every thread of both CTAs arrives (threads need not be converged).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void arrive_at(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr)
               : "memory");
}

// Bounded wait with cluster-scope acquire (barriers that a peer CTA or the
// pair's tensor core arrives on).
__device__ bool wait_cl(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = sm100::globaltimer_ns();
  for (uint32_t k = 0;; ++k) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(sm100::smem_addr(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((k & 255u) == 255u && sm100::globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// TMA load whose completion is counted on the mbarrier of the pair's leader.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(sm100::smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}

template <bool kTf32>
__device__ __forceinline__ void mma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         bool accumulate) {
  if constexpr (kTf32) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
        : "memory");
  }
}

// Arrive on `bar` (same offset) in both CTAs of the pair once the issuing
// thread's MMAs have completed.
__device__ __forceinline__ void commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(sm100::smem_addr(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

// Bounded wait until *flag == epoch.
__device__ bool wait_flag(const uint32_t* flag, uint32_t epoch, uint64_t limit_ns) {
  if (ld_acquire_u32(flag) == epoch) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire_u32(flag) == epoch) return true;
    if (sm100::globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// ---------------------------------------------------------------------------
// The kernel. Main operands: x and W (unswapped: x is the A side; swapped: W
// is). Adapter operands: T and Bm (unswapped: T on the A side; swapped: Bm).
// T tiles: x and the LoRA down weight A (unswapped: A on the B side, swapped:
// on the A side). Every projection of a grouped launch has its own W, Bm, T,
// A and outputs; x is shared.
// ---------------------------------------------------------------------------
template <typename T, int BN, bool SWAP, bool PAIR>
__global__ void __launch_bounds__(kGemmThreads, 1)
    dual_kernel(const __grid_constant__ DualMaps m, const __grid_constant__ GemmParams p) {
  static_assert(!(PAIR && SWAP), "the CTA pair serves the unswapped layout");
  constexpr int STAGES = stages_for<BN, PAIR>();
  constexpr int kAbytes = kBM * kRowBytes;
  constexpr int kBrows = PAIR ? BN / 2 : BN;   // rows of W (B side) per CTA and K-block
  constexpr int KBI = kblocks_per_item<PAIR>();  // K-blocks per ring item
  constexpr int kKb = kblock_bytes<BN, PAIR>();   // bytes of one K-block in a stage
  constexpr int kStage = stage_bytes<BN, PAIR>();
  constexpr int kRows = PAIR ? 2 * kBM : kBM;  // output rows of a tile (both CTAs)
  constexpr bool kTf32 = sizeof(T) == 4;
  constexpr int kElemsPerRow = kRowBytes / static_cast<int>(sizeof(T));
  constexpr uint32_t kIdesc = sm100::instr_desc(kTf32, kRows, BN);
  constexpr int kEpiArrivals = PAIR ? 8 : 4;  // epilogue warps of the pair / the CTA
  constexpr int kAcc = pow2_at_least(BN);  // columns of one accumulator buffer
  constexpr uint32_t kTmemCols = 2 * kAcc;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256 && kTmemCols <= 512, "BN");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * kStage);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* acc_full = empty_bar + STAGES;  // [2] main product done
  uint64_t* ar_read = acc_full + 2;         // [2] epilogue drained y_ar
  uint64_t* draft_full = ar_read + 2;       // [2] adapter product done
  uint64_t* acc_empty = draft_full + 2;     // [2] epilogue drained the buffer
  uint64_t* t_stored = acc_empty + 2;       // [1] epilogue warps stored a T tile
  uint64_t* mma_done = t_stored + 1;        // [2] every MMA of issuer e has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 2);
  int* order = reinterpret_cast<int*>(tmem_holder + 1);  // next ring item to issue
  // swapped layout with row statistics: [4 epilogue warps][2 outputs][BN] (m, z)
  float2* srs = reinterpret_cast<float2*>(smem + STAGES * kStage + 256);
  const bool swap_stats = SWAP && (p.g[0].stats_ar != nullptr || p.g[0].stats_draft != nullptr);
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // With the CTA pair, rank 0 (the leader) issues the MMAs for both SMs; each
  // CTA loads and drains its own 128 rows of the 256-row tile.
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int my_rows = static_cast<int>(rank) * kBM;     // this CTA's row offset in a tile
  const int my_brows = static_cast<int>(rank) * kBrows;  // and in the B operand
  const int nt_all = p.nT * p.ngroups;  // T tiles of all projections come first
  const int n_split = p.main_tiles - (p.split_start - nt_all);  // tiles of the split round
  const int ntiles = p.split_start + n_split * p.split_k;
  const int G = static_cast<int>(gridDim.x) / (PAIR ? 2 : 1);
  const int C = static_cast<int>(blockIdx.x) / (PAIR ? 2 : 1);
  const int nmine = (ntiles > C) ? (ntiles - 1 - C) / G + 1 : 0;
  // This CTA's T tiles are its first nt_mine tiles (their global indices are
  // the lowest); main tile li has ordinal li - nt_mine among its main tiles,
  // which indexes the ar_read / draft_full barriers and their phases.
  const int nt_mine = (nt_all > C) ? (nt_all - 1 - C) / G + 1 : 0;
  const int nkb = p.kb_total;
  const bool adapter = p.nkb_adapt > 0;
  const int nad = adapter ? p.nkb_adapt : 0;
  constexpr int kInsertItems = (kInsert + KBI - 1) / KBI;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full_bar[s], 1);
      sm100::mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(&acc_full[b], 2);  // one commit per MMA issuer
      sm100::mbar_init(&ar_read[b], kEpiArrivals);
      sm100::mbar_init(&draft_full[b], 2);
      sm100::mbar_init(&acc_empty[b], kEpiArrivals);
    }
    sm100::mbar_init(t_stored, kEpiArrivals);
    sm100::mbar_init(&mma_done[0], 1);
    sm100::mbar_init(&mma_done[1], 1);
    *order = 0;
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == kFirstProducer && lane == 0) {
    sm100::tma_prefetch_desc(&m.x);
    for (int g = 0; g < p.ngroups; ++g) {
      sm100::tma_prefetch_desc(&m.w[g]);
      if (adapter) {
        sm100::tma_prefetch_desc(&m.bm[g]);
        sm100::tma_prefetch_desc(&m.t[g]);
        sm100::tma_prefetch_desc(&m.l[g]);
      }
    }
  }
  if (warp == kMmaWarp0) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       sm100::smem_addr(tmem_holder)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      sm100::tmem_alloc(tmem_holder, kTmemCols);
    }
  }
  sm100::tc_fence_before();
  if constexpr (PAIR) cluster_sync();  // barriers of both CTAs initialised
  else __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // Set-up above overlaps the previous kernel on the stream; global memory
  // (x, T, outputs, flags) is touched only after it has completed.
  uno::launch_dependents();
  uno::grid_dependency_wait();

  // Local tile li of this CTA: global tile t = C + li * G. The T tiles of
  // all projections come first, projection-major: t < nT * ngroups is T tile
  // t % nT of projection t / nT (its A rows start at that index * kRows:
  // rows of x, or with swapped operands rows of the LoRA A). Then main tile
  // u = t - nT * ngroups, projection-major, at (v % tiles_a, v / tiles_a)
  // with v its index within the projection.
  struct Tile {
    bool is_t;
    int g;       // projection
    int a0, b0;  // first A row, first B row
    int tt;      // T tile index within the projection
    int kb0, kb1;  // K-blocks of this unit (a piece of a split tile covers a part)
    int piece;   // piece of a split tile (0: the one that finishes the tile)
    int sidx;    // index of the split tile (-1: not split)
  };
  auto tile_at = [&](int li) {
    const int t = C + li * G;
    Tile x;
    x.is_t = t < nt_all;
    x.kb0 = 0;
    x.kb1 = nkb;
    x.piece = 0;
    x.sidx = -1;
    if (x.is_t) {
      x.g = t / p.nT;
      x.tt = t - x.g * p.nT;
      x.a0 = x.tt * kRows;
      x.b0 = 0;
    } else {
      int u = t - nt_all;
      if (t >= p.split_start) {
        const int j = t - p.split_start;
        x.sidx = j / p.split_k;
        x.piece = j - x.sidx * p.split_k;
        x.kb0 = x.piece * nkb / p.split_k;  // balanced: no piece is empty (nkb >= split_k)
        x.kb1 = (x.piece + 1) * nkb / p.split_k;
        u = p.split_start - nt_all + x.sidx;
      }
      int g = 0;
      while (g + 1 < p.ngroups && u >= p.g[g + 1].tile0) ++g;
      const int v = u - p.g[g].tile0;
      x.g = g;
      x.tt = 0;
      x.a0 = (v % p.g[g].tiles_a) * kRows;
      x.b0 = (v / p.g[g].tiles_a) * BN;
    }
    return x;
  };
  // Ring items of local tile li (KBI K-blocks each, the last of a kind may
  // hold fewer): the first main items of tile li, the adapter items of tile
  // li-1 (if that was a main tile other than the last: its adapter
  // accumulates in place onto its drained y_ar), the remaining main items,
  // and for this CTA's last tile (a main tile) its own adapter items into the
  // other accumulator buffer, so that one drain writes both outputs.
  struct Counts {
    int nmain, nprev, nself;  // K-blocks of each kind
    int imain, iprev, iself;  // ring items of each kind
  };
  auto counts = [&](int li) {
    Counts c;
    const Tile x = tile_at(li);
    c.nmain = x.kb1 - x.kb0;
    c.nprev = (li > 0 && adapter && !tile_at(li - 1).is_t) ? nad : 0;
    c.nself = (li == nmine - 1 && adapter && !x.is_t && x.piece == 0) ? nad : 0;
    c.imain = (c.nmain + KBI - 1) / KBI;
    c.iprev = (c.nprev + KBI - 1) / KBI;
    c.iself = (c.nself + KBI - 1) / KBI;
    return c;
  };
  // Item q of tile li: kind (0 main, 1 previous tile's adapter, 2 own adapter)
  // and its item index j within that kind (K-blocks j * KBI onwards).
  auto item_of = [&](const Counts& c, int q) -> int2 {
    const int head = min(kInsertItems, c.imain);
    if (q < head) return make_int2(0, q);
    if (q < head + c.iprev) return make_int2(1, q - head);
    if (q < c.imain + c.iprev) return make_int2(0, q - c.iprev);
    return make_int2(2, q - c.imain - c.iprev);
  };
  // K-blocks in item j of a kind that has n K-blocks.
  auto item_kbs = [&](int j, int n) { return min(KBI, n - j * KBI); };

  if (warp >= kFirstProducer) {
    if (lane == 0) {
      // ---- TMA producers ----
      // Producer pr issues ring items it with it % kProducers == pr. A thread
      // that has TMA copies in flight stalls at its next mbarrier operation
      // until they land, so one producer would keep a single stage in
      // flight; kProducers of them keep kProducers stages in flight.
      const int pr = warp - kFirstProducer;
      int it = 0;
      bool ok = true;
      int t_ready = -1;  // (projection, row block) whose T this producer saw published
      // Stage of the current ring item, once it is free (null on failure).
      // b_rows: rows of the B box; nk: K-blocks in the item (both CTAs of a
      // pair load the same shapes; the leader expects the bytes of both).
      uint32_t bar_pair = 0;
      auto begin_item = [&](int b_rows, int nk) -> uint8_t* {
        const int s = it % STAGES;
        if (it >= STAGES && !sm100::mbar_wait(&empty_bar[s], ((it / STAGES) - 1) & 1, p.wait_ns)) {
          set_fault(kFaultProducer, &abort_flag);
          ok = false;
          return nullptr;
        }
        if (abort_flag) {
          ok = false;
          return nullptr;
        }
        const uint32_t bytes = static_cast<uint32_t>(nk * (kAbytes + b_rows * kRowBytes));
        if constexpr (PAIR) {
          if (leader) sm100::mbar_arrive_expect_tx(&full_bar[s], 2 * bytes);
          bar_pair = cluster_addr(&full_bar[s], 0);
        } else {
          sm100::mbar_arrive_expect_tx(&full_bar[s], bytes);
        }
        return smem + s * kStage;
      };
      // The A and B boxes of one K-block, at K-block slot j of the stage.
      auto load_kb = [&](uint8_t* stage, int j, const CUtensorMap* ma, int ay,
                         const CUtensorMap* mb, int by, int kx) {
        uint8_t* sa = stage + j * kKb;
        const int s = it % STAGES;
        if constexpr (PAIR) {
          tma_load_2d_pair(sa, ma, bar_pair, kx, ay);
          tma_load_2d_pair(sa + kAbytes, mb, bar_pair, kx, by);
        } else {
          sm100::tma_load_2d(sa, ma, &full_bar[s], kx, ay);
          sm100::tma_load_2d(sa + kAbytes, mb, &full_bar[s], kx, by);
        }
      };
      // Main item j of tile x: K-blocks x.kb0 + j * KBI onwards.
      auto load_main = [&](const Tile& x, int j, int nk) {
        const int b_rows = (x.is_t && !SWAP) ? p.t_brows : kBrows;
        uint8_t* stage = begin_item(b_rows, nk);
        if (!stage) return;
        for (int jj = 0; jj < nk; ++jj) {
          const int kb = x.kb0 + j * KBI + jj;  // K-block within d_in
          const int kx = kb * kElemsPerRow;
          // The CTAs of one weight tile (all row blocks of x) ask for the same
          // K-block at about the same time; the first of them warms L2 for
          // K-block kb + kPrefetch so that none of them waits on DRAM.
          if constexpr (!SWAP) {
            if (!x.is_t && x.a0 == 0 && kb + kPrefetch < nkb)
              sm100::tma_prefetch_l2_2d(&m.w[x.g], kx + kPrefetch * kElemsPerRow,
                                        x.b0 + my_brows);
          }
          if (x.is_t) {
            if constexpr (SWAP) load_kb(stage, jj, &m.l[x.g], x.a0, &m.x, 0, kx);
            else load_kb(stage, jj, &m.x, x.a0 + my_rows, &m.l[x.g],
                         static_cast<int>(rank) * p.t_brows, kx);
          } else {
            if constexpr (SWAP) load_kb(stage, jj, &m.w[x.g], x.a0, &m.x, x.b0, kx);
            else load_kb(stage, jj, &m.x, x.a0 + my_rows, &m.w[x.g], x.b0 + my_brows, kx);
          }
        }
      };
      int last_mine = -1;  // this producer's last ring item
      for (int li = 0; li < nmine && ok; ++li) {
        const Counts c = counts(li);
        const Tile cur = tile_at(li);
        const Tile prev = (li > 0) ? tile_at(li - 1) : cur;
        const int items = c.imain + c.iprev + c.iself;
        for (int q = 0; q < items && ok; ++q, ++it) {
          if (it % kProducers != pr) continue;
          last_mine = it;
          const int2 ik = item_of(c, q);
          const int kind = ik.x, j = ik.y;
          if (kind == 0) {
            load_main(cur, j, item_kbs(j, c.nmain));
            continue;
          }
          const Tile owner = (kind == 1) ? prev : cur;
          const int key = (owner.g << 26) | owner.a0;
          if (t_ready != key) {
            // T must be stored before its TMA load: wait for the T tile(s)
            bool ready = true;
            const uint32_t* fl = p.g[owner.g].t_flags;
            if constexpr (SWAP) {
              for (int t = 0; t < p.nT && ready; ++t)
                ready = wait_flag(fl + t, p.t_wait_epoch, p.wait_ns);
            } else {
              ready = wait_flag(fl + owner.a0 / kRows, p.t_wait_epoch, p.wait_ns);
            }
            if (!ready) {
              set_fault(kFaultProducer, &abort_flag);
              ok = false;
              break;
            }
            fence_proxy_async_global();
            t_ready = key;
          }
          const int nk = item_kbs(j, nad);
          uint8_t* stage = begin_item(kBrows, nk);
          if (!stage) break;
          for (int jj = 0; jj < nk; ++jj) {
            const int kx = (j * KBI + jj) * kElemsPerRow;
            if constexpr (SWAP)
              load_kb(stage, jj, &m.bm[owner.g], owner.a0, &m.t[owner.g], owner.b0, kx);
            else
              load_kb(stage, jj, &m.t[owner.g], owner.a0 + my_rows, &m.bm[owner.g],
                      owner.b0 + my_brows, kx);
          }
        }
      }
      // No copy may still be landing when the CTA exits: wait for this
      // producer's items among the last STAGES (the leader's full barriers
      // count the copies of both CTAs; the pair then meets at a cluster barrier).
      for (int k = (it > STAGES ? it - STAGES : 0); leader && k < it && k <= last_mine; ++k)
        if (k % kProducers == pr &&
            !sm100::mbar_wait(&full_bar[k % STAGES], (k / STAGES) & 1, p.wait_ns))
          set_fault(kFaultProducer, &abort_flag);
    }
  } else if (warp == kMmaWarp0 || warp == kMmaWarp0 + 1) {
    if (lane == 0 && leader) {
      // ---- MMA issuers ----
      // Two threads (warps 4 and 5) issue alternate ring items: item it is
      // issued by issuer it & 1, in ring order, handed over through `order`
      // (a tcgen05 fence on each side of the hand-over orders the MMAs). A
      // thread that has committed stalls at its next wait until its own
      // MMAs finish; with two issuers the other thread's item keeps the
      // tensor pipe busy meanwhile. Per-tile barriers (acc_full, draft_full)
      // take one commit from each issuer, each tracking its own MMAs.
      const int e = warp - kMmaWarp0;
      int it = 0;
      bool ok = true;
      auto fail = [&]() {
        set_fault(kFaultMma, &abort_flag);
        ok = false;
      };
      auto commit = [&](uint64_t* bar) {
        if constexpr (PAIR) commit_pair(bar);
        else sm100::mma_commit(bar);
      };
      // The MMAs of ring item `it` (nk K-blocks of 4 MMAs each); the first
      // MMA overwrites the accumulator unless accumulate_first.
      auto issue = [&](uint32_t d, uint32_t idesc, bool accumulate_first, int nk) {
        const int s = it % STAGES;
        if (!wait_order(order, it, &abort_flag, p.wait_ns) ||
            !sm100::mbar_wait(&full_bar[s], (it / STAGES) & 1, p.wait_ns)) {
          fail();
          return;
        }
        sm100::tc_fence_after();
        const uint32_t sa = sm100::smem_addr(smem + s * kStage);
#pragma unroll
        for (int jj = 0; jj < KBI; ++jj) {
          if (jj < nk) {
            const uint64_t da = sm100::smem_desc_k_sw128(sa + jj * kKb);
            const uint64_t db = sm100::smem_desc_k_sw128(sa + jj * kKb + kAbytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const bool acc = accumulate_first || (jj > 0) || (k > 0);
              if constexpr (PAIR)
                mma_pair<kTf32>(d, da + 2 * k, db + 2 * k, idesc, acc);
              else
                sm100::mma<kTf32>(d, da + 2 * k, db + 2 * k, idesc, acc);
            }
          }
        }
        sm100::tc_fence_before();
        st_release_shared(order, it + 1);
        commit(&empty_bar[s]);
      };
      for (int li = 0; li < nmine && ok; ++li) {
        const Counts c = counts(li);
        const int buf = li & 1, pbuf = buf ^ 1;
        const uint32_t d = tmem + static_cast<uint32_t>(buf * kAcc);
        const uint32_t pd = tmem + static_cast<uint32_t>(pbuf * kAcc);
        const uint32_t idesc = (tile_at(li).is_t && !SWAP) ? p.idesc_t : kIdesc;
        const int items = c.imain + c.iprev + c.iself;
        const int mo = li - 1 - nt_mine;  // main ordinal of the previous tile
        for (int q = 0; q < items && ok; ++q, ++it) {
          const bool mine = (it & 1) == e;
          const int2 ik = item_of(c, q);
          const int kind = ik.x, j = ik.y;
          if (kind == 1) {
            if (mine) {
              if (j == 0) {
                if (!wait_cl(&ar_read[mo & 1], (mo >> 1) & 1, p.wait_ns)) {
                  fail();
                  break;
                }
                sm100::tc_fence_after();
              }
              // adds T Bm^T onto y_ar of the previous tile
              issue(pd, kIdesc, true, item_kbs(j, c.nprev));
            }
            if (ok && j == c.iprev - 1) commit(&draft_full[mo & 1]);
          } else if (kind == 2) {
            if (mine) {
              if (j == 0 && li >= 1) {
                // the other buffer is free once tile li-1 has been drained
                if (!wait_cl(&acc_empty[pbuf], ((li - 1) >> 1) & 1, p.wait_ns)) {
                  fail();
                  break;
                }
                sm100::tc_fence_after();
              }
              issue(pd, kIdesc, j > 0, item_kbs(j, c.nself));  // T Bm^T of this tile, on its own
            }
            if (ok && j == c.iself - 1) commit(&acc_full[buf]);
          } else {
            if (mine) {
              if (j == 0 && li >= 2) {
                if (!wait_cl(&acc_empty[buf], ((li >> 1) - 1) & 1, p.wait_ns)) {
                  fail();
                  break;
                }
                sm100::tc_fence_after();
              }
              issue(d, idesc, j > 0, item_kbs(j, c.nmain));
            }
            if (ok && j == c.imain - 1 && c.nself == 0) commit(&acc_full[buf]);
          }
        }
      }
      // Before TMEM is released every MMA this thread issued must have
      // completed, on the normal path and after an abort alike: a commit
      // tracks all of them (with the pair it also arrives, unused, on the
      // second CTA's barrier).
      commit(&mma_done[e]);
      if (!sm100::mbar_wait(&mma_done[e], 0, p.wait_ns)) set_fault(kFaultMma, &abort_flag);
    } else if constexpr (PAIR) {
      // the second CTA: the leader's last commits arrive here too; wait for
      // them so that no arrival targets this CTA's shared memory after it exits
      if (lane == 0 && !sm100::mbar_wait(&mma_done[warp - kMmaWarp0], 0, p.wait_ns))
        set_fault(kFaultMma, &abort_flag);
    }
  } else {
    // ---- epilogue: warps 0..3, TMEM lane quarter = warp ----
    const int quarter = warp;
    // Epilogue barriers live in the leader; a pair's second CTA arrives remotely.
    auto arrive_leader = [&](uint64_t* bar) {
      if constexpr (PAIR) arrive_at(cluster_addr(bar, 0));
      else sm100::mbar_arrive(bar);
    };
    const int rr = quarter * 32 + lane;
    // Swapped layout: one lane holds one output column for 32 rows. The
    // statistics of this warp's 32 columns for rows cbase..cbase+31 (sv[e] =
    // the stored value of row cbase + e, -inf where there is none) go through
    // the warp's 32 x 33 shared-memory scratch (the pad makes both the column
    // writes and the row reads conflict-free), so that lane l holds row
    // cbase + l's 32 values; it folds them (their maximum, then one 2^x per
    // value against it) and merges the pair into the CTA's running pair for
    // that row (this warp's own slot). Pairs (m, z) are in the log2 domain as
    // everywhere: m = max value times log2 e, z = sum of 2^(v log2 e - m).
    // The pair with the larger reference keeps its sum; only the other one's
    // is rescaled (one 2^x per merge; 2^-inf = 0 covers an empty pair, and
    // two empty pairs stay (-inf, 0)).
    auto merge_mz = [](float& m, float& z, float m2, float z2) {
      const bool first = m >= m2;
      const float hi = first ? m : m2, lo = first ? m2 : m;
      const float zhi = first ? z : z2, zlo = first ? z2 : z;
      z = fmaf(zlo, uno::ex2(lo == -INFINITY ? -INFINITY : lo - hi), zhi);
      m = hi;
    };
    float* sxp = reinterpret_cast<float*>(srs + 4 * 2 * BN) + quarter * 32 * 33;
    auto swap_row_stats = [&](const float* sv, int out, int cbase) {
      constexpr float kL2e = 1.4426950408889634f;
#pragma unroll
      for (int e = 0; e < 32; ++e) sxp[e * 33 + lane] = sv[e];
      __syncwarp();
      float v[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = sxp[lane * 33 + c];
      __syncwarp();  // the next chunk may overwrite the scratch
      float mx = v[0];
#pragma unroll
      for (int c = 1; c < 32; ++c) mx = fmaxf(mx, v[c]);
      if (mx == -INFINITY) return;  // no stored value in this row's 32 columns
      const float ml = mx * kL2e;
      float zp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 32; ++c) zp[c & 3] += uno::ex2(fmaf(v[c], kL2e, -ml));
      float2* slot = srs + (quarter * 2 + out) * BN + cbase + lane;
      float2 acc = *slot;
      merge_mz(acc.x, acc.y, ml, (zp[0] + zp[1]) + (zp[2] + zp[3]));
      *slot = acc;
    };
    if (swap_stats)
      for (int q = 0; q < 2 * BN; q += 32)
        srs[quarter * 2 * BN + q + lane] = make_float2(-INFINITY, 0.f);
    // outputs of the projection of the tile being drained
    T* ya = nullptr;
    T* yd = nullptr;
    T* tb = nullptr;
    int ncols = 0, gi = 0;
    // Drain accumulator columns [0, ncol) into y (row-major, ld columns, nrows rows).
    // gate: for T tiles, the per-row adapter gate (rows of x: the A rows
    // unswapped, the B rows swapped); a closed row stores T = 0.
    auto drain = [&](uint32_t acc, int a0, int b0, T* y, int ld, int nrows, int ncol,
                     float mul, const uint8_t* gate = nullptr, float2* stats = nullptr,
                     int stats_tiles = 0, int stat_out = 0) {
      if (!y) return;
      const uint32_t tq = acc + (static_cast<uint32_t>(quarter * 32) << 16);
      const int arow = a0 + rr;
      if constexpr (!SWAP) {
        if (gate && arow < nrows && gate[arow] == 0) mul = 0.f;
      }
      RowStats rs;
      rs.init();
      for (int c = 0; c < ncol; c += 32) {
        uint32_t v[32];
        sm100::tmem_ld_32x32b_x32(tq + c, v);
        sm100::tmem_ld_wait();
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]) * mul;
        const int brow = b0 + c;
        if constexpr (SWAP) {
          if (gate) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (brow + e < nrows && gate[brow + e] == 0) f[e] = 0.f;
          }
        }
        if constexpr (!SWAP) {
          // row = A row, column = B row
          if (arow < nrows && brow < ld)
            store_row32<T>(y + static_cast<size_t>(arow) * ld + brow, f, ld - brow);
          if (stats && brow < ld) {
            float sv[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[e] = stored_value<T>(f[e]);
            rs.add(sv, min(32, ld - brow));
          }
        } else {
          // row = B row, column = A row
          if (arow < ld) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (brow + e < nrows)
                store_one<T>(y + static_cast<size_t>(brow + e) * ld + arow, f[e]);
          }
          if (stats) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              f[e] = (arow < ld && brow + e < nrows) ? stored_value<T>(f[e]) : -INFINITY;
            swap_row_stats(f, stat_out, c);
          }
        }
      }
      if constexpr (!SWAP) {
        if (stats && arow < nrows)
          stats[static_cast<size_t>(arow) * stats_tiles + b0 / BN] = make_float2(rs.m, rs.z);
      }
    };
    // Drain y_ar = acc and y_draft = acc + adp (both BN columns wide).
    // Last tile with bf16 outputs and the pair layout: the ring is idle by
    // now, so each warp stages its 32 rows of y_ar and y_draft in shared
    // memory (128-byte swizzled boxes of 32 rows x 64 columns, 16 KB per
    // output) and writes them with TMA stores: full 128-byte rows instead of
    // 64-byte pieces 8 KB apart.
    auto drain2_tma = [&](uint32_t acc, uint32_t adp, int a0, int b0) {
      const uint32_t lq = static_cast<uint32_t>(quarter * 32) << 16;
      uint8_t* stage_ar = smem + quarter * 32768;
      uint8_t* stage_dr = stage_ar + 16384;
      const uint32_t sw = static_cast<uint32_t>(lane & 7);
      float2* st_ar = p.g[gi].stats_ar;
      float2* st_dr = p.g[gi].stats_draft;
      RowStats rs_ar, rs_dr;
      rs_ar.init();
      rs_dr.init();
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32], w[32];
        sm100::tmem_ld_32x32b_x32(acc + lq + c, v);
        sm100::tmem_ld_32x32b_x32(adp + lq + c, w);
        sm100::tmem_ld_wait();
        // columns c..c+31 = 4 chunks of 16 bytes in box c/64, chunks (c%64)/8..+3
        float sva[32], svd[32];
        const int box = c >> 6;
        const uint32_t chunk0 = static_cast<uint32_t>((c & 63) >> 3);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float* fv = reinterpret_cast<const float*>(v) + 8 * g;
          uint4 a, d;
          a.x = pack_bf16x2(fv[0], fv[1]);
          a.y = pack_bf16x2(fv[2], fv[3]);
          a.z = pack_bf16x2(fv[4], fv[5]);
          a.w = pack_bf16x2(fv[6], fv[7]);
          float t[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) t[e] = fv[e] + __uint_as_float(w[8 * g + e]);
          d.x = pack_bf16x2(t[0], t[1]);
          d.y = pack_bf16x2(t[2], t[3]);
          d.z = pack_bf16x2(t[4], t[5]);
          d.w = pack_bf16x2(t[6], t[7]);
          const uint32_t off = static_cast<uint32_t>(box * 4096 + lane * 128) +
                               (((chunk0 + g) ^ sw) << 4);
          *reinterpret_cast<uint4*>(stage_ar + off) = a;
          *reinterpret_cast<uint4*>(stage_dr + off) = d;
          if (st_ar || st_dr) {  // the stored (rounded) values, unpacked again
            const uint32_t pa[4] = {a.x, a.y, a.z, a.w}, pd[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              sva[8 * g + 2 * h] = __uint_as_float(pa[h] << 16);
              sva[8 * g + 2 * h + 1] = __uint_as_float(pa[h] & 0xFFFF0000u);
              svd[8 * g + 2 * h] = __uint_as_float(pd[h] << 16);
              svd[8 * g + 2 * h + 1] = __uint_as_float(pd[h] & 0xFFFF0000u);
            }
          }
        }
        if (st_ar || st_dr) {
          const int nvalid = min(32, ncols - (b0 + c));
          if (st_ar) rs_ar.add(sva, nvalid);
          if (st_dr) rs_dr.add(svd, nvalid);
        }
        if ((c & 63) == 32) {
          // a 64-column box of this warp's 32 rows is staged: store it now,
          // so the stores overlap the rest of the drain
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            if (ya) sm100::tma_store_2d(&m.ya[gi], stage_ar + box * 4096, b0 + 64 * box, a0);
            sm100::tma_store_2d(&m.yd[gi], stage_dr + box * 4096, b0 + 64 * box, a0);
            sm100::bulk_commit_group();
          }
        }
      }
      {
        const int arow = a0 + lane;
        if (arow < p.M) {
          const size_t at = static_cast<size_t>(arow) * p.g[gi].stats_tiles + b0 / BN;
          if (st_ar) st_ar[at] = make_float2(rs_ar.m, rs_ar.z);
          if (st_dr) st_dr[at] = make_float2(rs_dr.m, rs_dr.z);
        }
      }
      // the staging buffers must stay intact until the stores have read them
      if (lane == 0) sm100::bulk_wait_group_read_0();
      __syncwarp();
    };
    auto drain2 = [&](uint32_t acc, uint32_t adp, int a0, int b0) {
      const uint32_t lq = static_cast<uint32_t>(quarter * 32) << 16;
      const int arow = a0 + rr;
      float2* st2[2] = {p.g[gi].stats_ar, p.g[gi].stats_draft};
      RowStats rs2[2];
      rs2[0].init();
      rs2[1].init();
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32], w[32];
        sm100::tmem_ld_32x32b_x32(acc + lq + c, v);
        sm100::tmem_ld_32x32b_x32(adp + lq + c, w);
        sm100::tmem_ld_wait();
        float f[32];
        const int brow = b0 + c;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          T* y = pass ? yd : ya;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            f[e] = pass ? f[e] + __uint_as_float(w[e]) : __uint_as_float(v[e]);
          if (!y) continue;
          if constexpr (!SWAP) {
            if (arow < p.M && brow < ncols)
              store_row32<T>(y + static_cast<size_t>(arow) * ncols + brow, f, ncols - brow);
            if (st2[pass] && brow < ncols) {
              float sv[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) sv[e] = stored_value<T>(f[e]);
              rs2[pass].add(sv, min(32, ncols - brow));
            }
          } else {
            if (arow < ncols) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (brow + e < p.M) store_one<T>(y + static_cast<size_t>(brow + e) * ncols + arow, f[e]);
            }
            if (st2[pass]) {
              float sv[32];
#pragma unroll
              for (int e = 0; e < 32; ++e)
                sv[e] = (arow < ncols && brow + e < p.M) ? stored_value<T>(f[e]) : -INFINITY;
              swap_row_stats(sv, pass, c);
            }
          }
        }
      }
      if constexpr (!SWAP) {
        if (arow < p.M) {
          const size_t at = static_cast<size_t>(arow) * p.g[gi].stats_tiles + b0 / BN;
#pragma unroll
          for (int pass = 0; pass < 2; ++pass)
            if (st2[pass]) st2[pass][at] = make_float2(rs2[pass].m, rs2[pass].z);
        }
      }
    };
    for (int li = 0; li < nmine; ++li) {
      const int buf = li & 1;
      const uint32_t acc = tmem + static_cast<uint32_t>(buf * kAcc);
      const Tile x = tile_at(li);
      const bool got = __all_sync(0xFFFFFFFFu, wait_cl(&acc_full[buf], (li >> 1) & 1, p.wait_ns));
      if (!got || abort_flag) {
        if (lane == 0) set_fault(kFaultEpilogue, &abort_flag);
        break;
      }
      sm100::tc_fence_after();
      gi = x.g;
      ya = static_cast<T*>(p.g[gi].y_ar);
      yd = static_cast<T*>(p.g[gi].y_draft);
      tb = static_cast<T*>(p.g[gi].t_buf);
      ncols = p.g[gi].ncols;
      if (x.is_t) {
        // T = scale * x A^T: non-swapped, rows of x by r columns; swapped, r
        // rows (rows of A) by the M columns of x.
        if constexpr (!SWAP) drain(acc, x.a0 + my_rows, 0, tb, p.r, p.M, p.r, p.g[gi].scale, p.gate);
        else drain(acc, x.a0, 0, tb, p.r, p.M, BN, p.g[gi].scale, p.gate);
        sm100::tc_fence_before();
        __threadfence();
        __syncwarp();
        // One thread publishes the tile once all four epilogue warps stored
        // their rows. T tiles are this CTA's tiles 0..nt_mine-1, so li counts
        // the completed phases of t_stored; warp 0 frees the accumulator only
        // after its wait, so the other warps cannot get two T tiles ahead.
        if (lane == 0) {
          arrive_leader(t_stored);
          if (warp == 0 && leader) {
            if (wait_cl(t_stored, li & 1, p.wait_ns)) {
              fence_proxy_async_global();
              st_release_u32(p.g[gi].t_flags + x.tt, p.epoch);
            } else {
              set_fault(kFaultEpilogue, &abort_flag);
            }
          }
          arrive_leader(&acc_empty[buf]);
        }
        __syncwarp();
        continue;
      }
      if (x.sidx >= 0) {
        // a tile split along K (the last round): pieces > 0 hand their fp32
        // partial to piece 0, which adds them before its epilogue
        const int nranks = PAIR ? 2 : 1;
        const uint32_t lq = static_cast<uint32_t>(quarter * 32) << 16;
        auto slot = [&](int piece) {
          const size_t sl =
              (static_cast<size_t>(x.sidx) * (p.split_k - 1) + (piece - 1)) * nranks + rank;
          return p.part_buf + sl * (static_cast<size_t>(kBM) * BN) + static_cast<size_t>(rr) * BN;
        };
        uint32_t* pflags = p.part_flags + static_cast<size_t>(x.sidx) * (p.split_k - 1);
        if (x.piece > 0) {
          float* dst = slot(x.piece);
          for (int c = 0; c < BN; c += 32) {
            uint32_t v[32];
            sm100::tmem_ld_32x32b_x32(acc + lq + c, v);
            sm100::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              __stcg(reinterpret_cast<float4*>(dst + c + e),
                     make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                 __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])));
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) {
            arrive_leader(t_stored);  // this CTA's T tiles used phases 0 .. nt_mine-1
            if (warp == 0 && leader) {
              if (wait_cl(t_stored, nt_mine & 1, p.wait_ns))
                st_release_u32(pflags + (x.piece - 1), p.epoch);
              else
                set_fault(kFaultEpilogue, &abort_flag);
            }
          }
          __syncwarp();
          break;  // a split piece is this CTA's last tile
        }
        // piece 0: wait for the other pieces, add their partials into TMEM
        bool ready = true;
        if (lane == 0)
          for (int q = 1; q < p.split_k && ready; ++q)
            ready = wait_flag(pflags + (q - 1), p.epoch, p.wait_ns);
        ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
        __syncwarp();  // orders lane 0's acquire before the other lanes' loads
        if (!ready) {
          if (lane == 0) set_fault(kFaultEpilogue, &abort_flag);
          break;
        }
        // every piece's loads of a 32-column chunk are issued before any is
        // used (up to 24 x 16 bytes in flight per thread: one L2 round trip
        // per chunk, not one per chunk and piece)
        for (int c = 0; c < BN; c += 32) {
          float4 f[kMaxSplit - 1][8];
#pragma unroll
          for (int q = 1; q < kMaxSplit; ++q)
            if (q < p.split_k) {
              const float* src = slot(q) + c;
#pragma unroll
              for (int e = 0; e < 8; ++e)
                f[q - 1][e] = __ldcg(reinterpret_cast<const float4*>(src + 4 * e));
            }
          uint32_t v[32];
          sm100::tmem_ld_32x32b_x32(acc + lq + c, v);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int q = 1; q < kMaxSplit; ++q)
            if (q < p.split_k) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                v[4 * e] = __float_as_uint(__uint_as_float(v[4 * e]) + f[q - 1][e].x);
                v[4 * e + 1] = __float_as_uint(__uint_as_float(v[4 * e + 1]) + f[q - 1][e].y);
                v[4 * e + 2] = __float_as_uint(__uint_as_float(v[4 * e + 2]) + f[q - 1][e].z);
                v[4 * e + 3] = __float_as_uint(__uint_as_float(v[4 * e + 3]) + f[q - 1][e].w);
              }
            }
          sm100::tmem_st_32x32b_x32(acc + lq + c, v);
        }
        sm100::tmem_st_wait();
      }
      if (adapter && li == nmine - 1) {
        // last tile: y_ar in this buffer, T Bm^T in the other; one pass
        if constexpr (PAIR && sizeof(T) == 2)
          drain2_tma(acc, tmem + static_cast<uint32_t>((buf ^ 1) * kAcc),
                     x.a0 + my_rows + quarter * 32, x.b0);
        else
          drain2(acc, tmem + static_cast<uint32_t>((buf ^ 1) * kAcc), x.a0 + my_rows, x.b0);
        break;
      }
      drain(acc, x.a0 + my_rows, x.b0, ya, ncols, p.M, BN, 1.f, nullptr, p.g[gi].stats_ar,
            p.g[gi].stats_tiles, 0);
      sm100::tc_fence_before();
      __syncwarp();
      const int mo = li - nt_mine;
      if (lane == 0) arrive_leader(adapter ? &ar_read[mo & 1] : &acc_empty[buf]);
      if (!adapter) continue;
      const bool got2 = __all_sync(0xFFFFFFFFu, wait_cl(&draft_full[mo & 1], (mo >> 1) & 1, p.wait_ns));
      if (!got2 || abort_flag) {
        if (lane == 0) set_fault(kFaultEpilogue, &abort_flag);
        break;
      }
      sm100::tc_fence_after();
      drain(acc, x.a0 + my_rows, x.b0, yd, ncols, p.M, BN, 1.f, nullptr, p.g[gi].stats_draft,
            p.g[gi].stats_tiles, 1);
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(&acc_empty[buf]);
    }
    if (swap_stats) {
      // this CTA's pair per row: the four warps' pairs merged, written to its
      // slot (slot = CTA index; CTA 0 marks the slots of absent CTAs empty)
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
      if (quarter == 0) {
        const int T_ = p.g[0].stats_tiles;
        for (int out = 0; out < 2; ++out) {
          float2* st = out ? p.g[0].stats_draft : p.g[0].stats_ar;
          if (!st) continue;
          for (int cb = 0; cb < BN; cb += 32) {
            const int row = cb + lane;
            float m = -INFINITY, z = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const float2 v = srs[(w * 2 + out) * BN + row];
              merge_mz(m, z, v.x, v.y);
            }
            if (row < p.M && static_cast<int>(blockIdx.x) < T_)
              st[static_cast<size_t>(row) * T_ + blockIdx.x] = make_float2(m, z);
          }
          if (blockIdx.x == 0)
            for (int sl = static_cast<int>(gridDim.x); sl < T_; ++sl)
              for (int row = lane; row < p.M; row += 32)
                st[static_cast<size_t>(row) * T_ + sl] = make_float2(-INFINITY, 0.f);
        }
      }
    }
  }

  sm100::tc_fence_before();
  if constexpr (PAIR) cluster_sync();  // neither CTA leaves while its peer may touch it
  else __syncthreads();
  if (warp == kMmaWarp0) {
    sm100::tc_fence_after();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
    else
      sm100::tmem_dealloc(tmem, kTmemCols);
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

// Row-major bf16 [rows][cols] output: boxes of 64 columns (128 bytes) x 32
// rows, 128-byte swizzle; the TMA store skips whatever lies out of bounds.
bool make_store_map(CUtensorMap* map, void* ptr, int cols, int rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

// A fresh value per call for the T-tile flags. Seeded from the clock so that
// a workspace left over from another process is not mistaken for this call's.
// Failure-path test hook (uno_dualpath_test_hooks): a shorter limit for every
// bounded wait, and a skew that makes producers wait for a T-flag value no
// tile writes. Zero: normal operation.
std::atomic<uint64_t> g_test_wait_ns{0};
std::atomic<uint32_t> g_test_t_skew{0};

uint32_t next_epoch() {
  static std::atomic<uint32_t> counter{0};
  static std::once_flag once;
  std::call_once(once, [] {
    const auto now = std::chrono::high_resolution_clock::now().time_since_epoch().count();
    counter.store(static_cast<uint32_t>(now) * 2654435761u);
  });
  uint32_t e;
  do {
    e = counter.fetch_add(1) + 1;
  } while (e == 0);
  return e;
}

int bn_for(int rows) { return rows <= 32 ? 32 : rows <= 64 ? 64 : rows <= 128 ? 128 : 256; }

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Clusters of two that can be resident at once (cached per device).
template <typename K>
int max_pairs(K kern, int bytes) {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return sm_count() / 2;
  if (cached[dev]) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sm_count() & ~1));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(bytes);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = sm_count() / 2;
  }
  cached[dev] = n;
  return n;
}

template <typename T, int BN, bool SWAP, bool PAIR>
int launch_dual(const DualMaps& maps, const GemmParams& p, cudaStream_t st) {
  constexpr int bytes = smem_bytes<BN, PAIR>();
  auto kern = dual_kernel<T, BN, SWAP, PAIR>;
  static std::atomic<uint64_t> attr_done{0};  // devices with the shared-memory opt-in
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return UNO_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (!bit || !(attr_done.load(std::memory_order_relaxed) & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return UNO_ERR_CUDA;
    attr_done.fetch_or(bit, std::memory_order_relaxed);
  }
  const long long units0 = static_cast<long long>(p.nT) * p.ngroups + p.main_tiles;
  long long resident = PAIR ? max_pairs(kern, bytes) : sm_count();
  // the swapped layout's row statistics have one slot per CTA: the launch
  // (and the split plan below, which assumes every CTA is resident) uses at
  // most that many CTAs
  if (SWAP && (p.g[0].stats_ar || p.g[0].stats_draft) && resident > p.g[0].stats_tiles)
    resident = p.g[0].stats_tiles;
  // Split the last, partial round of main tiles along K over the CTAs (or
  // pairs) it would leave idle: 3 or 4 pieces, each of at least 2 K-blocks.
  // (Two pieces do not pay for the hand-off of the fp32 partial: measured on
  // 256 x 256 tiles, the round got slower.)
  GemmParams q = p;
  q.split_start = static_cast<int>(units0);
  q.split_k = 1;
  long long tiles = units0;
  if (units0 > resident) {
    const long long rem = units0 % resident;
    int k = rem > 0 ? static_cast<int>(std::min<long long>(kMaxSplit, resident / rem)) : 1;
    while (k > 1 && p.kb_total < 2 * k) --k;
    const size_t per_slot = static_cast<size_t>(PAIR ? 2 : 1) * kBM * BN * sizeof(float);
    const size_t slots = static_cast<size_t>(rem) * (k - 1);
    const size_t need = slots * per_slot + align256(slots * sizeof(uint32_t));
    if (k >= 3 && units0 - rem >= static_cast<long long>(p.nT) * p.ngroups &&
        need <= p.part_capacity) {
      q.split_k = k;
      q.split_start = static_cast<int>(units0 - rem);
      q.part_flags = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(p.part_buf) +
                                                 slots * per_slot);
      tiles = units0 - rem + rem * k;
    }
  }
  if constexpr (PAIR) {
    long long pairs = resident;
    if (pairs > tiles) pairs = tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, maps, q) != cudaSuccess) return UNO_ERR_CUDA;
  } else {
    long long grid = resident;
    if (grid > tiles) grid = tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, maps, q) != cudaSuccess) return UNO_ERR_CUDA;
  }
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

template <typename T>
int launch_swapped(int bn, const DualMaps& maps, const GemmParams& p, cudaStream_t st) {
  switch (bn) {
    case 32: return launch_dual<T, 32, true, false>(maps, p, st);
    case 64: return launch_dual<T, 64, true, false>(maps, p, st);
    case 128: return launch_dual<T, 128, true, false>(maps, p, st);
    default: return launch_dual<T, 256, true, false>(maps, p, st);
  }
}


bool dual_sizes_ok(int M, int d_in, int d_out, int r, int dtype) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return false;
  const int q = (dtype == UNO_BF16) ? 8 : 4;
  return M >= 0 && M <= (1 << 24) && d_in >= 1 && d_out >= 1 && r >= 1 && r <= 256 &&
         d_in % q == 0 && d_out % q == 0 && r % q == 0 && d_in <= (1 << 24) &&
         d_out <= (1 << 24);
}

// Per-projection workspace: T [M][r] in the operand type, then its T-tile flags.
struct Plan {
  bool swap;
  int esize, kb_main, kb_adapt, nT;
  size_t t_bytes, flag_bytes;  // per projection
  size_t part_bytes;           // per launch: partials of a K-split last round
};

// Partials of a split round: at most (resident - 1) slots of 128 x BN fp32
// per CTA, sized for 148 SMs so that the size does not depend on the device
// (a device that would need more simply splits less).
constexpr int kSizingSms = 148;

Plan make_plan(int M, int d_in, int r, int dtype) {
  Plan pl{};
  pl.esize = (dtype == UNO_BF16) ? 2 : 4;
  pl.swap = M <= 256;
  pl.kb_main = (d_in * pl.esize + kRowBytes - 1) / kRowBytes;
  pl.kb_adapt = (r * pl.esize + kRowBytes - 1) / kRowBytes;
  // with M > 256 a CTA pair computes 256-row tiles, so one T tile per 256 rows
  pl.nT = pl.swap ? (r + kBM - 1) / kBM : (M + 2 * kBM - 1) / (2 * kBM);
  pl.t_bytes = align256(static_cast<size_t>(M) * r * pl.esize);
  pl.flag_bytes = align256(static_cast<size_t>(pl.nT) * sizeof(uint32_t));
  const int bn = pl.swap ? bn_for(M) : 256;
  const size_t per_slot = static_cast<size_t>(pl.swap ? 1 : 2) * kBM * bn * sizeof(float);
  const size_t slots = static_cast<size_t>(pl.swap ? kSizingSms : kSizingSms / 2) - 1;
  pl.part_bytes = slots * per_slot + align256(slots * sizeof(uint32_t));
  return pl;
}

template <typename T>
int run_dualpath(int n, const void* x, const void* const* W, const void* const* A,
                 const void* const* Bm, const float* scale, const uint8_t* gate,
                 void* const* y_ar, void* const* y_draft, int M, int d_in, const int* d_out,
                 int r, int dtype, void* workspace, cudaStream_t st,
                 float* const* stats_ar = nullptr, float* const* stats_draft = nullptr) {
  const Plan pl = make_plan(M, d_in, r, dtype);
  const bool adapter = (y_draft[0] != nullptr);
  const bool tf32 = (dtype == UNO_F32);
  GemmParams gp{};
  gp.kb_total = pl.kb_main;
  gp.nkb_adapt = adapter ? pl.kb_adapt : 0;
  gp.M = M;
  gp.nT = adapter ? pl.nT : 0;
  gp.ngroups = n;
  gp.r = r;
  gp.gate = gate;
  gp.epoch = next_epoch();
  {
    const uint64_t w = g_test_wait_ns.load();
    const uint32_t skew = g_test_t_skew.load();
    gp.wait_ns = w ? w : kWaitNs;
    gp.t_wait_epoch = gp.epoch + skew;
    if (skew != 0 && gp.t_wait_epoch == 0) gp.t_wait_epoch = 1;  // 0 is a cleared flag
  }
  DualMaps maps;
  const int bn = pl.swap ? bn_for(M) : 256;
  const int n_t = (r + 15) / 16 * 16;  // N of the unswapped T tiles
  bool ok = pl.swap ? make_map(&maps.x, x, dtype, d_in, M, bn) : make_map(&maps.x, x, dtype, d_in, M, kBM);
  char* ws = static_cast<char*>(workspace);
  int tile0 = 0;
  for (int g = 0; g < n && ok; ++g) {
    GroupArgs& a = gp.g[g];
    a.ncols = d_out[g];
    a.scale = scale[g];
    a.y_ar = y_ar[g];
    a.y_draft = y_draft[g];
    a.stats_ar = stats_ar ? reinterpret_cast<float2*>(stats_ar[g]) : nullptr;
    a.stats_draft = stats_draft ? reinterpret_cast<float2*>(stats_draft[g]) : nullptr;
    // row statistics: one pair per 256-column tile (CTA pairs), or per CTA
    // (swapped layout: each CTA accumulates over all of its tiles)
    a.stats_tiles = pl.swap ? kSizingSms : (d_out[g] + 255) / 256;
    a.t_buf = ws;
    a.t_flags = reinterpret_cast<uint32_t*>(ws + pl.t_bytes);
    ws += pl.t_bytes + pl.flag_bytes;
    if (pl.swap) {
      a.tiles_a = (d_out[g] + kBM - 1) / kBM;
      a.tiles = a.tiles_a * ((M + bn - 1) / bn);
      ok = make_map(&maps.w[g], W[g], dtype, d_in, d_out[g], kBM);
      if (adapter)
        ok = ok && make_map(&maps.bm[g], Bm[g], dtype, r, d_out[g], kBM) &&
             make_map(&maps.t[g], a.t_buf, dtype, r, M, bn) &&
             make_map(&maps.l[g], A[g], dtype, d_in, r, kBM);
    } else {
      // a CTA pair per 256 x 256 tile (each CTA: 128 rows of x, 128 rows of W);
      // the T tiles' N is r rounded up to 16, half of it per CTA
      a.tiles_a = (M + 2 * kBM - 1) / (2 * kBM);
      a.tiles = a.tiles_a * ((d_out[g] + 255) / 256);
      ok = make_map(&maps.w[g], W[g], dtype, d_in, d_out[g], kBM);
      if (adapter)
        ok = ok && make_map(&maps.bm[g], Bm[g], dtype, r, d_out[g], kBM) &&
             make_map(&maps.t[g], a.t_buf, dtype, r, M, kBM) &&
             make_map(&maps.l[g], A[g], dtype, d_in, r, n_t / 2);
      // output maps of the TMA-store epilogue (bf16): 32 rows x 64 columns
      if (ok && adapter && dtype == UNO_BF16) {
        ok = make_store_map(&maps.yd[g], y_draft[g], d_out[g], M);
        if (ok && y_ar[g]) ok = make_store_map(&maps.ya[g], y_ar[g], d_out[g], M);
      }
    }
    a.tile0 = tile0;
    tile0 += a.tiles;
  }
  if (!ok) return UNO_ERR_CUDA;
  gp.main_tiles = tile0;
  gp.part_buf = reinterpret_cast<float*>(ws);  // after the n per-projection areas
  gp.part_capacity = pl.part_bytes;
  {
    // A captured launch replays with the epoch it was captured with, so under
    // stream capture the flags are cleared by nodes of their own first.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return UNO_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone &&
        (cudaMemsetAsync(workspace, 0, n * (pl.t_bytes + pl.flag_bytes), st) != cudaSuccess ||
         cudaMemsetAsync(ws, 0, pl.part_bytes, st) != cudaSuccess))
      return UNO_ERR_CUDA;
  }
  if (pl.swap) {
    gp.idesc_t = sm100::instr_desc(tf32, kBM, bn);
    gp.t_brows = bn;
    return launch_swapped<T>(bn, maps, gp, st);
  }
  gp.idesc_t = sm100::instr_desc(tf32, 2 * kBM, n_t);
  gp.t_brows = n_t / 2;
  return launch_dual<T, 256, false, true>(maps, gp, st);
}

// Argument checks shared by the single and the grouped entry points.
int check_dual_args(int n, const void* x, const void* const* W, const void* const* A,
                    const void* const* Bm, void* const* y_ar, void* const* y_draft, int M,
                    int d_in, const int* d_out, int r, int dtype, const void* workspace,
                    size_t workspace_bytes) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (n < 1 || n > kMaxGroups) return UNO_ERR_SIZE;
  if (!W || !y_ar || !y_draft || !d_out) return UNO_ERR_NULL;
  for (int g = 0; g < n; ++g)
    if (!dual_sizes_ok(M, d_in, d_out[g], r, dtype)) return UNO_ERR_SIZE;
  if (M == 0) return UNO_OK;
  if (!x) return UNO_ERR_NULL;
  const bool adapter = y_draft[0] != nullptr;
  for (int g = 0; g < n; ++g) {
    if (!W[g] || (!y_ar[g] && !y_draft[g])) return UNO_ERR_NULL;
    if ((y_draft[g] != nullptr) != adapter) return UNO_ERR_NULL;  // all or none
    if (adapter && (!A || !Bm || !A[g] || !Bm[g])) return UNO_ERR_NULL;
    for (const void* ptr : {static_cast<const void*>(W[g]), static_cast<const void*>(y_ar[g]),
                            static_cast<const void*>(y_draft[g]),
                            adapter ? A[g] : nullptr, adapter ? Bm[g] : nullptr})
      if (!uno_host::aligned(ptr, 16)) return UNO_ERR_ALIGN;
  }
  if (!workspace) return UNO_ERR_WORKSPACE;
  if (!uno_host::aligned(x, 16) || !uno_host::aligned(workspace, 16)) return UNO_ERR_ALIGN;
  const Plan pl = make_plan(M, d_in, r, dtype);
  if (workspace_bytes < static_cast<size_t>(n) * (pl.t_bytes + pl.flag_bytes) + pl.part_bytes)
    return UNO_ERR_WORKSPACE;
  return 1;  // proceed
}

int dispatch(int n, const void* x, const void* const* W, const void* const* A,
             const void* const* Bm, const float* scale, const uint8_t* gate, void* const* y_ar,
             void* const* y_draft, int M, int d_in, const int* d_out, int r, int dtype,
             void* workspace, size_t workspace_bytes, void* stream,
             float* const* stats_ar = nullptr, float* const* stats_draft = nullptr) {
  const int chk = check_dual_args(n, x, W, A, Bm, y_ar, y_draft, M, d_in, d_out, r, dtype,
                                  workspace, workspace_bytes);
  if (chk != 1) return chk;
  const int dev = uno_host::check_device();
  if (dev != UNO_OK) return dev;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == UNO_BF16)
    return run_dualpath<uint16_t>(n, x, W, A, Bm, scale, gate, y_ar, y_draft, M, d_in, d_out, r,
                                  dtype, workspace, st, stats_ar, stats_draft);
  return run_dualpath<float>(n, x, W, A, Bm, scale, gate, y_ar, y_draft, M, d_in, d_out, r,
                             dtype, workspace, st, stats_ar, stats_draft);
}

}  // namespace

extern "C" size_t uno_dualpath_workspace_bytes(int M, int d_in, int d_out, int r, int dtype) {
  if (!dual_sizes_ok(M, d_in, d_out, r, dtype)) return 0;
  const Plan pl = make_plan(M, d_in, r, dtype);
  return pl.t_bytes + pl.flag_bytes + pl.part_bytes;
}

extern "C" size_t uno_dualpath_grouped_workspace_bytes(int n, int M, int d_in, const int* d_out,
                                                       int r, int dtype) {
  if (n < 1 || n > kMaxGroups || !d_out) return 0;
  for (int g = 0; g < n; ++g)
    if (!dual_sizes_ok(M, d_in, d_out[g], r, dtype)) return 0;
  const Plan pl = make_plan(M, d_in, r, dtype);
  return static_cast<size_t>(n) * (pl.t_bytes + pl.flag_bytes) + pl.part_bytes;
}

extern "C" int uno_dualpath_linear(const void* x, const void* W, const void* A, const void* Bm,
                                   float scale, void* y_ar, void* y_draft, int M, int d_in,
                                   int d_out, int r, int dtype, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return dispatch(1, x, &W, &A, &Bm, &scale, nullptr, &y_ar, &y_draft, M, d_in, &d_out, r, dtype,
                  workspace, workspace_bytes, stream);
}

extern "C" int uno_dualpath_linear_gated(const void* x, const void* W, const void* A,
                                         const void* Bm, float scale, const uint8_t* gate,
                                         void* y_ar, void* y_draft, int M, int d_in, int d_out,
                                         int r, int dtype, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  return dispatch(1, x, &W, &A, &Bm, &scale, gate, &y_ar, &y_draft, M, d_in, &d_out, r, dtype,
                  workspace, workspace_bytes, stream);
}

extern "C" int uno_dualpath_linear_grouped(int n, const void* x, const void* const* W,
                                           const void* const* A, const void* const* Bm,
                                           const float* scale, const uint8_t* gate,
                                           void* const* y_ar, void* const* y_draft, int M,
                                           int d_in, const int* d_out, int r, int dtype,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream) {
  if (!scale) return UNO_ERR_NULL;
  return dispatch(n, x, W, A, Bm, scale, gate, y_ar, y_draft, M, d_in, d_out, r, dtype,
                  workspace, workspace_bytes, stream);
}

extern "C" int uno_dualpath_stats_tiles(int M, int d_out) {
  if (M < 1 || d_out < 1) return 0;
  // CTA pairs (M > 256): one pair per 256-column tile; swapped layout: one
  // per CTA of the launch (at most kSizingSms CTAs; absent ones write empty
  // pairs)
  return (M <= 256) ? kSizingSms : (d_out + 255) / 256;
}

extern "C" int uno_dualpath_linear_stats(const void* x, const void* W, const void* A,
                                         const void* Bm, float scale, const uint8_t* gate,
                                         void* y_ar, void* y_draft, float* stats_ar,
                                         float* stats_draft, int M, int d_in, int d_out, int r,
                                         int dtype, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  if ((stats_ar && !y_ar) || (stats_draft && !y_draft)) return UNO_ERR_NULL;
  if (!uno_host::aligned(stats_ar, 8) || !uno_host::aligned(stats_draft, 8)) return UNO_ERR_ALIGN;
  return dispatch(1, x, &W, &A, &Bm, &scale, gate, &y_ar, &y_draft, M, d_in, &d_out, r, dtype,
                  workspace, workspace_bytes, stream, &stats_ar, &stats_draft);
}

extern "C" int uno_dualpath_test_hooks(uint64_t wait_ns, uint32_t t_flag_skew) {
  g_test_wait_ns.store(wait_ns);
  g_test_t_skew.store(t_flag_skew);
  return UNO_OK;
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
