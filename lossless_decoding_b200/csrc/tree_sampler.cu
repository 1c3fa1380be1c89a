// Tree variant of the Psi-Spec sampler on sm_100a.
//
// "Unlocking Lossless Speedups in LLMs via Discrete Diffusion": the reader
// page's "The Psi-Speculative Sampler" (worked example (B, K, V) = (3, 2, 2):
// K^(B-1) candidate sequences ranked by joint log-probability, the top V
// kept, every prefix verified by the frozen AR model, the longest valid one
// accepted) and "Sampler Extensions"; the summary page's "Psi-Speculative
// Sampler" (tree sampler: top-K at each position). The pages' (B, K, V) are
// here depth D = B - 1 (positions after the block's AR-only first token),
// top_k and budget.
//
// Drafting, two launches:
//   tree_topk_part_kernel   one CTA per (row, slab): a row of a few sequences
//                      is split over several CTAs so that low-batch drafting
//                      still keeps the SMs' loads in flight. Each thread keeps
//                      a sorted register list of its best logits (larger
//                      first, ties to the smaller id) and a running (max, sum
//                      of 2^(x - max)); only logits at or above a warp
//                      threshold (the top_k-th largest lane maximum so far)
//                      are offered to the lists. The CTA merges the lists in
//                      top_k argmax rounds and writes the slab's list and
//                      (max, sum) to the workspace.
//   tree_build_kernel  one CTA per sequence: one warp per row merges its
//                      slabs and writes the ids and log softmax(q)(id) =
//                      x - logsumexp; then the budget best sequences by
//                      joint log-probability, one position at a time (the
//                      best budget sequences of j + 1 positions extend the
//                      best budget of j positions); a candidate (prefix p,
//                      choice s) can only be kept if (p + 1)(s + 1) <= budget,
//                      so a step ranks at most ~budget ln(budget) candidates.
//                      Ties: the rank tuple packed 4 bits per position,
//                      position 0 in the top nibble, so integer order is
//                      lexicographic order. Then the prefix tree: distinct
//                      prefixes by depth, then by rank tuple.
// Verification, two launches:
//   draws              one inverse-CDF draw per tree node from its AR row
//                      (the sampler's row-draw kernel, uniform = word 1 of
//                      the Philox block (b, depth, step));
//   tree_walk_kernel   one CTA per sequence: the tree in shared memory, each
//                      node's children located there; one thread follows the
//                      draw while it is the token of a child, emits it and
//                      stops otherwise.
#include <algorithm>
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include "uno.h"
#include "uno_device.cuh"
#include "uno_host.h"

namespace {

constexpr int kTopThreads = 128;
constexpr int kTopWarps = kTopThreads / 32;
constexpr int kTopInFlight = 4;   // 16-byte loads in flight per thread
constexpr int kMaxTopK = 16;      // rank of a choice fits 4 bits
constexpr int kMaxDepth = 16;     // 16 positions x 4 bits = one 64-bit tuple
constexpr int kMaxBudget = 64;
constexpr int kBuildThreads = 512;  // a warp per row for the merge (D <= 16)
constexpr int kMaxCand = 256;     // candidates of one position step
constexpr int kWalkThreads = 128;
constexpr int kMaxNodes = 1 + kMaxDepth * kMaxBudget;  // nodes of a tree, at most
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

// A thread's best KM logits, sorted (better first); empty slots (-inf, INT_MAX).
template <int KM>
struct TopList {
  float v[KM];
  int i[KM];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int e = 0; e < KM; ++e) {
      v[e] = -INFINITY;
      i[e] = INT_MAX;
    }
  }
  __device__ __forceinline__ void offer(float x, int idx) {
    // -inf (probability 0) and NaN are never candidates
    if (!(x > -INFINITY) || !better(x, idx, v[KM - 1], i[KM - 1])) return;
    v[KM - 1] = x;
    i[KM - 1] = idx;
#pragma unroll
    for (int e = KM - 1; e > 0; --e) {
      if (better(v[e], i[e], v[e - 1], i[e - 1])) {
        const float tv = v[e];
        v[e] = v[e - 1];
        v[e - 1] = tv;
        const int ti = i[e];
        i[e] = i[e - 1];
        i[e - 1] = ti;
      }
    }
  }
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int e = 0; e < KM - 1; ++e) {
      v[e] = v[e + 1];
      i[e] = i[e + 1];
    }
    v[KM - 1] = -INFINITY;
    i[KM - 1] = INT_MAX;
  }
};

struct TopkParams {
  const void* q;  // [rows][V]
  int rows, V, top_k;
  int slabs;      // CTAs per row
  int slab_len;   // elements per slab (a multiple of 8)
  int32_t* part_id;  // [rows][slabs][top_k] workspace: each slab's best ids
  float* part_val;   // [rows][slabs][top_k] their logits
  float* part_m;     // [rows][slabs] slab maximum (log2 domain)
  float* part_s;     // [rows][slabs] sum over the slab of 2^(x log2 e - part_m)
  int32_t* ids;      // [rows][top_k]
  float* logq;       // [rows][top_k]
};

// Stage 1: one CTA per (row, slab); each thread keeps a sorted register list
// of its best logits and a running (max, sum) over its share of the slab; the
// CTA merges the lists in top_k block-argmax rounds.
template <typename T, int KM>
__global__ void __launch_bounds__(kTopThreads) tree_topk_part_kernel(const TopkParams P) {
  __shared__ float s_v[2][kTopWarps];
  __shared__ int s_i[2][kTopWarps];
  __shared__ float s_m[kTopWarps], s_s[kTopWarps];
  uno::launch_dependents();
  uno::grid_dependency_wait();
  using R = uno::LogitRow<T>;
  constexpr int kVec = R::kVec;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rw = blockIdx.x / P.slabs, slab = blockIdx.x - rw * P.slabs;
  const int V = P.V;
  const T* row = static_cast<const T*>(P.q) + static_cast<size_t>(rw) * V;
  const long long e0 = static_cast<long long>(slab) * P.slab_len;
  const long long e1 = min(e0 + P.slab_len, static_cast<long long>(V));
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  // whole vectors of the slab (e0 is a multiple of kVec), then a scalar tail
  const long long v_lo = vec ? e0 / kVec : 0, v_hi = vec ? e1 / kVec : 0;
  const long long tail0 = vec ? max(v_hi * kVec, e0) : e0;

  TopList<KM> top;
  top.init();
  float lm = -INFINITY, ls = 0.f;  // running max (log2 domain) and sum of 2^(x log2 e - lm)
  // folds n values into (lm, ls); returns their maximum
  auto stat = [&](const float* f, int n) {
    float mx = f[0];
    for (int e = 1; e < n; ++e) mx = fmaxf(mx, f[e]);
    const float mk = mx * kLog2e;
    if (mk > lm) {
      ls *= uno::ex2(lm - mk);
      lm = mk;
    }
    if (lm > -INFINITY) {
      float add = 0.f;
      for (int e = 0; e < n; ++e) add += uno::ex2(fmaf(f[e], kLog2e, -lm));
      ls += add;
    }
    return mx;
  };
  // A value below the warp's threshold cannot be among the slab's top_k:
  // top_k values at least that large have been seen (the threshold is the
  // top_k-th largest of the lanes' round maxima, one per lane, and only
  // grows). Offering only values at or above it keeps most of the list
  // insertions -- chains of dependent compares that also split the warp --
  // out of the stream; the kept set and its order are unchanged.
  float thr = -INFINITY;
  auto kth_of_lanes = [&](float x) {
    float kth = -INFINITY;
    for (int r = 0; r < P.top_k; ++r) {
      float m = x;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      kth = m;
      if (!(m > -INFINITY)) break;  // the same in every lane
      const unsigned holders = __ballot_sync(0xFFFFFFFFu, x == m);
      if (lane == __ffs(holders) - 1) x = -INFINITY;  // one lane gives up its value
    }
    return kth;
  };
  // rounds of kTopInFlight vectors per thread; every thread runs every round
  // (the threshold's shuffles need whole warps)
  for (long long r0 = v_lo; r0 < v_hi; r0 += kTopThreads * kTopInFlight) {
    uint4 raw[kTopInFlight];
#pragma unroll
    for (int k = 0; k < kTopInFlight; ++k) {
      const long long vi = r0 + tid + static_cast<long long>(k) * kTopThreads;
      raw[k] = (vi < v_hi) ? __ldg(reinterpret_cast<const uint4*>(row) + vi)
                           : make_uint4(0u, 0u, 0u, 0u);
    }
    float rmax = -INFINITY;
#pragma unroll
    for (int k = 0; k < kTopInFlight; ++k) {
      const long long vi = r0 + tid + static_cast<long long>(k) * kTopThreads;
      if (vi < v_hi) {
        float f[kVec];
        R::unpack(raw[k], f);
        rmax = fmaxf(rmax, stat(f, kVec));
      }
    }
    // (top_k rounds of shuffles per round: they cost more than they save at
    // top_k 16, measured; such lists take every value)
    if (P.top_k <= 8) thr = fmaxf(thr, kth_of_lanes(rmax));
#pragma unroll
    for (int k = 0; k < kTopInFlight; ++k) {
      const long long vi = r0 + tid + static_cast<long long>(k) * kTopThreads;
      if (vi < v_hi) {
        float f[kVec];
        R::unpack(raw[k], f);
#pragma unroll
        for (int e = 0; e < kVec; ++e)
          if (f[e] >= thr) top.offer(f[e], static_cast<int>(vi * kVec + e));
      }
    }
  }
  for (long long v = tail0 + tid; v < e1; v += kTopThreads) {
    const float f = R::at(row, v);
    stat(&f, 1);
    top.offer(f, static_cast<int>(v));
  }

  // ---- the slab's (max, sum) ----
  {
    float m = lm;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    float sum = (lm > -INFINITY) ? ls * uno::ex2(lm - m) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) {
      s_m[warp] = m;
      s_s[warp] = sum;
    }
  }
  __syncthreads();
  const size_t part = static_cast<size_t>(rw) * P.slabs + slab;
  if (tid == 0) {
    float M = -INFINITY;
    for (int w = 0; w < kTopWarps; ++w) M = fmaxf(M, s_m[w]);
    float S = 0.f;
    for (int w = 0; w < kTopWarps; ++w)
      if (s_m[w] > -INFINITY) S += s_s[w] * uno::ex2(s_m[w] - M);
    P.part_m[part] = M;
    P.part_s[part] = S;
  }

  // ---- the slab's best top_k: block-wide argmax rounds over the list heads ----
  int32_t* out_i = P.part_id + part * P.top_k;
  float* out_v = P.part_val + part * P.top_k;
  for (int r = 0; r < P.top_k; ++r) {
    const int buf = r & 1;
    float bv = top.v[0];
    int bi = top.i[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      s_v[buf][warp] = bv;
      s_i[buf][warp] = bi;
    }
    __syncthreads();
    float wv = s_v[buf][0];
    int wi = s_i[buf][0];
    for (int w = 1; w < kTopWarps; ++w)
      if (better(s_v[buf][w], s_i[buf][w], wv, wi)) {
        wv = s_v[buf][w];
        wi = s_i[buf][w];
      }
    const bool found = wv > -INFINITY;
    if (found && top.i[0] == wi) top.pop();  // ids are unique: one thread holds it
    if (tid == 0) {
      out_i[r] = found ? wi : -1;
      out_v[r] = found ? wv : -INFINITY;
    }
  }
}

// Stage 2 (first part of the build launch): one warp merges a row's slab
// lists and (max, sum) pairs and writes the row's top_k ids with log softmax
// = x - logsumexp, to global memory and to the given shared arrays.
template <int KM>
__device__ void merge_row(const TopkParams& P, int rw, int lane, int32_t* s_id, float* s_lq) {
  const size_t p0 = static_cast<size_t>(rw) * P.slabs;
  // the slabs' candidates, a batch of loads at a time; the first batch is in
  // flight while the (max, sum) pairs are merged
  const int n = P.slabs * P.top_k;
  const float* pv = P.part_val + p0 * P.top_k;
  const int32_t* pi = P.part_id + p0 * P.top_k;
  constexpr int kBatch = 8;
  float v[kBatch];
  int id[kBatch];
  auto load_batch = [&](int c0) {
#pragma unroll
    for (int e = 0; e < kBatch; ++e) {
      const int c = c0 + 32 * e;
      v[e] = (c < n) ? __ldcg(pv + c) : -INFINITY;
      id[e] = (c < n) ? __ldcg(pi + c) : INT_MAX;
    }
  };
  load_batch(lane);
  // the slabs' (max, sum) pairs: a lane merges its slabs (at most two when
  // there are 64), then the warp
  float m = -INFINITY, sum = 0.f;
  for (int sl = lane; sl < P.slabs; sl += 64) {
    const bool two = sl + 32 < P.slabs;
    const float m1 = __ldcg(P.part_m + p0 + sl), s1 = __ldcg(P.part_s + p0 + sl);
    const float m2 = two ? __ldcg(P.part_m + p0 + sl + 32) : -INFINITY;
    const float s2 = two ? __ldcg(P.part_s + p0 + sl + 32) : 0.f;
    const float mm = fmaxf(m, fmaxf(m1, m2));
    if (mm > -INFINITY) {
      sum = ((m > -INFINITY) ? sum * uno::ex2(m - mm) : 0.f) +
            ((m1 > -INFINITY) ? s1 * uno::ex2(m1 - mm) : 0.f) +
            ((m2 > -INFINITY) ? s2 * uno::ex2(m2 - mm) : 0.f);
      m = mm;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    const float s2 = __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    const float mm = fmaxf(m, m2);
    if (mm > -INFINITY) {
      sum = ((m > -INFINITY) ? sum * uno::ex2(m - mm) : 0.f) +
            ((m2 > -INFINITY) ? s2 * uno::ex2(m2 - mm) : 0.f);
      m = mm;
    }
  }
  const float lse = (m > -INFINITY) ? (m + log2f(sum)) * kLn2 : -INFINITY;

  TopList<KM> top;
  top.init();
  for (int c0 = lane; c0 < n; c0 += 32 * kBatch) {
    if (c0 != lane) load_batch(c0);
#pragma unroll
    for (int e = 0; e < kBatch; ++e) top.offer(v[e], id[e]);
  }
  int32_t* out_i = P.ids + static_cast<size_t>(rw) * P.top_k;
  float* out_l = P.logq + static_cast<size_t>(rw) * P.top_k;
  for (int r = 0; r < P.top_k; ++r) {
    float bv = top.v[0];
    int bi = top.i[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    const bool found = bv > -INFINITY;
    if (found && top.i[0] == bi) top.pop();
    if (lane == 0) {
      const int id = found ? bi : -1;
      const float lq = found ? bv - lse : -INFINITY;
      out_i[r] = id;
      out_l[r] = lq;
      s_id[r] = id;
      s_lq[r] = lq;
    }
  }
}

struct BuildParams {
  int B, D, top_k, budget, N;
  int32_t* node_token;   // [B][N]
  int32_t* node_parent;  // [B][N]
  int32_t* node_depth;   // [B][N]
  int32_t* n_nodes;      // [B]
};

__device__ __forceinline__ unsigned long long prefix_of(unsigned long long t, int j) {
  return t >> (4 * (kMaxDepth - j));  // the first j ranks (1 <= j <= kMaxDepth)
}

// One CTA per sequence: the merge of its D rows' slab lists (stage 2), then
// the kept set and its prefix tree.
template <int KM>
__global__ void __launch_bounds__(kBuildThreads) tree_build_kernel(const TopkParams TP,
                                                                   const BuildParams P) {
  __shared__ float k_score[2][kMaxBudget];
  __shared__ unsigned long long k_tup[2][kMaxBudget];
  __shared__ float c_score[kMaxCand];
  __shared__ unsigned long long c_tup[kMaxCand];
  __shared__ float s_lq[kMaxDepth][kMaxTopK];
  __shared__ int32_t s_ids[kMaxDepth][kMaxTopK];
  __shared__ int s_avail[kMaxDepth];
  // s_coff[a][p]: first candidate slot of prefix p when a choices are available
  // (prefix p owns min(a, budget / (p + 1)) slots); s_coff[a][nk] = their number
  __shared__ int s_coff[kMaxTopK + 1][kMaxBudget + 1];
  __shared__ int s_cap[kMaxBudget];  // budget / (p + 1)
  // s_slot_p[a][c]: the prefix that owns candidate slot c when a choices are
  // available (so each candidate is written by its own thread)
  __shared__ unsigned char s_slot_p[kMaxTopK + 1][kMaxCand];
  __shared__ unsigned char s_rep[kMaxDepth][kMaxBudget];
  __shared__ int s_cnt[kMaxDepth + 1];
  __shared__ int s_off[kMaxDepth + 2];
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int D = P.D, k = P.top_k, budget = P.budget;
  for (int q = tid; q < budget; q += kBuildThreads) s_cap[q] = budget / (q + 1);
  // the D rows' merges, one warp per row
  for (int j = warp; j < D; j += kBuildThreads / 32)
    merge_row<KM>(TP, b * D + j, lane, s_ids[j], s_lq[j]);
  __syncthreads();
  for (int a = tid; a <= k; a += kBuildThreads) {
    int off = 0;
    for (int q = 0; q < budget; ++q) {
      s_coff[a][q] = off;
      off += min(a, s_cap[q]);
    }
    s_coff[a][budget] = off;
  }
  __syncthreads();
  for (int w = tid; w < (k + 1) * budget; w += kBuildThreads) {
    const int a = w / budget, q = w - a * budget;
    for (int c = s_coff[a][q]; c < s_coff[a][q + 1]; ++c) s_slot_p[a][c] = static_cast<unsigned char>(q);
  }
  if (tid == 0) {
    k_score[0][0] = 0.f;  // the empty prefix
    k_tup[0][0] = 0ull;
  }
  __syncthreads();
  if (tid < D) {
    int a = 0;  // candidates of position tid (finite entries come first)
    for (int s = 0; s < k; ++s) a += (s_lq[tid][s] > -INFINITY) ? 1 : 0;
    s_avail[tid] = a;
  }
  __syncthreads();
  // The kept set, position by position, by the whole CTA: per step the
  // candidates are written (one thread per candidate slot), then ranked, a
  // barrier after each. A candidate's rank (the candidates ahead of it) is
  // counted by kRankLanes threads, each comparing it with every kRankLanes-th
  // candidate, and summed by shuffles within the group, so a step costs a few
  // comparisons per thread instead of one pass over all candidates.
  constexpr int kRankLanes = 8;
  constexpr int kRankGroups = kBuildThreads / kRankLanes;
  const int sub = tid & (kRankLanes - 1);
  int cur = 0, nk = 1;
  for (int j = 0; j < D; ++j) {
    const int avail = s_avail[j];
    // candidates (p, s) with (p + 1)(s + 1) <= budget: prefix p owns a run
    // of min(avail, budget / (p + 1)) slots from s_coff[avail][p]
    const int nc = s_coff[avail][nk];
    const unsigned long long shift = 4ull * (kMaxDepth - 1 - j);
    for (int c = tid; c < nc; c += kBuildThreads) {
      const int p = s_slot_p[avail][c];
      const int sl = c - s_coff[avail][p];
      c_score[c] = k_score[cur][p] + s_lq[j][sl];
      c_tup[c] = k_tup[cur][p] | (static_cast<unsigned long long>(sl) << shift);
    }
    __syncthreads();
    const int nxt = cur ^ 1;
    const int keep = min(budget, nc);
    // every thread runs the same iterations (the shuffles need whole warps)
    for (int base = 0; base < nc; base += kRankGroups) {
      const int c = base + tid / kRankLanes;
      const bool mine = c < nc;
      int ahead = 0;
      float sc = 0.f;
      unsigned long long tu = 0ull;
      if (mine) {
        sc = c_score[c];
        tu = c_tup[c];
#pragma unroll 8
        for (int o = sub; o < nc; o += kRankLanes) {  // branch-free: both loads always
          const float so = c_score[o];
          const unsigned long long to = c_tup[o];
          ahead += static_cast<int>((so > sc) | ((so == sc) & (to < tu)));
        }
      }
#pragma unroll
      for (int w = kRankLanes / 2; w > 0; w >>= 1) ahead += __shfl_xor_sync(0xFFFFFFFFu, ahead, w);
      if (mine && sub == 0 && ahead < keep) {
        k_score[nxt][ahead] = sc;
        k_tup[nxt][ahead] = tu;
      }
    }
    __syncthreads();
    cur = nxt;
    nk = keep;
  }

  // ---- the prefix tree of the kept sequences ----
  int32_t* tok = P.node_token + static_cast<size_t>(b) * P.N;
  int32_t* par = P.node_parent + static_cast<size_t>(b) * P.N;
  int32_t* dep = P.node_depth + static_cast<size_t>(b) * P.N;
  for (int n = tid; n < P.N; n += kBuildThreads) {
    tok[n] = -1;
    par[n] = -1;
    dep[n] = (n == 0) ? 0 : -1;
  }
  // s_rep[j-1][m]: kept sequence m is the first (smallest m) with its depth-j prefix
  for (int w = tid; w < D * nk; w += kBuildThreads) {
    const int j = w / nk + 1, m = w - (j - 1) * nk;
    const unsigned long long pre = prefix_of(k_tup[cur][m], j);
    bool rep = true;
#pragma unroll 4
    for (int m2 = 0; m2 < m; ++m2) rep &= prefix_of(k_tup[cur][m2], j) != pre;
    s_rep[j - 1][m] = rep ? 1 : 0;
  }
  __syncthreads();
  // nodes per depth, one warp per depth, then their offsets
  for (int j = warp + 1; j <= D; j += kBuildThreads / 32) {
    int c = 0;
    for (int m = lane; m < nk; m += 32) c += s_rep[j - 1][m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    if (lane == 0) s_cnt[j] = c;
  }
  __syncthreads();
  if (tid == 0) {
    s_off[1] = 1;
    for (int j = 1; j <= D; ++j) s_off[j + 1] = s_off[j] + s_cnt[j];
    P.n_nodes[b] = s_off[D + 1];
  }
  __syncthreads();  // also orders the padding stores before the node stores
  auto node_id = [&](int j, unsigned long long pre) {  // node of a depth-j prefix
    int rank = 0;
#pragma unroll 4
    for (int m2 = 0; m2 < nk; ++m2)
      rank += static_cast<int>((s_rep[j - 1][m2] != 0) & (prefix_of(k_tup[cur][m2], j) < pre));
    return s_off[j] + rank;
  };
  for (int w = tid; w < D * nk; w += kBuildThreads) {
    const int j = w / nk + 1, m = w - (j - 1) * nk;
    if (!s_rep[j - 1][m]) continue;
    const unsigned long long t = k_tup[cur][m];
    const int id = node_id(j, prefix_of(t, j));
    const int s = static_cast<int>((t >> (4 * (kMaxDepth - j))) & 15ull);  // rank at position j-1
    tok[id] = s_ids[j - 1][s];
    par[id] = (j == 1) ? 0 : node_id(j - 1, prefix_of(t, j - 1));
    dep[id] = j;
  }
}

struct WalkParams {
  const int32_t* draw;  // [B][N] draw of each node
  const int32_t* node_token;
  const int32_t* node_parent;
  const int32_t* n_nodes;
  int B, D, N;
  int32_t* out;  // [B][D+1]
  int32_t* acc;  // [B]
};

// One CTA per sequence: the tree (draws, tokens, parents) comes into shared
// memory in one round trip, each node's children are located there (first
// child and count), and one thread walks.
__global__ void __launch_bounds__(kWalkThreads) tree_walk_kernel(const WalkParams P) {
  __shared__ int32_t s_draw[kMaxNodes], s_tok[kMaxNodes], s_par[kMaxNodes];
  __shared__ int s_first[kMaxNodes], s_nchild[kMaxNodes];
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int b = blockIdx.x, tid = threadIdx.x;
  const size_t base = static_cast<size_t>(b) * P.N;
  const int n = min(max(P.n_nodes[b], 1), P.N);
  for (int c = tid; c < n; c += kWalkThreads) {
    s_draw[c] = P.draw[base + c];
    s_tok[c] = P.node_token[base + c];
    s_par[c] = P.node_parent[base + c];
    s_first[c] = INT_MAX;
    s_nchild[c] = 0;
  }
  __syncthreads();
  for (int c = 1 + tid; c < n; c += kWalkThreads) {
    const int pa = s_par[c];
    if (pa >= 0 && pa < c) {
      atomicMin(&s_first[pa], c);
      atomicAdd(&s_nchild[pa], 1);
    }
  }
  __syncthreads();
  if (tid != 0) return;
  int32_t* out = P.out + static_cast<size_t>(b) * (P.D + 1);
  int node = 0, acc = -1;
  for (int j = 0; j <= P.D; ++j) {
    const int y = s_draw[node];
    if (y < 0) break;  // a row with no distribution on the walk: invalid
    out[j] = y;
    int child = -1;
    if (j < P.D) {
      // the node's children in index order: the first with the drawn token
      int left = s_nchild[node];
      for (int c = s_first[node]; left > 0 && c < n && child < 0; ++c) {
        if (s_par[c] != node) continue;
        --left;
        if (s_tok[c] == y) child = c;
      }
    }
    if (child < 0) {
      acc = j;
      break;
    }
    node = child;
  }
  for (int j = acc + 1; j <= P.D; ++j) out[j] = -1;
  P.acc[b] = acc;
}

int max_candidates(int budget, int top_k) {
  int n = 0;
  for (int p = 0; p < budget; ++p) n += std::min(top_k, budget / (p + 1));
  return n;
}

bool tree_sizes_ok(int B, int D, int V, int top_k, int budget) {
  if (B < 0 || B > (1 << 20) || D < 1 || D > kMaxDepth || V < 1 || V > (1 << 28)) return false;
  if (top_k < 1 || top_k > kMaxTopK || budget < 1 || budget > kMaxBudget) return false;
  const long long N = 1 + static_cast<long long>(D) * budget;
  return static_cast<long long>(B) * D <= (1 << 28) && static_cast<long long>(B) * N <= (1 << 28);
}

template <typename Kern, typename Params, typename Params2>
int launch_pdl2(Kern kern, dim3 grid, dim3 block, const Params& p, const Params2& p2,
                cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p, p2) != cudaSuccess) return UNO_ERR_CUDA;
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

template <typename Kern, typename Params>
int launch_pdl(Kern kern, dim3 grid, dim3 block, const Params& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return UNO_ERR_CUDA;
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

// Slabs per row: about four 128-thread CTAs per SM over all rows (sized for
// 148 SMs, so the workspace does not depend on the device), at least 2048
// logits per slab, at most 64 slabs.
constexpr int kSizingSms = 148;

int slabs_for(long long rows, int V) {
  long long s = (4LL * kSizingSms + rows - 1) / rows;
  s = std::min<long long>(s, std::max<long long>(1, V / 2048));
  return static_cast<int>(std::max<long long>(1, std::min<long long>(s, 64)));
}

struct TopkPlan {
  int slabs, slab_len;
  size_t id_off, val_off, m_off, s_off, bytes;
};

TopkPlan topk_plan(long long rows, int V, int top_k) {
  TopkPlan pl{};
  pl.slabs = slabs_for(rows, V);
  const long long per = (static_cast<long long>(V) + pl.slabs - 1) / pl.slabs;
  pl.slab_len = static_cast<int>((per + 7) / 8 * 8);
  const size_t n = static_cast<size_t>(rows) * pl.slabs;
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  pl.id_off = 0;
  pl.val_off = a256(n * top_k * sizeof(int32_t));
  pl.m_off = pl.val_off + a256(n * top_k * sizeof(float));
  pl.s_off = pl.m_off + a256(n * sizeof(float));
  pl.bytes = pl.s_off + a256(n * sizeof(float));
  return pl;
}

// The two drafting launches: the slabs' top-k lists, then per sequence the
// merge of its rows and the tree.
template <typename T, int KM>
int launch_draft_km(const TopkParams& tp, const BuildParams& bp, cudaStream_t st) {
  const int rc = launch_pdl(tree_topk_part_kernel<T, KM>,
                            dim3(static_cast<unsigned>(tp.rows * tp.slabs)), dim3(kTopThreads),
                            tp, st);
  if (rc != UNO_OK) return rc;
  return launch_pdl2(tree_build_kernel<KM>, dim3(static_cast<unsigned>(bp.B)),
                     dim3(kBuildThreads), tp, bp, st);
}

template <typename T>
int launch_draft(const TopkParams& tp, const BuildParams& bp, cudaStream_t st) {
  if (tp.top_k <= 4) return launch_draft_km<T, 4>(tp, bp, st);
  if (tp.top_k <= 8) return launch_draft_km<T, 8>(tp, bp, st);
  return launch_draft_km<T, 16>(tp, bp, st);
}

}  // namespace

extern "C" int uno_tree_nodes(int depth, int budget) {
  if (depth < 1 || depth > kMaxDepth || budget < 1 || budget > kMaxBudget) return 0;
  return 1 + depth * budget;
}

extern "C" size_t uno_tree_draft_workspace_bytes(int B, int D, int V, int top_k) {
  if (!tree_sizes_ok(B, D, V, top_k, 1)) return 0;
  return topk_plan(static_cast<long long>(B) * D, V, top_k).bytes;
}

extern "C" int uno_tree_draft(const void* q_logits, int B, int D, int V, int dtype, int top_k,
                              int budget, int32_t* topk_ids, float* topk_logq,
                              int32_t* node_token, int32_t* node_parent, int32_t* node_depth,
                              int32_t* n_nodes, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (!tree_sizes_ok(B, D, V, top_k, budget) || max_candidates(budget, top_k) > kMaxCand)
    return UNO_ERR_SIZE;
  if (B == 0) return UNO_OK;
  if (!q_logits || !topk_ids || !topk_logq || !node_token || !node_parent || !node_depth ||
      !n_nodes)
    return UNO_ERR_NULL;
  if (!uno_host::aligned(q_logits, dtype == UNO_BF16 ? 2 : 4) ||
      !uno_host::aligned(topk_ids, 4) || !uno_host::aligned(topk_logq, 4) ||
      !uno_host::aligned(node_token, 4) || !uno_host::aligned(node_parent, 4) ||
      !uno_host::aligned(node_depth, 4) || !uno_host::aligned(n_nodes, 4))
    return UNO_ERR_ALIGN;
  const TopkPlan pl = topk_plan(static_cast<long long>(B) * D, V, top_k);
  if (!workspace || workspace_bytes < pl.bytes || !uno_host::aligned(workspace, 256))
    return UNO_ERR_WORKSPACE;
  const int dev = uno_host::check_device();
  if (dev != UNO_OK) return dev;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  TopkParams tp{};
  tp.q = q_logits;
  tp.rows = B * D;
  tp.V = V;
  tp.top_k = top_k;
  tp.slabs = pl.slabs;
  tp.slab_len = pl.slab_len;
  tp.part_id = reinterpret_cast<int32_t*>(ws + pl.id_off);
  tp.part_val = reinterpret_cast<float*>(ws + pl.val_off);
  tp.part_m = reinterpret_cast<float*>(ws + pl.m_off);
  tp.part_s = reinterpret_cast<float*>(ws + pl.s_off);
  tp.ids = topk_ids;
  tp.logq = topk_logq;
  BuildParams bp{B, D, top_k, budget, 1 + D * budget, node_token, node_parent, node_depth,
                 n_nodes};
  return (dtype == UNO_BF16) ? launch_draft<uint16_t>(tp, bp, st)
                             : launch_draft<float>(tp, bp, st);
}

extern "C" int uno_tree_verify(const void* p_logits, const int32_t* node_token,
                               const int32_t* node_parent, const int32_t* node_depth,
                               const int32_t* n_nodes, int B, int D, int budget, int V, int dtype,
                               uint64_t seed, uint64_t step, int32_t* node_draw,
                               int32_t* out_tokens, int32_t* accepted_len, void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (!tree_sizes_ok(B, D, V, 1, budget)) return UNO_ERR_SIZE;
  if (B == 0) return UNO_OK;
  if (!p_logits || !node_token || !node_parent || !node_depth || !n_nodes || !node_draw ||
      !out_tokens || !accepted_len)
    return UNO_ERR_NULL;
  if (!uno_host::aligned(p_logits, dtype == UNO_BF16 ? 2 : 4) ||
      !uno_host::aligned(node_token, 4) || !uno_host::aligned(node_parent, 4) ||
      !uno_host::aligned(node_depth, 4) || !uno_host::aligned(n_nodes, 4) ||
      !uno_host::aligned(node_draw, 4) || !uno_host::aligned(out_tokens, 4) ||
      !uno_host::aligned(accepted_len, 4))
    return UNO_ERR_ALIGN;
  const int dev = uno_host::check_device();
  if (dev != UNO_OK) return dev;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = 1 + D * budget;
  uno_host::RowDraws r{};
  r.logits = p_logits;
  r.B = B;
  r.rows_per_seq = N;
  r.V = V;
  r.dtype = dtype;
  r.row_key = node_depth;  // depth j draws with the sampling uniform of position j
  r.n_rows = n_nodes;
  r.word = 1;
  r.seed = seed;
  r.step = step;
  r.out = node_draw;
  int rc = uno_host::sample_rows(r, st);
  if (rc != UNO_OK) return rc;
  WalkParams wp{node_draw, node_token, node_parent, n_nodes, B, D, N, out_tokens, accepted_len};
  return launch_pdl(tree_walk_kernel, dim3(static_cast<unsigned>(B)), dim3(kWalkThreads), wp, st);
}
