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
// Drafting, three launches:
//   tree_topk_part_kernel   one CTA per (row, slab): a row of a few sequences
//                      is split over several CTAs so that low-batch drafting
//                      still keeps the SMs' loads in flight. Each thread keeps
//                      a sorted register list of its best logits (larger
//                      first, ties to the smaller id) and a running (max, sum
//                      of 2^(x - max)); the CTA merges the lists in top_k
//                      argmax rounds and writes the slab's list and (max, sum)
//                      to the workspace.
//   tree_topk_merge_kernel  one warp per row merges its slabs and writes the
//                      ids and log softmax(q)(id) = x - logsumexp.
//   tree_build_kernel  one CTA per sequence: the budget best sequences by
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
//   tree_walk_kernel   one thread per sequence: follow the draw while it is
//                      the token of a child, emit it and stop otherwise.
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
constexpr int kBuildThreads = 256;
constexpr int kMaxCand = 256;     // candidates of one position step
constexpr int kWalkThreads = 128;
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
  auto take = [&](const float* f, int n, long long x0) {
    float mk = f[0];
    for (int e = 1; e < n; ++e) mk = fmaxf(mk, f[e]);
    mk *= kLog2e;
    if (mk > lm) {
      ls *= uno::ex2(lm - mk);
      lm = mk;
    }
    if (lm > -INFINITY) {
      float add = 0.f;
      for (int e = 0; e < n; ++e) add += uno::ex2(fmaf(f[e], kLog2e, -lm));
      ls += add;
    }
    for (int e = 0; e < n; ++e) top.offer(f[e], static_cast<int>(x0 + e));
  };
  for (long long base = v_lo + tid; base < v_hi; base += kTopThreads * kTopInFlight) {
    uint4 raw[kTopInFlight];
#pragma unroll
    for (int k = 0; k < kTopInFlight; ++k) {
      const long long vi = base + static_cast<long long>(k) * kTopThreads;
      raw[k] = (vi < v_hi) ? __ldg(reinterpret_cast<const uint4*>(row) + vi)
                           : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kTopInFlight; ++k) {
      const long long vi = base + static_cast<long long>(k) * kTopThreads;
      if (vi < v_hi) {
        float f[kVec];
        R::unpack(raw[k], f);
        take(f, kVec, vi * kVec);
      }
    }
  }
  for (long long v = tail0 + tid; v < e1; v += kTopThreads) {
    const float f = R::at(row, v);
    take(&f, 1, v);
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

// Stage 2: one warp per row merges the slabs' lists and (max, sum) pairs and
// writes the row's top_k ids with log softmax = x - logsumexp.
template <int KM>
__global__ void __launch_bounds__(32) tree_topk_merge_kernel(const TopkParams P) {
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int lane = threadIdx.x, rw = blockIdx.x;
  const size_t p0 = static_cast<size_t>(rw) * P.slabs;
  float m = -INFINITY;
  for (int sl = lane; sl < P.slabs; sl += 32) m = fmaxf(m, P.part_m[p0 + sl]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  float sum = 0.f;
  for (int sl = lane; sl < P.slabs; sl += 32) {
    const float ms = P.part_m[p0 + sl];
    if (ms > -INFINITY) sum += P.part_s[p0 + sl] * uno::ex2(ms - m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  const float lse = (m > -INFINITY) ? (m + log2f(sum)) * kLn2 : -INFINITY;

  TopList<KM> top;
  top.init();
  const int n = P.slabs * P.top_k;
  for (int c = lane; c < n; c += 32) top.offer(P.part_val[p0 * P.top_k + c], P.part_id[p0 * P.top_k + c]);
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
      out_i[r] = found ? bi : -1;
      out_l[r] = found ? bv - lse : -INFINITY;
    }
  }
}

struct BuildParams {
  const int32_t* ids;  // [B][D][top_k]
  const float* logq;   // [B][D][top_k]
  int B, D, top_k, budget, N;
  int32_t* node_token;   // [B][N]
  int32_t* node_parent;  // [B][N]
  int32_t* node_depth;   // [B][N]
  int32_t* n_nodes;      // [B]
};

__device__ __forceinline__ unsigned long long prefix_of(unsigned long long t, int j) {
  return t >> (4 * (kMaxDepth - j));  // the first j ranks (1 <= j <= kMaxDepth)
}

__global__ void __launch_bounds__(kBuildThreads) tree_build_kernel(const BuildParams P) {
  __shared__ float k_score[2][kMaxBudget];
  __shared__ unsigned long long k_tup[2][kMaxBudget];
  __shared__ float c_score[kMaxCand];
  __shared__ unsigned long long c_tup[kMaxCand];
  __shared__ float s_lq[kMaxDepth][kMaxTopK];
  __shared__ int s_avail[kMaxDepth];
  __shared__ unsigned char s_rep[kMaxDepth][kMaxBudget];
  __shared__ int s_off[kMaxDepth + 2];
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int b = blockIdx.x, tid = threadIdx.x;
  const int D = P.D, k = P.top_k, budget = P.budget;
  const float* lq = P.logq + static_cast<size_t>(b) * D * k;
  const int32_t* ids = P.ids + static_cast<size_t>(b) * D * k;
  // every position's log-probabilities in one round trip
  for (int e = tid; e < D * k; e += kBuildThreads) s_lq[e / k][e % k] = lq[e];
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
  int cur = 0, nk = 1;
  for (int j = 0; j < D; ++j) {
    const int avail = s_avail[j];
    // candidates (p, s) with (p + 1)(s + 1) <= budget: prefix p owns a run of
    // min(avail, budget / (p + 1)) slots starting at the sum of the runs before
    int nc = 0, off = 0;
    for (int p = 0; p < nk; ++p) {
      const int c = min(avail, budget / (p + 1));
      if (p < tid) off += c;
      nc += c;
    }
    if (tid < nk) {
      const float ps = k_score[cur][tid];
      const unsigned long long pt = k_tup[cur][tid];
      const int cnt = min(avail, budget / (tid + 1));
      for (int s = 0; s < cnt; ++s) {
        c_score[off + s] = ps + s_lq[j][s];
        c_tup[off + s] = pt | (static_cast<unsigned long long>(s) << (4 * (kMaxDepth - 1 - j)));
      }
    }
    __syncthreads();
    const int nxt = cur ^ 1;
    const int keep = min(budget, nc);
    for (int c = tid; c < nc; c += kBuildThreads) {
      const float sc = c_score[c];
      const unsigned long long tu = c_tup[c];
      int rank = 0;
      for (int o = 0; o < nc; ++o) {
        const float so = c_score[o];
        rank += (so > sc || (so == sc && c_tup[o] < tu)) ? 1 : 0;
      }
      if (rank < keep) {
        k_score[nxt][rank] = sc;
        k_tup[nxt][rank] = tu;
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
    for (int m2 = 0; m2 < m && rep; ++m2) rep = prefix_of(k_tup[cur][m2], j) != pre;
    s_rep[j - 1][m] = rep ? 1 : 0;
  }
  __syncthreads();
  if (tid == 0) {
    s_off[1] = 1;
    for (int j = 1; j <= D; ++j) {
      int cnt = 0;
      for (int m = 0; m < nk; ++m) cnt += s_rep[j - 1][m];
      s_off[j + 1] = s_off[j] + cnt;
    }
    P.n_nodes[b] = s_off[D + 1];
  }
  __syncthreads();  // also orders the padding stores before the node stores
  auto node_id = [&](int j, unsigned long long pre) {  // node of a depth-j prefix
    int rank = 0;
    for (int m2 = 0; m2 < nk; ++m2)
      rank += (s_rep[j - 1][m2] && prefix_of(k_tup[cur][m2], j) < pre) ? 1 : 0;
    return s_off[j] + rank;
  };
  for (int w = tid; w < D * nk; w += kBuildThreads) {
    const int j = w / nk + 1, m = w - (j - 1) * nk;
    if (!s_rep[j - 1][m]) continue;
    const unsigned long long t = k_tup[cur][m];
    const int id = node_id(j, prefix_of(t, j));
    const int s = static_cast<int>((t >> (4 * (kMaxDepth - j))) & 15ull);  // rank at position j-1
    tok[id] = ids[(j - 1) * k + s];
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

__global__ void __launch_bounds__(kWalkThreads) tree_walk_kernel(const WalkParams P) {
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int b = blockIdx.x * kWalkThreads + threadIdx.x;
  if (b >= P.B) return;
  const size_t base = static_cast<size_t>(b) * P.N;
  const int32_t* draw = P.draw + base;
  const int32_t* tok = P.node_token + base;
  const int32_t* par = P.node_parent + base;
  const int n = min(max(P.n_nodes[b], 1), P.N);
  int32_t* out = P.out + static_cast<size_t>(b) * (P.D + 1);
  int node = 0, acc = -1;
  for (int j = 0; j <= P.D; ++j) {
    const int y = draw[node];
    if (y < 0) break;  // a row with no distribution on the walk: invalid
    out[j] = y;
    int child = -1;
    if (j < P.D)
      for (int c = node + 1; c < n && child < 0; ++c)
        if (par[c] == node && tok[c] == y) child = c;
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

template <typename T, int KM>
int launch_topk_km(const TopkParams& tp, cudaStream_t st) {
  const int rc = launch_pdl(tree_topk_part_kernel<T, KM>,
                            dim3(static_cast<unsigned>(tp.rows * tp.slabs)), dim3(kTopThreads),
                            tp, st);
  if (rc != UNO_OK) return rc;
  return launch_pdl(tree_topk_merge_kernel<KM>, dim3(static_cast<unsigned>(tp.rows)), dim3(32),
                    tp, st);
}

template <typename T>
int launch_topk(const TopkParams& tp, cudaStream_t st) {
  if (tp.top_k <= 4) return launch_topk_km<T, 4>(tp, st);
  if (tp.top_k <= 8) return launch_topk_km<T, 8>(tp, st);
  return launch_topk_km<T, 16>(tp, st);
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
  const int rc = (dtype == UNO_BF16) ? launch_topk<uint16_t>(tp, st) : launch_topk<float>(tp, st);
  if (rc != UNO_OK) return rc;
  BuildParams bp{topk_ids, topk_logq, B, D, top_k, budget, 1 + D * budget,
                 node_token, node_parent, node_depth, n_nodes};
  return launch_pdl(tree_build_kernel, dim3(static_cast<unsigned>(B)), dim3(kBuildThreads), bp,
                    st);
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
  return launch_pdl(tree_walk_kernel, dim3(static_cast<unsigned>((B + kWalkThreads - 1) /
                                                                 kWalkThreads)),
                    dim3(kWalkThreads), wp, st);
}
