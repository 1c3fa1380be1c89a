// Drafting a block with the linear Psi-Spec sampler on sm_100a.
//
// "Unlocking Lossless Speedups in LLMs via Discrete Diffusion", reader page,
// "The Psi-Speculative Sampler": the block's candidate tokens are sampled from
// the joint proposal; the linear sampler draws every position in parallel
// from its own marginal. Here x_{b,i} ~ softmax(q_{b,i}) by the inverse CDF
// over exp(q - max) in index order, with the uniform taken from word 2 of the
// Philox block of (b, i, step) under the verifier's key (words 0 and 1 serve
// the accept test and the resample), so drafting, verification and
// resampling draw independent uniforms from one stream.
//
// One cluster of kCluster CTAs per row (b, i), one pass over the row in HBM:
// each warp of the cluster takes chunks of the row (at least kMinSteps 16-byte
// vectors per lane, so the warp reduction is paid once per several vectors)
// and streams them in rounds of kRound 16-byte vectors per lane through a
// ring of kStages shared-memory stages (cp.async): kStages - 1 rounds are in
// flight while one is folded into a per-lane (running maximum, sum of
// 2^(x - maximum)) in the log2 domain with packed float32x2 arithmetic. The
// warp reduces each chunk to one such pair (the lanes' sums rescaled to the
// warp's maximum and added in float64) in the leading CTA's shared memory
// (distributed shared memory), and the others leave after a cluster barrier.
// The leader then rescales the chunk sums to the largest maximum, takes
// their float64 running sum, finds the chunk where u * total is crossed and
// scans only that chunk (in L2 by then): each thread sums a contiguous
// segment, one block scan places the segments, and the thread whose segment
// crosses finds the token.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include <cooperative_groups.h>

#include "logstat.cuh"
#include "uno.h"
#include "uno_device.cuh"
#include "uno_host.h"

namespace {

namespace cg = cooperative_groups;

constexpr int kMaxChunks = 2048;  // chunk table entries (shared memory, 8 bytes each)
constexpr int kMinSteps = 8;      // vectors per lane in a chunk, at least (2 rounds)

// Launch shapes. Many rows (a 64 x 16 block of drafts): two 128-thread CTAs
// per row, 8 per SM, in about two waves that the hardware balances over the
// SMs. Few rows (a tree's node rows at batch 1, a single sequence's drafts):
// clusters of four or eight 256-thread CTAs per row, 4 per SM, so that a
// handful of rows still keeps enough loads in flight in one wave.
template <int THREADS, int CTAS_PER_SM, int CLUSTER>
struct Shape {
  static constexpr int kThreads = THREADS;
  static constexpr int kWarps = THREADS / 32;
  static constexpr int kCtasPerSm = CTAS_PER_SM;
  static constexpr int kCluster = CLUSTER;  // CTAs per row
};
using Narrow = Shape<128, 8, 2>;
using Wide = Shape<256, 4, 4>;      // at most kWideRows rows
using Widest = Shape<256, 4, 8>;    // at most kWidestRows rows
constexpr int kRound = 4;   // 16-byte vectors per lane per round (a chunk is whole rounds)
constexpr int kStages = 3;  // ring stages per warp, one round each
constexpr int kWideRows = 2 * 148;   // rows of the wide shape, at most
constexpr int kWidestRows = 74;      // rows of the widest shape: one wave of 8-CTA clusters
using uno::kLog2e;

struct SampleParams {
  const void* q;       // [B][seq_rows][V], rows 0..rows-1 of each block drawn
  int B, rows, V;      // rows: rows drawn per sequence
  int seq_rows;        // rows per sequence in memory (>= rows)
  int chunk_len;       // elements per chunk (a multiple of 32 * kVec and of kThreads)
  int nchunks;
  const int32_t* row_key;  // [B][rows] Philox position of each row (null: the row index)
  const int32_t* n_rows;   // [B] rows in use per sequence (null: all)
  int word;                // Philox output word of the uniform (1 or 2)
  uint64_t seed, step;
  int32_t* out;        // [B][rows]
};

// Dynamic shared memory: the warps' copy rings (kStages rounds each), then the
// chunk table: cs[nchunks] (float64: sum over the chunk of 2^(x log2 e - cm))
// and cm[nchunks] (the chunk's maximum times log2 e, -inf when empty).
template <int kWarps>
constexpr int ring_bytes() {
  return kWarps * kStages * kRound * 32 * 16;
}

template <int kWarps>
struct Shared {
  double warp_tot[kWarps];
  float warp_max[kWarps];
  double carry;
  int chunk, last_pos, token;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Exclusive running sum (float64, thread order) across the CTA; the total is
// returned through *total.
template <int kWarps>
__device__ double block_exclusive_scan(double mine, Shared<kWarps>& sh, double* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double up = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += up;
  }
  if (lane == 31) sh.warp_tot[warp] = incl;
  __syncthreads();
  double before = 0.0, all = 0.0;
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) before += sh.warp_tot[w];
    all += sh.warp_tot[w];
  }
  *total = all;
  __syncthreads();
  return before + incl - mine;
}

// 2^(x log2 e - ref) for a logit x and a reference in the log2 domain
// (x = -inf gives 0).
__device__ __forceinline__ float w2(float x, float ref) {
  return uno::ex2(fmaf(x, kLog2e, -ref));
}

template <typename T, typename S>
__global__ void __launch_bounds__(S::kThreads, S::kCtasPerSm)
    sample_drafts_kernel(const SampleParams P) {
  constexpr int kThreads = S::kThreads, kWarps = S::kWarps, kCluster = S::kCluster;
  __shared__ Shared<kWarps> sh;
  extern __shared__ __align__(16) uint4 dyn[];  // rings, then the chunk table (the leader's)
  uno::launch_dependents();
  uno::grid_dependency_wait();
  constexpr int kVec = uno::LogitRow<T>::kVec;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = static_cast<int>(blockIdx.x) % kCluster;  // 1-D clusters of kCluster
  const int bi = static_cast<int>(blockIdx.x) / kCluster;    // b * rows + n
  if (P.n_rows != nullptr && bi % P.rows >= P.n_rows[bi / P.rows]) {
    if (tid == 0 && rank == 0) P.out[bi] = -1;  // a row not in use: the cluster leaves
    return;
  }
  cg::cluster_group cluster = cg::this_cluster();
  const int seq = bi / P.rows;
  const T* row = static_cast<const T*>(P.q) +
                 (static_cast<size_t>(seq) * P.seq_rows + (bi - seq * P.rows)) * P.V;
  const int V = P.V, L = P.chunk_len;
  uint4* ring = dyn + warp * (kStages * kRound * 32);
  double* cs = reinterpret_cast<double*>(dyn + kWarps * kStages * kRound * 32);
  float* cm = reinterpret_cast<float*>(cs + P.nchunks);

  // ---- pass 1: per-chunk (reference, sum of 2^(x - reference)) ----
  // Warp w of the cluster (gw = rank * kWarps + w) takes chunks gw, gw + nw,
  // ... (nw = kCluster * kWarps); a chunk is rpc rounds, a round
  // kRound whole 16-byte vectors per lane (a load instruction of the warp
  // reads 512 contiguous bytes). Elements outside whole vectors (the row's
  // tail, or the whole row when it is not 16-byte aligned) are read one by
  // one at the end of their chunk.
  const bool aligned = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  const int nvec = aligned ? V / kVec : 0;  // whole vectors of the row
  const uint4* vrow = reinterpret_cast<const uint4*>(row);
  const int cvec = L / kVec;                // vectors per chunk
  const int rpc = cvec / (32 * kRound);     // rounds per chunk
  constexpr int nw = kCluster * kWarps;
  const int gw = rank * kWarps + warp;
  const int my_chunks = (gw < P.nchunks) ? (P.nchunks - gw + nw - 1) / nw : 0;
  const int n_rounds = my_chunks * rpc;
  int lc = gw, lr = 0;  // chunk and round of the next copies
  // round j goes to stage j mod kStages; one commit group per round (empty
  // past the end), so wait<kStages - 1> always means "round k has landed"
  auto issue = [&](int j) {
    if (j < n_rounds) {
      uint4* dst = ring + (j % kStages) * (kRound * 32) + lane;
      const int vb = lc * cvec + lr * (32 * kRound) + lane;
#pragma unroll
      for (int k = 0; k < kRound; ++k)
        if (vb + k * 32 < nvec) uno::cp_async16(dst + k * 32, vrow + vb + k * 32);
      if (++lr == rpc) {
        lr = 0;
        lc += nw;
      }
    }
    uno::cp_async_commit();
  };
#pragma unroll
  for (int j = 0; j < kStages - 1; ++j) issue(j);
  float lm = -INFINITY, ls = 0.f;
  int c = gw, r = 0;  // chunk and round being folded
  for (int k = 0; k < n_rounds; ++k) {
    issue(k + kStages - 1);
    uno::cp_async_wait<kStages - 1>();
    uint4 cur[kRound];
    {
      const uint4* src = ring + (k % kStages) * (kRound * 32) + lane;
#pragma unroll
      for (int j = 0; j < kRound; ++j) cur[j] = src[j * 32];
    }
    const int vb = c * cvec + r * (32 * kRound) + lane;
    if (vb + (kRound - 1) * 32 < nvec) {  // every vector of the round is whole
#pragma unroll
      for (int j = 0; j < kRound; j += 2) uno::fold_vecs_max<T, 2>(lm, ls, cur + j);
    } else {
#pragma unroll
      for (int j = 0; j < kRound; ++j)
        if (vb + j * 32 < nvec) uno::fold_vecs_max<T, 1>(lm, ls, cur + j);
    }
    if (++r == rpc) {  // the chunk is complete
      // its elements outside whole vectors, one by one
      const int e0 = max(c * L, nvec * kVec), e1 = min((c + 1) * L, V);
      for (int e = e0 + lane; e < e1; e += 32) {
        uno::fold_one_max(lm, ls, uno::LogitRow<T>::at(row, e));
      }
      // the warp's pair: the largest reference, each lane's sum rescaled to
      // it once, in float64 (32 exact-ish exponentials per chunk)
      float mm = lm;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, o));
      double zd = (lm > -INFINITY)
                      ? static_cast<double>(ls) *
                            exp2(static_cast<double>(lm) - static_cast<double>(mm))
                      : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zd += __shfl_xor_sync(0xFFFFFFFFu, zd, o);
      if (lane == 0) {  // into the leader's table
        *cluster.map_shared_rank(cm + c, 0) = mm;
        *cluster.map_shared_rank(cs + c, 0) = (mm > -INFINITY) ? zd : 0.0;
      }
      lm = -INFINITY;
      ls = 0.f;
      r = 0;
      c += nw;
    }
  }
  uno::cp_async_wait<0>();
  // the table is complete and visible to the leader (release / acquire)
  cluster.sync();
  if (rank != 0) return;

  // ---- the largest chunk reference M and the chunk sums rescaled to it ----
  float mx = -INFINITY;
  for (int c = tid; c < P.nchunks; c += kThreads) mx = fmaxf(mx, cm[c]);
  mx = warp_max(mx);
  if (lane == 0) sh.warp_max[warp] = mx;
  if (tid == 0) {
    sh.chunk = INT_MAX;
    sh.last_pos = -1;
    sh.token = INT_MAX;
  }
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh.warp_max[w]);
  if (M == -INFINITY) {  // no finite logit: no distribution
    if (tid == 0) P.out[bi] = -1;
    return;
  }
  const int b = bi / P.rows;
  const int i = (P.row_key != nullptr) ? P.row_key[bi] : bi - b * P.rows;
  const uint4 words = uno::verify_block_words(P.seed, P.step, b, static_cast<uint32_t>(i));
  const float u = uno::uniform24(P.word == 1 ? words.y : words.z);
  // thread t owns chunks [t * per, (t + 1) * per)
  const int per = (P.nchunks + kThreads - 1) / kThreads;
  const int c_lo = tid * per, c_hi = min(c_lo + per, P.nchunks);
  double mine = 0.0;
  int last_pos_chunk = -1;
  for (int c = c_lo; c < c_hi; ++c) {
    const double w = (cm[c] > -INFINITY)
                         ? cs[c] * exp2(static_cast<double>(cm[c]) - static_cast<double>(M))
                         : 0.0;
    mine += w;
    if (w > 0.0) last_pos_chunk = c;
  }
  double total = 0.0;
  const double before = block_exclusive_scan(mine, sh, &total);
  const double t = static_cast<double>(u) * total;
  {
    double run = before;
    int found = -1;
    for (int c = c_lo; c < c_hi && found < 0; ++c) {
      const double w = (cm[c] > -INFINITY)
                           ? cs[c] * exp2(static_cast<double>(cm[c]) - static_cast<double>(M))
                           : 0.0;
      if (run + w > t) found = c;
      else run += w;
    }
    if (found >= 0) atomicMin(&sh.chunk, found);
    if (last_pos_chunk >= 0) atomicMax(&sh.last_pos, last_pos_chunk);
    __syncthreads();
    if (found >= 0 && found == sh.chunk) sh.carry = run;  // running sum before that chunk
  }
  __syncthreads();
  // Rounding can leave no crossing: then the last chunk with positive weight.
  const bool crossed = sh.chunk != INT_MAX;
  const int ch = crossed ? sh.chunk : sh.last_pos;
  double carry = crossed ? sh.carry : 0.0;
  __syncthreads();
  if (tid == 0) sh.last_pos = -1;
  __syncthreads();

  // ---- scan the chosen chunk: thread t sums the contiguous segment
  // [v_lo + t seg, v_lo + (t + 1) seg), a block scan places the segments, and
  // the segment where the running sum crosses u * total holds the token ----
  const long long v_lo = static_cast<long long>(ch) * L;
  const long long v_hi = min(v_lo + L, static_cast<long long>(V));
  const int seg = L / kThreads;
  const long long s_lo = min(v_lo + static_cast<long long>(tid) * seg, v_hi);
  const long long s_hi = min(s_lo + seg, v_hi);
  double seg_sum = 0.0;
  int seg_last = -1;
  for (long long v = s_lo; v < s_hi; ++v) {
    const float w = w2(uno::LogitRow<T>::at(row, v), M);
    seg_sum += static_cast<double>(w);
    if (w > 0.f) seg_last = static_cast<int>(v);
  }
  double chunk_total = 0.0;
  double run = carry + block_exclusive_scan(seg_sum, sh, &chunk_total);
  if (seg_last >= 0) atomicMax(&sh.last_pos, seg_last);
  if (crossed && seg_sum > 0.0 && run + seg_sum > t) {
    for (long long v = s_lo; v < s_hi; ++v) {
      const float w = w2(uno::LogitRow<T>::at(row, v), M);
      if (w > 0.f && run + static_cast<double>(w) > t) {
        atomicMin(&sh.token, static_cast<int>(v));
        break;
      }
      run += static_cast<double>(w);
    }
  }
  __syncthreads();
  if (tid == 0) P.out[bi] = (sh.token != INT_MAX) ? sh.token : sh.last_pos;
}

bool sample_sizes_ok(int B, int K, int V, int dtype) {
  return (dtype == UNO_BF16 || dtype == UNO_F32) && B >= 0 && B <= (1 << 20) && K >= 1 &&
         K <= 256 && V >= 1 && V <= (1 << 28) && static_cast<long long>(B) * K <= (1 << 28);
}

// Dynamic shared memory above the default 48 KB needs an opt-in, once per
// kernel instantiation and device.
constexpr int kMaxDevices = 64;
template <typename T, typename S>
bool allow_smem(int bytes) {
  static std::atomic<int> allowed[kMaxDevices];  // zero-initialised (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::atomic<int>* a = (dev >= 0 && dev < kMaxDevices) ? &allowed[dev] : nullptr;
  if (a && bytes <= a->load()) return true;
  if (cudaFuncSetAttribute(sample_drafts_kernel<T, S>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  if (a) a->store(bytes);
  return true;
}

template <typename T, typename S>
int run(const uno_host::RowDraws& r, cudaStream_t st) {
  constexpr int kStep = 32 * uno::LogitRow<T>::kVec;  // elements per vector step of a warp
  // a chunk is a whole number of rounds (kRound warp steps) and of CTA-wide
  // segments (both powers of two: the larger is a multiple of the other)
  constexpr int kSegSteps = (S::kThreads > kStep) ? S::kThreads / kStep : 1;
  constexpr int kStepsMult = (kSegSteps > kRound) ? kSegSteps : kRound;
  const int V = r.V;
  SampleParams P{};
  P.q = r.logits;
  P.B = r.B;
  P.rows = r.rows_per_seq;
  P.seq_rows = (r.seq_rows > 0) ? r.seq_rows : r.rows_per_seq;
  P.V = V;
  P.row_key = r.row_key;
  P.n_rows = r.n_rows;
  P.word = r.word;
  P.seed = r.seed;
  P.step = r.step;
  P.out = r.out;
  const long long steps = (static_cast<long long>(V) + kStep - 1) / kStep;
  long long per_chunk =
      std::max<long long>(kMinSteps, (steps + kMaxChunks - 1) / kMaxChunks);  // steps per chunk
  per_chunk = (per_chunk + kStepsMult - 1) / kStepsMult * kStepsMult;
  P.chunk_len = static_cast<int>(per_chunk * kStep);
  P.nchunks = static_cast<int>((V + P.chunk_len - 1) / P.chunk_len);
  cudaLaunchConfig_t cfg = {};
  const int smem = ring_bytes<S::kWarps>() +
                   P.nchunks * static_cast<int>(sizeof(double) + sizeof(float));
  if (!allow_smem<T, S>(smem)) return UNO_ERR_CUDA;
  cfg.gridDim = dim3(static_cast<unsigned>(r.B * r.rows_per_seq * S::kCluster));
  cfg.blockDim = dim3(S::kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S::kCluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, sample_drafts_kernel<T, S>, P) != cudaSuccess)
    return UNO_ERR_CUDA;
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

}  // namespace

int uno_host::sample_rows(const RowDraws& r, cudaStream_t st) {
  if (r.B == 0 || r.rows_per_seq == 0) return UNO_OK;
  const long long rows = static_cast<long long>(r.B) * r.rows_per_seq;
  if (rows <= kWidestRows)
    return (r.dtype == UNO_BF16) ? run<uint16_t, Widest>(r, st) : run<float, Widest>(r, st);
  if (rows <= kWideRows)
    return (r.dtype == UNO_BF16) ? run<uint16_t, Wide>(r, st) : run<float, Wide>(r, st);
  return (r.dtype == UNO_BF16) ? run<uint16_t, Narrow>(r, st) : run<float, Narrow>(r, st);
}

extern "C" int uno_sample_drafts_blocks(const void* logits, int B, int K, int block_rows, int V,
                                        int dtype, uint64_t seed, uint64_t step,
                                        int32_t* draft_tokens, void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (!sample_sizes_ok(B, K, V, dtype) || block_rows < K || block_rows > 4096 ||
      static_cast<long long>(B) * block_rows > (1LL << 28))
    return UNO_ERR_SIZE;
  if (B == 0) return UNO_OK;
  if (!logits || !draft_tokens) return UNO_ERR_NULL;
  if (!uno_host::aligned(logits, dtype == UNO_BF16 ? 2 : 4) ||
      !uno_host::aligned(draft_tokens, 4))
    return UNO_ERR_ALIGN;
  const int dev = uno_host::check_device();
  if (dev != UNO_OK) return dev;
  uno_host::RowDraws r{};
  r.logits = logits;
  r.B = B;
  r.rows_per_seq = K;
  r.seq_rows = block_rows;
  r.V = V;
  r.dtype = dtype;
  r.word = 2;  // drafting: word 2 of the (b, i, step) block
  r.seed = seed;
  r.step = step;
  r.out = draft_tokens;
  return uno_host::sample_rows(r, static_cast<cudaStream_t>(stream));
}

extern "C" int uno_sample_drafts(const void* q_logits, int B, int K, int V, int dtype,
                                 uint64_t seed, uint64_t step, int32_t* draft_tokens,
                                 void* stream) {
  return uno_sample_drafts_blocks(q_logits, B, K, K, V, dtype, seed, step, draft_tokens, stream);
}
