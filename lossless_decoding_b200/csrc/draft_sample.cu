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
// One CTA per row (b, i), one pass over the row in HBM: each warp takes
// chunks of the row (at least kMinSteps 16-byte vectors per lane, so the warp
// reduction is paid once per several vectors), reduces each chunk to (chunk
// max, sum of 2^(x - chunk max)) in the log2 domain and keeps it in shared
// memory. The CTA then rescales the chunk sums to the row maximum, takes their
// float64 running sum, finds the chunk where u * total is crossed and scans
// only that chunk (in L2 by then): each thread sums a contiguous segment, one
// block scan places the segments, and the thread whose segment crosses finds
// the token.
#include <algorithm>
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include "uno.h"
#include "uno_device.cuh"
#include "uno_host.h"

namespace {

constexpr int kMaxChunks = 2048;  // chunk table in shared memory (16 KB)
constexpr int kMinSteps = 8;      // vectors per lane in a chunk, at least

// Launch shapes. Many rows (a 64 x 16 block of drafts): 128-thread CTAs, 8 per
// SM, one wave. Few rows (a tree's node rows at batch 1): 512-thread CTAs, so
// that a handful of rows still keeps enough loads in flight. Four chunks in
// flight per warp either way (more spill registers).
template <int THREADS, int IN_FLIGHT, int CTAS_PER_SM>
struct Shape {
  static constexpr int kThreads = THREADS;
  static constexpr int kWarps = THREADS / 32;
  static constexpr int kInFlight = IN_FLIGHT;  // chunks a warp loads before reducing them
  static constexpr int kCtasPerSm = CTAS_PER_SM;
};
using Narrow = Shape<128, 4, 8>;
using Wide = Shape<512, 4, 2>;
constexpr int kWideRows = 2 * 148;  // at most this many rows: the wide shape
constexpr float kLog2e = 1.4426950408889634f;

struct SampleParams {
  const void* q;       // [B][rows][V]
  int B, rows, V;      // rows: rows per sequence
  int chunk_len;       // elements per chunk (a multiple of 32 * kVec and of kThreads)
  int nchunks;
  const int32_t* row_key;  // [B][rows] Philox position of each row (null: the row index)
  const int32_t* n_rows;   // [B] rows in use per sequence (null: all)
  int word;                // Philox output word of the uniform (1 or 2)
  uint64_t seed, step;
  int32_t* out;        // [B][rows]
};

template <int kWarps>
struct Shared {
  float cm[kMaxChunks];  // chunk maximum (log2 domain), -inf when empty
  float cs[kMaxChunks];  // sum over the chunk of 2^(x log2 e - cm)
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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
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
  constexpr int kThreads = S::kThreads, kWarps = S::kWarps, kInFlight = S::kInFlight;
  __shared__ Shared<kWarps> sh;
  uno::launch_dependents();
  uno::grid_dependency_wait();
  constexpr int kVec = uno::LogitRow<T>::kVec;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bi = blockIdx.x;  // b * rows + n
  if (P.n_rows != nullptr && bi % P.rows >= P.n_rows[bi / P.rows]) {
    if (tid == 0) P.out[bi] = -1;  // a row not in use: the whole CTA leaves
    return;
  }
  const T* row = static_cast<const T*>(P.q) + static_cast<size_t>(bi) * P.V;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  const int V = P.V, L = P.chunk_len;

  // ---- pass 1: per-chunk (max, sum of 2^(x - max)) ----
  // Each step a warp issues one 16-byte load per lane for kInFlight chunks
  // before it reduces any of them. Every lane keeps its own reference (its
  // running maximum, raised only when a larger value arrives) and sum; the
  // warp combines them once per chunk.
  for (int c0 = warp; c0 < P.nchunks; c0 += kWarps * kInFlight) {
    float lm[kInFlight], ls[kInFlight];
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      lm[k] = -INFINITY;
      ls[k] = 0.f;
    }
    // a chunk is L / (32 kVec) steps of one vector per lane
    for (int s = 0; s < L; s += 32 * kVec) {
      uint4 raw[kInFlight];
#pragma unroll
      for (int k = 0; k < kInFlight; ++k) {
        const int c = c0 + k * kWarps;
        const long long v0 = static_cast<long long>(c) * L + s + lane * kVec;
        raw[k] = (c < P.nchunks && vec && v0 + kVec <= V)
                     ? __ldg(reinterpret_cast<const uint4*>(row + v0))
                     : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < kInFlight; ++k) {
        const int c = c0 + k * kWarps;
        const long long v0 = static_cast<long long>(c) * L + s + lane * kVec;
        float f[kVec];  // logits as read (natural log domain)
        if (c < P.nchunks && vec && v0 + kVec <= V) {
          uno::LogitRow<T>::unpack(raw[k], f);
        } else {
#pragma unroll
          for (int e = 0; e < kVec; ++e)
            f[e] = (c < P.nchunks && v0 + e < V) ? uno::LogitRow<T>::at(row, v0 + e) : -INFINITY;
        }
        float mk = f[0];
#pragma unroll
        for (int e = 1; e < kVec; ++e) mk = fmaxf(mk, f[e]);
        mk *= kLog2e;
        if (mk > lm[k]) {  // a larger value: move the reference up
          ls[k] *= uno::ex2(lm[k] - mk);
          lm[k] = mk;
        }
        if (lm[k] > -INFINITY) {
          float add = 0.f;
#pragma unroll
          for (int e = 0; e < kVec; ++e) add += w2(f[e], lm[k]);
          ls[k] += add;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      const int c = c0 + k * kWarps;
      const float m = warp_max(lm[k]);
      const float t = warp_sum((lm[k] > -INFINITY) ? ls[k] * uno::ex2(lm[k] - m) : 0.f);
      if (lane == 0 && c < P.nchunks) {
        sh.cm[c] = m;
        sh.cs[c] = (m > -INFINITY) ? t : 0.f;
      }
    }
  }
  __syncthreads();

  // ---- the row maximum and the rescaled chunk sums ----
  float mx = -INFINITY;
  for (int c = tid; c < P.nchunks; c += kThreads) mx = fmaxf(mx, sh.cm[c]);
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
    const double w = (sh.cm[c] > -INFINITY) ? static_cast<double>(sh.cs[c]) *
                                                  static_cast<double>(uno::ex2(sh.cm[c] - M))
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
      const double w = (sh.cm[c] > -INFINITY) ? static_cast<double>(sh.cs[c]) *
                                                    static_cast<double>(uno::ex2(sh.cm[c] - M))
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

template <typename T, typename S>
int run(const uno_host::RowDraws& r, cudaStream_t st) {
  constexpr int kStep = 32 * uno::LogitRow<T>::kVec;  // elements per vector step of a warp
  // a chunk is a whole number of warp steps and of CTA-wide segments
  constexpr int kStepsMult = (S::kThreads > kStep) ? S::kThreads / kStep : 1;
  const int V = r.V;
  SampleParams P{};
  P.q = r.logits;
  P.B = r.B;
  P.rows = r.rows_per_seq;
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
  cfg.gridDim = dim3(static_cast<unsigned>(r.B * r.rows_per_seq));
  cfg.blockDim = dim3(S::kThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, sample_drafts_kernel<T, S>, P) != cudaSuccess)
    return UNO_ERR_CUDA;
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

}  // namespace

int uno_host::sample_rows(const RowDraws& r, cudaStream_t st) {
  if (r.B == 0 || r.rows_per_seq == 0) return UNO_OK;
  if (static_cast<long long>(r.B) * r.rows_per_seq <= kWideRows)
    return (r.dtype == UNO_BF16) ? run<uint16_t, Wide>(r, st) : run<float, Wide>(r, st);
  return (r.dtype == UNO_BF16) ? run<uint16_t, Narrow>(r, st) : run<float, Narrow>(r, st);
}

extern "C" int uno_sample_drafts(const void* q_logits, int B, int K, int V, int dtype,
                                 uint64_t seed, uint64_t step, int32_t* draft_tokens,
                                 void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (!sample_sizes_ok(B, K, V, dtype)) return UNO_ERR_SIZE;
  if (B == 0) return UNO_OK;
  if (!q_logits || !draft_tokens) return UNO_ERR_NULL;
  if (!uno_host::aligned(q_logits, dtype == UNO_BF16 ? 2 : 4) ||
      !uno_host::aligned(draft_tokens, 4))
    return UNO_ERR_ALIGN;
  const int dev = uno_host::check_device();
  if (dev != UNO_OK) return dev;
  uno_host::RowDraws r{};
  r.logits = q_logits;
  r.B = B;
  r.rows_per_seq = K;
  r.V = V;
  r.dtype = dtype;
  r.word = 2;  // drafting: word 2 of the (b, i, step) block
  r.seed = seed;
  r.step = step;
  r.out = draft_tokens;
  return uno_host::sample_rows(r, static_cast<cudaStream_t>(stream));
}
