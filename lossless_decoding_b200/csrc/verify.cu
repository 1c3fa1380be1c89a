// Block verifier of the linear Psi-Spec sampler on sm_100a.
//
// Operation: "Unlocking Lossless Speedups in LLMs via Discrete Diffusion",
// paperglide reader, "The Psi-Speculative Sampler" (verify every drafted
// position against the frozen AR model, keep the longest accepted prefix, and
// emit one more token from the verifier when all are accepted) and "Sampler
// Extensions" (the linear sampler replaces a rejected tail with one token drawn
// from the verifier), with the standard speculative accept rule
// u < p(x)/q(x) and residual max(0, p - q) that the pages cite.
//
// Two launches per call; no CTA ever waits for another:
//  1. verify_stream_kernel streams every logit row once. One CTA per slab
//     (up to 256 KB of one row, a whole number of 16 KB rounds) issues 16-byte
//     loads, four per thread in use plus the next four prefetched, folds them
//     with packed float32x2 arithmetic into a running (reference, sum of
//     2^(x - reference)) in the log2 domain and writes one partial per slab;
//     the first slab of a drafted row also records the logit at the draft id.
//     Slabs are left to the hardware's CTA scheduler, which hands them to SMs
//     as they free up (SMs do not all get the same bandwidth, so a static
//     split of the rows over one wave of CTAs ends later).
//  2. verify_draw_kernel runs SD CTAs per sequence. Each first decides the
//     sequence (the same decision in every one of them, so that none waits for
//     another): it merges the partials of the sequence's 2K+1 rows,
//     evaluates the accept tests with Philox uniforms and finds the first
//     rejection by ballot. It then sums, over its range of fixed-size
//     vocabulary chunks, the weights of the final draw -- the residual
//     max(0, p_n - q_n) or the bonus row p_K -- with 16-byte loads. The CTA
//     that completes a sequence (atomic counter) takes the running sum of the
//     chunk sums, finds the chunk where u' * total is crossed, scans it token
//     by token and writes the outputs.
// With the LM head's row statistics (uno_verify_block_head) the stream launch
// is replaced by verify_decide_kernel, one CTA per sequence, which merges the
// head's per-tile partials, decides and records the decision for the draw.
//
// Precision of the draw: a token's weight is 2^(x log2 e - L) on the SFU, L
// the row's log2-sum-exp from the decision (two floats) and the argument
// formed by FMAs with log2 e in two parts, so its error is three float32
// roundings of the argument; a vector's weights are summed in float32, all
// longer sums in float64.
#include <atomic>
#include <cfloat>
#include <climits>
#include <cstdint>
#include <cstdio>

#include <cuda_runtime.h>

#include "uno.h"
#include "logstat.cuh"
#include "uno_device.cuh"
#include "uno_host.h"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStreamCtasPerSm = 4;
constexpr int kRound = 4;                 // 16-byte vectors per thread per round
constexpr int kSlabBytes = 262144;        // target bytes streamed by one CTA
constexpr int kMinSlabBytes = kThreads * 16;
constexpr int kMaxK = 256;
constexpr int kMaxRows = 2 * kMaxK + 1;
static_assert(kMaxK <= kThreads, "the decision takes one position per thread");
constexpr int kChunkMin = 256;            // vocabulary entries per inverse-CDF chunk
constexpr int kMaxChunks = 4096;          // chunks per row (the chunk length grows beyond)
constexpr int kDrawCtasPerSm = 4;
constexpr int kDrawCtasTarget = 148 * kDrawCtasPerSm;  // one wave of draw CTAs
constexpr int kSizingSms = 148;           // fixed, so the workspace size is device-independent
using uno::kLog2e;
constexpr float kLn2 = 0.6931471805599453f;

struct Partial {
  float m;  // reference in the log2 domain (see fold)
  float z;  // sum over the slab of 2^(l * log2(e) - m)
};

// What the draw needs to know about one sequence.
struct __align__(16) Decision {
  int n;        // first rejected position (K: all accepted)
  int invalid;  // a draft id was out of range
  int mode;     // 0: residual max(0, p_n - q_n); 1: the row p_n itself
  int pad;
  double lp, lq;  // log2-sum-exp of the draw rows (lq unused in mode 1)
};

struct VerifyParams {
  const void* p_logits;
  const void* q_logits;
  const int32_t* draft;
  int B, K, V;
  int S;          // slabs per row
  int nchunks;    // inverse-CDF chunks per row
  int chunk_len;  // vocabulary entries per chunk
  int SD;         // draw CTAs per sequence
  uint64_t seed, step;
  int32_t* out_tokens;
  int32_t* accepted_len;
  float* p_at_draft;
  float* q_at_draft;
  float* row_lse;
  Partial* partials;    // [B][2K+1][slots]
  double* chunk_sums;   // [B][nchunks] draw-weight sums of the chunks
  int* draw_count;      // [B], set to 0 before the draw launch
  Decision* decisions;  // [B] (the LM-head path: written by the decision launch)
  // [B][2K+1]: logit of row j at its sequence's draft id (rows j != K; 0 for
  // an id out of range), recorded by the stream launch; null without it
  float* draft_logit = nullptr;
  int ring = 0;  // the draw launch has a copy ring in dynamic shared memory
  // Rows of q per sequence in memory: K (q is [B][K][V]) or K+1 (q is the
  // draft-pathway output of the same B x (K+1) rows as p, bonus rows unused).
  int q_rows = 0;
  // Row statistics written by the LM-head GEMM (null: the stream launch
  // computes them): ext_T partials per logit row, in the partial convention.
  const Partial* ext_p = nullptr;  // [B][K+1][ext_T]
  const Partial* ext_q = nullptr;  // [B][q_rows][ext_T]
  int ext_T = 0;
};

// ---- element access ------------------------------------------------------------

template <typename T>
using Elem = uno::LogitRow<T>;

using uno::fold;
using uno::fold_pair;
using uno::merge;
using uno::warp_merge;

// A row is a scalar head up to the first 16-byte boundary, nvec full 16-byte
// vectors, then a scalar tail.
struct RowGeom {
  int head, nvec, tail;
};

template <typename T>
__device__ __forceinline__ RowGeom row_geom(size_t elem_offset, int V) {
  constexpr int kVec = Elem<T>::kVec;
  const int mis = static_cast<int>(elem_offset % kVec);
  int head = mis ? (kVec - mis) : 0;
  if (head > V) head = V;
  const int nvec = (V - head) / kVec;
  return {head, nvec, V - head - nvec * kVec};
}

// Row j of sequence b: j = 0..K are the AR rows p_0..p_K, j = K+1..2K the draft
// rows q_0..q_{K-1}.
template <typename T>
__device__ __forceinline__ const T* row_ptr(const VerifyParams& P, int b, int j, size_t* off) {
  const int K = P.K;
  size_t row;
  const T* base;
  if (j <= K) {
    row = static_cast<size_t>(b) * (K + 1) + j;
    base = static_cast<const T*>(P.p_logits);
  } else {
    row = static_cast<size_t>(b) * P.q_rows + (j - K - 1);
    base = static_cast<const T*>(P.q_logits);
  }
  *off = row * static_cast<size_t>(P.V);
  return base + *off;
}

// ---- launch 1: streaming ----------------------------------------------------------------

template <typename T>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm)
    verify_stream_kernel(const VerifyParams P) {
  constexpr int kVec = Elem<T>::kVec;
  __shared__ float red_m[kWarps], red_z[kWarps];
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = 2 * P.K + 1;
  const int s = blockIdx.x % P.S;
  const int rj = blockIdx.x / P.S;
  const int j = rj % R, b = rj / R;

  size_t off;
  const T* row = row_ptr<T>(P, b, j, &off);
  const RowGeom g = row_geom<T>(off, P.V);
  constexpr int kStep = kRound * kThreads;  // vectors per round of the whole CTA
  // Every slab but the last of a row holds a whole number of rounds.
  const int per = ((g.nvec + P.S - 1) / P.S + kStep - 1) / kStep * kStep;
  const int v0 = min(s * per, g.nvec), v1 = min(v0 + per, g.nvec);
  const uint4* vrow = reinterpret_cast<const uint4*>(row + g.head);

  // The first slab's thread 0 of each drafted row also records the logit at
  // the draft id: the id is loaded first, the logit while the first round is
  // folded, so neither load stalls the stream.
  const bool rec = (P.draft_logit != nullptr) && s == 0 && j != P.K && tid == 0;
  int xq = -1;
  float xl = 0.f;
  if (rec) xq = __ldg(P.draft + static_cast<size_t>(b) * P.K + (j < P.K ? j : j - P.K - 1));

  float m = -INFINITY, z = 0.f;
  const int rounds = (v1 - v0 + kStep - 1) / kStep;  // the last one may be partial
  uint4 cur[kRound], nxt[kRound];
#pragma unroll
  for (int k = 0; k < kRound; ++k) {
    const int idx = v0 + k * kThreads + tid;
    cur[k] = (idx < v1) ? __ldg(vrow + idx) : make_uint4(0, 0, 0, 0);
  }
  for (int r = 0; r < rounds; ++r) {
    const int base = v0 + r * kStep;
    if (r + 1 < rounds) {  // prefetch the next round (predicated: it may be partial)
#pragma unroll
      for (int k = 0; k < kRound; ++k) {
        const int idx = base + kStep + k * kThreads + tid;
        nxt[k] = (idx < v1) ? __ldg(vrow + idx) : make_uint4(0, 0, 0, 0);
      }
    }
    if (rec && r == 0 && xq >= 0 && xq < P.V) xl = Elem<T>::at(row, xq);
    if (base + kStep <= v1) {  // a full round: no predication
#pragma unroll
      for (int k = 0; k < kRound; k += 2) fold_pair<T>(m, z, cur + k);
    } else {
#pragma unroll
      for (int k = 0; k < kRound; ++k) {
        if (base + k * kThreads + tid < v1) {
          float f[kVec];
          Elem<T>::unpack(cur[k], f);
          fold<kVec>(m, z, f);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kRound; ++k) cur[k] = nxt[k];
  }
  if (rec && rounds == 0 && xq >= 0 && xq < P.V) xl = Elem<T>::at(row, xq);
  if (s == 0 && tid < g.head) {
    const float v = Elem<T>::at(row, tid);
    fold<1>(m, z, &v);
  }
  if (s == P.S - 1 && tid < g.tail) {
    const float v =
        Elem<T>::at(row, static_cast<size_t>(g.head) + static_cast<size_t>(g.nvec) * kVec + tid);
    fold<1>(m, z, &v);
  }
  warp_merge(m, z);
  if (lane == 0) {
    red_m[warp] = m;
    red_z[warp] = z;
  }
  __syncthreads();
  if (warp == 0) {
    m = (lane < kWarps) ? red_m[lane] : -INFINITY;
    z = (lane < kWarps) ? red_z[lane] : 0.f;
    warp_merge(m, z);
    if (lane == 0) {
      P.partials[static_cast<size_t>(blockIdx.x)] = Partial{m, z};
      if (rec) P.draft_logit[static_cast<size_t>(b) * R + j] = xl;
      // the draw launch counts its CTAs of this sequence from 0
      if (j == 0 && s == 0) P.draw_count[b] = 0;
    }
  }
}

// ---- the decision of one sequence (a whole CTA) ------------------------------------

struct DecideShared {
  float row_m[kMaxRows], row_z[kMaxRows];
  int x[kMaxK];  // the sequence's draft ids
  int first_reject, invalid;
  Decision d;
};

// Merges the row statistics of sequence b (the slab partials, or the LM head's
// tile partials when P.ext_p is set), runs the K accept tests, finds the first
// rejection and leaves the decision in sh.d. With `outputs`, also writes
// row_lse, p/q at the drafts and the outputs of a sequence with an invalid
// draft id (the draw writes the others).
template <typename T>
__device__ void decide_sequence(const VerifyParams& P, int b, DecideShared& sh, bool outputs) {
  const int tid = threadIdx.x;
  const int K = P.K, R = 2 * K + 1, V = P.V;
  // Thread i < K (K <= kThreads) loads draft x_i and the logits at it first
  // (recorded by the stream launch when it ran: then no load waits for x_i),
  // and draws its Philox words, all overlapping the merge of the statistics.
  int x = -1;
  float lpx = 0.f, lqx = 0.f;
  uint4 words = make_uint4(0, 0, 0, 0);
  if (tid < K) {
    x = P.draft[static_cast<size_t>(b) * K + tid];
    if (P.draft_logit != nullptr) {
      lpx = __ldcg(P.draft_logit + static_cast<size_t>(b) * R + tid);
      lqx = __ldcg(P.draft_logit + static_cast<size_t>(b) * R + K + 1 + tid);
    } else if (x >= 0 && x < V) {
      size_t off;
      lpx = Elem<T>::at(row_ptr<T>(P, b, tid, &off), x);
      lqx = Elem<T>::at(row_ptr<T>(P, b, K + 1 + tid, &off), x);
    }
    words = uno::verify_block_words(P.seed, P.step, b, tid);
    sh.x[tid] = x;
  }
  if (P.ext_p == nullptr) {
    const int S = P.S;
    for (int j = tid; j < R; j += kThreads) {
      const Partial* pp = P.partials + (static_cast<size_t>(b) * R + j) * S;
      float m = -INFINITY, z = 0.f;
      for (int s0 = 0; s0 < S; s0 += 8) {  // eight loads in flight, merged in slab order
        Partial v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = (s0 + k < S) ? pp[s0 + k] : Partial{-INFINITY, 0.f};
#pragma unroll
        for (int k = 0; k < 8; ++k) merge(m, z, v[k].m, v[k].z);
      }
      sh.row_m[j] = m;
      sh.row_z[j] = z;
    }
  } else {
    // the LM head's column-tile partials (hundreds per row): one warp per row,
    // lanes over the tiles, then a shuffle reduction
    const int lane = tid & 31, warp = tid >> 5;
    for (int j = warp; j < R; j += kWarps) {
      const Partial* pp = (j <= K)
          ? P.ext_p + (static_cast<size_t>(b) * (K + 1) + j) * P.ext_T
          : P.ext_q + (static_cast<size_t>(b) * P.q_rows + (j - K - 1)) * P.ext_T;
      float m = -INFINITY, z = 0.f;
      for (int t0 = lane; t0 < P.ext_T; t0 += 32 * 4) {  // four loads in flight per lane
        Partial v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int t = t0 + 32 * k;
          v[k] = (t < P.ext_T) ? pp[t] : Partial{-INFINITY, 0.f};
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) merge(m, z, v[k].m, v[k].z);
      }
      warp_merge(m, z);
      if (lane == 0) {
        sh.row_m[j] = m;
        sh.row_z[j] = z;
      }
    }
  }
  if (tid == 0) {
    sh.first_reject = K;
    sh.invalid = 0;
  }
  __syncthreads();
  if (outputs && P.row_lse)
    for (int j = tid; j < R; j += kThreads)
      P.row_lse[static_cast<size_t>(b) * R + j] = (sh.row_m[j] + log2f(sh.row_z[j])) * kLn2;

  // accept tests, one thread per position; first rejection by ballot
  {
    const int i = tid;
    bool rejected = false;
    if (i < K) {
      if (x < 0 || x >= V) {
        atomicOr(&sh.invalid, 1);
      } else {
        const float pp = uno::ex2(fmaf(lpx, kLog2e, -sh.row_m[i])) / sh.row_z[i];
        const float qq = uno::ex2(fmaf(lqx, kLog2e, -sh.row_m[K + 1 + i])) / sh.row_z[K + 1 + i];
        rejected = !(uno::uniform24(words.x) * qq < pp);
        if (outputs && P.p_at_draft) P.p_at_draft[static_cast<size_t>(b) * K + i] = pp;
        if (outputs && P.q_at_draft) P.q_at_draft[static_cast<size_t>(b) * K + i] = qq;
      }
    }
    const unsigned ballot = __ballot_sync(0xFFFFFFFFu, rejected);
    if (ballot && (tid & 31) == 0) atomicMin(&sh.first_reject, (tid & ~31) + __ffs(ballot) - 1);
  }
  __syncthreads();
  const int n = sh.first_reject;
  if (outputs && sh.invalid) {
    int32_t* out = P.out_tokens + static_cast<size_t>(b) * (K + 1);
    for (int i = tid; i <= K; i += kThreads) out[i] = -1;
    if (tid == 0) P.accepted_len[b] = -1;
  }
  if (tid == 0) {
    Decision d{};
    d.n = n;
    d.invalid = sh.invalid;
    d.mode = (n < K) ? 0 : 1;
    d.lp = static_cast<double>(sh.row_m[n]) + static_cast<double>(log2f(sh.row_z[n]));
    // a q row with no finite logit has q = 0 everywhere: max(0, p - q) = p
    if (n < K && !(sh.row_z[K + 1 + n] > 0.f)) d.mode = 1;
    if (d.mode == 0)
      d.lq = static_cast<double>(sh.row_m[K + 1 + n]) +
             static_cast<double>(log2f(sh.row_z[K + 1 + n]));
    sh.d = d;
  }
  __syncthreads();
}

// The LM-head path: one CTA per sequence decides and records the decision.
template <typename T>
__global__ void __launch_bounds__(kThreads) verify_decide_kernel(const VerifyParams P) {
  __shared__ DecideShared sh;
  uno::launch_dependents();
  uno::grid_dependency_wait();
  decide_sequence<T>(P, blockIdx.x, sh, true);
  if (threadIdx.x == 0) {
    P.decisions[blockIdx.x] = sh.d;
    P.draw_count[blockIdx.x] = 0;
  }
}

// ---- launch 2: the draw -------------------------------------------------------------------

// log2(e) as a float32 and the float32 of its remainder.
constexpr float kLog2eHi = 1.44269502162933349609375f;
constexpr float kLog2eLo = 1.925963033500011e-08f;

// The row's log2-sum-exp L as two floats, L = hi + lo to float64 accuracy.
struct SplitL {
  float hi, lo;
};
__device__ __forceinline__ SplitL split_l(double L) {
  SplitL v;
  v.hi = static_cast<float>(L);
  v.lo = static_cast<float>(L - static_cast<double>(v.hi));
  return v;
}

// Exponent argument l log2 e - L of a token in float32 (three roundings, each
// at most 2^-24 of |argument|, and no error from log2 e itself).
__device__ __forceinline__ float arg_of(float l, SplitL L) {
  return fmaf(l, kLog2eLo, fmaf(l, kLog2eHi, -L.hi)) - L.lo;
}

// Weight of a token: mode 0: max(0, p - q), both exponentials skipped when
// p <= q; mode 1: p. p = 2^(arg_p) on the SFU, the row's normalised
// probability (up to the streaming pass's float32 normaliser).
__device__ __forceinline__ float token_weight(int mode, SplitL Lp, SplitL Lq, float lp, float lq) {
  const float ap = arg_of(lp, Lp);
  if (mode) return uno::ex2(ap);
  const float aq = arg_of(lq, Lq);
  if (!(ap > aq)) return 0.f;
  return fmaxf(0.f, uno::ex2(ap) - uno::ex2(aq));
}

// Chunk sums of chunks c0 + w0, c0 + w0 + wstep, ... (< c1) of the draw rows,
// one warp per chunk: the vector path, VPL 16-byte vectors per lane and chunk,
// kMaxVecs (chunk, vector) pairs per lane in flight per row, all loads of a
// pass issued before any is used. A vector's weights are added in float32 as
// a balanced tree, vectors and lanes in float64.
template <typename T, int VPL>
__device__ void chunk_sums_vec(const VerifyParams& P, const Decision& d, const T* rp, const T* rq,
                               double* out, int c0, int c1, int w0, int wstep) {
  constexpr int kVec = Elem<T>::kVec;
  constexpr int kMaxVecs = 4;
  constexpr int kPerPass = kMaxVecs / VPL;  // chunks per pass
  const int lane = threadIdx.x & 31;
  const uint4* vp = reinterpret_cast<const uint4*>(rp);
  const uint4* vq = reinterpret_cast<const uint4*>(rq);
  const int cvec = P.chunk_len / kVec;  // vectors per chunk
  const int nvec_row = P.V / kVec;      // vectors per row (the last chunk may be partial)
  const SplitL Lp = split_l(d.lp), Lq = split_l(d.mode ? 0.0 : d.lq);
  for (int cb = c0 + w0; cb < c1; cb += wstep * kPerPass) {
    uint4 a[kMaxVecs], bq[kMaxVecs];
    bool in[kMaxVecs];
#pragma unroll
    for (int k = 0; k < kMaxVecs; ++k) {
      const int c = cb + (k / VPL) * wstep;
      const int vi = c * cvec + (k % VPL) * 32 + lane;
      in[k] = (c < c1) && (vi < nvec_row);
      a[k] = in[k] ? __ldg(vp + vi) : make_uint4(0, 0, 0, 0);
      bq[k] = (in[k] && d.mode == 0) ? __ldg(vq + vi) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int ci = 0; ci < kPerPass; ++ci) {
      const int c = cb + ci * wstep;
      double t = 0.0;
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        if (!in[ci * VPL + q]) continue;
        float fp[kVec], fq[kVec], w[kVec];
        Elem<T>::unpack(a[ci * VPL + q], fp);
        Elem<T>::unpack(bq[ci * VPL + q], fq);
#pragma unroll
        for (int e = 0; e < kVec; ++e) w[e] = token_weight(d.mode, Lp, Lq, fp[e], fq[e]);
#pragma unroll
        for (int st = 1; st < kVec; st *= 2) {
#pragma unroll
          for (int e = 0; e + st < kVec; e += 2 * st) w[e] += w[e + st];
        }
        t += w[0];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
      if (lane == 0 && c < c1) out[c] = t;
    }
  }
}

// Stages of a warp's copy ring for VPL vectors per lane and chunk (0: no ring).
__host__ __device__ constexpr int ring_stages(int vpl) { return vpl == 1 ? 4 : (vpl == 2 ? 3 : 0); }

// Shared-memory bytes of the draw CTA's copy ring.
__host__ __device__ constexpr int ring_bytes(int vpl) {
  return kWarps * ring_stages(vpl) * 2 * vpl * 32 * 16;
}

// The vector path of chunk_sums through a ring of D shared-memory stages per
// warp, one chunk of both draw rows per stage: while a chunk's weights are
// computed, the copies of the next D - 1 chunks are in flight (cp.async), so
// the loads overlap the SFU work. Each lane copies and reads back only its own
// 16-byte slots; a stage is refilled only after the lane has read it.
template <typename T, int VPL>
__device__ void chunk_sums_ring(const VerifyParams& P, const Decision& d, const T* rp, const T* rq,
                                double* out, int c0, int c1, int w0, int wstep, uint4* ring) {
  constexpr int kVec = Elem<T>::kVec;
  constexpr int D = ring_stages(VPL);
  constexpr int kStage = 2 * VPL * 32;  // 16-byte slots per stage and warp
  const int lane = threadIdx.x & 31;
  uint4* my = ring + (threadIdx.x >> 5) * (D * kStage);
  const uint4* vp = reinterpret_cast<const uint4*>(rp);
  const uint4* vq = reinterpret_cast<const uint4*>(rq);
  const int cvec = P.chunk_len / kVec;
  const int nvec_row = P.V / kVec;
  const bool two = (d.mode == 0);
  const int first = c0 + w0;
  const int nk = (first < c1) ? (c1 - first + wstep - 1) / wstep : 0;
  const SplitL Lp = split_l(d.lp), Lq = split_l(two ? d.lq : 0.0);
  // every call commits one group per chunk slot, empty past the end, so that
  // wait<D - 1> always refers to the chunk about to be used
  auto issue = [&](int k) {
    if (k < nk) {
      const int c = first + k * wstep;
      uint4* dst = my + (k % D) * kStage;
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        const int vi = c * cvec + q * 32 + lane;
        if (vi < nvec_row) {
          uno::cp_async16(dst + q * 32 + lane, vp + vi);
          if (two) uno::cp_async16(dst + (VPL + q) * 32 + lane, vq + vi);
        }
      }
    }
    uno::cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < D - 1; ++k) issue(k);
  for (int k = 0; k < nk; ++k) {
    issue(k + D - 1);
    uno::cp_async_wait<D - 1>();
    const int c = first + k * wstep;
    const uint4* src = my + (k % D) * kStage;
    double t = 0.0;
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int vi = c * cvec + q * 32 + lane;
      if (vi < nvec_row) {
        float fp[kVec], fq[kVec], w[kVec];
        Elem<T>::unpack(src[q * 32 + lane], fp);
        Elem<T>::unpack(two ? src[(VPL + q) * 32 + lane] : make_uint4(0, 0, 0, 0), fq);
#pragma unroll
        for (int e = 0; e < kVec; ++e) w[e] = token_weight(d.mode, Lp, Lq, fp[e], fq[e]);
#pragma unroll
        for (int st = 1; st < kVec; st *= 2) {
#pragma unroll
          for (int e = 0; e + st < kVec; e += 2 * st) w[e] += w[e + st];
        }
        t += w[0];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
    if (lane == 0) out[c] = t;
  }
  uno::cp_async_wait<0>();  // nothing in flight once the ring is reused or left
}

// Chunk sums of chunks c0 + w0, c0 + w0 + wstep, ... (< c1): 16-byte vectors
// when both rows are 16-byte aligned and V and the chunk length are whole
// vectors (through the copy ring when `ring` is given and the chunk is one or
// two vectors per lane), otherwise scalar loads.
template <typename T>
__device__ void chunk_sums(const VerifyParams& P, int b, const Decision& d, const T* rp,
                           const T* rq, int c0, int c1, int w0, int wstep, uint4* ring) {
  constexpr int kVec = Elem<T>::kVec;
  const int lane = threadIdx.x & 31;
  double* out = P.chunk_sums + static_cast<size_t>(b) * P.nchunks;
  const int vpl = P.chunk_len / (32 * kVec);  // vectors per lane per chunk
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(rp) | reinterpret_cast<uintptr_t>(rq)) & 15) == 0 &&
                      (P.V % kVec) == 0 && (P.chunk_len % (32 * kVec)) == 0;
  if (vec_ok && ring && vpl == 1)
    return chunk_sums_ring<T, 1>(P, d, rp, rq, out, c0, c1, w0, wstep, ring);
  if (vec_ok && ring && vpl == 2)
    return chunk_sums_ring<T, 2>(P, d, rp, rq, out, c0, c1, w0, wstep, ring);
  if (vec_ok && vpl == 1) return chunk_sums_vec<T, 1>(P, d, rp, rq, out, c0, c1, w0, wstep);
  if (vec_ok && vpl == 2) return chunk_sums_vec<T, 2>(P, d, rp, rq, out, c0, c1, w0, wstep);
  if (vec_ok && vpl == 4) return chunk_sums_vec<T, 4>(P, d, rp, rq, out, c0, c1, w0, wstep);
  const SplitL Lp = split_l(d.lp), Lq = split_l(d.mode ? 0.0 : d.lq);
  for (int c = c0 + w0; c < c1; c += wstep) {
    const int v0 = c * P.chunk_len;
    const int v1 = min(v0 + P.chunk_len, P.V);
    double acc = 0.0;
    for (int v = v0 + lane; v < v1; v += 32)
      acc += token_weight(d.mode, Lp, Lq, Elem<T>::at(rp, v), d.mode ? 0.f : Elem<T>::at(rq, v));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) out[c] = acc;
  }
}

struct DrawShared {
  double warp_tot[kWarps];
  double total;
  double carry;
  int is_last, chunk, last_chunk, token_min, last_in_chunk;
};

// Exclusive running sum (float64, index order) of per-thread values across the
// CTA; also leaves the grand total in sh.total.
__device__ double block_exclusive_scan(double mine, DrawShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double up = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += up;
  }
  if (lane == 31) sh.warp_tot[warp] = incl;
  __syncthreads();
  double before = 0.0;
  for (int w = 0; w < warp; ++w) before += sh.warp_tot[w];
  if (threadIdx.x == kThreads - 1) sh.total = before + incl;
  __syncthreads();
  return before + incl - mine;
}

template <typename T>
__device__ __forceinline__ double weight_at(const Decision& d, SplitL Lp, SplitL Lq, const T* rp,
                                            const T* rq, int v) {
  return token_weight(d.mode, Lp, Lq, Elem<T>::at(rp, v), d.mode ? 0.f : Elem<T>::at(rq, v));
}

// Largest index with positive weight in chunk c (the whole CTA), or -1.
template <typename T>
__device__ int last_positive_in_chunk(const VerifyParams& P, const Decision& d, const T* rp,
                                      const T* rq, int c, DrawShared& sh) {
  const SplitL Lp = split_l(d.lp), Lq = split_l(d.mode ? 0.0 : d.lq);
  if (threadIdx.x == 0) sh.last_in_chunk = -1;
  __syncthreads();
  const int v0 = c * P.chunk_len, v1 = min(v0 + P.chunk_len, P.V);
  for (int v = v0 + threadIdx.x; v < v1; v += kThreads)
    if (weight_at<T>(d, Lp, Lq, rp, rq, v) > 0.0) atomicMax(&sh.last_in_chunk, v);
  __syncthreads();
  return sh.last_in_chunk;
}

// Final inverse-CDF step of sequence b (the whole CTA); returns the token.
// Thread t takes the sums of chunks [t * per, (t + 1) * per) (read twice).
template <typename T>
__device__ int finish_draw(const VerifyParams& P, int b, Decision d, const T* rp, const T* rq,
                           DrawShared& sh, uint4* ring) {
  const int tid = threadIdx.x;
  const double* cs = P.chunk_sums + static_cast<size_t>(b) * P.nchunks;
  const float u = uno::uniform24(uno::verify_block_words(P.seed, P.step, b, d.n).y);
  const int per = (P.nchunks + kThreads - 1) / kThreads;
  const int c0 = min(tid * per, P.nchunks), c1 = min(c0 + per, P.nchunks);
  constexpr int kKeep = 4;  // a thread's chunk sums kept in registers (more are reloaded)
  double keep[kKeep];
  double before = 0.0;
  for (int pass = 0; pass < 2; ++pass) {
    double mine = 0.0;
#pragma unroll
    for (int k = 0; k < kKeep; ++k) {
      keep[k] = (c0 + k < c1) ? __ldcg(cs + c0 + k) : 0.0;
      mine += keep[k];
    }
    for (int c = c0 + kKeep; c < c1; ++c) mine += __ldcg(cs + c);
    before = block_exclusive_scan(mine, sh);
    if (sh.total > 0.0 || d.mode == 1) break;
    // The residual mass is zero (possible only through rounding): draw from p_n.
    d.mode = 1;
    rq = rp;
    chunk_sums<T>(P, b, d, rp, rp, 0, P.nchunks, threadIdx.x >> 5, kWarps, ring);
    __threadfence();
    __syncthreads();
  }
  if (tid == 0) {
    sh.chunk = INT_MAX;
    sh.last_chunk = -1;
    sh.token_min = INT_MAX;
    sh.last_in_chunk = -1;
  }
  __syncthreads();
  const double t = static_cast<double>(u) * sh.total;
  {
    double run = before;
    int found = -1, last_pos_chunk = -1;
    for (int c = c0; c < c1; ++c) {
      double w = 0.0;
#pragma unroll
      for (int k = 0; k < kKeep; ++k)
        if (c == c0 + k) w = keep[k];
      if (c >= c0 + kKeep) w = __ldcg(cs + c);
      const double nxt = run + w;
      if (found < 0 && nxt > t) found = c;
      if (w > 0.0) last_pos_chunk = c;
      if (found < 0) run = nxt;
    }
    if (found >= 0) atomicMin(&sh.chunk, found);
    if (last_pos_chunk >= 0) atomicMax(&sh.last_chunk, last_pos_chunk);
    __syncthreads();
    if (found >= 0 && found == sh.chunk) sh.carry = run;  // running sum before that chunk
  }
  __syncthreads();
  const int ch = sh.chunk;
  if (ch == INT_MAX) {
    // Rounding left no crossing: the largest index with positive weight.
    return (sh.last_chunk >= 0) ? last_positive_in_chunk<T>(P, d, rp, rq, sh.last_chunk, sh) : -1;
  }
  // Within the chunk, token by token from the running sum before it; if the
  // chunk's weights end before the threshold (summation order), its last
  // token with positive weight is taken.
  const SplitL Lp = split_l(d.lp), Lq = split_l(d.mode ? 0.0 : d.lq);
  double carry = sh.carry;
  const int v0 = ch * P.chunk_len, v1 = min(v0 + P.chunk_len, P.V);
  for (int base = v0; base < v1; base += kThreads) {
    const int v = base + tid;
    const double w = (v < v1) ? weight_at<T>(d, Lp, Lq, rp, rq, v) : 0.0;
    const double bef = carry + block_exclusive_scan(w, sh);
    if ((w > 0.0) && (bef + w > t)) atomicMin(&sh.token_min, v);
    if (w > 0.0) atomicMax(&sh.last_in_chunk, v);
    carry += sh.total;
    __syncthreads();
    if (sh.token_min != INT_MAX) break;
  }
  return (sh.token_min != INT_MAX) ? sh.token_min : sh.last_in_chunk;
}

// DECIDE: each CTA decides its sequence from the slab partials (the first of
// a sequence's CTAs also writes the decision's outputs); otherwise the
// decision launch recorded it.
template <typename T, bool DECIDE>
__global__ void __launch_bounds__(kThreads, kDrawCtasPerSm) verify_draw_kernel(const VerifyParams P) {
  __shared__ DrawShared sh;
  __shared__ DecideShared dsh;
  extern __shared__ __align__(16) uint4 ring_smem[];  // ring_bytes(vpl) bytes, or none
  uint4* ring = P.ring ? ring_smem : nullptr;
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int tid = threadIdx.x, warp = tid >> 5;
  const int b = blockIdx.x / P.SD, du = blockIdx.x % P.SD;
  const int K = P.K;
  if constexpr (DECIDE) {
    decide_sequence<T>(P, b, dsh, du == 0);
  } else {
    if (tid == 0) dsh.d = P.decisions[b];
    if (tid < K) dsh.x[tid] = P.draft[static_cast<size_t>(b) * K + tid];
    __syncthreads();
  }
  const Decision d = dsh.d;
  if (d.invalid) return;  // the decision wrote this sequence's outputs
  size_t off;
  const T* rp = row_ptr<T>(P, b, d.n, &off);
  const T* rq = (d.mode == 0) ? row_ptr<T>(P, b, K + 1 + d.n, &off) : rp;
  const int per_cta = (P.nchunks + P.SD - 1) / P.SD;
  const int c0 = du * per_cta;
  const int c1 = min(c0 + per_cta, P.nchunks);
  chunk_sums<T>(P, b, d, rp, rq, c0, c1, warp, kWarps, ring);
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    sh.is_last = (atomicAdd(P.draw_count + b, 1) == P.SD - 1);
  }
  __syncthreads();
  if (!sh.is_last) return;

  // the CTA that completes the sequence picks the token and writes outputs
  __threadfence();
  const int y = finish_draw<T>(P, b, d, rp, rq, sh, ring);
  const int n = d.n;
  int32_t* out = P.out_tokens + static_cast<size_t>(b) * (K + 1);
  for (int i = tid; i <= K; i += kThreads) out[i] = (i < n) ? dsh.x[i] : ((i == n) ? y : -1);
  if (tid == 0) P.accepted_len[b] = n;
}

// ---- host side -----------------------------------------------------------------------

struct Geometry {
  int S, nchunks, chunk_len, SD;
  long long stream_ctas, draw_ctas;
  size_t off_counts, off_decisions, off_partials, off_chunks, off_xlogit, bytes;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool verify_sizes_ok(int B, int K, int V, int dtype) {
  return (dtype == UNO_BF16 || dtype == UNO_F32) && B >= 0 && B <= (1 << 20) && K >= 1 &&
         K <= kMaxK && V >= 1 && V <= (1 << 28);
}

// Slabs, chunks and the workspace layout: a function of (B, K, V, dtype) only.
Geometry geometry(int B, int K, int V, int dtype) {
  Geometry g{};
  const size_t esize = (dtype == UNO_BF16) ? 2 : 4;
  const long long rows = static_cast<long long>(B) * (2 * K + 1);
  const size_t row_bytes = static_cast<size_t>(V) * esize;
  long long s = static_cast<long long>((row_bytes + kSlabBytes - 1) / kSlabBytes);
  // at least one wave of stream CTAs; two waves of the smaller slabs this
  // gives few rows were measured slower (B = 1, K = 16: 25.6 against 21.5 us
  // per call; B = 4 to 64 unchanged)
  const long long want = static_cast<long long>(kSizingSms) * kStreamCtasPerSm;
  if (rows > 0 && s * rows < want) s = (want + rows - 1) / rows;
  long long smax = static_cast<long long>(row_bytes / kMinSlabBytes);
  if (smax < 1) smax = 1;
  if (s > smax) s = smax;
  if (s < 1) s = 1;
  g.S = static_cast<int>(s);
  int cl = (V + kMaxChunks - 1) / kMaxChunks;
  cl = ((cl + kChunkMin - 1) / kChunkMin) * kChunkMin;
  if (cl < kChunkMin) cl = kChunkMin;
  g.chunk_len = cl;
  g.nchunks = (V + cl - 1) / cl;
  // draw CTAs per sequence: at most one wave in total (a second, partial wave
  // would double the time of the sequences it holds), at least 8 chunks each
  long long sd = (B > 0) ? kDrawCtasTarget / B : 1;
  const long long sd_max = (g.nchunks + 7) / 8;
  if (sd > sd_max) sd = sd_max;
  if (sd < 1) sd = 1;
  g.SD = static_cast<int>(sd);
  g.stream_ctas = rows * g.S;
  g.draw_ctas = static_cast<long long>(B) * g.SD;
  g.off_counts = 0;
  g.off_decisions = align_up(sizeof(int) * static_cast<size_t>(B), 256);
  g.off_partials = align_up(g.off_decisions + sizeof(Decision) * static_cast<size_t>(B), 256);
  g.off_chunks =
      align_up(g.off_partials + sizeof(Partial) * static_cast<size_t>(g.stream_ctas), 256);
  g.off_xlogit = align_up(g.off_chunks + sizeof(double) * static_cast<size_t>(B) * g.nchunks, 256);
  g.bytes = align_up(g.off_xlogit + sizeof(float) * static_cast<size_t>(rows), 256);
  return g;
}

// Launch with programmatic stream serialisation: the kernel's CTAs may start
// while the previous kernel on the stream finishes (each waits for it before
// touching global memory).
template <typename Kern>
int launch_pdl(Kern kern, long long grid, cudaStream_t st, const VerifyParams& P,
               int smem_bytes = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P) == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

// The draw kernel's dynamic shared memory: the copy ring, opted in above the
// default 48 KB limit once per kernel instantiation and device.
constexpr int kMaxDevices = 64;
template <typename T, bool DECIDE>
bool allow_draw_smem(int bytes) {
  static std::atomic<int> allowed[kMaxDevices];  // zero-initialised (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::atomic<int>* a = (dev >= 0 && dev < kMaxDevices) ? &allowed[dev] : nullptr;
  if (a && bytes <= a->load()) return true;
  if (cudaFuncSetAttribute(verify_draw_kernel<T, DECIDE>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  if (a) a->store(bytes);
  return true;
}

template <typename T>
int launch(VerifyParams P, const Geometry& g, cudaStream_t st) {
  const int vpl = P.chunk_len / (32 * Elem<T>::kVec);
  const int smem = ring_bytes(vpl);
  P.ring = smem > 0;
  if (P.ext_p == nullptr) {
    if (!allow_draw_smem<T, true>(smem)) return UNO_ERR_CUDA;
    if (launch_pdl(verify_stream_kernel<T>, g.stream_ctas, st, P) != UNO_OK) return UNO_ERR_CUDA;
    if (launch_pdl(verify_draw_kernel<T, true>, g.draw_ctas, st, P, smem) != UNO_OK)
      return UNO_ERR_CUDA;
  } else {
    if (!allow_draw_smem<T, false>(smem)) return UNO_ERR_CUDA;
    if (launch_pdl(verify_decide_kernel<T>, P.B, st, P) != UNO_OK) return UNO_ERR_CUDA;
    if (launch_pdl(verify_draw_kernel<T, false>, g.draw_ctas, st, P, smem) != UNO_OK)
      return UNO_ERR_CUDA;
  }
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}

}  // namespace

extern "C" size_t uno_verify_workspace_bytes(int B, int K, int V, int dtype) {
  if (!verify_sizes_ok(B, K, V, dtype)) return 0;
  return geometry(B, K, V, dtype).bytes;
}

extern "C" int uno_verify_block(const void* p_logits, const void* q_logits,
                                const int32_t* draft_tokens, int B, int K, int V, int dtype,
                                uint64_t seed, uint64_t step, int32_t* out_tokens,
                                int32_t* accepted_len, float* p_at_draft, float* q_at_draft,
                                float* row_lse, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (!verify_sizes_ok(B, K, V, dtype)) return UNO_ERR_SIZE;
  if (B == 0) return UNO_OK;
  if (!p_logits || !q_logits || !draft_tokens || !out_tokens || !accepted_len)
    return UNO_ERR_NULL;
  if (!workspace) return UNO_ERR_WORKSPACE;
  if (!uno_host::aligned(p_logits, 16) || !uno_host::aligned(q_logits, 16) ||
      !uno_host::aligned(workspace, 16) || !uno_host::aligned(draft_tokens, 4) ||
      !uno_host::aligned(out_tokens, 4) || !uno_host::aligned(accepted_len, 4) ||
      !uno_host::aligned(p_at_draft, 4) || !uno_host::aligned(q_at_draft, 4) ||
      !uno_host::aligned(row_lse, 4))
    return UNO_ERR_ALIGN;
  const Geometry g = geometry(B, K, V, dtype);
  if (workspace_bytes < g.bytes) return UNO_ERR_WORKSPACE;
  if (g.stream_ctas > INT_MAX || g.draw_ctas > INT_MAX) return UNO_ERR_SIZE;
  const int dev_status = uno_host::check_device();
  if (dev_status != UNO_OK) return dev_status;

  char* ws = static_cast<char*>(workspace);
  VerifyParams P;
  P.p_logits = p_logits;
  P.q_logits = q_logits;
  P.draft = draft_tokens;
  P.B = B;
  P.K = K;
  P.V = V;
  P.S = g.S;
  P.nchunks = g.nchunks;
  P.chunk_len = g.chunk_len;
  P.SD = g.SD;
  P.seed = seed;
  P.step = step;
  P.out_tokens = out_tokens;
  P.accepted_len = accepted_len;
  P.p_at_draft = p_at_draft;
  P.q_at_draft = q_at_draft;
  P.row_lse = row_lse;
  P.draw_count = reinterpret_cast<int*>(ws + g.off_counts);
  P.decisions = reinterpret_cast<Decision*>(ws + g.off_decisions);
  P.partials = reinterpret_cast<Partial*>(ws + g.off_partials);
  P.chunk_sums = reinterpret_cast<double*>(ws + g.off_chunks);
  P.draft_logit = reinterpret_cast<float*>(ws + g.off_xlogit);
  P.q_rows = K;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (dtype == UNO_BF16) ? launch<uint16_t>(P, g, st) : launch<float>(P, g, st);
}

extern "C" int uno_verify_block_head(const void* y_ar, const void* y_draft, const float* stats_ar,
                                     const float* stats_draft, int stats_tiles,
                                     const int32_t* draft_tokens, int B, int K, int V, int dtype,
                                     uint64_t seed, uint64_t step, int32_t* out_tokens,
                                     int32_t* accepted_len, float* p_at_draft, float* q_at_draft,
                                     float* row_lse, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  if (!verify_sizes_ok(B, K, V, dtype) || stats_tiles < 1 || stats_tiles > (1 << 20))
    return UNO_ERR_SIZE;
  if (B == 0) return UNO_OK;
  if (!y_ar || !y_draft || !stats_ar || !stats_draft || !draft_tokens || !out_tokens ||
      !accepted_len)
    return UNO_ERR_NULL;
  if (!workspace) return UNO_ERR_WORKSPACE;
  if (!uno_host::aligned(y_ar, 16) || !uno_host::aligned(y_draft, 16) ||
      !uno_host::aligned(stats_ar, 8) || !uno_host::aligned(stats_draft, 8) ||
      !uno_host::aligned(workspace, 16) || !uno_host::aligned(draft_tokens, 4) ||
      !uno_host::aligned(out_tokens, 4) || !uno_host::aligned(accepted_len, 4) ||
      !uno_host::aligned(p_at_draft, 4) || !uno_host::aligned(q_at_draft, 4) ||
      !uno_host::aligned(row_lse, 4))
    return UNO_ERR_ALIGN;
  const Geometry g = geometry(B, K, V, dtype);
  if (workspace_bytes < g.bytes) return UNO_ERR_WORKSPACE;
  if (g.draw_ctas > INT_MAX) return UNO_ERR_SIZE;
  const int dev_status = uno_host::check_device();
  if (dev_status != UNO_OK) return dev_status;

  char* ws = static_cast<char*>(workspace);
  VerifyParams P;
  P.p_logits = y_ar;
  P.q_logits = y_draft;
  P.draft = draft_tokens;
  P.B = B;
  P.K = K;
  P.V = V;
  P.S = g.S;
  P.nchunks = g.nchunks;
  P.chunk_len = g.chunk_len;
  P.SD = g.SD;
  P.seed = seed;
  P.step = step;
  P.out_tokens = out_tokens;
  P.accepted_len = accepted_len;
  P.p_at_draft = p_at_draft;
  P.q_at_draft = q_at_draft;
  P.row_lse = row_lse;
  P.draw_count = reinterpret_cast<int*>(ws + g.off_counts);
  P.decisions = reinterpret_cast<Decision*>(ws + g.off_decisions);
  P.partials = reinterpret_cast<Partial*>(ws + g.off_partials);
  P.chunk_sums = reinterpret_cast<double*>(ws + g.off_chunks);
  P.q_rows = K + 1;
  P.ext_p = reinterpret_cast<const Partial*>(stats_ar);
  P.ext_q = reinterpret_cast<const Partial*>(stats_draft);
  P.ext_T = stats_tiles;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (dtype == UNO_BF16) ? launch<uint16_t>(P, g, st) : launch<float>(P, g, st);
}
