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
// Three launches per call; no CTA ever waits for another:
//  1. verify_stream_kernel streams every logit row once. One CTA per slab
//     (up to 256 KB of one row, a whole number of 16 KB rounds) issues 16-byte
//     loads, four per thread in flight plus the next four prefetched, folds
//     them into a running (reference, sum of 2^(x - reference)) in the log2
//     domain and writes one partial per slab. Nothing else happens on this
//     path.
//  2. verify_decide_kernel, one CTA per sequence, merges the slab partials of
//     the sequence's 2K+1 rows in slab order, evaluates the accept tests with
//     Philox uniforms, finds the first rejection by ballot and records what the
//     draw needs (which rows, their statistics).
//  3. verify_draw_kernel runs SD CTAs per sequence; each sums the residual
//     weights max(0, p_n - q_n) (or the bonus row p_K) over its range of
//     fixed-size vocabulary chunks with 16-byte loads. The CTA that completes a
//     sequence (atomic counter) takes the float64 running sum of the chunk
//     sums, finds the chunk where u' * total is crossed, scans it with warp
//     prefix sums to pick the token and writes the outputs.
#include <atomic>
#include <cfloat>
#include <climits>
#include <cstdint>
#include <cstdio>

#include <cuda_runtime.h>

#include "uno.h"
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
constexpr int kChunkMin = 256;            // vocabulary entries per inverse-CDF chunk
constexpr int kMaxChunks = 4096;          // chunks per row (the chunk length grows beyond)
constexpr int kDrawCtasPerSm = 2;
constexpr int kDrawCtasTarget = 148 * kDrawCtasPerSm;  // one wave of draw CTAs
constexpr int kSizingSms = 148;           // fixed, so the workspace size is device-independent
constexpr float kLog2e = 1.4426950408889634f;
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
  float mp, izp, mq, izq;  // draw rows: reference (log2 domain) and 1 / sum
  float c;                 // residual sign threshold (log2 domain)
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
  Partial* partials;  // [B][2K+1][S]
  float* chunk_sums;  // [B][nchunks]
  int* draw_count;    // [B], set to 0 by the decision launch
  Decision* decisions;  // [B]
  // Rows of q per sequence in memory: K (q is [B][K][V]) or K+1 (q is the
  // draft-pathway output of the same B x (K+1) rows as p, bonus rows unused).
  int q_rows = 0;
  // Row statistics written by the LM-head GEMM (null: the stream launch
  // computes them): ext_T partials per logit row, in the partial convention.
  const Partial* ext_p = nullptr;  // [B][K+1][ext_T]
  const Partial* ext_q = nullptr;  // [B][q_rows][ext_T]
  int ext_T = 0;
};

// ---- element access -----------------------------------------------------------

template <typename T>
struct Elem;

template <>
struct Elem<uint16_t> {  // bfloat16 bits
  static constexpr int kVec = 8;
  __device__ static __forceinline__ float at(const uint16_t* p, size_t i) {
    return uno::bf16_bits_to_float(__ldg(p + i));
  }
  __device__ static __forceinline__ void unpack(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};

template <>
struct Elem<float> {
  static constexpr int kVec = 4;
  __device__ static __forceinline__ float at(const float* p, size_t i) { return __ldg(p + i); }
  __device__ static __forceinline__ void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
};

// ---- (max, sum-exp) algebra in the log2 domain ----------------------------------

__device__ __forceinline__ void merge(float& m, float& z, float m2, float z2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;  // both empty
  const float a = (m == -INFINITY) ? 0.f : z * uno::ex2(m - mm);
  const float b = (m2 == -INFINITY) ? 0.f : z2 * uno::ex2(m2 - mm);
  m = mm;
  z = a + b;
}

// Fold N natural-log logits into the running (m, z). m is a reference, not
// necessarily the running maximum: z = sum of 2^(x - m) over the values seen,
// x = l * log2(e). The common path adds the group's sum against the current
// reference; only when that sum reaches 2^70 (or is not finite, e.g. while m
// is still -inf) does the group move the reference to its own maximum. So every
// term stays below 2^70 and z below 2^84, and a term that underflows against
// the reference is below 2^-126 of it, hence negligible against the true
// maximum. Merges and p = 2^(x - m) / z do not depend on which reference is
// kept.
template <int N>
__device__ __forceinline__ float sum_ex2(const float* v, float m) {
  float t[N];
#pragma unroll
  for (int e = 0; e < N; ++e) t[e] = uno::ex2(fmaf(v[e], kLog2e, -m));
#pragma unroll
  for (int w = 1; w < N; w *= 2) {
#pragma unroll
    for (int e = 0; e + w < N; e += 2 * w) t[e] += t[e + w];
  }
  return t[0];
}

template <int N>
__device__ __forceinline__ void fold(float& m, float& z, const float* v) {
  const float s = sum_ex2<N>(v, m);
  if (s < 0x1p70f) {  // false for inf and NaN
    z += s;
    return;
  }
  float gm = v[0];
#pragma unroll
  for (int e = 1; e < N; ++e) gm = fmaxf(gm, v[e]);
  if (gm == -INFINITY) return;
  gm *= kLog2e;
  if (gm > m) {
    z = (m == -INFINITY) ? 0.f : z * uno::ex2(m - gm);
    m = gm;
  }
  z += sum_ex2<N>(v, m);
}

__device__ __forceinline__ void warp_merge(float& m, float& z) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    const float z2 = __shfl_xor_sync(0xFFFFFFFFu, z, o);
    merge(m, z, m2, z2);
  }
}

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
    if (base + kStep <= v1) {  // a full round: no predication
#pragma unroll
      for (int k = 0; k < kRound; k += 2) {
        float f[2 * kVec];
        Elem<T>::unpack(cur[k], f);
        Elem<T>::unpack(cur[k + 1], f + kVec);
        fold<2 * kVec>(m, z, f);
      }
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
    if (lane == 0) P.partials[static_cast<size_t>(blockIdx.x)] = Partial{m, z};
  }
}

// ---- launch 2: decision and draw ----------------------------------------------------------

using DrawRows = Decision;

// Weight of token v. mode 0: max(0, p(v) - q(v)), skipping both exponentials
// where the log-domain test shows p(v) < q(v) by a clear margin; mode 1: p(v).
template <typename T>
__device__ __forceinline__ float weight(const DrawRows& d, const T* rp, const T* rq, int v) {
  const float lp = Elem<T>::at(rp, v) * kLog2e;
  if (d.mode) return uno::ex2(lp - d.mp) * d.izp;
  const float lq = Elem<T>::at(rq, v) * kLog2e;
  if (lp - lq < d.c - 1e-3f) return 0.f;
  const float pv = uno::ex2(lp - d.mp) * d.izp;
  const float qv = uno::ex2(lq - d.mq) * d.izq;
  return fmaxf(0.f, pv - qv);
}

// Sums of chunks c0 + w0, c0 + w0 + wstep, ... (< c1) of the draw rows of
// sequence b, one warp per chunk, stored to the workspace. Returns this lane's
// largest positive-weight index, or -1. When both rows are 16-byte aligned and
// V and the chunk length are whole vectors, each lane loads 16-byte vectors,
// all of the warp's chunks at once; otherwise it falls back to scalar loads.
template <typename T>
__device__ int chunk_sums(const VerifyParams& P, int b, const DrawRows& d, const T* rp,
                          const T* rq, int c0, int c1, int w0, int wstep) {
  constexpr int kVec = Elem<T>::kVec;
  constexpr int kMaxVecs = 8;  // vectors per lane held in flight per row
  const int lane = threadIdx.x & 31;
  int last = -1;
  const int vpl = P.chunk_len / (32 * kVec);  // vectors per lane per chunk
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(rp) | reinterpret_cast<uintptr_t>(rq)) & 15) == 0 &&
                      (P.V % kVec) == 0 && (P.chunk_len % (32 * kVec)) == 0 && vpl >= 1 &&
                      vpl <= kMaxVecs;
  if (vec_ok) {
    const uint4* vp = reinterpret_cast<const uint4*>(rp);
    const uint4* vq = reinterpret_cast<const uint4*>(rq);
    const int cvec = P.chunk_len / kVec;  // vectors per chunk
    const int nvec_row = P.V / kVec;      // vectors per row (V is a multiple of kVec here)
    // Each pass covers up to kMaxVecs (chunk, vector) pairs per lane: all loads
    // of a pass are issued before any is used.
    const int per_pass_chunks = max(1, kMaxVecs / vpl);
    for (int cb = c0 + w0; cb < c1; cb += wstep * per_pass_chunks) {
      uint4 a[kMaxVecs], bq[kMaxVecs];
#pragma unroll
      for (int k = 0; k < kMaxVecs; ++k) {
        const int c = cb + (k / vpl) * wstep;
        const int q = k % vpl;
        const int vi = c * cvec + q * 32 + lane;
        const bool in = (k < per_pass_chunks * vpl) && (c < c1) && (q < vpl) && (vi < nvec_row);
        a[k] = in ? __ldg(vp + vi) : make_uint4(0, 0, 0, 0);
        bq[k] = (in && d.mode == 0) ? __ldg(vq + vi) : make_uint4(0, 0, 0, 0);
      }
      float s[kMaxVecs / 1];
#pragma unroll
      for (int k = 0; k < kMaxVecs; ++k) {
        const int c = cb + (k / vpl) * wstep;
        const int q = k % vpl;
        s[k] = 0.f;
        const int vi = c * cvec + q * 32 + lane;
        if (!((k < per_pass_chunks * vpl) && (c < c1) && (q < vpl) && (vi < nvec_row))) continue;
        float fp[kVec], fq[kVec];
        Elem<T>::unpack(a[k], fp);
        Elem<T>::unpack(bq[k], fq);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          float w;
          const float lp = fp[e] * kLog2e;
          if (d.mode) {
            w = uno::ex2(lp - d.mp) * d.izp;
          } else {
            const float lq = fq[e] * kLog2e;
            w = (lp - lq < d.c - 1e-3f)
                    ? 0.f
                    : fmaxf(0.f, uno::ex2(lp - d.mp) * d.izp - uno::ex2(lq - d.mq) * d.izq);
          }
          s[k] += w;
          if (w > 0.f) last = max(last, vi * kVec + e);
        }
      }
      // one sum per chunk of this pass
#pragma unroll
      for (int k0 = 0; k0 < kMaxVecs; k0 += 1) {
        if (k0 % vpl != 0 || k0 >= per_pass_chunks * vpl) continue;
        float t = 0.f;
        for (int q = 0; q < vpl && k0 + q < kMaxVecs; ++q) t += s[k0 + q];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
        const int c = cb + (k0 / vpl) * wstep;
        if (lane == 0 && c < c1) P.chunk_sums[static_cast<size_t>(b) * P.nchunks + c] = t;
      }
    }
    return last;
  }
  for (int c = c0 + w0; c < c1; c += wstep) {
    const int v0 = c * P.chunk_len;
    const int v1 = min(v0 + P.chunk_len, P.V);
    float s = 0.f;
    for (int base = v0; base < v1; base += 32 * 8) {
      float w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int v = base + k * 32 + lane;
        w[k] = (v < v1) ? weight<T>(d, rp, rq, v) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        s += w[k];
        if (w[k] > 0.f) last = max(last, base + k * 32 + lane);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane == 0) P.chunk_sums[static_cast<size_t>(b) * P.nchunks + c] = s;
  }
  return last;
}

// ---- launch 2: the decision of each sequence (one CTA per sequence) ---------------------

struct DecideShared {
  float row_m[kMaxRows], row_z[kMaxRows];
  int first_reject, invalid;
};

template <typename T>
__global__ void __launch_bounds__(kThreads) verify_decide_kernel(const VerifyParams P) {
  __shared__ DecideShared sh;
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int tid = threadIdx.x;
  const int b = blockIdx.x;
  const int K = P.K, R = 2 * K + 1, S = P.S, V = P.V;

  // row statistics: merge the slab partials of every row in slab order
  if (P.ext_p == nullptr) {
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
      if (P.row_lse) P.row_lse[static_cast<size_t>(b) * R + j] = (m + log2f(z)) * kLn2;
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
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
        const float z2 = __shfl_xor_sync(0xFFFFFFFFu, z, o);
        merge(m, z, m2, z2);
      }
      if (lane == 0) {
        sh.row_m[j] = m;
        sh.row_z[j] = z;
        if (P.row_lse) P.row_lse[static_cast<size_t>(b) * R + j] = (m + log2f(z)) * kLn2;
      }
    }
  }
  if (tid == 0) {
    sh.first_reject = K;
    sh.invalid = 0;
    P.draw_count[b] = 0;
  }
  __syncthreads();

  // accept tests, one thread per position; first rejection by ballot
  for (int i0 = 0; i0 < K; i0 += kThreads) {
    const int i = i0 + tid;
    bool rejected = false;
    if (i < K) {
      const int x = P.draft[static_cast<size_t>(b) * K + i];
      if (x < 0 || x >= V) {
        atomicOr(&sh.invalid, 1);
      } else {
        size_t off;
        const T* rp = row_ptr<T>(P, b, i, &off);
        const T* rq = row_ptr<T>(P, b, K + 1 + i, &off);
        const float pp = uno::ex2(fmaf(Elem<T>::at(rp, x), kLog2e, -sh.row_m[i])) / sh.row_z[i];
        const float qq = uno::ex2(fmaf(Elem<T>::at(rq, x), kLog2e, -sh.row_m[K + 1 + i])) /
                         sh.row_z[K + 1 + i];
        const uint4 w = uno::verify_block_words(P.seed, P.step, b, i);
        rejected = !(uno::uniform24(w.x) * qq < pp);
        if (P.p_at_draft) P.p_at_draft[static_cast<size_t>(b) * K + i] = pp;
        if (P.q_at_draft) P.q_at_draft[static_cast<size_t>(b) * K + i] = qq;
      }
    }
    const unsigned ballot = __ballot_sync(0xFFFFFFFFu, rejected);
    if (ballot && (tid & 31) == 0)
      atomicMin(&sh.first_reject, i0 + (tid & ~31) + __ffs(ballot) - 1);
  }
  __syncthreads();
  const int n = sh.first_reject;
  if (sh.invalid) {
    int32_t* out = P.out_tokens + static_cast<size_t>(b) * (K + 1);
    for (int i = tid; i <= K; i += kThreads) out[i] = -1;
  }
  if (tid == 0) {
    Decision d{};
    d.n = n;
    d.invalid = sh.invalid;
    d.mode = (n < K) ? 0 : 1;
    d.mp = sh.row_m[n];
    d.izp = 1.f / sh.row_z[n];
    if (n < K) {
      d.mq = sh.row_m[K + 1 + n];
      d.izq = 1.f / sh.row_z[K + 1 + n];
      d.c = (sh.row_m[n] + log2f(sh.row_z[n])) -
            (sh.row_m[K + 1 + n] + log2f(sh.row_z[K + 1 + n]));
    }
    P.decisions[b] = d;
    if (sh.invalid) P.accepted_len[b] = -1;
  }
}

// ---- launch 3: the draw -------------------------------------------------------------------

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

// Largest index with positive weight in chunk c (the whole CTA), or -1.
template <typename T>
__device__ int last_positive_in_chunk(const VerifyParams& P, const DrawRows& d, const T* rp,
                                      const T* rq, int c, DrawShared& sh) {
  if (threadIdx.x == 0) sh.last_in_chunk = -1;
  __syncthreads();
  const int v0 = c * P.chunk_len, v1 = min(v0 + P.chunk_len, P.V);
  for (int v = v0 + threadIdx.x; v < v1; v += kThreads)
    if (weight<T>(d, rp, rq, v) > 0.f) atomicMax(&sh.last_in_chunk, v);
  __syncthreads();
  return sh.last_in_chunk;
}

// Final inverse-CDF step of sequence b (the whole CTA); returns the token.
// Thread t holds the sums of chunks [t * per, (t + 1) * per) in registers.
template <typename T>
__device__ int finish_draw(const VerifyParams& P, int b, DrawRows d, const T* rp, const T* rq,
                           DrawShared& sh) {
  constexpr int kMaxPer = kMaxChunks / kThreads;
  const int tid = threadIdx.x;
  float* cs = P.chunk_sums + static_cast<size_t>(b) * P.nchunks;
  const float u = uno::uniform24(uno::verify_block_words(P.seed, P.step, b, d.n).y);
  const int per = (P.nchunks + kThreads - 1) / kThreads;
  const int c0 = tid * per;
  float mine_cs[kMaxPer];
  double mine = 0.0, before = 0.0;
  for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k)
      mine_cs[k] = (k < per && c0 + k < P.nchunks) ? __ldcg(cs + c0 + k) : 0.f;
    mine = 0.0;
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) mine += static_cast<double>(mine_cs[k]);
    before = block_exclusive_scan(mine, sh);
    if (sh.total > 0.0 || d.mode == 1) break;
    // The residual mass is zero (possible only through rounding): draw from p_n.
    d.mode = 1;
    rq = rp;
    chunk_sums<T>(P, b, d, rp, rp, 0, P.nchunks, threadIdx.x >> 5, kWarps);
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
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
      if (k < per && c0 + k < P.nchunks) {
        const double nxt = run + static_cast<double>(mine_cs[k]);
        if (found < 0 && nxt > t) found = c0 + k;
        if (mine_cs[k] > 0.f) last_pos_chunk = c0 + k;
        if (found < 0) run = nxt;
      }
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
  double carry = sh.carry;
  const int v0 = ch * P.chunk_len, v1 = min(v0 + P.chunk_len, P.V);
  for (int base = v0; base < v1; base += kThreads) {
    const int v = base + tid;
    const float w = (v < v1) ? weight<T>(d, rp, rq, v) : 0.f;
    const double bef = carry + block_exclusive_scan(static_cast<double>(w), sh);
    if ((w > 0.f) && (bef + static_cast<double>(w) > t)) atomicMin(&sh.token_min, v);
    if (w > 0.f) atomicMax(&sh.last_in_chunk, v);
    carry += sh.total;
    __syncthreads();
    if (sh.token_min != INT_MAX) break;
  }
  return (sh.token_min != INT_MAX) ? sh.token_min : sh.last_in_chunk;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, kDrawCtasPerSm) verify_draw_kernel(const VerifyParams P) {
  __shared__ DrawShared sh;
  uno::launch_dependents();
  uno::grid_dependency_wait();
  const int tid = threadIdx.x, warp = tid >> 5;
  const int b = blockIdx.x / P.SD, du = blockIdx.x % P.SD;
  const int K = P.K;
  const Decision d = P.decisions[b];
  if (d.invalid) return;  // the decision launch wrote this sequence's outputs
  size_t off;
  const T* rp = row_ptr<T>(P, b, d.n, &off);
  const T* rq = (d.mode == 0) ? row_ptr<T>(P, b, K + 1 + d.n, &off) : rp;
  const int per_cta = (P.nchunks + P.SD - 1) / P.SD;
  const int c0 = du * per_cta;
  const int c1 = min(c0 + per_cta, P.nchunks);
  chunk_sums<T>(P, b, d, rp, rq, c0, c1, warp, kWarps);
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    sh.is_last = (atomicAdd(P.draw_count + b, 1) == P.SD - 1);
  }
  __syncthreads();
  if (!sh.is_last) return;

  // the CTA that completes the sequence picks the token and writes outputs
  __threadfence();
  const int y = finish_draw<T>(P, b, d, rp, rq, sh);
  const int n = d.n;
  int32_t* out = P.out_tokens + static_cast<size_t>(b) * (K + 1);
  const int32_t* x = P.draft + static_cast<size_t>(b) * K;
  for (int i = tid; i <= K; i += kThreads) out[i] = (i < n) ? x[i] : ((i == n) ? y : -1);
  if (tid == 0) P.accepted_len[b] = n;
}

// ---- host side -----------------------------------------------------------------------

struct Geometry {
  int S, nchunks, chunk_len, SD;
  long long stream_ctas, draw_ctas;
  size_t off_counts, off_decisions, off_partials, off_chunks, bytes;
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
  const long long want = static_cast<long long>(kSizingSms) * kStreamCtasPerSm * 2;
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
  g.bytes = align_up(g.off_chunks + sizeof(float) * static_cast<size_t>(B) * g.nchunks, 256);
  return g;
}

// Launch with programmatic stream serialisation: the kernel's CTAs may start
// while the previous kernel on the stream finishes (each waits for it before
// touching global memory).
template <typename Kern>
int launch_pdl(Kern kern, long long grid, cudaStream_t st, const VerifyParams& P) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P) == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

template <typename T>
int launch(const VerifyParams& P, const Geometry& g, cudaStream_t st) {
  if (P.ext_p == nullptr &&
      launch_pdl(verify_stream_kernel<T>, g.stream_ctas, st, P) != UNO_OK)
    return UNO_ERR_CUDA;
  if (launch_pdl(verify_decide_kernel<T>, P.B, st, P) != UNO_OK) return UNO_ERR_CUDA;
  if (launch_pdl(verify_draw_kernel<T>, g.draw_ctas, st, P) != UNO_OK) return UNO_ERR_CUDA;
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
  P.chunk_sums = reinterpret_cast<float*>(ws + g.off_chunks);
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
  P.chunk_sums = reinterpret_cast<float*>(ws + g.off_chunks);
  P.q_rows = K + 1;
  P.ext_p = reinterpret_cast<const Partial*>(stats_ar);
  P.ext_q = reinterpret_cast<const Partial*>(stats_draft);
  P.ext_T = stats_tiles;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (dtype == UNO_BF16) ? launch<uint16_t>(P, g, st) : launch<float>(P, g, st);
}
