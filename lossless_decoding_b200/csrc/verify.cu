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
// One launch does the whole step. Work unit = (sequence b, row j, slab s):
// rows j = 0..K are the AR rows p_0..p_K, rows K+1..2K the draft rows
// q_0..q_{K-1}; a slab is a contiguous stretch of one row's vocabulary. Each
// CTA streams its slab once with 16-byte loads and keeps a running
// (max, sum of exponentials) per thread, merged by warp shuffles and then
// across warps. The CTA that completes a sequence's last unit (an atomic
// counter per sequence, no waiting) merges the slab partials of the
// sequence's 2K+1 rows, evaluates the accept tests, finds the first rejection
// with a warp ballot, draws the residual (or bonus) token by inverse CDF over
// one or two rows that were just streamed (mostly still in L2), writes the
// outputs, and clears the partials and the counter it used, so the workspace
// is zero-filled again when the call completes.
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
constexpr int kUnroll = 4;            // 16-byte vectors per thread per iteration
constexpr int kMaxK = 256;
constexpr int kMaxRows = 2 * kMaxK + 1;
constexpr int kMaxChunks = 2048;      // inverse-CDF chunk sums held in shared memory
constexpr int kMinVecPerSlab = kThreads * kUnroll;  // at least one full iteration
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Partial {
  float m;  // max over the slab of l * log2(e)
  float z;  // sum over the slab of 2^(l * log2(e) - m)
};

struct VerifyParams {
  const void* p_logits;
  const void* q_logits;
  const int32_t* draft;
  int B, K, V, S;
  uint64_t seed, step;
  int32_t* out_tokens;
  int32_t* accepted_len;
  float* p_at_draft;
  float* q_at_draft;
  float* row_lse;
  Partial* partials;  // [B][2K+1][S]
  int* counters;      // [B]
};

// ---- element access --------------------------------------------------------

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

// ---- (max, sum-exp) algebra in the log2 domain ------------------------------

__device__ __forceinline__ void merge(float& m, float& z, float m2, float z2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;  // both empty
  const float a = (m == -INFINITY) ? 0.f : z * uno::ex2(m - mm);
  const float b = (m2 == -INFINITY) ? 0.f : z2 * uno::ex2(m2 - mm);
  m = mm;
  z = a + b;
}

// Fold n values (natural-log logits) into the running (m, z).
template <int N>
__device__ __forceinline__ void fold(float& m, float& z, const float* v) {
  float cm = v[0];
#pragma unroll
  for (int e = 1; e < N; ++e) cm = fmaxf(cm, v[e]);
  if (cm == -INFINITY) return;
  const float cm2 = cm * kLog2e;
  if (cm2 > m) {
    z *= uno::ex2(m - cm2);  // m = -inf gives 0
    m = cm2;
  }
  float t[N];
#pragma unroll
  for (int e = 0; e < N; ++e) t[e] = uno::ex2(fmaf(v[e], kLog2e, -m));
  // pairwise sum of the chunk, then one add into the running total
#pragma unroll
  for (int w = 1; w < N; w *= 2) {
#pragma unroll
    for (int e = 0; e + w < N; e += 2 * w) t[e] += t[e + w];
  }
  z += t[0];
}

// Geometry of one row: a scalar head up to the first 16-byte boundary, then
// nvec full vectors, then a scalar tail.
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

template <typename T>
__device__ __forceinline__ const T* row_ptr(const VerifyParams& P, int b, int j, size_t* off) {
  const int K = P.K;
  size_t row;
  const T* base;
  if (j <= K) {
    row = static_cast<size_t>(b) * (K + 1) + j;
    base = static_cast<const T*>(P.p_logits);
  } else {
    row = static_cast<size_t>(b) * K + (j - K - 1);
    base = static_cast<const T*>(P.q_logits);
  }
  *off = row * static_cast<size_t>(P.V);
  return base + *off;
}

// ---- block reductions -------------------------------------------------------

__device__ __forceinline__ void warp_merge(float& m, float& z) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    const float z2 = __shfl_xor_sync(0xFFFFFFFFu, z, o);
    merge(m, z, m2, z2);
  }
}

// ---- the draw: inverse CDF over one row's weights ---------------------------

struct DrawShared {
  float chunk_sum[kMaxChunks];
  double t;          // threshold u' * total
  int chunk;         // chunk where the running sum crosses t
  int last_pos;      // largest index with positive weight
  int token;
};

// Weight of token v. mode 0: max(0, p(v) - q(v)); mode 1: p(v).
template <typename T>
__device__ __forceinline__ float weight(int mode, const T* rp, const T* rq, int v, float mp,
                                        float izp, float mq, float izq) {
  const float pv = uno::ex2(fmaf(Elem<T>::at(rp, v), kLog2e, -mp)) * izp;
  if (mode) return pv;
  const float qv = uno::ex2(fmaf(Elem<T>::at(rq, v), kLog2e, -mq)) * izq;
  return fmaxf(0.f, pv - qv);
}

// All threads of the CTA call this. Returns the drawn token, or -1 when every
// weight is zero.
template <typename T>
__device__ int draw_token(DrawShared& sh, int mode, const T* rp, const T* rq, int V, float mp,
                          float izp, float mq, float izq, float u) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int chunk_len = (V + kMaxChunks - 1) / kMaxChunks;
  chunk_len = chunk_len < 256 ? 256 : ((chunk_len + 31) / 32) * 32;
  const int nchunks = (V + chunk_len - 1) / chunk_len;

  if (tid == 0) sh.last_pos = -1;
  __syncthreads();
  // Phase A: every chunk's weight sum (one warp per chunk, fixed order inside).
  int my_last = -1;
  for (int c = warp; c < nchunks; c += kWarps) {
    const int v0 = c * chunk_len;
    const int v1 = min(v0 + chunk_len, V);
    float s = 0.f;
    for (int v = v0 + lane; v < v1; v += 32) {
      const float w = weight<T>(mode, rp, rq, v, mp, izp, mq, izq);
      s += w;
      if (w > 0.f) my_last = v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane == 0) sh.chunk_sum[c] = s;
  }
  if (my_last >= 0) atomicMax(&sh.last_pos, my_last);
  __syncthreads();
  if (sh.last_pos < 0) return -1;  // all weights zero (uniform value for every thread)

  // Phase B (warp 0): running sum of chunk sums in float64; find the chunk.
  if (warp == 0) {
    const int per = (nchunks + 31) / 32;
    const int c0 = lane * per, c1 = min(c0 + per, nchunks);
    double mine = 0.0;
    for (int c = c0; c < c1; ++c) mine += static_cast<double>(sh.chunk_sum[c]);
    double incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double up = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += up;
    }
    const double total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    const double t = static_cast<double>(u) * total;
    double run = incl - mine;  // exclusive prefix of this lane's block
    int found = INT_MAX;
    for (int c = c0; c < c1; ++c) {
      const double nxt = run + static_cast<double>(sh.chunk_sum[c]);
      if (nxt > t) { found = c; break; }
      run = nxt;
    }
    const unsigned hit = __ballot_sync(0xFFFFFFFFu, found != INT_MAX);
    const int src = hit ? (__ffs(hit) - 1) : 31;
    const int chunk = __shfl_sync(0xFFFFFFFFu, found, src);
    if (lane == 0) {
      sh.t = t;
      sh.chunk = (chunk == INT_MAX) ? -1 : chunk;
      sh.token = -1;
    }
    // Phase C: scan inside the chosen chunk.
    const int ch = __shfl_sync(0xFFFFFFFFu, chunk, 0);
    if (ch != INT_MAX) {
      double carry = 0.0;
      for (int c = 0; c < ch; ++c) carry += static_cast<double>(sh.chunk_sum[c]);
      const int v0 = ch * chunk_len, v1 = min(v0 + chunk_len, V);
      int tok = -1, last_pos_in_chunk = -1;
      for (int base = v0; base < v1 && tok < 0; base += 32) {
        const int v = base + lane;
        const float w = (v < v1) ? weight<T>(mode, rp, rq, v, mp, izp, mq, izq) : 0.f;
        float incl_w = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float up = __shfl_up_sync(0xFFFFFFFFu, incl_w, o);
          if (lane >= o) incl_w += up;
        }
        const bool cross = (v < v1) && (w > 0.f) && (carry + static_cast<double>(incl_w) > t);
        const unsigned m = __ballot_sync(0xFFFFFFFFu, cross);
        const unsigned pos = __ballot_sync(0xFFFFFFFFu, (v < v1) && (w > 0.f));
        if (pos) last_pos_in_chunk = base + 31 - __clz(pos);
        if (m) tok = base + __ffs(m) - 1;
        carry += static_cast<double>(__shfl_sync(0xFFFFFFFFu, incl_w, 31));
      }
      if (lane == 0) sh.token = (tok >= 0) ? tok : last_pos_in_chunk;
    }
  }
  __syncthreads();
  const int tok = sh.token;
  return tok >= 0 ? tok : sh.last_pos;
}

// ---- finalize (runs in the CTA that completes sequence b) --------------------

struct FinalShared {
  float m[kMaxRows];
  float z[kMaxRows];
  int first_reject;
  int invalid;
  DrawShared draw;
};

template <typename T>
__device__ void finalize_sequence(const VerifyParams& P, int b, FinalShared& sh) {
  const int K = P.K, R = 2 * K + 1, S = P.S, V = P.V;
  const int tid = threadIdx.x;
  if (tid == 0) {
    sh.first_reject = K;
    sh.invalid = 0;
  }
  // 1. merge slab partials of every row, slabs in index order, and clear them
  //    so the workspace is zero-filled again when the call completes.
  for (int j = tid; j < R; j += kThreads) {
    Partial* pp = P.partials + (static_cast<size_t>(b) * R + j) * S;
    float m = -INFINITY, z = 0.f;
    for (int s = 0; s < S; ++s) {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(pp + s));
      merge(m, z, v.x, v.y);
      pp[s] = Partial{0.f, 0.f};
    }
    sh.m[j] = m;
    sh.z[j] = z;
    if (P.row_lse) P.row_lse[static_cast<size_t>(b) * R + j] = (m + log2f(z)) * kLn2;
  }
  __syncthreads();

  // 2. accept tests, one thread per drafted position; first rejection by ballot.
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
        const float pp = uno::ex2(fmaf(Elem<T>::at(rp, x), kLog2e, -sh.m[i])) / sh.z[i];
        const float qq =
            uno::ex2(fmaf(Elem<T>::at(rq, x), kLog2e, -sh.m[K + 1 + i])) / sh.z[K + 1 + i];
        const uint4 w = uno::verify_block_words(P.seed, P.step, b, i);
        const float u = uno::uniform24(w.x);
        rejected = !(u * qq < pp);
        if (P.p_at_draft) P.p_at_draft[static_cast<size_t>(b) * K + i] = pp;
        if (P.q_at_draft) P.q_at_draft[static_cast<size_t>(b) * K + i] = qq;
      }
    }
    const unsigned ballot = __ballot_sync(0xFFFFFFFFu, rejected);
    if (ballot && (tid & 31) == 0) atomicMin(&sh.first_reject, i0 + (tid & ~31) + __ffs(ballot) - 1);
  }
  __syncthreads();

  const int n = sh.first_reject;
  int32_t* out = P.out_tokens + static_cast<size_t>(b) * (K + 1);
  if (sh.invalid) {
    for (int i = tid; i <= K; i += kThreads) out[i] = -1;
    if (tid == 0) P.accepted_len[b] = -1;
    return;
  }

  // 3. residual (n < K) or bonus (n == K) draw with u'_n.
  size_t off;
  const T* rp = row_ptr<T>(P, b, n, &off);
  const T* rq = (n < K) ? row_ptr<T>(P, b, K + 1 + n, &off) : rp;
  const float u = uno::uniform24(uno::verify_block_words(P.seed, P.step, b, n).y);
  const float mp = sh.m[n], izp = 1.f / sh.z[n];
  const float mq = (n < K) ? sh.m[K + 1 + n] : 0.f;
  const float izq = (n < K) ? 1.f / sh.z[K + 1 + n] : 0.f;
  int y = draw_token<T>(sh.draw, (n < K) ? 0 : 1, rp, rq, V, mp, izp, mq, izq, u);
  if (y < 0) y = draw_token<T>(sh.draw, 1, rp, rp, V, mp, izp, 0.f, 0.f, u);  // empty residual

  // 4. outputs.
  const int32_t* x = P.draft + static_cast<size_t>(b) * K;
  for (int i = tid; i <= K; i += kThreads) out[i] = (i < n) ? x[i] : ((i == n) ? y : -1);
  if (tid == 0) P.accepted_len[b] = n;
}

// ---- the kernel ----------------------------------------------------------------

template <typename T>
__global__ void __launch_bounds__(kThreads, 4) verify_kernel(const VerifyParams P) {
  constexpr int kVec = Elem<T>::kVec;
  __shared__ FinalShared sh_final;
  __shared__ float red_m[kWarps], red_z[kWarps];
  __shared__ int is_last;

  const int R = 2 * P.K + 1;
  const int unit = blockIdx.x;
  const int s = unit % P.S;
  const int rj = unit / P.S;
  const int j = rj % R;
  const int b = rj / R;
  const int tid = threadIdx.x;

  size_t off;
  const T* row = row_ptr<T>(P, b, j, &off);
  const RowGeom g = row_geom<T>(off, P.V);
  const int per = (g.nvec + P.S - 1) / P.S;
  const int v_begin = min(s * per, g.nvec);
  const int v_end = min(v_begin + per, g.nvec);

  float m = -INFINITY, z = 0.f;
  const uint4* vrow = reinterpret_cast<const uint4*>(row + g.head);
  for (int base = v_begin; base < v_end; base += kThreads * kUnroll) {
    uint4 raw[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int idx = base + k * kThreads + tid;
      raw[k] = (idx < v_end) ? __ldg(vrow + idx)
                             : make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
    }
    float f[kUnroll * kVec];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int idx = base + k * kThreads + tid;
      Elem<T>::unpack(raw[k], f + k * kVec);
      if (idx >= v_end) {
#pragma unroll
        for (int e = 0; e < kVec; ++e) f[k * kVec + e] = -INFINITY;
      }
    }
    fold<kUnroll * kVec>(m, z, f);
  }
  // scalar head (first slab) and tail (last slab)
  if (s == 0 && tid < g.head) {
    const float v = Elem<T>::at(row, tid);
    fold<1>(m, z, &v);
  }
  if (s == P.S - 1 && tid < g.tail) {
    const float v = Elem<T>::at(row, static_cast<size_t>(g.head) + static_cast<size_t>(g.nvec) * kVec + tid);
    fold<1>(m, z, &v);
  }

  warp_merge(m, z);
  const int lane = tid & 31, warp = tid >> 5;
  if (lane == 0) {
    red_m[warp] = m;
    red_z[warp] = z;
  }
  __syncthreads();
  if (tid == 0) {
    float bm = red_m[0], bz = red_z[0];
    for (int w = 1; w < kWarps; ++w) merge(bm, bz, red_m[w], red_z[w]);
    P.partials[static_cast<size_t>(rj) * P.S + s] = Partial{bm, bz};
    __threadfence();
    const int prev = atomicAdd(P.counters + b, 1);
    is_last = (prev == R * P.S - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  finalize_sequence<T>(P, b, sh_final);
  if (tid == 0) P.counters[b] = 0;  // leave the workspace zero-filled
}

// ---- host side -----------------------------------------------------------------

int choose_slabs(int B, int K, int V, int dtype) {
  const int vec = (dtype == UNO_BF16) ? 8 : 4;
  const long long rows = static_cast<long long>(B) * (2 * K + 1);
  const long long nvec = V / vec;
  long long smax = nvec / kMinVecPerSlab;
  if (smax < 1) smax = 1;
  const long long target = 148LL * 32;  // about four waves of eight CTAs per SM
  long long s = (target + rows - 1) / rows;
  if (s > smax) s = smax;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool verify_sizes_ok(int B, int K, int V, int dtype) {
  return (dtype == UNO_BF16 || dtype == UNO_F32) && B >= 0 && B <= (1 << 20) && K >= 1 &&
         K <= kMaxK && V >= 1 && V <= (1 << 28);
}

}  // namespace

extern "C" size_t uno_verify_workspace_bytes(int B, int K, int V, int dtype) {
  if (!verify_sizes_ok(B, K, V, dtype)) return 0;
  const int S = choose_slabs(B, K, V, dtype);
  const size_t partial = static_cast<size_t>(B) * (2 * K + 1) * S * sizeof(Partial);
  return align_up(partial, 16) + align_up(static_cast<size_t>(B) * sizeof(int), 16);
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
  const size_t need = uno_verify_workspace_bytes(B, K, V, dtype);
  if (workspace_bytes < need) return UNO_ERR_WORKSPACE;
  const int dev_status = uno_host::check_device();
  if (dev_status != UNO_OK) return dev_status;

  VerifyParams P;
  P.p_logits = p_logits;
  P.q_logits = q_logits;
  P.draft = draft_tokens;
  P.B = B;
  P.K = K;
  P.V = V;
  P.S = choose_slabs(B, K, V, dtype);
  P.seed = seed;
  P.step = step;
  P.out_tokens = out_tokens;
  P.accepted_len = accepted_len;
  P.p_at_draft = p_at_draft;
  P.q_at_draft = q_at_draft;
  P.row_lse = row_lse;
  const size_t partial_bytes =
      align_up(static_cast<size_t>(B) * (2 * K + 1) * P.S * sizeof(Partial), 16);
  P.partials = static_cast<Partial*>(workspace);
  P.counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + partial_bytes);

  const long long grid = static_cast<long long>(B) * (2 * K + 1) * P.S;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == UNO_BF16)
    verify_kernel<uint16_t><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(P);
  else
    verify_kernel<float><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(P);
  return (cudaGetLastError() == cudaSuccess) ? UNO_OK : UNO_ERR_CUDA;
}
