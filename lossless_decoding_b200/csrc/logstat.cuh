// Row statistics in the log2 domain: a running (reference m, sum z) pair with
// z = sum of 2^(x - m) over the values seen, x = l * log2(e) for a natural-log
// logit l. Shared by the verifier's stream and the draft sampler.
#pragma once

#include <cstdint>

#include "uno_device.cuh"

namespace uno {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void merge(float& m, float& z, float m2, float z2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;  // both empty
  const float a = (m == -INFINITY) ? 0.f : z * ex2(m - mm);
  const float b = (m2 == -INFINITY) ? 0.f : z2 * ex2(m2 - mm);
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
  for (int e = 0; e < N; ++e) t[e] = ex2(fmaf(v[e], kLog2e, -m));
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
    z = (m == -INFINITY) ? 0.f : z * ex2(m - gm);
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

// Folds NV 16-byte vectors (8 NV bfloat16 or 4 NV float32 values) with
// packed float32x2 arithmetic: the exponent arguments by fma.f32x2, 2^(.) on
// the SFU, a balanced sum tree by add.f32x2 (fold's tree, pair by pair). Same
// reference rule as fold.
template <typename T, int NV>
__device__ __forceinline__ void fold_vecs(float& m, float& z, const uint4* v) {
  constexpr bool kBf16 = sizeof(T) == 2;
  constexpr int kP = (kBf16 ? 4 : 2) * NV;  // float pairs
  uint64_t x[kP];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    if constexpr (kBf16) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        x[4 * k + i] = pack2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    } else {
#pragma unroll
      for (int i = 0; i < 2; ++i)
        x[2 * k + i] = pack2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
    }
  }
  auto sum = [&](float ref) {
    const uint64_t l2e = pack2(kLog2e, kLog2e), nref = pack2(-ref, -ref);
    uint64_t e[kP];
#pragma unroll
    for (int i = 0; i < kP; ++i) {
      const float2 a = unpack2(fma2(x[i], l2e, nref));
      e[i] = pack2(ex2(a.x), ex2(a.y));
    }
#pragma unroll
    for (int w = 1; w < kP; w *= 2) {
#pragma unroll
      for (int i = 0; i + w < kP; i += 2 * w) e[i] = add2(e[i], e[i + w]);
    }
    const float2 s = unpack2(e[0]);
    return s.x + s.y;
  };
  const float s = sum(m);
  if (s < 0x1p70f) {  // false for inf and NaN
    z += s;
    return;
  }
  float gm = -INFINITY;
#pragma unroll
  for (int i = 0; i < kP; ++i) {
    const float2 p = unpack2(x[i]);
    gm = fmaxf(gm, fmaxf(p.x, p.y));
  }
  if (gm == -INFINITY) return;
  gm *= kLog2e;
  if (gm > m) {
    z = (m == -INFINITY) ? 0.f : z * ex2(m - gm);
    m = gm;
  }
  z += sum(m);
}

// The same fold with m kept at the running maximum (times log2 e) instead of a
// lazy reference: the group's maximum is taken first and m moves up to it
// before the sum, so every exponent argument is <= 0. Costs one more max per
// value; in return a weight's error from its argument's rounding is at most
// about 2^-24 ln 2 |argument| 2^argument of the maximum's weight, which keeps
// a sampler's chunk sums (not only their ratios) accurate to a few float32
// roundings.
template <typename T, int NV>
__device__ __forceinline__ void fold_vecs_max(float& m, float& z, const uint4* v) {
  constexpr bool kBf16 = sizeof(T) == 2;
  constexpr int kP = (kBf16 ? 4 : 2) * NV;  // float pairs
  uint64_t x[kP];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    if constexpr (kBf16) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        x[4 * k + i] = pack2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    } else {
#pragma unroll
      for (int i = 0; i < 2; ++i)
        x[2 * k + i] = pack2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
    }
  }
  float gm = -INFINITY;
#pragma unroll
  for (int i = 0; i < kP; ++i) {
    const float2 p = unpack2(x[i]);
    gm = fmaxf(gm, fmaxf(p.x, p.y));
  }
  if (gm == -INFINITY) return;  // nothing finite in the group
  gm *= kLog2e;
  if (gm > m) {
    z = (m == -INFINITY) ? 0.f : z * ex2(m - gm);
    m = gm;
  }
  const uint64_t l2e = pack2(kLog2e, kLog2e), nref = pack2(-m, -m);
  uint64_t e[kP];
#pragma unroll
  for (int i = 0; i < kP; ++i) {
    const float2 a = unpack2(fma2(x[i], l2e, nref));
    e[i] = pack2(ex2(a.x), ex2(a.y));
  }
#pragma unroll
  for (int w = 1; w < kP; w *= 2) {
#pragma unroll
    for (int i = 0; i + w < kP; i += 2 * w) e[i] = add2(e[i], e[i + w]);
  }
  const float2 s = unpack2(e[0]);
  z += s.x + s.y;
}

// One value, m kept at the running maximum (times log2 e).
__device__ __forceinline__ void fold_one_max(float& m, float& z, float x) {
  if (!(x > -INFINITY)) return;
  const float g = x * kLog2e;
  if (g > m) {
    z = (m == -INFINITY) ? 0.f : z * ex2(m - g);
    m = g;
  }
  z += ex2(fmaf(x, kLog2e, -m));
}

template <typename T>
__device__ __forceinline__ void fold_pair(float& m, float& z, const uint4* v) {
  fold_vecs<T, 2>(m, z, v);
}

}  // namespace uno
