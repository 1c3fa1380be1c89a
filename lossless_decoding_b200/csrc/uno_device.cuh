// Device-side helpers shared by the Uno sm_100a kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace uno {

// ---------------------------------------------------------------------------
// Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11). Ten rounds; each
// round multiplies counter words 0 and 2 by the two Philox multipliers, takes
// the high and low halves of the 64-bit products, and mixes in the key, which
// is bumped by the two Weyl constants between rounds.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t m0 = 0xD2511F53u, m1 = 0xCD9E8D57u;
    const uint32_t lo0 = m0 * c.x, hi0 = __umulhi(m0, c.x);
    const uint32_t lo1 = m1 * c.z, hi1 = __umulhi(m1, c.z);
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
    k.x += 0x9E3779B9u;
    k.y += 0xBB67AE85u;
  }
  return c;
}

// Top 24 bits of a Philox word as a float in [0, 1): exact in float32.
__device__ __forceinline__ float uniform24(uint32_t w) {
  return static_cast<float>(w >> 8) * 5.9604644775390625e-08f;  // 2^-24
}

// Uniforms of sequence b, position i: counter (b, i, step lo, step hi),
// key (seed lo, seed hi). Word 0 -> accept test, word 1 -> token draw.
__device__ __forceinline__ uint4 verify_block_words(uint64_t seed, uint64_t step, uint32_t b,
                                                    uint32_t i) {
  return philox4x32_10(make_uint4(b, i, static_cast<uint32_t>(step),
                                  static_cast<uint32_t>(step >> 32)),
                       make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)));
}

// Programmatic dependent launch. A kernel launched with programmatic stream
// serialisation may start while the previous kernel on the stream is still
// running; it calls grid_dependency_wait() before it touches global memory the
// previous kernel may write or read, which returns once that kernel has
// completed and its writes are visible. launch_dependents() lets the next
// kernel start (its CTAs only get SMs as this kernel's CTAs leave).
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Asynchronous 16-byte copy global -> shared (cp.async.cg, cached in L2 only).
// Completion is per thread: copies are grouped by commit, and wait<N> returns
// once at most the N most recent groups of this thread are still in flight.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Packed float32 pairs (PTX .f32x2 arithmetic, sm_100): one instruction does
// the operation on both halves, each rounded as its scalar form would be.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x on the SFU (PTX ex2.approx, flush-to-zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h16) {
  return __uint_as_float(h16 << 16);
}

// Round-to-nearest-even float -> bfloat16 bits (finite inputs; NaN kept NaN).
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

// A row of logits in memory: element reads and 16-byte vector unpacking for
// bfloat16 (raw bits, 8 per vector) and float32 (4 per vector).
template <typename T>
struct LogitRow;

template <>
struct LogitRow<uint16_t> {
  static constexpr int kVec = 8;
  __device__ static __forceinline__ float at(const uint16_t* p, long long i) {
    return bf16_bits_to_float(__ldg(p + i));
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
struct LogitRow<float> {
  static constexpr int kVec = 4;
  __device__ static __forceinline__ float at(const float* p, long long i) { return __ldg(p + i); }
  __device__ static __forceinline__ void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
};

}  // namespace uno
