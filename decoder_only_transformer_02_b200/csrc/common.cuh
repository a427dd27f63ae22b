// Shared device helpers for the GPT-2 training-step kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

typedef __nv_bfloat16 bf16;

// Library-wide device error word.  Kernels never trap: a bounded wait that
// gives up, or an out-of-range index, records a code here and the kernel
// returns.  The host reads and clears it at its sync points.
enum DeviceErr : int {
  DERR_NONE = 0,
  DERR_TOKEN_RANGE = 1,     // a token or target id >= padded vocab
  DERR_WAIT_TIMEOUT = 2,    // an mbarrier wait ran past its limit
  DERR_NONFINITE = 3,       // non-finite gradient norm (update skipped)
};

// (the library is one translation unit, so this is its single definition)
__device__ int g_device_err = 0;

__device__ __forceinline__ void set_device_err(int code) { atomicCAS(&g_device_err, 0, code); }

// Time after which a pipeline wait (a warp waiting for its producer or
// consumer) gives up, in nanoseconds of %globaltimer.  Settable from the host
// (gpt2_set_wait_limit_ns) so that the give-up path can be exercised; the
// waits that drain a kernel's own in-flight copies and MMAs before it exits
// keep the fixed DRAIN_LIMIT_NS instead.
constexpr unsigned long long DEFAULT_WAIT_LIMIT_NS = 2000000000ull;
constexpr unsigned long long DRAIN_LIMIT_NS = 2000000000ull;
__device__ unsigned long long g_wait_limit_ns = DEFAULT_WAIT_LIMIT_NS;

// --------------------------------------------------------------- numerics
__device__ __forceinline__ float bf2f(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ bf16 f2bf(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Two-wide fp32 arithmetic (sm_100): one instruction for two lanes, each
// rounded as the scalar operation would be, so results are bit-identical.
__device__ __forceinline__ uint64_t f2_bits(float2 a) {
  return (uint64_t)__float_as_uint(a.x) | ((uint64_t)__float_as_uint(a.y) << 32);
}
__device__ __forceinline__ float2 f2_val(uint64_t d) {
  return make_float2(__uint_as_float((uint32_t)d), __uint_as_float((uint32_t)(d >> 32)));
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return f2_val(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_val(d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_val(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_val(d);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

// hardware tanh approximation (max rel. error ~2^-11), used where the result
// is rounded to bf16 anyway
__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU, tanh form: 0.5*u*(1+tanh(sqrt(2/pi)*(u+0.044715*u^3)))
#define GELU_K 0.7978845608028654f
#define GELU_A 0.044715f
// FAST (the bf16 GEMM epilogues): tanh.approx, and the polynomials
// factored into fused multiply-adds,
//   t = u (K + K A u^2),  gelu = h + h tanh(t) with h = u / 2,
//   gelu' = (1 + th) / 2 + (1 - th^2) u (K/2 + 3 K A u^2 / 2);
// otherwise (the fp32 parity mode) tanhf and the formulas as written.
template <bool FAST>
__device__ __forceinline__ float gelu_tanh(float u) {
  if (FAST) {
    const float th = tanh_fast(u * fmaf(GELU_K * GELU_A, u * u, GELU_K));
    const float h = 0.5f * u;
    return fmaf(h, th, h);
  }
  float t = GELU_K * (u + GELU_A * u * u * u);
  float th = tanhf(t);
  return 0.5f * u * (1.0f + th);
}
template <bool FAST>
__device__ __forceinline__ float gelu_tanh_grad(float u) {
  if (FAST) {
    const float u2 = u * u;
    const float th = tanh_fast(u * fmaf(GELU_K * GELU_A, u2, GELU_K));
    const float q = u * fmaf(1.5f * GELU_K * GELU_A, u2, 0.5f * GELU_K);
    return fmaf(q, fmaf(-th, th, 1.0f), fmaf(0.5f, th, 0.5f));
  }
  float t = GELU_K * (u + GELU_A * u * u * u);
  float th = tanhf(t);
  return 0.5f * (1.0f + th) + 0.5f * u * (1.0f - th * th) * GELU_K * (1.0f + 3.0f * GELU_A * u * u);
}

// The FAST forms above on two values with the two-wide instructions: the
// same operations in the same order on each lane, so the same bits.
__device__ __forceinline__ float2 gelu_tanh2(float2 u) {
  const float2 t = mul2(u, fma2(mul2(u, u), make_float2(GELU_K * GELU_A, GELU_K * GELU_A), make_float2(GELU_K, GELU_K)));
  const float2 th = make_float2(tanh_fast(t.x), tanh_fast(t.y));
  const float2 h = mul2(make_float2(0.5f, 0.5f), u);
  return fma2(h, th, h);
}
__device__ __forceinline__ float2 gelu_tanh_grad2(float2 u) {
  const float2 u2 = mul2(u, u);
  const float2 t = mul2(u, fma2(u2, make_float2(GELU_K * GELU_A, GELU_K * GELU_A), make_float2(GELU_K, GELU_K)));
  const float2 th = make_float2(tanh_fast(t.x), tanh_fast(t.y));
  const float2 q = mul2(u, fma2(u2, make_float2(1.5f * GELU_K * GELU_A, 1.5f * GELU_K * GELU_A),
                                make_float2(0.5f * GELU_K, 0.5f * GELU_K)));
  const float2 omt = fma2(mul2(th, make_float2(-1.f, -1.f)), th, make_float2(1.f, 1.f));
  return fma2(q, omt, fma2(make_float2(0.5f, 0.5f), th, make_float2(0.5f, 0.5f)));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Softmax-statistics merge: (m, s, i) <- (m, s, i) (+) (om, os, oi), where m is
// a maximum, s = sum of exp(z - m) and i the lowest index attaining m.  The
// same fixed merge serves the GEMM epilogue's per-tile partials and the
// cross-entropy kernels' reductions.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float LOG2E_F = 1.4426950408889634f;
__device__ __forceinline__ void softmax_stats_merge(float& m, float& s, int& i, float om, float os, int oi) {
  const float nm = fmaxf(m, om);
  const float a = (m == -INFINITY) ? 0.f : ex2_approx((m - nm) * LOG2E_F);
  const float b = (om == -INFINITY) ? 0.f : ex2_approx((om - nm) * LOG2E_F);
  s = s * a + os * b;
  if (om > m || (om == m && oi < i)) i = oi;
  m = nm;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

static inline int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }

// Host-side set-up that must run once on every device a kernel is launched on
// (cudaFuncSetAttribute applies to the current device only).
struct DeviceOnce {
  std::mutex mu;
  bool done[64] = {};
};
template <class F>
static cudaError_t run_once_per_device(DeviceOnce& once, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(once.mu);
  if (once.done[dev]) return cudaSuccess;
  e = setup();
  if (e == cudaSuccess) once.done[dev] = true;
  return e;
}
