// Causal multi-head self-attention, forward and backward.
//
// Layout: the fused projection output qkv is [B, T, 3C] (row = token); q, k, v
// are its column blocks [0,C), [C,2C), [2C,3C) and head h owns columns
// h*d .. h*d+d-1 of each block.  The attention output o is [B, T, C] with the
// same head-column convention, and lse is [B, H, T] fp32 (natural log of the
// softmax denominator of the scaled scores, saved for the backward pass).
//
//   s_ij = q_i . k_j / sqrt(d)      (j <= i; later keys are masked)
//   p_ij = exp(s_ij - lse_i)        o_i = sum_j p_ij v_j
// backward, with D_i = sum_d do_i . o_i = sum_j p_ij (do_i . v_j):
//   dv_j = sum_i p_ij do_i          dp_ij = do_i . v_j
//   ds_ij = p_ij (dp_ij - D_i)      dq_i = sum_j ds_ij k_j / sqrt(d)
//   dk_j = sum_i ds_ij q_i / sqrt(d)
//
// bf16 path (d = 64): the tcgen05 kernels in attention_tc.cuh (forward) and
// attention_tc_bwd.cuh (backward, which also forms D).
// fp32 path (this file): plain per-row kernels (fp32 parity mode, small shapes).
#pragma once
#include "common.cuh"

namespace attn {

constexpr int HD = 64;   // head dim of the bf16 path
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// ------------------------------------------------------------ fp32 path
// one warp per (b, h, query i): lse_i and o_i
__global__ void naive_fwd_kernel(const float* __restrict__ qkv, float* __restrict__ out, float* __restrict__ lse,
                                 int B, int T, int H, int d) {
  const int C = H * d;
  const long ld = 3L * C;
  const long nrows = (long)B * H * T;
  const int lane = threadIdx.x & 31;
  const float scale = 1.f / sqrtf((float)d);
  for (long w = (blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5; w < nrows;
       w += ((long)gridDim.x * blockDim.x) >> 5) {
    const int i = (int)(w % T);
    const int h = (int)((w / T) % H);
    const long b = w / ((long)T * H);
    const float* q = qkv + (b * T + i) * ld + h * d;
    // pass 1: max of the scaled scores
    float mx = -INFINITY;
    for (int j = 0; j <= i; ++j) {
      const float* k = qkv + (b * T + j) * ld + C + h * d;
      float s = 0.f;
      for (int e = lane; e < d; e += 32) s += q[e] * k[e];
      s = warp_sum(s) * scale;
      mx = fmaxf(mx, s);
    }
    // pass 2: denominator and weighted sum of values
    float den = 0.f;
    float acc0 = 0.f, acc1 = 0.f;
    for (int j = 0; j <= i; ++j) {
      const float* k = qkv + (b * T + j) * ld + C + h * d;
      const float* v = k + C;
      float s = 0.f;
      for (int e = lane; e < d; e += 32) s += q[e] * k[e];
      s = warp_sum(s) * scale;
      const float p = expf(s - mx);
      den += p;
      if (lane < d) acc0 += p * v[lane];
      if (lane + 32 < d) acc1 += p * v[lane + 32];
    }
    float* o = out + (b * T + i) * C + h * d;
    if (lane < d) o[lane] = acc0 / den;
    if (lane + 32 < d) o[lane + 32] = acc1 / den;
    if (lane == 0) lse[(b * H + h) * T + i] = mx + logf(den);
  }
}

// one warp per (b, h, query i): D_i and dq_i
__global__ void naive_bwd_dq_kernel(const float* __restrict__ qkv, const float* __restrict__ out,
                                    const float* __restrict__ dout, const float* __restrict__ lse,
                                    float* __restrict__ Dv, float* __restrict__ dqkv, int B, int T, int H, int d) {
  const int C = H * d;
  const long ld = 3L * C;
  const long nrows = (long)B * H * T;
  const int lane = threadIdx.x & 31;
  const float scale = 1.f / sqrtf((float)d);
  for (long w = (blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5; w < nrows;
       w += ((long)gridDim.x * blockDim.x) >> 5) {
    const int i = (int)(w % T);
    const int h = (int)((w / T) % H);
    const long b = w / ((long)T * H);
    const float* q = qkv + (b * T + i) * ld + h * d;
    const float* o = out + (b * T + i) * C + h * d;
    const float* dO = dout + (b * T + i) * C + h * d;
    float Di = 0.f;
    for (int e = lane; e < d; e += 32) Di += dO[e] * o[e];
    Di = warp_sum(Di);
    const float L = lse[(b * H + h) * T + i];
    float acc0 = 0.f, acc1 = 0.f;
    for (int j = 0; j <= i; ++j) {
      const float* k = qkv + (b * T + j) * ld + C + h * d;
      const float* v = k + C;
      float s = 0.f, dp = 0.f;
      for (int e = lane; e < d; e += 32) {
        s += q[e] * k[e];
        dp += dO[e] * v[e];
      }
      s = warp_sum(s) * scale;
      dp = warp_sum(dp);
      const float ds = expf(s - L) * (dp - Di);
      if (lane < d) acc0 += ds * k[lane];
      if (lane + 32 < d) acc1 += ds * k[lane + 32];
    }
    float* dq = dqkv + (b * T + i) * ld + h * d;
    if (lane < d) dq[lane] = acc0 * scale;
    if (lane + 32 < d) dq[lane + 32] = acc1 * scale;
    if (lane == 0) Dv[(b * H + h) * T + i] = Di;
  }
}

// one warp per (b, h, key j): dk_j and dv_j (needs D from the dq kernel)
__global__ void naive_bwd_dkdv_kernel(const float* __restrict__ qkv, const float* __restrict__ dout,
                                      const float* __restrict__ lse, const float* __restrict__ Dv,
                                      float* __restrict__ dqkv, int B, int T, int H, int d) {
  const int C = H * d;
  const long ld = 3L * C;
  const long nrows = (long)B * H * T;
  const int lane = threadIdx.x & 31;
  const float scale = 1.f / sqrtf((float)d);
  for (long w = (blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5; w < nrows;
       w += ((long)gridDim.x * blockDim.x) >> 5) {
    const int j = (int)(w % T);
    const int h = (int)((w / T) % H);
    const long b = w / ((long)T * H);
    const float* k = qkv + (b * T + j) * ld + C + h * d;
    const float* v = k + C;
    float dk0 = 0.f, dk1 = 0.f, dv0 = 0.f, dv1 = 0.f;
    for (int i = j; i < T; ++i) {
      const float* q = qkv + (b * T + i) * ld + h * d;
      const float* dO = dout + (b * T + i) * C + h * d;
      float s = 0.f, dp = 0.f;
      for (int e = lane; e < d; e += 32) {
        s += q[e] * k[e];
        dp += dO[e] * v[e];
      }
      s = warp_sum(s) * scale;
      dp = warp_sum(dp);
      const float p = expf(s - lse[(b * H + h) * T + i]);
      const float ds = p * (dp - Dv[(b * H + h) * T + i]);
      if (lane < d) {
        dk0 += ds * q[lane];
        dv0 += p * dO[lane];
      }
      if (lane + 32 < d) {
        dk1 += ds * q[lane + 32];
        dv1 += p * dO[lane + 32];
      }
    }
    float* dk = dqkv + (b * T + j) * ld + C + h * d;
    float* dv = dk + C;
    if (lane < d) {
      dk[lane] = dk0 * scale;
      dv[lane] = dv0;
    }
    if (lane + 32 < d) {
      dk[lane + 32] = dk1 * scale;
      dv[lane + 32] = dv1;
    }
  }
}

static inline int naive_blocks(long rows) {
  long b = (rows * 32 + 255) / 256;
  return (int)(b > 148 * 32 ? 148 * 32 : b);
}

static inline cudaError_t naive_forward(const float* qkv, float* out, float* lse, int B, int T, int H, int d,
                                        cudaStream_t st) {
  naive_fwd_kernel<<<naive_blocks((long)B * H * T), 256, 0, st>>>(qkv, out, lse, B, T, H, d);
  return cudaGetLastError();
}
static inline cudaError_t naive_backward(const float* qkv, const float* out, const float* dout, const float* lse,
                                         float* dqkv, float* Dv, int B, int T, int H, int d, cudaStream_t st) {
  naive_bwd_dq_kernel<<<naive_blocks((long)B * H * T), 256, 0, st>>>(qkv, out, dout, lse, Dv, dqkv, B, T, H, d);
  naive_bwd_dkdv_kernel<<<naive_blocks((long)B * H * T), 256, 0, st>>>(qkv, dout, lse, Dv, dqkv, B, T, H, d);
  return cudaGetLastError();
}

}  // namespace attn
