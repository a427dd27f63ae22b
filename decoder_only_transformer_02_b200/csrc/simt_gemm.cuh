// fp32 GEMM on the CUDA cores (FFMA, no TF32) for the fp32 parity mode.
//
//   D[M,N] = sum_k A[m,k] * B[n,k]
// A element (m,k) at A[m*sam + k*sak]; B element (n,k) at B[n*sbn + k*sbk]
// (any of the forward / dgrad / wgrad layouts by choice of strides), with the
// same fused epilogues as the tensor-core GEMM, all in fp32.
#pragma once
#include "common.cuh"

namespace simt {

enum Epi : int {
  EPI_F32 = 0,        // out = acc (+ bias)
  EPI_RESID = 1,      // out = resid + acc (+ bias)
  EPI_GELU = 2,       // out = u = acc + bias ; out2 = gelu_tanh(u)
  EPI_DGELU = 3,      // out = acc * gelu_tanh'(aux)
  EPI_ACCUM = 4,      // out += acc
};

struct Args {
  const float* A;
  long sam, sak;
  const float* B;
  long sbn, sbk;
  int M, N, K;
  int epi;
  const float* bias;
  const float* resid;
  float* out;
  float* out2;
  const float* aux;
  long ldc;
};

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) simt_gemm_kernel(const Args a) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += TK) {
    for (int i = threadIdx.x; i < TK * TM; i += 256) {
      int kk = i % TK, mm = i / TK;
      int m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < a.M && k < a.K) ? a.A[(long)m * a.sam + (long)k * a.sak] : 0.f;
      int n = n0 + mm;
      Bs[kk][mm] = (n < a.N && k < a.K) ? a.B[(long)n * a.sbn + (long)k * a.sbk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= a.N) continue;
      const long o = (long)m * a.ldc + n;
      float v = acc[i][j];
      switch (a.epi) {
        case EPI_F32:
          a.out[o] = a.bias ? v + a.bias[n] : v;
          break;
        case EPI_RESID:
          a.out[o] = a.resid[o] + (a.bias ? v + a.bias[n] : v);
          break;
        case EPI_GELU: {
          float u = a.bias ? v + a.bias[n] : v;
          a.out[o] = u;
          a.out2[o] = gelu_tanh<false>(u);
        } break;
        case EPI_DGELU:
          a.out[o] = v * gelu_tanh_grad<false>(a.aux[o]);
          break;
        case EPI_ACCUM:
          a.out[o] += v;
          break;
      }
    }
  }
}

static inline cudaError_t gemm(const Args& a, cudaStream_t st) {
  dim3 grid(ceil_div(a.N, TN), ceil_div(a.M, TM));
  simt_gemm_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace simt
