// Memory-bound kernels of the GPT-2 step: embedding, LayerNorm, softmax
// cross-entropy, bias-gradient column sums, gradient norm, AdamW, init.
// Every reduction runs in a fixed order (no floating-point atomics), so results
// are bit-reproducible run to run.
#pragma once
#include "common.cuh"

namespace k {

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<bf16>(const bf16* p) { return bf2f(*p); }
template <typename T>
__device__ __forceinline__ void st_f(T* p, float v);
template <>
__device__ __forceinline__ void st_f<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_f<bf16>(bf16* p, float v) { *p = f2bf(v); }

// ------------------------------------------------------------ embedding
// x0[b,t,:] = wte[tok[b,t],:] + wpe[t,:]; an id >= V marks the error word and
// the row is written as wpe only.  Also checks targets (may be null).
__global__ void embed_fwd_kernel(const int32_t* __restrict__ tok, const int32_t* __restrict__ tgt,
                                 const float* __restrict__ wte, const float* __restrict__ wpe, float* __restrict__ x,
                                 int M, int T, int C, int V, int* __restrict__ bad) {
  const int c4 = C / 4;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < (long)M * c4; i += (long)gridDim.x * blockDim.x) {
    const int row = (int)(i / c4), c = (int)(i % c4);
    const int id = tok[row];
    const int t = row % T;
    float4 p = reinterpret_cast<const float4*>(wpe + (long)t * C)[c];
    if (id >= 0 && id < V) {
      float4 w = reinterpret_cast<const float4*>(wte + (long)id * C)[c];
      p.x += w.x;
      p.y += w.y;
      p.z += w.z;
      p.w += w.w;
    } else if (c == 0) {
      atomicExch(bad, 1);
    }
    if (c == 0 && tgt != nullptr) {
      const int y = tgt[row];
      if (y < 0 || y >= V) atomicExch(bad, 1);
    }
    reinterpret_cast<float4*>(x + (long)row * C)[c] = p;
  }
}

// single-CTA bitonic sort of the keys (token << 16 | position), n <= capacity
// (a power of two, padded with 0xffffffff).  Sorting (token, position) pairs
// gives every token's positions in ascending order: the fixed summation order
// of the embedding scatter-add.
// An id outside [0, V) sorts under the sentinel token 0xffff (never a valid
// row: V <= 65472) and is skipped by the scatter.
__global__ void sort_keys_kernel(const int32_t* __restrict__ tok, int M, int V, uint32_t* __restrict__ keys_out,
                                 int cap) {
  extern __shared__ uint32_t sk[];
  for (int i = threadIdx.x; i < cap; i += blockDim.x) {
    uint32_t key = 0xffffffffu;
    if (i < M) {
      const int t = tok[i];
      key = ((t >= 0 && t < V) ? (uint32_t)t : 0xffffu) << 16 | (uint32_t)i;
    }
    sk[i] = key;
  }
  __syncthreads();
  for (int size = 2; size <= cap; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < cap / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = ((lo & size) == 0);
        const uint32_t a = sk[lo], b = sk[hi];
        if ((a > b) == up) {
          sk[lo] = b;
          sk[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < M; i += blockDim.x) keys_out[i] = sk[i];
}

// Stage 1 of the deterministic scatter-add.  Sorted entries are cut into
// chunks of EMB_CH; chunk c sums each run of equal tokens it holds (positions
// in ascending order) and writes the run's sum to part[first sorted index of
// the run].  dx0 is fp32 [M, C]; one CTA per chunk, one thread per 4 columns
// (blockDim >= C/4); the chunk's keys sit in shared memory and eight rows'
// loads are in flight at a time.
constexpr int EMB_CH = 32;
__global__ void embed_bwd_partial_kernel(const uint32_t* __restrict__ keys, const float* __restrict__ dx, int M, int C,
                                         float* __restrict__ part) {
  __shared__ uint32_t ks[EMB_CH];
  const int c0 = blockIdx.x * EMB_CH;
  const int n = min(EMB_CH, M - c0);
  for (int i = threadIdx.x; i < n; i += blockDim.x) ks[i] = keys[c0 + i];
  __syncthreads();
  const int c4 = threadIdx.x;
  if (c4 >= C / 4) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int run_start = 0;
  for (int s0 = 0; s0 < n; s0 += 8) {
    float4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (s0 + j < n) v[j] = reinterpret_cast<const float4*>(dx + (long)(ks[s0 + j] & 0xffffu) * C)[c4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int s = s0 + j;
      if (s < n) {
        acc.x += v[j].x;
        acc.y += v[j].y;
        acc.z += v[j].z;
        acc.w += v[j].w;
        if (s + 1 == n || (ks[s + 1] >> 16) != (ks[s] >> 16)) {
          reinterpret_cast<float4*>(part + (long)(c0 + run_start) * C)[c4] = acc;
          acc = make_float4(0.f, 0.f, 0.f, 0.f);
          run_start = s + 1;
        }
      }
    }
  }
}

// Stage 2: one CTA per sorted index (launched with a grid of M); the CTAs at a
// token's first sorted index sum the run partials of that token's segment (in
// sorted order) into dwte[token].  One thread per 4 columns.
__global__ void embed_bwd_reduce_kernel(const uint32_t* __restrict__ keys, const float* __restrict__ part, int M, int C,
                                        int V, float* __restrict__ dwte) {
  for (int s = blockIdx.x; s < M; s += gridDim.x) {
    const uint32_t tokn = keys[s] >> 16;
    if (tokn >= (uint32_t)V) continue;                   // out-of-range id (already flagged)
    if (s > 0 && (keys[s - 1] >> 16) == tokn) continue;  // not a segment start
    // segment end: the keys are sorted by token, so binary-search the first
    // index past s whose token differs
    int lo = s + 1, hi = M;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if ((keys[mid] >> 16) == tokn)
        lo = mid + 1;
      else
        hi = mid;
    }
    const int e = lo;
    for (int c4 = threadIdx.x; c4 < C / 4; c4 += blockDim.x) {
      // run partials start at s and at each chunk boundary inside [s, e)
      float4 acc = reinterpret_cast<const float4*>(part + (long)s * C)[c4];
#pragma unroll 4
      for (int cb = (s / EMB_CH + 1) * EMB_CH; cb < e; cb += EMB_CH) {
        const float4 v = reinterpret_cast<const float4*>(part + (long)cb * C)[c4];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      float4* d = reinterpret_cast<float4*>(dwte + (long)tokn * C) + c4;
      const float4 o = *d;
      *d = make_float4(o.x + acc.x, o.y + acc.y, o.z + acc.z, o.w + acc.w);
    }
  }
}


// g[i] += slots[0][i] + slots[1][i] + ... (in split order), and the slots
// are cleared for the next accumulation.  n % 4 == 0, splits <= SLOT_MAX; all
// of a thread's loads are issued before its adds and stores.
constexpr int SLOT_MAX = 16;
__global__ void slot_fold_kernel(float* __restrict__ g, float* __restrict__ slots, long n, int splits) {
  const long n4 = n / 4;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x) {
    float4 v[SLOT_MAX];
#pragma unroll
    for (int s = 0; s < SLOT_MAX; ++s)
      if (s < splits) v[s] = reinterpret_cast<const float4*>(slots + s * n)[i];
    float4 acc = reinterpret_cast<const float4*>(g)[i];
#pragma unroll
    for (int s = 0; s < SLOT_MAX; ++s)
      if (s < splits) {
        acc.x += v[s].x;
        acc.y += v[s].y;
        acc.z += v[s].z;
        acc.w += v[s].w;
      }
    reinterpret_cast<float4*>(g)[i] = acc;
#pragma unroll
    for (int s = 0; s < SLOT_MAX; ++s)
      if (s < splits) reinterpret_cast<float4*>(slots + s * n)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dwpe[t] += sum_b dx0[b,t] (in batch order); one thread per 4 columns of a
// position
__global__ void wpe_bwd_kernel(const float* __restrict__ dx, int B, int T, int C, float* __restrict__ dwpe) {
  const int C4 = C / 4;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < (long)T * C4; i += (long)gridDim.x * blockDim.x) {
    const long t = i / C4, c = i % C4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int b = 0; b < B; ++b) {
      const float4 v = reinterpret_cast<const float4*>(dx + ((long)b * T + t) * C)[c];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    float4* d = reinterpret_cast<float4*>(dwpe + t * C) + c;
    const float4 o = *d;
    *d = make_float4(o.x + acc.x, o.y + acc.y, o.z + acc.z, o.w + acc.w);
  }
}

// ------------------------------------------------------------ LayerNorm
// One warp per row, the row held in registers (C = 128 * NV), two-pass
// mean/variance, biased variance, eps 1e-5.  Writes y (bf16 or fp32) and the
// row's mean and rstd.
template <int NV, typename TO>
__global__ void __launch_bounds__(256, 2) ln_fwd_kernel(const float* __restrict__ x, const float* __restrict__ gam,
                                                     const float* __restrict__ bet, TO* __restrict__ y,
                                                     float* __restrict__ mean, float* __restrict__ rstd, int M) {
  constexpr int C = 128 * NV;
  const int lane = threadIdx.x & 31;
  const long nw = (long)gridDim.x * (blockDim.x >> 5);  // warps in the grid: the row stride
  long row = (blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5;
  if (row >= M) return;
  float4 v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = reinterpret_cast<const float4*>(x + row * C)[lane + 32 * i];
  for (;;) {
    // the warp's next row loads while this one is normalised
    const long next = row + nw;
    float4 vn[NV];
    if (next < M) {
#pragma unroll
      for (int i = 0; i < NV; ++i) vn[i] = reinterpret_cast<const float4*>(x + next * C)[lane + 32 * i];
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) s += v[i].x + v[i].y + v[i].z + v[i].w;
    const float mu = warp_sum(s) * (1.f / C);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float a = v[i].x - mu, b = v[i].y - mu, c = v[i].z - mu, d = v[i].w - mu;
      q += a * a + b * b + c * c + d * d;
    }
    const float var = warp_sum(q) * (1.f / C);
    const float rs = rsqrtf(var + 1e-5f);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 4 * (lane + 32 * i);
      const float4 gg = reinterpret_cast<const float4*>(gam)[lane + 32 * i];
      const float4 bb = reinterpret_cast<const float4*>(bet)[lane + 32 * i];
      const float o0 = (v[i].x - mu) * rs * gg.x + bb.x;
      const float o1 = (v[i].y - mu) * rs * gg.y + bb.y;
      const float o2 = (v[i].z - mu) * rs * gg.z + bb.z;
      const float o3 = (v[i].w - mu) * rs * gg.w + bb.w;
      if constexpr (sizeof(TO) == 2) {
        uint2 w = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
        *reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(y) + row * C + c) = w;
      } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + row * C + c) = make_float4(o0, o1, o2, o3);
      }
    }
    if (lane == 0) {
      mean[row] = mu;
      rstd[row] = rs;
    }
    if (next >= M) break;
    row = next;
#pragma unroll
    for (int i = 0; i < NV; ++i) v[i] = vn[i];
  }
}

// LayerNorm backward fused with the residual stream, per row:
//   dxhat = dy*g ; dx = rstd*(dxhat - mean(dxhat) - xhat*mean(dxhat*xhat))
//   dres = (accumulate ? dres : 0) + dx     (fp32, in place)   and a bf16 copy
// and per-block partial column sums (fixed row ranges, fixed order) of
//   dy*xhat (-> dgamma), dy (-> dbeta), dres_out (-> the bias gradient of the
//   linear layer whose output is this residual point).
// A CTA owns a fixed range of rows.  One producer thread streams them into
// shared memory with bulk asynchronous copies (dy, x and the incoming dres of
// LN_BWD_WARPS consecutive rows per stage, one copy per array, LnBwd<NV>::STAGES
// stages), so the bytes in flight do not depend on registers; each compute warp takes one row of a
// stage, reads it from shared memory, writes dres / dres_bf to global memory,
// and keeps its columns' sums in registers.  At the end the warps' sums are
// combined in warp order.  Rows per CTA: a multiple of LN_BWD_WARPS.
constexpr int LN_BWD_WARPS = 7;  // compute warps (with the producer: 256 threads, so 255 registers each)
template <int NV>
struct LnBwd {
  static constexpr int C = 128 * NV;
  static constexpr int ROW = 3 * C;                     // floats per staged row: dy, x, dres
  static constexpr int STAGES = NV <= 6 ? 3 : 2;
  static constexpr int STAGE_FLOATS = LN_BWD_WARPS * ROW;
  static size_t smem_bytes(int rpb) { return (size_t)STAGES * STAGE_FLOATS * 4 + (size_t)2 * rpb * 4 + 2 * STAGES * 8; }
};
template <int NV>
__global__ void __launch_bounds__(32 * (LN_BWD_WARPS + 1), 1)
    ln_bwd_kernel(const float* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ mean,
                  const float* __restrict__ rstd, const float* __restrict__ gam, float* __restrict__ dres,
                  bf16* __restrict__ dres_bf, int M, int rows_per_block, int accumulate, float* __restrict__ part) {
  using L = LnBwd<NV>;
  constexpr int C = L::C, S = L::STAGES, W = LN_BWD_WARPS;
  extern __shared__ float4 ln_smem4[];
  float* stage = reinterpret_cast<float*>(ln_smem4);  // [S][dy | x | dres][W][C]
  float* mr = stage + S * L::STAGE_FLOATS;              // mean [rows_per_block], rstd [rows_per_block]
  uint64_t* full = reinterpret_cast<uint64_t*>(mr + 2 * rows_per_block);
  uint64_t* empty = full + S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long r0 = (long)blockIdx.x * rows_per_block;
  const int nrows = (int)(min((long)M, r0 + rows_per_block) - r0);
  const int nbatch = (nrows + W - 1) / W;
  for (int i = threadIdx.x; i < nrows; i += blockDim.x) {
    mr[i] = mean[r0 + i];
    mr[rows_per_block + i] = rstd[r0 + i];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tcg::mbar_init(&full[s], 1);
      tcg::mbar_init(&empty[s], W);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  float4 adg[NV], adb[NV], adr[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) adg[i] = adb[i] = adr[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (warp == W) {
    if (lane == 0) {
      // ------------------------------------------------------ producer
      bool ok = true;
      int issued = 0;
      for (int k = 0; k < nbatch; ++k, ++issued) {
        const int s = k % S;
        if (!tcg::mbar_wait(&empty[s], ((k / S) & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        // the batch's rows are contiguous in each array: one copy per array
        const int nr = min(W, nrows - k * W);
        const uint32_t bytes = (uint32_t)(nr * C * 4);
        const long row = r0 + (long)k * W;
        float* dst = stage + (long)s * L::STAGE_FLOATS;
        tcg::mbar_expect_tx(&full[s], (accumulate ? 3 : 2) * bytes);
        tcfa::bulk_load(tcg::smem_u32(dst), dy + row * C, bytes, &full[s]);
        tcfa::bulk_load(tcg::smem_u32(dst + W * C), x + row * C, bytes, &full[s]);
        if (accumulate) tcfa::bulk_load(tcg::smem_u32(dst + 2 * W * C), dres + row * C, bytes, &full[s]);
      }
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tcfa::drain_ring(full, S, (uint32_t)issued);
    }
  } else {
    // ------------------------------------------------- compute warps
    float4 g[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) g[i] = reinterpret_cast<const float4*>(gam)[lane + 32 * i];
    bool ok = true;
    for (int k = 0; k < nbatch; ++k) {
      const int s = k % S;
      if (!tcfa::warp_wait(&full[s], (k / S) & 1u)) {
        ok = false;
        break;
      }
      const int ri = k * W + warp;
      if (ri < nrows) {
        const long row = r0 + ri;
        // this warp's row of the stage's dy, x and dres blocks
        const float4* src = reinterpret_cast<const float4*>(stage + (long)s * L::STAGE_FLOATS + warp * C);
        const float mu = mr[ri], rs = mr[rows_per_block + ri];
        float4 dyv[NV], xv[NV];
        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          dyv[i] = src[lane + 32 * i];
          const float4 xr = src[W * C / 4 + lane + 32 * i];
          xv[i] = make_float4((xr.x - mu) * rs, (xr.y - mu) * rs, (xr.z - mu) * rs, (xr.w - mu) * rs);
          const float d0 = dyv[i].x * g[i].x, d1 = dyv[i].y * g[i].y, d2 = dyv[i].z * g[i].z, d3 = dyv[i].w * g[i].w;
          s1 += d0 + d1 + d2 + d3;
          s2 += d0 * xv[i].x + d1 * xv[i].y + d2 * xv[i].z + d3 * xv[i].w;
        }
        s1 = warp_sum(s1) * (1.f / C);
        s2 = warp_sum(s2) * (1.f / C);
        float4* dr = reinterpret_cast<float4*>(dres + row * C) + lane;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int c4 = lane + 32 * i;
          const float4 rv = accumulate ? src[W * C / 2 + c4] : make_float4(0.f, 0.f, 0.f, 0.f);
          float4 o;
          o.x = rv.x + rs * (dyv[i].x * g[i].x - s1 - xv[i].x * s2);
          o.y = rv.y + rs * (dyv[i].y * g[i].y - s1 - xv[i].y * s2);
          o.z = rv.z + rs * (dyv[i].z * g[i].z - s1 - xv[i].z * s2);
          o.w = rv.w + rs * (dyv[i].w * g[i].w - s1 - xv[i].w * s2);
          dr[32 * i] = o;
          if (dres_bf != nullptr)
            reinterpret_cast<uint2*>(dres_bf + row * C)[c4] = make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
          adg[i].x += dyv[i].x * xv[i].x;
          adg[i].y += dyv[i].y * xv[i].y;
          adg[i].z += dyv[i].z * xv[i].z;
          adg[i].w += dyv[i].w * xv[i].w;
          adb[i].x += dyv[i].x;
          adb[i].y += dyv[i].y;
          adb[i].z += dyv[i].z;
          adb[i].w += dyv[i].w;
          adr[i].x += o.x;
          adr[i].y += o.y;
          adr[i].z += o.z;
          adr[i].w += o.w;
        }
      }
      __syncwarp();
      if (lane == 0) tcg::mbar_arrive(&empty[s]);
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
  }
  __syncthreads();  // every row is done and every copy has landed: the stages are free
  // combine the warps' column sums in warp order
  float4* acc = reinterpret_cast<float4*>(stage);  // [W][3][C/4]
  if (warp < W) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c4 = lane + 32 * i;
      acc[(warp * 3 + 0) * (C / 4) + c4] = adg[i];
      acc[(warp * 3 + 1) * (C / 4) + c4] = adb[i];
      acc[(warp * 3 + 2) * (C / 4) + c4] = adr[i];
    }
  }
  __syncthreads();
  const float* af = reinterpret_cast<const float*>(acc);
  for (int idx = threadIdx.x; idx < 3 * C; idx += blockDim.x) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) t += af[w * 3 * C + idx];
    part[(long)blockIdx.x * 3 * C + idx] += t;  // (accumulates over the micro-steps)
  }
}

// Sum per-block partial rows (fixed order) into up to three outputs:
// part is [nblk][ncols]; column j goes to out[j / C][j % C] (+=).  A cluster
// of PR_SPLIT CTAs serves 32 columns: warp w of CTA y sums the partial rows
// b = 8y + w (mod 8*PR_SPLIT) in ascending order, each CTA combines its warps
// in warp order, and CTA 0 adds the CTAs' sums in rank order through
// distributed shared memory, so the result is independent of timing.
constexpr int PR_SPLIT = 8;
__global__ void __cluster_dims__(1, PR_SPLIT, 1) __launch_bounds__(256)
    partials_reduce_kernel(const float* __restrict__ part, int nblk, int ncols, int C, float* __restrict__ out0,
                           float* __restrict__ out1, float* __restrict__ out2) {
  __shared__ float red[8][32];
  __shared__ float tot[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + lane;
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  float s = 0.f;
  if (col < ncols) {
#pragma unroll 4
    for (int b = 8 * (int)rank + warp; b < nblk; b += 8 * PR_SPLIT) s += part[(long)b * ncols + col];
  }
  red[warp][lane] = s;
  __syncthreads();
  if (warp == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][lane];
    tot[lane] = t;
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (rank == 0 && warp == 0) {
    const uint32_t local = (uint32_t)__cvta_generic_to_shared(&tot[lane]);
    float t = 0.f;
#pragma unroll
    for (uint32_t r = 0; r < PR_SPLIT; ++r) {
      uint32_t remote;
      float v;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(r));
      asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
      t += v;
    }
    if (col < ncols) {
      const int which = col / C, c = col % C;
      float* o = which == 0 ? out0 : (which == 1 ? out1 : out2);
      if (o != nullptr) o[c] += t;
    }
  }
  // no CTA leaves while CTA 0 may still read its shared memory
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Column sums of an [M, N] matrix, stage 1: block (x, y) sums 32 column
// groups of 16 bytes (8 bf16 or 4 fp32 columns each) over rows
// [y*rows_per_block, ...), 8 row lanes per group, combined in lane order.
// N must be a multiple of 16 / sizeof(T).
template <typename T>
__global__ void __launch_bounds__(256) colsum_partial_kernel(const T* __restrict__ a, int M, int N, int rows_per_block,
                                                             float* __restrict__ part) {
  constexpr int VEC = 16 / sizeof(T);
  __shared__ float red[8][32 * VEC];
  const int cg = threadIdx.x & 31, rl = threadIdx.x >> 5;
  const int c0 = (blockIdx.x * 32 + cg) * VEC;
  const int r0 = blockIdx.y * rows_per_block;
  const int r1 = min(M, r0 + rows_per_block);
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
  if (c0 < N) {
#pragma unroll 8
    for (int r = r0 + rl; r < r1; r += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(a + (long)r * N + c0);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] += ld_f(e + i);
    }
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) red[rl][cg * VEC + i] = acc[i];
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * VEC; i += 256) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w][i];
    const int col = blockIdx.x * 32 * VEC + i;
    if (col < N) part[(long)blockIdx.y * N + col] += t;  // (accumulates over the micro-steps)
  }
}

// ------------------------------------------------------- cross-entropy
// One CTA per row of logits z[M, V] (the row kept in shared memory):
//   lse = max + log(sum exp(z - max)); loss_row = lse - z[y]; argmax (lowest
//   index among maxima).  When write_grad, the row is overwritten in place by
//   dz = (exp(z - lse) - [j == y]) * gscale.
// One pass over global memory in and (with write_grad) one out: the load pass
// keeps a per-thread running (max, argmax, sum of exp) with rescaling per
// 16-byte chunk, and the gradient pass reads and writes 16-byte chunks.
// V * sizeof(T) must be a multiple of 16.
constexpr float CE_LOG2E = 1.4426950408889634f;
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
template <typename T>
__device__ __forceinline__ void ce_combine(float& m, float& s, int& i, float om, float os, int oi) {
  // merge (m, s, i) with (om, os, oi): max, rescaled sum, lowest argmax
  const float nm = fmaxf(m, om);
  const float a = (m == -INFINITY) ? 0.f : exp2_approx((m - nm) * CE_LOG2E);
  const float b = (om == -INFINITY) ? 0.f : exp2_approx((om - nm) * CE_LOG2E);
  s = s * a + os * b;
  if (om > m || (om == m && oi < i)) i = oi;
  m = nm;
}

template <typename T>
__global__ void __launch_bounds__(1024) ce_kernel(T* __restrict__ z, const int32_t* __restrict__ y, int V,
                                                  float* __restrict__ lse_out, float* __restrict__ loss_row,
                                                  int32_t* __restrict__ amax_out, int write_grad, float gscale) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  uint4* row_s = reinterpret_cast<uint4*>(sm_raw);
  __shared__ float red_m[32], red_s[32];
  __shared__ int red_i[32];
  const long row = blockIdx.x;
  T* zr = z + row * (long)V;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  constexpr int EPC = 16 / sizeof(T);
  const int nch = V / EPC;
  float m = -INFINITY, se = 0.f;
  int mi = 0x7fffffff;
  for (int c = tid; c < nch; c += blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(zr)[c];
    row_s[c] = u;
    const T* e = reinterpret_cast<const T*>(&u);
    float v[EPC];
    float cm = -INFINITY;
    int ci = 0;
#pragma unroll
    for (int k = 0; k < EPC; ++k) {
      v[k] = ld_f(e + k);
      if (v[k] > cm) {
        cm = v[k];
        ci = c * EPC + k;
      }
    }
    float cs = 0.f;
    const float ncm = -cm * CE_LOG2E;
#pragma unroll
    for (int k = 0; k < EPC; ++k) cs += exp2_approx(fmaf(v[k], CE_LOG2E, ncm));
    ce_combine<T>(m, se, mi, cm, cs, ci);
  }
  // (max, sum, lowest argmax) across the warp, then across warps
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o);
    const float os = __shfl_xor_sync(0xffffffffu, se, o);
    const int oi = __shfl_xor_sync(0xffffffffu, mi, o);
    ce_combine<T>(m, se, mi, om, os, oi);
  }
  if (lane == 0) {
    red_m[warp] = m;
    red_s[warp] = se;
    red_i[warp] = mi;
  }
  __syncthreads();
  if (warp == 0) {
    m = lane < nw ? red_m[lane] : -INFINITY;
    se = lane < nw ? red_s[lane] : 0.f;
    mi = lane < nw ? red_i[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, m, o);
      const float os = __shfl_xor_sync(0xffffffffu, se, o);
      const int oi = __shfl_xor_sync(0xffffffffu, mi, o);
      ce_combine<T>(m, se, mi, om, os, oi);
    }
    if (lane == 0) {
      red_m[0] = m;
      red_s[0] = se;
      red_i[0] = mi;
    }
  }
  __syncthreads();
  const float lse = red_m[0] + logf(red_s[0]);
  const int tgt = y ? y[row] : -1;
  if (tid == 0) {
    if (lse_out) lse_out[row] = lse;
    if (amax_out) amax_out[row] = red_i[0];
    if (loss_row) {
      float zt = 0.f;
      if (tgt >= 0 && tgt < V) zt = ld_f(reinterpret_cast<const T*>(row_s) + tgt);
      loss_row[row] = (tgt >= 0 && tgt < V) ? lse - zt : 0.f;
    }
  }
  if (write_grad) {
    // gscale * exp(z - lse) = 2^(z*log2(e) + log2(gscale) - lse*log2(e)): one FFMA and one ex2
    const float off = __log2f(gscale) - lse * CE_LOG2E;
    for (int c = tid; c < nch; c += blockDim.x) {
      const uint4 u = row_s[c];
      const T* e = reinterpret_cast<const T*>(&u);
      uint4 w;
      T* o = reinterpret_cast<T*>(&w);
#pragma unroll
      for (int k = 0; k < EPC; ++k) {
        float p = exp2_approx(fmaf(ld_f(e + k), CE_LOG2E, off));
        if (c * EPC + k == tgt) p -= gscale;
        st_f(o + k, p);
      }
      reinterpret_cast<uint4*>(zr)[c] = w;
    }
  }
}

// Cross-entropy from the lm_head GEMM's softmax statistics (bf16 mode).  The
// GEMM epilogue stored the bf16 logits z[M, V] and, per row and half tile of
// 128 columns, (max, sum of exp(z - max), lowest argmax) of the stored values.
// One CTA per row merges the row's partials in a fixed order:
//   lse = max + log(sum);  loss_row = lse - z[y];  argmax (lowest index)
// and, when write_grad, streams the row once, overwriting it in place with
//   dz = (exp(z - lse) - [j == y]) * gscale.
// V must be a multiple of 8.
constexpr int CEF_THREADS = 256;
__global__ void __launch_bounds__(CEF_THREADS) ce_finish_kernel(bf16* __restrict__ z, const float* __restrict__ part,
                                                               int nh, const int32_t* __restrict__ y, int V,
                                                               float* __restrict__ lse_out,
                                                               float* __restrict__ loss_row,
                                                               int32_t* __restrict__ amax_out, int write_grad,
                                                               float gscale) {
  __shared__ float red_m[CEF_THREADS / 32], red_s[CEF_THREADS / 32];
  __shared__ int red_i[CEF_THREADS / 32];
  const long row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float m = -INFINITY, s = 0.f;
  int mi = 0x7fffffff;
  const float* pr = part + row * (long)nh * 3;
  for (int k = tid; k < nh; k += CEF_THREADS)
    softmax_stats_merge(m, s, mi, pr[3 * k], pr[3 * k + 1], __float_as_int(pr[3 * k + 2]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o);
    const float os = __shfl_xor_sync(0xffffffffu, s, o);
    const int oi = __shfl_xor_sync(0xffffffffu, mi, o);
    softmax_stats_merge(m, s, mi, om, os, oi);
  }
  if (lane == 0) {
    red_m[warp] = m;
    red_s[warp] = s;
    red_i[warp] = mi;
  }
  __syncthreads();
  m = red_m[0];
  s = red_s[0];
  mi = red_i[0];
#pragma unroll
  for (int w = 1; w < CEF_THREADS / 32; ++w) softmax_stats_merge(m, s, mi, red_m[w], red_s[w], red_i[w]);
  const float lse = m + logf(s);
  bf16* zr = z + row * (long)V;
  const int tgt = y ? y[row] : -1;
  if (tid == 0) {
    if (lse_out) lse_out[row] = lse;
    if (amax_out) amax_out[row] = mi;
    if (loss_row) loss_row[row] = (tgt >= 0 && tgt < V) ? lse - bf2f(zr[tgt]) : 0.f;
  }
  if (!write_grad) return;
  // every thread read the target logit above (tid 0) before any row chunk is
  // overwritten: the target's chunk is written by a thread that first syncs
  __syncthreads();
  // gscale * exp(z - lse) = 2^(z*log2(e) + log2(gscale) - lse*log2(e)): one FFMA and one ex2
  const float off = __log2f(gscale) - lse * LOG2E_F;
  const int nch = V / 8;
  uint4* zc = reinterpret_cast<uint4*>(zr);
  for (int c0 = tid; c0 < nch; c0 += 4 * CEF_THREADS) {
    uint4 u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (c0 + k * CEF_THREADS < nch) u[k] = zc[c0 + k * CEF_THREADS];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = c0 + k * CEF_THREADS;
      if (c >= nch) break;
      uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16x2(w[e]);
        float p0 = ex2_approx(fmaf(f.x, LOG2E_F, off));
        float p1 = ex2_approx(fmaf(f.y, LOG2E_F, off));
        if (c * 8 + 2 * e == tgt) p0 -= gscale;
        if (c * 8 + 2 * e + 1 == tgt) p1 -= gscale;
        w[e] = pack_bf16x2(p0, p1);
      }
      zc[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// dz = (exp(z - lse) - onehot) * gscale in place, from the saved lse
template <typename T>
__global__ void ce_bwd_kernel(T* __restrict__ z, const int32_t* __restrict__ y, const float* __restrict__ lse, int V,
                              float gscale) {
  const long row = blockIdx.x;
  T* zr = z + row * (long)V;
  const float off = __log2f(gscale) - lse[row] * CE_LOG2E;  // the same expression as ce_kernel's
  const int tgt = y[row];
  for (int j = threadIdx.x; j < V; j += blockDim.x) {
    float p = exp2_approx(fmaf(ld_f(zr + j), CE_LOG2E, off));
    if (j == tgt) p -= gscale;
    st_f(zr + j, p);
  }
}

// mean of the row losses into *loss (+= when accumulate), fixed order, 1 CTA
__global__ void loss_mean_kernel(const float* __restrict__ rows, int M, float* __restrict__ loss, float* __restrict__ acc,
                                 float acc_scale) {
  __shared__ float red[32];
  float s = 0.f;
  for (int i = threadIdx.x; i < M; i += blockDim.x) s += rows[i];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    s = warp_sum(s);
    if (threadIdx.x == 0) {
      const float m = s / (float)M;
      *loss = m;
      if (acc) *acc += m * acc_scale;
    }
  }
}

// ------------------------------------------------------------ optimizer
// sum of squares of the flat gradient, stage 1: per-block partials (fixed
// chunking: block b owns a contiguous range), fp64 accumulation
__global__ void sumsq_partial_kernel(const float* __restrict__ g, long n, long per_block, double* __restrict__ part) {
  __shared__ double red[32];
  const long lo = blockIdx.x * per_block;
  const long hi = min(n, lo + per_block);
  double s = 0.0;
  for (long i = lo + threadIdx.x * 4; i < hi; i += (long)blockDim.x * 4) {
    if (i + 3 < hi) {
      const float4 v = *reinterpret_cast<const float4*>(g + i);
      s += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
    } else {
      for (long j = i; j < hi; ++j) s += (double)g[j] * g[j];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    part[blockIdx.x] = t;
  }
}
// stage 2, 1 CTA of 32 threads: out = [norm, clip scale, finite flag, bias
// correction 1 - b1^t, bias correction 1 - b2^t]; the step counter t advances
// only when the norm is finite (a non-finite norm skips the update).
__global__ void norm_finish_kernel(const double* __restrict__ part, int nblk, float max_norm, float b1, float b2,
                                   float* __restrict__ out, long long* __restrict__ step) {
  double s = 0.0;
  for (int i = threadIdx.x; i < nblk; i += 32) s += part[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (threadIdx.x == 0) {
    const double n = sqrt(s);
    const bool fin = isfinite(n);
    out[0] = (float)n;
    const double sc = (double)max_norm / (n + 1e-6);
    out[1] = (float)(sc < 1.0 ? sc : 1.0);
    out[2] = fin ? 1.f : 0.f;
    long long t = *step;
    if (fin) {
      t += 1;
      *step = t;
    }
    out[3] = (float)(1.0 - pow((double)b1, (double)t));
    out[4] = (float)(1.0 - pow((double)b2, (double)t));
  }
}

struct AdamSeg {
  long begin;  // first flat index of a tensor (segments sorted, contiguous)
  int decay;
};

// One launch over the whole flat arena.  Segment table in shared memory; each
// thread handles 4 consecutive elements (every tensor size is a multiple of 4).
//   g' = g * clip;  p *= (1 - lr*wd*decay);  m = b1 m + (1-b1) g';
//   v = b2 v + (1-b2) g'^2;  p -= lr * (m / bc1) / (sqrt(v / bc2) + eps)
// Skipped entirely (params untouched) when the norm is not finite.
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    bf16* __restrict__ pbf, long n, const AdamSeg* __restrict__ segs,
                                                    int nseg, const float* __restrict__ normbuf, float lr, float wd,
                                                    float b1, float b2, float eps) {
  __shared__ long s_begin[160];
  __shared__ int s_decay[160];
  for (int i = threadIdx.x; i < nseg; i += blockDim.x) {
    s_begin[i] = segs[i].begin;
    s_decay[i] = segs[i].decay;
  }
  __syncthreads();
  if (normbuf[2] == 0.f) return;
  const float clip = normbuf[1];
  const float bc1 = normbuf[3], bc2 = normbuf[4];
  const float rbc2 = rsqrtf(bc2);
  const float step = lr / bc1;
  for (long i = (blockIdx.x * (long)blockDim.x + threadIdx.x) * 4; i < n; i += (long)gridDim.x * blockDim.x * 4) {
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_begin[mid] <= i)
        lo = mid;
      else
        hi = mid - 1;
    }
    const float dec = s_decay[lo] ? (1.f - lr * wd) : 1.f;
    float4 pv = *reinterpret_cast<float4*>(p + i);
    const float4 gv = *reinterpret_cast<const float4*>(g + i);
    float4 mv = *reinterpret_cast<float4*>(m + i);
    float4 vv = *reinterpret_cast<float4*>(v + i);
    float pa[4] = {pv.x, pv.y, pv.z, pv.w}, ga[4] = {gv.x, gv.y, gv.z, gv.w};
    float ma[4] = {mv.x, mv.y, mv.z, mv.w}, va[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float gg = ga[e] * clip;
      ma[e] = b1 * ma[e] + (1.f - b1) * gg;
      va[e] = b2 * va[e] + (1.f - b2) * gg * gg;
      const float denom = sqrtf(va[e]) * rbc2 + eps;
      pa[e] = pa[e] * dec - step * ma[e] / denom;
    }
    *reinterpret_cast<float4*>(p + i) = make_float4(pa[0], pa[1], pa[2], pa[3]);
    *reinterpret_cast<float4*>(m + i) = make_float4(ma[0], ma[1], ma[2], ma[3]);
    *reinterpret_cast<float4*>(v + i) = make_float4(va[0], va[1], va[2], va[3]);
    if (pbf != nullptr)
      *reinterpret_cast<uint2*>(pbf + i) = make_uint2(pack_bf16x2(pa[0], pa[1]), pack_bf16x2(pa[2], pa[3]));
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ a, bf16* __restrict__ b, long n) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    b[i] = f2bf(a[i]);
}

// ------------------------------------------------------------ init
// counter-based N(0, std): splitmix64 of (seed, index) -> two uniforms ->
// Box-Muller (cosine branch)
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}
__global__ void init_normal_kernel(float* __restrict__ p, long n, uint64_t seed, long offset, float std) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const uint64_t h = splitmix64(seed * 0x2545F4914F6CDD1Dull + (uint64_t)(offset + i));
    const float u1 = ((float)(h >> 40) + 1.f) * (1.f / 16777217.f);  // (0, 1]
    const float u2 = (float)((h >> 16) & 0xFFFFFFu) * (1.f / 16777216.f);
    p[i] = std * sqrtf(-2.f * logf(u1)) * cospif(2.f * u2);
  }
}
__global__ void fill_kernel(float* __restrict__ p, long n, float v) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) p[i] = v;
}

}  // namespace k
