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
// bf16 backward (d = 64): flash-style tiling, bf16 tensor-core MMAs (m16n8k16)
// with fp32 accumulation; S and P never leave the chip.  Two deterministic
// kernels (no atomics): one owns a key block and produces dk, dv; the other owns
// a query block and produces dq.  (The bf16 forward is the tcgen05 kernel in
// attention_tc.cuh.)
// fp32 path: plain per-row kernels (fp32 parity mode, small shapes).
#pragma once
#include "common.cuh"

namespace attn {

constexpr int HD = 64;   // head dim of the bf16 path
constexpr int BQ = 64;   // query rows per CTA
constexpr int BKV = 64;  // keys per tile
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte offset of element (r, c) of a [64][64] bf16 tile with 16-byte chunks
// XOR-swizzled by row (conflict-free ldmatrix)
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// load rows [row0, row0+64) x 64 columns of a row-major bf16 matrix (row
// stride ld elements) into a swizzled tile; rows >= nrows are zero-filled.
__device__ __forceinline__ void load_tile(uint8_t* tile, const bf16* g, long ld, int row0, int nrows) {
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(tile);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = threadIdx.x + i * 128;  // 512 chunks of 16 B
    const int r = idx >> 3, ch = idx & 7;
    const int gr = row0 + r;
    const bool ok = gr < nrows;
    const bf16* src = g + (long)(ok ? gr : 0) * ld + ch * 8;
    cp_async16(base + swz(r, ch * 8), src, ok ? 16 : 0);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragments (16 rows x 64 cols, 4 k-steps) of rows [r0, r0+16) of a tile
__device__ __forceinline__ void load_a_frags(const uint8_t* tile, int r0, uint32_t (&f)[4][4]) {
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(tile);
  const int lane = threadIdx.x & 31;
  const int r = r0 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int c = kk * 16 + 8 * (lane >> 4);
    ldsm_x4(base + swz(r, c), f[kk][0], f[kk][1], f[kk][2], f[kk][3]);
  }
}

// acc[16 x 64] += A(16 x 64, registers) . tile_rows^T where the tile holds 64
// rows of the "n" operand, each with 64 "k" values (B stored [n][k]).
__device__ __forceinline__ void mma_a_bt(float (&acc)[8][4], const uint32_t (&a)[4][4], const uint8_t* tile) {
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(tile);
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int n = p * 16 + (lane & 7) + 8 * (lane >> 4);
      const int k = kk * 16 + 8 * ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(base + swz(n, k), b0, b1, b2, b3);
      mma16816(acc[2 * p], a[kk], b0, b1);
      mma16816(acc[2 * p + 1], a[kk], b2, b3);
    }
  }
}

// acc[16 x 64] += P(16 x 64, registers, K = tile rows) . tile where the tile
// holds 64 rows of "k", each with 64 "n" values (B stored [k][n]).
__device__ __forceinline__ void mma_a_b(float (&acc)[8][4], const uint32_t (&a)[4][4], const uint8_t* tile) {
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(tile);
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int k = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
      const int n = p * 16 + 8 * (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(base + swz(k, n), b0, b1, b2, b3);
      mma16816(acc[2 * p], a[kk], b0, b1);
      mma16816(acc[2 * p + 1], a[kk], b2, b3);
    }
  }
}

// C fragments of a 16 x 64 fp32 tile -> bf16 A fragments (K = 64)
__device__ __forceinline__ void c_to_a(const float (&c)[8][4], uint32_t (&a)[4][4]) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    a[kk][0] = pack_bf16x2(c[2 * kk][0], c[2 * kk][1]);
    a[kk][1] = pack_bf16x2(c[2 * kk][2], c[2 * kk][3]);
    a[kk][2] = pack_bf16x2(c[2 * kk + 1][0], c[2 * kk + 1][1]);
    a[kk][3] = pack_bf16x2(c[2 * kk + 1][2], c[2 * kk + 1][3]);
  }
}

// ------------------------------------------------------------ backward
// D[b,h,t] = sum_d do[b,t,h,d] * o[b,t,h,d]
__global__ void bwd_dot_kernel(const bf16* __restrict__ o, const bf16* __restrict__ dout, float* __restrict__ Dv,
                               int B, int T, int H) {
  const int C = H * HD;
  const long rows = (long)B * T * H;
  const int lane = threadIdx.x & 31;
  for (long w = (blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5; w < rows;
       w += ((long)gridDim.x * blockDim.x) >> 5) {
    const long bt = w / H;
    const int h = (int)(w % H);
    const long off = bt * C + h * HD + 2 * lane;
    const float2 a = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(o + off));
    const float2 c = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(dout + off));
    float s = warp_sum(a.x * c.x + a.y * c.y);
    if (lane == 0) {
      const long b = bt / T, t = bt % T;
      Dv[(b * H + h) * T + t] = s;
    }
  }
}

// one CTA per key block: dk, dv for its 64 keys (warp w owns keys 16w..16w+15)
__global__ void __launch_bounds__(128) flash_bwd_dkdv_kernel(const bf16* __restrict__ qkv, const bf16* __restrict__ dout,
                                                             const float* __restrict__ lse,
                                                             const float* __restrict__ Dv, bf16* __restrict__ dqkv,
                                                             int T, int H, float scale, float sl2) {
  // dynamic shared memory: K, V tiles, two (Q, dO) tiles, two (lse, D) rows
  extern __shared__ __align__(128) uint8_t dkdv_smem[];
  uint8_t* sK = dkdv_smem;
  uint8_t* sV = dkdv_smem + 8192;
  uint8_t* sQ[2] = {dkdv_smem + 16384, dkdv_smem + 24576};
  uint8_t* sO[2] = {dkdv_smem + 32768, dkdv_smem + 40960};
  float(*sL)[64] = reinterpret_cast<float(*)[64]>(dkdv_smem + 49152);
  float(*sD)[64] = reinterpret_cast<float(*)[64]>(dkdv_smem + 49152 + 512);
  const int kb = blockIdx.x;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD;
  const long ld = 3L * C;
  const bf16* Qg = qkv + (long)b * T * ld + h * HD;
  const bf16* Kg = Qg + C;
  const bf16* Vg = Qg + 2 * C;
  const bf16* dOg = dout + (long)b * T * C + h * HD;
  const float* Lg = lse + ((long)b * H + h) * T;
  const float* Dg = Dv + ((long)b * H + h) * T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int nqb = (T + BQ - 1) / BQ;

  load_tile(sK, Kg, ld, kb * BKV, T);
  load_tile(sV, Vg, ld, kb * BKV, T);
  auto load_q = [&](int i, int buf) {
    load_tile(sQ[buf], Qg, ld, i * BQ, T);
    load_tile(sO[buf], dOg, C, i * BQ, T);
    if (threadIdx.x < 64) {
      const int qr = i * BQ + threadIdx.x;
      sL[buf][threadIdx.x] = qr < T ? Lg[qr] * LOG2E : INFINITY;
      sD[buf][threadIdx.x] = qr < T ? Dg[qr] : 0.f;
    }
  };
  load_q(kb, 0);
  cp_commit();

  uint32_t kf[4][4], vf[4][4];
  float dk[8][4] = {}, dv[8][4] = {};
  const int key0 = kb * BKV + warp * 16 + g;  // this thread's keys: key0, key0 + 8

  for (int i = kb; i < nqb; ++i) {
    const int buf = (i - kb) & 1;
    cp_wait<0>();
    __syncthreads();
    if (i + 1 < nqb) load_q(i + 1, buf ^ 1);
    cp_commit();
    if (i == kb) {
      load_a_frags(sK, warp * 16, kf);
      load_a_frags(sV, warp * 16, vf);
    }
    // S^T (keys x queries) and dP^T
    float st[8][4] = {}, dpt[8][4] = {};
    mma_a_bt(st, kf, sQ[buf]);
    mma_a_bt(dpt, vf, sO[buf]);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = nt * 8 + 2 * t4 + (e & 1);
        const int qr = i * BQ + ql;
        const int key = key0 + ((e >> 1) << 3);
        float p = ex2(st[nt][e] * sl2 - sL[buf][ql]);
        if (qr < key) p = 0.f;
        st[nt][e] = p;
        dpt[nt][e] = p * (dpt[nt][e] - sD[buf][ql]);
      }
    uint32_t pf[4][4], dsf[4][4];
    c_to_a(st, pf);
    c_to_a(dpt, dsf);
    mma_a_b(dv, pf, sO[buf]);
    mma_a_b(dk, dsf, sQ[buf]);
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int key = key0 + hr * 8;
    if (key < T) {
      bf16* krow = dqkv + ((long)b * T + key) * ld + C + h * HD;
      bf16* vrow = krow + C;
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        *reinterpret_cast<uint32_t*>(krow + dt * 8 + 2 * t4) =
            pack_bf16x2(dk[dt][2 * hr] * scale, dk[dt][2 * hr + 1] * scale);
        *reinterpret_cast<uint32_t*>(vrow + dt * 8 + 2 * t4) = pack_bf16x2(dv[dt][2 * hr], dv[dt][2 * hr + 1]);
      }
    }
  }
}

// one CTA per query block: dq for its 64 queries (warp w owns queries 16w..)
__global__ void __launch_bounds__(128) flash_bwd_dq_kernel(const bf16* __restrict__ qkv, const bf16* __restrict__ dout,
                                                           const float* __restrict__ lse, const float* __restrict__ Dv,
                                                           bf16* __restrict__ dqkv, int T, int H, float scale,
                                                           float sl2) {
  __shared__ __align__(128) uint8_t sQ[64 * 128];
  __shared__ __align__(128) uint8_t sO[64 * 128];
  __shared__ __align__(128) uint8_t sK[2][64 * 128];
  __shared__ __align__(128) uint8_t sV[2][64 * 128];
  const int qb = gridDim.x - 1 - blockIdx.x;
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD;
  const long ld = 3L * C;
  const bf16* Qg = qkv + (long)b * T * ld + h * HD;
  const bf16* Kg = Qg + C;
  const bf16* Vg = Qg + 2 * C;
  const bf16* dOg = dout + (long)b * T * C + h * HD;
  const float* Lg = lse + ((long)b * H + h) * T;
  const float* Dg = Dv + ((long)b * H + h) * T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;

  load_tile(sQ, Qg, ld, qb * BQ, T);
  load_tile(sO, dOg, C, qb * BQ, T);
  load_tile(sK[0], Kg, ld, 0, T);
  load_tile(sV[0], Vg, ld, 0, T);
  cp_commit();

  const int q_row0 = qb * BQ + warp * 16 + g;
  float lrow[2], drow[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int qr = q_row0 + hr * 8;
    lrow[hr] = qr < T ? Lg[qr] * LOG2E : INFINITY;
    drow[hr] = qr < T ? Dg[qr] : 0.f;
  }
  uint32_t qf[4][4], of[4][4];
  float dq[8][4] = {};
  const int nkv = qb + 1;
  for (int j = 0; j < nkv; ++j) {
    cp_wait<0>();
    __syncthreads();
    if (j + 1 < nkv) {
      load_tile(sK[(j + 1) & 1], Kg, ld, (j + 1) * BKV, T);
      load_tile(sV[(j + 1) & 1], Vg, ld, (j + 1) * BKV, T);
    }
    cp_commit();
    if (j == 0) {
      load_a_frags(sQ, warp * 16, qf);
      load_a_frags(sO, warp * 16, of);
    }
    float s[8][4] = {}, dp[8][4] = {};
    mma_a_bt(s, qf, sK[j & 1]);
    mma_a_bt(dp, of, sV[j & 1]);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1;
        const int key = j * BKV + nt * 8 + 2 * t4 + (e & 1);
        const int qr = q_row0 + hr * 8;
        float p = ex2(s[nt][e] * sl2 - lrow[hr]);
        if (key > qr) p = 0.f;
        s[nt][e] = p * (dp[nt][e] - drow[hr]);
      }
    uint32_t dsf[4][4];
    c_to_a(s, dsf);
    mma_a_b(dq, dsf, sK[j & 1]);
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int qr = q_row0 + hr * 8;
    if (qr < T) {
      bf16* row = dqkv + ((long)b * T + qr) * ld + h * HD;
#pragma unroll
      for (int dt = 0; dt < 8; ++dt)
        *reinterpret_cast<uint32_t*>(row + dt * 8 + 2 * t4) =
            pack_bf16x2(dq[dt][2 * hr] * scale, dq[dt][2 * hr + 1] * scale);
    }
  }
}

// Dv: caller-provided fp32 scratch of B*H*T elements
static inline cudaError_t flash_backward(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                                         bf16* dqkv, float* Dv, int B, int T, int H, cudaStream_t st) {
  const float scale = 1.f / sqrtf((float)HD);
  const float sl2 = LOG2E * scale;
  const long rows = (long)B * T * H;
  int blocks = (int)((rows * 32 + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  bwd_dot_kernel<<<blocks, 256, 0, st>>>(out, dout, Dv, B, T, H);
  dim3 grid((T + BQ - 1) / BQ, B * H);
  constexpr int DKDV_SMEM = 49152 + 1024;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(flash_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKDV_SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  flash_bwd_dkdv_kernel<<<grid, 128, DKDV_SMEM, st>>>(qkv, dout, lse, Dv, dqkv, T, H, scale, sl2);
  flash_bwd_dq_kernel<<<grid, 128, 0, st>>>(qkv, dout, lse, Dv, dqkv, T, H, scale, sl2);
  return cudaGetLastError();
}

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
