// Causal attention on the 5th-generation tensor cores (tcgen05): the forward
// kernel and the constants and helpers the backward kernels share.
//
// bf16 qkv [B, T, 3C] (q, k, v column blocks, head h in columns h*64..),
// head dim 64; output o [B, T, C] bf16 and lse [B, H, T] fp32.  One CTA owns
// 128 queries of one (batch, head) and walks the key blocks of 64 keys up to
// its last query:
//   S_j  = Q K_j^T        tcgen05.mma, M=128 x N=64 x K=64, fp32 in TMEM
//   P_j  = exp(S_j/sqrt(d) - m_j)  (online softmax, one thread per query row,
//          read from TMEM; bf16 P written to shared memory in the 128-byte
//          swizzled K-major layout the MMA reads)
//   PV_j = P_j V_j        tcgen05.mma, M=128 x N=64 x K=64, fp32 in TMEM
//   O    = alpha_j (O + PV_{j-1}) in registers, O/l at the end.  The
//          reference maximum m_j is updated lazily (only when a block raises
//          some row's maximum by more than 2^8), so most blocks need no
//          rescale: then alpha_j = 1 and O + PV_{j-1} is all that is done.
// Warp 0 loads Q once and K_j, V_j through a 3-stage TMA ring; warp 1 issues
// the MMAs (S_{j+1} is computed while the softmax warps work on S_j); warps
// 2..5 do the softmax (warp w reads TMEM lanes 32*(w%4)..+31).  S and PV are
// double-buffered in TMEM.  All waits are bounded.
#pragma once
#include "common.cuh"

namespace tcfa {

using namespace tcg;

constexpr int BQ = 128;       // queries per CTA
constexpr int BKV = 128;      // keys per block
constexpr int HD = 64;        // head dim
constexpr int KV_STAGES = 3;
constexpr int TILE = 128 * 64 * 2;          // one 128 x 64 bf16 tile (16 KB)
constexpr int Q_OFF = 0;
constexpr int KV_OFF = TILE;                // stage s: K at +2s*TILE, V at +(2s+1)*TILE
constexpr int P_OFF = KV_OFF + 2 * KV_STAGES * TILE;  // two P buffers of 2 tiles each
constexpr int BAR_OFF = P_OFF + 4 * TILE;
constexpr int SMEM_BYTES = BAR_OFF + 512 + 1024;
constexpr uint32_t TMEM_COLS = 512;         // S0 0, S1 128, PV0 256, PV1 320

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte offset of element (r, c) in a 128-row, 64-column bf16 K-major tile with
// the 128-byte swizzle (16-byte chunk c/8 of row r stored at chunk (c/8)^(r%8))
__device__ __forceinline__ uint32_t sw128(int r, int chunk) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4));
}

// ---------------------------------------------------------------- forward
// The forward walks 64-key blocks so that one CTA needs 256 TMEM columns and
// about 97 KB of shared memory: two CTAs share an SM, and every SM
// sub-partition runs two softmax warps, one CTA's softmax overlapping the
// other's MMAs.
constexpr int FBKV = 64;                        // keys per block (forward)
constexpr int F_STAGES = 3;
constexpr int HTILE = 64 * 64 * 2;              // one 64 x 64 bf16 tile (8 KB)
constexpr int FQ_OFF = 0;                       // Q: 128 x 64, loaded as two 64-row boxes
constexpr int FKV_OFF = TILE;                   // stage s: K at +2s*HTILE, V at +(2s+1)*HTILE
constexpr int FP_OFF = FKV_OFF + 2 * F_STAGES * HTILE;  // two P buffers of 128 x 64 bf16
constexpr int FBAR_OFF = FP_OFF + 2 * TILE;
constexpr int F_SMEM = FBAR_OFF + 256 + 1024;
constexpr uint32_t F_TMEM_COLS = 256;           // S0 0, S1 64, PV0 128, PV1 192
constexpr float RESCALE_LOG2 = 8.f;             // lazy-rescale threshold (log2 units)

__global__ void __launch_bounds__(192, 2)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse, int T,
               int H, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FBAR_OFF);
  uint64_t* q_full = bars;                 // 1
  uint64_t* kv_full = bars + 1;            // F_STAGES
  uint64_t* kv_empty = kv_full + F_STAGES;
  uint64_t* s_full = kv_empty + F_STAGES;  // 2
  uint64_t* s_free = s_full + 2;           // 2 (count 4)
  uint64_t* p_full = s_free + 2;           // 2 (count 4)
  uint64_t* pv_full = p_full + 2;          // 2
  uint64_t* pv_free = pv_full + 2;         // 2 (count 4)
  uint64_t* drain = pv_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest blocks first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD;
  const int qlast = min(qb * BQ + BQ - 1, T - 1);  // last query position of the block
  const int nkv = qlast / FBKV + 1;
  const int row0 = b * T;  // first row of this batch in the [B*T, 3C] view

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < F_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_full[i], 1);
      mbar_init(&pv_free[i], 4);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(F_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------- producer
      mbar_expect_tx(q_full, TILE);
      tma_load_2d(smem_u32(smem + FQ_OFF), &tm_qkv, h * HD, row0 + qb * BQ, q_full);
      tma_load_2d(smem_u32(smem + FQ_OFF + HTILE), &tm_qkv, h * HD, row0 + qb * BQ + 64, q_full);
      uint32_t issued = 0;
      for (int j = 0; j < nkv; ++j, ++issued) {
        const int s = j % F_STAGES;
        if (!mbar_wait(&kv_empty[s], ((j / F_STAGES) & 1u) ^ 1u)) {
          set_device_err(DERR_WAIT_TIMEOUT);
          break;
        }
        mbar_expect_tx(&kv_full[s], 2 * HTILE);
        const uint32_t kd = smem_u32(smem + FKV_OFF + 2 * s * HTILE);
        tma_load_2d(kd, &tm_qkv, C + h * HD, row0 + j * FBKV, &kv_full[s]);
        tma_load_2d(kd + HTILE, &tm_qkv, 2 * C + h * HD, row0 + j * FBKV, &kv_full[s]);
      }
      // drain: every issued K/V load has been consumed by its PV MMA
      for (int s = 0; s < F_STAGES; ++s) {
        if ((uint32_t)s < issued) {
          const uint32_t last = issued - 1 - ((issued - 1 - s) % F_STAGES);
          if (!mbar_wait(&kv_empty[s], (last / F_STAGES) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
      if (!mbar_wait(q_full, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      // S: A = Q (K-major), B = K_j (K-major), M=128, N=64
      const uint32_t id_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(FBKV >> 3) << 17) |
                            ((uint32_t)(BQ >> 4) << 24);
      // PV: A = P_j (K-major over keys), B = V_j (MN-major: d contiguous), M=128, N=64
      const uint32_t id_pv = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(HD >> 3) << 17) |
                             ((uint32_t)(BQ >> 4) << 24);
      bool ok = mbar_wait(q_full, 0);
      tc_fence_after();
      const uint32_t qa = smem_u32(smem + FQ_OFF);
      auto do_pv = [&](int i) -> bool {
        const int pb = i & 1;
        if (!mbar_wait(&p_full[pb], (i >> 1) & 1u)) return false;
        if (i >= 2 && !mbar_wait(&pv_free[pb], ((i - 2) >> 1) & 1u)) return false;
        tc_fence_after();
        const int s = i % F_STAGES;
        const uint32_t pa = smem_u32(smem + FP_OFF + pb * TILE);
        const uint32_t va = smem_u32(smem + FKV_OFF + (2 * s + 1) * HTILE);
        const uint32_t d = tmem + 128 + pb * HD;
#pragma unroll
        for (int kk = 0; kk < FBKV / 16; ++kk) {
          const uint64_t ad = make_sdesc(pa + kk * 32, 0);
          const uint64_t bd = make_sdesc(va + kk * 2048, 1);
          tc_mma(d, ad, bd, id_pv, kk > 0 ? 1u : 0u);
        }
        tc_commit(&pv_full[pb]);
        tc_commit(&kv_empty[s]);
        return true;
      };
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % F_STAGES, sb = j & 1;
        if (!mbar_wait(&kv_full[s], (j / F_STAGES) & 1u)) {
          ok = false;
          break;
        }
        if (j >= 2 && !mbar_wait(&s_free[sb], ((j - 2) >> 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + FKV_OFF + 2 * s * HTILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t ad = make_sdesc(qa + kk * 32, 0);
          const uint64_t bd = make_sdesc(ka + kk * 32, 0);
          tc_mma(tmem + sb * FBKV, ad, bd, id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        if (j >= 1 && !do_pv(j - 1)) ok = false;
      }
      if (ok && !do_pv(nkv - 1)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(drain);
      if (!mbar_wait(drain, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------- softmax warps
    const int qw = warp & 3;                // TMEM lane quarter
    const int r = qw * 32 + lane;           // query row within the block
    const int q = qb * BQ + r;              // query position in the sequence
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    float o[HD];
#pragma unroll
    for (int i = 0; i < HD; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the 64-key row of S in registers (one TMEM wait), buffer released
      uint32_t v[FBKV];
      tmem_ld32(tl + sb * FBKV, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld32(tl + sb * FBKV + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      // causal mask on the blocks that reach past the block's first query
      if (j * FBKV + FBKV - 1 > qb * BQ) {
#pragma unroll
        for (int e = 0; e < FBKV; ++e)
          if (j * FBKV + e > q) v[e] = __float_as_uint(-INFINITY);
      }
      // row maximum of the raw scores in 8 chains; the positive scale
      // 1/sqrt(d)*log2(e) is applied to the maximum
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(v[i]);
#pragma unroll
      for (int e = 8; e < FBKV; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // lazy rescaling: the reference maximum m moves only when some row of
      // the warp sees a block maximum more than 2^RESCALE_LOG2 above it (and
      // always for the first block).  O, l and P share the reference, so the
      // result is exact for any choice of it; P stays <= 2^RESCALE_LOG2.
      const bool rescale = __any_sync(0xffffffffu, mx * sl2 > m + RESCALE_LOG2);
      float m_new = m, alpha = 1.f;
      if (rescale) {
        m_new = fmaxf(m, mx * sl2);
        alpha = ex2f(m - m_new);
      }
      // p = 2^(s*sl2 - m_new) (one FFMA + ex2), row sum in 8 chains, bf16 P
      // into shared memory in the swizzled K-major layout
      float rs8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) rs8[i] = 0.f;
      uint8_t* pbuf = smem + FP_OFF + sb * TILE;
#pragma unroll
      for (int k = 0; k < FBKV / 8; ++k) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = ex2f(fmaf(__uint_as_float(v[8 * k + e]), sl2, -m_new));
          rs8[e] += pv[e];
        }
        const uint4 w = make_uint4(pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]), pack_bf16x2(pv[4], pv[5]),
                                   pack_bf16x2(pv[6], pv[7]));
        *reinterpret_cast<uint4*>(pbuf + sw128(r, k)) = w;
      }
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
      l = l * alpha + rs;
      m = m_new;
      if (j >= 1) {
        const int pb = (j - 1) & 1;
        if (!mbar_wait(&pv_full[pb], ((j - 1) >> 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t a0[32], a1[32];
        tmem_ld32(tl + 128 + pb * HD, a0);
        tmem_ld32(tl + 128 + pb * HD + 32, a1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pv_free[pb]);
        if (!rescale) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            o[i] += __uint_as_float(a0[i]);
            o[32 + i] += __uint_as_float(a1[i]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            o[i] = (o[i] + __uint_as_float(a0[i])) * alpha;
            o[32 + i] = (o[32 + i] + __uint_as_float(a1[i])) * alpha;
          }
        }
      }
    }
    if (ok) {
      const int pb = (nkv - 1) & 1;
      if (mbar_wait(&pv_full[pb], ((nkv - 1) >> 1) & 1u)) {
        tc_fence_after();
        uint32_t a0[32], a1[32];
        tmem_ld32(tl + 128 + pb * HD, a0);
        tmem_ld32(tl + 128 + pb * HD + 32, a1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          o[i] += __uint_as_float(a0[i]);
          o[32 + i] += __uint_as_float(a1[i]);
        }
        if (q < T) {
          const float inv = 1.f / l;
          bf16* orow = out + ((long)b * T + q) * C + h * HD;
#pragma unroll
          for (int i = 0; i < HD; i += 8)
            *reinterpret_cast<uint4*>(orow + i) =
                make_uint4(pack_bf16x2(o[i] * inv, o[i + 1] * inv), pack_bf16x2(o[i + 2] * inv, o[i + 3] * inv),
                           pack_bf16x2(o[i + 4] * inv, o[i + 5] * inv), pack_bf16x2(o[i + 6] * inv, o[i + 7] * inv));
          lse[((long)b * H + h) * T + q] = (m + __log2f(l)) * 0.6931471805599453f;
        }
      } else {
        ok = false;
      }
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(F_TMEM_COLS) : "memory");
  }
}

static inline cudaError_t forward(const bf16* qkv, bf16* out, float* lse, int B, int T, int H, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, F_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap tm;
  const int C = H * HD;
  if (make_tmap(&tm, qkv, 3L * C, (long)B * T, 3L * C, 64, 64) != 0) return cudaErrorInvalidValue;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
  dim3 grid((T + BQ - 1) / BQ, B * H);
  fwd_kernel<<<grid, 192, F_SMEM, st>>>(tm, out, lse, T, H, sl2);
  return cudaGetLastError();
}

}  // namespace tcfa
