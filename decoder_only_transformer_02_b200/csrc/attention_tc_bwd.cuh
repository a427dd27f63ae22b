// Causal attention backward on tcgen05 (bf16 operands, fp32 TMEM accumulators).
//
// With P = exp(S/sqrt(d) - lse) and D_q = sum_d dO_q . O_q:
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dK = dS^T Q / sqrt(d),
//   dQ = dS K / sqrt(d).
// Two deterministic kernels (no atomics), each with one CTA per SM and
// 128 x 128 score tiles:
//  dq_kernel (runs first): one CTA owns 128 queries of one (batch, head) and
//     walks the 128-key blocks up to its last query:
//       S = Q K_j^T, dP = dO V_j^T        (M=128 queries, N=128 keys, K=64)
//       dS = P * (dP - D)                  (eight compute warps, bf16 into TMEM)
//       dQ += dS K_j                       (A = dS read from TMEM, K=128 keys)
//     It also forms D for its queries (from the dO tile in shared memory and
//     the rows of O) and writes lse*log2(e) and D per 128-query block into a
//     padded fp32 array (+inf / 0 past T) that dkdv_kernel streams by bulk copy.
//  dkdv_kernel: one CTA owns 128 keys and walks the 128-query blocks that
//     reach them:
//       S^T = K Q_i^T, dP^T = V dO_i^T     (M=128 keys, N=128 queries, K=64)
//       P^T, dS^T                          (bf16 into TMEM)
//       dV += P^T dO_i, dK += dS^T Q_i     (A from TMEM, K=128 queries)
// The score tiles never touch shared memory: S and dP are read from TMEM into
// registers, and P / dS go back into TMEM as the A operand of the next MMAs.
// Warp 0 streams the operand tiles through a 4-stage TMA ring, warp 1 issues
// the MMAs (one thread), warps 2..9 do the element-wise math: warps w and w+4
// share TMEM lane quarter w%4 (one row each) and take the two 64-column halves
// of the tile.  While the warps work on tile j, the tensor cores already run
// S_{j+1} and dP_{j+1} (and the accumulating MMAs of tile j-1).  Every wait is
// bounded; the waits that drain a CTA's own copies and MMAs before it exits
// have their own fixed limit.
#pragma once
#include "attention.cuh"
#include "attention_tc.cuh"

namespace tcfa {

constexpr int BW_THREADS = 320;               // producer, MMA issuer, 8 compute warps
constexpr int BW_STAGES = 4;                  // operand ring depth
constexpr int BT = 128;                       // rows of a score tile (queries or keys)
constexpr int LD_FLOATS = 2 * BT;             // per 128-query block: lse*log2(e)[128], D[128]
constexpr uint32_t BW_TMEM_COLS = 512;

// Store 32 consecutive fp32 accumulator columns of one row as bf16 (x scale).
__device__ __forceinline__ void store_row32(bf16* dst, const uint32_t (&a)[32], float scale) {
#pragma unroll
  for (int e = 0; e < 32; e += 8)
    *reinterpret_cast<uint4*>(dst + e) = make_uint4(
        pack_bf16x2(__uint_as_float(a[e]) * scale, __uint_as_float(a[e + 1]) * scale),
        pack_bf16x2(__uint_as_float(a[e + 2]) * scale, __uint_as_float(a[e + 3]) * scale),
        pack_bf16x2(__uint_as_float(a[e + 4]) * scale, __uint_as_float(a[e + 5]) * scale),
        pack_bf16x2(__uint_as_float(a[e + 6]) * scale, __uint_as_float(a[e + 7]) * scale));
}

// ----------------------------------------------------------------- dQ
// Shared memory: Q 128x64, dO 128x64 (16 KB each, 128-byte swizzled K-major
// rows of 64 bf16), then the ring of K_j, V_j tiles (32 KB per stage).
constexpr int DQ_Q_OFF = 0;
constexpr int DQ_DO_OFF = TILE;
constexpr int DQ_RING_OFF = 2 * TILE;  // stage s: K at +2s*TILE, V at +(2s+1)*TILE
constexpr int DQ_BAR_OFF = DQ_RING_OFF + 2 * BW_STAGES * TILE;
constexpr int DQ_RED_OFF = DQ_BAR_OFF + 256;
constexpr int DQ_SMEM = DQ_RED_OFF + 2 * 4 * 32 * 4 + 1024;
// TMEM columns: S [0,128), dP [128,256), dQ [256,320), dS (bf16 pairs) [320,384)
constexpr uint32_t DQ_T_S = 0, DQ_T_DP = 128, DQ_T_DQ = 256, DQ_T_DS = 320;

__global__ void __launch_bounds__(BW_THREADS, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
              const bf16* __restrict__ out, const float* __restrict__ lse, float* __restrict__ ld_out,
              bf16* __restrict__ dqkv, float* __restrict__ colsum, int T, int H, float scale, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_BAR_OFF);
  uint64_t* q_full = bars;                   // Q and dO tiles landed
  uint64_t* kv_full = bars + 1;              // BW_STAGES
  uint64_t* kv_empty = kv_full + BW_STAGES;  // BW_STAGES
  uint64_t* s_full = kv_empty + BW_STAGES;   // S_j and dP_j in TMEM
  uint64_t* s_free = s_full + 1;             // count 8: S_j and dP_j are in registers
  uint64_t* ds_full = s_free + 1;            // count 8: dS_j in TMEM
  uint64_t* ds_free = ds_full + 1;           // dQ += dS_j K_j has read dS_j
  uint64_t* acc_done = ds_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);
  float* red = reinterpret_cast<float*>(smem + DQ_RED_OFF);  // [2 halves][4 quarters][32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = gridDim.x;
  const int qb = nqb - 1 - blockIdx.x;  // most key blocks first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD;
  const int row0 = b * T;
  const int qlast = min(qb * BT + BT - 1, T - 1);
  const int nblk = qlast / BT + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < BW_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(ds_full, 8);
    mbar_init(ds_free, 1);
    mbar_init(acc_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(BW_TMEM_COLS)
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
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_qkv)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_do)) : "memory");
      mbar_expect_tx(q_full, 2 * TILE);
      tma_load_2d(smem_u32(smem + DQ_Q_OFF), &tm_qkv, h * HD, row0 + qb * BT, q_full);
      tma_load_2d(smem_u32(smem + DQ_DO_OFF), &tm_do, h * HD, row0 + qb * BT, q_full);
      uint32_t issued = 0;
      for (int j = 0; j < nblk; ++j, ++issued) {
        const int s = j % BW_STAGES;
        if (!mbar_wait(&kv_empty[s], ((j / BW_STAGES) & 1u) ^ 1u)) {
          set_device_err(DERR_WAIT_TIMEOUT);
          break;
        }
        mbar_expect_tx(&kv_full[s], 2 * TILE);
        const uint32_t dst = smem_u32(smem + DQ_RING_OFF + 2 * s * TILE);
        tma_load_2d(dst, &tm_qkv, C + h * HD, row0 + j * BT, &kv_full[s]);
        tma_load_2d(dst + TILE, &tm_qkv, 2 * C + h * HD, row0 + j * BT, &kv_full[s]);
      }
      // drain: every issued load has landed before the CTA exits
      for (int s = 0; s < BW_STAGES; ++s) {
        if ((uint32_t)s < issued) {
          const uint32_t last = issued - 1 - ((issued - 1 - s) % BW_STAGES);
          if (!mbar_wait_drain(&kv_full[s], (last / BW_STAGES) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
      if (!mbar_wait_drain(q_full, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t id_s = att_idesc(BT, 0);   // S, dP: N = 128 keys, K = 64 (d)
      constexpr uint32_t id_dq = att_idesc(HD, 1);  // dQ: N = 64 (d), K = 128 keys, K_j MN-major
      bool ok = mbar_wait(q_full, 0);
      const uint32_t qa = smem_u32(smem + DQ_Q_OFF), doa = smem_u32(smem + DQ_DO_OFF);
      auto dq_step = [&](int i) -> bool {
        if (!mbar_wait(ds_full, i & 1u)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + DQ_RING_OFF + 2 * (i % BW_STAGES) * TILE);
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          tc_mma_ts(tmem + DQ_T_DQ, tmem + DQ_T_DS + kk * 8, make_sdesc(ka + kk * 2048, 1), id_dq,
                    (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&kv_empty[i % BW_STAGES]);
        tc_commit(ds_free);
        return true;
      };
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % BW_STAGES;
        if (!mbar_wait(&kv_full[s], (j / BW_STAGES) & 1u)) {
          ok = false;
          break;
        }
        if (j >= 1 && !mbar_wait(s_free, (j - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + DQ_RING_OFF + 2 * s * TILE);
        const uint32_t va = ka + TILE;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          tc_mma(tmem + DQ_T_S, make_sdesc(qa + kk * 32, 0), make_sdesc(ka + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
          tc_mma(tmem + DQ_T_DP, make_sdesc(doa + kk * 32, 0), make_sdesc(va + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
        if (j >= 1 && !dq_step(j - 1)) ok = false;
      }
      if (ok && !dq_step(nblk - 1)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(acc_done);
      if (!mbar_wait_drain(acc_done, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------- compute warps
    const int qw = warp & 3;             // TMEM lane quarter
    const int hf = (warp - 2) >> 2;      // which 64 keys of the 128-key tile
    const int r = qw * 32 + lane;        // query row within the block
    const int q = qb * BT + r;           // query position
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    const float l2 = q < T ? lse[(long)bh * T + q] * 1.4426950408889634f : INFINITY;
    bool ok = warp_wait(q_full, 0);
    // D_q = sum_d dO[q,d] O[q,d] (the row of O from global memory, dO from the
    // tile in shared memory)
    float dq_ = 0.f;
    if (ok && q < T) {
      const bf16* orow = out + ((long)row0 + q) * C + h * HD;
      const uint8_t* dorow = smem + DQ_DO_OFF;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < HD / 8; ++c) {
        const uint4 ov = *reinterpret_cast<const uint4*>(orow + 8 * c);
        const uint4 dv = *reinterpret_cast<const uint4*>(dorow + sw128(r, c));
        const uint32_t o4[4] = {ov.x, ov.y, ov.z, ov.w}, d4[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 of = unpack_bf16x2(o4[e]), df = unpack_bf16x2(d4[e]);
          acc[e] = fmaf(of.x, df.x, fmaf(of.y, df.y, acc[e]));
        }
      }
      dq_ = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    if (ok && hf == 0) {
      float* ldb = ld_out + ((long)bh * nqb + qb) * LD_FLOATS;
      ldb[r] = l2;
      ldb[BT + r] = dq_;
    }
    for (int j = 0; ok && j < nblk; ++j) {
      if (!warp_wait(s_full, j & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[64], dv[64];
      tmem_ld64(tl + DQ_T_S + hf * 64, sv);
      tmem_ld64(tl + DQ_T_DP + hf * 64, dv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      const int k0 = j * BT + hf * 64;      // first key of this warp's columns
      const bool diag = k0 + 63 > qb * BT;  // some key of the columns follows some query of the block
      // dS = P * (dP - D), packed to bf16 pairs in place
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float p0 = ex2f(fmaf(__uint_as_float(sv[c]), sl2, -l2));
        float p1 = ex2f(fmaf(__uint_as_float(sv[c + 1]), sl2, -l2));
        if (diag) {
          if (k0 + c > q) p0 = 0.f;
          if (k0 + c + 1 > q) p1 = 0.f;
        }
        sv[c >> 1] = pack_bf16x2(p0 * (__uint_as_float(dv[c]) - dq_), p1 * (__uint_as_float(dv[c + 1]) - dq_));
      }
      // dQ += dS_{j-1} K_{j-1} has read the dS buffer
      if (j >= 1 && !warp_wait(ds_free, (j - 1) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st32(tl + DQ_T_DS + hf * 32, sv);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    float cs[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) cs[i] = 0.f;
    if (ok && warp_wait(acc_done, 0)) {
      tc_fence_after();
      uint32_t a[32];
      tmem_ld32(tl + DQ_T_DQ + hf * 32, a);
      tmem_wait_ld();
      if (q < T) {
        store_row32(dqkv + ((long)row0 + q) * (3L * C) + h * HD + hf * 32, a, scale);
#pragma unroll
        for (int i = 0; i < 32; ++i) cs[i] = __uint_as_float(a[i]) * scale;
      }
    } else {
      ok = false;
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
    if (colsum) red[(hf * 4 + qw) * 32 + lane] = warp_colsum32(cs, lane);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BW_TMEM_COLS) : "memory");
  }
  // column sums of dQ over the block's rows (the query bias gradient), as
  // one partial row per 128-row block, quarters added in a fixed order
  if (colsum && warp >= 2 && warp < 4) {
    const int hf = warp - 2;
    const float t = ((red[(hf * 4) * 32 + lane] + red[(hf * 4 + 1) * 32 + lane]) + red[(hf * 4 + 2) * 32 + lane]) +
                    red[(hf * 4 + 3) * 32 + lane];
    colsum[((long)b * nqb + qb) * (3L * C) + h * HD + hf * 32 + lane] = t;
  }
}

// ------------------------------------------------------------ dK, dV
// Shared memory: K, V 128x64 (16 KB each), then the ring of Q_i, dO_i tiles and
// the block's lse*log2(e) / D rows (33 KB per stage).
constexpr int DKV_K_OFF = 0;
constexpr int DKV_V_OFF = TILE;
constexpr int DKV_STAGE_BYTES = 2 * TILE + LD_FLOATS * 4;
constexpr int DKV_RING_OFF = 2 * TILE;  // stage s: Q, dO, lse2/D
constexpr int DKV_BAR_OFF = DKV_RING_OFF + BW_STAGES * DKV_STAGE_BYTES;
constexpr int DKV_RED_OFF = DKV_BAR_OFF + 256;
constexpr int DKV_SMEM = DKV_RED_OFF + 2 * 2 * 4 * 32 * 4 + 1024;
// TMEM columns: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384),
// P^T (bf16 pairs) [384,448), dS^T (bf16 pairs) [448,512)
constexpr uint32_t DKV_T_S = 0, DKV_T_DP = 128, DKV_T_DV = 256, DKV_T_DK = 320, DKV_T_P = 384, DKV_T_DS = 448;
static_assert(DKV_STAGE_BYTES % 1024 == 0, "ring stages keep the 1024-byte swizzle alignment");

__global__ void __launch_bounds__(BW_THREADS, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                const float* __restrict__ ld_in, bf16* __restrict__ dqkv, float* __restrict__ colsum, int T, int H,
                float scale, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DKV_BAR_OFF);
  uint64_t* kv_full = bars;                  // K and V tiles
  uint64_t* qd_full = bars + 1;              // BW_STAGES
  uint64_t* qd_empty = qd_full + BW_STAGES;  // BW_STAGES
  uint64_t* s_full = qd_empty + BW_STAGES;   // S^T and dP^T in TMEM
  uint64_t* s_free = s_full + 1;             // count 8
  uint64_t* p_full = s_free + 1;             // count 8: P^T and dS^T in TMEM
  uint64_t* p_free = p_full + 1;             // the dV / dK MMAs have read them
  uint64_t* acc_done = p_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);
  float* red = reinterpret_cast<float*>(smem + DKV_RED_OFF);  // [dK, dV][2 halves][4 quarters][32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = gridDim.x;
  const int kb = blockIdx.x;  // key block; small kb = most query blocks, launched first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD;
  const int row0 = b * T;
  const int nblk = nqb - kb;  // query blocks kb .. nqb-1

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < BW_STAGES; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(p_full, 8);
    mbar_init(p_free, 1);
    mbar_init(acc_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(BW_TMEM_COLS)
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
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_qkv)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_do)) : "memory");
      mbar_expect_tx(kv_full, 2 * TILE);
      tma_load_2d(smem_u32(smem + DKV_K_OFF), &tm_qkv, C + h * HD, row0 + kb * BT, kv_full);
      tma_load_2d(smem_u32(smem + DKV_V_OFF), &tm_qkv, 2 * C + h * HD, row0 + kb * BT, kv_full);
      uint32_t issued = 0;
      for (int n = 0; n < nblk; ++n, ++issued) {
        const int i = kb + n, s = n % BW_STAGES;
        if (!mbar_wait(&qd_empty[s], ((n / BW_STAGES) & 1u) ^ 1u)) {
          set_device_err(DERR_WAIT_TIMEOUT);
          break;
        }
        mbar_expect_tx(&qd_full[s], DKV_STAGE_BYTES);
        const uint32_t dst = smem_u32(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES);
        tma_load_2d(dst, &tm_qkv, h * HD, row0 + i * BT, &qd_full[s]);
        tma_load_2d(dst + TILE, &tm_do, h * HD, row0 + i * BT, &qd_full[s]);
        bulk_load(dst + 2 * TILE, ld_in + ((long)bh * nqb + i) * LD_FLOATS, LD_FLOATS * 4, &qd_full[s]);
      }
      // drain: every issued load has landed before the CTA exits
      for (int s = 0; s < BW_STAGES; ++s) {
        if ((uint32_t)s < issued) {
          const uint32_t last = issued - 1 - ((issued - 1 - s) % BW_STAGES);
          if (!mbar_wait_drain(&qd_full[s], (last / BW_STAGES) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
      if (!mbar_wait_drain(kv_full, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t id_s = att_idesc(BT, 0);    // S^T, dP^T: N = 128 queries, K = 64 (d)
      constexpr uint32_t id_acc = att_idesc(HD, 1);  // dV, dK: N = 64 (d), K = 128 queries, B MN-major
      bool ok = mbar_wait(kv_full, 0);
      const uint32_t ka = smem_u32(smem + DKV_K_OFF), va = smem_u32(smem + DKV_V_OFF);
      auto acc_step = [&](int n) -> bool {
        if (!mbar_wait(p_full, n & 1u)) return false;
        tc_fence_after();
        const int s = n % BW_STAGES;
        const uint32_t qa = smem_u32(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES);
        const uint32_t doa = qa + TILE;
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
          tc_mma_ts(tmem + DKV_T_DV, tmem + DKV_T_P + kk * 8, make_sdesc(doa + kk * 2048, 1), id_acc, acc);
          tc_mma_ts(tmem + DKV_T_DK, tmem + DKV_T_DS + kk * 8, make_sdesc(qa + kk * 2048, 1), id_acc, acc);
        }
        tc_commit(&qd_empty[s]);
        tc_commit(p_free);
        return true;
      };
      for (int n = 0; ok && n < nblk; ++n) {
        const int s = n % BW_STAGES;
        if (!mbar_wait(&qd_full[s], (n / BW_STAGES) & 1u)) {
          ok = false;
          break;
        }
        if (n >= 1 && !mbar_wait(s_free, (n - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t qa = smem_u32(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES);
        const uint32_t doa = qa + TILE;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          tc_mma(tmem + DKV_T_S, make_sdesc(ka + kk * 32, 0), make_sdesc(qa + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
          tc_mma(tmem + DKV_T_DP, make_sdesc(va + kk * 32, 0), make_sdesc(doa + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
        if (n >= 1 && !acc_step(n - 1)) ok = false;
      }
      if (ok && nblk > 0 && !acc_step(nblk - 1)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(acc_done);
      if (!mbar_wait_drain(acc_done, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------- compute warps
    const int qw = warp & 3;
    const int hf = (warp - 2) >> 2;  // which 64 queries of the 128-query tile
    const int kr = qw * 32 + lane;   // key row within the block
    const int key = kb * BT + kr;    // key position
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    bool ok = true;
    for (int n = 0; n < nblk; ++n) {
      const int i = kb + n, s = n % BW_STAGES;
      if (!warp_wait(s_full, n & 1u) || !warp_wait(&qd_full[s], (n / BW_STAGES) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[64], dv[64];
      tmem_ld64(tl + DKV_T_S + hf * 64, sv);
      tmem_ld64(tl + DKV_T_DP + hf * 64, dv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      const int q0 = i * BT + hf * 64;                // first query of this warp's columns
      const bool diag = q0 < kb * BT + BT - 1;        // some query of the columns precedes some key
      const float* ldl =
          reinterpret_cast<const float*>(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES + 2 * TILE) + hf * 64;
      // P^T and dS^T of this block, packed to bf16 pairs in place
#pragma unroll
      for (int c = 0; c < 64; c += 8) {
        const float4 la = *reinterpret_cast<const float4*>(ldl + c);
        const float4 lb = *reinterpret_cast<const float4*>(ldl + c + 4);
        const float4 da = *reinterpret_cast<const float4*>(ldl + BT + c);
        const float4 db = *reinterpret_cast<const float4*>(ldl + BT + c + 4);
        const float l8[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
        const float d8[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
        float p[8], ds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float pe = ex2f(fmaf(__uint_as_float(sv[c + e]), sl2, -l8[e]));
          if (diag && (q0 + c + e < key)) pe = 0.f;
          p[e] = pe;
          ds[e] = pe * (__uint_as_float(dv[c + e]) - d8[e]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sv[(c >> 1) + e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
          dv[(c >> 1) + e] = pack_bf16x2(ds[2 * e], ds[2 * e + 1]);
        }
      }
      // the previous block's dV / dK MMAs have read P^T and dS^T
      if (n >= 1 && !warp_wait(p_free, (n - 1) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st32(tl + DKV_T_P + hf * 32, sv);
      tmem_st32(tl + DKV_T_DS + hf * 32, dv);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    float cv[32], ck[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) cv[i] = ck[i] = 0.f;
    if (ok && warp_wait(acc_done, 0)) {
      tc_fence_after();
      uint32_t a[32];
      tmem_ld32(tl + DKV_T_DV + hf * 32, a);
      tmem_wait_ld();
      if (key < T) {
        store_row32(dqkv + ((long)row0 + key) * (3L * C) + 2 * C + h * HD + hf * 32, a, 1.f);
#pragma unroll
        for (int i = 0; i < 32; ++i) cv[i] = __uint_as_float(a[i]);
      }
      tmem_ld32(tl + DKV_T_DK + hf * 32, a);
      tmem_wait_ld();
      if (key < T) {
        store_row32(dqkv + ((long)row0 + key) * (3L * C) + C + h * HD + hf * 32, a, scale);
#pragma unroll
        for (int i = 0; i < 32; ++i) ck[i] = __uint_as_float(a[i]) * scale;
      }
    } else {
      ok = false;
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
    if (colsum) {
      red[(hf * 4 + qw) * 32 + lane] = warp_colsum32(ck, lane);
      red[256 + (hf * 4 + qw) * 32 + lane] = warp_colsum32(cv, lane);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BW_TMEM_COLS) : "memory");
  }
  // column sums of dK and dV over the block's rows (the key and value bias
  // gradients), one partial row per 128-row block, quarters in a fixed order
  if (colsum && warp >= 2 && warp < 6) {
    const int kv = (warp - 2) >> 1, hf = (warp - 2) & 1;  // kv 0: dK, 1: dV
    const float* rr = red + kv * 256 + hf * 128;
    const float t = ((rr[lane] + rr[32 + lane]) + rr[64 + lane]) + rr[96 + lane];
    colsum[((long)b * nqb + kb) * (3L * C) + (1 + kv) * C + h * HD + hf * 32 + lane] = t;
  }
}

// fp32 scratch of the backward: lse*log2(e) and D per query, padded to whole
// 128-query blocks
static inline long backward_scratch_floats(int B, int T, int H) {
  return (long)B * H * ((T + BT - 1) / BT) * LD_FLOATS;
}

// dq_kernel first (it also writes lse*log2(e) and D into `ld`), then
// dkdv_kernel.  ld: fp32 scratch of backward_scratch_floats(B, T, H) elements,
// 16-byte aligned.  colsum (may be null): [B * ceil(T/128)][3C] fp32 partial
// column sums of dqkv, one row per 128-row block of each batch (summing them
// over the rows gives the qkv bias gradient).
static inline cudaError_t backward(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, bf16* dqkv,
                                   float* ld, int B, int T, int H, cudaStream_t st, float* colsum = nullptr) {
  static DeviceOnce once;
  cudaError_t e = run_once_per_device(once, [] {
    cudaError_t r = cudaFuncSetAttribute(dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKV_SMEM);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM);
    return r;
  });
  if (e != cudaSuccess) return e;
  if (reinterpret_cast<uintptr_t>(ld) & 15) return cudaErrorInvalidValue;
  const int C = H * HD;
  CUtensorMap tq, td;
  if (make_tmap(&tq, qkv, 3L * C, (long)B * T, 3L * C, 64, BT) != 0) return cudaErrorInvalidValue;
  if (make_tmap(&td, dout, C, (long)B * T, C, 64, BT) != 0) return cudaErrorInvalidValue;
  const float scale = 1.f / sqrtf((float)HD);
  const float sl2 = 1.4426950408889634f * scale;
  dim3 grid((T + BT - 1) / BT, B * H);
  dq_kernel<<<grid, BW_THREADS, DQ_SMEM, st>>>(tq, td, out, lse, ld, dqkv, colsum, T, H, scale, sl2);
  dkdv_kernel<<<grid, BW_THREADS, DKV_SMEM, st>>>(tq, td, ld, dqkv, colsum, T, H, scale, sl2);
  return cudaGetLastError();
}

}  // namespace tcfa
