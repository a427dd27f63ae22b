// Causal attention backward on tcgen05 (bf16 operands, fp32 TMEM accumulators).
//
// With P = exp(S/sqrt(d) - lse), D_q = sum_d dO_q . O_q (computed by dq_kernel):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dK = dS^T Q / sqrt(d),
//   dQ = dS K / sqrt(d).
// Two deterministic kernels (no atomics), in the structure of the forward:
//  dkdv_kernel: one CTA owns 128 keys and walks the query blocks i >= kb:
//     S^T = K Q_i^T and dP^T = V dO_i^T (M=128 keys, N=128 queries, K=64) into
//     TMEM; four compute warps (one key row per thread) form bf16 P^T and dS^T
//     in shared memory (128-byte swizzled, K-major over queries); then
//     dV += P^T dO_i and dK += dS^T Q_i (M=128, N=64, K=128) accumulate in TMEM.
//  dq_kernel: one CTA owns 128 queries and walks the 64-key blocks up to its
//     last query: S = Q K_j^T, dP = dO V_j^T, dS = P * (dP - D) (one query row
//     per thread), dQ += dS K_j; two CTAs per SM.
// Q_i / dO_i (resp. K_j / V_j) stream through a 2-stage TMA ring; the same
// swizzled tile serves as a K-major operand (contraction over d) and as an
// MN-major one (contraction over its rows).
#pragma once
#include "attention.cuh"
#include "attention_tc.cuh"

namespace tcfa {

constexpr int B_STAGES = 2;

// ------------------------------------------------------------ dK, dV
// One CTA owns 128 keys and walks the 64-query blocks from the first that
// reaches them.  256 TMEM columns and ~98 KB of shared memory, so two CTAs
// share an SM.  S^T and dP^T are released as soon as the compute warps hold
// them in registers, so S^T_{n+1} and dP^T_{n+1} run on the tensor cores while
// the warps form P^T_n and dS^T_n; the warps store those only after
// dV += P^T_{n-1} dO and dK += dS^T_{n-1} Q have read the previous ones.
constexpr int DKV_K_OFF = 0;                                      // K 128 x 64 (two 64-row boxes)
constexpr int DKV_V_OFF = TILE;                                   // V 128 x 64
constexpr int DKV_RING_OFF = 2 * TILE;                            // stage s: Q at +2s*HTILE, dO at +(2s+1)*HTILE
constexpr int DKV_P_OFF = DKV_RING_OFF + 2 * B_STAGES * HTILE;    // P^T 128 keys x 64 queries
constexpr int DKV_DS_OFF = DKV_P_OFF + TILE;                      // dS^T 128 x 64
constexpr int DKV_LD_OFF = DKV_DS_OFF + TILE;                     // stage s: lse*log2(e)[64], D[64]
constexpr int DKV_BAR_OFF = DKV_LD_OFF + B_STAGES * 512;
constexpr int DKV_SMEM = DKV_BAR_OFF + 256 + 1024;
constexpr uint32_t DKV_TMEM_COLS = 256;                           // S^T 0, dP^T 64, dV 128, dK 192

__global__ void __launch_bounds__(192, 2)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_qkv64, const __grid_constant__ CUtensorMap tm_do64,
                const float* __restrict__ lse, const float* __restrict__ Dv, bf16* __restrict__ dqkv, int T, int H,
                float scale, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DKV_BAR_OFF);
  uint64_t* kv_full = bars;                // K and V tiles
  uint64_t* qd_full = bars + 1;            // B_STAGES
  uint64_t* qd_empty = qd_full + B_STAGES;
  uint64_t* s_full = qd_empty + B_STAGES;  // S^T and dP^T ready
  uint64_t* s_free = s_full + 1;           // count 4
  uint64_t* p_full = s_free + 1;           // count 4
  uint64_t* pt_free = p_full + 1;          // P^T / dS^T consumed
  uint64_t* acc_done = pt_free + 1;
  uint64_t* ld_full = acc_done + 1;        // B_STAGES: lse / D of the stage's queries
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ld_full + B_STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x;  // key block; small kb = most query blocks, launched first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD;
  const int nq64 = (T + FBKV - 1) / FBKV;  // 64-query blocks in the sequence
  const int i0 = 2 * kb;                   // first query block that reaches key kb*128
  const int row0 = b * T;
  const int nblk = nq64 - i0;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < B_STAGES; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
      mbar_init(&ld_full[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(pt_free, 1);
    mbar_init(acc_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(DKV_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    // lane 0 drives the TMA ring; the whole warp stages each query block's
    // lse (log2 units; +inf past T) and D (0 past T) next to its Q / dO tiles
    if (lane == 0) {
      mbar_expect_tx(kv_full, 2 * TILE);
      const uint32_t kd = smem_u32(smem + DKV_K_OFF), vd = smem_u32(smem + DKV_V_OFF);
      tma_load_2d(kd, &tm_qkv64, C + h * HD, row0 + kb * BKV, kv_full);
      tma_load_2d(kd + HTILE, &tm_qkv64, C + h * HD, row0 + kb * BKV + 64, kv_full);
      tma_load_2d(vd, &tm_qkv64, 2 * C + h * HD, row0 + kb * BKV, kv_full);
      tma_load_2d(vd + HTILE, &tm_qkv64, 2 * C + h * HD, row0 + kb * BKV + 64, kv_full);
    }
    const float* lrow = lse + ((long)b * H + h) * T;
    const float* drow = Dv + ((long)b * H + h) * T;
    uint32_t issued = 0;
    for (int n = 0; n < nblk; ++n, ++issued) {
      const int i = i0 + n, s = n % B_STAGES;
      int got = 1;
      if (lane == 0) got = mbar_wait(&qd_empty[s], ((n / B_STAGES) & 1u) ^ 1u) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        if (lane == 0) set_device_err(DERR_WAIT_TIMEOUT);
        break;
      }
      float* ld = reinterpret_cast<float*>(smem + DKV_LD_OFF + s * 512);
      for (int c = lane; c < FBKV; c += 32) {
        const int q = i * FBKV + c;
        ld[c] = q < T ? lrow[q] * 1.4426950408889634f : INFINITY;
        ld[FBKV + c] = q < T ? drow[q] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ld_full[s]);
        mbar_expect_tx(&qd_full[s], 2 * HTILE);
        const uint32_t dst = smem_u32(smem + DKV_RING_OFF + 2 * s * HTILE);
        tma_load_2d(dst, &tm_qkv64, h * HD, row0 + i * FBKV, &qd_full[s]);
        tma_load_2d(dst + HTILE, &tm_do64, h * HD, row0 + i * FBKV, &qd_full[s]);
      }
    }
    if (lane == 0) {
      for (int s = 0; s < B_STAGES; ++s) {
        if ((uint32_t)s < issued) {
          const uint32_t last = issued - 1 - ((issued - 1 - s) % B_STAGES);
          if (!mbar_wait(&qd_empty[s], (last / B_STAGES) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
      if (!mbar_wait(kv_full, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      // S^T, dP^T: M=128 keys, N=64 queries, K=64 (d), both operands K-major
      const uint32_t id_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(FBKV >> 3) << 17) |
                            ((uint32_t)(BKV >> 4) << 24);
      // dV, dK: M=128 keys, N=64 (d), K=64 queries; dO / Q read MN-major
      const uint32_t id_acc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(HD >> 3) << 17) |
                              ((uint32_t)(BKV >> 4) << 24);
      bool ok = mbar_wait(kv_full, 0);
      const uint32_t ka = smem_u32(smem + DKV_K_OFF), va = smem_u32(smem + DKV_V_OFF);
      const uint32_t pa = smem_u32(smem + DKV_P_OFF), dsa = smem_u32(smem + DKV_DS_OFF);
      auto acc_step = [&](int n) -> bool {
        if (!mbar_wait(p_full, n & 1u)) return false;
        tc_fence_after();
        const int s = n % B_STAGES;
        const uint32_t qa = smem_u32(smem + DKV_RING_OFF + 2 * s * HTILE);
        const uint32_t doa = qa + HTILE;
#pragma unroll
        for (int kk = 0; kk < FBKV / 16; ++kk) {
          const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
          tc_mma(tmem + 128, make_sdesc(pa + kk * 32, 0), make_sdesc(doa + kk * 2048, 1), id_acc, acc);
          tc_mma(tmem + 192, make_sdesc(dsa + kk * 32, 0), make_sdesc(qa + kk * 2048, 1), id_acc, acc);
        }
        tc_commit(&qd_empty[s]);
        tc_commit(pt_free);
        return true;
      };
      for (int n = 0; ok && n < nblk; ++n) {
        const int s = n % B_STAGES;
        if (!mbar_wait(&qd_full[s], (n / B_STAGES) & 1u)) {
          ok = false;
          break;
        }
        if (n >= 1 && !mbar_wait(s_free, (n - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t qa = smem_u32(smem + DKV_RING_OFF + 2 * s * HTILE);
        const uint32_t doa = qa + HTILE;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          tc_mma(tmem, make_sdesc(ka + kk * 32, 0), make_sdesc(qa + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
          tc_mma(tmem + 64, make_sdesc(va + kk * 32, 0), make_sdesc(doa + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
        if (n >= 1 && !acc_step(n - 1)) ok = false;
      }
      if (ok && nblk > 0 && !acc_step(nblk - 1)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(acc_done);
      if (!mbar_wait(acc_done, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------- compute warps
    const int qw = warp & 3;
    const int kr = qw * 32 + lane;            // key row within the block
    const int key = kb * BKV + kr;            // key position
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    bool ok = true;
    for (int n = 0; n < nblk; ++n) {
      const int i = i0 + n, s = n % B_STAGES;
      if (!mbar_wait(&ld_full[s], (n / B_STAGES) & 1u) || !mbar_wait(s_full, n & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[64], dv[64];
      tmem_ld32(tl, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tl + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(tl + 64, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
      tmem_ld32(tl + 96, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      const bool diag = i * FBKV < kb * BKV + BKV - 1;  // some query of the block precedes some key
      const float* ldl = reinterpret_cast<const float*>(smem + DKV_LD_OFF + s * 512);
      // P^T and dS^T of this block, packed to bf16 pairs in place
#pragma unroll
      for (int k = 0; k < FBKV / 8; ++k) {
        const int c0 = 8 * k;
        const int q0 = i * FBKV + c0;
        const float4 la = *reinterpret_cast<const float4*>(ldl + c0);
        const float4 lb = *reinterpret_cast<const float4*>(ldl + c0 + 4);
        const float4 da = *reinterpret_cast<const float4*>(ldl + FBKV + c0);
        const float4 db = *reinterpret_cast<const float4*>(ldl + FBKV + c0 + 4);
        const float l8[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
        const float d8[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
        float p[8], ds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float pe = ex2f(fmaf(__uint_as_float(sv[c0 + e]), sl2, -l8[e]));
          if (diag && (q0 + e < key)) pe = 0.f;
          p[e] = pe;
          ds[e] = pe * (__uint_as_float(dv[c0 + e]) - d8[e]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sv[c0 + e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
          dv[c0 + e] = pack_bf16x2(ds[2 * e], ds[2 * e + 1]);
        }
      }
      // the previous block's dV / dK MMAs have read P^T and dS^T
      if (n >= 1 && !mbar_wait(pt_free, (n - 1) & 1u)) {
        ok = false;
        break;
      }
      uint8_t* pt = smem + DKV_P_OFF;
      uint8_t* dst = smem + DKV_DS_OFF;
#pragma unroll
      for (int k = 0; k < FBKV / 8; ++k) {
        *reinterpret_cast<uint4*>(pt + sw128(kr, k)) =
            make_uint4(sv[8 * k], sv[8 * k + 1], sv[8 * k + 2], sv[8 * k + 3]);
        *reinterpret_cast<uint4*>(dst + sw128(kr, k)) =
            make_uint4(dv[8 * k], dv[8 * k + 1], dv[8 * k + 2], dv[8 * k + 3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(acc_done, 0)) {
      tc_fence_after();
      uint32_t a[64];
      tmem_ld32(tl + 128, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
      tmem_ld32(tl + 160, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
      tmem_wait_ld();
      if (key < T) {
        bf16* vrow = dqkv + ((long)b * T + key) * (3L * C) + 2 * C + h * HD;
#pragma unroll
        for (int e = 0; e < HD; e += 8)
          *reinterpret_cast<uint4*>(vrow + e) = make_uint4(
              pack_bf16x2(__uint_as_float(a[e]), __uint_as_float(a[e + 1])),
              pack_bf16x2(__uint_as_float(a[e + 2]), __uint_as_float(a[e + 3])),
              pack_bf16x2(__uint_as_float(a[e + 4]), __uint_as_float(a[e + 5])),
              pack_bf16x2(__uint_as_float(a[e + 6]), __uint_as_float(a[e + 7])));
      }
      tmem_ld32(tl + 192, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
      tmem_ld32(tl + 224, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
      tmem_wait_ld();
      if (key < T) {
        bf16* krow = dqkv + ((long)b * T + key) * (3L * C) + C + h * HD;
#pragma unroll
        for (int e = 0; e < HD; e += 8)
          *reinterpret_cast<uint4*>(krow + e) = make_uint4(
              pack_bf16x2(__uint_as_float(a[e]) * scale, __uint_as_float(a[e + 1]) * scale),
              pack_bf16x2(__uint_as_float(a[e + 2]) * scale, __uint_as_float(a[e + 3]) * scale),
              pack_bf16x2(__uint_as_float(a[e + 4]) * scale, __uint_as_float(a[e + 5]) * scale),
              pack_bf16x2(__uint_as_float(a[e + 6]) * scale, __uint_as_float(a[e + 7]) * scale));
      }
    } else {
      ok = false;
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(DKV_TMEM_COLS) : "memory");
  }
}

// ----------------------------------------------------------------- dQ
// One CTA owns 128 queries and walks the 64-key blocks up to its last query.
// 256 TMEM columns and ~97 KB of shared memory, so two CTAs share an SM.  S and
// dP are released as soon as the compute warps hold them in registers, so
// S_{j+1}, dP_{j+1} and dQ += dS_j K_j run on the tensor cores while the warps
// form dS_{j+1}; dS is double-buffered in shared memory.
constexpr int DQ_STAGES = 2;
constexpr int DQ_Q_OFF = 0;                                       // Q 128 x 64 (two 64-row boxes)
constexpr int DQ_DO_OFF = TILE;                                   // dO 128 x 64
constexpr int DQ_RING_OFF = 2 * TILE;                             // stage s: K at +2s*HTILE, V at +(2s+1)*HTILE
constexpr int DQ_DS_OFF = DQ_RING_OFF + 2 * DQ_STAGES * HTILE;    // two dS buffers of 128 x 64
constexpr int DQ_BAR_OFF = DQ_DS_OFF + 2 * TILE;
constexpr int DQ_SMEM = DQ_BAR_OFF + 256 + 1024;
constexpr uint32_t DQ_TMEM_COLS = 256;                            // S 0, dP 64, dQ 128

__global__ void __launch_bounds__(192, 2)
    dq_kernel(const __grid_constant__ CUtensorMap tm_qkv64, const __grid_constant__ CUtensorMap tm_do,
              const bf16* __restrict__ out, const float* __restrict__ lse, float* __restrict__ Dv,
              bf16* __restrict__ dqkv, int T, int H, float scale, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_BAR_OFF);
  uint64_t* q_full = bars;                 // Q and dO tiles
  uint64_t* kv_full = bars + 1;            // DQ_STAGES
  uint64_t* kv_empty = kv_full + DQ_STAGES;
  uint64_t* s_full = kv_empty + DQ_STAGES;
  uint64_t* s_free = s_full + 1;           // count 4
  uint64_t* p_full = s_free + 1;           // 2, count 4
  uint64_t* acc_done = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;  // most key blocks first
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD;
  const int row0 = b * T;
  const int qlast = min(qb * BQ + BQ - 1, T - 1);
  const int nblk = qlast / FBKV + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < DQ_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(&p_full[0], 4);
    mbar_init(&p_full[1], 4);
    mbar_init(acc_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(DQ_TMEM_COLS)
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
      mbar_expect_tx(q_full, 2 * TILE);
      tma_load_2d(smem_u32(smem + DQ_Q_OFF), &tm_qkv64, h * HD, row0 + qb * BQ, q_full);
      tma_load_2d(smem_u32(smem + DQ_Q_OFF + HTILE), &tm_qkv64, h * HD, row0 + qb * BQ + 64, q_full);
      tma_load_2d(smem_u32(smem + DQ_DO_OFF), &tm_do, h * HD, row0 + qb * BQ, q_full);
      uint32_t issued = 0;
      for (int j = 0; j < nblk; ++j, ++issued) {
        const int s = j % DQ_STAGES;
        if (!mbar_wait(&kv_empty[s], ((j / DQ_STAGES) & 1u) ^ 1u)) {
          set_device_err(DERR_WAIT_TIMEOUT);
          break;
        }
        mbar_expect_tx(&kv_full[s], 2 * HTILE);
        const uint32_t dst = smem_u32(smem + DQ_RING_OFF + 2 * s * HTILE);
        tma_load_2d(dst, &tm_qkv64, C + h * HD, row0 + j * FBKV, &kv_full[s]);
        tma_load_2d(dst + HTILE, &tm_qkv64, 2 * C + h * HD, row0 + j * FBKV, &kv_full[s]);
      }
      for (int s = 0; s < DQ_STAGES; ++s) {
        if ((uint32_t)s < issued) {
          const uint32_t last = issued - 1 - ((issued - 1 - s) % DQ_STAGES);
          if (!mbar_wait(&kv_empty[s], (last / DQ_STAGES) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
      if (!mbar_wait(q_full, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      // S, dP: M=128 queries, N=64 keys, K=64 (d), both operands K-major
      const uint32_t id_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(FBKV >> 3) << 17) |
                            ((uint32_t)(BQ >> 4) << 24);
      // dQ += dS K_j: M=128, N=64 (d), K=64 keys; K_j read MN-major
      const uint32_t id_acc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(HD >> 3) << 17) |
                              ((uint32_t)(BQ >> 4) << 24);
      bool ok = mbar_wait(q_full, 0);
      const uint32_t qa = smem_u32(smem + DQ_Q_OFF), doa = smem_u32(smem + DQ_DO_OFF);
      const uint32_t dsa = smem_u32(smem + DQ_DS_OFF);
      auto dq_step = [&](int i) -> bool {
        const int pb = i & 1;
        if (!mbar_wait(&p_full[pb], (i >> 1) & 1u)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + DQ_RING_OFF + 2 * (i % DQ_STAGES) * HTILE);
#pragma unroll
        for (int kk = 0; kk < FBKV / 16; ++kk)
          tc_mma(tmem + 128, make_sdesc(dsa + pb * TILE + kk * 32, 0), make_sdesc(ka + kk * 2048, 1), id_acc,
                 (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&kv_empty[i % DQ_STAGES]);
        return true;
      };
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % DQ_STAGES;
        if (!mbar_wait(&kv_full[s], (j / DQ_STAGES) & 1u)) {
          ok = false;
          break;
        }
        if (j >= 1 && !mbar_wait(s_free, (j - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + DQ_RING_OFF + 2 * s * HTILE);
        const uint32_t va = ka + HTILE;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          tc_mma(tmem, make_sdesc(qa + kk * 32, 0), make_sdesc(ka + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
          tc_mma(tmem + 64, make_sdesc(doa + kk * 32, 0), make_sdesc(va + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
        if (j >= 1 && !dq_step(j - 1)) ok = false;
      }
      if (ok && !dq_step(nblk - 1)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(acc_done);
      if (!mbar_wait(acc_done, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------- compute warps
    const int qw = warp & 3;
    const int r = qw * 32 + lane;  // query row within the block
    const int q = qb * BQ + r;
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    const float l2 = q < T ? lse[((long)b * H + h) * T + q] * 1.4426950408889634f : INFINITY;
    // D_q = sum_d dO[q,d] O[q,d] from the dO tile in shared memory and this
    // query's row of O; written out for dkdv_kernel, which runs next
    bool ok = mbar_wait(q_full, 0);
    float dq_ = 0.f;
    if (ok && q < T) {
      const bf16* orow = out + ((long)b * T + q) * C + h * HD;
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
      Dv[((long)b * H + h) * T + q] = dq_;
    }
    for (int j = 0; ok && j < nblk; ++j) {
      if (!mbar_wait(s_full, j & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[64], dv[64];
      tmem_ld32(tl, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tl + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(tl + 64, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
      tmem_ld32(tl + 96, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      const bool diag = j * FBKV + FBKV - 1 > qb * BQ;
      uint8_t* dst = smem + DQ_DS_OFF + (j & 1) * TILE;
#pragma unroll
      for (int k = 0; k < FBKV / 8; ++k) {
        float ds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int key = j * FBKV + 8 * k + e;
          float pe = ex2f(fmaf(__uint_as_float(sv[8 * k + e]), sl2, -l2));
          if (diag && key > q) pe = 0.f;
          ds[e] = pe * (__uint_as_float(dv[8 * k + e]) - dq_);
        }
        *reinterpret_cast<uint4*>(dst + sw128(r, k)) =
            make_uint4(pack_bf16x2(ds[0], ds[1]), pack_bf16x2(ds[2], ds[3]), pack_bf16x2(ds[4], ds[5]),
                       pack_bf16x2(ds[6], ds[7]));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
    }
    if (ok && mbar_wait(acc_done, 0)) {
      tc_fence_after();
      uint32_t a[64];
      tmem_ld32(tl + 128, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
      tmem_ld32(tl + 160, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
      tmem_wait_ld();
      if (q < T) {
        bf16* qrow = dqkv + ((long)b * T + q) * (3L * C) + h * HD;
#pragma unroll
        for (int e = 0; e < HD; e += 8)
          *reinterpret_cast<uint4*>(qrow + e) = make_uint4(
              pack_bf16x2(__uint_as_float(a[e]) * scale, __uint_as_float(a[e + 1]) * scale),
              pack_bf16x2(__uint_as_float(a[e + 2]) * scale, __uint_as_float(a[e + 3]) * scale),
              pack_bf16x2(__uint_as_float(a[e + 4]) * scale, __uint_as_float(a[e + 5]) * scale),
              pack_bf16x2(__uint_as_float(a[e + 6]) * scale, __uint_as_float(a[e + 7]) * scale));
      }
    } else {
      ok = false;
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(DQ_TMEM_COLS) : "memory");
  }
}

// dq_kernel first (it also writes D = rowsum(dO * O) to Dv), then dkdv_kernel.
// Dv: caller-provided fp32 scratch of B*H*T elements.
static inline cudaError_t backward(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, bf16* dqkv,
                                   float* Dv, int B, int T, int H, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKV_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dkdv_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int C = H * HD;
  CUtensorMap tq64, td, td64;
  if (make_tmap(&tq64, qkv, 3L * C, (long)B * T, 3L * C, 64, 64) != 0) return cudaErrorInvalidValue;
  if (make_tmap(&td, dout, C, (long)B * T, C, 64, 128) != 0) return cudaErrorInvalidValue;
  if (make_tmap(&td64, dout, C, (long)B * T, C, 64, 64) != 0) return cudaErrorInvalidValue;
  const float scale = 1.f / sqrtf((float)HD);
  const float sl2 = 1.4426950408889634f * scale;
  dim3 grid((T + BQ - 1) / BQ, B * H);
  dq_kernel<<<grid, 192, DQ_SMEM, st>>>(tq64, td, out, lse, Dv, dqkv, T, H, scale, sl2);
  dkdv_kernel<<<grid, 192, DKV_SMEM, st>>>(tq64, td64, lse, Dv, dqkv, T, H, scale, sl2);
  return cudaGetLastError();
}

}  // namespace tcfa
