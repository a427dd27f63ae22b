// Causal attention backward on tcgen05 (bf16 operands, fp32 TMEM accumulators).
//
// With P = exp(S/sqrt(d) - lse) and D_q = sum_d dO_q . O_q:
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dK = dS^T Q / sqrt(d),
//   dQ = dS K / sqrt(d).
// Deterministic (no atomics).  The tile kernels are persistent with one CTA
// per SM and 128 x 128 score tiles; a CTA takes work items longest first in
// a snake order, and its pipeline runs across item boundaries (the next
// item's tiles load and its first MMAs run while the current item's results
// are written).
//  ld_kernel: lse*log2(e) and D per query, padded to whole 128-query blocks
//     (+inf / 0 past T), unless the caller already formed them.
//  dkdv_kernel: an item is 128 keys of one (batch, head); it walks the
//     128-query blocks that reach them:
//       S^T = K Q_i^T, dP^T = V dO_i^T     (M=128 keys, N=128 queries, K=64)
//       P^T, dS^T                          (sixteen compute warps, bf16 into TMEM)
//       dV += P^T dO_i, dK += dS^T Q_i     (A from TMEM, K=128 queries)
//     and stores every dS^T block as a bf16 tile: the compute warps write it
//     into a swizzled staging tile in shared memory, a store warp issues the
//     TMA stores.
//  dq_mma_kernel: dQ_i = sum_j dS_ij K_j / sqrt(d) from the stored tiles, so
//     no score is formed twice.
// Without room for the dS tiles (the no-allocation entry point), dq_kernel
// forms D and dQ from recomputed scores per 128-query block instead:
//       S = Q K_j^T, dP = dO V_j^T, dS = P * (dP - D), dQ += dS K_j
// and dkdv_kernel runs without its stores.  The score tiles go from TMEM to
// registers and back into TMEM as the A operand of the next MMAs.  Warp 0
// streams the operand tiles through a TMA ring, warp 1 issues the MMAs (one
// thread), warps 2..17 do the element-wise math: warps w, w+4, w+8 and w+12
// share TMEM lane quarter w%4 (one row each) and take the four 32-column
// quarters of the tile, so every SM sub-partition has four warps to hide the
// TMEM and shared-memory latencies with.  While the warps work on tile j, the
// tensor cores already run the next tile's score MMAs (and the accumulating
// MMAs of tile j-1).  The kernels can also add per-(128-row block, lane
// quarter) column sums of what they store (the qkv bias gradient) into a
// caller's buffer.  Every wait is bounded; the waits that drain a CTA's own
// copies and MMAs before it exits have their own fixed limit.
#pragma once
#include "attention.cuh"
#include "attention_tc.cuh"

namespace tcfa {

constexpr int BW_CWARPS = 16;                 // compute warps: four per TMEM lane quarter
constexpr int BW_THREADS = 64 + 32 * BW_CWARPS; // producer, MMA issuer, compute warps
constexpr int BW_CW = 128 / (BW_CWARPS / 4);    // score-tile columns per compute warp (32)
constexpr int BW_EW = 64 / (BW_CWARPS / 4);     // accumulator columns per compute warp (16)
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

__device__ __forceinline__ void store_row16(bf16* dst, const uint32_t (&a)[16], float scale) {
#pragma unroll
  for (int e = 0; e < 16; e += 8)
    *reinterpret_cast<uint4*>(dst + e) = make_uint4(
        pack_bf16x2(__uint_as_float(a[e]) * scale, __uint_as_float(a[e + 1]) * scale),
        pack_bf16x2(__uint_as_float(a[e + 2]) * scale, __uint_as_float(a[e + 3]) * scale),
        pack_bf16x2(__uint_as_float(a[e + 4]) * scale, __uint_as_float(a[e + 5]) * scale),
        pack_bf16x2(__uint_as_float(a[e + 6]) * scale, __uint_as_float(a[e + 7]) * scale));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// Transposing warp reduction of 16 columns: lane L holds v[0..15] (one row);
// returns to lanes L and L+16 the sum over the 32 lanes of column L (L < 16),
// in a fixed order.
__device__ __forceinline__ float warp_colsum16(float (&v)[16], int lane) {
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}
static_assert(BW_CW == 32 && BW_EW == 16, "the compute-warp code below handles 32 score and 16 output columns");

// wait (bounded) until every issued phase of a ring of n barriers has
// completed: the drain of a CTA's own in-flight copies before it exits
__device__ __forceinline__ void drain_ring(uint64_t* bars, int n, uint32_t issued) {
  for (int s = 0; s < n; ++s) {
    if ((uint32_t)s < issued) {
      const uint32_t last = issued - 1 - ((issued - 1 - s) % n);
      if (!mbar_wait_drain(&bars[s], (last / n) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  }
}

// TMA tile store shared -> global (bulk-group completion) and its waits
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int c0, int c1, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the committed stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// the committed stores are complete
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ----------------------------------------------------------------- dQ
// Shared memory: two buffers of (Q, dO) 128x64 tiles (16 KB each, 128-byte
// swizzled K-major rows of 64 bf16), then the ring of K_j, V_j tiles.
constexpr int DQ_QD_OFF = 0;                               // buffer b: Q at +2b*TILE, dO at +(2b+1)*TILE
constexpr int DQ_RING_OFF = 4 * TILE;                      // stage s: K at +2s*TILE, V at +(2s+1)*TILE
constexpr int DQ_D_OFF = DQ_RING_OFF + 2 * BW_STAGES * TILE;  // per item parity: lse*log2(e)[128], D[128]
constexpr int DQ_BAR_OFF = DQ_D_OFF + 2 * 2 * BT * 4;
constexpr int DQ_SMEM = DQ_BAR_OFF + 256 + 1024;
// TMEM columns: S [0,128), dP [128,256), dQ of item parity 0 / 1 [256,320) /
// [320,384), dS (bf16 pairs) [384,448)
constexpr uint32_t DQ_T_S = 0, DQ_T_DP = 128, DQ_T_DQ = 256, DQ_T_DS = 384;

__global__ void __launch_bounds__(BW_THREADS, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
              const bf16* __restrict__ out, const float* __restrict__ lse, float* __restrict__ ld_out,
              bf16* __restrict__ dqkv, float* __restrict__ colsum, int T, int H, int BH, float scale, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_BAR_OFF);
  uint64_t* q_full = bars;                   // 2: Q and dO tiles landed
  uint64_t* q_empty = bars + 2;              // 2, count 5: last S/dP MMA done and D formed
  uint64_t* kv_full = bars + 4;              // BW_STAGES
  uint64_t* kv_empty = kv_full + BW_STAGES;  // BW_STAGES
  uint64_t* s_full = kv_empty + BW_STAGES;   // S and dP in TMEM
  uint64_t* s_free = s_full + 1;             // count BW_CWARPS: S and dP are in registers
  uint64_t* ds_full = s_free + 1;            // count BW_CWARPS: dS in TMEM
  uint64_t* ds_free = ds_full + 1;           // dQ += dS K has read dS
  uint64_t* acc_full = ds_free + 1;          // 2: the item's dQ is complete
  uint64_t* acc_empty = acc_full + 2;        // 2, count 16: the item's dQ is in registers
  uint64_t* d_ready = acc_empty + 2;         // count 4: the item's lse*log2(e) and D are in shared memory
  uint64_t* drain = d_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BT - 1) / BT;
  const int nitems = nqb * BH;
  const int C = H * HD;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1 + BW_CWARPS / 4);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], BW_CWARPS);
    }
    for (int s = 0; s < BW_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, BW_CWARPS);
    mbar_init(ds_full, BW_CWARPS);
    mbar_init(ds_free, 1);
    mbar_init(d_ready, BW_CWARPS / 4);
    mbar_init(drain, 1);
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
      uint32_t g = 0, t = 0;
      bool ok = true;
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
        int qb, bh;
        item_desc(w, nqb, BH, qb, bh);
        const int b = bh / H, h = bh % H, row0 = b * T;
        const int nblk = min(qb * BT + BT - 1, T - 1) / BT + 1;
        const uint32_t qbuf = t & 1u;
        if (!mbar_wait(&q_empty[qbuf], ((t >> 1) & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&q_full[qbuf], 2 * TILE);
        const uint32_t qd = smem_u32(smem + DQ_QD_OFF + 2 * qbuf * TILE);
        tma_load_2d(qd, &tm_qkv, h * HD, row0 + qb * BT, &q_full[qbuf]);
        tma_load_2d(qd + TILE, &tm_do, h * HD, row0 + qb * BT, &q_full[qbuf]);
        for (int j = 0; j < nblk; ++j, ++g) {
          const int s = g % BW_STAGES;
          if (!mbar_wait(&kv_empty[s], ((g / BW_STAGES) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&kv_full[s], 2 * TILE);
          const uint32_t dst = smem_u32(smem + DQ_RING_OFF + 2 * s * TILE);
          tma_load_2d(dst, &tm_qkv, C + h * HD, row0 + j * BT, &kv_full[s]);
          tma_load_2d(dst + TILE, &tm_qkv, 2 * C + h * HD, row0 + j * BT, &kv_full[s]);
        }
      }
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      drain_ring(kv_full, BW_STAGES, g);
      drain_ring(q_full, 2, t);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t id_s = att_idesc(BT, 0);   // S, dP: N = 128 keys, K = 64 (d)
      constexpr uint32_t id_dq = att_idesc(HD, 1);  // dQ: N = 64 (d), K = 128 keys, K_j MN-major
      uint32_t g = 0, t = 0;
      int pj = 0, plast = 0;   // step g-1: block index within its item, last block of it?
      uint32_t pt = 0;         // step g-1: item counter
      bool ok = true;
      auto dq_step = [&](uint32_t gp, int jp, uint32_t tp, int last) -> bool {
        const uint32_t ab = tp & 1u;
        if (jp == 0 && !mbar_wait(&acc_empty[ab], ((tp >> 1) & 1u) ^ 1u)) return false;
        if (!mbar_wait(ds_full, gp & 1u)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + DQ_RING_OFF + 2 * (gp % BW_STAGES) * TILE);
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          tc_mma_ts(tmem + DQ_T_DQ + ab * HD, tmem + DQ_T_DS + kk * 8, make_sdesc(ka + kk * 2048, 1), id_dq,
                    (jp > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&kv_empty[gp % BW_STAGES]);
        tc_commit(ds_free);
        if (last) tc_commit(&acc_full[ab]);
        return true;
      };
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
        int qb, bh;
        item_desc(w, nqb, BH, qb, bh);
        const int nblk = min(qb * BT + BT - 1, T - 1) / BT + 1;
        const uint32_t qbuf = t & 1u;
        if (!mbar_wait(&q_full[qbuf], (t >> 1) & 1u)) {
          ok = false;
          break;
        }
        const uint32_t qa = smem_u32(smem + DQ_QD_OFF + 2 * qbuf * TILE), doa = qa + TILE;
        for (int j = 0; j < nblk; ++j, ++g) {
          const int s = g % BW_STAGES;
          if (!mbar_wait(&kv_full[s], (g / BW_STAGES) & 1u) || (g >= 1 && !mbar_wait(s_free, (g - 1) & 1u))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ka = smem_u32(smem + DQ_RING_OFF + 2 * s * TILE);
          const uint32_t va = ka + TILE;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            tc_mma(tmem + DQ_T_S, make_sdesc(qa + kk * 32, 0), make_sdesc(ka + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
            tc_mma(tmem + DQ_T_DP, make_sdesc(doa + kk * 32, 0), make_sdesc(va + kk * 32, 0), id_s,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
          if (j == nblk - 1) tc_commit(&q_empty[qbuf]);
          if (g >= 1 && !dq_step(g - 1, pj, pt, plast)) {
            ok = false;
            break;
          }
          pj = j;
          pt = t;
          plast = j == nblk - 1;
        }
      }
      if (ok && g >= 1 && !dq_step(g - 1, pj, pt, plast)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------- compute warps
    const int qw = warp & 3;             // TMEM lane quarter
    const int cq = (warp - 2) >> 2;      // which 32 keys of the 128-key tile (and 16 dQ columns)
    const int r = qw * 32 + lane;        // query row within the block
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    float* Dsm = reinterpret_cast<float*>(smem + DQ_D_OFF);  // [item parity][lse2 128, D 128]
    uint32_t g = 0, t = 0;
    bool ok = true;
    for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
      int qb, bh;
      item_desc(w, nqb, BH, qb, bh);
      const int b = bh / H, h = bh % H, row0 = b * T;
      const int q = qb * BT + r;          // query position
      const int nblk = min(qb * BT + BT - 1, T - 1) / BT + 1;
      const uint32_t qbuf = t & 1u;
      float* dsm = Dsm + (t & 1u) * 2 * BT;
      if (cq == 0) {
        // D_q = sum_d dO[q,d] O[q,d] (the row of O from global memory, dO
        // from the tile in shared memory) and lse*log2(e), for the item's
        // four warps of this lane quarter and for dkdv_kernel
        const float l2 = q < T ? lse[(long)bh * T + q] * 1.4426950408889634f : INFINITY;
        if (!warp_wait(&q_full[qbuf], (t >> 1) & 1u)) {
          ok = false;
          break;
        }
        float dq_ = 0.f;
        if (q < T) {
          const bf16* orow = out + ((long)row0 + q) * C + h * HD;
          const uint8_t* dorow = smem + DQ_QD_OFF + (2 * qbuf + 1) * TILE;
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
        dsm[r] = l2;
        dsm[BT + r] = dq_;
        float* ldb = ld_out + ((long)bh * nqb + qb) * LD_FLOATS;
        ldb[r] = l2;
        ldb[BT + r] = dq_;
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&q_empty[qbuf]);  // this warp is done with the dO tile
          mbar_arrive(d_ready);
        }
      }
      if (!warp_wait(d_ready, t & 1u)) {
        ok = false;
        break;
      }
      const float l2 = dsm[r], dq_ = dsm[BT + r];
      for (int j = 0; j < nblk; ++j, ++g) {
        if (!warp_wait(s_full, g & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[32], dv[32];
        tmem_ld32(tl + DQ_T_S + cq * 32, sv);
        tmem_ld32(tl + DQ_T_DP + cq * 32, dv);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        const int k0 = j * BT + cq * 32;      // first key of this warp's columns
        const bool diag = k0 + 31 > qb * BT;  // some key of the columns follows some query of the block
        // dS = P * (dP - D), packed to bf16 pairs in place
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const bool fma_pipe = EX2_FMA_EVERY > 0 && (c / 2) % (EX2_FMA_EVERY > 0 ? EX2_FMA_EVERY : 1) ==
                                                         (EX2_FMA_EVERY > 0 ? EX2_FMA_EVERY : 1) - 1;
          const float a0 = fmaf(__uint_as_float(sv[c]), sl2, -l2), a1 = fmaf(__uint_as_float(sv[c + 1]), sl2, -l2);
          float p0 = fma_pipe ? ex2_fma(a0) : ex2f(a0);
          float p1 = fma_pipe ? ex2_fma(a1) : ex2f(a1);
          if (diag) {
            if (k0 + c > q) p0 = 0.f;
            if (k0 + c + 1 > q) p1 = 0.f;
          }
          sv[c >> 1] = pack_bf16x2(p0 * (__uint_as_float(dv[c]) - dq_), p1 * (__uint_as_float(dv[c + 1]) - dq_));
        }
        // the previous step's dQ MMA has read the dS buffer
        if (g >= 1 && !warp_wait(ds_free, (g - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st16(tl + DQ_T_DS + cq * 16, sv);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (!ok) break;
      // item epilogue: dQ (scaled) and its column sums
      const uint32_t ab = t & 1u;
      if (!warp_wait(&acc_full[ab], (t >> 1) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t a[16];
      tmem_ld16(tl + DQ_T_DQ + ab * HD + cq * 16, a);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      float cs[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) cs[i] = q < T ? __uint_as_float(a[i]) * scale : 0.f;
      if (q < T) store_row16(dqkv + ((long)row0 + q) * (3L * C) + h * HD + cq * 16, a, scale);
      if (colsum) {
        const float tot = warp_colsum16(cs, lane);
        if (lane < 16) colsum[(((long)b * nqb + qb) * 4 + qw) * (3L * C) + h * HD + cq * 16 + lane] += tot;
      }
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BW_TMEM_COLS) : "memory");
  }
}

// ------------------------------------------------------------ dK, dV
// Shared memory: two buffers of (K, V) 128x64 tiles, then the ring of Q_i,
// dO_i tiles and the block's lse*log2(e) / D rows (33 KB per stage), then the
// staging tile of dS^T for its TMA store (four 64x64 boxes, [key half][query
// half], 128-byte swizzled rows).
constexpr int DKV_STAGES = 3;
constexpr int DKV_STORE_WARP = 2 + BW_CWARPS;           // the warp that issues the dS^T TMA stores
constexpr int DKV_THREADS = BW_THREADS + 32;
constexpr int DKV_KV_OFF = 0;                              // buffer b: K at +2b*TILE, V at +(2b+1)*TILE
constexpr int DKV_STAGE_BYTES = 2 * TILE + LD_FLOATS * 4;
constexpr int DKV_RING_OFF = 4 * TILE;                     // stage s: Q, dO, lse2/D
constexpr int DKV_DS_OFF = DKV_RING_OFF + DKV_STAGES * DKV_STAGE_BYTES;
constexpr int DKV_BAR_OFF = DKV_DS_OFF + 2 * TILE;
constexpr int DKV_SMEM = DKV_BAR_OFF + 256 + 1024;
// TMEM columns: three 128-column score regions, then dV [384,448) and dK
// [448,512).  Block g of a CTA's sequence puts S^T in region g%3 and dP^T in
// region (g+1)%3; once both are in registers, P^T and dS^T (bf16 pairs) go
// back into S^T's region, each warp into the 32 columns it read: P^T of its
// 32 queries in the first 16, dS^T in the last 16 (so the 16-query K step kk
// of the dV / dK MMAs reads columns 32(kk/2) + 8(kk%2) and 16 further on).
// The MMAs run in issue order, so a region is rewritten only after the MMAs
// that read it, and the compute warps need not wait for the previous block's
// dV / dK MMAs before writing P^T and dS^T.
constexpr uint32_t DKV_T_DV = 384, DKV_T_DK = 448;
__device__ __forceinline__ uint32_t dkv_region(uint32_t g) { return 128u * (g % 3u); }
static_assert(DKV_STAGE_BYTES % 1024 == 0, "ring stages keep the 1024-byte swizzle alignment");

__global__ void __launch_bounds__(DKV_THREADS, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_ds, const float* __restrict__ ld_in, bf16* __restrict__ dqkv,
                float* __restrict__ colsum, int store_ds, int T, int H, int BH, float scale, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DKV_BAR_OFF);
  uint64_t* kv_full = bars;                  // 2: K and V tiles
  uint64_t* kv_empty = bars + 2;             // 2: the item's last S^T / dP^T MMA has read them
  uint64_t* qd_full = bars + 4;              // DKV_STAGES
  uint64_t* qd_empty = qd_full + DKV_STAGES;  // DKV_STAGES
  uint64_t* s_full = qd_empty + DKV_STAGES;   // S^T and dP^T in TMEM
  uint64_t* s_free = s_full + 1;             // count BW_CWARPS
  // p_full: P^T and dS^T in TMEM, count BW_CWARPS, one per block parity (the
  // compute warps no longer wait for the issuer between blocks, so with a
  // single barrier they could complete a second phase before it waits on the
  // first)
  uint64_t* p_full = s_free + 1;             // 2
  uint64_t* acc_done = p_full + 2;           // the item's dV / dK are complete
  uint64_t* drain = acc_done + 1;
  uint64_t* st_full = drain + 1;             // count BW_CWARPS: the dS^T staging tile is written
  uint64_t* st_free = st_full + 1;           // the previous tile's TMA store has read the staging tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(st_free + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BT - 1) / BT;
  const int nitems = nqb * BH;
  const int C = H * HD;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int s = 0; s < DKV_STAGES; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, BW_CWARPS);
    mbar_init(&p_full[0], BW_CWARPS);
    mbar_init(&p_full[1], BW_CWARPS);
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    mbar_init(st_full, BW_CWARPS);
    mbar_init(st_free, 1);
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

  // items in ascending key block: key block 0 meets the most query blocks
  auto item = [&](int w, int& kb, int& bh) {
    kb = w / BH;
    bh = w % BH;
  };

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------- producer
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_qkv)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_do)) : "memory");
      uint32_t g = 0, t = 0;
      bool ok = true;
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
        int kb, bh;
        item(w, kb, bh);
        const int b = bh / H, h = bh % H, row0 = b * T;
        const int nblk = nqb - kb;  // query blocks kb .. nqb-1
        const uint32_t kvb = t & 1u;
        if (!mbar_wait(&kv_empty[kvb], ((t >> 1) & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&kv_full[kvb], 2 * TILE);
        const uint32_t kd = smem_u32(smem + DKV_KV_OFF + 2 * kvb * TILE);
        tma_load_2d(kd, &tm_qkv, C + h * HD, row0 + kb * BT, &kv_full[kvb]);
        tma_load_2d(kd + TILE, &tm_qkv, 2 * C + h * HD, row0 + kb * BT, &kv_full[kvb]);
        for (int n = 0; n < nblk; ++n, ++g) {
          const int i = kb + n, s = g % DKV_STAGES;
          if (!mbar_wait(&qd_empty[s], ((g / DKV_STAGES) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&qd_full[s], DKV_STAGE_BYTES);
          const uint32_t dst = smem_u32(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES);
          tma_load_2d(dst, &tm_qkv, h * HD, row0 + i * BT, &qd_full[s]);
          tma_load_2d(dst + TILE, &tm_do, h * HD, row0 + i * BT, &qd_full[s]);
          bulk_load(dst + 2 * TILE, ld_in + ((long)bh * nqb + i) * LD_FLOATS, LD_FLOATS * 4, &qd_full[s]);
        }
      }
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      drain_ring(qd_full, DKV_STAGES, g);
      drain_ring(kv_full, 2, t);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t id_s = att_idesc(BT, 0);    // S^T, dP^T: N = 128 queries, K = 64 (d)
      constexpr uint32_t id_acc = att_idesc(HD, 1);  // dV, dK: N = 64 (d), K = 128 queries, B MN-major
      uint32_t g = 0, t = 0;
      int pn = 0, plast = 0;  // step g-1: block index within its item, last block of it?
      bool ok = true;
      auto acc_step = [&](uint32_t gp, int np, int last) -> bool {
        if (!mbar_wait(&p_full[gp & 1u], (gp >> 1) & 1u)) return false;
        tc_fence_after();
        const int s = gp % DKV_STAGES;
        const uint32_t qa = smem_u32(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES);
        const uint32_t doa = qa + TILE;
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          const uint32_t acc = (np > 0 || kk > 0) ? 1u : 0u;
          const uint32_t pa = tmem + dkv_region(gp) + (kk >> 1) * 32 + (kk & 1) * 8;
          tc_mma_ts(tmem + DKV_T_DV, pa, make_sdesc(doa + kk * 2048, 1), id_acc, acc);
          tc_mma_ts(tmem + DKV_T_DK, pa + 16, make_sdesc(qa + kk * 2048, 1), id_acc, acc);
        }
        tc_commit(&qd_empty[s]);
        if (last) tc_commit(acc_done);
        return true;
      };
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
        int kb, bh;
        item(w, kb, bh);
        const int nblk = nqb - kb;
        const uint32_t kvb = t & 1u;
        if (!mbar_wait(&kv_full[kvb], (t >> 1) & 1u)) {
          ok = false;
          break;
        }
        const uint32_t ka = smem_u32(smem + DKV_KV_OFF + 2 * kvb * TILE), va = ka + TILE;
        for (int n = 0; n < nblk; ++n, ++g) {
          const int s = g % DKV_STAGES;
          if (!mbar_wait(&qd_full[s], (g / DKV_STAGES) & 1u) || (g >= 1 && !mbar_wait(s_free, (g - 1) & 1u))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qa = smem_u32(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES);
          const uint32_t doa = qa + TILE;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            tc_mma(tmem + dkv_region(g), make_sdesc(ka + kk * 32, 0), make_sdesc(qa + kk * 32, 0), id_s,
                   kk > 0 ? 1u : 0u);
            tc_mma(tmem + dkv_region(g + 1), make_sdesc(va + kk * 32, 0), make_sdesc(doa + kk * 32, 0), id_s,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
          if (n == nblk - 1) tc_commit(&kv_empty[kvb]);
          if (g >= 1 && !acc_step(g - 1, pn, plast)) {
            ok = false;
            break;
          }
          pn = n;
          plast = n == nblk - 1;
        }
      }
      if (ok && g >= 1 && !acc_step(g - 1, pn, plast)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else if (warp == DKV_STORE_WARP) {
    if (lane == 0 && store_ds) {
      // ------------------------------------------------- dS^T store warp
      // once the compute warps have written a block's dS^T into the staging
      // tile: four TMA stores to tile (bh, query block i, key block kb), and
      // the staging tile is handed back once the stores have read it
      uint32_t g = 0;
      bool ok = true;
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k)) {
        int kb, bh;
        item(w, kb, bh);
        const int nblk = nqb - kb;
        for (int n = 0; n < nblk; ++n, ++g) {
          const int i = kb + n;
          if (!mbar_wait(st_full, g & 1u)) {
            ok = false;
            break;
          }
          const int y = (bh * (nqb * (nqb + 1) / 2) + i * (i + 1) / 2 + kb) * BT;
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_store_2d(&tm_ds, (bx & 1) * 64, y + (bx >> 1) * 64, smem_u32(smem + DKV_DS_OFF + bx * 8192));
          bulk_commit();
          bulk_wait_read0();
          mbar_arrive(st_free);
        }
      }
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      bulk_wait0();  // the dS^T stores are complete before the CTA exits
    }
  } else {
    // ---------------------------------------------------- compute warps
    const int qw = warp & 3;
    const int cq = (warp - 2) >> 2;  // which 32 queries of the 128-query tile (and 16 dK/dV columns)
    const int kr = qw * 32 + lane;   // key row within the block
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t g = 0, t = 0;
    bool ok = true;
    for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
      int kb, bh;
      item(w, kb, bh);
      const int b = bh / H, h = bh % H, row0 = b * T;
      const int nblk = nqb - kb;
      const int key = kb * BT + kr;  // key position
      for (int n = 0; n < nblk; ++n, ++g) {
        const int i = kb + n, s = g % DKV_STAGES;
        if (!warp_wait(s_full, g & 1u) || !warp_wait(&qd_full[s], (g / DKV_STAGES) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[32], dv[32];
        tmem_ld32(tl + dkv_region(g) + cq * 32, sv);
        tmem_wait_ld();
        tmem_ld32(tl + dkv_region(g + 1) + cq * 32, dv);  // (lands while P is formed)
        const int q0 = i * BT + cq * 32;          // first query of this warp's columns
        const bool diag = q0 < kb * BT + BT - 1;  // some query of the columns precedes some key
        const float* ldl =
            reinterpret_cast<const float*>(smem + DKV_RING_OFF + s * DKV_STAGE_BYTES + 2 * TILE) + cq * 32;
        // P^T in fp32, in place of S^T
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          const float4 la = *reinterpret_cast<const float4*>(ldl + c);
          const float4 lb = *reinterpret_cast<const float4*>(ldl + c + 4);
          const float l8[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = fmaf(__uint_as_float(sv[c + e]), sl2, -l8[e]);
            float pe = (EX2_FMA_EVERY > 0 && ((c + e) / 2) % (EX2_FMA_EVERY > 0 ? EX2_FMA_EVERY : 1) ==
                                                  (EX2_FMA_EVERY > 0 ? EX2_FMA_EVERY : 1) - 1)
                           ? ex2_fma(a)
                           : ex2f(a);
            if (diag && (q0 + c + e < key)) pe = 0.f;
            sv[c + e] = __float_as_uint(pe);
          }
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        // dS^T, then P^T and dS^T packed to bf16 pairs in place
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          const float4 da = *reinterpret_cast<const float4*>(ldl + BT + c);
          const float4 db = *reinterpret_cast<const float4*>(ldl + BT + c + 4);
          const float d8[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
          float p[8], ds[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            p[e] = __uint_as_float(sv[c + e]);
            p[e + 1] = __uint_as_float(sv[c + e + 1]);
            const float2 d = mul2(make_float2(p[e], p[e + 1]),
                                  sub2(make_float2(__uint_as_float(dv[c + e]), __uint_as_float(dv[c + e + 1])),
                                       make_float2(d8[e], d8[e + 1])));
            ds[e] = d.x;
            ds[e + 1] = d.y;
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sv[(c >> 1) + e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
            dv[(c >> 1) + e] = pack_bf16x2(ds[2 * e], ds[2 * e + 1]);
          }
        }
        if (store_ds) {
          // dS^T of this block for dq_mma_kernel: written into the swizzled
          // staging tile once the store warp's previous TMA store has read it
          if (!warp_wait(st_free, (g & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          const int rb = (qw & 1) * 32 + lane;  // row within its 64-row box
          uint8_t* box = smem + DKV_DS_OFF + ((qw >> 1) * 2 + (cq >> 1)) * 8192;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(box + sw128(rb, (cq & 1) * 4 + c4)) =
                make_uint4(dv[4 * c4], dv[4 * c4 + 1], dv[4 * c4 + 2], dv[4 * c4 + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(st_full);
        }
        // into the 32 columns of S^T's region that this warp has read
        tmem_st16(tl + dkv_region(g) + cq * 32, sv);
        tmem_st16(tl + dkv_region(g) + cq * 32 + 16, dv);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g & 1u]);
      }
      if (!ok) break;
      // item epilogue: dV, dK (scaled) and their column sums.  The next item's
      // first dV / dK MMAs overwrite the accumulators; they wait for that
      // item's first P^T / dS^T, which these warps write only after the loads
      // below.
      if (!warp_wait(acc_done, t & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t av[16], ak[16];
      tmem_ld16(tl + DKV_T_DV + cq * 16, av);
      tmem_ld16(tl + DKV_T_DK + cq * 16, ak);
      tmem_wait_ld();
      tc_fence_before();
      if (key < T) {
        store_row16(dqkv + ((long)row0 + key) * (3L * C) + 2 * C + h * HD + cq * 16, av, 1.f);
        store_row16(dqkv + ((long)row0 + key) * (3L * C) + C + h * HD + cq * 16, ak, scale);
      }
      if (colsum) {
        float cs[16];
        const long prow = (((long)b * nqb + kb) * 4 + qw) * (3L * C);
#pragma unroll
        for (int i = 0; i < 16; ++i) cs[i] = key < T ? __uint_as_float(ak[i]) * scale : 0.f;
        const float tk = warp_colsum16(cs, lane);
#pragma unroll
        for (int i = 0; i < 16; ++i) cs[i] = key < T ? __uint_as_float(av[i]) : 0.f;
        const float tv = warp_colsum16(cs, lane);
        if (lane < 16) {
          colsum[prow + C + h * HD + cq * 16 + lane] += tk;
          colsum[prow + 2 * C + h * HD + cq * 16 + lane] += tv;
        }
      }
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BW_TMEM_COLS) : "memory");
  }
}

// ------------------------------------------------------- lse / D rows
// The per-query values the backward kernels stream: lse*log2(e) and
// D = sum_d dO[q,d] O[q,d], padded to whole 128-query blocks (+inf and 0 past
// T), in ld[((b*H + h)*nqb + qb)*LD_FLOATS + r] and [... + BT + r].  One thread
// per (batch, head, padded position), positions fastest: a thread reads its
// row's 128 bytes in whole sectors and a warp writes 32 consecutive floats.
// The sum runs in the same order as in dq_kernel (four chains over pairs of
// columns), so either route gives the same bits.  V32: out and dout are
// 32-byte aligned (rows are read as 32-byte vectors), else 16-byte vectors.
template <bool V32>
__global__ void __launch_bounds__(256) ld_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout,
                                                 const float* __restrict__ lse, float* __restrict__ ld, int B, int T,
                                                 int H) {
  const int nqb = (T + BT - 1) / BT;
  const long n = (long)B * nqb * BT * H;
  const long gi = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= n) return;
  const int q = (int)(gi % ((long)nqb * BT));
  const long bhi = gi / ((long)nqb * BT);
  const int h = (int)(bhi % H), b = (int)(bhi / H);
  const int C = H * HD;
  float l2 = INFINITY, dq_ = 0.f;
  if (q < T) {
    l2 = lse[((long)b * H + h) * T + q] * 1.4426950408889634f;
    const bf16* orow = out + ((long)b * T + q) * C + h * HD;
    const bf16* drow = dout + ((long)b * T + q) * C + h * HD;
    // the whole 128-byte rows in flight at once
    uint32_t ov[HD / 16][8], dv[HD / 16][8];
#pragma unroll
    for (int c = 0; c < HD / 16; ++c) {
      if constexpr (V32) {
        ld32(orow + 16 * c, ov[c]);
        ld32(drow + 16 * c, dv[c]);
      } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint4 o = *reinterpret_cast<const uint4*>(orow + 16 * c + 8 * hh);
          const uint4 d = *reinterpret_cast<const uint4*>(drow + 16 * c + 8 * hh);
          ov[c][4 * hh] = o.x, ov[c][4 * hh + 1] = o.y, ov[c][4 * hh + 2] = o.z, ov[c][4 * hh + 3] = o.w;
          dv[c][4 * hh] = d.x, dv[c][4 * hh + 1] = d.y, dv[c][4 * hh + 2] = d.z, dv[c][4 * hh + 3] = d.w;
        }
      }
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < HD / 8; ++c) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 of = unpack_bf16x2(ov[c / 2][4 * (c % 2) + e]), df = unpack_bf16x2(dv[c / 2][4 * (c % 2) + e]);
        acc[e] = fmaf(of.x, df.x, fmaf(of.y, df.y, acc[e]));
      }
    }
    dq_ = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  }
  float* ldb = ld + (((long)b * H + h) * nqb + q / BT) * LD_FLOATS;
  ldb[q % BT] = l2;
  ldb[BT + q % BT] = dq_;
}

// ----------------------------------------------------- dQ from stored dS
// dQ_i = sum_{j <= i} dS_ij K_j / sqrt(d), with the bf16 dS tiles that
// dkdv_kernel stored (tile (bh, i, j) holds dS^T: row = key, 128 queries), so
// no score is formed twice.  Persistent, one CTA per SM, items (128 queries of
// one (batch, head)) longest first.  Warp 0 streams (dS_ij, K_j) through a
// 4-stage TMA ring; warp 1 issues dQ += dS_ij K_j (M = 128 queries, N = 64,
// K = 128 keys, A and B both MN-major in shared memory) into one of two TMEM
// accumulators (by item parity); warps 2..5 scale dQ, store it as bf16 and
// form its column sums, while the next item's MMAs run.  The MMAs add the key
// blocks in the order dq_kernel does, on the same bf16 values.
constexpr int DQM_STAGES = 4;
constexpr int DQM_STAGE = 3 * TILE;  // dS tile as four 64x64 boxes [key half][query half], then K_j
constexpr int DQM_BAR_OFF = DQM_STAGES * DQM_STAGE;
constexpr int DQM_SMEM = DQM_BAR_OFF + 256 + 1024;
constexpr uint32_t DQM_TMEM_COLS = 128;  // two 64-column dQ accumulators

__global__ void __launch_bounds__(192, 1)
    dq_mma_kernel(const __grid_constant__ CUtensorMap tm_ds, const __grid_constant__ CUtensorMap tm_qkv,
                  bf16* __restrict__ dqkv, float* __restrict__ colsum, int T, int H, int BH, float scale) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQM_BAR_OFF);
  uint64_t* full = bars;                    // DQM_STAGES
  uint64_t* empty = full + DQM_STAGES;      // DQM_STAGES
  uint64_t* acc_full = empty + DQM_STAGES;  // 2: the item's dQ is complete
  uint64_t* acc_empty = acc_full + 2;       // 2, count 4: the item's dQ is in registers
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BT - 1) / BT;
  const int nitems = nqb * BH;
  const int ntri = nqb * (nqb + 1) / 2;
  const int C = H * HD;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DQM_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(DQM_TMEM_COLS)
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
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_ds)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_qkv)) : "memory");
      uint32_t g = 0;
      bool ok = true;
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k)) {
        int qb, bh;
        item_desc(w, nqb, BH, qb, bh);
        const int b = bh / H, h = bh % H, row0 = b * T;
        const long trow = ((long)bh * ntri + (long)qb * (qb + 1) / 2) * BT;  // first row of tile (bh, qb, 0)
        for (int kb = 0; kb <= qb; ++kb, ++g) {
          const int s = g % DQM_STAGES;
          if (!mbar_wait(&empty[s], ((g / DQM_STAGES) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[s], DQM_STAGE);
          const uint32_t dst = smem_u32(smem + s * DQM_STAGE);
          const int y = (int)(trow + (long)kb * BT);
          tma_load_2d(dst, &tm_ds, 0, y, &full[s]);
          tma_load_2d(dst + 8192, &tm_ds, 64, y, &full[s]);
          tma_load_2d(dst + 16384, &tm_ds, 0, y + 64, &full[s]);
          tma_load_2d(dst + 24576, &tm_ds, 64, y + 64, &full[s]);
          tma_load_2d(dst + 2 * TILE, &tm_qkv, C + h * HD, row0 + kb * BT, &full[s]);
        }
      }
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      drain_ring(full, DQM_STAGES, g);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = att_idesc(HD, 1) | (1u << 15);  // N = 64, A and B MN-major
      uint32_t g = 0, t = 0;
      bool ok = true;
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
        int qb, bh;
        item_desc(w, nqb, BH, qb, bh);
        const uint32_t ab = t & 1u;
        if (!mbar_wait(&acc_empty[ab], ((t >> 1) & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb <= qb; ++kb, ++g) {
          const int s = g % DQM_STAGES;
          if (!mbar_wait(&full[s], (g / DQM_STAGES) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * DQM_STAGE);
#pragma unroll
          for (int kk = 0; kk < BT / 16; ++kk)
            tc_mma(tmem + ab * HD, make_sdesc(base + (kk >> 2) * 16384 + (kk & 3) * 2048, 1),
                   make_sdesc(base + 2 * TILE + kk * 2048, 1), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
          if (kb == qb) tc_commit(&acc_full[ab]);
        }
      }
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------- epilogue
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t t = 0;
    bool ok = true;
    for (int k = 0, w = snake_item(0); w < nitems; w = snake_item(++k), ++t) {
      int qb, bh;
      item_desc(w, nqb, BH, qb, bh);
      const int b = bh / H, h = bh % H, row0 = b * T;
      const int q = qb * BT + r;
      const uint32_t ab = t & 1u;
      if (!warp_wait(&acc_full[ab], (t >> 1) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t a0[32], a1[32];
      tmem_ld32(tl + ab * HD, a0);
      tmem_ld32(tl + ab * HD + 32, a1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      if (q < T) {
        bf16* dst = dqkv + ((long)row0 + q) * (3L * C) + h * HD;
        store_row32(dst, a0, scale);
        store_row32(dst + 32, a1, scale);
      }
      if (colsum) {
        const long prow = (((long)b * nqb + qb) * 4 + qw) * (3L * C) + h * HD;
        float cs[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) cs[i] = q < T ? __uint_as_float(a0[i]) * scale : 0.f;
        const float t0 = warp_colsum32(cs, lane);
#pragma unroll
        for (int i = 0; i < 32; ++i) cs[i] = q < T ? __uint_as_float(a1[i]) * scale : 0.f;
        const float t1 = warp_colsum32(cs, lane);
        colsum[prow + lane] += t0;
        colsum[prow + 32 + lane] += t1;
      }
    }
    if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(DQM_TMEM_COLS) : "memory");
  }
}

// fp32 scratch of the backward: lse*log2(e) and D per query, padded to whole
// 128-query blocks
static inline long backward_scratch_floats(int B, int T, int H) {
  return (long)B * H * ((T + BT - 1) / BT) * LD_FLOATS;
}
// bf16 elements of the stored dS tiles: 128 x 128 per (batch, head, query
// block, key block at or below it)
static inline long backward_ds_elems(int B, int T, int H) {
  const long nqb = (T + BT - 1) / BT;
  return (long)B * H * (nqb * (nqb + 1) / 2) * BT * BT;
}
// rows of the column-sum partials: one per (batch, 128-row block, lane quarter)
static inline long backward_colsum_rows(int B, int T) { return (long)B * ((T + BT - 1) / BT) * 4; }

// The attention backward.  ld: fp32 scratch of backward_scratch_floats(B, T,
// H) elements, 16-byte aligned.  colsum (may be null): [backward_colsum_rows(B,
// T)][3C] fp32 partial column sums of dqkv, added to what it holds (summing
// them over the rows gives the qkv bias gradient).
//  ds given (backward_ds_elems(B, T, H) bf16, 16-byte aligned): ld_kernel forms
//     lse*log2(e) and D (unless ld_ready: the caller already wrote them into
//     ld), dkdv_kernel forms P and dS once per score and stores dS,
//     dq_mma_kernel reads it back for dQ (three launches, or two).
//  ds null: dq_kernel forms D and dQ from recomputed scores, then dkdv_kernel
//     (two launches, no scratch beyond ld).
// Both routes run the same arithmetic on every score (the products of S and
// dP are the same bf16 pairs in either operand order, and every sum runs in
// the same order), so their results agree bit for bit.
static inline cudaError_t backward(const bf16* qkv, const bf16* out, const bf16* dout, const float* lse, bf16* dqkv,
                                   float* ld, int B, int T, int H, cudaStream_t st, float* colsum = nullptr,
                                   bf16* ds = nullptr, bool ld_ready = false) {
  static DeviceOnce once;
  cudaError_t e = run_once_per_device(once, [] {
    cudaError_t r = cudaFuncSetAttribute(dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKV_SMEM);
    if (r == cudaSuccess) r = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(dq_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQM_SMEM);
    return r;
  });
  if (e != cudaSuccess) return e;
  if ((reinterpret_cast<uintptr_t>(ld) & 15) || (reinterpret_cast<uintptr_t>(ds) & 15)) return cudaErrorInvalidValue;
  const int C = H * HD;
  CUtensorMap tq, td;
  if (make_tmap(&tq, qkv, 3L * C, (long)B * T, 3L * C, 64, BT) != 0) return cudaErrorInvalidValue;
  if (make_tmap(&td, dout, C, (long)B * T, C, 64, BT) != 0) return cudaErrorInvalidValue;
  const float scale = 1.f / sqrtf((float)HD);
  const float sl2 = 1.4426950408889634f * scale;
  const int items = ((T + BT - 1) / BT) * B * H;
  const int grid = items < num_sms_attn() ? items : num_sms_attn();
  if (ds != nullptr) {
    // (the TMA row coordinates of the dS tiles are 32-bit)
    if (backward_ds_elems(B, T, H) / BT >= (1L << 31)) return cudaErrorInvalidValue;
    CUtensorMap tds;
    if (make_tmap(&tds, ds, BT, backward_ds_elems(B, T, H) / BT, BT, 64, 64) != 0) return cudaErrorInvalidValue;
    const long n = (long)B * ((T + BT - 1) / BT) * BT * H;
    if (ld_ready) {
      // lse*log2(e) and D are already in ld (formed by the kernel that wrote dout)
    } else if (((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(dout)) & 31) == 0)
      ld_kernel<true><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(out, dout, lse, ld, B, T, H);
    else
      ld_kernel<false><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(out, dout, lse, ld, B, T, H);
    dkdv_kernel<<<grid, DKV_THREADS, DKV_SMEM, st>>>(tq, td, tds, ld, dqkv, colsum, 1, T, H, B * H, scale, sl2);
    dq_mma_kernel<<<grid, 192, DQM_SMEM, st>>>(tds, tq, dqkv, colsum, T, H, B * H, scale);
  } else {
    dq_kernel<<<grid, BW_THREADS, DQ_SMEM, st>>>(tq, td, out, lse, ld, dqkv, colsum, T, H, B * H, scale, sl2);
    dkdv_kernel<<<grid, DKV_THREADS, DKV_SMEM, st>>>(tq, td, tq, ld, dqkv, colsum, 0, T, H, B * H, scale, sl2);
  }
  return cudaGetLastError();
}

}  // namespace tcfa
