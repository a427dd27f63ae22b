// Causal attention on the 5th-generation tensor cores (tcgen05): the forward
// kernel and the helpers the backward kernels share.
//
// bf16 qkv [B, T, 3C] (q, k, v column blocks, head h in columns h*64..),
// head dim 64; output o [B, T, C] bf16 and lse [B, H, T] fp32.  One CTA owns
// 128 queries of one (batch, head) and walks the blocks of 128 keys up to its
// last query:
//   S_j  = Q K_j^T        tcgen05.mma, M=128 x N=128 x K=64, fp32 in TMEM
//   P_j  = exp(S_j/sqrt(d) - m)   (online softmax, one thread per query row
//          holding the row's 128 scores; bf16 P written back into TMEM)
//   O   += P_j V_j        tcgen05.mma with A = P_j read from TMEM (K = 128
//          keys), B = V_j from shared memory; O accumulates in TMEM.
// The reference maximum m of a row moves lazily: only when a block raises some
// row's maximum by more than 2^8 (and for the first block).  Then O is
// rescaled in TMEM (load, multiply, store) before the block's PV MMA; most
// blocks need no rescale.  O/l at the end.
// Warp 0 loads Q once and K_j, V_j through a 2-stage TMA ring, warp 1 issues
// the MMAs (S_{j+1} runs while the softmax warps work on S_j), warps 2..5 do
// the softmax (warp w reads TMEM lanes 32*(w%4)..+31).  A CTA needs 256 TMEM
// columns and ~82 KB of shared memory, so two CTAs share an SM and each SM
// sub-partition runs two softmax warps.  All waits are bounded.
#pragma once
#include "common.cuh"

namespace tcfa {

using namespace tcg;

constexpr int BQ = 128;                     // queries per CTA
constexpr int BKV = 128;                    // keys per block
constexpr int HD = 64;                      // head dim
constexpr int TILE = 128 * 64 * 2;          // one 128 x 64 bf16 tile (16 KB)

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA and integer pipes, to take part of the exponentials off the
// MUFU unit without using any other MUFU-pipe instruction (no float/int
// conversion, no rounding instruction): adding 1.5 * 2^23 rounds x to the
// nearest integer n in the low mantissa bits, f = x - n lies in [-0.5, 0.5],
// 2^f comes from a cubic fitted here to minimise the maximum relative error
// on that interval (7.5e-5, below the 2^-9 rounding of the bf16 values it
// feeds), and n is shifted into the exponent field.  Results below 2^-125
// (and x = -inf) give 0, as ex2.approx.ftz flushes those below 2^-126.
__device__ __forceinline__ float ex2_fma(float x) {
  const float xc = fmaxf(x, -127.f);
  const float t = xc + 12582912.f;  // 1.5 * 2^23
  const float f = xc - (t - 12582912.f);
  const float p = fmaf(fmaf(fmaf(0.05517144f, f, 0.24261081f), f, 0.69326099f), f, 0.99992809f);
  const float y = __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
  return x < -125.f ? 0.f : y;
}

// byte offset of element (r, c) in a 128-row, 64-column bf16 K-major tile with
// the 128-byte swizzle (16-byte chunk c/8 of row r stored at chunk (c/8)^(r%8))
__device__ __forceinline__ uint32_t sw128(int r, int chunk) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4));
}

// bf16 kind::f16 instruction descriptor: fp32 accumulate, M=128, N given, B
// K-major (b_mn = 0) or MN-major (b_mn = 1); A K-major (shared memory or TMEM)
__host__ __device__ constexpr uint32_t att_idesc(int n, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]  (A: 128 lanes x 16 bf16 = 8 columns per MMA)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 64 consecutive fp32 TMEM columns of this thread's lane (two loads, no wait)
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t* r) {
  tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(r));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
}
// Bounded wait by every lane of a warp, with a warp-uniform outcome: the warp
// goes on only if every lane saw the phase complete, so the warp-collective
// tcgen05.ld / tcgen05.st that follow never run on part of a warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}
// Transposing warp reduction: lane L holds v[0..31] (one row, 32 columns);
// returns to lane L the sum over the 32 lanes of column L, in a fixed order.
__device__ __forceinline__ float warp_colsum32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

// 1-D bulk copy global -> shared, completing on an mbarrier (16-byte aligned, size % 16 == 0)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- forward
// Persistent: a CTA takes work items (one 128-query block of one (batch,
// head)) in a fixed order, longest first, and the pipeline runs across item
// boundaries: the next item's Q and first K/V blocks load and its first S MMA
// runs while the softmax warps finish the current item's output.
constexpr int F_STAGES = 2;
constexpr int FQ_OFF = 0;                                 // two Q buffers of 128 x 64
constexpr int FKV_OFF = 2 * TILE;                         // stage s: K at +2s*TILE, V at +(2s+1)*TILE
constexpr int FBAR_OFF = FKV_OFF + 2 * F_STAGES * TILE;
constexpr int F_SMEM = FBAR_OFF + 256 + 1024;
constexpr uint32_t F_TMEM_COLS = 256;                     // S [0,128), P (bf16 pairs) [128,192), O [192,256)
constexpr uint32_t FT_S = 0, FT_P = 128, FT_O = 192;
constexpr float RESCALE_LOG2 = 8.f;                       // lazy-rescale threshold (log2 units)
#ifndef EX2_FMA_EVERY
#define EX2_FMA_EVERY 0  // > 0: one pair of exponentials in EX2_FMA_EVERY through ex2_fma instead of MUFU
#endif

// The k-th work item of this CTA: items are numbered longest first and dealt
// to the CTAs in a snake order (CTA c takes c, 2G-1-c, 2G+c, 4G-1-c, ... for a
// grid of G), so each CTA's long and short items balance out; the sequence
// increases in k.
__device__ __forceinline__ int snake_item(int k) {
  const int G = gridDim.x, c = blockIdx.x;
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// The w-th work item in descending order of length: 128-row block index and
// (batch, head) row of the grid.
__device__ __forceinline__ void item_desc(int w, int nblk, int BH, int& blk, int& bh) {
  blk = nblk - 1 - w / BH;
  bh = w % BH;
}

__global__ void __launch_bounds__(192, 2)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse, int T,
               int H, int BH, float sl2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + FBAR_OFF);
  uint64_t* q_full = bars;                  // 2
  uint64_t* q_empty = bars + 2;             // 2: the item's last S MMA has read Q
  uint64_t* kv_full = bars + 4;             // F_STAGES
  uint64_t* kv_empty = kv_full + F_STAGES;  // F_STAGES
  uint64_t* s_full = kv_empty + F_STAGES;   // S in TMEM
  uint64_t* s_free = s_full + 1;            // count 4: S is in registers
  uint64_t* p_full = s_free + 1;            // count 4: P in TMEM (and O rescaled)
  uint64_t* pv_done = p_full + 1;           // O += P V complete
  uint64_t* drain = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BQ - 1) / BQ;
  const int nitems = nqb * BH;
  const int C = H * HD;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int s = 0; s < F_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
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
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_qkv)) : "memory");
      uint32_t g = 0, t = 0;
      bool ok = true;
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
        int qb, bh;
        item_desc(w, nqb, BH, qb, bh);
        const int b = bh / H, h = bh % H, row0 = b * T;
        const int nkv = min(qb * BQ + BQ - 1, T - 1) / BKV + 1;
        const uint32_t qbuf = t & 1u;
        if (!mbar_wait(&q_empty[qbuf], ((t >> 1) & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&q_full[qbuf], TILE);
        tma_load_2d(smem_u32(smem + FQ_OFF + qbuf * TILE), &tm_qkv, h * HD, row0 + qb * BQ, &q_full[qbuf]);
        for (int j = 0; j < nkv; ++j, ++g) {
          const int s = g % F_STAGES;
          if (!mbar_wait(&kv_empty[s], ((g / F_STAGES) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&kv_full[s], 2 * TILE);
          const uint32_t kd = smem_u32(smem + FKV_OFF + 2 * s * TILE);
          tma_load_2d(kd, &tm_qkv, C + h * HD, row0 + j * BKV, &kv_full[s]);
          tma_load_2d(kd + TILE, &tm_qkv, 2 * C + h * HD, row0 + j * BKV, &kv_full[s]);
        }
      }
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      // drain: every issued load has landed before the CTA exits
      for (int s = 0; s < F_STAGES; ++s) {
        if ((uint32_t)s < g) {
          const uint32_t last = g - 1 - ((g - 1 - s) % F_STAGES);
          if (!mbar_wait_drain(&kv_full[s], (last / F_STAGES) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
      for (uint32_t i = 0; i < 2; ++i) {
        if (i < t) {
          const uint32_t last = t - 1 - ((t - 1 - i) % 2);
          if (!mbar_wait_drain(&q_full[i], (last >> 1) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t id_s = att_idesc(BKV, 0);  // S: A = Q, B = K_j, both K-major, N = 128 keys
      constexpr uint32_t id_pv = att_idesc(HD, 1);  // PV: A = P (TMEM), B = V_j MN-major, N = 64
      uint32_t g = 0, t = 0;
      int prev_j = 0;  // block index (within its item) of step g-1
      bool ok = true;
      auto do_pv = [&](uint32_t gp, int jp) -> bool {
        if (!mbar_wait(p_full, gp & 1u)) return false;
        tc_fence_after();
        const int s = gp % F_STAGES;
        const uint32_t va = smem_u32(smem + FKV_OFF + (2 * s + 1) * TILE);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          tc_mma_ts(tmem + FT_O, tmem + FT_P + kk * 8, make_sdesc(va + kk * 2048, 1), id_pv,
                    (jp > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&kv_empty[s]);
        tc_commit(pv_done);
        return true;
      };
      for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k), ++t) {
        int qb, bh;
        item_desc(w, nqb, BH, qb, bh);
        const int nkv = min(qb * BQ + BQ - 1, T - 1) / BKV + 1;
        const uint32_t qbuf = t & 1u;
        if (!mbar_wait(&q_full[qbuf], (t >> 1) & 1u)) {
          ok = false;
          break;
        }
        const uint32_t qa = smem_u32(smem + FQ_OFF + qbuf * TILE);
        for (int j = 0; j < nkv; ++j, ++g) {
          const int s = g % F_STAGES;
          if (!mbar_wait(&kv_full[s], (g / F_STAGES) & 1u) || (g >= 1 && !mbar_wait(s_free, (g - 1) & 1u))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ka = smem_u32(smem + FKV_OFF + 2 * s * TILE);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            tc_mma(tmem + FT_S, make_sdesc(qa + kk * 32, 0), make_sdesc(ka + kk * 32, 0), id_s, kk > 0 ? 1u : 0u);
          tc_commit(s_full);
          if (j == nkv - 1) tc_commit(&q_empty[qbuf]);
          if (g >= 1 && !do_pv(g - 1, prev_j)) {
            ok = false;
            break;
          }
          prev_j = j;
        }
      }
      if (ok && g >= 1 && !do_pv(g - 1, prev_j)) ok = false;
      if (!ok) set_device_err(DERR_WAIT_TIMEOUT);
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------- softmax warps
    const int qw = warp & 3;                // TMEM lane quarter
    const int r = qw * 32 + lane;           // query row within the block
    const uint32_t tl = tmem + ((uint32_t)(qw * 32) << 16);
    uint32_t g = 0;
    bool ok = true;
    for (int k = 0, w = snake_item(0); ok && w < nitems; w = snake_item(++k)) {
      int qb, bh;
      item_desc(w, nqb, BH, qb, bh);
      const int b = bh / H, h = bh % H;
      const int q = qb * BQ + r;            // query position in the sequence
      const int nkv = min(qb * BQ + BQ - 1, T - 1) / BKV + 1;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv; ++j, ++g) {
        if (!warp_wait(s_full, g & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the 128-key row of S in registers (one TMEM wait), buffer released
        uint32_t v[BKV];
        tmem_ld64(tl + FT_S, v);
        tmem_ld64(tl + FT_S + 64, v + 64);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        // causal mask on the block that reaches past the block's first query
        if (j * BKV + BKV - 1 > qb * BQ) {
#pragma unroll
          for (int e = 0; e < BKV; ++e)
            if (j * BKV + e > q) v[e] = __float_as_uint(-INFINITY);
        }
        // row maximum of the raw scores in 8 chains; the positive scale
        // 1/sqrt(d)*log2(e) is applied to the maximum
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(v[i]);
#pragma unroll
        for (int e = 8; e < BKV; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e]));
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
        // p = 2^(s*sl2 - m_new) (one FFMA + ex2), row sum in 8 chains, packed
        // to bf16 pairs in place
        float rs8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) rs8[i] = 0.f;
#pragma unroll
        for (int e = 0; e < BKV; e += 2) {
          // one pair in every EX2_FMA_EVERY goes through the FMA pipe
          const bool fma_pipe = EX2_FMA_EVERY > 0 && (e / 2) % (EX2_FMA_EVERY > 0 ? EX2_FMA_EVERY : 1) ==
                                                         (EX2_FMA_EVERY > 0 ? EX2_FMA_EVERY : 1) - 1;
          const float a0 = fmaf(__uint_as_float(v[e]), sl2, -m_new);
          const float a1 = fmaf(__uint_as_float(v[e + 1]), sl2, -m_new);
          const float p0 = fma_pipe ? ex2_fma(a0) : ex2f(a0);
          const float p1 = fma_pipe ? ex2_fma(a1) : ex2f(a1);
          rs8[e & 7] += p0;
          rs8[(e + 1) & 7] += p1;
          v[e >> 1] = pack_bf16x2(p0, p1);
        }
        const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
        l = l * alpha + rs;
        m = m_new;
        // O += P V of the item's previous block is complete: the P buffer is
        // free and O final up to it; rescale O in TMEM when the reference
        // moved.  (For an item's first block the previous item's epilogue
        // already waited for its last PV.)
        if (j >= 1) {
          if (!warp_wait(pv_done, (g - 1) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (rescale) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t o[32];
              tmem_ld32(tl + FT_O + half * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tl + FT_O + half * 32, o);
            }
          }
        }
        tmem_st32(tl + FT_P, v);
        tmem_st32(tl + FT_P + 32, v + 32);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      // item epilogue: O / l and the log-sum-exp
      if (!warp_wait(pv_done, (g - 1) & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t o[HD];
      tmem_ld64(tl + FT_O, o);
      tmem_wait_ld();
      tc_fence_before();
      if (q < T) {
        const float inv = 1.f / l;
        bf16* orow = out + ((long)b * T + q) * C + h * HD;
#pragma unroll
        for (int i = 0; i < HD; i += 8)
          *reinterpret_cast<uint4*>(orow + i) = make_uint4(
              pack_bf16x2(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv),
              pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv),
              pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv),
              pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv));
        lse[((long)b * H + h) * T + q] = (m + __log2f(l)) * 0.6931471805599453f;
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

static int num_sms_attn() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

static inline cudaError_t forward(const bf16* qkv, bf16* out, float* lse, int B, int T, int H, cudaStream_t st) {
  static DeviceOnce once;
  cudaError_t e = run_once_per_device(once, [] {
    cudaError_t r = cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, F_SMEM);
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (e != cudaSuccess) return e;
  CUtensorMap tm;
  const int C = H * HD;
  if (make_tmap(&tm, qkv, 3L * C, (long)B * T, 3L * C, 64, BKV) != 0) return cudaErrorInvalidValue;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
  const int items = ((T + BQ - 1) / BQ) * B * H;
  const int grid = items < 2 * num_sms_attn() ? items : 2 * num_sms_attn();
  fwd_kernel<<<grid, 192, F_SMEM, st>>>(tm, out, lse, T, H, B * H, sl2);
  return cudaGetLastError();
}

}  // namespace tcfa
