// bf16 GEMM on the 5th-generation tensor cores (tcgen05) for sm_100a.
//
//   D[M,N] = sum_k A[m,k] * B[n,k]      (bf16 operands, fp32 accumulation)
//
// with the epilogue fused (bias, GELU, GELU', residual add, gradient
// accumulation, split-K partials).  Every matrix product of the GPT-2 step is
// one of three forms of this contraction:
//   forward  Y = X W^T        A = X  [M,K] K-major   B = W  [N,K] K-major
//   dgrad   dX = dY W         A = dY [M,N] K-major   B = W  viewed [K,N] MN-major
//   wgrad   dW += dY^T X      A = dY viewed MN-major B = X  viewed MN-major
// ("K-major": the contraction index is contiguous in memory; "MN-major": the
// output index is contiguous.)  Both layouts are read straight from global
// memory by TMA with the 128-byte swizzle; no transposed copy is ever made.
//
// Design (one persistent CTA per SM, 10 warps):
//   warp 0      TMA producer: fills a ring of shared-memory stages (A tile
//               128x64, B tile BNx64 per stage) and signals an mbarrier.
//   warp 1      allocates TMEM and issues tcgen05.mma (one thread): 4 MMAs of
//               128xBNx16 per stage; tcgen05.commit frees the stage and, at the
//               end of a tile, marks the accumulator ready.
//   warps 2..9  epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane per
//               row), fused math, vectorised global stores.  Warps w and w+4
//               share a TMEM lane quarter and take the two column halves of the
//               tile, so every SM sub-partition runs two epilogue warps.  Two
//               accumulator buffers in TMEM let the epilogue of tile i overlap
//               the MMAs of tile i+1.
// Every mbarrier wait is bounded (about two seconds); a wait that gives up
// records an error in g_device_err and the kernel drains its own in-flight
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include "common.cuh"
#include "tc_gemm.h"

namespace tcg {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;

template <int BN>
struct Layout {
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
};

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete: gives up
// (returns false) after g_wait_limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  // (mbarrier.try_wait itself suspends the thread for a while before it
  // reports an incomplete phase, so the clock is read on every retry)
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    if (globaltimer_ns() - t0 > *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns)) return false;
  }
}
// The same with the fixed limit, for the waits that drain a kernel's own
// in-flight TMA copies and MMAs before it exits.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    if (globaltimer_ns() - t0 > DRAIN_LIMIT_NS) return false;
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bit.
//  K-major : rows of 128 B (64 bf16 along K); 8-row groups 1024 B apart (SBO).
//  MN-major: rows of 128 B (64 bf16 along M or N), one row per K index;
//            8-row K groups 1024 B apart (SBO); 64-wide M/N chunks 8 KB apart (LBO).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, int mn_major) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((mn_major ? (8192u >> 4) : 1u) & 0x3FFFu) << 16;
  d |= (uint64_t)((1024u >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor for kind::f16: bf16 x bf16 -> fp32, M=128, N=BN.
template <int BN>
__device__ __forceinline__ uint32_t make_idesc(int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void decode_tile(const Params& p, int tile, int& mb, int& nb, int& split) {
  int per_split = p.num_m * p.num_n;
  split = tile / per_split;
  int t = tile - split * per_split;
  mb = t % p.num_m;
  nb = t / p.num_m;
}

// 32-byte vector global accesses: one lane writes (or reads) a whole 32-byte
// sector in one instruction.  Used when the row stride keeps every 32-column
// chunk 32-byte aligned.
__device__ __forceinline__ void st32(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                     uint32_t f, uint32_t g, uint32_t h) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d), "r"(e),
               "r"(f), "r"(g), "r"(h)
               : "memory");
}
// (read-once streams: the residual, accumulator and pre-activation inputs of
// the epilogues do not allocate in L1, which keeps the bias there)
__device__ __forceinline__ void ld32(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}
// bias loads: every lane of a warp reads the same 16 bytes, tile after tile,
// so they are kept in L1 with the highest priority
__device__ __forceinline__ float4 ldg_keep(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::evict_last.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st_bf16x16(bf16* o, const float* v) {
  st32(o, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]),
       pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
}
__device__ __forceinline__ void st_f32x8(float* o, const float* v) {
  st32(o, __float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]),
       __float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]), __float_as_uint(v[7]));
}

// ------------------------------------------------------------- epilogue
// Fused math on the 32 consecutive columns [col0, col0+32) of one row.
// FULL: all 32 columns lie inside N and every 32-column chunk is 32-byte
// aligned (32-byte vector accesses); otherwise element-wise with masks.
template <bool FULL>
__device__ __forceinline__ void epi_store(const Params& p, int row, int col0, int split, const uint32_t (&r)[32]) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  const long base = (long)row * p.ldc + col0;
  if (p.bias != nullptr && p.epi != EPI_DGELU && p.epi != EPI_ACCUM_F32 && p.epi != EPI_PARTIAL_F32) {
    if (FULL) {
      const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 b = ldg_keep(b4 + i);
        v[4 * i] += b.x;
        v[4 * i + 1] += b.y;
        v[4 * i + 2] += b.z;
        v[4 * i + 3] += b.w;
      }
    } else {
      for (int i = 0; i < 32; ++i)
        if (col0 + i < p.N) v[i] += __ldg(p.bias + col0 + i);
    }
  }
  switch (p.epi) {
    case EPI_BF16: {
      bf16* o = reinterpret_cast<bf16*>(p.out) + base;
      if (FULL) {
        st_bf16x16(o, v);
        st_bf16x16(o + 16, v + 16);
      } else {
        for (int i = 0; i < 32; ++i)
          if (col0 + i < p.N) o[i] = f2bf(v[i]);
      }
    } break;
    case EPI_F32:
    case EPI_PARTIAL_F32: {
      float* o = (p.epi == EPI_F32 ? reinterpret_cast<float*>(p.out) : p.partial + (long)split * p.M * p.ldc) + base;
      if (FULL) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) st_f32x8(o + i, v + i);
      } else {
        for (int i = 0; i < 32; ++i)
          if (col0 + i < p.N) o[i] = v[i];
      }
    } break;
    case EPI_RESID_F32:
    case EPI_ACCUM_F32: {
      const long soff = p.epi == EPI_ACCUM_F32 ? (long)split * p.split_stride : 0;
      const float* rs = (p.epi == EPI_RESID_F32 ? p.resid : reinterpret_cast<const float*>(p.out) + soff) + base;
      float* o = reinterpret_cast<float*>(p.out) + soff + base;
      if (FULL) {
        uint32_t x[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) ld32(rs + 8 * i, x[i]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[8 * i + e] += __uint_as_float(x[i][e]);
          st_f32x8(o + 8 * i, v + 8 * i);
        }
      } else {
        for (int i = 0; i < 32; ++i)
          if (col0 + i < p.N) o[i] = rs[i] + v[i];
      }
    } break;
    case EPI_GELU: {
      bf16* o = reinterpret_cast<bf16*>(p.out) + base;
      bf16* o2 = p.out2 + base;
      float u[32], g[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        u[i] = bf2f(f2bf(v[i]));  // the stored pre-activation, as rounded
        g[i] = gelu_tanh<true>(u[i]);
      }
      if (FULL) {
        st_bf16x16(o, u);
        st_bf16x16(o + 16, u + 16);
        st_bf16x16(o2, g);
        st_bf16x16(o2 + 16, g + 16);
      } else {
        for (int i = 0; i < 32; ++i)
          if (col0 + i < p.N) {
            o[i] = f2bf(u[i]);
            o2[i] = f2bf(g[i]);
          }
      }
    } break;
    case EPI_DGELU: {
      bf16* o = reinterpret_cast<bf16*>(p.out) + base;
      const bf16* ua = p.aux + base;
      if (FULL) {
        uint32_t uw[2][8];
        ld32(ua, uw[0]);
        ld32(ua + 16, uw[1]);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 f = unpack_bf16x2(uw[h][e]);
            v[16 * h + 2 * e] *= gelu_tanh_grad<true>(f.x);
            v[16 * h + 2 * e + 1] *= gelu_tanh_grad<true>(f.y);
          }
        st_bf16x16(o, v);
        st_bf16x16(o + 16, v + 16);
      } else {
        for (int i = 0; i < 32; ++i)
          if (col0 + i < p.N) o[i] = f2bf(v[i] * gelu_tanh_grad<true>(bf2f(ua[i])));
      }
    } break;
    default:
      break;
  }
}

// The epilogues that read no memory besides the bias (EPI_BF16, EPI_F32,
// EPI_PARTIAL_F32, EPI_GELU) on 16 consecutive columns [col0, col0+16) of one
// row.  Vector path (32-byte accesses) when all 16 lie inside N; the caller
// has checked p.vec32.
__device__ __forceinline__ void epi_store16(const Params& p, int row, int col0, int split, const uint32_t (&r)[16]) {
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  const long base = (long)row * p.ldc + col0;
  const bool bias = p.bias != nullptr && p.epi != EPI_PARTIAL_F32;
  if (col0 + 16 > p.N) {
    for (int i = 0; i < 16 && col0 + i < p.N; ++i) {
      const float x = v[i] + (bias ? __ldg(p.bias + col0 + i) : 0.f);
      if (p.epi == EPI_BF16) {
        reinterpret_cast<bf16*>(p.out)[base + i] = f2bf(x);
      } else if (p.epi == EPI_GELU) {
        const float u = bf2f(f2bf(x));  // the stored pre-activation, as rounded
        reinterpret_cast<bf16*>(p.out)[base + i] = f2bf(u);
        p.out2[base + i] = f2bf(gelu_tanh<true>(u));
      } else {
        (p.epi == EPI_F32 ? reinterpret_cast<float*>(p.out) : p.partial + (long)split * p.M * p.ldc)[base + i] = x;
      }
    }
    return;
  }
  if (bias) {
    const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 b = ldg_keep(b4 + i);
      const float2 lo = add2(make_float2(v[4 * i], v[4 * i + 1]), make_float2(b.x, b.y));
      const float2 hi = add2(make_float2(v[4 * i + 2], v[4 * i + 3]), make_float2(b.z, b.w));
      v[4 * i] = lo.x;
      v[4 * i + 1] = lo.y;
      v[4 * i + 2] = hi.x;
      v[4 * i + 3] = hi.y;
    }
  }
  if (p.epi == EPI_BF16) {
    st_bf16x16(reinterpret_cast<bf16*>(p.out) + base, v);
  } else if (p.epi == EPI_GELU) {
    // u rounded to bf16 once; gelu of the rounded u
    uint32_t wu[8], wg[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      wu[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
      const float2 g = gelu_tanh2(unpack_bf16x2(wu[e]));
      wg[e] = pack_bf16x2(g.x, g.y);
    }
    st32(reinterpret_cast<bf16*>(p.out) + base, wu[0], wu[1], wu[2], wu[3], wu[4], wu[5], wu[6], wu[7]);
    st32(p.out2 + base, wg[0], wg[1], wg[2], wg[3], wg[4], wg[5], wg[6], wg[7]);
  } else {
    float* o = (p.epi == EPI_F32 ? reinterpret_cast<float*>(p.out) : p.partial + (long)split * p.M * p.ldc) + base;
    st_f32x8(o, v);
    st_f32x8(o + 8, v + 8);
  }
}

// Softmax statistics epilogue: the 64 accumulator columns [col0, col0+64) of
// one row are rounded to bf16 and stored (the logits), and their statistics
// (maximum, sum of exp(z - max), lowest index of the maximum), computed from
// the rounded values over the columns below N, are merged into (m, s, mi).
__device__ __forceinline__ void epi_ce_chunk(const Params& p, int row, int col0, uint32_t (&r)[64], float& m,
                                             float& s, int& mi) {
  bf16* o = reinterpret_cast<bf16*>(p.out) + (long)row * p.ldc + col0;
  float cm = -INFINITY;
  int ci = 0x7fffffff;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float z = bf2f(f2bf(__uint_as_float(r[i])));
    r[i] = __float_as_uint(z);
    if (col0 + i < p.N && z > cm) {
      cm = z;
      ci = col0 + i;
    }
  }
  if (col0 + 64 <= p.N && p.vec32) {
    float v[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[16 * q + i]);
      st_bf16x16(o + 16 * q, v);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i)
      if (col0 + i < p.N) o[i] = f2bf(__uint_as_float(r[i]));
  }
  if (cm == -INFINITY) return;  // no column below N
  float cs[4] = {0.f, 0.f, 0.f, 0.f};
  const float nb = -cm * LOG2E_F;
#pragma unroll
  for (int i = 0; i < 64; ++i)
    if (col0 + i < p.N) cs[i & 3] += ex2_approx(fmaf(__uint_as_float(r[i]), LOG2E_F, nb));
  softmax_stats_merge(m, s, mi, cm, (cs[0] + cs[1]) + (cs[2] + cs[3]), ci);
}

// Fused math on 32 columns whose residual / accumulator (fp32, 4 x 32-byte
// words) or GELU pre-activation (bf16, 2 x 32-byte words) the caller already
// loaded into x: the vectorised epilogue of EPI_RESID_F32, EPI_ACCUM_F32 and
// EPI_DGELU.
__device__ __forceinline__ void epi_store_loaded(const Params& p, int row, int col0, int split,
                                                 const uint32_t (&r)[32], const uint32_t (*x)[8],
                                                 float (&dot)[4]) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  const long base = (long)row * p.ldc + col0;
  if (p.epi == EPI_ROWDOT) {
    // the stored bf16 values, and their products with aux in four chains
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      const float2 a = unpack_bf16x2(w[i]), o = unpack_bf16x2(x[i / 8][i % 8]);
      dot[i & 3] = fmaf(a.x, o.x, fmaf(a.y, o.y, dot[i & 3]));
    }
    bf16* ob = reinterpret_cast<bf16*>(p.out) + base;
    st32(ob, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    st32(ob + 16, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
    return;
  }
  if (p.epi == EPI_DGELU) {
    bf16* o = reinterpret_cast<bf16*>(p.out) + base;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 d = mul2(make_float2(v[16 * hh + 2 * e], v[16 * hh + 2 * e + 1]),
                              gelu_tanh_grad2(unpack_bf16x2(x[hh][e])));
        v[16 * hh + 2 * e] = d.x;
        v[16 * hh + 2 * e + 1] = d.y;
      }
    st_bf16x16(o, v);
    st_bf16x16(o + 16, v + 16);
    return;
  }
  if (p.bias != nullptr && p.epi == EPI_RESID_F32) {
    const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 bb = ldg_keep(b4 + i);
      const float2 lo = add2(make_float2(v[4 * i], v[4 * i + 1]), make_float2(bb.x, bb.y));
      const float2 hi = add2(make_float2(v[4 * i + 2], v[4 * i + 3]), make_float2(bb.z, bb.w));
      v[4 * i] = lo.x;
      v[4 * i + 1] = lo.y;
      v[4 * i + 2] = hi.x;
      v[4 * i + 3] = hi.y;
    }
  }
  float* o = reinterpret_cast<float*>(p.out) + (p.epi == EPI_ACCUM_F32 ? (long)split * p.split_stride : 0) + base;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float2 s =
          add2(make_float2(v[8 * i + e], v[8 * i + e + 1]),
               make_float2(__uint_as_float(x[i][e]), __uint_as_float(x[i][e + 1])));
      v[8 * i + e] = s.x;
      v[8 * i + e + 1] = s.y;
    }
    st_f32x8(o + 8 * i, v + 8 * i);
  }
}

// The epilogue of one accumulator tile for one warp: its TMEM lane quarter
// (rows `row` of the tile, one per lane) and its half of the columns
// [cbase, cbase + BN/2).  wait_acc() waits for the accumulator (false: gave
// up); release() hands the accumulator buffer back to the MMA issuer once the
// warp's last columns are in registers (called by lane 0).  The epilogues that
// read memory (residual, accumulator, GELU pre-activation) issue a chunk's
// loads before they wait for its accumulator columns, the first chunk's even
// before the accumulator is complete.  Returns false when wait_acc gave up.
template <int BN, bool CE, class Wait, class Release>
__device__ __forceinline__ bool epilogue_tile(const Params& p, int row, int nb, int split, uint32_t tbase, int cbase,
                                              int whalf, int lane, Wait wait_acc, Release release) {
  constexpr int CHUNKS = BN / 64 / (EPI_WARPS / 4);  // 64-column chunks per warp
  if constexpr (CE) {
    if (!wait_acc()) return false;
    // logits and their per-(row, half tile) softmax statistics
    float m = -INFINITY, s = 0.f;
    int mi = 0x7fffffff;
#pragma unroll 1
    for (int j = 0; j < CHUNKS; ++j) {
      uint32_t r[64];
      tmem_ld32(tbase + cbase + j * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(tbase + cbase + j * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_wait_ld();
      if (j == CHUNKS - 1) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release();
      }
      const int col0 = nb * BN + cbase + j * 64;
      if (row < p.M && col0 < p.N) epi_ce_chunk(p, row, col0, r, m, s, mi);
    }
    if (row < p.M) {
      float* cp = p.ce_part + ((long)row * p.ce_nh + nb * 2 + whalf) * 3;
      cp[0] = m;
      cp[1] = s;
      cp[2] = __int_as_float(mi);
    }
  } else {
    const bool f32_in = p.epi == EPI_RESID_F32 || p.epi == EPI_ACCUM_F32;
    const bool in_loads = f32_in || p.epi == EPI_DGELU || p.epi == EPI_ROWDOT;
    if (!in_loads && p.vec32) {
      // 16 accumulator columns per TMEM load, each load issued while the
      // previous 16 columns are processed
      constexpr int NP = CHUNKS * 4;
      const int colw = nb * BN + cbase;
      uint32_t pa[16], pb[16];
      if (!wait_acc()) return false;
      tmem_ld16(tbase + cbase, pa);
      tmem_wait_ld();
#pragma unroll 1
      for (int q = 0; q < NP; q += 2) {
        tmem_ld16(tbase + cbase + 16 * (q + 1), pb);
        if (row < p.M && colw + 16 * q < p.N) epi_store16(p, row, colw + 16 * q, split, pa);
        tmem_wait_ld();
        if (q + 2 < NP) {
          tmem_ld16(tbase + cbase + 16 * (q + 2), pa);
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release();
        }
        if (row < p.M && colw + 16 * (q + 1) < p.N) epi_store16(p, row, colw + 16 * (q + 1), split, pb);
        if (q + 2 < NP) tmem_wait_ld();
      }
      return true;
    }
    const bool loads = in_loads && p.vec32 && row < p.M;
    // 64 accumulator columns per TMEM wait; the buffer is handed back to the
    // MMA warp as soon as its last columns are in registers
#pragma unroll 1
    for (int j = 0; j < CHUNKS; ++j) {
      const int col = nb * BN + cbase + j * 64;
      const bool pre = loads && col + 64 <= p.N;
      uint32_t x[8][8];
      if (pre) {
        if (f32_in) {
          const float* src = (p.epi == EPI_RESID_F32
                                  ? p.resid
                                  : reinterpret_cast<const float*>(p.out) + (long)split * p.split_stride) +
                             (long)row * p.ldc + col;
#pragma unroll
          for (int i = 0; i < 8; ++i) ld32(src + 8 * i, x[i]);
        } else {
          const bf16* src = p.aux + (long)row * p.ldc + col;
#pragma unroll
          for (int i = 0; i < 4; ++i) ld32(src + 16 * i, x[i]);
        }
      }
      if (j == 0 && !wait_acc()) return false;
      float dot[4] = {0.f, 0.f, 0.f, 0.f};  // EPI_ROWDOT: the chunk's 64 columns are one group
      // the chunk's two 32-column halves, one TMEM load and wait each
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        tmem_ld32(tbase + cbase + j * 64 + 32 * h, r);
        tmem_wait_ld();
        if (j == CHUNKS - 1 && h == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release();
        }
        const int col0 = col + h * 32;
        if (pre) {
          if (f32_in)
            epi_store_loaded(p, row, col0, split, r, &x[4 * h], dot);
          else
            epi_store_loaded(p, row, col0, split, r, &x[2 * h], dot);
        } else if (row < p.M && col0 < p.N) {
          if (col0 + 32 <= p.N && p.vec32)
            epi_store<true>(p, row, col0, split, r);
          else
            epi_store<false>(p, row, col0, split, r);
        }
      }
      if (p.epi == EPI_ROWDOT && pre) {
        const int T = p.rd_T, H = p.N / 64, nqb = T / 128;
        const int b = row / T, q = row % T, hd = col / 64;
        float* ld = p.rd_out + (((long)b * H + hd) * nqb + q / 128) * 256 + q % 128;
        ld[0] = p.rd_lse[((long)b * H + hd) * T + q] * 1.4426950408889634f;
        ld[128] = (dot[0] + dot[1]) + (dot[2] + dot[3]);
      }
    }
  }
  return true;
}

// --------------------------------------------------------------- kernel
// CE: the softmax-statistics epilogue (EPI_CE_STATS) in its own instantiation,
// so that its registers do not weigh on the other epilogues.
template <int BN, bool CE>
__global__ void __launch_bounds__(THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                   const Params p) {
  using L = Layout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + L::STAGES;
  uint64_t* tfull = empty + L::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_WARPS);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)L::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tma_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tma_b)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
        int mb, nb, split;
        decode_tile(p, tile, mb, nb, split);
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % L::STAGES;
          const uint32_t ph = (it / L::STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) {
            set_device_err(DERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          mbar_expect_tx(&full[s], L::STAGE_BYTES);
          const uint32_t a_dst = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t b_dst = a_dst + L::A_BYTES;
          const int k0 = kb * BK;
          if (!p.a_mn) {
            tma_load_2d(a_dst, &tma_a, k0, mb * BM, &full[s]);
          } else {
            tma_load_2d(a_dst, &tma_a, mb * BM, k0, &full[s]);
            tma_load_2d(a_dst + 8192, &tma_a, mb * BM + 64, k0, &full[s]);
          }
          if (!p.b_mn) {
            tma_load_2d(b_dst, &tma_b, k0, nb * BN, &full[s]);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(b_dst + j * 8192, &tma_b, nb * BN + 64 * j, k0, &full[s]);
          }
        }
      }
      // drain: every issued stage load has landed before the CTA exits
      const uint32_t issued = it;
      for (int s = 0; s < L::STAGES; ++s) {
        if ((uint32_t)s < issued) {
          const uint32_t last = issued - 1 - ((issued - 1 - s) % L::STAGES);
          if (!mbar_wait_drain(&full[s], (last / L::STAGES) & 1u)) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      const uint32_t idesc = make_idesc<BN>(p.a_mn, p.b_mn);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++tc) {
        int mb, nb, split;
        decode_tile(p, tile, mb, nb, split);
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
        const uint32_t buf = tc & 1u;
        if (!mbar_wait(&tempty[buf], ((tc >> 1) & 1u) ^ 1u)) {
          set_device_err(DERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % L::STAGES;
          const uint32_t ph = (it / L::STAGES) & 1u;
          if (!mbar_wait(&full[s], ph)) {
            set_device_err(DERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t b_addr = a_addr + L::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = make_sdesc(a_addr + (p.a_mn ? k * 2048 : k * 32), p.a_mn);
            const uint64_t bd = make_sdesc(b_addr + (p.b_mn ? k * 2048 : k * 32), p.b_mn);
            tc_mma(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&tfull[buf]);
      }
      // drain: all MMAs issued by this thread have completed
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    constexpr int CHUNKS = BN / 64 / (EPI_WARPS / 4);  // 64-column chunks per warp
    const int cbase = ((warp - 2) >> 2) * CHUNKS * 64;  // first column of this warp's half
    uint32_t tc = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++tc) {
      int mb, nb, split;
      decode_tile(p, tile, mb, nb, split);
      const uint32_t buf = tc & 1u;
      const int row = mb * BM + q * 32 + lane;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
      const bool ok = epilogue_tile<BN, CE>(
          p, row, nb, split, tbase, cbase, (warp - 2) >> 2, lane,
          [&] {
            const bool got = mbar_wait(&tfull[buf], (tc >> 1) & 1u);
            tc_fence_after();
            return got;
          },
          [&] { mbar_arrive(&tempty[buf]); });
      if (!ok) {
        set_device_err(DERR_WAIT_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)L::TMEM_COLS)
                 : "memory");
  }
}


// ------------------------------------------------------ 2-SM kernel
// A cluster of two CTAs (one per SM) computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256): CTA r of the pair loads rows
// [r*128, r*128+128) of the tile's A block and rows [r*128, r*128+128) of its
// B block (the N half) into the same shared-memory offsets, the leader CTA's
// MMA thread issues the MMAs for both, and each CTA's TMEM receives its 128
// rows x 256 columns of the accumulator.  Per SM this halves the shared-memory
// traffic of the B operand against the 1-SM 128 x 256 tile.
// Barriers: the leader's full[s] counts the bytes of both CTAs' loads (the
// peer's TMA loads signal it across the pair); the MMA commits release empty[s]
// and signal tfull[buf] in both CTAs; both CTAs' epilogue warps arrive on the
// leader's tempty[buf].
struct Layout2 {
  static constexpr int STAGES = 6;
  static constexpr int A_BYTES = BM * BK * 2;   // this CTA's 128 rows of A
  static constexpr int B_BYTES = 128 * BK * 2;  // this CTA's 128 rows (N half) of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 512;         // two 256-column accumulators
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t mapa_rank(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory that completes on an mbarrier of
// either CTA of the pair (bar: shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
// arrive once on the barrier at this offset in both CTAs of the pair when the
// MMAs issued so far are complete
__device__ __forceinline__ void tc_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// (CTA-scope release: what the MMA issuer needs ordered before it reuses the
// accumulator are the warp's TMEM loads, which tcgen05.wait::ld and
// tcgen05.fence::before_thread_sync already order; a cluster-scope release
// would also wait for the warp's global stores to be acknowledged)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <bool CE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    tc_gemm2_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                    const Params p) {
  using L = Layout2;
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + L::STAGES;
  uint64_t* tfull = empty + L::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * EPI_WARPS);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)L::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the pair's barriers are initialised before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tma_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tma_b)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < p.total_tiles; tile += ncl) {
        int mb, nb, split;
        decode_tile(p, tile, mb, nb, split);
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
        const int m0 = mb * 256 + (int)rank * 128, n0 = nb * 256 + (int)rank * 128;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % L::STAGES;
          const uint32_t ph = (it / L::STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) {
            set_device_err(DERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          if (rank == 0) mbar_expect_tx(&full[s], 2 * L::STAGE_BYTES);
          const uint32_t bar = mapa_rank(smem_u32(&full[s]), 0);
          const uint32_t a_dst = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t b_dst = a_dst + L::A_BYTES;
          const int k0 = kb * BK;
          if (!p.a_mn) {
            tma_load_2d_pair(a_dst, &tma_a, k0, m0, bar);
          } else {
            tma_load_2d_pair(a_dst, &tma_a, m0, k0, bar);
            tma_load_2d_pair(a_dst + 8192, &tma_a, m0 + 64, k0, bar);
          }
          if (!p.b_mn) {
            tma_load_2d_pair(b_dst, &tma_b, k0, n0, bar);
          } else {
            tma_load_2d_pair(b_dst, &tma_b, n0, k0, bar);
            tma_load_2d_pair(b_dst + 8192, &tma_b, n0 + 64, k0, bar);
          }
        }
      }
      // drain: every stage this CTA loaded has been consumed by the pair's
      // MMAs (so its copies have landed) before the CTA goes on to exit
      const uint32_t issued = it;
      for (int s = 0; s < L::STAGES; ++s) {
        if ((uint32_t)s < issued) {
          const uint32_t last = issued - 1 - ((issued - 1 - s) % L::STAGES);
          if (!mbar_wait_drain(&empty[s], ((last / L::STAGES) & 1u))) set_device_err(DERR_WAIT_TIMEOUT);
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      // -------------------------------------------- MMA issuer (leader CTA)
      // kind::f16, bf16 x bf16 -> fp32, M = 256 (the pair), N = 256
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)p.a_mn << 15) |
                             ((uint32_t)p.b_mn << 16) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < p.total_tiles; tile += ncl, ++tc) {
        int mb, nb, split;
        decode_tile(p, tile, mb, nb, split);
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
        const uint32_t buf = tc & 1u;
        if (!mbar_wait(&tempty[buf], ((tc >> 1) & 1u) ^ 1u)) {
          set_device_err(DERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % L::STAGES;
          const uint32_t ph = (it / L::STAGES) & 1u;
          if (!mbar_wait(&full[s], ph)) {
            set_device_err(DERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t b_addr = a_addr + L::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = make_sdesc(a_addr + (p.a_mn ? k * 2048 : k * 32), p.a_mn);
            const uint64_t bd = make_sdesc(b_addr + (p.b_mn ? k * 2048 : k * 32), p.b_mn);
            tc_mma_pair(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit_pair_both(&empty[s]);
        }
        if (!ok) break;
        tc_commit_pair_both(&tfull[buf]);
      }
      // drain: all MMAs issued by this thread have completed
      tc_commit_pair_local(drain);
      if (!mbar_wait_drain(drain, 0)) set_device_err(DERR_WAIT_TIMEOUT);
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;
    constexpr int CHUNKS = BN / 64 / (EPI_WARPS / 4);
    const int cbase = ((warp - 2) >> 2) * CHUNKS * 64;
    uint32_t tc = 0;
    for (int tile = cid; tile < p.total_tiles; tile += ncl, ++tc) {
      int mb, nb, split;
      decode_tile(p, tile, mb, nb, split);
      const uint32_t buf = tc & 1u;
      const int row = mb * 256 + (int)rank * 128 + q * 32 + lane;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
      const uint32_t tempty_leader = mapa_rank(smem_u32(&tempty[buf]), 0);
      const bool ok = epilogue_tile<BN, CE>(
          p, row, nb, split, tbase, cbase, (warp - 2) >> 2, lane,
          [&] {
            const bool got = mbar_wait(&tfull[buf], (tc >> 1) & 1u);
            tc_fence_after();
            return got;
          },
          [&] { mbar_arrive_cluster(tempty_leader); });
      if (!ok) {
        set_device_err(DERR_WAIT_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while its pair may still use its shared memory or TMEM
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)L::TMEM_COLS)
                 : "memory");
  }
}

// Deterministic split-K reduction: out[i] += sum_s partial[s][i] (fixed order).
__global__ void splitk_reduce_kernel(float* __restrict__ out, const float* __restrict__ partial, long n4, long stride,
                                     int splits) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(out)[i];
    for (int s = 0; s < splits; ++s) {
      float4 v = reinterpret_cast<const float4*>(partial + s * stride)[i];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    reinterpret_cast<float4*>(out)[i] = acc;
  }
}

// ------------------------------------------------------------------ host
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2-D bf16 tensor map: `inner` contiguous elements per row, `outer` rows,
// rows `ld` elements apart; box box_inner x box_outer; 128-byte swizzle.
static int make_tmap(CUtensorMap* m, const void* base, long inner, long outer, long ld, int box_inner,
                     int box_outer) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return -1;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

static int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int BN, bool CE>
static cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& tb, const Params& p, int grid, cudaStream_t st) {
  using L = Layout<BN>;
  static DeviceOnce once;
  cudaError_t e = run_once_per_device(once, [] {
    return cudaFuncSetAttribute(tc_gemm_kernel<BN, CE>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  tc_gemm_kernel<BN, CE><<<grid, THREADS, L::SMEM_BYTES, st>>>(ta, tb, p);
  return cudaGetLastError();
}

template <bool CE>
static cudaError_t launch2(const CUtensorMap& ta, const CUtensorMap& tb, const Params& p, int grid, cudaStream_t st) {
  static DeviceOnce once;
  cudaError_t e = run_once_per_device(once, [] {
    return cudaFuncSetAttribute(tc_gemm2_kernel<CE>, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout2::SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  tc_gemm2_kernel<CE><<<grid, THREADS, Layout2::SMEM_BYTES, st>>>(ta, tb, p);
  return cudaGetLastError();
}

// Which kernel serves a shape: the 2-SM pair kernel for N > 128 with more
// than 128 rows, unless GPT2_GEMM_2SM=0 is set in the environment (then the
// 1-SM kernel serves every shape; read at each call, for comparisons).
static bool use_pair_kernel(int M, int N, int bn) {
  const char* e = getenv("GPT2_GEMM_2SM");
  const bool pair = !(e != nullptr && e[0] == '0');
  return pair && bn == 256 && M > BM && N > 128;
}

int choose_splits(int tiles, int kb_total, int units) {
  const int sms = units;
  if (tiles >= sms) return 1;
  int best = 1;
  double best_eff = (double)tiles / (double)(((tiles + sms - 1) / sms) * sms);
  for (int s = 2; s <= 16; ++s) {
    if (kb_total / s < 4) break;
    const int t = tiles * s;
    const double eff = (double)t / (double)(((t + sms - 1) / sms) * sms);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

int accum_slot_splits(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 1;
  const int bn = (N <= 128) ? 128 : 256;
  const bool pair = use_pair_kernel(M, N, bn);
  const int tiles = pair ? ceil_div(M, 256) * ceil_div(N, 256) : ceil_div(M, BM) * ceil_div(N, bn);
  const int kbt = ceil_div(K, BK);
  const int s = choose_splits(tiles, kbt, pair ? num_sms() / 2 : num_sms());
  return ceil_div(kbt, ceil_div(kbt, s));
}

size_t splitk_workspace_bytes(int M, int N, int K, int bn) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  if (bn != 128) bn = (N <= 128) ? 128 : 256;
  const bool pair = use_pair_kernel(M, N, bn);
  const int tiles = pair ? ceil_div(M, 256) * ceil_div(N, 256) : ceil_div(M, BM) * ceil_div(N, bn);
  const int kbt = ceil_div(K, BK);
  const int s = choose_splits(tiles, kbt, pair ? num_sms() / 2 : num_sms());
  return s > 1 ? (size_t)s * M * N * sizeof(float) : 0;
}

int gemm(const GemmArgs& g, cudaStream_t st) {
  // shape / layout checks (TMA needs 16-byte row strides and base addresses)
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return -1;
  if ((g.lda % 8) || (g.ldb % 8) || (g.ldc % 8)) return -1;
  if ((reinterpret_cast<uintptr_t>(g.A) & 15) || (reinterpret_cast<uintptr_t>(g.B) & 15) ||
      (reinterpret_cast<uintptr_t>(g.out) & 15))
    return -1;
  const int bn = (g.bn == 128 || g.N <= 128) ? 128 : 256;
  const bool pair = use_pair_kernel(g.M, g.N, bn);
  CUtensorMap ta, tb;
  if (!g.a_mn) {
    if (make_tmap(&ta, g.A, g.K, g.M, g.lda, 64, BM)) return -2;
  } else {
    if (make_tmap(&ta, g.A, g.M, g.K, g.lda, 64, 64)) return -2;
  }
  if (!g.b_mn) {
    if (make_tmap(&tb, g.B, g.K, g.N, g.ldb, 64, pair ? 128 : bn)) return -2;
  } else {
    if (make_tmap(&tb, g.B, g.N, g.K, g.ldb, 64, 64)) return -2;
  }
  Params p{};
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.a_mn = g.a_mn;
  p.b_mn = g.b_mn;
  p.num_m = pair ? ceil_div(g.M, 256) : ceil_div(g.M, BM);
  p.num_n = ceil_div(g.N, bn);
  p.kb_total = ceil_div(g.K, BK);
  p.epi = g.epi;
  p.bias = g.bias;
  p.resid = g.resid;
  p.out = g.out;
  p.out2 = g.out2;
  p.aux = g.aux;
  p.ldc = g.ldc;
  p.ce_part = g.ce_part;
  p.ce_nh = ce_halves(g.N);
  p.rd_out = g.rd_out;
  p.rd_lse = g.rd_lse;
  p.rd_T = g.rd_T;
  if (g.epi == EPI_ROWDOT && (g.rd_out == nullptr || g.rd_lse == nullptr || g.aux == nullptr || g.rd_T <= 0 ||
                              g.rd_T % 128 != 0 || g.N % 64 != 0 || g.M % g.rd_T != 0 || g.ldc != g.N || g.bias))
    return -1;
  if (g.epi == EPI_CE_STATS && (g.ce_part == nullptr || bn != 256)) return -1;
  {
    // 32-byte vector epilogue: every 32-column chunk of every row (and of the
    // residual / aux / split-K partial buffers) must start on 32 bytes
    const size_t es =
        (g.epi == EPI_BF16 || g.epi == EPI_GELU || g.epi == EPI_DGELU || g.epi == EPI_CE_STATS || g.epi == EPI_ROWDOT)
            ? 2
            : 4;
    auto al32 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 31) == 0; };
    bool ok = (g.ldc * (long)es) % 32 == 0 && al32(g.out);
    if (g.epi == EPI_RESID_F32) ok = ok && al32(g.resid);
    if (g.epi == EPI_GELU) ok = ok && al32(g.out2);
    if (g.epi == EPI_DGELU || g.epi == EPI_ROWDOT) ok = ok && al32(g.aux);
    if (g.workspace) ok = ok && al32(g.workspace) && (g.ldc * 4L) % 32 == 0;
    p.vec32 = ok ? 1 : 0;
    if (g.epi == EPI_ROWDOT && !ok) return -1;  // its row dots are formed on the vector path only
  }
  const int units = pair ? num_sms() / 2 : num_sms();
  int splits = 1;       // K splits
  bool reduce = false;  // split-K partials in g.workspace, summed into out by a reduction kernel
  if (g.epi == EPI_ACCUM_F32 && g.slots != nullptr) {
    // persistent per-split accumulators: no scratch, no reduction
    if (g.ldc != g.N || (reinterpret_cast<uintptr_t>(g.slots) & 15)) return -1;
    splits = choose_splits(p.num_m * p.num_n, p.kb_total, units);
    if (splits > g.slot_splits) splits = g.slot_splits;
    if (splits < 1) splits = 1;
    p.out = g.slots;
    p.split_stride = (long)g.M * g.ldc;
    p.vec32 = p.vec32 && (reinterpret_cast<uintptr_t>(g.slots) & 31) == 0;
  } else if (g.epi == EPI_ACCUM_F32 && g.workspace != nullptr && g.ldc == g.N) {
    splits = choose_splits(p.num_m * p.num_n, p.kb_total, units);
    if (splits > 1 && g.workspace_bytes < (size_t)splits * g.M * g.ldc * sizeof(float)) splits = 1;
    reduce = splits > 1;
  }
  {
    // every split gets at least one k-block
    const int kps = ceil_div(p.kb_total, splits);
    p.splits = ceil_div(p.kb_total, kps);
    p.kb_per_split = kps;
  }
  if (reduce) {
    p.epi = EPI_PARTIAL_F32;
    p.partial = g.workspace;
  }
  p.total_tiles = p.num_m * p.num_n * p.splits;
  cudaError_t e;
  if (pair) {
    // one cluster of two CTAs per pair of SMs, persistent over the tiles
    const int pairs = p.total_tiles < num_sms() / 2 ? p.total_tiles : num_sms() / 2;
    e = p.epi == EPI_CE_STATS ? launch2<true>(ta, tb, p, 2 * pairs, st) : launch2<false>(ta, tb, p, 2 * pairs, st);
  } else {
    const int grid = p.total_tiles < num_sms() ? p.total_tiles : num_sms();
    e = p.epi == EPI_CE_STATS ? launch<256, true>(ta, tb, p, grid, st)
        : (bn == 128)         ? launch<128, false>(ta, tb, p, grid, st)
                              : launch<256, false>(ta, tb, p, grid, st);
  }
  if (e != cudaSuccess) return -3;
  if (reduce) {
    const long n = (long)g.M * g.N;
    const long n4 = n / 4;
    int blocks = (int)((n4 + 255) / 256);
    if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
    splitk_reduce_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<float*>(g.out), g.workspace, n4, n, p.splits);
    if (cudaGetLastError() != cudaSuccess) return -3;
  }
  return 0;
}

}  // namespace tcg
