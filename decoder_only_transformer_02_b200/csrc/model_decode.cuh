// Generation: the forward pass one token at a time with a KV cache, and an
// on-device top-k sampler ("Let's reproduce GPT-2 (124M)", Chapters:
// sampling init, prefix tokens; sampling loop).
//
// A prefill runs the training forward on the prefix [B, T0] and copies every
// layer's keys and values into the cache; each decode step then takes one new
// token per sequence at the next position, computes its 12 layers with M = B
// rows (the tcgen05 GEMMs, a one-query attention over the cached keys), the
// lm_head logits [B, Vp] and the next token.  bf16 mode only.
//
// Sampling rule (the pages name a sampling loop but no rule): top-k sampling
// from softmax(logits / temperature) over the k largest logits of the real
// vocabulary [0, V), ties at the k-th place to the lower id; k = 1 or
// temperature 0 is the greedy argmax.  The uniform u of row b for the token at
// position p is the top 53 bits of splitmix64(seed * 2^32 + p * 2^16 + b)
// (Steele, Lea and Flood's generator), so a CPU restatement draws the same u.
#pragma once
#include "model_pass.cuh"

namespace gen {

constexpr int SAMPLE_THREADS = 1024;
constexpr int MAX_TOP_K = 64;

// x[b] = wte[tok[b]] + wpe[pos] (fp32); ids outside [0, Vp) flag the error
// word and embed as wpe only
__global__ void embed_kernel(const int32_t* __restrict__ tok, const float* __restrict__ wte,
                             const float* __restrict__ wpe, float* __restrict__ x, int B, int C, int Vp, int pos,
                             int* __restrict__ bad) {
  const int c4 = C / 4;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B * c4; i += gridDim.x * blockDim.x) {
    const int b = i / c4, c = i % c4;
    const int id = tok[b];
    float4 p = reinterpret_cast<const float4*>(wpe + (long)pos * C)[c];
    if (id >= 0 && id < Vp) {
      const float4 w = reinterpret_cast<const float4*>(wte + (long)id * C)[c];
      p.x += w.x;
      p.y += w.y;
      p.z += w.z;
      p.w += w.w;
    } else if (c == 0) {
      atomicExch(bad, 1);
    }
    reinterpret_cast<float4*>(x + (long)b * C)[c] = p;
  }
}

// kv[b][t][0:C] = k, kv[b][t][C:2C] = v of rows b*T0 + t of one layer's qkv
// [B*T0, 3C] (t < T0), 16 bytes per thread
__global__ void fill_cache_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ kv, int B, int T0, int C,
                                  int P) {
  const int c8 = 2 * C / 8;  // 16-byte chunks of k and v
  const long n = (long)B * T0 * c8;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const long r = i / c8;
    const int c = (int)(i % c8);
    const int b = (int)(r / T0), t = (int)(r % T0);
    const uint4 v = reinterpret_cast<const uint4*>(qkv + r * 3L * C + C)[c];
    reinterpret_cast<uint4*>(kv + ((long)b * P + t) * 2L * C)[c] = v;
  }
}

// One query per (sequence, head) against the cached keys 0..pos: stores the
// new key and value at pos, then o = softmax(q k^T / sqrt(d)) v with the
// scores in shared memory and fixed-order reductions.  qkv [B, 3C], kv layer
// base [max_B][P][2C], out [B, C].  Dynamic shared memory: (pos+1) floats.
__global__ void __launch_bounds__(256) attn_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ kv,
                                                   bf16* __restrict__ out, int H, int P, int pos, float sl2) {
  extern __shared__ float sc[];
  __shared__ float qs[64];
  __shared__ float red[256];
  const int b = blockIdx.x / H, h = blockIdx.x % H;
  const int C = H * 64;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bf16* row = qkv + (long)b * 3 * C;
  bf16* cache = kv + (long)b * P * 2 * C;
  if (tid < 16) {
    // the new key (threads 0-7) and value (8-15) at position pos
    const int part = tid >> 3, c = tid & 7;
    reinterpret_cast<uint4*>(cache + (long)pos * 2 * C + part * C + h * 64)[c] =
        reinterpret_cast<const uint4*>(row + (1 + part) * C + h * 64)[c];
  }
  if (tid < 64) qs[tid] = bf2f(row[h * 64 + tid]);
  __syncthreads();
  // scores in log2 units
  float mx = -INFINITY;
  for (int t = tid; t <= pos; t += 256) {
    const uint4* kr = reinterpret_cast<const uint4*>(cache + (long)t * 2 * C + h * 64);
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 u = kr[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16x2(w[e]);
        s = fmaf(qs[8 * c + 2 * e], f.x, fmaf(qs[8 * c + 2 * e + 1], f.y, s));
      }
    }
    s *= sl2;
    sc[t] = s;
    mx = fmaxf(mx, s);
  }
  red[tid] = mx;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (tid < o) red[tid] = fmaxf(red[tid], red[tid + o]);
    __syncthreads();
  }
  mx = red[0];
  __syncthreads();
  float sum = 0.f;
  for (int t = tid; t <= pos; t += 256) {
    const float e = exp2f(sc[t] - mx);
    sc[t] = e;
    sum += e;
  }
  red[tid] = sum;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (tid < o) red[tid] += red[tid + o];
    __syncthreads();
  }
  const float inv = 1.f / red[0];
  __syncthreads();
  // o[d] = sum_t p_t v_t[d]: thread (slice, d) takes the keys t = slice mod 4
  const int d = tid & 63, sl = tid >> 6;
  float acc = 0.f;
  for (int t = sl; t <= pos; t += 4) acc = fmaf(sc[t], bf2f(cache[(long)t * 2 * C + C + h * 64 + d]), acc);
  red[tid] = acc;
  __syncthreads();
  if (tid < 64) {
    const float o = ((red[d] + red[64 + d]) + red[128 + d]) + red[192 + d];
    out[(long)b * C + h * 64 + d] = f2bf(o * inv);
  }
  (void)lane;
  (void)warp;
}

__device__ __forceinline__ uint64_t sm64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

// (v, i) precedes (w, j) in the sampler's order: larger logit first, lower id on ties
__device__ __forceinline__ bool before(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

// One CTA per sequence: the next token from its logits row z (bf16 [Vp],
// row stride ld) over ids [0, V).  k rounds each find the next element in
// (logit desc, id asc) order; p_i = exp((z_i - z_top) / temperature) in
// double, inverse CDF at u.  top_k <= 1 or temperature <= 0: argmax.
__global__ void __launch_bounds__(SAMPLE_THREADS) sample_kernel(const bf16* __restrict__ z, long ld, int V,
                                                               float temperature, int top_k, uint64_t seed,
                                                               int pos_next, int32_t* __restrict__ next) {
  __shared__ float bv[SAMPLE_THREADS / 32];
  __shared__ int bi[SAMPLE_THREADS / 32];
  __shared__ float top_v[MAX_TOP_K];
  __shared__ int top_i[MAX_TOP_K];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bf16* zr = z + (long)b * ld;
  const int k = (top_k <= 1 || temperature <= 0.f) ? 1 : min(top_k, min(V, MAX_TOP_K));
  float pv = INFINITY;  // previous selection (the order starts above every logit)
  int pi = -1;
  for (int r = 0; r < k; ++r) {
    float v = -INFINITY;
    int i = 0x7fffffff;
    for (int j = tid; j < V; j += SAMPLE_THREADS) {
      const float x = bf2f(zr[j]);
      if (before(pv, pi, x, j) && before(x, j, v, i)) {
        v = x;
        i = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, v, o);
      const int oi = __shfl_xor_sync(0xffffffffu, i, o);
      if (before(ov, oi, v, i)) {
        v = ov;
        i = oi;
      }
    }
    if (lane == 0) {
      bv[warp] = v;
      bi[warp] = i;
    }
    __syncthreads();
    v = bv[0];
    i = bi[0];
    for (int w = 1; w < SAMPLE_THREADS / 32; ++w)
      if (before(bv[w], bi[w], v, i)) {
        v = bv[w];
        i = bi[w];
      }
    if (tid == 0) {
      top_v[r] = v;
      top_i[r] = i;
    }
    pv = v;
    pi = i;
    __syncthreads();
  }
  if (tid == 0) {
    int pick = top_i[0];
    if (k > 1) {
      double p[MAX_TOP_K], tot = 0.0;
      for (int r = 0; r < k; ++r) {
        p[r] = exp(((double)top_v[r] - (double)top_v[0]) / (double)temperature);
        tot += p[r];
      }
      const uint64_t key = ((seed & 0xFFFFFFFFull) << 32) | ((uint64_t)(pos_next & 0xFFFF) << 16) | (uint64_t)(b & 0xFFFF);
      const double u = (double)(sm64(key) >> 11) * (1.0 / 9007199254740992.0);
      double c = 0.0;
      pick = top_i[k - 1];
      for (int r = 0; r < k; ++r) {
        c += p[r];
        if (c / tot > u) {
          pick = top_i[r];
          break;
        }
      }
    }
    next[b] = pick;
  }
}

}  // namespace gen

static int gen_alloc(gpt2* h) {
  if (h->kv != nullptr) return GPT2_OK;
  const long mb = h->maxB, C = h->C;
  ALLOC(h, h->kv, (size_t)h->L * mb * h->P * 2 * C * 2);
  ALLOC(h, h->dec_x, (size_t)mb * C * 4);
  ALLOC(h, h->dec_mean, (size_t)mb * 4);
  ALLOC(h, h->dec_rstd, (size_t)mb * 4);
  ALLOC(h, h->dec_ln, (size_t)mb * C * 2);
  ALLOC(h, h->dec_qkv, (size_t)mb * 3 * C * 2);
  ALLOC(h, h->dec_att, (size_t)mb * C * 2);
  ALLOC(h, h->dec_u, (size_t)mb * 4 * C * 2);
  ALLOC(h, h->dec_a, (size_t)mb * 4 * C * 2);
  ALLOC(h, h->dec_logits, (size_t)mb * h->Vp * 2);
  return GPT2_OK;
}

static int gen_check(gpt2* h, float temperature, int top_k, int32_t* d_next) {
  if (h->prec != GPT2_BF16) return set_err(h, GPT2_EINVAL, "generation needs bf16 mode");
  if (d_next == nullptr) return set_err(h, GPT2_EINVAL, "next-token pointer is NULL");
  if (top_k < 1 || top_k > gen::MAX_TOP_K || !(temperature >= 0.f))
    return set_err(h, GPT2_EINVAL, "top_k must lie in [1, 64] and temperature must be >= 0");
  return gen_alloc(h);
}

static int gen_sample(gpt2* h, const bf16* rows, long ld, int B, float temperature, int top_k, uint64_t seed,
                      int pos_next, int32_t* d_next) {
  gen::sample_kernel<<<B, gen::SAMPLE_THREADS, 0, h->stream>>>(rows, ld, h->V, temperature, top_k, seed, pos_next,
                                                              d_next);
  LAUNCH_CHECK(h);
  return GPT2_OK;
}

// Prefill: the training forward on [B, T0] (logits only), every layer's keys
// and values into the cache, the last position's logits kept and sampled.
static int prefill_impl(gpt2* h, const int32_t* tok, int B, int T0, float temperature, int top_k, uint64_t seed,
                        int32_t* d_next) {
  RET_IF(gen_check(h, temperature, top_k, d_next));
  if (T0 > h->P) return set_err(h, GPT2_EINVAL, "prefix longer than block_size");
  RET_IF(forward_impl(h, tok, nullptr, B, T0, false, 1.f));
  const int C = h->C;
  Views w{h};
  for (int l = 0; l < h->L; ++l) {
    const long n = (long)B * T0 * (2 * C / 8);
    gen::fill_cache_kernel<<<grid_for(n, 256), 256, 0, h->stream>>>(
        (const bf16*)w.qkv(l), h->kv + (size_t)l * h->maxB * h->P * 2 * C, B, T0, C, h->P);
    LAUNCH_CHECK(h);
  }
  // the last position's logits of every sequence: rows b*T0 + T0-1
  CU_CHECK(h, cudaMemcpy2DAsync(h->dec_logits, (size_t)h->Vp * 2, (const bf16*)h->logits + (size_t)(T0 - 1) * h->Vp,
                                (size_t)T0 * h->Vp * 2, (size_t)h->Vp * 2, B, cudaMemcpyDeviceToDevice, h->stream));
  RET_IF(gen_sample(h, h->dec_logits, h->Vp, B, temperature, top_k, seed, T0, d_next));
  h->gen_B = B;
  h->gen_len = T0;
  return GPT2_OK;
}

// One decode step: tokens [B] at position pos (= the number of positions the
// cache holds), all layers with M = B, logits [B, Vp], the next token.
static int decode_impl(gpt2* h, const int32_t* tok, int B, int pos, float temperature, int top_k, uint64_t seed,
                       int32_t* d_next) {
  RET_IF(gen_check(h, temperature, top_k, d_next));
  if (tok == nullptr) return set_err(h, GPT2_EINVAL, "tokens pointer is NULL");
  if (B != h->gen_B || B < 1) return set_err(h, GPT2_ESTATE, "decode needs a prefill with the same batch first");
  if (pos != h->gen_len) return set_err(h, GPT2_ESTATE, "decode position must follow the cached positions");
  if (pos >= h->P) return set_err(h, GPT2_EINVAL, "position reaches block_size");
  const int C = h->C, L = h->L;
  {
    KTimer kt(h, KC_EMB, 0.0, 8.0 * B * C);
    gen::embed_kernel<<<grid_for((long)B * C / 4, 256), 256, 0, h->stream>>>(tok, h->P32(h->wte), h->P32(h->wpe),
                                                                             h->dec_x, B, C, h->Vp, pos, h->d_bad);
    LAUNCH_CHECK(h);
  }
  const float sl2 = 1.4426950408889634f / sqrtf((float)(C / h->H));
  for (int l = 0; l < L; ++l) {
    const LayerOffsets& o = h->lo[l];
    RET_IF(op_ln_fwd(h, h->dec_x, o.ln1g, o.ln1b, h->dec_ln, h->dec_mean, h->dec_rstd, B));
    RET_IF(op_lin_fwd(h, h->dec_ln, B, C, o.attnw, 3 * C, o.attnb, LIN_PLAIN, h->dec_qkv, nullptr, nullptr));
    {
      KTimer kt(h, KC_ATTN_F, 4.0 * B * (pos + 1.0) * C, 0.0);
      gen::attn_kernel<<<B * h->H, 256, (size_t)(pos + 1) * 4, h->stream>>>(
          h->dec_qkv, h->kv + (size_t)l * h->maxB * h->P * 2 * C, h->dec_att, h->H, h->P, pos, sl2);
      LAUNCH_CHECK(h);
    }
    RET_IF(op_lin_fwd(h, h->dec_att, B, C, o.projw, C, o.projb, LIN_RESID, h->dec_x, nullptr, h->dec_x));
    RET_IF(op_ln_fwd(h, h->dec_x, o.ln2g, o.ln2b, h->dec_ln, h->dec_mean, h->dec_rstd, B));
    RET_IF(op_lin_fwd(h, h->dec_ln, B, C, o.fcw, 4 * C, o.fcb, LIN_GELU, h->dec_u, h->dec_a, nullptr));
    RET_IF(op_lin_fwd(h, h->dec_a, B, 4 * C, o.mpw, C, o.mpb, LIN_RESID, h->dec_x, nullptr, h->dec_x));
  }
  RET_IF(op_ln_fwd(h, h->dec_x, h->lnfg, h->lnfb, h->dec_ln, h->dec_mean, h->dec_rstd, B));
  RET_IF(op_lin_fwd(h, h->dec_ln, B, C, h->wte, h->Vp, NO_OFF, LIN_NOBIAS, h->dec_logits, nullptr, nullptr));
  RET_IF(gen_sample(h, h->dec_logits, h->Vp, B, temperature, top_k, seed, pos + 1, d_next));
  h->gen_len = pos + 1;
  return GPT2_OK;
}
