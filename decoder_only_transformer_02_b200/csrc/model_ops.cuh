// Building-block launches of the GPT-2 step, one helper per operation, in both
// precisions (bf16 tensor-core path and fp32 CUDA-core parity path).
#pragma once
#include "model_core.cuh"


// ----------------------------------------------------------------- LayerNorm
template <typename TO>
static int ln_fwd_dispatch(gpt2* h, const float* x, const float* g, const float* b, TO* y, float* mean, float* rstd,
                           long M) {
  // a warp per row, looping over rows with a stride of the grid's warps: at
  // most two 8-warp CTAs per SM (what the kernel's registers allow)
  int blocks = (int)((M * 32 + 255) / 256);
  if (blocks > 2 * tcg::num_sms()) blocks = 2 * tcg::num_sms();
  switch (h->C / 128) {
#define LNF(NV) \
  case NV:      \
    k::ln_fwd_kernel<NV, TO><<<blocks, 256, 0, h->stream>>>(x, g, b, y, mean, rstd, (int)M); break;
    LNF(1) LNF(2) LNF(3) LNF(4) LNF(5) LNF(6) LNF(7) LNF(8)
#undef LNF
    default:
      return set_err(h, GPT2_EINVAL, "n_embd must be a multiple of 128 up to 1024");
  }
  LAUNCH_CHECK(h);
  return GPT2_OK;
}

static int op_ln_fwd(gpt2* h, const float* x, size_t goff, size_t boff, void* y, float* mean, float* rstd, long M) {
  KTimer kt(h, KC_LN_F, 0.0, (double)M * h->C * (4 + h->es) + 8.0 * M);
  if (h->prec == GPT2_BF16)
    return ln_fwd_dispatch<bf16>(h, x, h->P32(goff), h->P32(boff), (bf16*)y, mean, rstd, M);
  return ln_fwd_dispatch<float>(h, x, h->P32(goff), h->P32(boff), (float*)y, mean, rstd, M);
}

// the LayerNorm backward's dynamic shared memory limit (set once per device
// to the most a CTA may have)
constexpr size_t LN_BWD_SMEM_MAX = 227 * 1024;
template <int NV>
static bool ln_bwd_attr() {
  static DeviceOnce once;
  return run_once_per_device(once, [] {
           return cudaFuncSetAttribute(k::ln_bwd_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)LN_BWD_SMEM_MAX);
         }) == cudaSuccess;
}

// LayerNorm backward into the running residual gradient h->dres.  dy is fp32
// [M, C].  Its partial column sums (dgamma, dbeta and the bias gradient of the
// projection feeding this residual point) add into h->psums[inst].
static int op_ln_bwd(gpt2* h, const float* dy, const float* x, const float* mean, const float* rstd, size_t goff,
                     int inst, long M, int accumulate) {
  KTimer kt(h, KC_LN_B, 0.0, (double)M * h->C * (12 + (accumulate ? 4 : 0) + (h->prec == GPT2_BF16 ? 2 : 0)) + 8.0 * M);
  const int rpb = ln_rows_per_block(M);
  const int nblk = (int)((M + rpb - 1) / rpb);
  bf16* dbf = h->prec == GPT2_BF16 ? h->dres_bf : nullptr;
  float* part = h->psums[inst].buf;
  switch (h->C / 128) {
#define LNB(NV)                                                                                                     \
  case NV:                                                                                                          \
    if (k::LnBwd<NV>::smem_bytes(rpb) > LN_BWD_SMEM_MAX) return set_err(h, GPT2_EINVAL, "layernorm: rows");     \
    if (!ln_bwd_attr<NV>()) return set_err(h, GPT2_ECUDA, "layernorm backward shared memory");                  \
    k::ln_bwd_kernel<NV><<<nblk, (k::LN_BWD_WARPS + 1) * 32, k::LnBwd<NV>::smem_bytes(rpb), h->stream>>>(       \
        dy, x, mean, rstd, h->P32(goff), h->dres, dbf, (int)M, rpb, accumulate, part);                              \
    break;
    LNB(1) LNB(2) LNB(3) LNB(4) LNB(5) LNB(6) LNB(7) LNB(8)
#undef LNB
    default:
      return set_err(h, GPT2_EINVAL, "n_embd must be a multiple of 128 up to 1024");
  }
  LAUNCH_CHECK(h);
  h->accum_dirty = true;
  return GPT2_OK;
}

// ------------------------------------------------------------------ linear
enum LinKind { LIN_PLAIN, LIN_RESID, LIN_GELU, LIN_NOBIAS };

static int tc_call(gpt2* h, tcg::GemmArgs& g) {
  const int r = tcg::gemm(g, h->stream);
  if (r == -1) return set_err(h, GPT2_EINVAL, "matmul: bad shape / stride / alignment");
  if (r != 0) return set_err(h, GPT2_ECUDA, "matmul: tensor map or launch failure");
  h->launches += 1;
  return GPT2_OK;
}
static int simt_call(gpt2* h, const simt::Args& a) {
  if (simt::gemm(a, h->stream) != cudaSuccess) return set_err(h, GPT2_ECUDA, "simt matmul launch failure");
  h->launches++;
  return GPT2_OK;
}

// out[M,N] = X[M,K] W[N,K]^T (+ b): W at param offset woff, b at boff
static int op_lin_fwd(gpt2* h, const void* X, long M, int K, size_t woff, int N, size_t boff, LinKind kind, void* out,
                      void* out2, const float* resid) {
  KTimer kt(h, KC_GEMM, 2.0 * M * N * K, 0.0);
  const float* bias = boff == NO_OFF ? nullptr : h->P32(boff);
  if (h->prec == GPT2_BF16) {
    tcg::GemmArgs g;
    g.A = (const bf16*)X;
    g.lda = K;
    g.a_mn = 0;
    g.B = h->PBF(woff);
    g.ldb = K;
    g.b_mn = 0;
    g.M = (int)M;
    g.N = N;
    g.K = K;
    g.bias = bias;
    g.out = out;
    g.ldc = N;
    switch (kind) {
      case LIN_PLAIN:
      case LIN_NOBIAS: g.epi = tcg::EPI_BF16; break;
      case LIN_RESID: g.epi = tcg::EPI_RESID_F32; g.resid = resid; break;
      case LIN_GELU: g.epi = tcg::EPI_GELU; g.out2 = (bf16*)out2; break;
    }
    return tc_call(h, g);
  }
  simt::Args a{};
  a.A = (const float*)X;
  a.sam = K;
  a.sak = 1;
  a.B = h->P32(woff);
  a.sbn = K;
  a.sbk = 1;
  a.M = (int)M;
  a.N = N;
  a.K = K;
  a.bias = bias;
  a.out = (float*)out;
  a.ldc = N;
  switch (kind) {
    case LIN_PLAIN:
    case LIN_NOBIAS: a.epi = simt::EPI_F32; break;
    case LIN_RESID: a.epi = simt::EPI_RESID; a.resid = resid; break;
    case LIN_GELU: a.epi = simt::EPI_GELU; a.out2 = (float*)out2; break;
  }
  return simt_call(h, a);
}

// bf16 lm_head with the softmax-statistics epilogue: logits[M, Vp] = xf wte^T
// and h->ce_part
static int op_lm_head_ce(gpt2* h, long M) {
  KTimer kt(h, KC_GEMM, 2.0 * M * h->Vp * h->C, 0.0);
  tcg::GemmArgs g;
  g.A = (const bf16*)h->lnf;
  g.lda = h->C;
  g.B = h->PBF(h->wte);
  g.ldb = h->C;
  g.M = (int)M;
  g.N = h->Vp;
  g.K = h->C;
  g.out = h->logits;
  g.ldc = h->Vp;
  g.epi = tcg::EPI_CE_STATS;
  g.ce_part = h->ce_part;
  return tc_call(h, g);
}

// fp32 out / activation-typed out / x gelu'(aux) / bf16 out plus the attention
// backward's lse*log2(e) and D rows of layer `aux_layer` (the output is dO)
enum DgradKind { DG_F32, DG_ACT, DG_DGELU, DG_ACT_ROWDOT };

// dX[M,Kin] = dY[M,N] W[N,Kin]
static int op_lin_dgrad(gpt2* h, const void* dY, long M, int N, size_t woff, int Kin, DgradKind kind, void* out,
                        const void* aux, int aux_layer = -1) {
  KTimer kt(h, KC_GEMM, 2.0 * M * N * Kin, 0.0);
  if (h->prec == GPT2_BF16) {
    tcg::GemmArgs g;
    g.A = (const bf16*)dY;
    g.lda = N;
    g.a_mn = 0;
    g.B = h->PBF(woff);
    g.ldb = Kin;
    g.b_mn = 1;
    g.M = (int)M;
    g.N = Kin;
    g.K = N;
    g.out = out;
    g.ldc = Kin;
    g.epi = kind == DG_F32 ? tcg::EPI_F32 : (kind == DG_ACT ? tcg::EPI_BF16 : tcg::EPI_DGELU);
    g.aux = (const bf16*)aux;
    if (kind == DG_ACT_ROWDOT) {
      // aux: the layer's attention output O; the row dots D = rowsum(dO * O)
      // and lse*log2(e) go to the attention backward's scratch
      g.epi = tcg::EPI_ROWDOT;
      g.aux = (const bf16*)(h->att + (size_t)aux_layer * h->Mmax() * h->C * h->es);
      g.rd_out = h->attn_D;
      g.rd_lse = h->lse + (size_t)aux_layer * h->Mmax() * h->H;
      g.rd_T = h->T;
    }
    return tc_call(h, g);
  }
  simt::Args a{};
  a.A = (const float*)dY;
  a.sam = N;
  a.sak = 1;
  a.B = h->P32(woff);
  a.sbn = 1;
  a.sbk = Kin;
  a.M = (int)M;
  a.N = Kin;
  a.K = N;
  a.out = (float*)out;
  a.ldc = Kin;
  a.epi = kind == DG_DGELU ? simt::EPI_DGELU : simt::EPI_F32;
  a.aux = (const float*)aux;
  return simt_call(h, a);
}

// grads[W (N x Kin)] += dY[M,N]^T X[M,Kin]
static int op_lin_wgrad(gpt2* h, const void* dY, long M, int N, const void* X, int Kin, size_t woff) {
  KTimer kt(h, KC_GEMM, 2.0 * M * N * Kin, 0.0);
  if (h->prec == GPT2_BF16) {
    tcg::GemmArgs g;
    g.A = (const bf16*)dY;
    g.lda = N;
    g.a_mn = 1;
    g.B = (const bf16*)X;
    g.ldb = Kin;
    g.b_mn = 1;
    g.M = N;
    g.N = Kin;
    g.K = (int)M;
    g.out = h->G32(woff);
    g.ldc = Kin;
    g.epi = tcg::EPI_ACCUM_F32;
    for (const auto& ws : h->wslots)
      if (ws.woff == woff) {
        g.slots = ws.ptr;
        g.slot_splits = ws.splits;
        h->accum_dirty = true;
      }
    return tc_call(h, g);
  }
  simt::Args a{};
  a.A = (const float*)dY;
  a.sam = 1;
  a.sak = N;
  a.B = (const float*)X;
  a.sbn = 1;
  a.sbk = Kin;
  a.M = N;
  a.N = Kin;
  a.K = (int)M;
  a.out = h->G32(woff);
  a.ldc = Kin;
  a.epi = simt::EPI_ACCUM;
  return simt_call(h, a);
}

// Partial column sums of a[M, N] (activation type), added into
// h->psums[inst] (folded into the bias gradient later).
static int op_colsum(gpt2* h, const void* a, long M, int N, int inst) {
  KTimer kt(h, KC_OTHER, 0.0, (double)M * N * h->es);
  const int rpb = colsum_rows_per_block(M);
  const int nblk = (int)((M + rpb - 1) / rpb);
  const int vec = h->prec == GPT2_BF16 ? 8 : 4;
  dim3 grid((N + 32 * vec - 1) / (32 * vec), nblk);
  float* part = h->psums[inst].buf;
  if (h->prec == GPT2_BF16)
    k::colsum_partial_kernel<bf16><<<grid, 256, 0, h->stream>>>((const bf16*)a, (int)M, N, rpb, part);
  else
    k::colsum_partial_kernel<float><<<grid, 256, 0, h->stream>>>((const float*)a, (int)M, N, rpb, part);
  LAUNCH_CHECK(h);
  h->accum_dirty = true;
  return GPT2_OK;
}

// --------------------------------------------------------------- attention
static int op_attn_fwd(gpt2* h, int l) {
  KTimer kt(h, KC_ATTN_F, 2.0 * h->B * (double)h->T * h->T * h->C, 0.0);
  const long M = h->M();
  uint8_t* qkv = h->qkv + (size_t)l * h->Mmax() * 3 * h->C * h->es;
  uint8_t* att = h->att + (size_t)l * h->Mmax() * h->C * h->es;
  float* lse = h->lse + (size_t)l * h->Mmax() * h->H;
  (void)M;
  if (h->prec == GPT2_BF16) {
    if (tcfa::forward((const bf16*)qkv, (bf16*)att, lse, h->B, h->T, h->H, h->stream) != cudaSuccess)
      return set_err(h, GPT2_ECUDA, "attention forward launch");
    h->launches++;
  } else {
    if (attn::naive_forward((const float*)qkv, (float*)att, lse, h->B, h->T, h->H, h->C / h->H, h->stream) !=
        cudaSuccess)
      return set_err(h, GPT2_ECUDA, "attention forward launch");
    h->launches++;
  }
  return GPT2_OK;
}

// T a multiple of 128: the attention-output projection's dgrad forms the
// backward's lse*log2(e) and D rows (EPI_ROWDOT) instead of a separate kernel
static bool attn_rows_fused(const gpt2* h) { return h->prec == GPT2_BF16 && h->T % 128 == 0; }

static int op_attn_bwd(gpt2* h, int l) {
  KTimer kt(h, KC_ATTN_B, 4.0 * h->B * (double)h->T * h->T * h->C, 0.0);
  uint8_t* qkv = h->qkv + (size_t)l * h->Mmax() * 3 * h->C * h->es;
  uint8_t* att = h->att + (size_t)l * h->Mmax() * h->C * h->es;
  float* lse = h->lse + (size_t)l * h->Mmax() * h->H;
  if (h->prec == GPT2_BF16) {
    if (tcfa::backward((const bf16*)qkv, (const bf16*)att, (const bf16*)h->datt, lse, (bf16*)h->dqkv, h->attn_D,
                       h->B, h->T, h->H, h->stream, h->psums[3 * h->L + 1 + l].buf, h->attn_ds,
                       attn_rows_fused(h)) != cudaSuccess)
      return set_err(h, GPT2_ECUDA, "attention backward launch");
    h->launches += attn_rows_fused(h) ? 2 : 3;
    h->accum_dirty = true;
  } else {
    if (attn::naive_backward((const float*)qkv, (const float*)att, (const float*)h->datt, lse, (float*)h->dqkv,
                             h->attn_D, h->B, h->T, h->H, h->C / h->H, h->stream) != cudaSuccess)
      return set_err(h, GPT2_ECUDA, "attention backward launch");
    h->launches += 2;
  }
  return GPT2_OK;
}
