// Handle creation: argument checks, arena allocation, device-side init.
#pragma once
#include "model_ops.cuh"

static int validate_config(const gpt2_config* c, std::string& why) {
  if (c->n_layer < 1 || c->n_head < 1 || c->n_embd < 128 || c->n_embd > 1024 || c->n_embd % 128) {
    why = "n_layer >= 1, n_head >= 1, n_embd a multiple of 128 in [128, 1024]";
    return GPT2_EINVAL;
  }
  if (c->n_embd % c->n_head) {
    why = "n_embd must be divisible by n_head";
    return GPT2_EINVAL;
  }
  if (c->padded_vocab < c->vocab_size || c->vocab_size < 1 || c->padded_vocab % 64 || c->padded_vocab > 65472 ||
      (c->precision == GPT2_FP32 && c->padded_vocab > 51200)) {
    why = "padded_vocab: a multiple of 64, >= vocab_size, <= 65472 (<= 51200 in fp32 mode)";
    return GPT2_EINVAL;
  }
  if (c->block_size < 1 || c->max_T < 1 || c->max_T > c->block_size || c->max_B < 1) {
    why = "need 1 <= max_T <= block_size and max_B >= 1";
    return GPT2_EINVAL;
  }
  if ((long)c->max_B * c->max_T > 32768) {
    why = "max_B * max_T must be at most 32768 (embedding scatter-add sort capacity)";
    return GPT2_EINVAL;
  }
  if (c->precision != GPT2_FP32 && c->precision != GPT2_BF16) {
    why = "precision must be GPT2_FP32 or GPT2_BF16";
    return GPT2_EINVAL;
  }
  if (c->precision == GPT2_BF16 && c->n_embd / c->n_head != 64) {
    why = "bf16 mode needs head dim 64";
    return GPT2_EINVAL;
  }
  if (c->precision == GPT2_FP32 && c->n_embd / c->n_head > 64) {
    why = "fp32 mode supports head dim up to 64";
    return GPT2_EINVAL;
  }
  return GPT2_OK;
}

static int init_params_device(gpt2* h, uint64_t seed) {
  const float resid_std = 0.02f / sqrtf(2.f * h->L);
  for (const TensorInfo& t : h->tensors) {
    float* p = h->params + t.offset;
    const bool is_gain = t.name.size() >= 2 && t.name.compare(t.name.size() - 2, 2, ".g") == 0;
    const bool is_bias = t.name.size() >= 2 && t.name.compare(t.name.size() - 2, 2, ".b") == 0;
    const bool is_resid = t.name.find("proj.w") != std::string::npos;  // attn proj and mlp proj
    const int blocks = grid_for((long)t.numel, 256);
    if (is_gain)
      k::fill_kernel<<<blocks, 256, 0, h->stream>>>(p, (long)t.numel, 1.f);
    else if (is_bias)
      k::fill_kernel<<<blocks, 256, 0, h->stream>>>(p, (long)t.numel, 0.f);
    else
      k::init_normal_kernel<<<blocks, 256, 0, h->stream>>>(p, (long)t.numel, seed, (long)t.offset,
                                                           is_resid ? resid_std : 0.02f);
    LAUNCH_CHECK(h);
  }
  return GPT2_OK;
}

static int refresh_bf16(gpt2* h) {
  if (h->prec != GPT2_BF16) return GPT2_OK;
  k::f32_to_bf16_kernel<<<grid_for((long)h->nparams, 256), 256, 0, h->stream>>>(h->params, h->pbf, (long)h->nparams);
  LAUNCH_CHECK(h);
  return GPT2_OK;
}

static int create_impl(gpt2* h, const gpt2_config* c, uint64_t seed) {
  std::string why;
  if (validate_config(c, why) != GPT2_OK) return set_err(h, GPT2_EINVAL, why);
  {
    const cudaError_t stale = cudaGetLastError();
    if (stale != cudaSuccess)
      return set_err(h, GPT2_ECUDA, std::string("CUDA error pending before create: ") + cudaGetErrorString(stale));
  }
  h->cfg = *c;
  h->L = c->n_layer;
  h->H = c->n_head;
  h->C = c->n_embd;
  h->V = c->vocab_size;
  h->Vp = c->padded_vocab;
  h->P = c->block_size;
  h->maxB = c->max_B;
  h->maxT = c->max_T;
  h->prec = c->precision;
  h->es = h->prec == GPT2_BF16 ? 2 : 4;
  build_tensor_table(h);
  const size_t N = h->nparams, es = h->es;
  const long Mx = h->Mmax();
  const int L = h->L, C = h->C, H = h->H;

  ALLOC(h, h->params, N * 4);
  ALLOC(h, h->grads, N * 4);
  ALLOC(h, h->m, N * 4);
  ALLOC(h, h->v, N * 4);
  if (h->prec == GPT2_BF16) ALLOC(h, h->pbf, N * 2);
  ALLOC(h, h->res, (size_t)(2 * L + 1) * Mx * C * 4);
  ALLOC(h, h->ln1, (size_t)L * Mx * C * es);
  ALLOC(h, h->ln2, (size_t)L * Mx * C * es);
  ALLOC(h, h->ln1_mean, (size_t)L * Mx * 4);
  ALLOC(h, h->ln1_rstd, (size_t)L * Mx * 4);
  ALLOC(h, h->ln2_mean, (size_t)L * Mx * 4);
  ALLOC(h, h->ln2_rstd, (size_t)L * Mx * 4);
  ALLOC(h, h->qkv, (size_t)L * Mx * 3 * C * es);
  ALLOC(h, h->att, (size_t)L * Mx * C * es);
  ALLOC(h, h->lse, (size_t)L * Mx * H * 4);
  ALLOC(h, h->fcu, (size_t)L * Mx * 4 * C * es);
  ALLOC(h, h->fca, (size_t)L * Mx * 4 * C * es);
  ALLOC(h, h->lnf, (size_t)Mx * C * es);
  ALLOC(h, h->lnf_mean, (size_t)Mx * 4);
  ALLOC(h, h->lnf_rstd, (size_t)Mx * 4);
  ALLOC(h, h->logits, (size_t)Mx * h->Vp * es);
  ALLOC(h, h->ce_lse, (size_t)Mx * 4);
  if (h->prec == GPT2_BF16) {
    ALLOC(h, h->ce_part, (size_t)Mx * tcg::ce_halves(h->Vp) * 3 * 4);
    ALLOC(h, h->attn_ds, (size_t)tcfa::backward_ds_elems(h->maxB, h->maxT, H) * 2);
  }
  ALLOC(h, h->losses, (size_t)Mx * 4);
  ALLOC(h, h->d_loss, 16);
  ALLOC(h, h->argmax, (size_t)Mx * 4);
  ALLOC(h, h->dres, (size_t)Mx * C * 4);
  ALLOC(h, h->dln, (size_t)Mx * C * 4);
  if (h->prec == GPT2_BF16) ALLOC(h, h->dres_bf, (size_t)Mx * C * 2);
  ALLOC(h, h->dbig, (size_t)Mx * 4 * C * es);
  ALLOC(h, h->dqkv, (size_t)Mx * 3 * C * es);
  ALLOC(h, h->datt, (size_t)Mx * C * es);
  {
    // attention backward scratch: per query, lse*log2(e) and D (bf16 mode, padded
    // to 128-query blocks), or D alone (fp32 mode); the larger of the two
    const long nb = tcfa::backward_scratch_floats(h->maxB, h->maxT, H);
    ALLOC(h, h->attn_D, (size_t)(nb > Mx * H ? nb : Mx * H) * 4);
  }
  {
    // partial column sums accumulated over the micro-steps (see PartialSums)
    const int rpb = ln_rows_per_block(Mx);
    const int nblk = (int)((Mx + rpb - 1) / rpb);
    const int crpb = colsum_rows_per_block(Mx);
    const int cblk = (int)((Mx + crpb - 1) / crpb);
    const int qrows = h->prec == GPT2_BF16 ? (int)tcfa::backward_colsum_rows(h->maxB, h->maxT) : cblk;
    h->psums.resize(4 * L + 1);
    for (int l = 0; l < L; ++l) {
      const LayerOffsets& o = h->lo[l];
      h->psums[2 * l] = {nullptr, nblk, 3 * C, C, {o.ln1g, o.ln1b, l > 0 ? h->lo[l - 1].mpb : NO_OFF}};
      h->psums[2 * l + 1] = {nullptr, nblk, 3 * C, C, {o.ln2g, o.ln2b, o.projb}};
      h->psums[2 * L + 1 + l] = {nullptr, cblk, 4 * C, 4 * C, {o.fcb, NO_OFF, NO_OFF}};
      h->psums[3 * L + 1 + l] = {nullptr, qrows, 3 * C, 3 * C, {o.attnb, NO_OFF, NO_OFF}};
    }
    h->psums[2 * L] = {nullptr, nblk, 3 * C, C, {h->lnfg, h->lnfb, h->lo[L - 1].mpb}};
    size_t total = 0;
    for (auto& ps : h->psums) total += (size_t)ps.rows * ps.ncols;
    h->psum_floats = total;
    ALLOC(h, h->psum_buf, total * 4);
    CU_CHECK(h, cudaMemsetAsync(h->psum_buf, 0, total * 4, h->stream));
    size_t at = 0;
    for (auto& ps : h->psums) {
      ps.buf = h->psum_buf + at;
      at += (size_t)ps.rows * ps.ncols;
    }
  }
  if (h->prec == GPT2_BF16) {
    // per-split accumulators of the weight gradients that the tcgen05 GEMM
    // splits over the tokens (the lm_head's has tiles enough and goes straight
    // into grads)
    size_t total = 0;
    for (int l = 0; l < L; ++l) {
      const LayerOffsets& o = h->lo[l];
      const size_t w[4][3] = {{o.attnw, (size_t)3 * C, (size_t)C},
                              {o.projw, (size_t)C, (size_t)C},
                              {o.fcw, (size_t)4 * C, (size_t)C},
                              {o.mpw, (size_t)C, (size_t)4 * C}};
      for (auto& x : w) {
        const int sp = tcg::accum_slot_splits((int)x[1], (int)x[2], (int)Mx);
        if (sp < 2) continue;
        const long n = (long)(x[1] * x[2]);
        h->wslots.push_back({x[0], nullptr, sp, n});
        total += (size_t)sp * n;
      }
    }
    h->slot_floats = total;
    if (total) {
      ALLOC(h, h->slot_buf, total * 4);
      CU_CHECK(h, cudaMemsetAsync(h->slot_buf, 0, total * 4, h->stream));
      size_t at = 0;
      for (auto& ws : h->wslots) {
        ws.ptr = h->slot_buf + at;
        at += (size_t)ws.splits * ws.n;
      }
    }
  }
  ALLOC(h, h->emb_keys, (size_t)Mx * 4);
  ALLOC(h, h->emb_part, (size_t)Mx * C * 4);
  h->sort_cap = 1;
  while (h->sort_cap < Mx) h->sort_cap <<= 1;
  ALLOC(h, h->normbuf, 32);
  ALLOC(h, h->d_step, 8);
  h->norm_blocks = 2 * 148;
  ALLOC(h, h->norm_part, (size_t)h->norm_blocks * 8);
  {
    std::vector<k::AdamSeg> segs;
    for (const TensorInfo& t : h->tensors) segs.push_back(k::AdamSeg{(long)t.offset, t.decay});
    h->nseg = (int)segs.size();
    if (h->nseg > 160) return set_err(h, GPT2_EINVAL, "too many tensors for the AdamW segment table (max 160)");
    ALLOC(h, h->segs, segs.size() * sizeof(k::AdamSeg));
    CU_CHECK(h, cudaMemcpy(h->segs, segs.data(), segs.size() * sizeof(k::AdamSeg), cudaMemcpyHostToDevice));
  }
  ALLOC(h, h->d_bad, 16);
  ALLOC(h, h->tok_dev, (size_t)Mx * 4);
  ALLOC(h, h->tgt_dev, (size_t)Mx * 4);

  CU_CHECK(h, cudaMemsetAsync(h->grads, 0, N * 4, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->m, 0, N * 4, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->v, 0, N * 4, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->d_bad, 0, 16, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->d_loss, 0, 16, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->d_step, 0, 8, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->normbuf, 0, 32, h->stream));
  int r = init_params_device(h, seed);
  if (r != GPT2_OK) return r;
  r = refresh_bf16(h);
  if (r != GPT2_OK) return r;
  // kernels with large dynamic shared memory
  // (exactly the dynamic shared memory each launch asks for; the opt-in limit
  // covers static plus dynamic shared memory)
  const int ce_smem = (int)((size_t)h->Vp * h->es);
  if (h->prec != GPT2_BF16)
    CU_CHECK(h, cudaFuncSetAttribute(k::ce_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, ce_smem));
  CU_CHECK(h, cudaFuncSetAttribute(k::sort_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, h->sort_cap * 4));
  CU_CHECK(h, cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking));
  CU_CHECK(h, cudaStreamCreateWithFlags(&h->side_stream, cudaStreamNonBlocking));
  CU_CHECK(h, cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
  CU_CHECK(h, cudaEventCreateWithFlags(&h->ev_sorted, cudaEventDisableTiming));
  CU_CHECK(h, cudaEventCreateWithFlags(&h->ev_in, cudaEventDisableTiming));
  CU_CHECK(h, cudaEventCreateWithFlags(&h->ev_out, cudaEventDisableTiming));
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}
