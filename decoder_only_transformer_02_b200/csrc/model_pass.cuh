// The training step itself: forward, backward, clip + AdamW.
#pragma once
#include "model_create.cuh"

struct Views {
  gpt2* h;
  float* res(int i) const { return h->res + (size_t)i * h->Mmax() * h->C; }
  uint8_t* ln1(int l) const { return h->ln1 + (size_t)l * h->Mmax() * h->C * h->es; }
  uint8_t* ln2(int l) const { return h->ln2 + (size_t)l * h->Mmax() * h->C * h->es; }
  float* ln1m(int l) const { return h->ln1_mean + (size_t)l * h->Mmax(); }
  float* ln1r(int l) const { return h->ln1_rstd + (size_t)l * h->Mmax(); }
  float* ln2m(int l) const { return h->ln2_mean + (size_t)l * h->Mmax(); }
  float* ln2r(int l) const { return h->ln2_rstd + (size_t)l * h->Mmax(); }
  uint8_t* qkv(int l) const { return h->qkv + (size_t)l * h->Mmax() * 3 * h->C * h->es; }
  uint8_t* att(int l) const { return h->att + (size_t)l * h->Mmax() * h->C * h->es; }
  uint8_t* fcu(int l) const { return h->fcu + (size_t)l * h->Mmax() * 4 * h->C * h->es; }
  uint8_t* fca(int l) const { return h->fca + (size_t)l * h->Mmax() * 4 * h->C * h->es; }
};

#define RET_IF(x)                \
  do {                           \
    int r__ = (x);               \
    if (r__ != GPT2_OK) return r__; \
  } while (0)

// fuse: the softmax gradient (scaled by loss_scale / M) overwrites the logits
// in the same pass that computes the loss
// The embedding backward's (token, position) sort needs only the ids: it runs
// on the side stream, forked just before the cross-entropy pass, whose many
// small CTAs share the SMs with its one CTA (the persistent GEMM and attention
// kernels of the forward would wait for the SM it holds); the backward joins
// it before the embedding scatter-add.
static int fork_embedding_sort(gpt2* h, bool with_targets) {
  if (!with_targets || h->timing) return GPT2_OK;
  CU_CHECK(h, cudaEventRecord(h->ev_fork, h->stream));
  CU_CHECK(h, cudaStreamWaitEvent(h->side_stream, h->ev_fork, 0));
  k::sort_keys_kernel<<<1, 1024, (size_t)h->sort_cap * 4, h->side_stream>>>(h->tok_dev, (int)h->M(), h->Vp,
                                                                             h->emb_keys, h->sort_cap);
  LAUNCH_CHECK(h);
  CU_CHECK(h, cudaEventRecord(h->ev_sorted, h->side_stream));
  h->sort_pending = true;
  return GPT2_OK;
}

static int forward_impl(gpt2* h, const int32_t* tok, const int32_t* tgt, int B, int T, bool fuse, float loss_scale) {
  if (tok == nullptr) return set_err(h, GPT2_EINVAL, "tokens pointer is NULL");
  if (B < 1 || T < 1 || B > h->maxB || T > h->maxT)
    return set_err(h, GPT2_EINVAL, "B, T must satisfy 1 <= B <= max_B and 1 <= T <= max_T");
  if (fuse && tgt == nullptr) return set_err(h, GPT2_EINVAL, "fused forward-backward needs targets");
  h->B = B;
  h->T = T;
  h->have_fwd = false;
  const long M = h->M();
  const int C = h->C, L = h->L;
  Views w{h};
  if (h->sort_pending) {
    // a sort forked by an earlier forward that no backward joined still reads
    // the ids: join it before they are overwritten
    CU_CHECK(h, cudaStreamWaitEvent(h->stream, h->ev_sorted, 0));
    h->sort_pending = false;
  }
  // keep private copies of the ids: the backward pass reads them again
  if (tok != h->tok_dev) CU_CHECK(h, cudaMemcpyAsync(h->tok_dev, tok, M * 4, cudaMemcpyDeviceToDevice, h->stream));
  if (tgt && tgt != h->tgt_dev)
    CU_CHECK(h, cudaMemcpyAsync(h->tgt_dev, tgt, M * 4, cudaMemcpyDeviceToDevice, h->stream));
  const int32_t* dtgt = tgt ? h->tgt_dev : nullptr;

  {
    KTimer kt(h, KC_EMB, 0.0, 12.0 * M * C);
    k::embed_fwd_kernel<<<grid_for(M * C / 4, 256), 256, 0, h->stream>>>(
        h->tok_dev, dtgt, h->P32(h->wte), h->P32(h->wpe), w.res(0), (int)M, T, C, h->Vp, h->d_bad);
    LAUNCH_CHECK(h);
  }
  for (int l = 0; l < L; ++l) {
    const LayerOffsets& o = h->lo[l];
    RET_IF(op_ln_fwd(h, w.res(2 * l), o.ln1g, o.ln1b, w.ln1(l), w.ln1m(l), w.ln1r(l), M));
    RET_IF(op_lin_fwd(h, w.ln1(l), M, C, o.attnw, 3 * C, o.attnb, LIN_PLAIN, w.qkv(l), nullptr, nullptr));
    RET_IF(op_attn_fwd(h, l));
    RET_IF(op_lin_fwd(h, w.att(l), M, C, o.projw, C, o.projb, LIN_RESID, w.res(2 * l + 1), nullptr, w.res(2 * l)));
    RET_IF(op_ln_fwd(h, w.res(2 * l + 1), o.ln2g, o.ln2b, w.ln2(l), w.ln2m(l), w.ln2r(l), M));
    RET_IF(op_lin_fwd(h, w.ln2(l), M, C, o.fcw, 4 * C, o.fcb, LIN_GELU, w.fcu(l), w.fca(l), nullptr));
    RET_IF(op_lin_fwd(h, w.fca(l), M, 4 * C, o.mpw, C, o.mpb, LIN_RESID, w.res(2 * l + 2), nullptr,
                      w.res(2 * l + 1)));
  }
  RET_IF(op_ln_fwd(h, w.res(2 * L), h->lnfg, h->lnfb, h->lnf, h->lnf_mean, h->lnf_rstd, M));
  const float gscale = loss_scale / (float)M;
  if (h->prec == GPT2_BF16) {
    // tied lm_head: logits = xf wte^T (no bias); the GEMM epilogue also emits
    // per-(row, 128-column) softmax statistics of the stored logits, so the
    // cross-entropy pass only merges them and streams the row once for the
    // gradient
    RET_IF(op_lm_head_ce(h, M));
    RET_IF(fork_embedding_sort(h, dtgt != nullptr));
    KTimer kt(h, KC_CE, 0.0, (double)M * h->Vp * 2 * (fuse ? 2 : 0) + (double)M * tcg::ce_halves(h->Vp) * 12);
    k::ce_finish_kernel<<<(unsigned)M, k::CEF_THREADS, 0, h->stream>>>(
        (bf16*)h->logits, h->ce_part, tcg::ce_halves(h->Vp), dtgt, h->Vp, h->ce_lse, dtgt ? h->losses : nullptr,
        h->argmax, fuse ? 1 : 0, gscale);
    LAUNCH_CHECK(h);
  } else {
    RET_IF(op_lin_fwd(h, h->lnf, M, C, h->wte, h->Vp, NO_OFF, LIN_NOBIAS, h->logits, nullptr, nullptr));
    RET_IF(fork_embedding_sort(h, dtgt != nullptr));
    const size_t smem = (size_t)h->Vp * h->es;
    KTimer kt(h, KC_CE, 0.0, (double)M * h->Vp * h->es * (fuse ? 2 : 1));
    k::ce_kernel<float><<<(unsigned)M, 1024, smem, h->stream>>>((float*)h->logits, dtgt, h->Vp, h->ce_lse,
                                                                 dtgt ? h->losses : nullptr, h->argmax, fuse ? 1 : 0,
                                                                 gscale);
    LAUNCH_CHECK(h);
  }
  if (dtgt) {
    KTimer kt(h, KC_OTHER, 0.0, 4.0 * M);
    k::loss_mean_kernel<<<1, 1024, 0, h->stream>>>(h->losses, (int)M, h->d_loss, h->d_loss + 1,
                                                   fuse ? loss_scale : 0.f);
    LAUNCH_CHECK(h);
  }
  h->have_fwd = true;
  h->have_targets = dtgt != nullptr;
  h->logits_valid = !fuse;
  return GPT2_OK;
}

static int backward_impl(gpt2* h, float loss_scale, bool fused) {
  if (!h->have_fwd || !h->have_targets)
    return set_err(h, GPT2_ESTATE, "backward needs a preceding forward with targets");
  if (!fused && !h->logits_valid) return set_err(h, GPT2_ESTATE, "the logits of the last forward were consumed");
  const long M = h->M();
  const int C = h->C, L = h->L, B = h->B, T = h->T;
  Views w{h};
  if (!fused) {
    KTimer kt(h, KC_CE, 0.0, 2.0 * M * h->Vp * h->es);
    const float gscale = loss_scale / (float)M;
    if (h->prec == GPT2_BF16)
      k::ce_bwd_kernel<bf16><<<(unsigned)M, 512, 0, h->stream>>>((bf16*)h->logits, h->tgt_dev, h->ce_lse, h->Vp,
                                                                 gscale);
    else
      k::ce_bwd_kernel<float><<<(unsigned)M, 512, 0, h->stream>>>((float*)h->logits, h->tgt_dev, h->ce_lse, h->Vp,
                                                                  gscale);
    LAUNCH_CHECK(h);
    h->logits_valid = false;
  }
  const void* dlog = h->logits;
  const bool bf = h->prec == GPT2_BF16;
  const void* dres_act = bf ? (const void*)h->dres_bf : (const void*)h->dres;
  // lm_head (tied): dwte += dlogits^T xf ; dxf = dlogits wte
  RET_IF(op_lin_wgrad(h, dlog, M, h->Vp, h->lnf, C, h->wte));
  RET_IF(op_lin_dgrad(h, dlog, M, h->Vp, h->wte, C, DG_F32, h->dln, nullptr));
  RET_IF(op_ln_bwd(h, h->dln, w.res(2 * L), h->lnf_mean, h->lnf_rstd, h->lnfg, 2 * L, M, 0));
  for (int l = L - 1; l >= 0; --l) {
    const LayerOffsets& o = h->lo[l];
    // MLP half: x_out = x_mid + mproj(gelu(fc(ln2(x_mid))))
    RET_IF(op_lin_wgrad(h, dres_act, M, C, w.fca(l), 4 * C, o.mpw));
    RET_IF(op_lin_dgrad(h, dres_act, M, C, o.mpw, 4 * C, DG_DGELU, h->dbig, w.fcu(l)));
    RET_IF(op_colsum(h, h->dbig, M, 4 * C, 2 * L + 1 + l));
    RET_IF(op_lin_wgrad(h, h->dbig, M, 4 * C, w.ln2(l), C, o.fcw));
    RET_IF(op_lin_dgrad(h, h->dbig, M, 4 * C, o.fcw, C, DG_F32, h->dln, nullptr));
    RET_IF(op_ln_bwd(h, h->dln, w.res(2 * l + 1), w.ln2m(l), w.ln2r(l), o.ln2g, 2 * l + 1, M, 1));
    // attention half: x_mid = x_in + proj(attn(qkv(ln1(x_in))))
    RET_IF(op_lin_wgrad(h, dres_act, M, C, w.att(l), C, o.projw));
    RET_IF(op_lin_dgrad(h, dres_act, M, C, o.projw, C, attn_rows_fused(h) ? DG_ACT_ROWDOT : DG_ACT, h->datt, nullptr,
                        l));
    RET_IF(op_attn_bwd(h, l));  // (bf16: with the qkv bias partial sums)
    if (h->prec != GPT2_BF16) RET_IF(op_colsum(h, h->dqkv, M, 3 * C, 3 * L + 1 + l));
    RET_IF(op_lin_wgrad(h, h->dqkv, M, 3 * C, w.ln1(l), C, o.attnw));
    RET_IF(op_lin_dgrad(h, h->dqkv, M, 3 * C, o.attnw, C, DG_F32, h->dln, nullptr));
    RET_IF(op_ln_bwd(h, h->dln, w.res(2 * l), w.ln1m(l), w.ln1r(l), o.ln1g, 2 * l, M, 1));
  }
  // embeddings: dwte[tok] += dx0 (sorted, fixed order), dwpe[t] += sum_b dx0[b, t]
  KTimer kt(h, KC_EMB, 0.0, 8.0 * M * C + 8.0 * T * C);
  if (h->sort_pending) {
    CU_CHECK(h, cudaStreamWaitEvent(h->stream, h->ev_sorted, 0));
    h->sort_pending = false;
  } else {
    k::sort_keys_kernel<<<1, 1024, (size_t)h->sort_cap * 4, h->stream>>>(h->tok_dev, (int)M, h->Vp, h->emb_keys,
                                                                          h->sort_cap);
    LAUNCH_CHECK(h);
  }
  const int eth = C / 4;  // one thread per 4 columns (n_embd <= 1024)
  k::embed_bwd_partial_kernel<<<(unsigned)((M + k::EMB_CH - 1) / k::EMB_CH), eth, 0, h->stream>>>(
      h->emb_keys, h->dres, (int)M, C, h->emb_part);
  LAUNCH_CHECK(h);
  k::embed_bwd_reduce_kernel<<<(unsigned)M, eth, 0, h->stream>>>(h->emb_keys, h->emb_part, (int)M, C, h->Vp,
                                                                 h->G32(h->wte));
  LAUNCH_CHECK(h);
  k::wpe_bwd_kernel<<<grid_for((long)T * C / 4, 256), 256, 0, h->stream>>>(h->dres, B, T, C, h->G32(h->wpe));
  LAUNCH_CHECK(h);
  h->have_bwd_keys = true;
  h->have_targets = false;  // one backward per forward
  return GPT2_OK;
}

// Fold the accumulators (the per-split weight gradients and the partial
// column sums) into grads, in a fixed order, and clear them.
static int fold_accumulators(gpt2* h) {
  if (!h->accum_dirty) return GPT2_OK;
  KTimer kt(h, KC_OPT, 0.0, 12.0 * (double)h->slot_floats + 4.0 * (double)h->psum_floats);
  for (const auto& ws : h->wslots) {
    k::slot_fold_kernel<<<grid_for(ws.n / 4, 256, 4), 256, 0, h->stream>>>(h->G32(ws.woff), ws.ptr, ws.n, ws.splits);
    LAUNCH_CHECK(h);
  }
  for (const auto& ps : h->psums) {
    float* o[3];
    for (int j = 0; j < 3; ++j) o[j] = ps.off[j] == NO_OFF ? nullptr : h->G32(ps.off[j]);
    k::partials_reduce_kernel<<<dim3((ps.ncols + 31) / 32, k::PR_SPLIT), 256, 0, h->stream>>>(
        ps.buf, ps.rows, ps.ncols, ps.C, o[0], o[1], o[2]);
    LAUNCH_CHECK(h);
  }
  CU_CHECK(h, cudaMemsetAsync(h->psum_buf, 0, h->psum_floats * 4, h->stream));
  h->accum_dirty = false;
  return GPT2_OK;
}
// Discard whatever the accumulators hold (with the gradients being zeroed).
static int clear_accumulators(gpt2* h) {
  if (!h->accum_dirty) return GPT2_OK;
  if (h->slot_buf) CU_CHECK(h, cudaMemsetAsync(h->slot_buf, 0, h->slot_floats * 4, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->psum_buf, 0, h->psum_floats * 4, h->stream));
  h->accum_dirty = false;
  return GPT2_OK;
}

static int adamw_impl(gpt2* h, float lr, float wd, float b1, float b2, float eps, float clip) {
  RET_IF(fold_accumulators(h));
  const long n = (long)h->nparams;
  KTimer kt(h, KC_OPT, 0.0, 34.0 * n);
  long per = (n + h->norm_blocks - 1) / h->norm_blocks;
  per = (per + 3) / 4 * 4;
  k::sumsq_partial_kernel<<<h->norm_blocks, 256, 0, h->stream>>>(h->grads, n, per, h->norm_part);
  LAUNCH_CHECK(h);
  k::norm_finish_kernel<<<1, 32, 0, h->stream>>>(h->norm_part, h->norm_blocks, clip, b1, b2, h->normbuf, h->d_step);
  LAUNCH_CHECK(h);
  k::adamw_kernel<<<grid_for(n / 4, 256, 4), 256, 0, h->stream>>>(h->params, h->grads, h->m, h->v,
                                                                  h->prec == GPT2_BF16 ? h->pbf : nullptr, n, h->segs,
                                                                  h->nseg, h->normbuf, lr, wd, b1, b2, eps);
  LAUNCH_CHECK(h);
  return GPT2_OK;
}

// Sync point: surface device-side flags (token range, bounded-wait timeouts).
static int check_device_flags(gpt2* h) {
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  int bad = 0;
  CU_CHECK(h, cudaMemcpy(&bad, h->d_bad, 4, cudaMemcpyDeviceToHost));
  int derr = 0;
  CU_CHECK(h, cudaMemcpyFromSymbol(&derr, g_device_err, 4));
  if (derr) {
    int zero = 0;
    cudaMemcpyToSymbol(g_device_err, &zero, 4);
    return set_err(h, GPT2_ECUDA, "a device-side wait timed out (error code " + std::to_string(derr) + ")");
  }
  if (bad) {
    CU_CHECK(h, cudaMemset(h->d_bad, 0, 4));
    return set_err(h, GPT2_ETOKEN, "a token or target id lies outside [0, padded_vocab)");
  }
  return GPT2_OK;
}

// One fused micro-step (forward with targets + backward, loss scaled by
// loss_scale).  The ids are first copied to the handle's private buffers.  With
// graphs enabled and timing off, the kernel sequence is captured into a CUDA
// graph the second time a (B, T, loss_scale) combination is seen (the first
// run is eager and also initialises the kernels' one-time attributes) and
// replayed afterwards on a private stream joined to the handle's stream with
// events.  A failed capture falls back to eager launches for that key.
static int fused_micro_step(gpt2* h, const int32_t* tok, const int32_t* tgt, int B, int T, float loss_scale) {
  if (tok == nullptr || tgt == nullptr) return set_err(h, GPT2_EINVAL, "fused forward-backward needs ids and targets");
  if (B < 1 || T < 1 || B > h->maxB || T > h->maxT)
    return set_err(h, GPT2_EINVAL, "B, T must satisfy 1 <= B <= max_B and 1 <= T <= max_T");
  const long M = (long)B * T;
  if (tok != h->tok_dev) CU_CHECK(h, cudaMemcpyAsync(h->tok_dev, tok, M * 4, cudaMemcpyDeviceToDevice, h->stream));
  if (tgt != h->tgt_dev) CU_CHECK(h, cudaMemcpyAsync(h->tgt_dev, tgt, M * 4, cudaMemcpyDeviceToDevice, h->stream));
  auto eager = [&]() -> int {
    RET_IF(forward_impl(h, h->tok_dev, h->tgt_dev, B, T, true, loss_scale));
    return backward_impl(h, loss_scale, true);
  };
  if (!h->use_graphs || h->timing) return eager();
  uint32_t sb;
  memcpy(&sb, &loss_scale, 4);
  gpt2::GraphEntry* e = nullptr;
  for (auto& g : h->graphs)
    if (g.B == B && g.T == T && g.scale_bits == sb) e = &g;
  if (e == nullptr) {
    h->graphs.push_back(gpt2::GraphEntry{B, T, sb, 0, nullptr, 0});
    return eager();
  }
  if (e->state < 0) return eager();
  if (e->state == 0) {
    // capture on the private stream
    cudaStream_t user = h->stream;
    CU_CHECK(h, cudaEventRecord(h->ev_in, user));
    CU_CHECK(h, cudaStreamWaitEvent(h->cap_stream, h->ev_in, 0));
    CU_CHECK(h, cudaStreamSynchronize(h->cap_stream));
    if (cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      cudaGetLastError();
      e->state = -1;
      return eager();
    }
    h->stream = h->cap_stream;
    const int64_t l0 = h->launches;
    const int r = eager();
    h->stream = user;
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(h->cap_stream, &graph);
    cudaGraphExec_t exec = nullptr;
    if (r != GPT2_OK || ce != cudaSuccess || graph == nullptr ||
        cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
      cudaGetLastError();
      if (graph) cudaGraphDestroy(graph);
      e->state = -1;
      if (r != GPT2_OK) return r;
      h->launches = l0;
      return eager();
    }
    cudaGraphDestroy(graph);
    e->exec = exec;
    e->nlaunch = h->launches - l0;
    h->launches = l0;
    e->state = 1;
  }
  CU_CHECK(h, cudaEventRecord(h->ev_in, h->stream));
  CU_CHECK(h, cudaStreamWaitEvent(h->cap_stream, h->ev_in, 0));
  CU_CHECK(h, cudaGraphLaunch(e->exec, h->cap_stream));
  CU_CHECK(h, cudaEventRecord(h->ev_out, h->cap_stream));
  CU_CHECK(h, cudaStreamWaitEvent(h->stream, h->ev_out, 0));
  h->launches += e->nlaunch;
  // the host-side state the replayed sequence implies
  h->B = B;
  h->T = T;
  h->have_fwd = true;
  h->have_targets = false;
  h->logits_valid = false;
  h->have_bwd_keys = true;
  h->accum_dirty = true;  // its gradients went into the accumulators
  return GPT2_OK;
}
