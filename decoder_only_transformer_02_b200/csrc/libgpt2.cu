// libgpt2: the C ABI declared in include/gpt2.h.  Single translation unit: the
// kernels, the GEMM and the runtime are all included here so that they share
// one device error word.
#include "tc_gemm.cu"
#include "attention_tc.cuh"
#include "attention_tc_bwd.cuh"
#include "model_pass.cuh"
#include "model_decode.cuh"

#include <mutex>


static std::string g_null_handle_err = "handle is NULL";

// Scratch of gpt2_attention_backward_noalloc: a fixed device array (two fp32
// per attention row, rows padded to 128-query blocks), so that entry point
// never allocates.  Host code cannot
// use the symbol itself as a device address: the address is looked up once per
// device, with that device current, and cached.
static __device__ __align__(256) float g_attn_noalloc_scratch[2 * GPT2_ATTN_NOALLOC_MAX_ROWS];
static std::mutex g_noalloc_mu;
static float* g_noalloc_addr[256] = {};

static float* noalloc_scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_addr[dev] = static_cast<float*>(p);
  }
  return g_noalloc_addr[dev];
}

extern "C" {

int gpt2_create(const gpt2_config* cfg, uint64_t seed, gpt2_t** out) {
  if (cfg == nullptr || out == nullptr) return GPT2_EINVAL;
  *out = nullptr;
  gpt2* h = new (std::nothrow) gpt2();
  if (h == nullptr) return GPT2_ENOMEM;
  const int r = create_impl(h, cfg, seed);
  if (r != GPT2_OK) {
    fprintf(stderr, "gpt2_create: %s\n", h->err.c_str());
    free_all(h);
    delete h;
    return r;
  }
  *out = h;
  return GPT2_OK;
}

void gpt2_destroy(gpt2_t* h) {
  if (h == nullptr) return;
  cudaStreamSynchronize(h->stream);
  if (h->cap_stream) cudaStreamSynchronize(h->cap_stream);
  for (auto& g : h->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  if (h->side_stream) {
    cudaStreamSynchronize(h->side_stream);
    cudaStreamDestroy(h->side_stream);
  }
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_sorted) cudaEventDestroy(h->ev_sorted);
  if (h->ev_in) cudaEventDestroy(h->ev_in);
  if (h->ev_out) cudaEventDestroy(h->ev_out);
  for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
  free_all(h);
  delete h;
}

int gpt2_set_stream(gpt2_t* h, void* s) {
  if (h == nullptr) return GPT2_EINVAL;
  h->stream = reinterpret_cast<cudaStream_t>(s);
  return GPT2_OK;
}

int gpt2_forward(gpt2_t* h, const int32_t* tok, const int32_t* tgt, int B, int T, float* h_loss) {
  if (h == nullptr) return GPT2_EINVAL;
  RET_IF(forward_impl(h, tok, tgt, B, T, false, 1.f));
  if (h_loss) {
    RET_IF(check_device_flags(h));
    if (!tgt) return set_err(h, GPT2_ESTATE, "no loss without targets");
    CU_CHECK(h, cudaMemcpy(h_loss, h->d_loss, 4, cudaMemcpyDeviceToHost));
  }
  return GPT2_OK;
}

int gpt2_backward(gpt2_t* h, float loss_scale) {
  if (h == nullptr) return GPT2_EINVAL;
  return backward_impl(h, loss_scale, false);
}

int gpt2_forward_backward(gpt2_t* h, const int32_t* tok, const int32_t* tgt, int B, int T, float loss_scale,
                          float* h_loss) {
  if (h == nullptr) return GPT2_EINVAL;
  RET_IF(fused_micro_step(h, tok, tgt, B, T, loss_scale));
  if (h_loss) {
    RET_IF(check_device_flags(h));
    CU_CHECK(h, cudaMemcpy(h_loss, h->d_loss, 4, cudaMemcpyDeviceToHost));
  }
  return GPT2_OK;
}

int gpt2_zero_grad(gpt2_t* h) {
  if (h == nullptr) return GPT2_EINVAL;
  RET_IF(clear_accumulators(h));
  CU_CHECK(h, cudaMemsetAsync(h->grads, 0, h->nparams * 4, h->stream));
  return GPT2_OK;
}

int gpt2_adamw_step(gpt2_t* h, float lr, float wd, float b1, float b2, float eps, float clip, float* h_norm) {
  if (h == nullptr) return GPT2_EINVAL;
  RET_IF(adamw_impl(h, lr, wd, b1, b2, eps, clip));
  if (h_norm) {
    RET_IF(check_device_flags(h));
    float nb[3];
    CU_CHECK(h, cudaMemcpy(nb, h->normbuf, 12, cudaMemcpyDeviceToHost));
    *h_norm = nb[0];
    if (nb[2] == 0.f) return set_err(h, GPT2_ENONFINITE, "non-finite gradient norm: update skipped");
  }
  return GPT2_OK;
}

int gpt2_train_step(gpt2_t* h, const int32_t* h_tok, const int32_t* h_tgt, int n_micro, int B, int T, float lr,
                    float wd, float b1, float b2, float eps, float clip, float* h_loss, float* h_norm) {
  if (h == nullptr) return GPT2_EINVAL;
  if (h_tok == nullptr || h_tgt == nullptr || n_micro < 1) return set_err(h, GPT2_EINVAL, "bad train_step arguments");
  if (B < 1 || T < 1 || B > h->maxB || T > h->maxT) return set_err(h, GPT2_EINVAL, "B or T out of range");
  const long M = (long)B * T;
  RET_IF(clear_accumulators(h));
  CU_CHECK(h, cudaMemsetAsync(h->grads, 0, h->nparams * 4, h->stream));
  CU_CHECK(h, cudaMemsetAsync(h->d_loss + 1, 0, 4, h->stream));
  const float scale = 1.f / (float)n_micro;
  for (int k = 0; k < n_micro; ++k) {
    CU_CHECK(h, cudaMemcpyAsync(h->tok_dev, h_tok + k * M, M * 4, cudaMemcpyHostToDevice, h->stream));
    CU_CHECK(h, cudaMemcpyAsync(h->tgt_dev, h_tgt + k * M, M * 4, cudaMemcpyHostToDevice, h->stream));
    RET_IF(fused_micro_step(h, h->tok_dev, h->tgt_dev, B, T, scale));
  }
  RET_IF(adamw_impl(h, lr, wd, b1, b2, eps, clip));
  if (h_loss || h_norm) {
    RET_IF(check_device_flags(h));
    float nb[3];
    CU_CHECK(h, cudaMemcpy(nb, h->normbuf, 12, cudaMemcpyDeviceToHost));
    if (h_norm) *h_norm = nb[0];
    if (h_loss) CU_CHECK(h, cudaMemcpy(h_loss, h->d_loss + 1, 4, cudaMemcpyDeviceToHost));
    if (nb[2] == 0.f) return set_err(h, GPT2_ENONFINITE, "non-finite gradient norm: update skipped");
  }
  return GPT2_OK;
}

double gpt2_lr_at(int it, double max_lr, double min_lr, int warmup, int max_steps) {
  if (it < warmup) return max_lr * (it + 1) / warmup;
  if (it > max_steps) return min_lr;
  const double ratio = (double)(it - warmup) / (double)(max_steps - warmup);
  const double coeff = 0.5 * (1.0 + cos(M_PI * ratio));
  return min_lr + coeff * (max_lr - min_lr);
}

int64_t gpt2_num_params(const gpt2_t* h) { return h ? (int64_t)h->nparams : -1; }

int gpt2_get_params(gpt2_t* h, float* dst) {
  if (h == nullptr || dst == nullptr) return GPT2_EINVAL;
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  CU_CHECK(h, cudaMemcpy(dst, h->params, h->nparams * 4, cudaMemcpyDeviceToHost));
  return GPT2_OK;
}

int gpt2_set_params(gpt2_t* h, const float* src) {
  if (h == nullptr || src == nullptr) return GPT2_EINVAL;
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  CU_CHECK(h, cudaMemcpy(h->params, src, h->nparams * 4, cudaMemcpyHostToDevice));
  RET_IF(refresh_bf16(h));
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  return GPT2_OK;
}

int gpt2_get_grads(gpt2_t* h, float* dst) {
  if (h == nullptr || dst == nullptr) return GPT2_EINVAL;
  RET_IF(fold_accumulators(h));
  RET_IF(check_device_flags(h));
  CU_CHECK(h, cudaMemcpy(dst, h->grads, h->nparams * 4, cudaMemcpyDeviceToHost));
  return GPT2_OK;
}

int gpt2_get_adam_state(gpt2_t* h, float* hm, float* hv, int64_t* step) {
  if (h == nullptr) return GPT2_EINVAL;
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  if (hm) CU_CHECK(h, cudaMemcpy(hm, h->m, h->nparams * 4, cudaMemcpyDeviceToHost));
  if (hv) CU_CHECK(h, cudaMemcpy(hv, h->v, h->nparams * 4, cudaMemcpyDeviceToHost));
  if (step) {
    long long t = 0;
    CU_CHECK(h, cudaMemcpy(&t, h->d_step, 8, cudaMemcpyDeviceToHost));
    *step = t;
  }
  return GPT2_OK;
}

int gpt2_set_adam_state(gpt2_t* h, const float* hm, const float* hv, int64_t step) {
  if (h == nullptr || hm == nullptr || hv == nullptr || step < 0) return GPT2_EINVAL;
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  CU_CHECK(h, cudaMemcpy(h->m, hm, h->nparams * 4, cudaMemcpyHostToDevice));
  CU_CHECK(h, cudaMemcpy(h->v, hv, h->nparams * 4, cudaMemcpyHostToDevice));
  long long t = step;
  CU_CHECK(h, cudaMemcpy(h->d_step, &t, 8, cudaMemcpyHostToDevice));
  return GPT2_OK;
}

int gpt2_get_logits(gpt2_t* h, float* dst) {
  if (h == nullptr || dst == nullptr) return GPT2_EINVAL;
  if (!h->have_fwd || !h->logits_valid) return set_err(h, GPT2_ESTATE, "no valid logits (none computed, or consumed)");
  RET_IF(check_device_flags(h));
  const size_t n = (size_t)h->M() * h->Vp;
  if (h->prec == GPT2_BF16) {
    std::vector<uint16_t> tmp(n);
    CU_CHECK(h, cudaMemcpy(tmp.data(), h->logits, n * 2, cudaMemcpyDeviceToHost));
    for (size_t i = 0; i < n; ++i) {
      uint32_t u = (uint32_t)tmp[i] << 16;
      memcpy(dst + i, &u, 4);
    }
  } else {
    CU_CHECK(h, cudaMemcpy(dst, h->logits, n * 4, cudaMemcpyDeviceToHost));
  }
  return GPT2_OK;
}

int gpt2_get_argmax(gpt2_t* h, int32_t* dst) {
  if (h == nullptr || dst == nullptr) return GPT2_EINVAL;
  if (!h->have_fwd) return set_err(h, GPT2_ESTATE, "no forward yet");
  RET_IF(check_device_flags(h));
  CU_CHECK(h, cudaMemcpy(dst, h->argmax, h->M() * 4, cudaMemcpyDeviceToHost));
  return GPT2_OK;
}

int gpt2_get_losses(gpt2_t* h, float* dst) {
  if (h == nullptr || dst == nullptr) return GPT2_EINVAL;
  if (!h->have_fwd) return set_err(h, GPT2_ESTATE, "no forward yet");
  RET_IF(check_device_flags(h));
  CU_CHECK(h, cudaMemcpy(dst, h->losses, h->M() * 4, cudaMemcpyDeviceToHost));
  return GPT2_OK;
}

int gpt2_last_loss(gpt2_t* h, float* loss) {
  if (h == nullptr || loss == nullptr) return GPT2_EINVAL;
  if (!h->have_fwd) return set_err(h, GPT2_ESTATE, "no forward yet");
  RET_IF(check_device_flags(h));
  CU_CHECK(h, cudaMemcpy(loss, h->d_loss, 4, cudaMemcpyDeviceToHost));
  return GPT2_OK;
}

int gpt2_get_embed_keys(gpt2_t* h, uint32_t* dst) {
  if (h == nullptr || dst == nullptr) return GPT2_EINVAL;
  if (!h->have_bwd_keys) return set_err(h, GPT2_ESTATE, "no backward yet");
  RET_IF(check_device_flags(h));
  CU_CHECK(h, cudaMemcpy(dst, h->emb_keys, h->M() * 4, cudaMemcpyDeviceToHost));
  return GPT2_OK;
}

int64_t gpt2_kernel_launches(const gpt2_t* h) { return h ? h->launches : -1; }

int gpt2_check_guards(gpt2_t* h, int64_t* n_bad) {
  if (h == nullptr || n_bad == nullptr) return GPT2_EINVAL;
  if (cudaStreamSynchronize(h->stream) != cudaSuccess) return set_err(h, GPT2_ECUDA, "stream synchronise");
  if (h->side_stream && cudaStreamSynchronize(h->side_stream) != cudaSuccess)
    return set_err(h, GPT2_ECUDA, "stream synchronise");
  int64_t bad = 0;
  unsigned char buf[GUARD_BYTES];
  for (const auto& g : h->guards) {
    if (cudaMemcpy(buf, static_cast<const uint8_t*>(g.first) + g.second, GUARD_BYTES, cudaMemcpyDeviceToHost) !=
        cudaSuccess)
      return set_err(h, GPT2_ECUDA, "guard read");
    for (size_t i = 0; i < GUARD_BYTES; ++i) bad += buf[i] != GUARD_BYTE;
  }
  *n_bad = bad;
  return GPT2_OK;
}

int gpt2_debug_overwrite_guard(gpt2_t* h, int index) {
  if (h == nullptr || index < 0 || index >= (int)h->guards.size()) return GPT2_EINVAL;
  const auto& g = h->guards[index];
  return cudaMemset(static_cast<uint8_t*>(g.first) + g.second, 0, 1) == cudaSuccess ? GPT2_OK : GPT2_ECUDA;
}

int gpt2_set_graphs(gpt2_t* h, int enable) {
  if (h == nullptr) return GPT2_EINVAL;
  h->use_graphs = enable != 0;
  return GPT2_OK;
}

int gpt2_set_timing(gpt2_t* h, int enable) {
  if (h == nullptr) return GPT2_EINVAL;
  h->timing = enable != 0;
  return GPT2_OK;
}

int gpt2_get_timing(gpt2_t* h, double* ms, int64_t* ops, double* flops, double* bytes) {
  if (h == nullptr) return GPT2_EINVAL;
  CU_CHECK(h, cudaStreamSynchronize(h->stream));
  double t[GPT2_NUM_KCLASSES] = {};
  int64_t n[GPT2_NUM_KCLASSES] = {};
  for (size_t i = 0; i < h->ev_used; ++i) {
    float e = 0.f;
    CU_CHECK(h, cudaEventElapsedTime(&e, h->ev_pool[2 * i], h->ev_pool[2 * i + 1]));
    t[h->ev_class[i]] += e;
    n[h->ev_class[i]]++;
  }
  for (int c = 0; c < GPT2_NUM_KCLASSES; ++c) {
    if (ms) ms[c] = t[c];
    if (ops) ops[c] = n[c];
    if (flops) flops[c] = h->t_flops[c];
    if (bytes) bytes[c] = h->t_bytes[c];
    h->t_flops[c] = h->t_bytes[c] = 0.0;
  }
  h->ev_used = 0;
  return GPT2_OK;
}

const char* gpt2_last_error(const gpt2_t* h) { return h ? h->err.c_str() : g_null_handle_err.c_str(); }

// ------------------------------------------------------------ standalone ops
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// The attention kernels launch one grid row per (batch, head): grid.y = B*H.
static bool attn_sizes_ok(int B, int T, int H) {
  return B >= 1 && T >= 1 && H >= 1 && (long)B * H <= 65535L && (long)B * T * 3 * 64 * H < (1L << 31);
}

int gpt2_attention_forward(const void* qkv, void* out, float* lse, int B, int T, int H, void* stream) {
  if (!qkv || !out || !lse || !attn_sizes_ok(B, T, H)) return GPT2_EINVAL;
  if (!aligned16(qkv) || !aligned16(out)) return GPT2_EINVAL;
  return tcfa::forward((const bf16*)qkv, (bf16*)out, lse, B, T, H, (cudaStream_t)stream) == cudaSuccess
             ? GPT2_OK
             : GPT2_ECUDA;
}

int64_t gpt2_attention_workspace_floats(int B, int T, int H) {
  if (B < 1 || T < 1 || H < 1) return 0;
  // lse*log2(e) and D rows, then the bf16 dS tiles (1 KB aligned)
  return (int64_t)tcfa::backward_scratch_floats(B, T, H) + (tcfa::backward_ds_elems(B, T, H) + 1) / 2;
}

int gpt2_attention_backward(const void* qkv, const void* out, const void* dout, const float* lse, void* dqkv,
                            float* work, int B, int T, int H, void* stream) {
  if (!qkv || !out || !dout || !lse || !dqkv || !work || !attn_sizes_ok(B, T, H)) return GPT2_EINVAL;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(dout) || !aligned16(dqkv) || !aligned16(work))
    return GPT2_EINVAL;
  bf16* ds = reinterpret_cast<bf16*>(work + tcfa::backward_scratch_floats(B, T, H));
  return tcfa::backward((const bf16*)qkv, (const bf16*)out, (const bf16*)dout, lse, (bf16*)dqkv, work, B, T, H,
                        (cudaStream_t)stream, nullptr, ds) == cudaSuccess
             ? GPT2_OK
             : GPT2_ECUDA;
}

int gpt2_matmul_bf16(const void* A, int64_t lda, int a_mn, const void* Bm, int64_t ldb, int b_mn, int M, int N, int K,
                     int epi, const float* bias, const float* resid, void* out, void* out2, const void* aux,
                     int64_t ldc, float* work, size_t work_bytes, void* stream) {
  if (!A || !Bm || !out || epi < 0 || epi > 5) return GPT2_EINVAL;
  if ((epi == 2 && !resid) || (epi == 3 && !out2) || (epi == 4 && !aux)) return GPT2_EINVAL;
  tcg::GemmArgs g;
  g.A = (const bf16*)A;
  g.lda = lda;
  g.a_mn = a_mn ? 1 : 0;
  g.B = (const bf16*)Bm;
  g.ldb = ldb;
  g.b_mn = b_mn ? 1 : 0;
  g.M = M;
  g.N = N;
  g.K = K;
  g.epi = epi;
  g.bias = bias;
  g.resid = resid;
  g.out = out;
  g.out2 = (bf16*)out2;
  g.aux = (const bf16*)aux;
  g.ldc = ldc;
  g.workspace = work;
  g.workspace_bytes = work_bytes;
  const int r = tcg::gemm(g, (cudaStream_t)stream);
  return r == 0 ? GPT2_OK : (r == -1 ? GPT2_EINVAL : GPT2_ECUDA);
}

size_t gpt2_matmul_workspace_bytes(int M, int N, int K) { return tcg::splitk_workspace_bytes(M, N, K, 0); }

int gpt2_attention_backward_noalloc(const void* qkv, const void* out, const void* dout, const float* lse, void* dqkv,
                                    int B, int T, int H, void* stream) {
  if (!qkv || !out || !dout || !lse || !dqkv || !attn_sizes_ok(B, T, H)) return GPT2_EINVAL;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(dout) || !aligned16(dqkv)) return GPT2_EINVAL;
  if (tcfa::backward_scratch_floats(B, T, H) > 2L * GPT2_ATTN_NOALLOC_MAX_ROWS) return GPT2_EINVAL;
  float* scratch = noalloc_scratch_on_current_device();
  if (scratch == nullptr) return GPT2_ECUDA;
  return tcfa::backward((const bf16*)qkv, (const bf16*)out, (const bf16*)dout, lse, (bf16*)dqkv, scratch, B, T,
                              H, (cudaStream_t)stream) == cudaSuccess
             ? GPT2_OK
             : GPT2_ECUDA;
}

int gpt2_check_device_error(void* stream) {
  const cudaError_t se = cudaStreamSynchronize((cudaStream_t)stream);
  if (se != cudaSuccess) {
    cudaGetLastError();
    return GPT2_ECUDA;
  }
  int derr = 0;
  if (cudaMemcpyFromSymbol(&derr, g_device_err, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return GPT2_ECUDA;
  }
  if (derr == 0) return GPT2_OK;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_err, &zero, sizeof(int)) != cudaSuccess) cudaGetLastError();
  return GPT2_ECUDA;
}

int gpt2_set_wait_limit_ns(uint64_t limit_ns) {
  const unsigned long long v = limit_ns == 0 ? DEFAULT_WAIT_LIMIT_NS : (unsigned long long)limit_ns;
  if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return GPT2_ECUDA;
  }
  return GPT2_OK;
}

int gpt2_prefill(gpt2_t* h, const int32_t* d_tokens, int B, int T0, float temperature, int top_k, uint64_t seed,
                 int32_t* d_next) {
  if (h == nullptr) return GPT2_EINVAL;
  return prefill_impl(h, d_tokens, B, T0, temperature, top_k, seed, d_next);
}

int gpt2_decode_step(gpt2_t* h, const int32_t* d_tokens, int B, int pos, float temperature, int top_k, uint64_t seed,
                     int32_t* d_next) {
  if (h == nullptr) return GPT2_EINVAL;
  return decode_impl(h, d_tokens, B, pos, temperature, top_k, seed, d_next);
}

int gpt2_get_decode_logits(gpt2_t* h, float* dst) {
  if (h == nullptr || dst == nullptr) return GPT2_EINVAL;
  if (h->gen_B == 0) return set_err(h, GPT2_ESTATE, "no prefill yet");
  RET_IF(check_device_flags(h));
  const size_t n = (size_t)h->gen_B * h->Vp;
  std::vector<uint16_t> tmp(n);
  CU_CHECK(h, cudaMemcpy(tmp.data(), h->dec_logits, n * 2, cudaMemcpyDeviceToHost));
  for (size_t i = 0; i < n; ++i) {
    const uint32_t u = (uint32_t)tmp[i] << 16;
    memcpy(dst + i, &u, 4);
  }
  return GPT2_OK;
}

}  // extern "C"
