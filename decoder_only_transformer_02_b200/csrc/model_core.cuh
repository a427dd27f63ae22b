// Host-side runtime of the GPT-2 step: the handle, its device arenas and the
// per-layer views into them.  Included by libgpt2.cu (single translation unit).
#pragma once
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/gpt2.h"
#include "attention.cuh"
#include "common.cuh"
#include "kernels.cuh"
#include "simt_gemm.cuh"
#include "tc_gemm.h"

struct TensorInfo {
  std::string name;
  size_t offset;
  size_t numel;
  int rows, cols;  // cols == 0 for 1-D tensors
  int decay;
};

static const size_t NO_OFF = (size_t)-1;  // no parameter

struct LayerOffsets {
  size_t ln1g, ln1b, attnw, attnb, projw, projb, ln2g, ln2b, fcw, fcb, mpw, mpb;
};

struct gpt2 {
  gpt2_config cfg{};
  int L = 0, H = 0, C = 0, V = 0, Vp = 0, P = 0, maxB = 0, maxT = 0, prec = 0;
  size_t es = 4;  // bytes per activation element (2 in bf16 mode)
  cudaStream_t stream = nullptr;
  std::string err = "ok";
  // guard bytes after every device allocation: (allocation, offset of its guard)
  std::vector<std::pair<void*, size_t>> guards;
  int64_t launches = 0;

  // parameters, flat
  std::vector<TensorInfo> tensors;
  std::vector<LayerOffsets> lo;
  size_t wte = 0, wpe = 0, lnfg = 0, lnfb = 0;
  size_t nparams = 0;
  float *params = nullptr, *grads = nullptr, *m = nullptr, *v = nullptr;
  bf16* pbf = nullptr;  // bf16 copy of the weights (bf16 mode)
  int64_t adam_t = 0;

  // activations (element type: bf16 in bf16 mode, fp32 otherwise, unless noted)
  float* res = nullptr;  // fp32 residual stream, (2L+1) points x [M, C]
  uint8_t *ln1 = nullptr, *ln2 = nullptr;
  float *ln1_mean = nullptr, *ln1_rstd = nullptr, *ln2_mean = nullptr, *ln2_rstd = nullptr;
  uint8_t *qkv = nullptr, *att = nullptr, *fcu = nullptr, *fca = nullptr, *lnf = nullptr, *logits = nullptr;
  float *lse = nullptr, *lnf_mean = nullptr, *lnf_rstd = nullptr;
  float *ce_lse = nullptr, *losses = nullptr, *d_loss = nullptr;
  float* ce_part = nullptr;  // lm_head softmax statistics per (row, 128 columns) (bf16 mode)
  bf16* attn_ds = nullptr;   // the attention backward's dS tiles, one layer at a time (bf16 mode)
  int32_t* argmax = nullptr;

  // backward scratch
  float *dres = nullptr, *dln = nullptr, *attn_D = nullptr;
  bf16* dres_bf = nullptr;
  uint8_t *dbig = nullptr, *dqkv = nullptr, *datt = nullptr;
  // bf16 weight gradients of the layers' linear weights accumulate over K
  // splits into one buffer per split (no per-call reduction); they are folded
  // into grads, in split order, before anything reads the gradients
  struct WgradSlots {
    size_t woff;  // the weight's offset in the parameter arena
    float* ptr;   // [splits][n]
    int splits;
    long n;
  };
  std::vector<WgradSlots> wslots;
  float* slot_buf = nullptr;
  size_t slot_floats = 0;
  // per-block partial column sums (LayerNorm dgamma / dbeta / bias of the
  // projection feeding the residual point, the fc and qkv biases) likewise
  // accumulate over the micro-steps in one buffer per use, and are reduced in
  // row order with the fold.  Index: 2l / 2l+1 LayerNorm 1 / 2 of layer l,
  // 2L the final LayerNorm, 2L+1+l the fc bias, 3L+1+l the qkv bias of layer l.
  struct PartialSums {
    float* buf;     // [rows][ncols]
    int rows, ncols, C;
    size_t off[3];  // column j sums into grads[off[j / C] + j % C] (NO_OFF: dropped)
  };
  std::vector<PartialSums> psums;
  float* psum_buf = nullptr;
  size_t psum_floats = 0;
  bool accum_dirty = false;  // the accumulators hold sums not yet folded into grads
  uint32_t* emb_keys = nullptr;
  float* emb_part = nullptr;
  int sort_cap = 0;

  // optimizer
  float* normbuf = nullptr;  // [norm, clip scale, finite flag, 1-b1^t, 1-b2^t]
  long long* d_step = nullptr;  // AdamW step counter t (device)
  double* norm_part = nullptr;
  int norm_blocks = 0;
  k::AdamSeg* segs = nullptr;
  int nseg = 0;

  int* d_bad = nullptr;  // token-range flag
  int32_t *tok_dev = nullptr, *tgt_dev = nullptr;

  // state of the last forward
  int B = 0, T = 0;
  bool have_fwd = false, have_targets = false, logits_valid = false, have_bwd_keys = false;

  // generation (bf16 mode): KV cache [L][max_B][block][2C] (k then v) and the
  // per-step activations of up to max_B sequences, allocated on first use
  bf16* kv = nullptr;
  float *dec_x = nullptr, *dec_mean = nullptr, *dec_rstd = nullptr;
  bf16 *dec_ln = nullptr, *dec_qkv = nullptr, *dec_att = nullptr, *dec_u = nullptr, *dec_a = nullptr;
  bf16* dec_logits = nullptr;  // [max_B, Vp] logits of the last prefill / decode step
  int gen_B = 0, gen_len = 0;  // sequences and positions held in the cache
  const int32_t* last_tok = nullptr;
  const int32_t* last_tgt = nullptr;

  // CUDA graphs of the fused micro-step, one per (B, T, loss scale)
  struct GraphEntry {
    int B, T;
    uint32_t scale_bits;
    int state;  // 0: seen once (ran eagerly), 1: captured, -1: capture failed
    cudaGraphExec_t exec;
    int64_t nlaunch;
  };
  std::vector<GraphEntry> graphs;
  bool use_graphs = true;
  cudaStream_t cap_stream = nullptr;
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
  // the embedding backward's key sort runs beside the cross-entropy pass on side_stream
  cudaStream_t side_stream = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_sorted = nullptr;
  bool sort_pending = false;

  // opt-in per-class device timing (measurement support)
  bool timing = false;
  std::vector<cudaEvent_t> ev_pool;   // 2 events per timed operation
  std::vector<int> ev_class;          // class of each timed operation
  size_t ev_used = 0;                 // operations recorded since the last read
  double t_flops[GPT2_NUM_KCLASSES] = {}, t_bytes[GPT2_NUM_KCLASSES] = {};

  long M() const { return (long)B * T; }
  long Mmax() const { return (long)maxB * maxT; }
  float* P32(size_t off) { return params + off; }
  float* G32(size_t off) { return grads + off; }
  const bf16* PBF(size_t off) { return pbf + off; }
};

static int set_err(gpt2* h, int code, const std::string& msg) {
  if (h) h->err = msg;
  return code;
}

#define CU_CHECK(h, call)                                                                         \
  do {                                                                                            \
    cudaError_t e_ = (call);                                                                      \
    if (e_ != cudaSuccess) {                                                                      \
      cudaGetLastError(); /* clear a non-sticky error so the handle stays usable */              \
      return set_err((h), GPT2_ECUDA, std::string(#call) + ": " + cudaGetErrorString(e_));       \
    }                                                                                             \
  } while (0)

#define LAUNCH_CHECK(h)                                                                           \
  do {                                                                                            \
    (h)->launches++;                                                                              \
    cudaError_t e_ = cudaGetLastError();                                                          \
    if (e_ != cudaSuccess)                                                                        \
      return set_err((h), GPT2_ECUDA,                                                             \
                     std::string("launch at ") + __FILE__ + ":" + std::to_string(__LINE__) + ": " +  \
                         cudaGetErrorString(e_));                                                 \
  } while (0)

static int grid_for(long n, int threads, int cap_per_sm = 8) {
  long b = (n + threads - 1) / threads;
  long cap = 148L * cap_per_sm;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return (int)b;
}

static void build_tensor_table(gpt2* h) {
  h->tensors.clear();
  h->lo.assign(h->L, LayerOffsets{});
  size_t off = 0;
  auto add = [&](const std::string& n, int rows, int cols, int decay) -> size_t {
    TensorInfo t;
    t.name = n;
    t.offset = off;
    t.rows = rows;
    t.cols = cols;
    t.numel = (size_t)rows * (cols ? cols : 1);
    t.decay = decay;
    h->tensors.push_back(t);
    off += t.numel;
    return t.offset;
  };
  const int C = h->C;
  h->wte = add("wte", h->Vp, C, 1);
  h->wpe = add("wpe", h->P, C, 1);
  for (int l = 0; l < h->L; ++l) {
    const std::string p = "h" + std::to_string(l) + ".";
    LayerOffsets& o = h->lo[l];
    o.ln1g = add(p + "ln1.g", C, 0, 0);
    o.ln1b = add(p + "ln1.b", C, 0, 0);
    o.attnw = add(p + "attn.w", 3 * C, C, 1);
    o.attnb = add(p + "attn.b", 3 * C, 0, 0);
    o.projw = add(p + "proj.w", C, C, 1);
    o.projb = add(p + "proj.b", C, 0, 0);
    o.ln2g = add(p + "ln2.g", C, 0, 0);
    o.ln2b = add(p + "ln2.b", C, 0, 0);
    o.fcw = add(p + "fc.w", 4 * C, C, 1);
    o.fcb = add(p + "fc.b", 4 * C, 0, 0);
    o.mpw = add(p + "mproj.w", C, 4 * C, 1);
    o.mpb = add(p + "mproj.b", C, 0, 0);
  }
  h->lnfg = add("lnf.g", C, 0, 0);
  h->lnfb = add("lnf.b", C, 0, 0);
  h->nparams = off;
}

// Every device allocation is rounded up to 256 bytes and followed by
// GUARD_BYTES of GUARD_BYTE: a kernel that writes past the end of a buffer
// changes them, and gpt2_check_guards reports it.
constexpr size_t GUARD_BYTES = 256;
constexpr unsigned char GUARD_BYTE = 0xA5;
static int dev_alloc(gpt2* h, void** p, size_t bytes) {
  const size_t body = ((bytes == 0 ? 16 : bytes) + 255) & ~size_t(255);
  cudaError_t e = cudaMalloc(p, body + GUARD_BYTES);
  if (e == cudaSuccess) e = cudaMemset(static_cast<uint8_t*>(*p) + body, GUARD_BYTE, GUARD_BYTES);
  if (e != cudaSuccess) {
    if (*p) cudaFree(*p);
    *p = nullptr;
    return set_err(h, GPT2_ENOMEM, std::string("cudaMalloc(") + std::to_string(bytes) + "): " + cudaGetErrorString(e));
  }
  h->guards.emplace_back(*p, body);
  return GPT2_OK;
}
#define ALLOC(h, ptr, bytes)                                                    \
  do {                                                                          \
    int r_ = dev_alloc((h), reinterpret_cast<void**>(&(ptr)), (size_t)(bytes)); \
    if (r_ != GPT2_OK) return r_;                                               \
  } while (0)

static void free_all(gpt2* h) {
  void* ptrs[] = {h->params,  h->grads,   h->m,        h->v,        h->pbf,      h->res,      h->ln1,
                  h->ln2,     h->ln1_mean, h->ln1_rstd, h->ln2_mean, h->ln2_rstd, h->qkv,      h->att,
                  h->fcu,     h->fca,     h->lnf,      h->logits,   h->lse,      h->lnf_mean, h->lnf_rstd,
                  h->ce_lse,  h->losses,  h->d_loss,   h->argmax,   h->dres,     h->dln,      h->attn_D,
                  h->psum_buf, h->dres_bf,  h->dbig,     h->dqkv,     h->datt,     h->slot_buf,
                  h->emb_keys, h->emb_part, h->normbuf, h->d_step, h->norm_part, h->segs,    h->d_bad,    h->tok_dev,
                  h->tgt_dev, h->ce_part, h->attn_ds, h->kv, h->dec_x, h->dec_mean, h->dec_rstd, h->dec_ln,
                  h->dec_qkv, h->dec_att, h->dec_u, h->dec_a, h->dec_logits};
  for (void* p : ptrs)
    if (p) cudaFree(p);
}

// rows handled per CTA by the LayerNorm backward: one CTA per SM, a whole
// number of stages of k::LN_BWD_WARPS rows
static int ln_rows_per_block(long M) {
  long r = (M + 147) / 148;
  r = (r + k::LN_BWD_WARPS - 1) / k::LN_BWD_WARPS * k::LN_BWD_WARPS;
  return (int)r;
}
// rows per CTA of the column-sum kernel: at most 64 row blocks
static int colsum_rows_per_block(long M) {
  long r = (M + 63) / 64;
  return (int)(r < 64 ? 64 : r);
}

// Times one operation (all launches in its scope) when timing is enabled.
struct KTimer {
  gpt2* h;
  int cls;
  bool on;
  KTimer(gpt2* hh, int c, double flops, double bytes) : h(hh), cls(c), on(hh->timing) {
    if (!on) return;
    if (h->ev_used * 2 + 2 > h->ev_pool.size()) {
      for (int i = 0; i < 2; ++i) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) {
          on = false;
          return;
        }
        h->ev_pool.push_back(e);
      }
      h->ev_class.push_back(c);
    }
    h->ev_class[h->ev_used] = c;
    cudaEventRecord(h->ev_pool[h->ev_used * 2], h->stream);
    h->t_flops[c] += flops;
    h->t_bytes[c] += bytes;
  }
  ~KTimer() {
    if (!on) return;
    cudaEventRecord(h->ev_pool[h->ev_used * 2 + 1], h->stream);
    h->ev_used++;
  }
};
enum KClass { KC_GEMM = 0, KC_ATTN_F, KC_ATTN_B, KC_LN_F, KC_LN_B, KC_CE, KC_OPT, KC_EMB, KC_OTHER };
