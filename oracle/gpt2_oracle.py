"""CPU oracle for one GPT-2 training step.  TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module.  The product
path (the CUDA library and its Python binding) never imports, calls or links it,
and this module imports nothing from the product package.

It is a plain, slow, explicit NumPy restatement of what one training step
computes: every formula is written out, nothing is fused, blocked or reordered
beyond what the definition states, and there is no autograd.  The default
precision is float64; float32 is accepted for large shapes and for the timed CPU
baseline.

Sources (titles of the pages the method is described on):
  [V]  "Let's reproduce GPT-2 (124M)" -- video summary, Key Takeaways bullets
       (architecture; optimization hyperparameters; gradient accumulation;
       weight tying and vocab padding).
  [C]  "Let's reproduce GPT-2 (124M)" -- video page, Chapters list (cross
       entropy loss; parameter sharing wte and lm_head; model initialization
       std 0.02 + residual init; AdamW and gradient clipping; learning rate
       scheduler warmup + cosine decay; gradient accumulation).
  [D]  "From Scratch: Building GPT-2 for Efficient Language Modeling" -- Key
       Features list and Training Setup table (iterations 19073, warmup 715,
       total batch 524,288, vocab 50304, AdamW betas/eps).

Where the pages are silent the plainest reading is taken; each one is marked
"reading:" at the function that makes it.

Parity status: every function below is pinned by a CPU test (closed forms,
finite differences, textbook library reductions, the pages' printed numbers).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# --------------------------------------------------------------------------
# configuration
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class Config:
    n_layer: int = 12
    n_head: int = 12
    n_embd: int = 768
    vocab_size: int = 50257      # real token ids live in [0, vocab_size)
    padded_vocab: int = 50304    # rows of wte / columns of the logits
    block_size: int = 1024       # rows of wpe (max sequence length)

    @property
    def head_dim(self) -> int:
        return self.n_embd // self.n_head


# [V] architecture bullet: 12 layers, 768 channels, vocab 50,257, seq 1024;
# [V] weight tying & padding bullet: 50257 -> 50304.
GPT2_124M = Config()
# tiny fp32 parity model (layer/width/vocab shrunk, same structure)
TINY = Config(n_layer=2, n_head=4, n_embd=128, vocab_size=512, padded_vocab=512, block_size=64)

LN_EPS = 1e-5  # reading: the pages name LayerNorm but no epsilon; the usual 1e-5, biased variance.


def param_specs(cfg: Config):
    """Flat parameter order: list of (name, shape, decayed).

    [V] architecture bullet (pre-norm blocks, extra final LayerNorm, GELU MLP),
    [V] weight tying bullet (one matrix serves as token embedding and lm_head,
    so it appears once).  Linear weights are stored [out, in].
    reading: every Linear in a block carries a bias and the lm_head has none;
    the closed-form count 124,439,808 at vocab 50257 pins this.
    [V] hyperparameter bullet: weight decay only on 2D tensors (embeddings and
    matrices), never on biases or LayerNorm parameters.
    """
    C, V, P = cfg.n_embd, cfg.padded_vocab, cfg.block_size
    specs = [("wte", (V, C), True), ("wpe", (P, C), True)]
    for l in range(cfg.n_layer):
        specs += [
            (f"h{l}.ln1.g", (C,), False), (f"h{l}.ln1.b", (C,), False),
            (f"h{l}.attn.w", (3 * C, C), True), (f"h{l}.attn.b", (3 * C,), False),
            (f"h{l}.proj.w", (C, C), True), (f"h{l}.proj.b", (C,), False),
            (f"h{l}.ln2.g", (C,), False), (f"h{l}.ln2.b", (C,), False),
            (f"h{l}.fc.w", (4 * C, C), True), (f"h{l}.fc.b", (4 * C,), False),
            (f"h{l}.mproj.w", (C, 4 * C), True), (f"h{l}.mproj.b", (C,), False),
        ]
    specs += [("lnf.g", (C,), False), ("lnf.b", (C,), False)]
    return specs


def num_params(cfg: Config) -> int:
    return int(sum(int(np.prod(s)) for _, s, _ in param_specs(cfg)))


def unflatten(flat: np.ndarray, cfg: Config) -> dict:
    """Views (not copies) of the flat vector, keyed by parameter name."""
    out, off = {}, 0
    for name, shape, _ in param_specs(cfg):
        n = int(np.prod(shape))
        out[name] = flat[off:off + n].reshape(shape)
        off += n
    assert off == flat.size, (off, flat.size)
    return out


def decay_mask(cfg: Config, dtype=np.float64) -> np.ndarray:
    """1 where a flat parameter is weight-decayed, 0 elsewhere."""
    parts = [np.full(int(np.prod(s)), 1.0 if d else 0.0, dtype=dtype) for _, s, d in param_specs(cfg)]
    return np.concatenate(parts)


def init_params(cfg: Config, seed: int, dtype=np.float64) -> np.ndarray:
    """[C] chapter "model initialization: std 0.02, residual init".

    reading: all matrices and both embeddings ~ N(0, 0.02) (the padded wte rows
    included); the two projections that write into the residual stream
    (attention output projection, MLP output projection) ~ N(0, 0.02/sqrt(2L));
    biases 0; LayerNorm gain 1 and shift 0.
    """
    rng = np.random.default_rng(seed)
    flat = np.zeros(num_params(cfg), dtype=dtype)
    p = unflatten(flat, cfg)
    resid_std = 0.02 / math.sqrt(2 * cfg.n_layer)
    for name, shape, _ in param_specs(cfg):
        if name.endswith(".g"):
            p[name][...] = 1.0
        elif name.endswith(".b"):
            p[name][...] = 0.0
        elif name.endswith("proj.w"):            # attn proj and mlp proj
            p[name][...] = rng.normal(0.0, resid_std, size=shape)
        else:                                    # wte, wpe, attn.w, fc.w
            p[name][...] = rng.normal(0.0, 0.02, size=shape)
    return flat


# --------------------------------------------------------------------------
# building blocks (each written out from its definition)
# --------------------------------------------------------------------------

def layernorm_forward(x, g, b, eps=LN_EPS):
    """y = (x - mean) / sqrt(var + eps) * g + b over the last axis (biased var).
    [V] architecture bullet: LayerNorm before attention, before the MLP and once
    more before the classifier."""
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (x - mean) * rstd
    return xhat * g + b, mean[..., 0], rstd[..., 0]


def layernorm_backward(dy, x, mean, rstd, g):
    """Chain rule through layernorm_forward.
    dxhat = dy*g ; dx = rstd*(dxhat - mean(dxhat) - xhat*mean(dxhat*xhat));
    dg = sum_rows dy*xhat ; db = sum_rows dy."""
    xhat = (x - mean[..., None]) * rstd[..., None]
    dxhat = dy * g
    dx = rstd[..., None] * (dxhat - dxhat.mean(axis=-1, keepdims=True)
                            - xhat * (dxhat * xhat).mean(axis=-1, keepdims=True))
    dg = (dy * xhat).reshape(-1, x.shape[-1]).sum(axis=0)
    db = dy.reshape(-1, x.shape[-1]).sum(axis=0)
    return dx, dg, db


GELU_K = math.sqrt(2.0 / math.pi)
GELU_A = 0.044715


def gelu_tanh(u):
    """[V] architecture bullet: GELU (the historical tanh approximation).
    gelu(u) = 0.5*u*(1 + tanh(sqrt(2/pi)*(u + 0.044715*u^3)))."""
    return 0.5 * u * (1.0 + np.tanh(GELU_K * (u + GELU_A * u ** 3)))


def gelu_tanh_grad(u):
    """d gelu / du = 0.5*(1+th) + 0.5*u*(1-th^2)*sqrt(2/pi)*(1+3*0.044715*u^2)."""
    th = np.tanh(GELU_K * (u + GELU_A * u ** 3))
    return 0.5 * (1.0 + th) + 0.5 * u * (1.0 - th * th) * GELU_K * (1.0 + 3.0 * GELU_A * u * u)


def linear_forward(x, w, b=None):
    """y = x @ w^T (+ b); w is stored [out, in]."""
    y = x @ w.T
    return y if b is None else y + b


def linear_backward(dy, x, w):
    """dx = dy @ w ; dw = dy^T @ x ; db = column sums of dy."""
    x2 = x.reshape(-1, x.shape[-1])
    dy2 = dy.reshape(-1, dy.shape[-1])
    return (dy @ w), dy2.T @ x2, dy2.sum(axis=0)


def split_heads(qkv, n_head):
    """qkv [B,T,3C] -> q, k, v each [B,H,T,d]; columns [0,C) are q, [C,2C) k,
    [2C,3C) v, and head h owns columns h*d..(h+1)*d of each."""
    B, T, C3 = qkv.shape
    C = C3 // 3
    d = C // n_head
    q, k, v = qkv[..., :C], qkv[..., C:2 * C], qkv[..., 2 * C:]
    f = lambda t: t.reshape(B, T, n_head, d).transpose(0, 2, 1, 3)
    return f(q), f(k), f(v)


def merge_heads(o):
    """[B,H,T,d] -> [B,T,H*d]."""
    B, H, T, d = o.shape
    return o.transpose(0, 2, 1, 3).reshape(B, T, H * d)


def causal_softmax_probs(q, k):
    """P = softmax_j(q.k_j / sqrt(d)) with j > i masked out (decoder-only:
    a position never sees later tokens).  Max-subtracted exponentials."""
    d = q.shape[-1]
    T = q.shape[-2]
    s = (q @ np.swapaxes(k, -1, -2)) / math.sqrt(d)
    future = np.triu(np.ones((T, T), dtype=bool), k=1)
    s = np.where(future, -np.inf, s)
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def attention_forward(qkv, n_head):
    """Causal multi-head self-attention core: o = softmax(q k^T/sqrt(d), causal) v.
    Returns o [B,T,C] and the per-row log-sum-exp [B,H,T] of the scaled scores."""
    q, k, v = split_heads(qkv, n_head)
    d = q.shape[-1]
    T = q.shape[-2]
    s = (q @ np.swapaxes(k, -1, -2)) / math.sqrt(d)
    future = np.triu(np.ones((T, T), dtype=bool), k=1)
    s = np.where(future, -np.inf, s)
    m = s.max(axis=-1, keepdims=True)
    lse = (m + np.log(np.exp(s - m).sum(axis=-1, keepdims=True)))[..., 0]
    p = causal_softmax_probs(q, k)
    return merge_heads(p @ v), lse


def attention_backward(do, qkv, n_head):
    """Chain rule through attention_forward (P recomputed from q, k):
    dv = P^T do ; dP = do v^T ; dS = P*(dP - rowsum(dP*P)) ;
    dq = dS k / sqrt(d) ; dk = dS^T q / sqrt(d).  Returns dqkv [B,T,3C]."""
    q, k, v = split_heads(qkv, n_head)
    B, H, T, d = q.shape
    p = causal_softmax_probs(q, k)
    do_h = do.reshape(B, T, H, d).transpose(0, 2, 1, 3)
    dv = np.swapaxes(p, -1, -2) @ do_h
    dp = do_h @ np.swapaxes(v, -1, -2)
    ds = p * (dp - (dp * p).sum(axis=-1, keepdims=True))
    dq = (ds @ k) / math.sqrt(d)
    dk = (np.swapaxes(ds, -1, -2) @ q) / math.sqrt(d)
    return np.concatenate([merge_heads(dq), merge_heads(dk), merge_heads(dv)], axis=-1)


def cross_entropy(z, y, loss_scale=1.0):
    """[C] chapter "cross entropy loss".  z [M,V] logits over the padded
    vocabulary, y [M] targets.  reading: the softmax runs over all padded
    columns; the loss is the mean over all M positions with no ignore index.

    loss = mean_i (lse_i - z_i[y_i]);  dz = (softmax(z) - onehot(y)) * loss_scale / M;
    argmax = lowest index among the maxima of each row.
    """
    M = z.shape[0]
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    sumexp = e.sum(axis=1, keepdims=True)
    lse = (zmax + np.log(sumexp))[:, 0]
    rows = np.arange(M)
    losses = lse - z[rows, y]
    prob = e / sumexp
    dz = prob.copy()
    dz[rows, y] -= 1.0
    dz *= loss_scale / M
    return float(losses.mean()), losses, dz, np.argmax(z, axis=1).astype(np.int32)


# --------------------------------------------------------------------------
# the model
# --------------------------------------------------------------------------

def forward(flat, cfg: Config, tokens, targets=None, dtype=None):
    """Logits (and loss) for tokens [B,T] (int) given the flat parameters.

    [D] Key Features (token + positional embeddings, attention with layer norm
    and residual connections, GELU MLP), [V] architecture bullet (pre-norm,
    extra final LayerNorm), [V]/[C] weight tying (logits = xf @ wte^T).
    Returns a state dict that ``backward`` consumes.
    """
    dtype = dtype or flat.dtype
    p = unflatten(flat.astype(dtype, copy=False), cfg)
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    assert T <= cfg.block_size
    C, H = cfg.n_embd, cfg.n_head
    x = p["wte"][tokens] + p["wpe"][:T][None]           # [B,T,C]
    cache = {"tokens": tokens, "layers": []}
    for l in range(cfg.n_layer):
        pre = f"h{l}."
        c = {"x_in": x}
        h, c["ln1_mean"], c["ln1_rstd"] = layernorm_forward(x, p[pre + "ln1.g"], p[pre + "ln1.b"])
        c["ln1"] = h
        qkv = linear_forward(h, p[pre + "attn.w"], p[pre + "attn.b"])
        c["qkv"] = qkv
        o, c["lse"] = attention_forward(qkv, H)
        c["att"] = o
        x = x + linear_forward(o, p[pre + "proj.w"], p[pre + "proj.b"])
        c["x_mid"] = x
        h2, c["ln2_mean"], c["ln2_rstd"] = layernorm_forward(x, p[pre + "ln2.g"], p[pre + "ln2.b"])
        c["ln2"] = h2
        u = linear_forward(h2, p[pre + "fc.w"], p[pre + "fc.b"])
        c["fc_pre"] = u
        a = gelu_tanh(u)
        c["fc_act"] = a
        x = x + linear_forward(a, p[pre + "mproj.w"], p[pre + "mproj.b"])
        cache["layers"].append(c)
    cache["x_final"] = x
    xf, cache["lnf_mean"], cache["lnf_rstd"] = layernorm_forward(x, p["lnf.g"], p["lnf.b"])
    cache["lnf"] = xf
    logits = linear_forward(xf, p["wte"])                 # [B,T,Vp], no bias
    state = {"cfg": cfg, "params": p, "flat_dtype": dtype, "cache": cache,
             "logits": logits, "B": B, "T": T}
    if targets is not None:
        targets = np.asarray(targets)
        loss, losses, dz, amax = cross_entropy(logits.reshape(B * T, -1), targets.reshape(-1))
        state.update(loss=loss, losses=losses.reshape(B, T), dz_unit=dz, argmax=amax.reshape(B, T))
    return state


def backward(state, loss_scale=1.0):
    """Every parameter gradient, in the flat order, for loss * loss_scale.

    [C] chapter "gradient accumulation" / [V] accumulation bullet: each
    micro-step's loss is divided by the number of micro-steps, which is
    ``loss_scale``.  The tied wte gradient is the sum of its lm_head use and its
    embedding use (np.add.at scatter).
    """
    cfg, p, c = state["cfg"], state["params"], state["cache"]
    B, T, C = state["B"], state["T"], cfg.n_embd
    dtype = state["flat_dtype"]
    grads = np.zeros(num_params(cfg), dtype=dtype)
    g = unflatten(grads, cfg)
    dz = (state["dz_unit"] * loss_scale).reshape(B, T, -1)
    # lm_head (tied): logits = xf @ wte^T
    dxf, dw, _ = linear_backward(dz, c["lnf"], p["wte"])
    g["wte"] += dw
    dx, dg, db = layernorm_backward(dxf, c["x_final"], c["lnf_mean"], c["lnf_rstd"], p["lnf.g"])
    g["lnf.g"] += dg
    g["lnf.b"] += db
    for l in reversed(range(cfg.n_layer)):
        pre, cl = f"h{l}.", c["layers"][l]
        # x_out = x_mid + mproj(gelu(fc(ln2(x_mid))))
        da, dw, db = linear_backward(dx, cl["fc_act"], p[pre + "mproj.w"])
        g[pre + "mproj.w"] += dw
        g[pre + "mproj.b"] += db
        du = da * gelu_tanh_grad(cl["fc_pre"])
        dh2, dw, db = linear_backward(du, cl["ln2"], p[pre + "fc.w"])
        g[pre + "fc.w"] += dw
        g[pre + "fc.b"] += db
        dln, dg, db = layernorm_backward(dh2, cl["x_mid"], cl["ln2_mean"], cl["ln2_rstd"], p[pre + "ln2.g"])
        g[pre + "ln2.g"] += dg
        g[pre + "ln2.b"] += db
        dx = dx + dln                                     # residual
        # x_mid = x_in + proj(attn(qkv(ln1(x_in))))
        do, dw, db = linear_backward(dx, cl["att"], p[pre + "proj.w"])
        g[pre + "proj.w"] += dw
        g[pre + "proj.b"] += db
        dqkv = attention_backward(do, cl["qkv"], cfg.n_head)
        dh, dw, db = linear_backward(dqkv, cl["ln1"], p[pre + "attn.w"])
        g[pre + "attn.w"] += dw
        g[pre + "attn.b"] += db
        dln, dg, db = layernorm_backward(dh, cl["x_in"], cl["ln1_mean"], cl["ln1_rstd"], p[pre + "ln1.g"])
        g[pre + "ln1.g"] += dg
        g[pre + "ln1.b"] += db
        dx = dx + dln
    # embeddings: x0 = wte[tok] + wpe[t]
    tok = c["tokens"]
    np.add.at(g["wte"], tok.reshape(-1), dx.reshape(B * T, C))
    g["wpe"][:T] += dx.sum(axis=0)
    return grads


# --------------------------------------------------------------------------
# optimizer
# --------------------------------------------------------------------------

def grad_norm(grads) -> float:
    """Global L2 norm over every gradient (the tied wte counted once)."""
    return float(np.sqrt(np.sum(np.asarray(grads, dtype=np.float64) ** 2)))


def clip_scale(norm: float, max_norm: float = 1.0) -> float:
    """[V] hyperparameter bullet: clip the global gradient norm at 1.0.
    reading: s = min(1, max_norm / (norm + 1e-6))."""
    return min(1.0, max_norm / (norm + 1e-6))


def adamw_step(params, grads, m, v, t, lr, cfg: Config, wd=0.1, beta1=0.9, beta2=0.95,
               eps=1e-8, max_norm=1.0):
    """Clip then one AdamW update; returns (params, m, v, norm) as new arrays.

    [V] hyperparameter bullet / [D] Key Features: AdamW, betas (0.9, 0.95),
    eps 1e-8, weight decay 0.1 on 2D tensors only.
    reading: decoupled decay p <- p*(1 - lr*wd) before the moment update;
    bias correction of both moments with step count t (t >= 1); eps added
    after the bias-corrected sqrt(v).
    """
    assert t >= 1
    norm = grad_norm(grads)
    s = clip_scale(norm, max_norm)
    gs = grads * s
    mask = decay_mask(cfg, dtype=params.dtype)
    p = params * (1.0 - lr * wd * mask)
    m = beta1 * m + (1.0 - beta1) * gs
    v = beta2 * v + (1.0 - beta2) * gs * gs
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v, norm


def lr_at(it: int, max_lr=6e-4, min_lr=6e-5, warmup=715, max_steps=19073) -> float:
    """[C] chapter "learning rate scheduler: warmup + cosine decay"; [V]
    hyperparameter bullet (max 6e-4, warm up over 375M tokens, decay to 10% of
    max); [D] Training Setup table (715 warmup steps, 19073 iterations).
    reading: lr = max*(it+1)/warmup while it < warmup; min after max_steps;
    cosine in between."""
    if it < warmup:
        return max_lr * (it + 1) / warmup
    if it > max_steps:
        return min_lr
    ratio = (it - warmup) / (max_steps - warmup)
    coeff = 0.5 * (1.0 + math.cos(math.pi * ratio))
    return min_lr + coeff * (max_lr - min_lr)


def train_step(params, m, v, t, cfg: Config, micro_batches, lr, **adamw_kw):
    """One optimizer step: accumulate gradients over the micro-batches
    (loss scale 1/n each), clip, AdamW.  micro_batches: list of (tokens, targets).
    Returns (params, m, v, mean micro-loss, grad norm)."""
    n = len(micro_batches)
    grads = np.zeros_like(params)
    losses = []
    for tok, tgt in micro_batches:
        st = forward(params, cfg, tok, tgt)
        grads += backward(st, loss_scale=1.0 / n)
        losses.append(st["loss"])
    p, m, v, norm = adamw_step(params, grads, m, v, t, lr, cfg, **adamw_kw)
    return p, m, v, float(np.mean(losses)), norm


# --------------------------------------------------------------------------
# generation
# --------------------------------------------------------------------------
# [C] chapters "sampling init, prefix tokens, tokenization", "sampling loop":
# the model continues a prefix one token at a time, each new token drawn from
# the distribution its logits give at the last position.  The pages name no
# sampling rule.  reading: top-k sampling from softmax(logits / temperature)
# over the k largest logits of the real vocabulary [0, V) (padded ids are not
# tokens), ties at the k-th place going to the lower id; k = 1 (or
# temperature 0) is the greedy argmax.  What KV caching changes is only how
# the logits are computed: the reference for the logits at position t is
# forward() on the prefix tokens[:t+1], whose last row they are.

_SM64_GAMMA = 0x9E3779B97F4A7C15
_MASK64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """The splitmix64 generator's output function (Steele, Lea and Flood,
    "Fast splittable pseudorandom number generators", OOPSLA 2014): add the
    golden-ratio increment, then two xor-shift-multiply rounds and a final
    xor-shift, all modulo 2^64."""
    z = (x + _SM64_GAMMA) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def sample_uniform(seed: int, row: int, pos: int) -> float:
    """Counter-based uniform in [0, 1) for sequence `row` at position `pos`:
    the top 53 bits of splitmix64(seed * 2^32 + pos * 2^16 + row).
    reading: the pages fix no generator; this one is defined here and in the
    device sampler alike, so both draw the same u."""
    key = ((seed & 0xFFFFFFFF) << 32 | (pos & 0xFFFF) << 16 | (row & 0xFFFF)) & _MASK64
    return (splitmix64(key) >> 11) * (1.0 / (1 << 53))


def sample_next(logits_row, vocab: int, temperature: float, top_k: int, u: float) -> int:
    """One draw of the next token from one row of logits (see the reading
    above): keep the top_k largest logits among ids [0, vocab), form
    p_i = exp((z_i - z_max) / temperature) / sum, and return the first id (in
    descending-logit order) whose cumulative probability exceeds u."""
    z = np.asarray(logits_row, dtype=np.float64)[:vocab]
    if top_k <= 1 or temperature <= 0.0:
        return int(np.argmax(z))
    k = min(top_k, vocab)
    order = np.lexsort((np.arange(vocab), -z))[:k]  # descending logit, lower id first on ties
    zk = z[order]
    p = np.exp((zk - zk[0]) / temperature)
    cdf = np.cumsum(p) / p.sum()
    i = int(np.searchsorted(cdf, u, side="right"))
    return int(order[min(i, k - 1)])
