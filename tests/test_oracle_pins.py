"""Pins of the CPU oracle against things other than itself: the numbers the
pages print, closed forms, finite differences, and PyTorch library routines.
None of these tests needs a GPU."""
import inspect
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import gpt2_oracle as O
from tests import torch_reference as TR

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")))
MICRO = O.Config(n_layer=1, n_head=2, n_embd=16, vocab_size=30, padded_vocab=32, block_size=8)


def _g(k):
    return GOLD[k]["value"]


# ---------------------------------------------------------------- constants

def test_oracle_constants_match_pages():
    c = O.GPT2_124M
    assert (c.n_layer, c.n_embd, c.vocab_size, c.block_size, c.padded_vocab) == (
        _g("n_layer"), _g("n_embd"), _g("vocab_size"), _g("block_size"), _g("padded_vocab"))
    lr = inspect.signature(O.lr_at).parameters
    assert lr["max_lr"].default == _g("max_lr")
    assert math.isclose(lr["min_lr"].default, _g("min_lr_fraction_of_max") * _g("max_lr"))
    assert lr["warmup"].default == _g("warmup_steps")
    assert lr["max_steps"].default == _g("max_steps")
    ad = inspect.signature(O.adamw_step).parameters
    assert ad["beta1"].default == _g("adamw_beta1")
    assert ad["beta2"].default == _g("adamw_beta2")
    assert ad["eps"].default == _g("adamw_eps")
    assert ad["wd"].default == _g("weight_decay")
    assert ad["max_norm"].default == _g("grad_clip")


def test_warmup_tokens_agree_with_warmup_steps():
    # 375M tokens of warm-up at 524,288 tokens per step is 715 whole steps
    assert int(_g("warmup_tokens") // _g("total_batch_tokens")) == _g("warmup_steps")


def test_accumulation_counts():
    assert _g("total_batch_tokens") // (16 * 1024) == 32
    assert _g("total_batch_tokens") // (_g("short_context_micro_batch") * _g("short_context_seq_len")) == 32


# ------------------------------------------------------------- param counts

def _closed_form(V, C=768, P=1024, L=12):
    return V * C + P * C + L * (12 * C * C + 13 * C) + 2 * C


def test_param_count_closed_form_and_pages():
    assert O.num_params(O.Config(vocab_size=50257, padded_vocab=50257)) == 124_439_808
    assert O.num_params(O.GPT2_124M) == 124_475_904
    assert _closed_form(50257) == 124_439_808 and _closed_form(50304) == 124_475_904
    assert O.num_params(O.TINY) == _closed_form(512, 128, 64, 2) == 470_528
    assert round(O.num_params(O.GPT2_124M) / 1e6) == _g("model_size_millions")
    # tying: the shared V x C matrix is ~30% of the (tied) parameter count
    tied = O.num_params(O.GPT2_124M)
    frac = 50304 * 768 / tied
    assert abs(frac - _g("tying_saves_fraction_approx")) < 0.05
    assert abs(frac - 0.3104) < 1e-3


def test_decay_set():
    specs = O.param_specs(O.GPT2_124M)
    dec = [(n, s) for n, s, d in specs if d]
    nod = [(n, s) for n, s, d in specs if not d]
    assert len(specs) == 148 and len(dec) == 50 and len(nod) == 98
    assert sum(int(np.prod(s)) for _, s in dec) == 124_354_560
    assert sum(int(np.prod(s)) for _, s in nod) == 121_344
    assert all(len(s) == 2 for _, s in dec) and all(len(s) == 1 for _, s in nod)


# ---------------------------------------------------------------------- init

@pytest.mark.parametrize("cfg", [O.TINY, O.GPT2_124M], ids=["tiny", "124m"])
def test_init_statistics(cfg):
    flat = O.init_params(cfg, seed=1234, dtype=np.float32)
    p = O.unflatten(flat, cfg)
    rs = 0.02 / math.sqrt(2 * cfg.n_layer)
    for name, shape, _ in O.param_specs(cfg):
        x = p[name].astype(np.float64)
        if name.endswith(".g"):
            assert np.all(x == 1.0)
        elif name.endswith(".b"):
            assert np.all(x == 0.0)
        else:
            want = rs if name.endswith("proj.w") else 0.02
            n = x.size
            tol = max(0.01, 5.0 / math.sqrt(2 * n))
            assert abs(x.std() / want - 1) < tol, (name, x.std(), want)
            assert abs(x.mean()) < 5 * want / math.sqrt(n), name


@pytest.mark.parametrize("cfg,T,tol", [(O.TINY, 64, 0.05), (O.GPT2_124M, 32, 0.35)], ids=["tiny", "124m"])
def test_initial_loss_near_ln_vocab(cfg, T, tol):
    # Near-uniform logits give a loss of about ln(V).  With tied weights the
    # logit of a position's own input token is xf.wte[tok] ~ 0.02*C*0.7, which
    # at C=768 (about 10) lifts the log-sum-exp by a few tenths; at C=128 the
    # lift is about 0.01.
    flat = O.init_params(cfg, seed=1234, dtype=np.float32)
    rng = np.random.default_rng(7)
    tok = rng.integers(0, cfg.vocab_size, size=(2, T))
    tgt = rng.integers(0, cfg.vocab_size, size=(2, T))
    st = O.forward(flat, cfg, tok, tgt)
    assert math.log(cfg.padded_vocab) - 0.02 < st["loss"] < math.log(cfg.padded_vocab) + tol


# ------------------------------------------------------------------- LR

def test_lr_schedule_points():
    assert math.isclose(O.lr_at(0), 6e-4 / 715)
    assert math.isclose(O.lr_at(714), 6e-4)
    assert math.isclose(O.lr_at(715), 6e-4)
    assert math.isclose(O.lr_at(715 + (19073 - 715) // 2), 3.3e-4, rel_tol=1e-9)
    assert math.isclose(O.lr_at(19073), 6e-5)
    assert math.isclose(O.lr_at(50000), 6e-5)
    # monotone: rises during warm-up, never rises afterwards
    w = [O.lr_at(i) for i in range(0, 715)]
    assert all(a < b for a, b in zip(w, w[1:]))
    d = [O.lr_at(i) for i in range(715, 19100, 37)]
    assert all(a >= b for a, b in zip(d, d[1:]))


# -------------------------------------------------------------- causality

def test_causal_invariance():
    cfg = O.TINY
    flat = O.init_params(cfg, 3)
    rng = np.random.default_rng(0)
    tok = rng.integers(0, cfg.vocab_size, size=(2, 48))
    base = O.forward(flat, cfg, tok)["logits"]
    for t in (0, 10, 30, 46):
        tok2 = tok.copy()
        tok2[:, t + 1] = (tok2[:, t + 1] + 17) % cfg.vocab_size
        got = O.forward(flat, cfg, tok2)["logits"]
        assert np.array_equal(got[:, :t + 1], base[:, :t + 1])
        assert not np.allclose(got[:, t + 1], base[:, t + 1])


# ------------------------------------------------------- finite differences

def _loss_at(flat, cfg, tok, tgt):
    return O.forward(flat, cfg, tok, tgt)["loss"]


def test_finite_difference_gradients():
    cfg = MICRO
    flat = O.init_params(cfg, 11)
    # larger weights than init so that every term matters
    rng = np.random.default_rng(5)
    flat = flat + rng.normal(0, 0.3, flat.size) * (O.decay_mask(cfg) + 0.5)
    tok = rng.integers(0, cfg.vocab_size, size=(2, 8))
    tgt = rng.integers(0, cfg.vocab_size, size=(2, 8))
    st = O.forward(flat, cfg, tok, tgt)
    g = O.backward(st, loss_scale=1.0)
    names = [n for n, _, _ in O.param_specs(cfg)]
    offs = np.cumsum([0] + [int(np.prod(s)) for _, s, _ in O.param_specs(cfg)])
    idx = set(rng.choice(flat.size, 200, replace=False).tolist())
    for i, n in enumerate(names):            # every bias and gain element
        if n.endswith(".b") or n.endswith(".g"):
            idx.update(range(offs[i], offs[i + 1]))
    # central differences: truncation ~h^2, round-off ~1e-16/h; at h=1e-5 both
    # stay below 1e-9 absolute, so relative error <= 1e-6 with a 1e-3 floor
    h = 1e-5
    worst = 0.0
    for j in sorted(idx):
        e = np.zeros_like(flat)
        e[j] = h
        fd = (_loss_at(flat + e, cfg, tok, tgt) - _loss_at(flat - e, cfg, tok, tgt)) / (2 * h)
        worst = max(worst, abs(fd - g[j]) / (abs(g[j]) + 1e-3))
    assert worst < 1e-6, worst


def test_loss_scale_is_linear():
    cfg = MICRO
    flat = O.init_params(cfg, 2)
    rng = np.random.default_rng(1)
    tok = rng.integers(0, cfg.vocab_size, size=(2, 8))
    tgt = rng.integers(0, cfg.vocab_size, size=(2, 8))
    st = O.forward(flat, cfg, tok, tgt)
    np.testing.assert_allclose(O.backward(st, 0.25), 0.25 * O.backward(st, 1.0), rtol=1e-12, atol=0)


# ------------------------------------------------- library-routine reductions

def test_layernorm_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 2, (5, 7, 24)) + 3
    g, b = rng.normal(1, 0.3, 24), rng.normal(0, 0.3, 24)
    dy = rng.normal(0, 1, x.shape)
    y, mu, rs = O.layernorm_forward(x, g, b)
    xt, gt, bt = (torch.tensor(a, requires_grad=True) for a in (x, g, b))
    yt = F.layer_norm(xt, (24,), gt, bt, 1e-5)
    yt.backward(torch.tensor(dy))
    np.testing.assert_allclose(y, yt.detach().numpy(), rtol=1e-12, atol=1e-12)
    dx, dg, db = O.layernorm_backward(dy, x, mu, rs, g)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_gelu_matches_torch():
    u = np.linspace(-8, 8, 4001)
    ut = torch.tensor(u, requires_grad=True)
    yt = F.gelu(ut, approximate="tanh")
    yt.sum().backward()
    np.testing.assert_allclose(O.gelu_tanh(u), yt.detach().numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(O.gelu_tanh_grad(u), ut.grad.numpy(), rtol=1e-11, atol=1e-13)


def test_attention_matches_sdpa_and_autograd():
    rng = np.random.default_rng(3)
    B, T, H, d = 2, 19, 3, 8
    qkv = rng.normal(0, 1, (B, T, 3 * H * d))
    do = rng.normal(0, 1, (B, T, H * d))
    o, lse = O.attention_forward(qkv, H)
    qt = torch.tensor(qkv, requires_grad=True)
    q, k, v = qt.split(H * d, dim=-1)
    f = lambda t: t.view(B, T, H, d).transpose(1, 2)
    ot = F.scaled_dot_product_attention(f(q), f(k), f(v), is_causal=True).transpose(1, 2).reshape(B, T, H * d)
    ot.backward(torch.tensor(do))
    np.testing.assert_allclose(o, ot.detach().numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(O.attention_backward(do, qkv, H), qt.grad.numpy(), rtol=1e-9, atol=1e-11)
    # lse against a direct log-sum-exp of the masked scaled scores
    s = torch.einsum("bhid,bhjd->bhij", f(q), f(k)).detach() / math.sqrt(d)
    s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_cross_entropy_matches_torch():
    rng = np.random.default_rng(4)
    z = rng.normal(0, 3, (37, 50))
    y = rng.integers(0, 45, 37)
    z[5, 7] = z[5, 9] = z[5].max() + 1.0          # a tie: lowest index wins
    loss, losses, dz, amax = O.cross_entropy(z, y, loss_scale=0.5)
    zt = torch.tensor(z, requires_grad=True)
    lt = F.cross_entropy(zt, torch.tensor(y))
    (0.5 * lt).backward()
    assert math.isclose(loss, lt.item(), rel_tol=1e-12)
    np.testing.assert_allclose(dz, zt.grad.numpy(), rtol=1e-10, atol=1e-14)
    assert amax[5] == 7
    assert np.array_equal(amax, np.argmax(z, 1))


def test_full_model_matches_torch_autograd():
    cfg = O.Config(n_layer=2, n_head=2, n_embd=16, vocab_size=40, padded_vocab=48, block_size=12)
    flat = O.init_params(cfg, 8)
    rng = np.random.default_rng(9)
    flat = flat + rng.normal(0, 0.1, flat.size)
    tok = rng.integers(0, cfg.vocab_size, size=(3, 12))
    tgt = rng.integers(0, cfg.vocab_size, size=(3, 12))
    st = O.forward(flat, cfg, tok, tgt)
    g = O.backward(st, loss_scale=1.0)
    p = TR.make_params(flat, cfg)
    logits, loss = TR.model_loss(p, cfg, tok, tgt)
    loss.backward()
    np.testing.assert_allclose(st["logits"], logits.detach().numpy(), rtol=1e-10, atol=1e-12)
    assert math.isclose(st["loss"], loss.item(), rel_tol=1e-12)
    np.testing.assert_allclose(g, TR.flatten_grads(p, cfg), rtol=1e-8, atol=1e-12)


@pytest.mark.parametrize("t", [1, 5])
def test_train_step_matches_torch_adamw(t):
    cfg = O.Config(n_layer=1, n_head=2, n_embd=16, vocab_size=40, padded_vocab=48, block_size=12)
    flat = O.init_params(cfg, 8)
    rng = np.random.default_rng(t)
    mbs = [(rng.integers(0, 40, (2, 12)), rng.integers(0, 40, (2, 12))) for _ in range(3)]
    m = np.abs(rng.normal(0, 1e-3, flat.size)) if t > 1 else np.zeros_like(flat)
    v = np.abs(rng.normal(0, 1e-5, flat.size)) if t > 1 else np.zeros_like(flat)
    # lr and a large step count so that the clip and decay both act
    for clip in (1.0, 1e-3):
        p1, m1, v1, loss, n1 = O.train_step(flat, m, v, t, cfg, mbs, lr=1e-2, max_norm=clip)
        p2, m2, v2, n2 = TR.torch_train_step(flat, m, v, t, cfg, mbs, lr=1e-2, clip=clip)
        assert math.isclose(n1, n2, rel_tol=1e-10)
        np.testing.assert_allclose(m1, m2, rtol=1e-9, atol=1e-15)
        np.testing.assert_allclose(v1, v2, rtol=1e-9, atol=1e-18)
        np.testing.assert_allclose(p1, p2, rtol=1e-9, atol=1e-13)


def test_grad_accumulation_equals_big_batch():
    # mean-loss over 2 micro-batches of B=2 equals one batch of B=4
    cfg = MICRO
    flat = O.init_params(cfg, 4)
    rng = np.random.default_rng(2)
    tok = rng.integers(0, cfg.vocab_size, (4, 8))
    tgt = rng.integers(0, cfg.vocab_size, (4, 8))
    g_big = O.backward(O.forward(flat, cfg, tok, tgt), 1.0)
    g_acc = (O.backward(O.forward(flat, cfg, tok[:2], tgt[:2]), 0.5)
             + O.backward(O.forward(flat, cfg, tok[2:], tgt[2:]), 0.5))
    np.testing.assert_allclose(g_acc, g_big, rtol=1e-10, atol=1e-14)


# ------------------------------------------------------ training dynamics

@pytest.mark.slow
def test_overfit_single_batch():
    cfg = O.TINY
    flat = O.init_params(cfg, 1234, dtype=np.float32)
    rng = np.random.default_rng(1235)
    tok = rng.integers(0, 512, (4, 64))
    tgt = np.roll(tok, -1, axis=1)
    m = np.zeros_like(flat)
    v = np.zeros_like(flat)
    losses = []
    for t in range(1, 301):
        flat, m, v, loss, _ = O.train_step(flat, m, v, t, cfg, [(tok, tgt)], lr=6e-4)
        losses.append(loss)
    ma = np.convolve(losses, np.ones(10) / 10, mode="valid")
    assert np.all(np.diff(ma[:50]) < 0)
    assert losses[-1] < 0.1 * math.log(512), losses[-1]


# ------------------------------------------------ the pins catch mistakes

@pytest.mark.parametrize("mistake", ["gelu_const", "ln_drop_term", "attn_scale", "resid_drop"])
def test_planted_oracle_mistakes_are_caught(monkeypatch, mistake):
    """Plant a plausible mistake in the oracle (CPU only) and check that the
    torch-autograd pin notices it."""
    cfg = O.Config(n_layer=1, n_head=2, n_embd=16, vocab_size=40, padded_vocab=48, block_size=12)
    if mistake == "gelu_const":
        monkeypatch.setattr(O, "GELU_A", 0.04)
    elif mistake == "ln_drop_term":
        def bad(dy, x, mean, rstd, g):
            xhat = (x - mean[..., None]) * rstd[..., None]
            dxhat = dy * g
            dx = rstd[..., None] * (dxhat - dxhat.mean(axis=-1, keepdims=True))
            return dx, (dy * xhat).reshape(-1, x.shape[-1]).sum(0), dy.reshape(-1, x.shape[-1]).sum(0)
        monkeypatch.setattr(O, "layernorm_backward", bad)
    elif mistake == "attn_scale":
        orig = O.causal_softmax_probs
        monkeypatch.setattr(O, "causal_softmax_probs", lambda q, k: orig(q * 0.9, k))
    elif mistake == "resid_drop":
        orig_lb = O.layernorm_backward
        calls = {"n": 0}

        def drop(dy, x, mean, rstd, g):
            calls["n"] += 1
            dx, dg, db = orig_lb(dy, x, mean, rstd, g)
            return (dx * 0.0 if calls["n"] == 2 else dx), dg, db
        monkeypatch.setattr(O, "layernorm_backward", drop)
    flat = O.init_params(cfg, 8) + np.random.default_rng(0).normal(0, 0.1, O.num_params(cfg))
    rng = np.random.default_rng(9)
    tok = rng.integers(0, 40, (2, 12))
    tgt = rng.integers(0, 40, (2, 12))
    st = O.forward(flat, cfg, tok, tgt)
    g = O.backward(st, 1.0)
    p = TR.make_params(flat, cfg)
    logits, loss = TR.model_loss(p, cfg, tok, tgt)
    loss.backward()
    ok = (np.allclose(st["logits"], logits.detach().numpy(), rtol=1e-8, atol=1e-10)
          and np.allclose(g, TR.flatten_grads(p, cfg), rtol=1e-6, atol=1e-10))
    assert not ok


# ------------------------------------------------------------- generation

def test_splitmix64_published_sequence():
    """The generator's output for a sequence seeded with 1234567 (state
    advanced by the golden-ratio increment per draw), as printed with the
    reference C implementation of splitmix64."""
    s, g = 1234567, O._SM64_GAMMA
    got = [O.splitmix64((s + i * g) & O._MASK64) for i in range(5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423, 4593380528125082431,
                   16408922859458223821]


def test_sample_uniform_range_and_spread():
    u = np.array([O.sample_uniform(7, b, p) for b in range(16) for p in range(256)])
    assert np.all((u >= 0) & (u < 1))
    assert abs(u.mean() - 0.5) < 0.02 and abs(u.var() - 1 / 12) < 0.01
    assert len(set(u.tolist())) == u.size


def test_sample_next_greedy_and_edges():
    rng = np.random.default_rng(3)
    z = rng.normal(0, 2, 64)
    V = 60           # ids 60..63 are padding and never drawn
    z[61] = 100.0
    best = int(np.argmax(z[:V]))
    assert O.sample_next(z, V, 1.0, 1, 0.7) == best
    assert O.sample_next(z, V, 0.0, 50, 0.7) == best
    order = np.argsort(-z[:V], kind="stable")
    assert O.sample_next(z, V, 1.0, 5, 0.0) == order[0]          # u = 0: the largest logit
    assert O.sample_next(z, V, 1.0, 5, 1 - 1e-12) == order[4]    # u -> 1: the k-th largest
    assert O.sample_next(z, V, 1e-6, 5, 0.999) == order[0]       # temperature -> 0: greedy


def test_sample_next_ties_go_to_lower_id():
    z = np.array([1.0, 3.0, 2.0, 2.0, 2.0, 0.0])
    # top 2 = id 1 and, among the three tied at 2.0, the lowest id 2
    draws = {O.sample_next(z, 6, 1.0, 2, u) for u in np.linspace(0, 0.999, 200)}
    assert draws == {1, 2}


def test_sample_next_frequencies_follow_softmax():
    """Over u spread evenly in [0, 1) the draws land on each of the top-k ids
    with the softmax(z / T) probability restricted to them (the inverse-CDF
    rule), up to the 1/n grid."""
    z = np.array([0.5, 2.0, -1.0, 1.5, 0.0, 3.0, -2.0, 1.0])
    T, k, n = 0.7, 4, 20000
    counts = np.zeros(len(z))
    for u in (np.arange(n) + 0.5) / n:
        counts[O.sample_next(z, len(z), T, k, u)] += 1
    top = np.argsort(-z)[:k]
    p = np.zeros(len(z))
    p[top] = np.exp(z[top] / T) / np.exp(z[top] / T).sum()
    np.testing.assert_allclose(counts / n, p, atol=2.0 / n)
