"""The whole training step through the C ABI against the CPU oracle.

fp32 mode (tiny config): per-tensor max|err|/max|ref| <= 1e-4 for logits and
gradients.  bf16 mode: |dloss| <= 1e-2 and per-tensor gradient cosine >= 0.999
against the fp32 oracle on the same fp32 master weights.  Integer work
(argmax, embedding sort keys) bit-exact.  Host-side fault paths (bad ids,
calls out of order, non-finite gradients) return their status codes."""
import math

import numpy as np
import pytest

from tests.gpu_util import cosine, need_gpu, per_tensor, rel_max_err, torch

pytestmark = pytest.mark.gpu

TINY_CFG = dict(n_layer=2, n_head=4, n_embd=128, vocab_size=512, padded_vocab=512, block_size=64)
BF_CFG = dict(n_layer=2, n_head=2, n_embd=128, vocab_size=500, padded_vocab=512, block_size=256)


def make(cfgd, B, T, prec, seed=1234):
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    from oracle import gpt2_oracle as O
    cfg = O.Config(**cfgd)
    m = G.GPT2(G.GPT2Config(**cfgd, max_B=B, max_T=T, precision=prec), seed=seed)
    return G, O, cfg, m


def batch(kind, V, B, T, seed, n=1):
    from decoder_only_transformer_02_b200.synthetic import token_batches
    return token_batches(kind, V, B, T, n, seed)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


# ------------------------------------------------------------------ fp32

def test_fp32_tiny_forward_backward_parity():
    G, O, cfg, m = make(TINY_CFG, 4, 64, 0)
    flat = O.init_params(cfg, 1234)
    m.set_params(flat.astype(np.float32))
    (tok, tgt), = batch("uniform", 512, 4, 64, 1235)
    loss = m.forward(dev(tok), dev(tgt), want_loss=True)
    logits = m.get_logits()
    m.backward(1.0)
    g = m.get_grads()
    st = O.forward(flat, cfg, tok, tgt)
    gref = O.backward(st, 1.0)
    assert rel_max_err(logits, st["logits"]) <= 1e-4
    assert abs(loss - st["loss"]) <= 1e-4 * abs(st["loss"])
    errs = per_tensor(g, gref, cfg, rel_max_err)
    bad = {k: v for k, v in errs.items() if v > 1e-4}
    assert not bad, bad
    np.testing.assert_array_equal(m.get_argmax(), np.argmax(logits, axis=-1))


def test_fp32_tiny_adamw_step_parity():
    """AdamW + clip on the device against the oracle's update applied to the
    same parameters and the device's own gradients (isolates the optimizer)."""
    G, O, cfg, m = make(TINY_CFG, 4, 64, 0)
    flat = O.init_params(cfg, 7).astype(np.float32)
    m.set_params(flat)
    (tok, tgt), = batch("uniform", 512, 4, 64, 8)
    m.forward_backward(dev(tok), dev(tgt), 1.0)
    g = m.get_grads().astype(np.float64)
    for step, (lr, clip) in enumerate([(6e-4, 1.0), (3e-3, 1e-2)], start=1):
        p0 = m.get_params().astype(np.float64)
        m0, v0, t0 = m.get_adam_state()
        norm = m.adamw_step(lr, clip=clip, want_norm=True)
        p1 = m.get_params()
        m1, v1, t1 = m.get_adam_state()
        pr, mr, vr, nr = O.adamw_step(p0, g, m0.astype(np.float64), v0.astype(np.float64), step, lr, cfg,
                                      max_norm=clip)
        assert t1 == t0 + 1 == step
        assert math.isclose(norm, nr, rel_tol=1e-5)
        assert rel_max_err(m1, mr) < 1e-5 and rel_max_err(v1, vr) < 1e-5
        assert np.max(np.abs(p1 - pr)) < 1e-6 + 1e-5 * np.max(np.abs(pr))


def test_fp32_gradient_accumulation_matches_big_batch():
    G, O, cfg, m = make(TINY_CFG, 2, 64, 0)
    flat = O.init_params(cfg, 3)
    m.set_params(flat.astype(np.float32))
    mbs = batch("uniform", 512, 2, 64, 4, n=2)
    m.zero_grad()
    for tok, tgt in mbs:
        m.forward(dev(tok), dev(tgt))
        m.backward(0.5)
    g = m.get_grads()
    tok = np.concatenate([b[0] for b in mbs])
    tgt = np.concatenate([b[1] for b in mbs])
    gref = O.backward(O.forward(flat, cfg, tok, tgt), 1.0)
    errs = per_tensor(g, gref, cfg, rel_max_err)
    assert max(errs.values()) <= 1e-4, errs


def test_fp32_causal_invariance_bit_exact():
    G, O, cfg, m = make(TINY_CFG, 4, 64, 0)
    (tok, _), = batch("uniform", 512, 4, 64, 11)
    m.forward(dev(tok))
    base = m.get_logits()
    for t in (0, 20, 62):
        tok2 = tok.copy()
        tok2[:, t + 1:] = (tok2[:, t + 1:] + 1) % 512
        m.forward(dev(tok2))
        got = m.get_logits()
        assert np.array_equal(got[:, :t + 1], base[:, :t + 1])


# ------------------------------------------------------------------ bf16

@pytest.mark.parametrize("B,T", [(2, 128), (3, 200), (1, 256)])
def test_bf16_forward_backward_parity(B, T):
    G, O, cfg, m = make(BF_CFG, B, T, 1)
    flat = O.init_params(cfg, 1234).astype(np.float32)
    m.set_params(flat)
    (tok, tgt), = batch("zipf", cfg.vocab_size, B, T, 99)
    loss = m.forward(dev(tok), dev(tgt), want_loss=True)
    logits = m.get_logits()
    amax = m.get_argmax()
    m.backward(1.0)
    g = m.get_grads()
    st = O.forward(flat.astype(np.float64), cfg, tok, tgt)
    gref = O.backward(st, 1.0)
    assert abs(loss - st["loss"]) <= 1e-2
    np.testing.assert_allclose(m.get_losses(), st["losses"], atol=5e-2)
    assert rel_max_err(logits, st["logits"]) < 3e-2
    cos = per_tensor(g, gref, cfg, cosine)
    bad = {k: v for k, v in cos.items() if v < 0.999}
    assert not bad, bad
    # integer work on the device's own logits: bit-exact, lowest index on ties
    np.testing.assert_array_equal(amax, np.argmax(logits, axis=-1))
    keys = m.embed_keys()
    flat_tok = tok.reshape(-1).astype(np.uint64)
    want = np.sort((flat_tok << 16) | np.arange(flat_tok.size, dtype=np.uint64)).astype(np.uint32)
    np.testing.assert_array_equal(keys, want)


def test_bf16_fused_forward_backward_equals_separate():
    G, O, cfg, m = make(BF_CFG, 2, 128, 1)
    (tok, tgt), = batch("zipf", cfg.vocab_size, 2, 128, 5)
    m.zero_grad()
    l1 = m.forward(dev(tok), dev(tgt), want_loss=True)
    m.backward(0.25)
    g1 = m.get_grads()
    m.zero_grad()
    l2 = m.forward_backward(dev(tok), dev(tgt), 0.25, want_loss=True)
    g2 = m.get_grads()
    assert l1 == l2
    np.testing.assert_array_equal(g1, g2)


def test_graph_replay_equals_eager_launches():
    """The fused micro-step is captured into a CUDA graph on the second use of a
    (B, T, loss scale) and replayed afterwards: the results must be the very
    bits the eager launches give, for new batches and after a shape change."""
    runs = {}
    for graphs in (False, True):
        G, O, cfg, m = make(BF_CFG, 2, 128, 1, seed=7)
        m.set_graphs(graphs)
        seq = [(2, 128, 0), (2, 128, 1), (2, 128, 2), (1, 96, 3), (2, 128, 4), (1, 96, 5), (1, 96, 6)]
        out = []
        for B, T, seed in seq:
            (tok, tgt), = batch("zipf", cfg.vocab_size, B, T, 40 + seed)
            m.zero_grad()
            loss = m.forward_backward(dev(tok), dev(tgt), 0.5, want_loss=True)
            out.append((loss, m.get_grads()))
        m.adamw_step(6e-4)
        out.append((0.0, m.get_params()))
        runs[graphs] = out
        m.close()
    for (la, ga), (lb, gb) in zip(runs[False], runs[True]):
        assert la == lb
        np.testing.assert_array_equal(ga, gb)


def test_graph_replay_with_split_accumulators_equals_eager():
    """Two optimizer steps of three micro-steps each, with the weight
    gradients split over 1024 tokens into per-split accumulators: the second
    step replays every micro-step from the CUDA graph, and the accumulators
    must still be folded into the gradients before the update.  The
    parameters must be the very bits of all-eager launches."""
    cfgd = dict(n_layer=2, n_head=4, n_embd=256, vocab_size=500, padded_vocab=512, block_size=256)
    params = {}
    for graphs in (False, True):
        G, O, cfg, m = make(cfgd, 4, 256, 1, seed=9)
        m.set_graphs(graphs)
        for step in range(2):
            m.zero_grad()
            for k, (tok, tgt) in enumerate(batch("zipf", cfg.vocab_size, 4, 256, 90 + 10 * step, n=3)):
                m.forward_backward(dev(tok), dev(tgt), 1.0 / 3)
            m.adamw_step(6e-4)
        params[graphs] = m.get_params()
        m.close()
    assert not np.array_equal(params[False], 0)
    np.testing.assert_array_equal(params[False], params[True])


def test_bf16_accumulated_optimizer_step_matches_oracle():
    """The accumulated optimizer step in bf16 mode: four micro-steps with
    distinct batches at loss scale 1/4 (the first eager, the second captured
    into a CUDA graph, the last two replayed), then the global-norm clip
    (active: clip 1e-2) and AdamW, against the oracle's train_step arithmetic
    on the same fp32 master weights and moments.  The moments start from a
    seeded non-zero state at t = 10, so the update is a smooth function of
    the gradient (at t = 1 it is lr*sign(g), which no tolerance on g bounds).
    Bars: |dloss| <= 1e-2, per-tensor gradient cosine >= 0.999 (read before
    the step), norm within 1%, per-tensor cosine of the update dp >= 0.999."""
    cfgd = dict(n_layer=2, n_head=4, n_embd=256, vocab_size=500, padded_vocab=512, block_size=256)
    # (1024 tokens per micro-step: the layers' weight gradients are split over
    # the tokens into per-split accumulators, folded before they are read)
    B, T, n_micro, lr, clip = 4, 256, 4, 6e-4, 1e-2
    G, O, cfg, m = make(cfgd, B, T, 1, seed=5)
    flat = O.init_params(cfg, 5).astype(np.float32)
    m.set_params(flat)
    mbs = batch("zipf", cfg.vocab_size, B, T, 77, n=n_micro)
    # oracle: accumulated gradients and mean micro-loss, fp64 on the same weights
    p64 = flat.astype(np.float64)
    gref = np.zeros_like(p64)
    lref = []
    for tok, tgt in mbs:
        st = O.forward(p64, cfg, tok, tgt)
        gref += O.backward(st, 1.0 / n_micro)
        lref.append(st["loss"])
    rng = np.random.default_rng(3)
    sg = np.abs(gref) + np.mean(np.abs(gref))
    m0 = (rng.standard_normal(p64.size) * sg * clip).astype(np.float32)
    v0 = ((np.abs(rng.standard_normal(p64.size)) + 0.5) * sg * clip) ** 2
    v0 = v0.astype(np.float32)
    t0 = 10
    m.set_adam_state(m0, v0, t0)
    m.zero_grad()
    losses = [m.forward_backward(dev(tok), dev(tgt), 1.0 / n_micro, want_loss=True) for tok, tgt in mbs]
    g = m.get_grads()
    norm = m.adamw_step(lr, clip=clip, want_norm=True)
    p1 = m.get_params()
    m1, v1, t1 = m.get_adam_state()
    pr, mr, vr, nr = O.adamw_step(p64, gref, m0.astype(np.float64), v0.astype(np.float64), t0 + 1, lr, cfg,
                                  max_norm=clip)
    assert t1 == t0 + 1
    assert abs(float(np.mean(losses)) - float(np.mean(lref))) <= 1e-2
    cos = per_tensor(g, gref, cfg, cosine)
    bad = {k: v for k, v in cos.items() if v < 0.999}
    assert not bad, bad
    assert abs(norm - nr) / nr < 1e-2
    assert nr > 10 * clip  # the clip is active
    dcos = per_tensor(p1.astype(np.float64) - p64, pr - p64, cfg, cosine)
    bad = {k: v for k, v in dcos.items() if v < 0.999}
    assert not bad, bad
    mcos = per_tensor(m1, mr, cfg, cosine)
    assert min(mcos.values()) >= 0.999, mcos


def test_bf16_deterministic_step():
    outs = []
    for _ in range(2):
        G, O, cfg, m = make(BF_CFG, 2, 128, 1, seed=42)
        (tok, tgt), = batch("zipf", cfg.vocab_size, 2, 128, 6)
        m.forward_backward(dev(tok), dev(tgt), 1.0)
        m.adamw_step(6e-4)
        outs.append(m.get_params())
        m.close()
    np.testing.assert_array_equal(outs[0], outs[1])


def test_bf16_causal_invariance_bit_exact():
    G, O, cfg, m = make(BF_CFG, 2, 200, 1)
    (tok, _), = batch("zipf", cfg.vocab_size, 2, 200, 12)
    m.forward(dev(tok))
    base = m.get_logits()
    for t in (0, 63, 64, 150):
        tok2 = tok.copy()
        tok2[:, t + 1] = (tok2[:, t + 1] + 7) % cfg.vocab_size
        m.forward(dev(tok2))
        got = m.get_logits()
        assert np.array_equal(got[:, :t + 1], base[:, :t + 1])


def test_bf16_device_init_statistics():
    G, O, cfg, m = make(dict(BF_CFG, n_layer=4), 1, 64, 1, seed=77)
    p = m.get_params()
    off = 0
    rs = 0.02 / math.sqrt(2 * cfg.n_layer)
    for name, shape, _ in O.param_specs(cfg):
        n = int(np.prod(shape))
        x = p[off:off + n].astype(np.float64)
        off += n
        if name.endswith(".g"):
            assert np.all(x == 1)
        elif name.endswith(".b"):
            assert np.all(x == 0)
        else:
            want = rs if name.endswith("proj.w") else 0.02
            assert abs(x.std() / want - 1) < max(0.01, 5 / math.sqrt(2 * n)), name
            assert abs(x.mean()) < 5 * want / math.sqrt(n), name


def test_train_step_host_buffers_matches_device_calls():
    G, O, cfg, m = make(BF_CFG, 2, 128, 1, seed=3)
    mbs = batch("zipf", cfg.vocab_size, 2, 128, 21, n=3)
    h_tok = np.ascontiguousarray(np.stack([b[0] for b in mbs]), dtype=np.int32)
    h_tgt = np.ascontiguousarray(np.stack([b[1] for b in mbs]), dtype=np.int32)
    p0 = m.get_params()
    loss, norm = m.train_step(h_tok, h_tgt, 3, 2, 128, 6e-4)
    p_a = m.get_params()
    # same step through the device-pointer calls
    m.set_params(p0)
    m.set_adam_state(np.zeros_like(p0), np.zeros_like(p0), 0)
    m.zero_grad()
    ls = [m.forward_backward(dev(t), dev(y), 1 / 3, want_loss=True) for t, y in mbs]
    n2 = m.adamw_step(6e-4, want_norm=True)
    np.testing.assert_array_equal(m.get_params(), p_a)
    assert math.isclose(loss, float(np.mean(ls)), rel_tol=1e-6) and norm == n2


def test_overfit_single_batch_bf16():
    G, O, cfg, m = make(BF_CFG, 2, 128, 1, seed=1)
    (tok, tgt), = batch("zipf", cfg.vocab_size, 2, 128, 2)
    losses = []
    for _ in range(60):
        m.zero_grad()
        losses.append(m.forward_backward(dev(tok), dev(tgt), 1.0, want_loss=True))
        m.adamw_step(1e-3)
    ma = np.convolve(losses, np.ones(10) / 10, mode="valid")
    assert np.all(np.diff(ma) < 0)
    assert losses[-1] < 0.5 * losses[0]


# -------------------------------------------------------------- fault paths

def test_out_of_range_token_reports_etoken():
    G, O, cfg, m = make(BF_CFG, 2, 64, 1)
    (tok, tgt), = batch("zipf", cfg.vocab_size, 2, 64, 1)
    tok[1, 5] = 512
    with pytest.raises(G.GPT2Error) as e:
        m.forward(dev(tok), dev(tgt), want_loss=True)
    assert e.value.name == "ETOKEN"
    tok[1, 5] = -3
    with pytest.raises(G.GPT2Error) as e:
        m.forward(dev(tok), dev(tgt), want_loss=True)
    assert e.value.name == "ETOKEN"
    # the handle stays usable
    tok[1, 5] = 3
    assert math.isfinite(m.forward(dev(tok), dev(tgt), want_loss=True))


def test_calls_out_of_order_and_bad_sizes():
    G, O, cfg, m = make(BF_CFG, 2, 64, 1)
    with pytest.raises(G.GPT2Error) as e:
        m.backward(1.0)
    assert e.value.name == "ESTATE"
    (tok, tgt), = batch("zipf", cfg.vocab_size, 2, 64, 1)
    with pytest.raises(G.GPT2Error) as e:
        m._check(m._lib.gpt2_forward(m._h, dev(tok).data_ptr(), None, 3, 64, None))
    assert e.value.name == "EINVAL"
    m.forward(dev(tok))
    with pytest.raises(G.GPT2Error) as e:
        m.backward(1.0)           # forward had no targets
    assert e.value.name == "ESTATE"
    m.forward_backward(dev(tok), dev(tgt), 1.0)
    with pytest.raises(G.GPT2Error) as e:
        m.get_logits()            # consumed by the fused backward
    assert e.value.name == "ESTATE"


def test_nonfinite_gradient_skips_update():
    G, O, cfg, m = make(BF_CFG, 2, 64, 1)
    p = m.get_params()
    p[10] = np.nan
    m.set_params(p)
    (tok, tgt), = batch("zipf", cfg.vocab_size, 2, 64, 1)
    m.forward_backward(dev(tok), dev(tgt), 1.0)
    before = m.get_params()
    with pytest.raises(G.GPT2Error) as e:
        m.adamw_step(6e-4, want_norm=True)
    assert e.value.name == "ENONFINITE"
    after = m.get_params()
    np.testing.assert_array_equal(np.isnan(after), np.isnan(before))
    np.testing.assert_array_equal(after[~np.isnan(after)], before[~np.isnan(before)])
    assert m.get_adam_state()[2] == 0


# ---------------------------------------------------------- guard bytes

def test_guard_bytes_intact_after_steps_and_generation():
    """Every device buffer is followed by guard bytes: after bf16 and fp32
    optimizer steps at ragged shapes and a generation run, none has changed."""
    G, O, cfg, m = make(BF_CFG, 3, 200, 1)
    (tok, tgt), = batch("uniform", 500, 3, 200, 7)
    for k in range(2):
        m.forward_backward(dev(tok), dev(tgt), 0.5)
    m.adamw_step(6e-4)
    nxt = torch.empty(3, dtype=torch.int32, device="cuda")
    m.prefill(dev(tok[:, :37]), nxt, temperature=0.8, top_k=5, seed=11)
    for pos in range(37, 45):
        m.decode_step(nxt.clone(), pos, nxt, temperature=0.8, top_k=5, seed=11)
    assert m.check_guards() == 0
    m.close()
    G, O, cfg, m = make(TINY_CFG, 4, 64, 0)
    (tok, tgt), = batch("uniform", 512, 4, 64, 8)
    m.forward_backward(dev(tok), dev(tgt), 1.0)
    m.adamw_step(6e-4)
    assert m.check_guards() == 0
    m.close()


def test_guard_check_reports_an_overwritten_guard():
    G, O, cfg, m = make(TINY_CFG, 4, 64, 0)
    assert m.check_guards() == 0
    m.debug_overwrite_guard(3)
    assert m.check_guards() == 1
    with pytest.raises(G.GPT2Error):
        m.debug_overwrite_guard(1 << 20)
    m.close()

