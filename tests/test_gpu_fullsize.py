"""GPT-2 124M at the benchmark's launch configuration (bf16, B=16 x T=1024 and
B=32 x T=512), checked against the fp32 oracle on outputs it can compute in
seconds:

* per-position losses and sampled logits rows of two distinct sequences of a
  batch (the oracle runs those sequences alone: positions only see their own
  sequence);
* gradients of a batch made of one sequence repeated B times: the batch-mean
  loss then has exactly the single sequence's gradient, which the oracle
  computes at the same shapes per sequence.
"""
import numpy as np
import pytest

from tests.gpu_util import cosine, need_gpu, per_tensor, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=[(16, 1024), (32, 512)], ids=["B16xT1024", "B32xT512"])
def setup(request):
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    from oracle import gpt2_oracle as O
    B, T = request.param
    m = G.GPT2(G.GPT2Config(12, 12, 768, 50257, 50304, 1024, B, T, G.GPT2_BF16), seed=1234)
    flat = m.get_params()
    yield G, O, m, flat, B, T
    m.close()


def _seq(seed, T):
    from decoder_only_transformer_02_b200.synthetic import token_batches
    (x, y), = token_batches("zipf", 50257, 1, T, 1, seed=seed)
    return x, y


def test_fullsize_losses_and_logits_of_sampled_sequences(setup):
    G, O, m, flat, B, T = setup
    from decoder_only_transformer_02_b200.synthetic import token_batches
    (tok, tgt), = token_batches("zipf", 50257, B, T, 1, seed=31)
    m.forward(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
    losses = m.get_losses()
    amax = m.get_argmax()
    logits = m.get_logits()
    for b in (0, B - 1):
        st = O.forward(flat, O.GPT2_124M, tok[b:b + 1], tgt[b:b + 1])
        assert abs(float(losses[b].mean()) - st["loss"]) <= 1e-2
        assert np.max(np.abs(losses[b] - st["losses"][0])) < 0.1
        rows = np.random.default_rng(b).choice(T, 8, replace=False)
        ref = st["logits"][0, rows]
        got = logits[b, rows]
        assert np.max(np.abs(got - ref)) < 0.05 * max(1.0, np.max(np.abs(ref)))
        for i in range(len(rows)):
            assert cosine(got[i], ref[i]) > 0.9999
    np.testing.assert_array_equal(amax, np.argmax(logits, axis=-1))


def test_fullsize_gradients_repeated_sequence(setup):
    G, O, m, flat, B, T = setup
    x, y = _seq(41, T)
    tok = np.repeat(x, B, axis=0)
    tgt = np.repeat(y, B, axis=0)
    m.zero_grad()
    loss = m.forward_backward(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda(), 1.0, want_loss=True)
    g = m.get_grads()
    st = O.forward(flat, O.GPT2_124M, x, y)
    gref = O.backward(st, 1.0)
    assert abs(loss - st["loss"]) <= 1e-2
    cos = per_tensor(g, gref, O.GPT2_124M, cosine)
    bad = {k: v for k, v in cos.items() if v < 0.999}
    assert not bad, bad
    norm = m.adamw_step(6e-4, want_norm=True)
    assert abs(norm - O.grad_norm(gref)) / O.grad_norm(gref) < 1e-2
    # every kernel of the step stayed inside its buffers
    assert m.check_guards() == 0
