"""Generation with the KV cache (gpt2_prefill / gpt2_decode_step) through the C
ABI against the oracle.

The reference for the logits at position t is the oracle's forward on the
prefix tokens[:t+1] (its last row): the cache changes how they are computed,
not what they are.  The bf16 logits are held to the bf16 forward's tolerance.
The sampled token is integer work and is checked bit-exactly against the
oracle's top-k rule applied to the device's own logits with the same
counter-based uniform draw."""
import numpy as np
import pytest

from tests.gpu_util import cosine, need_gpu, torch

pytestmark = pytest.mark.gpu

TINY = dict(n_layer=2, n_head=2, n_embd=128, vocab_size=500, padded_vocab=512, block_size=256)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _run(cfgd, B, T0, steps, temperature, top_k, seed, check_rows=None, max_T=None, oracle_dtype=np.float64):
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    from decoder_only_transformer_02_b200.synthetic import token_batches
    from oracle import gpt2_oracle as O
    cfg = O.Config(**cfgd)
    m = G.GPT2(G.GPT2Config(**cfgd, max_B=B, max_T=max_T or T0, precision=G.GPT2_BF16), seed=11)
    flat = O.init_params(cfg, 21).astype(np.float32)
    m.set_params(flat)
    (prompt, _), = token_batches("zipf", cfg.vocab_size, B, T0, 1, seed=5)
    seq = prompt.copy()
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    m.prefill(_dev(prompt), nxt, temperature, top_k, seed)
    rows = range(B) if check_rows is None else check_rows
    for step in range(steps + 1):
        t = seq.shape[1] - 1  # position of the logits row the draw used
        logits = m.get_decode_logits(B)
        got = nxt.cpu().numpy()
        ref = O.forward(flat.astype(oracle_dtype), cfg, seq[list(rows)])["logits"][:, t]
        for i, b in enumerate(rows):
            assert np.max(np.abs(logits[b] - ref[i])) < 0.05 * max(1.0, np.max(np.abs(ref[i]))), (step, b)
            assert cosine(logits[b], ref[i]) > 0.9999, (step, b)
        for b in range(B):
            want = O.sample_next(logits[b], cfg.vocab_size, temperature, top_k, O.sample_uniform(seed, b, t + 1))
            assert got[b] == want, (step, b, got[b], want)
            assert 0 <= got[b] < cfg.vocab_size
        seq = np.concatenate([seq, got[:, None]], axis=1)
        if step < steps:
            m.decode_step(_dev(got), t + 1, nxt, temperature, top_k, seed)
    m.close()
    return seq


def test_greedy_generation_matches_oracle():
    seq = _run(TINY, B=2, T0=5, steps=40, temperature=1.0, top_k=1, seed=3)
    assert seq.shape == (2, 46)


def test_top_k_sampling_matches_oracle_rule():
    _run(TINY, B=3, T0=7, steps=30, temperature=0.8, top_k=20, seed=12345)


def test_generation_reaches_block_size():
    # prefix 200 + 56 steps: the last step caches position 255 = block_size - 1
    _run(TINY, B=1, T0=200, steps=56, temperature=1.0, top_k=5, seed=9)


def test_generation_124m_after_long_prefix():
    """GPT-2 124M: a 1000-token prefix, then decode steps; the oracle (fp32 at
    this size) checks the logits of sequence 0, the rule every sequence."""
    cfgd = dict(n_layer=12, n_head=12, n_embd=768, vocab_size=50257, padded_vocab=50304, block_size=1024)
    _run(cfgd, B=2, T0=1000, steps=3, temperature=1.0, top_k=50, seed=77, check_rows=[0], oracle_dtype=np.float32)


def test_generation_call_order_and_arguments():
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    m = G.GPT2(G.GPT2Config(**TINY, max_B=2, max_T=16, precision=G.GPT2_BF16), seed=1)
    tok = _dev(np.zeros((2, 4)))
    nxt = torch.empty(2, dtype=torch.int32, device="cuda")
    with pytest.raises(G.GPT2Error) as e:
        m.decode_step(_dev(np.zeros(2)), 0, nxt)          # no prefill yet
    assert e.value.name == "ESTATE"
    with pytest.raises(G.GPT2Error) as e:
        m.prefill(tok, nxt, 1.0, 65, 0)                    # top_k beyond 64
    assert e.value.name == "EINVAL"
    m.prefill(tok, nxt, 1.0, 1, 0)
    with pytest.raises(G.GPT2Error) as e:
        m.decode_step(_dev(np.zeros(2)), 5, nxt)          # not the next position
    assert e.value.name == "ESTATE"
    m.decode_step(_dev(np.zeros(2)), 4, nxt)
    m.close()
