"""The bounded-wait failure path on the GPU, without a fault.

Every pipeline wait inside the tcgen05 kernels gives up after a limit, records
an error code in the device's error word and lets the kernel return (its own
in-flight copies and MMAs are drained first, under a separate fixed limit).
Here the limit is shortened so that the waits run out, and the tests check
that the error reaches the host, that nothing is left hung, and that the
library gives correct results again once the limit is restored."""
import math

import numpy as np
import pytest

from tests.gpu_util import bf16_round, from_dev, need_gpu, rel_max_err, to_dev_bf16, torch

pytestmark = pytest.mark.gpu


@pytest.fixture
def G():
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    G.check_device_error()  # start from a clear error word
    yield G
    G.set_wait_limit_ns(0)
    torch.cuda.synchronize()


def _gemm(G, A, Bm, M, N, K):
    o = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    G.matmul_bf16(A, K, 0, Bm, K, 0, M, N, K, 0, out=o, ldc=N)
    return o


def test_gemm_wait_timeout_is_reported_and_recovers(G):
    from decoder_only_transformer_02_b200.synthetic import normal_array
    M, N, K = 2048, 1024, 16384  # tiles long enough that the epilogue has to wait
    a = bf16_round(normal_array((M, K), 21))
    b = bf16_round(normal_array((N, K), 22))
    A, Bm = to_dev_bf16(a), to_dev_bf16(b)
    G.set_wait_limit_ns(1)  # every wait that has to spin gives up at once
    _gemm(G, A, Bm, M, N, K)
    with pytest.raises(G.GPT2Error) as e:
        G.check_device_error()
    assert e.value.name == "ECUDA"
    G.check_device_error()  # the check cleared the word
    G.set_wait_limit_ns(0)
    o = _gemm(G, A, Bm, M, N, K)
    G.check_device_error()
    ref = a @ b.T
    assert rel_max_err(from_dev(o), ref) < 2e-2


def test_model_step_wait_timeout_is_reported_and_handle_stays_usable(G):
    from decoder_only_transformer_02_b200.synthetic import token_batches
    cfgd = dict(n_layer=2, n_head=2, n_embd=128, vocab_size=500, padded_vocab=512, block_size=256)
    m = G.GPT2(G.GPT2Config(**cfgd, max_B=2, max_T=128, precision=G.GPT2_BF16), seed=9)
    m.set_graphs(False)
    (tok, tgt), = token_batches("zipf", 500, 2, 128, 1, seed=4)
    dtok, dtgt = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    m.zero_grad()
    ref = m.forward_backward(dtok, dtgt, 1.0, want_loss=True)
    g_ref = m.get_grads()
    G.set_wait_limit_ns(1)
    with pytest.raises(G.GPT2Error) as e:
        m.forward_backward(dtok, dtgt, 1.0, want_loss=True)
    assert e.value.name == "ECUDA"
    G.set_wait_limit_ns(0)
    m.zero_grad()
    again = m.forward_backward(dtok, dtgt, 1.0, want_loss=True)
    assert math.isfinite(again) and again == ref
    np.testing.assert_array_equal(m.get_grads(), g_ref)
    m.close()
