"""gpt2_attention_backward_noalloc: the attention backward for callers that
cannot allocate device memory (its scratch is a fixed array inside the
library).  Called through the C ABI twice in a row, with different and larger
inputs the second time so that the array's leftover contents are exercised, and
compared with the allocating entry point gpt2_attention_backward at the
attention tests' tolerance.  Both entry points run the same deterministic
kernels on the same inputs, so the outputs must be bit-identical.  Kept in a
file of its own that collects last."""
import numpy as np
import pytest

from tests.gpu_util import from_dev, need_gpu, to_dev_bf16, torch

pytestmark = pytest.mark.gpu


def _inputs(B, T, H, seed):
    from decoder_only_transformer_02_b200 import gpt2 as G
    from decoder_only_transformer_02_b200.synthetic import normal_array
    C = 64 * H
    qkv = to_dev_bf16(normal_array((B, T, 3 * C), seed))
    do = to_dev_bf16(normal_array((B, T, C), seed + 1))
    out = torch.empty(B, T, C, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
    G.attention_forward(qkv, out, lse, B, T, H)
    return qkv, do, out, lse


def test_noalloc_attention_backward_matches_allocating_entry_point():
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    for B, T, H, seed in [(2, 200, 3, 11), (8, 1024, 12, 12)]:
        C = 64 * H
        qkv, do, out, lse = _inputs(B, T, H, seed)
        ref = torch.empty(B, T, 3 * C, dtype=torch.bfloat16, device="cuda")
        work = torch.empty(G.attention_workspace_floats(B, T, H), dtype=torch.float32, device="cuda")
        G.attention_backward(qkv, out, do, lse, ref, work, B, T, H)
        got = torch.full((B, T, 3 * C), float("nan"), dtype=torch.bfloat16, device="cuda")
        G.attention_backward_noalloc(qkv, out, do, lse, got, B, T, H)
        G.check_device_error()
        assert np.all(np.isfinite(from_dev(got)))
        assert torch.equal(got, ref)


def test_noalloc_rejects_sizes_beyond_its_array():
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    B, H = 1, 1
    T = G.ATTN_NOALLOC_MAX_ROWS + 64
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(G.GPT2Error) as e:
        G.attention_backward_noalloc(dummy, dummy, dummy, lse, dummy, B, T, H)
    assert e.value.name == "EINVAL"
    # B*H beyond one grid row per (batch, head), with B*H*T inside the array
    with pytest.raises(G.GPT2Error) as e:
        G.attention_backward_noalloc(dummy, dummy, dummy, lse, dummy, 65536, 1, 1)
    assert e.value.name == "EINVAL"
