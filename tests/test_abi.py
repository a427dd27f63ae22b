"""The C-ABI library builds, loads and exports every entry point the header
declares; host-side argument checks reject bad configurations before any
device work.  No GPU needed."""
import ctypes
import math
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gpt2.h")


@pytest.fixture(scope="module")
def lib():
    from decoder_only_transformer_02_b200 import build, gpt2
    build.build()
    return gpt2.load_library()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt2_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_names():
    from decoder_only_transformer_02_b200 import gpt2
    assert declared_symbols() == sorted(gpt2.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    from decoder_only_transformer_02_b200 import gpt2
    out = subprocess.run(["nm", "-D", "--defined-only", gpt2.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (gpt2_\w+)", out))
    for s in declared_symbols():
        assert s in exported, s
        assert hasattr(lib, s)


def test_library_is_built_for_sm100a(lib):
    from decoder_only_transformer_02_b200 import gpt2
    out = subprocess.run(["cuobjdump", "--list-elf", gpt2.library_path()], capture_output=True, text=True).stdout
    assert "sm_100a" in out


def test_lr_schedule_matches_oracle(lib):
    from decoder_only_transformer_02_b200 import gpt2
    from oracle import gpt2_oracle as O
    for it in (0, 1, 100, 714, 715, 716, 5000, 9894, 19072, 19073, 19074, 30000):
        assert math.isclose(gpt2.lr_at(it), O.lr_at(it), rel_tol=1e-12, abs_tol=0)


@pytest.mark.parametrize("bad", [
    dict(n_embd=96), dict(n_embd=100, n_head=4), dict(padded_vocab=500), dict(padded_vocab=100000),
    dict(max_T=2048), dict(max_B=64), dict(precision=7), dict(n_head=3, n_embd=384),
])
def test_create_rejects_bad_config_without_device_work(lib, bad):
    from decoder_only_transformer_02_b200 import gpt2
    cfg = dict(n_layer=2, n_head=2, n_embd=128, vocab_size=500, padded_vocab=512, block_size=1024, max_B=16,
               max_T=1024, precision=gpt2.GPT2_BF16)
    cfg.update(bad)
    c = gpt2._Config(*[cfg[k] for k, _ in gpt2._Config._fields_])
    h = ctypes.c_void_p()
    assert lib.gpt2_create(ctypes.byref(c), 1, ctypes.byref(h)) == -1
    assert not h.value


def test_null_arguments_rejected(lib):
    assert lib.gpt2_create(None, 1, None) == -1
    assert lib.gpt2_forward(None, None, None, 1, 1, None) == -1
    assert lib.gpt2_attention_forward(None, None, None, 1, 1, 1, None) == -1
    assert lib.gpt2_matmul_bf16(None, 8, 0, None, 8, 0, 8, 8, 8, 0, None, None, None, None, None, 8, None, 0,
                                None) == -1
    assert lib.gpt2_last_error(None) == b"handle is NULL"
    lib.gpt2_destroy(None)
