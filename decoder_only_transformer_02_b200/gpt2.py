"""Thin Python binding of libgpt2 (include/gpt2.h): argument marshalling only.

Every step of the training step runs in the library's CUDA kernels; this module
converts Python / torch / numpy arguments to the C ABI's plain pointers and
sizes and turns status codes into exceptions.  There is no other code path:
if the library is missing the import of this module's functions fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgpt2.so")
_lib = None

GPT2_FP32 = 0
GPT2_BF16 = 1
_ERRS = {-1: "EINVAL", -2: "ECUDA", -3: "ETOKEN", -4: "ENOMEM", -5: "ESTATE", -6: "ENONFINITE"}

EXPORTED = [
    "gpt2_create", "gpt2_destroy", "gpt2_set_stream", "gpt2_forward", "gpt2_backward", "gpt2_forward_backward",
    "gpt2_zero_grad", "gpt2_adamw_step", "gpt2_train_step", "gpt2_lr_at", "gpt2_num_params", "gpt2_get_params",
    "gpt2_set_params", "gpt2_get_grads", "gpt2_get_adam_state", "gpt2_set_adam_state", "gpt2_get_logits",
    "gpt2_get_argmax", "gpt2_get_losses", "gpt2_last_loss", "gpt2_get_embed_keys", "gpt2_kernel_launches",
    "gpt2_last_error", "gpt2_attention_forward", "gpt2_attention_backward", "gpt2_attention_workspace_floats",
    "gpt2_matmul_bf16", "gpt2_matmul_workspace_bytes", "gpt2_set_timing", "gpt2_get_timing",
    "gpt2_attention_backward_noalloc", "gpt2_set_graphs", "gpt2_check_device_error", "gpt2_set_wait_limit_ns",
    "gpt2_prefill", "gpt2_decode_step", "gpt2_get_decode_logits", "gpt2_check_guards",
    "gpt2_debug_overwrite_guard",
]
ATTN_NOALLOC_MAX_ROWS = 1 << 19  # padded (batch, head, position) rows
KCLASSES = ["matmul", "attention_fwd", "attention_bwd", "layernorm_fwd", "layernorm_bwd", "cross_entropy",
            "optimizer", "embedding", "other"]


class GPT2Error(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{_ERRS.get(code, code)}: {msg}")
        self.code = code
        self.name = _ERRS.get(code, str(code))


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("n_layer", "n_head", "n_embd", "vocab_size", "padded_vocab",
                                             "block_size", "max_B", "max_T", "precision")]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libgpt2.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libgpt2.so not built ({_LIB_PATH}); run python -m decoder_only_transformer_02_b200.build")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F, D, L, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "gpt2_create": (I, [ctypes.POINTER(_Config), ctypes.c_uint64, ctypes.POINTER(P)]),
        "gpt2_destroy": (None, [P]),
        "gpt2_set_stream": (I, [P, P]),
        "gpt2_forward": (I, [P, P, P, I, I, P]),
        "gpt2_backward": (I, [P, F]),
        "gpt2_forward_backward": (I, [P, P, P, I, I, F, P]),
        "gpt2_zero_grad": (I, [P]),
        "gpt2_adamw_step": (I, [P, F, F, F, F, F, F, P]),
        "gpt2_train_step": (I, [P, P, P, I, I, I, F, F, F, F, F, F, P, P]),
        "gpt2_lr_at": (D, [I, D, D, I, I]),
        "gpt2_num_params": (L, [P]),
        "gpt2_get_params": (I, [P, P]),
        "gpt2_set_params": (I, [P, P]),
        "gpt2_get_grads": (I, [P, P]),
        "gpt2_get_adam_state": (I, [P, P, P, P]),
        "gpt2_set_adam_state": (I, [P, P, P, L]),
        "gpt2_get_logits": (I, [P, P]),
        "gpt2_get_argmax": (I, [P, P]),
        "gpt2_get_losses": (I, [P, P]),
        "gpt2_last_loss": (I, [P, P]),
        "gpt2_get_embed_keys": (I, [P, P]),
        "gpt2_kernel_launches": (L, [P]),
        "gpt2_check_guards": (I, [P, P]),
        "gpt2_debug_overwrite_guard": (I, [P, I]),
        "gpt2_last_error": (ctypes.c_char_p, [P]),
        "gpt2_attention_forward": (I, [P, P, P, I, I, I, P]),
        "gpt2_attention_backward": (I, [P, P, P, P, P, P, I, I, I, P]),
        "gpt2_attention_workspace_floats": (L, [I, I, I]),
        "gpt2_matmul_bf16": (I, [P, L, I, P, L, I, I, I, I, I, P, P, P, P, P, L, P, S, P]),
        "gpt2_matmul_workspace_bytes": (S, [I, I, I]),
        "gpt2_set_timing": (I, [P, I]),
        "gpt2_get_timing": (I, [P, P, P, P, P]),
        "gpt2_attention_backward_noalloc": (I, [P, P, P, P, P, I, I, I, P]),
        "gpt2_set_graphs": (I, [P, I]),
        "gpt2_check_device_error": (I, [P]),
        "gpt2_set_wait_limit_ns": (I, [ctypes.c_uint64]),
        "gpt2_prefill": (I, [P, P, I, I, F, I, ctypes.c_uint64, P]),
        "gpt2_decode_step": (I, [P, P, I, I, F, I, ctypes.c_uint64, P]),
        "gpt2_get_decode_logits": (I, [P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _ptr(x):
    """Address of a torch tensor (data_ptr), numpy array, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        assert x.flags["C_CONTIGUOUS"]
        return x.ctypes.data
    return x.data_ptr()  # torch.Tensor


def _stream_ptr(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream  # torch.cuda.Stream


@dataclass
class GPT2Config:
    n_layer: int = 12
    n_head: int = 12
    n_embd: int = 768
    vocab_size: int = 50257
    padded_vocab: int = 50304
    block_size: int = 1024
    max_B: int = 16
    max_T: int = 1024
    precision: int = GPT2_BF16


class GPT2:
    """Handle on one model instance living on the current CUDA device."""

    def __init__(self, cfg: GPT2Config, seed: int = 1234, stream=None):
        lib = load_library()
        self.cfg = cfg
        c = _Config(cfg.n_layer, cfg.n_head, cfg.n_embd, cfg.vocab_size, cfg.padded_vocab, cfg.block_size,
                    cfg.max_B, cfg.max_T, cfg.precision)
        h = ctypes.c_void_p()
        r = lib.gpt2_create(ctypes.byref(c), ctypes.c_uint64(seed), ctypes.byref(h))
        if r != 0:
            raise GPT2Error(r, "gpt2_create failed (see stderr)")
        self._h = h
        self._lib = lib
        self.B = self.T = 0
        if stream is not None:
            self.set_stream(stream)

    # -- lifetime
    def close(self):
        if getattr(self, "_h", None):
            self._lib.gpt2_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, r):
        if r != 0:
            raise GPT2Error(r, self._lib.gpt2_last_error(self._h).decode())

    # -- step
    def set_stream(self, stream):
        self._check(self._lib.gpt2_set_stream(self._h, _stream_ptr(stream)))

    def forward(self, tokens, targets=None, want_loss=False):
        B, T = tokens.shape
        self.B, self.T = B, T
        out = ctypes.c_float()
        self._check(self._lib.gpt2_forward(self._h, _ptr(tokens), _ptr(targets), B, T,
                                           ctypes.byref(out) if want_loss else None))
        return out.value if want_loss else None

    def backward(self, loss_scale=1.0):
        self._check(self._lib.gpt2_backward(self._h, loss_scale))

    def forward_backward(self, tokens, targets, loss_scale=1.0, want_loss=False):
        B, T = tokens.shape
        self.B, self.T = B, T
        out = ctypes.c_float()
        self._check(self._lib.gpt2_forward_backward(self._h, _ptr(tokens), _ptr(targets), B, T, loss_scale,
                                                    ctypes.byref(out) if want_loss else None))
        return out.value if want_loss else None

    def zero_grad(self):
        self._check(self._lib.gpt2_zero_grad(self._h))

    def adamw_step(self, lr, wd=0.1, b1=0.9, b2=0.95, eps=1e-8, clip=1.0, want_norm=False):
        n = ctypes.c_float()
        self._check(self._lib.gpt2_adamw_step(self._h, lr, wd, b1, b2, eps, clip,
                                              ctypes.byref(n) if want_norm else None))
        return n.value if want_norm else None

    def train_step(self, h_tokens, h_targets, n_micro, B, T, lr, wd=0.1, b1=0.9, b2=0.95, eps=1e-8, clip=1.0,
                   want=True):
        """h_tokens / h_targets: HOST int32 buffers of n_micro*B*T ids (numpy
        array or pinned CPU torch tensor)."""
        self.B, self.T = B, T
        loss, norm = ctypes.c_float(), ctypes.c_float()
        self._check(self._lib.gpt2_train_step(self._h, _ptr(h_tokens), _ptr(h_targets), n_micro, B, T, lr, wd,
                                              b1, b2, eps, clip, ctypes.byref(loss) if want else None,
                                              ctypes.byref(norm) if want else None))
        return (loss.value, norm.value) if want else None

    def set_graphs(self, enable: bool):
        self._check(self._lib.gpt2_set_graphs(self._h, 1 if enable else 0))

    # -- generation
    def prefill(self, tokens, next_out, temperature=1.0, top_k=1, seed=0):
        """tokens: device int32 [B, T0]; next_out: device int32 [B] (receives
        the token at position T0)."""
        B, T0 = tokens.shape
        self._check(self._lib.gpt2_prefill(self._h, _ptr(tokens), B, T0, temperature, top_k, seed, _ptr(next_out)))

    def decode_step(self, tokens, pos, next_out, temperature=1.0, top_k=1, seed=0):
        """tokens: device int32 [B] at position pos; next_out: device int32 [B]."""
        B = tokens.shape[0]
        self._check(self._lib.gpt2_decode_step(self._h, _ptr(tokens), B, pos, temperature, top_k, seed,
                                               _ptr(next_out)))

    def get_decode_logits(self, B) -> np.ndarray:
        a = np.empty((B, self.cfg.padded_vocab), dtype=np.float32)
        self._check(self._lib.gpt2_get_decode_logits(self._h, a.ctypes.data))
        return a

    # -- measurement support
    def set_timing(self, enable: bool):
        self._check(self._lib.gpt2_set_timing(self._h, 1 if enable else 0))

    def get_timing(self) -> dict:
        """Per kernel class: device ms, operations, algorithmic FLOPs and bytes
        since the last call (then reset)."""
        n = len(KCLASSES)
        ms = np.zeros(n, dtype=np.float64)
        ops = np.zeros(n, dtype=np.int64)
        fl = np.zeros(n, dtype=np.float64)
        by = np.zeros(n, dtype=np.float64)
        self._check(self._lib.gpt2_get_timing(self._h, ms.ctypes.data, ops.ctypes.data, fl.ctypes.data,
                                              by.ctypes.data))
        return {k: dict(ms=float(ms[i]), ops=int(ops[i]), flops=float(fl[i]), bytes=float(by[i]))
                for i, k in enumerate(KCLASSES)}

    # -- accessors
    @property
    def num_params(self) -> int:
        return int(self._lib.gpt2_num_params(self._h))

    @property
    def kernel_launches(self) -> int:
        return int(self._lib.gpt2_kernel_launches(self._h))

    def check_guards(self) -> int:
        """Number of guard bytes after the handle's device buffers that some
        kernel overwrote (0 when every write stayed inside its buffer)."""
        n = ctypes.c_int64(0)
        self._check(self._lib.gpt2_check_guards(self._h, ctypes.byref(n)))
        return int(n.value)

    def debug_overwrite_guard(self, index: int):
        self._check(self._lib.gpt2_debug_overwrite_guard(self._h, index))

    def get_params(self) -> np.ndarray:
        a = np.empty(self.num_params, dtype=np.float32)
        self._check(self._lib.gpt2_get_params(self._h, a.ctypes.data))
        return a

    def set_params(self, flat: np.ndarray):
        a = np.ascontiguousarray(flat, dtype=np.float32)
        assert a.size == self.num_params
        self._check(self._lib.gpt2_set_params(self._h, a.ctypes.data))

    def get_grads(self) -> np.ndarray:
        a = np.empty(self.num_params, dtype=np.float32)
        self._check(self._lib.gpt2_get_grads(self._h, a.ctypes.data))
        return a

    def get_adam_state(self):
        m = np.empty(self.num_params, dtype=np.float32)
        v = np.empty(self.num_params, dtype=np.float32)
        t = ctypes.c_int64()
        self._check(self._lib.gpt2_get_adam_state(self._h, m.ctypes.data, v.ctypes.data, ctypes.byref(t)))
        return m, v, t.value

    def set_adam_state(self, m, v, t):
        m = np.ascontiguousarray(m, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        self._check(self._lib.gpt2_set_adam_state(self._h, m.ctypes.data, v.ctypes.data, int(t)))

    def get_logits(self) -> np.ndarray:
        a = np.empty((self.B, self.T, self.cfg.padded_vocab), dtype=np.float32)
        self._check(self._lib.gpt2_get_logits(self._h, a.ctypes.data))
        return a

    def get_argmax(self) -> np.ndarray:
        a = np.empty((self.B, self.T), dtype=np.int32)
        self._check(self._lib.gpt2_get_argmax(self._h, a.ctypes.data))
        return a

    def get_losses(self) -> np.ndarray:
        a = np.empty((self.B, self.T), dtype=np.float32)
        self._check(self._lib.gpt2_get_losses(self._h, a.ctypes.data))
        return a

    def last_loss(self) -> float:
        x = ctypes.c_float()
        self._check(self._lib.gpt2_last_loss(self._h, ctypes.byref(x)))
        return x.value

    def embed_keys(self) -> np.ndarray:
        a = np.empty(self.B * self.T, dtype=np.uint32)
        self._check(self._lib.gpt2_get_embed_keys(self._h, a.ctypes.data))
        return a


# ------------------------------------------------------------ standalone ops

def _op_check(r, what):
    if r != 0:
        raise GPT2Error(r, what)


def attention_forward(qkv, out, lse, B, T, H, stream=None):
    _op_check(load_library().gpt2_attention_forward(_ptr(qkv), _ptr(out), _ptr(lse), B, T, H, _stream_ptr(stream)),
              "gpt2_attention_forward")


def attention_workspace_floats(B, T, H) -> int:
    return int(load_library().gpt2_attention_workspace_floats(B, T, H))


def attention_backward(qkv, out, dout, lse, dqkv, work, B, T, H, stream=None):
    _op_check(load_library().gpt2_attention_backward(_ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dqkv),
                                                     _ptr(work), B, T, H, _stream_ptr(stream)),
              "gpt2_attention_backward")


def attention_backward_noalloc(qkv, out, dout, lse, dqkv, B, T, H, stream=None):
    """gpt2_attention_backward with the library's fixed scratch array (no
    allocation; B*H*ceil(T/128)*128 <= ATTN_NOALLOC_MAX_ROWS; calls must not overlap)."""
    _op_check(load_library().gpt2_attention_backward_noalloc(_ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse),
                                                             _ptr(dqkv), B, T, H, _stream_ptr(stream)),
              "gpt2_attention_backward_noalloc")


def matmul_bf16(A, lda, a_mn, Bm, ldb, b_mn, M, N, K, epi, bias=None, resid=None, out=None, out2=None, aux=None,
                ldc=None, work=None, work_bytes=0, stream=None):
    _op_check(load_library().gpt2_matmul_bf16(_ptr(A), lda, a_mn, _ptr(Bm), ldb, b_mn, M, N, K, epi, _ptr(bias),
                                              _ptr(resid), _ptr(out), _ptr(out2), _ptr(aux),
                                              N if ldc is None else ldc, _ptr(work), work_bytes,
                                              _stream_ptr(stream)),
              "gpt2_matmul_bf16")


def matmul_workspace_bytes(M, N, K) -> int:
    return int(load_library().gpt2_matmul_workspace_bytes(M, N, K))


def check_device_error(stream=None):
    """Synchronise `stream`, then read and clear the device's error word:
    raises GPT2Error (ECUDA) when a kernel gave up on a wait since the last check."""
    _op_check(load_library().gpt2_check_device_error(_stream_ptr(stream)), "a device-side wait gave up")


def set_wait_limit_ns(limit_ns: int):
    """Testing support: the device-side pipeline wait limit (0 = default 2 s)."""
    _op_check(load_library().gpt2_set_wait_limit_ns(int(limit_ns)), "gpt2_set_wait_limit_ns")


def lr_at(it, max_lr=6e-4, min_lr=6e-5, warmup=715, max_steps=19073) -> float:
    return float(load_library().gpt2_lr_at(it, max_lr, min_lr, warmup, max_steps))
