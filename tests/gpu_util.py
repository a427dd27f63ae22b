"""Helpers shared by the GPU parity tests (comparison metrics, bf16 rounding)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to the nearest bf16 (as the device does), return fp64."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.float().numpy().astype(np.float64)


def to_dev_bf16(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def from_dev(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def rel_max_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref)) / (den if den > 0 else 1.0))


def cosine(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(np.dot(a, b) / (na * nb))


def per_tensor(flat_got, flat_ref, cfg, metric):
    from oracle import gpt2_oracle as O
    out = {}
    off = 0
    for name, shape, _ in O.param_specs(cfg):
        n = int(np.prod(shape))
        out[name] = metric(flat_got[off:off + n], flat_ref[off:off + n])
        off += n
    return out
