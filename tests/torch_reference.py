"""An independent CPU restatement of the GPT-2 step built from PyTorch library
routines (F.layer_norm, F.linear, F.scaled_dot_product_attention, F.gelu,
F.cross_entropy, torch.autograd, torch.optim.AdamW, clip_grad_norm_).

Test-only: it pins the NumPy oracle against textbook library implementations.
It shares no code with the oracle (it only reads the same flat-order layout).
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F


def _specs(cfg):
    C, V, P = cfg.n_embd, cfg.padded_vocab, cfg.block_size
    s = [("wte", (V, C)), ("wpe", (P, C))]
    for l in range(cfg.n_layer):
        s += [(f"h{l}.ln1.g", (C,)), (f"h{l}.ln1.b", (C,)), (f"h{l}.attn.w", (3 * C, C)),
              (f"h{l}.attn.b", (3 * C,)), (f"h{l}.proj.w", (C, C)), (f"h{l}.proj.b", (C,)),
              (f"h{l}.ln2.g", (C,)), (f"h{l}.ln2.b", (C,)), (f"h{l}.fc.w", (4 * C, C)),
              (f"h{l}.fc.b", (4 * C,)), (f"h{l}.mproj.w", (C, 4 * C)), (f"h{l}.mproj.b", (C,))]
    s += [("lnf.g", (C,)), ("lnf.b", (C,))]
    return s


def make_params(flat: np.ndarray, cfg, dtype=torch.float64):
    out, off = {}, 0
    for name, shape in _specs(cfg):
        n = int(np.prod(shape))
        t = torch.tensor(flat[off:off + n].reshape(shape), dtype=dtype, requires_grad=True)
        out[name] = t
        off += n
    return out


def flatten_grads(params, cfg) -> np.ndarray:
    return np.concatenate([params[n].grad.detach().numpy().reshape(-1) for n, _ in _specs(cfg)])


def flatten_values(params, cfg) -> np.ndarray:
    return np.concatenate([params[n].detach().numpy().reshape(-1) for n, _ in _specs(cfg)])


def model_loss(p, cfg, tokens, targets, eps=1e-5):
    tok = torch.as_tensor(np.asarray(tokens), dtype=torch.long)
    tgt = torch.as_tensor(np.asarray(targets), dtype=torch.long)
    B, T = tok.shape
    C, H = cfg.n_embd, cfg.n_head
    d = C // H
    x = F.embedding(tok, p["wte"]) + p["wpe"][:T]
    for l in range(cfg.n_layer):
        pre = f"h{l}."
        h = F.layer_norm(x, (C,), p[pre + "ln1.g"], p[pre + "ln1.b"], eps)
        qkv = F.linear(h, p[pre + "attn.w"], p[pre + "attn.b"])
        q, k, v = qkv.split(C, dim=-1)
        q = q.view(B, T, H, d).transpose(1, 2)
        k = k.view(B, T, H, d).transpose(1, 2)
        v = v.view(B, T, H, d).transpose(1, 2)
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
        o = o.transpose(1, 2).reshape(B, T, C)
        x = x + F.linear(o, p[pre + "proj.w"], p[pre + "proj.b"])
        h2 = F.layer_norm(x, (C,), p[pre + "ln2.g"], p[pre + "ln2.b"], eps)
        a = F.gelu(F.linear(h2, p[pre + "fc.w"], p[pre + "fc.b"]), approximate="tanh")
        x = x + F.linear(a, p[pre + "mproj.w"], p[pre + "mproj.b"])
    xf = F.layer_norm(x, (C,), p["lnf.g"], p["lnf.b"], eps)
    logits = F.linear(xf, p["wte"])
    loss = F.cross_entropy(logits.reshape(B * T, -1), tgt.reshape(-1))
    return logits, loss


def torch_train_step(flat, m, v, t, cfg, micro_batches, lr, wd=0.1, betas=(0.9, 0.95), eps=1e-8, clip=1.0):
    """Accumulate over micro-batches (loss / n), clip_grad_norm_, torch AdamW
    with decay only on 2D tensors.  Returns new flat params, m, v, norm."""
    p = make_params(flat, cfg)
    names = [n for n, _ in _specs(cfg)]
    decay = [p[n] for n in names if p[n].dim() >= 2]
    nodecay = [p[n] for n in names if p[n].dim() < 2]
    opt = torch.optim.AdamW([{"params": decay, "weight_decay": wd},
                             {"params": nodecay, "weight_decay": 0.0}],
                            lr=lr, betas=betas, eps=eps, foreach=False, fused=False)
    # load moments and step count
    off = 0
    for n, shape in _specs(cfg):
        k = int(np.prod(shape))
        if t > 1:
            st = opt.state[p[n]]
            st["step"] = torch.tensor(float(t - 1), dtype=torch.float64)
            st["exp_avg"] = torch.tensor(m[off:off + k].reshape(shape), dtype=torch.float64)
            st["exp_avg_sq"] = torch.tensor(v[off:off + k].reshape(shape), dtype=torch.float64)
        off += k
    nmb = len(micro_batches)
    for tok, tgt in micro_batches:
        _, loss = model_loss(p, cfg, tok, tgt)
        (loss / nmb).backward()
    norm = torch.nn.utils.clip_grad_norm_([p[n] for n in names], clip)
    opt.step()
    mm = np.concatenate([opt.state[p[n]]["exp_avg"].numpy().reshape(-1) for n in names])
    vv = np.concatenate([opt.state[p[n]]["exp_avg_sq"].numpy().reshape(-1) for n in names])
    return flatten_values(p, cfg), mm, vv, float(norm)
