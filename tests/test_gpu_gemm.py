"""tcgen05 GEMM through the C ABI (gpt2_matmul_bf16) against the oracle's
linear-layer formulas evaluated in fp64 on the same bf16-rounded operands.
Covers the forward (K-major x K-major), dgrad (K-major x MN-major) and wgrad
(MN-major x MN-major) layouts, every fused epilogue, ragged M/N/K tails and the
split-K path."""
import numpy as np
import pytest

from tests.gpu_util import bf16_round, from_dev, need_gpu, rel_max_err, to_dev_bf16, torch

pytestmark = pytest.mark.gpu


def _lib():
    need_gpu()
    from decoder_only_transformer_02_b200 import gpt2 as G
    G.load_library()
    return G


@pytest.fixture(params=["pair", "single"], autouse=True)
def kernel(request, monkeypatch):
    """Run every case on both GEMM kernels: the 2-SM pair kernel (the default
    for N > 128 and M > 128) and the 1-SM kernel (GPT2_GEMM_2SM=0)."""
    if request.param == "single":
        monkeypatch.setenv("GPT2_GEMM_2SM", "0")
    else:
        monkeypatch.delenv("GPT2_GEMM_2SM", raising=False)
    return request.param


def _operands(M, N, K, seed):
    from decoder_only_transformer_02_b200.synthetic import normal_array
    A = bf16_round(normal_array((M, K), seed))        # logical A[m, k]
    Bm = bf16_round(normal_array((N, K), seed + 1))   # logical B[n, k]
    return A, Bm


def _dev(A, mn):
    # K-major: stored [M][K]; MN-major: stored [K][M]
    return to_dev_bf16(A.T.copy() if mn else A)


SHAPES = [(256, 256, 128), (304, 384, 200), (128, 128, 64), (1000, 2304, 768), (136, 144, 72)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1), (1, 0)])
def test_gemm_fp32_out_all_layouts(M, N, K, a_mn, b_mn):
    G = _lib()
    A, Bm = _operands(M, N, K, 10 + M)
    out = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    G.matmul_bf16(_dev(A, a_mn), M if a_mn else K, a_mn, _dev(Bm, b_mn), N if b_mn else K, b_mn, M, N, K, 1,
                  out=out, ldc=N)
    torch.cuda.synchronize()
    ref = A @ Bm.T
    assert rel_max_err(from_dev(out), ref) < 1e-5


@pytest.mark.parametrize("M,N,K", [(300, 384, 200), (1000, 2304, 768), (200, 136, 64)])
def test_gemm_epilogues(M, N, K):
    from oracle import gpt2_oracle as O
    G = _lib()
    from decoder_only_transformer_02_b200.synthetic import normal_array
    A, W = _operands(M, N, K, 3)
    bias = normal_array((N,), 5).astype(np.float32)
    resid = normal_array((M, N), 6).astype(np.float32)
    dA, dW = to_dev_bf16(A), to_dev_bf16(W)
    db = torch.from_numpy(bias).cuda()
    acc = O.linear_forward(A, W, bias.astype(np.float64))
    # 0: bf16 out + bias
    o = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    G.matmul_bf16(dA, K, 0, dW, K, 0, M, N, K, 0, bias=db, out=o)
    torch.cuda.synchronize()
    assert rel_max_err(from_dev(o), acc) < 8e-3
    # 2: residual fp32
    dr = torch.from_numpy(resid).cuda()
    o2 = torch.empty(M, N, dtype=torch.float32, device="cuda")
    G.matmul_bf16(dA, K, 0, dW, K, 0, M, N, K, 2, bias=db, resid=dr, out=o2)
    torch.cuda.synchronize()
    assert rel_max_err(from_dev(o2), acc + resid) < 1e-5
    # 3: GELU (u stored in bf16, gelu of the stored u)
    u = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    G.matmul_bf16(dA, K, 0, dW, K, 0, M, N, K, 3, bias=db, out=u, out2=a)
    torch.cuda.synchronize()
    u_ref = bf16_round(acc)
    assert np.max(np.abs(from_dev(u) - u_ref)) <= 1e-6 + 8e-3 * np.max(np.abs(acc))
    assert rel_max_err(from_dev(a), O.gelu_tanh(u_ref)) < 8e-3
    # 4: dgrad with GELU' of aux
    aux = u
    o4 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    acc0 = A @ W.T
    G.matmul_bf16(dA, K, 0, dW, K, 0, M, N, K, 4, out=o4, aux=aux)
    torch.cuda.synchronize()
    ref4 = acc0 * O.gelu_tanh_grad(from_dev(aux))
    assert rel_max_err(from_dev(o4), ref4) < 8e-3
    # 5: accumulate into fp32 (no split)
    o5 = torch.from_numpy(resid.copy()).cuda()
    G.matmul_bf16(dA, K, 0, dW, K, 0, M, N, K, 5, out=o5)
    torch.cuda.synchronize()
    assert rel_max_err(from_dev(o5), resid + acc0) < 1e-5


@pytest.mark.parametrize("N,Kin,M", [(768, 768, 16384), (2304, 768, 4096), (256, 384, 3000)])
def test_wgrad_split_k_matches_oracle(N, Kin, M):
    """dW[N,Kin] += dY[M,N]^T X[M,Kin] with the split-K scratch path."""
    from oracle import gpt2_oracle as O
    G = _lib()
    from decoder_only_transformer_02_b200.synthetic import normal_array
    dY = bf16_round(normal_array((M, N), 1))
    X = bf16_round(normal_array((M, Kin), 2))
    g0 = normal_array((N, Kin), 3).astype(np.float32)
    ws_bytes = G.matmul_workspace_bytes(N, Kin, M)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device="cuda")
    out = torch.from_numpy(g0.copy()).cuda()
    G.matmul_bf16(to_dev_bf16(dY), N, 1, to_dev_bf16(X), Kin, 1, N, Kin, M, 5, out=out, ldc=Kin, work=ws,
                  work_bytes=ws_bytes)
    torch.cuda.synchronize()
    _, dw_ref, _ = O.linear_backward(dY, X, np.zeros((N, Kin)))
    assert rel_max_err(from_dev(out), g0 + dw_ref) < 1e-5
    # deterministic: a second identical call gives bit-identical results
    out2 = torch.from_numpy(g0.copy()).cuda()
    G.matmul_bf16(to_dev_bf16(dY), N, 1, to_dev_bf16(X), Kin, 1, N, Kin, M, 5, out=out2, ldc=Kin, work=ws,
                  work_bytes=ws_bytes)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_lm_head_shape_sampled_rows():
    """The forward launch shape of the tied lm_head (M=16384, N=50304, K=768):
    sampled rows against the oracle computed row by row."""
    G = _lib()
    from decoder_only_transformer_02_b200.synthetic import normal_array
    M, N, K = 16384, 50304, 768
    X = torch.from_numpy(normal_array((M, K), 7)).to(torch.bfloat16).cuda()
    W = (torch.from_numpy(normal_array((N, K), 8)) * 0.02).to(torch.bfloat16).cuda()
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    G.matmul_bf16(X, K, 0, W, K, 0, M, N, K, 0, out=out)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(M, 24, replace=False)
    Wd = from_dev(W)
    for r in rows:
        ref = from_dev(X[r:r + 1]) @ Wd.T
        assert rel_max_err(from_dev(out[r:r + 1]), ref) < 8e-3


def test_bad_alignment_rejected():
    G = _lib()
    a = torch.zeros(64 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(64, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(G.GPT2Error):
        G.matmul_bf16(a[1:].data_ptr(), 64, 0, a, 64, 0, 64, 64, 64, 1, out=o)
    with pytest.raises(G.GPT2Error):
        G.matmul_bf16(a, 60, 0, a, 64, 0, 64, 64, 60, 1, out=o)
