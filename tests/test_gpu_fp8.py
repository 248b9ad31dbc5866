"""The FP8 (e4m3) GEMM path against the oracle: per-tensor quantization
codes and scales bit-exact (the scaled value is formed in fp32 on both sides,
so the rounding decision is the same), the product within 1e-5 of the fp64
product of the decoded codes (products of e4m3 codes are exact in fp32; only
the fp32 accumulation rounds), on both tile forms, with ragged edges and a K
that is not a multiple of the 128-element k-block."""

import numpy as np
import pytest

from oracle import fp8
from tests.helpers import rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


def gpu_quantize(g, x, dtype):
    import torch
    xd = torch.from_numpy(x).cuda()
    if dtype == "bf16":
        xd = xd.to(torch.bfloat16)
    q = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(g.fp8_quantize_workspace_bytes(), dtype=torch.uint8, device="cuda")
    g.fp8_quantize(xd, g.DTYPE_BF16 if dtype == "bf16" else g.DTYPE_F32, x.size, q, s, ws, ws.numel())
    torch.cuda.synchronize()
    return q, s


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_bit_exact(g, dtype):
    import torch
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(1 << 18) * 0.02, rng.standard_normal(1000) * 1e-7,
                        [0.0, -0.0, 1e-30, -1e-30]]).astype(np.float32)
    if dtype == "bf16":
        x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    q, s = gpu_quantize(g, x, dtype)
    qo, so = fp8.quantize(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    assert s.item() == float(so)


@pytest.fixture(params=[1, 0], ids=["sm_pairs", "one_sm"])
def tiles(request, g):
    g.gptx_set_gemm_cta_pairs(request.param)
    yield request.param
    g.gptx_set_gemm_cta_pairs(1)


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (200, 384, 160), (777, 520, 1024), (2048, 768, 768)])
def test_fp8_gemm_matches_oracle(g, tiles, M, N, K):
    import torch
    rng = np.random.default_rng(M + N + K)
    A = (rng.standard_normal((M, K)) * 0.05).astype(np.float32)
    B = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qa, sa = gpu_quantize(g, A.reshape(-1), "f32")
    qb, sb = gpu_quantize(g, B.reshape(-1), "f32")
    qao, sao = fp8.quantize(A.reshape(-1))
    qbo, sbo = fp8.quantize(B.reshape(-1))
    ref = fp8.gemm(qao.reshape(M, K), sao, qbo.reshape(N, K), sbo)
    C = torch.full((M, N), 9.0, dtype=torch.float32, device="cuda")
    g.gptx_gemm_fp8(M, N, K, qa, K, qb, K, sa, sb, g.DTYPE_F32, C, N)
    torch.cuda.synchronize()
    assert g.ngram_sync_status() == g.GPT_OK
    assert rel_l2(C.cpu().numpy(), ref) < 1e-5
    Cb = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    g.gptx_gemm_fp8(M, N, K, qa, K, qb, K, sa, sb, g.DTYPE_BF16, Cb, N)
    torch.cuda.synchronize()
    assert rel_l2(Cb.float().cpu().numpy(), ref) < 4e-3
    # and against the unquantized product: the e4m3 rounding error of the path
    assert rel_l2(C.cpu().numpy(), A.astype(np.float64) @ B.astype(np.float64).T) < 6e-2
