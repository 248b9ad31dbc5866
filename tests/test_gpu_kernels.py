"""Kernel-level parity on the GPU, through the C ABI: the tcgen05 GEMM in every
operand layout, and the bigram-table hash / gather / sparse update against the
fp64 oracle (bit-exact on row ids and updated-row sets)."""

import numpy as np
import pytest

from oracle import hashing, optim
from synthetic import round_to_bf16, zipf_stream
from tests.helpers import device_ints, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    return g


def _bf16_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


@pytest.fixture(params=[1, 0], ids=["sm_pairs", "one_sm"])
def tiles(request, g):
    """Both tile forms: CTA pairs (256 x 256 tiles over two SMs) and one SM per tile."""
    g.gptx_set_gemm_cta_pairs(request.param)
    yield request.param
    g.gptx_set_gemm_cta_pairs(1)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 384, 160), (776, 264, 520), (256, 768, 768),
                                   (2048, 768, 320)])  # one SM: the last one runs on 192-column tiles
@pytest.mark.parametrize("a_k,b_k", [(1, 1), (1, 0), (0, 0), (0, 1)])
def test_gemm_layouts_match_fp64(g, tiles, M, N, K, a_k, b_k):
    import torch
    rng = np.random.default_rng(M * 7 + N * 3 + K + 11 * a_k + 5 * b_k)
    A = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    B = round_to_bf16(rng.standard_normal((N, K)).astype(np.float32))
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    Ad = _bf16_dev(A if a_k else A.T)
    Bd = _bf16_dev(B if b_k else B.T)
    C = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    g.gptx_gemm_bf16(M, N, K, Ad, K if a_k else M, a_k, Bd, K if b_k else N, b_k, C, N, 0, 1, None, 0)
    torch.cuda.synchronize()
    assert g.ngram_sync_status() == g.GPT_OK
    err = rel_l2(C.cpu().numpy(), ref)
    assert err < 1e-5, err
    # beta = 1 accumulates
    g.gptx_gemm_bf16(M, N, K, Ad, K if a_k else M, a_k, Bd, K if b_k else N, b_k, C, N, 1, 1, None, 0)
    torch.cuda.synchronize()
    assert rel_l2(C.cpu().numpy(), 2 * ref) < 1e-5


def test_gemm_split_k_is_deterministic_and_exact(g, tiles):
    import torch
    M, N, K = 768, 768, 4096
    rng = np.random.default_rng(5)
    A = round_to_bf16(rng.standard_normal((K, M)).astype(np.float32))   # stored [K, M]
    B = round_to_bf16(rng.standard_normal((K, N)).astype(np.float32))   # stored [K, N]
    ref = A.astype(np.float64).T @ B.astype(np.float64)
    ws = torch.empty(8 * M * N * 4, dtype=torch.uint8, device="cuda")
    outs = []
    for splits in (1, 4, 4):
        C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
        g.gptx_gemm_bf16(M, N, K, _bf16_dev(A), M, 0, _bf16_dev(B), N, 0, C, N, 0, splits, ws, ws.numel())
        torch.cuda.synchronize()
        outs.append(C.cpu().numpy())
    assert rel_l2(outs[0], ref) < 1e-5 and rel_l2(outs[1], ref) < 1e-5
    np.testing.assert_array_equal(outs[1], outs[2])


def test_ngram_hash_bit_exact(g):
    import torch
    B, T, V = 4, 333, 50304
    tok = zipf_stream(B * T, V, 3).reshape(B, T)
    for rows in (2097152, 1048576, 1000003):
        out = torch.empty((B, T), dtype=torch.int32, device="cuda")
        g.ngram_hash(device_ints(tok), B, T, V, 2654435761, 2246822519, rows, out)
        torch.cuda.synchronize()
        ref = hashing.bigram_rows(tok, V, 2654435761, 2246822519, rows)
        np.testing.assert_array_equal(out.cpu().numpy(), ref)
    assert g.ngram_sync_status() == g.GPT_OK


def test_ngram_hash_rejects_bad_tokens(g):
    import torch
    tok = np.array([[1, 2, 70000, 3]])
    out = torch.empty((1, 4), dtype=torch.int32, device="cuda")
    g.ngram_hash(device_ints(tok), 1, 4, 50304, 2654435761, 2246822519, 1024, out)
    assert g.ngram_sync_status() == g.GPT_ERR_INPUT
    assert g.ngram_sync_status() == g.GPT_OK   # cleared


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("R,d,n", [(5000, 768, 1000), (3000, 136, 999), (300, 2048, 33)])
def test_ngram_gather(g, dtype, R, d, n):
    """Rows of any width (whole and partial 16-byte passes, two passes of a
    warp), an odd number of rows (the bf16 kernel takes two a warp)."""
    import torch
    rng = np.random.default_rng(2)
    tab = rng.standard_normal((R, d)).astype(np.float32)
    if dtype == "bf16":
        tab = round_to_bf16(tab)
    rows = rng.integers(0, R, n)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dt = g.DTYPE_BF16 if dtype == "bf16" else g.DTYPE_F32
    T = torch.from_numpy(tab).to(tdt).cuda()
    out = torch.ones((n, d), dtype=tdt, device="cuda")
    g.ngram_gather(device_ints(rows), n, T, R, d, dt, out, 0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.float().cpu().numpy(), tab[rows])
    g.ngram_gather(device_ints(rows), n, T, R, d, dt, out, 1)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out.float().cpu().numpy(), 2 * tab[rows], rtol=1e-2 if dtype == "bf16" else 0)


@pytest.mark.parametrize("dtype,R,n,d", [("f32", 1000, 3000, 128), ("bf16", 2048, 6000, 768),
                                         ("bf16", 2097152, 32768, 768)])
def test_ngram_sparse_update_matches_oracle(g, dtype, R, n, d):
    """Zipf-skewed bigram rows: long segments, singletons, ragged piece tails."""
    import torch
    rng = np.random.default_rng(R + n)
    tok = zipf_stream(n + 1, 50304, R).reshape(1, n + 1)[:, :n]
    rows = hashing.bigram_rows(tok, 50304, 2654435761, 2246822519, R).reshape(-1)
    grad = rng.standard_normal((n, d)).astype(np.float32)
    touched = np.unique(rows)
    # build only the touched rows on the host; the table is initialised on the device
    tab0 = rng.standard_normal((len(touched), d)).astype(np.float32) * 0.02
    if dtype == "bf16":
        tab0 = round_to_bf16(tab0)
    s0 = np.abs(rng.standard_normal(len(touched))) * 0.1
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    T = torch.zeros((R, d), dtype=tdt, device="cuda")
    S = torch.zeros(R, dtype=torch.float32, device="cuda")
    idx = torch.from_numpy(touched).cuda()
    T[idx] = torch.from_numpy(tab0).to(tdt).cuda()
    S[idx] = torch.from_numpy(s0.astype(np.float32)).cuda()
    ws_bytes = g.ngram_sparse_update_workspace_bytes(n, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    upd = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    nupd = torch.zeros(1, dtype=torch.int32, device="cuda")
    lr, beta, eps = 0.01, 0.95, 1e-10
    g.ngram_sparse_update(T, S, R, d, g.DTYPE_BF16 if dtype == "bf16" else g.DTYPE_F32,
                          device_ints(rows), torch.from_numpy(grad).cuda(), n, lr, beta, eps,
                          upd, nupd, ws, ws_bytes)
    assert g.ngram_sync_status() == g.GPT_OK
    k = int(nupd.item())
    np.testing.assert_array_equal(upd[:k].cpu().numpy(), touched)
    # oracle on the touched rows only (compact index space); at full size a
    # sample of rows (the most frequent ones plus random ones), since each
    # row's update depends only on its own positions
    sel = np.arange(len(touched))
    if n > 8000:
        counts = np.bincount(np.searchsorted(touched, rows), minlength=len(touched))
        sel = np.unique(np.concatenate([np.argsort(-counts)[:40],
                                        rng.choice(len(touched), 200, replace=False)]))
    keep = np.isin(rows, touched[sel])
    remap = {r: i for i, r in enumerate(touched[sel])}
    crow = np.array([remap[r] for r in rows[keep]])
    W1, s1, u = optim.table_update(tab0[sel].astype(np.float64),
                                   s0[sel].astype(np.float32).astype(np.float64),
                                   crow, grad[keep].astype(np.float64), lr, beta, eps)
    tab0 = tab0[sel]
    Wg = T[idx[torch.from_numpy(sel).cuda()]].float().cpu().numpy()
    Sg = S[idx[torch.from_numpy(sel).cuda()]].cpu().numpy()
    tol = 2e-2 if dtype == "bf16" else 1e-4
    assert rel_l2(Wg - tab0, W1 - tab0) < tol
    assert rel_l2(Sg, s1) < tol
    # untouched rows stay zero
    mask = torch.ones(R, dtype=torch.bool, device="cuda")
    mask[idx] = False
    assert int((T[mask] != 0).sum()) == 0 and int((S[mask] != 0).sum()) == 0


def _run_update(g, rows, d, R, seed, dtype="bf16"):
    """One ngram_sparse_update on a small table; returns host copies and the oracle's."""
    import torch
    rng = np.random.default_rng(seed)
    n = len(rows)
    grad = rng.standard_normal((n, d)).astype(np.float32)
    tab0 = rng.standard_normal((R, d)).astype(np.float32) * 0.02
    if dtype == "bf16":
        tab0 = round_to_bf16(tab0)
    s0 = (np.abs(rng.standard_normal(R)) * 0.1).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    T = torch.from_numpy(tab0).to(tdt).cuda()
    S = torch.from_numpy(s0).cuda()
    ws_bytes = g.ngram_sparse_update_workspace_bytes(n, d)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    upd = torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")
    nupd = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    g.ngram_sparse_update(T, S, R, d, g.DTYPE_BF16 if dtype == "bf16" else g.DTYPE_F32,
                          device_ints(np.asarray(rows, dtype=np.int32)), torch.from_numpy(grad).cuda(), n,
                          0.01, 0.95, 1e-10, upd, nupd, ws, ws_bytes)
    status = g.ngram_sync_status()
    valid = (np.asarray(rows) >= 0) & (np.asarray(rows) < R)
    W1, s1, touched = optim.table_update(tab0.astype(np.float64), s0.astype(np.float64),
                                         np.asarray(rows)[valid], grad[valid].astype(np.float64),
                                         0.01, 0.95, 1e-10)
    k = int(nupd.item())
    return status, T.float().cpu().numpy(), S.cpu().numpy(), upd[:k].cpu().numpy(), tab0, s0, W1, s1, touched


@pytest.mark.parametrize("case", ["one", "33_same", "long_mid_chunk", "aligned_32_runs", "offset_32_runs",
                                  "all_same_4096", "ragged_1001"])
def test_ngram_sparse_update_run_shapes(g, case):
    """Runs of equal rows against the chunk edges of the bucketed update: a run
    inside one chunk, runs exactly one chunk long (aligned and straddling),
    a run over many chunks, every position one row, a ragged tail."""
    rng = np.random.default_rng(5)
    R, d = 512, 768
    if case == "one":
        rows = [17]
    elif case == "33_same":
        rows = [3] * 33
    elif case == "long_mid_chunk":
        rows = list(rng.integers(0, R, 13)) + [R - 1] * 700 + list(rng.integers(0, R, 40))
    elif case == "aligned_32_runs":
        rows = [int(r) for r in rng.permutation(R)[:40] for _ in range(32)]
    elif case == "offset_32_runs":
        rows = [int(r) for r in rng.permutation(R)[:40] for _ in range(32)][16:] + [7] * 5
    elif case == "all_same_4096":
        rows = [R - 1] * 4096
    else:
        rows = list(rng.integers(0, R, 1001))
    st, Wg, Sg, upd, tab0, s0, W1, s1, touched = _run_update(g, rows, d, R, seed=len(rows))
    assert st == g.GPT_OK
    np.testing.assert_array_equal(upd, np.unique(rows))
    assert rel_l2(Wg - tab0, W1 - tab0) < 2e-2
    assert rel_l2(Sg, s1) < 1e-5
    untouched = np.setdiff1d(np.arange(R), touched)
    np.testing.assert_array_equal(Wg[untouched], tab0[untouched])
    np.testing.assert_array_equal(Sg[untouched], s0[untouched])


def test_ngram_sparse_update_invalid_rows_touch_nothing(g):
    """Ids outside [0, R) set the input error and are skipped; the valid
    positions (including ones on the last row, R - 1) are still applied."""
    rng = np.random.default_rng(9)
    R, d = 256, 128
    rows = np.concatenate([rng.integers(0, R, 300), [R - 1] * 40, [-1, R, R + 5, 1 << 30], [R - 1] * 3])
    rows = rng.permutation(rows).astype(np.int64)
    st, Wg, Sg, upd, tab0, s0, W1, s1, touched = _run_update(g, rows, d, R, seed=9, dtype="f32")
    assert st == g.GPT_ERR_INPUT
    np.testing.assert_array_equal(upd, touched)
    assert rel_l2(Wg - tab0, W1 - tab0) < 1e-4
    assert rel_l2(Sg, s1) < 1e-5
    untouched = np.setdiff1d(np.arange(R), touched)
    np.testing.assert_array_equal(Wg[untouched], tab0[untouched])


@pytest.mark.parametrize("b_k", [1, 0])
def test_gemm_epilogue_modes_match_fp64(g, tiles, b_k):
    """Every epilogue of the tensor-core GEMM against its definition on the fp64 product."""
    import torch
    M, N, K = 200, 640, 192
    rng = np.random.default_rng(17 + b_k)
    A = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    B = round_to_bf16(rng.standard_normal((N, K)).astype(np.float32))
    acc = A.astype(np.float64) @ B.astype(np.float64).T
    Ad, Bd = _bf16_dev(A), _bf16_dev(B if b_k else B.T)
    ldb = K if b_k else N
    aux = round_to_bf16(np.maximum(rng.standard_normal((M, N)), 0).astype(np.float32) ** 2)
    auxd = _bf16_dev(aux)
    ws = torch.zeros(M * 5 * 8 + M * 4, dtype=torch.uint8, device="cuda")
    tgt = rng.integers(0, N, M).astype(np.int32)
    tgt[::7] = -1
    tgtd = torch.from_numpy(tgt).cuda()
    tile_max = np.repeat(np.stack([acc[:, 128 * j:128 * (j + 1)].max(axis=1) for j in range(5)], 1), 128, 1)[:, :N]
    cases = {
        g.EPI_STORE: (torch.bfloat16, acc, 4e-3),
        g.EPI_STORE_F32: (torch.float32, acc, 1e-5),
        g.EPI_RELU2: (torch.bfloat16, np.maximum(acc, 0) ** 2, 4e-3),
        g.EPI_DRELU2: (torch.bfloat16, 2 * np.sqrt(aux.astype(np.float64)) * acc, 4e-3),
        g.EPI_LOGITS: (torch.bfloat16, np.exp(acc - tile_max), 4e-3),
    }
    for mode, (dt, ref, tol) in cases.items():
        C = torch.full((M, N), 3.0, dtype=dt, device="cuda")
        g.gptx_gemm_bf16(M, N, K, Ad, K, 1, Bd, ldb, b_k, C, N, 0, 1, ws, ws.numel(), mode=mode,
                         aux=auxd if mode == g.EPI_DRELU2 else (tgtd if mode == g.EPI_LOGITS else None))
        torch.cuda.synchronize()
        assert g.ngram_sync_status() == g.GPT_OK
        assert rel_l2(C.float().cpu().numpy(), ref) < tol, mode
    # logits statistics: per (row, 128-column block) max and sum of exp(z - max)
    st = ws[:M * 5 * 8].view(torch.float32).view(M, 5, 2).cpu().numpy().astype(np.float64)
    for j in range(5):
        z = acc[:, 128 * j:128 * (j + 1)]
        mx = z.max(axis=1)
        np.testing.assert_allclose(st[:, j, 0], mx, rtol=1e-5, atol=1e-4)
        np.testing.assert_allclose(st[:, j, 1], np.exp(z - mx[:, None]).sum(axis=1), rtol=1e-4)
    # the logit at each row's target column (rows without a target are left alone)
    zt = ws[M * 5 * 8:].view(torch.float32).cpu().numpy()
    rows = np.nonzero(tgt >= 0)[0]
    np.testing.assert_allclose(zt[rows], acc[rows, tgt[rows]], rtol=1e-5, atol=1e-4)
    # accumulate with beta = 1 adds into C (TMA reduce-add)
    C = torch.from_numpy(rng.standard_normal((M, N)).astype(np.float32)).cuda()
    C0 = C.cpu().numpy().astype(np.float64)
    g.gptx_gemm_bf16(M, N, K, Ad, K, 1, Bd, ldb, b_k, C, N, 1, 1, None, 0, mode=g.EPI_ACCUM_F32)
    torch.cuda.synchronize()
    assert rel_l2(C.cpu().numpy(), C0 + acc) < 1e-5


def test_gemm_tile_forms_agree_bitwise(g):
    """SM pairs and single-SM tiles add the same products in the same order
    per output element: identical fp32 results, several tiles and a ragged edge."""
    import torch
    M, N, K = 1000, 1280, 704
    rng = np.random.default_rng(23)
    Ad = _bf16_dev(round_to_bf16(rng.standard_normal((M, K)).astype(np.float32)))
    Bd = _bf16_dev(round_to_bf16(rng.standard_normal((K, N)).astype(np.float32)))  # MN-major B
    outs = []
    for on in (1, 0):
        g.gptx_set_gemm_cta_pairs(on)
        C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
        g.gptx_gemm_bf16(M, N, K, Ad, K, 1, Bd, N, 0, C, N, 0, 1, None, 0)
        torch.cuda.synchronize()
        outs.append(C.cpu().numpy())
    g.gptx_set_gemm_cta_pairs(1)
    assert g.ngram_sync_status() == g.GPT_OK
    np.testing.assert_array_equal(outs[0], outs[1])
