"""The allocation-free table update (built-in scratch) against the workspace one.

Some callers cannot hand the library any scratch memory (a runtime that owns
all device memory through its own pool, a plugin given tensors but no
allocator); for them ngram_sparse_update_noalloc uses a buffer compiled into
the library.  Both calls run the same kernels in the same order, and the
update is bit-reproducible, so the two results must be identical bit for bit.
Two calls in a row check that whatever the first call left in that shared
buffer does not leak into the second; the result of both calls is also
compared with the oracle's two updates.  This file is collected last on
purpose, so a failure here comes after every other test has run.
"""

import numpy as np
import pytest

from oracle import hashing, optim
from synthetic import round_to_bf16, zipf_stream
from tests.helpers import device_ints, rel_l2

pytestmark = pytest.mark.gpu


def test_noalloc_update_matches_workspace_update_on_two_calls():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    assert torch.cuda.is_available()
    R, d, n = 4096, 768, 6000
    rng = np.random.default_rng(99)
    tab0 = round_to_bf16(rng.standard_normal((R, d)).astype(np.float32) * 0.02)
    T_ws = torch.from_numpy(tab0).to(torch.bfloat16).cuda()
    T_na = T_ws.clone()
    S_ws = torch.zeros(R, dtype=torch.float32, device="cuda")
    S_na = S_ws.clone()
    ws_bytes = g.ngram_sparse_update_workspace_bytes(n, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    W_ref, S_ref = tab0.astype(np.float64), np.zeros(R)
    for call in range(2):
        tok = zipf_stream(n + 1, 50304, 1234 + call).reshape(1, n + 1)[:, :n]
        rows_h = hashing.bigram_rows(tok, 50304, 2654435761, 2246822519, R).reshape(-1)
        rows = device_ints(rows_h)
        grad_h = rng.standard_normal((n, d)).astype(np.float32)
        grad = torch.from_numpy(grad_h).cuda()
        u_ws = torch.full((n,), -1, dtype=torch.int32, device="cuda")
        u_na = torch.full((n,), -2, dtype=torch.int32, device="cuda")
        k_ws = torch.zeros(1, dtype=torch.int32, device="cuda")
        k_na = torch.zeros(1, dtype=torch.int32, device="cuda")
        g.ngram_sparse_update(T_ws, S_ws, R, d, g.DTYPE_BF16, rows, grad, n, 0.01, 0.95, 1e-10,
                              u_ws, k_ws, ws, ws_bytes)
        g.ngram_sparse_update_noalloc(T_na, S_na, R, d, g.DTYPE_BF16, rows, grad, n, 0.01, 0.95, 1e-10,
                                      u_na, k_na)
        assert g.ngram_sync_status() == g.GPT_OK
        k = int(k_ws.item())
        assert int(k_na.item()) == k
        np.testing.assert_array_equal(u_na[:k].cpu().numpy(), u_ws[:k].cpu().numpy())
        np.testing.assert_array_equal(T_na.view(torch.int16).cpu().numpy(), T_ws.view(torch.int16).cpu().numpy())
        np.testing.assert_array_equal(S_na.cpu().numpy(), S_ws.cpu().numpy())
        # and both against the oracle's update (fp64; the GPU rounds rows to bf16)
        W_ref, S_ref, uniq = optim.table_update(W_ref, S_ref, rows_h, grad_h.astype(np.float64), 0.01, 0.95, 1e-10)
        np.testing.assert_array_equal(u_na[:k].cpu().numpy(), uniq)
        assert rel_l2(T_na.float().cpu().numpy() - tab0, W_ref - tab0) < 2e-2
        assert rel_l2(S_na.cpu().numpy(), S_ref) < 2e-2


def test_noalloc_update_rejects_sizes_beyond_its_buffer():
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    n, d = 196608, 768     # needs about 75 MiB of scratch (16 n + 2 ceil(n / 16) d 4 bytes)
    tab = torch.zeros((16, d), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(g.GptError) as e:
        g.ngram_sparse_update_noalloc(tab, st, 16, d, g.DTYPE_BF16, None, None, n, 0.01, 0.95, 1e-10,
                                      None, None)
    assert e.value.code == g.GPT_ERR_WORKSPACE
    assert "scratch" in str(e.value)
