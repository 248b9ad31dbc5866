"""The C-ABI library loads and exports every symbol include/gpt.h declares;
host-only entry points validate configurations (no GPU needed)."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gpt.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    import gpt_pretraining_step_decoder_b200 as g
    lib = ctypes.CDLL(g.LIB_PATH)
    names = declared_functions()
    assert "gpt_create" in names and "ngram_sparse_update" in names
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", g.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for n in names:
        assert n in exported, n


def test_host_entry_points_match_oracle_counts():
    import gpt_pretraining_step_decoder_b200 as g
    from oracle import counts
    from synthetic import WORKLOADS
    from tests.helpers import to_cfg
    for name, w in WORKLOADS.items():
        cfg = to_cfg(w)
        f, fc = g.gpt_flops_per_token(cfg)
        assert f == counts.flops_per_token(w), name
        assert fc == counts.flops_per_token(w, causal=True), name
        assert g.gpt_workspace_bytes(cfg) > 0


@pytest.mark.parametrize("bad", [
    dict(d_model=130),                       # != n_head * head_dim
    dict(n_kv_head=2),                       # grouped KV heads unsupported
    dict(dtype="bf16"),                      # bf16 needs head_dim 128
    dict(n_layer=0),
    dict(head_dim=33, d_model=132),
])
def test_config_validation(bad):
    import gpt_pretraining_step_decoder_b200 as g
    cfg = g.make_config(**bad)
    with pytest.raises(g.GptError) as e:
        g.gpt_workspace_bytes(cfg)
    assert e.value.code == g.GPT_ERR_CONFIG
    assert g.gpt_last_error()


def test_argument_errors_without_gpu():
    import gpt_pretraining_step_decoder_b200 as g
    with pytest.raises(g.GptError) as e:
        g.gpt_create(g.make_config(), 0, None, 0)
    assert e.value.code == g.GPT_ERR_ARG
    assert g._lib.gpt_backward_step(None, 1.0) == g.GPT_ERR_ARG
    with pytest.raises(g.GptError):
        g.ngram_sparse_update_workspace_bytes(-1, 768)


def test_muon_and_table_exchange_argument_errors_without_gpu():
    """The new entry points validate their arguments before any device work:
    these calls return their error codes on a machine without a GPU."""
    import gpt_pretraining_step_decoder_b200 as g
    lib = g._lib
    assert lib.gpt_set_table_exchange(None, 1) == g.GPT_ERR_ARG
    for bad in ((100, 128), (128, 0), (8, 12)):
        with pytest.raises(g.GptError) as e:
            g.muon_update_workspace_bytes(*bad)
        assert e.value.code == g.GPT_ERR_ARG
    assert g.muon_update_workspace_bytes(768, 2304) > 0
    W, M, G = 1 << 20, 2 << 20, 3 << 20  # aligned stand-in addresses, never dereferenced
    args = dict(rows=64, cols=128, out_rows=1, lr=0.02, momentum=0.95, nesterov=1, ns_steps=5)

    def call(**kw):
        a = dict(args, **kw)
        return lib.muon_update(kw.get("W", W), M, G, a["rows"], a["cols"], a["out_rows"], a["lr"], a["momentum"],
                               a["nesterov"], a["ns_steps"], kw.get("ws", 4 << 20), kw.get("ws_bytes", 16), None)

    assert lib.muon_update(None, M, G, 64, 128, 1, 0.02, 0.95, 1, 5, None, 0, None) == g.GPT_ERR_ARG
    assert call(rows=60) == g.GPT_ERR_ARG            # not a multiple of 8
    assert call(momentum=1.0) == g.GPT_ERR_ARG       # momentum must be < 1
    assert call(ns_steps=65) == g.GPT_ERR_ARG
    assert call(W=W + 4) == g.GPT_ERR_ARG            # not 16-byte aligned
    assert call() == g.GPT_ERR_WORKSPACE             # 16 bytes of workspace
    assert "workspace" in g.gpt_last_error()
