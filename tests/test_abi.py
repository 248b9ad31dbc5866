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
