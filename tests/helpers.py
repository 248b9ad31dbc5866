"""Shared test helpers: workload dict -> C config, parameter import/export,
relative-L2 comparison."""

import numpy as np


def to_cfg(w):
    import gpt_pretraining_step_decoder_b200 as g
    keys = [f[0] for f in g.GptConfig._fields_]
    return g.make_config(**{k: v for k, v in w.items() if k in keys})


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def import_params(model, params):
    """Write seeded host parameters into the model arena, refresh bf16 copies."""
    import torch
    import gpt_pretraining_step_decoder_b200 as g
    for name, val in params.items():
        t = model.tensor(name, g.KIND_PARAM)
        t.copy_(torch.from_numpy(np.asarray(val, dtype=np.float32)).to(t.dtype))
    g.gpt_params_changed(model.h)


def export(model, name, kind=0):
    return model.tensor(name, kind).float().cpu().numpy().astype(np.float64)


def device_ints(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
