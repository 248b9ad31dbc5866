"""Forward pass and hand-derived backward pass of the decoder (fp64 oracle).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  Everything is float64
NumPy; matrix products use ``@`` as a library primitive and nothing is tiled,
fused or reordered beyond the definitions below.

Model (nanochat discussion #8, user-pasted GPT module, ``GPT.forward`` and
``Block.forward``; modded-nanogpt README "Other general differences"):

    h   = norm(wte[x_t]);  x0 = h + Hx[rx_t]            (x0 table optional)
    per layer:
        u = norm(x)
        q, k, v = split(u @ Wqkv.T);  v += Hv[rv_t]        (value table optional)
                                      v += vproj S3[r3_t]  (frozen trigram statistics, optional;
                                                            oracle/trigram.py)
        q, k = norm_head(rope(q)), norm_head(rope(k))      (QK-norm after RoPE)
        o = softmax(q k^T / sqrt(hd) + causal) v
        x = x + o @ Wo.T
        u2 = norm(x)
        x = x + relu(u2 @ W1.T)^2 @ W2.T                  (ReLU^2 MLP)
    z = norm(x) @ W_lm.T  [softcap c*tanh(z/c) when c > 0]
    loss = mean over targets != -1 of logsumexp(z_t) - z_t[y_t]

The pasted module squares a GELU in its MLP; the modded-nanogpt README and
the decoder-rtx posts both name ReLU^2, which is what is computed here.
"""

import numpy as np


# --------------------------------------------------------------------------- norms
def rmsnorm(x, eps):
    """Parameter-free RMSNorm over the last axis (``norm`` in the pasted module,
    ``F.rms_norm(x, (x.size(-1),))``): y = x / sqrt(mean(x^2) + eps).

    Returns (y, rstd) with rstd = 1/sqrt(mean(x^2)+eps) of shape x.shape[:-1].
    """
    ms = np.mean(x * x, axis=-1)
    rstd = 1.0 / np.sqrt(ms + eps)
    return x * rstd[..., None], rstd


def rmsnorm_bwd(dy, y, rstd):
    """Gradient of y = x*rstd(x): dx = rstd * (dy - y * mean(dy*y))."""
    c = np.mean(dy * y, axis=-1, keepdims=True)
    return rstd[..., None] * (dy - y * c)


# --------------------------------------------------------------------------- RoPE
def rope_tables(T, hd, base):
    """cos, sin [T, hd/2] with theta[t, i] = t * base^(-2i/hd)
    (``_precompute_rotary_embeddings``: inv_freq = 1/base^(arange(0,hd,2)/hd))."""
    i = np.arange(0, hd, 2, dtype=np.float64)
    inv_freq = 1.0 / (base ** (i / hd))
    theta = np.outer(np.arange(T, dtype=np.float64), inv_freq)
    return np.cos(theta), np.sin(theta)


def rope(x, cos, sin):
    """Half-split rotation (``apply_rotary_emb``) on x [..., T, hd]:
    y1 = x1*cos + x2*sin, y2 = -x1*sin + x2*cos, x1/x2 = first/second half."""
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * cos + x2 * sin, -x1 * sin + x2 * cos], axis=-1)


def rope_bwd(dy, cos, sin):
    """Transpose of the rotation: rotation by -theta."""
    h = dy.shape[-1] // 2
    d1, d2 = dy[..., :h], dy[..., h:]
    return np.concatenate([d1 * cos - d2 * sin, d1 * sin + d2 * cos], axis=-1)


# --------------------------------------------------------------------------- attention
def causal_attention(q, k, v):
    """Causal softmax attention (``F.scaled_dot_product_attention(is_causal=True)``
    in ``CausalSelfAttention.forward``), default scale 1/sqrt(hd).

    q, k, v: [B, H, T, hd].  Returns (o, P) with P the [B, H, T, T] probabilities.
    """
    hd = q.shape[-1]
    T = q.shape[-2]
    s = (q @ np.swapaxes(k, -1, -2)) / np.sqrt(hd)
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)
    s = np.where(mask, -np.inf, s)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ v, p


def causal_attention_bwd(do, q, k, v, p):
    """Gradients of o = P v, P = softmax(q k^T/sqrt(hd) + causal)."""
    hd = q.shape[-1]
    scale = 1.0 / np.sqrt(hd)
    dv = np.swapaxes(p, -1, -2) @ do
    dp = do @ np.swapaxes(v, -1, -2)
    ds = p * (dp - np.sum(dp * p, axis=-1, keepdims=True))
    dq = (ds @ k) * scale
    dk = (np.swapaxes(ds, -1, -2) @ q) * scale
    return dq, dk, dv


# --------------------------------------------------------------------------- model
def _heads(x, B, T, H, hd):
    return x.reshape(B, T, H, hd).transpose(0, 2, 1, 3)


def _unheads(x):
    B, H, T, hd = x.shape
    return x.transpose(0, 2, 1, 3).reshape(B * T, H * hd)


def forward(cfg, P, tokens, targets, rows_x=None, rows_v=None, rows_3=None):
    """Forward pass; returns (loss, per_token_loss, cache).

    P: dict of float64 parameters in the ``synthetic.param_shapes`` layout
    (plus the frozen trigram statistics "h3" when "vproj" is present).
    tokens/targets: int [B, T]; targets == -1 are ignored.  rows_x/rows_v are
    the bigram table rows [B, T] when the tables are present, rows_3 the
    trigram table rows.
    """
    B, T = tokens.shape
    d, H, hd, V = cfg["d_model"], cfg["n_head"], cfg["head_dim"], cfg["vocab"]
    eps = cfg["norm_eps"]
    N = B * T
    tok = tokens.reshape(N)
    c = {"B": B, "T": T}

    emb = P["wte"][tok]
    h, c["emb_rstd"] = rmsnorm(emb, eps)
    c["h"] = h
    x = h.copy()
    if "hx" in P:
        x = x + P["hx"][rows_x.reshape(N)]
    cos, sin = rope_tables(T, hd, cfg["rope_base"])
    c["cos"], c["sin"] = cos, sin
    vbias3 = None
    if "vproj" in P:
        c["s3g"] = P["h3"][rows_3.reshape(N)]      # [N, width] statistics of each position
        vbias3 = c["s3g"] @ P["vproj"].T           # [N, a], the same in every layer

    layers = []
    for layer in range(cfg["n_layer"]):
        L = {}
        u, L["rstd1"] = rmsnorm(x, eps)
        L["u"] = u
        qkv = u @ P[f"h{layer}.wqkv"].T
        a = H * hd
        q, k, v = qkv[:, :a], qkv[:, a:2 * a], qkv[:, 2 * a:]
        if "hv" in P:
            v = v + P["hv"][rows_v.reshape(N)]
        if vbias3 is not None:
            v = v + vbias3
        qh, kh, vh = _heads(q, B, T, H, hd), _heads(k, B, T, H, hd), _heads(v, B, T, H, hd)
        qr, kr = rope(qh, cos, sin), rope(kh, cos, sin)
        if cfg["qk_norm"]:
            qn, L["rstd_q"] = rmsnorm(qr, eps)
            kn, L["rstd_k"] = rmsnorm(kr, eps)
        else:
            qn, kn = qr, kr
        o, p = causal_attention(qn, kn, vh)
        L.update(qn=qn, kn=kn, vh=vh, p=p)
        o2 = _unheads(o)
        L["o"] = o2
        x = x + o2 @ P[f"h{layer}.wo"].T
        u2, L["rstd2"] = rmsnorm(x, eps)
        L["u2"] = u2
        a1 = u2 @ P[f"h{layer}.w1"].T
        r = np.maximum(a1, 0.0)
        g = r * r
        L["r"], L["g"] = r, g
        x = x + g @ P[f"h{layer}.w2"].T
        layers.append(L)
    c["layers"] = layers

    xf, c["rstd_f"] = rmsnorm(x, eps)
    c["xf"] = xf
    w_lm = P["wte"] if cfg["tie_embeddings"] else P["lm_head"]
    z = xf @ w_lm.T
    cap = cfg["softcap"]
    if cap > 0:
        z = cap * np.tanh(z / cap)
    c["z"] = z
    y = targets.reshape(N)
    valid = y >= 0
    zmax = z.max(axis=-1, keepdims=True)
    lse = (zmax + np.log(np.sum(np.exp(z - zmax), axis=-1, keepdims=True)))[:, 0]
    per_tok = np.zeros(N)
    per_tok[valid] = lse[valid] - z[np.arange(N)[valid], y[valid]]
    n_valid = int(valid.sum())
    loss = float(per_tok.sum() / n_valid) if n_valid > 0 else 0.0
    c.update(lse=lse, y=y, valid=valid, n_valid=n_valid, tok=tok)
    return loss, per_tok.reshape(B, T), c


def backward(cfg, P, c, scale=1.0):
    """Exact gradient of ``scale * loss`` w.r.t. every dense parameter.

    Returns (grads, gx0, gv): grads in the ``param_shapes`` layout (tables
    excluded), gx0 [N, d] = d/dx0 per position, gv [N, a] = sum over layers of
    d/dv per position (the gradients that reach the two bigram tables).
    Written out by hand, as in the decoder-rtx hand-written backward.
    """
    B, T = c["B"], c["T"]
    d, H, hd, V = cfg["d_model"], cfg["n_head"], cfg["head_dim"], cfg["vocab"]
    N = B * T
    a = H * hd
    G = {}
    # ---- loss head
    z, lse, y, valid = c["z"], c["lse"], c["y"], c["valid"]
    dz = np.zeros_like(z)
    if c["n_valid"] > 0:
        sm = np.exp(z - lse[:, None])
        dz[valid] = sm[valid]
        dz[np.arange(N)[valid], y[valid]] -= 1.0
        dz *= scale / c["n_valid"]
    cap = cfg["softcap"]
    if cap > 0:
        dz = dz * (1.0 - (z / cap) ** 2)
    w_lm = P["wte"] if cfg["tie_embeddings"] else P["lm_head"]
    dxf = dz @ w_lm
    dw_lm = dz.T @ c["xf"]
    dx = rmsnorm_bwd(dxf, c["xf"], c["rstd_f"])
    gv = np.zeros((N, a))
    cos, sin = c["cos"], c["sin"]
    for layer in reversed(range(cfg["n_layer"])):
        L = c["layers"][layer]
        # ---- MLP: x += relu(u2 W1^T)^2 W2^T
        W1, W2 = P[f"h{layer}.w1"], P[f"h{layer}.w2"]
        G[f"h{layer}.w2"] = dx.T @ L["g"]
        dg = dx @ W2
        da1 = 2.0 * L["r"] * dg
        G[f"h{layer}.w1"] = da1.T @ L["u2"]
        du2 = da1 @ W1
        dx = dx + rmsnorm_bwd(du2, L["u2"], L["rstd2"])
        # ---- attention: x += o Wo^T
        Wo = P[f"h{layer}.wo"]
        G[f"h{layer}.wo"] = dx.T @ L["o"]
        do = _heads(dx @ Wo, B, T, H, hd)
        dqn, dkn, dvh = causal_attention_bwd(do, L["qn"], L["kn"], L["vh"], L["p"])
        if cfg["qk_norm"]:
            dqr = rmsnorm_bwd(dqn, L["qn"], L["rstd_q"])
            dkr = rmsnorm_bwd(dkn, L["kn"], L["rstd_k"])
        else:
            dqr, dkr = dqn, dkn
        dq = _unheads(rope_bwd(dqr, cos, sin))
        dk = _unheads(rope_bwd(dkr, cos, sin))
        dv = _unheads(dvh)
        gv += dv
        dqkv = np.concatenate([dq, dk, dv], axis=1)
        G[f"h{layer}.wqkv"] = dqkv.T @ L["u"]
        du = dqkv @ P[f"h{layer}.wqkv"]
        dx = dx + rmsnorm_bwd(du, L["u"], L["rstd1"])
    gx0 = dx
    if "vproj" in P:
        G["vproj"] = gv.T @ c["s3g"]
    # ---- embedding: h = norm(wte[tok])
    dh = rmsnorm_bwd(gx0, c["h"], c["emb_rstd"])
    dwte = np.zeros_like(P["wte"])
    np.add.at(dwte, c["tok"], dh)
    if cfg["tie_embeddings"]:
        dwte += dw_lm
    else:
        G["lm_head"] = dw_lm
    G["wte"] = dwte
    return G, gx0, gv
