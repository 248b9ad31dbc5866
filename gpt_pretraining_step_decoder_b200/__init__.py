"""Python binding of libgpt_b200.so (ctypes; argument marshalling only).

Every function below forwards to the C entry point of the same name declared
in include/gpt.h; every step of the training path runs in the library's CUDA
kernels.  PyTorch is used only to own device memory (the model arena) and to
name CUDA streams.  Importing this package raises if the compiled library is
missing: there is no fallback path.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgpt_b200.so")

GPT_OK, GPT_ERR_ARG, GPT_ERR_CONFIG, GPT_ERR_WORKSPACE, GPT_ERR_STATE = 0, 1, 2, 3, 4
GPT_ERR_INPUT, GPT_ERR_NONFINITE, GPT_ERR_CUDA, GPT_ERR_TIMEOUT = 5, 6, 7, 8
DTYPE_F32, DTYPE_BF16, DTYPE_I32 = 0, 1, 2
KIND_PARAM, KIND_GRAD, KIND_ADAM_M, KIND_ADAM_V, KIND_ROW_STATE, KIND_PARAM_LP, KIND_ACT = range(7)
MATRIX_ADAMW, MATRIX_MUON = 0, 1

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python gpt_pretraining_step_decoder_b200/build.py` "
        "(there is no CPU fallback)")
_lib = ctypes.CDLL(LIB_PATH)


class GptConfig(ctypes.Structure):
    _fields_ = [
        ("n_layer", ctypes.c_int), ("d_model", ctypes.c_int), ("n_head", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("n_kv_head", ctypes.c_int), ("d_ff", ctypes.c_int),
        ("vocab", ctypes.c_int), ("seq_len", ctypes.c_int), ("micro_batch", ctypes.c_int),
        ("grad_accum", ctypes.c_int), ("dtype", ctypes.c_int), ("tie_embeddings", ctypes.c_int),
        ("qk_norm", ctypes.c_int), ("rope_base", ctypes.c_float), ("norm_eps", ctypes.c_float),
        ("softcap", ctypes.c_float), ("init_std", ctypes.c_float), ("adam_b1", ctypes.c_float),
        ("adam_b2", ctypes.c_float), ("adam_eps", ctypes.c_float), ("weight_decay", ctypes.c_float),
        ("grad_clip", ctypes.c_float), ("lr_mult_embed", ctypes.c_float),
        ("lr_mult_head", ctypes.c_float), ("lr_mult_matrix", ctypes.c_float),
        ("lr_mult_table", ctypes.c_float), ("x0_rows", ctypes.c_longlong),
        ("v_rows", ctypes.c_longlong), ("table_beta", ctypes.c_float),
        ("table_eps", ctypes.c_float), ("hash_p1", ctypes.c_ulonglong),
        ("hash_p2", ctypes.c_ulonglong), ("lm_chunk_rows", ctypes.c_int),
        ("matrix_optimizer", ctypes.c_int), ("muon_momentum", ctypes.c_float),
        ("muon_ns_steps", ctypes.c_int), ("muon_nesterov", ctypes.c_int),
        ("tri_rows", ctypes.c_longlong), ("tri_width", ctypes.c_int), ("hash_p3", ctypes.c_ulonglong),
    ]


class GptProfEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("scopes", ctypes.c_longlong),
                ("launches", ctypes.c_longlong), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


_P, _I, _LL, _SZ, _F, _ULL = (ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t,
                              ctypes.c_float, ctypes.c_ulonglong)
_SIGS = {
    "gpt_default_config": [ctypes.POINTER(GptConfig)],
    "gpt_workspace_bytes": [ctypes.POINTER(GptConfig), ctypes.POINTER(_SZ)],
    "gpt_create": [ctypes.POINTER(GptConfig), _ULL, _P, _SZ, _P, ctypes.POINTER(_P)],
    "gpt_destroy": [_P],
    "gpt_set_stream": [_P, _P],
    "gpt_forward_loss": [_P, _P, _P, _P],
    "gpt_backward_step": [_P, _F],
    "gpt_backward": [_P, _F],
    "gpt_optimizer_step": [_P, _F],
    "gpt_set_table_exchange": [_P, _I],
    "gpt_grad_sumsq": [_P, _LL, _LL, _P],
    "gpt_optimizer_step_range": [_P, _F, _LL, _LL, _P],
    "gpt_launch_count": [ctypes.POINTER(_LL)],
    "gpt_profile_enable": [_P, _I],
    "gpt_profile_read": [_P, ctypes.POINTER(GptProfEntry), _I, ctypes.POINTER(_I)],
    "gpt_num_params": [_P, ctypes.POINTER(_LL), ctypes.POINTER(_LL)],
    "gpt_flops_per_token": [ctypes.POINTER(GptConfig), ctypes.POINTER(_LL), ctypes.POINTER(_LL)],
    "gpt_tensor": [_P, ctypes.c_char_p, _I, ctypes.POINTER(_P), ctypes.POINTER(_I), _LL * 4],
    "gpt_params_changed": [_P],
    "gpt_sync_status": [_P],
    "ngram_hash": [_P, _I, _I, _I, _ULL, _ULL, _LL, _P, _P],
    "ngram_gather": [_P, _I, _P, _LL, _I, _I, _P, _I, _P],
    "ngram_sparse_update_workspace_bytes": [_I, _I, ctypes.POINTER(_SZ)],
    "ngram_sparse_update": [_P, _P, _LL, _I, _I, _P, _P, _I, _F, _F, _F, _P, _P, _P, _SZ, _P],
    "ngram_sync_status": [_P],
    "ngram_sparse_update_noalloc": [_P, _P, _LL, _I, _I, _P, _P, _I, _F, _F, _F, _P, _P, _P],
    "gptx_gemm_bf16": [_I, _I, _I, _P, _LL, _I, _P, _LL, _I, _I, _P, _LL, _P, _I, _I, _P, _SZ, _P],
    "gptx_set_gemm_cta_pairs": [_I],
    "gptx_wait_probe": [_I, _P],
    "fp8_quantize_workspace_bytes": [ctypes.POINTER(_SZ)],
    "fp8_quantize": [_P, _I, _LL, _P, _P, _P, _SZ, _P],
    "gptx_gemm_fp8": [_I, _I, _I, _P, _LL, _P, _LL, _P, _P, _I, _P, _LL, _P],
    "trigram_tally_workspace_bytes": [_LL, _I, ctypes.POINTER(_SZ)],
    "trigram_tally": [_P, _I, _I, _I, _ULL, _ULL, _ULL, _LL, _I, _I, _P, _P, _SZ, _P],
    "muon_update_workspace_bytes": [_I, _I, ctypes.POINTER(_SZ)],
    "muon_update": [_P, _P, _P, _I, _I, _I, _F, _F, _I, _I, _P, _SZ, _P],
}
for _name, _args in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int
_lib.gpt_last_error.argtypes = []
_lib.gpt_last_error.restype = ctypes.c_char_p


class GptError(RuntimeError):
    def __init__(self, code, fn):
        self.code = code
        msg = _lib.gpt_last_error().decode(errors="replace")
        super().__init__(f"{fn} returned {code}: {msg}")


def _check(code, fn):
    if code != GPT_OK:
        raise GptError(code, fn)
    return code


def _ptr(x):
    """Device/host address of a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ------------------------------------------------------------------ raw entry points
def gpt_last_error():
    return _lib.gpt_last_error().decode(errors="replace")


def make_config(**fields):
    """GptConfig from gpt_default_config() plus keyword overrides (dtype may be 'f32'/'bf16')."""
    c = GptConfig()
    _check(_lib.gpt_default_config(ctypes.byref(c)), "gpt_default_config")
    for k, v in fields.items():
        if k == "dtype" and isinstance(v, str):
            v = DTYPE_BF16 if v == "bf16" else DTYPE_F32
        if k == "matrix_optimizer" and isinstance(v, str):
            v = {"adamw": MATRIX_ADAMW, "muon": MATRIX_MUON}[v]
        if any(k == f[0] for f in GptConfig._fields_):
            setattr(c, k, v)
    if c.n_kv_head == 0 or "n_kv_head" not in fields:
        c.n_kv_head = c.n_head
    return c


def gpt_workspace_bytes(cfg):
    n = ctypes.c_size_t()
    _check(_lib.gpt_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "gpt_workspace_bytes")
    return n.value


def gpt_flops_per_token(cfg):
    f, fc = ctypes.c_longlong(), ctypes.c_longlong()
    _check(_lib.gpt_flops_per_token(ctypes.byref(cfg), ctypes.byref(f), ctypes.byref(fc)),
           "gpt_flops_per_token")
    return f.value, fc.value


def gpt_create(cfg, seed, arena, arena_bytes, stream=None):
    h = ctypes.c_void_p()
    _check(_lib.gpt_create(ctypes.byref(cfg), seed, _ptr(arena), arena_bytes, _stream(stream),
                           ctypes.byref(h)), "gpt_create")
    return h.value


def gpt_destroy(h):
    return _check(_lib.gpt_destroy(h), "gpt_destroy")


def gpt_set_stream(h, stream):
    return _check(_lib.gpt_set_stream(h, _stream(stream)), "gpt_set_stream")


def gpt_forward_loss(h, tokens, targets, loss):
    return _check(_lib.gpt_forward_loss(h, _ptr(tokens), _ptr(targets), _ptr(loss)), "gpt_forward_loss")


def gpt_backward_step(h, lr):
    return _check(_lib.gpt_backward_step(h, float(lr)), "gpt_backward_step")


def gpt_backward(h, lr):
    return _check(_lib.gpt_backward(h, float(lr)), "gpt_backward")


def gpt_optimizer_step(h, lr):
    return _check(_lib.gpt_optimizer_step(h, float(lr)), "gpt_optimizer_step")


def gpt_launch_count():
    n = ctypes.c_longlong()
    _check(_lib.gpt_launch_count(ctypes.byref(n)), "gpt_launch_count")
    return n.value


def gpt_profile_enable(h, on):
    return _check(_lib.gpt_profile_enable(h, int(on)), "gpt_profile_enable")


def gpt_profile_read(h, cap=64):
    """{class name: dict(scopes, launches, ms, flops, bytes)} since the last read."""
    arr = (GptProfEntry * cap)()
    n = ctypes.c_int()
    _check(_lib.gpt_profile_read(h, arr, cap, ctypes.byref(n)), "gpt_profile_read")
    return {arr[i].name.decode(): dict(scopes=arr[i].scopes, launches=arr[i].launches,
                                       ms=arr[i].ms, flops=arr[i].flops, bytes=arr[i].bytes)
            for i in range(min(n.value, cap))}


def gpt_num_params(h):
    d, t = ctypes.c_longlong(), ctypes.c_longlong()
    _check(_lib.gpt_num_params(h, ctypes.byref(d), ctypes.byref(t)), "gpt_num_params")
    return d.value, t.value


def gpt_tensor(h, name, kind):
    p, dt, shape = ctypes.c_void_p(), ctypes.c_int(), (ctypes.c_longlong * 4)()
    _check(_lib.gpt_tensor(h, name.encode(), kind, ctypes.byref(p), ctypes.byref(dt), shape),
           "gpt_tensor")
    return p.value, dt.value, tuple(shape)


def gpt_params_changed(h):
    return _check(_lib.gpt_params_changed(h), "gpt_params_changed")


def gpt_sync_status(h):
    """Returns the status code (does not raise): GPT_OK or a device-reported error."""
    return _lib.gpt_sync_status(h)


def ngram_hash(tokens, B, T, vocab, p1, p2, rows, rows_out, stream=None):
    return _check(_lib.ngram_hash(_ptr(tokens), B, T, vocab, p1, p2, rows, _ptr(rows_out),
                                  _stream(stream)), "ngram_hash")


def ngram_gather(rows, n, table, n_rows, d, dtype, out, accumulate, stream=None):
    return _check(_lib.ngram_gather(_ptr(rows), n, _ptr(table), n_rows, d, dtype, _ptr(out),
                                    accumulate, _stream(stream)), "ngram_gather")


def ngram_sparse_update_workspace_bytes(n, d):
    b = ctypes.c_size_t()
    _check(_lib.ngram_sparse_update_workspace_bytes(n, d, ctypes.byref(b)),
           "ngram_sparse_update_workspace_bytes")
    return b.value


def ngram_sparse_update(table, row_state, n_rows, d, dtype, rows, grad, n, lr, beta, eps,
                        updated_rows_out, n_updated_out, workspace, ws_bytes, stream=None):
    return _check(_lib.ngram_sparse_update(
        _ptr(table), _ptr(row_state), n_rows, d, dtype, _ptr(rows), _ptr(grad), n, lr, beta, eps,
        _ptr(updated_rows_out), _ptr(n_updated_out), _ptr(workspace), ws_bytes, _stream(stream)),
        "ngram_sparse_update")


def ngram_sparse_update_noalloc(table, row_state, n_rows, d, dtype, rows, grad, n, lr, beta, eps,
                                updated_rows_out, n_updated_out, stream=None):
    """ngram_sparse_update with the library's built-in scratch (no device allocation)."""
    return _check(_lib.ngram_sparse_update_noalloc(
        _ptr(table), _ptr(row_state), n_rows, d, dtype, _ptr(rows), _ptr(grad), n, lr, beta, eps,
        _ptr(updated_rows_out), _ptr(n_updated_out), _stream(stream)), "ngram_sparse_update_noalloc")


def ngram_sync_status(stream=None):
    return _lib.ngram_sync_status(_stream(stream))


def muon_update_workspace_bytes(rows, cols):
    b = ctypes.c_size_t(0)
    _check(_lib.muon_update_workspace_bytes(rows, cols, ctypes.byref(b)), "muon_update_workspace_bytes")
    return b.value


def muon_update(W, M, G, rows, cols, out_rows, lr, momentum, nesterov, ns_steps, workspace, ws_bytes,
                stream=None):
    return _check(_lib.muon_update(_ptr(W), _ptr(M), _ptr(G), rows, cols, int(out_rows), float(lr),
                                   float(momentum), int(nesterov), ns_steps, _ptr(workspace), ws_bytes,
                                   _stream(stream)), "muon_update")


EPI_STORE, EPI_STORE_F32, EPI_ACCUM_F32, EPI_RELU2, EPI_DRELU2, EPI_LOGITS = range(6)


def gptx_gemm_bf16(M, N, K, A, lda, a_kmajor, B, ldb, b_kmajor, C, ldc, beta=0, splits=1,
                   workspace=None, ws_bytes=0, stream=None, mode=EPI_ACCUM_F32, aux=None):
    return _check(_lib.gptx_gemm_bf16(M, N, K, _ptr(A), lda, a_kmajor, _ptr(B), ldb, b_kmajor, mode,
                                      _ptr(C), ldc, _ptr(aux), beta, splits, _ptr(workspace), ws_bytes,
                                      _stream(stream)), "gptx_gemm_bf16")


def trigram_tally_workspace_bytes(rows, width):
    n = ctypes.c_size_t()
    _check(_lib.trigram_tally_workspace_bytes(rows, width, ctypes.byref(n)), "trigram_tally_workspace_bytes")
    return n.value


def trigram_tally(streams, S, L, vocab, p1, p2, p3, rows, width, dtype, table, workspace, ws_bytes, stream=None):
    """Fill the frozen trigram statistics table from token streams [S, L] (device int32)."""
    return _check(_lib.trigram_tally(_ptr(streams), S, L, vocab, p1, p2, p3, rows, width, dtype, _ptr(table),
                                     _ptr(workspace), ws_bytes, _stream(stream)), "trigram_tally")


def fp8_quantize_workspace_bytes():
    n = ctypes.c_size_t()
    _check(_lib.fp8_quantize_workspace_bytes(ctypes.byref(n)), "fp8_quantize_workspace_bytes")
    return n.value


def fp8_quantize(x, dtype, n, q, scale, workspace, ws_bytes, stream=None):
    """Per-tensor e4m3 codes of x into q (uint8) and its scale (device float)."""
    return _check(_lib.fp8_quantize(_ptr(x), dtype, n, _ptr(q), _ptr(scale), _ptr(workspace), ws_bytes,
                                    _stream(stream)), "fp8_quantize")


def gptx_gemm_fp8(M, N, K, A, lda, B, ldb, scale_a, scale_b, out_dtype, C, ldc, stream=None):
    return _check(_lib.gptx_gemm_fp8(M, N, K, _ptr(A), lda, _ptr(B), ldb, _ptr(scale_a), _ptr(scale_b), out_dtype,
                                     _ptr(C), ldc, _stream(stream)), "gptx_gemm_fp8")


def gptx_set_gemm_cta_pairs(on):
    """Run later GEMMs with N >= 256 on SM pairs (True, the default) or one SM per tile."""
    return _check(_lib.gptx_set_gemm_cta_pairs(int(bool(on))), "gptx_set_gemm_cta_pairs")


def gptx_wait_probe(limit_us, stream=None):
    """Enqueue one bounded wait that nothing satisfies; it gives up after
    limit_us and the next ngram_sync_status(stream) reports GPT_ERR_TIMEOUT."""
    return _check(_lib.gptx_wait_probe(int(limit_us), _stream(stream)), "gptx_wait_probe")


# ------------------------------------------------------------------ convenience
class Model:
    """A model whose arena is a torch uint8 CUDA tensor (memory ownership only)."""

    def __init__(self, cfg, seed=0, device="cuda", stream=None):
        import torch
        self.torch = torch
        self.cfg = cfg
        self.bytes = gpt_workspace_bytes(cfg)
        self.arena = torch.empty(self.bytes + 256, dtype=torch.uint8, device=device)
        base = self.arena.data_ptr()
        self.base = (base + 255) & ~255
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.h = gpt_create(cfg, seed, self.base, self.bytes, self.stream)
        self.loss = torch.zeros(1, dtype=torch.float32, device=device)
        self.table_exchange = False

    def tensor(self, name, kind=KIND_PARAM):
        """torch view of a named tensor inside the arena (no copy)."""
        torch = self.torch
        p, dt, shape = gpt_tensor(self.h, name, kind)
        tdt = {DTYPE_F32: torch.float32, DTYPE_BF16: torch.bfloat16, DTYPE_I32: torch.int32}[dt]
        esz = 2 if dt == DTYPE_BF16 else 4
        rows, cols = shape[0], shape[1]
        off = p - self.arena.data_ptr()
        return self.arena[off:off + rows * cols * esz].view(tdt).view(rows, cols)

    def forward_loss(self, tokens, targets):
        gpt_forward_loss(self.h, tokens, targets, self.loss)
        return self.loss

    def backward_step(self, lr):
        gpt_backward_step(self.h, lr)

    def backward(self, lr):
        """Backward of the last forward without the dense optimizer step (the
        table updates run inline unless set_table_exchange is on); pair with
        optimizer_step."""
        gpt_backward(self.h, lr)

    def optimizer_step(self, lr):
        gpt_optimizer_step(self.h, lr)

    def set_table_exchange(self, on):
        """Leave the bigram-table gradients to the caller instead of applying
        them inside backward (data-parallel replicas: see dp.exchange_tables)."""
        _check(_lib.gpt_set_table_exchange(self.h, int(on)), "gpt_set_table_exchange")
        self.table_exchange = bool(on)

    def grad_sumsq(self, lo, hi, out):
        """Sum of squares of the flat gradient over [lo, hi) into `out` (device float64 [1])."""
        _check(_lib.gpt_grad_sumsq(self.h, lo, hi, _ptr(out)), "gpt_grad_sumsq")

    def optimizer_step_range(self, lr, lo, hi, grad_sumsq=None):
        """AdamW on the flat elements [lo, hi) only (a sharded optimizer step)."""
        _check(_lib.gpt_optimizer_step_range(self.h, lr, lo, hi, _ptr(grad_sumsq)), "gpt_optimizer_step_range")

    def flat_param(self):
        """The whole fp32 dense master buffer as one flat torch view (no copy)."""
        p, _, shape = gpt_tensor(self.h, "*", KIND_PARAM)
        off = p - self.arena.data_ptr()
        return self.arena[off:off + shape[0] * 4].view(self.torch.float32)

    def params_changed(self):
        gpt_params_changed(self.h)

    def flat_grad(self):
        """The whole fp32 dense gradient as one flat torch view (no copy)."""
        p, _, shape = gpt_tensor(self.h, "*", KIND_GRAD)
        off = p - self.arena.data_ptr()
        return self.arena[off:off + shape[0] * 4].view(self.torch.float32)

    def sync_status(self):
        return gpt_sync_status(self.h)

    def close(self):
        if self.h:
            gpt_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
