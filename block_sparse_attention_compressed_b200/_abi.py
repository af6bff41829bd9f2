"""ctypes binding of libbsa.so (include/bsa.h). Argument marshalling only: every step of the
computation runs in the library's CUDA kernels. The functions keep the C names and take torch
tensors (device memory owned by torch) plus an optional stream (default: torch's current stream).
There is no fallback: if the library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbsa.so")

BSA_OK = 0
BSA_ERR_INVALID_ARG = 1
BSA_ERR_UNSUPPORTED = 2
BSA_ERR_WORKSPACE = 3
BSA_ERR_CUDA = 4
BSA_ERR_DEVICE_CHECK = 5

BSA_F32 = 0
BSA_BF16 = 1
BSA_MAX_LAYERS = 16

DEVERR_SEQ_LEN = 1 << 0
DEVERR_CAPACITY = 1 << 1
DEVERR_BLOCK_IDX = 1 << 2
DEVERR_N_SEL = 1 << 3


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class Params(ctypes.Structure):
    """Mirror of bsa_params_t."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("cmp_kernel", ctypes.c_int32), ("cmp_stride", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("n_init", ctypes.c_int32), ("n_local", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("max_seq_len", ctypes.c_int64),
        ("num_layers", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
        ("score_tau", ctypes.c_float),
    ]

    def __repr__(self):
        return "Params(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class Sizes(ctypes.Structure):
    """Mirror of bsa_sizes_t."""
    _fields_ = [("nc_cap", ctypes.c_int64), ("nb_cap", ctypes.c_int64), ("sel_cap", ctypes.c_int32),
                ("group", ctypes.c_int32), ("workspace_bytes", ctypes.c_size_t)]


_lib = None
_lock = threading.Lock()
_P = ctypes.c_void_p
_S = ctypes.c_int
_PP = ctypes.POINTER(Params)

_SIGS = {
    "bsa_status_string": (ctypes.c_char_p, [_S]),
    "bsa_abi_version": (ctypes.c_int32, []),
    "bsa_check_params": (_S, [_PP]),
    "bsa_get_sizes": (_S, [_PP, ctypes.POINTER(Sizes)]),
    "bsa_workspace_size": (ctypes.c_size_t, [_PP]),
    "bsa_workspace_init": (_S, [_PP, _P, ctypes.c_size_t, _P]),
    "bsa_compress_keys": (_S, [_PP, _P, _P, _P, _P]),
    "bsa_compress_append": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "bsa_select_blocks": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "bsa_select_blocks_forecast": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "bsa_sparse_decode": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "bsa_sparse_decode_layers": (_S, [_PP, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]),
    "bsa_decode_step": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                             ctypes.c_size_t, _P]),
    "bsa_decode_step_fused": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                   ctypes.c_size_t, _P]),
    "bsa_decode_step_lookahead": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                       ctypes.c_size_t, _P]),
    "bsa_decode_step_clsa": (_S, [_PP, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "bsa_clsa_workspace_size": (ctypes.c_size_t, [_PP]),
    "bsa_prefill": (_S, [_PP, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "bsa_prefill_attend": (_S, [_PP, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                _P]),
    "bsa_prefill_tiles": (ctypes.c_int32, [ctypes.c_int32, ctypes.c_int32]),
    "bsa_decode_step_anchored": (_S, [_PP, ctypes.c_int32, _P, ctypes.c_int32, _P, _P, _P, _P, _P,
                                      _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "bsa_read_device_error": (_S, [_P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32), _P]),
    "bsa_decode_step_info": (_S, [_PP, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.POINTER(ctypes.c_int32)]),
    "bsa_sparse_decode_noalloc": (_S, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
}


def lib():
    """The loaded libbsa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libbsa.so not found at {LIB_PATH}: build it with "
                    "`python -m block_sparse_attention_compressed_b200.build` (nvcc, sm_100a)")
            h = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(h, name)
                fn.restype = res
                fn.argtypes = args
            _lib = h
    return _lib


def status_string(status: int) -> str:
    return lib().bsa_status_string(status).decode()


def _check(status: int, where: str):
    if status != BSA_OK:
        raise BsaError(status, where)


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t, name, dtype=None, numel=None, optional=False):
    """Device pointer of a contiguous CUDA tensor after shape/dtype checks."""
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")
    return ctypes.c_void_p(t.data_ptr())


def make_params(batch, num_q_heads, num_kv_heads, head_dim, max_seq_len, dtype="bf16", n_init=1,
                n_local=2, top_k=16, cmp_kernel=32, cmp_stride=16, block_size=64, num_layers=1,
                scale=0.0, score_tau=0.0) -> Params:
    return Params(batch=batch, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                  head_dim=head_dim, cmp_kernel=cmp_kernel, cmp_stride=cmp_stride,
                  block_size=block_size, n_init=n_init, n_local=n_local, top_k=top_k,
                  max_seq_len=max_seq_len, num_layers=num_layers,
                  dtype=BSA_F32 if dtype in ("f32", "float32", BSA_F32) else BSA_BF16,
                  scale=scale, score_tau=score_tau)


def _elem(p: Params):
    import torch
    return torch.float32 if p.dtype == BSA_F32 else torch.bfloat16


def bsa_abi_version() -> int:
    return lib().bsa_abi_version()


def bsa_check_params(p: Params) -> int:
    return lib().bsa_check_params(ctypes.byref(p))


def bsa_get_sizes(p: Params) -> Sizes:
    s = Sizes()
    _check(lib().bsa_get_sizes(ctypes.byref(p), ctypes.byref(s)), "bsa_get_sizes")
    return s


def bsa_workspace_size(p: Params) -> int:
    return int(lib().bsa_workspace_size(ctypes.byref(p)))


def bsa_workspace_init(p: Params, ws, stream=None):
    _check(lib().bsa_workspace_init(ctypes.byref(p), _ptr(ws, "workspace"), ws.numel() * ws.element_size(),
                                    _stream(stream)), "bsa_workspace_init")


def alloc_workspace(p: Params, device="cuda"):
    """A zero-initialised workspace tensor of bsa_workspace_size bytes (torch allocates it)."""
    import torch
    n = bsa_workspace_size(p)
    if n == 0:
        raise BsaError(bsa_check_params(p), "bsa_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _shapes(p: Params):
    s = bsa_get_sizes(p)
    pairs = p.batch * p.num_kv_heads
    return dict(
        q=p.batch * p.num_q_heads * p.head_dim,
        cache=pairs * p.max_seq_len * p.head_dim,
        ck=pairs * s.nc_cap * p.head_dim,
        new=pairs * p.head_dim,
        idx=pairs * s.sel_cap,
        pairs=pairs,
        scores=pairs * s.nb_cap,
        lse=p.batch * p.num_q_heads,
    )


def bsa_compress_keys(p: Params, k_cache, seq_lens, ck, stream=None):
    import torch
    n, e = _shapes(p), _elem(p)
    _check(lib().bsa_compress_keys(ctypes.byref(p), _ptr(k_cache, "k_cache", e, n["cache"]),
                                   _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
                                   _ptr(ck, "ck", e, n["ck"]), _stream(stream)),
           "bsa_compress_keys")


def bsa_compress_append(p: Params, k_cache, v_cache, k_new, v_new, seq_lens, ck, ws=None,
                        stream=None):
    import torch
    n, e = _shapes(p), _elem(p)
    _check(lib().bsa_compress_append(
        ctypes.byref(p), _ptr(k_cache, "k_cache", e, n["cache"]),
        _ptr(v_cache, "v_cache", e, n["cache"]), _ptr(k_new, "k_new", e, n["new"]),
        _ptr(v_new, "v_new", e, n["new"]), _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(ck, "ck", e, n["ck"]), _ptr(ws, "workspace", optional=True),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_compress_append")


def bsa_select_blocks(p: Params, q, ck, seq_lens, block_idx, n_sel, block_scores, ws,
                      stream=None):
    import torch
    n, e = _shapes(p), _elem(p)
    _check(lib().bsa_select_blocks(
        ctypes.byref(p), _ptr(q, "q", e, n["q"]), _ptr(ck, "ck", e, n["ck"]),
        _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"]),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"]),
        _ptr(block_scores, "block_scores", torch.float32, n["scores"], optional=True),
        _ptr(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_select_blocks")


def bsa_select_blocks_forecast(p: Params, f, ck, seq_lens, block_idx, n_sel, block_scores, ws,
                               stream=None):
    """Selection from one Forecast vector per (batch, kv head), f [B][Hkv][d]."""
    import torch
    n, e = _shapes(p), _elem(p)
    _check(lib().bsa_select_blocks_forecast(
        ctypes.byref(p), _ptr(f, "f", e, n["pairs"] * p.head_dim), _ptr(ck, "ck", e, n["ck"]),
        _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"]),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"]),
        _ptr(block_scores, "block_scores", torch.float32, n["scores"], optional=True),
        _ptr(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_select_blocks_forecast")


def bsa_sparse_decode(p: Params, q, k_cache, v_cache, seq_lens, block_idx, n_sel, out, lse, ws,
                      stream=None):
    import torch
    n, e = _shapes(p), _elem(p)
    _check(lib().bsa_sparse_decode(
        ctypes.byref(p), _ptr(q, "q", e, n["q"]), _ptr(k_cache, "k_cache", e, n["cache"]),
        _ptr(v_cache, "v_cache", e, n["cache"]), _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"]),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"]), _ptr(out, "out", e, n["q"]),
        _ptr(lse, "lse", torch.float32, n["lse"], optional=True), _ptr(ws, "workspace"),
        ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_sparse_decode")


def bsa_sparse_decode_noalloc(p: Params, q, k_cache, v_cache, seq_lens, block_idx, n_sel, out,
                              lse=None, device_error=None, stream=None):
    """bsa_sparse_decode without a workspace, for callers that cannot allocate device memory: the
    library keeps the split partials in its own fixed per-device scratch. ``device_error`` is an
    optional int32 tensor of one element that receives the device error bits (OR-ed in)."""
    import torch
    n, e = _shapes(p), _elem(p)
    _check(lib().bsa_sparse_decode_noalloc(
        ctypes.byref(p), _ptr(q, "q", e, n["q"]), _ptr(k_cache, "k_cache", e, n["cache"]),
        _ptr(v_cache, "v_cache", e, n["cache"]), _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"]),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"]), _ptr(out, "out", e, n["q"]),
        _ptr(lse, "lse", torch.float32, n["lse"], optional=True),
        _ptr(device_error, "device_error", torch.int32, 1, optional=True), _stream(stream)),
        "bsa_sparse_decode_noalloc")


def bsa_sparse_decode_layers(p: Params, qs, k_caches, v_caches, seq_lens, block_idx, n_sel, outs,
                             lses, ws, stream=None):
    import torch
    n, e = _shapes(p), _elem(p)
    L = len(qs)
    if not (len(k_caches) == len(v_caches) == len(outs) == L) or (lses is not None and len(lses) != L):
        raise ValueError("per-layer lists must have the same length")
    arr = ctypes.c_void_p * L
    q_a = arr(*[_ptr(t, "q", e, n["q"]) for t in qs])
    k_a = arr(*[_ptr(t, "k_cache", e, n["cache"]) for t in k_caches])
    v_a = arr(*[_ptr(t, "v_cache", e, n["cache"]) for t in v_caches])
    o_a = arr(*[_ptr(t, "out", e, n["q"]) for t in outs])
    l_a = None if lses is None else arr(*[_ptr(t, "lse", torch.float32, n["lse"], optional=True)
                                          for t in lses])
    _check(lib().bsa_sparse_decode_layers(
        ctypes.byref(p), L, q_a, k_a, v_a, _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"]),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"]), o_a, l_a, _ptr(ws, "workspace"),
        ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_sparse_decode_layers")


def bsa_clsa_workspace_size(p: Params) -> int:
    """Workspace bytes of bsa_decode_step_clsa (0 when unsupported)."""
    return int(lib().bsa_clsa_workspace_size(ctypes.byref(p)))


def alloc_clsa_workspace(p: Params, device="cuda"):
    """A zero-initialised workspace of bsa_clsa_workspace_size bytes (torch allocates it)."""
    import torch
    n = bsa_clsa_workspace_size(p)
    if n == 0:
        raise BsaError(BSA_ERR_UNSUPPORTED, "bsa_clsa_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def bsa_decode_step_clsa(p: Params, qs, k_caches, v_caches, seq_lens, tok_idx, n_tok, outs, lses, ws,
                         stream=None):
    """bsa_decode_step_clsa: layer 0's token-level index, attended by every layer of the lists."""
    import torch
    n, e = _shapes(p), _elem(p)
    L = len(qs)
    if not (len(k_caches) == len(v_caches) == len(outs) == L) or (lses is not None and len(lses) != L):
        raise ValueError("per-layer lists must have the same length")
    arr = ctypes.c_void_p * L
    tok_cap = (p.n_init + p.n_local + p.top_k) * p.block_size
    q_a = arr(*[_ptr(t, "q", e, n["q"]) for t in qs])
    k_a = arr(*[_ptr(t, "k_cache", e, n["cache"]) for t in k_caches])
    v_a = arr(*[_ptr(t, "v_cache", e, n["cache"]) for t in v_caches])
    o_a = arr(*[_ptr(t, "out", e, n["q"]) for t in outs])
    l_a = None if lses is None else arr(*[_ptr(t, "lse", torch.float32, n["lse"], optional=True) for t in lses])
    _check(lib().bsa_decode_step_clsa(
        ctypes.byref(p), L, q_a, k_a, v_a, _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(tok_idx, "tok_idx", torch.int32, n["pairs"] * tok_cap), _ptr(n_tok, "n_tok", torch.int32, n["pairs"]),
        o_a, l_a, _ptr(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_decode_step_clsa")


def bsa_decode_step_anchored(p: Params, anchors, qs, k_caches, v_caches, cks, seq_lens, block_idx,
                             n_sel, outs, lses, ws, stream=None):
    """Anchored index reuse: one selection per anchor layer, reused by the layers up to the next
    anchor. block_idx is [num_anchors][B][Hkv][SEL_cap], n_sel [num_anchors][B][Hkv]; cks lists one
    compressed-key tensor per layer (None where the layer is not an anchor)."""
    import torch
    n, e = _shapes(p), _elem(p)
    L, A = len(qs), len(anchors)
    if not (len(k_caches) == len(v_caches) == len(outs) == len(cks) == L) or \
            (lses is not None and len(lses) != L):
        raise ValueError("per-layer lists must have the same length")
    arr = ctypes.c_void_p * L
    anc = set(int(a) for a in anchors)
    q_a = arr(*[_ptr(t, "q", e, n["q"]) for t in qs])
    k_a = arr(*[_ptr(t, "k_cache", e, n["cache"]) for t in k_caches])
    v_a = arr(*[_ptr(t, "v_cache", e, n["cache"]) for t in v_caches])
    c_a = arr(*[_ptr(t, "ck", e, n["ck"]) if i in anc else None for i, t in enumerate(cks)])
    o_a = arr(*[_ptr(t, "out", e, n["q"]) for t in outs])
    l_a = None if lses is None else arr(*[_ptr(t, "lse", torch.float32, n["lse"], optional=True)
                                          for t in lses])
    a_a = (ctypes.c_int32 * A)(*[int(a) for a in anchors])
    _check(lib().bsa_decode_step_anchored(
        ctypes.byref(p), L, a_a, A, q_a, k_a, v_a, c_a,
        _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"] * A),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"] * A), o_a, l_a, _ptr(ws, "workspace"),
        ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_decode_step_anchored")


def bsa_decode_step_info(p: Params, append: bool = False) -> tuple[bool, int]:
    """(fused, launches) of bsa_decode_step for these parameters: whether one kernel runs the
    whole step, and the kernel launches of one call (with the append when ``append``)."""
    fused, launches = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().bsa_decode_step_info(ctypes.byref(p), int(bool(append)), ctypes.byref(fused),
                                      ctypes.byref(launches)), "bsa_decode_step_info")
    return bool(fused.value), int(launches.value)


def bsa_decode_step(p: Params, q, k_cache, v_cache, ck, k_new, v_new, seq_lens, block_idx, n_sel,
                    block_scores, out, lse, ws, stream=None, fused=False):
    """bsa_decode_step (or, with ``fused``, bsa_decode_step_fused)."""
    import torch
    n, e = _shapes(p), _elem(p)
    name = "bsa_decode_step_fused" if fused else "bsa_decode_step"
    _check(getattr(lib(), name)(
        ctypes.byref(p), _ptr(q, "q", e, n["q"]), _ptr(k_cache, "k_cache", e, n["cache"]),
        _ptr(v_cache, "v_cache", e, n["cache"]), _ptr(ck, "ck", e, n["ck"]),
        _ptr(k_new, "k_new", e, n["new"], optional=True),
        _ptr(v_new, "v_new", e, n["new"], optional=True),
        _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"]),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"]),
        _ptr(block_scores, "block_scores", torch.float32, n["scores"], optional=True),
        _ptr(out, "out", e, n["q"]), _ptr(lse, "lse", torch.float32, n["lse"], optional=True),
        _ptr(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)),
        name)


def bsa_decode_step_lookahead(p: Params, q, k_cache, v_cache, block_idx, n_sel, f, ck_next, seq_lens,
                              block_idx_next, n_sel_next, block_scores_next, out, lse, ws,
                              stream=None):
    """bsa_decode_step_lookahead: this layer attends block_idx / n_sel while the next layer's
    blocks are chosen from f (one Forecast vector per (batch, kv head)) against ck_next."""
    import torch
    n, e = _shapes(p), _elem(p)
    _check(lib().bsa_decode_step_lookahead(
        ctypes.byref(p), _ptr(q, "q", e, n["q"]), _ptr(k_cache, "k_cache", e, n["cache"]),
        _ptr(v_cache, "v_cache", e, n["cache"]),
        _ptr(block_idx, "block_idx", torch.int32, n["idx"]),
        _ptr(n_sel, "n_sel", torch.int32, n["pairs"]),
        _ptr(f, "f", e, n["pairs"] * p.head_dim), _ptr(ck_next, "ck_next", e, n["ck"]),
        _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
        _ptr(block_idx_next, "block_idx_next", torch.int32, n["idx"]),
        _ptr(n_sel_next, "n_sel_next", torch.int32, n["pairs"]),
        _ptr(block_scores_next, "block_scores_next", torch.float32, n["scores"], optional=True),
        _ptr(out, "out", e, n["q"]), _ptr(lse, "lse", torch.float32, n["lse"], optional=True),
        _ptr(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)),
        "bsa_decode_step_lookahead")


def bsa_prefill_tiles(chunk: int, block_size: int = 64) -> int:
    """Query tiles per (batch, kv head) pair of a prefill chunk."""
    return int(lib().bsa_prefill_tiles(int(chunk), int(block_size)))


def _prefill_ptrs(p: Params, chunk, q, seq_lens, block_idx, n_sel, out, lse):
    import torch
    e = _elem(p)
    pairs = p.batch * p.num_kv_heads
    tiles = bsa_prefill_tiles(chunk, p.block_size)
    sel_cap = p.n_init + p.n_local + p.top_k
    qn = p.batch * chunk * p.num_q_heads * p.head_dim
    return (_ptr(q, "q", e, qn), _ptr(seq_lens, "seq_lens", torch.int32, p.batch),
            _ptr(block_idx, "block_idx", torch.int32, pairs * tiles * sel_cap),
            _ptr(n_sel, "n_sel", torch.int32, pairs * tiles), _ptr(out, "out", e, qn),
            _ptr(lse, "lse", torch.float32, p.batch * chunk * p.num_q_heads, optional=True))


def bsa_prefill(p: Params, chunk: int, q, k_cache, v_cache, ck, seq_lens, block_idx, n_sel, out, lse, ws,
                stream=None):
    """bsa_prefill: the last `chunk` positions of every sequence, one selection per query tile."""
    n, e = _shapes(p), _elem(p)
    qp, sp, ip, np_, op, lp = _prefill_ptrs(p, chunk, q, seq_lens, block_idx, n_sel, out, lse)
    _check(lib().bsa_prefill(ctypes.byref(p), int(chunk), qp, _ptr(k_cache, "k_cache", e, n["cache"]),
                             _ptr(v_cache, "v_cache", e, n["cache"]), _ptr(ck, "ck", e, n["ck"]), sp, ip, np_,
                             op, lp, _ptr(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)),
           "bsa_prefill")


def bsa_prefill_attend(p: Params, chunk: int, q, k_cache, v_cache, seq_lens, block_idx, n_sel, out, lse, ws,
                       stream=None):
    """bsa_prefill_attend: the prefill attention with the tiles' blocks given."""
    n, e = _shapes(p), _elem(p)
    qp, sp, ip, np_, op, lp = _prefill_ptrs(p, chunk, q, seq_lens, block_idx, n_sel, out, lse)
    _check(lib().bsa_prefill_attend(ctypes.byref(p), int(chunk), qp, _ptr(k_cache, "k_cache", e, n["cache"]),
                                    _ptr(v_cache, "v_cache", e, n["cache"]), sp, ip, np_, op, lp,
                                    _ptr(ws, "workspace"), ws.numel() * ws.element_size(), _stream(stream)),
           "bsa_prefill_attend")


def bsa_read_device_error(ws, stream=None) -> int:
    """Device error bits (and clears them); synchronizes the stream."""
    flags = ctypes.c_uint32(0)
    st = lib().bsa_read_device_error(_ptr(ws, "workspace"), ws.numel() * ws.element_size(),
                                     ctypes.byref(flags), _stream(stream))
    if st not in (BSA_OK, BSA_ERR_DEVICE_CHECK):
        raise BsaError(st, "bsa_read_device_error")
    return int(flags.value)


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
