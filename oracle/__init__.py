"""CPU oracle for block-sparse compressed-key decode attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. The product path (the CUDA library and its binding) never imports it, and it never
imports the product path.

The arithmetic lives in ``bsa_oracle.c`` (plain C, IEEE double, one function per step of the
method, each citing the passage it follows; the readings of the pages are listed in
``bsa_oracle.h``). This module only builds that library on demand and marshals numpy arrays.

Storage conventions: bf16 tensors are passed as ``numpy.uint16`` bit patterns, fp32 tensors as
``numpy.float32``. ``raw(t)`` converts a torch tensor (any device) to that form.

Pins (what holds this oracle to something other than itself) are in
``tests/test_oracle_pins.py``; every public function here has at least one.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
import subprocess
import threading

import numpy as np

F32 = 0
BF16 = 1
NO_ROUND = -1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsa_oracle.c")
_HDR = os.path.join(_HERE, "bsa_oracle.h")
_LIB_PATH = os.path.join(_HERE, "libbsa_oracle.so")
_lock = threading.Lock()
_lib = None


def compile_source(src: str, out: str, include_dir: str = _HERE) -> str:
    """gcc -O2, OpenMP, no FMA contraction: ``src`` -> shared library ``out``."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-Wall", "-shared", "-fPIC",
           "-I", include_dir, src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libbsa_oracle.so`` when it is missing or stale."""
    stale = (not os.path.exists(_LIB_PATH)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB_PATH) for p in (_SRC, _HDR))
    if force or stale:
        compile_source(_SRC, _LIB_PATH)
    return _LIB_PATH


class Problem(ctypes.Structure):
    """Mirror of ``orc_problem_t``."""
    _fields_ = [
        ("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("cmp_kernel", ctypes.c_int), ("cmp_stride", ctypes.c_int),
        ("block_size", ctypes.c_int), ("n_init", ctypes.c_int), ("n_local", ctypes.c_int),
        ("top_k", ctypes.c_int), ("max_seq_len", ctypes.c_int64), ("dtype", ctypes.c_int),
        ("scale", ctypes.c_double), ("tau", ctypes.c_double),
    ]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_D = ctypes.c_double


def _bind(path: str):
    lib = ctypes.CDLL(path)
    sig = {
        "bsa_oracle_round": (_D, [_D, _INT]),
        "bsa_oracle_round_array": (None, [_P, _I64, _INT, _P]),
        "bsa_oracle_load": (_D, [_P, _INT, _I64]),
        "bsa_oracle_num_windows": (_I64, [_I64, _INT, _INT]),
        "bsa_oracle_num_blocks": (_I64, [_I64, _INT]),
        "bsa_oracle_compress": (_I64, [_P, _INT, _I64, _INT, _INT, _INT, _INT, _P]),
        "bsa_oracle_group_scores": (None, [_P, _P, _I64, _INT, _INT, _D, _P]),
        "bsa_oracle_forecast_scores": (None, [_P, _P, _I64, _INT, _P]),
        "bsa_oracle_block_scores": (None, [_P, _I64, _I64, _INT, _INT, _INT, _P]),
        "bsa_oracle_select": (_INT, [_P, _I64, _INT, _INT, _INT, _P, _P]),
        "bsa_oracle_attend": (None, [_P, _P, _P, _INT, _I64, _INT, _INT, _P, _INT, _INT,
                                     _D, _P, _P]),
        "bsa_oracle_decode": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _INT,
                                     _P, _P, _P, _P, _P, _P, _P, _P]),
        "bsa_oracle_decode_forecast": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P,
                                              _INT, _P, _P, _P, _P, _P, _P]),
        "bsa_oracle_attend_pairs": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P,
                                           _INT, _P, _P, _P, _P]),
        "bsa_oracle_compress_cache": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _INT,
                                             _P]),
        "bsa_oracle_num_threads": (_INT, []),
        "bsa_oracle_set_num_threads": (None, [_INT]),
        "bsa_oracle_decode_ck": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P, _INT,
                                        _P, _P, _P, _P, _P, _P]),
        "bsa_oracle_decode_forecast_ck": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P, _P,
                                                 _INT, _P, _P, _P, _P, _P, _P]),
        "bsa_oracle_select_forecast_ck": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _INT,
                                                 _P, _P, _P, _P]),
        "bsa_oracle_prefill": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _INT, _P, _INT, _INT,
                                      _P, _P, _P, _P, _P]),
        "bsa_oracle_token_select": (_INT, [ctypes.POINTER(Problem), _P, _P, _P, _P, _INT, _P, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


@contextlib.contextmanager
def using(path: str):
    """Run the wrappers against another build of the oracle source (a planted-mistake copy in the
    mutation tests), then switch back."""
    global _lib
    other = _bind(path)
    _load()
    with _lock:
        saved, _lib = _lib, other
    try:
        yield
    finally:
        with _lock:
            _lib = saved


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _raw_check(a: np.ndarray, dtype: int) -> np.ndarray:
    want = np.float32 if dtype == F32 else np.uint16
    if a.dtype != want:
        raise TypeError(f"expected storage array of {want.__name__}, got {a.dtype}")
    return np.ascontiguousarray(a)


def raw(t) -> tuple[np.ndarray, int]:
    """(storage array, dtype code) of a torch tensor: bf16 -> uint16 bits, fp32 -> float32."""
    import torch
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), BF16
    if t.dtype == torch.float32:
        return t.numpy(), F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def widen(a: np.ndarray, dtype: int) -> np.ndarray:
    """Storage array -> float64 array of the same shape."""
    if dtype == F32:
        return a.astype(np.float64)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def num_threads() -> int:
    return _load().bsa_oracle_num_threads()


@contextlib.contextmanager
def threads(n: int):
    """Run the OpenMP loops over pairs on n threads inside the block (timing only)."""
    lib = _load()
    saved = lib.bsa_oracle_num_threads()
    lib.bsa_oracle_set_num_threads(n)
    try:
        yield
    finally:
        lib.bsa_oracle_set_num_threads(saved)


def round_to(x, dtype: int) -> np.ndarray:
    """Round doubles to the nearest bf16 / fp32 value (ties to even), returned as float64."""
    x = _f64(x)
    y = np.empty_like(x)
    _load().bsa_oracle_round_array(_ptr(x), x.size, dtype, _ptr(y))
    return y


def num_windows(T: int, l: int, s: int) -> int:
    return int(_load().bsa_oracle_num_windows(T, l, s))


def num_blocks(T: int, block_size: int) -> int:
    return int(_load().bsa_oracle_num_blocks(T, block_size))


def compress(k: np.ndarray, dtype: int, l: int = 32, s: int = 16,
             round_dtype: int | None = None) -> np.ndarray:
    """Eq. (2) on one [T][d] key matrix -> float64 [nc][d]; rounded to ``dtype`` by default."""
    k = _raw_check(k, dtype)
    T, d = k.shape
    nc = num_windows(T, l, s)
    out = np.zeros((max(nc, 0), d), dtype=np.float64)
    rd = dtype if round_dtype is None else round_dtype
    _load().bsa_oracle_compress(_ptr(k), dtype, T, d, l, s, rd, _ptr(out))
    return out


def group_scores(q, ck, tau: float) -> np.ndarray:
    """Eq. (6) target form for one group: q [G][d], ck [nc][d] -> S [nc]."""
    q, ck = _f64(q), _f64(ck)
    G, d = q.shape
    nc = ck.shape[0]
    S = np.zeros(nc, dtype=np.float64)
    _load().bsa_oracle_group_scores(_ptr(q), _ptr(ck), nc, G, d, tau, _ptr(S))
    return S


def forecast_scores(f, ck) -> np.ndarray:
    """Eq. (4) with the Compact Forecast Indexer: f [d], ck [nc][d] -> S [nc] = f . ck_j."""
    f, ck = _f64(f), _f64(ck)
    nc, d = ck.shape
    S = np.zeros(nc, dtype=np.float64)
    _load().bsa_oracle_forecast_scores(_ptr(f), _ptr(ck), nc, d, _ptr(S))
    return S


def block_scores(S, nb: int, l: int = 32, s: int = 16, block_size: int = 64) -> np.ndarray:
    S = _f64(S)
    sb = np.zeros(nb, dtype=np.float64)
    _load().bsa_oracle_block_scores(_ptr(S), S.size, nb, l, s, block_size, _ptr(sb))
    return sb


def select(sb, n_init: int, n_local: int, top_k: int) -> tuple[np.ndarray, np.ndarray]:
    """Eq. (1)/(4): ascending selected block indices and (k-th taken, best left-out) scores."""
    sb = _f64(sb)
    idx = np.full(n_init + n_local + top_k + 1, -1, dtype=np.int32)
    bnd = np.zeros(2, dtype=np.float64)
    n = _load().bsa_oracle_select(_ptr(sb), sb.size, n_init, n_local, top_k, _ptr(idx), _ptr(bnd))
    return idx[:n].copy(), bnd


def attend(q, k: np.ndarray, v: np.ndarray, dtype: int, T: int, idx, block_size: int = 64,
           scale: float | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Eq. (5) for one group: q [G][d] (float64), K/V [rows][d] storage arrays -> out, lse."""
    q = _f64(q)
    k, v = _raw_check(k, dtype), _raw_check(v, dtype)
    G, d = q.shape
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((G, d), dtype=np.float64)
    lse = np.zeros(G, dtype=np.float64)
    _load().bsa_oracle_attend(_ptr(q), _ptr(k), _ptr(v), dtype, T, d, G, _ptr(idx), idx.size,
                              block_size, scale, _ptr(out), _ptr(lse))
    return out, lse


def make_problem(batch, num_q_heads, num_kv_heads, head_dim, max_seq_len, dtype, n_init, n_local,
                 top_k, cmp_kernel=32, cmp_stride=16, block_size=64, scale=None, tau=None):
    return Problem(batch=batch, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                   head_dim=head_dim, cmp_kernel=cmp_kernel, cmp_stride=cmp_stride,
                   block_size=block_size, n_init=n_init, n_local=n_local, top_k=top_k,
                   max_seq_len=max_seq_len, dtype=dtype,
                   scale=(1.0 / math.sqrt(head_dim)) if scale is None else scale,
                   tau=math.sqrt(head_dim) if tau is None else tau)


def _sizes(P: Problem):
    G = P.num_q_heads // P.num_kv_heads
    sel_cap = P.n_init + P.n_local + P.top_k
    nb_cap = num_blocks(P.max_seq_len, P.block_size)
    return G, sel_cap, nb_cap


def decode(P: Problem, q, k_cache, v_cache, seq_lens, pairs=None, given_idx=None,
           given_n_sel=None, ck=None) -> dict:
    """Select + attend for the listed (batch, kv-head) pairs (all pairs by default).

    q/k_cache/v_cache are storage arrays ([B][Hq][d], [B][Hkv][T_cap][d]); returns a dict with
    idx [n][sel_cap], n_sel [n], block_scores [n][nb_cap], boundary [n][2], out [n][G][d],
    lse [n][G]. With ``given_idx`` the selection is skipped and those blocks are attended. With
    ``ck`` (float64 [n][nc_cap][d], as ``compress_cache`` returns for the same pairs) the
    compressed keys are taken from it instead of being formed from the cache.
    """
    q = _raw_check(q, P.dtype)
    k_cache, v_cache = _raw_check(k_cache, P.dtype), _raw_check(v_cache, P.dtype)
    seq_lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    if pairs is None:
        pairs = np.arange(P.batch * P.num_kv_heads, dtype=np.int32)
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    n = pairs.size
    G, sel_cap, nb_cap = _sizes(P)
    d = P.head_dim
    if given_idx is not None:
        given_idx = np.ascontiguousarray(np.asarray(given_idx, dtype=np.int32).reshape(n, sel_cap))
        given_n_sel = np.ascontiguousarray(np.asarray(given_n_sel, dtype=np.int32).reshape(n))
    res = dict(
        idx=np.full((n, sel_cap), -1, dtype=np.int32),
        n_sel=np.zeros(n, dtype=np.int32),
        block_scores=np.full((n, nb_cap), -np.inf, dtype=np.float64),
        boundary=np.full((n, 2), np.nan, dtype=np.float64),
        out=np.zeros((n, G, d), dtype=np.float64),
        lse=np.zeros((n, G), dtype=np.float64),
    )
    if ck is not None:
        if given_idx is not None:
            raise ValueError("given compressed keys are for a selection, not given indices")
        nc_cap = num_windows(P.max_seq_len, P.cmp_kernel, P.cmp_stride)
        ck = np.ascontiguousarray(np.asarray(ck, dtype=np.float64))
        if ck.shape != (n, max(nc_cap, 0), d):
            raise ValueError(f"ck must be [{n}][{nc_cap}][{d}] float64")
        rc = _load().bsa_oracle_decode_ck(
            ctypes.byref(P), _ptr(q), _ptr(ck), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
            _ptr(pairs), n, _ptr(res["idx"]), _ptr(res["n_sel"]), _ptr(res["block_scores"]),
            _ptr(res["boundary"]), _ptr(res["out"]), _ptr(res["lse"]))
    else:
        rc = _load().bsa_oracle_decode(
            ctypes.byref(P), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), _ptr(pairs), n,
            _ptr(given_idx), _ptr(given_n_sel), _ptr(res["idx"]), _ptr(res["n_sel"]),
            _ptr(res["block_scores"]), _ptr(res["boundary"]), _ptr(res["out"]), _ptr(res["lse"]))
    if rc != 0:
        raise ValueError("bsa_oracle_decode rejected its arguments")
    return res


def decode_forecast(P: Problem, f, q, k_cache, v_cache, seq_lens, pairs=None, ck=None) -> dict:
    """As ``decode``, with the blocks selected from the Forecast vectors f [B][Hkv][d] (storage
    array of the problem's dtype) instead of the queries; q attends them. ``ck`` as in ``decode``."""
    f = _raw_check(f, P.dtype)
    q = _raw_check(q, P.dtype)
    k_cache, v_cache = _raw_check(k_cache, P.dtype), _raw_check(v_cache, P.dtype)
    seq_lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    if pairs is None:
        pairs = np.arange(P.batch * P.num_kv_heads, dtype=np.int32)
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    n = pairs.size
    G, sel_cap, nb_cap = _sizes(P)
    res = dict(
        idx=np.full((n, sel_cap), -1, dtype=np.int32),
        n_sel=np.zeros(n, dtype=np.int32),
        block_scores=np.full((n, nb_cap), -np.inf, dtype=np.float64),
        boundary=np.full((n, 2), np.nan, dtype=np.float64),
        out=np.zeros((n, G, P.head_dim), dtype=np.float64),
        lse=np.zeros((n, G), dtype=np.float64),
    )
    if ck is not None:
        nc_cap = num_windows(P.max_seq_len, P.cmp_kernel, P.cmp_stride)
        ck = np.ascontiguousarray(np.asarray(ck, dtype=np.float64))
        if ck.shape != (n, max(nc_cap, 0), P.head_dim):
            raise ValueError(f"ck must be [{n}][{nc_cap}][{P.head_dim}] float64")
        rc = _load().bsa_oracle_decode_forecast_ck(
            ctypes.byref(P), _ptr(f), _ptr(q), _ptr(ck), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
            _ptr(pairs), n, _ptr(res["idx"]), _ptr(res["n_sel"]), _ptr(res["block_scores"]),
            _ptr(res["boundary"]), _ptr(res["out"]), _ptr(res["lse"]))
    else:
        rc = _load().bsa_oracle_decode_forecast(
            ctypes.byref(P), _ptr(f), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
            _ptr(pairs), n, _ptr(res["idx"]), _ptr(res["n_sel"]), _ptr(res["block_scores"]),
            _ptr(res["boundary"]), _ptr(res["out"]), _ptr(res["lse"]))
    if rc != 0:
        raise ValueError("bsa_oracle_decode_forecast rejected its arguments")
    return res


def select_forecast(P: Problem, f, ck, seq_lens, pairs=None) -> dict:
    """The Forecast selection alone (SparDA Architecture, Eq. 4): the blocks that f [B][Hkv][d]
    (storage array of the problem's dtype) chooses among the compressed keys ck (float64
    [n][nc_cap][d], as ``compress_cache`` returns them for the same pairs). Returns idx, n_sel,
    block_scores and boundary as ``decode``."""
    f = _raw_check(f, P.dtype)
    seq_lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    if pairs is None:
        pairs = np.arange(P.batch * P.num_kv_heads, dtype=np.int32)
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    n = pairs.size
    G, sel_cap, nb_cap = _sizes(P)
    nc_cap = num_windows(P.max_seq_len, P.cmp_kernel, P.cmp_stride)
    ck = np.ascontiguousarray(np.asarray(ck, dtype=np.float64))
    if ck.shape != (n, max(nc_cap, 0), P.head_dim):
        raise ValueError(f"ck must be [{n}][{nc_cap}][{P.head_dim}] float64")
    res = dict(idx=np.full((n, sel_cap), -1, dtype=np.int32), n_sel=np.zeros(n, dtype=np.int32),
               block_scores=np.full((n, nb_cap), -np.inf, dtype=np.float64),
               boundary=np.full((n, 2), np.nan, dtype=np.float64))
    rc = _load().bsa_oracle_select_forecast_ck(
        ctypes.byref(P), _ptr(f), _ptr(ck), _ptr(seq_lens), _ptr(pairs), n, _ptr(res["idx"]),
        _ptr(res["n_sel"]), _ptr(res["block_scores"]), _ptr(res["boundary"]))
    if rc != 0:
        raise ValueError("bsa_oracle_select_forecast_ck rejected its arguments")
    return res


def lookahead_step(P: Problem, q, k_cache, v_cache, idx, n_sel, f, ck_next, seq_lens,
                   pairs=None) -> dict:
    """One layer l of one-layer-lookahead decoding (SparDA Architecture, Eqs. 4 and 5): layer l's
    queries attend the blocks chosen for it beforehand (idx, n_sel), and layer l + 1's blocks are
    chosen from layer l's Forecast vectors f against layer l + 1's compressed keys ck_next.
    Returns out, lse (layer l) and idx, n_sel, block_scores, boundary (layer l + 1)."""
    att = attend_pairs(P, q, k_cache, v_cache, seq_lens, idx, n_sel, pairs)
    nxt = select_forecast(P, f, ck_next, seq_lens, pairs)
    return dict(out=att["out"], lse=att["lse"], **nxt)


def prefill_tiles_cap(chunk: int, block_size: int = 64) -> int:
    """Most query tiles a chunk of ``chunk`` positions can span (one more when it starts mid-block)."""
    return -(-chunk // block_size) + 1


def prefill(P: Problem, q, k_cache, v_cache, seq_lens, chunk: int, pairs=None) -> dict:
    """Block-sparse prefill of the last ``chunk`` positions of each sequence (see
    ``bsa_oracle_prefill``): q is the chunk's queries [B][C][Hq][d] (storage array of the
    problem's dtype). Returns idx [n][tiles][sel_cap], n_sel [n][tiles] (tile i covers block
    (T - C) // BS + i), boundary [n][tiles][2] (the k-th taken and best rejected block score),
    out [n][C][G][d] and lse [n][C][G]."""
    q = _raw_check(q, P.dtype)
    k_cache, v_cache = _raw_check(k_cache, P.dtype), _raw_check(v_cache, P.dtype)
    seq_lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    if pairs is None:
        pairs = np.arange(P.batch * P.num_kv_heads, dtype=np.int32)
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    n = pairs.size
    G, sel_cap, _ = _sizes(P)
    tiles = prefill_tiles_cap(chunk, P.block_size)
    res = dict(idx=np.full((n, tiles, sel_cap), -1, dtype=np.int32),
               n_sel=np.zeros((n, tiles), dtype=np.int32),
               boundary=np.full((n, tiles, 2), np.nan, dtype=np.float64),
               out=np.zeros((n, chunk, G, P.head_dim), dtype=np.float64),
               lse=np.zeros((n, chunk, G), dtype=np.float64))
    rc = _load().bsa_oracle_prefill(ctypes.byref(P), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(seq_lens), chunk, _ptr(pairs), n, tiles, _ptr(res["idx"]),
                                    _ptr(res["n_sel"]), _ptr(res["boundary"]), _ptr(res["out"]),
                                    _ptr(res["lse"]))
    if rc != 0:
        raise ValueError("bsa_oracle_prefill rejected its arguments")
    return res


def token_select(P: Problem, q, k_cache, seq_lens, pairs=None) -> dict:
    """CLSA's token-level index (``bsa_oracle_token_select``): idx [n][tok_cap] (ascending tokens,
    -1 padded; tok_cap = (n_init + n_local + top_k) * block_size), n_sel [n], boundary [n][2] and
    the token scores [n][max_seq_len] (-inf past each sequence)."""
    q = _raw_check(q, P.dtype)
    k_cache = _raw_check(k_cache, P.dtype)
    seq_lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    if pairs is None:
        pairs = np.arange(P.batch * P.num_kv_heads, dtype=np.int32)
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    n = pairs.size
    tok_cap = (P.n_init + P.n_local + P.top_k) * P.block_size
    res = dict(idx=np.full((n, tok_cap), -1, dtype=np.int32), n_sel=np.zeros(n, dtype=np.int32),
               boundary=np.full((n, 2), np.nan, dtype=np.float64),
               scores=np.full((n, P.max_seq_len), -np.inf, dtype=np.float64))
    rc = _load().bsa_oracle_token_select(ctypes.byref(P), _ptr(q), _ptr(k_cache), _ptr(seq_lens), _ptr(pairs),
                                         n, _ptr(res["idx"]), _ptr(res["n_sel"]), _ptr(res["boundary"]),
                                         _ptr(res["scores"]))
    if rc != 0:
        raise ValueError("bsa_oracle_token_select rejected its arguments")
    return res


def clsa(P: Problem, qs, k_caches, v_caches, seq_lens, pairs=None) -> dict:
    """CLSA decode over the layers of qs / k_caches / v_caches (lists, layer 0 the index layer):
    the token index of layer 0, attended by every layer (tokens as blocks of one). Returns idx,
    n_sel, boundary and out [L][n][G][d], lse [L][n][G]."""
    sel = token_select(P, qs[0], k_caches[0], seq_lens, pairs)
    P1 = Problem.from_buffer_copy(P)  # tokens as blocks of one; the index is given
    P1.top_k = (P.n_init + P.n_local + P.top_k) * P.block_size
    P1.block_size, P1.n_init, P1.n_local = 1, 0, 0
    outs, lses = [], []
    for q, k, v in zip(qs, k_caches, v_caches):
        r = attend_pairs(P1, q, k, v, seq_lens, sel["idx"], sel["n_sel"], pairs)
        outs.append(r["out"])
        lses.append(r["lse"])
    return dict(sel, out=np.stack(outs), lse=np.stack(lses))


def attend_pairs(P: Problem, q, k_cache, v_cache, seq_lens, idx, n_sel, pairs=None) -> dict:
    """Shared-index mode: attend one layer with block indices selected on another layer."""
    q = _raw_check(q, P.dtype)
    k_cache, v_cache = _raw_check(k_cache, P.dtype), _raw_check(v_cache, P.dtype)
    seq_lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    if pairs is None:
        pairs = np.arange(P.batch * P.num_kv_heads, dtype=np.int32)
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    n = pairs.size
    G, sel_cap, _ = _sizes(P)
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(n, sel_cap))
    n_sel = np.ascontiguousarray(np.asarray(n_sel, dtype=np.int32).reshape(n))
    out = np.zeros((n, G, P.head_dim), dtype=np.float64)
    lse = np.zeros((n, G), dtype=np.float64)
    rc = _load().bsa_oracle_attend_pairs(ctypes.byref(P), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(seq_lens), _ptr(pairs), n, _ptr(idx), _ptr(n_sel),
                                         _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("bsa_oracle_attend_pairs rejected its arguments")
    return dict(out=out, lse=lse)


def compress_cache(P: Problem, k_cache, seq_lens, pairs=None) -> np.ndarray:
    """Eq. (2) over whole caches -> float64 [n][nc_cap][d] (rounded to the cache dtype)."""
    k_cache = _raw_check(k_cache, P.dtype)
    seq_lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    if pairs is None:
        pairs = np.arange(P.batch * P.num_kv_heads, dtype=np.int32)
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32))
    nc_cap = num_windows(P.max_seq_len, P.cmp_kernel, P.cmp_stride)
    ck = np.zeros((pairs.size, max(nc_cap, 0), P.head_dim), dtype=np.float64)
    rc = _load().bsa_oracle_compress_cache(ctypes.byref(P), _ptr(k_cache), _ptr(seq_lens),
                                           _ptr(pairs), pairs.size, _ptr(ck))
    if rc != 0:
        raise ValueError("bsa_oracle_compress_cache rejected its arguments")
    return ck
