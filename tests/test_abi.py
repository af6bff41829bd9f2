"""The C-ABI library loads, exports every function include/bsa.h declares, and validates its
arguments on the host. No test here makes a CUDA call: every call below is rejected (or is a pure
host query) before the library touches the GPU."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_compressed_b200 as bsa
from block_sparse_attention_compressed_b200 import build as bsa_build
from block_sparse_attention_compressed_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


@pytest.fixture(scope="module")
def lib():
    bsa_build.build()
    return bsa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["bsa_compress_keys", "bsa_compress_append", "bsa_select_blocks",
                 "bsa_sparse_decode", "bsa_sparse_decode_layers", "bsa_decode_step",
                 "bsa_workspace_size", "bsa_workspace_init", "bsa_read_device_error",
                 "bsa_status_string", "bsa_check_params", "bsa_get_sizes", "bsa_abi_version"]:
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_status_strings(lib):
    assert bsa.bsa_abi_version() == 1
    for code, name in [(0, "BSA_OK"), (1, "BSA_ERR_INVALID_ARG"), (2, "BSA_ERR_UNSUPPORTED"),
                       (3, "BSA_ERR_WORKSPACE"), (4, "BSA_ERR_CUDA"), (5, "BSA_ERR_DEVICE_CHECK")]:
        assert bsa.status_string(code) == name
    assert bsa.status_string(99) == "BSA_ERR_UNKNOWN"


def test_params_struct_layout_matches_header(lib):
    # 10 int32, one int64 (8-aligned at offset 40), 2 int32, 2 float
    assert ctypes.sizeof(bsa.Params) == 64
    assert bsa.Params.max_seq_len.offset == 40


def _p(**kw):
    base = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, max_seq_len=4096,
                dtype="bf16", n_init=1, n_local=2, top_k=8)
    base.update(kw)
    return bsa.make_params(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(num_q_heads=7), bsa.BSA_ERR_INVALID_ARG),
    (dict(num_q_heads=32, num_kv_heads=2), bsa.BSA_ERR_UNSUPPORTED),   # G = 16
    (dict(head_dim=96), bsa.BSA_ERR_UNSUPPORTED),
    (dict(block_size=40), bsa.BSA_ERR_UNSUPPORTED),
    (dict(block_size=512), bsa.BSA_ERR_UNSUPPORTED),
    (dict(cmp_kernel=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(cmp_stride=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(n_init=0, n_local=0, top_k=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(top_k=-1), bsa.BSA_ERR_INVALID_ARG),
    (dict(top_k=5000), bsa.BSA_ERR_UNSUPPORTED),                       # SEL_cap > 4096
    (dict(max_seq_len=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(max_seq_len=64 * 32768 + 1), bsa.BSA_ERR_UNSUPPORTED),       # nb_cap > 32768
    (dict(num_layers=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(num_layers=17), bsa.BSA_ERR_UNSUPPORTED),
    (dict(scale=-1.0), bsa.BSA_ERR_INVALID_ARG),
    (dict(score_tau=float("inf")), bsa.BSA_ERR_INVALID_ARG),
])
def test_invalid_params_rejected(lib, kw, status):
    p = _p(**kw)
    assert bsa.bsa_check_params(p) == status
    assert bsa.bsa_workspace_size(p) == 0


@pytest.mark.parametrize("batch,kv_heads,T", [(64, 8, 1 << 20), (16, 8, 1 << 21), (1, 1, 1 << 21)])
def test_long_contexts_supported_at_any_pair_count(lib, batch, kv_heads, T):
    # up to NB_cap = 32768 blocks, whatever the number of (batch, kv-head) pairs
    p = _p(batch=batch, num_q_heads=4 * kv_heads, num_kv_heads=kv_heads, max_seq_len=T, top_k=64)
    assert bsa.bsa_check_params(p) == bsa.BSA_OK
    assert bsa.bsa_workspace_size(p) > 0


def test_cache_rows_beyond_tma_coordinates_rejected(lib):
    # B * Hkv * T_cap cache rows must stay below 2^31 (32-bit TMA row coordinates)
    p = _p(batch=128, num_q_heads=32, num_kv_heads=8, max_seq_len=1 << 21, top_k=64)
    assert bsa.bsa_check_params(p) == bsa.BSA_ERR_UNSUPPORTED


def test_unsupported_dtype(lib):
    p = _p()
    p.dtype = 7
    assert bsa.bsa_check_params(p) == bsa.BSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_sizes_of_workloads(lib, name):
    w = WORKLOADS[name]
    cap = w.seq_len + w.append_steps
    p = bsa.make_params(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, cap, w.dtype,
                        w.n_init, w.n_local, w.top_k, num_layers=w.layers)
    assert bsa.bsa_check_params(p) == bsa.BSA_OK
    s = bsa.bsa_get_sizes(p)
    assert s.nc_cap == (cap - 32) // 16 + 1
    assert s.nb_cap == -(-cap // 64)
    assert s.sel_cap == w.n_init + w.n_local + w.top_k
    assert s.group == w.group
    ws = bsa.bsa_workspace_size(p)
    assert ws == s.workspace_bytes and ws % 256 == 0
    # the fp32 window logits alone: pairs * nc_cap * G floats
    assert ws >= w.batch * w.num_kv_heads * s.nc_cap * w.group * 4


# Fake, never-dereferenced device addresses: every call below fails validation first.
A = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10002)          # not 16-byte aligned
S0 = ctypes.c_void_p(0)                 # default stream handle


def test_entry_points_reject_bad_arguments_before_launch(lib):
    p = _p()
    P = ctypes.byref(p)
    ws_need = bsa.bsa_workspace_size(p)
    N = None
    # null / misaligned pointers
    assert lib.bsa_select_blocks(P, N, A, A, A, A, N, A, ws_need, S0) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_select_blocks(P, MIS, A, A, A, A, N, A, ws_need, S0) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_sparse_decode(P, A, A, A, A, A, A, N, N, A, ws_need, S0) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_compress_keys(P, N, A, A, S0) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_compress_append(P, A, A, A, N, A, A, N, 0, S0) == bsa.BSA_ERR_INVALID_ARG
    # workspace too small / missing / misaligned
    assert lib.bsa_select_blocks(P, A, A, A, A, A, N, A, ws_need - 1, S0) == bsa.BSA_ERR_WORKSPACE
    assert lib.bsa_select_blocks(P, A, A, A, A, A, N, N, ws_need, S0) == bsa.BSA_ERR_WORKSPACE
    assert lib.bsa_sparse_decode(P, A, A, A, A, A, A, A, N, ctypes.c_void_p(0x10010), ws_need,
                                 S0) == bsa.BSA_ERR_WORKSPACE
    assert lib.bsa_workspace_init(P, A, ws_need - 256, S0) == bsa.BSA_ERR_WORKSPACE
    # k_new without v_new
    assert lib.bsa_decode_step(P, A, A, A, A, A, N, A, A, A, N, A, N, A, ws_need,
                               S0) == bsa.BSA_ERR_INVALID_ARG
    # more layers than the workspace was sized for
    arr = (ctypes.c_void_p * 2)(A, A)
    assert lib.bsa_sparse_decode_layers(P, 2, arr, arr, arr, A, A, A, arr, N, A, ws_need,
                                        S0) == bsa.BSA_ERR_INVALID_ARG
    # invalid parameters are reported as such by every entry point
    bad = _p(head_dim=96)
    assert lib.bsa_select_blocks(ctypes.byref(bad), A, A, A, A, A, N, A, 1 << 30,
                                 S0) == bsa.BSA_ERR_UNSUPPORTED
    flags = ctypes.c_uint32(0)
    assert lib.bsa_read_device_error(N, 0, ctypes.byref(flags), S0) == bsa.BSA_ERR_WORKSPACE
    assert lib.bsa_read_device_error(A, 4, None, S0) == bsa.BSA_ERR_INVALID_ARG


def test_anchored_schedule_validated_before_launch(lib):
    """bsa_decode_step_anchored: the anchor list must start at layer 0, ascend and stay below
    num_layers; the Forecast selection validates like bsa_select_blocks."""
    p = _p(num_layers=4)
    P = ctypes.byref(p)
    ws_need = bsa.bsa_workspace_size(p)
    N = None
    arr = (ctypes.c_void_p * 4)(A, A, A, A)

    def run(anchors, layers=4, ws=ws_need):
        a = (ctypes.c_int32 * len(anchors))(*anchors)
        return lib.bsa_decode_step_anchored(P, layers, a, len(anchors), arr, arr, arr, arr, A, A, A,
                                            arr, N, A, ws, S0)
    for bad in ([1], [0, 0], [0, 3, 2], [0, 4], [0, 1, 2, 3, 3]):
        assert run(bad) == bsa.BSA_ERR_INVALID_ARG, bad
    assert run([0, 2], layers=5) == bsa.BSA_ERR_INVALID_ARG       # more layers than planned
    assert run([0, 2], ws=ws_need - 1) == bsa.BSA_ERR_WORKSPACE
    assert lib.bsa_decode_step_anchored(P, 4, N, 1, arr, arr, arr, arr, A, A, A, arr, N, A,
                                        ws_need, S0) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_select_blocks_forecast(P, N, A, A, A, A, N, A, ws_need, S0) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_select_blocks_forecast(P, MIS, A, A, A, A, N, A, ws_need, S0) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_select_blocks_forecast(P, A, A, A, A, A, N, A, ws_need - 1,
                                          S0) == bsa.BSA_ERR_WORKSPACE


def test_binding_rejects_host_tensors(lib):
    import torch
    p = _p()
    with pytest.raises(ValueError):
        bsa.bsa_compress_keys(p, torch.zeros(4), torch.zeros(2, dtype=torch.int32), torch.zeros(4))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from block_sparse_attention_compressed_b200 import _abi
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "libbsa.so"))
    with pytest.raises(RuntimeError, match="libbsa.so not found"):
        _abi.lib()
