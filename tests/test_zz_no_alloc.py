"""bsa_sparse_decode_noalloc: the sparse attention for callers that cannot allocate device memory.
Its split partials live in a fixed scratch array inside libbsa instead of a caller workspace; it
must give the results of bsa_sparse_decode, call after call. This file is collected last, so the
entry point is exercised both after every other test and (run alone) in a fresh process."""
import ctypes

import pytest
import torch

import block_sparse_attention_compressed_b200 as bsa
from block_sparse_attention_compressed_b200.workloads import WORKLOADS
from gpu_helpers import LSE_ATOL, OUT_ATOL, GpuCase

CASES = {
    "gqa4-bf16-128k-b16": WORKLOADS["gqa4-bf16-128k-b16"],
    "bf16-g4-d128-ragged": WORKLOADS["gqa4-bf16-32k-b1"].replace(
        name="x", batch=2, seq_len=4096 + 37, top_k=8, needles=4),
    "tiny-f32-2k": WORKLOADS["tiny-f32-2k"],
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_decode(name, cuda_device):
    w = CASES[name]
    run = GpuCase(w)
    run.compress()
    run.select()
    run.decode()  # the workspace entry point
    torch.cuda.synchronize()
    assert run.device_errors() == 0
    ref_out, ref_lse = run.out[0].clone(), run.lse[0].clone()
    d = run.data
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    outs = [torch.full_like(ref_out, 77.0) for _ in range(2)]
    lses = [torch.full_like(ref_lse, 77.0) for _ in range(2)]
    # two calls in a row on the stream, no host sync between them; the second reports no errors.
    # The second call's parameters name four layers: the call attends one, and its scratch is
    # sized for one (at 128K x 16, four layers' partials would not fit the scratch).
    p4 = bsa.make_params(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, run.T_cap, w.dtype,
                         w.n_init, w.n_local, w.top_k, w.cmp_kernel, w.cmp_stride, w.block_size,
                         num_layers=4)
    for i in range(2):
        bsa.bsa_sparse_decode_noalloc(run.p if i == 0 else p4, run.q[0], d["k"][0], d["v"][0],
                                      d["seq_lens"], run.block_idx, run.n_sel, outs[i], lses[i],
                                      device_error=err if i == 0 else None)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for out, lse in zip(outs, lses):
        torch.testing.assert_close(out.float(), ref_out.float(), atol=OUT_ATOL[w.dtype], rtol=0)
        torch.testing.assert_close(lse, ref_lse, atol=LSE_ATOL[w.dtype], rtol=0)
    del run
    torch.cuda.empty_cache()


def test_noalloc_rejects_problems_beyond_its_scratch():
    """A parameter set whose partials exceed the fixed scratch is refused on the host, before any
    CUDA call (fake, never-dereferenced device addresses)."""
    bsa.lib()
    w = WORKLOADS["append-bf16-16k-b128"]  # 1024 (batch, kv-head) pairs: > 4 MiB of partials
    p = bsa.make_params(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.seq_len + 64,
                        w.dtype, w.n_init, w.n_local, w.top_k)
    A = ctypes.c_void_p(0x10000)
    st = bsa.lib().bsa_sparse_decode_noalloc(ctypes.byref(p), A, A, A, A, A, A, A, None, None,
                                             ctypes.c_void_p(0))
    assert st == bsa.BSA_ERR_WORKSPACE
    # misaligned arguments are refused as usual
    st = bsa.lib().bsa_sparse_decode_noalloc(ctypes.byref(p), ctypes.c_void_p(0x10002), A, A, A,
                                             A, A, A, None, None, ctypes.c_void_p(0))
    assert st == bsa.BSA_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="host-side check with fake device addresses")
def test_noalloc_scratch_is_sized_for_one_layer():
    """The call attends one layer: a parameter set naming more layers is not refused for the size
    of partials it will never write. (On a machine without a GPU the call then stops at its first
    CUDA call, which is all this host-side check needs.)"""
    bsa.lib()
    w = WORKLOADS["gqa4-bf16-128k-b16"]  # 1.3 MiB of partials for one layer, 5.3 MiB for four
    A = ctypes.c_void_p(0x10000)
    for layers in (1, 4, 16):
        p = bsa.make_params(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.seq_len, w.dtype,
                            w.n_init, w.n_local, w.top_k, num_layers=layers)
        st = bsa.lib().bsa_sparse_decode_noalloc(ctypes.byref(p), A, A, A, A, A, A, A, None, None,
                                                 ctypes.c_void_p(0))
        assert st not in (bsa.BSA_OK, bsa.BSA_ERR_WORKSPACE), (layers, st)
