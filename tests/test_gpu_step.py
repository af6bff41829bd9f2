"""The fused decode step (bsa_decode_step_fused), vs the CPU oracle, through the C ABI.

For bf16 caches whose blocks are four windows long (BS = 4s, l = s or 2s, BS a multiple of 64; the
paper's 64 / 16 / 32), bsa_decode_step_fused runs one kernel in which a CTA takes a whole
(batch, kv-head) pair: it scores the pair's compressed keys (window terms kept in tensor memory),
selects its blocks and attends them. bsa_decode_step takes that path when there are enough pairs to
keep most SMs streaming, else it chains the separate kernels. These cases cover every padded group
size, both head dims, both window lengths, blocks of 64 and 128 tokens, ragged lengths (down to no
window and an empty sequence), last blocks cut inside either 32-token half, more pairs than SMs
(the persistent loop over pairs) and the selection edge cases (top-k covering every candidate,
k = 0, no init or local blocks); geometries the fused kernel does not take run through
bsa_decode_step's chained path.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_compressed_b200 as bsa
from block_sparse_attention_compressed_b200.workloads import WORKLOADS
from gpu_helpers import GpuCase, full_check, sample_pairs

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["gqa4-bf16-32k-b1"]

STEP = {
    "g4-d128-ragged": (BASE.replace(name="x", batch=2, seq_len=4096 + 37, top_k=8, needles=4), None),
    "g8-d64": (BASE.replace(name="x", batch=2, num_q_heads=16, num_kv_heads=2, head_dim=64,
                            seq_len=3000, top_k=6, needles=3), None),
    "g1-d128": (BASE.replace(name="x", batch=1, num_q_heads=3, num_kv_heads=3, seq_len=1500, top_k=5,
                             needles=2), None),
    "g2-d64-bs32-l16s8": (BASE.replace(name="x", batch=1, num_q_heads=4, num_kv_heads=2, head_dim=64,
                                       seq_len=2000, block_size=32, cmp_kernel=16, cmp_stride=8,
                                       top_k=10, needles=3), None),
    "g4-bs128": (BASE.replace(name="x", batch=1, seq_len=5000, block_size=128, top_k=7, needles=2),
                 None),
    "g4-bs128-l64s32": (BASE.replace(name="x", batch=2, seq_len=7000 + 45, block_size=128,
                                     cmp_kernel=64, cmp_stride=32, top_k=6, needles=2), None),
    "g4-bs256-l32s16": (BASE.replace(name="x", batch=2, seq_len=9000, block_size=256, top_k=5,
                                     needles=2), None),
    "g4-l16s16": (BASE.replace(name="x", batch=2, seq_len=6100, cmp_kernel=16, cmp_stride=16,
                               top_k=9, needles=3), None),
    "g3-padded-heads": (BASE.replace(name="x", batch=2, num_q_heads=12, num_kv_heads=4, seq_len=3333,
                                     top_k=7, needles=2), None),
    "last-block-10-tokens": (BASE.replace(name="x", batch=1, seq_len=64 * 40 + 10, top_k=6,
                                          needles=2), None),
    "last-block-50-tokens": (BASE.replace(name="x", batch=1, seq_len=64 * 40 + 50, top_k=6,
                                          needles=2), None),
    "ragged": (BASE.replace(name="x", batch=5, seq_len=5000, top_k=9, needles=3),
               [5000, 64, 31, 0, 4097]),
    "more-pairs-than-sms": (BASE.replace(name="x", batch=40, seq_len=3000, top_k=6, needles=2), None),
    "topk-covers-all": (BASE.replace(name="x", batch=1, seq_len=1000, top_k=1000, needles=0), None),
    "no-init-no-local": (BASE.replace(name="x", batch=1, seq_len=648, n_init=0, n_local=0, top_k=4,
                                      needles=0), None),
    "no-local-partial-last": (BASE.replace(name="x", batch=2, seq_len=64 * 30 + 20, n_local=0,
                                           top_k=6, needles=2), None),
    "k0": (BASE.replace(name="x", batch=1, seq_len=700, top_k=0, needles=0), None),
    "short": (BASE.replace(name="x", batch=1, seq_len=20, top_k=3, needles=0), None),
}


def _run(case):
    w, lens = STEP[case]
    run = GpuCase(w, seq_lens=lens)
    if lens is not None:
        # rows past each sequence's length hold other data here; they must never be read
        run.data["k"][0].view(-1)[:] = run.data["k"][0].view(-1).flip(0)
    run.compress()
    return w, run


def _fused_ok(w) -> bool:
    """The fused kernel's geometry (bf16, BS = 4s, l = s or 2s, BS a multiple of 64, a cache of at
    least one window)."""
    return (w.dtype == "bf16" and w.block_size == 4 * w.cmp_stride and w.block_size % 64 == 0
            and w.cmp_kernel in (w.cmp_stride, 2 * w.cmp_stride) and w.seq_len >= w.cmp_kernel)


@pytest.mark.parametrize("case", sorted(STEP))
def test_step_matches_oracle(case, cuda_device):
    w, run = _run(case)
    assert bsa.bsa_get_sizes(run.p).workspace_bytes > 0
    run.step(fused=_fused_ok(w))
    assert run.device_errors() == 0
    full_check(run, sample_pairs(w, 48))


@pytest.mark.parametrize("case", ["g4-d128-ragged", "g8-d64", "g2-d64-bs32-l16s8", "ragged",
                                  "more-pairs-than-sms", "no-local-partial-last", "g4-l16s16",
                                  "g4-bs128-l64s32", "g3-padded-heads"])
def test_step_selection_equals_separate_selection(case, cuda_device):
    """The step's block scores and selection are those of bsa_select_blocks, bit for bit: both
    weigh the same stored window terms by the same per-chunk softmax weights."""
    w, run = _run(case)
    run.step(fused=_fused_ok(w))
    got = (run.block_idx.clone(), run.n_sel.clone(), run.block_scores.clone())
    run.select()
    assert torch.equal(got[0], run.block_idx)
    assert torch.equal(got[1], run.n_sel)
    assert torch.equal(got[2], run.block_scores)


def test_step_empty_sequence_outputs(cuda_device):
    """A sequence of length 0 selects nothing and attends nothing: zero output, -inf LSE."""
    w, run = _run("ragged")
    run.step(fused=True)
    Hkv = w.num_kv_heads
    assert (run.n_sel.view(-1)[3 * Hkv:4 * Hkv] == 0).all()
    assert (run.block_idx[3] == -1).all()
    assert (run.out[0][3] == 0).all() and torch.isneginf(run.lse[0][3]).all()


def test_step_repeats_bit_for_bit(cuda_device):
    """Queued steps without a host sync give the first step's results bit for bit."""
    w, run = _run("more-pairs-than-sms")
    run.step(fused=True)
    torch.cuda.synchronize()
    first = (run.block_idx.clone(), run.out[0].clone(), run.lse[0].clone())
    for _ in range(30):
        run.step(fused=True)
    torch.cuda.synchronize()
    assert run.device_errors() == 0
    for a, b in zip(first, (run.block_idx, run.out[0], run.lse[0])):
        assert torch.equal(a, b)


def test_step_path_choice_and_unsupported_geometry(cuda_device):
    """bsa_decode_step takes the fused kernel only with enough pairs to fill most SMs; the fused
    entry point refuses a geometry it does not handle (blocks of eight strides) on the host."""
    small, _ = STEP["g4-d128-ragged"]
    big, _ = STEP["more-pairs-than-sms"]
    for w, want in ((small, False), (big, True)):
        p = bsa.make_params(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.seq_len, w.dtype,
                            w.n_init, w.n_local, w.top_k, w.cmp_kernel, w.cmp_stride, w.block_size)
        assert bsa.bsa_decode_step_info(p)[0] is want
    w, run = _run("g4-bs128")
    with pytest.raises(bsa.BsaError) as e:
        run.step(fused=True)
    assert e.value.status == bsa.BSA_ERR_UNSUPPORTED


def test_fused_step_graph_replay(cuda_device):
    """The fused step captured in a CUDA graph (its launch attributes included) and replayed gives
    the eager call's results bit for bit."""
    w, run = _run("more-pairs-than-sms")
    run.step(fused=True)
    torch.cuda.synchronize()
    ref = (run.block_idx.clone(), run.out[0].clone(), run.lse[0].clone())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            bsa.bsa_decode_step(run.p, run.q[0], run.data["k"][0], run.data["v"][0], run.ck[0],
                                None, None, run.data["seq_lens"], run.block_idx, run.n_sel, None,
                                run.out[0], run.lse[0], run.ws, stream=s, fused=True)
    torch.cuda.current_stream().wait_stream(s)
    run.out[0].fill_(0)
    run.block_idx.fill_(-5)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert run.device_errors() == 0
    for a, b in zip(ref, (run.block_idx, run.out[0], run.lse[0])):
        assert torch.equal(a, b)
