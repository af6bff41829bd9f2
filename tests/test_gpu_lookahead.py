"""One-layer-lookahead decoding (bsa_decode_step_lookahead) vs the CPU oracle, through the C ABI.

Page "SparDA: Sparse Decoupled Attention for Efficient Long-Context LLM Inference", SparDA
Architecture, Eqs. 4-5: layer l attends the blocks chosen for it beforehand while layer l + 1's
blocks are chosen from layer l's Forecast vectors against layer l + 1's compressed keys, in one
kernel. The attention is checked against the oracle attending the same given blocks, the selection
against the oracle's Forecast selection (near-tie rule, raw-score tolerance) and, bit for bit,
against the separate bsa_select_blocks_forecast; a three-layer chain checks every layer.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_compressed_b200 as bsa
import oracle
from block_sparse_attention_compressed_b200.workloads import WORKLOADS
from gpu_helpers import (GpuCase, check_output, check_selection, oracle_problem, sample_pairs)

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["gqa4-bf16-32k-b1"].replace(layers=2)

CASES = {
    "g4-d128-ragged": (BASE.replace(name="x", batch=2, seq_len=4096 + 37, top_k=8, needles=4), None),
    "g8-d64": (BASE.replace(name="x", batch=2, num_q_heads=16, num_kv_heads=2, head_dim=64,
                            seq_len=3000, top_k=6, needles=3), None),
    "g1-d128": (BASE.replace(name="x", batch=1, num_q_heads=3, num_kv_heads=3, seq_len=1500, top_k=5,
                             needles=2), None),
    "g4-bs128-l64s32": (BASE.replace(name="x", batch=2, seq_len=7000 + 45, block_size=128, cmp_kernel=64,
                                     cmp_stride=32, top_k=6, needles=2), None),
    "g4-l16s16": (BASE.replace(name="x", batch=2, seq_len=6100, cmp_kernel=16, cmp_stride=16, top_k=9,
                               needles=3), None),
    "ragged": (BASE.replace(name="x", batch=5, seq_len=5000, top_k=9, needles=3), [5000, 64, 31, 0, 4097]),
    "more-pairs-than-sms": (BASE.replace(name="x", batch=40, seq_len=3000, top_k=6, needles=2), None),
    "no-init-no-local": (BASE.replace(name="x", batch=1, seq_len=648, n_init=0, n_local=0, top_k=4,
                                      needles=0), None),
    "k0": (BASE.replace(name="x", batch=1, seq_len=700, top_k=0, needles=0), None),
    "topk-covers-all": (BASE.replace(name="x", batch=1, seq_len=1000, top_k=1000, needles=0), None),
}


def _forecast(w, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(w.batch, w.num_kv_heads, w.head_dim, generator=g, device="cuda").to(w.torch_dtype)


class Lookahead:
    """A GpuCase with the next layer's selection buffers and the lookahead call."""

    def __init__(self, case):
        w, lens = CASES[case]
        self.w, self.run = w, GpuCase(w, seq_lens=lens)
        self.run.compress()
        s = self.run.sizes
        B, Hkv = w.batch, w.num_kv_heads
        self.idx1 = torch.full((B, Hkv, s.sel_cap), -7, dtype=torch.int32, device="cuda")
        self.ns1 = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
        self.bs1 = torch.zeros(B, Hkv, s.nb_cap, dtype=torch.float32, device="cuda")

    def call(self, layer, f, idx, ns, idx_next, ns_next, bs_next):
        r = self.run
        bsa.bsa_decode_step_lookahead(r.p, r.q[layer], r.data["k"][layer], r.data["v"][layer], idx, ns, f,
                                      r.ck[layer + 1], r.data["seq_lens"], idx_next, ns_next, bs_next,
                                      r.out[layer], r.lse[layer], r.ws)


def _oracle_attend(run, pairs, layer, idx, ns):
    """The oracle attending the given blocks of the listed pairs (layer `layer`)."""
    w = run.w
    G, Hkv = w.group, w.num_kv_heads
    seq = run.data["seq_lens"].cpu()
    qs, ks, vs, lens = [], [], [], []
    for pr in pairs:
        b, h = divmod(pr, Hkv)
        qs.append(run.q[layer][b, h * G:(h + 1) * G])
        ks.append(run.data["k"][layer][b, h:h + 1])
        vs.append(run.data["v"][layer][b, h:h + 1])
        lens.append(int(seq[b]))
    P = oracle_problem(w, len(pairs), run.T_cap)
    fi = idx.view(-1, run.sizes.sel_cap).cpu().numpy()[pairs]
    fn = ns.view(-1).cpu().numpy()[pairs]
    res = oracle.attend_pairs(P, oracle.raw(torch.stack(qs))[0], oracle.raw(torch.stack(ks))[0],
                              oracle.raw(torch.stack(vs))[0], lens, fi, fn)
    res["seq_lens"] = lens
    return res


def _oracle_select(run, pairs, layer, f):
    """The oracle's Forecast selection of layer `layer` for the listed pairs, and the raw-score
    tolerance of each (fp32 accumulation of d exact products: 1e-5 |f|_1 max|K|)."""
    w = run.w
    Hkv = w.num_kv_heads
    seq = run.data["seq_lens"].cpu()
    ks, fs, lens, atol = [], [], [], []
    for pr in pairs:
        b, h = divmod(pr, Hkv)
        ks.append(run.data["k"][layer][b, h:h + 1])
        fs.append(f[b, h:h + 1])
        lens.append(int(seq[b]))
        kmax = float(run.data["k"][layer][b, h, :lens[-1]].float().abs().max()) if lens[-1] else 0.0
        atol.append(1e-5 * float(f[b, h].float().abs().sum()) * kmax + 1e-30)
    P = oracle_problem(w, len(pairs), run.T_cap)
    ck = oracle.compress_cache(P, oracle.raw(torch.stack(ks))[0], lens)
    res = oracle.select_forecast(P, oracle.raw(torch.stack(fs))[0], ck, lens)
    res["seq_lens"] = lens
    return res, np.array(atol)


def _check_next(la, pairs, layer, f, idx, ns, bs):
    """The selection written for layer `layer` (into idx / ns / bs) vs the oracle."""
    run = la.run
    saved = (run.block_idx, run.n_sel, run.block_scores)
    run.block_idx, run.n_sel, run.block_scores = idx, ns, bs
    try:
        orc, atol = _oracle_select(run, pairs, layer, f)
        check_selection(run, pairs, orc, score_atol=atol)
    finally:
        run.block_idx, run.n_sel, run.block_scores = saved


@pytest.mark.parametrize("case", sorted(CASES))
def test_lookahead_matches_oracle(case, cuda_device):
    la = Lookahead(case)
    run, w = la.run, la.w
    run.select(0)  # layer 0's blocks (its own queries)
    idx0, ns0 = run.block_idx.clone(), run.n_sel.clone()
    f = _forecast(w, 5)
    la.call(0, f, idx0, ns0, la.idx1, la.ns1, la.bs1)
    assert run.device_errors() == 0
    pairs = sample_pairs(w, 40)
    check_output(run, pairs, _oracle_attend(run, pairs, 0, idx0, ns0), 0)
    _check_next(la, pairs, 1, f, la.idx1, la.ns1, la.bs1)
    # bit for bit the separate Forecast selection
    idx_s = torch.full_like(la.idx1, -7)
    ns_s = torch.full_like(la.ns1, -7)
    bs_s = torch.zeros_like(la.bs1)
    bsa.bsa_select_blocks_forecast(run.p, f, run.ck[1], run.data["seq_lens"], idx_s, ns_s, bs_s, run.ws)
    assert torch.equal(idx_s, la.idx1) and torch.equal(ns_s, la.ns1) and torch.equal(bs_s, la.bs1)


def test_lookahead_unsupported_geometry(cuda_device):
    """Blocks that are not four compression strides long have no fused kernel: refused."""
    w = BASE.replace(name="x", batch=1, seq_len=5000, block_size=128, top_k=7, needles=2)
    CASES["bs128-s16"] = (w, None)
    try:
        la = Lookahead("bs128-s16")
    finally:
        del CASES["bs128-s16"]
    run = la.run
    run.select(0)
    with pytest.raises(bsa.BsaError) as e:
        la.call(0, _forecast(w, 8), run.block_idx.clone(), run.n_sel.clone(), la.idx1, la.ns1, la.bs1)
    assert e.value.status == bsa.BSA_ERR_UNSUPPORTED


def test_lookahead_given_blocks_any_order_with_holes(cuda_device):
    """The given blocks may come in any order, with -1 holes and entries past the sequence's
    blocks (skipped); n_sel = 0 attends nothing (zero output, -inf LSE)."""
    la = Lookahead("ragged")
    run, w = la.run, la.w
    run.select(0)
    idx0, ns0 = run.block_idx.clone(), run.n_sel.clone()
    g = torch.Generator().manual_seed(3)
    flat, fns = idx0.view(-1, run.sizes.sel_cap), ns0.view(-1)
    for pr in range(flat.shape[0]):
        n = int(fns[pr])
        row = flat[pr, :n][torch.randperm(n, generator=g).to(flat.device)]
        flat[pr, :n] = row
        if n >= 3:
            flat[pr, 1] = -1
            flat[pr, 2] = 1 << 20
    fns[1] = 0
    f = _forecast(w, 6)
    la.call(0, f, idx0, ns0, la.idx1, la.ns1, la.bs1)
    assert run.device_errors() == 0
    pairs = list(range(w.batch * w.num_kv_heads))
    check_output(run, pairs, _oracle_attend(run, pairs, 0, idx0, ns0), 0)
    assert (run.out[0][0, w.group:2 * w.group] == 0).all() and torch.isneginf(run.lse[0][0, w.group:2 * w.group]).all()
    _check_next(la, pairs, 1, f, la.idx1, la.ns1, la.bs1)


def test_lookahead_three_layer_chain(cuda_device):
    """Layer 0's blocks from its own queries; layers 0 and 1 each choose the next layer's blocks
    while attending theirs; the last layer attends with bsa_sparse_decode. Every layer's output
    and every selection against the oracle."""
    w = BASE.replace(name="x", batch=3, seq_len=6000, top_k=8, needles=3, layers=3)
    CASES["chain"] = (w, None)
    try:
        la = Lookahead("chain")
    finally:
        del CASES["chain"]
    run = la.run
    run.select(0)
    idx = [run.block_idx.clone(), la.idx1, torch.full_like(la.idx1, -7)]
    ns = [run.n_sel.clone(), la.ns1, torch.full_like(la.ns1, -7)]
    bs = [None, la.bs1, torch.zeros_like(la.bs1)]
    fs = [_forecast(w, 10 + L) for L in range(2)]
    for L in range(2):
        la.call(L, fs[L], idx[L], ns[L], idx[L + 1], ns[L + 1], bs[L + 1])
    bsa.bsa_sparse_decode(run.p, run.q[2], run.data["k"][2], run.data["v"][2], run.data["seq_lens"], idx[2],
                          ns[2], run.out[2], run.lse[2], run.ws)
    assert run.device_errors() == 0
    pairs = list(range(w.batch * w.num_kv_heads))
    for L in range(3):
        check_output(run, pairs, _oracle_attend(run, pairs, L, idx[L], ns[L]), L)
    for L in range(1, 3):
        _check_next(la, pairs, L, fs[L - 1], idx[L], ns[L], bs[L])


def test_lookahead_graph_replay_and_overlap_check(cuda_device):
    """Replays of a captured lookahead step give the eager results bit for bit; overlapping input
    and output selections are refused."""
    la = Lookahead("more-pairs-than-sms")
    run, w = la.run, la.w
    run.select(0)
    idx0, ns0 = run.block_idx.clone(), run.n_sel.clone()
    f = _forecast(w, 7)
    la.call(0, f, idx0, ns0, la.idx1, la.ns1, la.bs1)
    torch.cuda.synchronize()
    ref = (la.idx1.clone(), la.bs1.clone(), run.out[0].clone(), run.lse[0].clone())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(3):
                bsa.bsa_decode_step_lookahead(run.p, run.q[0], run.data["k"][0], run.data["v"][0], idx0, ns0, f,
                                              run.ck[1], run.data["seq_lens"], la.idx1, la.ns1, la.bs1,
                                              run.out[0], run.lse[0], run.ws, stream=s)
    for _ in range(4):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ref[0], la.idx1) and torch.equal(ref[1], la.bs1)
    assert torch.equal(ref[2], run.out[0]) and torch.equal(ref[3], run.lse[0])
    with pytest.raises(bsa.BsaError):
        bsa.bsa_decode_step_lookahead(run.p, run.q[0], run.data["k"][0], run.data["v"][0], idx0, ns0, f,
                                      run.ck[1], run.data["seq_lens"], idx0, la.ns1, None, run.out[0],
                                      run.lse[0], run.ws)


@pytest.mark.slow
def test_full_lookahead_workload(cuda_device):
    """The bench's lookahead workload (128K tokens x 16 sequences, two layers) on sampled pairs."""
    w = WORKLOADS["lookahead-bf16-128k-b16"]
    CASES["full"] = (w, None)
    try:
        la = Lookahead("full")
    finally:
        del CASES["full"]
    run = la.run
    run.select(0)
    idx0, ns0 = run.block_idx.clone(), run.n_sel.clone()
    f = run.data["f"]
    la.call(0, f, idx0, ns0, la.idx1, la.ns1, la.bs1)
    assert run.device_errors() == 0
    pairs = sample_pairs(w, 12, seed=5)
    check_output(run, pairs, _oracle_attend(run, pairs, 0, idx0, ns0), 0)
    _check_next(la, pairs, 1, f, la.idx1, la.ns1, la.bs1)
