"""CUDA path vs the CPU oracle, element by element, through the C ABI (via the ctypes binding).

Small cases span several tiles and ragged tails; the full-size workloads run in the launch
configuration the benchmark times and are checked on sampled (batch, kv-head) pairs.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_compressed_b200 as bsa
import oracle
from block_sparse_attention_compressed_b200.workloads import WORKLOADS, Workload
from gpu_helpers import (GpuCase, check_output, check_selection, forecast_check, full_check,
                         near_tie, oracle_on_pairs, sample_pairs)

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["gqa4-bf16-32k-b1"]

SMALL = {
    "tiny-f32-2k": WORKLOADS["tiny-f32-2k"],
    "bf16-g4-d128-ragged": BASE.replace(name="x", batch=2, seq_len=4096 + 37, top_k=8, needles=4),
    "bf16-g8-d64": BASE.replace(name="x", batch=2, num_q_heads=16, num_kv_heads=2, head_dim=64,
                                seq_len=3000, top_k=6, needles=3),
    "bf16-g1-d128": BASE.replace(name="x", batch=1, num_q_heads=3, num_kv_heads=3, seq_len=1500,
                                 top_k=5, needles=2),
    "bf16-g2-d64-bs32-l16s8": BASE.replace(name="x", batch=1, num_q_heads=4, num_kv_heads=2,
                                           head_dim=64, seq_len=2000, block_size=32, cmp_kernel=16,
                                           cmp_stride=8, top_k=10, needles=3),
    "bf16-g4-bs128": BASE.replace(name="x", batch=1, seq_len=5000, block_size=128, top_k=7,
                                  needles=2),
    "f32-g4-d128": BASE.replace(name="x", dtype="f32", batch=1, seq_len=2500, top_k=6, needles=2),
    "f32-g2-d64-bs128": BASE.replace(name="x", dtype="f32", batch=2, num_q_heads=4, num_kv_heads=2,
                                     head_dim=64, seq_len=1800, block_size=128, top_k=3, needles=1),
    "bf16-topk-covers-all": BASE.replace(name="x", batch=1, seq_len=1000, top_k=1000, needles=0),
    "bf16-no-init-no-local": BASE.replace(name="x", batch=1, seq_len=648, n_init=0, n_local=0,
                                          top_k=4, needles=0),
    "bf16-k0": BASE.replace(name="x", batch=1, seq_len=700, top_k=0, needles=0),
    "bf16-short": BASE.replace(name="x", batch=1, seq_len=20, top_k=3, needles=0),
}


@pytest.mark.parametrize("case", sorted(SMALL))
def test_small_select_and_decode(case, cuda_device):
    w = SMALL[case]
    run = GpuCase(w)
    run.compress()
    run.select()
    run.decode()
    assert run.device_errors() == 0
    full_check(run, sample_pairs(w, 64))


@pytest.mark.parametrize("case", ["tiny-f32-2k", "bf16-g4-d128-ragged", "bf16-g8-d64", "f32-g4-d128",
                                  "bf16-g2-d64-bs32-l16s8"])
def test_compress_bit_exact(case, cuda_device):
    w = SMALL[case]
    run = GpuCase(w)
    run.compress()
    P = oracle.make_problem(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, run.T_cap,
                            oracle.F32 if w.dtype == "f32" else oracle.BF16, w.n_init, w.n_local,
                            w.top_k, w.cmp_kernel, w.cmp_stride, w.block_size)
    kr, _ = oracle.raw(run.data["k"][0])
    want = oracle.compress_cache(P, kr, run.data["seq_lens"].cpu().numpy())
    got = run.ck[0].float().cpu().numpy().astype(np.float64).reshape(want.shape)
    assert np.array_equal(got, want)


def test_ragged_batch_lengths(cuda_device):
    """Sequences of different lengths in one batch, down to no window (T < l) and empty (T = 0)."""
    w = BASE.replace(name="x", batch=5, seq_len=5000, top_k=9, needles=3)
    run = GpuCase(w, seq_lens=[5000, 64, 31, 0, 4097])
    # rows past each sequence's length hold random data here; the kernels must never read them
    run.data["k"][0].view(-1)[:] = run.data["k"][0].view(-1).flip(0)
    run.compress()
    run.select()
    run.decode()
    assert run.device_errors() == 0
    pairs = list(range(w.batch * w.num_kv_heads))
    full_check(run, pairs)
    # the empty sequence: no block, zero output, -inf lse
    e = 3 * w.num_kv_heads
    assert (run.n_sel.view(-1)[e:e + w.num_kv_heads] == 0).all()
    assert (run.out[0][3] == 0).all() and torch.isneginf(run.lse[0][3]).all()


def test_equal_scores_take_lowest_blocks(cuda_device):
    """q = 0: every window has the same score, so every candidate block ties and the lowest
    candidate blocks are taken."""
    w = BASE.replace(name="x", batch=1, num_q_heads=4, num_kv_heads=1, seq_len=5000, top_k=8,
                     needles=0)
    run = GpuCase(w)
    run.data["q"][0].zero_()
    run.compress()
    run.select()
    run.decode()
    assert run.device_errors() == 0
    nb = -(-5000 // w.block_size)
    init_end, chi = w.n_init, nb - w.n_local
    want = list(range(init_end)) + list(range(init_end, init_end + w.top_k)) + list(range(chi, nb))
    assert run.n_sel[0, 0].item() == len(want)
    assert run.block_idx[0, 0, :len(want)].tolist() == want
    full_check(run, [0])


@pytest.mark.parametrize("seq_len", [20000, 40000])
def test_periodic_keys_many_ties(seq_len, cuda_device):
    """Keys that repeat every 256 tokens give block scores that repeat every four blocks: the k-th
    largest sits in a group of equal scores (about 80 or 160 of them), ranked by block index."""
    w = BASE.replace(name="x", batch=1, num_q_heads=8, num_kv_heads=2, seq_len=seq_len, top_k=50,
                     needles=0)
    run = GpuCase(w)
    k = run.data["k"][0]
    period = 256
    reps = -(-seq_len // period)
    tiled = k[:, :, :period].repeat(1, 1, reps, 1)[:, :, :seq_len]
    k[:, :, :seq_len] = tiled
    run.compress()
    run.select()
    run.decode()
    assert run.device_errors() == 0
    full_check(run, [0, 1])


def test_long_context_large_block_count(cuda_device):
    """nb_cap = 16384 blocks: the selection keeps 64 KB of keys in shared memory."""
    w = BASE.replace(name="x", batch=1, num_q_heads=4, num_kv_heads=1, seq_len=300000, top_k=40,
                     needles=10)
    run = GpuCase(w, T_cap=1 << 20)
    run.compress()
    run.select()
    run.decode()
    assert run.device_errors() == 0
    full_check(run, [0])


@pytest.mark.parametrize("q_heads,kv_heads,d", [(16, 2, 64), (16, 8, 128), (8, 8, 64)])
def test_one_cta_per_pair_selection_every_group_size(q_heads, kv_heads, d, cuda_device):
    """Enough pairs (>= 75) for one selection CTA per pair, with groups of 8, 2 and 1 query heads:
    the shared-memory ring, the shuffle block maxima and the top-k of select_single_kernel for
    every padded group size."""
    B = -(-80 // kv_heads)
    w = BASE.replace(name="x", batch=B, num_q_heads=q_heads, num_kv_heads=kv_heads, head_dim=d,
                     seq_len=3000 + 11, top_k=9, needles=3)
    run = GpuCase(w)
    run.compress()
    run.select()
    run.decode()
    assert run.device_errors() == 0
    full_check(run, sample_pairs(w, 24))


@pytest.mark.slow
def test_select_streams_rows_longer_than_the_ring(cuda_device):
    """80 pairs get one selection CTA each; at T = 150000 a pair's 9374 windows of window terms
    (150 KB) exceed the 128 KB shared-memory ring, so the stages are refilled as they are read."""
    w = BASE.replace(name="x", batch=10, seq_len=150000, top_k=16, needles=4)
    run = GpuCase(w)
    run.compress()
    run.select()
    run.decode()
    assert run.device_errors() == 0
    full_check(run, sample_pairs(w, 4, seed=4))
    del run
    torch.cuda.empty_cache()


def test_decode_with_given_indices_any_order(cuda_device):
    """Eq. 5 only depends on the set of blocks: shuffled indices and -1 holes give the same
    output as the oracle on the same set."""
    w = SMALL["bf16-g4-d128-ragged"]
    run = GpuCase(w)
    run.compress()
    run.select()
    pairs = list(range(w.batch * w.num_kv_heads))
    orc = oracle_on_pairs(run, pairs)
    idx = run.block_idx.clone().view(-1, run.sizes.sel_cap)
    ns = run.n_sel.clone().view(-1)
    g = torch.Generator().manual_seed(3)
    for i in range(idx.shape[0]):
        n = int(ns[i])
        perm = torch.randperm(n, generator=g)
        row = idx[i, :n][perm.to(idx.device)].clone()
        idx[i, :n] = row
    run.decode(0, idx.view_as(run.block_idx), ns.view_as(run.n_sel))
    check_output(run, pairs, orc)


def test_deterministic(cuda_device):
    w = SMALL["bf16-g4-d128-ragged"]
    run = GpuCase(w)
    run.compress()
    outs = []
    for _ in range(2):
        run.select()
        run.decode()
        outs.append((run.block_idx.clone(), run.block_scores.clone(), run.out[0].clone(),
                     run.lse[0].clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_decode_step_entry_point(cuda_device):
    """bsa_decode_step selects exactly what bsa_select_blocks selects (the same block scores, bit
    for bit) and its output matches the oracle. (For bf16 it runs one CTA per pair, attending all of
    a pair's blocks in one softmax pass: its output rounds differently from the split partials of
    bsa_sparse_decode, so outputs are checked against the oracle's tolerance, not bit for bit.)"""
    w = SMALL["bf16-g4-d128-ragged"]
    run = GpuCase(w)
    run.compress()
    run.select()
    ref = (run.block_idx.clone(), run.n_sel.clone(), run.block_scores.clone())
    run.out[0].fill_(5)
    run.block_idx.fill_(-3)
    run.block_scores.fill_(3)
    run.step()
    assert run.device_errors() == 0
    assert torch.equal(ref[0], run.block_idx)
    assert torch.equal(ref[1], run.n_sel)
    assert torch.equal(ref[2], run.block_scores)
    full_check(run, sample_pairs(w, 64))


def test_cuda_graph_replay(cuda_device):
    """The step can be captured in a CUDA graph (launch attributes included) and replayed."""
    w = SMALL["bf16-g4-d128-ragged"]
    run = GpuCase(w)
    run.compress()
    run.step()
    ref = run.out[0].clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            bsa.bsa_decode_step(run.p, run.q[0], run.data["k"][0], run.data["v"][0], run.ck[0],
                                None, None, run.data["seq_lens"], run.block_idx, run.n_sel, None,
                                run.out[0], run.lse[0], run.ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    run.out[0].fill_(0)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(ref, run.out[0])


# --------------------------------------------------------------------------- growing cache (append)
def test_append_matches_full_compression(cuda_device):
    """Appending tokens one by one (new windows completed on the fly) gives the same compressed keys
    as compressing the final cache, bit for bit, and as the oracle."""
    w = BASE.replace(name="x", batch=3, seq_len=100, top_k=2, needles=0)
    run = GpuCase(w, T_cap=200, steps=0)
    run.data["seq_lens"] = torch.tensor([100, 31, 47], dtype=torch.int32, device="cuda")
    run.compress()
    g = torch.Generator(device="cuda").manual_seed(9)
    for step in range(60):
        kn = torch.randn(w.batch, w.num_kv_heads, w.head_dim, generator=g, device="cuda").to(w.torch_dtype)
        vn = torch.randn(w.batch, w.num_kv_heads, w.head_dim, generator=g, device="cuda").to(w.torch_dtype)
        bsa.bsa_compress_append(run.p, run.data["k"][0], run.data["v"][0], kn, vn,
                                run.data["seq_lens"], run.ck[0], run.ws)
    assert run.data["seq_lens"].tolist() == [160, 91, 107]
    assert run.device_errors() == 0
    fresh = torch.zeros_like(run.ck[0])
    bsa.bsa_compress_keys(run.p, run.data["k"][0], run.data["seq_lens"], fresh)
    assert torch.equal(fresh, run.ck[0])
    P = oracle.make_problem(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, run.T_cap,
                            oracle.BF16, w.n_init, w.n_local, w.top_k)
    kr, _ = oracle.raw(run.data["k"][0])
    want = oracle.compress_cache(P, kr, run.data["seq_lens"].cpu().numpy())
    assert np.array_equal(run.ck[0].float().cpu().numpy().astype(np.float64).reshape(want.shape), want)


def test_append_capacity_flag(cuda_device):
    w = BASE.replace(name="x", batch=2, seq_len=64, top_k=1, needles=0)
    run = GpuCase(w, T_cap=65, steps=0)
    run.data["seq_lens"] = torch.tensor([64, 65], dtype=torch.int32, device="cuda")
    kn = torch.ones(w.batch, w.num_kv_heads, w.head_dim, dtype=w.torch_dtype, device="cuda")
    bsa.bsa_compress_append(run.p, run.data["k"][0], run.data["v"][0], kn, kn,
                            run.data["seq_lens"], run.ck[0], run.ws)
    assert run.data["seq_lens"].tolist() == [65, 65]
    assert run.device_errors() == bsa.DEVERR_CAPACITY
    assert run.device_errors() == 0   # reading clears the word


def test_device_error_flags(cuda_device):
    w = BASE.replace(name="x", batch=2, seq_len=640, top_k=2, needles=0)
    run = GpuCase(w)
    run.compress()
    run.data["seq_lens"][1] = run.T_cap + 5          # beyond capacity: pair skipped, flagged
    run.select()
    assert run.device_errors() == bsa.DEVERR_SEQ_LEN
    assert (run.n_sel[1] == 0).all()
    run.data["seq_lens"][1] = 640
    run.select()
    idx = run.block_idx.clone()
    idx[0, 0, 0] = 10                               # nb = 10: out of range
    run.decode(0, idx)
    assert run.device_errors() == bsa.DEVERR_BLOCK_IDX
    assert run.device_errors() == 0


# ------------------------------------------------------------------------------- full workloads
def _full_run(name):
    w = WORKLOADS[name]
    run = GpuCase(w)
    run.compress()
    return w, run


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny-f32-2k", "gqa4-bf16-32k-b1", "gqa4-bf16-128k-b16"])
def test_full_workload(name, cuda_device):
    w, run = _full_run(name)
    bsa.bsa_decode_step(run.p, run.q[0], run.data["k"][0], run.data["v"][0], run.ck[0], None,
                        None, run.data["seq_lens"], run.block_idx, run.n_sel, run.block_scores,
                        run.out[0], run.lse[0], run.ws)
    assert run.device_errors() == 0
    _, ties = full_check(run, sample_pairs(w, 12, seed=1))
    # planted needles are found (a property of the synthetic data, checked on every pair)
    nd = run.data["needles"]
    if nd.size:
        idx = run.block_idx.cpu().numpy()
        hit = np.mean([np.isin(nd[b, h], idx[b, h]).mean() for b in range(w.batch)
                       for h in range(w.num_kv_heads)])
        assert hit > 0.9, hit
    del run
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_back_to_back_calls_are_stable(cuda_device):
    """Many selections and decodes queued without a host sync between them (the launches overlap
    through programmatic dependent launch and the persistent rings run at full speed) give the
    first call's results bit for bit and raise no device error: pipeline races show up here."""
    w = WORKLOADS["gqa4-bf16-128k-b16"]
    run = GpuCase(w)
    run.compress()
    run.select()
    run.decode()
    torch.cuda.synchronize()
    first = (run.block_idx.clone(), run.n_sel.clone(), run.block_scores.clone(),
             run.out[0].clone(), run.lse[0].clone())
    for _ in range(60):
        run.select()
    for _ in range(60):
        run.decode()
    for _ in range(20):
        run.select()
        run.decode()
    torch.cuda.synchronize()
    assert run.device_errors() == 0
    now = (run.block_idx, run.n_sel, run.block_scores, run.out[0], run.lse[0])
    for a, b in zip(first, now):
        assert torch.equal(a, b)
    del run
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_shared_index_workload(cuda_device):
    """Selection on layer 0, reused by the sparse attention of all four layers (one launch)."""
    w, run = _full_run("shared-index-4x64k-b8")
    run.select(0)
    run.decode_layers()
    assert run.device_errors() == 0
    pairs = sample_pairs(w, 10, seed=2)
    orc0, ties = full_check(run, pairs, layer=0)
    # layers 1..3: attend with the layer-0 selection; near-tie pairs use the oracle's indices
    gi, gn = run.block_idx.clone(), run.n_sel.clone()
    if ties:
        from gpu_helpers import oracle_idx_tensor
        gi, gn = oracle_idx_tensor(run, pairs, orc0)
        run.decode_layers(gi, gn)
    fi = gi.view(-1, run.sizes.sel_cap).cpu().numpy()
    fn = gn.view(-1).cpu().numpy()
    for L in range(1, w.layers):
        orc = oracle_on_pairs(run, pairs, layer=L, given_idx=fi[pairs], given_n_sel=fn[pairs])
        check_output(run, pairs, orc, layer=L)
    del run
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_append_workload(cuda_device):
    """Growing cache: 20 steps of append + select + decode at batch 128, crossing a window
    completion; then the compressed keys and the last step are checked against the oracle."""
    w = WORKLOADS["append-bf16-16k-b128"]
    steps = 20
    run = GpuCase(w, steps=steps)
    run.compress()
    d = run.data
    for i in range(steps):
        bsa.bsa_decode_step(run.p, d["q_steps"][i], d["k"][0], d["v"][0], run.ck[0],
                            d["k_new"][i], d["v_new"][i], d["seq_lens"], run.block_idx, run.n_sel,
                            run.block_scores, run.out[0], run.lse[0], run.ws)
    assert run.device_errors() == 0
    assert (d["seq_lens"] == w.seq_len + steps).all()
    pairs = sample_pairs(w, 10, seed=3)
    # compressed keys of the sampled pairs, including the windows completed while appending
    P = oracle.make_problem(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, run.T_cap,
                            oracle.BF16, w.n_init, w.n_local, w.top_k)
    for pr in pairs[:3]:
        b, h = divmod(pr, w.num_kv_heads)
        kr, _ = oracle.raw(d["k"][0][b, h])
        want = oracle.compress(kr, oracle.BF16)
        got = run.ck[0][b, h, :want.shape[0]].float().cpu().numpy().astype(np.float64)
        assert np.array_equal(got, want)
    # the last step's selection and output
    run_q = d["q_steps"][steps - 1]
    orc = oracle_on_pairs(run, pairs, q=run_q)
    ties = check_selection(run, pairs, orc)
    check_output(run, pairs, orc, skip=set(ties))
    del run
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ Forecast indexer (SparDA Eq. 4)
FORECAST = {
    # few pairs: the selection splits each pair's windows over several CTAs
    "bf16-g4-d128-ragged": BASE.replace(name="x", batch=2, seq_len=4096 + 37, top_k=8, needles=4,
                                        forecast=True),
    "bf16-g8-d64": BASE.replace(name="x", batch=2, num_q_heads=16, num_kv_heads=2, head_dim=64,
                                seq_len=3000, top_k=6, needles=3, forecast=True),
    "f32-g4-d128": BASE.replace(name="x", dtype="f32", batch=1, seq_len=2500, top_k=6, needles=2,
                                forecast=True),
    "bf16-bs32-l16s8": BASE.replace(name="x", batch=1, num_q_heads=4, num_kv_heads=2, head_dim=64,
                                    seq_len=2000, block_size=32, cmp_kernel=16, cmp_stride=8,
                                    top_k=10, needles=3, forecast=True),
    # enough pairs for one CTA per pair (the shared-memory ring and shuffle block maxima)
    "bf16-256-pairs": BASE.replace(name="x", batch=32, seq_len=6000, top_k=12, needles=3,
                                   forecast=True),
}


@pytest.mark.parametrize("case", sorted(FORECAST))
def test_forecast_select_and_decode(case, cuda_device):
    """Blocks chosen by one Forecast vector per group (raw scores f . K~, no softmax), attended by
    the group's queries."""
    w = FORECAST[case]
    run = GpuCase(w)
    run.compress()
    f = run.data["f"]
    bsa.bsa_select_blocks_forecast(run.p, f, run.ck[0], run.data["seq_lens"], run.block_idx,
                                   run.n_sel, run.block_scores, run.ws)
    run.decode()
    assert run.device_errors() == 0
    forecast_check(run, sample_pairs(w, 48), f)


def test_forecast_ragged_lengths(cuda_device):
    """Different lengths in one batch, down to no window and an empty sequence."""
    w = BASE.replace(name="x", batch=5, seq_len=5000, top_k=9, needles=3, forecast=True)
    run = GpuCase(w, seq_lens=[5000, 64, 31, 0, 4097])
    run.compress()
    bsa.bsa_select_blocks_forecast(run.p, run.data["f"], run.ck[0], run.data["seq_lens"],
                                   run.block_idx, run.n_sel, run.block_scores, run.ws)
    run.decode()
    assert run.device_errors() == 0
    forecast_check(run, list(range(w.batch * w.num_kv_heads)), run.data["f"])


@pytest.mark.slow
def test_forecast_full_workload(cuda_device):
    w = WORKLOADS["forecast-bf16-128k-b16"]
    run = GpuCase(w)
    run.compress()
    bsa.bsa_select_blocks_forecast(run.p, run.data["f"], run.ck[0], run.data["seq_lens"],
                                   run.block_idx, run.n_sel, run.block_scores, run.ws)
    run.decode()
    assert run.device_errors() == 0
    forecast_check(run, sample_pairs(w, 12, seed=2), run.data["f"])
    # the needles lie along each group's mean query, which is the Forecast vector here
    nd = run.data["needles"]
    idx = run.block_idx.cpu().numpy()
    hit = np.mean([np.isin(nd[b, h], idx[b, h]).mean() for b in range(w.batch)
                   for h in range(w.num_kv_heads)])
    assert hit > 0.9, hit
    del run
    torch.cuda.empty_cache()


# ----------------------------------------------------------- anchored index reuse (Kascade, CLSA)
@pytest.mark.parametrize("anchors,dtype", [((0, 2), "bf16"), ((0, 1, 3), "bf16"), ((0, 2), "f32")])
def test_anchored_reuse(anchors, dtype, cuda_device):
    """Each anchor layer selects its own blocks per kv head; the layers up to the next anchor
    attend those blocks."""
    w = BASE.replace(name="x", batch=2, seq_len=3000 + 29, top_k=6, needles=3, layers=4,
                     anchors=anchors, dtype=dtype)
    run = GpuCase(w)
    run.compress()
    A, s = len(anchors), run.sizes
    idx = torch.full((A, w.batch, w.num_kv_heads, s.sel_cap), -7, dtype=torch.int32, device="cuda")
    ns = torch.full((A, w.batch, w.num_kv_heads), -7, dtype=torch.int32, device="cuda")
    bsa.bsa_decode_step_anchored(run.p, anchors, [run.q[L] for L in range(w.layers)], run.data["k"],
                                 run.data["v"], run.ck, run.data["seq_lens"], idx, ns, run.out,
                                 run.lse, run.ws)
    assert run.device_errors() == 0
    pairs = list(range(w.batch * w.num_kv_heads))
    bounds = list(anchors) + [w.layers]
    for i in range(A):
        a0, a1 = bounds[i], bounds[i + 1]
        orc = oracle_on_pairs(run, pairs, a0)           # the anchor layer's own selection
        gi, gn = idx[i].view(len(pairs), -1).cpu().numpy(), ns[i].view(-1).cpu().numpy()
        for j, pr in enumerate(pairs):
            n_o = int(orc["n_sel"][j])
            assert int(gn[pr]) == n_o
            if not near_tie(orc["boundary"][j]):
                assert gi[pr, :n_o].tolist() == orc["idx"][j, :n_o].tolist(), (i, pr)
        # every layer of the group attends the anchor's (GPU) selection
        for L in range(a0, a1):
            ref = oracle_on_pairs(run, pairs, L, given_idx=gi, given_n_sel=gn)
            check_output(run, pairs, ref, L)


@pytest.mark.slow
def test_full_anchored_workload(cuda_device):
    """The 4 x 64K x 8 workload with anchors at layers 0 and 2, in the bench's launch
    configuration (one anchored call), checked on sampled pairs."""
    w, run = _full_run("anchors-2of4-64k-b8")
    A, s = len(w.anchors), run.sizes
    idx = torch.full((A, w.batch, w.num_kv_heads, s.sel_cap), -7, dtype=torch.int32, device="cuda")
    ns = torch.full((A, w.batch, w.num_kv_heads), -7, dtype=torch.int32, device="cuda")
    bsa.bsa_decode_step_anchored(run.p, w.anchors, [run.q[L] for L in range(w.layers)],
                                 run.data["k"], run.data["v"], run.ck, run.data["seq_lens"], idx, ns,
                                 run.out, run.lse, run.ws)
    assert run.device_errors() == 0
    pairs = sample_pairs(w, 6, seed=3)
    bounds = list(w.anchors) + [w.layers]
    for i in range(A):
        orc = oracle_on_pairs(run, pairs, bounds[i])
        gi = idx[i].view(-1, s.sel_cap).cpu().numpy()
        gn = ns[i].view(-1).cpu().numpy()
        for j, pr in enumerate(pairs):
            n_o = int(orc["n_sel"][j])
            assert int(gn[pr]) == n_o
            if not near_tie(orc["boundary"][j]):
                assert gi[pr, :n_o].tolist() == orc["idx"][j, :n_o].tolist(), (i, pr)
        for L in range(bounds[i], bounds[i + 1]):
            ref = oracle_on_pairs(run, pairs, L, given_idx=gi[pairs], given_n_sel=gn[pairs])
            check_output(run, pairs, ref, L)
    del run
    torch.cuda.empty_cache()

