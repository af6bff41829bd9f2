"""Pins for the CPU oracle: checks against facts that do not come from the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
  * a library routine that computes the same quantity in a special case (torch avg_pool1d,
    max_pool1d, softmax, scaled_dot_product_attention, logsumexp, dtype casts, all in float64 on
    the CPU),
  * a closed form worked out by hand,
  * an invariant of the method, or
  * brute force over all candidates on tiny inputs.
The pytest wrappers are in test_oracle_pins.py; test_oracle_mutations.py runs the same functions
against copies of the oracle with planted mistakes and requires that some pin fails for each.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
rng_seed = 1234


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _randn(shape, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)


def golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------- rounding
def pin_round_bf16_matches_torch():
    """Values exactly representable in fp32 (so torch's cast rounds once) round like torch does."""
    x32 = torch.cat([
        _randn((4000,), 1) * 3.0,
        _randn((500,), 2) * 1e-38,          # bf16 subnormal range
        _randn((500,), 3) * 1e30,
        torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8, 0.0, -0.0]),
    ])
    want = x32.to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_to(x32.to(torch.float64).numpy(), oracle.BF16)
    assert np.array_equal(got, want), "bf16 rounding differs from torch"


def pin_round_ties_even():
    """Halfway cases of bf16 (8 significant bits) go to the even neighbour (closed form): between
    1 and 1 + 2^-7 the midpoint 1 + 2^-8 rounds to 1; between 1 + 2^-7 and 1 + 2^-6 the midpoint
    1 + 3*2^-8 rounds to 1 + 2^-6; just above a midpoint rounds up."""
    cases = [(1.0 + 2.0 ** -8, 1.0), (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),
             (-(1.0 + 2.0 ** -8), -1.0), (1.0 + 2.0 ** -8 + 2.0 ** -30, 1.0 + 2.0 ** -7),
             (2.0 ** -130 * 1.5, 2.0 ** -130 * 1.5), (3.0 * 2.0 ** -134, 2.0 ** -132)]
    for x, want in cases:
        got = float(oracle.round_to([x], oracle.BF16)[0])
        assert got == want, (x, got, want)


def pin_round_f32_matches_numpy():
    x = np.random.default_rng(5).standard_normal(4000) * np.logspace(-40, 30, 4000)
    got = oracle.round_to(x, oracle.F32)
    assert np.array_equal(got, x.astype(np.float32).astype(np.float64))


# ------------------------------------------------------------------------------------- compression
def pin_compress_matches_avg_pool():
    """Eq. (2) is a 1-D average pool of each key channel, kernel l, stride s, no padding."""
    for (T, d, l, s) in [(300, 8, 32, 16), (64, 4, 32, 16), (31, 4, 32, 16), (97, 3, 8, 4),
                         (50, 2, 6, 3)]:
        k32 = _randn((T, d), 10 + T)
        bits = _bf16_bits(k32)
        kk = oracle.widen(bits, oracle.BF16)
        ck = oracle.compress(bits, oracle.BF16, l, s, round_dtype=oracle.NO_ROUND)
        if T < l:
            assert ck.shape[0] == 0
            continue
        ref = F.avg_pool1d(torch.from_numpy(kk).T.unsqueeze(0), kernel_size=l, stride=s)[0].T
        assert ck.shape == tuple(ref.shape), (ck.shape, ref.shape)
        np.testing.assert_allclose(ck, ref.numpy(), rtol=0, atol=1e-15)
        # stored form: rounded once to bf16
        ckr = oracle.compress(bits, oracle.BF16, l, s)
        want = ref.to(torch.bfloat16).to(torch.float64).numpy()
        # torch's cast goes through fp32; the pooled doubles here are exact in fp32 (sums of
        # at most l bf16 values scaled by 1/l with l a power of two or a short exact sum)
        mism = np.count_nonzero(ckr != want)
        assert mism <= max(1, ckr.size // 1000), f"{mism} rounding mismatches"


def pin_compress_constant_windows():
    """A window whose rows are all equal compresses to that row (closed form)."""
    T, d, l, s = 128, 4, 32, 16
    rows = torch.zeros(T, d)
    for c in range(T // s):
        rows[c * s:(c + 1) * s] = float(c + 1) * torch.tensor([1.0, -0.5, 0.25, 2.0])
    ck = oracle.compress(rows.numpy(), oracle.F32, l, s, round_dtype=oracle.NO_ROUND)
    nc = (T - l) // s + 1
    assert ck.shape == (nc, d)
    for j in range(nc):
        # window j covers chunks j and j+1 with values (j+1) and (j+2): mean (2j+3)/2
        np.testing.assert_allclose(ck[j], (2 * j + 3) / 2 * np.array([1.0, -0.5, 0.25, 2.0]),
                                   rtol=0, atol=0)


def pin_window_and_block_counts():
    g = golden("page_constants.json")
    l, s = g["cmp_kernel"], g["cmp_stride"]
    for T, nc in [(31, 0), (32, 1), (47, 1), (48, 2), (2048, 127), (131072, 8191), (16384, 1023)]:
        assert oracle.num_windows(T, l, s) == nc, (T, nc)
    for T, nb in [(1, 1), (64, 1), (65, 2), (2048, 32), (131072, 2048)]:
        assert oracle.num_blocks(T, 64) == nb


def pin_compress_cache_matches_per_pair():
    P = oracle.make_problem(2, 4, 2, 8, 200, oracle.BF16, 1, 1, 2)
    k = _bf16_bits(_randn((2, 2, 200, 8), 77))
    lens = np.array([200, 77], dtype=np.int32)
    ck = oracle.compress_cache(P, k, lens)
    nc_cap = oracle.num_windows(200, 32, 16)
    for pair in range(4):
        T = int(lens[pair // 2])
        one = oracle.compress(k[pair // 2, pair % 2, :T].copy(), oracle.BF16)
        assert np.array_equal(ck[pair, :one.shape[0]], one)
        assert not ck[pair, one.shape[0]:nc_cap].any()


# -------------------------------------------------------------------------------------- scoring
def pin_scores_single_head_is_softmax():
    q = _randn((1, 16), 20).double()
    ck = _randn((40, 16), 21).double()
    tau = 4.0
    S = oracle.group_scores(q.numpy(), ck.numpy(), tau)
    ref = torch.softmax((q @ ck.T)[0] / tau, dim=0).numpy()
    np.testing.assert_allclose(S, ref, rtol=1e-13, atol=1e-300)


def pin_scores_group_sum_of_softmaxes():
    """G heads: the sum over heads of each head's own softmax over the windows (library softmax)."""
    G, d, nc = 4, 16, 57
    q = _randn((G, d), 22).double()
    ck = _randn((nc, d), 23).double()
    tau = math.sqrt(d)
    S = oracle.group_scores(q.numpy(), ck.numpy(), tau)
    ref = torch.softmax(q @ ck.T / tau, dim=1).sum(dim=0).numpy()
    np.testing.assert_allclose(S, ref, rtol=1e-13, atol=1e-300)
    assert abs(S.sum() - G) < 1e-12


def pin_scores_closed_form():
    """Two windows whose scaled logits are 0 and ln 2: softmax is (1/3, 2/3); two identical heads
    double it."""
    tau = 3.0
    q = np.array([[1.0, 0.0], [1.0, 0.0]])
    ck = np.array([[0.0, 5.0], [math.log(2.0) * tau, -1.0]])
    S = oracle.group_scores(q, ck, tau)
    np.testing.assert_allclose(S, [2.0 / 3.0, 4.0 / 3.0], rtol=1e-15)


def pin_forecast_scores_closed_form():
    """Compact Forecast Indexer: one vector per group, raw dot products, no softmax."""
    f = np.array([1.0, 2.0, -1.0])
    ck = np.array([[3.0, 4.0, 0.0], [-1.0, 0.5, 2.0], [0.0, 0.0, 0.0]])
    np.testing.assert_array_equal(oracle.forecast_scores(f, ck), [11.0, -2.0, 0.0])


def pin_forecast_scores_unit_vectors():
    """f = e_t reads coordinate t of every compressed key."""
    d, nc = 16, 23
    ck = _randn((nc, d), 24).double().numpy()
    for t in range(d):
        f = np.zeros(d)
        f[t] = 1.0
        np.testing.assert_array_equal(oracle.forecast_scores(f, ck), ck[:, t])


# ------------------------------------------------------------------------------- block reduction
def pin_block_scores_match_max_pool():
    """With l=32, s=16, BS=64 the overlapping windows of block b are 4b-1 .. 4b+3: a max pool of
    kernel 5, stride 4, padding 1 over the window scores."""
    g = golden("page_constants.json")
    l, s = g["cmp_kernel"], g["cmp_stride"]
    for T in [2048, 4096 + 64, 640]:
        nc = oracle.num_windows(T, l, s)
        nb = oracle.num_blocks(T, 64)
        S = np.random.default_rng(T).random(nc)
        sb = oracle.block_scores(S, nb, l, s, 64)
        ref = F.max_pool1d(torch.from_numpy(S)[None, None], kernel_size=5, stride=4,
                           padding=1)[0, 0].numpy()
        assert ref.shape[0] == nb
        np.testing.assert_array_equal(sb, ref)


def pin_block_scores_brute_force_overlap():
    """Other geometries: enumerate the token sets of windows and blocks directly."""
    for (T, l, s, BS) in [(200, 8, 4, 16), (130, 32, 16, 64), (77, 6, 5, 16), (100, 16, 16, 32)]:
        nc = oracle.num_windows(T, l, s)
        nb = oracle.num_blocks(T, BS)
        S = np.random.default_rng(T + l).random(nc)
        sb = oracle.block_scores(S, nb, l, s, BS)
        for b in range(nb):
            btoks = set(range(b * BS, (b + 1) * BS))
            vals = [S[j] for j in range(nc) if btoks & set(range(j * s, j * s + l))]
            want = max(vals) if vals else -math.inf
            assert sb[b] == want, (T, l, s, BS, b)


# ------------------------------------------------------------------------------------- selection
def _dominance_topk(sb, cand, k):
    """All k-subsets of ``cand`` that no single swap improves, where a candidate beats another
    when its score is higher, or equal with a lower block index (brute force)."""
    winners = []
    for sub in itertools.combinations(cand, k):
        inside = set(sub)
        ok = True
        for c in inside:
            for o in cand:
                if o in inside:
                    continue
                if sb[o] > sb[c] or (sb[o] == sb[c] and o < c):
                    ok = False
                    break
            if not ok:
                break
        if ok:
            winners.append(inside)
    return winners


def pin_select_brute_force():
    rng = np.random.default_rng(42)
    for trial in range(60):
        nb = int(rng.integers(1, 12))
        n_init, n_local, k = (int(x) for x in rng.integers(0, 4, size=3))
        sb = rng.integers(0, 5, size=nb).astype(np.float64)   # many exact ties
        if trial % 3 == 0:
            sb[rng.integers(0, nb)] = -math.inf
        idx, bnd = oracle.select(sb, n_init, n_local, k)
        fixed = set(range(min(n_init, nb))) | set(range(max(nb - n_local, 0), nb))
        cand = [b for b in range(nb) if b not in fixed]
        kk = min(k, len(cand))
        winners = _dominance_topk(sb, cand, kk)
        assert len(winners) == 1, (sb, n_init, n_local, k, winners)
        want = sorted(fixed | winners[0])
        assert idx.tolist() == want, (sb.tolist(), n_init, n_local, k, idx.tolist(), want)
        taken = sorted(winners[0], key=lambda b: (-sb[b], b))
        rest = sorted(set(cand) - winners[0], key=lambda b: (-sb[b], b))
        if taken:
            assert bnd[0] == sb[taken[-1]]
        else:
            assert math.isnan(bnd[0])
        if rest:
            assert bnd[1] == sb[rest[0]]
        else:
            assert math.isnan(bnd[1])


def pin_select_invariants():
    rng = np.random.default_rng(7)
    for nb in [2, 5, 32, 512, 2048]:
        for (n_init, n_local, k) in [(1, 2, 4), (1, 4, 64), (0, 0, 3), (3, 3, 0)]:
            sb = rng.random(nb)
            idx, _ = oracle.select(sb, n_init, n_local, k)
            assert np.all(np.diff(idx) > 0), "ascending and distinct"
            fixed = set(range(min(n_init, nb))) | set(range(max(nb - n_local, 0), nb))
            assert fixed <= set(idx.tolist())
            assert len(idx) == len(fixed) + min(k, nb - len(fixed))


def pin_select_closed_form_ties():
    """Hand example: blocks 0 (init) and 7 (local) fixed; candidates 1..6 scores
    [5, 9, 9, 1, 9, 2]; k=2 takes the two lowest-index 9s (blocks 2 and 3)."""
    sb = np.array([0.0, 5, 9, 9, 1, 9, 2, 0])
    idx, bnd = oracle.select(sb, 1, 1, 2)
    assert idx.tolist() == [0, 2, 3, 7]
    assert bnd.tolist() == [9.0, 9.0]


# ------------------------------------------------------------------------------------- attention
def _sdpa(q, k, v, scale):
    """q [G][d], k/v [n][d] float64 -> out [G][d], lse [G] from torch's library routines."""
    q, k, v = (torch.as_tensor(a, dtype=torch.float64) for a in (q, k, v))
    out = F.scaled_dot_product_attention(q[None, :, None, :], k[None, None].expand(1, q.shape[0], -1, -1),
                                         v[None, None].expand(1, q.shape[0], -1, -1), scale=scale)
    lse = torch.logsumexp(q @ k.T * scale, dim=-1)
    return out[0, :, 0, :].numpy(), lse.numpy()


def pin_attend_all_blocks_is_dense():
    for (T, d, G, dt) in [(256, 16, 4, oracle.BF16), (200, 8, 2, oracle.F32), (64, 4, 1, oracle.F32)]:
        q = _randn((G, d), 30 + T).double().numpy()
        k32, v32 = _randn((T, d), 31 + T), _randn((T, d), 32 + T)
        if dt == oracle.BF16:
            kr, vr = _bf16_bits(k32), _bf16_bits(v32)
        else:
            kr, vr = k32.numpy(), v32.numpy()
        nb = oracle.num_blocks(T, 64)
        scale = 1.0 / math.sqrt(d)
        out, lse = oracle.attend(q, kr, vr, dt, T, np.arange(nb), 64, scale)
        ro, rl = _sdpa(q, oracle.widen(kr, dt), oracle.widen(vr, dt), scale)
        np.testing.assert_allclose(out, ro, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, rl, rtol=1e-13, atol=1e-13)


def pin_attend_subset_is_gathered_dense():
    """Selected blocks 0, 2 and the partial last block of T=150: dense attention over exactly
    tokens 0..63, 128..149."""
    T, d, G = 150, 8, 2
    q = _randn((G, d), 40).double().numpy()
    k, v = _randn((T, d), 41).numpy(), _randn((T, d), 42).numpy()
    out, lse = oracle.attend(q, k, v, oracle.F32, T, [0, 2], 64, 0.3)
    toks = list(range(0, 64)) + list(range(128, 150))
    ro, rl = _sdpa(q, k[toks].astype(np.float64), v[toks].astype(np.float64), 0.3)
    np.testing.assert_allclose(out, ro, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, rl, rtol=1e-13)


def pin_attend_identical_keys_mean_of_v():
    """Equal keys give equal weights: the output is the mean of the attended V rows, and the
    log-sum-exp is score + log(n)."""
    T, d = 128, 4
    k = np.tile(np.array([[0.5, -1.0, 2.0, 0.0]], dtype=np.float32), (T, 1))
    v = _randn((T, d), 50).numpy()
    q = np.array([[1.0, 1.0, 1.0, 1.0]])
    out, lse = oracle.attend(q, k, v, oracle.F32, T, [1], 64, 0.5)
    np.testing.assert_allclose(out[0], v[64:128].astype(np.float64).mean(axis=0), rtol=1e-12)
    np.testing.assert_allclose(lse[0], 0.5 * 1.5 + math.log(64), rtol=1e-14)
    ones = np.ones((T, d), dtype=np.float32)
    out1, _ = oracle.attend(_randn((3, d), 51).double().numpy(), _randn((T, d), 52).numpy(), ones,
                            oracle.F32, T, [0, 1], 64, 1.0)
    np.testing.assert_allclose(out1, 1.0, rtol=1e-14)   # weights sum to one


# ------------------------------------------------------------------------------- whole decode step
def pin_decode_full_coverage_is_dense_gqa():
    """top_k >= number of candidates: every block is selected and each query head h attends
    densely to kv head h // G (torch SDPA with the kv heads repeated per group)."""
    B, Hq, Hkv, d, T_cap = 2, 8, 2, 16, 300
    lens = np.array([300, 170], dtype=np.int32)
    q = _randn((B, Hq, d), 60)
    k, v = _randn((B, Hkv, T_cap, d), 61), _randn((B, Hkv, T_cap, d), 62)
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    P = oracle.make_problem(B, Hq, Hkv, d, T_cap, oracle.BF16, 1, 1, 100)
    res = oracle.decode(P, qb, kb, vb, lens)
    G = Hq // Hkv
    qd = torch.from_numpy(oracle.widen(qb, oracle.BF16))
    kd = torch.from_numpy(oracle.widen(kb, oracle.BF16)).repeat_interleave(G, dim=1)
    vd = torch.from_numpy(oracle.widen(vb, oracle.BF16)).repeat_interleave(G, dim=1)
    for b in range(B):
        T = int(lens[b])
        ref = F.scaled_dot_product_attention(qd[b][:, None], kd[b][:, :T], vd[b][:, :T],
                                             scale=1.0 / math.sqrt(d))[:, 0]
        for kvh in range(Hkv):
            i = b * Hkv + kvh
            nb = oracle.num_blocks(T, 64)
            assert res["idx"][i, :res["n_sel"][i]].tolist() == list(range(nb))
            np.testing.assert_allclose(res["out"][i], ref[kvh * G:(kvh + 1) * G].numpy(),
                                       rtol=1e-12, atol=1e-13)


def pin_decode_selection_composes():
    """The batch driver's selection equals compress -> group scores -> block scores -> select on
    each pair, and its output equals attending the selected blocks."""
    B, Hq, Hkv, d, T = 1, 4, 2, 16, 64 * 20
    q, k, v = _randn((B, Hq, d), 70), _randn((B, Hkv, T, d), 71), _randn((B, Hkv, T, d), 72)
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    P = oracle.make_problem(B, Hq, Hkv, d, T, oracle.BF16, 1, 2, 3)
    res = oracle.decode(P, qb, kb, vb, [T])
    G = Hq // Hkv
    for kvh in range(Hkv):
        ck = oracle.compress(kb[0, kvh].copy(), oracle.BF16)
        qg = oracle.widen(qb[0, kvh * G:(kvh + 1) * G], oracle.BF16)
        S = oracle.group_scores(qg, ck, math.sqrt(d))
        sb = oracle.block_scores(S, oracle.num_blocks(T, 64))
        idx, _ = oracle.select(sb, 1, 2, 3)
        assert res["idx"][kvh, :res["n_sel"][kvh]].tolist() == idx.tolist()
        np.testing.assert_array_equal(res["block_scores"][kvh, :sb.size], sb)
        out, lse = oracle.attend(qg, kb[0, kvh].copy(), vb[0, kvh].copy(), oracle.BF16, T, idx)
        np.testing.assert_array_equal(res["out"][kvh], out)


def pin_decode_given_compressed_keys_composes():
    """A decode step on keys compressed beforehand (compress_cache, then decode with ck) gives the
    selection, block scores and output of the driver that compresses on its own, bit for bit, on
    ragged lengths and a pair subset; the thread count changes nothing."""
    B, Hq, Hkv, d, Tc = 2, 6, 3, 16, 64 * 18
    q, k, v = _randn((B, Hq, d), 86), _randn((B, Hkv, Tc, d), 87), _randn((B, Hkv, Tc, d), 88)
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    P = oracle.make_problem(B, Hq, Hkv, d, Tc, oracle.BF16, 1, 2, 4)
    lens, pairs = [Tc, 64 * 11 + 23], [0, 2, 4, 5]
    ref = oracle.decode(P, qb, kb, vb, lens, pairs=pairs)
    ck = oracle.compress_cache(P, kb, lens, pairs=pairs)
    for n in (1, 3):
        with oracle.threads(n):
            got = oracle.decode(P, qb, kb, vb, lens, pairs=pairs, ck=ck)
        for key in ("idx", "n_sel", "block_scores", "out", "lse"):
            np.testing.assert_array_equal(got[key], ref[key])
    # the Forecast driver too
    f = _bf16_bits(_randn((B, Hkv, d), 89))
    ref_f = oracle.decode_forecast(P, f, qb, kb, vb, lens, pairs=pairs)
    got_f = oracle.decode_forecast(P, f, qb, kb, vb, lens, pairs=pairs, ck=ck)
    for key in ("idx", "n_sel", "block_scores", "out", "lse"):
        np.testing.assert_array_equal(got_f[key], ref_f[key])


def pin_shared_index_identical_layers():
    """[CLSA]/[Kascade] reuse: attending an identical layer with layer 0's index reproduces layer
    0's output; a different layer gives its own dense-over-selected result."""
    B, Hq, Hkv, d, T = 1, 4, 1, 8, 64 * 6
    q, k, v = _randn((B, Hq, d), 80), _randn((B, Hkv, T, d), 81), _randn((B, Hkv, T, d), 82)
    P = oracle.make_problem(B, Hq, Hkv, d, T, oracle.F32, 1, 1, 1)
    r0 = oracle.decode(P, q.numpy(), k.numpy(), v.numpy(), [T])
    r1 = oracle.attend_pairs(P, q.numpy(), k.numpy(), v.numpy(), [T], r0["idx"], r0["n_sel"])
    np.testing.assert_array_equal(r0["out"], r1["out"])
    np.testing.assert_array_equal(r0["lse"], r1["lse"])
    v2 = _randn((B, Hkv, T, d), 83)
    r2 = oracle.attend_pairs(P, q.numpy(), k.numpy(), v2.numpy(), [T], r0["idx"], r0["n_sel"])
    toks = [t for b in r0["idx"][0, :r0["n_sel"][0]] for t in range(b * 64, b * 64 + 64)]
    ro, _ = _sdpa(q[0].double().numpy(), k[0, 0, toks].double().numpy(),
                  v2[0, 0, toks].double().numpy(), 1.0 / math.sqrt(d))
    np.testing.assert_allclose(r2["out"][0], ro, rtol=1e-12, atol=1e-13)


def pin_forecast_decode_composes():
    """The forecast driver selects each pair with its own Forecast vector f[b][kvh]: compress ->
    forecast scores -> block scores -> select, then q attends the selected blocks."""
    B, Hq, Hkv, d, T = 2, 4, 2, 16, 64 * 20
    q, k, v = _randn((B, Hq, d), 90), _randn((B, Hkv, T, d), 91), _randn((B, Hkv, T, d), 92)
    f = _randn((B, Hkv, d), 93)
    qb, kb, vb, fb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v), _bf16_bits(f)
    P = oracle.make_problem(B, Hq, Hkv, d, T, oracle.BF16, 1, 2, 3)
    lens = [T, T - 100]
    res = oracle.decode_forecast(P, fb, qb, kb, vb, lens)
    G = Hq // Hkv
    for b in range(B):
        for kvh in range(Hkv):
            i = b * Hkv + kvh
            Tb = lens[b]
            ck = oracle.compress(kb[b, kvh, :Tb].copy(), oracle.BF16)
            S = oracle.forecast_scores(oracle.widen(fb[b, kvh], oracle.BF16), ck)
            sb = oracle.block_scores(S, oracle.num_blocks(Tb, 64))
            idx, _ = oracle.select(sb, 1, 2, 3)
            assert res["idx"][i, :res["n_sel"][i]].tolist() == idx.tolist()
            np.testing.assert_array_equal(res["block_scores"][i, :sb.size], sb)
            qg = oracle.widen(qb[b, kvh * G:(kvh + 1) * G], oracle.BF16)
            out, _ = oracle.attend(qg, kb[b, kvh].copy(), vb[b, kvh].copy(), oracle.BF16, Tb, idx)
            np.testing.assert_array_equal(res["out"][i], out)


def pin_forecast_one_head_matches_base_selector():
    """With one query head per group, the base selector's softmax is monotone in q . K~, so a
    Forecast vector equal to q selects the same blocks (and q attends them identically); doubling
    f doubles every block score exactly and keeps the selection."""
    B, Hq, Hkv, d, T = 1, 3, 3, 16, 64 * 24
    q, k, v = _randn((B, Hq, d), 94), _randn((B, Hkv, T, d), 95), _randn((B, Hkv, T, d), 96)
    P = oracle.make_problem(B, Hq, Hkv, d, T, oracle.F32, 1, 2, 5)
    qn, kn, vn = q.numpy(), k.numpy(), v.numpy()
    base = oracle.decode(P, qn, kn, vn, [T])
    fc = oracle.decode_forecast(P, qn.reshape(B, Hkv, d), qn, kn, vn, [T])
    assert np.array_equal(base["idx"], fc["idx"]) and np.array_equal(base["n_sel"], fc["n_sel"])
    np.testing.assert_array_equal(base["out"], fc["out"])
    fc2 = oracle.decode_forecast(P, (2.0 * qn).reshape(B, Hkv, d), qn, kn, vn, [T])
    assert np.array_equal(fc2["idx"], fc["idx"])
    np.testing.assert_array_equal(fc2["block_scores"], 2.0 * fc["block_scores"])


def pin_lookahead_step_brute_force():
    """One-layer lookahead (SparDA Architecture, Eqs. 4-5): layer 0 attends the blocks given for it
    (the gathered tokens through torch's SDPA, in float64), and layer 1's blocks are those whose
    raw Forecast score f . K~_j (numpy dot products over the windows of each block) rank highest,
    ties to the lower block, from a plain sort, united with the init and local blocks."""
    B, Hq, Hkv, d, Tc = 1, 4, 2, 16, 64 * 14
    q, k0, v0 = _randn((B, Hq, d), 97), _randn((B, Hkv, Tc, d), 98), _randn((B, Hkv, Tc, d), 99)
    k1, f = _randn((B, Hkv, Tc, d), 100), _randn((B, Hkv, d), 101)
    P = oracle.make_problem(B, Hq, Hkv, d, Tc, oracle.F32, 1, 2, 3)
    T = 64 * 11 + 40
    qn, k0n, v0n, k1n, fn = (x.numpy() for x in (q, k0, v0, k1, f))
    idx0 = np.array([[0, 4, 5, 9, 11, -1], [0, 2, 7, 8, 10, 11]], dtype=np.int32)
    nsel0 = np.array([5, 6], dtype=np.int32)
    ck1 = oracle.compress_cache(P, k1n, [T])
    res = oracle.lookahead_step(P, qn, k0n, v0n, idx0, nsel0, fn, ck1, [T])
    G = Hq // Hkv
    nb = -(-T // 64)
    nc = (T - 32) // 16 + 1
    for kvh in range(Hkv):
        toks = [t for b in idx0[kvh, :nsel0[kvh]] for t in range(b * 64, min(b * 64 + 64, T))]
        ro, rl = _sdpa(qn[0, kvh * G:(kvh + 1) * G].astype(np.float64), k0n[0, kvh, toks].astype(np.float64),
                       v0n[0, kvh, toks].astype(np.float64), 1.0 / math.sqrt(d))
        np.testing.assert_allclose(res["out"][kvh], ro, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(res["lse"][kvh], rl, rtol=1e-12, atol=1e-13)
        # layer 1: windows j cover tokens [16j, 16j + 32); block b takes the max over the windows
        # that overlap its tokens
        kk = k1n[0, kvh].astype(np.float64)
        win = np.array([kk[16 * j:16 * j + 32].mean(0) for j in range(nc)])
        win = win.astype(np.float32).astype(np.float64)  # the cache dtype (fp32) rounding
        raw = win @ fn[0, kvh].astype(np.float64)
        sb = [max(raw[j] for j in range(nc) if 16 * j < 64 * (b + 1) and 16 * j + 32 > 64 * b)
              for b in range(nb)]
        fixed = {0} | {nb - 2, nb - 1}
        cand = sorted((b for b in range(nb) if b not in fixed), key=lambda b: (-sb[b], b))
        want = sorted(fixed | set(cand[:3]))
        assert res["idx"][kvh, :res["n_sel"][kvh]].tolist() == want
        np.testing.assert_allclose(res["block_scores"][kvh, :nb], sb, rtol=1e-12, atol=1e-12)


def pin_prefill_single_position_is_decode():
    """A prefill chunk of one query at the first position of a block is a decode step at that
    length: the windows complete before the block are those complete one token later, the tile's
    score is that one query's, and it attends tokens up to itself, so selection and output agree
    bit for bit."""
    B, Hq, Hkv, d, Tc = 1, 6, 2, 16, 64 * 16
    k, v = _randn((B, Hkv, Tc, d), 102), _randn((B, Hkv, Tc, d), 103)
    kb, vb = _bf16_bits(k), _bf16_bits(v)
    P = oracle.make_problem(B, Hq, Hkv, d, Tc, oracle.BF16, 1, 2, 4)
    for r in (0, 1, 5, 13):
        T = 64 * r + 1
        q = _bf16_bits(_randn((B, 1, Hq, d), 104 + r))
        pre = oracle.prefill(P, q, kb, vb, [T], 1)
        dec = oracle.decode(P, q[:, 0], kb, vb, [T])
        for i in range(Hkv):
            n = int(dec["n_sel"][i])
            assert int(pre["n_sel"][i, 0]) == n and pre["idx"][i, 0, :n].tolist() == dec["idx"][i, :n].tolist()
            assert (pre["n_sel"][i, 1:] == 0).all()
            np.testing.assert_array_equal(pre["out"][i, 0], dec["out"][i])
            np.testing.assert_array_equal(pre["lse"][i, 0], dec["lse"][i])


def pin_prefill_all_blocks_is_causal_dense():
    """With top-k covering every candidate each query attends every earlier token and itself:
    causal dense attention (torch SDPA in float64 with a causal mask), for a chunk that starts and
    ends inside blocks."""
    B, Hq, Hkv, d = 1, 4, 2, 16
    T, C = 64 * 5 + 20, 100
    q, k, v = _randn((B, C, Hq, d), 105), _randn((B, Hkv, T, d), 106), _randn((B, Hkv, T, d), 107)
    P = oracle.make_problem(B, Hq, Hkv, d, T, oracle.F32, 1, 1, 64)
    res = oracle.prefill(P, q.numpy(), k.numpy(), v.numpy(), [T], C)
    G = Hq // Hkv
    for kvh in range(Hkv):
        for c in range(C):
            pos = T - C + c
            ro, rl = _sdpa(q[0, c, kvh * G:(kvh + 1) * G].double().numpy(), k[0, kvh, :pos + 1].double().numpy(),
                           v[0, kvh, :pos + 1].double().numpy(), 1.0 / math.sqrt(d))
            np.testing.assert_allclose(res["out"][kvh, c], ro, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(res["lse"][kvh, c], rl, rtol=1e-12, atol=1e-13)


def pin_prefill_tile_selection_brute_force():
    """Each query tile's blocks by brute force: per position and head a softmax (torch) over the
    windows complete before the tile's block, summed; the block score the largest over the
    overlapping windows (plain loops); the top-k from a plain sort, ties to the lower block."""
    B, Hq, Hkv, d = 1, 4, 1, 8
    T, C = 64 * 9 + 37, 64 * 3 + 5
    q, k, v = _randn((B, C, Hq, d), 108), _randn((B, Hkv, T, d), 109), _randn((B, Hkv, T, d), 110)
    n_init, n_local, top_k = 1, 2, 3
    P = oracle.make_problem(B, Hq, Hkv, d, T, oracle.F32, n_init, n_local, top_k)
    res = oracle.prefill(P, q.numpy(), k.numpy(), v.numpy(), [T], C)
    kk = k[0, 0].double()
    t0 = T - C
    r_lo, r_hi = t0 // 64, (T - 1) // 64
    assert res["idx"].shape[1] == oracle.prefill_tiles_cap(C) and (res["n_sel"][0, r_hi - r_lo + 1:] == 0).all()
    for r in range(r_lo, r_hi + 1):
        nc = max((64 * r - 32) // 16 + 1, 0) if 64 * r >= 32 else 0
        win = torch.stack([kk[16 * j:16 * j + 32].mean(0) for j in range(nc)]) if nc else torch.zeros(0, d, dtype=torch.float64)
        win = win.float().double()  # the cache dtype (fp32)
        S = torch.zeros(nc, dtype=torch.float64)
        for pos in range(max(t0, 64 * r), min(T, 64 * r + 64)):
            for h in range(Hq):
                if nc:
                    S += torch.softmax(win @ q[0, pos - t0, h].double() / math.sqrt(d), dim=0)
        nb = r + 1
        sb = [max([float(S[j]) for j in range(nc) if 16 * j < 64 * (b + 1) and 16 * j + 32 > 64 * b], default=-math.inf)
              for b in range(nb)]
        fixed = set(range(min(n_init, nb))) | set(range(max(nb - n_local, min(n_init, nb)), nb))
        cand = sorted((b for b in range(nb) if b not in fixed), key=lambda b: (-sb[b], b))
        want = sorted(fixed | set(cand[:top_k]))
        ti = r - r_lo
        got = res["idx"][0, ti, :res["n_sel"][0, ti]].tolist()
        assert got == want, (r, got, want)


def pin_clsa_token_index_brute_force():
    """CLSA's token index: per pair the sum over the group's heads of a softmax (torch) over every
    token's key, the first and last tokens of the budget always taken and the rest by a plain sort
    (ties to the lower token); every layer's output is SDPA over exactly those tokens."""
    B, Hq, Hkv, d, T, BS = 1, 4, 2, 8, 200, 16
    n_init, n_local, top_k = 1, 1, 3
    L = 2
    qs = [_randn((B, Hq, d), 111 + 3 * l) for l in range(L)]
    ks = [_randn((B, Hkv, T, d), 112 + 3 * l) for l in range(L)]
    vs = [_randn((B, Hkv, T, d), 113 + 3 * l) for l in range(L)]
    P = oracle.make_problem(B, Hq, Hkv, d, T, oracle.F32, n_init, n_local, top_k, block_size=BS)
    Tn = 170
    res = oracle.clsa(P, [q.numpy() for q in qs], [k.numpy() for k in ks], [v.numpy() for v in vs], [Tn])
    G = Hq // Hkv
    for kvh in range(Hkv):
        S = sum(torch.softmax(ks[0][0, kvh, :Tn].double() @ qs[0][0, kvh * G + h].double() / math.sqrt(d), dim=0)
                for h in range(G))
        fixed = set(range(n_init * BS)) | set(range(Tn - n_local * BS, Tn))
        cand = sorted((t for t in range(Tn) if t not in fixed), key=lambda t: (-float(S[t]), t))
        want = sorted(fixed | set(cand[:top_k * BS]))
        assert res["idx"][kvh, :res["n_sel"][kvh]].tolist() == want
        assert (res["idx"][kvh, res["n_sel"][kvh]:] == -1).all()
        for l in range(L):
            ro, rl = _sdpa(qs[l][0, kvh * G:(kvh + 1) * G].double().numpy(), ks[l][0, kvh, want].double().numpy(),
                           vs[l][0, kvh, want].double().numpy(), 1.0 / math.sqrt(d))
            np.testing.assert_allclose(res["out"][l, kvh], ro, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(res["lse"][l, kvh], rl, rtol=1e-12, atol=1e-13)


ALL_PINS = [
    pin_round_bf16_matches_torch, pin_round_ties_even, pin_round_f32_matches_numpy,
    pin_compress_matches_avg_pool, pin_compress_constant_windows, pin_window_and_block_counts,
    pin_compress_cache_matches_per_pair,
    pin_scores_single_head_is_softmax, pin_scores_group_sum_of_softmaxes, pin_scores_closed_form,
    pin_forecast_scores_closed_form, pin_forecast_scores_unit_vectors,
    pin_block_scores_match_max_pool, pin_block_scores_brute_force_overlap,
    pin_select_brute_force, pin_select_invariants, pin_select_closed_form_ties,
    pin_attend_all_blocks_is_dense, pin_attend_subset_is_gathered_dense,
    pin_attend_identical_keys_mean_of_v,
    pin_decode_full_coverage_is_dense_gqa, pin_decode_selection_composes,
    pin_decode_given_compressed_keys_composes,
    pin_shared_index_identical_layers,
    pin_forecast_decode_composes, pin_forecast_one_head_matches_base_selector,
    pin_lookahead_step_brute_force,
    pin_prefill_single_position_is_decode, pin_prefill_all_blocks_is_causal_dense,
    pin_prefill_tile_selection_brute_force, pin_clsa_token_index_brute_force,
]
