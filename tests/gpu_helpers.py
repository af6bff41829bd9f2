"""Shared helpers of the GPU parity tests: run the CUDA path on a workload, run the oracle on a
sample of its (batch, kv-head) pairs, and compare with the pass rules:

  * compressed keys: bit-identical (fp64 window sums on both sides, one rounding each);
  * block indices: identical, except for pairs whose oracle k-th and (k+1)-th block scores are
    within 1e-3 relative (several correct answers); those are checked for validity and their
    output is checked by attending the oracle's indices on the GPU;
  * block scores: relative 1e-4 (fp32 on the GPU vs fp64);
  * outputs: max-abs 1e-5 (fp32) or 1e-2 (bf16 output, fp32 accumulation); LSE 1e-5 / 1e-4.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_attention_compressed_b200 as bsa
import oracle
from block_sparse_attention_compressed_b200.workloads import Workload, generate

NEAR_TIE_REL = 1e-3
SCORE_RTOL = 1e-4
OUT_ATOL = {"f32": 1e-5, "bf16": 1e-2}
LSE_ATOL = {"f32": 1e-5, "bf16": 1e-4}


def params_for(w: Workload, T_cap: int, layers: int | None = None) -> bsa.Params:
    return bsa.make_params(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, T_cap, w.dtype,
                           w.n_init, w.n_local, w.top_k, w.cmp_kernel, w.cmp_stride, w.block_size,
                           num_layers=layers or w.layers)


def oracle_problem(w: Workload, n: int, T_cap: int):
    return oracle.make_problem(n, w.group, 1, w.head_dim, T_cap,
                               oracle.F32 if w.dtype == "f32" else oracle.BF16, w.n_init, w.n_local,
                               w.top_k, w.cmp_kernel, w.cmp_stride, w.block_size)


class GpuCase:
    """Buffers of one workload on the GPU, and the library calls on them."""

    def __init__(self, w: Workload, device="cuda", seq_lens=None, T_cap=None, steps=None):
        self.w = w
        self.data = generate(w, device=device, seq_cap=T_cap, steps=steps)
        self.T_cap = self.data["seq_cap"]
        if seq_lens is not None:
            self.data["seq_lens"] = torch.tensor(seq_lens, dtype=torch.int32, device=device)
        self.p = params_for(w, self.T_cap)
        s = bsa.bsa_get_sizes(self.p)
        self.sizes = s
        B, Hkv, d = w.batch, w.num_kv_heads, w.head_dim
        dt = w.torch_dtype
        self.ck = [torch.zeros(B, Hkv, s.nc_cap, d, dtype=dt, device=device) for _ in range(w.layers)]
        self.ws = bsa.alloc_workspace(self.p, device)
        bsa.bsa_workspace_init(self.p, self.ws)
        self.block_idx = torch.full((B, Hkv, s.sel_cap), -7, dtype=torch.int32, device=device)
        self.n_sel = torch.full((B, Hkv), -7, dtype=torch.int32, device=device)
        self.block_scores = torch.zeros(B, Hkv, s.nb_cap, dtype=torch.float32, device=device)
        self.out = [torch.full((B, w.num_q_heads, d), 77.0, dtype=dt, device=device)
                    for _ in range(w.layers)]
        self.lse = [torch.full((B, w.num_q_heads), 77.0, dtype=torch.float32, device=device)
                    for _ in range(w.layers)]

    @property
    def q(self):
        return self.data["q"]

    def compress(self):
        for L in range(self.w.layers):
            bsa.bsa_compress_keys(self.p, self.data["k"][L], self.data["seq_lens"], self.ck[L])

    def select(self, layer=0, q=None):
        bsa.bsa_select_blocks(self.p, self.q[layer] if q is None else q, self.ck[layer],
                              self.data["seq_lens"], self.block_idx, self.n_sel, self.block_scores,
                              self.ws)

    def decode(self, layer=0, block_idx=None, n_sel=None, q=None):
        bsa.bsa_sparse_decode(self.p, self.q[layer] if q is None else q, self.data["k"][layer],
                              self.data["v"][layer], self.data["seq_lens"],
                              self.block_idx if block_idx is None else block_idx,
                              self.n_sel if n_sel is None else n_sel, self.out[layer],
                              self.lse[layer], self.ws)

    def step(self, q=None, block_scores=True, fused=False):
        """bsa_decode_step on layer 0 (no append): selection and attention in one call; with
        ``fused``, bsa_decode_step_fused (the one-kernel step, whatever the number of pairs)."""
        bsa.bsa_decode_step(self.p, self.q[0] if q is None else q, self.data["k"][0],
                            self.data["v"][0], self.ck[0], None, None, self.data["seq_lens"],
                            self.block_idx, self.n_sel, self.block_scores if block_scores else None,
                            self.out[0], self.lse[0], self.ws, fused=fused)

    def decode_layers(self, block_idx=None, n_sel=None):
        L = self.w.layers
        bsa.bsa_sparse_decode_layers(self.p, [self.q[i] for i in range(L)], self.data["k"],
                                     self.data["v"], self.data["seq_lens"],
                                     self.block_idx if block_idx is None else block_idx,
                                     self.n_sel if n_sel is None else n_sel, self.out, self.lse,
                                     self.ws)

    def device_errors(self) -> int:
        return bsa.bsa_read_device_error(self.ws)


def sample_pairs(w: Workload, n: int, seed: int = 0) -> list[int]:
    total = w.batch * w.num_kv_heads
    if total <= n:
        return list(range(total))
    rng = np.random.default_rng(seed)
    picks = set(rng.choice(total, size=n - 2, replace=False).tolist())
    picks.update({0, total - 1})
    return sorted(picks)


def oracle_on_pairs(run: GpuCase, pairs: list[int], layer=0, given_idx=None, given_n_sel=None,
                    q=None) -> dict:
    """Oracle over a sub-batch made of the listed pairs (one kv head each, its G query heads)."""
    w = run.w
    G, Hkv = w.group, w.num_kv_heads
    qfull = run.q[layer] if q is None else q
    qs, ks, vs, lens = [], [], [], []
    seq = run.data["seq_lens"].cpu()
    for pr in pairs:
        b, h = divmod(pr, Hkv)
        qs.append(qfull[b, h * G:(h + 1) * G])
        ks.append(run.data["k"][layer][b, h:h + 1])
        vs.append(run.data["v"][layer][b, h:h + 1])
        lens.append(int(seq[b]))
    qr, _ = oracle.raw(torch.stack(qs))
    kr, _ = oracle.raw(torch.stack(ks))
    vr, _ = oracle.raw(torch.stack(vs))
    P = oracle_problem(w, len(pairs), run.T_cap)
    res = oracle.decode(P, qr, kr, vr, lens, given_idx=given_idx, given_n_sel=given_n_sel)
    res["seq_lens"] = lens
    return res


def near_tie(boundary) -> bool:
    a, b = float(boundary[0]), float(boundary[1])
    if not (math.isfinite(a) and math.isfinite(b)):
        return a == b and not math.isnan(a)   # e.g. two -inf scores
    return abs(a - b) <= NEAR_TIE_REL * max(abs(a), abs(b))


def check_selection(run: GpuCase, pairs: list[int], orc: dict, score_atol=None) -> list[int]:
    """Compare the GPU selection of the listed pairs with the oracle. Returns the indices (into
    ``pairs``) of near-tie pairs whose GPU selection may legitimately differ.

    ``score_atol`` (one per listed pair) switches the block scores to an absolute tolerance, for
    raw dot-product scores that may sit near zero; two boundary scores then tie when they are
    within twice that tolerance."""
    w = run.w
    idx = run.block_idx.view(-1, run.sizes.sel_cap).cpu().numpy()
    ns = run.n_sel.view(-1).cpu().numpy()
    sc = run.block_scores.view(-1, run.sizes.nb_cap).cpu().numpy().astype(np.float64)
    ties = []
    for i, pr in enumerate(pairs):
        T = orc["seq_lens"][i]
        nb = -(-T // w.block_size)
        # block scores
        want = orc["block_scores"][i]
        got = sc[pr]
        assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"pair {pr}: -inf pattern"
        fin = np.isfinite(want)
        if fin.any() and score_atol is None:
            err = np.abs(got[fin] - want[fin]) / np.maximum(np.abs(want[fin]), 1e-30)
            assert err.max() <= SCORE_RTOL, f"pair {pr}: block score rel err {err.max():.3g}"
        elif fin.any():
            err = np.abs(got[fin] - want[fin]).max()
            assert err <= score_atol[i], f"pair {pr}: block score abs err {err:.3g} > {score_atol[i]:.3g}"
        # indices
        n_o = int(orc["n_sel"][i])
        bd = orc["boundary"][i]
        if score_atol is None:
            tie = near_tie(bd)
        else:
            tie = (math.isfinite(bd[0]) and math.isfinite(bd[1]) and abs(bd[0] - bd[1]) <= 2 * score_atol[i]) \
                or (bd[0] == bd[1] and not math.isnan(bd[0]))
        if tie:
            ties.append(i)
            n_g = int(ns[pr])
            g = idx[pr, :n_g]
            assert n_g == n_o, f"pair {pr}: n_sel {n_g} vs {n_o}"
            assert np.all(np.diff(g) > 0) and (n_g == 0 or (g[0] >= 0 and g[-1] < nb))
            fixed = set(range(min(w.n_init, nb))) | set(range(max(nb - w.n_local, 0), nb))
            assert fixed <= set(g.tolist())
        else:
            assert int(ns[pr]) == n_o, f"pair {pr}: n_sel {ns[pr]} vs oracle {n_o}"
            assert idx[pr, :n_o].tolist() == orc["idx"][i, :n_o].tolist(), \
                f"pair {pr}: idx {idx[pr, :n_o].tolist()} vs oracle {orc['idx'][i, :n_o].tolist()}"
        assert np.all(idx[pr, n_o:] == -1), f"pair {pr}: padding"
        # the selection is exactly the top-k of the kernel's own block scores (ties: lower block)
        want_idx = topk_union_of(sc[pr, :nb].astype(np.float32), nb, w.n_init, w.n_local, w.top_k)
        assert idx[pr, :int(ns[pr])].tolist() == want_idx, \
            f"pair {pr}: selection is not the top-k of the returned block scores"
    return ties


def topk_union_of(scores: np.ndarray, nb: int, n_init: int, n_local: int, top_k: int) -> list[int]:
    """Init blocks, the top_k candidates by score (ties: lower block first) and the local blocks,
    ascending: the selection rule applied to given block scores."""
    init_end = min(n_init, nb)
    chi = max(nb - n_local, init_end)
    cand = np.arange(init_end, chi)
    kk = min(top_k, len(cand))
    order = cand[np.lexsort((cand, -scores[cand].astype(np.float64)))] if len(cand) else cand
    return list(range(init_end)) + sorted(order[:kk].tolist()) + list(range(chi, nb))


def check_output(run: GpuCase, pairs: list[int], orc: dict, layer=0, skip=()):
    w = run.w
    G, Hkv = w.group, w.num_kv_heads
    out = run.out[layer].float().cpu().numpy().astype(np.float64)
    lse = run.lse[layer].cpu().numpy().astype(np.float64)
    tol, ltol = OUT_ATOL[w.dtype], LSE_ATOL[w.dtype]
    for i, pr in enumerate(pairs):
        if i in skip:
            continue
        b, h = divmod(pr, Hkv)
        got = out[b, h * G:(h + 1) * G]
        err = np.abs(got - orc["out"][i]).max()
        assert err <= tol, f"pair {pr}: output max-abs err {err:.3g} > {tol}"
        gl, ol = lse[b, h * G:(h + 1) * G], orc["lse"][i]
        assert np.array_equal(np.isneginf(gl), np.isneginf(ol)), f"pair {pr}: lse -inf pattern"
        fin = np.isfinite(ol)
        if fin.any():
            lerr = np.abs(gl[fin] - ol[fin]).max()
            assert lerr <= ltol, f"pair {pr}: lse err {lerr:.3g} > {ltol}"


def oracle_idx_tensor(run: GpuCase, pairs: list[int], orc: dict):
    """GPU block_idx/n_sel with the listed pairs' rows replaced by the oracle's selection."""
    idx = run.block_idx.clone()
    ns = run.n_sel.clone()
    fi, fn = idx.view(-1, run.sizes.sel_cap), ns.view(-1)
    for i, pr in enumerate(pairs):
        fi[pr] = torch.from_numpy(orc["idx"][i]).to(fi.device)
        fn[pr] = int(orc["n_sel"][i])
    return idx, ns


def forecast_check(run: GpuCase, pairs: list[int], f: torch.Tensor):
    """Forecast-indexer selection on the GPU (already run into run.block_idx / block_scores) and
    the decode of q over it, vs the oracle on the sampled pairs. Block scores are raw fp32 dot
    products f . K~_j: their tolerance is 1e-5 * |f|_1 * max|K| of the pair (fp32 accumulation of
    d exact products, each at most |f_t| max|K|)."""
    w = run.w
    G, Hkv = w.group, w.num_kv_heads
    seq = run.data["seq_lens"].cpu()
    qs, ks, vs, fs, lens, atol = [], [], [], [], [], []
    for pr in pairs:
        b, h = divmod(pr, Hkv)
        qs.append(run.q[0][b, h * G:(h + 1) * G])
        ks.append(run.data["k"][0][b, h:h + 1])
        vs.append(run.data["v"][0][b, h:h + 1])
        fs.append(f[b, h:h + 1])
        lens.append(int(seq[b]))
        kmax = float(run.data["k"][0][b, h, :lens[-1]].float().abs().max()) if lens[-1] else 0.0
        atol.append(1e-5 * float(f[b, h].float().abs().sum()) * kmax + 1e-30)
    P = oracle_problem(w, len(pairs), run.T_cap)
    orc = oracle.decode_forecast(P, oracle.raw(torch.stack(fs))[0], oracle.raw(torch.stack(qs))[0],
                                 oracle.raw(torch.stack(ks))[0], oracle.raw(torch.stack(vs))[0], lens)
    orc["seq_lens"] = lens
    ties = check_selection(run, pairs, orc, score_atol=np.array(atol))
    check_output(run, pairs, orc, 0, skip=set(ties))
    if ties:
        idx, ns = oracle_idx_tensor(run, pairs, orc)
        run.decode(0, idx, ns)
        check_output(run, [pairs[i] for i in ties], {k: (v[ties] if isinstance(v, np.ndarray) else v)
                                                     for k, v in orc.items()}, 0)
    return orc, ties


def full_check(run: GpuCase, pairs: list[int], layer=0):
    """Select + decode on the GPU vs the oracle for the sampled pairs, with the near-tie rule."""
    orc = oracle_on_pairs(run, pairs, layer)
    ties = check_selection(run, pairs, orc)
    check_output(run, pairs, orc, layer, skip=set(ties))
    if ties:
        idx, ns = oracle_idx_tensor(run, pairs, orc)
        run.decode(layer, idx, ns)
        check_output(run, [pairs[i] for i in ties], {k: (v[ties] if isinstance(v, np.ndarray) else v)
                                                     for k, v in orc.items()}, layer)
    return orc, ties
