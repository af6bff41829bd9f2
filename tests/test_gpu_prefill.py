"""Block-sparse prefill (bsa_prefill, bsa_prefill_attend) vs the CPU oracle, through the C ABI.

The last `chunk` positions of every sequence are queried; every query tile (the chunk's positions
inside one block) of every (batch, kv head) pair selects its blocks from the windows complete before
its block (the scoring on the tensor cores, tcgen05), and each query attends its tile's blocks
causally. Selections are compared tile by tile (identical, except tiles whose oracle k-th and
(k+1)-th block scores are within 1e-3 relative: those are checked for validity); outputs are
compared with the oracle attending the oracle's selection (bsa_prefill_attend), and bsa_prefill's
own outputs on the tiles whose selection matched.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_compressed_b200 as bsa
import oracle
from block_sparse_attention_compressed_b200.workloads import WORKLOADS, generate
from gpu_helpers import LSE_ATOL, OUT_ATOL, near_tie, oracle_problem, params_for, sample_pairs

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["gqa4-bf16-32k-b1"]

CASES = {
    # name: (workload, seq_lens, chunk)
    "g4-mid-block": (BASE.replace(name="x", batch=2, num_kv_heads=2, num_q_heads=8, seq_len=3000, top_k=6,
                                  needles=3), [3000, 2517], 300),
    "g2": (BASE.replace(name="x", batch=1, num_kv_heads=3, num_q_heads=6, seq_len=2000, top_k=5, needles=2),
           None, 640),
    "whole-sequence": (BASE.replace(name="x", batch=1, num_kv_heads=1, num_q_heads=4, seq_len=700, top_k=4,
                                    needles=0), None, 700),
    "aligned": (BASE.replace(name="x", batch=1, num_kv_heads=2, num_q_heads=8, seq_len=4096, top_k=8, needles=2),
                None, 1024),
    "short-chunk": (BASE.replace(name="x", batch=3, num_kv_heads=2, num_q_heads=8, seq_len=2600, top_k=7,
                                 needles=2), [2600, 1900, 65], 17),
    "topk-covers-all": (BASE.replace(name="x", batch=1, num_kv_heads=1, num_q_heads=4, seq_len=900, top_k=64,
                                     needles=0), None, 400),
    "long-context": (BASE.replace(name="x", batch=1, num_kv_heads=2, num_q_heads=8, seq_len=20000, top_k=16,
                                  needles=4), None, 256),
}


class Prefill:
    def __init__(self, w, lens, chunk, seed=7):
        self.w, self.chunk = w, chunk
        self.data = generate(w, device="cuda")
        if lens is not None:
            self.data["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device="cuda")
        self.T_cap = self.data["seq_cap"]
        self.p = params_for(w, self.T_cap)
        s = bsa.bsa_get_sizes(self.p)
        self.sizes = s
        B, Hkv, Hq, d = w.batch, w.num_kv_heads, w.num_q_heads, w.head_dim
        g = torch.Generator(device="cuda").manual_seed(seed)
        self.q = torch.randn(B, chunk, Hq, d, generator=g, device="cuda").to(torch.bfloat16)
        self.ck = torch.zeros(B, Hkv, s.nc_cap, d, dtype=torch.bfloat16, device="cuda")
        bsa.bsa_compress_keys(self.p, self.data["k"][0], self.data["seq_lens"], self.ck)
        self.ws = bsa.alloc_workspace(self.p)
        bsa.bsa_workspace_init(self.p, self.ws)
        self.tiles = bsa.bsa_prefill_tiles(chunk, w.block_size)
        self.idx = torch.full((B, Hkv, self.tiles, s.sel_cap), -7, dtype=torch.int32, device="cuda")
        self.ns = torch.full((B, Hkv, self.tiles), -7, dtype=torch.int32, device="cuda")
        self.out = torch.full((B, chunk, Hq, d), 77.0, dtype=torch.bfloat16, device="cuda")
        self.lse = torch.full((B, chunk, Hq), 77.0, dtype=torch.float32, device="cuda")

    def run(self):
        bsa.bsa_prefill(self.p, self.chunk, self.q, self.data["k"][0], self.data["v"][0], self.ck,
                        self.data["seq_lens"], self.idx, self.ns, self.out, self.lse, self.ws)

    def attend(self, idx, ns):
        bsa.bsa_prefill_attend(self.p, self.chunk, self.q, self.data["k"][0], self.data["v"][0],
                               self.data["seq_lens"], idx, ns, self.out, self.lse, self.ws)

    def oracle(self, pairs):
        w = self.w
        G, Hkv = w.group, w.num_kv_heads
        seq = self.data["seq_lens"].cpu()
        qs, ks, vs, lens = [], [], [], []
        for pr in pairs:
            b, h = divmod(pr, Hkv)
            qs.append(self.q[b, :, h * G:(h + 1) * G])
            ks.append(self.data["k"][0][b, h:h + 1])
            vs.append(self.data["v"][0][b, h:h + 1])
            lens.append(int(seq[b]))
        P = oracle_problem(w, len(pairs), self.T_cap)
        res = oracle.prefill(P, oracle.raw(torch.stack(qs))[0], oracle.raw(torch.stack(ks))[0],
                             oracle.raw(torch.stack(vs))[0], lens, self.chunk)
        res["seq_lens"] = lens
        return res


def _check_selection(pf, pairs, orc):
    """Tile selections vs the oracle; returns the (pair index, tile) pairs whose selection matched."""
    w = pf.w
    idx = pf.idx.view(-1, pf.tiles, pf.sizes.sel_cap).cpu().numpy()
    ns = pf.ns.view(-1, pf.tiles).cpu().numpy()
    matched = set()
    for i, pr in enumerate(pairs):
        T = orc["seq_lens"][i]
        r_lo, r_hi = (T - pf.chunk) // w.block_size, (T - 1) // w.block_size
        for ti in range(pf.tiles):
            n_o = int(orc["n_sel"][i, ti])
            if ti > r_hi - r_lo:
                assert ns[pr, ti] == 0 and (idx[pr, ti] == -1).all(), f"pair {pr} tile {ti}: past the chunk"
                continue
            nb = r_lo + ti + 1
            g = idx[pr, ti, :int(ns[pr, ti])]
            assert int(ns[pr, ti]) == n_o, f"pair {pr} tile {ti}: n_sel {ns[pr, ti]} vs {n_o}"
            assert (idx[pr, ti, n_o:] == -1).all(), f"pair {pr} tile {ti}: padding"
            if near_tie(orc["boundary"][i, ti]):
                assert np.all(np.diff(g) > 0) and (n_o == 0 or (g[0] >= 0 and g[-1] < nb))
                fixed = set(range(min(w.n_init, nb))) | set(range(max(nb - w.n_local, min(w.n_init, nb)), nb))
                assert fixed <= set(g.tolist())
            else:
                assert g.tolist() == orc["idx"][i, ti, :n_o].tolist(), \
                    f"pair {pr} tile {ti}: {g.tolist()} vs oracle {orc['idx'][i, ti, :n_o].tolist()}"
            if g.tolist() == orc["idx"][i, ti, :n_o].tolist():
                matched.add((i, ti))
    return matched


def _check_output(pf, pairs, orc, only=None):
    """out / lse of the listed pairs vs the oracle (positions of the matched tiles when `only`)."""
    w = pf.w
    G, Hkv = w.group, w.num_kv_heads
    out = pf.out.float().cpu().numpy().astype(np.float64)
    lse = pf.lse.cpu().numpy().astype(np.float64)
    tol, ltol = OUT_ATOL["bf16"], LSE_ATOL["bf16"]
    for i, pr in enumerate(pairs):
        b, h = divmod(pr, Hkv)
        T = orc["seq_lens"][i]
        t0 = T - pf.chunk
        for c in range(pf.chunk):
            ti = (t0 + c) // w.block_size - t0 // w.block_size
            if only is not None and (i, ti) not in only:
                continue
            err = np.abs(out[b, c, h * G:(h + 1) * G] - orc["out"][i, c]).max()
            assert err <= tol, f"pair {pr} position {t0 + c}: output err {err:.3g}"
            lerr = np.abs(lse[b, c, h * G:(h + 1) * G] - orc["lse"][i, c]).max()
            assert lerr <= ltol, f"pair {pr} position {t0 + c}: lse err {lerr:.3g}"


def _oracle_idx(pf, pairs, orc):
    idx, ns = pf.idx.clone(), pf.ns.clone()
    fi, fn = idx.view(-1, pf.tiles, pf.sizes.sel_cap), ns.view(-1, pf.tiles)
    for i, pr in enumerate(pairs):
        fi[pr] = torch.from_numpy(orc["idx"][i]).to(fi.device)
        fn[pr] = torch.from_numpy(orc["n_sel"][i]).to(fn.device)
    return idx, ns


@pytest.mark.parametrize("case", sorted(CASES))
def test_prefill_matches_oracle(case, cuda_device):
    w, lens, chunk = CASES[case]
    pf = Prefill(w, lens, chunk)
    pf.run()
    assert bsa.bsa_read_device_error(pf.ws) == 0
    pairs = sample_pairs(w, 6)
    orc = pf.oracle(pairs)
    matched = _check_selection(pf, pairs, orc)
    _check_output(pf, pairs, orc, only=matched)
    idx, ns = _oracle_idx(pf, pairs, orc)
    pf.attend(idx, ns)
    assert bsa.bsa_read_device_error(pf.ws) == 0
    _check_output(pf, pairs, orc)


def test_prefill_repeats_and_refuses_unsupported(cuda_device):
    """Queued prefills give the first one's results bit for bit; eight heads per group are refused."""
    w, lens, chunk = CASES["g4-mid-block"]
    pf = Prefill(w, lens, chunk)
    pf.run()
    torch.cuda.synchronize()
    first = (pf.idx.clone(), pf.out.clone(), pf.lse.clone())
    for _ in range(5):
        pf.run()
    torch.cuda.synchronize()
    assert torch.equal(first[0], pf.idx) and torch.equal(first[1], pf.out) and torch.equal(first[2], pf.lse)
    w8 = w.replace(num_q_heads=16)
    pf8 = Prefill(w8, lens, chunk)
    with pytest.raises(bsa.BsaError) as e:
        pf8.run()
    assert e.value.status == bsa.BSA_ERR_UNSUPPORTED


@pytest.mark.slow
def test_full_prefill_workload(cuda_device):
    """The bench's prefill workload (4 sequences of 32K tokens, the last 4096 queried) on sampled pairs."""
    w = WORKLOADS["prefill-bf16-32k-b4"]
    pf = Prefill(w, None, w.prefill_chunk, seed=w.seed)
    pf.run()
    assert bsa.bsa_read_device_error(pf.ws) == 0
    pairs = sample_pairs(w, 2, seed=3)
    orc = pf.oracle(pairs)
    matched = _check_selection(pf, pairs, orc)
    _check_output(pf, pairs, orc, only=matched)
