"""CLSA token-level shared index (bsa_decode_step_clsa) vs the CPU oracle, through the C ABI.

Layer 0's base selector scores every token (softmax per head over the tokens, summed over the
group), the block configuration's token budget picks the tokens (first and last tokens always, the
rest by score, ties to the lower token), and every layer attends exactly those tokens. The token
list is compared with the oracle's: identical, or, when the oracle's boundary scores are within
1e-3 relative, every token scoring clearly above the boundary taken and every token clearly below
it left out. Each layer's output is compared with the oracle attending the GPU's token list.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_compressed_b200 as bsa
import oracle
from block_sparse_attention_compressed_b200.workloads import WORKLOADS, generate
from gpu_helpers import LSE_ATOL, OUT_ATOL, near_tie, oracle_problem, params_for, sample_pairs

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["shared-index-4x64k-b8"].replace(layers=3)

CASES = {
    "g4-d128": (BASE.replace(name="x", batch=2, num_kv_heads=2, num_q_heads=8, seq_len=3000, n_local=1,
                             top_k=4, needles=3), None),
    "g1": (BASE.replace(name="x", batch=1, num_kv_heads=3, num_q_heads=3, seq_len=2500, top_k=5, needles=2), None),
    "g8-d64": (BASE.replace(name="x", batch=1, num_kv_heads=2, num_q_heads=16, head_dim=64, seq_len=4000,
                            top_k=6, needles=2), None),
    "ragged": (BASE.replace(name="x", batch=4, num_kv_heads=2, num_q_heads=8, seq_len=5000, top_k=6, needles=2),
               [5000, 700, 64, 0]),
    "budget-covers-all": (BASE.replace(name="x", batch=1, num_kv_heads=1, num_q_heads=4, seq_len=900, top_k=16,
                                       needles=0), None),
}


class Clsa:
    def __init__(self, w, lens):
        self.w = w
        self.data = generate(w, device="cuda")
        if lens is not None:
            self.data["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device="cuda")
        self.T_cap = self.data["seq_cap"]
        self.p = params_for(w, self.T_cap)
        B, Hkv, Hq, d = w.batch, w.num_kv_heads, w.num_q_heads, w.head_dim
        self.tok_cap = (w.n_init + w.n_local + w.top_k) * w.block_size
        self.ws = bsa.alloc_clsa_workspace(self.p)
        self.idx = torch.full((B, Hkv, self.tok_cap), -7, dtype=torch.int32, device="cuda")
        self.nt = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
        self.out = [torch.full((B, Hq, d), 77.0, dtype=torch.bfloat16, device="cuda") for _ in range(w.layers)]
        self.lse = [torch.full((B, Hq), 77.0, dtype=torch.float32, device="cuda") for _ in range(w.layers)]

    def run(self, stream=None):
        L = self.w.layers
        bsa.bsa_decode_step_clsa(self.p, [self.data["q"][l] for l in range(L)], self.data["k"], self.data["v"],
                                 self.data["seq_lens"], self.idx, self.nt, self.out, self.lse, self.ws, stream=stream)

    def pair_arrays(self, pairs, layer):
        w = self.w
        G, Hkv = w.group, w.num_kv_heads
        seq = self.data["seq_lens"].cpu()
        qs, ks, vs, lens = [], [], [], []
        for pr in pairs:
            b, h = divmod(pr, Hkv)
            qs.append(self.data["q"][layer][b, h * G:(h + 1) * G])
            ks.append(self.data["k"][layer][b, h:h + 1])
            vs.append(self.data["v"][layer][b, h:h + 1])
            lens.append(int(seq[b]))
        return (oracle.raw(torch.stack(qs))[0], oracle.raw(torch.stack(ks))[0], oracle.raw(torch.stack(vs))[0],
                lens)


def check_clsa(c, pairs):
    w = c.w
    P = oracle_problem(w, len(pairs), c.T_cap)
    q0, k0, _, lens = c.pair_arrays(pairs, 0)
    orc = oracle.token_select(P, q0, k0, lens)
    idx = c.idx.view(-1, c.tok_cap).cpu().numpy()
    nt = c.nt.view(-1).cpu().numpy()
    for i, pr in enumerate(pairs):
        T = lens[i]
        n_o = int(orc["n_sel"][i])
        g = idx[pr, :int(nt[pr])]
        assert int(nt[pr]) == n_o, f"pair {pr}: {nt[pr]} tokens vs {n_o}"
        assert (idx[pr, n_o:] == -1).all(), f"pair {pr}: padding"
        assert np.all(np.diff(g) > 0) and (n_o == 0 or (g[0] >= 0 and g[-1] < T)), f"pair {pr}: not ascending"
        if g.tolist() == orc["idx"][i, :n_o].tolist():
            continue
        bd = orc["boundary"][i]
        assert near_tie(bd), f"pair {pr}: token list differs from the oracle's away from a near tie"
        S = orc["scores"][i, :T]
        init_end = min(w.n_init * w.block_size, T)
        chi = max(T - w.n_local * w.block_size, init_end)
        taken = set(g.tolist())
        assert set(range(init_end)) <= taken and set(range(chi, T)) <= taken
        hi, lo = max(bd) * (1 + 1e-3), min(bd) * (1 - 1e-3)
        for t in range(init_end, chi):
            if S[t] > hi:
                assert t in taken, f"pair {pr}: token {t} scores above the boundary but is not taken"
            elif S[t] < lo:
                assert t not in taken, f"pair {pr}: token {t} scores below the boundary but is taken"
    # every layer's output: the oracle attending the GPU's token list
    P1 = oracle_problem(w, len(pairs), c.T_cap)
    P1.top_k = c.tok_cap
    P1.block_size, P1.n_init, P1.n_local = 1, 0, 0
    gi = np.stack([idx[pr] for pr in pairs])
    gn = np.array([nt[pr] for pr in pairs], dtype=np.int32)
    G, Hkv = w.group, w.num_kv_heads
    for layer in range(w.layers):
        q, k, v, lens = c.pair_arrays(pairs, layer)
        ro = oracle.attend_pairs(P1, q, k, v, lens, gi, gn)
        out = c.out[layer].float().cpu().numpy().astype(np.float64)
        lse = c.lse[layer].cpu().numpy().astype(np.float64)
        for i, pr in enumerate(pairs):
            b, h = divmod(pr, Hkv)
            err = np.abs(out[b, h * G:(h + 1) * G] - ro["out"][i]).max()
            assert err <= OUT_ATOL["bf16"], f"layer {layer} pair {pr}: output err {err:.3g}"
            gl, ol = lse[b, h * G:(h + 1) * G], ro["lse"][i]
            assert np.array_equal(np.isneginf(gl), np.isneginf(ol))
            fin = np.isfinite(ol)
            if fin.any():
                assert np.abs(gl[fin] - ol[fin]).max() <= LSE_ATOL["bf16"], f"layer {layer} pair {pr}: lse"


@pytest.mark.parametrize("case", sorted(CASES))
def test_clsa_matches_oracle(case, cuda_device):
    w, lens = CASES[case]
    c = Clsa(w, lens)
    c.run()
    assert bsa.bsa_read_device_error(c.ws) == 0
    check_clsa(c, sample_pairs(w, 8))


def test_clsa_graph_replay_and_unsupported(cuda_device):
    """Replays of a captured CLSA step give the eager results bit for bit; caches longer than
    about 50K tokens and fp32 are refused."""
    w, lens = CASES["g4-d128"]
    c = Clsa(w, lens)
    c.run()
    torch.cuda.synchronize()
    ref = (c.idx.clone(), [o.clone() for o in c.out])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(2):
                c.run(stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ref[0], c.idx) and all(torch.equal(a, b) for a, b in zip(ref[1], c.out))
    assert bsa.bsa_clsa_workspace_size(params_for(w, 60000)) == 0
    assert bsa.bsa_clsa_workspace_size(params_for(w.replace(dtype="f32"), 4096)) == 0


@pytest.mark.slow
def test_full_clsa_workload(cuda_device):
    """The bench's CLSA workload (4 layers, 8 sequences of 32K tokens) on sampled pairs."""
    w = WORKLOADS["clsa-4x32k-b8"]
    c = Clsa(w, None)
    c.run()
    assert bsa.bsa_read_device_error(c.ws) == 0
    check_clsa(c, sample_pairs(w, 3, seed=4))
