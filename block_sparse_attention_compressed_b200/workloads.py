"""Seeded synthetic decode workloads.

These generators produce the inputs of the decode step -- q, the K/V caches, the sequence lengths
and, for the growing-cache workload, the per-step new tokens -- for both the CUDA path and the CPU
oracle. They hold none of the method's arithmetic: no compression, scoring, selection or
attention happens here.

Recipe (every workload):
  * q, K, V ~ N(0, 1) drawn with ``torch.randn`` from a ``torch.Generator`` seeded with
    ``seed + 100 * layer`` on the target device, in fp32, then cast to the element type.
  * Cache rows at or past the sequence length are zero.
  * "Needle" blocks: per (batch, kv head), ``needles`` distinct 64-token blocks drawn uniformly
    (numpy ``default_rng(seed)``, so the positions do not depend on the device) from the blocks that
    can be top-k candidates, i.e. not init and not local. Every key of a needle block is shifted by
    ``2.0 * qbar / ||qbar||`` where ``qbar`` is the mean of the group's query vectors, so the block
    is attractive to that group and selection is not trivial. With several layers the positions are
    the same in every layer and each layer uses its own ``qbar``.
  * The growing-cache workload pre-draws, per step, new q, k and v rows from the same generator.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    seq_len: int            # context length T (tokens already in the cache, incl. the current one)
    dtype: str              # "f32" or "bf16"
    n_init: int
    n_local: int
    top_k: int
    needles: int = 0
    seed: int = 0
    layers: int = 1         # >1: several caches that share one selection
    append_steps: int = 0   # >0: every step appends one token per sequence first
    cmp_kernel: int = 32
    cmp_stride: int = 16
    block_size: int = 64
    needle_shift: float = 2.0
    forecast: bool = False  # select with one Forecast vector per GQA group (f = the group's mean q)
    lookahead: bool = False  # (two layers, forecast) layer 0 attends given blocks and selects layer 1's
    prefill_chunk: int = 0   # >0: block-sparse prefill of the last prefill_chunk positions
    token_index: bool = False  # (several layers) CLSA: layer 0's token-level index, reused by every layer
    anchors: tuple = (0,)   # multi-layer: layers that select; the others reuse the last anchor's

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The workloads: one small parity case, eight decode throughput cases and one prefill case.
WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny-f32-2k", batch=1, num_q_heads=1, num_kv_heads=1, head_dim=64, seq_len=2048,
                 dtype="f32", n_init=1, n_local=2, top_k=4, needles=0, seed=1001),
        Workload("gqa4-bf16-32k-b1", batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=32768, dtype="bf16", n_init=1, n_local=2, top_k=32, needles=8, seed=1002),
        Workload("gqa4-bf16-128k-b16", batch=16, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=131072, dtype="bf16", n_init=1, n_local=4, top_k=64, needles=16,
                 seed=1003),
        Workload("shared-index-4x64k-b8", batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=65536, dtype="bf16", n_init=1, n_local=2, top_k=48, needles=8, seed=1004,
                 layers=4),
        Workload("append-bf16-16k-b128", batch=128, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=16384, dtype="bf16", n_init=1, n_local=2, top_k=16, needles=4, seed=1005,
                 append_steps=64),
        Workload("forecast-bf16-128k-b16", batch=16, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=131072, dtype="bf16", n_init=1, n_local=4, top_k=64, needles=16,
                 seed=1006, forecast=True),
        Workload("anchors-2of4-64k-b8", batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=65536, dtype="bf16", n_init=1, n_local=2, top_k=48, needles=8, seed=1007,
                 layers=4, anchors=(0, 2)),
        Workload("lookahead-bf16-128k-b16", batch=16, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=131072, dtype="bf16", n_init=1, n_local=4, top_k=64, needles=16,
                 seed=1008, layers=2, forecast=True, lookahead=True),
        Workload("prefill-bf16-32k-b4", batch=4, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=32768, dtype="bf16", n_init=1, n_local=4, top_k=64, needles=8, seed=1009,
                 prefill_chunk=4096),
        Workload("clsa-4x32k-b8", batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 seq_len=32768, dtype="bf16", n_init=1, n_local=2, top_k=48, needles=8, seed=1010,
                 layers=4, token_index=True),
    ]
}
DEFAULT_WORKLOAD = "gqa4-bf16-128k-b16"


def _num_blocks(T: int, bs: int) -> int:
    return -(-T // bs)


def needle_blocks(w: Workload) -> np.ndarray:
    """[B][Hkv][needles] block indices, drawn from the non-init, non-local blocks."""
    nb = _num_blocks(w.seq_len, w.block_size)
    lo, hi = w.n_init, nb - w.n_local
    n = min(w.needles, max(hi - lo, 0))
    rng = np.random.default_rng(w.seed)
    out = np.zeros((w.batch, w.num_kv_heads, n), dtype=np.int64)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            out[b, h] = np.sort(rng.choice(np.arange(lo, hi), size=n, replace=False))
    return out


def _plant_needles(k32: torch.Tensor, q32: torch.Tensor, blocks: np.ndarray, w: Workload, T: int):
    """k32: [Hkv][T_cap][d] fp32 of one sequence; q32: [Hq][d] fp32 of the same sequence."""
    G = w.group
    qbar = q32.view(w.num_kv_heads, G, w.head_dim).mean(dim=1)             # [Hkv][d]
    u = qbar / qbar.norm(dim=-1, keepdim=True)
    for h in range(w.num_kv_heads):
        for blk in blocks[h].tolist():
            lo, hi = blk * w.block_size, min((blk + 1) * w.block_size, T)
            k32[h, lo:hi] += w.needle_shift * u[h]


def generate(w: Workload, device="cpu", seq_cap: int | None = None, steps: int | None = None,
             layers: list[int] | None = None) -> dict:
    """Materialise a workload on ``device``.

    Returns a dict with
      q        [L][B][Hq][d]          queries of the (first) decode step, per layer
      k, v     [L][B][Hkv][T_cap][d]  caches, zero at rows >= seq_len
      seq_lens [B] int32              (on ``device``)
      needles  [B][Hkv][n] numpy      needle block positions
      f        [B][Hkv][d]            Forecast vectors (forecast workloads): the mean of each
                                      group's query vectors of the first layer, in the cache type
                                      (lookahead: of the second layer, the one f selects for)
    and, when ``steps`` > 0 (growing-cache workload):
      q_steps  [steps][B][Hq][d], k_new / v_new [steps][B][Hkv][d]
    ``seq_cap`` is the cache capacity T_cap (default: seq_len + steps).
    """
    steps = w.append_steps if steps is None else steps
    T = w.seq_len
    T_cap = seq_cap if seq_cap is not None else T + max(steps, 0)
    if T_cap < T:
        raise ValueError("seq_cap must be >= seq_len")
    dt = w.torch_dtype
    layer_ids = list(range(w.layers)) if layers is None else list(layers)
    blocks = needle_blocks(w)
    out_q, out_k, out_v = [], [], []
    extra = {}
    for layer in layer_ids:
        g = torch.Generator(device=device)
        g.manual_seed(w.seed + 100 * layer)
        q32 = torch.randn(w.batch, w.num_q_heads, w.head_dim, generator=g, device=device)
        k = torch.zeros(w.batch, w.num_kv_heads, T_cap, w.head_dim, dtype=dt, device=device)
        v = torch.zeros_like(k)
        for b in range(w.batch):
            k32 = torch.randn(w.num_kv_heads, T, w.head_dim, generator=g, device=device)
            if w.needles:
                _plant_needles(k32, q32[b], blocks[b], w, T)
            k[b, :, :T] = k32.to(dt)
            del k32
            v[b, :, :T] = torch.randn(w.num_kv_heads, T, w.head_dim, generator=g,
                                      device=device).to(dt)
        out_q.append(q32.to(dt))
        out_k.append(k)
        out_v.append(v)
        if steps and layer == layer_ids[0]:
            extra["q_steps"] = torch.randn(steps, w.batch, w.num_q_heads, w.head_dim, generator=g,
                                           device=device).to(dt)
            extra["k_new"] = torch.randn(steps, w.batch, w.num_kv_heads, w.head_dim, generator=g,
                                         device=device).to(dt)
            extra["v_new"] = torch.randn(steps, w.batch, w.num_kv_heads, w.head_dim, generator=g,
                                         device=device).to(dt)
    res = dict(
        q=torch.stack(out_q) if len(out_q) > 1 else out_q[0].unsqueeze(0),
        k=out_k, v=out_v,
        seq_lens=torch.full((w.batch,), T, dtype=torch.int32, device=device),
        needles=blocks, seq_cap=T_cap,
    )
    if w.forecast:
        qf = res["q"][1 if w.lookahead and len(out_q) > 1 else 0]
        q0 = qf.float().view(w.batch, w.num_kv_heads, w.group, w.head_dim)
        res["f"] = q0.mean(dim=2).to(dt).contiguous()
    res.update(extra)
    return res


def prefill_flops(w: Workload) -> dict:
    """FLOPs of one block-sparse prefill of the last ``prefill_chunk`` positions (every sequence at
    seq_len): the scoring of every (position, head) against the windows complete before its tile's
    block (2 d per product), and the attention of every (position, head) over its tile's selected
    tokens up to itself (4 d per key: the score and the weighted value)."""
    C, T, d, BS = w.prefill_chunk, w.seq_len, w.head_dim, w.block_size
    heads = w.batch * w.num_q_heads
    score = attn = 0
    for pos in range(T - C, T):
        r = pos // BS
        start = BS * r
        nc = 0 if start < w.cmp_kernel else (start - w.cmp_kernel) // w.cmp_stride + 1
        score += nc
        nsel = min(w.n_init + w.n_local + w.top_k, r + 1)
        keys = BS * (nsel - 1) + (pos - start + 1) if w.n_local > 0 else BS * nsel
        attn += keys
    return dict(score=2 * d * heads * score, attend=4 * d * heads * attn,
                total=2 * d * heads * score + 4 * d * heads * attn)


def algorithmic_bytes(w: Workload, T: int | None = None) -> dict:
    """Minimum bytes one decode step moves: the compressed keys of the scored layer, the K and V
    rows of the selected blocks of every layer, q read and the output written, and for the
    growing-cache workload the appended rows (new k/v read and written, plus one compressed-key
    window of l rows read and one row written every s steps, amortised per step)."""
    T = w.seq_len if T is None else T
    e, d = w.elem_bytes, w.head_dim
    pairs = w.batch * w.num_kv_heads
    nc = 0 if T < w.cmp_kernel else (T - w.cmp_kernel) // w.cmp_stride + 1
    nb = _num_blocks(T, w.block_size)
    n_sel = min(w.n_init + w.n_local + w.top_k, nb)
    sel_tokens = n_sel * w.block_size
    if w.n_local > 0 or n_sel == nb:          # the last (possibly partial) block is selected
        sel_tokens -= nb * w.block_size - T
    ck = pairs * nc * d * e * len(w.anchors)   # every anchor layer scores its compressed keys
    attended = 1 if w.lookahead else w.layers  # lookahead: one layer attends, the next one is scored
    if w.token_index:
        # CLSA: the index layer's every key is scored; each layer reads the taken tokens' rows
        ck = pairs * T * d * e
        sel_tokens = min((w.n_init + w.n_local + w.top_k) * w.block_size, T)
    kv = attended * pairs * sel_tokens * d * e * 2
    qo = attended * w.batch * w.num_q_heads * d * e * 2
    app = 0
    if w.append_steps:
        app = pairs * d * e * 4 + pairs * (w.cmp_kernel + 1) * d * e / w.cmp_stride
    fv = pairs * d * e if w.forecast else 0   # the Forecast vectors read by the scoring
    return dict(ck=ck, kv=kv, qo=qo, append=app, f=fv, total=ck + kv + qo + app + fv)
