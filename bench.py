"""Decode-step benchmark of the B200 block-sparse compressed-key attention library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bsa|reference] [--workload NAME]

One step = one decode step of the workload: group scoring of q against the compressed keys,
block reduction, top-k + init/local selection and sparse attention over the selected blocks, for
all sequences of the batch (shared-index workload: selection on layer 0, attention on every layer;
growing-cache workload: the token append with its compressed-key update first).

Prints one JSON line. ``value`` is decode steps/s over all ranks (weak scaling: every rank runs its
own copy of the workload on its own GPU, no collective on the data path), device-timed with CUDA
events between barriers + synchronizes, max over ranks. ``e2e`` is the same metric through the
Python binding, with every step's inputs (each layer's q; the new k/v rows when the cache grows)
copied in from pinned host memory and its outputs (every layer) copied back. The copies are
double-buffered on two copy streams, so a step's transfers overlap its neighbours' compute.
``roofline`` is for the largest single launch of the step (the fused step kernel where
bsa_decode_step runs one, else the sparse attention with its combine), from a second, identical pass
that brackets every library call with CUDA events; ``hbm_target`` is the whole step's algorithmic
bytes over 8 TB/s against the 0.70 target. ``cpu_baseline`` (rank 0, one GPU only) and ``--impl
reference`` time the CPU oracle's decode step (keys compressed beforehand, as at decode time) on a
bounded sample of the same workload, on all host cores and on one.

With ``--gpus N`` and no WORLD_SIZE in the environment, the script starts the N ranks itself
(torch.distributed.run on 127.0.0.1); under a launcher it checks that WORLD_SIZE is N.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse decode steps/s & achieved HBM GB/s (select+attn) at 128K ctx"
# the library kernel behind each single-launch phase of a step, by dtype
KERNEL_OF_PHASE = {"step": {"bf16": "step_kernel"},
                   "prefill": {"bf16": "prefill_select_kernel+prefill_attend_kernel"},
                   "clsa": {"bf16": "score_tma_kernel+token_topk_kernel+token_decode_kernel"},
                   "decode": {"bf16": "decode_tma_kernel+combine_kernel", "f32": "decode_f32_kernel"},
                   "append": {"bf16": "append_kernel", "f32": "append_kernel"},
                   "select": {"bf16": "score_tma_kernel+select_kernel",
                              "f32": "score_f32_kernel+select_kernel"}}
TARGET_FRAC_OF_8TBS = 0.70  # of 8 TB/s, for the fused select + sparse attention at 128K
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="bsa", choices=["bsa", "reference"])
    ap.add_argument("--workload", default=None)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (small cases for profiling only)")
    ap.add_argument("--no-graph", action="store_true", help="launch steps directly (no CUDA graph)")
    ap.add_argument("--path", default="auto", choices=["auto", "fused", "chained"],
                    help="single-layer steps: bsa_decode_step's own choice, the fused one-kernel step "
                         "(bsa_decode_step_fused), or the chained selection and attention kernels")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


# ------------------------------------------------------------------------------------ distributed
def dist_init(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local) if backend == "nccl" else None)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a host float over ranks (timing only; not on the data path)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# -------------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.text = ""

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.text, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.text, _ = self.proc.communicate()

    def summary(self) -> dict:
        rows = []
        for row in csv.reader(io.StringIO(self.text or "")):
            if not row or row[0].strip() == "index":
                continue
            rows.append([c.strip() for c in row])
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(s):
            m = re.match(r"([\d.]+)", s)
            return float(m.group(1)) if m else None

        sm = [num(r[1]) for r in rows if len(r) > 1 and num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if len(r) > 2 and num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if len(r) > 5 + i and r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        loaded = [x for x in sm if mx and x > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------------- workload run
class Bench:
    def __init__(self, w, device, seed_offset: int, steps_total: int, path: str = "auto"):
        import torch
        import block_sparse_attention_compressed_b200 as bsa
        from block_sparse_attention_compressed_b200.workloads import generate
        self.torch, self.bsa, self.w, self.dev = torch, bsa, w, device
        ws_ = w.replace(seed=w.seed + seed_offset)
        self.append = w.append_steps > 0
        steps = max(steps_total, w.append_steps) if self.append else 0
        self.data = generate(ws_, device=device, steps=steps)
        self.T_cap = self.data["seq_cap"]
        self.p = bsa.make_params(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, self.T_cap,
                                 w.dtype, w.n_init, w.n_local, w.top_k, w.cmp_kernel, w.cmp_stride,
                                 w.block_size, num_layers=w.layers)
        s = bsa.bsa_get_sizes(self.p)
        self.sizes = s
        dt = w.torch_dtype
        B, Hkv, d = w.batch, w.num_kv_heads, w.head_dim
        self.ck = torch.zeros(B, Hkv, s.nc_cap, d, dtype=dt, device=device)
        bsa.bsa_compress_keys(self.p, self.data["k"][0], self.data["seq_lens"], self.ck)
        # anchored index reuse: compressed keys of every anchor layer, one selection per anchor
        self.anchored = len(w.anchors) > 1
        self.cks = [self.ck if L == 0 else None for L in range(w.layers)]
        for L in w.anchors[1:]:
            self.cks[L] = torch.zeros_like(self.ck)
            bsa.bsa_compress_keys(self.p, self.data["k"][L], self.data["seq_lens"], self.cks[L])
        self.ws = bsa.alloc_workspace(self.p, device)
        bsa.bsa_workspace_init(self.p, self.ws)
        A = len(w.anchors)
        self.block_idx_all = torch.zeros(A, B, Hkv, s.sel_cap, dtype=torch.int32, device=device)
        self.n_sel_all = torch.zeros(A, B, Hkv, dtype=torch.int32, device=device)
        self.block_idx, self.n_sel = self.block_idx_all[0], self.n_sel_all[0]
        self.out = [torch.zeros(B, w.num_q_heads, d, dtype=dt, device=device)
                    for _ in range(w.layers)]
        self.lse = [torch.zeros(B, w.num_q_heads, dtype=torch.float32, device=device)
                    for _ in range(w.layers)]
        self.seq0 = self.data["seq_lens"].clone()
        # one kernel per step (the fused path) for the single-layer workloads: bsa_decode_step's
        # own choice, or the path asked for
        single = w.layers == 1 and not w.forecast
        self.path = path if single else "auto"
        self.fused = single and (path == "fused" or (path == "auto" and bsa.bsa_decode_step_info(self.p)[0]))
        self.lookahead = bool(w.lookahead)
        self.clsa = bool(w.token_index)
        if self.clsa:
            # CLSA: layer 0's token-level index, attended by every layer (three launches per step)
            self.ws = bsa.alloc_clsa_workspace(self.p, device)
            self.tok_cap = (w.n_init + w.n_local + w.top_k) * w.block_size
            self.tok_idx = torch.zeros(B, Hkv, self.tok_cap, dtype=torch.int32, device=device)
            self.n_tok = torch.zeros(B, Hkv, dtype=torch.int32, device=device)
            self.fused = True
        self.prefill = w.prefill_chunk > 0
        if self.prefill:
            # block-sparse prefill of the last prefill_chunk positions: queries drawn like q
            C = w.prefill_chunk
            g = torch.Generator(device=device).manual_seed(w.seed + 7 + seed_offset)
            self.q_chunk = torch.randn(B, C, w.num_q_heads, d, generator=g, device=device).to(dt)
            self.data["q_chunk"] = self.q_chunk
            self.tiles = bsa.bsa_prefill_tiles(C, w.block_size)
            self.p_idx = torch.zeros(B, Hkv, self.tiles, s.sel_cap, dtype=torch.int32, device=device)
            self.p_ns = torch.zeros(B, Hkv, self.tiles, dtype=torch.int32, device=device)
            self.out = [torch.zeros(B, C, w.num_q_heads, d, dtype=dt, device=device)]
            self.lse = [torch.zeros(B, C, w.num_q_heads, dtype=torch.float32, device=device)]
            self.fused = True
        if self.lookahead:
            # layer 0 attends blocks chosen beforehand (here by its own queries, outside the timed
            # region) while layer 1's are chosen from the Forecast vectors: one kernel per step
            self.ck_next = torch.zeros_like(self.ck)
            bsa.bsa_compress_keys(self.p, self.data["k"][1], self.data["seq_lens"], self.ck_next)
            bsa.bsa_select_blocks(self.p, self.data["q"][0], self.ck, self.data["seq_lens"], self.block_idx,
                                  self.n_sel, None, self.ws)
            self.idx_next = torch.zeros_like(self.block_idx)
            self.n_sel_next = torch.zeros_like(self.n_sel)
            self.fused = True
        elif w.forecast and (w.layers > 1 or self.append):
            raise ValueError("the Forecast-indexer workloads are single-layer, fixed-length")
        torch.cuda.synchronize()

    def q_of(self, i):
        if self.prefill:
            return self.q_chunk
        return self.data["q_steps"][i] if self.append else self.data["q"][0]

    # the library calls of one step, on `stream`; `events` (optional) brackets every launch
    def step(self, i, stream=None, events=None, q=None):
        bsa, d = self.bsa, self.data
        q = self.q_of(i) if q is None else q
        ev = (lambda k: events[k].record(stream)) if events is not None else (lambda k: None)
        if self.clsa:
            ev(0)
            bsa.bsa_decode_step_clsa(self.p, [q] + [d["q"][L] for L in range(1, self.w.layers)], d["k"], d["v"],
                                     d["seq_lens"], self.tok_idx, self.n_tok, self.out, self.lse, self.ws,
                                     stream=stream)
            ev(1)
            return
        if self.prefill:
            ev(0)
            bsa.bsa_prefill(self.p, self.w.prefill_chunk, self.q_chunk, d["k"][0], d["v"][0], self.ck,
                            d["seq_lens"], self.p_idx, self.p_ns, self.out[0], self.lse[0], self.ws,
                            stream=stream)
            ev(1)
            return
        if self.lookahead:
            ev(0)
            bsa.bsa_decode_step_lookahead(self.p, q, d["k"][0], d["v"][0], self.block_idx, self.n_sel,
                                          d["f"], self.ck_next, d["seq_lens"], self.idx_next,
                                          self.n_sel_next, None, self.out[0], self.lse[0], self.ws,
                                          stream=stream)
            ev(1)
            return
        if self.w.forecast:
            ev(0)
            bsa.bsa_select_blocks_forecast(self.p, d["f"], self.ck, d["seq_lens"], self.block_idx,
                                           self.n_sel, None, self.ws, stream=stream)
            ev(1)
            bsa.bsa_sparse_decode(self.p, q, d["k"][0], d["v"][0], d["seq_lens"], self.block_idx,
                                  self.n_sel, self.out[0], self.lse[0], self.ws, stream=stream)
            ev(2)
            return
        if self.w.layers > 1:
            qs = [q] + [d["q"][L] for L in range(1, self.w.layers)]
            if self.anchored and events is None:
                bsa.bsa_decode_step_anchored(self.p, self.w.anchors, qs, d["k"], d["v"], self.cks,
                                             d["seq_lens"], self.block_idx_all, self.n_sel_all,
                                             self.out, self.lse, self.ws, stream=stream)
                return
            # one selection per anchor (the calls bsa_decode_step_anchored chains), each reused
            # by the layers up to the next anchor
            anchors = list(self.w.anchors) + [self.w.layers]
            for i in range(len(anchors) - 1):
                a0, a1 = anchors[i], anchors[i + 1]
                ev(2 * i)
                bsa.bsa_select_blocks(self.p, qs[a0], self.cks[a0], d["seq_lens"],
                                      self.block_idx_all[i], self.n_sel_all[i], None, self.ws,
                                      stream=stream)
                ev(2 * i + 1)
                bsa.bsa_sparse_decode_layers(self.p, qs[a0:a1], d["k"][a0:a1], d["v"][a0:a1],
                                             d["seq_lens"], self.block_idx_all[i],
                                             self.n_sel_all[i], self.out[a0:a1], self.lse[a0:a1],
                                             self.ws, stream=stream)
            ev(2 * (len(anchors) - 1))
            return
        if events is None and self.path != "chained":
            bsa.bsa_decode_step(self.p, q, d["k"][0], d["v"][0], self.ck,
                                d["k_new"][i] if self.append else None,
                                d["v_new"][i] if self.append else None, d["seq_lens"],
                                self.block_idx, self.n_sel, None, self.out[0], self.lse[0], self.ws,
                                stream=stream, fused=self.fused)
            return
        k = 0
        if self.append:
            ev(k); k += 1
            bsa.bsa_compress_append(self.p, d["k"][0], d["v"][0], d["k_new"][i], d["v_new"][i],
                                    d["seq_lens"], self.ck, self.ws, stream=stream)
        if self.fused:
            # the step kernel alone (the append, if any, was bracketed above)
            ev(k)
            bsa.bsa_decode_step(self.p, q, d["k"][0], d["v"][0], self.ck, None, None, d["seq_lens"],
                                self.block_idx, self.n_sel, None, self.out[0], self.lse[0], self.ws,
                                stream=stream, fused=True)
            ev(k + 1)
            return
        ev(k)
        bsa.bsa_select_blocks(self.p, q, self.ck, d["seq_lens"], self.block_idx, self.n_sel, None,
                              self.ws, stream=stream)
        ev(k + 1)
        bsa.bsa_sparse_decode(self.p, q, d["k"][0], d["v"][0], d["seq_lens"], self.block_idx,
                              self.n_sel, self.out[0], self.lse[0], self.ws, stream=stream)
        ev(k + 2)

    # one step with caller-given input and output buffers (the end-to-end pass); for the
    # Forecast-indexer workloads qs is [q, f]
    def step_io(self, qs, outs, lses, stream, k_new=None, v_new=None):
        bsa, d = self.bsa, self.data
        if self.clsa:
            bsa.bsa_decode_step_clsa(self.p, qs, d["k"], d["v"], d["seq_lens"], self.tok_idx, self.n_tok, outs, lses,
                                     self.ws, stream=stream)
            return
        if self.prefill:
            bsa.bsa_prefill(self.p, self.w.prefill_chunk, qs[0], d["k"][0], d["v"][0], self.ck, d["seq_lens"],
                            self.p_idx, self.p_ns, outs[0], lses[0], self.ws, stream=stream)
            return
        if self.lookahead:
            bsa.bsa_decode_step_lookahead(self.p, qs[0], d["k"][0], d["v"][0], self.block_idx, self.n_sel,
                                          qs[1], self.ck_next, d["seq_lens"], self.idx_next,
                                          self.n_sel_next, None, outs[0], lses[0], self.ws, stream=stream)
            return
        if self.w.forecast:
            bsa.bsa_select_blocks_forecast(self.p, qs[1], self.ck, d["seq_lens"], self.block_idx,
                                           self.n_sel, None, self.ws, stream=stream)
            bsa.bsa_sparse_decode(self.p, qs[0], d["k"][0], d["v"][0], d["seq_lens"], self.block_idx,
                                  self.n_sel, outs[0], lses[0], self.ws, stream=stream)
            return
        if self.w.layers > 1:
            if self.anchored:
                bsa.bsa_decode_step_anchored(self.p, self.w.anchors, qs, d["k"], d["v"], self.cks,
                                             d["seq_lens"], self.block_idx_all, self.n_sel_all,
                                             outs, lses, self.ws, stream=stream)
                return
            bsa.bsa_select_blocks(self.p, qs[0], self.ck, d["seq_lens"], self.block_idx, self.n_sel,
                                  None, self.ws, stream=stream)
            bsa.bsa_sparse_decode_layers(self.p, qs, d["k"], d["v"], d["seq_lens"], self.block_idx,
                                         self.n_sel, outs, lses, self.ws, stream=stream)
            return
        if self.path == "chained":
            if k_new is not None:
                bsa.bsa_compress_append(self.p, d["k"][0], d["v"][0], k_new, v_new, d["seq_lens"],
                                        self.ck, self.ws, stream=stream)
            bsa.bsa_select_blocks(self.p, qs[0], self.ck, d["seq_lens"], self.block_idx, self.n_sel,
                                  None, self.ws, stream=stream)
            bsa.bsa_sparse_decode(self.p, qs[0], d["k"][0], d["v"][0], d["seq_lens"], self.block_idx,
                                  self.n_sel, outs[0], lses[0], self.ws, stream=stream)
            return
        bsa.bsa_decode_step(self.p, qs[0], d["k"][0], d["v"][0], self.ck, k_new, v_new, d["seq_lens"],
                            self.block_idx, self.n_sel, None, outs[0], lses[0], self.ws,
                            stream=stream, fused=self.fused)

    def kernel_names(self):
        """The phases pass B brackets with events, in launch order."""
        if self.prefill:
            return ["prefill"]
        if self.clsa:
            return ["clsa"]
        if self.fused:
            return (["append"] if self.append else []) + ["step"]
        names = ["select", "decode"] * (len(self.w.anchors) if self.w.layers > 1 else 1)
        return (["append"] + names) if (self.append and self.w.layers == 1) else names

    def launches_per_step(self):
        if self.prefill:
            return 2  # the selection (tcgen05) and the attention
        if self.clsa:
            return 3  # token scoring, token top-k, token attention (all layers)
        if self.fused:
            return 1 + (1 if self.append else 0)
        # bsa_select_blocks launches two kernels (scoring, selection), the bf16 sparse attention two
        # (attention, combine), the fp32 one one
        n = self.kernel_names()
        return len(n) + n.count("select") + (n.count("decode") if self.w.dtype == "bf16" else 0)

    def reset_lengths(self):
        self.data["seq_lens"].copy_(self.seq0)


def algorithmic(w, T):
    from block_sparse_attention_compressed_b200.workloads import algorithmic_bytes
    return algorithmic_bytes(w, T)


def load_tensor_peak():
    """Measured dense bf16 GEMM throughput (burst, TFLOP/s), else the fallback figure."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


# The sources that decide a kernel's code and launch plan: its own file, the shared headers and
# the host side that plans the launch.
KERNEL_SOURCES = {"step": "step_kernels.cu", "decode": "decode_kernels.cu", "combine": "decode_kernels.cu",
                  "score": "select_kernels.cu", "select": "select_kernels.cu",
                  "compress": "compress_kernels.cu", "append": "compress_kernels.cu",
                  "prefill": "prefill_kernels.cu", "token": "clsa_kernels.cu"}


def _code_only(text: str) -> str:
    """C/C++/CUDA source without its comments and with whitespace runs collapsed, so that a
    comment edit does not count as a change of the compiled code."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":          # string or char literal, kept whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(kernel: str | None = None) -> str:
    """sha256 (16 hex digits) of the kernel's sources with comments removed (see _code_only), or
    of every kernel source when None."""
    import glob
    csrc = os.path.join(ROOT, "block_sparse_attention_compressed_b200", "csrc")
    if kernel is None:
        paths = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh")))
    else:
        own = next(f for k, f in KERNEL_SOURCES.items() if kernel.startswith(k))
        # the kernel's own file and the headers it includes, transitively (the host-side launch
        # code is left out)
        names, todo = [], [own]
        while todo:
            n = todo.pop(0)
            if n in names or not os.path.exists(os.path.join(csrc, n)):
                continue  # (the public header lies outside csrc/)
            names.append(n)
            with open(os.path.join(csrc, n), encoding="utf-8") as f:
                todo += re.findall(r'^#include "([^"]+)"', f.read(), flags=re.M)
        paths = [os.path.join(csrc, n) for n in names if os.path.exists(os.path.join(csrc, n))]
    h = hashlib.sha256()
    for p in paths:
        with open(p, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summaries of the workload, if they were taken on
    the kernel's current sources (each summary records their hash: kernel_source_hash(kernel)).

    A summary ``profiles/<name>_<workload>.md`` gives, per kernel, the lines
    ``dram_bytes_per_launch[<kernel>]: N`` and ``kernel_sources_sha256_16[<kernel>]: H`` (or, in
    ``profiles/<kernel>_<workload>.md``, the same two lines without the bracket). A phase of two
    kernels ("a+b") adds up both kernels' bytes."""
    if "+" in kernel:
        parts = [profile_traffic(k, workload) for k in kernel.split("+")]
        return None if any(v is None for v in parts) else sum(parts)
    import glob
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"*_{workload}.md"))):
        text = open(path).read()
        tag = re.escape(f"[{kernel}]")
        m = re.search(r"dram_bytes_per_launch" + tag + r":\s*([\d.eE+]+)", text)
        hm = re.search(r"kernel_sources_sha256_16" + tag + r":\s*([0-9a-f]+)", text)
        if not m and os.path.basename(path) == f"{kernel}_{workload}.md":
            m = re.search(r"dram_bytes_per_launch:\s*([\d.eE+]+)", text)
            hm = re.search(r"kernel_sources_sha256_16:\s*([0-9a-f]+)", text)
        if m and hm:
            return float(m.group(1)) if hm.group(1) == kernel_source_hash(kernel) else None
    return None


# ------------------------------------------------------------------------------- CPU (oracle) leg
def cpu_oracle_sample(w, data, seconds: float):
    """The CPU oracle's decode step on a bounded sample of the workload's (batch, kv-head) pairs:
    group scoring, block reduction, top-k and attention on the scoring layers (the compressed keys
    formed beforehand, as at decode time), attention with their selection on the other layers.
    Returns a dict: steps/s scaled to the whole batch on all host threads and on one, the threads,
    the compression's CPU time per step-equivalent cache (reported apart), and a description."""
    import torch
    import oracle
    G, Hkv = w.group, w.num_kv_heads
    total = w.batch * Hkv
    T_cap = data["seq_cap"]
    seq = data["seq_lens"].cpu().tolist()
    threads = oracle.num_threads()
    n0 = min(max(threads, 1), total)
    pairs = [divmod(p, Hkv) for p in range(n0)]

    def layer_arrays(L):
        if w.prefill_chunk:
            qs = torch.stack([data["q_chunk"][b, :, h * G:(h + 1) * G] for b, h in pairs])
        else:
            q = data["q_steps"][0] if ("q_steps" in data and L == 0) else data["q"][L]
            qs = torch.stack([q[b, h * G:(h + 1) * G] for b, h in pairs])
        ks = torch.stack([data["k"][L][b, h:h + 1] for b, h in pairs])
        vs = torch.stack([data["v"][L][b, h:h + 1] for b, h in pairs])
        return oracle.raw(qs)[0], oracle.raw(ks)[0], oracle.raw(vs)[0]

    arrays = [layer_arrays(L) for L in range(w.layers)]
    lens = [seq[b] for b, _ in pairs]
    P = oracle.make_problem(n0, G, 1, w.head_dim, T_cap,
                            oracle.F32 if w.dtype == "f32" else oracle.BF16, w.n_init, w.n_local,
                            w.top_k, w.cmp_kernel, w.cmp_stride, w.block_size)
    f_arr = (oracle.raw(torch.stack([data["f"][b, h:h + 1] for b, h in pairs]))[0]
             if w.forecast else None)
    # A1, the compression of every scoring layer's keys (once per cache; timed apart)
    scored = [1] if w.lookahead else ([] if (w.prefill_chunk or w.token_index) else list(w.anchors))
    t0 = time.perf_counter()
    cks = {L: oracle.compress_cache(P, arrays[L][1], lens) for L in scored}
    compress_s = (time.perf_counter() - t0) * (total / n0) / max(len(scored), 1)
    # lookahead: layer 0's blocks, chosen beforehand (by its own queries; untimed)
    sel0 = oracle.decode(P, *arrays[0], lens) if w.lookahead else None

    def one(sub=None):
        idx = slice(None) if sub is None else slice(0, sub)
        r = None
        for L in range(w.layers):
            q_, k_, v_ = arrays[L]
            if sub is not None:
                q_, k_, v_ = q_[idx], k_[idx], v_[idx]
            Ps = P if sub is None else oracle.make_problem(
                sub, G, 1, w.head_dim, T_cap, P.dtype, w.n_init, w.n_local, w.top_k, w.cmp_kernel,
                w.cmp_stride, w.block_size)
            ln = lens if sub is None else lens[:sub]
            if w.token_index:
                if L == 0:
                    oracle.clsa(Ps, [a[0][idx] for a in arrays], [a[1][idx] for a in arrays],
                                [a[2][idx] for a in arrays], ln)
                return
            if w.prefill_chunk:
                # the chunk's block-sparse prefill (its compression included: the chunk's keys
                # complete new windows)
                oracle.prefill(Ps, q_, k_, v_, ln, w.prefill_chunk)
                return
            if w.lookahead:
                # layer 0 attends its blocks, layer 1's are chosen from the Forecast vectors
                oracle.lookahead_step(Ps, q_, k_, v_, sel0["idx"][idx], sel0["n_sel"][idx], f_arr[idx],
                                      cks[1][idx], ln)
                return
            if w.forecast:
                oracle.decode_forecast(Ps, f_arr[idx], q_, k_, v_, ln, ck=cks[0][idx])
            elif L in w.anchors:
                r = oracle.decode(Ps, q_, k_, v_, ln, ck=cks[L][idx])  # select + attend
            else:
                oracle.attend_pairs(Ps, q_, k_, v_, ln, r["idx"], r["n_sel"])

    def timed(fn, budget):
        t0 = time.perf_counter()
        fn()
        dt0 = time.perf_counter() - t0
        reps = max(1, int(budget / max(dt0, 1e-6)))
        t0 = time.perf_counter()
        for _ in range(reps):
            fn()
        return (time.perf_counter() - t0) / reps, reps

    dt, reps = timed(one, seconds)
    with oracle.threads(1):
        dt1, reps1 = timed(lambda: one(1), seconds / 4)   # one pair on one thread
    layers = f" x {w.layers} layers" if w.layers > 1 and not w.lookahead else ""
    desc = (f"CPU oracle (fp64) decode step on {n0} of {total} (batch, kv-head) pairs{layers}: "
            f"scoring, block reduction, top-k and attention with the keys compressed beforehand "
            f"(their compression, {compress_s:.2f} s per full cache, is timed apart), "
            f"{reps} repetitions on {threads} threads scaled by {total}/{n0}, and one pair on one "
            f"thread ({reps1} repetitions) scaled by {total}")
    return {"value": 1.0 / (dt * total / n0), "single_thread_value": 1.0 / (dt1 * total),
            "cores": threads, "compress_s_per_cache": compress_s, "sample": desc}


# -------------------------------------------------------------------------------------------- main
def run_bsa(args, w, world, rank, local):
    import torch
    import block_sparse_attention_compressed_b200 as bsa  # noqa: F401  (fails loudly if unbuilt)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    K, W = args.steps, args.warmup
    bench = Bench(w, dev, seed_offset=10000 * rank, steps_total=K + W + 1, path=args.path)
    T_run = w.seq_len
    ab = algorithmic(w, T_run)
    stream = torch.cuda.Stream(device=dev)
    per_step_bytes = ab["total"]
    if w.prefill_chunk:
        # prefill: the chunk's queries and outputs, the compressed keys and (at least once) the K
        # and V rows of the whole prefix; the roofline of this workload is the tensor one
        e, d, pairs = w.elem_bytes, w.head_dim, w.batch * w.num_kv_heads
        per_step_bytes = (2 * w.batch * w.prefill_chunk * w.num_q_heads * d * e + ab["ck"]
                          + 2 * pairs * w.seq_len * d * e)
    flush = per_step_bytes < 4 * L2_BYTES
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if flush else None
    use_graph = not args.no_graph and not bench.append

    # CUDA graphs: with inputs larger than L2 the K timed steps are one graph, replayed once (the
    # way a decode loop is captured: consecutive steps overlap their launch with the previous
    # step's tail, each still waiting for it before reading anything); with an L2 flush between
    # steps, a graph of one step is replayed K times with the flush in between
    graph = graph_k = None
    with torch.cuda.stream(stream):
        for i in range(W):
            bench.step(i, stream)
        if use_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                bench.step(0, stream)
            graph.replay()
            if not flush:
                graph_k = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph_k, stream=stream):
                    for i in range(K):
                        bench.step(W + i, stream)
                graph_k.replay()  # warm-up of the captured loop (untimed)
    stream.synchronize()

    def run_step(i):
        if graph is not None:
            graph.replay()
        else:
            bench.step(W + i, stream)

    # ---- pass A: the headline
    if bench.append:
        bench.reset_lengths()
        with torch.cuda.stream(stream):
            for i in range(W):
                bench.step(i, stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            if flush:
                starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
                ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
                for i in range(K):
                    flush_buf.fill_(i & 0xff)
                    starts[i].record(stream)
                    run_step(i)
                    ends[i].record(stream)
            else:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                if graph_k is not None:
                    graph_k.replay()
                else:
                    for i in range(K):
                        run_step(i)
                e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
    barrier(world)
    if flush:
        local_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    else:
        local_ms = e0.elapsed_time(e1)
    total_ms = max_over_ranks(local_ms, world)
    ms_per_step = total_ms / K
    clocks = clk.summary()

    # the same K steps as K replays of the one-step graph (each replay waits for the previous one
    # to finish before its kernels launch): reported beside the headline, not instead of it
    one_step_graphs_ms = None
    if graph_k is not None:
        torch.cuda.synchronize()
        barrier(world)
        with torch.cuda.stream(stream):
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for i in range(K):
                graph.replay()
            g1.record(stream)
        stream.synchronize()
        one_step_graphs_ms = max_over_ranks(g0.elapsed_time(g1), world) / K

    # ---- pass B: per-kernel breakdown (same work, every launch bracketed by events)
    names = bench.kernel_names()
    nk = len(names)
    if bench.append:
        bench.reset_lengths()
        with torch.cuda.stream(stream):
            for i in range(W):
                bench.step(i, stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(K)]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(K):
            if flush:
                flush_buf.fill_(i & 0xff)
            bench.step(W + i if bench.append else 0, stream, events=evs[i])
    stream.synchronize()
    kern_ms = {}  # per phase, summed over the phase's calls in a step (one per anchor)
    for j, n in enumerate(names):
        kern_ms[n] = kern_ms.get(n, 0.0) + sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)) / K

    # ---- e2e: through the binding, every step's inputs copied in from pinned host memory and its
    # outputs (every layer) copied back, double-buffered: step i+1's inputs land and step i's
    # outputs return on copy streams while step i+1 computes
    import torch as _t
    L_ = 1 if w.lookahead else w.layers  # lookahead: one layer attends per step
    NBUF = 2
    def step_q(i):  # the query of every layer for timed step i (then the Forecast vectors)
        return ([bench.q_of(W + i if bench.append else 0)] + [bench.data["q"][l] for l in range(1, L_)]
                + ([bench.data["f"]] if w.forecast else []))
    q_host = [[t.cpu().pin_memory() for t in step_q(i)] for i in range(K)]
    q_dev = [[_t.empty_like(t) for t in step_q(0)] for _ in range(NBUF)]
    out_dev = [[_t.empty_like(bench.out[l]) for l in range(L_)] for _ in range(NBUF)]
    lse_dev = [[_t.empty_like(bench.lse[l]) for l in range(L_)] for _ in range(NBUF)]
    out_host = [[_t.empty(bench.out[l].shape, dtype=bench.out[l].dtype).pin_memory() for l in range(L_)]
                for _ in range(NBUF)]
    if bench.append:
        bench.reset_lengths()
        with _t.cuda.stream(stream):
            for i in range(W):
                bench.step(i, stream)
        kn_host = [bench.data["k_new"][W + i].cpu().pin_memory() for i in range(K)]
        vn_host = [bench.data["v_new"][W + i].cpu().pin_memory() for i in range(K)]
        kn_dev = [_t.empty_like(bench.data["k_new"][0]) for _ in range(NBUF)]
        vn_dev = [_t.empty_like(bench.data["v_new"][0]) for _ in range(NBUF)]
    h2d_stream = _t.cuda.Stream(device=dev)
    d2h_stream = _t.cuda.Stream(device=dev)
    ev_in = [_t.cuda.Event() for _ in range(NBUF)]
    ev_step = [_t.cuda.Event() for _ in range(NBUF)]
    ev_back = [_t.cuda.Event() for _ in range(NBUF)]
    _t.cuda.synchronize()
    barrier(world)
    _t.cuda.synchronize()
    t_e2e0 = time.perf_counter()
    a0, a1 = _t.cuda.Event(enable_timing=True), _t.cuda.Event(enable_timing=True)
    a0.record(stream)
    h2d_stream.wait_event(a0)
    d2h_stream.wait_event(a0)
    for i in range(K):
        j = i % NBUF
        with _t.cuda.stream(h2d_stream):
            if i >= NBUF:
                h2d_stream.wait_event(ev_step[j])  # the step that last read buffer j is done
            for l in range(len(q_host[i])):
                q_dev[j][l].copy_(q_host[i][l], non_blocking=True)
            if bench.append:
                kn_dev[j].copy_(kn_host[i], non_blocking=True)
                vn_dev[j].copy_(vn_host[i], non_blocking=True)
            ev_in[j].record(h2d_stream)
        stream.wait_event(ev_in[j])
        if i >= NBUF:
            stream.wait_event(ev_back[j])  # buffer j's outputs have been copied back
        with _t.cuda.stream(stream):
            bench.step_io(q_dev[j], out_dev[j], lse_dev[j], stream,
                          kn_dev[j] if bench.append else None, vn_dev[j] if bench.append else None)
        ev_step[j].record(stream)
        with _t.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ev_step[j])
            for l in range(L_):
                out_host[j][l].copy_(out_dev[j][l], non_blocking=True)
            ev_back[j].record(d2h_stream)
    stream.wait_stream(h2d_stream)
    stream.wait_stream(d2h_stream)
    a1.record(stream)
    stream.synchronize()
    e2e_local = a0.elapsed_time(a1)
    e2e_ms = max_over_ranks(e2e_local, world)
    wall_e2e = time.perf_counter() - t_e2e0
    h2d = sum(t.numel() * t.element_size() for t in q_host[0])
    if bench.append:
        h2d += 2 * kn_host[0].numel() * kn_host[0].element_size()
    d2h = sum(o.numel() * o.element_size() for o in out_host[0])

    err = bench.bsa.bsa_read_device_error(bench.ws)
    if err:
        raise RuntimeError(f"device error flags set during the benchmark: {err:#x}")

    # ---- roofline of the largest single launch, and the spec fraction of the whole step
    peak, peak_kind = load_peaks()
    q_bytes = w.batch * w.num_q_heads * w.head_dim * w.elem_bytes
    fv = ab["f"] if w.forecast else 0
    kbytes = {"select": ab["ck"] + (fv if w.forecast else q_bytes),  # compressed keys + q (or f)
              "decode": ab["kv"] + ab["qo"],         # selected K/V rows + q + out, every layer
              "step": ab["ck"] + ab["kv"] + ab["qo"] + fv,  # the fused step: all of them
              "clsa": ab["ck"] + ab["kv"] + ab["qo"],       # the index layer's keys + every layer's tokens
              "append": ab["append"]}
    # the selection phase is two launches (scoring, then selection): the roofline is taken on the
    # largest phase that is one launch, or one launch and its combine
    single = {n: t for n, t in kern_ms.items() if n != "select"} or kern_ms
    dom = max(single, key=single.get)
    kname = KERNEL_OF_PHASE[dom][w.dtype]
    n_calls = names.count(dom)  # launches of that phase per step (one per anchor)
    if bench.prefill:
        # a contraction: algorithmic FLOPs (scoring + attention) over the measured bf16 GEMM peak
        from block_sparse_attention_compressed_b200.workloads import prefill_flops
        fl = prefill_flops(w)
        tpeak, tkind = load_tensor_peak()
        achieved = fl["total"] / (kern_ms[dom] * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": kname, "achieved": round(achieved, 2), "peak": tpeak,
                    "unit": "TFLOP/s", "frac": round(achieved / tpeak, 4),
                    "peak_kind": tkind + " bf16 GEMM throughput (MEASURED_PEAKS.json bf16_tflops)",
                    "traffic": profile_traffic(kname, w.name), "algorithmic_flops_per_launch": fl["total"],
                    "algorithmic_flops": fl, "kernel_ms": round(kern_ms[dom], 5),
                    "launches_timed": "the selection and the attention kernels of one bsa_prefill call"}
    else:
        achieved = kbytes[dom] / (kern_ms[dom] * 1e-3) / 1e9
        traffic = profile_traffic(kname, w.name)
        roofline = {"bound": "hbm", "kernel": kname, "achieved": round(achieved, 1),
                    "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                    "peak_kind": peak_kind + " copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                    "frac_of_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                    "traffic": traffic, "algorithmic_bytes_per_launch": kbytes[dom] / n_calls,
                    "kernel_ms": round(kern_ms[dom] / n_calls, 5),
                    "launches_timed": "one" if "+" not in kname else "the attention kernel and its combine"}

    steps_per_s = world * K / (total_ms * 1e-3)
    gbs = per_step_bytes * world * K / (total_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC,
        "value": round(steps_per_s, 2),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) q/K/V with planted needle blocks)"
                + ("; Forecast vectors = each GQA group's mean query" if w.forecast else ""),
        "config": {
            "workload": w.name, "batch": w.batch, "seq_len": w.seq_len, "q_heads": w.num_q_heads,
            "kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "n_init": w.n_init,
            "n_local": w.n_local, "top_k": w.top_k, "block_size": w.block_size,
            "cmp_kernel": w.cmp_kernel, "cmp_stride": w.cmp_stride, "layers": w.layers,
            "append": bool(bench.append), "forecast_indexer": bool(w.forecast),
            "anchors": list(w.anchors),
            "parallelism": f"replicas x{world} (batch-sharded)",
            "l2": ("L2 flushed (256 MB write) between timed steps" if flush else
                   f"inputs larger than L2: {per_step_bytes / 1e6:.0f} MB read per step vs 126 MB L2"),
            "cuda_graph": ("one graph of the K timed steps" if graph_k is not None else
                           "a one-step graph replayed per step" if graph is not None else False),
            "step_path": "fused" if bench.fused else "chained",
        },
        "tokens_per_s": round(steps_per_s * w.batch * (w.prefill_chunk or 1), 1),
        "hbm_gbs": round(gbs / world, 1),
        "frac_of_8tbs": round(gbs / world / NOMINAL_HBM_GBS, 4),
        "hbm_target": None if bench.prefill else {
            "basis": "compressed keys + selected K/V + q + out bytes of the whole step over 8 TB/s, "
                     "device-timed step", "frac_of_8tbs": round(gbs / world / NOMINAL_HBM_GBS, 4),
            "target": TARGET_FRAC_OF_8TBS, "met": bool(gbs / world / NOMINAL_HBM_GBS >= TARGET_FRAC_OF_8TBS)},
        "ms_per_step_one_step_graphs": (round(one_step_graphs_ms, 5) if one_step_graphs_ms is not None
                                        else None),
        "fused_step": bool(bench.fused),
        "algorithmic_bytes_per_step": per_step_bytes,
        "kernels_ms": {k: round(v, 5) for k, v in kern_ms.items()},
        "roofline": roofline,
        "e2e": {"value": round(world * K / (e2e_ms * 1e-3), 2), "unit": "steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "wall_s": round(wall_e2e, 4), "l2_flush": False},
        "gpu_launches": K * bench.launches_per_step(),
        "clocks": clocks,
        "kernel_sources_sha256_16": kernel_source_hash(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        c = cpu_oracle_sample(w, bench.data, args.cpu_seconds)
        result["cpu_baseline"] = {"value": round(c["value"], 4), "unit": "steps/s",
                                  "cores": c["cores"], "kind": "oracle",
                                  "single_thread_value": round(c["single_thread_value"], 5),
                                  "compress_s_per_cache": round(c["compress_s_per_cache"], 3),
                                  "sample": c["sample"]}
    return result


def run_reference(args, w, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the host cores."""
    import torch
    from block_sparse_attention_compressed_b200.workloads import generate
    if rank != 0:
        return None
    per_step = max(1.0, args.cpu_seconds / max(args.steps + args.warmup, 1))
    w_small = w
    data = generate(w_small, device="cuda" if torch.cuda.is_available() else "cpu",
                    steps=1 if w.append_steps else 0)
    for _ in range(args.warmup):
        cpu_oracle_sample(w, data, per_step / 4)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        c = cpu_oracle_sample(w, data, per_step)
        vals.append(c["value"])
    cores, desc = c["cores"], c["sample"]
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 / value, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) q/K/V with planted needle blocks)",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seq_len},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "steps/s", "cores": cores,
                         "kind": "oracle", "single_thread_value": round(c["single_thread_value"], 5),
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 2),
    }


def relaunch(n: int) -> int:
    """Start n ranks of this script on this node (torch.distributed.run, rendezvous on
    127.0.0.1, a free port) with the same arguments; rank 0 prints the JSON line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    args = parse()
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        sys.exit(relaunch(args.gpus))
    if world_env is not None and int(world_env) != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world_env}; "
                         "start one rank per GPU with the same N")
    from block_sparse_attention_compressed_b200.workloads import DEFAULT_WORKLOAD, WORKLOADS
    w = WORKLOADS[args.workload or DEFAULT_WORKLOAD]
    if args.batch:
        w = w.replace(batch=args.batch, name=f"{w.name}@batch{args.batch}")
    world, rank, local = dist_init(args)
    if args.impl == "reference":
        res = run_reference(args, w, world, rank)
    else:
        res = run_bsa(args, w, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
