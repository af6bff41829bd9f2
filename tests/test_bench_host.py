"""Host-side pieces of bench.py (no GPU): the source fingerprint that ties an ncu summary in
profiles/ to the code it was taken on, and the byte model of every workload."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from block_sparse_attention_compressed_b200.workloads import WORKLOADS, algorithmic_bytes  # noqa: E402


def test_code_only_drops_comments_and_keeps_literals():
    src = 'int a = 1;  // note\n/* block\n comment */ const char* s = "// kept /* too */";\nfloat  b;'
    assert bench._code_only(src) == 'int a = 1; const char* s = "// kept /* too */"; float b;'
    # a comment edit does not change the fingerprint input, a code edit does
    assert bench._code_only(src.replace("note", "other note")) == bench._code_only(src)
    assert bench._code_only(src.replace("a = 1", "a = 2")) != bench._code_only(src)


def test_kernel_source_hash_covers_each_kernel():
    for k in ("step_kernel", "decode_tma_kernel", "combine_kernel", "score_tma_kernel",
              "select_single_kernel", "compress_keys_kernel", "append_kernel"):
        h = bench.kernel_source_hash(k)
        assert len(h) == 16 and int(h, 16) >= 0
    assert bench.kernel_source_hash("decode_tma_kernel") != bench.kernel_source_hash("score_tma_kernel")


def test_profile_summaries_parse():
    """Every committed DRAM summary states, per kernel, its bytes per launch and a source
    fingerprint, and the bench finds the figure of the kernel it reports for each summarised
    workload (when the summary's fingerprint is the kernel's current one)."""
    import re
    import bench
    pdir = os.path.join(ROOT, "profiles")
    names = [n for n in os.listdir(pdir) if n.endswith(".md") and not n.startswith("launches_")]
    assert names
    for n in names:
        text = open(os.path.join(pdir, n)).read()
        tagged = re.findall(r"dram_bytes_per_launch\[(\w+)\]:\s*\d+", text)
        assert tagged, n
        for k in tagged:
            assert re.search(r"kernel_sources_sha256_16\[" + k + r"\]:\s*[0-9a-f]{16}", text), (n, k)
        for wl in WORKLOADS:
            if n.endswith(f"_{wl}.md"):
                for k in tagged:
                    got = bench.profile_traffic(k, wl)
                    assert got is None or got > 0, (n, k)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_algorithmic_bytes(name):
    """The byte model: compressed keys of every scoring layer, the selected K/V rows of every
    layer, q and out, the appended rows and the Forecast vectors, summed."""
    w = WORKLOADS[name]
    ab = algorithmic_bytes(w)
    assert ab["total"] == pytest.approx(ab["ck"] + ab["kv"] + ab["qo"] + ab["append"] + ab["f"])
    pairs, e, d = w.batch * w.num_kv_heads, w.elem_bytes, w.head_dim
    nc = (w.seq_len - w.cmp_kernel) // w.cmp_stride + 1
    if w.token_index:
        assert ab["ck"] == pairs * w.seq_len * d * e  # every key of the index layer is scored
    else:
        assert ab["ck"] == pairs * nc * d * e * len(w.anchors)
    assert ab["f"] == (pairs * d * e if w.forecast else 0)
    if name == "gqa4-bf16-128k-b16":
        assert ab["total"] == 558071808   # 268.40 MB of compressed keys + 289.41 MB of K/V + q, out


@pytest.mark.parametrize("name", ["forecast-bf16-128k-b16", "anchors-2of4-64k-b8", "gqa4-bf16-32k-b1",
                                  "lookahead-bf16-128k-b16", "prefill-bf16-32k-b4", "clsa-4x32k-b8"])
def test_cpu_oracle_leg_runs(name):
    """The bench's CPU-baseline / reference leg (the oracle on a bounded sample of pairs) for the
    Forecast-indexer, anchored, lookahead, prefill and plain workloads, on a shortened copy of each."""
    import torch
    from block_sparse_attention_compressed_b200.workloads import generate
    w = WORKLOADS[name].replace(batch=1, seq_len=4096, needles=2)
    if w.prefill_chunk:
        w = w.replace(prefill_chunk=96)
    data = generate(w, device="cpu")
    if w.prefill_chunk:
        data["q_chunk"] = torch.randn(w.batch, w.prefill_chunk, w.num_q_heads, w.head_dim).to(w.torch_dtype)
    c = bench.cpu_oracle_sample(w, data, seconds=0.05)
    assert c["value"] > 0 and c["single_thread_value"] > 0 and c["cores"] >= 1
    assert c["compress_s_per_cache"] >= 0
    assert "pairs" in c["sample"] and "compressed beforehand" in c["sample"]


def test_bench_starts_its_own_ranks():
    """`bench.py --gpus 2` without a launcher starts two ranks itself (gloo here, no GPU): the
    reference arm prints one JSON line, from rank 0, with n_gpus 2."""
    import json
    import subprocess
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl",
                        "reference", "--workload", "tiny-f32-2k", "--steps", "1", "--warmup", "0",
                        "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference"


def test_bench_refuses_a_mismatched_world():
    """Under a launcher whose WORLD_SIZE differs from --gpus the script stops at once."""
    import subprocess
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl",
                        "reference", "--workload", "tiny-f32-2k"], capture_output=True, text=True,
                       timeout=300, cwd=ROOT, env=env)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr


def test_forecast_vectors_are_group_mean_queries():
    """The synthetic Forecast vector of each (batch, kv head) is the mean of the group's query
    vectors of the first layer, stored in the cache type; other workloads carry none."""
    import torch
    from block_sparse_attention_compressed_b200.workloads import generate
    w = WORKLOADS["forecast-bf16-128k-b16"].replace(batch=2, seq_len=2048, needles=2)
    d = generate(w, device="cpu")
    f = d["f"]
    assert f.shape == (w.batch, w.num_kv_heads, w.head_dim) and f.dtype == w.torch_dtype
    q = d["q"][0].float().view(w.batch, w.num_kv_heads, w.group, w.head_dim)
    assert torch.equal(f, q.mean(dim=2).to(w.torch_dtype))
    assert "f" not in generate(WORKLOADS["gqa4-bf16-32k-b1"].replace(seq_len=1024, needles=0))
