"""bench.py on the CPU: the reference arm (the fp64 oracle on the host cores) keeps the one-JSON-line
contract, and the attention roofline counts the (query, key) pairs the method attends to.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                           "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_json_line():
    r = _run({"RANK": "0"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run({"RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("mode,T,S,g,n_e,bsz", [
    (0, 40, 1000, 2, 0, 0), (0, 30, 60, 3, 0, 0),
    (1, 700, 700, 2, 100, 64), (1, 1000, 1000, 1, 0, 64), (1, 300, 300, 2, 512, 256), (1, 2048, 2048, 2, 256, 96),
    (2, 700, 700, 2, 16, 0), (2, 3000, 3000, 2, 64, 0), (2, 100, 100, 2, 128, 0),
])
def test_roofline_pair_count_is_what_the_oracle_attends(mode, T, S, g, n_e, bsz, monkeypatch):
    """The (query, key) pairs behind the attention roofline's FLOPs equal the pairs the oracle's
    attention actually weighs: its weighted-softmax calls are counted (visible entries of each mask)."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle.thin_oracle as O
    import thinned_softmax_attention_b200 as TA
    import workloads as W

    seen = [0]
    real = O.weighted_attention

    def counting(q, K, V, scale, logw=None, mask=None):
        seen[0] += int(mask.sum()) if mask is not None else q.shape[0] * K.shape[0]
        return real(q, K, V, scale, logw, mask)

    monkeypatch.setattr(O, "weighted_attention", counting)
    w = W.Workload("count", 1, 1, T, S if mode == 0 else T, 8, 8, "fp32", mode > 0, g, 3, 1, "iid",
                   n_exact=n_e, batch=bsz, cache="A" if mode == 2 else "B")
    rng = np.random.default_rng(T + S)
    L = w.S
    q, k, v = rng.normal(size=(1, T, 1, 8)), rng.normal(size=(1, L, 1, 8)), rng.normal(size=(1, L, 1, 8))
    if mode == 0:
        O.thinformer(q, k, v, g, 3)
    elif mode == 1:
        O.express(q, k, v, n_e, bsz, g, 3)
    else:
        O.express_a(q, k, v, n_e, g, 3)
    plan = TA.ThinAttention(1, T, L, 1, 8, 8, w.torch_dtype, n_exact=n_e, batch=bsz).plan(w.mode, g)
    flops, _, pairs = bench.attention_work(w, plan)
    assert pairs == seen[0] > 0
    assert flops == 2.0 * (w.E + w.D) * pairs


@pytest.mark.parametrize("name", ["express32k", "express32k_a", "vit"])
def test_attention_work_of_row_shards_adds_up(name):
    """bench.attention_work over the query-row ranges of --shard seq: the shards' pairs and FLOPs sum
    to the whole launch's, and each shard's q/out bytes are its rows'."""
    import bench
    import thinned_softmax_attention_b200 as T
    import workloads as W
    w = W.WORKLOADS[name]
    plan = T.ThinAttention(w.B, w.T, w.T if w.causal else w.S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact,
                           batch=w.batch).plan(w.mode, w.g)
    full_f, full_b, full_p = bench.attention_work(w, plan)
    fs, ps = 0.0, 0
    for r in range(4):
        rows = bench.Shard(w, 4, r, "seq").rows
        f, b, p = bench.attention_work(w, plan, rows)
        fs += f
        ps += p
        assert b < full_b
    assert ps == full_p and fs == full_f


def test_halving_floors_put_hbm_on_top_at_express32k():
    """The halving launches' three floors (Gram on the tensor cores, one exponential per kernel
    evaluation on MUFU, algorithmic HBM bytes): at Express 32K's level-1 step HBM is the largest, so
    the reported fraction is against the binding one."""
    import bench
    import workloads as W

    class FakeHandle:
        def profile_steps(self):
            return {"calls": 1, "steps": [{"n": 64, "n_inst": 15872, "ms": 0.195}, {"n": 128, "n_inst": 3968, "ms": 0.183},
                                          {"n": 256, "n_inst": 992, "ms": 0.297}, {"n": 512, "n_inst": 224, "ms": 0.0}]}

    w = W.WORKLOADS["express32k"]
    r = bench.halving_roofline(w, FakeHandle(), {"thin_ms": 0.6, "merge_ms": 0.08, "calls": 1}, bench.peaks())
    assert r["bound"] == "hbm"
    for t in r["launches"]:
        f = t["floors_ms"]
        assert f["hbm_ms"] > f["tensor_ms"] and f["hbm_ms"] > f["mufu_ms"]
    lv1 = r["launches"][0]["floors_ms"]
    assert abs(lv1["hbm_ms"] - 780140544 / 6553e9 * 1e3) < 1e-4
