"""CPU checks of bench.py's reference arm (the oracle on a bounded sample):
the JSON line's contract, and that under several ranks only rank 0 prints."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")


def _run(args, env_extra=None):
    env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        env.pop(k, None)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       timeout=600, env=env, cwd=ROOT)
    return r


@pytest.mark.parametrize("workload", ["tiny-fp32", "draft-tiny"])
def test_reference_arm_prints_one_contract_line(workload):
    r = _run(["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is False
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == workload


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--workload", "tiny-fp32", "--steps", "1", "--warmup", "0", "--gpus", "2"],
             {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert not [l for l in r.stdout.splitlines() if l.strip().startswith("{")]


def _bench_module():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    return bench


def test_recorded_dram_traffic_names_the_kernel_sources_it_was_taken_on():
    """The traffic figure is reported only while the kernel sources hash to
    the value recorded with it; the hash covers every .cu / .cuh / .h file."""
    bench = _bench_module()
    t = bench.TRAFFIC_PI0_BF16
    assert len(t["kernel_sources_sha256"]) == 64 and int(t["kernel_sources_sha256"], 16) >= 0
    h1, h2 = bench.kernel_sources_sha256(), bench.kernel_sources_sha256()
    assert h1 == h2 and len(h1) == 64
    # DRAM traffic of a chunk cannot be below its algorithmic bytes by more than
    # the cross-step L2 reuse allows, nor far above them without re-reads
    from synthetic import get_config
    cfg = get_config("pi0-bf16")
    alg = bench.algorithmic_bytes_per_step(cfg) * cfg.n_steps
    assert 0.9 <= t["bytes_per_chunk"] / alg <= 1.1


def test_draft_bytes_drop_the_folded_query_projection():
    """On the tensor-core path (bf16) the action queries' q/k/v are computed
    once per graph: a forward reads their tiles instead of the q weights."""
    bench = _bench_module()
    from synthetic import get_draft_config
    d = get_draft_config("flash-draft")
    e, w = 2, d.width
    kv = d.n_vis * 2 * d.kv_dim * e
    unfolded = (d.block_params() - 2 * w) * e + 2 * w * 4 + d.action_dim * (w * e + 4) + d.n_queries * w * 4 + \
        d.n_vis * w * e + 2 * kv
    tiles = (d.n_q_heads // 2) * 128 * d.head_dim * 2 + 2 * d.n_kv_heads * 64 * d.head_dim * 2
    assert bench.draft_bytes(d) == unfolded - w * d.q_dim * e + tiles
    assert 215e6 < bench.draft_bytes(d) < 220e6
