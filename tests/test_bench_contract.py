"""The benchmark's reference arm on CPU: the JSON line it prints and its rank handling."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ, **(extra_env or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "0",
                           "--steps", "2", "--warmup", "1"], capture_output=True, text=True, env=env, cwd=ROOT,
                          timeout=300)


def test_reference_arm_line():
    r = _run()
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    sys.path.insert(0, ROOT)
    import bench
    from deepseek_mla_latent_b200 import workloads as wl
    assert line["impl"] == "reference" and line["unit"] == bench.UNIT and line["metric"] == bench.METRIC
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["higher_is_better"] is False and line["value"] > 0
    assert line["config"] == bench.workload_config(wl.workload(0), 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_prefill_flop_count_closed_form():
    """Workload 4: 4 sequences, query i of 1024 sees 3073 + i of 4096 keys, and each (query,
    visible key) pair costs 2 * 128 * (512 + 64 + 512) flop."""
    sys.path.insert(0, ROOT)
    import bench
    from deepseek_mla_latent_b200 import workloads as wl
    _, dims, sq, sk = wl.workload_shape(4)

    class W:
        pass
    w = W()
    w.dims, w.seqlens_q, w.seqlens_k = dims, sq, sk
    pairs = 4 * (1024 * 3073 + 1023 * 1024 // 2)
    assert bench.prefill_attention_flop(w) == pairs * 2 * 128 * (512 + 64 + 512)


def test_naive_prefill_flop_count_closed_form():
    """Workload 4 on the naive path: every one of the 4 x 4096 cache rows is expanded to all heads
    (2 * 128 * 256 * 512 flop per row), and each (query, visible key) pair costs
    2 * 128 * (128 + 64 + 128) flop."""
    sys.path.insert(0, ROOT)
    import bench
    from deepseek_mla_latent_b200 import workloads as wl
    _, dims, sq, sk = wl.workload_shape(4)

    class W:
        pass
    w = W()
    w.dims, w.seqlens_q, w.seqlens_k = dims, sq, sk
    w.total_k = sum(sk)
    pairs = 4 * (1024 * 3073 + 1023 * 1024 // 2)
    ex, at = bench.expanded_prefill_flop(w)
    assert ex == 4 * 4096 * 2 * 128 * 256 * 512
    assert at == pairs * 2 * 128 * (128 + 64 + 128)


def test_committed_attention_profile_matches_the_sources():
    """profiles/attn_decode_v3_decode_b8_t4096.md was captured on the current attention-kernel
    sources (its hash is bench.py's), so the bench line's roofline.traffic is not null; a kernel
    change without a new capture fails here."""
    sys.path.insert(0, ROOT)
    import bench
    traffic = bench.profiled_traffic("v3_decode_b8_t4096")
    assert traffic is not None, "attention profile is stale: recapture it on the current sources"
    # DRAM bytes per launch close to the algorithmic bytes (32768 x 1152 cache + q_abs, q_pe, o_lat)
    alg = 32768 * 1152 + 8 * 128 * (512 + 64 + 512) * 2
    assert 0.9 * alg <= traffic <= 1.1 * alg
