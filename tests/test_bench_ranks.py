"""bench.py on CPU: the N>1 path (two gloo ranks, each a replica, combine
their timings by max and their work by sum, the only collectives), the
algorithmic byte counts against the format arithmetic, and the keys of both
arms' JSON lines (the CUDA arm's assembled from a stand-in measurement)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                      RANK=str(rank), LOCAL_RANK=str(rank), KVQ_BENCH_BACKEND="gloo")
    import bench
    r, ws, dist = bench.dist_setup(2)
    assert (r, ws) == (rank, 2)
    bench.barrier(dist)
    mx = bench.max_over_ranks(dist, [1.0 + rank, 10.0 - rank])
    sm = bench.sum_over_ranks(dist, [3.0, float(rank)])
    q.put((rank, mx, sm))
    dist.destroy_process_group()


def test_two_gloo_ranks_max_and_sum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, sm in got:
        assert mx == [2.0, 10.0]
        assert sm == [6.0, 1.0]


def test_algorithmic_bytes_of_the_int4_workload():
    import bench
    from quantized_kv_cache_14_b200.workloads import workload
    w = workload(3)
    # 8192 quantized tokens: 8 heads x (64 + 64 codes + 2 + 2 scale bytes) per token,
    # no window tokens, plus q (32 x 128 bf16) and out (fp32), plus 512 table entries
    b = bench.decode_bytes(w, [8192])
    assert b == 8192 * 8 * 136 + 32 * 128 * 6 + 512 * 4
    # 16 sequences of 8192 quantized tokens: 142,606,336 bytes of codes and scales
    assert 16 * 8192 * 8 * 136 == 142_606_336
    # 63 window tokens are bf16 rows of K and V
    assert bench.decode_bytes(w, [8192 + 63]) - b == 63 * 8 * 2 * 128 * 2


def test_algorithmic_bytes_of_the_int8_and_int2_workloads():
    import bench
    from quantized_kv_cache_14_b200.workloads import workload
    # INT8 keys and values per token, G = 128, fp16 scales: (128 + 128 codes +
    # 2 + 2 scale bytes) per token and kv head, 16-token pages, no window
    w = workload(2)
    assert bench.decode_bytes(w, [4096]) == 4096 * 8 * 260 + 256 * 4 + 32 * 128 * 6
    # INT2 with fp16 scale and zero-point per group of 32: 32 + 32 code bytes,
    # keys 128 channels x 4 bytes per 32 tokens, values 4 groups x 4 bytes;
    # 31 window tokens as bf16 K and V rows
    w = workload(4)
    assert bench.decode_bytes(w, [131072 + 31]) == (131072 * 8 * 96 + 31 * 8 * 2 * 128 * 2 + 8192 * 4
                                                   + 32 * 128 * 6)


def test_append_bytes_of_a_decode_step():
    import bench
    from quantized_kv_cache_14_b200.workloads import workload
    w = workload(3)
    row = 8 * 128 * 2   # one token's bf16 row over the 8 kv heads
    # no group fills: the new K and V rows read, then written to the window
    assert bench.append_bytes(w, [10]) == 2 * row + 2 * row
    # the 64th token fills the key group: its rows read, the 63 earlier window
    # rows of K and V read again, 64 tokens of codes + value scales written
    # (8 heads x (128 code bytes + 4 scale bytes)) and the group's key scales
    # (8 heads x 128 channels x 2 bytes)
    assert bench.append_bytes(w, [63]) == 2 * row + 2 * row * 63 + 64 * 8 * 132 + 8 * 128 * 2


def test_bulk_append_bytes_of_the_int4_workload():
    import bench
    from quantized_kv_cache_14_b200.workloads import workload
    w = workload(3)
    # 8192 + 17 tokens: every K and V row read once (8 heads x 128 bf16), the
    # 8192 tokens of whole key groups written as codes + scales (136 B per
    # token-head), the 17 window tokens written as bf16 K and V rows
    row = 8 * 128 * 2
    assert bench.bulk_append_bytes(w, [8192 + 17]) == 2 * row * (8192 + 17) + 8192 * 8 * 136 + 2 * row * 17


def test_reference_arm_runs_the_requested_steps():
    """The oracle arm times the same K steps after W warm-up steps as the CUDA
    arm (tiny workload, CPU only) and prints one JSON line of the contract."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "1", "--steps", "4",
                        "--warmup", "3"], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 4 and d["warmup"] == 3
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["metric"] == "decode-attn KV GB/s" and d["higher_is_better"] is True


def test_bench_line_carries_the_contract_keys(monkeypatch, capsys):
    """The JSON line of the CUDA arm, assembled from a stand-in measurement
    (no GPU here): every key of the line's contract is present, `value` is
    the decode GB/s, the roofline divides the attention rate by the peak,
    and e2e declares its copies."""
    import json
    import sys
    import bench
    from quantized_kv_cache_14_b200.workloads import workload
    w = workload(3)
    meas = {"w": w, "K": 20, "launches": 60, "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
            "kv_gbs": 3000.0, "attn_gbs": 3500.0, "attn_bytes_per_launch": 1.455e8, "attn_us": 41.6,
            "decode_us": 48.5, "append_us": 9.4, "append_gbs": 22.0, "seq_tok_s": 2.3e9, "ms_per_step": 0.058,
            "e2e_gbs": 2100.0, "kv_bytes_per_step": 1.455e8, "lens_final": [8192] * 16,
            "h2d": 196608, "d2h": 262144, "bulk": None}
    monkeypatch.setattr(bench, "run_gpu", lambda *a, **k: meas)
    monkeypatch.setattr(bench, "run_oracle_sample", lambda *a, **k: (0.3, 10.0, 3.0e9, [8192] * 16, 16))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "20", "--warmup", "5", "--no-workloads",
                                      "--no-control"])
    bench.main()
    d = json.loads([ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")][-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks"):
        assert key in d, key
    assert d["value"] == 3000.0 and d["unit"] == "GB/s" and d["n_gpus"] == 1 and d["steps"] == 20
    assert d["warmup"] == 5 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert "workload" in d["config"]
    r = d["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    assert r["achieved"] == 3500.0 and abs(r["frac"] - 3500.0 / r["peak"]) < 1e-12
    assert set(d["cpu_baseline"]) >= {"value", "unit", "cores", "kind", "sample"}
    assert d["e2e"] == {"value": 2100.0, "unit": "GB/s", "h2d_bytes_per_step": 196608,
                        "d2h_bytes_per_step": 262144}
    assert d["gpu_launches"] == 60 and set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
