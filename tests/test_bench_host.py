"""Host-side logic of bench.py that decides what the roofline line may claim (no GPU)."""

import hashlib
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()


def test_traffic_is_reported_only_for_the_captured_sources():
    bench = _bench()
    rec = dict(bench.QBSA_NCU_TRAFFIC)
    # pretend the capture was taken on the current sources: traffic scales with the algorithmic bytes
    bench.QBSA_NCU_TRAFFIC = dict(rec, sources={rel: _sha(rel) for rel in rec["sources"]})
    t, src = bench.qbsa_traffic(65536, rec["keep"], 4 * rec["alg_bytes"])
    assert t == 4 * rec["bytes"] and "scaled" in src
    t, src = bench.qbsa_traffic(65536, 0.5, 4 * rec["alg_bytes"])
    assert t is None                                   # no capture at this keep fraction
    # any source change since the capture withdraws the figure
    first = next(iter(rec["sources"]))
    bench.QBSA_NCU_TRAFFIC = dict(rec, sources=dict(bench.QBSA_NCU_TRAFFIC["sources"], **{first: "0" * 40}))
    t, src = bench.qbsa_traffic(65536, rec["keep"], 4 * rec["alg_bytes"])
    assert t is None and "changed" in src


def test_algorithmic_work_of_the_workload():
    bench = _bench()
    inp = dict(N=40, S=65536, D=128, kept=40 * 512 * 51)
    executed, dense_eq, nbytes = bench.qbsa_work(inp)
    assert executed == 4.0 * 128 * 128 * 128 * 40 * 512 * 51     # 4 D 128^2 FLOP per kept block
    assert dense_eq == 4.0 * 128 * 65536 * 65536 * 40
    # Q, K, V bytes read once (int8 / e4m3), bf16 output, mask and scales
    assert nbytes == 3 * 40 * 65536 * 128 + 2 * 40 * 65536 * 128 + 40 * 512 * 512 + 4 * (2 * 40 * 512 + 40 * 128)


def test_step_stats_median_and_cv():
    bench = _bench()
    st = bench.step_stats([1.0, 1.0, 1.0, 1.0])
    assert st["median_ms"] == 1.0 and st["cv"] == 0.0 and st["stable"]
    st = bench.step_stats([1.0, 2.0, 3.0])  # pstdev sqrt(2/3), mean 2
    assert st["median_ms"] == 2.0 and st["min_ms"] == 1.0 and st["max_ms"] == 3.0
    assert abs(st["cv"] - (2.0 / 3.0) ** 0.5 / 2.0) < 1e-12 and not st["stable"]
    assert bench.step_stats([5.0])["cv"] == 0.0


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the CPU oracle (no GPU needed) and prints one JSON
    line with the reference arm's keys."""
    import json
    import subprocess
    import sys
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["metric"] == bench_metric() and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def bench_metric():
    return _bench().METRIC


def test_visited_tiles_count_matches_the_oracle_tile_sets():
    """The executed-FLOP count of the causal and TND lines counts the key tiles the schedule
    visits; it must equal the number of (query tile, key tile) pairs holding a kept element,
    counted by brute force over the element mask."""
    from oracle import dense
    from quantized_block_sparse_attn_b200 import build
    build.build()
    bench = _bench()
    for sq, skv, mode in [(4096, 4096, 3), (1024, 1024, 3), (5000, 5000, 3), (300, 333, 2), (333, 300, 3),
                          (640, 640, 0)]:
        want = sum(len(vis) for vis, _ in dense.tile_sets(sq, skv, mode))
        assert bench._visited_tiles(sq, skv, mode) == want, (sq, skv, mode)
    # causal, equal lengths: tile t visits t + 1 key tiles
    n = 4096 // 128
    assert bench._visited_tiles(4096, 4096, 3) == n * (n + 1) // 2
