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
