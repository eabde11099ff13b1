"""CPU checks of libqbsa.so: it loads, exports every declared symbol, validates arguments
before touching the GPU, and its tile schedule matches the oracle's brute-force sets."""

import ctypes
import os
import re

import numpy as np
import pytest

import quantized_block_sparse_attn_b200 as qb
from oracle import dense

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qbsa.h")
INF = qb.INF_TOKENS


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_block_sparse_attn_b200 import build
    build.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)) - {"if"})


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert {"attn_fwd", "qbsa_fwd", "qbsa_check", "qbsa_last_error"} <= set(names)
    raw = ctypes.CDLL(qb.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert qb.lib().qbsa_version() == 103  # 1.03: qbsa_fwd_host added


@pytest.mark.parametrize("nkb", [1, 2, 5, 7, 64, 255, 512, 1024, 2048])
@pytest.mark.parametrize("keep", [0.0, 0.05, 0.1, 0.25, 0.3, 0.5, 0.9, 1.0])
def test_block_topk_keep_count_rule(nkb, keep):
    """The kept-block count qbsa_block_topk_keep derives from a keep fraction equals the
    oracle's rule; a null q_mean then stops the call before any launch."""
    from oracle import estimate
    n = ctypes.c_int(-1)
    st = qb.lib().qbsa_block_topk_keep(None, None, 1, 1, 1, 1, nkb, 128, 0.1, keep, None, None, ctypes.byref(n),
                                       None)
    assert st == 1
    assert n.value == estimate.keep_count(nkb, keep)


@pytest.mark.parametrize("keep", [-0.1, 1.5, float("nan")])
def test_block_topk_keep_rejects_bad_fraction(keep):
    n = ctypes.c_int(-1)
    st = qb.lib().qbsa_block_topk_keep(None, None, 1, 1, 1, 1, 8, 128, 0.1, keep, None, None, ctypes.byref(n), None)
    assert st == 1 and n.value == -1


def _attn(**over):
    fake = ctypes.c_void_p(0x10000)
    a = dict(q=fake, k=fake, v=fake, B=1, Nq=2, Nkv=1, Sq=128, Skv=128, D=128, head_num=2, layout=0, mask=None,
             mshape=0, pse=None, bcast=0, scale=0.1, keep=1.0, mode=0, pre=INF, nxt=INF, cq=None, ck=None,
             out=fake, smax=None, ssum=None, stream=None)
    a.update(over)
    st = qb.lib().attn_fwd(a["q"], a["k"], a["v"], a["B"], a["Nq"], a["Nkv"], a["Sq"], a["Skv"], a["D"],
                           a["head_num"], a["layout"], a["mask"], a["mshape"], a["pse"], a["bcast"], a["scale"],
                           a["keep"], a["mode"], a["pre"], a["nxt"], a["cq"], a["ck"], a["out"], a["smax"],
                           a["ssum"], a["stream"])
    return st, qb.lib().qbsa_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(q=None), 1),
    (dict(q=ctypes.c_void_p(0x10004)), 1),
    (dict(head_num=3), 1),
    (dict(Nq=3, Nkv=2, head_num=3), 1),
    (dict(D=96), 2),
    (dict(D=0), 1),
    (dict(keep=0.5), 2),
    (dict(keep=0.0), 1),
    (dict(mode=1), 2),
    (dict(mode=4), 2),
    (dict(layout=7), 1),
    (dict(mshape=1), 1),
    (dict(scale=float("inf")), 1),
    (dict(layout=2), 1),
    (dict(cq=ctypes.c_void_p(0x10000)), 1),
    (dict(B=0), 1),
    (dict(mask=ctypes.c_void_p(0x10000)), 1),                             # a mask without its shape
    (dict(mask=ctypes.c_void_p(0x10000), mshape=5), 1),                   # unknown mask shape
    (dict(pse=ctypes.c_void_p(0x10008)), 1),                              # pse not 16-byte aligned
    (dict(layout=2, mask=ctypes.c_void_p(0x10000), mshape=1), 2),         # atten_mask with TND
    (dict(layout=2, pse=ctypes.c_void_p(0x10000)), 2),                    # pse with TND
])
def test_attn_fwd_rejects_before_launch(over, status):
    st, msg = _attn(**over)
    assert st == status, msg
    assert msg


def test_tnd_lengths_must_be_cumulative_and_match_totals():
    cq = np.array([100, 50], dtype=np.int64)
    ck = np.array([100, 150], dtype=np.int64)
    st, msg = _attn(layout=2, B=2, Sq=150, Skv=150, cq=cq.ctypes.data_as(ctypes.c_void_p),
                    ck=ck.ctypes.data_as(ctypes.c_void_p))
    assert st == 1 and "non-decreasing" in msg
    cq = np.array([100, 140], dtype=np.int64)
    st, msg = _attn(layout=2, B=2, Sq=150, Skv=150, cq=cq.ctypes.data_as(ctypes.c_void_p),
                    ck=ck.ctypes.data_as(ctypes.c_void_p))
    assert st == 1 and "equal" in msg


def test_qbsa_fwd_rejects_before_launch():
    fake = ctypes.c_void_p(0x10000)
    L = qb.lib()
    args = [fake] * 7 + [1, 2, 1, 256, 256, 128, 0.1, fake, None, None, None]
    bad = list(args)
    bad[12] = 64
    assert L.qbsa_fwd(*bad) == 2
    bad = list(args)
    bad[0] = None
    assert L.qbsa_fwd(*bad) == 1
    bad = list(args)
    bad[8], bad[9] = 3, 2
    assert L.qbsa_fwd(*bad) == 1
    bad = list(args)
    bad[11] = 300 * 1024
    assert L.qbsa_fwd(*bad) == 2


def test_qbsa_fwd_host_rejects_before_any_device_work():
    """The host-buffer entry point validates like qbsa_fwd (plus n_chunks) before it touches
    the device, so these calls return without a GPU."""
    fake = ctypes.c_void_p(0x10000)
    L = qb.lib()
    args = [fake] * 7 + [1, 2, 1, 256, 256, 128, 0.1, fake, None, None, 8, None]
    for idx, val, status in [(12, 64, 2), (0, None, 1), (14, None, 1), (8, 3, 1), (11, 300 * 1024, 2),
                             (17, 0, 1), (17, -2, 1), (13, float("nan"), 1)]:
        bad = list(args)
        bad[idx] = val
        if idx == 8:
            bad[9] = 2          # Nq = 3 is not a multiple of Nkv = 2
        st = L.qbsa_fwd_host(*bad)
        assert st == status, (idx, val, qb.lib().qbsa_last_error().decode())


def test_block_estimation_rejects_before_launch():
    fake = ctypes.c_void_p(0x10000)
    L = qb.lib()
    assert L.qbsa_block_mean(fake, 1, 2, 300, 96, fake, None) == 2           # D not in {64, 128, 256}
    assert L.qbsa_block_mean(None, 1, 2, 300, 128, fake, None) == 1
    assert L.qbsa_block_mean(ctypes.c_void_p(0x10008), 1, 2, 300, 128, fake, None) == 1  # misaligned
    args = [fake, fake, 1, 4, 2, 3, 512, 128, 0.1, 51, fake, None, None]
    bad = list(args)
    bad[9] = 0                                                                # n_keep < 1
    assert L.qbsa_block_topk(*bad) == 1
    bad[9] = 513                                                              # n_keep > nkb
    assert L.qbsa_block_topk(*bad) == 1
    bad = list(args)
    bad[4] = 3                                                                # Nq % Nkv != 0
    assert L.qbsa_block_topk(*bad) == 1
    bad = list(args)
    bad[6] = 4096                                                             # nkb above 2048
    assert L.qbsa_block_topk(*bad) == 2


SCHED_CASES = [
    (256, 256, 0, INF, INF), (300, 500, 0, INF, INF), (1000, 1000, 2, INF, INF), (1000, 777, 2, INF, INF),
    (777, 1000, 3, INF, INF), (1000, 777, 3, INF, INF), (129, 1, 3, INF, INF), (1, 129, 3, INF, INF),
    (640, 640, 0, 100, 0), (640, 640, 0, 0, 0), (640, 900, 0, 300, 5), (640, 640, 0, -50, 200),
    (640, 640, 0, 200, -50), (640, 640, 0, -300, 100), (5000, 5000, 3, INF, INF), (512, 1024, 0, 0, 600),
]


@pytest.mark.parametrize("sq,skv,mode,pre,nxt", SCHED_CASES)
def test_tile_schedule_matches_oracle_sets(sq, skv, mode, pre, nxt):
    kb, ke, fb, fe = qb.attn_tile_schedule(sq, skv, mode, pre, nxt)
    ref = dense.tile_sets(sq, skv, mode, pre, nxt)
    for t, (vis, part) in enumerate(ref):
        got_vis = list(range(kb[t], ke[t]))
        got_part = [x for x in got_vis if not (fb[t] <= x < fe[t])]
        assert got_vis == vis, (t, got_vis, vis)
        assert got_part == part, (t, got_part, part)


@pytest.mark.parametrize("fn", ["qbsa_quantize_qk", "qbsa_quantize_v"])
@pytest.mark.parametrize("over,status", [
    (dict(x=None), 1),
    (dict(x=ctypes.c_void_p(0x10002)), 1),
    (dict(codes=ctypes.c_void_p(0x10008)), 1),
    (dict(D=96), 2),
    (dict(D=0), 1),
    (dict(S=0), 1),
])
def test_quantisers_reject_before_launch(fn, over, status):
    fake = ctypes.c_void_p(0x10000)
    a = dict(x=fake, B=1, N=2, S=256, D=128, codes=fake, scales=fake)
    a.update(over)
    st = getattr(qb.lib(), fn)(a["x"], a["B"], a["N"], a["S"], a["D"], a["codes"], a["scales"], None)
    assert st == status, qb.lib().qbsa_last_error().decode()
