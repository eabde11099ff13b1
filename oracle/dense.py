"""Dense fused-attention forward, written as its plain definition in fp64.

Definition (npu_fusion_attention guide, "昇腾 NPU 融合注意力算子详解与迁移指南",
§2 算子数学原理):

    Attention(Q, K, V) = Dropout(Softmax(Mask(Q·Kᵀ·scale + pse)))·V

with keep_prob = 1 (no dropout).  The score matrix S is materialised here (the
tiled kernel never does that; §2 says the fused operator avoids storing it).

Readings where the guide is silent (each also listed in the design notes):

* atten_mask: 1 = masked, 0 = kept (§4.2); shapes SS, B1SS, BNSS (§4.2).
* sparse_mode (§4.3): 0 keeps (i, j) with i - pre_tokens <= j <= i + next_tokens
  (0-based, aligned at the top-left) combined with atten_mask; 2 keeps j <= i
  (causal, top-left vertex); 3 keeps j <= i + (S_kv - S_q) (causal, bottom-right
  vertex), evaluated per sequence for TND.  Modes 2 and 3 ignore pre/next/atten_mask.
* pse is added after the scale, exactly as the formula places it (§2), shape
  [B or 1, N_q, S_q, S_kv].
* TND: actual_seq_qlen / actual_seq_kvlen are cumulative end offsets, no leading 0
  (§4.3 "累加长度"); sequence b spans rows [cum[b-1], cum[b]).
* GQA (§7): query head h reads key/value head h // (N_q / N_kv).
* A row with no kept key returns O = 0, softmax_max = -inf, softmax_sum = 0.
* softmax_max is the row maximum of the masked score S (natural-log domain) and
  softmax_sum = Σ_j exp(S_ij - softmax_max_i) (§5 names both as the softmax's max
  and sum intermediates).

Parity pins (tests): a pure-Python triple loop on tiny shapes; torch's
scaled_dot_product_attention (float64, CPU) on the unmasked and top-left-causal
special cases; Q = 0 giving uniform weights whose softmax_sum is the integer count
of kept keys; constant V returning V; one kept key returning that key's V.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64

INF_TOKENS = 2147483647


# --------------------------------------------------------------------------------------
# mask
# --------------------------------------------------------------------------------------

def allowed(sq: int, skv: int, sparse_mode: int, pre_tokens: int = INF_TOKENS,
            next_tokens: int = INF_TOKENS, atten_mask2d=None) -> np.ndarray:
    """Boolean [sq, skv]: True where query row i may attend to key column j (§4.2, §4.3)."""
    i = np.arange(sq, dtype=np.int64)[:, None]
    j = np.arange(skv, dtype=np.int64)[None, :]
    if sparse_mode == 0:
        ok = (j >= i - np.int64(pre_tokens)) & (j <= i + np.int64(next_tokens))
        if atten_mask2d is not None:
            ok = ok & (np.asarray(atten_mask2d) == 0)
    elif sparse_mode == 2:
        ok = j <= i
    elif sparse_mode == 3:
        ok = j <= i + (skv - sq)
    else:
        raise ValueError(f"sparse_mode {sparse_mode} is outside {{0, 2, 3}}")
    return np.broadcast_to(ok, (sq, skv)).copy()


# --------------------------------------------------------------------------------------
# one (batch, head) slice
# --------------------------------------------------------------------------------------

def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, ok: np.ndarray,
           pse: np.ndarray | None = None, row_chunk: int = 1024):
    """fp64 attention of one head: q [sq, d], k [skv, d], v [skv, dv], ok [sq, skv].

    Returns (O [sq, dv], softmax_max [sq], softmax_sum [sq]).  Rows are processed in
    chunks only to bound memory; every row's softmax runs over its full key set.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    sq = q.shape[0]
    out = np.zeros((sq, v.shape[1]))
    mx = np.full(sq, -np.inf)
    sm = np.zeros(sq)
    for r0 in range(0, sq, row_chunk):
        r1 = min(sq, r0 + row_chunk)
        s = (q[r0:r1] @ k.T) * scale
        if pse is not None:
            s = s + np.asarray(pse[r0:r1], dtype=np.float64)
        s = np.where(ok[r0:r1], s, -np.inf)
        m = s.max(axis=1) if s.shape[1] else np.full(r1 - r0, -np.inf)
        live = np.isfinite(m)
        e = np.exp(s - np.where(live, m, 0.0)[:, None])
        e = np.where(ok[r0:r1], e, 0.0)
        tot = e.sum(axis=1)
        w = e / np.where(live, tot, 1.0)[:, None]
        out[r0:r1] = w @ v
        mx[r0:r1] = m
        sm[r0:r1] = np.where(live, tot, 0.0)
    return out, mx, sm


def attend_loops(q, k, v, scale, ok, pse=None):
    """The same head computed with explicit Python loops (tiny inputs only)."""
    import math
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    sq, d = q.shape
    skv, dv = v.shape
    out = np.zeros((sq, dv))
    mx = np.full(sq, -np.inf)
    sm = np.zeros(sq)
    for i in range(sq):
        scores = []
        for j in range(skv):
            if not ok[i, j]:
                continue
            t = 0.0
            for c in range(d):
                t += q[i, c] * k[j, c]
            t = t * scale + (float(pse[i, j]) if pse is not None else 0.0)
            scores.append((j, t))
        if not scores:
            continue
        m = max(t for _, t in scores)
        tot = sum(math.exp(t - m) for _, t in scores)
        for j, t in scores:
            w = math.exp(t - m) / tot
            for c in range(dv):
                out[i, c] += w * v[j, c]
        mx[i] = m
        sm[i] = tot
    return out, mx, sm


# --------------------------------------------------------------------------------------
# layouts
# --------------------------------------------------------------------------------------

def _as_f64(x):
    x = np.asarray(x)
    return bf16_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)


def _seq_bounds(cum):
    ends = [int(c) for c in cum]
    starts = [0] + ends[:-1]
    return list(zip(starts, ends))


def attention_forward(q, k, v, *, layout: str, scale: float, sparse_mode: int = 0,
                      pre_tokens: int = INF_TOKENS, next_tokens: int = INF_TOKENS,
                      atten_mask=None, pse=None, actual_seq_qlen=None, actual_seq_kvlen=None,
                      heads=None, q_rows=None):
    """Oracle of the whole operator on bf16 (uint16 bit patterns) or float inputs.

    layout "BNSD": q [B, Nq, Sq, D], k/v [B, Nkv, Skv, D]
    layout "BSND": q [B, Sq, Nq, D], k/v [B, Skv, Nkv, D]
    layout "TND" : q [Tq, Nq, D],    k/v [Tkv, Nkv, D], with cumulative lengths.
    atten_mask: uint8/bool, 1 = masked; shape [Sq, Skv], [B, 1, Sq, Skv] or [B, Nq, Sq, Skv].
    pse: [B or 1, Nq, Sq, Skv] (BNSD/BSND only).

    Returns (out, softmax_max, softmax_sum) in fp64: out in q's layout; stats
    [B, Nq, Sq] (BNSD/BSND) or [Nq, Tq] (TND).  ``heads`` (list of (b, h)) and
    ``q_rows`` (array of query rows, per sequence for TND) restrict the work for
    sampled checks; entries not computed stay NaN.
    """
    qf, kf, vf = _as_f64(q), _as_f64(k), _as_f64(v)
    if layout == "BSND":
        qf, kf, vf = (np.swapaxes(t, 1, 2) for t in (qf, kf, vf))
    if layout in ("BNSD", "BSND"):
        B, Nq, Sq, D = qf.shape
        Nkv, Skv = kf.shape[1], kf.shape[2]
        seqs = [((0, Sq), (0, Skv))] * B
    elif layout == "TND":
        Nq, D = qf.shape[1], qf.shape[2]
        Nkv = kf.shape[1]
        qb, kb = _seq_bounds(actual_seq_qlen), _seq_bounds(actual_seq_kvlen)
        assert len(qb) == len(kb)
        seqs = list(zip(qb, kb))
        B = len(seqs)
    else:
        raise ValueError(layout)
    if Nq % Nkv:
        raise ValueError("N_q must be a multiple of N_kv")
    group = Nq // Nkv
    Dv = vf.shape[-1]

    out = np.full(qf.shape[:-1] + (Dv,), np.nan)
    if layout == "TND":
        smax = np.full((Nq, qf.shape[0]), np.nan)
    else:
        smax = np.full((B, Nq, qf.shape[2]), np.nan)
    ssum = np.full_like(smax, np.nan)

    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(Nq)]
    am = None if atten_mask is None else np.asarray(atten_mask)
    for b, h in sel:
        g = h // group
        (q0, q1), (k0, k1) = seqs[b]
        sq, skv = q1 - q0, k1 - k0
        if layout == "TND":
            qh, kh, vh = qf[q0:q1, h], kf[k0:k1, g], vf[k0:k1, g]
        else:
            qh, kh, vh = qf[b, h], kf[b, g], vf[b, g]
        m2d = None
        if am is not None and sparse_mode == 0:
            if am.ndim == 2:
                m2d = am[:sq, :skv]
            elif am.shape[1] == 1:
                m2d = am[b, 0]
            else:
                m2d = am[b, h]
        ok = allowed(sq, skv, sparse_mode, pre_tokens, next_tokens, m2d)
        p2d = None
        if pse is not None:
            pf = _as_f64(pse)
            p2d = pf[0 if pf.shape[0] == 1 else b, h]
        rows = np.arange(sq) if q_rows is None else np.asarray(q_rows)
        rows = rows[rows < sq]
        o, mx, sm = attend(qh[rows], kh, vh, scale, ok[rows], None if p2d is None else p2d[rows])
        if layout == "TND":
            out[q0 + rows, h] = o
            smax[h, q0 + rows] = mx
            ssum[h, q0 + rows] = sm
        else:
            out[b, h, rows] = o
            smax[b, h, rows] = mx
            ssum[b, h, rows] = sm
    if layout == "BSND":
        out = np.swapaxes(out, 1, 2)
    return out, smax, ssum


# --------------------------------------------------------------------------------------
# K-tile sets of a 128 x 128 tiling (what a tiled kernel must visit)
# --------------------------------------------------------------------------------------

def tile_sets(sq: int, skv: int, sparse_mode: int, pre_tokens: int = INF_TOKENS,
              next_tokens: int = INF_TOKENS, tile: int = 128):
    """Per q-tile: (visited, partial) sets of k-tiles, by brute force over the element mask.

    visited = k-tiles holding at least one kept (i, j) for a row i of the q-tile;
    partial = visited k-tiles that also hold a masked (i, j) inside [0, sq) x [0, skv),
    or that reach past skv.  Computed from ``allowed`` only (atten_mask excluded).
    """
    ok = allowed(sq, skv, sparse_mode, pre_tokens, next_tokens)
    res = []
    for qt in range(-(-sq // tile)):
        r = ok[qt * tile: (qt + 1) * tile]
        vis, part = [], []
        for kt in range(-(-skv // tile)):
            blk = r[:, kt * tile: (kt + 1) * tile]
            if blk.any():
                vis.append(kt)
                if (not blk.all()) or (kt + 1) * tile > skv:
                    part.append(kt)
        res.append((vis, part))
    return res
