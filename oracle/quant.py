"""Quantized block-sparse attention forward (EagleQBSA), step by step in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing in the product path
imports this module.

Source: EagleQBSA article, "昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍".

* Section "EagleQBSA量化叠加稀疏方案设计" and Fig 2.1: Q and K are quantised to
  INT8, symmetric and linear, one scale per 128-token block of the sequence axis;
  V is quantised to FP8 E4M3 with one scale per channel (head-dim column) covering
  the whole sequence; the attention map P is rounded to FP8 before P·V.
* Section "昇腾亲和的量化叠加稀疏Attention算子优化": P is held in floating point
  (FP16 there) and converted to FP8; the conversion rounds each weight's mantissa at
  its own binary exponent.
* Section "MindIE SD调用方式": the operator receives the INT8 query/key, the E4M3
  value bytes, query_scale / key_scale / value_scale, a block_sparse_mask with
  block_shape [128, 128], scale_value (the softmax scale, 128^-0.5 in the example)
  and num_key_value_heads; the output is bf16.
* Section "背景介绍": only the selected blocks of the attention map are computed.

Readings where the article is silent (each also listed in the design notes):

* Quantiser: a = max |x| over the block (or channel) in float32; scale s = a / 127
  (INT8) or a / 448 (E4M3) in float32, and s = 1 when a = 0; INT8 codes are
  rint_half_even(x / s) clamped to [-127, 127]; E4M3 codes are x / s rounded to
  nearest even with saturation.  A tail block (S % 128 != 0) gets its own scale.
* Shapes: query_scale [B, N_q, ceil(S_q/128)], key_scale [B, N_kv, ceil(S_kv/128)],
  value_scale [B, N_kv, D]; block_sparse_mask uint8 [B, N_q, ceil(S_q/128),
  ceil(S_kv/128)] with 1 = compute the block.
* Score: s = t * s_q * s_k * scale, t the exact integer dot product of the INT8 rows.
* P is held in FP16 before its FP8 rounding, the precision the article gives for P
  (section "昇腾亲和的量化叠加稀疏Attention算子优化": the FP16 P matrix is converted
  to FP8): p8 = E4M3(FP16(p)), both nearest even; the FP8 decision is taken on the
  FP16 value on both sides.
* l = Σ p8, the sum of the ROUNDED weights (so constant V returns V exactly);
  O[:, c] = acc[:, c] / l · v_scale[c] with acc = Σ p8 · v8.
* A row with no kept block returns O = 0, softmax_max = -inf, softmax_sum = 0.

Which maximum p is taken against decides the FP8 codes, and the article does not say.
Two readings are written out here:

* ``qbsa_forward`` -- the plain online-softmax definition.  Kept blocks are visited
  in ascending key order, one 128-key block per step; the running max m (natural-log
  units) moves at every block, m_new = max(m, rowmax s); the accumulated l and acc
  are multiplied by e^(m - m_new) at every step; the block's weights are
  p8 = E4M3(FP16(e^(s - m_new))).  softmax_max = final m, softmax_sum = final l.
  No choice made for a kernel's speed enters it.
* ``qbsa_forward_pow2ref`` -- the reading the CUDA kernel takes.  The same visit
  order, but the weights are taken against a power-of-two reference R (an integer in
  log2 units, z = s · log2 e) that follows the running max lazily: at a block,
  m = max(m, rowmax z); if R is unset or m > R + 8, R = ceil(m) and l, acc are
  multiplied by the exact power of two 2^(R_old - R).  Then p8 = E4M3(FP16(2^(z - R)))
  with 2^(z - R) <= 2^8 (below E4M3's 448).  softmax_sum = l · 2^(R - m): the rounded
  weights' sum against the true row maximum.  Because R is a power of two, E4M3
  rounding commutes with every rescale, so the codes equal those against the last
  reference except for weights in E4M3's subnormal range; against the plain reading
  they differ by one rounding of each weight on a shifted grid, well inside the
  quantized tolerance.

Parity pins (tests): the quantiser codes meet the rounding bound |x - q s| <= s/2 and
hit ±127 at the block maximum; the E4M3 codec matches the OCP definition on every
code and torch's float8_e4m3fn cast on finite inputs, and the FP16 -> E4M3 double
rounding matches torch's float16 -> float8_e4m3fn casts on a dense grid; for both
readings, with P rounding switched off the result equals the direct softmax over the
kept blocks, q = 0 gives p8 = 1, softmax_sum = the kept-key count and O = the mean of
the dequantised V, constant V returns V, a pure-Python loop version agrees on tiny
inputs, and masked-out blocks have no influence; the plain reading with a single kept
block per row equals the closed form E4M3(FP16(e^(s - max s))), and both readings lie
within the per-weight E4M3 bound of the unrounded softmax.  The article prints no
quantisation error figure ("parity unpinned" for the article's own error level; only
VBench scores are given, out of scope).
"""

from __future__ import annotations

import math

import numpy as np

from .formats import bf16_to_f64, e4m3_encode, e4m3_decode

BLK = 128
LOG2E = 1.0 / math.log(2.0)
REF_SLACK = 8  # pow2 reading: the reference is re-set once the running max exceeds it by more than 8 (log2 units)


# --------------------------------------------------------------------------------------
# quantisers
# --------------------------------------------------------------------------------------

def _f32_values(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return bf16_to_f64(x).astype(np.float32)
    return x.astype(np.float32)


def quantize_qk_per_block(x, block: int = BLK):
    """x [B, N, S, D] (bf16 bits or float32) -> (int8 codes [B, N, S, D], float32 scales [B, N, nblk])."""
    xf = _f32_values(x)
    B, N, S, D = xf.shape
    nblk = -(-S // block)
    codes = np.zeros((B, N, S, D), dtype=np.int8)
    scales = np.zeros((B, N, nblk), dtype=np.float32)
    for kb in range(nblk):
        r0, r1 = kb * block, min(S, (kb + 1) * block)
        blk = xf[:, :, r0:r1, :]
        a = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        s = np.where(a == 0, np.float32(1.0), a / np.float32(127.0)).astype(np.float32)
        q = np.rint(blk / s[:, :, None, None])
        codes[:, :, r0:r1, :] = np.clip(q, -127, 127).astype(np.int8)
        scales[:, :, kb] = s
    return codes, scales


def quantize_v_per_channel(v):
    """v [B, N, S, D] (bf16 bits or float32) -> (E4M3 codes uint8 [B, N, S, D], float32 scales [B, N, D])."""
    vf = _f32_values(v)
    a = np.abs(vf).max(axis=2).astype(np.float32)
    s = np.where(a == 0, np.float32(1.0), a / np.float32(448.0)).astype(np.float32)
    codes = e4m3_encode((vf / s[:, :, None, :]).astype(np.float32))
    return codes, s


# --------------------------------------------------------------------------------------
# the forward
# --------------------------------------------------------------------------------------

def _fp8_weights(p):
    """p (fp64, >= 0) -> E4M3(FP16(p)) as fp64: the weight held in FP16, then rounded to FP8."""
    return e4m3_decode(e4m3_encode(p.astype(np.float16).astype(np.float32)))


def _block_scores(qi, k8, qs_b, ks_b, scale, c0, c1):
    """s = t · s_q · s_k · scale for one kept key block, t the exact integer dot products."""
    t = qi @ k8[c0:c1].astype(np.int64).T
    return t.astype(np.float64) * (float(qs_b) * float(ks_b) * scale)


def _log2_scale_f32(scale):
    """scale·log2(e) as the kernel's host code forms it: both factors in f32, one f32 product."""
    return np.float32(np.float32(scale) * np.float32(LOG2E))


def _block_products_f32(qi, k8, qs_b, ks_b, sl, c0, c1):
    """For the kernel's reading: t and c = f32(f32(s_q·s_k)·sl) for one kept key block, and
    the exact products t·c (|t| < 2^21 times a 24-bit c is exact in fp64)."""
    t = qi @ k8[c0:c1].astype(np.int64).T
    c = np.float32(np.float32(np.float32(qs_b) * np.float32(ks_b)) * sl)
    return t.astype(np.float64) * float(c)


def _head_plain(q8, k8, qs, ks, v8f, vs, mask_rows, scale, qbs, round_p=True):
    """Plain online-softmax reading for one (b, h): running max moved and l, acc rescaled
    at every kept block; weights E4M3(FP16(e^(s - m))) against that running max."""
    skv, D = k8.shape[0], v8f.shape[1]
    outs, mxs, sms = [], [], []
    for qb in qbs:
        r0, r1 = qb * BLK, min(q8.shape[0], (qb + 1) * BLK)
        rows = r1 - r0
        qi = q8[r0:r1].astype(np.int64)
        m = np.full(rows, -np.inf)     # running max of s (natural-log units)
        l = np.zeros(rows)
        acc = np.zeros((rows, D))
        for kb in np.nonzero(mask_rows[qb])[0]:                               # ascending
            c0, c1 = kb * BLK, min(skv, (kb + 1) * BLK)
            s = _block_scores(qi, k8, qs[qb], ks[kb], scale, c0, c1)
            m_new = np.maximum(m, s.max(axis=1))
            alpha = np.exp(m - m_new)                                          # 0 while m = -inf
            p = np.exp(s - m_new[:, None])
            if round_p:
                p = _fp8_weights(p)
            l = l * alpha + p.sum(axis=1)
            acc = acc * alpha[:, None] + p @ v8f[c0:c1]
            m = m_new
        live = l > 0
        outs.append(np.where(live[:, None], acc / np.where(live, l, 1.0)[:, None], 0.0) * vs[None, :])
        mxs.append(m)
        sms.append(np.where(live, l, 0.0))
    return outs, mxs, sms


def _head_pow2ref(q8, k8, qs, ks, v8f, vs, mask_rows, scale, qbs, round_p=True):
    """Kernel's reading for one (b, h): weights E4M3(FP16(2^(z - R))) against a lazily moved
    power-of-two reference R (re-set to ceil(m) only when m passes R + REF_SLACK).

    The FP16 and E4M3 codes of each weight are decided on z, so z is formed in the kernel's
    precision: c = s_q·s_k·scale·log2(e) in f32 (as the kernel forms it), the block maximum
    as f32(t_max·c), and z − R = f32(t·c − R) with one rounding (a fused multiply-add).
    2^(z − R) itself is exact here (the kernel's ex2.approx differs from it only in the last
    bits of f32)."""
    skv, D = k8.shape[0], v8f.shape[1]
    sl = _log2_scale_f32(scale)
    outs, mxs, sms = [], [], []
    for qb in qbs:
        r0, r1 = qb * BLK, min(q8.shape[0], (qb + 1) * BLK)
        rows = r1 - r0
        qi = q8[r0:r1].astype(np.int64)
        m = np.full(rows, -np.inf)     # running max of z (log2 units)
        ref = np.full(rows, -np.inf)   # power-of-two reference R (an integer)
        l = np.zeros(rows)
        acc = np.zeros((rows, D))
        for kb in np.nonzero(mask_rows[qb])[0]:                               # ascending
            c0, c1 = kb * BLK, min(skv, (kb + 1) * BLK)
            tc = _block_products_f32(qi, k8, qs[qb], ks[kb], sl, c0, c1)
            m = np.maximum(m, tc.max(axis=1).astype(np.float32).astype(np.float64))
            upd = np.isneginf(ref) | (m > ref + REF_SLACK)
            new_ref = np.where(upd, np.ceil(m), ref)
            unset = np.isneginf(ref)
            alpha = np.where(unset, 0.0, np.exp2(np.where(unset, 0.0, ref) - new_ref))  # exact powers of two
            l, acc, ref = l * alpha, acc * alpha[:, None], new_ref
            p = np.exp2((tc - ref[:, None]).astype(np.float32).astype(np.float64))
            if round_p:
                p = _fp8_weights(p)
            l = l + p.sum(axis=1)
            acc = acc + p @ v8f[c0:c1]
        live = l > 0
        outs.append(np.where(live[:, None], acc / np.where(live, l, 1.0)[:, None], 0.0) * vs[None, :])
        mxs.append(m / LOG2E)
        sms.append(np.where(live, l * np.exp2(np.where(live, ref, 0.0) - np.where(live, m, 0.0)), 0.0))
    return outs, mxs, sms


def _forward(head_fn, q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale, heads, q_blocks, round_p):
    q8 = np.asarray(q8)
    k8 = np.asarray(k8)
    B, Nq, Sq, D = q8.shape
    Nkv = k8.shape[1]
    group = Nq // Nkv
    nqb = -(-Sq // BLK)
    out = np.full((B, Nq, Sq, D), np.nan)
    smax = np.full((B, Nq, Sq), np.nan)
    ssum = np.full((B, Nq, Sq), np.nan)
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(Nq)]
    qbs = list(range(nqb)) if q_blocks is None else list(q_blocks)
    v8f_cache = {}
    for b, h in sel:
        g = h // group
        if (b, g) not in v8f_cache:
            v8f_cache[(b, g)] = e4m3_decode(v8[b, g])
        o, mx, sm = head_fn(q8[b, h], k8[b, g], q_scale[b, h], k_scale[b, g], v8f_cache[(b, g)],
                            np.asarray(v_scale[b, g], dtype=np.float64), block_mask[b, h], scale, qbs, round_p)
        for qb, oo, mm, ss in zip(qbs, o, mx, sm):
            r0, r1 = qb * BLK, min(Sq, (qb + 1) * BLK)
            out[b, h, r0:r1] = oo
            smax[b, h, r0:r1] = mm
            ssum[b, h, r0:r1] = ss
    return out, smax, ssum


def qbsa_forward(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale: float,
                 heads=None, q_blocks=None, round_p: bool = True):
    """Oracle of the quantized block-sparse forward (BNSD), plain online-softmax reading.

    q8 [B, Nq, Sq, D] int8; k8 [B, Nkv, Skv, D] int8; q_scale [B, Nq, ceil(Sq/128)];
    k_scale [B, Nkv, ceil(Skv/128)]; v8 [B, Nkv, Skv, D] E4M3 codes (uint8);
    v_scale [B, Nkv, D]; block_mask [B, Nq, ceil(Sq/128), ceil(Skv/128)] uint8, 1 = compute.

    Returns (out [B, Nq, Sq, D], softmax_max [B, Nq, Sq], softmax_sum [B, Nq, Sq]) in
    fp64.  ``heads`` / ``q_blocks`` restrict the work for sampled checks (other entries
    NaN).  ``round_p=False`` skips the FP8 rounding of P (used only by a pin).
    """
    return _forward(_head_plain, q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale, heads, q_blocks,
                    round_p)


def qbsa_forward_pow2ref(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale: float,
                         heads=None, q_blocks=None, round_p: bool = True):
    """The same forward with the weights taken against the lazily moved power-of-two
    reference (the CUDA kernel's reading; module docstring).  Same arguments and returns."""
    return _forward(_head_pow2ref, q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale, heads, q_blocks,
                    round_p)


def _loops(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale, pow2ref):
    q8 = np.asarray(q8)
    k8 = np.asarray(k8)
    B, Nq, Sq, D = q8.shape
    Nkv, Skv = k8.shape[1], k8.shape[2]
    group = Nq // Nkv
    out = np.zeros((B, Nq, Sq, D))
    smax = np.full((B, Nq, Sq), -np.inf)
    ssum = np.zeros((B, Nq, Sq))
    for b in range(B):
        for h in range(Nq):
            g = h // group
            for i in range(Sq):
                qb = i // BLK
                m, ref, l = -math.inf, -math.inf, 0.0
                acc = [0.0] * D
                for kb in range(block_mask.shape[3]):
                    if not block_mask[b, h, qb, kb]:
                        continue
                    cols = range(kb * BLK, min(Skv, (kb + 1) * BLK))
                    ts = [sum(int(q8[b, h, i, c]) * int(k8[b, g, j, c]) for c in range(D)) for j in cols]
                    s = [t * (float(q_scale[b, h, qb]) * float(k_scale[b, g, kb]) * scale) for t in ts]
                    if pow2ref:
                        # the kernel's precision: f32 c, f32 block max, z - R rounded once to f32
                        cf = float(np.float32(np.float32(np.float32(q_scale[b, h, qb]) * np.float32(k_scale[b, g, kb]))
                                              * np.float32(np.float32(scale) * np.float32(LOG2E))))
                        m = max(m, max(float(np.float32(t * cf)) for t in ts))
                        if ref == -math.inf or m > ref + REF_SLACK:
                            new_ref = math.ceil(m)
                            alpha = 0.0 if ref == -math.inf else 2.0 ** (ref - new_ref)
                            l *= alpha
                            acc = [a * alpha for a in acc]
                            ref = new_ref
                        ws = [2.0 ** float(np.float32(t * cf - ref)) for t in ts]
                    else:
                        m_new = max(m, max(s))
                        alpha = 0.0 if m == -math.inf else math.exp(m - m_new)
                        l *= alpha
                        acc = [a * alpha for a in acc]
                        m = m_new
                        ws = [math.exp(sj - m) for sj in s]
                    for j, w in zip(cols, ws):
                        p16 = np.float16(w)                                   # P held in FP16 first
                        p = float(e4m3_decode(e4m3_encode(np.float32(p16))))
                        l += p
                        vrow = e4m3_decode(v8[b, g, j])
                        for c in range(D):
                            acc[c] += p * vrow[c]
                if l > 0:
                    for c in range(D):
                        out[b, h, i, c] = acc[c] / l * float(v_scale[b, g, c])
                    if pow2ref:
                        smax[b, h, i] = m / LOG2E
                        ssum[b, h, i] = l * 2.0 ** (ref - m)
                    else:
                        smax[b, h, i] = m
                        ssum[b, h, i] = l
    return out, smax, ssum


def qbsa_forward_loops(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale: float):
    """``qbsa_forward`` with explicit Python loops over rows and keys (tiny inputs)."""
    return _loops(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale, pow2ref=False)


def qbsa_forward_pow2ref_loops(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale: float):
    """``qbsa_forward_pow2ref`` with explicit Python loops over rows and keys (tiny inputs)."""
    return _loops(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale, pow2ref=True)


# --------------------------------------------------------------------------------------
# how far the power-of-two reading may lie from the plain one
# --------------------------------------------------------------------------------------

# Relative error of one weight held in FP16 and then rounded to E4M3 in E4M3's normal
# range: half the E4M3 spacing, 2^-4, plus the FP16 step (2^-11 of the value) and slack
# for ex2.approx and the fp32 score arithmetic of a kernel.
P_ROUND_EPS = 2.0 ** -4 + 2.0 ** -10


def pow2ref_weight_error(w):
    """Largest |a - w| for one weight of the power-of-two reading, in units of the row max.

    w = e^(s - max s) is the exact weight.  The reading rounds x = w · 2^(m - R) with the
    row's log2 max m and R - m in [-8, 1) (R = ceil of a running max, moved once m passes
    R + 8), so x >= w / 2 and the error in row-max units is 2^(R - m) <= 2 times the error
    in reference units.  At x >= 2^-6 (E4M3 normal) that error is at most P_ROUND_EPS · x;
    below, the E4M3 spacing is 2^-9, so it is at most min(x, 2^-10) (a value under 2^-10
    rounds to 0) plus the FP16 step.  Hence e(w) = P_ROUND_EPS·w + [w < 2^-5]·min(w, 2^-9),
    with a 1e-3 margin on the threshold and the clamp, and 2^-24 for FP16's subnormal step.
    """
    w = np.asarray(w, dtype=np.float64)
    sub = np.where(w < 2.0 ** -5 * 1.001, np.minimum(1.001 * w, 2.0 ** -9), 0.0)
    return P_ROUND_EPS * w + sub + 2.0 ** -24


def qbsa_reading_gap_terms(q8, k8, q_scale, k_scale, v8, v_scale, block_mask, scale: float, center,
                           heads=None, q_blocks=None):
    """Terms of the bound on |O_a - O_p| between any output O_a whose weights a_i lie within
    pow2ref_weight_error(w_i) of the exact weights and the plain reading's output O_p.

    With A = Σ a_i, W = Σ w_i and O_w the unrounded output (qbsa_forward with round_p=False):
        O_a - O_p = [Σ_i (a_i - w_i)(v_i - O_p) + W (O_w - O_p)] / A,
    since Σ_i a_i (v_i - O_p) = A (O_a - O_p) and Σ_i w_i (v_i - O_p) = W (O_w - O_p).  So
        |O_a - O_p| <= [G + W |O_w - O_p|] / A,   G[c] = Σ_i e(w_i) |v_ic - O_p[c]|,
    and, for the row sums, |A - l_p| <= E + |W - l_p| with E = Σ_i e(w_i).

    ``center`` is O_p (the plain reading's output, [B, Nq, Sq, D]); v_ic is the dequantised
    value e4m3(v8)·v_scale.  Returns (G [B, Nq, Sq, D], E [B, Nq, Sq]) over the rows that
    ``heads`` / ``q_blocks`` select (NaN elsewhere); rows with no kept key get 0.
    """
    q8 = np.asarray(q8)
    k8 = np.asarray(k8)
    B, Nq, Sq, D = q8.shape
    Nkv, Skv = k8.shape[1], k8.shape[2]
    group = Nq // Nkv
    nqb = -(-Sq // BLK)
    G = np.full((B, Nq, Sq, D), np.nan)
    E = np.full((B, Nq, Sq), np.nan)
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(Nq)]
    qbs = list(range(nqb)) if q_blocks is None else list(q_blocks)
    for b, h in sel:
        g = h // group
        vdq = e4m3_decode(v8[b, g]) * np.asarray(v_scale[b, g], dtype=np.float64)[None, :]
        for qb in qbs:
            r0, r1 = qb * BLK, min(Sq, (qb + 1) * BLK)
            kept = np.nonzero(block_mask[b, h, qb])[0]
            if len(kept) == 0:
                G[b, h, r0:r1] = 0.0
                E[b, h, r0:r1] = 0.0
                continue
            qi = q8[b, h, r0:r1].astype(np.int64)
            s = np.concatenate([_block_scores(qi, k8[b, g], q_scale[b, h, qb], k_scale[b, g, kb], scale,
                                              kb * BLK, min(Skv, (kb + 1) * BLK)) for kb in kept], axis=1)
            cols = np.concatenate([np.arange(kb * BLK, min(Skv, (kb + 1) * BLK)) for kb in kept])
            e = pow2ref_weight_error(np.exp(s - s.max(axis=1, keepdims=True)))
            E[b, h, r0:r1] = e.sum(axis=1)
            vk = vdq[cols]
            for i in range(r1 - r0):
                G[b, h, r0 + i] = e[i] @ np.abs(vk - center[b, h, r0 + i][None, :])
    return G, E
