"""ctypes binding of libqbsa.so: argument marshalling only.

Every numeric step runs in the library's CUDA kernels.  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the library has not
been built (``python -m quantized_block_sparse_attn_b200.build``) or the CUDA path
cannot run, calls raise.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB = None
_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqbsa.so")

STATUS = {0: "QBSA_OK", 1: "QBSA_ERR_INVALID", 2: "QBSA_ERR_UNSUPPORTED", 3: "QBSA_ERR_CUDA", 4: "QBSA_ERR_TIMEOUT"}
LAYOUTS = {"BNSD": 0, "BSND": 1, "TND": 2}
MASK_SHAPES = {None: 0, "SS": 1, "B1SS": 2, "BNSS": 3}
INF_TOKENS = 2147483647

# exported symbol -> (restype, argtypes)
_P, _I, _I64, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P, _I, _F, _F, _I, _I64, _I64,
                      _P, _P, _P, _P, _P, _P]),
    "qbsa_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P]),
    "qbsa_fwd_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _I, _P]),
    "bsa_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P]),
    "qbsa_quantize_qk": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "qbsa_quantize_v": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "qbsa_quantize_v_noalloc": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "attn_tile_schedule": (_I, [_I64, _I64, _I, _I64, _I64, _P, _P, _P, _P, _I64]),
    "qbsa_block_lists": (_I, [_P, _I64, _I, _P, _P, _P]),
    "qbsa_block_mean": (_I, [_P, _I, _I, _I, _I, _P, _P]),
    "qbsa_block_topk": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P]),
    "qbsa_block_topk_keep": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _F, ctypes.c_double, _P, _P, _P, _P]),
    "qbsa_wait_selftest": (_I, [_P]),
    "qbsa_check": (_I, [_P]),
    "qbsa_last_error": (ctypes.c_char_p, []),
    "qbsa_version": (_I, []),
}


class QbsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def lib():
    """Load libqbsa.so (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m quantized_block_sparse_attn_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def _ck(status: int):
    if status != 0:
        raise QbsaError(status, lib().qbsa_last_error().decode("utf-8", "replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _on_cuda(tensors, device):
    """Host tensors are copied to the device (pinned, asynchronous); device tensors pass through."""
    import torch
    out = []
    for t in tensors:
        if t is None or t.is_cuda:
            out.append(t)
        else:
            src = t if t.is_pinned() else t.pin_memory()
            out.append(src.to(device, non_blocking=True))
    return out


def _split_outputs(host, outs):
    """In host mode, caller-given output tensors on the host become copy destinations and the kernel writes
    fresh device buffers; otherwise every given output must already be a device tensor."""
    dev_outs, dsts = [], []
    for t in outs:
        if t is not None and not t.is_cuda:
            if not host:
                raise ValueError("output tensors must be on the GPU when the inputs are")
            dev_outs.append(None)
            dsts.append(t)
        else:
            dev_outs.append(t)
            dsts.append(None)
    return dev_outs, dsts


def _to_host(results, dsts, device):
    """Copy device results into pinned host tensors (the caller's or new ones); waits for the copies."""
    import torch
    res = []
    for t, dst in zip(results, dsts):
        if t is None:
            res.append(None)
            continue
        if dst is None:
            dst = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        dst.copy_(t, non_blocking=True)
        res.append(dst)
    torch.cuda.current_stream(device).synchronize()
    return tuple(res)


def attn_fwd(q, k, v, head_num: int, input_layout: str = "BNSD", *, atten_mask=None, mask_shape=None, pse=None,
             scale: float = 1.0, keep_prob: float = 1.0, sparse_mode: int = 0, pre_tokens: int = INF_TOKENS,
             next_tokens: int = INF_TOKENS, actual_seq_qlen=None, actual_seq_kvlen=None, out=None,
             softmax_max=None, softmax_sum=None, return_stats: bool = True, device=None):
    """Dense fused attention forward (bf16).  Returns (attention_out, softmax_max, softmax_sum).

    Tensors may live on the GPU or on the host; host inputs are copied to ``device``
    (default cuda:0) and the results are copied back to the host.
    """
    import torch
    host = not q.is_cuda
    dev = torch.device(device or (q.device if q.is_cuda else "cuda:0"))
    q, k, v, atten_mask, pse = _on_cuda([q, k, v, atten_mask, pse], dev)
    (out, softmax_max, softmax_sum), dsts = _split_outputs(host, (out, softmax_max, softmax_sum))
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bfloat16 tensors")
    lay = LAYOUTS[input_layout]
    if input_layout == "BNSD":
        B, Nq, Sq, D = q.shape
        Nkv, Skv = k.shape[1], k.shape[2]
    elif input_layout == "BSND":
        B, Sq, Nq, D = q.shape
        Skv, Nkv = k.shape[1], k.shape[2]
    else:
        Sq, Nq, D = q.shape
        Skv, Nkv = k.shape[0], k.shape[1]
        B = len(actual_seq_qlen)
    cq = ck = None
    if input_layout == "TND":
        cq = np.ascontiguousarray(np.asarray(actual_seq_qlen, dtype=np.int64))
        ck = np.ascontiguousarray(np.asarray(actual_seq_kvlen, dtype=np.int64))
    if atten_mask is not None:
        if atten_mask.dtype == torch.bool:
            atten_mask = atten_mask.to(torch.uint8)
        atten_mask = atten_mask.contiguous()
        if mask_shape is None:
            mask_shape = {2: "SS", 4: "BNSS" if atten_mask.shape[1] == Nq and Nq > 1 else "B1SS"}[atten_mask.dim()]
    pse_bcast = 0
    if pse is not None:
        pse = pse.contiguous()
        pse_bcast = int(pse.shape[0] == 1 and B > 1)
    if out is None:
        out = torch.empty_like(q)
    if return_stats:
        sshape = (Nq, Sq) if input_layout == "TND" else (B, Nq, Sq)
        if softmax_max is None:
            softmax_max = torch.empty(sshape, dtype=torch.float32, device=dev)
        if softmax_sum is None:
            softmax_sum = torch.empty(sshape, dtype=torch.float32, device=dev)
    L = lib()
    _ck(L.attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, Nq, Nkv, Sq, Skv, D, head_num, lay, _ptr(atten_mask),
                   MASK_SHAPES[mask_shape], _ptr(pse), pse_bcast, scale, keep_prob, sparse_mode, pre_tokens,
                   next_tokens, None if cq is None else cq.ctypes.data_as(ctypes.c_void_p),
                   None if ck is None else ck.ctypes.data_as(ctypes.c_void_p), _ptr(out), _ptr(softmax_max),
                   _ptr(softmax_sum), _stream(dev)))
    if host:
        return _to_host((out, softmax_max, softmax_sum), dsts, dev)
    return out, softmax_max, softmax_sum


def bsa_fwd(q, k, v, block_mask, scale: float, *, out=None, softmax_max=None, softmax_sum=None,
            return_stats: bool = True, device=None):
    """bf16 block-sparse attention (BNSD): attn_fwd over the 128x128 blocks kept by block_mask."""
    import torch
    host = not q.is_cuda
    dev = torch.device(device or (q.device if q.is_cuda else "cuda:0"))
    q, k, v, block_mask = _on_cuda([q, k, v, block_mask], dev)
    (out, softmax_max, softmax_sum), dsts = _split_outputs(host, (out, softmax_max, softmax_sum))
    B, Nq, Sq, D = q.shape
    Nkv, Skv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if return_stats:
        if softmax_max is None:
            softmax_max = torch.empty((B, Nq, Sq), dtype=torch.float32, device=dev)
        if softmax_sum is None:
            softmax_sum = torch.empty((B, Nq, Sq), dtype=torch.float32, device=dev)
    _ck(lib().bsa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(block_mask), B, Nq, Nkv, Sq, Skv, D, scale, _ptr(out),
                      _ptr(softmax_max), _ptr(softmax_sum), _stream(dev)))
    if host:
        return _to_host((out, softmax_max, softmax_sum), dsts, dev)
    return out, softmax_max, softmax_sum


def _qbsa_fwd_host(q_i8, k_i8, q_scale, k_scale, v_fp8, v_scale, block_mask, scale, dsts, return_stats, dev,
                   n_chunks):
    """qbsa_fwd on host tensors through the library's qbsa_fwd_host (chunked copies that
    overlap the kernel, done natively); returns host tensors (the caller's, or new pinned ones)."""
    import torch
    B, Nq, Sq, D = q_i8.shape
    Nkv, Skv = k_i8.shape[1], k_i8.shape[2]
    hq = [t.contiguous() for t in (q_i8, k_i8, q_scale, k_scale, v_fp8, v_scale, block_mask)]
    h_out = dsts[0] if dsts[0] is not None else torch.empty((B, Nq, Sq, D), dtype=torch.bfloat16, pin_memory=True)
    h_max = h_sum = None
    if return_stats:
        h_max = dsts[1] if dsts[1] is not None else torch.empty((B, Nq, Sq), dtype=torch.float32, pin_memory=True)
        h_sum = dsts[2] if dsts[2] is not None else torch.empty((B, Nq, Sq), dtype=torch.float32, pin_memory=True)
    with torch.cuda.device(dev):
        _ck(lib().qbsa_fwd_host(*[_ptr(t) for t in hq], B, Nq, Nkv, Sq, Skv, D, scale, _ptr(h_out), _ptr(h_max),
                                _ptr(h_sum), n_chunks, _stream(dev)))
    return h_out, h_max, h_sum


def qbsa_fwd(q_i8, k_i8, q_scale, k_scale, v_fp8, v_scale, block_mask, scale: float, *, out=None,
             softmax_max=None, softmax_sum=None, return_stats: bool = True, device=None, host_chunks: int = 8):
    """Quantized block-sparse attention forward (BNSD, D = 128).  Returns (out, max, sum).

    Device tensors run as one launch on the current stream.  Host tensors go through the
    library's qbsa_fwd_host, which copies them in and the results out in about `host_chunks`
    (batch, kv-head) chunks whose transfers overlap the kernel (page-locked tensors overlap
    best); the host results are pinned tensors (or the caller's `out` / stats tensors)."""
    import torch
    host = not q_i8.is_cuda
    dev = torch.device(device or (q_i8.device if q_i8.is_cuda else "cuda:0"))
    if host and all(not t.is_cuda for t in (k_i8, q_scale, k_scale, v_fp8, v_scale, block_mask)):
        _, dsts = _split_outputs(True, (out, softmax_max, softmax_sum))
        return _qbsa_fwd_host(q_i8, k_i8, q_scale, k_scale, v_fp8, v_scale, block_mask, scale, dsts,
                              return_stats, dev, max(1, host_chunks))
    q_i8, k_i8, q_scale, k_scale, v_fp8, v_scale, block_mask = _on_cuda(
        [q_i8, k_i8, q_scale, k_scale, v_fp8, v_scale, block_mask], dev)
    (out, softmax_max, softmax_sum), dsts = _split_outputs(host, (out, softmax_max, softmax_sum))
    B, Nq, Sq, D = q_i8.shape
    Nkv, Skv = k_i8.shape[1], k_i8.shape[2]
    if out is None:
        out = torch.empty((B, Nq, Sq, D), dtype=torch.bfloat16, device=dev)
    if return_stats:
        if softmax_max is None:
            softmax_max = torch.empty((B, Nq, Sq), dtype=torch.float32, device=dev)
        if softmax_sum is None:
            softmax_sum = torch.empty((B, Nq, Sq), dtype=torch.float32, device=dev)
    L = lib()
    _ck(L.qbsa_fwd(_ptr(q_i8), _ptr(k_i8), _ptr(q_scale), _ptr(k_scale), _ptr(v_fp8), _ptr(v_scale),
                   _ptr(block_mask), B, Nq, Nkv, Sq, Skv, D, scale, _ptr(out), _ptr(softmax_max),
                   _ptr(softmax_sum), _stream(dev)))
    if host:
        return _to_host((out, softmax_max, softmax_sum), dsts, dev)
    return out, softmax_max, softmax_sum


def quantize_qk(x):
    """Per-128-block INT8 quantisation of a BNSD bf16 device tensor -> (codes int8, scales fp32)."""
    import torch
    B, N, S, D = x.shape
    codes = torch.empty((B, N, S, D), dtype=torch.int8, device=x.device)
    scales = torch.empty((B, N, -(-S // 128)), dtype=torch.float32, device=x.device)
    _ck(lib().qbsa_quantize_qk(_ptr(x), B, N, S, D, _ptr(codes), _ptr(scales), _stream(x.device)))
    return codes, scales


def quantize_v(v):
    """Per-channel E4M3 quantisation of a BNSD bf16 device tensor -> (codes uint8, scales fp32)."""
    import torch
    B, N, S, D = v.shape
    codes = torch.empty((B, N, S, D), dtype=torch.uint8, device=v.device)
    scales = torch.empty((B, N, D), dtype=torch.float32, device=v.device)
    _ck(lib().qbsa_quantize_v(_ptr(v), B, N, S, D, _ptr(codes), _ptr(scales), _stream(v.device)))
    return codes, scales


def attn_tile_schedule(sq: int, skv: int, sparse_mode: int = 0, pre_tokens: int = INF_TOKENS,
                       next_tokens: int = INF_TOKENS):
    """Host-only: per query tile, (kt_begin, kt_end, full_begin, full_end) arrays."""
    n = -(-sq // 128)
    arrs = [np.zeros(n, dtype=np.int32) for _ in range(4)]
    _ck(lib().attn_tile_schedule(sq, skv, sparse_mode, pre_tokens, next_tokens,
                                 *[a.ctypes.data_as(ctypes.c_void_p) for a in arrs], n))
    return tuple(arrs)


def block_lists(block_mask_rows):
    """Device mask compaction hook: (rows, n_kb) uint8 device tensor -> (lists int32, counts int32)."""
    import torch
    rows, n_kb = block_mask_rows.shape
    lists = torch.empty((rows, n_kb), dtype=torch.int32, device=block_mask_rows.device)
    counts = torch.empty((rows,), dtype=torch.int32, device=block_mask_rows.device)
    _ck(lib().qbsa_block_lists(_ptr(block_mask_rows.contiguous()), rows, n_kb, _ptr(lists), _ptr(counts),
                               _stream(block_mask_rows.device)))
    return lists, counts


def check(device=None):
    """Synchronise the current stream and raise if a kernel reported a device-side timeout."""
    import torch
    _ck(lib().qbsa_check(_stream(torch.device(device or "cuda:0"))))


def block_mean(x):
    """Mean row of every 128-token block of a BNSD bf16 device tensor -> fp32 [B, N, ceil(S/128), D]."""
    import torch
    B, N, S, D = x.shape
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bfloat16 CUDA tensor")
    out = torch.empty((B, N, -(-S // 128), D), dtype=torch.float32, device=x.device)
    _ck(lib().qbsa_block_mean(_ptr(x), B, N, S, D, _ptr(out), _stream(x.device)))
    return out


def block_topk(q_mean, k_mean, scale: float, *, keep: float = None, n_keep: int = None, return_scores: bool = False):
    """Block mask (uint8 [B, Nq, nqb, nkb], 1 = compute) keeping the n_keep best pooled scores per query
    block; with ``keep`` the library derives n_keep from the fraction (qbsa_block_topk_keep)."""
    import torch
    B, Nq, nqb, D = q_mean.shape
    Nkv, nkb = k_mean.shape[1], k_mean.shape[2]
    if (keep is None) == (n_keep is None):
        raise ValueError("give exactly one of keep and n_keep")
    for t in (q_mean, k_mean):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q_mean and k_mean must be contiguous float32 CUDA tensors")
    mask = torch.empty((B, Nq, nqb, nkb), dtype=torch.uint8, device=q_mean.device)
    scores = torch.empty((B, Nq, nqb, nkb), dtype=torch.float32, device=q_mean.device) if return_scores else None
    if keep is not None:
        _ck(lib().qbsa_block_topk_keep(_ptr(q_mean), _ptr(k_mean), B, Nq, Nkv, nqb, nkb, D, scale, float(keep),
                                       _ptr(mask), _ptr(scores), None, _stream(q_mean.device)))
    else:
        _ck(lib().qbsa_block_topk(_ptr(q_mean), _ptr(k_mean), B, Nq, Nkv, nqb, nkb, D, scale, n_keep, _ptr(mask),
                                  _ptr(scores), _stream(q_mean.device)))
    return (mask, scores) if return_scores else mask


def estimate_block_mask(q, k, scale: float, keep: float, *, return_scores: bool = False):
    """Block mask for block-sparse attention from bf16 BNSD Q and K: pool, score, keep the top blocks."""
    return block_topk(block_mean(q), block_mean(k), scale, keep=keep, return_scores=return_scores)

