"""Python binding of libblasst.so (BLASST blocked attention on B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/blasst.h``.  PyTorch supplies
device memory and streams.  There is no CPU fallback: if the shared library
is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "BlasstError", "lib", "prefill", "decode", "decode_noalloc", "calibrate", "calibrate_fit", "calibrate_threshold",
    "visited_pairs", "decode_workspace_bytes", "mask_words", "Opts", "STATUS", "prefill_backward",
    "backward_workspace_bytes", "decode_fp8", "decode_pick_splits",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libblasst.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "workspace too small",
          4: "CUDA error", 5: "device wait timed out"}


class BlasstError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        msg = f"{what}: {STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class Opts(ctypes.Structure):
    """Mirror of ``blasst_opts``."""

    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("dv", ctypes.c_int),
        ("block_n", ctypes.c_int),
        ("num_splits", ctypes.c_int),
        ("mode", ctypes.c_int),
        ("k_row_stride", ctypes.c_longlong),
        ("v_row_stride", ctypes.c_longlong),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("gaps_out", ctypes.c_void_p),
        ("status_word", ctypes.c_void_p),
        ("seed_splits", ctypes.c_int),
    ]

    def __init__(self, **kw):
        super().__init__()
        self.struct_size = ctypes.sizeof(Opts)
        for k, v in kw.items():
            setattr(self, k, v)


_ATTN_ARGS = [ctypes.c_void_p] * 4 + [ctypes.c_void_p] + [ctypes.c_int] * 6 + [ctypes.c_float, ctypes.c_float,
                                                                              ctypes.c_int, ctypes.c_void_p,
                                                                              ctypes.c_void_p, ctypes.c_void_p,
                                                                              ctypes.POINTER(Opts)]

_lib = None


def lib() -> ctypes.CDLL:
    """Load libblasst.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m block_sparse_flashattention_tcgen05_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name in ("blasst_prefill", "blasst_decode", "blasst_calibrate", "blasst_decode_noalloc",
                     "blasst_measure_prefill_novote"):
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = _ATTN_ARGS
        L.blasst_decode_paged.restype = ctypes.c_int
        L.blasst_decode_paged.argtypes = ([ctypes.c_void_p] * 7 + [ctypes.c_int] * 7 +
                                          [ctypes.c_float, ctypes.c_float, ctypes.c_int] + [ctypes.c_void_p] * 3 +
                                          [ctypes.POINTER(Opts)])
        L.blasst_decode_fp8.restype = ctypes.c_int
        L.blasst_decode_fp8.argtypes = ([ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 +
                                        [ctypes.c_float] * 4 + [ctypes.c_int] + [ctypes.c_void_p] * 3 +
                                        [ctypes.POINTER(Opts)])
        L.blasst_prefill_backward.restype = ctypes.c_int
        L.blasst_prefill_backward.argtypes = ([ctypes.c_void_p] * 9 + [ctypes.c_int] * 6 +
                                              [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.POINTER(Opts)])
        L.blasst_backward_workspace_bytes.restype = ctypes.c_size_t
        L.blasst_backward_workspace_bytes.argtypes = [ctypes.c_int] * 3
        L.blasst_calibrate_fit.restype = ctypes.c_int
        L.blasst_calibrate_fit.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                                                                   ctypes.POINTER(ctypes.c_double)]
        L.blasst_calibrate_threshold.restype = ctypes.c_int
        L.blasst_calibrate_threshold.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_double,
                                                 ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
        L.blasst_decode_pick_splits.restype = ctypes.c_int
        L.blasst_decode_pick_splits.argtypes = [ctypes.c_int] * 4
        L.blasst_decode_pick_splits_rows.restype = ctypes.c_int
        L.blasst_decode_pick_splits_rows.argtypes = [ctypes.c_int] * 5
        L.blasst_decode_workspace_bytes.restype = ctypes.c_size_t
        L.blasst_decode_workspace_bytes.argtypes = [ctypes.c_int] * 5
        L.blasst_visited_pairs.restype = ctypes.c_longlong
        L.blasst_visited_pairs.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(Opts)]
        L.blasst_status_string.restype = ctypes.c_char_p
        L.blasst_status_string.argtypes = [ctypes.c_int]
        L.blasst_last_error.restype = ctypes.c_char_p
        L.blasst_last_error.argtypes = []
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        detail = lib().blasst_last_error().decode() if rc in (3, 4) else ""
        raise BlasstError(rc, what, detail)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def mask_words(n_blocks: int) -> int:
    return (n_blocks + 31) // 32


def _dev_tensor(t, name):
    import torch

    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library takes device pointers)")
    return t


def _attn(fn_name, q, k, v, *, scale, lam, causal, o, lse, want_mask, want_count, opts, stream, mask_rows,
          n_blocks, B, Hq, Hkv, Lq, Lk, d, dv):
    import torch

    dev = q.device
    if want_mask is True:
        want_mask = torch.empty((mask_rows, mask_words(n_blocks)), dtype=torch.int32, device=dev)
    if want_count is True:
        want_count = torch.empty(1, dtype=torch.int64, device=dev)
    mask = want_mask if isinstance(want_mask, torch.Tensor) else None
    count = want_count if isinstance(want_count, torch.Tensor) else None
    rc = getattr(lib(), fn_name)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq, Lk, d, float(scale), float(lam),
        int(bool(causal)), _ptr(mask), _ptr(count), _stream(stream), ctypes.byref(opts))
    _check(rc, fn_name)
    return mask, count


def prefill(q, k, v, *, scale, lam=0.0, causal=True, o=None, lse=None, skip_mask=True, skip_count=True,
            status_word=None, stream=None, _entry="blasst_prefill"):
    """Prefill attention with block skipping.  q [B,Hq,Lq,128], k/v [B,Hkv,Lk,128] bf16 on CUDA.

    Returns (o, lse, skip_mask [B*Hq*ceil(Lq/128), W] int32 or None, skip_count [1] int64 or None).
    """
    import torch

    _dev_tensor(q, "q"), _dev_tensor(k, "k"), _dev_tensor(v, "v")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    if o is None:
        o = torch.empty((B, Hq, Lq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    opts = Opts(status_word=None if status_word is None else status_word.data_ptr())
    nq = (Lq + 127) // 128
    nb = (Lk + 127) // 128
    m, c = _attn(_entry, q, k, v, scale=scale, lam=lam, causal=causal, o=o, lse=lse,
                 want_mask=skip_mask, want_count=skip_count, opts=opts, stream=stream, mask_rows=B * Hq * nq,
                 n_blocks=nb, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d, dv=d)
    return o, lse, m, c


def measure_prefill_novote(q, k, v, **kw):
    """blasst_measure_prefill_novote (include/blasst_measure.h): prefill() with
    the skip decision compiled out, every visited block kept.  Measurement only:
    timed against prefill() at lam = 0 it gives the decision's cost."""
    return prefill(q, k, v, _entry="blasst_measure_prefill_novote", **kw)


def prefill_backward(q, k, v, o, lse, dout, *, scale, causal=True, skip_mask=None, dq=None, dk=None, dv=None,
                     workspace=None, status_word=None, stream=None):
    """Gradients (dq, dk, dv) of prefill attention with the forward's skip mask held fixed.

    q, k, v, o, lse: the forward's tensors; dout [B,Hq,Lq,128] bf16, the gradient of o;
    skip_mask: the forward's mask (int32 [B*Hq*ceil(Lq/128), W]) or None (nothing skipped).
    Returns bf16 dq [B,Hq,Lq,128], dk, dv [B,Hkv,Lk,128].
    """
    import torch

    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (dout, "dout")):
        _dev_tensor(t, n)
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    if dq is None:
        dq = torch.empty_like(q)
    if dk is None:
        dk = torch.empty_like(k)
    if dv is None:
        dv = torch.empty_like(v)
    opts = Opts(status_word=None if status_word is None else status_word.data_ptr())
    if workspace is not None:
        opts.workspace = workspace.data_ptr()
        opts.workspace_bytes = workspace.numel() * workspace.element_size()
    rc = lib().blasst_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                       _ptr(dv), B, Hq, Hkv, Lq, Lk, d, float(scale), int(bool(causal)),
                                       _ptr(skip_mask), _stream(stream), ctypes.byref(opts))
    _check(rc, "blasst_prefill_backward")
    return dq, dk, dv


def decode_pick_splits(B, Hkv, Lk, num_sms=None, rows=1) -> int:
    """The split count num_splits=-1 selects for tiles of ``rows`` = G * Lq query rows
    (num_sms: this device's SM count by default)."""
    if num_sms is None:
        import torch

        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return int(lib().blasst_decode_pick_splits_rows(B, Hkv, rows, Lk, num_sms))


def backward_workspace_bytes(B, Hq, Lq) -> int:
    return int(lib().blasst_backward_workspace_bytes(B, Hq, Lq))


def decode(q, k, v, *, scale, lam=0.0, causal=False, num_splits=None, dv=None, o=None, lse=None,
           skip_mask=True, skip_count=True, workspace=None, status_word=None, stream=None, seed_splits=False):
    """Split-KV decode with block skipping.

    GQA/MQA: q [B,Hq,Lq,128], k/v [B,Hkv,Lk,128] bf16 on CUDA (16 splits by default);
    (Hq/Hkv)*Lq <= 128 query rows per KV head.
    MLA: q [B,Hq,Lq,576], k [B,1,Lk,576], v = the same tensor as k, dv = 512 (V is
    the first 512 columns of each cache row; 2 splits by default).
    Returns (o, lse, skip_mask [B*Hkv, W] int32 or None, skip_count [1] int64 or None).
    ``workspace``: optional uint8 CUDA tensor of at least decode_workspace_bytes() bytes.
    ``seed_splits`` (d = 128): splits after the first start their running max at
    block 0's row maxima and have no forced first block.
    """
    import torch

    _dev_tensor(q, "q"), _dev_tensor(k, "k"), _dev_tensor(v, "v")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, krs = k.shape
    vrs = v.shape[-1]
    dv = vrs if dv is None else dv
    if o is None:
        o = torch.empty((B, Hq, Lq, dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    opts = Opts(num_splits=num_splits or 0, dv=dv, k_row_stride=krs, v_row_stride=vrs,
                status_word=None if status_word is None else status_word.data_ptr(),
                seed_splits=int(bool(seed_splits)))
    if workspace is not None:
        opts.workspace = workspace.data_ptr()
        opts.workspace_bytes = workspace.numel() * workspace.element_size()
    nb = (Lk + 63) // 64
    m, c = _attn("blasst_decode", q, k, v, scale=scale, lam=lam, causal=causal, o=o, lse=lse,
                 want_mask=skip_mask, want_count=skip_count, opts=opts, stream=stream, mask_rows=B * Hkv,
                 n_blocks=nb, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d, dv=dv)
    return o, lse, m, c


def decode_fp8(q, k8, v8, *, scale, k_scale, v_scale, lam=0.0, causal=False, num_splits=None, o=None, lse=None,
               skip_mask=True, skip_count=True, workspace=None, status_word=None, stream=None, seed_splits=False):
    """Split-KV decode over an FP8 (e4m3) cache: K = k_scale * k8, V = v_scale * v8.

    q [B,Hq,Lq,128] bf16; k8, v8 [B,Hkv,Lk,128] uint8 (or float8_e4m3fn) on CUDA; (Hq/Hkv)*Lq <= 16.
    Returns (o, lse, skip_mask [B*Hkv, W] int32 or None, skip_count [1] int64 or None).
    """
    import torch

    _dev_tensor(q, "q"), _dev_tensor(k8, "k8"), _dev_tensor(v8, "v8")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k8.shape
    if o is None:
        o = torch.empty((B, Hq, Lq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    opts = Opts(num_splits=num_splits or 0, status_word=None if status_word is None else status_word.data_ptr(),
                seed_splits=int(bool(seed_splits)))
    if workspace is not None:
        opts.workspace = workspace.data_ptr()
        opts.workspace_bytes = workspace.numel() * workspace.element_size()
    nb = (Lk + 63) // 64
    mask = torch.empty((B * Hkv, mask_words(nb)), dtype=torch.int32, device=q.device) if skip_mask is True else (
        skip_mask if isinstance(skip_mask, torch.Tensor) else None)
    count = torch.empty(1, dtype=torch.int64, device=q.device) if skip_count is True else (
        skip_count if isinstance(skip_count, torch.Tensor) else None)
    rc = lib().blasst_decode_fp8(_ptr(q), _ptr(k8), _ptr(v8), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq, Lk, d,
                                 float(scale), float(k_scale), float(v_scale), float(lam), int(bool(causal)),
                                 _ptr(mask), _ptr(count), _stream(stream), ctypes.byref(opts))
    _check(rc, "blasst_decode_fp8")
    return o, lse, mask, count


def decode_noalloc(q, k, v, *, scale, lam=0.0, causal=False, num_splits=None, dv=None, o=None, lse=None,
                   skip_mask=True, skip_count=True, status_word=None, stream=None):
    """Same as decode(), through blasst_decode_noalloc: the library allocates
    nothing (split partials in its fixed device array).  Output tensors that
    are not passed are created here, by the caller side of the interface."""
    import torch

    _dev_tensor(q, "q"), _dev_tensor(k, "k"), _dev_tensor(v, "v")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, krs = k.shape
    vrs = v.shape[-1]
    dv = vrs if dv is None else dv
    if o is None:
        o = torch.empty((B, Hq, Lq, dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    opts = Opts(num_splits=num_splits or 0, dv=dv, k_row_stride=krs, v_row_stride=vrs,
                status_word=None if status_word is None else status_word.data_ptr())
    nb = (Lk + 63) // 64
    m, c = _attn("blasst_decode_noalloc", q, k, v, scale=scale, lam=lam, causal=causal, o=o, lse=lse,
                 want_mask=skip_mask, want_count=skip_count, opts=opts, stream=stream, mask_rows=B * Hkv,
                 n_blocks=nb, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d, dv=dv)
    return o, lse, m, c


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, *, scale, lam=0.0, causal=False, num_splits=None,
                 o=None, lse=None, skip_mask=True, skip_count=True, workspace=None, status_word=None, stream=None,
                 seed_splits=False):
    """Decode over a paged, ragged KV cache.

    q [B,Hq,Lq,128]; k_pages/v_pages [num_pages, Hkv, 64, 128] bf16; block_table int32
    [B, max_pages] (page of each 64-key block of each sequence); seq_lens int32 [B].
    All CUDA tensors.  Returns (o, lse, skip_mask [B*Hkv, ceil(max_pages/32)] int32 or
    None, skip_count [1] int64 or None).
    """
    import torch

    for t, n in ((q, "q"), (k_pages, "k_pages"), (v_pages, "v_pages"), (block_table, "block_table"),
                 (seq_lens, "seq_lens")):
        _dev_tensor(t, n)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    B, Hq, Lq, d = q.shape
    num_pages, Hkv, page, dk = k_pages.shape
    if page != 64 or dk != d or tuple(v_pages.shape) != tuple(k_pages.shape):
        raise ValueError("pages must be [num_pages, Hkv, 64, d] for both k and v")
    if block_table.dim() != 2 or block_table.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_table [B, max_pages] and seq_lens [B] expected")
    max_pages = block_table.shape[1]
    if o is None:
        o = torch.empty((B, Hq, Lq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    opts = Opts(num_splits=num_splits or 0, status_word=None if status_word is None else status_word.data_ptr(),
                seed_splits=int(bool(seed_splits)))
    if workspace is not None:
        opts.workspace = workspace.data_ptr()
        opts.workspace_bytes = workspace.numel() * workspace.element_size()
    dev = q.device
    if skip_mask is True:
        skip_mask = torch.empty((B * Hkv, mask_words(max_pages)), dtype=torch.int32, device=dev)
    if skip_count is True:
        skip_count = torch.empty(1, dtype=torch.int64, device=dev)
    mask = skip_mask if isinstance(skip_mask, torch.Tensor) else None
    count = skip_count if isinstance(skip_count, torch.Tensor) else None
    rc = lib().blasst_decode_paged(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(o), _ptr(lse), _ptr(block_table), _ptr(seq_lens),
        B, Hq, Hkv, Lq, max_pages, num_pages, d, float(scale), float(lam), int(bool(causal)),
        _ptr(mask), _ptr(count), _stream(stream), ctypes.byref(opts))
    _check(rc, "blasst_decode_paged")
    return o, lse, mask, count


NOALLOC_SCRATCH_BYTES = 16 << 20


def calibrate(q, k, *, scale, lam=0.0, causal=True, mode="prefill", num_splits=None, dv=None, skip_mask=True,
              skip_count=True, stream=None, seed_splits=False):
    """Decision-only pass.  Returns (gaps [tiles, nb] fp32, skip_mask, skip_count)."""
    import torch

    _dev_tensor(q, "q"), _dev_tensor(k, "k")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    if mode == "prefill":
        nb = (Lk + 127) // 128
        tiles = B * Hq * ((Lq + 127) // 128)
        m = 0
    elif mode == "decode":
        nb = (Lk + 63) // 64
        tiles = B * Hkv
        m = 1
    else:
        raise ValueError(mode)
    gaps = torch.empty((tiles, nb), dtype=torch.float32, device=q.device)
    opts = Opts(mode=m, num_splits=num_splits or 0, gaps_out=gaps.data_ptr(), dv=dv or 0,
                seed_splits=int(bool(seed_splits)))
    mk, c = _attn("blasst_calibrate", q, k, None, scale=scale, lam=lam, causal=causal, o=None, lse=None,
                  want_mask=skip_mask, want_count=skip_count, opts=opts, stream=stream, mask_rows=tiles,
                  n_blocks=nb, B=B, Hq=Hq, Hkv=Hkv, Lq=Lq, Lk=Lk, d=d, dv=d)
    return gaps, mk, c


def calibrate_fit(L, lam, sparsity):
    """Host least squares of ln(lambda*L) = ln(alpha) + beta*s.  Returns (alpha, beta)."""
    import numpy as np

    L = np.ascontiguousarray(L, dtype=np.float64)
    lam = np.ascontiguousarray(lam, dtype=np.float64)
    s = np.ascontiguousarray(sparsity, dtype=np.float64)
    a = ctypes.c_double()
    b = ctypes.c_double()
    _check(lib().blasst_calibrate_fit(L.ctypes.data, lam.ctypes.data, s.ctypes.data, len(s), ctypes.byref(a),
                                      ctypes.byref(b)), "blasst_calibrate_fit")
    return a.value, b.value


def calibrate_threshold(gaps_host, target):
    """lambda for a target sparsity from host gaps (numpy float32).  Returns (lambda, achieved)."""
    import numpy as np

    g = np.ascontiguousarray(gaps_host, dtype=np.float32).ravel()
    lam = ctypes.c_double()
    ach = ctypes.c_double()
    _check(lib().blasst_calibrate_threshold(g.ctypes.data, g.size, float(target), ctypes.byref(lam),
                                            ctypes.byref(ach)), "blasst_calibrate_threshold")
    return lam.value, ach.value


def visited_pairs(B, Hq, Hkv, Lq, Lk, causal, is_decode) -> int:
    opts = Opts()
    return int(lib().blasst_visited_pairs(B, Hq, Hkv, Lq, Lk, int(bool(causal)), int(bool(is_decode)),
                                          ctypes.byref(opts)))


def decode_workspace_bytes(B, Hq, Lq, dv=128, num_splits=16) -> int:
    return int(lib().blasst_decode_workspace_bytes(B, Hq, Lq, dv, num_splits))
