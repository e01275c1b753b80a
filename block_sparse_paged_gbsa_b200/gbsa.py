"""Python binding of libgbsa (argument marshalling only).

Every step of the computation runs in the CUDA kernels behind the C ABI
declared in ``include/gbsa.h``; this module checks tensor shapes, strides and
devices, fills the C structs and calls the library on the current CUDA
stream.  There is no fallback: if ``libgbsa.so`` is missing or no CUDA device
is present the calls raise.

Function and argument names follow the PyTorch interface of the
GenericBlockSparseAttention article (cf-1.com/news/4865651), "Calling /
PyTorch API": ``generic_block_sparse_attention_metadata(sparse_block_idx,
sparse_block_count, num_heads_q, num_heads_kv, head_dim, block_shape, *,
cu_seqlens_q, seqused_q, seqused_kv, ...)`` and
``generic_block_sparse_attention(q, k, v, sparse_block_idx,
sparse_block_count, block_shape, *, metadata, cu_seqlens_q, seqused_q,
seqused_kv, block_table, softmax_scale, mask_mode, win_left, win_right,
return_softmax_lse, ...) -> (attention_out, softmax_lse)``.  The quantisation,
attention-mask and raw-KV arguments of that interface are not offered: the
article marks those modes unsupported.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libgbsa.so"
_lock = threading.Lock()
_lib = None

STATUS_NAMES = {0: "GBSA_OK", 1: "GBSA_ERR_INVALID_ARG", 2: "GBSA_ERR_UNSUPPORTED",
                3: "GBSA_ERR_SHAPE", 4: "GBSA_ERR_ALIGNMENT", 5: "GBSA_ERR_WORKSPACE_TOO_SMALL",
                6: "GBSA_ERR_METADATA_TOO_SMALL", 7: "GBSA_ERR_CUDA", 8: "GBSA_ERR_NO_DEVICE"}

DEV_BITS = {0x01: "BAD_SEQLEN", 0x02: "BAD_BLOCK_IDX", 0x04: "BAD_COUNT", 0x08: "BAD_PAGE",
            0x10: "META_MISMATCH", 0x20: "TIMEOUT", 0x40: "CAPACITY"}


class GbsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class _Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("N1", ctypes.c_int32),
                ("N2", ctypes.c_int32), ("D", ctypes.c_int32), ("block_x", ctypes.c_int32),
                ("block_y", ctypes.c_int32), ("total_q_blocks", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("kv_page_stride", ctypes.c_int64),
                ("scale", ctypes.c_double), ("mask_mode", ctypes.c_int32),
                ("win_left", ctypes.c_int32), ("win_right", ctypes.c_int32),
                ("is_packed_gqa", ctypes.c_int32), ("return_lse", ctypes.c_int32),
                ("has_seqused_q", ctypes.c_int32), ("num_ctas", ctypes.c_int32),
                ("max_blocks_per_split", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("softmax_precision", ctypes.c_int32), ("kv_layout", ctypes.c_int32),
                ("T_kv", ctypes.c_int32), ("q_scale", ctypes.c_double),
                ("k_scale", ctypes.c_double), ("v_scale", ctypes.c_double),
                ("wait_limit_ns", ctypes.c_int64)]


class _Tensors(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q", "k", "v", "sparse_idx", "sparse_count", "cu_seqlens_q", "seqused_q",
                 "seqused_kv", "block_table", "out", "lse", "cu_seqlens_kv")]


@dataclasses.dataclass
class Problem:
    """Host-known description of one call (mirrors ``gbsa_problem``)."""
    B: int
    T: int
    N1: int
    N2: int
    D: int
    block_x: int
    total_q_blocks: int
    top_k: int
    max_pages_per_seq: int = 1
    num_pages: int = 1
    kv_page_stride: int = 0
    scale: float = 0.0
    mask_mode: int = 1
    win_left: int = -1
    win_right: int = -1
    is_packed_gqa: int = 1
    return_lse: int = 0
    has_seqused_q: int = 0
    num_ctas: int = 0
    max_blocks_per_split: int = 0
    block_y: int = 128
    dtype: int = 0              # 0 = bf16, 1 = fp16, 2 = E4M3 (q, k, v; out bf16 for E4M3)
    softmax_precision: int = 0  # 0: fp32 softmax; 1: f16 exponentials, fp32 rescale and sums
    kv_layout: int = 0          # 0 = paged pool + block_table, 1 = TND + cu_seqlens_kv
    T_kv: int = 0               # TND: rows of k and v
    q_scale: float = 1.0        # E4M3: per-tensor dequantization scales
    k_scale: float = 1.0
    v_scale: float = 1.0
    wait_limit_ns: int = 0      # bound of a pipeline wait of the forward kernel; 0 = 1 s

    def as_c(self) -> _Problem:
        p = _Problem()
        for f, _ in _Problem._fields_:
            setattr(p, f, getattr(self, f))
        return p


ABI_VERSION = 6
# GBSA_METADATA_FUSED_MAX_B: up to this many sequences the metadata call is
# two kernel launches, above it three.
METADATA_FUSED_MAX_B = 1024
DTYPE_BF16, DTYPE_FP16, DTYPE_FP8_E4M3 = 0, 1, 2


def _dtype_code(t) -> int:
    import torch
    codes = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_FP16,
             torch.float8_e4m3fn: DTYPE_FP8_E4M3}
    if t.dtype not in codes:
        raise ValueError(f"expected bf16, fp16 or float8_e4m3fn, got {t.dtype}")
    return codes[t.dtype]


def _out_dtype(t):
    """Element type of out: q's type, except bf16 for E4M3 inputs."""
    import torch
    return torch.bfloat16 if t.dtype == torch.float8_e4m3fn else t.dtype


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m block_sparse_paged_gbsa_b200.build`")
        lib = ctypes.CDLL(path)
        P, Tn, vp, sz = ctypes.POINTER(_Problem), ctypes.POINTER(_Tensors), ctypes.c_void_p, ctypes.c_size_t
        lib.gbsa_abi_version.restype = ctypes.c_int32
        lib.gbsa_status_string.argtypes = [ctypes.c_int]
        lib.gbsa_status_string.restype = ctypes.c_char_p
        lib.gbsa_metadata_size.argtypes = [P, ctypes.POINTER(sz)]
        lib.gbsa_metadata_size.restype = ctypes.c_int
        lib.gbsa_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        lib.gbsa_workspace_size.restype = ctypes.c_int
        lib.gbsa_metadata.argtypes = [P, Tn, vp, sz, vp, vp]
        lib.gbsa_metadata.restype = ctypes.c_int
        lib.gbsa_forward.argtypes = [P, Tn, vp, vp, sz, vp, vp]
        lib.gbsa_forward.restype = ctypes.c_int
        lib.gbsa_backward_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        lib.gbsa_backward_workspace_size.restype = ctypes.c_int
        lib.gbsa_backward.argtypes = [P, Tn, vp, vp, vp, vp, vp, vp, sz, vp, vp]
        lib.gbsa_backward.restype = ctypes.c_int
        if lib.gbsa_abi_version() != ABI_VERSION:
            raise RuntimeError("libgbsa ABI version mismatch")
        _lib = lib
        return lib


def lib():
    """The loaded ctypes library (raises if missing)."""
    return _load()


def _check(status: int, what: str):
    if status != 0:
        raise GbsaError(status, what)


def metadata_size(problem: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(_load().gbsa_metadata_size(ctypes.byref(problem.as_c()), ctypes.byref(n)),
           "gbsa_metadata_size")
    return int(n.value)


def workspace_size(problem: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(_load().gbsa_workspace_size(ctypes.byref(problem.as_c()), ctypes.byref(n)),
           "gbsa_workspace_size")
    return int(n.value)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, name, dtype, ndim, device=None):
    import torch
    if t is None:
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != ndim:
        raise ValueError(f"{name}: expected a {ndim}-d {dtype} tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous (no silent copies)")
    return t


def _block_shape(block_shape: Sequence[int]):
    bx, by = (int(x) for x in block_shape)
    return bx, by


QUANT_NONE, QUANT_FP8_E4M3_STATIC_CAST_P = 0, 5  # the article's quant_mode values


def _check_layouts(layout_q, layout_kv, quant_mode):
    """The article's layout and quantisation arguments: TND queries, PA_BBND
    or TND keys/values, quant_mode 0 or 5 (anything else is unsupported)."""
    if layout_q != "TND":
        raise ValueError(f"layout_q: only 'TND' is supported, got {layout_q!r}")
    if layout_kv is not None and layout_kv not in ("PA_BBND", "TND"):
        raise ValueError(f"layout_kv: 'PA_BBND' or 'TND', got {layout_kv!r}")
    if quant_mode is not None and int(quant_mode) not in (QUANT_NONE, QUANT_FP8_E4M3_STATIC_CAST_P):
        raise ValueError(f"quant_mode: 0 or 5 are supported, got {quant_mode!r}")


def metadata(sparse_block_idx, sparse_block_count, num_heads_q: int, num_heads_kv: int,
             head_dim: int, block_shape: Sequence[int], *, cu_seqlens_q, seqused_kv,
             seqused_q=None, num_tokens: int = 0, is_packed_gqa: bool = True, mask_mode: int = 1,
             win_left: int = -1, win_right: int = -1, num_ctas: int = 0,
             max_blocks_per_split: int = 0, dev_status=None, out=None,
             softmax_precision: int = 0, cu_seqlens_kv=None, max_seqlen_q: int = -1,
             max_seqlen_kv: int = -1, layout_q: str = "TND", layout_kv: str = "PA_BBND",
             quant_mode: int = 0):
    """Builds the work list (int32 tensor) on the device of the inputs.

    The article's remaining metadata arguments are accepted: layout_q
    ('TND'), layout_kv ('PA_BBND' or 'TND') and quant_mode (0 or 5) are
    checked; cu_seqlens_kv and max_seqlen_q / max_seqlen_kv do not enter the
    work list (it depends on seqused_kv and the Q lengths only).

    softmax_precision: the article's softmaxPrecision; accepted here so that
    its calls run unchanged (the work list does not depend on it).

    num_tokens: T if known (enables the device check cu_seqlens_q[B] == T); 0 skips it.
    out: optional preallocated int32 buffer of at least metadata_size() bytes.
    """
    import torch
    _check_layouts(layout_q, layout_kv, quant_mode)
    idx = _need(sparse_block_idx, "sparse_block_idx", torch.int32, 3)
    dev = idx.device
    cnt = _need(sparse_block_count, "sparse_block_count", torch.int32, 2, dev)
    cu = _need(cu_seqlens_q, "cu_seqlens_q", torch.int64, 1, dev)
    sku = _need(seqused_kv, "seqused_kv", torch.int32, 1, dev)
    squ = None if seqused_q is None else _need(seqused_q, "seqused_q", torch.int32, 1, dev)
    bx, by = _block_shape(block_shape)
    N2, tqb, top_k = idx.shape
    if num_heads_kv != N2 or tuple(cnt.shape) != (N2, tqb):
        raise ValueError("sparse_block_idx / sparse_block_count shapes disagree with num_heads_kv")
    prob = Problem(B=cu.shape[0] - 1, T=int(num_tokens), N1=num_heads_q, N2=num_heads_kv,
                   D=head_dim, block_x=bx, block_y=by, total_q_blocks=tqb, top_k=top_k,
                   mask_mode=mask_mode, win_left=win_left, win_right=win_right,
                   is_packed_gqa=int(bool(is_packed_gqa)), has_seqused_q=int(squ is not None),
                   num_ctas=num_ctas, max_blocks_per_split=max_blocks_per_split,
                   softmax_precision=int(softmax_precision))
    nbytes = metadata_size(prob)
    with torch.cuda.device(dev):
        if out is None:
            meta = torch.empty((nbytes // 4,), dtype=torch.int32, device=dev)
        else:
            meta = _need(out, "out", torch.int32, 1, dev)
            if meta.numel() * 4 < nbytes:
                raise ValueError(f"out: needs {nbytes} bytes")
            nbytes = meta.numel() * 4
        if dev_status is not None:
            dev_status = _need(dev_status, "dev_status", torch.int32, 1, dev)
        ten = _Tensors(sparse_idx=_ptr(idx), sparse_count=_ptr(cnt), cu_seqlens_q=_ptr(cu),
                       seqused_q=_ptr(squ), seqused_kv=_ptr(sku))
        _check(_load().gbsa_metadata(ctypes.byref(prob.as_c()), ctypes.byref(ten),
                                     meta.data_ptr(), nbytes, _ptr(dev_status), _stream_handle()),
               "gbsa_metadata")
    return meta


def make_problem(q, k, sparse_block_idx, block_shape, block_table, cu_seqlens_q, *,
                 softmax_scale=0.0, mask_mode=1, win_left=-1, win_right=-1, is_packed_gqa=True,
                 return_softmax_lse=False, has_seqused_q=False, num_ctas=0,
                 max_blocks_per_split=0, dequant_scales=(1.0, 1.0, 1.0),
                 softmax_precision=0, wait_limit_ns=0) -> Problem:
    """The gbsa_problem a forward call with these tensors describes.  A 4-d k
    is the page pool (block_table given); a 3-d k is TND [T_kv, N2, D]."""
    T, N1, D = q.shape
    N2i, tqb, top_k = sparse_block_idx.shape
    bx, by = _block_shape(block_shape)
    if k.dim() == 3:
        T_kv, N2, Dk = k.shape
        paged = dict(kv_layout=1, T_kv=T_kv, max_pages_per_seq=0, num_pages=0, kv_page_stride=0)
    else:
        num_pages, page, N2, Dk = k.shape
        paged = dict(kv_layout=0, T_kv=0, max_pages_per_seq=block_table.shape[1],
                     num_pages=num_pages, kv_page_stride=k.stride(0))
    return Problem(B=cu_seqlens_q.shape[0] - 1, T=T, N1=N1, N2=N2, D=D, block_x=bx, block_y=by,
                   total_q_blocks=tqb, top_k=top_k, **paged, scale=float(softmax_scale),
                   mask_mode=mask_mode, win_left=win_left, win_right=win_right,
                   is_packed_gqa=int(bool(is_packed_gqa)), return_lse=int(bool(return_softmax_lse)),
                   has_seqused_q=int(bool(has_seqused_q)), num_ctas=num_ctas,
                   max_blocks_per_split=max_blocks_per_split, dtype=_dtype_code(q),
                   q_scale=float(dequant_scales[0]), k_scale=float(dequant_scales[1]),
                   v_scale=float(dequant_scales[2]), softmax_precision=int(softmax_precision),
                   wait_limit_ns=int(wait_limit_ns))


def forward(q, k, v, sparse_block_idx, sparse_block_count, block_shape: Sequence[int], *,
            metadata, cu_seqlens_q, seqused_kv, block_table=None, seqused_q=None,
            cu_seqlens_kv=None,
            softmax_scale: float = 0.0, mask_mode: int = 1, win_left: int = -1,
            win_right: int = -1, is_packed_gqa: bool = True, return_softmax_lse: bool = False,
            num_ctas: int = 0, max_blocks_per_split: int = 0, out=None, lse=None, workspace=None,
            dev_status=None, q_dequant_scale=None, k_dequant_scale=None, v_dequant_scale=None,
            softmax_precision: int = 0, attn_mask=None, p_quant_scale=None,
            layout_q: str = "TND", layout_kv=None, quant_mode=None, dst_type_max: float = 0.0,
            attention_out_dtype=None, wait_limit_ns: int = 0):
    """Block-sparse paged GQA attention.  q, k and v share one element type,
    bf16, fp16 or float8_e4m3fn.  K/V come as the page pool [num_pages, 128,
    N2, D] with ``block_table`` (PA_BBND), or, when ``cu_seqlens_kv`` is given,
    as TND [T_kv, N2, D] with sequence b in rows cu_seqlens_kv[b]..
    cu_seqlens_kv[b+1] (no block table).  E4M3 inputs (the quantised mode
    with static per-tensor scales) take ``q/k/v_dequant_scale`` as positive
    host floats (default 1.0; ignored for the 16-bit types) and give a bf16
    out.  Returns (out [T,N1,D] in q's type -- bf16 for E4M3 --, lse [T,N1,1]
    fp32, an empty tensor unless return_softmax_lse).  softmax_precision is the
    article's softmaxPrecision: 0 (the default here) is the fp32 online
    softmax; 1 forms the exponentials in half precision (an f16 exponent, one
    f16x2 exponential per pair of weights) with the running max, the O
    rescale and the row sums in fp32.  The article's PyTorch API defaults to
    1; this binding defaults to 0, the more accurate mode and the only one
    the article allows for bf16 on the hardware it names.

    The article's remaining arguments: attn_mask must be None (only the
    built-in causal mask, mask_mode 1, exists); layout_q is 'TND'; layout_kv,
    when given, must agree with the tensors ('TND' with cu_seqlens_kv,
    'PA_BBND' with block_table); quant_mode, when given, must agree with q's
    type (0: bf16 / fp16, 5: float8_e4m3fn); p_quant_scale must be None (the
    weights are cast with the fixed factor 2^8); attention_out_dtype, when
    given, must be the type of out (q's, bf16 for E4M3); dst_type_max is not
    used.

    wait_limit_ns bounds every pipeline wait of the forward kernel (0: 1 s);
    a wait that runs out sets the TIMEOUT device-status bit and the results
    are not valid."""
    import torch
    if q is None or q.dtype not in (torch.bfloat16, torch.float16, torch.float8_e4m3fn):
        raise ValueError("q: expected a bf16, fp16 or float8_e4m3fn tensor")
    _check_layouts(layout_q, layout_kv, quant_mode)
    if attn_mask is not None:
        raise ValueError("attn_mask: only the built-in causal mask (mask_mode 1) is supported")
    if p_quant_scale is not None:
        raise ValueError("p_quant_scale: the weights are cast with a fixed factor 2^8; pass None")
    fp8_in = q.dtype == torch.float8_e4m3fn
    if quant_mode is not None and (int(quant_mode) == QUANT_FP8_E4M3_STATIC_CAST_P) != fp8_in:
        raise ValueError("quant_mode: 5 goes with float8_e4m3fn inputs, 0 with bf16 / fp16")
    if attention_out_dtype is not None and attention_out_dtype != _out_dtype(q):
        raise ValueError(f"attention_out_dtype: this input type gives {_out_dtype(q)}")
    if layout_kv is not None and (layout_kv == "TND") != (cu_seqlens_kv is not None):
        raise ValueError("layout_kv: 'TND' goes with cu_seqlens_kv, 'PA_BBND' with block_table")
    q = _need(q, "q", q.dtype, 3)
    scales = tuple(1.0 if s is None else float(s)
                   for s in (q_dequant_scale, k_dequant_scale, v_dequant_scale))
    dev = q.device
    tnd = cu_seqlens_kv is not None
    if tnd:
        if k is None or v is None or k.dim() != 3 or v.dim() != 3:
            raise ValueError("k, v: expected [T_kv, N2, D] tensors (cu_seqlens_kv given)")
    elif k is None or v is None or k.dim() != 4 or v.dim() != 4:
        raise ValueError("k, v: expected [num_pages, 128, N2, D] tensors")
    for name, t in (("k", k), ("v", v)):
        if t.dtype != q.dtype or t.device != dev:
            raise ValueError(f"{name}: expected {q.dtype} (the type of q) on {dev}")
        if tnd:
            if not t.is_contiguous():
                raise ValueError(f"{name}: TND k / v must be contiguous")
            continue
        _, page, n2, d = t.shape
        if t.stride()[1:] != (n2 * d, d, 1):
            raise ValueError(f"{name}: only dim0 (the page axis) may be strided")
    if k.shape != v.shape or k.stride() != v.stride():
        raise ValueError("k and v must have the same shape and strides")
    idx = _need(sparse_block_idx, "sparse_block_idx", torch.int32, 3, dev)
    cnt = _need(sparse_block_count, "sparse_block_count", torch.int32, 2, dev)
    cu = _need(cu_seqlens_q, "cu_seqlens_q", torch.int64, 1, dev)
    sku = _need(seqused_kv, "seqused_kv", torch.int32, 1, dev)
    bt = None if tnd else _need(block_table, "block_table", torch.int32, 2, dev)
    cukv = _need(cu_seqlens_kv, "cu_seqlens_kv", torch.int64, 1, dev) if tnd else None
    squ = None if seqused_q is None else _need(seqused_q, "seqused_q", torch.int32, 1, dev)
    meta = _need(metadata, "metadata", torch.int32, 1, dev)
    prob = make_problem(q, k, idx, block_shape, bt, cu, softmax_scale=softmax_scale,
                        mask_mode=mask_mode, win_left=win_left, win_right=win_right,
                        is_packed_gqa=is_packed_gqa, return_softmax_lse=return_softmax_lse,
                        has_seqused_q=squ is not None, num_ctas=num_ctas,
                        max_blocks_per_split=max_blocks_per_split, dequant_scales=scales,
                        softmax_precision=softmax_precision, wait_limit_ns=wait_limit_ns)
    T, N1, D = q.shape
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty(q.shape, dtype=_out_dtype(q), device=dev)
        else:
            out = _need(out, "out", _out_dtype(q), 3, dev)
            if out.shape != q.shape:
                raise ValueError(f"out: expected shape {tuple(q.shape)}")
        if return_softmax_lse:
            if lse is None:
                lse = torch.empty((T, N1, 1), dtype=torch.float32, device=dev)
            else:
                lse = _need(lse, "lse", torch.float32, 3, dev)
                if tuple(lse.shape) != (T, N1, 1):
                    raise ValueError(f"lse: expected shape {(T, N1, 1)}")
        else:
            lse = torch.empty((0,), dtype=torch.float32, device=dev)
        ws_bytes = workspace_size(prob)
        if workspace is None:
            workspace = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device=dev)
        else:
            workspace = _need(workspace, "workspace", torch.uint8, 1, dev)
        if dev_status is not None:
            dev_status = _need(dev_status, "dev_status", torch.int32, 1, dev)
        ten = _Tensors(q=_ptr(q), k=_ptr(k), v=_ptr(v), sparse_idx=_ptr(idx),
                       sparse_count=_ptr(cnt), cu_seqlens_q=_ptr(cu), seqused_q=_ptr(squ),
                       seqused_kv=_ptr(sku), block_table=_ptr(bt), out=_ptr(out),
                       lse=_ptr(lse) if return_softmax_lse else None, cu_seqlens_kv=_ptr(cukv))
        _check(_load().gbsa_forward(ctypes.byref(prob.as_c()), ctypes.byref(ten),
                                    meta.data_ptr(), workspace.data_ptr(),
                                    workspace.numel() * workspace.element_size(),
                                    _ptr(dev_status), _stream_handle()),
               "gbsa_forward")
    return out, lse


def decode_dev_status(word: int) -> list:
    return [name for bit, name in DEV_BITS.items() if word & bit]


def backward(dout, q, k, v, out, lse, sparse_block_idx, sparse_block_count,
             block_shape: Sequence[int], *, metadata, cu_seqlens_q, seqused_kv, block_table=None,
             seqused_q=None, cu_seqlens_kv=None, softmax_scale: float = 0.0, win_left: int = -1,
             win_right: int = -1, num_ctas: int = 0, max_blocks_per_split: int = 0, dq=None,
             dk=None, dv=None, workspace=None, dev_status=None):
    """Gradients of out for the incoming gradient ``dout`` ([T, N1, D], the type
    of q): returns (dq, dk, dv) in fp32 -- dq [T, N1, D]; dk, dv compact
    [num_pages, 128, N2, D] for the page pool (whatever its page stride), or
    [T_kv, N2, D] for TND.  ``out`` and ``lse`` are the forward's results for
    the same inputs (lse [T, N1, 1] or [T, N1]); the other arguments, and
    ``metadata``, ``num_ctas`` and ``max_blocks_per_split``, are those of that
    forward call.  bf16 and fp16 only.  The pages give no backward: this is
    the exact gradient of the forward's function (a library addition)."""
    import torch
    q = _need(q, "q", q.dtype, 3)
    dev = q.device
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("backward: bf16 or fp16 inputs only")
    tnd = cu_seqlens_kv is not None
    for name, t in (("k", k), ("v", v)):
        if t is None or t.dtype != q.dtype or t.device != dev or t.dim() != (3 if tnd else 4):
            raise ValueError(f"{name}: expected {q.dtype} on {dev}, "
                             f"{'[T_kv, N2, D]' if tnd else '[num_pages, 128, N2, D]'}")
        if tnd and not t.is_contiguous():
            raise ValueError(f"{name}: TND k / v must be contiguous")
        if not tnd and t.stride()[1:] != (t.shape[2] * t.shape[3], t.shape[3], 1):
            raise ValueError(f"{name}: only dim0 (the page axis) may be strided")
    if k.shape != v.shape or k.stride() != v.stride():
        raise ValueError("k and v must have the same shape and strides")
    dout = _need(dout, "dout", q.dtype, 3, dev)
    out = _need(out, "out", q.dtype, 3, dev)
    if dout.shape != q.shape or out.shape != q.shape:
        raise ValueError("dout, out: expected the shape of q")
    T, N1, D = q.shape
    lse = _need(lse.reshape(T, N1) if lse is not None else None, "lse", torch.float32, 2, dev)
    idx = _need(sparse_block_idx, "sparse_block_idx", torch.int32, 3, dev)
    cnt = _need(sparse_block_count, "sparse_block_count", torch.int32, 2, dev)
    cu = _need(cu_seqlens_q, "cu_seqlens_q", torch.int64, 1, dev)
    sku = _need(seqused_kv, "seqused_kv", torch.int32, 1, dev)
    bt = None if tnd else _need(block_table, "block_table", torch.int32, 2, dev)
    cukv = _need(cu_seqlens_kv, "cu_seqlens_kv", torch.int64, 1, dev) if tnd else None
    squ = None if seqused_q is None else _need(seqused_q, "seqused_q", torch.int32, 1, dev)
    meta = _need(metadata, "metadata", torch.int32, 1, dev)
    prob = make_problem(q, k, idx, block_shape, bt, cu, softmax_scale=softmax_scale,
                        win_left=win_left, win_right=win_right, has_seqused_q=squ is not None,
                        num_ctas=num_ctas, max_blocks_per_split=max_blocks_per_split)
    kv_shape = (k.shape[0], k.shape[1], k.shape[2], k.shape[3]) if not tnd else tuple(k.shape)
    with torch.cuda.device(dev):
        dq = torch.empty((T, N1, D), dtype=torch.float32, device=dev) if dq is None else \
            _need(dq, "dq", torch.float32, 3, dev)
        dk = torch.empty(kv_shape, dtype=torch.float32, device=dev) if dk is None else dk
        dv = torch.empty(kv_shape, dtype=torch.float32, device=dev) if dv is None else dv
        for name, t in (("dk", dk), ("dv", dv)):
            if t.dtype != torch.float32 or tuple(t.shape) != kv_shape or not t.is_contiguous():
                raise ValueError(f"{name}: expected a contiguous fp32 tensor of shape {kv_shape}")
        n = ctypes.c_size_t(0)
        _check(_load().gbsa_backward_workspace_size(ctypes.byref(prob.as_c()), ctypes.byref(n)),
               "gbsa_backward_workspace_size")
        if workspace is None:
            workspace = torch.empty((max(int(n.value), 16),), dtype=torch.uint8, device=dev)
        if dev_status is not None:
            dev_status = _need(dev_status, "dev_status", torch.int32, 1, dev)
        ten = _Tensors(q=_ptr(q), k=_ptr(k), v=_ptr(v), sparse_idx=_ptr(idx),
                       sparse_count=_ptr(cnt), cu_seqlens_q=_ptr(cu), seqused_q=_ptr(squ),
                       seqused_kv=_ptr(sku), block_table=_ptr(bt), out=_ptr(out), lse=_ptr(lse),
                       cu_seqlens_kv=_ptr(cukv))
        _check(_load().gbsa_backward(ctypes.byref(prob.as_c()), ctypes.byref(ten), _ptr(dout),
                                     meta.data_ptr(), _ptr(dq), _ptr(dk), _ptr(dv),
                                     workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(),
                                     _ptr(dev_status), _stream_handle()),
               "gbsa_backward")
    return dq, dk, dv

