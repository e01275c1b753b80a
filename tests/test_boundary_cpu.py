"""The C-ABI library on the host: it loads without a GPU, exports every
function include/gbsa.h declares, and rejects every rule of the GBSA
article's "Constraints" section before anything is launched."""
import ctypes
import dataclasses
import os
import re

import pytest

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200 import build as build_mod
from block_sparse_paged_gbsa_b200.gbsa import Problem, _Tensors
from block_sparse_paged_gbsa_b200.workloads import workload
from oracle import scheduler

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "gbsa.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return gbsa.gbsa.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gbsa_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert {"gbsa_metadata", "gbsa_forward", "gbsa_metadata_size",
            "gbsa_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.gbsa_abi_version() == gbsa.gbsa.ABI_VERSION == 6
    for code in range(0, 9):
        assert lib.gbsa_status_string(code).decode().startswith("GBSA_")


def _problem(**kw):
    w = workload("tiny")
    base = dict(B=w.B, T=w.T, N1=w.N1, N2=w.N2, D=128, block_x=w.block_x,
                total_q_blocks=w.total_q_blocks, top_k=w.top_k,
                max_pages_per_seq=w.max_pages_per_seq, num_pages=w.num_pages,
                kv_page_stride=w.kv_page_stride, scale=w.scale, num_ctas=148, return_lse=1)
    base.update(kw)
    return Problem(**base), w


def test_header_constants_match_the_binding():
    text = open(HEADER).read()
    abi = int(re.search(r"#define GBSA_ABI_VERSION (\d+)", text).group(1))
    fused = int(re.search(r"#define GBSA_METADATA_FUSED_MAX_B (\d+)", text).group(1))
    assert abi == gbsa.gbsa.ABI_VERSION
    assert fused == gbsa.gbsa.METADATA_FUSED_MAX_B


def test_metadata_size_matches_format(lib):
    for ctas, forced in ((148, 0), (7, 3)):
        p, w = _problem(num_ctas=ctas, max_blocks_per_split=forced)
        g = scheduler.geometry(dict(w.problem_kwargs(), num_ctas=ctas,
                                    max_blocks_per_split=forced))
        assert gbsa.metadata_size(p) == 4 * g["total"]
        ws = gbsa.workspace_size(p)
        rpu = g["rows_per_unit"]
        o_bytes = g["slot_cap"] * rpu * 128 * 4
        assert ws == ((o_bytes + 255) // 256) * 256 + g["slot_cap"] * rpu * 4


CASES = [
    (dict(D=64), "GBSA_ERR_UNSUPPORTED"),
    (dict(block_y=64), "GBSA_ERR_UNSUPPORTED"),
    (dict(N1=6, N2=4), "GBSA_ERR_SHAPE"),
    (dict(N1=2, N2=4), "GBSA_ERR_SHAPE"),
    (dict(N1=258, N2=2), "GBSA_ERR_UNSUPPORTED"),
    (dict(top_k=257), "GBSA_ERR_UNSUPPORTED"),
    (dict(mask_mode=0), "GBSA_ERR_UNSUPPORTED"),
    (dict(is_packed_gqa=2), "GBSA_ERR_INVALID_ARG"),
    (dict(B=0), "GBSA_ERR_SHAPE"),
    (dict(top_k=0), "GBSA_ERR_SHAPE"),
    (dict(block_x=0), "GBSA_ERR_SHAPE"),
    (dict(win_left=-2), "GBSA_ERR_INVALID_ARG"),
    (dict(scale=-1.0), "GBSA_ERR_INVALID_ARG"),
    (dict(dtype=3), "GBSA_ERR_INVALID_ARG"),                # not bf16, fp16 or E4M3
    (dict(dtype=2, q_scale=0.0), "GBSA_ERR_INVALID_ARG"),   # E4M3 scales must be > 0
    (dict(dtype=2, k_scale=-1.0), "GBSA_ERR_INVALID_ARG"),
    (dict(dtype=2, v_scale=float("inf")), "GBSA_ERR_INVALID_ARG"),
    (dict(dtype=2, v_scale=float("nan")), "GBSA_ERR_INVALID_ARG"),
    (dict(dtype=2, q_scale=1e-20, k_scale=1e-20), "GBSA_ERR_INVALID_ARG"),  # folded scale underflows
    (dict(softmax_precision=2), "GBSA_ERR_INVALID_ARG"),
    (dict(softmax_precision=-1), "GBSA_ERR_INVALID_ARG"),
    (dict(kv_layout=2), "GBSA_ERR_INVALID_ARG"),            # neither paged nor TND
]


@pytest.mark.parametrize("kw,expected", CASES)
def test_problem_rules(lib, kw, expected):
    p, _ = _problem(**kw)
    with pytest.raises(gbsa.GbsaError) as e:
        gbsa.metadata_size(p)
    assert expected in str(e.value)


FWD_CASES = [
    (dict(kv_page_stride=128 * 2 * 128 - 256), "GBSA_ERR_SHAPE"),      # smaller than a page
    (dict(kv_page_stride=128 * 2 * 128 + 128), "GBSA_ERR_SHAPE"),      # not a multiple of N2*D
    (dict(num_pages=0), "GBSA_ERR_SHAPE"),
    (dict(T=0), "GBSA_ERR_SHAPE"),
    (dict(kv_layout=1, T_kv=0), "GBSA_ERR_SHAPE"),          # TND without rows
]


def _call_forward(lib, p, tensors, meta=16, ws=16, ws_bytes=1 << 30):
    return lib.gbsa_forward(ctypes.byref(p.as_c()), ctypes.byref(tensors), meta, ws, ws_bytes,
                            None, None)


def _fake_tensors(**kw):
    # addresses that are never dereferenced: every case fails validation first
    f = dict(q=1 << 20, k=2 << 20, v=3 << 20, sparse_idx=4 << 20, sparse_count=5 << 20,
             cu_seqlens_q=6 << 20, seqused_kv=7 << 20, block_table=8 << 20, out=9 << 20,
             lse=10 << 20)
    f.update(kw)
    return _Tensors(**f)


@pytest.mark.parametrize("kw,expected", FWD_CASES)
def test_forward_shape_rules(lib, kw, expected):
    p, _ = _problem(**kw)
    rc = _call_forward(lib, p, _fake_tensors())
    assert lib.gbsa_status_string(rc).decode() == expected


def test_forward_pointer_rules(lib):
    p, _ = _problem()
    assert _call_forward(lib, p, _fake_tensors(q=None)) == 1              # INVALID_ARG
    assert _call_forward(lib, p, _fake_tensors(lse=None)) == 1            # lse requested
    p2, _ = _problem(has_seqused_q=1)
    assert _call_forward(lib, p2, _fake_tensors()) == 1                   # seqused_q missing
    assert _call_forward(lib, p, _fake_tensors(k=(2 << 20) + 8)) == 4     # ALIGNMENT
    assert _call_forward(lib, p, _fake_tensors(), meta=24) == 4
    assert _call_forward(lib, p, _fake_tensors(), ws_bytes=0) == 5        # workspace too small


def _call_backward(lib, p, tensors, dout=11 << 20, meta=16, dq=12 << 20, dk=13 << 20,
                   dv=14 << 20, ws=16, ws_bytes=1 << 30):
    return lib.gbsa_backward(ctypes.byref(p.as_c()), ctypes.byref(tensors), dout, meta, dq, dk, dv,
                             ws, ws_bytes, None, None)


def test_backward_host_rules(lib):
    """gbsa_backward checks its arguments before any launch (these cases never
    reach the device)."""
    p, w = _problem()
    s = lambda rc: lib.gbsa_status_string(rc).decode()
    assert s(_call_backward(lib, p, _fake_tensors(), dout=None)) == "GBSA_ERR_INVALID_ARG"
    assert s(_call_backward(lib, p, _fake_tensors(), dk=None)) == "GBSA_ERR_INVALID_ARG"
    # lse is an input here, whatever return_lse says
    assert s(_call_backward(lib, _problem(return_lse=0)[0], _fake_tensors(lse=None))) == \
        "GBSA_ERR_INVALID_ARG"
    assert s(_call_backward(lib, p, _fake_tensors(), dq=(12 << 20) + 8)) == "GBSA_ERR_ALIGNMENT"
    assert s(_call_backward(lib, p, _fake_tensors(), dout=(11 << 20) + 2)) == "GBSA_ERR_ALIGNMENT"
    assert s(_call_backward(lib, p, _fake_tensors(), ws_bytes=16)) == "GBSA_ERR_WORKSPACE_TOO_SMALL"
    p8, _ = _problem(dtype=2, q_scale=1.0, k_scale=1.0, v_scale=1.0)
    assert s(_call_backward(lib, p8, _fake_tensors())) == "GBSA_ERR_UNSUPPORTED"
    n = ctypes.c_size_t(0)
    assert lib.gbsa_backward_workspace_size(ctypes.byref(p.as_c()), ctypes.byref(n)) == 0
    assert n.value == (w.T * w.N1 * 4 + 15) // 16 * 16


def test_no_device_means_no_default_cta_count(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    p, _ = _problem(num_ctas=0)
    with pytest.raises(gbsa.GbsaError) as e:
        gbsa.metadata_size(p)
    assert "NO_DEVICE" in str(e.value)


def test_metadata_pointer_rules(lib):
    p, _ = _problem()
    t = _fake_tensors(sparse_idx=None)
    rc = lib.gbsa_metadata(ctypes.byref(p.as_c()), ctypes.byref(t), 16, 1 << 30, None, None)
    assert rc == 1
    rc = lib.gbsa_metadata(ctypes.byref(p.as_c()), ctypes.byref(_fake_tensors()), 16, 8, None,
                           None)
    assert rc == 6                                                        # METADATA_TOO_SMALL


def test_softmax_precision_one_is_accepted(lib):
    # both modes are accepted for every element type; the work list (and its
    # size) does not depend on the mode
    for dt in (0, 1, 2):
        p, _ = _problem(dtype=dt, softmax_precision=1)
        assert gbsa.metadata_size(p) == gbsa.metadata_size(_problem(dtype=dt)[0])


def test_fp8_scales_are_ignored_for_16_bit_types(lib):
    # the dequantization scales belong to the E4M3 mode only
    for dt in (0, 1):
        p, _ = _problem(dtype=dt, q_scale=0.0, k_scale=float("nan"))
        assert gbsa.metadata_size(p) > 0
    p, _ = _problem(dtype=2, q_scale=0.5, k_scale=2.0, v_scale=3.0)
    assert gbsa.metadata_size(p) > 0


def test_binding_element_types():
    # the Python binding maps torch dtypes to gbsa_problem.dtype and out's type
    import torch
    from block_sparse_paged_gbsa_b200.gbsa import _dtype_code, _out_dtype, make_problem
    w = workload("tiny")
    for dt, code, out in ((torch.bfloat16, 0, torch.bfloat16), (torch.float16, 1, torch.float16),
                          (torch.float8_e4m3fn, 2, torch.bfloat16)):
        q = torch.zeros((w.T, w.N1, w.D), dtype=dt)
        k = torch.zeros((w.num_pages, 128, w.N2, w.D), dtype=dt)
        assert _dtype_code(q) == code and _out_dtype(q) == out
        idx = torch.zeros((w.N2, w.total_q_blocks, w.top_k), dtype=torch.int32)
        bt = torch.zeros((w.B, w.max_pages_per_seq), dtype=torch.int32)
        cu = torch.zeros((w.B + 1,), dtype=torch.int64)
        prob = make_problem(q, k, idx, [w.block_x, 128], bt, cu, dequant_scales=(0.5, 2.0, 4.0),
                            num_ctas=148)
        assert prob.dtype == code and (prob.q_scale, prob.k_scale, prob.v_scale) == (0.5, 2.0, 4.0)
        assert gbsa.metadata_size(prob) > 0
    with pytest.raises(ValueError):
        _dtype_code(torch.zeros(1, dtype=torch.float32))


def test_binding_rejects_other_element_types():
    # checked before anything touches a device
    import torch
    w = workload("tiny")
    q = torch.zeros((w.T, w.N1, w.D), dtype=torch.float32)
    z = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="bf16, fp16 or float8_e4m3fn"):
        gbsa.forward(q, q, q, z, z, [w.block_x, 128], metadata=z, cu_seqlens_q=z, seqused_kv=z,
                     block_table=z)


@pytest.mark.parametrize("kw,match", [
    (dict(layout_q="BSND"), "layout_q"),
    (dict(layout_kv="BNSD"), "layout_kv"),
    (dict(quant_mode=1), "quant_mode"),
    (dict(quant_mode=5), "quant_mode"),            # bf16 inputs with the E4M3 mode
    (dict(attn_mask=1), "attn_mask"),
    (dict(p_quant_scale=1.0), "p_quant_scale"),
    (dict(attention_out_dtype="float16"), "attention_out_dtype"),
    (dict(layout_kv="TND"), "layout_kv"),          # TND without cu_seqlens_kv
])
def test_article_arguments_are_checked_before_launch(kw, match):
    # the remaining arguments of the article's PyTorch API: accepted where the
    # library implements them, rejected (before any device use) otherwise
    import torch
    w = workload("tiny")
    q = torch.zeros((w.T, w.N1, w.D), dtype=torch.bfloat16)
    z = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError, match=match):
        gbsa.forward(q, q, q, z, z, [w.block_x, 128], metadata=z, cu_seqlens_q=z, seqused_kv=z,
                     block_table=z, **kw)


def test_article_arguments_accepted_forms_reach_the_device_checks():
    # consistent values pass the argument checks (and stop only at the
    # device check on a host without CUDA tensors)
    import torch
    w = workload("tiny")
    z = torch.zeros(1, dtype=torch.int32)
    for dt, qm, od in ((torch.bfloat16, 0, torch.bfloat16), (torch.float8_e4m3fn, 5, torch.bfloat16)):
        q = torch.zeros((w.T, w.N1, w.D), dtype=dt)
        with pytest.raises(ValueError, match="CUDA"):
            gbsa.forward(q, q, q, z, z, [w.block_x, 128], metadata=z, cu_seqlens_q=z,
                         seqused_kv=z, block_table=z, layout_q="TND", layout_kv="PA_BBND",
                         quant_mode=qm, attention_out_dtype=od, dst_type_max=0.0)
    with pytest.raises(ValueError, match="layout"):
        gbsa.metadata(z, z, 8, 2, 128, [64, 128], cu_seqlens_q=z, seqused_kv=z, layout_q="BSH")
