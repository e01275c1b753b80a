"""Pins of the oracle's gradients (oracle.attention_backward).  The pages give
no backward; the oracle takes the analytic gradient of the forward function.
It is pinned here against quantities that do not use that formula:

* central finite differences of the forward oracle's L = sum(dout * out),
  with Richardson extrapolation (error O(h^4)), at sampled coordinates of q,
  k and v; inputs are fp16 values on a 2^-6 grid, so x +- h is exact;
* closed forms: values V equal for every key (out is constant: dq = dk = 0);
  a single visible key per row (its weight is 1: dq = dk = 0, dv = sum of
  dout); the weights of a row sum to 1 (the dv of all keys sums to the dout
  of the rows that see a key) and the score gradients of a row sum to 0 (the
  dk of all keys sums to 0).

Five planted mistakes in the gradient code (test_mutant_is_caught) each
fail at least one of these pins.
"""
import numpy as np
import pytest

import oracle
from block_sparse_paged_gbsa_b200.workloads import generate

PAGE = 128


def _grid_values(rng, shape, lim=1.0):
    """fp16 values that are multiples of 2^-6 in [-lim, lim]."""
    return (rng.integers(-int(lim * 64), int(lim * 64) + 1, size=shape) / 64.0).astype(np.float64)


def _problem(seed, window=False, D=8, N1=4, N2=2):
    # keys and queries: short sequences over a few pages, several Q blocks
    w = generate(name=f"bwd{seed}", seed=seed, q_storage=[6, 9], q_used=[6, 8], kv_used=[200, 300],
                 N1=N1, N2=N2, block_x=4, top_k=3, selection="random_causal",
                 win_left=150 if window else -1, win_right=0 if window else -1,
                 list_order="shuffled")
    return w


def _kw(w, D, dtype="fp16", lib=None):
    npages = w.num_pages
    stride = PAGE * w.N2 * D
    return dict(kv_page_stride=stride, num_pages=npages, sparse_idx=w.sparse_idx,
                sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q,
                seqused_q=w.q_used if w.has_seqused_q else None, seqused_kv=w.kv_used,
                block_table=w.block_table, block_x=w.block_x, scale=D ** -0.5,
                win_left=w.win_left, win_right=w.win_right, dtype=dtype, lib=lib)


def _bits(x):
    b = x.astype(np.float16)
    assert np.array_equal(b.astype(np.float64), x)  # exact on the grid
    return b.view(np.uint16)


def _loss(q, k, v, g, kw):
    out, _ = oracle.attention(q_bits=_bits(q), k_bits=_bits(k), v_bits=_bits(v), **kw)
    return float(np.sum(g * out))


def _values(w, D, seed):
    rng = np.random.default_rng(seed)
    T = int(w.cu_seqlens_q[-1])
    q = _grid_values(rng, (T, w.N1, D))
    k = _grid_values(rng, (w.num_pages * PAGE * w.N2 * D,))
    v = _grid_values(rng, (w.num_pages * PAGE * w.N2 * D,))
    g = _grid_values(rng, (T, w.N1, D))
    return q, k, v, g


@pytest.mark.parametrize("window", [False, True])
def test_gradients_match_finite_differences(window, lib=None):
    D = 8
    w = _problem(11 + window, window, D)
    kw = _kw(w, D, lib=lib)
    q, k, v, g = _values(w, D, 3)
    dq, dk, dv = oracle.attention_backward(q_bits=_bits(q), k_bits=_bits(k), v_bits=_bits(v),
                                           dout_bits=_bits(g), **kw)
    rng = np.random.default_rng(5)
    h = 2.0 ** -7

    def numeric(arr, idx):
        def f(delta):
            a = arr.copy()
            a.flat[idx] += delta
            args = {"q": q, "k": k, "v": v}
            args[name] = a
            return _loss(args["q"], args["k"], args["v"], g, kw)
        d1 = (f(h) - f(-h)) / (2 * h)
        d2 = (f(h / 2) - f(-h / 2)) / h
        return (4 * d2 - d1) / 3

    checked = 0
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        flat = grad.reshape(-1)
        nz = np.flatnonzero(flat)
        assert nz.size > 0, name
        # coordinates with a gradient, and some without (keys nobody sees)
        pick = list(rng.choice(nz, size=min(30, nz.size), replace=False))
        pick += list(rng.choice(np.arange(flat.size), size=10, replace=False))
        for idx in pick:
            if abs(arr.flat[idx]) > 1.0 - h:  # keep x +- h on the grid's range
                continue
            num = numeric(arr, idx)
            assert abs(num - flat[idx]) <= 1e-7 + 1e-6 * abs(flat[idx]), (name, idx, num, flat[idx])
            checked += 1
    assert checked >= 60


def test_constant_values_give_no_query_or_key_gradient(lib=None):
    D = 8
    w = _problem(21, True, D)
    kw = _kw(w, D, lib=lib)
    q, k, v, g = _values(w, D, 4)
    c = _grid_values(np.random.default_rng(9), (w.N2, D))
    v = np.broadcast_to(c, (v.size // (w.N2 * D), w.N2, D)).reshape(-1).copy()  # one vector per head
    dq, dk, dv = oracle.attention_backward(q_bits=_bits(q), k_bits=_bits(k), v_bits=_bits(v),
                                           dout_bits=_bits(g), **kw)
    assert np.abs(dq).max() <= 1e-12 and np.abs(dk).max() <= 1e-12
    assert np.abs(dv).max() > 1e-3  # v still gets a gradient


def test_single_key_rows(lib=None):
    """block_x = 1, one-token rows at position 0 of their sequences: each
    row sees exactly key 0, with weight 1."""
    D = 8
    w = generate(name="one", seed=31, q_storage=[1, 1, 1], q_used=[1, 1, 1], kv_used=[1, 1, 1],
                 N1=4, N2=2, block_x=1, top_k=2, selection="all_causal")
    kw = _kw(w, D, lib=lib)
    q, k, v, g = _values(w, D, 6)
    dq, dk, dv = oracle.attention_backward(q_bits=_bits(q), k_bits=_bits(k), v_bits=_bits(v),
                                           dout_bits=_bits(g), **kw)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    dv4 = dv.reshape(-1, PAGE, w.N2, D)
    G = w.N1 // w.N2
    for b in range(3):
        page = w.block_table[b][0]
        for kvh in range(w.N2):
            expect = g[b, kvh * G:(kvh + 1) * G].sum(axis=0)  # the G heads that read this key
            assert np.array_equal(dv4[page, 0, kvh], expect)


def test_row_sums(lib=None):
    """sum over keys of dv = sum of dout over rows that see a key; sum over
    keys of dk = 0 (the score gradients of each row sum to zero)."""
    D = 8
    w = _problem(41, True, D)
    kw = _kw(w, D, lib=lib)
    q, k, v, g = _values(w, D, 8)
    dq, dk, dv = oracle.attention_backward(q_bits=_bits(q), k_bits=_bits(k), v_bits=_bits(v),
                                           dout_bits=_bits(g), **kw)
    _, lse = oracle.attention(q_bits=_bits(q), k_bits=_bits(k), v_bits=_bits(v), **kw)
    sees = np.isfinite(lse)                      # [T, N1]
    G = w.N1 // w.N2
    dv_h = dv.reshape(-1, w.N2, D).sum(axis=0)   # per KV head
    dk_h = dk.reshape(-1, w.N2, D).sum(axis=0)
    for kvh in range(w.N2):
        heads = slice(kvh * G, (kvh + 1) * G)
        expect = (g[:, heads] * sees[:, heads, None]).sum(axis=(0, 1))
        assert np.allclose(dv_h[kvh], expect, rtol=0, atol=1e-12)
        assert np.abs(dk_h[kvh]).max() <= 1e-12
    assert sees.any() and (~sees).any()


# Planted mistakes in the oracle's gradient code: every one must fail a pin.
MUTANTS = {
    "delta_dropped": ("const double ds = w * (gv - dlt);", "const double ds = w * gv;"),
    "dk_unscaled": ("dk[base + d] += scale * ds * c.widen(qrow[d]);",
                    "dk[base + d] += ds * c.widen(qrow[d]);"),
    "dv_unweighted": ("dv[base + d] += w * g;", "dv[base + d] += g;"),
    "dq_from_v": ("dqr[d] += scale * ds * c.widen(krow[d]);",
                  "dqr[d] += scale * ds * c.widen(vrow[d]);"),
    "weight_without_lse": ("const double w = exp(score[i] - lse);", "const double w = exp(score[i]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load_library(oracle.compile_to(str(path), str(tmp_path / f"{name}.so")))
    pins = (lambda: test_gradients_match_finite_differences(True, lib=lib),
            lambda: test_constant_values_give_no_query_or_key_gradient(lib=lib),
            lambda: test_single_key_rows(lib=lib), lambda: test_row_sums(lib=lib))
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"{name} passes every pin"



def test_tnd_layout_gives_the_paged_gradients():
    """The same logical keys in the TND layout (with NaN rows between the
    sequences) and in the paged pool give the same dq, and the same dk / dv
    at every (sequence, position, head)."""
    import torch

    from block_sparse_paged_gbsa_b200.workloads import make_values, pool_view, tnd_kv
    from tests.helpers import bf16_bits

    w = generate(name="bwdtnd", seed=51, q_storage=[40, 70], q_used=[40, 66], kv_used=[300, 150],
                 N1=4, N2=2, block_x=16, top_k=3, selection="random_causal", win_left=100,
                 win_right=0, page_stride_factor=1.5, list_order="shuffled")
    q, kf, vf = make_values(w, "cpu", dtype=torch.float16)
    g = torch.randn(q.shape, generator=torch.Generator().manual_seed(3)).to(torch.float16)
    kt, vt, cu_kv = tnd_kv(w, kf, vf, seed=1)
    common = dict(q_bits=bf16_bits(q), dout_bits=bf16_bits(g), sparse_idx=w.sparse_idx,
                  sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q,
                  seqused_q=w.seqused_q, seqused_kv=w.kv_used, block_x=w.block_x, scale=w.scale,
                  win_left=w.win_left, win_right=w.win_right, dtype="fp16")
    pq, pk, pv = oracle.attention_backward(k_bits=bf16_bits(kf), v_bits=bf16_bits(vf),
                                           kv_page_stride=w.kv_page_stride,
                                           num_pages=w.num_pages, block_table=w.block_table,
                                           **common)
    tq, tk, tv = oracle.attention_backward(k_bits=bf16_bits(kt), v_bits=bf16_bits(vt),
                                           kv_page_stride=0, num_pages=0, block_table=None,
                                           cu_seqlens_kv=cu_kv, **common)
    assert np.array_equal(pq, tq) and np.abs(pq).max() > 0
    D = w.D
    for b in range(w.B):
        for pos in range(int(w.kv_used[b])):
            page, r = int(w.block_table[b, pos // PAGE]), pos % PAGE
            for h in range(w.N2):
                po = page * w.kv_page_stride + (r * w.N2 + h) * D
                to = ((int(cu_kv[b]) + pos) * w.N2 + h) * D
                assert np.array_equal(pk[po:po + D], tk[to:to + D])
                assert np.array_equal(pv[po:po + D], tv[to:to + D])
    assert np.abs(tk).max() > 0
