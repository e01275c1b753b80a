"""Seeded synthetic inputs for block-sparse paged GQA attention.

This module only draws inputs: sequence lengths, page placement, block
tables, block selections and bf16 values.  It holds none of the attention
arithmetic, and both the CUDA path and the CPU oracle are fed from it.

Structure (lengths, pages, selections) comes from numpy ``PCG64(seed)`` on
the host; the bulk bf16 values (Q, K, V ~ N(0, 1)) come from a torch
generator seeded with the same seed on the device the values are made on.
Positions that no selection may legally read are filled with NaN so that a
stray read shows up in the output: pool pages that no sequence owns, the
padding between pages when the pool's page stride is larger than a page,
and the tail of each sequence's last page past seqused_kv.

Named workloads (``WORKLOADS``), with the readings used where the pages leave
a choice open:

* ``tiny``    -- 2 x 512 tokens, N1=8, N2=2, block [64,128], top_k=4, random
  causal selections that always hold the diagonal block.
* ``dense``   -- 4 x 4096 tokens, N1=32, N2=8, block [128,128], top_k=32,
  every causal block selected (dense causal attention).
* ``long``    -- 1 x 131072 tokens, N1=32, N2=4, block [128,128], top_k=64:
  block 0, the diagonal block and 62 more causal blocks drawn without
  replacement.
* ``decode``  -- 64 sequences of one query token, KV lengths ~ U[8192, 65536],
  N1=64, N2=8, block [1,128], top_k=256, count ~ U{64..min(256, blocks)}
  always holding the last (partial) page.
* ``ragged``  -- 16 sequences, storage lengths lognormal (median 4096,
  sigma 1.0, clipped to [512, 32768]), seqused = storage - U[0,127] for Q and
  KV, N1=40, N2=8, block [64,128], top_k=128 random causal selections,
  window (4096, 0), page stride 1.25 x 128*N2*D.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

PAGE = 128
HEAD_DIM = 128


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    B: int
    N1: int
    N2: int
    D: int
    block_x: int
    top_k: int
    win_left: int
    win_right: int
    return_lse: bool
    has_seqused_q: bool
    scale: float
    q_storage: np.ndarray      # int64 [B]
    q_used: np.ndarray         # int32 [B]
    kv_used: np.ndarray        # int32 [B]
    cu_seqlens_q: np.ndarray   # int64 [B+1]
    block_table: np.ndarray    # int32 [B, max_pages_per_seq]
    num_pages: int
    kv_page_stride: int        # elements
    sparse_idx: np.ndarray     # int32 [N2, total_q_blocks, top_k]
    sparse_count: np.ndarray   # int32 [N2, total_q_blocks]
    owned_pages: np.ndarray    # bool [num_pages]: page holds some sequence's keys

    @property
    def T(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def total_q_blocks(self) -> int:
        return int(self.sparse_count.shape[1])

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def G(self) -> int:
        return self.N1 // self.N2

    @property
    def seqused_q(self) -> Optional[np.ndarray]:
        return self.q_used if self.has_seqused_q else None

    @property
    def pool_elems(self) -> int:
        return self.num_pages * self.kv_page_stride

    def problem_kwargs(self) -> dict:
        return dict(B=self.B, T=self.T, N1=self.N1, N2=self.N2, D=self.D,
                    block_x=self.block_x, total_q_blocks=self.total_q_blocks,
                    top_k=self.top_k, max_pages_per_seq=self.max_pages_per_seq,
                    num_pages=self.num_pages, kv_page_stride=self.kv_page_stride,
                    scale=self.scale, win_left=self.win_left, win_right=self.win_right,
                    return_lse=self.return_lse, has_seqused_q=self.has_seqused_q)


def _q_blocks(q_storage, block_x):
    return [int(-(-int(s) // block_x)) for s in q_storage]


def _choose(rng, pool, k):
    pool = np.asarray(pool, np.int64)
    if k >= pool.size:
        return pool.copy()
    return rng.choice(pool, size=k, replace=False)


def generate(*, name="custom", seed=0, q_storage, q_used=None, kv_used=None, N1, N2, block_x,
             top_k, selection="random_causal", win_left=-1, win_right=-1, return_lse=True,
             has_seqused_q=None, scale=None, page_stride_factor=1.0, extra_pages=None,
             count_range=None, pad_fill="garbage", list_order="ascending") -> Workload:
    """Draws the structure of one workload (no bf16 values; see ``make_values``).

    selection: "random_causal" | "all_causal" | "sink_diag_random" | "decode" | "random_any".
    count_range: (lo, hi) bounds of the count draw where the selection uses one.
    list_order: order of each selection list -- "ascending" (the named
    workloads), "descending" (the diagonal / last block first) or "shuffled"
    (a random permutation); "drawn" keeps the order of the draw.
    """
    if list_order not in ("ascending", "descending", "shuffled", "drawn"):
        raise ValueError(list_order)
    rng = np.random.Generator(np.random.PCG64(seed))
    # shuffled lists draw from their own stream: the selections stay those of
    # the other orders
    order_rng = np.random.Generator(np.random.PCG64(seed + 31337))
    q_storage = np.asarray(q_storage, np.int64)
    B = int(q_storage.size)
    q_used = q_storage.astype(np.int32) if q_used is None else np.asarray(q_used, np.int32)
    kv_used = q_used.copy() if kv_used is None else np.asarray(kv_used, np.int32)
    if has_seqused_q is None:
        has_seqused_q = bool(np.any(q_used != q_storage))
    D = HEAD_DIM
    G = N1 // N2
    cu = np.zeros(B + 1, np.int64)
    cu[1:] = np.cumsum(q_storage)

    # Physical pages: every sequence owns ceil(kv_used/128) of them, placed by a
    # random permutation of the pool; a few spare pages belong to nobody.
    pages_per_seq = [int(-(-int(k) // PAGE)) for k in kv_used]
    need = sum(pages_per_seq)
    if extra_pages is None:
        extra_pages = max(1, need // 16)
    num_pages = max(1, need + int(extra_pages))
    perm = rng.permutation(num_pages).astype(np.int32)
    maxp = max(1, max(pages_per_seq))
    block_table = np.full((B, maxp), -1, np.int32)
    owned = np.zeros(num_pages, bool)
    cursor = 0
    for b, npg in enumerate(pages_per_seq):
        block_table[b, :npg] = perm[cursor:cursor + npg]
        owned[perm[cursor:cursor + npg]] = True
        cursor += npg
    page_elems = PAGE * N2 * D
    stride = int(math.ceil(page_elems * page_stride_factor / (N2 * D))) * (N2 * D)

    qblocks = _q_blocks(q_storage, block_x)
    tqb = sum(qblocks)
    idx = np.zeros((N2, tqb, top_k), np.int32)
    cnt = np.zeros((N2, tqb), np.int32)
    qb = 0
    for b in range(B):
        qs, qu, ku = int(q_storage[b]), int(q_used[b]), int(kv_used[b])
        nblk = pages_per_seq[b]
        off = ku - qu
        for qbl in range(qblocks[b]):
            t_lo = qbl * block_x
            t_hi = min(t_lo + block_x, qu)          # used rows of this Q block
            for h in range(N2):
                if selection == "decode":
                    lo, hi = count_range or (64, 256)
                    c = int(rng.integers(min(lo, nblk), min(hi, nblk) + 1)) if nblk else 0
                    chosen = [nblk - 1] + list(_choose(rng, np.arange(nblk - 1), c - 1)) if c else []
                elif selection == "random_any":
                    c = int(rng.integers(0, top_k + 1))
                    chosen = list(rng.integers(0, max(nblk, 1), size=c))
                elif t_hi <= t_lo or t_hi - 1 + off < 0:
                    chosen = []                       # no used row sees any key
                else:
                    nc = min((t_hi - 1 + off) // PAGE + 1, nblk)   # causal blocks
                    diag = nc - 1
                    if selection == "all_causal":
                        chosen = list(range(nc))[:top_k]
                    elif selection == "sink_diag_random":
                        if nc <= top_k:
                            chosen = list(range(nc))
                        elif top_k == 1:            # room for the diagonal block only
                            chosen = [diag]
                        else:
                            chosen = [0, diag] + list(_choose(rng, np.arange(1, diag), top_k - 2))
                    elif selection == "random_causal":
                        lo, hi = count_range or (1, top_k)
                        c = int(rng.integers(max(1, lo), min(hi, nc, top_k) + 1))
                        chosen = [diag] + list(_choose(rng, np.arange(diag), c - 1))
                    else:
                        raise ValueError(selection)
                chosen = np.asarray(chosen, np.int64)
                if list_order == "ascending":
                    chosen = np.sort(chosen)
                elif list_order == "descending":
                    chosen = np.sort(chosen)[::-1]
                elif list_order == "shuffled":
                    chosen = order_rng.permutation(np.sort(chosen))
                c = int(chosen.size)
                cnt[h, qb] = c
                idx[h, qb, :c] = chosen
                if pad_fill == "garbage" and c < top_k:
                    idx[h, qb, c:] = rng.integers(-3, 2 * nblk + 4, size=top_k - c)
            qb += 1
    return Workload(name=name, seed=seed, B=B, N1=N1, N2=N2, D=D, block_x=block_x, top_k=top_k,
                    win_left=win_left, win_right=win_right, return_lse=return_lse,
                    has_seqused_q=bool(has_seqused_q),
                    scale=float(1.0 / math.sqrt(D) if scale is None else scale),
                    q_storage=q_storage, q_used=q_used, kv_used=kv_used, cu_seqlens_q=cu,
                    block_table=block_table, num_pages=num_pages, kv_page_stride=stride,
                    sparse_idx=idx, sparse_count=cnt, owned_pages=owned)


def _lognormal_lengths(rng, n, median, sigma, lo, hi):
    x = np.exp(np.log(median) + sigma * rng.standard_normal(n))
    return np.clip(np.round(x), lo, hi).astype(np.int64)


def workload(name: str, seed: Optional[int] = None, scale_down: int = 1,
             list_order: str = "ascending") -> Workload:
    """One of the five named workloads.  ``scale_down`` > 1 shrinks sequence
    lengths (and the decode KV range) by that factor for oracle-sized cases
    that keep the same structure; ``list_order`` as in ``generate``."""
    s = scale_down
    o = dict(list_order=list_order)
    if name == "tiny":
        seed = 1001 if seed is None else seed
        return generate(name=name, seed=seed, q_storage=[512 // s] * 2, N1=8, N2=2, block_x=64,
                        top_k=4, selection="random_causal", **o)
    if name == "dense":
        seed = 1002 if seed is None else seed
        n = max(4096 // s, 128)
        return generate(name=name, seed=seed, q_storage=[n] * 4, N1=32, N2=8, block_x=128,
                        top_k=max(n // 128, 1), selection="all_causal", **o)
    if name == "long":
        seed = 1003 if seed is None else seed
        return generate(name=name, seed=seed, q_storage=[max(131072 // s, 256)], N1=32, N2=4,
                        block_x=128, top_k=64, selection="sink_diag_random", **o)
    if name == "decode":
        seed = 1004 if seed is None else seed
        rng = np.random.Generator(np.random.PCG64(seed + 7919))
        kv = rng.integers(8192 // s, 65536 // s + 1, size=64).astype(np.int32)
        top_k = 256
        return generate(name=name, seed=seed, q_storage=[1] * 64, q_used=[1] * 64, kv_used=kv,
                        N1=64, N2=8, block_x=1, top_k=top_k, selection="decode",
                        count_range=(max(64 // s, 1), 256), has_seqused_q=False, **o)
    if name == "ragged":
        seed = 1005 if seed is None else seed
        rng = np.random.Generator(np.random.PCG64(seed + 7919))
        qs = _lognormal_lengths(rng, 16, 4096 / s, 1.0, max(512 // s, 128), 32768 // s)
        used = (qs - rng.integers(0, 128, size=16)).astype(np.int32)
        used = np.maximum(used, 1)
        return generate(name=name, seed=seed, q_storage=qs, q_used=used, kv_used=used, N1=40,
                        N2=8, block_x=64, top_k=128, selection="random_causal",
                        win_left=4096 // s, win_right=0, page_stride_factor=1.25,
                        has_seqused_q=True, **o)
    raise KeyError(name)


WORKLOADS = ("tiny", "dense", "long", "decode", "ragged")


def make_values(w: Workload, device="cpu", nan_fill=True, dtype=None):
    """Draws q [T,N1,D] and the K/V pools on ``device``: N(0,1) rounded to
    ``dtype`` (torch.bfloat16, the default, torch.float16 or
    torch.float8_e4m3fn; unreadable pool slots are NaN in each).

    Returns (q, k_flat, v_flat): the pools are flat buffers of
    num_pages*kv_page_stride elements; ``pool_view`` gives the
    [num_pages, 128, N2, D] view with the page stride.
    """
    import torch

    dtype = torch.bfloat16 if dtype is None else dtype
    g = torch.Generator(device=device)
    g.manual_seed(int(w.seed))
    q = torch.randn((w.T, w.N1, w.D), generator=g, device=device, dtype=torch.float32)
    q = q.to(dtype)
    pools = []
    for _ in range(2):
        flat = torch.randn((w.pool_elems,), generator=g, device=device, dtype=torch.float32)
        if nan_fill:
            _fill_unreadable(w, flat)
        pools.append(flat.to(dtype))
    return q, pools[0], pools[1]


def _fill_unreadable(w: Workload, flat):
    import torch

    nan = float("nan")
    page_elems = PAGE * w.N2 * w.D
    view2d = flat.view(w.num_pages, w.kv_page_stride)
    if w.kv_page_stride > page_elems:
        view2d[:, page_elems:] = nan
    unowned = np.nonzero(~w.owned_pages)[0]
    if unowned.size:
        view2d[torch.as_tensor(unowned, device=flat.device)] = nan
    row = w.N2 * w.D
    for b in range(w.B):
        ku = int(w.kv_used[b])
        if ku % PAGE:
            last = int(w.block_table[b, ku // PAGE])
            view2d[last, (ku % PAGE) * row:page_elems] = nan


def pool_view(w: Workload, flat):
    """[num_pages, 128, N2, D] strided view of a flat pool buffer."""
    return flat.as_strided((w.num_pages, PAGE, w.N2, w.D),
                           (w.kv_page_stride, w.N2 * w.D, w.D, 1))


def tnd_kv(w: Workload, kf, vf, pad_rows=None, seed=0):
    """The same logical keys and values in the non-paged TND layout: k, v of
    shape [T_kv, N2, D] with sequence b in rows [cu_kv[b], cu_kv[b+1]); its
    first seqused_kv[b] rows are the positions 0.. of the paged pool, the rest
    (``pad_rows`` per sequence, default U[0,40]) are NaN.  Returns
    (k, v, cu_kv int64 [B+1]) on the pool's device."""
    import torch

    rng = np.random.Generator(np.random.PCG64(seed + 4242))
    pads = (rng.integers(0, 41, size=w.B) if pad_rows is None
            else np.broadcast_to(np.asarray(pad_rows), (w.B,)))
    kp, vp = pool_view(w, kf), pool_view(w, vf)
    ks, vs, lens = [], [], []
    for b in range(w.B):
        ku = int(w.kv_used[b])
        pages = [int(w.block_table[b, lb]) for lb in range(-(-ku // PAGE))]
        for src, dst in ((kp, ks), (vp, vs)):
            rows = (torch.cat([src[pg] for pg in pages], 0)[:ku] if pages
                    else src.new_zeros((0, w.N2, w.D)))
            pad = src.new_full((int(pads[b]), w.N2, w.D), float("nan"))
            dst.append(torch.cat([rows, pad], 0))
        lens.append(ku + int(pads[b]))
    cu = np.zeros(w.B + 1, np.int64)
    cu[1:] = np.cumsum(lens)
    return torch.cat(ks, 0).contiguous(), torch.cat(vs, 0).contiguous(), cu


def bf16_bits(t) -> np.ndarray:
    """uint16 numpy copy of the bit patterns of a 16-bit (bf16 or fp16) torch
    tensor."""
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
