"""Work accounting for the benchmark: FLOPs and algorithmic bytes of one
forward pass over a Workload (host numpy; measurement only).

Definitions (what the benchmark reports):
* live block: a listed KV block inside the sequence's keys that some used
  query row of its Q block can see (causal, window) -- the blocks the
  kernels actually process;
* block-granular FLOPs (headline): sum over (Q block, KV head, live block) of
  4 * used_rows * G * keys_in_block * D  (QK^T and PV, 2 FLOPs per MAC);
* element-exact FLOPs: 4 * D * the number of visible (query row, head, key)
  triples, i.e. without the masked parts of partial blocks;
* algorithmic bytes: Q and O (used rows; 2 bytes per element, Q 1 byte for
  E4M3 inputs), LSE (fp32) if requested, 2 x 128 x D elements of K+V per live
  (Q block, KV head, block) -- 64 KiB for 16-bit types, 32 KiB for E4M3: what
  the method moves without cache reuse -- plus the index, count and
  block-table words.
"""
from __future__ import annotations

import numpy as np

from .workloads import PAGE, Workload


def _items(w: Workload):
    """Per item (qb-major, then KV head): used rows, pos0, ku and storage info."""
    bx = w.block_x
    qs = np.asarray(w.q_storage, np.int64)
    qu = np.asarray(w.q_used if w.has_seqused_q else w.q_storage, np.int64)
    ku = np.asarray(w.kv_used, np.int64)
    nqb = -(-qs // bx)
    b_of_qb = np.repeat(np.arange(w.B), nqb)
    qbl = np.arange(nqb.sum()) - np.repeat(np.cumsum(nqb) - nqb, nqb)
    n_store = np.minimum(bx, qs[b_of_qb] - qbl * bx)
    n_used = np.clip(qu[b_of_qb] - qbl * bx, 0, n_store)
    pos0 = qbl * bx + ku[b_of_qb] - qu[b_of_qb]
    return b_of_qb, n_used, pos0, ku[b_of_qb]


def work(w: Workload, exact: bool = True, in_bytes: int = 2) -> dict:
    """in_bytes: bytes per element of q, k and v (2, or 1 for E4M3); out is
    always 2 bytes per element."""
    b_of_qb, n_used, pos0, ku = _items(w)
    n = np.clip(w.sparse_count.astype(np.int64), 0, w.top_k)           # [N2, TQB]
    j = np.arange(w.top_k)[None, None, :]
    lb = w.sparse_idx.astype(np.int64)
    nblk = -(-ku // PAGE)
    sel = (j < n[:, :, None])
    inrange = sel & (lb >= 0) & (lb < nblk[None, :, None])
    k_lo = lb * PAGE
    k_hi = np.minimum(k_lo + PAGE - 1, ku[None, :, None] - 1)
    p_lo = pos0[None, :, None]
    p_hi = (pos0 + n_used - 1)[None, :, None]
    live = inrange & (n_used[None, :, None] > 0) & (k_lo <= p_hi)
    if w.win_left >= 0:
        live &= k_hi + w.win_left >= p_lo
    keys = np.where(live, k_hi - k_lo + 1, 0)
    G, D = w.G, w.D
    flops_block = float((4 * n_used[None, :, None] * G * keys * D).sum())
    n_live = int(live.sum())
    res = dict(flops_block=flops_block, live_blocks=n_live, selected_blocks=int(sel.sum()),
               kv_bytes=float(n_live) * 2 * PAGE * D * in_bytes)
    used_rows = int(n_used.sum())
    res["q_bytes"] = float(used_rows * w.N1 * D * in_bytes)
    res["o_bytes"] = float(used_rows * w.N1 * D * 2)
    res["lse_bytes"] = float(used_rows * w.N1 * 4) if w.return_lse else 0.0
    res["index_bytes"] = float(w.sparse_idx.nbytes + w.sparse_count.nbytes + w.block_table.nbytes)
    res["bytes"] = (res["q_bytes"] + res["o_bytes"] + res["lse_bytes"] + res["kv_bytes"] +
                    res["index_bytes"])
    if exact:
        res["flops_exact"] = _exact_flops(w, live, lb, pos0, n_used, ku)
    return res


def _exact_flops(w, live, lb, pos0, n_used, ku) -> float:
    """4*D*G * sum over live (item, block) of visible (row, key) pairs."""
    total = 0
    N2, TQB, K = live.shape
    max_rows = int(n_used.max()) if n_used.size else 0
    r = np.arange(max_rows)
    chunk = max(1, 4_000_000 // max(1, max_rows * K))
    for q0 in range(0, TQB, chunk):
        q1 = min(TQB, q0 + chunk)
        pos = pos0[q0:q1, None] + r[None, :]                               # [q, R]
        rowok = r[None, :] < n_used[q0:q1, None]
        k_lo = (lb[:, q0:q1, :] * PAGE)[..., None]                          # [N2, q, K, 1]
        k_hi = np.minimum(k_lo + PAGE - 1, ku[None, q0:q1, None, None] - 1)
        hi = np.minimum(k_hi, pos[None, :, None, :])
        lo = k_lo if w.win_left < 0 else np.maximum(k_lo, pos[None, :, None, :] - w.win_left)
        cnt = np.clip(hi - lo + 1, 0, None) * rowok[None, :, None, :]
        cnt = cnt * live[:, q0:q1, :, None]
        total += int(cnt.sum())
    return float(4 * w.D * w.G * total)


def row_flops(w: Workload, rows: np.ndarray) -> float:
    """Block-granular FLOPs of a sample of (token, head) rows: 4*D*keys of
    every live block of the row's Q block (same convention as flops_block)."""
    b_of_qb, n_used, pos0, ku = _items(w)
    qbase = np.concatenate([[0], np.cumsum(-(-np.asarray(w.q_storage, np.int64) // w.block_x))])
    cu = np.asarray(w.cu_seqlens_q, np.int64)
    b = np.searchsorted(cu, rows[:, 0], side="right") - 1
    t = rows[:, 0] - cu[b]
    qb = qbase[b] + t // w.block_x
    kvh = rows[:, 1] // w.G
    n = np.clip(w.sparse_count[kvh, qb].astype(np.int64), 0, w.top_k)
    lb = w.sparse_idx[kvh, qb].astype(np.int64)
    j = np.arange(w.top_k)[None, :]
    kuq = ku[qb][:, None]
    nblk = -(-kuq // PAGE)
    k_lo = lb * PAGE
    k_hi = np.minimum(k_lo + PAGE - 1, kuq - 1)
    p_lo = pos0[qb][:, None]
    p_hi = (pos0[qb] + n_used[qb] - 1)[:, None]
    live = (j < n[:, None]) & (lb >= 0) & (lb < nblk) & (n_used[qb][:, None] > 0) & (k_lo <= p_hi)
    if w.win_left >= 0:
        live &= k_hi + w.win_left >= p_lo
    t_in_block = t - (qb - qbase[b]) * w.block_x
    used = (t_in_block < n_used[qb])[:, None]
    keys = np.where(live & used, k_hi - k_lo + 1, 0)
    return float((4 * w.D * keys).sum())
