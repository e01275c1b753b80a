"""Sequential CPU rebuild of the GBSA work list (metadata buffer, format 1).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  The metadata kernels on
the GPU must produce exactly these int32 words for the same inputs; this file
is written from the format specification below, not from the CUDA code.

The GBSA article (cf-1.com/news/4865651), "two-phase call", gives the
metadata its role -- a load-balanced task split computed before the main
operator -- but not its content; the content below is this library's own.

Format 1 (int32 words)
----------------------
Header, 32 words:
   0 magic 0x41534247       1 version 1            2 signature (FNV-1a, below)
   3 B                      4 n_items=N2*TQB       5 tile_tokens
   6 tiles_max              7 num_ctas             8 unit_capacity
   9 slot_capacity         10 combine_capacity    11 n_units
  12 n_slots               13 n_combine           14 split_len
  15 status bits           16/17 total_cost lo/hi 18 off_seq
  19 off_item              20 off_list            21 off_unit
  22 off_combine           23 total_words         24 rows_per_unit
  25 G                     26..31 zero (26, 27: the forward's unit counters,
                                           back at zero after every call)
Sequence table (B x 8):   qs, qu, ku, n_qblocks, qblock_base, tok_begin, 0, 0
Item table (n_items x 8): b, n_live, n_tiles, tok_begin, n_store, n_used, pos0, ku
  item i = qb * N2 + kvh  (Q-block major, then KV head)
Live lists (n_items x top_k): lb | mask<<24 | partial<<25, list order kept,
  dead entries dropped, the rest of each row zero.
Units (unit_capacity x 4):  item, tp, j0 | j1<<16, slot (-1: not split),
  longest first (stable); only the first n_units rows are defined.
Combine (combine_capacity x 4): item, tp, first_slot, n_pieces; first n_combine.

Definitions
-----------
G = N1/N2; tile_tokens = min(128 // G, block_x) query tokens x G heads form
one 128-row tile; tiles_max = ceil(block_x / tile_tokens); a unit is a pair
of tiles (tp) of one item; rows_per_unit = min(2, tiles_max)*tile_tokens*G.
For item (qb, kvh) of sequence b, qbl = qb - qblock_base[b]:
  n_store = min(block_x, qs - qbl*block_x); n_used = clamp(qu - qbl*block_x,
  0, n_store); n_tiles = ceil(n_store / tile_tokens); pos0 = qbl*block_x + ku - qu.
Entry j < clamp(count, 0, top_k) with lb in [0, ceil(ku/128)) is live iff
  n_used > 0, 128*lb <= pos0 + n_used - 1 (causal), and, when win_left >= 0,
  min(128*lb + 127, ku - 1) + win_left >= pos0 (window);
  mask = not(128*lb + 128 <= ku and 128*lb + 127 <= pos0 and
             (win_left < 0 or 128*lb >= pos0 + n_used - 1 - win_left));
  partial = 128*lb + 128 > ku.
total_cost = sum_i ceil(n_tiles_i/2) * n_live_i;
split_len L = forced if max_blocks_per_split > 0 else max(8, ceil(total_cost / (4 P)));
a unit with n > L blocks becomes k = ceil(n/L) pieces [q*n//k, (q+1)*n//k).
"""
from __future__ import annotations

import numpy as np

MAGIC = 0x41534247
VERSION = 1
HEADER_WORDS = 32
PAGE = 128

DEV_BAD_SEQLEN = 0x01
DEV_BAD_BLOCK_IDX = 0x02
DEV_BAD_COUNT = 0x04
DEV_CAPACITY = 0x40


def _cdiv(a, b):
    return -(-a // b)


def _round4(x):
    return (x + 3) // 4 * 4


def fnv1a32(words) -> int:
    h = 0x811C9DC5
    for w in words:
        for byte in int(w & 0xFFFFFFFF).to_bytes(4, "little"):
            h ^= byte
            h = (h * 0x01000193) & 0xFFFFFFFF
    return h


def signature(p: dict) -> int:
    return fnv1a32([p["B"], p["N1"], p["N2"], p["D"], p["block_x"], p["total_q_blocks"],
                    p["top_k"], p.get("mask_mode", 1), p["win_left"], p["win_right"],
                    int(p["has_seqused_q"]), p["num_ctas"], p.get("max_blocks_per_split", 0)])


def geometry(p: dict) -> dict:
    G = p["N1"] // p["N2"]
    tile_tokens = min(128 // G, p["block_x"])
    tiles_max = _cdiv(p["block_x"], tile_tokens)
    n_items = p["N2"] * p["total_q_blocks"]
    units_max = n_items * _cdiv(tiles_max, 2)
    P = p["num_ctas"]
    forced = p.get("max_blocks_per_split", 0)
    if forced > 0:
        extra = _cdiv(units_max * p["top_k"], forced)
        unit_cap = units_max + extra
        slot_cap = 2 * extra
        comb_cap = min(units_max, extra)
    else:
        unit_cap = units_max + 4 * P
        slot_cap = 8 * P
        comb_cap = min(units_max, 4 * P)
    off_seq = HEADER_WORDS
    off_item = off_seq + 8 * p["B"]
    off_list = off_item + 8 * n_items
    off_unit = off_list + _round4(n_items * p["top_k"])
    off_comb = off_unit + 4 * unit_cap
    total = off_comb + 4 * comb_cap
    return dict(G=G, tile_tokens=tile_tokens, tiles_max=tiles_max, n_items=n_items,
                unit_cap=unit_cap, slot_cap=slot_cap, comb_cap=comb_cap, off_seq=off_seq,
                off_item=off_item, off_list=off_list, off_unit=off_unit, off_comb=off_comb,
                total=total, rows_per_unit=min(2, tiles_max) * tile_tokens * G)


def build(p: dict, sparse_idx, sparse_count, cu_seqlens_q, seqused_q, seqused_kv) -> np.ndarray:
    """Returns the metadata words (int32) for problem ``p`` and these inputs.

    ``p`` holds the host-known problem fields (B, T, N1, N2, D, block_x,
    total_q_blocks, top_k, win_left, win_right, has_seqused_q, num_ctas,
    max_blocks_per_split).
    """
    g = geometry(p)
    B, N2, top_k, bx = p["B"], p["N2"], p["top_k"], p["block_x"]
    tqb = p["total_q_blocks"]
    wl = p["win_left"]
    idx = np.asarray(sparse_idx, np.int64).reshape(N2, tqb, top_k)
    cnt = np.asarray(sparse_count, np.int64).reshape(N2, tqb)
    cu = [int(x) for x in np.asarray(cu_seqlens_q, np.int64)]
    ku_all = [int(x) for x in np.asarray(seqused_kv, np.int64)]
    words = np.zeros(g["total"], np.int64)
    status = 0

    # -- sequence table ---------------------------------------------------
    seq = []
    base = 0
    for b in range(B):
        qs = cu[b + 1] - cu[b]
        qu = int(seqused_q[b]) if p["has_seqused_q"] else qs
        ku = ku_all[b]
        if qs < 0 or qu < 0 or qu > qs or ku < 0:
            status |= DEV_BAD_SEQLEN
        nqb = _cdiv(max(qs, 0), bx)
        seq.append((qs, qu, ku, nqb, base, cu[b]))
        words[g["off_seq"] + 8 * b: g["off_seq"] + 8 * b + 6] = (qs, qu, ku, nqb, base, cu[b])
        base += nqb
    if cu[0] != 0 or cu[B] != p["T"] or base != tqb:
        status |= DEV_BAD_SEQLEN

    # -- items and live lists ----------------------------------------------
    n_items = g["n_items"]
    n_live = [0] * n_items
    n_tiles = [0] * n_items
    for qb in range(tqb):
        # the sequence holding Q block qb: the last b with a block starting at or before qb
        b = 0
        for bb in range(B):
            if seq[bb][3] > 0 and seq[bb][4] <= qb:
                b = bb
        qs, qu, ku, nqb, qbase, tok0 = seq[b]
        qbl = qb - qbase
        n_store = min(bx, qs - qbl * bx)
        n_used = min(max(qu - qbl * bx, 0), n_store)
        tiles = _cdiv(n_store, g["tile_tokens"])
        pos0 = qbl * bx + ku - qu
        nblk = _cdiv(ku, PAGE)
        p_hi = pos0 + n_used - 1
        for kvh in range(N2):
            i = qb * N2 + kvh
            c = int(cnt[kvh, qb])
            if c < 0 or c > top_k:
                status |= DEV_BAD_COUNT
                c = min(max(c, 0), top_k)
            live = []
            for j in range(c):
                lb = int(idx[kvh, qb, j])
                if lb < 0 or lb >= nblk:
                    status |= DEV_BAD_BLOCK_IDX
                    continue
                if n_used <= 0:
                    continue
                k_lo = PAGE * lb
                k_hi = min(PAGE * lb + PAGE - 1, ku - 1)
                if k_lo > p_hi:
                    continue
                if wl >= 0 and k_hi + wl < pos0:
                    continue
                full = (PAGE * lb + PAGE <= ku and PAGE * lb + PAGE - 1 <= pos0
                        and (wl < 0 or PAGE * lb >= p_hi - wl))
                partial = PAGE * lb + PAGE > ku
                live.append(lb | ((0 if full else 1) << 24) | ((1 if partial else 0) << 25))
            n_live[i] = len(live)
            n_tiles[i] = tiles
            o = g["off_item"] + 8 * i
            words[o:o + 8] = (b, len(live), tiles, tok0 + qbl * bx, n_store, n_used, pos0, ku)
            o = g["off_list"] + top_k * i
            words[o:o + len(live)] = live

    # -- plan: units, split-KV pieces, longest-first order ------------------
    P = p["num_ctas"]
    forced = p.get("max_blocks_per_split", 0)
    pieces, combine = [], []
    total_cost, L = 0, 0
    n_slots = 0
    if not status & DEV_BAD_SEQLEN:
        total_cost = sum(_cdiv(n_tiles[i], 2) * n_live[i] for i in range(n_items))
        L = forced if forced > 0 else max(8, _cdiv(total_cost, 4 * P))
        for i in range(n_items):
            n = n_live[i]
            k = 1 if n <= L else _cdiv(n, L)
            for tp in range(_cdiv(n_tiles[i], 2)):
                if k > 1:
                    combine.append((i, tp, n_slots, k))
                for q in range(k):
                    j0, j1 = q * n // k, (q + 1) * n // k
                    slot = n_slots if k > 1 else -1
                    if k > 1:
                        n_slots += 1
                    pieces.append((i, tp, j0, j1, slot))
        if len(pieces) > g["unit_cap"] or n_slots > g["slot_cap"] or len(combine) > g["comb_cap"]:
            status |= DEV_CAPACITY
    if status & (DEV_BAD_SEQLEN | DEV_CAPACITY):
        pieces, combine, n_slots = [], [], 0
        if status & DEV_BAD_SEQLEN:
            total_cost, L = 0, 0
    order = sorted(range(len(pieces)), key=lambda u: (-(pieces[u][3] - pieces[u][2]), u))
    for r, u in enumerate(order):
        i, tp, j0, j1, slot = pieces[u]
        o = g["off_unit"] + 4 * r
        words[o:o + 4] = (i, tp, j0 | (j1 << 16), slot)
    for r, rec in enumerate(combine):
        o = g["off_comb"] + 4 * r
        words[o:o + 4] = rec

    hdr = [MAGIC, VERSION, signature(p), B, n_items, g["tile_tokens"], g["tiles_max"], P,
           g["unit_cap"], g["slot_cap"], g["comb_cap"], len(pieces), n_slots, len(combine), L,
           status, total_cost & 0xFFFFFFFF, (total_cost >> 32) & 0xFFFFFFFF, g["off_seq"],
           g["off_item"], g["off_list"], g["off_unit"], g["off_comb"], g["total"],
           g["rows_per_unit"], g["G"]]
    words[:len(hdr)] = hdr
    return (words & 0xFFFFFFFF).astype(np.uint32).view(np.int32)


def defined_mask(words: np.ndarray) -> np.ndarray:
    """Boolean mask of the words the format defines for this buffer (the unit
    and combine tables are defined only up to n_units / n_combine rows)."""
    w = np.asarray(words).view(np.int32)
    m = np.ones(w.size, bool)
    off_unit, off_comb, total = int(w[21]), int(w[22]), int(w[23])
    m[total:] = False
    m[off_unit + 4 * int(w[11]):off_comb] = False
    m[off_comb + 4 * int(w[13]):total] = False
    return m
