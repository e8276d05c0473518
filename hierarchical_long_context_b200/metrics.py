"""Algorithmic byte and flop counts of the LoD hot path (host-side, no GPU work).

These are the numerators of the roofline fractions: the unique bytes a step
must move, counted from the selections the step actually made, not the bytes
an implementation happens to move.

Decode, per (sequence b, KV head) and for its g query heads at position t:
  * every visible, non-empty group summary: mean key + mean value + count;
  * the window [ws, t] and the sinks: one K row and one V row per token;
  * for the union of the opened groups: every page mean key, the page mean
    values of pages left unopened by some head, page counts/offsets and the
    group's page range;
  * the K and V rows of the union of opened pages' members (read from the
    member-ordered copies, one contiguous run per page);
  * the queries and outputs.
"""
from __future__ import annotations

import numpy as np


def decode_touched_bytes(p, index, seq_lens, sel_groups, sel_pages) -> int:
    """Unique bytes touched by one lod_decode call (all arguments on host or
    device; index is an api.Index).  sel_* are that call's selections."""
    e = 4 if str(p.dtype).endswith("float32") else 2
    d, k, P, C = p.d, p.clusters, p.page_slots, p.chunk
    row = d * e
    seq_lens = np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens)
    sg = np.asarray(sel_groups.cpu())
    sp = np.asarray(sel_pages.cpu())
    gCnt = index.gCnt.cpu().numpy()
    pCnt = index.pCnt.cpu().numpy()
    gPage = index.gPage.cpu().numpy().astype(np.int64)
    total = 2 * p.B * p.Hq * row  # q and out
    nw = p.window // C
    for b in range(p.B):
        t = int(seq_lens[b]) - 1
        bt = t // C
        wb = max(0, bt - nw + 1)
        ws = wb * C
        ns = min(p.sinks, ws)
        for h in range(p.Hkv):
            gc = gCnt[b, h, :wb * k]
            total += int((gc > 0).sum()) * 2 * row + gc.size * 4
            total += ((t - ws + 1) + ns) * 2 * row
            heads = range(h * p.g, (h + 1) * p.g)
            groups = set(int(x) for hq in heads for x in sg[b, hq] if x >= 0)
            if p.top_pages == 0:  # two-tier: every opened group read whole, no page tier
                for gid in groups:
                    total += 2 * 2 + 2 + int(gCnt[b, h, gid]) * 2 * row  # page range, first offset, K and V
                continue
            opened = set(int(x) for hq in heads for x in sp[b, hq].ravel() if x >= 0)
            for gid in groups:
                c, j = divmod(gid, k)
                p0, p1 = gPage[b, h, c * (k + 1) + j], gPage[b, h, c * (k + 1) + j + 1]
                total += 2 * 2  # page range
                for s in range(p0, p1):
                    pid = c * P + s
                    total += row + 4 + 2  # page mean key, count, offset
                    # a page mean value is read by every head that leaves it unopened
                    closed_by_some = any(
                        gid in set(sg[b, hq].tolist()) and pid not in set(sp[b, hq].ravel().tolist())
                        for hq in heads)
                    if closed_by_some:
                        total += row
            for pid in opened:
                n = int(pCnt[b, h, pid])
                if p.kv_bits == 4:  # three-tier INT4: K and V codes + (scale, low) quantisers
                    total += n * 2 * (d // 2) + 2 * d * 8
                else:
                    total += n * 2 * row  # K and V rows (one contiguous run per page)
    return total


def decode_flops(p, seq_lens) -> float:
    """Multiply-adds x2 of one decode call: scores and weighted values of every
    visible group and window/sink token per query head (page and exact terms
    of the opened groups are added at 16 * top_groups * (2 + top_pages) rows)."""
    C, k = p.chunk, p.clusters
    nw = p.window // C
    f = 0.0
    for L in np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens):
        t = int(L) - 1
        wb = max(0, t // C - nw + 1)
        rows = wb * k + (t - wb * C + 1) + min(p.sinks, wb * C) + p.top_groups * (4 + 16 * p.top_pages)
        f += 4.0 * p.d * rows * p.Hq
    return f


def prefill_flops(p, q_begin: int, Tq: int) -> float:
    """Algorithmic flops of lod_prefill on [q_begin, q_begin + Tq): per query row,
    2d per score and 2d per weighted value over the visible groups, the window
    and sinks, and the opened groups' pages (mean keys, unopened mean values)
    and opened tokens (expected page counts: all pages of a k=4 group average
    4.5 of which top_pages are opened)."""
    C, k = p.chunk, p.clusters
    nw = p.window // C
    f = 0.0
    for t in range(q_begin, q_begin + Tq):
        wb = max(0, t // C - nw + 1)
        ws = wb * C
        rows = wb * k + (t - ws + 1) + min(p.sinks, ws)
        if wb * k > 0:
            g = min(p.top_groups, wb * k)
            rows += g * (4.5 + (4.5 - p.top_pages) + 16 * p.top_pages)
        f += 4.0 * p.d * rows
    return f * p.B * p.Hq


def build_bytes(p, nchunks: int) -> int:
    """Algorithmic bytes of one lod_build_index call over chunks [0, nchunks)
    of every sequence: the method's own reads and writes -- K and V read
    once, the group and page summaries, counts, page offsets, group page
    ranges and the member list written once."""
    e = 4 if str(p.dtype).endswith("float32") else 2
    units = p.B * p.Hkv
    k, P, C, d = p.clusters, p.page_slots, p.chunk, p.d
    per_chunk = 2 * C * d * e + 2 * k * d * e + k * 4 + 2 * P * d * e + P * (4 + 2) + (k + 1) * 2 + C * 2
    return units * nchunks * per_chunk


def build_design_bytes(p, nchunks: int) -> int:
    """Bytes the build writes beyond the method's own: the member-ordered K/V
    copies (every clustered token once, cache dtype; with kv_bits = 4 the
    4-bit codes and the per-page (scale, low) quantisers instead) and the
    packed group words.  These serve the decode's contiguous page reads."""
    e = 4 if str(p.dtype).endswith("float32") else 2
    units = p.B * p.Hkv
    k, P, C, d = p.clusters, p.page_slots, p.chunk, p.d
    toks = nchunks * C - (p.sinks if nchunks else 0)
    if p.kv_bits == 4:
        copies = 2 * toks * (d // 2) + 2 * nchunks * P * d * 8
    else:
        copies = 2 * toks * d * e
    return units * (copies + nchunks * k * 4)


def build_flops(p, nchunks: int) -> float:
    """Lloyd work of the build at the configured rounds: 2 flops per (key,
    centroid, dimension) per round, plus the initialisation and the sums."""
    C, k, d = p.chunk, p.clusters, p.d
    per = 2.0 * C * k * d * p.kmeans_iters + 3.0 * C * k * d + 2.0 * C * d * 2
    return p.B * p.Hkv * nchunks * per
