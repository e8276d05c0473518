"""The roofline numerators (metrics.py) against counts worked out by hand on
tiny indexes: a wrong term here would misstate every roofline fraction."""
import torch

from hierarchical_long_context_b200 import api, metrics


def _params(**kw):
    base = dict(B=1, Hq=1, Hkv=1, d=64, Tmax=768, dtype=torch.float32, clusters=2, window=256, sinks=1,
                top_groups=2, top_pages=2)
    base.update(kw)
    return api.Params(**base)


def _index(p):
    """Chunks 0 and 1 indexed: chunk 0 has groups of 100 and 155 keys (one sink
    left out), chunk 1 groups of 200 and 56; pages of 16, the last one partial."""
    ix = api.Index(p, device="cpu")
    k, P = p.clusters, p.page_slots
    for c, sizes in ((0, (100, 155)), (1, (200, 56))):
        first = 0
        ix.gPage[0, 0, c * (k + 1)] = 0
        for j, n in enumerate(sizes):
            ix.gCnt[0, 0, c * k + j] = n
            npg = (n + 15) // 16
            for s in range(npg):
                ix.pCnt[0, 0, c * P + first + s] = min(16, n - 16 * s)
            first += npg
            ix.gPage[0, 0, c * (k + 1) + j + 1] = first
    return ix


def test_decode_touched_bytes_by_hand():
    p = _params()
    ix = _index(p)
    # query at t = 767: window = chunk 2 (256 tokens), groups of chunks 0-1
    # visible, 1 sink; opened: groups 0 (chunk 0) and 2 (chunk 1), pages
    # 1 and 3 of group 0 (16 keys each), pages 0 and 12 of group 2 (16 and 8)
    seq = torch.tensor([768])
    sg = torch.tensor([[[0, 2]]], dtype=torch.int32)
    sp = torch.tensor([[[[1, 3], [18, 30]]]], dtype=torch.int32)
    row = 64 * 4
    expect = 2 * row                           # q and out
    expect += 4 * 2 * row + 4 * 4              # 4 visible groups: mean K, mean V; 4 counts
    expect += (256 + 1) * 2 * row              # window and one sink
    expect += 4 + 7 * (row + 6) + 5 * row      # group 0: page range, 7 page keys + counts/offsets, 5 closed values
    expect += 4 + 13 * (row + 6) + 11 * row    # group 2: 13 pages, 11 closed
    expect += (16 + 16 + 16 + 8) * 2 * row     # opened members' K and V
    assert metrics.decode_touched_bytes(p, ix, seq, sg, sp) == expect == 172176


def test_decode_touched_bytes_int4_and_two_tier_by_hand():
    ix = _index(_params())
    seq = torch.tensor([768])
    sg = torch.tensor([[[0, 2]]], dtype=torch.int32)
    sp = torch.tensor([[[[1, 3], [18, 30]]]], dtype=torch.int32)
    row = 64 * 4
    common = 2 * row + 4 * 2 * row + 4 * 4 + 257 * 2 * row
    pages = 4 + 7 * (row + 6) + 5 * row + 4 + 13 * (row + 6) + 11 * row
    # three-tier INT4: each opened member is 32 + 32 bytes of codes; each
    # opened page adds (scale, low) pairs for K and V (2 x 64 x 8 bytes)
    p4 = _params(kv_bits=4)
    ix4 = _index(p4)
    got = metrics.decode_touched_bytes(p4, ix4, seq, sg, sp)
    assert got == common + pages + 56 * 2 * 32 + 4 * 2 * 64 * 8
    # two-tier: the opened groups are read whole (100 + 200 members), no page tier
    p2 = _params(top_pages=0)
    ix2 = _index(p2)
    got = metrics.decode_touched_bytes(p2, ix2, seq, sg, torch.zeros(1, 1, 2, 0, dtype=torch.int32))
    assert got == common + 2 * (2 * 2 + 2) + (100 + 200) * 2 * row


def test_build_bytes_by_hand():
    p = _params()
    per_chunk = (2 * 256 * 64 * 4        # read K and V
                 + 2 * 2 * 64 * 4        # group mean K and V
                 + 2 * 4                 # group counts
                 + 2 * 18 * 64 * 4       # page mean K and V (18 slots)
                 + 18 * (4 + 2)          # page counts and offsets
                 + 3 * 2                 # group page ranges
                 + 256 * 2)              # member list
    assert metrics.build_bytes(p, 2) == 2 * per_chunk == 283892
    copies = 2 * (2 * 256 - 1) * 64 * 4  # member-ordered K and V, sinks excluded
    words = 2 * 2 * 4                    # packed group words (2 chunks x 2 groups)
    assert metrics.build_design_bytes(p, 2) == copies + words == 261648
    # three-tier INT4: 32 + 32 bytes of codes per token, (scale, low) per slot and channel
    p4 = _params(kv_bits=4)
    assert metrics.build_design_bytes(p4, 2) == 2 * 511 * 32 + 2 * 2 * 18 * 64 * 8 + words
