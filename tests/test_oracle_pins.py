"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test ties one part of the oracle to something it cannot restate: a
published generator output, a library rounding routine, a textbook Lloyd
implementation, a closed form (dense attention) that the method must reduce
to, or an invariant the method's description implies ("Level of Detail
Attention", How It Works).  The combination is chosen so that a dropped term
(ln count), a wrong index (page members, window bounds), a wrong sign or a
transposed operand fails at least one of them.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from hierarchical_long_context_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden_hex(name):
    vals = []
    for line in open(os.path.join(HERE, "golden", name)):
        line = line.strip()
        if line and not line.startswith("#"):
            vals.append(int(line, 16))
    return vals


# ---------------------------------------------------------------- primitives

def test_splitmix64_matches_published_outputs():
    gamma = 0x9E3779B97F4A7C15
    want = _golden_hex("splitmix64_state0.txt")
    got = [oracle.splitmix64((i * gamma) % 2**64) for i in range(len(want))]
    assert got == want


def test_round_bf16_matches_torch_rne():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-3, 3, 20000),
                        [1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 255.5, 3.0 / 7]]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------- k-means / index

def _cfg(w, **kw):
    base = dict(d=w.d, clusters=w.clusters[0], iters=w.iters, top_groups=w.top_groups,
                top_pages=w.top_pages, window=w.window, sinks=w.sinks,
                store_bf16=(w.dtype == "bf16"), seed=w.seed)
    base.update(kw)
    return oracle.Config(**base)


@pytest.fixture(scope="module")
def tiny():
    w = synth.WORKLOADS["decode_tiny_f32"]
    K, V = synth.unit_kv(w, 0, 0)
    cfg = _cfg(w)
    nch = w.T // 256
    idx = oracle.build_sequence(cfg, 0, K, V, nch, want_objective=True)
    return w, cfg, K, V, idx


@pytest.fixture(scope="module")
def tiny_bf16():
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=1, Hq=8, Hkv=1, T=2048)
    K, V = synth.unit_kv(w, 0, 0)
    cfg = _cfg(w)
    idx = oracle.build_sequence(cfg, 0, K, V, w.T // 256, want_objective=True)
    return w, cfg, K, V, idx


def _chunk_members(idx, cfg, c, j):
    C = cfg.chunk
    return np.nonzero(idx["assign"][c * C:(c + 1) * C] == j)[0]


@pytest.mark.parametrize("which", ["tiny", "tiny_bf16"])
def test_group_and_page_summaries_are_member_means(which, request):
    w, cfg, K, V, idx = request.getfixturevalue(which)
    C, k, P = cfg.chunk, cfg.clusters, cfg.page_slots
    rnd = (lambda a: oracle.round_bf16(a)) if cfg.store_bf16 else (lambda a: a.astype(np.float32).astype(np.float64))
    for c in range(idx["nchunks"]):
        seen = []
        for j in range(k):
            m = _chunk_members(idx, cfg, c, j)
            assert idx["gCnt"][c * k + j] == len(m)
            if len(m):
                np.testing.assert_array_equal(idx["gK"][c * k + j], rnd(K[c * C + m].astype(np.float64).mean(0)))
                np.testing.assert_array_equal(idx["gV"][c * k + j], rnd(V[c * C + m].astype(np.float64).mean(0)))
            # pages: ascending positions, runs of `page`, last one short
            p0, p1 = idx["gPage"][c * (k + 1) + j], idx["gPage"][c * (k + 1) + j + 1]
            assert p1 - p0 == -(-len(m) // cfg.page)
            pages = []
            for s in range(p0, p1):
                b, n = idx["pBeg"][c * P + s], idx["pCnt"][c * P + s]
                mem = idx["perm"][c * C + b:c * C + b + n]
                pages.append(mem)
                np.testing.assert_array_equal(idx["pK"][c * P + s], rnd(K[c * C + mem].astype(np.float64).mean(0)))
                np.testing.assert_array_equal(idx["pV"][c * P + s], rnd(V[c * C + mem].astype(np.float64).mean(0)))
            sizes = [len(x) for x in pages]
            assert all(s == cfg.page for s in sizes[:-1]) and (not sizes or 0 < sizes[-1] <= cfg.page)
            flat = np.concatenate(pages) if pages else np.zeros(0, int)
            np.testing.assert_array_equal(flat, m)          # page union = group, ascending
            seen.append(m)
        allm = np.sort(np.concatenate(seen))
        first = cfg.sinks if c == 0 else 0
        np.testing.assert_array_equal(allm, np.arange(first, C))  # groups partition the chunk minus sinks
        assert idx["gPage"][c * (k + 1) + k] <= C // cfg.page + k - 1
        assert np.all(idx["pCnt"][c * P + idx["gPage"][c * (k + 1) + k]:(c + 1) * P] == 0)


@pytest.mark.parametrize("which", ["tiny", "tiny_bf16"])
def test_lloyd_objective_never_increases(which, request):
    _, _, _, _, idx = request.getfixturevalue(which)
    obj = idx["objective"]
    assert np.all(np.diff(obj, axis=1) <= 1e-6 * obj[:, :-1])


def test_farthest_first_init_properties(tiny):
    w, cfg, K, V, idx = tiny
    C, k = cfg.chunk, cfg.clusters
    for c in range(idx["nchunks"]):
        first = cfg.sinks if c == 0 else 0
        X = K[c * C + first:(c + 1) * C].astype(np.float64)
        picks = idx["init_idx"][c * k:(c + 1) * k]
        assert picks[0] == oracle.splitmix64(cfg.seed ^ ((0 << 32) + c)) % len(X)
        assert len(set(map(tuple, X[picks]))) == k        # distinct keys exist, so picks are distinct
        for j in range(1, k):
            dmin = ((X[:, None, :] - X[picks[:j]][None]) ** 2).sum(-1).min(1)
            # the pick is a farthest point (brute force), up to fp32 rounding of the distances
            assert dmin[picks[j]] >= dmin.max() * (1 - 1e-5)


def test_lloyd_matches_sklearn_given_the_same_init(tiny):
    from sklearn.cluster import KMeans
    w, cfg, K, V, idx = tiny
    C, k = cfg.chunk, cfg.clusters
    compared = 0
    for c in range(idx["nchunks"]):
        # skip only chunks where some decision is within fp32-vs-fp64 noise
        if idx["min_margin"][c] <= 1e-6:
            continue
        first = cfg.sinks if c == 0 else 0
        X = K[c * C + first:(c + 1) * C].astype(np.float64)
        init = X[idx["init_idx"][c * k:(c + 1) * k]]
        # sklearn re-assigns once after its last update, so its labels after
        # iters-1 rounds are the oracle's last assignment; its centres after
        # `iters` rounds are the means of that assignment.
        lab = KMeans(k, init=init, n_init=1, max_iter=cfg.iters - 1, tol=0.0,
                     algorithm="lloyd").fit(X).labels_
        np.testing.assert_array_equal(lab, idx["assign"][c * C + first:(c + 1) * C])
        cen = KMeans(k, init=init, n_init=1, max_iter=cfg.iters, tol=0.0,
                     algorithm="lloyd").fit(X).cluster_centers_
        np.testing.assert_allclose(idx["gK"][c * k:(c + 1) * k], cen, rtol=0, atol=1e-6)
        compared += 1
    assert compared >= idx["nchunks"] - 2


# ---------------------------------------------------------------- attention

def _rows(w, n):
    rng = np.random.default_rng(7)
    return (rng.standard_normal((n, w.d)).astype(np.float32) / 8).astype(np.float32)


def test_zero_variance_groups_give_dense_attention():
    """Level of Detail Attention, How It Works: with zero-variance groups the
    method equals full attention."""
    w = synth.WORKLOADS["decode_tiny_f32_zero_variance"]
    K, V = synth.unit_kv(w, 0, 0)
    cfg = _cfg(w)
    idx = oracle.build_sequence(cfg, 0, K, V, w.T // 256)
    assert np.all(idx["min_margin"] > 1e-4)
    for q in _rows(w, 16):
        for t in (w.T - 1, 3000, 1023, 700):
            out, lse, sg, sp, st = oracle.attend_row(cfg, q, t, K, V, idx)
            dout, dlse = oracle.dense_row(cfg, q, t, K, V)
            if t >= 3000:   # enough visible groups for both kinds of coarse entries
                assert st["n_coarse_groups"] > 0 and st["n_coarse_pages"] > 0
            np.testing.assert_allclose(out, dout, rtol=0, atol=1e-10)
            assert abs(lse - dlse) < 1e-10


def test_everything_opened_gives_dense_attention(tiny):
    w, _, K, V, _ = tiny
    T = 1024
    cfg = _cfg(w, top_groups=64, top_pages=64)
    idx = oracle.build_sequence(cfg, 0, K[:T], V[:T], T // 256)
    for q in _rows(w, 8):
        for t in (T - 1, 900, 600):
            out, lse, sg, sp, st = oracle.attend_row(cfg, q, t, K, V, idx)
            dout, dlse = oracle.dense_row(cfg, q, t, K, V)
            assert st["n_coarse_groups"] == 0 and st["n_coarse_pages"] == 0
            assert st["n_exact"] == t + 1
            np.testing.assert_allclose(out, dout, rtol=0, atol=1e-12)


def test_two_tier_is_whole_group_attention_written_out(tiny):
    """Two-tier LoD (top_pages = 0): the opened groups' members are exact and
    no page tier exists.  Checked against the entry list written out here in
    numpy from the index arrays (window, sinks, whole opened groups exact,
    every other visible group as mean-key logit + ln n with its mean value)."""
    w, _, K, V, _ = tiny
    T = 2048
    cfg = _cfg(w, top_groups=3, top_pages=0)
    idx = oracle.build_sequence(cfg, 0, K[:T], V[:T], T // 256)
    k, C, sc = cfg.clusters, cfg.chunk, 1.0 / np.sqrt(cfg.d)
    Kd, Vd = K.astype(np.float64), V.astype(np.float64)
    for q in _rows(w, 6):
        for t in (T - 1, 1700, 1100):
            out, lse, sg, sp, st = oracle.attend_row(cfg, q, t, K, V, idx)
            assert sp.size == 0 and st["n_coarse_pages"] == 0
            ws = 256 * max(0, t // 256 - cfg.window // 256 + 1)
            qd = q.astype(np.float64)
            ids = [g for g in range((ws // C) * k) if idx["gCnt"][g] > 0]
            s32 = {g: float(np.float32(np.dot(q.astype(np.float32), idx["gK"][g].astype(np.float32)))
                            * np.float32(sc)) for g in ids}
            opened = sorted(ids, key=lambda g: (-s32[g], g))[:cfg.top_groups]
            assert list(sg[:len(opened)]) == opened
            lg, vals = [], []
            for pos in list(range(min(cfg.sinks, ws))) + list(range(ws, t + 1)):
                lg.append(sc * qd @ Kd[pos]); vals.append(Vd[pos])
            for g in ids:
                c, j = divmod(g, k)
                if g in opened:
                    off = int(np.sum(idx["gCnt"][c * k:c * k + j]))
                    for m in range(int(idx["gCnt"][g])):
                        pos = c * C + idx["perm"][c * C + off + m]
                        lg.append(sc * qd @ Kd[pos]); vals.append(Vd[pos])
                else:
                    lg.append(sc * qd @ idx["gK"][g] + np.log(idx["gCnt"][g])); vals.append(idx["gV"][g])
            lg = np.array(lg)
            wgt = np.exp(lg - lg.max())
            want = (wgt[:, None] * np.array(vals)).sum(0) / wgt.sum()
            np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)
            assert abs(lse - (lg.max() + np.log(wgt.sum()))) < 1e-12


def test_window_covering_everything_is_dense(tiny):
    w, cfg, K, V, idx = tiny
    for q in _rows(w, 4):
        for t in (0, 1, 100, 255):
            out, lse, *_ = oracle.attend_row(cfg, q, t, K, V, idx)
            dout, dlse = oracle.dense_row(cfg, q, t, K, V)
            np.testing.assert_allclose(out, dout, rtol=0, atol=1e-13)


@pytest.mark.parametrize("which", ["tiny", "tiny_bf16"])
def test_weights_sum_to_one_and_partition_covers_every_position(which, request):
    w, cfg, K, V, idx = request.getfixturevalue(which)
    T = idx["nchunks"] * 256
    for q in _rows(w, 6):
        for t in (T - 1, T - 200, 1500, 300, 256, 40):
            out, lse, sg, sp, st = oracle.attend_row(cfg, q, t, K, V, idx)
            assert abs(st["weight_sum"] - 1.0) < 1e-12
            assert st["covered"] == t + 1
            ws = st["window_start"]
            bt = t // 256
            assert ws == 256 * max(0, bt - cfg.window // 256 + 1)
            assert t + 1 - ws >= min(t + 1, cfg.window - 255)


def test_coarse_mass_is_conservative_jensen(tiny):
    """How It Works: with variance the coarse remainder is a conservative
    estimate of the attention mass, i.e. n exp(q.mean k) <= sum exp(q.k), so
    the LoD log-normaliser never exceeds the dense one (fp32 summaries)."""
    w, cfg, K, V, idx = tiny
    for q in _rows(w, 32) * 8:   # sharper logits make the gap visible
        out, lse, *_ = oracle.attend_row(cfg, q, w.T - 1, K, V, idx)
        _, dlse = oracle.dense_row(cfg, q, w.T - 1, K, V)
        assert lse <= dlse + 1e-6


@pytest.mark.parametrize("which", ["tiny", "tiny_bf16"])
def test_selection_is_the_enumerated_top_k(which, request):
    w, cfg, K, V, idx = request.getfixturevalue(which)
    k, P = cfg.clusters, cfg.page_slots
    sc = np.float32(1 / np.sqrt(w.d))
    t = idx["nchunks"] * 256 - 1
    nvis = t // 256 - cfg.window // 256 + 1
    for q in _rows(w, 12):
        out, lse, sg, sp, st = oracle.attend_row(cfg, q, t, K, V, idx)
        ids = [i for i in range(nvis * k) if idx["gCnt"][i] > 0]
        s = {i: float(np.dot(q.astype(np.float64), idx["gK"][i])) * sc for i in ids}
        opened = [g for g in sg if g >= 0]
        assert len(opened) == min(cfg.top_groups, len(ids)) and len(set(opened)) == len(opened)
        rest = [i for i in ids if i not in opened]
        for g in opened:
            for u in rest:
                assert s[g] > s[u] - 1e-5 and (s[g] != s[u] or g < u)
        assert all(s[a] >= s[b] - 1e-5 for a, b in zip(opened, opened[1:]))
        for r, g in enumerate(opened):
            c, j = divmod(g, k)
            slots = list(range(idx["gPage"][c * (k + 1) + j], idx["gPage"][c * (k + 1) + j + 1]))
            ps = {sl: float(np.dot(q.astype(np.float64), idx["pK"][c * P + sl])) * sc for sl in slots}
            op = [x - c * P for x in sp[r] if x >= 0]
            assert len(op) == min(cfg.top_pages, len(slots))
            for a in op:
                for b in set(slots) - set(op):
                    assert ps[a] > ps[b] - 1e-5


def test_ties_go_to_the_lower_group_id(tiny):
    """Two groups with bit-identical summaries: the lower global id wins."""
    w, cfg, K, V, idx = tiny
    idx = {k_: (v.copy() if isinstance(v, np.ndarray) else v) for k_, v in idx.items()}
    k = cfg.clusters
    q = _rows(w, 1)[0]
    t = w.T - 1
    _, _, sg, _, _ = oracle.attend_row(cfg, q, t, K, V, idx)
    best = sg[0]
    twin = 0 if best != 0 else 1           # copy the winner's summary into a lower/higher id
    idx["gK"][twin] = idx["gK"][best]
    _, _, sg2, _, _ = oracle.attend_row(cfg, q, t, K, V, idx)
    assert sg2[0] == min(twin, best) and sg2[1] == max(twin, best)


def test_forced_selection_reproduces_free_selection(tiny_bf16):
    w, cfg, K, V, idx = tiny_bf16
    t = idx["nchunks"] * 256 - 1
    for q in _rows(w, 4):
        out, lse, sg, sp, _ = oracle.attend_row(cfg, q, t, K, V, idx)
        out2, lse2, sg2, sp2, _ = oracle.attend_row(cfg, q, t, K, V, idx, sg, sp)
        np.testing.assert_allclose(out, out2, rtol=0, atol=1e-13)   # entry order differs
        np.testing.assert_array_equal(sg, sg2)


# ---------------------------------------------------------------- three-tier INT4

def _page_members(idx, cfg, pid):
    """(chunk, member-order rows, token offsets) of page slot `pid`."""
    C, P = cfg.chunk, cfg.page_slots
    c, b0, m = pid // P, idx["pBeg"][pid], idx["pCnt"][pid]
    rows = c * C + b0 + np.arange(m)
    return c, rows, c * C + idx["perm"][c * C + b0 + np.arange(m)]


def _fused(qz, rows, pid):
    """code * scale + low with one rounding to fp32 (the product of a 4-bit
    code and an fp32 scale, plus an fp32 low, is exact in fp64)."""
    return (qz["code"][rows].astype(np.float64) * qz["scale"][pid].astype(np.float64)
            + qz["low"][pid].astype(np.float64)).astype(np.float32)


@pytest.mark.parametrize("which", ["tiny", "tiny_bf16"])
def test_int4_codes_are_nearest_grid_points(which, request):
    """Three-tier INT4 reading: per page and channel the grid is low + c *
    scale, c = 0..15, low = min and low + 15 scale = max over the page's
    members; every member gets a nearest grid point.  Checked by enumerating
    all 16 grid points in fp64, independently of the oracle's rounding."""
    w, cfg, K, V, idx = request.getfixturevalue(which)
    for X in (K, V):
        X = np.asarray(X, np.float32)
        qz = oracle.quantize_pages(cfg, X, idx)
        assert qz["code"].max() <= 15
        used = np.nonzero(idx["pCnt"] > 0)[0]
        for pid in used[:: max(1, len(used) // 40)]:
            _, rows, toks = _page_members(idx, cfg, pid)
            x = X[toks].astype(np.float64)                       # [m, d]
            lo = qz["low"][pid].astype(np.float64)
            sc = qz["scale"][pid].astype(np.float64)
            np.testing.assert_array_equal(lo, x.min(0))
            np.testing.assert_allclose(lo + 15 * sc, x.max(0), rtol=1e-6, atol=1e-6)
            grid = lo[None, :] + np.arange(16)[:, None] * sc[None, :]    # [16, d]
            dist = np.abs(x[:, None, :] - grid[None, :, :])              # [m, 16, d]
            best = dist.min(1)
            got = np.take_along_axis(dist, qz["code"][rows].astype(np.int64)[:, None, :], 1)[:, 0]
            # the fp32 quotient may round a near-tie either way
            assert np.all(got <= best + 1e-6 * (np.abs(x) + 15 * sc[None, :]) + 1e-12)
            # round trip within half a step
            xh = (qz["code"][rows].astype(np.float32) * qz["scale"][pid] + qz["low"][pid]).astype(np.float64)
            assert np.all(np.abs(xh - x) <= sc[None, :] / 2 * (1 + 1e-5) + 1e-7 * np.abs(x) + 1e-12)


def test_int4_constant_pages_decompress_exactly():
    """A page whose members are equal in a channel has scale 0, code 0 and
    decompresses to the value itself: on the zero-variance cache every page
    is constant, so three-tier INT4 equals the cache-value path and dense
    attention (How It Works, zero-variance paragraph)."""
    w = synth.WORKLOADS["decode_tiny_f32_zero_variance"]
    K, V = synth.unit_kv(w, 0, 0)
    cfg = _cfg(w)
    idx = oracle.build_sequence(cfg, 0, K, V, w.T // 256)
    kq, vq = oracle.quantize_pages(cfg, K, idx), oracle.quantize_pages(cfg, V, idx)
    used = idx["pCnt"] > 0
    assert np.all(kq["scale"][used] == 0) and np.all(vq["scale"][used] == 0)
    assert np.all(kq["code"] == 0) and np.all(vq["code"] == 0)
    for q in _rows(w, 6):
        for t in (w.T - 1, 3000):
            o4, l4, sg4, sp4, _ = oracle.attend_row(cfg, q, t, K, V, idx, kq=kq, vq=vq)
            o, l, sg, sp, _ = oracle.attend_row(cfg, q, t, K, V, idx)
            np.testing.assert_array_equal(o4, o)
            assert l4 == l and np.array_equal(sg4, sg) and np.array_equal(sp4, sp)
            dout, dlse = oracle.dense_row(cfg, q, t, K, V)
            np.testing.assert_allclose(o4, dout, rtol=0, atol=1e-10)


def test_int4_everything_opened_is_dense_over_the_decompressed_cache(tiny_bf16):
    """With every group and page opened, three-tier INT4 attention is full
    attention over the cache in which each indexed position holds its
    decompressed key and value (sinks and window keep the cache values):
    the decompression is applied to exactly the opened members."""
    w, _, K, V, _ = tiny_bf16
    K = np.asarray(K, np.float32); V = np.asarray(V, np.float32)
    cfg = _cfg(w, top_groups=64, top_pages=64)
    T = 1536
    idx = oracle.build_sequence(cfg, 0, K[:T], V[:T], T // 256)
    kq, vq = oracle.quantize_pages(cfg, K[:T], idx), oracle.quantize_pages(cfg, V[:T], idx)
    P = cfg.page_slots
    for q in _rows(w, 4):
        for t in (T - 1, 1300):
            nvis = t // 256 - cfg.window // 256 + 1
            Kh, Vh = K[:t + 1].copy(), V[:t + 1].copy()
            for pid in range(nvis * P):
                if idx["pCnt"][pid] <= 0:
                    continue
                _, rows, toks = _page_members(idx, cfg, pid)
                Kh[toks] = _fused(kq, rows, pid)
                Vh[toks] = _fused(vq, rows, pid)
            out, lse, _, _, st = oracle.attend_row(cfg, q, t, K, V, idx, kq=kq, vq=vq)
            assert st["n_coarse_groups"] == 0 and st["n_coarse_pages"] == 0
            dout, dlse = oracle.dense_row(cfg, q, t, Kh, Vh)
            np.testing.assert_allclose(out, dout, rtol=0, atol=1e-9)
            assert abs(lse - dlse) < 1e-9
