"""Helpers shared by the GPU parity tests: parameter mapping, index transfer
between the CUDA layout and the oracle's arrays, and the comparison rules.

Comparison rules (tolerances fixed for the method's parity):
  * outputs: max-abs 1e-3 for fp32 caches, 2e-2 for bf16 caches;
  * top-k selections identical, except that a GPU selection differing from
    the oracle's is accepted when every swapped pair's oracle scores lie
    within 1e-3 (scaled logits); the output is then compared with the oracle
    re-run on the GPU's selection;
  * k-means assignments identical for every key whose best-vs-second margin
    exceeds 1e-4 relative; a chunk in which some earlier decision had a
    margin <= 1e-4 may diverge as a whole (an early flip cascades) and is
    then only checked for internal consistency, while attention is checked
    on the GPU-built index.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from hierarchical_long_context_b200 import api, synth

TOL = {"f32": 1e-3, "bf16": 2e-2}
TIE = 1e-3
MARGIN = 1e-4


def oracle_cfg(w: synth.Workload, k: int | None = None, **kw) -> oracle.Config:
    base = dict(d=w.d, clusters=k or w.clusters[0], iters=w.iters, top_groups=w.top_groups,
                top_pages=w.top_pages, window=w.window, sinks=w.sinks,
                store_bf16=(w.dtype == "bf16"), seed=w.seed)
    base.update(kw)
    return oracle.Config(**base)


def params_of(w: synth.Workload, k: int | None = None, Tmax: int | None = None, **kw) -> api.Params:
    T = Tmax or ((w.T + 255) // 256) * 256
    base = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, Tmax=T, dtype=w.torch_dtype,
                clusters=k or w.clusters[0], kmeans_iters=w.iters, top_groups=w.top_groups,
                top_pages=w.top_pages, window=w.window, sinks=w.sinks, seed=w.seed)
    base.update(kw)
    return api.Params(**base)


def unit_from_gpu(ix: api.Index, b: int, h: int, nchunks: int, p: api.Params) -> dict:
    """One (b, kvh) sequence of a GPU index, in the oracle's array layout."""
    k, P, C = p.clusters, p.page_slots, p.chunk
    f = lambda t, n: t[b, h, :n].float().cpu().numpy().astype(np.float64)
    i = lambda t, n: t[b, h, :n].cpu().numpy().astype(np.int32)
    return dict(gK=f(ix.gK, nchunks * k), gV=f(ix.gV, nchunks * k), gCnt=i(ix.gCnt, nchunks * k),
                pK=f(ix.pK, nchunks * P), pV=f(ix.pV, nchunks * P), pCnt=i(ix.pCnt, nchunks * P),
                pBeg=i(ix.pBeg, nchunks * P), gPage=i(ix.gPage, nchunks * (k + 1)),
                perm=i(ix.perm, nchunks * C), gMeta=i(ix.gMeta, nchunks * k), nchunks=nchunks)


def pack_meta(u: dict, k: int) -> np.ndarray:
    """gMeta of an index in the oracle's layout: size | first page << 16 | end page << 24."""
    n = u["nchunks"]
    gp = np.asarray(u["gPage"][:n * (k + 1)], dtype=np.int64).reshape(n, k + 1)
    cnt = np.asarray(u["gCnt"][:n * k], dtype=np.int64).reshape(n, k)
    return (cnt | (gp[:, :k] << 16) | (gp[:, 1:] << 24)).reshape(-1).astype(np.int32)


def pack_codes(code: np.ndarray) -> np.ndarray:
    """[rows, d] 4-bit codes -> [rows, d/2] bytes (channel 2i in the low nibble)."""
    code = np.asarray(code, np.uint8)
    return (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes."""
    packed = np.asarray(packed, np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), np.uint8)
    out[:, 0::2] = packed & 15
    out[:, 1::2] = packed >> 4
    return out


def quantized(u: dict, K: np.ndarray, V: np.ndarray, cfg: oracle.Config) -> dict:
    """u with the oracle's three-tier INT4 pages of K and V added (kq, vq)."""
    return dict(u, kq=oracle.quantize_pages(cfg, K, u), vq=oracle.quantize_pages(cfg, V, u))


def check_int4_pages(ix: api.Index, b: int, h: int, u: dict, K: np.ndarray, V: np.ndarray,
                     cfg: oracle.Config) -> int:
    """The GPU's INT4 codes and (scale, low) quantisers equal the oracle's
    quantiser applied to the GPU-built index, bit for bit (every member row,
    every used page slot).  Returns the number of member rows compared."""
    n, C, P = u["nchunks"], cfg.chunk, cfg.page_slots
    used = u["pCnt"][:n * P] > 0
    members = u["perm"][:n * C] >= 0
    for X, codes, qs in ((K, ix.qK, ix.qKs), (V, ix.qV, ix.qVs)):
        oq = oracle.quantize_pages(cfg, X, u)
        gq = qs[b, h, :n * P].cpu().numpy()
        np.testing.assert_array_equal(gq[used][..., 0], oq["scale"][used])
        np.testing.assert_array_equal(gq[used][..., 1], oq["low"][used])
        gc = unpack_codes(codes[b, h, :n * C].cpu().numpy())
        np.testing.assert_array_equal(gc[members], oq["code"][members])
    return int(members.sum())


def unit_to_gpu(ix: api.Index, b: int, h: int, u: dict, p: api.Params, K=None, V=None) -> None:
    """Write an oracle-built index of one sequence into a GPU index.  K, V
    (that sequence's cache rows, [T][d] tensors) fill the member-ordered
    copies: row m of chunk c is the token at offset perm[m]; with
    p.kv_bits = 4, u's INT4 pages (kq, vq of `quantized`) fill the codes."""
    n = u["nchunks"]
    k, P, C = p.clusters, p.page_slots, p.chunk
    dev = ix.gK.device
    put = lambda t, a, m: t[b, h, :m].copy_(torch.from_numpy(np.ascontiguousarray(a)).to(t.dtype).to(dev))
    put(ix.gK, u["gK"], n * k)
    put(ix.gV, u["gV"], n * k)
    put(ix.gCnt, u["gCnt"], n * k)
    put(ix.pK, u["pK"], n * P)
    put(ix.pV, u["pV"], n * P)
    put(ix.pCnt, u["pCnt"], n * P)
    put(ix.pBeg, u["pBeg"], n * P)
    put(ix.gPage, u["gPage"], n * (k + 1))
    put(ix.perm, u["perm"], n * C)
    put(ix.gMeta, pack_meta(u, k), n * k)
    if p.kv_bits == 4:
        for key, codes, qs in (("kq", ix.qK, ix.qKs), ("vq", ix.qV, ix.qVs)):
            q = u[key]
            codes[b, h, :n * C].copy_(torch.from_numpy(pack_codes(q["code"][:n * C])).to(dev))
            sl = np.stack([q["scale"][:n * P], q["low"][:n * P]], -1).astype(np.float32)
            qs[b, h, :n * P].copy_(torch.from_numpy(np.ascontiguousarray(sl)).to(dev))
    elif K is not None:
        perm = torch.from_numpy(np.asarray(u["perm"][:n * C], dtype=np.int64))
        rows = torch.arange(n * C) // C * C + perm
        ok = perm >= 0
        dst = torch.nonzero(ok).flatten()
        ix.mK[b, h, dst.to(dev)] = K.to(dev)[rows[ok].to(dev)].to(ix.mK.dtype)
        ix.mV[b, h, dst.to(dev)] = V.to(dev)[rows[ok].to(dev)].to(ix.mV.dtype)


def assignment(u: dict, k: int, C: int = 256) -> np.ndarray:
    """Group slot of every position, reconstructed from (gCnt, perm)."""
    n = u["nchunks"]
    a = np.full(n * C, -1, np.int32)
    for c in range(n):
        off = 0
        for j in range(k):
            cnt = int(u["gCnt"][c * k + j])
            for m in range(off, off + cnt):
                a[c * C + u["perm"][c * C + m]] = j
            off += cnt
    return a


def check_member_copies(ix: api.Index, b: int, h: int, K, V, nchunks: int, p: api.Params) -> None:
    """The member-ordered copies hold the cache rows bit for bit: row m of
    chunk c of mK / mV is row c * chunk + perm[m] of K / V (K, V: that
    sequence's [T][d] cache rows)."""
    C = p.chunk
    perm = ix.perm[b, h, :nchunks * C].long()
    ok = perm >= 0
    rows = torch.arange(nchunks * C, device=perm.device) // C * C + perm
    assert torch.equal(ix.mK[b, h, :nchunks * C][ok], K.to(perm.device)[rows[ok]])
    assert torch.equal(ix.mV[b, h, :nchunks * C][ok], V.to(perm.device)[rows[ok]])


def check_index_consistency(u: dict, K: np.ndarray, V: np.ndarray, cfg: oracle.Config, bf16: bool):
    """Internal consistency of an index, whoever built it: groups partition the
    chunk minus the sinks, pages cut each group into runs of 16 in ascending
    order, and every summary is its members' mean (to one storage ulp)."""
    k, P, C = cfg.clusters, cfg.page_slots, cfg.chunk
    if "gMeta" in u:
        np.testing.assert_array_equal(u["gMeta"], pack_meta(u, k))
    for c in range(u["nchunks"]):
        first = cfg.sinks if c == 0 else 0
        perm = u["perm"][c * C:(c + 1) * C]
        n = C - first
        assert sorted(perm[:n].tolist()) == list(range(first, C)), c
        assert np.all(perm[n:] == -1)
        off = 0
        for j in range(k):
            cnt = int(u["gCnt"][c * k + j])
            mem = perm[off:off + cnt]
            assert np.all(np.diff(mem) > 0)
            p0, p1 = u["gPage"][c * (k + 1) + j], u["gPage"][c * (k + 1) + j + 1]
            assert p1 - p0 == -(-cnt // 16)
            for s in range(p0, p1):
                b0, pc = u["pBeg"][c * P + s], u["pCnt"][c * P + s]
                assert b0 == off + (s - p0) * 16 and pc == min(16, cnt - (s - p0) * 16)
                _close_mean(u["pK"][c * P + s], K[c * C + perm[b0:b0 + pc]], bf16)
                _close_mean(u["pV"][c * P + s], V[c * C + perm[b0:b0 + pc]], bf16)
            if cnt:
                _close_mean(u["gK"][c * k + j], K[c * C + mem], bf16)
                _close_mean(u["gV"][c * k + j], V[c * C + mem], bf16)
            off += cnt


def _close_mean(got, rows, bf16):
    want = rows.astype(np.float64).mean(0)
    tol = (2.0 ** -8 * np.abs(want) + 1e-6) if bf16 else (1e-6 * np.abs(want) + 1e-6)
    assert np.all(np.abs(got - want) <= tol), np.max(np.abs(got - want) - tol)


def compare_builds(gu: dict, ou: dict, cfg: oracle.Config, bf16: bool) -> dict:
    """GPU vs oracle index of one sequence.  Returns counts for reporting."""
    k, C = cfg.clusters, cfg.chunk
    ga, oa = assignment(gu, k, C), assignment(ou, k, C)
    stats = dict(chunks=gu["nchunks"], fragile=0, diverged=0, keys_checked=0)
    for c in range(gu["nchunks"]):
        fragile = ou["min_margin"][c] <= MARGIN
        stats["fragile"] += int(fragile)
        sl = slice(c * C, (c + 1) * C)
        strong = ou["key_margin"][sl] > MARGIN
        mism = (ga[sl] != oa[sl]) & strong
        stats["keys_checked"] += int(strong.sum())
        if mism.any():
            assert fragile, "chunk %d: %d confident keys assigned differently" % (c, mism.sum())
            stats["diverged"] += 1
            continue
        if np.array_equal(ga[sl], oa[sl]):
            # same groups: same pages and the same summaries up to one storage ulp
            for key in ("gCnt",):
                np.testing.assert_array_equal(gu[key][c * k:(c + 1) * k], ou[key][c * k:(c + 1) * k])
            P = cfg.page_slots
            np.testing.assert_array_equal(gu["gPage"][c * (k + 1):(c + 1) * (k + 1)],
                                          ou["gPage"][c * (k + 1):(c + 1) * (k + 1)])
            np.testing.assert_array_equal(gu["perm"][sl], ou["perm"][sl])
            np.testing.assert_array_equal(gu["pCnt"][c * P:(c + 1) * P], ou["pCnt"][c * P:(c + 1) * P])
            for key, n in (("gK", k), ("gV", k), ("pK", P), ("pV", P)):
                g_, o_ = gu[key][c * n:(c + 1) * n], ou[key][c * n:(c + 1) * n]
                # the GPU rounds an fp32 sum and the oracle an fp64 sum of the
                # same members to bf16: the two sums differ by fp32 rounding,
                # so the results may straddle a rounding boundary and differ by
                # one bf16 ulp, at most 2^-7 of the value
                tol = (2.0 ** -7 * np.abs(o_) + 1e-6) if bf16 else (2e-6 * np.abs(o_) + 1e-6)
                assert np.all(np.abs(g_ - o_) <= tol), (c, key)
    return stats


def check_rows(cfg: oracle.Config, dtype: str, K: np.ndarray, V: np.ndarray, u: dict, rows,
               threads: int = 8) -> dict:
    """rows: list of (q[d] float32, t, gpu_out[d], gpu_lse, gpu_sel_groups, gpu_sel_pages).
    Checks selection (tie rule) and output against the oracle on index u
    (three-tier INT4 when u carries the pages' codes, see `quantized`)."""
    tol = TOL[dtype]
    sc = np.float32(cfg.scale if cfg.scale > 0 else 1.0 / np.sqrt(cfg.d))

    qk = dict(kq=u["kq"], vq=u["vq"]) if "kq" in u else {}

    def gscore(q, gid):
        return float(np.dot(q.astype(np.float64), u["gK"][gid])) * sc

    def check_order(q, t, sg, gsg):
        """The ABI's order of sel_groups: the opened groups best first, then
        -1 padding; as many opened groups as the oracle opens.  Neighbours
        may swap only within a score tie (TIE)."""
        gsg = np.asarray(gsg)
        nv = int((np.asarray(sg) >= 0).sum())
        assert np.all(gsg[:nv] >= 0) and np.all(gsg[nv:] == -1), (t, gsg, sg)
        s = [gscore(q, int(x)) for x in gsg[:nv]]
        for i in range(nv - 1):
            assert s[i] >= s[i + 1] - TIE, (t, gsg, s)
            if s[i] == s[i + 1]:
                assert gsg[i] < gsg[i + 1], (t, gsg)

    def one(row):
        q, t, gout, glse, gsg, gsp = row
        out, lse, sg, sp, st = oracle.attend_row(cfg, q, t, K, V, u, **qk)
        check_order(q, t, sg, gsg)
        forced = False
        if not (np.array_equal(np.sort(sg), np.sort(gsg))):
            # differing opened groups must be score ties within TIE
            s = lambda gid: gscore(q, gid)
            og = [x for x in sg if x >= 0 and x not in gsg]
            gg = [x for x in gsg if x >= 0 and x not in sg]
            assert len(og) == len(gg), (sg, gsg)
            assert max(abs(s(a) - s(b)) for a in og for b in gg) <= TIE, (t, og, gg)
            forced = True
        else:
            # same groups: the same pages, up to ties
            for r, gid in enumerate(gsg):
                if gid < 0:
                    continue
                orow = list(sg).index(gid)
                a, b = set(sp[orow][sp[orow] >= 0]), set(gsp[r][gsp[r] >= 0])
                if a != b:
                    s = lambda pid: float(np.dot(q.astype(np.float64), u["pK"][pid])) * sc
                    assert max(abs(s(x) - s(y)) for x in a - b for y in b - a) <= TIE
                    forced = True
        if forced:
            out, lse, *_ = oracle.attend_row(cfg, q, t, K, V, u, gsg, gsp, **qk)
        err = float(np.max(np.abs(out - gout)))
        assert err <= tol, "t=%d max-abs %.3g > %g" % (t, err, tol)
        lerr = abs(lse - glse)
        assert lerr <= 5 * tol, (t, lse, glse)
        return err, forced

    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(one, rows))
    return dict(rows=len(res), max_err=max(r[0] for r in res), forced=sum(r[1] for r in res))
