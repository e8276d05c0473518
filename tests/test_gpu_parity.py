"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Sizes are small enough for the oracle to finish in seconds yet span several
scan splits, several chunks per group split, and ragged tails.  The rules
(tolerances, tie handling, k-means margin rule) are in tests/lodtest.py.
"""
import numpy as np
import pytest
import torch

import oracle
from hierarchical_long_context_b200 import api, synth
from tests import lodtest as lt

pytestmark = pytest.mark.gpu


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda")


def _setup(w, k=None, T=None, **pkw):
    dev = _cuda()
    T = T or w.T
    Kc, Vc = synth.kv_cache(w, T)
    p = lt.params_of(w, k, Tmax=((T + 255) // 256) * 256, **pkw)
    Kd = torch.zeros((w.B, w.Hkv, p.Tmax, w.d), dtype=w.torch_dtype, device=dev)
    Vd = torch.zeros_like(Kd)
    Kd[:, :, :T] = Kc.to(dev)
    Vd[:, :, :T] = Vc.to(dev)
    return p, Kc, Vc, Kd, Vd


def _np(t):
    return t.float().cpu().numpy()


# ------------------------------------------------------------------ build

@pytest.mark.parametrize("name, k, T", [
    ("decode_tiny_f32", 4, 4096),
    ("decode_tiny_f32_zero_variance", 4, 4096),
    ("decode_tiny_f32_zero_variance", 8, 2048),   # more clusters than distinct keys: empty groups
    ("decode_gqa_32k_bf16", 4, 4096),
    ("build_128k_bf16", 8, 2048),
])
def test_build_matches_oracle(name, k, T):
    w = synth.WORKLOADS[name]
    w = w.with_(B=min(w.B, 2), Hkv=min(w.Hkv, 2), Hq=min(w.Hkv, 2) * w.g)
    p, Kc, Vc, Kd, Vd = _setup(w, k, T)
    ix = api.Index(p)
    nch = T // 256
    api.lod_build_index(p, Kd, Vd, 0, nch, ix)
    torch.cuda.synchronize()
    cfg = lt.oracle_cfg(w, k)
    tot = dict(chunks=0, fragile=0, diverged=0, keys_checked=0)
    for b in range(w.B):
        for h in range(w.Hkv):
            K, V = _np(Kc[b, h]), _np(Vc[b, h])
            gu = lt.unit_from_gpu(ix, b, h, nch, p)
            lt.check_index_consistency(gu, K, V, cfg, w.dtype == "bf16")
            lt.check_member_copies(ix, b, h, Kd[b, h], Vd[b, h], nch, p)
            ou = oracle.build_sequence(cfg, b * w.Hkv + h, K, V, nch)
            st = lt.compare_builds(gu, ou, cfg, w.dtype == "bf16")
            for key in tot:
                tot[key] += st[key]
    print(name, k, tot)
    assert tot["keys_checked"] > 0.9 * tot["chunks"] * 200
    assert tot["diverged"] <= max(1, tot["chunks"] // 20)


# ------------------------------------------------------------------ decode

def _decode_rows(p, w, Kd, Vd, ix, seq_lens, draws):
    dev = Kd.device
    rows = []
    ws = api.workspace(p, api._lib.LOD_OP_DECODE)
    for s in range(draws):
        q = synth.decode_queries(w, stream="queries%d" % s).to(dev)
        sl = torch.tensor(seq_lens, dtype=torch.int64, device=dev)
        lse = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
        sg = torch.empty(w.B, w.Hq, p.top_groups, dtype=torch.int32, device=dev)
        sp = torch.empty(w.B, w.Hq, p.top_groups, p.top_pages, dtype=torch.int32, device=dev)
        out = api.lod_decode(p, q, Kd, Vd, sl, ix, lse=lse, sel_groups=sg, sel_pages=sp, ws=ws)
        torch.cuda.synchronize()
        assert api.lod_get_status(ws) == 0
        for b in range(w.B):
            for hq in range(w.Hq):
                rows.append(((b, hq // w.g), _np(q[b, hq]), seq_lens[b] - 1, _np(out[b, hq]).astype(np.float64),
                             float(lse[b, hq]), sg[b, hq].cpu().numpy(), sp[b, hq].cpu().numpy()))
    return rows


def _check_decode(w, p, Kc, Vc, ix, rows, cfg, use):
    by_unit = {}
    for r in rows:
        by_unit.setdefault(r[0], []).append(r[1:])
    stats = []
    for (b, h), rr in by_unit.items():
        K, V = _np(Kc[b, h]), _np(Vc[b, h])
        nch = max(r[1] for r in rr) // 256 + 1
        u = use(b, h, K, V, nch)
        stats.append(lt.check_rows(cfg, w.dtype, K, V, u, rr))
    return stats


@pytest.mark.parametrize("name, T, seq_lens", [
    ("decode_tiny_f32", 4096, [4096]),
    ("decode_tiny_f32_zero_variance", 4096, [4096]),
    ("decode_gqa_32k_bf16", 8192, [8192, 5000]),
    ("decode_gqa_32k_bf16", 4096, [1, 700]),          # window covers everything: no index used
])
def test_decode_on_gpu_index_matches_oracle(name, T, seq_lens):
    w = synth.WORKLOADS[name]
    w = w.with_(B=len(seq_lens), Hkv=min(w.Hkv, 2), Hq=min(w.Hkv, 2) * w.g)
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    rows = _decode_rows(p, w, Kd, Vd, ix, seq_lens, draws=4 if w.Hq > 1 else 16)
    cfg = lt.oracle_cfg(w)
    st = _check_decode(w, p, Kc, Vc, ix, rows, cfg,
                       lambda b, h, K, V, n: lt.unit_from_gpu(ix, b, h, T // 256, p))
    print(name, st)


@pytest.mark.parametrize("kw", [
    dict(d=64, Hq=2, Hkv=2),                                                  # bf16 d=64 (CUDA-core scan), MHA
    dict(Hq=4, Hkv=2, clusters=(16,), top_groups=16, top_pages=4),            # g=2, k=16, widest selection
    dict(dtype="f32", Hq=8, Hkv=2, clusters=(1,), top_groups=1, top_pages=1),  # fp32 d=128, k=1, one page
    dict(Hq=16, Hkv=2, window=256, sinks=0),                                   # g=8, short window, no sinks
    dict(top_pages=0),                                                         # two-tier LoD, g=8
    dict(d=64, dtype="f32", Hq=4, Hkv=2, top_groups=16, top_pages=0),          # two-tier, CUDA-core scan
    dict(Hq=16, Hkv=2, sinks=100),                                             # more sinks than free lanes
    dict(Hq=2, Hkv=2),                                                         # bf16 d=128 MHA: one query row per scan unit
    dict(Hq=8, Hkv=2, top_groups=12),                                          # g=4, G between 8 and 16
])
def test_decode_parameter_sweep(kw):
    """Head ratios, head sizes, dtypes, cluster counts and selection widths at
    the edges of what lod_params accepts, each against the oracle."""
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, T=4096, **kw)
    T = 4096
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    rows = _decode_rows(p, w, Kd, Vd, ix, [T, T - 777], draws=2)
    cfg = lt.oracle_cfg(w)
    st = _check_decode(w, p, Kc, Vc, ix, rows, cfg,
                       lambda b, h, K, V, n: lt.unit_from_gpu(ix, b, h, T // 256, p))
    print(kw, st)


def test_decode_on_oracle_index_matches_oracle():
    """The attention kernels alone: the index is the oracle's, imported."""
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, Hkv=2, Hq=16)
    T = 6144
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    cfg = lt.oracle_cfg(w)
    ix = api.Index(p)
    ous = {}
    for b in range(w.B):
        for h in range(w.Hkv):
            ous[(b, h)] = oracle.build_sequence(cfg, b * w.Hkv + h, _np(Kc[b, h]), _np(Vc[b, h]), T // 256)
            lt.unit_to_gpu(ix, b, h, ous[(b, h)], p, Kd[b, h], Vd[b, h])
    rows = _decode_rows(p, w, Kd, Vd, ix, [T, T - 300], draws=4)
    st = _check_decode(w, p, Kc, Vc, ix, rows, cfg, lambda b, h, K, V, n: ous[(b, h)])
    print(st)


# ------------------------------------------------------------------ three-tier INT4

@pytest.mark.parametrize("name, k, T, kw", [
    ("decode_gqa_32k_bf16", 4, 4096, {}),
    ("decode_gqa_32k_bf16", 8, 2048, dict(d=64)),
    ("decode_tiny_f32", 4, 4096, {}),
])
def test_int4_build_matches_oracle(name, k, T, kw):
    """Three-tier INT4 build: the codes and per-page quantisers equal the
    oracle's quantiser on the GPU-built index bit for bit; the summaries
    follow the same rules as the cache-dtype build."""
    w = synth.WORKLOADS[name].with_(**kw)
    w = w.with_(B=min(w.B, 2), Hkv=min(w.Hkv, 2), Hq=min(w.Hkv, 2) * w.g)
    p, Kc, Vc, Kd, Vd = _setup(w, k, T, kv_bits=4)
    ix = api.Index(p)
    assert ix.mK.numel() == 0 and ix.qK.numel() > 0
    nch = T // 256
    api.lod_build_index(p, Kd, Vd, 0, nch, ix)
    torch.cuda.synchronize()
    cfg = lt.oracle_cfg(w, k)
    rows = 0
    tot = dict(chunks=0, fragile=0, diverged=0, keys_checked=0)
    for b in range(w.B):
        for h in range(w.Hkv):
            K, V = _np(Kc[b, h]), _np(Vc[b, h])
            gu = lt.unit_from_gpu(ix, b, h, nch, p)
            lt.check_index_consistency(gu, K, V, cfg, w.dtype == "bf16")
            rows += lt.check_int4_pages(ix, b, h, gu, K, V, cfg)
            ou = oracle.build_sequence(cfg, b * w.Hkv + h, K, V, nch)
            st = lt.compare_builds(gu, ou, cfg, w.dtype == "bf16")
            for key in tot:
                tot[key] += st[key]
    print(name, k, kw, rows, tot)
    assert rows > 0.9 * w.B * w.Hkv * nch * 256
    assert tot["diverged"] <= max(1, tot["chunks"] // 20)


@pytest.mark.parametrize("kw", [
    dict(),                                        # bf16 d=128, g=8 (tensor-core scan), two pages a group
    dict(Hq=4, Hkv=2, top_pages=4, top_groups=16),  # two page pairs a group, g=2
    dict(d=64, Hq=2, Hkv=2, top_pages=1),           # one page a group, CUDA-core scan, MHA
    dict(dtype="f32", Hq=8, Hkv=2),                 # fp32 cache
])
def test_int4_decode_matches_oracle(kw):
    """Three-tier INT4 decode on the GPU-built index against the oracle
    reading the same pages decompressed."""
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, T=4096, Hq=16, Hkv=2).with_(**kw)
    T = 4096
    p, Kc, Vc, Kd, Vd = _setup(w, None, T, kv_bits=4)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    rows = _decode_rows(p, w, Kd, Vd, ix, [T, T - 777], draws=2)
    cfg = lt.oracle_cfg(w)
    st = _check_decode(w, p, Kc, Vc, ix, rows, cfg,
                       lambda b, h, K, V, n: lt.quantized(lt.unit_from_gpu(ix, b, h, T // 256, p), K, V, cfg))
    print(kw, st)


def test_int4_decode_on_oracle_index_matches_oracle():
    """The INT4 attention kernels alone: index and codes are the oracle's."""
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, Hkv=2, Hq=16)
    T = 6144
    p, Kc, Vc, Kd, Vd = _setup(w, None, T, kv_bits=4)
    cfg = lt.oracle_cfg(w)
    ix = api.Index(p)
    ous = {}
    for b in range(w.B):
        for h in range(w.Hkv):
            K, V = _np(Kc[b, h]), _np(Vc[b, h])
            ous[(b, h)] = lt.quantized(oracle.build_sequence(cfg, b * w.Hkv + h, K, V, T // 256), K, V, cfg)
            lt.unit_to_gpu(ix, b, h, ous[(b, h)], p)
    rows = _decode_rows(p, w, Kd, Vd, ix, [T, T - 300], draws=4)
    st = _check_decode(w, p, Kc, Vc, ix, rows, cfg, lambda b, h, K, V, n: ous[(b, h)])
    print(st)


# ------------------------------------------------------------------ online build

def test_online_build_during_decode_matches_bulk_build():
    """The index built online -- lod_build_ready issued every decode step on a
    second stream, concurrently with lod_decode -- equals the bulk build bit
    for bit, and the decodes of those steps equal decodes on the bulk-built
    index (the chunk being built is not yet visible to them)."""
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=4, Hkv=2, Hq=16)
    T = 4096
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    dev = Kd.device
    L0 = [2045, 2041, 2047, 1900]   # three sequences complete chunk 7 at different steps
    steps = 12
    ix_on, ix_bulk = api.Index(p), api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, 7, ix_on)
    api.lod_build_index(p, Kd, Vd, 0, 8, ix_bulk)
    ws_b = api.workspace(p, api._lib.LOD_OP_BUILD)
    ws_d = api.workspace(p, api._lib.LOD_OP_DECODE)
    ws_r = api.workspace(p, api._lib.LOD_OP_DECODE)
    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    outs_on, outs_ref = [], []
    for s in range(steps):
        sl = torch.tensor([x + s + 1 for x in L0], dtype=torch.int64, device=dev)
        q = synth.decode_queries(w, stream="queries%d" % s).to(dev)
        side.wait_stream(main)             # the step's inputs (lengths) are ready
        api.lod_build_ready(p, Kd, Vd, sl, ix_on, ws=ws_b, stream=side)
        outs_on.append(api.lod_decode(p, q, Kd, Vd, sl, ix_on, ws=ws_d))
        outs_ref.append(api.lod_decode(p, q, Kd, Vd, sl, ix_bulk, ws=ws_r))
        sl.record_stream(side)
    main.wait_stream(side)
    torch.cuda.synchronize()
    assert api.lod_get_status(ws_d) == 0 and api.lod_get_status(ws_b) == 0
    for a, b in zip(outs_on, outs_ref):
        assert torch.equal(a, b)
    k, P, C = p.clusters, p.page_slots, p.chunk
    fresh = api.Index(p)
    per = {"gK": k, "gV": k, "gCnt": k, "pK": P, "pV": P, "pCnt": P, "pBeg": P, "gPage": k + 1,
           "perm": C, "mK": C, "mV": C, "gMeta": k}
    for f, n in per.items():
        on, bulk = getattr(ix_on, f), getattr(ix_bulk, f)
        for b in range(w.B):
            built = 8 if b < 3 else 7        # sequence 3 never reaches 2048 tokens
            assert torch.equal(on[b, :, :built * n], bulk[b, :, :built * n]), (f, b)
            if b == 3:                        # its chunk 7 is untouched
                assert torch.equal(on[b, :, 7 * n:8 * n], getattr(fresh, f)[b, :, 7 * n:8 * n]), f


def test_head_shard_builds_the_unsharded_index_slice():
    """A process holding KV heads [2, 4) of a 4-head model (head_shard) builds
    exactly those heads' slice of the unsharded index, and decodes them alike."""
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, Hkv=4, Hq=16)
    T = 2048
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    ws_ = synth.shard(w, "heads", 1, 2)
    ps = lt.params_of(ws_, Tmax=p.Tmax, head_shard=(ws_.hkv_model << 16) | ws_.kvh0)
    Ks, Vs = Kd[:, 2:4].contiguous(), Vd[:, 2:4].contiguous()
    ixs = api.Index(ps)
    api.lod_build_index(ps, Ks, Vs, 0, T // 256, ixs)
    for f in api._lib.INDEX_FIELDS:
        a, b = getattr(ix, f), getattr(ixs, f)
        if a.numel():
            assert torch.equal(a[:, 2:4], b), f
    sl = torch.full((w.B,), T, dtype=torch.int64, device=Kd.device)
    q = synth.decode_queries(w).to(Kd.device)
    out = api.lod_decode(p, q, Kd, Vd, sl, ix)
    outs = api.lod_decode(ps, q[:, 8:16].contiguous(), Ks, Vs, sl, ixs)
    assert torch.equal(out[:, 8:16], outs)


def test_append_kv_writes_the_current_rows_only():
    """lod_append_kv writes each sequence's new key/value rows at seq_len - 1
    and nothing else; a length outside [1, Tmax] leaves that sequence alone."""
    dev = _cuda()
    p = api.Params(B=3, Hq=16, Hkv=2, d=128, Tmax=1024, dtype=torch.bfloat16)
    g = torch.Generator(device=dev).manual_seed(5)
    K = torch.randn(3, 2, 1024, 128, generator=g, device=dev).to(torch.bfloat16)
    V = torch.randn(3, 2, 1024, 128, generator=g, device=dev).to(torch.bfloat16)
    K0, V0 = K.clone(), V.clone()
    kn = torch.randn(3, 2, 128, generator=g, device=dev).to(torch.bfloat16)
    vn = torch.randn(3, 2, 128, generator=g, device=dev).to(torch.bfloat16)
    sl = torch.tensor([5, 1024, 0], dtype=torch.int64, device=dev)
    api.lod_append_kv(p, K, V, sl, kn, vn)
    torch.cuda.synchronize()
    K0[0, :, 4], V0[0, :, 4] = kn[0], vn[0]
    K0[1, :, 1023], V0[1, :, 1023] = kn[1], vn[1]
    assert torch.equal(K, K0) and torch.equal(V, V0)


def test_pinned_host_buffers_are_used_in_place():
    """q, the new K/V rows and out in pinned host memory: the kernels read and
    write them directly, with the device buffers' result; pageable host memory
    and another device's memory are refused before anything is enqueued."""
    from hierarchical_long_context_b200 import _lib
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, Hq=16, Hkv=2, T=4096)
    p, Kc, Vc, Kd, Vd = _setup(w)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, w.T // 256, ix)
    q = synth.decode_queries(w).cuda()
    sl = torch.full((w.B,), w.T, dtype=torch.int64, device="cuda")
    ref = api.lod_decode(p, q, Kd, Vd, sl, ix)
    hq = q.cpu().pin_memory()
    hout = torch.zeros(q.shape, dtype=q.dtype).pin_memory()
    api.lod_decode(p, hq, Kd, Vd, sl, ix, out=hout)
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu())
    g = torch.Generator().manual_seed(3)
    kn = torch.randn(w.B, w.Hkv, w.d, generator=g).to(w.torch_dtype).pin_memory()
    vn = torch.randn(w.B, w.Hkv, w.d, generator=g).to(w.torch_dtype).pin_memory()
    K2, V2 = Kd.clone(), Vd.clone()
    api.lod_append_kv(p, K2, V2, sl, kn, vn)
    torch.cuda.synchronize()
    assert torch.equal(K2[:, :, w.T - 1].cpu(), kn) and torch.equal(V2[:, :, w.T - 1].cpu(), vn)
    assert torch.equal(K2[:, :, :w.T - 1], Kd[:, :, :w.T - 1])
    # refused: pageable host memory (no kernel is launched for these calls)
    pageable_q, pageable_out, pageable_k = q.cpu(), torch.zeros(q.shape, dtype=q.dtype), kn.clone()
    assert not pageable_q.is_pinned() and not pageable_k.is_pinned()
    for call in (lambda: api.lod_decode(p, pageable_q, Kd, Vd, sl, ix, out=hout),
                 lambda: api.lod_decode(p, hq, Kd, Vd, sl, ix, out=pageable_out),
                 lambda: api.lod_append_kv(p, K2, V2, sl, pageable_k, vn)):
        with pytest.raises(_lib.LodError) as e:
            call()
        assert e.value.code == _lib.LOD_EINVAL and "pageable" in str(e.value)
    assert torch.equal(pageable_out, torch.zeros_like(pageable_out))


def test_zero_variance_decode_equals_dense():
    """Level of Detail Attention, How It Works: zero-variance groups give full
    attention -- checked on the GPU path directly against dense softmax."""
    w = synth.WORKLOADS["decode_tiny_f32_zero_variance"]
    p, Kc, Vc, Kd, Vd = _setup(w)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, w.T // 256, ix)
    cfg = lt.oracle_cfg(w)
    K, V = _np(Kc[0, 0]), _np(Vc[0, 0])
    for s in range(8):
        q = synth.decode_queries(w, stream="dense%d" % s).cuda()
        out = api.lod_decode(p, q, Kd, Vd, torch.tensor([w.T], device="cuda"), ix)
        dout, _ = oracle.dense_row(cfg, _np(q[0, 0]), w.T - 1, K, V)
        assert np.max(np.abs(_np(out[0, 0]) - dout)) < 1e-5


@pytest.mark.parametrize("B, Hkv", [(1, 1), (4, 8)])
def test_tied_group_scores_open_the_smallest_ids_across_splits(B, Hkv):
    """Groups with equal scores rank by smaller id (D8) however the scan
    splits the unit's groups: a best key S sits in every 37th chunk and a
    second key G in every chunk, every chunk's four keys repeated 64 times,
    so the index's group means are those keys exactly and all S groups (and
    all G groups) tie.  The query points at S: the 8 opened groups must be
    the S groups of chunks 0, 37, .., 222 by id, then the G group of chunk 0
    (with B = 4, Hkv = 8 each split scans several group tiles)."""
    dev = _cuda()
    T, k, d = 65536, 4, 128
    w = synth.WORKLOADS["decode_gqa_128k_bf16"].with_(B=B, Hkv=Hkv, Hq=8 * Hkv, T=T)
    p = lt.params_of(w, k, Tmax=T)
    e = torch.eye(d)
    S, G = 2.0 * e[0], 1.0 * e[0]
    filler = [e[1] * 0.5, e[2] * 0.5, e[3] * 0.5, e[4] * 0.5]
    keys = torch.zeros(T // 256, 4, d)
    for c in range(T // 256):
        ks = [S, G, filler[0], filler[1]] if c % 37 == 0 else [G, filler[0], filler[1], filler[2]]
        keys[c] = torch.stack(ks)
    Kc = keys.repeat_interleave(64, dim=1).reshape(T, d)  # each key on 64 consecutive positions
    Kd = Kc.to(torch.bfloat16).to(dev).expand(B, Hkv, T, d).contiguous()
    Vd = torch.randn(B, Hkv, T, d, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).to(dev)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    q = torch.zeros(B, 8 * Hkv, d)
    q[..., 0] = 1.0
    q = q.to(torch.bfloat16).to(dev)
    sg = torch.empty(B, 8 * Hkv, p.top_groups, dtype=torch.int32, device=dev)
    ws = api.workspace(p, api._lib.LOD_OP_DECODE)
    api.lod_decode(p, q, Kd, Vd, torch.full((B,), T, dtype=torch.int64, device=dev), ix, sel_groups=sg, ws=ws)
    torch.cuda.synchronize()
    assert api.lod_get_status(ws) == 0
    gK = ix.gK.float().cpu()
    sgc = sg.cpu()
    vis = (T // 256 - p.window // 256) * k  # groups of the complete chunks before the window
    for b in range(B):
        for h in range(Hkv):
            def slot_of(c, key):
                hit = [j for j in range(k) if torch.equal(gK[b, h, c * k + j], key)]
                assert len(hit) == 1, (c, hit)
                return c * k + hit[0]
            want = [slot_of(c, S) for c in range(0, T // 256, 37) if (c + 1) * k <= vis]
            want = (want + [slot_of(0, G)])[: p.top_groups]
            for hq in range(h * 8, h * 8 + 8):
                assert sgc[b, hq].tolist() == want, (b, hq, sgc[b, hq].tolist(), want)


# ------------------------------------------------------------------ prefill

@pytest.mark.parametrize("name, T, split, kv_bits", [
    ("prefill_128k_bf16", 2048 + 100, None, 0),      # ragged tail, one call
    ("prefill_128k_bf16", 2048 + 100, 1024, 0),      # two calls: the second continues the first
    ("decode_tiny_f32", 1536 + 37, None, 0),
    ("decode_gqa_32k_bf16", 1024 + 300, None, 0),    # g = 8: one position per scan unit
    ("prefill_128k_bf16", 2048 + 100, 1024, 4),      # three-tier INT4
])
def test_prefill_matches_oracle(name, T, split, kv_bits):
    w = synth.WORKLOADS[name]
    w = w.with_(B=1, Hkv=min(w.Hkv, 2), Hq=min(w.Hkv, 2) * w.g, T=T)
    p, Kc, Vc, Kd, Vd = _setup(w, None, T, kv_bits=kv_bits)
    dev = Kd.device
    qc = synth.prefill_queries(w, 0, T)
    q = qc.to(dev)
    ix = api.Index(p)
    lse = torch.empty(w.B, w.Hq, T, dtype=torch.float32, device=dev)
    sg = torch.empty(w.B, w.Hq, T, p.top_groups, dtype=torch.int32, device=dev)
    sp = torch.empty(w.B, w.Hq, T, p.top_groups, p.top_pages, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    ws = api.workspace(p, api._lib.LOD_OP_PREFILL)
    cuts = [0, T] if split is None else [0, split, T]
    for lo, hi in zip(cuts, cuts[1:]):
        _prefill_piece(p, q, lo, hi, Kd, Vd, ix, out, lse, sg, sp, ws)
    torch.cuda.synchronize()
    assert api.lod_get_status(ws) == 0
    cfg = lt.oracle_cfg(w)
    rng = np.random.default_rng(3)
    nch = T // 256
    for h in range(w.Hkv):
        K, V = _np(Kc[0, h]), _np(Vc[0, h])
        u = lt.unit_from_gpu(ix, 0, h, nch, p)
        lt.check_index_consistency(u, K, V, cfg, w.dtype == "bf16")
        if kv_bits == 4:
            lt.check_int4_pages(ix, 0, h, u, K, V, cfg)
            u = lt.quantized(u, K, V, cfg)
        ts = sorted(set(rng.integers(0, T, 48).tolist()) | {0, 255, 256, 511, 512, T - 1})
        rows = []
        for hq in range(h * w.g, (h + 1) * w.g):
            for t in ts:
                rows.append((_np(q[0, hq, t]), t, _np(out[0, hq, t]).astype(np.float64),
                             float(lse[0, hq, t]), sg[0, hq, t].cpu().numpy(), sp[0, hq, t].cpu().numpy()))
        print(lt.check_rows(cfg, w.dtype, K, V, u, rows))


@pytest.mark.parametrize("kw, T", [
    (dict(Hq=2, Hkv=2), 2048 + 100),                                       # g = 1: 128 positions per tile
    (dict(Hq=4, Hkv=2), 2048 + 100),                                       # g = 2
    (dict(top_pages=0), 2048 + 100),                                       # two-tier LoD: groups opened whole
    (dict(clusters=(16,), top_groups=16, top_pages=4), 2048 + 100),        # k = 16, widest selection
    (dict(clusters=(1,), top_groups=2, top_pages=1), 3072 + 5),            # k = 1: groups of 252-256 members
    (dict(clusters=(2,), sinks=100, window=256), 2048 + 100),              # a sink tile with 100 live rows
    (dict(Hq=8, Hkv=2, window=1024), 2048 + 100),                          # window of four chunks
])
def test_grouped_prefill_sweep(kw, T):
    """The grouped tensor-core prefill over the head ratios, selection widths,
    cluster counts (group sizes up to a whole chunk), windows and sinks that
    lod_params accepts, each against the oracle on sampled rows."""
    w = synth.WORKLOADS["prefill_128k_bf16"].with_(B=1, Hkv=2, Hq=8).with_(**kw)
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    dev = Kd.device
    q = synth.prefill_queries(w, 0, T).to(dev)
    ix = api.Index(p)
    lse = torch.empty(w.B, w.Hq, T, dtype=torch.float32, device=dev)
    sg = torch.empty(w.B, w.Hq, T, p.top_groups, dtype=torch.int32, device=dev)
    sp = torch.empty(w.B, w.Hq, T, p.top_groups, max(p.top_pages, 1), dtype=torch.int32, device=dev)
    ws = api.workspace(p, api._lib.LOD_OP_PREFILL)
    out = api.lod_prefill(p, q, 0, Kd, Vd, ix, lse=lse, sel_groups=sg, sel_pages=sp if p.top_pages else None,
                          ws=ws)
    torch.cuda.synchronize()
    assert api.lod_get_status(ws) == 0
    assert torch.isfinite(out.float()).all()
    cfg = lt.oracle_cfg(w)
    rng = np.random.default_rng(5)
    nch = T // 256
    for h in range(w.Hkv):
        K, V = _np(Kc[0, h]), _np(Vc[0, h])
        u = lt.unit_from_gpu(ix, 0, h, nch, p)
        ts = sorted(set(rng.integers(0, T, 24).tolist()) | {0, 511, 512, 767, 1024, T - 1})
        rows = []
        for hq in range(h * w.g, (h + 1) * w.g):
            for t in ts:
                gsp = sp[0, hq, t].cpu().numpy() if p.top_pages else np.zeros((p.top_groups, 0), np.int32)
                rows.append((_np(q[0, hq, t]), t, _np(out[0, hq, t]).astype(np.float64),
                             float(lse[0, hq, t]), sg[0, hq, t].cpu().numpy(), gsp))
        print(kw, lt.check_rows(cfg, w.dtype, K, V, u, rows))


def test_grouped_prefill_several_waves_match_one_call_per_chunk():
    """A prefill longer than one wave of query chunks (at most 128 chunks)
    equals the same queries prefilled one chunk per call: the wave boundaries,
    the next wave's index built on a second stream while a wave attends, and
    the pair bookkeeping leave every row's result unchanged, bit for bit."""
    w = synth.WORKLOADS["prefill_128k_bf16"].with_(B=1, Hkv=1, Hq=4)
    T = 2 * 128 * 256 + 700
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    dev = Kd.device
    q = synth.prefill_queries(w, 0, T).to(dev)
    ws = api.workspace(p, api._lib.LOD_OP_PREFILL)
    ix = api.Index(p)
    lse = torch.empty(w.B, w.Hq, T, dtype=torch.float32, device=dev)
    out = api.lod_prefill(p, q, 0, Kd, Vd, ix, lse=lse, ws=ws)
    ix2 = api.Index(p)
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    for lo in range(0, T, 256):
        hi = min(T, lo + 256)
        o = torch.empty_like(q[:, :, lo:hi].contiguous())
        l_ = torch.empty(w.B, w.Hq, hi - lo, dtype=torch.float32, device=dev)
        api.lod_prefill(p, q[:, :, lo:hi].contiguous(), lo, Kd, Vd, ix2, out=o, lse=l_, ws=ws)
        out2[:, :, lo:hi] = o
        lse2[:, :, lo:hi] = l_
    torch.cuda.synchronize()
    assert api.lod_get_status(ws) == 0
    assert torch.equal(out, out2)
    assert torch.equal(lse, lse2)


def _prefill_piece(p, q, lo, hi, Kd, Vd, ix, out, lse, sg, sp, ws):
    o = torch.empty_like(q[:, :, lo:hi].contiguous())
    l_ = torch.empty(q.shape[0], q.shape[1], hi - lo, dtype=torch.float32, device=q.device)
    g_ = torch.empty(q.shape[0], q.shape[1], hi - lo, p.top_groups, dtype=torch.int32, device=q.device)
    p_ = torch.empty(q.shape[0], q.shape[1], hi - lo, p.top_groups, p.top_pages, dtype=torch.int32,
                     device=q.device)
    api.lod_prefill(p, q[:, :, lo:hi].contiguous(), lo, Kd, Vd, ix, out=o, lse=l_, sel_groups=g_,
                    sel_pages=p_, ws=ws)
    out[:, :, lo:hi] = o
    lse[:, :, lo:hi] = l_
    sg[:, :, lo:hi] = g_
    sp[:, :, lo:hi] = p_


# ------------------------------------------------------------------ faults

def test_bad_index_values_are_skipped_and_reported():
    """A corrupted index entry is bounds-checked by the kernel, skipped, and
    reported through the status word; nothing out of range is dereferenced."""
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=1, Hkv=1, Hq=8)
    T = 4096
    p, Kc, Vc, Kd, Vd = _setup(w, None, T)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    ws = api.workspace(p, api._lib.LOD_OP_DECODE)
    q = synth.decode_queries(w).cuda()
    sl = torch.tensor([T], device="cuda")
    sg = torch.empty(1, 8, p.top_groups, dtype=torch.int32, device="cuda")
    api.lod_decode(p, q, Kd, Vd, sl, ix, sel_groups=sg, ws=ws)
    assert api.lod_get_status(ws) == 0
    # move every page's member run of the chunks the first head opens past the chunk end
    P = p.page_slots
    for gid in sg[0, 0].tolist():
        c = gid // p.clusters
        ix.pBeg[0, 0, c * P:(c + 1) * P] = 250
    api.lod_decode(p, q, Kd, Vd, sl, ix, ws=ws)
    st = api.lod_get_status(ws)
    assert st & api._lib.LOD_ST_BAD_MEMBER
    assert api.lod_get_status(ws) == 0          # read clears it
    # a sequence length beyond the cache
    api.lod_decode(p, q, Kd, Vd, torch.tensor([T + 1], device="cuda"), ix, ws=ws)
    assert api.lod_get_status(ws) & api._lib.LOD_ST_BAD_SEQLEN
    # page ranges past the chunk's slots in the packed group words
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    api.lod_decode(p, q, Kd, Vd, sl, ix, ws=ws)
    assert api.lod_get_status(ws) == 0
    ix.gMeta[0, 0] = (ix.gMeta[0, 0] & 0xffff) | (200 << 24)
    out = api.lod_decode(p, q, Kd, Vd, sl, ix, ws=ws)
    assert api.lod_get_status(ws) & api._lib.LOD_ST_BAD_PAGE
    assert torch.isfinite(out.float()).all()
