"""Seeded synthetic inputs shaped like the long-context workloads of LoD attention.

This module holds no LoD arithmetic: it only draws keys, values and queries.
It is the one piece shared by the CUDA path's tests and benchmark and by the
CPU oracle's tests, so both see identical numbers.

Recipe (one independent PCG64 stream per (workload, batch entry, KV head)):
  * centres mu_j: Gaussian vectors normalised to unit length;
  * key at position t: mu_z + sigma * N(0, I), z uniform over the centres;
  * optional outlier channels: a few seeded channels get +/- magnitude added;
  * optional RoPE (rotate-half pairing (i, i + d/2), inverse frequency
    theta^(-2i/d)) applied to each key at its position, after the outliers;
  * values N(0, 1); queries N(0, 1) / 8;
  * zero-variance variant: every 256-token chunk draws `clusters` (key, value)
    pairs and each position of the chunk copies one of them, so every k-means
    group holds identical keys and values.
Keys, values and queries are drawn in float32 and then rounded to the cache
dtype (bfloat16, round-to-nearest-even, via torch) where the workload says so.
"""
from __future__ import annotations

import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    dtype: str                 # "f32" or "bf16": the KV-cache dtype
    n_centers: int
    sigma: float = 0.3
    rope_theta: float = 0.0    # 0: no RoPE
    n_outliers: int = 0
    outlier_mag: float = 8.0
    clusters: tuple = (4,)
    iters: int = 8
    top_groups: int = 8
    top_pages: int = 2
    window: int = 256
    sinks: int = 1
    seed: int = 0
    zero_variance: bool = False
    mode: str = "decode"       # decode | prefill | build
    chunk: int = 256
    page: int = 16
    note: str = ""
    kvh0: int = 0              # global index of the first KV head (a head shard's slice)
    hkv_model: int = 0         # a head shard's model-wide KV head count (0: not sharded)

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the method's measurement plan, named by what they are.
WORKLOADS = {
    "decode_tiny_f32": Workload(
        "decode_tiny_f32", B=1, Hq=1, Hkv=1, d=64, T=4096, dtype="f32", n_centers=64,
        window=256, sinks=1, note="tiny single-head decode, fp32"),
    "decode_tiny_f32_zero_variance": Workload(
        "decode_tiny_f32_zero_variance", B=1, Hq=1, Hkv=1, d=64, T=4096, dtype="f32",
        n_centers=64, window=256, sinks=1, zero_variance=True,
        note="tiny decode with zero-variance groups: LoD equals dense attention"),
    "decode_gqa_32k_bf16": Workload(
        "decode_gqa_32k_bf16", B=8, Hq=64, Hkv=8, d=128, T=32768, dtype="bf16",
        n_centers=512, rope_theta=1e6, n_outliers=4, window=512, sinks=4,
        note="GQA decode at 32K"),
    "decode_gqa_128k_bf16": Workload(
        "decode_gqa_128k_bf16", B=4, Hq=64, Hkv=8, d=128, T=131072, dtype="bf16",
        n_centers=512, rope_theta=1e6, n_outliers=4, window=512, sinks=4,
        note="GQA decode at 128K (decode headline)"),
    "prefill_128k_bf16": Workload(
        "prefill_128k_bf16", B=1, Hq=32, Hkv=8, d=128, T=131072, dtype="bf16",
        n_centers=512, rope_theta=1e6, window=512, sinks=4, mode="prefill",
        note="chunked causal prefill at 128K"),
    "decode_gqa_1m_bf16": Workload(
        "decode_gqa_1m_bf16", B=1, Hq=64, Hkv=8, d=128, T=1048576, dtype="bf16",
        n_centers=512, rope_theta=1e6, n_outliers=4, window=512, sinks=4,
        note="long-context GQA decode at 1M (one sequence); device-generated (kv_cache_device)"),
    "build_128k_bf16": Workload(
        "build_128k_bf16", B=1, Hq=8, Hkv=8, d=128, T=131072, dtype="bf16",
        n_centers=2048, rope_theta=1e6, clusters=(4, 8), window=512, sinks=4, mode="build",
        note="index build at 128K, k=4 and k=8"),
}


def _unit_rng(w: Workload, b: int, kvh: int, stream: str) -> np.random.Generator:
    tag = zlib.crc32(w.name.replace("_zero_variance", "").encode())
    s2 = zlib.crc32(stream.encode())
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, tag, b, kvh + w.kvh0, s2])))


def shard(w: Workload, mode: str, rank: int, world: int) -> Workload:
    """Rank `rank`'s part of workload `w` on `world` GPUs.  "batch": every
    rank decodes its own batch (a replica with its own seed; weak scaling).
    "heads": the ranks split the KV heads (with their query heads) of the one
    batch, as tensor-parallel attention does; rank r generates exactly its
    slice of the global inputs (strong scaling).  No data crosses ranks."""
    if world == 1:
        return w
    if mode == "batch":
        return w.with_(seed=w.seed + rank)
    if mode == "heads":
        if w.Hkv % world:
            raise ValueError("%d KV heads do not split over %d ranks" % (w.Hkv, world))
        h = w.Hkv // world
        return w.with_(Hkv=h, Hq=h * w.g, kvh0=w.kvh0 + rank * h, hkv_model=w.hkv_model or w.Hkv)
    raise ValueError("shard mode %r" % mode)


def _rope(x: np.ndarray, theta: float, pos0: int = 0) -> np.ndarray:
    T, d = x.shape
    h = d // 2
    inv = theta ** (-2.0 * np.arange(h, dtype=np.float64) / d)
    ang = (np.arange(pos0, pos0 + T, dtype=np.float64)[:, None] * inv[None, :])
    c = np.cos(ang).astype(np.float32)
    s = np.sin(ang).astype(np.float32)
    x1, x2 = x[:, :h], x[:, h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def _mixture_keys(w: Workload, rng: np.random.Generator, T: int) -> np.ndarray:
    cen = rng.standard_normal((w.n_centers, w.d), dtype=np.float32)
    cen /= np.linalg.norm(cen, axis=1, keepdims=True)
    z = rng.integers(0, w.n_centers, size=T)
    k = cen[z] + np.float32(w.sigma) * rng.standard_normal((T, w.d), dtype=np.float32)
    return k


def unit_kv(w: Workload, b: int, kvh: int, T: int | None = None):
    """Keys and values of one (batch entry, KV head): float32 [T, d] arrays
    holding cache-dtype values (already rounded to bf16 where needed)."""
    T = w.T if T is None else T
    rk = _unit_rng(w, b, kvh, "keys")
    rv = _unit_rng(w, b, kvh, "values")
    if w.zero_variance:
        nch = (T + w.chunk - 1) // w.chunk
        npair = w.clusters[0]
        pk = _mixture_keys(w, rk, nch * npair).reshape(nch, npair, w.d)
        pv = rv.standard_normal((nch, npair, w.d), dtype=np.float32)
        pick = rk.integers(0, npair, size=(nch, w.chunk))
        K = np.take_along_axis(pk, pick[:, :, None], axis=1).reshape(-1, w.d)[:T]
        V = np.take_along_axis(pv, pick[:, :, None], axis=1).reshape(-1, w.d)[:T]
        K = np.ascontiguousarray(K)
        V = np.ascontiguousarray(V)
    else:
        K = _mixture_keys(w, rk, T)
        if w.n_outliers:
            ro = _unit_rng(w, b, kvh, "outliers")
            ch = ro.choice(w.d, size=w.n_outliers, replace=False)
            sg = ro.choice(np.array([-1.0, 1.0], dtype=np.float32), size=w.n_outliers)
            K[:, ch] += np.float32(w.outlier_mag) * sg
        if w.rope_theta:
            K = _rope(K, w.rope_theta)
        V = rv.standard_normal((T, w.d), dtype=np.float32)
    return to_cache_values(w, K), to_cache_values(w, V)


def unit_queries(w: Workload, b: int, kvh: int, n_pos: int = 1, stream: str = "queries"):
    """Queries of the g query heads of one KV head: float32 [g, n_pos, d]
    (cache-dtype values), N(0, 1) / 8."""
    r = _unit_rng(w, b, kvh, stream)
    q = r.standard_normal((w.g, n_pos, w.d), dtype=np.float32) / np.float32(8.0)
    return to_cache_values(w, q)


def to_cache_values(w: Workload, a: np.ndarray) -> np.ndarray:
    if w.dtype == "f32":
        return np.ascontiguousarray(a, dtype=np.float32)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.to(torch.float32).numpy()


def kv_cache(w: Workload, T: int | None = None, threads: int = 8):
    """The whole KV cache as torch CPU tensors [B, Hkv, T, d] in the cache dtype."""
    T = w.T if T is None else T
    K = torch.empty((w.B, w.Hkv, T, w.d), dtype=w.torch_dtype)
    V = torch.empty_like(K)

    def fill(u):
        b, h = divmod(u, w.Hkv)
        k, v = unit_kv(w, b, h, T)
        K[b, h] = torch.from_numpy(k).to(w.torch_dtype)
        V[b, h] = torch.from_numpy(v).to(w.torch_dtype)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(fill, range(w.B * w.Hkv)))
    return K, V


def kv_cache_device(w: Workload, device, T: int | None = None):
    """The KV cache [B, Hkv, T, d] (cache dtype) generated on `device` with
    the same recipe as unit_kv (unit-norm Gaussian centres, key = centre +
    sigma N(0, I), seeded outlier channels before RoPE, N(0, 1) values) from
    seeded torch generators instead of numpy: for contexts whose host
    generation would take minutes.  Deterministic for (w, device type)."""
    T = w.T if T is None else T
    K = torch.empty((w.B, w.Hkv, T, w.d), dtype=w.torch_dtype, device=device)
    V = torch.empty_like(K)
    h2 = w.d // 2
    inv = w.rope_theta ** (-2.0 * torch.arange(h2, dtype=torch.float64, device=device) / w.d)
    step = 65536
    for b in range(w.B):
        for h in range(w.Hkv):
            tag = zlib.crc32(("%s/%d/%d" % (w.name, b, h + w.kvh0)).encode())
            g = torch.Generator(device=device).manual_seed((w.seed << 32) ^ tag)
            cen = torch.randn((w.n_centers, w.d), generator=g, device=device)
            cen /= cen.norm(dim=1, keepdim=True)
            ch = torch.randperm(w.d, generator=g, device=device)[:w.n_outliers]
            sg = torch.randint(0, 2, (w.n_outliers,), generator=g, device=device).float() * 2 - 1
            for t0 in range(0, T, step):
                n = min(step, T - t0)
                z = torch.randint(0, w.n_centers, (n,), generator=g, device=device)
                k = cen[z] + w.sigma * torch.randn((n, w.d), generator=g, device=device)
                if w.n_outliers:
                    k[:, ch] += w.outlier_mag * sg
                if w.rope_theta:
                    ang = torch.arange(t0, t0 + n, dtype=torch.float64, device=device)[:, None] * inv[None, :]
                    c, s = torch.cos(ang).float(), torch.sin(ang).float()
                    k = torch.cat([k[:, :h2] * c - k[:, h2:] * s, k[:, h2:] * c + k[:, :h2] * s], dim=1)
                K[b, h, t0:t0 + n] = k.to(w.torch_dtype)
                V[b, h, t0:t0 + n] = torch.randn((n, w.d), generator=g, device=device).to(w.torch_dtype)
    return K, V


def decode_queries(w: Workload, stream: str = "queries"):
    """Decode queries as a torch CPU tensor [B, Hq, d] in the cache dtype."""
    q = torch.empty((w.B, w.Hq, w.d), dtype=w.torch_dtype)
    for b in range(w.B):
        for h in range(w.Hkv):
            q[b, h * w.g:(h + 1) * w.g] = torch.from_numpy(
                unit_queries(w, b, h, 1, stream)[:, 0]).to(w.torch_dtype)
    return q


def prefill_queries(w: Workload, q_begin: int, Tq: int, stream: str = "queries"):
    """Prefill queries [B, Hq, Tq, d] (torch CPU, cache dtype) for positions
    [q_begin, q_begin + Tq).  Drawn per position block so any window of
    positions is reproducible on its own."""
    q = torch.empty((w.B, w.Hq, Tq, w.d), dtype=w.torch_dtype)
    for b in range(w.B):
        for h in range(w.Hkv):
            q[b, h * w.g:(h + 1) * w.g] = torch.from_numpy(
                unit_queries(w, b, h, q_begin + Tq, stream)[:, q_begin:]).to(w.torch_dtype)
    return q
