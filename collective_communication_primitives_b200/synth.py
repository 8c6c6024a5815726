"""Seeded synthetic inputs for the collectives, shared by the tests, the smoke check and the bench.

This module holds no collective arithmetic: it only turns (seed, stream label, element index) into
numbers. Both the oracle side and the CUDA side receive the same arrays from here.

Generator (counter based, so any element can be drawn alone):
  key  = splitmix64(seed * 2^32 + crc32(label))
  z(i) = splitmix64(key + (i + 1) * 0x9E3779B97F4A7C15)         (all uint64, wrapping)
where splitmix64 is the output mix of Steele, Lea and Flood's SplitMix64 generator. From z:
  uniform integers in [lo, hi]:  lo + z mod (hi - lo + 1)
  uniform fp32 in [-1, 1):        (z >> 40) * 2^-23 - 1            (exact in fp32)
  N(0, sigma):                    Box-Muller, u1 = ((z(2i) >> 11) + 1) * 2^-53,
                                  u2 = (z(2i+1) >> 11) * 2^-53, x = sigma * sqrt(-2 ln u1) cos(2 pi u2)
                                  in float64, rounded to fp32, then to bf16 (both ties-to-even).
"""
import os
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z):
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(label: str, seed: int = 0) -> np.uint64:
    with np.errstate(over="ignore"):
        base = np.uint64((seed << 32) + zlib.crc32(label.encode()))
        return _mix(np.array([base], dtype=np.uint64))[0]


def _z(key, start, count):
    """z(i) for i in [start, start + count)."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(key + i * _GOLDEN)


def _threads():
    return max(1, min(32, os.cpu_count() or 1))


def _fill(out, fn):
    """Fill a 1-D array chunk by chunk, in parallel (numpy releases the GIL in its loops)."""
    n = out.size
    starts = list(range(0, n, _CHUNK))

    def work(s):
        e = min(n, s + _CHUNK)
        out[s:e] = fn(s, e - s)

    if len(starts) <= 1:
        for s in starts:
            work(s)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, starts))
    return out


def ints(label, n, lo, hi, seed=0):
    """Uniform integers in [lo, hi] as int32."""
    key = stream_key(label, seed)
    span = np.uint64(hi - lo + 1)
    out = np.empty(n, dtype=np.int32)
    return _fill(out, lambda s, c: (np.int64(lo) + (_z(key, s, c) % span).astype(np.int64)).astype(np.int32))


def uniform_pm1(label, n, seed=0):
    """Uniform fp32 in [-1, 1) on the 2^-23 grid."""
    key = stream_key(label, seed)
    out = np.empty(n, dtype=np.float32)
    return _fill(out, lambda s, c: ((_z(key, s, c) >> np.uint64(40)).astype(np.float64) * 2.0**-23 - 1.0)
                 .astype(np.float32))


def _normal64(key, s, c, sigma):
    z = _z(key, 2 * s, 2 * c)
    u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0**-53
    u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * 2.0**-53
    return sigma * np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def fp32_to_bf16_bits(x):
    """fp32 -> bf16 bit patterns, round to nearest with ties to even on the dropped 16 bits.
    (The generator never produces NaN, so no NaN case is needed.)"""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def normal(label, n, sigma, dtype="fp32", seed=0):
    """N(0, sigma) as fp32, or as bf16 bit patterns (uint16) when dtype == 'bf16'."""
    key = stream_key(label, seed)
    f32 = np.empty(n, dtype=np.float32)
    _fill(f32, lambda s, c: _normal64(key, s, c, sigma).astype(np.float32))
    if dtype == "fp32":
        return f32
    if dtype == "bf16":
        out = np.empty(n, dtype=np.uint16)
        return _fill(out, lambda s, c: fp32_to_bf16_bits(f32[s:s + c]))
    raise ValueError(dtype)


def uniform01(label, n, seed=0):
    """Uniform float64 in [0, 1) with 53 random bits."""
    key = stream_key(label, seed)
    return (_z(key, 0, n) >> np.uint64(11)).astype(np.float64) * 2.0**-53


def moe_routes(p=8, tokens=8192, experts=64, topk=2, zipf_s=1.1, seed=0):
    """Router output of a top-k MoE layer: expert ids, int32 array [p][tokens][topk].

    Every source rank routes ``tokens`` tokens; each picks ``topk`` distinct experts, the first with
    probability w_e ∝ (e+1)^-s, each next one from w renormalised without the experts already
    picked. Expert e lives on rank e // (experts / p), so rank 0 holds the most popular experts.
    """
    if experts % p:
        raise ValueError("experts must split evenly over ranks")
    w = (np.arange(experts, dtype=np.float64) + 1.0) ** (-zipf_s)
    routes = np.zeros((p, tokens, topk), dtype=np.int32)
    for i in range(p):
        u = uniform01(f"moe.route.rank{i}", tokens * topk, seed).reshape(tokens, topk)
        avail = np.ones((tokens, experts), dtype=bool)
        for k in range(topk):
            wk = np.where(avail, w[None, :], 0.0)
            cdf = np.cumsum(wk, axis=1)
            target = u[:, k] * cdf[:, -1]
            e = (cdf <= target[:, None]).sum(axis=1)
            e = np.minimum(e, experts - 1)
            # never land on an expert already taken (zero weight) because of float ties
            taken = ~avail[np.arange(tokens), e]
            if taken.any():
                for t in np.nonzero(taken)[0]:
                    cand = np.nonzero(avail[t])[0]
                    e[t] = cand[np.searchsorted(cdf[t, cand], target[t], side="right").clip(max=len(cand) - 1)]
            avail[np.arange(tokens), e] = False
            routes[i, :, k] = e
    return routes


def moe_counts(p=8, tokens=8192, experts=64, topk=2, zipf_s=1.1, hidden=4096, seed=0):
    """Send-count matrix c[i][j] (elements) of a top-k MoE dispatch: the assignments of
    :func:`moe_routes` counted per destination rank, ``hidden`` elements per assignment."""
    routes = moe_routes(p, tokens, experts, topk, zipf_s, seed)
    per_rank = experts // p
    counts = np.zeros((p, p), dtype=np.int64)
    for i in range(p):
        counts[i] = np.bincount(routes[i].ravel() // per_rank, minlength=p)
    return counts * hidden


def moe_gate_weights(p=8, tokens=8192, topk=2, seed=0):
    """Gate weights of the router output, fp32 [p][tokens][topk]: positive, each token's summing to 1
    (up to fp32 rounding)."""
    out = np.zeros((p, tokens, topk), dtype=np.float32)
    for i in range(p):
        u = 0.05 + uniform01(f"moe.gate.rank{i}", tokens * topk, seed).reshape(tokens, topk)
        out[i] = (u / u.sum(axis=1, keepdims=True)).astype(np.float32)
    return out


def count_matrix_stats(counts):
    """Diagnostics of a send/recv count matrix: max row, max column, zero fraction."""
    c = np.asarray(counts)
    return {"max_row": int(c.sum(axis=1).max()), "max_col": int(c.sum(axis=0).max()),
            "zero_fraction": float((c == 0).mean())}
