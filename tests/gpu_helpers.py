"""Shared helpers of the GPU parity tests: tensors with guard bands, dtype conversions, tolerances."""
import math

import numpy as np
import torch

from collective_communication_primitives_b200 import synth as S

GUARD = 1024              # elements of guard band on each side of every device buffer
SENT = {"int32": np.int32(-0x5A5A5A5B), "fp32": np.float32(-7.0e33), "bf16": np.uint16(0xFEFE)}
TORCH = {"int32": torch.int32, "fp32": torch.float32, "bf16": torch.bfloat16}
U = 2.0 ** -24


def to_torch(a, dtype, device="cuda"):
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16) if dtype == "bf16" else a)
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.to(device)


def to_numpy(t, dtype):
    t = t.detach().cpu()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


class Guarded:
    """A device buffer of n elements with sentinel-filled guard bands on both sides."""

    def __init__(self, n, dtype, offset=0, fill=None):
        self.n, self.dtype, self.offset = n, dtype, offset
        host = np.full(GUARD * 2 + n + offset, SENT[dtype])
        if fill is not None:
            host[GUARD + offset:GUARD + offset + n] = fill
        self.full = to_torch(host, dtype)
        self.t = self.full[GUARD + offset:GUARD + offset + n]

    def guards_intact(self):
        h = to_numpy(self.full, self.dtype)
        s = SENT[self.dtype]
        head = h[:GUARD + self.offset]
        tail = h[GUARD + self.offset + self.n:]
        return np.array_equal(head, np.full(head.shape, s)) and np.array_equal(tail, np.full(tail.shape, s))

    def numpy(self):
        return to_numpy(self.t, self.dtype)


def make_inputs(kind, p, n, dtype, label, seed=0, sigma=1.0):
    """Per-rank host arrays: 'int8' uniform integers in [-8, 8]; 'int24' in [-2^24, 2^24];
    'normal' N(0, sigma); 'pm1' uniform(-1, 1)."""
    out = []
    for r in range(p):
        lab = f"{label}.rank{r}"
        if kind == "int8":
            v = S.ints(lab, n, -8, 8, seed)
        elif kind == "int24":
            v = S.ints(lab, n, -2**24, 2**24, seed)
        elif kind == "normal":
            v = S.normal(lab, n, sigma, "bf16" if dtype == "bf16" else "fp32", seed)
            out.append(v if dtype != "int32" else v.astype(np.int32))
            continue
        elif kind == "pm1":
            v = S.uniform_pm1(lab, n, seed)
        else:
            raise ValueError(kind)
        if dtype == "fp32":
            v = v.astype(np.float32)
        elif dtype == "bf16":
            v = S.fp32_to_bf16_bits(v.astype(np.float32))
        out.append(v)
    return out


def as_f64(a, dtype):
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def bf16_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 2.0 ** -133)))
    return 2.0 ** np.maximum(e - 7, -133)


def check_sum_tolerance(got, ins, dtype, op, p):
    """fp32: |got - exact| <= 2·p·2^-24·Σ_r|x_r| (AVG: that bound over p, plus 3 ulps of the mean);
    bf16 output: |got - exact| <= 1 bf16 ulp of the exact value."""
    vals = np.stack([as_f64(x, dtype) for x in ins])
    exact = vals.sum(axis=0)
    absum = np.abs(vals).sum(axis=0)
    if op == "avg":
        exact = exact / p
    g = as_f64(got, dtype)
    err = np.abs(g - exact)
    if dtype == "bf16":
        bound = bf16_ulp(exact)
    elif op == "avg":
        bound = 2 * p * U * absum / p + 3 * U * np.abs(exact)
    else:
        bound = 2 * p * U * absum
    bad = err > bound
    assert not bad.any(), f"{int(bad.sum())} elements outside the bound; worst {float((err - bound).max())}"
