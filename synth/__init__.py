"""Seeded synthetic inputs for the nanochat decoder step.

This module is shared by the fp64 oracle tests, the CUDA parity tests and the
bench.  It holds none of the model's arithmetic: only a counter-based random
stream (SplitMix64), normal and Zipf draws, the initialisation scheme of the
weights, bf16 rounding of the drawn values, and the five workload recipes.

The stand-in data: the pages train on FineWeb-EDU tokenised with a 65,536-entry
BPE vocabulary at a 2,048-token context (nanochat pages: "Five training stages"
and "1. Tokenizer").  Neither the dataset nor the tokenizer is available, so
token ids are drawn iid, either uniform or Zipf(1.1) (the usual heavy head of
natural-language token frequencies), with targets = tokens shifted by one.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

# tags that separate the random streams of one seed
TAG_TOKENS = 1
TAG_WEIGHTS = 1000


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function (Steele, Lea & Flood, OOPSLA 2014)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_base(seed: int, tag: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([(seed * 0x9E3779B97F4A7C15 + tag) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
        return _mix64(s)[0]


def splitmix64(seed: int, tag: int, n: int, offset: int = 0) -> np.ndarray:
    """Values offset..offset+n-1 of the SplitMix64 sequence started at the
    state derived from (seed, tag): x_i = mix(base + (i+1)*gamma)."""
    base = _stream_base(seed, tag)
    out = np.empty(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for lo in range(0, n, _CHUNK):
            hi = min(n, lo + _CHUNK)
            i = np.arange(offset + lo + 1, offset + hi + 1, dtype=np.uint64)
            out[lo:hi] = _mix64(base + i * GAMMA)
    return out


def uniform01(seed: int, tag: int, n: int) -> np.ndarray:
    """n doubles in [0,1) from the top 53 bits of each SplitMix64 value."""
    z = splitmix64(seed, tag, n)
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


_WCHUNK = 1 << 20


def _normal_pairs(seed, tag, lo, hi):
    """Normals 2*lo .. 2*hi-1 of the stream (Box-Muller on uniform pairs lo..hi-1)."""
    z = splitmix64(seed, tag, 2 * (hi - lo), offset=2 * lo)
    u = (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    u1 = 1.0 - u[0::2]  # (0, 1]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * math.pi * u2
    out = np.empty(2 * (hi - lo))
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out


def normal(seed: int, tag: int, n: int) -> np.ndarray:
    """n standard normals by Box-Muller, two per pair of uniforms.  Chunks are
    independent (counter-based stream), so they are filled by a thread pool;
    the values do not depend on the split."""
    m = (n + 1) // 2
    out = np.empty(2 * m, dtype=np.float64)
    spans = [(lo, min(m, lo + _CHUNK)) for lo in range(0, m, _CHUNK)]

    def fill(sp):
        out[2 * sp[0]:2 * sp[1]] = _normal_pairs(seed, tag, sp[0], sp[1])

    if len(spans) <= 1:
        for sp in spans:
            fill(sp)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(len(spans), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, spans))
    return out[:n]


def zipf_cdf(vocab: int, s: float = 1.1) -> np.ndarray:
    p = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(p)
    return c / c[-1]


def token_rows(seed: int, B: int, T: int, vocab: int, dist: str) -> tuple[np.ndarray, np.ndarray]:
    """B rows of T+1 iid ids; tokens = ids[:, :T], targets = ids[:, 1:]."""
    u = uniform01(seed, TAG_TOKENS, B * (T + 1))
    if dist == "uniform":
        ids = np.minimum((u * vocab).astype(np.int64), vocab - 1)
    elif dist == "zipf":
        ids = np.searchsorted(zipf_cdf(vocab), u, side="right")
        ids = np.minimum(ids, vocab - 1)
    else:
        raise ValueError(dist)
    ids = ids.astype(np.int32).reshape(B, T + 1)
    return np.ascontiguousarray(ids[:, :T]), np.ascontiguousarray(ids[:, 1:])


# ---------------------------------------------------------------------------
# bf16 storage: round-to-nearest-even of the fp32 value, kept as raw bits.

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    nan = (b & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    rounded = np.where(nan, b | np.uint32(0x00400000), rounded)
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# weights: the initialisation scheme of the workloads

def init_std(name: str, rows: int, cols: int) -> float:
    """Std of the N(0, std) draw of one weight tensor: the token embedding 1,
    the unembedding 0.001, every other matrix 1/sqrt(fan_in)."""
    if name == "wte":
        return 1.0
    if name == "lm_head":
        return 0.001
    return 1.0 / math.sqrt(cols)


def make_weights(layout, seed: int, dtype: str, std_override: dict | None = None, want_f64: bool = True,
                 values: dict | None = None):
    """Draw every tensor of `layout` (a list of (name, rows, cols)).

    Returns (flat, f64) where `flat` is the storage a device buffer receives
    (float32, or uint16 bf16 bits) in layout order, and `f64` maps each name to
    the float64 value of exactly what was stored (empty if not want_f64).
    Work is split into independent (tensor, chunk) jobs run by a thread pool;
    every element is computed the same way whatever the split.  `values`
    maps a tensor name to fixed values (an array of its shape) stored instead
    of a draw, rounded like the draws.
    """
    from concurrent.futures import ThreadPoolExecutor
    std_override = std_override or {}
    total = sum(r * c for _, r, c in layout)
    flat = np.empty(total, dtype=np.float32 if dtype == "f32" else np.uint16)
    f64 = {name: np.empty((rows, cols)) for name, rows, cols in layout} if want_f64 else {}
    jobs = []
    off = 0
    for i, (name, rows, cols) in enumerate(layout):
        n = rows * cols
        m = (n + 1) // 2
        for lo in range(0, m, _WCHUNK):
            jobs.append((i, name, off, n, lo, min(m, lo + _WCHUNK), std_override.get(name, init_std(name, rows, cols))))
        off += n

    def run(job):
        i, name, base, n, lo, hi, std = job
        tmp = _normal_pairs(seed, TAG_WEIGHTS + i, lo, hi)
        a, b = 2 * lo, min(n, 2 * hi)
        w32 = (tmp[:b - a] * std).astype(np.float32)
        if dtype == "f32":
            flat[base + a:base + b] = w32
            if want_f64:
                f64[name].reshape(-1)[a:b] = w32
        else:
            bits = f32_to_bf16_bits(w32)
            flat[base + a:base + b] = bits
            if want_f64:
                f64[name].reshape(-1)[a:b] = bf16_bits_to_f64(bits)

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(run, jobs))
    off = 0
    for name, rows, cols in layout:
        n = rows * cols
        if values and name in values:
            w32 = np.asarray(values[name], dtype=np.float64).reshape(-1).astype(np.float32)
            assert w32.size == n, name
            if dtype == "f32":
                flat[off:off + n] = w32
                if want_f64:
                    f64[name] = w32.astype(np.float64).reshape(rows, cols)
            else:
                bits = f32_to_bf16_bits(w32)
                flat[off:off + n] = bits
                if want_f64:
                    f64[name] = bf16_bits_to_f64(bits).reshape(rows, cols)
        off += n
    return flat, f64


def full_block_values(depth: int, n_ve: int, resid: float = 1.0, x0: float = 0.1, gate: float = 1.0) -> dict:
    """Values of the full block's scalars: the pages' initial resid_lambdas
    (1.0) and x0_lambdas (0.1); the value-embedding gate has no initial value
    on the pages (1.0 here)."""
    return {"resid_lambdas": np.full((1, depth), resid), "x0_lambdas": np.full((1, depth), x0),
            "ve_gates": np.full((1, n_ve), gate)}


# ---------------------------------------------------------------------------
# the five workloads

@dataclass(frozen=True)
class Workload:
    name: str
    depth: int
    B: int
    T: int
    dtype: str  # "f32" or "bf16"
    tokens: str  # "uniform" or "zipf"
    seed: int
    vocab: int = 65536
    seq: int = 2048


WORKLOADS = {
    "d4": Workload("d4", 4, 2, 256, "f32", "uniform", 0),
    "d12": Workload("d12", 12, 8, 1024, "bf16", "zipf", 1),
    "d20": Workload("d20", 20, 16, 2048, "bf16", "zipf", 2),
    "d24": Workload("d24", 24, 8, 2048, "bf16", "zipf", 3),
    "d32": Workload("d32", 32, 4, 2048, "bf16", "zipf", 4),
}
