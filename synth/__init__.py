"""Seeded synthetic inputs for the MSA hot path, bit-identical on the host and on the device.

This module holds no part of the attention method's arithmetic. It only draws random
numbers, rounds them to bf16, and builds the planted-block structure of the 32K workload.
Both the CPU oracle (through numpy arrays) and the CUDA library (through torch device
tensors) take their inputs from here.

Generator
---------
SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014) run in counter mode. Element ``i`` of stream ``s`` under seed ``S`` is

    mix64(key(S, s) + (i + 1) * GAMMA)        (all arithmetic mod 2**64)
    key(S, s) = mix64(S + (s + 1) * GAMMA2)

where ``mix64`` is SplitMix64's output finaliser. The top 18 bits of that word pick one
of 2**18 equiprobable buckets of the standard normal distribution; the value is the
bucket's midpoint quantile rounded to bf16 (round to nearest, ties to even). The quantile
table is computed once on the host (``scipy.special.ndtri``) and copied to the device, and
everything else is integer arithmetic, so the host (numpy) and device (torch) generators
return the same bits. The distribution is N(0,1) discretised to 2**18 quantiles, which is
finer than bf16 resolution over the body; the tails are cut at +-4.62 sigma (mass 4e-6).

Element indices are row-major offsets into each tensor's *logical* shape (documented in
``Workload``), never into a padded device allocation, so any subset of a tensor can be
regenerated on the host for sampled checks.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
GAMMA2 = 0xD1B54A32D192ED03
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
TABLE_BITS = 18

# stream ids
STREAM_Q, STREAM_K, STREAM_V, STREAM_QI, STREAM_KI, STREAM_PLANT = 0, 1, 2, 3, 4, 5


def _mix64_int(z: int) -> int:
    z &= M64
    z = ((z ^ (z >> 30)) * MIX1) & M64
    z = ((z ^ (z >> 27)) * MIX2) & M64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    return _mix64_int(seed + (stream + 1) * GAMMA2)


# --------------------------------------------------------------------------- bf16 helpers
def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values (finite, normal range) to bf16, nearest-even, as uint16 bits."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    r = np.round(m * 256.0)                  # numpy rounds half to even
    y = np.ldexp(r / 256.0, e).astype(np.float32)   # exact: 8 significant bits
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values (finite) to bf16, nearest-even, as uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


_TABLE: Optional[np.ndarray] = None


def normal_table() -> np.ndarray:
    """2**18 bf16 bit patterns: N(0,1) quantiles at bucket midpoints."""
    global _TABLE
    if _TABLE is None:
        import scipy.special
        k = np.arange(1 << TABLE_BITS, dtype=np.float64)
        _TABLE = f64_to_bf16_bits(scipy.special.ndtri((k + 0.5) / float(1 << TABLE_BITS)))
    return _TABLE


# --------------------------------------------------------------------------- host generator
def raw_u64(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """SplitMix64 words for element indices ``idx`` (any integer array) of one stream."""
    idx = np.asarray(idx, dtype=np.uint64)
    z = np.uint64(stream_key(seed, stream)) + (idx + np.uint64(1)) * np.uint64(GAMMA)
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
    return z ^ (z >> np.uint64(31))


def normal_bf16_at(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """bf16 bits (uint16) of the elements at flat indices ``idx``."""
    with np.errstate(over="ignore"):
        z = raw_u64(seed, stream, idx)
    return normal_table()[(z >> np.uint64(64 - TABLE_BITS)).astype(np.int64)]


def normal_bf16(seed: int, stream: int, shape: Sequence[int], start: int = 0) -> np.ndarray:
    """A whole tensor of bf16 bits: element with row-major offset i uses counter start + i.
    Large tensors are generated in 4M-element chunks on a thread pool (numpy releases the
    interpreter lock inside its array operations); the result does not depend on it."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    step = 1 << 22

    def fill(lo):
        hi = min(n, lo + step)
        out[lo:hi] = normal_bf16_at(seed, stream, np.arange(start + lo, start + hi, dtype=np.uint64))

    chunks = list(range(0, n, step))
    if len(chunks) > 1:
        import concurrent.futures
        import os
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(chunks), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, chunks))
    elif chunks:
        fill(0)
    return out.reshape(shape)


# --------------------------------------------------------------------------- device generator
def _i64(u: int) -> int:
    u &= M64
    return u - (1 << 64) if u >= (1 << 63) else u


_DEV_TABLES = {}


def _device_table(device):
    import torch
    key = str(device)
    if key not in _DEV_TABLES:
        _DEV_TABLES[key] = torch.from_numpy(normal_table().view(np.int16).copy()).to(device)
    return _DEV_TABLES[key]


def _srl(z, s: int):
    """Logical right shift of int64 tensors holding uint64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def normal_bf16_torch(seed: int, stream: int, n: int, device, start: int = 0, out=None):
    """Device tensor (torch.bfloat16, flat, length n) equal bit for bit to ``normal_bf16``."""
    import torch
    table = _device_table(device)
    if out is None:
        out = torch.empty(n, dtype=torch.bfloat16, device=device)
    out16 = out.view(torch.int16)
    key = _i64(stream_key(seed, stream))
    g, m1, m2 = _i64(GAMMA), _i64(MIX1), _i64(MIX2)
    step = 1 << 25
    for lo in range(0, n, step):
        hi = min(n, lo + step)
        z = torch.arange(start + lo + 1, start + hi + 1, dtype=torch.int64, device=device)
        z = z * g + key
        z = (z ^ _srl(z, 30)) * m1
        z = (z ^ _srl(z, 27)) * m2
        z = z ^ _srl(z, 31)
        out16[lo:hi] = table[_srl(z, 64 - TABLE_BITS)]
    return out


# --------------------------------------------------------------------------- workloads
@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload. Logical tensor shapes (row-major element indices):

    prefill: q [B,N,Hq,d] (stream 0), k [B,G,N,d] (1), v [B,G,N,d] (2),
             q_I [B,N,G,dI] (3), k_I [B,N,G,dI] (4); planted blocks use stream 5.
    decode:  sequence b uses seed + 16*b and has L = ctx[b] + 1 tokens (the new one last):
             k, v [G,L,d] (1, 2), k_I [L,G,dI] (4), q [Hq,d] (0), q_I [G,dI] (3).
    """
    name: str
    kind: str                      # "prefill" | "decode"
    B: int
    Hq: int
    G: int
    N: int = 0                     # prefill length
    ctx: tuple = ()                # decode: tokens already cached per sequence (L_b)
    d: int = 128
    dI: int = 64
    Bk: int = 128
    topk: int = 16
    seed: int = 0
    planted: int = 0               # planted high-affinity blocks per group (prefill)

    @property
    def Hg(self) -> int:
        return self.Hq // self.G


def _cfg(i: int, **kw) -> Workload:
    return Workload(seed=0x4D5341 + i, **kw)


WORKLOADS = {
    # prefill, 4K tokens, one GQA group of 4 query heads
    "prefill_4k_h4g1": _cfg(1, name="prefill_4k_h4g1", kind="prefill", B=1, N=4096, Hq=4, G=1),
    # prefill, 32K tokens, 64/8 heads, 16 planted high-affinity blocks per group
    "prefill_32k_h64g8_planted": _cfg(2, name="prefill_32k_h64g8_planted", kind="prefill", B=1,
                                      N=32768, Hq=64, G=8, planted=16),
    # prefill, 128K tokens, 64/8 heads
    "prefill_128k_h64g8": _cfg(3, name="prefill_128k_h64g8", kind="prefill", B=1, N=131072,
                               Hq=64, G=8),
    # decode step, batch 16 at 128K context
    "decode_128k_b16_h64g8": _cfg(4, name="decode_128k_b16_h64g8", kind="decode", B=16, Hq=64,
                                  G=8, ctx=(131072,) * 16),
    # decode step, ragged batch of 4 up to 1M context
    "decode_1m_ragged_b4_h64g8": _cfg(5, name="decode_1m_ragged_b4_h64g8", kind="decode", B=4,
                                      Hq=64, G=8, ctx=(1048576, 524288, 262144, 65536)),
}


def seq_seed(w: Workload, b: int) -> int:
    return w.seed + 16 * b


# --------------------------------------------------------------------------- planting (32K)
def planted_blocks(w: Workload, b: int, g: int, nb: int) -> np.ndarray:
    """w.planted distinct block ids drawn from [0, nb-1) by a seeded partial Fisher-Yates."""
    n = nb - 1
    a = np.arange(n, dtype=np.int64)
    base = (b * w.G + g) * 64
    with np.errstate(over="ignore"):
        z = raw_u64(w.seed, STREAM_PLANT, np.arange(base, base + w.planted, dtype=np.uint64))
    for i in range(w.planted):
        j = i + int(z[i] % np.uint64(n - i))
        a[i], a[j] = a[j], a[i]
    return np.sort(a[: w.planted])


def plant_shift(q_idx_bits: np.ndarray) -> np.ndarray:
    """Per (b, g): 2 * unit vector along the mean index query of the group, as float32.

    q_idx_bits: [B, N, G, dI] bf16 bits. Returns [B, G, dI] float32.
    """
    q = bf16_bits_to_f32(q_idx_bits).astype(np.float64)
    mu = q.mean(axis=1)                                    # [B, G, dI]
    mu /= np.linalg.norm(mu, axis=-1, keepdims=True)
    return (2.0 * mu).astype(np.float32)


def apply_plant_np(k_idx_bits: np.ndarray, shift: np.ndarray, blocks: dict, Bk: int) -> np.ndarray:
    """k_I[b, t, g] <- bf16(f32(k_I) + shift[b, g]) for t in the planted blocks of (b, g)."""
    out = k_idx_bits.copy()
    for (b, g), blks in blocks.items():
        for j in blks:
            rows = bf16_bits_to_f32(out[b, j * Bk:(j + 1) * Bk, g, :]) + shift[b, g][None, :]
            out[b, j * Bk:(j + 1) * Bk, g, :] = f32_to_bf16_bits(rows.astype(np.float32))
    return out


def plant_plan(w: Workload, q_idx_bits: np.ndarray):
    """(shift [B,G,dI] f32, {(b,g): block ids}) for a planted prefill workload."""
    nb = w.N // w.Bk
    shift = plant_shift(q_idx_bits)
    blocks = {(b, g): planted_blocks(w, b, g, nb) for b in range(w.B) for g in range(w.G)}
    return shift, blocks


# --------------------------------------------------------------------------- whole workloads
def prefill_inputs_np(w: Workload) -> dict:
    """All prefill tensors as host bf16 bit arrays (small workloads only)."""
    assert w.kind == "prefill"
    x = {
        "q": normal_bf16(w.seed, STREAM_Q, (w.B, w.N, w.Hq, w.d)),
        "k": normal_bf16(w.seed, STREAM_K, (w.B, w.G, w.N, w.d)),
        "v": normal_bf16(w.seed, STREAM_V, (w.B, w.G, w.N, w.d)),
        "q_idx": normal_bf16(w.seed, STREAM_QI, (w.B, w.N, w.G, w.dI)),
        "k_idx": normal_bf16(w.seed, STREAM_KI, (w.B, w.N, w.G, w.dI)),
    }
    if w.planted:
        shift, blocks = plant_plan(w, x["q_idx"])
        x["k_idx"] = apply_plant_np(x["k_idx"], shift, blocks, w.Bk)
    return x


def prefill_inputs_torch(w: Workload, device) -> dict:
    """All prefill tensors generated on ``device`` (torch.bfloat16), equal to the host ones."""
    import torch
    shapes = {
        "q": (STREAM_Q, (w.B, w.N, w.Hq, w.d)),
        "k": (STREAM_K, (w.B, w.G, w.N, w.d)),
        "v": (STREAM_V, (w.B, w.G, w.N, w.d)),
        "q_idx": (STREAM_QI, (w.B, w.N, w.G, w.dI)),
        "k_idx": (STREAM_KI, (w.B, w.N, w.G, w.dI)),
    }
    x = {}
    for name, (s, shp) in shapes.items():
        x[name] = normal_bf16_torch(w.seed, s, int(np.prod(shp)), device).view(shp)
    if w.planted:
        qi_host = normal_bf16(w.seed, STREAM_QI, (w.B, w.N, w.G, w.dI))
        shift, blocks = plant_plan(w, qi_host)
        kt = x["k_idx"]
        for (b, g), blks in blocks.items():
            sh = torch.from_numpy(shift[b, g]).to(device)
            for j in blks:
                rows = kt[b, j * w.Bk:(j + 1) * w.Bk, g, :].float() + sh[None, :]
                kt[b, j * w.Bk:(j + 1) * w.Bk, g, :] = f32_to_bf16_torch(rows)
    return x


def f32_to_bf16_torch(x):
    """Round-to-nearest-even float32 -> bfloat16 with integer ops (matches f32_to_bf16_bits)."""
    import torch
    u = x.contiguous().view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    u = torch.where(u >= 0x8000, u - 0x10000, u)
    return u.to(torch.int16).view(torch.bfloat16)


def decode_seq_np(w: Workload, b: int, what: str, pos_lo: int = 0, pos_hi: Optional[int] = None,
                  g: Optional[int] = None) -> np.ndarray:
    """Host bits of one decode sequence's tensor, optionally restricted to a position range
    and/or one group. what in {"k", "v", "k_idx", "q", "q_idx"}."""
    L = w.ctx[b] + 1
    s = seq_seed(w, b)
    if pos_hi is None:
        pos_hi = L
    if what in ("k", "v"):
        stream = STREAM_K if what == "k" else STREAM_V
        groups = range(w.G) if g is None else [g]
        out = []
        for gg in groups:
            start = (gg * L + pos_lo) * w.d
            out.append(normal_bf16(s, stream, (pos_hi - pos_lo, w.d), start=start))
        return np.stack(out) if g is None else out[0]
    if what == "k_idx":
        pos = np.arange(pos_lo, pos_hi, dtype=np.uint64)
        if g is None:                    # whole rows: a contiguous range of counters
            return normal_bf16(s, STREAM_KI, (pos_hi - pos_lo, w.G, w.dI), start=pos_lo * w.G * w.dI)
        else:
            idx = (pos[:, None] * np.uint64(w.G) + np.uint64(g)) * np.uint64(w.dI) \
                + np.arange(w.dI, dtype=np.uint64)[None, :]
        return normal_bf16_at(s, STREAM_KI, idx)
    if what == "q":
        return normal_bf16(s, STREAM_Q, (w.Hq, w.d))
    if what == "q_idx":
        return normal_bf16(s, STREAM_QI, (w.G, w.dI))
    raise ValueError(what)


def decode_seq_torch(w: Workload, b: int, what: str, device):
    """Device tensor of one decode sequence's whole tensor (logical shape, see Workload)."""
    L = w.ctx[b] + 1
    s = seq_seed(w, b)
    shape = {"k": (w.G, L, w.d), "v": (w.G, L, w.d), "k_idx": (L, w.G, w.dI),
             "q": (w.Hq, w.d), "q_idx": (w.G, w.dI)}[what]
    stream = {"k": STREAM_K, "v": STREAM_V, "k_idx": STREAM_KI, "q": STREAM_Q,
              "q_idx": STREAM_QI}[what]
    return normal_bf16_torch(s, stream, int(np.prod(shape)), device).view(shape)


def small_workload(kind="prefill", **kw) -> Workload:
    """Ad-hoc workload for tests (seeded, with the same stream conventions)."""
    base = dict(name="adhoc", kind=kind, B=1, Hq=4, G=1, seed=12345)
    base.update(kw)
    return Workload(**base)
