"""Seeded synthetic workloads for the DART forward path.

This module is the one piece shared by the float64 oracle (``oracle/``) and the
CUDA library (``ssm_state_memory_b200``): it draws the inputs and rounds them to
the storage dtype, and it holds none of the method's arithmetic. Both sides
receive the *same rounded values*: the GPU gets the bf16/fp32 storage arrays,
the oracle gets the exact float64 upcast of those same values.

Workloads (shapes and value distributions follow the DART paper,
"DART: Decoded Attention over Recurrent States", §5.3 "Kernel Forward Time and
Inference Cache" for the bf16 / N=128 / P=64 / S=256 kernel setting, §4 eq (14)
for the decode cache, App. D.2 for the Mamba-2-370M shape):

* ``tiny_f32``      -- batch 1, 1 head, L=512, S=64, N=16, P=8, fp32, g=0.5.
* ``mixer_bf16``    -- batch 2, 8 heads, L=4096, S=256, N=128, P=64, bf16, g=1.
* ``m370m_bf16``    -- batch 4, 32 heads, L=8192, S=256, N=128, P=64, bf16,
                       per-head gate g ~ U[0,1] (d_model 1024, expand 2).
* ``long_bf16``     -- batch 1, 32 heads, L=65536, S=256, bf16, planted
                       key/value pairs, logA = -1e-3.
* ``decode_bf16``   -- batch 64, 32 heads, 256 cached chunk memories.

Random streams: numpy ``Generator(PCG64(seed))``, default seed 20260 + the
workload's index in the list above. The decode cache (4.3e9 bf16 values) is
drawn from a counter-based generator (SplitMix64 of Steele, Lea & Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014, summed as an
Irwin-Hall(4) variate) that is implemented twice, here in numpy and in
``workloads/csrc/gen.cu`` for the device, so that both sides see bit-identical
values without a host->device copy of 8.6 GB.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np

BASE_SEED = 20260

# ---------------------------------------------------------------------------
# dtype rounding (storage formats)
# ---------------------------------------------------------------------------


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the raw 16-bit patterns as uint16. Inputs must be finite.
    """
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Stored:
    """One input tensor: its storage array and the exact float64 of its values."""

    storage: np.ndarray  # float32, or uint16 bf16 bit patterns
    dtype: str  # "f32" | "bf16"

    @property
    def f64(self) -> np.ndarray:
        if self.dtype == "bf16":
            return bf16_bits_to_f32(self.storage).astype(np.float64)
        return self.storage.astype(np.float64)

    @property
    def shape(self):
        return self.storage.shape


def store(x: np.ndarray, dtype: str) -> Stored:
    """Round float64 draws once to the storage dtype (f64 -> f32 -> bf16 RNE)."""
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "bf16":
        return Stored(f32_to_bf16_bits(x32), "bf16")
    if dtype == "f32":
        return Stored(np.ascontiguousarray(x32), "f32")
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# workload descriptions
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class LayerWorkload:
    name: str
    index: int
    batch: int
    nheads: int
    ngroups: int
    seqlen: int
    chunk: int
    dstate: int
    headdim: int
    dtype: str
    logA: str  # "tiny" | "mamba2" | "const"
    gate: str  # "scalar:<v>" | "per_head_uniform"
    planted: bool = False

    @property
    def nchunks(self) -> int:
        return -(-self.seqlen // self.chunk)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def with_(self, **kw) -> "LayerWorkload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    index: int
    batch: int
    nheads: int
    ngroups: int
    n_chunks: int
    chunk: int
    dstate: int
    headdim: int
    dtype: str
    cache_sigma: float

    def with_(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


TINY_F32 = LayerWorkload("tiny_f32", 0, 1, 1, 1, 512, 64, 16, 8, "f32", "tiny", "scalar:0.5")
MIXER_BF16 = LayerWorkload("mixer_bf16", 1, 2, 8, 1, 4096, 256, 128, 64, "bf16", "mamba2", "scalar:1.0")
M370M_BF16 = LayerWorkload("m370m_bf16", 2, 4, 32, 1, 8192, 256, 128, 64, "bf16", "mamba2", "per_head_uniform")
LONG_BF16 = LayerWorkload("long_bf16", 3, 1, 32, 1, 65536, 256, 128, 64, "bf16", "const", "scalar:1.0",
                          planted=True)
# sigma of the cached chunk memories: the standard deviation of the chunk state memories
# that the mixer_bf16 distributions produce (about 0.027; checked in tests/test_workloads.py).
DECODE_BF16 = DecodeWorkload("decode_bf16", 4, 64, 32, 1, 256, 256, 128, 64, "bf16", cache_sigma=0.027)

LAYER_WORKLOADS = {w.name: w for w in (TINY_F32, MIXER_BF16, M370M_BF16, LONG_BF16)}
DECODE_WORKLOADS = {DECODE_BF16.name: DECODE_BF16}


# ---------------------------------------------------------------------------
# layer inputs
# ---------------------------------------------------------------------------


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def _gate(w: LayerWorkload, rng: np.random.Generator) -> Tuple[np.ndarray, Tuple[int, int, int]]:
    """Gate g as an fp32 array plus (stride_b, stride_t, stride_h) in elements (0 = broadcast)."""
    if w.gate.startswith("scalar:"):
        return np.array([float(w.gate.split(":", 1)[1])], dtype=np.float32), (0, 0, 0)
    if w.gate == "per_head_uniform":
        return rng.uniform(0.0, 1.0, size=(w.nheads,)).astype(np.float32), (0, 0, 1)
    if w.gate == "per_token":
        return rng.uniform(0.0, 1.0, size=(w.batch, w.seqlen, w.nheads)).astype(np.float32), (
            w.seqlen * w.nheads, w.nheads, 1)
    raise ValueError(w.gate)


def _logA(w: LayerWorkload, rng: np.random.Generator) -> np.ndarray:
    shape = (w.batch, w.seqlen, w.nheads)
    if w.logA == "tiny":
        return -_softplus(rng.standard_normal(shape)) * 0.1
    if w.logA == "mamba2":
        # Mamba-2 reading: one A per head (exp of U[-4,-1]), one dt per (b, t, h).
        a_head = np.exp(rng.uniform(-4.0, -1.0, size=(w.nheads,)))
        dt = _softplus(rng.standard_normal(shape) + 1.0)
        return -(a_head[None, None, :] * dt)
    if w.logA == "const":
        return np.full(shape, -1e-3)
    if w.logA == "zero":
        return np.zeros(shape)
    raise ValueError(w.logA)


def _plant_pairs(w: LayerWorkload, rng: np.random.Generator, X, B, Q, E) -> Dict[str, object]:
    """Planted recall pairs for the long-context workload (in place, float64).

    One early chunk c* ~ U{1..15}; 16 distinct positions s_k inside it. Each of the
    last 64 tokens t gets k = (t - (L-64)) mod 16 and has Q_t (and, per head, E_t)
    replaced by a vector of the same norm whose cosine with B_{s_k} (X_{s_k,h}) is 0.9.
    """
    S, L = w.chunk, w.seqlen
    c_star = int(rng.integers(1, min(16, w.nchunks)))
    pos = np.sort(rng.choice(S, size=16, replace=False)) + c_star * S
    last = np.arange(L - 64, L)

    def aligned(target: np.ndarray, old: np.ndarray) -> np.ndarray:
        t_hat = target / np.linalg.norm(target)
        z = rng.standard_normal(target.shape)
        z -= np.dot(z, t_hat) * t_hat
        z /= np.linalg.norm(z)
        return np.linalg.norm(old) * (0.9 * t_hat + math.sqrt(1.0 - 0.81) * z)

    for b in range(w.batch):
        for t in last:
            k = (t - (L - 64)) % 16
            s = pos[k]
            for gidx in range(w.ngroups):
                Q[b, t, gidx] = aligned(B[b, s, gidx], Q[b, t, gidx])
            for h in range(w.nheads):
                E[b, t, h] = aligned(X[b, s, h], E[b, t, h])
    return {"c_star": c_star, "positions": pos, "queries": last}


def make_layer_inputs(w: LayerWorkload, seed: Optional[int] = None) -> Dict[str, object]:
    """Seeded inputs of one layer-forward workload.

    Returns a dict with ``X, B, C, Q, E`` (``Stored``), ``logA`` (fp32 [b, L, H]),
    ``g`` (fp32) and ``g_strides`` (elements), plus ``plant`` metadata when planted.
    Layouts: X, E [b, L, H, P]; B, C, Q [b, L, G, N]; logA [b, L, H].
    """
    if seed is None:
        seed = BASE_SEED + w.index
    rng = np.random.Generator(np.random.PCG64(seed))
    Bt, L, H, G, N, P = w.batch, w.seqlen, w.nheads, w.ngroups, w.dstate, w.headdim
    X = rng.standard_normal((Bt, L, H, P)) / math.sqrt(P)
    Bm = rng.standard_normal((Bt, L, G, N)) / math.sqrt(N)
    C = rng.standard_normal((Bt, L, G, N)) / math.sqrt(N)
    Q = rng.standard_normal((Bt, L, G, N)) / math.sqrt(N)
    E = rng.standard_normal((Bt, L, H, P)) / math.sqrt(P)
    logA = _logA(w, rng).astype(np.float32)
    g, g_strides = _gate(w, rng)
    out: Dict[str, object] = {}
    if w.planted:
        out["plant"] = _plant_pairs(w, rng, X, Bm, Q, E)
    out.update(
        X=store(X, w.dtype), B=store(Bm, w.dtype), C=store(C, w.dtype), Q=store(Q, w.dtype),
        E=store(E, w.dtype), logA=np.ascontiguousarray(logA), g=g, g_strides=g_strides,
    )
    return out


def make_readout_grad(w: LayerWorkload, seed: Optional[int] = None) -> np.ndarray:
    """Seeded upstream gradient dLoss/dR for the SMA backward: fp32 [b, L, H, P], entries N(0, 1/P)
    (the scale of a gradient reaching a head's P outputs through a unit-variance projection)."""
    rng = np.random.default_rng(BASE_SEED + 5000 + w.index if seed is None else seed)
    dR = rng.standard_normal((w.batch, w.seqlen, w.nheads, w.headdim)) / np.sqrt(w.headdim)
    return dR.astype(np.float32)


def gate_dense(g: np.ndarray, g_strides, batch: int, seqlen: int, nheads: int) -> np.ndarray:
    """Expand a strided gate to a dense float64 [b, L, H] array (index arithmetic only)."""
    sb, st, sh = g_strides
    b = np.arange(batch)[:, None, None]
    t = np.arange(seqlen)[None, :, None]
    h = np.arange(nheads)[None, None, :]
    return g.reshape(-1)[b * sb + t * st + h * sh].astype(np.float64)


# ---------------------------------------------------------------------------
# counter-based generator (SplitMix64 -> Irwin-Hall(4)), numpy side
# ---------------------------------------------------------------------------

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(key: int, idx: np.ndarray) -> np.ndarray:
    """SplitMix64 output for counter values ``idx`` under stream ``key``.

    state = key + (idx + 1) * 0x9E3779B97F4A7C15 (mod 2^64), then the SplitMix64
    finaliser (xor-shift 30, multiply, xor-shift 27, multiply, xor-shift 31).
    """
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (idx.astype(np.uint64) + np.uint64(1)) * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


# standard deviation of the sum of four independent uniforms on {0..65535}
IRWIN_HALL_STD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)


def irwin_hall_bf16(key: int, start: int, count: int, sigma: float) -> np.ndarray:
    """bf16 bits of sigma-scaled Irwin-Hall(4) variates for counters start..start+count-1.

    value = bf16_rne( float32(s) * float32(sigma / IRWIN_HALL_STD) ), with
    s = u0+u1+u2+u3 - 131070 from the four 16-bit fields of one SplitMix64 output.
    """
    z = splitmix64(key, np.arange(start, start + count, dtype=np.uint64))
    m = np.uint64(0xFFFF)
    s = ((z & m) + ((z >> np.uint64(16)) & m) + ((z >> np.uint64(32)) & m) + (z >> np.uint64(48))).astype(np.int64)
    s -= 131070
    scale = np.float32(sigma / IRWIN_HALL_STD)
    v = s.astype(np.float32) * scale
    return f32_to_bf16_bits(v)


def cache_key(seed: int) -> int:
    return (seed * 0x5851F42D4C957F2D + 0x14057B7EF767814F) & 0xFFFFFFFFFFFFFFFF


# ---------------------------------------------------------------------------
# decode inputs
# ---------------------------------------------------------------------------


def make_decode_inputs(w: DecodeWorkload, seed: Optional[int] = None) -> Dict[str, object]:
    """Per-token decode inputs (Q, C [b, G, N]; E, Y [b, H, P]; g), the inputs of a decode step's
    state update (X [b, H, P], B [b, G, N], logA [b, H] fp32, drawn after the others with the layer
    workloads' recipes) and the cache key.

    The chunk-memory cache [b, H, n_chunks, N, P] is *not* materialised here: element
    i of the flat cache is ``irwin_hall_bf16(key, i, 1, sigma)``. Use
    :func:`decode_cache_slice` on the host or ``workloads.device.fill_cache`` on the GPU.
    """
    if seed is None:
        seed = BASE_SEED + w.index
    rng = np.random.Generator(np.random.PCG64(seed))
    Bt, H, G, N, P = w.batch, w.nheads, w.ngroups, w.dstate, w.headdim
    Q = rng.standard_normal((Bt, G, N)) / math.sqrt(N)
    C = rng.standard_normal((Bt, G, N)) / math.sqrt(N)
    E = rng.standard_normal((Bt, H, P)) / math.sqrt(P)
    Y = rng.standard_normal((Bt, H, P)) / math.sqrt(P)
    X = rng.standard_normal((Bt, H, P)) / math.sqrt(P)
    B = rng.standard_normal((Bt, G, N)) / math.sqrt(N)
    a_head = np.exp(rng.uniform(-4.0, -1.0, size=(H,)))  # the "mamba2" log-decay recipe, one token
    logA = -(a_head[None, :] * _softplus(rng.standard_normal((Bt, H)) + 1.0))
    return dict(Q=store(Q, w.dtype), C=store(C, w.dtype), E=store(E, w.dtype), Y=store(Y, w.dtype),
                X=store(X, w.dtype), B=store(B, w.dtype), logA=np.ascontiguousarray(logA.astype(np.float32)),
                g=np.array([1.0], dtype=np.float32), g_strides=(0, 0), key=cache_key(seed))


def decode_cache_slice(w: DecodeWorkload, key: int, b: int, h: int, chunk_stride: Optional[int] = None) -> Stored:
    """Host copy of cache[b, h, :n_chunks] (bf16) from the counter-based generator."""
    cs = w.n_chunks if chunk_stride is None else chunk_stride
    per = w.dstate * w.headdim
    start = ((b * w.nheads + h) * cs) * per
    bits = irwin_hall_bf16(key, start, w.n_chunks * per, w.cache_sigma)
    return Stored(bits.reshape(w.n_chunks, w.dstate, w.headdim), "bf16")
