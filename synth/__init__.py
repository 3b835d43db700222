"""Seeded synthetic inputs for the HySparse2 hot path.

This module is shared by the CPU oracle tests, the GPU parity tests and the benchmark. It
holds no attention arithmetic: it only draws random numbers (numpy PCG64, one independent
child stream per tensor), adds the planted direction, and rounds float32 samples to bf16
once (round to nearest even), so that the oracle and the CUDA path consume the very same
bf16 values.

Workloads (shapes from the five synthetic configurations the method is measured on):

* ``tiny_prefill``  B=1, L=2048, 16 Q heads, head_dim 64, scale 1/8, 1 sparse layer
* ``decode_32k``    B=32 sequences, 32,768-token cache, 1 query token, 64 heads, d=128, 4 sparse layers
* ``prefill_32k``   B=1, L=32,768, 64 heads, d=128, 4 sparse layers, plus a KV Bridging
                    projection H[32768 x 2048] through 4 layers' W_k, W_v [2048 x 128]
* ``decode_256k``   B=8, 262,144-token cache
* ``decode_1m``     B=2, 1,048,576-token cache

Distribution: Q, K, V (and every sparse layer's own Q) are i.i.d. N(0, 1). A unit direction
u (a normalised N(0, I_d) draw) is added with gain 3 to exactly floor(0.02 * Lk) key
positions per sequence (drawn without replacement) and to every query vector (all heads,
all layers), so that the top-k selection is not trivial. V is not planted. The bridge
hidden state is N(0, 1) and the projection weights are N(0, 0.02^2).

Backward pass: the upstream gradient of each layer's output is N(0, 1), rounded to bf16
(``grad_out``).

FP8 cache: the same float32 K and V samples stored as OCP e4m3 codes (1 sign, 4 exponent bits
with bias 7, 3 mantissa bits, subnormals, no infinities) times one power-of-two scale per
tensor, the smallest for which the largest magnitude fits under 448; each value rounds to the
nearest code, ties to the even code.
"""
from __future__ import annotations

import math
import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from functools import cached_property

import numpy as np

WINDOW = 128   # most recent tokens always selected
TOPK = 1024    # older tokens selected by score
PLANT_FRAC = 0.02
PLANT_GAIN = 3.0
W_STD = 0.02


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Lq: int
    Lk: int
    H: int
    d: int
    scale: float
    n_sparse: int
    window: int = WINDOW
    topk: int = TOPK
    bridge_T: int = 0
    bridge_hidden: int = 0
    bridge_layers: int = 0

    @property
    def S(self) -> int:
        return self.window + self.topk

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny_prefill": Workload("tiny_prefill", 1, 2048, 2048, 16, 64, 1.0 / 8.0, 1),
    "decode_32k": Workload("decode_32k", 32, 1, 32768, 64, 128, 1.0 / math.sqrt(128), 4),
    "prefill_32k": Workload("prefill_32k", 1, 32768, 32768, 64, 128, 1.0 / math.sqrt(128), 4,
                            bridge_T=32768, bridge_hidden=2048, bridge_layers=4),
    "decode_256k": Workload("decode_256k", 8, 1, 262144, 64, 128, 1.0 / math.sqrt(128), 4),
    "decode_1m": Workload("decode_1m", 2, 1, 1048576, 64, 128, 1.0 / math.sqrt(128), 4),
}


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns the uint16 bit patterns.
    Large arrays are converted in chunks on several threads (element-wise: same result)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1)
    out = np.empty(flat.shape, np.uint16)

    def conv(lo, hi):
        u = flat[lo:hi].view(np.uint32)
        out[lo:hi] = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)

    n = flat.size
    if n <= _CHUNK:
        conv(0, n)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(lambda c: conv(c, min(n, c + _CHUNK)), range(0, n, _CHUNK)))
    return out.reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


E4M3_MAX = 448.0


def e4m3_scale(x: np.ndarray) -> float:
    """The power-of-two scale 2^e with max|x| / 2^e <= 448 for the smallest such e."""
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    if amax == 0.0:
        return 1.0
    e = math.ceil(math.log2(amax / E4M3_MAX))
    if amax / 2.0 ** e > E4M3_MAX:  # log2 rounding at an exact power of two
        e += 1
    return float(2.0 ** e)


def f32_to_e4m3(x: np.ndarray, scale: float) -> np.ndarray:
    """Codes of x / scale rounded to e4m3 (nearest, ties to even); |x / scale| must be <= 448."""
    a = np.asarray(x, dtype=np.float64).reshape(-1) / scale
    if not np.all(np.isfinite(a)) or np.max(np.abs(a), initial=0.0) > E4M3_MAX:
        raise ValueError("value outside the e4m3 range")
    sign = np.signbit(a).astype(np.int64)
    m = np.abs(a)
    code = np.empty(m.shape, np.int64)
    sub = m < 2.0 ** -6
    # subnormal range: steps of 2^-9 (code = steps; 8 steps is the smallest normal, code 8)
    code[sub] = np.rint(m[sub] * 2.0 ** 9).astype(np.int64)
    nrm = ~sub
    if np.any(nrm):
        _, ex = np.frexp(m[nrm])           # m = f * 2^ex, f in [0.5, 1)
        e = ex.astype(np.int64) - 1        # m in [2^e, 2^(e+1))
        steps = np.rint(np.ldexp(m[nrm], (3 - e).astype(np.int32))).astype(np.int64)  # 8..16
        code[nrm] = (e + 6) * 8 + steps    # (e + 7) * 8 + (steps - 8); 16 steps carries into e + 1
    if np.any(code > 0x7E):
        raise ValueError("value rounds above 448")
    return (code | (sign << 7)).astype(np.uint8).reshape(np.shape(x))


_CHUNK = 1 << 24  # elements per independent sub-stream for large tensors


def _normal_f32(seq: np.random.SeedSequence, shape) -> np.ndarray:
    """N(0,1) float32 array; large arrays are filled chunk by chunk from spawned streams."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    n_chunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    kids = seq.spawn(n_chunks)

    def fill(c):  # each chunk from its own stream: the result does not depend on the threads
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        np.random.Generator(np.random.PCG64(kids[c])).standard_normal(hi - lo, dtype=np.float32, out=out[lo:hi])

    if n_chunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(n_chunks)))
    return out.reshape(shape)


class SyntheticInputs:
    """Lazily generated, cached inputs of one workload (uint16 bf16 bit patterns)."""

    N_STREAMS = 16

    def __init__(self, wl: Workload, seed: int = 0):
        self.wl = wl
        self.seed = seed
        root = np.random.SeedSequence([seed, zlib.crc32(wl.name.encode())])
        self._s = root.spawn(self.N_STREAMS)

    @cached_property
    def u(self) -> np.ndarray:
        g = np.random.Generator(np.random.PCG64(self._s[0]))
        u = g.standard_normal(self.wl.d)
        return (u / np.linalg.norm(u)).astype(np.float32)

    @cached_property
    def planted(self) -> np.ndarray:
        """[B, n_planted] sorted key positions that carry the planted direction."""
        wl = self.wl
        g = np.random.Generator(np.random.PCG64(self._s[1]))
        n = int(math.floor(PLANT_FRAC * wl.Lk))
        return np.stack([np.sort(g.choice(wl.Lk, size=n, replace=False)) for _ in range(wl.B)]).astype(np.int64)

    def _query(self, stream: int) -> np.ndarray:
        wl = self.wl
        q = _normal_f32(self._s[stream], (wl.B, wl.Lq, wl.H, wl.d))
        q += PLANT_GAIN * self.u
        return f32_to_bf16_bits(q)

    @cached_property
    def q(self) -> np.ndarray:
        """[B, Lq, H, d] query of the full-attention layer."""
        return self._query(2)

    @cached_property
    def k(self) -> np.ndarray:
        """[B, Lk, d] keys (one KV head)."""
        return f32_to_bf16_bits(self._k_f32)

    @cached_property
    def _v_f32(self) -> np.ndarray:
        # drawn once: a SeedSequence hands out new children on every spawn, so a second draw
        # from the same stream would be a different sample
        wl = self.wl
        return _normal_f32(self._s[4], (wl.B, wl.Lk, wl.d))

    @cached_property
    def v(self) -> np.ndarray:
        """[B, Lk, d] values (one KV head)."""
        return f32_to_bf16_bits(self._v_f32)

    @cached_property
    def _k_f32(self) -> np.ndarray:
        wl = self.wl
        k = _normal_f32(self._s[3], (wl.B, wl.Lk, wl.d))
        for b in range(wl.B):
            k[b, self.planted[b]] += PLANT_GAIN * self.u
        return k

    @cached_property
    def k8(self) -> tuple[np.ndarray, float]:
        """([B, Lk, d] e4m3 codes, power-of-two scale) of the same key samples as ``k``."""
        k = self._k_f32
        sc = e4m3_scale(k)
        return f32_to_e4m3(k, sc), sc

    @cached_property
    def v8(self) -> tuple[np.ndarray, float]:
        """([B, Lk, d] e4m3 codes, power-of-two scale) of the same value samples as ``v``."""
        v = self._v_f32
        sc = e4m3_scale(v)
        return f32_to_e4m3(v, sc), sc

    def q_sparse(self, layer: int) -> np.ndarray:
        """[B, Lq, H, d] query of sparse layer `layer` (same distribution as q)."""
        assert 0 <= layer < self.wl.n_sparse and layer < self.N_STREAMS - 8
        key = f"_qs{layer}"
        if key not in self.__dict__:
            self.__dict__[key] = self._query(8 + layer)
        return self.__dict__[key]

    def grad_out(self, layer: int) -> np.ndarray:
        """[B, Lq, H, d] upstream gradient dL/d(out) of layer `layer` of the hybrid block (0: the
        full layer, 1..n_sparse: the sparse layers), N(0, 1) rounded to bf16, for the backward
        pass. Each layer draws from its own child of stream 7, derived by its spawn key so that
        the draw does not depend on the order of the calls."""
        assert 0 <= layer <= self.wl.n_sparse
        key = f"_go{layer}"
        if key not in self.__dict__:
            parent = self._s[7]
            child = np.random.SeedSequence(parent.entropy, spawn_key=tuple(parent.spawn_key) + (layer,),
                                           pool_size=parent.pool_size)
            wl = self.wl
            self.__dict__[key] = f32_to_bf16_bits(_normal_f32(child, (wl.B, wl.Lq, wl.H, wl.d)))
        return self.__dict__[key]

    @cached_property
    def bridge_h(self) -> np.ndarray:
        """[T, hidden] hidden state feeding the KV Bridging projections."""
        wl = self.wl
        return f32_to_bf16_bits(_normal_f32(self._s[5], (wl.bridge_T, wl.bridge_hidden)))

    @cached_property
    def bridge_w(self) -> np.ndarray:
        """[n_layers, 2 (K, V), hidden, d] projection weights."""
        wl = self.wl
        w = _normal_f32(self._s[6], (wl.bridge_layers, 2, wl.bridge_hidden, wl.d)) * np.float32(W_STD)
        return f32_to_bf16_bits(w)

    # single new token row of each sequence (used for the end-to-end decode measurement)
    def new_token_kv(self) -> tuple[np.ndarray, np.ndarray]:
        return self.k[:, -1:, :].copy(), self.v[:, -1:, :].copy()


def small(name: str, **kw) -> Workload:
    """A copy of a named workload with some fields overridden (for reduced-size tests)."""
    return WORKLOADS[name].with_(name=name + "_" + "_".join(f"{k}{v}" for k, v in sorted(kw.items())), **kw)
