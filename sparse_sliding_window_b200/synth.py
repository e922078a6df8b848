"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module holds no attention arithmetic: it only draws numbers and builds
the integer attention mask structure (which tokens are local, global or
padding).  Both the CUDA path and the CPU oracle consume its output; neither
imports the other.

Generator (counter based, so any element can be recomputed on its own):
  * splitmix64 finaliser ``mix(z)`` (Steele, Lea & Flood, "Fast splittable
    pseudorandom number generators", OOPSLA 2014):
    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
    z *= 0x94D049BB133111EB; z ^= z >> 31.
  * stream key = mix(seed * G ^ mix(stream_id + 1)), G = 0x9E3779B97F4A7C15;
    the k-th 64-bit word of a stream = mix(key + (k + 1) * G).
  * uniforms: u = (word >> 11) * 2**-53 in [0, 1); u1 uses (word >> 11) + 1 so
    it lies in (0, 1].
  * normals (Box-Muller, cosine branch): z_k = sqrt(-2 ln u1) cos(2 pi u2)
    with u1, u2 taken from words 2k and 2k + 1.
  * values are scaled, then rounded to the run's dtype with round-to-nearest-
    even (float16 / float32 by numpy's casts, bfloat16 by rounding the float32
    bit pattern).  ``as_float64`` returns exactly the rounded values.

Workload structure (the five synthetic workloads of the longformer pages'
shapes, see ``WORKLOADS``):
  * attention_mask codes: 0 = no attention (padding), 1 = local, 2 = global;
  * lengths / global positions are drawn from their own streams.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

_G = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream ids of the tensors a workload draws
STREAMS = {"qs": 1, "ks": 2, "vs": 3, "qg": 4, "kg": 5, "vg": 6, "do": 7,
           "lengths": 8, "globals": 9,
           # the projections around the attention: hidden states, input
           # weights and biases, attention output, output weights and bias
           "x": 10, "w": 11, "b": 12, "o": 13, "wo": 14, "bo": 15}


def _mix(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([seed], dtype=np.uint64) * _G
        t = _mix(np.array([stream + 1], dtype=np.uint64))
        return _mix(s ^ t)[0]


def words(seed: int, stream: int, count: int, start: int = 0) -> np.ndarray:
    """64-bit words ``start .. start+count-1`` of stream ``stream``."""
    k = _key(seed, stream)
    ctr = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(k + ctr * _G)


def uniforms(seed: int, stream: int, count: int, start: int = 0) -> np.ndarray:
    w = words(seed, stream, count, start)
    return (w >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normals(seed: int, stream: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.float64)
    chunk = 1 << 22
    for s in range(0, count, chunk):
        c = min(chunk, count - s)
        w = words(seed, stream, 2 * c, 2 * s)
        u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
        u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        out[s:s + c] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return out


# ---------------------------------------------------------------- rounding --

DTYPES = ("f32", "bf16", "f16")


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to ``dtype`` (RNE).  Returns the storage array:
    float32, float16, or uint16 bit patterns for bfloat16."""
    if dtype == "f32":
        return x.astype(np.float32)
    if dtype == "f16":
        return x.astype(np.float16)
    if dtype == "bf16":
        b = x.astype(np.float32).view(np.uint32)
        lsb = (b >> np.uint32(16)) & np.uint32(1)
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
        return r.astype(np.uint16)
    raise ValueError(dtype)


def as_float64(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of a storage array produced by ``round_to``."""
    if dtype == "bf16":
        return (stored.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return stored.astype(np.float64)


def tensor(seed: int, name: str, shape: Sequence[int], dtype: str, scale: float = 1.0) -> np.ndarray:
    """A seeded N(0,1)*scale tensor, rounded to dtype (storage array)."""
    count = int(np.prod(shape))
    return round_to(normals(seed, STREAMS[name], count).reshape(shape) * scale, dtype)


# -------------------------------------------------------------- workloads --

@dataclasses.dataclass
class Workload:
    name: str
    B: int
    H: int
    n: int
    head_dim: int
    r: int                      # one-sided window (w = 2r)
    dilation: List[int]         # per head
    causal: bool
    dtype: str
    in_scale: float             # inputs ~ N(0, 1) * in_scale
    mask_kind: str              # see build_mask
    seed: int
    backward: bool = False
    n_global_random: int = 0    # extra random global positions (batched)
    description: str = ""

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _wl(idx, **kw) -> Workload:
    return Workload(seed=20260000 + idx, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": _wl(1, name="tiny_f32", B=1, H=2, n=1024, head_dim=64, r=64, dilation=[1, 1],
                    causal=False, dtype="f32", in_scale=1.0, mask_kind="global0",
                    description="tiny fp32 forward, B1 H2 n1024 hd64 w128, token 0 global"),
    "base_bf16": _wl(2, name="base_bf16", B=1, H=12, n=4096, head_dim=64, r=256, dilation=[1] * 12,
                     causal=False, dtype="bf16", in_scale=0.5, mask_kind="question65",
                     description="longformer-base shape forward, B1 H12 n4096 hd64 w512, "
                                 "globals 0..64 (QA question block)"),
    "batched_f16": _wl(3, name="batched_f16", B=8, H=12, n=4096, head_dim=64, r=256,
                       dilation=[1] * 12, causal=False, dtype="f16", in_scale=1.0,
                       mask_kind="padded", n_global_random=16,
                       description="batched padded forward, B8 H12 n4096 hd64 w512, lengths "
                                   "U[2048,4096], tail mask 0, token 0 + 16 random globals"),
    "charlm_bf16": _wl(4, name="charlm_bf16", B=1, H=8, n=23040, head_dim=64, r=512,
                       dilation=[2, 2, 1, 1, 1, 1, 1, 1], causal=True, dtype="bf16", in_scale=1.0,
                       mask_kind="local",
                       description="autoregressive dilated char-LM, B1 H8 n23040 hd64 causal "
                                   "one-sided 512, d=2 on heads 0-1"),
    "led_bf16": _wl(5, name="led_bf16", B=2, H=16, n=16384, head_dim=64, r=512, dilation=[1] * 16,
                    causal=False, dtype="bf16", in_scale=1.0, mask_kind="global0", backward=True,
                    description="LED-large-encoder-sized forward+backward, B2 H16 n16384 hd64 "
                                "w1024, token 0 global"),
}


def build_mask(wl: Workload) -> np.ndarray:
    """int32 [B, n] attention_mask of a workload (0 pad / 1 local / 2 global)."""
    B, n = wl.B, wl.n
    m = np.ones((B, n), dtype=np.int32)
    if wl.mask_kind == "local":
        pass
    elif wl.mask_kind == "global0":
        m[:, 0] = 2
    elif wl.mask_kind == "question65":
        m[:, 0:min(65, n)] = 2
    elif wl.mask_kind == "padded":
        lo, hi = n // 2, n
        u = uniforms(wl.seed, STREAMS["lengths"], B)
        lengths = lo + np.floor(u * (hi - lo + 1)).astype(np.int64)
        lengths = np.minimum(lengths, hi)
        for b in range(B):
            L = int(lengths[b])
            m[b, L:] = 0
            m[b, 0] = 2
            k = min(wl.n_global_random, max(L - 1, 0))
            # k distinct positions in [1, L): partial Fisher-Yates on the stream
            pool = np.arange(1, L, dtype=np.int64)
            uu = uniforms(wl.seed, STREAMS["globals"] + 16 * (b + 1), k)
            for t in range(k):
                s = t + int(np.floor(uu[t] * (len(pool) - t)))
                pool[t], pool[s] = pool[s], pool[t]
            m[b, pool[:k]] = 2
    else:
        raise ValueError(wl.mask_kind)
    return m


def make_inputs(wl: Workload, with_do: Optional[bool] = None) -> Dict[str, np.ndarray]:
    """All inputs of a workload as storage arrays (+ 'mask', 'dilation')."""
    shape = (wl.B, wl.H, wl.n, wl.head_dim)
    out = {}
    names = ["qs", "ks", "vs", "qg", "kg", "vg"]
    if wl.backward if with_do is None else with_do:
        names.append("do")
    for name in names:
        out[name] = tensor(wl.seed, name, shape, wl.dtype, wl.in_scale if name != "do" else 1.0)
    out["mask"] = build_mask(wl)
    out["dilation"] = np.asarray(wl.dilation, dtype=np.int32)
    return out


def custom(name: str, B: int, H: int, n: int, r: int, dilation, causal: bool, dtype: str,
           mask: np.ndarray, seed: int, in_scale: float = 1.0, head_dim: int = 64,
           backward: bool = False) -> Workload:
    """A small ad-hoc workload for tests (mask given explicitly)."""
    wl = Workload(name=name, B=B, H=H, n=n, head_dim=head_dim, r=r, dilation=list(dilation),
                  causal=causal, dtype=dtype, in_scale=in_scale, mask_kind="explicit", seed=seed,
                  backward=backward)
    wl._mask = np.ascontiguousarray(mask, dtype=np.int32)  # type: ignore[attr-defined]
    return wl


def inputs_for(wl: Workload, with_do: Optional[bool] = None) -> Dict[str, np.ndarray]:
    """Like make_inputs but honours an explicit mask attached by ``custom``."""
    if wl.mask_kind == "explicit":
        shape = (wl.B, wl.H, wl.n, wl.head_dim)
        out = {}
        names = ["qs", "ks", "vs", "qg", "kg", "vg"]
        if wl.backward if with_do is None else with_do:
            names.append("do")
        for name in names:
            out[name] = tensor(wl.seed, name, shape, wl.dtype, wl.in_scale if name != "do" else 1.0)
        out["mask"] = wl._mask.copy()  # type: ignore[attr-defined]
        out["dilation"] = np.asarray(wl.dilation, dtype=np.int32)
        return out
    return make_inputs(wl, with_do)
