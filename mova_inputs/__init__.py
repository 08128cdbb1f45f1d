"""Seeded synthetic inputs for the MoVA value path.

This module only draws random numbers and stores them in the formats the
value path consumes (fp32, bf16 bit patterns, int8 indices, fp16 weights).
It holds none of the method's arithmetic: no routing, no activation, no
mixing.  Both the fp64 CPU oracle and the CUDA library are fed from here,
and nothing else is shared between them.

Workloads (all on one MoVA layer of 64 value experts, d_model 2560, expert
width 8 heads x 128 = 1024, top-4; shapes as stated by "MoVA: routing the
value vectors, and why the KV cache does not notice", sections "Where the
routing happens" and "So what does it cost?"):

  pr1        T=128, everything fp32 (the small case the oracle finishes fast)
  decode     T=8, bf16 x and experts, fp32 router
  prefill    T=4096, as decode
  skewed     T=16384, router bias 2*ln(p_e) with p_e a Zipf(1.2) law over e
  given      L=32768 cached x rows with precomputed routing: int8 top-4
             indices (first 4 of a uniform permutation of the 64 experts)
             and fp16 weights 2.5*g/sum(g), g ~ Exp(1) i.i.d.

Distributions: x ~ N(0,1); router weight ~ N(0, 0.02) (std); router bias
~ N(0, 0.01); expert weight ~ N(0, 1/sqrt(2560)) (the second parameter is
the standard deviation in every case).

bf16 values are produced by round-to-nearest-even from fp32 draws and are
kept as raw uint16 bit patterns, so both consumers see the same numbers.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

D_MODEL = 2560
N_EXPERTS = 64
TOP_K = 4
N_HEADS = 8
HEAD_DIM = 128
N_OUT = N_HEADS * HEAD_DIM
SCALE = 2.5

# Fixed stream ids: each tensor of a layer draws from its own child stream.
_STREAM = {"x": 1, "wr": 2, "br": 3, "wv": 4, "idx": 5, "w": 6, "probs": 7}

WORKLOADS = {
    # name: (tokens, activation dtype, routing mode, bias law)
    "pr1": dict(T=128, dtype="f32", mode="routed", bias="normal"),
    "decode": dict(T=8, dtype="bf16", mode="routed", bias="normal"),
    "prefill": dict(T=4096, dtype="bf16", mode="routed", bias="normal"),
    "skewed": dict(T=16384, dtype="bf16", mode="routed", bias="zipf"),
    "given": dict(T=32768, dtype="bf16", mode="given", bias="normal"),
    # one query token's attention (32 heads) over 32768 cached positions whose
    # values are recomputed from the compact cache (the given workload's)
    "attend": dict(T=32768, dtype="bf16", mode="attend", bias="normal"),
}
ATTEND_HEADS = 32


@dataclasses.dataclass
class Layer:
    """Weights of one MoVA value layer in storage format.

    Wr: (E, d) fp32 router weight; br: (E,) fp32 router bias;
    Wv: (E, n, d) expert weights, fp32 or bf16 bits (uint16), row-major
    (each expert stored output-major like a linear layer's weight).
    """
    Wr: np.ndarray
    br: np.ndarray
    Wv: np.ndarray
    wv_dtype: str


@dataclasses.dataclass
class Batch:
    """Per-step activations (and, for routing-given mode, the routing)."""
    x: np.ndarray                 # (T, d) fp32 or bf16 bits
    x_dtype: str
    idx: Optional[np.ndarray] = None   # (T, k) int8, routing-given mode
    w: Optional[np.ndarray] = None     # (T, k) fp16, routing-given mode
    probs: Optional[np.ndarray] = None  # (H, T) fp32, attend mode


def _rng(seed: int, layer: int, stream: str, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(
        np.random.PCG64(np.random.SeedSequence([int(seed), int(layer), _STREAM[stream], int(sub)])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def _f32_to_bf16_bits_fast(a: np.ndarray) -> np.ndarray:
    # torch's float->bfloat16 cast is round-to-nearest-even as well; it is
    # only used for speed on the large expert tensors (checked against the
    # numpy path in the input tests).
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def zipf_bias(E: int = N_EXPERTS, s: float = 1.2, gain: float = 2.0) -> np.ndarray:
    """Skewed router bias: gain * ln p_e, p_e proportional to (e+1)^-s over
    e = 0..E-1, normalised to sum 1 (expert 0 is Zipf rank 1)."""
    p = (np.arange(1, E + 1, dtype=np.float64)) ** (-s)
    p /= p.sum()
    return (gain * np.log(p)).astype(np.float32)


def make_layer(seed: int = 0, layer: int = 0, *, d: int = D_MODEL, E: int = N_EXPERTS,
               n: int = N_OUT, wv_dtype: str = "bf16", bias: str = "normal",
               threads: int = 8) -> Layer:
    Wr = _rng(seed, layer, "wr").standard_normal((E, d), dtype=np.float32) * np.float32(0.02)
    if bias == "zipf":
        br = zipf_bias(E)
    else:
        br = _rng(seed, layer, "br").standard_normal(E, dtype=np.float32) * np.float32(0.01)
    std = np.float32(1.0 / np.sqrt(float(d)))
    Wv32 = np.empty((E, n, d), dtype=np.float32)

    def fill(e: int) -> None:
        _rng(seed, layer, "wv", e).standard_normal(out=Wv32[e], dtype=np.float32)
        Wv32[e] *= std

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range(E)))
    if wv_dtype == "bf16":
        Wv = _f32_to_bf16_bits_fast(Wv32)
    elif wv_dtype == "f32":
        Wv = Wv32
    else:
        raise ValueError(wv_dtype)
    return Layer(Wr=np.ascontiguousarray(Wr), br=np.ascontiguousarray(br), Wv=Wv, wv_dtype=wv_dtype)


def make_batch(T: int, seed: int = 0, step: int = 0, *, d: int = D_MODEL, dtype: str = "bf16",
               mode: str = "routed", E: int = N_EXPERTS, k: int = TOP_K,
               scale: float = SCALE) -> Batch:
    x32 = _rng(seed, 1000 + step, "x").standard_normal((T, d), dtype=np.float32)
    if dtype == "bf16":
        x = _f32_to_bf16_bits_fast(x32)
    elif dtype == "f32":
        x = x32
    else:
        raise ValueError(dtype)
    b = Batch(x=x, x_dtype=dtype)
    if mode in ("given", "attend"):
        # Routing of the compact cache: k distinct experts per token, the
        # first k entries of a uniform random permutation of the experts.
        r = _rng(seed, 1000 + step, "idx")
        keys = r.random((T, E))
        b.idx = np.argsort(keys, axis=1)[:, :k].astype(np.int8)
        g = _rng(seed, 1000 + step, "w").exponential(1.0, size=(T, k))
        b.w = (scale * g / g.sum(axis=1, keepdims=True)).astype(np.float16)
    if mode == "attend":
        b.probs = make_attention_probs(ATTEND_HEADS, T, seed, step)
    return b


def make_attention_probs(H: int, L: int, seed: int = 0, step: int = 0, *, spread: float = 2.0,
                         support: int = 0) -> np.ndarray:
    """Attention probabilities of one query token's H heads over L cached
    positions, (H, L) fp32: a softmax of N(0, spread) scores per head (the
    shape decode attention produces; no trained model is involved).  With
    support > 0 each head puts all its probability on `support` random
    positions (softmax over those only), the rest exactly zero."""
    r = _rng(seed, 2000 + step, "probs")
    z = r.standard_normal((H, L)) * spread
    if support > 0:
        keep = np.zeros((H, L), dtype=bool)
        for h in range(H):
            keep[h, r.choice(L, size=min(support, L), replace=False)] = True
        z = np.where(keep, z, -np.inf)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def workload(name: str, seed: int = 0, layer: int = 0, step: int = 0):
    """(Layer, Batch) of a named workload."""
    cfg = WORKLOADS[name]
    wdt = "f32" if cfg["dtype"] == "f32" else "bf16"
    lay = make_layer(seed, layer, wv_dtype=wdt, bias=cfg["bias"])
    bat = make_batch(cfg["T"], seed, step, dtype=cfg["dtype"], mode=cfg["mode"])
    return lay, bat
