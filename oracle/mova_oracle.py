"""fp64 CPU oracle of the MoVA value path -- TEST INFRASTRUCTURE ONLY.

This file is the plain, slow, obviously correct statement of what the value
path computes.  Only the tests, the smoke check and the CPU-baseline leg of
the benchmark may import it; the CUDA library never does, and it shares no
code with it.

Source of the method: "MoVA: routing the value vectors, and why the KV cache
does not notice" (ai.thesatyajit.com), section "Where the routing happens":
the attention layer's v_proj is replaced by a 2560->64 router applied to the
flattened hidden states without its bias, a sigmoid-gated top-4 selection to
which the router bias is handed separately, a renormalisation of the four
sigmoid scores scaled by 2.5, and a mixture of the four selected
2560->1024 expert projections, each passed through SiLU, weighted and
summed; the (tokens, 1024) result is viewed as (tokens, 8 heads, 128).

Readings of points the page leaves open (each also listed in the design
notes):
  * the router bias is added to the sigmoid scores and steers the selection
    only; the weights use the unbiased scores;
  * ties in the biased score go to the lower expert index; slot 0 holds the
    highest biased score;
  * renormalise over the k selected scores, then multiply by the scale;
  * no bias in the expert projections; SiLU is applied per expert before
    weighting; slots are summed in ascending slot order;
  * in routing-given mode (the compact cache of "IFM K2 Horizon Deep Dive",
    Section 4, Option B) the stored fp16 weights are used as they are.

Every computation is in float64 on exactly converted inputs.  A matrix
product from numpy and a stable argsort serve as steps; nothing is blocked,
fused or reordered beyond the definition.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Exact conversion of stored inputs to float64
# ---------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (a bf16 is the top
    half of an fp32)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Stored tensor -> float64.  dtype in {"f32", "bf16", "f16", "f64"}."""
    if dtype == "bf16":
        return bf16_bits_to_f64(a)
    if dtype in ("f32", "f16", "f64"):
        return np.asarray(a).astype(np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Router: "Where the routing happens"
# ---------------------------------------------------------------------------


def router_logits(x: np.ndarray, Wr: np.ndarray) -> np.ndarray:
    """logits[t, e] = sum_j x[t, j] * Wr[e, j]; the router's linear map is
    applied WITHOUT its bias (the bias is handed to the gate separately).
    x: (T, d) fp64, Wr: (E, d) fp64 -> (T, E) fp64."""
    return x @ Wr.T


def router_logits_partitioned(x: np.ndarray, Wr: np.ndarray, partitions: int) -> np.ndarray:
    """Router logits with the reduction over d split into `partitions`
    equal consecutive ranges, as a router GEMM partitioned along K computes
    them: each range's dot product is formed (exactly, in fp64) and rounded
    once to fp32, and the fp32 partial sums are added in range order with
    fp32 rounding.  "Mixture of Value Attention" (robotsatlas.com),
    "Implementation pitfalls", names keeping the router's numerics through
    its GEMM partitioning; the serving recipe of "IFM/K2-Horizon-MoVA-36B-A4B"
    (paperfeed.app) sets two partitions.  The reading -- halves of d, each
    rounded to fp32, then added first + second -- is this oracle's.
    x: (T, d) fp64, Wr: (E, d) fp64, d divisible by `partitions`
    -> (T, E) fp64 holding fp32 values."""
    d = x.shape[1]
    assert d % partitions == 0
    step = d // partitions
    acc = None
    for p in range(partitions):
        part = (x[:, p * step:(p + 1) * step] @ Wr[:, p * step:(p + 1) * step].T).astype(np.float32)
        acc = part if acc is None else (acc + part).astype(np.float32)
    return acc.astype(np.float64)


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Logistic function 1 / (1 + exp(-z)), in fp64."""
    return 1.0 / (1.0 + np.exp(-z))


def select_top_k(b: np.ndarray, k: int) -> np.ndarray:
    """The k experts with the largest biased score b, in descending order of
    b; equal scores go to the lower expert index.  Done as a full stable
    sort of -b, so it is the plain definition of "top-k".
    b: (T, E) -> (T, k) int64."""
    order = np.argsort(-b, axis=1, kind="stable")
    return order[:, :k]


def route(x: np.ndarray, Wr: np.ndarray, br: np.ndarray, k: int, scale: float,
          partitions: int = 1):
    """Sigmoid gate, bias-assisted top-k, renormalise, scale.

    s = sigmoid(logits); b = s + br (selection only); idx = top-k of b;
    w[t, slot] = scale * s[t, idx] / sum over the k slots of s[t, idx].
    partitions > 1 takes the logits of router_logits_partitioned.
    Returns dict(idx (T,k) int64, w (T,k), s (T,E), b (T,E), logits (T,E)).
    """
    logits = router_logits(x, Wr) if partitions == 1 else router_logits_partitioned(x, Wr, partitions)
    s = sigmoid(logits)
    b = s + br[None, :]
    idx = select_top_k(b, k)
    s_sel = np.take_along_axis(s, idx, axis=1)
    w = scale * s_sel / s_sel.sum(axis=1, keepdims=True)
    return dict(idx=idx, w=w, s=s, b=b, logits=logits)


def weights_for(s: np.ndarray, idx: np.ndarray, scale: float) -> np.ndarray:
    """Renormalised, scaled weights of a given selection (used when a
    near-tie admits another valid selection)."""
    s_sel = np.take_along_axis(s, idx, axis=1)
    return scale * s_sel / s_sel.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# Experts and mixture: "Where the routing happens"
# ---------------------------------------------------------------------------


def silu(h: np.ndarray) -> np.ndarray:
    """SiLU(h) = h * sigmoid(h)."""
    return h * sigmoid(h)


def combine(x: np.ndarray, idx: np.ndarray, w: np.ndarray, Wv, wv_dtype: str = "f64") -> np.ndarray:
    """v[t] = sum over slots (ascending) of w[t, slot] * SiLU(Wv[idx[t, slot]] @ x[t]).

    x: (T, d) fp64; idx: (T, k) ints; w: (T, k) fp64;
    Wv: (E, n, d) stored expert weights (converted per expert on demand).
    Returns v (T, n) fp64.
    """
    T = x.shape[0]
    k = idx.shape[1]
    n = Wv.shape[1]
    v = np.zeros((T, n), dtype=np.float64)
    cache = {}

    def expert(e: int) -> np.ndarray:
        if e not in cache:
            cache[e] = to_f64(Wv[e], wv_dtype)
        return cache[e]

    for slot in range(k):
        for e in np.unique(idx[:, slot]):
            rows = np.nonzero(idx[:, slot] == e)[0]
            h = x[rows] @ expert(int(e)).T
            v[rows] += w[rows, slot][:, None] * silu(h)
    return v


def value_routed(x: np.ndarray, Wr: np.ndarray, br: np.ndarray, Wv, k: int, scale: float,
                 wv_dtype: str = "f64"):
    """Full path: route, then mix.  Returns (v (T, n), routing dict)."""
    r = route(x, Wr, br, k, scale)
    v = combine(x, r["idx"], r["w"], Wv, wv_dtype)
    return v, r


def as_gqa(v: np.ndarray, head_dim: int = 128) -> np.ndarray:
    """(T, heads*head_dim) -> (T, heads, head_dim): the value tensor a GQA
    v_proj writes per token (the page's reshape to 128-wide heads)."""
    T, n = v.shape
    return v.reshape(T, n // head_dim, head_dim)


def attend(x: np.ndarray, idx: np.ndarray, w: np.ndarray, Wv, probs: np.ndarray,
           wv_dtype: str = "f64", head_dim: int = 128) -> np.ndarray:
    """The value side of one query token's attention over L cached positions
    whose values are rematerialised from the compact cache ("IFM K2 Horizon
    Deep Dive", Section 4, Option B: x, the top-k indices and the stored
    weights per position; V recomputed inside attention):

        V = combine(x, idx, w, Wv) viewed as (L, n / 128, 128)  (KV heads)
        o[h] = sum over l of probs[h, l] * V[l, h // G],  G = H / (n / 128)

    (query heads grouped onto KV heads as in GQA, consecutive query heads
    sharing one).  probs: (H, L); returns o (H, head_dim) fp64."""
    V = as_gqa(combine(x, idx, w, Wv, wv_dtype), head_dim)
    H = probs.shape[0]
    G = H // V.shape[1]
    o = np.zeros((H, head_dim), dtype=np.float64)
    for h in range(H):
        o[h] = probs[h].astype(np.float64) @ V[:, h // G, :]
    return o


# ---------------------------------------------------------------------------
# Grouping of (token, slot) pairs by expert
# ---------------------------------------------------------------------------


def permutation(idx: np.ndarray, E: int):
    """Group the flat pairs f = t*k + slot by expert, stably.

    counts[e]   = number of pairs routed to e
    offsets[e]  = sum of counts[e'] for e' < e  (length E+1)
    perm[p]     = the flat pair at position p of the order sorted by
                  (expert, f)
    pos[f]      = the position of pair f in that order (perm's inverse)
    """
    flat = np.asarray(idx).reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int64)
    pos = np.empty_like(perm)
    pos[perm] = np.arange(perm.size, dtype=np.int64)
    return dict(counts=counts, offsets=offsets, perm=perm, pos=pos)


# ---------------------------------------------------------------------------
# Closed-form sizes ("So what does it cost?")
# ---------------------------------------------------------------------------


def expert_params_per_layer(E: int, d: int, n: int) -> int:
    """Stored value-expert parameters of one layer: E experts of n x d."""
    return E * d * n


def macs_per_token(d: int, n: int, k: int) -> int:
    """Expert multiply-accumulates per token: k projections of n x d."""
    return k * d * n


def router_params(d: int, E: int) -> int:
    """Router weights (without the E biases): E x d."""
    return d * E


def flops_per_token(d: int, n: int, k: int) -> int:
    """Expert flops per token, 2 per multiply-accumulate."""
    return 2 * macs_per_token(d, n, k)
