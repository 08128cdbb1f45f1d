"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Comparison rules are in tests/_parity.py."""
import ctypes

import numpy as np
import pytest
import torch

import mova_inputs as MI
from oracle import mova_oracle as O
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from mixture_value_routing_b200 import build
    build.build()
    from mixture_value_routing_b200 import api as A
    return A


def _layer(seed, d, E, n, dtype, bias="normal"):
    return MI.make_layer(seed, 0, d=d, E=E, n=n, wv_dtype=dtype, bias=bias)


def _routing_ref(bat, lay, k, scale=2.5):
    x = O.to_f64(bat.x, bat.x_dtype)
    return x, O.route(x, lay.Wr.astype(np.float64), lay.br.astype(np.float64), k, scale)


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

ROUTE_CASES = [
    # T, d, E, k, dtype
    (1, 256, 8, 1, "f32"),
    (3, 512, 64, 4, "bf16"),
    (8, 2560, 64, 4, "bf16"),
    (31, 256, 8, 8, "f32"),
    (33, 2560, 64, 4, "bf16"),
    (65, 1024, 17, 3, "f32"),
    (128, 2560, 64, 4, "f32"),
    (300, 2560, 64, 4, "bf16"),
    (4096, 2560, 64, 4, "bf16"),
]


@pytest.mark.parametrize("T,d,E,k,dtype", ROUTE_CASES)
def test_route(api, T, d, E, k, dtype):
    lay = _layer(11, d, E, 128, dtype)
    bat = MI.make_batch(T, 11, dtype=dtype, d=d)
    _, ref = _routing_ref(bat, lay, k)
    idx, w = api.route(P.dev(bat.x, dtype), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), k, 2.5)
    torch.cuda.synchronize()
    P.check_routing(idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), ref, k, 2.5)


def test_route_ties_go_to_lower_index(api):
    """Identical router rows and zero bias: all scores tie exactly, so the
    selection must be experts 0..k-1 in order."""
    d, E, k, T = 256, 16, 4, 5
    Wr = np.tile(np.random.default_rng(0).standard_normal(d).astype(np.float32) * 0.02, (E, 1))
    br = np.zeros(E, np.float32)
    x = np.random.default_rng(1).standard_normal((T, d)).astype(np.float32)
    idx, w = api.route(P.dev(x, "f32"), P.dev(Wr, "f32"), P.dev(br, "f32"), k, 2.5)
    assert (idx.cpu().numpy() == np.arange(k)[None, :]).all()
    np.testing.assert_allclose(w.cpu().numpy(), 2.5 / k, rtol=1e-6)


# ---------------------------------------------------------------------------
# Grouping by expert
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,kind", [
    (1, 64, 4, "distinct"), (7, 5, 2, "distinct"), (33, 64, 8, "distinct"),
    (1000, 64, 4, "distinct"), (4096, 64, 4, "distinct"), (32768, 64, 4, "distinct"),
    (3000, 64, 4, "skewed"), (2000, 3, 3, "duplicates"), (999, 1, 1, "distinct"),
])
def test_permute(api, T, E, k, kind):
    rng = np.random.default_rng(T + E + k)
    if kind == "distinct":
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    elif kind == "skewed":
        p = 1.0 / np.arange(1, E + 1) ** 2.0
        idx = rng.choice(E, size=(T, k), p=p / p.sum()).astype(np.int32)
    else:
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    got = api.permute(P.dev(idx, "i32"), E)
    torch.cuda.synchronize()
    P.check_permutation(got, idx, E)


def test_permute_rejects_bad_index(api):
    idx = np.array([[0, 1], [2, 7], [1, 0]], np.int32)  # 7 >= E = 4
    got = api.permute(P.dev(idx, "i32"), 4)
    status, detail = api.get_status(got["ws"])
    assert status == "MOVA_ERR_DEVICE_CHECK" and detail == 3
    assert got["offsets"].cpu().numpy()[-1] == 6  # every pair still placed, none out of bounds


# ---------------------------------------------------------------------------
# Routing-given mixture (compact-cache recompute)
# ---------------------------------------------------------------------------

GIVEN_CASES = [
    # T, d, E, k, n, dtype, idx dtype, w dtype, path
    (5, 256, 8, 2, 128, "f32", "i32", "f32", "stream"),
    (5, 256, 8, 2, 128, "bf16", "i8", "f16", "stream"),
    (8, 2560, 64, 4, 1024, "bf16", "i8", "f16", "stream"),
    (37, 512, 4, 4, 256, "bf16", "i32", "f32", "stream"),
    (128, 2560, 64, 4, 1024, "f32", "i8", "f16", "stream"),
    (1, 64, 1, 1, 128, "f32", "i32", "f32", "stream"),
]


@pytest.mark.parametrize("T,d,E,k,n,dtype,idt,wdt,path", GIVEN_CASES)
def test_value_given(api, T, d, E, k, n, dtype, idt, wdt, path):
    lay = _layer(5, d, E, n, dtype)
    rng = np.random.default_rng(T * 7 + E)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    g = rng.exponential(1.0, size=(T, k))
    w = (2.5 * g / g.sum(axis=1, keepdims=True))
    w = w.astype(np.float16 if wdt == "f16" else np.float32)
    bat = MI.make_batch(T, 5, dtype=dtype, d=d)
    v = api.value(P.dev(bat.x, dtype), P.dev(idx, idt), P.dev(w, wdt), P.dev(lay.Wv, dtype),
                  path=path)
    torch.cuda.synchronize()
    status, _ = api.get_status()
    assert status == "MOVA_OK"
    x = O.to_f64(bat.x, dtype)
    v_ref = O.combine(x, idx, w.astype(np.float64), lay.Wv, dtype)
    assert v.shape == (T, n) and v.dtype == (torch.bfloat16 if dtype == "bf16" else torch.float32)
    P.check_values(P.host_f64(v), v_ref, dtype)


def test_value_given_duplicate_experts(api):
    """A stored routing may name one expert in several slots of a token: every
    pair still counts once (here one expert receives all 6 x 4 pairs)."""
    d, E, k, n, T = 512, 8, 4, 256, 6
    lay = _layer(8, d, E, n, "bf16")
    bat = MI.make_batch(T, 8, dtype="bf16", d=d)
    idx = np.full((T, k), 3, np.int32)
    idx[0, 1] = 5
    w = np.random.default_rng(3).random((T, k)).astype(np.float32)
    v = api.value(P.dev(bat.x, "bf16"), P.dev(idx, "i32"), P.dev(w, "f32"), P.dev(lay.Wv, "bf16"),
                  path="stream")
    torch.cuda.synchronize()
    v_ref = O.combine(O.to_f64(bat.x, "bf16"), idx, w.astype(np.float64), lay.Wv, "bf16")
    P.check_values(P.host_f64(v), v_ref, "bf16")


def test_value_given_bad_index_is_flagged(api):
    d, E, k, n, T = 256, 8, 2, 128, 4
    lay = _layer(6, d, E, n, "bf16")
    bat = MI.make_batch(T, 6, dtype="bf16", d=d)
    idx = np.array([[0, 1], [2, 3], [4, -1], [6, 7]], np.int8)
    w = np.full((T, k), 1.25, np.float16)
    v = api.value(P.dev(bat.x, "bf16"), P.dev(idx, "i8"), P.dev(w, "f16"), P.dev(lay.Wv, "bf16"))
    status, detail = api.get_status()
    assert status == "MOVA_ERR_DEVICE_CHECK" and detail == 5
    assert torch.isfinite(v.float()).all()


# ---------------------------------------------------------------------------
# Full path
# ---------------------------------------------------------------------------

def _full(api, T, d, E, k, n, dtype, seed=0, bias="normal", sample=None, path="auto", record=None):
    """The whole path through mova_value_routed: routing against the oracle's
    (near-tie rule), the grouping the expert kernels actually ran on (read back
    from the workspace) bit-exact against the oracle's stable counting sort of
    the GPU's routing, and the values (every token, or a seeded sample)."""
    lay = _layer(seed, d, E, n, dtype, bias)
    bat = MI.make_batch(T, seed, dtype=dtype, d=d)
    x, ref = _routing_ref(bat, lay, k)
    ws = torch.empty(api.workspace_size(T, d, E, k, n), dtype=torch.uint8, device="cuda")
    v, idx, w = api.value_routed(P.dev(bat.x, dtype), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"),
                                 P.dev(lay.Wv, dtype), k, 2.5, return_routing=True, path=path, ws=ws)
    torch.cuda.synchronize()
    assert api.get_status(ws)[0] == "MOVA_OK"
    idx_g = idx.cpu().numpy().astype(np.int64)
    rc = P.check_routing(idx_g, w.cpu().numpy().astype(np.float64), ref, k, 2.5)
    P.check_permutation(api.grouping(ws, T, d, E, k, n), idx_g, E)
    rows = np.arange(T) if sample is None else np.sort(
        np.random.default_rng(seed + 99).choice(T, size=min(sample, T), replace=False))
    # Values of the GPU's (validated) selection with the oracle's weights.
    w_ref = O.weights_for(ref["s"][rows], idx_g[rows], 2.5)
    v_ref = O.combine(x[rows], idx_g[rows], w_ref, lay.Wv, dtype)
    err = P.check_values(P.host_f64(v)[rows], v_ref, dtype)
    if record is not None:
        record("near_tie_tokens", int(rc.near.size))
        record("differently_chosen_near_ties", int(rc.differ.size))
        record("value_rows_checked", int(rows.size))
        record("max_abs_err", err)
    return err, v, idx


def test_full_pr1_fp32(api):
    """T=128, all fp32, d=2560, 64 experts, top-4 (every output element)."""
    _full(api, 128, 2560, 64, 4, 1024, "f32")


def test_full_decode_bf16(api):
    """T=8 bf16 decode step at full dimensions (every output element)."""
    _full(api, 8, 2560, 64, 4, 1024, "bf16")


@pytest.mark.parametrize("T,E,k,n", [(1, 64, 4, 1024), (2, 8, 8, 128), (3, 1, 1, 256),
                                     (17, 16, 4, 384)])
def test_full_edge_shapes(api, T, E, k, n):
    _full(api, T, 256, E, k, n, "bf16", seed=T)


@pytest.mark.parametrize("T,d,E,k,n", [(8, 256, 16, 4, 2048), (8, 2560, 64, 8, 1024), (7, 512, 64, 8, 128)])
def test_full_decode_column_ranges(api, T, d, E, k, n):
    """Decode batches whose CTAs own more than 8 output columns (n = 2048:
    13 or 14 per CTA), whose SiLU tiles need the largest buffer (k = 8 of 64
    experts: up to 64 active, which leaves room for three weight stages), and
    whose slabs each span up to 8 experts (n = 128: one column per CTA, some
    CTAs none)."""
    _full(api, T, d, E, k, n, "bf16", seed=n + k, path="stream")


def test_full_stream_widest_rows_many_experts(api):
    """Decode batch with wide rows (d = 4544) and k = 8 of 64 experts, n =
    1024: the resident mode's buffers do not fit next to its x tile and two
    stages, so the batch takes the per-chunk mode with a separate combine,
    and is still supported."""
    _full(api, 8, 4544, 64, 8, 1024, "bf16", seed=4544, path="stream")


@pytest.mark.parametrize("T,d", [(8, 3072), (4, 4096), (3, 4544), (8, 4608)])
def test_full_stream_resident_boundary(api, T, d):
    """Decode batches at and near the widest rows the weight-streaming
    kernel holds: two stages of 8 rows plus the x tile (resident up to
    d = 4544 here; d = 4608 runs the per-chunk mode)."""
    _full(api, T, d, 16, 4, 256, "bf16", seed=d, path="stream")


@pytest.mark.parametrize("T,n", [(8, 128), (1, 128), (5, 384)])
def test_full_stream_fewer_columns_than_ctas(api, T, n):
    """Decode batches whose n output columns are fewer than, or not a
    multiple of, the CTAs the streaming kernel runs (one per SM): at n = 128
    some CTAs own no column at all and must leave without work, the others
    one; every value still matches the oracle."""
    _full(api, T, 2560, 64, 4, n, "bf16", seed=n + T, path="stream")


@pytest.mark.parametrize("T", [24, 64])
def test_full_stream_mid(api, T):
    """Weight-streaming path with more than 8 tokens on some experts."""
    _full(api, T, 2560, 64, 4, 1024, "bf16", seed=T, path="stream")


# ---------------------------------------------------------------------------
# tcgen05 grouped GEMM (bf16)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,d,E,k,n", [(1, 256, 8, 4, 128), (3, 512, 64, 4, 256), (40, 256, 4, 2, 384),
                                       (300, 2560, 64, 4, 1024), (700, 512, 2, 2, 128)])
@pytest.mark.parametrize("path", ["tensor", "tensor_1cta"])
def test_full_tensor_path(api, T, d, E, k, n, path):
    """The tcgen05 paths (SM-pair and single-CTA grouped GEMM) at small and
    ragged sizes: one token, tiles of 16, n not a multiple of 256 (the odd
    CTA's weight rows run past the expert), several token tiles per expert
    (700 x 2 pairs over 2 experts = 3 token tiles)."""
    _full(api, T, d, E, k, n, "bf16", seed=T + 1, path=path)


def test_tensor_given(api):
    d, E, k, n, T = 512, 8, 4, 256, 333
    lay = _layer(9, d, E, n, "bf16")
    bat = MI.make_batch(T, 9, dtype="bf16", d=d, mode="given", E=E, k=k)
    v = api.value(P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16"),
                  P.dev(lay.Wv, "bf16"), path="tensor")
    torch.cuda.synchronize()
    assert api.get_status()[0] == "MOVA_OK"
    v_ref = O.combine(O.to_f64(bat.x, "bf16"), bat.idx.astype(np.int64), bat.w.astype(np.float64),
                      lay.Wv, "bf16")
    P.check_values(P.host_f64(v), v_ref, "bf16")


@pytest.mark.parametrize("path", ["auto", "tensor_1cta"])
def test_full_prefill_4096(api, path, record_property):
    """Prefill workload at full size (T=4096): routing, grouping and the value
    of every token, element by element."""
    _full(api, 4096, 2560, 64, 4, 1024, "bf16", path=path, record=record_property)


def test_full_skewed_16384(api, record_property):
    """Skewed prefill (router bias 2 ln Zipf(1.2)), T=16384: routing and
    grouping of every token, values of 1024 sampled tokens."""
    _full(api, 16384, 2560, 64, 4, 1024, "bf16", bias="zipf", sample=1024, record=record_property)


def test_given_32768(api):
    """Routing-given recompute at L=32768 (int8 indices, fp16 weights): the
    grouping of every pair bit-exact, values of 1024 sampled rows."""
    L, d, E, k, n = 32768, 2560, 64, 4, 1024
    lay = _layer(0, d, E, n, "bf16")
    bat = MI.make_batch(L, 0, dtype="bf16", mode="given")
    ws = torch.empty(api.workspace_size(L, d, E, k, n), dtype=torch.uint8, device="cuda")
    v = api.value(P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16"),
                  P.dev(lay.Wv, "bf16"), ws=ws)
    torch.cuda.synchronize()
    assert api.get_status(ws)[0] == "MOVA_OK"
    P.check_permutation(api.grouping(ws, L, d, E, k, n), bat.idx.astype(np.int64), E)
    rows = np.sort(np.random.default_rng(5).choice(L, 1024, replace=False))
    v_ref = O.combine(O.to_f64(bat.x[rows], "bf16"), bat.idx[rows].astype(np.int64),
                      bat.w[rows].astype(np.float64), lay.Wv, "bf16")
    P.check_values(P.host_f64(v)[rows], v_ref, "bf16")


# ---------------------------------------------------------------------------
# Attend: the PV product with V recomputed from the compact cache
# ---------------------------------------------------------------------------


def _attend_ref(bat, lay, probs, rows=None):
    x = O.to_f64(bat.x, "bf16")
    idx = bat.idx.astype(np.int64)
    w = bat.w.astype(np.float64)
    p = probs.astype(np.float64)
    if rows is not None:
        x, idx, w, p = x[rows], idx[rows], w[rows], p[:, rows]
    return O.attend(x, idx, w, lay.Wv, p, "bf16")


@pytest.mark.parametrize("L,H", [(1, 32), (65, 32), (300, 8), (1000, 32), (4096, 16)])
def test_value_attend(api, L, H):
    """o (H, 128) against the oracle's attend: the experts' dot products and
    SiLU in fp32, weighted by p * w in fp32, summed per tile and then over
    tiles in a fixed order; |err| <= 1e-4 max(1, |ref|)."""
    d, E, k, n = 2560, 64, 4, 1024
    lay = _layer(51, d, E, n, "bf16")
    bat = MI.make_batch(L, 51, dtype="bf16", mode="given")
    probs = MI.make_attention_probs(H, L, 51)
    o = api.value_attend(P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16"),
                         P.dev(lay.Wv, "bf16"), torch.from_numpy(probs).cuda())
    torch.cuda.synchronize()
    assert o.shape == (H, 128) and o.dtype == torch.float32
    ref = _attend_ref(bat, lay, probs)
    err = np.abs(o.cpu().numpy().astype(np.float64) - ref)
    assert (err <= 1e-4 * np.maximum(1.0, np.abs(ref))).all(), err.max()


def test_value_attend_i32_f32_routing(api):
    """int32 indices and fp32 weights (the other accepted compact-cache
    formats), E = 16, k = 2, n = 512 (4 KV heads, 4 query heads each)."""
    d, E, k, n, L, H = 1024, 16, 2, 512, 700, 16
    lay = _layer(55, d, E, n, "bf16")
    bat = MI.make_batch(L, 55, dtype="bf16", d=d, mode="given", E=E, k=k)
    probs = MI.make_attention_probs(H, L, 55)
    o = api.value_attend(P.dev(bat.x, "bf16"), P.dev(bat.idx.astype(np.int32), "i32"),
                         P.dev(bat.w.astype(np.float32), "f32"), P.dev(lay.Wv, "bf16"),
                         torch.from_numpy(probs).cuda())
    torch.cuda.synchronize()
    ref = _attend_ref(bat, lay, probs)
    err = np.abs(o.cpu().numpy().astype(np.float64) - ref)
    assert (err <= 1e-4 * np.maximum(1.0, np.abs(ref))).all(), err.max()


def test_value_attend_one_hot_is_the_value_row(api):
    """All of head h's probability on position j: o[h] is row j of the value
    tensor (the routing-given call) in KV head h // G."""
    d, E, k, n, L, H = 2560, 64, 4, 1024, 200, 32
    lay = _layer(52, d, E, n, "bf16")
    bat = MI.make_batch(L, 52, dtype="bf16", mode="given")
    js = np.random.default_rng(52).integers(0, L, size=H)
    probs = np.zeros((H, L), dtype=np.float32)
    probs[np.arange(H), js] = 1.0
    args = (P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16"), P.dev(lay.Wv, "bf16"))
    o = api.value_attend(*args, torch.from_numpy(probs).cuda())
    v = api.value(*args, path="tensor")
    torch.cuda.synchronize()
    V = v.float().cpu().numpy().reshape(L, 8, 128)
    G = H // 8
    for h in range(H):
        # v is rounded to bf16 once; o is not
        np.testing.assert_allclose(o[h].cpu().numpy(), V[js[h], h // G], rtol=1e-2, atol=1e-2)


def test_value_attend_32768_sparse(api):
    """L = 32768 cached positions (the routing-given workload), every one
    recomputed on the GPU; each head's probability on 64 random positions,
    so the oracle needs only those."""
    d, E, k, n, L, H = 2560, 64, 4, 1024, 32768, 32
    lay = _layer(0, d, E, n, "bf16")
    bat = MI.make_batch(L, 0, dtype="bf16", mode="given")
    probs = MI.make_attention_probs(H, L, 53, support=64)
    o = api.value_attend(P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16"),
                         P.dev(lay.Wv, "bf16"), torch.from_numpy(probs).cuda())
    torch.cuda.synchronize()
    rows = np.nonzero(probs.any(axis=0))[0]
    ref = _attend_ref(bat, lay, probs, rows)
    err = np.abs(o.cpu().numpy().astype(np.float64) - ref)
    assert (err <= 1e-4 * np.maximum(1.0, np.abs(ref))).all(), err.max()


def test_value_attend_zero_positions(api):
    """No cached positions: o is zero (nothing to attend to)."""
    Wv = P.dev(_layer(56, 256, 8, 256, "bf16").Wv, "bf16")
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    o = api.value_attend(x, idx, w, Wv, torch.empty((8, 0), dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert o.shape == (8, 128) and not o.any()


def test_value_attend_deterministic(api):
    d, E, k, n, L, H = 2560, 64, 4, 1024, 3000, 32
    lay = _layer(54, d, E, n, "bf16")
    bat = MI.make_batch(L, 54, dtype="bf16", mode="given")
    probs = torch.from_numpy(MI.make_attention_probs(H, L, 54)).cuda()
    args = (P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16"), P.dev(lay.Wv, "bf16"), probs)
    first = api.value_attend(*args).clone()
    for _ in range(3):
        assert torch.equal(api.value_attend(*args), first)


def test_back_to_back_sizes_share_a_workspace(api):
    """A large bf16 call followed, with no synchronisation, by a smaller one on
    the same stream and the same workspace: the second call's kernels start
    while the first call's last kernels may still run (programmatic dependent
    launch), and the workspace offsets of the two layouts overlap.  Both
    results must match the oracle."""
    d, E, k, n = 2560, 64, 4, 1024
    lay = _layer(31, d, E, n, "bf16")
    ws = torch.empty(api.workspace_size(4096, d, E, k, n), dtype=torch.uint8, device="cuda")
    args = (P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16"))
    outs = []
    for T, seed in ((4096, 31), (128, 32), (8, 33), (4096, 34)):
        bat = MI.make_batch(T, seed, dtype="bf16", d=d)
        v, idx, _ = api.value_routed(P.dev(bat.x, "bf16"), *args, k, 2.5, return_routing=True, ws=ws)
        outs.append((bat, v, idx))
    torch.cuda.synchronize()
    assert api.get_status(ws)[0] == "MOVA_OK"
    for bat, v, idx in outs:
        x, ref = _routing_ref(bat, lay, k)
        idx_g = idx.cpu().numpy().astype(np.int64)
        rows = np.arange(min(bat.x.shape[0], 512))
        P.check_values(P.host_f64(v)[rows],
                       O.combine(x[rows], idx_g[rows], O.weights_for(ref["s"][rows], idx_g[rows], 2.5),
                                 lay.Wv, "bf16"), "bf16")


def test_tensor_deterministic(api):
    lay = _layer(4, 2560, 64, 1024, "bf16")
    bat = MI.make_batch(512, 4, dtype="bf16")
    args = (P.dev(bat.x, "bf16"), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"),
            P.dev(lay.Wv, "bf16"))
    first = api.value_routed(*args, path="tensor").clone()
    for _ in range(4):
        assert torch.equal(api.value_routed(*args, path="tensor"), first)


@pytest.mark.parametrize("T,d,E,k", [(65, 2560, 64, 4), (130, 512, 17, 3), (777, 256, 64, 8)])
def test_tensor_router_and_tile_grouping(api, T, d, E, k):
    """bf16 batches above 64 tokens route on the tensor cores (exact three-way
    bf16 split of the fp32 router) and group with the tile kernels; the
    expert step is forced onto the streaming kernel to isolate them."""
    _full(api, T, d, E, k, 256, "bf16", seed=T, path="stream")


@pytest.mark.parametrize("E,d", [(64, 2560), (17, 512)])
def test_router_planes_prepared(api, E, d):
    """mova_router_planes: the three bf16 planes sum exactly to the fp32 router
    weight (every plane's rows past E zero), and a call handed the prepared
    planes routes and computes bit for bit what a call that splits the
    weight itself does."""
    lay = _layer(41, d, E, 256, "bf16")
    Wr = P.dev(lay.Wr, "f32")
    planes = api.router_planes(Wr)
    torch.cuda.synchronize()
    pl = planes[: 3 * 64 * d].view(3, 64, d).double().cpu().numpy()
    assert np.array_equal(pl[0, :E] + pl[1, :E] + pl[2, :E], lay.Wr.astype(np.float32).astype(np.float64))
    assert not pl[:, E:].any()
    bat = MI.make_batch(300, 42, dtype="bf16", d=d)
    args = (P.dev(bat.x, "bf16"), Wr, P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16"), 4, 2.5)
    v0, i0, w0 = api.value_routed(*args, return_routing=True)
    v1, i1, w1 = api.value_routed(*args, return_routing=True, planes=planes)
    assert torch.equal(i0, i1) and torch.equal(w0, w1) and torch.equal(v0, v1)


def test_bounded_wait_reports_timeout(api):
    """A device wait that can never complete gives up after its limit and
    reports MOVA_ERR_TIMEOUT; the context stays usable for a normal call."""
    from mixture_value_routing_b200 import _lib
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.mova_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), 2_000_000, stream) == _lib.OK
    status, _ = api.get_status(ws)
    assert status == "MOVA_ERR_TIMEOUT"
    _full(api, 8, 256, 8, 2, 128, "bf16", seed=77)


def test_stream_stall_reports_timeout_and_recovers(api):
    """Failure detection in the weight-streaming kernel itself: the first CTA
    stops issuing weight copies at stage 2 and the waits are limited to about
    a millisecond, so its consumers' wait must run out.  The call reports
    MOVA_ERR_TIMEOUT, every warp leaves (the call completes), and the next
    call on the same context gives correct values."""
    lay = _layer(41, 2560, 64, 1024, "bf16")
    bat = MI.make_batch(8, 41, dtype="bf16")
    args = (P.dev(bat.x, "bf16"), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16"))
    ws = torch.empty(api.workspace_size(8, 2560, 64, 4, 1024), dtype=torch.uint8, device="cuda")
    api.arm_stream_stall(2, 2_000_000)
    api.value_routed(*args, ws=ws)
    status, detail = api.get_status(ws)
    assert status == "MOVA_ERR_TIMEOUT" and detail == 0  # the first CTA gave up
    _full(api, 8, 2560, 64, 4, 1024, "bf16", seed=41)


def test_full_zero_tokens(api):
    lay = _layer(0, 256, 8, 128, "bf16")
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    v = api.value_routed(x, P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16"))
    assert v.shape == (0, 128)


def test_full_gqa_view(api):
    _, v, _ = _full(api, 8, 2560, 64, 4, 1024, "bf16", seed=3)
    g = v.view(8, 8, 128)
    assert torch.equal(g[2, 5], v[2, 5 * 128:6 * 128])


def test_deterministic(api):
    lay = _layer(2, 2560, 64, 1024, "bf16")
    bat = MI.make_batch(8, 2, dtype="bf16")
    args = (P.dev(bat.x, "bf16"), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"),
            P.dev(lay.Wv, "bf16"))
    first = api.value_routed(*args).clone()
    for _ in range(9):
        assert torch.equal(api.value_routed(*args), first)


def test_decode_step_kernel_count(api):
    """A bf16 decode step is one persistent kernel with decode_launches=1
    (logits, grid barrier, selection, grouping, weight stream, combine), or
    two by default (the logits kernel, then the streaming kernel); fp32 runs
    selection/grouping and the combine as kernels of their own."""
    for dtype, launches, want in (("bf16", 1, 1), ("bf16", 0, 2), ("bf16", 2, 2), ("f32", 0, 4)):
        lay = _layer(5, 2560, 64, 1024, dtype)
        bat = MI.make_batch(8, 5, dtype=dtype)
        args = (P.dev(bat.x, dtype), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, dtype))
        api.value_routed(*args, decode_launches=launches)
        torch.cuda.synchronize()
        before = api.launch_count()
        api.value_routed(*args, decode_launches=launches)
        assert api.launch_count() - before == want, (dtype, launches)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T", [1, 8])
def test_decode_two_launches(api, T):
    """The two-launch decode path (logits kernel + streaming kernel) gives the
    same values as the one-launch kernel, bit for bit, and passes the full
    parity checks."""
    lay = _layer(12, 2560, 64, 1024, "bf16")
    bat = MI.make_batch(T, 12, dtype="bf16")
    args = (P.dev(bat.x, "bf16"), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16"))
    one = api.value_routed(*args, decode_launches=1).clone()
    two, idx, w = api.value_routed(*args, return_routing=True, decode_launches=2)
    torch.cuda.synchronize()
    assert torch.equal(one, two)
    x, ref = _routing_ref(bat, lay, 4)
    idx_g = idx.cpu().numpy().astype(np.int64)
    P.check_routing(idx_g, w.cpu().numpy().astype(np.float64), ref, 4, 2.5)
    P.check_values(P.host_f64(two), O.combine(x, idx_g, O.weights_for(ref["s"], idx_g, 2.5), lay.Wv, "bf16"),
                   "bf16")


def test_decode_grid_barrier_timeout_and_recovery(api):
    """The one-launch decode kernel's grid barrier is a bounded wait: with the
    first CTA armed not to arrive and the waits limited to about a
    millisecond, every CTA gives up, the call reports MOVA_ERR_TIMEOUT and
    completes; reading the status restores the barrier words, and the next
    calls (more than the ring of barrier words, so the damaged word comes
    round again) give correct values."""
    lay = _layer(43, 2560, 64, 1024, "bf16")
    bat = MI.make_batch(8, 43, dtype="bf16")
    args = (P.dev(bat.x, "bf16"), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16"))
    ws = torch.empty(api.workspace_size(8, 2560, 64, 4, 1024), dtype=torch.uint8, device="cuda")
    ref = api.value_routed(*args, decode_launches=2).clone()
    api.arm_stream_stall(-2, 2_000_000)
    api.value_routed(*args, ws=ws, decode_launches=1)
    assert api.get_status(ws)[0] == "MOVA_ERR_TIMEOUT"
    for _ in range(70):
        assert torch.equal(api.value_routed(*args, ws=ws, decode_launches=1), ref)
    assert api.get_status(ws)[0] == "MOVA_OK"


# ---------------------------------------------------------------------------
# Router partitions (mova_options.router_partitions = 2)
# ---------------------------------------------------------------------------

def _cancel_inputs(T, d, E, dtype):
    """Every token: expert 0's first half of d sums to 2^25 and its second
    half to -2^25 + 1, which fp32 rounds to -2^25 (a tie, to even): the
    partitioned logit is 0, the exact one 1.  Other experts' logits are 0."""
    x = np.zeros((T, d), np.float32)
    Wr = np.zeros((E, d), np.float32)
    h = d // 2
    x[:, 0] = x[:, h] = 2.0 ** 12
    x[:, h + 1] = 1.0
    Wr[0, 0], Wr[0, h], Wr[0, h + 1] = 2.0 ** 13, -2.0 ** 13, 1.0
    br = np.full(E, -1.0, np.float32)
    br[0], br[1] = 0.0, 0.1
    xs = MI.f32_to_bf16_bits(x) if dtype == "bf16" else x
    return xs, Wr, br


@pytest.mark.parametrize("T,dtype", [(1, "bf16"), (8, "bf16"), (8, "f32"), (16, "f32"), (40, "bf16")])
def test_route_partitions_cancellation(api, T, dtype):
    """The fp32 CUDA-core routers in two-partition mode (the tiled router of
    mova_route, and for decode batches of the full path the logits kernel)
    take the selection the partitioned oracle takes, which differs from the
    exact one.  (The tensor-core router is checked on random inputs below:
    how its accumulator rounds a 16-product block sum is not specified, so
    this exact tie is not asked of it.)"""
    d, E, k = 128, 8, 2
    xs, Wr, br = _cancel_inputs(T, d, E, dtype)
    x64 = O.to_f64(xs, dtype)
    ref = O.route(x64, Wr.astype(np.float64), br.astype(np.float64), k, 2.5, partitions=2)
    exact = O.route(x64, Wr.astype(np.float64), br.astype(np.float64), k, 2.5)
    assert (ref["idx"] == [1, 0]).all() and (exact["idx"] == [0, 1]).all()
    idx, w = api.route(P.dev(xs, dtype), P.dev(Wr, "f32"), P.dev(br, "f32"), k, 2.5, partitions=2)
    torch.cuda.synchronize()
    assert (idx.cpu().numpy() == ref["idx"]).all()
    np.testing.assert_allclose(w.cpu().numpy(), 1.25, rtol=1e-6)
    if dtype == "bf16" and T <= 8:
        # The decode batches of the full path route in the logits kernel.
        Wv = _layer(3, d, E, 128, "bf16").Wv
        for launches in (1, 2):  # the one-launch kernel and the logits kernel
            _, idx2, w2 = api.value_routed(P.dev(xs, dtype), P.dev(Wr, "f32"), P.dev(br, "f32"),
                                           P.dev(Wv, "bf16"), k, 2.5, return_routing=True, partitions=2,
                                           decode_launches=launches)
            torch.cuda.synchronize()
            assert (idx2.cpu().numpy() == ref["idx"]).all()
            np.testing.assert_allclose(w2.cpu().numpy(), 1.25, rtol=1e-6)


@pytest.mark.parametrize("T,d,dtype", [(8, 2560, "bf16"), (33, 2560, "bf16"), (130, 2560, "bf16"),
                                       (4096, 2560, "bf16"), (128, 2560, "f32")])
def test_route_partitions_random(api, T, d, dtype):
    """Two-partition routing on random inputs, every router kernel (decode
    logits, tiled SIMT, tensor-core with two accumulators), against the
    partitioned oracle under the near-tie rule."""
    E, k = 64, 4
    lay = _layer(13, d, E, 128, dtype)
    bat = MI.make_batch(T, 13, dtype=dtype, d=d)
    x = O.to_f64(bat.x, dtype)
    ref = O.route(x, lay.Wr.astype(np.float64), lay.br.astype(np.float64), k, 2.5, partitions=2)
    idx, w = api.route(P.dev(bat.x, dtype), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), k, 2.5,
                       partitions=2)
    torch.cuda.synchronize()
    P.check_routing(idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), ref, k, 2.5)


@pytest.mark.parametrize("T", [8, 300])
def test_value_routed_partitions(api, T):
    """The whole path in two-partition mode: routing as the partitioned
    oracle's, values of the GPU's selection."""
    d, E, k, n = 2560, 64, 4, 1024
    lay = _layer(17, d, E, n, "bf16")
    bat = MI.make_batch(T, 17, dtype="bf16", d=d)
    x = O.to_f64(bat.x, "bf16")
    ref = O.route(x, lay.Wr.astype(np.float64), lay.br.astype(np.float64), k, 2.5, partitions=2)
    v, idx, w = api.value_routed(P.dev(bat.x, "bf16"), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"),
                                 P.dev(lay.Wv, "bf16"), k, 2.5, return_routing=True, partitions=2)
    torch.cuda.synchronize()
    idx_g = idx.cpu().numpy().astype(np.int64)
    P.check_routing(idx_g, w.cpu().numpy().astype(np.float64), ref, k, 2.5)
    rows = np.arange(min(T, 128))
    v_ref = O.combine(x[rows], idx_g[rows], O.weights_for(ref["s"][rows], idx_g[rows], 2.5), lay.Wv, "bf16")
    P.check_values(P.host_f64(v)[rows], v_ref, "bf16")


def test_partitions_unsupported_width(api):
    from mixture_value_routing_b200 import _lib
    x = torch.zeros((4, 192), dtype=torch.bfloat16, device="cuda")  # 192 % 128 != 0
    with pytest.raises(_lib.MovaError) as e:
        api.route(x, torch.zeros((8, 192), device="cuda"), torch.zeros(8, device="cuda"), 2, 2.5,
                  partitions=2)
    assert e.value.code == _lib.ERR_UNSUPPORTED


# ---------------------------------------------------------------------------
# Head-parallel slices (mova_options.wv_expert_stride)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,path", [(8, "auto"), (24, "auto"), (300, "auto"), (300, "tensor_1cta"),
                                    (4096, "auto")])
def test_head_parallel_slices(api, T, path):
    """Two ranks' halves of the 8 value heads (rows 0..511 and 512..1023 of
    every expert, read in place from the full Wv): each equals the oracle's
    columns and, concatenated, the full call bit for bit (the same dot
    products in the same order)."""
    d, E, k, n = 2560, 64, 4, 1024
    lay = _layer(23, d, E, n, "bf16")
    bat = MI.make_batch(T, 23, dtype="bf16", d=d)
    args = (P.dev(bat.x, "bf16"), P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16"))
    full, idx, _ = api.value_routed(*args, return_routing=True, path=path)
    halves = [api.value_routed(*args, path=path, rows=(r * 512, 512)) for r in range(2)]
    torch.cuda.synchronize()
    for h in halves:
        assert h.shape == (T, 512)
    assert torch.equal(torch.cat(halves, dim=1), full)
    x, ref = _routing_ref(bat, lay, k)
    idx_g = idx.cpu().numpy().astype(np.int64)
    rows = np.arange(min(T, 256))
    v_ref = O.combine(x[rows], idx_g[rows], O.weights_for(ref["s"][rows], idx_g[rows], 2.5), lay.Wv, "bf16")
    for r, h in enumerate(halves):
        P.check_values(P.host_f64(h)[rows], v_ref[:, r * 512:(r + 1) * 512], "bf16")


def test_head_parallel_given(api):
    """Routing-given recompute of one head slice (rows 256..639, three heads)."""
    d, E, k, n, T = 512, 8, 4, 1024, 333
    lay = _layer(9, d, E, n, "bf16")
    bat = MI.make_batch(T, 9, dtype="bf16", d=d, mode="given", E=E, k=k)
    v = api.value(P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16"), P.dev(lay.Wv, "bf16"),
                  rows=(256, 384))
    torch.cuda.synchronize()
    v_ref = O.combine(O.to_f64(bat.x, "bf16"), bat.idx.astype(np.int64), bat.w.astype(np.float64),
                      lay.Wv, "bf16")
    P.check_values(P.host_f64(v), v_ref[:, 256:640], "bf16")


# ---------------------------------------------------------------------------
# Host-buffer forms (batch and result in pinned host memory)
# ---------------------------------------------------------------------------

def _pinned(t):
    return t.cpu().pin_memory()


@pytest.mark.parametrize("T", [8, 300])
def test_value_routed_host_buffers(api, T):
    """mova_value_routed_host (copy in, the device call, copy out on one
    stream) gives the device form's v and routing bit for bit, and v against
    the oracle."""
    d, E, k, n = 2560, 64, 4, 1024
    lay = _layer(T + 3, d, E, n, "bf16")
    bat = MI.make_batch(T, T + 3, dtype="bf16", d=d)
    Wr, br, Wv = P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16")
    xd = P.dev(bat.x, "bf16")
    v_dev, idx_dev, w_dev = api.value_routed(xd, Wr, br, Wv, k, 2.5, return_routing=True)
    ws = torch.empty(api.workspace_size_host(T, d, E, k, n), dtype=torch.uint8, device="cuda")
    v, idx, w = api.value_routed_host(_pinned(xd), Wr, br, Wv, k, 2.5, ws=ws, return_routing=True)
    torch.cuda.synchronize()
    assert not v.is_cuda and v.shape == (T, n) and v.dtype == torch.bfloat16
    assert torch.equal(v, v_dev.cpu()) and torch.equal(idx, idx_dev.cpu()) and torch.equal(w, w_dev.cpu())
    x, ref = _routing_ref(bat, lay, k)
    idx_g = idx.numpy().astype(np.int64)
    P.check_routing(idx_g, w.numpy().astype(np.float64), ref, k, 2.5)
    rows = np.arange(min(T, 64))
    v_ref = O.combine(x[rows], idx_g[rows], O.weights_for(ref["s"][rows], idx_g[rows], 2.5), lay.Wv, "bf16")
    P.check_values(P.host_f64(v)[rows], v_ref, "bf16")


@pytest.mark.parametrize("T,path", [(37, "stream"), (1000, "auto")])
def test_value_host_buffers(api, T, path):
    """mova_value_host with int8 indices and fp16 weights in host memory gives
    the device form's v bit for bit, and v against the oracle."""
    d, E, k, n = 512, 16, 4, 256
    lay = _layer(T, d, E, n, "bf16")
    rng = np.random.default_rng(T)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int8)
    g = rng.exponential(1.0, size=(T, k))
    w = (2.5 * g / g.sum(axis=1, keepdims=True)).astype(np.float16)
    bat = MI.make_batch(T, T, dtype="bf16", d=d)
    xd, idxd, wd, Wv = P.dev(bat.x, "bf16"), P.dev(idx, "i8"), P.dev(w, "f16"), P.dev(lay.Wv, "bf16")
    v_dev = api.value(xd, idxd, wd, Wv, path=path)
    v = api.value_host(_pinned(xd), _pinned(idxd), _pinned(wd), Wv)
    torch.cuda.synchronize()
    assert torch.equal(v, v_dev.cpu())
    v_ref = O.combine(O.to_f64(bat.x, "bf16"), idx.astype(np.int64), w.astype(np.float64), lay.Wv, "bf16")
    P.check_values(P.host_f64(v), v_ref, "bf16")


@pytest.mark.parametrize("L", [0, 65])
def test_value_attend_host_buffers(api, L):
    """mova_value_attend_host: o equals the device form's bit for bit (zeros
    for L = 0, written through the workspace's staging)."""
    d, E, k, n, H = 2560, 64, 4, 1024, 32
    lay = _layer(52, d, E, n, "bf16")
    Wv = P.dev(lay.Wv, "bf16")
    if L == 0:
        x = torch.empty((0, d), dtype=torch.bfloat16).pin_memory()
        idx = torch.empty((0, k), dtype=torch.int8).pin_memory()
        w = torch.empty((0, k), dtype=torch.float16).pin_memory()
        p = torch.empty((H, 0), dtype=torch.float32).pin_memory()
        o = api.value_attend_host(x, idx, w, Wv, p, out=torch.full((H, 128), 7.0).pin_memory())
        torch.cuda.synchronize()
        assert torch.equal(o, torch.zeros((H, 128)))
        return
    bat = MI.make_batch(L, 52, dtype="bf16", mode="given")
    probs = MI.make_attention_probs(H, L, 52)
    xd, idxd, wd = P.dev(bat.x, "bf16"), P.dev(bat.idx, "i8"), P.dev(bat.w, "f16")
    pd = torch.from_numpy(probs).cuda()
    o_dev = api.value_attend(xd, idxd, wd, Wv, pd)
    o = api.value_attend_host(_pinned(xd), _pinned(idxd), _pinned(wd), Wv, _pinned(pd))
    torch.cuda.synchronize()
    assert torch.equal(o, o_dev.cpu())
    ref = _attend_ref(bat, lay, probs)
    err = np.abs(o.numpy().astype(np.float64) - ref)
    assert (err <= 1e-4 * np.maximum(1.0, np.abs(ref))).all(), err.max()


def test_host_buffer_calls_on_two_streams(api):
    """Two host-buffer calls in flight on two streams, each with its own
    workspace (as the benchmark's end-to-end loop runs them), give the same
    results as the same calls one after another: the library keeps no state
    between calls that two streams could share."""
    d, E, k, n = 2560, 64, 4, 1024
    lay = _layer(77, d, E, n, "bf16")
    Wr, br, Wv = P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16")
    batches = [MI.make_batch(T, 77, step=s, dtype="bf16", d=d) for s, T in enumerate((8, 8, 300, 300))]
    xs = [_pinned(P.dev(b.x, "bf16")) for b in batches]
    ref = [api.value_routed_host(x, Wr, br, Wv, k, 2.5) for x in xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(2)]
    wss = [torch.empty(api.workspace_size_host(300, d, E, k, n), dtype=torch.uint8, device="cuda")
           for _ in range(2)]
    for rep in range(3):
        outs = []
        for i, x in enumerate(xs):
            out = torch.empty((x.shape[0], n), dtype=torch.bfloat16).pin_memory()
            outs.append(api.value_routed_host(x, Wr, br, Wv, k, 2.5, out=out, ws=wss[i % 2],
                                              stream=streams[i % 2]))
        torch.cuda.synchronize()
        for i in range(len(xs)):
            assert torch.equal(outs[i], ref[i]), f"call {i} of round {rep} differs"


def test_default_workspaces_on_two_streams(api):
    """Calls given no workspace, in flight on two streams at once -- the
    host-buffer form with `stream=` and the device form under a stream
    context -- give the results of the same calls made one after another:
    each stream has a default workspace of its own, so no call reads another
    stream's routing, grouping or expert rows."""
    d, E, k, n = 2560, 64, 4, 1024
    lay = _layer(78, d, E, n, "bf16")
    Wr, br, Wv = P.dev(lay.Wr, "f32"), P.dev(lay.br, "f32"), P.dev(lay.Wv, "bf16")
    batches = [MI.make_batch(T, 78, step=s, dtype="bf16", d=d) for s, T in enumerate((8, 300, 8, 300))]
    xd = [P.dev(b.x, "bf16") for b in batches]
    xs = [_pinned(x) for x in xd]
    ref = [api.value_routed(x, Wr, br, Wv, k, 2.5).cpu() for x in xd]  # serial, current stream
    streams = [torch.cuda.Stream() for _ in range(2)]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    for rep in range(3):
        host_out = [api.value_routed_host(x, Wr, br, Wv, k, 2.5, stream=streams[i % 2]) for i, x in enumerate(xs)]
        dev_out = []
        for i, x in enumerate(xd):
            with torch.cuda.stream(streams[i % 2]):
                dev_out.append(api.value_routed(x, Wr, br, Wv, k, 2.5))
        torch.cuda.synchronize()
        for i in range(len(xs)):
            assert torch.equal(host_out[i], ref[i]), f"host-buffer call {i} of round {rep} differs"
            assert torch.equal(dev_out[i].cpu(), ref[i]), f"device call {i} of round {rep} differs"
    for s in streams:
        assert api.get_status(stream=s)[0] == "MOVA_OK"
