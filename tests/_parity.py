"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
running the fp64 oracle on the same inputs, and the comparison rules.

Comparison rules (all written here, in one place):
  * expert indices: bit-exact, except tokens whose oracle biased scores have a
    gap < NEAR_TIE between the k-th and (k+1)-th (membership) or between two
    adjacent selected experts (slot order); such tokens are logged, and the
    GPU's choice must still be a valid top-k within the tie band;
  * routing weights: |w_gpu - w_ref| <= W_ATOL + W_RTOL*|w_ref|, w_ref being
    the oracle's weights of the GPU's selection;
  * values: max |v_gpu - v_ref| <= TOL * max(1, |v_ref|) elementwise, with
    TOL = 1e-2 for bf16 outputs and 1e-4 for fp32 outputs;
  * grouping (counts, offsets, perm, pos): bit-exact.
"""
from __future__ import annotations

from typing import NamedTuple

import numpy as np
import torch

from oracle import mova_oracle as O

NEAR_TIE = 1e-5
W_ATOL = 1e-6
W_RTOL = 1e-5
TOL = {"bf16": 1e-2, "f32": 1e-4}


def dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Storage-format numpy array -> CUDA tensor of the same bits."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    if dtype == "f16":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float16)).cuda()
    if dtype == "i8":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).cuda()
    if dtype == "i32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    raise ValueError(dtype)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class RoutingCheck(NamedTuple):
    differ: np.ndarray  # tokens whose GPU selection differs from the oracle's (inside the band)
    near: np.ndarray    # every token with a near tie


def check_routing(idx_gpu: np.ndarray, w_gpu: np.ndarray, ref: dict, k: int, scale: float,
                  log=print) -> RoutingCheck:
    """Compare the GPU's routing with the oracle's.  Returns the near-tie
    tokens and those whose selection differs inside the near-tie band (their
    value references must use the GPU's selection)."""
    b = ref["b"]
    T, E = b.shape
    order = np.argsort(-b, axis=1, kind="stable")
    sb = np.take_along_axis(b, order, axis=1)
    member_gap = (sb[:, k - 1] - sb[:, k]) if k < E else np.full(T, np.inf)
    slot_gap = np.min(sb[:, :k - 1] - sb[:, 1:k], axis=1) if k > 1 else np.full(T, np.inf)
    differ = np.nonzero((idx_gpu != ref["idx"]).any(axis=1))[0]
    for t in differ:
        near = min(member_gap[t], slot_gap[t]) < NEAR_TIE
        assert near, (f"token {t}: GPU idx {idx_gpu[t].tolist()} != oracle {ref['idx'][t].tolist()} "
                      f"without a near tie (gaps {member_gap[t]:.3e}, {slot_gap[t]:.3e})")
        sel = idx_gpu[t]
        assert len(set(sel.tolist())) == k and (sel >= 0).all() and (sel < E).all()
        kth = sb[t, k - 1]
        assert (b[t, sel] >= kth - NEAR_TIE).all(), f"token {t}: GPU picked outside the tie band"
        assert (np.diff(b[t, sel]) <= NEAR_TIE).all(), f"token {t}: GPU slot order not descending"
        log(f"near-tie token {t}: gpu {sel.tolist()} oracle {ref['idx'][t].tolist()} "
            f"gap45={member_gap[t]:.3e} gap_slots={slot_gap[t]:.3e}")
    # Weights of the GPU's selection, from the oracle's unbiased scores.
    w_ref = O.weights_for(ref["s"], idx_gpu.astype(np.int64), scale)
    err = np.abs(w_gpu - w_ref)
    assert (err <= W_ATOL + W_RTOL * np.abs(w_ref)).all(), f"w max err {err.max():.3e}"
    near_all = np.nonzero(np.minimum(member_gap, slot_gap) < NEAR_TIE)[0]
    for t in near_all:
        if t not in set(differ.tolist()):
            log(f"near-tie token {t} (same choice): gap45={member_gap[t]:.3e} "
                f"gap_slots={slot_gap[t]:.3e}")
    log(f"routing of {T} tokens: {near_all.size} near-tie tokens, {differ.size} chosen differently "
        f"inside the band")
    return RoutingCheck(differ=differ, near=near_all)


def check_values(v_gpu: np.ndarray, v_ref: np.ndarray, dtype: str, what: str = "v"):
    tol = TOL[dtype]
    bound = tol * np.maximum(1.0, np.abs(v_ref))
    err = np.abs(v_gpu - v_ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance; worst err "
                           f"{err.max():.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}")
    return float(err.max())


def check_permutation(got: dict, idx: np.ndarray, E: int):
    ref = O.permutation(idx, E)
    for key in ("counts", "offsets", "perm", "pos"):
        g = got[key].cpu().numpy().astype(np.int64)
        assert (g == ref[key]).all(), f"{key} differs at {np.nonzero(g != ref[key])[0][:10]}"
