"""The no-allocation entry point, mova_value_routed_noalloc, for callers that
cannot allocate device memory where they run the value projection (inside a
stream capture, under a memory pool that owns the device, or as a plug-in that
is handed only its tensors).  It must give the same values as the regular
entry point, mova_value_routed, call after call, although every call reuses
the one workspace array built into the library -- including calls of
different sizes, which take different kernel sequences (T <= 8: the logits
kernel and the weight-streaming kernel with the combine fused in; 9 <= T <= 30:
the tiled router, the grouping kernel, the weight-streaming kernel and the
combine kernel).  Both entry points are also checked against the fp64 oracle.

This file is collected last on purpose and sets up everything it needs itself,
so it passes both on its own in a fresh process and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import mova_inputs as MI
from oracle import mova_oracle as O

pytestmark = pytest.mark.gpu

TOL = 1e-2  # bf16 outputs: |err| <= TOL * max(1, |ref|), as in the parity tests


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _within(v, ref):
    err = (v.double() - ref).abs()
    return bool(torch.isfinite(v.double()).all()) and bool((err <= TOL * torch.clamp(ref.abs(), min=1.0)).all())


@pytest.mark.parametrize("sizes", [(8, 8), (30, 30), (30, 8)], ids=lambda s: "T=" + "-then-".join(map(str, s)))
def test_noalloc_matches_regular_entry_point_on_consecutive_calls(sizes):
    assert torch.cuda.is_available(), "GPU test"
    from mixture_value_routing_b200 import _lib, build
    build.build()
    lib = _lib.load()
    from mixture_value_routing_b200 import api

    d, E, k, n = 2560, 64, 4, 1024
    lay = MI.make_layer(21, 0, wv_dtype="bf16")
    Wr = torch.from_numpy(lay.Wr).cuda()
    br = torch.from_numpy(lay.br).cuda()
    Wv = _dev_bf16(lay.Wv)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731

    for step, T in enumerate(sizes):  # calls in a row, different tokens each time
        bat = MI.make_batch(T, 21, step=step)
        x = _dev_bf16(bat.x)
        v_ref, idx, _ = api.value_routed(x, Wr, br, Wv, k, 2.5, return_routing=True)
        v = torch.full((T, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = lib.mova_value_routed_noalloc(p(x), _lib.BF16, p(Wr), p(br), p(Wv), _lib.BF16, T, d, E, k,
                                           n, 2.5, p(v), stream)
        assert st == _lib.OK, _lib.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        assert _within(v, v_ref.double()), f"call {step} (T={T}): differs from mova_value_routed"
        # Both against the oracle, with the oracle's weights of the GPU's selection.
        x64 = O.to_f64(bat.x, "bf16")
        r = O.route(x64, lay.Wr.astype(np.float64), lay.br.astype(np.float64), k, 2.5)
        idx_g = idx.cpu().numpy().astype(np.int64)
        oracle = torch.from_numpy(O.combine(x64, idx_g, O.weights_for(r["s"], idx_g, 2.5), lay.Wv, "bf16"))
        assert _within(v.cpu(), oracle), f"call {step} (T={T}): differs from the oracle"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from mixture_value_routing_b200 import _lib, build
    build.build()
    lib = _lib.load()
    T, d, E, k, n = 4096, 2560, 64, 4, 1024
    assert lib.mova_workspace_size(T, d, E, k, n) > (2 << 20)
    fake = ctypes.c_void_p(4096)  # rejected before any pointer is used
    st = lib.mova_value_routed_noalloc(fake, _lib.BF16, fake, fake, fake, _lib.BF16, T, d, E, k, n, 2.5,
                                       fake, None)
    assert st == _lib.ERR_UNSUPPORTED
