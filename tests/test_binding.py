"""Host logic of the Python binding, without a GPU: the workspaces that calls
made without `ws` use.  Calls on different streams may overlap on the GPU, so
each (device, stream) gets its own workspace; calls on one stream share it,
and it is allocated with its stream current, so that torch's caching
allocator ties the memory to the stream that uses it."""
import contextlib

import pytest
import torch

from mixture_value_routing_b200 import api


class _FakeStream:
    def __init__(self, handle):
        self.cuda_stream = handle


@pytest.fixture
def fresh(monkeypatch):
    monkeypatch.setattr(api, "_WS", {})
    current = {"handle": 0x1000}
    monkeypatch.setattr(api, "_current_stream_handle", lambda: current["handle"])
    entered = []

    @contextlib.contextmanager
    def fake_stream_ctx(s):
        entered.append(s.cuda_stream)
        yield

    monkeypatch.setattr(api.torch.cuda, "stream", fake_stream_ctx)
    return current, entered


def test_one_workspace_per_stream(fresh):
    current, _ = fresh
    a = api._workspace(1000, "cpu")
    assert api._workspace(500, "cpu") is a  # same stream: reused
    current["handle"] = 0x2000
    b = api._workspace(1000, "cpu")
    assert b is not a and b.data_ptr() != a.data_ptr()
    current["handle"] = 0x1000
    assert api._workspace(1000, "cpu") is a
    assert len(api._WS) == 2


def test_workspace_grows_in_place_of_the_streams_own(fresh):
    current, _ = fresh
    a = api._workspace(1000, "cpu")
    big = api._workspace(5000, "cpu")
    assert big.numel() >= 5000 and big is not a
    assert api._WS[(torch.device("cpu"), current["handle"])].buf is big
    assert len(api._WS) == 1


def test_explicit_stream_allocates_with_that_stream_current(fresh):
    current, entered = fresh
    s = _FakeStream(0x3000)
    a = api._workspace(1000, "cpu", s)
    assert entered == [0x3000]
    assert (torch.device("cpu"), 0x3000) in api._WS
    assert api._workspace(1000, "cpu") is not a  # the current stream has its own
    assert api._workspace(800, "cpu", _FakeStream(0x3000)) is a


def test_status_without_a_call_on_this_stream_is_an_error(fresh):
    current, _ = fresh
    api._workspace(1000, "cpu")
    current["handle"] = 0x5000
    with pytest.raises(ValueError, match="default workspace"):
        api.get_status(device="cpu")


def test_release_drops_every_default_workspace(fresh):
    current, _ = fresh
    api._workspace(1000, "cpu")
    current["handle"] = 0x2000
    api._workspace(1000, "cpu")
    assert len(api._WS) == 2
    api.release_workspaces()
    assert api._WS == {}
    with pytest.raises(ValueError):
        api.get_status(device="cpu")


class _Tensor:
    """Shape-only stand-in for a device tensor: the device checks are
    skipped below, so the shape checks run without a GPU."""

    def __init__(self, *shape, dtype=torch.bfloat16):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device("cpu")

    def dim(self):
        return len(self.shape)


@pytest.mark.parametrize("case", ["Wr rows", "Wr width", "br", "Wv width", "out"])
def test_value_routed_refuses_mismatched_shapes(monkeypatch, case):
    """A tensor whose shape disagrees with x's and Wv's is refused before
    the library sees its pointer (which it would read or write out of bounds)."""
    monkeypatch.setattr(api, "_need", lambda *a, **k: None)
    T, d, E, n = 8, 2560, 64, 1024
    x, Wv = _Tensor(T, d), _Tensor(E, n, d)
    Wr, br, out = _Tensor(E, d, dtype=torch.float32), _Tensor(E, dtype=torch.float32), _Tensor(T, n)
    if case == "Wr rows":
        Wr = _Tensor(E - 1, d, dtype=torch.float32)
    elif case == "Wr width":
        Wr = _Tensor(E, d - 64, dtype=torch.float32)
    elif case == "br":
        br = _Tensor(E + 1, dtype=torch.float32)
    elif case == "Wv width":
        Wv = _Tensor(E, n, d - 64)
    else:
        out = _Tensor(T - 1, n)
    with pytest.raises(ValueError, match="shape"):
        api.value_routed(x, Wr, br, Wv, out=out)


@pytest.mark.parametrize("case", ["idx rows", "w shape", "Wv width"])
def test_value_refuses_mismatched_shapes(monkeypatch, case):
    monkeypatch.setattr(api, "_need", lambda *a, **k: None)
    T, d, E, n, k = 8, 2560, 64, 1024, 4
    x, Wv = _Tensor(T, d), _Tensor(E, n, d)
    idx, w = _Tensor(T, k, dtype=torch.int8), _Tensor(T, k, dtype=torch.float16)
    if case == "idx rows":
        idx = _Tensor(T - 1, k, dtype=torch.int8)
    elif case == "w shape":
        w = _Tensor(T, k + 1, dtype=torch.float16)
    else:
        Wv = _Tensor(E, n, d + 64)
    with pytest.raises(ValueError, match="shape"):
        api.value(x, idx, w, Wv)
