"""Python face of the MoVA value path: the C ABI of libmova.so, called with
torch CUDA tensors (torch only provides device memory and the stream).

    v = value_routed(x, Wr, br, Wv)            # (T, 1024) -> view (T, 8, 128)
    idx, w = route(x, Wr, br)
    v = value(x, idx, w, Wv)                    # routing given (compact cache)

Every function enqueues on torch's current CUDA stream (the host-buffer forms:
on `stream` if given) and returns without synchronising.  Device-side checks
are read with get_status().  A call given no `ws` uses the workspace this
module keeps for its device and stream, so calls on different streams may
overlap on the GPU.  Calls that share a `ws` must run on one stream.
"""
from __future__ import annotations

import ctypes
import functools
from typing import Optional

import torch

from . import _lib

_DT = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16, torch.float16: _lib.F16,
       torch.int32: _lib.I32, torch.int8: _lib.I8}
_PATH = {"auto": _lib.PATH_AUTO, "stream": _lib.PATH_STREAM, "tensor": _lib.PATH_TENSOR,
         "tensor_1cta": _lib.PATH_TENSOR_1CTA}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


try:
    _raw_stream = torch._C._cuda_getCurrentRawStream  # the current stream's handle, without a Stream object
except AttributeError:  # pragma: no cover - older torch
    _raw_stream = None


def _current_stream_handle() -> int:
    """The handle of the current stream of the current device."""
    if _raw_stream is not None:
        return int(_raw_stream(torch.cuda.current_device()))
    return int(torch.cuda.current_stream().cuda_stream)


def _stream(stream: Optional["torch.cuda.Stream"] = None):
    """The handle of `stream`, else of the current stream of the current device."""
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(_current_stream_handle())


def _need(t: torch.Tensor, name: str, dtypes=None, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _shape(t: torch.Tensor, name: str, want) -> None:
    """The library sees only pointers and the sizes passed with them, so a
    tensor of the wrong shape would be read or written out of bounds: refuse
    it here."""
    if t.shape != want:
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(want)}")


class Workspace:
    """A device workspace that grows on demand."""

    def __init__(self):
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != torch.device(device):
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


# The workspaces of calls made without `ws`: one per (device, stream).  A call
# leaves its routing, grouping and expert rows in its workspace until its last
# kernel has run, so calls that may overlap on the GPU -- calls on different
# streams -- must not share one.  Calls on one stream run in order and share
# that stream's workspace.
_WS = {}


def _devkey(device) -> torch.device:
    dev = torch.device(device)
    if dev.type == "cuda" and dev.index is None:
        dev = torch.device(dev.type, torch.cuda.current_device())
    return dev


def _workspace(nbytes: int, device, stream: Optional["torch.cuda.Stream"] = None) -> torch.Tensor:
    """The default workspace of `stream` (else of the current stream) on
    `device`, grown to at least `nbytes`.  It is allocated while that stream is
    current: torch's caching allocator then keeps the memory of a buffer that
    a later, larger call replaces from every other stream's allocations until
    this stream has passed its last use."""
    dev = _devkey(device)
    handle = int(stream.cuda_stream) if stream is not None else _current_stream_handle()
    key = (dev, handle)
    if key not in _WS:
        _WS[key] = Workspace()
    if stream is None:
        return _WS[key].get(nbytes, dev)
    with torch.cuda.stream(stream):
        return _WS[key].get(nbytes, dev)


def release_workspaces() -> None:
    """Drop the default workspaces (each stream that ran a call without `ws`
    keeps one, sized for its largest call, until this is called).  Safe with
    calls still in flight: torch's caching allocator reuses a freed buffer
    only for later work on the stream that used it."""
    _WS.clear()


@functools.lru_cache(maxsize=256)
def workspace_size(T: int, d: int, E: int, k: int, n: int) -> int:
    return int(_lib.load().mova_workspace_size(T, d, E, k, n))


@functools.lru_cache(maxsize=256)
def workspace_size_host(T: int, d: int, E: int, k: int, n: int) -> int:
    """Device workspace of the host-buffer value calls (value_routed_host, value_host)."""
    return int(_lib.load().mova_workspace_size_host(T, d, E, k, n))


@functools.lru_cache(maxsize=256)
def attend_workspace_size_host(L: int, d: int, E: int, k: int, n: int, H: int) -> int:
    """Device workspace of value_attend_host."""
    return int(_lib.load().mova_attend_workspace_size_host(L, d, E, k, n, H))


def auto_path(T: int, dtype: torch.dtype) -> str:
    code = _lib.load().mova_auto_path(T, _DT[dtype])
    return {v: k for k, v in _PATH.items()}[code]


def launch_count() -> int:
    """Kernel launches the library has enqueued in this process so far."""
    return int(_lib.load().mova_launch_count())


def _opts(path="auto", events=None, wv_stride=0, partitions=0, decode_launches=0, planes=None):
    """A mova_options value (kept alive by the caller for the call)."""
    ev = _events(events)
    o = _lib.Options(_PATH[path], ctypes.cast(ev, ctypes.c_void_p) if ev is not None else None,
                     int(wv_stride), int(partitions), int(decode_launches),
                     None if planes is None else ctypes.c_void_p(planes.data_ptr()))
    return o, ev


def router_planes(Wr: torch.Tensor) -> torch.Tensor:
    """The router weight split exactly into three bf16 planes (mova_router_planes),
    to hand to value_routed(planes=...) so that calls skip the split."""
    _need(Wr, "Wr", (torch.float32,), 2)
    E, d = Wr.shape
    lib = _lib.load()
    nbytes = int(lib.mova_router_planes_bytes(d))
    planes = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=Wr.device)
    _lib.check(lib.mova_router_planes(_ptr(Wr), E, d, _ptr(planes), _stream()), "mova_router_planes")
    return planes


def route(x: torch.Tensor, Wr: torch.Tensor, br: torch.Tensor, k: int = 4, scale: float = 2.5,
          partitions: int = 0):
    """(idx (T, k) int32, w (T, k) fp32).  partitions=2 sums the router's two
    halves of d separately in fp32 and then adds them (mova_options)."""
    _need(x, "x", (torch.float32, torch.bfloat16), 2)
    _need(Wr, "Wr", (torch.float32,), 2)
    _need(br, "br", (torch.float32,), 1)
    T, d = x.shape
    E = Wr.shape[0]
    _shape(Wr, "Wr", (E, d))
    _shape(br, "br", (E,))
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    lib = _lib.load()
    o, _ = _opts(partitions=partitions)
    _lib.check(lib.mova_route_opts(_ptr(x), _DT[x.dtype], _ptr(Wr), _ptr(br), T, d, E, k, float(scale),
                                   _ptr(idx), _ptr(w), ctypes.byref(o), _stream()), "mova_route")
    return idx, w


def permute(idx: torch.Tensor, E: int):
    """Stable grouping of the (token, slot) pairs by expert:
    dict(counts (E), offsets (E+1), perm (T*k), pos (T*k)), all int32."""
    _need(idx, "idx", (torch.int32,), 2)
    T, k = idx.shape
    dev = idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    nbytes = workspace_size(T, 64, E, k, 128)
    ws = _workspace(nbytes, dev)
    lib = _lib.load()
    _lib.check(lib.mova_permute(_ptr(idx), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm),
                                _ptr(pos), _ptr(ws), ws.numel(), _stream()), "mova_permute")
    return dict(counts=counts, offsets=offsets, perm=perm, pos=pos, ws=ws)


def _events(events):
    """Array of raw cudaEvent_t handles (or None) for the _ex entry points."""
    if events is None:
        return None
    assert len(events) == _lib.STAGE_EVENTS
    return (ctypes.c_void_p * _lib.STAGE_EVENTS)(*[ctypes.c_void_p(e.cuda_event) for e in events])


def _expert_view(Wv: torch.Tensor, rows: Optional[tuple]):
    """(E, n, stride in rows, base tensor) of the experts' rows a call reads:
    all of Wv, or rows = (row0, count) of every expert (head-parallel slice)."""
    E, n_total, _ = Wv.shape
    if rows is None:
        return E, n_total, 0, Wv
    row0, count = rows
    if not (0 <= row0 and count > 0 and row0 + count <= n_total):
        raise ValueError(f"rows {rows} outside the {n_total} rows of each expert")
    return E, count, n_total, Wv[:, row0:, :]


def head_slice(n_total: int, world: int, rank: int, head_dim: int = 128) -> tuple:
    """(row0, count) of the expert rows -- whole value heads -- that rank
    `rank` of `world` head-parallel ranks computes: the heads are dealt in
    contiguous blocks, the first n_heads % world ranks taking one extra."""
    if n_total % head_dim != 0:
        raise ValueError("n_total must be whole heads")
    heads = n_total // head_dim
    if not 0 <= rank < world or world > heads:
        raise ValueError(f"rank {rank} of {world} over {heads} heads")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    nh = base + (1 if rank < extra else 0)
    return h0 * head_dim, nh * head_dim


def value(x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, Wv: torch.Tensor,
          path: str = "auto", ws: Optional[torch.Tensor] = None,
          events=None, rows: Optional[tuple] = None) -> torch.Tensor:
    """Routing-given mixture: v (T, n) in x's dtype.  rows=(row0, count)
    computes only rows [row0, row0+count) of every expert (v is (T, count)),
    reading them in place from the full Wv."""
    _need(x, "x", (torch.float32, torch.bfloat16), 2)
    _need(idx, "idx", (torch.int32, torch.int8), 2)
    _need(w, "w", (torch.float32, torch.float16), 2)
    _need(Wv, "Wv", (x.dtype,), 3)
    T, d = x.shape
    E, n, stride, Wb = _expert_view(Wv, rows)
    k = idx.shape[1]
    _shape(idx, "idx", (T, k))
    _shape(w, "w", (T, k))
    _shape(Wv, "Wv", (E, Wv.shape[1], d))
    v = torch.empty((T, n), dtype=x.dtype, device=x.device)
    nbytes = workspace_size(T, d, E, k, n)
    if ws is None:
        ws = _workspace(nbytes, x.device)
    lib = _lib.load()
    o, _ev = _opts(path, events, stride)
    _lib.check(lib.mova_value_opts(_ptr(x), _DT[x.dtype], _ptr(idx), _DT[idx.dtype], _ptr(w),
                                   _DT[w.dtype], _ptr(Wb), _DT[Wv.dtype], T, d, E, k, n, _ptr(v),
                                   _ptr(ws), ws.numel(), ctypes.byref(o), _stream()),
               "mova_value")
    return v


def attend_workspace_size(L: int, d: int, E: int, k: int, n: int, H: int) -> int:
    return int(_lib.load().mova_attend_workspace_size(L, d, E, k, n, H))


def value_attend(x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, Wv: torch.Tensor,
                 probs: torch.Tensor, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One query token's attention output over L cached positions whose
    values are recomputed from the compact cache (x, idx, w) and never
    stored: o (H, 128) fp32 = sum_l probs[h, l] * V[l, h // G]."""
    _need(x, "x", (torch.bfloat16,), 2)
    _need(idx, "idx", (torch.int32, torch.int8), 2)
    _need(w, "w", (torch.float32, torch.float16), 2)
    _need(Wv, "Wv", (torch.bfloat16,), 3)
    _need(probs, "probs", (torch.float32,), 2)
    L, d = x.shape
    E, n = Wv.shape[0], Wv.shape[1]
    k = idx.shape[1]
    H = probs.shape[0]
    if probs.shape[1] != L:
        raise ValueError("probs: (H, L) for the L cached positions of x")
    _shape(idx, "idx", (L, k))
    _shape(w, "w", (L, k))
    _shape(Wv, "Wv", (E, n, d))
    o = torch.empty((H, 128), dtype=torch.float32, device=x.device)
    lib = _lib.load()
    nbytes = int(lib.mova_attend_workspace_size(L, d, E, k, n, H))
    if ws is None:
        ws = _workspace(nbytes, x.device)
    _lib.check(lib.mova_value_attend(_ptr(x), _ptr(idx), _DT[idx.dtype], _ptr(w), _DT[w.dtype], _ptr(Wv),
                                     L, d, E, k, n, _ptr(probs), H, _ptr(o), _ptr(ws), ws.numel(),
                                     _stream()), "mova_value_attend")
    return o


def value_routed(x: torch.Tensor, Wr: torch.Tensor, br: torch.Tensor, Wv: torch.Tensor,
                 k: int = 4, scale: float = 2.5, return_routing: bool = False,
                 path: str = "auto", ws: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, events=None, rows: Optional[tuple] = None,
                 partitions: int = 0, decode_launches: int = 0,
                 planes: Optional[torch.Tensor] = None):
    """Full value path: v (T, n) in x's dtype [, idx (T, k) int32, w (T, k) fp32].
    rows=(row0, count): only those rows of every expert (a head-parallel
    slice, v is (T, count)); partitions=2: the router's two-partition sum;
    decode_launches=1: decode batches as one persistent kernel (default two);
    planes: the router's bf16 planes from router_planes(Wr), made once."""
    _need(x, "x", (torch.float32, torch.bfloat16), 2)
    _need(Wr, "Wr", (torch.float32,), 2)
    _need(br, "br", (torch.float32,), 1)
    _need(Wv, "Wv", (x.dtype,), 3)
    T, d = x.shape
    E, n, stride, Wb = _expert_view(Wv, rows)
    _shape(Wr, "Wr", (E, d))
    _shape(br, "br", (E,))
    _shape(Wv, "Wv", (E, Wv.shape[1], d))
    dev = x.device
    if out is not None:
        _need(out, "out", (x.dtype,), 2)
        _shape(out, "out", (T, n))
    v = out if out is not None else torch.empty((T, n), dtype=x.dtype, device=dev)
    idx = w = None
    if return_routing:
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
    nbytes = workspace_size(T, d, E, k, n)
    if ws is None:
        ws = _workspace(nbytes, dev)
    lib = _lib.load()
    if planes is not None:
        _need(planes, "planes", (torch.bfloat16,), 1)
        if planes.numel() * 2 < int(lib.mova_router_planes_bytes(d)):
            raise ValueError("planes: too small for this d; make them with router_planes(Wr)")
    o, _ev = _opts(path, events, stride, partitions, decode_launches, planes)
    _lib.check(lib.mova_value_routed_opts(_ptr(x), _DT[x.dtype], _ptr(Wr), _ptr(br), _ptr(Wb),
                                          _DT[Wv.dtype], T, d, E, k, n, float(scale), _ptr(v),
                                          _ptr(idx), _ptr(w), _ptr(ws), ws.numel(), ctypes.byref(o),
                                          _stream()), "mova_value_routed")
    if return_routing:
        return v, idx, w
    return v


def _need_host(t: torch.Tensor, name: str, dtypes=None, ndim=None):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor; pinned memory makes the copy asynchronous")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _host_out(out, shape, dtype, name="out"):
    if out is None:
        return torch.empty(shape, dtype=dtype, pin_memory=True)
    _need_host(out, name, (dtype,), len(shape))
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(out.shape)}, expected {tuple(shape)}")
    return out


def value_routed_host(x: torch.Tensor, Wr: torch.Tensor, br: torch.Tensor, Wv: torch.Tensor,
                      k: int = 4, scale: float = 2.5, out: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None, stream=None, return_routing: bool = False):
    """value_routed for a batch in host memory (mova_value_routed_host): x is a
    CPU tensor (pinned for an asynchronous copy), the weights are on the
    device, and v (and the routing) come back in host tensors, valid once the
    stream has passed the call."""
    _need_host(x, "x", (torch.float32, torch.bfloat16), 2)
    _need(Wr, "Wr", (torch.float32,), 2)
    _need(br, "br", (torch.float32,), 1)
    _need(Wv, "Wv", (x.dtype,), 3)
    T, d = x.shape
    E, n = Wv.shape[0], Wv.shape[1]
    _shape(Wr, "Wr", (E, d))
    _shape(br, "br", (E,))
    _shape(Wv, "Wv", (E, n, d))
    v = _host_out(out, (T, n), x.dtype)
    idx = w = None
    if return_routing:
        idx = torch.empty((T, k), dtype=torch.int32, pin_memory=True)
        w = torch.empty((T, k), dtype=torch.float32, pin_memory=True)
    if ws is None:
        ws = _workspace(workspace_size_host(T, d, E, k, n), Wv.device, stream)
    _lib.check(_lib.load().mova_value_routed_host(
        _ptr(x), _DT[x.dtype], _ptr(Wr), _ptr(br), _ptr(Wv), _DT[Wv.dtype], T, d, E, k, n, float(scale),
        _ptr(v), _ptr(idx), _ptr(w), _ptr(ws), ws.numel(), _stream(stream)), "mova_value_routed_host")
    return (v, idx, w) if return_routing else v


def value_host(x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, Wv: torch.Tensor,
               out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """value for a batch and stored routing in host memory (mova_value_host);
    v comes back in a host tensor, valid once the stream has passed the call."""
    _need_host(x, "x", (torch.float32, torch.bfloat16), 2)
    _need_host(idx, "idx", (torch.int32, torch.int8), 2)
    _need_host(w, "w", (torch.float32, torch.float16), 2)
    _need(Wv, "Wv", (x.dtype,), 3)
    T, d = x.shape
    E, n = Wv.shape[0], Wv.shape[1]
    k = idx.shape[1]
    _shape(idx, "idx", (T, k))
    _shape(w, "w", (T, k))
    _shape(Wv, "Wv", (E, n, d))
    v = _host_out(out, (T, n), x.dtype)
    if ws is None:
        ws = _workspace(workspace_size_host(T, d, E, k, n), Wv.device, stream)
    _lib.check(_lib.load().mova_value_host(
        _ptr(x), _DT[x.dtype], _ptr(idx), _DT[idx.dtype], _ptr(w), _DT[w.dtype], _ptr(Wv), _DT[Wv.dtype],
        T, d, E, k, n, _ptr(v), _ptr(ws), ws.numel(), _stream(stream)), "mova_value_host")
    return v


def value_attend_host(x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor, Wv: torch.Tensor,
                      probs: torch.Tensor, out: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """value_attend for a compact cache and probabilities in host memory
    (mova_value_attend_host); o (H, 128) fp32 comes back in a host tensor,
    valid once the stream has passed the call."""
    _need_host(x, "x", (torch.bfloat16,), 2)
    _need_host(idx, "idx", (torch.int32, torch.int8), 2)
    _need_host(w, "w", (torch.float32, torch.float16), 2)
    _need_host(probs, "probs", (torch.float32,), 2)
    _need(Wv, "Wv", (torch.bfloat16,), 3)
    L, d = x.shape
    E, n = Wv.shape[0], Wv.shape[1]
    k = idx.shape[1]
    H = probs.shape[0]
    if probs.shape[1] != L:
        raise ValueError("probs: (H, L) for the L cached positions of x")
    _shape(idx, "idx", (L, k))
    _shape(w, "w", (L, k))
    _shape(Wv, "Wv", (E, n, d))
    o = _host_out(out, (H, 128), torch.float32)
    if ws is None:
        ws = _workspace(attend_workspace_size_host(L, d, E, k, n, H), Wv.device, stream)
    _lib.check(_lib.load().mova_value_attend_host(
        _ptr(x), _ptr(idx), _DT[idx.dtype], _ptr(w), _DT[w.dtype], _ptr(Wv), L, d, E, k, n, _ptr(probs), H,
        _ptr(o), _ptr(ws), ws.numel(), _stream(stream)), "mova_value_attend_host")
    return o


def workspace_parts(T: int, d: int, E: int, k: int, n: int) -> dict:
    """Byte offsets of the routing and grouping a value call leaves in its
    workspace: dict(idx, w, counts, offsets, perm, pos) -> offset."""
    offs = (ctypes.c_size_t * len(_lib.WS_PARTS))()
    _lib.check(_lib.load().mova_workspace_parts(T, d, E, k, n, offs), "mova_workspace_parts")
    return dict(zip(_lib.WS_PARTS, (int(o) for o in offs)))


def grouping(ws: torch.Tensor, T: int, d: int, E: int, k: int, n: int) -> dict:
    """The grouping by expert (counts, offsets, perm, pos; int32 copies) that
    the last value call with these sizes ran on, read from its workspace
    (call after the stream has passed that call)."""
    offs = workspace_parts(T, d, E, k, n)
    size = {"counts": E, "offsets": E + 1, "perm": T * k, "pos": T * k}
    out = {}
    for name, count in size.items():
        o = offs[name]
        out[name] = ws[o:o + 4 * count].view(torch.int32).clone()
    return out


def arm_stream_stall(stall_stage: int, limit_cycles: int) -> None:
    """Test hook: the next weight-streaming launch stops issuing weight copies
    in its first CTA at `stall_stage` and gives up waiting after
    `limit_cycles`, reporting MOVA_ERR_TIMEOUT (mova_selftest_arm_stream_stall)."""
    _lib.check(_lib.load().mova_selftest_arm_stream_stall(int(stall_stage), int(limit_cycles)),
               "mova_selftest_arm_stream_stall")


def get_status(ws: Optional[torch.Tensor] = None, device=None, stream=None):
    """(status name, detail) of the last value call on this workspace; without
    `ws`, on the default workspace of `stream` (else of the current stream),
    i.e. of the last call made there without `ws`.  Waits for that stream."""
    if ws is None:
        dev = _devkey(device if device is not None else "cuda")
        handle = int(stream.cuda_stream) if stream is not None else _current_stream_handle()
        entry = _WS.get((dev, handle))
        if entry is None or entry.buf is None:
            raise ValueError(f"no call on {dev} has used the default workspace of this stream")
        ws = entry.buf
    detail = ctypes.c_int32(0)
    code = _lib.load().mova_get_status(_ptr(ws), ctypes.byref(detail), _stream(stream))
    return _lib.STATUS_NAMES.get(code, str(code)), int(detail.value)
