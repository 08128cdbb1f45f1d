"""The C-ABI library: it builds, loads without a GPU, exports every entry point
include/mova.h declares, and rejects bad arguments on the host (no compute
call is made here)."""
import ctypes
import os
import re

import pytest

from mixture_value_routing_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mova.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mova_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ["mova_route", "mova_value", "mova_value_routed", "mova_permute",
                 "mova_workspace_size", "mova_get_status", "mova_status_str"]:
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(_lib.SIGNATURES)


def test_status_strings(lib):
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.mova_status_str(code).decode() == name
    assert lib.mova_status_str(99).decode() == "MOVA_ERR_UNKNOWN"


def test_workspace_size(lib):
    assert lib.mova_workspace_size(0, 2560, 64, 4, 1024) == 0
    a = lib.mova_workspace_size(8, 2560, 64, 4, 1024)
    b = lib.mova_workspace_size(4096, 2560, 64, 4, 1024)
    assert a > 0 and b > a and b % 256 == 0
    # P rows dominate: T*k*n fp32
    assert b >= 4096 * 4 * 1024 * 4
    # unsupported or invalid sizes give 0
    assert lib.mova_workspace_size(8, 2560, 65, 4, 1024) == 0
    assert lib.mova_workspace_size(8, 2561, 64, 4, 1024) == 0
    assert lib.mova_workspace_size(8, 2560, 64, 9, 1024) == 0
    assert lib.mova_workspace_size(8, 2560, 64, 4, 1000) == 0
    assert lib.mova_workspace_size(-1, 2560, 64, 4, 1024) == 0
    assert lib.mova_workspace_size(8, 2560, 4, 5, 1024) == 0
    assert lib.mova_workspace_size(40000, 2560, 64, 4, 1024) == 0  # above the pair limit


def test_host_side_validation(lib):
    """Errors found on the host return before anything touches a GPU."""
    fake = ctypes.c_void_p(4096)  # never dereferenced: every call below fails validation first
    st = lib.mova_route(None, _lib.BF16, None, None, 0, 2560, 64, 4, 2.5, None, None, None)
    assert st == _lib.OK  # T == 0 is a no-op
    st = lib.mova_route(None, _lib.BF16, None, None, 8, 2560, 64, 4, 2.5, None, None, None)
    assert st == _lib.ERR_INVALID_ARG
    st = lib.mova_route(fake, _lib.F16, fake, fake, 8, 2560, 64, 4, 2.5, fake, fake, None)
    assert st == _lib.ERR_UNSUPPORTED
    st = lib.mova_route(fake, _lib.BF16, fake, fake, 8, 2560, 64, 65, 2.5, fake, fake, None)
    assert st == _lib.ERR_INVALID_ARG
    # misaligned x
    st = lib.mova_route(ctypes.c_void_p(4098), _lib.BF16, fake, fake, 8, 2560, 64, 4, 2.5, fake,
                        fake, None)
    assert st == _lib.ERR_INVALID_ARG
    # value: wv dtype must equal x dtype; workspace too small
    st = lib.mova_value_routed(fake, _lib.BF16, fake, fake, fake, _lib.F32, 8, 2560, 64, 4, 1024,
                               2.5, fake, None, None, fake, 1 << 30, None)
    assert st == _lib.ERR_UNSUPPORTED
    st = lib.mova_value_routed(fake, _lib.BF16, fake, fake, fake, _lib.BF16, 8, 2560, 64, 4, 1024,
                               2.5, fake, None, None, fake, 16, None)
    assert st == _lib.ERR_INVALID_ARG
    st = lib.mova_value(fake, _lib.BF16, fake, _lib.F32, fake, _lib.F16, fake, _lib.BF16, 8, 2560,
                        64, 4, 1024, fake, fake, 1 << 30, None)
    assert st == _lib.ERR_UNSUPPORTED  # idx must be int32 or int8
    st = lib.mova_value_ex(fake, _lib.BF16, fake, _lib.I8, fake, _lib.F16, fake, _lib.BF16, 8, 2560,
                           64, 4, 1024, fake, fake, 1 << 30, 7, None, None)
    assert st == _lib.ERR_INVALID_ARG  # unknown path
    st = lib.mova_permute(None, 0, 64, 4, None, None, None, None, None, 0, None)
    assert st == _lib.OK
    st = lib.mova_get_status(None, None, None)
    assert st == _lib.ERR_INVALID_ARG


def test_launch_counter_ignores_rejected_calls(lib):
    # A call rejected on the host enqueues nothing, so the counter is unchanged.
    before = lib.mova_launch_count()
    st = lib.mova_value_routed(None, _lib.BF16, None, None, None, _lib.BF16, 8, 2560, 64, 4, 1024,
                               ctypes.c_float(2.5), None, None, None, None, 0, None)
    assert st == _lib.ERR_INVALID_ARG
    assert lib.mova_launch_count() == before


def test_noalloc_scratch_admits_the_documented_batch(lib):
    # include/mova.h: the built-in 2 MiB workspace admits T <= 30 at the
    # decode dimensions (d = 2560, E = 64, k = 4, n = 1024).
    scratch = 2 << 20
    assert lib.mova_workspace_size(30, 2560, 64, 4, 1024) <= scratch
    assert lib.mova_workspace_size(31, 2560, 64, 4, 1024) > scratch


def test_noalloc_validates_like_the_regular_entry_point(lib):
    """The no-allocation entry point checks its arguments exactly as
    mova_value_routed does; T == 0 is a no-op only for valid sizes."""
    for args in ((0, 2560, 64, 4, 1024), (0, -1, 64, 4, 1024), (0, 2560, 65, 4, 1024),
                 (8, 2561, 64, 4, 1024), (8, 2560, 64, 9, 1024)):
        want = lib.mova_value_routed(None, _lib.BF16, None, None, None, _lib.BF16, *args,
                                     ctypes.c_float(2.5), None, None, None, None, 0, None)
        got = lib.mova_value_routed_noalloc(None, _lib.BF16, None, None, None, _lib.BF16, *args,
                                            ctypes.c_float(2.5), None, None)
        assert got == want, (args, got, want)


def test_workspace_parts(lib):
    """The routing and grouping parts of the workspace lie inside it, in
    order, 256-byte aligned and large enough for their arrays."""
    T, d, E, k, n = 4096, 2560, 64, 4, 1024
    offs = (ctypes.c_size_t * len(_lib.WS_PARTS))()
    assert lib.mova_workspace_parts(T, d, E, k, n, offs) == _lib.OK
    o = dict(zip(_lib.WS_PARTS, offs))
    size = dict(idx=T * k * 4, w=T * k * 4, counts=E * 4, offsets=(E + 1) * 4, perm=T * k * 4,
                pos=T * k * 4)
    total = lib.mova_workspace_size(T, d, E, k, n)
    names = list(_lib.WS_PARTS)
    for a, b in zip(names, names[1:]):
        assert o[a] % 256 == 0 and o[a] + size[a] <= o[b]
    assert o["pos"] + size["pos"] <= total
    assert lib.mova_workspace_parts(0, d, E, k, n, offs) == _lib.ERR_INVALID_ARG
    assert lib.mova_workspace_parts(T, d, 65, k, n, offs) == _lib.ERR_UNSUPPORTED
    assert lib.mova_workspace_parts(T, d, E, k, n, None) == _lib.ERR_INVALID_ARG


def test_stream_stall_arming_is_validated(lib):
    assert lib.mova_selftest_arm_stream_stall(-1, 1000) == _lib.ERR_INVALID_ARG
    assert lib.mova_selftest_arm_stream_stall(-3, 1000) == _lib.ERR_INVALID_ARG
    assert lib.mova_selftest_arm_stream_stall(2, 0) == _lib.ERR_INVALID_ARG
    assert lib.mova_selftest_arm_stream_stall(2, 1 << 40) == _lib.ERR_INVALID_ARG


def test_attend_host_side_validation(lib):
    """mova_value_attend: head counts and sizes checked on the host."""
    fake = ctypes.c_void_p(4096)
    I32, F16 = _lib.I32, _lib.F16
    args = lambda H, o: (fake, fake, I32, fake, F16, fake, 64, 2560, 64, 4, 1024, fake, H, o, fake, 1 << 30, None)
    assert lib.mova_value_attend(*args(0, fake)) == _lib.ERR_INVALID_ARG     # no heads
    assert lib.mova_value_attend(*args(12, fake)) == _lib.ERR_UNSUPPORTED    # not a multiple of 8 KV heads
    assert lib.mova_value_attend(*args(48, fake)) == _lib.ERR_UNSUPPORTED    # 6 query heads per KV head
    assert lib.mova_value_attend(*args(32, None)) == _lib.ERR_INVALID_ARG    # no output
    assert lib.mova_attend_workspace_size(64, 2560, 64, 4, 1024, 32) > lib.mova_workspace_size(64, 2560, 64, 4, 1024)
    assert lib.mova_attend_workspace_size(64, 2560, 64, 4, 1024, 40) == 0
    assert lib.mova_attend_workspace_size(0, 2560, 64, 4, 1024, 32) == 0


def test_host_buffer_forms_validation(lib):
    """The host-buffer value calls check their arguments and workspace on the
    host before enqueueing any copy; their workspace is the device call's plus
    aligned staging for the batch and the result."""
    fake = ctypes.c_void_p(4096)
    BF16, F32, I8, F16 = _lib.BF16, _lib.F32, _lib.I8, _lib.F16
    T, d, E, k, n = 8, 2560, 64, 4, 1024
    base = lib.mova_workspace_size(T, d, E, k, n)
    host = lib.mova_workspace_size_host(T, d, E, k, n)
    staging = 2560 * 8 * 4 + 1024 * 8 * 4 + 2 * 256  # x and v at 4 B an element, idx and w rounded up
    assert host == ((base + 255) & ~255) + staging
    assert lib.mova_workspace_size_host(0, d, E, k, n) == 0
    assert lib.mova_workspace_size_host(T, d + 1, E, k, n) == 0
    routed = lambda x_dt, wv_dt, T_, ws_bytes, v: lib.mova_value_routed_host(
        fake, x_dt, fake, fake, fake, wv_dt, T_, d, E, k, n, 2.5, v, None, None, fake, ws_bytes, None)
    assert routed(BF16, BF16, 0, 0, None) == _lib.OK                       # T == 0: nothing to do
    assert routed(BF16, F32, T, host, fake) == _lib.ERR_UNSUPPORTED         # Wv dtype must equal x's
    assert routed(BF16, BF16, T, host, None) == _lib.ERR_INVALID_ARG        # no output buffer
    assert routed(BF16, BF16, T, base, fake) == _lib.ERR_INVALID_ARG        # room for the call, not the staging
    # rows wider than the streaming kernel holds (d = 4672 at T = 8): refused before any copy is enqueued
    wide = lib.mova_workspace_size_host(T, 4672, E, k, n)
    assert lib.mova_value_routed_host(fake, BF16, fake, fake, fake, BF16, T, 4672, E, k, n, 2.5, fake, None, None,
                                      fake, wide, None) == _lib.ERR_UNSUPPORTED
    assert lib.mova_value_host(fake, BF16, fake, F32, fake, F16, fake, BF16, T, d, E, k, n, fake, fake,
                               host, None) == _lib.ERR_UNSUPPORTED        # idx must be int32 or int8
    assert lib.mova_value_host(fake, BF16, fake, I8, fake, F16, fake, BF16, T, d, E, k, n, fake, fake,
                               host - 256, None) == _lib.ERR_INVALID_ARG  # workspace too small
    assert lib.mova_value_host(fake, BF16, fake, I8, fake, F16, ctypes.c_void_p(4100), BF16, T, d, E, k, n,
                               fake, fake, host, None) == _lib.ERR_INVALID_ARG  # misaligned Wv
    # attend: staging for o even at L == 0 (zeros are written through it)
    assert lib.mova_attend_workspace_size_host(0, d, E, k, n, 32) == 32 * 128 * 4
    assert lib.mova_attend_workspace_size_host(64, d, E, k, n, 40) == 0
    assert lib.mova_attend_workspace_size_host(64, d, E, k, n, 32) > lib.mova_attend_workspace_size(64, d, E, k, n, 32)
    attend = lambda H, o, ws_bytes: lib.mova_value_attend_host(fake, fake, I8, fake, F16, fake, 64, d, E, k, n,
                                                               fake, H, o, fake, ws_bytes, None)
    assert attend(0, fake, 1 << 30) == _lib.ERR_INVALID_ARG
    assert attend(12, fake, 1 << 30) == _lib.ERR_UNSUPPORTED
    assert attend(32, None, 1 << 30) == _lib.ERR_INVALID_ARG
    assert attend(32, fake, 4096) == _lib.ERR_INVALID_ARG


def _c_type_to_ctypes(decl: str):
    """The ctypes type that marshals a C parameter or return type of the header."""
    t = " ".join(decl.replace("const", " ").split())
    if "*" in t:
        return ctypes.c_char_p if t.startswith("char") else ctypes.c_void_p
    base = re.sub(r"\s*\b[A-Za-z_]\w*$", "", t) if len(t.split()) > 1 else t
    return {"size_t": ctypes.c_size_t, "long long": ctypes.c_longlong,
            "unsigned long long": ctypes.c_ulonglong, "float": ctypes.c_float, "int": ctypes.c_int,
            "int32_t": ctypes.c_int32, "mova_dtype": ctypes.c_int, "mova_path": ctypes.c_int,
            "mova_status": ctypes.c_int}[base]


def _prototypes():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = {}
    for m in re.finditer(r"([A-Za-z_][\w \t\*]*?)\s*\b(mova_[a-z_]+)\s*\(([^()]*)\)\s*;", src):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        ret = ret.split("\n")[-1].strip()
        args = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        out[name] = (_c_type_to_ctypes(ret + " r"), [_c_type_to_ctypes(a) for a in args])
    return out


def test_binding_signatures_match_the_header():
    """Every ctypes prototype of the binding has the header's return type and
    parameter types, one for one: a dropped, swapped or mistyped argument
    would otherwise reach the library as garbage without any error."""
    protos = _prototypes()
    assert set(protos) == set(_lib.SIGNATURES)
    for name, (ret, args) in protos.items():
        b_ret, b_args = _lib.SIGNATURES[name]
        assert b_ret == ret, (name, "return", b_ret, ret)
        assert len(b_args) == len(args), (name, len(b_args), len(args))
        for i, (b, h) in enumerate(zip(b_args, args)):
            assert b == h or (ctypes.sizeof(b) == ctypes.sizeof(h) and b not in (ctypes.c_float,)
                              and h not in (ctypes.c_float,) and (b is ctypes.c_void_p) == (h is ctypes.c_void_p)), \
                (name, i, b, h)


def test_options_struct_matches_the_header():
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct mova_options \{(.*?)\} mova_options;", src, re.S).group(1)
    fields = [f.strip() for f in body.split(";") if f.strip()]
    names = [re.search(r"(\w+)$", f).group(1) for f in fields]
    assert names == [n for n, _ in _lib.Options._fields_]
    for f, (_, ct) in zip(fields, _lib.Options._fields_):
        assert ctypes.sizeof(ct) == ctypes.sizeof(_c_type_to_ctypes(f)), f


def test_header_is_plain_c_and_links(lib, tmp_path):
    """The header compiles as C11 with warnings as errors, and a C program
    linked against libmova.so makes host-only calls: the library is usable
    without Python or C++."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    prog = tmp_path / "abi.c"
    prog.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "mova.h"
int main(void) {
  if (strcmp(mova_status_str(MOVA_ERR_TIMEOUT), "MOVA_ERR_TIMEOUT") != 0) return 1;
  if (mova_workspace_size(8, 2560, 64, 4, 1024) == 0) return 2;
  if (mova_workspace_size(8, 2560, 65, 4, 1024) != 0) return 3;      /* E > 64 unsupported */
  if (mova_auto_path(4096, MOVA_BF16) != MOVA_PATH_TENSOR) return 4;
  if (mova_value_routed(NULL, MOVA_BF16, NULL, NULL, NULL, MOVA_BF16, 8, 2560, 64, 4, 1024, 2.5f,
                        NULL, NULL, NULL, NULL, 0, NULL) != MOVA_ERR_INVALID_ARG) return 5;
  mova_options o;
  memset(&o, 0, sizeof o);
  o.router_partitions = 3;                                          /* unsupported */
  if (mova_route_opts(NULL, MOVA_BF16, NULL, NULL, 8, 2560, 64, 4, 2.5f, NULL, NULL, &o, NULL)
      != MOVA_ERR_UNSUPPORTED) return 6;
  puts("ok");
  return 0;
}
''')
    exe = tmp_path / "abi"
    libdir = os.path.dirname(_lib.LIB_PATH)
    r = subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(prog), "-o", str(exe), "-L", libdir, "-lmova", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
