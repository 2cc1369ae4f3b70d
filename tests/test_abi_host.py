"""Host-side checks of libssd.so: it loads, exports what include/ssd.h declares,
and rejects bad arguments before touching the GPU.

No test here launches anything: every ssd_fwd call below fails argument
validation, which runs on the host before the first CUDA call.
"""
import ctypes
import os
import re

import pytest

from structured_state_space_ssd_b200 import ssd
from structured_state_space_ssd_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return ssd.load()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SSD_API\s+[\w\s\*]*?\b(ssd_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(ssd.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.lib_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(ssd_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)
    # nothing but the declared API leaks out
    assert exported == set(_declared())


def test_version_and_status_strings(lib):
    assert lib.ssd_version() >= 100
    for code in range(5):
        assert ssd.status_string(code)
    assert ssd.status_string(99) == "unknown status"


def test_workspace_bytes(lib):
    f = lib.ssd_fwd_workspace_bytes
    w = f(4, 2048, 80, 64, 1, 128, 256, 1)      # fused tensor-core path: flags + the state rings
    assert w % 256 == 0
    nc = 8
    tile = 128 * 64 * 2                # a bf16 state tile (N = 128 rows of 64)
    ring = 4 * 80 * (64 * 128 * 4 + 3 * tile)   # per (batch, head): one fp32 state, three bf16 tiles
    assert ring <= w < ring + (1 << 16)
    w256 = f(8, 4096, 32, 64, 1, 256, 256, 1)   # N = 256: two halves, each with its own flags and rings
    ring256 = 2 * 8 * 32 * (64 * 128 * 4 + 3 * tile)
    assert ring256 <= w256 < ring256 + (1 << 17)
    wlong = f(1, 131072, 48, 64, 8, 128, 256, 1)   # look-back over 4 chunks: 8 slots of S~ and L
    ringlong = 48 * 8 * 2 * 64 * 128 * 4
    assert ringlong <= wlong < ringlong + (1 << 17)
    assert f(8, 4096, 32, 64, 1, 64, 256, 1) < (8 * 32 * (64 * 64 * 4 + 3 * 64 * 64 * 2)) + (1 << 16)  # 64-row tiles
    # the shapes the allocation-free entry point serves fit its 32 MiB scratch
    assert w <= (32 << 20) and wlong <= (32 << 20)
    w32p = f(8, 4096, 32, 32, 1, 128, 256, 1)   # P = 32 is padded: the ring still holds 64 rows
    assert w32p == f(8, 4096, 32, 64, 1, 128, 256, 1)
    assert f(8, 4096, 32, 128, 1, 256, 256, 1) == 2 * w256   # four launches of 64 x 128 states
    w32 = f(4, 2048, 80, 64, 1, 128, 256, 0)    # CUDA-core path: every chunk state
    assert w32 >= 4 * nc * 80 * 64 * 128 * 4 + 4 * 80 * nc * 256 * 4
    assert f(0, 2048, 80, 64, 1, 128, 256, 1) == 0      # batch < 1
    assert f(4, 2048, 80, 64, 3, 128, 256, 1) == 0      # H % G != 0
    assert f(4, 2048, 80, 64, 1, 128, 256, 7) == 0      # bad dtype
    assert f(4, 2048, 80, 256, 1, 128, 256, 1) == 0     # P above the limit
    assert f(1, 0, 2, 16, 1, 16, 64, 0) > 0             # empty sequence is valid


def test_launch_count(lib):
    assert lib.ssd_fwd_launch_count(4, 2048, 80, 64, 1, 128, 256, 1) == 1    # one fused launch
    assert lib.ssd_fwd_launch_count(8, 4096, 32, 64, 1, 256, 256, 1) == 2    # N = 256: two state halves
    assert lib.ssd_fwd_stage_name(8, 4096, 32, 64, 1, 256, 256, 1, 1) == b"ssd_fused_n128_255"
    assert lib.ssd_fwd_launch_count(2, 4096, 32, 128, 1, 128, 256, 1) == 2   # P = 128: two column halves
    assert lib.ssd_fwd_stage_name(2, 4096, 32, 128, 1, 128, 256, 1, 1) == b"ssd_fused_p64_127"
    assert lib.ssd_fwd_launch_count(2, 4096, 32, 128, 1, 256, 256, 1) == 4   # both splits
    assert lib.ssd_fwd_stage_name(2, 4096, 32, 128, 1, 256, 256, 1, 2) == b"ssd_fused_p0_63_n128_255"
    assert lib.ssd_fwd_launch_count(2, 4096, 32, 32, 1, 128, 256, 1) == 1    # P = 32: padded, one launch
    assert lib.ssd_fwd_launch_count(2, 4096, 32, 36, 1, 128, 256, 1) == 4    # P % 8 != 0: CUDA-core stages
    assert lib.ssd_fwd_launch_count(1, 0, 2, 16, 1, 16, 64, 0) == 0
    assert lib.ssd_fwd_launch_count(1, 10, 3, 16, 2, 16, 64, 0) == 0


def _call(lib, **over):
    """ssd_fwd with fake (never dereferenced) pointers; only validation runs."""
    args = dict(x=0x10000, dt=0x20000, A=0x30000, B=0x40000, C=0x50000, D=0x60000, Q=64, init=None,
                y=0x70000, fin=None, batch=1, T=256, H=2, P=16, G=1, N=16, dtype=0, ws=0x80000, wsb=0,
                stream=None)
    args.update(over)
    v = lambda a: None if a is None else ctypes.c_void_p(a)  # noqa: E731
    return lib.ssd_fwd(v(args["x"]), v(args["dt"]), v(args["A"]), v(args["B"]), v(args["C"]), v(args["D"]),
                       args["Q"], v(args["init"]), v(args["y"]), v(args["fin"]), args["batch"], args["T"],
                       args["H"], args["P"], args["G"], args["N"], args["dtype"], v(args["ws"]),
                       ctypes.c_size_t(args["wsb"]), v(args["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(x=None), 1), (dict(dt=None), 1), (dict(A=None), 1), (dict(B=None), 1), (dict(C=None), 1),
    (dict(D=None), 1), (dict(y=None), 1), (dict(ws=None), 1),
    (dict(batch=0), 1), (dict(T=-1), 1), (dict(H=0), 1), (dict(P=0), 1), (dict(N=0), 1), (dict(Q=0), 1),
    (dict(G=0), 1), (dict(H=3, G=2), 1), (dict(dtype=5), 1),
    (dict(P=129), 2), (dict(N=257), 2), (dict(Q=257), 2),
    (dict(x=0x10002), 1),                 # fp32 tensor not 4-byte aligned
    (dict(ws=0x80010), 1),                # workspace not 256-byte aligned
    (dict(wsb=16), 1),                    # workspace too small
    (dict(y=0x10000, wsb=1 << 30), 1),    # y aliases x
])
def test_invalid_arguments_are_rejected_on_the_host(lib, over, code):
    assert _call(lib, **over) == code


def _step(lib, **over):
    """ssd_step with fake (never dereferenced) pointers; only validation runs."""
    args = dict(state=0x100000, x=0x10000, dt=0x20000, A=0x30000, B=0x40000, C=0x50000, D=0x60000, y=0x70000,
                batch=1, H=2, P=16, G=1, N=16, dtype=0, stream=None)
    args.update(over)
    v = lambda a: None if a is None else ctypes.c_void_p(a)  # noqa: E731
    return lib.ssd_step(v(args["state"]), v(args["x"]), v(args["dt"]), v(args["A"]), v(args["B"]), v(args["C"]),
                        v(args["D"]), v(args["y"]), args["batch"], args["H"], args["P"], args["G"], args["N"],
                        args["dtype"], v(args["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(state=None), 1), (dict(x=None), 1), (dict(dt=None), 1), (dict(A=None), 1), (dict(B=None), 1),
    (dict(C=None), 1), (dict(D=None), 1), (dict(y=None), 1),
    (dict(batch=0), 1), (dict(H=0), 1), (dict(P=0), 1), (dict(N=0), 1), (dict(G=0), 1), (dict(H=3, G=2), 1),
    (dict(dtype=4), 1), (dict(N=1025), 2),
    (dict(x=0x10002), 1),                 # fp32 tensor not 4-byte aligned
    (dict(y=0x100000 + 64), 1),           # y inside the state
    (dict(y=0x10000), 1),                 # y aliases x
])
def test_step_rejects_invalid_arguments_on_the_host(lib, over, code):
    assert _step(lib, **over) == code


def _gn(lib, **over):
    """ssd_gate_norm with fake (never dereferenced) pointers; only validation runs."""
    args = dict(y=0x100000, z=0x200000, w=None, b=None, out=0x300000, rows=4, ch=64, ng=4, eps=1e-5, dtype=1,
                stream=None)
    args.update(over)
    v = lambda a: None if a is None else ctypes.c_void_p(a)  # noqa: E731
    return lib.ssd_gate_norm(v(args["y"]), v(args["z"]), v(args["w"]), v(args["b"]), v(args["out"]), args["rows"],
                             args["ch"], args["ng"], ctypes.c_float(args["eps"]), args["dtype"], v(args["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(y=None), 1), (dict(z=None), 1), (dict(out=None), 1), (dict(rows=-1), 1), (dict(ch=0), 1),
    (dict(ng=0), 1), (dict(ng=5), 1), (dict(eps=-1.0), 1), (dict(dtype=3), 1),
    (dict(ch=8192, ng=1), 2),             # a group larger than the kernel holds
    (dict(y=0x100001), 1),                # bf16 tensor not 2-byte aligned
    (dict(out=0x200000), 1),              # out aliases z
    (dict(out=0x100000 + 64), 1),         # out partly overlaps y
    (dict(rows=0), 0),                    # nothing to do
])
def test_gate_norm_rejects_invalid_arguments_on_the_host(lib, over, code):
    assert _gn(lib, **over) == code


@pytest.mark.parametrize("call,code", [
    (lambda L, v: L.ssd_split_logdecay(None, v(1), v(2), v(3), 1, 8, 2, None), 1),
    (lambda L, v: L.ssd_split_logdecay(v(4), v(8), v(12), v(16), 1, 0, 2, None), 1),          # T < 1
    (lambda L, v: L.ssd_split_combine(v(4), v(8), None, 2, 2, v(12), None, 1, 2, 4, 4, None), 1),  # k >= K
    (lambda L, v: L.ssd_split_combine(v(4), v(8), None, -1, 2, v(12), None, 1, 2, 4, 4, None), 1),
    (lambda L, v: L.ssd_split_correct(v(4), v(8), v(12), v(16), 1, 8, 3, 4, 2, 4, 0, None), 1),  # H % G
    (lambda L, v: L.ssd_split_correct(v(4), v(8), v(12), v(16), 1, 8, 2, 4, 1, 512, 0, None), 2),  # N > 256
    (lambda L, v: L.ssd_split_correct(v(4), v(8), v(12), v(16), 1, 0, 2, 4, 1, 4, 0, None), 0),  # nothing to do
])
def test_split_entry_points_validate_on_the_host(lib, call, code):
    v = lambda a: ctypes.c_void_p(0x100000 * a)  # noqa: E731  (never dereferenced)
    assert call(lib, v) == code


def test_bwd_workspace_bytes(lib):
    f = lib.ssd_bwd_workspace_bytes
    w = f(4, 2048, 80, 64, 1, 128, 256, 1)
    # two sets of chunk states and the per-head dB, dC terms at least
    assert w % 256 == 0 and w >= 2 * (4 * 8 * 80 * 64 * 128 * 4) + 2 * (4 * 2048 * 80 * 128 * 4)
    assert f(4, 2048, 80, 64, 3, 128, 256, 1) == 0      # H % G != 0
    assert f(4, 2048, 80, 256, 1, 128, 256, 1) == 0     # P above the limit
    assert f(1, 0, 2, 16, 1, 16, 64, 0) > 0             # empty sequence is valid


def test_bwd_workspace_holds_the_head_sums(lib):
    # the tensor-core dB and dC scans keep, in the per-head terms' regions, one 128-row partial sum per
    # (CTA, (chunk, 128-row block, group)) slot (up to 256 CTAs) plus two half-row dot products per
    # (batch, token, head); with one head per group and a ragged last chunk that exceeds the per-head terms
    f = lib.ssd_bwd_workspace_bytes
    for batch, T, H, G, N, Q in [(1, 130, 2, 2, 128, 256), (4, 2048, 80, 1, 128, 256), (2, 600, 8, 2, 64, 128)]:
        nc = -(-T // Q)
        keys = batch * nc * (Q // 128) * G
        sums = (256 + keys) * 128 * N * 4 + 2 * batch * T * H * 4
        perhead = batch * T * H * N * 4
        assert f(batch, T, H, 64, G, N, Q, 1) >= 2 * max(sums, perhead)


def _bwd(lib, **over):
    """ssd_bwd with fake (never dereferenced) pointers; only validation runs."""
    args = dict(x=0x10000, dt=0x20000, A=0x30000, B=0x40000, C=0x50000, D=0x60000, Q=64, init=None, dy=0x70000,
                dfin=None, dx=0x80000, ddt=0x90000, dA=0xa0000, dB=0xb0000, dC=0xc0000, dD=0xd0000, dinit=None,
                batch=1, T=256, H=2, P=16, G=1, N=16, dtype=0, ws=0x100000, wsb=1 << 40, stream=None)
    args.update(over)
    v = lambda a: None if a is None else ctypes.c_void_p(a)  # noqa: E731
    a = args
    return lib.ssd_bwd(v(a["x"]), v(a["dt"]), v(a["A"]), v(a["B"]), v(a["C"]), v(a["D"]), a["Q"], v(a["init"]),
                       v(a["dy"]), v(a["dfin"]), v(a["dx"]), v(a["ddt"]), v(a["dA"]), v(a["dB"]), v(a["dC"]),
                       v(a["dD"]), v(a["dinit"]), a["batch"], a["T"], a["H"], a["P"], a["G"], a["N"], a["dtype"],
                       v(a["ws"]), ctypes.c_size_t(a["wsb"]), v(a["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(x=None), 1), (dict(dy=None), 1), (dict(dx=None), 1), (dict(ddt=None), 1), (dict(dA=None), 1),
    (dict(dB=None), 1), (dict(dC=None), 1), (dict(dD=None), 1), (dict(ws=None), 1),
    (dict(H=3, G=2), 1), (dict(dtype=5), 1), (dict(Q=0), 1), (dict(P=256), 2), (dict(batch=70000), 2),
    (dict(wsb=16), 1),                                    # workspace too small
    (dict(ws=0x100010), 1),                               # workspace not 256-byte aligned
    (dict(dtype=1, x=0x10001), 1),                        # bf16 tensor not 2-byte aligned
    (dict(dx=0x10000), 1),                                # dx aliases x
    (dict(dB=0x70000 + 64), 1),                           # dB inside dy
    (dict(dfin=0x200000, dinit=0x200000), 1),             # dinit aliases dfinal
    (dict(dC=0xb0000), 1),                                # two outputs on one buffer
    (dict(dD=0x100000 + 256), 1),                         # an output inside the workspace
])
def test_bwd_rejects_invalid_arguments_on_the_host(lib, over, code):
    assert _bwd(lib, **over) == code
