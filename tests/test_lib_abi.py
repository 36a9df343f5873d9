"""The C-ABI library: it builds, loads, exports every symbol include/mhc.h
declares, and its host-side checks reject bad arguments before touching a GPU.
CPU only: no call here reaches a kernel launch."""

import ctypes
import os
import re

import pytest

from mhc_residual_stream_b200 import build
from mhc_residual_stream_b200 import mhc as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mhc.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return M.lib()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"MHC_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_header_declares_the_boundary_calls():
    names = set(declared_functions())
    for want in ("mhc_boundary_post_pre", "mhc_boundary_residual_only", "mhc_boundary_moe_finalize",
                 "mhc_coeffs", "mxfp8_quantize_rows", "mhc_workspace_bytes", "mhc_get_device_status"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    # nothing beyond the header leaks out
    out = os.popen(f"nm -D --defined-only {M.LIB_PATH}").read().split("\n")
    exported = {line.split()[-1] for line in out if " T " in line}
    assert exported == set(names)


def test_sizes(L):
    assert M.mhc_mxfp8_scale_bytes(32, 7168, True) == 128 * 224
    assert M.mhc_mxfp8_scale_bytes(130, 192, True) == 256 * 8
    assert M.mhc_mxfp8_scale_bytes(5, 7168, False) == 5 * 224
    assert M.mhc_mxfp8_scale_bytes(5, 100, True) == 0
    ws = M.mhc_workspace_bytes(32, 7168, 4)
    assert ws >= 1024 + 32 * 112 * 4 + 32 * 112 * 32 * 4
    assert M.mhc_workspace_bytes(16, 7168, 4) <= ws  # smaller rows fit a larger workspace
    for bad in ((0, 7168, 4), (129, 7168, 4), (4, 7100, 4), (4, 7168, 3), (4, 7168, 8), (4, 9536, 4)):
        assert M.mhc_workspace_bytes(*bad) == 0
    assert M.mhc_workspace_bytes(4, 9472, 4) > 0  # H/64 = 148 blocks is the largest
    # packed fn: per 64-column block [3][CP8][n*64 + 8] bf16, CP8 = C rounded up to 8
    assert M.mhc_projection_pack_bytes(7168, 4) == 112 * 3 * 24 * 264 * 2
    assert M.mhc_projection_pack_bytes(320, 2) == 5 * 3 * 8 * 136 * 2
    assert M.mhc_projection_pack_bytes(64, 1) == 1 * 3 * 8 * 72 * 2
    for bad in ((7100, 4), (7168, 3), (9536, 4), (0, 4)):
        assert M.mhc_projection_pack_bytes(*bad) == 0


def test_status_strings(L):
    for code, name in M.STATUS_NAMES.items():
        assert M.mhc_status_string(code) == name


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_host_checks_reject_before_launch(L):
    f = L.mhc_boundary_post_pre
    a = _fake()
    args = dict(partials=a, P=8, stride=32 * 256, residual=a, post=a, comb=a, pre=None, nw=None, eps=0.0,
                coeffs=None, res_out=a, aux=None, li=None, q=None, po=None, co=None, pr=None, R=32, H=256, n=4,
                ws=None, wsb=0, s=None)

    def call(**kw):
        d = dict(args)
        d.update(kw)
        return f(*d.values())

    assert call(R=0) == M.UNSUPPORTED_SHAPE
    assert call(R=129) == M.UNSUPPORTED_SHAPE
    assert call(H=100) == M.UNSUPPORTED_SHAPE
    assert call(n=3) == M.UNSUPPORTED_SHAPE
    assert call(P=0) == M.UNSUPPORTED_SHAPE
    assert call(P=17) == M.UNSUPPORTED_SHAPE
    assert call(partials=None) == M.INVALID_ARG
    assert call(partials=_fake(0x10008)) == M.INVALID_ARG  # not 16-byte aligned
    assert call(stride=12) == M.INVALID_ARG
    assert call(residual=None) == M.INVALID_ARG
    # residual-only with a tail argument is a contradiction
    assert call(li=a) == M.INVALID_ARG
    # full boundary without a workspace
    assert call(pre=a, nw=a, li=a) == M.WORKSPACE
    assert call(pre=a, nw=a, li=a, ws=_fake(0x10010), wsb=1 << 20) == M.WORKSPACE  # misaligned
    assert call(pre=a, nw=a, li=a, ws=a, wsb=100) == M.WORKSPACE  # too small
    assert call(pre=a, nw=a, li=a, eps=-1.0, ws=a, wsb=1 << 20) == M.INVALID_ARG
    bad_coeff = M.CoeffArgs(0x10000, 0x10000, 0x10000, 1e-6, 1e-6, 1e-6, 2.0, -1)
    assert call(pre=a, nw=a, li=a, ws=a, wsb=1 << 20, coeffs=ctypes.byref(bad_coeff)) == M.INVALID_ARG
    ok_coeff = M.CoeffArgs(0x10000, 0x10000, 0x10000, 1e-6, 1e-6, 1e-6, 2.0, 20)
    # coefficients requested without outputs
    assert call(pre=a, nw=a, li=a, ws=a, wsb=1 << 20, coeffs=ctypes.byref(ok_coeff)) == M.INVALID_ARG
    q = M.Mxfp8Out(0x10004, 0x10000, 1)  # data not 8-byte aligned
    assert call(pre=a, nw=a, li=a, ws=a, wsb=1 << 20, q=ctypes.byref(q)) == M.INVALID_ARG
    assert call(aux=_fake(0x10008)) == M.INVALID_ARG  # aux not 16-byte aligned


def test_other_entry_points_host_checks(L):
    a = _fake()
    assert L.mhc_boundary_residual_only(a, 8, 0, a, a, a, a, None, 4, 256, 4, None) == M.INVALID_ARG  # stride 0
    assert L.mhc_boundary_residual_only(a, 1, 0, a, a, a, a, None, 4, 256, 5, None) == M.UNSUPPORTED_SHAPE
    assert L.mhc_boundary_residual_only(a, 1, 0, a, a, a, a, _fake(0x10004), 4, 256, 4, None) == M.INVALID_ARG
    c = M.CoeffArgs(0x10000, 0x10000, 0x10000, 1e-6, 1e-6, 1e-6, 2.0, 20)
    # both residual and x, or neither
    assert L.mhc_coeffs(a, ctypes.byref(c), None, a, None, None, 0.0, None, a, a, a, 4, 256, 4, a, 1 << 20, None) \
        == M.INVALID_ARG
    assert L.mhc_coeffs(None, ctypes.byref(c), None, None, None, None, 0.0, None, a, a, a, 4, 256, 4, a, 1 << 20,
                        None) == M.INVALID_ARG
    # first layer takes no pre_mix
    assert L.mhc_coeffs(None, ctypes.byref(c), a, a, None, None, 0.0, None, a, a, a, 4, 256, 4, a, 1 << 20, None) \
        == M.INVALID_ARG
    # finalize: top_k out of range
    assert L.mhc_boundary_moe_finalize(a, 64, a, a, 17, a, a, a, a, None, None, 0.0, None, a, None, None, None,
                                       None, None, None, 4, 256, 4, a, 1 << 20, None) == M.UNSUPPORTED_SHAPE
    q = M.Mxfp8Out(0x10000, 0x10000, 1)
    assert L.mxfp8_quantize_rows(a, 4, 48, ctypes.byref(q), None) == M.UNSUPPORTED_SHAPE
    assert L.mxfp8_quantize_rows(None, 4, 64, ctypes.byref(q), None) == M.INVALID_ARG
    assert L.mxfp8_quantize_rows(a, 4, 64, None, None) == M.INVALID_ARG
    assert L.mhc_projection_pack(a, a, 7100, 4, None) == M.UNSUPPORTED_SHAPE
    assert L.mhc_projection_pack(None, a, 7168, 4, None) == M.INVALID_ARG
    assert L.mhc_projection_pack(a, _fake(0x10008), 7168, 4, None) == M.INVALID_ARG  # packed not 16-aligned
    # coefficients with neither fn nor packed fn, or a misaligned packed fn
    for bad in (M.CoeffArgs(None, 0x10000, 0x10000, 1e-6, 1e-6, 1e-6, 2.0, 20, None),
                M.CoeffArgs(None, 0x10000, 0x10000, 1e-6, 1e-6, 1e-6, 2.0, 20, 0x10008)):
        assert L.mhc_coeffs(a, ctypes.byref(bad), None, None, None, None, 0.0, None, a, a, a, 4, 256, 4, a,
                            1 << 20, None) == M.INVALID_ARG
    # the partial table: bad table, entries and counts are refused before any launch
    res = dict(residual=a, post=a, comb=a)

    def ptrs(table, n_parts, R=4, H=256, n=4):
        t = None if table is None else ctypes.cast((ctypes.c_void_p * len(table))(*table), ctypes.c_void_p)
        return L.mhc_boundary_post_pre_ptrs(t, n_parts, res["residual"], res["post"], res["comb"], None, None, 0.0,
                                            None, a, None, None, None, None, None, None, R, H, n, None, 0, None)
    assert ptrs(None, 2) == M.INVALID_ARG
    assert ptrs([0x10000, None], 2) == M.INVALID_ARG
    assert ptrs([0x10000, 0x10008], 2) == M.INVALID_ARG  # a partial not 16-byte aligned
    assert ptrs([0x10000], 0) == M.UNSUPPORTED_SHAPE
    assert ptrs([0x10000] * 17, 17) == M.UNSUPPORTED_SHAPE
    assert ptrs([0x10000], 1, H=100) == M.UNSUPPORTED_SHAPE
    # IPC helpers: argument checks only (no GPU here)
    assert M.lib().mhc_ipc_handle_bytes() == 72
    assert L.mhc_ipc_export(None, a) == M.INVALID_ARG
    assert L.mhc_ipc_export(a, None) == M.INVALID_ARG
    assert L.mhc_ipc_import(None, None) == M.INVALID_ARG
    assert L.mhc_ipc_release(ctypes.c_void_p(0x12340)) == M.INVALID_ARG  # never imported
    # mailbox: sizes (header 256, slots [2][W][max_rows][H] bf16) and refusals
    assert M.mhc_mailbox_bytes(2, 32, 7168) == 256 + 2 * 2 * 32 * 7168 * 2
    assert M.mhc_mailbox_bytes(8, 128, 64) == 256 + 2 * 8 * 128 * 64 * 2
    for bad in ((0, 32, 7168), (17, 32, 7168), (2, 0, 7168), (2, 129, 7168), (2, 32, 100)):
        assert M.mhc_mailbox_bytes(*bad) == 0
    mbs = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    tbl = ctypes.cast(mbs, ctypes.c_void_p)
    pub = L.mhc_mailbox_publish  # (x, rows, hidden, rank, round, mailboxes, world, max_rows, stream)
    assert pub(a, 4, 256, 2, 0, tbl, 2, 4, None) == M.INVALID_ARG  # rank >= world
    assert pub(a, 4, 256, 0, 0xFFFFFFFF, tbl, 2, 4, None) == M.INVALID_ARG
    assert pub(_fake(0x10008), 4, 256, 0, 0, tbl, 2, 4, None) == M.INVALID_ARG
    assert pub(a, 4, 256, 0, 0, None, 2, 4, None) == M.INVALID_ARG
    assert pub(a, 4, 256, 0, 0, tbl, 17, 4, None) == M.UNSUPPORTED_SHAPE
    assert pub(a, 5, 256, 0, 0, tbl, 2, 4, None) == M.UNSUPPORTED_SHAPE  # rows > capacity
    assert pub(a, 4, 100, 0, 0, tbl, 2, 4, None) == M.UNSUPPORTED_SHAPE
    bad_mbs = (ctypes.c_void_p * 2)(0x10000, 0x20080)  # a mailbox not 256-byte aligned
    assert pub(a, 4, 256, 0, 0, ctypes.cast(bad_mbs, ctypes.c_void_p), 2, 4, None) == M.INVALID_ARG
    col = L.mhc_boundary_collect  # (mailbox, world, max_rows, round, ... as post_pre_ptrs from residual on)
    tail = (a, a, a, None, None, 0.0, None, a, None, None, None, None, None, None, 4, 256, 4)
    assert col(_fake(0x10080), 2, 4, 0, *tail, a, 1 << 20, None) == M.INVALID_ARG  # not 256-byte aligned
    assert col(a, 0, 4, 0, *tail, a, 1 << 20, None) == M.UNSUPPORTED_SHAPE
    assert col(a, 2, 3, 0, *tail, a, 1 << 20, None) == M.UNSUPPORTED_SHAPE  # rows 4 > capacity 3
    assert col(a, 2, 4, 0xFFFFFFFF, *tail, a, 1 << 20, None) == M.INVALID_ARG
    assert col(a, 2, 4, 0, *tail, None, 0, None) == M.WORKSPACE  # the slot wait needs the status word
    assert L.mhc_mailbox_init(_fake(0x10010), 4096, None) == M.INVALID_ARG
    assert L.mhc_mailbox_init(a, 4100, None) == M.INVALID_ARG  # not whole 16-byte units
    assert L.mhc_workspace_init(None, 4096, None) == M.WORKSPACE
    assert L.mhc_get_device_status(None, None) == M.WORKSPACE


def test_phase_stamps_apply_to_the_current_kernels():
    # bench.py --phases instruments a copy of the kernel source at fixed anchors;
    # every anchor must still be found once (the stamped copy is built on the GPU machine)
    from mhc_residual_stream_b200 import build, phase_stamps
    with open(build.SOURCES[0]) as f:
        src = f.read()
    out = phase_stamps.instrument(src)
    assert out.count("mhc::g_ts[tslot]") >= 7 and out.count("mhc::g_tt[tslot]") >= 7
    assert "mhc_phase_read" in out and "mhc_phase_reset" in out
