"""Thin ctypes binding of libmhc.so, the CUDA library of the mHC boundary.

Argument marshalling only: every function here checks the tensors' dtype,
device and layout, passes their device pointers and the current CUDA stream to
the C entry point of the same name (include/mhc.h), and raises MhcError on a
non-OK status. All arithmetic runs in the library's kernels. There is no CPU
fallback: without the built library every call raises.

Shapes follow the C ABI: residual [R, n, H] bf16, partials [P, R, H] bf16 (any
stride between partials), post [R, n], comb [R, n, n], pre [R, n] fp32,
norm_weight [H] bf16, fn [n*H, 2n+n^2] fp32.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmhc.so")

OK, INVALID_ARG, UNSUPPORTED_SHAPE, WORKSPACE, CUDA, DEVICE_TIMEOUT, DEVICE_INDEX = range(7)
STATUS_NAMES = {0: "MHC_OK", 1: "MHC_ERR_INVALID_ARG", 2: "MHC_ERR_UNSUPPORTED_SHAPE",
                3: "MHC_ERR_WORKSPACE", 4: "MHC_ERR_CUDA", 5: "MHC_ERR_DEVICE_TIMEOUT",
                6: "MHC_ERR_DEVICE_INDEX"}


class MhcError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class CoeffArgs(ctypes.Structure):
    _fields_ = [("fn", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("base", ctypes.c_void_p),
                ("rms_eps", ctypes.c_float), ("pre_eps", ctypes.c_float),
                ("sinkhorn_eps", ctypes.c_float), ("post_alpha", ctypes.c_float),
                ("sinkhorn_iters", ctypes.c_int), ("fn_packed", ctypes.c_void_p)]


class Mxfp8Out(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("swizzled_128x4", ctypes.c_int)]


@dataclass
class Coeffs:
    """Device tensors and scalars of the next-coefficient step (mhc_coeff_args).
    `fn_packed` (optional) is fn as mhc_projection_pack wrote it; with it set the
    kernels read it instead of fn, and fn may be None."""
    fn: Optional[torch.Tensor]
    scale: torch.Tensor
    base: torch.Tensor
    rms_eps: float = 1e-6
    pre_eps: float = 1e-6
    sinkhorn_eps: float = 1e-6
    post_alpha: float = 2.0
    sinkhorn_iters: int = 20
    fn_packed: Optional[torch.Tensor] = None

    @classmethod
    def from_weights(cls, w, device, packed: bool = False) -> "Coeffs":
        """From any object with the same fields (e.g. synthetic.CoeffWeights) on the CPU;
        `packed` also packs fn (mhc_projection_pack) on `device`."""
        fn = w.fn.to(device).contiguous()
        c = cls(fn=fn, scale=w.scale.to(device).contiguous(), base=w.base.to(device).contiguous(),
                rms_eps=w.rms_eps, pre_eps=w.pre_eps, sinkhorn_eps=w.sinkhorn_eps, post_alpha=w.post_alpha,
                sinkhorn_iters=w.sinkhorn_iters)
        if packed:
            n = int(round((fn.shape[1] + 1) ** 0.5)) - 1  # C = n^2 + 2n
            c.fn_packed = mhc_projection_pack(fn, fn.shape[0] // n, n)
        return c


_lib = None
_vp, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mhc_residual_stream_b200.build` "
                           "(the mHC boundary has no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "mhc_workspace_bytes": (_sz, [_i, _i, _i]),
        "mhc_mxfp8_scale_bytes": (_sz, [_i, _i, _i]),
        "mhc_workspace_init": (_i, [_vp, _sz, _vp]),
        "mhc_boundary_post_pre": (_i, [_vp, _i, _i64, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
        "mhc_boundary_post_pre_noalloc": (_i, [_vp, _i, _i64, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
        "mhc_boundary_moe_finalize": (_i, [_vp, _i, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _f, _vp,
                                           _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
        "mhc_boundary_residual_only": (_i, [_vp, _i, _i64, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
        "mhc_coeffs": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
        "mxfp8_quantize_rows": (_i, [_vp, _i, _i, _vp, _vp]),
        "mhc_get_device_status": (_i, [_vp, _vp]),
        "mhc_status_string": (ctypes.c_char_p, [_i]),
        "mhc_debug_set_wait": (_i64, [_i64, _i]),
        "mhc_boundary_post_pre_ptrs": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, _vp,
                                            _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
        "mhc_mailbox_bytes": (_sz, [_i, _i, _i]),
        "mhc_mailbox_init": (_i, [_vp, _sz, _vp]),
        "mhc_mailbox_publish": (_i, [_vp, _i, _i, _i, ctypes.c_uint32, _vp, _i, _i, _vp]),
        "mhc_boundary_collect": (_i, [_vp, _i, _i, ctypes.c_uint32, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, _vp,
                                      _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
        "mhc_ipc_handle_bytes": (_sz, []),
        "mhc_ipc_export": (_i, [_vp, _vp]),
        "mhc_ipc_import": (_i, [_vp, ctypes.POINTER(ctypes.c_void_p)]),
        "mhc_ipc_release": (_i, [_vp]),
        "mhc_projection_pack_bytes": (_sz, [_i, _i]),
        "mhc_projection_pack": (_i, [_vp, _vp, _i, _i, _vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


# ------------------------------------------------------------------ marshalling helpers

def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _need(t, dtype, name, dims=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got {tuple(t.shape)}")


def _contig(t, name):
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check(status: int, where: str):
    if status != OK:
        raise MhcError(status, where)


def _coeff_struct(c: Optional[Coeffs]):
    if c is None:
        return None
    _need(c.fn, torch.float32, "fn", 2)
    _need(c.fn_packed, torch.uint8, "fn_packed", 1)
    _need(c.scale, torch.float32, "scale", 1)
    _need(c.base, torch.float32, "base", 1)
    for t, n in ((c.fn, "fn"), (c.fn_packed, "fn_packed"), (c.scale, "scale"), (c.base, "base")):
        _contig(t, n)
    return CoeffArgs(_p(c.fn), c.scale.data_ptr(), c.base.data_ptr(), c.rms_eps, c.pre_eps,
                     c.sinkhorn_eps, c.post_alpha, int(c.sinkhorn_iters), _p(c.fn_packed))


def _mxfp8_struct(q):
    if q is None:
        return None
    data, scale, swizzled = q
    _need(data, torch.uint8, "mxfp8 data", 2)
    _need(scale, torch.uint8, "mxfp8 scale")
    _contig(data, "mxfp8 data")
    _contig(scale, "mxfp8 scale")
    return Mxfp8Out(data.data_ptr(), scale.data_ptr(), 1 if swizzled else 0)


def _ref(s):
    return None if s is None else ctypes.byref(s)


# ------------------------------------------------------------------ sizes / workspace

def mhc_workspace_bytes(rows: int, hidden: int, hc_mult: int) -> int:
    return int(lib().mhc_workspace_bytes(rows, hidden, hc_mult))


def mhc_mxfp8_scale_bytes(rows: int, hidden: int, swizzled_128x4: bool = True) -> int:
    return int(lib().mhc_mxfp8_scale_bytes(rows, hidden, 1 if swizzled_128x4 else 0))


def new_workspace(rows: int, hidden: int, hc_mult: int, device=None) -> torch.Tensor:
    """A zeroed workspace (torch's caching allocator returns 512-byte aligned blocks)."""
    n = mhc_workspace_bytes(rows, hidden, hc_mult)
    if n == 0:
        raise MhcError(UNSUPPORTED_SHAPE, "mhc_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def mhc_workspace_init(workspace: torch.Tensor, stream=None):
    _check(lib().mhc_workspace_init(_p(workspace), workspace.numel(), _stream(stream)), "mhc_workspace_init")


def mhc_get_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise `stream`, then read and clear the status a kernel recorded."""
    return int(lib().mhc_get_device_status(_p(workspace), _stream(stream)))


def mhc_projection_pack_bytes(hidden: int, hc_mult: int) -> int:
    return int(lib().mhc_projection_pack_bytes(hidden, hc_mult))


def mhc_projection_pack(fn: torch.Tensor, hidden: int, hc_mult: int, out: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """fn [n*H, C] fp32 rewritten into the projection's tile form (a uint8 device
    tensor of mhc_projection_pack_bytes); done once per weight, at load time."""
    _need(fn, torch.float32, "fn", 2)
    _contig(fn, "fn")
    n = mhc_projection_pack_bytes(hidden, hc_mult)
    if n == 0:
        raise MhcError(UNSUPPORTED_SHAPE, "mhc_projection_pack_bytes")
    C = 2 * hc_mult + hc_mult * hc_mult
    if tuple(fn.shape) != (hc_mult * hidden, C):
        raise ValueError(f"fn must be [{hc_mult * hidden}, {C}], got {tuple(fn.shape)}")
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=fn.device)
    _need(out, torch.uint8, "packed", 1)
    if out.numel() < n:
        raise ValueError(f"packed needs {n} bytes")
    _check(lib().mhc_projection_pack(_p(fn), _p(out), hidden, hc_mult, _stream(stream)), "mhc_projection_pack")
    return out


def mhc_debug_set_wait(budget_ns: int, extra_units: int) -> int:
    """Test hook: the time limit of the kernels' bounded wait, and extra 16-byte
    units that wait should expect (so that it runs out)."""
    return int(lib().mhc_debug_set_wait(int(budget_ns), int(extra_units)))


# ------------------------------------------------------------------ entry points

def _mix_args(residual, post, comb, residual_out):
    _need(residual, torch.bfloat16, "residual", 3)
    _need(post, torch.float32, "post", 2)
    _need(comb, torch.float32, "comb", 3)
    _need(residual_out, torch.bfloat16, "residual_out", 3)
    for t, n in ((residual, "residual"), (post, "post"), (comb, "comb"), (residual_out, "residual_out")):
        _contig(t, n)
    R, n, H = residual.shape
    if tuple(residual_out.shape) != (R, n, H) or tuple(post.shape) != (R, n) or tuple(comb.shape) != (R, n, n):
        raise ValueError("residual/post/comb/residual_out shapes disagree")
    return R, n, H


def _partials_args(partials, R, H):
    _need(partials, torch.bfloat16, "partials", 3)
    if partials.shape[1:] != (R, H) or partials.stride(2) != 1 or partials.stride(1) != H:
        raise ValueError("partials must be [P, R, H] with contiguous rows")
    return partials.shape[0], partials.stride(0)


def _tail_args(pre, norm_weight, layer_input, post_out, comb_out, pre_out, R, n, H):
    _need(pre, torch.float32, "pre", 2)
    _need(norm_weight, torch.bfloat16, "norm_weight", 1)
    _need(layer_input, torch.bfloat16, "layer_input", 2)
    for t, n_, shp in ((post_out, "post_out", (R, n)), (comb_out, "comb_out", (R, n, n)), (pre_out, "pre_out", (R, n))):
        _need(t, torch.float32, n_)
        _contig(t, n_)
        if t is not None and tuple(t.shape) != shp:
            raise ValueError(f"{n_} must be {shp}")
    for t, n_ in ((pre, "pre"), (norm_weight, "norm_weight"), (layer_input, "layer_input")):
        _contig(t, n_)


def _aux_arg(aux, R, H):
    _need(aux, torch.bfloat16, "aux", 2)
    _contig(aux, "aux")
    if aux is not None and tuple(aux.shape) != (R, H):
        raise ValueError(f"aux must be [{R}, {H}]")


def mhc_boundary_post_pre(partials, residual, post, comb, pre, norm_weight, norm_eps, coeffs: Optional[Coeffs],
                          residual_out, layer_input=None, mxfp8=None, post_out=None, comb_out=None,
                          pre_out=None, workspace=None, stream=None, aux=None):
    """Boundary after a partial-output sublayer. mxfp8 = (data, scale, swizzled) or None;
    aux (optional, bf16 [R, H]) receives the mean of the new streams."""
    R, n, H = _mix_args(residual, post, comb, residual_out)
    P, stride = _partials_args(partials, R, H)
    _tail_args(pre, norm_weight, layer_input, post_out, comb_out, pre_out, R, n, H)
    _aux_arg(aux, R, H)
    cs, qs = _coeff_struct(coeffs), _mxfp8_struct(mxfp8)
    st = lib().mhc_boundary_post_pre(
        _p(partials), P, stride, _p(residual), _p(post), _p(comb), _p(pre), _p(norm_weight), float(norm_eps),
        _ref(cs), _p(residual_out), _p(aux), _p(layer_input), _ref(qs), _p(post_out), _p(comb_out), _p(pre_out),
        R, H, n, _p(workspace), 0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "mhc_boundary_post_pre")


def mhc_boundary_post_pre_ptrs(partial_ptrs, residual, post, comb, pre, norm_weight, norm_eps,
                               coeffs: Optional[Coeffs], residual_out, layer_input=None, mxfp8=None, post_out=None,
                               comb_out=None, pre_out=None, workspace=None, stream=None, aux=None):
    """mhc_boundary_post_pre with the partials as a list of device addresses (ints),
    each a [R, H] bf16 partial that may live in another GPU's memory (the
    tensor-parallel boundary; see PeerPartials in tp.py)."""
    R, n, H = _mix_args(residual, post, comb, residual_out)
    ptrs = [int(a) for a in partial_ptrs]
    if not 1 <= len(ptrs) <= 16:
        raise MhcError(UNSUPPORTED_SHAPE, "mhc_boundary_post_pre_ptrs")
    _tail_args(pre, norm_weight, layer_input, post_out, comb_out, pre_out, R, n, H)
    _aux_arg(aux, R, H)
    table = (ctypes.c_void_p * len(ptrs))(*ptrs)
    cs, qs = _coeff_struct(coeffs), _mxfp8_struct(mxfp8)
    st = lib().mhc_boundary_post_pre_ptrs(
        ctypes.cast(table, ctypes.c_void_p), len(ptrs), _p(residual), _p(post), _p(comb), _p(pre), _p(norm_weight),
        float(norm_eps), _ref(cs), _p(residual_out), _p(aux), _p(layer_input), _ref(qs), _p(post_out),
        _p(comb_out), _p(pre_out), R, H, n, _p(workspace), 0 if workspace is None else workspace.numel(),
        _stream(stream))
    _check(st, "mhc_boundary_post_pre_ptrs")


def mhc_mailbox_bytes(world: int, max_rows: int, hidden: int) -> int:
    return int(lib().mhc_mailbox_bytes(world, max_rows, hidden))


def mhc_mailbox_init(mailbox: torch.Tensor, stream=None):
    """Header zero, every slot element negative zero ("not yet written")."""
    _check(lib().mhc_mailbox_init(_p(mailbox), mailbox.numel(), _stream(stream)), "mhc_mailbox_init")


def new_mailbox(world: int, max_rows: int, hidden: int, device=None, stream=None) -> torch.Tensor:
    """An initialised mailbox (uint8 device tensor) for a group of `world`
    producers and up to `max_rows` tokens a round."""
    n = mhc_mailbox_bytes(world, max_rows, hidden)
    if n == 0:
        raise MhcError(UNSUPPORTED_SHAPE, "mhc_mailbox_bytes")
    mb = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    mhc_mailbox_init(mb, stream)
    return mb


def mhc_mailbox_publish(x: torch.Tensor, rank: int, round_: int, mailbox_ptrs, max_rows: int, stream=None):
    """Producer `rank`: store x [R, H] bf16 (R <= max_rows) into slot
    [round & 1][rank] of every consumer's mailbox (device addresses, rank order)."""
    _need(x, torch.bfloat16, "x", 2)
    _contig(x, "x")
    ptrs = [int(a) for a in mailbox_ptrs]
    table = (ctypes.c_void_p * len(ptrs))(*ptrs)
    R, H = x.shape
    _check(lib().mhc_mailbox_publish(_p(x), R, H, int(rank), int(round_), ctypes.cast(table, ctypes.c_void_p),
                                     len(ptrs), int(max_rows), _stream(stream)), "mhc_mailbox_publish")


def mhc_boundary_collect(mailbox, world: int, max_rows: int, round_: int, residual, post, comb, pre, norm_weight,
                         norm_eps, coeffs: Optional[Coeffs], residual_out, layer_input=None, mxfp8=None, post_out=None,
                         comb_out=None, pre_out=None, workspace=None, stream=None, aux=None):
    """The consumer's boundary of round `round_` over the `world` slots of its mailbox
    (a tensor from new_mailbox, or a device address)."""
    R, n, H = _mix_args(residual, post, comb, residual_out)
    _tail_args(pre, norm_weight, layer_input, post_out, comb_out, pre_out, R, n, H)
    _aux_arg(aux, R, H)
    mb = mailbox.data_ptr() if isinstance(mailbox, torch.Tensor) else int(mailbox)
    cs, qs = _coeff_struct(coeffs), _mxfp8_struct(mxfp8)
    st = lib().mhc_boundary_collect(
        mb, int(world), int(max_rows), int(round_), _p(residual), _p(post), _p(comb), _p(pre), _p(norm_weight), float(norm_eps),
        _ref(cs), _p(residual_out), _p(aux), _p(layer_input), _ref(qs), _p(post_out), _p(comb_out), _p(pre_out),
        R, H, n, _p(workspace), 0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "mhc_boundary_collect")


def ipc_export(t: torch.Tensor) -> bytes:
    """The handle another process passes to ipc_import to map t's memory."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("ipc_export needs a CUDA tensor")
    buf = ctypes.create_string_buffer(int(lib().mhc_ipc_handle_bytes()))
    _check(lib().mhc_ipc_export(_p(t), buf), "mhc_ipc_export")
    return buf.raw


def ipc_import(handle: bytes) -> int:
    """Device address of memory another process exported (release with ipc_release)."""
    out = ctypes.c_void_p()
    _check(lib().mhc_ipc_import(ctypes.create_string_buffer(handle, len(handle)), ctypes.byref(out)),
           "mhc_ipc_import")
    return int(out.value)


def ipc_release(addr: int):
    _check(lib().mhc_ipc_release(ctypes.c_void_p(addr)), "mhc_ipc_release")


def mhc_boundary_post_pre_noalloc(partials, residual, post, comb, pre, norm_weight, norm_eps,
                                  coeffs: Optional[Coeffs], residual_out, layer_input=None, mxfp8=None,
                                  post_out=None, comb_out=None, pre_out=None, stream=None, aux=None):
    """mhc_boundary_post_pre without a workspace, for callers that cannot allocate
    device memory (a runtime that owns all memory, graph capture, allocation-free
    serving loops): the scratch is a fixed array inside the library. Limits:
    rows <= 128, hidden <= 7168, hc_mult <= 4. Calls on one device must not
    overlap on the GPU."""
    R, n, H = _mix_args(residual, post, comb, residual_out)
    P, stride = _partials_args(partials, R, H)
    _tail_args(pre, norm_weight, layer_input, post_out, comb_out, pre_out, R, n, H)
    _aux_arg(aux, R, H)
    cs, qs = _coeff_struct(coeffs), _mxfp8_struct(mxfp8)
    st = lib().mhc_boundary_post_pre_noalloc(
        _p(partials), P, stride, _p(residual), _p(post), _p(comb), _p(pre), _p(norm_weight), float(norm_eps),
        _ref(cs), _p(residual_out), _p(aux), _p(layer_input), _ref(qs), _p(post_out), _p(comb_out), _p(pre_out),
        R, H, n, _stream(stream))
    _check(st, "mhc_boundary_post_pre_noalloc")


def mhc_boundary_moe_finalize(gemm2_permuted, expert_weights, expanded_idx_to_permuted_idx, shared_output,
                              residual, post, comb, pre, norm_weight, norm_eps, coeffs: Optional[Coeffs],
                              residual_out, layer_input=None, mxfp8=None, post_out=None, comb_out=None,
                              pre_out=None, workspace=None, stream=None, aux=None):
    """Boundary after a MoE sublayer left unfinalized; aux as in mhc_boundary_post_pre."""
    R, n, H = _mix_args(residual, post, comb, residual_out)
    _need(gemm2_permuted, torch.bfloat16, "gemm2_permuted", 2)
    _need(expert_weights, torch.float32, "expert_weights", 2)
    _need(expanded_idx_to_permuted_idx, torch.int32, "expanded_idx_to_permuted_idx", 1)
    _need(shared_output, torch.bfloat16, "shared_output", 2)
    for t, n_ in ((gemm2_permuted, "gemm2_permuted"), (expert_weights, "expert_weights"),
                  (expanded_idx_to_permuted_idx, "expanded_idx_to_permuted_idx"), (shared_output, "shared_output")):
        _contig(t, n_)
    k = expert_weights.shape[1]
    if gemm2_permuted.shape[1] != H or tuple(shared_output.shape) != (R, H) or expert_weights.shape[0] != R \
            or expanded_idx_to_permuted_idx.numel() != R * k:
        raise ValueError("MoE finalize shapes disagree")
    _tail_args(pre, norm_weight, layer_input, post_out, comb_out, pre_out, R, n, H)
    _aux_arg(aux, R, H)
    cs, qs = _coeff_struct(coeffs), _mxfp8_struct(mxfp8)
    st = lib().mhc_boundary_moe_finalize(
        _p(gemm2_permuted), gemm2_permuted.shape[0], _p(expert_weights), _p(expanded_idx_to_permuted_idx), k,
        _p(shared_output), _p(residual), _p(post), _p(comb), _p(pre), _p(norm_weight), float(norm_eps), _ref(cs),
        _p(residual_out), _p(aux), _p(layer_input), _ref(qs), _p(post_out), _p(comb_out), _p(pre_out), R, H, n,
        _p(workspace), 0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "mhc_boundary_moe_finalize")


def mhc_boundary_residual_only(partials, residual, post, comb, residual_out, stream=None, aux=None):
    R, n, H = _mix_args(residual, post, comb, residual_out)
    P, stride = _partials_args(partials, R, H)
    _aux_arg(aux, R, H)
    st = lib().mhc_boundary_residual_only(_p(partials), P, stride, _p(residual), _p(post), _p(comb),
                                          _p(residual_out), _p(aux), R, H, n, _stream(stream))
    _check(st, "mhc_boundary_residual_only")


def mhc_coeffs(coeffs: Coeffs, post_out, comb_out, pre_out, residual=None, pre_mix=None, x=None,
               residual_out=None, norm_weight=None, norm_eps=0.0, layer_input=None, workspace=None,
               hc_mult=None, stream=None):
    """Stock mHC pre: coefficients of `residual` [R, n, H] (layer input from pre_mix), or the
    first layer on the embedding `x` [R, H] broadcast to hc_mult streams."""
    if residual is not None:
        _need(residual, torch.bfloat16, "residual", 3)
        _contig(residual, "residual")
        R, n, H = residual.shape
    else:
        _need(x, torch.bfloat16, "x", 2)
        _contig(x, "x")
        R, H = x.shape
        n = int(hc_mult if hc_mult is not None else post_out.shape[1])
        _need(residual_out, torch.bfloat16, "residual_out", 3)
        _contig(residual_out, "residual_out")
    _tail_args(pre_mix, norm_weight, layer_input, post_out, comb_out, pre_out, R, n, H)
    cs = _coeff_struct(coeffs)
    st = lib().mhc_coeffs(_p(residual), _ref(cs), _p(pre_mix), _p(x), _p(residual_out), _p(norm_weight),
                          float(norm_eps), _p(layer_input), _p(post_out), _p(comb_out), _p(pre_out), R, H, n,
                          _p(workspace), 0 if workspace is None else workspace.numel(), _stream(stream))
    _check(st, "mhc_coeffs")


def mxfp8_quantize_rows(x, data, scale, swizzled_128x4: bool = True, stream=None):
    _need(x, torch.bfloat16, "x", 2)
    _contig(x, "x")
    R, H = x.shape
    qs = _mxfp8_struct((data, scale, swizzled_128x4))
    st = lib().mxfp8_quantize_rows(_p(x), R, H, ctypes.byref(qs), _stream(stream))
    _check(st, "mxfp8_quantize_rows")


def mhc_status_string(status: int) -> str:
    return lib().mhc_status_string(int(status)).decode()
