"""Thin Python binding of the m3 C ABI (include/m3.h).

Argument marshalling only: every step of the method runs in the CUDA
library ``libm3.so`` built from ``csrc/``.  PyTorch supplies device memory and
streams.  There is no fallback: if the library is missing, the first call
raises ImportError, and every call checks that its tensors live on a CUDA
device.  With ``M3_BOUNDS=1`` in the environment when the library is first
loaded, the binding loads the bounds build ``libm3_bounds.so`` instead (the
same ABI with device-side index checks; ``device_checks()`` tells which).
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libm3.so")
BOUNDS_LIB_PATH = os.path.join(_HERE, "libm3_bounds.so")

M3_OK, M3_ERR_INVALID_ARG, M3_ERR_UNSUPPORTED, M3_ERR_CUDA, M3_ERR_TIMEOUT, M3_ERR_BOUNDS = range(6)
M3_F32, M3_BF16 = 0, 1
M3_FLAG_A_PER_TOKEN = 1
M3_FLAG_THETA_PER_HEAD = 2
ALGO_AUTO, ALGO_SIMT, ALGO_TC = 0, 1, 2
KERNEL_NONE, KERNEL_SIMT, KERNEL_TC, KERNEL_TC32 = 0, 1, 2, 3
PLAN_STATIC = 1


def ALGO_TC_SEGMENTS(s: int) -> int:
    """The tensor-core path with every sequence split into `s` segments."""
    return ALGO_TC | (int(s) << 8)

_STATUS = {0: "M3_OK", 1: "M3_ERR_INVALID_ARG", 2: "M3_ERR_UNSUPPORTED", 3: "M3_ERR_CUDA", 4: "M3_ERR_TIMEOUT",
           5: "M3_ERR_BOUNDS"}


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("rank", ctypes.c_int64),
                ("io", ctypes.c_int32), ("flags", ctypes.c_int32)]


class CBCNorm(ctypes.Structure):
    _fields_ = [("wB", ctypes.c_void_p), ("wC", ctypes.c_void_p), ("bB", ctypes.c_void_p),
                ("bC", ctypes.c_void_p), ("eps", ctypes.c_float)]


class BCNorm(NamedTuple):
    """BC-norm prologue parameters (device fp32 tensors): RMS-norm weights
    wB, wC [N] and head-specific biases bB, bC [H, R, N]; eps > 0."""
    wB: torch.Tensor
    wC: torch.Tensor
    bB: torch.Tensor
    bC: torch.Tensor
    eps: float = 1e-6


def _cbcn(b: BCNorm):
    return ctypes.byref(CBCNorm(b.wB.data_ptr(), b.wC.data_ptr(), b.bB.data_ptr(), b.bC.data_ptr(), float(b.eps)))


class CMimoProj(ctypes.Structure):
    _fields_ = [("wx", ctypes.c_void_p), ("wB", ctypes.c_void_p), ("wC", ctypes.c_void_p), ("wy", ctypes.c_void_p)]


class MimoProj(NamedTuple):
    """MIMO projection weights (device fp32 tensors): wx, wy [H, R, P] and
    wB, wC [H, R, N]; with them x, B, C and y hold one row per token-head
    (see m3_mimo_proj in include/m3.h)."""
    wx: torch.Tensor
    wB: torch.Tensor
    wC: torch.Tensor
    wy: torch.Tensor


def _cproj(p: MimoProj):
    return ctypes.byref(CMimoProj(p.wx.data_ptr(), p.wB.data_ptr(), p.wC.data_ptr(), p.wy.data_ptr()))


class CPlanInfo(ctypes.Structure):
    _fields_ = [("workspace_bytes", ctypes.c_size_t), ("kernel", ctypes.c_int32), ("segments", ctypes.c_int32),
                ("launches", ctypes.c_int32), ("reserved", ctypes.c_int32), ("ctas", ctypes.c_int64)]


class CState(ctypes.Structure):
    _fields_ = [("h", ctypes.c_void_p), ("b_prev", ctypes.c_void_p), ("x_prev", ctypes.c_void_p)]


class M3Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class State(NamedTuple):
    h: torch.Tensor       # [Bt, H, N, P] fp32
    b_prev: torch.Tensor  # [Bt, H, R, N] fp32
    x_prev: torch.Tensor  # [Bt, H, R, P] fp32


def lib_path() -> str:
    """The library the binding loads: the bounds build if M3_BOUNDS=1."""
    return BOUNDS_LIB_PATH if os.environ.get("M3_BOUNDS", "") == "1" else LIB_PATH


def _load():
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(f"m3 CUDA library not built ({path} missing); "
                          "run `python -m state_space_sequence_ssm_b200.build`")
    lib = ctypes.CDLL(path)
    vp, dp = ctypes.c_void_p, ctypes.POINTER(Dims)
    sp = ctypes.POINTER(CState)
    lib.m3_scan_workspace_size.argtypes = [dp, ctypes.POINTER(ctypes.c_size_t)]
    lib.m3_scan_plan.argtypes = [ctypes.c_int, dp, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_int),
                                 ctypes.POINTER(ctypes.c_int)]
    lib.m3_scan_plan_info.argtypes = [ctypes.c_int, dp, ctypes.c_int, ctypes.POINTER(CPlanInfo)]
    lib.m3_scan_plan_info.restype = ctypes.c_int
    lib.m3_scan_fwd.argtypes = [dp] + [vp] * 8 + [sp, vp, sp, vp, ctypes.c_size_t, vp]
    lib.m3_scan_fwd_algo.argtypes = [ctypes.c_int, dp] + [vp] * 8 + [sp, vp, sp, vp, ctypes.c_size_t, vp]
    bp_ = ctypes.POINTER(CBCNorm)
    lib.m3_scan_fwd_bcnorm.argtypes = [ctypes.c_int, dp, bp_] + [vp] * 8 + [sp, vp, sp, vp, ctypes.c_size_t, vp]
    lib.m3_scan_fwd_bcnorm.restype = ctypes.c_int
    lib.m3_step_bcnorm.argtypes = [dp, bp_] + [vp] * 8 + [sp, vp, vp]
    lib.m3_step_bcnorm.restype = ctypes.c_int
    pp_ = ctypes.POINTER(CMimoProj)
    lib.m3_scan_fwd_proj.argtypes = [ctypes.c_int, dp, pp_] + [vp] * 8 + [sp, vp, sp, vp, ctypes.c_size_t, vp]
    lib.m3_scan_fwd_proj.restype = ctypes.c_int
    lib.m3_step_proj.argtypes = [dp, pp_] + [vp] * 8 + [sp, vp, vp]
    lib.m3_step_proj.restype = ctypes.c_int
    lib.m3_scan_fwd_static.argtypes = [ctypes.c_int, dp] + [vp] * 8 + [sp, vp, sp, vp]
    lib.m3_scan_fwd_static.restype = ctypes.c_int
    lib.m3_step.argtypes = [dp] + [vp] * 8 + [sp, vp, vp]
    i64p = ctypes.POINTER(ctypes.c_int64)
    lib.m3_scan_host_plan.argtypes = [dp, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t), i64p, i64p, i64p, i64p]
    lib.m3_scan_host_plan.restype = ctypes.c_int
    lib.m3_scan_fwd_host.argtypes = [dp, ctypes.POINTER(CBCNorm)] + [vp] * 8 + [sp, vp, sp, vp, ctypes.c_size_t, vp]
    lib.m3_scan_fwd_host.restype = ctypes.c_int
    for f in (lib.m3_scan_workspace_size, lib.m3_scan_plan, lib.m3_scan_fwd, lib.m3_scan_fwd_algo, lib.m3_step):
        f.restype = ctypes.c_int
    lib.m3_selftest_segment_timeout.argtypes = [dp, ctypes.c_int] + [vp] * 8 + [sp, vp, sp, vp, ctypes.c_size_t, vp]
    lib.m3_selftest_segment_timeout.restype = ctypes.c_int
    lib.m3_selftest_wait_timeout.argtypes = [vp]
    lib.m3_selftest_wait_timeout.restype = ctypes.c_int
    lib.m3_stream_status.argtypes = [vp]
    lib.m3_stream_status.restype = ctypes.c_int
    lib.m3_last_error.argtypes = []
    lib.m3_last_error.restype = ctypes.c_char_p
    lib.m3_version.restype = ctypes.c_int
    lib.m3_device_checks.restype = ctypes.c_int
    return lib


_lib = None


def get_lib():
    """The loaded library (raises ImportError if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def __getattr__(name):
    if name == "lib":
        return get_lib()
    raise AttributeError(name)


def _check(status: int):
    if status != M3_OK:
        raise M3Error(status, get_lib().m3_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    """The call's stream as a cudaStream_t: `stream`, else the current stream
    of `device` (the tensors' GPU).  A given stream must belong to `device`."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise ValueError(f"m3: stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _require_cuda(*ts):
    """Check that every given tensor is a contiguous CUDA tensor and that they
    all sit on one GPU; return that device (None if no tensor was given).

    The C library launches on the CUDA runtime's current device, so each call
    below runs with this device made current: pointers of a tensor on another
    GPU never reach a kernel on this one."""
    dev = None
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("m3: tensors must be on a CUDA device (no CPU path)")
            if not t.is_contiguous():
                raise ValueError("m3: tensors must be contiguous")
            if dev is None:
                dev = t.device
            elif t.device != dev:
                raise ValueError(f"m3: tensors on different devices ({dev} and {t.device})")
    return dev


def _scratch(nbytes: int, device, stream):
    """A workspace the binding allocates for one call: marked as used by the
    call's stream, so that the caching allocator does not hand it out again
    before that stream has finished with it."""
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if stream is not None:
        ws.record_stream(stream)
    return ws


def make_dims(Bt, T, H, P, N, R, dtype, a_per_token: bool = False, theta_per_head: bool = False) -> Dims:
    io = M3_BF16 if dtype == torch.bfloat16 else M3_F32
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("io dtype must be float32 or bfloat16")
    flags = (M3_FLAG_A_PER_TOKEN if a_per_token else 0) | (M3_FLAG_THETA_PER_HEAD if theta_per_head else 0)
    return Dims(Bt, T, H, P, N, R, io, flags)


def _cstate(s: State | None):
    if s is None:
        return None
    return ctypes.pointer(CState(s.h.data_ptr(), s.b_prev.data_ptr(), s.x_prev.data_ptr()))


def empty_state(Bt, H, N, P, R, device="cuda") -> State:
    f = dict(device=device, dtype=torch.float32)
    return State(torch.zeros(Bt, H, N, P, **f), torch.zeros(Bt, H, R, N, **f), torch.zeros(Bt, H, R, P, **f))


def workspace_size(dims: Dims, algo: int = ALGO_AUTO) -> int:
    """Workspace bytes m3_scan_fwd_algo(algo, dims, ...) needs."""
    return scan_plan(dims, algo)[0]


class Plan(NamedTuple):
    workspace_bytes: int
    segments: int   # per sequence (1 = not split)
    launches: int   # kernel launches of one call


def scan_plan(dims: Dims, algo: int = ALGO_AUTO) -> Plan:
    """How one prefill call with this `algo` runs on the current device."""
    n, sg, ln = ctypes.c_size_t(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(get_lib().m3_scan_plan(algo, ctypes.byref(dims), ctypes.byref(n), ctypes.byref(sg), ctypes.byref(ln)))
    return Plan(n.value, sg.value, ln.value)


class PlanInfo(NamedTuple):
    workspace_bytes: int
    kernel: int     # KERNEL_SIMT, KERNEL_TC or KERNEL_TC32 (KERNEL_NONE: nothing to run)
    segments: int   # per sequence (1 = not split)
    launches: int   # kernel launches of one call
    ctas: int       # CTAs of the (main) launch

    @property
    def kernel_name(self) -> str:
        return {KERNEL_NONE: "none", KERNEL_SIMT: "prefill_simt_kernel", KERNEL_TC: "prefill_tc_kernel",
                KERNEL_TC32: "prefill_tc32_kernel"}[self.kernel]


def scan_plan_info(dims: Dims, algo: int = ALGO_AUTO, flags: int = 0) -> PlanInfo:
    """Which kernel and schedule one prefill call runs on the current device
    (flags: PLAN_STATIC for scan_fwd_static)."""
    info = CPlanInfo()
    _check(get_lib().m3_scan_plan_info(algo, ctypes.byref(dims), flags, ctypes.byref(info)))
    return PlanInfo(info.workspace_bytes, info.kernel, info.segments, info.launches, info.ctas)


def scan_fwd(x, B, C, dt, lam, theta, A, D, init: State | None = None, *, want_state: bool = True,
             y=None, final: State | None = None, workspace=None, algo: int = ALGO_AUTO, stream=None,
             bcnorm: BCNorm | None = None, proj: MimoProj | None = None):
    """Prefill scan (with the BC-norm prologue when `bcnorm` is given).  x [Bt,T,H,R,P], B/C [Bt,T,H,R,N], dt/lam [Bt,T,H],
    theta [Bt,T,H,N/2] (or [H,N/2]: fixed per head) in one io dtype (fp32 or
    bf16); D [H] fp32; A [H] fp32, or [Bt,T,H] fp32 for a data-dependent A_t.
    With the MIMO projections `proj`: x [Bt,T,H,P], B/C [Bt,T,H,N] and y
    [Bt,T,H,P], widened to the rank of proj's weights on chip.
    Returns (y, final State or None)."""
    dev = _require_cuda(x, B, C, dt, lam, theta, A, D, y, workspace, *(init or ()), *(final or ()),
                        *(bcnorm[:4] if bcnorm is not None else ()), *(proj or ()))
    if proj is not None:
        if bcnorm is not None:
            raise M3Error(M3_ERR_UNSUPPORTED, "the MIMO projections do not combine with the BC-norm prologue")
        Bt, T, H, P = x.shape
        R = proj.wx.shape[1]
    else:
        Bt, T, H, R, P = x.shape
    N = B.shape[-1]
    dims = make_dims(Bt, T, H, P, N, R, x.dtype, a_per_token=A.dim() == 3, theta_per_head=theta.dim() == 2)
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty_like(x)
        if final is None and want_state:
            final = State(torch.empty(Bt, H, N, P, device=dev), torch.empty(Bt, H, R, N, device=dev),
                          torch.empty(Bt, H, R, P, device=dev))
        ws_need = workspace_size(dims, algo) if algo != ALGO_SIMT else 0
        if workspace is None and ws_need:
            workspace = _scratch(ws_need, dev, stream)
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        args = (*map(_ptr, (x, B, C, dt, lam, theta, A, D)), _cstate(init), _ptr(y), _cstate(final),
                _ptr(workspace), ws_bytes, _stream(stream, dev))
        if proj is not None:
            _check(get_lib().m3_scan_fwd_proj(algo, ctypes.byref(dims), _cproj(proj), *args))
        elif bcnorm is None:
            _check(get_lib().m3_scan_fwd_algo(algo, ctypes.byref(dims), *args))
        else:
            _check(get_lib().m3_scan_fwd_bcnorm(algo, ctypes.byref(dims), _cbcn(bcnorm), *args))
    return y, final


def scan_fwd_static(x, B, C, dt, lam, theta, A, D, init: State | None = None, *, want_state: bool = True,
                    y=None, final: State | None = None, algo: int = ALGO_AUTO, stream=None):
    """scan_fwd without a workspace: split sequences use the library's own
    device scratch (see m3_scan_fwd_static in include/m3.h for its limits)."""
    dev = _require_cuda(x, B, C, dt, lam, theta, A, D, y, *(init or ()), *(final or ()))
    Bt, T, H, R, P = x.shape
    N = B.shape[-1]
    dims = make_dims(Bt, T, H, P, N, R, x.dtype, a_per_token=A.dim() == 3, theta_per_head=theta.dim() == 2)
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty_like(x)
        if final is None and want_state:
            final = State(torch.empty(Bt, H, N, P, device=dev), torch.empty(Bt, H, R, N, device=dev),
                          torch.empty(Bt, H, R, P, device=dev))
        _check(get_lib().m3_scan_fwd_static(algo, ctypes.byref(dims), *map(_ptr, (x, B, C, dt, lam, theta, A, D)),
                                            _cstate(init), _ptr(y), _cstate(final), _stream(stream, dev)))
    return y, final


class HostPlan(NamedTuple):
    workspace_bytes: int    # device staging memory scan_fwd_host needs
    slice_tokens: int       # tokens per time slice (every group but the last)
    last_slice_tokens: int  # tokens per time slice of the last group
    group_batch: int        # sequences per group
    units: int              # (group, slice) units of one call


def scan_host_plan(dims: Dims, bcnorm: bool = False) -> HostPlan:
    """How scan_fwd_host cuts a problem of these dims into pipelined units."""
    n = ctypes.c_size_t(0)
    ts, tl, gb, u = (ctypes.c_int64(0) for _ in range(4))
    _check(get_lib().m3_scan_host_plan(ctypes.byref(dims), int(bool(bcnorm)), ctypes.byref(n), ctypes.byref(ts),
                                       ctypes.byref(tl), ctypes.byref(gb), ctypes.byref(u)))
    return HostPlan(n.value, ts.value, tl.value, gb.value, u.value)


def _require_host(*ts):
    for t in ts:
        if t is not None:
            if t.is_cuda:
                raise ValueError("m3: scan_fwd_host takes host tensors (pinned for overlapped copies)")
            if not t.is_contiguous():
                raise ValueError("m3: tensors must be contiguous")


def _hstate(s: State | None):
    if s is None:
        return None
    _require_host(*s)
    return ctypes.pointer(CState(s.h.data_ptr(), s.b_prev.data_ptr(), s.x_prev.data_ptr()))


def scan_fwd_host(x, B, C, dt, lam, theta, A, D, init: State | None = None, *, want_state: bool = True,
                  y=None, final: State | None = None, workspace=None, stream=None, bcnorm: BCNorm | None = None):
    """scan_fwd over host tensors (same shapes as scan_fwd; pinned memory lets
    the copies overlap): the library copies the inputs in, runs the scan and
    copies y (and the final state) back, pipelined over time slices, all
    ordered on `stream`.  `workspace` is a CUDA uint8 tensor of at least
    scan_host_plan(dims).workspace_bytes (allocated when None).  Returns
    (y, final State or None) as host tensors, complete once `stream` has
    reached the end of the call.  `bcnorm` (host fp32 tensors) adds the
    BC-norm prologue."""
    _require_host(x, B, C, dt, lam, theta, A, D, y)
    cb = None
    if bcnorm is not None:
        _require_host(bcnorm.wB, bcnorm.wC, bcnorm.bB, bcnorm.bC)
        cb = ctypes.byref(CBCNorm(bcnorm.wB.data_ptr(), bcnorm.wC.data_ptr(), bcnorm.bB.data_ptr(),
                                  bcnorm.bC.data_ptr(), float(bcnorm.eps)))
    Bt, T, H, R, P = x.shape
    N = B.shape[-1]
    dims = make_dims(Bt, T, H, P, N, R, x.dtype, a_per_token=A.dim() == 3, theta_per_head=theta.dim() == 2)
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    if final is None and want_state:
        f = dict(dtype=torch.float32, pin_memory=True)
        final = State(torch.empty(Bt, H, N, P, **f), torch.empty(Bt, H, R, N, **f), torch.empty(Bt, H, R, P, **f))
    # the device: the workspace's, else the stream's, else the current one
    dev = _require_cuda(workspace) or (stream.device if stream is not None else
                                       torch.device("cuda", torch.cuda.current_device()))
    with torch.cuda.device(dev):
        if workspace is None:
            workspace = _scratch(max(scan_host_plan(dims, bcnorm is not None).workspace_bytes, 1), dev, stream)
        ws_bytes = workspace.numel() * workspace.element_size()
        _check(get_lib().m3_scan_fwd_host(ctypes.byref(dims), cb, *map(_ptr, (x, B, C, dt, lam, theta, A, D)),
                                          _hstate(init), _ptr(y), _hstate(final), _ptr(workspace), ws_bytes,
                                          _stream(stream, dev)))
    return y, final


def selftest_wait_timeout(stream=None):
    """Queue a kernel whose bounded device wait gives up; the next
    stream_status() on that stream raises M3Error(M3_ERR_TIMEOUT)."""
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(get_lib().m3_selftest_wait_timeout(_stream(stream, dev)))


def selftest_segment_timeout(x, B, C, dt, lam, theta, A, D, segments: int, init: State | None = None, *,
                             stream=None):
    """The split prefill without its summary pass (m3_selftest_segment_timeout):
    the look-back waits of segments >= 1 give up (about 1 s) and the next
    stream_status() raises M3Error(M3_ERR_TIMEOUT) with code 0x8.  Returns the
    (incomplete) y and final state."""
    dev = _require_cuda(x, B, C, dt, lam, theta, A, D, *(init or ()))
    Bt, T, H, R, P = x.shape
    N = B.shape[-1]
    dims = make_dims(Bt, T, H, P, N, R, x.dtype, a_per_token=A.dim() == 3, theta_per_head=theta.dim() == 2)
    with torch.cuda.device(dev):
        y = torch.empty_like(x)
        final = State(torch.empty(Bt, H, N, P, device=dev), torch.empty(Bt, H, R, N, device=dev),
                      torch.empty(Bt, H, R, P, device=dev))
        need = workspace_size(dims, ALGO_TC_SEGMENTS(segments))
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        _check(get_lib().m3_selftest_segment_timeout(
            ctypes.byref(dims), segments, *map(_ptr, (x, B, C, dt, lam, theta, A, D)), _cstate(init), _ptr(y),
            _cstate(final), _ptr(ws), need, _stream(stream, dev)))
    return y, final


def device_checks() -> bool:
    """True when the loaded library is the bounds build (device index checks)."""
    return bool(get_lib().m3_device_checks())


def stream_status(stream=None):
    """Synchronise the stream and raise if a kernel's bounded wait gave up
    (on any stream of the stream's device since the previous check), or, in
    the bounds build, if a device index check failed (M3_ERR_BOUNDS)."""
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(get_lib().m3_stream_status(_stream(stream, dev)))


def step(x, B, C, dt, lam, theta, A, D, state: State, *, y=None, stream=None, bcnorm: BCNorm | None = None,
         proj: MimoProj | None = None):
    """One decode step in place on `state`.  x [Bt,H,R,P], B/C [Bt,H,R,N],
    dt/lam [Bt,H], theta [Bt,H,N/2] (or [H,N/2]: fixed per head); A [H] fp32,
    or [Bt,H] fp32 for a data-dependent A_t.  Returns y [Bt,H,R,P].  With the
    MIMO projections `proj`: x [Bt,H,P], B/C [Bt,H,N], y [Bt,H,P]."""
    dev = _require_cuda(x, B, C, dt, lam, theta, A, D, y, *state, *(bcnorm[:4] if bcnorm is not None else ()),
                        *(proj or ()))
    if proj is not None:
        Bt, H, P = x.shape
        R = proj.wx.shape[1]
    else:
        Bt, H, R, P = x.shape
    N = B.shape[-1]
    dims = make_dims(Bt, 1, H, P, N, R, x.dtype, a_per_token=A.dim() == 2, theta_per_head=theta.dim() == 2)
    with torch.cuda.device(dev):
        if y is None:
            y = torch.empty_like(x)
        args = (*map(_ptr, (x, B, C, dt, lam, theta, A, D)), _cstate(state), _ptr(y), _stream(stream, dev))
        if proj is not None:
            _check(get_lib().m3_step_proj(ctypes.byref(dims), _cproj(proj), *args))
        elif bcnorm is None:
            _check(get_lib().m3_step(ctypes.byref(dims), *args))
        else:
            _check(get_lib().m3_step_bcnorm(ctypes.byref(dims), _cbcn(bcnorm), *args))
    return y
