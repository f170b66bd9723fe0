"""Host-side checks of the C ABI: the library loads, exports every entry point
include/m3.h declares, and rejects bad arguments with a status (never a
crash) before touching any device memory.  CPU-only."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "m3.h")


@pytest.fixture(scope="module")
def m3():
    from state_space_sequence_ssm_b200 import build
    build.build()
    import state_space_sequence_ssm_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(m3_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(m3):
    names = declared_functions()
    assert {"m3_scan_fwd", "m3_step", "m3_scan_workspace_size", "m3_last_error"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", m3.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (m3_[a-z0-9_]+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in names:
        getattr(m3.lib, n)  # resolvable through ctypes


def test_only_abi_symbols_exported(m3):
    out = subprocess.run(["nm", "-D", "--defined-only", m3.LIB_PATH], capture_output=True, text=True).stdout
    ours = set(re.findall(r"\bT (m3\w*)", out))
    assert ours == set(declared_functions())


def dims(m3, Bt=2, T=8, H=2, P=8, N=8, R=1, io=0, flags=0):
    return m3.Dims(Bt, T, H, P, N, R, io, flags)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def call_scan(m3, d, ptrs=None, init=None, fin=None, y=None, algo=0):
    p = ptrs or [FAKE + i * 0x100000 for i in range(8)]
    vp = [ctypes.c_void_p(v) if v is not None else None for v in p]
    yv = ctypes.c_void_p(y if y is not None else FAKE + 9 * 0x100000)
    return m3.lib.m3_scan_fwd_algo(algo, ctypes.byref(d) if d is not None else None, *vp, init, yv, fin,
                                   None, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(N=7), 1), (dict(N=0), 1), (dict(H=0), 1), (dict(P=0), 1), (dict(R=0), 1),
    (dict(Bt=-1), 1), (dict(T=-2), 1), (dict(io=5), 1), (dict(flags=4), 1), (dict(flags=-1), 1),
    (dict(N=512), 2), (dict(R=16), 2), (dict(P=6), 2),
])
def test_bad_dims_rejected(m3, kw, status):
    assert call_scan(m3, dims(m3, **kw)) == status
    assert m3.lib.m3_last_error().decode()


def test_null_dims(m3):
    assert call_scan(m3, None) == 1
    n = ctypes.c_size_t(7)
    assert m3.lib.m3_scan_workspace_size(None, ctypes.byref(n)) == 1


def test_missing_tensor_rejected(m3):
    p = [FAKE + i * 0x100000 for i in range(8)]
    p[1] = None
    assert call_scan(m3, dims(m3), ptrs=p) == 1
    assert "required" in m3.lib.m3_last_error().decode()


def test_misaligned_rejected(m3):
    p = [FAKE + i * 0x100000 for i in range(8)]
    p[0] += 4
    assert call_scan(m3, dims(m3), ptrs=p) == 1
    assert "aligned" in m3.lib.m3_last_error().decode()


def test_y_overlapping_input_rejected(m3):
    p = [FAKE + i * 0x100000 for i in range(8)]
    assert call_scan(m3, dims(m3), ptrs=p, y=p[2] + 16) == 1
    assert "overlap" in m3.lib.m3_last_error().decode()


def test_partial_state_overlap_rejected(m3):
    base = 0x4000000
    init = m3.CState(base, base + 0x10000, base + 0x20000)
    fin = m3.CState(base + 0x100, base + 0x30000, base + 0x40000)   # h overlaps init.h partially
    assert call_scan(m3, dims(m3), init=ctypes.pointer(init), fin=ctypes.pointer(fin)) == 1
    assert "overlap" in m3.lib.m3_last_error().decode()


def test_incomplete_state_rejected(m3):
    init = m3.CState(0x4000000, None, 0x4020000)
    assert call_scan(m3, dims(m3), init=ctypes.pointer(init)) == 1


def test_tc_algo_refuses_fp32_io(m3):
    assert call_scan(m3, dims(m3, io=0), algo=2) == 2


def test_unknown_algo(m3):
    assert call_scan(m3, dims(m3), algo=9) == 1


def call_scan_proj(m3, d, proj, algo=0, y=None):
    p = [ctypes.c_void_p(FAKE + i * 0x100000) for i in range(8)]
    yv = ctypes.c_void_p(y if y is not None else FAKE + 9 * 0x100000)
    return m3.lib.m3_scan_fwd_proj(algo, ctypes.byref(d), proj, *p, None, yv, None, None, 0, None)


def test_proj_validation_on_the_host(m3):
    """m3_scan_fwd_proj rejects a missing or incomplete weight set, misaligned
    weights and y overlapping a weight array, and refuses fp32 I/O and the SIMT
    algo, all before any launch (the tensors are fake addresses)."""
    W = FAKE + 20 * 0x100000
    ok = m3.CMimoProj(W, W + 0x10000, W + 0x20000, W + 0x30000)
    d = dims(m3, P=64, N=64, R=2, io=1)
    assert call_scan_proj(m3, d, None) == 1
    assert call_scan_proj(m3, d, ctypes.byref(m3.CMimoProj(W, None, W + 0x20000, W + 0x30000))) == 1
    assert call_scan_proj(m3, d, ctypes.byref(m3.CMimoProj(W + 2, W + 0x10000, W + 0x20000, W + 0x30000))) == 1
    assert call_scan_proj(m3, d, ctypes.byref(ok), y=W + 0x30000) == 1  # y over wy
    assert call_scan_proj(m3, dims(m3, P=64, N=64, R=2, io=0), ctypes.byref(ok)) == 2
    assert call_scan_proj(m3, d, ctypes.byref(ok), algo=1) == 2


def test_step_validation(m3):
    d = dims(m3)
    vp = [ctypes.c_void_p(FAKE + i * 0x100000) for i in range(8)]
    assert m3.lib.m3_step(ctypes.byref(d), *vp, None, ctypes.c_void_p(FAKE + 9 * 0x100000), None) == 1
    st = m3.CState(FAKE + 3 * 0x100000, 0x7000000, 0x7100000)  # h overlaps C
    assert m3.lib.m3_step(ctypes.byref(d), *vp, ctypes.pointer(st), ctypes.c_void_p(0x7200000), None) == 1


def test_workspace_query_is_host_only(m3):
    n = ctypes.c_size_t(123)
    assert m3.lib.m3_scan_workspace_size(ctypes.byref(dims(m3, io=0)), ctypes.byref(n)) == 0
    assert n.value == 0  # fp32 I/O runs the SIMT path, which needs none


def test_version(m3):
    assert m3.lib.m3_version() == 103
    assert m3.lib.m3_device_checks() == 0  # the normal build


def test_scan_plan_info_host_side(m3):
    """m3_scan_plan_info on the host: the kernel that runs is reported (fp32
    I/O: the SIMT kernel, one CTA per slice, no workspace), bad flags and a
    NULL result are refused, an empty batch runs nothing."""
    d = dims(m3, Bt=3, H=5, io=0)
    info = m3.scan_plan_info(d)
    assert info == m3.PlanInfo(0, m3.KERNEL_SIMT, 1, 1, 15)
    assert info.kernel_name == "prefill_simt_kernel"
    assert m3.scan_plan_info(d, flags=m3.PLAN_STATIC).kernel == m3.KERNEL_SIMT
    assert m3.scan_plan_info(dims(m3, Bt=0)) == m3.PlanInfo(0, m3.KERNEL_NONE, 1, 0, 0)
    out = m3.CPlanInfo()
    assert m3.lib.m3_scan_plan_info(0, ctypes.byref(d), 2, ctypes.byref(out)) == 1
    assert "flags" in m3.lib.m3_last_error().decode()
    assert m3.lib.m3_scan_plan_info(0, ctypes.byref(d), 0, None) == 1
    assert m3.lib.m3_scan_plan_info(m3.ALGO_TC, ctypes.byref(d), 0, ctypes.byref(out)) == 2


def test_segment_count_only_with_tc(m3):
    # a segment count belongs to the tensor-core choice only; out-of-range counts are refused
    assert call_scan(m3, dims(m3, io=1), algo=m3.ALGO_SIMT | (3 << 8)) == 1
    assert call_scan(m3, dims(m3, io=1), algo=m3.ALGO_AUTO | (3 << 8)) == 1
    assert call_scan(m3, dims(m3, io=1), algo=m3.ALGO_TC_SEGMENTS(5000)) == 1
    assert "segment" in m3.lib.m3_last_error().decode()


def test_scan_plan_host_side(m3):
    size, segs, launches = ctypes.c_size_t(7), ctypes.c_int(7), ctypes.c_int(7)
    d = dims(m3, io=0)
    assert m3.lib.m3_scan_plan(m3.ALGO_AUTO, ctypes.byref(d), ctypes.byref(size), ctypes.byref(segs),
                               ctypes.byref(launches)) == 0
    assert (size.value, segs.value, launches.value) == (0, 1, 1)  # fp32 I/O: one SIMT launch, no workspace
    z = dims(m3, Bt=0, io=0)
    assert m3.lib.m3_scan_plan(m3.ALGO_SIMT, ctypes.byref(z), None, None, ctypes.byref(launches)) == 0
    assert launches.value == 0
    assert m3.lib.m3_scan_plan(m3.ALGO_TC, ctypes.byref(d), None, None, None) == 2  # TC refuses fp32 I/O
    assert m3.lib.m3_scan_plan(9, ctypes.byref(d), None, None, None) == 1
    assert m3.lib.m3_scan_plan(m3.ALGO_AUTO, None, None, None, None) == 1


@pytest.mark.parametrize("Bt,T,H,P,N,R,io,flags", [
    (8, 4096, 32, 64, 128, 1, 1, 0),   # 8 whole sequences
    (2, 1000, 2, 64, 128, 1, 1, 0),    # 2 sequences x 4 slices of 256
    (12, 300, 1, 64, 64, 1, 1, 1),     # groups of 2 x 2 slices, per-token A
    (1, 2600, 3, 64, 64, 4, 1, 2),     # one sequence in slices of 384, theta per head
    (16, 100, 2, 16, 32, 2, 0, 0),     # T <= 128: one slice, 8 groups of 2
    (3, 0, 2, 8, 8, 1, 0, 0),          # empty sequences
])
def test_host_plan_units_and_staging(m3, Bt, T, H, P, N, R, io, flags):
    """m3_scan_host_plan on the host: slices are multiples of 128 tokens (or
    the whole sequence), the units cover the problem, and the workspace holds
    at least two staging slots and three state sets of one unit's size."""
    d = dims(m3, Bt=Bt, T=T, H=H, P=P, N=N, R=R, io=io, flags=flags)
    ws = ctypes.c_size_t(0)
    ts, tl, gb, u = (ctypes.c_int64(0) for _ in range(4))
    assert m3.lib.m3_scan_host_plan(ctypes.byref(d), 0, ctypes.byref(ws), ctypes.byref(ts), ctypes.byref(tl),
                                    ctypes.byref(gb), ctypes.byref(u)) == 0
    ts, tl, gb, u = ts.value, tl.value, gb.value, u.value
    for s in (ts, tl):
        assert s == T if T <= 128 else (s % 128 == 0 and s <= T + 127)
    nslice = 1 if T <= 128 else -(-T // ts)
    nlast = 1 if T <= 128 else -(-T // tl)
    groups = -(-Bt // gb)
    assert u == nslice * (groups - 1) + nlast
    # the documented rule: up to 8 groups of whole sequences, then time slices toward 8 units;
    # the last group in at least 4 slices where the sequence has 4 chunks of 128 tokens
    assert gb == -(-Bt // min(Bt, 8))
    want = -(-8 // groups)
    if T > 128:
        assert ts == -(-(-(-T // min(-(-T // 128), want))) // 128) * 128
        assert tl == -(-(-(-T // min(-(-T // 128), max(nslice, 4)))) // 128) * 128
        assert tl <= ts
    es = 2 if io == 1 else 4
    per_tok = H * (2 * R * P * es + 2 * R * N * es + 2 * es + (0 if flags & 2 else N // 2 * es)
                   + (4 if flags & 1 else 0))
    staging = 2 * gb * ts * per_tok + 3 * gb * H * (N * P + R * N + R * P) * 4
    assert ws.value >= staging


def test_host_plan_empty_batch_and_bad_dims(m3):
    ws = ctypes.c_size_t(7)
    d = dims(m3, Bt=0, T=500)
    assert m3.lib.m3_scan_host_plan(ctypes.byref(d), 0, ctypes.byref(ws), None, None, None, None) == 0
    assert ws.value == 0
    bad = dims(m3, N=7)
    assert m3.lib.m3_scan_host_plan(ctypes.byref(bad), 0, None, None, None, None, None) == 1
    # the BC-norm parameters take room in the staging area
    d = dims(m3, Bt=2, T=300, H=2, P=8, N=8, R=2)
    w0, w1 = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert m3.lib.m3_scan_host_plan(ctypes.byref(d), 0, ctypes.byref(w0), None, None, None, None) == 0
    assert m3.lib.m3_scan_host_plan(ctypes.byref(d), 1, ctypes.byref(w1), None, None, None, None) == 0
    assert w1.value >= w0.value + 2 * 8 * 4 + 2 * 2 * 2 * 8 * 4
    # the host entry point validates before touching the device
    assert m3.lib.m3_scan_fwd_host(None, None, *([None] * 8), None, None, None, None, 0, None) == 1


def test_library_has_no_unresolved_internal_symbols(m3):
    """Every internal (namespace m3) function the library calls is defined in
    it: a missing definition would only surface when the GPU loads it."""
    out = subprocess.run(["nm", "-D", "--undefined-only", m3.LIB_PATH], capture_output=True, text=True).stdout
    missing = [l.split()[-1] for l in out.splitlines() if "_ZN2m3" in l]
    assert not missing, f"undefined library-internal symbols: {missing}"
    ctypes.CDLL(m3.LIB_PATH, mode=os.RTLD_NOW)  # resolves every symbol now


def _undefined_names(path):
    """Names a function of `path` loads but that are bound nowhere: not in the
    function (or an enclosing one), not at module level, not a builtin."""
    import ast
    import builtins
    tree = ast.parse(open(path).read())
    module_names = set(dir(builtins))
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef, ast.ClassDef)):
            module_names.add(node.name)
        elif isinstance(node, (ast.Import, ast.ImportFrom)):
            module_names.update((a.asname or a.name).split(".")[0] for a in node.names)
    for node in tree.body:
        for t in ast.walk(node) if isinstance(node, (ast.Assign, ast.AnnAssign)) else []:
            if isinstance(t, ast.Name):
                module_names.add(t.id)
    missing = set()

    def visit(fn, bound):
        local = set(bound)
        for n in ast.walk(fn):
            if isinstance(n, ast.Name) and isinstance(n.ctx, (ast.Store, ast.Del)):
                local.add(n.id)
            elif isinstance(n, ast.arg):
                local.add(n.arg)
            elif isinstance(n, (ast.FunctionDef, ast.Lambda)) and n is not fn and isinstance(n, ast.FunctionDef):
                local.add(n.name)
            elif isinstance(n, (ast.Import, ast.ImportFrom)):
                local.update((a.asname or a.name).split(".")[0] for a in n.names)
            elif isinstance(n, ast.ExceptHandler) and n.name:
                local.add(n.name)
        for n in ast.walk(fn):
            if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load) and n.id not in local | module_names:
                missing.add(n.id)

    for node in tree.body:
        if isinstance(node, ast.FunctionDef):
            visit(node, set())
    return missing


def test_bench_has_no_undefined_names():
    """bench.py's GPU legs cannot run here; at least every name they load is bound."""
    assert _undefined_names(os.path.join(ROOT, "bench.py")) == set()


def test_bench_clock_summary():
    """The bench's clock record: median SM clock of the loaded samples, the
    throttle reasons any sample showed, and no reasons when none was active."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    row = "0, GPU-x, {sm}, 1965, {pw}, 0x0, Not Active, Not Active, Not Active, {cap}"
    text = "\n".join([row.format(sm=1965, pw=600, cap="Not Active"), row.format(sm=1950, pw=900, cap="Active"),
                      row.format(sm=1965, pw=950, cap="Not Active"), row.format(sm=210, pw=80, cap="Not Active")])
    s = bench.ClockSampler.summarise(text)
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["samples"] == 4
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 950
    quiet = bench.ClockSampler.summarise(row.format(sm=1965, pw=500, cap="Not Active"))
    assert quiet["reasons"] == []
    assert bench.ClockSampler.summarise("") is None


class _FakeCudaTensor:
    """Stand-in for a CUDA tensor (no GPU here): only what the binding's
    device check reads."""

    def __init__(self, index, contiguous=True):
        import torch
        self.device = torch.device("cuda", index)
        self.is_cuda = True
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous


def test_binding_refuses_tensors_on_two_gpus(m3):
    """Tensors of one call on different GPUs are refused before any pointer
    reaches the library; the common device is returned otherwise."""
    a, b = _FakeCudaTensor(0), _FakeCudaTensor(1)
    assert m3._require_cuda(a, None, _FakeCudaTensor(0)) == a.device
    with pytest.raises(ValueError, match="different devices"):
        m3._require_cuda(a, b)
    with pytest.raises(ValueError, match="contiguous"):
        m3._require_cuda(_FakeCudaTensor(0, contiguous=False))
    with pytest.raises(ValueError, match="different devices"):
        m3.scan_fwd(a, a, a, a, a, a, a, b)
    with pytest.raises(ValueError, match="different devices"):
        m3.step(a, a, a, a, a, a, a, a, m3.State(a, a, b))


def test_binding_refuses_a_stream_of_another_gpu(m3):
    import torch

    class _S:
        device = torch.device("cuda", 1)
        cuda_stream = 0

    with pytest.raises(ValueError, match="stream is on"):
        m3._stream(_S(), torch.device("cuda", 0))
