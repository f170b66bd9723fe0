"""GPU tests of the library inside CUDA graphs and under concurrent host
threads: prefill (whole and split sequences, the SIMT kernel, fp32 I/O on
the tensor cores) and decode steps captured once
and replayed give the same bits as eager calls; two host threads driving
m3_scan_fwd_host on their own streams give the same bits as one at a time."""
import threading

import pytest
import torch

from m3_inputs import Shape, make_prefill, make_state, make_steps
from m3_testutil import KEYS

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
else:
    m3 = None


def dev(d):
    return {k: v.cuda() for k, v in d.items()}


@pytest.mark.parametrize("algo_name,segs", [("auto", 0), ("split", 3), ("simt", 0), ("tc32", 0)])
def test_prefill_graph_replay_matches_eager(algo_name, segs):
    s = Shape(2, 700, 4, 64, 128, 1, "bf16", 401)
    if algo_name == "tc32":  # fp32 I/O on the tensor cores (split operands)
        s = Shape(2, 700, 4, 64, 64, 2, "f32", 405)
    algo = {"auto": m3.ALGO_AUTO, "split": m3.ALGO_TC_SEGMENTS(segs), "simt": m3.ALGO_SIMT,
            "tc32": m3.ALGO_TC}[algo_name]
    inp = dev(make_prefill(s))
    init = m3.State(*(t.cuda() for t in make_state(s)))
    dims = m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io)
    plan = m3.scan_plan(dims, algo)
    ws = torch.empty(max(plan.workspace_bytes, 16), dtype=torch.uint8, device="cuda")
    y_ref, f_ref = m3.scan_fwd(*(inp[k] for k in KEYS), init, workspace=ws, algo=algo)
    y = torch.empty_like(y_ref)
    fin = m3.State(*(torch.empty_like(t) for t in f_ref))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on a side stream before capture
        m3.scan_fwd(*(inp[k] for k in KEYS), init, y=y, final=fin, workspace=ws, algo=algo)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m3.scan_fwd(*(inp[k] for k in KEYS), init, y=y, final=fin, workspace=ws, algo=algo)
    for _ in range(2):
        y.zero_()
        fin.h.zero_()
        g.replay()
        torch.cuda.synchronize()
        m3.stream_status()
        assert torch.equal(y, y_ref)
        for a, b in zip(fin, f_ref):
            assert torch.equal(a, b)


@pytest.mark.parametrize("rank", [1, 4])
@pytest.mark.parametrize("batch", [8, 40])  # 32 and 160 slices: rank 4 with and without dependent launch
def test_decode_graph_replay_matches_eager(rank, batch):
    s = Shape(batch, 64, 4, 64, 128, rank, "bf16", 402)
    pre = dev(make_prefill(s))
    nsteps = 4
    steps = make_steps(s, nsteps, device="cuda")
    _, st0 = m3.scan_fwd(*(pre[k] for k in KEYS), None)
    eager = m3.State(*(t.clone() for t in st0))
    ys_ref = [m3.step(*(steps[k][i] for k in KEYS[:6]), pre["A"], pre["D"], eager) for i in range(nsteps)]
    st = m3.State(*(t.clone() for t in st0))
    ys = [torch.empty_like(y) for y in ys_ref]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        m3.step(*(steps[k][0] for k in KEYS[:6]), pre["A"], pre["D"], m3.State(*(t.clone() for t in st0)))
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(nsteps):
            m3.step(*(steps[k][i] for k in KEYS[:6]), pre["A"], pre["D"], st, y=ys[i])
    for a, b in zip(st, st0):  # capture ran nothing
        a.copy_(b)
    g.replay()
    torch.cuda.synchronize()
    m3.stream_status()
    for y, yr in zip(ys, ys_ref):
        assert torch.equal(y, yr)
    for a, b in zip(st, eager):
        assert torch.equal(a, b)


def test_host_scan_from_two_threads():
    shapes = [Shape(3, 600, 2, 64, 128, 1, "bf16", 403), Shape(2, 900, 2, 64, 64, 4, "bf16", 404)]
    inputs = [{k: v.pin_memory() for k, v in make_prefill(s).items()} for s in shapes]
    refs = []
    for inp in inputs:
        y, f = m3.scan_fwd_host(*(inp[k] for k in KEYS))
        torch.cuda.synchronize()
        refs.append((y.clone(), m3.State(*(t.clone() for t in f))))
    results = [None, None]
    errors = []

    def run(i):
        try:
            stream = torch.cuda.Stream()
            outs = []
            for _ in range(3):
                y, f = m3.scan_fwd_host(*(inputs[i][k] for k in KEYS), stream=stream)
                outs.append((y, f))
            stream.synchronize()
            results[i] = outs
        except Exception as e:  # reported below, in the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    m3.stream_status()
    for i in range(2):
        for y, f in results[i]:
            assert torch.equal(y, refs[i][0])
            for a, b in zip(f, refs[i][1]):
                assert torch.equal(a, b)
