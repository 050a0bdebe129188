"""Runtime behaviour on the GPU: the bounded-wait failure path (no fault: a
wait that nothing completes runs out and the host reads the status), and
stream/graph capture of the whole step (multi-step decode by graph replay)."""
import pytest
import torch

from tests import parity
from top_kv_span_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    from top_kv_span_b200 import build
    build.build()
    from top_kv_span_b200 import reatt
    return reatt


def test_bounded_wait_times_out_and_context_survives(R):
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert R.reatt_workspace_status(ws) == R.OK
    R.reatt_selftest_bounded_wait(ws, 20_000_000)        # 20 ms
    torch.cuda.synchronize()
    assert R.reatt_workspace_status(ws) == R.ETIMEOUT
    assert R.reatt_workspace_status(ws) == R.OK          # read clears it
    # the context is still fine: a normal step runs and checks out
    w = wl.WORKLOADS["tiny_f32_4k"]
    x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
    d = R.dims_of(w)
    b = R.alloc_outputs(d)
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                 b["out"], b["ws"])
    torch.cuda.synchronize()
    assert R.reatt_workspace_status(b["ws"]) == R.OK
    assert torch.isfinite(b["out"]).all()


def test_selftest_rejects_bad_arguments(R):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert R.reatt_selftest_bounded_wait(None, 1000, check=False) == R.EINVAL
    assert R.reatt_selftest_bounded_wait(ws, 0, check=False) == R.EINVAL
    assert R.reatt_selftest_bounded_wait(ws, 11 * 10**9, check=False) == R.EINVAL


@pytest.mark.parametrize("name", ["llama3_8b_128k", "llama3_8b_prefill_256k"])
def test_step_captured_in_cuda_graph(R, name):
    """Several layers' steps captured once and replayed: same results as eager
    calls (nothing returns to the host inside a step)."""
    base = wl.WORKLOADS[name]
    w = base.replace(T=20000, n_needles=0) if base.C == 1 else base.replace(T=12000, C=256)
    layers = [w.replace(seed=500 + i) for i in range(3)]
    xs = [{n: t.cuda() for n, t in wl.make_inputs(l).items() if n != "needles"} for l in layers]
    d = R.dims_of(w)
    bufs = [R.alloc_outputs(d) for _ in layers]
    ref = []
    for x, b in zip(xs, bufs):
        R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                     b["out"], b["ws"])
        torch.cuda.synchronize()
        ref.append((b["sel"].clone(), b["out"].clone()))
        b["out"].fill_(float("nan"))
        b["sel"].fill_(-7)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for x, b in zip(xs, bufs):
            R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                         b["out"], b["ws"], stream=s)
    for _ in range(3):
        g.replay()
        torch.cuda.synchronize()
        for (rs, ro), b in zip(ref, bufs):
            assert torch.equal(b["sel"], rs)
            assert float((b["out"] - ro).abs().max()) <= parity.OUT_TOL[w.dtype]
