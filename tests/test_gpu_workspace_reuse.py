"""One workspace shared by calls of different geometries (decode steps of two
cache lengths and a prefill chunk, interleaved): every call must give exactly
what the same call gives on a workspace of its own (nothing a call leaves in
the workspace may leak into the next)."""
import pytest
import torch

from top_kv_span_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LLAMA = wl.WORKLOADS["llama3_8b_128k"]


@pytest.fixture(scope="module")
def R():
    from top_kv_span_b200 import build
    build.build()
    from top_kv_span_b200 import reatt
    return reatt


def _step(R, d, x, b):
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                 b["out"], b["ws"])
    torch.cuda.synchronize()
    return b["sel"].clone(), b["out"].clone()


def test_geometry_change_on_one_workspace(R):
    """Alternating geometries (and a prefill chunk) on one workspace: each call
    matches a call of the same geometry on a fresh workspace."""
    wa = LLAMA.replace(name="ga", Hq=8, Hkv=2, n_needles=2, seed=41)
    wb = LLAMA.replace(name="gb", Hq=8, Hkv=2, T=100000, n_needles=2, seed=42)
    wc = LLAMA.replace(name="gc", Hq=8, Hkv=2, C=16, n_needles=0, seed=43)
    ws_bytes = max(R.reatt_workspace_bytes(R.dims_of(w)) for w in (wa, wb, wc))
    shared = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    cases = {}
    for w in (wa, wb, wc):
        x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
        d = R.dims_of(w)
        b = R.alloc_outputs(d)
        cases[w.name] = (d, x, _step(R, d, x, b))
    for name in ["ga", "ga", "gb", "ga", "gc", "ga", "ga", "gb", "gb"]:
        d, x, expect = cases[name]
        b = R.alloc_outputs(d)
        b["ws"] = shared
        got = _step(R, d, x, b)
        assert torch.equal(got[0], expect[0]), name
        assert torch.equal(got[1], expect[1]), name
