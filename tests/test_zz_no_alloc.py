"""The no-allocation step (reatt_step_fixed_scratch) against the ordinary
step.  It serves callers that cannot allocate device memory (a plugin
interface without an allocator, a latency-critical loop where cudaMalloc
would synchronize the device), so its workspace is the library's fixed
16 MiB device array.  This file is collected last on purpose."""
import ctypes

import numpy as np
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


CASES = [
    wl.WORKLOADS["tiny_f32_4k"],
    wl.WORKLOADS["llama3_8b_128k"].replace(name="mid", T=40000, n_needles=2, seed=77),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fixed_scratch_matches_workspace_step(R, w):
    x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
    d = R.dims_of(w)
    b = R.alloc_outputs(d)
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                 b["out"], b["ws"])
    torch.cuda.synchronize()
    for _ in range(2):   # two calls in a row share the fixed array
        sel = torch.full_like(b["sel"], -7)
        out = torch.full_like(b["out"], float("nan"))
        rc = R.lib.reatt_step_fixed_scratch(
            ctypes.byref(d), x["q"].data_ptr(), x["k_cache"].data_ptr(), x["v_cache"].data_ptr(),
            x["k_cur"].data_ptr(), x["v_cur"].data_ptr(), sel.data_ptr(), out.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert rc == R.OK, R.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(sel, b["sel"])
        err = float((out.double() - b["out"].double()).abs().max())
        assert np.isfinite(err) and err <= parity.OUT_TOL[w.dtype]


def test_fixed_scratch_rejects_oversized_work(R):
    w = wl.WORKLOADS["llama3_8b_1m_x4"].replace(T=1 << 30)
    d = R.dims_of(w)
    assert R.reatt_workspace_bytes(d) > (16 << 20)
    fake = 0x10000   # never used: the size check comes first
    rc = R.lib.reatt_step_fixed_scratch(ctypes.byref(d), fake, fake, fake, fake, fake, None, fake,
                                        None)
    assert rc == R.EUNSUPPORTED


def test_fixed_scratch_status_word_reports_a_timeout(R):
    """A bounded-wait timeout in the fixed array is visible to the caller
    through its address, the read clears it, and the next step is normal."""
    torch.cuda.init()
    ws = R.reatt_fixed_scratch_address()
    assert ws % 256 == 0
    assert R.reatt_fixed_scratch_address() == ws
    assert R.reatt_workspace_status(ws) == R.OK
    R.reatt_selftest_bounded_wait(ws, 20_000_000)        # 20 ms
    torch.cuda.synchronize()
    assert R.reatt_workspace_status(ws) == R.ETIMEOUT
    assert R.reatt_workspace_status(ws) == R.OK          # read clears it
    w = CASES[0]
    x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
    d = R.dims_of(w)
    b = R.alloc_outputs(d)
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                 b["out"], b["ws"])
    sel = torch.empty_like(b["sel"])
    out = torch.empty_like(b["out"])
    R.reatt_step_fixed_scratch(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"],
                               sel, out)
    torch.cuda.synchronize()
    assert R.reatt_workspace_status(ws) == R.OK
    assert torch.equal(sel, b["sel"])
