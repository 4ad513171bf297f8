"""Failure detection on the GPU without a fault: a kernel whose bounded wait
cannot complete gives up after a short limit, the library reports
MTA_ERR_TIMEOUT, and the context and the workspace stay usable (the next
normal call on the same workspace returns MTA_OK with the oracle's output)."""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle as O
from token_attention_b200 import build, mta, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    mta.lib()


def test_wait_that_cannot_complete_reports_timeout_then_recovers():
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=1, H=4, L=300, seed=31)
    cfg = mta.make_cfg(wl.B, wl.H, wl.L, wl.d, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                       mta.BF16)
    nbytes = mta.lib().mta_attn_workspace_bytes(ctypes.byref(cfg))
    ws = mta.workspace(nbytes)
    stream = torch.cuda.current_stream()
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    cfg.stream = stream.cuda_stream
    torch.cuda.synchronize()

    limit_ms = 20
    t0 = time.perf_counter()
    assert mta.lib().mta_selftest_wait_timeout(ctypes.byref(cfg), limit_ms * 1000) == 0
    assert mta.lib().mta_sync_status(ctypes.byref(cfg)) == 5          # MTA_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert elapsed >= limit_ms / 1e3 * 0.9
    assert elapsed < 10.0                                             # the wait was bounded
    counters = ws[4:12].view(torch.int32).cpu().numpy()
    # every thread's first wait gave up (one by the limit, the rest by the abort
    # flag), and every second wait returned at once after the abort
    assert counters.tolist() == [128, 128]

    # the same workspace serves a normal call: the status is clear again and the
    # output is the oracle's
    inp = synth.make_attn_inputs(wl)
    dev = lambda x, bf=True: (lambda t: t.to(torch.bfloat16) if bf else t)(
        torch.from_numpy(np.ascontiguousarray(x)).cuda())
    out = mta.attn_fwd(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["theta"], False),
                       dev(inp["w"], False), wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                       ws=ws, check=True)
    assert mta.lib().mta_sync_status(ctypes.byref(cfg)) == 0
    ref = O.mta_attention(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h,
                          wl.kq_place, wl.head_place)
    g = out.double().cpu().numpy()
    rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    assert rel <= 1e-2 and np.abs(g - ref).max() <= 3e-2, rel
