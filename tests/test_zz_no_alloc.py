"""mta_layer_fwd_static: the MTA layer for callers that cannot allocate device
memory themselves (for example a runtime that is handed device pointers to its
inputs and outputs and has no allocator, or a loop that must not call cudaMalloc
because allocation can synchronise the device).  Its scratch lives in a static
buffer inside the library; these tests call it through the C ABI and compare
it with mta_layer_fwd given an ordinary workspace.

Each output is also compared with the fp64 oracle, so that a mistake shared by
both entry points cannot pass unseen, and the device's free memory is read
around calls to show that the entry point allocates nothing.

Named so that pytest collects it last; it passes alone in a fresh process and
after the other tests (the static buffer keeps whatever the last call left).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from token_attention_b200 import build, mta, synth

pytestmark = pytest.mark.gpu

STATIC_MAX = 16 * 1024 * 1024  # MTA_STATIC_SCRATCH_BYTES in include/mta.h


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    lib = mta.lib()
    P = ctypes.c_void_p
    lib.mta_layer_fwd_static.argtypes = [P, P, P, P, ctypes.POINTER(mta.MtaGn), P,
                                         ctypes.POINTER(mta.MtaCfg), P]
    lib.mta_layer_fwd_static.restype = ctypes.c_int
    return lib


def dev(x, bf16=True):
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t.to(torch.bfloat16) if bf16 else t


def static_call(L, wl, t, out):
    cfg = mta.make_cfg(wl.B, wl.H, wl.L, wl.d, wl.c_q, wl.c_k, wl.c_h, wl.kq_place,
                       wl.head_place, mta.BF16, stream=ctypes.c_void_p(
                           torch.cuda.current_stream().cuda_stream))
    gn = mta.MtaGn(t["gamma"].data_ptr(), t["beta"].data_ptr(), 1e-5, wl.depth, -1.0)
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    return L.mta_layer_fwd_static(p(t["x"]), p(t["wqkv"]), p(t["theta"]), p(t["w"]),
                                  ctypes.byref(gn), p(t["wo"]), ctypes.byref(cfg), p(out))


@pytest.mark.parametrize("name", ["layer_post_D2048_L4096", "layer_pre_D2048_L4096"])
def test_static_scratch_layer_matches_workspace_layer(L, name):
    """Two calls in a row with different inputs: each output matches the
    workspace-based entry point within the bf16 parity tolerance."""
    for call, seed in enumerate((501, 502)):
        wl = synth.shrink(synth.WORKLOADS[name], B=2, L=300, D=256, H=2, d=128, seed=seed)
        assert mta.layer_workspace_bytes(wl.B, wl.L, wl.H, wl.d, wl.c_q, wl.c_k, wl.c_h) <= STATIC_MAX
        inp = synth.make_layer_inputs(wl)
        t = {k: dev(inp[k], k in ("x", "wqkv", "wo")) for k in
             ("x", "wqkv", "wo", "theta", "w", "gamma", "beta")}
        out = torch.full((wl.B, wl.L, wl.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert static_call(L, wl, t, out) == 0
        ref = mta.layer_fwd(t["x"], t["wqkv"], t["theta"], t["w"], t["gamma"], t["beta"], t["wo"],
                            wl.H, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                            layer=wl.depth, check=True)
        torch.cuda.synchronize()
        g, r = out.double().cpu().numpy(), ref.double().cpu().numpy()
        rel = np.linalg.norm(g - r) / np.linalg.norm(r)
        assert rel <= 1e-2 and np.abs(g - r).max() <= 3e-2, (call, rel)
        o = O.mta_layer(inp["x"], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"], inp["beta"],
                        inp["eps"], O.depth_scale(wl.depth), inp["wo"], wl.H, wl.c_h, wl.kq_place,
                        wl.head_place)
        rel_o = np.linalg.norm(g - o) / np.linalg.norm(o)
        assert rel_o <= 1e-2 and np.abs(g - o).max() <= 3e-2, (call, rel_o)


def test_static_scratch_allocates_nothing(L):
    """Once a first call has run (with lazy module loading, the library's static
    buffer becomes resident on the device then), further calls leave the
    device's free memory exactly as it was: nothing is allocated per call."""
    wl = synth.shrink(synth.WORKLOADS["layer_post_D2048_L4096"], B=2, L=300, D=256, H=2, d=128, seed=503)
    inp = synth.make_layer_inputs(wl)
    t = {k: dev(inp[k], k in ("x", "wqkv", "wo")) for k in
         ("x", "wqkv", "wo", "theta", "w", "gamma", "beta")}
    out = torch.empty((wl.B, wl.L, wl.D), dtype=torch.bfloat16, device="cuda")
    assert static_call(L, wl, t, out) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert static_call(L, wl, t, out) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_static_scratch_rejects_sizes_beyond_the_buffer(L):
    """A layer whose scratch exceeds the static buffer is refused before
    anything is enqueued (MTA_ERR_WORKSPACE)."""
    wl = synth.WORKLOADS["layer_post_D2048_L4096"]
    assert mta.layer_workspace_bytes(wl.B, wl.L, wl.H, wl.d, wl.c_q, wl.c_k, wl.c_h) > STATIC_MAX
    fake = {k: torch.empty(16, device="cuda") for k in
            ("x", "wqkv", "wo", "theta", "w", "gamma", "beta")}
    out = torch.empty(16, device="cuda")
    assert static_call(L, wl, fake, out) == 3
