"""GPU parity of the layer's backward pass (mta_layer_bwd) and of its building
blocks (the GEMM in all operand layouts, the group norm's backward) against the
oracle, through the C ABI.

Tolerances.  The GEMMs and the group norm's backward take exact bf16 inputs and
accumulate in fp32: bf16 outputs are held to the forward's bf16 bound, fp32
outputs to a relative L2 error of 1e-4.

The layer is checked twice.  Step by step: the call leaves every intermediate in
its workspace (QKV, O, Y, dY, dO, dq/dk/dv, dQKV), and each step is compared
with the oracle's step applied to the GPU's own inputs of that step, at the
step's own tolerance (bf16 outputs: the bf16 bound; fp32 outputs of the GEMMs
and of the attention backward: 1e-4).  End to end: the gradients pass through
five bf16 roundings that the oracle does not make (QKV and O of the recomputed
forward, Y, dO, dQKV); each perturbs its tensor by at most 2^-9 relative and the
errors of the chain add, so the end-to-end gradients are held to a relative L2
error of 2e-2 (about 10 units of 2^-9) and a max-abs error of 5e-2 of the
largest reference magnitude.  One exception: with post-softmax mixing, dw[h][s]
sums dO_h . Z_{s->h} over tokens, and sum_s w[h][s] dw[h][s] = sum dO_h . O_h is
zero up to the norm's eps (the norm's gradient is orthogonal to its input), so
the entries are small differences of terms some 10^4 times larger: the bf16
roundings of the chain move them by far more than 2e-2 relative.  That dw is
compared step by step only (and end to end with pre-softmax mixing, which has
no such cancellation); step by step its tolerance is 1e-3, ten times the fp32
bound, because the same cancellation amplifies the fp32 rounding of the terms
(2^-24 times a factor of about 10^4).
"""
import numpy as np
import pytest
import torch

import oracle as O
from token_attention_b200 import build, mta, synth

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = (1e-2, 3e-2)
TOL_GRAD = (2e-2, 5e-2)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    mta.lib()


def dev(x, dtype="bf16"):
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def errs(gpu, ref):
    g = gpu.detach().double().cpu().numpy().reshape(ref.shape)
    diff = g - ref
    return (float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)),
            float(np.abs(diff).max()), float(np.abs(ref).max()))


# ---------------------------------------------------------------------------
# the GEMM in every operand layout the layer uses
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("a_mn,b_mn,f32", [(0, 0, 0), (0, 0, 1), (0, 1, 1), (1, 1, 1), (0, 1, 0), (1, 0, 1)])
@pytest.mark.parametrize("M,N,K", [(304, 520, 264), (96, 264, 136), (512, 256, 1000), (8, 8, 8)])
def test_gemm_layouts(a_mn, b_mn, f32, M, N, K):
    a = synth.round_bf16(synth.normal(5, 1, (M, K)))
    b = synth.round_bf16(synth.normal(5, 2, (N, K), std=0.05))
    a_in = a.T.copy() if a_mn else a
    b_in = b.T.copy() if b_mn else b
    c = mta.gemm_bf16(dev(a_in), dev(b_in), M, N, K, bool(a_mn), bool(b_mn), bool(f32))
    torch.cuda.synchronize()
    ref = a.astype(np.float64) @ b.astype(np.float64).T
    rel, mx, _ = errs(c, ref)
    if f32:
        assert rel <= TOL_F32, (rel, mx)
    else:
        assert rel <= TOL_BF16[0] and mx <= TOL_BF16[1], (rel, mx)


def test_gemm_layout_checks():
    a = torch.zeros((16, 12), dtype=torch.bfloat16, device="cuda")   # [K][M], M = 12
    b = torch.zeros((16, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mta.MtaError):   # a transposed A needs M % 8 == 0
        mta.gemm_bf16(a, b, 12, 16, 16, a_mn=True)


# ---------------------------------------------------------------------------
# group norm backward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [128, 96, 64, 32])
@pytest.mark.parametrize("gated", [False, True])
def test_group_norm_bwd(d, gated):
    T, H = 515, 6
    o = synth.round_bf16(synth.normal(6, 1, (T, H, d), mean=0.3, std=2.0))
    dy = synth.normal(6, 2, (T, H, d)).astype(np.float32)
    gamma = synth.normal(6, 3, (H * d,), mean=1.0, std=0.1)
    beta = synth.normal(6, 4, (H * d,), std=0.1)
    gate = synth.normal(6, 5, (H,)) if gated else None
    lam = O.depth_scale(12)
    y, do, dgamma, dbeta, dgate = mta.group_norm_scale_bwd(
        dev(o), dev(dy, "f32"), dev(gamma, "f32"), dev(beta, "f32"), 1e-5, lam,
        gate=dev(gate, "f32") if gated else None)
    torch.cuda.synchronize()
    mult = O.sigmoid_gate(gate) if gated else lam
    r_do, r_dg, r_db, r_dgate = O.group_norm_scale_bwd(o, gamma, beta, 1e-5, lam, dy, gate)
    for got, ref in ((y, O.group_norm_scale(o, gamma, beta, 1e-5, mult)), (do, r_do)):
        rel, mx, _ = errs(got, ref)
        assert rel <= TOL_BF16[0] and mx <= TOL_BF16[1], (rel, mx)
    for got, ref in ((dgamma, r_dg), (dbeta, r_db)) + (((dgate, r_dgate),) if gated else ()):
        rel, mx, _ = errs(got, ref)
        assert rel <= TOL_F32, (rel, mx)


def test_group_norm_bwd_full_size():
    """The layer workload's shape (8192 tokens x 16 heads x 128), every element."""
    T, H, d = 8192, 16, 128
    o = synth.round_bf16(synth.normal(7, 1, (T, H, d), std=1.5))
    dy = synth.normal(7, 2, (T, H, d)).astype(np.float32)
    gamma = synth.normal(7, 3, (H * d,), mean=1.0, std=0.1)
    beta = synth.normal(7, 4, (H * d,), std=0.1)
    lam = O.depth_scale(12)
    y, do, dgamma, dbeta, _ = mta.group_norm_scale_bwd(dev(o), dev(dy, "f32"), dev(gamma, "f32"),
                                                       dev(beta, "f32"), 1e-5, lam)
    torch.cuda.synchronize()
    r_do, r_dg, r_db, _ = O.group_norm_scale_bwd(o, gamma, beta, 1e-5, lam, dy)
    rel, mx, _ = errs(do, r_do)
    assert rel <= TOL_BF16[0] and mx <= TOL_BF16[1], (rel, mx)
    for got, ref in ((dgamma, r_dg), (dbeta, r_db)):
        rel, mx, _ = errs(got, ref)
        assert rel <= TOL_F32, (rel, mx)


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------

def up(x):
    return -(-x // 256) * 256


def workspace_views(ws, T, D):
    """The layer backward's intermediates, as laid out in its workspace."""
    off, out = 256, {}
    for name, n, dt, shape in (("qkv", T * 3 * D, torch.bfloat16, (T, 3 * D)), ("o", T * D, torch.bfloat16, (T, D)),
                               ("y", T * D, torch.bfloat16, (T, D)), ("dy", T * D, torch.float32, (T, D)),
                               ("do", T * D, torch.bfloat16, (T, D)), ("dq", T * D, torch.float32, (T, D)),
                               ("dk", T * D, torch.float32, (T, D)), ("dv", T * D, torch.float32, (T, D)),
                               ("dqkv", T * 3 * D, torch.bfloat16, (T, 3 * D))):
        nb = n * (2 if dt == torch.bfloat16 else 4)
        out[name] = ws[off:off + nb].view(dt).reshape(shape)
        off += up(nb)
    return out


def run_layer_bwd(wl, inp, dout, path=mta.PATH_AUTO, gate=None, ws=None):
    tp = None if inp.get("theta_post") is None else dev(inp["theta_post"], "f32")
    g = mta.layer_bwd(dev(inp["x"]), dev(inp["wqkv"]), dev(inp["theta"], "f32"), dev(inp["w"], "f32"),
                      dev(inp["gamma"], "f32"), dev(inp["beta"], "f32"), dev(inp["wo"]), dev(dout),
                      wl.H, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, eps=inp["eps"],
                      layer=wl.depth, path=path, check=True, theta_post=tp,
                      gate=None if gate is None else dev(gate, "f32"), ws=ws)
    torch.cuda.synchronize()
    return g


def oracle_layer_bwd(wl, inp, dout, gate=None):
    return O.mta_layer_bwd(inp["x"], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"], inp["beta"],
                           inp["eps"], O.depth_scale(wl.depth), inp["wo"], wl.H, wl.c_h, dout,
                           wl.kq_place, wl.head_place, theta_post=inp.get("theta_post"), gate=gate)


def compare_grads(g, ref, skip=()):
    report = {}
    for name in ("dx", "dwqkv", "dwo", "dgamma", "dbeta", "dtheta", "dw", "dtheta_post", "dgate"):
        if ref.get(name) is None or name in skip:
            continue
        rel, mx, scale = errs(g[name], ref[name])
        report[name] = (rel, mx / scale)
        assert rel <= TOL_GRAD[0] and mx <= TOL_GRAD[1] * scale, (name, rel, mx, scale)
    return report


CASES = [("layer_post_D2048_L4096", dict(B=2, L=150), None, False),
         ("layer_pre_D2048_L4096", dict(B=2, L=150), None, False),
         ("layer_post_D2048_L4096", dict(B=1, L=520), None, False),
         ("layer_post_D2048_L4096", dict(B=2, L=150), "gate", False),
         ("layer_post_D2048_L4096", dict(B=2, L=150), None, True)]


@pytest.mark.parametrize("name,shape,gated,kq_post", CASES)
@pytest.mark.parametrize("path", [mta.PATH_AUTO, mta.PATH_SIMT])
def test_layer_bwd_small(name, shape, gated, kq_post, path):
    wl = synth.shrink(synth.WORKLOADS[name], D=256, H=2, d=128, seed=321, kq_post=kq_post, **shape)
    inp = synth.make_layer_inputs(wl)
    gate = synth.normal(wl.seed, 77, (wl.H,)) if gated else None
    dout = synth.round_bf16(synth.normal(wl.seed, 78, (wl.B, wl.L, wl.D)))
    B, L, H, d, D = wl.B, wl.L, wl.H, wl.d, wl.D
    T = B * L
    tp = inp.get("theta_post")
    nb = mta.layer_bwd_workspace_bytes(B, L, H, d, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                                       kq_post=int(tp is not None))
    ws = mta.workspace(nb, "cuda")
    g = run_layer_bwd(wl, inp, dout, path, gate, ws)
    # end to end against the oracle
    compare_grads(g, oracle_layer_bwd(wl, inp, dout, gate), skip=("dw",) if wl.head_place == mta.POST else ())
    # step by step, each step on the GPU's own inputs to it
    V = {k: v.double().cpu().numpy() for k, v in workspace_views(ws, T, D).items()}
    def f32(got, ref):
        rel = errs(torch.from_numpy(np.asarray(got)), ref)[0]
        assert rel <= TOL_F32, rel
        return True

    def bf16_ok(got, ref):
        # a bf16 output: relative L2 and, element-wise, the bf16 rounding of the
        # largest magnitude (dO reaches |1/sigma| times dY, far above 1)
        rel, mx, scale = errs(torch.from_numpy(np.asarray(got)), ref)
        assert rel <= TOL_BF16[0] and mx <= TOL_BF16[0] * scale, (rel, mx, scale)
        return True
    x64, wqkv64, wo64 = (inp[n].astype(np.float64) for n in ("x", "wqkv", "wo"))
    assert bf16_ok(V["qkv"], x64.reshape(T, D) @ wqkv64.T)
    q, k, v = (V["qkv"][:, i * D:(i + 1) * D].reshape(B, L, H, d) for i in range(3))
    o_ref = O.mta_attention(q, k, v, inp["theta"], inp["w"], wl.c_h, wl.kq_place, wl.head_place, theta_post=tp)
    assert bf16_ok(V["o"], o_ref.reshape(T, D))
    assert f32(V["dy"], dout.reshape(T, D).astype(np.float64) @ wo64)
    lam = O.depth_scale(wl.depth)
    mult = O.sigmoid_gate(gate) if gated else lam
    o3 = V["o"].reshape(T, H, d)
    assert bf16_ok(V["y"], O.group_norm_scale(o3, inp["gamma"], inp["beta"], inp["eps"], mult).reshape(T, D))
    do_ref, dg_ref, db_ref, dgate_ref = O.group_norm_scale_bwd(o3, inp["gamma"], inp["beta"], inp["eps"], lam,
                                                               V["dy"].reshape(T, H, d), gate)
    assert bf16_ok(V["do"], do_ref.reshape(T, D))
    assert f32(g["dgamma"].cpu(), dg_ref) and f32(g["dbeta"].cpu(), db_ref)
    if gated:
        assert f32(g["dgate"].cpu(), dgate_ref)
    assert f32(g["dwo"].cpu(), dout.reshape(T, D).astype(np.float64).T @ V["y"])
    ga = O.mta_attention_bwd(q, k, v, inp["theta"], inp["w"], wl.c_h, V["do"].reshape(B, L, H, d), wl.kq_place,
                             wl.head_place, theta_post=tp)
    for n in ("dq", "dk", "dv"):
        assert f32(V[n], ga[n].reshape(T, D)), n
    for n in ("dtheta", "dw", "dtheta_post"):
        if ga[n] is not None:
            rel = errs(g[n], ga[n])[0]
            assert rel <= TOL_F32 * (10 if n == "dw" else 1), (n, rel)
    packed = np.concatenate([V["dq"], V["dk"], V["dv"]], axis=1)
    assert (torch.from_numpy(packed).float().to(torch.bfloat16).double().numpy() == V["dqkv"]).all()
    assert f32(g["dx"].cpu().reshape(T, D), V["dqkv"] @ wqkv64)
    assert f32(g["dwqkv"].cpu(), V["dqkv"].T @ x64.reshape(T, D))


@pytest.mark.parametrize("name", ["layer_pre_D2048_L4096", "layer_post_D2048_L4096"])
def test_layer_bwd_full_size_sparse_dout(name):
    """The layer workload at full size (B=2, L=4096, D=2048, H=16) with dout
    nonzero at a few tokens S of batch 0 only.  Then the oracle computes exactly,
    from the forward at those tokens alone: dWo = sum over S of dout^T Y, dgamma
    and dbeta (sums over S).  By causality (Mask_0 before the convolution, taps
    on past queries only) no token after max S, and no token of batch 1, gets a
    gradient: those rows of dx are exactly zero."""
    wl = synth.WORKLOADS[name]
    inp = synth.make_layer_inputs(wl)
    S = [5, 700, 2047, 3000]
    dout = np.zeros((wl.B, wl.L, wl.D), dtype=np.float32)
    dout[0, S] = synth.round_bf16(synth.normal(wl.seed, 79, (len(S), wl.D)))
    g = run_layer_bwd(wl, inp, dout)
    for name_ in ("dx", "dwqkv", "dwo", "dgamma", "dbeta"):
        assert torch.isfinite(g[name_]).all(), name_
    dx = g["dx"].cpu()
    assert (dx[0, max(S) + 1:] == 0).all() and (dx[1] == 0).all()
    assert (dx[0, S] != 0).any(dim=-1).all()
    # the forward at the tokens S: attention output o (fp64), Y
    H, d = wl.H, wl.d
    x64 = inp["x"][0].astype(np.float64)
    qkv = x64 @ inp["wqkv"].astype(np.float64).T
    q, k, v = (qkv[:, i * wl.D:(i + 1) * wl.D].reshape(1, wl.L, H, d) for i in range(3))
    o = O.mta_attention_rows(q, k, v, inp["theta"], inp["w"], wl.c_h, [(0, i) for i in S], wl.kq_place,
                             wl.head_place)
    o = np.asarray(o).reshape(len(S), H, d)
    lam = O.depth_scale(wl.depth)
    y = O.group_norm_scale(o, inp["gamma"], inp["beta"], inp["eps"], lam).reshape(len(S), wl.D)
    dS = dout[0, S].astype(np.float64)
    ref_dwo = dS.T @ y
    dy = (dS @ inp["wo"].astype(np.float64)).reshape(len(S), H, d)
    _, ref_dg, ref_db, _ = O.group_norm_scale_bwd(o, inp["gamma"], inp["beta"], inp["eps"], lam, dy)
    for got, ref in ((g["dwo"], ref_dwo), (g["dgamma"], ref_dg), (g["dbeta"], ref_db)):
        rel, mx, scale = errs(got, ref)
        assert rel <= TOL_GRAD[0] and mx <= TOL_GRAD[1] * scale, (rel, mx, scale)
