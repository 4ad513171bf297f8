"""GPU parity of the tensor-core attention backward (attn_bwd_tc.cu, path 3)
against the fp64 oracle's backward, through the C ABI.

Every gradient (q, k, v, theta, w) at the CUDA-core backward's fp32 tolerance
(relative L2 error 1e-4): the tensor-core path (d = 64, 96 or 128) takes the bf16 inputs themselves as
MMA operands and splits its computed operands (dS, A'') into two bf16 halves, so
its products carry about 16 significant bits and its sums fp32 accumulation.
Lengths span one query block (L <= 374 own rows, 369 with the convolution after the
softmax: blocks of 384 rows up to L = 3072), several blocks and a ragged tail; the pretraining recipe and the
convolution on both sides of the softmax run at their full length for one head
group.
"""
import numpy as np
import pytest
import torch

import oracle as O
from token_attention_b200 import build, mta, synth

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
GRAD_NAMES = ("dq", "dk", "dv", "dtheta", "dw", "dtheta_post")


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
    return float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)), float(np.abs(diff).max())


def run_bwd(wl, inp, dout, path):
    q, k, v = (dev(inp[n], wl.dtype) for n in ("q", "k", "v"))
    tp = None if inp.get("theta_post") is None else dev(inp["theta_post"], "f32")
    g = mta.attn_bwd(q, k, v, dev(inp["theta"], "f32"), dev(inp["w"], "f32"), dev(dout, wl.dtype),
                     wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, check=True, path=path, theta_post=tp)
    torch.cuda.synchronize()
    return g


def check(wl, inp, dout, path=mta.PATH_KQ):
    got = run_bwd(wl, inp, dout, path)
    ref = O.mta_attention_bwd(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h, dout,
                              wl.kq_place, wl.head_place, theta_post=inp.get("theta_post"))
    out = {}
    for n in GRAD_NAMES:
        if ref[n] is None:
            continue
        rel, mx = errs(got[n], ref[n])
        out[n] = rel
        assert rel <= TOL_F32, (n, rel, mx)
    return got, out


CASES = [(128, synth.POST, 9), (128, synth.POST, 375), (128, synth.PRE, 300), (128, synth.OFF, 70),
         (64, synth.POST, 800), (64, synth.PRE, 250), (64, synth.OFF, 119), (128, synth.POST, 374),
         (96, synth.POST, 500), (96, synth.PRE, 130), (128, synth.PRE, 760)]


@pytest.mark.parametrize("d,hp,L", CASES)
def test_bwd_tc_small(d, hp, L):
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=2, H=4, L=L, d=d, head_place=hp,
                      seed=901 + L + d + 3 * hp)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check(wl, inp, dout)


POST_CASES = [(128, synth.POST, 9), (128, synth.POST, 370), (128, synth.PRE, 250), (128, synth.OFF, 369),
              (64, synth.POST, 500), (96, synth.POST, 130), (128, synth.POST, 760)]


@pytest.mark.parametrize("d,hp,L", POST_CASES)
def test_bwd_tc_post_conv_small(d, hp, L):
    """The convolution on both sides of the softmax (the pages' default): every
    gradient, the post-softmax kernels' included, from one query block of 369 own
    rows to three."""
    wl = synth.shrink(synth.WORKLOADS["both_d128_L2048"], B=2, H=4, L=L, d=d, head_place=hp,
                      seed=931 + L + d + 3 * hp)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check(wl, inp, dout)


def test_bwd_tc_post_conv_full_length_one_group():
    """The convolution on both sides at L = 2048 (6 query blocks of 369 own rows), one head
    group."""
    wl = synth.shrink(synth.WORKLOADS["both_d128_L2048"], B=1, H=2, seed=955)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check(wl, inp, dout)


def test_bwd_tc_matches_cuda_core_path():
    """Both backward paths on the same inputs (L = 512: two query blocks, the second ragged)."""
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=1, H=4, L=512, seed=951)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    tc, _ = check(wl, inp, dout, mta.PATH_KQ)
    simt = run_bwd(wl, inp, dout, mta.PATH_SIMT)
    for n in GRAD_NAMES:
        if tc[n] is None:
            continue
        a, b = tc[n].double(), simt[n].double()
        assert float((a - b).norm() / b.norm()) <= 2 * TOL_F32, n


def test_bwd_tc_full_length_one_group():
    """The pretraining recipe at its full length L = 2048 (6 query blocks), one batch
    and one head group, against the oracle's full L x L backward of that group."""
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=1, H=2, seed=952)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check(wl, inp, dout)


def test_bwd_tc_taller_blocks_one_group():
    """Past L = 3072 the blocks are 512 rows tall (502 own rows): L = 3100, six full
    blocks and an 88-row tail, one head group, against the oracle's full backward."""
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=1, H=2, L=3100, seed=956)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check(wl, inp, dout)


def test_bwd_tc_d96_full_length_one_group():
    """The pages' 880M shape (d = 96: 1536 over 16 heads) at L = 2048, one head group:
    the operands' 96 channels are read as two 64-channel TMA boxes, the second half
    past d zero-filled."""
    wl = synth.shrink(synth.WORKLOADS["pretrain_d96_L2048"], B=1, H=2, seed=954)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check(wl, inp, dout)


def test_bwd_auto_takes_tensor_cores():
    """Path 0 with the workspace mta_attn_bwd_workspace_bytes asks for runs the
    tensor-core backward: its results equal path 3's bit for bit."""
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=1, H=2, L=200, seed=953)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    a = run_bwd(wl, inp, dout, mta.PATH_AUTO)
    b = run_bwd(wl, inp, dout, mta.PATH_KQ)
    # dq is at most two partial sums added into zeros (order-free): bit-exact; the
    # summed gradients agree to rounding
    assert torch.equal(a["dq"], b["dq"])
    for n in ("dk", "dv"):
        assert float((a[n] - b[n]).norm() / b[n].norm()) <= 1e-6
