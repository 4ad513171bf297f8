"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Tolerances (stated for the MTA forward): bf16 outputs within a relative L2
error of 1e-2 and a max-abs error of 3e-2 of the oracle; fp32 outputs within a
relative L2 error of 1e-4.  Small cases compare every element and span several
tiles plus a ragged tail; full-size workloads, in the launch configuration the
bench times, compare sampled tokens the oracle computes one by one.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from token_attention_b200 import build, mta, synth

pytestmark = pytest.mark.gpu

TOL_BF16 = (1e-2, 3e-2)
TOL_F32 = 1e-4


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


def assert_close(gpu, ref, dtype):
    rel, mx = errs(gpu, ref)
    if dtype == "bf16":
        assert rel <= TOL_BF16[0] and mx <= TOL_BF16[1], (rel, mx)
    else:
        assert rel <= TOL_F32, (rel, mx)
    return rel, mx


def run_attn(wl, inp, path=mta.PATH_AUTO, **kw):
    q, k, v = (dev(inp[n], wl.dtype) for n in ("q", "k", "v"))
    th, w = dev(inp["theta"], "f32"), dev(inp["w"], "f32")
    tp = None if inp.get("theta_post") is None else dev(inp["theta_post"], "f32")
    out = mta.attn_fwd(q, k, v, th, w, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                       path=path, check=True, theta_post=tp, **kw)
    torch.cuda.synchronize()
    return out


def oracle_full(wl, inp):
    return O.mta_attention(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h,
                           wl.kq_place, wl.head_place, theta_post=inp.get("theta_post"))


# ---------------------------------------------------------------------------
# small cases: every element
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", [mta.PATH_AUTO, mta.PATH_SIMT])
def test_tiny_f32_L256(path):
    wl = synth.WORKLOADS["tiny_f32_L256"]
    inp = synth.make_attn_inputs(wl)
    assert_close(run_attn(wl, inp, path), oracle_full(wl, inp), "f32")


SMALL = []
for d in (64, 96, 128):
    for hp in (synth.OFF, synth.PRE, synth.POST):
        for L in (1, 9, 300):
            SMALL.append((d, hp, L))


def tc_applies(wl):
    """Whether the direct tensor-core kernel serves this configuration."""
    return (wl.dtype == "bf16" and wl.d in (64, 128)
            and (wl.kq_place == synth.OFF or (wl.c_q, wl.c_k) == (6, 11))
            and (wl.head_place == synth.OFF or wl.c_h == 2))


def kq_applies(wl):
    """Whether the contraction kernel serves this configuration."""
    return (wl.dtype == "bf16" and wl.d in (64, 96, 128) and wl.kq_place in (synth.PRE, 3)
            and (wl.c_q, wl.c_k) == (6, 11)
            and (wl.head_place == synth.OFF or wl.c_h == 2))


@pytest.mark.parametrize("d,hp,L", SMALL)
@pytest.mark.parametrize("path", [mta.PATH_AUTO, mta.PATH_SIMT, mta.PATH_TC, mta.PATH_KQ])
def test_small_bf16(d, hp, L, path):
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=2, H=4, L=L, d=d, head_place=hp, seed=77 + L + d + hp)
    if path == mta.PATH_KQ and not kq_applies(wl):
        pytest.skip("the contraction kernel does not take this configuration")
    if path == mta.PATH_TC and not tc_applies(wl):
        pytest.skip("the direct tensor-core kernel does not take this configuration")
    inp = synth.make_attn_inputs(wl)
    assert_close(run_attn(wl, inp, path), oracle_full(wl, inp), "bf16")


@pytest.mark.parametrize("c_q,c_k,c_h,kq", [(1, 1, 1, synth.PRE), (3, 5, 4, synth.PRE),
                                            (6, 11, 1, synth.OFF), (8, 15, 2, synth.PRE)])
def test_small_bf16_other_kernels(c_q, c_k, c_h, kq):
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=8, L=200, d=64, c_q=c_q, c_k=c_k, c_h=c_h, kq_place=kq,
                      head_place=synth.POST if c_h > 1 else synth.OFF, seed=91 + c_q)
    inp = synth.make_attn_inputs(wl)
    ref = oracle_full(wl, inp)
    assert_close(run_attn(wl, inp), ref, "bf16")
    if tc_applies(wl):
        assert_close(run_attn(wl, inp, mta.PATH_TC), ref, "bf16")
    if kq_applies(wl):
        assert_close(run_attn(wl, inp, mta.PATH_KQ), ref, "bf16")


def test_tc_path_unsupported_is_reported():
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=8, L=64, d=64, c_h=4, seed=3)
    inp = synth.make_attn_inputs(wl)
    with pytest.raises(mta.MtaError) as e:
        run_attn(wl, inp, mta.PATH_TC)
    assert e.value.code == 2


def test_strided_qkv_views():
    """q, k, v as column blocks of one [B, L, 3*H*d] buffer (the layer's layout)."""
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=2, H=4, L=260, d=128, seed=5)
    inp = synth.make_attn_inputs(wl)
    B, L, H, d = wl.B, wl.L, wl.H, wl.d
    buf = torch.empty((B, L, 3, H, d), dtype=torch.bfloat16, device="cuda")
    for i, n in enumerate("qkv"):
        buf[:, :, i] = dev(inp[n])
    q, k, v = buf[:, :, 0], buf[:, :, 1], buf[:, :, 2]
    out = mta.attn_fwd(q, k, v, dev(inp["theta"], "f32"), dev(inp["w"], "f32"), wl.c_q, wl.c_k,
                       wl.c_h, wl.kq_place, wl.head_place, check=True)
    assert_close(out, oracle_full(wl, inp), "bf16")


@pytest.mark.parametrize("path", [mta.PATH_TC, mta.PATH_KQ])
def test_causality_on_gpu(path):
    """Outputs before position t do not change when q, k, v at >= t change."""
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=400, d=128, seed=8)
    inp = synth.make_attn_inputs(wl)
    a = run_attn(wl, inp, path)
    t = 201
    for n, s in (("q", 1), ("k", 2), ("v", 3)):
        x = inp[n].copy()
        x[:, t:] = synth.round_bf16(synth.normal(99, s, x[:, t:].shape))
        inp[n] = x
    b = run_attn(wl, inp, path)
    assert torch.equal(a[:, :t], b[:, :t])
    assert not torch.equal(a[:, t:], b[:, t:])


@pytest.mark.parametrize("eq,ek", [(15, -15), (-12, 12), (0, -20)])
def test_kq_operand_scales(eq, ek):
    """The contraction kernel keeps its fp16 operands in range: queries scaled by
    2^eq and keys by 2^ek (exact in bf16).  With eq = -ek the logits, and so the
    oracle's output, are those of the unscaled inputs; (0, -20) makes the keys
    tiny, so only the per-key-row exponents keep their precision."""
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=300, d=128, seed=12)
    inp = synth.make_attn_inputs(wl)
    inp["q"] = (inp["q"] * 2.0 ** eq).astype(np.float32)
    inp["k"] = (inp["k"] * 2.0 ** ek).astype(np.float32)
    ref = oracle_full(wl, inp)
    assert_close(run_attn(wl, inp, mta.PATH_KQ), ref, "bf16")


# ---------------------------------------------------------------------------
# full-size workloads: sampled tokens
# ---------------------------------------------------------------------------

def sample_rows(wl, n_extra=6, seed=0):
    """Tile-boundary rows, a few random ones and, for a workload with planted
    pairs, every planted query row r with the c_q-1 rows after it (the
    convolution carries q_r's spike into them) and every copied key p+1 as a
    query, in every batch."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 4, 5, 6, 122, 123, 127, 128, 129, 245, 246, wl.L // 2, wl.L - 2, wl.L - 1]
    rows = sorted({(int(rng.integers(wl.B)), i) for i in fixed if i < wl.L})
    rows += [(int(rng.integers(wl.B)), int(rng.integers(wl.L))) for _ in range(n_extra)]
    for p, r in synth.planted_positions(wl):
        for b in range(wl.B):
            rows += [(b, i) for i in range(r, min(wl.L, r + wl.c_q))] + [(b, p + 1)]
    return sorted(set(rows))


@pytest.mark.parametrize("name", ["identity_d64_L2048", "pretrain_d128_L2048", "long_d128_L16384"])
@pytest.mark.parametrize("path", [mta.PATH_AUTO, mta.PATH_TC])
def test_full_size_sampled(name, path):
    """Full-size workloads: the default path (the bench's launch configuration)
    and the direct tensor-core kernel."""
    wl = synth.WORKLOADS[name]
    assert tc_applies(wl) and kq_applies(wl)
    inp = synth.make_attn_inputs(wl)
    out = run_attn(wl, inp, path)
    rows = sample_rows(wl)
    ref = O.mta_attention_rows(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h,
                               rows, wl.kq_place, wl.head_place)
    got = torch.stack([out[b, i] for b, i in rows])
    assert_close(got, ref, "bf16")
    if wl.planted_pairs:
        # the planted rows are compared on their own too, so that a wrong spike row
        # cannot hide in the norm of the other rows
        planted = {(b, r + a) for p, r in synth.planted_positions(wl) for b in range(wl.B)
                   for a in range(wl.c_q) if r + a < wl.L}
        sel = [n for n, row in enumerate(rows) if row in planted]
        assert len(sel) >= wl.planted_pairs
        assert_close(got[sel], ref[sel], "bf16")


def spike_logits(wl, inp, h, r):
    """Row r of head h's convolved logits C (log2 units), composed from the
    oracle's steps: Mask_0, the key-query convolution, nothing after it (no
    pre-softmax mixing in these workloads)."""
    qh, kh = inp["q"][0, :, h][None], inp["k"][0, :, h][None]
    a_hat = O.attention_logits(qh, kh, 1 / np.sqrt(wl.d))
    qpos = np.arange(wl.L)
    c = O.key_query_conv(O.mask_zero(a_hat, qpos), inp["theta"][h:h + 1])
    return c[0, r, :r + 1] * np.log2(np.e)


SPIKES = [(140, 200), (150, 290), (20, 100)]  # spike in a diagonal key tile, an earlier one, the first


@pytest.mark.parametrize("path", [mta.PATH_AUTO, mta.PATH_TC, mta.PATH_SIMT])
def test_planted_spikes_small_full(path):
    """Planted high-similarity pairs (the long-context workload's recipe) at a
    size the oracle computes in full: the spike of row 200 sits in its own
    (diagonal) key tile 128..255, the spike of row 290 in the earlier tile
    128..255, and the spike of row 100 in the first tile.  For the first two the
    convolved logit at the spike exceeds every logit of the earlier key tiles by
    more than 8 (log2 units) in every head, so the kernels' online softmax takes
    its lazy rescale branch there (it rescales Z only when the running max grows by more
    than 2^8); every element is compared."""
    wl = synth.shrink(synth.WORKLOADS["long_d128_L16384"], B=1, H=4, L=300, planted_pairs=0,
                      seed=1104)
    inp = synth.make_attn_inputs(wl)
    synth.plant_pairs_at(inp["q"], inp["k"], SPIKES, wl.seed)
    inp["q"], inp["k"] = synth.round_bf16(inp["q"]), synth.round_bf16(inp["k"])
    for p, r in SPIKES[:2]:
        for h in range(wl.H):
            c = spike_logits(wl, inp, h, r)
            t_p = p // 128
            assert c[128 * t_p:].max() > c[:128 * t_p].max() + 8.0, (p, r, h)
    assert_close(run_attn(wl, inp, path), oracle_full(wl, inp), "bf16")


def test_identity_workload_equals_causal_attention():
    """Identity kernels: the whole output equals causal softmax attention (torch
    SDPA in fp32 on the same bf16 inputs)."""
    wl = synth.WORKLOADS["identity_d64_L2048"]
    inp = synth.make_attn_inputs(wl)
    out = run_attn(wl, inp)
    q, k, v = (dev(inp[n], "f32").permute(0, 2, 1, 3) for n in "qkv")
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    ref = ref.permute(0, 2, 1, 3).double().cpu().numpy()
    assert_close(out, ref, "bf16")


@pytest.mark.parametrize("name,calls", [("identity_d64_L2048", 2000), ("pretrain_d128_L2048", 500),
                                        ("layer_pre_D2048_L4096", 200), ("layer_post_D2048_L4096", 300),
                                        ("both_d128_L2048", 150)])
def test_repeated_calls_never_time_out(name, calls):
    """Back-to-back calls, the status word read after every one (each call clears it):
    the one-CTA kernel with and without pre- or post-softmax mixing, the CTA-pair
    kernel (L = 4096) and the two-pass kernel of the convolution after the softmax.
    With post-softmax mixing the two CTAs of a cluster exchange their partial outputs
    once per work item; the last items of the queue span a single key tile, so one CTA
    can finish an item's exchange while its peer still waits for the previous one.  A
    single exchange barrier then completed two phases under the waiter and its bounded
    wait ran out, about once per 250 calls at d = 64.  Every 100th call's output is
    also compared with the first call's: the same inputs give the same bits."""
    wl = synth.WORKLOADS[name]
    inp = synth.make_attn_inputs(wl)
    q, k, v = (dev(inp[n]) for n in "qkv")
    th, w = dev(inp["theta"], "f32"), dev(inp["w"], "f32")
    tp = dev(inp["theta_post"], "f32") if wl.kq_post else None
    cfg = mta.make_cfg(wl.B, wl.H, wl.L, wl.d, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, mta.BF16,
                       kq_post=int(wl.kq_post))
    ws = mta.workspace(mta.lib().mta_attn_workspace_bytes(ctypes.byref(cfg)))
    first = None
    out = torch.empty_like(q)
    for i in range(calls):
        mta.attn_fwd(q, k, v, th, w, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, out=out, ws=ws,
                     check=True, theta_post=tp)
        if first is None:
            first = out.clone()
        elif i % 100 == 0:
            assert torch.equal(out, first), f"call {i} differs from the first"


def test_no_LxL_buffer():
    """Peak device memory of a call stays at inputs + outputs + workspace."""
    wl = synth.WORKLOADS["pretrain_d128_L2048"]
    inp = synth.make_attn_inputs(wl)
    q, k, v = (dev(inp[n]) for n in "qkv")
    th, w = dev(inp["theta"], "f32"), dev(inp["w"], "f32")
    out = torch.empty_like(q)
    ws = mta.workspace(256)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.memory_allocated()
    mta.attn_fwd(q, k, v, th, w, wl.c_q, wl.c_k, wl.c_h, out=out, ws=ws, check=True)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == before
    lxl = wl.B * wl.H * wl.L * wl.L * 4
    assert before < lxl


# ---------------------------------------------------------------------------
# building blocks and the layer
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(300, 520, 264), (128, 256, 64), (1000, 96, 2048), (7, 9, 8)])
def test_gemm_bf16_nt(M, N, K):
    a = synth.round_bf16(synth.normal(3, 1, (M, K)))
    b = synth.round_bf16(synth.normal(3, 2, (N, K), std=0.05))
    c = mta.gemm_bf16_nt(dev(a), dev(b))
    torch.cuda.synchronize()
    assert_close(c, a.astype(np.float64) @ b.astype(np.float64).T, "bf16")


def test_group_norm_scale():
    o = synth.round_bf16(synth.normal(4, 1, (515, 16, 128), mean=0.3, std=2.0))
    gamma = synth.normal(4, 2, (16 * 128,), mean=1.0, std=0.1)
    beta = synth.normal(4, 3, (16 * 128,), std=0.1)
    y = mta.group_norm_scale(dev(o), dev(gamma, "f32"), dev(beta, "f32"), 1e-5, 0.97814)
    torch.cuda.synchronize()
    assert_close(y, O.group_norm_scale(o, gamma, beta, 1e-5, 0.97814), "bf16")
    o2 = o[:, :, :72].copy()
    y2 = mta.group_norm_scale(dev(o2), dev(gamma[:16 * 72], "f32"), dev(beta[:16 * 72], "f32"),
                              1e-5, 0.5)
    torch.cuda.synchronize()
    assert_close(y2, O.group_norm_scale(o2, gamma[:16 * 72], beta[:16 * 72], 1e-5, 0.5), "bf16")


def run_layer(wl, inp, path=mta.PATH_AUTO):
    x, wqkv, wo = dev(inp["x"]), dev(inp["wqkv"]), dev(inp["wo"])
    tp = None if inp.get("theta_post") is None else dev(inp["theta_post"], "f32")
    out = mta.layer_fwd(x, wqkv, dev(inp["theta"], "f32"), dev(inp["w"], "f32"),
                        dev(inp["gamma"], "f32"), dev(inp["beta"], "f32"), wo, wl.H, wl.c_q,
                        wl.c_k, wl.c_h, wl.kq_place, wl.head_place, eps=inp["eps"],
                        layer=wl.depth, path=path, check=True, theta_post=tp)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("name", ["layer_pre_D2048_L4096", "layer_post_D2048_L4096"])
@pytest.mark.parametrize("path", [mta.PATH_AUTO, mta.PATH_SIMT])
def test_layer_small(name, path):
    wl = synth.shrink(synth.WORKLOADS[name], B=2, L=300, D=256, H=2, d=128, seed=123)
    inp = synth.make_layer_inputs(wl)
    out = run_layer(wl, inp, path)
    ref = O.mta_layer(inp["x"], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"], inp["beta"],
                      inp["eps"], O.depth_scale(wl.depth), inp["wo"], wl.H, wl.c_h, wl.kq_place, wl.head_place)
    assert_close(out, ref, "bf16")


@pytest.mark.parametrize("name", ["layer_pre_D2048_L4096", "layer_post_D2048_L4096"])
def test_layer_full_size_sampled(name):
    wl = synth.WORKLOADS[name]
    inp = synth.make_layer_inputs(wl)
    out = run_layer(wl, inp)
    rows = [(0, 0), (0, 5), (0, 123), (0, 2048), (0, 4095), (1, 1), (1, 700), (1, 4094)]
    ref = O.mta_layer_rows(inp["x"], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"],
                           inp["beta"], inp["eps"], O.depth_scale(wl.depth), inp["wo"], wl.H, wl.c_h, rows,
                           wl.kq_place, wl.head_place)
    got = torch.stack([out[b, i] for b, i in rows])
    assert_close(got, ref, "bf16")


# ---------------------------------------------------------------------------
# exact causal indicator (kq_place = PRE_EXACT) and the sigmoid scalar gate
# ---------------------------------------------------------------------------

def oracle_exact(wl, inp):
    return O.mta_attention(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h,
                           O.PRE_EXACT, wl.head_place)


@pytest.mark.parametrize("d,hp,L", [(64, synth.OFF, 9), (128, synth.POST, 300), (64, synth.POST, 300),
                                    (128, synth.OFF, 1), (128, synth.PRE, 300), (64, synth.PRE, 130)])
@pytest.mark.parametrize("path", [mta.PATH_AUTO, mta.PATH_SIMT, mta.PATH_KQ])
def test_exact_indicator_small(d, hp, L, path):
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=2, H=4, L=L, d=d, head_place=hp, kq_place=mta.PRE_EXACT,
                      seed=301 + L + d + hp)
    inp = synth.make_attn_inputs(wl)
    assert_close(run_attn(wl, inp, path), oracle_exact(wl, inp), "bf16")


def test_exact_indicator_differs_from_mask0_on_gpu():
    """The two kernels of section 3.1 give different outputs near the diagonal."""
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=260, d=128, kq_place=mta.PRE_EXACT, seed=33)
    inp = synth.make_attn_inputs(wl)
    a = run_attn(wl, inp, mta.PATH_KQ)
    wl0 = synth.shrink(wl, kq_place=mta.PRE)
    b = run_attn(wl0, inp, mta.PATH_KQ)
    rel, _ = errs(a, b.double().cpu().numpy())
    assert rel > 1e-3


def test_exact_indicator_causality_on_gpu():
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=400, d=128, kq_place=mta.PRE_EXACT, seed=34)
    inp = synth.make_attn_inputs(wl)
    a = run_attn(wl, inp, mta.PATH_KQ)
    t = 201
    for n, s in (("q", 1), ("k", 2), ("v", 3)):
        x = inp[n].copy()
        x[:, t:] = synth.round_bf16(synth.normal(98, s, x[:, t:].shape))
        inp[n] = x
    b = run_attn(wl, inp, mta.PATH_KQ)
    assert torch.equal(a[:, :t], b[:, :t])
    assert not torch.equal(a[:, t:], b[:, t:])


def test_exact_indicator_full_size_sampled():
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], kq_place=mta.PRE_EXACT)
    inp = synth.make_attn_inputs(wl)
    out = run_attn(wl, inp)
    rows = sample_rows(wl, seed=5)
    ref = O.mta_attention_rows(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h, rows,
                               O.PRE_EXACT, wl.head_place)
    got = torch.stack([out[b, i] for b, i in rows])
    assert_close(got, ref, "bf16")


@pytest.mark.parametrize("name,path", [("layer_post_D2048_L4096", mta.PATH_AUTO),
                                       ("layer_pre_D2048_L4096", mta.PATH_AUTO),
                                       ("layer_post_D2048_L4096", mta.PATH_SIMT)])
def test_layer_sigmoid_gate(name, path):
    """The sigmoid scalar gate replaces the depth scale in every epilogue."""
    wl = synth.shrink(synth.WORKLOADS[name], B=2, L=300, D=256, H=2, d=128, seed=124)
    inp = synth.make_layer_inputs(wl)
    gate = np.array([-0.8, 1.3], np.float32)
    x, wqkv, wo = dev(inp["x"]), dev(inp["wqkv"]), dev(inp["wo"])
    out = mta.layer_fwd(x, wqkv, dev(inp["theta"], "f32"), dev(inp["w"], "f32"),
                        dev(inp["gamma"], "f32"), dev(inp["beta"], "f32"), wo, wl.H, wl.c_q,
                        wl.c_k, wl.c_h, wl.kq_place, wl.head_place, eps=inp["eps"],
                        layer=wl.depth, gate=dev(gate, "f32"), path=path, check=True)
    torch.cuda.synchronize()
    ref = O.mta_layer(inp["x"], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"], inp["beta"],
                      inp["eps"], O.sigmoid_gate(gate), inp["wo"], wl.H, wl.c_h, wl.kq_place,
                      wl.head_place)
    assert_close(out, ref, "bf16")


def test_group_norm_sigmoid_gate():
    o = synth.round_bf16(synth.normal(5, 1, (300, 4, 128), mean=0.1, std=1.5))
    gamma = synth.normal(5, 2, (4 * 128,), mean=1.0, std=0.1)
    beta = synth.normal(5, 3, (4 * 128,), std=0.1)
    gate = np.array([-2.0, 0.0, 0.4, 3.0], np.float32)
    y = mta.group_norm_scale(dev(o), dev(gamma, "f32"), dev(beta, "f32"), 1e-5, 1.0,
                             gate=dev(gate, "f32"))
    torch.cuda.synchronize()
    assert_close(y, O.group_norm_scale(o, gamma, beta, 1e-5, O.sigmoid_gate(gate)), "bf16")


# ---------------------------------------------------------------------------
# key-query convolution after the softmax as well (kq_post)
# ---------------------------------------------------------------------------

POST_SMALL = [("f32", synth.PRE, synth.POST, 9), ("f32", synth.OFF, synth.OFF, 70),
              ("bf16", synth.PRE, synth.POST, 150), ("bf16", synth.PRE, synth.PRE, 150),
              ("bf16", synth.PRE, synth.OFF, 33), ("bf16", synth.OFF, synth.POST, 150),
              ("bf16", mta.PRE_EXACT, synth.POST, 150), ("bf16", synth.PRE, synth.POST, 1)]


@pytest.mark.parametrize("dtype,kq,hp,L", POST_SMALL)
def test_post_conv_small(dtype, kq, hp, L):
    base = synth.WORKLOADS["both_d128_L2048"]
    wl = synth.shrink(base, B=2, H=4, L=L, d=64, kq_place=kq, head_place=hp, dtype=dtype,
                      seed=401 + L + kq + 3 * hp)
    inp = synth.make_attn_inputs(wl)
    assert inp["theta_post"] is not None
    assert_close(run_attn(wl, inp), oracle_full(wl, inp), dtype)


POST_PATHS = [(d, hp, L) for d in (64, 96, 128) for hp in (synth.OFF, synth.PRE, synth.POST)
              for L in (9, 300)]


@pytest.mark.parametrize("d,hp,L", POST_PATHS)
@pytest.mark.parametrize("path", [mta.PATH_SIMT, mta.PATH_KQ])
def test_post_conv_kernels(d, hp, L, path):
    """Both kernels that take the post-softmax convolution, with tiles of 123
    output rows on the contraction kernel (L = 300: three tiles, ragged tail)."""
    base = synth.WORKLOADS["both_d128_L2048"]
    wl = synth.shrink(base, B=2, H=4, L=L, d=d, head_place=hp, seed=501 + L + d + hp)
    inp = synth.make_attn_inputs(wl)
    assert_close(run_attn(wl, inp, path), oracle_full(wl, inp), "bf16")


@pytest.mark.parametrize("hp,L", [(synth.POST, 300), (synth.OFF, 130)])
def test_post_conv_exact_indicator_kq(hp, L):
    base = synth.WORKLOADS["both_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=L, d=128, head_place=hp, kq_place=mta.PRE_EXACT, seed=601 + L)
    inp = synth.make_attn_inputs(wl)
    assert_close(run_attn(wl, inp, mta.PATH_KQ), oracle_full(wl, inp), "bf16")


def test_post_conv_causality_kq():
    base = synth.WORKLOADS["both_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=400, d=128, seed=457)
    inp = synth.make_attn_inputs(wl)
    a = run_attn(wl, inp, mta.PATH_KQ)
    t = 250
    for n, s in (("q", 1), ("k", 2), ("v", 3)):
        x = inp[n].copy()
        x[:, t:] = synth.round_bf16(synth.normal(97, s, x[:, t:].shape))
        inp[n] = x
    b = run_attn(wl, inp, mta.PATH_KQ)
    assert torch.equal(a[:, :t], b[:, :t])
    assert not torch.equal(a[:, t:], b[:, t:])


def test_post_conv_other_kernel_sizes():
    base = synth.WORKLOADS["both_d128_L2048"]
    wl = synth.shrink(base, B=1, H=8, L=100, d=32, c_q=3, c_k=5, c_h=4, seed=455)
    inp = synth.make_attn_inputs(wl)
    assert_close(run_attn(wl, inp), oracle_full(wl, inp), "bf16")


def test_post_conv_causality_on_gpu():
    base = synth.WORKLOADS["both_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=200, d=64, seed=456)
    inp = synth.make_attn_inputs(wl)
    a = run_attn(wl, inp)
    t = 77
    for n, s in (("q", 1), ("k", 2), ("v", 3)):
        x = inp[n].copy()
        x[:, t:] = synth.round_bf16(synth.normal(99, s, x[:, t:].shape))
        inp[n] = x
    b = run_attn(wl, inp)
    assert torch.equal(a[:, :t], b[:, :t])
    assert not torch.equal(a[:, t:], b[:, t:])


def test_post_conv_full_size_sampled():
    """The pretraining-shaped workload with the convolution on both sides of the
    softmax, in the launch configuration the bench times."""
    wl = synth.WORKLOADS["both_d128_L2048"]
    inp = synth.make_attn_inputs(wl)
    out = run_attn(wl, inp)
    rows = sample_rows(wl, seed=6)
    ref = O.mta_attention_rows(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h, rows,
                               wl.kq_place, wl.head_place, theta_post=inp["theta_post"])
    got = torch.stack([out[b, i] for b, i in rows])
    assert_close(got, ref, "bf16")


@pytest.mark.parametrize("hp", [synth.PRE, synth.POST])
def test_post_conv_layer_small(hp):
    wl = synth.shrink(synth.WORKLOADS["layer_post_D2048_L4096"], B=2, L=200, D=256, H=2, d=128,
                      head_place=hp, kq_post=True, seed=125)
    inp = synth.make_layer_inputs(wl)
    out = run_layer(wl, inp)
    ref = O.mta_layer(inp["x"], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"], inp["beta"],
                      inp["eps"], O.depth_scale(wl.depth), inp["wo"], wl.H, wl.c_h, wl.kq_place, wl.head_place,
                      theta_post=inp["theta_post"])
    assert_close(out, ref, "bf16")


# ---------------------------------------------------------------------------
# head dimension 96 (the pages' 880M model: dimension 1536 over 16 heads)
# ---------------------------------------------------------------------------

def test_d96_full_size_sampled():
    wl = synth.WORKLOADS["pretrain_d96_L2048"]
    assert kq_applies(wl)
    inp = synth.make_attn_inputs(wl)
    out = run_attn(wl, inp)
    rows = sample_rows(wl, seed=7)
    ref = O.mta_attention_rows(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h, rows,
                               wl.kq_place, wl.head_place)
    got = torch.stack([out[b, i] for b, i in rows])
    assert_close(got, ref, "bf16")


@pytest.mark.parametrize("kq,post", [(synth.PRE, False), (mta.PRE_EXACT, False), (synth.PRE, True)])
def test_d96_kq_variants(kq, post):
    base = synth.WORKLOADS["pretrain_d96_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=260, kq_place=kq, kq_post=post, seed=701 + kq + 2 * post)
    inp = synth.make_attn_inputs(wl)
    assert_close(run_attn(wl, inp, mta.PATH_KQ), oracle_full(wl, inp), "bf16")


@pytest.mark.parametrize("hp", [synth.PRE, synth.POST])
def test_d96_layer_small(hp):
    wl = synth.shrink(synth.WORKLOADS["layer_post_D2048_L4096"], B=2, L=200, D=192, H=2, d=96,
                      head_place=hp, seed=126)
    inp = synth.make_layer_inputs(wl)
    out = run_layer(wl, inp)
    ref = O.mta_layer(inp["x"], inp["wqkv"], inp["theta"], inp["w"], inp["gamma"], inp["beta"],
                      inp["eps"], O.depth_scale(wl.depth), inp["wo"], wl.H, wl.c_h, wl.kq_place, wl.head_place)
    assert_close(out, ref, "bf16")


# ---------------------------------------------------------------------------
# backward pass (mta_attn_bwd): every gradient against the fp64 oracle
# ---------------------------------------------------------------------------

GRAD_NAMES = ("dq", "dk", "dv", "dtheta", "dw", "dtheta_post")


def run_bwd(wl, inp, dout):
    q, k, v = (dev(inp[n], wl.dtype) for n in ("q", "k", "v"))
    tp = None if inp.get("theta_post") is None else dev(inp["theta_post"], "f32")
    g = mta.attn_bwd(q, k, v, dev(inp["theta"], "f32"), dev(inp["w"], "f32"), dev(dout, wl.dtype),
                     wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place, check=True, theta_post=tp)
    torch.cuda.synchronize()
    return g


def check_grads(wl, inp, dout, tol=TOL_F32):
    got = run_bwd(wl, inp, dout)
    ref = O.mta_attention_bwd(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h, dout,
                              wl.kq_place, wl.head_place, theta_post=inp.get("theta_post"))
    for n in GRAD_NAMES:
        if ref[n] is None:
            assert got[n] is None
            continue
        rel, mx = errs(got[n], ref[n])
        assert rel <= tol, (n, rel, mx)


BWD_SMALL = [("f32", synth.PRE, synth.POST, 9), ("f32", synth.PRE, synth.PRE, 70),
             ("f32", synth.OFF, synth.OFF, 70), ("f32", mta.PRE_EXACT, synth.POST, 70),
             ("bf16", synth.PRE, synth.POST, 70), ("bf16", synth.PRE, synth.OFF, 33),
             ("bf16", synth.OFF, synth.POST, 40), ("bf16", mta.PRE_EXACT, synth.PRE, 50)]


@pytest.mark.parametrize("dtype,kq,hp,L", BWD_SMALL)
def test_bwd_small(dtype, kq, hp, L):
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=2, H=4, L=L, d=32, kq_place=kq, head_place=hp, dtype=dtype,
                      seed=801 + L + kq + 3 * hp)
    inp = synth.make_attn_inputs(wl)
    dout = synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d))
    if dtype == "bf16":
        dout = synth.round_bf16(dout)
    check_grads(wl, inp, dout)


def test_bwd_other_kernel_sizes():
    base = synth.WORKLOADS["pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=8, L=45, d=16, c_q=3, c_k=5, c_h=4, seed=850)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check_grads(wl, inp, dout)


def test_bwd_pretrain_recipe_L512():
    """The pretraining recipe (d = 128, c_q = 6, c_k = 11, post-softmax mixing) at a
    length the fp64 oracle finishes in seconds: four tiles of 128 keys."""
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=1, H=4, L=512, seed=851)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check_grads(wl, inp, dout)


BWD_POST = [("f32", synth.PRE, synth.POST, 9), ("f32", synth.PRE, synth.PRE, 40),
            ("bf16", synth.PRE, synth.POST, 70), ("bf16", synth.OFF, synth.POST, 50),
            ("bf16", mta.PRE_EXACT, synth.OFF, 45), ("bf16", synth.PRE, synth.OFF, 33)]


@pytest.mark.parametrize("dtype,kq,hp,L", BWD_POST)
def test_bwd_post_conv_small(dtype, kq, hp, L):
    """The backward with the key-query convolution also after the softmax: every
    gradient, the post-softmax kernels' included."""
    base = synth.WORKLOADS["both_d128_L2048"]
    wl = synth.shrink(base, B=2, H=4, L=L, d=32, kq_place=kq, head_place=hp, dtype=dtype,
                      seed=861 + L + kq + 3 * hp)
    inp = synth.make_attn_inputs(wl)
    dout = synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d))
    if dtype == "bf16":
        dout = synth.round_bf16(dout)
    check_grads(wl, inp, dout)


def test_bwd_post_conv_recipe_L300():
    wl = synth.shrink(synth.WORKLOADS["both_d128_L2048"], B=1, H=2, L=300, seed=862)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check_grads(wl, inp, dout)


def test_bwd_full_length_one_group():
    """The pretraining recipe at its full length L = 2048 (the length the bench's
    backward line runs) for one batch and one head group, against the fp64
    oracle's full L x L backward of that group."""
    wl = synth.shrink(synth.WORKLOADS["pretrain_d128_L2048"], B=1, H=2, seed=852)
    inp = synth.make_attn_inputs(wl)
    dout = synth.round_bf16(synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d)))
    check_grads(wl, inp, dout)


@pytest.mark.parametrize("post", [False, True])
def test_autograd_function_matches_oracle(post):
    """mta.mta_attention as a torch op: torch.autograd.grad through it returns the
    oracle's gradients (the op calls mta_attn_fwd and mta_attn_bwd)."""
    base = synth.WORKLOADS["both_d128_L2048" if post else "pretrain_d128_L2048"]
    wl = synth.shrink(base, B=1, H=4, L=90, d=64, dtype="f32", seed=871 + post)
    inp = synth.make_attn_inputs(wl)
    dout = synth.normal(wl.seed, 20, (wl.B, wl.L, wl.H, wl.d))
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda().requires_grad_(True)
    q, k, v, th, w = (t(inp[n]) for n in ("q", "k", "v", "theta", "w"))
    tp = t(inp["theta_post"]) if post else None
    out = mta.mta_attention(q, k, v, th, w, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                            theta_post=tp)
    leaves = [q, k, v, th, w] + ([tp] if post else [])
    grads = torch.autograd.grad(out, leaves, torch.from_numpy(dout).cuda())
    ref = O.mta_attention_bwd(inp["q"], inp["k"], inp["v"], inp["theta"], inp["w"], wl.c_h, dout,
                              wl.kq_place, wl.head_place, theta_post=inp["theta_post"])
    names = ["dq", "dk", "dv", "dtheta", "dw"] + (["dtheta_post"] if post else [])
    for n, g in zip(names, grads):
        rel, _ = errs(g, ref[n])
        assert rel <= TOL_F32, (n, rel)
    assert_close(out, oracle_full(wl, inp), "f32")
