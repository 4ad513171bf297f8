"""Pins of the fp64 oracle to facts other than itself.

Each test checks the oracle against a library routine, a closed form, an
invariant stated or implied by the pages, or a brute-force restatement on tiny
inputs, chosen so that a dropped term, a wrong sign or index or a transposed
operand anywhere in the oracle fails at least one of them.  Sources:
"Multi-Token Attention | Summary" (greeksharifa), sections 2, 3.1, 3.2, 3.3,
4.6 (identity initialisation) and appendix B.
"""
import itertools

import numpy as np
import pytest
import scipy.signal
import scipy.special
import torch

import oracle as O


def rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def sdpa(q, k, v, scale):
    """Causal softmax attention by torch's library routine, fp64.  q,k,v [H,L,d]."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q)[None], t(k)[None], t(v)[None], is_causal=True, scale=scale)[0].numpy()


def to_bhld(x):  # [B,L,H,d] -> [B,H,L,d]
    return np.ascontiguousarray(x.transpose(0, 2, 1, 3))


def delta_theta(H, cq, ck, a, t, tau=1.0):
    th = np.zeros((H, cq, ck))
    th[:, a, t] = tau
    return th


SHAPE = dict(B=2, L=23, H=4, d=8)


@pytest.fixture(scope="module")
def qkv():
    B, L, H, d = SHAPE["B"], SHAPE["L"], SHAPE["H"], SHAPE["d"]
    return rand((B, L, H, d), 1), rand((B, L, H, d), 2), rand((B, L, H, d), 3)


@pytest.mark.parametrize("head_place", [O.OFF, O.PRE, O.POST])
def test_identity_kernels_equal_causal_sdpa(qkv, head_place):
    """theta = delta at (0,0), w = I reduces MTA to standard causal multi-head
    attention (identity initialisation keeps the pretrained map, section 4.6)."""
    q, k, v = qkv
    B, L, H, d = q.shape
    cq, ck, ch = 3, 5, 2
    th = delta_theta(H, cq, ck, 0, ck // 2)
    w = np.tile(np.eye(ch), (H // ch, 1, 1))
    out = O.mta_attention(q, k, v, th, w, ch, O.PRE, head_place)
    ref = sdpa(to_bhld(q).reshape(B * H, L, d), to_bhld(k).reshape(B * H, L, d),
               to_bhld(v).reshape(B * H, L, d), 1 / np.sqrt(d))
    np.testing.assert_allclose(to_bhld(out).reshape(B * H, L, d), ref, rtol=0, atol=1e-12)


def _closed_form_attention(q, k, v, logit_fn, scale):
    """Brute force on one head: logits from a closed form, -inf on future keys,
    softmax by scipy, times V.  q,k,v [L,d]."""
    L = q.shape[0]
    lg = np.full((L, L), -np.inf)
    for i in range(L):
        for j in range(i + 1):
            lg[i, j] = logit_fn(i, j)
    return scipy.special.softmax(lg, axis=1) @ v


@pytest.mark.parametrize("a", [1, 2])
def test_query_shift_delta_closed_form(qkv, a):
    """theta = delta at (a, 0): C[i,j] = s q[i-a].k[j] if j <= i-a, and 0 for
    i-a < j <= i (Mask_0 zeroes the future of the shifted query), section 3.1."""
    q, k, v = qkv
    B, L, H, d = q.shape
    cq, ck = 3, 5
    s = 1 / np.sqrt(d)
    th = delta_theta(H, cq, ck, a, ck // 2)
    out = O.mta_attention(q, k, v, th, np.tile(np.eye(1), (H, 1, 1)), 1, O.PRE, O.OFF)
    for b, h in [(0, 0), (1, 3)]:
        qq, kk, vv = q[b, :, h], k[b, :, h], v[b, :, h]
        fn = lambda i, j: s * qq[i - a] @ kk[j] if (i - a >= 0 and j <= i - a) else 0.0
        np.testing.assert_allclose(out[b, :, h], _closed_form_attention(qq, kk, vv, fn, s),
                                   rtol=0, atol=1e-12)


@pytest.mark.parametrize("boff", [-2, -1, 1, 2])
def test_key_shift_delta_closed_form(qkv, boff):
    """theta = delta at (0, b): C[i,j] = s q[i].k[j-b] when 0 <= j-b <= i, else 0
    inside the causal region (pins the key orientation), section 3.1."""
    q, k, v = qkv
    B, L, H, d = q.shape
    cq, ck = 2, 5
    s = 1 / np.sqrt(d)
    th = delta_theta(H, cq, ck, 0, ck // 2 + boff)
    out = O.mta_attention(q, k, v, th, np.tile(np.eye(1), (H, 1, 1)), 1, O.PRE, O.OFF)
    for b, h in [(0, 1), (1, 2)]:
        qq, kk, vv = q[b, :, h], k[b, :, h], v[b, :, h]
        fn = lambda i, j: s * qq[i] @ kk[j - boff] if 0 <= j - boff <= i else 0.0
        np.testing.assert_allclose(out[b, :, h], _closed_form_attention(qq, kk, vv, fn, s),
                                   rtol=0, atol=1e-12)


def test_scaled_delta_is_temperature(qkv):
    """theta = tau * delta(0,0) gives softmax(tau s Q K^T) V (library SDPA with
    scale tau*s)."""
    q, k, v = qkv
    B, L, H, d = q.shape
    tau = 1.7
    th = delta_theta(H, 3, 5, 0, 2, tau)
    out = O.mta_attention(q, k, v, th, np.ones((H, 1, 1)), 1, O.PRE, O.OFF)
    ref = sdpa(to_bhld(q).reshape(B * H, L, d), to_bhld(k).reshape(B * H, L, d),
               to_bhld(v).reshape(B * H, L, d), tau / np.sqrt(d))
    np.testing.assert_allclose(to_bhld(out).reshape(B * H, L, d), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("head_place", [O.PRE, O.POST])
def test_causality_bit_exact(qkv, head_place):
    """Only current and past queries and keys matter (section 3.1, causal mask of
    section 2): perturbing position t leaves outputs at i < t bit-identical."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 5, 0.3)
    w = rand((H // 2, 2, 2), 6, 0.5)
    base = O.mta_attention(q, k, v, th, w, 2, O.PRE, head_place)
    t = 14
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, t:] += rand(q2[:, t:].shape, 7)
    k2[:, t:] += rand(k2[:, t:].shape, 8)
    v2[:, t:] += rand(v2[:, t:].shape, 9)
    pert = O.mta_attention(q2, k2, v2, th, w, 2, O.PRE, head_place)
    assert np.array_equal(base[:, :t], pert[:, :t])
    assert not np.allclose(base[:, t:], pert[:, t:])


def test_rows_sum_to_one_and_post_mix_row_sums(qkv):
    """Softmax rows sum to 1 (section 2); post-softmax mixing is a plain linear
    combination, so with V = 1 the output of head r is sum_s w[r,s] (section 3.2)."""
    q, k, _ = qkv
    B, L, H, d = q.shape
    ones = np.ones_like(q)
    th = rand((H, 3, 5), 11, 0.3)
    out = O.mta_attention(q, k, ones, th, np.ones((H, 1, 1)), 1, O.PRE, O.OFF)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)
    w = rand((H // 2, 2, 2), 12)
    out = O.mta_attention(q, k, ones, th, w, 2, O.PRE, O.POST)
    rs = w.sum(axis=2).reshape(H)               # head g*2+r -> sum_s w[g,r,s]
    np.testing.assert_allclose(out, np.broadcast_to(rs[None, None, :, None], out.shape),
                               rtol=0, atol=1e-12)


def test_post_mix_is_linear_in_w(qkv):
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 13, 0.3)
    w1, w2 = rand((H // 2, 2, 2), 14), rand((H // 2, 2, 2), 15)
    f = lambda w: O.mta_attention(q, k, v, th, w, 2, O.PRE, O.POST)
    np.testing.assert_allclose(f(w1 + w2), f(w1) + f(w2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(f(-2.5 * w1), -2.5 * f(w1), rtol=0, atol=1e-12)


def test_appendix_b_destination_values(qkv):
    """Appendix B: post-softmax mixing acts through the value projection, i.e.
    O^h = sum_h' w[h,h'] softmax-attention(Q^h', K^h', V^h).  With identity
    theta every term is the library's causal SDPA."""
    q, k, v = qkv
    B, L, H, d = q.shape
    ch = 2
    w = rand((H // ch, ch, ch), 16)
    th = delta_theta(H, 3, 5, 0, 2)
    out = O.mta_attention(q, k, v, th, w, ch, O.PRE, O.POST)
    s = 1 / np.sqrt(d)
    for b in range(B):
        for h in range(H):
            g, r = divmod(h, ch)
            ref = sum(w[g, r, sp] * sdpa(q[b, :, g * ch + sp][None], k[b, :, g * ch + sp][None],
                                         v[b, :, h][None], s)[0] for sp in range(ch))
            np.testing.assert_allclose(out[b, :, h], ref, rtol=0, atol=1e-12)


def test_first_row(qkv):
    """Query 0 sees only key 0: A[0,0] = 1, so O_0 = (sum_s w[r,s]) v_0 after a
    post mix and O_0 = v_0 without mixing or with a pre-softmax mix."""
    q, k, v = qkv
    B, L, H, d = q.shape
    th = rand((H, 3, 5), 17, 0.4)
    w = rand((H // 2, 2, 2), 18)
    out = O.mta_attention(q, k, v, th, w, 2, O.PRE, O.POST)
    rs = w.sum(axis=2).reshape(H)
    np.testing.assert_allclose(out[:, 0], rs[None, :, None] * v[:, 0], rtol=0, atol=1e-12)
    out = O.mta_attention(q, k, v, th, w, 2, O.PRE, O.PRE)
    np.testing.assert_allclose(out[:, 0], v[:, 0], rtol=0, atol=1e-12)


def test_conv_matches_scipy_convolve2d():
    """Conv2d_theta over (query, key) is a zero-padded 2-D convolution: scipy's
    'full' convolve2d of the masked map with theta, shifted by c_k//2 keys."""
    ch, L, cq, ck = 2, 19, 4, 7
    m = rand((ch, L, L), 21)
    th = rand((ch, cq, ck), 22)
    out = O.key_query_conv(m, th)
    for h in range(ch):
        full = scipy.signal.convolve2d(m[h], th[h], mode="full")   # [L+cq-1, L+ck-1]
        ref = full[:L, ck // 2: ck // 2 + L]
        np.testing.assert_allclose(out[h], ref, rtol=0, atol=1e-12)


def test_pipeline_matches_scipy_restatement(qkv):
    """Whole attention with random theta and w (pre and post mixing), restated
    with library pieces: logits by einsum, Mask_0 by np.tril, the convolution by
    scipy.signal.convolve2d, softmax by scipy.special.softmax."""
    q, k, v = qkv
    B, L, H, d = q.shape
    cq, ck, ch = 3, 5, 2
    th = rand((H, cq, ck), 23, 0.5)
    w = rand((H // ch, ch, ch), 24)
    s = 1 / np.sqrt(d)
    causal = np.tril(np.ones((L, L), bool))
    for head_place in (O.PRE, O.POST):
        out = O.mta_attention(q, k, v, th, w, ch, O.PRE, head_place)
        for b in range(B):
            lg = s * np.einsum("lhd,mhd->hlm", q[b], k[b])
            conv = np.stack([scipy.signal.convolve2d(np.tril(lg[h]), th[h], mode="full")
                             [:L, ck // 2: ck // 2 + L] for h in range(H)])
            conv = conv.reshape(H // ch, ch, L, L)
            if head_place == O.PRE:
                conv = np.einsum("grs,gslm->grlm", w, conv)
            p = scipy.special.softmax(np.where(causal, conv, -np.inf), axis=-1)
            if head_place == O.POST:
                p = np.einsum("grs,gslm->grlm", w, p)
            ref = np.einsum("hlm,mhd->lhd", p.reshape(H, L, L), v[b])
            np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def test_pre_mix_as_3d_convolution_bruteforce():
    """Section 3.3: key-query and head mixing on the same side of the softmax form
    one 3-D convolution over (head, query, key).  Pure-Python loops on a tiny
    case with theta3[h][h'][a][t] = w[h,h'] theta[h'][a][t]."""
    B, L, H, d, cq, ck, ch = 1, 7, 2, 3, 2, 3, 2
    q, k, v = rand((B, L, H, d), 31), rand((B, L, H, d), 32), rand((B, L, H, d), 33)
    th = rand((H, cq, ck), 34)
    w = rand((1, ch, ch), 35)
    out = O.mta_attention(q, k, v, th, w, ch, O.PRE, O.PRE)
    s = 1 / np.sqrt(d)
    c = ck // 2

    def m0(h, i, j):
        if i < 0 or j < 0 or j >= L or j > i:
            return 0.0
        return s * sum(q[0, i, h, x] * k[0, j, h, x] for x in range(d))

    for h in range(H):
        for i in range(L):
            row = []
            for j in range(i + 1):
                acc = 0.0
                for hp, a, t in itertools.product(range(ch), range(cq), range(ck)):
                    acc += w[0, h, hp] * th[hp, a, t] * m0(hp, i - a, j - (t - c))
                row.append(acc)
            mx = max(row)
            e = [np.exp(x - mx) for x in row]
            z = sum(e)
            ref = [sum(e[j] / z * v[0, j, h, x] for j in range(i + 1)) for x in range(d)]
            np.testing.assert_allclose(out[0, i, h], ref, rtol=0, atol=1e-12)


def test_group_norm_matches_torch():
    """Per-(token, head) group normalisation = torch group_norm with H groups over
    the D = H*d channels, affine gamma/beta, then the depth scale."""
    T, H, d = 9, 4, 6
    o = rand((T, H, d), 41, 3.0) + 2.0
    gamma, beta = 1 + rand((H * d,), 42, 0.1), rand((H * d,), 43, 0.1)
    lam, eps = 0.97814, 1e-5
    y = O.group_norm_scale(o, gamma, beta, eps, lam).reshape(T, H * d)
    ref = torch.nn.functional.group_norm(torch.from_numpy(o.reshape(T, H * d)), H,
                                         torch.from_numpy(gamma), torch.from_numpy(beta),
                                         eps).numpy() * lam
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def test_depth_scale_values():
    """The depth scale at the layer the workloads use (layer 12: 0.978141, the
    value the workload description states to six digits), its value 0.2 at the
    first layer, and its rise towards 1 with depth."""
    assert abs(O.depth_scale(12) - 0.978141) < 5e-7
    assert abs(O.depth_scale(0) - 0.2) < 1e-15
    vals = [O.depth_scale(n) for n in range(40)]
    assert all(b > a for a, b in zip(vals, vals[1:])) and 1 - vals[-1] < 1e-5


def test_group_norm_invariants():
    T, H, d = 5, 3, 16
    o = rand((T, H, d), 44, 2.0)
    eps = 1e-5
    y = O.group_norm_scale(o, np.ones(H * d), np.zeros(H * d), eps, 1.0)
    np.testing.assert_allclose(y.mean(-1), 0.0, atol=1e-12)
    var = o.var(-1)
    np.testing.assert_allclose(y.var(-1), var / (var + eps), rtol=1e-12)


def test_rows_match_full(qkv):
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 51, 0.3)
    w = rand((H // 2, 2, 2), 52)
    rows = [(0, 0), (0, 1), (1, 2), (1, 7), (0, 22)]
    for hp in (O.PRE, O.POST, O.OFF):
        full = O.mta_attention(q, k, v, th, w, 2, O.PRE, hp)
        part = O.mta_attention_rows(q, k, v, th, w, 2, rows, O.PRE, hp)
        for n, (b, i) in enumerate(rows):
            np.testing.assert_allclose(part[n], full[b, i], rtol=0, atol=1e-12)


def test_layer_matches_library_pipeline():
    """Layer: x W_qkv^T -> MTA attention -> torch group_norm * lambda -> Y W_o^T
    (section 2: projections and output projection; section 3.3: group norm)."""
    B, L, H, d, ch = 2, 11, 4, 4, 2
    D = H * d
    x = rand((B, L, D), 61)
    wqkv, wo = rand((3 * D, D), 62, 0.3), rand((D, D), 63, 0.3)
    th, w = rand((H, 3, 5), 64, 0.3), rand((H // ch, ch, ch), 65)
    gamma, beta = 1 + rand((D,), 66, 0.1), rand((D,), 67, 0.1)
    lam, eps = 0.9, 1e-5
    out = O.mta_layer(x, wqkv, th, w, gamma, beta, eps, lam, wo, H, ch, O.PRE, O.POST)
    qkv = np.einsum("bld,ed->ble", x, wqkv)
    q, k, v = (qkv[..., i * D:(i + 1) * D].reshape(B, L, H, d) for i in range(3))
    att = O.mta_attention(q, k, v, th, w, ch, O.PRE, O.POST).reshape(B * L, D)
    y = torch.nn.functional.group_norm(torch.from_numpy(att), H, torch.from_numpy(gamma),
                                       torch.from_numpy(beta), eps).numpy() * lam
    ref = (y @ wo.T).reshape(B, L, D)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-11)
    rows = [(0, 0), (1, 5), (1, 10)]
    part = O.mta_layer_rows(x, wqkv, th, w, gamma, beta, eps, lam, wo, H, ch, rows,
                            O.PRE, O.POST)
    for n, (b, i) in enumerate(rows):
        np.testing.assert_allclose(part[n], out[b, i], rtol=0, atol=1e-11)


# ---------------------------------------------------------------------------
# exact causal indicator (the variant section 3.1 contrasts with Mask_0)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("a", [1, 2])
def test_exact_indicator_query_shift_closed_form(qkv, a):
    """theta = delta at (a, 0) with the exact indicator: C[i,j] = s q[i-a].k[j] for
    every causal j <= i (keys after the shifted query i-a are kept, unlike Mask_0),
    and 0 when i-a < 0."""
    q, k, v = qkv
    B, L, H, d = q.shape
    cq, ck = 3, 5
    s = 1 / np.sqrt(d)
    th = delta_theta(H, cq, ck, a, ck // 2)
    out = O.mta_attention(q, k, v, th, np.tile(np.eye(1), (H, 1, 1)), 1, O.PRE_EXACT, O.OFF)
    for b, h in [(0, 2), (1, 0)]:
        qq, kk, vv = q[b, :, h], k[b, :, h], v[b, :, h]
        fn = lambda i, j: s * qq[i - a] @ kk[j] if i - a >= 0 else 0.0
        np.testing.assert_allclose(out[b, :, h], _closed_form_attention(qq, kk, vv, fn, s),
                                   rtol=0, atol=1e-12)


@pytest.mark.parametrize("boff", [-2, 1])
def test_exact_indicator_key_shift_closed_form(qkv, boff):
    """theta = delta at (1, b) with the exact indicator: C[i,j] = s q[i-1].k[j-b]
    when 0 <= j-b <= i (the key may lie after the shifted query i-1)."""
    q, k, v = qkv
    B, L, H, d = q.shape
    cq, ck = 2, 5
    s = 1 / np.sqrt(d)
    th = delta_theta(H, cq, ck, 1, ck // 2 + boff)
    out = O.mta_attention(q, k, v, th, np.tile(np.eye(1), (H, 1, 1)), 1, O.PRE_EXACT, O.OFF)
    for b, h in [(0, 3), (1, 1)]:
        qq, kk, vv = q[b, :, h], k[b, :, h], v[b, :, h]
        fn = lambda i, j: s * qq[i - 1] @ kk[j - boff] if (i >= 1 and 0 <= j - boff <= i) else 0.0
        np.testing.assert_allclose(out[b, :, h], _closed_form_attention(qq, kk, vv, fn, s),
                                   rtol=0, atol=1e-12)


def test_exact_indicator_equals_mask0_for_one_query_row(qkv):
    """With c_q = 1 the shifted query is the output query, so the two masks agree."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 1, 5), 31, 0.4)
    w = rand((H // 2, 2, 2), 32, 0.5)
    a = O.mta_attention(q, k, v, th, w, 2, O.PRE, O.POST)
    b = O.mta_attention(q, k, v, th, w, 2, O.PRE_EXACT, O.POST)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_exact_indicator_differs_from_mask0_only_near_the_diagonal():
    """The two convolutions differ only where a tap reads a key after the shifted
    query but not after the output query: 0 <= i-j < (c_q-1) + c."""
    cq, ck, L = 4, 5, 20
    c = ck // 2
    a_hat = rand((1, L, L), 33)
    th = rand((1, cq, ck), 34)
    qpos = np.arange(L)
    m0 = O.key_query_conv(O.mask_zero(a_hat, qpos), th)[0]
    ex = O.key_query_conv_exact(a_hat, th, qpos)[0]
    i, j = np.indices((L, L))
    band = (i - j >= 0) & (i - j < cq - 1 + c)
    causal = j <= i
    np.testing.assert_array_equal(ex[causal & ~band], m0[causal & ~band])
    assert np.abs(ex[band] - m0[band]).max() > 1e-3


@pytest.mark.parametrize("head_place", [O.PRE, O.POST])
def test_exact_indicator_causality_bit_exact(qkv, head_place):
    """The exact indicator still reads nothing after the output query."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 35, 0.3)
    w = rand((H // 2, 2, 2), 36, 0.5)
    base = O.mta_attention(q, k, v, th, w, 2, O.PRE_EXACT, head_place)
    t = 11
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, t:] += rand(q2[:, t:].shape, 37)
    k2[:, t:] += rand(k2[:, t:].shape, 38)
    v2[:, t:] += rand(v2[:, t:].shape, 39)
    pert = O.mta_attention(q2, k2, v2, th, w, 2, O.PRE_EXACT, head_place)
    assert np.array_equal(base[:, :t], pert[:, :t])
    assert not np.allclose(base[:, t:], pert[:, t:])


# ---------------------------------------------------------------------------
# sigmoid scalar gate (section 3.3)
# ---------------------------------------------------------------------------

def test_sigmoid_gate_values():
    """sigmoid(0) = 1/2, sigmoid(-g) = 1 - sigmoid(g), bounded in (0, 1)."""
    g = np.array([-30.0, -2.0, 0.0, 0.5, 3.0, 30.0])
    m = O.sigmoid_gate(g)
    assert m[2] == 0.5
    np.testing.assert_allclose(O.sigmoid_gate(-g), 1.0 - m, rtol=0, atol=1e-15)
    assert np.all(m > 0) and np.all(m < 1)
    np.testing.assert_allclose(m, scipy.special.expit(g), rtol=1e-15)


def test_gated_group_norm_invariants():
    """With gamma = 1, beta = 0 each (token, head) output has mean 0 and standard
    deviation sigmoid(g_h) * sqrt(var / (var + eps)): the gate scales head h alone."""
    T, H, d = 6, 4, 16
    o = rand((T, H, d), 45, 1.5)
    g = np.array([-1.0, 0.0, 0.7, 2.5])
    eps = 1e-5
    y = O.group_norm_scale(o, np.ones(H * d), np.zeros(H * d), eps, O.sigmoid_gate(g))
    np.testing.assert_allclose(y.mean(-1), 0.0, atol=1e-12)
    var = o.var(-1)
    np.testing.assert_allclose(y.std(-1), scipy.special.expit(g)[None, :] * np.sqrt(var / (var + eps)),
                               rtol=1e-12)


# ----------------------------------------------------------------------------
# post-softmax key-query convolution (section 3.1: the kernel acts before or
# after the softmax; after it, it combines attention weights additively)
# ----------------------------------------------------------------------------

def _softmax_weights(q, k, scale):
    """Causal softmax weights of one head by torch's library routine.  q,k [L,d]."""
    L = q.shape[0]
    lg = torch.from_numpy(scale * (q @ k.T))
    lg = lg.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
    return torch.softmax(lg, dim=1).numpy()


def test_post_conv_identity_is_no_op(qkv):
    """theta_post = delta at (0,0) leaves the attention unchanged."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 61, 0.3)
    w = rand((H // 2, 2, 2), 62)
    for hp in (O.OFF, O.PRE, O.POST):
        base = O.mta_attention(q, k, v, th, w, 2, O.PRE, hp)
        ident = O.mta_attention(q, k, v, th, w, 2, O.PRE, hp,
                                theta_post=delta_theta(H, 3, 5, 0, 2))
        np.testing.assert_allclose(ident, base, rtol=0, atol=1e-13)


@pytest.mark.parametrize("a", [1, 3])
def test_post_conv_query_shift_moves_output_rows(qkv, a):
    """theta_post = delta at (a, 0): A'[i] = A[i-a] (row i-a never reaches a key
    after i, so the final Mask_0 removes nothing), hence the output at i is the
    output the plain map gives at i-a, and 0 for i < a; with post-softmax mixing
    the mixed rows move the same way."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 63, 0.3)
    w = rand((H // 2, 2, 2), 64)
    for hp in (O.OFF, O.POST):
        base = O.mta_attention(q, k, v, th, w, 2, O.PRE, hp)
        out = O.mta_attention(q, k, v, th, w, 2, O.PRE, hp, theta_post=delta_theta(H, 4, 5, a, 2))
        np.testing.assert_allclose(out[:, a:], base[:, :-a], rtol=0, atol=1e-13)
        assert np.all(out[:, :a] == 0.0)


@pytest.mark.parametrize("boff", [-2, 1, 2])
def test_post_conv_key_shift_closed_form(qkv, boff):
    """theta_post = delta at (0, b): A'[i][j] = A[i][j-b] for keys j <= i, so
    out[i] = sum over keys j' with 0 <= j'+b <= i of A[i][j'] v[j'+b]: the weights
    move b keys later (b > 0: the last b weights of the row fall past the query
    and are dropped) or |b| keys earlier (b < 0: the first |b| fall off the
    sequence).  A from torch's softmax, the sum by loops."""
    q, k, v = qkv
    B, L, H, d = q.shape
    ck = 5
    th_post = delta_theta(H, 2, ck, 0, ck // 2 + boff)
    out = O.mta_attention(q, k, v, None, None, 1, O.OFF, O.OFF, theta_post=th_post)
    for b in range(B):
        for h in range(H):
            A = _softmax_weights(q[b, :, h], k[b, :, h], 1 / np.sqrt(d))
            ref = np.zeros((L, d))
            for i in range(L):
                for jp in range(L):
                    if 0 <= jp + boff <= i:
                        ref[i] += A[i, jp] * v[b, jp + boff, h]
            np.testing.assert_allclose(out[b, :, h], ref, rtol=0, atol=1e-12)


def test_post_conv_is_linear_in_theta_post(qkv):
    """After the softmax the convolution combines weights additively (section 3.1):
    the output is linear in theta_post."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 65, 0.3)
    w = rand((H // 2, 2, 2), 66)
    t1, t2 = rand((H, 3, 5), 67), rand((H, 3, 5), 68)
    f = lambda tp: O.mta_attention(q, k, v, th, w, 2, O.PRE, O.POST, theta_post=tp)
    np.testing.assert_allclose(f(t1 + t2), f(t1) + f(t2), rtol=0, atol=1e-11)
    np.testing.assert_allclose(f(-2.5 * t1), -2.5 * f(t1), rtol=0, atol=1e-11)


@pytest.mark.parametrize("head_place", [O.OFF, O.PRE, O.POST])
def test_post_conv_causality_bit_exact(qkv, head_place):
    """With the convolution on both sides of the softmax, perturbing position t
    still leaves outputs at i < t bit-identical."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 69, 0.3)
    tp = rand((H, 3, 5), 70, 0.3)
    w = rand((H // 2, 2, 2), 71, 0.5)
    base = O.mta_attention(q, k, v, th, w, 2, O.PRE, head_place, theta_post=tp)
    t = 11
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, t:] += rand(q2[:, t:].shape, 72)
    k2[:, t:] += rand(k2[:, t:].shape, 73)
    v2[:, t:] += rand(v2[:, t:].shape, 74)
    pert = O.mta_attention(q2, k2, v2, th, w, 2, O.PRE, head_place, theta_post=tp)
    assert np.array_equal(base[:, :t], pert[:, :t])
    assert not np.allclose(base[:, t:], pert[:, t:])


def test_both_sides_bruteforce_tiny():
    """Pure-Python restatement on a tiny case: pre-softmax convolution of the
    Mask_0 logits, softmax over past keys, post-softmax convolution of the weights
    with the future keys zeroed again, post-softmax head mixing, times the
    destination head's V; every sum an explicit loop."""
    L, H, d, cq, ck, ch = 7, 2, 3, 3, 3, 2
    c = ck // 2
    q, k, v = rand((1, L, H, d), 75), rand((1, L, H, d), 76), rand((1, L, H, d), 77)
    th, tp = rand((H, cq, ck), 78, 0.5), rand((H, cq, ck), 79, 0.5)
    w = rand((1, ch, ch), 80)
    s = 1 / np.sqrt(d)

    def m0(h, i, j):
        if i < 0 or j < 0 or j >= L or j > i:
            return 0.0
        return s * sum(q[0, i, h, e] * k[0, j, h, e] for e in range(d))

    A = np.zeros((H, L, L))
    for h in range(H):
        for i in range(L):
            C = [sum(th[h, a, t] * m0(h, i - a, j - (t - c)) for a in range(cq) for t in range(ck))
                 for j in range(i + 1)]
            mx = max(C)
            e = [np.exp(x - mx) for x in C]
            for j in range(i + 1):
                A[h, i, j] = e[j] / sum(e)

    def a_at(h, i, j):
        return A[h, i, j] if 0 <= i < L and 0 <= j < L else 0.0

    Ap = np.zeros((H, L, L))
    for h in range(H):
        for i in range(L):
            for j in range(i + 1):
                Ap[h, i, j] = sum(tp[h, a, t] * a_at(h, i - a, j - (t - c))
                                  for a in range(cq) for t in range(ck))
    ref = np.zeros((1, L, H, d))
    for r in range(H):
        for i in range(L):
            for j in range(L):
                wt = sum(w[0, r, s_] * Ap[s_, i, j] for s_ in range(H))
                ref[0, i, r] += wt * v[0, j, r]
    out = O.mta_attention(q, k, v, th, w, ch, O.PRE, O.POST, theta_post=tp)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_post_conv_rows_match_full(qkv):
    """The row-wise oracle widens its query window to 2 c_q - 1 rows when the
    convolution also acts after the softmax."""
    q, k, v = qkv
    H = q.shape[2]
    th = rand((H, 3, 5), 81, 0.3)
    tp = rand((H, 3, 5), 82, 0.3)
    w = rand((H // 2, 2, 2), 83)
    rows = [(0, 0), (0, 3), (1, 4), (1, 9), (0, 22)]
    for kq in (O.PRE, O.OFF):
        for hp in (O.PRE, O.POST, O.OFF):
            full = O.mta_attention(q, k, v, th, w, 2, kq, hp, theta_post=tp)
            part = O.mta_attention_rows(q, k, v, th, w, 2, rows, kq, hp, theta_post=tp)
            for n, (b, i) in enumerate(rows):
                np.testing.assert_allclose(part[n], full[b, i], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# backward pass: pinned to central finite differences of the forward, and to
# torch's autograd of its causal attention for identity kernels
# ----------------------------------------------------------------------------

def _fd_check(kq, hp, post, seed):
    B, L, H, d, cq, ck, ch = 1, 7, 2, 3, 3, 3, 2
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, L, H, d)) for _ in range(3))
    th = rng.standard_normal((H, cq, ck)) * 0.5
    tp = rng.standard_normal((H, cq, ck)) * 0.5 if post else None
    w = rng.standard_normal((1, ch, ch))
    dout = rng.standard_normal((B, L, H, d))
    hpl = hp if hp != O.OFF else O.OFF

    def f(q_, k_, v_, th_, w_, tp_):
        o = O.mta_attention(q_, k_, v_, th_, w_, ch, kq, hpl, theta_post=tp_)
        return float(np.sum(o * dout))

    g = O.mta_attention_bwd(q, k, v, th, w, ch, dout, kq, hpl, theta_post=tp)
    base = dict(q_=q, k_=k, v_=v, th_=th, w_=w, tp_=tp)
    checks = [("q_", "dq"), ("k_", "dk"), ("v_", "dv")]
    if kq != O.OFF:
        checks.append(("th_", "dtheta"))
    if hp != O.OFF:
        checks.append(("w_", "dw"))
    if post:
        checks.append(("tp_", "dtheta_post"))
    eps = 1e-6
    for name, gname in checks:
        for rep in range(2):
            u = rng.standard_normal(base[name].shape)
            plus = dict(base); plus[name] = base[name] + eps * u
            minus = dict(base); minus[name] = base[name] - eps * u
            fd = (f(**plus) - f(**minus)) / (2 * eps)
            an = float(np.sum(g[gname] * u))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (kq, hp, post, gname, fd, an)


@pytest.mark.parametrize("kq", [O.OFF, O.PRE, O.PRE_EXACT])
@pytest.mark.parametrize("hp", [O.OFF, O.PRE, O.POST])
@pytest.mark.parametrize("post", [False, True])
def test_backward_matches_finite_differences(kq, hp, post):
    """Every gradient (q, k, v, the kernels, the mixing weights) against central
    differences of the forward, along random directions."""
    _fd_check(kq, hp, post, seed=900 + 7 * kq + 3 * hp + post)


def test_backward_identity_kernels_equal_torch_autograd():
    """theta = delta(0,0), w = I: the gradients are those of causal softmax
    attention, taken here by torch's autograd through its SDPA routine."""
    B, L, H, d, cq, ck, ch = 2, 11, 4, 5, 3, 5, 2
    rng = np.random.default_rng(5)
    q, k, v, dout = (rng.standard_normal((B, L, H, d)) for _ in range(4))
    th = delta_theta(H, cq, ck, 0, ck // 2)
    w = np.tile(np.eye(ch), (H // ch, 1, 1))
    g = O.mta_attention_bwd(q, k, v, th, w, ch, dout, O.PRE, O.POST)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x.transpose(0, 2, 1, 3))).requires_grad_(True)
    tq, tk, tv = t(q), t(k), t(v)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=1 / np.sqrt(d))
    o.backward(torch.from_numpy(np.ascontiguousarray(dout.transpose(0, 2, 1, 3))))
    for name, tt in (("dq", tq), ("dk", tk), ("dv", tv)):
        np.testing.assert_allclose(g[name], tt.grad.numpy().transpose(0, 2, 1, 3), rtol=0, atol=1e-12)
    # the kernel gradient of the identity kernel's centre tap is the logits' own gradient . logits
    assert g["dtheta"].shape == (H, cq, ck)


# ----------------------------------------------------------------------------
# backward of the full layer: central finite differences of mta_layer, and the
# group norm's backward against torch's autograd of its group_norm routine
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("hp,post,gated", [(O.POST, False, False), (O.PRE, False, False),
                                           (O.POST, True, False), (O.POST, False, True)])
def test_layer_backward_matches_finite_differences(hp, post, gated):
    """Every gradient of the layer (x, Wqkv, Wo, the kernels, the mixing weights,
    gamma, beta and the gate logits) against central differences of the forward
    along random directions."""
    B, L, H, d, cq, ck, ch = 1, 6, 2, 3, 3, 3, 2
    D = H * d
    rng = np.random.default_rng(950 + hp + 2 * post + 4 * gated)
    x = rng.standard_normal((B, L, D))
    wqkv = rng.standard_normal((3 * D, D)) * 0.4
    wo = rng.standard_normal((D, D)) * 0.4
    th = rng.standard_normal((H, cq, ck)) * 0.5
    tp = rng.standard_normal((H, cq, ck)) * 0.5 if post else None
    w = rng.standard_normal((1, ch, ch))
    gamma = 1 + 0.2 * rng.standard_normal(D)
    beta = 0.2 * rng.standard_normal(D)
    gate = rng.standard_normal(H) if gated else None
    eps, lam = 1e-5, 0.8
    dout = rng.standard_normal((B, L, D))

    def f(x_, wqkv_, wo_, th_, w_, tp_, gamma_, beta_, gate_):
        mult = O.sigmoid_gate(gate_) if gate_ is not None else lam
        out = O.mta_layer(x_, wqkv_, th_, w_, gamma_, beta_, eps, mult, wo_, H, ch, O.PRE, hp,
                          theta_post=tp_)
        return float(np.sum(out * dout))

    g = O.mta_layer_bwd(x, wqkv, th, w, gamma, beta, eps, lam, wo, H, ch, dout, O.PRE, hp,
                        theta_post=tp, gate=gate)
    base = dict(x_=x, wqkv_=wqkv, wo_=wo, th_=th, w_=w, tp_=tp, gamma_=gamma, beta_=beta, gate_=gate)
    checks = [("x_", "dx"), ("wqkv_", "dwqkv"), ("wo_", "dwo"), ("th_", "dtheta"), ("w_", "dw"),
              ("gamma_", "dgamma"), ("beta_", "dbeta")]
    if post:
        checks.append(("tp_", "dtheta_post"))
    if gated:
        checks.append(("gate_", "dgate"))
    eps_fd = 1e-6
    for name, gname in checks:
        for _ in range(2):
            u = rng.standard_normal(base[name].shape)
            plus = dict(base); plus[name] = base[name] + eps_fd * u
            minus = dict(base); minus[name] = base[name] - eps_fd * u
            fd = (f(**plus) - f(**minus)) / (2 * eps_fd)
            an = float(np.sum(g[gname] * u))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (hp, post, gated, gname, fd, an)


def test_group_norm_backward_matches_torch_autograd():
    T, H, d = 7, 3, 8
    rng = np.random.default_rng(61)
    o = rng.standard_normal((T, H, d)) * 2 + 0.5
    gamma, beta = 1 + 0.1 * rng.standard_normal(H * d), 0.1 * rng.standard_normal(H * d)
    dy = rng.standard_normal((T, H, d))
    lam, eps = 0.9, 1e-5
    do, dgamma, dbeta, _ = O.group_norm_scale_bwd(o, gamma, beta, eps, lam, dy)
    to = torch.from_numpy(o.reshape(T, H * d)).requires_grad_(True)
    tg = torch.from_numpy(gamma).requires_grad_(True)
    tb = torch.from_numpy(beta).requires_grad_(True)
    y = torch.nn.functional.group_norm(to, H, tg, tb, eps) * lam
    y.backward(torch.from_numpy(dy.reshape(T, H * d)))
    np.testing.assert_allclose(do.reshape(T, H * d), to.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dgamma, tg.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dbeta, tb.grad.numpy(), rtol=0, atol=1e-10)
