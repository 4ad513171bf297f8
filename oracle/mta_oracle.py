"""fp64 CPU oracle of the Multi-Token Attention (MTA) forward pass.

TEST INFRASTRUCTURE ONLY.  Imported by tests/, by __graft_entry__.smoke() and by
the CPU-baseline leg of bench.py; the library (token_attention_b200) never
imports, links or runs anything here, and nothing here imports the library.

It is the plain definition written out: the full L x L logit, convolution and
attention maps are materialised per head group in float64 and every step is a
separate array operation, in the order the pages give it.  Sources (page title,
section):

  [MTA-2]   "Multi-Token Attention | Summary" (greeksharifa), section 2
            "Background on multi-head attention": per-head Q, K, V; logits
            A_hat = Q K^T / sqrt(d); causal -inf mask; softmax over keys; A V;
            concatenation; output projection.
  [MTA-3.1] same page, section 3.1 "Key-query convolution":
            A = Softmax(Mask_-inf(Conv2d_theta(Mask_0(A_hat)))), a separate 2-D
            kernel per head over (query, key) offsets, using only the current and
            previous queries.
  [MTA-3.2] same page, section 3.2 "Head mixing convolution": heads split into
            M/c_h groups; A1_new = w11 A1 + w12 A2, ...; applied to logits
            (before softmax) or to attention weights (after softmax).
  [MTA-3.3] same page, section 3.3 "Putting everything together": both on the
            same side of the softmax = one 3-D convolution; group normalisation
            of head outputs before concatenation, with a scale.
  [MTA-B]   same page, appendix B "MTA Architecture": post-softmax mixing acts
            through the value/output projections.
  [bycloud] "Multi-Token Attention" (bycloud), "Understanding Multi-Token
            Attention (MTA) Mechanism", item 3: group normalisation with depth
            scaling.

Readings where the pages leave a step open:
  * Mask_0 zeroes logits of future keys (key j > query i) before the
    convolution; indices outside [0, L) contribute 0 (zero padding).
  * theta[h][a][t] multiplies Mask_0(A_hat)[i - a][j - (t - c_k//2)]:
    a = 0..c_q-1 steps back over queries, t over keys centred on j.  No bias.
  * Pre-softmax head mixing is applied after the key-query convolution.
  * Post-softmax mixing is a plain linear combination (no renormalisation) and
    the mixed map of head r multiplies head r's own values.
  * Group norm: per (token, head) over the d channels, biased variance,
    eps, affine gamma/beta of length D; then times lambda.
  * Exact causal indicator (the variant section 3.1 contrasts with Mask_0: the
    simpler mask "removes slightly more information than necessary"): a tap of
    the convolution at output (i, j) reads A_hat[i - a][j - b] whenever its key
    j - b is not after the output query i, even if it is after the shifted
    query i - a.  Outputs stay causal (nothing after i is read).
  * Sigmoid scalar gate (section 3.3: "a learned sigmoid scalar gate, a bounded
    multiplier"): one learned logit g_h per head; the normalised output of head h
    is multiplied by sigmoid(g_h) in place of the depth scale.
  * Post-softmax key-query convolution (section 3.1 applies the kernel "before
    or after" the softmax; section 4 uses both by default, and only the
    pre-softmax formula is printed): its own per-head kernel theta_post of the
    same c_q x c_k shape convolves the attention weights A (already 0 at future
    keys), then Mask_0 zeroes the future keys again, so
    A' = Mask_0(Conv2d_theta_post(A)); no renormalisation.  With head mixing
    after the softmax, the convolution comes first, as before the softmax.
"""
from __future__ import annotations

import numpy as np

OFF, PRE, POST, PRE_EXACT = 0, 1, 2, 3

__all__ = ["OFF", "PRE", "POST", "PRE_EXACT", "attention_logits", "mask_zero", "key_query_conv",
           "key_query_conv_exact", "sigmoid_gate", "post_softmax_conv",
           "head_mix", "mask_neg_inf", "softmax_rows", "mta_attention_group",
           "mta_attention", "mta_attention_rows", "depth_scale", "group_norm_scale", "mta_layer",
           "key_query_conv_adjoint", "key_query_conv_grad_theta", "mta_attention_group_bwd",
           "mta_attention_bwd",
           "mta_layer_rows", "group_norm_scale_bwd", "mta_layer_bwd"]


# ----------------------------------------------------------------------------
# the steps, each on arrays of one head group: [c_h, rows, keys]
# ----------------------------------------------------------------------------

def attention_logits(q_rows: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """A_hat[h, r, j] = scale * q[h, r] . k[h, j]   [MTA-2].

    q_rows [c_h, R, d], k [c_h, L, d] -> [c_h, R, L] float64."""
    return scale * np.matmul(q_rows.astype(np.float64), k.astype(np.float64).transpose(0, 2, 1))


def _future(qpos: np.ndarray, L: int) -> np.ndarray:
    """Boolean [R, L]: True where key j lies in the future of query qpos[r]."""
    return np.arange(L)[None, :] > qpos[:, None]


def mask_zero(a: np.ndarray, qpos: np.ndarray) -> np.ndarray:
    """Mask_0: entries with key j > query position qpos[r] become 0  [MTA-3.1]."""
    return np.where(_future(qpos, a.shape[-1])[None], 0.0, a)


def key_query_conv(m: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Conv2d_theta over (query, key) per head  [MTA-3.1].

    m [c_h, R, L]: rows are consecutive queries (row r-1 is the query before
    row r); rows before the first and keys outside [0, L) count as 0.
    theta [c_h, c_q, c_k].
    out[h, r, j] = sum_a sum_t theta[h, a, t] * m[h, r - a, j - (t - c_k//2)].
    """
    ch, R, L = m.shape
    cq, ck = theta.shape[1], theta.shape[2]
    c = ck // 2
    out = np.zeros_like(m, dtype=np.float64)
    for a in range(cq):                       # a queries back
        if a >= R:
            break
        for t in range(ck):
            b = t - c                          # key offset: reads key j - b
            j_lo, j_hi = max(0, b), min(L, L + b)
            if j_lo >= j_hi:
                continue
            coef = theta[:, a, t].astype(np.float64)[:, None, None]
            out[:, a:, j_lo:j_hi] += coef * m[:, :R - a, j_lo - b:j_hi - b]
    return out


def key_query_conv_exact(a_hat: np.ndarray, theta: np.ndarray, qpos: np.ndarray) -> np.ndarray:
    """Conv2d_theta over (query, key) with the exact causal indicator  [MTA-3.1].

    a_hat [c_h, R, L] (unmasked logits; rows are consecutive queries qpos).
    out[h, r, j] = sum_a sum_t theta[h, a, t] * a_hat[h, r - a, j - b] * [j - b <= qpos[r]],
    b = t - c_k//2; rows before the first and keys outside [0, L) count as 0."""
    ch, R, L = a_hat.shape
    cq, ck = theta.shape[1], theta.shape[2]
    c = ck // 2
    out = np.zeros_like(a_hat, dtype=np.float64)
    keys = np.arange(L)
    for a in range(cq):
        if a >= R:
            break
        for t in range(ck):
            b = t - c
            j_lo, j_hi = max(0, b), min(L, L + b)
            if j_lo >= j_hi:
                continue
            shifted = np.zeros((ch, R, L), np.float64)
            shifted[:, a:, j_lo:j_hi] = a_hat[:, :R - a, j_lo - b:j_hi - b]
            allowed = (keys[None, :] - b) <= np.asarray(qpos)[:, None]       # [R, L]
            coef = theta[:, a, t].astype(np.float64)[:, None, None]
            out += coef * np.where(allowed[None], shifted, 0.0)
    return out


def sigmoid_gate(gate: np.ndarray) -> np.ndarray:
    """The bounded per-head multiplier sigmoid(g) of the scalar gate  [MTA-3.3]."""
    return 1.0 / (1.0 + np.exp(-np.asarray(gate, np.float64)))


def head_mix(a: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Within-group linear combination: out[r] = sum_s w[r, s] * a[s]  [MTA-3.2]."""
    return np.einsum("rs,s...->r...", w.astype(np.float64), a)


def mask_neg_inf(c: np.ndarray, qpos: np.ndarray) -> np.ndarray:
    """Mask_-inf: entries with key j > query qpos[r] become -inf  [MTA-2, MTA-3.1]."""
    return np.where(_future(qpos, c.shape[-1])[None], -np.inf, c)


def softmax_rows(c: np.ndarray) -> np.ndarray:
    """Softmax over keys (last axis)  [MTA-2]."""
    mx = np.max(c, axis=-1, keepdims=True)
    e = np.exp(c - mx)
    return e / np.sum(e, axis=-1, keepdims=True)


def post_softmax_conv(attn: np.ndarray, theta_post: np.ndarray, qpos: np.ndarray) -> np.ndarray:
    """Key-query convolution of the attention weights after the softmax, then
    Mask_0 again  [MTA-3.1]: A' = Mask_0(Conv2d_theta_post(A)).  attn [c_h, R, L]
    (rows are the consecutive queries qpos), theta_post [c_h, c_q, c_k]."""
    return mask_zero(key_query_conv(attn, theta_post), qpos)


def mta_attention_group(q_rows, k, v, theta, w, qpos, scale, kq_place, head_place,
                        theta_post=None):
    """MTA attention of one head group for the query rows `qpos` (consecutive).

    q_rows [c_h, R, d] (queries at positions qpos), k, v [c_h, L, d],
    theta [c_h, c_q, c_k], w [c_h, c_h], theta_post [c_h, c_q, c_k] or None (no
    post-softmax convolution).  Returns [c_h, R, d] float64.
    Steps in the pages' order [MTA-2, MTA-3.1, MTA-3.2, MTA-3.3]."""
    qpos = np.asarray(qpos)
    a_hat = attention_logits(q_rows, k, scale)
    if kq_place == PRE:
        c = key_query_conv(mask_zero(a_hat, qpos), theta)
    elif kq_place == PRE_EXACT:
        c = key_query_conv_exact(a_hat, theta, qpos)
    else:
        c = a_hat
    if head_place == PRE:
        c = head_mix(c, w)
    attn = softmax_rows(mask_neg_inf(c, qpos))
    if theta_post is not None:
        attn = post_softmax_conv(attn, theta_post, qpos)
    if head_place == POST:
        attn = head_mix(attn, w)
    return np.matmul(attn, v.astype(np.float64))        # head r: A_r V_r


# ----------------------------------------------------------------------------
# backward pass of one head group (gradients by the chain rule, each forward
# step taken in reverse order; the pages train with this forward, section 4)
# ----------------------------------------------------------------------------

def key_query_conv_adjoint(g: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Adjoint of key_query_conv in its input: for out = key_query_conv(m, theta),
    d m[h, r', j'] = sum_a sum_t theta[h, a, t] * g[h, r' + a, j' + (t - c_k//2)]
    (entries outside the array count as 0)."""
    ch, R, L = g.shape
    cq, ck = theta.shape[1], theta.shape[2]
    c = ck // 2
    out = np.zeros_like(g, dtype=np.float64)
    for a in range(cq):
        if a >= R:
            break
        for t in range(ck):
            b = t - c
            j_lo, j_hi = max(0, b), min(L, L + b)
            if j_lo >= j_hi:
                continue
            coef = theta[:, a, t].astype(np.float64)[:, None, None]
            out[:, :R - a, j_lo - b:j_hi - b] += coef * g[:, a:, j_lo:j_hi]
    return out


def key_query_conv_grad_theta(g: np.ndarray, m: np.ndarray, cq: int, ck: int) -> np.ndarray:
    """Gradient of key_query_conv in its kernel: d theta[h, a, t] =
    sum_{r, j} g[h, r, j] * m[h, r - a, j - (t - c_k//2)]."""
    ch, R, L = g.shape
    c = ck // 2
    out = np.zeros((ch, cq, ck), np.float64)
    for a in range(cq):
        if a >= R:
            break
        for t in range(ck):
            b = t - c
            j_lo, j_hi = max(0, b), min(L, L + b)
            if j_lo >= j_hi:
                continue
            out[:, a, t] = np.einsum("hrj,hrj->h", g[:, a:, j_lo:j_hi], m[:, :R - a, j_lo - b:j_hi - b])
    return out


def _exact_indicator_terms(a_hat, theta, qpos):
    """The shifted, indicator-masked logits of key_query_conv_exact, one per tap:
    yields (a, t, shifted * [key <= query])."""
    ch, R, L = a_hat.shape
    cq, ck = theta.shape[1], theta.shape[2]
    c = ck // 2
    keys = np.arange(L)
    for a in range(min(cq, R)):
        for t in range(ck):
            b = t - c
            j_lo, j_hi = max(0, b), min(L, L + b)
            if j_lo >= j_hi:
                continue
            allowed = ((keys[None, :] - b) <= np.asarray(qpos)[:, None]).astype(np.float64)
            yield a, t, b, j_lo, j_hi, allowed


def mta_attention_group_bwd(q_rows, k, v, theta, w, qpos, scale, kq_place, head_place, dout,
                            theta_post=None):
    """Gradients of mta_attention_group for all its query rows (qpos = 0 .. L-1).

    dout [c_h, R, d]: gradient of the output.  Returns dict with dq [c_h, R, d],
    dk, dv [c_h, L, d], dtheta [c_h, c_q, c_k] (None if the convolution is off),
    dw [c_h, c_h] (None without head mixing) and dtheta_post (None without the
    post-softmax convolution), all float64."""
    qpos = np.asarray(qpos)
    q64, k64, v64 = (x.astype(np.float64) for x in (q_rows, k, v))
    g_out = dout.astype(np.float64)
    # forward, keeping every intermediate map
    a_hat = attention_logits(q_rows, k, scale)
    if kq_place == PRE:
        m0 = mask_zero(a_hat, qpos)
        c = key_query_conv(m0, theta)
    elif kq_place == PRE_EXACT:
        c = key_query_conv_exact(a_hat, theta, qpos)
    else:
        c = a_hat
    c2 = head_mix(c, w) if head_place == PRE else c
    attn = softmax_rows(mask_neg_inf(c2, qpos))
    attn2 = post_softmax_conv(attn, theta_post, qpos) if theta_post is not None else attn
    attn3 = head_mix(attn2, w) if head_place == POST else attn2
    res = {"dtheta": None, "dw": None, "dtheta_post": None}
    # out[r] = attn3[r] v[r]
    res["dv"] = np.matmul(attn3.transpose(0, 2, 1), g_out)
    d_attn3 = np.matmul(g_out, v64.transpose(0, 2, 1))
    if head_place == POST:                      # attn3[r] = sum_s w[r, s] attn2[s]
        res["dw"] = np.einsum("rij,sij->rs", d_attn3, attn2)
        d_attn2 = np.einsum("rs,rij->sij", w.astype(np.float64), d_attn3)
    else:
        d_attn2 = d_attn3
    if theta_post is not None:                  # attn2 = Mask_0(conv(attn, theta_post))
        g_pre = mask_zero(d_attn2, qpos)
        res["dtheta_post"] = key_query_conv_grad_theta(g_pre, attn, theta_post.shape[1], theta_post.shape[2])
        d_attn = key_query_conv_adjoint(g_pre, theta_post)
    else:
        d_attn = d_attn2
    # softmax over keys: d c2 = attn * (d attn - sum_j d attn * attn); masked keys have attn 0
    dc2 = attn * (d_attn - np.sum(d_attn * attn, axis=-1, keepdims=True))
    if head_place == PRE:                       # c2[r] = sum_s w[r, s] c[s]
        res["dw"] = np.einsum("rij,sij->rs", dc2, c)
        dc = np.einsum("rs,rij->sij", w.astype(np.float64), dc2)
    else:
        dc = dc2
    if kq_place == PRE:                         # c = conv(Mask_0(a_hat), theta)
        res["dtheta"] = key_query_conv_grad_theta(dc, m0, theta.shape[1], theta.shape[2])
        d_a_hat = mask_zero(key_query_conv_adjoint(dc, theta), qpos)
    elif kq_place == PRE_EXACT:                 # c = sum_taps theta * shifted(a_hat) * [key <= query]
        ch, R, L = a_hat.shape
        d_a_hat = np.zeros_like(a_hat)
        dth = np.zeros(theta.shape, np.float64)
        for a, t, b, j_lo, j_hi, allowed in _exact_indicator_terms(a_hat, theta, qpos):
            g = dc * allowed[None]               # gradient reaching the shifted logits
            dth[:, a, t] = np.einsum("hrj,hrj->h", g[:, a:, j_lo:j_hi], a_hat[:, :R - a, j_lo - b:j_hi - b])
            coef = theta[:, a, t].astype(np.float64)[:, None, None]
            d_a_hat[:, :R - a, j_lo - b:j_hi - b] += coef * g[:, a:, j_lo:j_hi]
        res["dtheta"] = dth
    else:
        d_a_hat = dc
    # a_hat = scale q k^T
    res["dq"] = scale * np.matmul(d_a_hat, k64)
    res["dk"] = scale * np.matmul(d_a_hat.transpose(0, 2, 1), q64)
    return res


# ----------------------------------------------------------------------------
# whole tensors in the library's layout: q, k, v, out [B][L][H][d]
# ----------------------------------------------------------------------------

def _group(x: np.ndarray, b: int, g: int, ch: int) -> np.ndarray:
    """[L, H, d] slice of batch b -> heads of group g as [c_h, L, d]."""
    return np.ascontiguousarray(x[b, :, g * ch:(g + 1) * ch, :].transpose(1, 0, 2))


def _sel(x, idx):
    """x[idx], or None for a parameter that is absent (its step is off)."""
    return None if x is None else x[idx]


def _default_scale(d: int, scale) -> float:
    return 1.0 / np.sqrt(d) if not scale else float(scale)


def mta_attention(q, k, v, theta, w, c_h, kq_place=PRE, head_place=POST, scale=None,
                  theta_post=None):
    """Full MTA attention.  q, k, v [B][L][H][d]; theta [H][c_q][c_k];
    w [H/c_h][c_h][c_h]; theta_post [H][c_q][c_k] or None.
    Returns out [B][L][H][d] float64."""
    B, L, H, d = q.shape
    s = _default_scale(d, scale)
    out = np.zeros((B, L, H, d), np.float64)
    qpos = np.arange(L)
    for b in range(B):
        for g in range(H // c_h):
            hs = slice(g * c_h, (g + 1) * c_h)
            og = mta_attention_group(_group(q, b, g, c_h), _group(k, b, g, c_h),
                                     _group(v, b, g, c_h), _sel(theta, hs), _sel(w, g),
                                     qpos, s, kq_place, head_place,
                                     None if theta_post is None else theta_post[hs])
            out[b, :, hs, :] = og.transpose(1, 0, 2)
    return out


def mta_attention_bwd(q, k, v, theta, w, c_h, dout, kq_place=PRE, head_place=POST, scale=None,
                      theta_post=None):
    """Gradients of mta_attention.  q, k, v, dout [B][L][H][d].  Returns dict with
    dq, dk, dv [B][L][H][d], dtheta [H][c_q][c_k] (summed over batches),
    dw [H/c_h][c_h][c_h] and dtheta_post, float64 (None where the step is off)."""
    B, L, H, d = q.shape
    s = _default_scale(d, scale)
    G = H // c_h
    out = {n: np.zeros((B, L, H, d), np.float64) for n in ("dq", "dk", "dv")}
    dth = np.zeros((H,) + theta.shape[1:], np.float64) if theta is not None and kq_place else None
    dw = np.zeros((G, c_h, c_h), np.float64) if head_place else None
    dtp = np.zeros(theta_post.shape, np.float64) if theta_post is not None else None
    qpos = np.arange(L)
    for b in range(B):
        for g in range(G):
            hs = slice(g * c_h, (g + 1) * c_h)
            r = mta_attention_group_bwd(_group(q, b, g, c_h), _group(k, b, g, c_h), _group(v, b, g, c_h),
                                        _sel(theta, hs), _sel(w, g), qpos, s, kq_place, head_place,
                                        _group(dout, b, g, c_h),
                                        None if theta_post is None else theta_post[hs])
            for n in ("dq", "dk", "dv"):
                out[n][b, :, hs, :] = r[n].transpose(1, 0, 2)
            if dth is not None:
                dth[hs] += r["dtheta"]
            if dw is not None:
                dw[g] += r["dw"]
            if dtp is not None:
                dtp[hs] += r["dtheta_post"]
    out["dtheta"], out["dw"], out["dtheta_post"] = dth, dw, dtp
    return out


def mta_attention_rows(q, k, v, theta, w, c_h, rows, kq_place=PRE, head_place=POST,
                       scale=None, theta_post=None):
    """MTA attention output at selected tokens only.

    rows: sequence of (b, i).  Returns [n, H, d] float64.  Each row is computed
    from the window of queries ending at i that the convolutions read (c_q rows,
    2 c_q - 1 with the post-softmax convolution), with exactly the same steps as
    mta_attention."""
    B, L, H, d = q.shape
    cq = 1 if theta is None else theta.shape[1]
    back = cq - 1 + (0 if theta_post is None else theta_post.shape[1] - 1)
    s = _default_scale(d, scale)
    out = np.zeros((len(rows), H, d), np.float64)
    for n, (b, i) in enumerate(rows):
        lo = max(0, i - back)
        qpos = np.arange(lo, i + 1)
        for g in range(H // c_h):
            hs = slice(g * c_h, (g + 1) * c_h)
            qg = np.ascontiguousarray(q[b, lo:i + 1, hs, :].transpose(1, 0, 2))
            og = mta_attention_group(qg, _group(k, b, g, c_h), _group(v, b, g, c_h),
                                     _sel(theta, hs), _sel(w, g), qpos, s, kq_place,
                                     head_place,
                                     None if theta_post is None else theta_post[hs])
            out[n, hs, :] = og[:, -1, :]
    return out


def depth_scale(layer: int) -> float:
    """Depth-dependent multiplier of the normalised head outputs [bycloud, MTA-3.3]:
    lambda = 1 - 0.8 * exp(-0.3 * layer).  The pages name the scaling without a
    formula; this form (the Differential-Transformer one) is the workload's reading."""
    return 1.0 - 0.8 * np.exp(-0.3 * float(layer))


def group_norm_scale(o, gamma, beta, eps, lam):
    """Per-(token, head) normalisation over d, affine, then depth scale
    [MTA-3.3, bycloud].  o [..., H, d]; gamma, beta [H*d]; lam a scalar (depth
    scale) or a per-head [H] multiplier (the sigmoid gate).  Returns float64."""
    o = o.astype(np.float64)
    H, d = o.shape[-2], o.shape[-1]
    mu = np.mean(o, axis=-1, keepdims=True)
    var = np.mean((o - mu) ** 2, axis=-1, keepdims=True)
    y = (o - mu) / np.sqrt(var + eps)
    y = y * gamma.astype(np.float64).reshape(H, d) + beta.astype(np.float64).reshape(H, d)
    lam = np.asarray(lam, np.float64)
    return (lam.reshape(H, 1) if lam.ndim else lam) * y


def _split_qkv(qkv, H, d):
    D = H * d
    shp = qkv.shape[:-1] + (H, d)
    return (qkv[..., :D].reshape(shp), qkv[..., D:2 * D].reshape(shp),
            qkv[..., 2 * D:].reshape(shp))


def mta_layer(x, wqkv, theta, w, gamma, beta, eps, lam, wo, H, c_h,
              kq_place=PRE, head_place=POST, theta_post=None):
    """Full MTA attention layer  [MTA-2, MTA-3.x, bycloud].
    x [B][L][D]; wqkv [3D][D]; wo [D][D].  Returns out [B][L][D] float64."""
    B, L, D = x.shape
    d = D // H
    qkv = np.matmul(x.astype(np.float64), wqkv.astype(np.float64).T)      # x W^T
    q, k, v = _split_qkv(qkv, H, d)
    o = mta_attention(q, k, v, theta, w, c_h, kq_place, head_place, theta_post=theta_post)
    y = group_norm_scale(o, gamma, beta, eps, lam).reshape(B, L, D)
    return np.matmul(y, wo.astype(np.float64).T)


def group_norm_scale_bwd(o, gamma, beta, eps, lam, dy, gate=None):
    """Gradients of group_norm_scale  [MTA-3.3, bycloud]: given dy = dL/dy,
    returns (do, dgamma [H*d], dbeta [H*d], dgate [H] or None).  lam is the depth
    scale (a scalar, no gradient); with gate logits the multiplier of head h is
    sigmoid(gate[h]) and dgate is its gradient.  Chain rule of
    y = m_h * (xhat * gamma + beta), xhat = (o - mean) / sqrt(var + eps), biased var."""
    o = o.astype(np.float64)
    dy = dy.astype(np.float64)
    H, d = o.shape[-2], o.shape[-1]
    g = gamma.astype(np.float64).reshape(H, d)
    b = beta.astype(np.float64).reshape(H, d)
    mu = np.mean(o, axis=-1, keepdims=True)
    var = np.mean((o - mu) ** 2, axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (o - mu) * rstd
    m = sigmoid_gate(gate).reshape(H, 1) if gate is not None else np.asarray(lam, np.float64)
    lead = tuple(range(o.ndim - 2))
    dgamma = np.sum(m * dy * xhat, axis=lead).reshape(H * d)
    dbeta = np.sum(m * dy, axis=lead).reshape(H * d)
    dgate = None
    if gate is not None:
        sg = sigmoid_gate(gate)
        dgate = np.sum(dy * (xhat * g + b), axis=lead + (o.ndim - 1,)) * sg * (1.0 - sg)
    dxhat = m * dy * g
    do = rstd * (dxhat - np.mean(dxhat, axis=-1, keepdims=True)
                 - xhat * np.mean(dxhat * xhat, axis=-1, keepdims=True))
    return do, dgamma, dbeta, dgate


def mta_layer_bwd(x, wqkv, theta, w, gamma, beta, eps, lam, wo, H, c_h, dout,
                  kq_place=PRE, head_place=POST, theta_post=None, gate=None):
    """Gradients of mta_layer  [MTA-2, MTA-3.x, bycloud], each step of the forward
    taken in reverse: out = Y Wo^T, Y = group norm (depth scale or gate) of the
    attention output, attention as mta_attention_bwd, QKV = x Wqkv^T.
    dout [B][L][D].  Returns dict with dx [B][L][D], dwqkv [3D][D], dwo [D][D],
    dtheta, dw, dtheta_post (as mta_attention_bwd), dgamma, dbeta [D] and dgate [H]
    (None without a gate), float64.  With a gate, lam is ignored."""
    B, L, D = x.shape
    d = D // H
    x64 = x.astype(np.float64)
    qkv = np.matmul(x64, wqkv.astype(np.float64).T)
    q, k, v = _split_qkv(qkv, H, d)
    o = mta_attention(q, k, v, theta, w, c_h, kq_place, head_place, theta_post=theta_post)
    mult = sigmoid_gate(gate) if gate is not None else lam
    y = group_norm_scale(o, gamma, beta, eps, mult).reshape(B, L, D)
    g_out = dout.astype(np.float64)
    dy = np.matmul(g_out, wo.astype(np.float64)).reshape(B, L, H, d)         # out = y Wo^T
    dwo = np.matmul(g_out.reshape(-1, D).T, y.reshape(-1, D))
    do, dgamma, dbeta, dgate = group_norm_scale_bwd(o, gamma, beta, eps, lam, dy, gate)
    ga = mta_attention_bwd(q, k, v, theta, w, c_h, do, kq_place, head_place, theta_post=theta_post)
    dqkv = np.concatenate([ga[n].reshape(B, L, D) for n in ("dq", "dk", "dv")], axis=-1)
    dx = np.matmul(dqkv, wqkv.astype(np.float64))                            # qkv = x Wqkv^T
    dwqkv = np.matmul(dqkv.reshape(-1, 3 * D).T, x64.reshape(-1, D))
    return {"dx": dx, "dwqkv": dwqkv, "dwo": dwo, "dtheta": ga["dtheta"], "dw": ga["dw"],
            "dtheta_post": ga["dtheta_post"], "dgamma": dgamma, "dbeta": dbeta, "dgate": dgate}


def mta_layer_rows(x, wqkv, theta, w, gamma, beta, eps, lam, wo, H, c_h, rows,
                   kq_place=PRE, head_place=POST, theta_post=None):
    """mta_layer at selected tokens (b, i) only: K, V of the token's batch in
    full, queries of the convolution window.  Returns [n, D] float64."""
    B, L, D = x.shape
    d = D // H
    wq = wqkv.astype(np.float64)
    out = np.zeros((len(rows), D), np.float64)
    cache = {}
    for n, (b, i) in enumerate(rows):
        if b not in cache:
            qkv_b = np.matmul(x[b].astype(np.float64), wq.T)              # [L, 3D]
            cache = {b: _split_qkv(qkv_b, H, d)}
        q, k, v = cache[b]
        o = mta_attention_rows(q[None], k[None], v[None], theta, w, c_h, [(0, i)],
                               kq_place, head_place, theta_post=theta_post)[0]  # [H, d]
        y = group_norm_scale(o, gamma, beta, eps, lam).reshape(D)
        out[n] = y @ wo.astype(np.float64).T
    return out
