"""Planted mistakes in the fp64 oracle, for checking that its pins catch them.

A pytest plugin, loaded only by tests/test_oracle_mutations.py in a child
process (`-p oracle_mutants`).  It replaces one oracle function by a wrong
variant, named by the environment variable MTA_ORACLE_MUTANT, before the pins
of tests/test_oracle_pins.py run.  Every variant is a plausible slip in
writing the method down: a dropped tap, a flipped key or query offset, a
transposed mixing matrix, a mask off by one, a wrong scale, a missing re-mask,
mixing with the source heads' values instead of the destination head's, the
unbiased variance in the norm, a strict exact indicator, the gate's sign, and
wrong adjoints in the backward pass.  The mistakes live in the CPU oracle only;
nothing here touches the CUDA library.
"""
import os

import numpy as np

import oracle
import oracle.mta_oracle as M

_ORIG = {n: getattr(M, n) for n in (
    "attention_logits", "mask_zero", "mask_neg_inf", "key_query_conv", "head_mix",
    "post_softmax_conv", "mta_attention_group", "group_norm_scale",
    "key_query_conv_adjoint", "key_query_conv_grad_theta", "key_query_conv_exact",
    "sigmoid_gate")}


def _drop_tap(m, theta):
    """The last key tap of every row of the kernel is left out."""
    th = np.array(theta, np.float64, copy=True)
    th[:, :, -1] = 0.0
    return _ORIG["key_query_conv"](m, th)


def _flip_key(m, theta):
    """Key offset with the wrong sign: reads key j + b instead of j - b."""
    return _ORIG["key_query_conv"](m, np.asarray(theta)[:, :, ::-1])


def _future_queries(m, theta):
    """Query offset with the wrong sign: reads row r + a instead of r - a."""
    return _ORIG["key_query_conv"](m[:, ::-1], theta)[:, ::-1]


def _transpose_mix(a, w):
    return _ORIG["head_mix"](a, np.asarray(w).T)


def _mask_diagonal(a, qpos):
    """Mask_0 that also zeroes the diagonal (j >= i instead of j > i)."""
    fut = np.arange(a.shape[-1])[None, :] >= np.asarray(qpos)[:, None]
    return np.where(fut[None], 0.0, a)


def _no_mask0(a, qpos):
    return a


def _no_causal_softmax(c, qpos):
    return c


def _wrong_scale(q_rows, k, scale):
    return _ORIG["attention_logits"](q_rows, k, 1.25 * scale)


def _no_remask(attn, theta_post, qpos):
    """The convolution after the softmax without Mask_0 after it."""
    return M.key_query_conv(attn, theta_post)


def _source_values(q_rows, k, v, theta, w, qpos, scale, kq_place, head_place, theta_post=None):
    """Post-softmax mixing of the heads' outputs, sum_s w[r][s] A_s V_s, instead of
    mixing the weights against the destination head's values."""
    if head_place != M.POST:
        return _ORIG["mta_attention_group"](q_rows, k, v, theta, w, qpos, scale, kq_place,
                                            head_place, theta_post)
    o = _ORIG["mta_attention_group"](q_rows, k, v, theta, w, qpos, scale, kq_place, M.OFF,
                                     theta_post)
    return _ORIG["head_mix"](o, w)


def _unbiased_variance(o, gamma, beta, eps, lam):
    o = o.astype(np.float64)
    H, d = o.shape[-2], o.shape[-1]
    mu = np.mean(o, axis=-1, keepdims=True)
    var = np.sum((o - mu) ** 2, axis=-1, keepdims=True) / (d - 1)
    y = (o - mu) / np.sqrt(var + eps)
    y = y * gamma.astype(np.float64).reshape(H, d) + beta.astype(np.float64).reshape(H, d)
    lam = np.asarray(lam, np.float64)
    return (lam.reshape(H, 1) if lam.ndim else lam) * y


def _adjoint_flipped(g, theta):
    """The convolution's adjoint with its key taps in the forward's order."""
    return _ORIG["key_query_conv_adjoint"](g, np.asarray(theta)[:, :, ::-1])


def _grad_theta_flipped(g, m, cq, ck):
    """The kernel gradient with its key taps reversed."""
    return _ORIG["key_query_conv_grad_theta"](g, m, cq, ck)[:, :, ::-1]


def _exact_strict(a_hat, theta, qpos):
    """The exact indicator with a strict inequality: a tap may not read the
    output query's own key."""
    return _ORIG["key_query_conv_exact"](a_hat, theta, np.asarray(qpos) - 1)


def _gate_sign(gate):
    """The scalar gate with the wrong sign inside the sigmoid."""
    return _ORIG["sigmoid_gate"](-np.asarray(gate, np.float64))


MUTANTS = {
    "drop_tap": ("key_query_conv", _drop_tap),
    "flip_key_offset": ("key_query_conv", _flip_key),
    "future_queries": ("key_query_conv", _future_queries),
    "transposed_mix": ("head_mix", _transpose_mix),
    "mask0_on_diagonal": ("mask_zero", _mask_diagonal),
    "no_mask0": ("mask_zero", _no_mask0),
    "non_causal_softmax": ("mask_neg_inf", _no_causal_softmax),
    "wrong_scale": ("attention_logits", _wrong_scale),
    "post_conv_without_remask": ("post_softmax_conv", _no_remask),
    "mix_with_source_values": ("mta_attention_group", _source_values),
    "unbiased_variance": ("group_norm_scale", _unbiased_variance),
    "adjoint_flipped": ("key_query_conv_adjoint", _adjoint_flipped),
    "grad_theta_flipped": ("key_query_conv_grad_theta", _grad_theta_flipped),
    "exact_indicator_strict": ("key_query_conv_exact", _exact_strict),
    "gate_sign": ("sigmoid_gate", _gate_sign),
}


def pytest_configure(config):
    name = os.environ.get("MTA_ORACLE_MUTANT", "none")
    if name == "none":
        return
    attr, fn = MUTANTS[name]
    setattr(M, attr, fn)
    if hasattr(oracle, attr):
        setattr(oracle, attr, fn)
