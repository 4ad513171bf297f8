"""Seeded synthetic inputs for the MTA forward path.

This module only draws numbers: normal samples, bf16 rounding of those samples
and the planted high-similarity key pairs of the long-context workload.  It holds
none of the method's arithmetic, so both the fp64 oracle (tests, bench CPU
baseline) and the CUDA path (tests, bench) take their inputs from here.

Every workload is named by what it is, with its sizes.  The value recipes follow
the pages' workloads: Multi-Token Attention (greeksharifa summary), section 4.2
(c_q=6, c_k=11, identity initialisation of the convolutions, section 4.6) and
appendix D (880M model: D=1536, 16 heads, context 2048).
"""
from __future__ import annotations

import dataclasses

import numpy as np

# Placements (same integer codes as the C-ABI's mta_place).
OFF, PRE, POST = 0, 1, 2


def rng_for(seed: int, stream: int) -> np.random.Generator:
    """Independent PCG64 stream `stream` of workload seed `seed`."""
    return np.random.default_rng([int(seed), int(stream)])


def normal(seed: int, stream: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """float32 samples of N(mean, std^2)."""
    x = rng_for(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32
    arrays whose values are exactly representable in bf16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(x.shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of bf16-exact float32 values (upper halves)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("values are not bf16-exact; call round_bf16 first")
    return (u >> 16).astype(np.uint16)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    c_q: int
    c_k: int
    c_h: int
    kq_place: int
    head_place: int
    dtype: str            # "f32" or "bf16": dtype of q/k/v/out (or x/W/out)
    seed: int
    theta_kind: str       # "identity" or "delta_noise"
    theta_std: float
    w_kind: str           # "identity" or "eye_noise"
    w_std: float
    layer: bool = False   # full layer (QKV projection .. output projection)
    D: int = 0
    depth: int = 12       # layer index of the depth scale (the scale itself is the method's)
    planted_pairs: int = 0
    kq_post: bool = False # key-query convolution after the softmax as well (own kernels)

    @property
    def tokens(self) -> int:
        return self.B * self.L

    @property
    def causal_pairs(self) -> int:
        """Causal (query, key) pairs over all batches and heads: B*H*L(L+1)/2."""
        return self.B * self.H * self.L * (self.L + 1) // 2


WORKLOADS = {
    # tiny fp32 case the oracle finishes in seconds
    "tiny_f32_L256": Workload("tiny_f32_L256", B=1, H=4, L=256, d=32, c_q=3, c_k=5, c_h=2,
                              kq_place=PRE, head_place=POST, dtype="f32", seed=1001,
                              theta_kind="delta_noise", theta_std=0.1,
                              w_kind="eye_noise", w_std=0.1),
    # identity kernels: must equal standard causal attention
    "identity_d64_L2048": Workload("identity_d64_L2048", B=2, H=16, L=2048, d=64, c_q=6, c_k=11,
                                   c_h=2, kq_place=PRE, head_place=POST, dtype="bf16",
                                   seed=1002, theta_kind="identity", theta_std=0.0,
                                   w_kind="identity", w_std=0.0),
    # pretraining-shaped attention (B*L = 8192 tokens, 16 heads, d=128)
    "pretrain_d128_L2048": Workload("pretrain_d128_L2048", B=4, H=16, L=2048, d=128, c_q=6,
                                    c_k=11, c_h=2, kq_place=PRE, head_place=POST, dtype="bf16",
                                    seed=1003, theta_kind="delta_noise", theta_std=0.05,
                                    w_kind="eye_noise", w_std=0.1),
    # long context with planted high-similarity key pairs
    "long_d128_L16384": Workload("long_d128_L16384", B=1, H=16, L=16384, d=128, c_q=6, c_k=11,
                                 c_h=2, kq_place=PRE, head_place=POST, dtype="bf16",
                                 seed=1004, theta_kind="delta_noise", theta_std=0.05,
                                 w_kind="eye_noise", w_std=0.1, planted_pairs=8),
    # full layer, pre-softmax head mixing
    "layer_pre_D2048_L4096": Workload("layer_pre_D2048_L4096", B=2, H=16, L=4096, d=128, c_q=6,
                                      c_k=11, c_h=2, kq_place=PRE, head_place=PRE, dtype="bf16",
                                      seed=1005, theta_kind="delta_noise", theta_std=0.05,
                                      w_kind="eye_noise", w_std=0.1, layer=True, D=2048),
    # full layer, post-softmax head mixing
    "layer_post_D2048_L4096": Workload("layer_post_D2048_L4096", B=2, H=16, L=4096, d=128, c_q=6,
                                       c_k=11, c_h=2, kq_place=PRE, head_place=POST,
                                       dtype="bf16", seed=1005, theta_kind="delta_noise",
                                       theta_std=0.05, w_kind="eye_noise", w_std=0.1,
                                       layer=True, D=2048),
    # the pages' 880M pretraining shape: dimension 1536 over 16 heads (d = 96), L = 2048
    "pretrain_d96_L2048": Workload("pretrain_d96_L2048", B=4, H=16, L=2048, d=96, c_q=6, c_k=11,
                                   c_h=2, kq_place=PRE, head_place=POST, dtype="bf16", seed=1007,
                                   theta_kind="delta_noise", theta_std=0.05, w_kind="eye_noise",
                                   w_std=0.1),
    # the convolution on both sides of the softmax (the pages' default setting),
    # pretraining-shaped: post kernels drawn like the pre kernels
    "both_d128_L2048": Workload("both_d128_L2048", B=4, H=16, L=2048, d=128, c_q=6, c_k=11,
                                c_h=2, kq_place=PRE, head_place=POST, dtype="bf16", seed=1006,
                                theta_kind="delta_noise", theta_std=0.05, w_kind="eye_noise",
                                w_std=0.1, kq_post=True),
}


def shrink(wl: Workload, **changes) -> Workload:
    """Same value recipe at other sizes (used for small parity cases)."""
    return dataclasses.replace(wl, **changes)


# stream ids (fixed so that a tensor does not change when another one is added)
_S_Q, _S_K, _S_V, _S_THETA, _S_W, _S_X, _S_WQKV, _S_WO, _S_GAMMA, _S_BETA, _S_PLANT = range(11)
_S_THETA_POST = 11


def make_theta(wl: Workload, stream: int = _S_THETA) -> np.ndarray:
    """Key-query kernels [H][c_q][c_k], float32.  "(0,0)" is the current query
    and the centre key: theta[h][0][c_k//2]."""
    th = np.zeros((wl.H, wl.c_q, wl.c_k), np.float32)
    if wl.theta_kind == "delta_noise":
        th += normal(wl.seed, stream, th.shape, std=wl.theta_std)
    elif wl.theta_kind != "identity":
        raise ValueError(wl.theta_kind)
    th[:, 0, wl.c_k // 2] += 1.0
    return th


def make_theta_post(wl: Workload):
    """Post-softmax key-query kernels [H][c_q][c_k] (same recipe as the pre-softmax
    ones, their own stream), or None when the workload has none."""
    return make_theta(wl, _S_THETA_POST) if wl.kq_post else None


def make_w(wl: Workload) -> np.ndarray:
    """Head-mixing weights [H/c_h][c_h][c_h], float32: w[g][r][s] weighs source
    head g*c_h+s in destination head g*c_h+r."""
    G = wl.H // wl.c_h
    w = np.zeros((G, wl.c_h, wl.c_h), np.float32)
    if wl.w_kind == "eye_noise":
        w += normal(wl.seed, _S_W, w.shape, std=wl.w_std)
    elif wl.w_kind != "identity":
        raise ValueError(wl.w_kind)
    w += np.eye(wl.c_h, dtype=np.float32)[None]
    return w


def _plant_draws(wl: Workload) -> list:
    """The seeded draws of the planted pairs, in stream order: (p, r, noise) with
    noise [B][H][d] float32 for key p+1."""
    rng = rng_for(wl.seed, _S_PLANT)
    L = wl.L
    draws = []
    for _ in range(wl.planted_pairs):
        p = int(rng.integers(wl.c_k, L - 2))
        r = int(rng.integers(p + 2, L)) if p + 2 < L else L - 1
        noise = rng.standard_normal(size=(wl.B, wl.H, wl.d), dtype=np.float32) * 0.05
        draws.append((p, r, noise))
    return draws


def planted_positions(wl: Workload) -> list:
    """(p, r) of every planted pair of the workload: key p+1 is a near copy of key
    p and query r is 2*k_p (the same draws make_attn_inputs uses)."""
    return [(p, r) for p, r, _ in _plant_draws(wl)]


def plant_pairs_at(q: np.ndarray, k: np.ndarray, positions, seed: int) -> None:
    """Plants pairs at the given (p, r) positions in q, k [B][L][H][d] (in place),
    with the key noise drawn from the plant stream of `seed`."""
    rng = rng_for(seed, _S_PLANT)
    draws = [(p, r, rng.standard_normal(size=(k.shape[0], k.shape[2], k.shape[3]), dtype=np.float32) * 0.05)
             for p, r in positions]
    _apply_pairs(q, k, draws)


def _apply_pairs(q: np.ndarray, k: np.ndarray, draws) -> None:
    for p, r, noise in draws:
        k[:, p + 1] = k[:, p] + noise
        q[:, r] = 2.0 * k[:, p]


def _plant_pairs(wl: Workload, q: np.ndarray, k: np.ndarray) -> None:
    """Planted high-similarity pairs (reading of "a few planted high-similarity
    key pairs at random positions"): for n seeded positions p, key p+1 becomes a
    near copy of key p and a later query r > p+1 becomes 2*k_p, in every head."""
    _apply_pairs(q, k, _plant_draws(wl))


def make_attn_inputs(wl: Workload) -> dict:
    """q, k, v as [B][L][H][d] float32 (bf16-exact when dtype is bf16), plus
    theta [H][c_q][c_k] and w [H/c_h][c_h][c_h]."""
    shape = (wl.B, wl.L, wl.H, wl.d)
    q = normal(wl.seed, _S_Q, shape)
    k = normal(wl.seed, _S_K, shape)
    v = normal(wl.seed, _S_V, shape)
    if wl.planted_pairs:
        _plant_pairs(wl, q, k)
    if wl.dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return dict(q=q, k=k, v=v, theta=make_theta(wl), w=make_w(wl), theta_post=make_theta_post(wl))


def make_layer_inputs(wl: Workload) -> dict:
    """x [B][L][D], Wqkv [3D][D] (rows Q|K|V, head-major), Wo [D][D] (out x in),
    all bf16-exact float32; theta, w, gamma [D], beta [D] float32."""
    D = wl.D
    x = round_bf16(normal(wl.seed, _S_X, (wl.B, wl.L, D)))
    wqkv = round_bf16(normal(wl.seed, _S_WQKV, (3 * D, D), std=0.02))
    wo = round_bf16(normal(wl.seed, _S_WO, (D, D), std=0.02))
    gamma = normal(wl.seed, _S_GAMMA, (D,), mean=1.0, std=0.1)
    beta = normal(wl.seed, _S_BETA, (D,), std=0.1)
    return dict(x=x, wqkv=wqkv, wo=wo, theta=make_theta(wl), w=make_w(wl),
                theta_post=make_theta_post(wl), gamma=gamma, beta=beta, eps=1e-5)
