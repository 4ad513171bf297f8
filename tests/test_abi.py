"""The C-ABI library: it builds, loads, exports every function include/mta.h
declares, and rejects bad arguments on the host before any CUDA call (these
tests need no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from token_attention_b200 import build, mta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return mta.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mta.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mta_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(mta.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", mta.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(L, f)


def test_version_and_strings(L):
    assert L.mta_abi_version() == 3
    for code in range(6):
        assert L.mta_status_string(code)
    assert L.mta_status_string(0) == b"ok"


def good_cfg(**kw):
    base = dict(B=2, H=4, L=64, d=64, c_q=6, c_k=11, c_h=2, kq_place=mta.PRE,
                head_place=mta.POST, dtype=mta.BF16)
    base.update(kw)
    return mta.make_cfg(**base)


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every case below fails a host check


def fake(i):
    """Distinct addresses 1 GiB apart (no two tensors of these shapes overlap),
    never dereferenced."""
    return ctypes.c_void_p((1 << 36) + (i << 30))


def call_attn(L, cfg, q=None, theta=FAKE, w=FAKE, out=None, k=None, v=None, default_q=True):
    q = fake(1) if q is None and default_q else q
    out = fake(6) if out is None else out
    return L.mta_attn_fwd(q, fake(2) if k is None else k, fake(3) if v is None else v, theta, w,
                          ctypes.byref(cfg) if cfg else None, out)


def up(x):
    return -(-x // 256) * 256


def test_workspace_query(L):
    cfg = good_cfg()   # the contraction kernel applies: its operands are counted
    B, H, Ls, d, cq, M = 2, 4, 64, 64, 6, 6 - 1 + 2 * (11 // 2)
    lpad = -(-Ls // 128) * 128
    items = B * (H // 2) * 1     # (batch, head group, query tile) work items
    xg = min(160, 2 * items) * 2 * 2 * d * 128 * 4   # exchange buffer of the persistent CTAs
    kq = up(B * H * cq * Ls * d * 2) + up(B * H * lpad * 4) + up(B * H * Ls * M * 4) + xg
    assert L.mta_attn_workspace_bytes(ctypes.byref(cfg)) == 256 + kq
    t = 2 * 64
    D = 4 * 64
    base = 256 + up(t * 3 * D * 2) + 2 * up(t * D * 2)
    assert L.mta_layer_workspace_bytes(ctypes.byref(cfg)) == base + kq
    other = good_cfg(c_q=3)   # not a contraction shape: fixed scratch only
    assert L.mta_attn_workspace_bytes(ctypes.byref(other)) == 256
    assert L.mta_layer_workspace_bytes(ctypes.byref(other)) == base
    post = good_cfg(kq_post=1)   # adds the values convolved by the post-softmax kernels
    vt = up(B * H * Ls * 2 * cq * d * 2)   # both heads of the group (post-softmax mixing)
    assert L.mta_attn_workspace_bytes(ctypes.byref(post)) == 256 + kq + vt
    assert L.mta_layer_workspace_bytes(ctypes.byref(post)) == base + kq + vt
    post_nomix = good_cfg(kq_post=1, head_place=mta.OFF)
    kq0 = kq - xg
    assert L.mta_attn_workspace_bytes(ctypes.byref(post_nomix)) == 256 + kq0 + up(B * H * Ls * cq * d * 2)
    post_off = good_cfg(kq_post=1, kq_place=mta.OFF)   # CUDA-core kernel only
    assert L.mta_attn_workspace_bytes(ctypes.byref(post_off)) == 256
    # L >= 4096: the CTA-pair kernel serves d = 64 with post-softmax mixing; its
    # mixing scratch is per (batch, head group, query tile): two heads x two parts
    # of d x 128 fp32, then a counter per slot
    for Ll in (4096, 8192):
        long_cfg = good_cfg(L=Ll)
        slots = B * (H // 2) * (Ll // 128)
        xg_pair = slots * 2 * 2 * d * 128 * 4 + up(slots * 4)
        kq_long = up(B * H * cq * Ll * d * 2) + up(B * H * Ll * 4) + up(B * H * Ll * M * 4) + xg_pair
        assert L.mta_attn_workspace_bytes(ctypes.byref(long_cfg)) == 256 + kq_long
    assert L.mta_attn_workspace_bytes(ctypes.byref(good_cfg(c_k=4))) == 0
    assert L.mta_attn_workspace_bytes(None) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(c_k=4), 1), (dict(c_k=17), 1), (dict(c_q=0), 1), (dict(c_q=9), 1),
    (dict(H=5), 1), (dict(c_h=0), 1), (dict(B=0), 1), (dict(L=0), 1),
    (dict(kq_place=2), 1), (dict(kq_place=4), 1), (dict(head_place=3), 1), (dict(dtype=7), 1), (dict(path=4), 1), (dict(path=-1), 1),
    (dict(scale=-1.0), 1), (dict(qkv_row_stride=10), 1), (dict(kq_post=2), 1), (dict(kq_post=-1), 1),
    (dict(kq_post=1, kq_place=mta.OFF, path=mta.PATH_KQ), 2), (dict(kq_post=1, path=mta.PATH_TC), 2),
    (dict(d=200), 2), (dict(d=20), 2), (dict(B=70000), 2),
    (dict(n_events=-1), 1), (dict(n_events=65), 1), (dict(n_events=2), 1),
])
def test_bad_config_rejected(L, kw, code):
    cfg = good_cfg(**kw)
    cfg.workspace, cfg.workspace_bytes = 0x100000, 1 << 20
    assert call_attn(L, cfg) == code


def test_null_and_workspace_errors(L):
    assert call_attn(L, None) == 1
    cfg = good_cfg()
    cfg.workspace, cfg.workspace_bytes = 0x100000, 1 << 20
    assert call_attn(L, cfg, default_q=False) == 1
    assert L.mta_attn_fwd(fake(1), fake(2), fake(3), FAKE, FAKE, ctypes.byref(cfg), None) == 1
    assert call_attn(L, cfg, theta=None) == 1           # kq_place PRE needs theta
    assert call_attn(L, cfg, w=None) == 1               # head mixing needs w
    post_only = good_cfg(kq_place=mta.OFF, kq_post=1)
    post_only.workspace, post_only.workspace_bytes = 0x100000, 1 << 20
    assert call_attn(L, post_only, theta=None) == 1     # the post-softmax kernels are theta
    nomix = good_cfg(kq_place=mta.OFF, head_place=mta.OFF)
    nomix.workspace, nomix.workspace_bytes = 0x100000, 1 << 20
    assert call_attn(L, nomix, q=ctypes.c_void_p(fake(1).value + 1)) == 1   # misaligned bf16
    cfg.workspace_bytes = 16
    assert call_attn(L, cfg) == 3
    cfg.workspace, cfg.workspace_bytes = 0x100010, 1 << 20   # not 256-byte aligned
    assert call_attn(L, cfg) == 3
    cfg.workspace = None
    assert call_attn(L, cfg) == 3


def test_layer_argument_errors(L):
    cfg = good_cfg()
    cfg.workspace, cfg.workspace_bytes = 0x100000, 1 << 30
    gn = mta.MtaGn(0x20000, 0x20000, 1e-5, 12, -1.0)
    f = lambda c, g=ctypes.byref(gn), x=fake(1), out=fake(6): L.mta_layer_fwd(
        x, fake(2), FAKE, FAKE, g, fake(3), ctypes.byref(c), out)
    assert f(cfg, g=None) == 1
    assert f(cfg, x=None) == 1
    f32 = good_cfg(dtype=mta.F32)
    f32.workspace, f32.workspace_bytes = 0x100000, 1 << 30
    assert f(f32) == 2
    small = good_cfg()
    small.workspace, small.workspace_bytes = 0x100000, 1024
    assert f(small) == 3
    forced = good_cfg(path=mta.PATH_KQ)   # the contraction kernel without room for its operands
    base = L.mta_layer_workspace_bytes(ctypes.byref(good_cfg(c_q=3)))
    forced.workspace, forced.workspace_bytes = 0x100000, base
    assert f(forced) == 3
    # the output must not overlap x, Wqkv or Wo
    assert f(cfg, out=fake(1)) == 1
    assert f(cfg, out=ctypes.c_void_p(fake(2).value + 256)) == 1
    assert f(cfg, out=fake(3)) == 1


def test_output_aliasing_rejected(L):
    """An output that shares bytes with an input is refused (MTA_ERR_INVALID)
    before anything is enqueued; distinct buffers pass on to the workspace check."""
    cfg = good_cfg()
    cfg.workspace, cfg.workspace_bytes = 0x100000, 16   # too small: a call that passes the
    assert call_attn(L, cfg) == 3                        # pointer checks stops at the workspace
    for n in ("q", "k", "v"):
        i = {"q": 1, "k": 2, "v": 3}[n]
        assert call_attn(L, cfg, out=fake(i)) == 1
        # a view starting inside the input (e.g. the second token)
        assert call_attn(L, cfg, out=ctypes.c_void_p(fake(i).value + 4 * 64 * 2)) == 1
    # an output ending just before q starts does not overlap
    n_out = 2 * 64 * 4 * 64 * 2
    assert call_attn(L, cfg, out=ctypes.c_void_p(fake(1).value - n_out)) == 3
    # strided q/k/v (a [B][L][3][H][d] buffer): out inside the span of the last token
    st = good_cfg(qkv_row_stride=3 * 4 * 64)
    st.workspace, st.workspace_bytes = 0x100000, 16
    span = ((2 * 64 - 1) * 3 * 4 * 64 + 4 * 64) * 2
    assert call_attn(L, st, out=ctypes.c_void_p(fake(3).value + span - 2)) == 1
    assert call_attn(L, st, out=ctypes.c_void_p(fake(3).value + span)) == 3
    # the backward pass: gradients must not overlap the inputs or each other
    g = lambda dq, dk, dv: L.mta_attn_bwd(fake(1), fake(2), fake(3), FAKE, FAKE, fake(4),
                                         ctypes.byref(cfg), dq, dk, dv, None, None)
    assert g(fake(11), fake(12), fake(13)) == 3
    assert g(fake(4), fake(12), fake(13)) == 1
    assert g(fake(11), fake(11), fake(13)) == 1
    assert g(fake(11), fake(12), fake(2)) == 1


def test_building_block_argument_errors(L):
    assert L.mta_gemm_bf16_nt(FAKE, FAKE, FAKE, 0, 8, 8, None) == 1
    assert L.mta_gemm_bf16_nt(FAKE, FAKE, FAKE, 8, 8, 12, None) == 1   # K % 8
    gn = mta.MtaGn(0x20000, 0x20000, 1e-5, 12, -1.0)
    assert L.mta_group_norm_scale(FAKE, ctypes.byref(gn), 4, 2, 0, FAKE, None) == 1
    assert L.mta_group_norm_scale(FAKE, None, 4, 2, 64, FAKE, None) == 1
    # the general GEMM: flags are 0 or 1; the contiguous extent of each operand a
    # multiple of 8 (K for [rows][K], M or N for a transposed operand); C apart from A, B
    g = lambda M, N, K, am=0, bm=0, f=0, c=fake(3): L.mta_gemm_bf16(fake(1), fake(2), c, M, N, K, am, bm, f, None)
    assert g(16, 16, 16, am=2) == 1
    assert g(16, 16, 16, f=3) == 1
    assert g(12, 16, 16, am=1) == 1     # transposed A: M % 8
    assert g(16, 12, 16, bm=1) == 1     # transposed B: N % 8
    assert g(16, 16, 12) == 1           # K-major: K % 8
    assert g(16, 16, 16, c=fake(1)) == 1   # C overlaps A
    # the group norm's backward: d in {32, 64, 96, 128}; the gate's gradient when gated
    gb = lambda d, g_=ctypes.byref(gn), dgate=None: L.mta_group_norm_scale_bwd(
        fake(1), fake(2), g_, 4, 2, d, fake(3), fake(4), fake(5), fake(6), dgate, None)
    assert gb(48) == 2
    assert gb(64, g_=None) == 1
    gated = mta.MtaGn(0x20000, 0x20000, 1e-5, 12, -1.0, 0x30000)
    assert gb(64, g_=ctypes.byref(gated)) == 1   # no dgate


def test_layer_backward_argument_errors(L):
    """mta_layer_bwd checks its arguments on the host and enqueues nothing on error."""
    cfg = good_cfg()
    cfg.workspace, cfg.workspace_bytes = 0x100000, 1 << 40
    gn = mta.MtaGn(0x20000, 0x20000, 1e-5, 12, -1.0)
    f = lambda c, g=ctypes.byref(gn), dx=fake(11), dwq=fake(12), dwo=fake(13), dout=fake(4): L.mta_layer_bwd(
        fake(1), fake(2), FAKE, FAKE, g, fake(3), dout, ctypes.byref(c) if c else None,
        dx, dwq, dwo, None, None, fake(14), fake(15), None)
    assert f(None) == 1
    assert f(cfg, g=None) == 1
    assert f(cfg, dx=None) == 1
    assert f(cfg, dout=None) == 1
    assert f(cfg, dx=fake(1)) == 1                      # dx overlaps x
    assert f(cfg, dwo=fake(12)) == 1                    # two outputs overlap
    bad = good_cfg(dtype=mta.F32)
    bad.workspace, bad.workspace_bytes = 0x100000, 1 << 40
    assert f(bad) == 2
    odd = good_cfg(d=48)                                # d outside {32, 64, 96, 128}
    odd.workspace, odd.workspace_bytes = 0x100000, 1 << 40
    assert f(odd) == 2
    small = good_cfg()
    small.workspace, small.workspace_bytes = 0x100000, 1 << 10
    assert f(small) == 3
    gated = mta.MtaGn(0x20000, 0x20000, 1e-5, 12, -1.0, 0x30000)
    assert f(cfg, g=ctypes.byref(gated)) == 1           # gated without dgate


def test_layer_backward_workspace_query(L):
    """The fixed part (status; QKV, O, Y bf16; dY fp32; dO bf16; dq, dk, dv fp32; dQKV
    bf16), then the larger of the forward recompute's contraction operands and the
    tensor-core backward's strips."""
    B, H, Ls, d = 2, 4, 64, 64
    T, D = B * Ls, H * d
    fixed = 256 + 2 * up(T * 3 * D * 2) + 3 * up(T * D * 2) + 4 * up(T * D * 4)
    cfg = good_cfg()
    attn_bwd = L.mta_attn_bwd_workspace_bytes(ctypes.byref(cfg)) - 256
    attn_fwd = L.mta_attn_workspace_bytes(ctypes.byref(cfg)) - 256
    assert L.mta_layer_bwd_workspace_bytes(ctypes.byref(cfg)) == fixed + max(attn_bwd, attn_fwd)
    other = good_cfg(c_q=3)   # neither the contraction kernel nor the tensor-core backward
    assert L.mta_layer_bwd_workspace_bytes(ctypes.byref(other)) == fixed


def test_backward_argument_errors(L):
    """mta_attn_bwd checks its arguments on the host and enqueues nothing on error."""
    cfg = good_cfg()
    cfg.workspace, cfg.workspace_bytes = 0x100000, 1 << 20
    f = lambda c, dq=fake(11), theta=FAKE, dout=fake(4): L.mta_attn_bwd(
        fake(1), fake(2), fake(3), theta, FAKE, dout, ctypes.byref(c) if c else None,
        dq, fake(12), fake(13), FAKE, FAKE)
    assert f(None) == 1
    assert f(cfg, dq=None) == 1
    assert f(cfg, dout=None) == 1
    assert f(cfg, theta=None) == 1                      # kq_place PRE needs the kernels
    assert f(cfg, dq=ctypes.c_void_p(fake(11).value + 2)) == 1   # fp32 gradients, 4-byte aligned
    forced = good_cfg(path=mta.PATH_TC)                 # no direct tensor-core backward
    forced.workspace, forced.workspace_bytes = 0x100000, 1 << 20
    assert f(forced) == 2
    kq = good_cfg(path=mta.PATH_KQ)                     # the tensor-core backward, strips too small
    kq.workspace, kq.workspace_bytes = 0x100000, 1 << 20
    assert f(kq) == 3
    other = good_cfg(path=mta.PATH_KQ, c_q=3)           # a shape it does not serve
    other.workspace, other.workspace_bytes = 0x100000, 1 << 20
    assert f(other) == 2
    small = good_cfg()
    small.workspace, small.workspace_bytes = 0x100000, 16
    assert f(small) == 3
    # the status word, then the tensor-core backward's strips for one query block of
    # every head (B H = 8, pitch 64; blocks of R = 384 rows up to L = 3072): S [R rows]
    # and A, dA/dC [R - 5 rows] fp32, the dS and A'' halves [2R rows] bf16
    Z, P, R = 2 * 4, 64, 384
    rc = R - 5
    strips = up(Z * R * P * 4) + 2 * up(Z * rc * P * 4) + 2 * up(Z * 2 * R * P * 2)
    assert L.mta_attn_bwd_workspace_bytes(ctypes.byref(good_cfg())) == 256 + strips
    # pre-softmax mixing keeps the unmixed C as well
    assert L.mta_attn_bwd_workspace_bytes(ctypes.byref(good_cfg(head_place=mta.PRE))) == \
        256 + strips + up(Z * rc * P * 4)
    # the convolution after the softmax: blocks of R - 3 (c_q - 1) own rows, the same
    # R - 5 row strips, and its output gradient G [R - 5], dA / dC [R - 10] and A' [R - 15]
    assert L.mta_attn_bwd_workspace_bytes(ctypes.byref(good_cfg(kq_post=1))) == \
        256 + strips + up(Z * (R - 5) * P * 4) + up(Z * (R - 10) * P * 4) + up(Z * (R - 15) * P * 4)
    # past L = 3072 the blocks have R = 512 rows
    Ll, Rl = 4096, 512
    long_strips = (up(Z * Rl * Ll * 4) + 2 * up(Z * (Rl - 5) * Ll * 4) + 2 * up(Z * 2 * Rl * Ll * 2))
    assert L.mta_attn_bwd_workspace_bytes(ctypes.byref(good_cfg(L=Ll))) == 256 + long_strips
    assert L.mta_attn_bwd_workspace_bytes(ctypes.byref(good_cfg(c_q=3))) == 256   # CUDA cores only
    assert L.mta_attn_bwd_workspace_bytes(ctypes.byref(good_cfg(c_k=4))) == 0


# ---------------------------------------------------------------------------
# the Python binding rejects tensors the C ABI cannot take, before any call
# ---------------------------------------------------------------------------

class FakeCuda:
    """Stands in for a CUDA tensor on a machine without a GPU: only the
    attributes the binding's checks read."""

    def __init__(self, shape, dtype, contiguous=True, index=0):
        import torch
        self.shape, self.dtype, self._c = tuple(shape), dtype, contiguous
        self.is_cuda, self.device = True, torch.device("cuda", index)

    def is_contiguous(self):
        return self._c


def test_binding_checks_device_dtype_shape_layout():
    import torch
    dv = torch.device("cuda", 0)
    f32 = torch.float32
    mta._need("t", None, dv, f32, (2, 3))                     # optional argument left out
    mta._need("t", FakeCuda((2, 3), f32), dv, f32, (2, 3))
    with pytest.raises(ValueError, match="CUDA tensor"):
        mta._need("t", torch.zeros(2, 3), dv, f32, (2, 3))   # host memory
    with pytest.raises(ValueError, match="CUDA tensor"):
        mta._need("t", FakeCuda((2, 3), f32, index=1), dv)    # another GPU
    with pytest.raises(TypeError, match="bfloat16"):
        mta._need("t", FakeCuda((2, 3), f32), dv, torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        mta._need("t", FakeCuda((3, 2), f32), dv, f32, (2, 3))
    with pytest.raises(ValueError, match="contiguous"):
        mta._need("t", FakeCuda((2, 3), f32, contiguous=False), dv, f32)
    mta._need("t", FakeCuda((2, 3), f32, contiguous=False), dv, f32, contiguous=False)


def test_binding_rejects_host_tensors():
    """Host tensors would hand host pointers to the kernels: every entry point
    refuses them with a ValueError before calling the library."""
    import torch
    B, L, H, d = 1, 8, 2, 32
    bf = lambda *s: torch.zeros(s, dtype=torch.bfloat16)
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32)
    q = bf(B, L, H, d)
    th, w = f32(H, 3, 5), f32(1, 2, 2)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mta.attn_fwd(q, q, q, th, w, 3, 5, 2)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mta.attn_bwd(q, q, q, th, w, q, 3, 5, 2)
    D = H * d
    with pytest.raises(ValueError, match="CUDA tensor"):
        mta.layer_fwd(bf(B, L, D), bf(3 * D, D), th, w, f32(D), f32(D), bf(D, D), H, 3, 5, 2)
    with pytest.raises(ValueError, match="multiple of H"):
        mta.layer_fwd(bf(B, L, 65), bf(195, 65), th, w, f32(65), f32(65), bf(65, 65), H, 3, 5, 2)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mta.gemm_bf16_nt(bf(16, 8), bf(4, 8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        mta.group_norm_scale(q, f32(H * d), f32(H * d))


def test_plain_c_caller(L, tmp_path):
    """include/mta.h is plain C99: a C program that includes only the header
    compiles warning-free against it, links libmta.so and gets the documented
    status codes from the host-side checks (tests/abi_host.c)."""
    exe = tmp_path / "abi_host"
    lib_dir = os.path.dirname(mta.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                         "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_host.c"),
                         "-o", str(exe), mta.LIB_PATH, f"-Wl,-rpath,{lib_dir}"],
                        capture_output=True, text=True, timeout=120)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr


# ---------------------------------------------------------------------------
# kernel selection, asked of the library on the host (mta_attn_kernel)
# ---------------------------------------------------------------------------

def _cfg_for(wl, ws_bytes=None, path=mta.PATH_AUTO):
    d = wl.D // wl.H if wl.layer else wl.d
    cfg = mta.make_cfg(wl.B, wl.H, wl.L, d, wl.c_q, wl.c_k, wl.c_h, wl.kq_place, wl.head_place,
                       mta.F32 if wl.dtype == "f32" else mta.BF16, path=path, kq_post=int(wl.kq_post))
    cfg.workspace_bytes = mta.lib().mta_attn_workspace_bytes(ctypes.byref(cfg)) if ws_bytes is None else ws_bytes
    return cfg


def test_kernel_choice_matches_the_bench_launch_count(L):
    """bench.py counts the kernels a step launches from its own reading of the
    selection rules; the library's own choice (with the workspace the bench
    gives it) must agree for every workload."""
    import bench
    from token_attention_b200 import synth
    for name, wl in synth.WORKLOADS.items():
        want = mta.PATH_KQ if bench.uses_contraction(wl) else mta.PATH_TC if bench.uses_direct_tc(wl) \
            else mta.PATH_SIMT
        assert mta.attn_kernel(_cfg_for(wl)) == want, name


def test_kernel_choice_rules(L):
    from token_attention_b200 import synth
    wl = synth.WORKLOADS["pretrain_d128_L2048"]
    assert mta.attn_kernel(_cfg_for(wl)) == mta.PATH_KQ
    # without room for the convolved keys, path 0 takes the direct tensor-core kernel,
    # and a forced contraction kernel reports the workspace
    assert mta.attn_kernel(_cfg_for(wl, ws_bytes=256)) == mta.PATH_TC
    with pytest.raises(mta.MtaError) as e:
        mta.attn_kernel(_cfg_for(wl, ws_bytes=256, path=mta.PATH_KQ))
    assert e.value.code == 3
    assert mta.attn_kernel(_cfg_for(wl, path=mta.PATH_SIMT)) == mta.PATH_SIMT
    assert mta.attn_kernel(_cfg_for(wl, path=mta.PATH_TC)) == mta.PATH_TC
    # fp32 has only the CUDA-core kernel
    tiny = synth.WORKLOADS["tiny_f32_L256"]
    for path, code in ((mta.PATH_TC, 2), (mta.PATH_KQ, 2)):
        with pytest.raises(mta.MtaError) as e:
            mta.attn_kernel(_cfg_for(tiny, path=path))
        assert e.value.code == code
    # the post-softmax convolution: contraction kernel or CUDA-core kernel, never the direct form
    both = synth.WORKLOADS["both_d128_L2048"]
    assert mta.attn_kernel(_cfg_for(both, ws_bytes=256)) == mta.PATH_SIMT
    with pytest.raises(mta.MtaError) as e:
        mta.attn_kernel(_cfg_for(both, path=mta.PATH_TC))
    assert e.value.code == 2
    # an invalid configuration, and a workspace too small for the error word
    bad = _cfg_for(wl)
    bad.c_k = 4
    with pytest.raises(mta.MtaError) as e:
        mta.attn_kernel(bad)
    assert e.value.code == 1
    with pytest.raises(mta.MtaError) as e:
        mta.attn_kernel(_cfg_for(wl, ws_bytes=64))
    assert e.value.code == 3


@pytest.mark.parametrize("B,H,L_,d,cq,ck,ch,kq,hp,dt,post", [
    (1, 16, 300, 128, 8, 15, 16, mta.PRE, mta.POST, mta.F32, 1),
    (1, 16, 300, 128, 8, 15, 16, mta.PRE_EXACT, mta.PRE, mta.BF16, 1),
    (1, 16, 300, 16, 1, 1, 1, mta.OFF, mta.OFF, mta.F32, 0),
    (65535, 1, 1, 16, 1, 1, 1, mta.OFF, mta.OFF, mta.BF16, 0),
])
def test_extreme_documented_shapes_have_a_kernel(L, B, H, L_, d, cq, ck, ch, kq, hp, dt, post):
    """The ends of the ranges the header documents (c_q = 8, c_k = 15, c_h = 16,
    d = 16 and 128, B = 65535, both convolutions) are not refused: the library
    selects a kernel for them (the CUDA-core kernel with fewer rows per CTA).
    This checks the host's choice only; these shapes are not among the GPU
    parity cases."""
    cfg = mta.make_cfg(B, H, L_, d, cq, ck, ch, kq, hp, dt, kq_post=post)
    cfg.workspace_bytes = L.mta_attn_workspace_bytes(ctypes.byref(cfg))
    assert mta.attn_kernel(cfg) == mta.PATH_SIMT


def test_selftest_wait_timeout_argument_errors(L):
    """The bounded-wait diagnostic checks its arguments on the host."""
    cfg = good_cfg()
    cfg.workspace, cfg.workspace_bytes = 0x100000, 1 << 20
    assert L.mta_selftest_wait_timeout(None, 1000) == 1
    assert L.mta_selftest_wait_timeout(ctypes.byref(cfg), 0) == 1
    assert L.mta_selftest_wait_timeout(ctypes.byref(cfg), 2000001) == 1
    cfg.workspace = None
    assert L.mta_selftest_wait_timeout(ctypes.byref(cfg), 1000) == 3
    cfg.workspace, cfg.workspace_bytes = 0x100010, 1 << 20
    assert L.mta_selftest_wait_timeout(ctypes.byref(cfg), 1000) == 3
