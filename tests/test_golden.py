"""Values the pages print, checked against the shapes this library uses."""
import json
import os

from token_attention_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def test_param_delta_880m_matches_table8():
    """The MTA-minus-Transformer parameter count of the 880M model (29,592) is
    reproduced by per-head key-query kernels [H][c_q][c_k], per-group head-mixing
    matrices [H/c_h][c_h][c_h], a norm weight and bias over d, and one scalar per
    layer -- the parameter shapes this library takes."""
    g = json.load(open(os.path.join(HERE, "golden", "param_count_880m.json")))
    m = g["model"]
    wl = synth.Workload("880m", B=1, H=m["heads"], L=8, d=m["D"] // m["heads"], c_q=m["c_q"],
                        c_k=m["c_k"], c_h=m["c_h"], kq_place=synth.PRE,
                        head_place=synth.POST, dtype="bf16", seed=0,
                        theta_kind="identity", theta_std=0.0, w_kind="identity", w_std=0.0)
    kq_layers = m["layers"] // m["kq_every"]
    per_side = kq_layers * synth.make_theta(wl).size + m["layers"] * synth.make_w(wl).size
    norm = m["layers"] * 2 * wl.d
    scalars = m["layers"]
    assert m["sides"] * per_side + norm + scalars == g["mta_params"] - g["transformer_params"]
