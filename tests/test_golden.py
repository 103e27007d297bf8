"""Stored fixtures written by tests/golden/make_golden.py (oracle only): the
oracle must keep reproducing them, and the CUDA path must match them."""
import glob
import json
import os

import numpy as np
import pytest

from helpers import check_fwd, check_grad

HERE = os.path.dirname(os.path.abspath(__file__))
FILES = sorted(glob.glob(os.path.join(HERE, "golden", "*.json")))


def _load(path):
    d = json.load(open(path))
    s = d["shape"]
    shp = {"q": (s["B"], s["Sq"], s["H"], s["D"]), "do": (s["B"], s["Sq"], s["H"], s["D"]),
           "k": (s["B"], s["Sk"], s["H"], s["D"]), "v": (s["B"], s["Sk"], s["H"], s["D"])}
    bits = {n: np.array(d["inputs_bf16_bits"][n], dtype=np.uint16).reshape(shp[n]) for n in shp}
    lse = np.array([float(x) for x in d["lse"]]).reshape(s["B"], s["H"], s["Sq"])
    ref = {"o": np.array(d["o"]).reshape(shp["q"]), "lse": lse,
           "dq": np.array(d["dq"]).reshape(shp["q"]), "dk": np.array(d["dk"]).reshape(shp["k"]),
           "dv": np.array(d["dv"]).reshape(shp["v"])}
    return d, bits, ref


@pytest.mark.parametrize("path", FILES, ids=[os.path.basename(f) for f in FILES])
def test_oracle_reproduces_fixture(path):
    import oracle
    from synth import bf16_bits_to_f32
    d, bits, ref = _load(path)
    w = {n: bf16_bits_to_f32(b).astype(np.float64) for n, b in bits.items()}
    m = d["mask"]
    g = oracle.attention_backward(w["q"], w["k"], w["v"], w["do"], d["scale"], m["causal"],
                                  m["win_left"], m["win_right"])
    for n in ("o", "dq", "dk", "dv"):
        np.testing.assert_allclose(g[n], ref[n], rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(np.isinf(g["lse"]), np.isinf(ref["lse"]))


@pytest.mark.gpu
@pytest.mark.parametrize("path", FILES, ids=[os.path.basename(f) for f in FILES])
def test_cuda_path_matches_fixture(path):
    import torch
    from exact_attention_156_b200 import attn_bwd, attn_fwd, get_last_device_error
    from helpers import to_device, to_f64
    d, bits, ref = _load(path)
    m = d["mask"]
    win = (m["win_left"], m["win_right"])
    q, k, v, do = (to_device(bits[n]) for n in ("q", "k", "v", "do"))
    o, lse = attn_fwd(q, k, v, softmax_scale=d["scale"], causal=bool(m["causal"]), window_size=win)
    dq, dk, dv = attn_bwd(q, k, v, o, do, lse, softmax_scale=d["scale"], causal=bool(m["causal"]),
                          window_size=win)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), ref["o"], ref["lse"], path)
    floor = 1e-3 * max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
    for n, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(to_f64(g), ref[n], n, floor)
