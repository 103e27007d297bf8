"""Writes tests/golden/*.json from the float64 oracle (and nothing else).

Each fixture stores seeded bf16 inputs (as bit patterns), the mask settings and
the oracle's O (float64) and LSE for a case small enough to read.  The
definition it encodes is the standard three-step attention of the
FlashAttention-2 overview (lshu.cn), section 2.1, with the causal mask of
section 4.2 problem 4 and the window of the flash-attn install guide
(yfxerp.com), section 1, under the readings stated in the oracle's header.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from synth import bf16_bits_to_f32, make_inputs  # noqa: E402

CASES = [
    # name, B, Sq, Sk, H, D, causal, win_left, win_right, seed
    ("tiny_causal_window", 1, 6, 8, 1, 64, 1, 3, 0, 4242),
    ("tiny_noncausal", 1, 5, 5, 1, 64, 0, -1, -1, 4243),
]


def main():
    for name, B, Sq, Sk, H, D, causal, wl, wr, seed in CASES:
        bits = make_inputs(B, Sq, Sk, H, D, seed, 1.0, with_dout=True)
        w = {n: bf16_bits_to_f32(bits[n]).astype(np.float64) for n in bits}
        scale = 1.0 / np.sqrt(D)
        g = oracle.attention_backward(w["q"], w["k"], w["v"], w["do"], scale, causal, wl, wr)
        doc = {
            "source": "oracle.attention_backward (float64) via tests/golden/make_golden.py",
            "cite": "FlashAttention-2 overview (lshu.cn) section 2.1; causal: section 4.2 problem 4; "
                    "window: flash-attn install guide (yfxerp.com) section 1",
            "shape": {"B": B, "Sq": Sq, "Sk": Sk, "H": H, "D": D},
            "mask": {"causal": causal, "win_left": wl, "win_right": wr}, "scale": scale,
            "inputs_bf16_bits": {n: bits[n].reshape(-1).tolist() for n in ("q", "k", "v", "do")},
            "o": g["o"].reshape(-1).tolist(),
            "lse": [x if np.isfinite(x) else "-inf" for x in g["lse"].reshape(-1).tolist()],
            "dq": g["dq"].reshape(-1).tolist(),
            "dk": g["dk"].reshape(-1).tolist(),
            "dv": g["dv"].reshape(-1).tolist(),
        }
        with open(os.path.join(HERE, name + ".json"), "w") as f:
            json.dump(doc, f, separators=(",", ":"))


if __name__ == "__main__":
    main()
