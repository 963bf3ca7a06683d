"""Write worked_examples.json: tiny cases of the MoE layer with zero experts,
each solved by hand in closed form.

The LongCat-Flash write-up ("Meituan's large model goes viral for its
speed", itouyu.top, section "Zero-computation experts") defines the layer by
its glossary (softmax router R over N FFN experts plus Z zero experts that
return their input, expert bias b_i, K picks per token) but prints no worked
example.  The cases below are small enough that the picks, gates and outputs
follow by hand; this script only evaluates those hand-derived expressions
with the math module.  It does not call the oracle or the CUDA library.

    python tests/golden/make_worked_examples.py
"""
import json
import math
import os

SOURCE = (
    "LongCat-Flash write-up 'Meituan's large model goes viral for its speed' "
    "(itouyu.top), section 'Zero-computation experts'. The page prints no worked "
    "example; each case below is derived by hand from its definition (softmax over "
    "all N+Z experts, bias added to the score for selection only, gates = unbiased "
    "softmax, zero experts return x, SwiGLU FFN experts, ties to the lower index)."
)


def silu(z):
    return z / (1.0 + math.exp(-z))


def main():
    e = math.e
    zs = e + 1.0 + 1.0 / e
    p = [e / zs, 1.0 / zs, (1.0 / e) / zs]
    h = [silu(2.0) * 3.0, silu(1.0) * 1.0]
    y = [h[0], h[0] - h[1]]
    ex1_out = [p[2] * 2.0 + p[0] * y[0], p[2] * 1.0 + p[0] * y[1]]
    examples = [
        {
            "name": "one_ffn_one_zero",
            "derivation": "x=[2,1]; W_r rows [0.5,0],[0,0],[-0.5,0] give logits [1,0,-1]; "
                          "p = [e,1,1/e]/(e+1+1/e). b=[0,0,0.5] -> s=p+b picks {0 (FFN), 2 (zero)}. "
                          "Expert 0: W_gate=I, W_up=[[1,1],[0.5,0]], W_down=[[1,0],[1,-1]] -> "
                          "a=[2,1], u=[3,1], h=[3 silu(2), silu(1)], y=[h0, h0-h1]. out = p2*x + p0*y.",
            "N": 2, "Z": 1, "K": 2,
            "x": [[2.0, 1.0]],
            "W_r": [[0.5, 0.0], [0.0, 0.0], [-0.5, 0.0]],
            "b": [0.0, 0.0, 0.5],
            "W_gate": [[[1.0, 0.0], [0.0, 1.0]], [[0.0, 0.0], [0.0, 0.0]]],
            "W_up": [[[1.0, 1.0], [0.5, 0.0]], [[0.0, 0.0], [0.0, 0.0]]],
            "W_down": [[[1.0, 0.0], [1.0, -1.0]], [[0.0, 0.0], [0.0, 0.0]]],
            "expected_idx_set": [[0, 2]],
            "expected_gate": [[p[0], p[2]]],
            "expected_out": [ex1_out],
            "expected_load": [1, 0, 1],
        },
        {
            "name": "equal_logits_bias_decides",
            "derivation": "d=1, x=2, all logits 0 -> p=1/3 each. b=[0,0.1,0.05]: picks {1 (FFN), "
                          "2 (zero)}, gates 1/3. Expert 1 with W_gate=W_up=W_down=1 (I=1): "
                          "y = silu(2)*2. out = (x + y)/3.",
            "N": 2, "Z": 1, "K": 2,
            "x": [[2.0]],
            "W_r": [[0.0], [0.0], [0.0]],
            "b": [0.0, 0.1, 0.05],
            "W_gate": [[[0.0]], [[1.0]]],
            "W_up": [[[0.0]], [[1.0]]],
            "W_down": [[[0.0]], [[1.0]]],
            "expected_idx_set": [[1, 2]],
            "expected_gate": [[1.0 / 3.0, 1.0 / 3.0]],
            "expected_out": [[(2.0 + silu(2.0) * 2.0) / 3.0]],
            "expected_load": [0, 1, 1],
        },
        {
            "name": "exact_tie_lower_index",
            "derivation": "d=1, x=1, all logits 0 -> p=1/4 each (N=2, Z=2, K=1), b=0: all four "
                          "scores tie, so the lower index (expert 0) wins. Expert 0 with all "
                          "weights 1 (I=1): y = silu(1). out = y/4.",
            "N": 2, "Z": 2, "K": 1,
            "x": [[1.0]],
            "W_r": [[0.0], [0.0], [0.0], [0.0]],
            "b": [0.0, 0.0, 0.0, 0.0],
            "W_gate": [[[1.0]], [[1.0]]],
            "W_up": [[[1.0]], [[1.0]]],
            "W_down": [[[1.0]], [[1.0]]],
            "expected_idx_set": [[0]],
            "expected_gate": [[0.25]],
            "expected_out": [[silu(1.0) / 4.0]],
            "expected_load": [1, 0, 0, 0],
        },
    ]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "worked_examples.json")
    with open(path, "w") as f:
        json.dump({"source": SOURCE, "examples": examples}, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
