"""Writes tests/golden/worked_example.json: a hand-sized MoE block whose output
is known in closed form.

The pages print no worked example, so this one is derived by hand from the
block's definition (router softmax over all experts, renormalised top-k,
SwiGLU experts with the gate in the first half of w13, one shared expert of
weight 1, residual add; page "Hyper Optimizing Kimi K3 in vLLM: Moving Fast
and Responsibly", section "Recovering time between operators", names these
steps).  Every input is exactly representable in bf16.  With sigma(z) =
1/(1+exp(-z)) and silu(z) = z*sigma(z):

  x = [1, 0.5];  R = [[2, 1, 0], [0.5, -1, 3]]   -> logits [2.25, 0.5, 1.5]
  top-2 = [0, 2];  w = [sigma(0.75), sigma(-0.75)]
  expert 0: W13 = [[1, 1], [0, 2]]     -> g = 1,  u = 2 -> a = 2 sigma(1)
            W2  = [[1, -1]]             -> y0 = [a, -a]
  expert 1: large weights, never selected
  expert 2: W13 = [[-1, 0.5], [-2, 1]] -> g = -2, u = 1 -> a = -2 sigma(-2)
            W2  = [[0.25, 4]]           -> y2 = [0.25 a, 4 a]
  shared:   W13 = [[0.5, 1], [1, 0]]   -> g = 1,  u = 1 -> a = sigma(1)
            W2  = [[2, 0.5]]            -> s = [2 a, 0.5 a]
  out = x + w0 y0 + w2 y2 + s

Only the closed form above (math.exp) produces the stored values.
Run:  python tests/golden/make_worked_example.py
"""
import json
import math
import os


def sigma(z):
    return 1.0 / (1.0 + math.exp(-z))


def main():
    x = [1.0, 0.5]
    R = [[2.0, 1.0, 0.0], [0.5, -1.0, 3.0]]
    w13 = [[[1.0, 1.0], [0.0, 2.0]], [[3.0, 3.0], [3.0, 3.0]], [[-1.0, 0.5], [-2.0, 1.0]]]
    w2 = [[[1.0, -1.0]], [[5.0, 5.0]], [[0.25, 4.0]]]
    sw13 = [[0.5, 1.0], [1.0, 0.0]]
    sw2 = [[2.0, 0.5]]
    logits = [2.25, 0.5, 1.5]
    w0, w2_ = sigma(0.75), sigma(-0.75)
    a0 = 2.0 * sigma(1.0)
    a2 = -2.0 * sigma(-2.0)
    as_ = sigma(1.0)
    y0 = [a0, -a0]
    y2 = [0.25 * a2, 4.0 * a2]
    s = [2.0 * as_, 0.5 * as_]
    out = [x[h] + w0 * y0[h] + w2_ * y2[h] + s[h] for h in range(2)]
    data = {
        "citation": "hand-derived closed form; see the docstring of make_worked_example.py",
        "shape": {"hidden": 2, "n_experts": 3, "top_k": 2, "inter": 1, "shared_inter": 1},
        "x": [x], "router_w": R, "w13": w13, "w2": w2, "shared_w13": sw13, "shared_w2": sw2,
        "expected": {"logits": [logits], "topk_ids": [[0, 2]], "topk_w": [[w0, w2_]], "out": [out]},
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "worked_example.json")
    with open(path, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    print(path)


if __name__ == "__main__":
    main()
