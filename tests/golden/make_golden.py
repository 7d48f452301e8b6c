"""Write tests/golden/semantics_cases.json from the decimal brute force.

Calls only oracle/ (the Python-decimal brute force); the inputs are small
exact values written out in this file.  Each case cites the passage whose
semantics it fixes.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import brute  # noqa: E402

CASES = [
    {
        "name": "fully_masked_row_is_zero",
        "cite": "Karume v0.8.0 release notes, Breaking Changes, softmax NaN item: a fully "
                "masked row of fused attention yields exactly 0",
        "q": [[[0.5, -1.0]]], "k": [[[1.0, 2.0]]], "v": [[[3.0, 4.0]]],
        "pos": [-1], "window": 0, "scale": 1.0,
    },
    {
        "name": "nan_score_row_is_nan",
        "cite": "Karume v0.8.0 release notes, Breaking Changes, softmax NaN item: the row max "
                "is NaN-preserving, an all-NaN row yields NaN",
        "q": [[["nan", 1.0]]], "k": [[[1.0, 2.0]], [[0.5, 0.25]]], "v": [[[3.0, 4.0]], [[1.0, 1.0]]],
        "pos": [1], "window": 0, "scale": 1.0,
    },
    {
        "name": "two_keys_logistic",
        "cite": "states-form attention, Karume v0.12.0 release notes, Performance, first item: "
                "softmax of the QK scores applied to V over the KV state",
        "q": [[[1.0]]], "k": [[[0.0]], [[3.0]]], "v": [[[1.0]], [[-2.0]]],
        "pos": [1], "window": 0, "scale": 0.25,
    },
    {
        "name": "chunk_rows_causal_and_window",
        "cite": "Karume v0.8.0 release notes, Features, run-time window item: chunk rows "
                "attend to the cached rows before them and causally within the chunk; "
                "window 2 keeps keys [pos-1, pos]",
        "q": [[[0.5, -0.25], [1.5, 0.75]], [[-1.0, 2.0], [0.125, 0.5]], [[2.0, -2.0], [1.0, 1.0]]],
        "k": [[[0.25, 1.0]], [[-0.5, 0.5]], [[1.0, -1.0]], [[2.0, 0.0]], [[0.0, 0.75]]],
        "v": [[[1.0, 0.0]], [[0.0, 1.0]], [[-1.0, 2.0]], [[0.5, 0.5]], [[3.0, -3.0]]],
        "pos": [2, 3, 4], "window": 2, "scale": 0.7071067811865476,
    },
    {
        "name": "grouped_heads_share_kv_head",
        "cite": "grouped-query heads: query heads 0-1 read KV head 0, heads 2-3 KV head 1",
        "q": [[[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [-1.0, 0.5]]],
        "k": [[[1.0, 0.5], [0.0, -1.0]], [[0.25, 2.0], [1.5, 1.0]], [[-1.0, 1.0], [0.5, 0.5]]],
        "v": [[[2.0, 1.0], [0.0, 0.0]], [[-1.0, 0.5], [1.0, 3.0]], [[0.5, 0.5], [-2.0, 4.0]]],
        "pos": [2], "window": 0, "scale": 0.5, "n_kv_heads": 2,
    },
]


def _f(x):
    return float(x)


def cases():
    """The cases with their expected outputs from the brute force (as strings)."""
    out = []
    for c in CASES:
        import numpy as np
        q = np.array([[[_f(x) for x in h] for h in r] for r in c["q"]], dtype=np.float32)
        k = np.array([[[_f(x) for x in h] for h in r] for r in c["k"]], dtype=np.float32)
        v = np.array([[[_f(x) for x in h] for h in r] for r in c["v"]], dtype=np.float32)
        res = brute.attention(q, k, v, c["pos"], window=c["window"], scale=c["scale"],
                              n_kv_heads=c.get("n_kv_heads", 1))
        case = dict(c)
        case["expected"] = [[[str(x) for x in row] for row in head] for head in res]
        out.append(case)
    return out


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "semantics_cases.json")
    with open(path, "w") as f:
        json.dump({"generator": "tests/golden/make_golden.py (oracle.brute, 50 digits)",
                   "cases": cases()}, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
