"""Reader for the hand-derived golden micro cases under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_cases(fname="micro_cases.txt"):
    cases, cur = {}, None
    with open(os.path.join(GOLDEN, fname)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("case "):
                cur = {}
                cases[line.split()[1]] = cur
                continue
            key, val = [s.strip() for s in line.split("=", 1)]
            if key == "sizes":
                for kv in val.split():
                    a, b = kv.split("=")
                    cur[a] = int(b)
            else:
                cur[key] = np.array([float(v) for v in val.split()], dtype=np.float64)
    return cases


def shaped(case):
    """The case's tensors in their natural shapes."""
    T, H, E, I = case["T"], case["H"], case["E"], case["I"]
    out = dict(hidden=case["hidden"].reshape(T, H), router_w=case["router_w"].reshape(E, H))
    if "fc1_interleaved" in case:
        out["fc1"] = case["fc1_interleaved"].reshape(E, 2 * I, H)
        out["layout"] = "interleaved"
    if "fc1_chunked" in case:
        out["fc1"] = case["fc1_chunked"].reshape(E, 2 * I, H)
        out["layout"] = "chunked"
    if "fc2" in case:
        out["fc2"] = case["fc2"].reshape(E, H, I)
    return out
