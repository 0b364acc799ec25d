"""Reader for the hand-derived golden block fixtures in this folder.

Format: '#' comments; 'key values...' lines; 'case NAME' starts a case (files
without it hold one case); 'mode page|floor' starts the expected values of
that scale mode. Values may be written 'v*n' for n copies. Inputs shorter than
the block are padded with +0.0, whose expected output is +0, nibble 0, no
saturation.
"""
from __future__ import annotations

import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _expand(tokens):
    out = []
    for t in tokens:
        if "*" in t:
            v, n = t.split("*")
            out += [v] * int(n)
        else:
            out.append(t)
    return out


def load(name: str):
    """Returns (header dict, list of cases); a case is dict(name, input, modes)."""
    head, cases, case, mode = {}, [], None, None
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "case":
                case = dict(name=vals[0], input=None, modes={})
                cases.append(case)
                mode = None
            elif key == "input":
                if case is None:
                    case = dict(name=name, input=None, modes={})
                    cases.append(case)
                case["input"] = _expand(vals)
            elif key == "mode":
                mode = {}
                case["modes"][vals[0]] = mode
            elif mode is not None:
                mode[key] = _expand(vals)
            else:
                head[key] = vals[0]
    block = int(head["block"])
    for c in cases:
        raw = [int(v, 16) for v in c["input"]]
        dt = np.uint16 if head["dtype"] == "bf16" else np.uint32
        inp = np.zeros(block, dt)
        inp[: len(raw)] = raw
        c["input"] = inp if head["dtype"] == "bf16" else inp.view(np.float32)
        for m in c["modes"].values():
            o = np.zeros(block, dt)
            vals = [int(v, 16) for v in m["out"]]
            o[: len(vals)] = vals
            m["out"] = o
            nb = np.zeros(block, np.uint8)
            nv = [int(v) for v in m["nibble"]]
            nb[: len(nv)] = nv
            m["nibble"] = nb
            s = np.zeros(block, bool)
            s[[int(v) for v in m.get("sat", [])]] = True
            m["sat"] = s
            m["e8m0"] = int(m["e8m0"][0])
    return head, cases
