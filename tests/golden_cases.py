"""Parser for the hand-worked quantization fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
HOT, D = 32, 128


def _kv(s):
    return {"K": 0, "V": 1}[s]


def parse_cases(fname):
    """Returns {case_name: dict(quant_bits, tokens{(pos, kv): {ch: val}}, ops[...])}
    where ops are ("append", n) and ("check", dict) in file order."""
    cases = {}
    cur = None
    with open(os.path.join(GOLDEN, fname), encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "case":
                cur = dict(quant_bits=8, tokens={}, ops=[], bytes=[])
                cases[tok[1]] = cur
            elif tok[0] == "end":
                cur = None
            elif tok[0] == "config":
                for kv in tok[1:]:
                    k, v = kv.split("=")
                    cur[k] = int(v)
            elif tok[0] == "tok":
                pos, kv = int(tok[1]), _kv(tok[2])
                vals = {int(a): float(b) for a, b in (x.split("=") for x in tok[3:])}
                cur["tokens"][(pos, kv)] = vals
            elif tok[0] == "append":
                cur["ops"].append(("append", int(tok[1].split("=")[1])))
            elif tok[0] == "migrate":
                cur["ops"].append(("migrate", int(tok[1].split("=")[1])))
            elif tok[0] == "check":
                spec = {}
                codes = None
                i = 1
                while i < len(tok):
                    if tok[i] == "codes":
                        codes = {int(a): int(b) for a, b in (x.split("=") for x in tok[i + 1:])}
                        break
                    k, v = tok[i].split("=")
                    spec[k] = v
                    i += 1
                spec["codes"] = codes
                cur["ops"].append(("check", spec))
            elif tok[0] == "byte":
                spec = dict(x.split("=") for x in tok[1:])
                cur["bytes"].append((_kv(spec["kv"]), int(spec["off"]), int(spec["val"], 16)))
            else:
                raise ValueError("bad fixture line: %r" % raw)
    return cases


def token_arrays(case, start, n):
    """FP16 K, V for positions [start, start+n): [1][n][1][D] each."""
    k = np.zeros((1, n, 1, D), np.float32)
    v = np.zeros((1, n, 1, D), np.float32)
    for (pos, kv), vals in case["tokens"].items():
        if start <= pos < start + n:
            arr = k if kv == 0 else v
            for ch, val in vals.items():
                arr[0, pos - start, 0, ch] = val
    return k.astype(np.float16), v.astype(np.float16)
