"""Readers for the hand-written fixtures under tests/golden/."""
import math
import os
from fractions import Fraction

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line.split()


def code_table(name):
    """{code: value} from a two-column fixture; values may be 'nan' or '-0'."""
    out = {}
    for code, val in _lines(name):
        if val == "nan":
            out[int(code, 16)] = math.nan
        elif val == "-0":
            out[int(code, 16)] = -0.0
        else:
            out[int(code, 16)] = float(Fraction(val))
    return out


def hand_case():
    d = {"scale": {}, "codes": {}, "out": {}}
    for tok in _lines("hand_1x16x2.txt"):
        if tok[0] == "gscale":
            d["gscale"] = float(Fraction(tok[1]))
        elif tok[0] == "scale":
            d["scale"][int(tok[1])] = int(tok[2], 16)
        elif tok[0] == "codes":
            d["codes"][int(tok[1])] = [int(x) for x in tok[2:]]
        elif tok[0] == "out":
            d["out"][tok[1]] = [float(x) for x in tok[2:]]
    return d
