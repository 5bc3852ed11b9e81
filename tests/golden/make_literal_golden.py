"""Write tests/golden/literal_*.txt: small random rational cases of the update
in its printed matrix form, evaluated exactly by oracle.literal.

Calls only oracle/.  Source of the form: "Gated DeltaNet-2" LIT-802 review,
"Key takeaways" 1 (paper Sec. 3.1, Eqs. 8-10).  Run from the repo root:
    python tests/golden/make_literal_golden.py
"""

import os
import random
import sys
from fractions import Fraction

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "..", ".."))
from oracle import literal  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def rat(rng, lo, hi, den=8):
    return Fraction(rng.randint(lo * den, hi * den), den)


def case(seed, T, dk, dv):
    rng = random.Random(seed)
    S0 = [[rat(rng, -2, 2) for _ in range(dv)] for _ in range(dk)]
    seq = []
    for _ in range(T):
        seq.append(dict(
            q=[rat(rng, -1, 1) for _ in range(dk)],
            k=[rat(rng, -1, 1) for _ in range(dk)],
            v=[rat(rng, -2, 2) for _ in range(dv)],
            alpha=[Fraction(rng.randint(4, 8), 8) for _ in range(dk)],
            b=[Fraction(rng.randint(0, 16), 8) for _ in range(dk)],   # erase gate in [0, 2]
            w=[Fraction(rng.randint(0, 8), 8) for _ in range(dv)],
        ))
    ST, outs = literal.run(S0, seq)
    path = os.path.join(HERE, f"literal_T{T}_k{dk}_v{dv}_s{seed}.txt")
    with open(path, "w") as f:
        f.write("# Written by tests/golden/make_literal_golden.py (oracle.literal, exact "
                "rationals).\n# Printed matrix form of the update: \"Gated DeltaNet-2\" "
                "LIT-802 review, Key takeaways 1 (Sec. 3.1 Eqs. 8-10).\n")
        f.write(f"dims {T} {dk} {dv}\n")
        f.write("S0 " + " ".join(str(x) for row in S0 for x in row) + "\n")
        for t, tok in enumerate(seq):
            for n in ("q", "k", "v", "alpha", "b", "w"):
                f.write(f"{n}{t} " + " ".join(str(x) for x in tok[n]) + "\n")
        for t, o in enumerate(outs):
            f.write(f"o{t} " + " ".join(str(x) for x in o) + "\n")
        f.write("ST " + " ".join(str(x) for row in ST for x in row) + "\n")
    return path


if __name__ == "__main__":
    for args in ((1, 3, 3, 2), (2, 4, 2, 3), (3, 5, 4, 4)):
        print(case(*args))
