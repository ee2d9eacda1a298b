"""Writes tests/golden/oracle_small.txt by calling only the oracle (and the seeded generator).

The fixture freezes the oracle's output on two tiny seeded cases so that an
accidental change to its arithmetic shows up as a failing regression test.
The values themselves are pinned by the closed-form tests.
"""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))

import oracle  # noqa: E402
from synthetic import gaussian, rng_for  # noqa: E402


def main():
    G = gaussian(rng_for(42, 0), 5, 3)
    out = ["# oracle.orthogonalize on gaussian(rng_for(42, 0), 5, 3), eps=1e-7",
           "# case cubic10_5x3: 10 cubic steps (1.5, -0.5, 0) of the 5x3 input",
           "# case quintic5_3x5: 5 quintic steps (3.4445, -4.7750, 2.0315) of its transpose"]
    O, _ = oracle.orthogonalize(G, [oracle.CUBIC] * 10)
    out.append("case cubic10_5x3")
    out += [" ".join(repr(float(v)) for v in row) for row in O]
    O, _ = oracle.orthogonalize(G.T, [oracle.QUINTIC] * 5)
    out.append("case quintic5_3x5")
    out += [" ".join(repr(float(v)) for v in row) for row in O]
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.txt"), "w") as f:
        f.write("\n".join(out) + "\n")


if __name__ == "__main__":
    main()
