"""Write the frozen noise-spec fixture (noise_spec_seed0.txt) from the CPU oracle only.

The fixture freezes the noise specification: any later change to the oracle's
noise arithmetic changes these values and fails the regression test, so such a
change has to be deliberate (and justified by the pages or the spec).
Run:  python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

# (seed, layer, draw, token, channel, stream): corners of every counter word and
# all four channel slots of one Philox call.
CASES = [
    (0, 0, 0, 0, 0, 0), (0, 0, 0, 0, 1, 0), (0, 0, 0, 0, 2, 0), (0, 0, 0, 0, 3, 0),
    (0, 0, 0, 0, 4, 0), (0, 0, 1, 0, 0, 0), (0, 0, 0, 1, 0, 0), (0, 1, 0, 0, 0, 0),
    (1, 0, 0, 0, 0, 0), (0, 0, 0, 0, 0, 1), (0, 3, 16383, 16383, 2047, 0),
    (0, 9, 4095, 65535, 4095, 0), (7, 2, 1023, 12345, 1023, 0),
    (4294967295, 4294967295, 4294967295, 4294967295, 4294967295, 4294967295),
    (123456789, 42, 77, 88, 99, 1),
]


def main():
    path = os.path.join(HERE, "noise_spec_seed0.txt")
    with open(path, "w") as f:
        f.write("# Frozen values of the Philox4x32-10 + Box-Muller noise specification.\n")
        f.write("# Written by tests/golden/make_golden.py from the CPU oracle only.\n")
        f.write("# seed layer draw token channel stream -> binary32 bits (hex) | x0 x1 x2 x3 of the Philox call\n")
        for (s, l, d, t, c, st) in CASES:
            v = oracle.gauss(s, l, d, t, c, st)
            words = oracle.philox4x32_10([c >> 2, t, d, st], [s, l])
            bits = int(v.view("uint32"))
            f.write(f"{s} {l} {d} {t} {c} {st} {bits:08x} | " + " ".join(f"{int(w):08x}" for w in words) + "\n")
    print(path)


if __name__ == "__main__":
    main()
