"""Write hash_kat.json: known-answer values of the counter-based random
numbers, computed once by the CPU oracle and frozen, so that any later
change to the generator shows up. Calls only the oracle."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402


def main():
    rand16 = []
    for seed in (0, 1, 2, 5, 0xDEADBEEFCAFEF00D):
        for stream in (0, 1, 2):
            for i in (0, 1, 2, 3, 1000001, (1 << 33) + 7):
                rand16.append({"seed": seed, "stream": stream, "i": i,
                               "r": O.rand16(seed, stream, i)})
    signs = [{"seed": s, "c": c, "s": O.rht_sign(s, c)}
             for s in (2, 7) for c in (0, 1, 31, 32, 14335)]
    out = {"about": "Frozen outputs of the oracle's counter-based generator "
                    "(written by make_golden.py, which calls only the oracle).",
           "rand16": rand16, "rht_sign": signs}
    with open(os.path.join(HERE, "hash_kat.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
