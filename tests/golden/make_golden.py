"""Writes tests/golden/oracle_tiny.txt from the fp64 oracle alone.

The fixture freezes the oracle's output on one tiny seeded case, so a later
change to the oracle's arithmetic shows up as a diff that must be justified.
It calls only the oracle and the seeded input generator.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sliding_window_attention_sink_b200 import workloads as wl  # noqa: E402

CASE = dict(seqlens=[13, 11], Hq=2, Hkv=1, D=8, window=5, sigma=1.0,
            sink="uniform2", seed=0)


def compute():
    c = wl.prefill_case(CASE["seqlens"], CASE["Hq"], CASE["Hkv"], CASE["D"],
                        CASE["window"], sigma=CASE["sigma"], sink=CASE["sink"],
                        seed=CASE["seed"])
    return oracle.prefill(c["q"], c["k"], c["v"], c["cu_seqlens"], CASE["Hq"],
                          CASE["Hkv"], CASE["D"], CASE["window"], sink=c["sink"],
                          nthreads=1)


def main():
    o, lse, _ = compute()
    path = os.path.join(HERE, "oracle_tiny.txt")
    with open(path, "w") as f:
        f.write("# fp64 oracle snapshot; written by make_golden.py; case %r\n" % (CASE,))
        f.write("# lines: 'lse h t value' then 'o t h d value'\n")
        for h in range(lse.shape[0]):
            for t in range(lse.shape[1]):
                f.write("lse %d %d %r\n" % (h, t, float(lse[h, t])))
        for t in range(o.shape[0]):
            for h in range(o.shape[1]):
                for d in range(o.shape[2]):
                    f.write("o %d %d %d %r\n" % (t, h, d, float(o[t, h, d])))
    print(path)


if __name__ == "__main__":
    main()
