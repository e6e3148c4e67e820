"""Compile the fp64 oracle (plain C) into ``oracle/liboracle.so``.  Test infrastructure only.

``-ffp-contract=off`` keeps every multiply and add a separate IEEE operation, so two oracle
functions that perform the same operation sequence give identical bits.
"""
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))


def build(force: bool = False) -> str:
    srcs = [os.path.join(_HERE, f) for f in ("gdn_oracle.c", "gdn_vjp.c")]
    out = os.path.join(_HERE, "liboracle.so")
    if force or not os.path.exists(out) or os.path.getmtime(out) < max(os.path.getmtime(s) for s in srcs):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                               "-o", out, *srcs, "-lm"])
    return out


if __name__ == "__main__":
    print(build(force=True))
