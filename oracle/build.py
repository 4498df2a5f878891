"""Compile the CPU oracle (oracle.c) into liboracle.so beside this file.

Test infrastructure: the product library never links or loads the result.
Extra ``defines`` exist only so that tests can build deliberately broken
copies of the oracle (planted mistakes) into a separate directory and check
that the pins catch them.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
FLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
         "-Wall", "-Wextra", "-shared", "-fPIC"]


def build(out_path=None, defines=(), force=False):
    """Build the oracle; return the path of the shared library."""
    out = out_path or os.path.join(HERE, "liboracle.so")
    deps = [SRC, os.path.join(HERE, "oracle.h")]
    if (not force and not defines and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(d) for d in deps)):
        return out
    cmd = ["gcc", *FLAGS, *[f"-D{d}" for d in defines], SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True, cwd=HERE)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
