"""Build the CPU oracle (plain C, gcc) into a shared library.

Test infrastructure: the oracle is loaded only by the test suite, the smoke
check and the benchmark's CPU-baseline leg.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "fd_oracle.c")
LIBRARY = os.path.join(HERE, "libfd_oracle.so")


def build(out_path: str = LIBRARY, mutant: int = 0, force: bool = False) -> str:
    """Compile fd_oracle.c to ``out_path``; ``mutant`` != 0 plants the
    numbered mistake (used only by the tests that show the pins catch it)."""
    if (not force and mutant == 0 and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(SOURCE)):
        return out_path
    # -O2 without -ffast-math: IEEE double semantics, libm exp/log.
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-Wall", "-Wextra", f"-DFDO_MUTANT={int(mutant)}",
           "-o", out_path, SOURCE, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


if __name__ == "__main__":
    print(build(force=True))
