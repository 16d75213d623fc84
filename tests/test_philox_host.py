"""The library's sampling generator (csrc/philox.cuh), built for the host,
against the generator's published known-answer vectors and against the
oracle's independent restatement (oracle/sampling.py): identical words and
identical fp32 uniforms.  CPU only (g++)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import sampling as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_diffusion_speculative_layers_b200", "csrc")
GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="module")
def host_bin(tmp_path_factory):
    cxx = shutil.which("g++")
    if not cxx:
        pytest.skip("no g++")
    out = str(tmp_path_factory.mktemp("philox") / "philox_host")
    subprocess.run([cxx, "-O2", "-std=c++17", "-I", CSRC, os.path.join(ROOT, "tests", "host", "philox_host.cpp"),
                    "-o", out], check=True)
    return out


def _run(binary, text):
    return subprocess.run([binary], input=text, capture_output=True, text=True, check=True).stdout.split("\n")


def test_host_build_matches_known_answers(host_bin):
    rows = [l for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l.strip() and l[0] != "#"]
    cmds, want = [], []
    for l in rows:
        ctr, key, out = (part.split() for part in l.split("|"))
        cmds.append("p " + " ".join(ctr + key))
        want.append(" ".join(out))
    got = _run(host_bin, "\n".join(cmds) + "\n")
    assert got[:len(want)] == want


def test_host_build_draws_equal_the_oracle(host_bin):
    rng = np.random.default_rng(4)
    cases = [(int(rng.integers(0, 2 ** 63)), int(rng.integers(0, 10 ** 6)), int(rng.integers(0, 64)),
              int(rng.integers(1, 5)), int(rng.integers(1, 40))) for _ in range(20)]
    cases.append((2 ** 64 - 1, 2 ** 31, 255, S.TARGET, 9))
    text = "".join(f"u {seed} {pos} {slot} {purpose} {n}\n" for seed, pos, slot, purpose, n in cases)
    lines = iter(l for l in _run(host_bin, text) if l)
    for seed, pos, slot, purpose, n in cases:
        want = S.uniform_vector(seed, slot, pos, purpose, n)
        got = np.array([float.fromhex(next(lines)) for _ in range(n)])
        np.testing.assert_array_equal(got, want)
        scalar = next(lines)
        assert scalar.startswith("s ") and float.fromhex(scalar[2:]) == S.uniform_scalar(seed, slot, pos, purpose)
