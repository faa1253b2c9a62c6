"""The selection's first radix digit, checked on the host (no GPU): the library's key -> bin map,
its bin floors and its shared-prefix claims, compiled from the library's own header, against
the bin rule restated here from the float bits.

Rule: with a the bits [17, 31) of the fp32 score's pattern (exponent and top 6 mantissa bits of
|z|) and m = clamp(a - (119 * 64 - 1), 0, 1023), the bin is 1024 + m for z >= +0 and 1023 - m for
z < 0.  An order key is the float's bits with the sign bit set for z >= +0 and all bits flipped
for z < 0."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    return None


def _rule_from_keys(keys):
    keys = keys.astype(np.uint32)
    u = np.where(keys & 0x80000000, keys & 0x7FFFFFFF, ~keys).astype(np.uint32)
    m = np.clip(((u >> 17) & 0x3FFF).astype(np.int64) - (119 * 64 - 1), 0, 1023)
    return np.where((u >> 31) == 1, 1023 - m, 1024 + m)


def test_digit1_map_matches_the_rule_and_its_invariants(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = tmp_path / "digit1_check"
    subprocess.check_call([nvcc, "-std=c++17", "--expt-relaxed-constexpr", "-o", str(exe),
                           os.path.join(ROOT, "tests", "digit1_host_check.cu")])
    res = subprocess.run([str(exe)], capture_output=True, timeout=120)
    head, _, body = res.stdout.partition(b"\n")
    assert head == b"bad 0", head
    assert res.returncode == 0
    got = np.frombuffer(body, dtype="<u2").reshape(32768, 2).astype(np.int64)
    t = np.arange(32768, dtype=np.uint64)
    want_lo = _rule_from_keys((t << 17).astype(np.uint32))
    want_hi = _rule_from_keys(((t << 17) | 0x1FFFF).astype(np.uint32))
    assert np.array_equal(got[:, 0], want_lo)
    assert np.array_equal(got[:, 1], want_hi)
    # the four catch-all bins and the window's ends, by value
    z = np.array([-300.0, -250.0, -2 ** -8, -0.003, 0.0, 0.003, 2 ** -8, 250.0, 300.0], np.float32)
    u = z.view(np.uint32)
    keys = np.where(u >> 31, ~u, u | 0x80000000).astype(np.uint32)
    assert _rule_from_keys(keys).tolist() == [0, 1, 1022, 1023, 1024, 1024, 1025, 2046, 2047]
