"""The frozen tiny-GTA fixture still matches the generator and the oracle."""
import os

import numpy as np

from tests.golden import make_golden


def _parse(text):
    sha, lse, out = None, {}, {}
    for line in text.splitlines():
        if line.startswith("#") or not line.strip():
            continue
        f = line.split()
        if f[0] == "inputs_sha256":
            sha = f[1]
        elif f[0] == "lse":
            lse[(int(f[1]), int(f[2]))] = float(f[3])
        else:
            out[(int(f[1]), int(f[2]))] = np.array([float(x) for x in f[3:]])
    return sha, lse, out


def test_gta_tiny_fixture_is_reproduced():
    with open(make_golden.OUT) as fh:
        sha0, lse0, out0 = _parse(fh.read())
    sha1, lse1, out1 = _parse(make_golden.render())
    assert sha0 == sha1, "the seeded generator changed"
    for k in lse0:
        assert abs(lse0[k] - lse1[k]) <= 1e-13
        np.testing.assert_allclose(out0[k], out1[k], rtol=0, atol=1e-13)
