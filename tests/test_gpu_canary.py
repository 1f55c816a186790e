"""Canary-padded buffers and the debug build (the sanitizer substitute).

The cases of tests/canary_cases.py run every writing entry point of the
forward and decode paths with each buffer inside a canary-filled allocation.
With the release library the pads must stay intact and the device status
clean.  The same cases run in a child process with CSA_DEBUG=1, i.e. through
libcsa_debug.so, whose kernels check the indices they compute before each
global access and record CSA_ERR_DEVICE_BOUNDS instead of accessing: its
status must be clean as well, its pads intact, and every buffer it wrote
bit-identical to the release library's."""
import os
import subprocess
import sys

import numpy as np
import pytest

import canary_cases

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def release():
    return canary_cases.run_all()


def _check_clean(res, which):
    for k, v in res.items():
        if k.endswith("/status"):
            assert int(v[0]) == 0, f"{which}: {k} = {int(v[0])}"
        if k.endswith("/pads_intact"):
            assert bool(v[0]), f"{which}: canary overwritten around {k[:-len('/pads_intact')]}"


def test_release_pads_intact_and_status_clean(release):
    _check_clean(release, "release")
    # index rows are written in full: no canary word (0xA5A5A5A5) is left in any of them
    for k, v in release.items():
        if "/idx" in k and not k.endswith("pads_intact"):
            assert not (v.view(np.uint32) == 0xA5A5A5A5).any(), f"{k}: rows left unwritten"


def test_debug_build_matches_release_bit_for_bit(release, tmp_path):
    path = str(tmp_path / "debug.npz")
    env = dict(os.environ, CSA_DEBUG="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "canary_cases.py"), path], env=env, cwd=HERE,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    debug = dict(np.load(path))
    _check_clean(debug, "debug build")
    assert set(debug) == set(release)
    for k in release:
        if k.endswith(("/status", "/pads_intact")):
            continue
        assert np.array_equal(debug[k], release[k]), f"{k}: the debug build's result differs"
