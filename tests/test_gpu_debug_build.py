"""The bounds-checked debug build (librib_debug.so, RIB_DEBUG).

Every work entry point runs once in each build, in a process of its own
(tests/debug_build_run.py): in the debug build no guarded access may fall
outside its buffer, and every output must equal the release build's, bit
for bit, except the query-side gradients of the attention backward, whose
fp32 sums run in CTA-scheduling order (compared within the parity bounds).
A self-test entry point then makes a guard refuse an index on purpose and
checks what is recorded; nothing out of range is touched.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

from windowed_attention_implicit_b200 import build as B

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _env(debug):
    env = dict(os.environ)
    env.pop("RIB_DEBUG_LIBRARY", None)
    if debug:
        env["RIB_DEBUG_LIBRARY"] = "1"
    return env


def _run_all(tmp_path, debug):
    path = tmp_path / ("debug.npz" if debug else "release.npz")
    r = subprocess.run([sys.executable, "-m", "tests.debug_build_run", str(path)], cwd=ROOT,
                       env=_env(debug), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout + r.stderr)[-3000:]
    print(("debug: " if debug else "release: ") + r.stdout.strip().splitlines()[-1])
    return np.load(path)


def test_debug_build_in_bounds_and_equal_to_release(tmp_path):
    B.build(debug=True)
    rel = _run_all(tmp_path, False)
    dbg = _run_all(tmp_path, True)
    assert rel["_debug_build"][0] == 0 and dbg["_debug_build"][0] == 1
    assert sorted(rel.files) == sorted(dbg.files)
    bad = []
    for k in rel.files:
        if k.startswith("_"):
            continue
        a, b = rel[k], dbg[k]
        if k.startswith("~"):
            d = np.abs(a - b)
            if d.max() > 2e-2 or d.mean() > 2e-3:
                bad.append(f"{k}: max {d.max():.3e} mean {d.mean():.3e}")
        elif not np.array_equal(a, b):
            bad.append(f"{k}: differs (max |d| {np.abs(a - b).max():.3e})")
    assert not bad, bad


_SELFTEST = r"""
import ctypes
import windowed_attention_implicit_b200 as R
from windowed_attention_implicit_b200 import _abi
lib = R.library()
info = (ctypes.c_ulonglong * 2)()
assert lib.rib_debug_build() == 1
assert lib.rib_debug_guard_selftest(3, 4, None) == _abi.RIB_OK     # in range: let through
assert R.rib_last_status() == (0, 0)
assert lib.rib_debug_guard_info(info) == 0 and tuple(info) == (0, 0)
assert lib.rib_debug_guard_selftest(5, 4, None) == _abi.RIB_OK     # past the end: refused
code, site = R.rib_last_status()
assert code == _abi.RIB_ERR_BOUNDS and site == 190, (code, site)
assert lib.rib_debug_guard_info(info) == 0 and tuple(info) == (5, 4), tuple(info)
assert lib.rib_debug_guard_info(info) == 0 and tuple(info) == (0, 0)   # cleared by the read
assert R.rib_last_status() == (0, 0)
print("selftest ok")
"""

_RELEASE = r"""
import ctypes
import windowed_attention_implicit_b200 as R
from windowed_attention_implicit_b200 import _abi
lib = R.library()
info = (ctypes.c_ulonglong * 2)()
assert lib.rib_debug_build() == 0
assert lib.rib_debug_guard_selftest(5, 4, None) == _abi.RIB_ERR_UNSUPPORTED
assert lib.rib_debug_guard_info(info) == 0 and tuple(info) == (0, 0)
print("release ok")
"""


@pytest.mark.parametrize("debug,code,word", [(True, _SELFTEST, "selftest ok"),
                                             (False, _RELEASE, "release ok")])
def test_guard_refuses_and_records(debug, code, word):
    if debug:
        B.build(debug=True)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=_env(debug),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and word in r.stdout, (r.stdout + r.stderr)[-3000:]
