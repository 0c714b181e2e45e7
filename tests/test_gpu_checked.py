"""The checked build (liblora_linear_checked.so, compiled with -DLORA_CHECKED=1): every
TMA producer tests its tile coordinates and box origins before a copy.  On the ragged
parity shapes, a grouped and a feed-forward case it must give the same parity with
status LORA_OK and every output element written (NaN canaries); on the tensor-core
rank-r pass launched with one tile past the last row it must report
LORA_ERR_DEVICE_BOUNDS, while the regular build, which does not test, computes the real
tiles and stays at LORA_OK (the extra tile's copies are TMA zero fills and its epilogue
writes nothing).  Each case runs in a subprocess that loads the library it names."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "qlora_linear_b200")


def _run(lib_path, what):
    env = dict(os.environ, LORA_LIB_PATH=lib_path)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_worker.py"), what], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1]
    return json.loads(line)


@pytest.fixture(scope="module")
def checked_lib():
    sys.path.insert(0, PKG)
    import build
    return build.build(checked=True)


def test_checked_build_parity_and_bounds(checked_lib):
    import qlora_linear_b200 as q
    d = _run(checked_lib, "all")
    assert d["lib"] == "liblora_linear_checked.so"
    assert len(d["ok"]) >= 12
    assert d["tile"]["launch"] == q.LORA_OK
    assert d["tile"]["device_status"] == q.LORA_ERR_DEVICE_BOUNDS


def test_regular_build_does_not_test_the_extra_tile():
    import qlora_linear_b200 as q
    d = _run(q.LIB_PATH, "tile")
    assert d["lib"] == "liblora_linear.so"
    assert d["tile"]["launch"] == q.LORA_OK and d["tile"]["device_status"] == q.LORA_OK
    assert d["tile"]["rel_err"] < 1e-2  # the real tiles are computed
