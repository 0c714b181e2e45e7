"""Programmatic dependent launch keeps the stream order of every read and write: the
layer kernels launched with it (the default) give the same bits as launched plainly
(LORA_PDL=0), on stream-K shapes of both GEMM kernels, every weight format, both kinds of
rank-r pass and the feed-forward block.  Each setting runs in its own subprocess, since
the library reads the variable once per process."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(pdl):
    env = dict(os.environ, LORA_PDL="1" if pdl else "0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "pdl_worker.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1]
    return json.loads(line)


def test_pdl_gives_the_bits_of_plain_launches():
    on, off = _run(True), _run(False)
    assert on["pdl"] and not off["pdl"]
    assert len(on["cases"]) == 7 and on["cases"].keys() == off["cases"].keys()
    for name in on["cases"]:
        assert on["cases"][name] == off["cases"][name], name
