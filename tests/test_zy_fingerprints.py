"""Whole-result bit-identity across processes: the fingerprint method of "Add WMSE weight scale
search calibration" (PR #2283, "Refactor safety"). This process and two fresh ones calibrate
the same layer and must agree on every byte of H, P, the token counts, g, the codes, Wq and the
losses. A kernel that read uninitialised workspace, or summed in an order that varies between
runs, would show here.
"""
import json
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")

from tests import fingerprint as F  # noqa: E402

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import scale_calibration_lh_b200 as L
    from scale_calibration_lh_b200 import build

    build.build()
    L.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


@pytest.mark.parametrize("name,sizes", [
    ("dense", dict(tokens=700, cin=512, rows=96)),
    ("act", dict(tokens=900, cin=256, rows=64)),  # input quantizer fused
    ("moe", dict(tokens=80, cin=96, rows=24, groups=6, top_k=2)),
])
def test_fingerprint_is_identical_across_processes(name, sizes):
    here = F.digest(name, sizes)
    env = dict(os.environ, PYTHONPATH=os.pathsep.join(p for p in (ROOT, os.environ.get("PYTHONPATH")) if p))
    for _ in range(2):
        r = subprocess.run([sys.executable, "-m", "tests.fingerprint", name, json.dumps(sizes)], cwd=ROOT, env=env,
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-3000:]
        assert r.stdout.strip().splitlines()[-1] == here, name
