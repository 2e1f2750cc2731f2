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


def _other_processes_may_open_the_gpu() -> bool:
    """False when NVML reports an exclusive compute mode for the current GPU (read-only query);
    True when it reports the default mode or cannot tell."""
    try:
        import pynvml

        pynvml.nvmlInit()
        vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
        key = vis[torch.cuda.current_device()] if vis else str(torch.cuda.current_device())
        h = (pynvml.nvmlDeviceGetHandleByIndex(int(key)) if key.isdigit()
             else pynvml.nvmlDeviceGetHandleByUUID(key))
        return pynvml.nvmlDeviceGetComputeMode(h) == pynvml.NVML_COMPUTEMODE_DEFAULT
    except Exception:
        return True


@pytest.mark.parametrize("name,sizes", [
    ("dense", dict(tokens=700, cin=512, rows=96)),
    ("act", dict(tokens=900, cin=256, rows=64)),  # input quantizer fused
    ("moe", dict(tokens=80, cin=96, rows=24, groups=6, top_k=2)),
])
def test_fingerprint_is_identical_across_processes(name, sizes):
    if not _other_processes_may_open_the_gpu():
        pytest.skip("the GPU is in an exclusive compute mode: a second process cannot open it")
    here = F.digest(name, sizes)
    env = dict(os.environ, PYTHONPATH=os.pathsep.join(p for p in (ROOT, os.environ.get("PYTHONPATH")) if p))
    for _ in range(2):
        r = subprocess.run([sys.executable, "-m", "tests.fingerprint", name, json.dumps(sizes)], cwd=ROOT, env=env,
                           capture_output=True, text=True, timeout=600)
        if r.returncode != 0 and "busy or unavailable" in r.stderr:
            pytest.skip("a second process could not open the GPU")
        assert r.returncode == 0, r.stderr[-3000:]
        assert r.stdout.strip().splitlines()[-1] == here, name
