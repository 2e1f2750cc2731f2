"""Bit-identity fingerprint of one calibration: SHA-256 over the bytes of every output.

Run as ``python -m tests.fingerprint <workload> '<json sizes>'`` from the repository root,
it prints the fingerprint of a fresh process's run. The GPU tests compare it across
processes; this is the whole-result bit-identity check of "Add WMSE weight scale search
calibration" (PR #2283, "Refactor safety").
"""
import hashlib
import json
import sys


def digest(name: str, sizes: dict, seed: int = 91) -> str:
    import torch

    import scale_calibration_lh_b200 as L
    from tests import parity as P

    layer = P.make_layer(name, seed, **sizes)
    d = P.layer_to_device(layer)
    b = L.calibrate(layer.mode, d["x"], d["w"], group_offsets=d["offs"], token_ids=d["ids"], act_gx=d["act_gx"])
    torch.cuda.synchronize()
    h = hashlib.sha256()
    for t in (b.h, b.p, b.counts, b.g, b.codes, b.wq, b.loss):
        if t is not None:
            h.update(t.contiguous().cpu().numpy().tobytes())
    return h.hexdigest()


if __name__ == "__main__":
    print(digest(sys.argv[1], json.loads(sys.argv[2])))
