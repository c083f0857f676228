"""Failure detection on the GPU without a fault: a bounded wait that runs out.

A child process sets BITNET_TEST_STALL=1, which makes the first TMA-staged
GEMV launch skip one box request, so one warp's wait on that box can never
complete.  The wait gives up after its time limit (1 s), the kernel records
BITNET_ERR_DEVICE_TIMEOUT and returns; the host reads the status with
bitnet_get_device_error, which clears it, and the context stays usable: the
next call on the same stream is exact again.
"""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu

CHILD = r"""
import json, sys, time
import numpy as np, torch
sys.path.insert(0, ROOT)
import oracle
import ternary_weight_bit_w2a8_b200 as bn
from ternary_weight_bit_w2a8_b200 import synth
N, K = 1000, 2560
q, w = synth.uniform_int8_ternary(N, K, seed=5)
qd = torch.from_numpy(q).cuda()
packed = bn.bitnet_pack_weights(torch.from_numpy(w).cuda())
t0 = time.time()
bn.bitnet_w2a8_gemm(qd, packed, N)          # the stalled launch
status = bn.bitnet_get_device_error()
dt = time.time() - t0
again = bn.bitnet_get_device_error()         # cleared by the first read
y = bn.bitnet_w2a8_gemm(qd, packed, N).cpu().numpy()
exact = bool(np.array_equal(y, oracle.gemm_i32(q, w)))
print(json.dumps({"status": status, "again": again, "exact_after": exact, "seconds": dt,
                  "final": bn.bitnet_get_device_error()}))
"""


# the planner's variant; 16 warps; per-slice staging barriers
@pytest.mark.parametrize("tune", [None, "0,0,0,0,-1,0,3", "0,0,0,0,-1,0,-1,0,-1,0,0,-1,-1,-1,1"])
def test_bounded_wait_reports_timeout_and_context_survives(tune):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_weight_bit_w2a8_b200 as bn
    env = dict(os.environ)
    env["BITNET_TEST_STALL"] = "1"
    env.pop("BITNET_GEMV_TUNE", None)
    if tune is not None:
        env["BITNET_GEMV_TUNE"] = tune
    r = subprocess.run([sys.executable, "-c", "ROOT = " + repr(ROOT) + "\n" + CHILD], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["status"] == bn.BITNET_ERR_DEVICE_TIMEOUT
    assert res["again"] == bn.BITNET_OK
    assert res["exact_after"]
    assert res["final"] == bn.BITNET_OK
    assert 0.5 < res["seconds"] < 60
