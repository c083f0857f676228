"""Parity of the TMA-staged decode GEMV on small and ragged shapes.

Full-size shapes reach the TMA path on their own (packed weights >= 6 MB); here
a child process forces it (BITNET_GEMV_TUNE, read once per process: whole row
blocks per CTA or split mode, several warp/stage variants) for shapes
with ragged row blocks (N not a multiple of 32), partial K-slices (K_pad/4 not
a multiple of 128) and a single row block, int32 and fused-BitLinear outputs.
"""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu

CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
import oracle
import ternary_weight_bit_w2a8_b200 as bn
from ternary_weight_bit_w2a8_b200 import synth
out = {}
for (N, K) in [(1, 512), (5, 640), (31, 700), (33, 1000), (100, 3200), (257, 2560), (1000, 5120)]:
    q, w = synth.uniform_int8_ternary(N, K, seed=N + K)
    packed = bn.bitnet_pack_weights(torch.from_numpy(w).cuda())
    y = bn.bitnet_w2a8_gemm(torch.from_numpy(q).cuda(), packed, N).cpu().numpy()
    ok_i = bool(np.array_equal(y, oracle.gemm_i32(q, w)))
    x, W = synth.bitlinear_inputs(1, N, K, seed=N)
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    yb = bn.bitnet_bitlinear(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16),
                             bn.bitnet_pack_weights(torch.from_numpy(wt).cuda()),
                             torch.tensor([float(g)], dtype=torch.float32, device="cuda"), N)
    yr = oracle.bitlinear(x, wt, g)[0]
    yf = yb.float().cpu().numpy().astype(np.float64)
    err = np.abs(yf - yr)
    ok_b = bool(np.where(np.abs(yr) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(yr)).all())
    out[f"{N}x{K}"] = [ok_i, ok_b]
torch.cuda.synchronize()
out["device_error"] = bn.bitnet_get_device_error()
print(json.dumps(out))
"""


@pytest.mark.parametrize("tune", ["0,0,0,0,-1,0,1",    # TMA path, whole row blocks per CTA
                                  "0,0,0,0,-1,1,1",    # TMA path, split mode (parts + fixup)
                                  "0,0,0,0,-1,1,4",    # split mode, 8 warps x 2 boxes
                                  "0,0,0,0,-1,0,5"])   # 4 warps x 4 boxes
def test_tma_path_forced_small_shapes(tune):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ)
    env["BITNET_GEMV_TUNE"] = tune
    code = "ROOT = " + repr(ROOT) + "\n" + CHILD
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res.pop("device_error") == 0
    bad = {k: v for k, v in res.items() if v != [True, True]}
    assert not bad, bad
