"""Parity of the TMA-staged decode GEMV under every launch variant.

A child process forces the variant (BITNET_GEMV_TUNE, read once per process:
warps per CTA, ring depth, CTAs per SM) on shapes with ragged row blocks (N
not a multiple of 32), partial K-slices (K_pad/4 not a multiple of 128), a
single row block, several row blocks per CTA, and 1, 3, 8 or 13 tokens (the
last three on the MMA product); int32 and BitLinear outputs.
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
sys.path.insert(0, ROOT + "/tests")
import oracle
from guarded import Guarded
import ternary_weight_bit_w2a8_b200 as bn
from ternary_weight_bit_w2a8_b200 import synth
out = {}
SHAPES = [(1, 512), (5, 640), (31, 700), (33, 1000), (100, 3200), (257, 2560), (1000, 5120), (70, 10240),
          (65, 16384), (300, 27648), (4800, 3200), (4832, 27648), (20000, 3200)]
for (N, K) in SHAPES:
    for M in (1, 3, 8, 13):
        q, w = synth.uniform_int8_ternary(N, K, seed=N + K + M, M=M)
        q[0, :5] = -128
        packed = bn.bitnet_pack_weights(torch.from_numpy(w).cuda())
        yg = Guarded(torch, (M, N), torch.int32, fill=-7)
        bn.bitnet_w2a8_gemm(torch.from_numpy(q).cuda(), packed, N, y=yg.t)
        ok_i = bool(np.array_equal(yg.t.cpu().numpy(), oracle.gemm_i32(q, w))) and yg.intact()
        ok_b = True
        if M in (1, 3, 13):
            x, W = synth.bitlinear_inputs(M, N, K, seed=N + M)
            g = oracle.absmean(W)
            wt = oracle.ternarize(W, g)
            ybg = Guarded(torch, (M, N), torch.int16, fill=0x7F7F)
            bn.bitnet_bitlinear(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16),
                                bn.bitnet_pack_weights(torch.from_numpy(wt).cuda()),
                                torch.tensor([float(g)], dtype=torch.float32, device="cuda"), N,
                                y=ybg.t.view(torch.bfloat16))
            yb = ybg.t.view(torch.bfloat16)
            yr = oracle.bitlinear(x, wt, g)[0]
            yf = yb.float().cpu().numpy().astype(np.float64)
            err = np.abs(yf - yr)
            ok_b = bool(np.where(np.abs(yr) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(yr)).all()) and ybg.intact()
        out[f"{M}x{N}x{K}"] = [ok_i, ok_b]
torch.cuda.synchronize()
out["device_error"] = bn.bitnet_get_device_error()
print(json.dumps(out))
"""


# BITNET_GEMV_TUNE = "G,R,U,ctas_per_sm,prefetch,S,variant,ring,fuse,qwpt,rows,cores,mma,l2,sflags":
# variant 1..5 = 8x4, 12x3, 16x2, 8x2, 4x4 (warps x most boxes per warp), rows
# per block 16 or 32, cores = 1 the co-residency mode (two CTAs per SM), mma =
# 1 / 0 the MMA or the dp4a product for one token, l2 = 0 weights without the
# L2 evict-first policy, sflags = 1 / 0 per-slice staging barriers always /
# never.  4832 x 27648 and 20000 x
# 3200 leave 3 and 136 CTAs with one 32-row block more than the others.
@pytest.mark.parametrize("tune", ["0,0,0,0,-1,0,-1",     # the planner's own choice
                                  "0,0,0,0,-1,0,1",      # 8 warps, ring up to 4
                                  "0,0,0,0,-1,0,3",      # 16 warps, ring up to 2
                                  "0,0,0,2,-1,0,4",      # 8 warps, ring up to 2, 2 CTAs per SM
                                  "0,0,0,0,-1,0,5",      # 4 warps, ring up to 4
                                  "0,0,0,0,-1,0,2,1",    # 12 warps, ring of 1
                                  "0,0,0,0,-1,0,-1,0,-1,0,16",   # 16-row blocks (two lanes per row)
                                  "0,0,0,0,-1,0,1,0,-1,0,16",    # 16-row blocks, 8 warps, ring up to 4
                                  "0,0,0,0,-1,0,-1,0,-1,0,0,1",  # co-residency mode (16-row blocks below 148)
                                  "0,0,0,0,-1,0,-1,0,-1,0,32,1",  # co-residency mode, 32-row blocks
                                  "0,0,0,0,-1,0,-1,0,-1,0,0,-1,1",  # MMA product for one token too
                                  "0,0,0,0,-1,0,1,0,-1,0,16,-1,1",  # MMA, 16-row blocks, 8 warps
                                  "0,0,0,0,-1,0,2,0,-1,0,0,-1,1",  # MMA, 12 warps
                                  "0,0,0,0,-1,0,-1,0,-1,0,0,-1,0",  # dp4a product for one token
                                  "0,0,0,0,-1,0,-1,0,-1,0,0,-1,-1,0",  # weights without the evict-first policy
                                  "0,0,0,0,-1,0,-1,0,-1,0,0,-1,-1,-1,1",  # per-slice staging barriers always
                                  "0,0,0,0,-1,0,5,0,-1,0,16,-1,-1,-1,1",  # the same, 4 warps, 16-row blocks
                                  "0,0,0,0,-1,0,-1,0,-1,0,0,-1,-1,-1,0"])  # never
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
