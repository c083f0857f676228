"""Parity of the tcgen05 tensor-core GEMM (M > 1) with the oracle.

Ragged shapes (M, N not multiples of the tile, K not a multiple of the
128-byte stage or of 16, which makes the library repack the activations), every
token-tile width with and without a K-split (forced in child processes through
BITNET_GEMV_TUNE, read once per process, with outputs and workspaces between
guard bands), problems with many work units per persistent CTA, int32 and
BitLinear bf16 outputs.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle
import ternary_weight_bit_w2a8_b200 as bn
from conftest import ROOT
from ternary_weight_bit_w2a8_b200 import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ternary_weight_bit_w2a8_b200 import build
    build.build()
    yield
    torch.cuda.synchronize()
    assert bn.bitnet_get_device_error() == 0


@pytest.mark.parametrize("M,N,K", [(2, 1, 128), (2, 16, 128), (127, 100, 256), (129, 257, 384), (255, 1000, 1040),
                                   (130, 300, 200), (64, 513, 2560), (300, 96, 999)])
def test_tc_gemm_ragged_exact(M, N, K):
    q, w = synth.uniform_int8_ternary(N, K, seed=M + N + K, M=M)
    q[0, :] = -128  # the int8 extreme in one token
    y = bn.bitnet_w2a8_gemm(torch.from_numpy(q).cuda(), bn.bitnet_pack_weights(torch.from_numpy(w).cuda()), N)
    assert np.array_equal(y.cpu().numpy(), oracle.gemm_i32(q, w))


def test_tc_gemm_misaligned_activation_rows():
    # rows of q start at odd offsets: the library repacks them into a workspace
    M, N, K = 5, 200, 777
    q, w = synth.uniform_int8_ternary(N, K, seed=3, M=M)
    base = torch.zeros(M * K + 1, dtype=torch.int8, device="cuda")
    qd = base[1:].view(M, K)
    qd.copy_(torch.from_numpy(q))
    y = bn.bitnet_w2a8_gemm(qd, bn.bitnet_pack_weights(torch.from_numpy(w).cuda()), N)
    assert np.array_equal(y.cpu().numpy(), oracle.gemm_i32(q, w))


@pytest.mark.parametrize("M,N,K", [(2, 33, 300), (129, 200, 2560)])
def test_tc_bitlinear(M, N, K):
    x, W = synth.bitlinear_inputs(M, N, K, seed=1)
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    y = bn.bitnet_bitlinear(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16),
                            bn.bitnet_pack_weights(torch.from_numpy(wt).cuda()),
                            torch.tensor([float(g)], dtype=torch.float32, device="cuda"), N)
    y_ref = oracle.bitlinear(x, wt, g)[0]
    yf = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(yf - y_ref)
    assert np.where(np.abs(y_ref) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(y_ref)).all()


CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import oracle
import ternary_weight_bit_w2a8_b200 as bn
from guarded import Guarded, guarded_workspace
from ternary_weight_bit_w2a8_b200 import synth
out = {}
for (M, N, K) in [(130, 300, 1000), (256, 520, 2560), (9, 1000, 384), (40, 129, 640), (300, 64, 4096),
                  (2000, 4096, 256), (150, 257, 2900)]:
    q, w = synth.uniform_int8_ternary(N, K, seed=M * N + K, M=M)
    q[-1, :] = -128
    yg = Guarded(torch, (M, N), torch.int32, fill=-7)
    wsg = guarded_workspace(torch, bn, M, N, K)
    bn.bitnet_w2a8_gemm(torch.from_numpy(q).cuda(), bn.bitnet_pack_weights(torch.from_numpy(w).cuda()), N,
                        y=yg.t, ws=wsg.t)
    out[f"{M}x{N}x{K}"] = bool(np.array_equal(yg.t.cpu().numpy(), oracle.gemm_i32(q, w)))
    out[f"{M}x{N}x{K} guards"] = yg.intact() and wsg.intact()
for (M, N, K) in [(33, 200, 1000), (260, 96, 512), (150, 257, 2900)]:
    x, W = synth.bitlinear_inputs(M, N, K, seed=M)
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    yg = Guarded(torch, (M, N), torch.int16, fill=0x7F7F)
    wsg = guarded_workspace(torch, bn, M, N, K)
    bn.bitnet_bitlinear(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16),
                        bn.bitnet_pack_weights(torch.from_numpy(wt).cuda()),
                        torch.tensor([float(g)], dtype=torch.float32, device="cuda"), N,
                        y=yg.t.view(torch.bfloat16), ws=wsg.t)
    yr = oracle.bitlinear(x, wt, g)[0]
    yf = yg.t.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
    err = np.abs(yf - yr)
    out[f"bitlinear {M}x{N}x{K}"] = bool(np.isfinite(yf).all() and
                                         np.where(np.abs(yr) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(yr)).all())
    out[f"bitlinear {M}x{N}x{K} guards"] = yg.intact() and wsg.intact()
torch.cuda.synchronize()
out["device_error"] = bn.bitnet_get_device_error()
print(json.dumps(out))
"""


# variant 1..10 = token tiles of 192, 128 (512-k stages), 64, 32, 16, then 128,
# 96 and 64 with 4, 5 and 6 code stages, then 128 and 192 with one accumulator
# (6 and 5 code stages); S = K-splits (0: none when forced).  The
# 2000 x 4096 problem gives every persistent CTA several work units, so both
# accumulators are reused many times; K = 2900 is not a multiple of the
# 128-token tile's 512-k stage, so (2, 3) splits with a partial last stage.
# Outputs (257 columns: direct stores) and workspaces sit between guard bands.
@pytest.mark.parametrize("tile,S", [(1, 0), (2, 0), (3, 0), (4, 0), (5, 0), (6, 0), (7, 0), (8, 0), (9, 0), (10, 0),
                                    (1, 3), (2, 3), (3, 5), (5, 2), (6, 4), (9, 3)])
def test_tc_every_tile_width(tile, S):
    env = dict(os.environ)
    env["BITNET_GEMV_TUNE"] = f"0,-{tile},0,0,-1,{S},-1"
    r = subprocess.run([sys.executable, "-c", "ROOT = " + repr(ROOT) + "\n" + CHILD], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res.pop("device_error") == 0
    assert all(res.values()), res


def test_bitlinear_with_quantisation_inside_the_gemm_launch():
    """The alternative prefill path (tuning field fuse = 1): the GEMM launch
    quantises the activations itself, its CTAs meeting at a grid barrier
    before the first activation load; same cases, guard bands and checks."""
    env = dict(os.environ)
    env["BITNET_GEMV_TUNE"] = "0,0,0,0,-1,0,-1,0,1"
    r = subprocess.run([sys.executable, "-c", "ROOT = " + repr(ROOT) + "\n" + CHILD], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res.pop("device_error") == 0
    assert all(res.values()), res
