"""Parity of the small-batch decode (2..16 tokens through the TMA-staged GEMV's
MMA product, every weight box read once for all tokens): int32 and BitLinear
outputs on ragged shapes and token counts that leave unused token slots."""
import numpy as np
import pytest

import oracle
import ternary_weight_bit_w2a8_b200 as bn
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


@pytest.mark.parametrize("M,N,K", [(2, 1000, 2560), (3, 33, 700), (4, 257, 1024), (5, 300, 5120), (7, 64, 3200),
                                   (8, 2560, 6912), (6, 13824, 2560), (9, 300, 2560), (13, 33, 700),
                                   (12, 2560, 6912), (16, 13824, 2560), (16, 5120, 3200)])
def test_small_batch_int32_exact(M, N, K):
    q, w = synth.uniform_int8_ternary(N, K, seed=M * 1000 + N + K, M=M)
    q[-1, :7] = -128
    y = bn.bitnet_w2a8_gemm(torch.from_numpy(q).cuda(), bn.bitnet_pack_weights(torch.from_numpy(w).cuda()), N)
    assert np.array_equal(y.cpu().numpy(), oracle.gemm_i32(q, w))


# 2..4 tokens are quantised inside the GEMV prologue, 5..16 in a pass of their
# own first: both sides of that boundary are here
@pytest.mark.parametrize("M,N,K", [(2, 500, 2560), (3, 6912, 2560), (4, 257, 1536), (5, 300, 3200),
                                   (8, 2560, 6912), (11, 300, 3200), (16, 2560, 6912)])
def test_small_batch_bitlinear(M, N, K):
    x, W = synth.bitlinear_inputs(M, N, K, seed=M)
    x[1] = 0  # a zero token among them
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    y = bn.bitnet_bitlinear(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16),
                            bn.bitnet_pack_weights(torch.from_numpy(wt).cuda()),
                            torch.tensor([float(g)], dtype=torch.float32, device="cuda"), N)
    y_ref = oracle.bitlinear(x, wt, g)[0]
    yf = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(yf - y_ref)
    assert np.where(np.abs(y_ref) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(y_ref)).all()
    assert not y.view(torch.int16).cpu().numpy()[1].any()


def test_bitlinear_same_bits_on_every_path():
    """A token's bf16 output does not depend on which path quantised it: the
    single-token prologue (1 token), the multi-token prologue (2..4), a
    quantisation pass before the GEMV (5..16) or before the tensor-core GEMM
    (17 and more).  All of them take the scale and the codes with the same fp32
    operations and rescale the same way, so the shared tokens' outputs must be
    identical bit for bit (a one-ulp scale difference would change codes)."""
    N, K = 300, 2560
    x, W = synth.bitlinear_inputs(20, N, K, seed=5)
    x[7, :] = 0
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    packed = bn.bitnet_pack_weights(torch.from_numpy(wt).cuda())
    gamma = torch.tensor([float(g)], dtype=torch.float32, device="cuda")
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    outs = {M: bn.bitnet_bitlinear(xd[:M].contiguous(), packed, gamma, N).view(torch.int16).cpu().numpy()
            for M in (1, 2, 3, 4, 5, 8, 9, 12, 16, 17, 20)}
    full = outs[20]
    for M, y in outs.items():
        assert np.array_equal(y, full[:M]), f"{M} tokens: bf16 bits differ from the 20-token run"
    y_ref = oracle.bitlinear(x, wt, g)[0]
    yf = torch.from_numpy(full).view(torch.bfloat16).float().numpy().astype(np.float64)
    err = np.abs(yf - y_ref)
    assert np.where(np.abs(y_ref) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(y_ref)).all()


FUSED_CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
import oracle
import ternary_weight_bit_w2a8_b200 as bn
from ternary_weight_bit_w2a8_b200 import synth
out = {}
for (M, N, K) in [(5, 300, 3200), (8, 2560, 6912), (11, 300, 3200), (13, 33, 700), (16, 2560, 2560)]:
    x, W = synth.bitlinear_inputs(M, N, K, seed=M + N)
    x[1] = 0
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    y = bn.bitnet_bitlinear(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16),
                            bn.bitnet_pack_weights(torch.from_numpy(wt).cuda()),
                            torch.tensor([float(g)], dtype=torch.float32, device="cuda"), N)
    yr = oracle.bitlinear(x, wt, g)[0]
    err = np.abs(y.float().cpu().numpy().astype(np.float64) - yr)
    out[f"{M}x{N}x{K}"] = bool(np.where(np.abs(yr) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(yr)).all()
                               and not y.view(torch.int16).cpu().numpy()[1].any())
# the bits do not depend on the token count (prologue for 1..16, GEMM launch beyond)
N, K = 300, 2560
x, W = synth.bitlinear_inputs(20, N, K, seed=5)
g = oracle.absmean(W)
wt = oracle.ternarize(W, g)
packed = bn.bitnet_pack_weights(torch.from_numpy(wt).cuda())
gamma = torch.tensor([float(g)], dtype=torch.float32, device="cuda")
xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
outs = {M: bn.bitnet_bitlinear(xd[:M].contiguous(), packed, gamma, N).view(torch.int16).cpu().numpy()
        for M in (1, 2, 4, 5, 8, 9, 16, 20)}
for M, y in outs.items():
    out[f"same bits {M}"] = bool(np.array_equal(y, outs[20][:M]))
torch.cuda.synchronize()
out["device_error"] = bn.bitnet_get_device_error()
print(json.dumps(out))
"""


def test_bitlinear_quantised_inside_the_launch_for_every_token_count():
    """Tuning field fuse = 1: 2..16 tokens are quantised inside the GEMV's
    prologue (all tokens of a CTA's launch at once) instead of a pass of their
    own; outputs within the oracle's tolerance and bit-identical to the
    20-token run's (quantised inside the tensor-core GEMM launch)."""
    import json
    import os
    import subprocess
    import sys
    from conftest import ROOT
    env = dict(os.environ)
    env["BITNET_GEMV_TUNE"] = "0,0,0,0,-1,0,-1,0,1"
    r = subprocess.run([sys.executable, "-c", "ROOT = " + repr(ROOT) + "\n" + FUSED_CHILD], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res.pop("device_error") == 0
    bad = {k: v for k, v in res.items() if not v}
    assert not bad, bad
