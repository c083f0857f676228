"""Out-of-bounds writes: every output, quantised-activation buffer and
workspace handed to the library sits between guard bands of canary bytes (see
guarded.py), and each case checks both the bands and the result against the
oracle.  The cases reach every store path: the TMA GEMV epilogue on ragged row
blocks, the register GEMV and its K-split partials in the workspace, the
tensor-core GEMM's TMA-box stores and its direct stores (output rows whose
byte length is not a multiple of 16), its K-split (zeroed output plus TMA
reduce-add), the repack of unaligned activations into the workspace, the
BitLinear quantisation into the workspace and the rescale after a K-split,
and the offline kernels (absmean, ternarise, pack, activation quantisation).
"""
import numpy as np
import pytest

import oracle
import ternary_weight_bit_w2a8_b200 as bn
from guarded import Guarded, guarded_workspace
from ternary_weight_bit_w2a8_b200 import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

BF16_SENTINEL = 0x7F7F  # 3.39e38 as bf16: an output left unwritten fails the tolerance


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ternary_weight_bit_w2a8_b200 import build
    build.build()
    oracle._lib()
    yield
    torch.cuda.synchronize()
    assert bn.bitnet_get_device_error() == 0


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_ok(y, y_ref):
    yf = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(yf - y_ref)
    ok = np.where(np.abs(y_ref) < 0.1, err <= 1e-3, err <= 1e-2 * np.abs(y_ref))
    return bool(np.isfinite(yf).all() and ok.all())


# (M, N, K): which path each takes under the default plan
GEMM_CASES = [
    (1, 257, 2560),    # TMA GEMV, ragged last row block
    (1, 1000, 5120),   # TMA GEMV, several row blocks per CTA
    (1, 5115, 27648),  # TMA GEMV, 160 row blocks on 148 CTAs (12 take two), ragged last block
    (13, 300, 2560),   # small batch, 16-token MMA tiles
    (1, 300, 300),     # register GEMV (K < 512)
    (1, 64, 65536),    # register GEMV... or TMA; either way the plan's scratch is guarded
    (1, 20, 200000),   # K-split register GEMV: int32 partials in the workspace
    (3, 100, 3200),    # small batch (TMA GEMV, 4-token slots, one unused)
    (8, 33, 1024),     # small batch, 8 tokens
    (40, 257, 1024),   # tensor-core GEMM, direct stores (257 * 4 bytes is not a multiple of 16)
    (200, 512, 2560),  # tensor-core GEMM, TMA-box stores
    (64, 200, 8192),   # tensor-core GEMM with a K-split (2 tiles for 148 SMs)
    (20, 130, 999),    # K not a multiple of 16: activations repacked into the workspace
]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_gemm_guard_bands(M, N, K):
    q, w = synth.uniform_int8_ternary(N, K, seed=M * 7 + N + K, M=M)
    q[0, :3] = -128
    qg = Guarded(torch, (M, K), torch.int8, fill=torch.from_numpy(q))
    pg = Guarded(torch, (bn.bitnet_packed_bytes(N, K),), torch.uint8)
    bn.bitnet_pack_weights(dev(w), packed=pg.t)
    yg = Guarded(torch, (M, N), torch.int32, fill=-7)
    wsg = guarded_workspace(torch, bn, M, N, K)
    bn.bitnet_w2a8_gemm(qg.t, pg.t, N, y=yg.t, ws=wsg.t)
    torch.cuda.synchronize()
    assert np.array_equal(yg.t.cpu().numpy(), oracle.gemm_i32(q, w))
    yg.check("y")
    wsg.check("the workspace")
    qg.check("q (read only)")
    pg.check("the packed weights")
    assert np.array_equal(pg.t.cpu().numpy(), oracle.pack_device(w)[0].reshape(-1))


BITLINEAR_CASES = [
    (1, 257, 2560),    # fused quantisation in the GEMV prologue
    (3, 130, 1536),    # 3 tokens fused
    (6, 300, 3200),    # 6 tokens: quantised into the workspace first
    (40, 257, 1024),   # tensor-core GEMM, bf16 direct stores (257 * 2 bytes)
    (130, 512, 2560),  # tensor-core GEMM, bf16 TMA-box stores
    (64, 200, 8192),   # K-split: int32 sums in the workspace, then the rescale
    (9, 40, 300),      # tensor-core path with K < 512
]


@pytest.mark.parametrize("M,N,K", BITLINEAR_CASES)
def test_bitlinear_guard_bands(M, N, K):
    x, W = synth.bitlinear_inputs(M, N, K, seed=M + N)
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    xg = Guarded(torch, (M, K), torch.int16, fill=torch.from_numpy(x.view(np.int16)))
    yg = Guarded(torch, (M, N), torch.int16, fill=BF16_SENTINEL)
    wsg = guarded_workspace(torch, bn, M, N, K)
    gg = Guarded(torch, (1,), torch.float32, fill=float(g))
    bn.bitnet_bitlinear(xg.t.view(torch.bfloat16), bn.bitnet_pack_weights(dev(wt)), gg.t, N,
                        y=yg.t.view(torch.bfloat16), ws=wsg.t)
    torch.cuda.synchronize()
    assert bf16_ok(yg.t.view(torch.bfloat16), oracle.bitlinear(x, wt, g)[0])
    yg.check("y")
    wsg.check("the workspace")
    xg.check("x (read only)")
    gg.check("gamma (read only)")


@pytest.mark.parametrize("M,K", [(1, 7), (3, 4097), (5, 2560)])
def test_quant_act_guard_bands(M, K):
    x = synth.bf16_activations(M, K, seed=M + K)
    qg = Guarded(torch, (M, K), torch.int8, fill=99)
    sg = Guarded(torch, (M,), torch.float32)
    rg = Guarded(torch, (M,), torch.int32)
    bn.bitnet_quant_act(dev(x.view(np.int16)).view(torch.bfloat16), q=qg.t, s=sg.t, rowsum=rg.t)
    q_ref, s_ref, rs_ref = oracle.quant_act(x)
    assert np.array_equal(qg.t.cpu().numpy(), q_ref)
    assert np.array_equal(sg.t.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(rg.t.cpu().numpy(), rs_ref)
    for b, name in ((qg, "q"), (sg, "s"), (rg, "rowsum")):
        b.check(name)


@pytest.mark.parametrize("N,K", [(1, 1), (3, 129), (7, 33), (33, 1000)])
def test_offline_kernels_guard_bands(N, K):
    W = synth.bf16_weights(N, K, seed=N + K)
    Wd = dev(W.view(np.int16)).view(torch.bfloat16)
    gg = Guarded(torch, (1,), torch.float32)
    wsg = guarded_workspace(torch, bn, 0, N, K)
    bn.bitnet_absmean(Wd, gamma=gg.t, ws=wsg.t)
    g_ref = oracle.absmean(W)
    assert abs(float(gg.t.item()) - float(g_ref)) <= 1e-6 * float(g_ref)
    tg = Guarded(torch, (N, K), torch.int8)
    bn.bitnet_ternarize(Wd, dev(np.array([g_ref], np.float32)), W_t=tg.t)
    wt_ref = oracle.ternarize(W, g_ref)
    assert np.array_equal(tg.t.cpu().numpy(), wt_ref)
    pg = Guarded(torch, (bn.bitnet_packed_bytes(N, K),), torch.uint8)
    cg = Guarded(torch, (1,), torch.int32)
    bn.bitnet_pack_weights(tg.t, packed=pg.t, invalid_count=cg.t)
    assert np.array_equal(pg.t.cpu().numpy(), oracle.pack_device(wt_ref)[0].reshape(-1))
    assert int(cg.t.item()) == 0
    for b, name in ((gg, "gamma"), (wsg, "the absmean workspace"), (tg, "W_t"), (pg, "packed"),
                    (cg, "invalid_count")):
        b.check(name)
