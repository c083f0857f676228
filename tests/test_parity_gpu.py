"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same
seeded inputs: bit-exact for packing, ternary codes, int8 codes and the int32
contraction; bf16 BitLinear outputs within max relative error 1e-2 (absolute
1e-3 where |y_ref| < 0.1) of the fp64 oracle.

Full-size cases use the same entry points, and hence the same launch plans,
as bench.py."""
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
    oracle._lib()
    yield
    torch.cuda.synchronize()
    assert bn.bitnet_get_device_error() == 0


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def pack_on_gpu(w):
    return bn.bitnet_pack_weights(dev(w))


def bf16_tensor(bits):
    return dev(bits.view(np.int16)).view(torch.bfloat16)


def check_bf16(y_gpu, y_ref):
    """max relative error 1e-2, absolute 1e-3 where |y_ref| < 0.1."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(y).all(), "non-finite bf16 output"
    err = np.abs(y - y_ref)
    near = np.abs(y_ref) < 0.1
    bad = np.where(near, err > 1e-3, err > 1e-2 * np.abs(y_ref))
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside tolerance; worst abs err "
                           f"{err.max():.3g}")


# ------------------------------------------------------------------ packing

@pytest.mark.parametrize("N,K", [(1, 1), (3, 17), (5, 64), (2, 127), (4, 128), (3, 129), (17, 1000),
                                 (64, 2560), (31, 6912)])
def test_pack_bit_exact(N, K):
    _, w = synth.uniform_int8_ternary(N, K, seed=N + K)
    got = host(pack_on_gpu(w))
    ref, bad = oracle.pack_device(w)
    assert bad == 0
    assert np.array_equal(got, ref.reshape(-1))


def test_pack_invalid_count():
    w = np.array([[1, 2, -1, -5, 0, 127, 1, 1]] * 3, dtype=np.int8)
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = host(bn.bitnet_pack_weights(dev(w), invalid_count=cnt))
    ref, bad = oracle.pack_device(w)
    assert int(cnt.item()) == bad == 9
    assert np.array_equal(got, ref.reshape(-1))


# ------------------------------------------------------------------ ternarisation

@pytest.mark.parametrize("N,K", [(1, 1), (7, 33), (256, 2560), (6912, 2560)])
def test_absmean_and_ternarize(N, K):
    W = synth.bf16_weights(N, K, seed=N * 7 + K)
    g_ref = oracle.absmean(W)
    g = bn.bitnet_absmean(bf16_tensor(W))
    assert abs(float(g.item()) - float(g_ref)) <= 1e-6 * float(g_ref)
    # the ternary decision is taken with the oracle's scale on both sides
    wt = bn.bitnet_ternarize(bf16_tensor(W), dev(np.array([g_ref], np.float32)))
    assert np.array_equal(host(wt), oracle.ternarize(W, g_ref))


def test_ternarize_golden_ties_and_zero():
    W = np.array([[0x3E80, 0xBE80, 0x3F40, 0x0000, 0x3F00, 0xC000]], np.uint16)
    g = np.float32(0.5)
    wt = host(bn.bitnet_ternarize(bf16_tensor(W), dev(np.array([g], np.float32))))
    assert wt.tolist() == oracle.ternarize(W, g).tolist() == [[0, 0, 1, 0, 1, -1]]
    z = host(bn.bitnet_ternarize(bf16_tensor(W), dev(np.array([0.0], np.float32))))
    assert not z.any()
    gz = bn.bitnet_absmean(bf16_tensor(np.zeros((3, 5), np.uint16)))
    assert float(gz.item()) == 0.0


# ------------------------------------------------------------------ activation quant

@pytest.mark.parametrize("M,K", [(1, 1), (1, 7), (3, 100), (1, 2560), (1, 6912), (5, 4097), (128, 2560)])
def test_quant_act_bit_exact(M, K):
    x = synth.bf16_activations(M, K, seed=M * 31 + K)
    q, s, rs = bn.bitnet_quant_act(bf16_tensor(x))
    q_ref, s_ref, rs_ref = oracle.quant_act(x)
    assert np.array_equal(host(q), q_ref)
    assert np.array_equal(host(s).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(host(rs), rs_ref)


def test_quant_act_golden():
    x = synth.f32_to_bf16_bits(np.array([[2, -1, 0.5], [127, 2.5, -0.5], [0, 0, 0]], np.float32))
    q, s, rs = bn.bitnet_quant_act(bf16_tensor(x))
    assert host(q).tolist() == [[127, -64, 32], [127, 2, 0], [0, 0, 0]]
    assert host(rs).tolist() == [95, 129, 0]


# ------------------------------------------------------------------ GEMV (M = 1)

def gemv_case(N, K, seed, gen=synth.uniform_int8_ternary, M=1):
    q, w = gen(N, K, seed=seed, M=M)
    packed = pack_on_gpu(w)
    y = host(bn.bitnet_w2a8_gemm(dev(q), packed, N))
    return q, w, y


@pytest.mark.parametrize("N,K", [(1, 1), (1, 16), (3, 17), (17, 64), (65, 127), (129, 129), (257, 300),
                                 (1000, 2624), (33, 3200), (8, 10240), (100, 6912), (7, 27648)])
def test_gemv_small_shapes_exact(N, K):
    q, w, y = gemv_case(N, K, seed=N * 13 + K)
    assert np.array_equal(y, oracle.gemm_i32(q, w))


def test_gemv_extreme_values():
    N, K = 96, 8192
    w = np.ones((N, K), np.int8)
    w[N // 2:] = -1
    packed = pack_on_gpu(w)
    for val in (-128, 127):
        q = np.full((1, K), val, np.int8)
        y = host(bn.bitnet_w2a8_gemm(dev(q), packed, N))
        assert np.array_equal(y, oracle.gemm_i32(q, w))
    # codes of 2 and activations of -128 at the maximal K the tests afford
    K = 1 << 17
    w = np.ones((3, K), np.int8)
    q = np.full((1, K), -128, np.int8)
    y = host(bn.bitnet_w2a8_gemm(dev(q), pack_on_gpu(w), 3))
    assert y.tolist() == [[-128 * K] * 3]


# The TMA-staged GEMV keeps one row's whole K on one lane: |acc_j| <= 4096 K per
# lane is exact for K <= 2^19, and its shared-memory plan caps K well below
# that.  Forced to its smallest ring (4 warps x 1 box: the most room for the
# activations), it takes K = 208896 in one CTA; all weights +1 (code 2, the
# largest scaled code) against activations of -128 is the extreme there.
TMA_MAX_K_CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
import ternary_weight_bit_w2a8_b200 as bn
out = {}
for (N, K) in [(32, 208896), (5, 163840), (64, 131072)]:
    w = np.ones((N, K), np.int8)
    packed = bn.bitnet_pack_weights(torch.from_numpy(w).cuda())
    for val in (-128, 127):
        q = np.full((1, K), val, np.int8)
        y = bn.bitnet_w2a8_gemm(torch.from_numpy(q).cuda(), packed, N).cpu().numpy()
        out[f"{N}x{K}x{val}"] = bool((y == val * K).all())
    w[:, 1::2] = -1
    q = np.full((1, K), -128, np.int8)
    y = bn.bitnet_w2a8_gemm(torch.from_numpy(q).cuda(), bn.bitnet_pack_weights(torch.from_numpy(w).cuda()),
                            N).cpu().numpy()
    out[f"{N}x{K} alternating"] = bool((y == 0).all())
torch.cuda.synchronize()
out["device_error"] = bn.bitnet_get_device_error()
out["launches"] = bn.bitnet_launch_count()
print(json.dumps(out))
"""


def test_gemv_tma_largest_k_extremes():
    import json
    import os
    import subprocess
    import sys
    from conftest import ROOT
    env = dict(os.environ)
    env["BITNET_GEMV_TUNE"] = "0,0,0,0,-1,0,5,1"  # TMA GEMV variant of 4 warps, ring of one box
    r = subprocess.run([sys.executable, "-c", "ROOT = " + repr(ROOT) + "\n" + TMA_MAX_K_CHILD], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res.pop("device_error") == 0
    assert res.pop("launches") > 0
    assert all(res.values()), res


@pytest.mark.parametrize("N,K", [(64, 65536), (3, 100000), (200, 200000)])
def test_gemv_split_k_exact(N, K):
    q, w, y = gemv_case(N, K, seed=K)
    assert np.array_equal(y, oracle.gemm_i32(q, w))


@pytest.mark.parametrize("N,K", [(2560, 2560)])
def test_gemv_small_config_exact(N, K):
    q, w, y = gemv_case(N, K, seed=0)
    assert np.array_equal(y, oracle.gemm_i32(q, w))


@pytest.mark.parametrize("N,K", synth.SWEEP_SHAPES)
def test_gemv_shape_sweep_exact(N, K):
    q, w, y = gemv_case(N, K, seed=0)
    assert np.array_equal(y, oracle.gemm_i32(q, w))


@pytest.mark.parametrize("N,K", synth.LARGE_SHAPES)
def test_gemv_large_exact(N, K):
    q, w, y = gemv_case(N, K, seed=0, gen=synth.sparse_ternary_normal_int8)
    assert np.array_equal(y, oracle.gemm_i32(q, w))


def test_empty_and_zero_k():
    q = torch.zeros((1, 0), dtype=torch.int8, device="cuda")
    packed = torch.zeros(16, dtype=torch.uint8, device="cuda")
    y = torch.full((1, 5), 7, dtype=torch.int32, device="cuda")
    bn.bitnet_w2a8_gemm(q, packed, 5, y=y)
    assert host(y).tolist() == [[0] * 5]
    y0 = torch.empty((0, 5), dtype=torch.int32, device="cuda")
    bn.bitnet_w2a8_gemm(torch.zeros((0, 4), dtype=torch.int8, device="cuda"), packed, 5, y=y0)


# ------------------------------------------------------------------ BitLinear

def bitlinear_case(M, N, K, seed, outliers=True):
    x, W = synth.bitlinear_inputs(M, N, K, seed=seed, outliers=outliers)
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    packed = pack_on_gpu(wt)
    gamma = dev(np.array([g], np.float32))
    y = bn.bitnet_bitlinear(bf16_tensor(x), packed, gamma, N)
    return x, wt, g, packed, y


@pytest.mark.parametrize("N,K", synth.BITLINEAR_DECODE_SHAPES + [(33, 100), (1, 4096)])
def test_bitlinear_decode(N, K):
    x, wt, g, packed, y = bitlinear_case(1, N, K, seed=0)
    y_ref, acc_ref, q_ref, s_ref = oracle.bitlinear(x, wt, g)
    check_bf16(y, y_ref)
    # the int32 stage on the GPU's own codes is exact
    q, s, _ = bn.bitnet_quant_act(bf16_tensor(x))
    assert np.array_equal(host(q), q_ref)
    acc = host(bn.bitnet_w2a8_gemm(q, packed, N))
    assert np.array_equal(acc, acc_ref)


def test_bitlinear_zero_token_and_weights():
    M, N, K = 3, 40, 300
    x, W = synth.bitlinear_inputs(M, N, K, seed=2)
    x[1] = 0
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    y = bn.bitnet_bitlinear(bf16_tensor(x), pack_on_gpu(wt), dev(np.array([g], np.float32)), N)
    check_bf16(y, oracle.bitlinear(x, wt, g)[0])
    assert not host(y.view(torch.int16))[1].any()


# ------------------------------------------------------------------ M > 1

@pytest.mark.parametrize("M,N,K", [(2, 3, 17), (3, 129, 1000), (5, 64, 2560), (17, 300, 129)])
def test_gemm_small_batch_exact(M, N, K):
    q, w, y = gemv_case(N, K, seed=M + N + K, M=M)
    assert np.array_equal(y, oracle.gemm_i32(q, w))


@pytest.mark.parametrize("M", synth.PREFILL_M)
@pytest.mark.parametrize("N,K", synth.PREFILL_SHAPES)
def test_prefill_int32_and_bf16(M, N, K):
    """Production-size prefill, every output element: int32 bit-exact against
    the oracle's full contraction, bf16 within the stated tolerance of its fp64
    rescale; outputs and workspaces sit between guard bands."""
    from guarded import Guarded, guarded_workspace
    x, W = synth.bitlinear_inputs(M, N, K, seed=0, outliers=False)
    g = oracle.absmean(W)
    wt = oracle.ternarize(W, g)
    packed = pack_on_gpu(wt)
    q, s, _ = bn.bitnet_quant_act(bf16_tensor(x))
    q_ref, s_ref, _ = oracle.quant_act(x)
    assert np.array_equal(host(q), q_ref)
    yg = Guarded(torch, (M, N), torch.int32, fill=-7)
    wsg = guarded_workspace(torch, bn, M, N, K)
    bn.bitnet_w2a8_gemm(q, packed, N, y=yg.t, ws=wsg.t)
    acc_ref = oracle.gemm_i32(q_ref, wt)
    assert np.array_equal(host(yg.t), acc_ref)
    yg.check("the int32 output")
    wsg.check("the workspace")
    bg = Guarded(torch, (M, N), torch.int16, fill=0x7F7F)
    wsb = guarded_workspace(torch, bn, M, N, K)
    bn.bitnet_bitlinear(bf16_tensor(x), packed, dev(np.array([g], np.float32)), N,
                        y=bg.t.view(torch.bfloat16), ws=wsb.t)
    check_bf16(bg.t.view(torch.bfloat16), oracle.rescale(acc_ref, g, s_ref))
    bg.check("the bf16 output")
    wsb.check("the BitLinear workspace")
