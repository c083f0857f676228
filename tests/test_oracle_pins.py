"""Pins for the CPU oracle: each test checks it against something other than
itself -- hand-worked values from the pages' definitions (tests/golden/),
brute force on tiny inputs, closed forms, invariants and error bounds.

None of these tests needs a GPU.
"""
import itertools

import numpy as np
import pytest

from conftest import read_golden
from ternary_weight_bit_w2a8_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _py_matmul(q, w):
    """Brute-force triple loop in Python integers."""
    M, K = q.shape
    N = w.shape[0]
    out = [[0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = 0
            for k in range(K):
                acc += int(q[m, k]) * int(w[n, k])
            out[m][n] = acc
    return np.array(out, dtype=np.int64)


# ----------------------------------------------------------------- codes / packing

def test_code_mapping_golden(oracle_mod):
    rows = [r[0].split() for r in read_golden("code_mapping.txt")]
    for value, code in rows:
        w = np.array([[int(value)]], dtype=np.int8)
        canon = oracle_mod.pack_canonical(w)
        assert canon[0, 0] & 3 == int(code, 2)
        dev, bad = oracle_mod.pack_device(w)
        assert bad == 0
        assert dev[0, 0] & 3 == int(code, 2)
    # 11 is never produced: every field of a packed random matrix is < 3
    _, w = synth.uniform_int8_ternary(7, 300, seed=3)
    dev, _ = oracle_mod.pack_device(w)
    for shift in (0, 2, 4, 6):
        assert ((dev >> shift) & 3).max() <= 2


def test_canonical_pack_golden(oracle_mod):
    for K, vals, hexbytes in read_golden("canonical_pack.txt"):
        K = int(K)
        w = np.array([[int(v) for v in vals.split()]], dtype=np.int8)
        assert w.shape[1] == K
        got = oracle_mod.pack_canonical(w)[0]
        assert [int(h, 16) for h in hexbytes.split()] == list(got)


def test_device_pack_golden(oracle_mod):
    for K, vals, hexbytes in read_golden("device_pack_v1.txt"):
        K = int(K)
        w = np.array([[int(v) for v in vals.split()]], dtype=np.int8)
        assert w.shape[1] == K
        packed, bad = oracle_mod.pack_device(w)
        assert bad == 0
        row = list(packed[0])
        assert len(row) == 32  # K_pad = 128 -> 32 bytes
        lead = [int(h, 16) for h in hexbytes.split()]
        assert row[:len(lead)] == lead
        assert all(b == 0x55 for b in row[len(lead):])


@pytest.mark.parametrize("N,K", [(1, 1), (1, 3), (3, 17), (5, 64), (2, 127), (4, 128),
                                 (3, 129), (7, 300), (17, 1000)])
def test_pack_roundtrip(oracle_mod, N, K):
    _, w = synth.uniform_int8_ternary(N, K, seed=N * 1000 + K)
    c = oracle_mod.pack_canonical(w)
    assert c.shape == (N, (K + 3) // 4)
    assert np.array_equal(oracle_mod.unpack_canonical(c, N, K), w)
    d, bad = oracle_mod.pack_device(w)
    assert bad == 0
    assert d.size == oracle_mod.device_packed_bytes(N, K) == N * ((K + 127) // 128) * 32
    u, bad2 = oracle_mod.unpack_device(d, N, K)
    assert bad2 == 0
    assert np.array_equal(u, w)


def test_device_layout_word_property(oracle_mod):
    """Each little-endian 32-bit word covers 16 consecutive k; shifting it right
    by 2j and masking 0x03030303 leaves, in byte b, the code of k = 16i + 4j + b."""
    _, w = synth.uniform_int8_ternary(3, 256, seed=11)
    d, _ = oracle_mod.pack_device(w)
    words = d.view("<u4")
    for n in range(3):
        for i in range(256 // 16):
            for j in range(4):
                v = (int(words[n, i]) >> (2 * j)) & 0x03030303
                for b in range(4):
                    assert (v >> (8 * b)) & 0xFF == int(w[n, 16 * i + 4 * j + b]) + 1


def test_pack_invalid_values(oracle_mod):
    w = np.array([[1, 2, -1, -5, 0, 127]], dtype=np.int8)
    d, bad = oracle_mod.pack_device(w)
    assert bad == 3
    u, _ = oracle_mod.unpack_device(d, 1, 6)
    assert list(u[0]) == [1, 0, -1, 0, 0, 0]
    # unused code 11 decodes to zero and is counted; byte 0 holds k = 0, 4,
    # 8, 12, of which k = 0 and k = 4 lie inside K = 6
    d[0, 0] = 0xFF
    u, bad = oracle_mod.unpack_device(d, 1, 6)
    assert bad == 2 and u[0, 0] == 0 and u[0, 4] == 0


# ----------------------------------------------------------------- ternarisation

def test_ternarize_golden(oracle_mod):
    for hexw, gamma, vals in read_golden("ternarize_cases.txt"):
        W = np.array([[int(h, 16) for h in hexw.split()]], dtype=np.uint16)
        g = oracle_mod.absmean(W)
        assert g == np.float32(float(gamma))
        wt = oracle_mod.ternarize(W, g)
        assert [int(v) for v in vals.split()] == list(wt[0])


def test_absmean_matches_library_mean(oracle_mod):
    W = synth.bf16_weights(37, 411, seed=5)
    f = synth.bf16_bits_to_f32(W).astype(np.float64)
    ref = np.float32(np.mean(np.abs(f)))
    g = oracle_mod.absmean(W)
    assert abs(float(g) - float(ref)) <= float(np.spacing(ref))


def test_absmean_whole_matrix_not_per_row(oracle_mod):
    # two rows with different magnitudes: a per-row scale would ternarise both
    # rows to all +1; the whole-matrix scale (mean 0.5625) zeroes row 0.
    W = synth.f32_to_bf16_bits(np.array([[0.125, 0.125], [1.0, 1.0]], np.float32))
    g = oracle_mod.absmean(W)
    assert g == np.float32(0.5625)
    assert oracle_mod.ternarize(W, g).tolist() == [[0, 0], [1, 1]]


def test_ternarize_invariants(oracle_mod):
    W = synth.bf16_weights(64, 257, seed=9)
    g = oracle_mod.absmean(W)
    wt = oracle_mod.ternarize(W, g)
    r = synth.bf16_bits_to_f32(W) / g  # fp32 division, as the definition
    assert set(np.unique(wt)) <= {-1, 0, 1}
    assert np.all(wt[np.abs(r) < 0.5] == 0)
    big = np.abs(r) > 0.5
    assert np.array_equal(wt[big], np.sign(r[big]).astype(np.int8))
    # Gaussian weights: |w| > mean|w|/2 happens with probability ~0.69
    frac_nonzero = np.count_nonzero(wt) / wt.size
    assert 0.6 < frac_nonzero < 0.78


# ----------------------------------------------------------------- activation quant

def test_quant_golden(oracle_mod):
    for xs, s, qs, rowsum in read_golden("quant_cases.txt"):
        x = synth.f32_to_bf16_bits(np.array([float(v) for v in xs.split()], np.float32))
        assert np.array_equal(synth.bf16_bits_to_f32(x), np.array([float(v) for v in xs.split()], np.float32))
        q, sc, rs = oracle_mod.quant_act(x.reshape(1, -1))
        assert [int(v) for v in qs.split()] == list(q[0])
        assert rs[0] == int(rowsum)
        if s != "-":
            assert sc[0] == np.float32(float(s))


def test_quant_invariants(oracle_mod):
    x = synth.bf16_activations(9, 1000, seed=4)
    q, s, rs = oracle_mod.quant_act(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    amax = np.abs(xf).max(axis=1)
    assert np.all(np.abs(q.astype(np.int64)).max(axis=1) == 127)
    np.testing.assert_allclose(s, 127.0 / amax, rtol=2e-7)
    # rounding error of each code is at most half a step (+ fp32 slack)
    err = np.abs(xf * s[:, None].astype(np.float64) - q)
    assert err.max() <= 0.5 + 1e-4
    assert np.array_equal(rs, q.astype(np.int64).sum(axis=1))


# ----------------------------------------------------------------- contraction

@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (1, 5, 7), (2, 3, 67), (3, 17, 13), (3, 4, 64)])
def test_gemm_bruteforce(oracle_mod, M, N, K):
    q, w = synth.uniform_int8_ternary(N, K, seed=M * 100 + N * 10 + K, M=M)
    y = oracle_mod.gemm_i32(q, w)
    assert np.array_equal(y, _py_matmul(q, w))
    # the int8 extreme -128 as well
    q2 = np.full((M, K), -128, dtype=np.int8)
    assert np.array_equal(oracle_mod.gemm_i32(q2, w), _py_matmul(q2, w))


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_gemm_exhaustive_rows(oracle_mod, K):
    rows = np.array(list(itertools.product([-1, 0, 1], repeat=K)), dtype=np.int8)
    rng = np.random.default_rng(K)
    q = rng.integers(-128, 128, size=(3, K), dtype=np.int8)
    y = oracle_mod.gemm_i32(q, rows)
    assert np.array_equal(y, _py_matmul(q, rows))
    # the set of all ternary rows is symmetric under negation: outputs sum to 0
    assert np.all(y.astype(np.int64).sum(axis=1) == 0)


def test_gemm_special_weights(oracle_mod):
    rng = np.random.default_rng(1)
    M, K = 4, 333
    q = rng.integers(-128, 128, size=(M, K), dtype=np.int8)
    rs = q.astype(np.int64).sum(axis=1)
    zero = np.zeros((6, K), np.int8)
    assert np.all(oracle_mod.gemm_i32(q, zero) == 0)
    ones = np.ones((6, K), np.int8)
    assert np.array_equal(oracle_mod.gemm_i32(q, ones), np.repeat(rs[:, None], 6, axis=1))
    assert np.array_equal(oracle_mod.gemm_i32(q, -ones), -np.repeat(rs[:, None], 6, axis=1))
    eye = np.eye(K, dtype=np.int8)
    assert np.array_equal(oracle_mod.gemm_i32(q, eye), q.astype(np.int32))
    assert np.array_equal(oracle_mod.gemm_i32(q, -eye), -q.astype(np.int32))
    # rectangular, asymmetric weights: output n uses row n of W (not column n)
    w = np.zeros((2, K), np.int8)
    w[0, 0] = 1
    w[1, K - 1] = -1
    y = oracle_mod.gemm_i32(q, w)
    assert np.array_equal(y[:, 0], q[:, 0]) and np.array_equal(y[:, 1], -q[:, K - 1])


def test_gemm_linearity(oracle_mod):
    rng = np.random.default_rng(2)
    K = 500
    q1 = rng.integers(-60, 61, size=(2, K), dtype=np.int8)
    q2 = rng.integers(-60, 61, size=(2, K), dtype=np.int8)
    _, w = synth.uniform_int8_ternary(31, K, seed=2)
    y1 = oracle_mod.gemm_i32(q1, w).astype(np.int64)
    y2 = oracle_mod.gemm_i32(q2, w).astype(np.int64)
    y12 = oracle_mod.gemm_i32((q1 + q2).astype(np.int8), w).astype(np.int64)
    assert np.array_equal(y1 + y2, y12)
    yneg = oracle_mod.gemm_i32((-q1).astype(np.int8), w).astype(np.int64)
    assert np.array_equal(yneg, -y1)


def test_gemm_sampled_matches_full(oracle_mod):
    q, w = synth.uniform_int8_ternary(40, 300, seed=8, M=3)
    y = oracle_mod.gemm_i32(q, w)
    ms = np.array([0, 2, 1, 2], np.int64)
    ns = np.array([39, 0, 17, 5], np.int64)
    assert np.array_equal(oracle_mod.gemm_i32_sampled(q, w, ms, ns), y[ms, ns])


# ----------------------------------------------------------------- rescale / bitlinear

def test_rescale_closed_form(oracle_mod):
    acc = np.array([[3, -8], [0, 1000]], np.int32)
    s = np.array([2.0, 0.5], np.float32)
    y = oracle_mod.rescale(acc, np.float32(0.5), s)
    assert y.tolist() == [[0.75, -2.0], [0.0, 1000.0]]


def test_bitlinear_within_quantisation_error(oracle_mod):
    """The BitLinear output approximates x @ (gamma * W_t)^T; the only error is
    the activation rounding, at most half a step (1/(2 s_m)) per element:
    |y - x (gamma W_t)^T| <= gamma * sum_k |W_t[n,k]| / (2 s_m).  A scale
    applied the wrong way round, or a dropped scale, breaks this bound."""
    M, N, K = 3, 29, 257
    x, W = synth.bitlinear_inputs(M, N, K, seed=3)
    g = oracle_mod.absmean(W)
    wt = oracle_mod.ternarize(W, g)
    y, acc, q, s = oracle_mod.bitlinear(x, wt, g)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    exact = xf @ (float(g) * wt.astype(np.float64)).T
    bound = float(g) * np.abs(wt).sum(axis=1)[None, :] / (2.0 * s[:, None].astype(np.float64))
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-6) + 1e-12)
    # and the quantisation is not trivially loose: the error is well inside
    assert np.abs(y - exact).max() < 0.2 * bound.max()
    # all-zero weights give 0; a zero token gives 0
    z = oracle_mod.bitlinear(x, np.zeros_like(wt), g)[0]
    assert np.all(z == 0)
    x0 = x.copy()
    x0[1] = 0
    assert np.all(oracle_mod.bitlinear(x0, wt, g)[0][1] == 0)
