"""Pins of the oracle's online-softmax attention with PNQ: the textbook case
with quantization off, Proposition 1 (induced weights sum to one), the output
rebuilt from those weights, a hand-computed PNQ example and closed-form
special cases."""
import math

import numpy as np
import pytest

import oracle
from conftest import golden
from mxfp4_bit_attention_b200 import inputs


def _softmax_attention(q, k, v, s):
    S = (q @ k.T) * s
    P = np.exp(S - S.max(axis=1, keepdims=True))
    return (P / P.sum(axis=1, keepdims=True)) @ v


@pytest.fixture(scope="module")
def tiny():
    g = inputs.generate("tiny")
    return [inputs.as_fp32(g[n], "fp32")[0] for n in "qkv"]


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_quant_off_equals_softmax_attention(tiny, rotate, tau):
    q, k, v = tiny
    s = 1 / math.sqrt(q.shape[1])
    res = oracle.forward_rows(q[None], k[None], v[None], np.arange(q.shape[0]), s, rotate=rotate,
                              quant=False, key_tile=64, tau=tau)
    ref = _softmax_attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), s)
    assert np.max(np.abs(res["out"][0] - ref)) <= 1e-5


@pytest.mark.parametrize("rule", [oracle.RULE_UOS, oracle.RULE_QMAX6, oracle.RULE_OCP])
@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_pnq_weights_sum_to_one(tiny, rule, tau):
    q, k, v = tiny
    qd, kd, vd = oracle.prepare_head(q, k, v, True, rule)
    r = oracle.attention_rows(qd, kd, vd, 0.125, 64, pnq=True, rule=rule, tau=tau, weights=True)
    assert np.max(np.abs(r["wsum"] - 1.0)) <= 1e-12
    assert np.max(np.abs(r["ocheck"] - r["out"])) <= 1e-12


def test_direct_placement_breaks_normalization(tiny):
    q, k, v = tiny
    qd, kd, vd = oracle.prepare_head(q, k, v, True, oracle.RULE_OCP)
    r = oracle.attention_rows(qd, kd, vd, 0.125, 64, pnq=False, rule=oracle.RULE_OCP, weights=True)
    dev = r["wsum"] - 1.0
    assert np.mean(np.abs(dev) > 1e-6) > 0.9
    assert np.max(np.abs(r["ocheck"] - r["out"])) <= 1e-12


def test_hand_computed_pnq_example():
    ex = golden("pnq_example.json")
    p = np.array(ex["p"])
    n = len(p)
    d = 8
    q = np.zeros((1, d)); q[0, 0] = 1.0
    k = np.zeros((n, d)); k[:, 0] = np.log(p).astype(np.float32)
    v = np.eye(n, d)
    for rule in (oracle.RULE_UOS, oracle.RULE_QMAX6, oracle.RULE_OCP):
        r = oracle.attention_rows(q, k, v, 1.0, 32, pnq=True, rule=rule, weights=True)
        assert np.allclose(r["out"][0], ex["out_pnq"], rtol=0, atol=1e-15)
        assert r["l"][0] == pytest.approx(ex["l_pnq"], abs=1e-15)
        assert r["wsum"][0] == pytest.approx(ex["wsum_pnq"], abs=1e-15)
        rd = oracle.attention_rows(q, k, v, 1.0, 32, pnq=False, rule=rule, weights=True)
        assert rd["l"][0] == pytest.approx(ex["l_direct"], rel=1e-6)
        assert np.allclose(rd["out"][0], np.array(ex["p_hat"]) / ex["l_direct"], rtol=1e-6)
        assert rd["wsum"][0] == pytest.approx(ex["wsum_direct"], rel=1e-6)


def test_equal_scores_give_mean_of_values():
    """All keys equal: every P~ is exp(0) = 1, which MXFP4 represents exactly,
    so l = N and O is the plain mean of V over N keys (ragged last tile)."""
    rng = np.random.default_rng(3)
    N, d = 150, 64
    q = rng.standard_normal((4, d))
    k = np.tile(rng.standard_normal((1, d)), (N, 1))
    v = rng.standard_normal((N, d))
    r = oracle.attention_rows(q, k, v, 0.125, 64, pnq=True)
    assert np.allclose(r["l"], N, rtol=0, atol=1e-12)
    assert np.allclose(r["out"], v.mean(axis=0)[None], rtol=0, atol=1e-12)


def test_single_dominant_key():
    """One key far above the rest: P~ underflows to zero elsewhere, O = v of that key."""
    N, d = 100, 32
    q = np.zeros((1, d)); q[0, 0] = 1
    k = np.zeros((N, d)); k[:, 0] = -200.0; k[37, 0] = 0.0
    v = np.arange(N * d, dtype=np.float64).reshape(N, d)
    r = oracle.attention_rows(q, k, v, 1.0, 64, pnq=True)
    assert np.array_equal(r["out"][0], v[37])


def test_rows_are_independent(tiny):
    q, k, v = tiny
    rows = np.array([0, 5, 200, 255])
    full = oracle.forward_rows(q[None], k[None], v[None], np.arange(256), 0.125)
    part = oracle.forward_rows(q[None], k[None], v[None], rows, 0.125)
    assert np.array_equal(full["out"][0][rows], part["out"][0])


@pytest.mark.parametrize("N", [64, 45])
def test_recorded_p_codes_rebuild_the_pnq_row_sum(tiny, N):
    """With one key tile there is no rescaling, so under PNQ the row sum l is exactly the sum of
    the quantized tile: the recorded codes and scale bytes, dequantized, must rebuild it; keys
    past N (ragged tile) must record code 0, and each group's largest value must sit on the
    E2M1 grid scaled by its recorded power of two."""
    q, k, v = (x.astype(np.float64) for x in tiny)
    r = oracle.attention_rows(q[:16], k[:N], v[:N], 0.125, tau=0.0, codes=True)
    pc, ps = r["p_codes"], r["p_scales"]
    assert pc.shape == (16, 64) and ps.shape == (16, 2)
    assert not pc[:, N:].any()
    vals = oracle.dequantize(pc, ps)
    np.testing.assert_allclose(vals.sum(axis=1), r["l"], rtol=1e-15, atol=0)
    # the group holding the row max (P~ = exp(0) = 1) is never all zero
    assert (vals.max(axis=1) > 0).all()


@pytest.mark.parametrize("tau", [0.0, 8.0])
def test_causal_quant_off_equals_masked_softmax_attention(tiny, tau):
    """Causal masking (row i sees keys 0..i) with quantization off is the textbook masked softmax."""
    q, k, v = tiny
    N, d = k.shape
    rows = np.array([0, 1, 2, 63, 64, 65, 127, 128, 200, N - 1])
    s = 0.125
    res = oracle.forward_rows(q[None], k[None], v[None], rows, s, quant=False, tau=tau, causal=True)["out"][0]
    qr = oracle.rotate_rows(q[rows]).astype(np.float64)
    kr = oracle.rotate_rows(k).astype(np.float64)
    S = (qr @ kr.T) * s
    S[np.arange(N)[None, :] > rows[:, None]] = -np.inf
    P = np.exp(S - S.max(axis=1, keepdims=True))
    ref = (P / P.sum(axis=1, keepdims=True)) @ v.astype(np.float64)
    np.testing.assert_allclose(res, ref, rtol=0, atol=1e-5)


def test_causal_first_row_sees_only_the_first_key(tiny):
    """Row 0 under causal masking: one key, P~ = exp(0) = 1 is exact in E2M1, l = 1, so the output
    is the (quantized) first value row exactly."""
    q, k, v = tiny
    res = oracle.forward_rows(q[None], k[None], v[None], np.array([0]), 0.125, causal=True)["out"][0, 0]
    vq = oracle.prepare_head(q[:1], k, v)[2]
    np.testing.assert_array_equal(res, vq[0])


def _packed(lengths, H, d, seed):
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    q, k, v = (rng.standard_normal((T, H, d)).astype(np.float32) for _ in range(3))
    return q, k, v, np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_quant_off_equals_block_diagonal_softmax(causal):
    """A packed batch with quantization off is softmax attention over the whole packed token axis
    with a block-diagonal mask (and the causal mask inside each block): built here densely."""
    lengths = [5, 0, 70, 1, 130]
    q, k, v, cu = _packed(lengths, 2, 64, seed=11)
    T = len(q)
    rows = np.arange(T)
    s = 0.125
    res = oracle.forward_varlen(q, k, v, cu, rows, s, quant=False, causal=causal)
    seq = np.repeat(np.arange(len(lengths)), lengths)
    for h in range(2):
        qr = oracle.rotate_rows(q[:, h]).astype(np.float64)
        kr = oracle.rotate_rows(k[:, h]).astype(np.float64)
        S = (qr @ kr.T) * s
        mask = seq[:, None] != seq[None, :]
        if causal:
            mask |= np.arange(T)[None, :] > np.arange(T)[:, None]
        S[mask] = -np.inf
        P = np.exp(S - S.max(axis=1, keepdims=True))
        ref = (P / P.sum(axis=1, keepdims=True)) @ v[:, h].astype(np.float64)
        np.testing.assert_allclose(res[:, h], ref, rtol=0, atol=1e-5)


def test_varlen_sequences_are_independent():
    """A sequence's output depends on its own tokens only: replacing every other sequence's Q, K and
    V (whose V groups would share 32-key blocks with it if the groups ran across the packing) leaves
    it unchanged bit for bit; packing the same tokens as one sequence does change it."""
    lengths = [40, 100, 29]
    q, k, v, cu = _packed(lengths, 1, 128, seed=12)
    rows = np.arange(cu[1], cu[2])
    a = oracle.forward_varlen(q, k, v, cu, rows, 0.09, tau=8.0)
    rng = np.random.default_rng(99)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for x in (q2, k2, v2):
        x[:cu[1]] = rng.standard_normal(x[:cu[1]].shape) * 7
        x[cu[2]:] = rng.standard_normal(x[cu[2]:].shape) * 7
    b = oracle.forward_varlen(q2, k2, v2, cu, rows, 0.09, tau=8.0)
    np.testing.assert_array_equal(a, b)
    whole = oracle.forward_varlen(q, k, v, np.array([0, len(q)]), rows, 0.09, tau=8.0)
    assert np.abs(whole - a).max() > 1e-3
    # one sequence of the whole batch is forward_rows on [H, T, d]
    one = oracle.forward_rows(q.transpose(1, 0, 2).copy(), k.transpose(1, 0, 2).copy(),
                              v.transpose(1, 0, 2).copy(), rows, 0.09, tau=8.0)["out"].transpose(1, 0, 2)
    np.testing.assert_array_equal(whole, one)


@pytest.mark.parametrize("key_tile", [64, 128])
@pytest.mark.parametrize("tau", [8.0, 3.0])
def test_lazy_max_moves_only_past_tau_log2_units(key_tile, tau):
    """The lazy running max (Pith review page, axioms ledger: the FlashAttention-2 running max;
    Fig. 4B) moves only when a tile's max exceeds it by more than tau in log2 units.  Two tiles:
    tile 0 has scores 0, tile 1 one key whose score sits eps below or above tau * ln 2 (natural
    units).  With eps far below the distance between the log2 and natural readings of tau (a
    factor ln 2), a units mistake moves the max in both cases or in neither."""
    d, T = 64, key_tile
    q = np.zeros((1, d))
    q[0, 0] = 1.0
    k = np.zeros((2 * T, d))
    v = np.random.default_rng(0).standard_normal((2 * T, d))
    eps = 1e-4
    for sign, moves in ((-1, False), (+1, True)):
        b = float(np.float32(tau * math.log(2) * (1 + sign * eps)))
        k[T, 0] = b
        r = oracle.attention_rows(q, k, v, 1.0, key_tile, tau=tau, codes=True)
        assert r["m"][0] == (b if moves else 0.0)
        # the group holding the big key: P~ = e^b (about 2^tau) against the old max, or 1 against
        # the new one; its UOS scale byte is 127 + ceil(log2(P~max / 7.25)) either way
        pmax = math.exp(b) if not moves else 1.0
        assert r["p_scales"][0, T // 32] == 127 + math.ceil(math.log2(pmax / 7.25))
        # tile 0 was quantized before any move: 64 ones, scale 2^-2 (code 6 = 4.0)
        assert r["p_scales"][0, 0] == 125 and np.all(r["p_codes"][0, :T] == 6)
