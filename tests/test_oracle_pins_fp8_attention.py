"""Pins of the oracle's FP8 attention ("Wan（通义万相）…" 5.3, "FlashAttention3
FP8": the Q/K inner product in INT8, O = P V in FP8, accumulation across key
blocks in FP32).

* the INT8 quantisers against torch's round-half-even, their bounds and ties,
  and the per-block quantiser as the per-row one over a flattened block;
* the per-channel e4m3 quantiser as the pinned per-row one of the transpose;
* the blockwise attention without the rounding of P against torch's
  scaled_dot_product_attention of the dequantised operands (any reference
  threshold, ragged key blocks), and exactly on operands the quantisers
  represent exactly;
* with P rounded to e4m3: within the rounding bound of e4m3 of the exact
  result, and really rounded.

Planted mistakes (monkeypatched on the CPU for one test): a K scale taken from
the wrong block, the running output not rescaled when the reference moves,
the values' scale left out.  The pins must fail on each.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as TF

from oracle import wan_oracle as O

RNG = np.random.default_rng(1234)


def sdpa(q, k, v):
    """torch's attention (float64) of one head: q [Nq, dh], k/v [Nk, dh]."""
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    return TF.scaled_dot_product_attention(t(q), t(k), t(v))[0, 0].numpy()


def dequantised(q, k, v, bk=128):
    q8, sq = O.quant_rows_int8(q)
    k8, sk = O.quant_blocks_int8(k, bk)
    v8, sv = O.quant_cols_e4m3(v)
    kb = np.repeat(np.asarray(sk, np.float64), bk)[:k.shape[0]]
    return q8 * np.asarray(sq, np.float64)[:, None], k8 * kb[:, None], v8 * np.asarray(sv, np.float64)[None, :]


def qkv(nq, nk, dh=128, scale=1.0, seed=0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((nq, dh)).astype(np.float32) * scale
    k = r.standard_normal((nk, dh)).astype(np.float32) * scale
    v = r.standard_normal((nk, dh)).astype(np.float32)
    # blocks of different size, so that each has its own scale
    k[:128] *= 0.5
    k[256:384] *= 1.7
    return q, k, v


# ---------------------------------------------------------------- quantisers
def test_int8_rows_match_torch_round_half_even():
    x = RNG.standard_normal((37, 128)).astype(np.float32) * RNG.uniform(0.01, 10, (37, 1)).astype(np.float32)
    codes, s = O.quant_rows_int8(x)
    xt = torch.from_numpy(x)
    st = (xt.abs().amax(dim=1) / 127.0).to(torch.float32)
    np.testing.assert_array_equal(s, st.numpy())
    want = torch.round(xt / st[:, None]).clamp(-127, 127)    # torch.round: ties to even
    np.testing.assert_array_equal(codes, want.double().numpy())


def test_int8_rows_bounds_ties_and_zero_rows():
    x = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5],
                  [0, 0, 0, 0, 0, 0, 0]], np.float32)
    codes, s = O.quant_rows_int8(x)
    np.testing.assert_array_equal(s, [1.0, 1.0])
    np.testing.assert_array_equal(codes[0], [127, 2, 4, -2, -0.0, 0, 2])   # halves to even
    np.testing.assert_array_equal(codes[1], 0)
    y = RNG.standard_normal((64, 96)).astype(np.float32) * 3
    c, sy = O.quant_rows_int8(y)
    assert np.abs(c).max() <= 127 and np.all(np.abs(c).max(axis=1) == 127)   # each row's amax -> +-127
    err = np.abs(y - c * sy[:, None].astype(np.float64))
    assert np.all(err <= sy[:, None] * (0.5 + 1e-5))                        # half a step (plus fp32 division)


def test_int8_blocks_are_rows_of_flattened_blocks():
    x = RNG.standard_normal((300, 64)).astype(np.float32)
    x[128:256] *= 4.0
    codes, s = O.quant_blocks_int8(x, 128)
    assert s.shape == (3,)
    for n, (a, b) in enumerate([(0, 128), (128, 256), (256, 300)]):   # ragged last block
        c1, s1 = O.quant_rows_int8(x[a:b].reshape(1, -1))
        assert s[n] == s1[0]
        np.testing.assert_array_equal(codes[a:b], c1.reshape(b - a, 64))


def test_e4m3_columns_are_rows_of_the_transpose():
    x = RNG.standard_normal((200, 48)).astype(np.float32) * RNG.uniform(0.1, 5, (1, 48)).astype(np.float32)
    codes, s = O.quant_cols_e4m3(x)
    ct, st = O.quant_rows_e4m3(x.T)
    np.testing.assert_array_equal(codes, ct.T)
    np.testing.assert_array_equal(s, st)
    assert np.all(np.abs(codes).max(axis=0) == 448.0)


# ---------------------------------------------------------------- the attention
@pytest.mark.parametrize("theta", [0.0, 8.0, 1e9])
@pytest.mark.parametrize("nk", [128, 300, 517])
def test_unrounded_p_is_sdpa_of_the_dequantised_operands(theta, nk):
    """Without the rounding of P the blockwise softmax (any reference
    threshold: 0 moves it at every growth, 1e9 only at the first block) is the
    exact attention of the dequantised q, k, v."""
    q, k, v = qkv(45, nk, scale=1.3, seed=nk)
    got = O.attention_fp8_head(q, k, v, theta=theta, quant_p=False)
    np.testing.assert_allclose(got, sdpa(*dequantised(q, k, v)), rtol=0, atol=1e-12)


def test_exactly_representable_operands():
    """Integer q with 127 in every row, K blocks with amax 127 and v on the e4m3
    grid with 448 in every column quantise to themselves (unit scales); the
    attention without P rounding is then torch's attention of the inputs."""
    r = np.random.default_rng(3)
    # small integers, with each row's 127 (q) or each block's 127 (k) in a column the other operand leaves zero
    q = r.integers(-2, 3, (20, 128)).astype(np.float32)
    q[:, 5], q[:, 6] = 127, 0
    k = r.integers(-2, 3, (256, 128)).astype(np.float32)
    k[:, 5] = 0
    k[0, 6] = k[128, 6] = 127
    v = O.e4m3(r.standard_normal((256, 128)) * 50).astype(np.float32)
    v[0] = 448.0
    for fn, arr in ((O.quant_rows_int8, q), (lambda a: O.quant_blocks_int8(a, 128), k), (O.quant_cols_e4m3, v)):
        c, s = fn(arr)
        np.testing.assert_array_equal(c, arr)
        np.testing.assert_array_equal(s, 1.0)
    got = O.attention_fp8_head(q, k, v, quant_p=False)
    np.testing.assert_allclose(got, sdpa(q, k, v), rtol=0, atol=1e-10 * np.abs(v).max())


@pytest.mark.parametrize("theta", [0.0, 8.0])
def test_rounded_p_within_the_e4m3_bound(theta):
    """P rounded to e4m3 changes each probability by at most half an e4m3 step
    (2^-4 relative, or 2^-10 absolute below 2^-6).  Against the row's own
    maximum (p_j <= 1, l = sum_j p_j) every output element then lies within
    sum_j max(2^-4 p_j, 2^-10) |v_j| / l of the exact one: the reference sits
    s = 2^(row max - m) >= 1 below, which scales p, its relative error bound and
    l by s alike and leaves the absolute term 2^-10 / s <= 2^-10.  The
    rounding is really applied."""
    q, k, v = qkv(30, 300, scale=1.3, seed=7)
    exact = O.attention_fp8_head(q, k, v, theta=theta, quant_p=False)
    got = O.attention_fp8_head(q, k, v, theta=theta, quant_p=True)
    qd, kd, vd = dequantised(q, k, v)
    t = qd @ kd.T / math.sqrt(128)
    p = np.exp(t - t.max(axis=1, keepdims=True))          # relative to the row max: <= 1
    l = p.sum(axis=1, keepdims=True)
    bound = np.maximum(p * 2.0 ** -4, 2.0 ** -10) @ np.abs(vd) / l
    err = np.abs(got - exact)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-12)
    assert err.max() > 1e-6 * np.abs(exact).max()


# ---------------------------------------------------------------- planted mistakes
def _wrong_block_scale(monkeypatch):
    real = O.quant_blocks_int8

    def shifted(x, bk=128):
        c, s = real(x, bk)
        return c, np.roll(s, 1)
    monkeypatch.setattr(O, "quant_blocks_int8", shifted)


def _no_rescale(monkeypatch):
    # the per-row factor 2^(m_old - m_new) (the only one-dimensional exp2) becomes 1
    monkeypatch.setattr(O.np, "exp2", lambda a, _e=np.exp2: np.ones_like(a) if np.ndim(a) == 1 else _e(a))


def _no_value_scale(monkeypatch):
    real = O.quant_cols_e4m3
    monkeypatch.setattr(O, "quant_cols_e4m3", lambda x: (real(x)[0], np.ones_like(real(x)[1])))


@pytest.mark.parametrize("plant", [_wrong_block_scale, _no_rescale, _no_value_scale])
def test_planted_mistakes_fail_the_sdpa_pin(monkeypatch, plant):
    q, k, v = qkv(45, 517, scale=1.3, seed=11)
    want = sdpa(*dequantised(q, k, v))
    with monkeypatch.context() as m:
        plant(m)
        got = O.attention_fp8_head(q, k, v, theta=0.0, quant_p=False)
    assert np.abs(got - want).max() > 1e-6
