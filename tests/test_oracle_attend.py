"""Pins of the oracle's attention over a compressed cache (reading R18) and
of its unrounded decode: the decode against the (separately pinned) bf16
decode; attention against closed forms (one token, a zero query, a very
sharp softmax), against an independent numpy statement of grouped-query
attention on the decoded vectors, and the transformed-domain identity that
lets a fused kernel score tokens without inverting the transform."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_compression_04_b200 import synth


def sylvester(d):
    h = np.array([[1.0]])
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def _cache(L=2, H=2, d=128, bits=4, g=64, lens=(300,), seed=3):
    w = synth.Workload("a", L, H, d, bits, g, seed=seed, kind="lognormal", scale_sigma=1.5,
                       tokens=sum(lens))
    kv = synth.dense_kv(w)
    # the dense order [layer][kv][head][token] is the stream order of requests
    # of these lengths concatenated along tokens
    x = synth.bf16_bits(kv).reshape(-1, d)
    desc = oracle.StreamDesc(bits, g, d, L, H, list(lens), 0)
    st, s = oracle.compress(desc, x)
    assert st == oracle.OK
    return desc, s, x


def _q(L, n_req, Hq, d, seed=1, scale=1.0):
    q = torch.randn(L, n_req, Hq, d, generator=torch.Generator().manual_seed(seed)) * scale
    return synth.bf16_bits(q.to(torch.bfloat16)).reshape(L, n_req, Hq, d)


def bf16_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_unrounded_decode_rounds_to_the_bf16_decode():
    desc, s, _ = _cache()
    st, vals = oracle.decode_values(s, desc)
    dst, xb = oracle.decompress(s, desc)
    assert st == dst == oracle.OK
    ref = bf16_to_f64(xb)
    # the bf16 decode rounds an fp32 evaluation of the same values: within a
    # bf16 ulp, and almost always the same rounding
    rel = np.abs(ref - vals) / np.maximum(np.abs(vals), 1e-30)
    assert np.all((rel <= 2.0 ** -8) | (np.abs(ref - vals) < 1e-35))
    back = synth.bf16_bits(torch.from_numpy(vals).to(torch.bfloat16))
    assert (back == xb).mean() > 0.999


def test_attend_single_token_returns_its_value():
    desc, s, _ = _cache(lens=(1,))
    _, vals = oracle.decode_values(s, desc)
    q = _q(2, 1, 4, 128)
    st, out = oracle.attend(s, desc, q, 2, 0.1)
    assert st == oracle.OK
    V = vals.reshape(2, 2, 2, 1, 128)[:, 1]          # [layer][head][token][d]
    for l in range(2):
        for j in range(4):
            assert np.array_equal(out[l, 0, j], V[l, j // 2, 0])


def test_attend_zero_query_is_the_mean_value():
    desc, s, _ = _cache(lens=(257,))
    _, vals = oracle.decode_values(s, desc)
    q = np.zeros((2, 1, 2, 128), np.uint16)
    st, out = oracle.attend(s, desc, q, 1, 1.0)
    assert st == oracle.OK
    V = vals.reshape(2, 2, 2, 257, 128)[:, 1]
    assert np.allclose(out[:, 0], V.mean(axis=2), rtol=1e-12, atol=1e-15)


def test_attend_sharp_softmax_picks_the_argmax_key():
    desc, s, _ = _cache(lens=(200,))
    _, vals = oracle.decode_values(s, desc)
    q = _q(2, 1, 2, 128, seed=5)
    scale = 50.0
    st, out = oracle.attend(s, desc, q, 1, scale)
    assert st == oracle.OK
    K = vals.reshape(2, 2, 2, 200, 128)[:, 0]
    V = vals.reshape(2, 2, 2, 200, 128)[:, 1]
    for l in range(2):
        for j in range(2):
            sc = scale * K[l, j] @ bf16_to_f64(q[l, 0, j])
            order = np.argsort(sc)
            gap = sc[order[-1]] - sc[order[-2]]
            if gap < 40:
                continue
            # every other weight is below exp(-gap)
            bound = 200 * np.exp(-gap) * 2 * np.abs(V[l, j]).max()
            assert np.abs(out[l, 0, j] - V[l, j, order[-1]]).max() <= bound


@pytest.mark.parametrize("lens,q_per_kv", [((300,), 4), ((37, 0, 140), 2)])
def test_attend_matches_numpy_gqa(lens, q_per_kv):
    """Independent statement: scores by einsum, softmax by numpy, on the
    decoded vectors read in [layer][kv][head][request][token] order."""
    L, H, d = 2, 2, 128
    T = sum(lens)
    desc, s, _ = _cache(L=L, H=H, lens=lens)
    _, vals = oracle.decode_values(s, desc)
    n_req = len(lens)
    q = _q(L, n_req, H * q_per_kv, d, seed=7)
    scale = 1.0 / np.sqrt(d)
    st, out = oracle.attend(s, desc, q, q_per_kv, scale)
    assert st == oracle.OK
    X = vals.reshape(L, 2, H, T, d)
    cum = np.concatenate([[0], np.cumsum(lens)])
    qf = bf16_to_f64(q)
    for r in range(n_req):
        for l in range(L):
            for j in range(H * q_per_kv):
                h = j // q_per_kv
                K = X[l, 0, h, cum[r]:cum[r + 1]]
                V = X[l, 1, h, cum[r]:cum[r + 1]]
                if K.shape[0] == 0:
                    assert not out[l, r, j].any()
                    continue
                sc = scale * np.einsum("td,d->t", K, qf[l, r, j])
                p = np.exp(sc - sc.max())
                want = (p[:, None] * V).sum(0) / p.sum()
                assert np.allclose(out[l, r, j], want, rtol=1e-10, atol=1e-13)


def test_transformed_domain_identity():
    """x^ = D H y^ / d with H symmetric and H H = d I, so y^ = H D x^ and
    q . x^ = (H D q) . y^ / d, and sum_t p_t x^_t = D H (sum_t p_t y^_t) / d:
    a fused attention kernel scores and accumulates in the transformed
    domain and inverts the transform once."""
    desc, s, _ = _cache(lens=(64,))
    _, vals = oracle.decode_values(s, desc)
    d = 128
    Hm = sylvester(d)
    sign = np.array([-1.0 if (int(oracle.sign_words(0, d)[c // 64]) >> (c % 64)) & 1 else 1.0
                     for c in range(d)])
    X = vals[:64]
    Y = (Hm @ (sign[:, None] * X.T)).T                # y^ recovered from x^
    assert np.allclose((sign[None, :] * (Hm @ Y.T).T) / d, X, rtol=0, atol=1e-12)
    rng = np.random.default_rng(0)
    qv = rng.standard_normal(d)
    qt = Hm @ (sign * qv)
    assert np.allclose(X @ qv, Y @ qt / d, rtol=1e-12, atol=1e-12)
    p = rng.random(64)
    assert np.allclose(p @ X, sign * (Hm @ (p @ Y)) / d, rtol=1e-12, atol=1e-12)
