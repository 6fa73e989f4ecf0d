"""Pins of the float64 oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: a library
routine (scipy's Hadamard matrix, scipy's Beta law and quadrature, numpy's
float16 rounding, torch's bf16/E4M3 conversions, numpy sorting), a closed
form, a textbook table, the pages' printed numbers, or brute force.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.special
import scipy.stats
import torch

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# random streams
# --------------------------------------------------------------------------
def test_splitmix64_published_first_output():
    # SplitMix64 seeded with 0: first output is 0xE220A8397B1DCDAF (the
    # generator's reference implementation, Steele/Lea/Flood 2014).
    assert O.draw(0, 0, 0) == 0xE220A8397B1DCDAF


def test_signs_and_gaussian_statistics():
    P = O.make_params(128, 2, seed=123)
    assert set(np.unique(P.signs)) <= {-1, 1}
    big = O.make_params(1024, 2, seed=7)
    s = big.S.astype(np.float64).ravel()
    # bf16-exact entries
    assert np.all(torch.tensor(s, dtype=torch.float32).to(torch.bfloat16).float().numpy() == s)
    # iid N(0,1): moments and a Kolmogorov-Smirnov test against scipy's normal law
    assert abs(s.mean()) < 5 / math.sqrt(s.size)
    assert abs(s.var() - 1.0) < 5 * math.sqrt(2.0 / s.size) + 2e-5
    ks = scipy.stats.kstest(s[:200000], "norm")
    assert ks.pvalue > 1e-4
    sg = np.concatenate([O.make_params(1024, 2, seed=k, with_S=False).signs for k in range(8)])
    assert abs(sg.mean()) < 5 / math.sqrt(sg.size)


# --------------------------------------------------------------------------
# rounding to the storage formats
# --------------------------------------------------------------------------
def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-8, 5, 2000),
                           [0.0, 65504.0, 6.1e-5, 5.96e-8, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11]])
    for v in vals:
        assert O.round_fp16(v) == float(np.float16(v)), v


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(2)
    vals = (rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000)).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.bfloat16).double().numpy()
    for v, r in zip(vals.astype(np.float64), ref):
        assert O.round_bf16(v) == r, v


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(3)
    vals = (rng.standard_normal(4000) * 10.0 ** rng.uniform(-3, 2.6, 4000)).astype(np.float32)
    vals = vals[np.abs(vals) < 448.0]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals.astype(np.float64), ref):
        assert O.e4m3(v) == int(r), v
    # saturating beyond the largest finite value, signs kept
    assert O.e4m3(1e6) == 0x7E and O.e4m3(-1e6) == 0xFE
    assert O.e4m3_value(0x7E) == 448.0


# --------------------------------------------------------------------------
# rotation R = H D / sqrt(d)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [8, 128])
def test_rotation_equals_sylvester_matrix(d):
    P = O.make_params(d, 2, seed=5, with_S=False)
    H = scipy.linalg.hadamard(d).astype(np.float64)   # natural-order Sylvester
    R = H @ np.diag(P.signs.astype(np.float64)) / math.sqrt(d)
    rng = np.random.default_rng(d)
    X = rng.standard_normal((16, d))
    assert np.allclose(O.rotate(X, P.signs), X @ R.T, atol=1e-12, rtol=0)
    assert np.allclose(O.rotate_t(X, P.signs), X @ R, atol=1e-12, rtol=0)


@pytest.mark.parametrize("d", [8, 128, 1024])
def test_rotation_is_orthogonal(d):
    P = O.make_params(d, 2, seed=9, with_S=False)
    E = O.rotate(np.eye(d), P.signs)          # rows: R e_i -> columns of R
    assert np.allclose(E @ E.T, np.eye(d), atol=1e-12)
    x = np.random.default_rng(0).standard_normal((4, d))
    assert np.allclose(np.linalg.norm(O.rotate(x, P.signs), axis=1), np.linalg.norm(x, axis=1),
                       rtol=1e-13, atol=0)


# --------------------------------------------------------------------------
# Lloyd-Max codebook for the coordinate law of a random unit vector
# --------------------------------------------------------------------------
def _coord_law(d):
    # (T + 1) / 2 ~ Beta((d-1)/2, (d-1)/2) for one coordinate T of a uniform
    # random unit vector in R^d: an independent library description of f_d.
    a = (d - 1) / 2.0
    return scipy.stats.beta(a, a, loc=-1.0, scale=2.0)


@pytest.mark.parametrize("d,bits", [(8, 1), (8, 2), (8, 3), (128, 2), (128, 3), (128, 4),
                                    (1024, 4)])
def test_codebook_fixed_point_conditions(d, bits):
    c64, c32, t32 = O.codebook(d, bits)
    law = _coord_law(d)
    L = 1 << bits
    edges = np.concatenate([[-1.0], 0.5 * (c64[:-1] + c64[1:]), [1.0]])
    for j in range(L):
        lo, hi = edges[j], edges[j + 1]
        mass = law.cdf(hi) - law.cdf(lo)
        mom = scipy.integrate.quad(lambda t: t * law.pdf(t), lo, hi, epsabs=1e-15,
                                   epsrel=1e-13, limit=400)[0]
        assert abs(mom / mass - c64[j]) < 1e-10, (j, mom / mass, c64[j])
    # symmetry, and fp32 boundaries are midpoints of the fp32 levels
    assert np.all(c32 == -c32[::-1])
    assert np.all(t32 == ((c32[:-1].astype(np.float64) + c32[1:]) / 2).astype(np.float32))
    assert np.all(np.diff(c32) > 0)


@pytest.mark.parametrize("d", [8, 16, 128, 1024])
def test_codebook_one_bit_closed_form(d):
    # b = 1: the levels are +-E|T| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    c64, _, _ = O.codebook(d, 1)
    ref = math.exp(scipy.special.gammaln(d / 2) - scipy.special.gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    assert abs(c64[1] - ref) < 1e-12 and abs(c64[0] + ref) < 1e-12
    if d == 8:
        assert abs(c64[1] - 0.29103) < 5e-6


def test_codebook_tends_to_gaussian_lloyd_max():
    table = _gold("gaussian_lloyd_max.json")["levels"]
    for b in (1, 2, 3, 4):
        ref = np.array(table[str(b)])
        err = {}
        for d in (128, 1024):
            c64, _, _ = O.codebook(d, b)
            pos = math.sqrt(d) * c64[(1 << (b - 1)):]
            err[d] = np.max(np.abs(pos - ref) / ref)
        assert err[1024] < 6e-3, (b, err)
        assert err[1024] <= err[128] + 1e-4, (b, err)


def test_codebook_parameter_count_matches_pages():
    g = _gold("pages_numbers.json")
    c64, c32, t32 = O.codebook(128, 3)
    extra = g["turboquant_params_3bit_d128"]["value"] - g["dense_rotation_params_d128"]["value"]
    assert len(c32) + len(t32) == extra == 15
    assert 128 * 128 == g["dense_rotation_params_d128"]["value"]


# --------------------------------------------------------------------------
# quantizer: nearest codeword by brute force at d = 8
# --------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [2, 3])
def test_bucketize_is_nearest_codeword_bruteforce(bits):
    d = 8
    P = O.make_params(d, bits, seed=11)
    L = 1 << bits
    rng = np.random.default_rng(bits)
    X = rng.standard_normal((4, d))
    enc = O.encode(X, P, qjl=False)
    U = O.rotate(X, P.signs) / np.linalg.norm(X, axis=1, keepdims=True)
    c = P.c32.astype(np.float64)
    total = L ** d
    for v in range(X.shape[0]):
        best, bestd = None, np.inf
        for start in range(0, total, 1 << 20):
            ids = np.arange(start, min(total, start + (1 << 20)), dtype=np.int64)
            digits = (ids[:, None] // (L ** np.arange(d))[None, :]) % L
            dist = ((U[v][None, :] - c[digits]) ** 2).sum(1)
            k = int(np.argmin(dist))
            if dist[k] < bestd:
                bestd, best = dist[k], digits[k]
        assert np.array_equal(best, enc.idx[v].astype(np.int64))


# --------------------------------------------------------------------------
# distortion: within 2.7x of 4^-b (pages), and equal to the law's integral
# --------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_mse_within_pages_bound_and_matches_integral(bits):
    d, n = 128, 100_000
    P = O.make_params(d, bits, seed=21, with_S=False)
    X = np.random.default_rng(100 + bits).standard_normal((n, d))
    enc = O.encode(X, P, qjl=False, margins=False)
    Y = O.rotate(X, P.signs)
    rec = enc.nhat[:, None] * P.c32.astype(np.float64)[enc.idx]
    nmse = np.mean(np.sum((Y - rec) ** 2, 1) / np.sum(X ** 2, 1))
    bound = _gold("pages_numbers.json")["distortion_factor_vs_information_limit"]["value"] * 4.0 ** -bits
    assert nmse <= bound, (nmse, bound)
    # d * E[(T - Q(T))^2] under the coordinate law, by scipy quadrature
    law = _coord_law(d)
    c = P.c32.astype(np.float64)
    t = np.concatenate([[-1.0], P.t32.astype(np.float64), [1.0]])
    pred = d * sum(scipy.integrate.quad(lambda x, cj=c[j]: (x - cj) ** 2 * law.pdf(x), t[j], t[j + 1],
                                        epsabs=1e-14, limit=400)[0] for j in range(len(c)))
    assert abs(nmse - pred) / pred < 0.01, (nmse, pred)


# --------------------------------------------------------------------------
# QJL: the estimator is unbiased; without stage 2 it is biased
# --------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [2, 3])
def test_qjl_estimator_unbiased_over_seeds(bits):
    d, n_seeds = 128, 10_000
    rng = np.random.default_rng(7)
    k = rng.standard_normal(d)
    k[5] *= 20.0
    q = rng.standard_normal(d)
    q = q + 0.8 * k / np.linalg.norm(k) * np.linalg.norm(q)   # a sizeable <q, k>
    truth = float(q @ k)
    est_qjl = np.zeros(n_seeds)
    est_mse = np.zeros(n_seeds)
    for s in range(n_seeds):
        P = O.make_params(d, bits, seed=1000 + s)
        E = O.encode(k[None, :], P, qjl=True, margins=False)
        est_qjl[s] = O.estimate(q, P, E)[0]
        E0 = O.Encoded(bits, False, E.idx, E.nhat)
        est_mse[s] = O.estimate(q, P, E0)[0]
    se = est_qjl.std(ddof=1) / math.sqrt(n_seeds)
    assert abs(est_qjl.mean() - truth) < 3 * se, (est_qjl.mean(), truth, se)
    # the MSE-only estimate shrinks <q,k> (biased), as the pages state
    se0 = est_mse.std(ddof=1) / math.sqrt(n_seeds)
    assert abs(est_mse.mean() - truth) > 6 * se0, (est_mse.mean(), truth, se0)


# --------------------------------------------------------------------------
# attention and search
# --------------------------------------------------------------------------
def test_exact_attention_is_textbook_softmax():
    rng = np.random.default_rng(4)
    Q, K, V = rng.standard_normal((3, 5, 16)), rng.standard_normal((40, 16)), rng.standard_normal((40, 16))
    Q = Q[0]
    out = O.attend_exact(Q, K, V)
    ref = scipy.special.softmax(Q @ K.T / 4.0, axis=1) @ V
    assert np.allclose(out, ref, atol=1e-13)


def test_attention_single_key_returns_dequantized_value():
    d = 128
    rng = np.random.default_rng(8)
    Pk, Pv = O.make_params(d, 2, 1), O.make_params(d, 4, 2)
    K, V = rng.standard_normal((1, d)), rng.standard_normal((1, d))
    Ek, Ev = O.encode(K, Pk, qjl=True), O.encode(V, Pv, qjl=False)
    out, lse, logits = O.attend(rng.standard_normal((3, d)), Pk, Ek, Pv, Ev, want_logits=True)
    H = scipy.linalg.hadamard(d) / math.sqrt(d)
    vhat = (np.diag(Pv.signs.astype(float)) @ H @ (Ev.nhat[0] * Pv.c32.astype(float)[Ev.idx[0]]))
    assert np.allclose(out, vhat[None, :], atol=1e-12)
    assert np.allclose(lse, logits[:, 0], atol=1e-12)


def test_attention_weights_sum_to_one_and_causal_prefix():
    d, L = 128, 300
    rng = np.random.default_rng(9)
    Pk, Pv = O.make_params(d, 2, 3), O.make_params(d, 3, 4)
    K, V = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    Ek, Ev = O.encode(K, Pk, qjl=True), O.encode(V, Pv, qjl=False)
    Q = rng.standard_normal((4, d))
    out, lse, logits = O.attend(Q, Pk, Ek, Pv, Ev, want_logits=True)
    # logits are the estimates scaled by 1/sqrt(d); weights exp(l - lse) sum to 1
    for a in range(4):
        assert np.allclose(logits[a], O.estimate(Q[a], Pk, Ek) / math.sqrt(d), atol=1e-12)
        assert abs(np.exp(logits[a] - lse[a]).sum() - 1.0) < 1e-12
    # a query that sees a prefix equals attention over the truncated sequence
    nv = np.array([1, 57, 200, L], np.int32)
    o2, _, _ = O.attend(Q, Pk, Ek, Pv, Ev, nvis=nv)
    for a in range(4):
        sub = lambda E: O.Encoded(E.bits, E.qjl, E.idx[:nv[a]], E.nhat[:nv[a]],
                                  None if E.rho is None else E.rho[:nv[a]],
                                  None if E.sbits is None else E.sbits[:nv[a]])
        o3, _, _ = O.attend(Q[a:a + 1], Pk, sub(Ek), Pv, sub(Ev))
        assert np.allclose(o2[a], o3[0], atol=1e-13)


def test_search_topk_matches_sorting_with_ties():
    d, n = 64, 500
    rng = np.random.default_rng(10)
    P = O.make_params(d, 4, 5)
    X = rng.standard_normal((n, d))
    X[123] = X[45]          # identical vectors -> identical scores (a tie)
    X[400] = X[45]
    E = O.encode(X, P, qjl=True, margins=False)
    Q = rng.standard_normal((3, d))
    Q[0] = X[45] * 3.0      # make the tied vectors the best matches
    sc, ix = O.search(Q, P, E, 10)
    for a in range(3):
        est = O.estimate(Q[a], P, E)
        order = np.lexsort((np.arange(n), -est))[:10]      # score desc, index asc
        assert np.array_equal(ix[a], order)
        assert np.array_equal(sc[a], est[order])
    assert list(ix[0][:3]) == [45, 123, 400]


# --------------------------------------------------------------------------
# layout
# --------------------------------------------------------------------------
@pytest.mark.parametrize("kbits,kqjl,vbits,per_token", [(2, True, 4, 118), (2, True, 3, 102),
                                                        (8, False, 4, 196), (4, True, 4, 150),
                                                        (3, True, 3, 118)])
def test_layout_byte_counts(kbits, kqjl, vbits, per_token):
    lay = O.Layout(128, kbits, kqjl, vbits, page_tokens=64)
    assert lay.page_bytes == 64 * per_token
    # one fp16 norm per vector (plus rho for QJL keys): no per-block scales
    scale_bytes = sum(b for n, (o, b) in lay.fields.items() if n in ("kn", "kr", "vn"))
    assert scale_bytes == (6 if kqjl else 4)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, (50, 128)).astype(np.uint8)
    kap = O.to_kappa(idx, bits)
    assert np.array_equal(O.from_kappa(kap, bits), idx)
    for w in (1, 2, 4, 8):
        v = rng.integers(0, 1 << w, (7, 64)).astype(np.uint8)
        assert np.array_equal(O.unpack_fields(O.pack_fields(v, w), 64, w), v)
    # field i sits at bit offset i*w, little-endian
    v = np.zeros((1, 16), np.uint8)
    v[0, 3] = 0b1011
    assert O.pack_fields(v, 4)[0, 1] == 0b10110000


def test_cache_write_read_roundtrip():
    d = 128
    rng = np.random.default_rng(12)
    lay = O.Layout(d, 3, True, 3, page_tokens=16)
    Pk, Pv = O.make_params(d, 3, 1), O.make_params(d, 3, 2)
    X = rng.standard_normal((40, d))
    Ek, Ev = O.encode(X, Pk, qjl=True), O.encode(X[::-1].copy(), Pv, qjl=False)
    nheads = 2
    cache = np.zeros((4 * nheads, lay.page_bytes), np.uint8)
    slots = rng.permutation(64)[:40]
    O.write_cache(lay, cache, slots, 1, nheads, Ek, Ev)
    back = O.read_cache(lay, cache, slots, 1, nheads)
    assert np.array_equal(back["kidx"], Ek.idx) and np.array_equal(back["vidx"], Ev.idx)
    assert np.array_equal(back["ks"], Ek.sbits)
    assert np.array_equal(back["kn"], Ek.nhat) and np.array_equal(back["kr"], Ek.rho)
    assert np.array_equal(back["vn"], Ev.nhat)
    assert not cache[0::2].any()          # head 0 pages untouched


# --------------------------------------------------------------------------
# attention through the oracle's own compressed path, on keys and values
# that its codes represent exactly (the identity quantizer in code form)
# --------------------------------------------------------------------------
def _exact_from_codes(P, idx, nhat):
    """Vectors x_t = R^T (nhat_t c[idx_t]) built with scipy's Hadamard matrix,
    so that the oracle's encoded form (idx, nhat) reconstructs them exactly."""
    d = P.d
    R = scipy.linalg.hadamard(d).astype(np.float64) @ np.diag(P.signs.astype(np.float64)) / math.sqrt(d)
    Y = nhat[:, None] * P.c32.astype(np.float64)[idx]
    return Y @ R          # rows: (R^T y_t)^T


@pytest.mark.parametrize("L,nq", [(300, 5), (777, 3)])
def test_attend_equals_textbook_softmax_on_exactly_coded_kv(L, nq):
    d = 128
    rng = np.random.default_rng(L)
    Pk, Pv = O.make_params(d, 4, 31, with_S=False), O.make_params(d, 3, 32, with_S=False)
    kidx = rng.integers(0, 16, (L, d)).astype(np.uint8)
    vidx = rng.integers(0, 8, (L, d)).astype(np.uint8)
    kn = np.array([O.round_fp16(v) for v in rng.uniform(2.0, 30.0, L)])
    vn = np.array([O.round_fp16(v) for v in rng.uniform(0.5, 8.0, L)])
    Kx, Vx = _exact_from_codes(Pk, kidx, kn), _exact_from_codes(Pv, vidx, vn)
    Ek, Ev = O.Encoded(4, False, kidx, kn), O.Encoded(3, False, vidx, vn)
    Q = rng.standard_normal((nq, d)) * 1.5
    nvis = np.array([L, 1, L // 2, L - 3, 64][:nq], np.int32)
    out, lse, logits = O.attend(Q, Pk, Ek, Pv, Ev, nvis=nvis, want_logits=True)
    for a in range(nq):
        n = nvis[a]
        lg = Q[a] @ Kx[:n].T / math.sqrt(d)
        ref = scipy.special.softmax(lg) @ Vx[:n]
        assert np.allclose(out[a], ref, atol=1e-11, rtol=0), a
        assert abs(lse[a] - scipy.special.logsumexp(lg)) < 1e-11
        assert np.allclose(logits[a, :n], lg, atol=1e-11, rtol=0)
        assert np.all(np.isneginf(logits[a, n:]))


# --------------------------------------------------------------------------
# FP8 keys: code = torch's E4M3 cast of sqrt(d) R x / ||x||
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [8, 128, 1024])
def test_fp8_encode_matches_torch_e4m3_of_rotated_unit_vector(d):
    rng = np.random.default_rng(d + 5)
    P = O.make_params(d, 8, 77, with_S=False)
    X = rng.standard_normal((40, d)) * np.exp(rng.standard_normal(d))[None, :]
    X[3] = 0.0
    enc = O.encode(X, P, qjl=False)
    R = scipy.linalg.hadamard(d).astype(np.float64) @ np.diag(P.signs.astype(np.float64)) / math.sqrt(d)
    n = np.linalg.norm(X, axis=1)
    Y = X @ R.T
    U = np.where(n[:, None] > 0, Y / np.where(n > 0, n, 1.0)[:, None], 0.0)
    a = math.sqrt(d) * U
    # compare only where the oracle's value is not within 1e-9 of a rounding midpoint
    # (torch casts from fp32; the oracle rounds the float64 value)
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    clear = enc.umargin * math.sqrt(d) > 1e-6 * np.maximum(1.0, np.abs(a))
    assert clear.mean() > 0.99
    assert np.array_equal(enc.idx[clear], ref[clear])
    assert np.array_equal(enc.nhat, n.astype(np.float16).astype(np.float64))
    # reconstruction nhat e4m3(code) / sqrt(d) within half an E4M3 step of R x (plus the fp16 norm's rounding)
    val = torch.from_numpy(enc.idx.copy()).view(torch.float8_e4m3fn).double().numpy()
    rec = enc.nhat[:, None] * val / math.sqrt(d)
    half_step = np.where(np.abs(a) >= 2.0 ** -6, np.exp2(np.floor(np.log2(np.maximum(np.abs(a), 1e-300))) - 4),
                         2.0 ** -10)
    bound = n[:, None] * half_step / math.sqrt(d) * (1 + 1e-9) + np.abs(Y) * 2.0 ** -11
    assert np.all(np.abs(rec - Y) <= bound)
    assert np.all(enc.idx[3] == 0) and enc.nhat[3] == 0.0


# --------------------------------------------------------------------------
# exemption margins against direct numpy distances
# --------------------------------------------------------------------------
def test_code_and_sign_margins_match_direct_distances():
    d = 128
    rng = np.random.default_rng(55)
    P = O.make_params(d, 3, 91)
    X = rng.standard_normal((12, d))
    X[:, 5] *= 20.0
    enc = O.encode(X, P, qjl=True)
    R = scipy.linalg.hadamard(d).astype(np.float64) @ np.diag(P.signs.astype(np.float64)) / math.sqrt(d)
    n = np.linalg.norm(X, axis=1)
    U = (X @ R.T) / n[:, None]
    t = P.t32.astype(np.float64)
    um = np.min(np.abs(U[:, :, None] - t[None, None, :]), axis=2)
    assert np.allclose(enc.umargin, um, rtol=0, atol=1e-13)
    r = X @ R.T - enc.nhat[:, None] * P.c32.astype(np.float64)[enc.idx]
    Z = r @ P.S.astype(np.float64).T
    zm = np.abs(Z) / (np.linalg.norm(r, axis=1)[:, None] * np.linalg.norm(P.S.astype(np.float64), axis=1)[None, :])
    assert np.allclose(enc.zmargin, zm, rtol=1e-9, atol=1e-15)
    assert np.array_equal(enc.sbits, (Z >= 0).astype(np.uint8))


def test_fp8_margin_matches_direct_distance_to_rounding_midpoints():
    d = 64
    rng = np.random.default_rng(56)
    P = O.make_params(d, 8, 92, with_S=False)
    X = rng.standard_normal((6, d))
    enc = O.encode(X, P, qjl=False)
    vals = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()  # finite, >= 0
    mids = 0.5 * (vals[:-1] + vals[1:])
    R = scipy.linalg.hadamard(d).astype(np.float64) @ np.diag(P.signs.astype(np.float64)) / math.sqrt(d)
    a = math.sqrt(d) * (X @ R.T) / np.linalg.norm(X, axis=1)[:, None]
    mg = np.min(np.abs(np.abs(a)[:, :, None] - mids[None, None, :]), axis=2) / math.sqrt(d)
    assert np.allclose(enc.umargin, mg, rtol=0, atol=1e-13)


def test_attend_with_fp8_keys_equals_textbook_softmax_on_exactly_coded_kv():
    """The FP8-key estimator nhat <Rq, e4m3(code)> / sqrt(d) on keys that the
    codes represent exactly: attention equals scipy's softmax(QK^T/sqrt(d))V."""
    d, L, nq = 128, 400, 4
    rng = np.random.default_rng(8)
    Pk, Pv = O.make_params(d, 8, 33, with_S=False), O.make_params(d, 4, 34, with_S=False)
    codes = rng.integers(0, 0x7F, (L, d)).astype(np.uint8) | (rng.integers(0, 2, (L, d)).astype(np.uint8) << 7)
    kn = np.array([O.round_fp16(v) for v in rng.uniform(1.0, 40.0, L)])
    vidx = rng.integers(0, 16, (L, d)).astype(np.uint8)
    vn = np.array([O.round_fp16(v) for v in rng.uniform(0.5, 8.0, L)])
    vals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    R = scipy.linalg.hadamard(d).astype(np.float64) @ np.diag(Pk.signs.astype(np.float64)) / math.sqrt(d)
    Kx = (kn[:, None] * vals / math.sqrt(d)) @ R
    Vx = _exact_from_codes(Pv, vidx, vn)
    Ek, Ev = O.Encoded(8, False, codes, kn), O.Encoded(4, False, vidx, vn)
    Q = rng.standard_normal((nq, d))
    out, lse, logits = O.attend(Q, Pk, Ek, Pv, Ev, want_logits=True)
    lg = Q @ Kx.T / math.sqrt(d)
    assert np.allclose(logits, lg, atol=1e-11, rtol=0)
    assert np.allclose(out, scipy.special.softmax(lg, axis=1) @ Vx, atol=1e-11, rtol=0)
    assert np.allclose(lse, scipy.special.logsumexp(lg, axis=1), atol=1e-11, rtol=0)


# --------------------------------------------------------------------------
# dense random rotation (the alternative to H D / sqrt(d))
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d,seed", [(8, 3), (128, 5), (256, 6)])
def test_dense_rotation_is_numpy_qr_in_float32(d, seed):
    G, Q, Rm = O.dense_rotation(d, seed)
    # G: iid N(0,1) from its own stream (moments; a KS test against scipy's normal law)
    g = G.ravel()
    assert abs(g.mean()) < 5 / math.sqrt(g.size) and abs(g.var() - 1.0) < 5 * math.sqrt(2.0 / g.size)
    if d >= 128:
        assert scipy.stats.kstest(g, "norm").pvalue > 1e-4
    # rows of Q = Gram-Schmidt of the rows of G = numpy's QR of G^T with a positive diagonal
    q, r = np.linalg.qr(G.T)
    q = q * np.sign(np.diag(r))[None, :]
    assert np.allclose(Q, q.T, atol=1e-10, rtol=0)
    # stored entries: numpy's float32 rounding of Q
    assert np.array_equal(Rm, Q.astype(np.float32).astype(np.float64))
    # orthogonal to float32 precision
    assert np.max(np.abs(Rm @ Rm.T - np.eye(d))) < 1e-6
    # the rotation routines use it (y = Rm x, x = Rm^T y)
    P = O.make_params(d, 2, seed, with_S=False, rotation="dense")
    X = np.random.default_rng(d).standard_normal((5, d))
    assert np.allclose(O.rotate(X, P.signs, P.Rm), X @ Rm.T, atol=1e-12, rtol=0)
    assert np.allclose(O.rotate_t(X, P.signs, P.Rm), X @ Rm, atol=1e-12, rtol=0)


@pytest.mark.parametrize("bits", [2, 3])
def test_dense_rotation_bucketize_is_nearest_codeword_bruteforce(bits):
    d = 8
    P = O.make_params(d, bits, seed=12, rotation="dense")
    L = 1 << bits
    X = np.random.default_rng(20 + bits).standard_normal((4, d))
    enc = O.encode(X, P, qjl=False)
    Y = X @ P.Rm.T
    U = Y / np.linalg.norm(Y, axis=1, keepdims=True)            # n = ||R x|| for the dense rotation
    assert np.allclose(enc.nraw, np.linalg.norm(Y, axis=1), rtol=1e-14)
    c = P.c32.astype(np.float64)
    digits = (np.arange(L ** d)[:, None] // (L ** np.arange(d))[None, :]) % L
    for v in range(X.shape[0]):
        dist = ((U[v][None, :] - c[digits]) ** 2).sum(1)
        assert np.array_equal(digits[int(np.argmin(dist))], enc.idx[v].astype(np.int64))


def test_dense_rotation_mse_within_pages_bound_and_attention_textbook():
    d, n, bits = 128, 20000, 3
    P = O.make_params(d, bits, seed=31, with_S=False, rotation="dense")
    X = np.random.default_rng(5).standard_normal((n, d)) * np.exp(np.random.default_rng(6).standard_normal(d))
    enc = O.encode(X, P, qjl=False, margins=False)
    Y = X @ P.Rm.T
    rec = enc.nhat[:, None] * P.c32.astype(np.float64)[enc.idx]
    nmse = np.mean(np.sum((Y - rec) ** 2, 1) / np.sum(Y ** 2, 1))
    bound = _gold("pages_numbers.json")["distortion_factor_vs_information_limit"]["value"] * 4.0 ** -bits
    assert nmse <= bound, (nmse, bound)
    # attention with dense rotations, on K/V the codes represent exactly
    rng = np.random.default_rng(7)
    L = 200
    Pk, Pv = O.make_params(d, 4, 41, with_S=False, rotation="dense"), O.make_params(d, 2, 42, with_S=False,
                                                                                     rotation="dense")
    kidx, vidx = rng.integers(0, 16, (L, d)).astype(np.uint8), rng.integers(0, 4, (L, d)).astype(np.uint8)
    kn, vn = (np.array([O.round_fp16(v) for v in rng.uniform(1.0, 9.0, L)]) for _ in range(2))
    Kx = (kn[:, None] * Pk.c32.astype(np.float64)[kidx]) @ Pk.Rm
    Vx = (vn[:, None] * Pv.c32.astype(np.float64)[vidx]) @ Pv.Rm
    Q = rng.standard_normal((3, d))
    out, lse, _ = O.attend(Q, Pk, O.Encoded(4, False, kidx, kn), Pv, O.Encoded(2, False, vidx, vn))
    lg = Q @ Kx.T / math.sqrt(d)               # <Rm q, nhat c> = <q, Rm^T nhat c>
    assert np.allclose(out, scipy.special.softmax(lg, axis=1) @ Vx, atol=1e-10, rtol=0)
    assert np.allclose(lse, scipy.special.logsumexp(lg, axis=1), atol=1e-10, rtol=0)


# --------------------------------------------------------------------------
# fractional rates b + 1/2: coordinates 0 .. d/2-1 at b + 1 bits, the rest at b
# --------------------------------------------------------------------------
def test_fractional_rate_bucketize_is_nearest_codeword_bruteforce():
    d, rate = 8, 2.5
    P = O.make_params(d, rate, seed=13)
    assert (P.bits, P.bits2) == (3, 2)
    X = np.random.default_rng(25).standard_normal((3, d))
    enc = O.encode(X, P, qjl=False)
    U = O.rotate(X, P.signs) / np.linalg.norm(X, axis=1, keepdims=True)
    ca, cb = P.c32.astype(np.float64), P.c32b.astype(np.float64)
    da = (np.arange(8 ** 4)[:, None] // (8 ** np.arange(4))[None, :]) % 8
    db = (np.arange(4 ** 4)[:, None] // (4 ** np.arange(4))[None, :]) % 4
    for v in range(3):
        # the squared error separates over the two halves: each half's nearest codeword independently
        ea = ((U[v, :4][None, :] - ca[da]) ** 2).sum(1)
        eb = ((U[v, 4:][None, :] - cb[db]) ** 2).sum(1)
        best = np.concatenate([da[int(np.argmin(ea))], db[int(np.argmin(eb))]])
        assert np.array_equal(best, enc.idx[v].astype(np.int64))
        # and the joint search over all 8^4 x 4^4 code vectors agrees
        tot = ea[:, None] + eb[None, :]
        ia, ib = np.unravel_index(int(np.argmin(tot)), tot.shape)
        assert np.array_equal(np.concatenate([da[ia], db[ib]]), enc.idx[v].astype(np.int64))


@pytest.mark.parametrize("rate", [1.5, 2.5, 3.5])
def test_fractional_rate_mse_is_the_mean_of_its_two_codebooks(rate):
    d, n = 128, 40000
    P = O.make_params(d, rate, seed=27, with_S=False)
    X = np.random.default_rng(int(rate * 10)).standard_normal((n, d))
    enc = O.encode(X, P, qjl=False, margins=False)
    Y = O.rotate(X, P.signs)
    lv = np.concatenate([P.c32.astype(np.float64)[enc.idx[:, :64]], P.c32b.astype(np.float64)[enc.idx[:, 64:]]], 1)
    nmse = np.mean(np.sum((Y - enc.nhat[:, None] * lv) ** 2, 1) / np.sum(X ** 2, 1))
    law = _coord_law(d)

    def dist(c, t):
        e = np.concatenate([[-1.0], t.astype(np.float64), [1.0]])
        c = c.astype(np.float64)
        return d * sum(scipy.integrate.quad(lambda x, cj=c[j]: (x - cj) ** 2 * law.pdf(x), e[j], e[j + 1],
                                            epsabs=1e-14, limit=400)[0] for j in range(len(c)))
    pred = 0.5 * (dist(P.c32, P.t32) + dist(P.c32b, P.t32b))
    assert abs(nmse - pred) / pred < 0.02, (nmse, pred)
    lo, hi = O.make_params(d, P.bits, 1, with_S=False), O.make_params(d, P.bits2, 1, with_S=False)
    assert dist(lo.c32, lo.t32) < nmse < dist(hi.c32, hi.t32)


@pytest.mark.parametrize("kbits,kqjl,vbits,per_token", [(2.5, True, 3.5, 40 + 16 + 4 + 56 + 2),
                                                        (1.5, True, 2.5, 24 + 16 + 4 + 40 + 2),
                                                        (3.5, False, 2.5, 56 + 2 + 40 + 2)])
def test_fractional_layout_byte_counts_and_roundtrip(kbits, kqjl, vbits, per_token):
    d = 128
    lay = O.Layout(d, kbits, kqjl, vbits, page_tokens=16)
    assert lay.page_bytes == 16 * per_token
    rng = np.random.default_rng(3)
    Pk, Pv = O.make_params(d, kbits, 1), O.make_params(d, vbits, 2, with_S=False)
    X = rng.standard_normal((20, d))
    Ek, Ev = O.encode(X, Pk, qjl=kqjl), O.encode(X[::-1].copy(), Pv, qjl=False)
    cache = np.zeros((2 * 2, lay.page_bytes), np.uint8)
    slots = rng.permutation(32)[:20]
    O.write_cache(lay, cache, slots, 0, 2, Ek, Ev)
    back = O.read_cache(lay, cache, slots, 0, 2)
    assert np.array_equal(back["kidx"], Ek.idx) and np.array_equal(back["vidx"], Ev.idx)
    assert int(Ek.idx[:, :64].max()) < (1 << Pk.bits) and int(Ek.idx[:, 64:].max()) < (1 << Pk.bits2)


def test_fractional_rate_attention_and_qjl_unbiased():
    d = 128
    rng = np.random.default_rng(17)
    Pk, Pv = O.make_params(d, 3.5, 51, with_S=False), O.make_params(d, 2.5, 52, with_S=False)
    L = 150
    kidx = np.concatenate([rng.integers(0, 16, (L, 64)), rng.integers(0, 8, (L, 64))], 1).astype(np.uint8)
    vidx = np.concatenate([rng.integers(0, 8, (L, 64)), rng.integers(0, 4, (L, 64))], 1).astype(np.uint8)
    kn, vn = (np.array([O.round_fp16(v) for v in rng.uniform(1.0, 9.0, L)]) for _ in range(2))
    H = scipy.linalg.hadamard(d).astype(np.float64)
    R = lambda P: H @ np.diag(P.signs.astype(np.float64)) / math.sqrt(d)
    lvk = np.concatenate([Pk.c32.astype(np.float64)[kidx[:, :64]], Pk.c32b.astype(np.float64)[kidx[:, 64:]]], 1)
    lvv = np.concatenate([Pv.c32.astype(np.float64)[vidx[:, :64]], Pv.c32b.astype(np.float64)[vidx[:, 64:]]], 1)
    Kx, Vx = (kn[:, None] * lvk) @ R(Pk), (vn[:, None] * lvv) @ R(Pv)
    Q = rng.standard_normal((3, d))
    out, lse, _ = O.attend(Q, Pk, O.Encoded(3.5, False, kidx, kn), Pv, O.Encoded(2.5, False, vidx, vn))
    lg = Q @ Kx.T / math.sqrt(d)
    assert np.allclose(out, scipy.special.softmax(lg, axis=1) @ Vx, atol=1e-10, rtol=0)
    # stage 2 keeps the 2.5-bit estimate unbiased
    k = rng.standard_normal(d)
    q = rng.standard_normal(d) + 0.7 * k
    est = np.array([O.estimate(q, P, O.encode(k[None, :], P, qjl=True, margins=False))[0]
                    for P in (O.make_params(d, 2.5, 3000 + s) for s in range(3000))])
    assert abs(est.mean() - q @ k) < 3 * est.std(ddof=1) / math.sqrt(len(est))


# --------------------------------------------------------------------------
# PolarQuant: the polar-coordinate angle quantizer
# --------------------------------------------------------------------------
@pytest.mark.parametrize("k", [2, 4, 16, 64])
def test_polar_angle_codebook_fixed_point_under_beta_law(k):
    # for a random direction, the angle psi between two k-dimensional
    # sub-block radii has sin^2 psi ~ Beta(k/2, k/2) (ratio of chi-squares)
    c64, c32, t32 = O.polar_codebook(k, 2)
    law = scipy.stats.beta(k / 2, k / 2)
    pdf = lambda p: law.pdf(math.sin(p) ** 2) * 2 * math.sin(p) * math.cos(p)
    edges = np.concatenate([[0.0], 0.5 * (c64[:-1] + c64[1:]), [math.pi / 2]])
    for j in range(4):
        mass = scipy.integrate.quad(pdf, edges[j], edges[j + 1], epsabs=1e-14, limit=400)[0]
        mom = scipy.integrate.quad(lambda p: p * pdf(p), edges[j], edges[j + 1], epsabs=1e-14, limit=400)[0]
        assert abs(mom / mass - c64[j]) < 1e-9, (k, j)
    assert np.allclose(c64 + c64[::-1], math.pi / 2, atol=1e-14)
    assert np.all(t32 == ((c32[:-1].astype(np.float64) + c32[1:]) / 2).astype(np.float32))
    # and the law itself: angles of Gaussian sub-blocks (numpy) pass a KS test against it
    g = np.random.default_rng(k).standard_normal((20000, 2 * k))
    psi = np.arctan2(np.linalg.norm(g[:, k:], axis=1), np.linalg.norm(g[:, :k], axis=1))
    assert scipy.stats.kstest(np.sin(psi) ** 2, law.cdf).pvalue > 1e-4


def test_polar_d2_and_d4_against_numpy():
    P2 = O.polar_params(2, 3, with_S=False)
    X = np.random.default_rng(1).standard_normal((200, 2))
    E = O.encode_polar(X, P2, qjl=False)
    Y = O.rotate(X, P2.signs)
    th = np.mod(np.arctan2(Y[:, 1], Y[:, 0]), 2 * np.pi)
    code = np.floor(th / (2 * np.pi / 16)).astype(int)
    clear = E.margin1[:, 0] > 1e-9
    assert np.array_equal(E.codes1[clear, 0], code[clear])
    c = P2.c1.astype(np.float64)[E.codes1[:, 0]]
    assert np.allclose(E.yhat, E.nhat[:, None] * np.stack([np.cos(c), np.sin(c)], 1), atol=1e-14)
    P4 = O.polar_params(4, 4, with_S=False)
    X = np.random.default_rng(2).standard_normal((200, 4))
    E = O.encode_polar(X, P4, qjl=False)
    Y = O.rotate(X, P4.signs)
    psi = np.arctan2(np.hypot(Y[:, 2], Y[:, 3]), np.hypot(Y[:, 0], Y[:, 1]))
    ref = np.searchsorted(P4.th[0].astype(np.float64), psi, side="right")
    clear = E.marginh[:, 0] > 1e-9
    assert np.array_equal(E.codesh[clear, 0], ref[clear])
    ps = P4.ch[0].astype(np.float64)[E.codesh[:, 0]]
    t1, t2 = (P4.c1.astype(np.float64)[E.codes1[:, j]] for j in (0, 1))
    yh = E.nhat[:, None] * np.stack([np.cos(ps) * np.cos(t1), np.cos(ps) * np.sin(t1),
                                     np.sin(ps) * np.cos(t2), np.sin(ps) * np.sin(t2)], 1)
    assert np.allclose(E.yhat, yh, atol=1e-13)


def test_polar_decode_encode_idempotent_and_scale_free():
    d = 128
    P = O.polar_params(d, 6, with_S=False)
    X = np.random.default_rng(3).standard_normal((30, d)) * np.exp(np.random.default_rng(4).standard_normal(d))
    E = O.encode_polar(X, P, qjl=False)
    assert np.allclose(np.linalg.norm(E.yhat, axis=1), E.nhat, rtol=1e-13)     # only the radius is stored
    E2 = O.encode_polar(O.rotate_t(E.yhat, P.signs), P, qjl=False)              # the decoded vector re-encodes to itself
    assert np.array_equal(E2.codes1, E.codes1) and np.array_equal(E2.codesh, E.codesh)
    assert np.allclose(E2.yhat, E.yhat, atol=1e-12)
    E3 = O.encode_polar(4.0 * X, P, qjl=False)                                 # no scale besides the norm
    assert np.array_equal(E3.codes1, E.codes1) and np.array_equal(E3.codesh, E.codesh)
    assert np.array_equal(E3.nhat, 4.0 * E.nhat)
    # distortion: better than the 2-bit Lloyd-Max coordinate quantizer at ~3 bits per coordinate
    Xb = np.random.default_rng(5).standard_normal((5000, d))
    Eb = O.encode_polar(Xb, P, qjl=False)
    nm = np.mean(np.sum((O.rotate(Xb, P.signs) - Eb.yhat) ** 2, 1) / np.sum(Xb ** 2, 1))
    P2 = O.make_params(d, 2, 6, with_S=False)
    E2b = O.encode(Xb, P2, qjl=False, margins=False)
    n2 = np.mean(np.sum((O.rotate(Xb, P2.signs) - E2b.nhat[:, None] * P2.c32.astype(np.float64)[E2b.idx]) ** 2, 1)
                 / np.sum(Xb ** 2, 1))
    assert nm < n2


def test_polar_attention_textbook_and_qjl_unbiased():
    d, L = 64, 120
    rng = np.random.default_rng(8)
    Pk, Pv = O.polar_params(d, 61, with_S=False), O.polar_params(d, 62, with_S=False)

    def coded(P):
        c1 = rng.integers(0, 16, (L, d // 2)).astype(np.uint8)
        ch = rng.integers(0, 4, (L, d // 2 - 1)).astype(np.uint8)
        nh = np.array([O.round_fp16(v) for v in rng.uniform(1.0, 9.0, L)])
        yh = O.polar_decode(c1, ch, nh, P)
        return O.PolarEncoded(False, c1, ch, nh, yh), O.rotate_t(yh, P.signs)
    Ek, Kx = coded(Pk)
    Ev, Vx = coded(Pv)
    Q = rng.standard_normal((3, d))
    out, lse, logits = O.attend(Q, Pk, Ek, Pv, Ev, want_logits=True)
    lg = Q @ Kx.T / math.sqrt(d)
    assert np.allclose(logits, lg, atol=1e-11, rtol=0)
    assert np.allclose(out, scipy.special.softmax(lg, axis=1) @ Vx, atol=1e-11, rtol=0)
    # QJL on the polar residual keeps inner products unbiased
    k = rng.standard_normal(d)
    q = rng.standard_normal(d) + 0.6 * k
    est = np.array([O.estimate(q, P, O.encode_polar(k[None, :], P, qjl=True))[0]
                    for P in (O.polar_params(d, 4000 + s) for s in range(3000))])
    assert abs(est.mean() - q @ k) < 3 * est.std(ddof=1) / math.sqrt(len(est))
