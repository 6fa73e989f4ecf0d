"""Comparison rules between the CUDA path and the float64 oracle.

Codes and sign bits must match bit for bit, except:
  * a code whose oracle coordinate u_i lies within 1e-6 (unit-vector units)
    of a decision boundary (or an E4M3 rounding midpoint) - then the GPU code
    may be either neighbour;
  * a QJL sign whose |(S r)_j| / (||r|| ||S_j||) < 1e-6, and every sign of a
    vector with an exempt code or norm (its residual legitimately differs).
Norms (fp16) must be equal, or one fp16 ulp apart when the oracle's unrounded
value lies within 1e-5 relative of the rounding midpoint between them (the
GPU rounds from fp32); such a key's logits are exempt too.  Logits: |d| <= 1e-3 * max(|l_oracle|, rms of the
row's logits), on keys without exemptions.  Outputs (bf16): |d| <= 2e-3 +
half a bf16 ulp of the oracle value (the output rounding itself), plus, per
row, the most that exempt keys can move it (exempt_slack).
"""
from __future__ import annotations

import numpy as np

from oracle import oracle as O

CODE_MARGIN = 1e-6
SIGN_MARGIN = 1e-6
NORM_TIE_REL = 1e-5
LOGIT_REL = 1e-3
OUT_ABS = 2e-3


def fp16_match(gpu: np.ndarray, orc: np.ndarray, raw: np.ndarray):
    """(ok mask, tie mask) for fp16-valued norms."""
    g = np.asarray(gpu, np.float64)
    o = np.asarray(orc, np.float64)
    eq = g == o
    gb = g.astype(np.float16).view(np.int16).astype(np.int64)
    ob = o.astype(np.float16).view(np.int16).astype(np.int64)
    adj = (np.abs(gb - ob) == 1) & (np.sign(g) == np.sign(o))
    mid = 0.5 * (g + o)
    tie = (~eq) & adj & (np.abs(np.asarray(raw) - mid) <= NORM_TIE_REL * np.abs(raw))
    return eq | tie, tie


def compare_vectors(gpu: dict, Ek: O.Encoded, key: bool, bits: int):
    """Compare one head's decoded GPU fields with the oracle encoding.

    Returns (report dict, exempt_vector mask).  Raises AssertionError on a
    mismatch outside the exemptions."""
    rep = {}
    codes = gpu["kidx"] if key else gpu["vidx"]
    norms = gpu["kn"] if key else gpu["vn"]
    diff = codes != Ek.idx
    margin_ok = Ek.umargin < CODE_MARGIN
    bad = diff & ~margin_ok
    rep["code_exempt"] = int((diff & margin_ok).sum())
    assert not bad.any(), f"{int(bad.sum())} codes differ outside the boundary exemption " \
                          f"(first at {np.argwhere(bad)[0].tolist()})"
    if bits != 8:
        # an exempt code may only move to the neighbouring bucket
        assert np.all(np.abs(codes[diff].astype(int) - Ek.idx[diff].astype(int)) == 1)
    ok, tie = fp16_match(norms, Ek.nhat, Ek.nraw)
    assert ok.all(), f"{int((~ok).sum())} norms differ (first {np.argwhere(~ok)[0].tolist()})"
    rep["norm_tie"] = int(tie.sum())
    vec_exempt = diff.any(1) | tie
    if key and Ek.qjl:
        ok, rtie = fp16_match(gpu["kr"], Ek.rho, Ek.rraw)
        bad_r = ~ok & ~vec_exempt
        assert not bad_r.any(), f"{int(bad_r.sum())} residual norms differ"
        rep["rho_tie"] = int(rtie.sum())
        sdiff = gpu["ks"] != Ek.sbits
        sex = (Ek.zmargin < SIGN_MARGIN) | vec_exempt[:, None]
        bad_s = sdiff & ~sex
        rep["sign_exempt"] = int((sdiff & sex).sum())
        assert not bad_s.any(), f"{int(bad_s.sum())} QJL sign bits differ outside the exemption " \
                                f"(first {np.argwhere(bad_s)[0].tolist()})"
        # a residual norm rounded one ulp apart (a tie) changes that key's logit
        vec_exempt = vec_exempt | sdiff.any(1) | ~ok | rtie
    rep["vectors_exempt"] = int(vec_exempt.sum())
    return rep, vec_exempt


def check_logits(gpu: np.ndarray, orc: np.ndarray, exempt_keys: np.ndarray | None = None):
    """gpu, orc: [rows, L] over the visible keys."""
    rms = np.sqrt(np.mean(orc ** 2, axis=1, keepdims=True))
    tol = LOGIT_REL * np.maximum(np.abs(orc), rms)
    err = np.abs(gpu.astype(np.float64) - orc)
    bad = err > tol
    if exempt_keys is not None:
        bad &= ~exempt_keys[None, :]
    if bad.any():
        ratio = np.where(bad, err / np.maximum(tol, 1e-30), 0.0)
        order = np.argsort(ratio, axis=None)[::-1][:8]
        where = np.stack(np.unravel_index(order, ratio.shape), 1)
        detail = [(int(r), int(t), float(gpu[r, t]), float(orc[r, t]), float(rms[r, 0])) for r, t in where]
        raise AssertionError(f"{int(bad.sum())} logits outside tolerance; worst rel "
                             f"{float(np.max(err / np.maximum(tol, 1e-30)) * LOGIT_REL):.3e}; "
                             f"(row, key, gpu, oracle, rms): {detail}")
    return float(np.max(err / np.maximum(np.maximum(np.abs(orc), rms), 1e-30)))


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(x, np.float64))
    a = np.where(a == 0, 2.0 ** -133, a)
    e = np.floor(np.log2(a))
    return 0.5 * 2.0 ** (np.maximum(e, -126) - 7)


def levels_of(P: O.Params, idx: np.ndarray) -> np.ndarray:
    """Float64 levels of bucket indices [n, d] (fractional rates: the second
    codebook for coordinates d/2 .. d-1)."""
    lv = P.c32.astype(np.float64)[idx]
    if P.bits2:
        h = idx.shape[1] // 2
        lv[:, h:] = P.c32b.astype(np.float64)[idx[:, h:]]
    return lv


def exempt_slack(Pv: O.Params, Ev: O.Encoded, exempt: np.ndarray, logits: np.ndarray, lse: np.ndarray,
                 out: np.ndarray) -> np.ndarray:
    """Per-row bound on how far exempt keys can legitimately move an output.

    A key with an exempt (near-boundary) code, sign or norm is stored
    differently by the two sides, both correctly; its logit and dequantized
    value may differ.  Moving the weight p_t of such a key changes an output
    by at most 2 p_t (|v_t|_inf + |o|_inf), with p_t the oracle's softmax
    weight (exp(logit - lse)) and v_t the oracle's dequantized value."""
    rows = logits.shape[0]
    slack = np.zeros(rows)
    ex = np.flatnonzero(exempt)
    if ex.size == 0:
        return slack
    vhat = O.rotate_t(Ev.nhat[ex, None] * levels_of(Pv, Ev.idx[ex]), Pv.signs, Pv.Rm)
    vmax = np.abs(vhat).max(1)
    for r in range(rows):
        p = np.exp(logits[r, ex] - lse[r])
        p = np.where(np.isfinite(p), p, 0.0)
        slack[r] = 2.0 * np.sum(p * (vmax + np.abs(out[r]).max()))
    return slack


def check_outputs(gpu_bf16: np.ndarray, orc: np.ndarray, slack: np.ndarray | None = None):
    """gpu_bf16, orc: [rows, d]; slack: optional per-row allowance from
    exempt keys (exempt_slack)."""
    err = np.abs(gpu_bf16.astype(np.float64) - orc)
    tol = OUT_ABS + bf16_half_ulp(orc)
    if slack is not None:
        tol = tol + slack[:, None]
    bad = err > tol
    if bad.any():
        where = np.argwhere(bad)[:6]
        detail = [(int(r), int(c), float(gpu_bf16[r, c]), float(orc[r, c]),
                   float(slack[r]) if slack is not None else 0.0) for r, c in where]
        raise AssertionError(f"{int(bad.sum())} outputs outside tolerance; max err {float(err.max()):.3e}; "
                             f"(row, col, gpu, oracle, slack): {detail}")
    return float(err.max())


def compare_polar(gpu: dict, E: O.PolarEncoded, key: bool):
    """Polar codes: level-1 and higher-level angle codes bit-exact except
    where the oracle's angle lies within CODE_MARGIN (unit-vector units) of a
    bound (then either neighbour, and the vector's reconstruction is exempt);
    norms as compare_vectors; QJL signs and rho as compare_vectors.  Returns
    (report, exempt_vector mask)."""
    c1, ch = gpu["kidx"] if key else gpu["vidx"]
    norms = gpu["kn"] if key else gpu["vn"]
    d1, dh = c1 != E.codes1, ch != E.codesh
    bad = (d1 & ~(E.margin1 < CODE_MARGIN)) | np.zeros_like(d1)
    badh = dh & ~(E.marginh < CODE_MARGIN)
    assert not bad.any(), f"{int(bad.sum())} level-1 angle codes differ outside the exemption"
    assert not badh.any(), f"{int(badh.sum())} higher-level angle codes differ outside the exemption"
    ok, tie = fp16_match(norms, E.nhat, E.nraw)
    assert ok.all(), f"{int((~ok).sum())} norms differ"
    vec_exempt = d1.any(1) | dh.any(1) | tie
    rep = {"code_exempt": int(d1.sum() + dh.sum()), "norm_tie": int(tie.sum())}
    if key and E.qjl:
        okr, rtie = fp16_match(gpu["kr"], E.rho, E.rraw)
        assert not (~okr & ~vec_exempt).any(), "residual norms differ"
        sdiff = gpu["ks"] != E.sbits
        sex = (E.zmargin < SIGN_MARGIN) | vec_exempt[:, None]
        assert not (sdiff & ~sex).any(), f"{int((sdiff & ~sex).sum())} QJL sign bits differ outside the exemption"
        vec_exempt = vec_exempt | sdiff.any(1) | ~okr | rtie
    rep["vectors_exempt"] = int(vec_exempt.sum())
    return rep, vec_exempt


def exempt_slack_polar(Pv, Ev: O.PolarEncoded, exempt: np.ndarray, logits: np.ndarray, lse: np.ndarray,
                       out: np.ndarray) -> np.ndarray:
    """exempt_slack for polar-coded values (reconstruction y_hat)."""
    slack = np.zeros(logits.shape[0])
    ex = np.flatnonzero(exempt)
    if ex.size == 0:
        return slack
    vmax = np.abs(O.rotate_t(Ev.yhat[ex], Pv.signs, Pv.Rm)).max(1)
    for r in range(logits.shape[0]):
        p = np.exp(logits[r, ex] - lse[r])
        p = np.where(np.isfinite(p), p, 0.0)
        slack[r] = 2.0 * np.sum(p * (vmax + np.abs(out[r]).max()))
    return slack

