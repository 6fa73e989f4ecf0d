"""Python face of the float64 CPU oracle (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It never imports the product package and
the product package never imports it.  The arithmetic lives in
``tq_oracle.c`` (plain float64 loops, OpenMP over independent vectors and
queries); this file marshals numpy arrays and holds the oracle's own
implementation of the packed cache layout.

Sources, by page title and section:
  * "What is TurboQuant? mechanism, measured accuracy, status as of July 2026",
    sections on stage 1 (randomized Hadamard + per-coordinate Lloyd-Max),
    stage 2 (1-bit QJL residual, unbiased inner products) and the vLLM
    presets (k8v4 = FP8 keys + 4-bit values; 4-bit and 3-bit presets).
  * "TurboQuant and RotorQuant on DGX Spark", "Two-stage compression":
    rotation, no per-block scales (one norm per vector), 1-bit QJL correction.
  * "TurboQuant" overview (ai-work-lab.com), "QJL": +1/-1 sign bits; the same
    codec serves vector search.

The pages print no bit layout; the oracle implements the layout stated in the
design notes (packed little-endian code fields, sign-magnitude code order,
fp16 norms, structure-of-arrays pages of ``page_tokens`` tokens).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (float64, -O2, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    u64, i32, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p
    lib.orc_draw.restype = u64
    lib.orc_draw.argtypes = [u64, u64, u64]
    lib.orc_round_fp16.restype = ctypes.c_double
    lib.orc_round_fp16.argtypes = [ctypes.c_double]
    lib.orc_round_bf16.restype = ctypes.c_double
    lib.orc_round_bf16.argtypes = [ctypes.c_double]
    lib.orc_e4m3.restype = ctypes.c_uint8
    lib.orc_e4m3.argtypes = [ctypes.c_double]
    lib.orc_e4m3_value.restype = ctypes.c_double
    lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.orc_signs.argtypes = [i32, u64, vp]
    lib.orc_gauss_bf16.argtypes = [i32, i32, u64, vp]
    lib.orc_codebook.restype = i32
    lib.orc_codebook.argtypes = [i32, i32, vp, vp, vp]
    lib.orc_rotate.argtypes = [i32, vp, vp, vp, vp]
    lib.orc_rotate_t.argtypes = [i32, vp, vp, vp, vp]
    lib.orc_dense_rotation.argtypes = [i32, u64, vp, vp, vp]
    lib.orc_encode.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                               i32, vp, vp]
    lib.orc_encode_fp8.argtypes = [i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.orc_estimate.argtypes = [vp, i32, vp, vp]
    lib.orc_attend.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.orc_polar_codebook.restype = i32
    lib.orc_polar_codebook.argtypes = [i32, i32, vp, vp, vp]
    lib.orc_polar_decode.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.orc_encode_polar.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                     vp, vp, vp, vp, vp, vp]
    lib.orc_attend_exact.argtypes = [i32, i32, i32, vp, vp, vp, vp]
    lib.orc_search.argtypes = [i32, i32, i32, vp, vp, vp, vp]
    _lib = lib
    return lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------------------
# scalar helpers
# ---------------------------------------------------------------------------
def draw(seed: int, stream: int, i: int) -> int:
    """SplitMix64 output number stream*2^32 + i of the generator seeded with seed."""
    return int(_load().orc_draw(seed, stream, i))


def round_fp16(v: float) -> float:
    return float(_load().orc_round_fp16(float(v)))


def round_bf16(v: float) -> float:
    return float(_load().orc_round_bf16(float(v)))


def e4m3(v: float) -> int:
    return int(_load().orc_e4m3(float(v)))


def e4m3_value(code: int) -> float:
    return float(_load().orc_e4m3_value(int(code)))


# ---------------------------------------------------------------------------
# parameters
# ---------------------------------------------------------------------------
@dataclass
class Params:
    """Data-independent codec parameters for (d, bits, seed)."""
    d: int
    bits: int
    seed: int
    signs: np.ndarray            # int8 [d], +1/-1
    S: np.ndarray | None         # float32 [m, d] (bf16-exact), m = d
    c64: np.ndarray | None       # float64 levels (Lloyd-Max only)
    c32: np.ndarray | None       # float32 levels
    t32: np.ndarray | None       # float32 boundaries
    iters: int = 0
    Rm: np.ndarray | None = None  # dense rotation [d, d] (None: H D / sqrt(d))
    # fractional rates (bits = b + 1/2): coordinates d/2 .. d-1 use b bits
    # (bits2 = b) with their own codebook; coordinates 0 .. d/2-1 use b + 1
    bits2: int = 0
    c32b: np.ndarray | None = None
    t32b: np.ndarray | None = None
    c64b: np.ndarray | None = None

    @property
    def rate(self):
        """Bits per coordinate: bits, or bits - 1/2 for a fractional rate."""
        return self.bits - 0.5 if self.bits2 else self.bits


def make_params(d: int, bits: int, seed: int, with_S: bool = True, rotation: str = "hadamard") -> Params:
    """Signs, Gaussian S (m = d, bf16-exact) and, for bits in 1..4, the
    Lloyd-Max codebook of the coordinate law of a random unit vector in R^d.
    bits = 8 denotes FP8 (E4M3) codes and has no codebook.  rotation =
    "dense" replaces H D / sqrt(d) by the dense random rotation."""
    lib = _load()
    signs = np.zeros(d, np.int8)
    lib.orc_signs(d, seed, _p(signs))
    S = None
    if with_S:
        S = np.zeros((d, d), np.float32)
        lib.orc_gauss_bf16(d, d, seed, _p(S))
    c64 = c32 = t32 = None
    iters = 0
    bits2, cb = 0, (None, None, None)
    if bits in (1.5, 2.5, 3.5):
        bits2 = int(bits - 0.5)
        bits = bits2 + 1
        cb = codebook(d, bits2)
    if bits in (1, 2, 3, 4):
        c64, c32, t32 = codebook(d, bits)
    elif bits != 8:
        raise ValueError("bits must be 1..4, 8 or 1.5, 2.5, 3.5")
    Rm = None
    if rotation == "dense":
        Rm = dense_rotation(d, seed)[2]
    elif rotation != "hadamard":
        raise ValueError("rotation must be 'hadamard' or 'dense'")
    return Params(d, bits, seed, signs, S, c64, c32, t32, iters, Rm, bits2, cb[1], cb[2], cb[0])


def dense_rotation(d: int, seed: int):
    """(G, Q, Rm): the Gaussian matrix, its row-orthonormalised float64 form
    and the stored rotation (Q rounded to float32)."""
    G = np.zeros((d, d), np.float64)
    Q = np.zeros((d, d), np.float64)
    Rm = np.zeros((d, d), np.float64)
    _load().orc_dense_rotation(d, seed, _p(G), _p(Q), _p(Rm))
    return G, Q, Rm


_codebook_cache: dict = {}


def codebook(d: int, bits: int):
    """(c64, c32, t32) for (d, bits); cached since it does not depend on seed."""
    key = (d, bits)
    if key not in _codebook_cache:
        lib = _load()
        L = 1 << bits
        c64 = np.zeros(L, np.float64)
        c32 = np.zeros(L, np.float32)
        t32 = np.zeros(L - 1, np.float32)
        it = lib.orc_codebook(d, bits, _p(c64), _p(c32), _p(t32))
        if it < 0:
            raise RuntimeError("Lloyd-Max iteration did not converge")
        _codebook_cache[key] = (c64, c32, t32)
    return _codebook_cache[key]


def rotate(x: np.ndarray, signs: np.ndarray, Rm: np.ndarray | None = None) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    out = np.zeros_like(flat)
    lib = _load()
    Rm = None if Rm is None else np.ascontiguousarray(Rm, np.float64)
    for r in range(flat.shape[0]):
        lib.orc_rotate(d, _p(signs), _p(Rm), _p(flat[r]), _p(out[r]))
    return out.reshape(x.shape)


def rotate_t(y: np.ndarray, signs: np.ndarray, Rm: np.ndarray | None = None) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float64)
    d = y.shape[-1]
    flat = y.reshape(-1, d)
    out = np.zeros_like(flat)
    lib = _load()
    Rm = None if Rm is None else np.ascontiguousarray(Rm, np.float64)
    for r in range(flat.shape[0]):
        lib.orc_rotate_t(d, _p(signs), _p(Rm), _p(flat[r]), _p(out[r]))
    return out.reshape(y.shape)


# ---------------------------------------------------------------------------
# encode
# ---------------------------------------------------------------------------
@dataclass
class Encoded:
    """Oracle encoding of n vectors.  idx: bucket indices (Lloyd-Max) or E4M3
    codes (FP8).  nhat / rho hold fp16-exact values as float64."""
    bits: int
    qjl: bool
    idx: np.ndarray
    nhat: np.ndarray
    rho: np.ndarray | None = None
    sbits: np.ndarray | None = None
    umargin: np.ndarray | None = None
    zmargin: np.ndarray | None = None
    nraw: np.ndarray | None = None      # unrounded ||x||
    rraw: np.ndarray | None = None      # unrounded ||r||


def encode(X: np.ndarray, P: Params, qjl: bool, margins: bool = True) -> Encoded:
    X = np.ascontiguousarray(X, np.float64)
    n, d = X.shape
    assert d == P.d
    lib = _load()
    if P.bits == 8:
        code = np.zeros((n, d), np.uint8)
        nhat = np.zeros(n, np.float64)
        mg = np.zeros((n, d), np.float64) if margins else None
        nraw = np.zeros(n, np.float64)
        lib.orc_encode_fp8(n, d, _p(X), _p(P.signs), _p(P.Rm), _p(code), _p(nhat), _p(mg), _p(nraw))
        return Encoded(8, False, code, nhat, umargin=mg, nraw=nraw)
    idx = np.zeros((n, d), np.uint8)
    nhat = np.zeros(n, np.float64)
    rho = np.zeros(n, np.float64) if qjl else None
    sb = np.zeros((n, d), np.uint8) if qjl else None
    um = np.zeros((n, d), np.float64) if margins else None
    zm = np.zeros((n, d), np.float64) if (margins and qjl) else None
    if qjl:
        assert P.S is not None
    nraw = np.zeros(n, np.float64)
    rraw = np.zeros(n, np.float64) if qjl else None
    lib.orc_encode(n, d, P.bits, 1 if qjl else 0, _p(X), _p(P.signs), _p(P.Rm), _p(P.S), _p(P.c32),
                   _p(P.t32), _p(idx), _p(nhat), _p(rho), _p(sb), _p(um), _p(zm), _p(nraw), _p(rraw),
                   P.bits2, _p(P.c32b), _p(P.t32b))
    return Encoded(P.rate, qjl, idx, nhat, rho, sb, um, zm, nraw, rraw)


# ---------------------------------------------------------------------------
# PolarQuant: the polar-coordinate angle quantizer
# ---------------------------------------------------------------------------
@dataclass
class PolarParams:
    """Parameters of the polar quantizer: the rotation (signs / dense Rm), S
    for QJL, level-1 angle codebook (b1 bits, uniform cells on [0, 2 pi)) and
    one Lloyd-Max codebook of bh bits per level l = 2 .. log2 d."""
    d: int
    b1: int
    bh: int
    seed: int
    signs: np.ndarray
    S: np.ndarray | None
    c1: np.ndarray          # float32 [2^b1] level-1 centroids
    t1: np.ndarray          # float32 [2^b1 - 1] boundaries (midpoints of the fp32 centroids)
    ch: np.ndarray          # float32 [log2 d - 1][2^bh]
    th: np.ndarray          # float32 [log2 d - 1][2^bh - 1]
    ch64: np.ndarray        # float64 levels
    Rm: np.ndarray | None = None
    bits: str = "polar"


def polar_params(d: int, seed: int, b1: int = 4, bh: int = 2, with_S: bool = True,
                 rotation: str = "hadamard") -> PolarParams:
    base = make_params(d, 8, seed, with_S=with_S, rotation=rotation)
    L1 = 1 << b1
    c1_64 = (np.arange(L1) + 0.5) * (2.0 * np.pi / L1)      # the uniform law's Lloyd-Max levels: cell centres
    c1 = c1_64.astype(np.float32)
    t1 = ((c1[:-1].astype(np.float64) + c1[1:]) / 2).astype(np.float32)
    levels = int(np.log2(d))
    H = 1 << bh
    ch = np.zeros((levels - 1, H), np.float32)
    th = np.zeros((levels - 1, H - 1), np.float32)
    ch64 = np.zeros((levels - 1, H), np.float64)
    for l in range(2, levels + 1):
        c64, c32, t32 = polar_codebook(1 << (l - 1), bh)
        ch64[l - 2], ch[l - 2], th[l - 2] = c64, c32, t32
    return PolarParams(d, b1, bh, seed, base.signs, base.S, c1, t1, ch, th, ch64, base.Rm)


_polar_cache: dict = {}


def polar_codebook(k: int, bits: int):
    """(c64, c32, t32) of the level angle for sub-block dimension k."""
    if (k, bits) not in _polar_cache:
        L = 1 << bits
        c64, c32, t32 = np.zeros(L), np.zeros(L, np.float32), np.zeros(L - 1, np.float32)
        if _load().orc_polar_codebook(k, bits, _p(c64), _p(c32), _p(t32)) < 0:
            raise RuntimeError("polar Lloyd-Max iteration did not converge")
        _polar_cache[(k, bits)] = (c64, c32, t32)
    return _polar_cache[(k, bits)]


@dataclass
class PolarEncoded:
    qjl: bool
    codes1: np.ndarray      # uint8 [n, d/2] level-1 angle codes
    codesh: np.ndarray      # uint8 [n, d/2 - 1] higher-level codes (level 2 first)
    nhat: np.ndarray
    yhat: np.ndarray        # float64 [n, d] reconstruction in the rotated basis
    rho: np.ndarray | None = None
    sbits: np.ndarray | None = None
    margin1: np.ndarray | None = None
    marginh: np.ndarray | None = None
    zmargin: np.ndarray | None = None
    nraw: np.ndarray | None = None
    rraw: np.ndarray | None = None
    bits: str = "polar"


def encode_polar(X: np.ndarray, P: PolarParams, qjl: bool) -> PolarEncoded:
    X = np.ascontiguousarray(X, np.float64)
    n, d = X.shape
    h = d // 2
    c1, cd = np.zeros((n, h), np.uint8), np.zeros((n, h - 1), np.uint8)
    nhat, yhat, nraw = np.zeros(n), np.zeros((n, d)), np.zeros(n)
    m1, mh = np.zeros((n, h)), np.zeros((n, h - 1))
    rho = np.zeros(n) if qjl else None
    sb = np.zeros((n, d), np.uint8) if qjl else None
    zm = np.zeros((n, d)) if qjl else None
    rr = np.zeros(n) if qjl else None
    _load().orc_encode_polar(n, d, P.b1, P.bh, 1 if qjl else 0, _p(X), _p(P.signs), _p(P.Rm), _p(P.S), _p(P.c1),
                             _p(P.t1), _p(np.ascontiguousarray(P.ch)), _p(np.ascontiguousarray(P.th)), _p(c1), _p(cd),
                             _p(nhat), _p(yhat), _p(rho), _p(sb), _p(m1), _p(mh), _p(zm), _p(nraw), _p(rr))
    return PolarEncoded(qjl, c1, cd, nhat, yhat, rho, sb, m1, mh, zm, nraw, rr)


def polar_decode(codes1: np.ndarray, codesh: np.ndarray, nhat: np.ndarray, P: PolarParams) -> np.ndarray:
    n, h = codes1.shape
    d = 2 * h
    yhat = np.zeros((n, d))
    _load().orc_polar_decode(n, d, P.b1, P.bh, _p(np.ascontiguousarray(codes1, np.uint8)),
                             _p(np.ascontiguousarray(codesh, np.uint8)), _p(np.ascontiguousarray(nhat, np.float64)),
                             _p(P.c1), _p(np.ascontiguousarray(P.ch)), _p(yhat))
    return yhat


# ---------------------------------------------------------------------------
# estimator, attention, search
# ---------------------------------------------------------------------------
class _Keys(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("qjl", ctypes.c_int), ("d", ctypes.c_int),
                ("signs", ctypes.c_void_p), ("S", ctypes.c_void_p), ("c32", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("fp8", ctypes.c_void_p), ("nhat", ctypes.c_void_p),
                ("rho", ctypes.c_void_p), ("sbits", ctypes.c_void_p), ("Rm", ctypes.c_void_p),
                ("c32b", ctypes.c_void_p), ("yhat", ctypes.c_void_p)]


def _keys(P, E, keep: list) -> _Keys:
    if isinstance(E, PolarEncoded):
        arrs = [np.ascontiguousarray(a) if a is not None else None
                for a in (P.signs, P.S, E.nhat, E.rho, E.sbits, P.Rm, E.yhat)]
        keep.extend(arrs)
        signs, S, nhat, rho, sb, Rm, yh = arrs
        k = _Keys()
        k.kind, k.qjl, k.d = 2, 1 if E.qjl else 0, P.d
        k.signs, k.S, k.nhat, k.rho, k.sbits, k.Rm, k.yhat = (_p(a) for a in (signs, S, nhat, rho, sb, Rm, yh))
        return k
    arrs = [np.ascontiguousarray(a) if a is not None else None
            for a in (P.signs, P.S, P.c32, E.idx, E.nhat, E.rho, E.sbits, P.Rm, P.c32b)]
    keep.extend(arrs)
    signs, S, c32, idx, nhat, rho, sb, Rm, c32b = arrs
    k = _Keys()
    k.kind = 1 if E.bits == 8 else 0
    k.qjl = 1 if E.qjl else 0
    k.d = P.d
    k.signs = _p(signs)
    k.S = _p(S)
    k.c32 = _p(c32)
    k.idx = _p(idx) if E.bits != 8 else None
    k.fp8 = _p(idx) if E.bits == 8 else None
    k.nhat = _p(nhat)
    k.rho = _p(rho)
    k.sbits = _p(sb)
    k.Rm = _p(Rm)
    k.c32b = _p(c32b)
    return k


def estimate(q: np.ndarray, Pk: Params, Ek: Encoded) -> np.ndarray:
    """Estimates of <q, k_t> for every encoded key t (float64)."""
    keep: list = []
    K = _keys(Pk, Ek, keep)
    q = np.ascontiguousarray(q, np.float64)
    L = Ek.nhat.shape[0]
    est = np.zeros(L, np.float64)
    _load().orc_estimate(ctypes.byref(K), L, _p(q), _p(est))
    return est


def attend(Q: np.ndarray, Pk: Params, Ek: Encoded, Pv: Params, Ev: Encoded,
           nvis: np.ndarray | None = None, want_logits: bool = False):
    """Softmax attention of queries Q [nq, d] over one compressed sequence.
    Returns (out [nq, d], lse [nq], logits [nq, L] or None)."""
    keep: list = []
    K = _keys(Pk, Ek, keep)
    Q = np.ascontiguousarray(Q, np.float64)
    nq, d = Q.shape
    L = Ek.nhat.shape[0]
    out = np.zeros((nq, d), np.float64)
    lse = np.zeros(nq, np.float64)
    logits = np.zeros((nq, L), np.float64) if want_logits else None
    nv = None if nvis is None else np.ascontiguousarray(nvis, np.int32)
    vR = None if Pv.Rm is None else np.ascontiguousarray(Pv.Rm)
    if isinstance(Ev, PolarEncoded):
        vs, vn, vy = (np.ascontiguousarray(a) for a in (Pv.signs, Ev.nhat, Ev.yhat))
        _load().orc_attend(nq, L, d, _p(Q), _p(nv), ctypes.byref(K), _p(vs), _p(vR), None, None, _p(vy), None,
                           _p(vn), _p(logits), _p(out), _p(lse))
        return out, lse, logits
    vs, vc, vi, vn = (np.ascontiguousarray(a) for a in (Pv.signs, Pv.c32, Ev.idx, Ev.nhat))
    vcb = None if Pv.c32b is None else np.ascontiguousarray(Pv.c32b)
    _load().orc_attend(nq, L, d, _p(Q), _p(nv), ctypes.byref(K), _p(vs), _p(vR), _p(vc), _p(vcb), None, _p(vi),
                       _p(vn), _p(logits), _p(out), _p(lse))
    return out, lse, logits


def attend_exact(Q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    Q, K, V = (np.ascontiguousarray(a, np.float64) for a in (Q, K, V))
    nq, d = Q.shape
    out = np.zeros((nq, d), np.float64)
    _load().orc_attend_exact(nq, K.shape[0], d, _p(Q), _p(K), _p(V), _p(out))
    return out


def search(Q: np.ndarray, P: Params, E: Encoded, k: int):
    """Top-k estimated inner products per query; ties towards lower index."""
    keep: list = []
    K = _keys(P, E, keep)
    Q = np.ascontiguousarray(Q, np.float64)
    nq = Q.shape[0]
    sc = np.zeros((nq, k), np.float64)
    ix = np.zeros((nq, k), np.int64)
    _load().orc_search(nq, E.nhat.shape[0], k, _p(Q), ctypes.byref(K), _p(sc), _p(ix))
    return sc, ix


# ---------------------------------------------------------------------------
# packed page layout (the oracle's own implementation of the stated layout)
# ---------------------------------------------------------------------------
@dataclass
class Layout:
    """Structure-of-arrays page of ``page_tokens`` tokens of one KV head.

    kbits: 1..4 Lloyd-Max bits, 1.5 / 2.5 / 3.5 (fractional rates) or 8 for
    FP8 keys; kqjl: QJL sign bits + rho;
    vbits: 1..4, or 0 for no value fields (a search database).  Fields in order, each padded to 16 bytes:
      K codes  ("kc" for w in {1,2,4}; "kc_lo" (2-bit) + "kc_hi" (1-bit) for 3
               bits; "k8" bytes for FP8), "ks" QJL sign bits, "kn" fp16 norm,
      "kr" fp16 residual norm, V codes ("vc" or "vc_lo" + "vc_hi"), "vn".
    """
    d: int
    kbits: int
    kqjl: bool
    vbits: int
    page_tokens: int = 64
    fields: dict = field(default_factory=dict)
    page_bytes: int = 0

    def __post_init__(self):
        P, d = self.page_tokens, self.d
        off = 0

        def add(name, bytes_per_token):
            nonlocal off
            self.fields[name] = (off, bytes_per_token)
            off += -(-(P * bytes_per_token) // 16) * 16

        def codes(prefix, bits, n=d):
            if bits == "polar":
                # level-1 angles: 4-bit fields, d/2 of them; higher levels: 2-bit, d/2 slots (last unused)
                add(prefix[0] + "p1", d // 2 * 4 // 8)
                add(prefix[0] + "ph", d // 2 * 2 // 8)
            elif bits == 8:
                add(prefix[0] + "8", n)
            elif bits != int(bits):
                # fractional rate b + 1/2: coordinates 0 .. d/2-1 with b + 1 bits, then d/2 .. d-1 with b
                codes(prefix + "A", int(bits + 0.5), d // 2)
                codes(prefix + "B", int(bits - 0.5), d // 2)
            elif bits == 3:
                add(prefix + "_lo", n * 2 // 8)
                add(prefix + "_hi", n // 8)
            else:
                add(prefix, n * int(bits) // 8)

        codes("kc", self.kbits)
        if self.kqjl:
            add("ks", d // 8)
        add("kn", 2)
        if self.kqjl:
            add("kr", 2)
        if self.vbits == "polar" or self.vbits > 0:
            codes("vc", self.vbits)
            add("vn", 2)
        self.page_bytes = off


def to_kappa(idx: np.ndarray, bits: int) -> np.ndarray:
    """Sign-magnitude storage code of a bucket index: top bit set for the
    negative half, low bits the rank of |c[idx]| (0 = smallest magnitude)."""
    half = 1 << (bits - 1)
    idx = idx.astype(np.int64)
    neg = idx < half
    mag = np.where(neg, half - 1 - idx, idx - half)
    return ((neg.astype(np.int64) << (bits - 1)) | mag).astype(np.uint8)


def from_kappa(kap: np.ndarray, bits: int) -> np.ndarray:
    half = 1 << (bits - 1)
    kap = kap.astype(np.int64)
    neg = (kap >> (bits - 1)) & 1
    mag = kap & (half - 1)
    return np.where(neg == 1, half - 1 - mag, half + mag).astype(np.uint8)


def pack_fields(vals: np.ndarray, w: int) -> np.ndarray:
    """[n, d] values of w bits -> [n, d*w/8] bytes; value i at bit offset i*w
    of the little-endian byte string."""
    n, d = vals.shape
    out = np.zeros((n, d * w // 8), np.uint8)
    for i in range(d):
        for b in range(w):
            bit = i * w + b
            out[:, bit // 8] |= (((vals[:, i].astype(np.uint16) >> b) & 1) << (bit % 8)).astype(np.uint8)
    return out


def unpack_fields(packed: np.ndarray, d: int, w: int) -> np.ndarray:
    n = packed.shape[0]
    out = np.zeros((n, d), np.uint8)
    for i in range(d):
        for b in range(w):
            bit = i * w + b
            out[:, i] |= (((packed[:, bit // 8] >> (bit % 8)) & 1) << b).astype(np.uint8)
    return out


def _fp16_bytes(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, np.float64).astype(np.float16).view(np.uint8).reshape(-1, 2)


def _code_arrays(prefix: str, bits, codes) -> dict:
    if bits == "polar":
        E = codes
        ph = np.zeros((E.codesh.shape[0], E.codesh.shape[1] + 1), np.uint8)
        ph[:, :-1] = E.codesh
        return {prefix[0] + "p1": pack_fields(E.codes1, 4), prefix[0] + "ph": pack_fields(ph, 2)}
    if bits == 8:
        return {prefix[0] + "8": codes.astype(np.uint8)}
    if bits != int(bits):
        h = codes.shape[1] // 2
        out = _code_arrays(prefix + "A", int(bits + 0.5), codes[:, :h])
        out.update(_code_arrays(prefix + "B", int(bits - 0.5), codes[:, h:]))
        return out
    bits = int(bits)
    kap = to_kappa(codes, bits)
    if bits == 3:
        return {prefix + "_lo": pack_fields(kap & 3, 2), prefix + "_hi": pack_fields(kap >> 2, 1)}
    return {prefix: pack_fields(kap, bits)}


def token_records(lay: Layout, Ek: Encoded, Ev: Encoded) -> dict:
    """Per-token bytes of every field (name -> [n, bytes_per_token])."""
    rec = {}
    rec.update(_code_arrays("kc", lay.kbits, Ek if lay.kbits == "polar" else Ek.idx))
    if lay.kqjl:
        rec["ks"] = pack_fields(Ek.sbits, 1)
    rec["kn"] = _fp16_bytes(Ek.nhat)
    if lay.kqjl:
        rec["kr"] = _fp16_bytes(Ek.rho)
    if lay.vbits == "polar" or lay.vbits > 0:
        rec.update(_code_arrays("vc", lay.vbits, Ev if lay.vbits == "polar" else Ev.idx))
        rec["vn"] = _fp16_bytes(Ev.nhat)
    return rec


def _field_index(lay: Layout, slots: np.ndarray, head: int, n_heads: int, off: int, bpt: int):
    """(page rows, byte columns) of one field for each slot."""
    P = lay.page_tokens
    s = np.asarray(slots, np.int64)
    page = (s // P) * n_heads + head
    cols = off + (s % P)[:, None] * bpt + np.arange(bpt)[None, :]
    return page[:, None], cols


def write_cache(lay: Layout, cache: np.ndarray, slots: np.ndarray, head: int, n_heads: int,
                Ek: Encoded, Ev: Encoded) -> None:
    """Store the records of tokens with the given slots for one KV head into a
    cache array viewed as [num_blocks * n_heads, page_bytes] bytes."""
    rec = token_records(lay, Ek, Ev)
    for name, (off, bpt) in lay.fields.items():
        r, c = _field_index(lay, slots, head, n_heads, off, bpt)
        cache[r, c] = rec[name]


def read_cache(lay: Layout, cache: np.ndarray, slots: np.ndarray, head: int, n_heads: int) -> dict:
    """Decode the stored fields of the given slots of one KV head back into
    bucket indices / codes, sign bits and float64 norms."""
    d = lay.d
    raw = {}
    for name, (off, bpt) in lay.fields.items():
        r, c = _field_index(lay, slots, head, n_heads, off, bpt)
        raw[name] = np.ascontiguousarray(cache[r, c])

    def codes(prefix, bits, n=d):
        if bits == "polar":
            return (unpack_fields(raw[prefix[0] + "p1"], d // 2, 4),
                    unpack_fields(raw[prefix[0] + "ph"], d // 2, 2)[:, :-1].copy())
        if bits == 8:
            return raw[prefix[0] + "8"].copy()
        if bits != int(bits):
            return np.concatenate([codes(prefix + "A", int(bits + 0.5), d // 2),
                                   codes(prefix + "B", int(bits - 0.5), d // 2)], axis=1)
        bits = int(bits)
        if bits == 3:
            kap = unpack_fields(raw[prefix + "_lo"], n, 2) | (unpack_fields(raw[prefix + "_hi"], n, 1) << 2)
        else:
            kap = unpack_fields(raw[prefix], n, bits)
        return from_kappa(kap, bits)

    out = {"kidx": codes("kc", lay.kbits),
           "kn": raw["kn"].copy().view(np.float16).reshape(-1).astype(np.float64)}
    if lay.vbits == "polar" or lay.vbits > 0:
        out["vidx"] = codes("vc", lay.vbits)
        out["vn"] = raw["vn"].copy().view(np.float16).reshape(-1).astype(np.float64)
    if lay.kqjl:
        out["ks"] = unpack_fields(raw["ks"], d, 1)
        out["kr"] = raw["kr"].copy().view(np.float16).reshape(-1).astype(np.float64)
    return out
