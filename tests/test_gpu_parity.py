"""CUDA path vs the float64 oracle, through the C ABI, on seeded inputs.

Small cases compare every output; the full-size workloads (the 8B-layer
write path, the GQA decode over 32 x 32K tokens, the 262K-token decode and
2,048-query prefill, the 1M x 1024 search) compare sampled rows the oracle
recomputes one by one.  Exemptions and tolerances are in parity.py.
"""
import math

import numpy as np
import pytest
import torch

import parity
from kv_cache_vector_07_b200 import synth, tqkv
from oracle import oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
class Codec:
    """Library and oracle parameters for one cache configuration."""

    def __init__(self, d, kbits, kqjl, vbits, seed, page_tokens=64, H=1, dense=False):
        # fractional rates: TQ_BITS_HALF | b; "polar": the polar angle codes
        lib = lambda b: tqkv.TQ_BITS_POLAR if b == "polar" else (tqkv.half_bits(b) if b != int(b) else int(b))
        self.desc = tqkv.cache_desc(d, lib(kbits), kqjl, lib(vbits), page_tokens=page_tokens, n_kv_heads=H)
        self.lay = O.Layout(d, kbits, kqjl, vbits, page_tokens=page_tokens)
        rot, orot = (tqkv.TQ_ROT_DENSE, "dense") if dense else (tqkv.TQ_ROT_HADAMARD, "hadamard")
        op = lambda b, seed, **kw: (O.polar_params(d, seed, rotation=orot, **kw) if b == "polar"
                                    else O.make_params(d, b, seed, rotation=orot, **kw))
        self.kp = tqkv.make_params(d, lib(kbits), 1000 + seed, rot)
        self.Pk = op(kbits, 1000 + seed)
        self.vp = tqkv.make_params(d, lib(vbits), 2000 + seed, rot) if vbits else None
        self.Pv = op(vbits, 2000 + seed, with_S=False) if vbits else None
        self.d, self.kbits, self.kqjl, self.vbits, self.H, self.P = d, kbits, kqjl, vbits, H, page_tokens

    def encode(self, K, V, slots, num_blocks):
        cache = tqkv.alloc_cache(self.desc, num_blocks)
        ws = tqkv.encode(self.kp, self.vp, self.desc, K, V, slots, cache)
        torch.cuda.synchronize()
        return cache, tqkv.read_status(ws)

    def check_tokens(self, cache_np, slots_np, Kx, Vx, head):
        """Compare the stored fields of the given tokens of one head."""
        gpu = O.read_cache(self.lay, cache_np, slots_np, head, self.H)
        if self.kbits == "polar":
            Ek = O.encode_polar(Kx, self.Pk, qjl=self.kqjl)
            repk, exk = parity.compare_polar(gpu, Ek, key=True)
        else:
            Ek = O.encode(Kx, self.Pk, qjl=self.kqjl)
            repk, exk = parity.compare_vectors(gpu, Ek, key=True, bits=self.kbits)
        Ev = repv = None
        self.last_exempt = exk
        if self.vbits:
            if self.vbits == "polar":
                Ev = O.encode_polar(Vx, self.Pv, qjl=False)
                repv, exv = parity.compare_polar(gpu, Ev, key=False)
            else:
                Ev = O.encode(Vx, self.Pv, qjl=False)
                repv, exv = parity.compare_vectors(gpu, Ev, key=False, bits=self.vbits)
            self.last_exempt = exk | exv
        return Ek, Ev, exk, repk, repv

    def slack(self, Ev, logits, lse, out):
        """Per-row output allowance from the keys exempt in the last check."""
        if self.vbits == "polar":
            return parity.exempt_slack_polar(self.Pv, Ev, self.last_exempt, logits, lse, out)
        return parity.exempt_slack(self.Pv, Ev, self.last_exempt, logits, lse, out)


def cache_np(cache):
    return cache.view(cache.shape[0] * cache.shape[1], -1).cpu().numpy()


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


# ---------------------------------------------------------------------------
# single-head check: 1,024 keys/values (fp32, channels 5 and 77 x20), 16 queries
# ---------------------------------------------------------------------------
def test_single_head_small_check_every_output():
    d, L = 128, 1024
    Kh, Vh, Qh = synth.small_check(seed=0)
    cd = Codec(d, 3, True, 3, seed=0, page_tokens=64, H=1)
    bt, slots, nblk = synth.contiguous_block_table(1, L, 64, device=DEV, shuffle_seed=5)
    K = torch.from_numpy(Kh).to(DEV).view(L, 1, d)
    V = torch.from_numpy(Vh).to(DEV).view(L, 1, d)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    cn = cache_np(cache)
    Ek, Ev, exk, repk, repv = cd.check_tokens(cn, slots.cpu().numpy(), Kh.astype(np.float64),
                                              Vh.astype(np.float64), 0)
    # every query attends the whole cache: 16 sequences sharing one block table
    nq = Qh.shape[0]
    Qb = torch.from_numpy(Qh).to(DEV).to(torch.bfloat16).view(nq, 1, d)
    btq = bt.expand(nq, -1).contiguous()
    seq = torch.full((nq,), L, dtype=torch.int32, device=DEV)
    logits = torch.full((nq, 1, L), float("nan"), device=DEV)
    lse = torch.empty((nq, 1), device=DEV)
    out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Qb, btq, seq, L, cache, lse=lse, logits=logits)
    torch.cuda.synchronize()
    Qx = f64(Qb.view(nq, d))
    o_ref, lse_ref, lg_ref = O.attend(Qx, cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
    parity.check_logits(f64(logits.view(nq, L)), lg_ref, exk)
    parity.check_outputs(f64(out.view(nq, d)), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
    assert np.allclose(f64(lse.view(nq)), lse_ref, rtol=1e-3, atol=1e-3)
    # the same 16 queries as the last 16 positions of a prefill chunk
    C = nq
    outp = tqkv.prefill_attn(cd.kp, cd.vp, cd.desc, Qb, bt.view(-1), L, cache)
    torch.cuda.synchronize()
    nvis = np.arange(L - C + 1, L + 1, dtype=np.int32)
    o_p, lse_p, lg_p = O.attend(Qx, cd.Pk, Ek, cd.Pv, Ev, nvis=nvis, want_logits=True)
    parity.check_outputs(f64(outp.view(C, d)), o_p, cd.slack(Ev, lg_p, lse_p, o_p))


# ---------------------------------------------------------------------------
# write path of an 8B-dense-shaped layer: B=8, Hkv=8, d=128, 32,768 tokens
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("preset", ["k8v4", "k4qjl_v4"])
def test_write_path_full_size_sampled(preset):
    B, L, H, d, P = 8, 32768, 8, 128, 64
    n = B * L
    K = synth.lognormal_channels(n, H, d, seed=1, device=DEV)
    V = synth.lognormal_channels(n, H, d, seed=10001, device=DEV)
    cd = Codec(d, 8, False, 4, seed=1, H=H) if preset == "k8v4" else Codec(d, 4, True, 4, seed=1, H=H)
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=11)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    cn = cache_np(cache)
    rng = np.random.default_rng(3)
    toks = np.sort(rng.choice(n, 2048, replace=False))
    toks[0], toks[-1] = 0, n - 1
    sl = slots.cpu().numpy()[toks]
    Kt, Vt = f64(K[toks]), f64(V[toks])
    reports = []
    for h in range(H):
        _, _, _, repk, repv = cd.check_tokens(cn, sl, Kt[:, h], Vt[:, h], h)
        reports.append((repk, repv))
    print(preset, reports[0])
    if preset != "k8v4":
        # one GQA decode step (32 query heads) over the freshly written cache
        Q = synth.normal((B, 32, d), seed=12, device=DEV)
        seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
        logits = torch.full((B, 32, L), float("nan"), device=DEV)
        out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, logits=logits)
        torch.cuda.synchronize()
        for b, kvh in [(0, 0), (7, 5)]:
            idx = np.arange(b * L, (b + 1) * L)
            Ek, Ev, exk, _, _ = cd.check_tokens(cn, slots.cpu().numpy()[idx], f64(K[idx, kvh]), f64(V[idx, kvh]),
                                                kvh)
            rows = list(range(kvh * 4, kvh * 4 + 4))
            o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
            parity.check_logits(f64(logits[b, rows]), lg_ref, exk)
            parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))


# ---------------------------------------------------------------------------
# GQA decode: B=32, Hq=32 over Hkv=8, L=32,768, K 2-bit + QJL, V 4-bit
# ---------------------------------------------------------------------------
def test_decode_gqa_32x32k_sampled_rows():
    B, L, H, Hq, d, P = 32, 32768, 8, 32, 128, 64
    n = B * L
    K = synth.outlier_normal((n, H, d), seed=2, device=DEV)
    V = synth.outlier_normal((n, H, d), seed=20002, device=DEV)
    Q = synth.normal((B, Hq, d), seed=21, device=DEV)
    cd = Codec(d, 2, True, 4, seed=2, H=H)
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=22)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
    logits = torch.full((B, Hq, L), float("nan"), device=DEV)
    lse = torch.empty((B, Hq), device=DEV)
    out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, lse=lse, logits=logits)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for b, kvh in [(0, 0), (31, 7), (13, 3)]:
        idx = np.arange(b * L, (b + 1) * L)
        Ek, Ev, exk, repk, _ = cd.check_tokens(cn, sl[idx], f64(K[idx, kvh]), f64(V[idx, kvh]), kvh)
        rows = list(range(kvh * G, kvh * G + G))
        o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
        parity.check_logits(f64(logits[b, rows]), lg_ref, exk)
        parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
        assert np.allclose(f64(lse[b, rows]), lse_ref, rtol=1e-3, atol=1e-3)


# ---------------------------------------------------------------------------
# the alternative codecs at the size the bench times them: B=8 sequences x 8 KV
# heads x 8,192 tokens, 32 query heads (dense rotation, 3.5-bit fractional
# rates, polar codes); sampled (sequence, KV head) pairs: stored fields,
# logits and outputs
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kbits,vbits,dense", [(2, 4, True), (2.5, 3.5, False), ("polar", "polar", False)])
def test_alternative_codecs_bench_size_sampled(kbits, vbits, dense):
    B, L, H, Hq, d, P = 8, 8192, 8, 32, 128, 64
    n = B * L
    K = synth.outlier_normal((n, H, d), seed=51, device=DEV)
    V = synth.outlier_normal((n, H, d), seed=52, device=DEV)
    Q = synth.normal((B, Hq, d), seed=54, device=DEV)
    cd = Codec(d, kbits, True, vbits, seed=5, H=H, dense=dense)
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=53)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
    logits = torch.full((B, Hq, L), float("nan"), device=DEV)
    out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, logits=logits)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for b, kvh in [(0, 0), (7, 7), (3, 5)]:
        idx = np.arange(b * L, (b + 1) * L)
        Ek, Ev, exk, _, _ = cd.check_tokens(cn, sl[idx], f64(K[idx, kvh]), f64(V[idx, kvh]), kvh)
        rows = list(range(kvh * G, kvh * G + G))
        o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
        parity.check_logits(f64(logits[b, rows]), lg_ref, exk)
        parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))


# ---------------------------------------------------------------------------
# long context: B=1, Hq=32 over Hkv=4, L=262,144, 3-bit keys incl. QJL, 3-bit
# values; one decode step and one 2,048-query prefill chunk (causal inside)
# ---------------------------------------------------------------------------
def test_long_context_decode_and_prefill_sampled():
    L, H, Hq, d, P, C = 262144, 4, 32, 128, 64, 2048
    K = synth.outlier_normal((L, H, d), seed=3, device=DEV)
    V = synth.outlier_normal((L, H, d), seed=30003, device=DEV)
    cd = Codec(d, 2, True, 3, seed=3, H=H)
    bt, slots, nblk = synth.contiguous_block_table(1, L, P, device=DEV, shuffle_seed=33)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    Qd = synth.normal((1, Hq, d), seed=31, device=DEV)
    seq = torch.full((1,), L, dtype=torch.int32, device=DEV)
    logits = torch.full((1, Hq, L), float("nan"), device=DEV)
    out_d = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Qd, bt, seq, L, cache, logits=logits)
    Qp = synth.normal((C, Hq, d), seed=32, device=DEV)
    out_p = tqkv.prefill_attn(cd.kp, cd.vp, cd.desc, Qp, bt.view(-1), L, cache)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for kvh in (0, 3):
        Ek, Ev, exk, _, _ = cd.check_tokens(cn, sl, f64(K[:, kvh]), f64(V[:, kvh]), kvh)
        rows = list(range(kvh * G, kvh * G + G))
        o_ref, lse_ref, lg_ref = O.attend(f64(Qd[0, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
        parity.check_logits(f64(logits[0, rows]), lg_ref, exk)
        parity.check_outputs(f64(out_d[0, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
        for j in (0, 1, 777, C - 1):
            nvis = np.full(G, L - C + j + 1, np.int32)
            o_p, lse_p, lg_p = O.attend(f64(Qp[j, rows]), cd.Pk, Ek, cd.Pv, Ev, nvis=nvis, want_logits=True)
            parity.check_outputs(f64(out_p[j, rows]), o_p, cd.slack(Ev, lg_p, lse_p, o_p))


# ---------------------------------------------------------------------------
# tensor-core decode: every logit, output and lse on outlier-channel data
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kbits,vbits,B,Hq,H,L", [
    (2, 4, 3, 32, 8, 3000),       # k3v4 preset, G = 4, ragged lengths
    (4, 3, 2, 16, 2, 2500),       # G = 8
    (2, 3, 2, 8, 4, 4100),        # G = 2
    (8, 4, 3, 32, 8, 2200),       # k8v4 preset (FP8 keys, 4-bit values), G = 4
    (8, 3, 2, 16, 2, 1900),       # FP8 keys, G = 8
])
def test_decode_tensor_core_every_output(kbits, vbits, B, Hq, H, L):
    d, P = 128, 64
    seed = 60 + kbits * 10 + vbits
    K = synth.outlier_normal((B * L, H, d), seed=seed, device=DEV)
    V = synth.outlier_normal((B * L, H, d), seed=seed + 1, device=DEV)
    cd = Codec(d, kbits, kbits != 8, vbits, seed=seed, H=H)
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=seed)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    lens = [L - 37 * b for b in range(B)]
    seq = torch.tensor(lens, dtype=torch.int32, device=DEV)
    Q = synth.normal((B, Hq, d), seed=seed + 2, device=DEV)
    logits = torch.full((B, Hq, L), float("nan"), device=DEV)
    lse = torch.empty((B, Hq), device=DEV)
    out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, lse=lse, logits=logits)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for b in range(B):
        n = lens[b]
        idx = np.arange(b * L, b * L + n)
        for kvh in range(H):
            Ek, Ev, exk, _, _ = cd.check_tokens(cn, sl[idx], f64(K[idx, kvh]), f64(V[idx, kvh]), kvh)
            rows = list(range(kvh * G, kvh * G + G))
            o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
            parity.check_logits(f64(logits[b, rows, :n]), lg_ref, exk)
            parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
            assert np.allclose(f64(lse[b, rows]), lse_ref, rtol=1e-3, atol=1e-3)


# ---------------------------------------------------------------------------
# tensor-core prefill: every output and lse, ragged query tiles, ragged last
# page, several key splits, G = 1 .. 8
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kbits,vbits,Hq,H,C,L", [
    (2, 3, 32, 4, 100, 5000),     # G = 8: 16 positions per block, last block ragged, four key splits
    (3, 3, 8, 8, 64, 3100),       # G = 1: 128 positions per block, half used
    (4, 4, 16, 2, 40, 2600),      # G = 8, two KV heads
    (2, 2, 2, 1, 70, 1500),       # G = 2: 64 positions per block
    (3, 4, 8, 2, 33, 4096),       # G = 4, one position in the last block
    (8, 4, 16, 4, 24, 1500),      # k8v4: FP8 keys, each chunk position as a decode query group
])
def test_prefill_tensor_core_every_output(kbits, vbits, Hq, H, C, L):
    d, P = 128, 64
    seed = 40 + kbits * 10 + vbits
    K = synth.outlier_normal((L, H, d), seed=seed, device=DEV)
    V = synth.outlier_normal((L, H, d), seed=seed + 1, device=DEV)
    cd = Codec(d, kbits, kbits != 8, vbits, seed=seed, H=H)
    bt, slots, nblk = synth.contiguous_block_table(1, L, P, device=DEV, shuffle_seed=seed)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    Qp = synth.normal((C, Hq, d), seed=seed + 2, device=DEV)
    lse = torch.empty((C, Hq), device=DEV)
    out = tqkv.prefill_attn(cd.kp, cd.vp, cd.desc, Qp, bt.view(-1), L, cache, lse=lse)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for kvh in range(H):
        Ek, Ev, exk, _, _ = cd.check_tokens(cn, sl, f64(K[:, kvh]), f64(V[:, kvh]), kvh)
        rows = list(range(kvh * G, kvh * G + G))
        Qr = f64(Qp[:, rows]).reshape(C * G, d)
        nvis = np.repeat(np.arange(L - C + 1, L + 1, dtype=np.int32), G)
        o_p, lse_p, lg_p = O.attend(Qr, cd.Pk, Ek, cd.Pv, Ev, nvis=nvis, want_logits=True)
        parity.check_outputs(f64(out[:, rows]).reshape(C * G, d), o_p, cd.slack(Ev, lg_p, lse_p, o_p))
        assert np.allclose(f64(lse[:, rows]).reshape(C * G), lse_p, rtol=1e-3, atol=1e-3)


# ---------------------------------------------------------------------------
# search
# ---------------------------------------------------------------------------
def _search_case(n_db, n_q, seed, d=1024):
    X = synth.unit_normal(n_db, d, seed=seed, device=DEV)
    Qs = synth.unit_normal(n_q, d, seed=seed + 1, device=DEV)
    cd = Codec(d, 4, True, 0, seed=seed, H=1)
    nblk = -(-n_db // 64)
    slots = torch.arange(n_db, dtype=torch.int32, device=DEV)
    cache, flags = cd.encode(X, None, slots, nblk)
    assert flags == 0
    return X, Qs, cd, cache


def test_search_reduced_every_output():
    n_db, n_q, k = 20000, 16, 10
    X, Qs, cd, cache = _search_case(n_db, n_q, seed=4)
    sc, ix = tqkv.score(cd.kp, cd.desc, cache, n_db, Qs, k)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    Ek, _, exk, _, _ = cd.check_tokens(cn, np.arange(n_db), f64(X), None, 0)
    ref_sc, ref_ix = O.search(f64(Qs), cd.Pk, Ek, k + 1)
    gs, gi = f64(sc), ix.cpu().numpy()
    for a in range(n_q):
        est = O.estimate(f64(Qs[a]), cd.Pk, Ek)
        # GPU scores equal the oracle estimates of the returned vectors
        tol = 1e-3 * np.maximum(np.abs(est[gi[a]]), np.sqrt(np.mean(est ** 2)))
        ok = (np.abs(gs[a] - est[gi[a]]) <= tol) | exk[gi[a]]
        assert ok.all()
        # the returned set is the oracle's top-k unless the k-th/(k+1)-th gap is within tolerance
        if ref_sc[a, k - 1] - ref_sc[a, k] > 2e-3 * abs(ref_sc[a, k - 1]):
            assert set(gi[a]) == set(ref_ix[a, :k]) or exk[ref_ix[a, :k]].any()
        assert np.all(np.diff(gs[a]) <= 0)


def test_search_million_vectors_properties():
    n_db, n_q, k = 1_000_000, 1024, 10
    X, Qs, cd, cache = _search_case(n_db, n_q, seed=4)
    sc, ix = tqkv.score(cd.kp, cd.desc, cache, n_db, Qs, k)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    rng = np.random.default_rng(44)
    sample = np.sort(rng.choice(n_db, 1000, replace=False))
    cd.check_tokens(cn, sample, f64(X[sample]), None, 0)
    gs, gi = f64(sc), ix.cpu().numpy()
    for a in rng.choice(n_q, 8, replace=False):
        cand = np.unique(np.concatenate([gi[a], sample]))
        Ek, _, exk, _, _ = cd.check_tokens(cn, cand, f64(X[cand]), None, 0)
        est = O.estimate(f64(Qs[a]), cd.Pk, Ek)
        pos = {int(t): i for i, t in enumerate(cand)}
        mine = np.array([est[pos[int(t)]] for t in gi[a]])
        rms = np.sqrt(np.mean(est ** 2))
        assert np.all(np.abs(gs[a] - mine) <= 1e-3 * np.maximum(np.abs(mine), rms))
        others = np.array([est[pos[int(t)]] for t in sample if int(t) not in set(gi[a].tolist())])
        assert gs[a, k - 1] >= others.max() - 1e-3 * rms
    exact = torch.topk(Qs @ X.T, k, dim=1).indices.cpu().numpy()
    recall = np.mean([len(set(gi[a]) & set(exact[a])) / k for a in range(n_q)])
    print(f"recall@10 vs exact fp32: {recall:.4f}")
    assert recall > 0.3


@pytest.mark.parametrize("d,kbits,kqjl,n_db,n_q,k,qscale", [
    (128, 4, True, 3001, 130, 16, 1.0),      # tensor cores: two query tiles, ragged tails, largest k
    (256, 4, True, 1500, 5, 1, 1e5),         # tensor cores: k = 1, queries far beyond the fp16 range
    (512, 4, True, 777, 1, 3, 1e-6),         # tensor cores: one short tile, tiny query
    (1024, 4, True, 2600, 33, 6, 1.0),       # tensor cores: d = 1024, k between 4 and 8
    (64, 3, True, 2000, 9, 7, 1.0),          # general kernel (head dim below the tensor-core tile)
    (128, 2, False, 999, 3, 20, 1.0),        # general kernel (MSE-only codes, k above 16)
])
def test_search_configurations_every_output(d, kbits, kqjl, n_db, n_q, k, qscale):
    X = synth.unit_normal(n_db, d, seed=d + n_db, device=DEV)
    Qs = synth.unit_normal(n_q, d, seed=d + n_db + 1, device=DEV) * qscale
    cd = Codec(d, kbits, kqjl, 0, seed=d + k, H=1)
    nblk = -(-n_db // 64)
    slots = torch.arange(n_db, dtype=torch.int32, device=DEV)
    cache, flags = cd.encode(X, None, slots, nblk)
    assert flags == 0
    sc, ix = tqkv.score(cd.kp, cd.desc, cache, n_db, Qs, k)
    torch.cuda.synchronize()
    Ek, _, exk, _, _ = cd.check_tokens(cache_np(cache), np.arange(n_db), f64(X), None, 0)
    ref_sc, ref_ix = O.search(f64(Qs), cd.Pk, Ek, min(k + 1, n_db))
    gs, gi = f64(sc), ix.cpu().numpy()
    for a in range(n_q):
        assert len(set(gi[a].tolist())) == k and gi[a].min() >= 0 and gi[a].max() < n_db
        est = O.estimate(f64(Qs[a]), cd.Pk, Ek)
        tol = 1e-3 * np.maximum(np.abs(est[gi[a]]), np.sqrt(np.mean(est ** 2)))
        assert ((np.abs(gs[a] - est[gi[a]]) <= tol) | exk[gi[a]]).all()
        if k < n_db and ref_sc[a, k - 1] - ref_sc[a, k] > 2e-3 * abs(ref_sc[a, k - 1]):
            assert set(gi[a]) == set(ref_ix[a, :k]) or exk[ref_ix[a, :k]].any()
        assert np.all(np.diff(gs[a]) <= 0)


# ---------------------------------------------------------------------------
# edge cases: small and large head dims, ragged and empty sequences, skipped
# slots, zero vectors, out-of-range slots, G = 1 and 8
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,kbits,kqjl,vbits,P,Hq,H", [(8, 2, True, 1, 8, 2, 1), (16, 1, True, 2, 16, 8, 1),
                                                       (64, 3, True, 2, 16, 4, 2), (256, 4, False, 3, 32, 1, 1),
                                                       (128, 4, True, 4, 16, 8, 1), (32, 2, True, 4, 8, 6, 3),
                                                       (64, 8, False, 4, 16, 4, 2), (256, 8, False, 2, 32, 8, 1),
                                                       (128, 8, False, 4, 64, 3, 1)])
def test_small_dims_ragged_sequences(d, kbits, kqjl, vbits, P, Hq, H):
    seqs = [0, 1, 37, 3 * P + 5]
    B, Lmax = len(seqs), max(seqs)
    cd = Codec(d, kbits, kqjl, vbits, seed=d + kbits, page_tokens=P, H=H)
    bps = -(-Lmax // P)
    g = torch.Generator().manual_seed(d)
    phys = torch.randperm(B * bps + 3, generator=g)[:B * bps].view(B, bps).to(torch.int32)
    nblk = B * bps + 3
    toks, slot_list = [], []
    for b, Lb in enumerate(seqs):
        for t in range(Lb):
            toks.append((b, t))
            slot_list.append(int(phys[b, t // P]) * P + t % P)
    n = len(toks)
    # append two skipped tokens (slot -1): their inputs must not reach the cache
    slot_list += [-1, -1]
    K = synth.outlier_normal((n + 2, H, d), seed=d, device=DEV, dtype=torch.float32)
    V = synth.outlier_normal((n + 2, H, d), seed=d + 1, device=DEV, dtype=torch.float32)
    K[0].zero_()            # a zero vector
    slots = torch.tensor(slot_list, dtype=torch.int32, device=DEV)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    cn = cache_np(cache)
    sl = np.array(slot_list[:n])
    for h in range(H):
        cd.check_tokens(cn, sl, f64(K[:n, h]), f64(V[:n, h]), h)
    # bytes of pages no token was written to stay zero
    used = set(int(s) // P for s in slot_list[:n])
    unused = [blk for blk in range(nblk) if blk not in used]
    assert not cache[unused].any()
    Q = synth.normal((B, Hq, d), seed=d + 2, device=DEV)
    bt = phys.to(DEV)
    seq = torch.tensor(seqs, dtype=torch.int32, device=DEV)
    logits = torch.full((B, Hq, Lmax), float("nan"), device=DEV)
    lse = torch.empty((B, Hq), device=DEV)
    out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, Lmax, cache, lse=lse, logits=logits)
    torch.cuda.synchronize()
    G = Hq // H
    start = 0
    for b, Lb in enumerate(seqs):
        for kvh in range(H):
            rows = list(range(kvh * G, kvh * G + G))
            if Lb == 0:
                assert torch.all(out[b, rows] == 0)
                assert torch.all(torch.isneginf(lse[b, rows]))
                continue
            Ek, Ev, exk, _, _ = cd.check_tokens(cn, sl[start:start + Lb], f64(K[start:start + Lb, kvh]),
                                                f64(V[start:start + Lb, kvh]), kvh)
            o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
            parity.check_logits(f64(logits[b, rows, :Lb]), lg_ref, exk)
            parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
        start += Lb


def test_out_of_range_slot_is_flagged_and_skipped():
    cd = Codec(128, 2, True, 4, seed=9, page_tokens=16, H=1)
    K = synth.normal((4, 1, 128), seed=1, device=DEV)
    slots = torch.tensor([0, 1, 10_000, 2], dtype=torch.int32, device=DEV)
    cache, flags = cd.encode(K, K, slots, 1)
    assert flags & tqkv.TQ_DEV_SLOT_RANGE
    cn = cache_np(cache)
    Kx = f64(K[[0, 1, 3], 0])
    cd.check_tokens(cn, np.array([0, 1, 2]), Kx, Kx, 0)


def test_block_table_out_of_range_is_flagged():
    cd = Codec(128, 2, True, 4, seed=9, page_tokens=16, H=1)
    K = synth.normal((16, 1, 128), seed=1, device=DEV)
    slots = torch.arange(16, dtype=torch.int32, device=DEV)
    cache, _ = cd.encode(K, K, slots, 1)
    Q = synth.normal((1, 1, 128), seed=2, device=DEV)
    bt = torch.tensor([[0, 5]], dtype=torch.int32, device=DEV)     # block 5 does not exist
    seq = torch.tensor([20], dtype=torch.int32, device=DEV)
    ws = torch.zeros(tqkv.decode_workspace_bytes(cd.desc, 1, 1, 20), dtype=torch.uint8, device=DEV)
    tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, 20, cache, workspace=ws)
    assert tqkv.read_status(ws) & tqkv.TQ_DEV_BLOCK_RANGE


# ---------------------------------------------------------------------------
# fused decode step: the new token's write shares the query-prep launch
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,kbits,kqjl,vbits,B,Hq,H,L", [
    (128, 2, True, 4, 4, 32, 8, 777),      # k3v4, tensor-core decode
    (128, 8, False, 4, 3, 16, 4, 500),     # k8v4, tensor-core decode
    (128, 3, True, 3, 2, 8, 2, 300),       # 3-bit keys: general decode kernel
    (64, 4, True, 2, 3, 4, 1, 130),        # d = 64, general kernels
    (128, 2.5, True, 3.5, 2, 8, 2, 200),   # fractional rates
    (128, "polar", True, "polar", 2, 8, 4, 150),   # polar codes
])
def test_decode_step_writes_new_token_and_attends(d, kbits, kqjl, vbits, B, Hq, H, L):
    P = 64 if d == 128 else 16
    seed = 300 + d + (9 if kbits == "polar" else int(2 * kbits))
    cd = Codec(d, kbits, kqjl, vbits, seed=seed, page_tokens=P, H=H)
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=seed)
    K = synth.outlier_normal((B, L, H, d), seed=seed + 1, device=DEV)
    V = synth.outlier_normal((B, L, H, d), seed=seed + 2, device=DEV)
    sl = slots.view(B, L)
    old = sl[:, :L - 1].reshape(-1).contiguous()
    cache, flags = cd.encode(K[:, :L - 1].reshape(-1, H, d).contiguous(), V[:, :L - 1].reshape(-1, H, d).contiguous(),
                             old, nblk)
    assert flags == 0
    new_slots = sl[:, L - 1].contiguous().clone()
    new_slots[1] = -1                                   # sequence 1 writes nothing this step
    lens = [L] * B
    lens[1] = L - 1
    seq = torch.tensor(lens, dtype=torch.int32, device=DEV)
    Q = synth.normal((B, Hq, d), seed=seed + 3, device=DEV)
    ws = torch.zeros(tqkv.decode_workspace_bytes(cd.desc, B, Hq, L), dtype=torch.uint8, device=DEV)
    logits = torch.full((B, Hq, L), float("nan"), device=DEV)
    lse = torch.empty((B, Hq), device=DEV)
    out = tqkv.decode_step(cd.kp, cd.vp, cd.desc, K[:, L - 1].contiguous(), V[:, L - 1].contiguous(), new_slots, Q,
                           bt, seq, L, cache, lse=lse, logits=logits, workspace=ws)
    torch.cuda.synchronize()
    assert tqkv.read_status(ws) == 0
    cn = cache_np(cache)
    sln = sl.cpu().numpy()
    # the skipped token's slot stays empty
    lay = cd.lay
    back = O.read_cache(lay, cn, sln[1, L - 1:L], 0, H)
    assert np.all(back["kn"] == 0)
    G = Hq // H
    for b in range(B):
        n = lens[b]
        for kvh in range(H):
            Ek, Ev, exk, _, _ = cd.check_tokens(cn, sln[b, :n], f64(K[b, :n, kvh]), f64(V[b, :n, kvh]), kvh)
            rows = list(range(kvh * G, kvh * G + G))
            o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
            parity.check_logits(f64(logits[b, rows, :n]), lg_ref, exk)
            parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
            assert np.allclose(f64(lse[b, rows]), lse_ref, rtol=1e-3, atol=1e-3)


# ---------------------------------------------------------------------------
# dense random rotation: every path that rotates (encode, query preparation,
# the output's inverse rotation), with the tensor-core kernels downstream
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,kbits,kqjl,vbits,Hq,H,L,C", [
    (128, 2, True, 4, 32, 8, 700, 16),     # k3v4: tensor-core decode; prefill 16 x 4 heads
    (128, 8, False, 4, 16, 4, 500, 8),     # k8v4
    (64, 3, True, 3, 8, 2, 300, 4),        # general kernels
    (256, 4, True, 2, 4, 1, 200, 3),
])
def test_dense_rotation_encode_decode_prefill(d, kbits, kqjl, vbits, Hq, H, L, C):
    P = 64 if d == 128 else 16
    seed = 500 + d + kbits
    cd = Codec(d, kbits, kqjl, vbits, seed=seed, page_tokens=P, H=H, dense=True)
    assert np.array_equal(cd.kp.rotation_matrix().astype(np.float64), cd.Pk.Rm)
    B = 2
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=seed)
    K = synth.outlier_normal((B * L, H, d), seed=seed + 1, device=DEV)
    V = synth.outlier_normal((B * L, H, d), seed=seed + 2, device=DEV)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    Q = synth.normal((B, Hq, d), seed=seed + 3, device=DEV)
    seq = torch.tensor([L, L - 50], dtype=torch.int32, device=DEV)
    logits = torch.full((B, Hq, L), float("nan"), device=DEV)
    out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, logits=logits)
    Qp = synth.normal((C, Hq, d), seed=seed + 4, device=DEV)
    out_p = tqkv.prefill_attn(cd.kp, cd.vp, cd.desc, Qp, bt[0].contiguous(), L, cache)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for b in range(B):
        n = int(seq[b])
        idx = np.arange(b * L, b * L + n)
        for kvh in range(H):
            Ek, Ev, exk, _, _ = cd.check_tokens(cn, sl[idx], f64(K[idx, kvh]), f64(V[idx, kvh]), kvh)
            rows = list(range(kvh * G, kvh * G + G))
            o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
            parity.check_logits(f64(logits[b, rows, :n]), lg_ref, exk)
            parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
            if b == 0:
                for j in range(C):
                    nvis = np.full(G, L - C + j + 1, np.int32)
                    o_p, lse_p, lg_p = O.attend(f64(Qp[j, rows]), cd.Pk, Ek, cd.Pv, Ev, nvis=nvis, want_logits=True)
                    parity.check_outputs(f64(out_p[j, rows]), o_p, cd.slack(Ev, lg_p, lse_p, o_p))


@pytest.mark.parametrize("d", [128, 256])
def test_dense_rotation_search(d):
    n_db, n_q, k = 3000, 130, 10
    X = synth.unit_normal(n_db, d, seed=60 + d, device=DEV)
    Qs = synth.unit_normal(n_q, d, seed=61 + d, device=DEV)
    cd = Codec(d, 4, True, 0, seed=62 + d, H=1, dense=True)
    cache, flags = cd.encode(X, None, torch.arange(n_db, dtype=torch.int32, device=DEV), -(-n_db // 64))
    assert flags == 0
    sc, ix = tqkv.score(cd.kp, cd.desc, cache, n_db, Qs, k)
    torch.cuda.synchronize()
    E = O.encode(f64(X), cd.Pk, qjl=True)
    gpu = O.read_cache(cd.lay, cache_np(cache), np.arange(n_db), 0, 1)
    _, ex = parity.compare_vectors(gpu, E, key=True, bits=4)
    for q in range(0, n_q, 13):
        est = O.estimate(f64(Qs[q]), cd.Pk, E)
        rms = float(np.sqrt(np.mean(est ** 2)))
        got = ix[q].cpu().numpy()
        ok = ~ex[got]
        assert np.all(np.abs(sc[q].cpu().numpy()[ok] - est[got][ok]) <= 1e-3 * np.maximum(np.abs(est[got][ok]), rms))
        assert np.all(est[got] >= np.sort(est)[::-1][k - 1] - 2e-3 * rms)


# ---------------------------------------------------------------------------
# fractional rates (b + 1/2 bits per coordinate) through the general kernels
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,kbits,kqjl,vbits,Hq,H,L,P", [
    (128, 2.5, True, 3.5, 16, 4, 600, 64),     # 3.5-bit keys incl. QJL, 3.5-bit values
    (128, 1.5, True, 2.5, 8, 2, 400, 16),      # 2.5-bit keys incl. QJL, 2.5-bit values
    (64, 3.5, False, 1.5, 4, 1, 300, 16),
    (256, 2.5, True, 2.5, 8, 8, 150, 32),
    (16, 1.5, False, 3.5, 2, 2, 90, 8),
])
def test_fractional_rates_encode_decode_prefill(d, kbits, kqjl, vbits, Hq, H, L, P):
    seed = 700 + d + int(10 * kbits)
    cd = Codec(d, kbits, kqjl, vbits, seed=seed, page_tokens=P, H=H)
    B = 2
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=seed)
    K = synth.outlier_normal((B * L, H, d), seed=seed + 1, device=DEV, dtype=torch.float32)
    V = synth.outlier_normal((B * L, H, d), seed=seed + 2, device=DEV, dtype=torch.float32)
    K[3].zero_()
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    Q = synth.normal((B, Hq, d), seed=seed + 3, device=DEV)
    seq = torch.tensor([L, L - 21], dtype=torch.int32, device=DEV)
    logits = torch.full((B, Hq, L), float("nan"), device=DEV)
    out = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, logits=logits)
    C = 5
    Qp = synth.normal((C, Hq, d), seed=seed + 4, device=DEV)
    out_p = tqkv.prefill_attn(cd.kp, cd.vp, cd.desc, Qp, bt[0].contiguous(), L, cache)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for b in range(B):
        n = int(seq[b])
        idx = np.arange(b * L, b * L + n)
        for kvh in range(H):
            Ek, Ev, exk, _, _ = cd.check_tokens(cn, sl[idx], f64(K[idx, kvh]), f64(V[idx, kvh]), kvh)
            rows = list(range(kvh * G, kvh * G + G))
            o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), cd.Pk, Ek, cd.Pv, Ev, want_logits=True)
            parity.check_logits(f64(logits[b, rows, :n]), lg_ref, exk)
            parity.check_outputs(f64(out[b, rows]), o_ref, cd.slack(Ev, lg_ref, lse_ref, o_ref))
            if b == 0:
                for j in range(C):
                    nvis = np.full(G, L - C + j + 1, np.int32)
                    o_p, lse_p, lg_p = O.attend(f64(Qp[j, rows]), cd.Pk, Ek, cd.Pv, Ev, nvis=nvis, want_logits=True)
                    parity.check_outputs(f64(out_p[j, rows]), o_p, cd.slack(Ev, lg_p, lse_p, o_p))


@pytest.mark.parametrize("d,rate", [(128, 3.5), (256, 2.5)])
def test_fractional_rate_search(d, rate):
    n_db, n_q, k = 2500, 20, 10
    X = synth.unit_normal(n_db, d, seed=80 + d, device=DEV)
    Qs = synth.unit_normal(n_q, d, seed=81 + d, device=DEV)
    cd = Codec(d, rate, True, 0, seed=82 + d, H=1)
    cache, flags = cd.encode(X, None, torch.arange(n_db, dtype=torch.int32, device=DEV), -(-n_db // 64))
    assert flags == 0
    sc, ix = tqkv.score(cd.kp, cd.desc, cache, n_db, Qs, k)
    torch.cuda.synchronize()
    E = O.encode(f64(X), cd.Pk, qjl=True)
    gpu = O.read_cache(cd.lay, cache_np(cache), np.arange(n_db), 0, 1)
    _, ex = parity.compare_vectors(gpu, E, key=True, bits=rate)
    for q in range(n_q):
        est = O.estimate(f64(Qs[q]), cd.Pk, E)
        rms = float(np.sqrt(np.mean(est ** 2)))
        got = ix[q].cpu().numpy()
        ok = ~ex[got]
        assert np.all(np.abs(sc[q].cpu().numpy()[ok] - est[got][ok]) <= 1e-3 * np.maximum(np.abs(est[got][ok]), rms))
        assert np.all(est[got] >= np.sort(est)[::-1][k - 1] - 2e-3 * rms)


# ---------------------------------------------------------------------------
# PolarQuant codes (polar-coordinate angle quantizer) through the general kernels
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,kqjl,vpolar,Hq,H,L,P", [
    (128, True, True, 16, 4, 500, 64),       # polar keys + QJL, polar values
    (64, False, False, 8, 2, 300, 16),       # polar keys, 4-bit values
    (256, True, True, 4, 1, 160, 32),
    (8, True, True, 2, 1, 70, 8),
])
def test_polar_codes_encode_decode_prefill(d, kqjl, vpolar, Hq, H, L, P):
    seed = 900 + d
    vb = tqkv.TQ_BITS_POLAR if vpolar else 4
    desc = tqkv.cache_desc(d, tqkv.TQ_BITS_POLAR, kqjl, vb, page_tokens=P, n_kv_heads=H)
    kp, vp = tqkv.make_params(d, tqkv.TQ_BITS_POLAR, 1000 + seed), tqkv.make_params(d, vb, 2000 + seed)
    Pk = O.polar_params(d, 1000 + seed)
    Pv = O.polar_params(d, 2000 + seed, with_S=False) if vpolar else O.make_params(d, 4, 2000 + seed, with_S=False)
    lay = O.Layout(d, "polar", kqjl, "polar" if vpolar else 4, page_tokens=P)
    B = 2
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=seed)
    K = synth.outlier_normal((B * L, H, d), seed=seed + 1, device=DEV, dtype=torch.float32)
    V = synth.outlier_normal((B * L, H, d), seed=seed + 2, device=DEV, dtype=torch.float32)
    K[5].zero_()
    cache = tqkv.alloc_cache(desc, nblk)
    ws = tqkv.encode(kp, vp, desc, K, V, slots, cache)
    torch.cuda.synchronize()
    assert tqkv.read_status(ws) == 0
    Q = synth.normal((B, Hq, d), seed=seed + 3, device=DEV)
    seq = torch.tensor([L, L - 13], dtype=torch.int32, device=DEV)
    logits = torch.full((B, Hq, L), float("nan"), device=DEV)
    out = tqkv.decode_attn(kp, vp, desc, Q, bt, seq, L, cache, logits=logits)
    C = 4
    Qp = synth.normal((C, Hq, d), seed=seed + 4, device=DEV)
    out_p = tqkv.prefill_attn(kp, vp, desc, Qp, bt[0].contiguous(), L, cache)
    torch.cuda.synchronize()
    cn = cache_np(cache)
    sl = slots.cpu().numpy()
    G = Hq // H
    for b in range(B):
        n = int(seq[b])
        idx = np.arange(b * L, b * L + n)
        for kvh in range(H):
            gpu = O.read_cache(lay, cn, sl[idx], kvh, H)
            Ek = O.encode_polar(f64(K[idx, kvh]), Pk, qjl=kqjl)
            _, exk = parity.compare_polar(gpu, Ek, key=True)
            if vpolar:
                Ev = O.encode_polar(f64(V[idx, kvh]), Pv, qjl=False)
                _, exv = parity.compare_polar(gpu, Ev, key=False)
                slack = lambda lg, ls, o: parity.exempt_slack_polar(Pv, Ev, exk | exv, lg, ls, o)
            else:
                Ev = O.encode(f64(V[idx, kvh]), Pv, qjl=False)
                _, exv = parity.compare_vectors(gpu, Ev, key=False, bits=4)
                slack = lambda lg, ls, o: parity.exempt_slack(Pv, Ev, exk | exv, lg, ls, o)
            rows = list(range(kvh * G, kvh * G + G))
            o_ref, lse_ref, lg_ref = O.attend(f64(Q[b, rows]), Pk, Ek, Pv, Ev, want_logits=True)
            parity.check_logits(f64(logits[b, rows, :n]), lg_ref, exk)
            parity.check_outputs(f64(out[b, rows]), o_ref, slack(lg_ref, lse_ref, o_ref))
            if b == 0:
                for j in range(C):
                    nvis = np.full(G, L - C + j + 1, np.int32)
                    o_p, lse_p, lg_p = O.attend(f64(Qp[j, rows]), Pk, Ek, Pv, Ev, nvis=nvis, want_logits=True)
                    parity.check_outputs(f64(out_p[j, rows]), o_p, slack(lg_p, lse_p, o_p))


def test_decode_wait_timeout_is_flagged_and_context_survives():
    """A bounded on-chip wait that runs out (a barrier nothing completes, set
    up through the testing aid) sets TQ_DEV_WAIT_TIMEOUT, returns promptly,
    leaves nothing in flight, and the next call on the same context is exact."""
    import time
    cd = Codec(128, 2, True, 4, seed=19, H=2)
    B, Hq, L = 2, 8, 700
    K = synth.outlier_normal((B * L, 2, 128), seed=191, device=DEV)
    bt, slots, nblk = synth.contiguous_block_table(B, L, 64, device=DEV, shuffle_seed=19)
    cache, flags = cd.encode(K, K, slots, nblk)
    assert flags == 0
    Q = synth.normal((B, Hq, 128), seed=192, device=DEV)
    seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
    ws = torch.zeros(tqkv.decode_workspace_bytes(cd.desc, B, Hq, L), dtype=torch.uint8, device=DEV)
    ref = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, workspace=ws)
    torch.cuda.synchronize()
    assert tqkv.read_status(ws) == 0
    tqkv.test_stall_next_decode(2000)
    t0 = time.perf_counter()
    tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, workspace=ws)
    flags = tqkv.read_status(ws)
    assert time.perf_counter() - t0 < 5.0
    assert flags & tqkv.TQ_DEV_WAIT_TIMEOUT
    again = tqkv.decode_attn(cd.kp, cd.vp, cd.desc, Q, bt, seq, L, cache, workspace=ws)
    torch.cuda.synchronize()
    assert tqkv.read_status(ws) == 0
    assert torch.equal(again, ref)


# ---------------------------------------------------------------------------
# every configuration of the fused d = 128 bf16 encoder (fractional rates
# included): ragged tail tiles, skipped slots, a zero vector, three KV heads
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kbits,kqjl,vbits", [(4, True, 4), (2, True, 4), (2, True, 3), (3, True, 3), (3, True, 4),
                                              (8, False, 4), (4, False, 4), (3, False, 3), (4, True, 0),
                                              (2.5, True, 3.5), (1.5, True, 2.5), (3.5, True, 3.5),
                                              (2.5, True, 2.5)])
def test_fused_encoder_configurations(kbits, kqjl, vbits):
    d, H, P = 128, 3, 16
    n = 1000                                  # 3,000 vectors: 23 full tiles and a ragged one
    cd = Codec(d, kbits, kqjl, vbits, seed=int(40 + 2 * (kbits + vbits)), page_tokens=P, H=H)
    K = synth.lognormal_channels(n, H, d, seed=41, device=DEV)
    V = synth.lognormal_channels(n, H, d, seed=42, device=DEV) if vbits else None
    K[7].zero_()
    if V is not None:
        V[9].zero_()
    g = torch.Generator().manual_seed(43)
    nblk = -(-n // P) + 2
    perm = torch.randperm(nblk * P, generator=g)[:n].to(torch.int32)
    perm[[5, 500]] = -1                       # skipped tokens
    slots = perm.to(DEV)
    cache, flags = cd.encode(K, V, slots, nblk)
    assert flags == 0
    cn = cache_np(cache)
    keep = np.flatnonzero(perm.numpy() >= 0)
    sl = perm.numpy()[keep]
    for h in range(H):
        cd.check_tokens(cn, sl, f64(K[keep, h]), f64(V[keep, h]) if vbits else None, h)
