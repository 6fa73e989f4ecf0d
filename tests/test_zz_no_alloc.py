"""tq_decode_attn_noalloc: decode attention for callers that cannot allocate
device memory (an engine that keeps all device memory in its own pool, a
plug-in handed only one call's tensors, a path that cannot afford a blocking
cudaMalloc).  Its scratch is the library's static device array instead of a
caller workspace; its results must match tq_decode_attn's, call after call.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from kv_cache_vector_07_b200 import synth, tqkv

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(B, Hq, H, L, seed, kbits=2, vbits=4, d=128, P=64):
    desc = tqkv.cache_desc(d, kbits, True, vbits, page_tokens=P, n_kv_heads=H)
    kp, vp = tqkv.make_params(d, kbits, 500 + seed), tqkv.make_params(d, vbits, 600 + seed)
    bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=DEV, shuffle_seed=seed)
    K = synth.outlier_normal((B * L, H, d), seed=seed, device=DEV)
    V = synth.outlier_normal((B * L, H, d), seed=seed + 1, device=DEV)
    cache = tqkv.alloc_cache(desc, nblk, device=DEV)
    tqkv.encode(kp, vp, desc, K, V, slots, cache)
    lens = torch.tensor([L - 3 * b for b in range(B)], dtype=torch.int32, device=DEV)
    Q = synth.normal((B, Hq, d), seed=seed + 2, device=DEV)
    return desc, kp, vp, bt, lens, cache, Q


def _run(fn, desc, kp, vp, bt, lens, cache, Q, L):
    B, Hq, _ = Q.shape
    out = torch.empty_like(Q)
    lse = torch.empty((B, Hq), device=DEV)
    logits = torch.zeros((B, Hq, L), device=DEV)
    fn(kp, vp, desc, Q, bt, lens, L, cache, out=out, lse=lse, logits=logits)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), logits.cpu().numpy()


def _same(a, b):
    (o1, l1, g1), (o2, l2, g2) = a, b
    # output tolerance of the parity tests, for two bf16-rounded results
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(o2), 2.0 ** -126))) - 7)
    assert np.all(np.abs(o1 - o2) <= 2e-3 + ulp), np.abs(o1 - o2).max()
    rms = np.sqrt(np.mean(g2 ** 2, axis=-1, keepdims=True))
    assert np.all(np.abs(g1 - g2) <= 1e-3 * np.maximum(np.abs(g2), rms))  # logit tolerance of the parity tests
    assert np.allclose(l1, l2, rtol=1e-3, atol=1e-3)


def test_noalloc_decode_matches_workspace_decode_twice():
    L = 3000
    args = _case(B=4, Hq=16, H=4, L=L, seed=71)
    ref = _run(tqkv.decode_attn, *args, L)
    first = _run(tqkv.decode_attn_noalloc, *args, L)
    # a different problem in between leaves other contents in the shared array
    other = _case(B=2, Hq=8, H=1, L=700, seed=72, kbits=3, vbits=3)
    _run(tqkv.decode_attn_noalloc, *other, 700)
    second = _run(tqkv.decode_attn_noalloc, *args, L)
    _same(first, ref)
    _same(second, ref)


def test_noalloc_rejects_problems_beyond_its_static_scratch():
    desc = tqkv.cache_desc(128, 2, True, 4, page_tokens=64, n_kv_heads=8)
    B, Hq, L = 2048, 64, 1 << 20
    assert tqkv.decode_workspace_bytes(desc, B, Hq, L) > tqkv.TQ_NOALLOC_SCRATCH_BYTES
    kp, vp = tqkv.make_params(128, 2, 1), tqkv.make_params(128, 4, 2)
    Q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device=DEV)
    bt = torch.zeros((B, 1), dtype=torch.int32, device=DEV)
    lens = torch.zeros((B,), dtype=torch.int32, device=DEV)
    cache = torch.zeros((1, 8, tqkv.cache_bytes(desc)), dtype=torch.uint8, device=DEV)
    with pytest.raises(tqkv.TQError) as e:
        tqkv.decode_attn_noalloc(kp, vp, desc, Q, bt, lens, L, cache)
    assert e.value.code == tqkv.TQ_ESCRATCH


def test_noalloc_status_word_reports_a_block_out_of_range():
    # the no-allocation entry point's flags are readable: a block-table entry
    # beyond the cache sets TQ_DEV_BLOCK_RANGE; the next clean call reports 0
    desc, kp, vp, bt, lens, cache, Q = _case(B=2, Hq=8, H=2, L=500, seed=73)
    good = _run(tqkv.decode_attn_noalloc, desc, kp, vp, bt, lens, cache, Q, 500)
    assert tqkv.noalloc_read_status() == 0
    bad = bt.clone()
    bad[1, 3] = cache.shape[0] + 5
    _run(tqkv.decode_attn_noalloc, desc, kp, vp, bad, lens, cache, Q, 500)
    assert tqkv.noalloc_read_status() & tqkv.TQ_DEV_BLOCK_RANGE
    again = _run(tqkv.decode_attn_noalloc, desc, kp, vp, bt, lens, cache, Q, 500)
    assert tqkv.noalloc_read_status() == 0
    _same(again, good)

