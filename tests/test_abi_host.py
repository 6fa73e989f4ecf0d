"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function its header declares, builds the same parameters as the
oracle bit for bit, sizes pages like the oracle's layout, and rejects bad
arguments before touching the device."""
import ctypes

import numpy as np
import pytest

from kv_cache_vector_07_b200 import tqkv
from oracle import oracle as O


def test_every_declared_symbol_is_exported():
    names = tqkv.declared_functions()
    assert len(names) >= 14
    missing = [n for n in names if not tqkv.exported(n)]
    assert not missing, missing


@pytest.mark.parametrize("d", [8, 16, 64, 128, 1024])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_host_params_equal_oracle(d, bits):
    seed = 0xC0FFEE + d + bits
    signs, S, lv, bd = tqkv.compute_params_host(d, bits, seed)
    P = O.make_params(d, bits, seed)
    assert np.array_equal(signs, P.signs)
    assert np.array_equal(S, P.S)
    if bits != 8:
        assert np.array_equal(lv, P.c32)
        assert np.array_equal(bd, P.t32)


@pytest.mark.parametrize("d", [16, 128, 256])
@pytest.mark.parametrize("rate", [1.5, 2.5, 3.5])
def test_host_fractional_params_equal_oracle(d, rate):
    seed = 77 + d
    signs, S, lv, bd = tqkv.compute_params_host(d, tqkv.half_bits(rate), seed)
    P = O.make_params(d, rate, seed)
    assert np.array_equal(signs, P.signs) and np.array_equal(S, P.S)
    assert np.array_equal(lv, np.concatenate([P.c32, P.c32b]))
    assert np.array_equal(bd, np.concatenate([P.t32, P.t32b]))
    with pytest.raises(tqkv.TQError):
        tqkv.compute_params_host(8, tqkv.half_bits(rate), seed)        # d < 16 unsupported


@pytest.mark.parametrize("d,kbits,kqjl,vbits,P", [(128, 2.5, True, 3.5, 64), (64, 1.5, True, 2.5, 16),
                                                  (256, 3.5, False, 1.5, 32), (16, 2.5, True, 2.5, 8)])
def test_fractional_page_bytes_equal_oracle_layout(d, kbits, kqjl, vbits, P):
    desc = tqkv.cache_desc(d, tqkv.half_bits(kbits), kqjl, tqkv.half_bits(vbits), page_tokens=P, n_kv_heads=2)
    assert tqkv.cache_bytes(desc) == O.Layout(d, kbits, kqjl, vbits, page_tokens=P).page_bytes


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_host_polar_params_equal_oracle(d):
    seed = 91 + d
    signs, S, lv, bd = tqkv.compute_params_host(d, tqkv.TQ_BITS_POLAR, seed)
    P = O.polar_params(d, seed)
    assert np.array_equal(signs, P.signs) and np.array_equal(S, P.S)
    assert np.array_equal(lv, np.concatenate([P.c1, P.ch.ravel()]))
    assert np.array_equal(bd, np.concatenate([P.t1, P.th.ravel()]))
    for kq, vb in ((True, tqkv.TQ_BITS_POLAR), (False, 3)):
        desc = tqkv.cache_desc(d, tqkv.TQ_BITS_POLAR, kq, vb, page_tokens=16, n_kv_heads=2)
        lay = O.Layout(d, "polar", kq, "polar" if vb == tqkv.TQ_BITS_POLAR else vb, page_tokens=16)
        assert tqkv.cache_bytes(desc) == lay.page_bytes
    with pytest.raises(tqkv.TQError):
        tqkv.compute_params_host(512, tqkv.TQ_BITS_POLAR, seed)


@pytest.mark.parametrize("d", [8, 32, 128, 256])
@pytest.mark.parametrize("seed", [1, 1003, 0xBEEF])
def test_host_dense_rotation_equals_oracle(d, seed):
    # the library's Householder QR and the oracle's Gram-Schmidt, both in
    # float64, round to the same float32 matrix
    R = tqkv.compute_rotation_host(d, seed, tqkv.TQ_ROT_DENSE)
    assert np.array_equal(R.astype(np.float64), O.dense_rotation(d, seed)[2])
    H = tqkv.compute_rotation_host(d, seed, tqkv.TQ_ROT_HADAMARD)
    P = O.make_params(d, 2, seed, with_S=False)
    assert np.allclose(H, O.rotate(np.eye(d), P.signs).T, atol=1e-7, rtol=0)
    with pytest.raises(tqkv.TQError):
        tqkv.compute_rotation_host(512, seed, tqkv.TQ_ROT_DENSE)


@pytest.mark.parametrize("d,kbits,kqjl,vbits,P", [(128, 2, True, 4, 64), (128, 2, True, 3, 64), (128, 8, False, 4, 64),
                                                  (128, 4, True, 4, 64), (128, 3, True, 3, 16), (8, 2, True, 1, 8),
                                                  (1024, 4, True, 0, 64), (64, 1, False, 2, 32)])
def test_page_bytes_equal_oracle_layout(d, kbits, kqjl, vbits, P):
    desc = tqkv.cache_desc(d, kbits, kqjl, vbits, page_tokens=P, n_kv_heads=3)
    lay = O.Layout(d, kbits, kqjl, vbits, page_tokens=P)
    assert tqkv.cache_bytes(desc) == lay.page_bytes


def test_invalid_arguments_rejected_on_host():
    with pytest.raises(tqkv.TQError) as e:
        tqkv.compute_params_host(100, 2, 0)
    assert e.value.code == tqkv.TQ_EUNSUPPORTED
    with pytest.raises(tqkv.TQError):
        tqkv.compute_params_host(128, 5, 0)
    for bad in [tqkv.cache_desc(100, 2, True, 4), tqkv.cache_desc(128, 8, True, 4),
                tqkv.cache_desc(128, 2, True, 4, page_tokens=12), tqkv.cache_desc(128, 2, True, 5),
                tqkv.cache_desc(128, 2, True, 4, n_kv_heads=0)]:
        with pytest.raises(tqkv.TQError) as e:
            tqkv.cache_bytes(bad)
        assert e.value.code == tqkv.TQ_EINVAL
    lib = tqkv._lib
    desc = tqkv.cache_desc(128, 2, True, 4)
    # null parameter handles and pointers fail validation before any launch
    assert lib.tq_encode(None, None, ctypes.byref(desc), None, None, 0, 1, None, None, 1, None, 0, None) == tqkv.TQ_EINVAL
    assert lib.tq_decode_attn(None, None, ctypes.byref(desc), None, 1, 8, None, 1, None, 1, None, 1, None, None,
                              None, 0, None, 0, None) == tqkv.TQ_EINVAL
    assert lib.tq_score(None, ctypes.byref(desc), None, 1, None, 1, 1, None, None, None, 0, None) == tqkv.TQ_EINVAL
    assert tqkv.status_string(tqkv.TQ_EDEVICE).startswith("device-side")


def test_workspace_sizes_grow_with_problem():
    desc = tqkv.cache_desc(128, 2, True, 4, n_kv_heads=8)
    assert tqkv.encode_workspace_bytes(desc, 1000) > tqkv.encode_workspace_bytes(desc, 10) >= 256
    d0 = tqkv.decode_workspace_bytes(desc, 1, 32, 1000)
    d1 = tqkv.decode_workspace_bytes(desc, 32, 32, 32768)
    assert d1 > d0 >= 256
    sdesc = tqkv.cache_desc(1024, 4, True, 0)
    assert tqkv.score_workspace_bytes(sdesc, 10 ** 6, 1024, 10) > tqkv.score_workspace_bytes(sdesc, 1000, 8, 10)
    # an MSE-only cache needs no residual scratch
    assert tqkv.encode_workspace_bytes(tqkv.cache_desc(128, 3, False, 3), 10 ** 6) == 256
