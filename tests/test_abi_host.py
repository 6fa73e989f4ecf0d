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
