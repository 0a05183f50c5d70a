"""The library's Hilbert token order (a host computation, no GPU) against the
oracle's recursive definition of the curve, entry by entry, and its argument
checks."""
import ctypes

import numpy as np
import pytest

import oracle
import ultra_sparse_attention_b200 as usa


@pytest.mark.parametrize("h,w,frames,prefix", [(64, 64, 1, 0), (128, 128, 1, 0), (3, 5, 2, 4), (30, 45, 13, 226),
                                               (1, 1, 1, 0), (7, 1, 2, 3), (1, 9, 1, 0), (100, 37, 1, 11)])
def test_library_order_equals_oracle(h, w, frames, prefix):
    got = usa.rt_hilbert_order(h, w, frames=frames, prefix_tokens=prefix).numpy()
    assert np.array_equal(got, oracle.hilbert_order(h, w, frames=frames, prefix=prefix))


def test_hilbert_order_argument_validation():
    lib = usa.load_library()
    buf = (ctypes.c_int32 * 16)()
    assert lib.rt_hilbert_order(0, 1, 4, 4, buf) == usa.RT_OK
    assert lib.rt_hilbert_order(0, 1, 4, 4, None) == usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_hilbert_order(-1, 1, 4, 4, buf) == usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_hilbert_order(0, 0, 4, 4, buf) == usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_hilbert_order(0, 1, 0, 4, buf) == usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_hilbert_order(0, 1, 40000, 4, buf) == usa.RT_ERR_UNSUPPORTED
    assert lib.rt_hilbert_order(0, 70000, 32768, 32768, buf) == usa.RT_ERR_UNSUPPORTED


def test_permute_argument_validation():
    lib = usa.load_library()
    A16, MIS = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10002)
    ok = usa.RtShape(1, 2, 512, 64, 64, 64)
    assert lib.rt_permute_tokens(ctypes.byref(ok), A16, A16, 0, A16, None) == usa.RT_ERR_INVALID_ARGUMENT  # in place
    assert lib.rt_permute_tokens(ctypes.byref(ok), A16, None, 0, ctypes.c_void_p(0x20000), None) == \
        usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_permute_tokens(ctypes.byref(ok), MIS, A16, 0, ctypes.c_void_p(0x20000), None) == \
        usa.RT_ERR_INVALID_ARGUMENT
    bad = usa.RtShape(1, 2, 512, 64, 96, 64)
    assert lib.rt_permute_tokens(ctypes.byref(bad), A16, A16, 0, ctypes.c_void_p(0x20000), None) == \
        usa.RT_ERR_UNSUPPORTED
