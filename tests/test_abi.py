"""The C-ABI library builds for sm_100a, loads, exports what the header
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

import ultra_sparse_attention_b200 as usa
from ultra_sparse_attention_b200 import RtShape

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rettention.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rt_[a-z_]+)\s*\(", text)))


def test_header_declares_the_path_calls():
    names = _declared_functions()
    for n in ("rt_build_block_mask", "rt_attn_full_capture", "rt_attn_sparse_reshape", "rt_pair_query_blocks",
              "rt_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = usa.load_library()
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    assert usa.rt_abi_version() == 7
    for code in range(5):
        s = usa.rt_status_string(code)
        assert s.startswith("RT_")
    assert usa.rt_status_string(99) == "unknown rt_status"


# Fake, never-dereferenced device addresses: validation must reject before use.
A16 = ctypes.c_void_p(0x10000)
A4 = ctypes.c_void_p(0x10004)
MIS = ctypes.c_void_p(0x10002)


def _mask(lib, shape, q=A16, k=A16, scale=0.125, keep=2, forced=0, rp=A16, ci=A16, sc=None):
    return lib.rt_build_block_mask(ctypes.byref(shape) if shape is not None else None, q, k, scale, keep, forced,
                                   rp, ci, sc, None)


def _sparse(lib, shape, stats=(None, None, None, None), out=A16, scale=0.125, tiles=None):
    return lib.rt_attn_sparse_reshape(ctypes.byref(shape), A16, A16, A16, scale, A16, A16, tiles, *stats, out, None)


def _pair(lib, shape, rp=A16, ci=A16, tiles=A16, ws=None, ws_bytes=0):
    return lib.rt_pair_query_blocks(ctypes.byref(shape) if shape is not None else None, rp, ci, tiles, ws, ws_bytes,
                                    None)


def _capture(lib, shape, u=A16, m=A16, ws=None, ws_bytes=0):
    return lib.rt_attn_full_capture(ctypes.byref(shape), A16, A16, A16, 0.125, A16, A16, A16, m, A16, A16, u,
                                    ws, ws_bytes, None)


def test_mask_argument_validation():
    lib = usa.load_library()
    ok = RtShape(1, 2, 512, 64, 64, 64)
    assert _mask(lib, None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, RtShape(1, 2, 512, 64, 96, 64)) == usa.RT_ERR_UNSUPPORTED      # D
    assert _mask(lib, RtShape(1, 2, 512, 64, 64, 32)) == usa.RT_ERR_UNSUPPORTED      # block size
    assert _mask(lib, RtShape(1, 2, 512, 81, 80, 64)) == usa.RT_ERR_INVALID_ARGUMENT  # d > D
    assert _mask(lib, RtShape(0, 2, 512, 64, 64, 64)) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, RtShape(1, 1, 64 * 4097, 64, 64, 64)) == usa.RT_ERR_UNSUPPORTED  # too many blocks
    assert _mask(lib, ok, q=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, ok, q=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, ok, rp=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, ok, keep=0) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, ok, keep=9) == usa.RT_ERR_INVALID_ARGUMENT                     # > n_blocks
    assert _mask(lib, ok, keep=2, forced=130) == usa.RT_ERR_INVALID_ARGUMENT          # 3 forced > keep
    assert _mask(lib, ok, forced=-1) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, ok, scale=0.0) == usa.RT_ERR_INVALID_ARGUMENT
    assert _mask(lib, ok, scale=float("nan")) == usa.RT_ERR_INVALID_ARGUMENT


def test_attention_argument_validation():
    lib = usa.load_library()
    ok = RtShape(2, 3, 1000, 72, 80, 64)
    assert _sparse(lib, ok, stats=(A16, None, None, None)) == usa.RT_ERR_INVALID_ARGUMENT  # partial stats
    assert _sparse(lib, ok, stats=(A4, A4, A4, A4)) == usa.RT_ERR_INVALID_ARGUMENT        # U misaligned
    assert _sparse(lib, ok, out=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _sparse(lib, ok, scale=-1.0) == usa.RT_ERR_INVALID_ARGUMENT
    assert _sparse(lib, RtShape(2, 3, 1000, 72, 72, 64)) == usa.RT_ERR_UNSUPPORTED
    assert _sparse(lib, ok, tiles=MIS) == usa.RT_ERR_INVALID_ARGUMENT                     # table misaligned
    assert _capture(lib, ok, u=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _capture(lib, ok, u=A4) == usa.RT_ERR_INVALID_ARGUMENT
    assert _capture(lib, ok, m=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert _capture(lib, RtShape(2, 3, 1000, 72, 80, 256)) == usa.RT_ERR_UNSUPPORTED


def test_pairing_argument_validation():
    lib = usa.load_library()
    ok = RtShape(1, 2, 512, 64, 64, 64)
    assert _pair(lib, None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _pair(lib, ok, rp=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _pair(lib, ok, ci=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _pair(lib, ok, tiles=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert _pair(lib, ok, tiles=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert _pair(lib, RtShape(1, 2, 512, 64, 64, 32)) == usa.RT_ERR_UNSUPPORTED
    assert _pair(lib, RtShape(1, 1, 64 * 4097, 64, 64, 64)) == usa.RT_ERR_UNSUPPORTED


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        usa.rt_build_block_mask(q, q, head_dim=64, block_size=64, scale=0.125, keep_blocks=1)


def test_source_hash_covers_code_not_comments():
    """The build stamp (and the DRAM traffic keyed to it) changes with the code only."""
    from ultra_sparse_attention_b200 import build as b
    src = 'int a = 1; // note\n/* block\n note */ const char* s = "x // kept /* kept */";\nchar q = \'"\';  int  b;'
    assert b.code_text(src) == 'int a = 1; const char* s = "x // kept /* kept */"; char q = \'"\'; int b;'
    edited = src.replace("// note", "// another note\n// and a line more").replace("  int", "\n\nint")
    assert b.code_text(edited) == b.code_text(src)
    assert b.code_text(src.replace("a = 1", "a = 2")) != b.code_text(src)


def test_workspace_sizes_and_validation():
    """rt_workspace_bytes gives the capture's f16 copy of V plus its per-head maxima and the
    pairing's candidates; a caller workspace that is too small or misaligned is refused
    before any CUDA call."""
    cap, pair = usa.rt_workspace_bytes(2, 3, 1000, head_dim=72, head_dim_padded=80, block_size=64)
    assert cap == 2 * 3 * 1000 * 80 * 2 + 2 * 3 * 4
    assert pair == 2 * 3 * 16 * 16  # 16 blocks of 64, eight int16 candidates each
    assert usa.rt_workspace_bytes(2, 3, 1000, head_dim=72, head_dim_padded=80, block_size=128)[1] == 0
    with pytest.raises(usa.RtError):
        usa.rt_workspace_bytes(2, 3, 1000, head_dim=72, head_dim_padded=96, block_size=64)
    lib = usa.load_library()
    ok = RtShape(2, 3, 1000, 72, 80, 64)
    assert _capture(lib, ok, ws=A16, ws_bytes=cap - 1) == usa.RT_ERR_INVALID_ARGUMENT
    assert _capture(lib, ok, ws=A4, ws_bytes=cap) == usa.RT_ERR_INVALID_ARGUMENT
    assert _pair(lib, ok, ws=A16, ws_bytes=pair - 1) == usa.RT_ERR_INVALID_ARGUMENT
    assert _pair(lib, ok, ws=MIS, ws_bytes=pair) == usa.RT_ERR_INVALID_ARGUMENT


def test_compressed_cache_argument_validation():
    """The f16-U variants validate like the fp32 ones, and need U's scale array."""
    lib = usa.load_library()
    ok = RtShape(2, 3, 1000, 72, 80, 64)

    def cap16(u16=A16, us=A16, m=A16, shape=ok):
        return lib.rt_attn_full_capture_u16(ctypes.byref(shape), A16, A16, A16, 0.125, A16, A16, A16, m, A16, A16,
                                            u16, us, None, 0, None)

    def sp16(stats=(A16, A16, A16, A16, A16), shape=ok, out=A16):
        return lib.rt_attn_sparse_reshape_u16(ctypes.byref(shape), A16, A16, A16, 0.125, A16, A16, None, *stats,
                                              out, None)

    assert cap16(u16=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert cap16(us=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert cap16(u16=A4) == usa.RT_ERR_INVALID_ARGUMENT       # U must be 16-byte aligned
    assert cap16(us=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert cap16(m=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert cap16(shape=RtShape(2, 3, 1000, 72, 96, 64)) == usa.RT_ERR_UNSUPPORTED
    assert sp16(stats=(None, None, None, None, None)) == usa.RT_ERR_INVALID_ARGUMENT  # all five needed
    assert sp16(stats=(A16, A16, A16, A16, None)) == usa.RT_ERR_INVALID_ARGUMENT
    assert sp16(stats=(A16, A16, A16, A4, A16)) == usa.RT_ERR_INVALID_ARGUMENT
    assert sp16(out=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert sp16(shape=RtShape(2, 3, 1000, 72, 80, 32)) == usa.RT_ERR_UNSUPPORTED


def test_exact_mask_argument_validation():
    lib = usa.load_library()
    ok = RtShape(1, 2, 512, 64, 64, 64)

    def ex(shape=ok, q=A16, v=A16, keep=2, forced=0, rp=A16, mass=None, ws=None, ws_bytes=0, scale=0.125):
        return lib.rt_build_block_mask_exact(ctypes.byref(shape), q, A16, v, scale, keep, forced, rp, A16, mass, ws,
                                             ws_bytes, None)

    n = ctypes.c_size_t(0)
    assert lib.rt_exact_mask_workspace_bytes(ctypes.byref(ok), ctypes.byref(n)) == usa.RT_OK
    assert n.value >= 2 * 512 * 8 * 4  # at least the per-tile log-sum-exps
    assert ex(v=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(q=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(rp=None) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(mass=MIS) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(keep=0) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(keep=9) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(keep=1, forced=65) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(scale=float("inf")) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(ws=ctypes.c_void_p(0x10010), ws_bytes=n.value) == usa.RT_ERR_INVALID_ARGUMENT  # 256-byte alignment
    assert ex(ws=ctypes.c_void_p(0x10000), ws_bytes=n.value - 1) == usa.RT_ERR_INVALID_ARGUMENT
    assert ex(shape=RtShape(1, 2, 512, 64, 64, 32)) == usa.RT_ERR_UNSUPPORTED


def test_exp2_selftest_argument_validation():
    """Rejected before any launch (no GPU needed); n = 0 does nothing."""
    lib = usa.load_library()
    assert lib.rt_selftest_exp2_poly(None, None, 0, None) == usa.RT_OK
    assert lib.rt_selftest_exp2_poly(A16, A16, -1, None) == usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_selftest_exp2_poly(None, A16, 4, None) == usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_selftest_exp2_poly(A16, None, 4, None) == usa.RT_ERR_INVALID_ARGUMENT
    assert lib.rt_selftest_exp2_poly(ctypes.c_void_p(0x10002), A16, 4, None) == usa.RT_ERR_INVALID_ARGUMENT
