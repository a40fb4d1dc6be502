"""Host-side checks of libscion that need no GPU: the library loads, exports every
symbol include/scion.h declares, its host packers agree byte for byte with the
oracle's, and descriptor validation rejects bad layers before touching CUDA."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle
import ternary_quantized_moe_b200 as tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "scion.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(scion_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = tq._load()
    declared = _declared()
    assert len(declared) >= 13
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(tq.EXPORTS)


def test_block_bytes_and_status_strings():
    assert tq.scion_block_bytes(tq.SCION_PQ2_0) == 34
    assert tq.scion_block_bytes(tq.SCION_PTQ1_0) == 28
    assert tq.scion_block_bytes(7) == 0
    assert tq.scion_status_str(0) == "ok"
    assert "invalid code" in tq.scion_status_str(tq.SCION_EFORMAT)


@pytest.mark.parametrize("fmt", [tq.SCION_PQ2_0, tq.SCION_PTQ1_0])
def test_host_pack_matches_oracle(fmt):
    rng = np.random.default_rng(17)
    codes = rng.integers(-1, 2, size=(5, 7, 384)).astype(np.int8)
    scales = rng.integers(0, 1 << 16, size=(5, 7, 3)).astype(np.uint16)
    mine = tq.scion_pack_pq2(codes, scales) if fmt == tq.SCION_PQ2_0 else tq.scion_pack_ptq1(codes, scales)
    ref = oracle.pack(fmt, codes, scales)
    np.testing.assert_array_equal(mine, ref)
    c2, s2, st = tq.scion_unpack(fmt, ref)
    assert st == 0
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2, scales)


@pytest.mark.parametrize("fmt", [tq.SCION_PQ2_0, tq.SCION_PTQ1_0])
def test_host_unpack_flags_invalid_codes(fmt):
    bb = tq.scion_block_bytes(fmt)
    blk = oracle.pack(fmt, np.zeros((1, 128), np.int8), np.zeros((1, 1), np.uint16))
    bad = blk.copy()
    bad[0, 2] = 0xFF  # a 3 in every PQ2 field / a quintet byte above 242
    c, _, st = tq.scion_unpack(fmt, bad)
    assert st == tq.SCION_EFORMAT
    _, _, ost = oracle.unpack(fmt, bad)
    assert ost == oracle.EFORMAT
    assert blk.shape == (1, bb)


def test_host_pack_rejects_out_of_range_code():
    codes = np.zeros((1, 128), np.int8)
    codes[0, 3] = -2
    with pytest.raises(tq.ScionError) as ei:
        tq.scion_pack_pq2(codes, np.zeros((1, 1), np.uint16))
    assert ei.value.status == tq.SCION_EINVAL


def _desc(**over):
    D = tq._Desc()
    base = dict(d=256, n_experts=8, top_k=2, ffn=128, shared_ffn=0, rank=32, fmt=0, router_fp32=1, norm_topk=1)
    base.update(over)
    for k, v in base.items():
        setattr(D, k, v)
    for p in ("w_router", "w_router_delta", "gate_exps", "up_exps", "down_exps", "corr_a", "corr_b"):
        setattr(D, p, 0x1000)  # never dereferenced: validation fails first
    return D


@pytest.mark.parametrize("bad", [dict(d=200), dict(ffn=100), dict(top_k=0), dict(top_k=9), dict(top_k=33, n_experts=64),
                                 dict(fmt=5), dict(rank=8), dict(shared_ffn=64), dict(norm_topk=2),
                                 dict(n_experts=5000)])
def test_layer_create_rejects_bad_descriptors(bad):
    lib = tq._load()
    h = C.c_void_p()
    st = lib.scion_layer_create(C.byref(_desc(**bad)), 16, None, C.byref(h))
    assert st == tq.SCION_EINVAL and not h.value


def test_layer_create_rejects_null_banks_and_tokens():
    lib = tq._load()
    h = C.c_void_p()
    D = _desc()
    D.down_exps = None
    assert lib.scion_layer_create(C.byref(D), 16, None, C.byref(h)) == tq.SCION_EINVAL
    assert lib.scion_layer_create(C.byref(_desc()), 0, None, C.byref(h)) == tq.SCION_EINVAL
    assert lib.scion_moe_forward(None, 1, None, None, None) == tq.SCION_EINVAL


@pytest.mark.parametrize("off", [(2, 0, 0, 0), (0, 8, 0, 0), (0, 0, 4, 0), (0, 0, 0, 2)])
def test_static_router_rejects_misaligned_pointers_before_cuda(off):
    """x and the router matrices are read with 16-byte loads and logits written as fp32: a
    misaligned pointer is refused before any CUDA call (so this runs without a GPU; an aligned
    call here would reach the CUDA runtime and report SCION_ECUDA instead)."""
    lib = tq._load()
    base = 0x10000
    x, wr, wd, lg = (base + o for o in off)
    assert lib.scion_router_logits_static(x, 8, wr, wd, 64, 256, lg, None) == tq.SCION_EINVAL


def test_static_router_aligned_call_reaches_cuda():
    """Without a GPU an aligned call passes the argument checks and stops at the CUDA runtime.
    Skipped where a GPU is present: the pointers here are not device memory."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("fake pointers must not reach a real device")
    lib = tq._load()
    assert lib.scion_router_logits_static(0x10000, 8, 0x20000, 0x30000, 64, 256, 0x40000, None) == tq.SCION_ECUDA
