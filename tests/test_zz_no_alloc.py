"""The allocation-free router entry point (scion_router_logits_static).

Some callers cannot call cudaMalloc: their device memory belongs to another allocator, or
they run where allocation is not allowed.  They use this entry point to get the router logits
with the split-K scratch held in the library's static device array.  Its output is checked
against the oracle's fp64 router logits at the routing tolerance of the other parity tests,
on two calls in a row (the second call reuses the scratch the first one left behind), for
every token-tile width the kernel is built for (1, 2, 4 and 8 tiles of 8 tokens, ragged last
tiles included) and at the entry point's limits (E = 512, d = 4096, T = 64).  This file is
collected last on purpose."""
import ctypes as C

import numpy as np
import pytest

import oracle
from tests.helpers import u16_to_dev
from workloads import synth

torch = pytest.importorskip("torch")
import ternary_quantized_moe_b200 as tq  # noqa: E402

pytestmark = pytest.mark.gpu


def _router_case(E, d, T, seed):
    """bf16 router + delta with the workloads' distributions (std 1/sqrt(d) and a tenth of it)
    and bf16 x ~ N(0, 1); an oracle layer that holds only the router (routing reads nothing else)."""
    rng = synth.rng_for(seed)
    std = 1.0 / np.sqrt(d)
    wr = synth.to_bf16_bits(rng.standard_normal((E, d), dtype=np.float32) * np.float32(std))
    wd = synth.to_bf16_bits(rng.standard_normal((E, d), dtype=np.float32) * np.float32(0.1 * std))
    x = synth.to_bf16_bits(rng.standard_normal((T, d), dtype=np.float32))
    none = np.zeros(1, np.uint8)
    ol = oracle.OracleLayer(d=d, n_experts=E, top_k=1, ffn=128, fmt=synth.PQ2_0, w_router=wr, w_delta=wd,
                            gate_exps=none, up_exps=none, down_exps=none)
    logits, _, _ = oracle.route(ol, x)
    return wr, wd, x, logits


@pytest.mark.parametrize("E,d,T", [(96, 1152, 5), (40, 512, 12), (512, 4096, 24), (256, 2048, 64),
                                   (512, 4096, 64)])
def test_static_router_matches_oracle_twice(E, d, T):
    wr, wd, x, ref = _router_case(E, d, T, 9000 + E + T)
    xd = u16_to_dev(x, torch.bfloat16, "cuda")
    wrd = u16_to_dev(wr, torch.bfloat16, "cuda")
    wdd = u16_to_dev(wd, torch.bfloat16, "cuda")
    lib = tq._load()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        got = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.scion_router_logits_static(xd.data_ptr(), T, wrd.data_ptr(), wdd.data_ptr(), E, d, got.data_ptr(),
                                            stream)
        assert st == tq.SCION_OK
        torch.cuda.synchronize()
        g = got.cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        # fp32 tensor-core dot products over d against the fp64 logits (the a2 routing tolerance)
        np.testing.assert_allclose(g, ref, rtol=0, atol=2e-4 * max(1.0, np.abs(ref).max()))


def test_static_router_rejects_sizes_above_its_limit():
    lib = tq._load()
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    p = dummy.data_ptr()
    assert lib.scion_router_logits_static(p, 65, p, p, 64, 256, p, None) == tq.SCION_EINVAL
    assert lib.scion_router_logits_static(p, 8, p, p, 513, 256, p, None) == tq.SCION_EINVAL
    assert lib.scion_router_logits_static(p, 8, p, p, 64, 4224, p, None) == tq.SCION_EINVAL
    assert lib.scion_router_logits_static(p, 8, p, p, 64, 200, p, None) == tq.SCION_EINVAL
    assert lib.scion_router_logits_static(p + 2, 8, p, p, 64, 256, p, None) == tq.SCION_EINVAL
