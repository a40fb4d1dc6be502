"""The allocation-free router entry point (scion_router_logits_static).

Callers that cannot allocate device memory use it to get router logits with the split-K
scratch held in the library's static device array.  Its output must equal the router
logits of the regular forward (scion_moe_forward_debug) within the routing tolerance the
other parity tests use, on two calls in a row (the second call reuses the scratch the
first one left behind).  This file is collected last on purpose."""
import ctypes as C

import numpy as np
import pytest

from tests.helpers import device_layer, oracle_layer_packed, packed_banks, u16_to_dev, with_margin
from workloads import synth

torch = pytest.importorskip("torch")
import ternary_quantized_moe_b200 as tq  # noqa: E402

pytestmark = pytest.mark.gpu


def _layer(E, d, T):
    cfg = synth.Config("noalloc", 31, d, E, 4, 128, 0, synth.PQ2_0, 0, False, [T], 1)
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    x = with_margin(cfg, oracle_layer_packed(cfg, L, banks), synth.x_host(cfg, T))
    return cfg, L, banks, x


@pytest.mark.parametrize("E,d,T", [(256, 2048, 64), (96, 1152, 5)])
def test_static_router_matches_forward_twice(E, d, T):
    cfg, L, banks, x = _layer(E, d, T)
    layer = device_layer(cfg, L, banks, 64)
    xd = u16_to_dev(x, torch.bfloat16, "cuda")
    wr = u16_to_dev(L["w_router"], torch.bfloat16, "cuda")
    wd = u16_to_dev(L["w_delta"], torch.bfloat16, "cuda")
    out = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ref = torch.empty((T, E), dtype=torch.float32, device="cuda")
    tq.scion_moe_forward_debug(xd, T, layer, out, logits=ref)
    torch.cuda.synchronize()
    ref_np = ref.cpu().numpy().astype(np.float64)
    lib = tq._load()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        got = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.scion_router_logits_static(xd.data_ptr(), T, wr.data_ptr(), wd.data_ptr(), E, d, got.data_ptr(),
                                            stream)
        assert st == tq.SCION_OK
        torch.cuda.synchronize()
        g = got.cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        np.testing.assert_allclose(g, ref_np, rtol=0, atol=2e-4 * max(1.0, np.abs(ref_np).max()))


def test_static_router_rejects_sizes_above_its_limit():
    lib = tq._load()
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    p = dummy.data_ptr()
    assert lib.scion_router_logits_static(p, 65, p, p, 64, 256, p, None) == tq.SCION_EINVAL
    assert lib.scion_router_logits_static(p, 8, p, p, 513, 256, p, None) == tq.SCION_EINVAL
    assert lib.scion_router_logits_static(p, 8, p, p, 64, 4224, p, None) == tq.SCION_EINVAL
    assert lib.scion_router_logits_static(p, 8, p, p, 64, 200, p, None) == tq.SCION_EINVAL
