"""Expert parallelism on CPU (gloo, two and three ranks): the orchestration of
ternary_quantized_moe_b200.ep -- all-gather of the ranks' tokens, the routed part of each rank's
expert range, reduce-scatter, the dense part of each rank's own tokens -- with the oracle's parts
as the per-rank compute, against the oracle's block forward over all tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg():
    from workloads import synth

    return synth.Config("epc", 43, 256, 12, 3, 128, 128, synth.PQ2_0, 16, False, [8], 1)


class OracleBackend:
    """A rank's two forwards computed by the oracle: the routed part of experts [lo, lo + n) and
    the dense part, on bf16 bit patterns."""

    def __init__(self, ol, lo, n):
        self.ol, self.lo, self.n = ol, lo, n

    def routed(self, x_all, out_all):
        import oracle

        x = x_all.view(torch.int16).numpy().view(np.uint16)
        out_all.copy_(torch.from_numpy(oracle.forward_part(self.ol, x, self.lo, self.n, oracle.ROUTED)))

    def dense_add(self, x, out):
        import oracle

        xb = x.view(torch.int16).numpy().view(np.uint16)
        out.add_(torch.from_numpy(oracle.forward_part(self.ol, xb, 0, 0, oracle.DENSE)))


def _worker(rank, world, port, T, results):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from tests.helpers import oracle_layer_from
    from ternary_quantized_moe_b200 import ep
    from workloads import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = _cfg()
        ol = oracle_layer_from(cfg, synth.layer_host(cfg))
        lo, n = ep.expert_range(cfg.n_experts, world, rank)
        x_np = synth.x_host(cfg, T, stream=rank)  # this rank's tokens
        x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16)
        out = torch.empty((T, cfg.d), dtype=torch.float32)
        ep.ExpertParallelBlock(OracleBackend(ol, lo, n), cfg.d).forward(x, out)
        results[rank] = (lo, n, x_np, out.double().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_block_gloo(world):
    import oracle
    from tests.helpers import oracle_layer_from
    from ternary_quantized_moe_b200 import ep
    from workloads import synth

    T, port = 5, _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, T, results), nprocs=world, join=True)
        got = dict(results)
    cfg = _cfg()
    ol = oracle_layer_from(cfg, synth.layer_host(cfg))
    ranges = [got[r][:2] for r in range(world)]
    assert ranges == [ep.expert_range(cfg.n_experts, world, r) for r in range(world)]
    assert sum(n for _, n in ranges) == cfg.n_experts
    for r in range(world):
        x = got[r][2]
        ref, _, _ = oracle.forward(ol, x)
        # fp32 transport of the routed parts: agreement to fp32 rounding
        np.testing.assert_allclose(got[r][3], ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


def test_expert_range_covers_the_experts():
    from ternary_quantized_moe_b200 import ep

    for E, world in ((256, 8), (10, 3), (7, 7), (512, 6)):
        spans = [ep.expert_range(E, world, r) for r in range(world)]
        assert spans[0][0] == 0 and sum(n for _, n in spans) == E
        assert all(spans[i][0] + spans[i][1] == spans[i + 1][0] for i in range(world - 1))
        assert max(n for _, n in spans) - min(n for _, n in spans) <= 1
    with pytest.raises(ValueError):
        ep.expert_range(4, 5, 0)
