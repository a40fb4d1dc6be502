"""Expert parallelism through the library on the GPU: the orchestration of
ternary_quantized_moe_b200.ep with the library backend on a one-rank NCCL group (the only layout
one GPU allows: the collectives are identities), against the oracle; the multi-rank logic is
covered on CPU by tests/test_ep_cpu.py and the per-range parts by test_expert_parallel_parts."""
import os
import socket

import numpy as np
import pytest

import oracle
from tests.helpers import check_output, device_layer, oracle_layer_packed, packed_banks, u16_to_dev, with_margin
from workloads import synth

torch = pytest.importorskip("torch")
import ternary_quantized_moe_b200 as tq  # noqa: E402
from ternary_quantized_moe_b200 import ep  # noqa: E402

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("T,max_tokens", [(7, 64), (200, 200)])
def test_expert_parallel_block_one_rank_nccl(T, max_tokens):
    import torch.distributed as dist

    cfg = synth.Config("epg", 44, 256, 16, 4, 128, 128, synth.PTQ1_0, 16, False, [8], 1)
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    ol = oracle_layer_packed(cfg, L, banks)
    x = with_margin(cfg, ol, synth.x_host(cfg, T))
    lo, n = ep.expert_range(cfg.n_experts, 1, 0)
    layer = device_layer(cfg, L, banks, max_tokens, expert_lo=lo, n_local_experts=n)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        out = torch.full((T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        block = ep.ExpertParallelBlock(ep.LibraryBackend(layer), cfg.d)
        block.forward(u16_to_dev(x, torch.bfloat16, "cuda"), out)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref, _, _ = oracle.forward(ol, x)
    check_output(out.cpu().numpy().astype(np.float64), ref)
