"""Shared test helpers: oracle layers from the seeded generator, the top-k margin
filter, and the output tolerance check."""
from __future__ import annotations

import numpy as np

import oracle
from workloads import synth

# Output tolerance of the block: per-token relative L2 error and max-abs error
# relative to the largest reference magnitude.
REL_L2_TOL = 1e-3
MAX_ABS_TOL = 5e-3
# Minimum fp64 gap between the k-th and (k+1)-th logit of every test token, so that
# routing is decided identically by any correct fp32 implementation.
TOPK_MARGIN = 1e-3


def oracle_layer_from(cfg: synth.Config, L: dict, *, norm_topk: int = 1, corr_on_output: int = 0,
                      sh_gate_vec=None) -> oracle.OracleLayer:
    """Pack a generated layer with the oracle's own packer."""
    fmt = cfg.fmt
    return oracle.OracleLayer(
        d=cfg.d, n_experts=cfg.n_experts, top_k=cfg.top_k, ffn=cfg.ffn, fmt=fmt,
        w_router=L["w_router"], w_delta=L["w_delta"],
        gate_exps=oracle.pack(fmt, L["gate_codes"], L["gate_scales"]),
        up_exps=oracle.pack(fmt, L["up_codes"], L["up_scales"]),
        down_exps=oracle.pack(fmt, L["down_codes"], L["down_scales"]),
        shared_ffn=cfg.shared_ffn,
        sh_gate=L.get("sh_gate"), sh_up=L.get("sh_up"), sh_down=L.get("sh_down"),
        sh_gate_vec=sh_gate_vec,
        rank=cfg.rank, corr_a=L.get("corr_a"), corr_b=L.get("corr_b"),
        norm_topk=norm_topk, corr_on_output=corr_on_output,
    )


def topk_gap(logits: np.ndarray, k: int) -> np.ndarray:
    """Per-token fp64 gap between the k-th and (k+1)-th largest logit."""
    s = -np.sort(-logits, axis=1)
    if k >= logits.shape[1]:
        return np.full(logits.shape[0], np.inf)
    return s[:, k - 1] - s[:, k]


def with_margin(cfg: synth.Config, layer: oracle.OracleLayer, x: np.ndarray, margin: float = TOPK_MARGIN,
                seed: int = 12345, max_rounds: int = 50) -> np.ndarray:
    """Replace tokens whose top-k margin (oracle fp64 logits) is below `margin` with fresh
    draws from the generator until every token has the margin."""
    x = x.copy()
    bad = np.arange(x.shape[0])
    for rnd in range(max_rounds):
        logits, _, _ = oracle.route(layer, x[bad])
        gap = topk_gap(logits, cfg.top_k)
        bad = bad[gap < margin]
        if bad.size == 0:
            return x
        x[bad] = synth.x_rows_host(cfg, bad.size, seed + 7919 * rnd)
    raise RuntimeError("could not reach the top-k margin")


def check_output(got: np.ndarray, ref: np.ndarray, rel_l2: float = REL_L2_TOL, max_abs: float = MAX_ABS_TOL):
    """Per-token relative L2 <= rel_l2 and max |got-ref| <= max_abs * max|ref|."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return
    err = np.linalg.norm(got - ref, axis=1)
    nrm = np.linalg.norm(ref, axis=1)
    rel = err / np.maximum(nrm, 1e-300)
    worst = int(np.argmax(rel))
    assert rel.max() <= rel_l2, "token %d: relative L2 %.3e > %.1e" % (worst, rel.max(), rel_l2)
    mx = np.abs(got - ref).max()
    assert mx <= max_abs * np.abs(ref).max(), "max abs %.3e > %.1e * %.3e" % (mx, max_abs, np.abs(ref).max())


def f16(bits: np.ndarray) -> np.ndarray:
    """fp16 bit patterns -> float64 via numpy's float16 (a library routine)."""
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 via torch's bfloat16 (a library routine)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.double().numpy()


# ------------------------------------------------------------ device layers
def packed_banks(cfg: synth.Config, L: dict) -> dict:
    """Expert banks packed by the oracle's packer (the bytes both sides consume)."""
    return {n: oracle.pack(cfg.fmt, L[n + "_codes"], L[n + "_scales"]) for n in ("gate", "up", "down")}


def oracle_layer_packed(cfg: synth.Config, L: dict, banks: dict, **kw) -> oracle.OracleLayer:
    return oracle.OracleLayer(
        d=cfg.d, n_experts=cfg.n_experts, top_k=cfg.top_k, ffn=cfg.ffn, fmt=cfg.fmt,
        w_router=L["w_router"], w_delta=L["w_delta"], gate_exps=banks["gate"], up_exps=banks["up"],
        down_exps=banks["down"], shared_ffn=cfg.shared_ffn, sh_gate=L.get("sh_gate"), sh_up=L.get("sh_up"),
        sh_down=L.get("sh_down"), rank=cfg.rank, corr_a=L.get("corr_a"), corr_b=L.get("corr_b"), **kw)


def u16_to_dev(a, dtype, dev):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dtype).to(dev)


def packed_correction(cfg: synth.Config, seed: int = 55):
    """Ternary correction factors packed as PQ2_0 blocks by the oracle's packer: (A blocks
    [r, d/128*34], B blocks [d, r/128*34])."""
    rng = np.random.default_rng(seed)
    r, d = cfg.rank, cfg.d
    ca, sa = synth.ternary_codes(rng, (r, d)), synth.group_scales(rng, (r, d // 128))
    cb, sb = synth.ternary_codes(rng, (d, r)), synth.group_scales(rng, (d, r // 128))
    return oracle.pack(synth.PQ2_0, ca, sa), oracle.pack(synth.PQ2_0, cb, sb)


def device_layer(cfg: synth.Config, L: dict, banks: dict, max_tokens: int, dev="cuda", norm_topk: int = 1,
                 packed_corr=None, expert_lo: int = 0, n_local_experts: int = 0):
    import torch

    import ternary_quantized_moe_b200 as tq

    bf = torch.bfloat16
    if L["w_router"].dtype == np.float32:
        wr = torch.from_numpy(L["w_router"]).to(dev)
        wd = torch.from_numpy(L["w_delta"]).to(dev)
    else:
        wr = u16_to_dev(L["w_router"], bf, dev)
        wd = u16_to_dev(L["w_delta"], bf, dev)
    opt = lambda n: u16_to_dev(L[n], bf, dev) if n in L else None  # noqa: E731
    return tq.scion_layer_create(
        d=cfg.d, n_experts=cfg.n_experts, top_k=cfg.top_k, ffn=cfg.ffn, fmt=cfg.fmt, w_router=wr, w_router_delta=wd,
        gate_exps=torch.from_numpy(banks["gate"]).to(dev), up_exps=torch.from_numpy(banks["up"]).to(dev),
        down_exps=torch.from_numpy(banks["down"]).to(dev), shared_ffn=cfg.shared_ffn, sh_gate=opt("sh_gate"),
        sh_up=opt("sh_up"), sh_down=opt("sh_down"), rank=cfg.rank,
        corr_a=torch.from_numpy(packed_corr[0]).to(dev) if packed_corr else opt("corr_a"),
        corr_b=torch.from_numpy(packed_corr[1]).to(dev) if packed_corr else opt("corr_b"),
        corr_packed=1 if packed_corr else 0, norm_topk=norm_topk, max_tokens=max_tokens, expert_lo=expert_lo,
        n_local_experts=n_local_experts)


def range_mix(cfg: synth.Config, layer: oracle.OracleLayer, x: np.ndarray, seed: int = 4711) -> np.ndarray:
    """Activations far from N(0, 1), built from margin-filtered tokens x (bf16 bits): token t gets
    kind (t + 1) % 5 --
      0  unchanged (N(0, 1));
      1  four channels replaced by outliers of magnitude 1e2 .. 3e4 (log-uniform, random sign);
      2  the whole token times 2^-20 (values near 1e-6);
      3  the whole token times 2^8 (rms 256, max near 1e3);
      4  a hundred channels replaced by values near 1e-6.
    Power-of-two scalings are exact in bf16 and leave the fp64 logits scaled by the same factor,
    so those tokens keep their (relative) top-k margin; the outlier tokens are redrawn until their
    fp64 top-k gap is at least the absolute margin."""
    rng = np.random.default_rng(seed)
    xf = bf16(x).astype(np.float32)
    out = xf.copy()
    for t in range(x.shape[0]):
        kind = (t + 1) % 5
        if kind == 1:
            for _ in range(50):
                row = xf[t].copy()
                ch = rng.choice(cfg.d, 4, replace=False)
                row[ch] = (np.exp(rng.uniform(np.log(1e2), np.log(3e4), 4)) * rng.choice([-1.0, 1.0], 4))
                logits, _, _ = oracle.route(layer, synth.to_bf16_bits(row[None]))
                if topk_gap(logits, cfg.top_k)[0] >= TOPK_MARGIN:
                    out[t] = row
                    break
            else:
                raise RuntimeError("no outlier token with the top-k margin")
        elif kind == 2:
            out[t] = xf[t] * np.float32(2.0 ** -20)
        elif kind == 3:
            out[t] = xf[t] * np.float32(2.0 ** 8)
        elif kind == 4:
            ch = rng.choice(cfg.d, 100, replace=False)
            out[t, ch] = rng.standard_normal(100).astype(np.float32) * np.float32(1e-6)
    return synth.to_bf16_bits(out)
