"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same
seeded inputs.  Integer work (packing, routing ids, counts, offsets, the grouping
permutation) must match bit for bit; floating-point outputs must meet the block
tolerance (per-token relative L2 <= 1e-3, max-abs <= 5e-3 * max|ref|)."""
import numpy as np
import pytest

import oracle
from tests.helpers import (TOPK_MARGIN, bf16, check_output, device_layer, oracle_layer_packed, packed_banks,
                           packed_correction, range_mix, topk_gap, u16_to_dev, with_margin)
from workloads import synth

torch = pytest.importorskip("torch")
import ternary_quantized_moe_b200 as tq  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"


def small(name, fmt, router_f32, E=16, k=4, d=256, F=128, Fs=128, r=16, index=20):
    return synth.Config(name, index, d, E, k, F, Fs, fmt, r, router_f32, [8], 1)


def run_forward(layer, x_u16, T, debug=False, E=None, k=None, F=None, Kdense=None):
    x = u16_to_dev(x_u16, torch.bfloat16, DEV)
    out = torch.full((max(T, 1), layer.d), float("nan"), dtype=torch.float32, device=DEV)
    bufs = {}
    if debug:
        bufs = dict(
            logits=torch.empty((T, E), dtype=torch.float32, device=DEV),
            ids=torch.empty((T, k), dtype=torch.int32, device=DEV),
            gates=torch.empty((T, k), dtype=torch.float32, device=DEV),
            counts=torch.empty((E,), dtype=torch.int32, device=DEV),
            offsets=torch.empty((E + 1,), dtype=torch.int32, device=DEV),
            perm=torch.empty((T * k,), dtype=torch.int32, device=DEV),
            h=torch.empty((T * k, F), dtype=torch.float16, device=DEV),
        )
        if Kdense:
            bufs["hz"] = torch.empty((T, Kdense), dtype=torch.float16, device=DEV)
        tq.scion_moe_forward_debug(x, T, layer, out, **bufs)
    else:
        tq.scion_moe_forward(x, T, layer, out)
    torch.cuda.synchronize()
    return out[:T].cpu().numpy().astype(np.float64), {k_: v.cpu().numpy() for k_, v in bufs.items()}


# ------------------------------------------------------------------ formats
@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("n_groups", [1, 37, 1001])
def test_device_pack_unpack_match_oracle(fmt, n_groups):
    rng = np.random.default_rng(n_groups)
    codes = rng.integers(-1, 2, size=(n_groups, 128)).astype(np.int8)
    scales = rng.integers(0, 1 << 16, size=(n_groups, 1)).astype(np.uint16)
    ref = oracle.pack(fmt, codes, scales)
    dc = torch.from_numpy(codes).to(DEV)
    ds = torch.from_numpy(scales.view(np.int16)).to(DEV)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    blocks = tq.scion_pack_device(fmt, dc, ds, bad_count=bad)
    np.testing.assert_array_equal(blocks.cpu().numpy(), ref)
    assert int(bad.item()) == 0
    c2, s2 = tq.scion_unpack_device(fmt, torch.from_numpy(ref).to(DEV), bad_count=bad)
    np.testing.assert_array_equal(c2.cpu().numpy(), codes)
    np.testing.assert_array_equal(s2.cpu().numpy().view(np.uint16), scales)
    assert int(bad.item()) == 0


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
def test_device_unpack_counts_invalid_codes(fmt):
    blk = oracle.pack(fmt, np.zeros((4, 128), np.int8), np.zeros((4, 1), np.uint16))
    blk[1, 0] = 0xFF  # PQ2: four fields of 3; PTQ1: one quintet byte above 242
    if fmt == synth.PTQ1_0:
        blk[2, 25] = 27  # tail byte above 26
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    codes, _ = tq.scion_unpack_device(fmt, torch.from_numpy(blk).to(DEV), bad_count=bad)
    ref_codes, _, st = oracle.unpack(fmt, blk)
    assert st == oracle.EFORMAT
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    assert int(bad.item()) == (4 if fmt == synth.PQ2_0 else 2)


def test_device_pack_counts_out_of_range_codes():
    codes = np.zeros((2, 128), np.int8)
    codes[0, 5] = 3
    codes[1, 7] = -4
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    tq.scion_pack_device(synth.PQ2_0, torch.from_numpy(codes).to(DEV),
                         torch.zeros((2, 1), dtype=torch.int16, device=DEV), bad_count=bad)
    assert int(bad.item()) == 2


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
def test_create_rejects_invalid_bank(fmt):
    cfg = small("bad", fmt, False)
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    banks["down"] = banks["down"].copy()
    banks["down"][3, 17, 5] = 0xFF
    with pytest.raises(tq.ScionError) as ei:
        device_layer(cfg, L, banks, 8)
    assert ei.value.status == tq.SCION_EFORMAT


# ------------------------------------------------------------------ forward
def _case(cfg, T, norm_topk=1, stream=0):
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    ol = oracle_layer_packed(cfg, L, banks, norm_topk=norm_topk)
    x = synth.x_host(cfg, T, stream)
    if T:
        x = with_margin(cfg, ol, x)
    return L, banks, ol, x


def _check_routing(cfg, dbg, ol, x, T, stable=True, gate_rtol=1e-5):
    """stable: the permutation must be the oracle's stable (token, slot) order (decode path);
    otherwise (tensor-core path, whose grouping takes positions atomically) each expert's
    segment must hold exactly the oracle's entries, in any order.  gate_rtol: relative gate
    error allowed; a gate's relative error is about the absolute fp32 error of the logit
    differences, which grows with the logits' magnitude."""
    E, k = cfg.n_experts, cfg.top_k
    logits, ids, gates = oracle.route(ol, x)
    np.testing.assert_allclose(dbg["logits"], logits, rtol=0, atol=2e-4 * max(1.0, np.abs(logits).max()))
    np.testing.assert_array_equal(np.sort(dbg["ids"], 1), np.sort(ids, 1))
    # gates per (token, expert)
    for t in range(T):
        ref = dict(zip(ids[t].tolist(), gates[t].tolist()))
        for j in range(k):
            assert abs(dbg["gates"][t, j] - ref[int(dbg["ids"][t, j])]) <= gate_rtol * max(1e-3, ref[int(dbg["ids"][t, j])])
    counts, offsets, perm = oracle.group(ids, E)
    np.testing.assert_array_equal(dbg["counts"], counts)
    np.testing.assert_array_equal(dbg["offsets"], offsets)
    gp = dbg["perm"]
    if stable:
        # within each expert the tokens appear in increasing token order (unique)
        np.testing.assert_array_equal(gp // k, perm // k)
    else:
        np.testing.assert_array_equal(np.sort(gp), np.arange(T * k))  # a permutation
        for e in range(E):
            np.testing.assert_array_equal(np.sort(gp[offsets[e]:offsets[e + 1]] // k),
                                          np.sort(perm[offsets[e]:offsets[e + 1]] // k))
    # the slot part of each entry must point at that expert in the GPU's own ids
    for e in range(E):
        seg = gp[offsets[e]:offsets[e + 1]]
        assert (dbg["ids"].reshape(-1)[seg] == e).all()
    return ids


def _check_hidden(cfg, dbg, ol, x, T):
    """Expert SwiGLU hidden of every routed (token, expert) pair vs the oracle."""
    k = cfg.top_k
    worst = 0.0
    for p, entry in enumerate(dbg["perm"]):
        t, j = divmod(int(entry), k)
        e = int(dbg["ids"][t, j])
        h_ref, _ = oracle.expert(ol, e, x[t])
        got = dbg["h"][p].astype(np.float64)
        worst = max(worst, np.linalg.norm(got - h_ref) / max(np.linalg.norm(h_ref), 1e-30))
    assert worst <= 1e-3, worst


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("router_f32", [True, False])
@pytest.mark.parametrize("T", [1, 5, 13])
def test_forward_small_stagewise(fmt, router_f32, T):
    cfg = small("s", fmt, router_f32)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, 64)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    _check_routing(cfg, dbg, ol, x, T)
    _check_hidden(cfg, dbg, ol, x, T)
    hs, _ = oracle.shared(ol, x)
    z, _ = oracle.corr(ol, x)
    hz_ref = np.concatenate([hs, z], axis=1)
    check_output(dbg["hz"].astype(np.float64), hz_ref, rel_l2=1e-3)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("variant", ["tiny", "no_shared_no_corr", "norm_topk0", "k_eq_E", "E_not_mult16",
                                     "wide_d", "ptq1_F384"])
def test_forward_variants(variant):
    T, norm_topk = 16, 1
    if variant == "tiny":
        cfg = synth.CONFIGS["tiny"]
    elif variant == "no_shared_no_corr":
        cfg = small("v", synth.PQ2_0, False, Fs=0, r=0)
    elif variant == "norm_topk0":
        cfg, norm_topk = small("v", synth.PTQ1_0, False), 0
    elif variant == "k_eq_E":
        cfg = small("v", synth.PQ2_0, True, E=4, k=4)
    elif variant == "E_not_mult16":
        cfg = small("v", synth.PTQ1_0, False, E=24, k=3)
    elif variant == "wide_d":
        cfg = small("v", synth.PQ2_0, False, d=1152, F=256, Fs=256, r=48, E=32, k=6)
    else:
        cfg = small("v", synth.PTQ1_0, False, d=384, F=384, Fs=384, r=32, E=16, k=2)
    L, banks, ol, x = _case(cfg, T, norm_topk)
    layer = device_layer(cfg, L, banks, 64, norm_topk=norm_topk)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    _check_routing(cfg, dbg, ol, x, T)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("dense", ["shared_only", "corr_only"])
@pytest.mark.parametrize("T,max_tokens", [(1, 64), (13, 64), (40, 64), (200, 200)])
def test_forward_one_dense_part(fmt, dense, T, max_tokens):
    """A shared expert without a correction (the shared hidden then stored times 2^(2 s_t)) and a
    correction without a shared expert (z times 2^(s_t)), with range-scaled tokens, on the
    split-K, ring and tensor-core paths, at the 35B-A3B-class widths (d 2048, ffn 512)."""
    Fs, r = (512, 0) if dense == "shared_only" else (0, 512)
    cfg = small("od", fmt, False, E=16, k=4, d=2048, F=512, Fs=Fs, r=r)
    L, banks, ol, x = _case(cfg, T)
    x = range_mix(cfg, ol, x)
    layer = device_layer(cfg, L, banks, max_tokens)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    assert tq.scion_layer_check(layer) == 0
    assert np.isfinite(got).all()
    _, ids, _ = oracle.route(ol, x)
    np.testing.assert_array_equal(np.sort(dbg["ids"], 1), np.sort(ids, 1))
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("T,max_tokens", [(40, 64), (200, 200)])
def test_forward_narrow_correction_only(fmt, T, max_tokens):
    """A narrow layer (d 256, ffn 128) with a correction and no shared expert, on range-scaled
    tokens whose energy sits in a few outlier channels: their scaled expert hidden is small, and
    the tensor-core path keeps it out of the fp16 subnormals (no position factor on its operands)."""
    cfg = small("od", fmt, False, E=16, k=4, Fs=0, r=128)
    L, banks, ol, x = _case(cfg, T)
    x = range_mix(cfg, ol, x)
    layer = device_layer(cfg, L, banks, max_tokens)
    got, _ = run_forward(layer, x, T)
    assert tq.scion_layer_check(layer) == 0
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("E,k,T,norm_topk,max_tokens", [(64, 32, 1, 1, 64), (64, 32, 13, 0, 64), (64, 32, 64, 1, 64),
                                                       (512, 32, 40, 1, 64), (64, 32, 200, 0, 200),
                                                       (512, 32, 200, 1, 200)])
def test_forward_widest_topk(E, k, T, norm_topk, max_tokens):
    """k = 32 (the largest top-k the descriptor accepts) with E <= 512: the decode routing kernels
    (one CTA, and the multi-CTA form above 32 tokens) and the prefill top-k, both gate
    normalisations; routing bit-exact, output within the block tolerance."""
    cfg = small("wk", synth.PQ2_0 if E == 64 else synth.PTQ1_0, False, E=E, k=k)
    L, banks, ol, x = _case(cfg, T, norm_topk)
    layer = device_layer(cfg, L, banks, max_tokens, norm_topk=norm_topk)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    _check_routing(cfg, dbg, ol, x, T, stable=T <= 64)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("shape", ["d_max", "d_min"])
@pytest.mark.parametrize("T", [1, 16, 64, 100])
def test_forward_extreme_widths(fmt, shape, T):
    """The widest block the decode x-projection takes (d = 4096: eight 512-column chunks in one
    cluster) with the narrowest expert (F = 128: one group along the down projection's K) and
    k = 1, and the narrowest block (d = 128: one group along every gate/up row), on the split-K,
    ring and tensor-core paths (max_tokens = 128)."""
    if shape == "d_max":
        cfg = small("xw", fmt, False, E=8, k=1, d=4096, F=128, Fs=128, r=16)
    else:
        cfg = small("xn", fmt, False, E=8, k=2, d=128, F=128, Fs=128, r=16)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, 128)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    _check_routing(cfg, dbg, ol, x, T, stable=T <= 64)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("tc", [0, 1])
@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (5, 16, 4), (13, 16, 4), (64, 16, 4), (64, 4, 2), (37, 6, 3)])
def test_forward_stream_kernels(tc, fmt, T, E, k):
    """The persistent expert kernels of decode batches (selected for every batch size with
    SCION_OPT_STREAM_MIN_TOKENS = 1): tc = 1 the tcgen05 grouped GEMMs (one tile per active
    expert, 16-row boxes of the hidden, gate-weighted reductions into out), tc = 0 the mma.sync
    kernels fed by a bulk-copy ring (experts with more than one 8-token pass); stage by stage
    against the oracle, experts with up to 64 tokens (E = 4, k = 2)."""
    cfg = small("st", fmt, False, E=E, k=k)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, 64)
    tq.scion_layer_set_option(layer, tq.SCION_OPT_STREAM_MIN_TOKENS, 1)
    tq.scion_layer_set_option(layer, tq.SCION_OPT_DECODE_TC, tc)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    _check_routing(cfg, dbg, ol, x, T)
    _check_hidden(cfg, dbg, ol, x, T)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("E,k,T", [(64, 4, 5), (256, 8, 13), (512, 10, 5), (512, 10, 40), (256, 8, 200),
                                   (512, 10, 300)])
def test_topk_one_lane_holds_the_top(E, k, T):
    """Router rows built so that the experts e = 5 (mod 32), all held by one lane of the top-k
    warp, take most or all of the top k: that lane's candidate list runs dry and is refilled
    (decode single-CTA and multi-CTA routing, prefill top-k)."""
    cfg = small("tk", synth.PQ2_0, False, E=E, k=k, Fs=0, r=16)
    L = synth.layer_host(cfg)
    wr = bf16(L["w_router"]).astype(np.float32)
    hot = np.arange(5, E, 32)
    wr[hot, 0] = 8.0 + np.arange(hot.size, dtype=np.float32)  # exact in bf16
    L["w_router"] = synth.to_bf16_bits(wr)
    banks = packed_banks(cfg, L)
    ol = oracle_layer_packed(cfg, L, banks)
    x = synth.x_host(cfg, 4 * T)
    x[:, 0] = 0x3F80  # 1.0
    logits, ids, _ = oracle.route(ol, x)
    keep = topk_gap(logits, k) >= TOPK_MARGIN
    x, ids = x[keep][:T], ids[keep][:T]
    assert x.shape[0] == T
    assert (ids % 32 == 5).sum() >= min(k, hot.size) * T  # the hot lane holds the top
    layer = device_layer(cfg, L, banks, 64 if T <= 64 else T)
    got, dbg = run_forward(layer, x, T, debug=True, E=E, k=k, F=cfg.ffn, Kdense=cfg.shared_ffn + cfg.rank)
    # logits up to ~25 here (about 8x the standard cases): the gate bound scales with them
    _check_routing(cfg, dbg, ol, x, T, stable=T <= 64, gate_rtol=1e-4)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("T,max_tokens,dense,in_place", [(5, 64, True, False), (40, 64, True, True),
                                                          (64, 64, False, True), (150, 150, True, False),
                                                          (300, 300, False, True), (300, 300, True, True)])
def test_forward_residual(T, max_tokens, dense, in_place):
    """out = resid + block(x) on the decode kernels (split-K and ring passes) and the
    tensor-core path (with and without the shared expert and correction, whose dense down
    projection adds the residual; without them the combine does), in place and not."""
    cfg = small("rs", synth.PTQ1_0, False, E=16, k=4, Fs=128 if dense else 0, r=16 if dense else 0)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, max_tokens)
    rng = np.random.default_rng(77 + T)
    resid_h = rng.standard_normal((T, cfg.d)).astype(np.float32)
    resid = torch.from_numpy(resid_h).to(DEV)
    out = resid if in_place else torch.full((T, cfg.d), float("nan"), dtype=torch.float32, device=DEV)
    tq.scion_moe_forward_residual(u16_to_dev(x, torch.bfloat16, DEV), T, layer, resid, out)
    torch.cuda.synchronize()
    assert tq.scion_layer_check(layer) == 0
    if not in_place:
        np.testing.assert_array_equal(resid.cpu().numpy(), resid_h)  # only read
    ref, _, _ = oracle.forward(ol, x)
    check_output(out.cpu().numpy().astype(np.float64) - resid_h.astype(np.float64), ref)


@pytest.mark.parametrize("fmt,T,max_tokens", [(synth.PQ2_0, 5, 64), (synth.PTQ1_0, 13, 64), (synth.PQ2_0, 40, 64),
                                              (synth.PTQ1_0, 64, 64), (synth.PQ2_0, 200, 200),
                                              (synth.PTQ1_0, 300, 300)])
def test_forward_packed_correction(fmt, T, max_tokens):
    """Ternary correction factors in PQ2_0 blocks: decode (split-K and ring passes; A read from
    its blocks) and the tensor-core path (exact fp16 copies) against the oracle on the same
    packed bytes, with the stage outputs z (hz) checked too."""
    cfg = small("pc", fmt, False, E=16, k=4, Fs=128, r=256)
    L, banks, ol, x = _case(cfg, T)
    pa, pb = packed_correction(cfg)
    ol.corr_a, ol.corr_b, ol.corr_packed = pa, pb, 1
    x = with_margin(cfg, ol, x)
    layer = device_layer(cfg, L, banks, max_tokens, packed_corr=(pa, pb))
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    assert tq.scion_layer_check(layer) == 0
    hs, _ = oracle.shared(ol, x)
    z, _ = oracle.corr(ol, x)
    check_output(dbg["hz"].astype(np.float64), np.concatenate([hs, z], axis=1), rel_l2=1e-3)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("T,max_tokens", [(5, 64), (40, 64), (300, 300)])
def test_forward_packed_correction_activation_range(T, max_tokens):
    """Ternary correction factors with activations far outside N(0, 1) (outlier channels, tokens
    near 1e-6 or scaled by 256): the correction units read A from its blocks and scale z by the
    token's range exponent (decode), or use the exact fp16 copies (tensor-core path)."""
    cfg = small("pcr", synth.PQ2_0, False, E=16, k=4, Fs=128, r=256)
    L, banks, ol, x = _case(cfg, T)
    pa, pb = packed_correction(cfg)
    ol.corr_a, ol.corr_b, ol.corr_packed = pa, pb, 1
    x = range_mix(cfg, ol, with_margin(cfg, ol, x))
    layer = device_layer(cfg, L, banks, max_tokens, packed_corr=(pa, pb))
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    assert tq.scion_layer_check(layer) == 0
    assert np.isfinite(got).all()
    _, ids, _ = oracle.route(ol, x)
    np.testing.assert_array_equal(np.sort(dbg["ids"], 1), np.sort(ids, 1))
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


def test_packed_correction_rejects_invalid_codes_and_rank():
    cfg = small("pcx", synth.PQ2_0, False, E=16, k=4, Fs=128, r=256)
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    pa, pb = packed_correction(cfg)
    bad = pb.copy()
    bad[3, 5] = 0xFF  # four invalid fields
    with pytest.raises(tq.ScionError) as ei:
        device_layer(cfg, L, banks, 64, packed_corr=(pa, bad))
    assert ei.value.status == tq.SCION_EFORMAT
    cfg2 = small("pcr", synth.PQ2_0, False, E=16, k=4, Fs=128, r=16)
    L2 = synth.layer_host(cfg2)
    with pytest.raises(tq.ScionError) as ei:  # rank must be a multiple of 128 for packed factors
        device_layer(cfg2, L2, packed_banks(cfg2, L2), 64, packed_corr=packed_correction(cfg))
    assert ei.value.status == tq.SCION_EINVAL


@pytest.mark.parametrize("T", [64, 65, 150])
def test_forward_across_the_decode_limit(T):
    """One layer built for up to 160 tokens: T = 64 runs the decode kernels, T = 65 and 150 (one
    token past the limit, and a ragged 150) the tensor-core path; both against the oracle."""
    cfg = small("mp", synth.PTQ1_0, False, E=32, k=4)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, 160)
    got, _ = run_forward(layer, x, T)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("E,k,T", [(1024, 8, 1), (1024, 8, 13), (1024, 8, 64),
                                   pytest.param(4096, 32, 64, marks=pytest.mark.slow)])
def test_forward_decode_many_experts(E, k, T):
    """Decode routing for more than 512 experts (the single-CTA grouping kernel with the logits
    staged per warp in shared memory, then the slot records): ids, counts, offsets and the stable
    permutation bit-exact, gates, hidden and output within tolerance; E = 4096 with k = 32 is the
    largest layer the decode path accepts."""
    cfg = small("me", synth.PQ2_0, False, E=E, k=k, d=256, F=128, Fs=128, r=16)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, 64)
    del L, banks
    got, dbg = run_forward(layer, x, T, debug=True, E=E, k=k, F=cfg.ffn, Kdense=cfg.shared_ffn + cfg.rank)
    assert tq.scion_layer_check(layer) == 0
    _check_routing(cfg, dbg, ol, x, T)
    _check_hidden(cfg, dbg, ol, x, T)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("shape", ["a3b", "flashnext"])
@pytest.mark.parametrize("T", [1, 13, 64, 300])
def test_forward_activation_range(shape, T):
    """Activations far outside N(0, 1) -- outlier channels up to 3e4, whole tokens near 1e-6 or
    scaled by 256, tiny channels inside ordinary tokens -- through the decode kernels (T <= 64:
    split-K and ring passes) and the tensor-core path (T = 300), with the 35B-A3B-class (d 2048,
    ffn 512, PQ2_0, shared expert, rank 512) and FlashNext-class (d 3072, ffn 768, PTQ1_0) layer
    widths (32 experts).  Routing bit-exact, output within the block tolerance per token."""
    if shape == "a3b":
        cfg = small("ra", synth.PQ2_0, False, E=32, k=8, d=2048, F=512, Fs=512, r=512)
    else:
        cfg = small("rf", synth.PTQ1_0, False, E=32, k=10, d=3072, F=768, Fs=768, r=512)
    L, banks, ol, x = _case(cfg, T)
    x = range_mix(cfg, ol, x)
    layer = device_layer(cfg, L, banks, max(T, 64))
    del L, banks
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    assert tq.scion_layer_check(layer) == 0
    assert np.isfinite(got).all()
    _, ids, _ = oracle.route(ol, x)
    np.testing.assert_array_equal(np.sort(dbg["ids"], 1), np.sort(ids, 1))
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("packed", [0, 1])
@pytest.mark.parametrize("T,max_tokens,in_place", [(1, 64, False), (13, 64, True), (64, 64, False),
                                                   (300, 300, False), (300, 300, True)])
def test_attn_out_correction(packed, T, max_tokens, in_place):
    """The correction branch on the attention output, out = base + B (A v), with d_in != d_out:
    decode kernels (T <= 64) and tcgen05 GEMMs (T = 300), bf16 and PQ2_0 factors, in place and
    not, on activations that include tokens scaled by 2^-20 and 2^8 and outlier channels.  The
    branch (out - base) must meet the block tolerance against the oracle."""
    d_in, d_out, r = 1024, 512, 256
    rng = np.random.default_rng(91 + T + packed)
    if packed:
        ca, sa = synth.ternary_codes(rng, (r, d_in)), synth.group_scales(rng, (r, d_in // 128))
        cb, sb = synth.ternary_codes(rng, (d_out, r)), synth.group_scales(rng, (d_out, r // 128))
        a, b = oracle.pack(synth.PQ2_0, ca, sa), oracle.pack(synth.PQ2_0, cb, sb)
        ad, bd = torch.from_numpy(a).to(DEV), torch.from_numpy(b).to(DEV)
    else:
        a, b = synth.normal_bf16(rng, (r, d_in), 0.02), synth.normal_bf16(rng, (d_out, r), 0.02)
        ad, bd = u16_to_dev(a, torch.bfloat16, DEV), u16_to_dev(b, torch.bfloat16, DEV)
    vf = rng.standard_normal((T, d_in)).astype(np.float32)
    for t in range(T):
        kind = t % 4
        if kind == 1:
            vf[t] *= np.float32(2.0 ** -20)
        elif kind == 2:
            vf[t] *= np.float32(2.0 ** 8)
        elif kind == 3:
            vf[t, rng.choice(d_in, 3, replace=False)] = np.float32(2e4)
    v = synth.to_bf16_bits(vf)
    # base rows of the branch's own magnitude (a fp32 sum cannot hold a branch far below its base)
    br, _ = oracle.attn_corr(v, a, b, d_in, d_out, r, packed=packed)
    base = rng.standard_normal((T, d_out)) * np.sqrt((br ** 2).mean(axis=1, keepdims=True))
    base = base.astype(np.float32).astype(np.float64)
    ref, _ = oracle.attn_corr(v, a, b, d_in, d_out, r, packed=packed, base=base)
    h = tq.scion_corr_create(d_in, d_out, r, ad, bd, packed=packed, max_tokens=max_tokens)
    base_d = torch.from_numpy(base.astype(np.float32)).to(DEV)
    out = base_d if in_place else torch.full((T, d_out), float("nan"), dtype=torch.float32, device=DEV)
    tq.scion_corr_forward(u16_to_dev(v, torch.bfloat16, DEV), T, h, out, base=base_d)
    torch.cuda.synchronize()
    assert tq.scion_corr_check(h) == 0
    got = out.cpu().numpy().astype(np.float64)
    check_output(got - base, ref - base)


def test_attn_out_correction_rejects_bad_descriptors():
    dummy = torch.zeros(1 << 16, dtype=torch.bfloat16, device=DEV)
    for d_in, d_out, r, packed in [(1000, 512, 256, 0), (1024, 500, 256, 0), (1024, 512, 8, 0), (1024, 512, 64, 1),
                                   (8192, 512, 64, 0)]:
        with pytest.raises(tq.ScionError) as ei:
            tq.scion_corr_create(d_in, d_out, r, dummy, dummy, packed=packed)
        assert ei.value.status == tq.SCION_EINVAL


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("T,max_tokens", [(5, 64), (40, 64), (300, 300)])
def test_expert_parallel_parts(fmt, T, max_tokens):
    """The parts of an expert-parallel layout on one GPU: three handles holding experts [0, 10),
    [10, 18) and [18, 24) of a 24-expert layer (their slices of the banks), each computing its
    routed part (SCION_OPT_PARTS), and one dense part (shared expert + correction).  Each part
    against the oracle's part, their sum against the block (decode split-K and ring passes, the
    tensor-core path)."""
    cfg = small("ep", fmt, False, E=24, k=4)
    L, banks, ol, x = _case(cfg, T)
    full, _, _ = oracle.forward(ol, x)
    scale = np.linalg.norm(full, axis=1, keepdims=True)
    total = np.zeros_like(full)
    for lo, n in ((0, 10), (10, 8), (18, 6)):
        part_banks = {name: np.ascontiguousarray(banks[name][lo:lo + n]) for name in banks}
        layer = device_layer(cfg, L, part_banks, max_tokens, expert_lo=lo, n_local_experts=n)
        tq.scion_layer_set_option(layer, tq.SCION_OPT_PARTS, tq.SCION_PART_ROUTED)
        got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn)
        ref = oracle.forward_part(ol, x, lo, n, oracle.ROUTED)
        assert (np.linalg.norm(got - ref, axis=1, keepdims=True) <= 1e-3 * scale).all()
        # the grouping holds exactly the entries of the local experts (local indices)
        _, ids, _ = oracle.route(ol, x)
        loc = ids[(ids >= lo) & (ids < lo + n)] - lo
        np.testing.assert_array_equal(dbg["counts"][:n], np.bincount(loc, minlength=n))
        total += got
    layer = device_layer(cfg, L, banks, max_tokens)
    tq.scion_layer_set_option(layer, tq.SCION_OPT_PARTS, tq.SCION_PART_DENSE)
    dense, _ = run_forward(layer, x, T)
    check_output(dense, oracle.forward_part(ol, x, 0, 0, oracle.DENSE))
    check_output(total + dense, full)


def test_expert_range_rejects_bad_descriptors():
    cfg = small("epx", synth.PQ2_0, False, E=16, k=4)
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    for lo, n in ((3, 0), (-1, 4), (10, 8)):
        with pytest.raises(tq.ScionError) as ei:
            device_layer(cfg, L, banks, 64, expert_lo=lo, n_local_experts=n)
        assert ei.value.status == tq.SCION_EINVAL


@pytest.mark.parametrize("T,max_tokens", [(13, 64), (200, 200)])
def test_debug_route_matches_oracle(T, max_tokens):
    """scion_debug_route (the routing alone): ids as sets per token, offsets and the grouping
    bit-exact against the oracle, gates within the gate tolerance (decode and tensor-core path)."""
    cfg = small("dr", synth.PTQ1_0, False, E=32, k=4)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, max_tokens)
    ids = torch.empty((T, cfg.top_k), dtype=torch.int32, device=DEV)
    gates = torch.empty((T, cfg.top_k), dtype=torch.float32, device=DEV)
    offsets = torch.empty((cfg.n_experts + 1,), dtype=torch.int32, device=DEV)
    perm = torch.empty((T * cfg.top_k,), dtype=torch.int32, device=DEV)
    tq.scion_debug_route(u16_to_dev(x, torch.bfloat16, DEV), T, layer, ids=ids, gates=gates, offsets=offsets,
                         perm=perm)
    torch.cuda.synchronize()
    _, rids, rgates = oracle.route(ol, x)
    gi, gg = ids.cpu().numpy(), gates.cpu().numpy()
    np.testing.assert_array_equal(np.sort(gi, 1), np.sort(rids, 1))
    for t in range(T):
        ref = dict(zip(rids[t].tolist(), rgates[t].tolist()))
        for j in range(cfg.top_k):
            assert abs(gg[t, j] - ref[int(gi[t, j])]) <= 1e-5 * ref[int(gi[t, j])]
    _, roff, rperm = oracle.group(rids, cfg.n_experts)
    np.testing.assert_array_equal(offsets.cpu().numpy(), roff)
    gp = perm.cpu().numpy()
    for e in range(cfg.n_experts):
        np.testing.assert_array_equal(np.sort(gp[roff[e]:roff[e + 1]] // cfg.top_k),
                                      np.sort(rperm[roff[e]:roff[e + 1]] // cfg.top_k))
        assert (gi.reshape(-1)[gp[roff[e]:roff[e + 1]]] == e).all()


def test_empty_batch_and_limits():
    cfg = small("e", synth.PQ2_0, False)
    L, banks, ol, x = _case(cfg, 4)
    layer = device_layer(cfg, L, banks, 4)
    out = torch.zeros((4, cfg.d), device=DEV)
    xd = u16_to_dev(x, torch.bfloat16, DEV)
    tq.scion_moe_forward(xd, 0, layer, out)
    torch.cuda.synchronize()
    assert float(out.abs().sum()) == 0.0
    with pytest.raises(tq.ScionError) as ei:
        tq.scion_moe_forward(xd, 5, layer, out)
    assert ei.value.status == tq.SCION_EINVAL
    # out must be 16-byte aligned (the kernels store it with 16-byte accesses)
    flat = torch.zeros(4 * cfg.d + 1, device=DEV)
    with pytest.raises(tq.ScionError) as ei:
        tq.scion_moe_forward(xd, 4, layer, flat[1:].view(4, cfg.d))
    assert ei.value.status == tq.SCION_EINVAL


def test_host_buffer_forward_matches_device_forward():
    cfg = small("h", synth.PQ2_0, False)
    L, banks, ol, x = _case(cfg, 9)
    layer = device_layer(cfg, L, banks, 16)
    got_dev, _ = run_forward(layer, x, 9)
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty((9, cfg.d), dtype=torch.float32).pin_memory()
    tq.scion_moe_forward_host(xh, 9, layer, oh)
    torch.cuda.synchronize()
    ref, _, _ = oracle.forward(ol, x)
    check_output(oh.numpy().astype(np.float64), ref)
    check_output(got_dev, ref)


def test_repeated_calls_are_stable():
    """Back-to-back calls on one handle reuse the workspace (split-K counters reset)."""
    cfg = small("r", synth.PQ2_0, False, d=1024)
    L, banks, ol, x = _case(cfg, 8)
    layer = device_layer(cfg, L, banks, 8)
    a, _ = run_forward(layer, x, 8)
    for _ in range(3):
        b, _ = run_forward(layer, x, 8)
        check_output(b, a, rel_l2=1e-5, max_abs=1e-5)
    ref, _, _ = oracle.forward(ol, x)
    check_output(a, ref)


# ------------------------------------------------------------- full sizes
@pytest.mark.slow
@pytest.mark.parametrize("name", ["a3b_decode", "flashnext_decode"])
def test_full_size_decode(name):
    """One full layer of the decode shapes, every batch size the workload uses, all tokens."""
    cfg = synth.CONFIGS[name]
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    ol = oracle_layer_packed(cfg, L, banks)
    layer = device_layer(cfg, L, banks, max(cfg.tokens))
    del banks
    for T in cfg.tokens:
        x = with_margin(cfg, ol, synth.x_host(cfg, T))
        got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                               Kdense=cfg.shared_ffn + cfg.rank)
        _check_routing(cfg, dbg, ol, x, T)
        ref, _, _ = oracle.forward(ol, x)
        check_output(got, ref)
    # the largest batch again with activations far from N(0, 1) (outliers, tiny and large tokens)
    T = max(cfg.tokens)
    x = range_mix(cfg, ol, with_margin(cfg, ol, synth.x_host(cfg, T, 1)))
    got, _ = run_forward(layer, x, T)
    assert np.isfinite(got).all()
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.slow
def test_full_size_prefill_a3b_all_tokens():
    """The 4096-token a3b prefill on the GPU, every token against the oracle: routing (each
    expert's segment holds the oracle's entries) and the block output."""
    cfg = synth.CONFIGS["a3b_prefill"]
    T = cfg.tokens[0]
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    ol = oracle_layer_packed(cfg, L, banks)
    layer = device_layer(cfg, L, banks, T)
    del banks
    x = with_margin(cfg, ol, synth.x_host(cfg, T))
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    assert np.isfinite(got).all()
    # gates: the fp32 logits of K = 2048 tensor-core dot products carry absolute errors near 1e-5,
    # and a gate's relative error is the error of the logit differences (softmax), so 1e-4
    _check_routing(cfg, dbg, ol, x, T, stable=False, gate_rtol=1e-4)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.slow
def test_full_size_prefill_flashnext_sampled():
    """The 16384-token Zipf-loaded prefill on the GPU; the oracle checks a seeded sample of 2048
    tokens (flagged: not every token) that holds at least one token of every expert the batch
    uses.  Tokens are independent, so the sampled rows of the GPU output must equal the oracle's."""
    cfg = synth.CONFIGS["flashnext_prefill"]
    T, n_sample = cfg.tokens[0], 2048
    L = synth.layer_host(cfg)
    banks = packed_banks(cfg, L)
    ol = oracle_layer_packed(cfg, L, banks)
    layer = device_layer(cfg, L, banks, T)
    del banks
    x = with_margin(cfg, ol, synth.x_host(cfg, T))
    _, ids, _ = oracle.route(ol, x)
    rng = np.random.default_rng(4242)
    # one token per used expert (the first in a seeded order), then seeded fill
    order = rng.permutation(T)
    first = {}
    for t in order:
        for e in ids[t]:
            first.setdefault(int(e), int(t))
    picked = set(first.values())
    assert len(picked) <= n_sample
    rest = [int(t) for t in order if int(t) not in picked]
    sample = np.sort(np.array(sorted(picked) + rest[:n_sample - len(picked)]))
    covered = np.unique(ids[sample])
    np.testing.assert_array_equal(covered, np.unique(ids))
    got, _ = run_forward(layer, x, T)
    assert np.isfinite(got).all()
    ref, _, _ = oracle.forward(ol, x[sample])
    check_output(got[sample], ref)


# --------------------------------------------------------- tensor-core path
@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("router_f32", [False, True])
@pytest.mark.parametrize("T", [200, 500])
def test_prefill_stagewise(fmt, router_f32, T):
    """Batches above 64 tokens run as tcgen05 GEMMs; routing bit-exact, hidden and output
    within tolerance.  T = 200: 128-token gate/up tiles (50 tokens per expert on average);
    T = 500: 160-token gate/up tiles (125 on average, some experts past 128 tokens)."""
    cfg = small("p", fmt, router_f32, E=16, k=4, d=256, F=256, Fs=128, r=32)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, T)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    assert tq.scion_layer_check(layer) == 0
    _check_routing(cfg, dbg, ol, x, T, stable=False)
    _check_hidden(cfg, dbg, ol, x, T)
    hs, _ = oracle.shared(ol, x)
    z, _ = oracle.corr(ol, x)
    check_output(dbg["hz"].astype(np.float64), np.concatenate([hs, z], axis=1), rel_l2=1e-3)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("T", [65, 129, 250, 300, 500])
def test_prefill_multi_tile_experts(fmt, T):
    """Few experts, many tokens each: experts span several tiles, ragged tails (T = 65, 129:
    128-token tiles; T = 250, 300, 500: 160-token tiles, experts on both sides of 160 tokens and,
    at T = 500, across two tiles)."""
    cfg = small("m", fmt, False, E=4, k=2, d=384, F=128, Fs=0, r=16)
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, T)
    got, dbg = run_forward(layer, x, T, debug=True, E=cfg.n_experts, k=cfg.top_k, F=cfg.ffn,
                           Kdense=cfg.shared_ffn + cfg.rank)
    assert tq.scion_layer_check(layer) == 0
    _check_routing(cfg, dbg, ol, x, T, stable=False)
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)


@pytest.mark.parametrize("fmt", [synth.PQ2_0, synth.PTQ1_0])
@pytest.mark.parametrize("dense", [True, False])
def test_prefill_deterministic_combine(fmt, dense):
    """Both ways of adding the routed rows on the tensor-core path: one fp16 row per entry summed
    in slot order by the combine kernel (SCION_OPT_DETERMINISTIC = 1, the default), which repeats
    bit for bit, and fp32 reductions into out from the down projection's epilogue (0); with and
    without the dense down projection (without it out starts from zero, set by the x conversion
    or by the combine)."""
    cfg = small("dc", fmt, False, E=16, k=4, Fs=128 if dense else 0, r=16 if dense else 0)
    T = 300
    L, banks, ol, x = _case(cfg, T)
    layer = device_layer(cfg, L, banks, T)
    ref, _, _ = oracle.forward(ol, x)
    tq.scion_layer_set_option(layer, tq.SCION_OPT_DETERMINISTIC, 0)
    fused, _ = run_forward(layer, x, T)
    check_output(fused, ref)
    tq.scion_layer_set_option(layer, tq.SCION_OPT_DETERMINISTIC, 1)
    d1, _ = run_forward(layer, x, T)
    d2, _ = run_forward(layer, x, T)
    check_output(d1, ref)
    np.testing.assert_array_equal(d1, d2)


def test_prefill_matches_decode_passes():
    """The same tokens through both paths (a 64-token layer in two calls vs one 128-token call)."""
    cfg = small("pd", synth.PTQ1_0, False, E=32, k=4)
    L, banks, ol, x = _case(cfg, 128)
    dec = device_layer(cfg, L, banks, 64)
    pre = device_layer(cfg, L, banks, 128)
    a0, _ = run_forward(dec, x[:64], 64)
    a1, _ = run_forward(dec, x[64:], 64)
    b, _ = run_forward(pre, x, 128)
    check_output(b, np.concatenate([a0, a1]), rel_l2=1e-4, max_abs=1e-3)


# ------------------------------------------------------------------ quantizers
def _quant_inputs():
    rng = np.random.default_rng(2024)
    w = np.concatenate([rng.standard_normal((300, 128)), 0.01 * rng.laplace(size=(300, 128)),
                        rng.standard_t(3, size=(300, 128)), 1e3 * rng.standard_normal((20, 128)),
                        1e-4 * rng.standard_normal((20, 128))]).astype(np.float32)
    edge = np.zeros((6, 128), np.float32)
    edge[1] = 0.25
    edge[2] = np.where(np.arange(128) % 2, 3.0, -3.0)
    edge[3, 17] = -2.0
    edge[4, :64] = 1.0
    edge[5] = np.linspace(-1, 1, 128)
    return np.concatenate([w, edge])


@pytest.mark.parametrize("method", [tq.SCION_QUANT_ABSMEAN, tq.SCION_QUANT_LLOYD])
def test_quantize_matches_oracle(method):
    """Codes and fp16 scales bit-exact against the oracle (decisions in fp64 on both sides),
    then packed on the device into both containers and read back by the oracle's unpacker."""
    w = _quant_inputs()
    ref_c, ref_s = oracle.quantize(method, w, iters=30)
    wd = torch.from_numpy(w).to(DEV)
    codes = torch.empty(w.shape, dtype=torch.int8, device=DEV)
    scales = torch.empty(w.shape[0], dtype=torch.int16, device=DEV)
    tq.scion_quantize_device(method, wd, codes, scales, iters=30)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), ref_s)
    for fmt in (synth.PQ2_0, synth.PTQ1_0):
        blocks = tq.scion_pack_device(fmt, codes, scales)
        c2, s2, st = oracle.unpack(fmt, blocks.cpu().numpy())
        assert st == oracle.OK
        np.testing.assert_array_equal(c2.reshape(ref_c.shape), ref_c)
        np.testing.assert_array_equal(s2.reshape(-1), ref_s)


def test_quantize_rejects_bad_arguments():
    w = torch.zeros((2, 128), dtype=torch.float32, device=DEV)
    codes = torch.empty((2, 128), dtype=torch.int8, device=DEV)
    scales = torch.empty(2, dtype=torch.int16, device=DEV)
    with pytest.raises(tq.ScionError) as ei:
        tq.scion_quantize_device(7, w, codes, scales)
    assert ei.value.status == tq.SCION_EINVAL
    flat = torch.zeros(2 * 128 + 1, dtype=torch.float32, device=DEV)
    with pytest.raises(tq.ScionError) as ei:  # w must be 16-byte aligned
        tq.scion_quantize_device(tq.SCION_QUANT_ABSMEAN, flat[1:], codes, scales)
    assert ei.value.status == tq.SCION_EINVAL


# ------------------------------------------------------------------ failure path
def test_bounded_wait_gives_up_and_context_stays_usable():
    """A device wait on a barrier phase that nothing completes gives up after its limit with
    SCION_ETIMEOUT in the status word; the other waiter leaves on the abort flag; the context then
    still runs a forward correctly."""
    (status, first_ok, second_ok), ms = tq.scion_selftest_bounded_wait(50000)  # 50 ms
    assert status == tq.SCION_ETIMEOUT and first_ok == 0 and second_ok == 0
    assert 50.0 <= ms < 200.0, ms
    cfg = small("fw", synth.PQ2_0, False)
    L, banks, ol, x = _case(cfg, 5)
    layer = device_layer(cfg, L, banks, 64)
    got, _ = run_forward(layer, x, 5)
    assert tq.scion_layer_check(layer) == 0
    ref, _, _ = oracle.forward(ol, x)
    check_output(got, ref)
