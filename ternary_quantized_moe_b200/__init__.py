"""Python binding of libscion: the B200 forward pass of one ternary MoE block.

Argument marshalling only: every function here forwards to the C ABI declared in
``include/scion.h`` (same names), and every step of the block runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  If the
library has not been built, the first call raises -- there is no fallback.

Block ("Scion: ternary MoE quantization with trained corrections", The idea;
"Scion-35B-A3B" / "Scion-FlashNext-176B-A6B" model cards, Model Overview and
Weight Representation):

    out[t] = sum_j g_tj W_d,e (silu(W_g,e x_t) * (W_u,e x_t)) + S(x_t) + B (A x_t)
"""
from __future__ import annotations

import ctypes as C
import os
import threading
from typing import Optional

import numpy as np

__all__ = [
    "SCION_PQ2_0", "SCION_PTQ1_0", "ScionError", "scion_block_bytes", "scion_status_str",
    "scion_pack_pq2", "scion_pack_ptq1", "scion_unpack", "scion_pack_device", "scion_unpack_device",
    "scion_layer_create", "scion_layer_destroy", "scion_layer_device_bytes", "scion_moe_forward",
    "scion_moe_forward_host", "scion_moe_forward_debug", "Layer", "library_path", "EXPORTS",
    "scion_profile_begin", "scion_profile_end", "scion_kernel_launches", "STAGES", "scion_layer_check",
    "scion_router_logits_static", "scion_layer_set_option", "SCION_OPT_STREAM_MIN_TOKENS", "SCION_OPT_DECODE_TC",
    "SCION_OPT_DETERMINISTIC", "SCION_OPT_PARTS", "SCION_PART_ROUTED", "SCION_PART_DENSE",
    "scion_moe_forward_residual", "scion_quantize_device", "SCION_QUANT_ABSMEAN", "SCION_QUANT_LLOYD",
    "scion_selftest_bounded_wait", "scion_debug_route", "scion_corr_create", "scion_corr_forward", "Corr",
]

SCION_PQ2_0 = 0
SCION_PTQ1_0 = 1
SCION_OK, SCION_EINVAL, SCION_ENOMEM, SCION_ECUDA, SCION_EFORMAT, SCION_ETIMEOUT = 0, -1, -2, -3, -4, -5

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libscion.so")
_lock = threading.Lock()
_lib = None

# Every symbol include/scion.h declares.
EXPORTS = (
    "scion_block_bytes", "scion_status_str", "scion_pack_pq2", "scion_pack_ptq1", "scion_unpack",
    "scion_pack_device", "scion_unpack_device", "scion_layer_create", "scion_layer_destroy",
    "scion_layer_device_bytes", "scion_moe_forward", "scion_moe_forward_host", "scion_moe_forward_debug",
    "scion_profile_begin", "scion_profile_end", "scion_kernel_launches", "scion_layer_check",
    "scion_router_logits_static", "scion_layer_set_option", "scion_moe_forward_residual", "scion_quantize_device",
    "scion_selftest_bounded_wait", "scion_debug_route", "scion_corr_create", "scion_corr_destroy",
    "scion_corr_device_bytes", "scion_corr_forward", "scion_corr_check",
)
SCION_QUANT_ABSMEAN, SCION_QUANT_LLOYD = 0, 1
SCION_OPT_STREAM_MIN_TOKENS, SCION_OPT_DECODE_TC, SCION_OPT_DETERMINISTIC, SCION_OPT_PARTS = 1, 2, 3, 4
SCION_PART_ROUTED, SCION_PART_DENSE = 1, 2
STAGES = ("router_f32", "xproj", "route", "gateup", "down_routed", "down_dense", "x16", "combine")


class ScionError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__("%s: %s (%d)" % (where, scion_status_str(status), status))
        self.status = status


class _Desc(C.Structure):
    _fields_ = [
        ("d", C.c_int), ("n_experts", C.c_int), ("top_k", C.c_int), ("ffn", C.c_int),
        ("shared_ffn", C.c_int), ("rank", C.c_int), ("fmt", C.c_int), ("router_fp32", C.c_int),
        ("norm_topk", C.c_int),
        ("w_router", C.c_void_p), ("w_router_delta", C.c_void_p),
        ("gate_exps", C.c_void_p), ("up_exps", C.c_void_p), ("down_exps", C.c_void_p),
        ("sh_gate", C.c_void_p), ("sh_up", C.c_void_p), ("sh_down", C.c_void_p),
        ("sh_gate_vec", C.c_void_p), ("corr_a", C.c_void_p), ("corr_b", C.c_void_p),
        ("corr_packed", C.c_int), ("expert_lo", C.c_int), ("n_local_experts", C.c_int),
    ]


class _CorrDesc(C.Structure):
    _fields_ = [("d_in", C.c_int), ("d_out", C.c_int), ("rank", C.c_int), ("packed", C.c_int),
                ("corr_a", C.c_void_p), ("corr_b", C.c_void_p)]


class _Debug(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("logits", "ids", "gates", "counts", "offsets", "perm", "h", "hz")]


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError("libscion.so is not built (run __graft_entry__.build() or "
                              "python -m ternary_quantized_moe_b200.build); there is no fallback path")
        lib = C.CDLL(_LIB_PATH)
        vp, ci, i64 = C.c_void_p, C.c_int, C.c_int64
        sig = {
            "scion_block_bytes": (C.c_size_t, [ci]),
            "scion_status_str": (C.c_char_p, [ci]),
            "scion_pack_pq2": (ci, [vp, vp, i64, vp]),
            "scion_pack_ptq1": (ci, [vp, vp, i64, vp]),
            "scion_unpack": (ci, [ci, vp, i64, vp, vp]),
            "scion_pack_device": (ci, [ci, vp, vp, i64, vp, vp, vp]),
            "scion_unpack_device": (ci, [ci, vp, i64, vp, vp, vp, vp]),
            "scion_layer_create": (ci, [C.POINTER(_Desc), ci, vp, C.POINTER(vp)]),
            "scion_layer_destroy": (None, [vp]),
            "scion_layer_device_bytes": (C.c_size_t, [vp]),
            "scion_moe_forward": (ci, [vp, ci, vp, vp, vp]),
            "scion_moe_forward_residual": (ci, [vp, ci, vp, vp, vp, vp]),
            "scion_quantize_device": (ci, [ci, vp, i64, ci, vp, vp, vp]),
            "scion_selftest_bounded_wait": (ci, [ci, C.POINTER(C.c_int), C.POINTER(C.c_double), vp]),
            "scion_moe_forward_host": (ci, [vp, ci, vp, vp, vp]),
            "scion_moe_forward_debug": (ci, [vp, ci, vp, vp, C.POINTER(_Debug), vp]),
            "scion_debug_route": (ci, [vp, ci, vp, vp, vp, vp, vp, vp]),
            "scion_corr_create": (ci, [C.POINTER(_CorrDesc), ci, vp, C.POINTER(vp)]),
            "scion_corr_destroy": (None, [vp]),
            "scion_corr_device_bytes": (C.c_size_t, [vp]),
            "scion_corr_forward": (ci, [vp, ci, vp, vp, vp, vp]),
            "scion_corr_check": (ci, [vp, vp]),
            "scion_profile_begin": (ci, [ci]),
            "scion_profile_end": (ci, [ci, C.POINTER(C.c_double), C.POINTER(C.c_int64)]),
            "scion_kernel_launches": (C.c_int64, []),
            "scion_layer_check": (ci, [vp, vp]),
            "scion_router_logits_static": (ci, [vp, ci, vp, vp, ci, ci, vp, vp]),
            "scion_layer_set_option": (ci, [vp, ci, ci]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
        return lib


def _check(status: int, where: str):
    if status != SCION_OK:
        raise ScionError(status, where)


def _stream(stream):
    if stream is None:
        import torch

        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


def _dptr(t, name: str, dtypes=None):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("%s must be a contiguous CUDA tensor" % name)
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError("%s has dtype %s, expected one of %s" % (name, t.dtype, dtypes))
    return t.data_ptr()


def _hptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ---------------------------------------------------------------- formats
def scion_block_bytes(fmt: int) -> int:
    return int(_load().scion_block_bytes(int(fmt)))


def scion_status_str(status: int) -> str:
    return _load().scion_status_str(int(status)).decode()


def _host_pack(fn_name, codes, scales):
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    n = codes.size // 128
    fmt = SCION_PQ2_0 if fn_name == "scion_pack_pq2" else SCION_PTQ1_0
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] // 128 * scion_block_bytes(fmt),), np.uint8)
    _check(getattr(_load(), fn_name)(_hptr(codes), _hptr(scales), n, _hptr(out)), fn_name)
    return out


def scion_pack_pq2(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Host PQ2_0 packer: codes int8 [..., K] (K % 128 == 0), scales uint16 fp16 bits [..., K/128]."""
    return _host_pack("scion_pack_pq2", codes, scales)


def scion_pack_ptq1(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Host PTQ1_0 packer; same arguments as scion_pack_pq2."""
    return _host_pack("scion_pack_ptq1", codes, scales)


def scion_unpack(fmt: int, blocks: np.ndarray):
    """Host unpacker -> (codes int8, scales uint16, status)."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    bb = scion_block_bytes(fmt)
    n = blocks.size // bb
    codes = np.empty(blocks.shape[:-1] + (blocks.shape[-1] // bb * 128,), np.int8)
    scales = np.empty(blocks.shape[:-1] + (blocks.shape[-1] // bb,), np.uint16)
    st = _load().scion_unpack(int(fmt), _hptr(blocks), n, _hptr(codes), _hptr(scales))
    if st not in (SCION_OK, SCION_EFORMAT):
        _check(st, "scion_unpack")
    return codes, scales, int(st)


def scion_pack_device(fmt: int, codes, scales, out=None, bad_count=None, stream=None):
    """Device packer: codes int8 CUDA [..., K], scales fp16/int16 CUDA [..., K/128] -> uint8 CUDA blocks."""
    import torch

    n = codes.numel() // 128
    if out is None:
        out = torch.empty(codes.shape[:-1] + (codes.shape[-1] // 128 * scion_block_bytes(fmt),),
                          dtype=torch.uint8, device=codes.device)
    st = _load().scion_pack_device(int(fmt), _dptr(codes, "codes", (torch.int8,)),
                                   _dptr(scales, "scales", (torch.float16, torch.int16)), n,
                                   _dptr(out, "out", (torch.uint8,)), _dptr(bad_count, "bad_count", (torch.int64,)),
                                   _stream(stream))
    _check(st, "scion_pack_device")
    return out


def scion_selftest_bounded_wait(limit_us: int, stream=None):
    """Runs the bounded-wait failure check; returns ((status, first_ok, second_ok), elapsed_ms)."""
    res = (C.c_int * 3)()
    ms = C.c_double()
    st = _load().scion_selftest_bounded_wait(int(limit_us), res, C.byref(ms), _stream(stream))
    _check(st, "scion_selftest_bounded_wait")
    return (res[0], res[1], res[2]), ms.value


def scion_quantize_device(method: int, w, codes, scales, iters: int = 30, stream=None) -> None:
    """w: fp32 CUDA [n, 128] (groups of 128); codes: int8 CUDA [n, 128]; scales: int16 CUDA [n]
    (binary16 bit patterns).  method: SCION_QUANT_ABSMEAN or SCION_QUANT_LLOYD."""
    import torch

    n = w.numel() // 128
    if w.numel() != n * 128 or codes.numel() != n * 128 or scales.numel() != n:
        raise ValueError("w / codes / scales sizes do not match")
    st = _load().scion_quantize_device(int(method), _dptr(w, "w", (torch.float32,)), n, int(iters),
                                       _dptr(codes, "codes", (torch.int8,)),
                                       _dptr(scales, "scales", (torch.int16, torch.uint16)), _stream(stream))
    _check(st, "scion_quantize_device")


def scion_unpack_device(fmt: int, blocks, codes=None, scales=None, bad_count=None, stream=None):
    """Device unpacker -> (codes int8 CUDA, scales int16 CUDA holding fp16 bits)."""
    import torch

    bb = scion_block_bytes(fmt)
    n = blocks.numel() // bb
    if codes is None:
        codes = torch.empty(blocks.shape[:-1] + (blocks.shape[-1] // bb * 128,), dtype=torch.int8, device=blocks.device)
    if scales is None:
        scales = torch.empty(blocks.shape[:-1] + (blocks.shape[-1] // bb,), dtype=torch.int16, device=blocks.device)
    st = _load().scion_unpack_device(int(fmt), _dptr(blocks, "blocks", (torch.uint8,)), n,
                                     _dptr(codes, "codes", (torch.int8,)),
                                     _dptr(scales, "scales", (torch.int16, torch.float16)),
                                     _dptr(bad_count, "bad_count", (torch.int64,)), _stream(stream))
    _check(st, "scion_unpack_device")
    return codes, scales


# ------------------------------------------------------------------ layer
class Layer:
    """Owns a scion_layer handle; keeps the tensors the library reads in place alive."""

    def __init__(self, handle: int, keep: dict, d: int, n_experts: int, top_k: int, ffn: int,
                 shared_ffn: int, rank: int, max_tokens: int):
        self.handle = handle
        self._keep = keep
        self.d, self.n_experts, self.top_k, self.ffn = d, n_experts, top_k, ffn
        self.shared_ffn, self.rank, self.max_tokens = shared_ffn, rank, max_tokens

    def close(self):
        if self.handle:
            scion_layer_destroy(self)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def scion_layer_create(*, d: int, n_experts: int, top_k: int, ffn: int, fmt: int, w_router, w_router_delta,
                       gate_exps, up_exps, down_exps, shared_ffn: int = 0, sh_gate=None, sh_up=None,
                       sh_down=None, rank: int = 0, corr_a=None, corr_b=None, norm_topk: int = 1,
                       corr_packed: int = 0, max_tokens: int = 64, expert_lo: int = 0, n_local_experts: int = 0,
                       stream=None) -> Layer:
    """Builds a layer from CUDA tensors (see include/scion.h for layouts).

    w_router / w_router_delta: float32 (fp32 router) or bfloat16 [E, d]; banks: uint8 packed
    blocks; shared weights: bfloat16; correction factors: bfloat16, or (corr_packed = 1) uint8
    PQ2_0 blocks [rank, d/128*34] and [d, rank/128*34]."""
    import torch

    bf16 = (torch.bfloat16,)
    router_fp32 = 1 if w_router.dtype == torch.float32 else 0
    rdt = (torch.float32,) if router_fp32 else bf16
    D = _Desc()
    D.d, D.n_experts, D.top_k, D.ffn = d, n_experts, top_k, ffn
    D.shared_ffn, D.rank, D.fmt, D.router_fp32, D.norm_topk = shared_ffn, rank, fmt, router_fp32, norm_topk
    D.w_router = _dptr(w_router, "w_router", rdt)
    D.w_router_delta = _dptr(w_router_delta, "w_router_delta", rdt)
    D.gate_exps = _dptr(gate_exps, "gate_exps", (torch.uint8,))
    D.up_exps = _dptr(up_exps, "up_exps", (torch.uint8,))
    D.down_exps = _dptr(down_exps, "down_exps", (torch.uint8,))
    D.sh_gate = _dptr(sh_gate, "sh_gate", bf16)
    D.sh_up = _dptr(sh_up, "sh_up", bf16)
    D.sh_down = _dptr(sh_down, "sh_down", bf16)
    D.sh_gate_vec = None
    cdt = (torch.uint8,) if corr_packed else bf16
    D.corr_a = _dptr(corr_a, "corr_a", cdt)
    D.corr_b = _dptr(corr_b, "corr_b", cdt)
    D.corr_packed = int(corr_packed)
    D.expert_lo, D.n_local_experts = int(expert_lo), int(n_local_experts)
    h = C.c_void_p()
    st = _load().scion_layer_create(C.byref(D), int(max_tokens), _stream(stream), C.byref(h))
    _check(st, "scion_layer_create")
    keep = dict(w_router=w_router, w_router_delta=w_router_delta, sh_gate=sh_gate, sh_up=sh_up, corr_a=corr_a)
    if corr_packed:
        keep["corr_b"] = corr_b  # decode reads both factors' blocks in place
    return Layer(h.value, keep, d, n_experts, top_k, ffn, shared_ffn, rank, max_tokens)


def scion_layer_destroy(layer: Layer) -> None:
    if layer.handle:
        _load().scion_layer_destroy(C.c_void_p(layer.handle))
        layer.handle = 0
        layer._keep = {}


def scion_layer_check(layer: Layer, stream=None) -> int:
    """Waits for the stream and returns (and clears) the layer's device status word."""
    return int(_load().scion_layer_check(C.c_void_p(layer.handle), _stream(stream)))


def scion_layer_set_option(layer: Layer, option: int, value: int) -> None:
    _check(_load().scion_layer_set_option(C.c_void_p(layer.handle), int(option), int(value)),
           "scion_layer_set_option")


def scion_layer_device_bytes(layer: Layer) -> int:
    return int(_load().scion_layer_device_bytes(C.c_void_p(layer.handle)))


def scion_moe_forward(x, T: int, layer: Layer, out, stream=None) -> None:
    """x: bf16 CUDA [T, d]; out: fp32 CUDA [T, d] (overwritten)."""
    import torch

    st = _load().scion_moe_forward(_dptr(x, "x", (torch.bfloat16,)), int(T), C.c_void_p(layer.handle),
                                   _dptr(out, "out", (torch.float32,)), _stream(stream))
    _check(st, "scion_moe_forward")


def scion_moe_forward_residual(x, T: int, layer: Layer, resid, out, stream=None) -> None:
    """x: bf16 CUDA [T, d]; resid: fp32 CUDA [T, d] (may be `out` itself); out = resid + block(x)."""
    import torch

    st = _load().scion_moe_forward_residual(_dptr(x, "x", (torch.bfloat16,)), int(T), C.c_void_p(layer.handle),
                                            _dptr(resid, "resid", (torch.float32,)),
                                            _dptr(out, "out", (torch.float32,)), _stream(stream))
    _check(st, "scion_moe_forward_residual")


def scion_moe_forward_host(x_host, T: int, layer: Layer, out_host, stream=None) -> None:
    """x_host: bf16 CPU tensor [T, d] (pinned for async copies); out_host: fp32 CPU tensor [T, d]."""
    import torch

    for t, nm, dt in ((x_host, "x_host", torch.bfloat16), (out_host, "out_host", torch.float32)):
        if t.is_cuda or not t.is_contiguous() or t.dtype != dt:
            raise ValueError("%s must be a contiguous CPU %s tensor" % (nm, dt))
    st = _load().scion_moe_forward_host(x_host.data_ptr(), int(T), C.c_void_p(layer.handle), out_host.data_ptr(),
                                        _stream(stream))
    _check(st, "scion_moe_forward_host")


def scion_moe_forward_debug(x, T: int, layer: Layer, out, stream=None, **bufs) -> None:
    """Forward plus copies of intermediates into the given CUDA tensors (logits, ids, gates,
    counts, offsets, perm, h, hz; see scion_debug_out in include/scion.h)."""
    import torch

    dbg = _Debug()
    for name, _ in _Debug._fields_:
        setattr(dbg, name, _dptr(bufs.get(name), name))
    st = _load().scion_moe_forward_debug(_dptr(x, "x", (torch.bfloat16,)), int(T), C.c_void_p(layer.handle),
                                         _dptr(out, "out", (torch.float32,)), C.byref(dbg), _stream(stream))
    _check(st, "scion_moe_forward_debug")


def scion_debug_route(x, T: int, layer: Layer, ids=None, gates=None, offsets=None, perm=None, stream=None) -> None:
    """The batch's routing into the given CUDA tensors: ids int32 [T, k], gates fp32 [T, k],
    offsets int32 [E + 1], perm int32 [T * k] (each optional)."""
    import torch

    st = _load().scion_debug_route(_dptr(x, "x", (torch.bfloat16,)), int(T), C.c_void_p(layer.handle),
                                   _dptr(ids, "ids", (torch.int32,)), _dptr(gates, "gates", (torch.float32,)),
                                   _dptr(offsets, "offsets", (torch.int32,)), _dptr(perm, "perm", (torch.int32,)),
                                   _stream(stream))
    _check(st, "scion_debug_route")


# ------------------------------------------ correction branch on the attention output
class Corr:
    """Handle of the correction branch on the attention output (scion_corr_*).  Keeps the
    factor tensors alive for the handle's lifetime."""

    def __init__(self, handle: int, d_in: int, d_out: int, keep):
        self.handle, self.d_in, self.d_out, self._keep = handle, d_in, d_out, keep

    def close(self):
        if self.handle:
            _load().scion_corr_destroy(C.c_void_p(self.handle))
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def scion_corr_create(d_in: int, d_out: int, rank: int, corr_a, corr_b, packed: int = 0, max_tokens: int = 64,
                      stream=None) -> Corr:
    """corr_a / corr_b: bf16 CUDA [rank, d_in] / [d_out, rank], or (packed = 1) uint8 CUDA PQ2_0 blocks."""
    D = _CorrDesc()
    D.d_in, D.d_out, D.rank, D.packed = int(d_in), int(d_out), int(rank), int(packed)
    D.corr_a, D.corr_b = _dptr(corr_a, "corr_a"), _dptr(corr_b, "corr_b")
    h = C.c_void_p()
    _check(_load().scion_corr_create(C.byref(D), int(max_tokens), _stream(stream), C.byref(h)), "scion_corr_create")
    return Corr(h.value, d_in, d_out, (corr_a, corr_b))


def scion_corr_forward(v, T: int, corr: Corr, out, base=None, stream=None) -> None:
    """out = base + B (A v): v bf16 CUDA [T, d_in]; base / out fp32 CUDA [T, d_out] (base optional)."""
    import torch

    st = _load().scion_corr_forward(_dptr(v, "v", (torch.bfloat16,)), int(T), C.c_void_p(corr.handle),
                                    _dptr(base, "base", (torch.float32,)), _dptr(out, "out", (torch.float32,)),
                                    _stream(stream))
    _check(st, "scion_corr_forward")


def scion_corr_check(corr: Corr, stream=None) -> int:
    return int(_load().scion_corr_check(C.c_void_p(corr.handle), _stream(stream)))


# ------------------------------------------------------------ measurement
def scion_profile_begin(max_launches: int) -> None:
    _check(_load().scion_profile_begin(int(max_launches)), "scion_profile_begin")


def scion_profile_end() -> dict:
    """-> {stage name: (total ms, launches)}"""
    n = len(STAGES)
    ms = (C.c_double * n)()
    cnt = (C.c_int64 * n)()
    _check(_load().scion_profile_end(n, ms, cnt), "scion_profile_end")
    return {STAGES[i]: (float(ms[i]), int(cnt[i])) for i in range(n)}


def scion_kernel_launches() -> int:
    return int(_load().scion_kernel_launches())


# ------------------------------------------------------- no-allocation entry
def scion_router_logits_static(x, T: int, w_router, w_router_delta, logits, stream=None) -> None:
    """Router logits (x . W_r + x . delta, fp32) for callers that cannot allocate device
    memory: the library keeps the split-K scratch in a static device array.  x: bf16 CUDA
    [T, d]; weights: bf16 CUDA [E, d]; logits: fp32 CUDA [T, E].  T <= 64, E <= 512,
    d <= 4096.  Calls share the scratch, so issue them in order on one stream."""
    import torch

    E, d = w_router.shape
    st = _load().scion_router_logits_static(
        _dptr(x, "x", (torch.bfloat16,)), int(T), _dptr(w_router, "w_router", (torch.bfloat16,)),
        _dptr(w_router_delta, "w_router_delta", (torch.bfloat16,)), int(E), int(d),
        _dptr(logits, "logits", (torch.float32,)), _stream(stream))
    _check(st, "scion_router_logits_static")
