"""Python binding of libmoe, the sm_100a MoE-layer forward library.

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libmoe.so`` behind the C ABI declared in ``include/moe.h``.  PyTorch is used
for device memory and streams; tensors are passed as raw device pointers and
the current torch stream is used unless another one is given.  There is no
CPU fallback: if the library is missing, loading it raises.

Python names match the C entry points: ``moe_route``, ``moe_permute``,
``moe_expert_ffn``, ``moe_combine``, ``moe_layer_forward``, plus
``moe_scratch_size``, ``moe_workspace_size`` and ``moe_status_string``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "LIB_PATH", "MoeError", "moe_config", "moe_stats", "moe_ws_layout", "lib", "make_config",
    "moe_status_string", "moe_scratch_size", "moe_workspace_size", "moe_route", "moe_permute",
    "moe_expert_ffn", "moe_combine", "moe_layer_forward", "moe_convert_bf16_to_f16", "moe_permute_static",
    "moe_expert_ffn_combine", "MOE_STATIC_SCRATCH_BYTES", "prepare_w2", "moe_aux_coef_update",
    "moe_aux_coef_next", "moe_testing_set_expert_wait", "moe_segments_scratch_size", "moe_expert_ffn_segments",
    "moe_backward_workspace_size", "moe_layer_backward", "moe_mxfp8_weight_bytes", "moe_prepare_mxfp8_weights",
    "moe_workspace_size_mxfp8", "moe_layer_forward_mxfp8", "prepare_mxfp8", "moe_workspace_size_shared",
    "moe_layer_forward_shared",
    "read_stats", "STATS_BYTES", "MOE_ACT_RELU", "MOE_ACT_SWIGLU", "MOE_DTYPE_F32", "MOE_DTYPE_BF16",
    "MOE_DTYPE_F16", "MOE_DEV_TIMEOUT", "MOE_DEV_BOUNDS", "MOE_DEV_RANGE", "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_ACT_RELU, MOE_ACT_SWIGLU = 0, 1
MOE_DTYPE_F32, MOE_DTYPE_BF16, MOE_DTYPE_F16 = 0, 1, 2
MOE_DEV_TIMEOUT, MOE_DEV_BOUNDS, MOE_DEV_RANGE = 1, 2, 4
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA"}

EXPORTED_SYMBOLS = ["moe_status_string", "moe_scratch_size", "moe_workspace_size", "moe_route",
                    "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward",
                    "moe_convert_bf16_to_f16", "moe_permute_static", "moe_expert_ffn_combine",
                    "moe_aux_coef_update", "moe_aux_coef_next", "moe_testing_set_expert_wait",
                    "moe_segments_scratch_size", "moe_expert_ffn_segments", "moe_backward_workspace_size",
                    "moe_layer_backward", "moe_mxfp8_weight_bytes", "moe_prepare_mxfp8_weights",
                    "moe_workspace_size_mxfp8", "moe_layer_forward_mxfp8", "moe_workspace_size_shared",
                    "moe_layer_forward_shared"]
MOE_STATIC_SCRATCH_BYTES = 2 << 20


class moe_config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("F", ctypes.c_int32),
                ("k", ctypes.c_int32), ("act", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("lambda_", ctypes.c_float),
                ("hidden_dtype", ctypes.c_int32)]


class moe_stats(ctypes.Structure):
    _fields_ = [("drop_count", ctypes.c_int32), ("rows_kept", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("near_tie_count", ctypes.c_int32), ("drop_rate", ctypes.c_float), ("aux_loss", ctypes.c_float),
                ("status", ctypes.c_uint32), ("z_loss", ctypes.c_float)]


class moe_ws_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ["topk_idx", "topk_w", "gap", "counts", "kept", "offsets", "row_of", "src_tok", "row_w",
                 "xp", "h", "yp", "scratch", "total"]]


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)} ({moe_status_string(code)})")
        self.code = code


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m mixture_experts_layer_logit_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    cfgp = ctypes.POINTER(moe_config)
    st = ctypes.c_int
    L.moe_status_string.argtypes = [st]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_scratch_size.argtypes = [cfgp]
    L.moe_scratch_size.restype = ctypes.c_size_t
    L.moe_workspace_size.argtypes = [cfgp, ctypes.POINTER(moe_ws_layout)]
    L.moe_workspace_size.restype = ctypes.c_size_t
    L.moe_route.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_permute.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_expert_ffn.argtypes = [cfgp, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_combine.argtypes = [cfgp, P, P, P, P, P]
    L.moe_layer_forward.argtypes = [cfgp, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_convert_bf16_to_f16.argtypes = [P, P, ctypes.c_size_t, P]
    L.moe_permute_static.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P]
    L.moe_expert_ffn_combine.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    f32 = ctypes.c_float
    L.moe_aux_coef_update.argtypes = [P, P, f32, f32, P]
    L.moe_aux_coef_next.argtypes = [f32, f32, f32, f32, ctypes.POINTER(f32)]
    L.moe_testing_set_expert_wait.argtypes = [ctypes.c_uint64, ctypes.c_int32]
    i32 = ctypes.c_int32
    L.moe_segments_scratch_size.argtypes = [cfgp, i32, i32]
    L.moe_segments_scratch_size.restype = ctypes.c_size_t
    L.moe_expert_ffn_segments.argtypes = [cfgp, i32, i32, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    sz = ctypes.POINTER(ctypes.c_size_t)
    L.moe_mxfp8_weight_bytes.argtypes = [cfgp, sz, sz, sz, sz]
    L.moe_mxfp8_weight_bytes.restype = ctypes.c_size_t
    L.moe_prepare_mxfp8_weights.argtypes = [cfgp, P, P, P, P, P, P, P]
    L.moe_workspace_size_mxfp8.argtypes = [cfgp]
    L.moe_workspace_size_mxfp8.restype = ctypes.c_size_t
    L.moe_layer_forward_mxfp8.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_workspace_size_shared.argtypes = [cfgp, i32]
    L.moe_workspace_size_shared.restype = ctypes.c_size_t
    L.moe_layer_forward_shared.argtypes = [cfgp, i32, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.moe_backward_workspace_size.argtypes = [cfgp]
    L.moe_backward_workspace_size.restype = ctypes.c_size_t
    L.moe_layer_backward.argtypes = [cfgp, P, P, P, P, P, P, f32, f32, P, ctypes.c_size_t, P, P, P, P, P, P, P, P,
                                     ctypes.c_size_t, P]
    for n in ["moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward",
              "moe_convert_bf16_to_f16", "moe_permute_static", "moe_expert_ffn_combine", "moe_aux_coef_update",
              "moe_aux_coef_next", "moe_testing_set_expert_wait", "moe_expert_ffn_segments", "moe_layer_backward",
              "moe_prepare_mxfp8_weights", "moe_layer_forward_mxfp8", "moe_layer_forward_shared"]:
        getattr(L, n).restype = st
    _lib = L
    return L


_DTYPES = {"f32": MOE_DTYPE_F32, "bf16": MOE_DTYPE_BF16, "f16": MOE_DTYPE_F16}


def make_config(T: int, d: int, E: int, F: int, k: int, act: str = "relu", dtype: str = "bf16",
                capacity_factor: float = 0.0, lam: float = 0.0, hidden: Optional[str] = None) -> moe_config:
    """hidden: element type of the expert hidden activation and of W2 on the bf16
    path ("f16", the default, or "bf16"); always "f32" on the fp32 path."""
    if hidden is None:
        hidden = "f16" if dtype == "bf16" else "f32"
    return moe_config(T, d, E, F, k, MOE_ACT_SWIGLU if act == "swiglu" else MOE_ACT_RELU, _DTYPES[dtype],
                      capacity_factor, lam, _DTYPES[hidden])


def _ptr(t) -> Optional[int]:
    """Device pointer of a tensor (None -> NULL); also accepts raw ints."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _check(fn: str, code: int):
    if code != 0:
        raise MoeError(fn, code)


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def moe_scratch_size(cfg: moe_config) -> int:
    return lib().moe_scratch_size(ctypes.byref(cfg))


def moe_workspace_size(cfg: moe_config):
    """(bytes, moe_ws_layout) of the moe_layer_forward workspace."""
    L = moe_ws_layout()
    n = lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(L))
    return n, L


def moe_route(cfg, x, Wg, bg, topk_idx, topk_w, gap, prob_mean, ws, stream=None, z_loss=None):
    """z_loss: optional device fp32 scalar that receives the router z-loss."""
    _check("moe_route", lib().moe_route(ctypes.byref(cfg), _ptr(x), _ptr(Wg), _ptr(bg), _ptr(topk_idx),
                                        _ptr(topk_w), _ptr(gap), _ptr(prob_mean), _ptr(z_loss), _ptr(ws),
                                        _nbytes(ws), _stream(stream)))


def moe_permute(cfg, x, topk_idx, gap, prob_mean, counts, kept, offsets, row_of, src_tok, xp, stats, ws,
                stream=None):
    _check("moe_permute", lib().moe_permute(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(gap),
                                            _ptr(prob_mean), _ptr(counts), _ptr(kept), _ptr(offsets),
                                            _ptr(row_of), _ptr(src_tok), _ptr(xp), _ptr(stats), _ptr(ws),
                                            _nbytes(ws), _stream(stream)))


def moe_permute_static(cfg, x, topk_idx, gap, prob_mean, counts, kept, offsets, row_of, src_tok, xp, stats,
                       stream=None):
    """moe_permute with its scratch in the library's fixed device array (no
    workspace argument; calls that overlap in time race on that array)."""
    _check("moe_permute_static", lib().moe_permute_static(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(gap),
                                                          _ptr(prob_mean), _ptr(counts), _ptr(kept),
                                                          _ptr(offsets), _ptr(row_of), _ptr(src_tok), _ptr(xp),
                                                          _ptr(stats), _stream(stream)))


def moe_expert_ffn(cfg, xp, offsets, W1, W2, h, yp, stats, ws, stream=None):
    _check("moe_expert_ffn", lib().moe_expert_ffn(ctypes.byref(cfg), _ptr(xp), _ptr(offsets), _ptr(W1),
                                                  _ptr(W2), _ptr(h), _ptr(yp), _ptr(stats), _ptr(ws),
                                                  _nbytes(ws), _stream(stream)))


def moe_expert_ffn_combine(cfg, xp, offsets, src_tok, row_w, W1, W2, h, out, stats, ws, stream=None):
    """Steps 4-5 fused (bf16, k <= 2): out (zeroed by the caller) += gate-weighted expert outputs.
    ws is a moe_layer_forward workspace."""
    _check("moe_expert_ffn_combine",
           lib().moe_expert_ffn_combine(ctypes.byref(cfg), _ptr(xp), _ptr(offsets), _ptr(src_tok), _ptr(row_w),
                                        _ptr(W1), _ptr(W2), _ptr(h), _ptr(out), _ptr(stats), _ptr(ws), _nbytes(ws),
                                        _stream(stream)))


def moe_segments_scratch_size(cfg: moe_config, nseg: int, rows: int) -> int:
    return lib().moe_segments_scratch_size(ctypes.byref(cfg), nseg, rows)


def moe_expert_ffn_segments(cfg, nseg, rows, seg_offsets, xp, W1, W2, h, yp, stats, ws, stream=None):
    """Step 4 over nseg caller-given segments of a rows-row buffer; segment i
    runs through local expert i % cfg.E (the expert-parallel form)."""
    _check("moe_expert_ffn_segments",
           lib().moe_expert_ffn_segments(ctypes.byref(cfg), nseg, rows, _ptr(seg_offsets), _ptr(xp), _ptr(W1),
                                         _ptr(W2), _ptr(h), _ptr(yp), _ptr(stats), _ptr(ws), _nbytes(ws),
                                         _stream(stream)))


def moe_combine(cfg, yp, row_of, topk_w, out, stream=None):
    _check("moe_combine", lib().moe_combine(ctypes.byref(cfg), _ptr(yp), _ptr(row_of), _ptr(topk_w),
                                            _ptr(out), _stream(stream)))


def moe_layer_forward(cfg, x, Wg, bg, W1, W2, out, stats, ws, stream=None):
    _check("moe_layer_forward", lib().moe_layer_forward(ctypes.byref(cfg), _ptr(x), _ptr(Wg), _ptr(bg),
                                                        _ptr(W1), _ptr(W2), _ptr(out), _ptr(stats), _ptr(ws),
                                                        _nbytes(ws), _stream(stream)))


def moe_aux_coef_update(stats, coef, beta: float, xi: float, stream=None):
    """On the device: coef <- beta * coef + (1 - beta) * xi * stats.drop_rate
    (stats: device moe_stats bytes, coef: device fp32 scalar)."""
    _check("moe_aux_coef_update", lib().moe_aux_coef_update(_ptr(stats), _ptr(coef), beta, xi, _stream(stream)))


def moe_aux_coef_next(coef: float, drop_rate: float, beta: float, xi: float) -> float:
    """The same update on the host (no device involved)."""
    out = ctypes.c_float()
    _check("moe_aux_coef_next", lib().moe_aux_coef_next(coef, drop_rate, beta, xi, ctypes.byref(out)))
    return out.value


def moe_testing_set_expert_wait(wait_ns: int, extra_dependency: int):
    """Test hook: limit of the one-launch expert kernel's waits (0 = default)
    and an amount added to its layer-2 dependency target (> 0: unreachable)."""
    _check("moe_testing_set_expert_wait", lib().moe_testing_set_expert_wait(wait_ns, extra_dependency))


def moe_workspace_size_shared(cfg: moe_config, F_shared: int) -> int:
    return lib().moe_workspace_size_shared(ctypes.byref(cfg), F_shared)


def moe_layer_forward_shared(cfg, F_shared, x, Wg, bg, W1, W2, W1_shared, W2_shared, out, stats, ws, stream=None):
    """The layer plus a shared expert of hidden width F_shared (every token, weight 1)."""
    _check("moe_layer_forward_shared",
           lib().moe_layer_forward_shared(ctypes.byref(cfg), F_shared, _ptr(x), _ptr(Wg), _ptr(bg), _ptr(W1),
                                          _ptr(W2), _ptr(W1_shared), _ptr(W2_shared), _ptr(out), _ptr(stats),
                                          _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_mxfp8_weight_bytes(cfg: moe_config):
    """(total, (w1q, w1s, w2q, w2s)) bytes of the prepared FP8 weights (0 if unsupported)."""
    v = [ctypes.c_size_t() for _ in range(4)]
    n = lib().moe_mxfp8_weight_bytes(ctypes.byref(cfg), *[ctypes.byref(x) for x in v])
    return n, tuple(x.value for x in v)


def moe_prepare_mxfp8_weights(cfg, W1, W2, W1q, W1s, W2q, W2s, stream=None):
    _check("moe_prepare_mxfp8_weights",
           lib().moe_prepare_mxfp8_weights(ctypes.byref(cfg), _ptr(W1), _ptr(W2), _ptr(W1q), _ptr(W1s), _ptr(W2q),
                                           _ptr(W2s), _stream(stream)))


def prepare_mxfp8(cfg, W1, W2):
    """Weight preparation for the FP8 layer: four new uint8 device tensors
    (W1q, W1s, W2q, W2s) from bf16 W1, W2.  Run once at load time."""
    import torch
    n, sizes = moe_mxfp8_weight_bytes(cfg)
    if n == 0:
        raise MoeError("moe_mxfp8_weight_bytes", 2)
    bufs = [torch.empty(max(sz, 16), dtype=torch.uint8, device=W1.device) for sz in sizes]
    moe_prepare_mxfp8_weights(cfg, W1, W2, *bufs)
    return tuple(bufs)


def moe_workspace_size_mxfp8(cfg: moe_config) -> int:
    return lib().moe_workspace_size_mxfp8(ctypes.byref(cfg))


def moe_layer_forward_mxfp8(cfg, x, Wg, bg, W1q, W1s, W2q, W2s, out, stats, ws, stream=None):
    _check("moe_layer_forward_mxfp8",
           lib().moe_layer_forward_mxfp8(ctypes.byref(cfg), _ptr(x), _ptr(Wg), _ptr(bg), _ptr(W1q), _ptr(W1s),
                                         _ptr(W2q), _ptr(W2s), _ptr(out), _ptr(stats), _ptr(ws), _nbytes(ws),
                                         _stream(stream)))


def moe_backward_workspace_size(cfg: moe_config) -> int:
    return lib().moe_backward_workspace_size(ctypes.byref(cfg))


def moe_layer_backward(cfg, x, Wg, bg, W1, W2, dout, aux_coef, z_coef, fws, dx, dWg, dbg, dW1, dW2, dw, stats, ws,
                       stream=None):
    """Gradients of <dout, out> + aux_coef * aux + z_coef * z_loss for the forward
    whose workspace is fws (see include/moe.h)."""
    _check("moe_layer_backward",
           lib().moe_layer_backward(ctypes.byref(cfg), _ptr(x), _ptr(Wg), _ptr(bg), _ptr(W1), _ptr(W2), _ptr(dout),
                                    aux_coef, z_coef, _ptr(fws), _nbytes(fws), _ptr(dx), _ptr(dWg), _ptr(dbg),
                                    _ptr(dW1), _ptr(dW2), _ptr(dw), _ptr(stats), _ptr(ws), _nbytes(ws),
                                    _stream(stream)))


def moe_convert_bf16_to_f16(src, dst, n: Optional[int] = None, stream=None):
    """Weight preparation: dst = fp16(src) for bf16 src (device tensors)."""
    n = src.numel() if n is None else n
    _check("moe_convert_bf16_to_f16", lib().moe_convert_bf16_to_f16(_ptr(src), _ptr(dst), n, _stream(stream)))


def prepare_w2(cfg: moe_config, w2):
    """W2 in the storage type the layer expects (a new fp16 tensor when the
    hidden activation is fp16, else w2 itself).  Run once at load time."""
    if cfg.hidden_dtype != MOE_DTYPE_F16:
        return w2
    import torch
    out = torch.empty(w2.shape, dtype=torch.float16, device=w2.device)
    moe_convert_bf16_to_f16(w2, out)
    return out


def read_stats(stats_tensor) -> dict:
    """Copy a device moe_stats (a uint8 tensor of sizeof(moe_stats) bytes) to a dict (synchronises)."""
    raw = bytes(stats_tensor.cpu().numpy().tobytes())
    s = moe_stats.from_buffer_copy(raw[:ctypes.sizeof(moe_stats)])
    return {f: getattr(s, f) for f, _ in moe_stats._fields_}


STATS_BYTES = ctypes.sizeof(moe_stats)
