"""Host-side checks of the C ABI (no GPU needed, no compute call made).

The library must load, export every function include/moe.h declares, size its
workspaces consistently, and reject bad arguments synchronously -- before any
CUDA call -- with the documented status codes."""
import ctypes
import os
import re

import pytest

import mixture_experts_layer_logit_b200 as moe
from mixture_experts_layer_logit_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|size_t|moe_status)\s+(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ["moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward"]:
        assert name in fns
    assert sorted(moe.EXPORTED_SYMBOLS) == fns


def test_library_exports_every_declared_symbol(L):
    for name in header_functions():
        assert hasattr(L, name), name
    # and nothing is linked against libcuda / libtorch: check the dynamic deps
    import subprocess
    out = subprocess.run(["ldd", moe.LIB_PATH], capture_output=True, text=True).stdout
    assert "libtorch" not in out and "libcudart.so" not in out


def test_struct_sizes_match_header(L):
    assert ctypes.sizeof(moe.moe_config) == 10 * 4
    assert ctypes.sizeof(moe.moe_stats) == 8 * 4
    assert ctypes.sizeof(moe.moe_ws_layout) == 14 * 8


def test_status_strings(L):
    for code in range(5):
        assert moe.moe_status_string(code).startswith(moe.STATUS_NAMES[code])
    assert moe.moe_status_string(99) == "unknown moe_status"


def cfg(**kw):
    base = dict(T=100, d=64, E=8, F=128, k=2, act="relu", dtype="bf16", capacity_factor=1.0, lam=0.0)
    base.update(kw)
    return moe.make_config(**base)


@pytest.mark.parametrize("bad", [dict(k=9), dict(k=0), dict(T=-1), dict(d=0), dict(E=0), dict(F=0),
                                 dict(capacity_factor=float("nan")), dict(lam=float("inf"))])
def test_invalid_config_sizes_zero(L, bad):
    assert moe.moe_scratch_size(cfg(**bad)) == 0
    assert moe.moe_workspace_size(cfg(**bad))[0] == 0


@pytest.mark.parametrize("bad", [dict(E=257), dict(d=72), dict(F=40), dict(dtype="f32", d=66)])
def test_unsupported_config(L, bad):
    c = cfg(**bad)
    assert moe.moe_scratch_size(c) == 0
    # a step call reports the reason synchronously, before touching the device
    code = L.moe_combine(ctypes.byref(c), None, None, None, None, None)
    assert code == 2


def test_bad_enum_is_arg_error(L):
    c = cfg()
    c.act = 7
    assert L.moe_combine(ctypes.byref(c), None, None, None, None, None) == 1
    for dtype, hidden in [("bf16", "f32"), ("f32", "bf16"), ("f32", "f16")]:
        c = cfg(dtype=dtype, hidden=hidden)
        assert moe.moe_scratch_size(c) == 0
        assert L.moe_combine(ctypes.byref(c), None, None, None, None, None) == 1
    for hidden in ["bf16", "f16"]:
        assert moe.moe_scratch_size(cfg(hidden=hidden)) > 0
    c = cfg()
    c.dtype = 5
    assert L.moe_layer_forward(ctypes.byref(c), None, None, None, None, None, None, None, None, 0, None) == 1
    assert L.moe_route(None, None, None, None, None, None, None, None, None, None, 0, None) == 1


def test_null_and_misaligned_pointers(L):
    c = cfg()
    P = 1 << 20  # an aligned non-null stand-in: never dereferenced, the calls fail earlier
    # required pointers missing
    assert L.moe_route(ctypes.byref(c), None, P, None, P, P, P, None, None, P, 1 << 20, None) == 1
    assert L.moe_permute(ctypes.byref(c), P, P, None, None, P, P, P, P, P, P, None, P, 1 << 20, None) == 1
    assert L.moe_expert_ffn(ctypes.byref(c), P, None, P, P, P, P, P, P, 1 << 20, None) == 1
    # misaligned activations (TMA and 16-byte vectors need 16-byte alignment)
    assert L.moe_route(ctypes.byref(c), P + 8, P, None, P, P, P, None, None, P, 1 << 20, None) == 1
    assert L.moe_route(ctypes.byref(c), P, P, None, P, P, P, None, P + 2, P, 1 << 20, None) == 1   # z_loss misaligned
    assert L.moe_combine(ctypes.byref(c), P + 4, P, P, P, None) == 1


def test_fused_expert_combine_limits(L):
    P = 1 << 20
    for bad in [cfg(k=3, E=8), cfg(dtype="f32", d=64, F=128)]:
        full, _ = moe.moe_workspace_size(bad)
        assert L.moe_expert_ffn_combine(ctypes.byref(bad), P, P, P, P, P, P, P, P, P, P, full, None) == 2
    c = cfg(k=2)
    full, _ = moe.moe_workspace_size(c)
    assert L.moe_expert_ffn_combine(ctypes.byref(c), P, P, P, None, P, P, P, P, P, P, full, None) == 1   # no row_w
    assert L.moe_expert_ffn_combine(ctypes.byref(c), P, P, P, P, P, P, P, P, P, P, full - 1, None) == 3


def test_convert_rejects_bad_pointers(L):
    P = 1 << 20
    assert L.moe_convert_bf16_to_f16(None, P, 8, None) == 1
    assert L.moe_convert_bf16_to_f16(P + 2, P + 4096, 8, None) == 1   # misaligned
    assert L.moe_convert_bf16_to_f16(P, P + 8, 64, None) == 1         # overlapping
    assert L.moe_convert_bf16_to_f16(None, None, 0, None) == 0        # nothing to do


def test_workspace_checks(L):
    c = cfg()
    need = moe.moe_scratch_size(c)
    P = 1 << 20
    assert L.moe_route(ctypes.byref(c), P, P, None, P, P, P, None, None, None, need, None) == 3
    assert L.moe_route(ctypes.byref(c), P, P, None, P, P, P, None, None, P, need - 1, None) == 3
    assert L.moe_route(ctypes.byref(c), P, P, None, P, P, P, None, None, P + 16, need, None) == 3   # not 256-aligned
    full, layout = moe.moe_workspace_size(c)
    assert L.moe_layer_forward(ctypes.byref(c), P, P, None, P, P, P, P, P, full - 1, None) == 3


def test_workspace_layout_is_disjoint_and_aligned(L):
    for kw in [dict(), dict(T=32768, d=2048, E=64, F=1408, k=6, act="swiglu"), dict(T=1, E=1, k=1),
               dict(dtype="f32", d=64, F=96, T=300, E=5)]:
        c = cfg(**kw)
        total, lay = moe.moe_workspace_size(c)
        T, k, E, d, F = c.T, c.k, c.E, c.d, c.F
        es = 2 if c.dtype == moe.MOE_DTYPE_BF16 else 4
        A = T * k
        regions = [("topk_idx", 4 * A), ("topk_w", 4 * A), ("gap", 4 * T), ("counts", 4 * E), ("kept", 4 * E),
                   ("offsets", 4 * (E + 1)), ("row_of", 4 * A), ("src_tok", 4 * A), ("row_w", 4 * A),
                   ("xp", es * A * d),
                   ("h", es * A * F), ("yp", 4 * A * d), ("scratch", moe.moe_scratch_size(c))]
        spans = sorted((getattr(lay, n), getattr(lay, n) + sz, n) for n, sz in regions)
        for (a0, a1, an), (b0, b1, bn) in zip(spans, spans[1:]):
            assert a1 <= b0, (an, bn)
        for a0, a1, n in spans:
            assert a0 % 256 == 0, n
            assert a1 <= total
        assert lay.total == total


def test_scratch_grows_with_tokens(L):
    assert moe.moe_scratch_size(cfg(T=64)) < moe.moe_scratch_size(cfg(T=64 * 100))
    assert moe.moe_scratch_size(cfg(T=0)) > 0


def _max_tokens(limit, **kw):
    """Largest T whose scratch fits in `limit` bytes (binary search on the host size function)."""
    lo, hi = 1, 1 << 22
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if moe.moe_scratch_size(cfg(T=mid, **kw)) <= limit:
            lo = mid
        else:
            hi = mid - 1
    return lo


def test_static_scratch_limit_as_documented(L):
    # include/moe.h: E = 64, k = 2 fits about 342k tokens on the bf16 path
    # (its scratch also holds the expert kernel's tile-queue counters) and
    # 345k on fp32
    limit = 2 << 20
    t_bf16 = _max_tokens(limit, d=512, E=64, F=1024, k=2)
    t_f32 = _max_tokens(limit, d=512, E=64, F=1024, k=2, dtype="f32")
    assert abs(t_bf16 - 342_000) < 1_000, t_bf16
    assert abs(t_f32 - 345_000) < 1_000, t_f32


def test_route_scratch_holds_no_partial_logits(L):
    # the gate GEMM's model-width split (decode: 8 slices of one chunk) sums
    # its partial logits inside a thread-block cluster, through distributed
    # shared memory, so the scratch is the per-chunk tables and the
    # tile-queue counters alone (a few 256-byte alignment pads aside) on
    # every layer, split or not
    for T, d, F, k, act in ((64, 2048, 1408, 6, "swiglu"), (8192, 512, 1024, 2, "relu"),
                            (16384, 2048, 1408, 6, "swiglu"), (64, 512, 1408, 6, "swiglu")):
        s = moe.moe_scratch_size(cfg(T=T, d=d, E=64, F=F, k=k, act=act))
        nch = (T + 127) // 128
        tables = 4 * (3 * 64 * nch + nch + 1) + 4 * (2 + T * k // 128 + 64)
        assert s <= tables + 8 * 256, (T, d, s, tables)
    assert moe.moe_scratch_size(cfg(T=64, d=2048, E=64, F=1408, k=6, act="swiglu")) < 8 * 128 * 64 * 4


def test_adaptive_aux_coef_on_the_host_follows_the_oracle(L):
    """moe_aux_coef_next against the oracle's coefficient step over a scripted
    drop-rate sequence: the coefficient rises while the drop rate is high and
    falls once it drops."""
    from oracle import moe_oracle as om
    beta, xi = 0.9, 0.5
    rates = [0.30, 0.30, 0.25, 0.20, 0.05, 0.01, 0.0, 0.0, 0.12, 0.4]
    a_lib = a_ref = 0.01
    seq = []
    for d in rates:
        a_lib = moe.moe_aux_coef_next(a_lib, d, beta, xi)
        a_ref = om.adaptive_aux_coef(a_ref, d, beta, xi)
        assert abs(a_lib - a_ref) <= 1e-6 * max(1.0, abs(a_ref)), (d, a_lib, a_ref)
        seq.append(a_lib)
    assert seq[0] > 0.01 and seq[3] > seq[0]           # raised while many tokens drop
    assert seq[7] < seq[4]                              # lowered once the drop rate falls
    assert seq[9] > seq[8] > seq[7]                     # raised again


@pytest.mark.parametrize("args", [(0.1, -0.1, 0.9, 1.0), (0.1, 1.5, 0.9, 1.0), (0.1, 0.2, 1.5, 1.0),
                                  (0.1, 0.2, -0.1, 1.0), (0.1, 0.2, 0.9, -1.0), (float("nan"), 0.2, 0.9, 1.0),
                                  (0.1, 0.2, 0.9, float("inf"))])
def test_adaptive_aux_coef_rejects_bad_values(L, args):
    out = ctypes.c_float(-7.0)
    assert L.moe_aux_coef_next(*[ctypes.c_float(v) for v in args], ctypes.byref(out)) == 1
    assert out.value == -7.0
    assert L.moe_aux_coef_next(ctypes.c_float(0.1), ctypes.c_float(0.2), ctypes.c_float(0.9), ctypes.c_float(1.0),
                               None) == 1
    assert L.moe_aux_coef_update(None, None, ctypes.c_float(0.9), ctypes.c_float(1.0), None) == 1


def test_shared_expert_workspace_sizes(L):
    cfg = moe.make_config(64, 128, 4, 128, 2, "relu")
    assert moe.moe_workspace_size_shared(cfg, 0) == 0
    assert moe.moe_workspace_size_shared(cfg, 100) == 0          # not a multiple of 16 on the bf16 path
    assert moe.moe_workspace_size_shared(cfg, 128) > moe.moe_workspace_size(cfg)[0]


def test_mxfp8_shapes(L):
    ok = moe.make_config(64, 2048, 64, 1408, 6, "swiglu")
    n, (a, b, c, d) = moe.moe_mxfp8_weight_bytes(ok)
    assert a == 64 * 2816 * 2048 and c == 64 * 2048 * 1408
    assert b == a // 32 and d == c // 32 and n == a + b + c + d
    assert moe.moe_workspace_size_mxfp8(ok) > moe.moe_workspace_size(ok)[0]
    for bad in [moe.make_config(64, 192, 4, 256, 2, "relu"),               # d not a multiple of 128
                moe.make_config(64, 256, 4, 192, 2, "relu"),               # F not a multiple of 128
                moe.make_config(64, 256, 4, 256, 2, "relu", dtype="f32")]:
        assert moe.moe_workspace_size_mxfp8(bad) == 0
        assert moe.moe_mxfp8_weight_bytes(bad)[0] == 0
