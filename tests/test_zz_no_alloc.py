"""moe_permute_static: moe_permute with its scratch in the library's fixed
device array instead of a caller workspace.

The GPU test runs two such calls in a row, on two different layers (the
second with more experts, more chunks and a different capacity mode, so that
anything the first call left in the array would show), and compares every
output with the workspace entry point moe_permute on the same inputs, bit for
bit.  Outputs and stats are filled with garbage before each static call, so
that a value it fails to write (or to clear, for stats.status) shows too.
The file is named to be collected last: it must pass alone and after the
other tests, whatever they left on the device.  The CPU tests check that sizes
over the fixed array are rejected before any device work."""
import ctypes

import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
from mixture_experts_layer_logit_b200 import build as moe_build

W = mw.Workload
LAYERS = [
    W("na_relu_cap", T=777, d=256, E=12, F=320, k=3, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.1, seed=41),
    W("na_fine_dropless", T=2500, d=128, E=64, F=176, k=6, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True,
      seed=42),
]


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def cfg(**kw):
    base = dict(T=100, d=64, E=64, F=128, k=2, act="relu", dtype="bf16", capacity_factor=1.0, lam=0.0)
    base.update(kw)
    return moe.make_config(**base)


def largest_T(E):
    """Largest T whose scratch fits the fixed array, by bisection on moe_scratch_size."""
    lo, hi = 0, 1 << 22
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if moe.moe_scratch_size(cfg(T=mid, E=E)) <= moe.MOE_STATIC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid - 1
    return lo


def test_rejects_sizes_over_the_array(L):
    P = 1 << 20   # aligned non-null stand-ins, never dereferenced: the call fails first
    for E in (8, 64, 256):
        T = largest_T(E)
        assert T > 10000
        over = cfg(T=T + 128, E=E)
        assert moe.moe_scratch_size(over) > moe.MOE_STATIC_SCRATCH_BYTES
        code = L.moe_permute_static(ctypes.byref(over), P, P, None, None, P, P, P, P, P, P, P, None)
        assert code == 2   # MOE_ERR_UNSUPPORTED
        with pytest.raises(moe.MoeError, match="UNSUPPORTED"):
            moe.moe_permute_static(over, P, P, None, None, P, P, P, P, P, P, P, stream=0)
    # the limit stated in the header for E = 64
    assert 340_000 < largest_T(64) < 350_000


def test_argument_checks_match_moe_permute(L):
    c = cfg()
    P = 1 << 20
    assert L.moe_permute_static(ctypes.byref(c), P, P, None, None, P, P, P, P, P, P, None, None) == 1   # no stats
    assert L.moe_permute_static(ctypes.byref(c), P + 8, P, None, None, P, P, P, P, P, P, P, None) == 1  # misaligned x
    assert L.moe_permute_static(None, P, P, None, None, P, P, P, P, P, P, P, None) == 1


def _outputs(T, k, E, d, tdt, fill):
    A = max(T * k, 1)
    return dict(counts=torch.full((E,), fill, dtype=torch.int32, device="cuda"),
                kept=torch.full((E,), fill, dtype=torch.int32, device="cuda"),
                offsets=torch.full((E + 1,), fill, dtype=torch.int32, device="cuda"),
                row_of=torch.full((T, k), fill, dtype=torch.int32, device="cuda"),
                src_tok=torch.full((A,), fill, dtype=torch.int32, device="cuda"),
                xp=torch.full((A, d), float(fill), dtype=tdt, device="cuda"),
                stats=torch.full((moe.STATS_BYTES,), 0xFF, dtype=torch.uint8, device="cuda"))


@pytest.mark.gpu
def test_two_static_calls_match_moe_permute():
    from gpu_harness import DeviceLayer
    for w in LAYERS:
        lay = DeviceLayer(w)
        T, k, E, d = lay.T, w.k, w.E, w.d
        idx, _, gap, pm = lay.route()
        ref = lay.permute(idx, gap, pm)
        got = _outputs(T, k, E, d, lay.tdt, -3)
        moe.moe_permute_static(lay.cfg, lay.x, idx, gap, pm, got["counts"], got["kept"], got["offsets"],
                               got["row_of"], got["src_tok"], got["xp"], got["stats"])
        torch.cuda.synchronize()
        for name in ("counts", "kept", "offsets", "row_of"):
            assert torch.equal(got[name], ref[name]), (w.name, name)
        # every moe_stats field, bit for bit (z_loss is NaN from both: a
        # standalone permutation has no router scores)
        assert torch.equal(got["stats"], ref["stats"]), w.name
        rows = int(ref["offsets"][E].item())
        assert rows > 0
        assert torch.equal(got["src_tok"][:rows], ref["src_tok"][:rows]), w.name
        assert torch.equal(got["xp"][:rows].view(torch.int16), ref["xp"][:rows].view(torch.int16)), w.name
        st = moe.read_stats(got["stats"])
        assert st["status"] == 0 and st["rows_kept"] == rows, (w.name, st)
