"""Helpers shared by the GPU parity tests: upload a workload, run the layer
through the C ABI (step by step or whole), read results back, and compare
with the float64 oracle under the stated tolerances.

Tolerances:
* routing indices, per-expert counts, permutation and drop mask: bit-exact,
  except tokens whose oracle k-th/(k+1)-th score gap is below 1e-4 (near
  ties); those take the device's selection in the oracle (forced routing) and
  everything downstream is then compared exactly over all tokens;
* bf16 outputs: max|err| <= 2e-2 * RMS(oracle output);
* fp32 outputs: max|err| / max|oracle| <= 1e-4 (a norm-wise relative error;
  the element-wise |err| / max(|ref|, 1e-3 RMS) is printed beside it).
"""
from __future__ import annotations

import numpy as np
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
import oracle
from oracle import moe_oracle as om

NEAR_TIE = 1e-4
BF16_TOL = 2e-2     # x RMS(out)
F32_TOL = 1e-4      # relative to max |out|


def cfg_of(w: mw.Workload, T=None, hidden=None):
    return moe.make_config(w.T if T is None else T, w.d, w.E, w.F, w.k, w.act, w.dtype, w.capacity_factor, w.lam,
                           hidden)


def lcfg_of(w: mw.Workload, T=None):
    return oracle.LayerConfig.from_workload(w, T)


def dev_bytes(n):
    return torch.empty(max(int(n), 256), dtype=torch.uint8, device="cuda")


def view(ws, off, n, dtype):
    es = torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + n * es].view(dtype)


class DeviceLayer:
    """One workload's inputs on the device plus the outputs of a forward."""

    def __init__(self, w: mw.Workload, inp: mw.Inputs = None, hidden=None):
        self.w = w
        self.inp = inp if inp is not None else mw.generate(w)
        self.cfg = cfg_of(w, self.inp.x.shape[0], hidden)
        self.hidden = {moe.MOE_DTYPE_F16: "f16", moe.MOE_DTYPE_BF16: "bf16"}.get(self.cfg.hidden_dtype, "f32")
        self.T = self.inp.x.shape[0]
        self.x = mw.to_device(self.inp.x)
        self.wg = mw.to_device(self.inp.wg)
        self.bias = mw.to_device(self.inp.bias)
        self.w1 = mw.to_device(self.inp.w1)
        self.w2 = moe.prepare_w2(self.cfg, mw.to_device(self.inp.w2))   # weight preparation, once
        self.tdt = torch.bfloat16 if w.dtype == mw.BF16 else torch.float32
        self.hdt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[self.hidden]

    # ---------------------------------------------------------- whole layer
    def forward(self, poison=None):
        """poison: a byte value the workspace and out are filled with first."""
        n, L = moe.moe_workspace_size(self.cfg)
        assert n > 0
        ws = dev_bytes(n)
        out = torch.empty((self.T, self.w.d), dtype=torch.float32, device="cuda")
        if poison is not None:
            ws.fill_(poison)
            out.view(torch.uint8).fill_(poison)
        stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
        moe.moe_layer_forward(self.cfg, self.x, self.wg, self.bias, self.w1, self.w2, out, stats, ws)
        torch.cuda.synchronize()
        T, k, E, A = self.T, self.w.k, self.w.E, self.T * self.w.k
        r = dict(out=out, stats=moe.read_stats(stats), ws=ws, layout=L)
        r["topk_idx"] = view(ws, L.topk_idx, A, torch.int32).view(T, k).cpu().numpy()
        r["topk_w"] = view(ws, L.topk_w, A, torch.float32).view(T, k).cpu().numpy()
        r["gap"] = view(ws, L.gap, T, torch.float32).cpu().numpy()
        r["counts"] = view(ws, L.counts, E, torch.int32).cpu().numpy()
        r["kept"] = view(ws, L.kept, E, torch.int32).cpu().numpy()
        r["offsets"] = view(ws, L.offsets, E + 1, torch.int32).cpu().numpy()
        r["row_of"] = view(ws, L.row_of, A, torch.int32).view(T, k).cpu().numpy()
        nk = int(r["offsets"][-1])
        r["src_tok"] = view(ws, L.src_tok, nk, torch.int32).cpu().numpy()
        return r

    # ------------------------------------------------------------ the steps
    def scratch(self):
        return dev_bytes(moe.moe_scratch_size(self.cfg))

    def route(self, want_prob_mean=True, want_z_loss=False):
        T, k, E = self.T, self.w.k, self.w.E
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
        gap = torch.empty((T,), dtype=torch.float32, device="cuda")
        pm = torch.empty((E,), dtype=torch.float32, device="cuda") if want_prob_mean else None
        zl = torch.empty((1,), dtype=torch.float32, device="cuda") if want_z_loss else None
        moe.moe_route(self.cfg, self.x, self.wg, self.bias, idx, wt, gap, pm, self.scratch(), z_loss=zl)
        if want_z_loss:
            return idx, wt, gap, pm, zl
        return idx, wt, gap, pm

    def permute(self, idx, gap=None, prob_mean=None):
        T, k, E, d = self.T, self.w.k, self.w.E, self.w.d
        A = T * k
        counts = torch.empty(E, dtype=torch.int32, device="cuda")
        kept = torch.empty(E, dtype=torch.int32, device="cuda")
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        row_of = torch.empty((T, k), dtype=torch.int32, device="cuda")
        src_tok = torch.full((max(A, 1),), -7, dtype=torch.int32, device="cuda")
        xp = torch.empty((max(A, 1), d), dtype=self.tdt, device="cuda")
        stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
        moe.moe_permute(self.cfg, self.x, idx, gap, prob_mean, counts, kept, offsets, row_of, src_tok, xp, stats,
                        self.scratch())
        return dict(counts=counts, kept=kept, offsets=offsets, row_of=row_of, src_tok=src_tok, xp=xp, stats=stats)

    def expert_ffn(self, xp, offsets):
        A = max(self.T * self.w.k, 1)
        h = torch.empty((A, self.w.F), dtype=self.hdt, device="cuda")
        yp = torch.empty((A, self.w.d), dtype=torch.float32, device="cuda")
        stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
        moe.moe_expert_ffn(self.cfg, xp, offsets, self.w1, self.w2, h, yp, stats, self.scratch())
        return h, yp, stats

    def combine(self, yp, row_of, topk_w):
        out = torch.empty((self.T, self.w.d), dtype=torch.float32, device="cuda")
        moe.moe_combine(self.cfg, yp, row_of, topk_w, out)
        return out


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


# ----------------------------------------------------------------- checks
def near_tie_mask(r: om.Routing) -> np.ndarray:
    return r.gap < NEAR_TIE


def order_unique_mask(r: om.Routing) -> np.ndarray:
    """Tokens whose selected scores are pairwise >= 1e-4 apart, so the order of
    the selection (best first) is decided beyond fp32 rounding."""
    s_sel = np.take_along_axis(r.s, r.idx, axis=1)
    if s_sel.shape[1] < 2:
        return np.ones(s_sel.shape[0], bool)
    return np.all(-np.diff(s_sel, axis=1) >= NEAR_TIE, axis=1)


def check_routing(dev_idx: np.ndarray, r: om.Routing):
    """Returns (forced_mask, n_near_tie): asserts exact agreement off near ties."""
    nt = near_tie_mask(r)
    ou = order_unique_mask(r)
    exact = ~nt
    a = np.sort(dev_idx[exact], axis=1)
    b = np.sort(r.idx[exact], axis=1)
    bad = np.nonzero(np.any(a != b, axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens with a decided top-k differ, e.g. token {np.nonzero(exact)[0][bad[0]]}"
    oo = exact & ou
    assert np.array_equal(dev_idx[oo], r.idx[oo]), "selection order differs where it is decided"
    return nt, int(nt.sum())


def check_dispatch_exact(dev: dict, d: om.Dispatch, r: om.Routing, dev_idx: np.ndarray):
    """counts, kept, offsets, src_tok exact; row_of exact per (token, expert)."""
    assert np.array_equal(dev["counts"], d.counts), "counts"
    assert np.array_equal(dev["kept"], d.kept), "kept"
    assert np.array_equal(dev["offsets"], d.offsets), "offsets"
    n = int(d.offsets[-1])
    assert np.array_equal(dev["src_tok"][:n], d.src_tok), "src_tok"
    # row_of: compare as a map (token, expert) -> row, since slot order may
    # legitimately differ where selected scores are within rounding
    T, k = dev_idx.shape
    for name, idx_, rows_ in (("dev", dev_idx, dev["row_of"]), ("oracle", r.idx, d.row_of)):
        assert idx_.shape == rows_.shape, name
    key_dev = {(t, int(dev_idx[t, j])): int(dev["row_of"][t, j]) for t in range(T) for j in range(k)}
    key_ref = {(t, int(r.idx[t, j])): int(d.row_of[t, j]) for t in range(T) for j in range(k)}
    assert key_dev == key_ref, "row_of / drop mask"


def check_out(out_dev: np.ndarray, out_ref: np.ndarray, dtype: str, tol=BF16_TOL):
    """max|err| against the bar of the path's type: bf16 paths within tol *
    RMS(out) (tol None: measured, not asserted), fp32 paths within F32_TOL *
    max|out|.  Returns the error over the bar's scale."""
    if out_ref.size == 0:
        return 0.0
    err = np.max(np.abs(out_dev - out_ref))
    if dtype == mw.BF16:
        rms = float(np.sqrt(np.mean(out_ref ** 2)))
        assert tol is None or err <= tol * rms, f"max|err| {err:.3e} > {tol} * RMS {rms:.3e}"
        return err / rms
    scale = float(np.max(np.abs(out_ref)))
    assert err <= F32_TOL * scale, f"max|err| {err:.3e} > {F32_TOL} * max|ref| {scale:.3e}"
    # element-wise relative error with a floor of 1e-3 RMS, reported beside the bar
    rms = float(np.sqrt(np.mean(out_ref ** 2)))
    elem = float(np.max(np.abs(out_dev - out_ref) / np.maximum(np.abs(out_ref), 1e-3 * rms)))
    print(f"fp32 parity: max|err|/max|ref| = {err / scale:.2e}, element-wise (floor 1e-3 RMS) = {elem:.2e}")
    return err / scale
