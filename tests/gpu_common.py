"""Helpers shared by the GPU parity tests: run the CUDA library through its C
ABI, run the fp64 oracle on the same input bytes, compare."""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import stem_oracle as O
from block_sparse_attention_stem_b200 import inputs as I

TOL_OUT = {"bf16": 2e-2, "fp8": 6e-2}
TOL_LSE = 1e-3
TIE_REL = 1e-3


def to_device(inp: dict, dev="cuda"):
    out = {}
    for key, val in inp.items():
        out[key] = None if val is None else val.to(dev)
    return out


def oracle_arrays(inp: dict, dtype: str):
    """fp64 q, k, v exactly as the GPU sees them."""
    if dtype == "bf16":
        return tuple(O.dequant(I.raw_bits(inp[n]), "bf16") for n in ("q", "k", "v"))
    return tuple(O.dequant(I.raw_bits(inp[n]), "fp8", inp[n + "_scale"].numpy()) for n in ("q", "k", "v"))


def make_gpu_qkv(b, dinp: dict, cu):
    return b.make_qkv(dinp["q"], dinp["k"], dinp["v"], cu, q_scale=dinp["q_scale"], k_scale=dinp["k_scale"],
                      v_scale=dinp["v_scale"], cu_seqlens_dev=dinp["cu_seqlens"])


def check_scores(gpu: np.ndarray, ref: np.ndarray, cu, block=128):
    """Entries j <= i within tolerance; entries above the diagonal -inf."""
    seqs, _ = O.seq_blocks(cu, block)
    worst = 0.0
    for (_, _, nb, g0) in seqs:
        for i in range(nb):
            a = gpu[:, g0 + i, :i + 1]
            r = ref[:, g0 + i, :i + 1]
            err = np.abs(a - r) / np.maximum(1.0, np.abs(r))
            worst = max(worst, float(err.max()))
            assert np.all(gpu[:, g0 + i, i + 1:] == -np.inf)
    assert worst <= 1e-3, worst
    return worst


def compare_lists(rp_g, ci_g, rp_o, ci_o, ref_scores, cu, hq, sink, window, block=128):
    """Budgets/row_ptr must match exactly; within a row the sets may differ only
    by swaps between blocks whose oracle scores are within TIE_REL of each
    other.  Returns the number of rows that needed the near-tie allowance."""
    assert np.array_equal(rp_g, rp_o)
    seqs, nbtot = O.seq_blocks(cu, block)
    ties = 0
    for h in range(hq):
        for (_, _, nb, g0) in seqs:
            for i in range(nb):
                r = h * nbtot + g0 + i
                G = ci_g[rp_g[r]:rp_g[r + 1]]
                Os = ci_o[rp_o[r]:rp_o[r + 1]]
                assert np.all(np.diff(G) > 0) and G.max() == i
                assert set(O.forced_blocks(i, sink, window)) <= set(G.tolist())
                if np.array_equal(G, Os):
                    continue
                X = set(G.tolist()) - set(Os.tolist())
                Y = set(Os.tolist()) - set(G.tolist())
                assert len(X) == len(Y)
                row = ref_scores[h, g0 + i]
                for x in X:
                    for y in Y:
                        sx, sy = row[x], row[y]
                        assert abs(sx - sy) < TIE_REL * max(abs(sx), abs(sy)), (h, i, x, y, sx, sy)
                ties += 1
    return ties


def out_error(og, oo):
    """Output error scaled by max(1, |O_ref|): absolute where |O| <= 1 and
    relative above (reported beside the checked figures below)."""
    return float((np.abs(og - oo) / np.maximum(1.0, np.abs(oo))).max())


def bf16_rounding_interval(og):
    """[lo, hi]: the reals that round (to nearest) to each bf16 value in og.
    The bounds are the midpoints to the neighbouring bf16 values, taken from
    the bit pattern (the encoding is sign-magnitude)."""
    og = np.asarray(og, dtype=np.float64)
    bits = (og.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.int64)
    assert np.array_equal(((bits << 16).astype(np.uint32)).view(np.float32).astype(np.float64), og), \
        "not bf16 values"
    mag = bits & 0x7FFF
    sign = np.where(bits & 0x8000, -1.0, 1.0)

    def val(m):
        return ((m.astype(np.uint32) << np.uint32(16)).view(np.float32)).astype(np.float64)

    a = np.abs(og)
    up = (a + val(np.minimum(mag + 1, 0x7F7F))) / 2
    dn = np.where(mag > 0, (a + val(np.maximum(mag - 1, 0))) / 2, 0.0)
    lo = np.where(sign > 0, dn, -up)
    hi = np.where(sign > 0, up, -dn)
    return lo, hi


def out_error_abs(og, oo):
    """Absolute output errors: (max |O_gpu - O_ref|, max |O_gpu - bf16(O_ref)|,
    max distance from O_ref to the set of reals that round to O_gpu).  The
    last one is what the max-abs bound is checked on: the GPU's output is a bf16
    number, so the claim is that some value within the bound of the exact
    result rounds to it — the part of |O_gpu - O_ref| that is the output's own
    rounding (up to half a bf16 step, 2^-9 |O|) is not counted against the
    arithmetic."""
    og = np.asarray(og, dtype=np.float64)
    oo = np.asarray(oo, dtype=np.float64)
    raw = float(np.abs(og - oo).max()) if og.size else 0.0
    rounded_ref = oo.astype(np.float32)
    rounded_ref = (rounded_ref.view(np.uint32).astype(np.uint64) + 0x7FFF
                   + ((rounded_ref.view(np.uint32) >> 16) & 1)) >> 16  # RNE to bf16
    rounded_ref = ((rounded_ref.astype(np.uint32) << np.uint32(16)).view(np.float32)).astype(np.float64)
    vs_rounded = float(np.abs(og - rounded_ref).max()) if og.size else 0.0
    lo, hi = bf16_rounding_interval(og)
    dist = np.maximum(np.maximum(lo - oo, oo - hi), 0.0)
    return raw, vs_rounded, (float(dist.max()) if og.size else 0.0)


def check_attention(out_g, lse_g, out_o, lse_o, dtype, rows_mask=None):
    og = out_g.float().cpu().numpy().astype(np.float64)
    lg = lse_g.cpu().numpy().astype(np.float64)
    if rows_mask is not None:
        og, out_o = og[rows_mask], out_o[rows_mask]
        lg, lse_o = lg[:, rows_mask], lse_o[:, rows_mask]
    err = out_error(og, out_o)
    raw, vs_rounded, beyond_rounding = out_error_abs(og, out_o)
    lerr = float(np.abs(lg - lse_o).max())
    print(f"[{dtype}] max|dO| {raw:.3e}  vs bf16(O_ref) {vs_rounded:.3e}  beyond the output's rounding "
          f"{beyond_rounding:.3e}  scaled {err:.3e}  max|dLSE| {lerr:.3e}")
    assert beyond_rounding <= TOL_OUT[dtype], (beyond_rounding, raw, vs_rounded)
    assert err <= TOL_OUT[dtype], (err, raw)
    assert lerr <= TOL_LSE, lerr
    return err, lerr


def oparams(w: I.Workload) -> O.Params:
    return O.Params(**w.params())
