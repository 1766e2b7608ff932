"""Parity at the full workload sizes, in the launch configuration bench.py times
(stem_score_select -> stem_bsa_fwd on one stream).

Every row is checked for what is cheap at any size: budgets and row pointers
bit-exact against the oracle's closed form; each list strictly ascending,
ending at the diagonal, containing the sink and window blocks; finite outputs.
Sampled (query head, query block) rows are checked against the fp64 oracle one
by one: the block-score row (1e-3 relative), the selected list (exact up to
near-ties), and the attention output and LSE of the row computed with the
GPU's list.

On the 32K and 128K workloads, one mu = 0.7 layer of the fp8 varlen stack and
the sparsest point of the 64K sweep, every row is also checked in full: the
oracle scores the whole layer (one KV head at a time, so the fp64 arrays stay
small) and selects every row, and every GPU list must equal the oracle's up to
near-ties, every GPU score row must be within 1e-3 of the oracle's.
"""

import math

import numpy as np
import pytest
import torch

from oracle import stem_oracle as O
from block_sparse_attention_stem_b200 import inputs as I
from gpu_common import TIE_REL, TOL_LSE, TOL_OUT, make_gpu_qkv, out_error, out_error_abs

pytestmark = pytest.mark.gpu

b = pytest.importorskip("block_sparse_attention_stem_b200.binding")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def _run(w):
    """The bench's step (stem_score_select, then stem_bsa_fwd); the selection
    inside the scoring kernel (select_mode 1) must give the same scores and
    lists."""
    inp = I.make_inputs(w, device="cuda")
    qkv = make_gpu_qkv(b, inp, w.cu_seqlens())
    params = b.make_params(**w.params())
    scores, budgets, row_ptr, col_idx, ws = b.stem_score_select(qkv, params)
    out, lse, _ = b.stem_bsa_fwd(qkv, params, row_ptr, col_idx, ws=ws)
    torch.cuda.synchronize()
    assert b.stem_read_device_status(ws) == 0
    s2, _, rp2, ci2, ws2 = b.stem_score_select(qkv, b.make_params(**w.params(), select_mode=1))
    torch.cuda.synchronize()
    assert b.stem_read_device_status(ws2) == 0
    assert torch.equal(s2.view(torch.int32), scores.view(torch.int32))
    assert torch.equal(rp2, row_ptr) and torch.equal(ci2, col_idx)
    del s2, rp2, ci2, ws2
    return inp, qkv, dict(scores=scores, budgets=budgets, row_ptr=row_ptr, col_idx=col_idx, out=out, lse=lse)


def _head_slices(inp, w, s, h):
    """fp64 single-head arrays of sequence s for query head h (and its KV head)."""
    cu = w.cu_seqlens()
    o, e = cu[s], cu[s + 1]
    G = w.num_q_heads // w.num_kv_heads
    hk = h // G

    def sl(name, c):
        x = inp[name][o:e, c:c + 1].contiguous().cpu()
        if w.dtype == "bf16":
            return O.dequant(I.raw_bits(x), "bf16")
        sc = inp[name + "_scale"][c:c + 1].cpu().numpy()
        return O.dequant(I.raw_bits(x), "fp8", sc)

    return sl("q", h), sl("k", hk), sl("v", hk)


def _group_arrays(inp, w, hk):
    """fp64 q [T, G, d] (the query heads of KV head hk), k and v [T, 1, d]
    over every token of every sequence."""
    G = w.num_q_heads // w.num_kv_heads

    def sl(name, c0, c1):
        x = inp[name][:, c0:c1].contiguous().cpu()
        if w.dtype == "bf16":
            return O.dequant(I.raw_bits(x), "bf16")
        sc = inp[name + "_scale"][c0:c1].cpu().numpy()
        return O.dequant(I.raw_bits(x), "fp8", sc)

    return sl("q", hk * G, (hk + 1) * G), sl("k", hk, hk + 1), sl("v", hk, hk + 1)


def _check_every_row(w, inp, res):
    """The oracle's scores and lists for every row of the layer, against the
    GPU's: scores within 1e-3 (relative above 1), lists equal up to near-ties
    (a swapped pair's oracle scores within TIE_REL), forced blocks present."""
    p = O.Params(**w.params())
    cu = w.cu_seqlens()
    seqs, nbtot = O.seq_blocks(cu, p.block_size)
    G = w.num_q_heads // w.num_kv_heads
    rp = res["row_ptr"].cpu().numpy().astype(np.int64)
    ci = res["col_idx"].cpu().numpy().astype(np.int64)
    gscores = res["scores"]
    ties = rows = 0
    worst = 0.0
    for hk in range(w.num_kv_heads):
        q, k, v = _group_arrays(inp, w, hk)
        S = O.block_scores(q, k, v, cu, p)  # [G, NBtot, nb_max]
        _, orp, oci = O.select(S, cu, p, hkv=1)
        ranked = O.group_pooled_scores(S, 1) if p.list_mode else S
        gs = gscores[hk * G:(hk + 1) * G].cpu().numpy().astype(np.float64)
        for (_, _, nb, g0) in seqs:
            for i in range(nb):
                a, r = gs[:, g0 + i, :i + 1], S[:, g0 + i, :i + 1]
                worst = max(worst, float((np.abs(a - r) / np.maximum(1.0, np.abs(r))).max()))
        for e in range(G):
            h = hk * G + e
            for (_, _, nb, g0) in seqs:
                for i in range(nb):
                    r, ro = h * nbtot + g0 + i, e * nbtot + g0 + i
                    Gl, Ol = ci[rp[r]:rp[r + 1]], oci[orp[ro]:orp[ro + 1]]
                    rows += 1
                    assert len(Gl) == len(Ol), (h, i)
                    if np.array_equal(Gl, Ol):
                        continue
                    X = set(Gl.tolist()) - set(Ol.tolist())
                    Y = set(Ol.tolist()) - set(Gl.tolist())
                    assert len(X) == len(Y)
                    row = ranked[e, g0 + i]
                    for x in X:
                        for y in Y:
                            assert abs(row[x] - row[y]) < TIE_REL * max(abs(row[x]), abs(row[y])), \
                                (h, i, x, y, row[x], row[y])
                    ties += 1
        del q, k, v, S
    assert worst <= 1e-3, worst
    total = w.num_q_heads * nbtot
    assert rows == total
    print(f"{w.name}: every row: {rows} lists, {rows - ties} identical to the oracle's, {ties} differ only by "
          f"near-ties; max score err {worst:.2e}")
    return ties


def _check_workload(w, samples, every_row=False):
    inp, qkv, res = _run(w)
    p = O.Params(**w.params())
    cu = w.cu_seqlens()
    B = p.block_size
    seqs, nbtot = O.seq_blocks(cu, B)
    hq = w.num_q_heads
    # --- every row: budgets, row pointers, list structure
    bud = O.budgets(cu, p)
    assert np.array_equal(res["budgets"].cpu().numpy(), np.tile(bud, hq))
    rp = res["row_ptr"].cpu().numpy().astype(np.int64)
    ci = res["col_idx"].cpu().numpy().astype(np.int64)
    exp_rp = np.concatenate([[0], np.cumsum(np.tile(bud, hq))])
    assert np.array_equal(rp, exp_rp)
    first = np.zeros(len(ci), dtype=bool)
    first[rp[:-1][rp[:-1] < len(ci)]] = True
    assert np.all((np.diff(ci) > 0) | first[1:])  # strictly ascending inside each row
    for (o, L, nb, g0) in seqs:
        i_of_row = np.arange(nb)
        last = ci[rp[np.arange(hq)[:, None] * nbtot + g0 + i_of_row[None, :] + 1] - 1]
        assert np.array_equal(last, np.broadcast_to(i_of_row, last.shape))  # the diagonal ends each row
    assert torch.isfinite(res["out"].float()).all()
    assert torch.isfinite(res["lse"]).all()
    G = hq // w.num_kv_heads
    if p.list_mode:  # shared lists: the rows of a group's query heads are identical
        for hk in range(w.num_kv_heads):
            r0 = rp[hk * G * nbtot:(hk * G + 1) * nbtot + 1]
            for e in range(1, G):
                re_ = rp[(hk * G + e) * nbtot:(hk * G + e + 1) * nbtot + 1]
                assert np.array_equal(ci[r0[0]:r0[-1]], ci[re_[0]:re_[-1]])
    # --- sampled rows against the oracle
    ties = 0
    worst = [0.0, 0.0, 0.0, 0.0, 0.0]
    cache = {}
    for (s, h, i) in samples:
        o, L, nb, g0 = seqs[s]
        if (s, h) not in cache:
            cache = {(s, h): _head_slices(inp, w, s, h)}
        qh, kh, vh = cache[(s, h)]
        r = h * nbtot + g0 + i
        ref_row = O.block_score_row(qh, kh, vh, i, p)
        gpu_row = res["scores"][h, g0 + i, :i + 1].cpu().numpy().astype(np.float64)
        sel_row = ref_row
        if p.list_mode:  # the list is selected on the group's elementwise max (NaN as -inf)
            hk0 = (h // G) * G
            rows = [ref_row if e == h else O.block_score_row(*_head_slices(inp, w, s, e), i, p)
                    for e in range(hk0, hk0 + G)]
            sel_row = np.max(np.where(np.isnan(rows), -np.inf, rows), axis=0)
        err = float(np.max(np.abs(gpu_row - ref_row) / np.maximum(1.0, np.abs(ref_row))))
        worst[0] = max(worst[0], err)
        assert err <= 1e-3, (s, h, i, err)
        G_list = ci[rp[r]:rp[r + 1]]
        O_list = np.array(O.select_row(sel_row, i, int(bud[g0 + i]), p.sink_blocks, p.window_blocks))
        if not np.array_equal(G_list, O_list):
            X = set(G_list.tolist()) - set(O_list.tolist())
            Y = set(O_list.tolist()) - set(G_list.tolist())
            assert len(X) == len(Y)
            for x in X:
                for y in Y:
                    assert abs(sel_row[x] - sel_row[y]) < TIE_REL * max(abs(sel_row[x]), abs(sel_row[y]))
            ties += 1
        # attention of the row with the GPU's list
        rp1 = np.zeros(nb + 1, dtype=np.int64)
        rp1[i + 1:] = len(G_list)
        ro, rl = O.bsa(qh, kh, vh, [0, L], rp1, G_list, p, rows_subset=[(0, i)])
        t0, t1 = i * B, min((i + 1) * B, L)
        go = res["out"][o + t0:o + t1, h].float().cpu().numpy().astype(np.float64)
        gl = res["lse"][h, o + t0:o + t1].cpu().numpy().astype(np.float64)
        e_o = out_error(go, ro[t0:t1, 0])
        raw, _, beyond = out_error_abs(go, ro[t0:t1, 0])
        e_l = float(np.max(np.abs(gl - rl[0, t0:t1])))
        worst[1] = max(worst[1], e_o)
        worst[2] = max(worst[2], e_l)
        worst[3] = max(worst[3], raw)
        worst[4] = max(worst[4], beyond)
        assert e_o <= TOL_OUT[w.dtype] and e_l <= TOL_LSE, (s, h, i, e_o, e_l)
        assert beyond <= TOL_OUT[w.dtype], (s, h, i, beyond, raw)
    print(f"{w.name}: rows={len(samples)} near-tie rows={ties} max score err={worst[0]:.2e} "
          f"max out err (scaled)={worst[1]:.2e} max|dO|={worst[3]:.2e} beyond the output's rounding="
          f"{worst[4]:.2e} max lse err={worst[2]:.2e}")
    if every_row:
        _check_every_row(w, inp, res)


def _samples(w, heads, per_seq_blocks):
    out = []
    for s, L in enumerate(w.seqlens):
        nb = math.ceil(L / w.block_size)
        blocks = sorted({min(nb - 1, x) for x in per_seq_blocks(nb)})
        for h in heads:
            for i in blocks:
                out.append((s, h, i))
    return out


def test_fullsize_qwen32k():
    w = I.workload("qwen32k")
    _check_workload(w, _samples(w, (0, 13, 31), lambda nb: (0, 1, 5, nb // 2, nb - 2, nb - 1)), every_row=True)


def test_fullsize_qwen32k_64_token_blocks():
    """The 32K workload with 64-token blocks (512 blocks per row): every list
    against the oracle; sampled rows of both halves of attention tiles."""
    w = I.workload("qwen32k", block_size=64)
    _check_workload(w, _samples(w, (0, 13, 31), lambda nb: (0, 1, 2, 7, nb // 2, nb // 2 + 1, nb - 2, nb - 1)),
                    every_row=True)


def test_fullsize_long128k_bench_workload():
    w = I.workload("long128k")
    _check_workload(w, _samples(w, (0, 17, 31), lambda nb: (0, 3, nb // 3, nb - 1)), every_row=True)


@pytest.mark.parametrize("layer", [0, 5])
def test_fullsize_fp8_varlen_layers(layer):
    w = I.workload("fp8_varlen", mu=I.fp8_layer_mu(layer), seed=4000 + layer)
    _check_workload(w, _samples(w, (0, 30), lambda nb: (0, nb // 2, nb - 1)), every_row=(layer == 5))


@pytest.mark.parametrize("rho", [1.0, 0.1])
def test_fullsize_sweep64k_extremes(rho):
    w = I.workload("sweep64k", keep_ratio=rho)
    _check_workload(w, _samples(w, (7,), lambda nb: (2, nb - 1)), every_row=(rho == 0.1))


def test_fullsize_long128k_64_token_blocks():
    """The bench workload with 64-token blocks (2048 blocks per row), sampled
    rows."""
    w = I.workload("long128k", block_size=64)
    _check_workload(w, _samples(w, (0, 31), lambda nb: (0, 5, nb // 2 + 1, nb - 1)))


def test_fullsize_long128k_shared_lists():
    """The bench workload with one list per KV group (list_mode 1): the
    attention runs two query heads per CTA over K/V staged once for both."""
    w = I.workload("long128k", list_mode=1)
    _check_workload(w, _samples(w, (1, 18), lambda nb: (0, nb // 2, nb - 1)))


def test_rows_longer_than_the_staged_list():
    """Rows with more than 2048 listed blocks (the attention kernel stages at
    most 2048 list entries in shared memory and walks longer lists in global
    memory): one 270K-token sequence at keep ratio 0.99 with a uniform budget."""
    nb = 2112
    w = I.Workload(name="long_rows", seqlens=[nb * 128], num_q_heads=2, num_kv_heads=1, seed=41, keep_ratio=0.99,
                   mu=1.0, beta=0.2, sink_blocks=1, window_blocks=2)
    assert O.budgets(w.cu_seqlens(), O.Params(**w.params()))[-1] > 2048
    _check_workload(w, [(0, 0, nb - 1), (0, 1, nb - 40)])
