"""GPU parity: the CUDA library (called through its C ABI) against the fp64
oracle on the same seeded input bytes.

Acceptance (block scores relative 1e-3; budgets and row pointers bit-exact;
block lists bit-exact except at documented near-ties; attention output within
2e-2 (bf16) / 6e-2 (fp8) max-abs and LSE within 1e-3, computed with the GPU's
block lists).
"""

import numpy as np
import pytest
import torch

from oracle import stem_oracle as O
from block_sparse_attention_stem_b200 import inputs as I
from gpu_common import (check_attention, check_scores, compare_lists, make_gpu_qkv, oparams, oracle_arrays,
                        to_device)

pytestmark = pytest.mark.gpu

b = pytest.importorskip("block_sparse_attention_stem_b200.binding")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def W(seqlens, hq, hkv, dtype="bf16", seed=10, **kw):
    base = dict(keep_ratio=0.4, mu=0.7, beta=0.2, sink_blocks=1, window_blocks=2)
    base.update(kw)
    return I.Workload(name="case", seqlens=seqlens, num_q_heads=hq, num_kv_heads=hkv, dtype=dtype, seed=seed,
                      **base)


CASES = {
    "tiny": I.workload("tiny"),
    "one_block": W([128], 1, 1, keep_ratio=0.5, sink_blocks=1, window_blocks=1),
    "gqa4_ragged": W([1000], 4, 1, seed=11),
    "odd_len": W([1001], 2, 2, seed=12, stride=8),
    "varlen": W([1000, 128, 2088], 8, 2, seed=13, sink_blocks=2, window_blocks=1),
    "stride4": W([1536], 2, 1, seed=14, stride=4),
    "multi_tile": W([4096 + 640], 4, 2, seed=15, keep_ratio=0.3, sink_blocks=1, window_blocks=1),
    "tiny_fp8": I.workload("tiny", dtype="fp8"),
    "varlen_fp8": W([640, 2048, 77], 4, 2, dtype="fp8", seed=16),
    "many_seqs": W([128 * (k % 5 + 1) + 8 * k for k in range(11)], 2, 1, seed=17),
    "gqa3_odd_group": W([1500, 700], 6, 2, seed=18),  # three query heads per KV head
    # 36 KV heads of 2 MB of keys at 8K: the scoring CTAs run in two groups of
    # 18 KV heads (the most that fit in 64 MB), query tiles descending in each
    "mha36_grouped": W([8192], 36, 36, seed=24),
    # standardized value bonus (per-sequence, per-KV-head z-score of ln ||v||^2)
    "std_bonus_varlen": W([1000, 128, 2088], 8, 2, seed=19, bonus_mode=1),
    "std_bonus_fp8": W([640, 2048, 77], 4, 2, dtype="fp8", seed=20, bonus_mode=1),
    # one block list per KV head (max over its query heads), shared by the group
    "group_lists": W([1000, 128, 2088], 8, 2, seed=21, list_mode=1),
    "group_lists_odd_group": W([1500, 700], 6, 2, seed=22, list_mode=1, keep_ratio=0.25),
    "group_lists_fp8": W([640, 2048, 77], 4, 2, dtype="fp8", seed=23, list_mode=1),
    # 64-token blocks ("64x128" KV blocks): the attention's 128-row tile holds
    # query blocks 2p and 2p + 1 and walks the union of their lists; odd block
    # counts (2088 -> 33, 63 -> 1) leave a last tile with one query block
    "b64_varlen": W([1000, 128, 2088, 64, 63], 8, 2, seed=31, block_size=64, sink_blocks=2, window_blocks=2),
    "b64_fp8": W([640, 2112, 77], 4, 2, dtype="fp8", seed=32, block_size=64),
    "b64_stride4": W([1600], 2, 1, seed=33, stride=4, block_size=64, keep_ratio=0.3),
    "b64_multi_tile": W([4096 + 640 + 64], 4, 2, seed=34, keep_ratio=0.3, block_size=64, sink_blocks=1,
                        window_blocks=1),
    "b64_group_lists": W([1000, 2088], 8, 2, seed=35, list_mode=1, block_size=64),
    "b64_std_bonus_fp8": W([640, 2112, 77], 4, 2, dtype="fp8", seed=36, bonus_mode=1, block_size=64),
}


class Case:
    """Inputs, GPU results and oracle results of one workload (computed once)."""

    def __init__(self, w):
        self.w = w
        self.cu = w.cu_seqlens()
        self.inp = I.make_inputs(w)
        self.dinp = to_device(self.inp)
        self.qkv = make_gpu_qkv(b, self.dinp, self.cu)
        self.params = b.make_params(**w.params())
        self.p = oparams(w)
        self.q, self.k, self.v = oracle_arrays(self.inp, w.dtype)
        self.ref_scores = O.block_scores(self.q, self.k, self.v, self.cu, self.p)
        self.ref_bonus = O.value_bonus(self.v, self.cu, self.p.beta, self.p.block_size, mode=self.p.bonus_mode)


_cache = {}


def get_case(name):
    if name not in _cache:
        _cache[name] = Case(CASES[name])
    return _cache[name]


@pytest.mark.parametrize("name", list(CASES))
def test_scores_and_bonus(name):
    c = get_case(name)
    scores, vbonus, ws = b.stem_score(c.qkv, c.params)
    assert b.stem_read_device_status(ws) == 0
    check_scores(scores.cpu().numpy().astype(np.float64), c.ref_scores, c.cu, c.p.block_size)
    vb = vbonus.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(vb, c.ref_bonus, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("name", list(CASES))
def test_select_is_bit_exact_on_identical_fp32_scores(name):
    """Feed the oracle's scores rounded to fp32 to the GPU selection; the oracle
    selects on the very same fp32 values: budgets, row_ptr and col_idx must be
    identical (ties resolved by index on both sides)."""
    c = get_case(name)
    s32 = c.ref_scores.astype(np.float32)
    gb, grp, gci, ws = b.stem_select(c.qkv, c.params, torch.from_numpy(s32).cuda())
    assert b.stem_read_device_status(ws) == 0
    ob, orp, oci = O.select(s32.astype(np.float64), c.cu, c.p, hkv=c.w.num_kv_heads)
    assert np.array_equal(gb.cpu().numpy(), ob)
    assert np.array_equal(grp.cpu().numpy(), orp)
    assert np.array_equal(gci.cpu().numpy(), oci)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("select_mode", [0, 1])
def test_score_select_equals_score_then_select(name, select_mode):
    """stem_score_select gives exactly the two separate calls' scores and
    lists, with the selection kernel after the scoring kernel (select_mode 0)
    and with the scoring CTAs selecting their own rows (select_mode 1)."""
    c = get_case(name)
    scores, vbonus, ws = b.stem_score(c.qkv, c.params)
    gb, grp, gci, _ = b.stem_select(c.qkv, c.params, scores)
    params = b.make_params(**c.w.params(), select_mode=select_mode)
    s2, gb2, grp2, gci2, ws2 = b.stem_score_select(c.qkv, params)
    torch.cuda.synchronize()
    assert b.stem_read_device_status(ws2) == 0
    assert torch.equal(s2.view(torch.int32), scores.view(torch.int32))
    assert torch.equal(gb2, gb) and torch.equal(grp2, grp) and torch.equal(gci2, gci)


def test_select_ties_go_to_lowest_index():
    c = get_case("varlen")
    rng = np.random.default_rng(3)
    s32 = np.round(c.ref_scores * 2).astype(np.float32) / 2  # many exact ties
    s32[rng.random(s32.shape) < 0.05] = np.nan               # NaN ranks as -inf
    gb, grp, gci, _ = b.stem_select(c.qkv, c.params, torch.from_numpy(s32).cuda())
    ob, orp, oci = O.select(s32.astype(np.float64), c.cu, c.p, hkv=c.w.num_kv_heads)
    assert np.array_equal(grp.cpu().numpy(), orp)
    assert np.array_equal(gci.cpu().numpy(), oci)


def test_select_signed_zeros_tie_by_index():
    """Caller-given scores whose selection threshold falls on a -0.0 at a lower
    key block and a +0.0 at a higher one: the two are equal numbers, so the
    lower index is taken (the oracle's rule), not the +0.0."""
    c = get_case("multi_tile")
    rng = np.random.default_rng(5)
    s32 = c.ref_scores.astype(np.float32)
    bud = O.budgets(c.cu, c.p)
    seqs, nbtot = O.seq_blocks(c.cu)
    planted = []
    for h in range(c.w.num_q_heads):
        for (_, _, nb, g0) in seqs:
            for i in range(nb):
                F = set(O.forced_blocks(i, c.p.sink_blocks, c.p.window_blocks))
                cand = [j for j in range(i + 1) if j not in F]
                m = min(max(int(bud[g0 + i]) - len(F), 0), len(cand))
                if m < 1 or len(cand) < m + 1:
                    continue
                perm = rng.permutation(cand)
                top, zeros, rest = perm[:m - 1], sorted(perm[m - 1:m + 1]), perm[m + 1:]
                row = s32[h, g0 + i]
                row[top] = 1.0 + rng.random(len(top)).astype(np.float32)
                row[zeros[0]] = np.float32(-0.0)
                row[zeros[1]] = np.float32(0.0)
                row[rest] = -1.0 - rng.random(len(rest)).astype(np.float32)
                planted.append((h * nbtot + g0 + i, zeros[0], zeros[1]))
    assert len(planted) > 20
    gb, grp, gci, ws = b.stem_select(c.qkv, c.params, torch.from_numpy(s32).cuda())
    assert b.stem_read_device_status(ws) == 0
    ob, orp, oci = O.select(s32.astype(np.float64), c.cu, c.p, hkv=c.w.num_kv_heads)
    for (r, lo, hi) in planted:
        row = oci[orp[r]:orp[r + 1]].tolist()
        assert lo in row and hi not in row
    assert np.array_equal(grp.cpu().numpy(), orp)
    assert np.array_equal(gci.cpu().numpy(), oci)
    # the same rows through the KV-group-shared selection (max over the group)
    params1 = b.make_params(**dict(c.w.params(), list_mode=1))
    _, grp1, gci1, _ = b.stem_select(c.qkv, params1, torch.from_numpy(s32).cuda())
    p1 = O.Params(**dict(c.w.params(), list_mode=1))
    _, orp1, oci1 = O.select(s32.astype(np.float64), c.cu, p1, hkv=c.w.num_kv_heads)
    assert np.array_equal(grp1.cpu().numpy(), orp1)
    assert np.array_equal(gci1.cpu().numpy(), oci1)


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_end_to_end(name):
    c = get_case(name)
    out, lse, rp, ci, ws = b.stem_prefill(c.qkv, c.params)
    assert b.stem_read_device_status(ws) == 0
    rp, ci = rp.cpu().numpy(), ci.cpu().numpy()
    ob, orp, oci = O.select(c.ref_scores, c.cu, c.p, hkv=c.w.num_kv_heads)
    ranked = O.group_pooled_scores(c.ref_scores, c.w.num_kv_heads) if c.p.list_mode else c.ref_scores
    compare_lists(rp, ci, orp, oci, ranked, c.cu, c.w.num_q_heads, c.p.sink_blocks, c.p.window_blocks,
                  c.p.block_size)
    # attention with the GPU's own lists
    ro, rl = O.bsa(c.q, c.k, c.v, c.cu, rp, ci, c.p)
    check_attention(out, lse, ro, rl, c.w.dtype)
    # stem_prefill == stem_score -> stem_select -> stem_bsa_fwd
    scores, _, _ = b.stem_score(c.qkv, c.params)
    _, rp2, ci2, _ = b.stem_select(c.qkv, c.params, scores)
    assert np.array_equal(rp2.cpu().numpy(), rp) and np.array_equal(ci2.cpu().numpy(), ci)
    out2, lse2, _ = b.stem_bsa_fwd(c.qkv, c.params, rp2, ci2)
    assert torch.equal(out2, out) and torch.equal(lse2, lse)


@pytest.mark.parametrize("name", ["tiny", "varlen", "varlen_fp8", "multi_tile", "b64_varlen", "b64_fp8"])
def test_dense_comparator_is_causal_attention(name):
    """Every causal block listed: the result is ordinary causal attention."""
    c = get_case(name)
    rp, ci = O.full_csr(c.cu, c.w.num_q_heads, c.p.block_size)
    out, lse, ws = b.stem_bsa_fwd(c.qkv, c.params, torch.from_numpy(rp.astype(np.int32)).cuda(),
                                  torch.from_numpy(ci.astype(np.int32)).cuda())
    assert b.stem_read_device_status(ws) == 0
    ro, rl = O.bsa(c.q, c.k, c.v, c.cu, rp, ci, c.p)
    check_attention(out, lse, ro, rl, c.w.dtype)


def test_malformed_list_entries_are_skipped_and_reported():
    c = get_case("varlen")
    rp, ci = O.full_csr(c.cu, c.w.num_q_heads)
    bad = ci.copy()
    seqs, nbtot = O.seq_blocks(c.cu)
    # row of head 1, block 5 of sequence 0: replace its 3rd entry by a block above the diagonal
    r = 1 * nbtot + 5
    bad[rp[r] + 2] = 9
    out, lse, ws = b.stem_bsa_fwd(c.qkv, c.params, torch.from_numpy(rp.astype(np.int32)).cuda(),
                                  torch.from_numpy(bad.astype(np.int32)).cuda())
    assert b.stem_read_device_status(ws) == 7
    keep = np.ones(len(ci), dtype=bool)
    keep[rp[r] + 2] = False
    rp2 = rp.copy()
    rp2[r + 1:] -= 1
    ro, rl = O.bsa(c.q, c.k, c.v, c.cu, rp2, ci[keep], c.p)
    check_attention(out, lse, ro, rl, "bf16")


def test_malformed_list_entries_are_skipped_and_reported_64_token_blocks():
    """With 64-token blocks the bad entry sits in the second list of a tile
    (query block 7 = rows 64-127 of the tile of blocks 6 and 7)."""
    c = get_case("b64_varlen")
    rp, ci = O.full_csr(c.cu, c.w.num_q_heads, 64)
    seqs, nbtot = O.seq_blocks(c.cu, 64)
    r = 1 * nbtot + 7
    bad = ci.copy()
    bad[rp[r] + 2] = 9  # above the diagonal
    out, lse, ws = b.stem_bsa_fwd(c.qkv, c.params, torch.from_numpy(rp.astype(np.int32)).cuda(),
                                  torch.from_numpy(bad.astype(np.int32)).cuda())
    assert b.stem_read_device_status(ws) == 7
    keep = np.ones(len(ci), dtype=bool)
    keep[rp[r] + 2] = False
    rp2 = rp.copy()
    rp2[r + 1:] -= 1
    ro, rl = O.bsa(c.q, c.k, c.v, c.cu, rp2, ci[keep], c.p)
    check_attention(out, lse, ro, rl, "bf16")


def test_64_token_tiles_with_disjoint_lists():
    """Every unit of every tile belongs to one of its two query blocks only:
    block 2p lists its even blocks, block 2p + 1 its odd blocks (both end at
    their diagonal), so each unit is a -inf block for half of the tile's
    rows."""
    c = get_case("b64_varlen")
    seqs, nbtot = O.seq_blocks(c.cu, 64)
    rows = []
    for h in range(c.w.num_q_heads):
        for (_, _, nb, g0) in seqs:
            for i in range(nb):
                rows.append(list(range(i % 2, i + 1, 2)))
    rp = np.zeros(len(rows) + 1, dtype=np.int64)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([j for r in rows for j in r], dtype=np.int64)
    out, lse, ws = b.stem_bsa_fwd(c.qkv, c.params, torch.from_numpy(rp.astype(np.int32)).cuda(),
                                  torch.from_numpy(ci.astype(np.int32)).cuda())
    assert b.stem_read_device_status(ws) == 0
    ro, rl = O.bsa(c.q, c.k, c.v, c.cu, rp, ci, c.p)
    check_attention(out, lse, ro, rl, c.w.dtype)


@pytest.mark.parametrize("name", ["tiny", "b64_varlen"])
def test_empty_rows_give_zero_output_and_minus_inf_lse(name):
    c = get_case(name)
    nrows = c.w.num_q_heads * O.seq_blocks(c.cu, c.p.block_size)[1]
    rp = torch.zeros(nrows + 1, dtype=torch.int32, device="cuda")
    ci = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, ws = b.stem_bsa_fwd(c.qkv, c.params, rp, ci)
    assert b.stem_read_device_status(ws) == 0
    assert torch.all(out == 0)
    assert torch.all(torch.isneginf(lse))


def test_results_are_deterministic():
    c = get_case("multi_tile")
    a = b.stem_prefill(c.qkv, c.params)
    z = b.stem_prefill(c.qkv, c.params)
    for x, y in zip(a[:4], z[:4]):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name", ["group_lists", "group_lists_odd_group", "group_lists_fp8"])
def test_shared_list_pairs_equal_the_one_row_kernel(name):
    """With shared lists the attention runs two query heads per CTA on one
    staged K/V stream; per row it is the same arithmetic as one row per CTA,
    so the results are bit-identical (and match the oracle)."""
    c = get_case(name)
    _, _, rp, ci, _ = b.stem_prefill(c.qkv, c.params)
    out_pair, lse_pair, ws = b.stem_bsa_fwd(c.qkv, c.params, rp, ci)
    assert b.stem_read_device_status(ws) == 0
    per_row = b.make_params(**dict(c.w.params(), list_mode=0))
    out_row, lse_row, ws2 = b.stem_bsa_fwd(c.qkv, per_row, rp, ci)
    assert b.stem_read_device_status(ws2) == 0
    assert torch.equal(out_pair.view(torch.int16), out_row.view(torch.int16))
    assert torch.equal(lse_pair.view(torch.int32), lse_row.view(torch.int32))
    ro, rl = O.bsa(c.q, c.k, c.v, c.cu, rp.cpu().numpy(), ci.cpu().numpy(), c.p)
    check_attention(out_pair, lse_pair, ro, rl, c.w.dtype)


def test_shared_list_mode_reports_rows_that_differ():
    c = get_case("group_lists")
    _, _, rp, ci, _ = b.stem_prefill(c.qkv, c.params)
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy().copy()
    seqs, nbtot = O.seq_blocks(c.cu)
    # head 1 (second of the pair with head 0), block 12 of the third sequence
    # (global block 9 + 12): swap one listed block for an unlisted causal one
    r = 1 * nbtot + 9 + 12
    row = ci_h[rp_h[r]:rp_h[r + 1]]
    spare = [j for j in range(13) if j not in set(row.tolist())]
    assert spare and len(row) >= 2
    row[0] = spare[0]
    ci_h[rp_h[r]:rp_h[r + 1]] = np.sort(row)
    out, lse, ws = b.stem_bsa_fwd(c.qkv, c.params, rp, torch.from_numpy(ci_h).cuda())
    assert b.stem_read_device_status(ws) == 7  # STEM_ERR_BAD_BLOCKLIST


@pytest.mark.parametrize("list_mode", [0, 1])
def test_select_long_rows_on_given_scores(list_mode):
    """The standalone selection on rows of up to 2,500 key blocks (each warp's
    keys and histogram need more than the default 48 KB of shared memory per
    CTA), per query head and with KV-group-shared lists: seeded fp32 scores
    with repeated values (ties) and a few NaN, selected by the GPU and by the
    oracle on the very same values; the lists must be identical."""
    nb = 2500
    w = I.Workload(name="long_select", seqlens=[nb * 128 - 77], num_q_heads=4, num_kv_heads=2, seed=61,
                   keep_ratio=0.3, mu=0.7, beta=0.2, sink_blocks=2, window_blocks=3, list_mode=list_mode)
    cu = w.cu_seqlens()
    q = torch.zeros(1, w.num_q_heads, 128, dtype=torch.bfloat16, device="cuda")  # scores are given: never read
    qkv = b.make_qkv(q, q[:, :w.num_kv_heads].contiguous(), q[:, :w.num_kv_heads].contiguous(), cu,
                     cu_seqlens_dev=torch.tensor(cu, dtype=torch.int32, device="cuda"))
    qkv.desc.total_tokens = cu[-1]
    params = b.make_params(**w.params())
    rng = np.random.default_rng(7)
    s32 = (np.round(rng.standard_normal((w.num_q_heads, nb, nb)) * 8) / 8).astype(np.float32)
    s32[rng.random(s32.shape) < 0.001] = np.nan
    gb, grp, gci, ws = b.stem_select(qkv, params, torch.from_numpy(s32).cuda())
    torch.cuda.synchronize()
    assert b.stem_read_device_status(ws) == 0
    ob, orp, oci = O.select(s32.astype(np.float64), cu, O.Params(**w.params()), hkv=w.num_kv_heads)
    assert np.array_equal(gb.cpu().numpy(), ob)
    assert np.array_equal(grp.cpu().numpy(), orp)
    assert np.array_equal(gci.cpu().numpy(), oci)
