"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these checks re-types the oracle's own formula: each uses a closed form,
exact rational arithmetic, brute force on tiny inputs, a second formulation or a
library routine on a special case, so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import stem_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- encodings

def test_bf16_decode_matches_library_and_known_values():
    bits = np.arange(0, 1 << 16, 7, dtype=np.uint32).astype(np.uint16)
    ours = O.bf16_bits_to_f64(bits)
    lib = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    same = (ours == lib) | (np.isnan(ours) & np.isnan(lib))
    assert same.all()
    assert O.bf16_bits_to_f64(np.array([0x3F80, 0xC000, 0x0000, 0x4049], dtype=np.uint16)).tolist() == \
        [1.0, -2.0, 0.0, 3.140625]


def test_e4m3_decode_matches_library_and_format_extremes():
    b = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_bytes_to_f64(b)
    lib = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (ours == lib) | (np.isnan(ours) & np.isnan(lib))
    assert same.all()
    # largest normal 448 = 1.75 * 2^8, smallest subnormal 2^-9, NaN at 0x7F/0xFF
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])


def test_fp8_dequant_applies_per_head_scale():
    x = np.array([[[0x38, 0x40], [0x38, 0x40]]], dtype=np.uint8)  # 1.0, 2.0 per head
    out = O.dequant(x, "fp8", np.array([0.5, 3.0], dtype=np.float32))
    assert out.tolist() == [[[0.5, 1.0], [3.0, 6.0]]]


# ---------------------------------------------------------------- defaults

def test_defaults_match_documented_table():
    g = json.load(open(os.path.join(GOLDEN, "angelslim_defaults.json")))
    p = O.Params()
    assert p.block_size == g["block_size"] and p.stride == g["stride"]
    assert p.chunk_size == g["chunk_size"] and p.norm == g["norm"]
    assert p.sink_blocks == g["initial_blocks"] and p.window_blocks == g["window_size"]
    assert p.mu == g["mu_best"] and p.beta == g["beta_best"]


# ---------------------------------------------------------------- TPD budget

def _exact_k(i, nb, rho, mu, relative=True):
    """k(i) = floor(k_start - k_start (1-mu)/N * i) in exact rationals, with rho
    and mu taken as the decimals the caller wrote.  Also returns whether the
    real value sits exactly on an integer (where fp64 rounding may land on
    either side)."""
    rho, mu = Fraction(str(rho)), Fraction(str(mu))
    c = i + 1
    ks = math.ceil(rho * c) if relative else math.ceil(rho * nb)
    val = ks - ks * (1 - mu) / nb * i
    return ks, math.floor(val), val.denominator == 1


@pytest.mark.parametrize("rho,mu,nb", [(0.25, 0.7, 256), (0.5, 0.7, 16), (0.25, 0.7, 1024),
                                       (0.2, 1.0, 512), (0.1, 1.0, 512), (0.25, 0.7, 64),
                                       (0.3, 0.45, 100), (1.0, 0.7, 37)])
@pytest.mark.parametrize("relative", [True, False])
def test_tpd_closed_form_against_exact_rationals(rho, mu, nb, relative):
    p = O.Params(keep_ratio=rho, mu=mu, budget_mode=O.RELATIVE if relative else O.ABSOLUTE)
    for i in range(nb):
        ks, k = O.tpd_k(i, nb, p)
        eks, ek, on_integer = _exact_k(i, nb, rho, mu, relative)
        assert ks == eks
        # fp64 (the fixed evaluation order) may only differ from exact arithmetic
        # where the exact value is an integer, and then by one step down.
        if k != ek:
            assert on_integer and k == ek - 1, (i, k, ek)


def test_tpd_endpoints_and_uniform_limit():
    # i = 0 gives k_start; mu = 1 gives the uniform budget (k_end = mu k_start).
    for nb in (16, 256, 1000):
        for rho in (0.1, 0.25, 0.5):
            p1 = O.Params(keep_ratio=rho, mu=1.0)
            for i in range(nb):
                ks, k = O.tpd_k(i, nb, p1)
                assert k == ks
            p = O.Params(keep_ratio=rho, mu=0.7)
            ks0, k0 = O.tpd_k(0, nb, p)
            assert k0 == ks0 == math.ceil(rho)
    # absolute mode, i = N: k(N) = floor(mu * k_start) (the page's k_end)
    p = O.Params(keep_ratio=0.25, mu=0.7, budget_mode=O.ABSOLUTE)
    nb = 400
    ks = math.ceil(0.25 * nb)
    k_end = math.floor(ks - ks * (1 - Fraction("0.7")) / nb * nb)
    assert k_end == math.floor(Fraction("0.7") * ks)


def test_tpd_monotone_in_mu_and_full_density():
    nb = 300
    for i in range(nb):
        ks_prev = -1
        for mu in (0.1, 0.3, 0.5, 0.7, 0.9, 1.0):
            _, k = O.tpd_k(i, nb, O.Params(keep_ratio=0.25, mu=mu))
            assert k >= ks_prev
            ks_prev = k
    cu = [0, 128 * 50, 128 * 50 + 300]
    b = O.budgets(cu, O.Params(keep_ratio=1.0, mu=1.0, sink_blocks=0, window_blocks=1))
    expect = list(range(1, 51)) + list(range(1, 4))
    assert b.tolist() == expect


def test_forced_blocks_examples():
    assert O.forced_blocks(0, 4, 4) == [0]
    assert O.forced_blocks(5, 1, 1) == [0, 5]
    assert O.forced_blocks(5, 4, 4) == [0, 1, 2, 3, 4, 5]
    assert O.forced_blocks(9, 1, 2) == [0, 8, 9]
    assert O.forced_blocks(9, 0, 1) == [9]
    # budget never below |F| nor above c
    p = O.Params(keep_ratio=0.05, mu=0.5, sink_blocks=4, window_blocks=4)
    for i in range(40):
        b = O.tpd_budget(i, 40, p)
        assert len(O.forced_blocks(i, 4, 4)) <= b <= i + 1


# ---------------------------------------------------------------- selection

def test_selection_equals_subset_brute_force():
    rng = np.random.default_rng(7)
    for trial in range(60):
        i = int(rng.integers(0, 11))
        c = i + 1
        S, W = int(rng.integers(0, 3)), int(rng.integers(1, 3))
        F = O.forced_blocks(i, S, W)
        b = int(rng.integers(len(F), c + 1))
        row = rng.permutation(c).astype(np.float64) + rng.random(c) * 0.1  # distinct
        rest = [j for j in range(c) if j not in F]
        best, best_set = -math.inf, None
        for comb in itertools.combinations(rest, b - len(F)):
            tot = sum(row[j] for j in comb)
            if tot > best:
                best, best_set = tot, comb
        assert O.select_row(row, i, b, S, W) == sorted(F + list(best_set))


def test_selection_ties_nan_and_structure():
    row = np.array([0.0, 5.0, 5.0, 5.0, np.nan, -np.inf, 1.0, 9.0])
    # i=7, W=1 forces {7}; S=0; budget 3 -> two of {1,2,3} by lowest index
    assert O.select_row(row, 7, 3, 0, 1) == [1, 2, 7]
    # NaN ranks like -inf, behind 0.0; tie between NaN(4) and -inf(5) -> index 4
    assert O.select_row(row, 7, 7, 0, 1) == [0, 1, 2, 3, 4, 6, 7]
    rng = np.random.default_rng(3)
    cu = [0, 128 * 24]
    p = O.Params(keep_ratio=0.3, mu=0.7, sink_blocks=2, window_blocks=3)
    sc = rng.standard_normal((3, 24, 24))
    bud, rp, ci = O.select(sc, cu, p)
    for h in range(3):
        for i in range(24):
            r = h * 24 + i
            sel = ci[rp[r]:rp[r + 1]].tolist()
            assert len(sel) == bud[r] and sel == sorted(set(sel))
            assert set(O.forced_blocks(i, 2, 3)) <= set(sel) and max(sel) == i
    # -0.0 and +0.0 are equal numbers: between them the lower index wins,
    # whichever of the two carries the sign bit
    z = np.array([-1.0, 0.0, -0.0, 2.0, -0.0, 0.0, -3.0, 7.0])
    assert O.select_row(z, 7, 3, 0, 1) == [1, 3, 7]
    z2 = np.array([-1.0, -0.0, 0.0, 2.0, 0.0, -0.0, -3.0, 7.0])
    assert O.select_row(z2, 7, 3, 0, 1) == [1, 3, 7]
    assert O.select_row(z2, 7, 4, 0, 1) == [1, 2, 3, 7]
    # rho = 1, mu = 1 selects every causal block
    bud, rp, ci = O.select(sc, cu, O.Params(keep_ratio=1.0, mu=1.0, sink_blocks=0, window_blocks=1))
    rp2, ci2 = O.full_csr(cu, 3)
    assert rp.tolist() == rp2.tolist() and ci.tolist() == ci2.tolist()


# ---------------------------------------------------------------- scoring

@pytest.mark.parametrize("L,s,d,hq,hkv", [(64, 8, 16, 4, 2), (61, 8, 8, 2, 1), (40, 4, 8, 2, 2)])
def test_two_scoring_formulations_agree(L, s, d, hq, hkv):
    q = _rand((L, hq, d), 1)
    k = _rand((L, hkv, d), 2)
    A = O.downsampled_scores(q, k, s, 1.5)
    B = O.downsampled_scores_antidiag(q, k, s, 1.5)
    assert A.shape == B.shape
    np.testing.assert_allclose(A, B, rtol=0, atol=1e-12)


def test_scoring_closed_form_pairs_anti_diagonal():
    """q_t = t e0 and k_t = t e0: D[a][b] = sum_u (as+u)(bs+s-1-u)/(sqrt(d) s n),
    expanded with sum u = s(s-1)/2 and sum u^2 = (s-1)s(2s-1)/6; the main
    diagonal pairing would give a different value everywhere."""
    L, s, d, n = 48, 8, 4, 2.0
    t = np.arange(L, dtype=np.float64)
    q = np.zeros((L, 1, d)); q[:, 0, 0] = t
    k = np.zeros((L, 1, d)); k[:, 0, 0] = t
    D = O.downsampled_scores(q, k, s, n)[0]
    S1 = s * (s - 1) / 2
    S2 = (s - 1) * s * (2 * s - 1) / 6
    for a in range(L // s):
        for b in range(L // s):
            A_, B_ = a * s, b * s
            # (A+u)(B+s-1-u) = A(B+s-1) + u(B+s-1) - A u - u^2
            tot = s * A_ * (B_ + s - 1) + S1 * (B_ + s - 1) - A_ * S1 - S2
            assert D[a, b] == pytest.approx(tot / (math.sqrt(d) * s * n), rel=1e-14)
            diag = s * A_ * B_ + S1 * (A_ + B_) + S2
            if a == b == 0:
                continue
            assert abs(diag - tot) > 0.5


def test_block_scores_closed_form_with_bonus():
    """q_t = e0, k_t = t e0 (so D grows with the key group), and v_t = c_t e0:
    S_ij = (b_last s + (s-1)/2)/(sqrt(d) n) + beta max(0, ln max c_t^2),
    b_last the last group of key block j; -inf above the diagonal."""
    B, s, d = 32, 8, 4
    L = 4 * B + 20  # partial last block (20 tokens)
    t = np.arange(L, dtype=np.float64)
    q = np.zeros((L, 2, d)); q[:, :, 0] = 1.0
    k = np.zeros((L, 1, d)); k[:, 0, 0] = t
    c = np.exp(np.sin(t) * 2.0)  # norms spanning both sides of 1
    v = np.zeros((L, 1, d)); v[:, 0, 0] = c
    p = O.Params(block_size=B, stride=s, chunk_size=64, beta=0.2, norm=1.0)
    Sm = O.block_scores(q, k, v, [0, L], p)
    nb = 5
    ngv = math.ceil(L / s)
    for i in range(nb):
        for j in range(nb):
            if j > i:
                assert Sm[0, i, j] == -np.inf
                continue
            # key group b contributes sum of its valid token indices; the last
            # group of the partial block holds tokens 144..151 of which only
            # 144..147 exist (missing ones count as zero), so it is not the max
            dval = max(sum(tt for tt in range(b * s, b * s + s) if tt < L)
                       for b in range(j * (B // s), min((j + 1) * (B // s), ngv))) / (math.sqrt(d) * s)
            m = max(c[j * B:min((j + 1) * B, L)] ** 2)
            want = dval + 0.2 * max(0.0, math.log(m))
            assert Sm[0, i, j] == pytest.approx(want, rel=1e-13)
            assert Sm[1, i, j] == Sm[0, i, j]


def test_value_bonus_special_cases():
    # ||v||^2 = e^2 -> ln = 2 -> bonus 2 beta; ||v|| < 1 -> bonus 0; zero rows -> 0
    v = np.zeros((3 * 16, 1, 4))
    v[:16, 0, 1] = math.e
    v[16:32, 0, 2] = 0.5
    b = O.value_bonus(v, [0, 48], 0.2, block=16)
    assert b[0].tolist() == pytest.approx([0.4, 0.0, 0.0], abs=1e-15)


def _blocks_with_norms(sq_norms, block=16, d=4):
    """V [len(sq_norms) * block, 1, d] whose block j has max ||v_t||^2 = sq_norms[j]
    (one token at that norm, the others smaller)."""
    v = np.zeros((len(sq_norms) * block, 1, d))
    for j, n2 in enumerate(sq_norms):
        v[j * block, 0, 0] = math.sqrt(n2)
        v[j * block + 1: (j + 1) * block, 0, 1] = 0.5 * math.sqrt(n2)
    return v


def test_standardized_bonus_closed_forms():
    """Standardized OAM (AngelSlim doc §2.1: lambda ReLU(v_bar_j)): x_j = ln of
    the block's largest squared norm, z-scored over the sequence's blocks.
    Two blocks: z = -1, +1.  Three equally spaced x: z = -sqrt(3/2), 0, +sqrt(3/2)."""
    beta = 0.3
    b2 = O.value_bonus(_blocks_with_norms([math.exp(0.7), math.exp(5.0)]), [0, 32], beta, 16, O.BONUS_STANDARDIZED)
    assert b2[0].tolist() == pytest.approx([0.0, beta], abs=1e-12)
    b3 = O.value_bonus(_blocks_with_norms([1.0, math.e, math.e ** 2]), [0, 48], beta, 16, O.BONUS_STANDARDIZED)
    assert b3[0].tolist() == pytest.approx([0.0, 0.0, beta * math.sqrt(1.5)], abs=1e-12)
    # the log form on the same input: beta * max(0, x)
    b3l = O.value_bonus(_blocks_with_norms([1.0, math.e, math.e ** 2]), [0, 48], beta, 16, O.BONUS_LOG)
    assert b3l[0].tolist() == pytest.approx([0.0, beta, 2 * beta], abs=1e-12)


def test_standardized_bonus_is_scale_invariant_and_handles_degenerate_blocks():
    rng = np.random.default_rng(21)
    v = rng.standard_normal((5 * 16, 2, 4)) * np.exp(rng.standard_normal((5 * 16, 2, 1)))
    b = O.value_bonus(v, [0, 80], 0.2, 16, O.BONUS_STANDARDIZED)
    # scaling V scales every ||v||^2 by c^2: x shifts, z does not
    assert np.allclose(O.value_bonus(7.5 * v, [0, 80], 0.2, 16, O.BONUS_STANDARDIZED), b, rtol=0, atol=1e-12)
    assert not np.allclose(O.value_bonus(7.5 * v, [0, 80], 0.2, 16, O.BONUS_LOG),
                           O.value_bonus(v, [0, 80], 0.2, 16, O.BONUS_LOG))
    # z-scores of a head sum to zero: the bonus is the positive part, times beta
    x = np.array([[np.log(np.max(np.sum(v[j * 16:(j + 1) * 16, h] ** 2, axis=1))) for j in range(5)] for h in range(2)])
    z = (x - x.mean(axis=1, keepdims=True)) / x.std(axis=1, keepdims=True)
    assert np.allclose(b, 0.2 * np.maximum(0, z), atol=1e-12)
    # equal norms: std 0 -> no bonus; a zero block is left out of the statistics
    assert not O.value_bonus(_blocks_with_norms([2.0, 2.0, 2.0]), [0, 48], 0.2, 16, O.BONUS_STANDARDIZED).any()
    vz = _blocks_with_norms([1.0, 0.0, math.e ** 2])
    bz = O.value_bonus(vz, [0, 48], 0.5, 16, O.BONUS_STANDARDIZED)
    assert bz[0].tolist() == pytest.approx([0.0, 0.0, 0.5], abs=1e-12)  # z over {0, 2}: -1, +1
    # statistics are per sequence: a second sequence does not change the first one's bonus
    two = np.concatenate([vz, _blocks_with_norms([100.0, 1e-3])])
    assert O.value_bonus(two, [0, 48, 80], 0.5, 16, O.BONUS_STANDARDIZED)[0, :3].tolist() == bz[0].tolist()


def _rows(rp, ci):
    return [ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)]


def test_group_lists_pool_by_max_and_are_shared():
    """GQA-shared lists: for every (KV head, query block) the G query heads get
    one list, the per-head selection applied to the elementwise max of their
    score rows (checked against loops over the heads, not the vectorised max)."""
    rng = np.random.default_rng(31)
    hq, hkv, nb = 6, 2, 9
    cu = [0, nb * 16]
    p = O.Params(block_size=16, keep_ratio=0.4, mu=0.8, sink_blocks=1, window_blocks=1, list_mode=O.LIST_PER_GROUP)
    sc = np.full((hq, nb, nb), -np.inf)
    for h in range(hq):
        for i in range(nb):
            sc[h, i, :i + 1] = rng.standard_normal(i + 1)
    sc[4, 3, 1] = np.nan  # NaN counts as -inf in the pooling too
    bud, rp, ci = O.select(sc, cu, p, hkv=hkv)
    rows = _rows(rp, ci)
    G = hq // hkv
    for hk in range(hkv):
        for i in range(nb):
            pooled = []
            for j in range(i + 1):
                best = -math.inf
                for h in range(hk * G, (hk + 1) * G):
                    x = sc[h, i, j]
                    if not math.isnan(x) and x > best:
                        best = x
                pooled.append(best)
            want = O.select_row(np.array(pooled), i, int(bud[i]), 1, 1)
            for h in range(hk * G, (hk + 1) * G):
                assert rows[h * nb + i] == want


def test_group_lists_reduce_to_per_head_lists():
    rng = np.random.default_rng(32)
    hq, nb = 4, 7
    cu = [0, nb * 16]
    base = dict(block_size=16, keep_ratio=0.5, mu=0.7, sink_blocks=1, window_blocks=2)
    sc = np.full((hq, nb, nb), -np.inf)
    for i in range(nb):
        sc[:, i, :i + 1] = rng.standard_normal((hq, i + 1))
    per_head = _rows(*O.select(sc, cu, O.Params(**base))[1:])
    # one query head per KV head: the group is the head
    assert _rows(*O.select(sc, cu, O.Params(**base, list_mode=O.LIST_PER_GROUP), hkv=hq)[1:]) == per_head
    # identical heads in a group: nothing to pool
    same = np.repeat(sc[::2], 2, axis=0)
    assert (_rows(*O.select(same, cu, O.Params(**base, list_mode=O.LIST_PER_GROUP), hkv=2)[1:])
            == _rows(*O.select(same, cu, O.Params(**base))[1:]))
    # a dominant head decides its group's list
    dom = sc.copy()
    dom[0] += 100.0
    dom[2] += 100.0
    grp = _rows(*O.select(dom, cu, O.Params(**base, list_mode=O.LIST_PER_GROUP), hkv=2)[1:])
    ph = _rows(*O.select(dom, cu, O.Params(**base))[1:])
    for i in range(nb):
        assert grp[0 * nb + i] == grp[1 * nb + i] == ph[0 * nb + i]
        assert grp[2 * nb + i] == grp[3 * nb + i] == ph[2 * nb + i]


def test_paged_gather_is_the_page_table_lookup():
    rng = np.random.default_rng(41)
    cu, ps = [0, 150, 150 + 64, 150 + 64 + 1], 64
    kc = rng.standard_normal((cu[-1], 2, 4))
    # contiguous pages in order reproduce the packed tensor ...
    npg = [(cu[i + 1] - cu[i] + ps - 1) // ps for i in range(3)]
    pages = np.zeros((sum(npg), ps, 2, 4))
    table = np.zeros((3, max(npg)), dtype=np.int64)
    nxt = 0
    for sq in range(3):
        for pg in range(npg[sq]):
            n = min(ps, cu[sq + 1] - cu[sq] - pg * ps)
            pages[nxt, :n] = kc[cu[sq] + pg * ps: cu[sq] + pg * ps + n]
            table[sq, pg] = nxt
            nxt += 1
    assert np.array_equal(O.gather_paged(pages, table, cu, ps), kc)
    # ... and so does any permutation of the pool with the table permuted alike
    perm = rng.permutation(len(pages))
    inv = np.argsort(perm)
    assert np.array_equal(O.gather_paged(pages[perm], inv[table], cu, ps), kc)


def test_oam_log_form_ranks_like_product_form():
    """HPC-BSA article §2.2: the log turns the product exp(routing) * magnitude
    into a sum without changing the ranking.  Top-k by the additive score must
    equal top-k by exp(max D) * max(1, m_j)^beta on tiny inputs."""
    rng = np.random.default_rng(11)
    B, s, d = 16, 4, 8
    L = 12 * B
    q = rng.standard_normal((L, 1, d))
    k = rng.standard_normal((L, 1, d))
    v = rng.standard_normal((L, 1, d)) * np.exp(rng.standard_normal((L, 1, 1)))
    p = O.Params(block_size=B, stride=s, chunk_size=64, beta=0.7)
    Sm = O.block_scores(q, k, v, [0, L], p)[0]
    D = O.downsampled_scores(q, k, s, 1.0)[0]
    gpb = B // s
    for i in range(12):
        prod = []
        for j in range(i + 1):
            mx = D[i * gpb:(i + 1) * gpb, j * gpb:(j + 1) * gpb].max()
            m = max(np.sum(v[j * B:(j + 1) * B, 0] ** 2, axis=1))
            prod.append(math.exp(mx) * max(1.0, m) ** 0.7)
        for kk in range(1, i + 2):
            top_sum = set(np.argsort(-Sm[i, :i + 1], kind="stable")[:kk].tolist())
            top_prod = set(np.argsort(-np.array(prod), kind="stable")[:kk].tolist())
            assert top_sum == top_prod


def test_beta_zero_is_pure_routing():
    rng = np.random.default_rng(5)
    B, s, d, L = 16, 4, 8, 64
    q, k = rng.standard_normal((L, 1, d)), rng.standard_normal((L, 1, d))
    v = rng.standard_normal((L, 1, d)) * 10
    S0 = O.block_scores(q, k, v, [0, L], O.Params(block_size=B, stride=s, beta=0.0))
    D = O.downsampled_scores(q, k, s, 1.0)[0]
    for i in range(4):
        for j in range(i + 1):
            assert S0[0, i, j] == D[i * 4:(i + 1) * 4, j * 4:(j + 1) * 4].max()


def test_halving_the_block_refines_scores_and_bonus():
    """64x128 or 128x128 KV blocks (HPC-BSA article §3.1): with beta = 0 an
    off-diagonal score at block size B is the max of the four block-size-B/2
    scores it covers (both are maxima of the same downsampled entries), and the
    value bonus at B is the larger of its two halves' bonuses (the max over a
    union of tokens, then the monotone ln and max(0, .))."""
    rng = np.random.default_rng(21)
    B, s, d = 16, 4, 8
    L = 9 * B + 5  # ragged last block at both sizes
    q, k = rng.standard_normal((L, 2, d)), rng.standard_normal((L, 1, d))
    v = rng.standard_normal((L, 1, d)) * np.exp(rng.standard_normal((L, 1, 1)))
    S = O.block_scores(q, k, v, [0, L], O.Params(block_size=B, stride=s, beta=0.0))
    Sh = O.block_scores(q, k, v, [0, L], O.Params(block_size=B // 2, stride=s, beta=0.0))
    nb, nbh = S.shape[1], Sh.shape[1]
    assert nbh == O.cdiv(L, B // 2) and nb == O.cdiv(L, B)
    for h in range(2):
        for i in range(nb):
            for j in range(i):
                sub = [Sh[h, a, c] for a in (2 * i, 2 * i + 1) if a < nbh for c in (2 * j, 2 * j + 1)]
                assert S[h, i, j] == max(sub)
            # the diagonal also covers the sub-block above the half-size diagonal
            diag_sub = [Sh[h, a, c] for a in (2 * i, 2 * i + 1) if a < nbh for c in (2 * i, 2 * i + 1) if c <= a]
            assert S[h, i, i] >= max(diag_sub)
    bon = O.value_bonus(v, [0, L], 0.3, B)[0]
    bonh = O.value_bonus(v, [0, L], 0.3, B // 2)[0]
    for j in range(nb):
        assert bon[j] == max(bonh[2 * j:2 * j + 2])


def test_attention_with_refined_lists_equals_the_coarse_attention():
    """A list at block size B, refined to block size B/2 (both halves of every
    listed block, for both half-size query blocks), keeps the same causal key
    set for every query, so the attention is the same."""
    B, d = 16, 8
    seqlens = [7 * B + 3, 2 * B, 5]
    q, k, v, cu = _small_problem(seqlens, 4, 2, d, seed=23)
    rng = np.random.default_rng(24)
    p = O.Params(block_size=B)
    ph = O.Params(block_size=B // 2)
    seqs, nbtot = O.seq_blocks(cu, B)
    seqsh, nbtoth = O.seq_blocks(cu, B // 2)
    rows, rowsh = [], [[] for _ in range(4 * nbtoth)]
    for h in range(4):
        for (o, L, nb, g0), (_, _, nbh, g0h) in zip(seqs, seqsh):
            for i in range(nb):
                lst = sorted(set(rng.choice(i + 1, size=rng.integers(1, i + 2), replace=False).tolist()) | {i})
                rows.append(lst)
                for a in (2 * i, 2 * i + 1):
                    if a < nbh:
                        rowsh[h * nbtoth + g0h + a] = [c for j in lst for c in (2 * j, 2 * j + 1) if c <= a]

    def csr(rs):
        rp = np.zeros(len(rs) + 1, dtype=np.int64)
        rp[1:] = np.cumsum([len(r) for r in rs])
        return rp, np.array([j for r in rs for j in r], dtype=np.int64)

    rp, ci = csr(rows)
    rph, cih = csr(rowsh)
    O1, L1 = O.bsa(q, k, v, cu, rp, ci, p)
    O2, L2 = O.bsa(q, k, v, cu, rph, cih, ph)
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L1, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- attention

def _small_problem(seqlens, hq, hkv, d, seed):
    rng = np.random.default_rng(seed)
    T = sum(seqlens)
    q = rng.standard_normal((T, hq, d))
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).tolist()
    return q, k, v, cu


def test_gather_equals_minus_inf_mask():
    """HPC-BSA article §3.1: skipping a block is the same as -inf scores."""
    B = 16
    q, k, v, cu = _small_problem([100, 57], 4, 2, 8, 9)
    p = O.Params(block_size=B, stride=4, keep_ratio=0.4, mu=0.7, sink_blocks=1, window_blocks=1)
    S = O.block_scores(q, k, v, cu, p)
    bud, rp, ci = O.select(S, cu, p)
    A_o, A_l = O.bsa(q, k, v, cu, rp, ci, p)
    B_o, B_l = O.bsa_masked(q, k, v, cu, rp, ci, p)
    np.testing.assert_allclose(A_o, B_o, atol=1e-12)
    np.testing.assert_allclose(A_l, B_l, atol=1e-12)


def test_full_selection_is_dense_causal_attention_sdpa():
    """rho = 1, mu = 1 keeps every causal block: the result must be ordinary
    causal softmax attention (torch SDPA in fp64 on CPU, GQA heads repeated)."""
    B = 16
    seqlens = [70, 48]
    q, k, v, cu = _small_problem(seqlens, 4, 2, 8, 4)
    p = O.Params(block_size=B, stride=4, keep_ratio=1.0, mu=1.0, sink_blocks=0, window_blocks=1,
                 softmax_scale=0.3)
    res = O.prefill(q, k, v, cu, p)
    for s in range(2):
        o, e = cu[s], cu[s + 1]
        qt = torch.from_numpy(q[o:e]).permute(1, 0, 2)[None]
        kt = torch.from_numpy(k[o:e]).permute(1, 0, 2).repeat_interleave(2, 0)[None]
        vt = torch.from_numpy(v[o:e]).permute(1, 0, 2).repeat_interleave(2, 0)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.3)
        np.testing.assert_allclose(res["out"][o:e], ref[0].permute(1, 0, 2).numpy(), atol=1e-12)
        logits = 0.3 * torch.einsum("htd,hud->htu", qt[0], kt[0])
        mask = torch.ones(e - o, e - o, dtype=torch.bool).tril()
        lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
        np.testing.assert_allclose(res["lse"][:, o:e], lse.numpy(), atol=1e-12)


def test_first_token_sees_only_itself():
    B = 16
    q, k, v, cu = _small_problem([40], 2, 1, 8, 2)
    p = O.Params(block_size=B, stride=4, keep_ratio=0.5, mu=0.7, sink_blocks=1, window_blocks=1)
    rp, ci = O.full_csr(cu, 2, B)
    out, lse = O.bsa(q, k, v, cu, rp, ci, p)
    sig = 1 / math.sqrt(8)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], v[0, 0], atol=1e-15)
        assert lse[h, 0] == pytest.approx(sig * q[0, h] @ k[0, 0], abs=1e-14)


def test_skipped_block_changes_only_its_rows_weights():
    """Dropping one listed block equals renormalising the softmax without it:
    O_without = (l_full O_full - l_blk O_blk) / (l_full - l_blk)."""
    B = 16
    q, k, v, cu = _small_problem([64], 1, 1, 8, 12)
    p = O.Params(block_size=B, stride=4)
    rp_full, ci_full = O.full_csr(cu, 1, B)
    full_o, full_l = O.bsa(q, k, v, cu, rp_full, ci_full, p)
    # row of block 3 without key block 1
    rp = np.array([0, 1, 3, 6, 9])
    ci = np.array([0, 0, 1, 0, 1, 2, 0, 2, 3])
    o2, l2 = O.bsa(q, k, v, cu, rp, ci, p)
    only = np.array([0, 1, 2, 3, 4])
    rpb = np.array([0, 1, 2, 3, 4])
    cib = np.array([0, 1, 2, 1])  # block 3's row lists only key block 1
    ob, lb = O.bsa(q, k, v, cu, rpb, cib, p)
    t = slice(48, 64)
    lf, lbk = np.exp(full_l[0, t]), np.exp(lb[0, t])
    want = (lf[:, None] * full_o[t, 0] - lbk[:, None] * ob[t, 0]) / (lf - lbk)[:, None]
    np.testing.assert_allclose(o2[t, 0], want, atol=1e-10)
    np.testing.assert_allclose(np.exp(l2[0, t]), lf - lbk, rtol=1e-12)


@pytest.mark.parametrize("bonus_mode", [O.BONUS_LOG, O.BONUS_STANDARDIZED])
def test_single_row_scoring_equals_full_matrix_row(bonus_mode):
    rng = np.random.default_rng(21)
    B, s, d, L = 32, 8, 8, 5 * 32 + 9
    q = rng.standard_normal((L, 4, d))
    k = rng.standard_normal((L, 2, d))
    v = rng.standard_normal((L, 2, d)) * 3 * np.exp(rng.standard_normal((L, 2, 1)))
    p = O.Params(block_size=B, stride=s, chunk_size=64, beta=0.3, norm=1.3, bonus_mode=bonus_mode)
    full = O.block_scores(q, k, v, [0, L], p)
    for h in range(4):
        for i in range(6):
            row = O.block_score_row(q[:, h:h + 1], k[:, h // 2:h // 2 + 1], v[:, h // 2:h // 2 + 1], i, p)
            np.testing.assert_allclose(row, full[h, i, :i + 1], rtol=0, atol=1e-12)
