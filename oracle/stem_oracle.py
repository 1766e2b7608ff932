"""Plain fp64 CPU oracle of the Stem prefill hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module: only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, table or
helper with the CUDA library; it reads raw input bytes (bf16 bit patterns or
fp8 e4m3 bytes plus per-head scales), upcasts them exactly to fp64 and follows
the method step by step, in the order the pages give it.

Sources (cited by page title and section):

* [AngelSlim-doc]  "Stem: Rethinking Causal Information Flow in Sparse
  Attention", AngelSlim documentation (readthedocs, stem.md): §2.1 Block-Level
  Scoring (score formula with stride s and norm n), §2.2 Top-k Schedule (per-block
  budget from keep-ratio and alpha; initial blocks and sliding-window blocks are
  always kept), §2.3 Block-Sparse Attention, §6 parameter table (defaults).
* [gist-zh]  "Stem: Rethinking Causal Information Flow in Sparse Attention",
  gist.science summary (zh): §2.1 Token Position-Decay (the k(i) formula),
  §2.2 Output-Aware Metric (the M_ij formula; block-wise max-pooling of the
  value norms), §2.3 overall flow (anti-diagonal downsampled scoring, top-k per
  query block, exact softmax only over the chosen blocks).
* [gist-de]  same paper, gist.science summary (de): §2 Methodik A (TPD), B (OAM
  formula), C (anti-diagonal scoring, coarse-to-fine).
* [HPC-BSA]  youleyou article on Stem and the HPC-BSA operator: §2.2 (the log
  form turns the product into a sum and keeps the ranking), §3.1 (skipped
  blocks are equivalent to -inf scores; fixed 128x128 blocks).
* [zhichai]  zhichai.net summary of the AngelSlim Stem docs: §三 (sink and
  window blocks are additionally guaranteed), §四 Step 1 (stride 8, chunk 2048).

Readings taken where the pages are silent (each one is listed in the design
notes as well):

* keep-ratio -> k_start: relative, ks_i = ceil(rho * c_i) with c_i = i + 1
  causal key blocks of query block i; "absolute" mode ks = ceil(rho * NB).
* i and N in k(i): query-block index inside its sequence and the sequence's
  block count NB.
* k(i) evaluated in IEEE fp64 round-to-nearest in the order
  ks - ((ks * (1 - mu)) * i) / NB, then floor.
* forced blocks (sinks, window incl. the diagonal) count inside the budget:
  b_i = min(c_i, max(k_i, |F_i|)).
* value bonus: beta * max(0, ln max_{t in block} ||v_t||^2) (natural log).
* block score: max over the 16x16 downsampled entries of the block pair,
  plus the bonus of the key block; no causal mask inside scoring.
* anti-diagonal pairing (a*s + u, b*s + s - 1 - u), summed and divided by
  sqrt(d) * s * n.
* ties in top-k: lower key-block index wins; NaN scores rank as -inf.
* partial last block: only valid tokens; a downsampled group is valid when its
  first token is inside the sequence, its missing tokens count as zero.
* LSE: natural log of the softmax denominator over the selected causal keys.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force on tiny inputs, a second independent formulation,
library special cases).  The actual score values on realistic inputs have no
worked example on the pages, so beyond those pins the scoring is checked only by
its second formulation.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# --------------------------------------------------------------------------
# Parameters.  Defaults follow the AngelSlim-doc §6 parameter table
# (block_size 128, stride 8, chunk_size 2048, norm 1.0, initial_blocks 4,
# window_size 4) and gist-zh §4 ablation (mu = 0.7, beta = 0.2 best).
# --------------------------------------------------------------------------

RELATIVE = 0
ABSOLUTE = 1

# block-list granularity under GQA (see select)
LIST_PER_HEAD = 0   # every query head selects its own blocks
LIST_PER_GROUP = 1  # one list per KV head, from the max over its query heads

# value-magnitude bonus forms (see value_bonus)
BONUS_LOG = 0           # beta * max(0, ln ||v||^2)
BONUS_STANDARDIZED = 1  # beta * ReLU(z-score of ln ||v||^2)


@dataclass
class Params:
    block_size: int = 128
    stride: int = 8
    chunk_size: int = 2048
    norm: float = 1.0
    beta: float = 0.2
    keep_ratio: float = 0.25
    mu: float = 0.7
    sink_blocks: int = 4
    window_blocks: int = 4
    softmax_scale: float = 0.0  # 0 -> 1/sqrt(head_dim)
    budget_mode: int = RELATIVE
    bonus_mode: int = BONUS_LOG
    list_mode: int = LIST_PER_HEAD


# --------------------------------------------------------------------------
# Exact upcasts of the input encodings (definitions of the formats).
# --------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 is the upper half of an IEEE binary32: shift left by 16."""
    u32 = bits.astype(np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return u32.view(np.float32).astype(np.float64)


def _e4m3_value(byte: int) -> float:
    """OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa
    bits; no infinities; S.1111.111 is NaN; exponent field 0 is subnormal."""
    sign = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (-6)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_TABLE = np.array([_e4m3_value(b) for b in range(256)], dtype=np.float64)


def e4m3_bytes_to_f64(b: np.ndarray) -> np.ndarray:
    return _E4M3_TABLE[b.astype(np.uint8)]


def dequant(x_bits: np.ndarray, dtype: str, scale: np.ndarray | None = None) -> np.ndarray:
    """Exact fp64 values of a [T, H, d] tensor given as raw bits.

    dtype 'bf16': uint16 bit patterns.  dtype 'fp8': uint8 e4m3 bytes times a
    per-head fp32 scale (value = e4m3(byte) * scale[h])."""
    if dtype == "bf16":
        return bf16_bits_to_f64(x_bits)
    if dtype == "fp8":
        x = e4m3_bytes_to_f64(x_bits)
        s = np.asarray(scale, dtype=np.float32).astype(np.float64)
        return x * s[None, :, None]
    raise ValueError(dtype)


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


def seq_blocks(cu_seqlens, block: int = 128):
    """Per sequence (offset, length, NB) and the global block offset of each."""
    out = []
    g0 = 0
    for s in range(len(cu_seqlens) - 1):
        o, e = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        nb = cdiv(e - o, block)
        out.append((o, e - o, nb, g0))
        g0 += nb
    return out, g0


# --------------------------------------------------------------------------
# Step 1: value-magnitude bonus (gist-zh §2.2 / gist-de §2 B: the magnitude
# term beta * max(0, log ||V_j||^2); gist-zh §2.2 "block-wise downsampling and
# max-pooling of the value norms").  Max-pool of ||v||^2 over the tokens of the
# key block, then the log (log is monotone, so pooling before or after it is
# the same).
# --------------------------------------------------------------------------

def value_bonus(v: np.ndarray, cu_seqlens, beta: float, block: int = 128, mode: int = BONUS_LOG) -> np.ndarray:
    """v: fp64 [T, Hkv, d].  Returns bonus fp64 [Hkv, NBtot].

    x_j = ln max_{t in block j} ||v_t||^2 (gist-zh §2.2; the max is pooled
    over the block's tokens before the log, which is the same as pooling the
    logs).

    mode BONUS_LOG (gist-zh §2.2, gist-de §2 C): bonus_j = beta * max(0, x_j);
    ln 0 = -inf gives 0.

    mode BONUS_STANDARDIZED (AngelSlim doc §2.1 and the Stem overview's OAM
    formula: lambda * ReLU(v_bar_j), v_bar the standardized log value norm):
    v_bar_j = (x_j - mean) / std over the finite x of the same sequence and KV
    head (all its key blocks; population std); bonus_j = beta * max(0, v_bar_j).
    A block whose x is not finite gets 0, and so does every block when the std
    is 0 or fewer than one finite x exists.  The pages do not define the
    statistics' scope; this is the reading used here."""
    seqs, nbtot = seq_blocks(cu_seqlens, block)
    hkv = v.shape[1]
    bonus = np.zeros((hkv, nbtot), dtype=np.float64)
    for (o, L, nb, g0) in seqs:
        x = np.empty((hkv, nb), dtype=np.float64)
        for j in range(nb):
            rows = v[o + j * block: o + min((j + 1) * block, L)]  # [n, Hkv, d]
            sq = np.sum(rows * rows, axis=2)  # ||v_t||^2  [n, Hkv]
            m = np.max(sq, axis=0)  # max over the tokens of block j
            with np.errstate(divide="ignore"):
                x[:, j] = np.log(m)  # ln 0 = -inf
        if mode == BONUS_LOG:
            bonus[:, g0:g0 + nb] = beta * np.maximum(0.0, x)
            continue
        for h in range(hkv):
            fin = np.isfinite(x[h])
            if not fin.any():
                continue
            mean = x[h][fin].mean()
            std = math.sqrt(((x[h][fin] - mean) ** 2).mean())
            if std == 0.0:
                continue
            z = np.where(fin, (np.where(fin, x[h], 0.0) - mean) / std, -np.inf)
            bonus[h, g0:g0 + nb] = beta * np.maximum(0.0, z)
    return bonus


# --------------------------------------------------------------------------
# Step 2: anti-diagonal downsampled Q.K^T (AngelSlim-doc §2.1: score =
# Q.K^T / (sqrt(d) * s * n); gist-zh §2.3 and gist-de §2 C: anti-diagonal
# downsampling).  Group a of queries holds tokens a*s .. a*s+s-1; group b of
# keys likewise.  Query slot u is paired with key slot s-1-u.
# --------------------------------------------------------------------------

def _pad_groups(x: np.ndarray, s: int) -> np.ndarray:
    """x [L, H, d] -> [ceil(L/s)*s, H, d], missing tokens are zero."""
    L = x.shape[0]
    ng = cdiv(L, s)
    if ng * s == L:
        return x
    pad = np.zeros((ng * s - L,) + x.shape[1:], dtype=x.dtype)
    return np.concatenate([x, pad], axis=0)


def downsampled_scores(q: np.ndarray, k: np.ndarray, stride: int, norm: float,
                       groups: tuple[int, int] | None = None,
                       key_groups: int | None = None) -> np.ndarray:
    """Formulation A (via a BLAS product) for ONE sequence.

    q [L, Hq, d], k [L, Hkv, d] fp64.  Returns D [Hq, a1-a0, nk] with
    D[h, a, b] = sum_u q[a*s+u, h] . k[b*s+s-1-u, h//G] / (sqrt(d) * s * n)
    for query groups a in [a0, a1) (default: all) and key groups b < nk
    (default: all)."""
    s = stride
    L, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    ng = cdiv(L, s)
    a0, a1 = groups if groups is not None else (0, ng)
    nk = key_groups if key_groups is not None else ng
    qp = _pad_groups(q[a0 * s:min(a1 * s, L)], s)
    kp = _pad_groups(k[:min(nk * s, L)], s)
    na = qp.shape[0] // s
    # Q_ds[a] = concat_u q[a*s+u]      -> [na, s*d]
    # K_rev[b] = concat_u k[b*s+s-1-u] -> [nk, s*d]
    q_ds = qp.reshape(na, s, hq, d).transpose(2, 0, 1, 3).reshape(hq, na, s * d)
    k_rev = kp.reshape(nk, s, hkv, d)[:, ::-1].transpose(2, 0, 1, 3).reshape(hkv, nk, s * d)
    denom = math.sqrt(d) * s * norm
    out = np.empty((hq, na, nk), dtype=np.float64)
    for h in range(hq):
        out[h] = (q_ds[h] @ k_rev[h // G].T) / denom
    return out


def downsampled_scores_antidiag(q: np.ndarray, k: np.ndarray, stride: int, norm: float) -> np.ndarray:
    """Formulation B for ONE (tiny) sequence: the full fp64 attention logit
    matrix Q.K^T / sqrt(d), then the anti-diagonal of each s x s tile averaged
    (sum over the anti-diagonal divided by s) and divided by n."""
    s = stride
    L, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    qp = _pad_groups(q, s)
    kp = _pad_groups(k, s)
    Lp = qp.shape[0]
    ng = Lp // s
    out = np.zeros((hq, ng, ng), dtype=np.float64)
    for h in range(hq):
        P = (qp[:, h, :] @ kp[:, h // G, :].T) / math.sqrt(d)  # [Lp, Lp]
        for a in range(ng):
            for b in range(ng):
                acc = 0.0
                for u in range(s):
                    acc += P[a * s + u, b * s + (s - 1 - u)]
                out[h, a, b] = acc / s / norm
    return out


# --------------------------------------------------------------------------
# Step 3: block max-pooling plus the OAM bonus (gist-zh §2.2 M_ij = routing
# score + beta * max(0, log ||V_j||^2), evaluated block-wise on the
# downsampled scores).  Entries above the causal diagonal (j > i) are -inf.
# --------------------------------------------------------------------------

def block_scores(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens, p: Params) -> np.ndarray:
    """fp64 [Hq, NBtot, nb_max] block-score matrix, rows in sequence order.

    The query side is processed in chunks of ``chunk_size`` tokens (the pages'
    scoring chunk width); this changes nothing in the values."""
    B, s = p.block_size, p.stride
    gpb = B // s  # downsampled groups per block
    seqs, nbtot = seq_blocks(cu_seqlens, B)
    nb_max = max(nb for (_, _, nb, _) in seqs)
    hq, hkv = q.shape[1], k.shape[1]
    G = hq // hkv
    bonus = value_bonus(v, cu_seqlens, p.beta, B, p.bonus_mode)
    S = np.full((hq, nbtot, nb_max), -np.inf, dtype=np.float64)
    chunk_blocks = max(1, p.chunk_size // B)
    for (o, L, nb, g0) in seqs:
        qs, ks = q[o:o + L], k[o:o + L]
        ng_valid = cdiv(L, s)
        for i0 in range(0, nb, chunk_blocks):
            i1 = min(nb, i0 + chunk_blocks)
            a0, a1 = i0 * gpb, min(i1 * gpb, ng_valid)
            # only causal key blocks j <= i1-1 are needed for this chunk
            D = downsampled_scores(qs, ks, s, p.norm, groups=(a0, a1), key_groups=a1)
            for i in range(i0, i1):
                ra = slice(i * gpb - a0, min((i + 1) * gpb, ng_valid) - a0)
                for j in range(i + 1):
                    cb = slice(j * gpb, min((j + 1) * gpb, ng_valid))
                    blk = D[:, ra, cb]
                    S[:, g0 + i, j] = blk.reshape(hq, -1).max(axis=1) + bonus[np.arange(hq) // G, g0 + j]
    return S


def block_score_row(q: np.ndarray, k: np.ndarray, v: np.ndarray, i: int, p: Params) -> np.ndarray:
    """Row i of the block-score matrix of ONE sequence and ONE query head:
    q [L, 1, d], k/v [L, 1, d] fp64 (the query head and its KV head).  Same
    steps as block_scores, restricted to the query groups of block i and the
    key groups of blocks 0..i (used to check sampled rows of long inputs)."""
    B, s = p.block_size, p.stride
    gpb = B // s
    L = q.shape[0]
    ng_valid = cdiv(L, s)
    a0, a1 = i * gpb, min((i + 1) * gpb, ng_valid)
    D = downsampled_scores(q, k, s, p.norm, groups=(a0, a1), key_groups=min((i + 1) * gpb, ng_valid))[0]
    # the standardized form needs every block of the sequence; the log form
    # only blocks 0..i, so both take the whole sequence here
    bonus = value_bonus(v, [0, L], p.beta, B, p.bonus_mode)[0]
    out = np.empty(i + 1)
    for j in range(i + 1):
        out[j] = D[:, j * gpb:min((j + 1) * gpb, ng_valid)].max() + bonus[j]
    return out


# --------------------------------------------------------------------------
# Step 4: Token Position-Decay budget (gist-zh §2.1 / gist-de §2 A):
#   k(i) = floor(k_start - k_start * (1 - mu) / N * i),  k_end = mu * k_start,
# with the keep-ratio mapping and the forced blocks of AngelSlim-doc §2.2.
# --------------------------------------------------------------------------

def forced_blocks(i: int, sink: int, window: int) -> list[int]:
    """Sink blocks {0 .. min(S, c)-1} and the last W causal blocks
    {max(0, c-W) .. i} (window includes the diagonal), c = i + 1."""
    c = i + 1
    f = set(range(min(sink, c))) | set(range(max(0, c - window), c))
    return sorted(f)


def tpd_k(i: int, nb: int, p: Params) -> tuple[int, int]:
    """(k_start, k(i)) of query block i in a sequence of nb blocks, before the
    forced blocks and the causal cap are applied."""
    c = i + 1
    rho, mu = float(p.keep_ratio), float(p.mu)
    if p.budget_mode == RELATIVE:
        ks = math.ceil(rho * float(c))
    else:
        ks = math.ceil(rho * float(nb))
    ksf = float(ks)
    k = math.floor(ksf - ((ksf * (1.0 - mu)) * float(i)) / float(nb))
    return ks, k


def tpd_budget(i: int, nb: int, p: Params) -> int:
    """Budget b_i of query block i of a sequence with nb blocks."""
    _, k = tpd_k(i, nb, p)
    nf = len(forced_blocks(i, p.sink_blocks, p.window_blocks))
    return min(i + 1, max(k, nf))


def budgets(cu_seqlens, p: Params) -> np.ndarray:
    """int64 [NBtot]: one budget per query block (identical for every head)."""
    seqs, nbtot = seq_blocks(cu_seqlens, p.block_size)
    out = np.zeros(nbtot, dtype=np.int64)
    for (_, _, nb, g0) in seqs:
        for i in range(nb):
            out[g0 + i] = tpd_budget(i, nb, p)
    return out


# --------------------------------------------------------------------------
# Step 5: top-k block selection (gist-zh §2.3 "select the key blocks by OAM";
# AngelSlim-doc §2.2 sinks and window always kept; HPC-BSA §3.1 the inner loop
# only visits a pre-compacted list).
# --------------------------------------------------------------------------

def select_row(scores_row: np.ndarray, i: int, b: int, sink: int, window: int) -> list[int]:
    """Forced blocks first, then the best b-|F| of the remaining causal blocks
    by (score descending, index ascending); result in ascending order."""
    F = forced_blocks(i, sink, window)
    fs = set(F)
    rest = [j for j in range(i + 1) if j not in fs]

    def key(j):
        x = float(scores_row[j])
        return (math.inf if math.isnan(x) else -x, j)

    rest.sort(key=key)
    take = rest[: max(0, b - len(F))]
    return sorted(F + take)


def group_pooled_scores(scores: np.ndarray, hkv: int) -> np.ndarray:
    """GQA-shared lists (NEXT variant of the selection; HPC-BSA article §3.1
    block lists shared by the query heads of a KV head): every query head's
    score row becomes the elementwise max over the query heads of its KV
    group, NaN counted as -inf (the selection's NaN rule)."""
    hq = scores.shape[0]
    G = hq // hkv
    out = np.empty_like(scores)
    for hk in range(hkv):
        grp = scores[hk * G:(hk + 1) * G]
        pooled = np.where(np.isnan(grp), -np.inf, grp).max(axis=0)
        out[hk * G:(hk + 1) * G] = pooled
    return out


def select(scores: np.ndarray, cu_seqlens, p: Params, hkv: int | None = None):
    """scores fp64 [Hq, NBtot, nb_max] -> (budgets [Hq*NBtot], row_ptr
    [Hq*NBtot+1], col_idx [nnz]) with CSR row r = h*NBtot + g.  With
    p.list_mode == LIST_PER_GROUP (hkv required) the query heads of a KV
    group select on their pooled scores and so share one list."""
    if p.list_mode == LIST_PER_GROUP:
        scores = group_pooled_scores(scores, hkv)
    seqs, nbtot = seq_blocks(cu_seqlens, p.block_size)
    hq = scores.shape[0]
    bud = budgets(cu_seqlens, p)
    rows = []
    for h in range(hq):
        for (_, _, nb, g0) in seqs:
            for i in range(nb):
                rows.append(select_row(scores[h, g0 + i], i, int(bud[g0 + i]),
                                       p.sink_blocks, p.window_blocks))
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    col_idx = np.array([j for r in rows for j in r], dtype=np.int64)
    return np.tile(bud, hq), row_ptr, col_idx


# --------------------------------------------------------------------------
# Step 6: block-sparse attention (gist-zh §2.3 exact softmax and aggregation
# over the selected blocks only; HPC-BSA §3.1 the compacted list).
# --------------------------------------------------------------------------

def _softmax_scale(p: Params, d: int) -> float:
    return p.softmax_scale if p.softmax_scale > 0 else 1.0 / math.sqrt(d)


def bsa(q, k, v, cu_seqlens, row_ptr, col_idx, p: Params, rows_subset=None):
    """Formulation A: gather only the listed key blocks.

    q [T, Hq, d], k/v [T, Hkv, d] fp64.  Returns O fp64 [T, Hq, d] and LSE fp64
    [Hq, T].  Key set of query token t in block i: union over listed j of the
    tokens of block j that are <= t.  ``rows_subset`` optionally limits the
    work to a list of (h, g) CSR rows (others stay NaN)."""
    B = p.block_size
    T, hq, d = q.shape
    G = hq // k.shape[1]
    sigma = _softmax_scale(p, d)
    seqs, nbtot = seq_blocks(cu_seqlens, B)
    O = np.full((T, hq, d), np.nan)
    LSE = np.full((hq, T), np.nan)
    gmap = {}
    for (o, L, nb, g0) in seqs:
        for i in range(nb):
            gmap[g0 + i] = (o, L, i)
    todo = rows_subset if rows_subset is not None else [(h, g) for h in range(hq) for g in range(nbtot)]
    for (h, g) in todo:
        o, L, i = gmap[g]
        r = h * nbtot + g
        blocks = [int(j) for j in col_idx[row_ptr[r]:row_ptr[r + 1]]]
        t0, t1 = i * B, min((i + 1) * B, L)
        key_tok = np.concatenate([np.arange(j * B, min((j + 1) * B, L)) for j in blocks])
        Qi = q[o + t0:o + t1, h, :]
        Kj = k[o + key_tok, h // G, :]
        Vj = v[o + key_tok, h // G, :]
        logits = sigma * (Qi @ Kj.T)
        tq = np.arange(t0, t1)[:, None]
        logits = np.where(key_tok[None, :] <= tq, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        l = e.sum(axis=1, keepdims=True)
        O[o + t0:o + t1, h, :] = (e @ Vj) / l
        LSE[h, o + t0:o + t1] = (m + np.log(l))[:, 0]
    return O, LSE


def bsa_masked(q, k, v, cu_seqlens, row_ptr, col_idx, p: Params):
    """Formulation B (tiny inputs): the full causal logit matrix with -inf
    written into every key block that is not listed (HPC-BSA §3.1: a skipped
    block is the same as a block of -inf scores), then an ordinary softmax."""
    B = p.block_size
    T, hq, d = q.shape
    G = hq // k.shape[1]
    sigma = _softmax_scale(p, d)
    seqs, nbtot = seq_blocks(cu_seqlens, B)
    O = np.zeros((T, hq, d))
    LSE = np.zeros((hq, T))
    for (o, L, nb, g0) in seqs:
        for h in range(hq):
            logits = sigma * (q[o:o + L, h, :] @ k[o:o + L, h // G, :].T)
            keep = np.zeros((L, L), dtype=bool)
            for i in range(nb):
                r = h * nbtot + g0 + i
                for j in col_idx[row_ptr[r]:row_ptr[r + 1]]:
                    keep[i * B:(i + 1) * B, int(j) * B:(int(j) + 1) * B] = True
            causal = np.tril(np.ones((L, L), dtype=bool))
            logits = np.where(keep & causal, logits, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            l = e.sum(axis=1, keepdims=True)
            O[o:o + L, h, :] = (e @ v[o:o + L, h // G, :]) / l
            LSE[h, o:o + L] = (m + np.log(l))[:, 0]
    return O, LSE


def full_csr(cu_seqlens, hq: int, block: int = 128):
    """Every causal block of every query block (the dense comparator)."""
    seqs, nbtot = seq_blocks(cu_seqlens, block)
    rows = []
    for h in range(hq):
        for (_, _, nb, g0) in seqs:
            for i in range(nb):
                rows.append(list(range(i + 1)))
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    col_idx = np.array([j for r in rows for j in r], dtype=np.int64)
    return row_ptr, col_idx


def gather_paged(pages: np.ndarray, page_table: np.ndarray, cu_seqlens, page_size: int) -> np.ndarray:
    """Paged KV (AngelSlim doc's paged fp8 KV path for the block-sparse
    attention): the keys (or values) of sequence s, token t, live at
    pages[page_table[s][t // page_size], t % page_size].  pages [P, page_size,
    H, d]; page_table [num_seqs, max_pages] int.  Returns the packed [T, H, d]
    tensor that the contiguous path reads, which is all the paged path means:
    attention over paged K/V equals attention over this gather."""
    T = cu_seqlens[-1]
    out = np.empty((T,) + pages.shape[2:], dtype=pages.dtype)
    for s in range(len(cu_seqlens) - 1):
        for t in range(cu_seqlens[s + 1] - cu_seqlens[s]):
            out[cu_seqlens[s] + t] = pages[page_table[s][t // page_size], t % page_size]
    return out


def prefill(q, k, v, cu_seqlens, p: Params):
    """score -> select -> block-sparse attention, all in fp64."""
    S = block_scores(q, k, v, cu_seqlens, p)
    bud, row_ptr, col_idx = select(S, cu_seqlens, p, hkv=k.shape[1])
    O, LSE = bsa(q, k, v, cu_seqlens, row_ptr, col_idx, p)
    return dict(scores=S, budgets=bud, row_ptr=row_ptr, col_idx=col_idx, out=O, lse=LSE)


# --------------------------------------------------------------------------
# Work counts used to label oracle timings (the same algorithmic counts the
# GPU side reports).
# --------------------------------------------------------------------------

def nnz_blocks(cu_seqlens, p: Params, hq: int) -> int:
    return int(budgets(cu_seqlens, p).sum()) * hq
