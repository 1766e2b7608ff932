"""Host-side checks of the C ABI (no GPU needed, no kernel is launched).

* the shared library loads and exports every entry point include/stem.h
  declares;
* stem_plan's data-independent numbers (nnz, budgets sum, work counts) agree
  with the oracle;
* argument validation rejects every documented bad input before anything is
  enqueued (these calls return before touching CUDA).
"""

import ctypes
import math
import os
import re

import numpy as np
import pytest
import torch

from oracle import stem_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
b = pytest.importorskip("block_sparse_attention_stem_b200.binding")
from block_sparse_attention_stem_b200 import inputs as I  # noqa: E402


def header_functions():
    src = open(os.path.join(ROOT, "include", "stem.h")).read()
    return re.findall(r"STEM_API\s+[\w\s\*]+?\b(stem_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    names = header_functions()
    assert set(names) == set(b.EXPORTED)
    for n in names:
        assert hasattr(b.LIB, n), n
    assert b.LIB.stem_version() >= 100
    for code in range(8):
        assert b.stem_status_string(code) not in ("", "unknown status")
    assert b.stem_status_string(99) == "unknown status"


def fake_qkv(seqlens, hq, hkv, d=128, fp8=False):
    T = int(sum(seqlens))
    dt = torch.uint8 if fp8 else torch.bfloat16
    q = torch.zeros(max(T, 1), hq, d, dtype=dt)
    k = torch.zeros(max(T, 1), hkv, d, dtype=dt)
    cu = [0] + list(np.cumsum(seqlens))
    sc = torch.ones(hq, dtype=torch.float32) if fp8 else None
    return b.make_qkv(q, k, k.clone(), cu, q_scale=sc, k_scale=sc, v_scale=sc, cu_seqlens_dev=torch.zeros(1))


def oparams(**kw):
    return O.Params(**kw)


@pytest.mark.parametrize("name", ["tiny", "qwen32k", "long128k", "sweep64k", "fp8_varlen"])
def test_plan_nnz_matches_oracle_budgets(name):
    w = I.workload(name)
    qkv = fake_qkv(w.seqlens, w.num_q_heads, w.num_kv_heads, fp8=(w.dtype == "fp8"))
    pl = b.stem_plan(qkv, b.make_params(**w.params()))
    cu = w.cu_seqlens()
    bud = O.budgets(cu, O.Params(**w.params()))
    assert pl.nnz == int(bud.sum()) * w.num_q_heads
    assert pl.nb_total == len(bud)
    assert pl.nb_max == max(math.ceil(L / 128) for L in w.seqlens)
    # work counts: score FLOPs = 2 s d Hq sum NB(NB+1)/2 * 16^2
    s = w.stride
    pairs = sum(math.ceil(L / 128) * (math.ceil(L / 128) + 1) // 2 for L in w.seqlens)
    assert pl.score_flops == pytest.approx(2 * s * 128 * w.num_q_heads * pairs * (128 // s) ** 2)
    assert 0 < pl.attn_flops <= pl.dense_attn_flops
    # fp8: the workspace holds V widened to f16 [T, Hkv, d] for the attention
    T = sum(w.seqlens)
    assert pl.vwide_bytes == (T * w.num_kv_heads * 128 * 2 if w.dtype == "fp8" else 0)
    assert pl.ws_bytes >= pl.vwide_bytes and pl.ws_prefill_bytes >= pl.ws_bytes


def test_plan_density_of_the_128k_workload():
    w = I.workload("long128k")
    qkv = fake_qkv(w.seqlens, 32, 8)
    pl = b.stem_plan(qkv, b.make_params(**w.params()))
    assert pl.nnz_per_head == 104793
    assert pl.nnz_per_head / (1024 * 1025 / 2) == pytest.approx(0.1997, abs=5e-5)  # kept / causal blocks
    # FLOP density is a little lower: the always-kept diagonal blocks are half masked
    assert pl.attn_flops / pl.dense_attn_flops == pytest.approx(0.1989, abs=5e-4)


@pytest.mark.parametrize("rho,mu,mode,S,W", [(0.3, 0.45, 0, 4, 4), (0.1, 1.0, 0, 0, 1), (0.25, 0.7, 1, 1, 2),
                                             (1.0, 1.0, 0, 0, 1), (0.05, 0.2, 1, 3, 5)])
@pytest.mark.parametrize("B", [128, 64])
def test_plan_budgets_equal_oracle_on_odd_parameters(rho, mu, mode, S, W, B):
    seqlens = [12800, 1000, 129, 1]
    qkv = fake_qkv(seqlens, 4, 2)
    p = dict(keep_ratio=rho, mu=mu, budget_mode=mode, sink_blocks=S, window_blocks=W, block_size=B)
    pl = b.stem_plan(qkv, b.make_params(**p))
    bud = O.budgets([0] + list(np.cumsum(seqlens)), O.Params(**p))
    assert pl.nnz_per_head == int(bud.sum())
    assert pl.nb_total == sum(math.ceil(L / B) for L in seqlens) == len(bud)
    assert pl.nb_max == math.ceil(max(seqlens) / B)
    # score FLOPs: 2 s d Hq sum NB(NB+1)/2 (B/s)^2
    pairs = sum(math.ceil(L / B) * (math.ceil(L / B) + 1) // 2 for L in seqlens)
    assert pl.score_flops == pytest.approx(2 * 8 * 128 * 4 * pairs * (B // 8) ** 2)


def test_plan_rejects_64_token_blocks_past_the_bitmap_limit():
    # 64-token blocks keep each tile's two lists as bitmaps of 32768 blocks;
    # planning reads only the host offsets, so one-token tensors stand in
    t = torch.zeros(1, 2, 128, dtype=torch.bfloat16)

    def qkv(L):
        return b.make_qkv(t, t, t, [0, L], cu_seqlens_dev=torch.zeros(1))

    assert b.stem_plan(qkv(32768 * 64), b.make_params(block_size=64)).nb_max == 32768
    assert _status(lambda: b.stem_plan(qkv(32768 * 64 + 1), b.make_params(block_size=64))) == 2
    assert b.stem_plan(qkv(32768 * 64 + 1), b.make_params(block_size=128)).nb_max == 16385


def _status(fn):
    with pytest.raises(b.StemError) as e:
        fn()
    return e.value.code


def test_validation_rejects_bad_parameters():
    qkv = fake_qkv([256], 4, 2)
    P = b.make_params
    assert _status(lambda: b.stem_plan(qkv, P(keep_ratio=0.0))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(keep_ratio=1.5))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(mu=0.0))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(mu=1.01))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(window_blocks=0))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(sink_blocks=-1))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(norm=0.0))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(beta=-0.1))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(chunk_size=0))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(softmax_scale=-1.0))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(budget_mode=2))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(bonus_mode=2))) == 1
    b.stem_plan(qkv, P(bonus_mode=1))  # the standardized bonus is valid
    assert _status(lambda: b.stem_plan(qkv, P(list_mode=2))) == 1
    b.stem_plan(qkv, P(list_mode=1))  # GQA-shared lists are valid
    b.stem_plan(qkv, P(select_mode=1))  # the selection inside the scoring kernel is valid
    assert _status(lambda: b.stem_plan(qkv, P(select_mode=2))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(stride=3))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(stride=16))) == 2
    b.stem_plan(qkv, P(block_size=64))  # 64-token blocks are valid
    assert _status(lambda: b.stem_plan(qkv, P(block_size=32))) == 2
    assert _status(lambda: b.stem_plan(qkv, P(block_size=96))) == 2
    assert _status(lambda: b.stem_plan(qkv, P(block_size=0))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(block_size=64, stride=16))) == 2  # divides 64, not supported
    assert _status(lambda: b.stem_plan(qkv, P(block_size=64, stride=3))) == 1
    assert _status(lambda: b.stem_plan(qkv, P(norm=float("nan")))) == 1


def test_validation_rejects_bad_shapes_and_pointers():
    P = b.make_params()
    assert _status(lambda: b.stem_plan(fake_qkv([256], 4, 3), P)) == 1     # Hq % Hkv
    assert _status(lambda: b.stem_plan(fake_qkv([256], 2, 2, d=64), P)) == 2  # head_dim
    qkv = fake_qkv([256, 128], 2, 2)
    qkv.cu_host[1] = 400  # decreasing offsets (0, 400, 384)
    assert _status(lambda: b.stem_plan(qkv, P)) == 1
    qkv = fake_qkv([256], 2, 2)
    qkv.desc.total_tokens = 255  # inconsistent with cu_seqlens
    assert _status(lambda: b.stem_plan(qkv, P)) == 1
    # misaligned q pointer
    qkv = fake_qkv([256], 2, 2)
    qkv.desc.q = qkv.desc.q + 2
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    out = torch.zeros(256, 2, 128, dtype=torch.bfloat16)
    lse = torch.zeros(2, 256)
    rp = torch.zeros(5, dtype=torch.int32)
    code = b.LIB.stem_bsa_fwd(ctypes.byref(qkv.desc), ctypes.byref(P), rp.data_ptr(), rp.data_ptr(),
                              out.data_ptr(), lse.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert code == 4
    # fp8 without scales
    qkv = fake_qkv([256], 2, 2, fp8=True)
    qkv.desc.k_scale = None
    code = b.LIB.stem_prefill(ctypes.byref(qkv.desc), ctypes.byref(P), out.data_ptr(), lse.data_ptr(), None,
                              None, ws.data_ptr(), ws.numel(), None)
    assert code == 1


def test_paged_kv_validation():
    qkv = fake_qkv([1000, 300], 4, 2)
    P = b.make_params()
    fake = 1 << 20  # never dereferenced: validation fails first

    def kv(page_size, num_pages, max_pages):
        return b.StemPagedKV(page_size, num_pages, max_pages, fake, fake, fake)

    def call(d):  # straight through the C ABI: no device memory is touched
        return b.LIB.stem_bsa_fwd_paged(ctypes.byref(qkv.desc), ctypes.byref(d), ctypes.byref(P), None, None, None,
                                        None, None, 0, None)

    assert call(kv(96, 64, 16)) == 1   # not a multiple of 64
    assert call(kv(0, 64, 16)) == 1
    assert call(kv(128, 64, 7)) == 1   # 1000 tokens need 8 pages of 128
    assert call(kv(64, 0, 16)) == 1
    assert call(kv(128, 64, 8)) == 1   # valid pages, but no lists: rejected too


def test_workspace_too_small_is_reported_before_launch():
    qkv = fake_qkv([4096], 4, 2)
    P = b.make_params()
    pl = b.stem_plan(qkv, P)
    ws = torch.zeros(pl.ws_prefill_bytes - 1, dtype=torch.uint8)
    out = torch.zeros(4096, 4, 128, dtype=torch.bfloat16)
    lse = torch.zeros(4, 4096)
    code = b.LIB.stem_prefill(ctypes.byref(qkv.desc), ctypes.byref(P), out.data_ptr(), lse.data_ptr(), None, None,
                              ws.data_ptr(), ws.numel(), None)
    assert code == 3
    sc = torch.zeros(pl.scores_bytes // 4)
    code = b.LIB.stem_score(ctypes.byref(qkv.desc), ctypes.byref(P), sc.data_ptr(), None, ws.data_ptr(),
                            pl.ws_bytes - 1, None)
    assert code == 3
    assert pl.ws_bytes < pl.ws_prefill_bytes
    assert pl.ws_prefill_bytes >= pl.scores_bytes + pl.nnz * 4
