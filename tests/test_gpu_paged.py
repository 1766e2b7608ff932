"""Attention over paged K/V (stem_bsa_fwd_paged): the same results as the
packed path, bit for bit, for any page size that is a multiple of 64 and any
placement of the pages in the pool."""

import numpy as np
import pytest
import torch

from oracle import stem_oracle as O
from block_sparse_attention_stem_b200 import inputs as I
from gpu_common import check_attention, make_gpu_qkv

pytestmark = pytest.mark.gpu

b = pytest.importorskip("block_sparse_attention_stem_b200.binding")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def W(seqlens, hq, hkv, dtype="bf16", seed=50, **kw):
    base = dict(keep_ratio=0.4, mu=0.7, beta=0.2, sink_blocks=1, window_blocks=2)
    base.update(kw)
    return I.Workload(name="case", seqlens=seqlens, num_q_heads=hq, num_kv_heads=hkv, dtype=dtype, seed=seed, **base)


def to_pages(x, cu, page_size, rng, spare=3):
    """Packed [T, H, d] -> (pool [P, page_size, H, d], table int32 [S, max_pages]):
    each sequence padded to a multiple of 128 tokens with zeros, pages placed
    at random pool slots; spare pages hold NaN (never referenced)."""
    S = len(cu) - 1
    npg = [((cu[s + 1] - cu[s] + 127) // 128 * 128 + page_size - 1) // page_size for s in range(S)]
    P = sum(npg) + spare
    pool = torch.full((P, page_size) + tuple(x.shape[1:]), float("nan"), dtype=torch.float32).to(x.dtype)
    if x.dtype == torch.uint8:
        pool = torch.full((P, page_size) + tuple(x.shape[1:]), 0x7F, dtype=torch.uint8)  # e4m3 NaN
    slots = rng.permutation(P)
    table = np.zeros((S, max(npg)), dtype=np.int32)
    k = 0
    for s in range(S):
        L = cu[s + 1] - cu[s]
        for pg in range(npg[s]):
            page = torch.zeros((page_size,) + tuple(x.shape[1:]), dtype=x.dtype)
            n = max(0, min(page_size, L - pg * page_size))
            page[:n] = x[cu[s] + pg * page_size: cu[s] + pg * page_size + n].cpu()
            pool[slots[k]] = page
            table[s, pg] = slots[k]
            k += 1
    return pool, torch.from_numpy(table)


CASES = {
    "varlen_page64": (W([1000, 128, 2088], 8, 2), 64),
    "gqa_page128": (W([1500, 700], 6, 2, seed=51), 128),
    "fp8_page256": (W([640, 2048, 77], 4, 2, dtype="fp8", seed=52), 256),
    "shared_lists_page64": (W([1000, 128, 2088], 8, 2, seed=53, list_mode=1), 64),  # two heads per CTA
    # 64-token blocks: every 64-key unit is one page lookup
    "b64_page64": (W([1000, 128, 2088, 63], 8, 2, seed=54, block_size=64), 64),
    "b64_fp8_page128": (W([640, 2112, 77], 4, 2, dtype="fp8", seed=55, block_size=64), 128),
    "b64_shared_lists_page64": (W([1000, 2088], 8, 2, seed=56, block_size=64, list_mode=1), 64),
}


@pytest.mark.parametrize("name", list(CASES))
def test_paged_equals_packed(name):
    w, ps = CASES[name]
    cu = w.cu_seqlens()
    inp = I.make_inputs(w, device="cuda")
    qkv = make_gpu_qkv(b, inp, cu)
    params = b.make_params(**w.params())
    out_ref, lse_ref, rp, ci, ws = b.stem_prefill(qkv, params)
    rng = np.random.default_rng(7)
    kp, table = to_pages(inp["k"], cu, ps, rng)
    vp, table_v = to_pages(inp["v"], cu, ps, np.random.default_rng(7))
    assert torch.equal(table, table_v)
    kp, vp, table = kp.cuda(), vp.cuda(), table.cuda()
    kv = b.paged_kv(kp, vp, table, ps)
    out, lse, ws2 = b.stem_bsa_fwd_paged(qkv, kv, params, rp, ci)
    torch.cuda.synchronize()
    assert b.stem_read_device_status(ws2) == 0
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32))


@pytest.mark.parametrize("name", ["varlen_page64", "fp8_page256", "b64_page64", "b64_fp8_page128"])
def test_paged_attention_matches_oracle_through_the_gather(name):
    w, ps = CASES[name]
    cu = w.cu_seqlens()
    inp = I.make_inputs(w, device="cuda")
    qkv = make_gpu_qkv(b, inp, cu)
    params = b.make_params(**w.params())
    _, _, rp, ci, _ = b.stem_prefill(qkv, params)
    kp, table = to_pages(inp["k"], cu, ps, np.random.default_rng(3))
    vp, _ = to_pages(inp["v"], cu, ps, np.random.default_rng(3))
    out, lse, ws = b.stem_bsa_fwd_paged(qkv, b.paged_kv(kp.cuda(), vp.cuda(), table.cuda(), ps), params, rp, ci)
    torch.cuda.synchronize()
    assert b.stem_read_device_status(ws) == 0

    def pool_f64(pool, name):
        """fp64 values of a [P, page_size, H, d] pool (fp8: times the per-head scale)."""
        flat = pool.reshape(-1, *pool.shape[2:])
        if w.dtype == "bf16":
            x = O.dequant(I.raw_bits(flat), "bf16")
        else:
            x = O.dequant(I.raw_bits(flat), "fp8", inp[name + "_scale"].cpu().numpy())
        return x.reshape(pool.shape)

    if w.dtype == "bf16":
        q = O.dequant(I.raw_bits(inp["q"].cpu()), "bf16")
    else:
        q = O.dequant(I.raw_bits(inp["q"].cpu()), "fp8", inp["q_scale"].cpu().numpy())
    kg = O.gather_paged(pool_f64(kp, "k"), table.numpy(), cu, ps)
    vg = O.gather_paged(pool_f64(vp, "v"), table.numpy(), cu, ps)
    ro, rl = O.bsa(q, kg, vg, cu, rp.cpu().numpy(), ci.cpu().numpy(), O.Params(**w.params()))
    check_attention(out, lse, ro, rl, w.dtype)


def test_page_numbers_outside_the_pool_read_zeros():
    w, ps = CASES["gqa_page128"]
    cu = w.cu_seqlens()
    inp = I.make_inputs(w, device="cuda")
    qkv = make_gpu_qkv(b, inp, cu)
    params = b.make_params(**w.params())
    _, _, rp, ci, _ = b.stem_prefill(qkv, params)
    kp, table = to_pages(inp["k"], cu, ps, np.random.default_rng(5))
    vp, _ = to_pages(inp["v"], cu, ps, np.random.default_rng(5))
    bad = table.clone()
    bad[0, 2] = -1                  # before the pool
    bad[1, 0] = kp.shape[0] + 5     # past it
    out, lse, ws = b.stem_bsa_fwd_paged(qkv, b.paged_kv(kp.cuda(), vp.cuda(), bad.cuda(), ps), params, rp, ci)
    torch.cuda.synchronize()
    assert b.stem_read_device_status(ws) == 0
    # the packed path over K/V with those pages' tokens zeroed
    k0, v0 = inp["k"].clone(), inp["v"].clone()
    for s, pg in ((0, 2), (1, 0)):
        t0 = cu[s] + pg * ps
        t1 = min(cu[s + 1], t0 + ps)
        k0[t0:t1] = 0
        v0[t0:t1] = 0
    qkv0 = b.make_qkv(inp["q"], k0, v0, cu, cu_seqlens_dev=inp["cu_seqlens"])
    out0, lse0, _ = b.stem_bsa_fwd(qkv0, params, rp, ci)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out0.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), lse0.view(torch.int32))
