"""stem_prefill_host (host buffers, transfers overlapped with compute, one
KV-head group at a time) must give exactly stem_prefill's results."""

import pytest
import torch

from block_sparse_attention_stem_b200 import inputs as I
from gpu_common import make_gpu_qkv

pytestmark = pytest.mark.gpu

b = pytest.importorskip("block_sparse_attention_stem_b200.binding")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def W(seqlens, hq, hkv, dtype="bf16", seed=30, **kw):
    base = dict(keep_ratio=0.3, mu=0.7, beta=0.2, sink_blocks=1, window_blocks=2)
    base.update(kw)
    return I.Workload(name="case", seqlens=seqlens, num_q_heads=hq, num_kv_heads=hkv, dtype=dtype, seed=seed, **base)


CASES = {
    "varlen_gqa4": W([1000, 128, 2088], 8, 2),
    "odd_group": W([1500, 700], 6, 2, seed=31),
    "more_kv_heads_than_groups": W([640, 1024], 16, 16, seed=32),  # 16 KV heads -> 8 groups of 2
    "fp8_varlen": W([640, 2048, 77], 4, 2, dtype="fp8", seed=33),
    "qwen32k": I.workload("qwen32k"),
    "one_kv_head": W([1000, 300], 4, 1, seed=34),  # a single group
    "one_kv_head_odd_group": W([1500], 3, 1, seed=35),
    "mha": W([700], 2, 2, seed=38),  # one query head per KV head
    "std_bonus": W([1000, 128, 2088], 8, 2, seed=36, bonus_mode=1),  # per-KV-head z-score per group
    "group_lists": W([1000, 2088], 8, 2, seed=37, list_mode=1),  # the separate selection pass
    "b64_varlen": W([1000, 128, 2088, 63], 8, 2, seed=39, block_size=64),  # 64-token blocks
}


@pytest.mark.parametrize("name,select_mode", [(n, 0) for n in CASES] + [("varlen_gqa4", 1), ("fp8_varlen", 1)])
def test_prefill_host_matches_prefill(name, select_mode):
    """select_mode 1: each KV-head group's scoring kernel also selects its rows."""
    w = CASES[name]
    inp = I.make_inputs(w, device="cuda")
    qkv = make_gpu_qkv(b, inp, w.cu_seqlens())
    params = b.make_params(**w.params(), select_mode=select_mode)
    out_ref, lse_ref, _, _, _ = b.stem_prefill(qkv, params, return_lists=False)
    torch.cuda.synchronize()
    # host copies of the inputs; the device input tensors are overwritten by the call
    hq_t = inp["q"].cpu().pin_memory()
    hk_t = inp["k"].cpu().pin_memory()
    hv_t = inp["v"].cpu().pin_memory()
    dq, dk, dv = torch.zeros_like(inp["q"]), torch.zeros_like(inp["k"]), torch.zeros_like(inp["v"])
    qkv2 = b.make_qkv(dq, dk, dv, w.cu_seqlens(), q_scale=inp["q_scale"], k_scale=inp["k_scale"],
                      v_scale=inp["v_scale"], cu_seqlens_dev=inp["cu_seqlens"])
    T, hq = w.total_tokens, w.num_q_heads
    out_h = torch.full((T, hq, 128), float("nan"), dtype=torch.bfloat16).pin_memory()
    lse_h = torch.full((hq, T), float("nan"), dtype=torch.float32).pin_memory()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        _, _, ws = b.stem_prefill_host(qkv2, params, hq_t, hk_t, hv_t, out_h, lse_h, stream=stream)
    stream.synchronize()
    assert b.stem_read_device_status(ws) == 0
    assert torch.equal(dq, inp["q"]) and torch.equal(dk, inp["k"]) and torch.equal(dv, inp["v"])
    assert torch.equal(out_h.view(torch.int16), out_ref.cpu().view(torch.int16))
    assert torch.equal(lse_h.view(torch.int32), lse_ref.cpu().view(torch.int32))
