"""The allocation-free prefill entry point (stem_prefill_noalloc).

Some callers cannot allocate device memory for a workspace; this entry point
runs the same pipeline on a built-in 32 MiB device array instead.  These tests
call it through the C ABI and check it against stem_prefill with a
caller-allocated workspace, on two calls in a row with different inputs (the
built-in array keeps the previous call's contents, which must not leak into
the next result).  The file is named to be collected last.
"""

import numpy as np
import pytest
import torch

from block_sparse_attention_stem_b200 import inputs as I
from gpu_common import TOL_LSE, TOL_OUT, make_gpu_qkv, out_error, to_device

pytestmark = pytest.mark.gpu

b = pytest.importorskip("block_sparse_attention_stem_b200.binding")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def _case(seed, dtype="bf16", block_size=128, select_mode=0):
    w = I.Workload(name="noalloc", seqlens=[3000, 1000, 640], num_q_heads=8, num_kv_heads=2, dtype=dtype,
                   seed=seed, keep_ratio=0.3, mu=0.7, beta=0.2, sink_blocks=1, window_blocks=2,
                   block_size=block_size)
    dinp = to_device(I.make_inputs(w))
    return w, make_gpu_qkv(b, dinp, w.cu_seqlens()), b.make_params(**w.params(), select_mode=select_mode)


@pytest.mark.parametrize("dtype,block_size,select_mode", [("bf16", 128, 0), ("fp8", 128, 0), ("bf16", 64, 0),
                                                          ("bf16", 128, 1)])
def test_noalloc_matches_workspace_prefill_on_two_calls(dtype, block_size, select_mode):
    for seed in (101, 202):
        w, qkv, params = _case(seed, dtype, block_size, select_mode)
        ref_out, ref_lse, ref_rp, ref_ci, ws = b.stem_prefill(qkv, params)
        out, lse, rp, ci = b.stem_prefill_noalloc(qkv, params)
        torch.cuda.synchronize()
        assert b.stem_read_device_status(ws) == 0
        assert b.stem_noalloc_read_device_status() == 0  # the built-in workspace's own status word
        assert torch.equal(rp, ref_rp) and torch.equal(ci, ref_ci)
        err = out_error(out.float().cpu().numpy(), ref_out.float().cpu().numpy())
        assert err <= TOL_OUT[dtype]
        assert float((lse - ref_lse).abs().max()) <= TOL_LSE
        # same kernels on the same inputs: the results are in fact identical
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_noalloc_status_word_reads_ok_on_any_stream_of_the_device():
    """The built-in workspace's status word (where a timed-out wait or a
    malformed list entry would be recorded; a valid prefill produces neither)
    reads STEM_OK after calls on the default stream and on a side stream of
    the same device, which the device check accepts."""
    w, qkv, params = _case(303)
    b.stem_prefill_noalloc(qkv, params)
    assert b.stem_noalloc_read_device_status() == 0
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b.stem_prefill_noalloc(qkv, params, stream=s)
    assert b.stem_noalloc_read_device_status(s) == 0


def test_noalloc_rejects_problems_larger_than_its_workspace():
    w = I.Workload(name="big", seqlens=[65536], num_q_heads=32, num_kv_heads=8)
    q = torch.zeros(1, 32, 128, dtype=torch.bfloat16, device="cuda")  # never read: rejected on the host
    qkv = b.make_qkv(q, q[:, :8], q[:, :8].clone(), w.cu_seqlens())
    qkv.desc.total_tokens = 65536
    params = b.make_params()
    assert b.stem_plan(qkv, params).ws_prefill_bytes > (32 << 20)
    with pytest.raises(b.StemError) as e:
        b.stem_prefill_noalloc(qkv, params, out=q, lse=torch.zeros(1, device="cuda"), return_lists=False)
    assert e.value.code == 3  # STEM_ERR_WORKSPACE_TOO_SMALL
