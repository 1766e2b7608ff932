"""Failure detection on the GPU without a fault: a kernel waits on a barrier
that nothing arrives on; the bounded wait must give up, report
STEM_ERR_TIMEOUT through the workspace status word, and leave the context
usable for the next call."""

import time

import pytest
import torch

from block_sparse_attention_stem_b200 import inputs as I
from gpu_common import make_gpu_qkv, to_device

pytestmark = pytest.mark.gpu

b = pytest.importorskip("block_sparse_attention_stem_b200.binding")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    b.stem_selftest_wait_timeout(ws)
    status = b.stem_read_device_status(ws)
    elapsed = time.time() - t0
    assert status == 6, b.stem_status_string(status)  # STEM_ERR_TIMEOUT
    assert 1.5 < elapsed < 30.0
    # the context is still usable: a normal prefill runs and reports no error
    w = I.workload("tiny")
    d = to_device(I.make_inputs(w))
    qkv = make_gpu_qkv(b, d, w.cu_seqlens())
    out, lse, rp, ci, ws2 = b.stem_prefill(qkv, b.make_params(**w.params()))
    assert b.stem_read_device_status(ws2) == 0
    assert torch.isfinite(out.float()).all()
