"""Stem long-context prefill hot path for NVIDIA B200 (sm_100a).

``binding`` wraps the C ABI of ``libstem.so`` (include/stem.h): block scoring
with the output-aware metric, token position-decay top-k block selection and
causal block-sparse flash attention, in bf16 and fp8 e4m3, for GQA and
varlen-packed batches.  ``inputs`` draws the seeded synthetic workloads.
Submodules are imported on first use, so the input generators work on a
machine without the built library.
"""

import importlib

__all__ = ["binding", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
