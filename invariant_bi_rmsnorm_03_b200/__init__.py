"""Batch-invariant transformer forward kernels for B200 (sm_100a).

The computation lives in the CUDA library ``lib/libbi.so`` behind the C ABI of
``include/bi.h``; this package is its thin Python binding (torch tensors in,
torch tensors out).  Functions of the same names as the C entry points are
re-exported from the default (batch-invariant) build; ``load(variant=True)``
gives the variant-off build used to measure the cost of invariance.
"""
from .binding import (BIError, Library, PagedKV, Status, load, NOALLOC_SCRATCH_BYTES,  # noqa: F401
                      PAGE_SIZE, SPLIT_KEYS)


def _default():
    return load(False)


def bi_rmsnorm(*a, **k):
    return _default().bi_rmsnorm(*a, **k)


def bi_matmul(*a, **k):
    return _default().bi_matmul(*a, **k)


def bi_kv_write(*a, **k):
    return _default().bi_kv_write(*a, **k)


def bi_attention_decode(*a, **k):
    return _default().bi_attention_decode(*a, **k)


def bi_attention_prefill(*a, **k):
    return _default().bi_attention_prefill(*a, **k)


def bi_device_status(*a, **k):
    return _default().bi_device_status(*a, **k)


def bi_build_invariant():
    return _default().bi_build_invariant()
