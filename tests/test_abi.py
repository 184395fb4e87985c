"""The C-ABI library loads and exports every entry point include/bi.h
declares, and rejects bad arguments on the host before touching a device.
CPU only: no call here reaches a kernel launch."""
import ctypes
import os
import re

import pytest

import invariant_bi_rmsnorm_03_b200 as bi
from invariant_bi_rmsnorm_03_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bi.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bi_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module", params=[False, True], ids=["invariant", "variant_off"])
def lib(request):
    return bi.load(variant=request.param)


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("bi_rmsnorm", "bi_matmul", "bi_kv_write", "bi_attention_decode",
              "bi_attention_prefill", "bi_device_status"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib.lib, s), s
        assert ctypes.cast(getattr(lib.lib, s), ctypes.c_void_p).value


def test_header_constants_match_the_binding():
    text = open(HEADER).read()
    m = re.search(r"#define BI_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", text)
    assert m, "BI_NOALLOC_SCRATCH_BYTES not found"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == bi.NOALLOC_SCRATCH_BYTES
    assert re.search(r"#define BI_PAGE_SIZE %d\b" % bi.PAGE_SIZE, text)
    assert re.search(r"#define BI_SPLIT_KEYS %d\b" % bi.SPLIT_KEYS, text)


def test_build_flavour(lib):
    want = 0 if lib.path.endswith("libbi_variant.so") else 1
    assert lib.bi_build_invariant() == want


def test_status_strings(lib):
    for s in binding.Status:
        assert lib.bi_status_string(int(s))
    assert lib.bi_status_string(0) == "ok"


P = ctypes.c_void_p
FAKE = P(0x10000)  # a 16-byte aligned non-null value; never dereferenced


def test_rmsnorm_rejects_bad_sizes(lib):
    L = lib.lib
    assert L.bi_rmsnorm(FAKE, FAKE, FAKE, 4, 12, 1e-6, 0, None) == binding.Status.INVALID   # H % 8
    assert L.bi_rmsnorm(FAKE, FAKE, FAKE, -1, 64, 1e-6, 0, None) == binding.Status.INVALID
    assert L.bi_rmsnorm(FAKE, FAKE, FAKE, 4, 64, 1e-6, 7, None) == binding.Status.INVALID   # dtype
    assert L.bi_rmsnorm(FAKE, FAKE, FAKE, 4, 65544, 1e-6, 0, None) == binding.Status.INVALID
    assert L.bi_rmsnorm(FAKE, FAKE, FAKE, 4, 64, float("nan"), 0, None) == binding.Status.INVALID
    assert L.bi_rmsnorm(P(0x10008), FAKE, FAKE, 4, 64, 1e-6, 0, None) == binding.Status.INVALID
    assert L.bi_rmsnorm(None, FAKE, FAKE, 4, 64, 1e-6, 0, None) == binding.Status.INVALID
    assert L.bi_rmsnorm(None, None, None, 0, 64, 1e-6, 0, None) == binding.Status.OK  # M == 0


def test_matmul_rejects_bad_sizes(lib):
    L = lib.lib
    assert L.bi_matmul(FAKE, FAKE, FAKE, 4, 12, 64, 0, None, 0, None) == binding.Status.INVALID
    assert L.bi_matmul(FAKE, FAKE, FAKE, 4, 64, 12, 0, None, 0, None) == binding.Status.INVALID
    assert L.bi_matmul(FAKE, FAKE, FAKE, 4, 0, 64, 0, None, 0, None) == binding.Status.INVALID
    assert L.bi_matmul(None, FAKE, FAKE, 4, 64, 64, 0, None, 0, None) == binding.Status.INVALID
    assert L.bi_matmul(None, None, None, 0, 64, 64, 0, None, 0, None) == binding.Status.OK


def _kv(**over):
    f = dict(k_cache=0x10000, v_cache=0x20000, block_table=0x30000, max_pages_per_seq=4,
             num_pages=8, page_size=16, num_kv_heads=2, head_dim=128)
    f.update(over)
    return binding._PagedKV(**f)


def test_attention_rejects_bad_layouts(lib):
    L = lib.lib
    dec = lambda kv, Hq=4, B=1, mx=32: L.bi_attention_decode(  # noqa: E731
        ctypes.byref(kv), FAKE, FAKE, None, FAKE, B, Hq, mx, 0.1, 0, None, 0, None)
    assert dec(_kv(page_size=8)) == binding.Status.INVALID
    assert dec(_kv(), Hq=3) == binding.Status.INVALID               # Hq % Hkv
    assert dec(_kv(head_dim=96)) == binding.Status.UNSUPPORTED
    assert dec(_kv(k_cache=0x10004)) == binding.Status.INVALID       # alignment
    assert dec(_kv(), mx=65) == binding.Status.INVALID               # > max_pages * 16
    assert dec(_kv(), Hq=2 * 129) == binding.Status.INVALID          # group > 128
    assert dec(_kv(), B=0) == binding.Status.OK
    pre = lambda kv, Hq=4: L.bi_attention_prefill(  # noqa: E731
        ctypes.byref(kv), FAKE, FAKE, None, FAKE, FAKE, 1, Hq, 16, 16, 0.1, None, 0, None)
    assert pre(_kv(num_kv_heads=0)) == binding.Status.INVALID
    assert pre(_kv(head_dim=32)) == binding.Status.UNSUPPORTED
    assert L.bi_kv_write(ctypes.byref(_kv(page_size=32)), FAKE, FAKE, FAKE, 4, None) == \
        binding.Status.INVALID


def test_debug_wait_rejects_out_of_range_limits(lib):
    assert lib.lib.bi_debug_bounded_wait(10, None) == binding.Status.INVALID
    assert lib.lib.bi_debug_bounded_wait(10 ** 10, None) == binding.Status.INVALID


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        binding.Library(str(tmp_path / "libbi.so"))


def test_fused_matmuls_reject_bad_arguments(lib):
    L, INV, OK = lib.lib, binding.Status.INVALID, binding.Status.OK
    assert L.bi_fold_norm_weight(FAKE, FAKE, FAKE, 4, 12, None) == INV          # K % 8
    assert L.bi_fold_norm_weight(None, FAKE, FAKE, 4, 64, None) == INV
    assert L.bi_fold_norm_weight(None, None, None, 0, 64, None) == OK           # N == 0
    rm = lambda M=4, N=64, K=64, eps=1e-6, dt=0, ws=FAKE, nb=1024: L.bi_rmsnorm_matmul(  # noqa: E731
        FAKE, FAKE, FAKE, M, N, K, eps, dt, ws, nb, None)
    assert rm(N=12) == INV                 # N % 8
    assert rm(eps=-1.0) == INV
    assert rm(eps=float("inf")) == INV
    assert rm(dt=9) == INV
    assert rm(K=65544) == INV              # beyond the row reduction's limit
    assert rm(nb=8) == binding.Status.WORKSPACE
    assert rm(ws=None) == binding.Status.WORKSPACE
    assert L.bi_rmsnorm_matmul(None, None, None, 0, 64, 64, 1e-6, 0, None, 0, None) == OK  # M == 0
    assert L.bi_rmsnorm_matmul_workspace_bytes(5) == 256
    assert L.bi_matmul_residual(FAKE, FAKE, FAKE, FAKE, 4, 64, 12, None) == INV     # K % 8
    assert L.bi_matmul_residual(FAKE, FAKE, None, FAKE, 4, 64, 64, None) == INV     # no R
    assert L.bi_matmul_residual(None, None, None, None, 0, 64, 64, None) == OK


def test_qkv_epilogue_and_angle_table_reject_bad_arguments(lib):
    L, INV, OK = lib.lib, binding.Status.INVALID, binding.Status.OK
    assert L.bi_rope_table(FAKE, 0, 128, 10000.0, None) == INV                  # no positions
    assert L.bi_rope_table(FAKE, 16, 96, 10000.0, None) == INV                  # head_dim
    assert L.bi_rope_table(FAKE, 16, 128, 1.0, None) == INV                     # theta <= 1
    assert L.bi_rope_table(P(0x10004), 16, 128, 10000.0, None) == INV           # alignment
    call = lambda kv, Hq=4, T=3, K=64, ws=FAKE: L.bi_rmsnorm_matmul_rope_kv(  # noqa: E731
        FAKE, FAKE, 1e-6, ctypes.byref(kv), FAKE, 4096, FAKE, FAKE, FAKE, T, K, Hq, ws, 256, None)
    assert call(_kv(), ws=None) == binding.Status.WORKSPACE
    assert call(_kv(page_size=8)) == INV
    assert call(_kv(), Hq=3) == INV                                             # Hq % Hkv
    assert call(_kv(), K=12) == INV                                             # K % 8
    assert call(_kv(), T=0) == OK


def test_backward_passes_reject_bad_arguments(lib):
    L, INV, OK, WS = lib.lib, binding.Status.INVALID, binding.Status.OK, binding.Status.WORKSPACE
    bwd = lambda M=4, H=64, ws=FAKE, nb=1 << 20, eps=1e-6: L.bi_rmsnorm_backward(  # noqa: E731
        FAKE, FAKE, FAKE, FAKE, FAKE, M, H, eps, 0, ws, nb, None)
    assert bwd(H=12) == INV
    assert bwd(eps=float("nan")) == INV
    assert bwd(nb=0) == WS
    assert bwd(ws=None) == WS
    assert bwd(M=0) == OK
    assert L.bi_rmsnorm_backward_workspace_bytes(300, 64) >= 300 * 4 + 5 * 64 * 4
    assert L.bi_transpose(FAKE, FAKE, 8, 4, 7, None) == INV                     # ld_out < R
    assert L.bi_transpose(None, None, 0, 4, 0, None) == OK
    mb = lambda da=FAKE, dw=FAKE, M=4, nb=1 << 30: L.bi_matmul_backward(  # noqa: E731
        FAKE, FAKE, FAKE, da, dw, M, 64, 64, 0, FAKE, nb, None)
    assert mb(da=None, dw=None) == INV
    assert mb(nb=16) == WS
    assert mb(M=0) == OK
    # W^T, dC^T and A^T, each region rounded up to 256 bytes, rows padded to 8
    assert L.bi_matmul_backward_workspace_bytes(5, 64, 32) == 4096 + 1024 + 512


def test_swiglu_and_rope_backward_reject_bad_arguments(lib):
    L, INV, OK = lib.lib, binding.Status.INVALID, binding.Status.OK
    sw = lambda T=4, F=64, dt=0, p=FAKE: L.bi_swiglu_backward(p, FAKE, FAKE, T, F, dt, None)  # noqa: E731
    assert sw(F=12) == INV
    assert sw(F=0) == INV
    assert sw(T=-1) == INV
    assert sw(dt=5) == INV
    assert sw(p=P(0x10008)) == INV       # misaligned
    assert sw(T=0) == OK
    rb = lambda T=4, nh=2, d=128, ld=256, ldo=256, th=1e4, dt=0: L.bi_rope_backward(  # noqa: E731
        FAKE, ld, FAKE, FAKE, ldo, T, nh, d, th, dt, None)
    assert rb(d=96) == INV
    assert rb(nh=0) == INV
    assert rb(ld=255) == INV             # shorter than the heads it holds
    assert rb(ldo=260 - 2) == INV        # not a multiple of 8
    assert rb(th=1.0) == INV
    assert rb(th=float("inf")) == INV
    assert rb(dt=3) == INV
    assert rb(T=0) == OK


def test_attention_backward_rejects_bad_arguments(lib):
    import ctypes as C
    L, INV, OK, WS = lib.lib, binding.Status.INVALID, binding.Status.OK, binding.Status.WORKSPACE
    UNS = binding.Status.UNSUPPORTED

    def kv(d=128, heads=2, pages=8, mp=4):
        return binding._PagedKV(0x10000, 0x20000, 0x30000, mp, pages, 16, heads, d)

    def ab(k=None, Hq=8, B=2, T=10, mq=5, mkv=40, ws=FAKE, nb=1 << 20, dk=P(0x40000),
           dv=P(0x50000)):
        k = k or kv()
        return L.bi_attention_backward(C.byref(k), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, Hq, T,
                                       mq, mkv, 0.1, FAKE, dk, dv, ws, nb, None)
    assert ab(Hq=7) == INV                 # Hq % Hkv
    assert ab(k=kv(d=96)) == UNS
    assert ab(mkv=65) == INV               # beyond the page table (4 pages)
    assert ab(mq=50, mkv=40) == INV        # a chunk longer than its sequence
    assert ab(dk=P(0x10000)) == INV        # dk aliases the k cache
    assert ab(dk=P(0x50000)) == INV        # dk aliases dv
    assert ab(nb=8) == WS
    assert ab(ws=None) == WS
    assert ab(T=0) == OK
    assert ab(B=0) == OK
    assert L.bi_attention_backward_workspace_bytes(8, 10) == 2 * 8 * 10 * 4
