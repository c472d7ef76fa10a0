"""CPU tests of the C ABI: the library loads, exports every symbol that
include/lq.h declares, and rejects bad arguments with status codes before it
touches the GPU.  No call here launches a kernel."""

import ctypes
import os
import re

import pytest

from quantized_linear_gemm_b200 import lq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lq.h")

OK, INVALID, ALIGN, SHAPE, TABLE = 0, 1, 2, 3, 7
FAKE = 0x10000          # 16-byte aligned non-null "device pointer"; never dereferenced
MISALIGNED = 0x10008


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_what_binding_lists():
    assert declared_functions() == sorted(lq.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = lq.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_version_and_status_strings():
    assert lq.version().startswith("lq ")
    for code, name in lq.STATUS.items():
        assert lq.status_string(code) == name


def _mm(fmt=0, A=FAKE, a_s=FAKE, B=FAKE, b_s=FAKE, C=FAKE, M=16, N=128, K=128, variant=None):
    return lq.lib().lq_scaled_mm(fmt, A, a_s, B, b_s, C, M, N, K,
                                 ctypes.byref(variant) if variant is not None else None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(fmt=4), INVALID), (dict(fmt=-1), INVALID),
    (dict(A=None), INVALID), (dict(B=None), INVALID), (dict(C=None), INVALID),
    (dict(a_s=None), INVALID), (dict(b_s=None), INVALID),
    (dict(M=-1), INVALID), (dict(K=-16), INVALID),
    (dict(A=MISALIGNED), ALIGN), (dict(B=MISALIGNED), ALIGN), (dict(C=MISALIGNED), ALIGN),
    (dict(K=120), SHAPE), (dict(N=100), SHAPE),
    (dict(fmt=2, K=192), SHAPE), (dict(fmt=2, N=192), SHAPE),
    (dict(fmt=3, K=192), SHAPE), (dict(fmt=3, N=192), SHAPE), (dict(fmt=3, a_s=None), INVALID),
])
def test_scaled_mm_argument_checks(kw, code):
    assert _mm(**kw) == code


def test_int8_depth_bound():
    """W8A8_INT8 sums int8 products in int32: K up to 131071 cannot wrap
    (131071 * 128 * 128 < 2^31); deeper K is refused before any launch."""
    assert _mm(fmt=1, K=131072) == SHAPE
    assert _mm(fmt=1, K=131072 + 16) == SHAPE
    assert 131071 * 128 * 128 < 2 ** 31 <= 131072 * 128 * 128
    # the other formats accumulate in fp32 and take any K
    assert _mm(fmt=0, K=131072, M=0) == OK
    v = lq.make_variant(swap_ab=1, split_k=2, tile_n=32)
    rc = lq.lib().lq_grouped_scaled_mm(1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 16, 128, 131072,
                                       ctypes.byref(v), None)
    assert rc == SHAPE
    rc = lq.lib().lq_quant_scaled_mm(1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 128, 131072, None, None)
    assert rc == SHAPE


def test_default_variant_waits_before_reading_weights():
    """A NULL variant lowers the table's pdl 2 (weights streamed before the
    dependency wait) to 1 until the caller declares static weights."""
    prev = lq.declare_static_weights(False)
    try:
        shapes = [(1, 6144, 4096), (8, 4096, 4096), (32, 24576, 4096), (16, 4096, 12288)]
        for fmt in (0, 1, 2):
            for M, N, K in shapes:
                assert lq.select_variant(fmt, M, N, K).pdl <= 1
        assert lq.declare_static_weights(True) is False
        assert any(lq.select_variant(0, M, N, K).pdl == 2 for M, N, K in shapes)
        assert lq.declare_static_weights(False) is True
        assert all(lq.select_variant(0, M, N, K).pdl <= 1 for M, N, K in shapes)
    finally:
        lq.declare_static_weights(prev)


def test_quant_scaled_mm_checks_the_variant_before_launching():
    """The two-kernel path checks the caller's variant before it launches the
    quantization kernel: an invalid one launches nothing."""
    v = lq.make_variant(swap_ab=1, split_k=3, tile_n=16, reduce=2)   # split 3: not with the cluster reduction
    assert lq.lib().lq_quant_scaled_mm(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 128, 1024,
                                       ctypes.byref(v), None) == INVALID


def test_empty_problem_is_a_noop():
    # M == 0 or N == 0: nothing to do, no pointer is needed
    assert _mm(M=0, A=None, B=None, C=None, a_s=None, b_s=None) == OK
    assert _mm(N=0, A=None, B=None, C=None, a_s=None, b_s=None) == OK


@pytest.mark.parametrize("field,value", [
    ("split_k", 3), ("split_k", 512), ("split_k", 257), ("split_k", 0), ("split_k", -4), ("swap_ab", 2),
    ("tile_n", 48), ("stages", 1), ("stages", 15), ("reduce", 3), ("pdl", 5),
])
def test_variant_checks(field, value):
    v = lq.make_variant(swap_ab=1, split_k=2, tile_n=32, reduce=2)   # split 3: not with the cluster reduction
    setattr(v, field, value)
    assert _mm(variant=v) == INVALID


def test_explicit_variant_is_checked_before_the_pointers():
    """So that a valid variant with a misaligned C reports the pointer
    (LQ_ERR_ALIGNMENT: the variant was accepted) and an invalid one reports
    the variant whatever the pointers; the same for the allocation-free
    entry point, which applies its own reduction first."""
    bad = lq.make_variant(swap_ab=1, split_k=3, tile_n=16, reduce=2)
    good = lq.make_variant(swap_ab=1, split_k=3, tile_n=16, reduce=1)
    assert _mm(variant=bad, C=MISALIGNED) == INVALID
    assert _mm(variant=good, C=MISALIGNED) == ALIGN
    assert _mm(variant=bad, A=None) == INVALID
    f = lq.lib().lq_scaled_mm_noalloc
    assert f(0, FAKE, FAKE, FAKE, FAKE, MISALIGNED, 16, 128, 128, ctypes.byref(bad), None) == ALIGN   # reduce 0 there
    worse = lq.make_variant(swap_ab=1, split_k=2, tile_n=48)
    assert f(0, FAKE, FAKE, FAKE, FAKE, MISALIGNED, 16, 128, 128, ctypes.byref(worse), None) == INVALID


def test_split_counts_by_reduction():
    """Any split count 1..256 with the workspace reductions (0, 1); powers of
    two (at most 16) with the cluster reduction."""
    for S in (3, 5, 7, 12, 100, 256):
        for reduce in (0, 1):
            for sw, tn in ((1, 16), (0, 128)):
                v = lq.make_variant(swap_ab=sw, split_k=S, tile_n=tn, reduce=reduce)
                assert _mm(variant=v, C=MISALIGNED) == ALIGN, (S, reduce, sw)
        assert _mm(variant=lq.make_variant(swap_ab=1, split_k=S, tile_n=16, reduce=2)) == INVALID, S


def test_persistent_variant_rules():
    """persistent = 1 (one-SM tiles), 2 (CTA pairs) and 3 (stream-K; both
    tile_n 128 / 256) need the Standard orientation and FP8 / INT8; one
    split, except CTA pairs, which take any split count with reduce 0."""
    for pers in (1, 2, 3):
        ok = lq.make_variant(swap_ab=0, tile_n=256, split_k=1, persistent=pers)
        assert _mm(variant=ok, C=MISALIGNED) == ALIGN    # accepted up to the pointer checks
    for S in (2, 3, 5, 7, 256):
        ok = lq.make_variant(swap_ab=0, tile_n=256, split_k=S, reduce=0, persistent=2)
        assert _mm(variant=ok, C=MISALIGNED) == ALIGN, S
    for bad in (dict(swap_ab=0, tile_n=256, split_k=2, reduce=1, persistent=2),
                dict(swap_ab=0, tile_n=256, split_k=2, reduce=2, persistent=2),
                dict(swap_ab=0, tile_n=256, split_k=257, reduce=0, persistent=2),
                dict(swap_ab=0, tile_n=256, split_k=3, reduce=0, persistent=1),
                dict(swap_ab=0, tile_n=256, split_k=3, reduce=2, persistent=0),
                dict(swap_ab=1, tile_n=16, persistent=1), dict(swap_ab=0, tile_n=128, split_k=2, persistent=1),
                dict(swap_ab=0, tile_n=128, persistent=4), dict(swap_ab=0, tile_n=256, stages=5, persistent=1),
                dict(swap_ab=0, tile_n=64, persistent=2), dict(swap_ab=1, tile_n=32, persistent=2),
                dict(swap_ab=0, tile_n=64, persistent=3), dict(swap_ab=0, tile_n=256, split_k=2, persistent=3)):
        assert _mm(variant=lq.make_variant(**bad)) == INVALID, bad
    for fmt in (2, 3):
        assert _mm(fmt=fmt, K=256, N=256, variant=lq.make_variant(swap_ab=0, tile_n=128, persistent=1)) == INVALID
        # Block_FP8 (fp32 or UE8M0 scales) on CTA pairs: 256 x 128 tiles only
        ok = lq.make_variant(swap_ab=0, tile_n=128, persistent=2)
        assert _mm(fmt=fmt, K=256, N=256, variant=ok, C=MISALIGNED) == ALIGN
        assert _mm(fmt=fmt, K=256, N=256, variant=lq.make_variant(swap_ab=0, tile_n=256, persistent=2)) == INVALID


def test_variant_tile_rules():
    assert _mm(variant=lq.make_variant(swap_ab=1, tile_n=128)) == INVALID      # swap tiles are 16/32/64
    assert _mm(variant=lq.make_variant(swap_ab=0, tile_n=16)) == INVALID       # standard tiles are 64/128/256
    assert _mm(fmt=2, variant=lq.make_variant(swap_ab=0, tile_n=256)) == INVALID
    assert _mm(variant=lq.make_variant(swap_ab=0, tile_n=256, stages=5)) == INVALID   # > 227 KB smem


def test_quant_argument_checks():
    L = lq.lib()
    assert L.lq_quant_per_token(2, FAKE, FAKE, FAKE, 4, 128, None) == INVALID    # block fmt not per-token
    assert L.lq_quant_per_token(0, None, FAKE, FAKE, 4, 128, None) == INVALID
    assert L.lq_quant_per_token(0, MISALIGNED, FAKE, FAKE, 4, 128, None) == ALIGN
    assert L.lq_quant_per_token(0, FAKE, FAKE, FAKE, 4, 120, None) == SHAPE
    assert L.lq_quant_per_token(0, FAKE, FAKE, FAKE, 0, 128, None) == OK
    assert L.lq_quant_per_token_group128(FAKE, FAKE, FAKE, 4, 192, None) == SHAPE
    assert L.lq_quant_per_token_group128(None, FAKE, FAKE, 4, 256, None) == INVALID
    assert L.lq_quant_weight_block128(FAKE, FAKE, FAKE, 192, 256, None) == SHAPE
    assert L.lq_quant_weight_block128(FAKE, FAKE, FAKE, 0, 256, None) == OK


def test_quant_scaled_mm_argument_checks():
    L = lq.lib()
    assert L.lq_quant_scaled_mm(2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 128, None, None) == INVALID  # block
    assert L.lq_quant_scaled_mm(0, None, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 128, None, None) == INVALID
    assert L.lq_quant_scaled_mm(0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 128, 128, None, None) == INVALID
    assert L.lq_quant_scaled_mm(0, MISALIGNED, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 128, None, None) == ALIGN
    assert L.lq_quant_scaled_mm(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 100, 128, None, None) == SHAPE
    assert L.lq_quant_scaled_mm(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 128, 128, None, None) == OK


def test_producer_quant_argument_checks():
    L = lq.lib()
    rms = L.lq_rms_norm_dynamic_per_token_quant
    assert rms(2, FAKE, None, FAKE, 1e-6, FAKE, FAKE, 4, 128, None) == INVALID          # block fmt
    assert rms(0, None, None, FAKE, 1e-6, FAKE, FAKE, 4, 128, None) == INVALID
    assert rms(0, FAKE, None, None, 1e-6, FAKE, FAKE, 4, 128, None) == INVALID          # no weight
    assert rms(0, FAKE, None, FAKE, -1.0, FAKE, FAKE, 4, 128, None) == INVALID          # eps < 0
    assert rms(0, FAKE, None, FAKE, float("nan"), FAKE, FAKE, 4, 128, None) == INVALID
    assert rms(0, FAKE, None, FAKE, float("inf"), FAKE, FAKE, 4, 128, None) == INVALID
    assert rms(0, FAKE, MISALIGNED, FAKE, 1e-6, FAKE, FAKE, 4, 128, None) == ALIGN
    assert rms(0, FAKE, None, MISALIGNED, 1e-6, FAKE, FAKE, 4, 128, None) == ALIGN
    assert rms(0, FAKE, None, FAKE, 1e-6, FAKE, FAKE, 4, 120, None) == SHAPE
    assert rms(0, FAKE, None, FAKE, 1e-6, FAKE, FAKE, 4, 0, None) == SHAPE
    assert rms(0, FAKE, None, FAKE, 1e-6, FAKE, FAKE, 4, 32768 + 16, None) == SHAPE      # longest row: 32768
    assert rms(0, FAKE, None, FAKE, 1e-6, FAKE, FAKE, -1, 128, None) == INVALID
    assert rms(0, FAKE, None, FAKE, 1e-6, FAKE, FAKE, 0, 128, None) == OK
    blk = L.lq_rms_norm_per_block_quant
    assert blk(FAKE, None, FAKE, 1e-6, FAKE, FAKE, 4, 192, None) == SHAPE
    assert blk(FAKE, None, FAKE, 1e-6, None, FAKE, 4, 256, None) == INVALID
    assert blk(FAKE, None, FAKE, 1e-6, FAKE, FAKE, 0, 256, None) == OK
    silu = L.lq_silu_and_mul_dynamic_per_token_quant
    assert silu(2, FAKE, FAKE, FAKE, 4, 128, None) == INVALID
    assert silu(1, MISALIGNED, FAKE, FAKE, 4, 128, None) == ALIGN
    assert silu(1, FAKE, FAKE, FAKE, 4, 24, None) == SHAPE
    assert silu(1, FAKE, FAKE, FAKE, 4, 65536, None) == SHAPE
    assert silu(1, FAKE, FAKE, FAKE, 0, 128, None) == OK
    sblk = L.lq_silu_and_mul_per_block_quant
    assert sblk(FAKE, FAKE, FAKE, 4, 64, None) == SHAPE
    assert sblk(FAKE, FAKE, None, 4, 128, None) == INVALID
    assert sblk(FAKE, FAKE, FAKE, 0, 128, None) == OK


def test_grouped_argument_checks():
    L = lq.lib()
    g = L.lq_grouped_scaled_mm
    v_std = lq.make_variant(swap_ab=0, tile_n=128)
    assert g(2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 256, 128, None, None) == INVALID      # Block_FP8
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 256, 128, None, None) == INVALID      # tokens, no expert
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 64, 256, 128, None, None) == INVALID      # no offsets
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 256, 128, ctypes.byref(v_std), None) == INVALID
    assert g(0, FAKE, FAKE, FAKE, FAKE, MISALIGNED, FAKE, 4, 64, 256, 128, None, None) == ALIGN
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, 64, 256, 128, None, None) == ALIGN
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 256, 120, None, None) == SHAPE        # K % 16
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 252, 128, None, None) == SHAPE        # N % 8
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 70000, 2000000, 256, 128, None, None) == SHAPE   # grid y
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0, 256, 128, None, None) == OK
    assert g(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, 64, 256, 128, None, None) == INVALID


def test_ue8m0_quant_argument_checks():
    L = lq.lib()
    assert L.lq_quant_per_token_group128_ue8m0(FAKE, FAKE, FAKE, 4, 192, None) == SHAPE
    assert L.lq_quant_per_token_group128_ue8m0(None, FAKE, FAKE, 4, 256, None) == INVALID
    assert L.lq_quant_per_token_group128_ue8m0(MISALIGNED, FAKE, FAKE, 4, 256, None) == ALIGN
    assert L.lq_quant_per_token_group128_ue8m0(FAKE, FAKE, FAKE + 1, 0, 256, None) == OK     # bytes: any alignment
    assert L.lq_quant_weight_block128_ue8m0(FAKE, FAKE, FAKE, 192, 256, None) == SHAPE
    assert L.lq_quant_weight_block128_ue8m0(FAKE, FAKE, None, 128, 256, None) == INVALID
    assert L.lq_quant_weight_block128_ue8m0(FAKE, FAKE, FAKE, 0, 256, None) == OK
    # UE8M0 scales are bytes: an odd scale address passes the checks (M = 0 stops before any launch)
    assert _mm(fmt=3, a_s=FAKE + 1, b_s=FAKE + 3, M=0) == OK


def test_bias_argument_checks():
    L = lq.lib()
    b = L.lq_scaled_mm_bias
    assert b(0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16, 128, 128, None, None) == INVALID     # no bias
    assert b(0, FAKE, FAKE, FAKE, FAKE, FAKE + 1, FAKE, 16, 128, 128, None, None) == ALIGN  # odd bias address
    assert b(0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 128, 0, None, None) == SHAPE        # K = 0
    assert b(4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 128, 128, None, None) == INVALID    # format
    assert b(0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 0, 128, 128, None, None) == OK          # M = 0


def test_stall_hook_argument_check():
    assert lq.lib().lq_test_inject_stall(-2, 0) == INVALID
    assert lq.lib().lq_test_inject_stall(-1, 0) == OK


def test_silu_hook_argument_check():
    f = lq.lib().lq_test_silu_bf16
    assert f(FAKE, FAKE, -1, None) == INVALID
    assert f(None, None, 0, None) == OK
    assert f(None, FAKE, 8, None) == INVALID
    assert f(FAKE + 1, FAKE, 8, None) == ALIGN


def test_i32acc_needs_an_output():
    L = lq.lib()
    assert L.lq_scaled_mm_i32acc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 128, 128, None, None) == INVALID
    assert L.lq_scaled_mm_i32acc(FAKE, FAKE, FAKE, FAKE, FAKE, MISALIGNED, 4, 128, 128, None, None) == ALIGN


def test_heuristic_variant_shapes(tmp_path):
    empty = tmp_path / "empty.txt"
    empty.write_text("# no entries: every lookup falls back to the heuristic\n")
    lq.load_dispatch_table(str(empty))
    try:
        _check_heuristic()
    finally:
        lq.load_dispatch_table(None)


def _check_heuristic():
    v = lq.select_variant("fp8_dynamic", 1, 4096, 4096)
    assert v.swap_ab == 1 and v.tile_n == 16 and v.split_k >= 2
    v = lq.select_variant("fp8_dynamic", 24, 4096, 4096)
    assert v.swap_ab == 1 and v.tile_n == 32
    v = lq.select_variant("w8a8_int8", 8192, 5120, 25600)
    assert v.swap_ab == 0 and v.tile_n == 256 and v.split_k == 1
    v = lq.select_variant("block_fp8", 2048, 51200, 5120)
    assert v.swap_ab == 0 and v.tile_n == 128
    for M in (1, 2, 3, 17, 33, 64, 100, 4096):
        v = lq.select_variant("block_fp8", M, 5120, 25600)
        assert v.split_k & (v.split_k - 1) == 0 and 1 <= v.split_k <= 256


def test_dispatch_table_file(tmp_path):
    p = tmp_path / "table.txt"
    p.write_text("# fmt m_bucket N K swap split tile stages reduce pdl\n"
                 "fp8_dynamic 8 4096 4096 1 8 16 4 0 1\n"
                 "w8a8_int8 32 6144 4096 0 2 64 6 1 0   # trailing comment\n"
                 "fp8_dynamic 2048 51200 5120 0 1 256 4 1 2 1   # 11th column: persistent\n")
    try:
        lq.load_dispatch_table(str(p))
        assert lq.dispatch_table_size() == 3
        v = lq.select_variant("fp8_dynamic", 5, 4096, 4096)      # M=5 -> bucket 8
        assert v.as_dict() == dict(swap_ab=1, split_k=8, tile_n=16, stages=4, reduce=0, pdl=1, persistent=0)
        v = lq.select_variant("w8a8_int8", 32, 6144, 4096)
        assert v.as_dict() == dict(swap_ab=0, split_k=2, tile_n=64, stages=6, reduce=1, pdl=0, persistent=0)
        v = lq.select_variant("fp8_dynamic", 2048, 51200, 5120)
        assert v.as_dict() == dict(swap_ab=0, split_k=1, tile_n=256, stages=4, reduce=1, pdl=1, persistent=1)
        # workspace need follows the selected variant
        assert lq.workspace_bytes("fp8_dynamic", 5, 4096, 4096) == 8 * 5 * 4096 * 4
        bad = tmp_path / "bad.txt"
        bad.write_text("fp8_dynamic 8 4096 4096 1 3 16 4 2 1\n")   # split_k 3 with the cluster reduction
        with pytest.raises(lq.LQError) as e:
            lq.load_dispatch_table(str(bad))
        assert e.value.code == TABLE
        assert lq.dispatch_table_size() == 3                       # the table in force is kept
        with pytest.raises(lq.LQError):
            lq.load_dispatch_table(str(tmp_path / "missing.txt"))
    finally:
        lq.load_dispatch_table(None)


def test_token_buckets(tmp_path):
    """M rounds up to the next tuned decode size (1,2,4,8,16,24,32), then to powers of two."""
    buckets = (1, 2, 4, 8, 16, 24, 32, 64, 128)
    p = tmp_path / "buckets.txt"
    p.write_text("".join(f"fp8_dynamic {mb} 4096 4096 1 2 16 {2 + i} 1 1\n" for i, mb in enumerate(buckets)))
    try:
        lq.load_dispatch_table(str(p))
        for M, mb in [(1, 1), (2, 2), (3, 4), (5, 8), (9, 16), (17, 24), (25, 32), (33, 64), (65, 128)]:
            assert lq.select_variant("fp8_dynamic", M, 4096, 4096).stages == 2 + buckets.index(mb), M
    finally:
        lq.load_dispatch_table(None)


def test_fuse_limit_hook():
    """lq_set_fuse_limit returns the limit in force and restores the default."""
    default = lq.set_fuse_limit(-1)
    assert default == 0 or os.environ.get("LQ_FUSE_MAX_SLICE_BYTES")
    assert lq.set_fuse_limit(0) == default
    assert lq.set_fuse_limit(4096) == 0
    assert lq.set_fuse_limit(-1) == 4096
    assert lq.set_fuse_limit(-1) == default
