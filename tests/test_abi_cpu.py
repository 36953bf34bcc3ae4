"""The C-ABI library loads and exports what include/qsa.h declares; host-side
argument validation answers before anything touches a device (CPU only:
no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qsa.h")


@pytest.fixture(scope="module")
def capi():
    from top_sparse_attention_qsa_b200 import build
    build.build()
    from top_sparse_attention_qsa_b200 import _capi
    return _capi


@pytest.fixture(scope="module")
def dbg(capi):
    from top_sparse_attention_qsa_b200 import _debug
    return _debug


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert "qsa_sparse_prefill_fwd" in names
    assert "qsa_sparse_prefill_debug_gather" in names


def test_library_exports_every_declared_symbol(capi):
    lib = capi.library()
    for name in declared_functions():
        assert hasattr(lib, name), f"libqsa.so does not export {name}"
    assert sorted(capi.EXPORTS) == declared_functions()


def test_library_is_sm100a_only_and_static_runtime(capi):
    # the build flags the driver checks: one sm_100a target, static cudart
    from top_sparse_attention_qsa_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


def test_abi_version_and_status_strings(capi):
    m = re.search(r"#define QSA_ABI_VERSION (\d+)", open(HEADER).read())
    assert capi.abi_version() == int(m.group(1))
    for code in range(6):
        assert capi.status_string(code)
    assert capi.status_string(99) == "unknown status"


def _shape(capi, **kw):
    base = dict(num_tokens=4, num_q_heads=12, num_kv_heads=1, head_dim=256, topk=8,
                num_slots=64, q_stride_tok=12 * 256, q_stride_head=256, kv_stride_slot=256,
                kv_stride_head=256, idx_stride_tok=8, idx_stride_head=8, o_stride_tok=12 * 256,
                o_stride_head=256, lse_stride_tok=12)
    base.update(kw)
    return capi.Shape(**base)


# Fake, 16-byte-aligned addresses: every case below is rejected by the host
# checks before any CUDA call, so nothing is ever dereferenced.
P = 0x10000


def _fwd(capi, shape, q=P, k=P, v=P, idx=P, out=P, lse=None, nv=None):
    return capi.library().qsa_sparse_prefill_fwd(ctypes.byref(shape) if shape is not None else None,
                                                 q, k, v, idx, nv, 0.0, out, lse, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=128), 3),
    (dict(num_q_heads=34, num_kv_heads=2), 3),      # G = 17
    (dict(num_q_heads=7, num_kv_heads=2), 2),       # Hq % Hkv != 0
    (dict(num_tokens=-1), 2),
    (dict(topk=-3), 2),
    (dict(q_stride_head=260), 4),                   # rows not 16-byte aligned
    (dict(kv_stride_slot=-256), 2),
    (dict(kv_stride_slot=0), 2),
])
def test_shape_validation(capi, kw, code):
    assert _fwd(capi, _shape(capi, **kw)) == code


def test_null_and_alignment_checks(capi):
    s = _shape(capi)
    assert _fwd(capi, None) == 1
    assert _fwd(capi, s, q=None) == 1
    assert _fwd(capi, s, idx=None) == 1
    assert _fwd(capi, s, out=P + 8) == 4
    assert _fwd(capi, s, k=P + 2) == 4
    # with K == 0 the caches and lists are never read: NULL is fine there,
    # and T == 0 is a no-op that returns before any CUDA call
    assert _fwd(capi, _shape(capi, num_tokens=0), q=None, out=None) == 0
    lib = capi.library()
    assert lib.qsa_sparse_prefill_debug_gather(ctypes.byref(s), P, P, P, P, None, 0.0, P, None,
                                               None, None, None) == 1


def test_binding_rejects_host_tensors(capi):
    q = torch.zeros(2, 3, 256, dtype=torch.bfloat16)
    k = torch.zeros(8, 1, 256, dtype=torch.bfloat16)
    idx = torch.zeros(2, 1, 4, dtype=torch.int32)
    with pytest.raises(ValueError):
        capi.sparse_prefill_fwd(q, k, k, idx)
    with pytest.raises(TypeError):
        capi.sparse_prefill_fwd(q.float(), k, k, idx)


def test_stall_hook_needs_a_status_word(dbg, capi):
    s = _shape(capi)
    assert dbg.library().qsa_test_stalled_pipeline(ctypes.byref(s), P, P, P, P, None, 0.0, P, None,
                                                   None, None) == 1


def _ishape(capi, **kw):
    base = dict(num_tokens=4, num_heads=4, head_dim=128, num_blocks=64, block_size=4, reserved=0,
                q_stride_tok=512, q_stride_head=128, k_stride_block=128, score_stride_tok=64)
    base.update(kw)
    return capi.IndexerShape(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), 3),
    (dict(num_heads=3), 3),
    (dict(num_heads=16), 3),
    (dict(num_blocks=0), 2),
    (dict(block_size=0), 2),
    (dict(score_stride_tok=63), 2),
    (dict(q_stride_head=132), 4),
    (dict(k_stride_block=-128), 2),
])
def test_indexer_validation(capi, kw, code):
    lib = capi.library()
    assert lib.qsa_indexer_scores(ctypes.byref(_ishape(capi, **kw)), P, P, P, P, P, None, None) == code


def test_indexer_nulls_and_topk_limits(capi):
    lib = capi.library()
    s = _ishape(capi)
    assert lib.qsa_indexer_scores(None, P, P, P, P, P, None, None) == 1
    assert lib.qsa_indexer_scores(ctypes.byref(s), None, P, P, P, P, None, None) == 1
    assert lib.qsa_indexer_scores(ctypes.byref(s), P + 8, P, P, P, P, None, None) == 4
    assert lib.qsa_indexer_scores(ctypes.byref(_ishape(capi, num_tokens=0)), None, None, None, None, None,
                                  None, None) == 0
    # selection: rows longer than 32768 candidates are refused, widths checked
    big = _ishape(capi, num_blocks=32769, score_stride_tok=32772)
    sel = lib.qsa_topk_select
    assert sel(ctypes.byref(big), P, P, P, 8, 1, P, 9, P, 1, None, None) == 3
    assert sel(ctypes.byref(s), P, P, P, 8, 1, P, 8, P, 1, None, None) == 2   # stride < width
    assert sel(ctypes.byref(s), P, P, P, -1, 0, P, 8, P, 1, None, None) == 2
    assert sel(ctypes.byref(s), P, P, P, 8, 0, P, 8, P, 33, None, None) == 2  # copies
    assert sel(ctypes.byref(s), None, P, P, 8, 0, P, 8, P, 1, None, None) == 1
    assert sel(ctypes.byref(s), P + 4, P, P, 8, 0, P, 8, P, 1, None, None) == 4  # scores not 16-byte aligned
    odd = _ishape(capi, score_stride_tok=66)
    assert sel(ctypes.byref(odd), P, P, P, 8, 0, P, 8, P, 1, None, None) == 4   # row stride not 4 floats


def test_indexer_fold_validation(capi):
    lib = capi.library()
    fold = lib.qsa_indexer_fold_heads
    s = _ishape(capi)
    assert fold(None, P, P, None) == 1
    assert fold(ctypes.byref(s), None, P, None) == 1
    assert fold(ctypes.byref(s), P, None, None) == 1
    assert fold(ctypes.byref(s), P + 8, P, None) == 4            # q not 16-byte aligned
    assert fold(ctypes.byref(s), P, P + 8, None) == 4            # output not 16-byte aligned
    assert fold(ctypes.byref(_ishape(capi, q_stride_head=132)), P, P, None) == 4
    assert fold(ctypes.byref(_ishape(capi, num_heads=3)), P, P, None) == 3
    assert fold(ctypes.byref(_ishape(capi, head_dim=64)), P, P, None) == 3
    assert fold(ctypes.byref(_ishape(capi, num_tokens=0)), None, None, None) == 0


def test_fp8_entry_validation(capi):
    lib = capi.library()
    s = _shape(capi)
    fp8 = lib.qsa_sparse_prefill_fp8_fwd
    # kv strides must be multiples of 16 elements (bytes) for 16-byte copies
    odd = _shape(capi, kv_stride_slot=264, kv_stride_head=264)
    assert fp8(ctypes.byref(odd), 1, None, P, P, P, P, None, 0.0, 1.0, 1.0, P, None, None, None) == 4
    assert fp8(ctypes.byref(s), 3, None, P, P, P, P, None, 0.0, 1.0, 1.0, P, None, None, None) == 3
    assert fp8(ctypes.byref(s), 1, None, None, P, P, P, None, 0.0, 1.0, 1.0, P, None, None, None) == 1
    assert fp8(ctypes.byref(_shape(capi, head_dim=128)), 1, None, P, P, P, P, None, 0.0, 1.0, 1.0, P,
               None, None, None) == 3


def test_kernel_choice_validation(capi):
    """Kernel choices outside the enum are refused before anything is
    enqueued; the production library has no measurement-only choice."""
    lib = capi.library()
    s = _shape(capi)
    fwd_with = lib.qsa_sparse_prefill_fwd_with
    assert fwd_with(ctypes.byref(s), P, P, P, P, None, 0.0, P, None, None, 7, None) == 3
    assert fwd_with(ctypes.byref(s), P, P, P, P, None, 0.0, P, None, None, 3, None) == 3
    assert "KERNEL_GATHER_ONLY" not in open(HEADER).read()


def test_debug_gather_lists_validation(capi):
    lib = capi.library()
    s = _shape(capi)
    dl = lib.qsa_sparse_prefill_debug_gather_lists
    args = (P, P, P, P, None, 0.0, 1.0, 1.0, P, None, None)
    assert dl(ctypes.byref(s), 1, None, 0, *args, None, None) == 1          # no dump buffer
    assert dl(ctypes.byref(s), 3, None, 0, *args, P, None) == 3             # block size 3
    odd = _shape(capi, kv_stride_slot=264, kv_stride_head=264)
    assert dl(ctypes.byref(odd), 1, None, 1, *args, P, None) == 4           # FP8 strides
    assert dl(ctypes.byref(s), 1, None, 0, *args, P + 2, None) == 4         # dump not 4-byte aligned


# --- the debug library (measurement kernels, test hooks) ----------------------

DEBUG_HEADER = os.path.join(ROOT, "include", "qsa_debug.h")


def declared_debug_functions():
    src = re.sub(r"/\*.*?\*/", "", open(DEBUG_HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", src)))


def test_debug_library_exports_and_production_does_not(dbg, capi):
    names = declared_debug_functions()
    assert sorted(dbg.EXPORTS) == names
    for name in names:
        assert hasattr(dbg.library(), name), f"libqsa_debug.so does not export {name}"
        assert name not in capi.EXPORTS
        # the production library carries no test hook or measurement kernel
        with pytest.raises(AttributeError):
            getattr(ctypes.CDLL(capi.LIB_PATH), name)
    m = re.search(r"#define QSA_DEBUG_ABI_VERSION (\d+)", open(DEBUG_HEADER).read())
    assert dbg.abi_version() == int(m.group(1))


def test_debug_gather_only_validation(dbg, capi):
    lib = dbg.library()
    s = _shape(capi)
    assert lib.qsa_debug_gather_only(None, 0, P, P, P, P, None, None, None) == 1
    odd = _shape(capi, kv_stride_slot=264, kv_stride_head=264)
    assert lib.qsa_debug_gather_only(ctypes.byref(odd), 1, P, P, P, P, None, None, None) == 4
    assert lib.qsa_debug_gather_only(ctypes.byref(_shape(capi, head_dim=128)), 0, P, P, P, P, None, None,
                                     None) == 3


@pytest.mark.parametrize("args,code", [
    # table, rows, stride, row_bytes, ids, n_ids, method, depth, warps, ctas, sink, sink_words
    ((None, 64, 512, 512, P, 64, 0, 4, 8, 1, None, 0), 1),
    ((P, 64, 512, 384, P, 64, 0, 4, 8, 1, None, 0), 3),      # row bytes
    ((P, 64, 512, 512, P, 64, 0, 3, 8, 1, None, 0), 3),      # cp.async depth 3
    ((P, 64, 512, 512, P, 64, 0, 16, 2, 1, None, 0), 3),     # cp.async depth 16
    ((P, 64, 512, 512, P, 64, 1, 2, 8, 1, None, 0), 3),      # ld.v4 depth 2
    ((P, 64, 512, 512, P, 64, 2, 5, 8, 1, None, 0), 3),      # bulk depth 5
    ((P, 64, 512, 512, P, 64, 9, 4, 8, 1, None, 0), 3),      # method
    ((P, 64, 504, 512, P, 64, 0, 4, 8, 1, None, 0), 2),      # stride < row
    ((P, 64, 520, 512, P, 64, 0, 4, 8, 1, None, 0), 2),      # stride not 16-byte
    ((P, 0, 512, 512, P, 64, 0, 4, 8, 1, None, 0), 2),       # no rows
    ((P, 64, 512, 512, P, 64, 0, 4, 33, 1, None, 0), 2),     # warps
    ((P + 8, 64, 512, 512, P, 64, 0, 4, 8, 1, None, 0), 4),  # table alignment
])
def test_debug_gather_peak_validation(dbg, args, code):
    assert dbg.library().qsa_debug_gather_peak(*args, None, None) == code
