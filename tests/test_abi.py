"""The C ABI without a GPU: the library builds for sm_100a, loads, exports every entry point
include/fa_b200.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build_module():
    import importlib.util
    path = os.path.join(ROOT, "block_sparse_masked_x128_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_fa_b200_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def fa():
    _build_module().build()
    import block_sparse_masked_x128_b200 as fa
    return fa


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "fa_b200.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("fa_create_block_mask", "fa_forward", "fa_block_mask_get", "fa_get_device_status",
              "fa_destroy_block_mask", "fa_status_string", "fa_last_error_message"):
        assert n in names


def test_library_exports_every_declared_symbol(fa):
    lib = ctypes.CDLL(fa.library_path())
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(fa.EXPORTED) <= set(_declared_functions())


def test_library_is_built_for_sm100a_only():
    assert _build_module().ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings(fa):
    for code, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID_ARG"), (2, "FA_ERR_UNSUPPORTED"),
                       (3, "FA_ERR_CUDA"), (4, "FA_ERR_OOM"), (5, "FA_ERR_TIMEOUT"),
                       (6, "FA_ERR_INTERNAL")]:
        assert fa.fa_status_string(code) == name


def _create(fa, kind, params, B=0, H=0, Q=256, KV=256, BS=128):
    h = ctypes.c_void_p()
    st = fa._lib.fa_create_block_mask(kind, ctypes.byref(params) if params is not None else None,
                                      B, H, Q, KV, BS, None, ctypes.byref(h))
    return st, h.value


def test_create_block_mask_rejects_bad_arguments(fa):
    P = fa.FaMaskParams
    assert fa._lib.fa_create_block_mask(1, None, 0, 0, 256, 256, 128, None, None) == fa.FA_ERR_INVALID_ARG
    assert _create(fa, 1, None, BS=0)[0] == fa.FA_ERR_INVALID_ARG      # block sizes are positive
    assert "block sizes" in fa.fa_last_error_message()
    assert _create(fa, 1, None, BS=1, Q=16385, KV=16385)[0] == fa.FA_ERR_UNSUPPORTED
    assert "blocks per side" in fa.fa_last_error_message()
    assert _create(fa, 8, None)[0] == fa.FA_ERR_INVALID_ARG          # unknown kind bit
    assert _create(fa, 2, P(0, None, 1))[0] == fa.FA_ERR_INVALID_ARG  # window must be > 0
    assert _create(fa, 2, None)[0] == fa.FA_ERR_INVALID_ARG          # window missing
    assert _create(fa, 4, P(0, None, 1))[0] == fa.FA_ERR_INVALID_ARG  # doc_id missing
    assert _create(fa, 4, P(0, 0x1000, 1), Q=256, KV=512)[0] == fa.FA_ERR_INVALID_ARG
    assert _create(fa, 1, None, Q=0)[0] == fa.FA_ERR_INVALID_ARG
    assert _create(fa, 1, None, B=-1)[0] == fa.FA_ERR_INVALID_ARG
    assert _create(fa, 1, None, Q=128 * 16385)[0] == fa.FA_ERR_UNSUPPORTED


def _t(fa, B=1, H=2, S=256, D=64, dtype=1, data=0x10000, stride=None):
    st = stride or (H * S * D, S * D, D, 1)
    return fa.FaTensor(data, dtype, B, H, S, D, (ctypes.c_int64 * 4)(*st))


def _fwd(fa, q, k, v, out, mask=None, kind=0, params=None, lse=None):
    return fa._lib.fa_forward(ctypes.byref(q) if q else None, ctypes.byref(k), ctypes.byref(v), mask,
                              kind, ctypes.byref(params) if params else None, -1.0,
                              ctypes.byref(out), lse, None)


def test_forward_rejects_bad_arguments(fa):
    q, k, v, o = (_t(fa) for _ in range(4))
    assert _fwd(fa, None, k, v, o) == fa.FA_ERR_INVALID_ARG
    assert _fwd(fa, _t(fa, data=0), k, v, o) == fa.FA_ERR_INVALID_ARG
    assert _fwd(fa, _t(fa, data=0x10008), k, v, o) == fa.FA_ERR_INVALID_ARG      # misaligned
    assert _fwd(fa, _t(fa, dtype=7), k, v, o) == fa.FA_ERR_INVALID_ARG
    assert _fwd(fa, _t(fa, stride=(256 * 64 * 2, 256 * 64, 64, 2)), k, v, o) == fa.FA_ERR_INVALID_ARG
    assert _fwd(fa, _t(fa, stride=(256 * 64 * 2, 256 * 64, 60, 1)), k, v, o) == fa.FA_ERR_INVALID_ARG
    assert _fwd(fa, q, _t(fa, dtype=0), v, o) == fa.FA_ERR_INVALID_ARG          # dtype mismatch
    assert _fwd(fa, q, _t(fa, H=3), v, o) == fa.FA_ERR_INVALID_ARG              # H mismatch
    assert _fwd(fa, q, k, _t(fa, S=384), o) == fa.FA_ERR_INVALID_ARG            # k/v length mismatch
    assert _fwd(fa, q, k, v, _t(fa, S=384)) == fa.FA_ERR_INVALID_ARG            # out length
    d96 = [_t(fa, D=96) for _ in range(4)]
    assert _fwd(fa, *d96) == fa.FA_ERR_UNSUPPORTED
    assert "head_dim" in fa.fa_last_error_message()
    r = [_t(fa, S=200) for _ in range(4)]           # ragged lengths pass the shape checks:
    assert _fwd(fa, *r) == fa.FA_ERR_INVALID_ARG      # what stops this call is the NULL mask
    assert "block_mask" in fa.fa_last_error_message()
    assert _fwd(fa, q, k, v, o, kind=4) == fa.FA_ERR_INVALID_ARG                # unknown score bit
    assert _fwd(fa, q, k, v, o, kind=1) == fa.FA_ERR_INVALID_ARG                # soft-cap without params
    assert _fwd(fa, q, k, v, o, kind=1, params=fa.FaScoreParams(0.0, None)) == fa.FA_ERR_INVALID_ARG
    assert _fwd(fa, q, k, v, o, lse=0x10002) == fa.FA_ERR_INVALID_ARG           # misaligned lse
    assert _fwd(fa, q, k, v, o) == fa.FA_ERR_INVALID_ARG                        # NULL mask
    assert "block_mask" in fa.fa_last_error_message()


def test_null_handles_are_rejected_or_ignored(fa):
    assert fa._lib.fa_get_device_status(None, None) == fa.FA_ERR_INVALID_ARG
    info = fa.FaBlockMaskInfo()
    assert fa._lib.fa_block_mask_get(None, ctypes.byref(info)) == fa.FA_ERR_INVALID_ARG
    fa._lib.fa_destroy_block_mask(None)


def test_python_binding_raises_fa_error(fa):
    with pytest.raises(fa.FaError) as ei:
        fa.fa_create_block_mask(1, None, 0, 0, 256, 256, BLOCK_SIZE=0, stream=0)
    assert ei.value.status == fa.FA_ERR_INVALID_ARG
    # Caller block lists must come in multiples of the kernels' 128 x 128 tiles.
    dummy = ctypes.c_void_p(0x1000)
    h = ctypes.c_void_p()
    st = fa._lib.fa_block_mask_from_kv_blocks(1, None, 0, 0, 256, 256, 64, 128, dummy, dummy, None,
                                              None, None, ctypes.byref(h))
    assert st == fa.FA_ERR_UNSUPPORTED


def _header_constants():
    text = open(os.path.join(ROOT, "include", "fa_b200.h")).read()
    consts = {n: int(v) for n, v in re.findall(r"#define\s+(FA_[A-Z0-9_]+)\s+(\d+)u?\b", text)}
    for body in re.findall(r"typedef enum \w*\s*\{(.*?)\}", text, flags=re.S):
        body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
        consts.update({n: int(v) for n, v in re.findall(r"(FA_[A-Z_]+)\s*=\s*(\d+)", body)})
    return consts


def test_binding_constants_match_the_header(fa):
    consts = _header_constants()
    for name in ("FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA", "FA_ERR_OOM",
                 "FA_ERR_TIMEOUT", "FA_ERR_INTERNAL", "FA_MASK_CAUSAL", "FA_MASK_SLIDING_WINDOW",
                 "FA_MASK_DOCUMENT", "FA_SCORE_NONE", "FA_SCORE_SOFTCAP", "FA_SCORE_ALIBI",
                 "FA_DTYPE_F16", "FA_DTYPE_BF16"):
        assert name in consts, name
        assert getattr(fa, name) == consts[name], name


def test_struct_layouts_match_the_header(fa):
    # ctypes mirrors of the ABI structs: field order and sizes as declared (64-bit ABI).
    assert ctypes.sizeof(fa.FaMaskParams) == 40      # int32, pad, void*, int32 x 3, pad, void*
    assert ctypes.sizeof(fa.FaScoreParams) == 16     # float, pad, const float*
    assert ctypes.sizeof(fa.FaTensor) == 8 + 8 + 4 * 8 + 4 * 8
    text = open(os.path.join(ROOT, "include", "fa_b200.h")).read()
    for struct, fields in (("fa_mask_params", ["window", "doc_id", "separate_full_blocks",
                                               "dq_kv_order", "kv_block_size", "kv_lens"]),
                           ("fa_score_params", ["softcap", "alibi_slopes"]),
                           ("fa_tensor", ["data", "dtype", "B", "stride"])):
        body = re.search(r"typedef struct %s \{(.*?)\}" % struct, text, flags=re.S).group(1)
        body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
        pos = [body.index(f) for f in fields]
        assert pos == sorted(pos), struct


def test_binding_checks_lse_before_the_call(fa):
    import torch

    class _Mask:                      # never reached: the check comes first
        handle, device = 0, None
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    for bad in (torch.zeros(1, 2, 128), torch.zeros(1, 2, 128, dtype=torch.float64),
                torch.zeros(1, 2, 64)):
        with pytest.raises(ValueError):
            fa.flex_attention(q, q, q, _Mask(), lse=bad)


class _FakeCudaIds:
    """Stands in for a CUDA int32 tensor (no GPU here): only what check_doc_id reads."""

    def __init__(self, n, device="cuda:0", dims=1):
        import torch
        self.is_cuda = True
        self.dtype = torch.int32
        self.device = torch.device(device)
        self.shape = (n,) if dims == 1 else (1, n)
        self._n = n
        self._dims = dims

    def is_contiguous(self):
        return True

    def dim(self):
        return self._dims

    def numel(self):
        return self._n


def test_binding_rejects_a_doc_id_shorter_than_kv_len(fa):
    # The C ABI reads KV_LEN ids through a bare pointer; a short vector would be read out of
    # bounds on the device, so the binding refuses it before anything is launched.
    with pytest.raises(ValueError, match="KV_LEN=1024"):
        fa.check_doc_id(_FakeCudaIds(1000), 1024, "cuda:0")
    with pytest.raises(ValueError, match="KV_LEN"):
        fa.check_doc_id(_FakeCudaIds(1024, dims=2), 1024, "cuda:0")
    with pytest.raises(ValueError, match="lives on"):
        fa.check_doc_id(_FakeCudaIds(1024, device="cuda:1"), 1024, "cuda:0")
    fa.check_doc_id(_FakeCudaIds(1024), 1024, "cuda:0")
