"""Block-sparse masked attention forward for NVIDIA B200 (sm_100a).

A thin ctypes binding of the C ABI in ``include/fa_b200.h``.  It only marshals arguments:
every step of the computation runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams.  There is no CPU fallback: importing this package fails loudly if the
shared library has not been built (``python block_sparse_masked_x128_b200/build.py``).

Low-level names mirror the C entry points (``fa_create_block_mask``, ``fa_forward``, ...).
``create_block_mask`` and ``flex_attention`` are the convenience forms named after the
FlexAttention API the pages use ("How to Use FlexAttention on Apple Silicon", Setup).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

# FA_B200_LIBRARY may name another build of the same library (build.py --debug writes
# _lib/libfa_b200_debug.so, whose kernels check metadata indices); the default is the product.
_LIB_PATH = os.environ.get("FA_B200_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "_lib", "libfa_b200.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python block_sparse_masked_x128_b200/build.py`")
_lib = ctypes.CDLL(_LIB_PATH)

# ---------------------------------------------------------------- constants (fa_b200.h)
FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_OOM = 4
FA_ERR_TIMEOUT = 5
FA_ERR_INTERNAL = 6

FA_MASK_CAUSAL = 1
FA_MASK_SLIDING_WINDOW = 2
FA_MASK_DOCUMENT = 4
FA_SCORE_NONE = 0
FA_SCORE_SOFTCAP = 1
FA_SCORE_ALIBI = 2
FA_DTYPE_F16 = 0
FA_DTYPE_BF16 = 1

EXPORTED = ("fa_create_block_mask", "fa_forward", "fa_block_mask_get", "fa_get_device_status",
            "fa_destroy_block_mask", "fa_status_string", "fa_last_error_message",
            "fa_create_block_mask_noalloc", "fa_debug_set_stall", "fa_masked_softmax",
            "fa_masked_softmax_status", "fa_backward", "fa_backward_workspace_bytes",
            "fa_block_mask_from_kv_blocks", "fa_forward_paged", "fa_forward_paged_workspace_bytes")


class FaMaskParams(ctypes.Structure):
    _fields_ = [("window", ctypes.c_int32), ("doc_id", ctypes.c_void_p),
                ("separate_full_blocks", ctypes.c_int32), ("dq_kv_order", ctypes.c_int32),
                ("kv_block_size", ctypes.c_int32), ("kv_lens", ctypes.c_void_p)]


class FaScoreParams(ctypes.Structure):
    _fields_ = [("softcap", ctypes.c_float), ("alibi_slopes", ctypes.c_void_p)]


class FaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("S", ctypes.c_int64),
                ("D", ctypes.c_int64), ("stride", ctypes.c_int64 * 4)]


class FaBlockMaskInfo(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("Q_LEN", ctypes.c_int32),
                ("KV_LEN", ctypes.c_int32), ("BLOCK_SIZE", ctypes.c_int32),
                ("q_blocks", ctypes.c_int32), ("kv_blocks", ctypes.c_int32),
                ("mask_kind", ctypes.c_uint32), ("window", ctypes.c_int32),
                ("separate_full_blocks", ctypes.c_int32),
                ("kv_num_blocks", ctypes.c_void_p), ("kv_indices", ctypes.c_void_p),
                ("full_kv_num_blocks", ctypes.c_void_p), ("full_kv_indices", ctypes.c_void_p),
                ("q_num_blocks", ctypes.c_void_p), ("q_indices", ctypes.c_void_p),
                ("full_q_num_blocks", ctypes.c_void_p), ("full_q_indices", ctypes.c_void_p),
                ("dq_kv_order", ctypes.c_int32), ("KV_BLOCK_SIZE", ctypes.c_int32)]


_status = ctypes.c_int
_lib.fa_create_block_mask.argtypes = [ctypes.c_uint32, ctypes.POINTER(FaMaskParams), ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)]
_lib.fa_create_block_mask.restype = _status
_lib.fa_forward.argtypes = [ctypes.POINTER(FaTensor), ctypes.POINTER(FaTensor), ctypes.POINTER(FaTensor),
                            ctypes.c_void_p, ctypes.c_uint32, ctypes.POINTER(FaScoreParams),
                            ctypes.c_float, ctypes.POINTER(FaTensor), ctypes.c_void_p, ctypes.c_void_p]
_lib.fa_forward.restype = _status
_lib.fa_forward_paged.argtypes = [ctypes.POINTER(FaTensor), ctypes.POINTER(FaTensor), ctypes.POINTER(FaTensor),
                                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_uint32,
                                  ctypes.POINTER(FaScoreParams), ctypes.c_float, ctypes.POINTER(FaTensor),
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
_lib.fa_forward_paged.restype = _status
_lib.fa_forward_paged_workspace_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                  ctypes.c_int64, ctypes.c_int64]
_lib.fa_forward_paged_workspace_bytes.restype = ctypes.c_size_t
_lib.fa_create_block_mask_noalloc.argtypes = [
    ctypes.c_uint32, ctypes.POINTER(FaMaskParams), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
    ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
    ctypes.c_void_p]
_lib.fa_create_block_mask_noalloc.restype = _status
_lib.fa_block_mask_get.argtypes = [ctypes.c_void_p, ctypes.POINTER(FaBlockMaskInfo)]
_lib.fa_block_mask_get.restype = _status
_lib.fa_get_device_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
_lib.fa_get_device_status.restype = _status
_lib.fa_destroy_block_mask.argtypes = [ctypes.c_void_p]
_lib.fa_destroy_block_mask.restype = None
_lib.fa_status_string.argtypes = [ctypes.c_int]
_lib.fa_status_string.restype = ctypes.c_char_p
_lib.fa_last_error_message.argtypes = []
_lib.fa_last_error_message.restype = ctypes.c_char_p
_lib.fa_debug_set_stall.argtypes = [ctypes.c_int32]
_lib.fa_debug_set_stall.restype = _status
_lib.fa_masked_softmax.argtypes = [ctypes.POINTER(FaTensor), ctypes.c_uint32, ctypes.c_int64,
                                   ctypes.POINTER(FaTensor), ctypes.c_void_p]
_lib.fa_masked_softmax.restype = _status
_lib.fa_masked_softmax_status.argtypes = [ctypes.c_void_p]
_lib.fa_masked_softmax_status.restype = _status
_lib.fa_block_mask_from_kv_blocks.argtypes = [
    ctypes.c_uint32, ctypes.POINTER(FaMaskParams), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
    ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)]
_lib.fa_block_mask_from_kv_blocks.restype = _status
_lib.fa_backward_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
_lib.fa_backward_workspace_bytes.restype = ctypes.c_size_t
_lib.fa_backward.argtypes = [ctypes.POINTER(FaTensor)] * 5 + [
    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint32, ctypes.POINTER(FaScoreParams), ctypes.c_float,
    ctypes.POINTER(FaTensor), ctypes.POINTER(FaTensor), ctypes.POINTER(FaTensor), ctypes.c_void_p,
    ctypes.c_size_t, ctypes.c_void_p]
_lib.fa_backward.restype = _status


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.fa_last_error_message().decode()
        super().__init__(f"{where}: {_lib.fa_status_string(status).decode()}: {msg}")


def _check(status: int, where: str) -> None:
    if status != FA_OK:
        raise FaError(status, where)


def library_path() -> str:
    return _LIB_PATH


def fa_status_string(status: int) -> str:
    return _lib.fa_status_string(status).decode()


def fa_last_error_message() -> str:
    return _lib.fa_last_error_message().decode()


# ---------------------------------------------------------------- low-level entry points

def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return getattr(stream, "cuda_stream", stream)


def _dtype_code(dtype) -> int:
    import torch
    if dtype == torch.bfloat16:
        return FA_DTYPE_BF16
    if dtype == torch.float16:
        return FA_DTYPE_F16
    raise TypeError(f"unsupported dtype {dtype}: use torch.float16 or torch.bfloat16")


def fa_tensor(t) -> FaTensor:
    """Describe a 4-D (B, H, S, D) torch tensor for the C ABI (no copy)."""
    if t.dim() != 4:
        raise ValueError("expected a (B, H, S, D) tensor")
    st = (ctypes.c_int64 * 4)(*t.stride())
    B, H, S, D = t.shape
    return FaTensor(t.data_ptr(), _dtype_code(t.dtype), B, H, S, D, st)


def fa_create_block_mask(mask_kind: int, params: Optional[FaMaskParams], B: int, H: int,
                         Q_LEN: int, KV_LEN: int, BLOCK_SIZE: int = 128, stream=None) -> int:
    """Call fa_create_block_mask; returns the raw handle (raises FaError on failure)."""
    h = ctypes.c_void_p()
    st = _lib.fa_create_block_mask(mask_kind, ctypes.byref(params) if params is not None else None,
                                   B, H, Q_LEN, KV_LEN, BLOCK_SIZE, _stream_ptr(stream), ctypes.byref(h))
    _check(st, "fa_create_block_mask")
    return h.value


def fa_forward(q: FaTensor, k: FaTensor, v: FaTensor, block_mask: int, score_mod_kind: int,
               params: Optional[FaScoreParams], scale: float, out: FaTensor, lse_ptr: Optional[int],
               stream=None) -> None:
    st = _lib.fa_forward(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), block_mask, score_mod_kind,
                         ctypes.byref(params) if params is not None else None, scale, ctypes.byref(out),
                         lse_ptr, _stream_ptr(stream))
    _check(st, "fa_forward")


def fa_create_block_mask_noalloc(mask_kind: int, params: Optional[FaMaskParams], B: int, H: int,
                                 Q_LEN: int, KV_LEN: int, BLOCK_SIZE: int, kv_num_blocks: int,
                                 kv_indices: int, full_kv_num_blocks: int, full_kv_indices: int,
                                 stream=None) -> None:
    """Call fa_create_block_mask_noalloc: build the four lists into caller-owned device buffers
    (pointers as integers) without any device allocation by the library."""
    st = _lib.fa_create_block_mask_noalloc(mask_kind, ctypes.byref(params) if params is not None else None,
                                           B, H, Q_LEN, KV_LEN, BLOCK_SIZE, kv_num_blocks, kv_indices,
                                           full_kv_num_blocks, full_kv_indices, _stream_ptr(stream))
    _check(st, "fa_create_block_mask_noalloc")


def fa_block_mask_get(block_mask: int) -> FaBlockMaskInfo:
    info = FaBlockMaskInfo()
    _check(_lib.fa_block_mask_get(block_mask, ctypes.byref(info)), "fa_block_mask_get")
    return info


def fa_get_device_status(block_mask: int, stream=None) -> int:
    """Synchronise the stream and return the status code (FA_OK or FA_ERR_TIMEOUT ...)."""
    return _lib.fa_get_device_status(block_mask, _stream_ptr(stream))


def fa_destroy_block_mask(block_mask: int) -> None:
    _lib.fa_destroy_block_mask(block_mask)


def fa_backward_workspace_bytes(B: int, H: int, Q_LEN: int) -> int:
    return int(_lib.fa_backward_workspace_bytes(B, H, Q_LEN))


def fa_backward(q: FaTensor, k: FaTensor, v: FaTensor, out: FaTensor, dout: FaTensor, lse_ptr: int,
                block_mask: int, score_mod_kind: int, params: Optional[FaScoreParams], scale: float,
                dq: FaTensor, dk: FaTensor, dv: FaTensor, workspace_ptr: int, workspace_bytes: int,
                stream=None) -> None:
    st = _lib.fa_backward(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(out),
                          ctypes.byref(dout), lse_ptr, block_mask, score_mod_kind,
                          ctypes.byref(params) if params is not None else None, scale,
                          ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), workspace_ptr,
                          workspace_bytes, _stream_ptr(stream))
    _check(st, "fa_backward")


def fa_masked_softmax(scores: FaTensor, mask_kind: int, offset: int, probs: FaTensor,
                      stream=None) -> None:
    _check(_lib.fa_masked_softmax(ctypes.byref(scores), mask_kind, offset, ctypes.byref(probs),
                                  _stream_ptr(stream)), "fa_masked_softmax")


def fa_masked_softmax_status(stream=None) -> int:
    """Synchronise the stream and return FA_OK or FA_ERR_TIMEOUT for the softmax kernels."""
    return _lib.fa_masked_softmax_status(_stream_ptr(stream))


def fa_debug_set_stall(enable: bool) -> None:
    """Test hook: make every later forward's bounded K wait run out (see the C header)."""
    _check(_lib.fa_debug_set_stall(1 if enable else 0), "fa_debug_set_stall")


# ---------------------------------------------------------------- convenience API

class _DeviceArray:
    """Zero-copy view of library-owned int32 device memory (for torch.as_tensor)."""

    def __init__(self, ptr: int, shape):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": "<i4",
                                         "data": (ptr, False), "version": 3, "strides": None}


class BlockMask:
    """A block mask built on the GPU; release happens when the object is collected.

    Attributes ``kv_num_blocks``, ``kv_indices``, ``full_kv_num_blocks`` and
    ``full_kv_indices`` are int32 CUDA tensors copied out of the library's buffers.
    """

    def __init__(self, handle: int, device, keepalive=None):
        self.handle = handle
        self.device = device
        self._keepalive = keepalive
        self.info = fa_block_mask_get(handle)

    def _view(self, ptr, shape):
        import torch
        return torch.as_tensor(_DeviceArray(ptr, shape), device=self.device).clone()

    @property
    def shape_prefix(self):
        return (self.info.B, self.info.H, self.info.q_blocks)

    @property
    def kv_num_blocks(self):
        return self._view(self.info.kv_num_blocks, self.shape_prefix)

    @property
    def kv_indices(self):
        return self._view(self.info.kv_indices, self.shape_prefix + (self.info.kv_blocks,))

    @property
    def full_kv_num_blocks(self):
        return self._view(self.info.full_kv_num_blocks, self.shape_prefix)

    @property
    def full_kv_indices(self):
        return self._view(self.info.full_kv_indices, self.shape_prefix + (self.info.kv_blocks,))

    @property
    def q_num_blocks(self):
        return self._view(self.info.q_num_blocks, (self.info.B, self.info.H, self.info.kv_blocks))

    @property
    def q_indices(self):
        return self._view(self.info.q_indices, (self.info.B, self.info.H, self.info.kv_blocks,
                                                 self.info.q_blocks))

    @property
    def full_q_num_blocks(self):
        return self._view(self.info.full_q_num_blocks, (self.info.B, self.info.H, self.info.kv_blocks))

    @property
    def full_q_indices(self):
        return self._view(self.info.full_q_indices, (self.info.B, self.info.H, self.info.kv_blocks,
                                                      self.info.q_blocks))

    def device_status(self, stream=None) -> int:
        return fa_get_device_status(self.handle, stream)

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h:
            try:
                fa_destroy_block_mask(h)
            except Exception:
                pass


def check_doc_id(doc_id, KV_LEN: int, device) -> None:
    """Raise ValueError unless doc_id is a contiguous 1-D int32 tensor of KV_LEN ids on
    `device` (the library reads exactly KV_LEN ids through a bare pointer)."""
    import torch
    if not (doc_id.is_cuda and doc_id.dtype == torch.int32 and doc_id.is_contiguous()):
        raise ValueError("doc_id must be a contiguous int32 CUDA tensor")
    if doc_id.dim() != 1 or doc_id.numel() != int(KV_LEN):
        raise ValueError(f"doc_id must hold exactly KV_LEN={int(KV_LEN)} ids, got shape "
                         f"{tuple(doc_id.shape)}")
    if doc_id.device != torch.device(device):
        raise ValueError(f"doc_id lives on {doc_id.device}, the mask on {device}")


def _block_sizes(BLOCK_SIZE):
    if isinstance(BLOCK_SIZE, (tuple, list)):
        bq, bkv = BLOCK_SIZE
        return int(bq), int(bkv)
    return int(BLOCK_SIZE), int(BLOCK_SIZE)


def _mask_params(mask_kind, KV_LEN, window, doc_id, separate_full_blocks, dq_kv_order, bkv, dev,
                 kv_lens=None, B=None):
    import torch
    doc_ptr = None
    if doc_id is not None:
        # The C ABI reads KV_LEN ids through a bare pointer: check what it cannot.
        check_doc_id(doc_id, KV_LEN, dev)
        doc_ptr = doc_id.data_ptr()
    lens_ptr = None
    if kv_lens is not None:
        # ... and B context lengths, one per batch element.
        if not (kv_lens.is_cuda and kv_lens.dtype == torch.int32 and kv_lens.is_contiguous()
                and kv_lens.dim() == 1 and B and kv_lens.numel() == int(B)
                and kv_lens.device == torch.device(dev)):
            raise ValueError("kv_lens must be a contiguous int32 CUDA tensor of B lengths on the "
                             "mask's device (and B must be given)")
        lens_ptr = kv_lens.data_ptr()
    return FaMaskParams(int(window), doc_ptr, 1 if separate_full_blocks else 0,
                        1 if dq_kv_order else 0, int(bkv), lens_ptr)


def create_block_mask(mask_kind: int, B: Optional[int], H: Optional[int], Q_LEN: int, KV_LEN: int,
                      *, window: int = 0, doc_id=None, separate_full_blocks: bool = True,
                      dq_kv_order: bool = True, BLOCK_SIZE=128, kv_lens=None, device=None,
                      stream=None) -> BlockMask:
    """Build a block mask on the current CUDA device (B or H of None broadcasts).
    BLOCK_SIZE is an int or a (q, kv) pair: the block size of the lists read back.  kv_lens
    (int32 CUDA tensor of B lengths) masks keys past each batch element's context."""
    import torch
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    bq, bkv = _block_sizes(BLOCK_SIZE)
    params = _mask_params(mask_kind, KV_LEN, window, doc_id, separate_full_blocks, dq_kv_order, bkv, dev,
                          kv_lens, B)
    with torch.cuda.device(dev):
        h = fa_create_block_mask(int(mask_kind), params, int(B or 0), int(H or 0), int(Q_LEN),
                                 int(KV_LEN), bq, stream)
    # doc_id and kv_lens are copied on the stream; keep them alive until the stream has run.
    return BlockMask(h, dev, keepalive=(doc_id, kv_lens))


def block_mask_from_kv_blocks(kv_num_blocks, kv_indices, full_kv_num_blocks=None,
                              full_kv_indices=None, *, Q_LEN: int, KV_LEN: int, BLOCK_SIZE=128,
                              mask_kind: int = 0, window: int = 0, doc_id=None,
                              separate_full_blocks: bool = True, dq_kv_order: bool = True,
                              stream=None) -> BlockMask:
    """BlockMask.from_kv_blocks: a mask from caller block lists (int32 CUDA tensors of shape
    (B, H, QBu) and (B, H, QBu, KVBu)); block sizes must be multiples of 128.  mask_kind and
    its parameters give the mask_mod applied on partial blocks (0: none)."""
    import torch
    bq, bkv = _block_sizes(BLOCK_SIZE)
    dev = kv_indices.device
    B, H = kv_indices.shape[0], kv_indices.shape[1]
    lists = [kv_num_blocks, kv_indices] + ([full_kv_num_blocks, full_kv_indices]
                                           if full_kv_num_blocks is not None else [])
    QBu, KVBu = -(-int(Q_LEN) // bq), -(-int(KV_LEN) // bkv)
    for t, shape in zip(lists, [(B, H, QBu), (B, H, QBu, KVBu)] * 2):
        if not (t.is_cuda and t.dtype == torch.int32 and t.is_contiguous() and tuple(t.shape) == shape
                and t.device == dev):
            raise ValueError(f"block lists must be contiguous int32 CUDA tensors of shape {shape}")
    params = _mask_params(mask_kind, KV_LEN, window, doc_id, separate_full_blocks, dq_kv_order, bkv, dev)
    h = ctypes.c_void_p()
    with torch.cuda.device(dev):
        st = _lib.fa_block_mask_from_kv_blocks(
            int(mask_kind), ctypes.byref(params), B, H, int(Q_LEN), int(KV_LEN), bq, bkv,
            kv_num_blocks.data_ptr(), kv_indices.data_ptr(),
            full_kv_num_blocks.data_ptr() if full_kv_num_blocks is not None else None,
            full_kv_indices.data_ptr() if full_kv_indices is not None else None,
            _stream_ptr(stream), ctypes.byref(h))
    _check(st, "fa_block_mask_from_kv_blocks")
    return BlockMask(h.value, dev, keepalive=(doc_id, lists))


def flex_attention(q, k, v, block_mask: BlockMask, *, score_mod: int = FA_SCORE_NONE,
                   softcap: float = 30.0, alibi_slopes=None, scale: Optional[float] = None,
                   out=None, lse=None, return_lse: bool = True, page_table=None,
                   split_decode: bool = True, workspace=None, stream=None) -> Tuple:
    """Fused block-sparse attention forward: returns (out, lse) (lse None if not requested).
    With page_table (int32 CUDA tensor (B, n) of page indices), k and v are (n_pages, H, 128, D)
    page pools and the mask's KV_LEN is the logical context length; with at most 4 query rows
    and split_decode the split decode path runs (its workspace is allocated when not given)."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty(q.shape[0], q.shape[1], q.shape[2], device=q.device, dtype=torch.float32)
    if lse is not None:
        # The C ABI takes lse as a bare pointer to [B][H][Q_LEN] fp32: check what it cannot.
        if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
                and tuple(lse.shape) == tuple(q.shape[:3]) and lse.device == q.device):
            raise ValueError("lse must be a contiguous float32 CUDA tensor of shape (B, H, Q_LEN) "
                             "on q's device")
    params = FaScoreParams(float(softcap), _check_alibi(alibi_slopes, q))
    with torch.cuda.device(q.device if q.is_cuda else block_mask.device):
        if page_table is None:
            fa_forward(fa_tensor(q), fa_tensor(k), fa_tensor(v), block_mask.handle, int(score_mod), params,
                       float(scale) if scale is not None else -1.0, fa_tensor(out),
                       lse.data_ptr() if lse is not None else None, stream)
        else:
            # The C ABI reads the table through a bare pointer: rows of kv_blocks entries.
            if not (page_table.is_cuda and page_table.dtype == torch.int32 and page_table.dim() == 2
                    and page_table.stride(1) == 1 and page_table.shape[0] == q.shape[0]
                    and page_table.shape[1] >= -(-block_mask.info.KV_LEN // 128)
                    and page_table.device == q.device):
                raise ValueError("page_table must be an int32 CUDA tensor (B, >= kv blocks) with "
                                 "contiguous rows on q's device")
            ws_ptr, ws_bytes = None, 0
            if split_decode:
                need = int(_lib.fa_forward_paged_workspace_bytes(block_mask.handle, q.shape[0], q.shape[1],
                                                                 q.shape[2], q.shape[3]))
                if need > 0:
                    if workspace is None:
                        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
                    ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
            st = _lib.fa_forward_paged(ctypes.byref(fa_tensor(q)), ctypes.byref(fa_tensor(k)),
                                       ctypes.byref(fa_tensor(v)), page_table.data_ptr(),
                                       page_table.stride(0), block_mask.handle, int(score_mod),
                                       ctypes.byref(params), float(scale) if scale is not None else -1.0,
                                       ctypes.byref(fa_tensor(out)),
                                       lse.data_ptr() if lse is not None else None, ws_ptr, ws_bytes,
                                       _stream_ptr(stream))
            _check(st, "fa_forward_paged")
    return out, lse



def _check_alibi(alibi_slopes, q):
    if alibi_slopes is None:
        return None
    import torch
    # The kernels read slope h for h < H through a bare pointer: H contiguous floats.
    if not (alibi_slopes.is_cuda and alibi_slopes.dtype == torch.float32
            and alibi_slopes.is_contiguous() and alibi_slopes.numel() == q.shape[1]
            and alibi_slopes.device == q.device):
        raise ValueError("alibi_slopes must be a contiguous float32 CUDA tensor of H "
                         "values on q's device")
    return alibi_slopes.data_ptr()


def flex_attention_backward(q, k, v, out, lse, dout, block_mask: BlockMask, *,
                            score_mod: int = FA_SCORE_NONE, softcap: float = 30.0, alibi_slopes=None,
                            scale: Optional[float] = None, dq=None, dk=None, dv=None,
                            workspace=None, stream=None) -> Tuple:
    """Gradients (dq, dk, dv) of flex_attention for the upstream gradient dout, given the
    forward's out and lse; deterministic (bitwise repeatable)."""
    import torch
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
            and tuple(lse.shape) == tuple(q.shape[:3]) and lse.device == q.device):
        raise ValueError("lse must be the forward's contiguous float32 (B, H, Q_LEN) CUDA tensor")
    nbytes = fa_backward_workspace_bytes(q.shape[0], q.shape[1], q.shape[2])
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    elif workspace.numel() * workspace.element_size() < nbytes or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA buffer of at least {nbytes} bytes")
    params = FaScoreParams(float(softcap), _check_alibi(alibi_slopes, q))
    with torch.cuda.device(q.device):
        fa_backward(fa_tensor(q), fa_tensor(k), fa_tensor(v), fa_tensor(out), fa_tensor(dout),
                    lse.data_ptr(), block_mask.handle, int(score_mod), params,
                    float(scale) if scale is not None else -1.0, fa_tensor(dq), fa_tensor(dk),
                    fa_tensor(dv), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                    stream)
    return dq, dk, dv


def masked_softmax(scores, offset: Optional[int] = None, *, causal: bool = True, out=None,
                   stream=None):
    """softmax(where(q + offset >= kv, scores, finfo.min)) over the last axis of a
    (B, H, Q, K) fp16/bf16 CUDA tensor, in one fused kernel; offset defaults to K - Q.
    ``causal=False`` gives the plain softmax.  ``out`` may be ``scores`` (in place)."""
    import torch
    if offset is None:
        offset = scores.shape[3] - scores.shape[2]
    if out is None:
        out = torch.empty_like(scores)
    with torch.cuda.device(scores.device):
        fa_masked_softmax(fa_tensor(scores), FA_MASK_CAUSAL if causal else 0, int(offset),
                          fa_tensor(out), stream)
    return out
