"""fa_create_block_mask_noalloc: the block-mask build for callers that cannot let the library
allocate device memory (a framework whose allocator owns the GPU's memory, a runtime plugin
whose enqueue path must not allocate, a deployment that forbids allocation after start-up).

It writes the four lists into buffers the caller owns and keeps its only scratch (per-block
document statistics) in a fixed device array shared by all calls.  The test calls it through
the C ABI twice in a row per case -- with cases ordered so the shared scratch always holds
another mask's leftovers -- and checks every list against fa_create_block_mask and against
the oracle's brute force, bit for bit (the tolerance of the integer metadata).  A last test
checks the property the entry point exists for: repeated calls leave the device's free
memory unchanged.  Kept in its own file, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

C, SW, DOC = wl.MASK_CAUSAL, wl.MASK_SLIDING_WINDOW, wl.MASK_DOCUMENT


def _fa():
    import block_sparse_masked_x128_b200 as fa
    return fa


def _lists_noalloc(kind, B, H, Q, KV, window=0, doc=None, separate_full=True):
    fa = _fa()
    Bm, Hm = B or 1, H or 1
    QB, KVB = -(-Q // 128), -(-KV // 128)
    # Filled with a sentinel so an element the entry point forgets to write shows up.
    kvn = torch.full((Bm, Hm, QB), -7, dtype=torch.int32, device="cuda")
    kvi = torch.full((Bm, Hm, QB, KVB), -7, dtype=torch.int32, device="cuda")
    fn = torch.full((Bm, Hm, QB), -7, dtype=torch.int32, device="cuda")
    fi = torch.full((Bm, Hm, QB, KVB), -7, dtype=torch.int32, device="cuda")
    doc_t = torch.from_numpy(doc).cuda() if doc is not None else None
    if doc_t is not None:
        fa.check_doc_id(doc_t, KV, doc_t.device)   # the C ABI reads KV ids in place
    params = fa.FaMaskParams(int(window), doc_t.data_ptr() if doc_t is not None else None,
                             1 if separate_full else 0)
    st = fa._lib.fa_create_block_mask_noalloc(
        kind, ctypes.byref(params), B, H, Q, KV, 128, kvn.data_ptr(), kvi.data_ptr(), fn.data_ptr(),
        fi.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == fa.FA_OK, fa.fa_last_error_message()
    torch.cuda.synchronize()
    return {"kv_num_blocks": kvn, "kv_indices": kvi, "full_kv_num_blocks": fn, "full_kv_indices": fi}


def _lists_reference(kind, B, H, Q, KV, window=0, doc=None, separate_full=True):
    fa = _fa()
    doc_t = torch.from_numpy(doc).cuda() if doc is not None else None
    bm = fa.create_block_mask(kind, B or None, H or None, Q, KV, window=window, doc_id=doc_t,
                              separate_full_blocks=separate_full)
    torch.cuda.synchronize()
    return {n: getattr(bm, n) for n in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks",
                                        "full_kv_indices")}


rng = np.random.default_rng(3)
CASES = [
    ("document_packed_8k", dict(kind=C | DOC, B=0, H=0, Q=8192, KV=8192, doc=wl.make_doc_ids(wl.WORKLOADS[3]))),
    ("three_documents_8k", dict(kind=C | DOC, B=0, H=0, Q=8192, KV=8192, doc=wl.three_doc_ids_from_page())),
    ("interleaved_ids", dict(kind=DOC, B=0, H=0, Q=768, KV=768, doc=rng.integers(0, 3, 768).astype(np.int32))),
    ("doc_window_per_head", dict(kind=SW | DOC, B=2, H=3, Q=1000, KV=1000, window=200,
                                 doc=wl.doc_ids_from_lengths([100, 1, 876, 23]))),
    ("causal_window_no_scratch", dict(kind=C | SW, B=0, H=0, Q=8192, KV=8192, window=1024)),
    ("causal_32k_not_separated", dict(kind=C, B=0, H=0, Q=32768, KV=32768, separate_full=False)),
]


def _lists_oracle(kind, B, H, Q, KV, window=0, doc=None, separate_full=True):
    mm = oracle.make_mask_mod(kind, window=window or None, document_id=doc)
    one = oracle.create_block_mask(mm, None, None, Q, KV, separate_full_blocks=separate_full)
    Bm, Hm = B or 1, H or 1
    # These mask_mods do not depend on b or h: a per-(b, h) mask repeats the broadcast lists.
    return {n: np.broadcast_to(one[n], (Bm, Hm) + one[n].shape[2:])
            for n in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices")}


@pytest.mark.parametrize("name,case", CASES, ids=[c[0] for c in CASES])
def test_noalloc_lists_equal_create_block_mask_on_two_calls_in_a_row(name, case):
    ref = _lists_reference(**case)
    want_oracle = _lists_oracle(**case)
    for call in range(2):
        got = _lists_noalloc(**case)
        for key, want in ref.items():
            assert torch.equal(got[key], want), f"call {call}: {key} differs"
            assert np.array_equal(got[key].cpu().numpy(), want_oracle[key]), \
                f"call {call}: {key} differs from the oracle"


def test_noalloc_calls_allocate_no_device_memory():
    fa = _fa()
    kind, Q = C | DOC, 8192
    QB = Q // 128
    doc_t = torch.from_numpy(wl.make_doc_ids(wl.WORKLOADS[3])).cuda()
    kvn, fn = (torch.empty(QB, dtype=torch.int32, device="cuda") for _ in range(2))
    kvi, fi = (torch.empty(QB * QB, dtype=torch.int32, device="cuda") for _ in range(2))
    params = fa.FaMaskParams(0, doc_t.data_ptr(), 1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        st = fa._lib.fa_create_block_mask_noalloc(kind, ctypes.byref(params), 0, 0, Q, Q, 128,
                                                  kvn.data_ptr(), kvi.data_ptr(), fn.data_ptr(),
                                                  fi.data_ptr(), stream)
        assert st == fa.FA_OK, fa.fa_last_error_message()

    call()                       # first call on the device: looks up the scratch address
    torch.cuda.synchronize()
    free0, allocated0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(8):
        call()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == allocated0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    fa = _fa()
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = z.data_ptr()
    st = fa._lib.fa_create_block_mask_noalloc(C, None, 0, 0, 128 * 4097, 128, 128, p, p, p, p, None)
    assert st == fa.FA_ERR_UNSUPPORTED
    assert "4096 blocks" in fa.fa_last_error_message()


def test_noalloc_rejects_host_output_buffers():
    fa = _fa()
    dev = torch.zeros(4 * 4, dtype=torch.int32, device="cuda")
    host = torch.zeros(4 * 4, dtype=torch.int32).pin_memory()
    d, h = dev.data_ptr(), host.data_ptr()
    st = fa._lib.fa_create_block_mask_noalloc(C, None, 0, 0, 512, 512, 128, h, d, d, d, None)
    assert st == fa.FA_ERR_INVALID_ARG
    assert "kv_num_blocks" in fa.fa_last_error_message()
    torch.cuda.synchronize()
