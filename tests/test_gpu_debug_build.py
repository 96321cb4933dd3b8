"""The FA_DEBUG build (build.py --debug): its kernels check every index they read from a
mask's metadata and record a bad one instead of faulting.  Run in a child process that loads
that build (FA_B200_LIBRARY), on the forward and the backward of a small document mask: the
checks must not fire on valid metadata, and the results must equal the product build's."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_LIB = os.path.join(ROOT, "block_sparse_masked_x128_b200", "_lib", "libfa_b200_debug.so")

CHILD = r'''
import sys, torch
sys.path.insert(0, sys.argv[1])
import block_sparse_masked_x128_b200 as fa
import workloads as wl
w = wl.WORKLOADS[3].scaled(S=1024, H=2)
q, k, v = (t.cuda() for t in wl.make_qkv(w))
do = wl.make_dout(w).cuda()
doc = torch.from_numpy(wl.make_doc_ids(w)).cuda()
bm = fa.create_block_mask(w.mask_kind, None, None, w.S, w.S, doc_id=doc)
out, lse = fa.flex_attention(q, k, v, bm, scale=w.scale)
dq, dk, dv = fa.flex_attention_backward(q, k, v, out, lse, do, bm, scale=w.scale)
torch.cuda.synchronize()
assert bm.device_status() == fa.FA_OK, fa.fa_last_error_message()
torch.save([t.cpu() for t in (out, lse, dq, dk, dv)], sys.argv[2])
print(fa.library_path())
'''


def _run(lib, out_path):
    env = dict(os.environ)
    if lib:
        env["FA_B200_LIBRARY"] = lib
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, out_path], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout.strip().splitlines()[-1]


def test_debug_build_checks_pass_and_match_the_product(tmp_path):
    import torch
    assert os.path.exists(DEBUG_LIB), "build it with build.py --debug (the graft build step does)"
    loaded = _run(DEBUG_LIB, str(tmp_path / "dbg.pt"))
    assert loaded.endswith("libfa_b200_debug.so")
    _run(None, str(tmp_path / "prod.pt"))
    a = torch.load(tmp_path / "dbg.pt")
    b = torch.load(tmp_path / "prod.pt")
    assert all(torch.equal(x, y) for x, y in zip(a, b))
