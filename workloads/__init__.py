"""Seeded synthetic workloads for block-sparse masked attention.

This module holds the five workload shapes and the seeded generators of their
inputs, and nothing of the attention method itself: no mask predicate, no
softmax, no block classification.  Both the float64 oracle (through the tests)
and the CUDA library (through the tests and the benchmark) draw their inputs
from here, so the two sides always see the same rounded fp16/bf16 values.

Recipe (the same for every workload):
  * q, k, v are i.i.d. N(0, 1), drawn in float32 from
    ``torch.Generator('cpu').manual_seed(seed)`` in the order q, k, v, each of
    shape (B, H, S, D), then rounded to the workload's dtype.  The shape
    (batch, heads, sequence, head_dim) is the one FlexAttention shares with
    scaled_dot_product_attention ("How to Use FlexAttention on Apple Silicon",
    Setup section).
  * The masked-softmax workloads take materialised scores: i.i.d. N(0, 1) float32 (the
    distribution of scale * q k^T for unit-variance q and k), drawn from
    ``torch.Generator('cpu').manual_seed(seed)`` with shape (B, H, Q, K) and rounded to
    bf16.  Q is a chunk of 1024 query rows that closes a context of K keys, so the causal
    offset is K - Q (the 8K and 32K sequences of "Fuse the causal mask into the SDPA
    fallback softmax", MLX pull request 3919).
  * The decode workloads hold a batch of B sequences with seeded context lengths
    (``numpy.random.default_rng(seed).integers(lo, hi + 1, B)``), one new query token per
    sequence, and the keys and values in 128-token pages of one shared pool, placed by a
    seeded random permutation of the pages (PagedAttention through block indices, "PyTorch
    2.13 brings custom AI attention to Mac", "What Attention Patterns Does FlexAttention
    Support?").  q, k, v are drawn like the other workloads' (q of shape (B, H, 1, D), k and v
    of shape (B, H, max length, D)); the pool takes each sequence's pages from k and v.
  * The document-packed workload splits T = 8192 positions into 4 documents of
    seeded random lengths, each at least 512 long: three cut points drawn from
    ``numpy.random.default_rng(seed).integers(0, 6145, 3)`` and sorted give the
    gaps of [0, cuts, 6144]; each length is 512 plus its gap.  Document ids are
    0..3 in order, one int32 per position (the document_id vector of the
    "Mask 3: document-packed" section).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# Mask kinds (bit flags; OR means conjunction of the predicates).
MASK_NONE = 0
MASK_CAUSAL = 1
MASK_SLIDING_WINDOW = 2
MASK_DOCUMENT = 4

# Score-mod kinds (bit flags; both means soft-cap first, then the bias).
SCORE_NONE = 0
SCORE_SOFTCAP = 1
SCORE_ALIBI = 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    dtype: str            # "fp16" or "bf16"
    mask_kind: int
    window: int = 0
    n_docs: int = 0
    score_kind: int = SCORE_NONE
    softcap: float = 0.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    def scaled(self, S: Optional[int] = None, B: Optional[int] = None,
               H: Optional[int] = None) -> "Workload":
        """Same workload at another size (used for oracle-sized parity cases)."""
        return dataclasses.replace(self, S=S or self.S, B=B or self.B, H=H or self.H)


# The five workloads, in order.  The seed of each is its 1-based position.
WORKLOADS = [
    Workload("swa128_b1h2_s512_d64_fp16", B=1, H=2, S=512, D=64, dtype="fp16",
             mask_kind=MASK_CAUSAL | MASK_SLIDING_WINDOW, window=128, seed=1),
    Workload("causal_b1h16_s8192_d64_bf16", B=1, H=16, S=8192, D=64, dtype="bf16",
             mask_kind=MASK_CAUSAL, seed=2),
    Workload("swa1024_b2h16_s8192_d128_bf16", B=2, H=16, S=8192, D=128, dtype="bf16",
             mask_kind=MASK_CAUSAL | MASK_SLIDING_WINDOW, window=1024, seed=3),
    Workload("doc4_causal_b1h16_s8192_d128_bf16", B=1, H=16, S=8192, D=128, dtype="bf16",
             mask_kind=MASK_CAUSAL | MASK_DOCUMENT, n_docs=4, seed=4),
    Workload("causal_softcap30_alibi_b1h8_s32768_d128_bf16", B=1, H=8, S=32768, D=128,
             dtype="bf16", mask_kind=MASK_CAUSAL,
             score_kind=SCORE_SOFTCAP | SCORE_ALIBI, softcap=30.0, seed=5),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def torch_dtype(name: str):
    import torch
    return {"fp16": torch.float16, "bf16": torch.bfloat16}[name]


def make_qkv(w: Workload, seed: Optional[int] = None):
    """q, k, v on the CPU in the workload's dtype, drawn as the module doc says."""
    import torch
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.S, w.D)
    out = []
    for _ in range(3):
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        out.append(t.to(torch_dtype(w.dtype)))
    return tuple(out)


def make_dout(w: Workload, seed: Optional[int] = None):
    """Upstream gradient dO for the backward: i.i.d. N(0, 1) float32 of shape (B, H, S, D) from
    ``torch.Generator('cpu').manual_seed(seed + 7919)``, rounded to the workload's dtype."""
    import torch
    g = torch.Generator(device="cpu")
    g.manual_seed((w.seed if seed is None else seed) + 7919)
    t = torch.randn((w.B, w.H, w.S, w.D), generator=g, dtype=torch.float32)
    return t.to(torch_dtype(w.dtype))


def doc_lengths(total: int, n_docs: int, min_len: int, seed: int) -> list:
    """Seeded document lengths, each >= min_len, summing to total."""
    slack = total - n_docs * min_len
    if slack < 0:
        raise ValueError("documents cannot all reach the minimum length")
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.integers(0, slack + 1, n_docs - 1))
    edges = np.concatenate([[0], cuts, [slack]])
    return [int(min_len + g) for g in np.diff(edges)]


def doc_ids_from_lengths(lengths) -> np.ndarray:
    """int32 document id per position: 0 for the first document, 1 for the next..."""
    return np.repeat(np.arange(len(lengths), dtype=np.int32),
                     np.asarray(lengths, dtype=np.int64)).astype(np.int32)


def make_doc_ids(w: Workload, S: Optional[int] = None) -> Optional[np.ndarray]:
    """Document ids for a document-masked workload (None otherwise).

    At the workload's own length the split is the seeded one described above
    (min length 512).  At a reduced length S the same recipe runs with the
    minimum scaled down in proportion, so small parity cases still hold
    several documents with boundaries that do not fall on tile edges.
    """
    if not (w.mask_kind & MASK_DOCUMENT):
        return None
    S = S or w.S
    min_len = max(1, (512 * S) // 8192)
    return doc_ids_from_lengths(doc_lengths(S, w.n_docs, min_len, w.seed))


def three_doc_ids_from_page(S: int = 8192) -> np.ndarray:
    """The three-document split of "Mask 3: document-packed": boundaries at 2048 and 5000."""
    d = np.zeros(S, dtype=np.int32)
    d[2048:] = 1
    d[5000:] = 2
    return d


@dataclasses.dataclass(frozen=True)
class SoftmaxWorkload:
    """Causal-masked softmax over a (B, H, Q, K) tensor of materialised scores."""
    name: str
    B: int
    H: int
    Q: int
    K: int
    offset: int           # query row q sees keys kv <= q + offset
    dtype: str = "bf16"
    seed: int = 0

    def scaled(self, Q: Optional[int] = None, K: Optional[int] = None,
               H: Optional[int] = None) -> "SoftmaxWorkload":
        Q = Q or self.Q
        K = K or self.K
        return dataclasses.replace(self, Q=Q, K=K, H=H or self.H, offset=K - Q)


SOFTMAX_WORKLOADS = [
    SoftmaxWorkload("masked_softmax_b1h8_q1024_k32768_bf16", B=1, H=8, Q=1024, K=32768,
                    offset=32768 - 1024, seed=31),
    SoftmaxWorkload("masked_softmax_b1h8_q1024_k8192_bf16", B=1, H=8, Q=1024, K=8192,
                    offset=8192 - 1024, seed=32),
]
SOFTMAX_BY_NAME = {w.name: w for w in SOFTMAX_WORKLOADS}


def make_scores(w: SoftmaxWorkload, seed: Optional[int] = None):
    """Materialised scores on the CPU in the workload's dtype, as the module doc says."""
    import torch
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    t = torch.randn((w.B, w.H, w.Q, w.K), generator=g, dtype=torch.float32)
    return t.to(torch_dtype(w.dtype))


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """One decode step: B sequences of seeded lengths in [lo, hi], paged K/V, Q_LEN new tokens."""
    name: str
    B: int
    H: int
    D: int
    lo: int
    hi: int
    Q: int = 1
    dtype: str = "bf16"
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    def lengths(self) -> np.ndarray:
        return np.random.default_rng(self.seed).integers(self.lo, self.hi + 1, self.B).astype(np.int32)

    @property
    def kv_len(self) -> int:
        return int(self.lengths().max())


DECODE_WORKLOADS = [
    DecodeWorkload("decode_paged_b16h16_d128_ctx1k-8k_bf16", B=16, H=16, D=128, lo=1024, hi=8192,
                   seed=71),
]


def make_decode(w: DecodeWorkload):
    """q (B, H, Q, D), contiguous k, v (B, H, KV, D), page pools (n_pages, H, 128, D) and the page
    table (B, ceil(KV / 128)) int32, plus the lengths; all on the CPU."""
    import torch
    lens = w.lengths()
    KV = int(lens.max())
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    td = torch_dtype(w.dtype)
    q = torch.randn((w.B, w.H, w.Q, w.D), generator=g, dtype=torch.float32).to(td)
    k = torch.randn((w.B, w.H, KV, w.D), generator=g, dtype=torch.float32).to(td)
    v = torch.randn((w.B, w.H, KV, w.D), generator=g, dtype=torch.float32).to(td)
    nblk = -(-KV // 128)
    pages_per = [-(-int(n) // 128) for n in lens]
    n_pages = sum(pages_per)
    perm = np.random.default_rng(w.seed + 1).permutation(n_pages).astype(np.int32)
    table = np.zeros((w.B, nblk), dtype=np.int32)
    kp = torch.zeros((n_pages, w.H, 128, w.D), dtype=td)
    vp = torch.zeros((n_pages, w.H, 128, w.D), dtype=td)
    nxt = 0
    for b in range(w.B):
        for j in range(pages_per[b]):
            page = int(perm[nxt])
            nxt += 1
            table[b, j] = page
            rows = slice(j * 128, min((j + 1) * 128, KV))
            n = rows.stop - rows.start
            kp[page, :, :n] = k[b, :, rows]
            vp[page, :, :n] = v[b, :, rows]
    return q, k, v, kp, vp, torch.from_numpy(table), lens
