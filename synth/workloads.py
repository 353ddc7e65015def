"""Seeded synthetic prefill workloads shaped like the CoSA evaluation.

The CoSA pages ("CoSA: Accelerating Long-Context Inference via Proxy-Kernel
Co-Designed Sparse Attention", §5.1 Setup) evaluate Llama-3.1-8B and Qwen3-8B
on RULER / LongBench-v2 up to 128K tokens.  Neither the models nor the data
are available, so these generators stand in for them: random bf16 Q/K/V with
the attention heads' shapes (32 query heads, 8 KV heads, head_dim 128) and a
planted block structure (attention sinks, a local diagonal band, vertical
stripes, near-dense heads) so that block selection and in-kernel skipping have
something real to find.  The structure only changes how sparse the result is;
it never enters the method's definition.

Everything is deterministic in the seed: large tensors are filled in fixed
chunks of 2**22 values, each from its own child of a SeedSequence, so the
result does not depend on how many threads fill them.

Tensors are returned as bf16 bit patterns (uint16, round-to-nearest-even from
fp32) in the layouts the library consumes:
  q         [T, Hq, d]            T = sum of sequence lengths (packed)
  k_pages   [P, Hkv, b_p, d]      page pool, one (page, kv head) tile contiguous
  v_pages   [P, Hkv, b_p, d]
  page_table[B, max_pages] int32  physical page of each logical page, -1 pad
Token slots past a sequence's end inside its last page hold finite random
values, so any code that fails to mask them shows up in the comparisons.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_CHUNK = 1 << 22
_THREADS = max(1, min(16, os.cpu_count() or 1))


# ----------------------------------------------------------------------------
# bf16 encoding
# ----------------------------------------------------------------------------

def _parallel_chunks(n: int, fn) -> None:
    nchunks = (n + _CHUNK - 1) // _CHUNK
    if nchunks <= 1:
        for c in range(nchunks):
            fn(c)
        return
    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(fn, range(nchunks)))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest, ties to even.

    Inputs are finite; NaN handling is not needed for generated data.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    src = x.reshape(-1).view(np.uint32)
    dst = out.reshape(-1)

    def work(c):
        lo, hi = c * _CHUNK, min(src.size, (c + 1) * _CHUNK)
        u = src[lo:hi]
        r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
        dst[lo:hi] = r.astype(np.uint16)

    _parallel_chunks(src.size, work)
    return out


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 values (exact)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# random fills
# ----------------------------------------------------------------------------

def _normal(shape, seed: int, stream: tuple, scale: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1)
    nchunks = max(1, (flat.size + _CHUNK - 1) // _CHUNK)
    children = np.random.SeedSequence([seed, *stream]).spawn(nchunks)

    def work(c):
        g = np.random.Generator(np.random.PCG64(children[c]))
        lo, hi = c * _CHUNK, min(flat.size, (c + 1) * _CHUNK)
        g.standard_normal(out=flat[lo:hi], dtype=np.float32)
        if scale != 1.0:
            flat[lo:hi] *= np.float32(scale)

    _parallel_chunks(flat.size, work)
    return out


def _unit(rng: np.random.Generator, *shape) -> np.ndarray:
    v = rng.standard_normal(shape).astype(np.float64)
    v /= np.linalg.norm(v, axis=-1, keepdims=True)
    return v.astype(np.float32)


# ----------------------------------------------------------------------------
# planted structure
# ----------------------------------------------------------------------------

def _band(q, k, b, heads, G, rng):
    """Local diagonal band of 2 key blocks: q-block i aligns with key blocks i, i-1.

    Per kv head g and block c a random unit vector r[g, c].  Queries of block
    i (heads of group g) get + a_l r[g, i]; keys of block c get
    + a_l (r[g, c] + r[g, c+1]) / sqrt 2, so q.k/sqrt(d) gains about 8 nats
    for key blocks i and i-1 (a_l^2 = 8 sqrt(d) sqrt(2)).
    """
    L, _, d = q.shape
    nb = (L + b - 1) // b
    a_l = math.sqrt(8.0 * math.sqrt(d) * math.sqrt(2.0))
    idx = np.arange(L) // b
    r_all = _unit(rng, k.shape[1], nb + 1, d)
    for g in heads:
        r = r_all[g]
        rq = r[idx]
        q[:, g * G:(g + 1) * G, :] += np.float32(a_l) * rq[:, None, :]
        k[:, g, :] += np.float32(a_l / math.sqrt(2.0)) * (rq + r[idx + 1])


def _stripes(q, k, b, heads, G, rng, count=16):
    """Vertical stripes: `count` random key blocks in [1, nb-2] per kv head.

    Keys of the stripe blocks get + a_s gh (gh a unit vector per kv head) and
    the group's queries after the first stripe block get + a_s gh, so the
    stripes gain about 12 nats (a_s^2 = 12 sqrt(d)), beyond -ln(1e-4) = 9.2.
    """
    L, _, d = q.shape
    nb = (L + b - 1) // b
    if nb < 3:
        return
    a_s = np.float32(math.sqrt(12.0 * math.sqrt(d)))
    for g in heads:
        n = min(count, nb - 2)
        cs = np.sort(rng.choice(np.arange(1, nb - 1), size=n, replace=False))
        gh = _unit(rng, d)
        for c in cs:
            k[c * b:min(L, (c + 1) * b), g, :] += a_s * gh
        q[(cs[0] + 1) * b:, g * G:(g + 1) * G, :] += a_s * gh


def _llama_sequence(L, Hq, Hkv, d, b, seed, s):
    rng = np.random.default_rng([seed, s, 7])
    G = Hq // Hkv
    q = _normal((L, Hq, d), seed, (s, 0))
    k = _normal((L, Hkv, d), seed, (s, 1))
    v = _normal((L, Hkv, d), seed, (s, 2))
    _band(q, k, b, range(Hkv), G, rng)
    _stripes(q, k, b, range(Hkv), G, rng)
    k[:4] *= np.float32(4.0)  # attention sinks: first 4 keys, norm x4
    return q, k, v, {}


def _qwen_sequence(L, Hq, Hkv, d, b, seed, s):
    """Qwen3-8B-shaped mix: kv heads 0-1 band only (local), 2-5 band + stripes,
    6-7 near-dense (K ~ N(0, 0.3^2), no structure); every key then scaled by
    exp(0.5 z), z ~ N(0, 1) (log-normal key norms, sigma 0.5)."""
    assert Hkv == 8
    rng = np.random.default_rng([seed, s, 7])
    G = Hq // Hkv
    q = _normal((L, Hq, d), seed, (s, 0))
    k = _normal((L, Hkv, d), seed, (s, 1))
    v = _normal((L, Hkv, d), seed, (s, 2))
    k[:, 6:8, :] *= np.float32(0.3)
    _band(q, k, b, range(0, 6), G, rng)
    _stripes(q, k, b, range(2, 6), G, rng)
    z = _normal((L, Hkv), seed, (s, 3))
    k *= np.exp(np.float32(0.5) * z)[:, :, None]
    return q, k, v, {}


def _tiny_sequence(L, Hq, Hkv, d, b, seed, s):
    """Tiny case: N(0,1) Q/K/V, 4 planted salient key blocks and a sink block.

    Four distinct key blocks c in [1, nb-2] each pair with a random later
    q-block i > c; all keys of block c become 3 sqrt(d) times the unit mean
    query direction of q-block i (over all query heads).  Keys of block 0 get
    + 2 sqrt(d) times the unit mean of all queries (a sink block).
    """
    assert Hkv == 1
    rng = np.random.default_rng([seed, s, 7])
    nb = (L + b - 1) // b
    q = _normal((L, Hq, d), seed, (s, 0))
    k = _normal((L, Hkv, d), seed, (s, 1))
    v = _normal((L, Hkv, d), seed, (s, 2))
    cs = rng.choice(np.arange(1, nb - 1), size=4, replace=False)
    plants = []
    for c in cs:
        i = int(rng.integers(c + 1, nb))
        plants.append((int(c), i))
        m = q[i * b:min(L, (i + 1) * b)].astype(np.float64).mean(axis=(0, 1))
        u = (m / np.linalg.norm(m)).astype(np.float32)
        k[c * b:(c + 1) * b, 0, :] = np.float32(3.0 * math.sqrt(d)) * u
    m = q.astype(np.float64).mean(axis=(0, 1))
    k[0:b, 0, :] += np.float32(2.0 * math.sqrt(d)) * (m / np.linalg.norm(m)).astype(np.float32)
    return q, k, v, {"plants": plants}


def _random_sequence(L, Hq, Hkv, d, b, seed, s):
    return (_normal((L, Hq, d), seed, (s, 0)),
            _normal((L, Hkv, d), seed, (s, 1)),
            _normal((L, Hkv, d), seed, (s, 2)), {})


_STRUCTURES = {
    "llama": _llama_sequence,
    "qwen": _qwen_sequence,
    "tiny": _tiny_sequence,
    "random": _random_sequence,
}


# ----------------------------------------------------------------------------
# workload container
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    seqlens: tuple
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    page_size: int
    q: np.ndarray
    k_pages: np.ndarray
    v_pages: np.ndarray
    page_table: np.ndarray
    budgets: tuple = (0.1,)
    taus: tuple = (1e-4,)
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    @property
    def qblocks(self) -> np.ndarray:
        b = self.block_size
        return np.array([(L + b - 1) // b for L in self.seqlens], dtype=np.int32)

    @property
    def cu_qblocks(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.qblocks)]).astype(np.int32)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def total_qblocks(self) -> int:
        return int(self.qblocks.sum())

    @property
    def num_pages(self) -> int:
        return int(self.k_pages.shape[0])

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.page_table.shape[1])


def _paginate(ks, vs, Hkv, d, b_p, shuffle, seed):
    rng = np.random.default_rng([seed, 1 << 20])
    npages = [(k.shape[0] + b_p - 1) // b_p for k in ks]
    P = int(sum(npages))
    perm = rng.permutation(P) if shuffle else np.arange(P)
    table = np.full((len(ks), max(npages)), -1, dtype=np.int32)
    k_pages = np.empty((P, Hkv, b_p, d), dtype=np.uint16)
    v_pages = np.empty((P, Hkv, b_p, d), dtype=np.uint16)
    off = 0
    for s, (k, v) in enumerate(zip(ks, vs)):
        L, n = k.shape[0], npages[s]
        ids = perm[off:off + n]
        off += n
        table[s, :n] = ids
        pad = n * b_p - L
        for src, dst, sid in ((k, k_pages, 0), (v, v_pages, 1)):
            if pad:
                tail = bf16_bits(_normal((pad, Hkv, d), seed, (1 << 20, s, sid)))
                src = np.concatenate([src, tail], axis=0)
            dst[ids] = src.reshape(n, b_p, Hkv, d).transpose(0, 2, 1, 3)
    return k_pages, v_pages, table


def from_arrays(qs, ks, vs, block_size, page_size, shuffle=True, seed=0, budgets=(0.1,),
                taus=(1e-4,), name="constructed") -> Workload:
    """Workload from explicit per-sequence fp32 arrays q [L, Hq, d], k/v [L, Hkv, d].

    Values are rounded to bf16; pages are laid out as in make_custom.
    """
    Hq, d = qs[0].shape[1], qs[0].shape[2]
    Hkv = ks[0].shape[1]
    q_all = np.concatenate([bf16_bits(q) for q in qs], axis=0)
    k_pages, v_pages, table = _paginate([bf16_bits(k) for k in ks], [bf16_bits(v) for v in vs],
                                        Hkv, d, page_size, shuffle, seed)
    return Workload(name=name, seqlens=tuple(int(q.shape[0]) for q in qs), num_q_heads=Hq,
                    num_kv_heads=Hkv, head_dim=d, block_size=block_size, page_size=page_size,
                    q=q_all, k_pages=k_pages, v_pages=v_pages, page_table=table,
                    budgets=tuple(budgets), taus=tuple(taus), seed=seed,
                    meta={"structure": "constructed", "shuffled_pages": shuffle})


def make_custom(seqlens, num_q_heads, num_kv_heads, head_dim, block_size, page_size,
                structure="llama", shuffle=True, seed=0, budgets=(0.1,), taus=(1e-4,),
                name=None) -> Workload:
    """Build a workload with the given shapes and planted structure."""
    seqlens = tuple(int(L) for L in seqlens)
    gen = _STRUCTURES[structure]
    T = sum(seqlens)
    q_all = np.empty((T, num_q_heads, head_dim), dtype=np.uint16)
    ks, vs, infos = [], [], []
    off = 0
    for s, L in enumerate(seqlens):
        q, k, v, info = gen(L, num_q_heads, num_kv_heads, head_dim, block_size, seed, s)
        infos.append(info)
        q_all[off:off + L] = bf16_bits(q)
        del q
        ks.append(bf16_bits(k))
        vs.append(bf16_bits(v))
        off += L
    k_pages, v_pages, table = _paginate(ks, vs, num_kv_heads, head_dim, page_size, shuffle, seed)
    return Workload(
        name=name or f"{structure}_{'-'.join(map(str, seqlens))}",
        seqlens=seqlens, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, page_size=page_size,
        q=q_all, k_pages=k_pages, v_pages=v_pages, page_table=table,
        budgets=tuple(budgets), taus=tuple(taus), seed=seed,
        meta={"structure": structure, "shuffled_pages": shuffle, "sequences": infos})


# The five workloads: shapes of the Llama-3.1-8B / Qwen3-8B attention layers
# the pages evaluate, at 1K..128K tokens.
WORKLOADS = {
    1: dict(name="tiny_1k_d64", seqlens=(1024,), num_q_heads=2, num_kv_heads=1, head_dim=64,
            block_size=64, page_size=64, structure="tiny", shuffle=False,
            budgets=(0.25,), taus=(1e-4,)),
    2: dict(name="llama8b_32k", seqlens=(32768,), num_q_heads=32, num_kv_heads=8, head_dim=128,
            block_size=128, page_size=64, structure="llama", shuffle=False,
            budgets=(0.10,), taus=(1e-4,)),
    3: dict(name="llama8b_128k", seqlens=(131072,), num_q_heads=32, num_kv_heads=8,
            head_dim=128, block_size=128, page_size=64, structure="llama", shuffle=True,
            budgets=(0.05,), taus=(0.0, 1e-5, 1e-4, 1e-3)),
    4: dict(name="qwen8b_64k", seqlens=(65536,), num_q_heads=32, num_kv_heads=8, head_dim=128,
            block_size=128, page_size=64, structure="qwen", shuffle=True,
            budgets=(0.10,), taus=(1e-4,)),
    5: dict(name="ragged4_llama8b", seqlens=(16384, 40000, 90000, 131072), num_q_heads=32,
            num_kv_heads=8, head_dim=128, block_size=128, page_size=64, structure="llama",
            shuffle=True, budgets=(0.05, 0.10, 0.20), taus=(1e-4,)),
}


def make_workload(cfg: int, seed: int | None = None) -> Workload:
    """Workload `cfg` (1..5); the seed defaults to the workload number."""
    spec = dict(WORKLOADS[cfg])
    return make_custom(seed=cfg if seed is None else seed, **spec)
