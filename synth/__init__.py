"""Seeded synthetic inputs for the quantized paged-KV attention workloads.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark.  It holds none of the attention method's arithmetic: it only draws
fp32 keys, values and queries, picks outlier channels, needle blocks and page
permutations, and rounds queries to bf16 where a workload asks for bf16 input.
Quantisation, attention, block scoring and selection are implemented twice,
independently: in ``oracle/`` (float64 CPU) and in the CUDA library.

Shapes follow the model geometry printed on the Vulkan speculative-decoding
report (lcz.me/topic/1398, section "model structure"): 16 full-attention layers,
4 KV heads, key/value length 256, i.e. 16,384 K (or V) elements per token; the
query-head count 24 (GQA group 6) comes from the workload definitions.

Two generators exist:

* ``np_rng`` (numpy PCG64) for every case the oracle evaluates in full;
* ``torch_normal`` (torch Philox on the target device) for the multi-GB caches
  of the long-context workloads.  When the oracle checks a sample of such a
  workload, the test regenerates the sampled slice with the same seed and copies
  the generator's own output to the host; nothing the CUDA library computes is
  ever fed to the oracle.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

PAGE_TOKENS = 128
HEAD_DIM = 256

# --------------------------------------------------------------------------
# seeds and numpy draws
# --------------------------------------------------------------------------


def np_rng(seed: int, *stream: int) -> np.random.Generator:
    """A numpy PCG64 generator for (seed, *stream); streams keep draws apart."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, stream)])))


def derived_seed(seed: int, *stream: int) -> int:
    """A 63-bit integer seed for torch generators, derived from (seed, *stream)."""
    ss = np.random.SeedSequence([int(seed), *map(int, stream)])
    return int(ss.generate_state(2, dtype=np.uint32).astype(np.uint64).view(np.uint64)[0] & ((1 << 63) - 1))


def normal_f32(rng: np.random.Generator, shape) -> np.ndarray:
    """Standard normal fp32 draws."""
    return rng.standard_normal(shape, dtype=np.float32)


def outlier_channels(rng: np.random.Generator, dim: int = HEAD_DIM, frac: float = 0.01) -> np.ndarray:
    """Sorted channel indices that carry outliers: round(frac * dim) distinct channels."""
    n = int(round(frac * dim))
    return np.sort(rng.choice(dim, size=n, replace=False)).astype(np.int64)


def page_permutation(rng: np.random.Generator, n_pages: int) -> np.ndarray:
    """A random permutation of physical page ids 0..n_pages-1 (int32)."""
    return rng.permutation(n_pages).astype(np.int32)


def needle_blocks(rng: np.random.Generator, n_candidates: int, count: int) -> np.ndarray:
    """Sorted indices of `count` distinct blocks drawn from [0, n_candidates)."""
    return np.sort(rng.choice(n_candidates, size=count, replace=False)).astype(np.int64)


def plant_needles(k: np.ndarray, blocks, direction: np.ndarray, rng: np.random.Generator,
                  cosine: float = 0.9, page_tokens: int = PAGE_TOKENS) -> None:
    """Rotate every key of the given blocks so its cosine with `direction` is `cosine`.

    k: [T][D] fp32 keys of one (layer, KV head), modified in place.  Each key keeps
    its norm; its new direction is cosine * u + sqrt(1 - cosine^2) * w, with u the
    unit `direction` and w a fresh random unit vector orthogonal to u.
    """
    u = np.asarray(direction, dtype=np.float64)
    u = u / np.linalg.norm(u)
    s = math.sqrt(1.0 - cosine * cosine)
    for b in blocks:
        rows = slice(int(b) * page_tokens, (int(b) + 1) * page_tokens)
        kb = k[rows].astype(np.float64)
        norms = np.linalg.norm(kb, axis=1, keepdims=True)
        w = rng.standard_normal(kb.shape)
        w -= (w @ u)[:, None] * u[None, :]
        w /= np.linalg.norm(w, axis=1, keepdims=True)
        k[rows] = (norms * (cosine * u[None, :] + s * w)).astype(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returned as fp32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(np.shape(x))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The uint16 bit patterns of fp32 values that are exactly representable in bf16."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "values must already be bf16-representable"
    return (b >> 16).astype(np.uint16)


# --------------------------------------------------------------------------
# torch draws for multi-GB caches (device side)
# --------------------------------------------------------------------------


def torch_normal(seed: int, shape, device, dtype=None):
    """Standard normal draws from a torch Philox generator seeded with `seed`."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, device=device, dtype=dtype or torch.float32)


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic workload (no arithmetic of the method)."""

    name: str
    layers: int
    kv_heads: int
    q_heads: int
    context: int            # prior tokens in the cache when the step starts
    n_q: int                # query tokens per step (1 decode, 4 verify, chunk for prefill)
    k_fmt: str = "q8_0"
    v_fmt: str = "q4_0"
    outlier_frac: float = 0.0
    needles: int = 0
    budget_blocks: int = 0
    recent_blocks: int = 0
    ubatch: int = 0
    kv_split_tokens: int = 0
    steps: int = 1
    seed: int = 0

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads


WORKLOADS = {
    # 1 layer x 1 KV head x 6 query heads, 4,096 tokens in 32 shuffled pages, 1 query.
    "tiny": Workload("tiny", layers=1, kv_heads=1, q_heads=6, context=4096, n_q=1, seed=1001),
    # 16 x 4 x 256, 24 query heads, 131,072 tokens, 1% x8 outlier channels.
    "decode131k": Workload("decode131k", layers=16, kv_heads=4, q_heads=24, context=131072, n_q=1,
                           outlier_frac=0.01, seed=2002),
    "decode131k_q8q8": Workload("decode131k_q8q8", layers=16, kv_heads=4, q_heads=24, context=131072,
                                n_q=1, v_fmt="q8_0", outlier_frac=0.01, seed=2003),
    "decode131k_q4q4": Workload("decode131k_q4q4", layers=16, kv_heads=4, q_heads=24, context=131072,
                                n_q=1, k_fmt="q4_0", v_fmt="q4_0", outlier_frac=0.01, seed=2004),
    "decode131k_q51q4": Workload("decode131k_q51q4", layers=16, kv_heads=4, q_heads=24, context=131072,
                                 n_q=1, k_fmt="q5_1", v_fmt="q4_0", outlier_frac=0.01, seed=2005),
    # Q8_0 values under 4- and 5-bit keys, and the Q5_0 K / Q4_1 V cache of the MTP tuning notes.
    "decode131k_q4q8": Workload("decode131k_q4q8", layers=16, kv_heads=4, q_heads=24, context=131072,
                                n_q=1, k_fmt="q4_0", v_fmt="q8_0", outlier_frac=0.01, seed=2006),
    "decode131k_q51q8": Workload("decode131k_q51q8", layers=16, kv_heads=4, q_heads=24, context=131072,
                                 n_q=1, k_fmt="q5_1", v_fmt="q8_0", outlier_frac=0.01, seed=2007),
    "decode131k_q50q41": Workload("decode131k_q50q41", layers=16, kv_heads=4, q_heads=24, context=131072,
                                  n_q=1, k_fmt="q5_0", v_fmt="q4_1", outlier_frac=0.01, seed=2008),
    # 262,144 prior tokens, 4 verify tokens, 20 needles, budget 256 + recent 128 blocks.
    "verify262k": Workload("verify262k", layers=16, kv_heads=4, q_heads=24, context=262144, n_q=4,
                           needles=20, budget_blocks=256, recent_blocks=128, seed=3003),
    # 2,048-token bf16 chunk (4 ubatches of 512) over 524,288 prior tokens, 4,096-token KV splits.
    "prefill524k": Workload("prefill524k", layers=16, kv_heads=4, q_heads=24, context=524288, n_q=2048,
                            ubatch=512, kv_split_tokens=4096, seed=4004),
    # the same prefill over the other format pairs that chunked prefill takes
    "prefill524k_q4q4": Workload("prefill524k_q4q4", layers=16, kv_heads=4, q_heads=24, context=524288,
                                 n_q=2048, k_fmt="q4_0", ubatch=512, kv_split_tokens=4096, seed=4005),
    "prefill524k_q51q4": Workload("prefill524k_q51q4", layers=16, kv_heads=4, q_heads=24, context=524288,
                                  n_q=2048, k_fmt="q5_1", ubatch=512, kv_split_tokens=4096, seed=4006),
    "prefill524k_q50q41": Workload("prefill524k_q50q41", layers=16, kv_heads=4, q_heads=24, context=524288,
                                   n_q=2048, k_fmt="q5_0", v_fmt="q4_1", ubatch=512, kv_split_tokens=4096,
                                   seed=4007),
    "prefill524k_q8q8": Workload("prefill524k_q8q8", layers=16, kv_heads=4, q_heads=24, context=524288,
                                 n_q=2048, v_fmt="q8_0", ubatch=512, kv_split_tokens=4096, seed=4008),
    # 524,288 tokens in pinned host RAM, 256-block working set per (layer, head), 512 steps.
    "stream524k": Workload("stream524k", layers=16, kv_heads=4, q_heads=24, context=524288, n_q=1,
                           budget_blocks=256, recent_blocks=0, steps=512, seed=5005),
}


def plant_needles_torch(k, blocks, direction, seed: int, cosine: float = 0.9, page_tokens: int = PAGE_TOKENS):
    """Device version of plant_needles for multi-GB caches.

    k: torch fp32 [T][D] view of one (layer, KV head) (modified in place); blocks: iterable of
    block indices; direction: torch [D].  Random orthogonal parts come from torch_normal(seed)."""
    import torch

    u = direction.to(torch.float64)
    u = u / torch.linalg.norm(u)
    s = math.sqrt(1.0 - cosine * cosine)
    idx = torch.as_tensor([int(b) for b in blocks], device=k.device, dtype=torch.int64)
    rows = (idx[:, None] * page_tokens + torch.arange(page_tokens, device=k.device)[None, :]).reshape(-1)
    kb = k[rows].to(torch.float64)
    norms = torch.linalg.norm(kb, dim=1, keepdim=True)
    w = torch_normal(seed, kb.shape, k.device, torch.float64)
    w = w - (w @ u)[:, None] * u[None, :]
    w = w / torch.linalg.norm(w, dim=1, keepdim=True)
    k[rows] = (norms * (cosine * u[None, :] + s * w)).to(torch.float32)


def workload_layer_kv(w: Workload, layer: int, tokens: int, device, q=None):
    """K and V of one layer of a workload, fp32 torch [tokens][kv_heads][D] on `device`.

    Draws come from torch_normal with per-layer seeds; the workload's outlier channels are
    scaled x8 in K and V; with needles, every KV head gets w.needles seeded older blocks
    planted towards the summed last-token query of its group (q: [n_q][q_heads][D] of this
    layer).  Returns (k, v, needles) with needles {kv_head: sorted block indices}."""
    import torch

    H = w.kv_heads
    k = torch_normal(derived_seed(w.seed, 10, layer), (tokens, H, HEAD_DIM), device)
    v = torch_normal(derived_seed(w.seed, 11, layer), (tokens, H, HEAD_DIM), device)
    if w.outlier_frac:
        n_out = int(round(w.outlier_frac * HEAD_DIM))
        for h in range(H):
            ch = torch.from_numpy(np_rng(w.seed, 12, layer, h).choice(HEAD_DIM, n_out, replace=False)).to(device)
            k[:, h, ch] *= 8.0
            v[:, h, ch] *= 8.0
    needles = {}
    if w.needles:
        n_full = tokens // PAGE_TOKENS
        g = w.group
        for h in range(H):
            blocks = np.sort(np_rng(w.seed, 13, layer, h).choice(n_full - w.recent_blocks, w.needles, replace=False))
            needles[h] = blocks
            direction = q[-1, h * g:(h + 1) * g].to(torch.float64).sum(0)
            kh = k[:, h].contiguous()
            plant_needles_torch(kh, blocks, direction, derived_seed(w.seed, 14, layer, h))
            k[:, h] = kh
    return k, v, needles
