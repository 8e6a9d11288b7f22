"""Seeded synthetic inputs and workload shapes.

This module is shared by the CPU oracle side (tests, golden-value scripts,
the bench's CPU baseline) and by the CUDA side (tests, bench).  It holds no
arithmetic of the method itself: only shapes, seeds, random draws and the
rounding of those draws to the storage dtype.

Workloads follow the five problem statements of the chunk-attention study
(LingBot-World 2.0 inference at 832x464 with 16-frame chunks = 4 latent
frames, "kaarelkaarelson.com/lingbot", setup paragraph; the 6 + 8 + 4
latent-frame slot layout of "World in World", second paragraph).

Random recipe (the pages give seeds only):
  * ``numpy.random.Generator(PCG64(seed)).standard_normal(dtype=float32)``
    rounded to bf16 with round-to-nearest-even (fp32 workloads keep fp32),
  * per chunk the draws come in the order Q, K, V, each of shape [L, H, D].
"""
from __future__ import annotations

import dataclasses
from typing import Iterator, List, Optional, Tuple

import numpy as np

# --------------------------------------------------------------------------
# dtype helpers (storage only; no method arithmetic)
# --------------------------------------------------------------------------


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return float32.

    bf16 keeps the top 16 bits of an IEEE float32.  Adding 0x7FFF plus the
    lowest kept bit and truncating gives round-to-nearest-even for finite
    inputs (the inputs here are finite normal draws).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    # finite inputs stay below 2^32 after the addition (largest: 0xFF7FFFFF + 0x8000)
    rounded = (bits + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return rounded.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float32 values (exact)."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def draw(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """One N(0,1) draw of ``shape`` stored as ``dtype`` ('bf16' or 'f32'),
    returned as float32 values (bf16 draws are bf16-exact float32)."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return x
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# workload shapes
# --------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class RopeSpec:
    """3D rotary split: ``pairs_t + pairs_h + pairs_w == head_dim // 2``."""

    grid_h: int
    grid_w: int
    pairs_t: int
    pairs_h: int
    pairs_w: int
    base: float = 10000.0


def default_rope_pairs(head_dim: int) -> Tuple[int, int, int]:
    """Pair counts (t, h, w) for a head dimension.

    h and w get floor(D/6) pairs each and t gets the rest; at D = 128 this is
    22/21/21 pairs = 44/42/42 rotary dims, the split the 832x464 workload
    states.  At D = 64 it gives 12/10/10 pairs (24/20/20 dims).
    """
    ph = head_dim // 6
    return head_dim // 2 - 2 * ph, ph, ph


@dataclasses.dataclass(frozen=True)
class RolloutSpec:
    """Chunk-wise autoregressive rollout over a sink + window cache."""

    name: str
    heads: int
    head_dim: int
    grid_h: int
    grid_w: int
    chunk_frames: int
    sinks: int
    window: int
    n_chunks: int
    dtype: str  # 'bf16' | 'f32'
    seed: int
    layers: int = 1
    steps: int = 1
    # dynamic window schedule (None = static window)
    window_seed: Optional[int] = None
    window_lo: int = 2
    window_hi: int = 8
    # causal cross-attention (text keys): env tokens + local tokens per chunk
    text_env: int = 0
    text_local: int = 0

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def chunk_tokens(self) -> int:
        return self.chunk_frames * self.tokens_per_frame

    def rope(self) -> RopeSpec:
        pt, ph, pw = default_rope_pairs(self.head_dim)
        return RopeSpec(self.grid_h, self.grid_w, pt, ph, pw, 10000.0)

    def window_schedule(self) -> List[int]:
        """Per-chunk retained window (dynamic scheduler), or the static window."""
        if self.window_seed is None:
            return [self.window] * self.n_chunks
        rng = np.random.Generator(np.random.PCG64(self.window_seed))
        return [int(w) for w in rng.integers(self.window_lo, self.window_hi + 1, self.n_chunks)]

    def frames_of_chunk(self, c: int) -> List[int]:
        return list(range(c * self.chunk_frames, (c + 1) * self.chunk_frames))


@dataclasses.dataclass(frozen=True)
class MobaSpec:
    """MoBA training sequence [C1..Cn | N1..Nn | B (n_bidir chunks)]."""

    name: str
    heads: int
    head_dim: int
    n_chunks: int
    chunk_tokens: int
    n_bidir_chunks: int
    seed: int
    dtype: str = "bf16"

    @property
    def seq_len(self) -> int:
        return (2 * self.n_chunks + self.n_bidir_chunks) * self.chunk_tokens


# The five workloads.  Names describe what they are.
TINY_F32 = RolloutSpec("tiny_rollout_f32", heads=1, head_dim=64, grid_h=4, grid_w=4,
                       chunk_frames=2, sinks=2, window=2, n_chunks=6, dtype="f32", seed=0)
VIDEO_832x464 = RolloutSpec("chunk_attn_832x464_bf16", heads=12, head_dim=128, grid_h=29,
                            grid_w=52, chunk_frames=4, sinks=6, window=8, n_chunks=40,
                            dtype="bf16", seed=1)
VIDEO_832x464_30L = RolloutSpec("chunk_attn_832x464_30layers_4steps", heads=12, head_dim=128,
                                grid_h=29, grid_w=52, chunk_frames=4, sinks=6, window=8,
                                n_chunks=10, dtype="bf16", seed=2, layers=30, steps=4)
MOBA_8x6032 = MobaSpec("moba_8chunks_x6032", heads=12, head_dim=128, n_chunks=8,
                       chunk_tokens=4 * 1508, n_bidir_chunks=8, seed=3)
VIDEO_720P_DYN = RolloutSpec("dynwin_720p_crossattn", heads=12, head_dim=128, grid_h=45,
                             grid_w=80, chunk_frames=4, sinks=6, window=8, n_chunks=60,
                             dtype="bf16", seed=4, window_seed=4, text_env=256, text_local=256)

ALL_ROLLOUTS = (TINY_F32, VIDEO_832x464, VIDEO_832x464_30L, VIDEO_720P_DYN)


def shrink(spec: RolloutSpec, **kw) -> RolloutSpec:
    """A smaller copy of a rollout workload (for tests that must finish fast)."""
    return dataclasses.replace(spec, **kw)


# --------------------------------------------------------------------------
# draws
# --------------------------------------------------------------------------


def rollout_chunks(spec: RolloutSpec, layer: int = 0) -> Iterator[dict]:
    """Yield, per chunk and denoising step, the chunk's Q, K, V ([L, H, D]).

    One generator per layer (seed + layer); within it, chunk by chunk and step
    by step, the draws are Q, K, V.  Each yielded dict has keys
    ``chunk, step, frames, q, k, v`` (float32 arrays holding dtype-exact values).
    """
    rng = np.random.Generator(np.random.PCG64(spec.seed + layer))
    shape = (spec.chunk_tokens, spec.heads, spec.head_dim)
    for c in range(spec.n_chunks):
        for s in range(spec.steps):
            q = draw(rng, shape, spec.dtype)
            k = draw(rng, shape, spec.dtype)
            v = draw(rng, shape, spec.dtype)
            yield dict(chunk=c, step=s, frames=spec.frames_of_chunk(c), q=q, k=k, v=v)


def aux_frames(spec: RolloutSpec, chunk: int, n: int, seed_offset: int = 2000):
    """Auxiliary evidence frames for one chunk: K, V ([n * T, H, D]) and n ascending
    temporal positions drawn from the frames before the chunk (retrieved history,
    source-video observations), from PCG64(seed + seed_offset + chunk)."""
    rng = np.random.Generator(np.random.PCG64(spec.seed + seed_offset + chunk))
    shape = (n * spec.tokens_per_frame, spec.heads, spec.head_dim)
    k = draw(rng, shape, spec.dtype)
    v = draw(rng, shape, spec.dtype)
    first = spec.frames_of_chunk(chunk)[0]
    pos = sorted(int(x) for x in rng.integers(0, max(first, 1), size=n))
    return k, v, pos


def text_kv(spec: RolloutSpec) -> Iterator[dict]:
    """Cross-attention inputs: the shared env prompt K/V (drawn once) and, per
    chunk, the chunk's local-prompt K/V and the chunk's cross-attention queries.

    Generator seed = seed + 1000; env K, env V first, then per chunk q, k, v.
    """
    rng = np.random.Generator(np.random.PCG64(spec.seed + 1000))
    H, D = spec.heads, spec.head_dim
    env_k = draw(rng, (spec.text_env, H, D), spec.dtype)
    env_v = draw(rng, (spec.text_env, H, D), spec.dtype)
    for c in range(spec.n_chunks):
        q = draw(rng, (spec.chunk_tokens, H, D), spec.dtype)
        k = draw(rng, (spec.text_local, H, D), spec.dtype)
        v = draw(rng, (spec.text_local, H, D), spec.dtype)
        yield dict(chunk=c, env_k=env_k, env_v=env_v, q=q, k=k, v=v)


def moba_inputs(spec: MobaSpec) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Q, K, V ([L, H, D]) of a MoBA training sequence, drawn Q, K, V."""
    rng = np.random.Generator(np.random.PCG64(spec.seed))
    shape = (spec.seq_len, spec.heads, spec.head_dim)
    return (draw(rng, shape, spec.dtype), draw(rng, shape, spec.dtype),
            draw(rng, shape, spec.dtype))


def moba_grad_output(spec: MobaSpec) -> np.ndarray:
    """Upstream gradient dO ([L, H, D]) for the MoBA backward: N(0, 1) in the
    spec's dtype, from a stream of its own (the seed's PCG64 jumped once)."""
    rng = np.random.Generator(np.random.PCG64(spec.seed).jumped(1))
    return draw(rng, (spec.seq_len, spec.heads, spec.head_dim), spec.dtype)


def sample_rows(n_rows: int, n_sample: int, seed: int, always: Optional[List[int]] = None) -> np.ndarray:
    """Sorted unique row indices: ``n_sample`` seeded random rows plus ``always``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    pick = rng.choice(n_rows, size=min(n_sample, n_rows), replace=False)
    rows = set(int(r) for r in pick)
    if always:
        rows.update(int(r) for r in always if 0 <= r < n_rows)
    return np.array(sorted(rows), dtype=np.int64)
