"""Seeded synthetic inputs for the split-RVQ workloads.

This module holds no arithmetic of the method: it only draws random numbers
(numpy PCG64, fixed seeds), converts float32 to bf16 bit patterns, and builds
planted latents. Both the CUDA path (tests, bench) and the float64 oracle are
fed from here; neither side imports the other.

Workloads (sizes of the Mimi quantiser: latent 512, projection 256, 8 codebooks
of 2048, codebook 0 semantic, 1..7 acoustic):

* ``pr1_reference``   -- 1 stream x 250 frames, fp32 latents, 5 % planted frames;
* ``offline_batch``   -- 64 streams x 3750 frames = 240 000 fp32 frames;
* ``streaming_step``  -- B concurrent streams, one fp32 frame each, 1000 calls;
* ``bulk_tokenization`` -- 1 048 576 bf16 frames, encode only;
* ``decode_heavy``    -- 1 048 576 frames of codes (semantic uniform, acoustic Zipf(1.1)).
* ``moshi_input``     -- the language model's side of the codec: text tokens and two audio
  code streams (Moshi, user) of T frames, and 17 embedding tables (text 32 000 + 1 rows,
  16 audio tables of 2048 + 1 rows; the extra row is the pad token), d = 4096, bf16.

Generation recipe: W_in ~ N(0, 1/512) [256, 512]; W_out ~ N(0, 1/256) [512, 256];
S ~ N(0, 1) [2048, 256]; A_l ~ N(0, 0.5^(2l)) [2048, 256] for l = 1..7; latents
z ~ N(0, 1); drawn in that order from one generator seeded with the workload's
index (0..4).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

D_IN, D, K, Q = 512, 256, 2048, 8


@dataclass
class Model:
    W_in: np.ndarray   # [D, D_in] float32
    W_out: np.ndarray  # [D_in, D] float32
    C: np.ndarray      # [Q, K, D] float32; 0 = semantic, 1..Q-1 = acoustic levels


def generator(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def make_model(rng: np.random.Generator, d_in: int = D_IN, d: int = D, k: int = K,
               q: int = Q) -> Model:
    W_in = normal(rng, (d, d_in), (1.0 / d_in) ** 0.5)
    W_out = normal(rng, (d_in, d), (1.0 / d) ** 0.5)
    C = np.empty((q, k, d), np.float32)
    C[0] = normal(rng, (k, d))
    for level in range(1, q):
        C[level] = normal(rng, (k, d), 0.5 ** level)
    return Model(W_in, W_out, C)


def to_bf16_bits(x: np.ndarray, chunk: int = 1 << 24) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even. Finite inputs only."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1)
    out = np.empty(flat.shape, np.uint16)
    for s in range(0, flat.size, chunk):
        u = flat[s:s + chunk].view(np.uint32)
        bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
        out[s:s + chunk] = ((u + bias) >> 16).astype(np.uint16)
    return out.reshape(x.shape)


def from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def latents(rng: np.random.Generator, n: int, dtype: str = "f32", d_in: int = D_IN) -> np.ndarray:
    z = normal(rng, (n, d_in))
    return to_bf16_bits(z) if dtype == "bf16" else z


def zipf_codes(rng: np.random.Generator, shape, s: float = 1.1, k: int = K) -> np.ndarray:
    """Indices in [0, k) with P(i) proportional to (i + 1)^-s (rank 1 is index 0)."""
    p = np.arange(1, k + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    u = rng.random(shape)
    return np.minimum(np.searchsorted(cdf, u, side="right"), k - 1).astype(np.int16)


# ---------------------------------------------------------------- workloads


@dataclass
class Encode:
    model: Model
    z: np.ndarray                 # [N, D_in] float32, or uint16 bf16 bits
    dtype: str                    # "f32" | "bf16"
    planted: dict | None = None   # frame index -> ("acoustic"|"semantic", codes)


def plant_latent(model: Model, codes_by_level: dict) -> np.ndarray:
    """A float32 latent whose projection is (to fp32 rounding) the sum of the given codewords.

    y = sum_l C[l][code_l] is built in float64 and mapped back through the
    Moore-Penrose inverse of W_in (W_in has full row rank, so W_in pinv(W_in) = I).
    """
    y = np.zeros(model.C.shape[2], np.float64)
    for level, code in codes_by_level.items():
        y += model.C[level, code].astype(np.float64)
    pinv = np.linalg.pinv(model.W_in.astype(np.float64))
    return (pinv @ y).astype(np.float32)


def pr1_reference(n: int = 250, plant_frac: float = 0.05, accept=None, seed: int = 0) -> Encode:
    """250 fp32 frames with floor(5 %) planted frames, half acoustic plants
    (y = sum of one codeword per acoustic level 1..7) and half semantic plants
    (y = one semantic codeword). ``accept(z_row, kind, codes) -> bool`` may
    reject a draw (the tests use it to demand well-separated plants)."""
    rng = generator(seed)
    model = make_model(rng)
    z = latents(rng, n)
    n_plant = int(np.floor(plant_frac * n))
    where = np.sort(rng.choice(n, size=n_plant, replace=False))
    planted = {}
    q, k = model.C.shape[0], model.C.shape[1]
    for j, f in enumerate(where):
        kind = "acoustic" if j < n_plant - n_plant // 2 else "semantic"
        for _attempt in range(100):
            if kind == "acoustic":
                codes = {lvl: int(rng.integers(k)) for lvl in range(1, q)}
            else:
                codes = {0: int(rng.integers(k))}
            row = plant_latent(model, codes)
            if accept is None or accept(row, kind, codes):
                break
        else:
            raise RuntimeError("could not draw a well-separated plant")
        z[f] = row
        planted[int(f)] = (kind, codes)
    return Encode(model, z, "f32", planted)


def offline_batch(n: int = 240_000, seed: int = 1) -> Encode:
    rng = generator(seed)
    model = make_model(rng)
    return Encode(model, latents(rng, n), "f32")


def streaming_step(batch: int, calls: int = 1000, seed: int = 2):
    """Model and per-call latents [calls, batch, D_in] float32."""
    rng = generator(seed)
    model = make_model(rng)
    return model, normal(rng, (calls, batch, D_IN))


def bulk_tokenization(n: int = 1 << 20, seed: int = 3) -> Encode:
    rng = generator(seed)
    model = make_model(rng)
    return Encode(model, latents(rng, n, "bf16"), "bf16")


def decode_heavy(n: int = 1 << 20, seed: int = 4):
    """Model and codes [n, 8] int16: column 0 uniform on [0, 2048), 1..7 Zipf(1.1)."""
    rng = generator(seed)
    model = make_model(rng)
    codes = np.empty((n, Q), np.int16)
    codes[:, 0] = rng.integers(0, K, size=n).astype(np.int16)
    codes[:, 1:] = zipf_codes(rng, (n, Q - 1))
    return model, codes


TEXT_CARD, AUDIO_CARD, MOSHI_DIM = 32000, 2048, 4096


def moshi_streams(T: int, seed: int = 5, n_audio: int = 2):
    """text [T] int32 uniform on [0, 32000); audio [n_audio, T, 8] int16 with level 0
    uniform on [0, 2048) and levels 1..7 Zipf(1.1) (the decode-heavy code statistics)."""
    rng = generator(seed)
    text = rng.integers(0, TEXT_CARD, size=T).astype(np.int32)
    audio = np.empty((n_audio, T, Q), np.int16)
    for a in range(n_audio):
        audio[a, :, 0] = rng.integers(0, K, size=T).astype(np.int16)
        audio[a, :, 1:] = zipf_codes(rng, (T, Q - 1))
    return text, audio


def moshi_rows(n_audio: int = 2):
    """Row counts of the stacked embedding tables: text, then n_audio x 8 audio tables."""
    return [TEXT_CARD + 1] + [AUDIO_CARD + 1] * (n_audio * Q)


def moshi_tables(d: int = MOSHI_DIM, seed: int = 6, n_audio: int = 2, rows=None) -> np.ndarray:
    """Stacked embedding tables [sum(rows), d] as bf16 bit patterns, entries N(0, 1)."""
    rng = generator(seed)
    rows = moshi_rows(n_audio) if rows is None else rows
    out = np.empty((int(sum(rows)), d), np.uint16)
    step = max(1, (1 << 24) // d)
    for r0 in range(0, out.shape[0], step):
        r1 = min(out.shape[0], r0 + step)
        out[r0:r1] = to_bf16_bits(normal(rng, (r1 - r0, d)))
    return out
