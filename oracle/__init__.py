"""Float64 CPU oracle for the Mimi split-RVQ bottleneck -- test infrastructure.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never does, and the
two share no code: this module only marshals numpy arrays into the plain C in
``oracle.c`` (built by ``oracle/build.py``).

What it computes, and the passages it follows, is documented in ``oracle.c``:
y = W_in z (512 -> 256), a semantic plain VQ on y, a greedy 7-level acoustic
RVQ on y, codes (s, a_1..a_7); decode = W_out (S_s + sum_l A_{l,a_l}); and in
``moshi_streams.c``: the delay-pattern packing of the 17-stream frame, its
inverse, and the sum of per-stream embeddings that feeds the language model.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, library_path, sources

F32, BF16 = 0, 1
NEAR_TIE_REL = 1e-5  # gap <= 1e-5 * (1 + d_best) at some level marks a near-tie frame

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path) or os.path.getmtime(path) < max(os.path.getmtime(f)
                                                                 for f in sources()):
        build_oracle()
    lib = ctypes.CDLL(path)
    c_i64, c_int, c_vp, c_dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_double
    lib.oracle_encode.argtypes = [c_vp, c_int, c_i64, c_int, c_int, c_int, c_int, c_vp, c_vp,
                                  c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp]
    lib.oracle_encode.restype = c_int
    lib.oracle_encode_projected.argtypes = [c_vp, c_i64, c_int, c_int, c_int, c_vp, c_int, c_int,
                                            c_int, c_vp, c_vp, c_vp]
    lib.oracle_encode_projected.restype = c_int
    lib.oracle_project.argtypes = [c_vp, c_int, c_i64, c_int, c_int, c_vp, c_int, c_vp]
    lib.oracle_project.restype = c_int
    lib.oracle_decode.argtypes = [c_vp, c_i64, c_int, c_int, c_int, c_int, c_int, c_vp, c_vp,
                                  c_int, c_vp, c_vp]
    lib.oracle_decode.restype = c_int
    lib.oracle_frame_rate.argtypes = [c_dbl, c_vp, c_int]
    lib.oracle_frame_rate.restype = c_dbl
    lib.oracle_bits_per_code.argtypes = [c_i64]
    lib.oracle_bits_per_code.restype = c_int
    lib.oracle_bitrate.argtypes = [c_dbl, c_int, c_i64]
    lib.oracle_bitrate.restype = c_dbl
    lib.oracle_threads.argtypes = [c_int]
    lib.oracle_threads.restype = c_int
    lib.oracle_delay_pack.argtypes = [c_vp, c_vp, c_int, c_i64, c_int, c_vp, c_i64,
                                      ctypes.c_int32, ctypes.c_int32, c_vp]
    lib.oracle_delay_pack.restype = c_int
    lib.oracle_delay_unpack.argtypes = [c_vp, c_i64, c_int, c_int, c_int, c_vp, c_i64, c_vp]
    lib.oracle_delay_unpack.restype = c_int
    lib.oracle_delay_latency_ms.argtypes = [c_vp, c_int, c_dbl]
    lib.oracle_delay_latency_ms.restype = c_dbl
    lib.oracle_embed_sum.argtypes = [c_vp, c_int, c_int, c_vp, c_int, c_vp, c_i64, c_int, c_vp,
                                     c_vp]
    lib.oracle_embed_sum.restype = c_int
    _lib = lib
    return lib


class OracleError(RuntimeError):
    pass


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc == 2:
        raise OracleError(f"{what}: code outside [0, K)")
    if rc != 0:
        raise OracleError(f"{what}: invalid arguments (status {rc})")


def _latents(z):
    """Return (contiguous array, dtype flag). bf16 latents travel as uint16 bit patterns."""
    z = np.ascontiguousarray(z)
    if z.dtype == np.float32:
        return z, F32
    if z.dtype == np.uint16:
        return z, BF16
    raise TypeError("latents must be float32 or uint16 (bf16 bit patterns)")


def threads(nthreads: int = 0) -> int:
    """OpenMP threads the oracle uses for a request of ``nthreads`` (0 = default)."""
    return int(_load().oracle_threads(int(nthreads)))


def project(z, W_in, nthreads: int = 0) -> np.ndarray:
    """y = W_in z in float64. z [N, D_in] float32 or bf16 bits; W_in [D, D_in] float32."""
    lib = _load()
    z, dt = _latents(z)
    W_in = np.ascontiguousarray(W_in, dtype=np.float32)
    N, D_in = z.shape
    D = W_in.shape[0]
    assert W_in.shape[1] == D_in
    y = np.empty((N, D), np.float64)
    _check(lib.oracle_project(_ptr(z), dt, N, D_in, D, _ptr(W_in), nthreads, _ptr(y)), "project")
    return y


def encode(z, W_in, C, n_q: int | None = None, variant: int = 0, nthreads: int = 0,
           return_y: bool = False):
    """Encode latents. Returns (codes int16 [N, n_q], d_best [N, n_q], d_second [N, n_q]) and,
    with return_y, the float64 projection y [N, D] as a fourth item.

    C is [Q, K, D] float32 (codebook 0 semantic, 1..Q-1 acoustic levels).
    variant 0: acoustic RVQ on y; variant 1: acoustic RVQ on y - S_s.
    """
    lib = _load()
    z, dt = _latents(z)
    W_in = np.ascontiguousarray(W_in, dtype=np.float32)
    C = np.ascontiguousarray(C, dtype=np.float32)
    N, D_in = z.shape
    Q, K, D = C.shape
    assert W_in.shape == (D, D_in)
    n_q = Q if n_q is None else int(n_q)
    codes = np.empty((N, n_q), np.int16)
    db = np.empty((N, n_q), np.float64)
    ds = np.empty((N, n_q), np.float64)
    y = np.empty((N, D), np.float64) if return_y else None
    _check(lib.oracle_encode(_ptr(z), dt, N, D_in, D, K, Q, _ptr(W_in), _ptr(C), n_q, variant,
                             nthreads, _ptr(codes), _ptr(db), _ptr(ds), _ptr(y)), "encode")
    return (codes, db, ds, y) if return_y else (codes, db, ds)


def encode_projected(y, C, n_q: int | None = None, variant: int = 0, nthreads: int = 0):
    """Split RVQ of given float64 projected latents y [N, D]. Returns (codes, d_best, d_second)."""
    lib = _load()
    y = np.ascontiguousarray(y, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float32)
    N, D = y.shape
    Q, K, D2 = C.shape
    assert D == D2
    n_q = Q if n_q is None else int(n_q)
    codes = np.empty((N, n_q), np.int16)
    db = np.empty((N, n_q), np.float64)
    ds = np.empty((N, n_q), np.float64)
    _check(lib.oracle_encode_projected(_ptr(y), N, D, K, Q, _ptr(C), n_q, variant, nthreads,
                                       _ptr(codes), _ptr(db), _ptr(ds)), "encode_projected")
    return codes, db, ds


def decode(codes, C, W_out, nthreads: int = 0, return_q: bool = False):
    """x = W_out (sum of the chosen codewords), float64 [N, D_out]. codes [N, n_q] int16."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.int16)
    C = np.ascontiguousarray(C, dtype=np.float32)
    W_out = np.ascontiguousarray(W_out, dtype=np.float32)
    N, n_q = codes.shape
    Q, K, D = C.shape
    D_out = W_out.shape[0]
    assert W_out.shape[1] == D
    out = np.empty((N, D_out), np.float64)
    q = np.empty((N, D), np.float64) if return_q else None
    _check(lib.oracle_decode(_ptr(codes), N, D, K, Q, n_q, D_out, _ptr(C), _ptr(W_out),
                             nthreads, _ptr(out), _ptr(q)), "decode")
    return (out, q) if return_q else out


def near_tie(d_best, d_second, rel: float = NEAR_TIE_REL) -> np.ndarray:
    """Per-frame flag: some level's best-vs-second gap is <= rel * (1 + d_best)."""
    d_best = np.asarray(d_best)
    gap = np.asarray(d_second) - d_best
    return np.any(gap <= rel * (1.0 + d_best), axis=1)


def frame_rate(sample_rate: float, strides) -> float:
    lib = _load()
    s = np.ascontiguousarray(strides, dtype=np.int32)
    return float(lib.oracle_frame_rate(float(sample_rate), _ptr(s), len(s)))


def bits_per_code(K: int) -> int:
    return int(_load().oracle_bits_per_code(int(K)))


def bitrate(frame_rate_hz: float, Q: int, K: int) -> float:
    return float(_load().oracle_bitrate(float(frame_rate_hz), int(Q), int(K)))


# ----------------------------------------------------------------- Moshi token streams

TEXT_CARD, AUDIO_CARD = 32000, 2048
TEXT_PAD, AUDIO_PAD = TEXT_CARD, AUDIO_CARD  # pad ids: one past each vocabulary


def delay_pack(text, audio, delays, S: int | None = None, text_pad: int = TEXT_PAD,
               audio_pad: int = AUDIO_PAD) -> np.ndarray:
    """Multi-stream frame V [S, 1 + n_audio * Q] int32 from text [T] int32 (or None) and
    audio [n_audio, T, Q] int16 with per-level delays [Q]. S defaults to T + max delay."""
    lib = _load()
    audio = np.ascontiguousarray(audio, dtype=np.int16)
    n_audio, T, Q = audio.shape
    d = np.ascontiguousarray(delays, dtype=np.int32)
    assert d.shape == (Q,)
    S = T + int(d.max(initial=0)) if S is None else int(S)
    t = None if text is None else np.ascontiguousarray(text, dtype=np.int32)
    assert t is None or t.shape == (T,)
    V = np.empty((S, 1 + n_audio * Q), np.int32)
    _check(lib.oracle_delay_pack(_ptr(t), _ptr(audio), n_audio, T, Q, _ptr(d), S, text_pad,
                                 audio_pad, _ptr(V)), "delay_pack")
    return V


def delay_unpack(V, col0: int, delays, T: int | None = None) -> np.ndarray:
    """audio [T, Q] int16 from the Q columns of V starting at col0 (inverse of the shift).
    T defaults to S - max delay."""
    lib = _load()
    V = np.ascontiguousarray(V, dtype=np.int32)
    S, K = V.shape
    d = np.ascontiguousarray(delays, dtype=np.int32)
    Q = d.shape[0]
    T = S - int(d.max(initial=0)) if T is None else int(T)
    out = np.empty((T, Q), np.int16)
    _check(lib.oracle_delay_unpack(_ptr(V), S, K, col0, Q, _ptr(d), T, _ptr(out)),
           "delay_unpack")
    return out


def delay_latency_ms(delays, frame_ms: float = 80.0) -> float:
    d = np.ascontiguousarray(delays, dtype=np.int32)
    return float(_load().oracle_delay_latency_ms(_ptr(d), len(d), float(frame_ms)))


def embed_sum(tables, rows, V, nthreads: int = 0):
    """out [S, d] float64 = sum over k of row V[s, k] of table k; returns (out, n_bad).
    tables: the K tables' rows stacked [sum(rows), d], float32 or bf16 bit patterns (uint16)."""
    lib = _load()
    tables, dt = _latents(tables)
    r = np.ascontiguousarray(rows, dtype=np.int64)
    V = np.ascontiguousarray(V, dtype=np.int32)
    S, K = V.shape
    assert r.shape == (K,) and tables.shape[0] == int(r.sum())
    d = tables.shape[1]
    out = np.empty((S, d), np.float64)
    bad = np.zeros(1, np.int64)
    _check(lib.oracle_embed_sum(_ptr(tables), dt, K, _ptr(r), d, _ptr(V), S, nthreads, _ptr(out),
                                _ptr(bad)), "embed_sum")
    return out, int(bad[0])
