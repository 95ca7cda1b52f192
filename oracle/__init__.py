"""Float64 CPU oracle for the Mimi split-RVQ bottleneck -- test infrastructure.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never does, and the
two share no code: this module only marshals numpy arrays into the plain C in
``oracle.c`` (built by ``oracle/build.py``).

What it computes, and the passages it follows, is documented in ``oracle.c``:
y = W_in z (512 -> 256), a semantic plain VQ on y, a greedy 7-level acoustic
RVQ on y, codes (s, a_1..a_7); decode = W_out (S_s + sum_l A_{l,a_l}).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, library_path

F32, BF16 = 0, 1
NEAR_TIE_REL = 1e-5  # gap <= 1e-5 * (1 + d_best) at some level marks a near-tie frame

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    src = os.path.join(os.path.dirname(__file__), "oracle.c")
    if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(src):
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
