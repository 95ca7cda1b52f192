"""B200-native split residual vector quantiser of the Mimi codec (the tokenizer
bottleneck behind Moshi): encode 512-d latents to 8 codes per 80 ms frame
(1 semantic VQ + 7-level acoustic RVQ, 2048 codewords each) and decode them back.

This module is argument marshalling over the C ABI in ``include/mimi_rvq.h``
(``libmimi_rvq.so``, built by ``build.py``): every step of the computation runs
in the library's sm_100a kernels. PyTorch supplies device memory and streams
only. There is no fallback: if the library is missing or fails to load, using
this module raises.
"""
from __future__ import annotations

import ctypes
import os

LATENT_DIM, DIM, CODEBOOK_SIZE, NUM_CODEBOOKS = 512, 256, 2048, 8
F32, BF16 = 0, 1
STATUS = {0: "ok", -1: "invalid argument", -2: "out of device memory", -3: "CUDA error",
          -4: "code out of range", -5: "device is not sm_100", -6: "kernel wait timed out"}

LIBRARY_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmimi_rvq.so")
EXPORTS = ("mimi_rvq_create", "mimi_rvq_destroy", "mimi_rvq_encode", "mimi_rvq_encode_ex",
           "mimi_rvq_encode_step", "mimi_rvq_project", "mimi_rvq_encode_scan", "mimi_rvq_decode",
           "mimi_rvq_decode_ex", "mimi_rvq_get_error", "mimi_rvq_stats", "mimi_rvq_strerror",
           "mimi_rvq_encode_profile", "mimi_rvq_delay_pack", "mimi_rvq_delay_unpack",
           "mimi_rvq_embed_sum", "mimi_rvq_wait_selftest", "mimi_rvq_encode_step_ex",
           "mimi_rvq_encode_noalloc", "mimi_rvq_streams_get_error",
           "mimi_rvq_streams_wait_selftest")
TEXT_CARD, TEXT_PAD, AUDIO_PAD = 32000, 32000, 2048

_lib = None


class MimiRVQError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, 'unknown')} (status {status})")
        self.status = status


def library() -> ctypes.CDLL:
    """Load libmimi_rvq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY_PATH):
        raise ImportError(f"{LIBRARY_PATH} is missing: build it with "
                          "`python -m split_residual_vector_b200.build`")
    lib = ctypes.CDLL(LIBRARY_PATH)
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.mimi_rvq_create.argtypes = [vp, vp, vp, ctypes.POINTER(vp)]
    lib.mimi_rvq_create.restype = ci
    lib.mimi_rvq_destroy.argtypes = [vp]
    lib.mimi_rvq_destroy.restype = None
    lib.mimi_rvq_encode.argtypes = [vp, vp, ci, i64, vp, vp]
    lib.mimi_rvq_encode.restype = ci
    for name in ("mimi_rvq_encode_ex", "mimi_rvq_encode_scan"):
        getattr(lib, name).argtypes = [vp, vp, ci, i64, ci, ci, vp, vp]
        getattr(lib, name).restype = ci
    lib.mimi_rvq_encode_profile.argtypes = [vp, vp, ci, i64, vp, vp, vp]
    lib.mimi_rvq_encode_profile.restype = ci
    lib.mimi_rvq_project.argtypes = [vp, vp, ci, i64, vp, vp]
    lib.mimi_rvq_project.restype = ci
    lib.mimi_rvq_decode_ex.argtypes = [vp, vp, i64, ci, vp, vp]
    lib.mimi_rvq_decode_ex.restype = ci
    lib.mimi_rvq_encode_step.argtypes = [vp, vp, ci, ci, vp, vp]
    lib.mimi_rvq_encode_step.restype = ci
    lib.mimi_rvq_decode.argtypes = [vp, vp, i64, vp, vp]
    lib.mimi_rvq_decode.restype = ci
    lib.mimi_rvq_get_error.argtypes = [vp, vp]
    lib.mimi_rvq_get_error.restype = ci
    lib.mimi_rvq_stats.argtypes = [vp, vp, ctypes.POINTER(i64), ctypes.POINTER(i64)]
    lib.mimi_rvq_stats.restype = ci
    lib.mimi_rvq_strerror.argtypes = [ci]
    lib.mimi_rvq_strerror.restype = ctypes.c_char_p
    lib.mimi_rvq_encode_step_ex.argtypes = [vp, vp, ci, ci, ci, ci, vp, vp]
    lib.mimi_rvq_encode_step_ex.restype = ci
    lib.mimi_rvq_wait_selftest.argtypes = [vp, ci, vp]
    lib.mimi_rvq_wait_selftest.restype = ci
    lib.mimi_rvq_set_cluster_form.argtypes = [vp, ci]
    lib.mimi_rvq_set_cluster_form.restype = ci
    i32 = ctypes.c_int32
    lib.mimi_rvq_delay_pack.argtypes = [vp, vp, ci, i64, vp, i64, i32, i32, vp, vp]
    lib.mimi_rvq_delay_pack.restype = ci
    lib.mimi_rvq_delay_unpack.argtypes = [vp, i64, ci, ci, vp, i64, vp, vp]
    lib.mimi_rvq_delay_unpack.restype = ci
    lib.mimi_rvq_embed_sum.argtypes = [vp, ci, ci, vp, ci, vp, i64, vp, ci, vp, vp]
    lib.mimi_rvq_embed_sum.restype = ci
    lib.mimi_rvq_streams_get_error.argtypes = [vp]
    lib.mimi_rvq_streams_get_error.restype = ci
    lib.mimi_rvq_streams_wait_selftest.argtypes = [vp]
    lib.mimi_rvq_streams_wait_selftest.restype = ci
    _lib = lib
    return lib


def strerror(status: int) -> str:
    return library().mimi_rvq_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != 0:
        raise MimiRVQError(status, what)


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_flag(t):
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("latents must be float32 or bfloat16")


class Quantizer:
    """A library handle: codebooks [8, 2048, 256], W_in [256, 512], W_out [512, 256]
    (float32 CUDA tensors, copied at construction)."""

    def __init__(self, codebooks, W_in, W_out):
        import torch
        lib = library()
        cb = codebooks.detach().to(device="cuda", dtype=torch.float32).contiguous()
        wi = W_in.detach().to(device=cb.device, dtype=torch.float32).contiguous()
        wo = W_out.detach().to(device=cb.device, dtype=torch.float32).contiguous()
        assert cb.shape == (NUM_CODEBOOKS, CODEBOOK_SIZE, DIM), cb.shape
        assert wi.shape == (DIM, LATENT_DIM) and wo.shape == (LATENT_DIM, DIM)
        self.device = cb.device
        self._h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib.mimi_rvq_create(cb.data_ptr(), wi.data_ptr(), wo.data_ptr(),
                                       ctypes.byref(self._h)), "mimi_rvq_create")

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            library().mimi_rvq_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _codes_out(self, n, out, n_q=NUM_CODEBOOKS):
        import torch
        if out is None:
            out = torch.empty((n, n_q), dtype=torch.int16, device=self.device)
        assert out.dtype == torch.int16 and out.is_contiguous() and out.shape == (n, n_q)
        return out

    @staticmethod
    def _latents(latents):
        assert latents.dim() == 2 and latents.shape[1] == LATENT_DIM and latents.is_contiguous()
        return latents.shape[0], _dtype_flag(latents)

    def encode(self, latents, n_q=NUM_CODEBOOKS, variant=0, out=None, stream=None):
        """latents [N, 512] float32 / bfloat16 (CUDA) -> codes [N, n_q] int16."""
        n, dt = self._latents(latents)
        out = self._codes_out(n, out, n_q)
        if n_q == NUM_CODEBOOKS and variant == 0:
            st = library().mimi_rvq_encode(self._h, latents.data_ptr(), dt, n, out.data_ptr(),
                                           _stream(stream))
        else:
            st = library().mimi_rvq_encode_ex(self._h, latents.data_ptr(), dt, n, n_q, variant,
                                              out.data_ptr(), _stream(stream))
        _check(st, "mimi_rvq_encode")
        return out

    def encode_step(self, frames, out=None, stream=None, n_q=NUM_CODEBOOKS, variant=0):
        """frames [B, 512] (one frame per stream) -> codes [B, n_q] int16."""
        b, dt = self._latents(frames)
        out = self._codes_out(b, out, n_q)
        if n_q == NUM_CODEBOOKS and variant == 0:
            st = library().mimi_rvq_encode_step(self._h, frames.data_ptr(), dt, b, out.data_ptr(),
                                                _stream(stream))
        else:
            st = library().mimi_rvq_encode_step_ex(self._h, frames.data_ptr(), dt, b, n_q, variant,
                                                   out.data_ptr(), _stream(stream))
        _check(st, "mimi_rvq_encode_step")
        return out

    def project(self, latents, out=None, stream=None):
        """latents [N, 512] -> y = W_in z [N, 256] float32 (the encoder's projection step)."""
        import torch
        n, dt = self._latents(latents)
        if out is None:
            out = torch.empty((n, DIM), dtype=torch.float32, device=self.device)
        assert out.dtype == torch.float32 and out.is_contiguous() and out.shape == (n, DIM)
        _check(library().mimi_rvq_project(self._h, latents.data_ptr(), dt, n, out.data_ptr(),
                                          _stream(stream)), "mimi_rvq_project")
        return out

    def encode_scan(self, latents, n_q=NUM_CODEBOOKS, variant=0, out=None, stream=None):
        """Float32 full-scan encoder on CUDA cores (slow; for comparison)."""
        n, dt = self._latents(latents)
        out = self._codes_out(n, out, n_q)
        _check(library().mimi_rvq_encode_scan(self._h, latents.data_ptr(), dt, n, n_q, variant,
                                              out.data_ptr(), _stream(stream)),
               "mimi_rvq_encode_scan")
        return out

    def decode(self, codes, out=None, stream=None):
        """codes [N, n_q] int16 (CUDA) -> latents [N, 512] float32 (n_q = codes.shape[1])."""
        import torch
        assert codes.dtype == torch.int16 and codes.is_contiguous() and codes.dim() == 2
        n, n_q = codes.shape
        if out is None:
            out = torch.empty((n, LATENT_DIM), dtype=torch.float32, device=self.device)
        assert out.dtype == torch.float32 and out.is_contiguous() and out.shape == (n, LATENT_DIM)
        if n_q == NUM_CODEBOOKS:
            st = library().mimi_rvq_decode(self._h, codes.data_ptr(), n, out.data_ptr(),
                                           _stream(stream))
        else:
            st = library().mimi_rvq_decode_ex(self._h, codes.data_ptr(), n, n_q, out.data_ptr(),
                                              _stream(stream))
        _check(st, "mimi_rvq_decode")
        return out

    PROFILE_SLOTS = ("producer_wait_stage", "mma_wait_operands", "mma_wait_score_buffer",
                     "mma_wait_level_operand", "mma_wait_latents", "epi_wait_score_tile",
                     "epi_scan", "epi_pick", "epi_update", "epi_stage", "epi_barrier",
                     "cta_total", "n_chunks", "n_displaced", "n_runner_up", "n_more",
                     "pick_exchange_merge", "pick_rescore", "pick_select", "scan_drain",
                     "update_wait_operand", "update_work", "update_sync", "unused")
    PROFILE_COUNTS = ("n_chunks", "n_displaced", "n_runner_up", "n_more")

    def encode_profile(self, latents, out=None, stream=None):
        """Encode and return (codes, {role: cycles summed over CTAs}) from the kernel's
        self-profile; the PROFILE_COUNTS entries are event counts, not cycles."""
        import torch
        n, dt = self._latents(latents)
        out = self._codes_out(n, out)
        cyc = torch.zeros(len(self.PROFILE_SLOTS), dtype=torch.int64, device=self.device)
        _check(library().mimi_rvq_encode_profile(self._h, latents.data_ptr(), dt, n,
                                                 out.data_ptr(), cyc.data_ptr(), _stream(stream)),
               "mimi_rvq_encode_profile")
        vals = cyc.cpu().tolist()
        return out, dict(zip(self.PROFILE_SLOTS, vals))

    def wait_selftest(self, which: int, stream=None):
        """Launch a kernel whose wait never completes (0: mbarrier, 1: group barrier); it
        times out after ~50 ms. The next get_error() returns -6 (timed out)."""
        _check(library().mimi_rvq_wait_selftest(self._h, int(which), _stream(stream)),
               "mimi_rvq_wait_selftest")

    def set_cluster_form(self, enabled: bool):
        """Use the thread-block-cluster form of the float32 latency encoder (default where the
        device runs clusters) or the group form, for streaming steps of up to 256 frames and
        the float32 re-encode after a batch encode."""
        _check(library().mimi_rvq_set_cluster_form(self._h, 1 if enabled else 0),
               "mimi_rvq_set_cluster_form")

    def get_error(self, stream=None) -> int:
        """Synchronise the stream; return and clear the device error status (0 = ok)."""
        return int(library().mimi_rvq_get_error(self._h, _stream(stream)))

    def stats(self, stream=None):
        """(frames encoded, frames whose candidates could not be certified and were resolved in
        float32: re-encoded after a batch encode, scanned exactly in a sliced step) since create."""
        a, b = ctypes.c_int64(), ctypes.c_int64()
        _check(library().mimi_rvq_stats(self._h, _stream(stream), ctypes.byref(a),
                                        ctypes.byref(b)), "mimi_rvq_stats")
        return a.value, b.value


# ----------------------------------------------------------------- token streams


def _host_i32(values, n):
    arr = (ctypes.c_int32 * n)(*[int(v) for v in values])
    assert len(values) == n
    return arr


def delay_pack(text, audio, delays, S=None, text_pad=TEXT_PAD, audio_pad=AUDIO_PAD, out=None,
               stream=None):
    """Multi-stream sequence [S, 1 + 8 * n_audio] int32 from text [T] int32 (or None) and
    audio codes [n_audio, T, 8] int16 (CUDA), level q shifted later by delays[q] steps.
    S defaults to T + max(delays)."""
    import torch
    assert audio.dtype == torch.int16 and audio.dim() == 3 and audio.shape[2] == NUM_CODEBOOKS
    assert audio.is_contiguous()
    n_audio, T, _ = audio.shape
    S = T + max(int(v) for v in delays) if S is None else int(S)
    K = 1 + NUM_CODEBOOKS * n_audio
    if text is not None:
        assert text.dtype == torch.int32 and text.is_contiguous() and text.shape == (T,)
    if out is None:
        out = torch.empty((S, K), dtype=torch.int32, device=audio.device)
    assert out.dtype == torch.int32 and out.is_contiguous() and out.shape == (S, K)
    _check(library().mimi_rvq_delay_pack(None if text is None else text.data_ptr(),
                                         audio.data_ptr(), n_audio, T,
                                         _host_i32(delays, NUM_CODEBOOKS), S, int(text_pad),
                                         int(audio_pad), out.data_ptr(), _stream(stream)),
           "mimi_rvq_delay_pack")
    return out


def delay_unpack(packed, col0, delays, T=None, out=None, stream=None):
    """Audio codes [T, 8] int16 from the 8 columns of packed [S, K] int32 that start at col0
    (the inverse shift). T defaults to S - max(delays)."""
    import torch
    assert packed.dtype == torch.int32 and packed.dim() == 2 and packed.is_contiguous()
    S, K = packed.shape
    T = S - max(int(v) for v in delays) if T is None else int(T)
    if out is None:
        out = torch.empty((T, NUM_CODEBOOKS), dtype=torch.int16, device=packed.device)
    assert out.dtype == torch.int16 and out.is_contiguous() and out.shape == (T, NUM_CODEBOOKS)
    _check(library().mimi_rvq_delay_unpack(packed.data_ptr(), S, K, int(col0),
                                           _host_i32(delays, NUM_CODEBOOKS), T, out.data_ptr(),
                                           _stream(stream)), "mimi_rvq_delay_unpack")
    return out


def embed_sum(tables, rows, tokens, out_dtype=None, out=None, n_bad=None, stream=None):
    """out [S, d] = sum over k of row tokens[s, k] of table k. tables: stacked rows
    [sum(rows), d] float32 / bfloat16 (CUDA); rows: the K row counts; tokens [S, K] int32.
    n_bad: optional CUDA int64 [1] (caller-zeroed) counting tokens past their table."""
    import torch
    assert tables.dim() == 2 and tables.is_contiguous()
    assert tokens.dtype == torch.int32 and tokens.dim() == 2 and tokens.is_contiguous()
    S, K = tokens.shape
    d = tables.shape[1]
    assert len(rows) == K and sum(int(r) for r in rows) == tables.shape[0]
    if out is None:
        out = torch.empty((S, d), dtype=out_dtype or tables.dtype, device=tables.device)
    assert out.is_contiguous() and out.shape == (S, d)
    host_rows = (ctypes.c_int64 * K)(*[int(r) for r in rows])
    _check(library().mimi_rvq_embed_sum(tables.data_ptr(), _dtype_flag(tables), K, host_rows, d,
                                        tokens.data_ptr(), S, out.data_ptr(), _dtype_flag(out),
                                        None if n_bad is None else n_bad.data_ptr(),
                                        _stream(stream)), "mimi_rvq_embed_sum")
    return out


def streams_get_error(stream=None) -> int:
    """Synchronise the stream; return and clear the token-stream status word (0 = ok, -6 =
    a wait of embed_sum timed out)."""
    return int(library().mimi_rvq_streams_get_error(_stream(stream)))


def streams_wait_selftest(stream=None):
    """Launch the embedding-sum kernel in its self-test form: its wait never completes and
    times out after ~50 ms; the next streams_get_error() returns -6."""
    _check(library().mimi_rvq_streams_wait_selftest(_stream(stream)),
           "mimi_rvq_streams_wait_selftest")
