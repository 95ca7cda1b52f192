"""The allocation-free encode (mimi_rvq_encode_noalloc), for callers that cannot call
cudaMalloc: it takes the codebooks and W_in directly, needs no handle, and keeps its only
scratch (the codeword norms) in a static device array. It must give the same codes as the
handle's float32 full-scan entry point (mimi_rvq_encode_scan), on consecutive calls that
reuse the shared array. Collected last so that a failure here leaves the other tests run."""
import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _noalloc(lib, C, W_in, z, dtype_flag, n_q, codes):
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fn = lib.mimi_rvq_encode_noalloc
    fn.argtypes = [vp, vp, vp, ci, i64, ci, vp, vp]
    fn.restype = ci
    return fn(C.data_ptr(), W_in.data_ptr(), z.data_ptr(), dtype_flag, z.shape[0], n_q,
              codes.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_encode_matches_the_full_scan_entry_point():
    import split_residual_vector_b200 as pkg
    lib = pkg.library()
    rng = synth.generator(77)
    model = synth.make_model(rng)
    C = torch.from_numpy(model.C).cuda()
    W_in = torch.from_numpy(model.W_in).cuda()
    q = pkg.Quantizer(C, W_in, torch.from_numpy(model.W_out).cuda())
    # two calls in a row on different inputs (the second reuses the static array)
    calls = [(synth.latents(rng, 300), 8), (synth.latents(rng, 129), 5)]
    for z_np, n_q in calls:
        z = torch.from_numpy(z_np).cuda()
        got = torch.full((z.shape[0], n_q), -1, dtype=torch.int16, device="cuda")
        assert _noalloc(lib, C, W_in, z, pkg.F32, n_q, got) == 0
        ref = q.encode_scan(z, n_q=n_q)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), "no-alloc encode differs from mimi_rvq_encode_scan"
    # sizes beyond the static scratch are refused, and nothing is launched
    bad = torch.empty((4, 9), dtype=torch.int16, device="cuda")
    z = torch.from_numpy(calls[0][0][:4]).cuda()
    assert _noalloc(lib, C, W_in, z, pkg.F32, 9, bad) == -1
    assert _noalloc(lib, C, W_in, z, pkg.F32, 0, bad) == -1
    q.close()
