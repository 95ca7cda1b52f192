"""The allocation-free encode (mimi_rvq_encode_noalloc), for callers that cannot call
cudaMalloc: it takes the codebooks and W_in directly, needs no handle, and keeps its only
scratch (the codeword norms) in a static device array. It must give the same codes as the
handle's float32 full-scan entry point (mimi_rvq_encode_scan), on consecutive calls that
reuse the shared array, for float32 and bf16 latents, and it must not allocate device
memory. Collected last so that a failure here leaves the other tests run."""
import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _noalloc(lib, C, W_in, z, dtype_flag, n_q, codes, n=None):
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fn = lib.mimi_rvq_encode_noalloc
    fn.argtypes = [vp, vp, vp, ci, i64, ci, vp, vp]
    fn.restype = ci
    return fn(C.data_ptr(), W_in.data_ptr(), z.data_ptr(), dtype_flag,
              z.shape[0] if n is None else n, n_q, codes.data_ptr(),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.fixture(scope="module")
def setup():
    import split_residual_vector_b200 as pkg
    rng = synth.generator(77)
    model = synth.make_model(rng)
    C = torch.from_numpy(model.C).cuda()
    W_in = torch.from_numpy(model.W_in).cuda()
    q = pkg.Quantizer(C, W_in, torch.from_numpy(model.W_out).cuda())
    yield pkg, pkg.library(), rng, C, W_in, q
    q.close()


def test_noalloc_encode_matches_the_full_scan_entry_point(setup):
    pkg, lib, rng, C, W_in, q = setup
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


def test_noalloc_bf16_latents_at_a_two_byte_offset(setup):
    """bf16 latents (odd N) read from a slice that starts 2 bytes into a buffer, codes
    written to a slice 2 bytes in: both legal for this call; the codebooks still need 16."""
    pkg, lib, rng, C, W_in, q = setup
    bits = synth.to_bf16_bits(synth.latents(rng, 131))
    buf = torch.from_numpy(np.concatenate([np.zeros(1, np.uint16), bits.reshape(-1)])
                           .view(np.int16)).cuda().view(torch.bfloat16)
    z_off = buf[1:].view(131, 512)                   # data_ptr 2 bytes past an aligned one
    assert z_off.data_ptr() % 16 == 2
    z = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    codes_buf = torch.full((131 * 8 + 1,), -1, dtype=torch.int16, device="cuda")
    got = codes_buf[1:].view(131, 8)
    assert _noalloc(lib, C, W_in, z_off, pkg.BF16, 8, got) == 0
    ref = q.encode_scan(z)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    C_off = torch.empty(C.numel() + 1, dtype=torch.float32, device="cuda")[1:].view(C.shape)
    assert _noalloc(lib, C_off, W_in, z, pkg.BF16, 8, got) == -1


def test_noalloc_allocates_no_device_memory(setup):
    """After a warm-up call, calls on a new N and n_q leave the device's free memory as it
    was: the entry point allocates nothing."""
    pkg, lib, rng, C, W_in, q = setup
    z = torch.from_numpy(synth.latents(rng, 513)).cuda()
    out = torch.empty((513, 8), dtype=torch.int16, device="cuda")
    assert _noalloc(lib, C, W_in, z, pkg.F32, 8, out) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert _noalloc(lib, C, W_in, z, pkg.F32, 3, out, n=257) == 0
    assert _noalloc(lib, C, W_in, z, pkg.F32, 8, out, n=513) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
