"""GPU parity of the decode path (gather-sum of W_out . c rows) against the float64 oracle."""
import numpy as np
import pytest

import oracle
import synth
from parity import DECODE_TOL, assert_codes_match, decode_error

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def quantizer(model):
    import split_residual_vector_b200 as pkg
    return pkg.Quantizer(torch.from_numpy(model.C).cuda(), torch.from_numpy(model.W_in).cuda(),
                         torch.from_numpy(model.W_out).cuda())


@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000])
def test_decode_small(n):
    model, codes = synth.decode_heavy(n=n, seed=40 + n)
    q = quantizer(model)
    out = q.decode(torch.from_numpy(codes).cuda()).cpu().numpy()
    assert q.get_error() == 0
    ref = oracle.decode(codes, model.C, model.W_out)
    assert decode_error(out, ref) <= DECODE_TOL


def test_decode_heavy_full_size_sampled():
    """1 048 576 frames (semantic uniform, acoustic Zipf(1.1)) in one call; 2000 sampled rows
    (including the last ones) against the oracle."""
    model, codes = synth.decode_heavy()
    q = quantizer(model)
    out = q.decode(torch.from_numpy(codes).cuda())
    assert q.get_error() == 0
    rng = np.random.default_rng(3)
    idx = np.unique(np.concatenate([rng.choice(len(codes), 1990, replace=False),
                                    np.arange(len(codes) - 10, len(codes))]))
    sample = out[torch.from_numpy(idx).cuda()].cpu().numpy()
    ref = oracle.decode(codes[idx], model.C, model.W_out)
    err = decode_error(sample, ref)
    print("decode_heavy max-abs/RMS", err)
    assert err <= DECODE_TOL


def test_out_of_range_codes_are_clamped_and_reported():
    model, codes = synth.decode_heavy(n=16, seed=9)
    q = quantizer(model)
    bad = codes.copy()
    bad[3, 2] = 2048
    bad[5, 0] = -7
    out = q.decode(torch.from_numpy(bad).cuda()).cpu().numpy()
    assert q.get_error() == -4
    assert q.get_error() == 0  # the flag is cleared once read
    clamped = np.clip(bad, 0, 2047)
    ref = oracle.decode(clamped, model.C, model.W_out)
    assert decode_error(out, ref) <= DECODE_TOL


def test_encode_then_decode_round_trip():
    """decode(encode(z)) equals W_out applied to the sum of the chosen codewords."""
    work = synth.offline_batch(n=500, seed=12)
    q = quantizer(work.model)
    z = torch.from_numpy(work.z).cuda()
    codes = q.encode(z)
    out = q.decode(codes).cpu().numpy()
    codes = codes.cpu().numpy()
    ref_codes, db, ds = oracle.encode(work.z, work.model.W_in, work.model.C)
    assert_codes_match(codes, ref_codes, db, ds, "round trip")
    ref = oracle.decode(codes, work.model.C, work.model.W_out)
    assert decode_error(out, ref) <= DECODE_TOL


@pytest.mark.parametrize("n_q", [1, 3, 8])
def test_decode_fewer_codebooks(n_q):
    model, codes = synth.decode_heavy(n=300, seed=50)
    codes = np.ascontiguousarray(codes[:, :n_q])
    q = quantizer(model)
    out = q.decode(torch.from_numpy(codes).cuda()).cpu().numpy()
    ref = oracle.decode(codes, model.C, model.W_out)
    assert decode_error(out, ref) <= DECODE_TOL
