"""The failure path of the bounded waits, on the GPU, without hanging or faulting it: a
kernel waits on a flag that nothing sets, gives up after its (short) budget, records the
timeout, and returns; the host reads the status and the handle keeps working."""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ETIMEOUT = -6


@pytest.mark.parametrize("which", [0, 1], ids=["mbarrier", "group_barrier"])
def test_a_wait_that_never_completes_times_out_and_the_handle_recovers(which):
    import split_residual_vector_b200 as pkg
    model, frames = synth.streaming_step(64, calls=1)
    q = pkg.Quantizer(torch.from_numpy(model.C).cuda(), torch.from_numpy(model.W_in).cuda(),
                      torch.from_numpy(model.W_out).cuda())
    z = torch.from_numpy(frames[0]).cuda()
    before = q.encode_step(z).cpu().numpy()
    before_tc = q.encode(z).cpu().numpy()
    assert q.get_error() == 0
    q.wait_selftest(which)
    assert q.get_error() == ETIMEOUT          # reported once ...
    assert q.get_error() == 0                 # ... and cleared
    # both encoders (the streaming one uses the group barriers the timeout may have left
    # mid-count) still give the same codes
    assert np.array_equal(q.encode_step(z).cpu().numpy(), before)
    assert np.array_equal(q.encode(z).cpu().numpy(), before_tc)
    assert q.get_error() == 0
    with pytest.raises(pkg.MimiRVQError):
        q.wait_selftest(2)


def test_embedding_sum_wait_times_out_reports_and_recovers():
    """The embedding sum's bulk-copy wait, in its self-test form (no copy is ever issued):
    the consumers' wait runs out, the kernel records the timeout in the token-stream status
    word (no n_bad counter is involved), returns, and the next real call is exact."""
    import oracle
    import split_residual_vector_b200 as pkg
    rows = synth.moshi_rows()
    tables = synth.moshi_tables(seed=21)
    text, audio = synth.moshi_streams(40, seed=22)
    V = oracle.delay_pack(text, audio, [0, 1, 1, 1, 1, 1, 1, 1])
    tt = torch.from_numpy(tables.view(np.int16)).cuda().view(torch.bfloat16)
    tok = torch.from_numpy(np.ascontiguousarray(V)).cuda()
    before = pkg.embed_sum(tt, rows, tok, out_dtype=torch.float32).cpu().numpy()
    assert pkg.streams_get_error() == 0
    pkg.streams_wait_selftest()
    assert pkg.streams_get_error() == ETIMEOUT   # reported once ...
    assert pkg.streams_get_error() == 0          # ... and cleared
    after = pkg.embed_sum(tt, rows, tok, out_dtype=torch.float32).cpu().numpy()
    assert pkg.streams_get_error() == 0
    assert np.array_equal(after, before)
