"""GPU parity of the token-stream kernels (delay-pattern packing, its inverse, the
per-stream embedding sum) against the float64 oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

PATTERNS = {"staircase": [0, 1, 2, 3, 4, 5, 6, 7], "tau2": [0, 2, 2, 2, 2, 2, 2, 2],
            "tau1": [0, 1, 1, 1, 1, 1, 1, 1], "none": [0] * 8, "ragged": [3, 0, 5, 1, 0, 2, 7, 4]}


def pkg():
    import split_residual_vector_b200 as p
    return p


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("name", list(PATTERNS))
@pytest.mark.parametrize("n_audio,with_text", [(2, True), (1, True), (2, False), (0, True)])
def test_delay_pack_matches_oracle(name, n_audio, with_text):
    d = PATTERNS[name]
    text, audio = synth.moshi_streams(1000, seed=11, n_audio=max(n_audio, 1))
    audio = audio[:n_audio]
    T = 1000
    for S in (T + max(d), 17, T, T + 40):
        want = oracle.delay_pack(text if with_text else None, audio.reshape(n_audio, T, 8), d, S=S)
        got = pkg().delay_pack(dev(text) if with_text else None,
                               dev(audio.reshape(n_audio, T, 8)), d, S=S).cpu().numpy()
        assert np.array_equal(got, want), (name, S)


@pytest.mark.parametrize("name", list(PATTERNS))
def test_delay_unpack_matches_oracle_and_inverts_pack(name):
    d = PATTERNS[name]
    text, audio = synth.moshi_streams(777, seed=12)
    packed = pkg().delay_pack(dev(text), dev(audio), d)
    for a, col0 in ((0, 1), (1, 9)):
        got = pkg().delay_unpack(packed, col0, d).cpu().numpy()
        assert np.array_equal(got, oracle.delay_unpack(packed.cpu().numpy(), col0, d))
        assert np.array_equal(got, audio[a])


def test_token_stream_argument_errors():
    p = pkg()
    text, audio = synth.moshi_streams(10, seed=13)
    with pytest.raises(p.MimiRVQError):
        p.delay_pack(dev(text), dev(audio), [0, -1, 1, 1, 1, 1, 1, 1])
    packed = p.delay_pack(dev(text), dev(audio), PATTERNS["tau2"])
    with pytest.raises(p.MimiRVQError):
        p.delay_unpack(packed, 1, PATTERNS["staircase"], T=10)   # 10 + 7 > 12 steps
    with pytest.raises(p.MimiRVQError):
        p.delay_unpack(packed, 10, PATTERNS["tau2"])             # columns 10..17 > K = 17
    tables = torch.zeros((10, 12), dtype=torch.float32, device="cuda")  # d not a multiple of 8
    with pytest.raises(p.MimiRVQError):
        p.embed_sum(tables, [10], torch.zeros((3, 1), dtype=torch.int32, device="cuda"))


def _closed_form_tables(rows, d):
    blocks = []
    for k, n in enumerate(rows):
        r = np.arange(n)[:, None]
        i = np.arange(d)[None, :]
        blocks.append((64 * k + (r % 64) + (i % 16) / 16.0).astype(np.float32))
    return np.concatenate(blocks)


def test_embed_sum_exact_on_closed_form_tables():
    """Tables whose entries and every partial sum are exact in float32: the GPU sum must
    equal the float64 oracle bit for bit, absent and out-of-range tokens included."""
    rows = synth.moshi_rows()
    d = 64
    E = _closed_form_tables(rows, d)
    rng = np.random.default_rng(14)
    S = 513
    V = np.stack([rng.integers(0, n, size=S) for n in rows], axis=1).astype(np.int32)
    V[5, 0] = -1
    V[9, 3] = rows[3]
    V[10, 16] = 1 << 30
    want, bad = oracle.embed_sum(E, rows, V)
    n_bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    got = pkg().embed_sum(dev(E), rows, dev(V), n_bad=n_bad).cpu().numpy()
    assert np.array_equal(got.astype(np.float64), want)
    assert int(n_bad.item()) == bad == 2


def _abs_sum(tables_bits, rows, V):
    """Sum of |terms| per output element (for the float32 summation bound)."""
    return oracle.embed_sum(tables_bits & np.uint16(0x7FFF), rows, V)[0]


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_embed_sum_moshi_shapes_within_the_summation_bound(out_dtype):
    """17 bf16 tables (text 32 001 rows, 16 x 2049 audio rows), d = 4096, tokens from a packed
    tau = 1 stream (pads included). float32 recursive summation of K terms is within
    (K - 1) 2^-24 sum|terms| of the exact sum; a bf16 output adds 2^-8 of the value."""
    rows = synth.moshi_rows()
    tables = synth.moshi_tables(seed=15)
    text, audio = synth.moshi_streams(300, seed=16)
    V = oracle.delay_pack(text, audio, PATTERNS["tau1"])
    want, _ = oracle.embed_sum(tables, rows, V)
    absum = _abs_sum(tables, rows, V)
    tt = dev(tables.view(np.int16)).view(torch.bfloat16)
    od = torch.float32 if out_dtype == "f32" else torch.bfloat16
    got = pkg().embed_sum(tt, rows, dev(V), out_dtype=od).float().cpu().numpy().astype(np.float64)
    bound = 16 * 2.0 ** -24 * absum * (1 + 1e-6)
    if out_dtype == "bf16":  # |rn(x) - x| <= 2^-8 |x| and |x| <= |want| + bound
        bound = bound * (1 + 2.0 ** -7) + 2.0 ** -8 * np.abs(want) * (1 + 1e-6) + 2.0 ** -133
    assert np.all(np.abs(got - want) <= bound)


def test_embed_sum_full_size_sampled():
    """The benchmark's launch: 65 536 frames packed with tau = 1 (65 537 steps), bf16 tables
    and output; 256 sampled steps (the first and last included) against the oracle."""
    rows = synth.moshi_rows()
    tables = synth.moshi_tables()
    text, audio = synth.moshi_streams(1 << 16)
    p = pkg()
    packed = p.delay_pack(dev(text), dev(audio), PATTERNS["tau1"])
    tt = dev(tables.view(np.int16)).view(torch.bfloat16)
    out = p.embed_sum(tt, rows, packed)
    torch.cuda.synchronize()
    rng = np.random.default_rng(17)
    S = packed.shape[0]
    idx = np.unique(np.concatenate([[0, 1, S - 2, S - 1], rng.choice(S, 252, replace=False)]))
    V = packed.cpu().numpy()[idx]
    want, _ = oracle.embed_sum(tables, rows, V)
    absum = _abs_sum(tables, rows, V)
    got = out[torch.from_numpy(idx).cuda()].float().cpu().numpy().astype(np.float64)
    bound = (16 * 2.0 ** -24 * absum * (1 + 1e-6) * (1 + 2.0 ** -7)
             + 2.0 ** -8 * np.abs(want) * (1 + 1e-6) + 2.0 ** -133)
    assert np.all(np.abs(got - want) <= bound)


def test_embed_sum_many_tables_and_odd_widths():
    """Every code path of the embedding sum: K = 30 (register kernel), widths other than
    4096 (cp.async ring; 72 and 4104 columns leave partial stages) and d = 4096 with 9 and 1
    tables (bulk-copy ring with a short last row group), against the oracle within the
    float32 bound."""
    rng = np.random.default_rng(18)
    for K, d, rows_each in ((30, 256, 40), (28, 64, 30), (17, 72, 50), (5, 4104, 9), (9, 4096, 20),
                            (1, 4096, 7)):
        rows = [rows_each + k for k in range(K)]
        tables = synth.to_bf16_bits(rng.standard_normal((sum(rows), d)).astype(np.float32))
        V = np.stack([rng.integers(-1, n + 1, size=150) for n in rows], 1).astype(np.int32)
        want, bad = oracle.embed_sum(tables, rows, V)
        absum = _abs_sum(tables, rows, V)
        n_bad = torch.zeros(1, dtype=torch.int64, device="cuda")
        tt = dev(tables.view(np.int16)).view(torch.bfloat16)
        got = pkg().embed_sum(tt, rows, dev(V), out_dtype=torch.float32, n_bad=n_bad)
        got = got.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - want) <= K * 2.0 ** -24 * absum * (1 + 1e-6)), (K, d)
        assert int(n_bad.item()) == bad
