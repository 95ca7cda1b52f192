"""Pins of the float64 oracle for the Moshi token streams (delay-pattern packing, its
inverse, and the per-stream embedding sum) against what the pages and arithmetic fix."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PATTERNS = {"staircase": [0, 1, 2, 3, 4, 5, 6, 7], "tau2": [0, 2, 2, 2, 2, 2, 2, 2],
            "tau1": [0, 1, 1, 1, 1, 1, 1, 1], "none": [0] * 8}


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def _streams(rng, T, n_audio=2, Q=8):
    text = rng.integers(0, oracle.TEXT_CARD, size=T).astype(np.int32)
    audio = rng.integers(0, oracle.AUDIO_CARD, size=(n_audio, T, Q)).astype(np.int16)
    return text, audio


def test_worked_example():
    want = np.array([[int(v) for v in r.split()] for r in _golden_rows("delay_pack_example.txt")])
    audio = np.array([[[100 * q + t for q in range(3)] for t in range(3)]], np.int16)
    V = oracle.delay_pack(np.array([10, 11, 12], np.int32), audio, [0, 1, 2], text_pad=99,
                          audio_pad=77)
    assert V.tolist() == want.tolist()


def test_latency_of_the_pages_patterns():
    for row in _golden_rows("delay_pattern_latency.txt"):
        pattern, ms = row.split(";")
        assert oracle.delay_latency_ms([int(v) for v in pattern.split()]) == float(ms)


def test_zero_pattern_is_the_identity():
    rng = np.random.default_rng(0)
    text, audio = _streams(rng, 50)
    V = oracle.delay_pack(text, audio, PATTERNS["none"])
    assert V.shape == (50, 17)
    assert np.array_equal(V[:, 0], text)
    assert np.array_equal(V[:, 1:9], audio[0]) and np.array_equal(V[:, 9:17], audio[1])


@pytest.mark.parametrize("name", list(PATTERNS))
def test_seventeen_stream_layout_and_pads(name):
    """K = 17 columns: text, Moshi's 8 levels, the user's 8 levels; level q of each audio
    stream has exactly d_q leading pads and max(d) - d_q trailing pads; text has
    max(d) trailing pads."""
    d = PATTERNS[name]
    rng = np.random.default_rng(1)
    T = 40
    text, audio = _streams(rng, T)
    V = oracle.delay_pack(text, audio, d)
    m = max(d)
    assert V.shape == (T + m, 17)
    assert np.array_equal(V[:T, 0], text) and np.all(V[T:, 0] == oracle.TEXT_PAD)
    for a in range(2):
        for q in range(8):
            col = V[:, 1 + 8 * a + q]
            assert np.all(col[:d[q]] == oracle.AUDIO_PAD)
            assert np.array_equal(col[d[q]:d[q] + T], audio[a, :, q])
            assert np.all(col[d[q] + T:] == oracle.AUDIO_PAD)


def test_brute_force_against_the_definition():
    """Every entry of a small random packing against a direct evaluation of the reading,
    with arbitrary (non-monotone) delays and a truncated output length."""
    rng = np.random.default_rng(2)
    T, Q = 9, 4
    d = [3, 0, 5, 1]
    text = rng.integers(0, 50, size=T).astype(np.int32)
    audio = rng.integers(0, 50, size=(2, T, Q)).astype(np.int16)
    for S in (0, 4, T, T + 5, T + 8):
        V = oracle.delay_pack(text, audio, d, S=S, text_pad=-7, audio_pad=-9)
        for s in range(S):
            assert V[s, 0] == (text[s] if s < T else -7)
            for a in range(2):
                for q in range(Q):
                    t = s - d[q]
                    assert V[s, 1 + a * Q + q] == (audio[a, t, q] if 0 <= t < T else -9)


@pytest.mark.parametrize("name", list(PATTERNS))
def test_unpack_inverts_pack(name):
    d = PATTERNS[name]
    rng = np.random.default_rng(3)
    text, audio = _streams(rng, 33)
    V = oracle.delay_pack(text, audio, d)
    assert np.array_equal(oracle.delay_unpack(V, 1, d), audio[0])
    assert np.array_equal(oracle.delay_unpack(V, 9, d), audio[1])


def test_unpack_rejects_a_short_stream():
    V = np.zeros((5, 17), np.int32)
    with pytest.raises(oracle.OracleError):
        oracle.delay_unpack(V, 1, PATTERNS["staircase"], T=3)


def test_text_absent_and_single_audio_stream():
    rng = np.random.default_rng(4)
    _, audio = _streams(rng, 12, n_audio=1)
    V = oracle.delay_pack(None, audio, PATTERNS["tau1"])
    assert V.shape == (13, 9) and np.all(V[:, 0] == oracle.TEXT_PAD)


# ----------------------------------------------------------------- embedding sum

def _closed_form_tables(rows, d):
    """E_k[r][i] = 64 k + (r mod 64) + (i mod 16) / 16: exact in float32 and distinct per
    table, row and column, so a wrong table offset, row or column shows in the sum."""
    blocks = []
    for k, n in enumerate(rows):
        r = np.arange(n)[:, None]
        i = np.arange(d)[None, :]
        blocks.append((64 * k + (r % 64) + (i % 16) / 16.0).astype(np.float32))
    return np.concatenate(blocks)


def test_embed_sum_closed_form_at_moshi_row_counts():
    rows = [oracle.TEXT_CARD + 1] + [oracle.AUDIO_CARD + 1] * 16
    d = 48
    E = _closed_form_tables(rows, d)
    rng = np.random.default_rng(5)
    S = 60
    V = np.stack([rng.integers(0, n, size=S) for n in rows], axis=1).astype(np.int32)
    V[3, 0] = -1            # absent text token
    V[7, 5] = rows[5]       # past the table: adds nothing, counted
    V[8, 16] = rows[16] + 9
    out, bad = oracle.embed_sum(E, rows, V)
    assert bad == 2
    i = np.arange(d)
    for s in range(S):
        valid = [k for k in range(17) if 0 <= V[s, k] < rows[k]]
        want = sum(64 * k + V[s, k] % 64 for k in valid) + len(valid) * (i % 16) / 16.0
        assert np.array_equal(out[s], want), s


def test_embed_sum_one_table_is_a_row_lookup():
    rng = np.random.default_rng(6)
    E = rng.standard_normal((300, 40)).astype(np.float32)
    V = rng.integers(0, 300, size=(25, 1)).astype(np.int32)
    out, bad = oracle.embed_sum(E, [300], V)
    assert bad == 0 and np.array_equal(out, E[V[:, 0]].astype(np.float64))


def test_embed_sum_bf16_tables_widen_exactly():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 16, size=(2 * 64, 32), dtype=np.uint16)
    bits[(bits & 0x7F80) == 0x7F80] = 0  # no inf / nan patterns
    V = rng.integers(0, 64, size=(10, 2)).astype(np.int32)
    out, _ = oracle.embed_sum(bits, [64, 64], V)
    f = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    want = f[V[:, 0]] + f[64 + V[:, 1]]
    assert np.array_equal(out, want)


def test_embed_sum_of_stream_swap():
    """Swapping two tables together with their token columns leaves the sum unchanged up to
    the order of two float64 additions."""
    rng = np.random.default_rng(8)
    A = rng.standard_normal((30, 16)).astype(np.float32)
    B = rng.standard_normal((20, 16)).astype(np.float32)
    V = np.stack([rng.integers(0, 30, 12), rng.integers(0, 20, 12)], 1).astype(np.int32)
    o1, _ = oracle.embed_sum(np.concatenate([A, B]), [30, 20], V)
    o2, _ = oracle.embed_sum(np.concatenate([B, A]), [20, 30], V[:, ::-1])
    assert np.allclose(o1, o2, rtol=0, atol=1e-12)
