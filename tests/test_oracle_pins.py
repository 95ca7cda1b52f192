"""Pins for the float64 oracle: checks against what the pages and the mathematics fix,
never against the oracle itself. CPU only.

Which plausible mistake each pin catches:
  * brute force in exact integer arithmetic: greedy-vs-joint, wrong residual sign,
    wrong level order, tie-break, d_best / d_second bookkeeping;
  * scipy cdist nearest neighbour: the distance itself (dropped or mis-signed term);
  * planted frames: the split wiring (acoustic RVQ on y, not on y - S_s), the projection
    direction (a transposed W_in cannot map pinv(W_in) y back to y);
  * identity projection: projection indexing (rows vs columns of W_in);
  * decode invariants: a dropped codebook in the sum, a transposed W_out;
  * rates: the golden tables the pages print;
  * translation invariance of the distance: a score without the ||c||^2 term, a chain fed
    from the wrong vector (checked by planting -2 r.c as the score in the oracle: both
    variants fail);
  * codeword relabelling: an index or row-offset mistake (checked by planting a row offset
    of one: the pin fails).
"""
import itertools
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


# ----------------------------------------------------------- exact brute force


def _greedy_exact(y, C, n_q):
    """Greedy split RVQ in Python integers: first minimum per level, r -= chosen."""
    def dist(r, c):
        return sum((ri - ci) ** 2 for ri, ci in zip(r, c))

    codes, best, second = [], [], []
    r = list(y)
    for level in range(n_q):
        target = y if level == 0 else r
        ds = [dist(target, c) for c in C[level]]
        k = min(range(len(ds)), key=lambda i: (ds[i], i))
        others = [d for i, d in enumerate(ds) if i != k]
        codes.append(k)
        best.append(ds[k])
        second.append(min(others) if others else float("inf"))
        if level >= 1:
            r = [ri - ci for ri, ci in zip(r, C[level][k])]
    return codes, best, second


def _all_paths_greedy(y, C):
    """Enumerate every acoustic code path; return those where each level's code is the
    first minimum given the levels before it (exactly one such path exists)."""
    q, k = len(C), len(C[0])
    hits = []
    for path in itertools.product(range(k), repeat=q - 1):
        r = list(y)
        ok = True
        for level, a in enumerate(path, start=1):
            ds = [sum((ri - ci) ** 2 for ri, ci in zip(r, c)) for c in C[level]]
            first = min(range(k), key=lambda i: (ds[i], i))
            if a != first:
                ok = False
                break
            r = [ri - ci for ri, ci in zip(r, C[level][a])]
        if ok:
            hits.append(path)
    return hits


def test_greedy_matches_exhaustive_enumeration_exactly():
    """Tiny integer codebooks (K=4, D=2, 1 semantic + 3 acoustic levels): float64 is exact on
    them, so codes and distances must equal the Python-integer enumeration bit for bit."""
    rng = np.random.default_rng(123)
    for trial in range(300):
        K, Dm, Qn = 4, 2, 4
        C = rng.integers(-6, 7, size=(Qn, K, Dm))
        if trial % 5 == 0:  # force ties
            C[rng.integers(Qn), 3] = C[rng.integers(Qn), 1]
        y = rng.integers(-9, 10, size=Dm)
        Cl = C.tolist()
        paths = _all_paths_greedy(y.tolist(), Cl)
        assert len(paths) == 1
        ref_codes, ref_best, ref_second = _greedy_exact(y.tolist(), Cl, Qn)
        assert tuple(ref_codes[1:]) == paths[0]
        codes, db, ds = oracle.encode_projected(y[None].astype(np.float64), C.astype(np.float32))
        assert codes[0].tolist() == ref_codes
        assert db[0].tolist() == [float(v) for v in ref_best]
        assert ds[0].tolist() == [float(v) for v in ref_second]


def test_greedy_is_not_the_joint_optimum():
    """A case where the jointly optimal acoustic path reconstructs y exactly but greedy does
    not: the oracle must return the greedy path (per-level nearest on the residual)."""
    # D = 1. y = 4; level 1 {3, 6}; level 2 {-2, 2}. Greedy: 3 then 2 (error 1);
    # joint: 6 then -2 (error 0).
    C = np.array([[[0.0], [100.0]], [[3.0], [6.0]], [[-2.0], [2.0]]], np.float32)
    y = np.array([[4.0]])
    codes, db, _ = oracle.encode_projected(y, C)
    assert codes[0].tolist() == [0, 0, 1]
    joint = min(itertools.product(range(2), repeat=2),
                key=lambda p: (4.0 - C[1, p[0], 0] - C[2, p[1], 0]) ** 2)
    assert joint == (1, 0)
    assert db[0, 2] == 1.0  # greedy leaves residual -1


def test_nearest_neighbour_matches_scipy_cdist():
    scipy_distance = pytest.importorskip("scipy.spatial.distance")
    rng = np.random.default_rng(7)
    Qn, K, Dm, N = 5, 64, 16, 400
    C = rng.standard_normal((Qn, K, Dm)).astype(np.float32)
    C[1:] *= 0.5
    y = rng.standard_normal((N, Dm))
    codes, db, _ = oracle.encode_projected(y, C)
    Cd = C.astype(np.float64)
    d0 = scipy_distance.cdist(y, Cd[0], "sqeuclidean")
    assert np.array_equal(codes[:, 0], d0.argmin(1))
    np.testing.assert_allclose(db[:, 0], d0.min(1), rtol=1e-12)
    r = y.copy()
    for level in range(1, Qn):
        d = scipy_distance.cdist(r, Cd[level], "sqeuclidean")
        a = d.argmin(1)
        assert np.array_equal(codes[:, level], a)
        np.testing.assert_allclose(db[:, level], d.min(1), rtol=1e-12, atol=1e-12)
        r = r - Cd[level][a]


# ----------------------------------------------------------- planted frames


def _well_separated(model, variant=0):
    """Plant acceptance: the oracle's best-vs-second gap is >= 1e-3 (1 + d_best) at every
    planted level (a semantic plant's acoustic levels quantise an ordinary random vector and
    are not part of the plant)."""
    def accept(row, kind, codes):
        _, db, ds = oracle.encode(row[None], model.W_in, model.C, variant=variant)
        levels = sorted(codes)
        return bool(np.all(ds[0, levels] - db[0, levels] >= 1e-3 * (1.0 + db[0, levels])))
    return accept


def test_planted_frames_recovered_exactly():
    """pr1_reference workload at full shape: every planted acoustic frame (y = sum of one
    codeword per acoustic level) returns its 7 acoustic codes, every planted semantic frame
    (y = one semantic codeword) returns its semantic code at distance ~0."""
    probe = synth.pr1_reference()
    work = synth.pr1_reference(accept=_well_separated(probe.model))
    assert len(work.planted) == 12
    idx = np.array(sorted(work.planted))
    codes, db, _ = oracle.encode(work.z[idx], work.model.W_in, work.model.C)
    for row, f in enumerate(idx):
        kind, planted = work.planted[f]
        if kind == "acoustic":
            assert codes[row, 1:].tolist() == [planted[lvl] for lvl in range(1, 8)]
            assert db[row, 7] < 1e-6
        else:
            assert codes[row, 0] == planted[0]
            assert db[row, 0] < 1e-6
    kinds = [work.planted[f][0] for f in idx]
    assert kinds.count("acoustic") == 6 and kinds.count("semantic") == 6


def test_full_sum_plant_needs_semantic_residual_variant():
    """y = S_s + sum_l A_l: recovered in full when the acoustic RVQ runs on y - S_s
    (variant 1), and its acoustic codes are lost when it runs on y (variant 0), because
    S_s dominates the residual chain."""
    rng = synth.generator(11)
    model = synth.make_model(rng)
    hits0 = 0
    for _ in range(6):
        codes_true = {lvl: int(rng.integers(synth.K)) for lvl in range(8)}
        row = synth.plant_latent(model, codes_true)
        c1, _, _ = oracle.encode(row[None], model.W_in, model.C, variant=1)
        assert c1[0].tolist() == [codes_true[lvl] for lvl in range(8)]
        c0, _, _ = oracle.encode(row[None], model.W_in, model.C, variant=0)
        assert c0[0, 0] == codes_true[0]
        hits0 += c0[0, 1:].tolist() == [codes_true[lvl] for lvl in range(1, 8)]
    assert hits0 == 0


# ----------------------------------------------------------- special cases


def test_identity_projection_returns_the_codeword_index():
    """W_in = [I | 0] and z = (S_k, noise): y = S_k exactly, so s = k at distance 0."""
    rng = np.random.default_rng(3)
    Dm, K, Qn = 16, 64, 3
    W_in = np.hstack([np.eye(Dm), np.zeros((Dm, Dm))]).astype(np.float32)
    C = rng.standard_normal((Qn, K, Dm)).astype(np.float32)
    ks = np.array([0, 5, 17, 63])
    z = np.hstack([C[0, ks], rng.standard_normal((len(ks), Dm)).astype(np.float32)])
    codes, db, _, y = oracle.encode(z, W_in, C, return_y=True)
    assert np.array_equal(y, C[0, ks].astype(np.float64))
    assert codes[:, 0].tolist() == ks.tolist()
    assert np.all(db[:, 0] == 0.0)
    # the other half of an identity: W_in = [0 | I] reads the second half of z
    W2 = np.hstack([np.zeros((Dm, Dm)), np.eye(Dm)]).astype(np.float32)
    z2 = np.hstack([rng.standard_normal((len(ks), Dm)).astype(np.float32), C[0, ks]])
    codes2, db2, _ = oracle.encode(z2, W2, C)
    assert codes2[:, 0].tolist() == ks.tolist() and np.all(db2[:, 0] == 0.0)


def test_projection_matches_library_matmul():
    rng = np.random.default_rng(5)
    W_in = rng.standard_normal((32, 64)).astype(np.float32)
    z = rng.standard_normal((50, 64)).astype(np.float32)
    y = oracle.project(z, W_in)
    ref = z.astype(np.float64) @ W_in.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


def test_tie_goes_to_lowest_index():
    rng = np.random.default_rng(9)
    Dm, K, Qn = 8, 32, 3
    C = rng.standard_normal((Qn, K, Dm)).astype(np.float32)
    C[0, 21] = C[0, 4]            # semantic duplicate
    C[1, 30] = C[1, 2]            # acoustic duplicate
    y = np.vstack([C[0, 4], C[1, 2]]).astype(np.float64)
    codes, db, ds = oracle.encode_projected(y, C)
    assert codes[0, 0] == 4 and db[0, 0] == ds[0, 0] == 0.0
    assert codes[1, 1] == 2 and db[1, 1] == ds[1, 1] == 0.0
    assert oracle.near_tie(db, ds).all()


def test_codes_in_range_and_prefix_property():
    """Codes lie in [0, K); encoding with the first n_q codebooks (quantizer dropout) gives
    the first n_q columns of the full encode (greedy levels only look backwards)."""
    rng = synth.generator(21)
    model = synth.make_model(rng, d_in=64, d=32, k=128)
    z = synth.latents(rng, 200, d_in=64)
    codes, _, _ = oracle.encode(z, model.W_in, model.C)
    assert codes.min() >= 0 and codes.max() < 128
    for n_q in (1, 3, 8):
        c, _, _ = oracle.encode(z, model.W_in, model.C, n_q=n_q)
        assert np.array_equal(c, codes[:, :n_q])


def test_bf16_latents_widen_exactly():
    """Latents that are exactly bf16 values give identical results as fp32 or as bf16 bits."""
    rng = synth.generator(8)
    model = synth.make_model(rng, d_in=64, d=32, k=128)
    bits = synth.latents(rng, 64, "bf16", d_in=64)
    as_f32 = synth.from_bf16_bits(bits)
    a = oracle.encode(bits, model.W_in, model.C)
    b = oracle.encode(as_f32, model.W_in, model.C)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ----------------------------------------------------------- decode


def test_decode_is_projected_sum_of_chosen_codewords():
    rng = synth.generator(13)
    model = synth.make_model(rng, d_in=64, d=32, k=128)
    codes = rng.integers(0, 128, size=(100, 8)).astype(np.int16)
    out, q = oracle.decode(codes, model.C, model.W_out, return_q=True)
    Cd = model.C.astype(np.float64)
    ref_q = Cd[0][codes[:, 0]]
    for level in range(1, 8):
        ref_q = ref_q + Cd[level][codes[:, level]]
    assert np.array_equal(q, ref_q)
    np.testing.assert_allclose(out, ref_q @ model.W_out.astype(np.float64).T, rtol=1e-12,
                               atol=1e-12)
    # n_q < 8 sums only the first n_q codebooks
    out3, q3 = oracle.decode(codes[:, :3], model.C, model.W_out, return_q=True)
    assert np.array_equal(q3, Cd[0][codes[:, 0]] + Cd[1][codes[:, 1]] + Cd[2][codes[:, 2]])


def test_decode_of_encode_is_sum_of_chosen_codewords():
    """decode(encode(z)) with W_out = [I; 0] is exactly the sum of the chosen codewords."""
    rng = synth.generator(17)
    model = synth.make_model(rng, d_in=64, d=32, k=128)
    z = synth.latents(rng, 80, d_in=64)
    codes, _, _ = oracle.encode(z, model.W_in, model.C)
    W_out = np.vstack([np.eye(32), np.zeros((32, 32))]).astype(np.float32)
    out = oracle.decode(codes, model.C, W_out)
    Cd = model.C.astype(np.float64)
    ref = sum(Cd[level][codes[:, level]] for level in range(8))
    assert np.array_equal(out[:, :32], ref)
    assert np.all(out[:, 32:] == 0.0)


def test_decode_rejects_out_of_range_codes():
    rng = synth.generator(1)
    model = synth.make_model(rng, d_in=16, d=8, k=32)
    codes = np.zeros((2, 8), np.int16)
    codes[1, 3] = 32
    with pytest.raises(oracle.OracleError):
        oracle.decode(codes, model.C, model.W_out)
    codes[1, 3] = -1
    with pytest.raises(oracle.OracleError):
        oracle.decode(codes, model.C, model.W_out)


# ----------------------------------------------------------- rates (golden)


def test_rates_match_the_pages():
    g = _read_kv("mimi_rates.txt")
    sr = float(g["sample_rate_hz"][0])
    strides = [int(s) for s in g["strides"]]
    fr = oracle.frame_rate(sr, strides)
    assert fr == float(g["frame_rate_hz"][0])
    assert sr / fr == float(g["samples_per_frame"][0])
    assert 1000.0 / fr == float(g["frame_ms"][0])
    K, Qn = int(g["codebook_size"][0]), int(g["codebooks"][0])
    assert oracle.bits_per_code(K) == int(g["bits_per_code"][0])
    assert oracle.bitrate(fr, Qn, K) == float(g["bitrate_bps"][0])
    assert (synth.D_IN, synth.D, synth.K, synth.Q) == (int(g["latent_dim"][0]),
                                                      int(g["projected_dim"][0]), K, Qn)


def test_codec_table_bitrates():
    with open(os.path.join(GOLDEN, "codec_table.txt")) as f:
        rows = [line.split() for line in f if line.strip() and not line.startswith("#")]
    assert len(rows) == 6
    for name, tok, nq, kbps, size in rows:
        fr = float(tok) / int(nq)
        bps = oracle.bitrate(fr, int(nq), int(size))
        assert round(bps / 1000.0, 1) == float(kbps), name


def test_near_tie_rule():
    db = np.array([[10.0, 1.0], [10.0, 1.0]])
    ds = np.array([[10.0 + 2e-4, 2.0], [10.0 + 1e-3, 2.0]])
    # threshold 1e-5 * (1 + 10) = 1.1e-4 on level 0
    assert oracle.near_tie(db, ds).tolist() == [False, False]
    ds[0, 0] = 10.0 + 1e-4
    assert oracle.near_tie(db, ds).tolist() == [True, False]


# ----------------------------------------------------------- invariances of the distance


@pytest.mark.parametrize("variant", [0, 1])
def test_translation_invariance(variant):
    """Squared distances do not change when the target and every candidate move by the same
    vector t. Variant 0 quantises y with codebook 0 and with the acoustic chain from codebook 1,
    so shifting y, codebook 0 and codebook 1 by t leaves every code and distance as it was;
    variant 1 feeds the chain y - S_s, so shifting y and codebook 0 alone does. Integer data
    keep every float64 operation exact, ties included. Catches a score without the ||c||^2 term
    (-2 y.c alone is not translation invariant) and a chain fed from the wrong vector."""
    rng = np.random.default_rng(41 + variant)
    Q, K, D, N = 4, 24, 6, 40
    C = rng.integers(-6, 7, size=(Q, K, D)).astype(np.float32)
    y = rng.integers(-9, 10, size=(N, D)).astype(np.float64)
    t = rng.integers(-20, 21, size=D)
    C2 = C.copy()
    C2[0] += t
    if variant == 0:
        C2[1] += t
    codes, db, ds = oracle.encode_projected(y, C, variant=variant)
    codes2, db2, ds2 = oracle.encode_projected(y + t, C2, variant=variant)
    assert np.array_equal(codes, codes2)
    assert np.array_equal(db, db2) and np.array_equal(ds, ds2)
    # and the plain shift of y alone does move the codes (the data are not degenerate)
    codes3, _, _ = oracle.encode_projected(y + t, C, variant=variant)
    assert not np.array_equal(codes, codes3)


def test_codeword_permutation_equivariance():
    """Relabelling the codewords of every codebook relabels the codes the same way and leaves
    the distances bit for bit unchanged. Catches an index or row-offset mistake in the scan."""
    rng = np.random.default_rng(43)
    Q, K, D, N = 8, 64, 16, 200
    C = rng.standard_normal((Q, K, D)).astype(np.float32)
    for level in range(1, Q):
        C[level] *= 0.5 ** level
    y = rng.standard_normal((N, D))
    perms = [rng.permutation(K) for _ in range(Q)]       # new index j holds old codeword p[j]
    Cp = np.stack([C[level][perms[level]] for level in range(Q)])
    codes, db, ds = oracle.encode_projected(y, C)
    codes_p, db_p, ds_p = oracle.encode_projected(y, Cp)
    inverse = [np.argsort(p) for p in perms]
    for level in range(Q):
        assert np.array_equal(codes_p[:, level], inverse[level][codes[:, level]])
    assert np.array_equal(db, db_p) and np.array_equal(ds, ds_p)
