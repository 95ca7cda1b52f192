"""GPU parity of the encode path (tcgen05 kernel + certified re-score + full-scan fallback)
against the float64 oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import synth
from parity import assert_codes_match

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def quantizer(model):
    import split_residual_vector_b200 as pkg
    return pkg.Quantizer(torch.from_numpy(model.C).cuda(), torch.from_numpy(model.W_in).cuda(),
                         torch.from_numpy(model.W_out).cuda())


def to_device(z):
    if z.dtype == np.uint16:
        return torch.from_numpy(z.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(z).cuda()


@pytest.fixture(scope="module")
def offline_small():
    work = synth.offline_batch(n=1000)
    return work, quantizer(work.model)


def test_pr1_reference_with_planted_frames():
    def accept_factory(model):
        def accept(row, kind, codes):
            _, db, ds = oracle.encode(row[None], model.W_in, model.C)
            lv = sorted(codes)
            return bool(np.all(ds[0, lv] - db[0, lv] >= 1e-3 * (1.0 + db[0, lv])))
        return accept
    work = synth.pr1_reference(accept=accept_factory(synth.pr1_reference().model))
    q = quantizer(work.model)
    codes = q.encode(to_device(work.z)).cpu().numpy()
    assert q.get_error() == 0
    ref, db, ds = oracle.encode(work.z, work.model.W_in, work.model.C)
    stats = assert_codes_match(codes, ref, db, ds, "pr1_reference")
    for f, (kind, planted) in work.planted.items():
        if kind == "acoustic":
            assert codes[f, 1:].tolist() == [planted[lvl] for lvl in range(1, 8)]
        else:
            assert codes[f, 0] == planted[0]
    print("pr1_reference", stats)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 127, 128, 129, 300, 777])
def test_ragged_sizes(offline_small, n, dtype):
    work, q = offline_small
    z = work.z[:n] if dtype == "f32" else synth.to_bf16_bits(work.z[:n])
    codes = q.encode(to_device(z)).cpu().numpy()
    assert q.get_error() == 0
    ref, db, ds = oracle.encode(z, work.model.W_in, work.model.C)
    assert_codes_match(codes, ref, db, ds, f"n={n} {dtype}")
    assert codes.min() >= 0 and codes.max() < 2048


def test_scan_kernel_matches_oracle(offline_small):
    work, q = offline_small
    z = work.z[:300]
    codes = q.encode_scan(to_device(z)).cpu().numpy()
    ref, db, ds = oracle.encode(z, work.model.W_in, work.model.C)
    assert_codes_match(codes, ref, db, ds, "scan")


def test_tensor_core_and_scan_agree_on_a_large_batch(offline_small):
    """Both GPU encoders on 20 000 frames: they may only differ on near-ties, which are a few
    percent of frames at these distributions; check the disagreeing frames with the oracle."""
    _, q = offline_small
    work = synth.offline_batch(n=20000, seed=5)
    q2 = quantizer(work.model)
    z = to_device(work.z)
    a = q2.encode(z).cpu().numpy()
    b = q2.encode_scan(z).cpu().numpy()
    diff = np.nonzero(np.any(a != b, axis=1))[0]
    assert len(diff) < 0.05 * len(a)
    if len(diff):
        ref, db, ds = oracle.encode(work.z[diff], work.model.W_in, work.model.C)
        assert oracle.near_tie(db, ds).all(), "tensor-core and scan encoders differ off a near-tie"


def test_offline_batch_full_size_sampled():
    """240 000 fp32 frames encoded in one call (the launch the benchmark times); 1500 sampled
    frames (including the ragged last tile) checked against the oracle."""
    work = synth.offline_batch()
    q = quantizer(work.model)
    codes = q.encode(to_device(work.z)).cpu().numpy()
    assert q.get_error() == 0
    rng = np.random.default_rng(0)
    idx = np.unique(np.concatenate([rng.choice(len(work.z), 1400, replace=False),
                                    np.arange(len(work.z) - 100, len(work.z))]))
    ref, db, ds = oracle.encode(work.z[idx], work.model.W_in, work.model.C)
    print("offline sampled", assert_codes_match(codes[idx], ref, db, ds, "offline_batch"))
    enc, rescanned = q.stats()
    assert enc == len(work.z)
    # the certificate fails on about 0.2 % of frames at these distributions (full scan)
    assert rescanned <= len(work.z) // 100


def test_bulk_tokenization_bf16_full_size_sampled():
    work = synth.bulk_tokenization()
    q = quantizer(work.model)
    codes = q.encode(to_device(work.z)).cpu().numpy()
    assert q.get_error() == 0
    rng = np.random.default_rng(1)
    idx = np.unique(np.concatenate([rng.choice(len(work.z), 1400, replace=False),
                                    np.arange(len(work.z) - 64, len(work.z))]))
    ref, db, ds = oracle.encode(work.z[idx], work.model.W_in, work.model.C)
    print("bulk sampled", assert_codes_match(codes[idx], ref, db, ds, "bulk_tokenization"))


def test_every_frame_of_the_offline_batch_against_the_oracle():
    """All 240 000 frames of the offline batch, encoded in the launch the benchmark times,
    against the float64 oracle frame by frame (about half a minute of oracle time on the
    host's cores): bit-exact on every frame that is not a near-tie on the oracle's path."""
    work = synth.offline_batch()
    q = quantizer(work.model)
    codes = q.encode(to_device(work.z)).cpu().numpy()
    assert q.get_error() == 0
    ref, db, ds = oracle.encode(work.z, work.model.W_in, work.model.C)
    stats = assert_codes_match(codes, ref, db, ds, "offline_batch, every frame")
    print("offline every frame", stats)
    assert stats["frames"] == 240_000


def test_every_frame_of_the_bulk_tokenization():
    """Every frame of the 1 048 576-frame bf16 encode: the tensor-core codes are compared
    with the float32 full scan's on the GPU, and every frame where the two differ goes to the
    float64 oracle, which must find a near-tie there (the only frames where two correct float32
    encoders may disagree). The oracle would need minutes for every frame of this size; the
    offline batch above is checked against it frame by frame."""
    work = synth.bulk_tokenization()
    q = quantizer(work.model)
    z = to_device(work.z)
    tc = q.encode(z).cpu().numpy()
    scan = q.encode_scan(z).cpu().numpy()
    assert q.get_error() == 0
    diff = np.nonzero(np.any(tc != scan, axis=1))[0]
    print("bulk_tokenization frames where the encoders differ:", len(diff), "of", len(tc))
    assert len(diff) < 0.05 * len(tc)
    if len(diff):
        _, db, ds = oracle.encode(work.z[diff], work.model.W_in, work.model.C)
        assert oracle.near_tie(db, ds).all(), "the encoders differ off a near-tie"


@pytest.mark.parametrize("batch", [1, 16, 128, 1024])
def test_streaming_step(batch):
    model, frames = synth.streaming_step(batch, calls=3)
    q = quantizer(model)
    for call in range(3):
        codes = q.encode_step(to_device(np.ascontiguousarray(frames[call]))).cpu().numpy()
        ref, db, ds = oracle.encode(frames[call], model.W_in, model.C)
        assert_codes_match(codes, ref, db, ds, f"step B={batch} call {call}")
    assert q.get_error() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_streaming_steps_equal_the_full_scan(dtype):
    """Steps of at most 480 frames run the float32 latency encoder on thread-block clusters,
    whose scores are the full scan's (same sums in the same order): every code equals
    encode_scan's, near ties included. Sizes span clusters of 16 and of 8 CTAs, one to 32
    frames per cluster with ragged last clusters, every thread tile and every projection
    tile."""
    model, frames = synth.streaming_step(1024, calls=1)
    q = quantizer(model)
    z = frames[0] if dtype == "f32" else synth.to_bf16_bits(frames[0])
    zd = to_device(np.ascontiguousarray(z))
    sizes = (1, 2, 3, 15, 16, 17, 33, 45, 63, 64, 65, 90, 100, 127, 128, 129, 180, 200, 255,
             256, 257, 300, 361, 384, 450, 479, 480)
    for b in sizes:
        step = q.encode_step(zd[:b]).cpu().numpy()
        scan = q.encode_scan(zd[:b]).cpu().numpy()
        assert np.array_equal(step, scan), f"B={b}: {np.argwhere(step != scan)[:5]}"
    enc, _ = q.stats()
    assert enc == sum(sizes)
    assert q.get_error() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_group_form_steps_equal_the_full_scan(dtype):
    """With the cluster form off (as on a device without clusters) steps of at most 256
    frames run the group form of the latency encoder (groups of up to 64 frames over CTAs
    meeting at barriers in global memory): its codes equal encode_scan's too, for one to four
    groups, ragged tails and every thread tile, also under CUDA-graph replay."""
    model, frames = synth.streaming_step(256, calls=2)
    q = quantizer(model)
    q.set_cluster_form(False)
    z = frames[0] if dtype == "f32" else synth.to_bf16_bits(frames[0])
    zd = to_device(np.ascontiguousarray(z))
    sizes = (1, 2, 15, 16, 17, 33, 63, 64, 65, 127, 128, 129, 200, 255, 256)
    for b in sizes:
        step = q.encode_step(zd[:b]).cpu().numpy()
        scan = q.encode_scan(zd[:b]).cpu().numpy()
        assert np.array_equal(step, scan), f"B={b}: {np.argwhere(step != scan)[:5]}"
    out = torch.empty((128, 8), dtype=torch.int16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        q.encode_step(zd[:128], out=out, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    static_in = zd[:128].clone()
    with torch.cuda.graph(g):
        q.encode_step(static_in, out=out, stream=torch.cuda.current_stream())
    for call in range(2):
        zc = frames[call][:128] if dtype == "f32" else synth.to_bf16_bits(frames[call][:128])
        static_in.copy_(to_device(np.ascontiguousarray(zc)))
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), q.encode_scan(static_in).cpu().numpy())
    q.set_cluster_form(True)
    assert np.array_equal(q.encode_step(zd[:100]).cpu().numpy(), q.encode_scan(zd[:100]).cpu().numpy())
    assert q.get_error() == 0


def test_cluster_form_switch_rejects_bad_values():
    model, _ = synth.streaming_step(1, calls=1)
    q = quantizer(model)
    import split_residual_vector_b200 as pkg
    lib = pkg.library()
    assert lib.mimi_rvq_set_cluster_form(None, 1) == -1
    assert lib.mimi_rvq_set_cluster_form(q._h, 2) == -1
    assert lib.mimi_rvq_set_cluster_form(q._h, 0) == 0
    assert lib.mimi_rvq_set_cluster_form(q._h, 1) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sliced_streaming_steps_match_the_oracle(dtype):
    """Steps of more than 480 frames run the codebook-sliced tensor-core encoder (8 CTAs per
    128-frame group, candidate lists exchanged through global memory): codes equal the
    oracle's outside near-ties and the batch tensor-core encoder's on every other frame,
    for full and ragged groups, up to the 18 groups that fit the device at once."""
    model, frames = synth.streaming_step(2304, calls=1)
    q = quantizer(model)
    z = frames[0] if dtype == "f32" else synth.to_bf16_bits(frames[0])
    zd = to_device(np.ascontiguousarray(z))
    ref, db, ds = oracle.encode(z, model.W_in, model.C)
    near = oracle.near_tie(db, ds)
    enc0, _ = q.stats()
    sizes = (481, 511, 512, 513, 700, 896, 1000, 1024, 2304)
    for b in sizes:
        step = q.encode_step(zd[:b]).cpu().numpy()
        assert_codes_match(step, ref[:b], db[:b], ds[:b], f"sliced step B={b}")
        batch = q.encode(zd[:b]).cpu().numpy()
        differ = np.any(step != batch, axis=1)
        assert not np.any(differ & ~near[:b]), f"B={b}: sliced and batch encoders differ off a near-tie"
    enc, _ = q.stats()
    assert enc - enc0 == 2 * sum(sizes)   # every step and every batch encode counted once
    assert q.get_error() == 0


def test_sliced_step_uncertified_rows_take_the_exact_scan():
    """Every level-1 codeword has ~20 exact copies, so no row of a sliced streaming step can
    certify its candidate window at level 1: each takes the in-kernel exact float32 scan of
    every slice's codewords, merged over the group (ties between copies go to the lowest
    index). 600 frames: four full groups and a ragged one. The codes match the oracle, and the
    float32 full-scan kernel's off the oracle's near-ties; each frame is counted once."""
    model = _small_model(seed=33)
    model.C[1] = model.C[1][np.arange(2048) % 100]
    q = quantizer(model)
    rng = np.random.default_rng(36)
    z = rng.standard_normal((600, 512)).astype(np.float32)
    zd = to_device(z)
    codes = q.encode_step(zd).cpu().numpy()
    assert q.get_error() == 0
    _, uncertified = q.stats()
    assert uncertified == 600
    ref, db, ds = oracle.encode(z, model.W_in, model.C)
    assert_codes_match(codes, ref, db, ds, "sliced, all rows uncertified")
    assert (codes[:, 1] < 100).all()  # the lowest of the tied copies
    near = oracle.near_tie(db, ds)
    scan = q.encode_scan(zd).cpu().numpy()
    assert np.array_equal(codes[~near], scan[~near])


def test_streaming_step_fewer_codebooks_and_variant():
    model, frames = synth.streaming_step(600, calls=1)
    q = quantizer(model)
    zd = to_device(np.ascontiguousarray(frames[0]))
    for b in (100, 600):   # cluster latency encoder, sliced tensor-core encoder
        for n_q, variant in ((1, 0), (5, 0), (8, 1), (3, 1)):
            step = q.encode_step(zd[:b], n_q=n_q, variant=variant).cpu().numpy()
            assert step.shape == (b, n_q)
            ref, db, ds = oracle.encode(frames[0][:b], model.W_in, model.C, n_q=n_q,
                                        variant=variant)
            assert_codes_match(step, ref, db, ds, f"step B={b} n_q={n_q} variant={variant}")
    assert q.get_error() == 0


def test_cluster_steps_on_two_streams_at_once():
    """The cluster form reads only the handle's tables, so steps launched on two streams with
    no ordering between them may overlap: both return the full scan's codes."""
    model, frames = synth.streaming_step(192, calls=2)
    q = quantizer(model)
    za = to_device(np.ascontiguousarray(frames[0][:128]))
    zb = to_device(np.ascontiguousarray(frames[1][:64]))
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    oa = torch.empty((128, 8), dtype=torch.int16, device="cuda")
    ob = torch.empty((64, 8), dtype=torch.int16, device="cuda")
    torch.cuda.synchronize()
    for _ in range(20):
        with torch.cuda.stream(sa):
            q.encode_step(za, out=oa, stream=sa)
        with torch.cuda.stream(sb):
            q.encode_step(zb, out=ob, stream=sb)
    torch.cuda.synchronize()
    assert np.array_equal(oa.cpu().numpy(), q.encode_scan(za).cpu().numpy())
    assert np.array_equal(ob.cpu().numpy(), q.encode_scan(zb).cpu().numpy())
    assert q.get_error() == 0


@pytest.mark.parametrize("batch", [1025, 2305, 5000])
def test_streaming_step_large_batch(batch):
    """Up to 2304 frames (18 groups of 8 CTAs on 148 SMs) a step is sliced; above, a batch
    encode."""
    model, frames = synth.streaming_step(batch, calls=1)
    q = quantizer(model)
    codes = q.encode_step(to_device(np.ascontiguousarray(frames[0]))).cpu().numpy()
    idx = np.concatenate([np.arange(0, 200), np.arange(batch - 100, batch)])
    ref, db, ds = oracle.encode(frames[0][idx], model.W_in, model.C)
    assert_codes_match(codes[idx], ref, db, ds, f"step B={batch}")
    assert q.get_error() == 0


@pytest.mark.parametrize("batch", [1, 128, 1024])
def test_streaming_step_in_a_cuda_graph(batch):
    """A captured step replays correctly on new inputs (the same codes as an uncaptured step):
    the cluster form keeps no state between launches, and the sliced form's group barriers
    return to their starting state after every launch."""
    model, frames = synth.streaming_step(batch, calls=4)
    q = quantizer(model)
    static_in = to_device(np.ascontiguousarray(frames[0]))
    static_out = torch.empty((batch, 8), dtype=torch.int16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        q.encode_step(static_in, out=static_out, stream=s)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        q.encode_step(static_in, out=static_out, stream=torch.cuda.current_stream())
    for call in range(4):
        static_in.copy_(to_device(np.ascontiguousarray(frames[call])))
        g.replay()
        torch.cuda.synchronize()
        got = static_out.cpu().numpy()
        want = q.encode_step(static_in).cpu().numpy()
        assert np.array_equal(got, want), f"replay {call}"
        ref, db, ds = oracle.encode(frames[call], model.W_in, model.C)
        assert_codes_match(got, ref, db, ds, f"replay {call}")
    assert q.get_error() == 0


# ------------------------------------------------------------------ adversarial inputs


def _small_model(seed=31):
    return synth.make_model(synth.generator(seed))


def test_duplicated_codewords_pick_the_lowest_index():
    model = _small_model()
    C = model.C
    C[0, 1500] = C[0, 700]
    C[3, 2000] = C[3, 9]
    C[7, 1024] = C[7, 1023]
    q = quantizer(model)
    rows = [synth.plant_latent(model, {0: 700}), synth.plant_latent(model, {0: 1500})]
    rows += [synth.plant_latent(model, {lvl: 9 if lvl == 3 else 5 for lvl in range(1, 8)})]
    z = np.stack(rows)
    codes = q.encode(to_device(z)).cpu().numpy()
    ref, db, ds = oracle.encode(z, model.W_in, C)
    assert codes[0, 0] == 700 and codes[1, 0] == 700 and ref[0, 0] == 700
    assert ref[2, 3] == 9 and np.array_equal(codes[2], ref[2])
    assert np.array_equal(codes[:, 0], ref[:, 0])


def test_many_equal_codewords_go_to_the_full_scan():
    """Twenty identical codewords nearest to the frame, spread over the codebook: more ties
    than the candidate list holds, so the candidate set cannot be certified; the frame must be
    re-encoded by the full scan and still return the lowest of the tied indices."""
    model = _small_model(33)
    tied = [100 + 37 * j for j in range(20)]
    for j in tied:
        model.C[0, j] = model.C[0, tied[0]]
    q = quantizer(model)
    z = np.stack([synth.plant_latent(model, {0: tied[5]})] * 3)
    codes = q.encode(to_device(z)).cpu().numpy()
    assert (codes[:, 0] == tied[0]).all()
    _, rescanned = q.stats()
    assert rescanned == 3


@pytest.mark.parametrize("k", [3, 5, 7, 8, 11, 20])
def test_equal_codewords_inside_one_scan_chunk(k):
    """k identical codewords in one 32-codeword chunk of the semantic codebook (columns 64..95),
    nearest to the frame: the scan takes them from the chunk in ascending key order. Up to 7
    fit the candidate list and certify without a re-encode; twenty are more than the list
    holds, and the row is re-encoded by the float32 full scan. Either way the lowest tied
    index wins."""
    model = _small_model(35)
    tied = [64 + (3 * j if k <= 11 else j) for j in range(k)]
    for j in tied:
        model.C[0, j] = model.C[0, tied[0]]
    q = quantizer(model)
    z = np.stack([synth.plant_latent(model, {0: tied[-1]})] * 3)
    codes = q.encode(to_device(z)).cpu().numpy()
    assert q.get_error() == 0
    assert (codes[:, 0] == tied[0]).all()
    ref, _, _ = oracle.encode(z, model.W_in, model.C)
    assert (ref[:, 0] == tied[0]).all()
    _, rescanned = q.stats()
    if k <= 7:
        assert rescanned == 0
    elif k == 20:
        assert rescanned == 3


def test_self_profile_counts(offline_small):
    """The diagnostic entry point returns the same codes, cycle counters for every role, and
    branch counts that respect their nesting; one count per 32-column chunk scanned by each
    epilogue warp (8 warps x 4 chunks x 8 tiles of 256 codewords x 8 codebooks per 128-frame
    tile)."""
    work, q = offline_small
    z = to_device(work.z)
    codes = q.encode(z).cpu().numpy()
    pcodes, prof = q.encode_profile(z)
    assert q.get_error() == 0
    assert np.array_equal(pcodes.cpu().numpy(), codes)
    tiles = (len(work.z) + 127) // 128
    assert prof["n_chunks"] == tiles * 8 * 4 * 8 * 8
    assert prof["n_chunks"] >= prof["n_displaced"] >= 0
    assert prof["n_chunks"] >= prof["n_runner_up"] >= prof["n_more"] >= 0
    assert prof["cta_total"] > 0 and prof["epi_scan"] > 0


@pytest.mark.parametrize("cluster_form", [True, False])
def test_rescan_of_many_frames_in_several_batches(cluster_form):
    """Every level-1 codeword has ~20 exact copies, so no frame's candidate window can be
    certified and all 2500 frames are re-encoded by the float32 latency encoder: the cluster
    form in passes of 32 frames per cluster, or the group form 1024 at a time (three
    batches). Its scores are the full scan's, so the codes equal encode_scan's; they also
    match the oracle (ties between copies go to the lowest index on both sides)."""
    model = _small_model(seed=33)
    model.C[1] = model.C[1][np.arange(2048) % 100]
    q = quantizer(model)
    q.set_cluster_form(cluster_form)
    rng = np.random.default_rng(34)
    z = rng.standard_normal((2500, 512)).astype(np.float32)
    zd = to_device(z)
    codes = q.encode(zd).cpu().numpy()
    enc, rescanned = q.stats()
    assert enc == 2500 and rescanned == 2500
    assert np.array_equal(codes, q.encode_scan(zd).cpu().numpy())
    ref, db, ds = oracle.encode(z, model.W_in, model.C)
    assert_codes_match(codes, ref, db, ds, "all frames re-scanned")
    # the re-encode with fewer codebooks and with the acoustic chain on y - S_s
    for n_q, variant in ((3, 0), (5, 1)):
        got = q.encode(zd[:700], n_q=n_q, variant=variant).cpu().numpy()
        want = q.encode_scan(zd[:700], n_q=n_q, variant=variant).cpu().numpy()
        assert np.array_equal(got, want), f"n_q={n_q} variant={variant}"
    assert q.get_error() == 0


def test_zero_huge_and_tiny_latents():
    model = _small_model(35)
    q = quantizer(model)
    rng = np.random.default_rng(2)
    z = np.concatenate([np.zeros((5, 512), np.float32),
                        (1e4 * rng.standard_normal((5, 512))).astype(np.float32),
                        (1e-30 * rng.standard_normal((5, 512))).astype(np.float32),
                        np.full((5, 512), 1e-40, np.float32)])
    codes = q.encode(to_device(z)).cpu().numpy()
    assert q.get_error() == 0
    ref, db, ds = oracle.encode(z, model.W_in, model.C)
    assert_codes_match(codes, ref, db, ds, "adversarial magnitudes")


# ------------------------------------------------------------------ boundary behaviour


def test_argument_errors(offline_small):
    import split_residual_vector_b200 as pkg
    work, q = offline_small
    z = to_device(work.z[:4])
    with pytest.raises(pkg.MimiRVQError) as e:
        q.encode(torch.from_numpy(work.z[:4]))            # host pointer
    assert e.value.status == -1
    flat = torch.empty(4 * 512 + 1, device="cuda")
    with pytest.raises(pkg.MimiRVQError):
        q.encode(flat[1:].view(4, 512))                  # 4-byte aligned only
    empty = q.encode(z[:0])
    assert empty.shape == (0, 8)
    lib = pkg.library()
    assert lib.mimi_rvq_encode(q._h, z.data_ptr(), 7, 4, empty.data_ptr(), None) == -1  # dtype
    assert lib.mimi_rvq_encode(None, z.data_ptr(), 0, 4, empty.data_ptr(), None) == -1
    assert q.get_error() == 0


# ------------------------------------------------------------------ projection, n_q, variant


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_projection_step_matches_oracle(offline_small, dtype):
    """y = W_in z from the tensor-core split-precision projection, against float64."""
    work, q = offline_small
    z = work.z[:300] if dtype == "f32" else synth.to_bf16_bits(work.z[:300])
    y = q.project(to_device(z)).cpu().numpy().astype(np.float64)
    ref = oracle.project(z, work.model.W_in)
    err = float(np.abs(y - ref).max())
    print(f"projection {dtype}: max abs error {err:.3e}")
    assert err <= (1e-4 if dtype == "f32" else 3e-5)


@pytest.mark.parametrize("n_q", [1, 2, 5, 8])
def test_fewer_codebooks(offline_small, n_q):
    """Quantizer dropout at inference: the first n_q codebooks only."""
    work, q = offline_small
    z = work.z[:300]
    codes = q.encode(to_device(z), n_q=n_q).cpu().numpy()
    assert codes.shape == (300, n_q)
    ref, db, ds = oracle.encode(z, work.model.W_in, work.model.C, n_q=n_q)
    assert_codes_match(codes, ref, db, ds, f"n_q={n_q}")
    scan = q.encode_scan(to_device(z), n_q=n_q).cpu().numpy()
    assert_codes_match(scan, ref, db, ds, f"scan n_q={n_q}")


def test_semantic_residual_variant():
    """variant 1: the acoustic RVQ quantises y - S_s; full 8-codeword plants come back whole."""
    rng = synth.generator(44)
    model = synth.make_model(rng)
    q = quantizer(model)
    z = synth.latents(rng, 200)
    plants = []
    for f in range(0, 200, 20):
        codes_true = {lvl: int(rng.integers(synth.K)) for lvl in range(8)}
        z[f] = synth.plant_latent(model, codes_true)
        plants.append((f, [codes_true[lvl] for lvl in range(8)]))
    codes = q.encode(to_device(z), variant=1).cpu().numpy()
    ref, db, ds = oracle.encode(z, model.W_in, model.C, variant=1)
    assert_codes_match(codes, ref, db, ds, "variant 1")
    for f, true in plants:
        assert codes[f].tolist() == true
