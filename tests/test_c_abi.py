"""The C ABI from a plain C program (tests/c_abi_roundtrip.c): no Python or torch on the
caller's side. On CPU it must compile and link against include/ and libmimi_rvq.so; on a
B200 it runs encode, encode_step and decode, and its outputs are checked against the oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import synth
from parity import assert_codes_match, decode_error, DECODE_TOL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
LIBDIR = os.path.join(ROOT, "split_residual_vector_b200")


def build(tmp_path):
    from split_residual_vector_b200 import build as lib_build
    lib_build.build()
    exe = str(tmp_path / "c_abi_roundtrip")
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Wextra", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_abi_roundtrip.c"),
           "-L", LIBDIR, "-lmimi_rvq", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{LIBDIR}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_compiles_and_links(tmp_path):
    assert os.path.exists(build(tmp_path))


@pytest.mark.gpu
def test_c_program_round_trip(tmp_path):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    exe = build(tmp_path)
    work = synth.offline_batch(n=300, seed=21)
    m = work.model
    for name, a in (("codebooks.f32", m.C), ("W_in.f32", m.W_in), ("W_out.f32", m.W_out),
                    ("latents.f32", work.z)):
        np.ascontiguousarray(a, dtype=np.float32).tofile(str(tmp_path / name))
    r = subprocess.run([exe, str(tmp_path), str(len(work.z))], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    codes = np.fromfile(str(tmp_path / "codes.i16"), np.int16).reshape(-1, 8)
    step = np.fromfile(str(tmp_path / "step.i16"), np.int16).reshape(-1, 8)
    x = np.fromfile(str(tmp_path / "decoded.f32"), np.float32).reshape(-1, 512)
    ref, db, ds = oracle.encode(work.z, m.W_in, m.C)
    assert_codes_match(codes, ref, db, ds, "C encode")
    assert_codes_match(step, ref, db, ds, "C encode_step")
    assert decode_error(x, oracle.decode(codes, m.C, m.W_out)) <= DECODE_TOL
