"""Shared checks for the GPU parity tests: the CUDA path against the float64 oracle."""
import numpy as np

import oracle

DECODE_TOL = 1e-4  # max-abs error / RMS of the oracle output


def assert_codes_match(gpu_codes, ref_codes, d_best, d_second, context=""):
    """Bit-exact on every frame that is not a near-tie on the oracle's path; return stats."""
    gpu_codes = np.asarray(gpu_codes)
    near = oracle.near_tie(d_best, d_second)
    bad = np.nonzero(np.any(gpu_codes[~near] != ref_codes[~near], axis=1))[0]
    if len(bad):
        idx = np.nonzero(~near)[0][bad[:5]]
        raise AssertionError(f"{context}: {len(bad)} non-near-tie frames differ, e.g. frames "
                             f"{idx.tolist()}: gpu {gpu_codes[idx].tolist()} oracle "
                             f"{ref_codes[idx].tolist()}")
    exact_all = float(np.mean(np.all(gpu_codes == ref_codes, axis=1)))
    return {"frames": len(gpu_codes), "near_tie": int(near.sum()), "exact_incl_near": exact_all}


def decode_error(gpu_out, ref_out):
    ref_out = np.asarray(ref_out, np.float64)
    rms = np.sqrt(np.mean(ref_out ** 2))
    return float(np.abs(np.asarray(gpu_out, np.float64) - ref_out).max() / rms)
