"""The parity metric shared by the GPU tests and the CPU checks of the metric itself.

Per output tensor: the largest amount by which an element misses the reference, beyond the
rounding of the output's own storage type, relative to the largest reference magnitude:

    max_i max(|got_i - ref_i| - u |ref_i|, 0) / max_i |ref_i|

u is the unit roundoff of the output's storage (0 for fp32, 2^-11 for fp16, 2^-8 for bf16).
A 16-bit output is a rounding of the computed value, and that final rounding alone exceeds
the 3e-3 bound of the tensor-core path; nothing else is forgiven.
"""
import numpy as np

UNIT_ROUNDOFF_BY_NAME = {"float32": 0.0, "float16": 2.0 ** -11, "bfloat16": 2.0 ** -8}


def excess_rel_err(got, ref, u):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got))
    excess = np.maximum(np.abs(got - ref) - u * np.abs(ref), 0.0)
    return float(np.max(excess) / max(np.max(np.abs(ref)), 1e-30)) if got.size else 0.0
