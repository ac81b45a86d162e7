"""Shared helpers of the parity tests: moving the seeded host inputs to the GPU
and the error metric.  No arithmetic of the method lives here."""
import numpy as np

# Tolerance on float outputs (fp32 accumulation, fp16 operands), measured as
#   max_i |y_gpu_i - y_ref_i| / max(|y_ref_i|, rms(y_ref)).
# The GPU keeps the dequantisation exact (codes enter the MMA as exact fp16,
# scale and zero are applied in fp32 per group); the remaining error comes
# from fp32 accumulation, the fp16 rounding of the compensator's t = x V^T
# and, in the full layer, 1-ulp differences of the fp16 SwiGLU activations.
REL_TOL = 2e-3


def rel_err(y, ref) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref ** 2)))
    den = np.maximum(np.abs(ref), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(y - ref) / den))


def to_dev(a: np.ndarray, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def f16_dev(bits: np.ndarray):
    import torch
    return to_dev(bits.astype(np.uint16).view(np.int16), torch.float16)


def bf16_dev(bits: np.ndarray):
    import torch
    return to_dev(bits.astype(np.uint16).view(np.int16), torch.bfloat16)


def act_dev(bits: np.ndarray, dtype: str):
    return bf16_dev(bits) if dtype == "bf16" else f16_dev(bits)


def act_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    import workloads as wl
    f = wl.bf16_bits_to_f32(bits) if dtype == "bf16" else wl.f16_bits_to_f32(bits)
    return f.astype(np.float64)
