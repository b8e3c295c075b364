"""Shared helpers of the GPU parity tests: moving seeded workloads to the GPU
and the tolerances the HSTU specification states.

Tolerances (against the fp64 oracle): fp32 tensors max-abs <= 1e-4; bf16
tensors relative Frobenius <= 1e-2 and max-abs <= 3e-2; integer work (buckets,
masks, indices) bit-exact."""
import numpy as np
import torch

FP32_MAX_ABS = 1e-4
BF16_REL_FRO = 1e-2
BF16_MAX_ABS = 3e-2


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def torch_dtype(name):
    return torch.float32 if name == "f32" else torch.bfloat16


def layer_to_dev(p, dtype):
    from hstu_sequential_transducer_02_b200 import binding
    return binding.layer_weights_to_device(p, dtype)


def errors(got, ref):
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    diff = g - r
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, ref, dtype_name, what="", grad=False):
    """grad=True: the tensor is a gradient, whose magnitude is set by the loss
    rather than being O(1); its max-abs bound is taken relative to its largest
    reference magnitude, max(1, max|ref|), because storing a value of magnitude
    M in the tensor's dtype alone already errs by up to M * 2^-9 (bf16)."""
    if isinstance(got, torch.Tensor):
        got = got.float().cpu().numpy()
    max_abs, rel = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    scale = max(1.0, float(np.max(np.abs(ref)))) if (grad and np.size(ref)) else 1.0
    if dtype_name == "f32":
        assert max_abs <= FP32_MAX_ABS * scale, f"{what}: max-abs {max_abs:.3e} > {FP32_MAX_ABS * scale:.3e}"
    else:
        assert rel <= BF16_REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {BF16_REL_FRO}"
        assert max_abs <= BF16_MAX_ABS * scale, f"{what}: max-abs {max_abs:.3e} > {BF16_MAX_ABS * scale:.3e}"
    return max_abs, rel
