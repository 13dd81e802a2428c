"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and the
fp64 oracle on the same seeded bf16 inputs, and compare.

Tolerances: max |O_gpu - O_oracle| <= 1.5e-2 and max |LSE_gpu - LSE_oracle| <=
1e-3 (finite entries); masked-out rows must match exactly (O = 0, LSE = -inf).
"""
from __future__ import annotations

import math

import numpy as np
import torch

O_TOL = 1.5e-2
LSE_TOL = 1e-3


def gpu_prefill(Q, K, V, scale, causal=False, window=0, input_pos=0, k_lengths=None,
                q_lengths=None, want_lse=True):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    LSE = torch.full(Q.shape[:3], float("nan"), dtype=torch.float32, device=dev) if want_lse else None
    kl = k_lengths.to(dev) if k_lengths is not None else None
    ql = q_lengths.to(dev) if q_lengths is not None else None
    binding.attn_fwd(O, Qd, Kd, Vd, LSE, scale, causal, window, input_pos, kl, ql)
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return O.cpu(), (LSE.cpu() if LSE is not None else None)


def oracle_prefill(orc, Q, K, V, scale, causal=False, window=0, input_pos=0, k_lengths=None,
                   q_lengths=None, rows=None):
    Qs = Q if rows is None else Q[:, :, torch.as_tensor(rows, dtype=torch.long)]
    kl = None if k_lengths is None else k_lengths.numpy()
    ql = None if q_lengths is None else q_lengths.numpy()
    return orc.attn_fwd(Qs.double().numpy(), K.double().numpy(), V.double().numpy(), scale,
                        causal=causal, window=window, input_pos=input_pos, k_lengths=kl,
                        q_lengths=ql, rows=rows, Sq=Q.shape[2])


def compare(O_gpu, LSE_gpu, O_ref, LSE_ref, rows=None, what=""):
    """Element-wise comparison; returns (max O error, max LSE error)."""
    Og = O_gpu.double().numpy()
    if rows is not None:
        Og = Og[:, :, rows]
    assert np.all(np.isfinite(Og)), f"{what}: non-finite O"
    dO = float(np.abs(Og - O_ref).max()) if Og.size else 0.0
    assert dO <= O_TOL, f"{what}: max |dO| = {dO}"
    dL = 0.0
    if LSE_gpu is not None:
        Lg = LSE_gpu.double().numpy()
        if rows is not None:
            Lg = Lg[:, :, rows]
        ref_inf = np.isneginf(LSE_ref)
        assert np.array_equal(np.isneginf(Lg), ref_inf), f"{what}: -inf rows differ"
        assert not np.any(np.isnan(Lg)), f"{what}: NaN LSE"
        fin = ~ref_inf
        if fin.any():
            dL = float(np.abs(Lg[fin] - LSE_ref[fin]).max())
        assert dL <= LSE_TOL, f"{what}: max |dLSE| = {dL}"
        # rows the oracle says see nothing must be exactly zero
        Oz = Og[ref_inf]
        assert np.all(Oz == 0.0), f"{what}: empty rows not zero"
    return dO, dL


def sample_rows(Sq, seed, n_random=16, extra=()):
    """Boundary rows of every 128-row tile edge near the ends plus random rows."""
    rng = np.random.default_rng(seed)
    base = {0, 1, 63, 64, 127, 128, 129, 255, 256, Sq // 2, Sq - 129, Sq - 128, Sq - 2, Sq - 1}
    base |= {int(x) for x in extra}
    base |= set(int(x) for x in rng.integers(0, Sq, n_random))
    return np.array(sorted(r for r in base if 0 <= r < Sq), dtype=np.int32)


def gpu_decode(Q, K, V, lengths, n_splits):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    binding.attn_decode(O, Q.to(dev), K.to(dev), V.to(dev), lengths.to(dev), n_splits)
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return O.cpu()


def default_scale(D):
    return 1.0 / math.sqrt(D)
