"""Parity checks of CUDA results against the fp64 oracle (test-only helpers).

Tolerances (the stated targets, made precise):
  y, dx   |gpu - ref| <= rtol * (|ref| + kappa), rtol = 1e-5 for float32 I/O
          and 1e-2 for bf16 I/O; kappa is the error scale of the same
          expression evaluated with absolute values (from the oracle).
          Where the sign of Q(x) is undecidable in float32
          (|Q| < AMB_REL * sum_j |b_j||x|^j), dx may take the value of any of
          the three branches s = -1, 0, +1: each is a correct float32 result.
  dA, dB  |gpu - ref| <= 1e-4 * |ref| + 1e-5 * S_abs / sqrt(n_terms) + allowance.
          S_abs = sum of |term| and n_terms = elements per group, so
          S_abs / sqrt(n_terms) is the typical size of a sum of that many
          random-sign terms: the floor is a tenth of the relative budget at
          that size, and keeps a sum that cancels far below its own float32
          rounding noise (|ref| << S_abs) from being graded on relative error.
          The allowance is the most that the undecidable signs can move dB
          (2 |dy y x^j / D| summed over those elements; zero for dA, which does
          not depend on s).
"""
import numpy as np
import torch

import oracle
import synth

RTOL = {synth.F32: 1e-5, synth.BF16: 1e-2}
RTOL_COEF = 1e-4


def to_torch(arr, device="cuda"):
    """numpy float32 / uint16 (bf16 bits) -> torch tensor on the device."""
    if arr.dtype == np.uint16:
        return torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(arr).to(device)


def to_f64(t):
    """torch float32 / bf16 tensor -> numpy float64 (exact)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        u = t.view(torch.int16).numpy().view(np.uint16)
        return synth.bf16_bits_to_f32(u).astype(np.float64)
    return t.numpy().astype(np.float64)


def check_y(got, ref, kappa, rtol, what="y"):
    err = np.abs(got - ref)
    lim = rtol * (np.abs(ref) + kappa)
    bad = ~(err <= lim)
    assert not bad.any(), "%s: %d/%d outside tolerance, worst ratio %.3g" % (
        what, int(bad.sum()), bad.size, float(np.max(err / np.maximum(lim, 1e-300))))
    return float(np.max(err / np.maximum(np.abs(ref) + kappa, 1e-300)))


def check_dx(got, ref, ex, rtol, what="dx"):
    kappa = ex["kappa_dx"]
    err = np.abs(got - ref)
    ok = err <= rtol * (np.abs(ref) + kappa)
    amb = np.abs(ex["q"]) < oracle.AMB_REL * ex["kappa_q"]
    if amb.any():
        for t in range(3):
            alt = ex["dx_sign"][..., t]
            ok |= amb & (np.abs(got - alt) <= rtol * (np.abs(alt) + kappa))
    bad = ~ok
    assert not bad.any(), "%s: %d/%d outside tolerance (worst err %.3g)" % (
        what, int(bad.sum()), bad.size, float(np.max(np.where(bad, err, 0))))
    return int(amb.sum())


def check_coef(dA, dB, ref, n_terms, rtol=RTOL_COEF, floor=1e-5, what=""):
    """dA, dB: numpy arrays from the GPU; ref: oracle.coef_grads dict;
    n_terms: elements summed per group (rows * d_g). Returns the largest plain
    relative error (for information)."""
    dA = np.asarray(dA, np.float64)
    dB = np.asarray(dB, np.float64)
    s = float(np.sqrt(max(n_terms, 1)))
    eA = np.abs(dA - ref["dA"])
    eB = np.abs(dB - ref["dB"])
    okA = eA <= rtol * np.abs(ref["dA"]) + floor * ref["sabs_a"] / s
    okB = eB <= rtol * np.abs(ref["dB"]) + floor * ref["sabs_b"] / s + ref["amb_b"]
    relA = eA / np.maximum(np.abs(ref["dA"]), 1e-300)
    relB = eB / np.maximum(np.abs(ref["dB"]), 1e-300)
    assert okA.all(), "%s dA: max rel err %.3g at %s" % (what, float(relA.max()),
                                                         np.argwhere(~okA)[:4].tolist())
    assert okB.all(), "%s dB: max rel err %.3g at %s" % (what, float(relB.max()),
                                                         np.argwhere(~okB)[:4].tolist())
    return max(float(relA.max(initial=0)), float(relB.max(initial=0)))
