"""Parity checks of CUDA results against the fp64 oracle (test-only helpers).

Tolerances (the stated targets, made precise):
  y, dx   |gpu - ref| <= rtol * (|ref| + kappa), rtol = 1e-5 for float32 I/O
          and 1e-2 for bf16 I/O; kappa is the error scale of the same
          expression evaluated with absolute values (from the oracle).
          Where the sign of Q(x) is undecidable in float32
          (|Q| < AMB_REL * sum_j |b_j||x|^j), dx may take the value of any of
          the three branches s = -1, 0, +1: each is a correct float32 result.
  dA, dB  |gpu - ref| <= 1e-4 * |ref| + 2e-6 * sqrt(c2) + allowance.
          c2 (from the oracle) is the sum over the group's elements of
          (|term| (1 + c))^2, c the term's sensitivity to float32 rounding of
          P and Q. Random per-term and per-addition rounding errors add in
          quadrature, so the float32 noise of the sum is a few u * sqrt(c2)
          (u = 2^-24 = 6e-8; the per-addition part also grows with the square
          root of the summation depth, ~10 here): 2e-6 = 32 u leaves a margin
          of 5 to 20 above it. For random-sign, light-tailed terms sqrt(c2) ~
          |ref|, so the floor is 2% of the relative budget; it matters only for
          a sum that cancels far below its own rounding noise
          (|ref| << sum |term|) or one dominated by a few ill-conditioned,
          heavy-tailed terms, where float32 terms cannot reach 1e-4 relative.
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


def check_coef(dA, dB, ref, rtol=RTOL_COEF, floor=2e-6, what=""):
    """dA, dB: numpy arrays from the GPU; ref: oracle.coef_grads dict. Returns
    the largest plain relative error (for information)."""
    return coef_report(dA, dB, ref, rtol, floor, what)["max_rel"]


def coef_report(dA, dB, ref, rtol=RTOL_COEF, floor=2e-6, what="", plain=False):
    """Checks dA, dB as check_coef does and returns a summary: the largest plain
    relative error over all entries, the largest over the graded entries
    (|ref| >= 1e-8 sum |term|; sums that cancel below that are reported, not
    graded), and how many entries pass only through the noise floor or the
    sign-ambiguity allowance. With plain=True every graded entry must also meet
    the plain |gpu - ref| <= rtol |ref|."""
    dA = np.asarray(dA, np.float64)
    dB = np.asarray(dB, np.float64)
    eA = np.abs(dA - ref["dA"])
    eB = np.abs(dB - ref["dB"])
    okA = eA <= rtol * np.abs(ref["dA"]) + floor * np.sqrt(ref["c2_a"])
    okB = eB <= rtol * np.abs(ref["dB"]) + floor * np.sqrt(ref["c2_b"]) + ref["amb_b"]
    relA = eA / np.maximum(np.abs(ref["dA"]), 1e-300)
    relB = eB / np.maximum(np.abs(ref["dB"]), 1e-300)
    assert okA.all(), "%s dA: max rel err %.3g at %s" % (what, float(relA.max()),
                                                         np.argwhere(~okA)[:4].tolist())
    assert okB.all(), "%s dB: max rel err %.3g at %s" % (what, float(relB.max()),
                                                         np.argwhere(~okB)[:4].tolist())
    gA = np.abs(ref["dA"]) >= 1e-8 * ref["sabs_a"]
    gB = np.abs(ref["dB"]) >= 1e-8 * ref["sabs_b"]
    plainA = eA <= rtol * np.abs(ref["dA"])
    plainB = eB <= rtol * np.abs(ref["dB"])
    rep = {
        "max_rel": max(float(relA.max(initial=0)), float(relB.max(initial=0))),
        "max_rel_graded": max(float(relA[gA].max(initial=0)), float(relB[gB].max(initial=0))),
        "entries": int(relA.size + relB.size),
        "ungraded": int((~gA).sum() + (~gB).sum()),
        "floor_only": int((okA & ~plainA).sum() + (okB & ~plainB).sum()),
    }
    if plain:
        assert np.all(plainA[gA]) and np.all(plainB[gB]), \
            "%s: plain %.0e relative fails on graded entries (max %.3g)" % (
                what, rtol, rep["max_rel_graded"])
    return rep
