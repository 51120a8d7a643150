"""The seeded input generator: determinism, slicing, gathers, rounding and
distributions. CPU only."""
import math

import numpy as np
import pytest

import synth


def test_counter_based_slices_and_threads():
    full = np.empty(10000, np.float32)
    synth.fill(full, 7, synth.X_STREAM, synth.KIND_NORMAL, 1.0, nthreads=1)
    part = np.empty(1234, np.float32)
    synth.fill(part, 7, synth.X_STREAM, synth.KIND_NORMAL, 1.0, offset=5000, nthreads=3)
    assert np.array_equal(part, full[5000:6234])
    idx = np.array([0, 17, 9999, 5000, 3], np.int64)
    assert np.array_equal(synth.gather(idx, synth.F32, 7, synth.X_STREAM, synth.KIND_NORMAL, 1.0),
                          full[idx])


def test_streams_and_seeds_differ():
    a = np.empty(64, np.float32)
    b = np.empty(64, np.float32)
    c = np.empty(64, np.float32)
    synth.fill(a, 0, 1, synth.KIND_NORMAL, 1.0)
    synth.fill(b, 0, 2, synth.KIND_NORMAL, 1.0)
    synth.fill(c, 1, 1, synth.KIND_NORMAL, 1.0)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)


def test_bf16_is_rne_of_f32():
    f = np.empty(50000, np.float32)
    h = np.empty(50000, np.uint16)
    synth.fill(f, 3, 1, synth.KIND_NORMAL, 1.0)
    synth.fill(h, 3, 1, synth.KIND_NORMAL, 1.0)
    # round-to-nearest-even of the float32 bits, done independently here
    u = f.view(np.uint32).astype(np.uint64)
    want = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    assert np.array_equal(h, want)
    w = synth.bf16_bits_to_f32(h)
    assert np.all(np.abs(w - f) <= np.abs(f) * 2.0 ** -8)


def test_distributions():
    n = 400000
    z = np.empty(n, np.float32)
    synth.fill(z, 0, 1, synth.KIND_NORMAL, 1.0)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    s = np.empty(n, np.float32)
    synth.fill(s, 0, 1, synth.KIND_NORMAL, 1e-2)
    assert abs(s.std() - 1e-2) < 1e-4
    t = np.empty(n, np.float32)
    synth.fill(t, 0, 1, synth.KIND_STUDENT3, 1.0, 8.0)
    assert t.max() <= 8 and t.min() >= -8
    # Student-t(3): variance 3 before clipping; P(|t| > 8) = 0.0040
    assert 0.002 < np.mean(np.abs(t) >= 8) < 0.006
    assert abs(np.median(np.abs(t)) - 0.7649) < 0.01
    u = np.empty(n, np.float32)
    synth.fill(u, 0, 3, synth.KIND_UNIFORM, -0.5, 0.5)
    assert u.min() >= -0.5 and u.max() < 0.5 and abs(u.mean()) < 0.005


@pytest.mark.parametrize("name", synth.WORKLOADS)
def test_workloads(name):
    w = synth.workload(name)
    small = w.with_rows(3)
    x = small.x()
    dy = small.dy()
    a, b = small.coefficients()
    assert x.shape == (3, w.d) and dy.shape == (3, w.d)
    assert a.shape == (w.n_g, w.m + 1) and b.shape == (w.n_g, w.n)
    assert a.dtype == np.float32 and b.dtype == np.float32
    assert x.dtype == (np.float32 if w.dtype == synth.F32 else np.uint16)
    idx = np.array([0, w.d + 5, 3 * w.d - 1], np.int64)
    assert np.array_equal(small.x_at(idx), x.ravel()[idx])
    assert np.array_equal(small.dy_at(idx), dy.ravel()[idx])


def test_workload_shapes_match_kat():
    # KAT-T/S/B MLP hidden widths (4 x 192, 4 x 384, 4 x 768) and 197 tokens
    assert synth.workload("kat_t").d == 768 and synth.workload("kat_s").d == 1536
    assert synth.workload("kat_b").d == 3072 and synth.workload("kat_b").N == 197
    assert synth.workload("kat_b").elems == 309854208
    for g in (1, 8, 64):
        w = synth.workload("stress", n_g=g)
        assert w.n_g == g and w.d % g == 0


def test_identity_and_swish_bases():
    a, b = synth.workload("kat_t").coefficients()
    assert np.all(np.abs(a[:, 1] - 1.0) <= 0.1 + 1e-6) and np.all(np.abs(a[:, 0]) <= 0.1 + 1e-6)
    sa, sb = synth.swish_fit()
    xs = np.linspace(-4, 4, 101)
    P = sum(sa[i] * xs ** i for i in range(6))
    Q = sum(sb[j - 1] * xs ** j for j in range(1, 5))
    sw = xs / (1 + np.exp(-xs))
    assert np.max(np.abs(P / (1 + np.abs(Q)) - sw)) < 1e-4
    a, b = synth.workload("kat_s").coefficients()
    assert np.all(np.abs(a - sa[None, :]) <= 0.1 + 1e-6)
    assert math.isclose(float(np.mean(a[:, 1])), 0.5, abs_tol=0.1)
