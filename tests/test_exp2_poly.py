"""The FMA-pipe exp2 of the kernels (ex2_poly in csrc/ptx.cuh), emulated step
by step in IEEE fp32 on the CPU and checked against 2^x and the error bound of
its minimax polynomial; its constants must be the ones gen_exp2_poly.py
derives."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rank_latent_routing_flare_b200", "csrc")


def kernel_coeffs():
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = text[text.index("float ex2_poly(float x)"):]
    body = body[:body.index("}")]
    hexes = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    # Horner order in the source: c3, c2, c1, c0
    c3, c2, c1, c0 = (float.fromhex(h) for h in hexes)
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def generated_coeffs():
    spec = importlib.util.spec_from_file_location("gen", os.path.join(CSRC, "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, _ = gen.remez()
    return np.array(c, dtype=np.float32)


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fma32(a, b, c):
    # a*b is exact in float64 for float32 inputs; one final rounding to float32
    return f32(np.float64(a) * np.float64(b) + np.float64(c))


def ex2_poly_emulated(x, c):
    x = np.maximum(f32(x), np.float32(-125.0))
    t = f32(x.astype(np.float64) + 12582912.0)
    f = f32(x.astype(np.float64) - f32(t.astype(np.float64) - 12582912.0).astype(np.float64))
    p = fma32(c[3], f, c[2])
    p = fma32(p, f, c[1])
    p = fma32(p, f, c[0])
    bits = p.view(np.int32).astype(np.int64) + ((t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF)
    bits = ((bits + 2**31) % 2**32 - 2**31).astype(np.int32)
    return bits.view(np.float32)


def test_constants_come_from_the_generator():
    assert np.array_equal(kernel_coeffs(), generated_coeffs())


def test_relative_error_bound():
    c = kernel_coeffs()
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 0.0, 2_000_001), -rng.random(200_000) * 125.0,
                        np.arange(-125, 1, dtype=np.float64), np.arange(-125, 0) + 0.5,
                        [-1e-7, -0.4999999, -0.5000001, 0.25]])
    x = f32(x)
    got = ex2_poly_emulated(x, c).astype(np.float64)
    want = 2.0 ** x.astype(np.float64)
    rel = np.abs(got / want - 1.0)
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert rel.max() < 8e-5, rel.max()


def test_clamp_keeps_results_tiny_and_positive():
    c = kernel_coeffs()
    x = f32([-126.0, -200.0, -1e30, -np.inf])
    got = ex2_poly_emulated(x, c).astype(np.float64)
    assert np.all(got > 0) and np.all(got <= 2.0 ** -124.9)
