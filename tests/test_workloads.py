"""The seeded input recipe (moe_workloads): the values the input recipe fixes,
checked against numbers worked out by hand from it.  CPU only.

  x ~ N(0, 1); router bank and expert weights ~ N(0, 0.02^2); correction
  bias ~ U(-0.1, 0.1), or for the Zipf layer b_e = 0.5 * ln p_e with
  p_e = (e+1)^-1.1 / sum_e' (e'+1)^-1.1 (expert 0 most popular); x and the
  expert weights of bf16 layers rounded to bf16, the router bank and the
  bias kept fp32; every tensor drawn from its own seeded stream.
"""
from __future__ import annotations

import math

import torch

import moe_workloads as mw


def test_zipf_bias_values():
    b = mw.zipf_bias(256)
    # worked by hand: H_256(1.1) = sum_{n<=256} n^-1.1 = 4.8315...;
    # b_e = 0.5 * (-1.1 ln(e+1) - ln H)
    H = sum(n ** -1.1 for n in range(1, 257))
    for e, expect in ((0, -0.789), (7, -1.932), (255, -3.839)):
        assert abs(float(b[e]) - expect) < 1e-3, (e, float(b[e]))
        assert abs(float(b[e]) - 0.5 * (-1.1 * math.log(e + 1) - math.log(H))) < 1e-6
    assert bool((b[1:] < b[:-1]).all())                      # strictly decreasing
    p = torch.exp(2 * b.double())
    assert abs(float(p.sum()) - 1.0) < 1e-6                  # the p_e form a distribution


def test_distributions_and_dtypes():
    w = mw.tiny(T=512, H=256, E=16, k=2, S=1, I=128, dtype="bf16", route_scale=2.5, seed=11)
    d = mw.generate(w, threads=2)
    assert d["x"].dtype == torch.bfloat16 and d["w_gate_up"].dtype == torch.bfloat16
    assert d["w_router"].dtype == torch.float32 and d["corr_bias"].dtype == torch.float32
    x = d["x"].float()
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1.0) < 0.01
    for name in ("w_router", "w_gate_up", "w_down", "ws_gate_up", "ws_down"):
        assert abs(float(d[name].float().std()) - 0.02) < 0.001, name
    cb = d["corr_bias"]
    assert float(cb.min()) >= -0.1 and float(cb.max()) <= 0.1 and float(cb.std()) > 0.04
    # shapes in the [out, in] orientation
    assert tuple(d["w_gate_up"].shape) == (16, 256, 256) and tuple(d["w_down"].shape) == (16, 256, 128)


def test_seeded_and_stream_separated():
    w = mw.tiny(T=64, H=128, E=8, k=2, S=1, I=64, dtype="bf16", route_scale=2.5, seed=5)
    a, b = mw.generate(w, threads=1), mw.generate(w, threads=3)
    for name in a:
        assert torch.equal(a[name], b[name]), name          # same seed, any thread count
    c = mw.generate(w.replace(T=32), threads=1)
    assert torch.equal(c["w_router"], a["w_router"])          # weights do not depend on T
    assert torch.equal(c["w_gate_up"], a["w_gate_up"])
    d = mw.generate(w.replace(seed=6), threads=1)
    assert not torch.equal(d["w_router"], a["w_router"])
