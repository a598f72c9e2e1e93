"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each pin checks the oracle against something it cannot trivially agree with:
brute-force enumeration, a closed form, an invariant, a textbook special case,
a library sort, or a hand-worked example whose values are exact rationals
(tests/golden/two_token_example.json).  The last group plants mistakes in the
oracle (on the CPU) and checks that some pin fails for each.
"""
from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import moe_workloads as mw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_token_example.json")
F64 = torch.float64


# ----------------------------------------------------------------- helpers
def two_token_inputs():
    g = json.load(open(GOLDEN))
    ln3 = math.log(3.0)
    E = g["sizes"]["E"]
    inputs = {
        "x": torch.tensor(g["inputs"]["x"], dtype=F64),
        "w_router": torch.tensor(g["inputs"]["w_router_in_units_of_ln3"], dtype=F64) * ln3,
        "corr_bias": torch.tensor(g["inputs"]["corr_bias"], dtype=F64),
        "w_gate_up": torch.tensor(g["inputs"]["w_gate_up_each_expert"], dtype=F64).expand(E, 2, 2).clone(),
        "w_down": torch.stack([torch.tensor([[1.0], [float(e)]], dtype=F64) for e in range(E)]),
        "ws_gate_up": torch.tensor(g["inputs"]["ws_gate_up"], dtype=F64)[None],
        "ws_down": torch.tensor(g["inputs"]["ws_down"], dtype=F64)[None],
    }
    return g, inputs


def frac(a):
    return np.array([[float(Fraction(v)) for v in row] for row in a])


def check_two_token():
    g, inp = two_token_inputs()
    s = g["sizes"]
    r = oracle.moe_forward(inp, s["E"], s["k"], s["S"], s["route_scale"], s["global_scale"])
    ex = g["expected"]
    assert r["topk_idx"].tolist() == ex["topk_idx"]
    np.testing.assert_allclose(r["topk_w"].numpy(), frac(ex["topk_w"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(r["shared_gamma"].numpy(), frac(ex["shared_gamma"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(r["out"].numpy(), frac(ex["out_over_silu1"]) * ex["silu1"],
                               rtol=0, atol=1e-13)
    p = oracle.permute(r["topk_idx"], s["E"])
    assert p["offsets"].tolist() == ex["offsets"]
    assert p["perm_slot"].tolist() == ex["perm_slot"]
    assert p["inv_perm"].tolist() == ex["inv_perm"]


def textbook_swiglu_mlp(x, A_gate, B_up, D):
    """silu(x A^T) * (x B^T) @ D^T with separate gate and up matrices."""
    return (F.silu(x @ A_gate.T) * (x @ B_up.T)) @ D.T


def interleave_rows(A_gate, B_up):
    I, H = A_gate.shape
    W = torch.empty((2 * I, H), dtype=A_gate.dtype)
    for j in range(I):          # row 2j = gate_j, row 2j+1 = up_j
        W[2 * j] = A_gate[j]
        W[2 * j + 1] = B_up[j]
    return W


def check_interleave(seed=3):
    g = torch.Generator().manual_seed(seed)
    H, I, n = 12, 5, 7
    A = torch.randn(I, H, generator=g, dtype=F64)
    B = torch.randn(I, H, generator=g, dtype=F64)
    D = torch.randn(H, I, generator=g, dtype=F64)
    x = torch.randn(n, H, generator=g, dtype=F64)
    w = torch.rand(n, generator=g, dtype=F64) + 0.5
    got = oracle.expert_mlp(x, interleave_rows(A, B), D, w)
    want = w[:, None] * textbook_swiglu_mlp(x, A, B, D)
    np.testing.assert_allclose(got.numpy(), want.numpy(), rtol=1e-12, atol=1e-12)


def brute_force_topk(scores_row, k):
    """The unique k-subset whose every member beats every non-member under
    (score desc, index asc), found by enumerating all C(E, k) subsets."""
    E = len(scores_row)

    def beats(a, b):
        return scores_row[a] > scores_row[b] or (scores_row[a] == scores_row[b] and a < b)

    winners = [c for c in itertools.combinations(range(E), k)
               if all(beats(a, b) for a in c for b in range(E) if b not in c)]
    assert len(winners) == 1
    return set(winners[0])


def check_selection(seed, E, k, S, ties=False):
    g = torch.Generator().manual_seed(seed)
    H, T = 6, 9
    x = torch.randn(T, H, generator=g, dtype=F64)
    Wr = torch.randn(E + S, H, generator=g, dtype=F64)
    b = torch.rand(E, generator=g, dtype=F64) * 0.2 - 0.1
    if ties:   # duplicated router rows with equal bias force exact score ties
        for e in range(1, E, 2):
            Wr[e] = Wr[e - 1]
            b[e] = b[e - 1]
    r = oracle.gate(x, Wr, b, E, k, S, 1.0, 1.0)
    # independent score: plain Python floats
    for t in range(T):
        row = []
        for e in range(E):
            z = sum(float(x[t, h]) * float(Wr[e, h]) for h in range(H))
            row.append(1.0 / (1.0 + math.exp(-z)) + float(b[e]))
        got = r["topk_idx"][t].tolist()
        assert set(got) == brute_force_topk(row, k)
        for a, c in zip(got, got[1:]):  # returned best first
            assert row[a] > row[c] or (row[a] == row[c] and a < c)
        if ties:
            for a in got:
                if a % 2 == 1 and a - 1 not in got:
                    pytest.fail("a tie went to the higher index")


# -------------------------------------------------------------------- pins
def test_two_token_example():
    check_two_token()


@pytest.mark.parametrize("E,k,S", [(3, 1, 0), (5, 2, 1), (8, 2, 1), (9, 4, 2), (10, 3, 0), (6, 6, 1)])
def test_selection_brute_force(E, k, S):
    for seed in range(4):
        check_selection(seed, E, k, S)


@pytest.mark.parametrize("E,k", [(6, 2), (8, 3), (10, 5)])
def test_selection_exact_ties_go_to_lower_index(E, k):
    for seed in range(4):
        check_selection(100 + seed, E, k, 1, ties=True)


def check_weights_closed_form(seed=0, E=10, k=3, S=2, rs=2.5, gs=0.75):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(20, 16, generator=g, dtype=F64)
    Wr = torch.randn(E + S, 16, generator=g, dtype=F64)
    b = torch.rand(E, generator=g, dtype=F64) * 0.2 - 0.1
    r = oracle.gate(x, Wr, b, E, k, S, rs, gs)
    z = x @ Wr.T
    for t in range(x.shape[0]):
        sig_sel = [1.0 / (1.0 + math.exp(-float(z[t, e]))) for e in r["topk_idx"][t].tolist()]
        sig_sh = [1.0 / (1.0 + math.exp(-float(z[t, E + s]))) for s in range(S)]
        den = sum(sig_sel) + sum(sig_sh)
        np.testing.assert_allclose(r["topk_w"][t].numpy(), np.array(sig_sel) / den * rs * gs, rtol=1e-13)
        np.testing.assert_allclose(r["shared_gamma"][t].numpy(), np.array(sig_sh) / den * rs * gs, rtol=1e-13)
    total = r["topk_w"].sum(1) + r["shared_gamma"].sum(1)
    np.testing.assert_allclose(total.numpy(), rs * gs, rtol=1e-14)
    # the bias enters selection only: shifting every bias by a constant changes nothing
    r2 = oracle.gate(x, Wr, b + 0.3, E, k, S, rs, gs)
    assert torch.equal(r["topk_idx"], r2["topk_idx"])
    np.testing.assert_allclose(r2["topk_w"].numpy(), r["topk_w"].numpy(), rtol=1e-15)


def test_weights_closed_form_and_sum_invariant():
    for seed in range(3):
        check_weights_closed_form(seed)
    check_weights_closed_form(5, E=4, k=4, S=0, rs=1.0, gs=1.0)


def test_interleaved_swiglu_is_textbook_swiglu():
    check_interleave()


def test_single_routed_expert_no_shared_is_scaled_mlp():
    """S=0, E=k=1: the softmax has one entry, so out = route_scale*global_scale*MLP(x)."""
    g = torch.Generator().manual_seed(7)
    H, I, T = 16, 6, 11
    A, B = torch.randn(I, H, generator=g, dtype=F64), torch.randn(I, H, generator=g, dtype=F64)
    D = torch.randn(H, I, generator=g, dtype=F64)
    x = torch.randn(T, H, generator=g, dtype=F64)
    inputs = {"x": x, "w_router": torch.randn(1, H, generator=g, dtype=F64),
              "corr_bias": torch.zeros(1, dtype=F64), "w_gate_up": interleave_rows(A, B)[None],
              "w_down": D[None], "ws_gate_up": torch.zeros(0, 2 * I, H, dtype=F64),
              "ws_down": torch.zeros(0, H, I, dtype=F64)}
    r = oracle.moe_forward(inputs, 1, 1, 0, 2.5, 0.5)
    np.testing.assert_allclose(r["out"].numpy(), (1.25 * textbook_swiglu_mlp(x, A, B, D)).numpy(),
                               rtol=1e-12, atol=1e-12)


def test_full_layer_against_textbook_pieces():
    """E=3, k=2, S=2: the layer equals the closed-form weights times textbook
    SwiGLU MLPs, summed."""
    g = torch.Generator().manual_seed(9)
    H, I, T, E, k, S = 10, 4, 13, 3, 2, 2
    rs, gs = 2.5, 1.0
    mats = [(torch.randn(I, H, generator=g, dtype=F64), torch.randn(I, H, generator=g, dtype=F64),
             torch.randn(H, I, generator=g, dtype=F64)) for _ in range(E + S)]
    x = torch.randn(T, H, generator=g, dtype=F64)
    Wr = torch.randn(E + S, H, generator=g, dtype=F64)
    b = torch.tensor([0.05, -0.02, 0.0], dtype=F64)
    inputs = {"x": x, "w_router": Wr, "corr_bias": b,
              "w_gate_up": torch.stack([interleave_rows(a, bb) for a, bb, _ in mats[:E]]),
              "w_down": torch.stack([d for _, _, d in mats[:E]]),
              "ws_gate_up": torch.stack([interleave_rows(a, bb) for a, bb, _ in mats[E:]]),
              "ws_down": torch.stack([d for _, _, d in mats[E:]])}
    r = oracle.moe_forward(inputs, E, k, S, rs, gs)
    z = (x @ Wr.T).numpy()
    sig = 1.0 / (1.0 + np.exp(-z))
    for t in range(T):
        sel = sig[t, :E] + b.numpy()
        chosen = sorted(range(E), key=lambda e: (-sel[e], e))[:k]
        den = sig[t, chosen].sum() + sig[t, E:].sum()
        want = np.zeros(H)
        for e in chosen:
            A, B, D = mats[e]
            want += sig[t, e] / den * rs * gs * textbook_swiglu_mlp(x[t:t + 1], A, B, D)[0].numpy()
        for s in range(S):
            A, B, D = mats[E + s]
            want += sig[t, E + s] / den * rs * gs * textbook_swiglu_mlp(x[t:t + 1], A, B, D)[0].numpy()
        np.testing.assert_allclose(r["out"][t].numpy(), want, rtol=1e-11, atol=1e-12)


def check_permutation(seed=1, T=37, E=7, k=3, pad=False, repeats=False):
    rng = np.random.default_rng(seed)
    if repeats:   # an expert id may repeat inside a token (caller-given selections)
        idx = rng.integers(0, E, size=(T, k))
    else:
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    pm = torch.from_numpy(rng.random(T) < 0.3) if pad else None
    p = oracle.permute(torch.from_numpy(idx), E, pm)
    live = [t for t in range(T) if not (pad and bool(pm[t]))]
    rows = sorted((int(idx[t, j]), t, j) for t in live for j in range(k))   # Python's sort
    assert p["perm_slot"].tolist() == [t * k + j for _, t, j in rows]
    counts = [sum(1 for e, _, _ in rows if e == ee) for ee in range(E)]
    assert p["offsets"].tolist() == [sum(counts[:e]) for e in range(E + 1)]
    inv = p["inv_perm"].tolist()
    for r, (_, t, j) in enumerate(rows):
        assert inv[t * k + j] == r
    assert sum(1 for v in inv if v < 0) == (T - len(live)) * k


def test_permutation_against_python_sort():
    for seed in range(5):
        check_permutation(seed)
    check_permutation(11, T=1, E=4, k=2)
    check_permutation(12, T=50, E=3, k=3)   # every expert holds every token


def test_permutation_with_padding():
    for seed in range(3):
        check_permutation(seed, pad=True)


def test_permutation_with_repeated_ids_keeps_choice_order():
    # rows of one (expert, token) keep the order of their choices j
    for seed in range(3):
        check_permutation(seed, T=40, E=3, k=5, repeats=True)
        check_permutation(seed + 10, T=40, E=3, k=5, pad=True, repeats=True)


def test_padding_drops_routed_keeps_shared():
    w = mw.tiny(T=9, H=16, E=5, k=2, S=1, I=8)
    d = mw.generate(w, threads=1)
    pm = torch.zeros(w.T, dtype=torch.bool)
    pm[[1, 4]] = True
    r = oracle.moe_forward_workload(d, w, padding_mask=pm)
    assert torch.all(r["routed"][pm] == 0)
    np.testing.assert_allclose(r["out"][pm].numpy(), r["shared"][pm].numpy(), rtol=0, atol=0)
    r0 = oracle.moe_forward_workload(d, w)
    np.testing.assert_allclose(r["out"][~pm].numpy(), r0["out"][~pm].numpy(), rtol=0, atol=0)


def test_token_subset_equals_full_rows():
    w = mw.tiny(T=21, H=32, E=6, k=2, S=1, I=16, dtype="bf16")
    d = mw.generate(w, threads=1)
    full = oracle.moe_forward_workload(d, w)
    sub = torch.tensor([0, 5, 20])
    part = oracle.moe_forward_workload(d, w, tokens=sub)
    np.testing.assert_allclose(part["out"].numpy(), full["out"][sub].numpy(), rtol=1e-13, atol=1e-13)
    assert torch.equal(part["topk_idx"], full["topk_idx"][sub])


# --------------------------------------------------- planted mistakes
def _expect_pin_failure(monkeypatch, name, replacement, pins):
    monkeypatch.setattr(oracle, name, replacement)
    failed = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, pytest.fail.Exception, RuntimeError, ValueError, IndexError):
            failed += 1
    assert failed > 0, f"no pin caught the planted mistake in {name}"


def test_planted_swapped_gate_up_is_caught(monkeypatch):
    def bad(G, w):
        g, u = G[..., 1::2], G[..., 0::2]
        return w * (g * torch.sigmoid(g)) * u
    _expect_pin_failure(monkeypatch, "swiglu_interleaved", bad, [check_interleave])


def test_planted_weight_on_up_input_is_caught(monkeypatch):
    def bad(G, w):   # routing weight applied before the activation
        g, u = G[..., 0::2] * w, G[..., 1::2]
        return (g * torch.sigmoid(g)) * u
    _expect_pin_failure(monkeypatch, "swiglu_interleaved", bad, [check_interleave, check_two_token])


def test_planted_missing_bias_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "selection_scores", lambda z, b: torch.sigmoid(z))
    with pytest.raises(AssertionError):
        check_two_token()


def test_planted_reversed_tie_break_is_caught(monkeypatch):
    def bad(scores, k):
        s = scores.numpy()
        T, E = s.shape
        order = np.lexsort((-np.broadcast_to(np.arange(E), (T, E)), -s), axis=-1)
        return torch.from_numpy(np.ascontiguousarray(order[:, :k]))
    monkeypatch.setattr(oracle, "select_topk", bad)
    with pytest.raises(AssertionError):
        check_two_token()
    with pytest.raises((AssertionError, pytest.fail.Exception)):
        check_selection(100, 6, 2, 1, ties=True)


def test_planted_raw_shared_logits_is_caught(monkeypatch):
    """The other reading of the weights (no log-sigmoid on the shared logits)
    is told apart by the two-token example."""
    real_gate = oracle.gate

    def reading_b(x, w_router, corr_bias, E, k, S, rs, gs, given_topk_idx=None):
        r = real_gate(x, w_router, corr_bias, E, k, S, rs, gs, given_topk_idx)
        z = r["logits"]
        v = torch.cat([F.logsigmoid(torch.gather(z[:, :E], 1, r["topk_idx"])), z[:, E:E + S]], 1)
        p = torch.softmax(v, 1) * rs * gs
        return {**r, "topk_w": p[:, :k], "shared_gamma": p[:, k:]}
    monkeypatch.setattr(oracle, "gate", reading_b)
    with pytest.raises(AssertionError):
        check_two_token()


def test_planted_unsorted_permutation_is_caught(monkeypatch):
    real = oracle.permute

    def bad(topk_idx, E, padding_mask=None):
        r = real(topk_idx, E, padding_mask)
        ps = r["perm_slot"].clone()
        if ps.numel() > 2:
            ps[[0, 1]] = ps[[1, 0]]
        return {**r, "perm_slot": ps}
    monkeypatch.setattr(oracle, "permute", bad)
    with pytest.raises(AssertionError):
        check_permutation(0)


def test_planted_transposed_down_is_caught(monkeypatch):
    def bad(x_rows, w_gate_up, w_down, rw):
        G = x_rows @ w_gate_up.T
        h = oracle.swiglu_interleaved(G, rw[:, None])
        Wd = w_down.reshape(w_down.shape[1], w_down.shape[0])   # wrong orientation, same size
        return h @ Wd
    _expect_pin_failure(monkeypatch, "expert_mlp", bad, [check_interleave, check_two_token])


# ------------------------------------------------------------- dense layer
DENSE_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dense_mlp_example.json")


def check_dense_example():
    g = json.load(open(DENSE_GOLDEN))
    a = math.log(3.0)
    x = (torch.tensor(g["inputs"]["x_coeff_a"], dtype=F64) * a
         + torch.tensor(g["inputs"]["x_coeff_1"], dtype=F64))
    out = oracle.dense_mlp(x, torch.tensor(g["inputs"]["w_gate_up"], dtype=F64),
                           torch.tensor(g["inputs"]["w_down"], dtype=F64),
                           g["sizes"]["global_scale"])
    want = frac(g["expected"]["out_coeff_a"]) * a + frac(g["expected"]["out_coeff_a2"]) * a * a
    np.testing.assert_allclose(out.numpy(), want, rtol=0, atol=1e-14)


def check_dense_textbook(seed=5, gs=1.7):
    g = torch.Generator().manual_seed(seed)
    H, I = 10, 6
    A = torch.randn(I, H, generator=g, dtype=F64)
    B = torch.randn(I, H, generator=g, dtype=F64)
    D = torch.randn(H, I, generator=g, dtype=F64)
    x = torch.randn(2, 3, H, generator=g, dtype=F64)     # leading dims kept
    got = oracle.dense_mlp(x, interleave_rows(A, B), D, gs)
    assert got.shape == (2, 3, H)
    want = gs * textbook_swiglu_mlp(x.reshape(-1, H), A, B, D)
    np.testing.assert_allclose(got.reshape(-1, H).numpy(), want.numpy(), rtol=1e-12, atol=1e-12)


def test_dense_example():
    check_dense_example()


def test_dense_is_textbook_swiglu_mlp_times_global_scale():
    check_dense_textbook()


def test_dense_token_subset_equals_full_rows():
    w = mw.dense_tiny(T=20, H=64, I=64)
    d = mw.generate_dense(w)
    full = oracle.dense_mlp(d["x"], d["w_gate_up"], d["w_down"], 0.5)
    idx = torch.tensor([0, 7, 19])
    sub = oracle.dense_mlp(d["x"], d["w_gate_up"], d["w_down"], 0.5, tokens=idx)
    # same rows; the library matmul may block a 3-row product differently
    np.testing.assert_allclose(sub.numpy(), full[idx].numpy(), rtol=1e-12, atol=1e-14)


def test_dense_generator_slices_are_reproducible():
    w = mw.dense_tiny(T=4, H=64, I=300)     # 600 gate/up rows: three 256-row slices
    a = mw.generate_dense(w, threads=1)
    b = mw.generate_dense(w, threads=4)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert a["w_gate_up"].shape == (600, 64) and a["w_down"].shape == (64, 300)


def test_planted_dense_swapped_gate_up_is_caught(monkeypatch):
    def bad(G, w):
        g, u = G[..., 1::2], G[..., 0::2]
        return w * (g * torch.sigmoid(g)) * u
    _expect_pin_failure(monkeypatch, "swiglu_interleaved", bad, [check_dense_example])


def test_planted_dense_missing_global_scale_is_caught(monkeypatch):
    real = oracle.dense_mlp

    def bad(x, wgu, wd, global_scale=1.0, tokens=None):
        return real(x, wgu, wd, 1.0, tokens)
    monkeypatch.setattr(oracle, "dense_mlp", bad)
    for pin in (check_dense_example, check_dense_textbook):
        with pytest.raises(AssertionError):
            pin()


def test_planted_dense_transposed_down_is_caught(monkeypatch):
    real_mlp = oracle.dense_mlp

    def bad(x, wgu, wd, global_scale=1.0, tokens=None):
        return real_mlp(x, wgu, wd.T.contiguous().reshape(wd.shape), global_scale, tokens)
    monkeypatch.setattr(oracle, "dense_mlp", bad)
    for pin in (check_dense_example, check_dense_textbook):
        with pytest.raises(AssertionError):
            pin()


# ------------------------------------------------------------------ RMSNorm
RMS_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rmsnorm_example.json")


def check_rmsnorm_example():
    g = json.load(open(RMS_GOLDEN))
    for c in g["cases"]:
        y = oracle.rmsnorm(torch.tensor([c["x"]], dtype=F64), torch.tensor(c["weight"], dtype=F64),
                           c["eps"])
        np.testing.assert_allclose(y[0].numpy(), np.array(c["expected_over_sqrt2"]) * math.sqrt(2.0),
                                   rtol=0, atol=1e-15)


def check_rounding_cases():
    vals = [1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -30, -(1 + 2 ** -8 + 2 ** -30),
            1.5 * 2.0 ** -133, 2.5 * 2.0 ** -133]
    want = [1.0, 1 + 2 ** -6, 1 + 2 ** -7, -(1 + 2 ** -7), 2.0 ** -132, 2.0 ** -132]
    got = oracle.round_to_bf16(torch.tensor(vals, dtype=F64)).tolist()
    assert got == want


def check_rounding_matches_single_rounding_from_float32(seed=9):
    # float32 inputs: the library's float32 -> bfloat16 conversion rounds once
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(20000, generator=g, dtype=torch.float32) * 3
    ties = (torch.randint(-200, 200, (2000,), generator=g).float() + 0.5) * 2.0 ** -7  # exact ties
    a = torch.cat([a, ties.float(), -ties.float()])
    want = a.to(torch.bfloat16).double()
    got = oracle.round_to_bf16(a.double())
    assert torch.equal(got, want)


def check_rmsnorm_library_and_invariants(seed=4):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(5, 3, 48, generator=g, dtype=F64)
    w = torch.rand(48, generator=g, dtype=F64) + 0.5
    eps = 1e-6
    want = F.rms_norm(x, (48,), weight=w, eps=eps)     # library routine
    np.testing.assert_allclose(oracle.rmsnorm(x, w, eps).numpy(), want.numpy(), rtol=1e-13, atol=1e-14)
    ones = torch.ones(48, dtype=F64)
    y = oracle.rmsnorm(x, ones, 0.0)
    np.testing.assert_allclose(y.pow(2).mean(-1).numpy(), 1.0, rtol=1e-14)   # unit RMS
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * x, ones, 0.0).numpy(), y.numpy(), rtol=1e-14)


def test_rmsnorm_example():
    check_rmsnorm_example()


def test_round_to_bf16_cases():
    check_rounding_cases()
    check_rounding_matches_single_rounding_from_float32()


def test_rmsnorm_library_and_invariants():
    check_rmsnorm_library_and_invariants()


def test_rmsnorm_rounds_once_into_the_input_dtype():
    g = torch.Generator().manual_seed(2)
    x = torch.randn(4, 64, generator=g).to(torch.bfloat16)
    w = (torch.rand(64, generator=g) + 0.5).to(torch.bfloat16)
    y = oracle.rmsnorm(x, w, 1e-6, out_dtype=torch.bfloat16)
    assert y.dtype == torch.bfloat16
    assert torch.equal(y.double(), oracle.round_to_bf16(oracle.rmsnorm(x, w, 1e-6)).reshape(4, 64))
    y32 = oracle.rmsnorm(x.float(), w.float(), 1e-6, out_dtype=torch.float32)
    assert y32.dtype == torch.float32


def test_planted_eps_outside_sqrt_is_caught(monkeypatch):
    def bad(x, weight, eps, out_dtype=None):
        x64 = x.double()
        return x64 / (torch.sqrt((x64 * x64).mean(-1, keepdim=True)) + eps) * weight.double()
    _expect_pin_failure(monkeypatch, "rmsnorm", bad, [check_rmsnorm_example])


def test_planted_norm_over_wrong_axis_is_caught(monkeypatch):
    def bad(x, weight, eps, out_dtype=None):
        x64 = x.double()
        return x64 / torch.sqrt((x64 * x64).mean(0, keepdim=True) + eps) * weight.double()
    _expect_pin_failure(monkeypatch, "rmsnorm", bad, [check_rmsnorm_library_and_invariants])


def test_planted_missing_norm_weight_is_caught(monkeypatch):
    def bad(x, weight, eps, out_dtype=None):
        x64 = x.double()
        return x64 / torch.sqrt((x64 * x64).mean(-1, keepdim=True) + eps)
    _expect_pin_failure(monkeypatch, "rmsnorm", bad, [check_rmsnorm_example])


def test_planted_double_rounding_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "round_to_bf16", lambda y: y.to(torch.bfloat16).double())
    with pytest.raises(AssertionError):
        check_rounding_cases()
