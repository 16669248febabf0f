"""Pins of the fp64 CPU oracle against things other than itself.

Each test ties one oracle function to a hand-computed example, a closed form,
a brute-force rebuild, a library routine or an invariant, so that a dropped
term, a wrong sign or index, or a transposed operand fails here.  CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
EPS = oracle.EPS


def bf16(x):
    """float list -> bf16 bit patterns via torch's float32 -> bf16 rounding."""
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------- bf16

def test_bf16_roundtrip_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000),
                        [0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.0e38, 1e-40, -1e-41]])
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(x32.astype(np.float64))
    assert np.array_equal(got, ref)
    back = oracle.bf16_to_f64(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_rounds_directly_from_fp64():
    L = oracle.lib()
    # 1 + 2^-8 + 2^-30 lies just above the tie between 1.0 and 1.0078125;
    # rounding through fp32 first would lose the 2^-30 and land on 1.0.
    assert L.oracle_double_to_bf16(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert L.oracle_double_to_bf16(1.0 + 2 ** -8) == 0x3F80          # tie -> even
    assert L.oracle_double_to_bf16(-(1.0 + 3 * 2 ** -8)) == 0xBF82    # tie -> even
    assert L.oracle_double_to_bf16(1e300) == 0x7F80                   # overflow -> inf


# ----------------------------------------------------------------- dequant

def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "dequant_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            left, right = line.split("|")
            t = left.split()
            bits, word, s, b = int(t[0]), int(t[1], 16), float(t[2]), float(t[3])
            codes = [int(v) for v in t[4:]]
            vals = [float(v) for v in right.split()]
            rows.append((bits, word, s, b, codes, vals))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: f"{r[0]}bit-{r[1]:#010x}")
def test_dequant_worked_example(row):
    bits, word, s, b, codes, vals = row
    per = 32 // bits
    q = np.zeros((1, 64 * bits // 32), np.uint32)
    q[0, 0] = word
    out = oracle.dequant(q, bf16([s]), bf16([b]), 1, 64, bits)[0]
    assert list(out[:per]) == vals
    assert np.all(out[per:] == b)          # zero codes give the bias alone


def test_dequant_group_and_row_indexing():
    # two rows x 128 columns: each (row, group) has its own scale; codes = 1 everywhere
    q = np.full((2, 128 // 8), 0x11111111, np.uint32)
    s = bf16([1.0, 2.0, 4.0, 8.0])
    b = bf16([0.5, -0.5, 0.25, -0.25])
    out = oracle.dequant(q, s, b, 2, 128, 4)
    assert np.all(out[0, :64] == 1.5) and np.all(out[0, 64:] == 1.5)
    assert np.all(out[1, :64] == 4.25) and np.all(out[1, 64:] == 7.75)


def test_dequant_matches_packed_codes():
    rng = np.random.default_rng(1)
    for bits in (4, 8):
        codes = rng.integers(0, 1 << bits, size=(3, 192))
        q = synth.pack_codes(torch.from_numpy(codes), bits).numpy().view(np.uint32)
        s = bf16(rng.uniform(0.01, 0.05, size=9))
        b = bf16(rng.uniform(-0.5, 0.5, size=9))
        sd, bd = oracle.bf16_to_f64(s).reshape(3, 3), oracle.bf16_to_f64(b).reshape(3, 3)
        want = sd.repeat(64, axis=1) * codes + bd.repeat(64, axis=1)
        assert np.array_equal(oracle.dequant(q, s, b, 3, 192, bits), want)


# ------------------------------------------------------- one quantised matrix

@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: f"{r[0]}bit-{r[1]:#010x}")
def test_qmat_gemv_worked_example(row):
    """One row of the worked example times x = (1, 2, 3, ...): the hand-computed
    values weighted by their column number (the rest of the group is the bias)."""
    bits, word, s, b, codes, vals = row
    per = 32 // bits
    q = np.zeros((1, 64 * bits // 32), np.uint32)
    q[0, 0] = word
    x = np.arange(1, 65, dtype=np.float64)
    want = sum(v * (c + 1) for c, v in enumerate(vals)) + b * sum(range(per + 1, 65))
    assert oracle.qmat_gemv(q, bf16([s]), bf16([b]), 1, 64, x, bits=bits)[0, 0] == want


def test_qmat_gemv_unit_vectors_give_the_columns():
    rng = np.random.default_rng(4)
    rows, cols = 5, 128
    codes = rng.integers(0, 16, size=(rows, cols))
    q = synth.pack_codes(torch.from_numpy(codes), 4).numpy().view(np.uint32)
    s = bf16(rng.uniform(0.01, 0.05, size=rows * 2))
    b = bf16(rng.uniform(-0.5, 0.5, size=rows * 2))
    sd, bd = oracle.bf16_to_f64(s).reshape(rows, 2), oracle.bf16_to_f64(b).reshape(rows, 2)
    for j in (0, 63, 64, 127):
        e = np.zeros(cols)
        e[j] = 1.0
        y = oracle.qmat_gemv(q, s, b, rows, cols, e)[0]
        assert np.array_equal(y, sd[:, j // 64] * codes[:, j] + bd[:, j // 64])


def test_qmat_gemv_bias_only_and_linearity():
    rows, cols = 3, 192
    q = np.zeros((rows, cols // 8), np.uint32)   # every code 0: W = bias of each group
    b = bf16([1.0, -2.0, 0.5, 4.0, 0.25, -1.0, 3.0, 2.0, -0.5])
    s = bf16([0.125] * 9)
    x = np.arange(cols, dtype=np.float64)
    gsum = x.reshape(3, 64).sum(axis=1)
    bd = oracle.bf16_to_f64(b).reshape(rows, 3)
    assert np.array_equal(oracle.qmat_gemv(q, s, b, rows, cols, x)[0], bd @ gsum)
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 16, size=(rows, cols))
    q = synth.pack_codes(torch.from_numpy(codes), 4).numpy().view(np.uint32)
    x1, x2 = rng.standard_normal(cols), rng.standard_normal(cols)
    y = oracle.qmat_gemv(q, s, b, rows, cols, np.stack([x1, x2, 2.0 * x1 - 3.0 * x2]))
    assert np.allclose(y[2], 2.0 * y[0] - 3.0 * y[1], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- rmsnorm

def test_rmsnorm_constant_vector_closed_form():
    for c in (1.0, -3.0, 1e-3, 250.0):
        xn = oracle.rmsnorm_no_scale(np.full(64, c))
        assert np.allclose(xn, c / math.sqrt(c * c + EPS), rtol=1e-15, atol=0)


def test_rmsnorm_scale_invariance_and_unit_rms():
    h = np.random.default_rng(2).standard_normal(512)
    a = oracle.rmsnorm_no_scale(h, eps=0.0)
    b = oracle.rmsnorm_no_scale(h * 37.5, eps=0.0)
    assert np.allclose(a, b, rtol=1e-14)
    assert abs(np.mean(a * a) - 1.0) < 1e-14
    assert np.all(np.sign(a) == np.sign(h))


# ------------------------------------------------------------------ router

def _tiny_layer(cfg_id=0, seed=0, **over):
    cfg = synth.CONFIGS[cfg_id]
    w = synth.gen_layer(cfg, cfg_id, 0, seed=seed)
    w.update(over)
    return cfg, w


def _router_with_codes(cfg, w, codes):
    w = dict(w)
    w["router_q"] = synth.pack_codes(torch.from_numpy(codes), 8)
    return w


def test_router_one_hot_hidden_picks_one_column():
    cfg, w = _tiny_layer()
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 256, size=(cfg.E, cfg.H))
    w = _router_with_codes(cfg, w, codes)
    L = oracle.OracleLayer.from_config(w, cfg)
    rs = oracle.bf16_to_f64(w["router_scale"])
    s = oracle.bf16_to_f64(w["router_s"]).reshape(cfg.E, -1)
    b = oracle.bf16_to_f64(w["router_b"]).reshape(cfg.E, -1)
    for j in (0, 63, 64, cfg.H - 1):
        h = np.zeros((1, cfg.H), np.float32)
        h[0, j] = 2.0
        logits, _, _, _ = oracle.router(L, torch.from_numpy(h).to(torch.bfloat16))
        # xn_j = 2 / sqrt(4/H + eps); xs_j = xn_j * rs_j / sqrt(H)
        xs_j = 2.0 / math.sqrt(4.0 / cfg.H + EPS) * rs[j] / math.sqrt(cfg.H)
        want = (s[:, j // 64] * codes[:, j] + b[:, j // 64]) * xs_j
        assert np.allclose(logits[0], want, rtol=1e-13, atol=1e-15)


def test_router_constant_hidden_closed_form():
    cfg, w = _tiny_layer()
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 256, size=(cfg.E, cfg.H))
    w = _router_with_codes(cfg, w, codes)
    w["router_scale"] = torch.ones(cfg.H, dtype=torch.bfloat16)
    L = oracle.OracleLayer.from_config(w, cfg)
    s = oracle.bf16_to_f64(w["router_s"]).reshape(cfg.E, -1)
    b = oracle.bf16_to_f64(w["router_b"]).reshape(cfg.E, -1)
    row_sum = (s.repeat(64, axis=1) * codes + b.repeat(64, axis=1)).sum(1)
    c = 0.75
    logits, idx, wts, xn = oracle.router(L, torch.full((1, cfg.H), c, dtype=torch.bfloat16))
    want = row_sum * (c / math.sqrt(c * c + EPS)) / math.sqrt(cfg.H)
    assert np.allclose(logits[0], want, rtol=1e-12)


def test_topk_matches_full_sort_brute_force():
    rng = np.random.default_rng(5)
    for trial in range(300):
        E = int(rng.integers(1, 70))
        k = int(rng.integers(1, E + 1))
        if trial % 3 == 0:     # many exact ties
            lg = rng.integers(-3, 4, size=E).astype(np.float64)
        else:
            lg = rng.standard_normal(E)
        want = sorted(range(E), key=lambda e: (-lg[e], e))[:k]
        assert list(oracle.topk(lg, k)) == want


def test_topk_all_equal_takes_lowest_indices():
    assert list(oracle.topk(np.zeros(16), 4)) == [0, 1, 2, 3]


def test_softmax_weights_closed_forms():
    rng = np.random.default_rng(6)
    E, k = 32, 6
    lg = rng.standard_normal(E) * 3
    idx = oracle.topk(lg, k)
    pes = bf16(rng.uniform(0.5, 1.5, E))
    w, p = oracle.gate_weights(lg, idx, pes)
    assert abs(p.sum() - 1.0) < 1e-15
    for a in range(k):
        for c in range(k):
            assert math.isclose(p[a] / p[c], math.exp(lg[idx[a]] - lg[idx[c]]), rel_tol=1e-13)
    assert np.array_equal(w, p * oracle.bf16_to_f64(pes)[idx])     # no renormalisation after the scale
    # k = 1: the weight is the per-expert scale itself
    w1, p1 = oracle.gate_weights(lg, idx[:1], pes)
    assert p1[0] == 1.0 and w1[0] == oracle.bf16_to_f64(pes)[idx[0]]
    # equal logits: uniform softmax
    _, pu = oracle.gate_weights(np.zeros(E), np.arange(4, dtype=np.int32), pes)
    assert np.all(pu == 0.25)


def test_router_softmax_is_over_selected_logits_only():
    cfg, w = _tiny_layer()
    L = oracle.OracleLayer.from_config(w, cfg)
    h = synth.gen_hidden(cfg, 0, 0, 4)
    logits, idx, wts, _ = oracle.router(L, h)
    pes = oracle.bf16_to_f64(w["per_expert_scale"])
    for t in range(4):
        assert list(idx[t]) == sorted(range(cfg.E), key=lambda e: (-logits[t, e], e))[:cfg.k]
        p = wts[t] / pes[idx[t]]
        assert abs(p.sum() - 1.0) < 1e-14


# ------------------------------------------------------------------ bucket

def test_bucket_brute_force_and_invariants():
    rng = np.random.default_rng(7)
    for _ in range(100):
        E = int(rng.integers(1, 40))
        k = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(0, 30))
        idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
        offsets, perm, inv = oracle.bucket(idx, E)
        flat = idx.reshape(-1)
        want_perm = [p for e in range(E) for p in range(T * k) if flat[p] == e]
        want_off = np.concatenate([[0], np.cumsum([np.sum(flat == e) for e in range(E)])])
        assert list(perm) == want_perm
        assert np.array_equal(offsets, want_off) and offsets[E] == T * k
        assert sorted(perm) == list(range(T * k))
        assert np.array_equal(inv[perm], np.arange(T * k))
        for e in range(E):
            assert np.all(flat[perm[offsets[e]:offsets[e + 1]]] == e)


# ----------------------------------------------------------------- experts

def _const_matrix(n_mat, rows, cols, code, scale):
    """Every weight = scale * code (bias 0): words filled with one nibble."""
    word = sum(code << (4 * j) for j in range(8))
    word = word - (1 << 32) if word >= (1 << 31) else word
    q = torch.full((n_mat, rows, cols // 8), word, dtype=torch.int32)
    s = torch.full((n_mat, rows, cols // 64), scale, dtype=torch.bfloat16)
    b = torch.zeros((n_mat, rows, cols // 64), dtype=torch.bfloat16)
    return q, s, b


def test_expert_zero_when_codes_sit_at_the_bias_midpoint():
    cfg, w = _tiny_layer()
    for name in ("gate", "up", "sh_gate", "sh_up"):
        w[name + "_q"] = torch.full_like(w[name + "_q"], 0x88888888 - (1 << 32))
        w[name + "_b"] = (-8.0 * w[name + "_s"].float()).to(torch.bfloat16)   # exact: times 8
    L = oracle.OracleLayer.from_config(w, cfg)
    x = np.random.default_rng(8).standard_normal(cfg.H)
    for e in (-1, 0, cfg.E - 1):
        assert np.all(oracle.expert(L, e, x) == 0.0)


def test_expert_swiglu_closed_form():
    cfg, w = _tiny_layer()
    H, I = cfg.H, cfg.I
    cg, cu, cd = 3 * 0.125, 5 * 0.0625, 7 * 0.25          # exact bf16 products
    w["gate_q"], w["gate_s"], w["gate_b"] = _const_matrix(cfg.E, I, H, 3, 0.125)
    w["up_q"], w["up_s"], w["up_b"] = _const_matrix(cfg.E, I, H, 5, 0.0625)
    w["down_q"], w["down_s"], w["down_b"] = _const_matrix(cfg.E, H, I, 7, 0.25)
    L = oracle.OracleLayer.from_config(w, cfg)
    # x = v * 1 with g = cg * v * H = ln 3, so sigmoid(g) = 3/4 exactly
    v = math.log(3.0) / (cg * H)
    y = oracle.expert(L, 2, np.full(H, v))
    u = cu * v * H
    a = 0.75 * math.log(3.0) * u                  # silu(g) * u with silu applied to the gate
    assert np.allclose(y, cd * I * a, rtol=1e-13)
    # large gate: silu(g) -> g
    y2 = oracle.expert(L, 2, np.full(H, 40.0 / (cg * H)))
    u2 = cu * 40.0 / cg
    assert np.allclose(y2, cd * I * 40.0 * u2, rtol=1e-15)
    # zero gate: silu(0) = 0
    assert np.all(oracle.expert(L, 2, np.zeros(H)) == 0.0)


def _dense_expert(w, e, x, I, H):
    if e < 0:
        G = oracle.dequant(w["sh_gate_q"], w["sh_gate_s"], w["sh_gate_b"], I, H, 4)
        U = oracle.dequant(w["sh_up_q"], w["sh_up_s"], w["sh_up_b"], I, H, 4)
        D = oracle.dequant(w["sh_down_q"], w["sh_down_s"], w["sh_down_b"], H, I, 4)
    else:
        G = oracle.dequant(w["gate_q"][e], w["gate_s"][e], w["gate_b"][e], I, H, 4)
        U = oracle.dequant(w["up_q"][e], w["up_s"][e], w["up_b"][e], I, H, 4)
        D = oracle.dequant(w["down_q"][e], w["down_s"][e], w["down_b"][e], H, I, 4)
    g, u = G @ x, U @ x
    return D @ (g * u / (1.0 + np.exp(-g)))


def test_dense_equivalence_k_equals_E_unit_gates():
    """Routing every token to all E experts with unit gates equals the dense mixture."""
    cfg, w = _tiny_layer()
    L = oracle.OracleLayer(w, cfg.H, cfg.E, cfg.E, cfg.I, cfg.Is)   # k = E
    rng = np.random.default_rng(9)
    T = 3
    x = rng.standard_normal((T, cfg.H))
    idx = np.stack([rng.permutation(cfg.E) for _ in range(T)]).astype(np.int32)
    m = oracle.expert_ffn(L, x, idx, np.ones((T, cfg.E)), with_shared=True)
    for t in range(T):
        dense = sum(_dense_expert(w, e, x[t], cfg.I, cfg.H) for e in range(cfg.E))
        dense = dense + _dense_expert(w, -1, x[t], cfg.Is, cfg.H)
        assert np.allclose(m[t], dense, rtol=1e-11, atol=1e-11)


def test_expert_ffn_weights_and_shared_term():
    cfg, w = _tiny_layer()
    L = oracle.OracleLayer.from_config(w, cfg)
    rng = np.random.default_rng(10)
    x = rng.standard_normal((2, cfg.H))
    idx = np.array([[3, 0, 7, 12], [15, 1, 2, 3]], np.int32)
    wt = rng.uniform(0.1, 1.0, (2, 4))
    m0 = oracle.expert_ffn(L, x, idx, wt, with_shared=False)
    m1 = oracle.expert_ffn(L, x, idx, wt, with_shared=True)
    for t in range(2):
        want = sum(wt[t, s] * _dense_expert(w, idx[t, s], x[t], cfg.I, cfg.H) for s in range(4))
        assert np.allclose(m0[t], want, rtol=1e-11, atol=1e-12)
        assert np.allclose(m1[t] - m0[t], _dense_expert(w, -1, x[t], cfg.Is, cfg.H), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------- combine

def test_combine_closed_forms():
    rng = np.random.default_rng(11)
    H = 128
    h = torch.from_numpy(rng.standard_normal((2, H)).astype(np.float32)).to(torch.bfloat16)
    hd = oracle.bf16_to_f64(h)
    of, ob = oracle.combine(h, np.zeros((2, H)), layer_scalar=0.5)
    assert np.array_equal(of, hd * 0.5)                    # rmsnorm(0) = 0
    of, _ = oracle.combine(h, np.full((2, H), -4.0))
    assert np.allclose(of, hd - 4.0 / math.sqrt(16.0 + EPS), rtol=1e-15)
    m = rng.standard_normal((2, H))
    of, _ = oracle.combine(h, m, post_norm=False, layer_scalar=2.0)
    assert np.allclose(of, (hd + m) * 2.0, rtol=1e-15)
    a, _ = oracle.combine(h, m, eps=0.0)
    b, _ = oracle.combine(h, m * 1e3, eps=0.0)             # post-norm is scale invariant
    assert np.allclose(a, b, rtol=1e-13, atol=1e-14)
    assert np.allclose(a - hd, m / np.sqrt(np.mean(m * m, axis=1, keepdims=True)), rtol=1e-12)
    a, ob = oracle.combine(h, m)
    assert np.array_equal(ob, oracle.f64_to_bf16(a))


def test_layer_forward_is_the_composition_of_its_parts():
    cfg, w = _tiny_layer()
    L = oracle.OracleLayer.from_config(w, cfg)
    h = synth.gen_hidden(cfg, 0, 0, cfg.T)
    r = oracle.layer_forward(L, h)
    logits, idx, wt, xn = oracle.router(L, h)
    xe = oracle.bf16_to_f64(oracle.f64_to_bf16(xn))
    m = oracle.expert_ffn(L, xe, idx, wt)
    of, ob = oracle.combine(h, m)
    assert np.array_equal(r["idx"], idx) and np.array_equal(r["w"], wt)
    assert np.array_equal(r["m"], m) and np.array_equal(r["out_f64"], of) and np.array_equal(r["out_bf16"], ob)


# --------------------------------------------------------------- inputs

def test_zipf_planted_experts_are_the_ones_the_router_selects():
    """The Zipf(1.1) input construction must make the router pick the planted set."""
    cfg = synth.CONFIGS[3]
    w = synth.gen_router(cfg, 3, 0)
    w.update({n: np.zeros(1, np.uint32) for n in oracle._WORDS if n != "router_q"})
    for n in ("gate", "up", "down", "sh_gate", "sh_up", "sh_down"):
        w[n + "_s"] = w[n + "_b"] = np.zeros(1, np.uint16)
    L = oracle.OracleLayer.from_config(w, cfg)
    for step in range(3):
        h, target = synth.gen_zipf_hidden(cfg, 3, 0, step, w["router_codes"])
        logits, idx, _, _ = oracle.router(L, h)
        assert sorted(idx[0]) == sorted(target[0].tolist())
        gap = np.sort(logits[0])[::-1]
        assert gap[cfg.k - 1] - gap[cfg.k] > 1.0


def test_threaded_oracle_gives_the_same_bits():
    """The all-cores oracle (the row loops split over OpenMP threads) is the
    same computation: every row's sum runs in the same order, so the layer's
    outputs are bit-identical to the sequential oracle's."""
    cfg = synth.CONFIGS[2]
    w = synth.gen_layer(cfg, 2, 0)
    L = oracle.OracleLayer.from_config(w, cfg)
    h = synth.gen_hidden(cfg, 2, 0, 2)
    try:
        oracle.set_threads(1)
        a = oracle.layer_forward(L, h)
        oracle.set_threads(4)
        b = oracle.layer_forward(L, h)
    finally:
        oracle.set_threads(1)
    for key in ("idx", "w", "m", "out_f64", "out_bf16"):
        assert np.array_equal(a[key], b[key]), key


def test_stored_tiny_redraws_are_the_oracles():
    """The benchmark's tiny-configuration inputs follow a stored redraw table;
    recompute the first 120 steps with the oracle and compare."""
    import importlib.util
    import os
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_tiny_redraws", os.path.join(here, "make_tiny_redraws.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    table = synth.load_redraws(os.path.join(here, "tiny_redraws.txt"))
    cfg = synth.CONFIGS[0]
    w = {n: v.cpu() for n, v in synth.gen_layer(cfg, 0, 0).items()}
    L = oracle.OracleLayer(w, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is)
    for step in range(120):
        stream = mk.FIRST_STREAM + step
        h = synth.gen_hidden_redrawn(cfg, 0, stream, cfg.T, table)
        logits = oracle.router(L, h)[0]
        for t in range(cfg.T):
            assert mk.min_gap(logits[t], cfg.k) >= mk.GAP, (stream, t)
            if (stream, t) in table:   # a listed row's first draw was below the gap
                first = synth.gen_hidden(cfg, 0, stream, cfg.T)[t:t + 1]
                assert mk.min_gap(oracle.router(L, first)[0][0], cfg.k) < mk.GAP
