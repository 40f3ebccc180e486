"""Pins for the oracle's FP8 MoE layer (the single-path FP8 MoE of the page
"vLLM and Tencent Hunyuan upstream two HPC backends for NVIDIA Hopper GPUs",
section "FP8 MoE pipeline as a single execution path": routing, Gate-Up GEMM,
activation, quantisation, Down GEMM, top-k reduction).

Each stage is checked against something other than itself: routing against a
library sort and a float64 softmax (with a planted tie); the row layout
against its invariants; gate-up, down and combine against float64 library
arithmetic on the dequantised operands (within one bf16 ulp); the activation
quantisation against float64 SiLU within the e4m3 rounding bound; and the whole
layer against an unquantised float64 MoE (FP8 error bound), which fails if an
expert, a row or a weight were mixed up.
"""
import numpy as np
import pytest
import torch

import oracle


def _problem(T, H, I, E, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    logits = (torch.randn(T, E, generator=g) * 2).numpy().astype(np.float32)
    w1 = (torch.randn(E * 2 * I, H, generator=g) * 0.05).to(torch.bfloat16)
    w2 = (torch.randn(E * H, I, generator=g) * 0.05).to(torch.bfloat16)
    w1q, sw1 = oracle.quantize_per_token(oracle.FMT_FP8, w1)
    w2q, sw2 = oracle.quantize_per_token(oracle.FMT_FP8, w2)
    return (x, logits, w1q.reshape(E, 2 * I, H), sw1.reshape(E, 2 * I), w2q.reshape(E, H, I), sw2.reshape(E, H),
            w1.float().numpy().reshape(E, 2 * I, H), w2.float().numpy().reshape(E, H, I))


def _deq(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _ulp_bf16(v):
    return np.ldexp(1.0, np.frexp(np.maximum(np.abs(v), 1e-30))[1] - 8)


@pytest.fixture(scope="module")
def case():
    T, H, I, E, k = 37, 256, 128, 16, 4
    p = _problem(T, H, I, E, 3)
    x, logits = p[0], p[1]
    logits[5, 3] = logits[5, 9] = np.float32(50.0)   # a tie for the top place: the lower index wins
    o = oracle.moe_forward(x, logits, *p[2:6], topk=k)
    return dict(T=T, H=H, I=I, E=E, k=k, p=p, o=o)


def test_routing_is_topk_of_the_logits_with_softmax_weights(case):
    o, logits, k = case["o"], case["p"][1], case["k"]
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k]   # descending, ties to the lower index
    assert np.array_equal(o["topk_ids"], order)
    assert o["topk_ids"][5, 0] == 3 and o["topk_ids"][5, 1] == 9
    sel = np.take_along_axis(logits.astype(np.float64), order, axis=1)
    ref = np.exp(sel - sel[:, :1])
    ref /= ref.sum(axis=1, keepdims=True)
    assert np.allclose(o["topk_w"], ref, rtol=2e-6, atol=0)
    assert np.allclose(o["topk_w"].sum(axis=1), 1.0, rtol=1e-6)


def test_rows_group_tokens_by_expert_in_token_order(case):
    o, E, k, T = case["o"], case["E"], case["k"], case["T"]
    counts = np.bincount(o["topk_ids"].ravel(), minlength=E)
    assert np.array_equal(o["offsets"], np.r_[0, np.cumsum(counts)])
    rows = o["rows"]
    assert np.array_equal(np.sort(rows.ravel()), np.arange(T * k))
    for e in range(E):
        t_of = [t for t in range(T) for j in range(k) if o["topk_ids"][t, j] == e]
        r_of = [rows[t, j] for t in range(T) for j in range(k) if o["topk_ids"][t, j] == e]
        assert r_of == list(range(o["offsets"][e], o["offsets"][e + 1])) and t_of == sorted(t_of)


def test_gate_up_down_and_combine_stages(case):
    o, p = case["o"], case["p"]
    x, w1q, sw1, w2q, sw2 = p[0], p[2], p[3], p[4], p[5]
    T, H, I, k = case["T"], case["H"], case["I"], case["k"]
    xq, sx = oracle.quantize_per_token(oracle.FMT_FP8, x)
    g = oracle.bf16_bits_to_f32(o["g"]).astype(np.float64)
    y = oracle.bf16_bits_to_f32(o["y"]).astype(np.float64)
    for t in range(T):
        for j in range(k):
            e, r = o["topk_ids"][t, j], o["rows"][t, j]
            ref_g = (_deq(w1q[e]) @ _deq(xq[t])) * float(sx[t]) * sw1[e].astype(np.float64)
            assert np.all(np.abs(g[r] - ref_g) <= _ulp_bf16(ref_g)), (t, j)
            ref_y = (_deq(w2q[e]) @ _deq(o["h_q"][r])) * float(o["s_h"][r]) * sw2[e].astype(np.float64)
            assert np.all(np.abs(y[r] - ref_y) <= _ulp_bf16(ref_y)), (t, j)
    out = oracle.bf16_bits_to_f32(o["out"]).astype(np.float64)
    ref = np.zeros((T, H))
    for j in range(k):
        ref += o["topk_w"][:, j:j + 1].astype(np.float64) * y[o["rows"][:, j]]
    assert np.all(np.abs(out - ref) <= _ulp_bf16(ref) + 1e-6 * np.abs(ref).max())


def test_activation_quantisation(case):
    o, I = case["o"], case["I"]
    g = oracle.bf16_bits_to_f32(o["g"]).astype(np.float64)
    gate, up = g[:, :I], g[:, I:]
    h = gate / (1.0 + np.exp(-gate)) * up                      # float64 SiLU(gate) * up
    deq = _deq(o["h_q"]) * o["s_h"][:, None].astype(np.float64)
    amax = np.abs(h).max(axis=1)
    assert np.allclose(o["s_h"], amax / 448.0, rtol=1e-6)
    # e4m3 round to nearest: relative 2^-4 for normals, half a subnormal step otherwise
    bound = np.maximum(np.abs(h) * 2.0 ** -4, o["s_h"][:, None] * 2.0 ** -10) * 1.001 + 1e-30
    assert np.all(np.abs(deq - h) <= bound)
    nz = amax > 0
    assert np.all(np.abs(_deq(o["h_q"][nz])).max(axis=1) == 448.0)


def test_whole_layer_against_unquantised_float64_moe(case):
    o, p = case["o"], case["p"]
    x = p[0].float().numpy().astype(np.float64)
    w1, w2 = p[6].astype(np.float64), p[7].astype(np.float64)
    T, H, I, k = case["T"], case["H"], case["I"], case["k"]
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = o["topk_ids"][t, j]
            gg = w1[e] @ x[t]
            h = gg[:I] / (1 + np.exp(-gg[:I])) * gg[I:]
            ref[t] += float(o["topk_w"][t, j]) * (w2[e] @ h)
    out = oracle.bf16_bits_to_f32(o["out"]).astype(np.float64)
    err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert err < 0.08, err          # two FP8 GEMMs with per-token / per-channel scales
    # the same with the experts of every token shifted by one must be far off
    wrong = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = (o["topk_ids"][t, j] + 1) % case["E"]
            gg = w1[e] @ x[t]
            wrong[t] += float(o["topk_w"][t, j]) * (w2[e] @ (gg[:I] / (1 + np.exp(-gg[:I])) * gg[I:]))
    assert np.linalg.norm(out - wrong) / np.linalg.norm(wrong) > 0.5
