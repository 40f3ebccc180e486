"""GPU parity of the FP8 MoE path (routing, quantise-scatter, grouped GEMMs,
SiLU + quantisation, top-k combine; the single-path FP8 MoE of the page "vLLM
and Tencent Hunyuan upstream two HPC backends for NVIDIA Hopper GPUs") against
the oracle.

Each step is run through the C ABI on the oracle's (or the previous GPU
step's) inputs and compared: routing ids, offsets exactly, weights bitwise,
rows as a valid layout (the order inside an expert's group is free); the
quantised rows bit-exactly; the grouped GEMM within the FP8 tolerance (INT8
bit-exactly, including experts with no rows); the activation quantisation and
the combine bit-exactly against the oracle's own step on the same input; and
the whole layer (qlin_moe_forward, seven kernels chained with PDL) against the
oracle's layer.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL_ABS, TOL_REL, assert_fp_parity, assert_parity, bits_u8, bits_u16, check_status

pytestmark = pytest.mark.gpu


def _layer(T, H, I, E, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    logits = (torch.randn(T, E, generator=g) * 2).float()
    w1 = (torch.randn(E * 2 * I, H, generator=g) * 0.05).to(torch.bfloat16)
    w2 = (torch.randn(E * H, I, generator=g) * 0.05).to(torch.bfloat16)
    w1q, sw1 = oracle.quantize_per_token(oracle.FMT_FP8, w1)
    w2q, sw2 = oracle.quantize_per_token(oracle.FMT_FP8, w2)
    return x, logits, w1q, sw1, w2q, sw2


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    return t.cuda() if dtype is None else t.to(dtype).cuda()


@pytest.fixture(scope="module", params=[(64, 1024, 512, 32, 4), (5, 512, 256, 8, 2), (300, 512, 384, 16, 8)],
                ids=["decode64", "tiny", "prefill300"])
def case(request):
    T, H, I, E, k = request.param
    x, logits, w1q, sw1, w2q, sw2 = _layer(T, H, I, E, seed=T + E)
    o = oracle.moe_forward(x, logits.numpy(), w1q.reshape(E, 2 * I, H), sw1.reshape(E, 2 * I),
                           w2q.reshape(E, H, I), sw2.reshape(E, H), k)
    return dict(T=T, H=H, I=I, E=E, k=k, x=x, logits=logits, w1q=w1q, sw1=sw1, w2q=w2q, sw2=sw2, o=o)


def _route(c):
    from quantized_linear_layers_group_b200 import qlin

    T, E, k = c["T"], c["E"], c["k"]
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    rows = torch.empty(T, k, dtype=torch.int32, device="cuda")
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    qlin.qlin_moe_route(c["logits"].cuda(), k, ids, w, rows, offs)
    return ids, w, rows, offs


def test_routing_and_rows(case):
    o, E = case["o"], case["E"]
    ids, w, rows, offs = _route(case)
    torch.cuda.synchronize()
    check_status()
    assert np.array_equal(ids.cpu().numpy(), o["topk_ids"])
    assert np.array_equal(w.cpu().numpy().view(np.uint32), o["topk_w"].view(np.uint32))
    assert np.array_equal(offs.cpu().numpy(), o["offsets"])
    r = rows.cpu().numpy()
    assert np.array_equal(np.sort(r.ravel()), np.arange(r.size))        # every row used once
    e = o["topk_ids"]
    assert np.all((r >= o["offsets"][e]) & (r < o["offsets"][e + 1]))   # inside the expert's group


def test_quantize_scatter_grouped_mms_act_and_combine(case):
    from quantized_linear_layers_group_b200 import qlin

    c, o = case, case["o"]
    T, H, I, E, k = c["T"], c["H"], c["I"], c["E"], c["k"]
    R = T * k
    ids, w, rows, offs = _route(c)
    a_q = torch.empty(R, H, dtype=torch.uint8, device="cuda")
    s_a = torch.empty(R, dtype=torch.float32, device="cuda")
    qlin.qlin_moe_quantize_scatter(c["x"].cuda(), k, rows, a_q, s_a, flags=qlin.QLIN_PDL)
    g = torch.empty(R, 2 * I, dtype=torch.bfloat16, device="cuda")
    qlin.qlin_moe_grouped_mm(qlin.QLIN_FMT_FP8, E, a_q, s_a, offs, _dev(c["w1q"]), _dev(c["sw1"]), g,
                             flags=qlin.QLIN_PDL)
    torch.cuda.synchronize()
    check_status()
    rg, ro = rows.cpu().numpy().ravel(), o["rows"].ravel()
    xq, sx = oracle.quantize_per_token(oracle.FMT_FP8, c["x"])
    tok = np.repeat(np.arange(T), k)
    assert np.array_equal(bits_u8(a_q)[rg], xq[tok])
    assert np.array_equal(s_a.cpu().numpy()[rg].view(np.uint32), sx[tok].view(np.uint32))
    assert_fp_parity(bits_u16(g)[rg], o["g"][ro], "gate-up grouped GEMM")
    # activation + quantisation on the GPU's own G: bit-exact against the oracle's step
    h_q = torch.empty(R, I, dtype=torch.uint8, device="cuda")
    s_h = torch.empty(R, dtype=torch.float32, device="cuda")
    qlin.qlin_moe_act_quantize(g, h_q, s_h, flags=qlin.QLIN_PDL)
    y = torch.empty(R, H, dtype=torch.bfloat16, device="cuda")
    qlin.qlin_moe_grouped_mm(qlin.QLIN_FMT_FP8, E, h_q, s_h, offs, _dev(c["w2q"]), _dev(c["sw2"]), y,
                             flags=qlin.QLIN_PDL)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    qlin.qlin_moe_combine(y, w, rows, out, flags=qlin.QLIN_PDL)
    torch.cuda.synchronize()
    check_status()
    rhq, rsh = oracle.moe_act_quantize(bits_u16(g))
    assert np.array_equal(bits_u8(h_q), rhq)
    assert np.array_equal(s_h.cpu().numpy().view(np.uint32), rsh.view(np.uint32))
    # down GEMM on the GPU's h_q: the oracle's per-expert scaled_mm on the same rows
    offs_n = offs.cpu().numpy()
    yb = bits_u16(y)
    w2q, sw2 = c["w2q"].reshape(E, H, I), c["sw2"].reshape(E, H)
    for e in range(E):
        r0, r1 = offs_n[e], offs_n[e + 1]
        if r1 > r0:
            ref = oracle.scaled_mm(oracle.FMT_FP8, rhq[r0:r1], rsh[r0:r1], w2q[e], sw2[e])
            assert_fp_parity(yb[r0:r1], ref, f"down GEMM expert {e}")
    # combine on the GPU's y: bit-exact against the oracle's step
    assert np.array_equal(bits_u16(out), oracle.moe_combine(yb, w.cpu().numpy(), rows.cpu().numpy()))


def test_whole_layer_forward(case):
    from quantized_linear_layers_group_b200 import qlin

    c, o = case, case["o"]
    T, H, I, E, k = c["T"], c["H"], c["I"], c["E"], c["k"]
    ws = torch.empty(qlin.qlin_moe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    qlin.qlin_moe_forward(c["x"].cuda(), c["logits"].cuda(), k, _dev(c["w1q"]), _dev(c["sw1"]), _dev(c["w2q"]),
                          _dev(c["sw2"]), out, ws, flags=qlin.QLIN_PDL)
    torch.cuda.synchronize()
    check_status()
    got = oracle.bf16_bits_to_f32(bits_u16(out)).astype(np.float64)
    ref = oracle.bf16_bits_to_f32(o["out"]).astype(np.float64)
    # G within the FP8 tolerance can move an activation code by one step, so the
    # layer is compared in norm and elementwise against a bound scaled by the
    # row's magnitude
    assert np.linalg.norm(got - ref) <= 2e-2 * np.linalg.norm(ref)
    bound = TOL_REL * np.abs(ref) + TOL_ABS + 2e-2 * np.abs(ref).max(axis=1, keepdims=True)
    assert np.all(np.abs(got - ref) <= bound)


@pytest.mark.parametrize("variant,tile", [(3, 16), (3, 64), (1, 128), (1, 256)])
def test_int8_grouped_mm_exact_with_empty_and_uneven_experts(variant, tile):
    from quantized_linear_layers_group_b200 import qlin

    E, N, K = 6, 272, 384
    counts = np.array([0, 37, 1, 200, 0, 130])                   # empty experts and ragged groups
    offs = np.r_[0, np.cumsum(counts)].astype(np.int32)
    R = int(offs[-1])
    g = torch.Generator().manual_seed(9)
    a = torch.randn(R, K, generator=g).to(torch.bfloat16)
    wt = (torch.randn(E * N, K, generator=g) * 0.02).to(torch.bfloat16)
    aq, sa = oracle.quantize_per_token(oracle.FMT_INT8, a)
    wq, sw = oracle.quantize_per_token(oracle.FMT_INT8, wt)
    cdev = torch.full((R, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    qlin.qlin_moe_grouped_mm(qlin.QLIN_FMT_INT8, E, _dev(aq), _dev(sa), _dev(offs), _dev(wq), _dev(sw), cdev,
                             variant=variant, tile_n=tile)
    torch.cuda.synchronize()
    check_status()
    got = bits_u16(cdev)
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 > r0:
            ref = oracle.scaled_mm(oracle.FMT_INT8, aq[r0:r1], sa[r0:r1], wq[e * N:(e + 1) * N], sw[e * N:(e + 1) * N])
            assert_parity(oracle.FMT_INT8, got[r0:r1], ref, f"expert {e} variant {variant} tile {tile}")
