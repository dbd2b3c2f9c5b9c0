"""GPU parity of the routed experts on the FWHT128 grid against the CPU
oracle: expert ids, histogram, routing weights, the rotated x codes and
their bf16 group scales, the gated intermediate's rotated codes and group
scales, and the bf16 output, all bit for bit (the kernels take the oracle's
fp32 steps in its order: the butterflies stage by stage, each group's int32
product promoted with one fma in ascending group order, the k contributions
added in slot order)."""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import assert_bf16_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _rotate_experts(orc, w13b, w2b):
    """bf16 expert weights -> rotated group codes and bf16 scales, on the GPU
    and in the oracle (which must agree bit for bit)."""
    E, I2, H = w13b.shape
    I = I2 // 2
    g13 = w8a8.fwht128_quant(to_dev_bf16(w13b.reshape(E * I2, H)))
    g2 = w8a8.fwht128_quant(to_dev_bf16(w2b.reshape(E * H, I)))
    o13 = orc.fwht128_quant(w13b.reshape(E * I2, H))
    o2 = orc.fwht128_quant(w2b.reshape(E * H, I))
    assert np.array_equal(g13[0].cpu().numpy(), o13[0]) and np.array_equal(g2[0].cpu().numpy(), o2[0])
    assert np.array_equal(g13[1].view(torch.int16).cpu().numpy().view(np.uint16), o13[1])
    assert np.array_equal(g2[1].view(torch.int16).cpu().numpy().view(np.uint16), o2[1])
    gw = (g13[0].view(E, I2, H), g13[1].view(E, I2, H // 128), g2[0].view(E, H, I), g2[1].view(E, H, I // 128))
    ow = (o13[0].reshape(E, I2, H), o13[1].reshape(E, I2, H // 128), o2[0].reshape(E, H, I),
          o2[1].reshape(E, H, I // 128))
    return gw, ow


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _compare(orc, xb, lb, gw, ow, topk, tokens):
    y, dbg = w8a8.moe_g128_forward(to_dev_bf16(xb), to_dev_bf16(lb), *gw, topk, debug=True)
    y = from_dev_bf16(y)
    ids_all, _ = orc.route(lb, topk)
    E = gw[0].shape[0]
    assert np.array_equal(dbg["counts"].cpu().numpy(), np.bincount(ids_all.reshape(-1), minlength=E))
    assert np.array_equal(dbg["topk_ids"].cpu().numpy(), ids_all)
    ref = orc.moe_g128_forward(xb, lb, *ow, topk, tokens=tokens)
    t = ref["tokens"]
    assert np.array_equal(dbg["topk_w"].cpu().numpy()[t].view(np.uint32), ref["wts"].view(np.uint32))
    assert np.array_equal(dbg["qx"].cpu().numpy()[t], ref["qx"])
    assert np.array_equal(_bits(dbg["sx"])[t], ref["sx"])
    assert np.array_equal(dbg["qa"].cpu().numpy()[t], ref["qa"])
    assert np.array_equal(_bits(dbg["sa"])[t], ref["sa"])
    assert assert_bf16_close(y[t], ref["y32"], what="moe g128 y") == 1.0
    assert np.array_equal(y[t], ref["y"])


def _small(seed, T, E, H, I, skew=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if skew is not None:
        logits[:, skew] += 6.0
    w13 = inputs.weights(rng, (E, 2 * I, H))
    w2 = inputs.weights(rng, (E, H, I))
    return (inputs.to_bf16_bits(x), inputs.to_bf16_bits(logits), inputs.to_bf16_bits(w13),
            inputs.to_bf16_bits(w2))


@pytest.mark.parametrize("T,E,H,I,k,skew", [
    # token blocks of 16 rows (few rows per expert)
    (5, 8, 256, 128, 2, None), (1, 4, 128, 128, 4, None), (37, 8, 256, 128, 2, None),
    (9, 256, 2048, 512, 8, None),
    # 32- and 64-row blocks, several blocks per expert under skew
    (48, 8, 256, 128, 4, None), (64, 4, 256, 128, 2, None), (200, 8, 256, 256, 2, 2),
    # one group along H; an odd number of groups; the largest H and I
    (7, 8, 128, 128, 2, None), (100, 8, 384, 256, 4, None), (20, 8, 4096, 128, 2, None),
    (12, 4, 256, 2048, 2, None)])
def test_moe_g128_small_configs(orc, T, E, H, I, k, skew):
    xb, lb, w13, w2 = _small(T * 17 + E + H, T, E, H, I, skew)
    gw, ow = _rotate_experts(orc, w13, w2)
    _compare(orc, xb, lb, gw, ow, k, None)


def test_moe_g128_zero_token_row(orc):
    xb, lb, w13, w2 = _small(3, 6, 8, 256, 128)
    xb[4] = 0
    gw, _ = _rotate_experts(orc, w13, w2)
    y = from_dev_bf16(w8a8.moe_g128_forward(to_dev_bf16(xb), to_dev_bf16(lb), *gw, 2))
    assert not y[4].any() and y[3].any()


def test_moe_g128_rejects_bad_shapes():
    x = torch.zeros((2, 192), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((2, 4), dtype=torch.bfloat16, device="cuda")
    w13 = torch.zeros((4, 256, 192), dtype=torch.int8, device="cuda")
    s13 = torch.zeros((4, 256, 1), dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros((4, 192, 128), dtype=torch.int8, device="cuda")
    s2 = torch.zeros((4, 192, 1), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w8a8.W8A8Error):
        w8a8.moe_g128_forward(x, lg, w13, s13, w2, s2, 2)


@pytest.fixture(scope="module")
def full_experts(orc):
    w13, w2 = inputs.moe_weights(0)
    w13b, w2b = inputs.to_bf16_bits(w13), inputs.to_bf16_bits(w2)
    del w13, w2
    return _rotate_experts(orc, w13b, w2b)


@pytest.mark.parametrize("T", [1, 8, 512, 4096])
def test_moe_g128_full_size(orc, full_experts, T):
    gw, ow = full_experts
    xb, lb = inputs.moe_tokens(0, T)
    rng = np.random.default_rng(T)
    tokens = None if T <= 8 else np.unique(np.concatenate([rng.integers(0, T, 24), [0, T - 1]]))
    _compare(orc, xb, lb, gw, ow, 8, tokens)


def test_moe_g128_full_size_extreme_skew(orc, full_experts):
    """Every token's logits favour the same 8 experts: 512 rows each for those,
    none for the rest."""
    gw, ow = full_experts
    xb, lb = inputs.moe_tokens(5, 512)
    lf = inputs.bf16_bits_to_f32(lb).copy()
    lf[:, [3, 17, 64, 65, 128, 200, 254, 255]] += 8.0
    lb = inputs.to_bf16_bits(lf)
    tokens = np.unique(np.concatenate([np.random.default_rng(11).integers(0, 512, 20), [0, 511]]))
    _compare(orc, xb, lb, gw, ow, 8, tokens)


@pytest.mark.parametrize("T,E,k", [(1, 8, 1), (3, 2, 2), (16, 256, 8)])
def test_moe_g128_degenerate_routing(orc, T, E, k):
    """top-1 of 8, every expert of 2 selected, and 16 tokens over 256 experts."""
    xb, lb, w13, w2 = _small(T * 5 + E, T, E, 256, 128)
    gw, ow = _rotate_experts(orc, w13, w2)
    _compare(orc, xb, lb, gw, ow, k, None)
