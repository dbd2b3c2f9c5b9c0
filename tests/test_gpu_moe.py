"""GPU parity of the routed W8A8 MoE layer (a5 .. a11) against the CPU
oracle: expert ids, histogram, routing weights, x codes, the gated
intermediate's codes and scales bit for bit; the bf16 output bit for bit
while the slot-order combine is used (the kernels take the oracle's fp32
steps in the oracle's order), and for the large-T atomic combine within one
bf16 ulp plus the bound on reordering a sum of k fp32 terms."""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import assert_bf16_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _quant_experts_gpu(w13, w2):
    q13, s13 = w8a8.quant_rows_f32(_dev(w13))
    q2, s2 = w8a8.quant_rows_f32(_dev(w2))
    return q13, s13, q2, s2


def _quant_experts_orc(orc, w13, w2):
    E, I2, H = w13.shape
    q13, s13 = orc.quant_rows_f32(w13.reshape(E * I2, H))
    q2, s2 = orc.quant_rows_f32(w2.reshape(E * H, -1))
    return q13.reshape(w13.shape), s13.reshape(E, I2), q2.reshape(w2.shape), s2.reshape(E, H)


def _compare(orc, xb, lb, gpu_w, orc_w, topk, tokens, exact=None):
    q13, s13, q2, s2 = gpu_w
    y, dbg = w8a8.moe_forward(to_dev_bf16(xb), to_dev_bf16(lb), q13, s13, q2, s2, topk, debug=True)
    y = from_dev_bf16(y)
    ids_all, _ = orc.route(lb, topk)
    E = q13.shape[0]
    assert np.array_equal(dbg["counts"].cpu().numpy(), np.bincount(ids_all.reshape(-1), minlength=E))
    assert np.array_equal(dbg["topk_ids"].cpu().numpy(), ids_all)
    ref = orc.moe_forward(xb, lb, *orc_w, topk, tokens=tokens)
    t = ref["tokens"]
    assert np.array_equal(dbg["topk_ids"].cpu().numpy()[t], ref["ids"])
    assert np.array_equal(dbg["topk_w"].cpu().numpy()[t].view(np.uint32), ref["wts"].view(np.uint32))
    assert np.array_equal(dbg["qx"].cpu().numpy()[t], ref["qx"])
    assert np.array_equal(dbg["sx"].cpu().numpy()[t].view(np.uint32), ref["sx"].view(np.uint32))
    assert np.array_equal(dbg["qa"].cpu().numpy()[t], ref["qa"])
    assert np.array_equal(dbg["sa"].cpu().numpy()[t].view(np.uint32), ref["sa"].view(np.uint32))
    H = xb.shape[1]
    if exact is None:
        exact = xb.shape[0] * topk * H * 4 <= 64 << 20
    if exact:
        # slot-order combine: the oracle's fp32 steps exactly
        assert assert_bf16_close(y[t], ref["y32"], what="moe y") == 1.0
        assert np.array_equal(y[t], ref["y"])
    else:
        # large T: fp32 atomics, the k contributions added in some order
        assert_bf16_close(y[t], ref["y32"], extra=2.0 ** -18 * ref["yabs"].astype(np.float64), what="moe y")


def _small(seed, T, E, H, I, skew=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if skew is not None:
        logits[:, skew] += 6.0
    w13 = inputs.weights(rng, (E, 2 * I, H))
    w2 = inputs.weights(rng, (E, H, I))
    return inputs.to_bf16_bits(x), inputs.to_bf16_bits(logits), w13, w2


@pytest.mark.parametrize("T,E,H,I,k,skew", [(5, 8, 256, 64, 2, None), (37, 8, 256, 64, 2, None),
                                             (40, 16, 512, 128, 2, 3), (1, 4, 128, 64, 4, None),
                                             (9, 256, 2048, 512, 8, None),
                                             # swap-AB expert GEMMs: token blocks of 16 / 32 / 64 rows,
                                             # several blocks per expert under skew, I up to 2048,
                                             # a single 128-column group (H = 128)
                                             (48, 8, 256, 128, 4, None), (64, 4, 256, 128, 2, None),
                                             (100, 8, 256, 128, 4, None), (200, 8, 256, 128, 2, 2),
                                             (12, 4, 256, 2048, 2, None), (7, 8, 128, 128, 2, None),
                                             # 128-row tile path: more rows per expert
                                             (300, 4, 256, 128, 2, 1), (520, 8, 512, 256, 3, 5)])
def test_moe_small_configs(orc, T, E, H, I, k, skew):
    xb, lb, w13, w2 = _small(T * 31 + E, T, E, H, I, skew)
    gw = _quant_experts_gpu(w13, w2)
    ow = _quant_experts_orc(orc, w13, w2)
    assert np.array_equal(gw[0].cpu().numpy(), ow[0]) and np.array_equal(gw[2].cpu().numpy(), ow[2])
    _compare(orc, xb, lb, gw, ow, k, None)


def test_moe_zero_token_row(orc):
    xb, lb, w13, w2 = _small(3, 6, 8, 256, 64)
    xb[4] = 0
    gw = _quant_experts_gpu(w13, w2)
    y = from_dev_bf16(w8a8.moe_forward(to_dev_bf16(xb), to_dev_bf16(lb), *gw, 2))
    assert not y[4].any()


@pytest.fixture(scope="module")
def full_experts(orc):
    w13, w2 = inputs.moe_weights(0)
    gw = _quant_experts_gpu(w13, w2)
    ow = _quant_experts_orc(orc, w13, w2)
    assert np.array_equal(gw[0].cpu().numpy(), ow[0]) and np.array_equal(gw[1].cpu().numpy(), ow[1])
    assert np.array_equal(gw[2].cpu().numpy(), ow[2]) and np.array_equal(gw[3].cpu().numpy(), ow[3])
    del w13, w2
    return gw, ow


@pytest.mark.parametrize("T", [1, 8, 512, 4096])
def test_moe_full_size(orc, full_experts, T):
    gw, ow = full_experts
    xb, lb = inputs.moe_tokens(0, T)
    rng = np.random.default_rng(T)
    tokens = None if T <= 8 else np.unique(np.concatenate([rng.integers(0, T, 24), [0, T - 1]]))
    _compare(orc, xb, lb, gw, ow, 8, tokens)


def test_moe_full_size_exact_combine_t4096(orc, full_experts):
    """With the slot-order combine forced at every T, the T = 4096 layer is
    bit-exact with the oracle's bf16 on the sampled tokens."""
    gw, ow = full_experts
    xb, lb = inputs.moe_tokens(0, 4096)
    tokens = np.unique(np.concatenate([np.random.default_rng(41).integers(0, 4096, 24), [0, 4095]]))
    prev = w8a8.moe_set_combine(w8a8.MOE_COMBINE_EXACT)
    try:
        _compare(orc, xb, lb, gw, ow, 8, tokens, exact=True)
    finally:
        w8a8.moe_set_combine(prev)


def test_moe_full_size_every_token_t512(orc, full_experts):
    """Every token of the layer at T = 512 (4096 sorted rows over all 256
    experts), not a sample: every token block of every expert."""
    gw, ow = full_experts
    xb, lb = inputs.moe_tokens(0, 512)
    _compare(orc, xb, lb, gw, ow, 8, None)


def test_moe_full_size_extreme_skew(orc, full_experts):
    """Every token's logits favour the same 8 experts: 512 rows each for those
    (many token blocks per expert on the swap-AB path), 0 for the other 248."""
    gw, ow = full_experts
    xb, lb = inputs.moe_tokens(5, 512)
    lf = inputs.bf16_bits_to_f32(lb).copy()
    lf[:, [3, 17, 64, 65, 128, 200, 254, 255]] += 8.0
    lb = inputs.to_bf16_bits(lf)
    tokens = np.unique(np.concatenate([np.random.default_rng(11).integers(0, 512, 20), [0, 511]]))
    _compare(orc, xb, lb, gw, ow, 8, tokens)
