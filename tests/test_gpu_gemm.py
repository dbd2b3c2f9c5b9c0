"""GPU parity of the dense W8A8 path: int32 accumulators bit for bit
(tcgen05 GEMM and weight-streaming GEMV), bf16 dequant outputs within one
bf16 ulp of the oracle's fp32 value, at small ragged shapes and at the
workload shapes (decode in full, prefill at M = 512 in full and at M = 4096
on sampled outputs)."""
import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import assert_bf16_close, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _rand_codes(rng, r, c):
    return rng.integers(-127, 128, (r, c), dtype=np.int8)


@pytest.mark.parametrize("path", [w8a8.PATH_TCGEN05, w8a8.PATH_GEMV])
@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (3, 48, 96), (8, 512, 528), (13, 272, 1040), (32, 512, 5120),
                                   (3, 40, 96), (17, 136, 2064), (8, 1152, 17408)])
def test_gemm_s32_small(orc, path, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    a, b = _rand_codes(rng, M, K), _rand_codes(rng, N, K)
    acc = w8a8.gemm_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), path).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(a, b))


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (200, 520, 1040), (1000, 264, 2064), (384, 768, 4096),
                                   (129, 1024, 256), (3, 40, 96), (1, 8, 16)])
def test_gemm_s32_tcgen05_tiles_and_tails(orc, M, N, K):
    rng = np.random.default_rng(M + N * 3 + K)
    a, b = _rand_codes(rng, M, K), _rand_codes(rng, N, K)
    acc = w8a8.gemm_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), w8a8.PATH_TCGEN05).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(a, b))


def test_gemm_s32_extreme_codes(orc):
    K = 17408
    a = np.full((130, K), 127, np.int8)
    a[1::2] = -127
    b = np.full((272, K), 127, np.int8)
    acc = w8a8.gemm_s32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), w8a8.PATH_TCGEN05).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(a, b))
    acc = w8a8.gemm_s32(torch.from_numpy(a[:8]).cuda(), torch.from_numpy(b).cuda(), w8a8.PATH_GEMV).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(a[:8], b))


def _quantized(orc, seed, M, K, N):
    xb, w = inputs.dense_linear(seed, M, K, N)
    qw, sw = orc.quant_rows_f32(w)
    return xb, qw, sw


def test_linear_tiny_config(orc):
    xb, w = inputs.tiny_linear(0)
    qw, sw = orc.quant_rows_f32(w)
    y = w8a8.linear(to_dev_bf16(xb), torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda())
    yo, y32, _, _ = orc.linear(xb, qw, sw)
    exact = assert_bf16_close(from_dev_bf16(y), y32, what="tiny")
    assert exact == 1.0
    for path in (w8a8.PATH_TCGEN05, w8a8.PATH_GEMV):
        qx, sx = orc.quant_rows_bf16(xb)
        y2 = w8a8.gemm_q(torch.from_numpy(qx).cuda(), torch.from_numpy(sx).cuda(), torch.from_numpy(qw).cuda(),
                         torch.from_numpy(sw).cuda(), path)
        assert np.array_equal(from_dev_bf16(y2), yo)


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("shape", ["gate_up", "down"])
def test_linear_decode_full_size(orc, M, shape):
    d = inputs.GATE_UP if shape == "gate_up" else inputs.DOWN
    xb, qw, sw = _quantized(orc, 100 + M, M, d["K"], d["N"])
    y = w8a8.linear(to_dev_bf16(xb), torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda())
    yo, y32, _, _ = orc.linear(xb, qw, sw)
    exact = assert_bf16_close(from_dev_bf16(y), y32, what=f"decode {shape} M={M}")
    assert exact == 1.0


@pytest.mark.parametrize("M", [512, 4096])
@pytest.mark.parametrize("shape", ["gate_up", "down"])
def test_linear_prefill_full_size_sampled(orc, M, shape):
    d = inputs.GATE_UP if shape == "gate_up" else inputs.DOWN
    K, N = d["K"], d["N"]
    rng = np.random.default_rng(M + K)
    xb = inputs.dense_linear(200 + M, M, K, 16, with_weights=False)[0]
    w = inputs.weights(rng, (N, K))
    qw, sw = orc.quant_rows_f32(w)
    y = from_dev_bf16(w8a8.linear(to_dev_bf16(xb), torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda()))
    qx, sx = orc.quant_rows_bf16(xb)
    ms = np.concatenate([rng.integers(0, M, 3000), [0, M - 1, 127, 128, M - 1]])
    ns = np.concatenate([rng.integers(0, N, 3000), [0, N - 1, 255, 256, 0]])
    acc = orc.gemm_s32_at(qx, qw, ms, ns)
    y32 = (acc.astype(np.float32) * sx[ms]) * sw[ns]
    exact = assert_bf16_close(y[ms, ns], y32, what=f"prefill {shape} M={M}")
    assert exact == 1.0


@pytest.mark.parametrize("shape", ["gate_up", "down"])
def test_linear_prefill_m512_every_output(orc, shape):
    """Every output of the prefill shape at M = 512 (2.6 M / 17.8 M values),
    so that every tile of every wave of the persistent pair-tile scheduler is
    compared, not a sample."""
    d = inputs.GATE_UP if shape == "gate_up" else inputs.DOWN
    K, N, M = d["K"], d["N"], 512
    rng = np.random.default_rng(M + K + 1)
    xb = inputs.dense_linear(300 + M, M, K, 16, with_weights=False)[0]
    qw, sw = orc.quant_rows_f32(inputs.weights(rng, (N, K)))
    y = from_dev_bf16(w8a8.linear(to_dev_bf16(xb), torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda()))
    yo, y32, _, _ = orc.linear(xb, qw, sw)
    assert assert_bf16_close(y, y32, what=f"prefill {shape} M=512, every output") == 1.0
    assert np.array_equal(y, yo)


def test_linear_pair_tile_odd_k_blocks(orc):
    """The 144-column pair tile (chosen for N = 5120 at M = 512) loads two
    128-byte k blocks per ring stage; with K = 17280 (135 k blocks) its last
    stage's second block lies past K and must add nothing.  Every output."""
    M, N, K = 512, 5120, 17280
    rng = np.random.default_rng(17)
    xb = inputs.dense_linear(41, M, K, 16, with_weights=False)[0]
    qw, sw = orc.quant_rows_f32(inputs.weights(rng, (N, K)))
    y = from_dev_bf16(w8a8.linear(to_dev_bf16(xb), torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda()))
    yo, y32, _, _ = orc.linear(xb, qw, sw)
    assert assert_bf16_close(y, y32, what="pair tile, odd k blocks") == 1.0
    assert np.array_equal(y, yo)


def test_linear_prefill_ragged_rows(orc):
    xb, qw, sw = _quantized(orc, 5, 300, 1024, 776)
    y = w8a8.linear(to_dev_bf16(xb), torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda())
    yo, y32, _, _ = orc.linear(xb, qw, sw)
    assert assert_bf16_close(from_dev_bf16(y), y32, what="ragged") == 1.0


def test_gemv_rejects_more_than_32_tokens():
    a = torch.zeros(33, 96, dtype=torch.int8, device="cuda")
    b = torch.zeros(40, 96, dtype=torch.int8, device="cuda")
    with pytest.raises(w8a8.W8A8Error) as e:
        w8a8.gemm_s32(a, b, w8a8.PATH_GEMV)
    assert e.value.status == w8a8.ERR_UNSUPPORTED
    assert w8a8.gemm_s32(a, b).shape == (33, 40)


def test_linear_repeated_calls_and_workspace_reuse(orc):
    """Split-K counters are left zero, so back-to-back calls sharing a workspace agree."""
    xb, qw, sw = _quantized(orc, 9, 8, inputs.DOWN["K"], 1024)
    x, qwd, swd = to_dev_bf16(xb), torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda()
    ws = torch.empty(w8a8.linear_workspace_size(8, 1024, inputs.DOWN["K"]), dtype=torch.uint8, device="cuda")
    ys = [from_dev_bf16(w8a8.linear(x, qwd, swd, ws=ws)) for _ in range(3)]
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[1], ys[2])
    assert np.array_equal(ys[0], orc.linear(xb, qw, sw)[0])
