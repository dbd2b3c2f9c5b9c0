"""The allocation-free linear: same output as w8a8_linear.

Callers that cannot allocate device memory while the layer runs (a locked
allocator, a host that only passes its input and output buffers) use
w8a8_linear_noalloc, which keeps its scratch in the library's static device
array.  This file runs last so that, after the rest of the suite, it also
checks that the shared array's leftover contents do not leak into results.
"""
import ctypes

import numpy as np
import pytest
import torch

from moe_gemm_absmax_b200 import inputs, w8a8
from tests._util import bits_to_f64, bf16_ulp, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _weights(N, K, seed):
    w = inputs.weights(np.random.default_rng(seed), (N, K))
    return w8a8.quant_rows_f32(torch.from_numpy(w).cuda())


@pytest.mark.parametrize("M,N,K", [(8, 5120, 17408), (1, 34816, 5120), (5, 1024, 2048), (200, 1024, 5120)])
def test_noalloc_equals_linear_two_calls(M, N, K):
    xb = inputs.dense_linear(M + N, M, K, 16, with_weights=False)[0]
    x = to_dev_bf16(xb)
    qw, sw = _weights(N, K, M * 3 + K)
    L = w8a8.lib()
    assert L.w8a8_linear_noalloc_scratch_size(M, N, K) <= w8a8.NOALLOC_SCRATCH_BYTES
    ref = from_dev_bf16(w8a8.linear(x, qw, sw))
    for _ in range(2):
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        rc = L.w8a8_linear_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(qw.data_ptr()),
                                   ctypes.c_void_p(sw.data_ptr()), ctypes.c_void_p(y.data_ptr()), M, N, K,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == w8a8.OK
        got = from_dev_bf16(y)
        r = bits_to_f64(ref)
        assert np.all(np.abs(bits_to_f64(got) - r) <= bf16_ulp(r))
        assert np.array_equal(got, ref)
    assert w8a8.get_device_error() == (w8a8.OK, 0)


def test_noalloc_rejects_sizes_beyond_the_array():
    M, N, K = 4096, 256, 5120          # codes alone need 20 MiB
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    qw = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    with pytest.raises(w8a8.W8A8Error) as e:
        w8a8.linear_noalloc(x, qw, sw)
    assert e.value.status == w8a8.ERR_UNSUPPORTED
