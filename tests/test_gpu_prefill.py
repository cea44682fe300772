"""GPU parity of the tcgen05 prefill-chunk GEMM (Q4_0 weights, fp16 activations) against the
oracle (float64 products of the exact dequantized weights, one rounding to fp16)."""
import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
import synth
from oracle import prefill as op
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu

# (tokens, n, k): the three prefill configurations, partial token tiles, a partial feature
# tile, the smallest k, and shapes that exercise each k-split (cluster) size.
SHAPES = [(128, 1024, 4096), (128, 4096, 4096), (128, 14336, 4096), (1, 1024, 4096), (37, 144, 768),
          (100, 16, 256), (128, 272, 1280), (64, 2048, 2048)]


@pytest.mark.parametrize("tokens,n,k", SHAPES)
def test_prefill_matches_oracle(tokens, n, k):
    need_gpu()
    name = f"pf/{tokens}x{n}x{k}"
    W = synth.q4_0_matrix(n, k, 0, name + "/W")
    X = synth.normal_f16(0, synth.stream_id(name + "/X"), tokens * k).view(tokens, k)
    Y = bqg.qgemm_prefill(bqg.Q4_0, W.cuda(), X.cuda(), n, k)
    torch.cuda.synchronize()
    ref = op.prefill_f64(2, W.numpy(), X.numpy(), n, k)
    assert Y.dtype == torch.float16 and tuple(Y.shape) == (tokens, n)
    assert_close(Y.float(), ref, what=f"prefill {tokens}x{n}x{k}")
    # fp16 weights (one rounding of (q-8)*d) and one fp16 rounding of the output: the error stays
    # near the output's own half-ulp (2^-11 relative), well inside the tolerance
    assert_close(Y.float(), ref, tol=1e-3, what=f"prefill {tokens}x{n}x{k} (fp16 accuracy)")


def test_prefill_deterministic():
    need_gpu()
    n, k = 1024, 4096   # 8-way k split over a cluster
    W = synth.q4_0_matrix(n, k, 1, "pf/det").cuda()
    X = synth.normal_f16(1, 2, 128 * k).view(128, k).cuda()
    a = bqg.qgemm_prefill(bqg.Q4_0, W, X, n, k)
    b = bqg.qgemm_prefill(bqg.Q4_0, W, X, n, k)
    assert torch.equal(a, b)


def test_prefill_equals_gemv_rows():
    """Each token row of the prefill product is that token's GEMV (same weights)."""
    need_gpu()
    n, k, tokens = 512, 1024, 5
    W = synth.q4_0_matrix(n, k, 2, "pf/gemv").cuda()
    X = synth.normal_f16(2, 3, tokens * k).view(tokens, k).cuda()
    Y = bqg.qgemm_prefill(bqg.Q4_0, W, X, n, k).float()
    for t in range(tokens):
        y = bqg.qgemv(bqg.Q4_0, W, X[t].float().contiguous(), n, k)
        assert_close(Y[t], y.cpu().numpy(), tol=2e-3, what=f"row {t}")
