"""Pins for the oracle's prefill-chunk product (CPU only)."""
import numpy as np

import synth
from oracle import prefill as op
from oracle import qgemv as oq


def test_prefill_equals_independent_gemvs():
    T, N, K = 5, 40, 128
    W = synth.q4_0_matrix(N, K, 1, "pf").numpy()
    X = synth.normal_f16(1, 2, T * K).numpy().reshape(T, K)
    Y = op.prefill_f64(oq.FMT_Q4_0, W, X, N, K)
    for t in range(T):
        np.testing.assert_allclose(Y[t], oq.qgemv(oq.FMT_Q4_0, W, X[t].astype(np.float64), N, K),
                                   rtol=1e-12, atol=1e-12)


def test_prefill_tiny_triple_loop():
    T, N, K = 2, 3, 32
    W = synth.q4_0_matrix(N, K, 2, "pf2").numpy()
    X = synth.normal_f16(2, 3, T * K).numpy().reshape(T, K)
    Y = op.prefill(oq.FMT_Q4_0, W, X, N, K)
    raw = W.reshape(N, 18)
    for t in range(T):
        for n in range(N):
            d = float(raw[n, 0:2].view(np.float16)[0])
            acc = 0.0
            for i in range(K):
                byte = int(raw[n, 2 + i // 2])
                q = (byte & 0xF) if i % 2 == 0 else (byte >> 4)
                acc += float(X[t, i]) * d * (q - 8)
            assert Y[t, n] == np.float16(acc)


def test_prefill_output_is_fp16_round_to_nearest():
    T, N, K = 3, 17, 64
    W = synth.q4_0_matrix(N, K, 3, "pf3").numpy()
    X = synth.normal_f16(3, 4, T * K).numpy().reshape(T, K)
    Y = op.prefill(oq.FMT_Q4_0, W, X, N, K)
    Yd = op.prefill_f64(oq.FMT_Q4_0, W, X, N, K)
    assert Y.dtype == np.float16
    # |Y - Yd| is at most half an fp16 ulp of Y
    ulp = np.spacing(np.abs(Y).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(Y.astype(np.float64) - Yd) <= 0.5 * ulp + 1e-300)
