"""GPU parity of the MoE layer on the tensor-core path (grouped expert GEMM on tcgen05) against
the float64 oracle, through the C ABI, and against the CUDA-core path on the same inputs.

The shapes cover every weight format as routed and as shared expert, rows whose byte length
needs 1, 2 or 4 rows per tensor-map super-row, partial 128-row tiles, experts with more than 64
tokens (several token chunks per item) and the full-size Gemma-like and GLM-like geometry.

Two variants: kind::f16 (Q8_0, Q4_0 and int4 weights dequantized to fp16) and kind::i8 (layers
whose every family is int4 or int2 with k a multiple of 128: weights as exact unsigned bytes,
activations as 16-bit fixed-point digit pairs, int32 accumulation).

Tolerance: the benchmark spec's bound 2e-3 * max|y_ref|, and a stricter bound derived from the
arithmetic of each variant.  kind::f16: weights become fp16 with one rounding of (q - 8) * d or
q * d (relative error <= 2^-11; int4 values are exact), x and h become fp16 (<= 2^-11 each),
products accumulate in fp32.  The errors are independent per product, so a dot product's error
is about 2^-11 * sqrt(2) times the root-sum-square of its terms; through gate/up, the activation
and down this stays near 4e-4 of max|y| (measured: see the per-test assertions), hence 1e-3.
kind::i8: the sums over integers are exact; each x and h element carries a rounding error of at
most max|row| / 65278 (16-bit fixed point per row), i.e. ~1.5e-5 of the row's largest element,
and fp32 rounding of the scaled sums adds ~1e-7.  Relative to max|y| the row errors grow by the
row's max / rms ratio, up to ~10 for the gated products h = act(g) * u, hence 3e-4 (measured up
to 1.6e-4 over the specs below).
"""
import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
from synth import workloads as wl
from oracle import moe as om
from tests.moe_util import device_layer, oracle_layer, oracle_router_logits
from tests.util import assert_close, max_rel_err, need_gpu

pytestmark = pytest.mark.gpu

TC_TOL = 1e-3
I8_TOL = 3e-4


def i8_variant(spec) -> bool:
    """True when the tensor-core path takes the kind::i8 variant for this layer."""
    fams = [(spec.expert_fmt, spec.hidden), (spec.expert_fmt, spec.inter)]
    if spec.shared_inter:
        fams += [(spec.shared_fmt, spec.shared_inter)]
    return all(f in (bqg.I4_ROW, bqg.I2_ROW) and k % 128 == 0 for f, k in fams) and spec.hidden % 128 == 0

TC_SPECS = [
    # hidden, inter, shared_inter multiples of 64; rows of 1584 / 216 / 72 bytes etc.
    wl.MoESpec("tc_q4_gelu_shared", 8, 2, 256, 128, bqg.Q4_0, bqg.ACT_GELU_TANH, 192, bqg.Q8_0, False),
    wl.MoESpec("tc_q8_silu", 6, 3, 192, 320, bqg.Q8_0, bqg.ACT_SILU, 0, 0, False),
    wl.MoESpec("tc_i4_silu", 16, 8, 256, 128, bqg.I4_ROW, bqg.ACT_SILU, 0, 0, False),
    # Q4_0 rows of 704 values (396 bytes: 4 rows per super-row), down rows 320 = 256 + a partial tile
    wl.MoESpec("tc_q4_rows704", 5, 5, 320, 704, bqg.Q4_0, bqg.ACT_GELU_TANH, 0, 0, False),
    wl.MoESpec("tc_i4_shared_q8", 12, 4, 192, 128, bqg.I4_ROW, bqg.ACT_GELU_TANH, 128, bqg.Q8_0, False),
    wl.MoESpec("tc_q8_shared_q4", 4, 2, 128, 384, bqg.Q8_0, bqg.ACT_SILU, 448, bqg.Q4_0, False),
    # kind::i8 layers: int2 routed; int4 with an int4 shared expert; int2 with an int4 shared expert;
    # three 128-k stages and a down matrix of 384 rows (a 256-row item, then a one-tile item)
    wl.MoESpec("tc8_i2_silu", 8, 2, 256, 128, bqg.I2_ROW, bqg.ACT_SILU, 0, 0, False),
    wl.MoESpec("tc8_i4_shared_i4", 10, 3, 256, 256, bqg.I4_ROW, bqg.ACT_GELU_TANH, 128, bqg.I4_ROW, False),
    wl.MoESpec("tc8_i2_shared_i4", 6, 2, 384, 128, bqg.I2_ROW, bqg.ACT_SILU, 256, bqg.I4_ROW, False),
    wl.MoESpec("tc8_i4_rows384", 5, 2, 384, 384, bqg.I4_ROW, bqg.ACT_SILU, 0, 0, False),
    # int4 with inter 192 (not a multiple of 128): the kind::f16 variant
    wl.MoESpec("tc_i4_f16_inter192", 4, 2, 256, 192, bqg.I4_ROW, bqg.ACT_SILU, 0, 0, False),
    # inter 64: the down matrix's only stage is half a 128-k stage (four k steps, one per partial
    # accumulator); Q4_0 rows of 64 values are 36 bytes (4 rows per super-row)
    wl.MoESpec("tc_q4_inter64", 6, 2, 128, 64, bqg.Q4_0, bqg.ACT_SILU, 0, 0, False),
]


def _layer(spec, path, seed=0):
    L = wl.build_moe_layer(spec, seed, 0, device="cuda")
    return L, device_layer(L).with_path(path)


def _route(spec, seed, tokens):
    lg = wl.moe_logits(spec, seed, 0, tokens)
    idx, w = bqg.moe_router_topk(lg.cuda(), spec.top_k)
    ridx, rw = om.router_topk(lg.numpy(), spec.top_k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    return idx, w, ridx, rw


@pytest.mark.parametrize("spec", TC_SPECS, ids=lambda s: s.name)
@pytest.mark.parametrize("tokens", [1, 16, 40, 100, 200])
def test_tc_small_matches_oracle(spec, tokens):
    need_gpu()
    L, lay = _layer(spec, bqg.MOE_PATH_TENSOR_CORES)
    x = wl.moe_tokens(spec, 0, tokens)
    idx, w, ridx, rw = _route(spec, 0, tokens)
    y = bqg.moe_forward(lay, x.cuda(), idx, w)
    torch.cuda.synchronize()
    ref = om.moe_layer(oracle_layer(spec, 0, 0), x.numpy(), ridx, rw)
    assert_close(y, ref, what=f"{spec.name} T={tokens}")
    e = assert_close(y, ref, tol=TC_TOL, what=f"{spec.name} T={tokens} (fp16 operands)")
    if i8_variant(spec):
        assert_close(y, ref, tol=I8_TOL, what=f"{spec.name} T={tokens} (int8 digits)")
    print(f"{spec.name} T={tokens}: max rel err {e:.2e}")
    assert bqg.bqg_device_errors() == 0


@pytest.mark.parametrize("spec", TC_SPECS[:3], ids=lambda s: s.name)
def test_tc_agrees_with_cuda_core_path(spec):
    """Both expert paths on the same inputs; and the automatic choice takes the tensor cores
    from BQG_MOE_TC_MIN_TOKENS tokens on."""
    need_gpu()
    L, tc = _layer(spec, bqg.MOE_PATH_TENSOR_CORES)
    cc = tc.with_path(bqg.MOE_PATH_CUDA_CORES)
    auto = tc.with_path(bqg.MOE_PATH_AUTO)
    tokens = 24
    x = wl.moe_tokens(spec, 5, tokens).cuda()
    idx, w, _, _ = _route(spec, 5, tokens)
    y_tc = bqg.moe_forward(tc, x, idx, w)
    y_cc = bqg.moe_forward(cc, x, idx, w)
    y_auto = bqg.moe_forward(auto, x, idx, w)
    torch.cuda.synchronize()
    assert torch.equal(y_auto, y_tc)
    assert_close(y_tc, y_cc.cpu().numpy(), tol=TC_TOL, what="tensor-core vs CUDA-core path")


def test_tc_deterministic_and_identical_experts():
    """Identical experts: y = FFN(x) for any routing; two calls give identical bits."""
    need_gpu()
    spec = wl.MoESpec("tc_same", 4, 2, 128, 64, bqg.Q4_0, bqg.ACT_GELU_TANH, 0, 0, False)
    L = wl.build_moe_layer(spec, 1, 0, device="cuda")
    for fam, stride in ((L.gate, L.gate_stride), (L.up, L.up_stride), (L.down, L.down_stride)):
        for e in range(1, 4):
            fam[e * stride:(e + 1) * stride] = fam[0:stride]
    lay = device_layer(L).with_path(bqg.MOE_PATH_TENSOR_CORES)
    x = wl.moe_tokens(spec, 1, 33).cuda()
    idx, w = bqg.moe_router_topk(wl.moe_logits(spec, 1, 0, 33).cuda(), 2)
    y1 = bqg.moe_forward(lay, x, idx, w)
    y2 = bqg.moe_forward(lay, x, idx, w)
    assert torch.equal(y1, y2)
    ex = oracle_layer(spec, 1, 0).expert(0)
    ref = om.ffn_dense(ex, 64, 128, spec.act, x.cpu().numpy())
    assert_close(y1, ref, tol=TC_TOL, what="identical experts")


def test_tc_invalid_expert_id_is_skipped_and_flagged():
    need_gpu()
    spec = TC_SPECS[2]
    L, lay = _layer(spec, bqg.MOE_PATH_TENSOR_CORES)
    tokens = 20
    x = wl.moe_tokens(spec, 0, tokens)
    idx, w, ridx, rw = _route(spec, 0, tokens)
    bqg.bqg_device_errors()
    bad = idx.clone()
    bad[3, 2] = 999
    bad[11, 0] = -1
    y = bqg.moe_forward(lay, x.cuda(), bad, w)
    assert bqg.bqg_device_errors() & bqg.DEVERR_EXPERT_ID
    rw = rw.copy()
    rw[3, 2] = 0.0
    rw[11, 0] = 0.0
    ref = om.moe_layer(oracle_layer(spec, 0, 0), x.numpy(), ridx, rw)
    assert_close(y, ref, tol=TC_TOL, what="invalid ids skipped")


def test_tc_rejects_unsupported_shapes():
    """Forcing the tensor cores on a layer whose inter is not a multiple of 64 is refused
    before any launch; the automatic choice then stays on the CUDA cores."""
    need_gpu()
    spec = wl.MoESpec("tc_bad", 4, 2, 128, 96, bqg.Q4_0, bqg.ACT_SILU, 0, 0, False)
    L, lay = _layer(spec, bqg.MOE_PATH_TENSOR_CORES)
    x = torch.zeros(20, 128, device="cuda")
    idx = torch.zeros(20, 2, dtype=torch.int32, device="cuda")
    w = torch.zeros(20, 2, device="cuda")
    with pytest.raises(bqg.BQGError) as e:
        bqg.moe_forward(lay, x, idx, w)
    assert e.value.status == -3
    y = bqg.moe_forward(lay.with_path(bqg.MOE_PATH_AUTO), x, idx, w)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0


def _near_tie_ok(lg_ref, gidx, ridx):
    for t in np.nonzero((gidx != ridx).any(axis=1))[0]:
        a, b = set(gidx[t]) - set(ridx[t]), set(ridx[t]) - set(gidx[t])
        for e1, e2 in zip(sorted(a), sorted(b)):
            if abs(lg_ref[t, e1] - lg_ref[t, e2]) > 1e-5 * (1 + abs(lg_ref[t, e2])):
                return False
    return True


@pytest.mark.parametrize("tokens", [16, 128])
def test_gemma_like_prefill_chunk_every_token(tokens):
    """The MoE prefill chunk: hidden 2816, 128 Q4_0 GeGLU experts of 704, top-8, shared Q8_0 expert
    of 2112, fp32 router; every token compared (the automatic path takes the tensor cores)."""
    need_gpu()
    spec = wl.GEMMA_MOE
    L = wl.build_moe_layer(spec, 0, 0, device="cuda")
    x = wl.moe_tokens(spec, 0, tokens)
    lg = bqg.moe_router_logits(L.R, x.cuda())
    idx, w = bqg.moe_router_topk(lg, spec.top_k)
    lay = device_layer(L)
    y = bqg.moe_forward(lay, x.cuda(), idx, w)
    y_cc = bqg.moe_forward(lay.with_path(bqg.MOE_PATH_CUDA_CORES), x.cuda(), idx, w)
    torch.cuda.synchronize()
    lg_ref = oracle_router_logits(spec, 0, 0, x.numpy())
    ridx, rw = om.router_topk(lg_ref, spec.top_k)
    gidx = idx.cpu().numpy()
    assert _near_tie_ok(lg_ref, gidx, ridx)
    same = (gidx == ridx).all(axis=1)
    assert same.sum() >= max(1, int(0.95 * tokens))
    ref = om.moe_layer(oracle_layer(spec, 0, 0), x.numpy(), ridx, rw)
    assert_close(y.cpu().numpy()[same], ref[same], what=f"gemma-like chunk T={tokens}")
    e = assert_close(y.cpu().numpy()[same], ref[same], tol=TC_TOL, what=f"gemma-like chunk T={tokens} (fp16)")
    print(f"gemma-like T={tokens}: max rel err {e:.2e}")
    # the whole chunk (near-tie tokens included) agrees with the CUDA-core path on the same routing
    assert_close(y, y_cc.cpu().numpy(), tol=TC_TOL, what="tensor-core vs CUDA-core path")


def test_glm_like_geometry_every_token_t64():
    """The GLM-like kernel geometry (hidden 6144, int4 SwiGLU experts of 2048, top-8) with 16
    experts, so that the oracle can check every token of a 64-token step on both paths."""
    need_gpu()
    spec = wl.MoESpec("glm16", 16, 8, 6144, 2048, bqg.I4_ROW, bqg.ACT_SILU, 0, 0, False)
    L = wl.build_moe_layer(spec, 0, 0, device="cuda")
    lay = device_layer(L)
    tokens = 64
    x = wl.moe_tokens(spec, 0, tokens)
    idx, w, ridx, rw = _route(spec, 0, tokens)
    ref = om.moe_layer(oracle_layer(spec, 0, 0), x.numpy(), ridx, rw)
    for path in (bqg.MOE_PATH_TENSOR_CORES, bqg.MOE_PATH_CUDA_CORES):
        y = bqg.moe_forward(lay.with_path(path), x.cuda(), idx, w)
        torch.cuda.synchronize()
        assert_close(y, ref, what=f"glm geometry T=64 path {path}")
        tol = I8_TOL if path == bqg.MOE_PATH_TENSOR_CORES else 1e-4
        e = assert_close(y, ref, tol=tol, what=f"glm geometry T=64 path {path} (strict)")
        print(f"glm geometry T=64 path {path}: max rel err {e:.2e}")


def test_i8_zero_and_outlier_activations():
    """kind::i8 with degenerate rows: tokens whose x is all zero give exactly zero (scale 0, no
    division), and tokens with one large outlier (1e3 among N(0, 1) values, 16-bit fixed point per
    row then spends most of its range on the outlier) stay within the bounds of max|y|."""
    need_gpu()
    spec = wl.MoESpec("tc8_edge", 8, 2, 256, 128, bqg.I4_ROW, bqg.ACT_SILU, 0, 0, False)
    assert i8_variant(spec)
    L, lay = _layer(spec, bqg.MOE_PATH_TENSOR_CORES)
    tokens = 16
    x = wl.moe_tokens(spec, 3, tokens).clone()
    x[0] = 0.0
    x[5] = 0.0
    x[7, 17] = 1e3
    x[9, 200] = -1e3
    idx, w, ridx, rw = _route(spec, 3, tokens)
    y = bqg.moe_forward(lay, x.cuda(), idx, w)
    torch.cuda.synchronize()
    ref = om.moe_layer(oracle_layer(spec, 0, 0), x.numpy(), ridx, rw)
    yc = y.cpu().numpy()
    assert np.all(yc[0] == 0.0) and np.all(yc[5] == 0.0)
    assert_close(yc, ref, what="i8 zero / outlier rows")
    for t in (7, 9):  # each outlier token against its own scale
        assert_close(yc[t], ref[t], tol=I8_TOL, what=f"i8 outlier token {t}")
    normal = [t for t in range(tokens) if t not in (0, 5, 7, 9)]
    assert_close(yc[normal], ref[normal], tol=I8_TOL, what="i8 ordinary tokens")
    assert bqg.bqg_device_errors() == 0
