"""GPU: host-resident experts with a device slot cache (bqg_expert_cache_*), through the C ABI.

Every call is checked against the float64 oracle on the ORIGINAL expert ids, and the cache's
hit / miss / eviction / byte counts against an independent simulation of the replacement rule
(least frequently used among the slots the call does not need, least recently used among equal
counts, an empty slot first)."""
import numpy as np
import pytest
import torch

import block_quant_gemv_b200 as bqg
import synth
from oracle import moe as om
from synth import workloads as wl
from tests.moe_util import oracle_layer
from tests.util import assert_close, need_gpu

pytestmark = pytest.mark.gpu


class PolicySim:
    def __init__(self, n_experts, n_slots, expert_bytes):
        self.slot_of, self.expert_in = {}, [-1] * n_slots
        self.freq, self.last = [0] * n_slots, [-1] * n_slots
        self.calls, self.nb = 0, expert_bytes
        self.stats = dict(calls=0, hits=0, misses=0, evictions=0, bytes_copied=0)

    def step(self, idx, n_experts):
        order = []
        for e in np.asarray(idx).reshape(-1):
            e = int(e)
            if 0 <= e < n_experts and e not in order:
                order.append(e)
        needed = {self.slot_of[e] for e in order if e in self.slot_of}
        misses = []
        for e in order:
            if e in self.slot_of:
                continue
            free = [s for s in range(len(self.expert_in)) if s not in needed]
            empty = [s for s in free if self.expert_in[s] < 0]
            victim = empty[0] if empty else min(free, key=lambda s: (self.freq[s], self.last[s], s))
            if self.expert_in[victim] >= 0:
                del self.slot_of[self.expert_in[victim]]
                self.stats["evictions"] += 1
            self.expert_in[victim], self.slot_of[e], self.freq[victim] = e, victim, 0
            needed.add(victim)
            misses.append(e)
        for e in order:
            s = self.slot_of[e]
            self.freq[s] += 1
            self.last[s] = self.calls
        self.stats["hits"] += len(order) - len(misses)
        self.stats["misses"] += len(misses)
        self.stats["bytes_copied"] += len(misses) * self.nb
        self.stats["calls"] += 1
        self.calls += 1


def _cache(spec, n_slots, seed=0, with_shared=True):
    L = wl.build_moe_layer(spec, seed, 0, device="cpu")
    host = [t.pin_memory() for t in (L.gate, L.up, L.down)]
    shared = None
    if with_shared and L.shared is not None:
        shared = (spec.shared_fmt, spec.shared_inter) + tuple(t.cuda() for t in L.shared)
    c = bqg.ExpertCache(spec.n_experts, spec.top_k, spec.hidden, spec.inter, spec.expert_fmt, spec.act, *host,
                        L.gate_stride, L.up_stride, L.down_stride, n_slots, shared)
    nb = sum(spec.mat_bytes(m) for m in ("gate", "up", "down"))
    return c, PolicySim(spec.n_experts, n_slots, nb)


def _route(spec, seed, tokens, layer=0):
    lg = wl.moe_logits(spec, seed, layer, tokens)
    idx, w = bqg.moe_router_topk(lg.cuda(), spec.top_k)
    return idx.cpu().contiguous(), w


SMALL = wl.MoESpec("ec_q4_shared", 24, 4, 256, 128, bqg.Q4_0, bqg.ACT_GELU_TANH, 192, bqg.Q8_0, False)


def test_small_layer_sequence_matches_oracle_and_policy():
    need_gpu()
    spec = SMALL
    cache, sim = _cache(spec, n_slots=6)
    ref_layer = oracle_layer(spec, 0, 0)
    seeds = [1, 2, 1, 3, 4, 1, 5, 2, 2, 6]  # repeats give hits, new routings evict
    for call, seed in enumerate(seeds):
        tokens = 1
        x = wl.moe_tokens(spec, seed, tokens)
        idx_h, w = _route(spec, seed, tokens)
        y = cache.forward(x.cuda(), idx_h, w)
        torch.cuda.synchronize()
        sim.step(idx_h.numpy(), spec.n_experts)
        ref = om.moe_layer(ref_layer, x.numpy(), idx_h.numpy(), w.cpu().numpy())
        assert_close(y, ref, tol=1e-4, what=f"call {call}")
        assert cache.stats() == sim.stats, f"call {call}: {cache.stats()} != {sim.stats}"
    assert sim.stats["hits"] > 0 and sim.stats["evictions"] > 0
    assert bqg.bqg_device_errors() == 0


def test_two_tokens_and_invalid_id():
    """Two tokens (up to 8 distinct experts in 8 slots); an invalid id is skipped and flagged."""
    need_gpu()
    spec = SMALL
    cache, sim = _cache(spec, n_slots=8)
    ref_layer = oracle_layer(spec, 0, 0)
    bqg.bqg_device_errors()
    for call, seed in enumerate([7, 8, 7]):
        x = wl.moe_tokens(spec, seed, 2)
        idx_h, w = _route(spec, seed, 2)
        bad = call == 2
        if bad:
            idx_h[1, 2] = 999
        y = cache.forward(x.cuda(), idx_h, w)
        torch.cuda.synchronize()
        wr = w.cpu().numpy().copy()
        ir = idx_h.numpy().copy()
        if bad:
            wr[1, 2] = 0.0
            ir[1, 2] = 0
            assert bqg.bqg_device_errors() & bqg.DEVERR_EXPERT_ID
        sim.step(idx_h.numpy(), spec.n_experts)
        ref = om.moe_layer(ref_layer, x.numpy(), ir, wr)
        assert_close(y, ref, tol=1e-4, what=f"two tokens call {call}")
        assert cache.stats() == sim.stats


def test_more_experts_than_slots_is_refused():
    need_gpu()
    spec = SMALL
    cache, _ = _cache(spec, n_slots=4)
    x = wl.moe_tokens(spec, 9, 2)
    idx_h, w = _route(spec, 9, 2)
    assert len(set(idx_h.numpy().reshape(-1).tolist())) > 4
    with pytest.raises(bqg.BQGError) as e:
        cache.forward(x.cuda(), idx_h, w)
    assert e.value.status == -8
    assert cache.stats()["calls"] == 0


def test_glm_like_geometry_sixteen_slots():
    """GLM-like experts (hidden 6144, int4 SwiGLU of 2048, top-8) on the host, 16 device slots,
    one token per call: misses, full hits (the first routing again), and a mix."""
    need_gpu()
    spec = wl.MoESpec("ec_glm", 40, 8, 6144, 2048, bqg.I4_ROW, bqg.ACT_SILU, 0, 0, False)
    cache, sim = _cache(spec, n_slots=16)
    ref_layer = oracle_layer(spec, 0, 0)
    for call, seed in enumerate([11, 12, 11, 13]):
        x = wl.moe_tokens(spec, seed, 1)
        idx_h, w = _route(spec, seed, 1)
        y = cache.forward(x.cuda(), idx_h, w)
        torch.cuda.synchronize()
        sim.step(idx_h.numpy(), spec.n_experts)
        ref = om.moe_layer(ref_layer, x.numpy(), idx_h.numpy(), w.cpu().numpy())
        assert_close(y, ref, what=f"glm-like cache call {call}")
        assert_close(y, ref, tol=1e-4, what=f"glm-like cache call {call} (strict)")
        assert cache.stats() == sim.stats
    st = cache.stats()
    assert st["hits"] >= 8 and st["bytes_copied"] == st["misses"] * sim.nb


@pytest.mark.parametrize("spec,tol", [
    (SMALL, 1e-3),  # Q4_0 experts, Q8_0 shared expert: the kind::f16 tensor-core variant
    (wl.MoESpec("ec_i4", 16, 4, 256, 128, bqg.I4_ROW, bqg.ACT_SILU, 0, 0, False), 3e-4),  # kind::i8
], ids=["q4_shared_f16", "i4_i8"])
def test_many_tokens_take_the_tensor_cores(spec, tol):
    """Calls of 12 tokens take the tensor-core path in both passes (hits, then the misses after
    the copies, accumulated into the same output): every call against the oracle and the policy."""
    need_gpu()
    assert 12 >= bqg.MOE_TC_MIN_TOKENS
    cache, sim = _cache(spec, n_slots=spec.n_experts)
    ref_layer = oracle_layer(spec, 0, 0)
    for call, seed in enumerate([21, 21, 22, 23]):  # misses, all hits, then mixes
        x = wl.moe_tokens(spec, seed, 12)
        idx_h, w = _route(spec, seed, 12)
        y = cache.forward(x.cuda(), idx_h, w)
        torch.cuda.synchronize()
        sim.step(idx_h.numpy(), spec.n_experts)
        ref = om.moe_layer(ref_layer, x.numpy(), idx_h.numpy(), w.cpu().numpy())
        assert_close(y, ref, what=f"{spec.name} call {call}")
        assert_close(y, ref, tol=tol, what=f"{spec.name} call {call} (tensor cores)")
        assert cache.stats() == sim.stats
    st = cache.stats()
    assert st["hits"] > 0 and st["misses"] > 0
    assert bqg.bqg_device_errors() == 0
