"""The router projection fused with top-k (moe_router_topk) vs the CPU oracle.

The logits are fp32 sums on the GPU and fp64 sums in the oracle, so they agree
within the rounding bound of the GPU's summation: each logit is a chain of at
most H/32 fused multiply-adds followed by a 5-level butterfly, so
|gpu - exact| <= gamma_n * sum_h |x_h w_h| with n = H/32 + 5 and
gamma_n = n u / (1 - n u), u = 2^-24.  The routing decision is taken on the
GPU's own fp32 logits: ids and weights must equal the oracle's top-k of those
logits bit for bit; against the oracle's exact logits, ids must match wherever
the top k+1 logits are separated by more than twice the bound.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
import moe_router_softmax_b200 as moe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits_equal(a, b):
    return np.array_equal(np.ascontiguousarray(a).view(np.uint32), np.ascontiguousarray(b).view(np.uint32))


def _bound(x_bits, wr):
    H = x_bits.shape[1]
    n = H / 32 + 5
    u = 2.0 ** -24
    xf = syn.bf16_to_f32(x_bits).astype(np.float64)
    return (n * u / (1 - n * u)) * (np.abs(xf) @ np.abs(wr.astype(np.float64)).T)


def _run(T, H, E, k, seed, wr=None, x=None):
    x = syn.activations(T, H, seed=seed) if x is None else x
    wr = syn.router_weights(E, H, seed=seed) if wr is None else wr
    xd = torch.from_numpy(x.view(np.int16)).to(DEV)
    wd = torch.from_numpy(wr).to(DEV)
    ids, w, lg = moe.moe_router_topk(xd, wd, k, logits=True)
    torch.cuda.synchronize()
    return x, wr, ids.cpu().numpy(), w.cpu().numpy(), lg.cpu().numpy()


def _check(x, wr, ids, w, lg, k):
    exact = oracle.router_logits(x, wr)
    bound = _bound(x, wr)
    assert np.all(np.abs(lg.astype(np.float64) - exact) <= bound), float(np.max(np.abs(lg - exact) / bound))
    # the decision on the GPU's logits, in fp32, exactly as the oracle takes it
    oi, ow = oracle.route_topk(lg, k)
    assert np.array_equal(ids, oi)
    assert _bits_equal(w, ow)
    # against the exact logits where the order is not decided by rounding
    T, E = exact.shape
    checked = 0
    for t in range(T):
        top = np.sort(exact[t])[::-1][: min(k + 1, E)]
        if np.all(np.diff(-top) > 2 * bound[t].max()):
            want = np.argsort(-exact[t], kind="stable")[:k]
            assert np.array_equal(ids[t], want)
            checked += 1
    return checked


@pytest.mark.parametrize("T,H,E,k", [
    (1, 2816, 128, 8), (2, 2816, 128, 8), (3, 2816, 128, 8), (5, 2816, 128, 8), (8, 2816, 128, 8),
    (13, 2816, 128, 8), (64, 2816, 128, 8), (37, 260, 13, 3), (9, 64, 8, 2), (20, 512, 200, 32),
    (17, 1024, 1024, 8), (4, 128, 8, 8),
])
def test_router_topk_matches_oracle(T, H, E, k):
    x, wr, ids, w, lg = _run(T, H, E, k, seed=T * 7 + E)
    checked = _check(x, wr, ids, w, lg, k)
    assert checked >= T // 2


def test_router_topk_prefill_batch_full_size():
    """The 1024-token prefill batch at the Gemma shape: every token."""
    x, wr, ids, w, lg = _run(1024, 2816, 128, 8, seed=5)
    assert _check(x, wr, ids, w, lg, 8) >= 900


def test_router_topk_without_logits_output_is_the_same():
    T, H, E, k = 29, 2816, 128, 8
    x = syn.activations(T, H, seed=3)
    wr = syn.router_weights(E, H, seed=3)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV)
    wd = torch.from_numpy(wr).to(DEV)
    i1, w1, _ = moe.moe_router_topk(xd, wd, k, logits=True)
    i2, w2 = moe.moe_router_topk(xd, wd, k)
    assert torch.equal(i1, i2) and torch.equal(w1.view(torch.int32), w2.view(torch.int32))


def test_router_topk_equal_rows_tie_to_the_lower_id():
    """Identical router rows give bit-identical logits (same summation order),
    and equal logits rank the lower expert id first."""
    T, H, E, k = 16, 2816, 128, 8
    wr = syn.router_weights(E, H, seed=9)
    x = syn.activations(T, H, seed=9)
    exact = oracle.router_logits(x, wr)
    # copy the winning row of each token into a higher id: both must be chosen, lower id first
    for t in range(4):
        e = int(np.argmax(exact[t]))
        wr[(e + 50 + t) % E] = wr[e]
    x, wr, ids, w, lg = _run(T, H, E, k, seed=9, wr=wr, x=x)
    _check(x, wr, ids, w, lg, k)
    for t in range(4):
        e = int(np.argmax(exact[t]))
        dup = (e + 50 + t) % E
        pos = list(ids[t])
        if dup in pos and e in pos:
            assert pos.index(min(e, dup)) < pos.index(max(e, dup))
            assert lg[t, e] == lg[t, dup]


def test_router_topk_k_equals_e_is_a_softmax_and_t0_is_a_noop():
    T, H, E = 6, 320, 16
    x, wr, ids, w, lg = _run(T, H, E, E, seed=1)
    _check(x, wr, ids, w, lg, E)
    assert np.all(np.abs(w.sum(axis=1) - 1.0) < 1e-5)
    xd = torch.empty((0, H), dtype=torch.bfloat16, device=DEV)
    ids0, w0 = moe.moe_router_topk(xd, torch.from_numpy(wr).to(DEV), 4)
    assert ids0.shape == (0, 4)


def test_no_kernel_recorded_a_device_error():
    """The tensor-core kernels record the first failed index check or timed-out
    wait in a device word; after every GPU test so far it must still be clear."""
    code, info = moe.moe_take_device_errors()
    assert code == 0, (hex(code), info)
