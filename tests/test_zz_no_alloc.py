"""moe_grouped_ffn_noalloc: the grouped FFN for callers that cannot allocate
device memory (a runtime that hands the library only input and output buffers,
or a loop that must not call cudaMalloc).  Its scratch is a fixed device array
inside the library instead of a caller workspace, and it always runs the split-K
GEMV kernels.

Checked through the C ABI, on consecutive calls with different batches (so each
later call runs over the scratch contents the earlier one left behind), against
  - the CPU oracle, every row, at the FFN tolerance;
  - moe_grouped_ffn_path(..., MOE_FFN_GEMV) on the same inputs: bit-identical;
  - moe_grouped_ffn (the workspace entry point, AUTO path): within the tolerance.
The sequence includes a one-token call, which takes the GEMV kernels' one-token
instantiation.  This file is named to be collected last; it also passes on its
own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
import moe_router_softmax_b200 as moe
from gpu_support import FFN_TOL, device_weights_from_host, oracle_layer_for, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(L, x, k, counts, offsets, sr, rows):
    st = moe._lib.moe_grouped_ffn_noalloc(L.ref(), _ptr(x), x.shape[0], k, _ptr(counts), _ptr(offsets), _ptr(sr),
                                          _ptr(rows), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.MOE_OK, moe.moe_last_error()


@pytest.mark.parametrize("fmt", [moe.MOE_W_BF16, moe.MOE_W_INT8, moe.MOE_W_INT4])
def test_noalloc_matches_the_oracle_and_the_workspace_entry_point(fmt):
    E, H, I, k = 16, 1024, 320, 4
    w13, w2 = syn.expert_weights(E, H, I, seed=31)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    OL = oracle_layer_for(fmt, w13, w2)
    for call, T in enumerate((40, 1, 23)):
        xh = syn.activations(T, H, seed=40 + call)
        lgh = syn.router_logits(T, E, "normal", seed=50 + call)
        x = torch.from_numpy(xh.view(np.int16)).to(DEV).view(torch.bfloat16)
        ids, w = moe.moe_route_topk(torch.from_numpy(lgh).to(DEV), k)
        counts, offsets, sr, rp = moe.moe_permute(ids, E)
        gemv = moe.moe_grouped_ffn(L, x, k, counts, offsets, sr, path=moe.MOE_FFN_GEMV)
        auto = moe.moe_grouped_ffn(L, x, k, counts, offsets, sr)
        rows = torch.full((T * k, H), float("nan"), dtype=torch.float32, device=DEV)
        _noalloc(L, x, k, counts, offsets, sr, rows)
        torch.cuda.synchronize()
        n = int(offsets[-1])
        assert n == T * k
        got = rows[:n].cpu().numpy()
        assert np.array_equal(got.view(np.uint32), gemv[:n].cpu().numpy().view(np.uint32))
        assert rel_err(got, auto[:n].cpu().numpy()) <= FFN_TOL
        orows = oracle.ffn_routes(OL, xh, oracle.route_topk(lgh, k)[0])
        assert rel_err(got[rp.cpu().numpy()], orows) <= FFN_TOL


def test_noalloc_rejects_requests_beyond_its_scratch():
    E, H, I, k = 8, 256, 4096, 8
    home = torch.zeros(16, dtype=torch.uint8, device=DEV)
    L = moe.MoeLayer(moe.MOE_W_BF16, E, H, I, home, expert_bytes=moe.moe_expert_bytes(0, H, I))
    T = 1024  # 1024 * 8 routes * 4096 * 2 bytes = 64 MiB > 16 MiB
    x = torch.zeros((T, H), dtype=torch.bfloat16, device=DEV)
    z = torch.zeros(T * k, dtype=torch.int32, device=DEV)
    rows = torch.zeros(16, dtype=torch.float32, device=DEV)
    st = moe._lib.moe_grouped_ffn_noalloc(L.ref(), _ptr(x), T, k, _ptr(z), _ptr(z), _ptr(z), _ptr(rows), None)
    assert st == moe.MOE_ERR_INVALID_ARG
    assert "scratch" in moe.moe_last_error()
    # a bad layer is reported as what it is, not as a scratch overflow
    bad = moe.MoeLayer(moe.MOE_W_BF16, E, H, 4100, home, expert_bytes=moe.moe_expert_bytes(0, H, I))
    st = moe._lib.moe_grouped_ffn_noalloc(bad.ref(), _ptr(x), T, k, _ptr(z), _ptr(z), _ptr(z), _ptr(rows), None)
    assert st == moe.MOE_ERR_INVALID_ARG
    assert "I=4100" in moe.moe_last_error()
