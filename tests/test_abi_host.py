"""The C-ABI library on the host (no GPU): it loads, exports every symbol the
header declares, rejects bad arguments before any launch, and its host-side
placement calls match the oracle and the pages' vectors."""
import json
import os
import re

import numpy as np
import pytest

import oracle
import moe_router_softmax_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^MOE_API[^(]*?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    syms = header_symbols()
    assert len(syms) >= 20
    for s in syms:
        assert hasattr(moe._lib, s), s
    assert sorted(moe.EXPORTS) == syms


def test_version_and_expert_bytes_match_oracle():
    assert "sm_100a" in moe.moe_version()
    for fmt in (0, 1, 2):
        for H, I in [(2816, 704), (256, 128), (1024, 192)]:
            assert moe.moe_expert_bytes(fmt, H, I) == oracle.expert_bytes(fmt, H, I)
            assert moe.moe_blob_offsets(fmt, H, I) == oracle.blob_offsets(fmt, H, I)
    assert moe.moe_expert_bytes(0, 100, 704) == 0


def _null_layer(**kw):
    import ctypes
    c = moe._CLayer()
    c.fmt, c.E, c.H, c.I = kw.get("fmt", 0), kw.get("E", 8), kw.get("H", 256), kw.get("I", 128)
    c.home = kw.get("home", 256)
    c.pool = kw.get("pool", None)
    c.slot_table = kw.get("slot_table", None)
    c.expert_bytes = kw.get("expert_bytes", moe.moe_expert_bytes(c.fmt, c.H, c.I))
    c.pool_slots = kw.get("pool_slots", 0)
    return ctypes.byref(c)


@pytest.mark.parametrize("args,frag", [
    (dict(E=0), "E=0"), (dict(E=2000), "E=2000"), (dict(H=100), "H=100"), (dict(I=96), "I=96"),
    (dict(fmt=7), "format"), (dict(expert_bytes=1000), "expert_bytes"), (dict(home=8), "aligned"),
    (dict(slot_table=256), "pool"), (dict(slot_table=256, pool=512), "pool_slots"),
    (dict(slot_table=256, pool=512, pool_slots=-3), "pool_slots"),
])
def test_ffn_rejects_bad_layers_before_launch(args, frag):
    st = moe._lib.moe_grouped_ffn(_null_layer(**args), 256, 4, 2, 256, 256, 256, 256, 256, 1 << 20, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    assert frag in moe.moe_last_error()


def test_calls_reject_bad_shapes_and_null_pointers():
    L = moe._lib
    assert L.moe_route_topk(256, 4, 8, 9, 256, 256, None) == moe.MOE_ERR_INVALID_ARG   # k > E
    assert "k=9" in moe.moe_last_error()
    assert L.moe_route_topk(256, 4, 8, 33, 256, 256, None) == moe.MOE_ERR_INVALID_ARG  # k > 32
    assert L.moe_route_topk(None, 4, 8, 2, 256, 256, None) == moe.MOE_ERR_INVALID_ARG  # NULL logits
    assert L.moe_route_topk(256, -1, 8, 2, 256, 256, None) == moe.MOE_ERR_INVALID_ARG  # T < 0
    assert L.moe_route_topk(256, 1 << 28, 128, 8, 256, 256, None) == moe.MOE_ERR_INVALID_ARG  # T*k overflow
    assert L.moe_route_topk(None, 0, 8, 2, None, None, None) == moe.MOE_OK  # T == 0: no-op
    assert L.moe_permute(None, 4, 2, 8, 256, 256, 256, 256, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_hits(256, 10, 0, 256, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(256, 256, 256, 4, 2, 100, 256, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(264, 256, 256, 4, 2, 128, 256, None) == moe.MOE_ERR_INVALID_ARG  # misaligned rows
    assert L.moe_quantize_int4(256, 4, 100, 256, 256, None) == moe.MOE_ERR_INVALID_ARG  # K % 64
    assert L.moe_pack_expert(1, 256, None, 256, None, 256, 128, 256, None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    st = L.moe_grouped_ffn(_null_layer(), 256, 4, 2, 256, 256, 256, 256, 256, 16, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "workspace" in moe.moe_last_error()
    # forcing an unknown path
    st = L.moe_grouped_ffn_path(_null_layer(), 256, 4, 2, 256, 256, 256, 256, 256, 1 << 30, 9, None)
    assert st == moe.MOE_ERR_INVALID_ARG


def test_workspace_queries():
    lay = _null_layer(E=128, H=2816, I=704)
    need = moe._lib.moe_grouped_ffn_workspace(lay, 64, 8)
    assert need >= 64 * 8 * 704 * 2
    fw = moe._lib.moe_layer_forward_workspace(lay, 64, 8)
    assert fw >= need + 64 * 8 * 2816 * 4


# ------------------------------------------------------------------ placement

def test_placement_matches_page_vectors(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "expert_pool_vectors.json")))
    c = g["target_gpu_picks_top_by_count"]
    assert moe.moe_refresh_target(np.array(c["counts"]), c["budget"]).tolist() == c["target"]
    c = g["paired_swap_limits_demotions"]
    so = np.full(c["E"], -1, np.int32)
    so[c["resident"]] = np.arange(len(c["resident"]))
    so2, pr, de = moe.moe_apply_placement(so, c["budget"], np.array(c["target"]))
    assert (len(pr), len(de)) == (c["promotions"], c["demotions"])
    assert sorted(np.nonzero(so2 >= 0)[0].tolist()) == c["resident_after"]
    c = g["paired_swap_keeps_extra_residents"]
    so = np.full(c["E"], -1, np.int32)
    so[c["resident"]] = np.arange(len(c["resident"]))
    so2, pr, de = moe.moe_apply_placement(so, c["budget"], np.array(c["target"]))
    assert (len(pr), len(de)) == (c["promotions"], c["demotions"])
    assert int((so2 >= 0).sum()) == c["resident_count_after"]
    c = g["jump_steps_refresh_schedule"]
    for step, prefill, want in c["cases"]:
        assert moe.moe_should_refresh(c["budget"] < c["E"], False, step, prefill, c["interval"]) == want
    assert not moe.moe_should_refresh(False, True, 0, True, 1)   # no offload: never
    c = g["vram_budget_formula"]
    b = moe.moe_budget_from_vram(c["free_bytes"], c["reserve_bytes"], c["expert_bytes"], c["layers"],
                                 c["max_per_layer"], c["E"])
    assert 0 < b <= 128
    assert moe.moe_budget_from_vram(1, 2, 0, 0, 300, 128) == 128


def test_placement_matches_oracle_on_random_refreshes():
    rng = np.random.default_rng(0)
    for E, n_slots in [(128, 18), (16, 5), (8, 8)]:
        so_a = np.full(E, -1, np.int32)
        so_a[:n_slots] = np.arange(n_slots)
        so_b = so_a.copy()
        for _ in range(100):
            hits = rng.integers(0, 6, size=E).astype(np.uint32) * (rng.random(E) < 0.6)
            ta = moe.moe_refresh_target(hits, n_slots)
            tb = oracle.refresh_target(hits, n_slots)
            assert np.array_equal(ta, tb)
            so_a, pa, da = moe.moe_apply_placement(so_a, n_slots, ta)
            so_b, pb, db = oracle.apply_placement(so_b, n_slots, tb)
            assert np.array_equal(so_a, so_b) and np.array_equal(pa, pb) and np.array_equal(da, db)


def test_placement_rejects_bad_input():
    with pytest.raises(moe.MoeError):
        moe.moe_apply_placement(np.full(8, -1, np.int32), 2, np.array([1, 2, 3]))  # target > slots
    with pytest.raises(moe.MoeError):
        moe.moe_apply_placement(np.full(8, -1, np.int32), 4, np.array([1, 1]))  # duplicate
    so = np.full(8, -1, np.int32)
    so[[0, 1]] = 0
    with pytest.raises(moe.MoeError):
        moe.moe_apply_placement(so, 4, np.array([2]))  # slot held twice


def test_router_topk_rejects_bad_arguments_before_launch():
    L = moe._lib
    ok = dict(x=256, wr=256, T=4, H=2816, E=128, k=8, lg=None, ids=256, w=256)

    def call(**kw):
        a = {**ok, **kw}
        return L.moe_router_topk(a["x"], a["wr"], a["T"], a["H"], a["E"], a["k"], a["lg"], a["ids"], a["w"], None)

    assert call(k=129) == moe.MOE_ERR_INVALID_ARG           # k > E
    assert call(E=0) == moe.MOE_ERR_INVALID_ARG
    assert call(H=2818) == moe.MOE_ERR_INVALID_ARG          # H % 4
    assert call(x=None) == moe.MOE_ERR_INVALID_ARG
    assert call(wr=264) == moe.MOE_ERR_INVALID_ARG          # router weights not 16-byte aligned
    assert call(x=260) == moe.MOE_ERR_INVALID_ARG           # x not 8-byte aligned
    assert call(T=-1) == moe.MOE_ERR_INVALID_ARG
    assert call(T=70000 * 16) == moe.MOE_ERR_INVALID_ARG    # more than 65535 token groups
    st = call(T=1, H=120000)                                 # one row of 120000 bf16 exceeds 200 KiB
    assert st == moe.MOE_ERR_UNSUPPORTED and "shared memory" in moe.moe_last_error()
    assert call(T=0) == moe.MOE_OK                           # nothing to do


def test_hits_window_matches_oracle():
    rng = np.random.default_rng(2)
    ring = rng.integers(0, 50, size=(8, 128), dtype=np.uint32)
    assert np.array_equal(moe.moe_hits_window(ring), oracle.hits_window(ring))
    with pytest.raises(moe.MoeError):
        moe.moe_hits_window(np.zeros((0, 128), np.uint32))


def test_device_refresh_rejects_bad_arguments_before_launch():
    L = moe._lib
    assert L.moe_refresh_device(256, 128, 19, 256, 18, 256, 256, None) == moe.MOE_ERR_INVALID_ARG  # budget > slots
    assert L.moe_refresh_device(256, 0, 0, 256, 0, 256, 256, None) == moe.MOE_ERR_INVALID_ARG      # E = 0
    assert L.moe_refresh_device(256, 2000, 1, 256, 4, 256, 256, None) == moe.MOE_ERR_INVALID_ARG   # E > 1024
    assert L.moe_refresh_device(None, 128, 1, 256, 4, 256, 256, None) == moe.MOE_ERR_INVALID_ARG   # NULL hits
    assert L.moe_promote_copies(256, 256, 100, 256, 256, 4, None) == moe.MOE_ERR_INVALID_ARG       # size % 16
    assert L.moe_promote_copies(264, 256, 256, 256, 256, 4, None) == moe.MOE_ERR_INVALID_ARG       # unaligned
    assert L.moe_promote_copies(256, 256, 256, 256, 256, 0, None) == moe.MOE_OK                    # nothing to do


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover
    given = None


if given is not None:
    @st.composite
    def _placement_case(draw):
        E = draw(st.integers(1, 64))
        n_slots = draw(st.integers(0, E))
        budget = draw(st.integers(0, n_slots))
        hits = np.array(draw(st.lists(st.integers(0, 5), min_size=E, max_size=E)), np.uint32)
        n_res = draw(st.integers(0, n_slots))
        experts = draw(st.permutations(list(range(E))))[:n_res]
        slots = draw(st.permutations(list(range(n_slots))))[:n_res] if n_slots else []
        slot_of = np.full(E, -1, np.int32)
        slot_of[list(experts)] = list(slots)
        return hits, slot_of, n_slots, budget

    @settings(max_examples=300, deadline=None)
    @given(_placement_case())
    def test_placement_property_matches_oracle(case):
        """Generated hit histograms and slot tables (empty and full pools, zero
        budget, all-zero hits, ties): the library's host placement equals the
        oracle's, and the residency invariants hold."""
        hits, slot_of, n_slots, budget = case
        target = moe.moe_refresh_target(hits, budget)
        assert np.array_equal(target, oracle.refresh_target(hits, budget))
        so, pr, de = moe.moe_apply_placement(slot_of, n_slots, target)
        oso, opr, ode = oracle.apply_placement(slot_of, n_slots, target)
        assert np.array_equal(so, oso) and np.array_equal(pr, opr) and np.array_equal(de, ode)
        held = so[so >= 0]
        assert len(set(held.tolist())) == len(held) and (held < n_slots).all()
        assert all(so[t] >= 0 for t in target)
        assert len(held) == int((slot_of >= 0).sum()) - len(de) + len(pr)
        assert set(pr.tolist()).isdisjoint(de.tolist())
