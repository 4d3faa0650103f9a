"""C-ABI checks that need no GPU: the library loads, exports every function
the header declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from dynamic_block_sparse_fractal_b200 import api, workloads as W

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "sparse_attn.h")
FAKE = ctypes.c_void_p(0x10000000)  # never dereferenced: validation fails first


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(sparse_attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = api.lib()
    names = declared_functions()
    assert set(names) == set(api.SYMBOLS)
    for n in names:
        assert hasattr(L, n), n


def test_workspace_size_and_validation():
    d = api.desc_for(W.HUNYUAN)
    assert api.workspace_size(d) > 0
    bad = [
        dict(d=96), dict(P=4, N=16), dict(Hh=44), dict(thr=1.0), dict(thr=-0.1),
        dict(thr=float("nan")), dict(sta=(2, 3, 3)), dict(sta=(3, 0, 3)), dict(B=0),
    ]
    expect = [api.SA_ERR_UNSUPPORTED, api.SA_ERR_UNSUPPORTED, api.SA_ERR_UNSUPPORTED,
              api.SA_ERR_INVALID_ARG, api.SA_ERR_INVALID_ARG, api.SA_ERR_INVALID_ARG,
              api.SA_ERR_INVALID_ARG, api.SA_ERR_INVALID_ARG, api.SA_ERR_INVALID_ARG]
    base = dict(B=1, H=2, T=4, Hh=16, Ww=16, d=128, thr=0.1, sta=(0, 0, 0), N=64, P=8)
    for b, e in zip(bad, expect):
        kw = dict(base, **b)
        n = ctypes.c_size_t()
        st = api.lib().sparse_attn_workspace_size(ctypes.byref(api.make_desc(**kw)),
                                                  ctypes.byref(n))
        assert st == e, (b, st)
    # too many blocks per head for the mask kernel's shared memory
    big = api.make_desc(1, 1, 100, 64, 64, 128, 0.1)
    n = ctypes.c_size_t()
    assert api.lib().sparse_attn_workspace_size(ctypes.byref(big), ctypes.byref(n)) == \
        api.SA_ERR_UNSUPPORTED


def test_entry_points_reject_before_launch():
    L = api.lib()
    d = api.desc_for(W.TINY)
    need = api.workspace_size(d)
    st = L.sparse_attn_plan(ctypes.byref(d), FAKE, FAKE, FAKE, need - 1, None)
    assert st == api.SA_ERR_WORKSPACE
    st = L.sparse_attn_plan(ctypes.byref(d), None, FAKE, FAKE, need, None)
    assert st == api.SA_ERR_INVALID_ARG
    st = L.sparse_attn_plan(ctypes.byref(d), ctypes.c_void_p(0x10000008), FAKE, FAKE, need, None)
    assert st == api.SA_ERR_INVALID_ARG  # q not 16-byte aligned
    st = L.sparse_attn_fwd(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, need - 256, FAKE, None)
    assert st == api.SA_ERR_WORKSPACE
    st = L.sparse_attn_fwd(ctypes.byref(d), FAKE, FAKE, FAKE, ctypes.c_void_p(0x10000010),
                           need, FAKE, None)
    assert st == api.SA_ERR_INVALID_ARG  # workspace not 256-byte aligned
    st = L.sparse_attn_permute(ctypes.byref(d), FAKE, FAKE, 0, None)
    assert st == api.SA_ERR_INVALID_ARG  # x and y overlap
    st = L.sparse_attn_permute(ctypes.byref(d), FAKE, FAKE, 2, None)
    assert st == api.SA_ERR_INVALID_ARG
    v = api.SaMaskViews()
    assert L.sparse_attn_get_mask(ctypes.byref(d), FAKE, need - 1, ctypes.byref(v)) == \
        api.SA_ERR_WORKSPACE
    assert L.sparse_attn_check(ctypes.byref(d), FAKE, 0, None) == api.SA_ERR_WORKSPACE
    assert L.sparse_attn_get_mask(None, FAKE, need, ctypes.byref(v)) == api.SA_ERR_INVALID_ARG
    assert api.status_string(api.SA_ERR_DEVICE_TIMEOUT).startswith("a kernel")
    sz = ctypes.c_size_t
    scr = api.heatmap_scratch_size(d)
    assert scr == 2 * 256 * 4 * 4  # two CTAs of 256 rows x 4 blocks (fp32)

    def heat_call(ws_bytes, heat, scratch, scratch_bytes):
        return L.sparse_attn_block_heatmap(ctypes.byref(d), FAKE, FAKE, FAKE, sz(ws_bytes), heat,
                                           scratch, sz(scratch_bytes), None)
    assert heat_call(need, None, FAKE, scr) == api.SA_ERR_INVALID_ARG  # no heat buffer
    assert heat_call(need, ctypes.c_void_p(0x10000002), FAKE, scr) == \
        api.SA_ERR_INVALID_ARG  # heat not 4-byte aligned
    assert heat_call(need, FAKE, None, scr) == api.SA_ERR_INVALID_ARG  # no scratch
    assert heat_call(need - 1, FAKE, FAKE, scr) == api.SA_ERR_WORKSPACE
    assert heat_call(need, FAKE, FAKE, scr - 1) == api.SA_ERR_WORKSPACE
    h = ctypes.c_void_p()
    assert L.sparse_attn_graph_create(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, sz(need), FAKE, 1,
                                      None) == api.SA_ERR_INVALID_ARG  # nowhere to put it
    assert L.sparse_attn_graph_create(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, sz(need), FAKE, 2,
                                      ctypes.byref(h)) == api.SA_ERR_INVALID_ARG
    bad = api.make_desc(1, 1, 4, 8, 8, 96, 0.1)  # d = 96: rejected before any capture
    assert L.sparse_attn_graph_create(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, sz(need), FAKE, 1,
                                      ctypes.byref(h)) == api.SA_ERR_UNSUPPORTED
    assert L.sparse_attn_graph_launch(None, None) == api.SA_ERR_INVALID_ARG
    assert L.sparse_attn_graph_destroy(None) == api.SA_OK


@pytest.mark.parametrize("T,Hh,Ww", [(4, 8, 8), (33, 48, 80), (21, 32, 56), (3, 8, 24), (1, 16, 8)])
def test_tile_pairing_covers_every_block_once(T, Hh, Ww):
    d = api.make_desc(1, 1, T, Hh, Ww, 128, 0.1)
    nh, nw = Hh // 8, Ww // 8
    nb = T * nh * nw
    seen = []
    ntile = (T // 2) * nh * nw + (T % 2) * nh * ((nw + 1) // 2)
    for i in range(ntile):
        qa, qb = api.tile_blocks(d, i)
        seen.append(qa)
        if qb >= 0:
            seen.append(qb)
            ta, tb = qa // (nh * nw), qb // (nh * nw)
            # same patch in consecutive frames, or neighbours in the last odd frame
            assert (tb == ta + 1 and qb - qa == nh * nw) or (ta == tb == T - 1 and qb == qa + 1)
    assert sorted(seen) == list(range(nb))
    with pytest.raises(api.SparseAttnError):
        api.tile_blocks(d, ntile)


def test_tile_shape_validation():
    base = dict(B=1, H=2, T=8, Hh=32, Ww=32, d=128, thr=0.1)
    cases = [
        ((2, 4, 8), api.SA_OK),
        ((4, 4, 4), api.SA_OK),
        ((1, 8, 8), api.SA_OK),          # the square patch, given as a tile
        ((2, 4, 4), api.SA_ERR_UNSUPPORTED),   # 32 tokens, not N = 64
        ((3, 4, 8), api.SA_ERR_UNSUPPORTED),   # 96 tokens
        ((16, 2, 2), api.SA_ERR_UNSUPPORTED),  # T = 8 not divisible by 16
        ((1, 1, 64), api.SA_ERR_UNSUPPORTED),  # Ww = 32 not divisible by 64
        ((0, 8, 8), api.SA_ERR_INVALID_ARG),
        ((-2, -4, 8), api.SA_ERR_INVALID_ARG),
    ]
    for tile, expect in cases:
        n = ctypes.c_size_t()
        st = api.lib().sparse_attn_workspace_size(ctypes.byref(api.make_desc(**base, tile=tile)),
                                                  ctypes.byref(n))
        assert st == expect, (tile, st)
    # with a tile the patch edge is not used
    d = api.make_desc(**base, tile=(2, 4, 8), P=0)
    assert api.workspace_size(d) > 0


@pytest.mark.parametrize("T,Hh,Ww,tile", [(8, 32, 32, (2, 4, 8)), (8, 32, 32, (4, 4, 4)),
                                         (33, 48, 80, (1, 4, 16)), (6, 16, 32, (2, 2, 16))])
def test_tile_pairing_covers_every_block_once_3d(T, Hh, Ww, tile):
    pt, ph, pw = tile
    d = api.make_desc(1, 1, T, Hh, Ww, 128, 0.1, tile=tile)
    nt, nh, nw = T // pt, Hh // ph, Ww // pw
    nb = nt * nh * nw
    seen = []
    ntile = (nt // 2) * nh * nw + (nt % 2) * nh * ((nw + 1) // 2)
    for i in range(ntile):
        qa, qb = api.tile_blocks(d, i)
        seen.append(qa)
        if qb >= 0:
            seen.append(qb)
            ta, tb = qa // (nh * nw), qb // (nh * nw)
            assert (tb == ta + 1 and qb - qa == nh * nw) or (ta == tb == nt - 1 and qb == qa + 1)
    assert sorted(seen) == list(range(nb))


def test_per_head_shapes_split_into_runs():
    w = W.W8K  # 12 heads on an 8 x 32 x 32 grid
    d = api.desc_for(w)
    tiles = [(1, 8, 8)] * 4 + [(2, 4, 8)] * 4 + [(4, 4, 4)] * 2 + [(2, 4, 8)] * 2
    runs = api.heads_runs(d, tiles)
    assert [(r[0].H, r[1]) for r in runs] == [(4, 0), (4, 4), (2, 8), (2, 10)]
    assert [(r[0].pt, r[0].ph, r[0].pw) for r in runs] == [(1, 8, 8), (2, 4, 8), (4, 4, 4),
                                                           (2, 4, 8)]
    total = api.workspace_size_heads(d, tiles)
    off = 0
    for sub, _, ws_off, ws_bytes in runs:
        assert ws_off == off and ws_off % 256 == 0
        assert ws_bytes == api.workspace_size(sub)
        off = (ws_off + ws_bytes + 255) // 256 * 256
    assert total == off
    # one shape for every head: a single run with the whole problem
    one = api.heads_runs(d, [(2, 4, 8)] * 12)
    assert len(one) == 1 and one[0][0].H == 12
    # a bad shape in one head is that run's error; no tiles is an argument error
    with pytest.raises(api.SparseAttnError):
        api.workspace_size_heads(d, [(1, 8, 8)] * 11 + [(3, 4, 8)])
    n = ctypes.c_size_t()
    assert api.lib().sparse_attn_workspace_size_heads(ctypes.byref(d), None, ctypes.byref(n)) == \
        api.SA_ERR_INVALID_ARG
    # one scratch buffer serves the runs of the gradient and map calls in turn:
    # the largest run's size
    arr = (ctypes.c_int * 36)(*[x for t in tiles for x in t])
    for name, single in (("sparse_attn_bwd_scratch_size_heads", api.bwd_scratch_size),
                         ("sparse_attn_block_heatmap_scratch_size_heads",
                          api.heatmap_scratch_size)):
        assert getattr(api.lib(), name)(ctypes.byref(d), arr, ctypes.byref(n)) == api.SA_OK
        assert n.value == max(single(sub) for sub, *_ in runs)


def test_plan_profile_names_and_rejection():
    L = api.lib()
    names = []
    i = 0
    while L.sparse_attn_plan_stage_name(i) is not None:
        names.append(L.sparse_attn_plan_stage_name(i).decode())
        i += 1
    assert names and len(set(names)) == len(names)
    assert L.sparse_attn_plan_stage_name(-1) is None
    d = api.desc_for(W.TINY)
    us = (ctypes.c_float * 16)()
    n = ctypes.c_int(0)
    need = api.workspace_size(d)
    # too short an output array, zero repetitions: rejected before any launch
    assert L.sparse_attn_plan_profile(ctypes.byref(d), FAKE, FAKE, FAKE, need, 1, us,
                                      len(names) - 1, ctypes.byref(n), None) == \
        api.SA_ERR_INVALID_ARG
    assert L.sparse_attn_plan_profile(ctypes.byref(d), FAKE, FAKE, FAKE, need, 0, us, 16,
                                      ctypes.byref(n), None) == api.SA_ERR_INVALID_ARG


def test_radius_plan_rejects_bad_parameters_before_launch():
    L = api.lib()
    d = api.desc_for(W.TINY)
    need = api.workspace_size(d)
    for tau, gamma, vmin in ((0.0, 0.1, 1), (-1.0, 0.1, 1), (float("nan"), 0.1, 1),
                             (1.0, -0.5, 1), (1.0, float("inf"), 1), (1.0, 0.1, 0),
                             (1.0, 0.1, 65)):
        r = api.SaRadius(tau, gamma, vmin)
        assert L.sparse_attn_plan_radius(ctypes.byref(d), ctypes.byref(r), FAKE, FAKE, need,
                                         None) == api.SA_ERR_INVALID_ARG, (tau, gamma, vmin)
    r = api.SaRadius(1.0, 0.1, 1)
    assert L.sparse_attn_plan_radius(ctypes.byref(d), ctypes.byref(r), None, FAKE, need,
                                     None) == api.SA_ERR_INVALID_ARG
    assert L.sparse_attn_plan_radius(ctypes.byref(d), ctypes.byref(r), FAKE, FAKE, need - 1,
                                     None) == api.SA_ERR_WORKSPACE
    assert L.sparse_attn_token_entropy(ctypes.byref(d), FAKE, FAKE, FAKE, need, None,
                                       None) == api.SA_ERR_INVALID_ARG
