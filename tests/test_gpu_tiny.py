"""GPU parity of the whole layer and of each stage on the tiny workload
(T=64, H=512, I=256, 32 routed + 1 shared, top-6), through the C ABI."""
import numpy as np
import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import synth
from oracle import moe as om
from oracle import mx as omx

import parity

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["tiny"]


@pytest.fixture(scope="module")
def tiny(cuda_device):
    from routed_expert_ffn_sqrtsoftplus_b200 import build
    build.build()
    lay = synth.make_layer(WL.with_tokens(700), device="cpu")
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=700)
    yield lay, layer
    layer.close()


def _run(layer, x):
    y, idx, w = layer.forward_with_routing(x)
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK
    return y, idx, w


@pytest.mark.parametrize("T", [64, 1, 3, 17, 63, 33, 129])
def test_tiny_layer_parity(tiny, T):
    lay, layer = tiny
    x = lay["x"][:T].contiguous()
    y, idx, w = _run(layer, x)
    sub = dict(lay, x=x)
    rep = parity.compare_layer(sub, np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(),
                               WL.k, WL.route_scale, WL.swiglu_limit)
    assert rep["rel"] < parity.TOL_Y


@pytest.mark.parametrize("T", [300, 700])
def test_tiny_layer_parity_large_T(tiny, T):
    """T >= 256 takes the tensor-core router and the 128/256-token GEMM tiles."""
    lay, layer = tiny
    x = lay["x"][:T].contiguous()
    y, idx, w = _run(layer, x)
    rep = parity.compare_layer(dict(lay, x=x), np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(),
                               w.cpu().numpy(), WL.k, WL.route_scale, WL.swiglu_limit)
    assert rep["rel"] < parity.TOL_Y


@pytest.mark.parametrize("T", [300, 700])
def test_tiny_layer_parity_hot_experts(tiny, cuda_device, T):
    """A router bias of +6 on experts 0 and 1 sends every token to both: groups of
    T rows, more than the narrower many-token tile holds, so the permutation keeps
    the widest tiles and splits each hot expert over several of them."""
    lay, _ = tiny
    bias = torch.zeros(WL.E, dtype=torch.float32, device=cuda_device)
    bias[:2] = 6.0
    hot = dict(lay, bias=bias)
    layer = moe.MoELayer.from_layer(hot, top_k=WL.k, max_tokens=700)
    try:
        x = lay["x"][:T].contiguous()
        y, idx, w = _run(layer, x)
        cnt = np.bincount(idx.cpu().numpy().ravel(), minlength=WL.E)
        assert cnt[0] == T and cnt[1] == T
        rep = parity.compare_layer(dict(hot, x=x), np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(),
                                   w.cpu().numpy(), WL.k, WL.route_scale, WL.swiglu_limit)
        assert rep["rel"] < parity.TOL_Y
    finally:
        layer.close()


@pytest.mark.parametrize("T", [64, 300])
def test_permutation_is_exact(tiny, T):
    lay, layer = tiny
    x = lay["x"][:T].contiguous()
    _, idx, _ = _run(layer, x)
    G = WL.E + WL.n_shared
    cnt = layer.inspect(moe.BUF_COUNTS, torch.empty(G, dtype=torch.int32, device=x.device)).cpu().numpy()
    off = layer.inspect(moe.BUF_OFFSETS, torch.empty(G + 1, dtype=torch.int32, device=x.device)).cpu().numpy()
    perm = layer.inspect(moe.BUF_PERM, torch.empty(T * WL.k, dtype=torch.int32, device=x.device)).cpu().numpy()
    inv = layer.inspect(moe.BUF_INV, torch.empty(T * WL.k, dtype=torch.int32, device=x.device)).cpu().numpy()
    torch.cuda.synchronize()
    c_ref, o_ref, p_ref, i_ref = om.permutation_reference(idx.cpu().numpy(), WL.E)
    assert np.array_equal(cnt[:WL.E], c_ref) and np.all(cnt[WL.E:] == T)
    assert np.array_equal(off[:WL.E + 1], o_ref)
    assert np.array_equal(off[WL.E + 1:], T * WL.k + T * np.arange(1, WL.n_shared + 1))
    assert np.array_equal(perm, p_ref)
    assert np.array_equal(inv, i_ref)


def test_swiglu_rows_match_oracle(tiny):
    """The gate/up GEMM's epilogue output h, row by row, against the oracle's h."""
    lay, layer = tiny
    T = 64
    x = lay["x"][:T].contiguous()
    _, idx, _ = _run(layer, x)
    R = T * WL.k + WL.n_shared * T
    h = layer.inspect(moe.BUF_H, torch.empty((R, WL.I), dtype=torch.bfloat16, device=x.device))
    perm = layer.inspect(moe.BUF_PERM, torch.empty(T * WL.k, dtype=torch.int32, device=x.device))
    torch.cuda.synchronize()
    h = parity.f64(h)
    perm = perm.cpu().numpy()
    idx = idx.cpu().numpy()
    xf = parity.f64(x)
    ex = parity.LayerExperts(lay)
    # h is stored in BF16: each element carries at most 2^-9 relative rounding,
    # plus fp32 accumulation error far below it
    def check(h_gpu, h_or):
        bound = 2.0 ** -8 * np.abs(h_or) + 1e-3 * np.sqrt(np.mean(h_or ** 2))
        assert np.all(np.abs(h_gpu - h_or) <= bound), np.max(np.abs(h_gpu - h_or) / bound)
    for e in range(WL.E):
        rows = np.nonzero(idx.reshape(-1)[perm] == e)[0]
        if len(rows) == 0:
            continue
        toks = perm[rows] // WL.k
        _, h_or = om.expert_forward(xf[toks], *ex.routed(e), WL.swiglu_limit)
        check(h[rows], h_or)
    _, h_sh = om.expert_forward(xf, *ex.shared(0), WL.swiglu_limit)
    check(h[T * WL.k:], h_sh)


def test_deterministic(tiny):
    lay, layer = tiny
    x = lay["x"][:300].contiguous()
    y1, i1, w1 = _run(layer, x)
    y2, i2, w2 = _run(layer, x)
    assert torch.equal(y1, y2) and torch.equal(i1, i2) and torch.equal(w1, w2)


def test_token_order_invariance(tiny):
    lay, layer = tiny
    T = 64
    x = lay["x"][:T].contiguous()
    p = torch.randperm(T, generator=torch.Generator().manual_seed(0)).to(x.device)
    y, idx, w = _run(layer, x)
    yp, idxp, wp = _run(layer, x[p].contiguous())
    assert torch.equal(idxp, idx[p]) and torch.equal(wp, w[p])
    assert torch.allclose(yp.float(), y[p].float(), rtol=0, atol=0)


def test_zero_tokens(tiny):
    lay, layer = tiny
    x = lay["x"][:0]
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert y.shape == (0, WL.H)
    assert layer.status() == moe.MOE_OK


def test_rejects_too_many_tokens(tiny):
    lay, layer = tiny
    x = torch.zeros((701, WL.H), dtype=torch.bfloat16, device=lay["x"].device)
    with pytest.raises(moe.MoEError) as ei:
        layer.forward(x)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG


def test_forward_rejects_pointers_outside_the_device(tiny):
    """moe_forward, called through the C ABI with x or y in pinned host memory,
    returns MOE_ERR_INVALID_ARG before launching anything. (Pinned memory is
    readable from the device, so even an accepted pointer could not fault.)"""
    lay, layer = tiny
    T = 4
    xd = lay["x"][:T].contiguous()
    yd = torch.empty_like(xd)
    xh = xd.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    L = moe.lib()
    s = torch.cuda.current_stream().cuda_stream
    for xp, yp in ((xh, yd), (xd, yh)):
        st = L.moe_forward(layer._h, xp.data_ptr(), T, yp.data_ptr(), None, None, s)
        assert st == moe.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK
    # the same call with device buffers still runs
    assert L.moe_forward(layer._h, xd.data_ptr(), T, yd.data_ptr(), None, None, s) == moe.MOE_OK
    torch.cuda.synchronize()


def test_forward_host_matches_device(tiny):
    lay, layer = tiny
    T = 17
    x = lay["x"][:T].contiguous()
    y, idx, w = _run(layer, x)
    xh = x.cpu().pin_memory()
    yh = torch.empty((T, WL.H), dtype=torch.bfloat16).pin_memory()
    ih = torch.empty((T, WL.k), dtype=torch.int32).pin_memory()
    layer.forward_host(xh, yh, ih)
    torch.cuda.synchronize()
    assert torch.equal(yh, y.cpu()) and torch.equal(ih, idx.cpu())


def test_forward_host_async_pipeline_matches_device(tiny):
    """Calls of the pipelined host path with different batches back to back (copies on
    the library's streams overlapping the neighbouring layers): every y equals the
    device forward of its own x, bit for bit, also when the two staging slots are
    reused several times and T changes between calls."""
    lay, layer = tiny
    Ts = [17, 64, 5, 64, 33, 1, 64]
    xs, ys, ref = [], [], []
    for i, T in enumerate(Ts):
        x = lay["x"][:T].contiguous() if i % 2 == 0 else torch.flip(lay["x"][:T], dims=[0]).contiguous()
        y, _, _ = _run(layer, x)
        ref.append(y.cpu())
        xs.append(x.cpu().pin_memory())
        ys.append(torch.full((T, WL.H), float("nan"), dtype=torch.bfloat16).pin_memory())
    torch.cuda.synchronize()
    for xh, yh in zip(xs, ys):
        layer.forward_host_async(xh, yh)
    layer.forward_host_wait()
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK
    for i, (yh, r) in enumerate(zip(ys, ref)):
        assert torch.equal(yh, r), f"call {i} (T={Ts[i]})"


def test_bounded_wait_reports_timeout(tiny):
    _, layer = tiny
    assert layer.status() == moe.MOE_OK
    layer.selftest_wait_timeout(2_000_000)   # 2 ms wait that nothing completes
    assert layer.status() == moe.MOE_ERR_TIMEOUT
    assert layer.status() == moe.MOE_OK      # reading clears it


def test_router_tie_break_lower_index(cuda_device):
    """Identical router rows tie exactly: the lower expert index must win."""
    H, I, E, S, k = 128, 128, 8, 1, 2
    g = torch.Generator().manual_seed(4)
    x = torch.randn((5, H), generator=g).to(torch.bfloat16)
    wg = torch.randn((E, H), generator=g).to(torch.bfloat16) * 0.0
    wg[3] = wg[6] = wg[1] = 0.5        # three identical best rows
    w1 = (torch.randn((E, I, H), generator=g) / 11).to(torch.bfloat16)
    w3 = (torch.randn((E, I, H), generator=g) / 11).to(torch.bfloat16)
    w2 = (torch.randn((E, H, I), generator=g) / 11).to(torch.bfloat16)
    sh = [(torch.randn(s, generator=g) / 11).to(torch.bfloat16) for s in ((S, I, H), (S, I, H), (S, H, I))]
    d = {n: t.to(cuda_device) for n, t in dict(x=x, wg=wg, w1=w1, w3=w3, w2=w2, sh_w1=sh[0], sh_w3=sh[1],
                                                sh_w2=sh[2]).items()}
    layer = moe.MoELayer.from_layer(d, top_k=k, max_tokens=8)
    y, idx, w = layer.forward_with_routing(d["x"])
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    # z = x . row for rows 1, 3, 6 and 0 for the rest: z > 0 picks 1 then 3 (three-way
    # tie, lowest indices win); z < 0 leaves the zero-logit experts 0, 2, 4, 5, 7 tied on top
    for t in range(5):
        z = float((x[t].double() * 0.5).sum())
        assert list(idx[t]) == ([1, 3] if z > 0 else [0, 2] if z < 0 else [0, 1])
    rep = parity.compare_layer(d, np.arange(5), y.float().cpu().numpy(), idx, w.cpu().numpy(), k, 1.5, 10.0)
    layer.close()


def test_quantize_mxfp4_bitexact(cuda_device):
    g = torch.Generator().manual_seed(11)
    w = (torch.randn((48, 512), generator=g) * 0.03).to(torch.bfloat16)
    w[3, :32] = 0                                  # all-zero block
    w[4, 32:64] = 7.0                              # saturating block
    w[5, 64:96] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25] * 4)   # E2M1 midpoints at scale 1
    w[5, 64] = 4.0                                 # amax 4 -> scale code 127
    w[6, :32] = torch.finfo(torch.bfloat16).tiny   # smallest normal BF16
    q, s = moe.quantize_mxfp4(w.to(cuda_device))
    torch.cuda.synchronize()
    q_ref, s_ref = omx.quantize_mxfp4_packed(parity.f64(w))
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("T", [7, 37, 200])
def test_dspark_shaped_layer(cuda_device, T):
    """The DSpark drafter's routing shape (128 routed experts, 3 active; config.json
    dspark_n_routed_experts / dspark_n_activated_experts) at small widths."""
    wl = synth.Workload("dspark_small", T=T, H=512, I=256, E=128, k=3, seed=1005)
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in synth.make_layer(wl).items()}
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=T)
    try:
        y, idx, w = _run(layer, lay["x"])
        rep = parity.compare_layer(lay, np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(),
                                   wl.k, wl.route_scale, wl.swiglu_limit)
        assert rep["rel"] < parity.TOL_Y
    finally:
        layer.close()


@pytest.mark.parametrize("T,bad", [(16, 5), (300, 123)])
def test_nan_token_is_contained(tiny, T, bad):
    lay, layer = tiny
    parity.check_nan_token(layer, lay, T, bad, WL.k, WL.E, WL.route_scale, WL.swiglu_limit)


def test_nan_token_is_contained_warp_topk(cuda_device):
    """Above 1024 tokens the top-k runs one warp per token."""
    lay = synth.make_layer(WL.with_tokens(1100), device="cpu")
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=1100)
    try:
        parity.check_nan_token(layer, lay, 1100, 1037, WL.k, WL.E, WL.route_scale, WL.swiglu_limit)
    finally:
        layer.close()


def _check_tile_list(tiles, n_shared_end, cnt, off, E, gateup, longest_first):
    """Every group's rows covered once per weight tile; shared tiles first; with
    many tokens per expert each (group, weight tile)'s token tiles adjacent, full
    ones first, and the groups with a single token tile shorter than the widest at
    the end, by row count non-increasing; else the routed tiles in group order."""
    g = tiles[:, 0] & 0xFFFF
    mt = tiles[:, 0] >> 16
    y, z, rows = tiles[:, 1], tiles[:, 2], tiles[:, 3]
    assert np.all(g[:n_shared_end] >= E) and np.all(g[n_shared_end:] < E)
    r = rows[n_shared_end:]
    if longest_first:
        gr, mr = g[n_shared_end:], mt[n_shared_end:]
        key = gr * 65536 + mr
        runs = np.flatnonzero(np.r_[True, key[1:] != key[:-1]])          # starts of (group, m tile) runs
        assert len(np.unique(key[runs])) == len(runs), "a (group, m tile)'s token tiles are not adjacent"
        ends = np.r_[runs[1:], len(key)]
        for a_, b_ in zip(runs, ends):
            assert np.all(r[a_:b_ - 1] >= r[a_ + 1:b_]), "full token tiles do not come first"
        single = (ends - runs) == 1
        cold = single & (r[runs] < r.max())                               # no full tile for sure
        if cold.any():
            first = int(np.argmax(cold))
            assert np.all(cold[first:]), "groups without a full tile are not last"
            rc = r[runs[first:]]
            assert np.all(rc[:-1] >= rc[1:]), "the tail is not longest first"
    else:
        gr = g[n_shared_end:]
        full = r == r.max()
        assert np.all(gr[:-1] <= gr[1:]) or np.all(np.diff(gr[~full]) >= 0), "routed tiles not in group order"
    assert np.all(rows > 0)
    m_tiles = int(mt.max()) + 1
    for grp in range(len(cnt)):
        sel = g == grp
        if cnt[grp] == 0:
            assert not sel.any()
            continue
        assert set(mt[sel].tolist()) == set(range(m_tiles))
        for m in range(m_tiles):
            s2 = sel & (mt == m)
            cover = np.zeros(cnt[grp], dtype=np.int64)
            for zz, rr in zip(z[s2], rows[s2]):
                cover[zz - off[grp]: zz - off[grp] + rr] += 1
            assert np.all(cover == 1), f"group {grp} m tile {m}: rows covered {cover.min()}..{cover.max()} times"
    if gateup:
        shared = g >= E
        assert np.array_equal(y[~shared], z[~shared]) and np.array_equal(y[shared], z[shared] - off[g[shared]])
    else:
        assert np.array_equal(y, z)


@pytest.mark.parametrize("T,hot", [(17, False), (64, False), (300, False), (700, False), (300, True), (700, True)])
def test_tile_lists_are_complete_and_longest_first(tiny, cuda_device, T, hot):
    lay, layer = tiny
    made = None
    if hot:
        bias = torch.zeros(WL.E, dtype=torch.float32, device=cuda_device)
        bias[:2] = 6.0
        made = layer = moe.MoELayer.from_layer(dict(lay, bias=bias), top_k=WL.k, max_tokens=700)
    try:
        x = lay["x"][:T].contiguous()
        _run(layer, x)
        dev = x.device
        G = WL.E + WL.n_shared
        nt = layer.inspect(moe.BUF_NTILES, torch.empty(7, dtype=torch.int32, device=dev)).cpu().numpy()
        cnt = layer.inspect(moe.BUF_COUNTS, torch.empty(G, dtype=torch.int32, device=dev)).cpu().numpy()
        off = layer.inspect(moe.BUF_OFFSETS, torch.empty(G + 1, dtype=torch.int32, device=dev)).cpu().numpy()
        for which, n, ns, thin, gateup in ((moe.BUF_TILES_GU, nt[0], nt[2], nt[5], True),
                                           (moe.BUF_TILES_DN, nt[1], nt[3], nt[6], False)):
            tl = layer.inspect(which, torch.empty((int(n), 4), dtype=torch.int32, device=dev)).cpu().numpy()
            _check_tile_list(tl.astype(np.int64), int(ns), cnt.astype(np.int64), off.astype(np.int64), WL.E, gateup,
                             longest_first=T > 32)
            # the thin tail: tiles of routed groups of at most 32 rows in all, and every
            # such group's tiles when the list is ordered longest first (else it is empty)
            g = tl[:, 0] & 0xFFFF
            assert int(ns) <= int(thin) <= int(n)
            assert np.all(g[thin:] < WL.E) and np.all(cnt[g[thin:]] <= 32)
            if T > 32:
                assert np.all(cnt[g[ns:thin]] > 32)
            else:
                assert thin == n
    finally:
        if made is not None:
            made.close()


@pytest.mark.parametrize("T", [5, 40, 300, 700])
def test_poisoned_workspace_gives_the_same_bits(tiny, T):
    """Every scratch buffer filled with 0xFF bytes (NaN floats, -1 indices) between
    two forwards of the same tokens: the outputs are bit-identical, so no forward
    reads anything an earlier call left in the workspace."""
    lay, layer = tiny
    x = lay["x"][:T].contiguous()
    y1, i1, w1 = _run(layer, x)
    y1 = y1.clone()
    layer.fill_workspace(0xFF)
    y2, i2, w2 = _run(layer, x)
    assert torch.equal(y1, y2) and torch.equal(i1, i2) and torch.equal(w1, w2)


@pytest.mark.parametrize("n_ok", [0, 1, 4, 12, 20])
def test_create_failing_allocation_leaks_nothing(tiny, cuda_device, n_ok, monkeypatch):
    """moe_create whose (n_ok+1)-th device allocation fails returns MOE_ERR_OOM and
    hands back every byte it took (free device memory is unchanged). A BF16 layer
    makes about two dozen allocations, so every n_ok here fails one."""
    lay, _ = tiny
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(cuda_device)
    monkeypatch.setenv("MOE_TEST_FAIL_ALLOC_AFTER", str(n_ok))
    with pytest.raises(moe.MoEError) as ei:
        moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=700)
    assert ei.value.status == moe.MOE_ERR_OOM
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(cuda_device)
    assert abs(free1 - free0) <= 2 << 20, f"free memory moved by {free0 - free1} bytes"
    # a budget above the allocation count changes nothing
    monkeypatch.setenv("MOE_TEST_FAIL_ALLOC_AFTER", "1000")
    ok = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=64)
    ok.close()
    monkeypatch.delenv("MOE_TEST_FAIL_ALLOC_AFTER")
