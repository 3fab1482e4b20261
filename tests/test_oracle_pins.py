"""Pins for the CPU oracle: each check ties it to something other than itself.

* a hand-worked fixture (tests/golden/hand_3x3.json) from the definitions of M, N
  and the convolution on the SV-TAD page (Key Designs 1-2);
* all tokens kept -> torch's conv2d in float64 (a library routine);
* any mask -> scatter to a zero grid, torch conv2d, gather back: the page's
  claim that the sparse operator is lossless w.r.t. dense reconstruction;
* backward -> torch autograd of that dense pipeline, exact central differences
  (the operator is linear), adjoint identities;
* the neighbour table -> an O(n^2) brute-force search and its invariants;
* bf16 rounding -> torch's RNE cast; adapter -> the same stages composed from
  torch float64 ops.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from sparse_convolution_pruned_b200 import workloads as wl

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def torch_weight(Wt):
    """W[o][j][i] with j=(a*3+b) -> torch conv2d weight [o][i][a][b]."""
    Cout, _, Cin = Wt.shape
    return torch.from_numpy(np.asarray(Wt, np.float64)).reshape(Cout, 3, 3, Cin).permute(0, 3, 1, 2).contiguous()


def scatter_grid(X, coords, T, H, W):
    n, C = X.shape
    G = torch.zeros((T, C, H, W), dtype=torch.float64)
    c = torch.from_numpy(np.asarray(coords, np.int64))
    G[c[:, 0], :, c[:, 1], c[:, 2]] = torch.as_tensor(np.asarray(X, np.float64))
    return G


def dense_pipeline(X, Wt, bias, coords, T, H, W):
    """Dense reconstruction: scatter -> conv2d (padding 1) -> gather kept positions."""
    c = torch.from_numpy(np.asarray(coords, np.int64))
    G = scatter_grid(X, coords, T, H, W)
    b = None if bias is None else torch.as_tensor(np.asarray(bias, np.float64))
    Yg = F.conv2d(G, torch_weight(Wt), b, padding=1)
    return Yg[c[:, 0], :, c[:, 1], c[:, 2]]


def brute_nbr(coords):
    n = coords.shape[0]
    N = -np.ones((n, 9), dtype=np.int32)
    for k in range(n):
        t, y, x = coords[k]
        for j in range(9):
            dy, dx = j // 3 - 1, j % 3 - 1
            for m in range(n):
                if coords[m, 0] == t and coords[m, 1] == y + dy and coords[m, 2] == x + dx:
                    N[k, j] = m
    return N


# ---------------------------------------------------------------- hand fixture
def test_hand_fixture(orc):
    g = json.load(open(os.path.join(GOLD, "hand_3x3.json")))
    nbr, M, st = orc.build_index(np.array(g["coords"]), np.array(g["frame_off"]), g["T"], g["H"], g["W"])
    assert st == 0
    np.testing.assert_array_equal(nbr, np.array(g["N"]))
    np.testing.assert_array_equal(M, np.array(g["M"]))
    Wt = np.array(g["Wt"], np.float64).reshape(1, 9, 1)
    X = np.array(g["X"], np.float64).reshape(-1, 1)
    Y = orc.fwd(X, nbr, Wt, np.array([g["bias"]]))
    np.testing.assert_array_equal(Y[:, 0], np.array(g["Y"]))
    dY = np.array(g["dY"], np.float64).reshape(-1, 1)
    np.testing.assert_array_equal(orc.bwd_data(dY, nbr, Wt)[:, 0], np.array(g["dX"]))
    dW, db = orc.bwd_weight(dY, X, nbr)
    np.testing.assert_array_equal(dW.reshape(-1), np.array(g["dW"], np.float64))
    assert db[0] == g["db"]


# ---------------------------------------------------------------- index build
@pytest.mark.parametrize("seed,T,H,W,frac,shuffle", [
    (0, 3, 8, 8, 0.5, False), (1, 4, 7, 13, 0.3, True), (2, 2, 5, 4, 1.0, False),
    (3, 5, 6, 6, 0.1, True), (4, 3, 1, 9, 0.6, False)])
def test_index_bruteforce_and_invariants(orc, seed, T, H, W, frac, shuffle):
    w = wl.custom_conv(seed=seed, T=T, H=H, W=W, keep_frac=frac, Cin=4, Cout=4, dtype="f32",
                       shuffle=shuffle, empty_frames=(1,) if T > 2 else ())
    nbr, M, st = orc.build_index(w.coords, w.frame_off, T, H, W)
    assert st == 0
    np.testing.assert_array_equal(nbr, brute_nbr(w.coords))
    n = w.n
    assert (M >= 0).sum() == n
    for k in range(n):
        t, y, x = w.coords[k]
        assert M[t, y, x] == k
        assert nbr[k, 4] == k
        for j in range(9):
            m = nbr[k, j]
            if m >= 0:
                assert nbr[m, 8 - j] == k  # mirror symmetry
                assert tuple(w.coords[m]) == (t, y + j // 3 - 1, x + j % 3 - 1)


def test_index_permutation_equivariance(orc):
    w = wl.custom_conv(seed=7, T=3, H=6, W=9, keep_frac=0.5, Cin=4, Cout=4, dtype="f32")
    nbr, _, _ = orc.build_index(w.coords, w.frame_off, 3, 6, 9)
    rng = np.random.default_rng(0)
    perm = np.arange(w.n)
    for t in range(3):  # permute inside frames only: frames stay contiguous
        a, b = w.frame_off[t], w.frame_off[t + 1]
        perm[a:b] = a + rng.permutation(b - a)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(w.n)
    nbr2, _, _ = orc.build_index(w.coords[perm], w.frame_off, 3, 6, 9)
    expect = np.where(nbr[perm] >= 0, inv[np.maximum(nbr[perm], 0)], -1)
    np.testing.assert_array_equal(nbr2, expect)
    Y = orc.fwd(w.X, nbr, w.Wt, w.bias)
    Y2 = orc.fwd(w.X[perm], nbr2, w.Wt, w.bias)
    np.testing.assert_array_equal(Y2, Y[perm])


def test_index_error_flags(orc):
    coords = np.array([[0, 0, 0], [0, 1, 1], [1, 0, 0]], np.int32)
    off = np.array([0, 2, 3], np.int32)
    assert orc.build_index(coords, off, 2, 2, 2)[2] == 0
    bad = coords.copy(); bad[1, 2] = 2
    assert orc.build_index(bad, off, 2, 2, 2)[2] & orc.BAD_COORD
    dup = coords.copy(); dup[1] = dup[0]
    assert orc.build_index(dup, off, 2, 2, 2)[2] & orc.DUPLICATE
    wrong_t = coords.copy(); wrong_t[2, 0] = 0
    assert orc.build_index(wrong_t, off, 2, 2, 2)[2] & orc.BAD_FRAME
    assert orc.build_index(coords, np.array([0, 3, 2], np.int32), 2, 2, 2)[2] & orc.BAD_OFFSETS
    assert orc.build_index(coords, np.array([0, 2, 4], np.int32), 2, 2, 2)[2] & orc.BAD_OFFSETS


# ---------------------------------------------------------------- forward
def test_fwd_all_kept_equals_torch_conv2d(orc):
    T, H, W, Cin, Cout = 2, 5, 7, 3, 4
    w = wl.custom_conv(seed=11, T=T, H=H, W=W, keep_frac=1.0, Cin=Cin, Cout=Cout, dtype="f32")
    nbr, _, _ = orc.build_index(w.coords, w.frame_off, T, H, W)
    Y = orc.fwd(w.X, nbr, w.Wt, w.bias)
    ref = dense_pipeline(w.X, w.Wt, w.bias, w.coords, T, H, W).numpy()
    np.testing.assert_allclose(Y, ref, rtol=1e-13, atol=1e-13)
    # the oracle's own direct dense loop agrees with torch too
    G = scatter_grid(w.X, w.coords, T, H, W)[0].permute(1, 2, 0).numpy()
    Yd = orc.dense_conv(G, w.Wt, w.bias)
    Yt = F.conv2d(torch.from_numpy(G).permute(2, 0, 1)[None], torch_weight(w.Wt),
                  torch.from_numpy(w.bias.astype(np.float64)), padding=1)[0].permute(1, 2, 0).numpy()
    np.testing.assert_allclose(Yd, Yt, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("seed,T,H,W,frac,Cin,Cout", [
    (21, 3, 8, 8, 0.5, 4, 5), (22, 4, 7, 13, 0.25, 8, 3), (23, 2, 16, 16, 0.3, 16, 16)])
def test_fwd_lossless_vs_dense_reconstruction(orc, seed, T, H, W, frac, Cin, Cout):
    w = wl.custom_conv(seed=seed, T=T, H=H, W=W, keep_frac=frac, Cin=Cin, Cout=Cout, dtype="f32",
                       shuffle=True, empty_frames=(1,))
    nbr, _, _ = orc.build_index(w.coords, w.frame_off, T, H, W)
    Y = orc.fwd(w.X, nbr, w.Wt, w.bias)
    ref = dense_pipeline(w.X, w.Wt, w.bias, w.coords, T, H, W).numpy()
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-12)
    # bit-exact against the oracle's own dense loop on the zero-filled grid
    G = scatter_grid(w.X, w.coords, T, H, W).permute(0, 2, 3, 1).numpy()
    for t in range(T):
        Yd = orc.dense_conv(G[t], w.Wt, w.bias)
        a, b = w.frame_off[t], w.frame_off[t + 1]
        c = w.coords[a:b]
        assert np.array_equal(Y[a:b], Yd[c[:, 1], c[:, 2]])
    # row-subset mode returns the same rows
    rows = np.array([0, w.n - 1, w.n // 2], np.int64)
    np.testing.assert_array_equal(orc.fwd(w.X, nbr, w.Wt, w.bias, rows=rows), Y[rows])


# ---------------------------------------------------------------- backward
@pytest.mark.parametrize("seed,T,H,W,frac,Cin,Cout", [(31, 3, 6, 9, 0.45, 5, 3), (32, 2, 8, 8, 1.0, 4, 4)])
def test_bwd_vs_torch_autograd(orc, seed, T, H, W, frac, Cin, Cout):
    w = wl.custom_conv(seed=seed, T=T, H=H, W=W, keep_frac=frac, Cin=Cin, Cout=Cout, dtype="f32", shuffle=True)
    nbr, _, _ = orc.build_index(w.coords, w.frame_off, T, H, W)
    Xt = torch.tensor(w.X, dtype=torch.float64, requires_grad=True)
    Wtt = torch.tensor(w.Wt, dtype=torch.float64, requires_grad=True)
    bt = torch.tensor(w.bias, dtype=torch.float64, requires_grad=True)
    c = torch.from_numpy(w.coords.astype(np.int64))
    G = torch.zeros((T, H, W, Cin), dtype=torch.float64)
    G = G.index_put((c[:, 0], c[:, 1], c[:, 2]), Xt).permute(0, 3, 1, 2)
    wtorch = Wtt.reshape(Cout, 3, 3, Cin).permute(0, 3, 1, 2)
    Yg = F.conv2d(G, wtorch, bt, padding=1)
    Y = Yg[c[:, 0], :, c[:, 1], c[:, 2]]
    (Y * torch.from_numpy(w.dY.astype(np.float64))).sum().backward()
    dX = orc.bwd_data(w.dY, nbr, w.Wt)
    dW, db = orc.bwd_weight(w.dY, w.X, nbr)
    np.testing.assert_allclose(dX, Xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dW, Wtt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.bwd_bias(w.dY), bt.grad.numpy(), rtol=1e-12, atol=1e-12)
    rows = np.array([w.n - 1, 0, 3], np.int64)
    np.testing.assert_allclose(orc.bwd_data(w.dY, nbr, w.Wt, rows=rows), dX[rows], rtol=1e-13, atol=1e-13)
    ent = np.array([[0, 0, 0], [Cout - 1, 8, Cin - 1], [1, 4, 2]], np.int32)
    np.testing.assert_allclose(orc.bwd_weight_entries(w.dY, w.X, nbr, ent),
                               dW[ent[:, 0], ent[:, 1], ent[:, 2]], rtol=1e-13, atol=1e-13)


def test_bwd_finite_differences(orc):
    """Exact central differences (the operator is linear in X and in W)."""
    T, H, W, Cin, Cout = 2, 5, 4, 3, 2
    w = wl.custom_conv(seed=41, T=T, H=H, W=W, keep_frac=0.6, Cin=Cin, Cout=Cout, dtype="f32", bias=False)
    nbr, _, _ = orc.build_index(w.coords, w.frame_off, T, H, W)
    X, Wt, dY = w.X.astype(np.float64), w.Wt.astype(np.float64), w.dY.astype(np.float64)
    L = lambda Xv, Wv: float((orc.fwd(Xv, nbr, Wv) * dY).sum())
    dX = orc.bwd_data(dY, nbr, Wt)
    dW, _ = orc.bwd_weight(dY, X, nbr)
    h = 0.5
    for k in range(w.n):
        for i in range(Cin):
            Xp, Xm = X.copy(), X.copy()
            Xp[k, i] += h; Xm[k, i] -= h
            assert abs((L(Xp, Wt) - L(Xm, Wt)) / (2 * h) - dX[k, i]) <= 1e-9 * (1 + abs(dX[k, i]))
    for idx in np.ndindex(Wt.shape):
        Wp, Wm = Wt.copy(), Wt.copy()
        Wp[idx] += h; Wm[idx] -= h
        assert abs((L(X, Wp) - L(X, Wm)) / (2 * h) - dW[idx]) <= 1e-9 * (1 + abs(dW[idx]))


def test_adjoint_identities(orc):
    w = wl.custom_conv(seed=51, T=6, H=16, W=16, keep_frac=0.3, Cin=16, Cout=8, dtype="f32")
    nbr, _, _ = orc.build_index(w.coords, w.frame_off, 6, 16, 16)
    X, Wt, dY = w.X.astype(np.float64), w.Wt.astype(np.float64), w.dY.astype(np.float64)
    lhs = float((orc.fwd(X, nbr, Wt) * dY).sum())
    assert abs(lhs - float((orc.bwd_data(dY, nbr, Wt) * X).sum())) <= 1e-10 * (1 + abs(lhs))
    dW, db = orc.bwd_weight(dY, X, nbr)
    assert abs(lhs - float((dW * Wt).sum())) <= 1e-10 * (1 + abs(lhs))
    assert abs(db.sum() - dY.sum()) <= 1e-10 * (1 + abs(dY.sum()))


# ---------------------------------------------------------------- bf16 + adapter
def test_round_bf16_matches_torch_rne(orc):
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 6, 2000),
                           [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3.0 + 2 ** -7, 0.0]]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.round_bf16(float(v)) for v in vals])
    np.testing.assert_array_equal(got, ref)
    assert orc.round_bf16(1 + 2 ** -8) == 1.0  # tie -> even
    assert orc.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    # the generator's rounding agrees with torch as well
    np.testing.assert_array_equal(wl.round_to_bf16(vals), torch.from_numpy(vals).to(torch.bfloat16).float().numpy())


def test_adapter_vs_torch_composition(orc):
    a = wl.adapter_bf16(seed=9, T=6, D=64, R=32)
    nbr, _, _ = orc.build_index(a.coords, a.frame_off, a.T, a.H, a.W)
    r0, r1 = int(a.frame_off[2]), int(a.frame_off[5])
    got = orc.adapter_fwd(a.X, nbr, r0, r1, a.Wd, a.Wc, a.Wu)
    bf = lambda t: t.to(torch.bfloat16).to(torch.float64)
    X = torch.from_numpy(a.X.astype(np.float64))
    H1 = bf(X @ torch.from_numpy(a.Wd.astype(np.float64)).T)
    conv = dense_pipeline(H1.numpy(), a.Wc, None, a.coords, a.T, a.H, a.W)
    H2 = bf(F.gelu(conv, approximate="none"))
    out = bf(X + H2 @ torch.from_numpy(a.Wu.astype(np.float64)).T)[r0:r1].numpy()
    np.testing.assert_allclose(got, out, rtol=0, atol=1e-9)


# ------------------------------------------------------------------ frame-parallel oracle runs
def test_frame_parallel_oracle_equals_the_direct_calls(orc):
    """The full-size GPU checks run the oracle on frame ranges in worker processes; rows of
    Y, dX and the adapter are then bit-identical to one direct call (frames are independent),
    and the summed weight / bias gradients equal the direct sums up to fp64 rounding."""
    import oracle_pool
    from sparse_convolution_pruned_b200 import workloads as wl
    w = wl.custom_conv(seed=61, T=9, H=6, W=7, keep_frac=0.5, Cin=8, Cout=12, dtype="f32", shuffle=True,
                       empty_frames=(0, 4, 8))
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    got = oracle_pool.conv_full(w, ref_n)
    assert np.array_equal(got["Y"], orc.fwd(w.X, ref_n, w.Wt, w.bias))
    assert np.array_equal(got["dX"], orc.bwd_data(w.dY, ref_n, w.Wt))
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    np.testing.assert_allclose(got["dW"], rdW, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["db"], rdb, rtol=1e-12, atol=1e-12)
    a = wl.adapter_bf16(seed=12, T=10, D=64, R=64)
    an, _, _ = orc.build_index(a.coords, a.frame_off, a.T, a.H, a.W, want_map=False)
    assert np.array_equal(oracle_pool.adapter_full(a, an), orc.adapter_fwd(a.X, an, 0, a.n, a.Wd, a.Wc, a.Wu))


def test_frame_ranges_cover_every_frame_once():
    import oracle_pool
    off = np.array([0, 0, 5, 5, 9, 30, 31, 31, 40], np.int64)
    for parts in (1, 2, 3, 5, 8, 50):
        r = oracle_pool.frame_ranges(off, parts)
        assert r[0][0] == 0 and r[-1][1] == len(off) - 1
        assert all(a < b for a, b in r) and all(r[i][1] == r[i + 1][0] for i in range(len(r) - 1))


# ------------------------------------------------------------------ asymmetric cross-attention
def _xattn_case(seed, G=3, A=2, R=32, heads=2, sizes=(7, 0, 11)):
    rng = np.random.default_rng(seed)
    goff = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    H = rng.standard_normal((int(goff[-1]), R))
    aux = rng.standard_normal((G, A, R))
    return H, goff, aux


def test_xattn_aux_equals_torch_sdpa(orc):
    """Per group, torch's scaled_dot_product_attention in float64 (heads split the channels),
    plus the residual; an empty group leaves its auxiliary tokens unchanged."""
    import torch
    import torch.nn.functional as F
    for heads in (1, 2, 4):
        H, goff, aux = _xattn_case(3 + heads, heads=heads)
        G, A, R = aux.shape
        d = R // heads
        got = orc.xattn_aux(H, goff, aux, heads=heads)
        for g in range(G):
            r0, r1 = goff[g], goff[g + 1]
            if r1 == r0:
                assert np.array_equal(got[g], aux[g])
                continue
            q = torch.from_numpy(aux[g]).view(A, heads, d).permute(1, 0, 2)
            kv = torch.from_numpy(H[r0:r1]).view(r1 - r0, heads, d).permute(1, 0, 2)
            att = F.scaled_dot_product_attention(q, kv, kv).permute(1, 0, 2).reshape(A, R).numpy()
            np.testing.assert_allclose(got[g], aux[g] + att, rtol=1e-12, atol=1e-12)


def test_xattn_aux_closed_forms(orc):
    rng = np.random.default_rng(8)
    R = 16
    H = rng.standard_normal((9, R))
    # a group of one row: the softmax weight is 1, so the update is that row
    goff = np.array([0, 1, 9], np.int32)
    aux = rng.standard_normal((2, 1, R))
    got = orc.xattn_aux(H, goff, aux)
    np.testing.assert_allclose(got[0, 0], aux[0, 0] + H[0], rtol=0, atol=1e-14)
    # a zero query scores every row 0: uniform weights, the update is the rows' mean
    aux0 = np.zeros((2, 1, R))
    got = orc.xattn_aux(H, goff, aux0)
    np.testing.assert_allclose(got[1, 0], H[1:9].mean(0), rtol=0, atol=1e-14)
    # a query far more aligned with one row than with the others (scores ~ 1e3 apart):
    # the softmax saturates on that row (and nothing overflows)
    Hs = rng.standard_normal((5, R))
    q = 300.0 * Hs[3] / np.linalg.norm(Hs[3])
    Hs[3] = 40.0 * Hs[3] / np.linalg.norm(Hs[3])
    got = orc.xattn_aux(Hs, np.array([0, 5], np.int32), q.reshape(1, 1, R))
    np.testing.assert_allclose(got[0, 0], q + Hs[3], rtol=0, atol=1e-9)


def test_xattn_aux_row_order_does_not_matter(orc):
    H, goff, aux = _xattn_case(13, G=2, sizes=(10, 6), heads=1)
    perm = np.concatenate([np.random.default_rng(1).permutation(10), 10 + np.random.default_rng(2).permutation(6)])
    np.testing.assert_allclose(orc.xattn_aux(H[perm], goff, aux), orc.xattn_aux(H, goff, aux), rtol=1e-12,
                               atol=1e-12)


def test_down_proj_equals_torch_matmul_then_bf16(orc):
    """The adapter's first stage: float64 matmul, then torch's round-to-nearest-even bf16 cast."""
    import torch
    rng = np.random.default_rng(21)
    X = rng.standard_normal((37, 64))
    Wd = rng.standard_normal((16, 64)) / 8
    want = (torch.from_numpy(X) @ torch.from_numpy(Wd).T).to(torch.bfloat16).double().numpy()
    assert np.array_equal(orc.down_proj(X, Wd), want)
