"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bars (from the workload definitions): the neighbour table N and the map M are
bit-exact; fp32 outputs satisfy |err| <= 1e-5 * (1 + |ref|) element by element;
bf16-input outputs (fp32 accumulation) satisfy max|err| <= 2e-2 * max|ref| per
tensor.  Full-size configurations are checked in full, the oracle running on
frame ranges in parallel worker processes (frames are independent).
"""
import numpy as np
import pytest
import torch

from sparse_convolution_pruned_b200 import workloads as wl

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_convolution_pruned_b200 import build, svconv
    build.build()
    assert svconv.svconv_read_error_word() == 0
    return svconv


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def check_f32(got, ref, what):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    bad = err > F32_TOL * (1.0 + np.abs(ref))
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max err {err.max():.3e}"


def check_bf16(got, ref, what):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref).max() if ref.size else 0.0
    lim = BF16_TOL * (np.abs(ref).max() if ref.size else 0.0)
    assert err <= lim, f"{what}: max err {err:.4e} > {lim:.4e}"


def gpu_index(sv, w, want_map=True):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nbr, M = sv.svconv_build_index(dev(w.coords), dev(w.frame_off), w.T, w.H, w.W, want_map=want_map, status=st)
    torch.cuda.synchronize()
    return nbr, M, int(st.item())


# ------------------------------------------------------------------ index build
INDEX_CASES = [
    ("tiny", lambda: wl.tiny_f32()),
    ("small_c", lambda: wl.small_c_bf16()),
    ("large_c_fwd", lambda: wl.large_c_fwd_bf16()),
    ("large_c_bwd", lambda: wl.large_c_bwd_bf16()),
    ("all_kept_7x13", lambda: wl.custom_conv(seed=5, T=3, H=7, W=13, keep_frac=1.0, Cin=4, Cout=4, dtype="f32")),
    ("one_per_frame", lambda: wl.custom_conv(seed=6, T=9, H=5, W=5, keep_frac=1 / 25, Cin=4, Cout=4, dtype="f32")),
    ("shuffled_empty", lambda: wl.custom_conv(seed=7, T=6, H=16, W=16, keep_frac=0.4, Cin=4, Cout=4, dtype="f32",
                                              shuffle=True, empty_frames=(0, 3, 5))),
    ("max_grid_128x128", lambda: wl.custom_conv(seed=8, T=2, H=128, W=128, keep_frac=0.3, Cin=4, Cout=4,
                                                dtype="f32", shuffle=True)),
    ("single_row_1x40", lambda: wl.custom_conv(seed=9, T=4, H=1, W=40, keep_frac=0.5, Cin=4, Cout=4, dtype="f32")),
    # thousands of frames: several frames per CTA, empty frames among them, shuffled tokens
    ("many_frames_5x6", lambda: wl.custom_conv(seed=10, T=6000, H=5, W=6, keep_frac=0.5, Cin=4, Cout=4,
                                               dtype="f32", shuffle=True, empty_frames=tuple(range(0, 6000, 7)))),
]


@pytest.mark.parametrize("name,make", INDEX_CASES, ids=[c[0] for c in INDEX_CASES])
def test_index_bit_exact(sv, orc, name, make):
    w = make()
    ref_n, ref_m, ref_st = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W)
    assert ref_st == 0
    nbr, M, st = gpu_index(sv, w)
    assert st == 0
    np.testing.assert_array_equal(nbr.cpu().numpy(), ref_n)
    np.testing.assert_array_equal(M.cpu().numpy(), ref_m)


def test_index_adapter_size_and_empty(sv, orc):
    a = wl.adapter_bf16(T=3072, D=64, R=64)  # long-video token layout; features unused here
    ref_n, _, _ = orc.build_index(a.coords, a.frame_off, a.T, a.H, a.W, want_map=False)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nbr, _ = sv.svconv_build_index(dev(a.coords), dev(a.frame_off), a.T, a.H, a.W, status=st)
    np.testing.assert_array_equal(nbr.cpu().numpy(), ref_n)
    assert st.item() == 0
    # no tokens at all: M is all -1
    coords = torch.zeros((0, 3), dtype=torch.int32, device="cuda")
    off = torch.zeros(5, dtype=torch.int32, device="cuda")
    nbr, M = sv.svconv_build_index(coords, off, 4, 3, 3, want_map=True, status=st)
    assert nbr.shape == (0, 9) and bool((M == -1).all()) and st.item() == 0


def test_index_error_flags_in_multi_frame_ctas(sv, orc):
    """Thousands of one-token frames (several frames per CTA); one frame at a time carries a bad
    coordinate, a wrong frame number or a duplicate: flags equal the oracle's, and every other
    frame's rows are still exact."""
    T = 5000
    coords = np.zeros((2 * T, 3), np.int32)
    coords[:, 0] = np.repeat(np.arange(T), 2)
    coords[0::2, 1], coords[0::2, 2] = 0, 0
    coords[1::2, 1], coords[1::2, 2] = 0, 1
    off = np.arange(0, 2 * T + 1, 2, dtype=np.int32)
    for kind in ("coord", "frame", "dup"):
        c = coords.copy()
        k = 2 * 2501 + 1
        if kind == "coord":
            c[k, 2] = 9
        elif kind == "frame":
            c[k, 0] = 2500
        else:
            c[k, 1:] = c[k - 1, 1:]
        ref_n, _, ref_st = orc.build_index(c, off, T, 3, 3, want_map=False)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        nbr, _ = sv.svconv_build_index(dev(c), dev(off), T, 3, 3, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == ref_st, (kind, int(st.item()), ref_st)
        got = nbr.cpu().numpy()
        ok_rows = np.ones(2 * T, bool)
        ok_rows[2 * 2500: 2 * 2502] = False  # the frames touched by the bad token
        np.testing.assert_array_equal(got[ok_rows], ref_n[ok_rows])
    assert sv.svconv_read_error_word() == 0


def test_index_error_flags_match_oracle(sv, orc):
    base = np.array([[0, 0, 0], [0, 1, 1], [1, 0, 0], [1, 1, 0]], np.int32)
    off = np.array([0, 2, 4], np.int32)
    cases = []
    c = base.copy(); c[1, 2] = 2; cases.append((c, off))            # x out of range
    c = base.copy(); c[1] = c[0]; cases.append((c, off))            # duplicate
    c = base.copy(); c[2, 0] = 0; cases.append((c, off))            # wrong frame
    cases.append((base, np.array([0, 3, 2], np.int32)))             # non-monotone offsets
    cases.append((base, np.array([0, 2, 3], np.int32)))             # offsets do not end at n
    for coords, fo in cases:
        _, _, ref_st = orc.build_index(coords, fo, 2, 2, 2)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sv.svconv_build_index(dev(coords), dev(fo), 2, 2, 2, status=st)
        got = int(st.item())
        if ref_st & orc.BAD_OFFSETS:
            # frames are validated independently on the GPU: with inconsistent
            # offsets other bits may be raised too, BAD_OFFSETS must be
            assert got & sv.STATUS_BAD_OFFSETS, (fo.tolist(), got)
        else:
            assert got == ref_st, (coords.tolist(), fo.tolist(), got, ref_st)
    # valid input afterwards still works and leaves the library word clean
    assert sv.svconv_read_error_word() == 0


# ------------------------------------------------------------------ fp32 path
F32_CASES = [
    ("tiny_config", lambda: wl.tiny_f32()),
    ("ragged_7x13_C8x24", lambda: wl.custom_conv(seed=21, T=5, H=7, W=13, keep_frac=0.45, Cin=8, Cout=24,
                                                dtype="f32", shuffle=True, empty_frames=(2,))),
    ("all_kept_C32", lambda: wl.custom_conv(seed=22, T=2, H=8, W=8, keep_frac=1.0, Cin=32, Cout=16, dtype="f32")),
    ("C64", lambda: wl.custom_conv(seed=23, T=8, H=16, W=16, keep_frac=0.3, Cin=64, Cout=64, dtype="f32")),
]


@pytest.mark.parametrize("name,make", F32_CASES, ids=[c[0] for c in F32_CASES])
def test_f32_fwd_bwd(sv, orc, name, make):
    w = make()
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    nbr, _, _ = gpu_index(sv, w, want_map=False)
    X, Wt, dY = dev(w.X), dev(w.Wt), dev(w.dY)
    b = dev(w.bias) if w.bias is not None else None
    Y = sv.svconv_fwd(X, nbr, Wt, b)
    dX = sv.svconv_bwd_data(dY, nbr, Wt)
    dW, db = sv.svconv_bwd_weight(dY, X, nbr)
    torch.cuda.synchronize()
    check_f32(Y.cpu().numpy(), orc.fwd(w.X, ref_n, w.Wt, w.bias), "Y")
    check_f32(dX.cpu().numpy(), orc.bwd_data(w.dY, ref_n, w.Wt), "dX")
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    check_f32(dW.cpu().numpy(), rdW, "dW")
    check_f32(db.cpu().numpy(), rdb, "db")
    assert sv.svconv_read_error_word() == 0


# ------------------------------------------------------------------ bf16 tensor-core path
def run_bf16(sv, w):
    nbr, _, st = gpu_index(sv, w, want_map=False)
    assert st == 0
    X, Wt, dY = dev(w.X, torch.bfloat16), dev(w.Wt, torch.bfloat16), dev(w.dY, torch.bfloat16)
    b = dev(w.bias) if w.bias is not None else None
    Y = sv.svconv_fwd(X, nbr, Wt, b)
    dX = sv.svconv_bwd_data(dY, nbr, Wt)
    dW, db = sv.svconv_bwd_weight(dY, X, nbr)
    torch.cuda.synchronize()
    return nbr, Y.float().cpu().numpy(), dX.float().cpu().numpy(), dW.cpu().numpy(), db.cpu().numpy()


BF16_FULL_CASES = [
    ("small_c_config", lambda: wl.small_c_bf16()),
    ("C256_T24_bias", lambda: wl.large_c_fwd_bf16(T=24)),
    ("C128x192_ragged", lambda: wl.custom_conv(seed=31, T=7, H=9, W=14, keep_frac=0.55, Cin=128, Cout=192,
                                               dtype="bf16", shuffle=True, empty_frames=(3,))),
    ("C64x256_one_tile_tail", lambda: wl.custom_conv(seed=32, T=3, H=6, W=7, keep_frac=0.9, Cin=64, Cout=256,
                                                     dtype="bf16")),
    ("C320x64_allkept", lambda: wl.custom_conv(seed=33, T=2, H=12, W=12, keep_frac=1.0, Cin=320, Cout=64,
                                               dtype="bf16")),
    # W + 1 = 81 packed rows: vertical neighbours fall outside the kernels' staged
    # halo windows and are read from global memory
    ("wide_grid_5x80_C64", lambda: wl.custom_conv(seed=34, T=6, H=5, W=80, keep_frac=0.6, Cin=64, Cout=64,
                                                  dtype="bf16")),
]


@pytest.mark.parametrize("name,make", BF16_FULL_CASES, ids=[c[0] for c in BF16_FULL_CASES])
def test_bf16_full(sv, orc, name, make):
    w = make()
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    nbr, Y, dX, dW, db = run_bf16(sv, w)
    check_bf16(Y, orc.fwd(w.X, ref_n, w.Wt, w.bias), "Y")
    check_bf16(dX, orc.bwd_data(w.dY, ref_n, w.Wt), "dX")
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    check_bf16(dW, rdW, "dW")
    check_bf16(db, rdb, "db")
    assert sv.svconv_read_error_word() == 0


@pytest.mark.parametrize("make,with_bwd", [(wl.large_c_fwd_bf16, False), (wl.large_c_bwd_bf16, True)],
                         ids=["large_c_fwd", "large_c_bwd"])
def test_bf16_full_size_complete(sv, orc, make, with_bwd):
    """The large-channel workloads at full size, every output element against the oracle
    (run on frame ranges in parallel worker processes: frames are independent)."""
    import oracle_pool
    w = make()
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    nbr, Y, dX, dW, db = run_bf16(sv, w)
    np.testing.assert_array_equal(nbr.cpu().numpy(), ref_n)
    ref = oracle_pool.conv_full(w, ref_n, do_fwd=True, do_bwd=with_bwd)
    check_bf16(Y, ref["Y"], "Y")
    if with_bwd:
        check_bf16(dX, ref["dX"], "dX")
        check_bf16(dW, ref["dW"], "dW")
        check_bf16(db, ref["db"], "db")
    assert sv.svconv_read_error_word() == 0


FUSED_BWD_CASES = [
    ("small_c_concurrent", lambda: wl.small_c_bf16(), torch.bfloat16),
    # 256-channel multiples: the two gradients side by side on disjoint SMs (CTA budgets from the
    # cost model; the weight gradient with its own, smaller split count)
    ("C256_T48_concurrent", lambda: wl.large_c_bwd_bf16(T=48), torch.bfloat16),
    ("C512x256_concurrent", lambda: wl.custom_conv(seed=34, T=6, H=16, W=16, keep_frac=0.5, Cin=512, Cout=256,
                                                   dtype="bf16", shuffle=True, empty_frames=(2,)), torch.bfloat16),
    ("C64_tiny_frames_concurrent", lambda: wl.custom_conv(seed=42, T=5, H=4, W=4, keep_frac=[0.0, 1 / 16, 0.0, 1.0, 0.5],
                                                          Cin=64, Cout=64, dtype="bf16"), torch.bfloat16),
    ("C128x192_sequential", lambda: wl.custom_conv(seed=31, T=7, H=9, W=14, keep_frac=0.55, Cin=128, Cout=192,
                                                   dtype="bf16", shuffle=True, empty_frames=(3,)), torch.bfloat16),
    ("tiny_f32_sequential", lambda: wl.tiny_f32(), torch.float32),
]


@pytest.mark.parametrize("name,make,dtype", FUSED_BWD_CASES, ids=[c[0] for c in FUSED_BWD_CASES])
def test_fused_bwd(sv, orc, name, make, dtype):
    w = make()
    nbr, _, st = gpu_index(sv, w, want_map=False)
    assert st == 0
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    X, Wt, dY = dev(w.X, dtype), dev(w.Wt, dtype), dev(w.dY, dtype)
    dX, dW, db = sv.svconv_bwd(dY, X, nbr, Wt)
    dX2, dW2, db2 = sv.svconv_bwd(dY, X, nbr, Wt)
    dX_sep = sv.svconv_bwd_data(dY, nbr, Wt)
    torch.cuda.synchronize()
    assert torch.equal(dX, dX_sep)                                   # same kernel, same sums
    assert torch.equal(dX, dX2) and torch.equal(dW, dW2) and torch.equal(db, db2)  # deterministic
    check = check_bf16 if dtype == torch.bfloat16 else check_f32
    check(dX.float().cpu().numpy(), orc.bwd_data(w.dY, ref_n, w.Wt), "dX")
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    check(dW.cpu().numpy(), rdW, "dW")
    check(db.cpu().numpy(), rdb, "db")
    assert sv.svconv_read_error_word() == 0


@pytest.mark.parametrize("make", [lambda: wl.small_c_bf16(T=96), lambda: wl.large_c_bwd_bf16(T=24)], ids=["C64", "C256"])
def test_fused_bwd_in_cuda_graph(sv, make):
    w = make()
    nbr, _, st = gpu_index(sv, w, want_map=False)
    X, Wt, dY = dev(w.X, torch.bfloat16), dev(w.Wt, torch.bfloat16), dev(w.dY, torch.bfloat16)
    ref = [t.clone() for t in sv.svconv_bwd(dY, X, nbr, Wt)]  # first call outside capture
    dX = torch.zeros_like(ref[0])
    dW = torch.zeros_like(ref[1])
    db = torch.zeros_like(ref[2])
    ws = torch.empty(max(16, sv.svconv_bwd_workspace_size(sv.BF16, w.n, w.Cin, w.Cout)), dtype=torch.uint8,
                     device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            sv.svconv_bwd(dY, X, nbr, Wt, dX=dX, dW=dW, db=db, workspace=ws)
        g.replay()
    torch.cuda.synchronize()
    for got, want in zip((dX, dW, db), ref):
        assert torch.equal(got, want)
    assert sv.svconv_read_error_word() == 0


def test_bf16_deterministic(sv):
    w = wl.large_c_bwd_bf16(T=48)
    a = run_bf16(sv, w)
    b = run_bf16(sv, w)
    for x, y in zip(a[1:], b[1:]):
        assert np.array_equal(x, y)


def test_bf16_one_token_and_empty_frames(sv, orc):
    w = wl.custom_conv(seed=41, T=5, H=4, W=4, keep_frac=[0.0, 1 / 16, 0.0, 1.0, 0.5], Cin=64, Cout=64, dtype="bf16")
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    nbr, Y, dX, dW, db = run_bf16(sv, w)
    check_bf16(Y, orc.fwd(w.X, ref_n, w.Wt, w.bias), "Y")
    check_bf16(dX, orc.bwd_data(w.dY, ref_n, w.Wt), "dX")
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    check_bf16(dW, rdW, "dW")


def test_bwd_weight_empty_input_zeroes(sv):
    X = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    dY = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    nbr = torch.zeros((0, 9), dtype=torch.int32, device="cuda")
    dW = torch.full((64, 9, 64), 7.0, device="cuda")
    db = torch.full((64,), 7.0, device="cuda")
    sv.svconv_bwd_weight(dY, X, nbr, dW=dW, db=db)
    assert float(dW.abs().max()) == 0.0 and float(db.abs().max()) == 0.0


# ------------------------------------------------------------------ adapter
def adapter_gpu(sv, a, chunk_T):
    nbr, _, st = gpu_index(sv, a, want_map=False)
    assert st == 0
    off = a.frame_off.astype(np.int64)
    max_rows = int(max(off[min(t + chunk_T, a.T)] - off[t] for t in range(0, a.T, chunk_T)))
    X = dev(a.X, torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sv.svconv_adapter_fwd(X, nbr, dev(a.frame_off), a.T, dev(a.Wd, torch.bfloat16), dev(a.Wc, torch.bfloat16),
                          dev(a.Wu, torch.bfloat16), chunk_T=chunk_T, max_chunk_rows=max_rows, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return X


def test_adapter_small_full(sv, orc):
    a = wl.adapter_bf16(seed=11, T=20, D=256, R=128)
    ref_n, _, _ = orc.build_index(a.coords, a.frame_off, a.T, a.H, a.W, want_map=False)
    out = adapter_gpu(sv, a, chunk_T=6).float().cpu().numpy()
    ref = orc.adapter_fwd(a.X, ref_n, 0, a.n, a.Wd, a.Wc, a.Wu)
    check_bf16(out, ref, "adapter out")
    check_bf16(out - a.X, ref - a.X, "adapter delta")


@pytest.fixture(scope="module")
def long_video(orc):
    """The long-video adapter workload and its oracle output for every row (computed once)."""
    import oracle_pool
    a = wl.adapter_bf16()
    ref_n, _, _ = orc.build_index(a.coords, a.frame_off, a.T, a.H, a.W, want_map=False)
    return a, oracle_pool.adapter_full(a, ref_n)


@pytest.mark.parametrize("chunk_T", [512, 1024])  # 1024: the chunking bench.py times
def test_adapter_long_video_config(sv, long_video, chunk_T):
    """Full size, every row against the oracle: all chunk boundaries (frames 511/512,
    1023/1024, 2047/2048, ...) and the middle chunks included."""
    a, ref = long_video
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    out = adapter_gpu(sv, a, chunk_T=chunk_T)
    peak = torch.cuda.max_memory_allocated() - base
    assert peak <= 1 << 30, f"peak {peak / 2**20:.0f} MiB"
    out = out.float().cpu().numpy()
    check_bf16(out, ref, "adapter out")
    check_bf16(out - a.X, ref - a.X, "adapter delta")
    # each chunk boundary on its own (a local error there would be small against the global max)
    off = a.frame_off
    for t in range(chunk_T, a.T, chunk_T):
        r0, r1 = int(off[t - 6]), int(off[t + 6])
        check_bf16(out[r0:r1] - a.X[r0:r1], ref[r0:r1] - a.X[r0:r1], f"delta around frame {t}")
    assert sv.svconv_read_error_word() == 0


# ------------------------------------------------------------------ failure detection / host errors
def test_bounded_wait_times_out_cleanly(sv):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sv.svconv_selftest_timeout(st, 20000)  # 20 ms on a barrier nothing arrives at
    torch.cuda.synchronize()
    assert int(st.item()) & sv.STATUS_TIMEOUT
    # the context is still usable
    w = wl.tiny_f32()
    nbr, _, s2 = gpu_index(sv, w)
    assert s2 == 0


def test_host_errors_on_device(sv):
    X = torch.zeros((10, 96), dtype=torch.bfloat16, device="cuda")
    nbr = torch.zeros((10, 9), dtype=torch.int32, device="cuda")
    Wt = torch.zeros((64, 9, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sv.SvconvError) as e:
        sv.svconv_fwd(X, nbr, Wt)  # C_in = 96 is not a multiple of 64
    assert e.value.code == -3
    Wt2 = torch.zeros((64, 9, 64), dtype=torch.bfloat16, device="cuda")
    X3 = torch.zeros((10 * 64 + 4,), dtype=torch.bfloat16, device="cuda")[4:].view(10, 64)
    with pytest.raises(sv.SvconvError) as e:
        sv.svconv_fwd(X3, nbr, Wt2)  # 8-byte offset: rejected
    assert e.value.code == -4
    dW = torch.empty((64, 9, 64), device="cuda")
    ws = torch.empty((16,), dtype=torch.uint8, device="cuda")
    X4 = torch.zeros((10, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sv.SvconvError) as e:
        sv.svconv_bwd_weight(X4, X4, nbr, dW=dW, workspace=ws)
    assert e.value.code == -5


def test_bad_neighbour_index_is_flagged_not_faulted(sv):
    w = wl.custom_conv(seed=51, T=2, H=8, W=8, keep_frac=0.5, Cin=64, Cout=64, dtype="bf16")
    nbr, _, _ = gpu_index(sv, w, want_map=False)
    nbr[3, 2] = w.n + 1000  # outside the feature rows
    nbr[5, 7] = -77         # negative but not -1: still zero padding
    X = dev(w.X, torch.bfloat16)
    Wt = dev(w.Wt, torch.bfloat16)
    sv.svconv_fwd(X, nbr, Wt)
    sv.svconv_bwd_data(X, nbr, Wt)
    sv.svconv_bwd_weight(X, X, nbr)
    assert sv.svconv_read_error_word() & sv.STATUS_BAD_INDEX
    assert sv.svconv_read_error_word() == 0  # reading clears it


# ------------------------------------------------------------------ e4m3 forward (large channels)
def run_e4m3_fwd(sv, w):
    nbr, _, st = gpu_index(sv, w, want_map=False)
    assert st == 0
    X = dev(w.X).to(torch.float8_e4m3fn)
    Wt = dev(w.Wt).to(torch.float8_e4m3fn)
    assert torch.equal(X.float().cpu(), torch.from_numpy(w.X))  # the inputs are e4m3 values already
    b = dev(w.bias) if w.bias is not None else None
    Y = sv.svconv_fwd(X, nbr, Wt, b)
    Y2 = sv.svconv_fwd(X, nbr, Wt, b)
    torch.cuda.synchronize()
    assert Y.dtype == torch.bfloat16 and torch.equal(Y, Y2)
    return Y.float().cpu().numpy()


E4M3_CASES = [
    ("C256_T24", lambda: wl.large_c_fwd_e4m3(T=24)),
    ("C128x256_ragged_shuffled", lambda: wl.custom_conv(seed=35, T=7, H=9, W=14, keep_frac=0.55, Cin=128, Cout=256,
                                                        dtype="bf16", shuffle=True, empty_frames=(3,))),
    ("C384x512_wide_grid", lambda: wl.custom_conv(seed=36, T=4, H=5, W=80, keep_frac=0.6, Cin=384, Cout=512,
                                                  dtype="bf16")),
]


@pytest.mark.parametrize("name,make", E4M3_CASES, ids=[c[0] for c in E4M3_CASES])
def test_e4m3_fwd(sv, orc, name, make):
    w = make()
    w.X, w.Wt = wl.round_to_e4m3(w.X), wl.round_to_e4m3(w.Wt)
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    check_bf16(run_e4m3_fwd(sv, w), orc.fwd(w.X, ref_n, w.Wt, w.bias), "Y e4m3")
    assert sv.svconv_read_error_word() == 0


def test_e4m3_fwd_full_size_complete(sv, orc):
    import oracle_pool
    w = wl.large_c_fwd_e4m3()
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    Y = run_e4m3_fwd(sv, w)
    check_bf16(Y, oracle_pool.conv_full(w, ref_n, do_fwd=True, do_bwd=False)["Y"], "Y e4m3 full size")
    assert sv.svconv_read_error_word() == 0


def test_e4m3_rejects_unsupported_channels(sv):
    X = torch.zeros((10, 64), dtype=torch.float8_e4m3fn, device="cuda")
    nbr = torch.zeros((10, 9), dtype=torch.int32, device="cuda")
    Wt = torch.zeros((256, 9, 64), dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(sv.SvconvError) as e:
        sv.svconv_fwd(X, nbr, Wt)  # C_in = 64 is not a multiple of 128
    assert e.value.code == -3


# ------------------------------------------------------------------ single pass over dY (64 channels)
SINGLE_PASS_CASES = [
    ("small_c_config", lambda: wl.small_c_bf16()),
    ("tiny_and_empty_frames", lambda: wl.custom_conv(seed=43, T=5, H=4, W=4, keep_frac=[0.0, 1 / 16, 0.0, 1.0, 0.5],
                                                     Cin=64, Cout=64, dtype="bf16")),
    ("shuffled_ragged", lambda: wl.custom_conv(seed=44, T=9, H=11, W=13, keep_frac=0.6, Cin=64, Cout=64, dtype="bf16",
                                               shuffle=True, empty_frames=(4,))),
    # W + 1 = 81 packed rows: neighbours outside the staged windows are read from global memory
    ("wide_grid_5x80", lambda: wl.custom_conv(seed=45, T=6, H=5, W=80, keep_frac=0.6, Cin=64, Cout=64, dtype="bf16")),
]


@pytest.mark.parametrize("name,make", SINGLE_PASS_CASES, ids=[c[0] for c in SINGLE_PASS_CASES])
def test_bwd_single_pass(sv, orc, name, make):
    w = make()
    nbr, _, st = gpu_index(sv, w, want_map=False)
    assert st == 0
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    X, Wt, dY = dev(w.X, torch.bfloat16), dev(w.Wt, torch.bfloat16), dev(w.dY, torch.bfloat16)
    dX, dW, db = sv.svconv_bwd_single_pass(dY, X, nbr, Wt)
    dX2, dW2, db2 = sv.svconv_bwd_single_pass(dY, X, nbr, Wt)
    torch.cuda.synchronize()
    assert torch.equal(dX, dX2) and torch.equal(dW, dW2) and torch.equal(db, db2)  # deterministic
    assert torch.equal(dX, sv.svconv_bwd_data(dY, nbr, Wt))  # same products, same order per output
    check_bf16(dX.float().cpu().numpy(), orc.bwd_data(w.dY, ref_n, w.Wt), "dX")
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    check_bf16(dW.cpu().numpy(), rdW, "dW")
    check_bf16(db.cpu().numpy(), rdb, "db")
    assert sv.svconv_read_error_word() == 0
