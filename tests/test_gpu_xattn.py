"""GPU parity of the auxiliary-token cross-attention (SV-TAD page, Key Design 3) through the
C ABI, against the oracle: the standalone entry point over grouped rows, and the chunked
adapter with the cross-attention over its down-projected features.

Bar: bf16 inputs with fp32 accumulation, max|err| <= 2e-2 max|ref| per tensor, applied to the
attention's update (aux_out - aux) as well as to aux_out itself.
"""
import numpy as np
import pytest
import torch

from sparse_convolution_pruned_b200 import workloads as wl

pytestmark = pytest.mark.gpu
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_convolution_pruned_b200 import build, svconv
    build.build()
    assert svconv.svconv_read_error_word() == 0
    return svconv


def check(got, ref, aux, what):
    for g, r, name in ((got, ref, "out"), (got - aux, ref - aux, "update")):
        err = np.abs(g - r).max()
        lim = BF16_TOL * np.abs(r).max()
        assert err <= lim, f"{what} {name}: max err {err:.3e} > {lim:.3e}"


def inputs(seed, sizes, A, R, scale=1.0):
    rng = np.random.default_rng(seed)
    goff = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    H = wl.round_to_bf16((scale * rng.standard_normal((int(goff[-1]), R))).astype(np.float32))
    aux = wl.round_to_bf16(rng.standard_normal((len(sizes), A, R)).astype(np.float32))
    return H, goff, aux


CASES = [
    ("one_group_R256", 1, (3000,), 1, 256, 1),
    ("groups_empty_ragged_heads2", 2, (700, 0, 1, 257, 256, 1300), 2, 256, 2),
    ("R128_heads4_A5", 3, (513, 90, 2049), 5, 128, 4),
    ("R64_A16", 4, (300, 1000), 16, 64, 1),
    ("R8_heads1", 5, (40, 9), 3, 8, 1),
]


@pytest.mark.parametrize("name,seed,sizes,A,R,heads", CASES, ids=[c[0] for c in CASES])
def test_xattn_aux_vs_oracle(sv, orc, name, seed, sizes, A, R, heads):
    H, goff, aux = inputs(seed, sizes, A, R)
    d = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).to(dt) if dt else
                            torch.from_numpy(np.ascontiguousarray(a))).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = sv.svconv_xattn_aux(d(H, torch.bfloat16), d(goff), d(aux, torch.bfloat16), max_group_rows=max(sizes),
                              heads=heads, status=st)
    out2 = sv.svconv_xattn_aux(d(H, torch.bfloat16), d(goff), d(aux, torch.bfloat16), max_group_rows=max(sizes),
                               heads=heads, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(out, out2)  # fixed merge order: bitwise reproducible
    ref = orc.xattn_aux(H, goff, aux, heads=heads)
    got = out.cpu().double().numpy()
    check(got, ref, aux, name)
    for g, sz in enumerate(sizes):
        if sz == 0:
            assert np.array_equal(got[g], aux[g])  # no rows: unchanged
    assert sv.svconv_read_error_word() == 0


def test_xattn_aux_long_video_rows(sv, orc):
    """One video's worth of down-projected rows (282,624 x 256, the long-video adapter's
    size) attended by one CLS token, as bench.py times it; also a saturated softmax."""
    H, goff, aux = inputs(9, (282624,), 1, 256)
    d = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).to(dt) if dt else
                            torch.from_numpy(np.ascontiguousarray(a))).cuda()
    out = sv.svconv_xattn_aux(d(H, torch.bfloat16), d(goff), d(aux, torch.bfloat16), max_group_rows=282624)
    torch.cuda.synchronize()
    check(out.cpu().double().numpy(), orc.xattn_aux(H, goff, aux), aux, "long video")
    # query aligned with one row far more than with any other: the softmax saturates there
    Hs, goff_s, _ = inputs(10, (5000,), 1, 256)
    u = Hs[1234] / np.linalg.norm(Hs[1234])
    Hs[1234] = wl.round_to_bf16((40.0 * u).astype(np.float32))
    q = wl.round_to_bf16((300.0 * u).astype(np.float32)).reshape(1, 1, 256)
    out = sv.svconv_xattn_aux(d(Hs, torch.bfloat16), d(goff_s), d(q, torch.bfloat16), max_group_rows=5000)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    check(out.cpu().double().numpy(), orc.xattn_aux(Hs, goff_s, q), q, "saturated")


def test_xattn_group_larger_than_bound_is_flagged(sv):
    H = torch.zeros((600, 64), dtype=torch.bfloat16, device="cuda")
    goff = torch.tensor([0, 600], dtype=torch.int32, device="cuda")
    aux = torch.zeros((1, 1, 64), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sv.svconv_xattn_aux(H, goff, aux, max_group_rows=100, status=st)  # covers 256 rows of 600
    torch.cuda.synchronize()
    assert int(st.item()) & sv.STATUS_CHUNK_OVERFLOW


def _adapter(sv, a, chunk_T, aux, heads):
    st0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    nbr, _ = sv.svconv_build_index(torch.from_numpy(a.coords).cuda(), torch.from_numpy(a.frame_off).cuda(), a.T,
                                   a.H, a.W, status=st0)
    off = a.frame_off.astype(np.int64)
    max_rows = int(max(off[min(t + chunk_T, a.T)] - off[t] for t in range(0, a.T, chunk_T)))
    d = lambda x, dt=None: (torch.from_numpy(np.ascontiguousarray(x)).to(dt) if dt else
                            torch.from_numpy(np.ascontiguousarray(x))).cuda()
    args = (nbr, d(a.frame_off), a.T, d(a.Wd, torch.bfloat16), d(a.Wc, torch.bfloat16), d(a.Wu, torch.bfloat16))
    X1 = d(a.X, torch.bfloat16)
    st1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    X1, aux_out = sv.svconv_adapter_fwd_xattn(X1, *args, d(aux, torch.bfloat16), chunk_T=chunk_T,
                                              max_chunk_rows=max_rows, heads=heads, status=st1)
    X2 = d(a.X, torch.bfloat16)
    sv.svconv_adapter_fwd(X2, *args, chunk_T=chunk_T, max_chunk_rows=max_rows)
    torch.cuda.synchronize()
    assert int(st0.item()) == 0 and int(st1.item()) == 0
    assert torch.equal(X1, X2)  # the adapter's own output is untouched by the cross-attention
    return aux_out.cpu().double().numpy()


def test_adapter_with_xattn_small(sv, orc):
    a = wl.adapter_bf16(seed=13, T=21, D=256, R=128)
    aux = wl.round_to_bf16(np.random.default_rng(3).standard_normal((3, 128)).astype(np.float32))
    got = _adapter(sv, a, 5, aux, heads=2)
    H1 = orc.down_proj(a.X, a.Wd)
    ref = orc.xattn_aux(H1, np.array([0, a.n], np.int32), aux[None], heads=2)[0]
    check(got, ref, aux, "adapter+xattn")


def test_adapter_with_xattn_long_video(sv):
    """The long-video adapter at full size with one CLS token over all 282,624 rows (three
    1,024-frame chunks, as bench.py runs it)."""
    import oracle
    import oracle_pool
    a = wl.adapter_bf16()
    aux = wl.round_to_bf16(np.random.default_rng(4).standard_normal((1, a.R)).astype(np.float32))
    got = _adapter(sv, a, 1024, aux, heads=1)
    H1 = oracle_pool.down_proj_full(a.X, a.Wd)
    ref = oracle.xattn_aux(H1, np.array([0, a.n], np.int32), aux[None])[0]
    check(got, ref, aux, "long video adapter+xattn")
