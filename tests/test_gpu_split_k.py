"""The split-K tail of the CTA-pair GEMM (lm_fp8_gemm_ex with a workspace):
the persistent grid's last wave of r tiles runs as S units per tile over
ranges of K whose fp32 sums meet in the workspace (lm_fp8_gemm_split_plan
gives S).  With 2r <= C (the number of CTA pairs) the tiles are halved in one
round; fuller tails may take three or more parts over several rounds.
Shapes below are built from C so that the tail is split; the split tiles'
rows are checked in full or on a sample of every (CTA, warp) row group
against the oracle, other rows on a sample."""
import numpy as np
import pytest
import torch

from gpu_util import ELEM_REL, ELEM_REL_RELU2_BWD, assert_close, assert_close_f32, from_u8, u8, u16

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1
EPI_NONE, EPI_RELU2_FWD, EPI_RELU2_BWD, EPI_ACCUM_F32 = 0, 1, 2, 3
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}
PAT, PRE, POST = 0xA5, 256, 4096


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_gemms_b200 import _lib
    return _lib


@pytest.fixture(scope="module")
def clusters():
    return torch.cuda.get_device_properties(0).multi_processor_count // 2


def codes(fmt, shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(TORCH_DT[fmt]).view(torch.uint8).numpy()


def tail_rows(M, C, extra):
    """With N <= 256 every tile is one 256-row block, visited in order, so the
    split tiles are the last `extra` row blocks; add a sample of the rest."""
    first = 256 * C
    rows = np.arange(first, M)
    rng = np.random.default_rng(3)
    return np.sort(np.concatenate([rows, rng.choice(first, 64, replace=False)]))


def run(lib, A, fa, B, fb, M, N, ia, ib, flags=0, epi=EPI_NONE, aux=None, ws=True, D=None):
    ws_t = (torch.empty(lib.lm_fp8_gemm_workspace_size(), dtype=torch.uint8, device="cuda")
            if ws else None)
    ia_t = torch.tensor([ia], dtype=torch.float32, device="cuda")
    ib_t = torch.tensor([ib], dtype=torch.float32, device="cuda")
    if D is None:
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(1, device="cuda")
    At = from_u8(np.ascontiguousarray(A.T) if flags & 1 else A)
    Bt = from_u8(np.ascontiguousarray(B.T) if flags & 2 else B)
    lib.lm_fp8_gemm_ex(At, fa, Bt, fb, ia_t, ib_t, D, flags=flags, epi=epi,
                       aux=None if aux is None else torch.from_numpy(aux.view(np.int16)).cuda(),
                       amax_out=None if epi == EPI_ACCUM_F32 else am, workspace=ws_t)
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    return D, am


@pytest.mark.parametrize("epi", [EPI_NONE, EPI_RELU2_FWD, EPI_RELU2_BWD])
@pytest.mark.parametrize("N,K,flags", [(256, 512, 0), (200, 384, 0), (256, 1024, 3), (160, 256, 2)])
def test_split_tail_against_oracle(lib, orc, clusters, epi, N, K, flags):
    """C + 5 row blocks: the last wave's 5 tiles split (K = 384: halves of one
    and two k-blocks; N = 200 / 160: a ragged column edge in every tile)."""
    M = 256 * (clusters + 5)
    A, B = codes(E4M3, (M, K), 1), codes(E4M3, (N, K), 2)
    aux = None
    if epi == EPI_RELU2_BWD:
        g = torch.Generator().manual_seed(4)
        aux = u16(torch.randn(M, N, generator=g).to(torch.bfloat16))
    D, am = run(lib, A, E4M3, B, E4M3, M, N, 0.02, 0.5, flags=flags, epi=epi, aux=aux)
    rows = tail_rows(M, clusters, 5)
    ref, _ = orc.gemm(A, E4M3, B, E4M3, np.float32(0.02), np.float32(0.5), epi=epi, aux=aux,
                      rows=rows)
    got = u16(D)
    assert_close(got[rows], ref, f"split tail epi={epi} N={N} K={K} flags={flags}",
                 ELEM_REL_RELU2_BWD if epi == EPI_RELU2_BWD else ELEM_REL)
    # the epilogue's amax covers the final values only (not a half's partial sums)
    assert float(am.item()) == float(orc.amax(got, relu2_input=(epi == EPI_RELU2_FWD)))


def test_split_tail_accumulating_epilogue(lib, orc, clusters):
    M, N, K = 256 * (clusters + 3), 256, 512
    A, B = codes(E5M2, (M, K), 5), codes(E4M3, (N, K), 6)
    D0 = np.random.default_rng(7).standard_normal((M, N)).astype(np.float32) * 1e-3
    D = torch.from_numpy(D0.copy()).cuda()
    run(lib, A, E5M2, B, E4M3, M, N, 1e-4, 0.05, flags=3, epi=EPI_ACCUM_F32, D=D)
    rows = tail_rows(M, clusters, 3)
    ref = D0[rows].copy()
    orc.gemm_accum_f32(A[rows], E5M2, B, E4M3, np.float32(1e-4), np.float32(0.05), ref)
    assert_close_f32(D.cpu().numpy()[rows], ref, "split tail accumulate")


@pytest.mark.parametrize("M,N,K", [(512, 1024, 256), (256, 512, 2048), (300, 264, 640)])
def test_every_tile_split_when_the_grid_is_large(lib, orc, M, N, K):
    """Fewer tiles than half the CTA pairs: every tile becomes two half-K units."""
    A, B = codes(E4M3, (M, K), 8), codes(E4M3, (N, K), 9)
    D, _ = run(lib, A, E4M3, B, E4M3, M, N, 0.02, 0.5)
    ref, _ = orc.gemm(A, E4M3, B, E4M3, np.float32(0.02), np.float32(0.5))
    assert_close(u16(D), ref, f"all split M={M} N={N} K={K}", ELEM_REL)


def test_single_k_block_is_not_split(lib, orc):
    M, N, K = 512, 512, 128
    A, B = codes(E4M3, (M, K), 10), codes(E4M3, (N, K), 11)
    D, _ = run(lib, A, E4M3, B, E4M3, M, N, 0.02, 0.5)
    Dn, _ = run(lib, A, E4M3, B, E4M3, M, N, 0.02, 0.5, ws=False)
    assert torch.equal(D.view(torch.int16), Dn.view(torch.int16))


def test_split_is_deterministic_and_close_to_unsplit(lib, clusters):
    M, N, K = 256 * (clusters + 7), 256, 1536
    A, B = codes(E4M3, (M, K), 12), codes(E4M3, (N, K), 13)
    D1, a1 = run(lib, A, E4M3, B, E4M3, M, N, 0.02, 0.5, epi=EPI_RELU2_FWD)
    D2, a2 = run(lib, A, E4M3, B, E4M3, M, N, 0.02, 0.5, epi=EPI_RELU2_FWD)
    Dn, _ = run(lib, A, E4M3, B, E4M3, M, N, 0.02, 0.5, epi=EPI_RELU2_FWD, ws=False)
    assert torch.equal(D1.view(torch.int16), D2.view(torch.int16)) and torch.equal(a1, a2)
    # the unsplit tiles are the same bits; the split ones differ by fp32 summation order only
    head = 256 * clusters
    assert torch.equal(D1[:head].view(torch.int16), Dn[:head].view(torch.int16))
    g, r = D1[head:].float(), Dn[head:].float()
    assert float((g - r).abs().max()) <= 2.0 ** -7 * float(r.abs().max())


def test_split_writes_stay_inside_output_and_workspace(lib, clusters):
    from fp8_gemms_b200 import _lib
    M, N, K = 256 * (clusters + 5), 200, 512
    n_ws = _lib.lm_fp8_gemm_workspace_size()
    wbuf = torch.full((PRE + n_ws + POST,), PAT, dtype=torch.uint8, device="cuda")
    ws = wbuf[PRE:PRE + n_ws]
    nbytes = M * N * 2
    dbuf = torch.full((PRE + nbytes + POST,), PAT, dtype=torch.uint8, device="cuda")
    D = dbuf[PRE:PRE + nbytes].view(torch.bfloat16).view(M, N)
    g = torch.Generator(device="cuda").manual_seed(14)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.float8_e4m3fn).view(torch.uint8)
    B = torch.randn(N, K, device="cuda", generator=g).to(torch.float8_e4m3fn).view(torch.uint8)
    one = torch.full((1,), 0.01, device="cuda")
    _lib.lm_fp8_gemm_ex(A, 0, B, 0, one, one, D, workspace=ws)
    torch.cuda.synchronize()
    assert _lib.lm_get_error()[0] == 0
    for buf, n in [(wbuf, n_ws), (dbuf, nbytes)]:
        assert bool((buf[:PRE] == PAT).all()) and bool((buf[PRE + n:] == PAT).all())


def plan(lib, M, N, K):
    return lib.lm_fp8_gemm_split_plan(M, N, K, torch.cuda.get_device_properties(0).multi_processor_count)


def dev_codes(fmt, shape, seed):
    """FP8 codes drawn on the device (the deep-K operands below are too large to
    draw on the host); the oracle receives the rows it checks."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(*shape, device="cuda", generator=g).to(TORCH_DT[fmt]).view(torch.uint8)


def run_dev(lib, A, fa, B, fb, ia, ib, flags=0, epi=EPI_NONE, aux=None, D=None, ws=True):
    M, N = A.shape[0], B.shape[0]
    ws_t = (torch.empty(lib.lm_fp8_gemm_workspace_size(), dtype=torch.uint8, device="cuda")
            if ws else None)
    if D is None:
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(1, device="cuda")
    At = A.t().contiguous() if flags & 1 else A
    Bt = B.t().contiguous() if flags & 2 else B
    lib.lm_fp8_gemm_ex(At, fa, Bt, fb, torch.tensor([ia], device="cuda"),
                       torch.tensor([ib], device="cuda"), D, flags=flags, epi=epi, aux=aux,
                       amax_out=None if epi == EPI_ACCUM_F32 else am, workspace=ws_t)
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    return D, am


def rows_per_group(first_tile, last_tile, seed, extra=64):
    """One row of each of the 8 (CTA, TMEM lane quarter) groups of 32 rows in
    every 256-row tile from first_tile to last_tile, plus a sample of the rest."""
    r = np.random.default_rng(seed)
    rows = [t * 256 + g * 32 + r.integers(0, 32, 1) for t in range(first_tile, last_tile)
            for g in range(8)]
    rows = np.concatenate(rows)
    if extra and first_tile > 0:
        rows = np.concatenate([rows, r.choice(first_tile * 256, extra, replace=False)])
    return np.unique(rows)


# 44 tiles on 74 CTA pairs (more than half): three parts per tile, 24 tiles per
# round, two rounds, when K is deep enough to pay for reading two partials
THREE_PART = dict(tiles=44, K=32768)


@pytest.mark.parametrize("epi,flags,N,K", [(EPI_NONE, 3, 256, 32768),
                                           (EPI_RELU2_FWD, 0, 200, 32768 - 64),
                                           (EPI_RELU2_BWD, 2, 256, 32768)])
def test_three_part_tail_over_two_rounds(lib, orc, clusters, epi, flags, N, K):
    """Every tile runs as three parts (the last part reading the others' sums
    from global memory), with idle pairs in each round; K = 32704 leaves the
    last k-block partial and N = 200 a ragged column edge."""
    M = 256 * THREE_PART["tiles"]
    S, rem = plan(lib, M, N, K)
    assert S == 3 and rem == THREE_PART["tiles"], (S, rem)
    A, B = dev_codes(E4M3, (M, K), 21), dev_codes(E4M3, (N, K), 22)
    aux = None
    if epi == EPI_RELU2_BWD:
        g = torch.Generator(device="cuda").manual_seed(23)
        aux = torch.randn(M, N, device="cuda", generator=g).to(torch.bfloat16)
    D, am = run_dev(lib, A, E4M3, B, E4M3, 0.02, 0.5, flags=flags, epi=epi, aux=aux)
    rows = rows_per_group(0, THREE_PART["tiles"], 24)
    ref, _ = orc.gemm(u8(A[rows]), E4M3, u8(B), E4M3, np.float32(0.02), np.float32(0.5), epi=epi,
                      aux=None if aux is None else u16(aux)[rows])
    got = u16(D)
    assert_close(got[rows], ref, f"3-part tail epi={epi} N={N} K={K} flags={flags}",
                 ELEM_REL_RELU2_BWD if epi == EPI_RELU2_BWD else ELEM_REL)
    assert float(am.item()) == float(orc.amax(got, relu2_input=(epi == EPI_RELU2_FWD)))


def test_five_part_tail_in_one_round(lib, orc, clusters):
    """The LM head's dgrad shape class: a 14-tile tail on K = 50304, five
    parts per tile in one round, of uneven length (393 k-blocks: 78 or 79)."""
    M, N, K = 256 * (clusters + 14), 256, 50304
    S, rem = plan(lib, M, N, K)
    assert S == 5 and rem == 14, (S, rem)
    A, B = dev_codes(E4M3, (M, K), 25), dev_codes(E4M3, (N, K), 26)
    D, am = run_dev(lib, A, E4M3, B, E4M3, 0.02, 0.5, flags=1)
    rows = rows_per_group(clusters, clusters + 14, 27)
    ref, _ = orc.gemm(u8(A[rows]), E4M3, u8(B), E4M3, np.float32(0.02), np.float32(0.5))
    got = u16(D)
    assert_close(got[rows], ref, "5-part tail", ELEM_REL)
    assert float(am.item()) == float(orc.amax(got))


def test_three_part_tail_accumulating(lib, orc, clusters):
    """The wgrad of a gradient-accumulation step: fp32 D += A B^T s, each
    element added once although its tile ran as three parts."""
    M, N, K = 256 * THREE_PART["tiles"], 256, THREE_PART["K"]
    assert plan(lib, M, N, K)[0] == 3
    A, B = dev_codes(E5M2, (M, K), 28), dev_codes(E4M3, (N, K), 29)
    D0 = np.random.default_rng(30).standard_normal((M, N)).astype(np.float32) * 1e-3
    D = torch.from_numpy(D0.copy()).cuda()
    run_dev(lib, A, E5M2, B, E4M3, 1e-4, 0.05, flags=3, epi=EPI_ACCUM_F32, D=D)
    rows = rows_per_group(0, THREE_PART["tiles"], 31)
    ref = D0[rows].copy()
    orc.gemm_accum_f32(u8(A[rows]), E5M2, u8(B), E4M3, np.float32(1e-4), np.float32(0.05), ref)
    assert_close_f32(D.cpu().numpy()[rows], ref, "3-part tail accumulate")


def test_multi_part_tails_are_deterministic_and_close_to_unsplit(lib, clusters):
    for M, K in [(256 * THREE_PART["tiles"], THREE_PART["K"]), (256 * (clusters + 14), 50304)]:
        N = 256
        assert plan(lib, M, N, K)[0] >= 3
        A, B = dev_codes(E4M3, (M, K), 32), dev_codes(E4M3, (N, K), 33)
        D1, a1 = run_dev(lib, A, E4M3, B, E4M3, 0.02, 0.5)
        D2, a2 = run_dev(lib, A, E4M3, B, E4M3, 0.02, 0.5)
        Dn, _ = run_dev(lib, A, E4M3, B, E4M3, 0.02, 0.5, ws=False)
        assert torch.equal(D1.view(torch.int16), D2.view(torch.int16)) and torch.equal(a1, a2)
        g, r = D1.float(), Dn.float()
        assert float((g - r).abs().max()) <= 2.0 ** -7 * float(r.abs().max())


def test_multi_part_writes_stay_inside_output_and_workspace(lib, clusters):
    M, N, K = 256 * THREE_PART["tiles"], 200, THREE_PART["K"]
    assert plan(lib, M, N, K)[0] == 3
    n_ws = lib.lm_fp8_gemm_workspace_size()
    wbuf = torch.full((PRE + n_ws + POST,), PAT, dtype=torch.uint8, device="cuda")
    ws = wbuf[PRE:PRE + n_ws]
    nbytes = M * N * 2
    dbuf = torch.full((PRE + nbytes + POST,), PAT, dtype=torch.uint8, device="cuda")
    D = dbuf[PRE:PRE + nbytes].view(torch.bfloat16).view(M, N)
    A, B = dev_codes(E4M3, (M, K), 34), dev_codes(E4M3, (N, K), 35)
    one = torch.full((1,), 0.01, device="cuda")
    lib.lm_fp8_gemm_ex(A, 0, B, 0, one, one, D, workspace=ws)
    torch.cuda.synchronize()
    assert lib.lm_get_error()[0] == 0
    for buf, n in [(wbuf, n_ws), (dbuf, nbytes)]:
        assert bool((buf[:PRE] == PAT).all()) and bool((buf[PRE + n:] == PAT).all())
