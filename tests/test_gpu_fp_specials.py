"""Floating-point special values through the combine and its relatives, on the GPU.

The expert outputs a combine reads (Zyphra, English abstract: the dispatched tokens'
results are combined) and the rows the backward and the token shuffle add can hold any
bf16 value; the gates any fp32 value.  Every kernel that does arithmetic on rows is fed
rows drawn from the whole bf16 bit space -- +-0, subnormals, +-inf, NaNs with any
payload, values near the bf16 maximum whose fp32 sum overflows or rounds to a bf16
infinity -- and gates that are negative, zero, -0, above 1, subnormal, huge, infinite or
NaN.  The oracle runs the same fixed-order fp32 chains.

What must match (IEEE 754 leaves the payload and sign of a NaN result open, and the
pages fix no precision): every non-NaN output bit for bit; a NaN exactly where the
oracle has a NaN, whatever its payload or sign.  Where the chain and the float64
reference are both finite, the stated tolerance of the ordinary tests holds as well.
For the gate gradients (a dot product whose summation order is the kernel's) the rows
avoid finite overflow, so that NaN and infinity do not depend on the order: class
(NaN, +inf, -inf, finite) must match, finite values within the stated bound."""
import math

import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import DEV, cuda, host_bits, ulp_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def special_rows(n, H, seed, huge=True):
    """bf16 bit patterns [n, H]: a mix of rows of uniformly random bits (every class of
    value), ordinary N(0,1)-like values, values near the bf16 maximum, subnormals, and
    rows sprinkled with +-0, +-inf and NaNs of several payloads.  huge=False keeps every
    magnitude below 2^20 (no finite overflow anywhere)."""
    rng = np.random.default_rng(seed)
    kind = rng.integers(0, 5, n)
    out = np.empty((n, H), np.uint16)
    rand_bits = rng.integers(0, 1 << 16, (n, H), dtype=np.uint32).astype(np.uint16)
    ordinary = host_bits(workload.fill_bf16(n, H, seed, 9))
    sign = (rng.integers(0, 2, (n, H)) << 15).astype(np.uint16)
    near_max = sign | (0xFE << 7) | rng.integers(0, 128, (n, H)).astype(np.uint16)
    subn = sign | rng.integers(0, 128, (n, H)).astype(np.uint16)
    out[:] = ordinary
    out[kind == 0] = rand_bits[kind == 0]
    out[kind == 1] = near_max[kind == 1]
    out[kind == 2] = subn[kind == 2]
    specials = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFC0, 0x7F81, 0x7FFF,
                         0xFFA5, 0x0001, 0x8001, 0x7F7F, 0xFF7F], np.uint16)
    sprinkle = rng.random((n, H)) < 0.03
    out[sprinkle] = specials[rng.integers(0, len(specials), sprinkle.sum())]
    if not huge:
        f = workload.bf16_bits_to_float(out)
        big = np.isfinite(f) & (np.abs(f) >= 2.0 ** 20)
        out[big] = ordinary[big]
    return out


def mostly_ordinary(rows, seed, frac=0.2):
    """rows with all but a `frac` share of them replaced by ordinary N(0,1)-like values."""
    n, H = rows.shape
    keep = np.random.default_rng(seed + 7).random(n) < frac
    out = host_bits(workload.fill_bf16(n, H, seed, 10))
    out[keep] = rows[keep]
    return out


def special_gates(N, k, seed, huge=True):
    rng = np.random.default_rng(seed + 1000)
    g = rng.random((N, k)).astype(np.float32)
    pool = [-0.7, 0.0, -0.0, 1.0, 3.5, 1e4, -2.25, 1e-40, 1.4e-45, np.inf, -np.inf, np.nan]
    if huge:
        pool += [1e30, 3e38]
    pool = np.array(pool, np.float32)
    pick = rng.random((N, k)) < 0.35
    g[pick] = pool[rng.integers(0, len(pool), pick.sum())]
    return g


def to_dev_bits(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).to(DEV).view(torch.bfloat16)


def assert_bits_nan_as_nan(got, want, what):
    """Bit-exact, except that a NaN must meet a NaN (any payload or sign)."""
    if got.dtype == np.uint16:
        gv, wv = workload.bf16_bits_to_float(got), workload.bf16_bits_to_float(want)
    else:
        gv, wv = got.view(np.float32), want.view(np.float32)
        got, want = got.view(np.uint32), want.view(np.uint32)
    gn, wn = np.isnan(gv), np.isnan(wv)
    bad = np.nonzero(gn != wn)
    assert bad[0].size == 0, f"{what}: NaN at {bad[0][:4]},{bad[1][:4] if len(bad) > 1 else ''}"
    diff = np.nonzero((got != want) & ~wn)
    assert diff[0].size == 0, (f"{what}: {diff[0].size} non-NaN outputs differ, first "
                               f"got {got[diff][:4]} want {want[diff][:4]}")


def check_tolerance_where_finite(got_f, chain, ref64, mag, bf16):
    ok = (np.isfinite(chain) & np.isfinite(ref64) & np.isfinite(mag)
          & (np.abs(ref64) < 2.0 ** 127) & np.isfinite(got_f))
    with np.errstate(invalid="ignore", over="ignore"):
        d = np.abs(got_f.astype(np.float64) - ref64)
    tol = 1e-5 * mag + (ulp_bf16(ref64) if bf16 else 1e-30)
    assert (d[ok] <= tol[ok]).all()
    return int(ok.sum())


@pytest.mark.parametrize("k,H", [(1, 264), (3, 264), (8, 264), (2, 7168), (6, 1000)])
def test_combine_special_values(coact, k, H):
    N = 1031
    y = special_rows(N * k, H, 100 * k + H)
    g = special_gates(N, k, 7 * k + H)
    comb = np.random.default_rng(k).permutation(N * k).reshape(N, k).astype(np.int32)
    comb[5, 0] = -1                                    # an absent slot
    chain = oracle.combine_f32chain(y, g, comb)
    ref64 = oracle.combine_f64(y, g, comb)
    with np.errstate(invalid="ignore", over="ignore"):
        yf = workload.bf16_bits_to_float(y).astype(np.float64)
        mag = np.zeros((N, H))
        for j in range(k):
            v = comb[:, j] >= 0
            mag[v] += np.abs(g[v, j, None].astype(np.float64) * yf[comb[v, j]])
    yd = to_dev_bits(y)
    for dt in (torch.float32, torch.bfloat16):
        out = torch.empty((N, H), dtype=dt, device=DEV)
        coact.combine_scatter(yd, cuda(g), cuda(comb), out)
        torch.cuda.synchronize()
        if dt == torch.float32:
            got = out.cpu().numpy()
            assert_bits_nan_as_nan(got, chain, "combine fp32")
            n_ok = check_tolerance_where_finite(got, chain, ref64, mag, False)
        else:
            got = host_bits(out)
            want = oracle.bf16_rne(chain)
            assert_bits_nan_as_nan(got, want, "combine bf16")
            n_ok = check_tolerance_where_finite(workload.bf16_bits_to_float(got), chain, ref64,
                                                mag, True)
        # the ordinary part was checked too (with k = 8, about a quarter of the elements
        # have only finite terms and a finite sum)
        assert n_ok > N * H // 8
    assert np.isnan(chain).any() and np.isinf(chain).any()    # the specials were exercised


def test_combine_rounds_finite_sum_to_bf16_infinity(coact):
    """Sums that are finite in fp32 but above the largest bf16 value B = 2^127 + 127 * 2^120
    round to nearest-even: above the midpoint B + 2^119 to infinity, below it to B, and
    the tie itself to infinity (B's last mantissa bit is odd)."""
    H = 16
    B = 0x7F7F
    pairs = [(B, 0x7B40), (B, 0x7A80), (B, 0x7B00)]    # + 1.5*2^119, + 2^118, + 2^119
    y = np.repeat(np.array(pairs, np.uint16).reshape(-1, 1), H, axis=1)
    g = np.ones((3, 2), np.float32)
    comb = np.arange(6, dtype=np.int32).reshape(3, 2)
    chain = oracle.combine_f32chain(y, g, comb)
    assert np.isfinite(chain).all()
    want = oracle.bf16_rne(chain)
    assert (want[0] == 0x7F80).all() and (want[1] == B).all() and (want[2] == 0x7F80).all()
    out = torch.empty((3, H), dtype=torch.bfloat16, device=DEV)
    coact.combine_scatter(to_dev_bits(y), cuda(g), cuda(comb), out)
    assert np.array_equal(host_bits(out), want)


@pytest.mark.parametrize("k", [2, 6])
def test_combine_rows_and_gather_backward_special_values(coact, k):
    """The pre-reduced reverse path (partial rows per send row, then the transposed
    dispatch's fp32 add chain) on special values."""
    r = workload.make_routing(2 if k == 6 else 1, N=2053)
    c = r.cfg
    H = 264
    p = oracle.plan(r.ids, c.E, r.expert_rank, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    plan = coact.alloc_plan(r.N, r.k, c.E, c.R, DEV)
    coact.plan_dispatch(cuda(r.ids), c.E, cuda(r.expert_rank, np.int32), c.R, plan,
                        rank_node=cuda(r.rank_node, np.int32), n_nodes=c.n_nodes)
    D = p["D"]
    y = special_rows(r.N * r.k, H, 31 + k)
    g = special_gates(r.N, r.k, 17 + k)
    pre = torch.empty((D, H), dtype=torch.bfloat16, device=DEV)
    coact.combine_rows(to_dev_bits(y), cuda(g), plan.comb_row, plan.row_token, plan.row_kmask, pre)
    pre_o, out_o = oracle.combine_prereduced(y, g, p)
    torch.cuda.synchronize()
    assert_bits_nan_as_nan(host_bits(pre), pre_o, "combine_rows")
    # the transposed dispatch over rows of special values (its own input, not pre)
    gs = special_rows(D, H, 55 + k)
    gx = torch.empty((r.N, H), dtype=torch.float32, device=DEV)
    coact.dispatch_gather_backward(to_dev_bits(gs), plan.send_row, gx)
    want = oracle.gather_backward_f32chain(gs, p["send_row"])
    torch.cuda.synchronize()
    assert_bits_nan_as_nan(gx.cpu().numpy(), want, "dispatch_gather_backward fp32")
    gxb = torch.empty((r.N, H), dtype=torch.bfloat16, device=DEV)
    coact.dispatch_gather_backward(to_dev_bits(gs), plan.send_row, gxb)
    assert_bits_nan_as_nan(host_bits(gxb), oracle.bf16_rne(want), "dispatch_gather_backward bf16")
    assert np.isnan(want).any() and np.isinf(want).any()


@pytest.mark.parametrize("P", [3, 16])
def test_shuffle_reduce_special_values(coact, P):
    N, H = 777, 264
    parts = np.stack([special_rows(N, H, 300 + q) for q in range(P)])
    home = np.random.default_rng(P).integers(0, 8, N).astype(np.int32)
    order = oracle.shuffle_order(home, 8)
    rt = order["row_token"][:N]
    dev_parts = [to_dev_bits(parts[q]) for q in range(P)]
    bases = torch.tensor([t.data_ptr() for t in dev_parts], dtype=torch.int64, device=DEV)
    want = oracle.shuffle_reduce_f32chain(parts, rt)
    for dt in (torch.float32, torch.bfloat16):
        out = torch.empty((N, H), dtype=dt, device=DEV)
        coact.shuffle_reduce_scatter(bases, N, cuda(rt), out)
        torch.cuda.synchronize()
        if dt == torch.float32:
            assert_bits_nan_as_nan(out.cpu().numpy(), want, "shuffle fp32")
        else:
            assert_bits_nan_as_nan(host_bits(out), oracle.bf16_rne(want), "shuffle bf16")
    assert np.isnan(want).any() and np.isinf(want).any()


@pytest.mark.parametrize("k,H", [(2, 264), (8, 1000)])
def test_combine_backward_special_values(coact, k, H):
    """grad_y = bf16(gate * grad_out) bit for bit (NaN as NaN); grad_gates by class and,
    where finite, within the dot product's bound.  No finite overflow in the rows, so
    the class of a dot product does not depend on its summation order."""
    N = 517
    # special values in a fifth of the rows only, so that many dot products stay finite
    y = mostly_ordinary(special_rows(N * k, H, 11 * k + H, huge=False), 11 * k + H)
    go = mostly_ordinary(special_rows(N, H, 13 * k + H, huge=False), 13 * k + H)
    g = special_gates(N, k, 19 * k + H, huge=False)
    comb = np.random.default_rng(H).permutation(N * k).reshape(N, k).astype(np.int32)
    gy = torch.zeros((N * k, H), dtype=torch.bfloat16, device=DEV)
    gg = torch.empty((N, k), dtype=torch.float32, device=DEV)
    coact.combine_scatter_backward(to_dev_bits(y), cuda(g), cuda(comb), to_dev_bits(go), gy, gg)
    gy_o, gg_o, ga_o = oracle.combine_backward(y, g, comb, go)
    torch.cuda.synchronize()
    assert_bits_nan_as_nan(host_bits(gy), gy_o, "grad_y")
    got = gg.cpu().numpy().astype(np.float64)
    for name, cls in (("NaN", np.isnan), ("+inf", lambda a: np.isposinf(a)),
                      ("-inf", lambda a: np.isneginf(a))):
        assert np.array_equal(cls(got), cls(gg_o)), f"grad_gates {name}"
    fin = np.isfinite(gg_o)
    m = max(8 * math.ceil(H / 256), 16 * math.ceil(H / 512))
    bound = 1.01 * (m + 5) * 2.0 ** -24 * ga_o + 1e-30
    assert (np.abs(got[fin] - gg_o[fin]) <= bound[fin]).all()
    assert np.isnan(gg_o).any() and fin.sum() > N * k // 4


def test_device_nan_results_are_canonical(coact):
    """What the device emits for a NaN result, pinned: whatever the NaN's payload or sign in
    the inputs (signalling, quiet, negative), the fused multiply-adds give the canonical
    quiet NaN (fp32 0x7FFFFFFF) and its round to bf16 gives 0x7FFF.  The oracle keeps an
    input's payload instead (C library semantics); the contract compares NaN as NaN."""
    H = 64
    nans = np.array([0x7FC0, 0xFFC0, 0x7F81, 0xFF81, 0x7FFF, 0xFFA5, 0x7FAA], np.uint16)
    rows = np.repeat(nans.reshape(-1, 1), H, axis=1)
    k1 = len(nans)
    # k = 1: each token's only row is a NaN row; k = 2: a NaN row after an ordinary one, and
    # 0 * inf (an invalid operation from non-NaN inputs)
    ordinary = host_bits(workload.fill_bf16(k1, H, 0, 11))
    y1 = rows
    y2 = np.concatenate([ordinary, rows, np.full((1, H), 0x7F80, np.uint16)])
    comb2 = np.stack([np.arange(k1), k1 + np.arange(k1)], 1).astype(np.int32)
    comb2 = np.concatenate([comb2, [[0, 2 * k1]]]).astype(np.int32)
    g2 = np.ones(comb2.shape, np.float32)
    g2[-1, 1] = 0.0
    for y, comb, g in ((y1, np.arange(k1, dtype=np.int32).reshape(-1, 1),
                        np.full((k1, 1), 0.5, np.float32)), (y2, comb2, g2)):
        f32 = torch.empty((comb.shape[0], H), dtype=torch.float32, device=DEV)
        b16 = torch.empty((comb.shape[0], H), dtype=torch.bfloat16, device=DEV)
        coact.combine_scatter(to_dev_bits(y), cuda(g), cuda(comb), f32)
        coact.combine_scatter(to_dev_bits(y), cuda(g), cuda(comb), b16)
        torch.cuda.synchronize()
        got32 = f32.cpu().numpy().view(np.uint32)
        got16 = host_bits(b16)
        assert np.isnan(oracle.combine_f32chain(y, g, comb)).all()
        assert (got32 == 0x7FFFFFFF).all(), sorted({hex(v) for v in got32.ravel()})
        assert (got16 == 0x7FFF).all(), sorted({hex(v) for v in got16.ravel()})
