"""GPU parity of token shuffling fused into the post-attention reduce-scatter, through the
C ABI, against the CPU oracle: the permutation (plan of every token to its predicted home
rank) bit-exact, and the reduced rows bit-exact with the oracle's rank-order fp32 chain
(fp32 out) and its round-to-nearest-even (bf16 out).  P partial outputs live in P local
buffers addressed through the same base-pointer table that peers' buffers use on a GPU
group."""
import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import (DEV, assert_plan_equal, cuda, for_chunks, host_bits, plan_to_host,
                       rows_of)

pytestmark = pytest.mark.gpu

PART_STREAM = 100            # partial q: fill_bf16 stream PART_STREAM + q


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def zero_flag():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def partials(P, N, H, seed):
    return [workload.fill_bf16(N, H, seed, PART_STREAM + q, device=DEV) for q in range(P)]


def bases_of(parts):
    return torch.tensor([p.data_ptr() for p in parts], dtype=torch.int64, device=DEV)


def check_rows(out, parts_bits, row_token_local, rows=None):
    chain = oracle.shuffle_reduce_f32chain(parts_bits, row_token_local)
    got = out if rows is None else out[torch.as_tensor(rows, device=DEV)]
    if got.dtype == torch.float32:
        assert np.array_equal(got.cpu().numpy().view(np.uint32), chain.view(np.uint32))
    else:
        assert np.array_equal(host_bits(got), oracle.bf16_rne(chain))


def test_config4_full_size(coact):
    """Config 4 (N = 65536, H = 4096, R = 16): homes predicted by the library from the
    calibration counts, the shuffle plan, and the reduce-scatter over 16 partials, every
    row checked."""
    tl = workload.make_two_layer(workload.CONFIGS[4])
    c = tl.layer1.cfg
    N, H, R, E = c.N, c.H, c.R, c.E
    C12 = torch.zeros((E, E), dtype=torch.int64, device=DEV)
    coact.coact_count(cuda(tl.calib1), E, C12, ids2=cuda(tl.calib2), E2=E)
    home = torch.empty(N, dtype=torch.int32, device=DEV)
    coact.predict_home(cuda(tl.layer1.ids), E, C12, cuda(tl.layer2.expert_rank, np.int32), R, home)
    sp = coact.shuffle_plan(home, R)
    torch.cuda.synchronize()
    o = oracle.shuffle_order(home.cpu().numpy(), R)
    g = plan_to_host(sp)
    for key in ("rank_counts", "rank_offsets", "send_row"):
        assert np.array_equal(g[key], o[key]), key
    assert np.array_equal(g["row_token"][:N], o["row_token"][:N])
    parts = partials(R, N, H, 0)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    err = zero_flag()
    coact.shuffle_reduce_scatter(bases_of(parts), N, sp.row_token, out, err_flag=err)
    # each rank's own segment, as a rank computes it on a GPU group
    offs = o["rank_offsets"]
    segs = []
    for r in (0, 7, R - 1):
        seg = torch.empty((int(offs[r + 1] - offs[r]), H), dtype=torch.bfloat16, device=DEV)
        coact.shuffle_reduce_scatter(bases_of(parts), N, sp.row_token[int(offs[r]):], seg, err_flag=err)
        segs.append((r, seg))
    torch.cuda.synchronize()
    assert err.item() == 0
    for r, seg in segs:
        assert torch.equal(seg.view(torch.int16), out[int(offs[r]):int(offs[r + 1])].view(torch.int16))
    # every shuffled row: the 16 partials' rows of the oracle's token order, in chunks
    def prepare(i0, i1):
        toks = o["row_token"][i0:i1]
        pb = np.stack([rows_of(p, toks) for p in parts])
        got = host_bits(out[i0:i1])

        def job():
            chain = oracle.shuffle_reduce_f32chain(pb, np.arange(i1 - i0, dtype=np.int32))
            np.testing.assert_array_equal(got, oracle.bf16_rne(chain), err_msg=f"rows [{i0}, {i1})")
        return job

    for_chunks(N, 1024, prepare, workers=4)


@pytest.mark.parametrize("P,H", [(1, 8), (3, 1000), (16, 256), (64, 64), (5, 2056)])
def test_shapes(coact, P, H):
    rng = np.random.default_rng(P * 31 + H)
    N = 777
    R = max(P, 2)
    home = rng.integers(0, R, N).astype(np.int32)
    sp = coact.shuffle_plan(cuda(home), R)
    parts = partials(P, N, H, P)
    pb = np.stack([host_bits(p) for p in parts])
    o = oracle.shuffle_order(home, R)
    for dt in (torch.bfloat16, torch.float32):
        out = torch.empty((N, H), dtype=dt, device=DEV)
        coact.shuffle_reduce_scatter(bases_of(parts), N, sp.row_token, out)
        torch.cuda.synchronize()
        check_rows(out, pb, o["row_token"][:N])


def test_flags_invalid_tokens_and_bases(coact):
    N, H, P = 64, 32, 4
    parts = partials(P, N, H, 9)
    pb = np.stack([host_bits(p) for p in parts])
    rt = np.arange(N, dtype=np.int32)[::-1].copy()
    rt[5] = N + 3                               # outside [0, N): zero row, flagged
    rt[9] = -1
    out = torch.empty((N, H), dtype=torch.float32, device=DEV)
    err = zero_flag()
    coact.shuffle_reduce_scatter(bases_of(parts), N, cuda(rt), out, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == coact.EFLAG_ROW_RANGE
    assert (out[5] == 0).all() and (out[9] == 0).all()
    ok = np.array([i for i in range(N) if i not in (5, 9)])
    check_rows(out, pb, rt[ok], rows=ok)
    # a NULL and a misaligned partial base are skipped (never dereferenced) and flagged
    b = bases_of(parts)
    b[1] = 0
    b[2] = parts[2].data_ptr() + 2
    err.zero_()
    coact.shuffle_reduce_scatter(b, N, cuda(np.arange(N, dtype=np.int32)), out, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == coact.EFLAG_ROW_RANGE
    check_rows(out, pb[[0, 3]], np.arange(N, dtype=np.int32))


def test_rank_order_of_the_sum(coact):
    """Partials 1, 2^24, -2^24 (and the reverse): in rank order the fp32 sum is 0 (1 + 2^24
    rounds back to 2^24), in reverse order it is 1 -- the kernel must add in rank order."""
    H = 8
    vals = [1.0, 2.0 ** 24, -(2.0 ** 24)]
    for order, want in ((vals, 0.0), (vals[::-1], 1.0)):
        parts = [torch.full((1, H), v, dtype=torch.bfloat16, device=DEV) for v in order]
        out = torch.empty((1, H), dtype=torch.float32, device=DEV)
        coact.shuffle_reduce_scatter(bases_of(parts), 1, cuda(np.zeros(1, np.int32)), out)
        torch.cuda.synchronize()
        assert (out == want).all(), (order, out)
