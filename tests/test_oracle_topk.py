"""Pins of the oracle's Top-K dynamic block mask (oracle_topk_mask), each
against something other than the oracle itself: the closed form when every
block is kept, inputs whose ranking is known by construction (constant key
blocks scored against an all-ones query), the tie rule, the mean over the real
tokens of a partial last block, and an fp64 numpy restatement of the ranking on
random data (rows without a near-tie at the cut)."""
import numpy as np
import pytest

import oracle
import salad_inputs as si


def bf16(x):
    return si.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def shape_inputs(B, N, Hh, d, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, Hh, d), dtype=np.float32)
    k = rng.standard_normal((B, N, Hh, d), dtype=np.float32)
    return q, k


def rows(rp, ci):
    return [ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)]


def test_keep_at_least_nb_keeps_every_block():
    q, k = shape_inputs(2, 300, 3, 16)
    nb = (300 + 63) // 64
    rp, ci = oracle.topk_mask(bf16(q), bf16(k), 64, nb + 3)
    assert np.array_equal(rp, np.arange(2 * 3 * nb + 1) * nb)
    assert all(r == list(range(nb)) for r in rows(rp, ci))


def test_ranking_by_construction():
    # q = 1 everywhere; key block J holds the constant v[J] on every token and
    # feature, so score(I, J) = d * v[J] for every row I (exact in fp32)
    B, Hh, d, blk, nb = 1, 2, 32, 16, 10
    N = nb * blk
    v = np.array([3, -1, 7, 0, 5, 2, -4, 6, 1, 4], dtype=np.float32)
    q = np.ones((B, N, Hh, d), np.float32)
    k = np.repeat(v, blk)[None, :, None, None] * np.ones((B, N, Hh, d), np.float32)
    for keep in (1, 3, 6):
        rp, ci = oracle.topk_mask(bf16(q), bf16(k), blk, keep)
        want = sorted(np.argsort(-v, kind="stable")[:keep].tolist())
        assert all(r == want for r in rows(rp, ci)), (keep, rows(rp, ci)[0], want)


def test_ties_keep_the_smaller_blocks():
    B, Hh, d, blk, nb = 1, 1, 8, 8, 9
    q = np.ones((B, nb * blk, Hh, d), np.float32)
    k = np.full_like(q, 0.5)
    rp, ci = oracle.topk_mask(bf16(q), bf16(k), blk, 4)
    assert all(r == [0, 1, 2, 3] for r in rows(rp, ci))


def test_partial_last_block_is_the_mean_of_its_real_tokens():
    # the last key block has 3 real tokens of value 2; the others hold 1.9.  With
    # the mean over real tokens the last block scores highest; averaged over the
    # padded block size (2 * 3 / 8) it would score lowest.
    B, Hh, d, blk = 1, 1, 4, 8
    N = 3 * blk + 3
    q = np.ones((B, N, Hh, d), np.float32)
    k = np.full((B, N, Hh, d), 1.9, np.float32)
    k[:, 3 * blk:] = 2.0
    rp, ci = oracle.topk_mask(bf16(q), bf16(k), blk, 1)
    assert all(r == [3] for r in rows(rp, ci))


@pytest.mark.parametrize("B,N,Hh,d,blk,keep", [(1, 1000, 2, 64, 64, 5), (2, 517, 3, 32, 32, 7),
                                              (1, 2048, 1, 128, 128, 4)])
def test_matches_an_fp64_ranking_away_from_ties(B, N, Hh, d, blk, keep):
    q, k = shape_inputs(B, N, Hh, d, seed=N)
    qb, kb = bf16(q), bf16(k)
    rp, ci = oracle.topk_mask(qb, kb, blk, keep)
    nb = (N + blk - 1) // blk
    qf = si.bf16_bits_to_f32(qb).astype(np.float64)
    kf = si.bf16_bits_to_f32(kb).astype(np.float64)
    got = rows(rp, ci)
    checked = 0
    for b in range(B):
        for h in range(Hh):
            qm = np.stack([qf[b, I * blk:min(N, (I + 1) * blk), h].mean(0) for I in range(nb)])
            km = np.stack([kf[b, J * blk:min(N, (J + 1) * blk), h].mean(0) for J in range(nb)])
            sc = qm @ km.T
            for I in range(nb):
                order = np.argsort(-sc[I], kind="stable")
                kk = min(keep, nb)
                if kk < nb and abs(sc[I, order[kk - 1]] - sc[I, order[kk]]) < 1e-4 * (1 + abs(sc[I, order[kk]])):
                    continue  # a near-tie at the cut: fp32 and fp64 may order it differently
                assert got[(b * Hh + h) * nb + I] == sorted(order[:kk].tolist())
                checked += 1
    assert checked >= 0.9 * B * Hh * nb


def test_rows_are_sorted_unique_and_of_fixed_length():
    q, k = shape_inputs(2, 777, 2, 16, seed=5)
    rp, ci = oracle.topk_mask(bf16(q), bf16(k), 32, 9)
    nb = (777 + 31) // 32
    assert np.array_equal(np.diff(rp), np.full(2 * 2 * nb, 9))
    for r in rows(rp, ci):
        assert r == sorted(set(r)) and 0 <= r[0] and r[-1] < nb


def test_forward_with_rows_per_batch_element_reads_the_right_rows():
    # a per-(b, h) mask whose rows repeat the per-head window mask for every b
    # gives the per-head result; a different mask for b = 1 changes only b = 1
    wl = si.Workload("t", B=2, Hh=2, d=16, T=2, H=4, W=8, block=16, window=(0, 1, 2), seed=3)
    inp = si.make_inputs(wl)
    rp, ci = oracle.block_mask(wl.T, wl.H, wl.W, wl.block, inp.windows)
    nb = wl.nb
    counts = np.diff(rp)
    rp2 = np.concatenate([[0], np.cumsum(np.concatenate([counts, counts]))]).astype(np.int32)
    ci2 = np.concatenate([ci, ci]).astype(np.int32)
    ref = oracle.forward(inp.q, inp.k, inp.v, wl.block, rp, ci, inp.w_proj, inp.gate)
    got = oracle.forward(inp.q, inp.k, inp.v, wl.block, rp2, ci2, inp.w_proj, inp.gate, mask_per_bh=True)
    assert np.array_equal(got, ref)
    full = np.tile(np.arange(nb, dtype=np.int32), 2 * wl.Hh * nb)
    rp3 = np.concatenate([rp2[:wl.Hh * nb + 1], rp2[wl.Hh * nb] + np.arange(1, wl.Hh * nb + 1) * nb]).astype(np.int32)
    ci3 = np.concatenate([ci, full[:wl.Hh * nb * nb]]).astype(np.int32)
    got3 = oracle.forward(inp.q, inp.k, inp.v, wl.block, rp3, ci3, inp.w_proj, inp.gate, mask_per_bh=True)
    assert np.array_equal(got3[0], ref[0]) and not np.allclose(got3[1], ref[1])
