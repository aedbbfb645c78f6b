"""Pins for the oracle's attention (no GPU).

Each pin is independent of the oracle's own code path: a library routine
(PyTorch SDPA and scipy logsumexp in float64), closed forms, brute-force loops,
and invariants that the pages fix (paged attention equals dense attention over
the same tokens; physical page ids do not matter).
"""
import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import PageModel, PoolImage, attention as A
from oracle.stream import StreamOracle, bits16
import workload


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("T,L,H,D", [(7, 13, 2, 64), (262, 300, 3, 64), (5, 1, 1, 128)])
def test_dense_matches_torch_sdpa_fp64(T, L, H, D):
    q, k, v = rnd((T, H, D), 1), rnd((L, H, D), 2), rnd((L, H, D), 3)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).permute(1, 0, 2), torch.from_numpy(k).permute(1, 0, 2),
        torch.from_numpy(v).permute(1, 0, 2)).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(A.dense(q, k, v), want, rtol=0, atol=1e-12)


def test_equal_keys_give_mean_of_values():
    q = rnd((9, 2, 64), 4)
    k = np.broadcast_to(rnd((1, 2, 64), 5), (40, 2, 64)).copy()
    v = rnd((40, 2, 64), 6)
    np.testing.assert_allclose(A.dense(q, k, v), np.broadcast_to(v.mean(0), (9, 2, 64)),
                               rtol=0, atol=1e-12)


def test_constant_values_pass_through():
    q, k = rnd((9, 2, 64), 7), rnd((33, 2, 64), 8)
    v = np.full((33, 2, 64), 0.3125)
    np.testing.assert_allclose(A.dense(q, k, v), 0.3125, rtol=0, atol=1e-14)


def test_single_visible_token_returns_its_value():
    q, k, v = rnd((9, 3, 64), 9), rnd((1, 3, 64), 10), rnd((1, 3, 64), 11)
    np.testing.assert_allclose(A.dense(q, k, v), np.broadcast_to(v[0], (9, 3, 64)),
                               rtol=0, atol=1e-14)


def test_dominant_key_selects_its_value():
    q = np.zeros((1, 1, 64)); q[0, 0, 0] = 1.0
    k = np.zeros((5, 1, 64)); k[3, 0, 0] = 400.0      # score 50 vs 0 for the rest
    v = rnd((5, 1, 64), 12)
    np.testing.assert_allclose(A.dense(q, k, v)[0, 0], v[3, 0], rtol=0, atol=1e-18)


def test_probability_rows_sum_to_one():
    p = A.probs(rnd((50, 4, 64), 13) * 3, rnd((500, 4, 64), 14) * 3)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (p >= 0).all()


def test_brute_force_loops_match_vectorised():
    q, k, v = rnd((4, 2, 8), 15), rnd((6, 2, 8), 16), rnd((6, 2, 8), 17)
    np.testing.assert_allclose(A.brute(q, k, v), A.dense(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("cuts", [[1], [128, 256], [3, 4, 5, 100], [299]])
def test_partials_merge_to_full_softmax(cuts):
    q, k, v = rnd((11, 2, 64), 18), rnd((300, 2, 64), 19), rnd((300, 2, 64), 20)
    edges = [0] + cuts + [300]
    parts = [A.partial(q, k[a:b], v[a:b]) for a, b in zip(edges[:-1], edges[1:])]
    np.testing.assert_allclose(A.merge(parts), A.dense(q, k, v), rtol=0, atol=1e-12)
    # each chunk's log-sum-exp agrees with scipy's
    s = np.einsum("thd,lhd->thl", q, k[edges[0]:edges[1]]) / 8.0
    np.testing.assert_allclose(parts[0][1], logsumexp(s, axis=-1), rtol=0, atol=1e-12)


def test_decode_matches_torch_conversions():
    raw = np.array([0x3F80, 0xC000, 0x0001, 0x7F7F, 0x8000, 0x3C00, 0x4049], dtype=np.uint16)
    t = torch.from_numpy(raw.view(np.int16))
    np.testing.assert_array_equal(A.decode(raw, "bf16"), t.view(torch.bfloat16).double().numpy())
    np.testing.assert_array_equal(A.decode(raw, "fp16"), t.view(torch.float16).double().numpy())
    assert A.decode(np.array([0x3F80], np.uint16), "bf16")[0] == 1.0
    assert A.decode(np.array([0x3C00], np.uint16), "fp16")[0] == 1.0


def _frames(wl, n, seed=1):
    return [tuple(bits16(x) for x in workload.frame_qkv(wl, seed, f, 0)) for f in range(n)]


def _paged_run(wl, frames, perm=None):
    """Append `frames` through the page model + pool image; optionally relabel
    the physical page ids by `perm` (moving the pool rows to match)."""
    m = PageModel(wl.S, wl.W, wl.page_size, wl.max_pages, NS=wl.NS)
    pool = PoolImage(m, wl.H, wl.D)
    for f, (_, k, v) in enumerate(frames):
        page, sp0 = m.append(f)
        m.evict()
        pool.write(page, sp0, k, v)
    table, last = m.page_table()
    bits = pool.bits
    if perm is not None:
        moved = np.empty_like(bits)
        moved[perm] = bits
        pool.bits = moved
        table = [int(perm[p]) for p in table]
    k, v = pool.gather(table, last)
    return A.decode(k, wl.dtype), A.decode(v, wl.dtype)


def test_paged_equals_dense_when_nothing_evicted():
    wl = workload.WORKLOADS[0]                       # S=2, W=4: 6 frames fit
    frames = _frames(wl, wl.S + wl.W)
    kp, vp = _paged_run(wl, frames)
    kd = np.concatenate([A.decode(k, wl.dtype) for _, k, _ in frames])
    vd = np.concatenate([A.decode(v, wl.dtype) for _, _, v in frames])
    assert kp.shape == kd.shape
    q = A.decode(frames[-1][0], wl.dtype)
    np.testing.assert_allclose(A.dense(q, kp, vp), A.dense(q, kd, vd), rtol=0, atol=1e-12)


def test_physical_page_relabelling_changes_nothing():
    wl = workload.WORKLOADS[0]
    frames = _frames(wl, 12)
    perm = np.random.default_rng(21).permutation(wl.max_pages)
    k0, v0 = _paged_run(wl, frames)
    k1, v1 = _paged_run(wl, frames, perm)
    np.testing.assert_array_equal(k0, k1)
    np.testing.assert_array_equal(v0, v1)


def test_stream_oracle_sees_the_page_models_tokens():
    """The stream oracle (frame lists, no pages) and the page model + pool image
    hold the same visible K/V rows after eviction has recycled pages."""
    wl = workload.WORKLOADS[0]
    frames = _frames(wl, 12)
    so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, lambda f: frames[f])
    for f in range(12):
        so.begin_frame(f)
    ks, vs = so.visible_kv()
    ks, vs = ks.astype(np.float64), vs.astype(np.float64)
    kp, vp = _paged_run(wl, frames)
    key = lambda k, v: sorted(map(bytes, np.concatenate([k, v], axis=-1).reshape(k.shape[0], -1)))
    assert key(ks, vs) == key(kp, vp)
    q = so.q
    np.testing.assert_allclose(so.expected(), A.dense(q, kp, vp), rtol=0, atol=1e-12)
