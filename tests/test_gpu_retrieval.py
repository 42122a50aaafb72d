"""GPU parity of full-catalog retrieval (hstu_retrieval_topk, through the C
ABI) against the oracle (oracle.retrieval) on the same seeded inputs.

* Integer-valued embeddings and user vectors (|values| <= 2, exact in bf16)
  make every score an integer below 2^24, exact in the GPU's fp32 and in the
  oracle's float64: ids (including the order of the many equal scores, which
  must be by ascending id) and scores are compared exactly.
* N(0,1) inputs: the GPU decides in fp32, the oracle in float64, so the check
  is validity within the fp32 accumulation bound tol_um = d * 2^-23 *
  sum_k |E_mk h_uk|: every returned score within tol of the exact score of
  its id, no item whose exact score beats the oracle's K-th by 2 tol missing,
  no returned item below the oracle's K-th by 2 tol, scores non-increasing.
"""
import numpy as np
import pytest

import hstu_workloads as hw
from oracle import retrieval as R

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def _bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


def _run(Hd, Ed, K, offsets=None, n_users=None):
    import torch
    import hstu_sequential_transducer_layer_b200 as H
    U = n_users if n_users is not None else (len(offsets) - 1 if offsets is not None else Hd.shape[0])
    M, d = Ed.shape
    ws = torch.empty(H.hstu_retrieval_workspace_size(U, M, d, K, offsets is not None),
                     dtype=torch.uint8, device="cuda")
    s = torch.full((U, K), float("nan"), dtype=torch.float32, device="cuda")
    i = torch.full((U, K), -1, dtype=torch.int64, device="cuda")
    off = None if offsets is None else torch.from_numpy(np.asarray(offsets, np.int64)).cuda()
    H.hstu_retrieval_topk(Hd, Ed, K, s, i, ws, user_offsets=off, n_users=U)
    st = H.hstu_read_status(ws)
    return st, s.cpu().numpy(), i.cpu().numpy()


def _ints(rng, shape):
    return rng.integers(-2, 3, size=shape).astype(np.float32)


@pytest.mark.parametrize("U,M,d,K", [(3, 20000, 64, 1), (3, 20000, 128, 7), (4, 20000, 1024, 100),
                                     (2, 20000, 64, 1024), (130, 8193, 64, 50), (5, 100, 64, 100),
                                     (1, 257, 192, 256)])
def test_integer_inputs_exact(U, M, d, K):
    rng = np.random.default_rng(U * 1000 + K)
    E, Hh = _ints(rng, (M, d)), _ints(rng, (U, d))
    st, s, i = _run(_bf16(Hh), _bf16(E), K)
    assert st == 0
    rv, ri = R.retrieve(E, Hh, K)
    np.testing.assert_array_equal(i, ri)
    np.testing.assert_array_equal(s.astype(np.float64), rv)


def test_user_vectors_from_encoder_rows():
    rng = np.random.default_rng(5)
    offsets = np.array([0, 7, 7, 30, 31, 60])          # user 1 has no rows
    Y = _ints(rng, (60, 128))
    E = _ints(rng, (5000, 128))
    st, s, i = _run(_bf16(Y), _bf16(E), 20, offsets=offsets)
    assert st == 0
    rv, ri = R.retrieve(E, R.user_vectors(Y, offsets), 20)
    np.testing.assert_array_equal(i, ri)
    np.testing.assert_array_equal(s.astype(np.float64), rv)
    assert i[1].tolist() == list(range(20)) and not s[1].any()   # empty user: first ids


def test_bad_offsets_set_status():
    rng = np.random.default_rng(6)
    Y, E = _ints(rng, (10, 64)), _ints(rng, (300, 64))
    st, _, _ = _run(_bf16(Y), _bf16(E), 5, offsets=np.array([0, 6, 4, 10]))
    assert st == 5
    st, _, _ = _run(_bf16(Y), _bf16(E), 5, offsets=np.array([0, 6, 11]))
    assert st == 5


def test_host_argument_errors():
    import torch
    import hstu_sequential_transducer_layer_b200 as H
    from hstu_sequential_transducer_layer_b200 import HstuError
    E = _bf16(np.zeros((100, 64)))
    Hd = _bf16(np.zeros((2, 64)))
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    s = torch.empty((2, 200), dtype=torch.float32, device="cuda")
    i = torch.empty((2, 200), dtype=torch.int64, device="cuda")
    for K in (0, 101, 2000):      # K outside 1..min(M, 1024)
        with pytest.raises(HstuError):
            H.hstu_retrieval_topk(Hd, E, K, s, i, ws)
    with pytest.raises(HstuError):                         # d not a multiple of 64
        H.hstu_retrieval_topk(_bf16(np.zeros((2, 96))), _bf16(np.zeros((100, 96))), 5, s, i, ws)


def _exact(E64, H64):
    """Float64 scores and the bound's sums |h||E| (item blocks of 64K rows)."""
    S = np.empty((H64.shape[0], E64.shape[0]))
    A = np.empty_like(S)
    for m0 in range(0, E64.shape[0], 1 << 16):
        Eb = np.asarray(E64[m0:m0 + (1 << 16)], np.float64)
        S[:, m0:m0 + len(Eb)] = R.scores(Eb, H64)
        A[:, m0:m0 + len(Eb)] = np.abs(H64) @ np.abs(Eb).T
    return S, A


def _validity(s, i, S, A, d, K):
    """The fp32 decisions against the float64 scores (module docstring)."""
    tol = d * 2.0 ** -23 * A
    rv, ri = R.topk(S, K)
    for u in range(S.shape[0]):
        assert len(set(i[u].tolist())) == K and (i[u] >= 0).all()
        ex = S[u, i[u]]
        assert np.all(np.abs(s[u] - ex) <= tol[u, i[u]]), u
        assert np.all(np.diff(s[u]) <= 0), u
        eq = np.diff(s[u]) == 0
        assert np.all(np.diff(i[u])[eq] > 0), u              # equal scores: ascending ids
        kth = rv[u, -1]
        t2 = 2 * tol[u].max()
        assert np.all(ex >= kth - t2), u
        must = np.nonzero(S[u] > kth + t2)[0]
        assert set(must.tolist()) <= set(i[u].tolist()), u
        # the exact top-K and the GPU's agree except within the tolerance band
        assert len(set(ri[u].tolist()) ^ set(i[u].tolist())) <= 2 * np.count_nonzero(
            np.abs(S[u] - kth) <= t2), u


def test_normal_inputs_valid():
    rng = np.random.default_rng(8)
    U, M, d, K = 16, 50000, 256, 100
    E = hw.round_to_bf16(rng.standard_normal((M, d)).astype(np.float32))
    Hh = hw.round_to_bf16(rng.standard_normal((U, d)).astype(np.float32))
    st, s, i = _run(_bf16(Hh), _bf16(E), K)
    assert st == 0
    S, A = _exact(E, Hh.astype(np.float64))
    _validity(s, i, S, A, d, K)


def test_full_catalog_at_full_size():
    """The bench's configuration: 128 users, the 1M x 1024 content table of
    the full-stack raw workload, K = 100; the oracle checks 8 sampled users
    against the whole catalog."""
    import torch
    M, d, K, U = 1_000_000, 1024, 100, 128
    Ed = hw.device_embedding_table(0, 0, M, d, "cuda")
    rng = np.random.default_rng(9)
    Hh = hw.round_to_bf16(rng.standard_normal((U, d)).astype(np.float32) / 32.0)
    st, s, i, ws = _run_ws(_bf16(Hh), Ed, K)
    assert st == 0 and not _fallback_taken(ws)   # the filtering path decided
    users = [0, 1, 37, 64, 90, 101, 126, 127]
    Eb = Ed.view(torch.int16).cpu().numpy().view(np.uint16)
    E32 = (Eb.astype(np.uint32) << np.uint32(16)).view(np.float32)   # exact bf16 values
    del Eb
    S, A = _exact(E32, Hh[users].astype(np.float64))
    _validity(s[users], i[users], S, A, d, K)


def _fallback_taken(ws):
    import hstu_sequential_transducer_layer_b200 as H
    return H.hstu_retrieval_fallback_taken(ws)


def _run_ws(Hd, Ed, K):
    import torch
    import hstu_sequential_transducer_layer_b200 as H
    U, (M, d) = Hd.shape[0], Ed.shape
    ws = torch.empty(H.hstu_retrieval_workspace_size(U, M, d, K), dtype=torch.uint8, device="cuda")
    s = torch.full((U, K), float("nan"), dtype=torch.float32, device="cuda")
    i = torch.full((U, K), -1, dtype=torch.int64, device="cuda")
    H.hstu_retrieval_topk(Hd, Ed, K, s, i, ws)
    return H.hstu_read_status(ws), s.cpu().numpy(), i.cpu().numpy(), ws


@pytest.mark.parametrize("U,M,K", [(7, 70000, 100), (3, 100003, 1024), (2, 65536, 1)])
def test_filter_path_integer_inputs_exact(U, M, K):
    """Catalogs of 65,536 items or more take the sample-threshold filtering
    path; integer scores tie often, so the tie order is exercised too."""
    rng = np.random.default_rng(M + K)
    E, Hh = _ints(rng, (M, 64)), _ints(rng, (U, 64))
    st, s, i, ws = _run_ws(_bf16(Hh), _bf16(E), K)
    assert st == 0 and not _fallback_taken(ws)
    rv, ri = R.retrieve(E, Hh, K)
    np.testing.assert_array_equal(i, ri)
    np.testing.assert_array_equal(s.astype(np.float64), rv)


def test_fallback_when_every_score_ties():
    # every item equal: all pass the threshold, the candidate lists overflow,
    # the direct path runs and returns the first K ids
    rng = np.random.default_rng(13)
    E = np.ones((70000, 64), np.float32)
    Hh = _ints(rng, (3, 64))
    st, s, i, ws = _run_ws(_bf16(Hh), _bf16(E), 50)
    assert st == 0 and _fallback_taken(ws)
    rv, ri = R.retrieve(E, Hh, 50)
    np.testing.assert_array_equal(i, ri)
    np.testing.assert_array_equal(s.astype(np.float64), rv)


def test_no_users():
    import torch
    import hstu_sequential_transducer_layer_b200 as H
    E = _bf16(np.ones((300, 64), np.float32))
    Hd = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.full((H.hstu_retrieval_workspace_size(0, 300, 64, 5),), 7, dtype=torch.uint8,
                    device="cuda")
    s = torch.empty((0, 5), dtype=torch.float32, device="cuda")
    i = torch.empty((0, 5), dtype=torch.int64, device="cuda")
    H.hstu_retrieval_topk(Hd, E, 5, s, i, ws)
    assert H.hstu_read_status(ws) == 0   # a stale word from an earlier call would not be 0
