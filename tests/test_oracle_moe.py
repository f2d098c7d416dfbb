"""Pins for the oracle's MoE routing and combine (256 routed experts, 8 active per
token on the DeepSeek-V3 page; block-scale fused MoE on the ROCm/AITER page, 2.3).

What fixes the expected values:
- a hand-worked case with ties (T = 3, E = 4, k = 2);
- selection against numpy's stable sort of (-score, expert) on random scores; offsets
  against numpy's bincount / cumsum; the sorted rows against numpy's lexsort of
  (token, expert); token_row as the inverse permutation;
- weights: fp32 sum in selection order and one IEEE division, recomputed with numpy
  float32; the zero-sum case gives 1/k;
- combine: with unit weights on one expert it reduces to the block GEMM row; in
  general it is the weighted sum of per-expert GEMM rows, each pinned elsewhere.
"""
import numpy as np

import oracle as O


def test_hand_case_with_ties():
    s = np.array([[0.5, 0.9, 0.5, 0.1],      # picks 1, then 0 (tie 0/2 -> lower index)
                  [0.2, 0.2, 0.2, 0.2],      # picks 0, 1
                  [0.0, 0.0, 0.3, 0.0]],     # picks 2, then 0
                 np.float32)
    r = O.moe_route(s, 2)
    assert r["ids"].tolist() == [[1, 0], [0, 1], [2, 0]]
    assert r["w"][0].tolist() == [np.float32(0.9) / np.float32(np.float32(0.9) + np.float32(0.5)),
                                  np.float32(0.5) / np.float32(np.float32(0.9) + np.float32(0.5))]
    assert r["w"][1].tolist() == [0.5, 0.5]
    assert r["w"][2].tolist() == [1.0, 0.0]
    # expert 0 <- tokens 0, 1, 2; expert 1 <- tokens 0, 1; expert 2 <- token 2; expert 3 <- none
    assert r["offsets"].tolist() == [0, 3, 5, 6, 6]
    assert r["row_token"].tolist() == [0, 1, 2, 0, 1, 2]
    assert r["token_row"].tolist() == [3, 0, 1, 4, 5, 2]


def test_zero_scores_give_equal_weights():
    r = O.moe_route(np.zeros((2, 5), np.float32), 4)
    assert r["ids"].tolist() == [[0, 1, 2, 3]] * 2
    assert (r["w"] == np.float32(0.25)).all()


def test_random_routing_against_numpy():
    rng = np.random.default_rng(8)
    T, E, k = 300, 64, 8
    s = rng.random((T, E), dtype=np.float32)
    s[5, :] = 0.5                                             # a row of ties
    r = O.moe_route(s, k)
    order = np.lexsort((np.arange(E)[None, :].repeat(T, 0), -s), axis=1)   # by -score, then index
    assert np.array_equal(r["ids"], order[:, :k])
    sel = np.take_along_axis(s, r["ids"].astype(np.int64), 1)
    tot = np.zeros(T, np.float32)
    for j in range(k):
        tot = tot + sel[:, j]                                 # fp32, selection order
    assert np.array_equal(r["w"], sel / tot[:, None])
    cnt = np.bincount(r["ids"].ravel(), minlength=E)
    assert np.array_equal(r["offsets"], np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32))
    tok = np.repeat(np.arange(T), k)
    exp = r["ids"].ravel()
    srt = np.lexsort((tok, exp))
    assert np.array_equal(r["row_token"], tok[srt])
    assert np.array_equal(r["row_weight"], r["w"].ravel()[srt])
    inv = np.empty(T * k, np.int64)
    inv[srt] = np.arange(T * k)
    assert np.array_equal(r["token_row"], inv)


def test_combine_reduces_to_gemm_rows():
    rng = np.random.default_rng(9)
    T, E, N, K, k = 6, 3, 256, 256, 2
    qa = rng.integers(0x20, 0x50, (T, K)).astype(np.uint8)
    sa = np.exp2(rng.integers(-3, 3, (T, K // 128))).astype(np.float32)
    qw = rng.integers(0x20, 0x50, (E, N, K)).astype(np.uint8)
    sw = np.exp2(rng.integers(-3, 3, (E, N // 128, K // 128))).astype(np.float32)
    ids = np.array([[e % E, (e + 1) % E] for e in range(T)], np.int32)
    w1 = np.tile(np.array([[1.0, 0.0]], np.float32), (T, 1))
    out, _ = O.moe_combine_rows(qa, sa, qw, sw, ids, w1, np.arange(T))
    for t in range(T):
        y, _ = O.gemm_rows(qa, sa, qw[ids[t, 0]], sw[ids[t, 0]], rows=[t])
        assert np.array_equal(out[t], y[0])
    w = rng.random((T, k)).astype(np.float32)
    out, bound = O.moe_combine_rows(qa, sa, qw, sw, ids, w, np.arange(T))
    for t in range(T):
        ref = sum(np.float64(w[t, j]) * O.gemm_rows(qa, sa, qw[ids[t, j]], sw[ids[t, j]], rows=[t])[0][0]
                  for j in range(k))
        assert np.array_equal(out[t], ref)
    assert (bound >= np.abs(out)).all()
