"""Pins of the oracle's dense and clustered LM heads."""
import numpy as np

from oracle import lm_head as H


def test_dense_basis_vectors_pick_weight_columns():
    """h = e_i gives logits[v] = W[v, i]: catches a transposed operand."""
    rng = np.random.default_rng(0)
    W = rng.standard_normal((37, 11))
    h = np.eye(11)[[3, 0, 10]]
    out = H.lm_head(h, W)
    np.testing.assert_array_equal(out, W[:, [3, 0, 10]].T)


def test_dense_one_hot_rows_pick_hidden_coordinates():
    rng = np.random.default_rng(1)
    h = rng.standard_normal((4, 6))
    W = np.eye(6)[[5, 5, 0, 2]]
    np.testing.assert_array_equal(H.lm_head(h, W), h[:, [5, 5, 0, 2]])


def test_dense_cols_subset_equals_slice():
    rng = np.random.default_rng(2)
    h, W = rng.standard_normal((3, 8)), rng.standard_normal((50, 8))
    cols = np.array([49, 0, 17])
    np.testing.assert_array_equal(H.lm_head(h, W, cols), H.lm_head(h, W)[:, cols])


def _clustered(seed, C=16, cs=8, d=12, M=5):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(C * cs).reshape(C, cs)
    w_cm = rng.standard_normal((C, cs, d))
    W = np.empty((C * cs, d))
    W[perm.ravel()] = w_cm.reshape(-1, d)
    cent = w_cm.mean(axis=1)
    h = rng.standard_normal((M, d))
    return h, W, w_cm, cent, perm


def test_clustered_keeping_all_clusters_equals_dense():
    h, W, w_cm, cent, perm = _clustered(3)
    logits, sel, gap = H.clustered_lm_head(h, cent, w_cm, perm, top_c=16)
    np.testing.assert_allclose(logits, H.lm_head(h, W), rtol=1e-13, atol=1e-13)
    assert np.all(np.isinf(gap))


def test_clustered_logits_equal_dense_inside_and_neg_inf_outside():
    h, W, w_cm, cent, perm = _clustered(4)
    logits, sel, _ = H.clustered_lm_head(h, cent, w_cm, perm, top_c=3)
    dense = H.lm_head(h, W)
    for m in range(h.shape[0]):
        keep = perm[sel[m]].ravel()
        np.testing.assert_allclose(logits[m, keep], dense[m, keep], rtol=1e-13, atol=1e-13)
        mask = np.ones(W.shape[0], bool)
        mask[keep] = False
        assert np.all(logits[m, mask] == -np.inf)
        assert np.isfinite(logits[m]).sum() == 3 * 8


def test_centroid_score_is_mean_of_member_logits_and_selection_is_top():
    h, W, w_cm, cent, perm = _clustered(5)
    scores = H.cluster_scores(h, cent)
    dense = H.lm_head(h, W)
    np.testing.assert_allclose(scores, dense[:, perm].mean(axis=2), rtol=1e-12, atol=1e-12)
    _, sel, gap = H.clustered_lm_head(h, cent, w_cm, perm, top_c=4)
    for m in range(h.shape[0]):
        kept = np.sort(scores[m, sel[m]])
        rest = np.delete(scores[m], sel[m])
        assert kept.min() >= rest.max()
        assert np.isclose(gap[m], kept.min() - rest.max())
        assert np.all(np.diff(sel[m]) > 0)  # ascending id order


def test_top_clusters_ties_prefer_lower_id():
    scores = np.array([[1.0, 2.0, 2.0, 2.0, 0.0]])
    sel, gap = H.top_clusters(scores, 2)
    assert sel.tolist() == [[1, 2]]
    assert gap[0] == 0.0
