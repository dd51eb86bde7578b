"""Pins for the oracle's greedy tree verify (CPU only): hand-built trees
whose expected path is read off the rule by eye -- a node is matched when
its token is the AR argmax of its parent's row and its parent is matched;
the deepest matched node (lowest index on ties) ends the path; the bonus is
the argmax of that node's own row (row 0 = root, row k+1 = node k)."""
import numpy as np

import oracle

V = 6


def rows(argmaxes):
    """One f32 row per entry, largest logit at the given index."""
    r = np.zeros((len(argmaxes), V), np.float32)
    for j, a in enumerate(argmaxes):
        r[j, a] = 2.0
    return r


def run(argmaxes, tokens, parents):
    ar = rows(argmaxes)[None]
    return oracle.verify_tree_greedy(ar, np.array([tokens]), np.array([parents]))


def check(res, path, toks, status=0):
    M = res["path_nodes"].shape[1]
    assert res["path_len"][0] == len(path)
    assert res["path_nodes"][0].tolist() == path + [-1] * (M - len(path))
    assert res["tokens"][0].tolist() == toks + [-1] * (M + 1 - len(toks))
    assert res["status"] == status


def test_chain_full_match():
    a = [1, 3, 0, 5]                       # argmax of root, node0, node1, node2 rows
    check(run(a, [1, 3, 0], [-1, 0, 1]), [0, 1, 2], [1, 3, 0, 5])


def test_chain_mismatch_in_middle():
    a = [1, 3, 0, 5]
    check(run(a, [1, 4, 0], [-1, 0, 1]), [0], [1, 3])


def test_star_duplicate_siblings_lowest_index():
    a = [2, 0, 1, 4, 5]
    check(run(a, [5, 1, 2, 2], [-1, -1, -1, -1]), [2], [2, 4])


def test_no_match_emits_root_argmax():
    a = [2, 0, 1, 4]
    check(run(a, [0, 1, 3], [-1, -1, 0]), [], [2])


def test_later_sibling_with_deeper_subtree_wins():
    # nodes 0 and 1 both carry the root argmax; only node 1 has a matching child
    a = [4, 1, 3, 2]
    check(run(a, [4, 4, 3], [-1, -1, 1]), [1, 2], [4, 3, 2])


def test_equal_depth_branches_lowest_index():
    # node0 -> node2, node1 -> node3, both depth 2 and matched
    a = [4, 1, 1, 0, 5]
    check(run(a, [4, 4, 1, 1], [-1, -1, 0, 1]), [0, 2], [4, 1, 0])


def test_unmatched_parent_blocks_child():
    a = [4, 1, 3]
    check(run(a, [2, 1], [-1, 0]), [], [4])


def test_bad_parent_flagged():
    a = [4, 1, 3]
    res = run(a, [4, 1], [-1, 1])          # parent must precede the child
    check(res, [0], [4, 1], status=oracle.BAD_PARENT)
    res = run(a, [4, 1], [-1, -2])
    check(res, [0], [4, 1], status=oracle.BAD_PARENT)


def test_bad_token_flagged():
    a = [4, 1, 3]
    check(run(a, [4, 99], [-1, 0]), [0], [4, 1], status=oracle.BAD_TOKEN_ID)


def test_ties_in_rows_pick_lowest_index():
    ar = np.zeros((1, 3, V), np.float32)
    ar[0, 0, [2, 4]] = 1.0                 # root argmax: 2 (tie with 4)
    ar[0, 1, :] = 0.5                      # node0 row: all equal -> 0
    res = oracle.verify_tree_greedy(ar, np.array([[2, 4]]), np.array([[-1, -1]]))
    check(res, [0], [2, 0])


def test_batch_rows_are_independent():
    a0, a1 = [1, 3, 0, 5], [2, 2, 2, 2]
    ar = np.stack([rows(a0), rows(a1)])
    res = oracle.verify_tree_greedy(ar, np.array([[1, 3, 0], [2, 2, 2]]),
                                    np.array([[-1, 0, 1], [-1, 0, 0]]))
    assert res["path_len"].tolist() == [3, 2]
    assert res["tokens"][1].tolist() == [2, 2, 2, -1]
