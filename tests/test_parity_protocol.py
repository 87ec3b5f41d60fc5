"""The host side of the parity protocol (the decision the GPU parity tests take): the logit error
relative to the logit scale, token admissibility at near-ties and the TOP-n commit rule.  These
run on CPU with hand-made logits whose answers are known."""
import numpy as np

import oracle
from smdm_testlib import logit_err, token_admissible, topn_commit_admissible


def test_logit_error_is_relative_to_scale_at_least_one():
    o = np.array([[0.5, -0.25]])
    assert abs(logit_err(o + 0.01, o) - 0.01) < 1e-15     # scale clamps to 1
    o2 = np.array([[10.0, -40.0]])
    assert abs(logit_err(o2 + 0.4, o2) - 0.01) < 1e-15   # scale = 40


def test_token_admissibility_near_ties():
    ref = np.array([[1.0, 0.995, 0.2],     # near tie between 0 and 1 (gap 0.005 < 2e-2)
                    [3.0, 2.0, 1.0],       # clear argmax 0 (scale 3: band 0.06)
                    [0.0, 0.0, 0.0]])      # exact three-way tie
    assert token_admissible(np.array([1, 0, 2]), ref, 2e-2).all()
    assert not token_admissible(np.array([2, 1, 0]), ref, 2e-2)[:2].any()
    assert token_admissible(np.array([0, 0, 1]), ref, 2e-2).all()


def test_topn_commit_rule():
    ref = np.array([[4.0, 0.0, 0.0],       # conf high
                    [1.0, 0.0, 0.0],       # conf mid
                    [1.001, 0.0, 0.0],     # near-tie with row 1 (slightly higher)
                    [0.0, 0.0, 0.0]])      # conf 1/3, lowest
    tol = 2e-2
    _, _, rows = oracle.unmask(ref, oracle.POLICY_TOPN, 2)
    assert list(rows) == [0, 2]
    assert topn_commit_admissible(ref, rows, 2, tol)
    assert topn_commit_admissible(ref, [0, 1], 2, tol)        # near-tie swap is admissible
    assert not topn_commit_admissible(ref, [0, 3], 2, tol)    # a clearly lower row is not
    assert not topn_commit_admissible(ref, [0], 2, tol)       # wrong count
    assert topn_commit_admissible(ref, [0, 1, 2, 3], 8, tol)  # n larger than the rows: all
