"""The work counters behind the bench's roofline figures, against brute force."""
import numpy as np
import pytest

from workloads import WORKLOADS, band_pairs, dswa_pairs, algorithmic_work, backward_work


def _pairs_brute(L, P, w, dil):
    t = np.arange(L)
    f, s = t // P, t % P
    r = (f // dil) * P + s
    same = (f[:, None] % dil) == (f[None, :] % dil)
    d = r[:, None] - r[None, :]
    return int((same & (d >= 0) & (d < w)).sum())


@pytest.mark.parametrize("L,P,w,dil", [(50, 1, 7, 1), (64, 8, 20, 1), (300, 32, 48, 3), (257, 50, 120, 4),
                                       (120, 10, 1, 2), (100, 16, 500, 5)])
def test_pair_counts_match_the_masks(L, P, w, dil):
    assert dswa_pairs(L, P, w, dil) == _pairs_brute(L, P, w, dil)
    assert band_pairs(L, w) == _pairs_brute(L, 1, w, 1)


def test_backward_attention_work_is_ten_over_four_of_the_forward():
    wl = WORKLOADS["rollout_480p"]
    f, b = algorithmic_work(wl), backward_work(wl)
    assert b["swa_flops"] * 4 == f["swa_flops"] * 10 and b["dswa_flops"] * 4 == f["dswa_flops"] * 10
    assert b["flops"] == b["swa_flops"] + b["dswa_flops"] + b["gdn_flops"]
