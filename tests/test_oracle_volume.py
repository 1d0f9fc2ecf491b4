"""Pins of the volume comparison in the oracle (V-IoU of inside sets, sign
agreement) against hand-counted closed forms (no GPU)."""
import numpy as np

from oracle import volume as OV


def test_v_iou_of_two_overlapping_boxes_by_hand():
    # boxes [0,4)^3 and [2,6)^3 of an 8^3 grid: 64 voxels each, overlap [2,4)^3 = 8,
    # union 120, so V-IoU = 8 / 120; sign agreement: 8^3 - (64 + 64 - 2 * 8) = 400
    a = np.ones((8, 8, 8), np.float32)
    b = np.ones((8, 8, 8), np.float32)
    a[:4, :4, :4] = -1
    b[2:6, 2:6, 2:6] = -2
    c = OV.compare_volumes(a, b)
    assert (c["inside_a"], c["inside_b"], c["inside_both"]) == (64, 64, 8)
    assert c["v_iou"] == 8 / 120
    assert c["same_sign"] == 512 - 112
    assert c["max_abs_diff"] == 3.0     # -1 against +2 ... and +1 against -2


def test_zero_counts_as_outside_and_identical_volumes():
    a = np.array([0.0, -0.0, -1e-30, 1e-30], np.float32)
    c = OV.compare_volumes(a, a)
    assert c["inside_a"] == 1 and c["v_iou"] == 1.0 and c["same_sign"] == 4
    empty = OV.compare_volumes(np.ones(5), np.ones(5))
    assert empty["v_iou"] == 1.0 and empty["inside_both"] == 0
