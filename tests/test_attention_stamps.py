"""The attention kernel's diagnostic clock stamps: the product library has
none (and says so), and the analysis of a stamp table returns the phase
durations planted in it."""
import ctypes as C

import numpy as np
import pytest

from image_generation_b200 import attention_stamps as S
from image_generation_b200 import h3dit as H


def test_product_library_has_no_stamp_points():
    n = H.H3DIT_ATTN_STAMP_SLOTS * H.H3DIT_ATTN_STAMP_STEPS
    buf = (C.c_uint64 * n)()
    assert H.lib.h3dit_attention_stamps(buf, H.H3DIT_ATTN_STAMP_SLOTS,
                                        H.H3DIT_ATTN_STAMP_STEPS) == H.H3DIT_ERR_UNSUPPORTED
    assert H.lib.h3dit_attention_stamps(None, 32, 300) == H.H3DIT_ERR_INVALID_ARG


def test_header_constants_match_the_kernel_layout():
    src = open(H.os.path.join(H.PKG, "csrc", "attention.cu")).read()
    assert f"kStampSlots = {H.H3DIT_ATTN_STAMP_SLOTS}, kStampSteps = {H.H3DIT_ATTN_STAMP_STEPS}" in src


def _table(period=1600, phases=(200, 100, 150, 900, 50, 80), offset=400, spread=(0, 60, 120, 30),
           steps=264):
    """A stamp table of a kernel whose every step takes `period` clocks, each
    softmax warp going through `phases` (wait for S, load, max, exp, store,
    hand-back) and tile 1 running `offset` clocks after tile 0."""
    st = np.zeros((S_STEPS, 32), np.int64)
    for j in range(steps):
        for t in (0, 1):
            t0 = 10_000 + j * period + t * offset + phases[0]
            c = t0
            st[j, 6 * t] = c
            for i in range(1, 6):
                c += phases[i]
                st[j, 6 * t + i] = c
            for k in range(4):
                st[j, 20 + 4 * t + k] = c + spread[k]
            last = c + max(spread)
            st[j, 12 + 3 * t] = last + 70           # issuer sees P
            st[j, 13 + 3 * t] = last + 70 + 500     # PV issued
            st[j, 14 + 3 * t] = last + 70 + 500 + 150 + 600  # S(j+2) issued
        st[j, 18] = 5_000 + j * period
    for j in range(2, steps):                        # K_j seen just before S_j is issued
        for t in (0, 1):
            st[j, 28 + t] = st[j - 2, 14 + 3 * t] - 600
    return st[:steps]


S_STEPS = 300


def test_analysis_recovers_planted_phases():
    r = S.analyse(_table())
    sm = r["softmax_tile0"]
    assert sm["period"] == 1600
    assert sm["S_seen_to_scores_loaded"] == 100 and sm["row_max_to_exponentials"] == 900
    assert sm["hand_back_after_first_warp"] == [0, 60, 120, 30] and sm["hand_back_spread"] == 120
    iss = r["issuer_tile1"]
    assert iss["last_hand_back_to_P_seen"] == 70 and iss["issue_PV"] == 500
    assert iss["wait_K_two_steps_ahead"] == 150 and iss["issue_S_two_steps_ahead"] == 600
    assert r["tile1_S_seen_minus_tile0"]["median"] == 400
    assert r["tma_stage_period"] == 1600
