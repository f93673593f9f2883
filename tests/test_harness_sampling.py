"""The full-size parity checks sample tokens and locate their rows without the CUDA
path (tests/gpu_harness.py: sample_tokens, token_rows_in_image, token_a, check_tokens).
Here, on the CPU, those helpers are run against the oracle's whole forward pass on
small cases: every sampled row must equal the oracle's row for that token, every
M-block must hold a sample, and a row moved to the wrong placeholder must fail."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import projector as O

from gpu_harness import check_tokens, custom, make_case, oracle_params, sample_tokens

CASES = {
    "untiled_ln_odd": (custom("s_untiled", 200, 3, 64, 96, 64, 4, 2, 200, has_ln=True),
                       [[25, 31], [9, 9], [3, 2], [30, 27]], "head"),
    "tiled_head_odd": (custom("s_tiled", 201, 2, 64, 96, 64, 3, 3, 120, tiled=True, tw=2, th=2),
                       [[5, 5]] * 15, "head"),
    "tiled_tail": (custom("s_tail", 202, 2, 64, 96, 64, 2, 2, 400, tiled=True, tw=3, th=2),
                   [[6, 7]] * 14, "tail"),
}


def _oracle_out(case):
    emb = O.bf16_bits_to_f64(case.prefill)
    full = O.forward(case.feats, case.hw, case.crop, case.wl.k, oracle_params(case), case.ids, W.IMAGE_TOKEN_ID,
                     emb, case.wl.ln_eps, not case.wl.feat_fp32, True, case.gvp)
    return torch.from_numpy(full)


@pytest.mark.parametrize("name", list(CASES))
def test_sampled_rows_equal_the_whole_forward(name):
    wl, hw, gvp = CASES[name]
    case = make_case(wl, np.array(hw, np.int32), gvp=gvp)
    out = _oracle_out(case)
    picks = sample_tokens(case, per_image=4, block=16)
    stats = check_tokens(case, out, picks)
    assert stats["max_abs_err"] < 1e-12


@pytest.mark.parametrize("name", list(CASES))
def test_every_block_of_tokens_is_sampled(name):
    wl, hw, gvp = CASES[name]
    case = make_case(wl, np.array(hw, np.int32), gvp=gvp)
    n_tok = [O.tokens_untiled(int(h), int(w), wl.k) for h, w in case.hw]
    start = np.concatenate([[0], np.cumsum(n_tok)])
    picks = sample_tokens(case, per_image=4, block=16)
    m = sorted(int(start[v]) + t for v, t in picks)
    assert set(range(0, int(start[-1]), 16)) <= {x - x % 16 for x in m}
    per = wl.views_per_image
    for img in range(wl.n_images):
        tot = sum(n_tok[img * per:(img + 1) * per])
        assert sum(1 for v, _ in picks if v // per == img) >= min(4, tot)


@pytest.mark.parametrize("name", list(CASES))
def test_a_row_at_the_wrong_placeholder_fails(name):
    wl, hw, gvp = CASES[name]
    case = make_case(wl, np.array(hw, np.int32), gvp=gvp)
    out = _oracle_out(case)
    pos = O.placeholder_positions(case.ids, W.IMAGE_TOKEN_ID)
    bad = out.clone()
    bad[pos[1:]] = out[pos[:-1]]                      # every row one placeholder late
    picks = sample_tokens(case, per_image=4, block=16)
    with pytest.raises(AssertionError):
        check_tokens(case, bad, picks)
