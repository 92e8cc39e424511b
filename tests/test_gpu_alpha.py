"""GPU alpha search against the oracle's quantize -> decode -> SNR at every candidate alpha.

The GPU decodes in fp32 (LUT * max) where the oracle decodes in fp64, so the SNRs agree to
1e-3 dB; the best alpha is unique only up to candidates within that margin, so the check is
that the GPU's choice is within 1e-3 dB of the oracle's best.
"""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_b200 as opq
import oracle
import workloads
from test_gpu_parity import DEV, no_device_error

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gs", [0, 128, 32])
@pytest.mark.parametrize("dist", ["student_t4", "normal"])
def test_alpha_search_matches_oracle(gs, dist):
    lin = workloads.Linear("alpha-search", 1, 257, 1024, w_seed=17 + gs, w_dist=dist)
    w = lin.make_weights("cpu")
    alphas = list(opq.ALPHA_GRID)
    best_g, snr_g = opq.alpha_search(w.to(DEV), alphas, gs)
    no_device_error()
    best_o, snr_o = oracle.alpha_search(w, alphas, gs)
    assert np.allclose(snr_g, snr_o, atol=1e-3, rtol=0), (snr_g, snr_o)
    assert snr_o[alphas.index(best_g)] >= max(snr_o) - 1e-3


def test_alpha_search_full_size():
    # the attention projection: the search runs on the GPU in one call per candidate
    w = workloads.dit_attn_proj().make_weights(DEV)
    best, snr = opq.alpha_search(w, (0.45, 0.6, 0.73, 0.9, 1.0))
    assert best in (0.45, 0.6, 0.73, 0.9, 1.0) and len(snr) == 5
    sample = w[:256].contiguous().cpu()
    _, snr_o = oracle.alpha_search(sample, [0.73], 0)
    _, snr_s = opq.alpha_search(sample.to(DEV), [0.73], 0)
    assert abs(snr_s[0] - snr_o[0]) < 1e-3
    no_device_error()


def test_alpha_search_errors():
    w = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(opq.OPQError):
        opq.alpha_search(w, [0.73, -1.0])
    with pytest.raises(opq.OPQError):
        opq.alpha_search(w, [0.73], 48)
    best, snr = opq.alpha_search(w, [0.5, 0.73])   # all-zero weights: zero error -> +inf, first alpha
    assert best == 0.5 and snr[0] == float("inf")
