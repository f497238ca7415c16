"""Pins of the oracle's token-grid and schedule arithmetic to the pages."""

import numpy as np
import pytest

from oracle import grid, schedule


def test_latent_shape_720p(gold):
    assert list(grid.latent_shape(81, 720, 1280)) == gold(
        "latent_shape_81f_720p")
    assert grid.latent_shape(81, 720, 1280)[1] == gold("latent_frames_81")[0]


def test_frame_count_must_be_4n_plus_1():
    # The page: 80 or 82 frames make the shapes not fit.
    for bad in (80, 82, 0):
        with pytest.raises(ValueError):
            grid.latent_shape(bad, 720, 1280)
    for ok in (1, 77, 81, 121):
        grid.latent_shape(ok, 720, 1280)


def test_tokens_720p(gold):
    g = grid.token_grid(81, 720, 1280)
    assert g == (21, 45, 80)
    assert g[1] * g[2] == gold("tokens_per_latent_frame_720p")[0]
    assert grid.token_count(g) == gold("tokens_81f_720p")[0]


def test_compression_numbers(gold):
    lat = int(np.prod(grid.latent_shape(81, 720, 1280)))
    pix = 81 * 720 * 1280 * 3
    assert abs(lat - gold("latent_values_81f_720p_approx")[0]) < 5e3
    assert abs(pix - gold("pixel_values_81f_720p_approx")[0]) < 5e5
    assert round(pix / lat) == gold("compression_ratio_approx")[0]


def test_long_video_token_counts(gold):
    # 480p (480 x 832): "~32.7k" at 81 frames and "~65.5k" at 165 frames.
    n81 = grid.token_count(grid.token_grid(81, 480, 832))
    n165 = grid.token_count(grid.token_grid(165, 480, 832))
    assert n81 == 32760 and n165 == 65520
    assert abs(n81 - gold("tokens_81f_480p_approx")[0]) < 100
    assert abs(n165 - gold("tokens_165f_480p_approx")[0]) < 100


def test_attention_flops(gold):
    f = grid.attention_flops(1, 40, 75600, 75600, 128)
    assert abs(f / gold("attention_flops_per_layer_approx")[0] - 1) < 0.005


def test_token_coords_roundtrip():
    g = (3, 5, 7)
    for n in range(grid.token_count(g)):
        f, h, w = grid.token_coords(n, g)
        assert (f * g[1] + h) * g[2] + w == n
        assert 0 <= f < 3 and 0 <= h < 5 and 0 <= w < 7


def test_printed_timesteps(gold):
    # The printed list is reproduced with s_max = 0.999 and truncation.
    want = [int(v) for v in gold("first_timesteps_shift12_40steps")]
    got = schedule.timesteps_int(40, 12.0, s_max=0.999)[:6]
    assert list(got) == want
    # With s_max = 1 only the first value differs (1000 instead of 999).
    got1 = schedule.timesteps_int(40, 12.0, s_max=1.0)[:6]
    assert list(got1[1:]) == want[1:] and got1[0] == 1000


@pytest.mark.parametrize("s_max", [1.0, 0.999])
def test_expert_split_and_median(gold, s_max):
    t = schedule.timesteps(40, 12.0, s_max)
    assert int((t >= 875).sum()) == gold("high_noise_steps_boundary_875")[0]
    assert int((t < 875).sum()) == gold("low_noise_steps_boundary_875")[0]
    # "half of the sampling points fall at t > 926"
    assert int((t > gold("median_timestep_shift12_above")[0]).sum()) == 20
    assert abs(np.median(t) - 926.4) < 0.2


def test_schedule_properties():
    s = schedule.sigmas(40, 12.0)
    assert s.shape == (41,)
    assert s[0] == 1.0 and s[-1] == 0.0
    assert np.all(np.diff(s) < 0)
    # shift = 1 leaves the uniform points unchanged.
    u = schedule.sigmas(40, 1.0)
    assert np.allclose(u[:-1], 1.0 - np.arange(40) / 40.0, atol=0, rtol=0)
    # the shift map fixes 0 and 1 and pushes interior points up
    assert schedule.shift_sigma(0.0, 5.0) == 0.0
    assert schedule.shift_sigma(1.0, 5.0) == 1.0
    assert schedule.shift_sigma(0.5, 5.0) > 0.5
    # shift 5, first step: s 1.0 -> 0.975 gives sigma 1.0 -> 4.875 / 4.9
    assert schedule.sigmas(40, 5.0)[1] == pytest.approx(4.875 / 4.9,
                                                        rel=1e-15)


def test_timestep_scale(gold):
    assert schedule.NUM_TRAIN_TIMESTEPS == gold("num_train_timesteps")[0]
    t = schedule.timesteps(10, 3.0)
    assert np.allclose(t / 1000.0, schedule.sigmas(10, 3.0)[:10],
                       rtol=1e-15)
